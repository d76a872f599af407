// Arguments shared by the attention kernels.
#pragma once
#include <stdint.h>

#include "common.cuh"

namespace csa2 {

struct AttnArgs {
    const uint16_t *q;          // bf16 [rows][H][512]
    int rows, T, H, K;
    const uint8_t *kv;          // main entries, kv_row_stride bytes apart
    int64_t kv_row_stride;
    const int64_t *seq_start;
    const int32_t *n_entries;   // [B] entries per sequence: ids at or above are refused (NULL: unchecked)
    const int64_t *shard_lo;    // context shards: [B] first global entry of this shard (NULL: none)
    const int32_t *shard_n;     //   [B] entries in the shard; selected ids outside it are skipped
    const int32_t *idx;         // [rows][K]
    const int32_t *cnt;         // [rows] or NULL
    const uint8_t *swa_codes;   // [B][swa_cap][512]
    const float *swa_scale;     // [B][swa_cap]
    int swa_cap;
    const int32_t *swa_start;   // [rows] or NULL
    const int32_t *swa_len;     // [rows]
    float softmax_scale;
    void *out;
    int out_dtype;
    float *lse;
    float *partials;            // workspace
    int splits;
    int hgroups;                // head groups of 64 (tensor-core kernel)
    int keys_per_split;         // keys handled by one split (tensor-core kernel)
};

// Floats of one tensor-core split partial: running max[64], row sum[64], O[64][512].
constexpr int kPartialFloats = 2 * 64 + 64 * 512;

// Split plan of a launch: head groups of 64, key splits per (row, head group), keys per split.
// With max_ws set, only plans whose split partials fit in max_ws bytes are considered (one
// split, which needs no partials, always fits).
void attn_plan(int rows, int H, int K, int &hgroups, int &splits, int &keys_per_split,
               size_t max_ws = SIZE_MAX);
// Workspace bytes of a plan (the split partials; 256 when there is one split).
size_t attn_plan_workspace(int rows, int hgroups, int splits);
// Workspace bytes of the default plan.
size_t attn_workspace_bytes(int rows, int H, int K);

// Launch with the default plan; the split merge (when splits > 1) follows on `st`.
cudaError_t launch_attn(AttnArgs a, cudaStream_t st);
// Launch with the plan already in `a` (hgroups, splits, keys_per_split).
cudaError_t launch_attn_planned(const AttnArgs &a, cudaStream_t st);
// As launch_attn, but the split merge runs on `side` once the attention kernel has finished
// (`attn_done` is recorded on `st` and waited on `side`); *merged says whether a merge was
// queued on `side`.
cudaError_t launch_attn_side_merge(AttnArgs a, cudaStream_t st, cudaStream_t side, cudaEvent_t attn_done,
                                   bool *merged);

}  // namespace csa2

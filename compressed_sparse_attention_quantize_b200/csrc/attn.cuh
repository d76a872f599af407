// Arguments shared by the attention kernels.
#pragma once
#include "common.cuh"

namespace csa2 {

struct AttnArgs {
    const uint16_t *q;          // bf16 [rows][H][512]
    int rows, T, H, K;
    const uint8_t *kv;          // main entries, kv_row_stride bytes apart
    int64_t kv_row_stride;
    const int64_t *seq_start;
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

cudaError_t launch_attn_tc(AttnArgs a, cudaStream_t st);
cudaError_t launch_attn_tc_side_merge(AttnArgs a, cudaStream_t st, cudaStream_t side, cudaEvent_t attn_done,
                                      bool *merged);
size_t tc_workspace_bytes(int rows, int H, int K);
void tc_plan(int rows, int H, int K, int &hgroups, int &splits, int &keys_per_split);

// Dispatch used by the C ABI.
size_t attn_workspace_bytes(int rows, int H, int K);
void attn_plan(int rows, int H, int K, int &hgroups, int &splits, int &keys_per_split);
cudaError_t launch_attn(AttnArgs a, cudaStream_t st);

}  // namespace csa2

// Launch description of csa2_index_topk shared by the C ABI and the index kernels.
#pragma once
#include "common.cuh"

namespace csa2 {

struct IndexLaunch {
    int mode;
    const uint8_t *q_codes;
    const uint8_t *q_scales;
    const float *w;
    int B, T, H;
    const uint8_t *k_codes;
    int64_t k_code_stride;
    const uint8_t *k_scales;
    int64_t k_scale_stride;
    const int64_t *seq_start;
    const int32_t *n_entries;
    int64_t max_n;
    const int32_t *q_pos;
    const int32_t *pool;
    const int32_t *pool_len;
    int P_in;
    int K;
    int32_t *out_idx;
    int32_t *out_cnt;
    int P;
    int32_t *out_pool;
    int32_t *out_pool_len;
    void *workspace;
    size_t ws_bytes;
    float *out_scores;          // FULL: scores of the selected entries [rows][K] (NULL: none)
};

// Scratch bytes for `rows` query rows with up to `n` candidates each.
size_t index_topk_workspace_bytes(int rows, int64_t n, int K, int P);
cudaError_t launch_index_topk(const IndexLaunch &L, cudaStream_t st);

// Device-side error word (bounded waits that expire write a csa2_status here).
csa2_status read_and_clear_device_error();

}  // namespace csa2

// Launch description of csa2_index_topk shared by the C ABI and the index kernels.
#pragma once
#include "common.cuh"

namespace csa2 {

// One head's dot product from its four block partials, added in block order: u[q] is the raw
// E2M1 product sum of block q (a multiple of 1/4 below 2^10: at most 12 significant bits) and
// c[q] = s_q * s_k the product of two E4M3 scales (at most 8 bits, exact), so every partial
// u[q] * c[q] is exact in fp32 and a fused multiply-add rounds only the sum: the result equals
// rounding each product (exactly) and then each sum.
CSA2_D float head_block_sum(const uint32_t *u, const float (&c)[4]) {
    float d = __fmul_rn(__uint_as_float(u[0]), c[0]);
    d = __fmaf_rn(__uint_as_float(u[1]), c[1], d);
    d = __fmaf_rn(__uint_as_float(u[2]), c[2], d);
    return __fmaf_rn(__uint_as_float(u[3]), c[3], d);
}

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

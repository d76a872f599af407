// Pieces of context-parallel decode: one long sequence whose compressed entries are split into
// consecutive shards, one per GPU.  Each GPU selects and attends within its shard; the exchange
// steps are an all-gather of every shard's scored top-K and of every shard's attention partial.
//
// [A] page "DeepSeek V4.1 Flash深度解析：KV缓存压缩437倍的技术路径", section "压缩吸收注意力（二代）":
// the indexer keeps the top 2048 blocks of the whole context (ranked by score, entry index on
// ties).  The global top-K lies inside the union of the shards' top-K lists, so merging those
// lists by the same order reproduces the single-GPU selection exactly.
// [B] page "DeepSeek V4.1 Flash 如何靠压缩 KV 缓存实现小模型干翻大模型", section
// "CSA2：三层压缩一次吃满": one joint softmax over the selected entries; shards' partial
// outputs merge through their log-sum-exp like any split of the key set.
#include "common.cuh"

namespace csa2 {
namespace cpx {

// Scores of the selected entries, read back from the Full-mode score buffer of a row chunk.
__global__ void gather_scores_kernel(const float *__restrict__ scores, int64_t score_stride,
                                     const int32_t *__restrict__ idx, int K, int row0, int nrows,
                                     float *__restrict__ out_scores) {
    const int lr = blockIdx.y;
    const int r = row0 + lr;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < K; i += gridDim.x * blockDim.x) {
        const int32_t e = idx[(int64_t)r * K + i];
        out_scores[(int64_t)r * K + i] = e >= 0 ? scores[(int64_t)lr * score_stride + e] : -INFINITY;
    }
}

// Shard lists -> one contiguous candidate list per row (shard order, so ids stay ascending).
__global__ void compact_shards_kernel(const float *__restrict__ scores, const int32_t *__restrict__ ids,
                                      const int64_t *__restrict__ id_offset,
                                      const int32_t *__restrict__ cnt, int G, int rows, int K_in,
                                      float *__restrict__ c_scores, int32_t *__restrict__ c_ids,
                                      int32_t *__restrict__ c_n) {
    const int r = blockIdx.x;
    const int64_t stride = (int64_t)G * K_in;
    int off = 0;
    for (int g = 0; g < G; ++g) {
        int n = cnt[(int64_t)g * rows + r];
        n = n < 0 ? 0 : (n > K_in ? K_in : n);
        const int64_t src = ((int64_t)g * rows + r) * K_in;
        const int64_t base = id_offset ? id_offset[(int64_t)g * rows + r] : 0;
        for (int i = threadIdx.x; i < n; i += blockDim.x) {
            c_scores[r * stride + off + i] = scores[src + i];
            c_ids[r * stride + off + i] = (int32_t)(ids[src + i] + base);
        }
        off += n;
    }
    if (threadIdx.x == 0) c_n[r] = off;
}

// Log-sum-exp merge of the shards' normalised outputs: out = sum_g exp(lse_g - M) out_g / L,
// lse = M + ln L, with M = max_g lse_g and L = sum_g exp(lse_g - M), shards in order.
// One CTA of 128 threads per (row, head), 4 channels per thread.
__global__ void __launch_bounds__(128) attn_merge_shards_kernel(const float *__restrict__ outs,
                                                                const float *__restrict__ lses, int G,
                                                                int rows, int H, int D, void *out,
                                                                int out_dtype, float *lse) {
    const int r = blockIdx.x, h = blockIdx.y;
    float M = -INFINITY;
    for (int g = 0; g < G; ++g) M = fmaxf(M, lses[((int64_t)g * rows + r) * H + h]);
    float L = 0.0f;
    for (int g = 0; g < G; ++g) {
        const float l = lses[((int64_t)g * rows + r) * H + h];
        if (l > -INFINITY) L += expf(l - M);
    }
    const float inv = L > 0.0f ? 1.0f / L : 0.0f;
    for (int c = threadIdx.x * 4; c < D; c += blockDim.x * 4) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int g = 0; g < G; ++g) {
            const float l = lses[((int64_t)g * rows + r) * H + h];
            if (!(l > -INFINITY)) continue;
            const float f = expf(l - M);
            const float4 v = *reinterpret_cast<const float4 *>(outs + (((int64_t)g * rows + r) * H + h) * D + c);
            acc[0] += f * v.x; acc[1] += f * v.y; acc[2] += f * v.z; acc[3] += f * v.w;
        }
        const int64_t oi = ((int64_t)r * H + h) * D + c;
        if (out_dtype == CSA2_DTYPE_F32) {
            *reinterpret_cast<float4 *>(reinterpret_cast<float *>(out) + oi) =
                make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
        } else {
            __nv_bfloat162 *o2 = reinterpret_cast<__nv_bfloat162 *>(reinterpret_cast<__nv_bfloat16 *>(out) + oi);
            o2[0] = __floats2bfloat162_rn(acc[0] * inv, acc[1] * inv);
            o2[1] = __floats2bfloat162_rn(acc[2] * inv, acc[3] * inv);
        }
    }
    if (threadIdx.x == 0 && lse) lse[(int64_t)r * H + h] = L > 0.0f ? M + logf(L) : -INFINITY;
}

}  // namespace cpx

cudaError_t launch_gather_scores(const float *scores, int64_t score_stride, const int32_t *idx, int K,
                                 int row0, int nrows, float *out_scores, cudaStream_t st) {
    dim3 grid((unsigned)((K + 255) / 256), (unsigned)nrows);
    cpx::gather_scores_kernel<<<grid, 256, 0, st>>>(scores, score_stride, idx, K, row0, nrows, out_scores);
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_topk_cluster(const float *scores, int64_t score_stride, const int32_t *cand,
                                int cand_stride, const int32_t *n_entries, const int32_t *q_pos,
                                const int32_t *pool_len, int T, int row0, int nrows, int K,
                                int32_t *out_idx, int32_t *out_cnt, int P, int32_t *out_pool,
                                int32_t *out_pool_len, int64_t max_n, cudaStream_t st);

int topk_row_chunks(int64_t max_n, int K, int P);
size_t topk_row_scratch_bytes(int rows, int64_t max_n, int K, int P);
cudaError_t launch_topk_row(const float *scores, int64_t score_stride, const int32_t *cand, int64_t cand_stride,
                            const int32_t *n_entries, const int32_t *q_pos, const int32_t *pool_len, int T,
                            int row0, int nrows, int K, int32_t *out_idx, int32_t *out_cnt, int P,
                            int32_t *out_pool, int32_t *out_pool_len, int64_t max_n, void *scratch,
                            cudaStream_t st);

// The largest selection scratch any K <= CSA2_MAX_TOPK needs for lists of up to n candidates.
static size_t merge_select_scratch(int rows, int64_t n) {
    size_t best = 0;
    for (int K = 1; K <= CSA2_MAX_TOPK; K *= 2) {
        const size_t b = topk_row_scratch_bytes(rows, n, K, 0);
        if (b > best) best = b;
    }
    const size_t b = topk_row_scratch_bytes(rows, n, CSA2_MAX_TOPK, 0);
    return b > best ? b : best;
}

static size_t merge_list_bytes(int G, int rows, int K_in) {
    const size_t cands = (size_t)rows * G * K_in;
    return (cands * 8 + (size_t)rows * 4 + 255) / 256 * 256;
}

size_t topk_merge_workspace_bytes(int G, int rows, int K_in) {
    return merge_list_bytes(G, rows, K_in) + merge_select_scratch(rows, (int64_t)G * K_in) + 256;
}

cudaError_t launch_topk_merge_shards(const float *scores, const int32_t *ids, const int64_t *id_offset,
                                     const int32_t *cnt, int G, int rows, int K_in, int K, int32_t *out_idx,
                                     int32_t *out_cnt, void *workspace, cudaStream_t st) {
    const int64_t stride = (int64_t)G * K_in;
    void *sel_scratch = reinterpret_cast<uint8_t *>(workspace) + merge_list_bytes(G, rows, K_in);
    const bool row_path = topk_row_chunks(stride, K, 0) > 0;
    if (G == 1 && id_offset == nullptr) {       // one list already in place: select from it directly
        if (row_path)
            return launch_topk_row(scores, K_in, ids, K_in, nullptr, nullptr, cnt, 1, 0, rows, K, out_idx, out_cnt, 0,
                                   nullptr, nullptr, K_in, sel_scratch, st);
        return launch_topk_cluster(scores, K_in, ids, K_in, nullptr, nullptr, cnt, 1, 0, rows, K, out_idx, out_cnt, 0,
                                   nullptr, nullptr, K_in, st);
    }
    float *c_scores = reinterpret_cast<float *>(workspace);
    int32_t *c_ids = reinterpret_cast<int32_t *>(c_scores + (size_t)rows * stride);
    int32_t *c_n = c_ids + (size_t)rows * stride;
    cpx::compact_shards_kernel<<<rows, 256, 0, st>>>(scores, ids, id_offset, cnt, G, rows, K_in, c_scores, c_ids,
                                                     c_n);
    note_launches(1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (row_path)
        return launch_topk_row(c_scores, stride, c_ids, stride, nullptr, nullptr, c_n, 1, 0, rows, K, out_idx, out_cnt,
                               0, nullptr, nullptr, stride, sel_scratch, st);
    return launch_topk_cluster(c_scores, stride, c_ids, (int)stride, nullptr, nullptr, c_n, 1, 0, rows, K,
                               out_idx, out_cnt, 0, nullptr, nullptr, stride, st);
}

cudaError_t launch_attn_merge_shards(const float *outs, const float *lses, int G, int rows, int H, int D,
                                     void *out, int out_dtype, float *lse, cudaStream_t st) {
    cpx::attn_merge_shards_kernel<<<dim3((unsigned)rows, (unsigned)H), 128, 0, st>>>(outs, lses, G, rows, H, D,
                                                                                    out, out_dtype, lse);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace csa2

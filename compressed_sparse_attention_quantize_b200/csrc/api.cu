// C ABI of the CSA2 library: argument validation, workspace sizing, launch sequencing.
//
// Every call validates all arguments before it enqueues anything, launches only on the
// caller's stream and never synchronises the host (csa2_device_error excepted).
#include <cstdio>

#include "common.cuh"
#include "attn.cuh"

namespace csa2 {
size_t topk_merge_workspace_bytes(int G, int rows, int K_in);
int64_t topk_cluster_max_n();
cudaError_t launch_topk_merge_shards(const float *, const int32_t *, const int64_t *, const int32_t *, int, int,
                                     int, int, int32_t *, int32_t *, void *, cudaStream_t);
cudaError_t launch_attn_merge_shards(const float *, const float *, int, int, int, int, void *, int, float *,
                                     cudaStream_t);

cudaError_t launch_selftest_bounded_wait(int, cudaStream_t);
cudaError_t launch_compress_fp4(const void *, int, int64_t, int, int, int64_t, const float *, int64_t,
                                uint8_t *, int64_t, uint8_t *, int64_t, const int64_t *, cudaStream_t);
cudaError_t launch_quant_fp4(const void *, int, int64_t, int, int64_t, uint8_t *, int64_t,
                             uint8_t *, int64_t, const int64_t *, cudaStream_t);
cudaError_t launch_quant_fp8_token(const void *, int, int64_t, int, int64_t, uint8_t *, int64_t,
                                   uint8_t *, int64_t, const int64_t *, cudaStream_t);
cudaError_t launch_quant_batch(const csa2_quant_job *, int, cudaStream_t);
cudaError_t launch_pool_extend(const int32_t *, const int32_t *, int, const int32_t *, const int32_t *,
                               const int32_t *, int, int, int, int32_t *, int32_t *, cudaStream_t);
}  // namespace csa2

#include "index_api.cuh"

#include <atomic>

#include <nvtx3/nvToolsExt.h>

namespace csa2 {
static std::atomic<uint64_t> g_launches{0};
void note_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }
}  // namespace csa2

using namespace csa2;

namespace {

inline bool aligned16(const void *p) { return (((uintptr_t)p) & 15u) == 0; }
inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }
thread_local char t_last_error[256] = "";
inline csa2_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return CSA2_OK;
    snprintf(t_last_error, sizeof(t_last_error), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
    return CSA2_ERR_CUDA;
}
// Host-timeline ranges for profilers: every public call, and each layer inside a group.  NVTX3
// is header-only; without an attached tool the push and pop are no-ops.
struct Range {
    explicit Range(const char *name) { nvtxRangePushA(name); }
    ~Range() { nvtxRangePop(); }
    Range(const Range &) = delete;
    Range &operator=(const Range &) = delete;
};
inline const char *layer_range_name(int mode) {
    return mode == CSA2_MODE_FULL ? "csa2 layer: Full" : mode == CSA2_MODE_REINDEX ? "csa2 layer: Reindex"
                                                                                   : "csa2 layer: Reuse";
}
constexpr size_t kAlign = 256;
inline size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

csa2_status check_index_args(int mode, const uint8_t *q_codes, const uint8_t *q_scales,
                             const float *w, int B, int T, int H_I, const uint8_t *k_codes,
                             int64_t k_code_stride, const uint8_t *k_scales, int64_t k_scale_stride,
                             const int64_t *seq_start, const int32_t *n_entries, int64_t max_n,
                             const int32_t *pool, const int32_t *pool_len, int P_in, int K,
                             int32_t *out_idx, int P, int32_t *out_pool) {
    if (mode != CSA2_MODE_FULL && mode != CSA2_MODE_REINDEX) return CSA2_ERR_INVALID_ARG;
    if (!q_codes || !q_scales || !w || !k_codes || !k_scales || !seq_start || !n_entries ||
        !out_idx)
        return CSA2_ERR_INVALID_ARG;
    if (B <= 0 || T <= 0 || (int64_t)B * T > (1 << 30)) return CSA2_ERR_SHAPE;
    if (H_I < 1 || H_I > CSA2_MAX_INDEX_HEADS) return CSA2_ERR_SHAPE;
    if (K < 1 || K > CSA2_MAX_TOPK) return CSA2_ERR_SHAPE;
    if (max_n < 0 || max_n > INT32_MAX) return CSA2_ERR_SHAPE;
    if (k_code_stride < 32 || k_scale_stride < 4) return CSA2_ERR_SHAPE;
    if (!aligned16(k_codes) || (k_code_stride & 15)) return CSA2_ERR_ALIGN;
    if (mode == CSA2_MODE_FULL) {
        if (P < 0 || P > CSA2_MAX_POOL) return CSA2_ERR_SHAPE;
        if (P > 0 && !out_pool) return CSA2_ERR_INVALID_ARG;
    } else {
        if (!pool || !pool_len) return CSA2_ERR_INVALID_ARG;
        if (P != 0) return CSA2_ERR_INVALID_ARG;
        if (P_in < 1 || P_in > CSA2_MAX_POOL) return CSA2_ERR_SHAPE;
    }
    return CSA2_OK;
}

csa2_status check_attn_args(const uint16_t *q, int B, int T, int H, int D, const uint8_t *kv,
                            int64_t kv_row_stride, const int64_t *seq_start, const int32_t *idx,
                            int K, const uint8_t *swa_codes, const float *swa_scale, int swa_cap,
                            const int32_t *swa_len, void *out, int out_dtype) {
    if (!q || !kv || !seq_start || !idx || !swa_len || !out) return CSA2_ERR_INVALID_ARG;
    if (out_dtype != CSA2_DTYPE_F32 && out_dtype != CSA2_DTYPE_BF16) return CSA2_ERR_INVALID_ARG;
    if (D != CSA2_LATENT_DIM) return CSA2_ERR_UNSUPPORTED;
    if (B <= 0 || T <= 0 || (int64_t)B * T > (1 << 30)) return CSA2_ERR_SHAPE;
    if (H < 16 || H > CSA2_MAX_HEADS || (H % 16)) return CSA2_ERR_SHAPE;
    if (K < 1 || K > CSA2_MAX_TOPK) return CSA2_ERR_SHAPE;
    if (swa_cap < 0) return CSA2_ERR_SHAPE;
    if (swa_cap > 0 && (!swa_codes || !swa_scale)) return CSA2_ERR_INVALID_ARG;
    if (kv_row_stride < kKvRowBytes) return CSA2_ERR_SHAPE;
    if (!aligned16(kv) || (kv_row_stride & 15)) return CSA2_ERR_ALIGN;
    if (swa_codes && !aligned16(swa_codes)) return CSA2_ERR_ALIGN;
    if (!aligned16(q) || !aligned16(out)) return CSA2_ERR_ALIGN;
    return CSA2_OK;
}

size_t attn_ws(int rows, int H, int K) { return round_up(attn_workspace_bytes(rows, H, K)); }

size_t index_ws(int mode, int rows, int64_t max_n, int K, int P) {
    const int64_t n = mode == CSA2_MODE_REINDEX ? (int64_t)P : max_n;
    return round_up(index_topk_workspace_bytes(rows, n, K, mode == CSA2_MODE_REINDEX ? 0 : P));
}

}  // namespace

extern "C" {

const char *csa2_status_string(csa2_status s) {
    switch (s) {
        case CSA2_OK: return "CSA2_OK";
        case CSA2_ERR_INVALID_ARG: return "CSA2_ERR_INVALID_ARG: a required pointer is NULL or an enum is unknown";
        case CSA2_ERR_SHAPE: return "CSA2_ERR_SHAPE: a size is out of range";
        case CSA2_ERR_ALIGN: return "CSA2_ERR_ALIGN: a pointer or stride is not 16-byte aligned";
        case CSA2_ERR_UNSUPPORTED: return "CSA2_ERR_UNSUPPORTED: valid but not implemented";
        case CSA2_ERR_CUDA: return "CSA2_ERR_CUDA: the CUDA runtime refused a launch";
        case CSA2_ERR_TIMEOUT: return "CSA2_ERR_TIMEOUT: a bounded device wait expired";
        case CSA2_ERR_WORKSPACE: return "CSA2_ERR_WORKSPACE: workspace missing or too small";
        case CSA2_ERR_HOST: return "CSA2_ERR_HOST: the operating system refused host memory";
    }
    return "CSA2: unknown status";
}

int csa2_version(void) { return 6; }

const char *csa2_last_error_string(void) { return t_last_error; }

uint64_t csa2_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

static csa2_status check_quant_args(int fmt, const void *x, int x_dtype, int64_t rows, int dim,
                                    int64_t x_stride, const uint8_t *codes, int64_t code_stride,
                                    const void *scales, int64_t scale_stride) {
    if (fmt != CSA2_FMT_FP4_E2M1_E4M3S16 && fmt != CSA2_FMT_FP8_E4M3_TOKEN) return CSA2_ERR_INVALID_ARG;
    if (x_dtype != CSA2_DTYPE_F32 && x_dtype != CSA2_DTYPE_BF16) return CSA2_ERR_INVALID_ARG;
    if (rows == 0) return CSA2_OK;                               // no-op, whatever the strides
    if (rows < 0 || dim <= 0 || (dim % 16) || dim > 65536 || x_stride < dim) return CSA2_ERR_SHAPE;
    if (!x || !codes || !scales) return CSA2_ERR_INVALID_ARG;
    if (fmt == CSA2_FMT_FP4_E2M1_E4M3S16) {
        if (code_stride < dim / 2 || scale_stride < dim / 16) return CSA2_ERR_SHAPE;
        return CSA2_OK;
    }
    if (code_stride < dim || scale_stride < 4) return CSA2_ERR_SHAPE;
    if ((((uintptr_t)scales) & 3u) || (scale_stride & 3)) return CSA2_ERR_ALIGN;
    return CSA2_OK;
}

csa2_status csa2_quantize_kv(int fmt, const void *x, int x_dtype, int64_t rows, int dim,
                             int64_t x_stride, uint8_t *codes, int64_t code_stride, void *scales,
                             int64_t scale_stride, const int64_t *dst_rows, void *stream) {
    const Range range("csa2_quantize_kv");
    const csa2_status s = check_quant_args(fmt, x, x_dtype, rows, dim, x_stride, codes, code_stride, scales,
                                           scale_stride);
    if (s != CSA2_OK || rows == 0) return s;
    if (fmt == CSA2_FMT_FP4_E2M1_E4M3S16)
        return cuda_status(launch_quant_fp4(x, x_dtype, rows, dim, x_stride, codes, code_stride,
                                            (uint8_t *)scales, scale_stride, dst_rows,
                                            as_stream(stream)));
    return cuda_status(launch_quant_fp8_token(x, x_dtype, rows, dim, x_stride, codes, code_stride,
                                              (uint8_t *)scales, scale_stride, dst_rows,
                                              as_stream(stream)));
}

csa2_status csa2_quantize_kv_batch(const csa2_quant_job *jobs, int n_jobs, void *stream) {
    const Range range("csa2_quantize_kv_batch");
    if (n_jobs < 0 || n_jobs > CSA2_MAX_QUANT_JOBS) return CSA2_ERR_SHAPE;
    if (n_jobs == 0) return CSA2_OK;
    if (!jobs) return CSA2_ERR_INVALID_ARG;
    for (int i = 0; i < n_jobs; ++i) {
        const csa2_quant_job &j = jobs[i];
        const csa2_status s = check_quant_args(j.fmt, j.x, j.x_dtype, j.rows, j.dim, j.x_stride, j.codes,
                                               j.code_stride, j.scales, j.scale_stride);
        if (s != CSA2_OK) return s;
    }
    return cuda_status(launch_quant_batch(jobs, n_jobs, as_stream(stream)));
}

csa2_status csa2_compress_quantize_kv(const void *x, int x_dtype, int64_t entries, int ratio, int dim,
                                      int64_t x_stride, const float *w, int64_t w_stride,
                                      uint8_t *codes, int64_t code_stride, uint8_t *scales,
                                      int64_t scale_stride, const int64_t *dst_rows, void *stream) {
    const Range range("csa2_compress_quantize_kv");
    if (x_dtype != CSA2_DTYPE_F32 && x_dtype != CSA2_DTYPE_BF16) return CSA2_ERR_INVALID_ARG;
    if (entries == 0) return CSA2_OK;
    if (entries < 0 || ratio < 1 || ratio > CSA2_MAX_COMPRESS_RATIO || dim <= 0 || (dim % 16) ||
        dim > 65536 || x_stride < dim)
        return CSA2_ERR_SHAPE;
    if (!x || !codes || !scales) return CSA2_ERR_INVALID_ARG;
    if ((w && w_stride < ratio) || code_stride < dim / 2 || scale_stride < dim / 16) return CSA2_ERR_SHAPE;
    return cuda_status(launch_compress_fp4(x, x_dtype, entries, ratio, dim, x_stride, w, w_stride, codes,
                                           code_stride, scales, scale_stride, dst_rows, as_stream(stream)));
}

csa2_status csa2_index_topk_workspace_size(int mode, int rows, int64_t max_n, int K, int P,
                                           size_t *bytes) {
    if (!bytes) return CSA2_ERR_INVALID_ARG;
    if (rows <= 0 || max_n < 0 || K < 1 || P < 0) return CSA2_ERR_SHAPE;
    *bytes = index_ws(mode, rows, max_n, K, P);
    return CSA2_OK;
}

csa2_status csa2_index_topk(int mode, const uint8_t *q_codes, const uint8_t *q_scales,
                            const float *w, int B, int T, int H_I, const uint8_t *k_codes,
                            int64_t k_code_stride, const uint8_t *k_scales, int64_t k_scale_stride,
                            const int64_t *seq_start, const int32_t *n_entries, int64_t max_n,
                            const int32_t *q_pos, const int32_t *pool, const int32_t *pool_len,
                            int P_in, int K, int32_t *out_idx, int32_t *out_cnt, int P,
                            int32_t *out_pool, int32_t *out_pool_len, void *workspace,
                            size_t ws_bytes, void *stream) {
    const Range range("csa2_index_topk");
    csa2_status s = check_index_args(mode, q_codes, q_scales, w, B, T, H_I, k_codes, k_code_stride,
                                     k_scales, k_scale_stride, seq_start, n_entries, max_n, pool,
                                     pool_len, P_in, K, out_idx, P, out_pool);
    if (s != CSA2_OK) return s;
    const int rows = B * T;
    const size_t need = index_ws(mode, rows, max_n, K, mode == CSA2_MODE_REINDEX ? P_in : P);
    if (!workspace || ws_bytes < need) return CSA2_ERR_WORKSPACE;
    IndexLaunch L;
    L.mode = mode; L.q_codes = q_codes; L.q_scales = q_scales; L.w = w;
    L.B = B; L.T = T; L.H = H_I;
    L.k_codes = k_codes; L.k_code_stride = k_code_stride;
    L.k_scales = k_scales; L.k_scale_stride = k_scale_stride;
    L.seq_start = seq_start; L.n_entries = n_entries; L.max_n = max_n; L.q_pos = q_pos;
    L.pool = pool; L.pool_len = pool_len; L.P_in = P_in;
    L.K = K; L.out_idx = out_idx; L.out_cnt = out_cnt;
    L.P = P; L.out_pool = out_pool; L.out_pool_len = out_pool_len;
    L.workspace = workspace; L.ws_bytes = ws_bytes;
    L.out_scores = nullptr;
    return cuda_status(launch_index_topk(L, as_stream(stream)));
}

csa2_status csa2_index_topk_scored(const uint8_t *q_codes, const uint8_t *q_scales, const float *w, int B,
                                   int T, int H_I, const uint8_t *k_codes, int64_t k_code_stride,
                                   const uint8_t *k_scales, int64_t k_scale_stride,
                                   const int64_t *seq_start, const int32_t *n_entries, int64_t max_n,
                                   const int32_t *q_pos, int K, int32_t *out_idx, int32_t *out_cnt,
                                   float *out_scores, void *workspace, size_t ws_bytes, void *stream) {
    const Range range("csa2_index_topk_scored");
    if (!out_scores) return CSA2_ERR_INVALID_ARG;
    csa2_status s = check_index_args(CSA2_MODE_FULL, q_codes, q_scales, w, B, T, H_I, k_codes, k_code_stride,
                                     k_scales, k_scale_stride, seq_start, n_entries, max_n, nullptr,
                                     nullptr, 0, K, out_idx, 0, nullptr);
    if (s != CSA2_OK) return s;
    const int rows = B * T;
    if (!workspace || ws_bytes < index_ws(CSA2_MODE_FULL, rows, max_n, K, 0)) return CSA2_ERR_WORKSPACE;
    IndexLaunch L;
    L.mode = CSA2_MODE_FULL; L.q_codes = q_codes; L.q_scales = q_scales; L.w = w;
    L.B = B; L.T = T; L.H = H_I;
    L.k_codes = k_codes; L.k_code_stride = k_code_stride;
    L.k_scales = k_scales; L.k_scale_stride = k_scale_stride;
    L.seq_start = seq_start; L.n_entries = n_entries; L.max_n = max_n; L.q_pos = q_pos;
    L.pool = nullptr; L.pool_len = nullptr; L.P_in = 0;
    L.K = K; L.out_idx = out_idx; L.out_cnt = out_cnt;
    L.P = 0; L.out_pool = nullptr; L.out_pool_len = nullptr;
    L.workspace = workspace; L.ws_bytes = ws_bytes;
    L.out_scores = out_scores;
    return cuda_status(launch_index_topk(L, as_stream(stream)));
}

csa2_status csa2_topk_merge_shards_workspace_size(int G, int rows, int K_in, size_t *bytes) {
    if (!bytes) return CSA2_ERR_INVALID_ARG;
    if (G <= 0 || rows <= 0 || K_in <= 0) return CSA2_ERR_SHAPE;
    *bytes = topk_merge_workspace_bytes(G, rows, K_in);
    return CSA2_OK;
}

csa2_status csa2_topk_merge_shards(const float *scores, const int32_t *ids, const int64_t *id_offset,
                                   const int32_t *cnt, int G, int rows, int K_in, int K, int32_t *out_idx,
                                   int32_t *out_cnt, void *workspace, size_t ws_bytes, void *stream) {
    const Range range("csa2_topk_merge_shards");
    if (!scores || !ids || !cnt || !out_idx) return CSA2_ERR_INVALID_ARG;
    if (G <= 0 || rows <= 0 || K_in <= 0 || K < 1 || K > CSA2_MAX_TOPK) return CSA2_ERR_SHAPE;
    if ((int64_t)G * K_in > topk_cluster_max_n()) return CSA2_ERR_UNSUPPORTED;
    if (!workspace || ws_bytes < topk_merge_workspace_bytes(G, rows, K_in)) return CSA2_ERR_WORKSPACE;
    return cuda_status(launch_topk_merge_shards(scores, ids, id_offset, cnt, G, rows, K_in, K, out_idx, out_cnt,
                                                workspace, as_stream(stream)));
}

csa2_status csa2_pool_extend(const int32_t *pool, const int32_t *pool_len, int P_in, const int32_t *n_ref,
                             const int32_t *n_entries, const int32_t *q_pos, int B, int T, int P_out,
                             int32_t *out_pool, int32_t *out_len, void *stream) {
    const Range range("csa2_pool_extend");
    if (!pool || !pool_len || !n_ref || !n_entries || !out_pool || !out_len) return CSA2_ERR_INVALID_ARG;
    if (B <= 0 || T <= 0 || (int64_t)B * T > (1 << 30) || P_in < 0 || P_out < 1 || P_out > CSA2_MAX_POOL)
        return CSA2_ERR_SHAPE;
    return cuda_status(launch_pool_extend(pool, pool_len, P_in, n_ref, n_entries, q_pos, B * T, T, P_out, out_pool,
                                          out_len, as_stream(stream)));
}

csa2_status csa2_attn_merge_shards(const float *outs, const float *lses, int G, int rows, int H, int D,
                                   void *out, int out_dtype, float *lse, void *stream) {
    const Range range("csa2_attn_merge_shards");
    if (!outs || !lses || !out) return CSA2_ERR_INVALID_ARG;
    if (out_dtype != CSA2_DTYPE_F32 && out_dtype != CSA2_DTYPE_BF16) return CSA2_ERR_INVALID_ARG;
    if (G <= 0 || rows <= 0 || H <= 0 || D <= 0 || (D % 4)) return CSA2_ERR_SHAPE;
    if ((((uintptr_t)outs) & 15u) || (((uintptr_t)out) & 15u)) return CSA2_ERR_ALIGN;
    return cuda_status(launch_attn_merge_shards(outs, lses, G, rows, H, D, out, out_dtype, lse, as_stream(stream)));
}

csa2_status csa2_sparse_attn_plan(int rows, int H, int K, int *hgroups, int *splits, int *keys_per_split) {
    if (!hgroups || !splits || !keys_per_split) return CSA2_ERR_INVALID_ARG;
    if (rows <= 0 || H <= 0 || K <= 0) return CSA2_ERR_SHAPE;
    attn_plan(rows, H, K, *hgroups, *splits, *keys_per_split);
    return CSA2_OK;
}

csa2_status csa2_sparse_attn_workspace_size(int rows, int H, int K, size_t *bytes) {
    if (!bytes) return CSA2_ERR_INVALID_ARG;
    if (rows <= 0 || H <= 0 || K <= 0) return CSA2_ERR_SHAPE;
    *bytes = attn_ws(rows, H, K);
    return CSA2_OK;
}

csa2_status csa2_sparse_attn(const uint16_t *q, int B, int T, int H, int D, const uint8_t *kv,
                             int64_t kv_row_stride, const int64_t *seq_start,
                             const int32_t *n_entries, const int32_t *idx,
                             const int32_t *cnt, int K, const uint8_t *swa_codes,
                             const float *swa_scale, int swa_cap, const int32_t *swa_start,
                             const int32_t *swa_len, float softmax_scale, void *out,
                             int out_dtype, float *lse, void *workspace, size_t ws_bytes,
                             void *stream) {
    const Range range("csa2_sparse_attn");
    csa2_status s = check_attn_args(q, B, T, H, D, kv, kv_row_stride, seq_start, idx, K, swa_codes,
                                    swa_scale, swa_cap, swa_len, out, out_dtype);
    if (s != CSA2_OK) return s;
    const int rows = B * T;
    if (!workspace || ws_bytes < attn_ws(rows, H, K)) return CSA2_ERR_WORKSPACE;
    if (!aligned16(workspace)) return CSA2_ERR_ALIGN;
    AttnArgs a;
    a.q = q; a.rows = rows; a.T = T; a.H = H; a.K = K;
    a.kv = kv; a.kv_row_stride = kv_row_stride; a.seq_start = seq_start; a.n_entries = n_entries;
    a.shard_lo = nullptr; a.shard_n = nullptr;
    a.idx = idx; a.cnt = cnt;
    a.swa_codes = swa_codes; a.swa_scale = swa_scale; a.swa_cap = swa_cap;
    a.swa_start = swa_start; a.swa_len = swa_len;
    a.softmax_scale = softmax_scale; a.out = out; a.out_dtype = out_dtype; a.lse = lse;
    a.partials = reinterpret_cast<float *>(workspace);
    a.splits = 1;
    return cuda_status(launch_attn(a, as_stream(stream)));
}

csa2_status csa2_sparse_attn_shard(const uint16_t *q, int B, int T, int H, int D, const uint8_t *kv,
                                   int64_t kv_row_stride, const int64_t *seq_start, const int64_t *shard_lo,
                                   const int32_t *shard_n, const int32_t *idx, const int32_t *cnt, int K,
                                   const uint8_t *swa_codes, const float *swa_scale, int swa_cap,
                                   const int32_t *swa_start, const int32_t *swa_len, float softmax_scale,
                                   float *out, float *lse, void *workspace, size_t ws_bytes, void *stream) {
    const Range range("csa2_sparse_attn_shard");
    if (!shard_lo || !shard_n || !lse) return CSA2_ERR_INVALID_ARG;
    csa2_status s = check_attn_args(q, B, T, H, D, kv, kv_row_stride, seq_start, idx, K, swa_codes,
                                    swa_scale, swa_cap, swa_len, out, CSA2_DTYPE_F32);
    if (s != CSA2_OK) return s;
    const int rows = B * T;
    if (!workspace || ws_bytes < attn_ws(rows, H, K)) return CSA2_ERR_WORKSPACE;
    if (!aligned16(workspace)) return CSA2_ERR_ALIGN;
    AttnArgs a;
    a.q = q; a.rows = rows; a.T = T; a.H = H; a.K = K;
    a.kv = kv; a.kv_row_stride = kv_row_stride; a.seq_start = seq_start; a.n_entries = nullptr;
    a.shard_lo = shard_lo; a.shard_n = shard_n;
    a.idx = idx; a.cnt = cnt;
    a.swa_codes = swa_codes; a.swa_scale = swa_scale; a.swa_cap = swa_cap;
    a.swa_start = swa_start; a.swa_len = swa_len;
    a.softmax_scale = softmax_scale; a.out = out; a.out_dtype = CSA2_DTYPE_F32; a.lse = lse;
    a.partials = reinterpret_cast<float *>(workspace);
    a.splits = 1;
    return cuda_status(launch_attn(a, as_stream(stream)));
}

// ------------------------------------------------------------------------------------------
// layer group
// ------------------------------------------------------------------------------------------
static csa2_status group_layout(const csa2_group_desc *g, const csa2_layer_desc *layers, int n,
                                size_t *idx_off, size_t *pool_off, size_t *idx_ws_off,
                                size_t *attn_off, size_t *total) {
    if (!g || !layers || n <= 0) return CSA2_ERR_INVALID_ARG;
    bool need_pool = false, seen_full = false;
    for (int l = 0; l < n; ++l) {
        const int m = layers[l].mode;
        if (m == CSA2_MODE_FULL) seen_full = true;
        else if (m == CSA2_MODE_REINDEX || m == CSA2_MODE_REUSE) {
            if (!seen_full) return CSA2_ERR_INVALID_ARG;
            if (m == CSA2_MODE_REINDEX) need_pool = true;
        } else return CSA2_ERR_INVALID_ARG;
    }
    if (need_pool && g->P <= 0) return CSA2_ERR_INVALID_ARG;
    if (g->B <= 0 || g->T <= 0) return CSA2_ERR_SHAPE;
    const bool keep = need_pool && g->pool_keep;
    if (keep) {
        if (!g->pool_keep_len || !g->pool_keep_n || g->q_pos) return CSA2_ERR_INVALID_ARG;
        if (g->max_new < 0 || (int64_t)g->P + g->max_new > CSA2_MAX_POOL) return CSA2_ERR_SHAPE;
    }
    // candidates the Reindex layers search: the pool, or the kept pool and the entries since
    const int p_search = keep ? g->P + g->max_new : g->P;
    const int rows = g->B * g->T;
    size_t off = 0;
    *idx_off = off; off += round_up((size_t)rows * g->K * 4 + (size_t)rows * 4);
    *pool_off = off;
    if (need_pool) off += round_up((size_t)rows * p_search * 4 + (size_t)rows * 4);
    *idx_ws_off = off;
    size_t iw = index_ws(CSA2_MODE_FULL, rows, g->max_n, g->K, need_pool ? g->P : 0);
    if (need_pool) {
        size_t iw2 = index_ws(CSA2_MODE_REINDEX, rows, g->max_n, g->K, p_search);
        if (iw2 > iw) iw = iw2;
    }
    *attn_off = off + iw;
    // two attention workspaces: layer l merges its splits from slot l % 2 on a second stream
    // while layer l + 1 runs
    off += iw + attn_ws(rows, g->H, g->K) * (n > 1 ? 2 : 1);
    *total = off;
    return CSA2_OK;
}

csa2_status csa2_layer_group_workspace_size(const csa2_group_desc *g, const csa2_layer_desc *layers,
                                            int n_layers, size_t *bytes) {
    if (!bytes) return CSA2_ERR_INVALID_ARG;
    size_t a, b, c, d;
    return group_layout(g, layers, n_layers, &a, &b, &c, &d, bytes);
}

// Per host thread and device: the stream the layer group runs its split merges on, and the
// events that order them (a thread's group calls never share them with another thread's).
struct GroupAux {
    cudaStream_t side = nullptr;
    cudaEvent_t attn_done = nullptr, merge_done[2] = {nullptr, nullptr};
};
static cudaError_t group_aux(GroupAux **out) {
    static thread_local GroupAux aux[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    GroupAux &a = aux[dev];
    if (!a.side) {
        e = cudaStreamCreateWithFlags(&a.side, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&a.attn_done, cudaEventDisableTiming);
        for (int i = 0; i < 2 && e == cudaSuccess; ++i)
            e = cudaEventCreateWithFlags(&a.merge_done[i], cudaEventDisableTiming);
        if (e != cudaSuccess) { a.side = nullptr; return e; }
    }
    *out = &a;
    return cudaSuccess;
}

csa2_status csa2_layer_group(const csa2_group_desc *g, const csa2_layer_desc *layers, int n_layers,
                             void *workspace, size_t ws_bytes, void *stream) {
    const Range range("csa2_layer_group");
    size_t idx_off, pool_off, iws_off, attn_off, total;
    csa2_status s = group_layout(g, layers, n_layers, &idx_off, &pool_off, &iws_off, &attn_off, &total);
    if (s != CSA2_OK) return s;
    if (!workspace || ws_bytes < total) return CSA2_ERR_WORKSPACE;
    if (!aligned16(workspace)) return CSA2_ERR_ALIGN;
    const int rows = g->B * g->T;
    bool need_pool = false;
    for (int l = 0; l < n_layers; ++l) need_pool |= layers[l].mode == CSA2_MODE_REINDEX;
    // kept pool: rebuilt by the Full layer on refresh, else extended by the entries written since
    const bool keep = need_pool && g->pool_keep;
    const bool rebuild = need_pool && (!keep || g->refresh);
    const int p_search = keep && !g->refresh ? g->P + g->max_new : g->P;
    // validate every layer before launching anything
    for (int l = 0; l < n_layers; ++l) {
        const csa2_layer_desc &L = layers[l];
        if (L.mode != CSA2_MODE_REUSE) {
            s = check_index_args(L.mode, L.iq_codes, L.iq_scales, L.iw, g->B, g->T, g->H_I,
                                 g->k_codes, g->k_code_stride, g->k_scales, g->k_scale_stride,
                                 g->seq_start, g->n_entries, g->max_n,
                                 L.mode == CSA2_MODE_REINDEX ? (const int32_t *)1 : nullptr,
                                 L.mode == CSA2_MODE_REINDEX ? (const int32_t *)1 : nullptr,
                                 p_search, g->K, (int32_t *)1,
                                 L.mode == CSA2_MODE_FULL && rebuild ? g->P : 0, (int32_t *)1);
            if (s != CSA2_OK) return s;
        }
        s = check_attn_args(L.q, g->B, g->T, g->H, g->D, g->kv, g->kv_row_stride, g->seq_start,
                            (const int32_t *)1, g->K, L.swa_codes, L.swa_scale, g->swa_cap,
                            g->swa_len, L.out, g->out_dtype);
        if (s != CSA2_OK) return s;
    }
    uint8_t *ws = reinterpret_cast<uint8_t *>(workspace);
    int32_t *idx = reinterpret_cast<int32_t *>(ws + idx_off);
    int32_t *cnt = idx + (size_t)rows * g->K;
    int32_t *pool = need_pool ? reinterpret_cast<int32_t *>(ws + pool_off) : nullptr;
    int32_t *pool_len = need_pool ? pool + (size_t)rows * p_search : nullptr;
    if (keep && g->refresh) {
        pool = g->pool_keep;
        pool_len = g->pool_keep_len;
    }
    void *iws = ws + iws_off;
    const size_t iws_bytes = attn_off - iws_off;
    void *aws = ws + attn_off;
    const size_t aws_one = attn_ws(rows, g->H, g->K);
    cudaStream_t st = as_stream(stream);
    GroupAux *aux = nullptr;
    {
        cudaError_t e = group_aux(&aux);
        if (e != cudaSuccess) return cuda_status(e);
    }
    if (keep && !g->refresh) {
        cudaError_t e = launch_pool_extend(g->pool_keep, g->pool_keep_len, g->P, g->pool_keep_n,
                                           g->n_entries, g->q_pos, rows, g->T, p_search, pool, pool_len, st);
        if (e != cudaSuccess) return cuda_status(e);
    }
    bool merge_pending[2] = {false, false};
    for (int l = 0; l < n_layers; ++l) {
        const csa2_layer_desc &L = layers[l];
        const Range layer_range(layer_range_name(L.mode));
        if (L.ready_event) {
            cudaError_t e = cudaStreamWaitEvent(st, reinterpret_cast<cudaEvent_t>(L.ready_event), 0);
            if (e != cudaSuccess) return cuda_status(e);
        }
        if (L.mode == CSA2_MODE_FULL) {
            s = csa2_index_topk(CSA2_MODE_FULL, L.iq_codes, L.iq_scales, L.iw, g->B, g->T, g->H_I,
                                g->k_codes, g->k_code_stride, g->k_scales, g->k_scale_stride,
                                g->seq_start, g->n_entries, g->max_n, g->q_pos, nullptr, nullptr, 0,
                                g->K, idx, cnt, rebuild ? g->P : 0, rebuild ? pool : nullptr,
                                rebuild ? pool_len : nullptr, iws, iws_bytes, stream);
            if (s == CSA2_OK && keep && g->refresh) {
                cudaError_t e = cudaMemcpyAsync(g->pool_keep_n, g->n_entries, (size_t)g->B * 4,
                                                cudaMemcpyDeviceToDevice, st);
                if (e != cudaSuccess) return cuda_status(e);
            }
        } else if (L.mode == CSA2_MODE_REINDEX) {
            s = csa2_index_topk(CSA2_MODE_REINDEX, L.iq_codes, L.iq_scales, L.iw, g->B, g->T,
                                g->H_I, g->k_codes, g->k_code_stride, g->k_scales,
                                g->k_scale_stride, g->seq_start, g->n_entries, g->max_n, g->q_pos,
                                pool, pool_len, p_search, g->K, idx, cnt, 0, nullptr, nullptr, iws,
                                iws_bytes, stream);
        }
        if (s != CSA2_OK) return s;
        // REUSE: idx/cnt still hold the preceding layer's selection
        if (L.idx_out) {
            cudaError_t e = cudaMemcpyAsync(L.idx_out, idx, (size_t)rows * g->K * 4,
                                            cudaMemcpyDeviceToDevice, st);
            if (e != cudaSuccess) return cuda_status(e);
        }
        if (L.attn_ready_event) {
            cudaError_t e = cudaStreamWaitEvent(st, reinterpret_cast<cudaEvent_t>(L.attn_ready_event), 0);
            if (e != cudaSuccess) return cuda_status(e);
        }
        // attention on `st`; its split merge on the side stream, overlapping the next layers.
        // Layer l uses workspace slot l % 2: before overwriting it, wait for layer l - 2's merge.
        const int slot = n_layers > 1 ? (l & 1) : 0;
        if (l >= 2 && merge_pending[slot]) {
            cudaError_t e = cudaStreamWaitEvent(st, aux->merge_done[slot], 0);
            if (e != cudaSuccess) return cuda_status(e);
            merge_pending[slot] = false;
        }
        AttnArgs a;
        a.q = L.q; a.rows = rows; a.T = g->T; a.H = g->H; a.K = g->K;
        a.kv = g->kv; a.kv_row_stride = g->kv_row_stride; a.seq_start = g->seq_start;
        a.n_entries = g->n_entries;
        a.shard_lo = nullptr; a.shard_n = nullptr;
        a.idx = idx; a.cnt = cnt;
        a.swa_codes = L.swa_codes; a.swa_scale = L.swa_scale; a.swa_cap = g->swa_cap;
        a.swa_start = g->swa_start; a.swa_len = g->swa_len;
        a.softmax_scale = g->softmax_scale; a.out = L.out; a.out_dtype = g->out_dtype; a.lse = L.lse;
        a.partials = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(aws) + slot * aws_one);
        a.splits = 1;
        bool merged = false;
        cudaError_t e = launch_attn_side_merge(a, st, aux->side, aux->attn_done, &merged);
        if (e != cudaSuccess) return cuda_status(e);
        if (merged) {
            e = cudaEventRecord(aux->merge_done[slot], aux->side);
            if (e != cudaSuccess) return cuda_status(e);
            merge_pending[slot] = true;
        }
        if (L.done_event) {
            e = cudaEventRecord(reinterpret_cast<cudaEvent_t>(L.done_event), merged ? aux->side : st);
            if (e != cudaSuccess) return cuda_status(e);
        }
    }
    // the group completes on `stream`: join every merge still running on the side stream
    for (int i = 0; i < 2; ++i) {
        if (!merge_pending[i]) continue;
        cudaError_t e = cudaStreamWaitEvent(st, aux->merge_done[i], 0);
        if (e != cudaSuccess) return cuda_status(e);
    }
    return CSA2_OK;
}

csa2_status csa2_selftest_bounded_wait(int skip_arrival, void *stream) {
    return cuda_status(launch_selftest_bounded_wait(skip_arrival != 0, as_stream(stream)));
}

csa2_status csa2_device_error(void *stream) {
    if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return CSA2_ERR_CUDA;
    return read_and_clear_device_error();
}

}  // extern "C"

// Indexer scoring and top-K block selection (Full and Reindex modes).
//
// [B] page "DeepSeek V4.1 Flash 如何靠压缩 KV 缓存实现小模型干翻大模型":
//   section "为什么 KV 缓存成了新瓶颈？" names the DSA-style indexer; section
//   "CSA2：三层压缩一次吃满" defines Full (own indexer query, full scan) and Reindex
//   (re-score an earlier layer's candidates with the layer's own query); section
//   "FP4 量化 + Bounded Replay" makes indexer Q and K FP4.
// [A] page "DeepSeek V4.1 Flash深度解析：KV缓存压缩437倍的技术路径", section
//   "压缩吸收注意力（二代）": the first layer picks 2048 blocks and keeps a candidate pool.
//
// Scores come from the tensor-core kernel in index_tc.cu (bit-identical to the fixed fp32
// summation order that csa2.h defines) into a bounded row-chunked buffer; selection runs on 8-CTA clusters
// (topk_cluster.cu) or, for rows longer than a cluster holds, on one CTA per row here: a 4-pass,
// 8-bit radix select on order-preserving keys, then one compaction pass in entry order
// (entries above the threshold key, plus the lowest-indexed entries equal to it, written in
// ascending index order).
#include "common.cuh"
#include "index_api.cuh"

namespace csa2 {

constexpr int kSelectThreads = 1024;

struct ScoreArgs {
    const uint8_t *q_codes;    // [rows][H][32]
    const uint8_t *q_scales;   // [rows][H][4]
    const float *w;            // [rows][H]
    int H;
    int T;
    const uint8_t *k_codes;
    int64_t k_code_stride;
    const uint8_t *k_scales;
    int64_t k_scale_stride;
    const int64_t *seq_start;
    const int32_t *n_entries;
    const int32_t *q_pos;      // nullable
    const int32_t *pool;       // Reindex: [rows][P_in]
    const int32_t *pool_len;
    int P_in;
    int row0;                  // first query row of this launch
    float *scores;             // [launch rows][score_stride]
    int64_t score_stride;
};

// Number of candidates of row r (visible entries, or pool length).
CSA2_D int64_t row_candidates(const ScoreArgs &a, int r) {
    if (a.pool) return a.pool_len[r];
    const int b = r / a.T;
    int64_t n = a.n_entries[b];
    if (a.q_pos) {
        int64_t v = ((int64_t)a.q_pos[r] + 1) / 4;
        n = v < n ? v : n;
        if (n < 0) n = 0;
    }
    return n;
}

// ---------------------------------------------------------------------------------------
// Block-wide helpers (blockDim.x == kSelectThreads)
// ---------------------------------------------------------------------------------------
// Exclusive prefix of a 0/1 flag over the block in thread order; returns the block total.
CSA2_D int block_exclusive_count(bool flag, int *warp_sums, int &total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned bal = __ballot_sync(0xffffffffu, flag);
    const int within = __popc(bal & ((1u << lane) - 1u));
    if (lane == 0) warp_sums[warp] = __popc(bal);
    __syncthreads();
    if (warp == 0) {
        int v = lane < (int)(blockDim.x >> 5) ? warp_sums[lane] : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        warp_sums[lane] = incl - v;                 // exclusive
        if (lane == 31) warp_sums[32] = incl;       // total
    }
    __syncthreads();
    const int res = warp_sums[warp] + within;
    total = warp_sums[32];
    __syncthreads();
    return res;
}

// Radix-select the threshold key of the k-th largest key among n; returns (key, how many
// entries equal to key must be taken).
__device__ void radix_threshold(const float *scores, int64_t n, int64_t k, uint32_t &thr,
                                int64_t &need_eq) {
    __shared__ unsigned int hist[256];
    __shared__ uint32_t s_prefix, s_mask;
    __shared__ long long s_remaining;
    if (threadIdx.x == 0) { s_prefix = 0u; s_mask = 0u; s_remaining = k; }
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0u;
        __syncthreads();
        const uint32_t prefix = s_prefix, mask = s_mask;
        for (int64_t j = threadIdx.x; j < n; j += blockDim.x) {
            const uint32_t key = float_key(scores[j]);
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            const int lane = threadIdx.x;
            // lane owns bins [8*lane, 8*lane+8); suffix sums from the top bin down
            unsigned int local = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) local += hist[lane * 8 + i];
            unsigned int suffix = local;               // inclusive sum of lanes >= lane
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                unsigned int t = __shfl_down_sync(0xffffffffu, suffix, o);
                if (lane + o < 32) suffix += t;
            }
            const long long rem = s_remaining;
            const unsigned int above = suffix - local;  // count in lanes > lane
            const bool crosses = (long long)above < rem && rem <= (long long)suffix;
            const unsigned bal = __ballot_sync(0xffffffffu, crosses);
            const int owner = __ffs(bal) - 1;
            if (lane == owner) {
                long long acc = above;
                int d = lane * 8 + 7;
                for (; d > lane * 8; --d) {
                    if (acc + hist[d] >= rem) break;
                    acc += hist[d];
                }
                s_remaining = rem - acc;
                s_prefix = prefix | ((uint32_t)d << shift);
                s_mask = mask | (255u << shift);
            }
        }
        __syncthreads();
    }
    thr = s_prefix;
    need_eq = s_remaining;
    __syncthreads();
}

// Select the top-k of one row into out[0..k) (ascending index, -1 padded); ids maps
// candidate positions to entry ids (NULL = identity).
__device__ void select_row(const float *scores, const int32_t *ids, int64_t n, int k,
                           int32_t *out, int32_t *out_cnt) {
    __shared__ int warp_sums[33];
    const int cnt = (int)(n < k ? n : k);
    if (n <= k) {
        for (int64_t j = threadIdx.x; j < n; j += blockDim.x) out[j] = ids ? ids[j] : (int32_t)j;
    } else {
        uint32_t thr;
        int64_t need_eq;
        radix_threshold(scores, n, k, thr, need_eq);
        int64_t run_out = 0, run_eq = 0;
        for (int64_t base = 0; base < n; base += blockDim.x) {
            const int64_t j = base + threadIdx.x;
            uint32_t key = 0u;
            if (j < n) key = float_key(scores[j]);
            const bool gt = j < n && key > thr;
            const bool eq = j < n && key == thr;
            int eq_total;
            const int eq_rank = block_exclusive_count(eq, warp_sums, eq_total);
            const bool sel = gt || (eq && run_eq + eq_rank < need_eq);
            int sel_total;
            const int pos = block_exclusive_count(sel, warp_sums, sel_total);
            if (sel && run_out + pos < k) out[run_out + pos] = ids ? ids[j] : (int32_t)j;
            run_out += sel_total;
            run_eq += eq_total;
        }
    }
    for (int i = cnt + threadIdx.x; i < k; i += blockDim.x) out[i] = -1;
    if (threadIdx.x == 0 && out_cnt) *out_cnt = cnt;
    __syncthreads();
}

struct SelectArgs {
    const float *scores;
    int64_t score_stride;
    ScoreArgs sa;              // for row_candidates()
    int K;
    int32_t *out_idx;
    int32_t *out_cnt;
    int P;
    int32_t *out_pool;
    int32_t *out_pool_len;
};

__global__ void __launch_bounds__(kSelectThreads)
select_kernel(SelectArgs a) {
    const int lr = blockIdx.x;
    const int r = a.sa.row0 + lr;
    int64_t n = row_candidates(a.sa, r);
    if (n > a.score_stride) n = a.score_stride;        // never read past the row's scores
    const float *s = a.scores + (int64_t)lr * a.score_stride;
    const int32_t *ids = a.sa.pool ? a.sa.pool + (int64_t)r * a.sa.P_in : nullptr;
    select_row(s, ids, n, a.K, a.out_idx + (int64_t)r * a.K, a.out_cnt ? a.out_cnt + r : nullptr);
    if (a.P > 0)
        select_row(s, ids, n, a.P, a.out_pool + (int64_t)r * a.P,
                   a.out_pool_len ? a.out_pool_len + r : nullptr);
}

// Rows processed per launch so the score buffer stays bounded.
static int64_t index_rows_per_chunk(int rows, int64_t max_n) {
    const int64_t cap = (int64_t)256 << 20;                       // 256 MB of scores
    int64_t per = cap / ((max_n > 0 ? max_n : 1) * 4);
    if (per < 1) per = 1;
    return per < rows ? per : rows;
}

int64_t topk_row_max_n();
int topk_row_chunks(int64_t max_n, int K, int P);
size_t topk_row_scratch_bytes(int rows, int64_t max_n, int K, int P);
cudaError_t launch_topk_row(const float *scores, int64_t score_stride, const int32_t *cand, int64_t cand_stride,
                            const int32_t *n_entries, const int32_t *q_pos, const int32_t *pool_len, int T,
                            int row0, int nrows, int K, int32_t *out_idx, int32_t *out_cnt, int P,
                            int32_t *out_pool, int32_t *out_pool_len, int64_t max_n, void *scratch,
                            cudaStream_t st);

// Scores of a row chunk, then the selection's scratch (two-phase path for long rows).
static size_t score_bytes(int64_t chunk, int64_t n) { return ((size_t)(chunk * (n > 0 ? n : 1) * 4) + 255) / 256 * 256; }

size_t index_topk_workspace_bytes(int rows, int64_t n, int K, int P) {
    const int64_t chunk = index_rows_per_chunk(rows, n);
    return score_bytes(chunk, n) + topk_row_scratch_bytes((int)chunk, n, K, P) + 256;
}

cudaError_t launch_index_score_tc(const IndexLaunch &L, int row0, int nrows, float *scores,
                                  int64_t score_stride, cudaStream_t st);
bool index_pipe_applies(const IndexLaunch &L);
cudaError_t launch_index_score_pipe(const IndexLaunch &L, int row0, int nrows, int R, float *scores,
                                    int64_t score_stride, cudaStream_t st);

int64_t topk_cluster_max_n();
cudaError_t launch_gather_scores(const float *scores, int64_t score_stride, const int32_t *idx, int K,
                                 int row0, int nrows, float *out_scores, cudaStream_t st);
cudaError_t launch_topk_cluster(const float *scores, int64_t score_stride, const int32_t *cand,
                                int cand_stride, const int32_t *n_entries, const int32_t *q_pos,
                                const int32_t *pool_len, int T, int row0, int nrows, int K,
                                int32_t *out_idx, int32_t *out_cnt, int P, int32_t *out_pool,
                                int32_t *out_pool_len, int64_t max_n, cudaStream_t st);

cudaError_t launch_index_topk(const IndexLaunch &L, cudaStream_t st) {
    ScoreArgs base;
    base.q_codes = L.q_codes; base.q_scales = L.q_scales; base.w = L.w;
    base.H = L.H; base.T = L.T;
    base.k_codes = L.k_codes; base.k_code_stride = L.k_code_stride;
    base.k_scales = L.k_scales; base.k_scale_stride = L.k_scale_stride;
    base.seq_start = L.seq_start; base.n_entries = L.n_entries; base.q_pos = L.q_pos;
    const bool reindex = L.mode == CSA2_MODE_REINDEX;
    base.pool = reindex ? L.pool : nullptr;
    base.pool_len = reindex ? L.pool_len : nullptr;
    base.P_in = L.P_in;
    const int rows = L.B * L.T;
    const int64_t max_n = reindex ? (int64_t)L.P_in : L.max_n;
    const int64_t chunk = index_rows_per_chunk(rows, max_n);
    // contiguous key ranges (Full mode) go to the pipelined score kernel
    const bool pipe = index_pipe_applies(L);
    float *scores = reinterpret_cast<float *>(L.workspace);
    for (int64_t r0 = 0; r0 < rows; r0 += chunk) {
        const int nr = (int)((rows - r0) < chunk ? (rows - r0) : chunk);
        ScoreArgs sa = base;
        sa.row0 = (int)r0;
        sa.scores = scores;
        sa.score_stride = max_n > 0 ? max_n : 1;
        if (max_n > 0) {
            cudaError_t e = pipe ? launch_index_score_pipe(L, (int)r0, nr, 1, scores, sa.score_stride, st)
                                 : launch_index_score_tc(L, (int)r0, nr, scores, sa.score_stride, st);
            if (e != cudaSuccess) return e;
        }
        const int sel_P = reindex ? 0 : L.P;
        // Few rows that the cluster kernel can hold: one cluster of CTAs per row keeps more SMs
        // busy than one CTA per row (measured faster for 16 and 32 rows of 32K-64K scores).
        const bool few_rows = max_n <= topk_cluster_max_n() && nr <= 64;
        if (!few_rows && topk_row_chunks(max_n, L.K, sel_P) > 0) {
            void *scratch = reinterpret_cast<uint8_t *>(L.workspace) + score_bytes(chunk, max_n);
            cudaError_t e = launch_topk_row(scores, sa.score_stride, sa.pool, sa.P_in, sa.n_entries, sa.q_pos,
                                            sa.pool_len, sa.T, sa.row0, nr, L.K, L.out_idx, L.out_cnt, sel_P,
                                            L.out_pool, L.out_pool_len, max_n, scratch, st);
            if (e == cudaSuccess && L.out_scores && !reindex)
                e = launch_gather_scores(scores, sa.score_stride, L.out_idx, L.K, sa.row0, nr, L.out_scores, st);
            if (e != cudaSuccess) return e;
            continue;
        }
        if (max_n <= topk_cluster_max_n()) {
            cudaError_t e = launch_topk_cluster(scores, sa.score_stride, sa.pool, sa.P_in, sa.n_entries,
                                                sa.q_pos, sa.pool_len, sa.T, sa.row0, nr, L.K, L.out_idx,
                                                L.out_cnt, reindex ? 0 : L.P, L.out_pool, L.out_pool_len,
                                                max_n, st);
            if (e == cudaSuccess && L.out_scores && !reindex)
                e = launch_gather_scores(scores, sa.score_stride, L.out_idx, L.K, sa.row0, nr, L.out_scores, st);
            if (e != cudaSuccess) return e;
            continue;
        }
        SelectArgs se;
        se.scores = scores;
        se.score_stride = sa.score_stride;
        se.sa = sa;
        se.K = L.K;
        se.out_idx = L.out_idx;
        se.out_cnt = L.out_cnt;
        se.P = reindex ? 0 : L.P;
        se.out_pool = L.out_pool;
        se.out_pool_len = L.out_pool_len;
        select_kernel<<<nr, kSelectThreads, 0, st>>>(se);
        note_launches(1);
        cudaError_t e = cudaGetLastError();
        if (e == cudaSuccess && L.out_scores && !reindex)
            e = launch_gather_scores(scores, sa.score_stride, L.out_idx, L.K, sa.row0, nr, L.out_scores, st);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// ---------------------------------------------------------------------------------------
// pool kept across decode steps: the kept pool followed by the entries written since
// ---------------------------------------------------------------------------------------
__global__ void pool_extend_kernel(const int32_t *__restrict__ pool, const int32_t *__restrict__ pool_len,
                                   int P_in, const int32_t *__restrict__ n_ref,
                                   const int32_t *__restrict__ n_entries, const int32_t *__restrict__ q_pos,
                                   int T, int P_out, int32_t *__restrict__ out_pool, int32_t *__restrict__ out_len) {
    const int r = blockIdx.x;
    const int b = r / T;
    const int kept = max(0, min(pool_len[r], P_in));
    int64_t n = n_entries[b];
    if (q_pos) {
        const int64_t v = ((int64_t)q_pos[r] + 1) / 4;
        n = v < n ? v : n;
    }
    const int64_t lo = max(0, n_ref[b]);
    const int64_t fresh = n > lo ? n - lo : 0;
    int64_t total = kept + fresh;
    if (total > P_out) {
        if (threadIdx.x == 0) raise_device_error(CSA2_ERR_SHAPE);
        total = P_out;
    }
    const int32_t *src = pool + (int64_t)r * P_in;
    int32_t *dst = out_pool + (int64_t)r * P_out;
    for (int64_t i = threadIdx.x; i < total; i += blockDim.x)
        dst[i] = i < kept ? src[i] : (int32_t)(lo + (i - kept));
    if (threadIdx.x == 0) out_len[r] = (int32_t)total;
}

cudaError_t launch_pool_extend(const int32_t *pool, const int32_t *pool_len, int P_in, const int32_t *n_ref,
                               const int32_t *n_entries, const int32_t *q_pos, int rows, int T, int P_out,
                               int32_t *out_pool, int32_t *out_len, cudaStream_t st) {
    pool_extend_kernel<<<rows, 256, 0, st>>>(pool, pool_len, P_in, n_ref, n_entries, q_pos, T, P_out, out_pool,
                                             out_len);
    note_launches(1);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------------------
// device error word
// ---------------------------------------------------------------------------------------
csa2_status read_and_clear_device_error() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess) return CSA2_ERR_CUDA;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return CSA2_ERR_CUDA;
    }
    return (csa2_status)v;
}

}  // namespace csa2

// Top-K (and pool) selection with one CTA per list, the list's keys held in shared memory.
//
// [A] page "DeepSeek V4.1 Flash深度解析：KV缓存压缩437倍的技术路径", section
// "压缩吸收注意力（二代）": the indexer keeps the 2048 best blocks of the context and the first
// layer's candidate pool; order = score descending, entry index ascending on ties; the selected
// ids are written ascending.
//
// A list is a sequence of (score, id) candidates whose ids ascend with the position (a row's
// consecutive entries, a Reindex pool, or the concatenated per-chunk selections of a long row),
// so "lower index first" on ties is "earlier position first".  One CTA of 1024 threads:
//   1. loads the list's order-preserving 32-bit keys into shared memory (16 independent loads in
//      flight per thread) and counts their top 8 bits on the way;
//   2. finds the exact threshold key of the k-th place in four 8-bit digits.  Histograms are
//      per lane (bin b of lane l at b * 32 + l), so the 32 lanes of a warp always add into 32
//      different banks.  After the first digit the keys of the threshold bin are copied into a
//      candidate array (when they fit), and the three refinement digits scan only those;
//   3. writes the selection in position order: each thread owns a consecutive run of keys, and
//      two block scans (equal keys before the run, then selected keys before it) give every
//      thread its output offset.  Lists with explicit ids first write positions, then map them
//      to ids in a second, coalesced pass.
// The pool (top-P of the same order) is a second selection over the same keys, reusing the first
// digit's histogram.  Lists longer than shared memory holds go through two phases: every chunk of
// a row selects its top-max(K, P) with their scores, then one CTA per row selects from the union
// of the chunk selections (the row's top-k lies inside it, and the union keeps position order).
#include "common.cuh"

namespace csa2 {
namespace tkr {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kUnroll = 16;                        // independent loads in flight per thread
constexpr int kMaxKeys = 36864;                    // keys per CTA in shared memory (144 KB)
constexpr int kCandCap = 8192;                     // keys of the threshold bin kept apart (32 KB)
constexpr int kChunk = 32768;                      // chunk length of the two-phase path
constexpr int kBins = 256;                         // 8-bit digits
constexpr int kMaxSeg = 32;                        // segments of a phase-2 list

// One CTA's list: nseg segments in order; segment s holds cnt[s] candidates with scores at
// score[s][i] and ids at id[s][i] (or id_base[s] + i when id[s] is NULL).
struct List {
    int nseg;
    const float *score[kMaxSeg];
    const int32_t *id[kMaxSeg];
    int64_t id_base[kMaxSeg];
    int cnt[kMaxSeg];
};

struct Args {
    // plain or phase 1 (nseg_in == 0): row lr's scores at scores + lr * score_stride; its length
    // from n_entries / q_pos (entries) or pool_len (candidate lists); ids from cand (+ row *
    // cand_stride) or the position.  Phase 1 takes chunk blockIdx.x of kChunk candidates.
    const float *scores;
    int64_t score_stride;
    const int32_t *cand;
    int64_t cand_stride;
    const int32_t *n_entries;
    const int32_t *q_pos;
    const int32_t *pool_len;
    int T;
    int row0;
    bool phase1;
    // phase 2 (nseg_in > 0): row lr's segments s at seg_scores / seg_ids + (lr * nseg_in + s) *
    // seg_stride, seg_cnt[lr * nseg_in + s] candidates each
    int nseg_in;
    const float *seg_scores;
    const int32_t *seg_ids;
    const int32_t *seg_cnt;
    int64_t seg_stride;
    // outputs.  Plain / phase 2: out_idx [rows][K] + out_cnt, out_pool [rows][P] + out_pool_len
    // (global row r = row0 + lr).  Phase 1: ids, scores and count of chunk c's top-kc at
    // ph1_ids / ph1_scores + (lr * gridDim.x + c) * kc, ph1_cnt[lr * gridDim.x + c].
    int K;
    int32_t *out_idx;
    int32_t *out_cnt;
    int P;
    int32_t *out_pool;
    int32_t *out_pool_len;
    int kc;
    int32_t *ph1_ids;
    float *ph1_scores;
    int32_t *ph1_cnt;
};

struct Shared {
    unsigned int hp[kBins * 32];                   // per-lane histograms
    unsigned int hist[kBins];                      // their sum (current digit)
    unsigned int hist1[kBins];                     // the first digit's sum over all keys (kept)
    int seg_start[kMaxSeg + 1];
    int warp_sums[kWarps + 1];
    uint32_t prefix, mask;
    int remaining;
    int ncand;
    List list;
};

CSA2_D float key_to_float(uint32_t k) {
    const uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
    return __uint_as_float(u);
}

// Block-wide exclusive sum of per-thread counts in thread order; total = the block's sum.
CSA2_D int block_excl_sum(int v, int *ws, int &total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += x;
    }
    if (lane == 31) ws[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int w = lane < kWarps ? ws[lane] : 0;
        int wincl = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int x = __shfl_up_sync(0xffffffffu, wincl, o);
            if (lane >= o) wincl += x;
        }
        ws[lane] = wincl - w;
        if (lane == 31) ws[kWarps] = wincl;
    }
    __syncthreads();
    const int res = ws[warp] + incl - v;
    total = ws[kWarps];
    __syncthreads();
    return res;
}

CSA2_D void hist_add(Shared &S, uint32_t bin) { atomicAdd(&S.hp[bin * 32 + (threadIdx.x & 31)], 1u); }

CSA2_D void hist_clear(Shared &S) {
    for (int i = threadIdx.x; i < kBins * 32; i += kThreads) S.hp[i] = 0u;
}

// dst[b] = sum over lanes of hp[b * 32 + lane]; warp w sums bins w, w + 32, ...
CSA2_D void hist_reduce(Shared &S, unsigned int *dst) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int b = warp; b < kBins; b += kWarps) {
        const unsigned v = __reduce_add_sync(0xffffffffu, S.hp[b * 32 + lane]);
        if (lane == 0) dst[b] = v;
    }
}

// Warp 0 finds, in histogram h, the digit d where the count from the top crosses S.remaining;
// it sets S.prefix |= d << shift, S.mask |= 0xFF << shift, S.remaining -= (count above d).
CSA2_D void pick_digit(Shared &S, const unsigned int *h, int shift) {
    if (threadIdx.x >= 32) return;
    const int lane = threadIdx.x;
    constexpr int per = kBins / 32;                // bins owned by a lane: [per*lane, per*lane+per)
    unsigned int bins[per];
    unsigned int local = 0;
#pragma unroll
    for (int i = 0; i < per; ++i) {
        bins[i] = h[lane * per + i];
        local += bins[i];
    }
    unsigned int suffix = local;                   // sum over lanes >= lane
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned int x = __shfl_down_sync(0xffffffffu, suffix, o);
        if (lane + o < 32) suffix += x;
    }
    const int rem = S.remaining;
    const unsigned int above = suffix - local;
    const bool crosses = (int)above < rem && rem <= (int)suffix;
    const unsigned bal = __ballot_sync(0xffffffffu, crosses);
    const int owner = __ffs(bal) - 1;
    if (lane == owner) {
        int acc = (int)above;
        int d = per - 1;
        for (; d > 0; --d) {
            if (acc + (int)bins[d] >= rem) break;
            acc += (int)bins[d];
        }
        S.remaining = rem - acc;
        S.prefix |= (uint32_t)(lane * per + d) << shift;
        S.mask |= 0xFFu << shift;
    }
}

// Threshold key of the k-th place among the m keys (k < m) and how many keys equal to it are
// taken.  S.hist1 holds the first digit's histogram of all keys.
CSA2_D void threshold(Shared &S, const uint32_t *keys, uint32_t *cand, int m, int k, uint32_t &thr,
                      int &need_eq) {
    if (threadIdx.x == 0) { S.prefix = 0u; S.mask = 0u; S.remaining = k; S.ncand = 0; }
    __syncthreads();
    pick_digit(S, S.hist1, 24);
    __syncthreads();
    // the keys of the threshold bin, when they fit the candidate array (order does not matter)
    const uint32_t d1 = S.prefix >> 24;
    const bool compact = S.hist1[d1] <= (unsigned)kCandCap;
    if (compact) {
        for (int base = 0; base < m; base += kThreads) {
            const int i = base + threadIdx.x;
            const uint32_t key = i < m ? keys[i] : 0u;
            const bool in = i < m && (key >> 24) == d1;
            const unsigned bal = __ballot_sync(0xffffffffu, in);
            int off = 0;
            if ((threadIdx.x & 31) == 0 && bal) off = atomicAdd(&S.ncand, __popc(bal));
            off = __shfl_sync(0xffffffffu, off, 0);
            if (in) cand[off + __popc(bal & ((1u << (threadIdx.x & 31)) - 1u))] = key;
        }
        __syncthreads();
    }
    const uint32_t *src = compact ? cand : keys;
    const int n = compact ? S.ncand : m;
    for (int pass = 1; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        hist_clear(S);
        __syncthreads();
        const uint32_t prefix = S.prefix, mask = S.mask;
        for (int i = threadIdx.x; i < n; i += kThreads) {
            const uint32_t key = src[i];
            if ((key & mask) == prefix) hist_add(S, (key >> shift) & 255u);
        }
        __syncthreads();
        hist_reduce(S, S.hist);
        __syncthreads();
        pick_digit(S, S.hist, shift);
        __syncthreads();
    }
    thr = S.prefix;
    need_eq = S.remaining;
    __syncthreads();
}

CSA2_D int seg_of(const Shared &S, int pos, int s) {
    while (pos >= S.seg_start[s + 1]) ++s;
    return s;
}

CSA2_D int32_t id_at(const Shared &S, int pos) {
    int lo = 0, hi = S.list.nseg - 1;              // last segment whose start <= pos
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (S.seg_start[mid] <= pos) lo = mid; else hi = mid - 1;
    }
    const int j = pos - S.seg_start[lo];
    return S.list.id[lo] ? __ldg(S.list.id[lo] + j) : (int32_t)(S.list.id_base[lo] + j);
}

// Writes the selection (k < m) or every candidate (k >= m) in position order to out[0..k) (ids),
// out_scores (optional), pads with -1 and stores the count.  `direct`: ids are positions plus
// id_base[0] (one segment without explicit ids), so they are written at once; otherwise the
// positions are written first and mapped to ids in a second pass.
CSA2_D void emit(Shared &S, const uint32_t *keys, int m, int k, bool select, uint32_t thr, int need_eq,
                 int32_t *out, float *out_scores, int32_t *cnt_out) {
    const bool direct = S.list.nseg == 1 && S.list.id[0] == nullptr;
    const int per = ((m + kThreads - 1) / kThreads) | 1;     // odd: a warp's lanes hit 32 banks
    const int i0 = min(m, (int)threadIdx.x * per), i1 = min(m, i0 + per);
    int my_gt = 0, my_eq = 0;
    if (select) {
        for (int i = i0; i < i1; ++i) {
            const uint32_t key = keys[i];
            my_gt += key > thr;
            my_eq += key == thr;
        }
    } else {
        my_gt = i1 - i0;
    }
    int eq_tot;
    const int eq_pre = block_excl_sum(my_eq, S.warp_sums, eq_tot);
    const int take = select ? min(my_eq, max(0, need_eq - eq_pre)) : 0;
    int sel_tot;
    int o = block_excl_sum(my_gt + take, S.warp_sums, sel_tot);
    int eq_seen = 0;
    const int64_t base = S.list.id_base[0];
    for (int i = i0; i < i1; ++i) {
        const uint32_t key = keys[i];
        const bool sel = !select || key > thr || (key == thr && eq_seen++ < take);
        if (sel) {
            if (o < k) {
                out[o] = direct ? (int32_t)(base + i) : i;
                if (out_scores) out_scores[o] = key_to_float(key);
            }
            ++o;
        }
    }
    const int c = min(k, m);
    for (int i = c + threadIdx.x; i < k; i += kThreads) {
        out[i] = -1;
        if (out_scores) out_scores[i] = -INFINITY;
    }
    if (threadIdx.x == 0 && cnt_out) *cnt_out = c;
    if (!direct) {
        __syncthreads();                            // every position is written
        for (int i0b = 0; i0b < c; i0b += kThreads * 8) {
            int32_t v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = i0b + u * kThreads + threadIdx.x;
                v[u] = i < c ? id_at(S, out[i]) : 0;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = i0b + u * kThreads + threadIdx.x;
                if (i < c) out[i] = v[u];
            }
        }
    }
    __syncthreads();
}

CSA2_D int64_t row_len(const Args &a, int r) {
    if (a.cand) return max(a.pool_len[r], 0);
    const int b = r / a.T;
    int64_t n = a.n_entries[b];
    if (a.q_pos) {
        const int64_t v = ((int64_t)a.q_pos[r] + 1) / 4;
        n = v < n ? v : n;
        if (n < 0) n = 0;
    }
    return n;
}

__global__ void __launch_bounds__(kThreads, 1) topk_row_kernel(Args a) {
    extern __shared__ __align__(16) uint32_t keys[];     // kMaxKeys keys, then kCandCap candidates
    uint32_t *cand = keys + kMaxKeys;
    __shared__ Shared S;
    const int lr = blockIdx.y;
    const int r = a.row0 + lr;
    // ---- the CTA's list
    if (threadIdx.x == 0) {
        List &L = S.list;
        if (a.nseg_in == 0) {
            int64_t n = row_len(a, r);
            if (n > a.score_stride) n = a.score_stride;       // never read past the row's scores
            int64_t lo = 0;
            if (a.phase1) {
                lo = (int64_t)blockIdx.x * kChunk;
                n = max((int64_t)0, min((int64_t)kChunk, n - lo));
            }
            L.nseg = 1;
            L.score[0] = a.scores + (int64_t)lr * a.score_stride + lo;
            L.id[0] = a.cand ? a.cand + (int64_t)r * a.cand_stride + lo : nullptr;
            L.id_base[0] = lo;
            L.cnt[0] = (int)n;
        } else {
            L.nseg = a.nseg_in;
            for (int s = 0; s < a.nseg_in; ++s) {
                const int64_t off = ((int64_t)lr * a.nseg_in + s) * a.seg_stride;
                L.score[s] = a.seg_scores + off;
                L.id[s] = a.seg_ids + off;
                L.id_base[s] = 0;
                L.cnt[s] = max(0, min((int)a.seg_stride, a.seg_cnt[(int64_t)lr * a.nseg_in + s]));
            }
        }
        int acc = 0;
        for (int s = 0; s < L.nseg; ++s) {
            S.seg_start[s] = acc;
            acc += L.cnt[s];
        }
        for (int s = L.nseg; s <= kMaxSeg; ++s) S.seg_start[s] = acc;
    }
    hist_clear(S);
    __syncthreads();
    const int m = S.seg_start[kMaxSeg];
    // ---- keys into shared memory, kUnroll independent loads per thread at a time; the first
    //      digit's histogram on the way
    const bool one_seg = S.list.nseg == 1;
    const float *sc0 = S.list.score[0];
    for (int base = 0; base < m; base += kThreads * kUnroll) {
        float v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int i = base + u * kThreads + threadIdx.x;
            v[u] = 0.0f;
            if (i < m) {
                if (one_seg) {
                    v[u] = __ldg(sc0 + i);
                } else {
                    const int s = seg_of(S, i, 0);
                    v[u] = __ldg(S.list.score[s] + (i - S.seg_start[s]));
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int i = base + u * kThreads + threadIdx.x;
            if (i < m) {
                const uint32_t key = float_key(v[u]);
                keys[i] = key;
                hist_add(S, key >> 24);
            }
        }
    }
    __syncthreads();
    hist_reduce(S, S.hist1);
    __syncthreads();
    // ---- selections
    if (a.phase1) {
        const int64_t o = ((int64_t)lr * gridDim.x + blockIdx.x) * a.kc;
        uint32_t thr = 0u;
        int need_eq = 0;
        const bool sel = a.kc < m;
        if (sel) threshold(S, keys, cand, m, a.kc, thr, need_eq);
        emit(S, keys, m, a.kc, sel, thr, need_eq, a.ph1_ids + o, a.ph1_scores + o,
             a.ph1_cnt + (int64_t)lr * gridDim.x + blockIdx.x);
        return;
    }
    for (int which = 0; which < 2; ++which) {
        const int k = which == 0 ? a.K : a.P;
        if (k <= 0) continue;
        int32_t *out = which == 0 ? a.out_idx + (int64_t)r * a.K : a.out_pool + (int64_t)r * a.P;
        int32_t *cnt = which == 0 ? (a.out_cnt ? a.out_cnt + r : nullptr)
                                  : (a.out_pool_len ? a.out_pool_len + r : nullptr);
        uint32_t thr = 0u;
        int need_eq = 0;
        const bool sel = k < m;
        if (sel) threshold(S, keys, cand, m, k, thr, need_eq);
        emit(S, keys, m, k, sel, thr, need_eq, out, nullptr, cnt);
    }
}

constexpr size_t kSmemBytes = (size_t)(kMaxKeys + kCandCap) * sizeof(uint32_t);

}  // namespace tkr

static SmemLimit g_topk_row_smem;

int64_t topk_row_max_n() { return tkr::kMaxKeys; }

// Chunks per row of the two-phase path for rows of up to max_n candidates (1: one CTA per row),
// or 0 when the union of the chunks' selections would not fit one CTA.
int topk_row_chunks(int64_t max_n, int K, int P) {
    if (max_n <= tkr::kMaxKeys) return 1;
    const int64_t chunks = ceil_div(max_n, (int64_t)tkr::kChunk);
    const int kc = K > P ? K : P;
    if (chunks > tkr::kMaxSeg || chunks * (int64_t)kc > tkr::kMaxKeys) return 0;
    return (int)chunks;
}

// Scratch of the two-phase path: ids + scores of every chunk's selection and the counts.
size_t topk_row_scratch_bytes(int rows, int64_t max_n, int K, int P) {
    const int chunks = topk_row_chunks(max_n, K, P);
    if (chunks <= 1) return 0;
    const int kc = K > P ? K : P;
    return (size_t)rows * chunks * ((size_t)kc * 8 + 4) + 256;
}

// Selection for rows [row0, row0 + nrows) from scores in global memory (row lr of this launch
// at scores + lr * score_stride).  cand: NULL (ids = positions) or the candidate ids [rows][stride].
cudaError_t launch_topk_row(const float *scores, int64_t score_stride, const int32_t *cand, int64_t cand_stride,
                            const int32_t *n_entries, const int32_t *q_pos, const int32_t *pool_len, int T,
                            int row0, int nrows, int K, int32_t *out_idx, int32_t *out_cnt, int P,
                            int32_t *out_pool, int32_t *out_pool_len, int64_t max_n, void *scratch,
                            cudaStream_t st) {
    cudaError_t e = ensure_smem_limit(g_topk_row_smem, tkr::topk_row_kernel, (int)tkr::kSmemBytes);
    if (e != cudaSuccess) return e;
    tkr::Args a{};
    a.scores = scores; a.score_stride = score_stride; a.cand = cand; a.cand_stride = cand_stride;
    a.n_entries = n_entries; a.q_pos = q_pos; a.pool_len = pool_len; a.T = T; a.row0 = row0;
    a.K = K; a.out_idx = out_idx; a.out_cnt = out_cnt; a.P = P; a.out_pool = out_pool;
    a.out_pool_len = out_pool_len;
    const int chunks = topk_row_chunks(max_n, K, P);
    if (chunks == 1) {
        tkr::topk_row_kernel<<<dim3(1, nrows), tkr::kThreads, tkr::kSmemBytes, st>>>(a);
        note_launches(1);
        return cudaGetLastError();
    }
    if (chunks == 0) return cudaErrorInvalidValue;
    const int kc = K > P ? K : P;
    int32_t *ids = reinterpret_cast<int32_t *>(scratch);
    float *sc = reinterpret_cast<float *>(ids + (size_t)nrows * chunks * kc);
    int32_t *cnt = reinterpret_cast<int32_t *>(sc + (size_t)nrows * chunks * kc);
    tkr::Args p1 = a;
    p1.phase1 = true;
    p1.kc = kc; p1.ph1_ids = ids; p1.ph1_scores = sc; p1.ph1_cnt = cnt;
    tkr::topk_row_kernel<<<dim3(chunks, nrows), tkr::kThreads, tkr::kSmemBytes, st>>>(p1);
    tkr::Args p2 = a;
    p2.cand = nullptr;
    p2.nseg_in = chunks; p2.seg_scores = sc; p2.seg_ids = ids; p2.seg_cnt = cnt; p2.seg_stride = kc;
    tkr::topk_row_kernel<<<dim3(1, nrows), tkr::kThreads, tkr::kSmemBytes, st>>>(p2);
    note_launches(2);
    return cudaGetLastError();
}

}  // namespace csa2

// Top-K (and pool) selection by a cluster of 8 CTAs of 512 threads per query row, or, for few
// rows, of 16 CTAs of 1024 threads (one CTA per SM) when all the rows' clusters fit on the GPU at once.
//
// [A] page "DeepSeek V4.1 Flash深度解析：KV缓存压缩437倍的技术路径", section
// "压缩吸收注意力（二代）": the indexer keeps 2048 blocks per query and the first layer's
// candidate pool; order = score descending, entry index ascending on ties; output ascending.
//
// Each CTA of the cluster owns a contiguous chunk of the row's candidates and keeps their
// order-preserving 32-bit keys in shared memory (read from global once).  Four 8-bit radix
// passes find the exact threshold key: every CTA builds a 256-bin histogram of its chunk,
// the cluster barrier publishes them, and every CTA sums the cluster's histograms through distributed
// shared memory (identical totals -> identical decisions, no broadcast needed).  Compaction:
// each CTA publishes how many of its keys are above / equal to the threshold; the CTA's output
// offset and its share of the "equal" keys (lowest indices first) follow from the lower-ranked
// CTAs' counts.  Inside the CTA each thread owns a consecutive run of keys; two block scans
// (equal keys before the thread, then selections before it) give every thread its output
// offset, so the selected ids come out in ascending order.
#include <cooperative_groups.h>

#include "common.cuh"

namespace csa2 {
namespace tkc {

namespace cg = cooperative_groups;

constexpr int kCluster = 8;                        // the portable cluster size
constexpr int kClusterWide = 16;                   // for few rows: twice the SMs per row
constexpr int kThreads = 512;                      // two CTAs per SM (8-CTA clusters)
constexpr int kThreadsWide = 1024;                 // one CTA per SM (16-CTA clusters, few rows)
constexpr int kMaxChunk = 32768;                   // keys per CTA (128 KB of shared memory)

struct Args {
    const float *scores;        // [rows][score_stride]
    int64_t score_stride;
    const int32_t *cand;        // NULL: row r has cand_len(r) candidates 0..n-1
    int cand_stride;            //  else [rows][cand_stride] entry ids (the Reindex pool)
    const int32_t *n_entries;   // (NULL cand) visible count per row via the helpers below
    const int32_t *q_pos;
    const int32_t *pool_len;    // (cand) candidates per row
    int T;
    int row0;
    int K;
    int32_t *out_idx;
    int32_t *out_cnt;
    int P;
    int32_t *out_pool;
    int32_t *out_pool_len;
};

CSA2_D int64_t row_n(const Args &a, int r) {
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

struct alignas(16) Shared {
    unsigned int hist[2][256];
    alignas(16) unsigned int total[256];
    int counts[2];              // [0] above threshold, [1] equal to it
    int warp_sums[33];
};

static_assert(kThreads % 32 == 0 && kThreadsWide % 32 == 0 && kThreadsWide <= 1024,
              "block scans need whole warps, at most 32");
static_assert(kThreads >= 256 && kThreadsWide >= 256, "one thread per histogram bin");
// Block-wide exclusive sum of per-thread counts in thread order (warp 0 scans one partial per
// warp and zero for lanes beyond the warp count); total = the block's sum.  kT = blockDim.x.
template <int kT>
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
        const int w = lane < kT / 32 ? ws[lane] : 0;
        int wincl = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int x = __shfl_up_sync(0xffffffffu, wincl, o);
            if (lane >= o) wincl += x;
        }
        ws[lane] = wincl - w;
        if (lane == 31) ws[32] = wincl;
    }
    __syncthreads();
    const int res = ws[warp] + incl - v;
    total = ws[32];
    __syncthreads();
    return res;
}

// The digit of the k-th place from the cluster's histogram totals (S.total): every warp reads
// the 256 totals and takes the same decision, so no barrier hands it out.  Updates the prefix,
// mask and the count still needed inside the chosen bin.
CSA2_D void choose_digit(const Shared &S, int shift, uint32_t &prefix, uint32_t &mask, int &remaining) {
    const int lane = threadIdx.x & 31;
    const uint4 t0 = reinterpret_cast<const uint4 *>(S.total)[2 * lane];
    const uint4 t1 = reinterpret_cast<const uint4 *>(S.total)[2 * lane + 1];
    const unsigned int bins[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
    unsigned int local = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) local += bins[i];
    unsigned int suffix = local;                    // sum over lanes >= lane
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned int x = __shfl_down_sync(0xffffffffu, suffix, o);
        if (lane + o < 32) suffix += x;
    }
    const unsigned int above = suffix - local;
    const bool crosses = (int)above < remaining && remaining <= (int)suffix;
    const int owner = __ffs(__ballot_sync(0xffffffffu, crosses)) - 1;
    // the owner lane walks its 8 bins from the top (unrolled: the bins stay in registers)
    int acc = (int)above, dsel = 0;
    bool found = false;
#pragma unroll
    for (int d = 7; d >= 0; --d) {
        if (!found && (d == 0 || acc + (int)bins[d] >= remaining)) {
            dsel = d;
            found = true;
        } else if (!found) {
            acc += (int)bins[d];
        }
    }
    const int take_rem = __shfl_sync(0xffffffffu, remaining - acc, owner);
    const int digit = __shfl_sync(0xffffffffu, lane * 8 + dsel, owner);
    remaining = take_rem;
    prefix |= (uint32_t)digit << shift;
    mask |= 255u << shift;
}

// One selection of the k largest keys of the row (k < n): writes ids ascending to out[0..k).
// kC CTAs per cluster, kT threads per CTA.
template <int kC, int kT>
CSA2_D void select_cluster(cg::cluster_group &cl, Shared &S, const uint32_t *keys, int chunk_len,
                           int64_t chunk_base, const int32_t *ids, int k, int32_t *out) {
    const int rank = (int)cl.block_rank();
    uint32_t prefix = 0u, mask = 0u;
    int remaining = k;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        unsigned int *h = S.hist[pass & 1];
        for (int i = threadIdx.x; i < 256; i += kT) h[i] = 0u;
        __syncthreads();
        // warp-aggregated: lanes with the same bin add once (the top digits of nearby scores
        // collide heavily, which would serialise plain shared-memory atomics)
        for (int base = 0; base < chunk_len; base += kT) {
            const int i = base + threadIdx.x;
            const uint32_t key = i < chunk_len ? keys[i] : 0u;
            const bool in = i < chunk_len && (key & mask) == prefix;
            const uint32_t bin = in ? ((key >> shift) & 255u) : 256u;
            const unsigned peers = __match_any_sync(0xffffffffu, bin);
            if (in && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&h[bin], (unsigned)__popc(peers));
        }
        cl.sync();                                  // every CTA's histogram is complete
        if (threadIdx.x < 256) {                    // bin t summed over the cluster (kC DSMEM loads)
            unsigned int v[kC];
#pragma unroll
            for (int c = 0; c < kC; ++c) v[c] = cl.map_shared_rank(h, c)[threadIdx.x];
            unsigned int sum = 0;
#pragma unroll
            for (int c = 0; c < kC; ++c) sum += v[c];
            S.total[threadIdx.x] = sum;
        }
        __syncthreads();
        choose_digit(S, shift, prefix, mask, remaining);
        // S.total is rewritten only after the next pass's cluster barrier, and the histograms
        // are double-buffered: the next pass writes the other buffer, and the pass after that is
        // separated from these remote reads by the next pass's cluster barrier
    }
    const uint32_t thr = prefix;
    const int need_eq = remaining;
    // ordered compaction of this chunk: thread t owns the consecutive keys [t*per, (t+1)*per).
    // One block scan of (above, equal) counts packed in 16-bit halves gives the thread's place
    // among this CTA's selections; the CTA's place follows from the lower-ranked CTAs' totals.
    const int per = ((chunk_len + kT - 1) / kT) | 1;     // odd: a warp's lanes hit 32 banks
    const int i0 = min(chunk_len, threadIdx.x * per), i1 = min(chunk_len, i0 + per);
    int my_gt = 0, my_eq = 0;
    for (int i = i0; i < i1; ++i) {
        const uint32_t key = keys[i];
        my_gt += key > thr;
        my_eq += key == thr;
    }
    int tot;
    const int pre = block_excl_sum<kT>((my_gt << 16) | my_eq, S.warp_sums, tot);   // counts < 2^16
    const int gt_pre = pre >> 16, eq_pre = pre & 0xFFFF;
    if (threadIdx.x == 0) { S.counts[0] = tot >> 16; S.counts[1] = tot & 0xFFFF; }
    cl.sync();
    int out_base = 0, eq_before = 0;
    for (int c = 0; c < rank; ++c) {
        const int *rc = cl.map_shared_rank(S.counts, c);
        const int g = rc[0], e = rc[1];
        const int take = min(e, max(0, need_eq - eq_before));
        out_base += g + take;
        eq_before += e;
    }
    // equal keys go to the lowest positions first: this thread's share, and the ones before it
    const int quota = max(0, need_eq - eq_before);
    const int take = min(my_eq, max(0, quota - eq_pre));
    int o = out_base + gt_pre + min(eq_pre, quota);
    int eq_seen = 0;
    for (int i = i0; i < i1; ++i) {
        const uint32_t key = keys[i];
        const bool sel = key > thr || (key == thr && eq_seen++ < take);
        if (sel) {
            if (o < k) out[o] = ids ? ids[chunk_base + i] : (int32_t)(chunk_base + i);   // never past k
            ++o;
        }
    }
    cl.sync();                                      // counts may be reused by the next selection
}

// Launched with a cluster of kC CTAs of kT threads per row (launch attribute).
template <int kC, int kT>
__global__ void __launch_bounds__(kT, 1024 / kT) topk_cluster_kernel(Args a) {
    extern __shared__ __align__(16) uint32_t keys[];
    __shared__ Shared S;
    cg::cluster_group cl = cg::this_cluster();
    const int rank = (int)cl.block_rank();
    const int lr = blockIdx.x / kC;
    const int r = a.row0 + lr;
    int64_t n = row_n(a, r);
    if (n > a.score_stride) n = a.score_stride;
    const int chunk = (int)((n + kC - 1) / kC);
    const int64_t cbase = (int64_t)rank * chunk;
    const int clen = (int)max((int64_t)0, min((int64_t)chunk, n - cbase));
    const float *s = a.scores + (int64_t)lr * a.score_stride;
    const int32_t *ids = a.cand ? a.cand + (int64_t)r * a.cand_stride : nullptr;
    for (int i = threadIdx.x; i < clen; i += kT) keys[i] = float_key(s[cbase + i]);
    __syncthreads();
    for (int which = 0; which < 2; ++which) {
        const int k = which == 0 ? a.K : a.P;
        if (k <= 0) continue;                       // uniform across the cluster
        int32_t *out = which == 0 ? a.out_idx + (int64_t)r * a.K : a.out_pool + (int64_t)r * a.P;
        int32_t *cnt = which == 0 ? a.out_cnt : a.out_pool_len;
        const int c = (int)min((int64_t)k, n);
        if (n <= k) {
            for (int i = threadIdx.x; i < clen; i += kT) {
                const int64_t j = cbase + i;
                out[j] = ids ? ids[j] : (int32_t)j;
            }
        } else {
            select_cluster<kC, kT>(cl, S, keys, clen, cbase, ids, k, out);
        }
        // padding: rank 0 writes -1 to out[c..k)
        if (rank == 0) {
            for (int i = c + threadIdx.x; i < k; i += kT) out[i] = -1;
            if (threadIdx.x == 0 && cnt) cnt[r] = c;
        }
    }
}

// Dynamic shared memory of a CTA holding `chunk` keys.
constexpr size_t smem_of(int chunk) { return (size_t)chunk * sizeof(uint32_t); }

}  // namespace tkc

int64_t topk_cluster_max_n() { return (int64_t)tkc::kCluster * tkc::kMaxChunk; }

static SmemLimit g_topk_smem, g_topk_smem_wide, g_topk_smem_wide_full;
// per device: how many 16-CTA clusters can be resident at once (0 unknown, -1 none), for CTAs of
// 512 threads ([0]) and of 1024 threads ([1])
static std::atomic<int> g_topk_wide_slots[2][kMaxDevices];

template <int kC, int kT>
static cudaError_t launch_topk_cluster_n(const tkc::Args &a, int nrows, int64_t max_n, SmemLimit &lim,
                                         cudaStream_t st) {
    const int chunk = (int)((max_n + kC - 1) / kC);
    const size_t smem = tkc::smem_of(chunk > 0 ? chunk : 1);
    cudaError_t e = ensure_smem_limit(lim, tkc::topk_cluster_kernel<kC, kT>, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(nrows * kC));
    cfg.blockDim = dim3(kT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kC;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, tkc::topk_cluster_kernel<kC, kT>, a);
    note_launches(1);
    return e;
}

// How many clusters of 16 CTAs of kT threads with `smem` bytes each can be resident at once on
// the current device (the size is not portable: it needs the opt-in attribute and enough SMs per
// GPC); 0 when none.  Queried once per device and thread count.
template <int kT>
static int topk_wide_slots(size_t smem) {
    constexpr int kC = tkc::kClusterWide;
    const int dev = current_device();
    if (dev < 0) return 0;
    std::atomic<int> &slot = g_topk_wide_slots[kT == tkc::kThreadsWide ? 1 : 0][dev];
    const int known = slot.load(std::memory_order_acquire);
    if (known != 0) return known > 0 ? known : 0;
    std::lock_guard<std::mutex> lock(settings_mutex());
    bool ok = cudaFuncSetAttribute(tkc::topk_cluster_kernel<kC, kT>,
                                   cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess &&
              cudaFuncSetAttribute(tkc::topk_cluster_kernel<kC, kT>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)tkc::smem_of(tkc::kMaxChunk)) == cudaSuccess;
    int clusters = 0;
    if (ok) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(kC);
        cfg.blockDim = dim3(kT);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = kC;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&clusters, tkc::topk_cluster_kernel<kC, kT>, &cfg) !=
            cudaSuccess)
            clusters = 0;
    }
    (void)cudaGetLastError();                   // a refused query leaves no error behind
    slot.store(clusters > 0 ? clusters : -1, std::memory_order_release);
    return clusters > 0 ? clusters : 0;
}

// Selection for rows [row0, row0+nrows) from scores in global memory (max_n <= topk_cluster_max_n()).
cudaError_t launch_topk_cluster(const float *scores, int64_t score_stride, const int32_t *cand,
                                int cand_stride, const int32_t *n_entries, const int32_t *q_pos,
                                const int32_t *pool_len, int T, int row0, int nrows, int K,
                                int32_t *out_idx, int32_t *out_cnt, int P, int32_t *out_pool,
                                int32_t *out_pool_len, int64_t max_n, cudaStream_t st) {
    tkc::Args a;
    a.scores = scores; a.score_stride = score_stride;
    a.cand = cand; a.cand_stride = cand_stride;
    a.n_entries = n_entries; a.q_pos = q_pos; a.pool_len = pool_len; a.T = T;
    a.row0 = row0; a.K = K; a.out_idx = out_idx; a.out_cnt = out_cnt;
    a.P = P; a.out_pool = out_pool; a.out_pool_len = out_pool_len;
    // few rows: clusters of 16 put twice the SMs on each row when the grid still has one CTA per
    // SM (measured: 4 rows x 256K scores 78 -> 59 us; 16 rows x 64K with a 16K pool, two CTAs per
    // SM, was slower at 16 than at 8).  Such a CTA has its SM to itself, so it runs 1024 threads
    // when every row's cluster can be resident at once (4 rows x 147K-254K scores: index + top-K
    // 56.4 -> 52.3 us; 16 rows x 64K with a 16K pool on 8-CTA clusters of 1024 threads: no change).
    const int64_t nsm = device_sm_count();
    const int64_t wide_chunk = (max_n + tkc::kClusterWide - 1) / tkc::kClusterWide;
    if ((int64_t)nrows * tkc::kClusterWide <= nsm && wide_chunk >= 1024) {
        const size_t smem = tkc::smem_of((int)wide_chunk);
        if (nrows <= topk_wide_slots<tkc::kThreadsWide>(smem))
            return launch_topk_cluster_n<tkc::kClusterWide, tkc::kThreadsWide>(a, nrows, max_n,
                                                                               g_topk_smem_wide_full, st);
        if (topk_wide_slots<tkc::kThreads>(smem) > 0)
            return launch_topk_cluster_n<tkc::kClusterWide, tkc::kThreads>(a, nrows, max_n, g_topk_smem_wide, st);
    }
    return launch_topk_cluster_n<tkc::kCluster, tkc::kThreads>(a, nrows, max_n, g_topk_smem, st);
}

}  // namespace csa2

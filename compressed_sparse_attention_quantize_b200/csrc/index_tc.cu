// Indexer scores on the tensor cores (tcgen05.mma kind::mxf4), exact in fp32.
//
// [B] page "DeepSeek V4.1 Flash 如何靠压缩 KV 缓存实现小模型干翻大模型": section "为什么 KV 缓存成了
// 新瓶颈？" (DSA-style indexer), "CSA2：三层压缩一次吃满" (Full / Reindex), "FP4 量化 + Bounded
// Replay" (indexer Q and K in FP4).
//
// I[r, j] = sum_h w_h * relu(q_h . k_j).  The MMA computes, for 128 keys at a time, the raw E2M1
// products of every (head, 16-channel block) pair: B holds the query "block-diagonally" --
// column (h, b) carries head h's codes for block b and zeros elsewhere -- and every block scale
// fed to the MMA is 1.0, so each output is a sum of 16 exact products (multiples of 1/4, at most
// 576): exact in fp32.  The epilogue multiplies by the two E4M3 scales (exact) and adds blocks
// and heads in the fixed order that csa2.h defines (explicitly rounded adds and multiplies), so
// the scores -- and therefore the selected sets -- are bit-identical to any implementation of
// that order (the oracle's is one).
//
// Operands in shared memory, K-major without swizzle: a 32-byte row of FP4 codes is two 16-byte
// planes (elements 0-31 and 32-63), rows 16 bytes apart inside a plane.  D: 128 lanes (keys) x
// N columns (4 per head, N rounded up to 16) fp32 in TMEM.  Each thread keeps the key rows of
// next tiles in flight: for a contiguous key range (Full mode) one thread streams the raw
// 32-byte rows of the next kStages tiles into a shared-memory ring with bulk copies; for a
// gathered pool (Reindex) every thread keeps its key rows of the next kDepth tiles in registers.
// Shared memory is reserved so that TMEM allocation never waits (at most 512 / columns CTAs).
#include "common.cuh"
#include "index_api.cuh"
#include "tc_ptx.cuh"

namespace csa2 {
namespace itc {

constexpr int kTile = 128;
constexpr int kThreads = 128;
constexpr int kMaxN = 4 * CSA2_MAX_INDEX_HEADS;      // 64 columns
constexpr int kDepth = 2;                            // gathered tiles in flight per thread
constexpr int kStages = 4;                           // contiguous tiles in flight per CTA (a 16 KB
                                                     // ring lets 8 CTAs share an SM)
constexpr int kRingBytes = kStages * kTile * 32;     // raw key rows, 32 bytes each

struct Args {
    const uint8_t *q_codes, *q_scales;
    const float *w;
    int H, T;
    const uint8_t *k_codes;
    int64_t k_code_stride;
    const uint8_t *k_scales;
    int64_t k_scale_stride;
    const int64_t *seq_start;
    const int32_t *n_entries;
    const int32_t *q_pos;
    const int32_t *pool;
    const int32_t *pool_len;
    int P_in;
    int row0;
    float *scores;
    int64_t score_stride;
    uint32_t tmem_cols;
    int tiles_per_cta;                 // consecutive 128-key tiles of a row per CTA
};

struct __align__(16) Smem {
    uint8_t a[2 * kTile * 16];         // keys: two 16-byte planes
    uint8_t b[2 * kMaxN * 16];         // block-diagonal query
    float qs[CSA2_MAX_INDEX_HEADS * 4];// query block scales
    float w[CSA2_MAX_INDEX_HEADS];
    uint64_t done, drain;
    uint64_t full[kStages];            // ring stage s holds its tile's key rows
    uint32_t tmem_base;
    int abort_flag;
};

CSA2_D int64_t candidates(const Args &a, int r) {
    if (a.pool) return a.pool_len[r];
    const int b = r / a.T;
    int64_t n = a.n_entries[b];
    if (a.q_pos) {
        const int64_t v = ((int64_t)a.q_pos[r] + 1) / 4;
        n = v < n ? v : n;
        if (n < 0) n = 0;
    }
    return n;
}

// Instruction descriptor, kind::mxf4 (block 32, UE8M0 scales): A, B = E2M1, K-major.
CSA2_HD constexpr uint32_t idesc_mxf4(int M, int N) {
    return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | (1u << 23) | ((uint32_t)(M >> 4) << 24);
}

CSA2_D uint64_t sdesc_noswizzle(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1u << 46;                          // version; layout type 0 = no swizzle
    return d;
}

CSA2_D void mma_mxf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                     uint32_t sfb) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, 0, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa), "r"(sfb)
        : "memory");
}

__global__ void __launch_bounds__(kThreads, 6)
index_score_tc_kernel(Args a) {
    __shared__ Smem S;
    extern __shared__ __align__(128) uint8_t ring[];     // kStages x 128 raw key rows (contiguous mode)
    const int t = threadIdx.x, warp = t >> 5;
    const int r = a.row0 + blockIdx.y;
    const int b = r / a.T;
    const int64_t n = min(candidates(a, r), a.score_stride);
    const int64_t j0 = (int64_t)blockIdx.x * a.tiles_per_cta * kTile;
    if (j0 >= n) return;                                  // uniform per CTA: nothing allocated yet
    const int ntiles = (int)min((int64_t)a.tiles_per_cta, (n - j0 + kTile - 1) / kTile);
    const int H = a.H;
    const int N = ((4 * H + 15) / 16) * 16;
    const uint32_t tmem_cols = a.tmem_cols;
    const uint32_t sf_col = N;

    // ---- setup: query (block-diagonal B), scales, weights, barriers, TMEM ----
    for (int i = t; i < (int)(sizeof(S.b) / 16); i += kThreads)
        reinterpret_cast<uint4 *>(S.b)[i] = make_uint4(0u, 0u, 0u, 0u);
    if (t == 0) {
        ptx::mbar_init(&S.done, 1);
        ptx::mbar_init(&S.drain, 1);
        for (int i = 0; i < kStages; ++i) ptx::mbar_init(&S.full[i], 1);
        S.abort_flag = 0;
        ptx::fence_async_smem();
    }
    if (warp == 0) {
        ptx::tmem_alloc(&S.tmem_base, tmem_cols);
        ptx::tmem_relinquish();
    }
    __syncthreads();
    for (int i = t; i < H * 4; i += kThreads) {
        const int h = i >> 2, blk = i & 3;
        const uint8_t *qc = a.q_codes + ((int64_t)r * H + h) * 32;
        // column n = 4h + blk: block blk's 8 code bytes at byte offset 8*blk of the 32-byte row
        const int plane = blk >> 1, within = (blk & 1) * 8;
        uint8_t *dst = S.b + plane * (kMaxN * 16) + i * 16 + within;
#pragma unroll
        for (int k = 0; k < 8; ++k) dst[k] = qc[8 * blk + k];
        S.qs[i] = e4m3_to_f32(a.q_scales[((int64_t)r * H + h) * 4 + blk]);
    }
    for (int i = t; i < H; i += kThreads) S.w[i] = a.w[(int64_t)r * H + i];
    ptx::fence_async_smem();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    // every block scale the MMA sees is 1.0 (UE8M0 0x7F): the true E4M3 scales are applied below
    {
        uint32_t ones[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) ones[i] = 0x7F7F7F7Fu;
        ptx::tmem_st32(lane_addr + sf_col, ones);
        ptx::tmem_st_wait();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();

    const uint32_t idesc = idesc_mxf4(128, N);
    const uint32_t b_addr = ptx::smem_u32(S.b);
    const uint64_t bdesc = sdesc_noswizzle(b_addr, kMaxN * 16, 128);
    const uint32_t sf = tmem + sf_col;
    volatile int *abort_flag = &S.abort_flag;
    const int64_t sbase = a.seq_start[b];

    const uint64_t adesc = sdesc_noswizzle(ptx::smem_u32(S.a), kTile * 16, 128);

    // One tile: stage this thread's key row in the two 16-byte planes, one MMA, then the
    // fixed-order epilogue.  Returns false when the CTA gives up (collective).
    // k0, k1: this thread's key row (planes 0 and 1), or with `chunked` the 16-byte chunks t and
    // t + 128 of the tile's raw rows (chunk c is plane c % 2 of row c / 2), which keeps both the
    // ring reads and the plane writes free of bank conflicts.
    auto run_tile = [&](int i, const uint4 &k0, const uint4 &k1, bool chunked, uint32_t sc_this,
                        bool valid_this) -> bool {
        if (chunked) {
            uint8_t *plane = S.a + (t & 1) * (kTile * 16);
            *reinterpret_cast<uint4 *>(plane + (t >> 1) * 16) = k0;
            *reinterpret_cast<uint4 *>(plane + (kTile / 2 + (t >> 1)) * 16) = k1;
        } else {
            *reinterpret_cast<uint4 *>(S.a + t * 16) = k0;
            *reinterpret_cast<uint4 *>(S.a + kTile * 16 + t * 16) = k1;
        }
        ptx::fence_async_smem();
        ptx::tc_fence_before();
        __syncthreads();
        if (t == 0) {
            ptx::tc_fence_after();
            mma_mxf4(tmem, adesc, bdesc, idesc, sf, sf);
            ptx::mma_commit(&S.done);
        }
        ptx::mbar_wait(&S.done, i & 1, abort_flag);
        if (__syncthreads_or(*abort_flag != 0)) return false;
        ptx::tc_fence_after();
        float sk[4];
        ptx::e4m3x4_to_f32(sc_this, sk);
        float acc = 0.0f;
        for (int hb = 0; hb * 8 < H; ++hb) {
            uint32_t u[32];
            ptx::tmem_ld32(lane_addr + hb * 32, u);
            ptx::tmem_ld_wait();
#pragma unroll
            for (int hh = 0; hh < 8; ++hh) {
                const int h = hb * 8 + hh;
                if (h < H) {
                    float c[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) c[q] = __fmul_rn(S.qs[h * 4 + q], sk[q]);
                    const float dot = head_block_sum(u + hh * 4, c);
                    const float rl = dot > 0.0f ? dot : 0.0f;
                    acc = __fadd_rn(acc, __fmul_rn(S.w[h], rl));
                }
            }
        }
        if (acc == 0.0f) acc = 0.0f;                     // -0 -> +0
        if (valid_this) a.scores[(int64_t)blockIdx.y * a.score_stride + j0 + (int64_t)i * kTile + t] = acc;
        return true;
    };

    // the four E4M3 block scales of key j (0 past the end)
    auto scale_of = [&](int i) -> uint32_t {
        const int64_t j = j0 + (int64_t)i * kTile + t;
        if (i >= ntiles || j >= n) return 0u;
        const int64_t e = sbase + (a.pool ? (int64_t)a.pool[(int64_t)r * a.P_in + j] : j);
        const uint8_t *ks = a.k_scales + e * a.k_scale_stride;
        if ((a.k_scale_stride & 3) == 0) return __ldg(reinterpret_cast<const uint32_t *>(ks));
        return (uint32_t)__ldg(ks) | ((uint32_t)__ldg(ks + 1) << 8) | ((uint32_t)__ldg(ks + 2) << 16) |
               ((uint32_t)__ldg(ks + 3) << 24);
    };

    bool aborted = false;
    const bool contiguous = a.pool == nullptr && a.k_code_stride == 32;
    if (contiguous) {
        // ---- Full mode: the CTA's keys are consecutive rows; thread 0 keeps kStages tiles of raw
        //      rows in flight with bulk copies (only the rows that exist are copied)
        const uint8_t *src0 = a.k_codes + (sbase + j0) * 32;
        auto issue = [&](int i) {
            const int st = i % kStages;
            const int64_t jt = (int64_t)i * kTile;
            const uint32_t bytes = (uint32_t)min((int64_t)kTile, n - j0 - jt) * 32u;
            ptx::mbar_arrive_expect_tx(&S.full[st], bytes);
            ptx::bulk_load_g2s(ring + st * kTile * 32, src0 + jt * 32, bytes, &S.full[st]);
        };
        int issued = 0;
        if (t == 0)
            for (; issued < kStages && issued < ntiles; ++issued) issue(issued);
        uint32_t s0 = scale_of(0), s1 = scale_of(1), s2 = scale_of(2);
        int i = 0;
        for (; i < ntiles; ++i) {
            const int st = i % kStages;
            ptx::mbar_wait(&S.full[st], (uint32_t)(i / kStages) & 1u, abort_flag);   // a miss aborts below
            const bool valid_this = j0 + (int64_t)i * kTile + t < n;
            // rows past the end were not copied: their codes are stale but finite (E2M1 has no
            // NaN), and their scores are never stored
            const uint4 *stage = reinterpret_cast<const uint4 *>(ring + st * kTile * 32);
            const uint4 k0 = stage[t], k1 = stage[t + kTile];
            const uint32_t sc_this = s0;
            s0 = s1;
            s1 = s2;
            s2 = scale_of(i + 3);
            if (!run_tile(i, k0, k1, true, sc_this, valid_this)) { aborted = true; break; }
            // every thread has read stage st (run_tile synchronised after staging)
            if (t == 0 && issued < ntiles) issue(issued++);
        }
        if (aborted && t == 0) {       // let the copies still in flight land before exiting
            for (int k = i; k < issued; ++k)
                ptx::mbar_wait_drain(&S.full[k % kStages], (uint32_t)(k / kStages) & 1u);
        }
    } else {
        // ---- gathered keys (Reindex pool) or strided rows: kDepth tiles in registers per thread
        auto key_row = [&](int i, uint4 &c0, uint4 &c1, bool &valid) {
            const int64_t j = j0 + (int64_t)i * kTile + t;
            valid = j < n;
            c0 = c1 = make_uint4(0u, 0u, 0u, 0u);
            if (valid) {
                const int64_t e = sbase + (a.pool ? (int64_t)a.pool[(int64_t)r * a.P_in + j] : j);
                const uint4 *kc = reinterpret_cast<const uint4 *>(a.k_codes + e * a.k_code_stride);
                c0 = __ldg(kc);
                c1 = __ldg(kc + 1);
            }
        };
        uint4 c0[kDepth], c1[kDepth];
        uint32_t sc[kDepth];
        bool valid[kDepth];
#pragma unroll
        for (int k = 0; k < kDepth; ++k) {
            key_row(k, c0[k], c1[k], valid[k]);
            sc[k] = scale_of(k);
        }
        for (int i0 = 0; i0 < ntiles && !aborted; i0 += kDepth) {
#pragma unroll
            for (int k = 0; k < kDepth; ++k) {
                const int i = i0 + k;
                if (i >= ntiles) break;
                const uint4 k0 = c0[k], k1 = c1[k];
                const uint32_t sc_this = sc[k];
                const bool valid_this = valid[k];
                if (i + kDepth < ntiles) {
                    key_row(i + kDepth, c0[k], c1[k], valid[k]);
                    sc[k] = scale_of(i + kDepth);
                }
                if (!run_tile(i, k0, k1, false, sc_this, valid_this)) { aborted = true; break; }
            }
        }
    }
    if (aborted && t == 0) {           // drain the tensor pipe before TMEM is released
        ptx::mma_commit(&S.drain);
        ptx::mbar_wait_drain(&S.drain, 0);
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, tmem_cols);
    }
}

}  // namespace itc

static SmemLimit g_index_smem;

// Resident CTAs of the score kernel on the current device for a dynamic shared-memory size:
// the minimum of the TMEM-column limit (per_sm), shared memory (1 KB reserved per CTA) and
// registers (the occupancy query does not account for the TMEM limit).  Cached per device and
// TMEM width (per_sm is 512 / columns: 1, 2, 4, 8 or 16).
static int index_resident_ctas(int per_sm, int dyn) {
    static std::atomic<int> cache[kMaxDevices][5];
    const int dev = current_device();
    int slot = 0;
    while ((1 << slot) < per_sm && slot < 4) ++slot;
    if (dev >= 0) {
        const int v = cache[dev][slot].load(std::memory_order_acquire);
        if (v > 0) return v;
    }
    int nsm = 148, smem_sm = 228 * 1024;
    if (dev >= 0) {
        nsm = device_sm_count();
        cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    }
    cudaFuncAttributes fa;
    int regs = 72;
    size_t stat = sizeof(itc::Smem);
    if (cudaFuncGetAttributes(&fa, itc::index_score_tc_kernel) == cudaSuccess) {
        regs = fa.numRegs > 0 ? fa.numRegs : regs;
        stat = fa.sharedSizeBytes;
    }
    int blocks = per_sm;
    blocks = min(blocks, smem_sm / (int)(stat + (size_t)dyn + 1024));
    blocks = min(blocks, 65536 / (regs * itc::kThreads));
    const int resident = max(blocks, 1) * nsm;
    if (dev >= 0) cache[dev][slot].store(resident, std::memory_order_release);
    return resident;
}

cudaError_t launch_index_score_tc(const IndexLaunch &L, int row0, int nrows, float *scores,
                                  int64_t score_stride, cudaStream_t st) {
    itc::Args a;
    a.q_codes = L.q_codes; a.q_scales = L.q_scales; a.w = L.w;
    a.H = L.H; a.T = L.T;
    a.k_codes = L.k_codes; a.k_code_stride = L.k_code_stride;
    a.k_scales = L.k_scales; a.k_scale_stride = L.k_scale_stride;
    a.seq_start = L.seq_start; a.n_entries = L.n_entries; a.q_pos = L.q_pos;
    const bool reindex = L.mode == CSA2_MODE_REINDEX;
    a.pool = reindex ? L.pool : nullptr;
    a.pool_len = reindex ? L.pool_len : nullptr;
    a.P_in = L.P_in;
    a.row0 = row0;
    a.scores = scores;
    a.score_stride = score_stride;
    // TMEM per CTA: D (N columns) + 32 columns of unit scale factors
    const int N = ((4 * L.H + 15) / 16) * 16;
    uint32_t cols = 32;
    while (cols < (uint32_t)(N + 32)) cols <<= 1;
    a.tmem_cols = cols;
    // reserve shared memory so that at most 512/cols CTAs are resident on an SM
    // (and at least the bulk-copy ring of the contiguous path)
    const int per_sm = 512 / (int)cols;
    const int smem_total = (227 * 1024) / per_sm - 1024;
    const int dyn = max(smem_total - (int)sizeof(itc::Smem), itc::kRingBytes);
    cudaError_t e = ensure_smem_limit(g_index_smem, itc::index_score_tc_kernel, dyn);
    if (e != cudaSuccess) return e;
    const int resident = index_resident_ctas(per_sm, dyn);
    // tiles per CTA: the fewest that fit every row's tiles into one wave of resident CTAs (a
    // partial second wave would cost a whole CTA time); with more rows than resident CTAs, 8
    const int64_t tiles_row = ceil_div(score_stride, (int64_t)itc::kTile);
    const int64_t per_row_ctas = resident / (nrows > 0 ? nrows : 1);
    int64_t tpc = per_row_ctas > 0 ? ceil_div(tiles_row, per_row_ctas) : 8;
    if (tpc < 1) tpc = 1;
    a.tiles_per_cta = (int)tpc;
    const int64_t per_cta = tpc * itc::kTile;
    dim3 grid((unsigned)ceil_div(score_stride, per_cta), (unsigned)nrows);
    itc::index_score_tc_kernel<<<grid, itc::kThreads, dyn, st>>>(a);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace csa2

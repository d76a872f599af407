// Sparse attention on the 5th-generation tensor cores (tcgen05 + TMEM), sm_100a.
//
// [B] page "DeepSeek V4.1 Flash 如何靠压缩 KV 缓存实现小模型干翻大模型", section
// "CSA2：三层压缩一次吃满": every layer keeps its own query and window and attends over the
// selected compressed entries, whose MLA-style latent is shared by the heads (keys = values =
// the 512-wide latent).  Section "FP4 量化 + Bounded Replay": entries are E2M1 with one E4M3
// scale per 16 channels; the window is the last 128 tokens, 8-bit.
//
// One CTA = (query row, group of 64 heads, split of the row's key list: selected entries
// followed by window tokens).  Per tile of 128 keys:
//   S^T[key, head] = V . Q^T   tcgen05.mma kind::f16, M=128 keys, N=64 heads, K=512 channels;
//                              A = V (K-major), B = Q (K-major), fp32 accumulator in TMEM.
//   online softmax             4 warps read S^T from TMEM (one key per thread), log2 domain,
//                              lazy rescale: the running max moves only when a tile's max
//                              exceeds it by more than 2^8.
//   O^T[chan, head] += V^T.P^T four MMAs M=128 channels, N=64 heads, K=128 keys; A = the same
//                              V bytes read as an MN-major operand, B = P^T (MN-major fp16).
//                              P is split as fp16(P) + fp16(P - fp16(P)) and both halves are
//                              accumulated: fp16 rounding of P alone (2^-11) times the x8
//                              outlier channels breaks the 2e-3 max-abs/RMS bound.
// V is dequantised once per tile into fp16 (E2M1 x E4M3 is exact in fp16); the window's
// per-token fp32 scale is applied to the logit and folded into P instead.  Q is converted to
// fp16 with a power-of-two pre-scale so small values keep full precision.
//
// Warp roles (9 warps): 0 = TMEM owner + MMA issuer; 1-8 = workers.  Worker warp w owns TMEM
// sub-partition w%4 (keys 32*(w%4)..+31) and one half: it dequantises channels 256*half..+255
// of its keys and runs the softmax for heads 32*half..+31.  Hand-offs use one mbarrier per
// channel half (every mbarrier wait costs the issuing thread ~140 cycles, measured), so the
// dequantisation of one half overlaps the MMAs on the other; the per-head max is only
// re-reduced when some logit exceeds the running max by 2^8.
// Every wait is bounded: on expiry the CTA records CSA2_ERR_TIMEOUT, drains, frees TMEM and exits.
#include "attn.cuh"
#include "tc_ptx.cuh"

namespace csa2 {

namespace tc {

constexpr int kTile = 128;                 // keys per tile (MMA M)
constexpr int kHeads = 64;                 // heads per CTA (MMA N)
constexpr int kRegions = 8;                // 64-channel blocks of the 512-wide latent
constexpr int kBlocks = 4;                 // 128-channel blocks (P.V MMA M)
constexpr int kQRegion = kHeads * 128;     // 8 KB
constexpr int kVRegion = kTile * 128;      // 16 KB
constexpr int kQBytes = kRegions * kQRegion;         // 64 KB
constexpr int kVBytes = kRegions * kVRegion;         // 128 KB
constexpr int kPBytes = kTile * kHeads * 2;          // 16 KB (one of P_hi, P_lo)
constexpr int kThreads = 288;             // warp 0: MMA issuer; warps 1-8: workers
constexpr int kWorkers = 256;
constexpr int kTmemCols = 512;
constexpr int kLCol = 64;                  // per-key row-sum partials at columns 64..127
// O^T accumulators from column 128.  The first kFolded 128-channel blocks run the P_hi and P_lo
// products as one N=128 MMA (B = [P_hi | P_lo]: the descriptor's leading-byte offset is the
// P_hi -> P_lo distance), so V is read once for both; their accumulators are [O(P_hi) | O(P_lo)]
// (128 columns, added in the epilogue).  The other blocks take both products into one 64-column
// accumulator.  TMEM holds two folded blocks next to S^T and the row sums.
constexpr int kFolded = 2;
CSA2_HD constexpr int o_col(int mb) {
    return mb < kFolded ? 128 + 128 * mb : 128 + 128 * kFolded + 64 * (mb - kFolded);
}
static_assert(o_col(kBlocks - 1) + kHeads <= kTmemCols, "O^T accumulators fit in TMEM");
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr int32_t kNoKey = INT32_MIN;

struct Smem {
    uint64_t v_full[kBlocks];              // 128-channel block mb of the tile is written
    uint64_t v_empty[kBlocks];             // P.V of 128-channel block mb has completed
    uint64_t s_full, p_full, pv_done, drain;
    uint64_t q_full;                       // the bulk copy of Q has landed in the staging area
    uint64_t q_ready;                      // the workers have written the fp16 Q operand
    uint32_t tmem_base;
    int abort_flag;
    int q_exp_max;
    float m_run[kHeads];
    float alpha[kHeads];
};

// Scratch that lives in the P_lo buffer while that buffer is free: the per-head max reduction
// (during a tile's softmax, after the previous tile's P.V has completed and before P_lo is
// rewritten) and the final row-sum reduction.
struct Scratch {
    float red[4][kHeads];
    float inv_l[kHeads];
};

constexpr int kSmemBytes = kQBytes + kVBytes + 2 * kPBytes + (int)sizeof(Smem) + 1024;

// Key x of row r, step 1: the entry number (>= 0), -1 - w for window position w, or kNoKey.
CSA2_D int32_t entry_of(const AttnArgs &a, int r, int x, int x_end, int n_sel) {
    if (x >= x_end) return kNoKey;
    if (x < n_sel) {
        const int32_t e = a.idx[(int64_t)r * a.K + x];
        return e < 0 ? kNoKey : e;
    }
    return -1 - (x - n_sel);
}

// Step 2: where the key's bytes are.
struct KeySrc {
    bool valid, swa;
    const uint8_t *ptr;      // main: 288-byte row; window: 512 E4M3 codes
    float scale;             // window token scale (1 for main entries, 0 if invalid)
};

// An id at or above its sequence's entry count (n_lim) or a window slot outside the window buffer
// breaks the caller contract: the key is skipped and the device error word records
// CSA2_ERR_INVALID_ARG, so nothing is read outside the caller's buffers.
CSA2_D KeySrc source_of(const AttnArgs &a, int r, int b, int64_t seq_start, int64_t n_lim, int32_t e) {
    KeySrc k{false, false, nullptr, 0.0f};
    if (e == kNoKey) return k;
    if (e >= 0 && a.shard_lo) {                   // context shard: global entry -> this shard's row
        const int64_t le = (int64_t)e - a.shard_lo[b];
        if (le < 0 || le >= a.shard_n[b]) return k;
        e = (int32_t)le;
    } else if (e >= n_lim) {
        raise_device_error(CSA2_ERR_INVALID_ARG);
        return k;
    }
    if (e >= 0) {
        k.valid = true;
        k.ptr = a.kv + (seq_start + e) * a.kv_row_stride;
        k.scale = 1.0f;
    } else {
        const int slot = (a.swa_start ? a.swa_start[r] : 0) + (-1 - e);
        if (slot < 0 || slot >= a.swa_cap) {
            raise_device_error(CSA2_ERR_INVALID_ARG);
            return k;
        }
        const int64_t srow = (int64_t)b * a.swa_cap + slot;
        k.valid = true;
        k.swa = true;
        k.ptr = a.swa_codes + srow * kLatent;
        k.scale = a.swa_scale[srow];
    }
    return k;
}

// Transpose-reduce 32 values across a warp: afterwards v[0] of lane L holds the max (or sum)
// over the 32 lanes of element L.  31 shuffles instead of 32 x 5.
template <bool kSum>
CSA2_D void warp_transpose_reduce(float (&v)[32], int lane) {
#pragma unroll
    for (int off = 16, n = 16; off >= 1; off >>= 1, n >>= 1) {
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < n; ++i) {
            const float send = upper ? v[i] : v[i + n];
            const float keep = upper ? v[i + n] : v[i];
            const float got = __shfl_xor_sync(0xffffffffu, send, off);
            v[i] = kSum ? keep + got : fmaxf(keep, got);
        }
    }
}

// swizzled 16-byte chunk c of row `row` inside a 128B-swizzled region
CSA2_D uint32_t sw128_off(int row, int c) {
    return (uint32_t)((row >> 3) * 1024 + (row & 7) * 128 + ((c ^ (row & 7)) << 4));
}

// The bytes of one main-entry key that a worker dequantises: regions 2mb + hsel (mb = 0..3),
// i.e. 32 code bytes and 4 scale bytes per region.  Window keys are read per region instead.
struct RowPart {
    uint4 codes[8];
    uint32_t sc[4];
};

// 32 bytes in one 256-bit load (p 32-byte aligned), read-only path
CSA2_D void ldg_32B(const void *p, uint4 &lo, uint4 &hi) {
    asm volatile("ld.global.nc.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(lo.x), "=r"(lo.y), "=r"(lo.z), "=r"(lo.w), "=r"(hi.x), "=r"(hi.y), "=r"(hi.z), "=r"(hi.w)
                 : "l"(p));
}

// Block mb of prefetch: the 32 code bytes of region 2mb + hsel; with the last block, the row's
// 32 scale bytes in one load (its four words 2mb + hsel are kept: every block of the current
// tile has been dequantised by then).  A tile's rows are requested one block at a time, each
// right after the previous tile's block has been dequantised, so that at most a few KB of
// gathers are in flight per block: a load queue full of gathers holds up every shared-memory
// access of the SM behind it (measured: the MMA issuer's barrier polls and the softmax's P
// stores waited for the gathers).  One scale load per row and half instead of four cuts a tile's
// gather requests from 16 to 10 per row.
CSA2_D void prefetch_block(const KeySrc &src, int hsel, int mb, RowPart &rp) {
    if (src.valid && !src.swa) {
        const uint8_t *p = src.ptr + 32 * (2 * mb + hsel);
        if ((reinterpret_cast<uintptr_t>(p) & 31u) == 0) {
            ldg_32B(p, rp.codes[2 * mb], rp.codes[2 * mb + 1]);
        } else {
            rp.codes[2 * mb] = __ldg(reinterpret_cast<const uint4 *>(p));
            rp.codes[2 * mb + 1] = __ldg(reinterpret_cast<const uint4 *>(p) + 1);
        }
        if (mb == kBlocks - 1) {
            const uint8_t *ps = src.ptr + 256;
            uint4 lo, hi;
            if ((reinterpret_cast<uintptr_t>(ps) & 31u) == 0) {
                ldg_32B(ps, lo, hi);
            } else {
                lo = __ldg(reinterpret_cast<const uint4 *>(ps));
                hi = __ldg(reinterpret_cast<const uint4 *>(ps) + 1);
            }
            rp.sc[0] = hsel ? lo.y : lo.x;
            rp.sc[1] = hsel ? lo.w : lo.z;
            rp.sc[2] = hsel ? hi.y : hi.x;
            rp.sc[3] = hsel ? hi.w : hi.z;
        }
    } else {                                     // always assigned: no stale registers live
        rp.codes[2 * mb] = rp.codes[2 * mb + 1] = make_uint4(0u, 0u, 0u, 0u);
        if (mb == kBlocks - 1) rp.sc[0] = rp.sc[1] = rp.sc[2] = rp.sc[3] = 0u;
    }
}

// Dequantise region rg = 2mb + hsel (64 channels) of one key into 8 fp16 chunks.
CSA2_D void dequant_region(const KeySrc &src, const RowPart &rp, int mb, int rg, uint4 (&out)[8]) {
    if (!src.valid) {
#pragma unroll
        for (int c = 0; c < 8; ++c) out[c] = make_uint4(0u, 0u, 0u, 0u);
    } else if (!src.swa) {
        const uint32_t sw = rp.sc[mb];
        const uint4 c0 = rp.codes[2 * mb], c1 = rp.codes[2 * mb + 1];
        const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        const uint32_t s01 = ptx::e4m3x2_to_f16x2((uint16_t)(sw & 0xFFFFu));
        const uint32_t s23 = ptx::e4m3x2_to_f16x2((uint16_t)(sw >> 16));
        const uint32_t sc[4] = {__byte_perm(s01, 0, 0x1010), __byte_perm(s01, 0, 0x3232),
                                __byte_perm(s23, 0, 0x1010), __byte_perm(s23, 0, 0x3232)};
#pragma unroll
        for (int wi = 0; wi < 8; ++wi) {                 // word wi = channels 8wi..8wi+7
            uint32_t hv[4];
            ptx::e2m1x8_to_f16x8(words[wi], hv);
            const uint32_t sv = sc[wi >> 1];
            out[wi] = make_uint4(ptx::hmul2_u32(hv[0], sv), ptx::hmul2_u32(hv[1], sv),
                                 ptx::hmul2_u32(hv[2], sv), ptx::hmul2_u32(hv[3], sv));
        }
    } else {
        const uint4 *p = reinterpret_cast<const uint4 *>(src.ptr + rg * 64);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 v = __ldg(p + i);                  // 16 codes = channels 16i..16i+15
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            uint32_t hv[8];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                hv[2 * k] = ptx::e4m3x2_to_f16x2((uint16_t)(w[k] & 0xFFFFu));
                hv[2 * k + 1] = ptx::e4m3x2_to_f16x2((uint16_t)(w[k] >> 16));
            }
            out[2 * i] = make_uint4(hv[0], hv[1], hv[2], hv[3]);
            out[2 * i + 1] = make_uint4(hv[4], hv[5], hv[6], hv[7]);
        }
    }
}

// bar.red.or over `threads` threads: a barrier that also tells every thread whether any flag was set.
CSA2_D bool block_any(bool flag, uint32_t barrier_id, uint32_t threads) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)flag), "r"(barrier_id), "r"(threads)
        : "memory");
    return r != 0;
}

// The MMA issuer (one thread).  Every MMA sequence is straight-line code: an mbarrier wait or any
// other memory instruction between two MMAs leaves the tensor pipe idle for a few hundred cycles
// (measured), so each tile has five waits: the four 128-channel blocks of V, then P.
// Kept out of line so that its few live values keep registers of their own.
__device__ __noinline__ void issue_mmas(uint32_t tmem, uint8_t *sQ, uint8_t *sV, uint8_t *sP, uint8_t *sPlo,
                                        Smem &S, int ntiles, volatile int *abort_flag) {
    constexpr uint32_t idesc_s = ptx::idesc_f16_f32(128, kHeads, false, false);
    constexpr uint32_t idesc_pv = ptx::idesc_f16_f32(128, kHeads, true, true);
    constexpr uint32_t idesc_pv2 = ptx::idesc_f16_f32(128, 2 * kHeads, true, true);
    // S^T = V . Q^T: A = V (K-major), B = Q (K-major); K step = 32 bytes, region = 64 channels
    const uint64_t s_a0 = ptx::sdesc_sw128(ptx::smem_u32(sV), 16, 1024);
    const uint64_t s_b0 = ptx::sdesc_sw128(ptx::smem_u32(sQ), 16, 1024);
    // O^T += V^T . P^T: A = V read MN-major (64 channels per 128-byte row, next 64 channels one
    // region further), B = P^T (MN-major, 64 heads per row); K step = 16 keys = 2048 bytes
    const uint64_t pv_a0 = ptx::sdesc_sw128(ptx::smem_u32(sV), kVRegion, 1024);
    const uint64_t pv_b0 = ptx::sdesc_sw128(ptx::smem_u32(sP), kPBytes, 1024);
    const uint64_t pvlo_b0 = ptx::sdesc_sw128(ptx::smem_u32(sPlo), kPBytes, 1024);
    for (int j = 0; j < ntiles; ++j) {
        const uint32_t ph = j & 1;
        // S(j) is issued after P.V(j-1), whose P the softmax warps released before p_full(j-1),
        // and s_full(j) completes only after P.V(j-1) has: no separate S-buffer hand-off.
        if (j == 0 && !ptx::mbar_wait(&S.q_ready, 0, abort_flag)) goto done;      // the fp16 Q operand
#pragma unroll
        for (int mb = 0; mb < kBlocks; ++mb) {
            if (!ptx::mbar_wait(&S.v_full[mb], ph, abort_flag)) goto done;
#pragma unroll
            for (int rl = 0; rl < 2; ++rl)
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int rg = mb * 2 + rl;
                    ptx::mma_f16_ss(tmem, s_a0 + (uint64_t)(rg * (kVRegion >> 4) + k * 2),
                                    s_b0 + (uint64_t)(rg * (kQRegion >> 4) + k * 2), idesc_s, (rg | k) != 0);
                }
        }
        ptx::mma_commit(&S.s_full);
        if (!ptx::mbar_wait(&S.p_full, ph, abort_flag)) break;
        ptx::tc_fence_after();
        // per 128-channel block: fp16(P) and P - fp16(P) (P exact to ~2^-22), then the block's V
        // bytes are released to the dequantisers.  Folded blocks: one N=128 MMA per key step into
        // [O(P_hi) | O(P_lo)]; the others: the two halves one after the other into one accumulator.
#pragma unroll
        for (int mb = 0; mb < kBlocks; ++mb) {
            const uint64_t a_mb = pv_a0 + (uint64_t)(mb * ((2 * kVRegion) >> 4));
            if (mb < kFolded) {
#pragma unroll
                for (int kk = 0; kk < kTile / 16; ++kk)
                    ptx::mma_f16_ss(tmem + o_col(mb), a_mb + (uint64_t)(kk * (2048 >> 4)),
                                    pv_b0 + (uint64_t)(kk * (2048 >> 4)), idesc_pv2, (j > 0 || kk > 0) ? 1u : 0u);
            } else {
#pragma unroll
                for (int kk = 0; kk < kTile / 16; ++kk)
                    ptx::mma_f16_ss(tmem + o_col(mb), a_mb + (uint64_t)(kk * (2048 >> 4)),
                                    pv_b0 + (uint64_t)(kk * (2048 >> 4)), idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < kTile / 16; ++kk)
                    ptx::mma_f16_ss(tmem + o_col(mb), a_mb + (uint64_t)(kk * (2048 >> 4)),
                                    pvlo_b0 + (uint64_t)(kk * (2048 >> 4)), idesc_pv, 1u);
            }
            ptx::mma_commit(&S.v_empty[mb]);
        }
        ptx::mma_commit(&S.pv_done);
    }
done:
    // every issued MMA must have completed before TMEM is released (also after an abort)
    ptx::mma_commit(&S.drain);
    ptx::mbar_wait_drain(&S.drain, 0);
}

__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(AttnArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *sQ = base;
    uint8_t *sV = base + kQBytes;
    uint8_t *sP = sV + kVBytes;                     // P_hi
    uint8_t *sPlo = sP + kPBytes;                   // P_lo
    Smem &S = *reinterpret_cast<Smem *>(sPlo + kPBytes);
    Scratch &X = *reinterpret_cast<Scratch *>(sPlo);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = blockIdx.x;                       // query row
    const int hg = blockIdx.y;                      // head group
    const int split = blockIdx.z;
    const int b = r / a.T;
    const int h0 = hg * kHeads;

    // counts outside [0, K] and window lengths outside [0, CSA2_SWA_WINDOW] break the caller
    // contract: they are clamped and the device error word records CSA2_ERR_SHAPE
    int n_sel = a.cnt ? a.cnt[r] : a.K;
    int wlen = a.swa_len[r];
    if (n_sel < 0 || n_sel > a.K || wlen < 0 || wlen > CSA2_SWA_WINDOW) {
        if (threadIdx.x == 0) raise_device_error(CSA2_ERR_SHAPE);
        n_sel = min(max(n_sel, 0), a.K);
        wlen = min(max(wlen, 0), CSA2_SWA_WINDOW);
    }
    const int total = n_sel + wlen;
    const int x_begin = split * a.keys_per_split;
    const int x_end = min(total, x_begin + a.keys_per_split);
    const int ntiles = x_end > x_begin ? (x_end - x_begin + kTile - 1) / kTile : 0;

    // worker roles: key t = sub*32 + lane (TMEM sub-partition = warp % 4); hsel picks the
    // channel regions 2mb + hsel it dequantises and the heads 32*hsel..+31 of its softmax
    const int sub = warp & 3;
    const int hsel = (warp - 1) >> 2;
    const int t = sub * 32 + lane;
    const int64_t seq_start = a.seq_start[b];
    const int64_t n_lim = a.n_entries ? (int64_t)a.n_entries[b] : INT64_MAX;
    // the first tile's rows are requested before anything else
    KeySrc src{false, false, nullptr, 0.0f};
    RowPart rp;
    if (warp > 0) {
        src = source_of(a, r, b, seq_start, n_lim, entry_of(a, r, x_begin + t, x_end, n_sel));
#pragma unroll
        for (int mb = 0; mb < kBlocks; ++mb) prefetch_block(src, hsel, mb, rp);
    }

    // ---------------- setup ----------------
    if (threadIdx.x == 0) {
        for (int i = 0; i < kBlocks; ++i) ptx::mbar_init(&S.v_full[i], kWorkers);
        for (int i = 0; i < kBlocks; ++i) ptx::mbar_init(&S.v_empty[i], 1);
        ptx::mbar_init(&S.s_full, 1);
        ptx::mbar_init(&S.p_full, kWorkers);
        ptx::mbar_init(&S.pv_done, 1);
        ptx::mbar_init(&S.drain, 1);
        ptx::mbar_init(&S.q_full, 1);
        ptx::mbar_init(&S.q_ready, kWorkers);
        S.abort_flag = 0;
        S.q_exp_max = 0;
        ptx::fence_async_smem();
    }
    if (threadIdx.x < kHeads) S.m_run[threadIdx.x] = -INFINITY;
    if (warp == 0) {
        ptx::tmem_alloc(&S.tmem_base, kTmemCols);
        ptx::tmem_relinquish();
    }
    // Q arrives by bulk copy (hcount heads x 1 KB, contiguous) into the upper half of the V buffer,
    // which the first tile's dequantisation writes last; the workers turn it into the swizzled fp16
    // operand between the first tile's channel blocks 1 and 2 (stage_q below).
    const uint16_t *qrow = a.q + ((int64_t)r * a.H + h0) * kLatent;
    const int hcount = min(kHeads, a.H - h0);
    uint8_t *sQstage = sV + 4 * kVRegion;                 // V regions 4..7 (64 KB)
    if (threadIdx.x == 0 && ntiles > 0) {
        const uint32_t bytes = (uint32_t)hcount * kLatent * 2;
        ptx::mbar_arrive_expect_tx(&S.q_full, bytes);
        for (uint32_t off = 0; off < bytes; off += 16384u)
            ptx::bulk_load_g2s(sQstage + off, reinterpret_cast<const uint8_t *>(qrow) + off,
                               min(16384u, bytes - off), &S.q_full);
    }
    ptx::fence_async_smem();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    volatile int *abort_flag = &S.abort_flag;

    if (warp == 0) {
        // ================= MMA issuer (lane 0 alone) =================
        if (lane == 0) issue_mmas(tmem, sQ, sV, sP, sPlo, S, ntiles, abort_flag);
        __syncwarp();
    } else {
        // ================= workers =================
        const int half = hsel;
        const int wt = threadIdx.x - 32;                 // 0..255
        const uint32_t lane_addr = tmem + ((uint32_t)(sub * 32) << 16);
        // A wait that fails (abort or timeout) only marks `bad`; every worker keeps taking the
        // same barriers, and the decision to stop is collective (bar.red.or) once per tile.
        bool bad = false, aborted = false;
        // Q from the staging area into the swizzled fp16 operand (workers only, once, between the
        // first tile's channel blocks 1 and 2): the largest bf16 exponent of the head group picks
        // a power-of-two pre-scale so that the fp16 copy keeps full precision for small values;
        // heads past the last are zero.  Returns that shift.
        auto stage_q = [&]() -> int {
            constexpr int kChunksPer = kHeads * (kLatent / 8) / kWorkers;    // 16-byte chunks per worker
            if (!ptx::mbar_wait(&S.q_full, 0, abort_flag)) bad = true;
            int emax = 0;
#pragma unroll 4
            for (int k = 0; k < kChunksPer; ++k) {
                const int i = wt + k * kWorkers;
                if ((i >> 6) < hcount) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(sQstage + i * 16);
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        emax = max(emax, (int)((w[e] >> 7) & 0xFFu));
                        emax = max(emax, (int)((w[e] >> 23) & 0xFFu));
                    }
                }
            }
            emax = __reduce_max_sync(0xffffffffu, emax);
            if (lane == 0) atomicMax(&S.q_exp_max, emax);
            ptx::named_barrier(1, kWorkers);
            // the largest |q| lands in [2^13, 2^14): far from fp16 overflow, far above its subnormals
            const int qs = S.q_exp_max == 0 ? 0 : (13 - (S.q_exp_max - 127));
            const float qmul = exp2f((float)qs);
#pragma unroll 4
            for (int k = 0; k < kChunksPer; ++k) {
                const int i = wt + k * kWorkers;
                const int h = i >> 6, c8 = i & 63;
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (h < hcount) v = *reinterpret_cast<const uint4 *>(sQstage + i * 16);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                uint32_t packed[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const __half2 hh = __floats2half2_rn(__uint_as_float(w[e] << 16) * qmul,
                                                         __uint_as_float(w[e] & 0xFFFF0000u) * qmul);
                    packed[e] = *reinterpret_cast<const uint32_t *>(&hh);
                }
                *reinterpret_cast<uint4 *>(sQ + (c8 >> 3) * kQRegion + sw128_off(h, c8 & 7)) =
                    make_uint4(packed[0], packed[1], packed[2], packed[3]);
            }
            ptx::fence_async_smem();
            ptx::mbar_arrive(&S.q_ready);
            ptx::named_barrier(1, kWorkers);             // every worker is done with the staging area
            return qs;
        };
        float qk_scale = 0.0f;
        // this key's share of the row sums lives in TMEM (lane = key, 32 columns per half)
        const uint32_t l_addr = lane_addr + kLCol + half * 32;
        {
            uint32_t zero[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) zero[i] = 0u;
            ptx::tmem_st32(l_addr, zero);
            ptx::tmem_st_wait();
        }
        // the entry number of the next tile is read one tile ahead of its use
        int32_t e_next = ntiles > 1 ? entry_of(a, r, x_begin + kTile + t, x_end, n_sel) : kNoKey;
        for (int j = 0; j < ntiles; ++j) {
            const uint32_t ph = j & 1;
            const KeySrc src_next = source_of(a, r, b, seq_start, n_lim, e_next);
            e_next = (j + 2 < ntiles) ? entry_of(a, r, x_begin + (j + 2) * kTile + t, x_end, n_sel) : kNoKey;
            // ---- dequantise regions 2mb + hsel of key t; block mb is free once P.V(j-1) has
            //      finished with it
#pragma unroll
            for (int mb = 0; mb < kBlocks; ++mb) {
                if (j == 0 && mb == 2)                   // Q's staging area is blocks 2 and 3
                    qk_scale = a.softmax_scale * 1.4426950408889634f * exp2f((float)-stage_q());
                if (j > 0 && !ptx::mbar_wait(&S.v_empty[mb], ph ^ 1, abort_flag)) bad = true;
                const int rg = 2 * mb + hsel;
                uint4 out[8];
                dequant_region(src, rp, mb, rg, out);
                uint8_t *dst = sV + rg * kVRegion;
#pragma unroll
                for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4 *>(dst + sw128_off(t, c)) = out[c];
                ptx::fence_async_smem();
                ptx::mbar_arrive(&S.v_full[mb]);
                // block mb of the next tile into the registers just consumed
                if (j + 1 < ntiles) prefetch_block(src_next, hsel, mb, rp);
            }
            const bool cur_valid = src.valid;
            const float cur_scale = src.scale;
            src = src_next;
            // ---- softmax over this thread's key for heads 32*half .. 32*half+31
            if (!ptx::mbar_wait(&S.s_full, ph, abort_flag)) bad = true;
            ptx::tc_fence_after();
            const float zs = qk_scale * cur_scale;
            const uint32_t s_addr = lane_addr + half * 32;
            bool over = false;
            {
                uint32_t u[2][16];
                ptx::tmem_ld16(s_addr, u[0]);
                ptx::tmem_ld16(s_addr + 16, u[1]);
                ptx::tmem_ld_wait();
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float zi = cur_valid ? __uint_as_float(u[hh][i]) * zs : -INFINITY;
                        over |= zi > S.m_run[half * 32 + hh * 16 + i] + kRescaleThreshold;
                    }
            }
            // the running max moves only when some logit exceeds it by more than 2^8.  The max
            // scratch lives in P_lo, free here: s_full(j) completed after P.V(j-1).  One barrier
            // decides both whether to stop (a failed wait anywhere) and whether the max moves;
            // a second one separates the two only when either happened.
            bool move = false;
            if (block_any(over || bad || *abort_flag != 0, 1, kWorkers)) {
                if (block_any(bad || *abort_flag != 0, 1, kWorkers)) { aborted = true; break; }
                move = true;
            }
            bool rescale = false;
            if (move) {
                float v[32];
                {
                    uint32_t u[32];
                    ptx::tmem_ld32(s_addr, u);
                    ptx::tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = cur_valid ? __uint_as_float(u[i]) * zs : -INFINITY;
                }
                warp_transpose_reduce<false>(v, lane);
                X.red[sub][half * 32 + lane] = v[0];
                ptx::named_barrier(1, kWorkers);
                bool moved_here = false;
                if (wt < kHeads) {
                    const float tmax = fmaxf(fmaxf(X.red[0][wt], X.red[1][wt]), fmaxf(X.red[2][wt], X.red[3][wt]));
                    const float mo = S.m_run[wt];
                    float al = 1.0f;
                    if (tmax > mo + kRescaleThreshold) {
                        S.m_run[wt] = tmax;
                        al = (mo == -INFINITY) ? 0.0f : ptx::ex2(mo - tmax);
                        moved_here = j > 0 && mo != -INFINITY;
                    }
                    S.alpha[wt] = al;
                }
                // barrier for the m_run / alpha writes, and whether any accumulated head moved
                rescale = block_any(moved_here, 1, kWorkers);
            }
            // per 16 heads: probabilities (log2 domain), row sums (per key in TMEM, reduced over
            // the keys once at the end), and the P^T line of key t: fp16 high halves to P_hi, low
            // halves (P - fp16(P)) to P_lo.  P.V(j-1) finished before s_full(j), and the max
            // scratch in P_lo was last read before the barrier above.
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                float z[16];
                {
                    uint32_t u[16];
                    ptx::tmem_ld16(s_addr + hh * 16, u);
                    ptx::tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float m = S.m_run[half * 32 + hh * 16 + i];
                        z[i] = (m == -INFINITY || !cur_valid) ? 0.0f : ptx::ex2(__uint_as_float(u[i]) * zs - m);
                    }
                }
                {
                    uint32_t u[16];
                    ptx::tmem_ld16(l_addr + hh * 16, u);
                    ptx::tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float lp = __uint_as_float(u[i]);
                        u[i] = __float_as_uint((move ? lp * S.alpha[half * 32 + hh * 16 + i] : lp) + z[i]);
                    }
                    ptx::tmem_st16(l_addr + hh * 16, u);
                }
#pragma unroll
                for (int c2 = 0; c2 < 2; ++c2) {
                    uint32_t hi4[4], lo4[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int i = 8 * c2 + 2 * k;
                        const float q0 = z[i] * cur_scale, q1 = z[i + 1] * cur_scale;
                        const __half2 hp = __floats2half2_rn(q0, q1);
                        const float2 back = __half22float2(hp);
                        const __half2 lp = __floats2half2_rn(q0 - back.x, q1 - back.y);
                        hi4[k] = *reinterpret_cast<const uint32_t *>(&hp);
                        lo4[k] = *reinterpret_cast<const uint32_t *>(&lp);
                    }
                    const int c = hh * 2 + c2;
                    *reinterpret_cast<uint4 *>(sP + sw128_off(t, half * 4 + c)) = make_uint4(hi4[0], hi4[1], hi4[2], hi4[3]);
                    *reinterpret_cast<uint4 *>(sPlo + sw128_off(t, half * 4 + c)) = make_uint4(lo4[0], lo4[1], lo4[2], lo4[3]);
                }
            }
            // O^T rescale for heads whose running max moved (columns of this half)
            if (rescale) {
                float al[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) al[i] = S.alpha[half * 32 + i];
#pragma unroll 1
                for (int acc = 0; acc < kBlocks + kFolded; ++acc) {      // every accumulator, lo halves last
                    uint32_t u[32];
                    const int mb = acc < kBlocks ? acc : acc - kBlocks;
                    const uint32_t addr = lane_addr + o_col(mb) + (acc < kBlocks ? 0 : kHeads) + half * 32;
                    ptx::tmem_ld32(addr, u);
                    ptx::tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * al[i]);
                    ptx::tmem_st32(addr, u);
                }
            }
            ptx::tmem_st_wait();
            ptx::fence_async_smem();
            ptx::tc_fence_before();
            ptx::mbar_arrive(&S.p_full);
        }
        // ---------------- epilogue ----------------
        if (!aborted && ntiles > 0 && !ptx::mbar_wait(&S.pv_done, (ntiles - 1) & 1, abort_flag)) bad = true;
        aborted = block_any(aborted || bad || *abort_flag != 0, 1, kWorkers);
        ptx::tc_fence_after();
        // row sums: reduce the per-key partials over this warp's 32 keys, then over the 4
        // sub-partitions
        {
            float v[32];
            {
                uint32_t u[32];
                ptx::tmem_ld32(l_addr, u);
                ptx::tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(u[i]);
            }
            warp_transpose_reduce<true>(v, lane);
            if (!aborted) X.red[sub][half * 32 + lane] = v[0];
        }
        ptx::named_barrier(1, kWorkers);
        if (!aborted) {
            // The result goes through shared memory (the Q and V buffers are free: every MMA has
            // completed) and leaves with bulk stores: a split's partial [m(64) | l(64) | O(64 x 512)]
            // fp32, or the single split's normalised output rows (heads h0 .. h0 + hcount - 1 of
            // row r are contiguous).  One worker issues the stores and waits for them.
            const bool single = a.splits == 1;
            float *stg = reinterpret_cast<float *>(sQ);
            if (wt < kHeads) {
                const float l = ntiles > 0 ? X.red[0][wt] + X.red[1][wt] + X.red[2][wt] + X.red[3][wt] : 0.0f;
                X.inv_l[wt] = l > 0.0f ? 1.0f / l : 0.0f;       // 1/l for the single-split output
                if (!single) {
                    stg[wt] = ntiles > 0 ? S.m_run[wt] : -INFINITY;
                    stg[kHeads + wt] = l;
                } else if (a.lse && h0 + wt < a.H) {
                    a.lse[(int64_t)r * a.H + h0 + wt] =
                        (l > 0.0f) ? (S.m_run[wt] + log2f(l)) * 0.6931471805599453f : -INFINITY;
                }
            }
            ptx::named_barrier(1, kWorkers);
            const bool bf16_out = single && a.out_dtype == CSA2_DTYPE_BF16;
#pragma unroll 1
            for (int mb = 0; mb < kBlocks; ++mb) {
                const int c = mb * 128 + t;               // this thread's channel
                uint32_t u[32];
                if (ntiles > 0) {
                    ptx::tmem_ld32(lane_addr + o_col(mb) + half * 32, u);
                    if (mb < kFolded) {                   // add the P_lo accumulator
                        uint32_t v[32];
                        ptx::tmem_ld32(lane_addr + o_col(mb) + kHeads + half * 32, v);
                        ptx::tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) + __uint_as_float(v[i]));
                    }
                    ptx::tmem_ld_wait();
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) u[i] = 0u;
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int h = half * 32 + i;
                    const float o = __uint_as_float(u[i]);
                    if (!single)
                        stg[2 * kHeads + h * kLatent + c] = o;
                    else if (!bf16_out)
                        stg[h * kLatent + c] = o * X.inv_l[h];
                    else
                        reinterpret_cast<__nv_bfloat16 *>(stg)[h * kLatent + c] = __float2bfloat16_rn(o * X.inv_l[h]);
                }
            }
            ptx::fence_async_smem();
            ptx::named_barrier(1, kWorkers);
            if (wt == 0) {
                uint8_t *dst;
                uint32_t bytes;
                if (!single) {
                    const int64_t part_idx = ((int64_t)r * a.hgroups + hg) * a.splits + split;
                    dst = reinterpret_cast<uint8_t *>(a.partials + part_idx * kPartialFloats);
                    bytes = (uint32_t)(kPartialFloats * sizeof(float));
                } else {
                    const int es = bf16_out ? 2 : 4;
                    dst = reinterpret_cast<uint8_t *>(a.out) + ((int64_t)r * a.H + h0) * kLatent * es;
                    bytes = (uint32_t)(hcount * kLatent * es);
                }
                const uint8_t *src8 = reinterpret_cast<const uint8_t *>(stg);
                for (uint32_t off = 0; off < bytes; off += 16384u)
                    ptx::bulk_store_s2g(dst + off, src8 + off, min(16384u, bytes - off));
                ptx::bulk_commit();
                ptx::bulk_wait_all();
            }
        }
    }

    // ---------------- teardown ----------------
    // the bulk copy of Q has landed before the CTA exits (already so unless the CTA gave up early)
    if (threadIdx.x == 0 && ntiles > 0) ptx::mbar_wait_drain(&S.q_full, 0);
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

// Merge split partials (log2-domain maxima): one CTA of 128 threads per (row, head).  Warp 0
// turns the splits' (m, l) into weights exp2(m - M) (one split per lane, up to 64 splits), then
// every thread adds its 4 channels of the splits in split order with independent loads.
constexpr int kMaxMergeSplits = 64;
static_assert((CSA2_MAX_TOPK + CSA2_SWA_WINDOW + kTile - 1) / kTile <= kMaxMergeSplits, "splits <= tiles");

__global__ void __launch_bounds__(128) attn_tc_merge_kernel(AttnArgs a) {
    __shared__ float fw[kMaxMergeSplits];
    __shared__ float inv_total;
    const int r = blockIdx.x, h = blockIdx.y;
    const int hg = h / kHeads, hl = h % kHeads;
    const float *base = a.partials + ((int64_t)r * a.hgroups + hg) * a.splits * kPartialFloats;
    const int ns = min(a.splits, kMaxMergeSplits);
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        float m[2], l[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int sidx = lane + 32 * k;
            m[k] = sidx < ns ? base[sidx * kPartialFloats + hl] : -INFINITY;
            l[k] = sidx < ns ? base[sidx * kPartialFloats + kHeads + hl] : 0.0f;
        }
        float M = fmaxf(m[0], m[1]);
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        float f[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) f[k] = (l[k] > 0.0f) ? exp2f(m[k] - M) : 0.0f;
        // L in split order: gather the terms to lane 0 order-preservingly through shared memory
#pragma unroll
        for (int k = 0; k < 2; ++k)
            if (lane + 32 * k < ns) fw[lane + 32 * k] = f[k];
        __syncwarp();
        if (lane == 0) {
            float L = 0.0f;
            for (int sidx = 0; sidx < ns; ++sidx) {
                const float ls = base[sidx * kPartialFloats + kHeads + hl];
                if (ls > 0.0f) L += ls * fw[sidx];
            }
            inv_total = L > 0.0f ? 1.0f / L : 0.0f;
            if (a.lse) a.lse[(int64_t)r * a.H + h] = L > 0.0f ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
        }
    }
    __syncthreads();
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const float *o = base + 2 * kHeads + hl * kLatent + threadIdx.x * 4;
    int sidx = 0;
    for (; sidx + 4 <= ns; sidx += 4) {
        float4 v[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) v[k] = *reinterpret_cast<const float4 *>(o + (int64_t)(sidx + k) * kPartialFloats);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float f = fw[sidx + k];
            if (f != 0.0f) {
                acc[0] += v[k].x * f; acc[1] += v[k].y * f; acc[2] += v[k].z * f; acc[3] += v[k].w * f;
            }
        }
    }
    for (; sidx < ns; ++sidx) {
        const float f = fw[sidx];
        if (f != 0.0f) {
            const float4 v = *reinterpret_cast<const float4 *>(o + (int64_t)sidx * kPartialFloats);
            acc[0] += v.x * f; acc[1] += v.y * f; acc[2] += v.z * f; acc[3] += v.w * f;
        }
    }
    const float inv = inv_total;
    const int64_t oi = ((int64_t)r * a.H + h) * kLatent + threadIdx.x * 4;
    if (a.out_dtype == CSA2_DTYPE_F32) {
        *reinterpret_cast<float4 *>(reinterpret_cast<float *>(a.out) + oi) =
            make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    } else {
        __nv_bfloat162 *o2 = reinterpret_cast<__nv_bfloat162 *>(reinterpret_cast<__nv_bfloat16 *>(a.out) + oi);
        o2[0] = __floats2bfloat162_rn(acc[0] * inv, acc[1] * inv);
        o2[1] = __floats2bfloat162_rn(acc[2] * inv, acc[3] * inv);
    }
}

}  // namespace tc

// ------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------
static SmemLimit g_attn_smem;

size_t attn_plan_workspace(int rows, int hgroups, int splits) {
    if (splits <= 1) return 256;
    return (size_t)rows * hgroups * splits * kPartialFloats * sizeof(float) + 256;
}

// Split plan (one CTA per SM).  Each CTA costs a fixed part (Q staging, first loads, epilogue:
// about 1.8 tile times, measured) plus its tiles; splits add merge work (about 0.009 tile times
// per row and split, plus the merge launch).  The remainder split is the slowest-varying grid
// index, so its short CTAs are the ones that wait for an SM when the grid exceeds the SMs.
// Pick the tiles per split with the smallest estimated finish time among the plans whose
// partials fit in max_ws bytes.
void attn_plan(int rows, int H, int K, int &hgroups, int &splits, int &keys_per_split, size_t max_ws) {
    hgroups = (H + tc::kHeads - 1) / tc::kHeads;
    const int max_keys = K + CSA2_SWA_WINDOW;
    const int tiles = (max_keys + tc::kTile - 1) / tc::kTile;
    const int per_split = rows * hgroups;                     // CTAs of one split index
    const int nsm = device_sm_count();
    const double fixed = 1.8, merge_per = 0.009, merge_launch = 0.3;
    double best = 1e30;
    int best_tp = tiles;
    for (int tp = 1; tp <= tiles; ++tp) {
        const int sp = (tiles + tp - 1) / tp;
        if (attn_plan_workspace(rows, hgroups, sp) > max_ws) continue;
        const int last = tiles - (sp - 1) * tp;
        const long long ctas = (long long)per_split * sp;
        double t;
        if (ctas <= nsm) {
            t = fixed + tp;
        } else if (ctas - nsm <= per_split) {                 // only remainder CTAs wait
            t = fixed + tp;
            const double second = 2.0 * (fixed + last);
            if (second > t) t = second;
        } else {
            t = (double)((ctas + nsm - 1) / nsm) * (fixed + tp);
        }
        if (sp > 1) t += merge_launch + merge_per * (double)per_split * sp;
        if (t < best - 1e-9) { best = t; best_tp = tp; }
    }
    splits = (tiles + best_tp - 1) / best_tp;
    keys_per_split = best_tp * tc::kTile;
}

size_t attn_workspace_bytes(int rows, int H, int K) {
    int hg, sp, kps;
    attn_plan(rows, H, K, hg, sp, kps);
    return attn_plan_workspace(rows, hg, sp);
}

// The attention kernel with the plan in `a`; the split merge (splits > 1) goes to `side` after
// `attn_done` when a side stream is given, else it follows on `st`.
static cudaError_t launch_with_plan(const AttnArgs &a, cudaStream_t st, cudaStream_t side, cudaEvent_t attn_done,
                                   bool *merged) {
    *merged = false;
    cudaError_t e = ensure_smem_limit(g_attn_smem, tc::attn_tc_kernel, tc::kSmemBytes);
    if (e != cudaSuccess) return e;
    dim3 grid(a.rows, a.hgroups, a.splits);
    tc::attn_tc_kernel<<<grid, tc::kThreads, tc::kSmemBytes, st>>>(a);
    int n = 1;
    if (a.splits > 1) {
        cudaStream_t ms = st;
        if (side) {
            e = cudaEventRecord(attn_done, st);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(side, attn_done, 0);
            if (e != cudaSuccess) return e;
            ms = side;
            *merged = true;
        }
        tc::attn_tc_merge_kernel<<<dim3(a.rows, a.H), 128, 0, ms>>>(a);
        ++n;
    }
    note_launches(n);
    return cudaGetLastError();
}

cudaError_t launch_attn_planned(const AttnArgs &a, cudaStream_t st) {
    bool merged;
    return launch_with_plan(a, st, nullptr, nullptr, &merged);
}

cudaError_t launch_attn(AttnArgs a, cudaStream_t st) {
    attn_plan(a.rows, a.H, a.K, a.hgroups, a.splits, a.keys_per_split);
    bool merged;
    return launch_with_plan(a, st, nullptr, nullptr, &merged);
}

cudaError_t launch_attn_side_merge(AttnArgs a, cudaStream_t st, cudaStream_t side, cudaEvent_t attn_done,
                                   bool *merged) {
    attn_plan(a.rows, a.H, a.K, a.hgroups, a.splits, a.keys_per_split);
    return launch_with_plan(a, st, side, attn_done, merged);
}

}  // namespace csa2

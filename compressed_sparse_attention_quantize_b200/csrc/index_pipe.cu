// Indexer scores of contiguous key ranges (Full mode) on the tensor cores, pipelined.
//
// [B] page "DeepSeek V4.1 Flash 如何靠压缩 KV 缓存实现小模型干翻大模型": section "为什么 KV 缓存成了
// 新瓶颈？" (DSA-style indexer), "CSA2：三层压缩一次吃满" (Full), "FP4 量化 + Bounded Replay"
// (indexer Q and K in FP4).
//
// The same scores as index_tc.cu (raw E2M1 products on the tensor cores with unit block scales,
// exact in fp32; E4M3 scales, ReLU and head weights applied in the fixed order of csa2.h), for
// the rows whose candidates are a contiguous run of 32-byte key rows.  Instead of one tile at a
// time, the stages overlap:
//   warp 0 (producer)   tile i's 128 key rows (4 KB) into ring stage i % kStages with one tensor
//                       copy that writes the MMA operand layout directly (32-byte rows,
//                       32-byte swizzle).  A tile that runs past the row's candidates is copied
//                       exactly with one bulk copy and swizzled by the warp (nothing is read past
//                       the candidates).  The keys' 4-byte scale words go to the stage's scale
//                       slots by asynchronous copies of the warp's lanes, tracked by the same
//                       barrier, so the epilogue never waits on a global load.
//   warp 1 (MMA)        one kind::mxf4 MMA per tile into TMEM buffer i % 3: M = 128 keys,
//                       N = R rows x 4 columns per head; it releases the ring stage when done.
//   warps 2-5           the epilogue of tile i (one key per thread) while the MMA of tile i+1
//                       and the copies of later tiles run.
// R query rows of one sequence may share a CTA (the rows of a prefill sequence see the same key
// range up to their causal limits); the launcher uses R = 1: the epilogue, not the key reads,
// bounds the kernel, and R > 1 needs more TMEM columns per CTA, so fewer CTAs share an SM
// (measured slower at 4 rows per CTA on 4096 prefill rows).
#include "common.cuh"
#include "index_api.cuh"
#include "tc_ptx.cuh"

namespace csa2 {
namespace ipk {

constexpr int kTile = 128;
constexpr int kStages = 6;
constexpr int kNBuf = 3;
constexpr int kMaxR = 4;
constexpr int kThreads = 192;
constexpr int kStageBytes = kTile * 32;               // 4 KB: 128 key rows, 32-byte swizzle
constexpr int kMaxN = kMaxR * 4 * CSA2_MAX_INDEX_HEADS; // B columns (rows x heads x blocks)
constexpr int kSfCols = 32;
constexpr int kRegHeads = 8;                          // heads of the register-held epilogue

struct Args {
    const uint8_t *q_codes, *q_scales;
    const float *w;
    int H, T, R, N1;                   // heads, tokens per sequence, rows per CTA, columns per row
    const uint8_t *k_codes;
    const uint8_t *k_scales;
    int64_t k_scale_stride;
    const int64_t *seq_start;
    const int32_t *n_entries;
    const int32_t *q_pos;
    int row0, nrows;
    float *scores;
    int64_t score_stride;
    uint32_t tmem_cols;
    int tiles_per_cta;
};

struct __align__(1024) Smem {
    uint8_t ring[kStages][kStageBytes];
    uint32_t scales[kStages][kTile];   // the stage's keys' four E4M3 block scales
    uint8_t tail[kTile * 32];          // raw rows of a tile that runs past the candidates
    uint8_t b[2][kMaxN * 16];          // block-diagonal queries of R rows: two 16-byte planes
    float qs[kMaxR][CSA2_MAX_INDEX_HEADS * 4];
    float w[kMaxR][CSA2_MAX_INDEX_HEADS];
    int64_t n_row[kMaxR];
    uint64_t full[kStages], empty[kStages];
    uint64_t tfull[kNBuf], tempty[kNBuf];
    uint64_t tail_bar, drain;
    uint32_t tmem_base;
    int abort_flag;
};

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

// K-major operand with 32-byte rows and the 32-byte swizzle (layout type 6): the 16-byte half c
// of row r sits at half c ^ ((r >> 2) & 1); 8-row groups 256 bytes apart.
CSA2_D uint64_t sdesc_sw32(uint32_t saddr) {
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)(16u >> 4) << 16;
    d |= (uint64_t)(256u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)6u << 61;
    return d;
}

// 4-byte asynchronous copy global -> shared, and an arrival on `bar` once this thread's copies
// so far have landed (the barrier's expected count includes it).
CSA2_D void cp_async_4(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(ptx::smem_u32(dst)), "l"(src) : "memory");
}
CSA2_D void cp_async_arrive(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(ptx::smem_u32(bar)) : "memory");
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

// Candidates of query row r: its sequence's entries, limited by the causal position in prefill.
CSA2_D int64_t row_candidates(const Args &a, int r) {
    int64_t n = a.n_entries[r / a.T];
    if (a.q_pos) {
        const int64_t v = ((int64_t)a.q_pos[r] + 1) / 4;
        n = v < n ? v : n;
        if (n < 0) n = 0;
    }
    return n;
}

__global__ void __launch_bounds__(kThreads, 4)
index_score_pipe_kernel(const Args a, const __grid_constant__ CUtensorMap keys) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // the swizzled stages want their 1024-byte alignment in the shared window
    Smem &S = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int g0 = a.row0 + blockIdx.y * a.R;              // first row of the group
    const int R = min(a.R, a.row0 + a.nrows - g0);
    const int b = g0 / a.T;
    const int H = a.H, N1 = a.N1, NT = R * N1;
    // the group's candidate range: the longest of its rows
    int64_t n = 0;
    for (int rr = 0; rr < R; ++rr) n = max(n, min(row_candidates(a, g0 + rr), a.score_stride));
    const int64_t j0 = (int64_t)blockIdx.x * a.tiles_per_cta * kTile;
    if (j0 >= n) return;                                  // uniform per CTA: nothing allocated yet
    const int ntiles = (int)min((int64_t)a.tiles_per_cta, (n - j0 + kTile - 1) / kTile);
    const int64_t sbase = a.seq_start[b];

    // ---- setup: queries (block-diagonal B), scales, weights, barriers, TMEM ----
    for (int i = t; i < (int)(sizeof(S.b) / 16); i += kThreads)
        reinterpret_cast<uint4 *>(&S.b[0][0])[i] = make_uint4(0u, 0u, 0u, 0u);
    if (t < R) S.n_row[t] = min(row_candidates(a, g0 + t), a.score_stride);
    if (t == 0) {
        for (int i = 0; i < kStages; ++i) {
            ptx::mbar_init(&S.full[i], 1 + 32);           // the code copy (or tail) + 32 lanes' scales
            ptx::mbar_init(&S.empty[i], 1 + 128);         // the MMA + the epilogue's scale reads
        }
        for (int i = 0; i < kNBuf; ++i) {
            ptx::mbar_init(&S.tfull[i], 1);
            ptx::mbar_init(&S.tempty[i], 128);
        }
        ptx::mbar_init(&S.tail_bar, 1);
        ptx::mbar_init(&S.drain, 1);
        S.abort_flag = 0;
        ptx::fence_async_smem();
    }
    if (warp == 0) {
        ptx::tmem_alloc(&S.tmem_base, a.tmem_cols);
        ptx::tmem_relinquish();
    }
    __syncthreads();
    for (int i = t; i < R * H * 4; i += kThreads) {
        const int rr = i / (H * 4), hb = i % (H * 4);
        const int h = hb >> 2, blk = hb & 3;
        const int r = g0 + rr;
        const uint8_t *qc = a.q_codes + ((int64_t)r * H + h) * 32;
        // column rr*N1 + 4h + blk: block blk's 8 code bytes at byte offset 8*blk of the 32-byte row
        const int col = rr * N1 + 4 * h + blk;
        const int plane = blk >> 1, within = (blk & 1) * 8;
        uint8_t *dst = &S.b[plane][col * 16 + within];
#pragma unroll
        for (int k = 0; k < 8; ++k) dst[k] = qc[8 * blk + k];
        S.qs[rr][hb] = e4m3_to_f32(a.q_scales[((int64_t)r * H + h) * 4 + blk]);
    }
    for (int i = t; i < R * H; i += kThreads) S.w[i / H][i % H] = a.w[(int64_t)(g0 + i / H) * H + i % H];
    ptx::fence_async_smem();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    const uint32_t sf_col = kNBuf * NT;
    // every block scale the MMA sees is 1.0 (UE8M0 0x7F): the true E4M3 scales are applied below
    if (warp >= 2) {
        uint32_t ones[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) ones[i] = 0x7F7F7F7Fu;
        ptx::tmem_st32(tmem + ((uint32_t)((warp & 3) * 32) << 16) + sf_col, ones);
        ptx::tmem_st_wait();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    volatile int *abort_flag = &S.abort_flag;

    if (warp == 0) {
        // ================= producer =================
        int issued = 0;
        for (int i = 0; i < ntiles; ++i) {
            const int st = i % kStages;
            if (i >= kStages) {
                bool ok = true;
                if (lane == 0) ok = ptx::mbar_wait(&S.empty[st], ((i / kStages) - 1) & 1, abort_flag);
                if (!__shfl_sync(0xffffffffu, (int)ok, 0)) break;
            }
            const int64_t j = j0 + (int64_t)i * kTile;
            const int rows = (int)min((int64_t)kTile, n - j);
            uint8_t *stage = S.ring[st];
            // the scale words of the tile's keys that exist
            for (int k = lane; k < rows; k += 32)
                cp_async_4(&S.scales[st][k], a.k_scales + (sbase + j + k) * a.k_scale_stride);
            cp_async_arrive(&S.full[st]);
            if (rows == kTile) {
                if (lane == 0) {
                    ptx::mbar_arrive_expect_tx(&S.full[st], (uint32_t)kStageBytes);
                    ptx::tma_load_2d(stage, &keys, 0, (int32_t)(sbase + j), &S.full[st]);
                }
            } else {
                // the last tile: exactly the candidates' rows, then swizzled (rows past the
                // candidates are zero; their scores are never stored)
                bool ok = true;
                if (lane == 0) {
                    ptx::mbar_arrive_expect_tx(&S.tail_bar, (uint32_t)rows * 32u);
                    ptx::bulk_load_g2s(S.tail, a.k_codes + (sbase + j) * 32, (uint32_t)rows * 32u, &S.tail_bar);
                    ok = ptx::mbar_wait(&S.tail_bar, 0, abort_flag);
                }
                if (!__shfl_sync(0xffffffffu, (int)ok, 0)) break;
                for (int row = lane; row < kTile; row += 32) {
                    uint4 p0 = make_uint4(0u, 0u, 0u, 0u), p1 = p0;
                    if (row < rows) {
                        p0 = *reinterpret_cast<const uint4 *>(S.tail + row * 32);
                        p1 = *reinterpret_cast<const uint4 *>(S.tail + row * 32 + 16);
                    }
                    const int sw = (row >> 2) & 1;
                    *reinterpret_cast<uint4 *>(stage + row * 32 + 16 * sw) = p0;
                    *reinterpret_cast<uint4 *>(stage + row * 32 + 16 * (sw ^ 1)) = p1;
                }
                ptx::fence_async_smem();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&S.full[st]);
            }
            issued = i + 1;
        }
        // the tensor copies still in flight land before the warp leaves
        if (lane == 0) {
            for (int i = issued > kStages ? issued - kStages : 0; i < issued; ++i)
                ptx::mbar_wait_drain(&S.full[i % kStages], (i / kStages) & 1);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ================= MMA issuer =================
        if (lane == 0) {
            const uint32_t idesc = idesc_mxf4(128, NT);
            const uint64_t bdesc = sdesc_noswizzle(ptx::smem_u32(&S.b[0][0]), kMaxN * 16, 128);
            const uint32_t sf = tmem + sf_col;
            for (int i = 0; i < ntiles; ++i) {
                const int st = i % kStages, buf = i % kNBuf;
                if (!ptx::mbar_wait(&S.full[st], (i / kStages) & 1, abort_flag)) break;
                if (i >= kNBuf && !ptx::mbar_wait(&S.tempty[buf], ((i / kNBuf) - 1) & 1, abort_flag)) break;
                ptx::tc_fence_after();
                const uint64_t adesc = sdesc_sw32(ptx::smem_u32(S.ring[st]));
                mma_mxf4(tmem + buf * NT, adesc, bdesc, idesc, sf, sf);
                ptx::mma_commit(&S.empty[st]);
                ptx::mma_commit(&S.tfull[buf]);
            }
            // every issued MMA has completed before TMEM is released
            ptx::mma_commit(&S.drain);
            ptx::mbar_wait_drain(&S.drain, 0);
        }
        __syncwarp();
    } else if (R == 1 && H == kRegHeads) {
        // ======= epilogue, one row of 8 heads: its scales and weights held in registers =======
        const int sub = warp & 3;
        const int key = sub * 32 + lane;                   // TMEM lane = key within the tile
        const uint32_t lane_addr = tmem + ((uint32_t)(sub * 32) << 16);
        float qs[kRegHeads][4], wh[kRegHeads];
#pragma unroll
        for (int h = 0; h < kRegHeads; ++h) {
            wh[h] = S.w[0][h];
#pragma unroll
            for (int q = 0; q < 4; ++q) qs[h][q] = S.qs[0][h * 4 + q];
        }
        const int64_t n_row = S.n_row[0];
        float *out = a.scores + (int64_t)(g0 - a.row0) * a.score_stride;
        for (int i = 0; i < ntiles; ++i) {
            const int buf = i % kNBuf;
            if (!ptx::mbar_wait(&S.tfull[buf], (i / kNBuf) & 1, abort_flag)) break;
            ptx::tc_fence_after();
            // heads 0-3, then 4-7: 16 accumulator columns at a time keep the registers in budget
            uint32_t u[16];
            ptx::tmem_ld16(lane_addr + buf * NT, u);
            const uint32_t sc_this = S.scales[i % kStages][key];
            ptx::mbar_arrive(&S.empty[i % kStages]);
            float sk[4];
            ptx::e4m3x4_to_f32(sc_this, sk);
            float acc = 0.0f;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                if (half == 1) ptx::tmem_ld16(lane_addr + buf * NT + 16, u);
                ptx::tmem_ld_wait();
                if (half == 1) {
                    ptx::tc_fence_before();
                    ptx::mbar_arrive(&S.tempty[buf]);      // the accumulator is in registers
                }
#pragma unroll
                for (int hh = 0; hh < 4; ++hh) {
                    const int h = half * 4 + hh;
                    float c[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) c[q] = __fmul_rn(qs[h][q], sk[q]);
                    const float dot = head_block_sum(u + hh * 4, c);
                    acc = __fadd_rn(acc, __fmul_rn(wh[h], dot > 0.0f ? dot : 0.0f));
                }
            }
            if (acc == 0.0f) acc = 0.0f;                     // -0 -> +0
            const int64_t j = j0 + (int64_t)i * kTile + key;
            if (j < n_row) out[j] = acc;
        }
    } else {
        // ================= epilogue: one key per thread =================
        const int sub = warp & 3;
        const int key = sub * 32 + lane;                   // TMEM lane = key within the tile
        const uint32_t lane_addr = tmem + ((uint32_t)(sub * 32) << 16);
        for (int i = 0; i < ntiles; ++i) {
            const int buf = i % kNBuf;
            if (!ptx::mbar_wait(&S.tfull[buf], (i / kNBuf) & 1, abort_flag)) break;
            ptx::tc_fence_after();
            // the key's scale words landed with its stage (tfull follows the stage's full barrier);
            // the stage is refilled only after every epilogue thread has read them
            const uint32_t sc_this = S.scales[i % kStages][key];
            ptx::mbar_arrive(&S.empty[i % kStages]);
            float sk[4];
            ptx::e4m3x4_to_f32(sc_this, sk);
            const int64_t j = j0 + (int64_t)i * kTile + key;
            for (int rr = 0; rr < R; ++rr) {
                float acc = 0.0f;
                for (int hb = 0; hb * 8 < H; ++hb) {
                    uint32_t u[32];
                    ptx::tmem_ld32(lane_addr + buf * NT + rr * N1 + hb * 32, u);
                    ptx::tmem_ld_wait();
#pragma unroll
                    for (int hh = 0; hh < 8; ++hh) {
                        const int h = hb * 8 + hh;
                        if (h < H) {
                            float c[4];
#pragma unroll
                            for (int q = 0; q < 4; ++q) c[q] = __fmul_rn(S.qs[rr][h * 4 + q], sk[q]);
                            const float dot = head_block_sum(u + hh * 4, c);
                            const float rl = dot > 0.0f ? dot : 0.0f;
                            acc = __fadd_rn(acc, __fmul_rn(S.w[rr][h], rl));
                        }
                    }
                }
                if (acc == 0.0f) acc = 0.0f;                 // -0 -> +0
                if (j < S.n_row[rr]) a.scores[(int64_t)(g0 - a.row0 + rr) * a.score_stride + j] = acc;
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(&S.tempty[buf]);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, a.tmem_cols);
    }
}

}  // namespace ipk

// cuTensorMapEncodeTiled from the driver, looked up once
using IpkEncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                      const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                      CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
static IpkEncodeTiledFn ipk_encode_tiled() {
    static const IpkEncodeTiledFn fn = []() -> IpkEncodeTiledFn {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<IpkEncodeTiledFn>(p);
    }();
    return fn;
}

static SmemLimit g_index_pipe_smem;

// Decode (one query row per sequence) with contiguous keys.  Prefill rows stay on index_tc.cu:
// its epilogue, which bounds both kernels, keeps more warps busy per SM there (measured 1.21 ms
// here against about 1.0 ms per 2000-row chunk of 33,792 keys).
bool index_pipe_applies(const IndexLaunch &L) {
    // 4-byte asynchronous copies of the scale words need them 4-byte aligned
    return L.mode == CSA2_MODE_FULL && L.T == 1 && L.k_code_stride == 32 && (L.k_scale_stride & 3) == 0 &&
           (reinterpret_cast<uintptr_t>(L.k_scales) & 3) == 0 && ipk_encode_tiled() != nullptr;
}

// R rows per CTA: row0 and T must be multiples of R so that a group's rows belong to one
// sequence.
cudaError_t launch_index_score_pipe(const IndexLaunch &L, int row0, int nrows, int R, float *scores,
                                    int64_t score_stride, cudaStream_t st) {
    if (R < 1 || R > ipk::kMaxR || row0 % R != 0 || L.T % R != 0) return cudaErrorInvalidValue;
    ipk::Args a;
    a.q_codes = L.q_codes; a.q_scales = L.q_scales; a.w = L.w;
    a.H = L.H; a.T = L.T;
    a.R = R;
    a.N1 = ((4 * L.H + 15) / 16) * 16;
    a.k_codes = L.k_codes;
    a.k_scales = L.k_scales; a.k_scale_stride = L.k_scale_stride;
    a.seq_start = L.seq_start; a.n_entries = L.n_entries; a.q_pos = L.q_pos;
    a.row0 = row0; a.nrows = nrows;
    a.scores = scores;
    a.score_stride = score_stride;
    const int NT = a.R * a.N1;
    uint32_t cols = 32;
    while (cols < (uint32_t)(ipk::kNBuf * NT + ipk::kSfCols)) cols <<= 1;
    a.tmem_cols = cols;
    // key codes: 32-byte rows, 128 rows per box, written with the 32-byte swizzle of the operand
    CUtensorMap keys;
    const IpkEncodeTiledFn enc = ipk_encode_tiled();
    if (!enc) return cudaErrorNotSupported;
    cudaError_t e = bind_current_context();
    if (e != cudaSuccess) return e;
    {
        const cuuint64_t dim[2] = {32, (cuuint64_t)INT32_MAX};
        const cuuint64_t stride[1] = {32};
        const cuuint32_t box[2] = {32, (cuuint32_t)ipk::kTile};
        const cuuint32_t ones[2] = {1, 1};
        if (enc(&keys, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(L.k_codes), dim, stride, box, ones,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    const int smem = (int)sizeof(ipk::Smem) + 1024;
    e = ensure_smem_limit(g_index_pipe_smem, ipk::index_score_pipe_kernel, smem);
    if (e != cudaSuccess) return e;
    // CTAs per SM: TMEM columns and shared memory
    const int per_sm = min(512 / (int)cols, (227 * 1024) / (smem + 1024));
    const int resident = max(per_sm, 1) * device_sm_count();
    const int groups = (nrows + a.R - 1) / a.R;
    // tiles per CTA: the fewest that fit every group's tiles into one wave of resident CTAs
    const int64_t tiles_row = ceil_div(score_stride, (int64_t)ipk::kTile);
    const int64_t per_group = resident / groups;
    int64_t tpc = per_group > 0 ? ceil_div(tiles_row, per_group) : 8;
    if (tpc < 1) tpc = 1;
    a.tiles_per_cta = (int)tpc;
    dim3 grid((unsigned)ceil_div(tiles_row, tpc), (unsigned)groups);
    ipk::index_score_pipe_kernel<<<grid, ipk::kThreads, smem, st>>>(a, keys);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace csa2

// Quantise-on-write kernels (FP4 main KV / indexer rows, FP8 sliding-window rows).
//
// [B] page "DeepSeek V4.1 Flash 如何靠压缩 KV 缓存实现小模型干翻大模型", section
// "FP4 量化 + Bounded Replay": E2M1 with one E4M3 scale per 16 channels, no second-level
// scale.  [A] page "DeepSeek V4.1 Flash深度解析：KV缓存压缩437倍的技术路径", section
// "压缩吸收注意力（二代）": the precision-sensitive sliding window stays at 8 bits.
//
// Exactness: every code is the quotient's exact value rounded once.
//  * FP4 scale s = E4M3(amax/6): amax/6 is divided in fp32 (round-to-nearest).  amax and 6*mu
//    share one fp32 grid for every E4M3 midpoint mu, so a non-exact quotient sits more than
//    half an fp32 ulp away from mu and the fp32 rounding cannot create a false tie.
//  * FP4 code = E2M1(x/s) without a division: |x| is compared with mu*s for the seven E2M1
//    midpoints mu.  mu has at most 3 significant bits and s (an E4M3 value) at most 4, so every
//    product is exact in fp32 and each comparison decides on the exact quotient.
//  * FP8 code = E4M3(x/s) with a full 24-bit s: an approximate quotient |x| * (1/s) (a few
//    fp32 ulps off) is rounded, and the one midpoint mu it may have crossed is tested exactly:
//    the sign of |x| - mu*s, one fma, rounded once, is the sign of the exact difference (s and
//    |x| first scaled by a power of two that brings s into [2^-100, 2^100]).
#include "common.cuh"

namespace csa2 {

template <typename T>
CSA2_D float load_as_f32(const T *p);
template <>
CSA2_D float load_as_f32<float>(const float *p) { return __ldg(p); }
template <>
CSA2_D float load_as_f32<uint16_t>(const uint16_t *p) { return bf16_bits_to_f32(__ldg(p)); }

// The seven E2M1 midpoints times an E4M3 scale s (all exact), and the signed code of x/s from
// them, nearest-even and saturating at 6: 0.25 -> 0, 0.75 -> 1.0, 1.25 -> 1.0, 1.75 -> 2,
// 2.5 -> 2, 3.5 -> 4, 5 -> 4.
struct E2M1Cuts {
    float c[7];
};
CSA2_D E2M1Cuts e2m1_cuts(float s) {
    return {{0.25f * s, 0.75f * s, 1.25f * s, 1.75f * s, 2.5f * s, 3.5f * s, 5.0f * s}};
}
CSA2_D uint32_t e2m1_code(float x, const E2M1Cuts &t) {
    const float a = fabsf(x);
    const uint32_t m = (uint32_t)(a > t.c[0]) + (uint32_t)(a >= t.c[1]) + (uint32_t)(a > t.c[2]) +
                       (uint32_t)(a >= t.c[3]) + (uint32_t)(a > t.c[4]) + (uint32_t)(a >= t.c[5]) +
                       (uint32_t)(a > t.c[6]);
    return m | (signbit(x) ? 8u : 0u);
}

// FP4 quantisation of one 16-channel block: 8 code bytes at cd, one E4M3 scale at *sd.
CSA2_D void quantize_block16(const float (&v)[16], uint8_t *cd, uint8_t *sd) {
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const uint32_t sc = e4m3_code_mag_rne(__fdiv_rn(amax, 6.0f));
    const float s = e4m3_to_f32(sc);
    uint32_t packed[2] = {0u, 0u};
    if (s != 0.0f) {
        const E2M1Cuts t = e2m1_cuts(s);
#pragma unroll
        for (int i = 0; i < 16; ++i) packed[i >> 3] |= e2m1_code(v[i], t) << ((i & 7) * 4);
    }
    // 8 code bytes; alignment of cd is only guaranteed to 1 byte in general
    if ((((uintptr_t)cd) & 7u) == 0) {
        *reinterpret_cast<uint2 *>(cd) = make_uint2(packed[0], packed[1]);
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) cd[i] = (uint8_t)(packed[i >> 2] >> ((i & 3) * 8));
    }
    *sd = (uint8_t)sc;
}

// One thread per 16-channel block.
template <typename T>
__global__ void quant_fp4_kernel(const T *__restrict__ x, int64_t rows, int dim, int64_t x_stride,
                                 uint8_t *__restrict__ codes, int64_t code_stride,
                                 uint8_t *__restrict__ scales, int64_t scale_stride,
                                 const int64_t *__restrict__ dst_rows) {
    const int nblk = dim >> 4;
    const int64_t total = rows * nblk;
    for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total;
         t += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = t / nblk;
        const int b = (int)(t - r * nblk);
        const T *xr = x + r * x_stride + b * 16;
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = load_as_f32<T>(xr + i);
        const int64_t d = dst_rows ? dst_rows[r] : r;
        quantize_block16(v, codes + d * code_stride + b * 8, scales + d * scale_stride + b);
    }
}

// Sequence compressor + quantise-on-write ([B] section "CSA2：三层压缩一次吃满": every m tokens
// become one entry).  Entry e = sum_k w[e][k] * x[m*e + k] in fp32, tokens in order, every
// product and sum rounded once (no fused multiply-add); w == NULL is the mean (w = 1/m).
// One thread per (entry, 16-channel block).
template <typename T>
__global__ void compress_fp4_kernel(const T *__restrict__ x, int64_t entries, int ratio, int dim,
                                    int64_t x_stride, const float *__restrict__ w, int64_t w_stride,
                                    uint8_t *__restrict__ codes, int64_t code_stride,
                                    uint8_t *__restrict__ scales, int64_t scale_stride,
                                    const int64_t *__restrict__ dst_rows) {
    const int nblk = dim >> 4;
    const int64_t total = entries * nblk;
    const float mean_w = __fdiv_rn(1.0f, (float)ratio);
    for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total;
         t += (int64_t)gridDim.x * blockDim.x) {
        const int64_t e = t / nblk;
        const int b = (int)(t - e * nblk);
        float v[16];
        for (int k = 0; k < ratio; ++k) {
            const float wk = w ? __ldg(w + e * w_stride + k) : mean_w;
            const T *xr = x + (e * ratio + k) * x_stride + b * 16;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float prod = __fmul_rn(wk, load_as_f32<T>(xr + i));
                v[i] = k == 0 ? prod : __fadd_rn(v[i], prod);
            }
        }
        const int64_t d = dst_rows ? dst_rows[e] : e;
        quantize_block16(v, codes + d * code_stride + b * 8, scales + d * scale_stride + b);
    }
}

// Per-row constants of the E4M3 codes of x/s: a power of two f that brings the scale into
// [2^-100, 2^100] (f = 1 for the scales of ordinary data), sf = s*f and rs = 1/sf.  Scaling
// |x| and s by f leaves the quotient as it is, and |x|*f is exact wherever the code can be
// non-zero: f > 1 only scales up, and f < 1 only loses bits of values below 2^-62 whose
// quotient is below 2^-100.
struct E4M3Row {
    float f, sf, rs;
};
CSA2_D E4M3Row e4m3_row(float s) {
    const float f = s < 0x1p-100f ? 0x1p64f : (s > 0x1p100f ? 0x1p-64f : 1.0f);
    const float sf = s * f;
    return {f, sf, __frcp_rn(sf)};
}

// E4M3 code of the exact quotient a/s (a >= 0, s > 0), rounded once, nearest-even, satfinite.
// q = (a*f) * rs is within a few fp32 ulps of the exact quotient, so its rounding is off by
// at most one code, and only across the midpoint mu between the rounded code and its
// neighbour on q's side.  That midpoint is tested exactly: a*f - mu*sf by one fma, rounded
// once, has the sign of the exact difference (mu*sf and a*f lie on a grid that fp32 resolves
// for sf in [2^-100, 2^100]).
CSA2_D uint32_t e4m3_code_of_quotient(float a, const E4M3Row &k) {
    const float af = a * k.f;
    const float q = af * k.rs;
    uint32_t c = e4m3_code_mag_rne(q);
    const float v = e4m3_to_f32(c);
    if (q > v && c < 0x7Eu) {
        const float d = fmaf(-0.5f * (v + e4m3_to_f32(c + 1u)), k.sf, af);
        if (d > 0.0f || (d == 0.0f && (c & 1u))) c += 1u;        // at or past the tie: up
    } else if (q < v && c > 0u) {
        const float d = fmaf(-0.5f * (v + e4m3_to_f32(c - 1u)), k.sf, af);
        if (d < 0.0f || (d == 0.0f && (c & 1u))) c -= 1u;        // at or below the tie: down
    }
    return c;
}

// Signed E4M3 code of x for its row's scale s (k = e4m3_row(s)); a zero scale gives code 0.
CSA2_D uint32_t e4m3_code_scaled(float x, float s, const E4M3Row &k) {
    if (s == 0.0f) return 0u;
    return e4m3_code_of_quotient(fabsf(x), k) | (signbit(x) ? 0x80u : 0u);
}

// One token row by one warp: the scale s = amax / 448 and every code.  Rows of up to 512
// channels are read once, all loads issued before the first is used (a loop that waits for each
// load in turn made a step's small window write latency-bound); longer rows take two passes.
template <typename Load>
CSA2_D void fp8_token_row(int lane, int dim, Load load, uint8_t *cd, float *scale) {
    constexpr int kPer = 16;
    if (dim <= 32 * kPer) {
        float v[kPer];
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            const int i = lane + 32 * k;
            v[k] = i < dim ? load(i) : 0.0f;
        }
        float amax = 0.0f;
#pragma unroll
        for (int k = 0; k < kPer; ++k) amax = fmaxf(amax, fabsf(v[k]));
        // non-negative floats order like their bit patterns
        amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
        const float s = __fdiv_rn(amax, 448.0f);
        const E4M3Row kr = e4m3_row(s);
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            const int i = lane + 32 * k;
            if (i < dim) cd[i] = (uint8_t)e4m3_code_scaled(v[k], s, kr);
        }
        if (lane == 0) *scale = s;
        return;
    }
    float amax = 0.0f;
    for (int i = lane; i < dim; i += 32) amax = fmaxf(amax, fabsf(load(i)));
    amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
    const float s = __fdiv_rn(amax, 448.0f);
    const E4M3Row kr = e4m3_row(s);
    for (int i = lane; i < dim; i += 32) cd[i] = (uint8_t)e4m3_code_scaled(load(i), s, kr);
    if (lane == 0) *scale = s;
}

// One warp per row.
template <typename T>
__global__ void quant_fp8_token_kernel(const T *__restrict__ x, int64_t rows, int dim,
                                       int64_t x_stride, uint8_t *__restrict__ codes,
                                       int64_t code_stride, uint8_t *__restrict__ scales,
                                       int64_t scale_stride, const int64_t *__restrict__ dst_rows) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t r = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
         r += warps) {
        const T *xr = x + r * x_stride;
        const int64_t d = dst_rows ? dst_rows[r] : r;
        fp8_token_row(lane, dim, [&](int i) { return load_as_f32<T>(xr + i); }, codes + d * code_stride,
                      reinterpret_cast<float *>(scales + d * scale_stride));
    }
}

// ---------------------------------------------------------------------------------------
// Several quantise-on-write jobs in one launch (a decode step writes a main-KV entry, its
// indexer key, window tokens and indexer queries: one launch instead of one per buffer).
// Block b belongs to the job whose block range holds it.  A thread takes 4 neighbouring
// channels of one row, read in one vector load where the row's alignment allows: an FP4 block
// is 4 neighbouring lanes (block amax by two shuffles), an FP8 row of up to 2048 channels is a
// group of 128 threads (row amax by a warp reduction, then the group's 4 warps through shared
// memory).  The step's writes are a few hundred rows, so the launch is one short wave and its
// time is the chain load -> amax -> scale -> codes -> store of one thread, kept short this way.
// Longer FP8 rows take one warp per row.
// ---------------------------------------------------------------------------------------
struct QuantJob {
    int fmt, x_dtype, dim;
    const void *x;
    int64_t rows, x_stride;
    uint8_t *codes;
    int64_t code_stride;
    uint8_t *scales;
    int64_t scale_stride;
    const int64_t *dst_rows;
};

constexpr int kMaxQuantJobs = 16;
static_assert(kMaxQuantJobs == CSA2_MAX_QUANT_JOBS, "one job table size");
constexpr int kQuantThreads = 256;
constexpr int kRowGroup = 128;                           // threads of one FP8 row
constexpr int kRowVecs = 4;                              // 4-channel groups a thread holds
constexpr int kRowMaxDim = kRowGroup * 4 * kRowVecs;     // longest FP8 row held in registers

struct QuantJobs {
    QuantJob job[kMaxQuantJobs];
    int64_t block_start[kMaxQuantJobs + 1];
    int n;
};

CSA2_D float load_elem(const void *x, int dtype, int64_t i) {
    return dtype == CSA2_DTYPE_F32 ? __ldg(reinterpret_cast<const float *>(x) + i)
                                   : bf16_bits_to_f32(__ldg(reinterpret_cast<const uint16_t *>(x) + i));
}

// Channels i .. i+3 of x (element offset i); vec: one 16-byte (f32) or 8-byte (bf16) load.
CSA2_D void load4(const void *x, int dtype, int64_t i, bool vec, float (&v)[4]) {
    if (dtype == CSA2_DTYPE_F32) {
        const float *p = reinterpret_cast<const float *>(x) + i;
        if (vec) {
            const float4 t = __ldg(reinterpret_cast<const float4 *>(p));
            v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
        } else {
#pragma unroll
            for (int k = 0; k < 4; ++k) v[k] = __ldg(p + k);
        }
    } else {
        const uint16_t *p = reinterpret_cast<const uint16_t *>(x) + i;
        if (vec) {
            const uint2 t = __ldg(reinterpret_cast<const uint2 *>(p));
            v[0] = bf16_bits_to_f32((uint16_t)(t.x & 0xFFFFu)); v[1] = bf16_bits_to_f32((uint16_t)(t.x >> 16));
            v[2] = bf16_bits_to_f32((uint16_t)(t.y & 0xFFFFu)); v[3] = bf16_bits_to_f32((uint16_t)(t.y >> 16));
        } else {
#pragma unroll
            for (int k = 0; k < 4; ++k) v[k] = bf16_bits_to_f32(__ldg(p + k));
        }
    }
}

// Rows start on a vector boundary: base aligned and the row stride a multiple of 4 elements.
CSA2_D bool rows_vec_aligned(const QuantJob &q) {
    const uintptr_t need = q.x_dtype == CSA2_DTYPE_F32 ? 15u : 7u;
    return ((reinterpret_cast<uintptr_t>(q.x) & need) == 0) && ((q.x_stride & 3) == 0);
}

// 4 code bytes (little-endian in w) at p: one 32-bit store when aligned.
CSA2_D void store4(uint8_t *p, uint32_t w, bool aligned) {
    if (aligned) {
        *reinterpret_cast<uint32_t *>(p) = w;
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) p[k] = (uint8_t)(w >> (8 * k));
    }
}

__global__ void __launch_bounds__(kQuantThreads) quant_batch_kernel(const __grid_constant__ QuantJobs J) {
    __shared__ float group_amax[kQuantThreads / 32];
    int j = 0;
    while (j + 1 < J.n && (int64_t)blockIdx.x >= J.block_start[j + 1]) ++j;
    const QuantJob &q = J.job[j];
    const int64_t lb = (int64_t)blockIdx.x - J.block_start[j];
    const int lane = threadIdx.x & 31;
    const bool vec = rows_vec_aligned(q);
    if (q.fmt == CSA2_FMT_FP4_E2M1_E4M3S16) {
        // thread t: row t / (dim/4), channels 4*(t % (dim/4)) ..; dim/4 is a multiple of 4, so
        // the 4 lanes of a block are lanes 4k .. 4k+3 of one warp
        const int64_t quads = q.dim >> 2;
        const int64_t t = lb * kQuantThreads + threadIdx.x;
        const bool live = t < q.rows * quads;
        float v[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        int64_t d = 0;
        int c4 = 0;
        if (live) {
            const int64_t r = t / quads;
            c4 = (int)(t - r * quads);
            load4(q.x, q.x_dtype, r * q.x_stride + 4 * c4, vec, v);
            d = q.dst_rows ? __ldg(q.dst_rows + r) : r;
        }
        float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        const uint32_t sc = e4m3_code_mag_rne(__fdiv_rn(amax, 6.0f));
        const float s = e4m3_to_f32(sc);
        uint32_t p = 0u;
        if (s != 0.0f) {
            const E2M1Cuts cuts = e2m1_cuts(s);
#pragma unroll
            for (int k = 0; k < 4; ++k) p |= e2m1_code(v[k], cuts) << (4 * k);
        }
        // lanes 4k and 4k+2 assemble code words 0 and 1 of the block (channels 0-7, 8-15)
        const uint32_t w = p | (__shfl_down_sync(0xffffffffu, p, 1) << 16);
        if (live && (c4 & 1) == 0) {
            uint8_t *cd = q.codes + d * q.code_stride + (c4 >> 2) * 8 + (c4 & 2) * 2;
            store4(cd, w, ((reinterpret_cast<uintptr_t>(q.codes) | (uintptr_t)q.code_stride) & 3u) == 0);
            if ((c4 & 3) == 0) q.scales[d * q.scale_stride + (c4 >> 2)] = (uint8_t)sc;
        }
    } else if (q.dim <= kRowMaxDim) {
        const int grp = threadIdx.x / kRowGroup, tr = threadIdx.x % kRowGroup;
        const int64_t r = lb * (kQuantThreads / kRowGroup) + grp;
        const bool live = r < q.rows;                        // uniform per group
        float v[kRowVecs][4];
        float amax = 0.0f;
#pragma unroll
        for (int k = 0; k < kRowVecs; ++k) {
            const int c = 4 * (tr + kRowGroup * k);
            if (live && c < q.dim) {
                load4(q.x, q.x_dtype, r * q.x_stride + c, vec, v[k]);
            } else {
                v[k][0] = v[k][1] = v[k][2] = v[k][3] = 0.0f;
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) amax = fmaxf(amax, fabsf(v[k][e]));
        }
        const int64_t d = live ? (q.dst_rows ? __ldg(q.dst_rows + r) : r) : 0;
        // non-negative floats order like their bit patterns
        amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
        if (lane == 0) group_amax[threadIdx.x >> 5] = amax;
        __syncthreads();
        const float *ga = group_amax + grp * (kRowGroup / 32);
        amax = fmaxf(fmaxf(ga[0], ga[1]), fmaxf(ga[2], ga[3]));
        const float s = __fdiv_rn(amax, 448.0f);
        const E4M3Row kr = e4m3_row(s);
        if (live) {
            uint8_t *cd = q.codes + d * q.code_stride;
            const bool al = ((reinterpret_cast<uintptr_t>(q.codes) | (uintptr_t)q.code_stride) & 3u) == 0;
#pragma unroll
            for (int k = 0; k < kRowVecs; ++k) {
                const int c = 4 * (tr + kRowGroup * k);
                if (c < q.dim) {
                    uint32_t w = 0u;
#pragma unroll
                    for (int e = 0; e < 4; ++e) w |= e4m3_code_scaled(v[k][e], s, kr) << (8 * e);
                    store4(cd + c, w, al);
                }
            }
            if (tr == 0) *reinterpret_cast<float *>(q.scales + d * q.scale_stride) = s;
        }
    } else {
        const int64_t r = lb * (kQuantThreads / 32) + (threadIdx.x >> 5);
        if (r >= q.rows) return;                                   // uniform per warp
        const int64_t base = r * q.x_stride;
        const int64_t d = q.dst_rows ? q.dst_rows[r] : r;
        fp8_token_row(lane, q.dim, [&](int i) { return load_elem(q.x, q.x_dtype, base + i); },
                      q.codes + d * q.code_stride, reinterpret_cast<float *>(q.scales + d * q.scale_stride));
    }
}

cudaError_t launch_quant_batch(const csa2_quant_job *jobs, int n, cudaStream_t st) {
    QuantJobs J;
    J.n = 0;
    int64_t blocks = 0;
    for (int i = 0; i < n; ++i) {
        const csa2_quant_job &s = jobs[i];
        if (s.rows == 0) continue;
        QuantJob &q = J.job[J.n];
        q.fmt = s.fmt; q.x_dtype = s.x_dtype; q.dim = s.dim; q.x = s.x; q.rows = s.rows;
        q.x_stride = s.x_stride; q.codes = s.codes; q.code_stride = s.code_stride;
        q.scales = reinterpret_cast<uint8_t *>(s.scales); q.scale_stride = s.scale_stride;
        q.dst_rows = s.dst_rows;
        J.block_start[J.n] = blocks;
        if (s.fmt == CSA2_FMT_FP4_E2M1_E4M3S16)
            blocks += ceil_div(s.rows * (s.dim / 4), kQuantThreads);
        else if (s.dim <= kRowMaxDim)
            blocks += ceil_div(s.rows, kQuantThreads / kRowGroup);
        else
            blocks += ceil_div(s.rows, kQuantThreads / 32);
        ++J.n;
    }
    J.block_start[J.n] = blocks;
    if (J.n == 0) return cudaSuccess;
    if (blocks > INT32_MAX) return cudaErrorInvalidConfiguration;
    quant_batch_kernel<<<(unsigned)blocks, kQuantThreads, 0, st>>>(J);
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_quant_fp4(const void *x, int x_dtype, int64_t rows, int dim, int64_t x_stride,
                             uint8_t *codes, int64_t code_stride, uint8_t *scales,
                             int64_t scale_stride, const int64_t *dst_rows, cudaStream_t st) {
    const int64_t total = rows * (dim / 16);
    const int threads = 256;
    int64_t blocks = ceil_div(total, threads);
    if (blocks > 148 * 64) blocks = 148 * 64;
    if (x_dtype == CSA2_DTYPE_F32)
        quant_fp4_kernel<float><<<(unsigned)blocks, threads, 0, st>>>(
            (const float *)x, rows, dim, x_stride, codes, code_stride, scales, scale_stride, dst_rows);
    else
        quant_fp4_kernel<uint16_t><<<(unsigned)blocks, threads, 0, st>>>(
            (const uint16_t *)x, rows, dim, x_stride, codes, code_stride, scales, scale_stride,
            dst_rows);
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_compress_fp4(const void *x, int x_dtype, int64_t entries, int ratio, int dim,
                                int64_t x_stride, const float *w, int64_t w_stride, uint8_t *codes,
                                int64_t code_stride, uint8_t *scales, int64_t scale_stride,
                                const int64_t *dst_rows, cudaStream_t st) {
    const int64_t total = entries * (dim / 16);
    const int threads = 256;
    int64_t blocks = ceil_div(total, threads);
    if (blocks > 148 * 64) blocks = 148 * 64;
    if (x_dtype == CSA2_DTYPE_F32)
        compress_fp4_kernel<float><<<(unsigned)blocks, threads, 0, st>>>(
            (const float *)x, entries, ratio, dim, x_stride, w, w_stride, codes, code_stride, scales,
            scale_stride, dst_rows);
    else
        compress_fp4_kernel<uint16_t><<<(unsigned)blocks, threads, 0, st>>>(
            (const uint16_t *)x, entries, ratio, dim, x_stride, w, w_stride, codes, code_stride, scales,
            scale_stride, dst_rows);
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_quant_fp8_token(const void *x, int x_dtype, int64_t rows, int dim,
                                   int64_t x_stride, uint8_t *codes, int64_t code_stride,
                                   uint8_t *scales, int64_t scale_stride, const int64_t *dst_rows,
                                   cudaStream_t st) {
    const int threads = 256;
    int64_t blocks = ceil_div(rows, threads / 32);
    if (blocks > 148 * 32) blocks = 148 * 32;
    if (x_dtype == CSA2_DTYPE_F32)
        quant_fp8_token_kernel<float><<<(unsigned)blocks, threads, 0, st>>>(
            (const float *)x, rows, dim, x_stride, codes, code_stride, scales, scale_stride, dst_rows);
    else
        quant_fp8_token_kernel<uint16_t><<<(unsigned)blocks, threads, 0, st>>>(
            (const uint16_t *)x, rows, dim, x_stride, codes, code_stride, scales, scale_stride,
            dst_rows);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace csa2

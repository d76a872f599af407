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
//  * FP4 code = E2M1(x/s): s has at most 4 significant bits, the same argument applies.
//  * FP8 code = E4M3(x/s) with a full 24-bit s: the fp32 quotient can land exactly on a
//    midpoint; the exact remainder x - q*s (one fma) then says which side the exact quotient
//    is on and the tie is re-resolved.
#include "common.cuh"

namespace csa2 {

template <typename T>
CSA2_D float load_as_f32(const T *p);
template <>
CSA2_D float load_as_f32<float>(const float *p) { return __ldg(p); }
template <>
CSA2_D float load_as_f32<uint16_t>(const uint16_t *p) { return bf16_bits_to_f32(__ldg(p)); }

// FP4 quantisation of one 16-channel block: 8 code bytes at cd, one E4M3 scale at *sd.
CSA2_D void quantize_block16(const float (&v)[16], uint8_t *cd, uint8_t *sd) {
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const uint32_t sc = e4m3_code_mag_rne(__fdiv_rn(amax, 6.0f));
    const float s = e4m3_to_f32(sc);
    uint32_t packed[2] = {0u, 0u};
    if (s != 0.0f) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float q = __fdiv_rn(fabsf(v[i]), s);
            uint32_t c = e2m1_code_mag_rne(q) | (signbit(v[i]) ? 8u : 0u);
            packed[i >> 3] |= c << ((i & 7) * 4);
        }
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

// E4M3 code of the exact quotient a/s (a >= 0, s > 0), rounded once, nearest-even, satfinite.
CSA2_D uint32_t e4m3_code_of_quotient(float a, float s) {
    const float q = __fdiv_rn(a, s);
    uint32_t c = e4m3_code_mag_rne(q);
    if (c < 0x7Eu || q <= 448.0f) {
        const float v = e4m3_to_f32(c);
        if (q > v && c < 0x7Eu) {
            const float up = e4m3_to_f32(c + 1u);
            if (q == 0.5f * (v + up) && fmaf(-q, s, a) > 0.0f) c += 1u;   // exact is above the tie
        } else if (q < v && c > 0u) {
            const float dn = e4m3_to_f32(c - 1u);
            if (q == 0.5f * (v + dn) && fmaf(-q, s, a) < 0.0f) c -= 1u;   // exact is below the tie
        }
    }
    return c;
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
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            const int i = lane + 32 * k;
            if (i < dim) {
                uint32_t c = 0u;
                if (s != 0.0f) c = e4m3_code_of_quotient(fabsf(v[k]), s) | (signbit(v[k]) ? 0x80u : 0u);
                cd[i] = (uint8_t)c;
            }
        }
        if (lane == 0) *scale = s;
        return;
    }
    float amax = 0.0f;
    for (int i = lane; i < dim; i += 32) amax = fmaxf(amax, fabsf(load(i)));
    amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
    const float s = __fdiv_rn(amax, 448.0f);
    for (int i = lane; i < dim; i += 32) {
        const float v = load(i);
        uint32_t c = 0u;
        if (s != 0.0f) c = e4m3_code_of_quotient(fabsf(v), s) | (signbit(v) ? 0x80u : 0u);
        cd[i] = (uint8_t)c;
    }
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
// Block b belongs to the job whose block range holds it; FP4 jobs take one thread per
// 16-channel block, FP8 jobs one warp per row, as the single-job kernels do.
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

struct QuantJobs {
    QuantJob job[kMaxQuantJobs];
    int64_t block_start[kMaxQuantJobs + 1];
    int n;
};

CSA2_D float load_elem(const void *x, int dtype, int64_t i) {
    return dtype == CSA2_DTYPE_F32 ? __ldg(reinterpret_cast<const float *>(x) + i)
                                   : bf16_bits_to_f32(__ldg(reinterpret_cast<const uint16_t *>(x) + i));
}

__global__ void __launch_bounds__(kQuantThreads) quant_batch_kernel(const __grid_constant__ QuantJobs J) {
    int j = 0;
    while (j + 1 < J.n && (int64_t)blockIdx.x >= J.block_start[j + 1]) ++j;
    const QuantJob &q = J.job[j];
    const int64_t lb = (int64_t)blockIdx.x - J.block_start[j];
    if (q.fmt == CSA2_FMT_FP4_E2M1_E4M3S16) {
        const int nblk = q.dim >> 4;
        const int64_t t = lb * kQuantThreads + threadIdx.x;
        if (t >= q.rows * nblk) return;
        const int64_t r = t / nblk;
        const int b = (int)(t - r * nblk);
        const int64_t base = r * q.x_stride + b * 16;
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = load_elem(q.x, q.x_dtype, base + i);
        const int64_t d = q.dst_rows ? q.dst_rows[r] : r;
        quantize_block16(v, q.codes + d * q.code_stride + b * 8, q.scales + d * q.scale_stride + b);
    } else {
        const int lane = threadIdx.x & 31;
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
        blocks += s.fmt == CSA2_FMT_FP4_E2M1_E4M3S16 ? ceil_div(s.rows * (s.dim / 16), kQuantThreads)
                                                     : ceil_div(s.rows, kQuantThreads / 32);
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

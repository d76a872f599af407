// Sparse attention over the selected FP4 entries + the 8-bit window, CUDA-core version.
//
// [B] page "DeepSeek V4.1 Flash 如何靠压缩 KV 缓存实现小模型干翻大模型", section
// "CSA2：三层压缩一次吃满": every layer keeps its own query and window; entries carry an
// MLA-style latent shared by the heads (keys = values = the 512-wide latent).  Section
// "FP4 量化 + Bounded Replay": the window is the last 128 tokens at 8 bits.
//
// One CTA = (query row, 8 heads, split of the key list); one warp per head, 16 channels
// per lane, fp32 online softmax.  Splits are merged by log-sum-exp in attn_merge_kernel.
// This path handles head counts the tensor-core kernel does not take and serves as the
// second, independent GPU implementation in the tests.
#include "common.cuh"
#include "attn.cuh"

namespace csa2 {

constexpr int kSimtWarps = 8;

CSA2_D void load_key_row(const AttnArgs &a, int r, int x, int n_sel, float *dst) {
    // dst: 512 floats in shared memory, filled by the whole block
    const int b = r / a.T;
    if (x < n_sel) {
        const int32_t e = a.idx[(int64_t)r * a.K + x];
        if (e < 0) {
            for (int c = threadIdx.x; c < kLatent; c += blockDim.x) dst[c] = 0.0f;
            return;
        }
        const uint8_t *row = a.kv + (a.seq_start[b] + e) * a.kv_row_stride;
        for (int c = threadIdx.x * 2; c < kLatent; c += blockDim.x * 2) {
            const uint8_t byte = row[c >> 1];
            const float s = e4m3_to_f32(row[kLatent / 2 + (c >> 4)]);
            dst[c] = e2m1_to_f32(byte & 15u) * s;
            dst[c + 1] = e2m1_to_f32(byte >> 4) * s;
        }
    } else {
        const int slot = (a.swa_start ? a.swa_start[r] : 0) + (x - n_sel);
        const int64_t srow = (int64_t)b * a.swa_cap + slot;
        const float s = a.swa_scale[srow];
        const uint8_t *codes = a.swa_codes + srow * kLatent;
        for (int c = threadIdx.x; c < kLatent; c += blockDim.x) dst[c] = e4m3_to_f32(codes[c]) * s;
    }
}

__global__ void __launch_bounds__(kSimtWarps * 32)
attn_simt_kernel(AttnArgs a) {
    const int r = blockIdx.x;
    const int h = blockIdx.y * kSimtWarps + (threadIdx.x >> 5);
    const int split = blockIdx.z;
    const int lane = threadIdx.x & 31;
    __shared__ float vs[2][kLatent];

    const int n_sel = a.cnt ? a.cnt[r] : a.K;
    const int n_swa = a.swa_len[r];
    const int total = n_sel + n_swa;
    const int per = (total + a.splits - 1) / a.splits;
    const int x0 = split * per;
    const int x1 = min(total, x0 + per);

    float q[16];
    const uint16_t *qh = a.q + ((int64_t)r * a.H + h) * kLatent + lane * 16;
#pragma unroll
    for (int i = 0; i < 16; ++i) q[i] = bf16_bits_to_f32(qh[i]);
    float o[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i] = 0.0f;
    float m = -INFINITY, l = 0.0f;
    int buf = 0;

    for (int x = x0; x < x1; ++x) {
        const bool skip = x < n_sel && a.idx[(int64_t)r * a.K + x] < 0;
        if (skip) continue;                       // uniform across the block
        float *v = vs[buf];
        buf ^= 1;                                 // loaded rows alternate buffers
        load_key_row(a, r, x, n_sel, v);
        __syncthreads();
        float d = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) d = fmaf(q[i], v[lane * 16 + i], d);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
        const float z = d * a.softmax_scale;
        const float mn = fmaxf(m, z);
        const float alpha = expf(m - mn);        // m == -inf -> 0
        const float p = expf(z - mn);
        l = l * alpha + p;
#pragma unroll
        for (int i = 0; i < 16; ++i) o[i] = o[i] * alpha + p * v[lane * 16 + i];
        m = mn;
        // the double buffer lets the next row load start without a second barrier
    }
    __syncthreads();

    // partial: [row][h][split] -> (m, l, o[512])
    float *part = a.partials + (((int64_t)r * a.H + h) * a.splits + split) * (kLatent + 2);
    if (lane == 0) { part[0] = m; part[1] = l; }
#pragma unroll
    for (int i = 0; i < 16; ++i) part[2 + lane * 16 + i] = o[i];
}

// Merge split partials: one CTA of 128 threads per (row, head), 4 channels per thread.
__global__ void attn_merge_kernel(AttnArgs a) {
    const int r = blockIdx.x, h = blockIdx.y;
    const float *base = a.partials + ((int64_t)r * a.H + h) * a.splits * (kLatent + 2);
    float M = -INFINITY;
    for (int s = 0; s < a.splits; ++s) M = fmaxf(M, base[s * (kLatent + 2)]);
    float L = 0.0f;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int s = 0; s < a.splits; ++s) {
        const float *p = base + s * (kLatent + 2);
        const float ls = p[1];
        if (ls == 0.0f) continue;
        const float f = expf(p[0] - M);
        L += ls * f;
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i] += p[2 + threadIdx.x * 4 + i] * f;
    }
    const float inv = L > 0.0f ? 1.0f / L : 0.0f;
    const int64_t o = ((int64_t)r * a.H + h) * kLatent + threadIdx.x * 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float v = acc[i] * inv;
        if (a.out_dtype == CSA2_DTYPE_F32)
            reinterpret_cast<float *>(a.out)[o + i] = v;
        else
            reinterpret_cast<__nv_bfloat16 *>(a.out)[o + i] = __float2bfloat16_rn(v);
    }
    if (threadIdx.x == 0 && a.lse) a.lse[(int64_t)r * a.H + h] = L > 0.0f ? M + logf(L) : -INFINITY;
}

int simt_splits(int rows, int H, int K) {
    const int groups = rows * (H / kSimtWarps);
    int s = (4 * 148 + groups - 1) / groups;
    const int max_s = (K + CSA2_SWA_WINDOW + 63) / 64;
    if (s > max_s) s = max_s;
    if (s < 1) s = 1;
    return s;
}

size_t simt_workspace_bytes(int rows, int H, int K) {
    return (size_t)rows * H * simt_splits(rows, H, K) * (kLatent + 2) * sizeof(float) + 256;
}

cudaError_t launch_attn_simt(AttnArgs a, cudaStream_t st) {
    a.splits = simt_splits(a.rows, a.H, a.K);
    dim3 grid(a.rows, a.H / kSimtWarps, a.splits);
    attn_simt_kernel<<<grid, kSimtWarps * 32, 0, st>>>(a);
    attn_merge_kernel<<<dim3(a.rows, a.H), 128, 0, st>>>(a);
    note_launches(2);
    return cudaGetLastError();
}

}  // namespace csa2

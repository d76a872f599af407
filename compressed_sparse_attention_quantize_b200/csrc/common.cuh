// Device helpers shared by the CSA2 kernels: number formats, keys, launch checks.
//
// Formats ([B] = page "DeepSeek V4.1 Flash 如何靠压缩 KV 缓存实现小模型干翻大模型",
// section "FP4 量化 + Bounded Replay"): E2M1 codes with one E4M3 scale per 16 channels;
// the 8-bit sliding window uses E4M3 with a per-token fp32 scale.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "../../include/csa2.h"

#define CSA2_HD __host__ __device__ __forceinline__
#define CSA2_D __device__ __forceinline__

namespace csa2 {

constexpr int kLatent = 512;
constexpr int kKvRowBytes = kLatent / 2 + kLatent / 16;   // 288
constexpr int kIndexDim = 64;

// ---------------------------------------------------------------------------------------
// E4M3 ("fn": bias 7, max 448, no inf) and E2M1
// ---------------------------------------------------------------------------------------

// Decode an E4M3 code to fp32 (exact).
CSA2_D float e4m3_to_f32(uint32_t code) {
    uint32_t e = (code >> 3) & 15u, m = code & 7u;
    float mag;
    if (e == 0) {
        mag = (float)m * 0.001953125f;                  // m * 2^-9
    } else {
        mag = __uint_as_float(((e + 120u) << 23) | (m << 20));
    }
    return (code & 0x80u) ? -mag : mag;
}

// Round a non-negative fp32 magnitude to an E4M3 magnitude code, nearest-even,
// saturating finite values above 448 to 448 (code 0x7E).
CSA2_D uint32_t e4m3_code_mag_rne(float a) {
    if (!(a < 448.0f)) return 0x7Eu;                     // also catches +inf
    if (a < 0.015625f) {                                  // below 2^-6: subnormal grid 2^-9
        return (uint32_t)__float2int_rn(a * 512.0f);      // exact scaling; ties to even
    }
    uint32_t bits = __float_as_uint(a);
    uint32_t e = bits >> 23;                              // biased fp32 exponent
    uint32_t code = ((e - 120u) << 3) | ((bits >> 20) & 7u);
    uint32_t rem = bits & 0xFFFFFu;
    if (rem > 0x80000u || (rem == 0x80000u && (code & 1u))) code += 1u;   // carry ok
    return code > 0x7Eu ? 0x7Eu : code;
}

// E2M1 magnitude table (codes 0..7).
CSA2_D float e2m1_mag(uint32_t c) {
    // 0, .5, 1, 1.5, 2, 3, 4, 6 without a memory table
    uint32_t e = (c >> 1) & 3u, m = c & 1u;
    float base = e == 0 ? 0.0f : __uint_as_float((126u + e) << 23);   // 2^(e-1)
    return e == 0 ? 0.5f * (float)m : base * (1.0f + 0.5f * (float)m);
}

CSA2_D float e2m1_to_f32(uint32_t c) {
    float v = e2m1_mag(c & 7u);
    return (c & 8u) ? -v : v;
}

// ---------------------------------------------------------------------------------------
// bf16
// ---------------------------------------------------------------------------------------
CSA2_D float bf16_bits_to_f32(uint16_t b) { return __uint_as_float(((uint32_t)b) << 16); }

// ---------------------------------------------------------------------------------------
// Order-preserving key: larger float -> larger unsigned key (for radix selection).
// ---------------------------------------------------------------------------------------
CSA2_HD uint32_t float_key(float f) {
#ifdef __CUDA_ARCH__
    uint32_t u = __float_as_uint(f);
#else
    uint32_t u;
    memcpy(&u, &f, 4);
#endif
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

CSA2_HD int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Device-side error word: a bounded wait that expires, or a kernel that meets an argument
// outside the caller contract, stores a csa2_status here (the first one sticks).
__device__ int g_device_error = 0;

CSA2_D void raise_device_error(int status) { atomicCAS(&g_device_error, 0, status); }

// ---------------------------------------------------------------------------------------
// Per-device launch settings
// ---------------------------------------------------------------------------------------
// A kernel's dynamic shared-memory limit is a per-device setting (cudaFuncSetAttribute acts on
// the current device) and launch plans depend on the device's SM count.  Launchers keep such
// settings in tables indexed by device; a table entry is filled once per device under one
// mutex, so first calls may come from several host threads and several devices at once.
constexpr int kMaxDevices = 64;

inline std::mutex &settings_mutex() {
    static std::mutex m;
    return m;
}

// The calling thread's current device, or -1 when there is none (or its number is too large).
inline int current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
    return dev;
}

// Makes the current device's primary context current for driver-API calls of this thread (the
// runtime binds it lazily, and a thread whose first call encodes a tensor map has none bound
// yet: the encode then fails).  Once per thread and device.
inline cudaError_t bind_current_context() {
    thread_local int bound = -1;
    const int dev = current_device();
    if (dev < 0) return cudaErrorInvalidDevice;
    if (dev == bound) return cudaSuccess;
    const cudaError_t e = cudaSetDevice(dev);
    if (e == cudaSuccess) bound = dev;
    return e;
}

// SM count of the current device; 148 (a B200) when no device can be queried, so that plans
// can still be inspected on a host without a GPU.
inline int device_sm_count() {
    static std::atomic<int> cache[kMaxDevices];
    const int dev = current_device();
    if (dev < 0) return 148;
    int n = cache[dev].load(std::memory_order_acquire);
    if (n > 0) return n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev].store(n, std::memory_order_release);
    return n;
}

// Dynamic shared-memory limit of one kernel on every device it has been raised on.
struct SmemLimit {
    std::atomic<int> bytes[kMaxDevices];
};

// Raises `kernel`'s dynamic shared-memory limit on the current device to at least `bytes`
// (the limit only grows; a launch asks for its own size).
template <typename Kernel>
inline cudaError_t ensure_smem_limit(SmemLimit &lim, Kernel kernel, int bytes) {
    const int dev = current_device();
    if (dev < 0) return cudaErrorInvalidDevice;
    if (lim.bytes[dev].load(std::memory_order_acquire) >= bytes) return cudaSuccess;
    std::lock_guard<std::mutex> lock(settings_mutex());
    if (lim.bytes[dev].load(std::memory_order_relaxed) >= bytes) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    lim.bytes[dev].store(bytes, std::memory_order_release);
    return cudaSuccess;
}

// Host-side count of kernel launches (csa2_launch_count); every launcher adds its launches.
void note_launches(int n);

}  // namespace csa2

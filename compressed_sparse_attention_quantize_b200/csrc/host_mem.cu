// Page-locked host staging buffers on 2 MB pages (csa2_host_alloc / csa2_host_free).
//
// A host<->device copy translates every page of its host range; from ordinary page-locked
// memory (4 KB pages) a decode step's 13 MB of inputs are some 3200 translations, and on a
// B200 over PCIe those copies ran at 32 GB/s and slowed the kernels beside them.  The same
// copies from 2 MB pages ran at 50 GB/s with the kernels beside them unaffected.  The buffer
// is an anonymous mapping with transparent huge pages requested, zero-filled by the calling
// thread (first touch places the pages on its NUMA node), then registered with CUDA.
#include <sys/mman.h>

#include <cstring>
#include <mutex>
#include <unordered_map>

#include "common.cuh"
// cuda_status (records the CUDA error text for csa2_last_error_string) comes from api.cu,
// which the library's single translation unit includes first.

namespace csa2 {
namespace {

constexpr size_t kHugePage = size_t(2) << 20;
constexpr size_t kMaxHostBytes = size_t(1) << 40;

struct HostMapping {
    void *base;    // what mmap returned
    size_t len;    // mapped length
};

std::mutex g_host_mu;
std::unordered_map<uintptr_t, HostMapping> &host_mappings() {
    static std::unordered_map<uintptr_t, HostMapping> m;
    return m;
}

}  // namespace
}  // namespace csa2

extern "C" csa2_status csa2_host_alloc(size_t bytes, void **ptr) {
    using namespace csa2;
    if (!ptr) return CSA2_ERR_INVALID_ARG;
    *ptr = nullptr;
    if (bytes == 0 || bytes > kMaxHostBytes) return CSA2_ERR_SHAPE;
    const size_t len = (bytes + kHugePage - 1) / kHugePage * kHugePage;
    const size_t map_len = len + kHugePage;                 // room to align the start
    void *base = mmap(nullptr, map_len, PROT_READ | PROT_WRITE, MAP_PRIVATE | MAP_ANONYMOUS, -1, 0);
    if (base == MAP_FAILED) return CSA2_ERR_HOST;
    const uintptr_t b = reinterpret_cast<uintptr_t>(base);
    void *p = reinterpret_cast<void *>((b + kHugePage - 1) / kHugePage * kHugePage);
    (void)madvise(p, len, MADV_HUGEPAGE);                   // advisory: 4 KB pages otherwise
    std::memset(p, 0, len);
    const cudaError_t e = cudaHostRegister(p, len, cudaHostRegisterDefault);
    if (e != cudaSuccess) {
        munmap(base, map_len);
        return cuda_status(e);
    }
    {
        std::lock_guard<std::mutex> lock(g_host_mu);
        host_mappings()[reinterpret_cast<uintptr_t>(p)] = HostMapping{base, map_len};
    }
    *ptr = p;
    return CSA2_OK;
}

extern "C" csa2_status csa2_host_free(void *ptr) {
    using namespace csa2;
    if (!ptr) return CSA2_OK;
    HostMapping m;
    {
        std::lock_guard<std::mutex> lock(g_host_mu);
        auto it = host_mappings().find(reinterpret_cast<uintptr_t>(ptr));
        if (it == host_mappings().end()) return CSA2_ERR_INVALID_ARG;
        m = it->second;
        host_mappings().erase(it);
    }
    const cudaError_t e = cudaHostUnregister(ptr);
    munmap(m.base, m.len);
    return e == cudaSuccess ? CSA2_OK : cuda_status(e);
}

// csa2_sparse_attn_noalloc: the attention call for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at all: code running under an allocator that owns the
// whole device pool, a plug-in loaded into a host process that forbids device allocations
// after start-up, or code recorded once and replayed where a fresh allocation would break the
// replay.  csa2_sparse_attn needs a caller-supplied workspace for its split partials; this
// variant keeps that scratch in a fixed buffer inside the library instead, so the caller only
// passes inputs and outputs.
//
// The scratch is a file-scope __device__ array (kNoAllocScratchBytes); every device that loads
// the library holds it until the process exits.  On first use on a device the call looks up
// the array's device address with cudaGetSymbolAddress while that device is current and keeps
// it; that first call should therefore happen before any stream capture.  The split plan is
// the best one whose partials fit in the array (csa2_sparse_attn may pick more splits when its
// workspace allows); one split per row needs no partials, so a fitting plan always exists.
// All calls share the one array and each call overwrites what it reads (every split writes its
// full partial before the merge reads it), so nothing needs clearing; calls whose kernels
// overlap on the GPU (two streams, or two host threads) race on it.
#include <mutex>

namespace csa2 {

constexpr size_t kNoAllocScratchBytes = (size_t)20 << 20;    // 20 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device (looked up once per device).
csa2_status noalloc_scratch(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_status(e);
    if (dev < 0 || dev >= kMaxDevices) return CSA2_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_status(e);
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return CSA2_OK;
}
}  // namespace

}  // namespace csa2

extern "C" csa2_status csa2_sparse_attn_noalloc(const uint16_t *q, int B, int T, int H, int D,
                                                const uint8_t *kv, int64_t kv_row_stride,
                                                const int64_t *seq_start, const int32_t *n_entries,
                                                const int32_t *idx, const int32_t *cnt, int K,
                                                const uint8_t *swa_codes, const float *swa_scale,
                                                int swa_cap, const int32_t *swa_start,
                                                const int32_t *swa_len, float softmax_scale, void *out,
                                                int out_dtype, float *lse, void *stream) {
    using namespace csa2;
    const Range range("csa2_sparse_attn_noalloc");
    csa2_status s = check_attn_args(q, B, T, H, D, kv, kv_row_stride, seq_start, idx, K, swa_codes,
                                    swa_scale, swa_cap, swa_len, out, out_dtype);
    if (s != CSA2_OK) return s;
    AttnArgs a;
    a.rows = B * T;
    attn_plan(a.rows, H, K, a.hgroups, a.splits, a.keys_per_split, kNoAllocScratchBytes);
    if (attn_plan_workspace(a.rows, a.hgroups, a.splits) > kNoAllocScratchBytes) return CSA2_ERR_WORKSPACE;
    void *scratch = nullptr;
    s = noalloc_scratch(&scratch);
    if (s != CSA2_OK) return s;
    a.q = q; a.T = T; a.H = H; a.K = K;
    a.kv = kv; a.kv_row_stride = kv_row_stride; a.seq_start = seq_start; a.n_entries = n_entries;
    a.idx = idx; a.cnt = cnt;
    a.swa_codes = swa_codes; a.swa_scale = swa_scale; a.swa_cap = swa_cap;
    a.swa_start = swa_start; a.swa_len = swa_len;
    a.softmax_scale = softmax_scale; a.out = out; a.out_dtype = out_dtype; a.lse = lse;
    a.partials = reinterpret_cast<float *>(scratch);
    a.shard_lo = nullptr;
    a.shard_n = nullptr;
    return cuda_status(launch_attn_planned(a, reinterpret_cast<cudaStream_t>(stream)));
}

// Attention dispatch: every launch goes to the tcgen05 tensor-core kernel (heads padded to
// groups of 64).  The CUDA-core kernel in attn_simt.cu is kept only as an independent GPU
// implementation for the tests (csa2_debug_attn_simt).
#include "attn.cuh"

namespace csa2 {

size_t attn_workspace_bytes(int rows, int H, int K) {
    const size_t a = tc_workspace_bytes(rows, H, K);
    const size_t b = simt_workspace_bytes(rows, H, K);
    return a > b ? a : b;
}

cudaError_t launch_attn(AttnArgs a, cudaStream_t st) { return launch_attn_tc(a, st); }

}  // namespace csa2

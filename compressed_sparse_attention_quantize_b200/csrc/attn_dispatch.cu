// Attention dispatch: chooses the kernel for a launch.
#include "attn.cuh"

namespace csa2 {

size_t attn_workspace_bytes(int rows, int H, int K) { return simt_workspace_bytes(rows, H, K); }

cudaError_t launch_attn(AttnArgs a, cudaStream_t st) { return launch_attn_simt(a, st); }

}  // namespace csa2

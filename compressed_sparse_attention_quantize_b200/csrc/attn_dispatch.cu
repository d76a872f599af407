// Attention dispatch: every launch goes to the tcgen05 tensor-core kernel (heads in groups of 64).
#include "attn.cuh"

namespace csa2 {

size_t attn_workspace_bytes(int rows, int H, int K) { return tc_workspace_bytes(rows, H, K); }

void attn_plan(int rows, int H, int K, int &hgroups, int &splits, int &keys_per_split) {
    tc_plan(rows, H, K, hgroups, splits, keys_per_split);
}

cudaError_t launch_attn(AttnArgs a, cudaStream_t st) { return launch_attn_tc(a, st); }

}  // namespace csa2

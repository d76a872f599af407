// Single translation unit of the CSA2 library (keeps device symbols in one module).
#include "quant.cu"
#include "index_topk.cu"
#include "index_tc.cu"
#include "topk_cluster.cu"
#include "attn_tc.cu"
#include "attn_dispatch.cu"
#include "api.cu"
#include "noalloc.cu"

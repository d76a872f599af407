/*
 * csa2.h -- C ABI of the CSA2 (Compressed Sparse Attention 2) hot-path library for
 * NVIDIA B200 (sm_100a).
 *
 * Sources for what each call computes (web pages about the DeepSeek V4.1 Flash report):
 *   [A] "DeepSeek V4.1 Flash深度解析：KV缓存压缩437倍的技术路径"
 *   [B] "DeepSeek V4.1 Flash 如何靠压缩 KV 缓存实现小模型干翻大模型"
 *
 * Conventions shared by every call
 *  - All array arguments are DEVICE pointers owned by the caller; the library keeps no
 *    reference after the call returns and allocates nothing (scratch space is the
 *    caller's `workspace`, sized by the matching *_workspace_size call).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).  Every
 *    call only enqueues work on it: nothing synchronises the host, so results are valid
 *    once the caller synchronises the stream.  Calls keep no data between calls.  The
 *    library keeps launch settings per device (kernels' shared-memory limits, the SM
 *    count), set once per device under a lock, and the layer group keeps a side stream
 *    per host thread and device; calls may come from several host threads, on their own
 *    streams, for any of the process's devices (the current device at the call).
 *  - Arguments are validated before anything is launched; a call that returns an error
 *    has enqueued nothing.  Faults that happen on the device surface at the caller's
 *    next synchronisation, as for any CUDA kernel.
 *  - Strides are in BYTES for quantised buffers and in ELEMENTS for float/bf16 inputs.
 *  - bf16 values are passed as their uint16_t bit patterns.
 *  - Indices are int32.  Entry j of sequence b is row seq_start[b] + j of the packed
 *    caches.  A query row is r = b * T + t.
 */
#ifndef CSA2_H
#define CSA2_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define CSA2_API __attribute__((visibility("default")))
#else
#define CSA2_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum csa2_status {
    CSA2_OK = 0,
    CSA2_ERR_INVALID_ARG = 1,   /* a required pointer is NULL or an enum is unknown      */
    CSA2_ERR_SHAPE = 2,         /* a size is negative, zero where it must not be, or too big */
    CSA2_ERR_ALIGN = 3,         /* a pointer or stride breaks the 16-byte rule stated below */
    CSA2_ERR_UNSUPPORTED = 4,   /* valid but not implemented (e.g. latent width != 512)  */
    CSA2_ERR_CUDA = 5,          /* the CUDA runtime refused a launch                     */
    CSA2_ERR_TIMEOUT = 6,       /* a bounded device-side wait gave up (see csa2_device_error) */
    CSA2_ERR_WORKSPACE = 7,     /* workspace NULL or smaller than the size query returned */
    CSA2_ERR_HOST = 8           /* the operating system refused host memory              */
} csa2_status;

/* quantised formats */
#define CSA2_FMT_FP4_E2M1_E4M3S16 0   /* E2M1 codes, one E4M3 scale per 16 channels */
#define CSA2_FMT_FP8_E4M3_TOKEN   1   /* E4M3 codes, one fp32 scale per row (token) */
/* float element types */
#define CSA2_DTYPE_F32  0
#define CSA2_DTYPE_BF16 1
/* layer modes ([B] section "CSA2：三层压缩一次吃满") */
#define CSA2_MODE_FULL    0
#define CSA2_MODE_REINDEX 1
#define CSA2_MODE_REUSE   2

/* Limits of this library. */
#define CSA2_LATENT_DIM   512     /* main-KV latent width (attention)            */
#define CSA2_INDEX_DIM    64      /* indexer key / query width                   */
#define CSA2_MAX_INDEX_HEADS 16
#define CSA2_MAX_TOPK     4096
#define CSA2_MAX_POOL     32768
#define CSA2_MAX_HEADS    128     /* main query heads; a multiple of 16          */
#define CSA2_SWA_WINDOW   128     /* at most this many window tokens per query   */
#define CSA2_MAX_COMPRESS_RATIO 64 /* tokens per compressed entry                  */

/* Human-readable name of a status code (static string, never NULL). */
CSA2_API const char *csa2_status_string(csa2_status s);

/* Library ABI version (increments on any signature change). */
CSA2_API int csa2_version(void);

/* ------------------------------------------------------------------------------------
 * csa2_quantize_kv -- quantise-on-write of cache rows.
 *
 * fmt == CSA2_FMT_FP4_E2M1_E4M3S16 ([B] section "FP4 量化 + Bounded Replay": main KV is
 *   E2M1 with one E4M3 scale per 16 channels and no second-level scale; the indexer Q
 *   and K use the same FP4 format):  per block of 16 channels
 *       s = E4M3_rne_satfinite(amax / 6);  code_i = E2M1_rne_satfinite(x_i / s)
 *   with each quotient rounded once from its exact value; s == 0 gives all-zero codes;
 *   a negative value that rounds to zero is stored as -0 (code 8).  Two codes per byte,
 *   channel 2i in the low nibble.  Row r writes dim/2 bytes at codes + d*code_stride and
 *   dim/16 E4M3 bytes at scales + d*scale_stride, d = dst_rows ? dst_rows[r] : r.
 *   dim must be a multiple of 16.
 * fmt == CSA2_FMT_FP8_E4M3_TOKEN (the 8-bit sliding window, [A] section
 *   "压缩吸收注意力（二代）"):  per row s = amax / 448 rounded to fp32 and stored as a
 *   float at scales + d*scale_stride; code_i = E4M3_rne_satfinite(x_i / s) rounded once
 *   from the exact quotient; s == 0 gives all-zero codes.  dim bytes per row.
 *
 * x: rows x dim elements of x_dtype (CSA2_DTYPE_F32 or CSA2_DTYPE_BF16), row r at
 *    x + r*x_stride elements.  dst_rows: optional int64 [rows] destination rows (a cache
 *    position, or a ring slot of the window); NULL writes row r to row r.
 * Errors: INVALID_ARG (NULL x/codes/scales, unknown fmt or dtype), SHAPE (rows < 0,
 *   dim <= 0 or not a multiple of 16, dim > 65536, x_stride < dim), ALIGN (scales for
 *   FP8 not 4-byte aligned or scale_stride not a multiple of 4), CUDA.
 * rows == 0 is a no-op returning CSA2_OK (checked after fmt and x_dtype, before the rest).
 * ---------------------------------------------------------------------------------- */
CSA2_API csa2_status csa2_quantize_kv(int fmt, const void *x, int x_dtype, int64_t rows, int dim,
                             int64_t x_stride, uint8_t *codes, int64_t code_stride,
                             void *scales, int64_t scale_stride, const int64_t *dst_rows,
                             void *stream);

/* ------------------------------------------------------------------------------------
 * csa2_quantize_kv_batch -- several csa2_quantize_kv jobs in one kernel launch.
 *
 * A decode step writes to several caches at once (the new compressed entry, its indexer key,
 * the step token's window entry of every layer, the indexer queries); this call quantises all
 * of them in one launch.  Each job has the arguments, meaning and result of csa2_quantize_kv
 * ([B] section "FP4 量化 + Bounded Replay"; [A] section "压缩吸收注意力（二代）").  Jobs must
 * not write overlapping bytes (they run concurrently).
 * jobs: host array of n_jobs descriptors (read during the call only), 0 <= n_jobs <=
 *   CSA2_MAX_QUANT_JOBS; jobs with rows == 0 are skipped.
 * Errors: INVALID_ARG (jobs NULL with n_jobs > 0), SHAPE (n_jobs out of range), and any job's
 *   csa2_quantize_kv error (nothing is launched then), CUDA.
 * ---------------------------------------------------------------------------------- */
#define CSA2_MAX_QUANT_JOBS 16

typedef struct csa2_quant_job {
    int fmt;                     /* CSA2_FMT_*                                          */
    int x_dtype;                 /* CSA2_DTYPE_F32 or CSA2_DTYPE_BF16                   */
    const void *x;               /* rows x dim elements, row r at x + r*x_stride         */
    int64_t rows;
    int dim;
    int64_t x_stride;
    uint8_t *codes;              /* as csa2_quantize_kv                                 */
    int64_t code_stride;
    void *scales;
    int64_t scale_stride;
    const int64_t *dst_rows;     /* NULL or int64 [rows] destination rows               */
} csa2_quant_job;

CSA2_API csa2_status csa2_quantize_kv_batch(const csa2_quant_job *jobs, int n_jobs, void *stream);

/* ------------------------------------------------------------------------------------
 * csa2_compress_quantize_kv -- sequence compressor fused with the FP4 quantise-on-write.
 *
 * [B] section "CSA2：三层压缩一次吃满": along the sequence every m tokens are compressed into
 * one entry (V4's CSA does this with learned weights, which are not on the pages).  Here the
 * caller supplies the per-token weights:
 *     entry e = sum_{k<m} w[e][k] * x[m*e + k]
 * in fp32, tokens in order k = 0..m-1, each product and each sum rounded once (no fused
 * multiply-add); w == NULL takes the mean, w = 1/m (an IEEE fp32 quotient).  The entry is then
 * quantised exactly as csa2_quantize_kv with CSA2_FMT_FP4_E2M1_E4M3S16 and written to
 * destination row d = dst_rows ? dst_rows[e] : e (dim/2 code bytes at codes + d*code_stride,
 * dim/16 E4M3 scale bytes at scales + d*scale_stride).
 *
 * x: entries*m token rows of dim elements of x_dtype (CSA2_DTYPE_F32 or CSA2_DTYPE_BF16), token
 *    row t at x + t*x_stride elements.  w: NULL or fp32 [entries][w_stride] (w_stride >= m).
 * Errors: INVALID_ARG (NULL x/codes/scales, unknown dtype), SHAPE (entries < 0, m < 1 or
 *   m > CSA2_MAX_COMPRESS_RATIO, dim <= 0, not a multiple of 16 or > 65536, x_stride < dim,
 *   w_stride < m, code_stride < dim/2, scale_stride < dim/16), CUDA.
 * entries == 0 is a no-op returning CSA2_OK (checked after x_dtype).
 * ---------------------------------------------------------------------------------- */
CSA2_API csa2_status csa2_compress_quantize_kv(const void *x, int x_dtype, int64_t entries, int ratio,
                                      int dim, int64_t x_stride, const float *w,
                                      int64_t w_stride, uint8_t *codes, int64_t code_stride,
                                      uint8_t *scales, int64_t scale_stride,
                                      const int64_t *dst_rows, void *stream);

/* ------------------------------------------------------------------------------------
 * csa2_index_topk -- indexer scoring + top-K block selection for Full and Reindex layers.
 *
 * Score ([B] section "为什么 KV 缓存成了新瓶颈？" names the DSA indexer; [B] section
 * "FP4 量化 + Bounded Replay" makes its Q and K FP4):  for query row r and entry j
 *     I[r, j] = sum_h w[r,h] * ReLU(q[r,h] . k[j])
 * with q, k the dequantised FP4 vectors (64 channels), computed in fp32: each 16-channel
 * block's partial is exact, blocks are added left to right, heads are accumulated left to
 * right as acc = acc + w*relu(dot) without fused multiply-add, and 0 is returned as +0.
 *
 * Selection ([A] section "压缩吸收注意力（二代）": the first layer picks 2048 blocks and
 * builds a candidate pool that later layers search):  the entries visible to row r are
 * ordered by (score descending, entry index ascending); the first min(K, n) are written to
 * out_idx[r][0..K) in ascending index order, padded with -1, and their number to
 * out_cnt[r].
 *   mode == CSA2_MODE_FULL: visible entries are j < n_vis(r), n_vis = n_entries[b] when
 *     q_pos is NULL (decode) else min(n_entries[b], (q_pos[r] + 1) / 4) (entry j covers
 *     tokens 4j..4j+3).  When P > 0 the first min(P, n) of the same order (the pool,
 *     which contains the top-K) go to out_pool[r][0..P) ascending, padded with -1, and
 *     their number to out_pool_len[r].
 *   mode == CSA2_MODE_REINDEX: only the entries listed in pool[r][0..pool_len[r]) (row
 *     stride P_in, ascending) are scored with this layer's own q and w; P must be 0.
 *
 * Layouts: q_codes [B*T][H_I][32] u8, q_scales [B*T][H_I][4] u8 (E4M3), w [B*T][H_I] f32;
 *   key codes of entry row e at k_codes + e*k_code_stride (32 bytes), its 4 E4M3 scales at
 *   k_scales + e*k_scale_stride; seq_start int64 [B]; n_entries int32 [B]; q_pos int32
 *   [B*T] or NULL; pool int32 [B*T][P_in]; pool_len int32 [B*T].
 *   max_n: an upper bound of n_entries[b] over the batch (sizes the launch; the device
 *   values are not read back).
 * Limits: 1 <= H_I <= CSA2_MAX_INDEX_HEADS, 1 <= K <= CSA2_MAX_TOPK, 0 <= P <=
 *   CSA2_MAX_POOL, P_in <= CSA2_MAX_POOL, max_n <= 2^31-1.
 * Workspace: csa2_index_topk_workspace_size(mode, B*T, max_n, K, P (or P_in), &bytes).
 * Errors: INVALID_ARG, SHAPE, ALIGN (k_codes or k_code_stride not 16-byte aligned),
 *   WORKSPACE, CUDA.
 * ---------------------------------------------------------------------------------- */
CSA2_API csa2_status csa2_index_topk_workspace_size(int mode, int rows, int64_t max_n, int K, int P,
                                           size_t *bytes);

CSA2_API csa2_status csa2_index_topk(int mode, const uint8_t *q_codes, const uint8_t *q_scales,
                            const float *w, int B, int T, int H_I,
                            const uint8_t *k_codes, int64_t k_code_stride,
                            const uint8_t *k_scales, int64_t k_scale_stride,
                            const int64_t *seq_start, const int32_t *n_entries, int64_t max_n,
                            const int32_t *q_pos,
                            const int32_t *pool, const int32_t *pool_len, int P_in,
                            int K, int32_t *out_idx, int32_t *out_cnt,
                            int P, int32_t *out_pool, int32_t *out_pool_len,
                            void *workspace, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------------------
 * csa2_pool_extend -- Reindex candidates between pool refreshes ([A] section
 * "压缩吸收注意力（二代）": later layers search the first layer's candidate pool; this call keeps
 * such a pool useful as entries are written after it was built).  For query row r (b = r / T):
 *     out_pool[r] = pool[r][0 .. pool_len[r]) followed by ids n_ref[b] .. n_vis(r) - 1
 * with n_vis(r) as in csa2_index_topk (n_entries[b], or min(n_entries[b], (q_pos[r] + 1) / 4)
 * when q_pos is given); out_len[r] = the count.  The kept pool's ids lie below n_ref[b], so the
 * list stays ascending.  Rows with more than P_out candidates keep the first P_out and the
 * device error word becomes CSA2_ERR_SHAPE (csa2_device_error).
 *   pool int32 [B*T][P_in], pool_len / out_len int32 [B*T], n_ref / n_entries int32 [B],
 *   q_pos int32 [B*T] or NULL, out_pool int32 [B*T][P_out] (may not overlap pool).
 * Errors: INVALID_ARG (NULL pool, pool_len, n_ref, n_entries, out_pool or out_len), SHAPE
 *   (B or T <= 0, P_in < 0, P_out < 1 or P_out > CSA2_MAX_POOL), CUDA.
 * ---------------------------------------------------------------------------------- */
CSA2_API csa2_status csa2_pool_extend(const int32_t *pool, const int32_t *pool_len, int P_in,
                                      const int32_t *n_ref, const int32_t *n_entries,
                                      const int32_t *q_pos, int B, int T, int P_out,
                                      int32_t *out_pool, int32_t *out_len, void *stream);

/* ------------------------------------------------------------------------------------
 * csa2_sparse_attn -- attention of each query row over its selected compressed entries
 * merged with its own 8-bit sliding window.
 *
 * [B] section "CSA2：三层压缩一次吃满": entries carry an MLA-style latent shared by all
 * heads, so keys = values = the dequantised 512-wide latent; every layer keeps its own
 * query and its own window.  [B] section "FP4 量化 + Bounded Replay": the window is
 * truncated to the last 128 tokens.  For row r and head h, with X = {selected entries}
 * followed by {window tokens}:
 *     z_x = softmax_scale * (q[r,h] . v_x);   out[r,h] = sum_x softmax(z)_x v_x
 * one joint softmax over X (the window is merged by the log-sum-exp of the two parts);
 * lse[r,h] = log(sum_x exp(z_x)) (natural log; -inf and out = 0 when X is empty).
 *
 * Layouts: q bf16 [B*T][H][D]; main entry e at kv + e*kv_row_stride holds D/2 bytes of
 *   E2M1 codes followed by D/16 E4M3 scales (288 bytes for D = 512); entry ids are
 *   relative to seq_start[b]; n_entries int32 [B] (entries of each sequence) or NULL;
 *   idx int32 [B*T][K] (-1 = empty slot, ignored); cnt int32 [B*T] or NULL (number of
 *   leading ids to read, 0 <= cnt <= K; NULL = scan all K);
 *   swa_codes u8 [B][swa_cap][D] (E4M3), swa_scale f32 [B][swa_cap]; row r uses slots
 *   swa_start[r] .. swa_start[r]+swa_len[r]-1 of its sequence (swa_start NULL = 0);
 *   out [B*T][H][D] of out_dtype (CSA2_DTYPE_F32 or CSA2_DTYPE_BF16); lse f32 [B*T][H]
 *   or NULL.
 * Caller contract: every non-negative id in idx names an entry of its own sequence (id <
 *   n_entries[b], so the row lies inside kv), 0 <= swa_len[r] <= CSA2_SWA_WINDOW and
 *   0 <= swa_start[r], swa_start[r] + swa_len[r] <= swa_cap.  csa2_index_topk's outputs
 *   always satisfy the first condition.  The kernel checks it as it reads: an id at or
 *   above n_entries[b] (checked only when n_entries is given) or a window slot outside
 *   [0, swa_cap) is skipped and the device error word becomes CSA2_ERR_INVALID_ARG; a cnt
 *   outside [0, K] or a swa_len outside [0, CSA2_SWA_WINDOW] is clamped and the word
 *   becomes CSA2_ERR_SHAPE (read and clear it with csa2_device_error).  The row of such a
 *   call is not meaningful, but nothing outside the caller's buffers is read.
 * Limits: D == 512; H a multiple of 16, 16 <= H <= CSA2_MAX_HEADS; 1 <= K <=
 *   CSA2_MAX_TOPK; swa_len <= CSA2_SWA_WINDOW; q, kv, kv_row_stride, swa_codes, out and
 *   workspace 16-byte aligned.
 * Workspace: csa2_sparse_attn_workspace_size(B*T, H, K, &bytes).
 * Errors: INVALID_ARG, SHAPE, ALIGN, UNSUPPORTED (D != 512), WORKSPACE, CUDA.
 * ---------------------------------------------------------------------------------- */
CSA2_API csa2_status csa2_sparse_attn_workspace_size(int rows, int H, int K, size_t *bytes);

/* ------------------------------------------------------------------------------------
 * csa2_sparse_attn_plan -- how csa2_sparse_attn splits a launch of `rows` query rows,
 * H heads and top-K on the current device (read-only; launches nothing).
 *   hgroups: head groups of 64 (one CTA each per row and split);
 *   splits: key splits per (row, head group), merged by log-sum-exp when > 1;
 *   keys_per_split: keys per split, a multiple of 128; the last split takes the rest of
 *     the K + CSA2_SWA_WINDOW keys.
 * The plan minimises an estimated finish time over the device's SMs (148 assumed when no
 * device is visible).  The workspace holds one partial of 131,584 bytes per (row, head
 * group, split) when splits > 1.
 * Errors: INVALID_ARG (NULL outputs), SHAPE (rows, H or K <= 0).
 * ---------------------------------------------------------------------------------- */
CSA2_API csa2_status csa2_sparse_attn_plan(int rows, int H, int K, int *hgroups, int *splits,
                                           int *keys_per_split);

CSA2_API csa2_status csa2_sparse_attn(const uint16_t *q, int B, int T, int H, int D,
                             const uint8_t *kv, int64_t kv_row_stride, const int64_t *seq_start,
                             const int32_t *n_entries, const int32_t *idx, const int32_t *cnt, int K,
                             const uint8_t *swa_codes, const float *swa_scale, int swa_cap,
                             const int32_t *swa_start, const int32_t *swa_len,
                             float softmax_scale, void *out, int out_dtype, float *lse,
                             void *workspace, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------------------
 * csa2_sparse_attn_noalloc -- csa2_sparse_attn for callers that cannot allocate device memory.
 *
 * No counterpart in the pages: this is an interface convenience, not part of the method.
 * Same arguments, layouts, limits and result as csa2_sparse_attn, without `workspace`: the
 * split partials go to a fixed 20 MiB scratch array inside the library (a static device
 * array that every device loading the library holds until the process exits).  Callers that
 * cannot call cudaMalloc -- an allocator that owns the whole device pool, a host process that
 * forbids device allocations after start-up -- use this call instead.
 *   - The first call on a device looks up the array's address (cudaGetSymbolAddress) with
 *     that device current; make that first call before any stream capture.
 *   - The split plan is the best one whose partials (131,584 bytes each) fit in the array;
 *     it may use fewer key splits than csa2_sparse_attn would.  One split per query row
 *     needs no partials, so every valid shape runs; CSA2_ERR_WORKSPACE would mean a plan
 *     that does not fit, which cannot happen for arguments that pass validation.
 *   - All calls share the array, and each call fully rewrites what it reads, so nothing needs
 *     clearing; calls whose kernels overlap on the GPU (other streams or host threads) race.
 *   - Otherwise the errors of csa2_sparse_attn.
 * ---------------------------------------------------------------------------------- */
CSA2_API csa2_status csa2_sparse_attn_noalloc(const uint16_t *q, int B, int T, int H, int D,
                                              const uint8_t *kv, int64_t kv_row_stride,
                                              const int64_t *seq_start, const int32_t *n_entries,
                                              const int32_t *idx,
                                              const int32_t *cnt, int K, const uint8_t *swa_codes,
                                              const float *swa_scale, int swa_cap,
                                              const int32_t *swa_start, const int32_t *swa_len,
                                              float softmax_scale, void *out, int out_dtype,
                                              float *lse, void *stream);

/* ------------------------------------------------------------------------------------
 * csa2_layer_group -- one group of CSA2 layers in order ([B] section
 * "CSA2：三层压缩一次吃满"; [A] section "压缩吸收注意力（二代）": in a group of six only
 * the first is Full and the rest Reuse).
 *   FULL    : csa2_index_topk(FULL) with the layer's own indexer query; when any later
 *             layer is REINDEX the Full layer also emits the pool of size P.
 *   REINDEX : re-scores the pool of the group's most recent Full layer with the layer's
 *             own indexer query and takes top-K from it.
 *   REUSE   : takes the preceding layer's selection as is (no indexer work).
 * Every layer then runs csa2_sparse_attn with its own main query and its own window over
 * the shared main KV.  Layers run in order on `stream`.
 * Per-layer events (optional, cudaEvent_t passed as void*, owned by the caller): the work of
 * layer l waits on `ready_event` (cudaStreamWaitEvent), e.g. the copy of that layer's indexer
 * query on another stream; its attention also waits on `attn_ready_event`, e.g. the copy of its
 * main query, so that the indexer can run while that copy is still in flight; `done_event` is
 * recorded once layer l's work is queued, e.g. to start reading its output back while later
 * layers run.  NULL skips any of them.
 * Rejected (INVALID_ARG): a REUSE or REINDEX layer before any FULL layer; REINDEX with
 * P == 0.
 * ---------------------------------------------------------------------------------- */
typedef struct csa2_group_desc {
    int B, T, H, D, H_I, K, P;
    const uint8_t *kv;           int64_t kv_row_stride;     /* main KV (shared)        */
    const uint8_t *k_codes;      int64_t k_code_stride;     /* indexer keys (shared)   */
    const uint8_t *k_scales;     int64_t k_scale_stride;
    const int64_t *seq_start;    const int32_t *n_entries;  int64_t max_n;
    const int32_t *q_pos;        /* NULL = decode (all entries visible)                */
    int swa_cap;                 const int32_t *swa_start;  const int32_t *swa_len;
    float softmax_scale;         int out_dtype;
    /* Candidate pool kept across decode steps (optional; pool_keep == NULL rebuilds it in every
     * call).  [A] section "压缩吸收注意力（二代）" has the first layer's scan build a pool that the
     * later layers search; how a pool is kept as the context grows is this library's own rule:
     *   refresh != 0: the Full layer rebuilds the pool -- top-min(P, n) of its order -- into
     *                 pool_keep [B*T][P] / pool_keep_len [B*T] and records pool_keep_n[b] =
     *                 n_entries[b] (the entry count at the rebuild);
     *   refresh == 0: the pool is kept, and the Reindex layers search it followed by the entries
     *                 written since (ids pool_keep_n[b] .. n - 1, see csa2_pool_extend), at most
     *                 max_new per sequence (P + max_new <= CSA2_MAX_POOL).
     * The caller owns the three arrays and calls with refresh != 0 first and every R steps.  The
     * Full layer's own top-K is always taken over every visible entry.  Ignored without REINDEX
     * layers.  Decode only: INVALID_ARG with q_pos != NULL or a NULL pool_keep_len /
     * pool_keep_n; SHAPE when max_new < 0 or P + max_new > CSA2_MAX_POOL; a step that has
     * written more than max_new entries since the refresh sets CSA2_ERR_SHAPE in the device
     * error word and searches the first P + max_new candidates. */
    int32_t *pool_keep;          int32_t *pool_keep_len;    int32_t *pool_keep_n;
    int refresh;                 int max_new;
} csa2_group_desc;

typedef struct csa2_layer_desc {
    int mode;                    /* CSA2_MODE_*                                        */
    const uint16_t *q;           /* main query, bf16 [B*T][H][D]                       */
    const uint8_t *iq_codes;     /* indexer query [B*T][H_I][32] (FULL / REINDEX)      */
    const uint8_t *iq_scales;    /* [B*T][H_I][4]                                      */
    const float *iw;             /* indexer head weights [B*T][H_I]                    */
    const uint8_t *swa_codes;    /* this layer's window [B][swa_cap][D]                */
    const float *swa_scale;      /* [B][swa_cap]                                       */
    void *out;                   /* [B*T][H][D] of out_dtype                           */
    float *lse;                  /* [B*T][H] or NULL                                   */
    int32_t *idx_out;            /* optional copy of this layer's selection [B*T][K]   */
    void *ready_event;           /* cudaEvent_t or NULL: the layer's kernels wait for it */
    void *done_event;            /* cudaEvent_t or NULL: recorded after the layer's work */
    void *attn_ready_event;      /* cudaEvent_t or NULL: the layer's attention (not its
                                    indexer) also waits for it, e.g. the copy of q        */
} csa2_layer_desc;

CSA2_API csa2_status csa2_layer_group_workspace_size(const csa2_group_desc *g,
                                            const csa2_layer_desc *layers, int n_layers,
                                            size_t *bytes);

CSA2_API csa2_status csa2_layer_group(const csa2_group_desc *g, const csa2_layer_desc *layers,
                             int n_layers, void *workspace, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------------------
 * Context parallelism: one long sequence whose compressed entries are split into
 * consecutive shards, one per GPU ([A] section "压缩吸收注意力（二代）": the top 2048 blocks
 * of the whole context, score descending, entry index ascending on ties; [B] section
 * "CSA2：三层压缩一次吃满": one joint softmax over the selection).  Each GPU runs
 * csa2_index_topk_scored and csa2_sparse_attn on its own shard; the caller all-gathers the
 * results (NCCL) and merges them with the two calls below.  The global top-K lies inside the
 * union of the shards' top-K lists, so the merged selection equals the single-GPU one.
 *
 * csa2_index_topk_scored -- csa2_index_topk in FULL mode (no pool) that also writes the
 *   fp32 score of every selected entry: out_scores [B*T][K], -inf in padded slots.  Same
 *   arguments, workspace and errors as csa2_index_topk; INVALID_ARG if out_scores is NULL.
 * ---------------------------------------------------------------------------------- */
CSA2_API csa2_status csa2_index_topk_scored(const uint8_t *q_codes, const uint8_t *q_scales,
                                   const float *w, int B, int T, int H_I,
                                   const uint8_t *k_codes, int64_t k_code_stride,
                                   const uint8_t *k_scales, int64_t k_scale_stride,
                                   const int64_t *seq_start, const int32_t *n_entries,
                                   int64_t max_n, const int32_t *q_pos, int K,
                                   int32_t *out_idx, int32_t *out_cnt, float *out_scores,
                                   void *workspace, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------------------
 * csa2_topk_merge_shards -- top-K of the union of G shards' scored candidate lists.
 *   scores, ids: [G][rows][K_in]; shard g's list for row r holds cnt[g*rows + r] valid
 *   candidates first (ids ascending).  id_offset: [G][rows] int64 added to shard g's ids
 *   (the shard's first global entry; NULL adds nothing).  After the offset, shard g's ids
 *   must all lie below shard g+1's.
 *   Output as csa2_index_topk: the selected ids ascending in out_idx [rows][K], -1 padded,
 *   out_cnt [rows] (nullable) = min(K, candidates).  Order: score descending, id ascending.
 *   workspace: csa2_topk_merge_shards_workspace_size(G, rows, K_in) bytes.
 * Errors: INVALID_ARG (NULL scores/ids/cnt/out_idx), SHAPE (G, rows, K_in <= 0, K < 1 or
 *   K > CSA2_MAX_TOPK), UNSUPPORTED (G*K_in above the selection's 262144 candidates),
 *   WORKSPACE, CUDA.
 * ---------------------------------------------------------------------------------- */
CSA2_API csa2_status csa2_topk_merge_shards_workspace_size(int G, int rows, int K_in, size_t *bytes);
CSA2_API csa2_status csa2_topk_merge_shards(const float *scores, const int32_t *ids,
                                   const int64_t *id_offset, const int32_t *cnt, int G, int rows,
                                   int K_in, int K,
                                   int32_t *out_idx, int32_t *out_cnt, void *workspace,
                                   size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------------------
 * csa2_sparse_attn_shard -- csa2_sparse_attn over one shard's part of the selection: idx
 *   holds GLOBAL entry numbers; entry e of sequence b is used only if it lies in the shard,
 *   shard_lo[b] <= e < shard_lo[b] + shard_n[b], and is read from this GPU's cache row
 *   seq_start[b] + e - shard_lo[b].  The window keys are taken as given (pass swa_len = 0 on
 *   every shard but the one that holds the window).  Output fp32 out [B*T][H][D] and the
 *   natural-log lse [B*T][H] (required): the inputs of csa2_attn_merge_shards.  Other
 *   arguments, workspace and errors as csa2_sparse_attn; INVALID_ARG if shard_lo, shard_n or
 *   lse is NULL.
 * ---------------------------------------------------------------------------------- */
CSA2_API csa2_status csa2_sparse_attn_shard(const uint16_t *q, int B, int T, int H, int D,
                                   const uint8_t *kv, int64_t kv_row_stride,
                                   const int64_t *seq_start, const int64_t *shard_lo,
                                   const int32_t *shard_n, const int32_t *idx, const int32_t *cnt,
                                   int K, const uint8_t *swa_codes, const float *swa_scale,
                                   int swa_cap, const int32_t *swa_start, const int32_t *swa_len,
                                   float softmax_scale, float *out, float *lse, void *workspace,
                                   size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------------------
 * csa2_attn_merge_shards -- log-sum-exp merge of G shards' attention results (each the
 *   fp32 output and natural-log LSE of csa2_sparse_attn over that shard's part of the key
 *   set): out = sum_g exp(lse_g - M) out_g / L, lse = M + ln L, M = max_g lse_g,
 *   L = sum_g exp(lse_g - M), shards added in order g = 0..G-1.  A shard with lse = -inf
 *   (no keys) contributes nothing.
 *   outs: fp32 [G][rows][H][D] (16-byte aligned); lses: [G][rows][H]; out: [rows][H][D] of
 *   out_dtype (16-byte aligned); lse: [rows][H] or NULL.
 * Errors: INVALID_ARG (NULL outs/lses/out, unknown dtype), SHAPE (G, rows, H, D <= 0, D not a
 *   multiple of 4), ALIGN, CUDA.
 * ---------------------------------------------------------------------------------- */
CSA2_API csa2_status csa2_attn_merge_shards(const float *outs, const float *lses, int G, int rows,
                                   int H, int D, void *out, int out_dtype, float *lse,
                                   void *stream);

/* ------------------------------------------------------------------------------------
 * csa2_device_error -- reads (and clears) the library's device-side error word for the
 * current device: 0 when nothing was recorded since the last call, otherwise the first
 * csa2_status code a kernel recorded: CSA2_ERR_TIMEOUT (a bounded wait expired),
 * CSA2_ERR_INVALID_ARG or CSA2_ERR_SHAPE (csa2_sparse_attn met an id, window slot or count
 * outside its caller contract).  Synchronises `stream` first.
 * ---------------------------------------------------------------------------------- */
CSA2_API csa2_status csa2_device_error(void *stream);

/* ------------------------------------------------------------------------------------
 * csa2_selftest_bounded_wait -- failure-detection self-test of the bounded device-side wait
 * that the pipelined kernels use (no page defines it; it checks this library's own error
 * path).  Launches one CTA on `stream`: a producer thread arrives on an mbarrier that a
 * consumer thread waits for, then waits for the consumer's reply.  skip_arrival != 0 makes the
 * producer skip its arrival, so the consumer's wait gives up after 2^10 polls, the device
 * error word becomes CSA2_ERR_TIMEOUT (read it with csa2_device_error) and the kernel
 * exits.  Nothing traps or faults, and the context stays usable.  With skip_arrival == 0 the
 * handshake completes and the error word is untouched.
 * Errors: CUDA (launch failure).
 * ---------------------------------------------------------------------------------- */
CSA2_API csa2_status csa2_selftest_bounded_wait(int skip_arrival, void *stream);

/* ------------------------------------------------------------------------------------
 * csa2_last_error_string -- description of the last CUDA runtime error a call of this
 * library met on the calling host thread (the reason behind CSA2_ERR_CUDA), or "" if none.
 * ---------------------------------------------------------------------------------- */
CSA2_API const char *csa2_last_error_string(void);

/* ------------------------------------------------------------------------------------
 * csa2_launch_count -- number of kernels this library has launched in this process
 * (all devices, all streams) since it was loaded.  A diagnostic for benchmarks.
 * ---------------------------------------------------------------------------------- */
CSA2_API uint64_t csa2_launch_count(void);

/* ------------------------------------------------------------------------------------
 * csa2_host_alloc / csa2_host_free -- page-locked host staging buffers for the inputs and
 * outputs a decode step copies between host and device (no page defines them; they serve
 * the end-to-end path).  csa2_host_alloc maps `bytes` rounded up to a multiple of 2 MB,
 * 2 MB-aligned, asks the kernel for transparent huge pages on it (where they are off the
 * buffer is still valid, on 4 KB pages), writes zeros to every byte from the calling thread
 * (so the pages sit on that thread's NUMA node under the default policy), page-locks and
 * registers it with CUDA (cudaHostRegister, default flags: usable by asynchronous copies on
 * every device and in CUDA graphs), and stores its address in *ptr.  Copies from 2 MB pages
 * need 512 times fewer address translations than from 4 KB pages: on a B200 over PCIe they
 * ran faster (50 against 32 GB/s for 2 MB copies) and slowed kernels running beside them less.
 * The caller owns the buffer until csa2_host_free(ptr), which unregisters and unmaps it.
 * Errors: INVALID_ARG (ptr NULL; csa2_host_free of an address csa2_host_alloc did not
 * return, or returned and already freed), SHAPE (bytes == 0 or above 2^40), HOST (the mapping
 * failed), CUDA (registration failed; nothing stays allocated).  csa2_host_free(NULL) is a
 * no-op returning OK.  Thread-safe.
 * ---------------------------------------------------------------------------------- */
CSA2_API csa2_status csa2_host_alloc(size_t bytes, void **ptr);
CSA2_API csa2_status csa2_host_free(void *ptr);

#ifdef __cplusplus
}
#endif
#endif /* CSA2_H */

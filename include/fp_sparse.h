/*
 * fp_sparse.h -- C ABI of the B200 (sm_100a) dynamic block-sparse prefill
 * attention library (Flex-Prefill method).
 *
 * The operation is defined by two web articles on FAST-Prefill:
 *   "FPGA24成果：FAST-Prefill稀疏注意力加速器，长上下文LLM推理提速2.5倍"
 *     section 1.1  causal attention softmax(Q K^T / sqrt(d)) V
 *     section 1.2  b x b block partition; per-head vertical-slash or
 *                  query-aware pattern chosen by a Jensen-Shannon divergence
 *     section 2.1  the last query block scores every key block (softmax,
 *                  block pooling)
 *     section 3.1  vertical and slash accumulators; blocks added until the
 *                  cumulative score reaches gamma
 *     section 3.3  INT8 multiply with INT32 accumulation
 *   "FPGA加速动态稀疏注意力技术解析与优化"
 *     section 1.1  representative last query block, JSD pattern decision with
 *                  threshold tau (usually 0.1), block-level index generation
 *
 * Conventions (all arguments): batch 1, tensors head-major and contiguous,
 * q[Hq][S][d], k[Hkv][S][d], v[Hkv][S][d], out[Hq][S][d]; query head h reads
 * KV head h / (Hq/Hkv).  Supported: d = 128, b in {64, 128, 256}, any S >= 1
 * with n = ceil(S/b) <= 1024 blocks, Hq a multiple of Hkv.  When b does not divide
 * S the last block is partial: it holds the S - (n-1)b rows (n-1)b .. S-1,
 * the statistics of steps 1-2 below average over those rows and every block
 * mean is taken over the rows the block actually has (the articles only
 * treat whole blocks; this is the reading that keeps every other step
 * unchanged).  Device pointers must be 16-byte aligned.  All calls are asynchronous on `stream` (a cudaStream_t,
 * NULL = legacy default stream) unless stated; the caller keeps every buffer
 * alive until the stream has passed the call.
 *
 * Batches: B sequences of equal length S are one call with the tensors
 * stacked sequence-major, i.e. q[B*Hq][S][d], k and v [B*Hkv][S][d], passing
 * B*Hq and B*Hkv as the head counts (query head b*Hq + h then reads KV head
 * b*Hkv + h/(Hq/Hkv), as it should).  Every step works per head, so the result
 * equals B separate calls.
 *
 * Errors: functions return FP_OK (0) or an FP_ERR_* code; nothing aborts the
 * process.  Argument errors are detected on the host before any launch.  A
 * device-side bounded wait that gives up records FP_ERR_TIMEOUT in a sticky
 * per-device word read by fp_get_device_error().
 */
#ifndef FP_SPARSE_H
#define FP_SPARSE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
    FP_OK = 0,
    FP_ERR_ARG = 1,      /* invalid argument (shape, pointer, alignment, range) */
    FP_ERR_CUDA = 2,     /* a CUDA runtime/driver call failed (launch, copy, alloc) */
    FP_ERR_TIMEOUT = 3,  /* a device-side bounded wait gave up */
    FP_ERR_STATE = 4     /* index used before it was built, or built for other shapes */
};

enum { FP_QK_BF16 = 0, FP_QK_INT8 = 1 };        /* element type of q and k */
enum { FP_PATTERN_VS = 0, FP_PATTERN_QA = 1 };  /* vertical-slash / query-aware */

/* Opaque, library-owned index: per-(head, query block) KV-block lists plus the
 * per-head statistics and pattern, resident in device memory. */
typedef struct fp_index fp_index;

/* Allocates an index and its device workspace for one layer shape on the
 * current CUDA device.  Sizes: S tokens, Hq query heads, Hkv KV heads, head
 * dim d, block size b (see the supported set above).  *out receives the
 * handle (NULL on error).  The workspace holds the worst case (gamma = 1),
 * Hq*n(n+1)/2 block indices, so building never allocates.
 * Returns FP_ERR_ARG for unsupported shapes, FP_ERR_CUDA if allocation fails. */
int fp_index_create(int S, int Hq, int Hkv, int d, int b, fp_index **out);

/* Frees an index and its workspace (NULL is ignored).  The workspace is
 * released in stream order once the index's most recent fp_build_index or
 * fp_sparse_attn call has finished on its stream; the call does not wait for
 * the device or for other streams (work of earlier calls still running on
 * other streams must be ordered before that last call by the caller, as for
 * any buffer it frees). */
void fp_index_free(fp_index *idx);

/* Sparse-index generation (articles above: section 2.1 and 3.1 of the
 * first; section 1.1 of the second).  For every query head h:
 *   1. the last query block (rows (n-1)b..S-1) is scored against every key
 *      j <= p and softmax-normalised per row;
 *   2. vertical vhat[c] and slash shat[o] statistics pool those probabilities
 *      over key blocks and over diagonal offset blocks floor((p-j)/b);
 *   3. P_est = softmax_c(qbar_{n-1} . kbar_c / sqrt(d)) from block means;
 *      JSD(vhat, P_est) < tau selects query-aware, otherwise vertical-slash;
 *   4. for every query block r: block scores over c <= r (VS: vhat[c] +
 *      shat[r-c]; QA: softmax of qbar_r . kbar_c / sqrt(d)), normalised; the
 *      diagonal block is kept, then blocks by descending score (ties: lower
 *      index) until the kept sum reaches gamma; gamma >= 1 keeps all.
 * q, k: device, bf16 (qk_dtype FP_QK_BF16) or int8 (FP_QK_INT8) in the layout
 * above.  q_scale[Hq], k_scale[Hkv]: device fp32 per-head dequantisation
 * scales for FP_QK_INT8 (logit = int32 dot * q_scale * k_scale / sqrt(d)),
 * NULL for bf16.  gamma in (0, 1]; tau >= 0.  S, Hq, Hkv, d, b must equal
 * the values idx was created with.  Writes only into idx. */
int fp_build_index(const void *q, const void *k, int S, int Hq, int Hkv, int d, int b,
                   float gamma, float tau, int qk_dtype, const float *q_scale,
                   const float *k_scale, fp_index *idx, void *stream);

/* Block-sparse GQA causal attention over exactly the blocks in idx (first
 * article: section 1.1 and figure 3; section 2.2 on KV reuse across the
 * heads of a GQA group): out[h][p] = sum over keys j <= p in the listed
 * blocks of softmax_j(q_p . k_j / sqrt(d)) v_j, fp32 softmax, bf16 output.
 * q, k: device bf16 or int8 (the qk_dtype idx was built with; scales as in
 * fp_build_index); v: device bf16; out: device bf16 [Hq][S][d].
 * Returns FP_ERR_STATE if idx has not been built. */
int fp_sparse_attn(const void *q, const void *k, const void *v, const float *q_scale,
                   const float *k_scale, const fp_index *idx, void *out, void *stream);

/* Shape of an index (any pointer may be NULL). */
int fp_index_info(const fp_index *idx, int *S, int *Hq, int *Hkv, int *d, int *b, int *qk_dtype);

/* Synchronises `stream` and returns the number of selected (head, query
 * block, key block) triples in *nnz. */
int fp_index_nnz(const fp_index *idx, int64_t *nnz, void *stream);

/* Synchronises `stream` and copies the index to HOST buffers (any may be
 * NULL): row_ptr[Hq*n + 1] and col[nnz] as CSR over rows h*n + r with
 * ascending key blocks; pattern[Hq] (FP_PATTERN_*); jsd[Hq]; vhat[Hq*n];
 * shat[Hq*n]; pest[Hq*n]. */
int fp_index_export(const fp_index *idx, int32_t *row_ptr, int32_t *col, uint8_t *pattern,
                    float *jsd, float *vhat, float *shat, float *pest, void *stream);

/* Head-pattern sharing (second article, section 5: similar heads share one
 * sparse pattern; the articles give no rule, so this is the written
 * convention).  Within each GQA group, in head order, head a joins the class
 * of the earliest earlier class representative b with JSD(vhat_a, vhat_b) <
 * eps (natural log, the divergence of the pattern decision); a head that
 * joins none represents its own class.  Every head of a class then attends to
 * the union of the class members' block lists for each query block, so every
 * head keeps at least its own gamma-coverage, and heads of one class walk the
 * same key blocks in fp_sparse_attn.  Rewrites the lists of a built index in
 * place (asynchronous on `stream`); eps >= 0 (eps = 0 shares nothing).
 * Returns FP_ERR_STATE before a build, FP_ERR_ARG for a negative or NaN eps
 * or more than 110 query heads per KV head. */
int fp_index_share(fp_index *idx, float eps, void *stream);

/* Compact block lists on the device (first article, section 3.2: compact
 * job lists).  row_ptr: device int32[Hq*n + 1] receives the CSR row offsets
 * over rows h*n + r (row_ptr[Hq*n] = nnz); col (device int32[nnz], or NULL
 * to get only row_ptr) the ascending key blocks of every row.  Both
 * caller-owned, 4-byte aligned; asynchronous on `stream`.  The attention
 * kernel itself reads the index's padded per-row lists (row (h, r) at a
 * fixed offset, written by the selection without a scan); this call
 * produces the compact form for other consumers. */
int fp_index_csr(const fp_index *idx, int32_t *row_ptr, int32_t *col, void *stream);

/* Per-(KV head, query block) union lists with head masks (first article,
 * section 2.2: a KV block loaded once serves the query heads of its GQA
 * group).  Rows j*n + r for KV head j: grp_ptr device int32[Hkv*n + 1]
 * (offsets), grp_col device int32[total] the ascending union of the g
 * query heads' blocks, grp_mask device uint32[total] with bit m set when
 * query head j*g + m lists that block.  grp_col and grp_mask both NULL to get
 * only grp_ptr (the total is grp_ptr[Hkv*n]).  g <= 32.  Caller-owned, 4-byte
 * aligned; asynchronous on `stream`. */
int fp_index_group_lists(const fp_index *idx, int32_t *grp_ptr, int32_t *grp_col, uint32_t *grp_mask,
                         void *stream);

/* Synchronises `stream` and copies the class representative of every query
 * head (absolute head index; h itself when not shared) to HOST cls[Hq]. */
int fp_index_classes(const fp_index *idx, int32_t *cls, void *stream);

/* Adaptive block size (second article, section 5: block size adjusted to the
 * complexity of the content; section 4.3: 64, 128, 256; the articles give no
 * rule, so this is the written convention).  From an index built with
 * b = 128: k_h = fewest key blocks whose vhat (the exact pooled last-block
 * attention of head h) sums to at least gamma, taken by descending vhat;
 * rho = mean over heads of k_h / n.  *b = 64 when rho < 0.1 and S/64 <= 1024
 * blocks, 256 when rho >= 0.5, else 128; *rho (may be NULL) receives rho.
 * The counts run on the device; synchronises `stream`.  Returns
 * FP_ERR_STATE unless idx is built with b = 128. */
int fp_choose_block_size(const fp_index *idx, float gamma, int *b, float *rho, void *stream);

/* Synchronises `stream`, returns FP_OK or the sticky device error recorded by
 * a kernel on the current device (FP_ERR_TIMEOUT), and clears it. */
int fp_get_device_error(void *stream);

/* Test hook for the bounded-wait path: launches one CTA that waits on a
 * barrier nothing will complete, giving up after timeout_us microseconds and
 * recording FP_ERR_TIMEOUT; the context stays usable.  timeout_us in
 * [1, 10000000]. */
int fp_debug_wait_timeout(int timeout_us, void *stream);

/* Test hook for the int8 score tiles: computes the exact int32 tile
 * out[i][t] = q8[h][p0 + i] . k8[h/g][j0 + t] for i, t in [0, 128) with the
 * same tensor-core path the int8 kernels use, into device out[128][128].
 * S a multiple of 128; p0, j0 multiples of 128 inside [0, S). */
int fp_debug_qk_tile_i8(const int8_t *q8, const int8_t *k8, int S, int Hq, int Hkv, int d, int h,
                        int p0, int j0, int32_t *out, void *stream);

/* Test hook for the int8 score tiles of the production kernels (first
 * article, section 3.3: INT8 multiply, exact INT32 accumulation).  Arms
 * (out != NULL) or disarms (out = NULL) a capture: while armed, every int8
 * fp_build_index (which = 0) or int8 fp_sparse_attn (which = 1) on any
 * device copies one raw 128 x 128 int32 score tile, exactly as the
 * tensor-core MMAs accumulated it and before any masking or scaling, to the
 * device buffer out[128][128] (row-major, 16-byte aligned, caller-owned):
 *   which = 0: the index pass's last-block scores of query head h, 128-row
 *              slice `tile` of the last block (rows (n-1)b + 128*tile ..),
 *              key chunk `chunk` (keys 128*chunk .. 128*chunk + 127);
 *   which = 1: the attention's scores of query head h, query tile `tile`
 *              (rows 128*tile ..), key chunk `chunk`; written only if that
 *              tile attends to that chunk (the chunk of a listed block).
 * Row i, column t of out is then q8[h][row0 + i] . k8[h/g][128*chunk + t].
 * The setting is process-wide; bf16 calls ignore it.  Returns FP_ERR_ARG for
 * which outside {0, 1}, a misaligned out or a negative coordinate. */
int fp_debug_capture_i8(int which, int h, int tile, int chunk, int32_t *out);

/* Per-head pattern statistics with no device allocation at all.  The papers
 * have no counterpart of this call; it exists for callers that must not
 * allocate device memory -- for example a host framework that owns every
 * byte of device memory through its own caching allocator or memory budget,
 * or a latency-critical loop that cannot afford the device-wide
 * synchronisation cudaMalloc/cudaFree imply.  It computes what
 * fp_build_index computes up to the pattern decision (steps 1-3 there):
 * vhat[Hq*n], shat[Hq*n], pest[Hq*n], jsd[Hq] and pattern[Hq]
 * (FP_PATTERN_*, int32), all caller-owned device buffers.  Inputs as in
 * fp_build_index (gamma is not needed).
 *
 * Scratch: a fixed 32 MiB array inside the library (a file-scope device
 * array; every GPU that loads the library keeps it until process exit).  A
 * problem needs at most 12*Hq*C*b + 512*Hkv*C + 512*Hkv*n bytes of it, with
 * C = ceil(S/128) column parts (2*ceil(S/128) when b = 64) and n = ceil(S/b),
 * plus 1.25 KiB of alignment; e.g. S=32768 with Hq=32, Hkv=8, b=128 fits, and
 * so does S=131072 with Hq=16, Hkv=4, b=128.
 * Larger problems are rejected with FP_ERR_ARG before anything is launched.
 * The first call on a device looks up the array's device address (set-up,
 * once per device, with that device current; after a device reset the next
 * call looks it up again); make that first call before any stream capture.  All calls share the one array and it keeps the last
 * call's contents; every scratch word a call reads is written earlier in
 * the same call, so nothing needs clearing.  Calls whose executions overlap
 * on the GPU (different streams, or different host threads) race on the
 * scratch and must be serialised by the caller.  Makes no cudaMalloc,
 * cudaFree or other allocating call. */
int fp_pattern_stats_noalloc(const void *q, const void *k, int S, int Hq, int Hkv, int d, int b,
                             float tau, int qk_dtype, const float *q_scale, const float *k_scale,
                             float *vhat, float *shat, float *pest, float *jsd, int32_t *pattern,
                             void *stream);

/* ---- Rotary-embedding epilogue with block pooling ----------------------
 * The projection step before the path (first article, section 1.1: Q = X W_q,
 * K = X W_k) ends with the rotary embedding; fp_rope_pool is that epilogue and
 * also emits the block means the index generation uses (section 2.1 block
 * pooling), so the index build need not read Q again to pool it.
 *
 * q_in [Hq][S][d], k_in [Hkv][S][d]: device bf16 before the rotation;
 * rope_cos, rope_sin: device fp32 [S][d/2] tables (cos and sin of the angle of
 * position p and frequency i); q_out, k_out: device bf16, same layouts (may be
 * q_in / k_in themselves); qbar [Hq][n][d], kbar [Hkv][n][d]: device fp32,
 * n = ceil(S/b).  Rotate-half convention: for i < d/2
 *   out[p][i] = x[p][i] cos[p][i] - x[p][i+d/2] sin[p][i],
 *   out[p][i+d/2] = x[p][i+d/2] cos[p][i] + x[p][i] sin[p][i],
 * computed in fp32 and stored as bf16 (nearest, ties to even); the means are
 * over the stored values of each block's rows.  Shapes as for fp_index_create;
 * all pointers 16-byte aligned; asynchronous on `stream`. */
int fp_rope_pool(const void *q_in, const void *k_in, const float *rope_cos, const float *rope_sin, int S, int Hq,
                 int Hkv, int d, int b, void *q_out, void *k_out, float *qbar, float *kbar, void *stream);

/* fp_build_index (bf16 q and k) with the block means supplied by the caller,
 * e.g. by fp_rope_pool: qbar [Hq][n][d] and kbar [Hkv][n][d] device fp32 must
 * be the block means of q and k.  The index pass then skips its own Q and K
 * pooling; the result is the one fp_build_index gives up to the summation
 * order of those means. */
int fp_build_index_pooled(const void *q, const void *k, const float *qbar, const float *kbar, int S, int Hq, int Hkv,
                          int d, int b, float gamma, float tau, fp_index *idx, void *stream);

/* ---- Packed sequences of different lengths ------------------------------
 * nseq sequences packed head-major: q[Hq][T][d], k and v [Hkv][T][d],
 * out [Hq][T][d], with sequence s at rows cu_seqlens[s] .. cu_seqlens[s+1]-1
 * of every head and T = cu_seqlens[nseq].  Every sequence is its own
 * problem (its own last block, statistics, pattern and block lists; causal
 * within the sequence, never across sequences), with the same supported
 * shapes as above for its length (lengths of 0 are allowed and skipped).
 * The articles treat one sequence at a time; this is that operation applied
 * to each sequence of a packed batch. */
typedef struct fp_varlen fp_varlen;

/* Allocates one index per non-empty sequence on the current device.
 * cu_seqlens: HOST int32[nseq + 1], cu_seqlens[0] = 0, non-decreasing.
 * Returns FP_ERR_ARG for bad offsets or shapes, FP_ERR_CUDA if allocation
 * fails. */
int fp_varlen_create(const int32_t *cu_seqlens, int nseq, int Hq, int Hkv, int d, int b, fp_varlen **out);

/* Frees the set and its indexes (NULL is ignored), each as fp_index_free does. */
void fp_varlen_free(fp_varlen *set);

/* fp_build_index for every sequence, queued in order on `stream`.  q, k:
 * packed device tensors as above (bf16 or int8); for FP_QK_INT8 the device
 * scales are per sequence and head: q_scale[nseq][Hq], k_scale[nseq][Hkv]. */
int fp_varlen_build_index(fp_varlen *set, const void *q, const void *k, float gamma, float tau, int qk_dtype,
                          const float *q_scale, const float *k_scale, void *stream);

/* fp_sparse_attn for every sequence over its own block lists; writes the
 * packed out [Hq][T][d] bf16.  Returns FP_ERR_STATE before a build. */
int fp_varlen_sparse_attn(const fp_varlen *set, const void *q, const void *k, const void *v, const float *q_scale,
                          const float *k_scale, void *out, void *stream);

/* Index of sequence `seq` (NULL for an empty sequence), owned by the set, for
 * fp_index_export / fp_index_nnz / fp_index_info (its S is the sequence
 * length).  fp_build_index and fp_sparse_attn refuse it with FP_ERR_STATE,
 * since its rows are spaced for the packed layout. */
int fp_varlen_index(const fp_varlen *set, int seq, const fp_index **out);

/* Static message for an FP_* code. */
const char *fp_strerror(int code);

#ifdef __cplusplus
}
#endif

#endif /* FP_SPARSE_H */

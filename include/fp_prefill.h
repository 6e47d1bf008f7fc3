/*
 * fp_prefill.h -- host-to-host prefill runtime over the C ABI of
 * fp_sparse.h: one call takes a layer's Q, K, V in host memory and returns
 * the attention output in host memory, overlapping the host-device copies
 * with the index build and the sparse attention.
 *
 * The articles on FAST-Prefill do not define this layer; it is the runtime
 * around the operation they define ("FPGA24成果：FAST-Prefill稀疏注意力加速器，
 * 长上下文LLM推理提速2.5倍", section 1.1 and figure 3, as computed by
 * fp_build_index and fp_sparse_attn).  Every head's index and output depend
 * only on that head's Q and on its KV head's K and V, so the layer is streamed
 * in groups of heads (whole KV heads with their query heads, or a share of
 * one KV head's query heads): group i is copied in while group i-1 is
 * computed and group i-2 is copied out, and consecutive runs overlap the same
 * way.  The result is
 * identical to fp_build_index + fp_sparse_attn over the whole layer.
 *
 * Layouts, supported shapes and the meaning of gamma and tau are those of
 * fp_sparse.h (q[Hq][S][d], k and v [Hkv][S][d], out [Hq][S][d]).
 */
#ifndef FP_PREFILL_H
#define FP_PREFILL_H

#include <stddef.h>
#include <stdint.h>

#include "fp_sparse.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Opaque pipeline: device copies of q, k, v, out and the int8 scales, one
 * fp_index per KV-head group, three streams (copy in, compute, copy out) and
 * their events, all on the device current at creation. */
typedef struct fp_prefill fp_prefill;

/* Creates a pipeline for one layer shape.  S, Hq, Hkv, d, b as in
 * fp_index_create; qk_dtype FP_QK_BF16 or FP_QK_INT8 (element type of the
 * host q and k); groups = number of head groups the layer is streamed in, 0
 * for Hkv (one KV head with its query heads per group).  A divisor of Hkv
 * makes groups of Hkv/groups whole KV heads; a multiple of Hkv that divides
 * Hq splits each KV head's query heads into groups/Hkv shares (K and V are
 * copied once, with the first share), which shortens the pipeline's start and
 * end at the price of one index build per share.  *out receives the
 * handle (NULL on error).  Returns FP_ERR_ARG for unsupported shapes or
 * groups, FP_ERR_CUDA if a device allocation or stream creation fails.  Device
 * memory: the layer's q, k, v and out plus the indexes of fp_index_create. */
int fp_prefill_create(int S, int Hq, int Hkv, int d, int b, int qk_dtype, int groups, fp_prefill **out);

/* Synchronises the device and frees the pipeline (NULL is ignored). */
void fp_prefill_free(fp_prefill *p);

/* Queues index build and sparse attention for one layer from host buffers to
 * a host buffer.  h_q [Hq][S][d] and h_k [Hkv][S][d] of the pipeline's
 * qk_dtype, h_v [Hkv][S][d] bf16, h_out [Hq][S][d] bf16 (written); h_q_scale[Hq]
 * and h_k_scale[Hkv] host fp32 for FP_QK_INT8 (read before the call returns),
 * NULL for bf16.  gamma in (0, 1], tau >= 0.  The work starts after everything
 * already queued on `stream` (a cudaStream_t, NULL = legacy default stream)
 * and runs on the pipeline's own streams; the call returns once it is queued.
 * Runs queued one after another on a pipeline overlap: run k+1 copies a
 * group's inputs in as soon as run k has computed that group, and writes a
 * group's output as soon as run k has copied it out, so a stream of layers
 * keeps the copies under the compute.  h_out of a run is complete once
 * fp_prefill_wait has made a stream wait for it and that stream has passed
 * that point; until then the run's host buffers must stay valid and h_q, h_k,
 * h_v unchanged.  Page-locked host memory (cudaHostAlloc, cudaHostRegister,
 * torch pin_memory) lets the copies overlap the compute; pageable memory gives
 * the same result with less overlap.  Calls on one pipeline must come from one
 * host thread at a time.  The call makes the pipeline's device current while
 * it queues work and then restores the caller's device; `stream` must belong
 * to the pipeline's device.  Returns FP_ERR_ARG for NULL buffers or
 * out-of-range gamma/tau (nothing is queued), FP_ERR_CUDA if queueing a copy,
 * launch or event fails (part of the run may then be queued: synchronise the
 * device before reusing the buffers); device-side wait timeouts are reported
 * by fp_get_device_error as for the other calls. */
int fp_prefill_enqueue(fp_prefill *p, const void *h_q, const void *h_k, const void *h_v,
                       const float *h_q_scale, const float *h_k_scale, float gamma, float tau, void *h_out,
                       void *stream);

/* Makes `stream` wait until the outputs of every run queued so far on the
 * pipeline are in host memory (nothing to wait for before the first run).
 * Returns FP_ERR_ARG for a NULL pipeline, FP_ERR_CUDA if the wait cannot be
 * queued. */
int fp_prefill_wait(fp_prefill *p, void *stream);

/* fp_prefill_enqueue followed by fp_prefill_wait on the same stream: events
 * recorded on `stream` around the call bracket the whole run, and
 * synchronising `stream` afterwards means h_out is complete. */
int fp_prefill_run(fp_prefill *p, const void *h_q, const void *h_k, const void *h_v, const float *h_q_scale,
                   const float *h_k_scale, float gamma, float tau, void *h_out, void *stream);

/* Index of head group `group` of the last run (query heads
 * group*Hq/groups .. (group+1)*Hq/groups - 1 and the KV heads they read), for
 * fp_index_export and fp_index_nnz; *out is owned by the pipeline.  Returns
 * FP_ERR_ARG for a bad group. */
int fp_prefill_group_index(const fp_prefill *p, int group, const fp_index **out);

#ifdef __cplusplus
}
#endif

#endif /* FP_PREFILL_H */

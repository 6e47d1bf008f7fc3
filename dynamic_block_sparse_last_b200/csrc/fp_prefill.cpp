// fp_prefill.cpp -- host-to-host prefill runtime (include/fp_prefill.h).
//
// Streams a layer through the device in groups of heads: whole KV heads with
// the query heads that read them, or (more groups than KV heads) one KV head
// with a share of its query heads, K and V then travelling with the first
// share.  The copy-in stream uploads group i while the compute stream runs
// fp_build_index + fp_sparse_attn on group i-1 and the copy-out stream
// downloads group i-2.  Consecutive runs overlap as well: run k+1 copies a
// group's inputs in once run k has computed that group, and overwrites a
// group's output once run k has copied it out.  Only the public C ABI of
// fp_sparse.h is used; every step of the computation runs in its kernels.
// Every head's index and output depend on that head's Q and its KV head's K
// and V alone, so the grouped result equals the whole-layer call.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include "fp_prefill.h"

struct fp_prefill {
  int S, Hq, Hkv, d, b, qk_dtype, groups;
  int device;
  size_t qk_elt;             // bytes per q/k element (2 bf16, 1 int8)
  void *d_q, *d_k, *d_v, *d_out;
  // int8 scales, two slots used by alternate runs: [Hq] q scales then [Hkv]
  // k scales, staged through page-locked host memory
  float *d_scales[2], *h_stage[2];
  std::vector<fp_index *> idx;
  cudaStream_t s_in, s_comp, s_out;
  cudaEvent_t ev_start, ev_last;
  cudaEvent_t ev_scale_in[2], ev_scale_free[2];    // slot copied in / last reader done
  std::vector<cudaEvent_t> ev_qk, ev_in, ev_comp, ev_out;  // per group: Q,K in; V in; computed; copied out
  long long runs;                                  // runs enqueued so far
};

namespace {

void release(fp_prefill *p) {
  if (!p) return;
  // all of the pipeline's work runs on its own three streams
  if (p->s_in) cudaStreamSynchronize(p->s_in);
  if (p->s_comp) cudaStreamSynchronize(p->s_comp);
  if (p->s_out) cudaStreamSynchronize(p->s_out);
  for (fp_index *i : p->idx) fp_index_free(i);
  for (cudaEvent_t e : p->ev_qk) if (e) cudaEventDestroy(e);
  for (cudaEvent_t e : p->ev_in) if (e) cudaEventDestroy(e);
  for (cudaEvent_t e : p->ev_comp) if (e) cudaEventDestroy(e);
  for (cudaEvent_t e : p->ev_out) if (e) cudaEventDestroy(e);
  for (int s = 0; s < 2; ++s) {
    if (p->ev_scale_in[s]) cudaEventDestroy(p->ev_scale_in[s]);
    if (p->ev_scale_free[s]) cudaEventDestroy(p->ev_scale_free[s]);
    if (p->d_scales[s]) cudaFree(p->d_scales[s]);
    if (p->h_stage[s]) cudaFreeHost(p->h_stage[s]);
  }
  if (p->ev_start) cudaEventDestroy(p->ev_start);
  if (p->ev_last) cudaEventDestroy(p->ev_last);
  if (p->s_in) cudaStreamDestroy(p->s_in);
  if (p->s_comp) cudaStreamDestroy(p->s_comp);
  if (p->s_out) cudaStreamDestroy(p->s_out);
  if (p->d_q) cudaFree(p->d_q);
  if (p->d_k) cudaFree(p->d_k);
  if (p->d_v) cudaFree(p->d_v);
  if (p->d_out) cudaFree(p->d_out);
  delete p;
}

// Shapes fp_index_create accepts (checked here too so that nothing is
// allocated for a shape it would reject).
bool shape_ok(int S, int Hq, int Hkv, int d, int b) {
  if (d != 128 || (b != 64 && b != 128 && b != 256)) return false;
  if (S <= 0 || (S + b - 1) / b > 1024) return false;
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return false;
  if ((int64_t)Hq * S > (int64_t)INT32_MAX) return false;
  return true;
}

// Makes the pipeline's device current for the scope of a call.
struct DeviceScope {
  int prev = -1;
  explicit DeviceScope(int dev) {
    if (cudaGetDevice(&prev) == cudaSuccess && prev != dev) cudaSetDevice(dev);
    else prev = -1;
  }
  ~DeviceScope() {
    if (prev >= 0) cudaSetDevice(prev);
  }
};

}  // namespace

extern "C" {

int fp_prefill_create(int S, int Hq, int Hkv, int d, int b, int qk_dtype, int groups, fp_prefill **out) {
  if (!out) return FP_ERR_ARG;
  *out = nullptr;
  if (!shape_ok(S, Hq, Hkv, d, b)) return FP_ERR_ARG;
  if (qk_dtype != FP_QK_BF16 && qk_dtype != FP_QK_INT8) return FP_ERR_ARG;
  if (groups == 0) groups = Hkv;
  if (groups < 1 || Hq % groups != 0) return FP_ERR_ARG;
  if (groups <= Hkv ? Hkv % groups != 0 : groups % Hkv != 0) return FP_ERR_ARG;
  fp_prefill *p = new (std::nothrow) fp_prefill();
  if (!p) return FP_ERR_CUDA;
  p->S = S; p->Hq = Hq; p->Hkv = Hkv; p->d = d; p->b = b; p->qk_dtype = qk_dtype; p->groups = groups;
  p->qk_elt = qk_dtype == FP_QK_INT8 ? 1 : 2;
  cudaGetDevice(&p->device);
  const size_t rq = (size_t)Hq * S * d, rkv = (size_t)Hkv * S * d;
  bool ok = cudaMalloc(&p->d_q, rq * p->qk_elt) == cudaSuccess && cudaMalloc(&p->d_k, rkv * p->qk_elt) == cudaSuccess &&
            cudaMalloc(&p->d_v, rkv * 2) == cudaSuccess && cudaMalloc(&p->d_out, rq * 2) == cudaSuccess;
  for (int s = 0; ok && s < 2; ++s)
    ok = cudaMalloc(reinterpret_cast<void **>(&p->d_scales[s]), (size_t)(Hq + Hkv) * sizeof(float)) == cudaSuccess &&
         cudaHostAlloc(reinterpret_cast<void **>(&p->h_stage[s]), (size_t)(Hq + Hkv) * sizeof(float),
                       cudaHostAllocDefault) == cudaSuccess &&
         cudaEventCreateWithFlags(&p->ev_scale_in[s], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&p->ev_scale_free[s], cudaEventDisableTiming) == cudaSuccess;
  ok = ok && cudaStreamCreateWithFlags(&p->s_in, cudaStreamNonBlocking) == cudaSuccess &&
       cudaStreamCreateWithFlags(&p->s_comp, cudaStreamNonBlocking) == cudaSuccess &&
       cudaStreamCreateWithFlags(&p->s_out, cudaStreamNonBlocking) == cudaSuccess &&
       cudaEventCreateWithFlags(&p->ev_start, cudaEventDisableTiming) == cudaSuccess &&
       cudaEventCreateWithFlags(&p->ev_last, cudaEventDisableTiming) == cudaSuccess;
  p->ev_qk.assign(groups, nullptr);
  p->ev_in.assign(groups, nullptr);
  p->ev_comp.assign(groups, nullptr);
  p->ev_out.assign(groups, nullptr);
  p->idx.assign(groups, nullptr);
  for (int i = 0; ok && i < groups; ++i) {
    ok = cudaEventCreateWithFlags(&p->ev_qk[i], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&p->ev_in[i], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&p->ev_comp[i], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&p->ev_out[i], cudaEventDisableTiming) == cudaSuccess &&
         fp_index_create(S, Hq / groups, groups <= Hkv ? Hkv / groups : 1, d, b, &p->idx[i]) == FP_OK;
  }
  if (!ok) {
    release(p);
    cudaGetLastError();  // clear a sticky allocation error
    return FP_ERR_CUDA;
  }
  *out = p;
  return FP_OK;
}

void fp_prefill_free(fp_prefill *p) {
  if (!p) return;
  DeviceScope scope(p->device);
  release(p);
}

int fp_prefill_enqueue(fp_prefill *p, const void *h_q, const void *h_k, const void *h_v, const float *h_q_scale,
                       const float *h_k_scale, float gamma, float tau, void *h_out, void *stream) {
  if (!p || !h_q || !h_k || !h_v || !h_out) return FP_ERR_ARG;
  if (!(gamma > 0.f && gamma <= 1.f) || !(tau >= 0.f) || std::isnan(gamma) || std::isnan(tau)) return FP_ERR_ARG;
  const bool i8 = p->qk_dtype == FP_QK_INT8;
  if (i8 && (!h_q_scale || !h_k_scale)) return FP_ERR_ARG;
  DeviceScope scope(p->device);
  cudaStream_t user = static_cast<cudaStream_t>(stream);
  // group i: query heads [i*hq, (i+1)*hq), KV heads [kv0(i), kv0(i) + hkv)
  const int G = p->groups, hq = p->Hq / G;
  const int hkv = G <= p->Hkv ? p->Hkv / G : 1, share = G <= p->Hkv ? 1 : G / p->Hkv;
  auto kv0 = [&](int i) { return (i / share) * hkv; };
  auto carries_kv = [&](int i) { return i % share == 0; };  // first share of its KV heads
  const size_t row = (size_t)p->S * p->d;                // elements of one head
  const size_t q_bytes = hq * row * p->qk_elt, kv_qk_bytes = hkv * row * p->qk_elt;
  const size_t v_bytes = hkv * row * 2, out_bytes = hq * row * 2;
  const char *hq8 = static_cast<const char *>(h_q), *hk8 = static_cast<const char *>(h_k);
  const char *hv8 = static_cast<const char *>(h_v);
  char *ho8 = static_cast<char *>(h_out);
  char *dq = static_cast<char *>(p->d_q), *dk = static_cast<char *>(p->d_k), *dv = static_cast<char *>(p->d_v);
  char *dout = static_cast<char *>(p->d_out);
  const bool prev = p->runs > 0;         // the per-group events hold the previous run's records
  const int slot = (int)(p->runs & 1);   // scale slot of this run
  const float *qs = i8 ? p->d_scales[slot] : nullptr, *ks = i8 ? p->d_scales[slot] + p->Hq : nullptr;

  // everything starts after the work already queued on the caller's stream
  if (cudaEventRecord(p->ev_start, user) != cudaSuccess) return FP_ERR_CUDA;
  if (cudaStreamWaitEvent(p->s_in, p->ev_start, 0) != cudaSuccess) return FP_ERR_CUDA;
  if (i8) {
    // the run two back copied this slot in long ago; wait for it before
    // refilling the staging buffer, and for its last reader on the device
    const size_t nsc = (size_t)(p->Hq + p->Hkv);
    if (p->runs >= 2 && cudaEventSynchronize(p->ev_scale_in[slot]) != cudaSuccess) return FP_ERR_CUDA;
    memcpy(p->h_stage[slot], h_q_scale, (size_t)p->Hq * sizeof(float));
    memcpy(p->h_stage[slot] + p->Hq, h_k_scale, (size_t)p->Hkv * sizeof(float));
    if ((p->runs >= 2 && cudaStreamWaitEvent(p->s_in, p->ev_scale_free[slot], 0) != cudaSuccess) ||
        cudaMemcpyAsync(p->d_scales[slot], p->h_stage[slot], nsc * sizeof(float), cudaMemcpyHostToDevice, p->s_in) !=
            cudaSuccess ||
        cudaEventRecord(p->ev_scale_in[slot], p->s_in) != cudaSuccess)
      return FP_ERR_CUDA;
  }
  // copy in, group by group: K and Q (all the index build reads), then V;
  // a later share of a KV head only brings its Q (stream order covers K, V).
  // A buffer is refilled once the previous run's compute no longer reads it.
  for (int i = 0; i < G; ++i) {
    const size_t ko = (size_t)kv0(i) / hkv * kv_qk_bytes, vo = (size_t)kv0(i) / hkv * v_bytes;
    const int last_reader = carries_kv(i) ? i + share - 1 : i;  // compute of every share of these KV heads
    if (prev && cudaStreamWaitEvent(p->s_in, p->ev_comp[last_reader], 0) != cudaSuccess) return FP_ERR_CUDA;
    if (carries_kv(i) &&
        cudaMemcpyAsync(dk + ko, hk8 + ko, kv_qk_bytes, cudaMemcpyHostToDevice, p->s_in) != cudaSuccess)
      return FP_ERR_CUDA;
    if (cudaMemcpyAsync(dq + i * q_bytes, hq8 + i * q_bytes, q_bytes, cudaMemcpyHostToDevice, p->s_in) != cudaSuccess ||
        cudaEventRecord(p->ev_qk[i], p->s_in) != cudaSuccess)
      return FP_ERR_CUDA;
    if (carries_kv(i) &&
        cudaMemcpyAsync(dv + vo, hv8 + vo, v_bytes, cudaMemcpyHostToDevice, p->s_in) != cudaSuccess)
      return FP_ERR_CUDA;
    if (cudaEventRecord(p->ev_in[i], p->s_in) != cudaSuccess) return FP_ERR_CUDA;
  }
  // compute: index then attention per group, each as soon as its inputs are
  // in and the previous run's output of the group has been copied out
  for (int i = 0; i < G; ++i) {
    if (cudaStreamWaitEvent(p->s_comp, p->ev_qk[i], 0) != cudaSuccess) return FP_ERR_CUDA;
    const void *gq = dq + i * q_bytes, *gk = dk + (size_t)kv0(i) / hkv * kv_qk_bytes;
    const void *gv = dv + (size_t)kv0(i) / hkv * v_bytes;
    const float *gqs = i8 ? qs + i * hq : nullptr, *gks = i8 ? ks + kv0(i) : nullptr;
    int rc = fp_build_index(gq, gk, p->S, hq, hkv, p->d, p->b, gamma, tau, p->qk_dtype, gqs, gks, p->idx[i],
                            p->s_comp);
    if (rc) return rc;
    if (cudaStreamWaitEvent(p->s_comp, p->ev_in[i], 0) != cudaSuccess) return FP_ERR_CUDA;
    if (prev && cudaStreamWaitEvent(p->s_comp, p->ev_out[i], 0) != cudaSuccess) return FP_ERR_CUDA;
    rc = fp_sparse_attn(gq, gk, gv, gqs, gks, p->idx[i], dout + i * out_bytes, p->s_comp);
    if (rc) return rc;
    if (cudaEventRecord(p->ev_comp[i], p->s_comp) != cudaSuccess) return FP_ERR_CUDA;
  }
  if (i8 && cudaEventRecord(p->ev_scale_free[slot], p->s_comp) != cudaSuccess) return FP_ERR_CUDA;
  // copy out: each group's output as soon as it is written
  for (int i = 0; i < G; ++i) {
    if (cudaStreamWaitEvent(p->s_out, p->ev_comp[i], 0) != cudaSuccess ||
        cudaMemcpyAsync(ho8 + i * out_bytes, dout + i * out_bytes, out_bytes, cudaMemcpyDeviceToHost, p->s_out) !=
            cudaSuccess ||
        cudaEventRecord(p->ev_out[i], p->s_out) != cudaSuccess)
      return FP_ERR_CUDA;
  }
  if (cudaEventRecord(p->ev_last, p->s_out) != cudaSuccess) return FP_ERR_CUDA;
  ++p->runs;
  return FP_OK;
}

int fp_prefill_wait(fp_prefill *p, void *stream) {
  if (!p) return FP_ERR_ARG;
  DeviceScope scope(p->device);
  if (p->runs == 0) return FP_OK;
  return cudaStreamWaitEvent(static_cast<cudaStream_t>(stream), p->ev_last, 0) == cudaSuccess ? FP_OK : FP_ERR_CUDA;
}

int fp_prefill_run(fp_prefill *p, const void *h_q, const void *h_k, const void *h_v, const float *h_q_scale,
                   const float *h_k_scale, float gamma, float tau, void *h_out, void *stream) {
  const int rc = fp_prefill_enqueue(p, h_q, h_k, h_v, h_q_scale, h_k_scale, gamma, tau, h_out, stream);
  return rc ? rc : fp_prefill_wait(p, stream);
}

int fp_prefill_group_index(const fp_prefill *p, int group, const fp_index **out) {
  if (!p || !out || group < 0 || group >= p->groups) return FP_ERR_ARG;
  *out = p->idx[group];
  return FP_OK;
}

}  // extern "C"

// fp_sparse.cu -- host side of the C ABI declared in include/fp_sparse.h:
// argument validation, the library-owned index workspace, TMA tensor maps
// and the kernel launches.  Every step of the computation runs in the CUDA
// kernels of index_kernels.cuh and attn_kernel.cuh; there is no host
// fallback.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "attn_kernel.cuh"
#include "fp_sparse.h"
#include "index_kernels.cuh"
#include "rope_pool.cuh"
#include "share_kernels.cuh"

using namespace fpk;

// One sticky error word per device (module-scope device variable).
static __device__ int g_fp_dev_error;

struct fp_index {
  int S, Hq, Hkv, d, b, n, nch, g;
  int npart;               // column parts of the statistics: nch, or 2 nch when b = 64 (one per block)
  int ld;                  // rows from one head to the next in q, k, v, out (S, or T when packed)
  int device;
  int built;
  int qk_dtype;
  void *slab;
  size_t slab_bytes;
  bool slab_pooled;        // slab from the stream-ordered allocator (else cudaMalloc)
  cudaStream_t own;        // the index's own stream: allocation and release of the slab
  cudaEvent_t last_use;    // recorded on the caller's stream at the end of every build / attention call
  float *pm, *plo, *phi;   // [Hq][npart][b]
  float *ksum;             // [Hkv][npart][128]
  float *kbar;             // [Hkv][n][128]
  float *qbar;             // [Hq][n][128]
  float *qsplit, *ksplit;  // [Hq][n][256], [Hkv][n][256]: tf32 hi | lo of the block means (logits operands)
  float *vhat, *shat, *pest;  // [Hq][n]
  float *jsd;              // [Hq]
  int *pattern;            // [Hq]
  int *counts;             // [Hq][n]
  int *cls;                // [Hq] head-sharing class representatives (fp_index_share)
  int *cover;              // [Hq] blocks covering gamma of vhat (fp_choose_block_size)
  int *gcount;             // [Hkv][n] union sizes of the group lists (fp_index_group_lists)
  int shared;              // the lists are class unions (fp_index_share ran after the last index build)
  int *cols;               // [Hq][n(n+1)/2]
  float *zlog;             // [Hq][n(n+1)/2] q-bar . k-bar logits (query-aware heads)
};

namespace {

std::mutex g_mu;

// Per-device set-up (device addresses of the library's __device__ arrays,
// raised shared-memory limits of the big kernels), valid for one context of
// that device: a device reset destroys the primary context and everything
// set up in it, so the entry is redone when the current context changes.
struct DevState {
  void *ctx;
  int *err;                 // g_fp_dev_error
  unsigned char *scratch;   // g_fp_stats_scratch (allocation-free call)
  bool attrs[2];            // set_smem_attrs<false>, <true>
};
DevState g_dev[128] = {};

// The calling thread's current context (the device's primary context once
// the runtime has made it current), through the driver entry point.
void *current_context() {
  using Fn = CUresult (*)(CUcontext *);
  static Fn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<Fn>(p);
  });
  CUcontext c = nullptr;
  if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
  if (!c) {
    cudaFree(nullptr);  // no-op that makes the runtime's primary context current
    if (fn(&c) != CUDA_SUCCESS) return nullptr;
  }
  return c;
}

// The current device's entry, refreshed when its context changed; call with
// g_mu held.  Returns null for an unusable device.
DevState *dev_state() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return nullptr;
  void *ctx = current_context();
  if (!ctx) return nullptr;
  DevState &d = g_dev[dev];
  if (d.ctx != ctx) d = DevState{ctx, nullptr, nullptr, {false, false}};
  return &d;
}

// Armed int8 tile captures (fp_debug_capture_i8); read when an int8 launch
// is prepared, so the captured tile comes from the normal launch path.
struct CaptureI8 {
  int32_t *score;
  int s_h, s_slice, s_ch;
  int32_t *attn;
  int a_h, a_qc, a_kc;
};
CaptureI8 g_cap = {nullptr, 0, 0, 0, nullptr, 0, 0, 0};

CaptureI8 capture_settings() {
  std::lock_guard<std::mutex> lk(g_mu);
  return g_cap;
}

int *device_error_word() {
  std::lock_guard<std::mutex> lk(g_mu);
  DevState *d = dev_state();
  if (!d) return nullptr;
  if (!d->err) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fp_dev_error) != cudaSuccess) return nullptr;
    d->err = static_cast<int *>(p);
  }
  return d->err;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D map over a [rows][128] tensor: boxes of 128 rows x 128 bytes
// (64 bf16 or 128 int8 columns), 128-byte swizzle.  For H heads of S rows
// spaced ld rows apart the map covers (H-1)*ld + S rows from the first head's
// first row, so no box reads past the last head's last row.
bool make_map(CUtensorMap *m, const void *ptr, bool i8, uint64_t rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {128, rows};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(128 * (i8 ? 1 : 2))};
  const cuuint32_t box[2] = {i8 ? 128u : 64u, 128u};
  const cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(m, i8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Rows of 256 fp32 (a block mean split as tf32 hi | lo), 32-column x 128-row
// boxes with the 128-byte swizzle: the operands of k_qa_logits.
bool make_map_split(CUtensorMap *m, const float *ptr, uint64_t rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {256, rows};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(256 * 4)};
  const cuuint32_t box[2] = {32u, 128u};
  const cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

uint64_t map_rows(int H, int ld, int S) { return (uint64_t)(H - 1) * (uint64_t)ld + (uint64_t)S; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool shape_ok(int S, int Hq, int Hkv, int d, int b) {
  if (d != 128) return false;
  if (b != 64 && b != 128 && b != 256) return false;
  if (S <= 0 || (S + b - 1) / b > kSelMaxN) return false;
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return false;
  if ((int64_t)Hq * S > (int64_t)INT32_MAX || (int64_t)Hkv * S > (int64_t)INT32_MAX) return false;
  return true;
}

int sm_count() {
  int dev = 0, n = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

template <typename T>
T *carve(char *&cur, size_t count) {
  T *p = reinterpret_cast<T *>(cur);
  cur += ((count * sizeof(T) + 255) / 256) * 256;
  return p;
}

int launch_status() { return cudaGetLastError() == cudaSuccess ? FP_OK : FP_ERR_CUDA; }

template <bool I8>
int set_smem_attrs() {
  std::lock_guard<std::mutex> lk(g_mu);  // first calls from several host threads
  DevState *d = dev_state();
  if (!d) return FP_ERR_CUDA;
  if (d->attrs[I8]) return FP_OK;
  if (cudaFuncSetAttribute(k_score_last<I8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           ScoreCfg<I8>::kSmem) != cudaSuccess)
    return FP_ERR_CUDA;
  if (cudaFuncSetAttribute(k_sparse_attn<I8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           AttnCfg<I8>::kSmem) != cudaSuccess)
    return FP_ERR_CUDA;
  if (cudaFuncSetAttribute(k_qa_logits, cudaFuncAttributeMaxDynamicSharedMemorySize, kLgSmem) != cudaSuccess)
    return FP_ERR_CUDA;
  d->attrs[I8] = true;
  return FP_OK;
}

// Shape, inputs and scratch of the pattern-statistics launches (steps 1-3 of
// fp_build_index), shared by the index build and the allocation-free call.
struct StatsJob {
  int S, Hq, Hkv, d, b, n, nch, g;
  int npart;  // column parts: nch, or 2 nch when b = 64
  int ld;  // rows from one head to the next
  const void *q, *k;
  const float *q_scale, *k_scale;  // int8 only
  float tau;
  float *pm, *plo, *phi, *ksum, *kbar;
  float *vhat, *shat, *pest, *jsd;
  int *pattern;
  const float *ext_kbar;  // K block means given by the caller (then ksum/kbar are not computed), or null
};

// k_score_last on `st`.
template <bool I8>
int launch_score(const StatsJob &J, int *err, cudaStream_t st) {
  CUtensorMap tq, tk;
  if (!make_map(&tq, J.q, I8, map_rows(J.Hq, J.ld, J.S)) || !make_map(&tk, J.k, I8, map_rows(J.Hkv, J.ld, J.S)))
    return FP_ERR_CUDA;
  const int nlast = J.S - (J.n - 1) * J.b;  // rows of the (possibly partial) last block
  const int tiles_per_head = (nlast + 127) / 128;
  const int tiles_per_group = J.g * tiles_per_head;
  const int tgroups = (tiles_per_group + ScoreCfg<I8>::kTiles - 1) / ScoreCfg<I8>::kTiles;
  int R = sm_count() / (tgroups * J.Hkv);
  if (R < 1) R = 1;
  if (R > J.nch) R = J.nch;
  const int cpc = (J.nch + R - 1) / R;
  R = (J.nch + cpc - 1) / cpc;
  ScoreParams sp;
  sp.S = J.S; sp.Hq = J.Hq; sp.Hkv = J.Hkv; sp.b = J.b; sp.n = J.n; sp.nch = J.nch; sp.g = J.g;
  sp.nsub = J.npart / J.nch;
  sp.ld = J.ld;
  sp.nlast = nlast;
  sp.tiles_per_head = tiles_per_head;
  sp.tiles_per_group = tiles_per_group;
  sp.chunks_per_cta = cpc;
  sp.scale2 = kLog2e / sqrtf((float)J.d);
  sp.q_scale = J.q_scale;
  sp.k_scale = J.k_scale;
  sp.pm = J.pm; sp.plo = J.plo; sp.phi = J.phi; sp.ksum = J.ext_kbar ? nullptr : J.ksum;
  sp.err = err;
  sp.cap = nullptr;
  sp.cap_h = sp.cap_slice = sp.cap_ch = 0;
  if (I8) {
    const CaptureI8 c = capture_settings();
    sp.cap = c.score;
    sp.cap_h = c.s_h; sp.cap_slice = c.s_slice; sp.cap_ch = c.s_ch;
  }
  k_score_last<I8><<<dim3(R, tgroups, J.Hkv), ScoreCfg<I8>::kThreads, ScoreCfg<I8>::kSmem, st>>>(tq, tk, sp);
  return launch_status();
}

// k_head_stats on `st` (after launch_score).
template <bool I8>
int launch_head_stats(const StatsJob &J, cudaStream_t st) {
  const int nlast = J.S - (J.n - 1) * J.b;
  HeadStatsParams hp;
  hp.S = J.S; hp.b = J.b; hp.n = J.n; hp.npart = J.npart; hp.g = J.g; hp.ld = J.ld; hp.nlast = nlast;
  hp.pm = J.pm; hp.plo = J.plo; hp.phi = J.phi;
  hp.ksum = J.ksum; hp.ext_kbar = J.ext_kbar; hp.k_scale = J.k_scale;
  hp.q = J.q; hp.q_scale = J.q_scale;
  hp.inv_sqrt_d = 1.0f / sqrtf((float)J.d);
  hp.tau = J.tau;
  hp.vhat = J.vhat; hp.shat = J.shat; hp.pest = J.pest; hp.jsd = J.jsd; hp.pattern = J.pattern;
  hp.kbar = J.kbar;
  k_head_stats<I8><<<dim3(kStatCta, J.Hq), kStatThreads, 0, st>>>(hp);
  return launch_status();
}

// ext_qbar / ext_kbar: block means of Q [Hq][n][128] and K [Hkv][n][128]
// computed by the caller (fp_rope_pool); when given, the index build does not
// pool Q or K itself.
template <bool I8>
int build_index_impl(const void *q, const void *k, float gamma, float tau, const float *q_scale,
                     const float *k_scale, fp_index *I, cudaStream_t st, const float *ext_qbar = nullptr,
                     const float *ext_kbar = nullptr) {
  int rc = set_smem_attrs<I8>();
  if (rc) return rc;
  int *err = device_error_word();
  if (!err) return FP_ERR_CUDA;
  StatsJob J;
  J.S = I->S; J.Hq = I->Hq; J.Hkv = I->Hkv; J.d = I->d; J.b = I->b; J.n = I->n; J.nch = I->nch; J.g = I->g;
  J.npart = I->npart;
  J.ld = I->ld;
  J.q = q; J.k = k; J.q_scale = q_scale; J.k_scale = k_scale; J.tau = tau;
  J.pm = I->pm; J.plo = I->plo; J.phi = I->phi;
  J.ksum = I->ksum; J.kbar = I->kbar;
  J.vhat = I->vhat; J.shat = I->shat; J.pest = I->pest; J.jsd = I->jsd; J.pattern = I->pattern;
  J.ext_kbar = ext_kbar;
  if ((rc = launch_score<I8>(J, err, st))) return rc;
  if ((rc = launch_head_stats<I8>(J, st))) return rc;
  // Q block means of the query-aware heads only, now that the pattern is known
  const float *qbar = ext_qbar;
  if (!qbar) {
    k_qpool<I8><<<dim3(I->n, I->Hq), 128, 0, st>>>(I->pattern, q, q_scale, I->S, I->ld, I->b, I->n, I->qbar);
    if ((rc = launch_status())) return rc;
    qbar = I->qbar;
  }
  const float inv_sqrt_d = 1.0f / sqrtf((float)I->d);
  const float *kbar = ext_kbar ? ext_kbar : I->kbar;
  if (I->n >= kLgTensorMinN) {
    // tensor cores: the logits' operands as tf32 hi | lo pairs (q-bar of the
    // query-aware heads only), 128 x 128 tiles
    const int qrows = I->Hq * I->n, krows = I->Hkv * I->n;
    k_split_tf32<<<(qrows + 7) / 8, 256, 0, st>>>(qbar, I->qsplit, qrows, I->n, I->pattern);
    if ((rc = launch_status())) return rc;
    k_split_tf32<<<(krows + 7) / 8, 256, 0, st>>>(kbar, I->ksplit, krows, I->n, nullptr);
    if ((rc = launch_status())) return rc;
    CUtensorMap tmq, tmk;
    if (!make_map_split(&tmq, I->qsplit, (uint64_t)qrows) || !make_map_split(&tmk, I->ksplit, (uint64_t)krows))
      return FP_ERR_CUDA;
    const int nt = (I->n + kLgTile - 1) / kLgTile;
    k_qa_logits<<<dim3(nt * (nt + 1) / 2, I->Hq), 128, kLgSmem, st>>>(tmq, tmk, I->pattern, I->g, I->n,
                                                                      inv_sqrt_d, err, I->zlog);
  } else {
    // too few 128 x 128 tiles to fill the GPU: 64 x 64 tiles on the FMA pipe
    const int nt = (I->n + kLgFmaTile - 1) / kLgFmaTile;
    k_qa_logits_fma<<<dim3(nt * (nt + 1) / 2, I->Hq), 256, 0, st>>>(I->pattern, qbar, kbar, I->g, I->n,
                                                                     inv_sqrt_d, I->zlog);
  }
  if ((rc = launch_status())) return rc;
  k_cut<<<(I->Hq * I->n + 7) / 8, 256, 0, st>>>(I->pattern, I->vhat, I->shat, I->zlog, I->Hq, I->n, gamma,
                                               I->counts, I->cols);
  if ((rc = launch_status())) return rc;
  return cudaEventRecord(I->last_use, st) == cudaSuccess ? FP_OK : FP_ERR_CUDA;
}

template <bool I8>
int attn_impl(const void *q, const void *k, const void *v, const float *q_scale, const float *k_scale,
              const fp_index *I, void *out, cudaStream_t st) {
  int rc = set_smem_attrs<I8>();
  if (rc) return rc;
  int *err = device_error_word();
  if (!err) return FP_ERR_CUDA;
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, q, I8, map_rows(I->Hq, I->ld, I->S)) || !make_map(&tk, k, I8, map_rows(I->Hkv, I->ld, I->S)) ||
      !make_map(&tv, v, false, map_rows(I->Hkv, I->ld, I->S)))
    return FP_ERR_CUDA;
  AttnParams ap;
  ap.S = I->S; ap.Hq = I->Hq; ap.Hkv = I->Hkv; ap.b = I->b; ap.n = I->n; ap.g = I->g; ap.ld = I->ld;
  ap.counts = I->counts;
  ap.cols = I->cols;
  ap.q_scale = q_scale;
  ap.k_scale = k_scale;
  ap.scale2 = kLog2e / sqrtf((float)I->d);
  ap.out = static_cast<__nv_bfloat16 *>(out);
  ap.err = err;
  ap.cap = nullptr;
  ap.cap_h = ap.cap_qc = ap.cap_kc = 0;
  if (I8) {
    const CaptureI8 c = capture_settings();
    ap.cap = c.attn;
    ap.cap_h = c.a_h; ap.cap_qc = c.a_qc; ap.cap_kc = c.a_kc;
  }
  const unsigned grid = (unsigned)attn_pairs(I->Hq, I->Hkv, I->S, I->b);
  k_sparse_attn<I8><<<grid, AttnCfg<I8>::kThreads, AttnCfg<I8>::kSmem, st>>>(tq, tk, tv, ap);
  if ((rc = launch_status())) return rc;
  return cudaEventRecord(I->last_use, st) == cudaSuccess ? FP_OK : FP_ERR_CUDA;
}

// Index for one sequence of S rows per head, heads ld rows apart.
int index_create(int S, int ld, int Hq, int Hkv, int d, int b, fp_index **out) {
  if (!out) return FP_ERR_ARG;
  *out = nullptr;
  if (!shape_ok(S, Hq, Hkv, d, b) || ld < S || (int64_t)Hq * ld > (int64_t)INT32_MAX) return FP_ERR_ARG;
  fp_index *I = static_cast<fp_index *>(calloc(1, sizeof(fp_index)));
  if (!I) return FP_ERR_CUDA;
  I->S = S; I->Hq = Hq; I->Hkv = Hkv; I->d = d; I->b = b; I->ld = ld;
  I->n = (S + b - 1) / b; I->nch = (S + 127) / 128; I->g = Hq / Hkv;
  I->npart = b < 128 ? I->nch * (128 / b) : I->nch;
  cudaGetDevice(&I->device);
  const size_t n = I->n, nch = I->npart, bb = b;  // statistics arrays are per column part
  const size_t tri = n * (n + 1) / 2;
  size_t need = 0;
  auto add = [&](size_t bytes) { need += ((bytes + 255) / 256) * 256; };
  for (int i = 0; i < 3; ++i) add((size_t)Hq * nch * bb * 4);
  add((size_t)Hkv * nch * 128 * 4);
  add((size_t)Hkv * n * 128 * 4);
  add((size_t)Hq * n * 128 * 4);
  const size_t nsplit = n >= (size_t)kLgTensorMinN ? n : 0;  // tf32 operands only where the tensor-core logits run
  add((size_t)Hq * nsplit * 256 * 4);
  add((size_t)Hkv * nsplit * 256 * 4);
  for (int i = 0; i < 3; ++i) add((size_t)Hq * n * 4);
  add((size_t)Hq * 4);
  add((size_t)Hq * 4);
  add((size_t)Hq * n * 4);
  add((size_t)Hq * 4);
  add((size_t)Hq * 4);
  add((size_t)Hkv * n * 4);
  add((size_t)Hq * tri * 4);
  add((size_t)Hq * tri * 4);
  if (cudaStreamCreateWithFlags(&I->own, cudaStreamNonBlocking) != cudaSuccess) {
    free(I);
    return FP_ERR_CUDA;
  }
  if (cudaEventCreateWithFlags(&I->last_use, cudaEventDisableTiming) != cudaSuccess) {
    cudaStreamDestroy(I->own);
    free(I);
    return FP_ERR_CUDA;
  }
  // stream-ordered allocation, so that freeing waits for this index's work
  // only; plain cudaMalloc where the device has no memory pools
  I->slab_pooled = cudaMallocAsync(&I->slab, need, I->own) == cudaSuccess &&
                   cudaStreamSynchronize(I->own) == cudaSuccess;
  if (!I->slab_pooled) {
    cudaGetLastError();
    I->slab = nullptr;
    if (cudaMalloc(&I->slab, need) != cudaSuccess) {
      cudaEventDestroy(I->last_use);
      cudaStreamDestroy(I->own);
      free(I);
      return FP_ERR_CUDA;
    }
  }
  I->slab_bytes = need;
  char *cur = static_cast<char *>(I->slab);
  I->pm = carve<float>(cur, (size_t)Hq * nch * bb);
  I->plo = carve<float>(cur, (size_t)Hq * nch * bb);
  I->phi = carve<float>(cur, (size_t)Hq * nch * bb);
  I->ksum = carve<float>(cur, (size_t)Hkv * nch * 128);
  I->kbar = carve<float>(cur, (size_t)Hkv * n * 128);
  I->qbar = carve<float>(cur, (size_t)Hq * n * 128);
  I->qsplit = carve<float>(cur, (size_t)Hq * nsplit * 256);
  I->ksplit = carve<float>(cur, (size_t)Hkv * nsplit * 256);
  I->vhat = carve<float>(cur, (size_t)Hq * n);
  I->shat = carve<float>(cur, (size_t)Hq * n);
  I->pest = carve<float>(cur, (size_t)Hq * n);
  I->jsd = carve<float>(cur, (size_t)Hq);
  I->pattern = carve<int>(cur, (size_t)Hq);
  I->counts = carve<int>(cur, (size_t)Hq * n);
  I->cls = carve<int>(cur, (size_t)Hq);
  I->cover = carve<int>(cur, (size_t)Hq);
  I->gcount = carve<int>(cur, (size_t)Hkv * n);
  I->cols = carve<int>(cur, (size_t)Hq * tri);
  I->zlog = carve<float>(cur, (size_t)Hq * tri);
  *out = I;
  return FP_OK;
}

}  // namespace

extern "C" {

int fp_index_create(int S, int Hq, int Hkv, int d, int b, fp_index **out) {
  return index_create(S, S, Hq, Hkv, d, b, out);
}

void fp_index_free(fp_index *I) {
  if (!I) return;
  int prev = -1;
  if (cudaGetDevice(&prev) == cudaSuccess && prev != I->device) cudaSetDevice(I->device);
  else prev = -1;
  if (I->slab_pooled) {
    // released in stream order after the index's last call; nothing else waits
    cudaStreamWaitEvent(I->own, I->last_use, 0);
    cudaFreeAsync(I->slab, I->own);
  } else if (I->slab) {
    cudaEventSynchronize(I->last_use);
    cudaFree(I->slab);
  }
  cudaEventDestroy(I->last_use);
  cudaStreamDestroy(I->own);  // returns at once; the stream's pending free still completes
  if (prev >= 0) cudaSetDevice(prev);
  free(I);
}

int fp_build_index(const void *q, const void *k, int S, int Hq, int Hkv, int d, int b, float gamma,
                   float tau, int qk_dtype, const float *q_scale, const float *k_scale, fp_index *idx,
                   void *stream) {
  if (!idx || !q || !k) return FP_ERR_ARG;
  if (!shape_ok(S, Hq, Hkv, d, b)) return FP_ERR_ARG;
  if (S != idx->S || Hq != idx->Hq || Hkv != idx->Hkv || d != idx->d || b != idx->b) return FP_ERR_STATE;
  if (idx->ld != idx->S) return FP_ERR_STATE;  // an index of a packed set: fp_varlen_* calls only
  if (!(gamma > 0.f && gamma <= 1.f) || !(tau >= 0.f) || std::isnan(gamma) || std::isnan(tau)) return FP_ERR_ARG;
  if (qk_dtype != FP_QK_BF16 && qk_dtype != FP_QK_INT8) return FP_ERR_ARG;
  if (qk_dtype == FP_QK_INT8 && (!q_scale || !k_scale)) return FP_ERR_ARG;
  if (!aligned16(q) || !aligned16(k)) return FP_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  idx->built = 0;
  idx->shared = 0;
  const int rc = qk_dtype == FP_QK_INT8 ? build_index_impl<true>(q, k, gamma, tau, q_scale, k_scale, idx, st)
                                        : build_index_impl<false>(q, k, gamma, tau, nullptr, nullptr, idx, st);
  if (rc == FP_OK) {
    idx->built = 1;
    idx->qk_dtype = qk_dtype;
  }
  return rc;
}

int fp_sparse_attn(const void *q, const void *k, const void *v, const float *q_scale, const float *k_scale,
                   const fp_index *idx, void *out, void *stream) {
  if (!idx || !q || !k || !v || !out) return FP_ERR_ARG;
  if (!idx->built || idx->ld != idx->S) return FP_ERR_STATE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return FP_ERR_ARG;
  if (idx->qk_dtype == FP_QK_INT8 && (!q_scale || !k_scale)) return FP_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return idx->qk_dtype == FP_QK_INT8 ? attn_impl<true>(q, k, v, q_scale, k_scale, idx, out, st)
                                     : attn_impl<false>(q, k, v, nullptr, nullptr, idx, out, st);
}

int fp_index_info(const fp_index *idx, int *S, int *Hq, int *Hkv, int *d, int *b, int *qk_dtype) {
  if (!idx) return FP_ERR_ARG;
  if (S) *S = idx->S;
  if (Hq) *Hq = idx->Hq;
  if (Hkv) *Hkv = idx->Hkv;
  if (d) *d = idx->d;
  if (b) *b = idx->b;
  if (qk_dtype) *qk_dtype = idx->qk_dtype;
  return FP_OK;
}

int fp_index_nnz(const fp_index *idx, int64_t *nnz, void *stream) {
  if (!idx || !nnz) return FP_ERR_ARG;
  if (!idx->built) return FP_ERR_STATE;
  std::vector<int> counts((size_t)idx->Hq * idx->n);
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FP_ERR_CUDA;
  if (cudaMemcpy(counts.data(), idx->counts, counts.size() * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
    return FP_ERR_CUDA;
  int64_t s = 0;
  for (int c : counts) s += c;
  *nnz = s;
  return FP_OK;
}

int fp_index_export(const fp_index *idx, int32_t *row_ptr, int32_t *col, uint8_t *pattern, float *jsd,
                    float *vhat, float *shat, float *pest, void *stream) {
  if (!idx) return FP_ERR_ARG;
  if (!idx->built) return FP_ERR_STATE;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FP_ERR_CUDA;
  const size_t Hn = (size_t)idx->Hq * idx->n;
  const size_t tri = (size_t)idx->n * (idx->n + 1) / 2;
  if (row_ptr || col) {
    std::vector<int> counts(Hn);
    if (cudaMemcpy(counts.data(), idx->counts, Hn * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
      return FP_ERR_CUDA;
    std::vector<int> padded;
    if (col) {
      padded.resize((size_t)idx->Hq * tri);
      if (cudaMemcpy(padded.data(), idx->cols, padded.size() * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
        return FP_ERR_CUDA;
    }
    int64_t pos = 0;
    for (int h = 0; h < idx->Hq; ++h)
      for (int r = 0; r < idx->n; ++r) {
        const size_t row = (size_t)h * idx->n + r;
        if (row_ptr) row_ptr[row] = (int32_t)pos;
        const int c = counts[row];
        if (col)
          memcpy(col + pos, padded.data() + (size_t)h * tri + (size_t)r * (r + 1) / 2, (size_t)c * 4);
        pos += c;
      }
    if (row_ptr) row_ptr[Hn] = (int32_t)pos;
  }
  if (pattern) {
    std::vector<int> p(idx->Hq);
    if (cudaMemcpy(p.data(), idx->pattern, p.size() * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
      return FP_ERR_CUDA;
    for (int h = 0; h < idx->Hq; ++h) pattern[h] = (uint8_t)p[h];
  }
  if (jsd && cudaMemcpy(jsd, idx->jsd, (size_t)idx->Hq * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
    return FP_ERR_CUDA;
  if (vhat && cudaMemcpy(vhat, idx->vhat, Hn * 4, cudaMemcpyDeviceToHost) != cudaSuccess) return FP_ERR_CUDA;
  if (shat && cudaMemcpy(shat, idx->shat, Hn * 4, cudaMemcpyDeviceToHost) != cudaSuccess) return FP_ERR_CUDA;
  if (pest && cudaMemcpy(pest, idx->pest, Hn * 4, cudaMemcpyDeviceToHost) != cudaSuccess) return FP_ERR_CUDA;
  return FP_OK;
}

int fp_get_device_error(void *stream) {
  int *err = device_error_word();
  if (!err) return FP_ERR_CUDA;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FP_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, err, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return FP_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpy(err, &zero, 4, cudaMemcpyHostToDevice) != cudaSuccess) return FP_ERR_CUDA;
    return (v & kDevErrTimeout) ? FP_ERR_TIMEOUT : FP_ERR_CUDA;
  }
  return FP_OK;
}

int fp_debug_wait_timeout(int timeout_us, void *stream) {
  if (timeout_us < 1 || timeout_us > 10000000) return FP_ERR_ARG;
  int *err = device_error_word();
  if (!err) return FP_ERR_CUDA;
  k_wait_timeout<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>((unsigned long long)timeout_us * 1000ull, err);
  return launch_status();
}

int fp_debug_qk_tile_i8(const int8_t *q8, const int8_t *k8, int S, int Hq, int Hkv, int d, int h, int p0,
                        int j0, int32_t *out, void *stream) {
  if (!q8 || !k8 || !out || d != 128 || S <= 0 || S % 128 || Hq <= 0 || Hkv <= 0 || Hq % Hkv) return FP_ERR_ARG;
  if (h < 0 || h >= Hq || p0 < 0 || j0 < 0 || p0 % 128 || j0 % 128 || p0 >= S || j0 >= S) return FP_ERR_ARG;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(out)) return FP_ERR_ARG;
  int *err = device_error_word();
  if (!err) return FP_ERR_CUDA;
  CUtensorMap tq, tk;
  if (!make_map(&tq, q8, true, (uint64_t)Hq * S) || !make_map(&tk, k8, true, (uint64_t)Hkv * S))
    return FP_ERR_CUDA;
  const int g = Hq / Hkv;
  k_qk_tile_i8<<<1, 128, 32768 + 1024, static_cast<cudaStream_t>(stream)>>>(
      tq, tk, h * S + p0, (h / g) * S + j0, out, err);
  return launch_status();
}

int fp_index_share(fp_index *idx, float eps, void *stream) {
  if (!idx || !(eps >= 0.f) || std::isnan(eps)) return FP_ERR_ARG;
  if (!idx->built) return FP_ERR_STATE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t smem = (size_t)idx->g * idx->g * sizeof(float);
  if (smem > 48 * 1024) return FP_ERR_ARG;
  k_share_classes<<<idx->Hkv, 256, smem, st>>>(idx->vhat, idx->n, idx->g, eps, idx->cls);
  int rc = launch_status();
  if (rc) return rc;
  k_share_union<<<(idx->Hq * idx->n + 7) / 8, 256, 0, st>>>(idx->cls, idx->Hq, idx->n, idx->g, idx->counts,
                                                            idx->cols);
  if ((rc = launch_status())) return rc;
  idx->shared = 1;
  return cudaEventRecord(idx->last_use, st) == cudaSuccess ? FP_OK : FP_ERR_CUDA;
}

int fp_index_csr(const fp_index *idx, int32_t *row_ptr, int32_t *col, void *stream) {
  if (!idx || !row_ptr) return FP_ERR_ARG;
  if (!idx->built) return FP_ERR_STATE;
  if (((uintptr_t)row_ptr & 3u) || ((uintptr_t)col & 3u)) return FP_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int N = idx->Hq * idx->n;
  k_scan_counts<<<1, 1024, 0, st>>>(idx->counts, N, row_ptr);
  int rc = launch_status();
  if (rc || !col) return rc;
  k_compact_rows<<<(N + 7) / 8, 256, 0, st>>>(idx->counts, idx->cols, row_ptr, idx->Hq, idx->n, col);
  return launch_status();
}

int fp_index_group_lists(const fp_index *idx, int32_t *grp_ptr, int32_t *grp_col, uint32_t *grp_mask,
                         void *stream) {
  if (!idx || !grp_ptr || (grp_col == nullptr) != (grp_mask == nullptr)) return FP_ERR_ARG;
  if (!idx->built) return FP_ERR_STATE;
  if (idx->g > 32) return FP_ERR_ARG;
  if (((uintptr_t)grp_ptr & 3u) || ((uintptr_t)grp_col & 3u) || ((uintptr_t)grp_mask & 3u)) return FP_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int N = idx->Hkv * idx->n;
  const size_t smem = (size_t)8 * idx->g * 32 * sizeof(uint32_t);
  // sizes of the unions (into the index's own counts scratch for the groups), their scan, then the lists
  k_group_lists<<<(N + 7) / 8, 256, smem, st>>>(idx->counts, idx->cols, idx->Hkv, idx->n, idx->g, nullptr,
                                                idx->gcount, nullptr, nullptr);
  int rc = launch_status();
  if (rc) return rc;
  k_scan_counts<<<1, 1024, 0, st>>>(idx->gcount, N, grp_ptr);
  if ((rc = launch_status()) || !grp_col) return rc;
  k_group_lists<<<(N + 7) / 8, 256, smem, st>>>(idx->counts, idx->cols, idx->Hkv, idx->n, idx->g, grp_ptr,
                                                nullptr, grp_col, grp_mask);
  return launch_status();
}

int fp_index_classes(const fp_index *idx, int32_t *cls, void *stream) {
  if (!idx || !cls) return FP_ERR_ARG;
  if (!idx->built) return FP_ERR_STATE;
  if (!idx->shared) {
    for (int h = 0; h < idx->Hq; ++h) cls[h] = h;
    return FP_OK;
  }
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FP_ERR_CUDA;
  return cudaMemcpy(cls, idx->cls, (size_t)idx->Hq * 4, cudaMemcpyDeviceToHost) == cudaSuccess ? FP_OK
                                                                                                : FP_ERR_CUDA;
}

int fp_choose_block_size(const fp_index *idx, float gamma, int *b, float *rho, void *stream) {
  if (!idx || !b || !(gamma > 0.f && gamma <= 1.f) || std::isnan(gamma)) return FP_ERR_ARG;
  if (!idx->built || idx->b != 128 || idx->ld != idx->S) return FP_ERR_STATE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  k_cover_count<<<(idx->Hq + 7) / 8, 256, 0, st>>>(idx->vhat, idx->Hq, idx->n, gamma, idx->cover);
  const int rc = launch_status();
  if (rc) return rc;
  std::vector<int> cover(idx->Hq);
  if (cudaStreamSynchronize(st) != cudaSuccess ||
      cudaMemcpy(cover.data(), idx->cover, cover.size() * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
    return FP_ERR_CUDA;
  double r = 0.0;
  for (int h = 0; h < idx->Hq; ++h) r += (double)cover[h] / idx->n;
  r /= idx->Hq;
  if (rho) *rho = (float)r;
  if (r < 0.1 && (idx->S + 63) / 64 <= kSelMaxN) *b = 64;
  else if (r >= 0.5) *b = 256;
  else *b = 128;
  return FP_OK;
}

int fp_debug_capture_i8(int which, int h, int tile, int chunk, int32_t *out) {
  if (which != 0 && which != 1) return FP_ERR_ARG;
  if (out && (!aligned16(out) || h < 0 || tile < 0 || chunk < 0)) return FP_ERR_ARG;
  std::lock_guard<std::mutex> lk(g_mu);
  if (which == 0) {
    g_cap.score = out;
    g_cap.s_h = h; g_cap.s_slice = tile; g_cap.s_ch = chunk;
  } else {
    g_cap.attn = out;
    g_cap.a_h = h; g_cap.a_qc = tile; g_cap.a_kc = chunk;
  }
  return FP_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free pattern statistics: the scratch of the statistics kernels
// lives in this fixed device array instead of an fp_index workspace.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
static __device__ __align__(256) unsigned char g_fp_stats_scratch[kNoAllocScratchBytes];

// Device address of g_fp_stats_scratch on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached; the lookup is
// redone in a new context of the device (after a device reset).
unsigned char *stats_scratch() {
  std::lock_guard<std::mutex> lk(g_mu);
  DevState *d = dev_state();
  if (!d) return nullptr;
  if (!d->scratch) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fp_stats_scratch) != cudaSuccess || p == nullptr) return nullptr;
    d->scratch = static_cast<unsigned char *>(p);
  }
  return d->scratch;
}

size_t round256(size_t x) { return ((x + 255) / 256) * 256; }

template <bool I8>
int stats_noalloc_impl(const void *q, const void *k, int S, int Hq, int Hkv, int d, int b, float tau,
                       const float *q_scale, const float *k_scale, float *vhat, float *shat, float *pest,
                       float *jsd, int32_t *pattern, cudaStream_t st) {
  const int n = (S + b - 1) / b, nch = (S + 127) / 128, npart = b < 128 ? nch * (128 / b) : nch;
  const size_t e_part = (size_t)Hq * npart * b;
  const size_t e_ksum = (size_t)Hkv * npart * 128, e_kbar = (size_t)Hkv * n * 128;
  const size_t need = 3 * round256(e_part * 4) + round256(e_ksum * 4) + round256(e_kbar * 4);
  if (need > kNoAllocScratchBytes) return FP_ERR_ARG;
  unsigned char *base = stats_scratch();
  if (!base) return FP_ERR_CUDA;
  int rc = set_smem_attrs<I8>();
  if (rc) return rc;
  int *err = device_error_word();
  if (!err) return FP_ERR_CUDA;
  char *cur = reinterpret_cast<char *>(base);
  float *pm = carve<float>(cur, e_part), *plo = carve<float>(cur, e_part), *phi = carve<float>(cur, e_part);
  float *ksum = carve<float>(cur, e_ksum), *kbar = carve<float>(cur, e_kbar);

  StatsJob J;
  J.S = S; J.Hq = Hq; J.Hkv = Hkv; J.d = d; J.b = b; J.n = n; J.nch = nch; J.g = Hq / Hkv;
  J.npart = npart;
  J.ld = S; J.ext_kbar = nullptr;
  J.q = q; J.k = k; J.q_scale = q_scale; J.k_scale = k_scale; J.tau = tau;
  J.pm = pm; J.plo = plo; J.phi = phi;
  J.ksum = ksum; J.kbar = kbar;
  J.vhat = vhat; J.shat = shat; J.pest = pest; J.jsd = jsd; J.pattern = pattern;
  if ((rc = launch_score<I8>(J, err, st))) return rc;
  return launch_head_stats<I8>(J, st);
}

bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

}  // namespace

extern "C" {

int fp_pattern_stats_noalloc(const void *q, const void *k, int S, int Hq, int Hkv, int d, int b, float tau,
                             int qk_dtype, const float *q_scale, const float *k_scale, float *vhat, float *shat,
                             float *pest, float *jsd, int32_t *pattern, void *stream) {
  if (!q || !k || !vhat || !shat || !pest || !jsd || !pattern) return FP_ERR_ARG;
  if (!shape_ok(S, Hq, Hkv, d, b)) return FP_ERR_ARG;
  if (!(tau >= 0.f) || std::isnan(tau)) return FP_ERR_ARG;
  if (qk_dtype != FP_QK_BF16 && qk_dtype != FP_QK_INT8) return FP_ERR_ARG;
  if (qk_dtype == FP_QK_INT8 && (!q_scale || !k_scale)) return FP_ERR_ARG;
  if (!aligned16(q) || !aligned16(k)) return FP_ERR_ARG;
  if (!aligned4(vhat) || !aligned4(shat) || !aligned4(pest) || !aligned4(jsd) || !aligned4(pattern))
    return FP_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return qk_dtype == FP_QK_INT8
             ? stats_noalloc_impl<true>(q, k, S, Hq, Hkv, d, b, tau, q_scale, k_scale, vhat, shat, pest, jsd,
                                        pattern, st)
             : stats_noalloc_impl<false>(q, k, S, Hq, Hkv, d, b, tau, nullptr, nullptr, vhat, shat, pest, jsd,
                                         pattern, st);
}

const char *fp_strerror(int code) {
  switch (code) {
    case FP_OK: return "ok";
    case FP_ERR_ARG: return "invalid argument";
    case FP_ERR_CUDA: return "CUDA call failed";
    case FP_ERR_TIMEOUT: return "device wait timed out";
    case FP_ERR_STATE: return "index not built or built for another shape";
    default: return "unknown error";
  }
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Packed variable-length sequences: one index per sequence over strided views
// of the packed [H][T][d] tensors (heads T rows apart, sequence s at rows
// cu_seqlens[s] .. cu_seqlens[s+1]-1 of every head).
// ---------------------------------------------------------------------------
struct fp_varlen {
  int nseq, T, Hq, Hkv, d, b;
  std::vector<int> cu;              // nseq + 1 offsets
  std::vector<fp_index *> idx;      // nullptr for empty sequences
  int built, qk_dtype;
};

extern "C" {

void fp_varlen_free(fp_varlen *V) {
  if (!V) return;
  for (fp_index *I : V->idx) fp_index_free(I);
  delete V;
}

int fp_varlen_create(const int32_t *cu_seqlens, int nseq, int Hq, int Hkv, int d, int b, fp_varlen **out) {
  if (!out) return FP_ERR_ARG;
  *out = nullptr;
  if (!cu_seqlens || nseq <= 0 || cu_seqlens[0] != 0) return FP_ERR_ARG;
  for (int s = 0; s < nseq; ++s) {
    const int len = cu_seqlens[s + 1] - cu_seqlens[s];
    if (len < 0 || (len > 0 && !shape_ok(len, Hq, Hkv, d, b))) return FP_ERR_ARG;
  }
  const int T = cu_seqlens[nseq];
  if (T <= 0 || !shape_ok(1, Hq, Hkv, d, b) || (int64_t)Hq * T > (int64_t)INT32_MAX) return FP_ERR_ARG;
  fp_varlen *V = new (std::nothrow) fp_varlen();
  if (!V) return FP_ERR_CUDA;
  V->nseq = nseq; V->T = T; V->Hq = Hq; V->Hkv = Hkv; V->d = d; V->b = b;
  V->cu.assign(cu_seqlens, cu_seqlens + nseq + 1);
  V->idx.assign(nseq, nullptr);
  V->built = 0;
  V->qk_dtype = FP_QK_BF16;
  for (int s = 0; s < nseq; ++s) {
    const int len = V->cu[s + 1] - V->cu[s];
    if (len == 0) continue;
    const int rc = index_create(len, T, Hq, Hkv, d, b, &V->idx[s]);
    if (rc) {
      fp_varlen_free(V);
      return rc;
    }
  }
  *out = V;
  return FP_OK;
}

int fp_varlen_build_index(fp_varlen *V, const void *q, const void *k, float gamma, float tau, int qk_dtype,
                          const float *q_scale, const float *k_scale, void *stream) {
  if (!V || !q || !k) return FP_ERR_ARG;
  if (!(gamma > 0.f && gamma <= 1.f) || !(tau >= 0.f) || std::isnan(gamma) || std::isnan(tau)) return FP_ERR_ARG;
  if (qk_dtype != FP_QK_BF16 && qk_dtype != FP_QK_INT8) return FP_ERR_ARG;
  const bool i8 = qk_dtype == FP_QK_INT8;
  if (i8 && (!q_scale || !k_scale)) return FP_ERR_ARG;
  if (!aligned16(q) || !aligned16(k)) return FP_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t elt = i8 ? 1 : 2;
  V->built = 0;
  for (int s = 0; s < V->nseq; ++s) {
    fp_index *I = V->idx[s];
    if (!I) continue;
    const size_t off = (size_t)V->cu[s] * V->d * elt;  // bytes to the sequence's first row in head 0
    const void *qs = static_cast<const char *>(q) + off, *ks = static_cast<const char *>(k) + off;
    I->built = 0;
    const int rc = i8 ? build_index_impl<true>(qs, ks, gamma, tau, q_scale + (size_t)s * V->Hq,
                                               k_scale + (size_t)s * V->Hkv, I, st)
                      : build_index_impl<false>(qs, ks, gamma, tau, nullptr, nullptr, I, st);
    if (rc) return rc;
    I->built = 1;
    I->qk_dtype = qk_dtype;
  }
  V->built = 1;
  V->qk_dtype = qk_dtype;
  return FP_OK;
}

int fp_varlen_sparse_attn(const fp_varlen *V, const void *q, const void *k, const void *v, const float *q_scale,
                          const float *k_scale, void *out, void *stream) {
  if (!V || !q || !k || !v || !out) return FP_ERR_ARG;
  if (!V->built) return FP_ERR_STATE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return FP_ERR_ARG;
  const bool i8 = V->qk_dtype == FP_QK_INT8;
  if (i8 && (!q_scale || !k_scale)) return FP_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t elt = i8 ? 1 : 2;
  for (int s = 0; s < V->nseq; ++s) {
    const fp_index *I = V->idx[s];
    if (!I) continue;
    const size_t row = (size_t)V->cu[s] * V->d;
    const void *qs = static_cast<const char *>(q) + row * elt, *ks = static_cast<const char *>(k) + row * elt;
    const void *vs = static_cast<const char *>(v) + row * 2;
    void *os = static_cast<char *>(out) + row * 2;
    const int rc = i8 ? attn_impl<true>(qs, ks, vs, q_scale + (size_t)s * V->Hq, k_scale + (size_t)s * V->Hkv, I,
                                        os, st)
                      : attn_impl<false>(qs, ks, vs, nullptr, nullptr, I, os, st);
    if (rc) return rc;
  }
  return FP_OK;
}

int fp_varlen_index(const fp_varlen *V, int seq, const fp_index **out) {
  if (!V || !out || seq < 0 || seq >= V->nseq) return FP_ERR_ARG;
  *out = V->idx[seq];
  return FP_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Rotary-embedding epilogue with block pooling, and the index build that
// takes its block means.
// ---------------------------------------------------------------------------
extern "C" {

int fp_rope_pool(const void *q_in, const void *k_in, const float *rope_cos, const float *rope_sin, int S, int Hq,
                 int Hkv, int d, int b, void *q_out, void *k_out, float *qbar, float *kbar, void *stream) {
  if (!q_in || !k_in || !rope_cos || !rope_sin || !q_out || !k_out || !qbar || !kbar) return FP_ERR_ARG;
  if (!shape_ok(S, Hq, Hkv, d, b)) return FP_ERR_ARG;
  if (!aligned16(q_in) || !aligned16(k_in) || !aligned16(rope_cos) || !aligned16(rope_sin) || !aligned16(q_out) ||
      !aligned16(k_out) || !aligned16(qbar) || !aligned16(kbar))
    return FP_ERR_ARG;
  const int n = (S + b - 1) / b;
  k_rope_pool<<<dim3(Hq + Hkv, n), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16 *>(q_in), static_cast<const __nv_bfloat16 *>(k_in), rope_cos, rope_sin, S, Hq, b,
      n, static_cast<__nv_bfloat16 *>(q_out), static_cast<__nv_bfloat16 *>(k_out), qbar, kbar);
  return launch_status();
}

int fp_build_index_pooled(const void *q, const void *k, const float *qbar, const float *kbar, int S, int Hq, int Hkv,
                          int d, int b, float gamma, float tau, fp_index *idx, void *stream) {
  if (!idx || !q || !k || !qbar || !kbar) return FP_ERR_ARG;
  if (!shape_ok(S, Hq, Hkv, d, b)) return FP_ERR_ARG;
  if (S != idx->S || Hq != idx->Hq || Hkv != idx->Hkv || d != idx->d || b != idx->b) return FP_ERR_STATE;
  if (idx->ld != idx->S) return FP_ERR_STATE;
  if (!(gamma > 0.f && gamma <= 1.f) || !(tau >= 0.f) || std::isnan(gamma) || std::isnan(tau)) return FP_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(qbar) || !aligned16(kbar)) return FP_ERR_ARG;
  idx->built = 0;
  const int rc = build_index_impl<false>(q, k, gamma, tau, nullptr, nullptr, idx, static_cast<cudaStream_t>(stream),
                                         qbar, kbar);
  if (rc == FP_OK) {
    idx->built = 1;
    idx->qk_dtype = FP_QK_BF16;
  }
  return rc;
}

}  // extern "C"

// share_kernels.cuh -- head-pattern sharing and the block-size statistic.
//
// The maplevalley article (section 5, future directions) names two variants
// without giving a rule: similar heads sharing one sparse pattern, and a
// block size adjusted to the complexity of the content.  Written conventions:
//   sharing     within a GQA group, in head order, head a joins the class of
//               the earliest earlier representative b with JSD(vhat_a,
//               vhat_b) < eps (natural log); every head of a class attends
//               to the union of the class members' block lists;
//   block size  k_h = fewest key blocks whose vhat (at b = 128) sums to at
//               least gamma; rho = mean_h k_h / n picks 64 (rho < 0.1 and
//               S/64 <= 1024), 256 (rho >= 0.5) or 128 (host side).
#pragma once

#include "ptx.cuh"

namespace fpk {

// k_share_classes: grid (Hkv), block 256.  cls[h] = the class representative
// (absolute head index) of every query head of KV head blockIdx.x.
__global__ void __launch_bounds__(256)
    k_share_classes(const float *__restrict__ vhat, int n, int g, float eps, int *__restrict__ cls) {
  extern __shared__ float jsd_s[];  // [g][g]
  const int kvh = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int h0 = kvh * g;
  // JSD of every pair a > b, one warp per pair, fixed-order sums
  for (int pr = warp; pr < g * g; pr += nw) {
    const int a = pr / g, b = pr % g;
    if (b >= a) continue;
    const float *pa = vhat + (size_t)(h0 + a) * n, *pb = vhat + (size_t)(h0 + b) * n;
    float js = 0.f;
    for (int c = lane; c < n; c += 32) {
      const float p = pa[c], q = pb[c], m = 0.5f * (p + q);
      if (p > 0.f) js += 0.5f * p * logf(p / m);
      if (q > 0.f) js += 0.5f * q * logf(q / m);
    }
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) js += __shfl_xor_sync(0xffffffffu, js, s);
    if (lane == 0) jsd_s[a * g + b] = js;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int a = 0; a < g; ++a) {
      int c = a;
      for (int b = 0; b < a; ++b)
        if (cls[h0 + b] == h0 + b && jsd_s[a * g + b] < eps) {
          c = b;
          break;
        }
      cls[h0 + a] = h0 + c;
    }
  }
}

// k_share_union: one warp per (representative head, query block r), block 256.
// The members' lists of row r are read into a 1024-bit shared bitmap, then
// the ascending union is written to every member's row (rows of different
// classes or blocks are disjoint, so no warp reads a row another writes).
__global__ void __launch_bounds__(256)
    k_share_union(const int *__restrict__ cls, int Hq, int n, int g, int *__restrict__ counts,
                  int *__restrict__ cols) {
  __shared__ uint32_t bm_s[8][32];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + w;
  if (row >= Hq * n) return;
  const int h = row / n, r = row % n;
  if (cls[h] != h) return;  // a member: its representative's warp writes its rows
  const int h0 = (h / g) * g;
  int members = 0;
  for (int m = h0; m < h0 + g; ++m) members += cls[m] == h;
  if (members < 2) return;
  uint32_t *bm = bm_s[w];
  bm[lane] = 0u;
  __syncwarp();
  const size_t tri = (size_t)n * (n + 1) / 2, off = (size_t)r * (r + 1) / 2;
  for (int m = h0; m < h0 + g; ++m) {
    if (cls[m] != h) continue;
    const int cnt = counts[(size_t)m * n + r];
    const int *list = cols + (size_t)m * tri + off;
    for (int e = lane; e < cnt; e += 32) atomicOr(&bm[list[e] >> 5], 1u << (list[e] & 31));
  }
  __syncwarp();
  const uint32_t word = bm[lane];
  // exclusive prefix of the set bits over the lanes (words in ascending order)
  uint32_t pre = __popc(word);
#pragma unroll
  for (int s = 1; s < 32; s <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, pre, s);
    if (lane >= s) pre += v;
  }
  const uint32_t total = __shfl_sync(0xffffffffu, pre, 31);
  pre -= __popc(word);
  for (int m = h0; m < h0 + g; ++m) {
    if (cls[m] != h) continue;
    int *list = cols + (size_t)m * tri + off;
    uint32_t wv = word;
    int pos = (int)pre;
    while (wv) {
      const int bit = __ffs(wv) - 1;
      wv &= wv - 1u;
      list[pos++] = lane * 32 + bit;
    }
    if (lane == 0) counts[(size_t)m * n + r] = (int)total;
  }
}

// k_cover_count: one warp per head, block 256.  cover[h] = fewest key blocks
// whose vhat sums to at least gamma, taken by descending vhat (ties by lower
// index); gamma >= 1 or a total below gamma gives n.  The threshold is found
// by bisection on the fp32 bit pattern, the sums in fixed point as in k_cut.
__global__ void __launch_bounds__(256)
    k_cover_count(const float *__restrict__ vhat, int Hq, int n, float gamma, int *__restrict__ cover) {
  const int h = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (h >= Hq) return;
  constexpr int NL = 32;  // n <= 1024
  constexpr float kFx = 1073741824.f;
  float v[NL];
#pragma unroll
  for (int i = 0; i < NL; ++i) {
    const int c = lane + 32 * i;
    v[i] = c < n ? fmaxf(vhat[(size_t)h * n + c], 0.f) : 0.f;
  }
  auto lane_sum = [&](uint32_t t, uint32_t &cnt) -> uint32_t {
    float f = 0.f;
    cnt = 0u;
#pragma unroll
    for (int i = 0; i < NL; ++i) {
      const bool ge = __float_as_uint(v[i]) >= t;
      f += ge ? v[i] : 0.f;
      cnt += ge ? 1u : 0u;
    }
    return __float2uint_rn(f * kFx);
  };
  const uint32_t need = __float2uint_ru(fminf(gamma, 1.f) * kFx);
  uint32_t cnt;
  const uint32_t tot = redux_add_u32(lane_sum(1u, cnt));
  if (gamma >= 1.f || tot < need) {
    if (lane == 0) cover[h] = n;
    return;
  }
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
#pragma unroll
  for (int i = 0; i < NL; ++i) {
    const uint32_t key = __float_as_uint(v[i]);
    if (key != 0u) {
      kmin = min(kmin, key);
      kmax = max(kmax, key);
    }
  }
  uint32_t lo = redux_min_u32(kmin), hi = redux_max_u32(kmax) + 1u;
  uint32_t c_lo = redux_add_u32(cnt), c_hi = 0u, f_hi = 0u;
  while (hi - lo > 1u && c_lo - c_hi > 1u) {
    const uint32_t mid = lo + ((hi - lo) >> 1);
    uint32_t cm;
    const uint32_t f = redux_add_u32(lane_sum(mid, cm)), cs = redux_add_u32(cm);
    if (f >= need) {
      lo = mid;
      c_lo = cs;
    } else {
      hi = mid;
      c_hi = cs;
      f_hi = f;
    }
  }
  uint32_t T;
  if (c_lo - c_hi == 1u) {
    uint32_t tb = 0u;
#pragma unroll
    for (int i = 0; i < NL; ++i) {
      const uint32_t key = __float_as_uint(v[i]);
      if (key >= lo && key < hi) tb = key;
    }
    T = redux_max_u32(tb);
  } else {
    T = lo;
  }
  // blocks above T, then ties at T until the sum reaches gamma
  uint32_t above = 0u, ties = 0u;
#pragma unroll
  for (int i = 0; i < NL; ++i) {
    const uint32_t key = __float_as_uint(v[i]);
    above += key > T ? 1u : 0u;
    ties += key == T ? 1u : 0u;
  }
  above = redux_add_u32(above);
  ties = redux_add_u32(ties);
  const uint32_t t_fx = __float2uint_rn(__uint_as_float(T) * kFx);
  uint32_t acc = f_hi, take = 0u;
  while (take < ties && acc < need) {
    acc += t_fx;
    ++take;
  }
  if (lane == 0) cover[h] = (int)(above + take);
}

}  // namespace fpk

namespace fpk {

// ---------------------------------------------------------------------------
// Compact block lists on the device (first article, section 3.2: compact job
// lists; second article, section 1.1 step 3: block-level index).
// ---------------------------------------------------------------------------

// k_scan_counts: one CTA of 1024 threads.  ptr[i] = sum_{j < i} counts[j] for
// i in [0, N], each thread scanning a contiguous segment.
__global__ void __launch_bounds__(1024) k_scan_counts(const int *__restrict__ counts, int N, int *__restrict__ ptr) {
  __shared__ int wsum[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int seg = (N + 1023) / 1024, lo = min(N, tid * seg), hi = min(N, lo + seg);
  int s = 0;
  for (int i = lo; i < hi; ++i) s += counts[i];
  int incl = s;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += v;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = wsum[lane];
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, w, d);
      if (lane >= d) w += v;
    }
    wsum[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  int run = incl - s + (warp > 0 ? wsum[warp - 1] : 0);
  for (int i = lo; i < hi; ++i) {
    ptr[i] = run;
    run += counts[i];
  }
  if (tid == 1023) ptr[N] = wsum[31];
}

// k_compact_rows: one warp per row (h, r): the padded list of the row to
// col[ptr[row] ..).
__global__ void __launch_bounds__(256)
    k_compact_rows(const int *__restrict__ counts, const int *__restrict__ cols, const int *__restrict__ ptr, int Hq,
                   int n, int *__restrict__ col) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= Hq * n) return;
  const int h = row / n, r = row % n;
  const int *src = cols + (size_t)h * ((size_t)n * (n + 1) / 2) + (size_t)r * (r + 1) / 2;
  const int cnt = counts[row];
  int *dst = col + ptr[row];
  for (int e = lane; e < cnt; e += 32) dst[e] = src[e];
}

// k_group_lists: one warp per (KV head j, query block r), block 256, dynamic
// shared memory 8 * g * 128 bytes.  The g query heads' lists of row r as
// 1024-bit maps; count mode (col == null) writes the size of their union to
// gcount[j*n + r]; write mode writes the union in ascending order to
// col[gptr[j*n + r] ..) with mask bit m set when head j*g + m lists the block.
__global__ void __launch_bounds__(256)
    k_group_lists(const int *__restrict__ counts, const int *__restrict__ cols, int Hkv, int n, int g,
                  const int *__restrict__ gptr, int *__restrict__ gcount, int *__restrict__ col,
                  uint32_t *__restrict__ mask) {
  extern __shared__ uint32_t gbm[];  // [8 warps][g][32 words]
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + w;
  if (row >= Hkv * n) return;
  const int j = row / n, r = row % n;
  uint32_t *bm = gbm + (size_t)w * g * 32;
  for (int m = 0; m < g; ++m) bm[m * 32 + lane] = 0u;
  __syncwarp();
  const size_t tri = (size_t)n * (n + 1) / 2, off = (size_t)r * (r + 1) / 2;
  for (int m = 0; m < g; ++m) {
    const int h = j * g + m;
    const int cnt = counts[(size_t)h * n + r];
    const int *list = cols + (size_t)h * tri + off;
    for (int e = lane; e < cnt; e += 32) atomicOr(&bm[m * 32 + (list[e] >> 5)], 1u << (list[e] & 31));
  }
  __syncwarp();
  uint32_t word = 0u;
  for (int m = 0; m < g; ++m) word |= bm[m * 32 + lane];
  uint32_t pre = __popc(word);
#pragma unroll
  for (int s = 1; s < 32; s <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, pre, s);
    if (lane >= s) pre += v;
  }
  const uint32_t total = __shfl_sync(0xffffffffu, pre, 31);
  pre -= __popc(word);
  if (col == nullptr) {
    if (lane == 0) gcount[row] = (int)total;
    return;
  }
  int pos = gptr[row] + (int)pre;
  uint32_t wv = word;
  while (wv) {
    const int bit = __ffs(wv) - 1;
    wv &= wv - 1u;
    uint32_t mk = 0u;
    for (int m = 0; m < g; ++m) mk |= ((bm[m * 32 + lane] >> bit) & 1u) << m;
    col[pos] = lane * 32 + bit;
    mask[pos] = mk;
    ++pos;
  }
}

}  // namespace fpk

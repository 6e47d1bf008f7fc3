// rope_pool.cuh -- rotary embedding epilogue with block pooling on sm_100a.
//
// The projection step of the FAST-Prefill article (section 1.1: Q = X W_q,
// K = X W_k) ends with the rotary embedding; this kernel is that epilogue,
// and while each rotated row is in registers it also accumulates the block
// means the index generation needs (section 2.1 block pooling), so the index
// pass does not read Q again to pool it.
//
// Rotate-half convention with the caller's tables: for i < 64,
//   out[p][i]      = x[p][i] cos[p][i] - x[p][i+64] sin[p][i]
//   out[p][i + 64] = x[p][i+64] cos[p][i] + x[p][i] sin[p][i]
// in fp32, stored as bf16 (round to nearest even); the means are over the
// stored (rounded) values, b rows per block or S - (n-1)b for a partial last
// block.  Pure streaming: 2 bytes read and 2 written per element plus the
// tables (shared by all heads, so mostly served from L2).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace fpk {

// grid (Hq + Hkv, n), block 256: the heads of a block of positions are
// neighbours in launch order, so that block's cos/sin rows come from DRAM
// once and from L2 for the other heads.  Thread = (row slot rs in 0..31, pair
// group j in 0..7): dims 8j..8j+7 and 64+8j..64+8j+7 of rows rs, rs+32, ...
__global__ void __launch_bounds__(256)
    k_rope_pool(const __nv_bfloat16 *q_in, const __nv_bfloat16 *k_in,
                const float *__restrict__ cosT, const float *__restrict__ sinT, int S, int Hq, int b, int n,
                __nv_bfloat16 *q_out, __nv_bfloat16 *k_out, float *__restrict__ qbar, float *__restrict__ kbar) {
  __shared__ float red[8][128];
  const int hh = blockIdx.x, r = blockIdx.y, tid = threadIdx.x;
  const bool isq = hh < Hq;
  const int h = isq ? hh : hh - Hq;
  // in and out may be the same tensor: every element is read, then written,
  // by the same thread
  const __nv_bfloat16 *in = (isq ? q_in : k_in) + (size_t)h * S * 128;
  __nv_bfloat16 *out = (isq ? q_out : k_out) + (size_t)h * S * 128;
  float *mean = (isq ? qbar : kbar) + ((size_t)h * n + r) * 128;
  const int p0 = r * b, rows = min(b, S - p0);
  const int j = tid & 7, rs = tid >> 3;
  float acc[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) acc[e] = 0.f;
#pragma unroll 4
  for (int rr = rs; rr < rows; rr += 32) {
    const size_t p = (size_t)(p0 + rr);
    const uint4 xl = *reinterpret_cast<const uint4 *>(in + p * 128 + 8 * j);
    const uint4 xh = *reinterpret_cast<const uint4 *>(in + p * 128 + 64 + 8 * j);
    const float4 c0 = *reinterpret_cast<const float4 *>(cosT + p * 64 + 8 * j);
    const float4 c1 = *reinterpret_cast<const float4 *>(cosT + p * 64 + 8 * j + 4);
    const float4 s0 = *reinterpret_cast<const float4 *>(sinT + p * 64 + 8 * j);
    const float4 s1 = *reinterpret_cast<const float4 *>(sinT + p * 64 + 8 * j + 4);
    const float cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
    const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
    const uint32_t wl[4] = {xl.x, xl.y, xl.z, xl.w}, wh[4] = {xh.x, xh.y, xh.z, xh.w};
    uint32_t ol[4], oh[4];
#pragma unroll
    for (int e2 = 0; e2 < 4; ++e2) {
      const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&wl[e2]));
      const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&wh[e2]));
      const int e = 2 * e2;
      const float lo0 = fmaf(a.x, cv[e], -c.x * sv[e]), lo1 = fmaf(a.y, cv[e + 1], -c.y * sv[e + 1]);
      const float hi0 = fmaf(c.x, cv[e], a.x * sv[e]), hi1 = fmaf(c.y, cv[e + 1], a.y * sv[e + 1]);
      const __nv_bfloat162 bl = __floats2bfloat162_rn(lo0, lo1), bh = __floats2bfloat162_rn(hi0, hi1);
      ol[e2] = *reinterpret_cast<const uint32_t *>(&bl);
      oh[e2] = *reinterpret_cast<const uint32_t *>(&bh);
      const float2 fl = __bfloat1622float2(bl), fh = __bfloat1622float2(bh);
      acc[e] += fl.x;
      acc[e + 1] += fl.y;
      acc[8 + e] += fh.x;
      acc[8 + e + 1] += fh.y;
    }
    *reinterpret_cast<uint4 *>(out + p * 128 + 8 * j) = make_uint4(ol[0], ol[1], ol[2], ol[3]);
    *reinterpret_cast<uint4 *>(out + p * 128 + 64 + 8 * j) = make_uint4(oh[0], oh[1], oh[2], oh[3]);
  }
  // column sums: the 4 row slots of a warp with the same j (lanes j, j+8,
  // j+16, j+24), then the 8 warps in order
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 8);
    acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 16);
  }
  const int warp = tid >> 5, lane = tid & 31;
  if (lane < 8) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      red[warp][8 * lane + e] = acc[e];
      red[warp][64 + 8 * lane + e] = acc[8 + e];
    }
  }
  __syncthreads();
  if (tid < 128) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) s += red[w][tid];
    mean[tid] = s / (float)rows;
  }
}

}  // namespace fpk

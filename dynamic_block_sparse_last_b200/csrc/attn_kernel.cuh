// attn_kernel.cuh -- block-sparse GQA causal flash attention on sm_100a.
//
// Each query block attends only to the key blocks its index lists (FAST-Prefill
// article, figure 3 and section 1.1): out_p = sum over listed keys j <= p of
// softmax_j(q_p . k_j / sqrt(d)) v_j.  Online softmax in fp32, bf16 P.V.
//
// CTA = (query head h, 128-row query tile qc).  CTAs are numbered heavy first
// (descending qc) and, inside one qc, by head, so the g heads of a GQA group
// run side by side and their K/V chunks are served from L2 after the first
// fetch.  A KV block of b keys is processed as b/128 chunks of 128 keys.
//
// Warp roles (192 threads):
//   warps 0-3  softmax / correction / epilogue; thread = one query row = one
//              TMEM lane
//   warp 4     TMA producer: Q tile once, then K chunks (3-stage ring) and V
//              chunks (2-stage ring) in list order
//   warp 5     TMEM owner and MMA issuer (one thread)
// TMEM (512 columns): S double buffer at [0,128) and [128,256), O at [256,384).
// Shared memory: Q 32 KiB, K 3 x 32 KiB, V 2 x 32 KiB, P 32 KiB (bf16 Q/K;
// half the Q/K bytes for int8), all in the 128-byte-swizzled K-major layout
// (V is read MN-major).
//
// Pipeline per chunk j (MMA thread order):
//   QK(j+1) -> S[(j+1)&1]      as soon as K(j+1) has landed
//   wait P(j), V(j); PV(j): O += P V
// Softmax thread for chunk j: S -> registers, rowmax, P = 2^(s*scale2 - m)
// with a lazily raised reference max m (raised only when the row max exceeds
// it by more than 2^8; the correction O *= 2^(m_old - m_new) then runs after
// PV(j-1) has completed), P -> shared memory, signal.
#pragma once

#include "ptx.cuh"

namespace fpk {

struct AttnParams {
  int S, Hq, Hkv, b, n, g;
  const int *counts;  // [Hq][n]
  const int *cols;    // padded lists, row (h, r) at h*n(n+1)/2 + r(r+1)/2
  const float *q_scale, *k_scale;  // int8 only
  float scale2;                    // log2(e)/sqrt(d)
  __nv_bfloat16 *out;              // [Hq][S][128]
  int *err;
};

template <bool I8>
struct AttnCfg {
  static constexpr int kQKTile = I8 ? 16384 : 32768;
  static constexpr int kVTile = 32768;
  static constexpr int kKStages = 3;
  static constexpr int kVStages = 2;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kQKTile;
  static constexpr int kVOff = kKOff + kKStages * kQKTile;
  static constexpr int kPOff = kVOff + kVStages * kVTile;
  static constexpr int kSmem = kPOff + 32768 + 1024;
  static constexpr int kThreads = 192;
};

// Number of 128-key chunks query tile qc attends to, given the list length of
// its query block (ascending block list whose last entry is the diagonal).
__device__ __forceinline__ int attn_chunks(int cnt, int b, int qc) {
  const int per = b / 128;
  return (cnt - 1) * per + (qc % per) + 1;
}

template <bool I8>
__global__ void __launch_bounds__(192, 1)
    k_sparse_attn(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, AttnParams P) {
  using C = AttnCfg<I8>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_q, bar_kfull[3], bar_kempty[3], bar_vfull[2], bar_vempty[2],
      bar_sfull[2], bar_pfull, bar_odone;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nq = P.S / 128;
  const int qc = nq - 1 - (int)(blockIdx.x / P.Hq);
  const int h = blockIdx.x % P.Hq;
  const int kvh = h / P.g;
  const int per = P.b / 128;
  const int r = (qc * 128) / P.b;
  const size_t list_off = (size_t)h * ((size_t)P.n * (P.n + 1) / 2) + (size_t)r * (r + 1) / 2;
  const int cnt = P.counts[(size_t)h * P.n + r];
  const int L = attn_chunks(cnt, P.b, qc);

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sq = base + C::kQOff, sk = base + C::kKOff, sv = base + C::kVOff, sp = base + C::kPOff;
  uint8_t *const p_gen = smem_raw + (sp - smem_u32(smem_raw));

  if (threadIdx.x == 0) {
    abort_sh = 0;
    mbar_init(smem_u32(&bar_q), 1);
    for (int s = 0; s < 3; ++s) {
      mbar_init(smem_u32(&bar_kfull[s]), 1);
      mbar_init(smem_u32(&bar_kempty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&bar_vfull[s]), 1);
      mbar_init(smem_u32(&bar_vempty[s]), 1);
      mbar_init(smem_u32(&bar_sfull[s]), 1);
    }
    mbar_init(smem_u32(&bar_pfull), 4);
    mbar_init(smem_u32(&bar_odone), 1);
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(&tmem_base_sh), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  volatile int *abort_flag = &abort_sh;

  if (warp == 4) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_map(&tm_q);
      tma_prefetch_map(&tm_k);
      tma_prefetch_map(&tm_v);
      const int qrow = h * P.S + qc * 128;
      mbar_expect_tx(smem_u32(&bar_q), C::kQKTile);
      tma_load_2d(sq, &tm_q, 0, qrow, smem_u32(&bar_q));
      if (!I8) tma_load_2d(sq + 16384, &tm_q, 64, qrow, smem_u32(&bar_q));
      const int *lst = P.cols + list_off;
      int j = 0;
      bool ok = true;
      for (int e = 0; e < cnt && ok; ++e) {
        const int c = lst[e];
        for (int k = 0; k < per && ok; ++k) {
          const int kc = c * per + k;
          if (kc > qc) break;
          const int krow = kvh * P.S + kc * 128;
          const int ks = j % 3, vs = j & 1;
          if (j >= 3 && !mbar_wait(smem_u32(&bar_kempty[ks]), ((j / 3) - 1) & 1, abort_flag, P.err)) {
            ok = false;
            break;
          }
          mbar_expect_tx(smem_u32(&bar_kfull[ks]), C::kQKTile);
          tma_load_2d(sk + ks * C::kQKTile, &tm_k, 0, krow, smem_u32(&bar_kfull[ks]));
          if (!I8) tma_load_2d(sk + ks * C::kQKTile + 16384, &tm_k, 64, krow, smem_u32(&bar_kfull[ks]));
          if (j >= 2 && !mbar_wait(smem_u32(&bar_vempty[vs]), ((j / 2) - 1) & 1, abort_flag, P.err)) {
            ok = false;
            break;
          }
          mbar_expect_tx(smem_u32(&bar_vfull[vs]), C::kVTile);
          tma_load_2d(sv + vs * C::kVTile, &tm_v, 0, krow, smem_u32(&bar_vfull[vs]));
          tma_load_2d(sv + vs * C::kVTile + 16384, &tm_v, 64, krow, smem_u32(&bar_vfull[vs]));
          ++j;
        }
      }
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_qk = I8 ? idesc_i8(128, 128) : idesc_bf16(128, 128, 0);
      const uint32_t id_pv = idesc_bf16(128, 128, 1);
      auto issue_qk = [&](int j) -> bool {
        const int ks = j % 3;
        if (!mbar_wait(smem_u32(&bar_kfull[ks]), (j / 3) & 1, abort_flag, P.err)) return false;
        tc_fence_after();
        const uint32_t kb = sk + ks * C::kQKTile;
        const uint32_t d_tmem = tmem + (j & 1) * 128;
        if (I8) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_i8_ss(d_tmem, umma_desc_sw128(sq + kk * 32, 16, 1024),
                      umma_desc_sw128(kb + kk * 32, 16, 1024), id_qk, kk > 0);
        } else {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            mma_bf16_ss(d_tmem, umma_desc_sw128(sq + off, 16, 1024),
                        umma_desc_sw128(kb + off, 16, 1024), id_qk, kk > 0);
          }
        }
        tc_commit(smem_u32(&bar_sfull[j & 1]));
        tc_commit(smem_u32(&bar_kempty[ks]));
        return true;
      };
      bool ok = mbar_wait(smem_u32(&bar_q), 0, abort_flag, P.err) && issue_qk(0);
      for (int j = 0; ok && j < L; ++j) {
        if (j + 1 < L && !issue_qk(j + 1)) break;
        if (!mbar_wait(smem_u32(&bar_pfull), j & 1, abort_flag, P.err)) break;
        const int vs = j & 1;
        if (!mbar_wait(smem_u32(&bar_vfull[vs]), (j >> 1) & 1, abort_flag, P.err)) break;
        tc_fence_after();
        const uint32_t vb = sv + vs * C::kVTile;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t aoff = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16_ss(tmem + 256, umma_desc_sw128(sp + aoff, 16, 1024),
                      umma_desc_sw128(vb + kk * 2048, 16384, 1024), id_pv, (j > 0 || kk > 0));
        }
        tc_commit(smem_u32(&bar_odone));
        tc_commit(smem_u32(&bar_vempty[vs]));
      }
    }
  } else {
    // ---------------------------------------------------------------- softmax
    const int row = warp * 32 + lane;
    const uint32_t lane_off = ((uint32_t)(warp * 32)) << 16;
    float scale2 = P.scale2;
    if (I8) scale2 *= P.q_scale[h] * P.k_scale[kvh];
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < L; ++j) {
      if (!mbar_wait(smem_u32(&bar_sfull[j & 1]), (j >> 1) & 1, abort_flag, P.err)) { ok = false; break; }
      tc_fence_after();
      float s[128];
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) {
        uint32_t rr[32];
        tmem_ld32(tmem + (j & 1) * 128 + lane_off + qq * 32, rr);
        tmem_ld_wait(rr);
#pragma unroll
        for (int e = 0; e < 32; ++e) s[qq * 32 + e] = I8 ? (float)(int)rr[e] : __uint_as_float(rr[e]);
      }
      if (j == L - 1) {
        // diagonal chunk: key t of the chunk is visible iff t <= row
#pragma unroll
        for (int t = 0; t < 128; ++t) s[t] = (t <= row) ? s[t] : -INFINITY;
      }
      float mx = s[0];
#pragma unroll
      for (int t = 1; t < 128; ++t) mx = fmaxf(mx, s[t]);
      const float rmax2 = mx * scale2;
      const bool raise = rmax2 > m_ref + 8.f;
      const float m_new = raise ? rmax2 : m_ref;
      const float alpha = raise ? ex2(m_ref - m_new) : 1.f;
      // P in bf16 (the P.V operand); the row sum adds the same rounded values
      // so numerator and denominator use identical weights.
      uint32_t pk[64];
      float rs = 0.f;
#pragma unroll
      for (int t = 0; t < 128; t += 2) {
        pk[t >> 1] = pack_bf16x2(ex2(fmaf(s[t], scale2, -m_new)), ex2(fmaf(s[t + 1], scale2, -m_new)));
        rs += __uint_as_float(pk[t >> 1] << 16) + __uint_as_float(pk[t >> 1] & 0xFFFF0000u);
      }
      l = l * alpha + rs;
      m_ref = m_new;
      if (j > 0) {
        // PV(j-1) complete: O is stable and the P buffer is free
        if (!mbar_wait(smem_u32(&bar_odone), (j - 1) & 1, abort_flag, P.err)) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, raise)) {
#pragma unroll 1
          for (int qq = 0; qq < 4; ++qq) {
            uint32_t o[32];
            tmem_ld32(tmem + 256 + lane_off + qq * 32, o);
            tmem_ld_wait(o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(tmem + 256 + lane_off + qq * 32, o);
          }
          tmem_st_wait();
        }
      }
      // P row -> shared memory, K-major 128-byte swizzle: key t of row `row`
      // lives in 64-key half t/64, 16-byte chunk ((t%64)/8) ^ (row%8).
#pragma unroll
      for (int c8 = 0; c8 < 16; ++c8) {
        const uint4 v = make_uint4(pk[c8 * 4 + 0], pk[c8 * 4 + 1], pk[c8 * 4 + 2], pk[c8 * 4 + 3]);
        const int half = c8 >> 3, chunk = (c8 & 7) ^ (row & 7);
        *reinterpret_cast<uint4 *>(p_gen + half * 16384 + row * 128 + chunk * 16) = v;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar_pfull));
    }
    if (ok && L > 0 && mbar_wait(smem_u32(&bar_odone), (L - 1) & 1, abort_flag, P.err)) {
      tc_fence_after();
      const float inv = 1.f / l;
      __nv_bfloat16 *orow = P.out + ((size_t)h * P.S + (size_t)qc * 128 + row) * 128;
#pragma unroll 1
      for (int qq = 0; qq < 4; ++qq) {
        uint32_t o[32];
        tmem_ld32(tmem + 256 + lane_off + qq * 32, o);
        tmem_ld_wait(o);
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(o[c8 * 8 + 0]) * inv, __uint_as_float(o[c8 * 8 + 1]) * inv);
          v.y = pack_bf16x2(__uint_as_float(o[c8 * 8 + 2]) * inv, __uint_as_float(o[c8 * 8 + 3]) * inv);
          v.z = pack_bf16x2(__uint_as_float(o[c8 * 8 + 4]) * inv, __uint_as_float(o[c8 * 8 + 5]) * inv);
          v.w = pack_bf16x2(__uint_as_float(o[c8 * 8 + 6]) * inv, __uint_as_float(o[c8 * 8 + 7]) * inv);
          *reinterpret_cast<uint4 *>(orow + qq * 32 + c8 * 8) = v;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// Test kernel: one exact int8 score tile through the same kind::i8 MMA and
// descriptors as the attention kernel; out[i][t] (int32, row-major 128x128).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128, 1)
    k_qk_tile_i8(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 int qrow, int krow, int32_t *out, int *err) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_ld, bar_mma;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  if (threadIdx.x == 0) {
    abort_sh = 0;
    mbar_init(smem_u32(&bar_ld), 1);
    mbar_init(smem_u32(&bar_mma), 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_base_sh), 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  volatile int *abort_flag = &abort_sh;
  if (threadIdx.x == 0) {
    mbar_expect_tx(smem_u32(&bar_ld), 32768);
    tma_load_2d(base, &tm_q, 0, qrow, smem_u32(&bar_ld));
    tma_load_2d(base + 16384, &tm_k, 0, krow, smem_u32(&bar_ld));
    if (mbar_wait(smem_u32(&bar_ld), 0, abort_flag, err)) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_i8_ss(tmem, umma_desc_sw128(base + kk * 32, 16, 1024),
                  umma_desc_sw128(base + 16384 + kk * 32, 16, 1024), idesc_i8(128, 128), kk > 0);
      tc_commit(smem_u32(&bar_mma));
    }
  }
  __syncwarp();
  if (mbar_wait(smem_u32(&bar_mma), 0, abort_flag, err)) {
    tc_fence_after();
    const int row = warp * 32 + lane;
    for (int qq = 0; qq < 4; ++qq) {
      uint32_t r[32];
      tmem_ld32(tmem + (((uint32_t)(warp * 32)) << 16) + qq * 32, r);
      tmem_ld_wait(r);
      for (int e = 0; e < 32; ++e) out[row * 128 + qq * 32 + e] = (int32_t)r[e];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// Test kernel: waits on a barrier that nothing completes, bounded by limit_ns.
__global__ void k_wait_timeout(unsigned long long limit_ns, int *err) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_sh;
  if (threadIdx.x == 0) {
    abort_sh = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, &abort_sh, err, limit_ns);
  __syncthreads();
}

}  // namespace fpk

// attn2_kernel.cuh -- block-sparse GQA causal attention with CTA-pair MMAs
// (tcgen05 cta_group::2, M = 256) for block size b = 256.
//
// Same operation as k_sparse_attn (FAST-Prefill article, figure 3 and
// section 1.1): out_p = sum over listed keys j <= p of softmax_j(q_p . k_j /
// sqrt(d)) v_j, fp32 online softmax, bf16 P.V.  With b = 256 the two 128-row
// halves of a query block share one block list, so they form one M = 256
// "pair tile": the top half in CTA rank 0 of a two-CTA cluster, the bottom
// half in rank 1.  Each Q.K^T and P.V is one pair MMA issued by rank 0: each
// CTA holds its own 128 rows of Q, S, P and O (same shared-memory offsets and
// TMEM columns), and only half of every K and V chunk (64 keys of K, 64
// columns of V); the tensor cores exchange the halves, so each SM reads and
// TMA-loads half the K/V bytes per tile of the one-CTA kernel.
// A cluster serves two pair tiles that read the same KV head (two heads of a
// GQA group, or two blocks of one head when g = 1; section 2.2, KV reuse
// across the group's heads) and walks the union of their chunk lists, a
// chunk one pair does not list being computed for the other pair only.
// Every chunk of a listed block up to the block's last row is computed for
// both halves; each half's softmax masks by absolute position (the top half
// sees none of the block's second chunk).
//
// Warp roles per CTA (608 threads), as in k_sparse_attn:
//   0-7 / 8-15 softmax, rescale and epilogue of pair tile 0 / 1 (this CTA's rows)
//   16         TMA producer: this CTA's Q tiles, then its K halves (ring)
//   17         TMEM owner (pair allocation in both CTAs); MMA issuer in rank 0
//   18         TMA producer of this CTA's V halves (ring)
// Barriers: K/V/Q "full" barriers live in rank 0 and count both CTAs' bytes
// (each CTA's TMA signals rank 0's barrier); S-full, O-done and the ring
// "empty" barriers exist in both CTAs and are signalled by one multicast
// commit; P-full lives in rank 0 and counts both CTAs' softmax warps.
#pragma once

#include "attn_kernel.cuh"

namespace fpk {

template <bool I8>
struct Attn2Cfg {
  static constexpr int kQTile = I8 ? 16384 : 32768;  // this CTA's 128 query rows
  static constexpr int kKHalf = I8 ? 8192 : 16384;   // 64 keys x 128 d of a chunk
  static constexpr int kVHalf = 16384;               // 128 keys x 64 d of a chunk (bf16)
  static constexpr int kKStages = 4, kVStages = 4;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + 2 * kQTile;
  static constexpr int kVOff = kKOff + kKStages * kKHalf;
  static constexpr int kSmem = kVOff + kVStages * kVHalf + 1024;
  static constexpr int kThreads = 608;
};

// Number of clusters for b = 256.
__host__ __device__ inline int attn2_units(int Hq, int Hkv, int S) {
  const int n = (S + 255) / 256, g = Hq / Hkv;
  if (g >= 2) return Hkv * ((g + 1) / 2) * n;
  return Hq * ((n + 1) / 2);
}

// Pair tiles of cluster `unit`: KV-head-major, heavy (late) blocks first.
// qc is set to the pair's last 128-row tile (2r + 1) so that the chunk maps
// hold every chunk of the listed blocks up to the block's end.
__device__ inline void attn2_unit_tiles(const AttnParams &P, int unit, AttnTile (&t)[2]) {
  const int n = P.n, g = P.g;
  int h0, h1, r0, r1, v1;
  if (g >= 2) {
    const int hp = (g + 1) / 2, per_kv = hp * n, kvh = unit / per_kv, rem = unit % per_kv;
    const int r = n - 1 - rem / hp, k = rem % hp;
    h0 = kvh * g + 2 * k;
    h1 = h0 + 1;
    v1 = (2 * k + 1) < g;
    r0 = r1 = r;
  } else {
    const int per = (n + 1) / 2, h = unit / per, m = per - 1 - unit % per;
    h0 = h1 = h;
    r0 = 2 * m;
    r1 = 2 * m + 1;
    v1 = r1 < n;
  }
  const int hs[2] = {h0, h1}, rs[2] = {r0, r1}, vs[2] = {1, v1};
  const size_t tri = (size_t)n * (n + 1) / 2;
  const int nq = (P.S + 127) / 128;
  for (int i = 0; i < 2; ++i) {
    t[i].valid = vs[i];
    t[i].h = hs[i];
    t[i].r = rs[i];
    t[i].qc = min(2 * rs[i] + 1, nq - 1);
    t[i].cnt = t[i].cnt1 = 0;
    t[i].list = t[i].list1 = nullptr;
    if (vs[i]) {
      t[i].cnt = P.counts[(size_t)hs[i] * n + rs[i]];
      t[i].list = P.cols + (size_t)hs[i] * tri + (size_t)rs[i] * (rs[i] + 1) / 2;
    }
  }
}

template <bool I8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(608, 1)
    k_sparse_attn2(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kh,
                   const __grid_constant__ CUtensorMap tm_v, AttnParams P) {
  using C = Attn2Cfg<I8>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_q, bar_kfull[C::kKStages], bar_kempty[C::kKStages], bar_vfull[C::kVStages],
      bar_vempty[C::kVStages], bar_sfull[2], bar_pfull[2], bar_odone[2], bar_xchg[2][4], bar_final;
  __shared__ float xmax[2][2][2][128];  // [chunk parity][tile][column half][row]
  __shared__ float xl[2][2][128];       // [tile][column half][row]
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  __shared__ uint32_t chunk_bm[2][kMaxChunkWords];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  AttnTile tl[2];
  attn2_unit_tiles(P, blockIdx.x >> 1, tl);
  const int kvh = tl[0].h / P.g;
  const int words = (max(tl[0].qc, tl[1].valid ? tl[1].qc : 0) >> 5) + 1;
  const int own_qc[2] = {2 * tl[0].r + (int)rank, 2 * tl[1].r + (int)rank};

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sq = base + C::kQOff, sk = base + C::kKOff, sv = base + C::kVOff;

  if (threadIdx.x == 0) {
    abort_sh = 0;
    mbar_init(smem_u32(&bar_q), 1);
    for (int s = 0; s < C::kKStages; ++s) {
      mbar_init(smem_u32(&bar_kfull[s]), 1);
      mbar_init(smem_u32(&bar_kempty[s]), 1);
    }
    for (int s = 0; s < C::kVStages; ++s) {
      mbar_init(smem_u32(&bar_vfull[s]), 1);
      mbar_init(smem_u32(&bar_vempty[s]), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(smem_u32(&bar_sfull[t]), 1);
      mbar_init(smem_u32(&bar_pfull[t]), 16);  // 8 softmax warps in each CTA of the pair
      mbar_init(smem_u32(&bar_odone[t]), 1);
      for (int q = 0; q < 4; ++q) mbar_init(smem_u32(&bar_xchg[t][q]), 2);
    }
    mbar_init(smem_u32(&bar_final), 1);
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < 2 * kMaxChunkWords; i += blockDim.x) (&chunk_bm[0][0])[i] = 0u;
  if (warp == 17) {
    tmem_alloc_pair(smem_u32(&tmem_base_sh), 512);
    tmem_relinquish_pair();
  }
  __syncthreads();
  if (warp == 16 || warp == 17) {
    const int lane64 = threadIdx.x - 512;
    build_chunk_bitmap(tl[0], 256, chunk_bm[0], nullptr, nullptr, lane64);
    build_chunk_bitmap(tl[1], 256, chunk_bm[1], nullptr, nullptr, lane64);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers initialised before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  volatile int *abort_flag = &abort_sh;
  const uint16_t kBoth = 3;

  if (warp == 16) {
    // ---------------------------------------------------------------- Q and K producer
    if (lane == 0) {
      tma_prefetch_map(&tm_q);
      tma_prefetch_map(&tm_kh);
      const int nt = tl[1].valid ? 2 : 1;
      const uint32_t qbar = mapa_shared(smem_u32(&bar_q), 0);
      if (leader) mbar_expect_tx(smem_u32(&bar_q), 2 * nt * C::kQTile);
      for (int t = 0; t < nt; ++t) {
        const int qrow = tl[t].h * P.ld + own_qc[t] * 128;
        const uint32_t dst = sq + t * C::kQTile;
        tma_load_2d_pair(dst, &tm_q, 0, qrow, qbar);
        if (!I8) tma_load_2d_pair(dst + 16384, &tm_q, 64, qrow, qbar);
      }
      UnionWalk wk;
      wk.init(chunk_bm[0], chunk_bm[1], words);
      int kc, mask;
      for (int u = 0; wk.next(kc, mask); ++u) {
        const int st = u % C::kKStages;
        const int krow = kvh * P.ld + kc * 128 + (int)rank * 64;  // this CTA's 64 keys of the chunk
        if (u >= C::kKStages &&
            !mbar_wait(smem_u32(&bar_kempty[st]), ((u / C::kKStages) - 1) & 1, abort_flag, P.err))
          break;
        const uint32_t fb = mapa_shared(smem_u32(&bar_kfull[st]), 0);
        if (leader) mbar_expect_tx(smem_u32(&bar_kfull[st]), 2 * C::kKHalf);
        tma_load_2d_pair(sk + st * C::kKHalf, &tm_kh, 0, krow, fb);
        if (!I8) tma_load_2d_pair(sk + st * C::kKHalf + 8192, &tm_kh, 64, krow, fb);
      }
    }
  } else if (warp == 18) {
    // ---------------------------------------------------------------- V producer
    if (lane == 0) {
      tma_prefetch_map(&tm_v);
      UnionWalk wv;
      wv.init(chunk_bm[0], chunk_bm[1], words);
      int kc, mask;
      for (int u = 0; wv.next(kc, mask); ++u) {
        const int st = u % C::kVStages, vrow = kvh * P.ld + kc * 128;
        if (u >= C::kVStages &&
            !mbar_wait(smem_u32(&bar_vempty[st]), ((u / C::kVStages) - 1) & 1, abort_flag, P.err))
          break;
        const uint32_t fb = mapa_shared(smem_u32(&bar_vfull[st]), 0);
        if (leader) mbar_expect_tx(smem_u32(&bar_vfull[st]), 2 * C::kVHalf);
        tma_load_2d_pair(sv + st * C::kVHalf, &tm_v, (int)rank * 64, vrow, fb);  // this CTA's 64 columns of V
      }
    }
  } else if (warp == 17) {
    // ---------------------------------------------------------------- MMA issuer (rank 0)
    if (lane == 0 && leader) {
      const uint32_t id_qk = I8 ? idesc_i8(256, 128) : idesc_bf16(256, 128, 0);
      const uint32_t id_pv = idesc_bf16(256, 128, 1);
      const uint64_t dq0 = umma_desc_sw128(sq, 16, 1024), dq1 = umma_desc_sw128(sq + C::kQTile, 16, 1024);
      UnionWalk uw;
      uw.init(chunk_bm[0], chunk_bm[1], words);
      int npv[2] = {0, 0};
      int prev = 0;
      bool ok = mbar_wait(smem_u32(&bar_q), 0, abort_flag, P.err);
      int u = 0;
      auto issue_pv = [&](int t, int vst) -> bool {
        if (!mbar_wait(smem_u32(&bar_pfull[t]), npv[t] & 1, abort_flag, P.err)) return false;
        tc_fence_after();
        const uint64_t dv = umma_desc_sw128(sv + vst * C::kVHalf, 16384, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts_pair(tmem + 256 + t * 128, tmem + t * 128 + kk * 8, dv + (uint64_t)((kk * 2048) >> 4), id_pv,
                           (npv[t] > 0 || kk > 0));
        tc_commit_pair(smem_u32(&bar_odone[t]), kBoth);
        ++npv[t];
        return true;
      };
      int kc, mask;
      while (ok) {
        const bool more = uw.next(kc, mask);
        if (prev) {
          const int pst = (u - 1) % C::kVStages;
          if (!mbar_wait(smem_u32(&bar_vfull[pst]), ((u - 1) / C::kVStages) & 1, abort_flag, P.err)) break;
        }
        bool kwaited = false;
        const int st = u % C::kKStages;
        for (int t = 0; t < 2 && ok; ++t) {
          if ((prev >> t) & 1) ok = issue_pv(t, (u - 1) % C::kVStages);
          if (ok && more && ((mask >> t) & 1)) {
            if (!kwaited) {
              if (!mbar_wait(smem_u32(&bar_kfull[st]), (u / C::kKStages) & 1, abort_flag, P.err)) {
                ok = false;
                break;
              }
              tc_fence_after();
              kwaited = true;
            }
            const uint64_t dq = t ? dq1 : dq0;
            const uint64_t dk = umma_desc_sw128(sk + st * C::kKHalf, 16, 1024);
            const uint32_t d_tmem = tmem + t * 128;
            if (I8) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_i8_ss_pair(d_tmem, dq + (uint64_t)((kk * 32) >> 4), dk + (uint64_t)((kk * 32) >> 4), id_qk, kk > 0);
            } else {
#pragma unroll
              for (int kk = 0; kk < 8; ++kk) {
                const uint64_t offq = (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
                const uint64_t offk = (uint64_t)(((kk >> 2) * 8192 + (kk & 3) * 32) >> 4);
                mma_bf16_ss_pair(d_tmem, dq + offq, dk + offk, id_qk, kk > 0);
              }
            }
            tc_commit_pair(smem_u32(&bar_sfull[t]), kBoth);
          }
        }
        if (!ok) break;
        if (prev) tc_commit_pair(smem_u32(&bar_vempty[(u - 1) % C::kVStages]), kBoth);
        if (!more) break;
        tc_commit_pair(smem_u32(&bar_kempty[st]), kBoth);
        prev = mask;
        ++u;
      }
      // every pair MMA issued has completed before the teardown frees TMEM
      tc_commit_pair(smem_u32(&bar_final), 1);
      mbar_wait(smem_u32(&bar_final), 0, abort_flag, P.err);
    }
  } else {
    // ---------------------------------------------------------------- softmax (this CTA's rows)
    const int t = warp >> 3, ch = (warp >> 2) & 1, lq = warp & 3;
    const AttnTile &me = tl[t];
    const int qc = own_qc[t];
    const int row = lq * 32 + lane;
    const uint32_t lane_off = ((uint32_t)(lq * 32)) << 16;
    const uint32_t s_tm = tmem + t * 128 + ch * 64 + lane_off;
    const uint32_t p_tm = tmem + t * 128 + ch * 32 + lane_off;
    const uint32_t o_tm = tmem + 256 + t * 128 + ch * 64 + lane_off;
    const uint32_t xbar = smem_u32(&bar_xchg[t][lq]);
    const uint32_t pbar = mapa_shared(smem_u32(&bar_pfull[t]), 0);
    float scale2 = P.scale2;
    if (I8 && me.valid) scale2 *= P.q_scale[me.h] * P.k_scale[kvh];
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    int L = 0;
    if (me.valid)
      for (int w = 0; w < words; ++w) L += __popc(chunk_bm[t][w]);
    int wi = 0;
    uint32_t cur = me.valid ? chunk_bm[t][0] : 0u;
    for (int j = 0; j < L; ++j) {
      while (cur == 0u) cur = chunk_bm[t][++wi];
      const int kc = wi * 32 + (__ffs(cur) - 1);
      cur &= cur - 1u;
      if (!mbar_wait(smem_u32(&bar_sfull[t]), j & 1, abort_flag, P.err)) { ok = false; break; }
      tc_fence_after();
      uint32_t rr[64];
      tmem_ld64(s_tm, rr);
      tmem_ld_wait64(rr);
      if constexpr (I8) {
        if (P.cap != nullptr && me.h == P.cap_h && qc == P.cap_qc && kc == P.cap_kc) {
          int4 *dst = reinterpret_cast<int4 *>(P.cap + (size_t)row * 128 + ch * 64);
#pragma unroll
          for (int e = 0; e < 16; ++e)
            dst[e] = make_int4((int)rr[4 * e], (int)rr[4 * e + 1], (int)rr[4 * e + 2], (int)rr[4 * e + 3]);
        }
      }
      float s[64];
#pragma unroll
      for (int e = 0; e < 64; ++e) s[e] = I8 ? i32_to_f32_small(rr[e]) : __uint_as_float(rr[e]);
      if (kc >= qc) {
        // the tile's own chunk: key 64ch+e visible iff it is <= row; a later chunk: none
        const int lim = kc == qc ? row - ch * 64 : -1;
#pragma unroll
        for (int e = 0; e < 64; ++e) s[e] = (e <= lim) ? s[e] : -INFINITY;
      }
      float m8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) m8[e] = s[e];
#pragma unroll
      for (int c = 8; c < 64; c += 16)
#pragma unroll
        for (int e = 0; e < 8; ++e) m8[e] = fmax3(m8[e], s[c + e], s[c + 8 + e]);
      const float pmx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
      xmax[j & 1][t][ch][row] = pmx;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(xbar);
      if (!mbar_wait(xbar, j & 1, abort_flag, P.err)) { ok = false; break; }
      tc_fence_after();
      const float mx = fmaxf(pmx, xmax[j & 1][t][ch ^ 1][row]);
      const float rmax2 = mx * scale2;
      const bool raise = rmax2 > m_ref + 8.f;
      const float m_new = raise ? rmax2 : m_ref;
      const float alpha = raise ? ex2(m_ref - m_new) : 1.f;
      const float m_sub = (m_new == -INFINITY) ? 0.f : m_new;
      uint32_t pk[32];
      float r8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) r8[e] = 0.f;
      const uint64_t sc2 = f2_pack(scale2, scale2), nm2 = f2_pack(-m_sub, -m_sub);
#pragma unroll
      for (int e = 0; e < 64; e += 2) {
        float x0, x1;
        f2_unpack(f2_fma(f2_pack(s[e], s[e + 1]), sc2, nm2), x0, x1);
        pk[e >> 1] = pack_bf16x2(ex2(x0), ex2(x1));
      }
      uint64_t a2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int e = 0; e < 32; ++e)
        a2[e & 3] = f2_add(a2[e & 3], f2_pack(__uint_as_float(pk[e] << 16), __uint_as_float(pk[e] & 0xFFFF0000u)));
#pragma unroll
      for (int e = 0; e < 4; ++e) f2_unpack(a2[e], r8[2 * e], r8[2 * e + 1]);
      const float rs = ((r8[0] + r8[1]) + (r8[2] + r8[3])) + ((r8[4] + r8[5]) + (r8[6] + r8[7]));
      l = l * alpha + rs;
      m_ref = m_new;
      if (j > 0 && __any_sync(0xffffffffu, raise)) {
#pragma unroll 1
        for (int qq = 0; qq < 2; ++qq) {
          uint32_t o[32];
          tmem_ld32(o_tm + qq * 32, o);
          tmem_ld_wait(o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(o_tm + qq * 32, o);
        }
      }
      tmem_st32(p_tm, pk);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(pbar);
    }
    if (ok && L > 0 && mbar_wait(smem_u32(&bar_odone[t]), (L - 1) & 1, abort_flag, P.err)) {
      tc_fence_after();
      xl[t][ch][row] = l;
      __syncwarp();
      if (lane == 0) mbar_arrive(xbar);
      if (mbar_wait(xbar, L & 1, abort_flag, P.err)) {
        const float inv = 1.f / (l + xl[t][ch ^ 1][row]);
        const bool store = qc * 128 + row < P.S;
        __nv_bfloat16 *orow = P.out + ((size_t)me.h * P.ld + (size_t)qc * 128 + row) * 128 + ch * 64;
#pragma unroll 1
        for (int qq = 0; qq < 2; ++qq) {
          uint32_t o[32];
          tmem_ld32(o_tm + qq * 32, o);
          tmem_ld_wait(o);
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(o[c8 * 8 + 0]) * inv, __uint_as_float(o[c8 * 8 + 1]) * inv);
            v.y = pack_bf16x2(__uint_as_float(o[c8 * 8 + 2]) * inv, __uint_as_float(o[c8 * 8 + 3]) * inv);
            v.z = pack_bf16x2(__uint_as_float(o[c8 * 8 + 4]) * inv, __uint_as_float(o[c8 * 8 + 5]) * inv);
            v.w = pack_bf16x2(__uint_as_float(o[c8 * 8 + 6]) * inv, __uint_as_float(o[c8 * 8 + 7]) * inv);
            if (store) *reinterpret_cast<uint4 *>(orow + qq * 32 + c8 * 8) = v;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // neither CTA frees the pair's TMEM while the other may still use it
  if (warp == 17) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace fpk

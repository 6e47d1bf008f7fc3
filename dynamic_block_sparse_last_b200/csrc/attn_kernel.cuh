// attn_kernel.cuh -- block-sparse GQA causal flash attention on sm_100a.
//
// Each query block attends only to the key blocks its index lists (FAST-Prefill
// article, figure 3 and section 1.1): out_p = sum over listed keys j <= p of
// softmax_j(q_p . k_j / sqrt(d)) v_j.  Online softmax in fp32, bf16 P.V.
//
// CTA = two 128-row query tiles that read the same KV head, so every K/V
// chunk the CTA loads serves both (KV reuse across the heads of a GQA group,
// FAST-Prefill article section 2.2):
//   b = 256:            the two 128-row halves of one 256-row query block
//   b <= 128, g >= 2:   the same query tile of two heads of one GQA group
//   b <= 128, g == 1:   two neighbouring query tiles of one head
// With b = 64 a tile holds two query blocks and a chunk two key blocks: the
// tile attends to a chunk if either of its blocks lists either key block, and
// each softmax warp, which owns one 32-row by 64-key quadrant and so exactly
// one (query block, key block) pair, masks the quadrant when that pair is not
// listed.
// The CTA walks the union of the two tiles' chunk lists (ascending 128-key
// chunks); a chunk only one tile needs is computed for that tile only.
// When 128 does not divide S the last query tile and the last key chunk run
// past S: the tensor maps read whatever follows (the next head's or the next
// packed sequence's rows, or zeros past the end of the tensor), the causal
// mask keeps those keys away from every real row, and rows at or past S are
// not stored.
// CTAs are numbered KV-head-major (all CTAs of one KV head together, so its
// K and V stay in L2 while they run; the GPU analogue of the article's
// KV-block-major schedule, section 3.2) and heavy first (descending query
// position) within a KV head.
//
// Warp roles (608 threads):
//   warps 0-7 / 8-15 softmax, correction and epilogue of tile 0 / tile 1:
//                    two warps per 32-row TMEM lane group, each taking half
//                    of the 128 keys of a chunk and half of the O columns
//   warp 16          TMA producer: Q tiles once, then K chunks (2-stage ring)
//   warp 17          TMEM owner and MMA issuer (one thread)
//   warp 18          TMA producer of V chunks (2-stage ring)
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512).
// Each softmax warp writes the P of its 64 keys (bf16, two per column) over
// the first 32 of its own 64 S columns, so P occupies columns 0-31 and 64-95
// of the S tile and no warp writes where another still reads. The P.V
// product reads P from TMEM (tcgen05.mma A operand in tensor memory), so P
// never touches shared memory.
//
// MMA issue order per union entry u: for each tile t, PV_t(u-1) then
// QK_t(u).  While softmax t works on S_t(u), the tensor pipe runs the other
// tile's PV and QK.  The exponentials of a chunk are taken against the
// row's current reference max at once; the reference moves (to the row max
// plus a headroom) only when the chunk's row sum exceeds kRefSum or the row
// has none yet, and
// the chunk is then recomputed, so no row max is formed in the common case.
// The correction O *= 2^(m_old - m_new) runs in TMEM after PV_t(u-1) has
// completed.
#pragma once

#include "ptx.cuh"

namespace fpk {

struct AttnParams {
  int S, Hq, Hkv, b, n, g;
  int ld;             // rows from one head to the next (S, or more for packed sequences)
  const int *counts;  // [Hq][n]
  const int *cols;    // padded lists, row (h, r) at h*n(n+1)/2 + r(r+1)/2
  const float *q_scale, *k_scale;  // int8 only
  float scale2;                    // log2(e)/sqrt(d)
  __nv_bfloat16 *out;              // [Hq][S][128]
  int *err;
  // int8 test capture (null in normal use): the raw int32 score tile of
  // query head cap_h, query tile cap_qc and key chunk cap_kc, copied from
  // tensor memory before masking, row-major [128][128]
  int32_t *cap;
  int cap_h, cap_qc, cap_kc;
};

template <bool I8>
struct AttnCfg {
  static constexpr int kQKTile = I8 ? 16384 : 32768;   // 128 rows x 128 elements
  static constexpr int kVTile = 32768;
  static constexpr int kKStages = 2, kVStages = 2;
  static constexpr int kQOff = 0;                                 // two Q tiles
  static constexpr int kKOff = kQOff + 2 * kQKTile;               // K ring
  static constexpr int kVOff = kKOff + kKStages * kQKTile;        // V ring
  static constexpr int kSmem = kVOff + kVStages * kVTile + 1024;
  static constexpr int kThreads = 608;
  // Every kExpFmaEvery-th exponential of an off-diagonal chunk runs on the
  // FMA pipe (ex2_fma) instead of MUFU; 0 keeps all on MUFU.  A share of 1/4
  // measured no faster on the 128K layer (power-capped clocks), so it is off.
  static constexpr int kExpFmaEvery = 0;
  // The reference max of a row moves when a chunk's row sum of P exceeds
  // this bound, so no P exceeds it (bf16 keeps its relative precision at any
  // magnitude; the sums and O accumulate in fp32).
  static constexpr float kRefSum = 256.f;
  // A moved reference is set this far (log2 units) above the row max, so the
  // next move needs the scores to rise about log2(kRefSum) + kRefHeadroom
  // above it.  Scores near the diagonal often exceed those of the first
  // chunks by tens of log2 units; with this headroom such rows rarely move
  // again.  P then starts near 2^-kRefHeadroom: bf16 keeps its relative
  // precision there, and only keys more than 126 - kRefHeadroom below the
  // row max flush to zero, whose weight relative to it is below 2^-62.
  static constexpr float kRefHeadroom = 64.f;
};

// Number of CTAs (tile pairs) for a layer shape.
__host__ __device__ inline int attn_pairs(int Hq, int Hkv, int S, int b) {
  const int nq = (S + 127) / 128, g = Hq / Hkv;
  if (b == 256) return Hq * ((S + b - 1) / b);
  if (g >= 2) return Hkv * ((g + 1) / 2) * nq;
  return Hq * ((nq + 1) / 2);
}

struct AttnTile {
  int valid, h, qc, r, cnt;
  const int *list;
  int cnt1;            // b = 64: the tile's second query block r + 1 (0 when past the last block)
  const int *list1;
};

// The two query tiles of CTA `pair`: KV-head-major, heavy pairs first within a head.
__device__ inline void attn_pair_tiles(const AttnParams &P, int pair, AttnTile (&t)[2]) {
  const int nq = (P.S + 127) / 128, g = P.g;
  int h0, h1, q0, q1, v1;
  // KV-head-major: all CTAs of one KV head (its K/V fit in L2), heavy first within it
  if (P.b == 256) {
    const int per_kv = g * P.n, kvh = pair / per_kv, rem = pair % per_kv;
    const int rr = P.n - 1 - rem / g;
    h0 = h1 = kvh * g + rem % g;
    q0 = 2 * rr;
    q1 = 2 * rr + 1;
    v1 = q1 < nq;  // a partial last block may have a single tile
  } else if (g >= 2) {
    const int hp = (g + 1) / 2, per_kv = hp * nq, kvh = pair / per_kv, rem = pair % per_kv;
    const int qc = nq - 1 - rem / hp, k = rem % hp;
    h0 = kvh * g + 2 * k;
    h1 = h0 + 1;
    v1 = (2 * k + 1) < g;
    q0 = q1 = qc;
  } else {
    const int per_kv = (nq + 1) / 2, h = pair / per_kv;
    const int m = per_kv - 1 - pair % per_kv;
    h0 = h1 = h;
    q0 = 2 * m;
    q1 = 2 * m + 1;
    v1 = q1 < nq;
  }
  const int hs[2] = {h0, h1}, qs[2] = {q0, q1}, vs[2] = {1, v1};
  const size_t tri = (size_t)P.n * (P.n + 1) / 2;
  for (int i = 0; i < 2; ++i) {
    t[i].valid = vs[i];
    t[i].h = hs[i];
    t[i].qc = qs[i];
    t[i].r = (qs[i] * 128) / P.b;
    t[i].cnt = t[i].cnt1 = 0;
    t[i].list = t[i].list1 = nullptr;
    if (vs[i]) {
      const int r = t[i].r;
      t[i].cnt = P.counts[(size_t)hs[i] * P.n + r];
      t[i].list = P.cols + (size_t)hs[i] * tri + (size_t)r * (r + 1) / 2;
      if (P.b < 128 && r + 1 < P.n) {
        t[i].cnt1 = P.counts[(size_t)hs[i] * P.n + r + 1];
        t[i].list1 = P.cols + (size_t)hs[i] * tri + (size_t)(r + 1) * (r + 2) / 2;
      }
    }
  }
}

// Chunk bitmaps: bit kc of tile t's map is set when the tile attends to the
// 128-key chunk kc.  Built once per CTA in shared memory from the block lists
// (coalesced loads by 64 lanes), so the producer and the MMA issuer walk the
// union without global-memory round trips.
constexpr int kMaxChunkWords = 64;  // 2048 chunks: S/128 <= 2048 for S/b <= 1024, b <= 256
constexpr int kMaxBlockWords = 32;  // b = 64: 1024 key blocks, one bit each

// b >= 128: chunk kc is attended when its block kc*128/b is listed.  b = 64:
// chunk kc when block 2kc or 2kc+1 is listed for either query block, and
// blk0 / blk1 get the listed key blocks of the tile's two query blocks.
__device__ inline void build_chunk_bitmap(const AttnTile &t, int b, uint32_t *bm, uint32_t *blk0, uint32_t *blk1,
                                          int lane64) {
  if (!t.valid) return;
  if (b >= 128) {
    const int per = b / 128;
    for (int e = lane64; e < t.cnt; e += 64) {
      const int c = t.list[e];
      for (int k = 0; k < per; ++k) {
        const int kc = c * per + k;
        if (kc <= t.qc) atomicOr(&bm[kc >> 5], 1u << (kc & 31));
      }
    }
    return;
  }
  for (int rb = 0; rb < 2; ++rb) {
    const int *list = rb ? t.list1 : t.list;
    const int cnt = rb ? t.cnt1 : t.cnt;
    uint32_t *blk = rb ? blk1 : blk0;
    for (int e = lane64; e < cnt; e += 64) {
      const int c = list[e], kc = c >> 1;
      atomicOr(&blk[c >> 5], 1u << (c & 31));
      if (kc <= t.qc) atomicOr(&bm[kc >> 5], 1u << (kc & 31));
    }
  }
}

// Iterates the union of the two tiles' chunk sets in ascending order.
struct UnionWalk {
  const uint32_t *a, *b;
  int words, wi;
  uint32_t cur;
  __device__ void init(const uint32_t *a_, const uint32_t *b_, int words_) {
    a = a_;
    b = b_;
    words = words_;
    wi = 0;
    cur = words > 0 ? (a[0] | b[0]) : 0u;
  }
  __device__ bool next(int &kc, int &mask) {
    while (cur == 0u) {
      if (++wi >= words) return false;
      cur = a[wi] | b[wi];
    }
    const int bit = __ffs(cur) - 1;
    cur &= cur - 1u;
    kc = wi * 32 + bit;
    mask = (int)((a[wi] >> bit) & 1u) | (int)(((b[wi] >> bit) & 1u) << 1);
    return true;
  }
};

template <bool I8>
__global__ void __launch_bounds__(608, 1)
    k_sparse_attn(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, AttnParams P) {
  using C = AttnCfg<I8>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_q, bar_kfull[2], bar_kempty[2], bar_vfull[2], bar_vempty[2],
      bar_sfull[2], bar_pfull[2], bar_odone[2], bar_xchg[2][4];
  __shared__ float xmax[2][2][2][128];  // [chunk parity][tile][column half][row]
  __shared__ float xl[2][2][128];       // [tile][column half][row]
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  __shared__ uint32_t chunk_bm[2][kMaxChunkWords];
  __shared__ uint32_t block_bm[2][2][kMaxBlockWords];  // b = 64: [tile][query block][key-block bits]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  AttnTile tl[2];
  attn_pair_tiles(P, blockIdx.x, tl);
  const int kvh = tl[0].h / P.g;
  const int words = (max(tl[0].qc, tl[1].valid ? tl[1].qc : 0) >> 5) + 1;

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sq = base + C::kQOff, sk = base + C::kKOff, sv = base + C::kVOff;

  if (threadIdx.x == 0) {
    abort_sh = 0;
    mbar_init(smem_u32(&bar_q), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&bar_kfull[s]), 1);
      mbar_init(smem_u32(&bar_kempty[s]), 1);
    }
    for (int t = 0; t < 2; ++t)
      for (int q = 0; q < 4; ++q) mbar_init(smem_u32(&bar_xchg[t][q]), 2);
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&bar_vfull[s]), 1);
      mbar_init(smem_u32(&bar_vempty[s]), 1);
      mbar_init(smem_u32(&bar_sfull[s]), 1);
      mbar_init(smem_u32(&bar_pfull[s]), 8);
      mbar_init(smem_u32(&bar_odone[s]), 1);
    }
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < 2 * kMaxChunkWords; i += blockDim.x) (&chunk_bm[0][0])[i] = 0u;
  for (int i = threadIdx.x; i < 4 * kMaxBlockWords; i += blockDim.x) (&block_bm[0][0][0])[i] = 0u;
  if (warp == 17) {
    tmem_alloc(smem_u32(&tmem_base_sh), 512);
    tmem_relinquish();
  }
  __syncthreads();
  if (warp == 16 || warp == 17) {
    const int lane64 = threadIdx.x - 512;
    build_chunk_bitmap(tl[0], P.b, chunk_bm[0], block_bm[0][0], block_bm[0][1], lane64);
    build_chunk_bitmap(tl[1], P.b, chunk_bm[1], block_bm[1][0], block_bm[1][1], lane64);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  volatile int *abort_flag = &abort_sh;

  if (warp == 16) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_map(&tm_q);
      tma_prefetch_map(&tm_k);
      const int nt = tl[1].valid ? 2 : 1;
      mbar_expect_tx(smem_u32(&bar_q), nt * C::kQKTile);
      for (int t = 0; t < nt; ++t) {
        const int qrow = tl[t].h * P.ld + tl[t].qc * 128;
        const uint32_t dst = sq + t * C::kQKTile;
        tma_load_2d(dst, &tm_q, 0, qrow, smem_u32(&bar_q));
        if (!I8) tma_load_2d(dst + 16384, &tm_q, 64, qrow, smem_u32(&bar_q));
      }
      // K runs up to two chunks ahead of the MMA issuer; V (warp 18) has
      // its own ring and producer, so neither waits on the other's slots.
      UnionWalk wk;
      wk.init(chunk_bm[0], chunk_bm[1], words);
      int kc, mask;
      for (int u = 0; wk.next(kc, mask); ++u) {
        const int st = u % C::kKStages, krow = kvh * P.ld + kc * 128;
        if (u >= C::kKStages &&
            !mbar_wait(smem_u32(&bar_kempty[st]), ((u / C::kKStages) - 1) & 1, abort_flag, P.err))
          break;
        mbar_expect_tx(smem_u32(&bar_kfull[st]), C::kQKTile);
        tma_load_2d(sk + st * C::kQKTile, &tm_k, 0, krow, smem_u32(&bar_kfull[st]));
        if (!I8) tma_load_2d(sk + st * C::kQKTile + 16384, &tm_k, 64, krow, smem_u32(&bar_kfull[st]));
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
        mbar_expect_tx(smem_u32(&bar_vfull[st]), C::kVTile);
        tma_load_2d(sv + st * C::kVTile, &tm_v, 0, vrow, smem_u32(&bar_vfull[st]));
        tma_load_2d(sv + st * C::kVTile + 16384, &tm_v, 64, vrow, smem_u32(&bar_vfull[st]));
      }
    }
  } else if (warp == 17) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_qk = I8 ? idesc_i8(128, 128) : idesc_bf16(128, 128, 0);
      const uint32_t id_pv = idesc_bf16(128, 128, 1);
      // Shared-memory descriptors built once: a byte offset d inside an
      // operand is the descriptor plus d >> 4 (start address field, bits 0-13).
      const uint64_t dq0 = umma_desc_sw128(sq, 16, 1024), dq1 = umma_desc_sw128(sq + C::kQKTile, 16, 1024);
      const uint64_t dk0 = umma_desc_sw128(sk, 16, 1024), dk1 = umma_desc_sw128(sk + C::kQKTile, 16, 1024);
      const uint64_t dv0 = umma_desc_sw128(sv, 16384, 1024), dv1 = umma_desc_sw128(sv + C::kVTile, 16384, 1024);
      UnionWalk uw;
      uw.init(chunk_bm[0], chunk_bm[1], words);
      int npv[2] = {0, 0};
      int prev = 0;
      bool ok = mbar_wait(smem_u32(&bar_q), 0, abort_flag, P.err);
      int u = 0;
      // issue_pv: O_t += P_t(TMEM) . V(stage), for the entry before u
      auto issue_pv = [&](int t, int vst) -> bool {
        if (!mbar_wait(smem_u32(&bar_pfull[t]), npv[t] & 1, abort_flag, P.err)) return false;
        tc_fence_after();
        const uint64_t dv = vst ? dv1 : dv0;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(tmem + 256 + t * 128, tmem + t * 128 + (kk >> 2) * 64 + (kk & 3) * 8,
                      dv + (uint64_t)((kk * 2048) >> 4), id_pv,
                      (npv[t] > 0 || kk > 0));
        tc_commit(smem_u32(&bar_odone[t]));
        ++npv[t];
        return true;
      };
      int kc, mask;
      while (ok) {
        const bool more = uw.next(kc, mask);
        if (prev) {
          const int pst = (u - 1) & 1;
          if (!mbar_wait(smem_u32(&bar_vfull[pst]), ((u - 1) >> 1) & 1, abort_flag, P.err)) break;
        }
        bool kwaited = false;
        const int st = u % C::kKStages;
        for (int t = 0; t < 2 && ok; ++t) {
          if ((prev >> t) & 1) ok = issue_pv(t, (u - 1) & 1);
          if (ok && more && ((mask >> t) & 1)) {
            if (!kwaited) {
              if (!mbar_wait(smem_u32(&bar_kfull[st]), (u / C::kKStages) & 1, abort_flag, P.err)) { ok = false; break; }
              tc_fence_after();
              kwaited = true;
            }
            const uint64_t dq = t ? dq1 : dq0, dk = st ? dk1 : dk0;
            const uint32_t d_tmem = tmem + t * 128;
            if (I8) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_i8_ss(d_tmem, dq + (uint64_t)((kk * 32) >> 4), dk + (uint64_t)((kk * 32) >> 4), id_qk, kk > 0);
            } else {
#pragma unroll
              for (int kk = 0; kk < 8; ++kk) {
                const uint64_t off = (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
                mma_bf16_ss(d_tmem, dq + off, dk + off, id_qk, kk > 0);
              }
            }
            tc_commit(smem_u32(&bar_sfull[t]));
          }
        }
        if (!ok) break;
        if (prev) tc_commit(smem_u32(&bar_vempty[(u - 1) & 1]));
        if (!more) break;
        tc_commit(smem_u32(&bar_kempty[st]));
        prev = mask;
        ++u;
      }
    }
  } else {
    // ---------------------------------------------------------------- softmax
    // Two warps share each 32-row group of a tile: warp half ch owns keys
    // 64ch .. 64ch+63 of every S chunk and O columns 64ch .. 64ch+63.  They
    // exchange their partial row maxima once per chunk through shared memory
    // (an mbarrier of count 2, waited with the usual time limit) and keep
    // partial row sums against the same reference max, added at the end.
    const int t = warp >> 3, ch = (warp >> 2) & 1, lq = warp & 3;
    const AttnTile &me = tl[t];
    const int row = lq * 32 + lane;
    const uint32_t lane_off = ((uint32_t)(lq * 32)) << 16;
    const uint32_t s_tm = tmem + t * 128 + ch * 64 + lane_off;    // this warp's S columns
    const uint32_t p_tm = tmem + t * 128 + ch * 64 + lane_off;    // packed P of its 64 keys, over its own S
    const uint32_t o_tm = tmem + 256 + t * 128 + ch * 64 + lane_off;
    const uint32_t xbar = smem_u32(&bar_xchg[t][lq]);
    float scale2 = P.scale2;
    if (I8 && me.valid) scale2 *= P.q_scale[me.h] * P.k_scale[kvh];
    float m_ref = -INFINITY, l = 0.f;
    int nx = 0;  // exchanges with the partner half so far (phase and buffer parity)
    bool ok = true;
    // this tile's chunks, ascending: the entries its S tile receives
    int L = 0;
    if (me.valid)
      for (int w = 0; w < words; ++w) L += __popc(chunk_bm[t][w]);
    int wi = 0;
    uint32_t cur = me.valid ? chunk_bm[t][0] : 0u;
    const uint32_t *vis_bm = block_bm[t][lq >= 2 ? 1 : 0];  // b = 64: this warp's query block
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
        if (P.cap != nullptr && me.h == P.cap_h && me.qc == P.cap_qc && kc == P.cap_kc) {
          int4 *dst = reinterpret_cast<int4 *>(P.cap + (size_t)row * 128 + ch * 64);
#pragma unroll
          for (int e = 0; e < 16; ++e)
            dst[e] = make_int4((int)rr[4 * e], (int)rr[4 * e + 1], (int)rr[4 * e + 2], (int)rr[4 * e + 3]);
        }
      }
      // S (this warp's 64 keys) as fp32 with the masks applied; -inf where
      // a key is not visible.  Called again when the reference must move.
      float s[64];
      auto load_s = [&](bool reload) {
        if (reload) {
          tmem_ld64(s_tm, rr);
          tmem_ld_wait64(rr);
        }
#pragma unroll
        for (int e = 0; e < 64; ++e) s[e] = I8 ? (float)(int)rr[e] : __uint_as_float(rr[e]);
        if (P.b < 128) {
          // the warp's quadrant is one (query block, key block 2kc + ch) pair
          const int kb = 2 * kc + ch;
          if (!((vis_bm[kb >> 5] >> (kb & 31)) & 1u)) {
#pragma unroll
            for (int e = 0; e < 64; ++e) s[e] = -INFINITY;
          }
        }
        if (j == L - 1) {
          // diagonal chunk: key 64ch+e of the chunk is visible iff it is <= row
#pragma unroll
          for (int e = 0; e < 64; ++e) s[e] = (ch * 64 + e <= row) ? s[e] : -INFINITY;
        }
      };
      // P in bf16 (the P.V operand) against reference m (log2 units; 0
      // stands for "none yet"), and the row sum of the same rounded values:
      // each bf16 added to an fp32 chain as it is (mixed-precision add), eight chains
      uint32_t pk[32];
      auto make_p = [&](float m) -> float {
        float r8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) r8[e] = 0.f;
        if (C::kExpFmaEvery > 0 && j != L - 1) {
          // every kExpFmaEvery-th exponential on the FMA pipe (ex2_fma); the
          // diagonal chunk has masked (-inf) entries and uses MUFU only
#pragma unroll
          for (int e = 0; e < 64; e += 2) {
            const float x0 = fmaf(s[e], scale2, -m), x1 = fmaf(s[e + 1], scale2, -m);
            const bool f1 = ((e + 1) % (C::kExpFmaEvery > 0 ? C::kExpFmaEvery : 1)) == 0;
            pk[e >> 1] = pack_bf16x2(ex2(x0), f1 ? ex2_fma(x1) : ex2(x1));
          }
        } else {
          // exponent arguments two at a time (packed fp32 FMA), then MUFU ex2
          const uint64_t sc2 = f2_pack(scale2, scale2), nm2 = f2_pack(-m, -m);
#pragma unroll
          for (int e = 0; e < 64; e += 2) {
            float x0, x1;
            f2_unpack(f2_fma(f2_pack(s[e], s[e + 1]), sc2, nm2), x0, x1);
            pk[e >> 1] = pack_bf16x2(ex2(x0), ex2(x1));
          }
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) add_bf16x2_f32(pk[e], r8[(2 * e) & 7], r8[(2 * e + 1) & 7]);
        return ((r8[0] + r8[1]) + (r8[2] + r8[3])) + ((r8[4] + r8[5]) + (r8[6] + r8[7]));
      };
      // one exchange with the partner half through shared memory (each warp
      // writes P only over its own S columns, so no tensor-memory ordering
      // between the two is needed here)
      auto exchange = [&](float v, float &partner) -> bool {
        xmax[nx & 1][t][ch][row] = v;
        __syncwarp();
        if (lane == 0) mbar_arrive(xbar);
        if (!mbar_wait(xbar, nx & 1, abort_flag, P.err)) return false;
        partner = xmax[nx & 1][t][ch ^ 1][row];
        ++nx;
        return true;
      };
      load_s(false);
      // Exponentials first, against the current reference m_ref.  The
      // reference moves only when the row's chunk sum (both halves) exceeds
      // kRefSum, which bounds every P of the chunk by it, or when the row has no
      // reference yet; then the row max is taken, S is read again (P has
      // not been written over it yet) and P is recomputed.  In the common
      // case no row max is computed at all.
      float rs = make_p(m_ref == -INFINITY ? 0.f : m_ref);
      float rs_other;
      if (!exchange(rs, rs_other)) { ok = false; break; }
      const bool trig = !(rs + rs_other <= C::kRefSum) || m_ref == -INFINITY;
      float alpha = 1.f;
      bool moved = false;
      if (__any_sync(0xffffffffu, trig)) {
        load_s(true);
        float m8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) m8[e] = s[e];
#pragma unroll
        for (int c = 8; c < 64; c += 16)
#pragma unroll
          for (int e = 0; e < 8; ++e) m8[e] = fmax3(m8[e], s[c + e], s[c + 8 + e]);
        const float pmx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
        float pmx_other;
        if (!exchange(pmx, pmx_other)) { ok = false; break; }
        const float m_new = trig ? fmaxf(m_ref, fmaxf(pmx, pmx_other) * scale2 + C::kRefHeadroom) : m_ref;
        moved = m_new > m_ref;
        alpha = moved ? ex2(m_ref - m_new) : 1.f;  // 0 when there was no reference
        m_ref = m_new;
        rs = make_p(m_ref == -INFINITY ? 0.f : m_ref);
      }
      l = l * alpha + rs;
      // The commit that signalled S(j) also covers PV(j-1), issued before
      // QK(j): O is stable here and may be rescaled in place.
      if (j > 0 && __any_sync(0xffffffffu, moved)) {
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
      if (lane == 0) mbar_arrive(smem_u32(&bar_pfull[t]));
    }
    if (ok && L > 0 && mbar_wait(smem_u32(&bar_odone[t]), (L - 1) & 1, abort_flag, P.err)) {
      tc_fence_after();
      // total row sum: this half's plus the partner's (exchange phase L)
      xl[t][ch][row] = l;
      __syncwarp();
      if (lane == 0) mbar_arrive(xbar);
      if (mbar_wait(xbar, nx & 1, abort_flag, P.err)) {
        const float inv = 1.f / (l + xl[t][ch ^ 1][row]);
        const bool store = me.qc * 128 + row < P.S;  // rows past S belong to a neighbour
        __nv_bfloat16 *orow = P.out + ((size_t)me.h * P.ld + (size_t)me.qc * 128 + row) * 128 + ch * 64;
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
  if (warp == 17) {
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

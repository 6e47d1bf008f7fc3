// index_kernels.cuh -- sparse-index generation on sm_100a.
//
// Method (FAST-Prefill article, sections 1.2, 2.1 and 3.1; maplevalley
// article, section 1.1): score the last query block of every head against
// all keys, pool the softmax probabilities into vertical (per key block) and
// slash (per diagonal offset block) statistics, decide the head's pattern by
// the Jensen-Shannon divergence between the exact pooled distribution and
// the block-mean estimate, then keep for every query block the smallest set
// of key blocks (diagonal forced) whose normalised score reaches gamma.
//
// Kernels, in launch order:
//   k_score_last   tcgen05 Q_last.K^T per 128-key chunk, K streamed once per
//                  KV group through a TMA ring; per (row, chunk) reference and the
//                  two offset-half sums; per-chunk K column sums.  Nothing of
//                  size S x b reaches global memory.
//   k_head_stats   one cluster per head: row max / sum, row-normalised
//                  block masses, vhat, shat, block means of K, P_est, JSD,
//                  pattern.
//   k_qpool        block means of Q of the query-aware heads.
//   k_qa_logits    q-bar . k-bar logits of query-aware heads: tf32 hi/lo split
//                  on the tensor cores (k_split_tf32 prepares the operands), or
//                  tiled fp32 FMAs (k_qa_logits_fma) when n is small.
//   k_cut          per (head, query block): scores, gamma cut, sorted list.
#pragma once

#include <cooperative_groups.h>

#include "ptx.cuh"

namespace fpk {

constexpr float kLog2e = 1.4426950408889634f;
// headroom (log2 units) above the piece max when the statistics loop of
// k_score_last moves a row's reference
constexpr float kScoreHeadroom = 64.f;

// ---------------------------------------------------------------------------
// k_score_last
//
// CTA = (KV head, group of up to 4 row tiles of 128 query rows of the last
// block, range of 128-key chunks).  A "tile" is (query head of the group,
// 128-row slice of the last block; ceil(nlast/128) slices for its nlast =
// S - (n-1)b rows, which is fewer than b when b does not divide S).  Rows of
// a slice past nlast are computed but not stored: every reader of the
// per-row partials stops at nlast.  Keys at or past S only meet the last
// block, where the causal mask already hides them from its real rows.
// Warps:
//   0..15  statistics: warpgroup t owns tile t; thread = one query row
//   16     TMA producer
//   17..20 MMA issuers, one per tile (warp 17 also owns TMEM): each tile's
//          chain (score a 64-key half, drain it, score the next) runs on its
//          own, so a slow tile never holds back the others
//   21, 22 K column sums for the block means, one 64-column half each (only
//          CTAs of tile group 0)
// TMEM: tile t's 128x128 fp32 score tile at columns [128t, 128t+128), filled
// and drained as two 64-key halves with their own barriers.
// ---------------------------------------------------------------------------
struct ScoreParams {
  int S, Hq, Hkv, b, n, nch, g;
  int nsub;             // column parts per 128-key chunk: 2 when b = 64 (one per block), else 1
  int ld;               // rows from one head to the next (S, or more for packed sequences)
  int nlast;            // rows of the last block, S - (n-1)b
  int tiles_per_head;   // ceil(nlast / 128)
  int tiles_per_group;  // g * tiles_per_head
  int chunks_per_cta;
  float scale2;          // log2(e)/sqrt(d) (bf16); int8: multiplied by per-head scales
  const float *q_scale;  // int8 only
  const float *k_scale;
  float *pm, *plo, *phi;  // [Hq][nch * nsub][b]: per (head, column part, last-block row)
  float *ksum;            // [Hkv][nch * nsub][128]: K column sums per part
  int *err;
  // int8 test capture (null in normal use): the raw int32 score tile of
  // query head cap_h, last-block row slice cap_slice and key chunk cap_ch,
  // copied from tensor memory as the MMAs left it, row-major [128][128]
  int32_t *cap;
  int cap_h, cap_slice, cap_ch;
};

template <bool I8>
struct ScoreCfg {
  // two bf16 K stages: a third measured no faster (the kernel is bound by its exponentials)
  static constexpr int kStages = I8 ? 4 : 2;
  static constexpr int kTileBytes = I8 ? 16384 : 32768;  // 128 rows x 128 elements
  static constexpr int kTiles = 4;       // row tiles per CTA
  static constexpr int kSumWarps = 2;
  static constexpr int kThreads = (17 + kTiles + kSumWarps) * 32;
  static constexpr int kSmem = kTiles * kTileBytes + kStages * kTileBytes + 1024;
  // warps 0-15 statistics, 16 producer, 17-20 MMA issuers, 21-22 K column sums
  static_assert(kThreads == 736, "k_score_last warp roles need exactly 23 warps");
};

template <bool I8>
__global__ void __launch_bounds__(736, 1)
    k_score_last(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 ScoreParams P) {
  using C = ScoreCfg<I8>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_q, bar_kfull[C::kStages], bar_kempty[C::kStages], bar_sfull[4][2],
      bar_sfree[4][2];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kvh = blockIdx.z;
  const int tg0 = blockIdx.y * 4;
  const int T = min(4, P.tiles_per_group - tg0);
  const int ch0 = blockIdx.x * P.chunks_per_cta;
  const int ch1 = min(P.nch, ch0 + P.chunks_per_cta);
  const int U = ch1 - ch0;
  const bool do_ksum = (blockIdx.y == 0) && P.ksum != nullptr;  // null: the caller gave the K means
  const int n_ksum_warps = do_ksum ? C::kSumWarps : 0;
  const int tiles_per_head = P.tiles_per_head;

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t q_smem = base;                                // 4 tiles
  const uint32_t k_smem = base + 4 * C::kTileBytes;            // ring
  uint8_t *const k_gen = smem_raw + (k_smem - smem_u32(smem_raw));

  if (threadIdx.x == 0) {
    abort_sh = 0;
    mbar_init(smem_u32(&bar_q), 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(smem_u32(&bar_kfull[s]), 1);
      mbar_init(smem_u32(&bar_kempty[s]), T + n_ksum_warps);
    }
    for (int t = 0; t < 4; ++t)
      for (int hf = 0; hf < 2; ++hf) {
        mbar_init(smem_u32(&bar_sfull[t][hf]), 1);
        mbar_init(smem_u32(&bar_sfree[t][hf]), 4);
      }
    fence_mbar_init();
  }
  if (warp == 17) {
    tmem_alloc(smem_u32(&tmem_base_sh), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  volatile int *abort_flag = &abort_sh;

  if (U > 0) {
    if (warp == 16) {
      // ------------------------------------------------------------ producer
      if (lane == 0) {
        tma_prefetch_map(&tm_q);
        tma_prefetch_map(&tm_k);
        mbar_expect_tx(smem_u32(&bar_q), T * C::kTileBytes);
        for (int t = 0; t < T; ++t) {
          const int tile = tg0 + t;
          const int hh = kvh * P.g + tile / tiles_per_head;
          const int row = hh * P.ld + (P.n - 1) * P.b + (tile % tiles_per_head) * 128;
          const uint32_t dst = q_smem + t * C::kTileBytes;
          if (I8) {
            tma_load_2d(dst, &tm_q, 0, row, smem_u32(&bar_q));
          } else {
            tma_load_2d(dst, &tm_q, 0, row, smem_u32(&bar_q));
            tma_load_2d(dst + 16384, &tm_q, 64, row, smem_u32(&bar_q));
          }
        }
        for (int u = 0; u < U; ++u) {
          const int st = u % C::kStages;
          if (u >= C::kStages &&
              !mbar_wait(smem_u32(&bar_kempty[st]), ((u / C::kStages) - 1) & 1, abort_flag, P.err))
            break;
          const uint32_t dst = k_smem + st * C::kTileBytes;
          const int row = kvh * P.ld + (ch0 + u) * 128;
          mbar_expect_tx(smem_u32(&bar_kfull[st]), C::kTileBytes);
          tma_load_2d(dst, &tm_k, 0, row, smem_u32(&bar_kfull[st]));
          if (!I8) tma_load_2d(dst + 16384, &tm_k, 64, row, smem_u32(&bar_kfull[st]));
        }
      }
    } else if (warp >= 17 && warp < 17 + C::kTiles) {
      // ------------------------------------------------------------ MMA issuers
      // Warp 17 + t scores tile t: each 128-key chunk as two 64-key halves,
      // a half once the statistics warps have drained it from the previous
      // chunk.  Every issuer commits its own MMAs (a commit tracks the
      // issuing thread's operations) to the K stage's empty barrier.
      const int t = warp - 17;
      if (lane == 0 && t < T) {
        const uint32_t idesc = I8 ? idesc_i8(128, 64) : idesc_bf16(128, 64, 0);
        const uint32_t qb = q_smem + t * C::kTileBytes;
        bool ok = mbar_wait(smem_u32(&bar_q), 0, abort_flag, P.err);
        for (int u = 0; ok && u < U; ++u) {
          const int st = u % C::kStages;
          if (!mbar_wait(smem_u32(&bar_kfull[st]), (u / C::kStages) & 1, abort_flag, P.err)) break;
          const uint32_t kb = k_smem + st * C::kTileBytes;
          for (int hf = 0; hf < 2; ++hf) {
            if (u > 0 && !mbar_wait(smem_u32(&bar_sfree[t][hf]), (u - 1) & 1, abort_flag, P.err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t d_tmem = tmem + t * 128 + hf * 64;
            const uint32_t kh = kb + hf * 8192;  // key rows 64*hf .. 64*hf+63
            if (I8) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_i8_ss(d_tmem, umma_desc_sw128(qb + kk * 32, 16, 1024), umma_desc_sw128(kh + kk * 32, 16, 1024),
                          idesc, kk > 0);
            } else {
#pragma unroll
              for (int kk = 0; kk < 8; ++kk) {
                const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                mma_bf16_ss(d_tmem, umma_desc_sw128(qb + off, 16, 1024), umma_desc_sw128(kh + off, 16, 1024), idesc,
                            kk > 0);
              }
            }
            tc_commit(smem_u32(&bar_sfull[t][hf]));
          }
          if (!ok) break;
          tc_commit(smem_u32(&bar_kempty[st]));
        }
      }
    } else if (warp >= 17 + C::kTiles) {
      // ------------------------------------------------------------ K column sums
      // warp 21 + kh sums key columns 64kh .. 64kh+63 over the chunk's keys
      // inside [0, S)
      const int kh = warp - 17 - C::kTiles;
      if (kh < n_ksum_warps) {
        for (int u = 0; u < U; ++u) {
          const int st = u % C::kStages;
          if (!mbar_wait(smem_u32(&bar_kfull[st]), (u / C::kStages) & 1, abort_flag, P.err)) break;
          const uint8_t *tile = k_gen + st * C::kTileBytes;
          const int nrows = min(128, P.S - (ch0 + u) * 128);
          // one column sum per part: rows [sub*prow, (sub+1)*prow) of the chunk
          const int prow = 128 / P.nsub;
          for (int sub = 0; sub < P.nsub; ++sub) {
          float *out = P.ksum + ((size_t)kvh * P.nch * P.nsub + (size_t)(ch0 + u) * P.nsub + sub) * 128 + kh * 64;
          const int r_lo = sub * prow, r_hi = min(nrows, r_lo + prow);
          if (I8) {
            // one 128-byte row per key; lane owns bytes 64kh + 2lane, +1
            const int c16 = 4 * kh + (lane >> 3), within = (2 * lane) & 15;
            int acc0 = 0, acc1 = 0;
#pragma unroll 4
            for (int r = r_lo; r < r_hi; ++r) {
              const int phys = ((c16 ^ (r & 7)) << 4) | within;
              const uint32_t w = *reinterpret_cast<const uint16_t *>(tile + r * 128 + phys);
              acc0 += (int)(int8_t)(w & 0xff);
              acc1 += (int)(int8_t)((w >> 8) & 0xff);
            }
            out[2 * lane] = (float)acc0;
            out[2 * lane + 1] = (float)acc1;
          } else {
            // 64-column half kh (a 16 KB swizzled block); lane owns columns
            // 2lane, 2lane+1: the bf16 pair widened by bit moves and added as
            // one packed fp32 pair, even and odd rows in separate chains
            const uint8_t *hsrc = tile + kh * 16384;
            uint64_t ae = 0ull, ao = 0ull;
            const int c16 = lane >> 2, within = (lane & 3) << 2;
            auto row_pair = [&](int r) -> uint64_t {
              const uint32_t w = *reinterpret_cast<const uint32_t *>(hsrc + r * 128 + (((c16 ^ (r & 7)) << 4) | within));
              return f2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
            };
            int r = r_lo;
#pragma unroll 2
            for (; r + 1 < r_hi; r += 2) {
              ae = f2_add(ae, row_pair(r));
              ao = f2_add(ao, row_pair(r + 1));
            }
            if (r < r_hi) ae = f2_add(ae, row_pair(r));
            float x0, x1, y0, y1;
            f2_unpack(ae, x0, x1);
            f2_unpack(ao, y0, y1);
            out[2 * lane] = x0 + y0;
            out[2 * lane + 1] = x1 + y1;
          }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&bar_kempty[st]));
        }
      }
    } else {
      // ------------------------------------------------------------ statistics
      const int t = warp >> 2;
      if (t < T) {
        const int tile = tg0 + t;
        const int hh = kvh * P.g + tile / tiles_per_head;
        const int rloc = (warp & 3) * 32 + lane;                 // TMEM lane
        const int i = (tile % tiles_per_head) * 128 + rloc;      // row of the last block
        float scale2 = P.scale2;
        if (I8) scale2 *= P.q_scale[hh] * P.k_scale[kvh];
        const uint32_t taddr = tmem + t * 128 + (((warp & 3) * 32) << 16);
        const bool cap_on = I8 && P.cap != nullptr && hh == P.cap_h && (tile % tiles_per_head) == P.cap_slice;
        const uint64_t sc2 = f2_pack(scale2, scale2);
        bool ok = true;
        float m = -INFINITY;
        uint64_t lo2 = 0ull, hi2 = 0ull;  // the part's lo / hi sums as packed fp32 pairs
        for (int u = 0; u < U && ok; ++u) {
          const int ch = ch0 + u;
          // One pass over the chunk in 32-column pieces: lo/hi are kept
          // relative to the row's reference m (see below) and rescaled when
          // it moves.  Columns t <= i (block-relative) go to lo, the
          // rest to hi; in the last block columns t > i are causally masked
          // (their exponentials are 0).  With b = 64 each 64-column half is a
          // block of its own and gets its own (reference, lo, hi) part; otherwise
          // the chunk is one part.
          for (int hf = 0; hf < 2; ++hf) {
            if (hf == 0 || P.nsub == 2) lo2 = hi2 = 0ull;  // the reference m carries over
            if (!mbar_wait(smem_u32(&bar_sfull[t][hf]), u & 1, abort_flag, P.err)) { ok = false; break; }
            tc_fence_after();
#pragma unroll 1
            for (int qq = 0; qq < 2; ++qq) {
              uint32_t r[32];
              tmem_ld32(taddr + hf * 64 + qq * 32, r);
              tmem_ld_wait(r);
              if constexpr (I8) {
                if (cap_on && ch == P.cap_ch) {
                  int4 *dst = reinterpret_cast<int4 *>(P.cap + (size_t)rloc * 128 + hf * 64 + qq * 32);
#pragma unroll
                  for (int e = 0; e < 8; ++e)
                    dst[e] = make_int4((int)r[4 * e], (int)r[4 * e + 1], (int)r[4 * e + 2], (int)r[4 * e + 3]);
                }
              }
              const int key0 = ch * 128 + hf * 64 + qq * 32;  // first key of the piece
              const int blk = key0 / P.b;
              if (blk > P.n - 1) continue;                    // past the last block: masked
              const int dlt = i - (key0 - blk * P.b);         // columns e <= dlt are on the lo side
              float s[32];
#pragma unroll
              for (int e = 0; e < 32; ++e) s[e] = I8 ? i32_to_f32_small(r[e]) : __uint_as_float(r[e]);
              if (blk == P.n - 1 && dlt < 31) {
#pragma unroll
                for (int e = 0; e < 32; ++e) s[e] = (e <= dlt) ? s[e] : -INFINITY;
              }
              // the piece's lo / hi sums of 2^((s - m) scale2), exponent
              // arguments two at a time (packed fp32 FMA), ex2, packed adds
              auto piece = [&](uint64_t &pl, uint64_t &ph) {
                const float nm = -m * scale2;
                const uint64_t nm2 = f2_pack(nm, nm);
                pl = ph = 0ull;
                if (dlt >= 31 || dlt < 0) {
                  uint64_t a0 = 0ull, a1 = 0ull;
#pragma unroll
                  for (int e = 0; e < 32; e += 4) {
                    float x0, x1, x2, x3;
                    f2_unpack(f2_fma(f2_pack(s[e], s[e + 1]), sc2, nm2), x0, x1);
                    f2_unpack(f2_fma(f2_pack(s[e + 2], s[e + 3]), sc2, nm2), x2, x3);
                    a0 = f2_add(a0, f2_pack(ex2(x0), ex2(x1)));
                    a1 = f2_add(a1, f2_pack(ex2(x2), ex2(x3)));
                  }
                  if (dlt >= 31) pl = f2_add(a0, a1);
                  else ph = f2_add(a0, a1);
                } else {
#pragma unroll
                  for (int e = 0; e < 32; e += 2) {
                    float x0, x1;
                    f2_unpack(f2_fma(f2_pack(s[e], s[e + 1]), sc2, nm2), x0, x1);
                    const float p0 = ex2(x0), p1 = ex2(x1);
                    const bool q0 = e <= dlt, q1 = e + 1 <= dlt;
                    pl = f2_add(pl, f2_pack(q0 ? p0 : 0.f, q1 ? p1 : 0.f));
                    ph = f2_add(ph, f2_pack(q0 ? 0.f : p0, q1 ? 0.f : p1));
                  }
                }
              };
              // Exponentials first, against the row's reference m (raw score
              // units).  The reference moves -- to the piece max plus
              // kScoreHeadroom (log2 units) -- only when the piece's sum
              // exceeds 2^8 or the row has no reference yet; the piece is then
              // recomputed and the part's sums so far rescaled.  The per-part
              // partials carry the reference in place of a maximum, which the
              // statistics kernel's log-sum-exp combination allows.
              uint64_t pl, ph;
              bool move = (m == -INFINITY);
              if (!move) {
                piece(pl, ph);
                float a, b2, c, d2;
                f2_unpack(pl, a, b2);
                f2_unpack(ph, c, d2);
                move = !((a + b2) + (c + d2) <= 256.f);
              }
              if (move) {
                float m8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) m8[e] = fmax3(s[e], s[8 + e], s[16 + e]);
#pragma unroll
                for (int e = 0; e < 8; ++e) m8[e] = fmaxf(m8[e], s[24 + e]);
                const float pmx =
                    fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
                if (pmx == -INFINITY) continue;  // whole piece masked and no reference yet
                const float nmv = fmaxf(m, pmx + kScoreHeadroom / scale2);
                if (nmv > m) {
                  const float f = (m == -INFINITY) ? 0.f : ex2((m - nmv) * scale2);
                  const uint64_t f2 = f2_pack(f, f);
                  lo2 = f2_mul(lo2, f2);
                  hi2 = f2_mul(hi2, f2);
                  m = nmv;
                }
                piece(pl, ph);
              }
              lo2 = f2_add(lo2, pl);
              hi2 = f2_add(hi2, ph);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&bar_sfree[t][hf]));
            if ((hf == 1 || P.nsub == 2) && i < P.nlast) {
              float l_a, l_b, h_a, h_b;
              f2_unpack(lo2, l_a, l_b);
              f2_unpack(hi2, h_a, h_b);
              const int part = ch * P.nsub + (P.nsub == 2 ? hf : 0);
              const size_t o = ((size_t)hh * P.nch * P.nsub + part) * P.b + i;
              P.pm[o] = m * scale2;
              P.plo[o] = l_a + l_b;
              P.phi[o] = h_a + h_b;
            }
          }
          if (!ok) break;
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
// k_head_stats: statistics finalise and pattern choice, one cluster of
// kStatCta CTAs per query head h (grid (kStatCta, Hq), 256 threads).  Rank
// k of the cluster owns the key blocks [k n / C, (k+1) n / C) and their
// column parts.  With nlast = S - (n-1)b rows in the last block and the
// score kernel's per-(row, part) partials (m, the reference the part's sums
// are taken against, in log2 units; lo; hi -- any reference gives the same
// combined statistics):
//   1. row statistics over the owned parts, combined over the cluster
//      through distributed shared memory (in rank order):
//        M_i = max_p m_ip,  L_i = sum_p (lo_ip + hi_ip) 2^(m_ip - M_i);
//      and a rank's slice of the last block's query rows summed per column
//      (qbar_last = mean of the nlast rows);
//   2. per owned part: LO_p = sum_i lo_ip 2^(m_ip - M_i) / L_i, HI_p alike;
//      per owned block: vhat[c] = (LO[c] + HI[c]) / nlast, the block mean
//      kbar_c of K, and the logit z_c = qbar_last . kbar_c / sqrt(d);
//   3. shat[o] = (LO[n-1-o] + HI[n-2-o]) / nlast (the mirrored blocks are
//      read from their owners), P_est = softmax_c(z_c) with the cluster's
//      max and sum, and JSD(vhat, P_est) (natural log) summed over ranks;
//      pattern = QA iff JSD < tau.
// Every reduction runs in a fixed order.  kbar is written for the KV head by
// the cluster of its first query head (h % g == 0); when the caller supplies
// the K block means (ext_kbar) they are read instead of the column sums.
// ---------------------------------------------------------------------------
constexpr int kStatCta = 8;
constexpr int kStatThreads = 512;  // two CTAs per SM: 256 clustered CTAs (32 heads) run in one wave
constexpr int kStatMaxOwnParts = 256;   // npart <= 2048
constexpr int kStatMaxOwnBlocks = 128;  // n <= 1024

struct HeadStatsParams {
  int S, b, n, npart, g, ld, nlast;
  const float *pm, *plo, *phi;   // [Hq][npart][b]
  const float *ksum;             // [Hkv][npart][128] K column sums per part
  const float *ext_kbar;         // [Hkv][n][128] block means given by the caller, or null
  const float *k_scale;          // int8 only
  const void *q;                 // last block rows for qbar_last
  const float *q_scale;          // int8 only
  float inv_sqrt_d, tau;
  float *vhat, *shat, *pest, *jsd;
  int *pattern;
  float *kbar;                   // [Hkv][n][128] out (when computed here)
};

__device__ __forceinline__ int stat_block0(int k, int n) { return (k * n) / kStatCta; }

template <bool I8>
__global__ void __cluster_dims__(kStatCta, 1, 1) __launch_bounds__(kStatThreads, 2)
    k_head_stats(HeadStatsParams P) {
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  __shared__ float grpM[kStatThreads], grpL[kStatThreads];   // per thread group, phase 1
  __shared__ float rowM[256], rowL[256];                     // this rank's row partials (shared)
  __shared__ float gM[256], gInvL[256];                      // cluster row statistics
  __shared__ float qpart[128], qb[128];                      // last-block query column sums / mean
  __shared__ float qgrp[kStatThreads / 128][128];            // per row group, before qpart
  __shared__ float LOp[kStatMaxOwnParts], HIp[kStatMaxOwnParts];
  __shared__ float LOb[kStatMaxOwnBlocks], HIb[kStatMaxOwnBlocks];  // owned blocks (shared)
  __shared__ float vh[kStatMaxOwnBlocks], zc[kStatMaxOwnBlocks];
  __shared__ float red[kStatThreads / 32];
  __shared__ float xch[4];                                    // [0] local max, [1] local sum, [2] local JSD

  const int k = (int)cl.block_rank(), h = blockIdx.y, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5, nwarp = kStatThreads / 32;
  const int b = P.b, n = P.n, npart = P.npart, nlast = P.nlast;
  const int kvh = h / P.g;
  const int per = b >= 128 ? b / 128 : 1;  // parts per block
  const int c0 = stat_block0(k, n), c1 = stat_block0(k + 1, n);
  const int p0 = min(npart, c0 * per), p1 = min(npart, c1 * per);
  const size_t hoff = (size_t)h * npart * b;

  // ---- 1. row statistics over the owned parts; query column sums of a row slice
  {
    const int G = kStatThreads / b, i = tid % b, j = tid / b;
    float M = -INFINITY, L = 0.f;
    if (i < nlast) {
      // four parts' partials in flight, then the running combine in part order
      for (int p = p0 + j; p < p1; p += 4 * G) {
        float mv[4], sv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int pp = p + u * G;
          const size_t o = hoff + (size_t)pp * b + i;
          const bool in = pp < p1;
          mv[u] = in ? P.pm[o] : -INFINITY;
          sv[u] = in ? P.plo[o] + P.phi[o] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float m = mv[u];
          if (m == -INFINITY) continue;
          if (m > M) {
            L = L * ex2(M - m) + sv[u];
            M = m;
          } else {
            L += sv[u] * ex2(m - M);
          }
        }
      }
    }
    grpM[tid] = M;
    grpL[tid] = L;
    {
      // rows r0 .. r1-1 of the last block, column tid % 128, row group tid / 128
      const int r0 = (k * nlast) / kStatCta, r1 = ((k + 1) * nlast) / kStatCta;
      const int c = tid & 127, rg = tid >> 7, RG = kStatThreads / 128;
      const size_t base = ((size_t)h * P.ld + (size_t)(n - 1) * b) * 128 + c;
      float acc = 0.f;
      if (I8) {
        const int8_t *q8 = reinterpret_cast<const int8_t *>(P.q);
        int ia = 0;
        for (int r = r0 + rg; r < r1; r += RG) ia += q8[base + (size_t)r * 128];
        acc = (float)ia;
      } else {
        const __nv_bfloat16 *qh = reinterpret_cast<const __nv_bfloat16 *>(P.q);
        for (int r = r0 + rg; r < r1; r += RG) acc += __bfloat162float(qh[base + (size_t)r * 128]);
      }
      qgrp[rg][c] = acc;
    }
    __syncthreads();
    if (tid < 128) {
      float a = 0.f;
      for (int rg = 0; rg < kStatThreads / 128; ++rg) a += qgrp[rg][tid];
      qpart[tid] = a;
    }
    if (tid < b) {
      float Mi = -INFINITY, Li = 0.f;
      for (int jj = 0; jj < G; ++jj) {
        const float m = grpM[jj * b + tid];
        if (m == -INFINITY) continue;
        const float l = grpL[jj * b + tid];
        if (m > Mi) {
          Li = Li * ex2(Mi - m) + l;
          Mi = m;
        } else {
          Li += l * ex2(m - Mi);
        }
      }
      rowM[tid] = Mi;
      rowL[tid] = Li;
    }
  }
  cl.sync();  // (1) row partials and query column sums of every rank visible
  if (tid < b) {
    float Mi = -INFINITY;
    for (int r = 0; r < kStatCta; ++r) Mi = fmaxf(Mi, cl.map_shared_rank(rowM, r)[tid]);
    float Li = 0.f;
    for (int r = 0; r < kStatCta; ++r) {
      const float m = cl.map_shared_rank(rowM, r)[tid];
      if (m != -INFINITY) Li += cl.map_shared_rank(rowL, r)[tid] * ex2(m - Mi);
    }
    gM[tid] = Mi;
    gInvL[tid] = (tid < nlast && Li > 0.f) ? 1.f / Li : 0.f;
  }
  if (tid < 128) {
    float a = 0.f;
    for (int r = 0; r < kStatCta; ++r) a += cl.map_shared_rank(qpart, r)[tid];
    qb[tid] = (I8 ? a * P.q_scale[h] : a) / (float)nlast;
  }
  __syncthreads();

  // ---- 2. part masses (warp per part, lanes over rows), block masses, kbar and logits
  for (int p = p0 + warp; p < p1; p += nwarp) {
    float a = 0.f, c = 0.f;
    float mv[8], lv[8], hv[8];  // the lane's rows i = lane + 32 t of the part (b <= 256)
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const int i = lane + 32 * t;
      const bool in = i < b && i < nlast;
      const size_t o = hoff + (size_t)p * b + i;
      mv[t] = in ? P.pm[o] : -INFINITY;
      lv[t] = in ? P.plo[o] : 0.f;
      hv[t] = in ? P.phi[o] : 0.f;
    }
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const int i = lane + 32 * t;
      const float w = (mv[t] == -INFINITY) ? 0.f : ex2(mv[t] - gM[i]) * gInvL[i];
      a += lv[t] * w;
      c += hv[t] * w;
    }
#pragma unroll
    for (int sft = 16; sft > 0; sft >>= 1) {
      a += __shfl_xor_sync(0xffffffffu, a, sft);
      c += __shfl_xor_sync(0xffffffffu, c, sft);
    }
    if (lane == 0) {
      LOp[p - p0] = a;
      HIp[p - p0] = c;
    }
  }
  __syncthreads();
  const float inv_nl = 1.f / (float)nlast;
  for (int c = c0 + tid; c < c1; c += kStatThreads) {
    float a = 0.f, e = 0.f;
    for (int q = 0; q < per && c * per + q < npart; ++q) {
      a += LOp[c * per + q - p0];
      e += HIp[c * per + q - p0];
    }
    LOb[c - c0] = a;
    HIb[c - c0] = e;
    vh[c - c0] = (a + e) * inv_nl;
    P.vhat[(size_t)h * n + c] = (a + e) * inv_nl;
  }
  // block means of K (warp per block) and the logits of P_est
  const bool write_kbar = (h % P.g) == 0 && P.ext_kbar == nullptr;
  for (int c = c0 + warp; c < c1; c += nwarp) {
    float kv[4];
    if (P.ext_kbar) {
#pragma unroll
      for (int t = 0; t < 4; ++t) kv[t] = P.ext_kbar[((size_t)kvh * n + c) * 128 + lane + 32 * t];
    } else {
      const int rows = min(b, P.S - c * b);
      float sc = 1.f / (float)rows;
      if (I8) sc *= P.k_scale[kvh];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        float s2 = 0.f;
        for (int q = 0; q < per && c * per + q < npart; ++q)
          s2 += P.ksum[((size_t)kvh * npart + c * per + q) * 128 + lane + 32 * t];
        kv[t] = s2 * sc;
        if (write_kbar) P.kbar[((size_t)kvh * n + c) * 128 + lane + 32 * t] = kv[t];
      }
    }
    float z = 0.f;
#pragma unroll
    for (int t = 0; t < 4; ++t) z = fmaf(qb[lane + 32 * t], kv[t], z);
#pragma unroll
    for (int sft = 16; sft > 0; sft >>= 1) z += __shfl_xor_sync(0xffffffffu, z, sft);
    if (lane == 0) zc[c - c0] = z * P.inv_sqrt_d;
  }
  __syncthreads();
  {
    float mx = -INFINITY;
    for (int c = c0 + tid; c < c1; c += kStatThreads) mx = fmaxf(mx, zc[c - c0]);
#pragma unroll
    for (int sft = 16; sft > 0; sft >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, sft));
    if (lane == 0) red[warp] = mx;
    __syncthreads();
    if (tid == 0) {
      float m = red[0];
      for (int w = 1; w < nwarp; ++w) m = fmaxf(m, red[w]);
      xch[0] = m;
    }
  }
  cl.sync();  // (2) block masses and logit maxima of every rank visible
  // slash statistics of the owned offsets from the mirrored blocks' owners
  for (int o = c0 + tid; o < c1; o += kStatThreads) {
    const int cl_ = n - 1 - o;
    int kr = kStatCta - 1;
    while (stat_block0(kr, n) > cl_) --kr;
    float sv = cl.map_shared_rank(LOb, kr)[cl_ - stat_block0(kr, n)];
    if (o <= n - 2) {
      const int ch = n - 2 - o;
      int kh = kStatCta - 1;
      while (stat_block0(kh, n) > ch) --kh;
      sv += cl.map_shared_rank(HIb, kh)[ch - stat_block0(kh, n)];
    }
    P.shat[(size_t)h * n + o] = sv * inv_nl;
  }
  float gmax = -INFINITY;
  for (int r = 0; r < kStatCta; ++r) gmax = fmaxf(gmax, cl.map_shared_rank(xch, r)[0]);
  {
    float sum = 0.f;
    for (int c = c0 + tid; c < c1; c += kStatThreads) {
      const float e = expf(zc[c - c0] - gmax);
      zc[c - c0] = e;
      sum += e;
    }
#pragma unroll
    for (int sft = 16; sft > 0; sft >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, sft);
    if (lane == 0) red[warp] = sum;
    __syncthreads();
    if (tid == 0) {
      float s2 = 0.f;
      for (int w = 0; w < nwarp; ++w) s2 += red[w];
      xch[1] = s2;
    }
  }
  cl.sync();  // (3) local exponential sums visible
  float gsum = 0.f;
  for (int r = 0; r < kStatCta; ++r) gsum += cl.map_shared_rank(xch, r)[1];
  {
    float js = 0.f;
    for (int c = c0 + tid; c < c1; c += kStatThreads) {
      const float pe = zc[c - c0] / gsum;
      P.pest[(size_t)h * n + c] = pe;
      const float pv = vh[c - c0];
      const float m = 0.5f * (pv + pe);
      if (pv > 0.f) js += 0.5f * pv * logf(pv / m);
      if (pe > 0.f) js += 0.5f * pe * logf(pe / m);
    }
#pragma unroll
    for (int sft = 16; sft > 0; sft >>= 1) js += __shfl_xor_sync(0xffffffffu, js, sft);
    __syncthreads();  // red[] reuse
    if (lane == 0) red[warp] = js;
    __syncthreads();
    if (tid == 0) {
      float s2 = 0.f;
      for (int w = 0; w < nwarp; ++w) s2 += red[w];
      xch[2] = s2;
    }
  }
  cl.sync();  // (4) local divergences visible
  if (k == 0 && tid == 0) {
    float tot = 0.f;
    for (int r = 0; r < kStatCta; ++r) tot += cl.map_shared_rank(xch, r)[2];
    P.jsd[h] = tot;
    P.pattern[h] = (tot < P.tau) ? 1 : 0;
  }
  cl.sync();  // (5) no rank leaves while another may still read its shared memory
}

// ---------------------------------------------------------------------------
// k_qpool: grid (n, Hq), block 128, at most 64 registers per thread, no
// shared memory, so that 8 CTAs (32 warps, 256 loads of 16 bytes in flight
// per SM sub-partition) share an SM.  For the query-aware heads only (the
// CTAs of the others exit at once): qbar[h][r][t] = mean of the Q rows of
// block r (b rows, or S - (n-1)b for a partial last block).  Runs after the
// pattern decision.  (Pooling every head beside k_score_last instead, on a
// second stream or in extra warps of that kernel, measured slower: the
// score kernel holds the register file and almost all shared memory of its
// SM, which leaves the pooling too few bytes in flight.)
// Warp w owns columns 32w .. 32w+31; lane (c = lane & 3, rr = lane >> 2)
// loads 16 bytes of rows rr, rr + 8, ..., eight rows' loads in flight, and
// the rows are summed across lanes with shuffles.  The block kPoolAhead
// blocks ahead is prefetched into L2 (bulk prefetch, no registers held).
// ---------------------------------------------------------------------------
constexpr int kPoolAhead = 4;

__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(p)), "r"(bytes)
               : "memory");
}

template <bool I8>
__global__ void __maxnreg__(64)
    k_qpool(const int *__restrict__ pattern, const void *__restrict__ q, const float *__restrict__ q_scale, int S,
            int ld, int b, int n, float *__restrict__ qbar) {
  const int r = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
  if (pattern[h] != 1) return;
  const size_t row0 = (size_t)h * ld + (size_t)r * b;
  const int rows = min(b, S - r * b);
  const int esz = I8 ? 1 : 2;
  if (tid == 0 && r + kPoolAhead < n) {
    const int ra = r + kPoolAhead;
    const int arows = min(b, S - ra * b);
    // 16-byte multiples: a row is 128 (int8) or 256 (bf16) bytes
    prefetch_l2(reinterpret_cast<const char *>(q) + ((size_t)h * ld + (size_t)ra * b) * 128 * esz,
                (uint32_t)arows * 128u * esz);
  }
  const int warp = tid >> 5, lane = tid & 31;
  float *out = qbar + ((size_t)h * n + r) * 128 + warp * 32;
  if (I8) {
    // warp's 32 columns = 32 bytes per row: lane (c = lane & 1, rr = lane >> 1) owns 16 columns, 16 rows per pass
    const int8_t *q8 = reinterpret_cast<const int8_t *>(q);
    const int c = lane & 1, rr = lane >> 1;
    int acc[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) acc[e] = 0;
    for (int p = rr; p < rows; p += 16 * 8) {
      int4 v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        v[j] = (p + 16 * j < rows)
                   ? *reinterpret_cast<const int4 *>(q8 + (row0 + p + 16 * j) * 128 + warp * 32 + c * 16)
                   : make_int4(0, 0, 0, 0);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int w4[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[e] += (int)(int8_t)((w4[e >> 2] >> (8 * (e & 3))) & 0xff);
      }
    }
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      int a = acc[e];
#pragma unroll
      for (int sft = 2; sft < 32; sft <<= 1) a += __shfl_xor_sync(0xffffffffu, a, sft);
      acc[e] = a;
    }
    if (lane < 2) {
#pragma unroll
      for (int e = 0; e < 16; ++e) out[c * 16 + e] = (float)acc[e] * q_scale[h] / (float)rows;
    }
  } else {
    // warp's 32 columns = 64 bytes per row: lane (c = lane & 3, rr = lane >> 2) owns 8 columns, 8 rows per pass
    const __nv_bfloat16 *qh = reinterpret_cast<const __nv_bfloat16 *>(q);
    const int c = lane & 3, rr = lane >> 2;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    for (int p = rr; p < rows; p += 8 * 8) {
      uint4 v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        v[j] = (p + 8 * j < rows)
                   ? *reinterpret_cast<const uint4 *>(qh + (row0 + p + 8 * j) * 128 + warp * 32 + c * 8)
                   : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t w4[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc[2 * e] += __uint_as_float(w4[e] << 16);
          acc[2 * e + 1] += __uint_as_float(w4[e] & 0xFFFF0000u);
        }
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
#pragma unroll
      for (int sft = 4; sft < 32; sft <<= 1) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], sft);
    }
    if (lane < 4) {
#pragma unroll
      for (int e = 0; e < 8; ++e) out[c * 8 + e] = acc[e] / (float)rows;
    }
  }
}

// ---------------------------------------------------------------------------
// k_qa_logits_fma: grid (nt(nt+1)/2, Hq) with nt = ceil(n/64), block 256.  The
// form for small n, where k_qa_logits (tensor cores, 128 x 128 tiles) has too
// few tiles to fill the GPU; same output.  For
// query-aware heads only (others exit): the lower triangle of
// Z = qbar kbar^T / sqrt(d), z[h][r][c] for c <= r, in the padded triangular
// layout (row r at h*n(n+1)/2 + r(r+1)/2).  Tiled fp32 product: 64 x 64
// output tile per CTA, 4 x 4 outputs per thread held as column pairs and
// updated with packed fp32 FMAs; d is staged through shared memory 32 at a
// time, double-buffered (the next slice is loaded into registers while the
// current one is multiplied).
// ---------------------------------------------------------------------------
constexpr int kLgFmaTile = 64;
constexpr int kLgK = 32;
constexpr int kLgStride = kLgFmaTile + 4;  // float4-aligned rows

__global__ void __launch_bounds__(256)
    k_qa_logits_fma(const int *__restrict__ pattern, const float *__restrict__ qbar,
                const float *__restrict__ kbar, int g, int n, float inv_sqrt_d, float *__restrict__ z) {
  const int h = blockIdx.y;
  if (pattern[h] != 1) return;
  __shared__ __align__(16) float As[2][kLgK][kLgStride];  // [buffer][k][row]
  __shared__ __align__(16) float Bs[2][kLgK][kLgStride];  // [buffer][k][col]
  // lower-triangular tile (tr, tc), tc <= tr, from the linear index
  const int x = blockIdx.x;
  int tr = (int)((sqrtf(8.f * (float)x + 1.f) - 1.f) * 0.5f);
  while ((tr + 1) * (tr + 2) / 2 <= x) ++tr;
  while (tr * (tr + 1) / 2 > x) --tr;
  const int tc = x - tr * (tr + 1) / 2;
  const int kvh = h / g;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int row0 = tr * kLgFmaTile, col0 = tc * kLgFmaTile;
  const float *qh = qbar + (size_t)h * n * 128;
  const float *kh = kbar + (size_t)kvh * n * 128;
  // this thread's share of a k-slice: rows rr0, rr0 + 32 of q-bar and k-bar, 4 consecutive k
  const int rr0 = tid >> 3, k4 = (tid & 7) * 4;
  float4 qa[2], kb[2];
  auto load = [&](int k0) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int rr = rr0 + 32 * u;
      qa[u] = (row0 + rr < n) ? *reinterpret_cast<const float4 *>(qh + (size_t)(row0 + rr) * 128 + k0 + k4)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
      kb[u] = (col0 + rr < n) ? *reinterpret_cast<const float4 *>(kh + (size_t)(col0 + rr) * 128 + k0 + k4)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  auto store = [&](int buf) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int rr = rr0 + 32 * u;
      As[buf][k4 + 0][rr] = qa[u].x; As[buf][k4 + 1][rr] = qa[u].y;
      As[buf][k4 + 2][rr] = qa[u].z; As[buf][k4 + 3][rr] = qa[u].w;
      Bs[buf][k4 + 0][rr] = kb[u].x; Bs[buf][k4 + 1][rr] = kb[u].y;
      Bs[buf][k4 + 2][rr] = kb[u].z; Bs[buf][k4 + 3][rr] = kb[u].w;
    }
  };
  uint64_t acc[4][2];  // rows ty*4 + a, column pairs tx*4 + 2p, +1
#pragma unroll
  for (int a = 0; a < 4; ++a) acc[a][0] = acc[a][1] = 0ull;
  load(0);
  store(0);
  __syncthreads();
#pragma unroll 1
  for (int kt = 0; kt < 128 / kLgK; ++kt) {
    const int buf = kt & 1;
    if (kt + 1 < 128 / kLgK) load((kt + 1) * kLgK);
#pragma unroll 8
    for (int k = 0; k < kLgK; ++k) {
      const float4 a4 = *reinterpret_cast<const float4 *>(&As[buf][k][ty * 4]);
      const float4 b4 = *reinterpret_cast<const float4 *>(&Bs[buf][k][tx * 4]);
      const uint64_t b01 = f2_pack(b4.x, b4.y), b23 = f2_pack(b4.z, b4.w);
      const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const uint64_t aa = f2_pack(av[a], av[a]);
        acc[a][0] = f2_fma(aa, b01, acc[a][0]);
        acc[a][1] = f2_fma(aa, b23, acc[a][1]);
      }
    }
    if (kt + 1 < 128 / kLgK) store(buf ^ 1);
    __syncthreads();
  }
  float *zh = z + (size_t)h * ((size_t)n * (n + 1) / 2);
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int r = row0 + ty * 4 + a;
    if (r >= n) continue;
    float v[4];
    f2_unpack(acc[a][0], v[0], v[1]);
    f2_unpack(acc[a][1], v[2], v[3]);
#pragma unroll
    for (int b2 = 0; b2 < 4; ++b2) {
      const int c = col0 + tx * 4 + b2;
      if (c <= r) zh[(size_t)r * (r + 1) / 2 + c] = v[b2] * inv_sqrt_d;
    }
  }
}

// ---------------------------------------------------------------------------
// k_split_tf32: one warp per row of 128 fp32 block means (block 256 = 8
// rows); row r of src becomes row r of dst as 256 floats: x_hi = tf32(x) in
// columns 0..127 and x_lo = tf32(x - x_hi) in columns 128..255 (nearest,
// ties away).  With pattern given, rows of heads that are not query-aware
// (head = row / n) are skipped.  The operands of k_qa_logits.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
    k_split_tf32(const float *__restrict__ src, float *__restrict__ dst, int rows, int n,
                 const int *__restrict__ pattern) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= rows) return;
  if (pattern != nullptr && pattern[row / n] != 1) return;
  const float4 v = *reinterpret_cast<const float4 *>(src + (size_t)row * 128 + lane * 4);
  const float a[4] = {v.x, v.y, v.z, v.w};
  uint32_t hi[4], lo[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    hi[e] = tf32_rna(a[e]);
    lo[e] = tf32_rna(a[e] - __uint_as_float(hi[e]));
  }
  *reinterpret_cast<uint4 *>(dst + (size_t)row * 256 + lane * 4) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
  *reinterpret_cast<uint4 *>(dst + (size_t)row * 256 + 128 + lane * 4) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
}

// ---------------------------------------------------------------------------
// k_qa_logits: grid (nt(nt+1)/2, Hq) with nt = ceil(n/128), block 128.  For
// query-aware heads only (others exit): the lower triangle of
// Z = qbar kbar^T / sqrt(d), z[h][r][c] for c <= r, in the padded triangular
// layout (row r at h*n(n+1)/2 + r(r+1)/2), one 128 x 128 tile per CTA on the
// tensor cores.  The operands come split by k_split_tf32 (x = x_hi + x_lo,
// both tf32); the tile accumulates hi.hi + hi.lo + lo.hi in fp32 in tensor
// memory (the dropped lo.lo term and the two roundings are each at most 2^-22
// of a product, together below 2^-20: fp32-class).  Thread 0 streams d in four
// slabs of 32 through one 64 KB shared-memory slot (q_hi, q_lo, k_hi, k_lo:
// 128 rows x 128 bytes each, TMA with the 128-byte swizzle) and issues 12
// MMAs (M = N = 128, K = 8) per slab; the slot is refilled once its MMAs
// have completed.  With one slot three CTAs share an SM and hide each
// other's load and MMA latencies (a two-slot ring with one CTA per SM
// measured slower).
// Epilogue: warp w reads rows 32w.. of the accumulator, scales by 1/sqrt(d)
// and stages them in the slot (column c of row r at c ^ (r % 32): no bank
// conflicts either way); the CTA then writes each row's c <= r part
// contiguously.
// ---------------------------------------------------------------------------
constexpr int kLgTile = 128;
// smallest n that takes this kernel.  Below it the 64 x 64 FMA form, with
// more CTAs and no split pass, is as fast or faster; measured index passes
// (32 heads, half query-aware), tensor cores (three CTAs per SM) vs FMA:
// 0.267 vs 0.261 ms at n = 512, 0.384 vs 0.397 at 768, 0.512 vs 0.529 at
// 1024 (0.501 vs 0.521 int8)
constexpr int kLgTensorMinN = 640;
constexpr int kLgSlab = 16384;            // 128 rows x 32 tf32
constexpr int kLgSlot = 4 * kLgSlab;      // q_hi, q_lo, k_hi, k_lo
constexpr int kLgSmem = kLgSlot + 1024;   // one slot: three CTAs share an SM
static_assert(kLgTile * kLgTile * 4 <= kLgSlot, "k_qa_logits staging exceeds the slot");

__global__ void __launch_bounds__(128, 3)
    k_qa_logits(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const int *__restrict__ pattern, int g, int n, float inv_sqrt_d, int *__restrict__ err,
                float *__restrict__ z) {
  const int h = blockIdx.y;
  if (pattern[h] != 1) return;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_full, bar_empty, bar_done;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  // lower-triangular tile (tr, tc), tc <= tr, from the linear index
  const int x = blockIdx.x;
  int tr = (int)((sqrtf(8.f * (float)x + 1.f) - 1.f) * 0.5f);
  while ((tr + 1) * (tr + 2) / 2 <= x) ++tr;
  while (tr * (tr + 1) / 2 > x) --tr;
  const int tc = x - tr * (tr + 1) / 2;
  const int kvh = h / g;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  float *const stage = reinterpret_cast<float *>(smem_raw + (base - smem_u32(smem_raw)));
  if (tid == 0) {
    abort_sh = 0;
    mbar_init(smem_u32(&bar_full), 1);
    mbar_init(smem_u32(&bar_empty), 1);
    mbar_init(smem_u32(&bar_done), 1);
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
  if (tid == 0) {
    tma_prefetch_map(&tm_q);
    tma_prefetch_map(&tm_k);
    const int qy = h * n + tr * kLgTile, ky = kvh * n + tc * kLgTile;
    auto load = [&](int sb) {  // slab sb of d into the slot
      const uint32_t bar = smem_u32(&bar_full);
      mbar_expect_tx(bar, kLgSlot);
      tma_load_2d(base + 0 * kLgSlab, &tm_q, 32 * sb, qy, bar);
      tma_load_2d(base + 1 * kLgSlab, &tm_q, 128 + 32 * sb, qy, bar);
      tma_load_2d(base + 2 * kLgSlab, &tm_k, 32 * sb, ky, bar);
      tma_load_2d(base + 3 * kLgSlab, &tm_k, 128 + 32 * sb, ky, bar);
    };
    const uint32_t idesc = idesc_tf32(128, 128);
    load(0);
    bool ok = true;
    for (int sb = 0; sb < 4 && ok; ++sb) {
      if (!mbar_wait(smem_u32(&bar_full), sb & 1, abort_flag, err)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t a_hi = umma_desc_sw128(base + 0 * kLgSlab + kk * 32, 16, 1024);
        const uint64_t a_lo = umma_desc_sw128(base + 1 * kLgSlab + kk * 32, 16, 1024);
        const uint64_t b_hi = umma_desc_sw128(base + 2 * kLgSlab + kk * 32, 16, 1024);
        const uint64_t b_lo = umma_desc_sw128(base + 3 * kLgSlab + kk * 32, 16, 1024);
        mma_tf32_ss(tmem, a_hi, b_hi, idesc, (sb > 0 || kk > 0));
        mma_tf32_ss(tmem, a_hi, b_lo, idesc, 1);
        mma_tf32_ss(tmem, a_lo, b_hi, idesc, 1);
      }
      if (sb + 1 < 4) {
        tc_commit(smem_u32(&bar_empty));
        if (!mbar_wait(smem_u32(&bar_empty), sb & 1, abort_flag, err)) { ok = false; break; }
        load(sb + 1);
      }
    }
    tc_commit(smem_u32(&bar_done));  // arrives once every MMA issued above has completed
  }
  __syncwarp();
  const bool ok = mbar_wait(smem_u32(&bar_done), 0, abort_flag, err) && !*abort_flag;
  if (ok) {
    tc_fence_after();
    // accumulator row 32w + lane -> staging row (scaled)
    const int row = warp * 32 + lane;
#pragma unroll 1
    for (int q4 = 0; q4 < 4; ++q4) {
      uint32_t v[32];
      tmem_ld32(tmem + (((uint32_t)(warp * 32)) << 16) + q4 * 32, v);
      tmem_ld_wait(v);
#pragma unroll
      for (int e = 0; e < 32; ++e) stage[row * kLgTile + ((q4 * 32 + e) ^ lane)] = __uint_as_float(v[e]) * inv_sqrt_d;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (ok) {
    // row r of the tile: columns tc*128 + c with c <= rq, one contiguous run
    float *zh = z + (size_t)h * ((size_t)n * (n + 1) / 2);
#pragma unroll 1
    for (int r = 0; r < kLgTile; ++r) {
      const int rq = tr * kLgTile + r;
      if (rq >= n) break;
      const int cmax = rq - tc * kLgTile;  // last column of the run, tile-relative
      if (tid <= cmax) zh[(size_t)rq * (rq + 1) / 2 + tc * kLgTile + tid] = stage[r * kLgTile + (tid ^ (r & 31))];
    }
  }
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// ---------------------------------------------------------------------------
// k_cut: one warp per (head, query block r), heavy rows first; block 256.
// Scores over c <= r:  VS: w_c = vhat[c] + shat[r - c];  QA: w_c = exp(z_c -
// max) (as 2^((z_c - max) log2 e)); normalised to sum 1 (times the reciprocal
// of the sum).  The diagonal is kept; the others are kept in
// order of descending score (ties: lower index) while the kept sum is below
// gamma.  The cut is found by bisection on the fp32 bit pattern of the
// scores (monotone for positive floats), between the smallest and the
// largest candidate: T = largest t with sum_{c < r, bits(w_c) >= t} w_c >=
// gamma - w_r, stopping as soon as one candidate is left between the
// bounds; everything above T is kept, then ties at T by ascending index
// until the target is reached.  The row lives in registers (element c in
// lane c % 32, slot c / 32; the diagonal's slot is zeroed once w_r is read,
// so a slot's bit pattern is its key and non-candidates never qualify).
// Sums: each lane adds its slots in fp32 in a fixed order; the lane sums
// are converted to fixed point (2^-30 units, exact integer addition) and
// reduced across the warp in one instruction, so every sum is deterministic
// and monotone in the threshold.
// Output: counts[h*n + r], ascending list at cols[h*n(n+1)/2 + r(r+1)/2].
// ---------------------------------------------------------------------------
constexpr int kSelMaxN = 1024;
constexpr float kCutFx = 1073741824.f;  // 2^30

template <int NL>
__device__ __forceinline__ void cut_row(int pat, int h, int r, int n, const float *__restrict__ vhat,
                                        const float *__restrict__ shat, const float *__restrict__ zrow,
                                        float gamma, int *__restrict__ out, int *__restrict__ count_out) {
  const int lane = threadIdx.x & 31;
  float v[NL];
  if (pat == 1) {
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < NL; ++i) {
      const int c = lane + 32 * i;
      float val = -INFINITY;
      if (c <= r) val = zrow[c];
      v[i] = val;
      mx = fmaxf(mx, val);
    }
    mx = redux_max_f32(mx);
#pragma unroll
    for (int i = 0; i < NL; ++i) v[i] = (lane + 32 * i <= r) ? ex2((v[i] - mx) * kLog2e) : 0.f;
  } else {
    const float *vh = vhat + (size_t)h * n, *sh = shat + (size_t)h * n;
#pragma unroll
    for (int i = 0; i < NL; ++i) {
      const int c = lane + 32 * i;
      float val = 0.f;
      if (c <= r) val = vh[c] + sh[r - c];
      v[i] = val;
    }
  }
  float zs = 0.f;
#pragma unroll
  for (int i = 0; i < NL; ++i) zs += v[i];
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) zs += __shfl_xor_sync(0xffffffffu, zs, s);
  const float inv_zs = __frcp_rn(zs);
#pragma unroll
  for (int i = 0; i < NL; ++i) v[i] = v[i] * inv_zs;
  // diagonal score w_r from lane r % 32, slot r / 32; then that slot is zeroed
  float wr_l = 0.f;
#pragma unroll
  for (int i = 0; i < NL; ++i)
    if (i == (r >> 5)) wr_l = v[i];
  const float wr = __shfl_sync(0xffffffffu, wr_l, r & 31);
#pragma unroll
  for (int i = 0; i < NL; ++i)
    if (lane + 32 * i == r) v[i] = 0.f;
  const float need = gamma - wr;
  // lane sum of the slots with key >= t (four chains, fixed order), in fixed point
  auto lane_sum_fx = [&](uint32_t t, uint32_t &cnt) -> uint32_t {
    float f4[4] = {0.f, 0.f, 0.f, 0.f};
    uint32_t c4[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int i = 0; i < NL; ++i) {
      const bool ge = __float_as_uint(v[i]) >= t;
      f4[i & 3] += ge ? v[i] : 0.f;
      c4[i & 3] += ge ? 1u : 0u;
    }
    cnt = (c4[0] + c4[1]) + (c4[2] + c4[3]);
    return __float2uint_rn(((f4[0] + f4[1]) + (f4[2] + f4[3])) * kCutFx);
  };
  int mode;  // 0 = all, 1 = diagonal only, 2 = cut at T
  uint32_t T = 0, need_fx = 0, s_gt = 0;
  if (gamma >= 1.f) {
    mode = 0;
  } else if (need <= 0.f) {
    mode = 1;
  } else {
    need_fx = __float2uint_ru(need * kCutFx);
    uint32_t cnt;
    const uint32_t tot = redux_add_u32(lane_sum_fx(1u, cnt));  // every candidate with w > 0
    if (tot < need_fx) {
      mode = 0;
    } else {
      mode = 2;
      // bracket: f(lo) >= need > f(hi); c_lo / c_hi count candidates with key >= lo / >= hi
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
        const uint32_t fl = lane_sum_fx(mid, cm);
        const uint32_t f = redux_add_u32(fl), cs = redux_add_u32(cm);
        if (f >= need_fx) {
          lo = mid;
          c_lo = cs;
        } else {
          hi = mid;
          c_hi = cs;
          f_hi = f;
        }
      }
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
      s_gt = f_hi;  // every candidate above T has key >= hi
    }
  }
  // Ties at T are taken in index order while the kept sum is below the
  // target: the count taken is the smallest k with s_gt + k t_fx >= need
  // (all of them if the target is not reached, or if T is below the fixed
  // point's resolution).  A tie's rank is its position among the ties in
  // index order (slot-major, then lane).
  uint32_t take_ties = 0u;
  if (mode == 2 && s_gt < need_fx) {
    const uint32_t t_fx = __float2uint_rn(__uint_as_float(T) * kCutFx);
    take_ties = t_fx ? (need_fx - s_gt + t_fx - 1u) / t_fx : 0xFFFFFFFFu;
  }
  const uint32_t lt_mask = (1u << lane) - 1u;
  int written = 0;
  uint32_t ties_before = 0u;
#pragma unroll
  for (int i = 0; i < NL; ++i) {
    const int c = lane + 32 * i;
    const uint32_t key = __float_as_uint(v[i]);
    const bool is_tie = mode == 2 && c < r && key == T;
    const uint32_t tm = __ballot_sync(0xffffffffu, is_tie);
    const bool keep = c <= r && (mode == 0 || c == r || (mode == 2 && key > T) ||
                                 (is_tie && ties_before + __popc(tm & lt_mask) < take_ties));
    ties_before += __popc(tm);
    const uint32_t km = __ballot_sync(0xffffffffu, keep);
    if (keep) out[written + __popc(km & lt_mask)] = c;
    written += __popc(km);
  }
  if (lane == 0) *count_out = written;
}

__global__ void __launch_bounds__(256)
    k_cut(const int *__restrict__ pattern, const float *__restrict__ vhat, const float *__restrict__ shat,
          const float *__restrict__ z, int Hq, int n, float gamma, int *__restrict__ counts,
          int *__restrict__ cols) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= Hq * n) return;
  const int r = n - 1 - row / Hq, h = row % Hq;  // longest rows first
  const size_t tri = (size_t)n * (n + 1) / 2, off = (size_t)h * tri + (size_t)r * (r + 1) / 2;
  const int pat = pattern[h];
  const float *zrow = z + off;
  int *out = cols + off, *cnt = counts + (size_t)h * n + r;
  const int nl = (r >> 5) + 1;  // elements per lane
  if (nl <= 1) cut_row<1>(pat, h, r, n, vhat, shat, zrow, gamma, out, cnt);
  else if (nl <= 2) cut_row<2>(pat, h, r, n, vhat, shat, zrow, gamma, out, cnt);
  else if (nl <= 4) cut_row<4>(pat, h, r, n, vhat, shat, zrow, gamma, out, cnt);
  else if (nl <= 8) cut_row<8>(pat, h, r, n, vhat, shat, zrow, gamma, out, cnt);
  else if (nl <= 16) cut_row<16>(pat, h, r, n, vhat, shat, zrow, gamma, out, cnt);
  else cut_row<32>(pat, h, r, n, vhat, shat, zrow, gamma, out, cnt);
}

}  // namespace fpk

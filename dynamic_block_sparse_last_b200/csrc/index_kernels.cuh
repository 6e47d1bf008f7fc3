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
//                  KV group through a TMA ring; per (row, chunk) max and the
//                  two offset-half sums; per-chunk K column sums.  Nothing of
//                  size S x b reaches global memory.
//   k_row_stats    per (head, row, chunk range): running max / sum.
//   k_block_mass   per (head, chunk): row-normalised lo/hi masses.
//   k_kbar         block means of K.
//   k_pattern      per head: vhat, shat, P_est, JSD, pattern.
//   k_qbar         block means of Q for query-aware heads only.
//   k_qa_logits    q-bar . k-bar logits of query-aware heads (tiled fp32).
//   k_cut          per (head, query block): scores, gamma cut, sorted list.
#pragma once

#include "ptx.cuh"

namespace fpk {

constexpr float kLog2e = 1.4426950408889634f;

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
  static constexpr int kStages = I8 ? 4 : 3;
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
        bool ok = true;
        float m = -INFINITY;
        float lo4[4] = {0.f, 0.f, 0.f, 0.f}, hi4[4] = {0.f, 0.f, 0.f, 0.f};
        for (int u = 0; u < U && ok; ++u) {
          const int ch = ch0 + u;
          // One pass over the chunk in 32-column pieces with an online max:
          // lo/hi are kept relative to the running max m and rescaled when a
          // piece raises it.  Columns t <= i (block-relative) go to lo, the
          // rest to hi; in the last block columns t > i are causally masked.
          // With b = 64 each 64-column half is a block of its own and gets
          // its own (max, lo, hi) part; otherwise the chunk is one part.
          for (int hf = 0; hf < 2; ++hf) {
            if (hf == 0 || P.nsub == 2) {
              m = -INFINITY;
#pragma unroll
              for (int w4 = 0; w4 < 4; ++w4) lo4[w4] = hi4[w4] = 0.f;
            }
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
              const bool last_block = blk == P.n - 1;
              const int t0 = key0 - blk * P.b;                // block-relative column of the piece
              const int dlt = i - t0;  // columns e <= dlt are on the lo side
              float pm4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                const float s = I8 ? (float)(int)r[e] : __uint_as_float(r[e]);
                const bool valid = !last_block || (e <= dlt);
                pm4[e & 3] = valid ? fmaxf(pm4[e & 3], s) : pm4[e & 3];
              }
              const float pmx = fmaxf(fmaxf(pm4[0], pm4[1]), fmaxf(pm4[2], pm4[3]));
              if (pmx == -INFINITY) continue;  // whole piece masked
              if (pmx > m) {
                const float f = (m == -INFINITY) ? 0.f : ex2((m - pmx) * scale2);
#pragma unroll
                for (int w4 = 0; w4 < 4; ++w4) {
                  lo4[w4] *= f;
                  hi4[w4] *= f;
                }
                m = pmx;
              }
              const float m2p = m * scale2;
              if (dlt >= 31) {
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                  const float s = I8 ? (float)(int)r[e] : __uint_as_float(r[e]);
                  lo4[e & 3] += ex2(fmaf(s, scale2, -m2p));
                }
              } else if (dlt < 0) {
                if (!last_block) {
#pragma unroll
                  for (int e = 0; e < 32; ++e) {
                    const float s = I8 ? (float)(int)r[e] : __uint_as_float(r[e]);
                    hi4[e & 3] += ex2(fmaf(s, scale2, -m2p));
                  }
                }
              } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                  const float s = I8 ? (float)(int)r[e] : __uint_as_float(r[e]);
                  const float p = ex2(fmaf(s, scale2, -m2p));
                  if (e <= dlt) lo4[e & 3] += p;
                  else if (!last_block) hi4[e & 3] += p;
                }
              }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&bar_sfree[t][hf]));
            if ((hf == 1 || P.nsub == 2) && i < P.nlast) {
              const float m2 = m * scale2;
              const float lo = (lo4[0] + lo4[1]) + (lo4[2] + lo4[3]);
              const float hi = (hi4[0] + hi4[1]) + (hi4[2] + hi4[3]);
              const int part = ch * P.nsub + (P.nsub == 2 ? hf : 0);
              const size_t o = ((size_t)hh * P.nch * P.nsub + part) * P.b + i;
              P.pm[o] = m2;
              P.plo[o] = lo;
              P.phi[o] = hi;
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
// k_row_stats: grid (Hq, R2), block b threads.  Row i's running max M and
// sum L = sum_chunks (lo + hi) 2^(m - M) over the CTA's chunk range; rows at
// or past nlast (absent from a partial last block) get M = -inf, L = 0.
// ---------------------------------------------------------------------------
__global__ void k_row_stats(const float *__restrict__ pm, const float *__restrict__ plo,
                            const float *__restrict__ phi, int nch, int b, int nlast, int chunks_per_part,
                            float *__restrict__ partM, float *__restrict__ partL) {
  const int h = blockIdx.x, part = blockIdx.y, R2 = gridDim.y, i = threadIdx.x;
  const int c0 = part * chunks_per_part, c1 = i < nlast ? min(nch, c0 + chunks_per_part) : c0;
  float M = -INFINITY, L = 0.f;
  for (int ch = c0; ch < c1; ch += 4) {
    // four chunks' loads in flight, then the running combine in order
    float mv[4], sv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const size_t o = ((size_t)h * nch + ch + u) * b + i;
      const bool in = ch + u < c1;
      mv[u] = in ? pm[o] : -INFINITY;
      sv[u] = in ? plo[o] + phi[o] : 0.f;
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
  partM[((size_t)h * R2 + part) * b + i] = M;
  partL[((size_t)h * R2 + part) * b + i] = L;
}

// ---------------------------------------------------------------------------
// k_block_mass: grid (Hq, R2), block b threads.  Combines the R2 partial row
// statistics, then for every chunk of the CTA's range sums over rows
//   LOc[ch] = sum_i lo_i 2^(m_i - M_i) / L_i,  HIc[ch] likewise,
// in a fixed order (per-warp shuffle tree, then warps in index order).
// ---------------------------------------------------------------------------
__global__ void k_block_mass(const float *__restrict__ pm, const float *__restrict__ plo,
                             const float *__restrict__ phi, const float *__restrict__ partM,
                             const float *__restrict__ partL, int nch, int b, int nlast,
                             int chunks_per_part, float *__restrict__ LOc, float *__restrict__ HIc) {
  extern __shared__ float red[];  // [nwarps][chunks_per_part][2]
  const int h = blockIdx.x, part = blockIdx.y, R2 = gridDim.y, i = threadIdx.x;
  const int warp = i >> 5, lane = i & 31, nw = blockDim.x >> 5;
  float M = -INFINITY;
  for (int r = 0; r < R2; ++r) M = fmaxf(M, partM[((size_t)h * R2 + r) * b + i]);
  float L = 0.f;
  for (int r = 0; r < R2; ++r) {
    const float m = partM[((size_t)h * R2 + r) * b + i];
    if (m != -INFINITY) L += partL[((size_t)h * R2 + r) * b + i] * ex2(m - M);
  }
  const float invL = 1.f / L;
  const int c0 = part * chunks_per_part, c1 = min(nch, c0 + chunks_per_part);
  for (int ch = c0; ch < c1; ch += 4) {
    float a[4], c[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const size_t o = ((size_t)h * nch + ch + u) * b + i;
      const bool in = i < nlast && ch + u < c1;  // rows past nlast hold no partials
      const float m = in ? pm[o] : -INFINITY;
      const float w = (m == -INFINITY) ? 0.f : ex2(m - M) * invL;
      a[u] = in ? plo[o] * w : 0.f;
      c[u] = in ? phi[o] * w : 0.f;
    }
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        a[u] += __shfl_xor_sync(0xffffffffu, a[u], s);
        c[u] += __shfl_xor_sync(0xffffffffu, c[u], s);
      }
    }
    if (lane == 0) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (ch + u < c1) {
          red[(warp * chunks_per_part + (ch + u - c0)) * 2 + 0] = a[u];
          red[(warp * chunks_per_part + (ch + u - c0)) * 2 + 1] = c[u];
        }
      }
    }
  }
  __syncthreads();
  for (int ch = c0 + i; ch < c1; ch += blockDim.x) {
    float a = 0.f, c = 0.f;
    for (int w = 0; w < nw; ++w) {
      a += red[(w * chunks_per_part + (ch - c0)) * 2 + 0];
      c += red[(w * chunks_per_part + (ch - c0)) * 2 + 1];
    }
    LOc[(size_t)h * nch + ch] = a;
    HIc[(size_t)h * nch + ch] = c;
  }
}

// ---------------------------------------------------------------------------
// k_kbar: grid (n, Hkv), block 128: kbar[kvh][c][t] = mean of the K rows of
// block c (b rows, or S - (n-1)b for a partial last block); for int8 keys the
// exact integer sum times k_scale[kvh].
// ---------------------------------------------------------------------------
__global__ void k_kbar(const float *__restrict__ ksum, const float *__restrict__ k_scale, int S, int nch,
                       int b, int n, float *__restrict__ kbar) {
  const int c = blockIdx.x, kvh = blockIdx.y, t = threadIdx.x;
  const int per = b >= 128 ? b / 128 : 1, rows = min(b, S - c * b);  // column parts per block
  float s = 0.f;
  for (int k = 0; k < per && c * per + k < nch; ++k) s += ksum[((size_t)kvh * nch + c * per + k) * 128 + t];
  if (k_scale) s *= k_scale[kvh];
  kbar[((size_t)kvh * n + c) * 128 + t] = s / (float)rows;
}

// ---------------------------------------------------------------------------
// k_pattern: grid (Hq), block 1024.  With nlast = S - (n-1)b rows in the
// last block: vhat[c] = (LO[c] + HI[c]) / nlast, shat[o] = (LO[n-1-o] +
// HI[n-2-o]) / nlast, P_est = softmax_c(qbar_last . kbar_c / sqrt(d)) with
// qbar_last the mean of those nlast rows, JSD(vhat, P_est) (natural log),
// pattern = QA iff JSD < tau.
// ---------------------------------------------------------------------------
template <bool I8>
__global__ void __launch_bounds__(1024)
    k_pattern(const void *__restrict__ q, const float *__restrict__ q_scale,
              const float *__restrict__ LOc, const float *__restrict__ HIc,
              const float *__restrict__ kbar, int S, int ld, int g, int b, int n, int nch, float inv_sqrt_d,
              float tau, float *__restrict__ vhat, float *__restrict__ shat,
              float *__restrict__ pest, float *__restrict__ jsd, int *__restrict__ pattern) {
  __shared__ float qb[128];
  __shared__ float part[1024 / 32];
  __shared__ float lo_s[1024], hi_s[1024];
  const int h = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int kvh = h / g, per = b >= 128 ? b / 128 : 1, nlast = S - (n - 1) * b;  // parts per block
  // block masses
  for (int c = tid; c < n; c += blockDim.x) {
    float a = 0.f, e = 0.f;
    for (int k = 0; k < per && c * per + k < nch; ++k) {
      a += LOc[(size_t)h * nch + c * per + k];
      e += HIc[(size_t)h * nch + c * per + k];
    }
    lo_s[c] = a / (float)nlast;
    hi_s[c] = e / (float)nlast;
  }
  // mean of the last block's query rows
  if (tid < 128) {
    const size_t base = ((size_t)h * ld + (size_t)(n - 1) * b) * 128 + tid;
    if (I8) {
      const int8_t *q8 = reinterpret_cast<const int8_t *>(q);
      int acc = 0;
      for (int r = 0; r < nlast; ++r) acc += q8[base + (size_t)r * 128];
      qb[tid] = (float)acc * q_scale[h] / (float)nlast;
    } else {
      const __nv_bfloat16 *qh = reinterpret_cast<const __nv_bfloat16 *>(q);
      float acc = 0.f;
      for (int r = 0; r < nlast; ++r) acc += __bfloat162float(qh[base + (size_t)r * 128]);
      qb[tid] = acc / (float)nlast;
    }
  }
  __syncthreads();
  for (int c = tid; c < n; c += blockDim.x) {
    vhat[(size_t)h * n + c] = lo_s[c] + hi_s[c];
    const int o = c;
    shat[(size_t)h * n + o] = lo_s[n - 1 - o] + (o <= n - 2 ? hi_s[n - 2 - o] : 0.f);
  }
  // logits of P_est, one warp per block c
  float *z = lo_s;  // reuse after vhat/shat are written
  __syncthreads();
  for (int c = warp; c < n; c += blockDim.x / 32) {
    const float *kr = kbar + ((size_t)kvh * n + c) * 128;
    float a = 0.f;
#pragma unroll
    for (int t = 0; t < 4; ++t) a = fmaf(qb[lane + 32 * t], kr[lane + 32 * t], a);
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) a += __shfl_xor_sync(0xffffffffu, a, s);
    if (lane == 0) z[c] = a * inv_sqrt_d;
  }
  __syncthreads();
  float mx = -INFINITY;
  for (int c = tid; c < n; c += blockDim.x) mx = fmaxf(mx, z[c]);
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, s));
  if (lane == 0) part[warp] = mx;
  __syncthreads();
  mx = part[0];
  for (int w = 1; w < (int)(blockDim.x / 32); ++w) mx = fmaxf(mx, part[w]);
  __syncthreads();
  float sum = 0.f;
  for (int c = tid; c < n; c += blockDim.x) {
    const float e = expf(z[c] - mx);
    hi_s[c] = e;
    sum += e;
  }
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, s);
  if (lane == 0) part[warp] = sum;
  __syncthreads();
  sum = 0.f;
  for (int w = 0; w < (int)(blockDim.x / 32); ++w) sum += part[w];
  __syncthreads();
  float js = 0.f;
  for (int c = tid; c < n; c += blockDim.x) {
    const float pe = hi_s[c] / sum;
    pest[(size_t)h * n + c] = pe;
    const float pv = vhat[(size_t)h * n + c];
    const float m = 0.5f * (pv + pe);
    if (pv > 0.f) js += 0.5f * pv * logf(pv / m);
    if (pe > 0.f) js += 0.5f * pe * logf(pe / m);
  }
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) js += __shfl_xor_sync(0xffffffffu, js, s);
  if (lane == 0) part[warp] = js;
  __syncthreads();
  if (tid == 0) {
    float tot = 0.f;
    for (int w = 0; w < (int)(blockDim.x / 32); ++w) tot += part[w];
    jsd[h] = tot;
    pattern[h] = (tot < tau) ? 1 : 0;
  }
}

// ---------------------------------------------------------------------------
// k_qbar: grid (n, Hq), block 256: qbar[h][r][t] = mean of the Q rows of
// block r (b rows, or S - (n-1)b for a partial last block), only for heads
// whose pattern is query-aware (others exit).
// ---------------------------------------------------------------------------
template <bool I8>
__global__ void __launch_bounds__(256)
    k_qbar(const void *__restrict__ q, const float *__restrict__ q_scale,
           const int *__restrict__ pattern, int S, int ld, int b, int n, float *__restrict__ qbar) {
  const int r = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
  if (pattern[h] != 1) return;
  __shared__ float red[16][128];
  const size_t row0 = (size_t)h * ld + (size_t)r * b;
  const int rows = min(b, S - r * b);
  if (I8) {
    // 8 threads per 128-byte row, 32 rows per pass; thread owns 16 columns
    const int8_t *q8 = reinterpret_cast<const int8_t *>(q);
    const int c16 = tid & 7, rr = tid >> 3;
    int acc[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) acc[e] = 0;
    for (int p = rr; p < rows; p += 32) {
      const int4 v = *reinterpret_cast<const int4 *>(q8 + (row0 + p) * 128 + c16 * 16);
      const int w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 16; ++e) acc[e] += (int)(int8_t)((w[e >> 2] >> (8 * (e & 3))) & 0xff);
    }
    // reduce over rr (32 groups) via shuffles within the 4 groups of a warp then smem
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      int a = acc[e];
      a += __shfl_xor_sync(0xffffffffu, a, 8);
      a += __shfl_xor_sync(0xffffffffu, a, 16);
      acc[e] = a;
    }
    const int warp = tid >> 5, lane = tid & 31;
    if (lane < 8) {
#pragma unroll
      for (int e = 0; e < 16; ++e) red[warp][lane * 16 + e] = (float)acc[e];
    }
    __syncthreads();
    if (tid < 128) {
      float s = 0.f;
      for (int w = 0; w < 8; ++w) s += red[w][tid];
      qbar[((size_t)h * n + r) * 128 + tid] = s * q_scale[h] / (float)rows;
    }
  } else {
    // 16 threads per 256-byte row, 16 rows per pass; thread owns 8 columns
    const __nv_bfloat16 *qh = reinterpret_cast<const __nv_bfloat16 *>(q);
    const int c8 = tid & 15, rr = tid >> 4;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll 4
    for (int p = rr; p < rows; p += 16) {
      const uint4 v = *reinterpret_cast<const uint4 *>(qh + (row0 + p) * 128 + c8 * 8);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[e]));
        acc[2 * e] += f.x;
        acc[2 * e + 1] += f.y;
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 16);
    const int warp = tid >> 5, lane = tid & 31;
    if (lane < 16) {
#pragma unroll
      for (int e = 0; e < 8; ++e) red[warp][lane * 8 + e] = acc[e];
    }
    __syncthreads();
    if (tid < 128) {
      float s = 0.f;
      for (int w = 0; w < 8; ++w) s += red[w][tid];
      qbar[((size_t)h * n + r) * 128 + tid] = s / (float)rows;
    }
  }
}

// ---------------------------------------------------------------------------
// k_qa_logits: grid (nt(nt+1)/2, Hq) with nt = ceil(n/64), block 256.  For
// query-aware heads only (others exit): the lower triangle of
// Z = qbar kbar^T / sqrt(d), z[h][r][c] for c <= r, in the padded triangular
// layout (row r at h*n(n+1)/2 + r(r+1)/2).  Tiled fp32 product: 64 x 64
// output tile per CTA, 4 x 4 outputs per thread, d staged through shared
// memory 32 at a time.
// ---------------------------------------------------------------------------
constexpr int kLgTile = 64;
constexpr int kLgK = 32;
constexpr int kLgStride = kLgTile + 4;  // float4-aligned rows

__global__ void __launch_bounds__(256)
    k_qa_logits(const int *__restrict__ pattern, const float *__restrict__ qbar,
                const float *__restrict__ kbar, int g, int n, float inv_sqrt_d, float *__restrict__ z) {
  const int h = blockIdx.y;
  if (pattern[h] != 1) return;
  __shared__ __align__(16) float As[kLgK][kLgStride];  // [k][row]
  __shared__ __align__(16) float Bs[kLgK][kLgStride];  // [k][col]
  // lower-triangular tile (tr, tc), tc <= tr, from the linear index
  const int x = blockIdx.x;
  int tr = (int)((sqrtf(8.f * (float)x + 1.f) - 1.f) * 0.5f);
  while ((tr + 1) * (tr + 2) / 2 <= x) ++tr;
  while (tr * (tr + 1) / 2 > x) --tr;
  const int tc = x - tr * (tr + 1) / 2;
  const int kvh = h / g;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int row0 = tr * kLgTile, col0 = tc * kLgTile;
  const float *qh = qbar + (size_t)h * n * 128;
  const float *kh = kbar + (size_t)kvh * n * 128;
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b2 = 0; b2 < 4; ++b2) acc[a][b2] = 0.f;
  for (int k0 = 0; k0 < 128; k0 += kLgK) {
    __syncthreads();
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int f = tid + u * 256, rr = f >> 3, k4 = (f & 7) * 4;
      const float4 qa = (row0 + rr < n) ? *reinterpret_cast<const float4 *>(qh + (size_t)(row0 + rr) * 128 + k0 + k4)
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
      const float4 kb = (col0 + rr < n) ? *reinterpret_cast<const float4 *>(kh + (size_t)(col0 + rr) * 128 + k0 + k4)
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
      As[k4 + 0][rr] = qa.x; As[k4 + 1][rr] = qa.y; As[k4 + 2][rr] = qa.z; As[k4 + 3][rr] = qa.w;
      Bs[k4 + 0][rr] = kb.x; Bs[k4 + 1][rr] = kb.y; Bs[k4 + 2][rr] = kb.z; Bs[k4 + 3][rr] = kb.w;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < kLgK; ++k) {
      const float4 a4 = *reinterpret_cast<const float4 *>(&As[k][ty * 4]);
      const float4 b4 = *reinterpret_cast<const float4 *>(&Bs[k][tx * 4]);
      const float av[4] = {a4.x, a4.y, a4.z, a4.w}, bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b2 = 0; b2 < 4; ++b2) acc[a][b2] = fmaf(av[a], bv[b2], acc[a][b2]);
    }
  }
  float *zh = z + (size_t)h * ((size_t)n * (n + 1) / 2);
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int r = row0 + ty * 4 + a;
    if (r >= n) continue;
#pragma unroll
    for (int b2 = 0; b2 < 4; ++b2) {
      const int c = col0 + tx * 4 + b2;
      if (c <= r) zh[(size_t)r * (r + 1) / 2 + c] = acc[a][b2] * inv_sqrt_d;
    }
  }
}

// ---------------------------------------------------------------------------
// k_cut: one warp per (head, query block r), heavy rows first; block 256.
// Scores over c <= r:  VS: w_c = vhat[c] + shat[r - c];  QA: w_c = exp(z_c -
// max); normalised to sum 1.  The diagonal is kept; the others are kept in
// order of descending score (ties: lower index) while the kept sum is below
// gamma.  The cut is found by bisection on the fp32 bit pattern of the
// scores (monotone for positive floats): T = largest t with
// sum_{c < r, bits(w_c) >= t} w_c >= gamma - w_r, stopping as soon as one
// candidate is left between the bounds; everything above T is kept, then
// ties at T by ascending index until the target is reached.  The row lives
// in registers (element c in lane c % 32, slot c / 32).
// Output: counts[h*n + r], ascending list at cols[h*n(n+1)/2 + r(r+1)/2].
// ---------------------------------------------------------------------------
constexpr int kSelMaxN = 1024;

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
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, s));
#pragma unroll
    for (int i = 0; i < NL; ++i) v[i] = (lane + 32 * i <= r) ? expf(v[i] - mx) : 0.f;
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
#pragma unroll
  for (int i = 0; i < NL; ++i) v[i] = v[i] / zs;
  // diagonal score w_r from lane r % 32, slot r / 32
  float wr_l = 0.f;
#pragma unroll
  for (int i = 0; i < NL; ++i)
    if (i == (r >> 5)) wr_l = v[i];
  const float wr = __shfl_sync(0xffffffffu, wr_l, r & 31);
  const float need = gamma - wr;
  // candidates: c < r (slot value 0 and bits 0 elsewhere never qualify)
  int mode;  // 0 = all, 1 = diagonal only, 2 = cut at T
  uint32_t T = 0;
  float s_gt = 0.f;
  if (gamma >= 1.f) {
    mode = 0;
  } else if (need <= 0.f) {
    mode = 1;
  } else {
    float tot = 0.f;
#pragma unroll
    for (int i = 0; i < NL; ++i) tot += (lane + 32 * i < r) ? v[i] : 0.f;
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, s);
    if (tot < need) {
      mode = 0;
    } else {
      mode = 2;
      // invariant: f(lo) >= need > f(hi); c_lo / c_hi count candidates with
      // bits >= lo / >= hi; f_hi = f(hi)
      uint32_t lo = 0u, hi = 0x7F800000u;
      int c_lo = r, c_hi = 0;
      float f_hi = 0.f;
      while (hi - lo > 1u && c_lo - c_hi > 1) {
        const uint32_t mid = lo + ((hi - lo) >> 1);
        // four independent accumulation chains
        float f4[4] = {0.f, 0.f, 0.f, 0.f};
        int c4[4] = {0, 0, 0, 0};
#pragma unroll
        for (int i = 0; i < NL; ++i) {
          const bool ge = (lane + 32 * i < r) && __float_as_uint(v[i]) >= mid;
          f4[i & 3] += ge ? v[i] : 0.f;
          c4[i & 3] += ge ? 1 : 0;
        }
        float f = (f4[0] + f4[1]) + (f4[2] + f4[3]);
        int cnt = (c4[0] + c4[1]) + (c4[2] + c4[3]);
#pragma unroll
        for (int s = 16; s > 0; s >>= 1) {
          f += __shfl_xor_sync(0xffffffffu, f, s);
          cnt += __shfl_xor_sync(0xffffffffu, cnt, s);
        }
        if (f >= need) {
          lo = mid;
          c_lo = cnt;
        } else {
          hi = mid;
          c_hi = cnt;
          f_hi = f;
        }
      }
      if (c_lo - c_hi == 1) {
        uint32_t tb = 0u;
#pragma unroll
        for (int i = 0; i < NL; ++i) {
          const uint32_t bits = __float_as_uint(v[i]);
          if (lane + 32 * i < r && bits >= lo && bits < hi) tb = bits;
        }
#pragma unroll
        for (int s = 16; s > 0; s >>= 1) tb = max(tb, __shfl_xor_sync(0xffffffffu, tb, s));
        T = tb;
      } else {
        T = lo;
      }
      s_gt = f_hi;  // every candidate above T has bits >= hi
    }
  }
  // emit ascending; ties at T in index order until the target is reached
  int written = 0;
  float tie_acc = s_gt;
  const float tval = __uint_as_float(T);
  bool ties_done = false;
#pragma unroll
  for (int i = 0; i < NL; ++i) {
    const int c = lane + 32 * i;
    bool keep = false, is_tie = false;
    if (c <= r) {
      if (mode == 0 || c == r) keep = true;
      else if (mode == 2) {
        const uint32_t bits = __float_as_uint(v[i]);
        keep = bits > T;
        is_tie = (bits == T);
      }
    }
    if (mode == 2) {
      uint32_t tmask = __ballot_sync(0xffffffffu, is_tie);
      uint32_t take = 0u;
      while (tmask && !ties_done) {
        if (tie_acc >= need) {
          ties_done = true;
          break;
        }
        take |= 1u << (__ffs(tmask) - 1);
        tie_acc += tval;
        tmask &= tmask - 1u;
      }
      if (take & (1u << lane)) keep = true;
    }
    const uint32_t km = __ballot_sync(0xffffffffu, keep);
    if (keep) out[written + __popc(km & ((1u << lane) - 1u))] = c;
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

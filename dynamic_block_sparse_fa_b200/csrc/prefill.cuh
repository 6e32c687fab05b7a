// prefill.cuh -- BLASST prefill forward on sm_100a: TMA-staged Q/K/V tiles,
// tcgen05 MMAs accumulating S = Q K^T and O += P V in tensor memory, a
// per-row max read back from tensor memory and a per-tile skip vote.  A
// skipped (tile, block) pair issues neither its V TMA load nor its P.V MMA,
// and computes no exp.
//
// Method: "BLASST: Dynamic BLocked Attention Sparsity via Softmax
// Thresholding" (gist.science summary, section 2 "Criterio de Pulo",
// "Acoes de Otimizacao"; MLSys'26 reading notes, "core method": each block
// updates the running max and, if m~ - m < ln(lambda), skips exp, V load and
// P.V MMA; "design trade-offs": the decision is per block).  The Hindi
// summary (section 2, kernel optimisation) says the prefill kernel there
// still loaded V to keep memory access predictable; this kernel does not
// load V for skipped blocks: the load is issued after the vote and overlaps
// the exp of the same block.
//
// CTA = 6 warps, one 128-row query tile (M = 128 tcgen05 MMA):
//   warp 0       TMA producer: Q once, K ring ahead, V on demand per kept
//                block (after reading the block's decision)
//   warp 1       MMA issuer (one thread): S_j = Q K_j^T into one of two TMEM
//                score buffers; P_j V_j into the TMEM output accumulator
//   warps 2..5   softmax: one thread per row; tcgen05.ld of the score row,
//                causal/ragged masking, row max, tile vote by barrier
//                AND-reduction, exp, bf16 P written back over the scores,
//                lazy O rescaling, epilogue
// Tensor memory columns: [S0 | S1 | O], P_j aliases the first Bc/2 columns
// of its score buffer (two bf16 per 32-bit column).
//
// Tiles with Br = 64 still run an M = 128 MMA: rows 64..127 belong to the
// next tile and are ignored (they neither vote nor get stored).
#pragma once

#include <cuda.h>

#include "ptx.cuh"

namespace blasst {

struct PrefillProblem {
  const void *q, *k, *v;
  void* o;
  float* lse;
  int B, Hq, Hkv, Lq, Lkv, d;
  float scale;
  int causal;
  float ln_lambda;
  int Br, Bc;
  unsigned long long* counters;
  unsigned char* mask;
  float* margin;  // decision margins, layout of mask (may be null)
  int window;  // 0 = none
};

struct __align__(64) PrefillParams {
  CUtensorMap tq, tk, tv;
  __nv_bfloat16* o;
  float* lse;
  unsigned long long* counters;
  unsigned char* mask;
  float* margin;
  int B, Hq, Hkv, Lq, Lkv, nq, nk, G;
  float scale, ln_lambda;
  int causal, stats_only;
  // causal sliding window: row r sees keys [diag_r - window + 1, diag_r]
  // (0 = no window; 128x128 tiles only)
  int window;
};

template <int D, int BN, int BRL>
struct PrefillCfg {
  static constexpr int BM = 128;  // MMA rows
  static constexpr int NKS = (D == 128 && BN == 128) ? 3 : 4;
  static constexpr int NVS = 2;
  static constexpr int R = 8;     // decision ring (> NKS)
  static_assert(R > NKS, "decision ring must exceed the K prefetch depth");
  static constexpr int BOX_Q = BM * 128;  // bytes of one 64-column box
  static constexpr int BOX_K = BN * 128;
  static constexpr int QBYTES = BM * D * 2;
  static constexpr int KBYTES = BN * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QBYTES;
  static constexpr int OFF_V = OFF_K + NKS * KBYTES;
  static constexpr int OFF_BAR = OFF_V + NVS * KBYTES;
  // barrier indices
  static constexpr int B_Q = 0;
  static constexpr int B_KF = 1;
  static constexpr int B_KE = B_KF + NKS;
  static constexpr int B_VF = B_KE + NKS;
  static constexpr int B_VE = B_VF + NVS;
  static constexpr int B_SF = B_VE + NVS;
  static constexpr int B_PF = B_SF + 2;
  static constexpr int B_DEC = B_PF + 2;
  static constexpr int B_OD = B_DEC + R;
  static constexpr int NBAR = B_OD + 1;
  static constexpr int OFF_DEC = OFF_BAR + NBAR * 8;
  static constexpr int OFF_TMEM = OFF_DEC + R * 4;
  static constexpr int OFF_XM = OFF_TMEM + 16;  // f32 [2][4]: warp margin maxima
  static constexpr int SMEM = OFF_XM + 32;
  static constexpr int SMEM_ALLOC = SMEM + 1024;  // slack for 1024 alignment
  static constexpr int TMEM_COLS = (2 * BN + D <= 256) ? 256 : 512;
  static constexpr int COL_S = 0;  // buffer b at COL_S + b * BN
  static constexpr int COL_O = 2 * BN;
  static constexpr int THREADS = 192;
};

constexpr float kPrefLog2e = 1.4426950408889634f;
// Lazy rescaling: O and l keep a reference max m_ref that trails the exact
// running max (used by the criterion) by at most kRescaleNats.
constexpr float kRescaleNats = 5.545177444479562f;  // 8 ln 2

template <int D, int BN, int BRL>
__global__ void __launch_bounds__(192, 1)
    prefill_kernel(const __grid_constant__ PrefillParams p) {
  using C = PrefillCfg<D, BN, BRL>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Work item: longest query tiles first over all heads.
  const int BH = p.B * p.Hq;
  const int lin = blockIdx.x;
  const int tile = p.nq - 1 - lin / BH;
  const int bh = lin - (lin / BH) * BH;
  const int b = bh / p.Hq;
  const int hq = bh - b * p.Hq;
  const int hkv = hq / p.G;
  const int row0 = tile * BRL;
  const int last_row = min(row0 + BRL, p.Lq) - 1;
  const int kmax = p.causal ? min(p.Lkv - 1, last_row + (p.Lkv - p.Lq))
                            : p.Lkv - 1;
  const int nblk = kmax / BN + 1;

  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  volatile int* dec_flag = reinterpret_cast<volatile int*>(smem + C::OFF_DEC);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM);

  if (threadIdx.x == 0) {
    mbar_init(&bar[C::B_Q], 1);
    for (int i = 0; i < C::NKS; ++i) {
      mbar_init(&bar[C::B_KF + i], 1);
      mbar_init(&bar[C::B_KE + i], 1);
    }
    for (int i = 0; i < C::NVS; ++i) {
      mbar_init(&bar[C::B_VF + i], 1);
      mbar_init(&bar[C::B_VE + i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar[C::B_SF + i], 1);
      mbar_init(&bar[C::B_PF + i], 4);  // one arrival per softmax warp
    }
    for (int i = 0; i < C::R; ++i) mbar_init(&bar[C::B_DEC + i], 1);
    mbar_init(&bar[C::B_OD], 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool stats_only = p.stats_only != 0;

  // Every role loop below is run by whole warps with warp-uniform control
  // flow; a single elected lane issues TMA / MMA instructions.
  constexpr unsigned FULL = 0xffffffffu;
  const bool leader = (lane == 0);

  if (warp == 0) {
    // ------------------------------------------------------------------
    // TMA producer
    // ------------------------------------------------------------------
    const uint64_t pol_q = policy_evict_first();
    const uint64_t pol_kv = policy_evict_last();
    const int zq = b * p.Hq + hq;
    const int zk = b * p.Hkv + hkv;
    auto issue_k = [&](int j) {
      const int st = j % C::NKS;
      mbar_arrive_expect_tx(&bar[C::B_KF + st], C::KBYTES);
#pragma unroll
      for (int c = 0; c < D / 64; ++c)
        tma_load_3d(sK + st * C::KBYTES + c * C::BOX_K, &p.tk,
                    &bar[C::B_KF + st], c * 64, j * BN, zk, pol_kv);
    };
    if (leader) {
      prefetch_tmap(&p.tq);
      prefetch_tmap(&p.tk);
      prefetch_tmap(&p.tv);
      mbar_arrive_expect_tx(&bar[C::B_Q], C::QBYTES);
#pragma unroll
      for (int c = 0; c < D / 64; ++c)
        tma_load_3d(sQ + c * C::BOX_Q, &p.tq, &bar[C::B_Q], c * 64, row0, zq,
                    pol_q);
      const int n0 = nblk < C::NKS ? nblk : C::NKS;
      for (int j = 0; j < n0; ++j) issue_k(j);
    }
    __syncwarp();
    int kept = 0;
    for (int j = 0; j < nblk; ++j) {
      if (j + C::NKS < nblk) {
        const bool w = mbar_wait(&bar[C::B_KE + j % C::NKS], (j / C::NKS) & 1,
                                 kWaitPrefillLoad, j, j % C::NKS);
        if (!__all_sync(FULL, w)) break;
        if (leader) issue_k(j + C::NKS);
        __syncwarp();
      }
      if (!stats_only) {
        const bool w = mbar_wait(&bar[C::B_DEC + j % C::R], (j / C::R) & 1,
                                 kWaitPrefillLoad, j, 100 + j % C::R);
        if (!__all_sync(FULL, w)) break;
        if (dec_flag[j % C::R]) {
          const int n = kept++;
          const int slot = n % C::NVS;
          if (n >= C::NVS) {
            const bool w2 = mbar_wait(&bar[C::B_VE + slot],
                                      ((n / C::NVS) - 1) & 1, kWaitPrefillLoad,
                                      j, 200 + slot);
            if (!__all_sync(FULL, w2)) break;
          }
          if (leader) {
            mbar_arrive_expect_tx(&bar[C::B_VF + slot], C::KBYTES);
#pragma unroll
            for (int c = 0; c < D / 64; ++c)
              tma_load_3d(sV + slot * C::KBYTES + c * C::BOX_K, &p.tv,
                          &bar[C::B_VF + slot], c * 64, j * BN, zk, pol_kv);
          }
          __syncwarp();
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------
    // MMA issuer
    // ------------------------------------------------------------------
    constexpr uint32_t idesc_s = idesc_bf16(128, BN, 0, 0);
    constexpr uint32_t idesc_o = idesc_bf16(128, D, 0, 1);
    const uint32_t aQ = smem_u32(sQ);
    const uint32_t aK = smem_u32(sK);
    const uint32_t aV = smem_u32(sV);
    bool ok = __all_sync(FULL, mbar_wait(&bar[C::B_Q], 0, kWaitPrefillMma, 0, 0));
    tc_fence_after();
    int kept = 0;
    for (int j = 0; j <= nblk && ok; ++j) {
      if (j < nblk) {
        const int st = j % C::NKS;
        ok = __all_sync(FULL, mbar_wait(&bar[C::B_KF + st], (j / C::NKS) & 1,
                                        kWaitPrefillMma, j, st));
        if (!ok) break;
        tc_fence_after();
        if (leader) {
          const uint32_t d_s = tmem + C::COL_S + (j & 1) * BN;
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t off = (uint32_t)(k & 3) * 32;  // 16 cols = 32 B
            const uint64_t da =
                smem_desc(aQ + (k >> 2) * C::BOX_Q + off, 16, 1024, 2);
            const uint64_t db = smem_desc(
                aK + st * C::KBYTES + (k >> 2) * C::BOX_K + off, 16, 1024, 2);
            mma_ss(d_s, da, db, idesc_s, k > 0 ? 1u : 0u);
          }
          mma_commit(&bar[C::B_SF + (j & 1)]);
          mma_commit(&bar[C::B_KE + st]);
        }
        __syncwarp();
      }
      if (j >= 1) {
        const int jj = j - 1;
        ok = __all_sync(FULL, mbar_wait(&bar[C::B_DEC + jj % C::R],
                                        (jj / C::R) & 1, kWaitPrefillMma, jj,
                                        100 + jj % C::R));
        if (!ok) break;
        if (!stats_only && dec_flag[jj % C::R]) {
          ok = __all_sync(FULL, mbar_wait(&bar[C::B_PF + (jj & 1)],
                                          (jj >> 1) & 1, kWaitPrefillMma, jj,
                                          300 + (jj & 1)));
          if (!ok) break;
          const int n = kept++;
          const int slot = n % C::NVS;
          ok = __all_sync(FULL, mbar_wait(&bar[C::B_VF + slot],
                                          (n / C::NVS) & 1, kWaitPrefillMma,
                                          jj, 200 + slot));
          if (!ok) break;
          tc_fence_after();
          if (leader) {
            const uint32_t a_p = tmem + C::COL_S + (jj & 1) * BN;
#pragma unroll
            for (int k = 0; k < BN / 16; ++k) {
              const uint64_t db = smem_desc(aV + slot * C::KBYTES + k * 2048,
                                            C::BOX_K, 1024, 2);
              mma_ts(tmem + C::COL_O, a_p + k * 8, db, idesc_o,
                     (n > 0 || k > 0) ? 1u : 0u);
            }
            mma_commit(&bar[C::B_VE + slot]);
            mma_commit(&bar[C::B_OD]);
          }
          __syncwarp();
        }
      }
    }
  } else {
    // ------------------------------------------------------------------
    // Softmax warpgroup: thread = query row
    // ------------------------------------------------------------------
    const int quad = warp & 3;  // TMEM lane quadrant this warp may access
    const int rr = quad * 32 + lane;
    const int row_g = row0 + rr;
    const bool active = rr < BRL && row_g < p.Lq;
    const int lim = p.causal ? min(row_g + (p.Lkv - p.Lq), p.Lkv - 1)
                             : p.Lkv - 1;
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    const float scale = p.scale;
    const float ln_lambda = p.ln_lambda;
    const float sl2 = scale * kPrefLog2e;
    const bool elected = (warp == 2 && lane == 0);
    const size_t mask_row =
        ((size_t)(b * p.Hq + hq) * p.nq + tile) * (size_t)p.nk;

    float m_crit = -INFINITY;  // exact running max (scaled units)
    float m_ref = -INFINITY;   // reference max of O and l
    float l = 0.f;
    int kept = 0;
    unsigned long long n_vis = 0, n_skp = 0;
    bool ok = true;

    // A failed bounded wait is voted on (OR over the warpgroup) at the top of
    // the next block, so the warpgroup always leaves the loop together.
    for (int j = 0; j < nblk; ++j) {
      const int buf = j & 1;
      if (ok)
        ok = mbar_wait(&bar[C::B_SF + buf], (j >> 1) & 1, kWaitPrefillSoftmax,
                       j, 400 + buf);
      tc_fence_after();
      if (named_sync_or(1, 128, !ok)) { ok = false; break; }
      uint32_t sr[BN / 32][32];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c)
        tmem_ld32(lane_base + C::COL_S + buf * BN + c * 32, sr[c]);
      tc_wait_ld();

      const int col0 = j * BN;
      if (col0 + BN - 1 > lim) {  // diagonal or ragged block: mask per entry
#pragma unroll
        for (int c = 0; c < BN / 32; ++c)
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            if (col0 + c * 32 + x > lim) sr[c][x] = __float_as_uint(-INFINITY);
          }
      }
      float mt;
      {
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < BN / 32; ++c)
#pragma unroll
          for (int x = 0; x < 32; ++x)
            m4[x & 3] = fmaxf(m4[x & 3], __uint_as_float(sr[c][x]));
        mt = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      }
      const float mt_s = mt * scale;  // -inf stays -inf (scale > 0)
      const bool pred = !active || mt_s == -INFINITY ||
                        (mt_s - m_crit < ln_lambda);
      float* xm = reinterpret_cast<float*>(smem + C::OFF_XM) + (j & 1) * 4;
      if (p.margin) {  // max over the rows of m~ - m, per warp
        float dl = (active && mt_s != -INFINITY) ? mt_s - m_crit : -INFINITY;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1)
          dl = fmaxf(dl, __shfl_xor_sync(0xffffffffu, dl, o));
        if (lane == 0) xm[warp & 3] = dl;
      }
      tc_fence_before();
      const bool skip =
          named_sync_and(1, 128, pred) && (ln_lambda > -INFINITY);
      if (elected) {
        ++n_vis;
        if (skip) ++n_skp;
        if (p.mask) p.mask[mask_row + j] = skip ? 2 : 1;
        if (p.margin)
          p.margin[mask_row + j] =
              fmaxf(fmaxf(xm[0], xm[1]), fmaxf(xm[2], xm[3])) - ln_lambda;
        dec_flag[j % C::R] = skip ? 0 : 1;
        mbar_arrive(&bar[C::B_DEC + j % C::R]);
      }
      if (skip || stats_only) {
        if (!stats_only) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar[C::B_PF + buf]);
        }
        if (active) m_crit = fmaxf(m_crit, mt_s);
        continue;
      }

      // Kept block: exp, P to tensor memory, O rescale if the max grew.
      float alpha = 1.f;
      bool rescale = false;
      if (active && mt_s != -INFINITY) {
        const float m_new = fmaxf(m_crit, mt_s);
        if (m_ref == -INFINITY || m_new > m_ref + kRescaleNats) {
          alpha = (m_ref == -INFINITY) ? 0.f
                                       : ex2_approx((m_ref - m_new) * kPrefLog2e);
          m_ref = m_new;
          rescale = true;
        }
      }
      const float mb = (active && m_ref != -INFINITY) ? m_ref * kPrefLog2e
                                                      : INFINITY;
      float rowsum = 0.f;
      uint32_t pk[BN / 2];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c)
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          const float p0 =
              ex2_approx(fmaf(__uint_as_float(sr[c][x]), sl2, -mb));
          const float p1 =
              ex2_approx(fmaf(__uint_as_float(sr[c][x + 1]), sl2, -mb));
          rowsum += p0 + p1;
          pk[(c * 32 + x) / 2] = pack_bf16x2(p0, p1);
        }
      l = alpha * l + rowsum;
#pragma unroll
      for (int c = 0; c < BN / 64; ++c) {
        uint32_t chunk[32];
#pragma unroll
        for (int x = 0; x < 32; ++x) chunk[x] = pk[c * 32 + x];
        tmem_st32(lane_base + C::COL_S + buf * BN + c * 32, chunk);
      }
      tc_wait_st();
      // Observe the completion of the previous kept block's P.V (the O
      // accumulator may only be touched once it is done).  The rescale is
      // done by whole warps (tcgen05.ld/st are warp-collective); rows that
      // do not rescale multiply by 1.
      if (kept > 0) {
        if (ok)
          ok = mbar_wait(&bar[C::B_OD], (kept - 1) & 1, kWaitPrefillSoftmax, j,
                         500);
        tc_fence_after();
        const bool warp_ok = __all_sync(FULL, ok);
        if (warp_ok && __any_sync(FULL, rescale)) {
          const float f = rescale ? alpha : 1.f;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t orow[32];
            tmem_ld32(lane_base + C::COL_O + c * 32, orow);
            tc_wait_ld();
#pragma unroll
            for (int x = 0; x < 32; ++x)
              orow[x] = __float_as_uint(__uint_as_float(orow[x]) * f);
            tmem_st32(lane_base + C::COL_O + c * 32, orow);
          }
          tc_wait_st();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[C::B_PF + buf]);
      ++kept;
      if (active) m_crit = fmaxf(m_crit, mt_s);
    }
    if (named_sync_or(1, 128, !ok)) ok = false;

    if (ok && elected) {
      if (p.counters) {
        atomicAdd(&p.counters[0], n_vis);
        atomicAdd(&p.counters[1], n_skp);
      }
      if (p.mask)
        for (int j = nblk; j < p.nk; ++j) p.mask[mask_row + j] = 0;
    }
    if (ok && !stats_only) {
      bool w = true;
      if (kept > 0)
        w = mbar_wait(&bar[C::B_OD], (kept - 1) & 1, kWaitPrefillEpilogue,
                      nblk, 600);
      tc_fence_after();
      if (__all_sync(FULL, w)) {
        const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
        __nv_bfloat16* orow_g =
            p.o + ((size_t)(b * p.Hq + hq) * p.Lq + row_g) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t orow[32];
          tmem_ld32(lane_base + C::COL_O + c * 32, orow);
          tc_wait_ld();
          if (active) {
            uint4* dst = reinterpret_cast<uint4*>(orow_g + c * 32);
#pragma unroll
            for (int x = 0; x < 32; x += 8) {
              uint4 w4;
              w4.x = pack_bf16x2(__uint_as_float(orow[x]) * inv_l,
                                 __uint_as_float(orow[x + 1]) * inv_l);
              w4.y = pack_bf16x2(__uint_as_float(orow[x + 2]) * inv_l,
                                 __uint_as_float(orow[x + 3]) * inv_l);
              w4.z = pack_bf16x2(__uint_as_float(orow[x + 4]) * inv_l,
                                 __uint_as_float(orow[x + 5]) * inv_l);
              w4.w = pack_bf16x2(__uint_as_float(orow[x + 6]) * inv_l,
                                 __uint_as_float(orow[x + 7]) * inv_l);
              dst[x / 8] = w4;
            }
          }
        }
        if (active && p.lse)
          p.lse[(size_t)(b * p.Hq + hq) * p.Lq + row_g] = m_ref + __logf(l);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Host side: tensor maps and launch
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t,
                                  void*, const cuuint64_t*, const cuuint64_t*,
                                  const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

inline EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr,
                                cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 3-D map over a [planes, rows, D] bf16 tensor, box = 64 columns x box_rows,
// 128-byte swizzle, out-of-range rows read as zero.
inline bool encode_map(CUtensorMap* m, const void* base, int D, int rows,
                       long long planes, int box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)planes};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)rows * D * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base),
                  dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 4-D map over a page pool [pages][heads][page_rows][D] bf16 whose pages
// are `page_stride` elements apart: box = 64 columns x box_rows rows of one
// head of one page, 128-byte swizzle.
inline bool encode_pool_map(CUtensorMap* m, const void* base, int D,
                            int page_rows, int heads, long long pages,
                            long long page_stride, int box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)page_rows, (cuuint64_t)heads,
                        (cuuint64_t)pages};
  cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)page_rows * D * 2,
                           (cuuint64_t)page_stride * 2};
  cuuint32_t box[4] = {64, (cuuint32_t)box_rows, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base),
                  dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The page pool at D = 128 as 5-D (64 columns, 2 column halves, page rows,
// heads, pages): one copy brings box_rows whole rows of a page (both halves,
// 256 bytes a row), each half a 128-byte line under the 128-byte swizzle.
inline bool encode_pool_map_rows(CUtensorMap* m, const void* base,
                                 int page_rows, int heads, long long pages,
                                 long long page_stride, int box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  constexpr int D = 128;
  cuuint64_t dims[5] = {64, 2, (cuuint64_t)page_rows, (cuuint64_t)heads,
                        (cuuint64_t)pages};
  cuuint64_t strides[4] = {128, (cuuint64_t)D * 2,
                           (cuuint64_t)page_rows * D * 2,
                           (cuuint64_t)page_stride * 2};
  cuuint32_t box[5] = {64, 2, (cuuint32_t)box_rows, 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base),
                  dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, int BN, int BRL>
cudaError_t launch_prefill_t(const PrefillProblem& pr, cudaStream_t st) {
  using C = PrefillCfg<D, BN, BRL>;
  PrefillParams p;
  memset(&p, 0, sizeof p);
  if (!encode_map(&p.tq, pr.q, D, pr.Lq, (long long)pr.B * pr.Hq, 128) ||
      !encode_map(&p.tk, pr.k, D, pr.Lkv, (long long)pr.B * pr.Hkv, BN) ||
      !encode_map(&p.tv, pr.v, D, pr.Lkv, (long long)pr.B * pr.Hkv, BN))
    return cudaErrorInvalidValue;
  p.o = static_cast<__nv_bfloat16*>(pr.o);
  p.lse = pr.lse;
  p.counters = pr.counters;
  p.mask = pr.mask;
  p.margin = pr.margin;
  p.B = pr.B;
  p.Hq = pr.Hq;
  p.Hkv = pr.Hkv;
  p.Lq = pr.Lq;
  p.Lkv = pr.Lkv;
  p.nq = (pr.Lq + BRL - 1) / BRL;
  p.nk = (pr.Lkv + BN - 1) / BN;
  p.G = pr.Hq / pr.Hkv;
  p.scale = pr.scale;
  p.ln_lambda = pr.ln_lambda;
  p.causal = pr.causal;
  p.stats_only = pr.o == nullptr ? 1 : 0;
  const long long grid = (long long)p.nq * pr.B * pr.Hq;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(prefill_kernel<D, BN, BRL>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  prefill_kernel<D, BN, BRL><<<(unsigned)grid, C::THREADS, C::SMEM_ALLOC, st>>>(p);
  return cudaGetLastError();
}

// 128x128 tiles run prefill2_kernel (prefill2.cuh); 64x64 tiles run the
// single-tile kernel above.
template <int D>
cudaError_t launch_prefill2(const PrefillProblem& pr, cudaStream_t st);

inline cudaError_t launch_prefill(const PrefillProblem& pr, cudaStream_t st) {
  if (pr.d == 128 && pr.Br == 128) return launch_prefill2<128>(pr, st);
  if (pr.d == 64 && pr.Br == 128) return launch_prefill2<64>(pr, st);
  if (pr.d == 128 && pr.Br == 64) return launch_prefill_t<128, 64, 64>(pr, st);
  return launch_prefill_t<64, 64, 64>(pr, st);
}

}  // namespace blasst

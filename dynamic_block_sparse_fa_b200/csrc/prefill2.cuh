// prefill2.cuh -- BLASST prefill forward on sm_100a for 128x128 tiles with
// two query tiles per CTA that take turns on the tensor core.
//
// Same method and decisions as prefill.cuh ("BLASST: Dynamic BLocked
// Attention Sparsity via Softmax Thresholding", gist.science summary,
// section 2; MLSys'26 reading notes, core method and design trade-offs): per
// (tile, block) pair the row maxima of S = Q K^T are voted on, and a skipped
// pair computes no exp, issues no P.V MMA, and (unless the other tile of the
// CTA keeps the block) issues no V TMA load.
//
// CTA = 10 warps, query tiles t0 = 2p and t1 = 2p+1 of one head:
//   warp 0        TMA producer: Q0, Q1 once; K ring (2 blocks); V per block
//                 that at least one of the two tiles keeps, issued as soon as
//                 the first keeping decision is known
//   warp 1        MMA issuer; per block j: [tile 0] P0.V_j then QK0(j+1),
//                 [tile 1] P1.V_j then QK1(j+1), so that while one tile's
//                 softmax runs the tensor core works on the other tile
//   warps 2..5    softmax of tile 0 (thread = row; TMEM lane quadrants
//                 2, 3, 0, 1)
//   warps 6..9    softmax of tile 1
// Tensor memory (512 columns): S0 | S1 | O0 | O1, each 128 columns; P_t
// aliases the first 64 columns of S_t (two bf16 per column).  Because the
// MMA warp issues QK_t(j+1) after P_t.V_j, the arrival of S_t(j+1) also
// certifies that O_t is no longer being written, so the softmax may rescale
// O_t without a further wait.
//
// SKIP = false builds the dense forward without the skip machinery (no vote
// barrier, no decision words; V is loaded for every block as soon as its
// slot is free).  The library runs it for ln lambda = -inf, so the cost of
// the vote on the dense path can be measured against the SKIP = true kernel
// run with a threshold that never skips (ln lambda = -FLT_MAX).
#pragma once

#include "prefill.cuh"

namespace blasst {

template <int D>
struct Prefill2Cfg {
  static constexpr int BM = 128;
  static constexpr int BN = 128;
  static constexpr int NKS = 2;  // K ring depth
  static constexpr int NVS = 2;
  static constexpr int R = 8;  // decision ring per tile (> NKS)
  static constexpr int BOX_Q = BM * 128;
  static constexpr int BOX_K = BN * 128;
  static constexpr int QBYTES = BM * D * 2;
  static constexpr int KBYTES = BN * D * 2;
  static constexpr int OFF_Q = 0;  // Q0 then Q1
  static constexpr int OFF_K = OFF_Q + 2 * QBYTES;
  static constexpr int OFF_V = OFF_K + NKS * KBYTES;
  static constexpr int OFF_BAR = OFF_V + NVS * KBYTES;
  static constexpr int B_Q = 0;
  static constexpr int B_KF = 1;
  static constexpr int B_KE = B_KF + NKS;
  static constexpr int B_VF = B_KE + NKS;
  static constexpr int B_VE = B_VF + NVS;
  static constexpr int B_SF = B_VE + NVS;  // [2]
  static constexpr int B_PF = B_SF + 2;    // [2]
  static constexpr int B_OD = B_PF + 2;    // [2]
  static constexpr int B_DEC = B_OD + 2;   // [2][R]
  static constexpr int NBAR = B_DEC + 2 * R;
  static constexpr int OFF_DEC = OFF_BAR + NBAR * 8;  // int [2][R]
  static constexpr int OFF_TMEM = OFF_DEC + 2 * R * 4;
  static constexpr int OFF_ABORT = OFF_TMEM + 4;      // int [2]
  static constexpr int WPT = 4;  // softmax warps per tile (thread = row)
  static constexpr int OFF_XM = OFF_ABORT + 8;  // f32 [2][2 tiles][4]: margins
  static constexpr int SMEM = OFF_XM + 64;
  static constexpr int SMEM_ALLOC = SMEM + 1024;
  static constexpr int TMEM_COLS = 512;
  static constexpr int COL_S = 0;    // tile t at COL_S + t * 128
  static constexpr int COL_O = 256;  // tile t at COL_O + t * 128
  static constexpr int THREADS = 64 + 2 * WPT * 32;
  static_assert(SMEM_ALLOC <= 232448, "shared memory per CTA");
};

// MARGIN: also write each visited pair's decision margin (p.margin); a
// separate instance, so that the timed kernel carries no code for it.
template <int D, bool SKIP, bool MARGIN>
__global__ void __launch_bounds__(64 + 2 * 4 * 32, 1)
    prefill2_kernel(const __grid_constant__ PrefillParams p) {
  using C = Prefill2Cfg<D>;
  constexpr int BN = C::BN;
  constexpr unsigned FULL = 0xffffffffu;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const bool leader = (lane == 0);

  // Work item: KV-head-major (the CTAs resident at any time share one KV
  // head's K and V, which then stay in L2), and within a KV head the
  // longest tile pairs first; the G query heads of a pair are adjacent.
  const int nq2 = (p.nq + 1) >> 1;
  const int per_kv = nq2 * p.G;
  const int lin = blockIdx.x;
  const int kvi = lin / per_kv;  // b * Hkv + hkv
  const int rem = lin - kvi * per_kv;
  const int pair = nq2 - 1 - rem / p.G;
  const int b = kvi / p.Hkv;
  const int hkv = kvi - b * p.Hkv;
  const int hq = hkv * p.G + (rem - (rem / p.G) * p.G);
  // Tile t visits blocks [jlo_t[t], nblk_t[t]): up to its last row's
  // diagonal, and from the block holding its first row's first key when a
  // sliding window is set.  The CTA walks [jlo, nblk); ring slots and
  // barrier phases count blocks from jlo (K, V) or from jlo_t (per tile).
  int nblk_t[2], jlo_t[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int tile = 2 * pair + t;
    jlo_t[t] = 0;
    if (tile >= p.nq) {
      nblk_t[t] = 0;
    } else {
      const int last_row = min((tile + 1) * 128, p.Lq) - 1;
      const int kmax = p.causal ? min(p.Lkv - 1, last_row + (p.Lkv - p.Lq))
                                : p.Lkv - 1;
      nblk_t[t] = kmax / BN + 1;
      if (p.window > 0)
        jlo_t[t] = max(0, tile * 128 + (p.Lkv - p.Lq) - p.window + 1) / BN;
    }
  }
  const int nblk = max(nblk_t[0], nblk_t[1]);
  const int jlo = jlo_t[0];
  auto in_range = [&](int t, int j) { return j >= jlo_t[t] && j < nblk_t[t]; };

  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  // Decision words [2][R]: ((jt + 1) << 1) | skip for block jt of a tile,
  // published with a release store right after the vote.
  uint32_t* dec_word = reinterpret_cast<uint32_t*>(smem + C::OFF_DEC);
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
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bar[C::B_SF + t], 1);
      mbar_init(&bar[C::B_PF + t], C::WPT);  // P written: one arrival per softmax warp, kept blocks only
      mbar_init(&bar[C::B_OD + t], 1);
      for (int i = 0; i < C::R; ++i) mbar_init(&bar[C::B_DEC + t * C::R + i], 1);
    }
    for (int i = 0; i < 2 * C::R; ++i) dec_word[i] = 0u;
    reinterpret_cast<volatile int*>(smem + C::OFF_ABORT)[0] = 0;
    reinterpret_cast<volatile int*>(smem + C::OFF_ABORT)[1] = 0;
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

  if (warp == 0) {
    // ------------------------------------------------------------------
    // TMA producer
    // ------------------------------------------------------------------
    const uint64_t pol_q = policy_evict_first();
    const uint64_t pol_kv = policy_evict_last();
    const int zq = b * p.Hq + hq;
    const int zk = b * p.Hkv + hkv;
    auto issue_k = [&](int j) {
      const int st = (j - jlo) % C::NKS;
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
      const int nt = nblk_t[1] > 0 ? 2 : 1;
      mbar_arrive_expect_tx(&bar[C::B_Q], C::QBYTES * nt);
      for (int t = 0; t < nt; ++t)
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(sQ + t * C::QBYTES + c * C::BOX_Q, &p.tq, &bar[C::B_Q],
                      c * 64, (2 * pair + t) * 128, zq, pol_q);
      const int n0 = nblk - jlo < C::NKS ? nblk - jlo : C::NKS;
      for (int j = jlo; j < jlo + n0; ++j) issue_k(j);
    }
    __syncwarp();
    // Per block: first the V load (needed by the P.V right after the exp of
    // this block), then the K prefetch two blocks ahead (needed only by the
    // next block's QK, and blocked until this block's QKs release a slot).
    int vcount = 0;
    for (int j = jlo; j < nblk; ++j) {
      if (!stats_only) {
        bool need = !SKIP && (in_range(0, j) || in_range(1, j)), ok = true;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (!SKIP || need || !in_range(t, j)) continue;
          const int jt = j - jlo_t[t];
          const bool w = mbar_wait(&bar[C::B_DEC + t * C::R + jt % C::R],
                                   (jt / C::R) & 1, kWaitPrefillLoad, j,
                                   100 + t * C::R + jt % C::R);
          if (!__all_sync(FULL, w)) { ok = false; break; }
          need = (ld_acquire_shared(&dec_word[t * C::R + jt % C::R]) & 1u) == 0;
        }
        if (!ok) break;
        if (need) {
          const int n = vcount++;
          const int slot = n % C::NVS;
          if (n >= C::NVS) {
            const bool w = mbar_wait(&bar[C::B_VE + slot], ((n / C::NVS) - 1) & 1,
                                     kWaitPrefillLoad, j, 200 + slot);
            if (!__all_sync(FULL, w)) break;
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
      if (j + C::NKS < nblk) {
        const int jr = j - jlo;
        const bool w = mbar_wait(&bar[C::B_KE + jr % C::NKS], (jr / C::NKS) & 1,
                                 kWaitPrefillLoad, j, jr % C::NKS);
        if (!__all_sync(FULL, w)) break;
        if (leader) issue_k(j + C::NKS);
        __syncwarp();
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------
    // MMA issuer
    // ------------------------------------------------------------------
    constexpr uint32_t idesc_s = idesc_bf16(128, BN, 0, 0);
    constexpr uint32_t idesc_o = idesc_bf16(128, D, 0, 1);
    // Descriptors of the operand buffers, built once.  Stepping through an
    // operand only adds (byte offset >> 4) to the start-address field: every
    // address stays below 256 KB, so the 14-bit field never carries.
    const uint64_t dQ0 = smem_desc(smem_u32(sQ), 16, 1024, 2);
    const uint64_t dQ1 = smem_desc(smem_u32(sQ) + C::QBYTES, 16, 1024, 2);
    const uint64_t dK0 = smem_desc(smem_u32(sK), 16, 1024, 2);
    const uint64_t dK1 = smem_desc(smem_u32(sK) + C::KBYTES, 16, 1024, 2);
    const uint64_t dV0 = smem_desc(smem_u32(sV), C::BOX_K, 1024, 2);
    const uint64_t dV1 = smem_desc(smem_u32(sV) + C::KBYTES, C::BOX_K, 1024, 2);
    static_assert(C::NKS == 2 && C::NVS == 2, "two K and two V slots");
    auto qk = [&](int t, int j) {
      const int st = (j - jlo) % C::NKS;
      const uint32_t d_s = tmem + C::COL_S + t * 128;
      const uint64_t da0 = t ? dQ1 : dQ0;
      const uint64_t db0 = st ? dK1 : dK0;
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        // 16 columns = 32 B within a 64-column box; boxes are BOX_* apart
        const uint64_t ka = (uint64_t)(((k >> 2) * C::BOX_Q + (k & 3) * 32) >> 4);
        const uint64_t kb = (uint64_t)(((k >> 2) * C::BOX_K + (k & 3) * 32) >> 4);
        mma_ss_elect(d_s, da0 + ka, db0 + kb, idesc_s, k > 0 ? 1u : 0u);
      }
      mma_commit_elect(&bar[C::B_SF + t]);
    };
    // The whole warp runs the loop; one elected lane issues each MMA and
    // commit.  Waits are taken by every lane and made warp-uniform.  All
    // waits of a tile's step come before its MMAs, so the P.V and the next
    // QK^T of a tile go to the tensor core back to back.
    {
      bool ok = mbar_wait(&bar[C::B_Q], 0, kWaitPrefillMma, 0, 0) &&
                mbar_wait(&bar[C::B_KF], 0, kWaitPrefillMma, 0, 0);
      ok = __all_sync(FULL, ok);
      tc_fence_after();
      if (ok) {
        for (int t = 0; t < 2; ++t)
          if (in_range(t, jlo)) qk(t, jlo);
        mma_commit_elect(&bar[C::B_KE]);
      }
      int vcount = 0;
      int npv[2] = {0, 0};  // kept blocks of each tile so far
      for (int j = jlo; j < nblk && ok; ++j) {
        int vslot = -1;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const bool cur = in_range(t, j);
          const bool more = in_range(t, j + 1);
          if (!ok || !(cur || more)) continue;
          const int jt = j - jlo_t[t];
          bool kept = false;
          if (cur && !SKIP) {
            kept = true;
            ok = mbar_wait(&bar[C::B_PF + t], npv[t] & 1, kWaitPrefillMma, j,
                           300 + t);
            if (!__all_sync(FULL, ok)) { ok = false; break; }
          } else if (cur) {
            // The decision word: a skipped block needs nothing more (its
            // scores were read before the vote), a kept one its P (B_PF,
            // one phase per kept block).
            const uint32_t want = (uint32_t)(jt + 1) << 1;
            uint32_t w = ld_acquire_shared(&dec_word[t * C::R + jt % C::R]);
            if ((w & ~1u) != want) {
              const long long t0 = clock64();
              while (((w = ld_acquire_shared(
                           &dec_word[t * C::R + jt % C::R])) & ~1u) != want) {
                if (clock64() - t0 > kWaitLimitCycles) {
                  record_error(kWaitPrefillMma, j, 0, 310 + t);
                  ok = false;
                  break;
                }
              }
              if (!__all_sync(FULL, ok)) { ok = false; break; }
            }
            kept = !stats_only && (w & 1u) == 0;
            if (kept) {
              ok = mbar_wait(&bar[C::B_PF + t], npv[t] & 1, kWaitPrefillMma, j,
                             300 + t);
              if (!__all_sync(FULL, ok)) { ok = false; break; }
            }
          }
          if (kept && vslot < 0) {
            vslot = vcount % C::NVS;
            ok = mbar_wait(&bar[C::B_VF + vslot], (vcount / C::NVS) & 1,
                           kWaitPrefillMma, j, 200 + vslot);
            ++vcount;
            if (!__all_sync(FULL, ok)) { ok = false; break; }
          }
          if (more) {
            const int jr1 = j + 1 - jlo;
            ok = mbar_wait(&bar[C::B_KF + jr1 % C::NKS], (jr1 / C::NKS) & 1,
                           kWaitPrefillMma, j + 1, jr1 % C::NKS);
            if (!__all_sync(FULL, ok)) { ok = false; break; }
          }
          tc_fence_after();
          if (kept) {
            const uint32_t a_p = tmem + C::COL_S + t * 128;
            const uint64_t dv0 = vslot ? dV1 : dV0;
#pragma unroll
            for (int k = 0; k < BN / 16; ++k)  // 16 keys = 16 rows of 128 B
              mma_ts_elect(tmem + C::COL_O + t * 128, a_p + k * 8,
                     dv0 + (uint64_t)((k * 2048) >> 4), idesc_o,
                     (npv[t] > 0 || k > 0) ? 1u : 0u);
            ++npv[t];
          }
          if (more)
            qk(t, j + 1);
          else
            mma_commit_elect(&bar[C::B_OD + t]);  // tile t has issued its last MMA
        }
        if (!__all_sync(FULL, ok)) { ok = false; break; }
        if (vslot >= 0) mma_commit_elect(&bar[C::B_VE + vslot]);
        if (j + 1 < nblk) mma_commit_elect(&bar[C::B_KE + (j + 1 - jlo) % C::NKS]);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------
    // Softmax: warps 2..5 tile 0, warps 6..9 tile 1; thread = row (the
    // warp's TMEM lane quadrant is warp % 4).
    // ------------------------------------------------------------------
    constexpr int CPT = BN;  // score columns per thread
    constexpr int OPT = D;   // output columns per thread
    const int gw = warp - 2;
    const int t = gw / C::WPT;
    const int wi = gw - t * C::WPT;
    const uint32_t bar_id = 1 + t;
    constexpr uint32_t kBarThreads = 32 * C::WPT;
    const int nb = nblk_t[t];
    const int quad = warp & 3;
    const int rr = quad * 32 + lane;
    const int tile = 2 * pair + t;
    const int row_g = tile * 128 + rr;
    const bool active = nb > 0 && row_g < p.Lq;
    const int lim = p.causal ? min(row_g + (p.Lkv - p.Lq), p.Lkv - 1)
                             : p.Lkv - 1;
    // first key of the row's sliding window (0 without a window)
    const int first = p.window > 0
                          ? max(0, row_g + (p.Lkv - p.Lq) - p.window + 1)
                          : 0;
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    const uint32_t col_s = C::COL_S + t * 128;  // the row's scores
    const uint32_t col_p = C::COL_S + t * 128;  // its P (bf16 pairs)
    const uint32_t col_o = C::COL_O + t * 128;  // its O
    const float scale = p.scale;
    const float ln_lambda = p.ln_lambda;
    const float sl2 = scale * kPrefLog2e;
    const bool elected = (wi == 0 && lane == 0);
    const size_t mask_row =
        ((size_t)(b * p.Hq + hq) * p.nq + tile) * (size_t)p.nk;
    volatile int* abort_t = reinterpret_cast<volatile int*>(smem + C::OFF_ABORT);

    float m_crit = -INFINITY;
    float m_ref = -INFINITY;
    float l = 0.f;  // the row normaliser
    unsigned long long n_vis = 0, n_skp = 0;
    bool ok = true;

    for (int j = jlo_t[t]; j < nb; ++j) {
      const int jt = j - jlo_t[t];  // blocks this tile has visited before j
      if (!mbar_wait(&bar[C::B_SF + t], jt & 1, kWaitPrefillSoftmax, j, 400 + t))
        abort_t[t] = 1;  // read by every thread of the tile after the vote
      tc_fence_after();
      uint32_t sr[CPT / 32][32];
#pragma unroll
      for (int c = 0; c < CPT / 32; ++c)
        tmem_ld32(lane_base + col_s + c * 32, sr[c]);
      tc_wait_ld();

      const int col0 = j * BN;  // the block's first key
      if (col0 + CPT - 1 > lim || col0 < first) {
#pragma unroll
        for (int c = 0; c < CPT / 32; ++c)
#pragma unroll
          for (int x = 0; x < 32; ++x)
            if (col0 + c * 32 + x > lim || col0 + c * 32 + x < first)
              sr[c][x] = __float_as_uint(-INFINITY);
      }
      float mt;
      {
        // 8 chains of three-input maxima (two comparisons per instruction)
        float m8[8];
#pragma unroll
        for (int x = 0; x < 8; ++x)
          m8[x] = fmaxf(__uint_as_float(sr[0][x]), __uint_as_float(sr[0][x + 8]));
#pragma unroll
        for (int i = 16; i + 16 <= CPT; i += 16)
#pragma unroll
          for (int x = 0; x < 8; ++x)
            m8[x] = fmax3(m8[x], __uint_as_float(sr[i >> 5][(i & 31) + x]),
                          __uint_as_float(sr[(i + 8) >> 5][((i + 8) & 31) + x]));
        mt = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]),
                   fmaxf(m8[6], m8[7]));
      }
      const float mt_s = mt * scale;  // the row's block max
      const bool pred = !active || mt_s == -INFINITY ||
                        (mt_s - m_crit < ln_lambda);
      float* xm = reinterpret_cast<float*>(smem + C::OFF_XM) + ((jt & 1) * 2 + t) * 4;
      if constexpr (MARGIN) {  // max over the rows of m~ - m, per warp
        float dl = (active && mt_s != -INFINITY) ? mt_s - m_crit : -INFINITY;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1)
          dl = fmaxf(dl, __shfl_xor_sync(FULL, dl, o));
        if (lane == 0) xm[wi] = dl;
      }
      tc_fence_before();
      bool skip = false;
      if constexpr (SKIP) {
        skip = named_sync_and(bar_id, kBarThreads, pred) &&
               (ln_lambda > -INFINITY);
        if (abort_t[t]) { ok = false; break; }
      } else {
        // no vote: every block is kept; a wait that gave up ends the warp
        __syncwarp();
        if (__any_sync(FULL, abort_t[t] != 0)) { ok = false; break; }
      }
      if (elected) {
        ++n_vis;
        if (skip) ++n_skp;
        if (p.mask) p.mask[mask_row + j] = skip ? 2 : 1;
        if (MARGIN)
          p.margin[mask_row + j] =
              fmaxf(fmaxf(xm[0], xm[1]), fmaxf(xm[2], xm[3])) - ln_lambda;
        if constexpr (SKIP) {
          st_release_shared(&dec_word[t * C::R + jt % C::R],
                            ((uint32_t)(jt + 1) << 1) | (skip ? 1u : 0u));
          mbar_arrive(&bar[C::B_DEC + t * C::R + jt % C::R]);
        }
      }
      if (skip || stats_only) {  // the issuer reads the decision word
        if (active) m_crit = fmaxf(m_crit, mt_s);
        continue;
      }

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
      float rs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < CPT / 32; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          const float a0 = fmaf(__uint_as_float(sr[c][x]), sl2, -mb);
          const float a1 = fmaf(__uint_as_float(sr[c][x + 1]), sl2, -mb);
          const float p0 = ex2_approx(a0);
          const float p1 = ex2_approx(a1);
          rs[(x >> 1) & 3] += p0 + p1;
          pk[x / 2] = pack_bf16x2(p0, p1);
        }
        tmem_st16(lane_base + col_p + c * 16, pk);
      }
      l = alpha * l + ((rs[0] + rs[1]) + (rs[2] + rs[3]));
      tc_wait_st();
      // O_t is idle here (see the header comment); rescale whole warps.
      if (__any_sync(FULL, rescale)) {
        const float f = rescale ? alpha : 1.f;
#pragma unroll
        for (int c = 0; c < OPT / 32; ++c) {
          uint32_t orow[32];
          tmem_ld32(lane_base + col_o + c * 32, orow);
          tc_wait_ld();
#pragma unroll
          for (int x = 0; x < 32; ++x)
            orow[x] = __float_as_uint(__uint_as_float(orow[x]) * f);
          tmem_st32(lane_base + col_o + c * 32, orow);
        }
        tc_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[C::B_PF + t]);
      if (active) m_crit = fmaxf(m_crit, mt_s);
    }

    if (ok && elected && nb > 0) {
      if (p.counters) {
        atomicAdd(&p.counters[0], n_vis);
        atomicAdd(&p.counters[1], n_skp);
      }
      if (p.mask)
        for (int j = 0; j < p.nk; ++j)
          if (j < jlo_t[t] || j >= nb) p.mask[mask_row + j] = 0;
    }
    if (ok && !stats_only && nb > 0) {
      const bool w = mbar_wait(&bar[C::B_OD + t], 0, kWaitPrefillEpilogue, nb,
                               600 + t);
      tc_fence_after();
      const float lrow = l;
      if (__all_sync(FULL, w)) {
        const float inv_l = (lrow > 0.f) ? 1.f / lrow : 0.f;
        __nv_bfloat16* orow_g =
            p.o + ((size_t)(b * p.Hq + hq) * p.Lq + row_g) * D;
#pragma unroll
        for (int c = 0; c < OPT / 32; ++c) {
          uint32_t orow[32];
          tmem_ld32(lane_base + col_o + c * 32, orow);
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
          p.lse[(size_t)(b * p.Hq + hq) * p.Lq + row_g] = m_ref + __logf(lrow);
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

template <int D, bool SKIP, bool MARGIN>
cudaError_t launch_prefill2_t(const PrefillProblem& pr, cudaStream_t st) {
  using C = Prefill2Cfg<D>;
  PrefillParams p;
  memset(&p, 0, sizeof p);
  if (!encode_map(&p.tq, pr.q, D, pr.Lq, (long long)pr.B * pr.Hq, 128) ||
      !encode_map(&p.tk, pr.k, D, pr.Lkv, (long long)pr.B * pr.Hkv, 128) ||
      !encode_map(&p.tv, pr.v, D, pr.Lkv, (long long)pr.B * pr.Hkv, 128))
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
  p.nq = (pr.Lq + 127) / 128;
  p.nk = (pr.Lkv + 127) / 128;
  p.G = pr.Hq / pr.Hkv;
  p.scale = pr.scale;
  p.ln_lambda = pr.ln_lambda;
  p.causal = pr.causal;
  p.stats_only = pr.o == nullptr ? 1 : 0;
  p.window = pr.window;
  const long long grid = (long long)((p.nq + 1) / 2) * pr.B * pr.Hq;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(prefill2_kernel<D, SKIP, MARGIN>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  prefill2_kernel<D, SKIP, MARGIN>
      <<<(unsigned)grid, C::THREADS, C::SMEM_ALLOC, st>>>(p);
  return cudaGetLastError();
}

// The dense forward (ln lambda = -inf, outputs requested) runs the kernel
// without the vote; every other call runs the skipping kernel.
template <int D>
cudaError_t launch_prefill2(const PrefillProblem& pr, cudaStream_t st) {
  if (pr.margin != nullptr) return launch_prefill2_t<D, true, true>(pr, st);
  if (pr.ln_lambda == -INFINITY && pr.o != nullptr)
    return launch_prefill2_t<D, false, false>(pr, st);
  return launch_prefill2_t<D, true, false>(pr, st);
}

}  // namespace blasst

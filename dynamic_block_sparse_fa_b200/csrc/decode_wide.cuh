// decode_wide.cuh -- BLASST decode on the tensor core for wide head groups:
// 16 to 128 query heads per KV head (MQA and large GQA ratios), d = 128.
//
// Same method as decode.cuh (per (sequence, KV head, split): blocks of 64
// keys in ascending order, the G heads of the KV head are the rows of one
// tile and vote together, V is read only for kept blocks, split outputs are
// merged by log-sum-exp), but the scores and P.V run as tcgen05 MMAs with
// the G heads as the M = 128 rows (padded), which the CUDA-core kernel
// cannot feed fast enough once G x d FMAs per key exceed the memory time.
//   warp 0      producer: K blocks (2-slot ring) ahead of the scores; V of
//               a block as soon as the tile's decision keeps it (2 slots)
//   warp 1      MMA issuer (one lane): S = Q K^T (TS, A = Q from TMEM);
//               O += P V (SS, P from shared memory, V MN-major) one block
//               behind: the P.V of a kept block goes out after the next
//               block's S, so its V load overlaps that block's score and
//               vote
//   warps 2..5  one thread per head: Q into TMEM, row max, vote, exp, P
//               (bf16, two shared-memory slots), lazy O rescale (after the
//               pending P.V is done), epilogue
// Tensor memory: Q [0, 64) (bf16 pairs), S [64, 128), O [128, 256): 256
// columns, two CTAs per SM.
//
// Tiles.  With T = G the G heads are one tile (one decision per block).
// With T = 8 < G the heads form G / 8 tiles of 8 consecutive heads, each
// voting on its own, exactly as the CUDA-core decode cuts wide groups: the
// block's V load and P.V run when any tile keeps it, and the rows of a tile
// that skips it get P = 0 (no exp) and keep their running state, so they
// come out as if the block had not been touched.
#pragma once

#include "prefill.cuh"

namespace blasst {

constexpr int kWideD = 128;
constexpr int kWideBc = 64;
constexpr int kWideThreads = 192;

struct WideArgs {
  CUtensorMap tk, tv;        // [B*Hkv][Lkv][128], box 64 x 64
  const __nv_bfloat16* q;    // [B, Hq, 128]
  float* o_part;             // [B*Hq, S, 128]
  float* lse_part;           // [B*Hq, S]
  unsigned long long* counters;
  unsigned char* mask;       // [B*Hkv*(G/T), nk]
  int Hkv, G, Lkv, nk, S;
  int T;                     // heads per tile: G, or 8 (G a multiple of 8)
  int window;                // sliding window: the last `window` keys (0 = all)
  float scale, ln_lambda;
  int stats_only;
};

struct WideCfg {
  static constexpr int BOX = 64 * 128;     // 64 rows x 128 bytes
  static constexpr int TILE = 2 * BOX;     // 64 keys x 128 dims, 16 KB
  static constexpr int NK = 2, NV = 2;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + NK * TILE;
  static constexpr int PT = 128 * kWideBc * 2;  // P tile: 128 rows x 64 keys
  static constexpr int OFF_P = OFF_V + NV * TILE;  // [2] P tiles
  static constexpr int OFF_BAR = OFF_P + 2 * PT;
  static constexpr int B_KF = 0;   // [NK]
  static constexpr int B_KE = 2;   // [NK]
  static constexpr int B_VF = 4;   // [NV]
  static constexpr int B_VE = 6;   // [NV]
  static constexpr int B_QR = 8;   // Q in TMEM (one arrival per row warp)
  static constexpr int B_SF = 9;   // S in TMEM
  static constexpr int B_PF = 10;  // [2] P slot written (one arrival per warp)
  static constexpr int B_PE = 12;  // [2] P slot read by its P.V
  static constexpr int B_PVD = 14; // a P.V done (one phase per kept block)
  static constexpr int B_OD = 15;  // last MMA done
  static constexpr int NBAR = 16;
  static constexpr int R = 4;      // decision-word ring
  static constexpr int OFF_DEC = OFF_BAR + NBAR * 8;
  static constexpr int OFF_TMEM = OFF_DEC + R * 4;
  static constexpr int SMEM = OFF_TMEM + 8;
  static constexpr int SMEM_ALLOC = SMEM + 1024;
  static constexpr uint32_t COL_Q = 0, COL_S = 64, COL_O = 128;
};

// Polls a decision word until it holds block jj's decision (bounded);
// returns the word, or 0 after recording a timeout.
__device__ __forceinline__ uint32_t wide_decision(uint32_t* word, int jj,
                                                  unsigned int slot) {
  const uint32_t want = (uint32_t)(jj + 1) << 1;
  uint32_t w = ld_acquire_shared(word);
  if ((w & ~1u) == want) return w;
  const long long t0 = clock64();
  while (((w = ld_acquire_shared(word)) & ~1u) != want) {
    if (clock64() - t0 > kWaitLimitCycles) {
      record_error(kWaitDecodeWide, jj, 0, slot);
      return 0u;
    }
  }
  return w;
}

__global__ void __launch_bounds__(kWideThreads, 2)
    decode_wide_kernel(const __grid_constant__ WideArgs a) {
  using C = WideCfg;
  constexpr unsigned FULL = 0xffffffffu;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int s = blockIdx.x % a.S;
  const int bh = blockIdx.x / a.S;  // b * Hkv + hkv
  // first visible key and its block (sliding window); the splits divide
  // the blocks from there on
  const int key_lo = (a.window > 0 && a.Lkv > a.window) ? a.Lkv - a.window : 0;
  const int jlo = key_lo / kWideBc;
  const int j0 = jlo + (int)(((long long)s * (a.nk - jlo)) / a.S);
  const int j1 = jlo + (int)(((long long)(s + 1) * (a.nk - jlo)) / a.S);
  const int nb = j1 - j0;
  const int ntile = a.G / a.T;  // tiles per KV head
  if (a.mask && s == 0)  // blocks left of the window are not visited
    for (int e = threadIdx.x; e < ntile * jlo; e += kWideThreads)
      a.mask[((size_t)bh * ntile + e / jlo) * a.nk + e % jlo] = 0;

  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint32_t* dec_word = reinterpret_cast<uint32_t*>(smem + C::OFF_DEC);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM);
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar[C::B_KF + i], 1);
      mbar_init(&bar[C::B_KE + i], 1);
      mbar_init(&bar[C::B_VF + i], 1);
      mbar_init(&bar[C::B_VE + i], 1);
    }
    mbar_init(&bar[C::B_QR], 4);
    mbar_init(&bar[C::B_SF], 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar[C::B_PF + i], 4);
      mbar_init(&bar[C::B_PE + i], 1);
    }
    mbar_init(&bar[C::B_PVD], 1);
    mbar_init(&bar[C::B_OD], 1);
    for (int i = 0; i < C::R; ++i) dec_word[i] = 0u;
    // a wait that gave up in any head thread, read by all after the vote
    *reinterpret_cast<volatile int*>(smem + C::OFF_TMEM + 4) = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool stats_only = a.stats_only != 0;

  if (warp == 0) {
    // ------------------------------------------------------------ loads
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      prefetch_tmap(&a.tk);
      prefetch_tmap(&a.tv);
      auto load_k = [&](int jj) {
        const int sl = jj % C::NK;
        mbar_arrive_expect_tx(&bar[C::B_KF + sl], C::TILE);
        for (int c = 0; c < 2; ++c)
          tma_load_3d(smem + C::OFF_K + sl * C::TILE + c * C::BOX, &a.tk,
                      &bar[C::B_KF + sl], c * 64, (j0 + jj) * kWideBc, bh, pol);
      };
      bool ok = true;
      if (nb > 0) load_k(0);
      int nv = 0;
      for (int jj = 0; jj < nb && ok; ++jj) {
        // the next K block first (its slot frees when block jj-1 is done)
        if (jj + 1 < nb) {
          if (jj + 1 >= C::NK)
            ok = mbar_wait(&bar[C::B_KE + (jj + 1) % C::NK],
                           (((jj + 1) / C::NK) - 1) & 1, kWaitDecodeWide, jj,
                           1);
          if (!ok) break;
          load_k(jj + 1);
        }
        if (stats_only) continue;
        // then V of block jj if the tile keeps it
        const uint32_t w = wide_decision(&dec_word[jj % C::R], jj, 2);
        if (w == 0u) { ok = false; break; }
        if (w & 1u) continue;
        const int sl = nv % C::NV;
        if (nv >= C::NV &&
            !mbar_wait(&bar[C::B_VE + sl], ((nv / C::NV) - 1) & 1,
                       kWaitDecodeWide, jj, 3))
          break;
        mbar_arrive_expect_tx(&bar[C::B_VF + sl], C::TILE);
        for (int c = 0; c < 2; ++c)
          tma_load_3d(smem + C::OFF_V + sl * C::TILE + c * C::BOX, &a.tv,
                      &bar[C::B_VF + sl], c * 64, (j0 + jj) * kWideBc, bh, pol);
        ++nv;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA
    if (lane == 0 && nb > 0) {
      constexpr uint32_t id_s = idesc_bf16(128, kWideBc, 0, 0);
      constexpr uint32_t id_o = idesc_bf16(128, kWideD, 0, 1);
      const uint32_t aK = smem_u32(smem + C::OFF_K);
      const uint32_t aV = smem_u32(smem + C::OFF_V);
      const uint32_t aP = smem_u32(smem + C::OFF_P);
      bool ok = mbar_wait(&bar[C::B_QR], 0, kWaitDecodeWide, 0, 10);
      int npv = 0;           // P.V products issued
      bool pending = false;  // a kept block whose P.V is not issued yet
      // P.V of kept block number npv: P and V slot npv % 2
      auto issue_pv = [&]() {
        const int sl = npv % 2;
        ok = ok &&
             mbar_wait(&bar[C::B_PF + sl], (npv / 2) & 1, kWaitDecodeWide, npv,
                       13) &&
             mbar_wait(&bar[C::B_VF + sl], (npv / C::NV) & 1, kWaitDecodeWide,
                       npv, 14);
        if (!ok) return;
        tc_fence_after();
        const uint32_t vb = aV + sl * C::TILE, pb = aP + sl * C::PT;
#pragma unroll
        for (int k = 0; k < kWideBc / 16; ++k)
          mma_ss(tmem + C::COL_O,
                 smem_desc(pb + k * 32, 16, 1024, 2),  // P: K-major, 128 B rows
                 smem_desc(vb + k * 2048, C::BOX, 1024, 2), id_o,
                 (npv > 0 || k > 0) ? 1u : 0u);
        mma_commit(&bar[C::B_PE + sl]);
        mma_commit(&bar[C::B_VE + sl]);
        mma_commit(&bar[C::B_PVD]);
        ++npv;
      };
      for (int jj = 0; jj < nb && ok; ++jj) {
        const int sl = jj % C::NK;
        ok = mbar_wait(&bar[C::B_KF + sl], (jj / C::NK) & 1, kWaitDecodeWide,
                       jj, 11);
        if (!ok) break;
        tc_fence_after();
        const uint32_t kb = aK + sl * C::TILE;
#pragma unroll
        for (int k = 0; k < kWideD / 16; ++k)
          mma_ts(tmem + C::COL_S, tmem + C::COL_Q + k * 8,
                 smem_desc(kb + (k >> 2) * C::BOX + (k & 3) * 32, 16, 1024, 2),
                 id_s, k > 0 ? 1u : 0u);
        mma_commit(&bar[C::B_SF]);
        mma_commit(&bar[C::B_KE + sl]);
        if (pending) {  // the previous kept block, behind this block's S
          issue_pv();
          pending = false;
          if (!ok) break;
        }
        const uint32_t w = wide_decision(&dec_word[jj % C::R], jj, 12);
        if (w == 0u) { ok = false; break; }
        pending = !stats_only && (w & 1u) == 0;
      }
      if (ok && pending) issue_pv();
      mma_commit(&bar[C::B_OD]);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------- head rows
    const int quad = warp & 3;
    const int h = quad * 32 + lane;  // head of the group = TMEM lane
    const bool active = h < a.G;
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    const bool elected = (quad == 0 && lane == 0);
    // the first row of each tile keeps the tile's statistics
    const bool tile_lead = active && (h % a.T) == 0;
    const size_t mask_row = ((size_t)bh * ntile + h / a.T) * a.nk;
    const uint32_t tbits = a.T >= 32 ? FULL : ((1u << a.T) - 1u);
    const int tshift = a.T >= 32 ? 0 : (lane / a.T) * a.T;
    const int b = bh / a.Hkv;
    const int hkv = bh - b * a.Hkv;
    const size_t qrow_i = (size_t)(b * a.Hkv + hkv) * a.G;  // first head row
    {
      // padding rows read the group's first head and store zeros: no
      // branch before the warp-collective TMEM stores
      const uint4* qrow = reinterpret_cast<const uint4*>(
          a.q + (qrow_i + (active ? h : 0)) * kWideD);
      const uint32_t keep = active ? 0xffffffffu : 0u;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t r[32];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint4 v = __ldg(qrow + c * 8 + u);
          r[4 * u] = v.x & keep;
          r[4 * u + 1] = v.y & keep;
          r[4 * u + 2] = v.z & keep;
          r[4 * u + 3] = v.w & keep;
        }
        __syncwarp();
        tmem_st32(lane_base + C::COL_Q + c * 32, r);
      }
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[C::B_QR]);
    }
    const float scale = a.scale, ln_lambda = a.ln_lambda;
    const float sl2 = scale * kPrefLog2e;
    float m_crit = -INFINITY, m_ref = -INFINITY, l = 0.f;
    unsigned long long n_vis = 0, n_skp = 0;
    int kp = 0;  // kept blocks so far (their P slot is kp % 2)
    uint8_t* sP = smem + C::OFF_P;
    bool ok = true;
    for (int jj = 0; jj < nb; ++jj) {
      const int j = j0 + jj;
      const bool w = mbar_wait(&bar[C::B_SF], jj & 1, kWaitDecodeWide, jj, 20);
      tc_fence_after();
      uint32_t sr[2][32];
      tmem_ld32(lane_base + C::COL_S, sr[0]);
      tmem_ld32(lane_base + C::COL_S + 32, sr[1]);
      tc_wait_ld();
      const int valid = min(kWideBc, a.Lkv - j * kWideBc);
      const int first = key_lo - j * kWideBc;  // keys below it are hidden
      if (valid < kWideBc || first > 0) {
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int x = 0; x < 32; ++x)
            if (c * 32 + x >= valid || c * 32 + x < first)
              sr[c][x] = __float_as_uint(-INFINITY);
      }
      float m8[8];
#pragma unroll
      for (int x = 0; x < 8; ++x)
        m8[x] = fmaxf(__uint_as_float(sr[0][x]), __uint_as_float(sr[0][x + 8]));
#pragma unroll
      for (int i = 16; i < 64; i += 16)
#pragma unroll
        for (int x = 0; x < 8; ++x)
          m8[x] = fmax3(m8[x], __uint_as_float(sr[i >> 5][(i & 31) + x]),
                        __uint_as_float(sr[(i + 8) >> 5][((i + 8) & 31) + x]));
      const float mt = fmax3(fmax3(m8[0], m8[1], m8[2]),
                             fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
      const float mt_s = mt * scale;
      const bool pred = !active || mt_s == -INFINITY ||
                        (mt_s - m_crit < ln_lambda);
      tc_fence_before();
      // a failed wait in any thread ends the loop for all, after the vote
      volatile int* abort_w = reinterpret_cast<volatile int*>(smem + C::OFF_TMEM + 4);
      if (!w) *abort_w = 1;
      // this row's tile: the AND of its T rows' votes (one warp holds a
      // tile of 8; a tile of all G rows is the whole vote below)
      const unsigned bal = __ballot_sync(FULL, pred);
      const bool all = named_sync_and(1, 128, pred && w);
      if (*abort_w) { ok = false; break; }
      const bool tile_all = a.T == a.G ? all
                                       : ((bal >> tshift) & tbits) == tbits;
      const bool skip = all && (ln_lambda > -INFINITY);        // the block
      const bool skip_row = tile_all && (ln_lambda > -INFINITY);  // my tile
      if (elected)
        st_release_shared(&dec_word[jj % C::R],
                          ((uint32_t)(jj + 1) << 1) | (skip ? 1u : 0u));
      if (tile_lead) {
        ++n_vis;
        if (skip_row) ++n_skp;
        if (a.mask) a.mask[mask_row + j] = skip_row ? 2 : 1;
      }
      if (skip || stats_only) {
        if (active) m_crit = fmaxf(m_crit, mt_s);
        continue;
      }
      float alpha = 1.f;
      bool rescale = false;
      if (active && !skip_row && mt_s != -INFINITY) {
        const float m_new = fmaxf(m_crit, mt_s);
        if (m_ref == -INFINITY || m_new > m_ref + kRescaleNats) {
          alpha = (m_ref == -INFINITY) ? 0.f
                                       : ex2_approx((m_ref - m_new) * kPrefLog2e);
          m_ref = m_new;
          rescale = true;
        }
      }
      // a row of a tile that skips the block gets P = 0: exp2(-inf)
      const float mb = (active && !skip_row && m_ref != -INFINITY)
                           ? m_ref * kPrefLog2e
                           : INFINITY;
      // P (bf16, this row's 64 keys = one 128-byte swizzled row) into P
      // slot kp % 2, once the P.V two kept blocks back has read it
      const int psl = kp & 1;
      bool wp = true;
      if (kp >= 2)
        wp = mbar_wait(&bar[C::B_PE + psl], ((kp >> 1) - 1) & 1,
                       kWaitDecodeWide, jj, 22);
      float rs = 0.f;
      uint32_t pk[32];
#pragma unroll
      for (int x = 0; x < 64; x += 2) {
        const float p0 =
            ex2_approx(fmaf(__uint_as_float(sr[x >> 5][x & 31]), sl2, -mb));
        const float p1 =
            ex2_approx(fmaf(__uint_as_float(sr[x >> 5][(x & 31) + 1]), sl2, -mb));
        rs += p0 + p1;
        pk[x / 2] = pack_bf16x2(p0, p1);
      }
      l = alpha * l + rs;
      uint8_t* prow = sP + psl * C::PT + h * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(prow + ((c ^ (h & 7)) * 16)) =
            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      fence_async_smem();
      // The O rescale waits for the P.V of the previous kept block (it may
      // still be running: P.V goes out one block behind).
      if (__any_sync(FULL, rescale)) {
        bool wv = true;
        if (kp >= 1)
          wv = mbar_wait(&bar[C::B_PVD], (kp - 1) & 1, kWaitDecodeWide, jj, 23);
        tc_fence_after();
        const float f = rescale ? alpha : 1.f;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t orow[32];
          tmem_ld32(lane_base + C::COL_O + c * 32, orow);
          tc_wait_ld();
#pragma unroll
          for (int x = 0; x < 32; ++x)
            orow[x] = __float_as_uint(__uint_as_float(orow[x]) * f);
          tmem_st32(lane_base + C::COL_O + c * 32, orow);
        }
        tc_wait_st();
        wp = wp && wv;
      }
      tc_fence_before();
      const bool wall = __all_sync(FULL, wp);  // every lane votes
      if (lane == 0 && wall) mbar_arrive(&bar[C::B_PF + psl]);
      ++kp;
      if (active) m_crit = fmaxf(m_crit, mt_s);
    }
    if (ok && tile_lead && a.counters && nb > 0) {
      atomicAdd(&a.counters[0], n_vis);
      atomicAdd(&a.counters[1], n_skp);
    }
    if (ok && !stats_only) {
      const size_t row = qrow_i + h;
      bool w2 = true;
      if (nb > 0) w2 = mbar_wait(&bar[C::B_OD], 0, kWaitDecodeWide, nb, 21);
      tc_fence_after();
      const bool done = __all_sync(FULL, w2) && nb > 0;  // every lane votes
      const bool have = done && l > 0.f;
      const float inv_l = have ? 1.f / l : 0.f;
      float* dst = a.o_part + (row * a.S + s) * kWideD;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t orow[32];
        if (done) {
          tmem_ld32(lane_base + C::COL_O + c * 32, orow);
          tc_wait_ld();
        }
        if (active) {
#pragma unroll
          for (int x = 0; x < 32; x += 4)
            *reinterpret_cast<float4*>(dst + c * 32 + x) =
                have ? make_float4(__uint_as_float(orow[x]) * inv_l,
                                   __uint_as_float(orow[x + 1]) * inv_l,
                                   __uint_as_float(orow[x + 2]) * inv_l,
                                   __uint_as_float(orow[x + 3]) * inv_l)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      if (active) a.lse_part[row * a.S + s] = have ? m_ref + __logf(l) : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace blasst

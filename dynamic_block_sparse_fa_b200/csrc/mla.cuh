// mla.cuh -- BLASST decode over a multi-head latent (MLA) cache on sm_100a.
//
// Every query head h of a token scores the shared latent cache row c_t
// (d_qk = 576: 512 latent + 64 rope dimensions) as scale * q_h . c_t, and the
// value is the latent part c_t[0:512] (the attention forms the method is
// stated to support: MLSys'26 reading notes; gist.science summary, section
// 3).  The H heads of a token form one decode tile (rows), blocks of 64 keys,
// the decode criterion and online softmax per split, split-KV merged by
// log-sum-exp: the same algorithm as decode.cuh with K = c and V = c[:512].
//
// One CTA pair (a cluster of 2) per (sequence, split), the work cut so that
// no cache byte is loaded twice and no score product is issued twice:
//   rank 0 scores columns [0, 256) of c_t (4 boxes of 64) and accumulates
//          value columns [0, 256): the same 4 boxes;
//   rank 1 scores columns [256, 576) (5 boxes) and accumulates value
//          columns [256, 512): the first 4 of its boxes.
// Each CTA's head threads read their partial scores from tensor memory,
// store them into the other CTA's shared memory with st.async (distributed
// shared memory, as [4-key group][head] float4s so that a warp's stores are
// contiguous, counted as transaction bytes on the other CTA's barrier), and
// add the other CTA's partial to their own.  IEEE addition commutes, so
// both CTAs hold the same scores bit for bit and take the same decisions
// without exchanging them.
//   warp 0      TMA producer: this rank's boxes of each cache block, ring of 4
//   warp 1      MMA issuer (whole warp, one elected lane issues): partial
//               S = Q_r c_r^T (TS, 16 or 20 products, N = 64), issued as soon
//               as the previous S has been read; for a kept block
//               O_r += P V_r (TS, 4 products, N = 256).  Order S(1), S(2),
//               PV(0), S(3), PV(1), ...: the scores run one block ahead
//   warps 2..5  one thread per head (TMEM lane): Q_r into TMEM, partial
//               score exchange one block ahead (block j+1's partial is read
//               and sent before block j is decided, so the exchange overlaps
//               the vote and the exps), row max, vote, exp, P, lazy O
//               rescale, epilogue
// Tensor memory: Q_r [0, 160) (bf16 pairs), P [160, 192), S [192, 256),
// O_r [256, 512).
#pragma once

#include "prefill.cuh"

namespace blasst {

constexpr int kMlaDqk = 576;
constexpr int kMlaDv = 512;
constexpr int kMlaBc = 64;
constexpr int kMlaRows = 128;  // heads per tile (at most)

struct MlaArgs {
  CUtensorMap tc;            // cache [B][L][576], box 64 x 64
  const __nv_bfloat16* q;    // [B, H, 576]
  float* o_part;             // [B*H, S, 512] normalised split outputs
  float* lse_part;           // [B*H, S]
  unsigned long long* counters;
  unsigned char* mask;       // [B, nk]
  int B, H, L, nk, S;
  float scale, ln_lambda;
  int stats_only;
};

constexpr int kMlaPairThreads = 192;

struct MlaPairCfg {
  static constexpr int BOX = 64 * 128;        // 64 keys x 64 columns (bf16)
  static constexpr int NBX = 5;               // boxes per ring slot (rank 1)
  static constexpr int SLOT = NBX * BOX;      // 40960 bytes
  static constexpr int NK = 4;                // ring slots
  static constexpr int XBYTES = 64 * 128 * 4; // a partial score block, f32
  static constexpr int OFF_K = 0;
  static constexpr int OFF_X = OFF_K + NK * SLOT;  // [2] partials from the peer
  static constexpr int OFF_BAR = OFF_X + 2 * XBYTES;
  static constexpr int B_KF = 0;            // [NK]
  static constexpr int B_KE = NK;           // [NK]
  static constexpr int B_QR = 2 * NK;       // Q in TMEM (per head warp)
  static constexpr int B_SF = B_QR + 1;     // partial S in TMEM
  static constexpr int B_SR = B_SF + 1;     // partial S read (per head warp)
  static constexpr int B_PF = B_SR + 1;     // P written (per head warp)
  static constexpr int B_PVD = B_PF + 1;    // a P.V done
  static constexpr int B_OD = B_PVD + 1;    // last MMA done
  static constexpr int B_XF = B_OD + 1;     // [2] my X[b] holds the peer's partial
  static constexpr int NBAR = B_XF + 2;
  static constexpr int R = 4;               // decision-word ring
  static constexpr int OFF_DEC = OFF_BAR + NBAR * 8;
  static constexpr int OFF_TMEM = OFF_DEC + R * 4;
  static constexpr int SMEM = OFF_TMEM + 8;
  static constexpr int SMEM_ALLOC = SMEM + 1024;
  static constexpr uint32_t COL_Q = 0, COL_P = 160, COL_S = 192, COL_O = 256;
  static_assert(SMEM_ALLOC <= 232448, "shared memory per CTA");
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kMlaPairThreads, 1)
    mla_pair_kernel(const __grid_constant__ MlaArgs a) {
  using C = MlaPairCfg;
  constexpr unsigned FULL = 0xffffffffu;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const uint32_t peer = rank ^ 1u;
  const int bs = blockIdx.x >> 1;  // b * S + s
  const int s = bs % a.S;
  const int b = bs / a.S;
  const int j0 = (int)(((long long)s * a.nk) / a.S);
  const int j1 = (int)(((long long)(s + 1) * a.nk) / a.S);
  const int nb = j1 - j0;
  const int box0 = rank ? 4 : 0;  // first cache box (64 columns) of mine
  const int nbx = rank ? 5 : 4;   // boxes I score
  const bool recorder = rank == 0;

  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint32_t* dec_word = reinterpret_cast<uint32_t*>(smem + C::OFF_DEC);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM);
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NK; ++i) {
      mbar_init(&bar[C::B_KF + i], 1);
      mbar_init(&bar[C::B_KE + i], 1);
    }
    mbar_init(&bar[C::B_QR], 4);
    mbar_init(&bar[C::B_SF], 1);
    mbar_init(&bar[C::B_SR], 4);
    mbar_init(&bar[C::B_PF], 4);
    mbar_init(&bar[C::B_PVD], 1);
    mbar_init(&bar[C::B_OD], 1);
    // X[b]'s phases: one arrival (this CTA arming the phase with the bytes
    // it expects) plus the peer's 32 KB of st.async transactions
    for (int i = 0; i < 2; ++i) mbar_init(&bar[C::B_XF + i], 1);
    for (int i = 0; i < C::R; ++i) dec_word[i] = 0u;
    // a wait that gave up in any head thread, read by all after the vote
    *reinterpret_cast<volatile int*>(smem + C::OFF_TMEM + 4) = 0;
    fence_mbar_init();
    for (int i = 0; i < 2; ++i) mbar_arrive_expect_tx(&bar[C::B_XF + i], C::XBYTES);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  // both CTAs' barriers are initialised before either arrives remotely
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool stats_only = a.stats_only != 0;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();  // each box is read once
      prefetch_tmap(&a.tc);
      for (int jj = 0; jj < nb; ++jj) {
        const int sl = jj % C::NK;
        if (jj >= C::NK &&
            !mbar_wait(&bar[C::B_KE + sl], ((jj / C::NK) - 1) & 1,
                       kWaitMlaPair, jj, sl))
          break;
        mbar_arrive_expect_tx(&bar[C::B_KF + sl], nbx * C::BOX);
#pragma unroll 1
        for (int c = 0; c < nbx; ++c)
          tma_load_3d(smem + C::OFF_K + sl * C::SLOT + c * C::BOX, &a.tc,
                      &bar[C::B_KF + sl], (box0 + c) * 64, (j0 + jj) * kMlaBc,
                      b, pol);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA
    if (nb > 0) {
      constexpr uint32_t id_s = idesc_bf16(128, kMlaBc, 0, 0);
      constexpr uint32_t id_o = idesc_bf16(128, 256, 0, 1);
      const uint32_t aK = smem_u32(smem + C::OFF_K);
      const int nmma = nbx * 4;  // K = 64 columns per box, 16 per product
      auto score = [&](int jj) {
        const uint32_t kb = aK + (jj % C::NK) * C::SLOT;
#pragma unroll 4
        for (int k = 0; k < nmma; ++k)
          mma_ts_elect(tmem + C::COL_S, tmem + C::COL_Q + k * 8,
                 smem_desc(kb + (k >> 2) * C::BOX + (k & 3) * 32, 16, 1024, 2),
                 id_s, k > 0 ? 1u : 0u);
        mma_commit_elect(&bar[C::B_SF]);
      };
      // P.V of block jj once its decision is known (kept: after its P),
      // then the block's ring slot is released
      int npv = 0;
      auto value = [&](int jj) -> bool {
        const int sl = jj % C::NK;
        const uint32_t want = (uint32_t)(jj + 1) << 1;
        uint32_t w = ld_acquire_shared(&dec_word[jj % C::R]);
        if ((w & ~1u) != want) {
          const long long t0 = clock64();
          bool tout = false;
          while (((w = ld_acquire_shared(&dec_word[jj % C::R])) & ~1u) != want) {
            if (clock64() - t0 > kWaitLimitCycles) {
              record_error(kWaitMlaPair, jj, 0, 13);
              tout = true;
              break;
            }
          }
          if (__any_sync(FULL, tout)) return false;
        }
        if (!stats_only && (w & 1u) == 0) {
          if (!__all_sync(FULL, mbar_wait(&bar[C::B_PF], npv & 1, kWaitMlaPair, jj, 14)))
            return false;
          tc_fence_after();
          // my 256 value columns: the slot's first 4 boxes, MN-major
          const uint32_t kb = aK + sl * C::SLOT;
#pragma unroll
          for (int k = 0; k < kMlaBc / 16; ++k)
            mma_ts_elect(tmem + C::COL_O, tmem + C::COL_P + k * 8,
                   smem_desc(kb + k * 2048, C::BOX, 1024, 2), id_o,
                   (npv > 0 || k > 0) ? 1u : 0u);
          ++npv;
          mma_commit_elect(&bar[C::B_PVD]);
        }
        mma_commit_elect(&bar[C::B_KE + sl]);
        return true;
      };
      bool ok = __all_sync(FULL, mbar_wait(&bar[C::B_QR], 0, kWaitMlaPair, 0, 10) &&
                                 mbar_wait(&bar[C::B_KF], 0, kWaitMlaPair, 0, 11));
      tc_fence_after();
      if (ok) score(0);
      // The head threads read S(jj+1) before they decide block jj, so the
      // scores of block jj+1 go to the tensor core ahead of P.V(jj-1):
      // order S(1), S(2), PV(0), S(3), PV(1), ...
      for (int jj = 0; jj < nb && ok; ++jj) {
        if (jj + 1 < nb) {
          // my partial S(jj) has been read: S(jj+1) overwrites it
          const int sn = (jj + 1) % C::NK;
          ok = __all_sync(FULL, mbar_wait(&bar[C::B_SR], jj & 1, kWaitMlaPair, jj, 16) &&
                                mbar_wait(&bar[C::B_KF + sn], ((jj + 1) / C::NK) & 1,
                                          kWaitMlaPair, jj + 1, 11 + sn));
          if (!ok) break;
          tc_fence_after();
          score(jj + 1);
        }
        if (jj >= 1) ok = value(jj - 1);
      }
      if (ok) value(nb - 1);
      mma_commit_elect(&bar[C::B_OD]);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------- head rows
    const int quad = warp & 3;
    const int h = quad * 32 + lane;  // head = TMEM lane
    const bool active = h < a.H;
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    const bool elected = (quad == 0 && lane == 0);
    // my part of the Q row into TMEM: nbx chunks of 64 bf16 (32 columns);
    // padding rows (h >= H) read head 0's row and store zeros (no branch
    // before the warp-collective TMEM stores)
    {
      const uint4* qrow = reinterpret_cast<const uint4*>(
          a.q + ((size_t)b * a.H + (active ? h : 0)) * kMlaDqk) + box0 * 8;
      const uint32_t keep = active ? 0xffffffffu : 0u;
#pragma unroll 1
      for (int c = 0; c < nbx; ++c) {
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
    // the exchange buffers: mine (written by the peer) and the peer's.
    // X[b] is written again (block jj+2) only after the peer has received
    // my partial of block jj+1, which I send after reading X[b] for block
    // jj: the two CTAs' steps interlock, so X[b] needs no "free" signal.
    const uint32_t x_mine = smem_u32(smem + C::OFF_X);
    const uint32_t x_peer = map_shared(x_mine, peer);
    const uint32_t xf_peer = map_shared(smem_u32(&bar[C::B_XF]), peer);
    const bool armer = quad == 0 && lane == 0;  // re-arms X[b]'s next phase
    const float scale = a.scale, ln_lambda = a.ln_lambda;
    const float sl2 = scale * kPrefLog2e;
    float m_crit = -INFINITY, m_ref = -INFINITY, l = 0.f;
    unsigned long long n_vis = 0, n_skp = 0;
    bool ok = true;
    int npv = 0;         // kept blocks so far (one P.V each)
    // Block jj's partial goes to the peer one step ahead: the head threads
    // read S(jj+1) and send it before they decide block jj, so that the
    // exchange of block jj+1 runs while block jj is voted on and
    // exponentiated.  cur: block jj's scores; nxt: block jj+1's partial.
    bool w = true;  // this thread's waits so far
    uint32_t cur[2][32], nxt[2][32];
    auto read_send = [&](int jj, uint32_t (&sr)[2][32]) {
      if (!mbar_wait(&bar[C::B_SF], jj & 1, kWaitMlaPair, jj, 20)) w = false;
      tc_fence_after();
      tmem_ld32(lane_base + C::COL_S, sr[0]);
      tmem_ld32(lane_base + C::COL_S + 32, sr[1]);
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[C::B_SR]);  // S(jj+1) may overwrite S
      // my partial into the peer's X[jj & 1] as [4-key group][head]
      // float4s, counted on the peer's X[jj & 1] barrier
      const uint32_t xp = x_peer + (jj & 1) * C::XBYTES + h * 16;
#pragma unroll
      for (int q4 = 0; q4 < 16; ++q4) {
        const uint32_t* v = &sr[q4 >> 3][(q4 & 7) * 4];
        st_async_v4(xp + q4 * 2048, v[0], v[1], v[2], v[3],
                    xf_peer + (jj & 1) * 8);
      }
    };
    if (nb > 0) read_send(0, cur);
    for (int jj = 0; jj < nb; ++jj) {
      const int j = j0 + jj;
      const int xb = jj & 1;
      if (jj > 0) {
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int x = 0; x < 32; ++x) cur[c][x] = nxt[c][x];
      }
      uint32_t (&sr)[2][32] = cur;
      // the peer's partial of block jj (sent one step ago), added to mine
      // (the peer adds in the other order: the same sums)
      if (!mbar_wait_cluster(&bar[C::B_XF + xb], (jj >> 1) & 1, kWaitMlaPair,
                             jj, 32 + xb))
        w = false;
      // X[xb]'s phase for block jj is complete (this thread has seen it):
      // arm the phase of block jj+2
      if (armer && jj + 2 < nb)
        mbar_arrive_expect_tx(&bar[C::B_XF + xb], C::XBYTES);
      const float4* xm =
          reinterpret_cast<const float4*>(smem + C::OFF_X + xb * C::XBYTES) + h;
#pragma unroll
      for (int q4 = 0; q4 < 16; ++q4) {
        const float4 o4 = xm[q4 * 128];
        uint32_t* v = &sr[q4 >> 3][(q4 & 7) * 4];
        v[0] = __float_as_uint(__uint_as_float(v[0]) + o4.x);
        v[1] = __float_as_uint(__uint_as_float(v[1]) + o4.y);
        v[2] = __float_as_uint(__uint_as_float(v[2]) + o4.z);
        v[3] = __float_as_uint(__uint_as_float(v[3]) + o4.w);
      }
      // X[xb] has been read: the peer may now refill it (block jj+2), which
      // it does only after it has received my partial of block jj+1
      if (jj + 1 < nb) read_send(jj + 1, nxt);
      const int valid = min(kMlaBc, a.L - j * kMlaBc);  // keys of the block
      if (valid < kMlaBc) {
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int x = 0; x < 32; ++x)
            if (c * 32 + x >= valid) sr[c][x] = __float_as_uint(-INFINITY);
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
      const bool all = named_sync_and(1, 128, pred && w);
      if (*abort_w) { ok = false; break; }
      const bool skip = all && (ln_lambda > -INFINITY);
      if (elected) {
        st_release_shared(&dec_word[jj % C::R],
                          ((uint32_t)(jj + 1) << 1) | (skip ? 1u : 0u));
        ++n_vis;
        if (skip) ++n_skp;
        if (recorder && a.mask) a.mask[(size_t)b * a.nk + j] = skip ? 2 : 1;
      }
      if (skip || stats_only) {
        if (active) m_crit = fmaxf(m_crit, mt_s);
        continue;
      }
      // P and O are free once the previous P.V is done
      if (npv > 0 &&
          !mbar_wait(&bar[C::B_PVD], (npv - 1) & 1, kWaitMlaPair, jj, 22))
        w = false;
      tc_fence_after();
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
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          const float p0 = ex2_approx(fmaf(__uint_as_float(sr[c][x]), sl2, -mb));
          const float p1 =
              ex2_approx(fmaf(__uint_as_float(sr[c][x + 1]), sl2, -mb));
          rs += p0 + p1;
          pk[x / 2] = pack_bf16x2(p0, p1);
        }
        tmem_st16(lane_base + C::COL_P + c * 16, pk);
      }
      l = alpha * l + rs;
      tc_wait_st();
      if (__any_sync(FULL, rescale)) {
        const float f = rescale ? alpha : 1.f;
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
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
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[C::B_PF]);
      ++npv;
      if (active) m_crit = fmaxf(m_crit, mt_s);
    }
    if (ok && elected && recorder && a.counters && nb > 0) {
      atomicAdd(&a.counters[0], n_vis);
      atomicAdd(&a.counters[1], n_skp);
    }
    if (ok && !stats_only) {
      const size_t row = (size_t)b * a.H + h;
      bool w2 = true;
      if (nb > 0) w2 = mbar_wait(&bar[C::B_OD], 0, kWaitMlaPair, nb, 21);
      tc_fence_after();
      // warp-wide: every lane takes part (padding heads included)
      const bool done = __all_sync(FULL, w2) && nb > 0;
      const bool have = done && l > 0.f;
      const float inv_l = have ? 1.f / l : 0.f;
      float* dst = a.o_part + (row * a.S + s) * kMlaDv + rank * 256;
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
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
      if (active && rank == 0)
        a.lse_part[row * a.S + s] = have ? m_ref + __logf(l) : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  // the peer's stores and arrivals into this CTA's shared memory are over
  // before either CTA exits
  cluster_sync_all();
}

// lse = ln sum_s exp(lse_s), o = sum_s exp(lse_s - lse) o_s -> bf16.  One
// CTA of 128 threads per (sequence, head), 4 value columns per thread.
__global__ void __launch_bounds__(128) mla_combine_kernel(
    const float* o_part, const float* lse_part, __nv_bfloat16* o, float* lse,
    int S) {
  const size_t row = blockIdx.x;
  const float* lp = lse_part + row * S;
  float mx = -INFINITY;
  for (int s = 0; s < S; ++s) mx = fmaxf(mx, lp[s]);
  float den = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (mx > -INFINITY) {
    for (int s = 0; s < S; ++s) {
      const float wgt = lp[s] == -INFINITY ? 0.f : __expf(lp[s] - mx);
      den += wgt;
      const float4 v =
          reinterpret_cast<const float4*>(o_part + (row * S + s) * kMlaDv)[threadIdx.x];
      acc.x += wgt * v.x;
      acc.y += wgt * v.y;
      acc.z += wgt * v.z;
      acc.w += wgt * v.w;
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  uint2 w;
  w.x = pack_bf16x2(acc.x * inv, acc.y * inv);
  w.y = pack_bf16x2(acc.z * inv, acc.w * inv);
  reinterpret_cast<uint2*>(o + row * kMlaDv)[threadIdx.x] = w;
  if (threadIdx.x == 0 && lse) lse[row] = den > 0.f ? mx + __logf(den) : -INFINITY;
}

}  // namespace blasst

// backward.cuh -- backward of the BLASST prefill forward on sm_100a, with the
// forward's skip decisions held fixed (128x128 tiles, d = 128).
//
// Fine-tuning with BLASST active ("BLASST: Dynamic BLocked Attention
// Sparsity via Softmax Thresholding", gist.science summary, section 2,
// "Treinamento Consciente de Esparsidade"; Hindi summary, algorithm design)
// differentiates the forward as it ran.  With its decisions fixed that
// forward is softmax attention restricted, per query tile, to its kept
// blocks, so only the kept (tile, block) pairs enter the backward:
//   D_r = dO_r . O_r;  P = exp(scale q k^T - lse);  dV += P^T dO;
//   dP = dO V^T;  dS = P o (dP - D);  dK += scale dS^T Q;  dQ += scale dS K
// A pair the forward skipped (or did not visit) does no MMA and loads
// nothing.
//
// Three kernels (five with a mask):
//   bwd_prep_kernel     D and lse * log2 e per query row (rows padded to 16
//                       bytes, for the producer's TMA), zeroes the f32 dQ
//                       accumulator
//   bwd_count_kernel,   with a mask: kept pairs per CTA, and the CTAs in
//   bwd_order_kernel    order of those counts, most first
//   bwd_dkdv_kernel     one CTA per (sequence, KV head, key block j): K_j and
//                       V_j stay in shared memory while the kept query tiles
//                       of the G query heads stream through; dK_j, dV_j
//                       accumulate in tensor memory, each pair's dQ tile is
//                       staged in shared memory (four 32-column boxes through
//                       two 16 KB halves) and added to the f32 accumulator
//                       by TMA bulk reductions
//   bwd_dq_kernel       dQ = bf16(scale * accumulator)
// bwd_dkdv_kernel: warp 0 TMA producer (Q_i, dO_i ring of 2), warp 1 MMA
// issuer (one lane), warps 2..5 one thread per tensor-memory lane.  Per kept
// pair the MMAs are
//   S^T  = K_j Q_i^T      (SS, K-major A and B)        -> TMEM [0, 128)
//   dP^T = V_j dO_i^T     (SS)                         -> TMEM [128, 256)
//   dV  += P^T dO_i       (TS, A = P^T (bf16) from TMEM [0, 64),
//                          B = dO_i MN-major)          -> [256, 384)
//   dK  += dS^T Q_i       (TS, A = dS^T from TMEM [128, 192),
//                          B = Q_i MN-major)           -> [384, 512)
//   dQ_i = dS K_j         (SS, A = dS MN-major from shared memory,
//                          B = K_j MN-major)           -> [128, 256)
// Pairs are pipelined one deep.  The threads take pair n's dS, then pair
// n+1's P while the tensor core runs dK_n and dQ_n, then read pair n's dQ
// tile out (it lands in the dP^T columns, which dP^T_{n+1} waits for).  The
// issuer's order per pair: dK_n, dQ_n | dV_{n+1} | dP^T_{n+1}, S^T_{n+2};
// S^T_{n+2} comes last because its Q slot is the one dK_n releases.  The
// producer brings each pair's lse (ring of 2) and D (one slot) by TMA.
// Tensor memory is the whole 512 columns: one CTA per SM.
#pragma once

#include "prefill.cuh"

namespace blasst {

struct BwdParams {
  CUtensorMap tq, tk, tv, tdo;
  CUtensorMap tdq;  // f32 dQ accumulator [B*Hq][Lq][D], box 32 x 128
  const __nv_bfloat16* o;     // [B, Hq, Lq, D]
  const __nv_bfloat16* dout;  // [B, Hq, Lq, D]
  const float* lse;           // [B, Hq, Lq] natural log
  const unsigned char* mask;  // [B, Hq, nq, nk]; 1 = kept (null: all kept)
  float* dq_acc;              // [B, Hq, Lq, D]
  float* delta;               // [B*Hq][Lqp]: D per query row
  float* lse2;                // [B*Hq][Lqp]: lse * log2 e per query row
  CUtensorMap tdel, tlse2;    // those two, 128-column boxes
  int Lqp;                    // Lq rounded up to 4 (16-byte row stride)
  __nv_bfloat16* dq;          // [B, Hq, Lq, D]
  __nv_bfloat16* dk;          // [B, Hkv, Lkv, D]
  __nv_bfloat16* dv;          // [B, Hkv, Lkv, D]
  int* counts;                // masked: kept pairs per grid slot (scratch)
  const int* order;           // masked: grid slot of each CTA (null: own)
  int B, Hq, Hkv, Lq, Lkv, nq, nk, G, causal;
  float scale;
};

constexpr int kBwdD = 128;
// the work order's rank kernel is quadratic in the CTA count: above this
// many CTAs the grid keeps its own order
constexpr long long kBwdOrderMaxSlots = 32768;
constexpr int kBwdThreads = 192;

struct BwdCfg {
  static constexpr int TILE = 128 * kBwdD * 2;  // 32 KB, two 64-column boxes
  static constexpr int BOX = 128 * 128;         // bytes of one box
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int OFF_Q = OFF_V + TILE;     // [2]
  static constexpr int OFF_DO = OFF_Q + 2 * TILE;  // [2]
  static constexpr int OFF_DS = OFF_DO + 2 * TILE;  // dS^T [keys][queries]
  static constexpr int OFF_LSE = OFF_DS + TILE;      // f32 [2][128] lse * log2 e
  static constexpr int OFF_DEL = OFF_LSE + 2 * 512;  // f32 [128] D
  static constexpr int OFF_BAR = OFF_DEL + 512;
  static constexpr int B_KV = 0;
  static constexpr int B_QF = 1;    // [2]
  static constexpr int B_QE = 3;    // [2]
  static constexpr int B_SF = 5;    // S^T in TMEM
  static constexpr int B_DPF = 6;   // dP^T in TMEM
  static constexpr int B_PR = 7;    // P^T written (one arrival per warp)
  static constexpr int B_DSR = 8;   // dS^T written (one arrival per warp)
  static constexpr int B_DQF = 9;   // dQ tile in TMEM
  static constexpr int B_DQR = 10;  // dQ tile read out (one arrival per warp)
  static constexpr int B_LF = 11;   // [2] a pair's lse in its ring slot
  static constexpr int B_LE = 13;   // [2] that slot read (one arrival per warp)
  static constexpr int B_DF = 15;   // the pair's D in shared memory
  static constexpr int NBAR = 16;
  static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_TMEM + 8;
  static constexpr int SMEM_ALLOC = SMEM + 1024;
  static_assert(SMEM_ALLOC <= 232448, "shared memory per CTA");
};

// global[box at (c0, c1, c2)] += shared box (f32 add), as a bulk group.
__device__ __forceinline__ void tma_reduce_add_3d(const void* tmap,
                                                  const void* src, int c0,
                                                  int c1, int c2) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group "
      "[%0, {%2, %3, %4}], [%1];" ::"l"(tmap),
      "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// the shared-memory sources of every committed bulk group have been read
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// all but the most recently committed bulk group have been read
__device__ __forceinline__ void bulk_wait_read_but_one() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// D_r = sum_e dO_re O_re (f32), and the row's dQ accumulator set to zero.
// One warp per query row, 4 elements per lane.
__global__ void __launch_bounds__(256) bwd_prep_kernel(const BwdParams p) {
  const long long rows = (long long)p.B * p.Hq * p.Lq;
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const uint2 a = reinterpret_cast<const uint2*>(p.o + row * kBwdD)[lane];
  const uint2 g = reinterpret_cast<const uint2*>(p.dout + row * kBwdD)[lane];
  float s = bf16lo(a.x) * bf16lo(g.x) + bf16hi(a.x) * bf16hi(g.x) +
            bf16lo(a.y) * bf16lo(g.y) + bf16hi(a.y) * bf16hi(g.y);
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) s += __shfl_xor_sync(0xffffffffu, s, m);
  if (lane == 0) {
    const long long r = row / p.Lq, q = row - r * p.Lq;
    p.delta[r * p.Lqp + q] = s;
    p.lse2[r * p.Lqp + q] = p.lse[row] * kPrefLog2e;
    if (q == p.Lq - 1)  // the row's padding columns: finite, never used
      for (int c = p.Lq; c < p.Lqp; ++c) {
        p.delta[r * p.Lqp + c] = 0.f;
        p.lse2[r * p.Lqp + c] = 0.f;
      }
  }
  reinterpret_cast<float4*>(p.dq_acc + row * kBwdD)[lane] =
      make_float4(0.f, 0.f, 0.f, 0.f);
}

// dQ = bf16(scale * accumulator), 8 elements per thread.
// Work order of a masked backward.  A CTA's work is its kept (head, tile)
// pairs, which a sparse mask spreads very unevenly over the key blocks, so
// the CTAs go out by kept pairs, most first (ties in grid order).  Grid slot
// s = jb * (B*Hkv) + b*Hkv + hkv is the CTA of key block jb; one warp counts
// a slot's pairs.
__global__ void __launch_bounds__(256) bwd_count_kernel(const BwdParams p) {
  const int nbk = p.B * p.Hkv;
  const long long n = (long long)nbk * p.nk;
  const long long s = ((long long)blockIdx.x * 256 + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (s >= n) return;
  const int jb = (int)(s / nbk);
  const int bk = (int)(s - (long long)jb * nbk);
  const int b = bk / p.Hkv;
  const int hkv = bk - b * p.Hkv;
  const int off = p.Lkv - p.Lq;
  int c = 0;
  const int cand = p.G * p.nq;
  for (int x = lane; x < cand; x += 32) {
    const int g = x / p.nq;
    const int i = x - g * p.nq;
    if (p.causal && min((i + 1) * 128, p.Lq) - 1 + off < jb * 128) continue;
    const int hq = hkv * p.G + g;
    c += __ldg(p.mask + ((size_t)(b * p.Hq + hq) * p.nq + i) * p.nk + jb) == 1;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if (lane == 0) p.counts[s] = c;
}

// order[rank of slot s] = s, rank = slots with more kept pairs, or as many
// and a lower index.  The ranks are a permutation of 0 .. n-1.
__global__ void __launch_bounds__(256) bwd_order_kernel(const BwdParams p,
                                                         int* order) {
  __shared__ int tile[2048];
  const int n = p.B * p.Hkv * p.nk;
  const int s = blockIdx.x * 256 + threadIdx.x;
  const int cs = s < n ? p.counts[s] : 0;
  int rank = 0;
  for (int t0 = 0; t0 < n; t0 += 2048) {
    const int m = min(2048, n - t0);
    __syncthreads();
    for (int u = threadIdx.x; u < m; u += 256) tile[u] = p.counts[t0 + u];
    __syncthreads();
    if (s < n)
      for (int u = 0; u < m; ++u) {
        const int cu = tile[u];
        rank += (cu > cs) || (cu == cs && t0 + u < s);
      }
  }
  if (s < n) order[rank] = s;
}

__global__ void __launch_bounds__(256) bwd_dq_kernel(const BwdParams p) {
  const long long n8 = (long long)p.B * p.Hq * p.Lq * (kBwdD / 8);
  const long long i = (long long)blockIdx.x * 256 + threadIdx.x;
  if (i >= n8) return;
  const float4 x = reinterpret_cast<const float4*>(p.dq_acc)[2 * i];
  const float4 y = reinterpret_cast<const float4*>(p.dq_acc)[2 * i + 1];
  const float sc = p.scale;
  uint4 w;
  w.x = pack_bf16x2(x.x * sc, x.y * sc);
  w.y = pack_bf16x2(x.z * sc, x.w * sc);
  w.z = pack_bf16x2(y.x * sc, y.y * sc);
  w.w = pack_bf16x2(y.z * sc, y.w * sc);
  reinterpret_cast<uint4*>(p.dq)[i] = w;
}

__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ BwdParams p) {
  using C = BwdCfg;
  constexpr unsigned FULL = 0xffffffffu;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Causal key block j has the most query tiles for j = 0: CTAs go out in
  // ascending j over all (sequence, KV head), longest first.
  const int nbk = p.B * p.Hkv;
  const int slot = p.order ? __ldg(p.order + blockIdx.x) : (int)blockIdx.x;
  const int jb = slot / nbk;         // key block
  const int bk = slot - jb * nbk;    // b * Hkv + hkv
  const int b = bk / p.Hkv;
  const int hkv = bk - b * p.Hkv;
  const int off = p.Lkv - p.Lq;      // bottom-right causal alignment
  // Pair (g, i) of query head hkv*G + g and query tile i enters the
  // backward iff the forward kept it (and, causal, it is visible at all).
  auto kept = [&](int g, int i) -> bool {
    if (p.causal && min((i + 1) * 128, p.Lq) - 1 + off < jb * 128) return false;
    if (!p.mask) return true;
    const int hq = hkv * p.G + g;
    return __ldg(p.mask + ((size_t)(b * p.Hq + hq) * p.nq + i) * p.nk + jb) == 1;
  };
  // the next kept pair after (g, i) in (head, tile) order; false at the end
  auto next_kept = [&](int& g, int& i) -> bool {
    ++i;
    while (g < p.G) {
      if (i >= p.nq) {
        ++g;
        i = 0;
        continue;
      }
      if (kept(g, i)) return true;
      ++i;
    }
    return false;
  };

  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM);
  if (threadIdx.x == 0) {
    mbar_init(&bar[C::B_KV], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar[C::B_QF + s], 1);
      mbar_init(&bar[C::B_QE + s], 1);
    }
    mbar_init(&bar[C::B_SF], 1);
    mbar_init(&bar[C::B_DPF], 1);
    mbar_init(&bar[C::B_PR], 4);
    mbar_init(&bar[C::B_DSR], 4);
    mbar_init(&bar[C::B_DQF], 1);
    mbar_init(&bar[C::B_DQR], 4);
    for (int r = 0; r < 2; ++r) {
      mbar_init(&bar[C::B_LF + r], 1);
      mbar_init(&bar[C::B_LE + r], 4);
    }
    mbar_init(&bar[C::B_DF], 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      const uint64_t pol_kv = policy_evict_first();
      const uint64_t pol_q = policy_evict_last();
      prefetch_tmap(&p.tq);
      prefetch_tmap(&p.tk);
      prefetch_tmap(&p.tv);
      prefetch_tmap(&p.tdo);
      prefetch_tmap(&p.tdq);
      mbar_arrive_expect_tx(&bar[C::B_KV], 2 * C::TILE);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        tma_load_3d(smem + C::OFF_K + c * C::BOX, &p.tk, &bar[C::B_KV], c * 64,
                    jb * 128, bk, pol_kv);
        tma_load_3d(smem + C::OFF_V + c * C::BOX, &p.tv, &bar[C::B_KV], c * 64,
                    jb * 128, bk, pol_kv);
      }
      int n = 0;
      bool ok = true;
      for (int g = 0; g < p.G && ok; ++g) {
        const int zq = b * p.Hq + hkv * p.G + g;
        for (int i = 0; i < p.nq; ++i) {
          if (!kept(g, i)) continue;
          const int s = n & 1;
          if (n >= 2 &&
              !mbar_wait(&bar[C::B_QE + s], ((n >> 1) - 1) & 1, kWaitBackward,
                         n, s)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar[C::B_QF + s], 2 * C::TILE);
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            tma_load_3d(smem + C::OFF_Q + s * C::TILE + c * C::BOX, &p.tq,
                        &bar[C::B_QF + s], c * 64, i * 128, zq, pol_q);
            tma_load_3d(smem + C::OFF_DO + s * C::TILE + c * C::BOX, &p.tdo,
                        &bar[C::B_QF + s], c * 64, i * 128, zq, pol_q);
          }
          // lse of pair n into slot s once pair n-2's P phase has read it
          if (n >= 2 &&
              !mbar_wait(&bar[C::B_LE + s], ((n >> 1) - 1) & 1, kWaitBackward,
                         n, 41)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar[C::B_LF + s], 512);
          tma_load_3d(smem + C::OFF_LSE + s * 512, &p.tlse2, &bar[C::B_LF + s],
                      i * 128, zq, 0, pol_q);
          // D of pair n once pair n-1's dS phase (its one reader) is over;
          // that phase needs this D's predecessor, so DSR cannot run ahead
          if (n >= 1 && !mbar_wait(&bar[C::B_DSR], (n - 1) & 1,
                                   kWaitBackward, n, 40)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar[C::B_DF], 512);
          tma_load_3d(smem + C::OFF_DEL, &p.tdel, &bar[C::B_DF], i * 128, zq,
                      0, pol_q);
          ++n;
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t id_kk = idesc_bf16(128, 128, 0, 0);  // K-major A, B
      constexpr uint32_t id_km = idesc_bf16(128, 128, 0, 1);  // B MN-major
      constexpr uint32_t id_mm = idesc_bf16(128, 128, 1, 1);  // A, B MN-major
      const uint32_t aK = smem_u32(smem + C::OFF_K);
      const uint32_t aV = smem_u32(smem + C::OFF_V);
      const uint32_t aQ = smem_u32(smem + C::OFF_Q);
      const uint32_t aDO = smem_u32(smem + C::OFF_DO);
      const uint32_t aDS = smem_u32(smem + C::OFF_DS);
      // K-major operand (128 rows x 128 elements, two 64-column boxes):
      // the 16-element step k is box k/4, 32 bytes k%4 into the row.
      auto kmaj = [&](uint32_t base, int k) {
        return smem_desc(base + (k >> 2) * C::BOX + (k & 3) * 32, 16, 1024, 2);
      };
      // MN-major operand (K runs down the rows): step k is rows 16k..16k+15,
      // the two 64-column boxes are C::BOX apart.
      auto mnmaj = [&](uint32_t base, int k) {
        return smem_desc(base + k * 2048, C::BOX, 1024, 2);
      };
      bool ok = mbar_wait(&bar[C::B_KV], 0, kWaitBackward, 0, 20);
      // S^T of pair n: K Q_n^T into [0, 128)
      auto issue_s = [&](int n) {
        const int s = n & 1;
        ok = ok && mbar_wait(&bar[C::B_QF + s], (n >> 1) & 1, kWaitBackward,
                             n, 21 + s);
        if (!ok) return;
        tc_fence_after();
        const uint32_t q_s = aQ + s * C::TILE;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_ss(tmem + 0, kmaj(aK, k), kmaj(q_s, k), id_kk, k > 0 ? 1u : 0u);
        mma_commit(&bar[C::B_SF]);
      };
      // dP^T of pair n: V dO_n^T into [128, 256) (its dO arrived with Q)
      auto issue_dp = [&](int n) {
        const uint32_t do_s = aDO + (n & 1) * C::TILE;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_ss(tmem + 128, kmaj(aV, k), kmaj(do_s, k), id_kk,
                 k > 0 ? 1u : 0u);
        mma_commit(&bar[C::B_DPF]);
      };
      // dV += P^T dO_n once the threads have written P^T of pair n
      auto issue_dv = [&](int n) {
        ok = ok && mbar_wait(&bar[C::B_PR], n & 1, kWaitBackward, n, 24);
        if (!ok) return;
        tc_fence_after();
        const uint32_t do_s = aDO + (n & 1) * C::TILE;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_ts(tmem + 256, tmem + 0 + k * 8, mnmaj(do_s, k), id_km,
                 (n > 0 || k > 0) ? 1u : 0u);
      };
      // Pairs are pipelined one deep: while the threads compute P of pair
      // n+1, the tensor core runs dK and dQ of pair n.  Per pair n:
      //   [dS_n written]  dK_n, dQ_n
      //   [P_{n+1}]       dV_{n+1}
      //   [dQ_n read]     dP^T_{n+1}, then S^T_{n+2}
      // S^T_{n+2} comes last: its Q slot is the one dK_n has just released.
      int g = 0, i = -1;
      bool have = next_kept(g, i);
      int n = 0;
      if (have && ok) {
        issue_s(0);
        if (ok) issue_dp(0);
        issue_dv(0);
        int g1 = g, i1 = i;
        if (next_kept(g1, i1)) issue_s(1);
      }
      while (have && ok) {
        const int s = n & 1;
        ok = mbar_wait(&bar[C::B_DSR], n & 1, kWaitBackward, n, 25);
        if (!ok) break;
        tc_fence_after();
        const uint32_t q_s = aQ + s * C::TILE;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_ts(tmem + 384, tmem + 128 + k * 8, mnmaj(q_s, k), id_km,
                 (n > 0 || k > 0) ? 1u : 0u);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_ss(tmem + 128, mnmaj(aDS, k), mnmaj(aK, k), id_mm,
                 k > 0 ? 1u : 0u);
        mma_commit(&bar[C::B_DQF]);
        mma_commit(&bar[C::B_QE + s]);
        int g2 = g, i2 = i;
        const bool h2 = next_kept(g2, i2);
        if (h2) {
          issue_dv(n + 1);
          // dP^T overwrites the columns dQ_n is read from
          ok = ok && mbar_wait(&bar[C::B_DQR], n & 1, kWaitBackward, n, 23);
          if (!ok) break;
          tc_fence_after();
          issue_dp(n + 1);
          int g3 = g2, i3 = i2;
          if (next_kept(g3, i3)) issue_s(n + 2);
        }
        ++n;
        g = g2;
        i = i2;
        have = h2;
      }
    }
    __syncwarp();
  } else {
    // ----------------------------------------------------------- threads
    const int quad = warp & 3;
    const int rr = quad * 32 + lane;  // TMEM lane of this thread
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    float* lse_s = reinterpret_cast<float*>(smem + C::OFF_LSE);
    float* del_s = reinterpret_cast<float*>(smem + C::OFF_DEL);
    uint8_t* sDS = smem + C::OFF_DS;
    const int key = jb * 128 + rr;
    const bool key_ok = key < p.Lkv;
    const float sl2 = p.scale * kPrefLog2e;
    int n = 0;
    bool ok = true;
    uint32_t pk[64];  // P^T of a pair, from its P phase to its dS phase
    // P^T of pair m (query tile i) into TMEM [0, 64); its lse in slot m & 1
    auto p_phase = [&](int m, int i) {
      const float* lse_m = lse_s + (m & 1) * 128;
      {
        const bool wl = ok && mbar_wait(&bar[C::B_LF + (m & 1)], (m >> 1) & 1,
                                        kWaitBackward, m, 33);
        ok = __all_sync(FULL, wl);
      }
        // P^T (thread = key row, 128 query columns) into TMEM [0, 64) as
        // bf16; the packed values stay in registers for dS.
        const bool w1 = ok && mbar_wait(&bar[C::B_SF], m & 1, kWaitBackward, m, 30);
        ok = __all_sync(FULL, w1);
        tc_fence_after();
        // rows that see every query column of the tile need no mask; a warp
        // whose 32 rows all do takes the unmasked loop
        const bool row_full = key_ok && i * 128 + 127 < p.Lq &&
                              (!p.causal || key <= i * 128 + off);
        const bool warp_full = __all_sync(FULL, row_full);
        const float4* lse4 = reinterpret_cast<const float4*>(lse_m);
        // chunk cc + 1 is read while chunk cc is exponentiated; P of chunk
        // cc goes to columns [16 cc, 16 cc + 16), all read already
        uint32_t svb[2][32];
        if (ok) {
          tmem_ld32(lane_base + 0, svb[0]);
          tc_wait_ld();
        }
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          if (!ok) break;
          if (cc < 3) tmem_ld32(lane_base + (cc + 1) * 32, svb[(cc + 1) & 1]);
          const uint32_t (&sv)[32] = svb[cc & 1];
          if (warp_full) {
#pragma unroll
            for (int x = 0; x < 32; x += 4) {
              const float4 l4 = lse4[(cc * 32 + x) >> 2];
              const float p0 = ex2_approx(fmaf(__uint_as_float(sv[x]), sl2, -l4.x));
              const float p1 = ex2_approx(fmaf(__uint_as_float(sv[x + 1]), sl2, -l4.y));
              const float p2 = ex2_approx(fmaf(__uint_as_float(sv[x + 2]), sl2, -l4.z));
              const float p3 = ex2_approx(fmaf(__uint_as_float(sv[x + 3]), sl2, -l4.w));
              pk[cc * 16 + (x >> 1)] = pack_bf16x2(p0, p1);
              pk[cc * 16 + (x >> 1) + 1] = pack_bf16x2(p2, p3);
            }
          } else {
#pragma unroll
          for (int x = 0; x < 32; x += 2) {
            float pv[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int c = cc * 32 + x + e;  // query column in the tile
              const int qr = i * 128 + c;
              const bool valid = key_ok && qr < p.Lq &&
                                 (!p.causal || key <= qr + off);
              pv[e] = valid ? ex2_approx(fmaf(__uint_as_float(sv[x + e]), sl2,
                                              -lse_m[c]))
                            : 0.f;
            }
            pk[cc * 16 + (x >> 1)] = pack_bf16x2(pv[0], pv[1]);
          }
          }
          uint32_t st16[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) st16[u] = pk[cc * 16 + u];
          tmem_st16(lane_base + 0 + cc * 16, st16);
          if (cc < 3) tc_wait_ld();
        }
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (ok && lane == 0) {
          mbar_arrive(&bar[C::B_PR]);
          mbar_arrive(&bar[C::B_LE + (m & 1)]);  // the lse slot is free
        }
    };
    // dS^T of pair m, once its D and its dP^T have arrived
    auto d_phase = [&](int m) {
      {
        const bool wd = ok && mbar_wait(&bar[C::B_DF], m & 1, kWaitBackward, m, 34);
        ok = __all_sync(FULL, wd);
      }
        // dS^T = P^T o (dP^T - D) into TMEM [128, 192) and shared memory
        const bool w2 =
            ok && mbar_wait(&bar[C::B_DPF], m & 1, kWaitBackward, m, 31);
        ok = __all_sync(FULL, w2);
        // the buffer holds the previous pair's last dQ staging until the
        // reduction has read it (its wait is taken here, after P)
        if (m > 0) {
          if (warp == 2 && lane == 0) bulk_wait_read_all();
          named_sync(1, 128);
        }
        tc_fence_after();
        // the same overlap: dS^T of chunk cc goes to [128 + 16 cc, +16),
        // below the dP^T columns still to be read
        uint32_t dpb[2][32];
        if (ok) {
          tmem_ld32(lane_base + 128, dpb[0]);
          tc_wait_ld();
        }
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          if (!ok) break;
          if (cc < 3) tmem_ld32(lane_base + 128 + (cc + 1) * 32, dpb[(cc + 1) & 1]);
          const uint32_t (&dp)[32] = dpb[cc & 1];
          uint32_t dk16[16];
#pragma unroll
          for (int x = 0; x < 32; x += 4) {
            const float4 d4 =
                reinterpret_cast<const float4*>(del_s)[(cc * 32 + x) >> 2];
            const uint32_t pw0 = pk[cc * 16 + (x >> 1)];
            const uint32_t pw1 = pk[cc * 16 + (x >> 1) + 1];
            dk16[x >> 1] = pack_bf16x2(
                bf16lo(pw0) * (__uint_as_float(dp[x]) - d4.x),
                bf16hi(pw0) * (__uint_as_float(dp[x + 1]) - d4.y));
            dk16[(x >> 1) + 1] = pack_bf16x2(
                bf16lo(pw1) * (__uint_as_float(dp[x + 2]) - d4.z),
                bf16hi(pw1) * (__uint_as_float(dp[x + 3]) - d4.w));
          }
          tmem_st16(lane_base + 128 + cc * 16, dk16);
          // dS^T row rr, query columns 32cc..32cc+31: box cc/2, 16-byte
          // chunks (cc%2)*4 .. +3 of the 128-byte row, 128-byte swizzle
          uint8_t* row = sDS + (cc >> 1) * C::BOX + rr * 128;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int ch = ((cc & 1) * 4 + u) ^ (rr & 7);
            *reinterpret_cast<uint4*>(row + ch * 16) =
                make_uint4(dk16[4 * u], dk16[4 * u + 1], dk16[4 * u + 2],
                           dk16[4 * u + 3]);
          }
          if (cc < 3) tc_wait_ld();
        }
        tc_wait_st();
        fence_async_smem();
        tc_fence_before();
        __syncwarp();
        if (ok && lane == 0) mbar_arrive(&bar[C::B_DSR]);
    };
    // the dQ tile of pair m (query tile i of head hq) out to the accumulator
    auto e_phase = [&](int m, int i, int hq) {
        // dQ tile (TMEM lane = query row) from [128, 256): staged in the dS
        // buffer (free once the dQ product is done) as two rounds of two
        // 32-column boxes (128-byte swizzle), each added to the f32
        // accumulator by TMA reductions issued by one thread.
        const bool w3 =
            ok && mbar_wait(&bar[C::B_DQF], m & 1, kWaitBackward, m, 32);
        ok = named_sync_and(1, 128, __all_sync(FULL, w3));
        if (ok) {
          tc_fence_after();
#pragma unroll 1
          for (int h = 0; h < 4; ++h) {
            // four 32-column boxes through the buffer's two 16 KB halves:
            // a half is written again once the reduction of the box two
            // rounds back has read it
            const int half = h & 1;
            if (h >= 2) {
              if (warp == 2 && lane == 0) bulk_wait_read_but_one();
              named_sync(1, 128);
            }
            uint32_t a[32];
            tmem_ld32(lane_base + 128 + h * 32, a);
            tc_wait_ld();
            uint8_t* row = sDS + half * (C::TILE / 2) + rr * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4*>(row + ((c ^ (rr & 7)) * 16)) =
                  make_uint4(a[4 * c], a[4 * c + 1], a[4 * c + 2],
                             a[4 * c + 3]);
            if (h == 3) {  // TMEM [128, 256) is free for the next dP^T
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&bar[C::B_DQR]);
            }
            fence_async_smem();
            named_sync(1, 128);
            if (warp == 2 && lane == 0) {
              tma_reduce_add_3d(&p.tdq, sDS + half * (C::TILE / 2), h * 32,
                                i * 128, b * p.Hq + hq);
              bulk_commit_group();
            }
          }
        }
    };
    // One pair deep: P of pair n+1 runs while the tensor core does dK and
    // dQ of pair n, then pair n's dQ tile is read out.
    int g = 0, i = -1;
    bool have = next_kept(g, i);
    if (have) {
      ok = named_sync_and(1, 128, ok);
      p_phase(0, i);
    }
    while (have && ok) {
      d_phase(n);
      int g2 = g, i2 = i;
      const bool h2 = next_kept(g2, i2);
      if (h2) {
        // All four warps leave together: a wait that gave up in any of them
        // ends the loop for all at this barrier (never between barriers).
        if (!named_sync_and(1, 128, ok)) {
          ok = false;
          break;
        }
        p_phase(n + 1, i2);
      }
      e_phase(n, i, hkv * p.G + g);
      ++n;
      g = g2;
      i = i2;
      have = h2;
    }
    // dK_j, dV_j (TMEM lane = key row); zero when no pair was kept.  The
    // tensor-memory loads are warp-collective, so every lane takes part and
    // only the stores depend on the row (a warp can straddle the cache end).
    if (ok) {
      __nv_bfloat16* dvr = p.dv + ((size_t)bk * p.Lkv + key) * kBwdD;
      __nv_bfloat16* dkr = p.dk + ((size_t)bk * p.Lkv + key) * kBwdD;
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        const uint32_t col = half == 0 ? 256u : 384u;
        const float f = half == 0 ? 1.f : p.scale;
        __nv_bfloat16* out = half == 0 ? dvr : dkr;
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t a[32];
          if (n > 0) {
            tmem_ld32(lane_base + col + cc * 32, a);
            tc_wait_ld();
          } else {
#pragma unroll
            for (int x = 0; x < 32; ++x) a[x] = 0u;
          }
          if (key_ok) {
#pragma unroll
            for (int x = 0; x < 32; x += 8) {
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(a[x]) * f, __uint_as_float(a[x + 1]) * f);
              w.y = pack_bf16x2(__uint_as_float(a[x + 2]) * f, __uint_as_float(a[x + 3]) * f);
              w.z = pack_bf16x2(__uint_as_float(a[x + 4]) * f, __uint_as_float(a[x + 5]) * f);
              w.w = pack_bf16x2(__uint_as_float(a[x + 6]) * f, __uint_as_float(a[x + 7]) * f);
              *reinterpret_cast<uint4*>(out + cc * 32 + x) = w;
            }
          }
        }
      }
    }
  }

  if (warp == 2 && lane == 0) bulk_wait_all();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// 3-D map over the f32 dQ accumulator [planes, rows, 128], box 32 columns
// (128 bytes) x 128 rows, 128-byte swizzle; rows past the end are clipped.
inline bool encode_map_f32(CUtensorMap* m, void* base, int rows,
                           long long planes) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kBwdD, (cuuint64_t)rows,
                        (cuuint64_t)planes};
  cuuint64_t strides[2] = {(cuuint64_t)kBwdD * 4,
                           (cuuint64_t)rows * kBwdD * 4};
  cuuint32_t box[3] = {32, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

struct BwdProblem {
  const void *q, *k, *v, *o, *dout;
  const float* lse;
  const unsigned char* mask;
  void *dq, *dk, *dv;
  float* workspace;  // dQ accumulator [B*Hq*Lq*D] then D [B*Hq*Lq]
  int B, Hq, Hkv, Lq, Lkv, causal;
  float scale;
};

inline size_t bwd_workspace_bytes(int B, int Hq, int Lq) {
  const size_t rows = (size_t)B * Hq * Lq;
  const size_t prow = (size_t)B * Hq * ((Lq + 3) & ~3);
  // dQ accumulator, then D and lse * log2 e with 16-byte row strides
  return rows * kBwdD * 4 + 2 * (((prow + 63) & ~(size_t)63) * 4);
}

// [planes][cols] f32 with a 16-byte row stride, 128-column boxes of one row
inline bool encode_rows_f32(CUtensorMap* m, void* base, int cols,
                            long long planes) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)planes, 1};
  cuuint64_t strides[2] = {(cuuint64_t)cols * 4,
                           (cuuint64_t)planes * cols * 4};
  cuuint32_t box[3] = {128, 1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

inline cudaError_t launch_backward(const BwdProblem& pr, cudaStream_t st) {
  BwdParams p;
  memset(&p, 0, sizeof p);
  if (!encode_map(&p.tq, pr.q, kBwdD, pr.Lq, (long long)pr.B * pr.Hq, 128) ||
      !encode_map(&p.tdo, pr.dout, kBwdD, pr.Lq, (long long)pr.B * pr.Hq, 128) ||
      !encode_map(&p.tk, pr.k, kBwdD, pr.Lkv, (long long)pr.B * pr.Hkv, 128) ||
      !encode_map(&p.tv, pr.v, kBwdD, pr.Lkv, (long long)pr.B * pr.Hkv, 128))
    return cudaErrorInvalidValue;
  p.o = static_cast<const __nv_bfloat16*>(pr.o);
  p.dout = static_cast<const __nv_bfloat16*>(pr.dout);
  p.lse = pr.lse;
  p.mask = pr.mask;
  const size_t rows = (size_t)pr.B * pr.Hq * pr.Lq;
  p.Lqp = (pr.Lq + 3) & ~3;
  const size_t prow = (size_t)pr.B * pr.Hq * p.Lqp;
  p.dq_acc = pr.workspace;
  p.delta = pr.workspace + rows * kBwdD;
  p.lse2 = p.delta + ((prow + 63) & ~(size_t)63);
  if (!encode_map_f32(&p.tdq, p.dq_acc, pr.Lq, (long long)pr.B * pr.Hq) ||
      !encode_rows_f32(&p.tdel, p.delta, p.Lqp, (long long)pr.B * pr.Hq) ||
      !encode_rows_f32(&p.tlse2, p.lse2, p.Lqp, (long long)pr.B * pr.Hq))
    return cudaErrorInvalidValue;
  p.dq = static_cast<__nv_bfloat16*>(pr.dq);
  p.dk = static_cast<__nv_bfloat16*>(pr.dk);
  p.dv = static_cast<__nv_bfloat16*>(pr.dv);
  p.B = pr.B;
  p.Hq = pr.Hq;
  p.Hkv = pr.Hkv;
  p.Lq = pr.Lq;
  p.Lkv = pr.Lkv;
  p.nq = (pr.Lq + 127) / 128;
  p.nk = (pr.Lkv + 127) / 128;
  p.G = pr.Hq / pr.Hkv;
  p.causal = pr.causal;
  p.scale = pr.scale;
  const long long prep_blocks = (long long)((rows + 7) / 8);
  const long long grid = (long long)pr.B * pr.Hkv * p.nk;
  const long long conv_blocks = (long long)((rows * (kBwdD / 8) + 255) / 256);
  if (prep_blocks > 0x7fffffffLL || grid > 0x7fffffffLL ||
      conv_blocks > 0x7fffffffLL)
    return cudaErrorInvalidConfiguration;
  bwd_prep_kernel<<<(unsigned)prep_blocks, 256, 0, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // With a mask, the CTAs go out by kept pairs.  The counts and the order
  // (2 ints per slot) live in dq, which only the last kernel writes; the
  // order is skipped when dq is too small for them or the slots are many.
  const size_t dq_bytes = rows * kBwdD * 2;
  if (p.mask && grid <= kBwdOrderMaxSlots &&
      (size_t)grid * 2 * sizeof(int) <= dq_bytes) {
    p.counts = static_cast<int*>(pr.dq);
    int* order = p.counts + grid;
    bwd_count_kernel<<<(unsigned)((grid * 32 + 255) / 256), 256, 0, st>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    bwd_order_kernel<<<(unsigned)((grid + 255) / 256), 256, 0, st>>>(p, order);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    p.order = order;
  }
  e = cudaFuncSetAttribute(bwd_dkdv_kernel,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           BwdCfg::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  bwd_dkdv_kernel<<<(unsigned)grid, kBwdThreads, BwdCfg::SMEM_ALLOC, st>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  bwd_dq_kernel<<<(unsigned)conv_blocks, 256, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace blasst

// decode_mma.cuh -- BLASST decode with the scores and P.V on warp-level
// tensor-core instructions (mma.sync m16n8k16, bf16 in, f32 accumulate):
// contiguous or paged bf16 KV cache, G <= 8 query heads per KV head, head
// dimension 64 or 128, split-KV.
//
// Method as in decode.cuh ("BLASST: Dynamic BLocked Attention Sparsity via
// Softmax Thresholding", gist.science summary, section 2 "Criterio de Pulo"
// and "Acoes de Otimizacao", section 3: in the memory-bound decode the
// saving is the V blocks never loaded): per (sequence, KV head, split) the
// G heads are the rows of one tile, blocks of 64 keys in ascending order,
// block j skipped when every head's block max lies more than |ln lambda|
// below its running max, V read only for kept blocks, then the split
// partials are merged by log-sum-exp (decode_combine_kernel).
//
// Why this form: the decode is bound by HBM, and the CUDA-core scoring of a
// block (G x 64 x 128 FMAs plus the bf16 unpacking and the cross-lane
// reductions, ~350 instructions a thread) left each CTA ~4k cycles per block,
// far from the ~1k at which 3 CTAs per SM keep HBM busy when most V blocks
// are skipped.  Here a warp scores its 16 keys of the block with 16 MMAs fed
// by 8 ldmatrix loads, and the score fragment it holds is, after the exp,
// exactly the A fragment of its 16-key slice of P.V, so P never leaves
// registers.  A tcgen05 MMA would need the scores to go through tensor
// memory and a cross-warp hand-off on every block (the wide kernel pays that
// chain); at M = G <= 8 rows the warp-level instruction keeps the whole
// per-block chain inside each warp.
//
// CTA = 4 warps per (b, hkv, split); warp w owns keys 16w .. 16w+15 of each
// block.  K and V blocks arrive by TMA as two 64-column boxes with the
// 128-byte swizzle (ldmatrix reads are then free of bank conflicts): a K
// ring of two blocks and a V ring of two.  The P.V of a kept block runs
// when the next kept block has been decided (its V load has had a block of
// scoring to land); its P and rescale factor wait in registers.
//
// Paged cache (PAGED): the page pool [num_pages][Hkv][page_size][d] is a
// tensor map whose box is min(page_size, 64) rows of one page, so a 64-key
// block is one to four TMA segments, each from the page the block table
// names.  At d = 128 the map is 5-D (64 columns, 2 halves, rows, heads,
// pages) and one copy brings a segment's whole 256-byte rows, stored row by
// row in shared memory; at d = 64 it is 4-D with one 64-column box.  Every page id a split will read is range-checked before the
// first load (a bad id or length sets the error word and the CTA leaves).
// Rows past the sequence's end that a segment brings in (the rest of its
// last page) or that no segment covers are masked in the scores and zeroed
// in V before the P.V, so whatever the pool holds there cannot reach o.
#pragma once

#include "decode.cuh"
#include "prefill.cuh"

namespace blasst {

struct DecodeMmaArgs {
  CUtensorMap tk, tv;        // [B*Hkv][Lkv][d] bf16, box 64 cols x 64 rows
  const __nv_bfloat16* q;    // [B, Hq, d]
  float* o_part;             // [B*Hq, S, d]
  float* lse_part;           // [B*Hq, S]
  unsigned long long* counters;
  unsigned char* mask;       // [B*Hkv, nk]
  float* margin;             // [B*Hkv, nk] decision margins (may be null)
  int Hkv, Lkv, nk, S;
  float scale, ln_lambda;
  int stats_only;
  int window;                // the last `window` keys (0 = all)
  // paged cache only (tk / tv then map the pools, see above)
  const int* block_table;    // [B, max_pages]
  const int* seq_lens;       // [B]; Lkv is then the upper bound on them
  int max_pages, num_pages, log2_page;
  int per_length;  // ln_lambda is ln a; sequence b uses min(0, ln a - ln L_b)
  const int* order;  // paged: sequence of each grid slot (NULL: slot b is b)
};

struct DecodeMmaCfg {
  static constexpr int BOX = 64 * 128;      // 64 rows x 128 bytes (64 dims)
  static constexpr int TILE = 2 * BOX;      // slot: 64 keys x up to 128 dims
  static constexpr int NK = 2, NV = 2;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + NK * TILE;
  static constexpr int OFF_M = OFF_V + NV * TILE;  // f32 [2][2][8 heads][4 warps]
  static constexpr int OFF_L = OFF_M + 2 * 2 * 8 * 4 * 4;  // f32 [4 warps][8]
  static constexpr int OFF_BAR = OFF_L + 4 * 8 * 4;    // u64 [NK + NV]
  static constexpr int SMEM = OFF_BAR + (NK + NV) * 8;
  static constexpr int SMEM_ALLOC = SMEM + 1024;  // 1024-byte alignment
  static_assert(4 * 8 * 128 * 4 <= NK * TILE, "reduction fits the K ring");
};

// D = A * B + C for one 16 x 8 x 16 step; rows 8..15 of A are zero (at most
// 8 heads), so only D rows 0..7 (d0, d1) are kept.
__device__ __forceinline__ void mma16816_top(float& d0, float& d1, uint32_t a0,
                                             uint32_t a2, uint32_t b0,
                                             uint32_t b1) {
  [[maybe_unused]] float x2, x3;  // rows 8..15 of D: always zero, unused
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%11,%12,%13};"
      : "=f"(d0), "=f"(d1), "=f"(x2), "=f"(x3)
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1), "f"(d0),
        "f"(d1), "f"(0.f), "f"(0.f));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0,
                                        uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile(
      "ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
      : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
      : "r"(addr)
      : "memory");
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0,
                                          uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile(
      "ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
      : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
      : "r"(addr)
      : "memory");
}

__device__ __forceinline__ void tma_load_4d(void* dst_smem, const void* tmap,
                                            uint64_t* bar, int c0, int c1,
                                            int c2, int c3, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_"
      "tx::bytes.L2::cache_hint [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(
          smem_u32(dst_smem)),
      "l"(tmap), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar)),
      "l"(policy)
      : "memory");
}

__device__ __forceinline__ void tma_load_5d(void* dst_smem, const void* tmap,
                                            uint64_t* bar, int c0, int c1,
                                            int c2, int c3, int c4,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_"
      "tx::bytes.L2::cache_hint [%0], [%1, {%2, %3, %4, %5, %6}], [%7], %8;" ::"r"(
          smem_u32(dst_smem)),
      "l"(tmap), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(smem_u32(bar)),
      "l"(policy)
      : "memory");
}

// Byte offset of the 16-byte chunk `chunk` (0..15: dims 8*chunk ..) of key
// row `key` in a block stored as two 64-column boxes with the 128-byte
// swizzle (chunk index XOR key % 8 within each 1024-byte group of rows).
__device__ __forceinline__ uint32_t swz_off(int key, int chunk) {
  return (uint32_t)((chunk >> 3) * DecodeMmaCfg::BOX + key * 128 +
                    (((chunk & 7) ^ (key & 7)) << 4));
}

// The same for a block stored row by row (paged cache, d = 128): key row
// `key` is 256 bytes, its two 64-column halves two consecutive 128-byte
// lines, and the 128-byte swizzle XORs the chunk with the line index % 8.
__device__ __forceinline__ uint32_t swz_off_rows(int key, int chunk) {
  const int line = 2 * key + (chunk >> 3);
  return (uint32_t)(line * 128 + (((chunk & 7) ^ (line & 7)) << 4));
}

// BATCH = 2: the batched decision rule (contiguous cache): blocks r and
// r+1 are scored before either is decided, and each is judged against
// Mb = max(running max before r, maxima of both blocks); kept blocks use Mb
// as the reference of P.  (A skip never moves the running max, so the
// running max is always the reference of O and l, in both rules.)
template <int G, int D, bool PAGED, int BATCH = 1>
__global__ void __launch_bounds__(kDecThreads, 3)
    decode_mma_kernel(const __grid_constant__ DecodeMmaArgs a) {
  static_assert(G >= 1 && G <= 8, "at most 8 heads per tile");
  static_assert(BATCH == 1 || (BATCH == 2 && !PAGED), "pairs: contiguous");
  static_assert(D == 64 || D == 128, "head dimension 64 or 128");
  constexpr int NBOX = D / 64;     // 64-column boxes per block
  // paged d = 128: a segment's rows arrive whole (both halves) in one copy
  constexpr bool ROWS = PAGED && NBOX == 2;
  auto kv_off = [](int key, int chunk) {
    if constexpr (ROWS) return swz_off_rows(key, chunk);
    else return swz_off(key, chunk);
  };
  constexpr int KST = D / 16;      // k-steps of the scores
  constexpr int NG = D / 8;        // 8-column groups of the output
  using C = DecodeMmaCfg;
  constexpr unsigned FULL = 0xffffffffu;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;

  const int s = blockIdx.x % a.S;
  const int slot = blockIdx.x / a.S;  // sequence slot * Hkv + hkv
  const int Hq = a.Hkv * G;
  const int hkv = slot % a.Hkv;
  int b = slot / a.Hkv;
  if constexpr (PAGED) {
    if (a.order) b = __ldg(a.order + b);
  }
  const int bh = b * a.Hkv + hkv;
  int Lb = a.Lkv;  // keys of this sequence
  float ln_lambda = a.ln_lambda;
  const int* bt_row = nullptr;
  if constexpr (PAGED) {
    Lb = __ldg(a.seq_lens + b);
    if (Lb < 0 || Lb > a.Lkv) {  // uniform across the CTA
      if (tid == 0) record_error(kBadSeqLen, (unsigned)b, (unsigned)Lb, 0);
      return;
    }
    // lambda = a / L with L this sequence's own context length
    if (a.per_length && ln_lambda > -INFINITY && Lb > 0)
      ln_lambda = fminf(0.f, ln_lambda - logf((float)Lb));
    bt_row = a.block_table + (size_t)b * a.max_pages;
  }
  const int nk_b = (Lb + kDecBc - 1) / kDecBc;
  const int key_lo = (a.window > 0 && Lb > a.window) ? Lb - a.window : 0;
  const int jlo = key_lo / kDecBc;
  const int j0 = jlo + (int)(((long long)s * (nk_b - jlo)) / a.S);
  const int j1 = jlo + (int)(((long long)(s + 1) * (nk_b - jlo)) / a.S);
  const int nblk = j1 - j0;
  const int ps = 1 << a.log2_page;       // paged: rows per page
  const int seg = ps < 64 ? ps : 64;     // paged: rows per TMA segment
  if constexpr (PAGED) {
    // every page id this split reads, before any load
    bool bad = false;
    const int t0 = j0 * kDecBc, t1 = min(j1 * kDecBc, Lb);
    if (t1 > t0)
      for (int pg = (t0 >> a.log2_page) + tid; pg <= ((t1 - 1) >> a.log2_page);
           pg += kDecThreads) {
        const int id = __ldg(bt_row + pg);
        if (id < 0 || id >= a.num_pages) {
          bad = true;
          record_error(kBadPageId, (unsigned)b, (unsigned)pg, (unsigned)id);
        }
      }
    if (__syncthreads_or(bad)) return;
  }
  if (a.mask && s == 0)  // blocks left of the window are not visited
    for (int j = tid; j < jlo; j += kDecThreads) a.mask[(size_t)bh * a.nk + j] = 0;

  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  float* sM = reinterpret_cast<float*>(smem + C::OFF_M);
  float* sL = reinterpret_cast<float*>(smem + C::OFF_L);
  uint64_t* kfull = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* vfull = kfull + C::NK;
  const bool stats_only = a.stats_only != 0;

  if (tid == 0) {
    for (int i = 0; i < C::NK; ++i) mbar_init(&kfull[i], 1);
    for (int i = 0; i < C::NV; ++i) mbar_init(&vfull[i], 1);
    fence_mbar_init();
  }
  __syncthreads();

  const uint64_t pol = policy_evict_first();
  auto load = [&](const CUtensorMap* map, uint8_t* dst, uint64_t* bar, int j) {
    if constexpr (!PAGED) {
      mbar_arrive_expect_tx(bar, NBOX * C::BOX);
#pragma unroll
      for (int c = 0; c < NBOX; ++c)
        tma_load_3d(dst + c * C::BOX, map, bar, c * 64, j * kDecBc, bh, pol);
    } else {
      // segments of `seg` rows that hold the block's keys (< Lb)
      const int rows = min(kDecBc, Lb - j * kDecBc);
      const int nseg = (rows + seg - 1) / seg;
      mbar_arrive_expect_tx(bar, (uint32_t)(nseg * seg * 128 * NBOX));
      for (int i = 0; i < nseg; ++i) {
        const int t = j * kDecBc + i * seg;
        const int id = __ldg(bt_row + (t >> a.log2_page));
        if constexpr (ROWS) {
          tma_load_5d(dst + i * seg * 256, map, bar, 0, 0, t & (ps - 1), hkv,
                      id, pol);
        } else {
#pragma unroll
          for (int c = 0; c < NBOX; ++c)
            tma_load_4d(dst + c * C::BOX + i * seg * 128, map, bar, c * 64,
                        t & (ps - 1), hkv, id, pol);
        }
      }
    }
  };
  if (tid == 0) {
    prefetch_tmap(&a.tk);
    prefetch_tmap(&a.tv);
    for (int r = 0; r < nblk && r < C::NK; ++r)
      load(&a.tk, sK + r * C::TILE, &kfull[r], j0 + r);
  }

  // A fragments of q (rows = heads; head h = lane / 4, zero for h >= G),
  // k-step t covers dims 16t .. 16t+15: qa[t][0] dims 16t + 2(lane%4) + {0,1},
  // qa[t][1] the same + 8.
  const int hr = lane >> 2;  // this lane's head (fragment row)
  const int q4 = lane & 3;
  uint32_t qa[KST][2];
  {
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
        a.q + ((size_t)b * Hq + hkv * G + (hr < G ? hr : 0)) * D);
#pragma unroll
    for (int t = 0; t < KST; ++t) {
      qa[t][0] = hr < G ? __ldg(qrow + 8 * t + q4) : 0u;
      qa[t][1] = hr < G ? __ldg(qrow + 8 * t + 4 + q4) : 0u;
    }
  }

  // ldmatrix row addresses: lane l serves row l % 8 of matrix l / 8.
  //  scores (K, no transpose): matrix m = chunk 2p + m of keys 16w + 8g + l%8
  //  P.V (V, transposed): matrix m = keys 16w + 8(m&1) + l%8, chunk 2p + m/2
  const int mi = lane >> 3, mr = lane & 7;
  const uint32_t aK = smem_u32(sK), aV = smem_u32(sV);

  float o[NG][2];  // O of head hr, dims 8n + 2 q4 + {0,1}
#pragma unroll
  for (int n = 0; n < NG; ++n) o[n][0] = o[n][1] = 0.f;
  float m_run[G];  // running max of each head (replicated in every thread)
#pragma unroll
  for (int g = 0; g < G; ++g) m_run[g] = -INFINITY;
  float l_part = 0.f;  // this lane's part of the normaliser of head hr
  // the kept block waiting for its P.V
  bool pend = false;
  uint32_t pp0 = 0, pp1 = 0;  // its P as A fragment (keys 16w + 2q4 (+8))
  float palpha = 1.f;          // its rescale factor for head hr
  int prows = kDecBc;          // its keys inside the sequence
  int kept = 0;                // kept blocks so far (V slot = index % 2)

  const float scale = a.scale;
  unsigned long long n_vis = 0, n_skp = 0;
  bool ok = true;

  auto pv = [&](int kidx) -> bool {
    const int slot = kidx % C::NV;
    if (!mbar_wait(&vfull[slot], (uint32_t)(kidx / C::NV) & 1u, kWaitDecodeV,
                   kidx, slot))
      return false;
#pragma unroll
    for (int n = 0; n < NG; ++n) {
      o[n][0] *= palpha;
      o[n][1] *= palpha;
    }
    const uint32_t vb = aV + slot * C::TILE;
    if (PAGED && prows < kDecBc) {
      // rows past the sequence end: zero this warp's share (16 rows) so
      // that P = 0 there multiplies zeros, whatever the pool held
      uint8_t* vs = sV + slot * C::TILE;
      for (int e = lane; e < 16 * NBOX * 8; e += 32) {
        const int row = 16 * warp + e / (NBOX * 8);
        const int c16 = e % (NBOX * 8);  // 16-byte chunk of the row
        // (every chunk of the row, so the swizzle order does not matter)
        const int off = ROWS ? row * 256 + c16 * 16
                             : (c16 >> 3) * C::BOX + row * 128 + (c16 & 7) * 16;
        if (row >= prows)
          *reinterpret_cast<uint4*>(vs + off) = make_uint4(0, 0, 0, 0);
      }
      fence_async_smem();  // before a later TMA load overwrites the slot
      __syncwarp();
    }
#pragma unroll
    for (int p = 0; p < NG / 2; ++p) {
      uint32_t r0, r1, r2, r3;
      ldsm_x4_t(vb + kv_off(16 * warp + 8 * (mi & 1) + mr, 2 * p + (mi >> 1)),
                r0, r1, r2, r3);
      mma16816_top(o[2 * p][0], o[2 * p][1], pp0, pp1, r0, r1);
      mma16816_top(o[2 * p + 1][0], o[2 * p + 1][1], pp0, pp1, r2, r3);
    }
    return true;
  };

  // Scores of this warp's 16 keys of block r of the split (sc[g][i] = key
  // 16w + 8g + 2q4 + i, scaled, -inf where hidden); returns the block max of
  // head hr over the warp's keys.
  auto score = [&](int r, float (&sc)[2][2]) -> float {
    const int j = j0 + r;
    const int stage = r % C::NK;
    if (!mbar_wait(&kfull[stage], (uint32_t)(r / C::NK) & 1u, kWaitDecodeK, r,
                   stage))
      ok = false;
    sc[0][0] = sc[0][1] = sc[1][0] = sc[1][1] = 0.f;
    if (ok) {
      const uint32_t kb = aK + stage * C::TILE;
#pragma unroll
      for (int p = 0; p < KST / 2; ++p) {  // k-steps 2p, 2p+1 (chunks 4p .. 4p+3)
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          uint32_t r0, r1, r2, r3;
          ldsm_x4(kb + kv_off(16 * warp + 8 * g + mr, 4 * p + mi), r0, r1, r2,
                  r3);
          mma16816_top(sc[g][0], sc[g][1], qa[2 * p][0], qa[2 * p][1], r0, r1);
          mma16816_top(sc[g][0], sc[g][1], qa[2 * p + 1][0], qa[2 * p + 1][1],
                       r2, r3);
        }
      }
    }
    const int kbase = j * kDecBc + 16 * warp + 2 * q4;
    float mx = -INFINITY;
#pragma unroll
    for (int g = 0; g < 2; ++g)
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int key = kbase + 8 * g + i;
        sc[g][i] = (key < Lb && key >= key_lo) ? sc[g][i] * scale : -INFINITY;
        mx = fmaxf(mx, sc[g][i]);
      }
    mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 1));
    return fmaxf(mx, __shfl_xor_sync(FULL, mx, 2));
  };
  // Statistics, mask and margin of block j (thread 0).
  auto record = [&](int j, bool skip, const float (&mt)[G], const float (&mref)[G]) {
    if (tid == 0) {
      ++n_vis;
      if (skip) ++n_skp;
      if (a.mask) a.mask[(size_t)bh * a.nk + j] = skip ? 2 : 1;
      if (a.margin) {  // max over the heads of m~ - m (+inf while m = -inf)
        float dl = -INFINITY;
#pragma unroll
        for (int g = 0; g < G; ++g) dl = fmaxf(dl, mt[g] - mref[g]);
        a.margin[(size_t)bh * a.nk + j] = dl - ln_lambda;
      }
    }
  };
  // A kept block: its V load, the previous kept block's P.V (its V has had
  // at least this block's scoring to land), then this block's P against
  // the new reference mn of head hr (mo the old one).
  auto keep = [&](int j, const float (&sc)[2][2], float mo, float mn) {
    if (tid == 0) load(&a.tv, sV + (kept % C::NV) * C::TILE, &vfull[kept % C::NV], j);
    if (pend && !pv(kept - 1)) ok = false;
    const float al = (mo == -INFINITY) ? 0.f : ex2_approx((mo - mn) * kLog2e);
    const float mb = mn * kLog2e;
    float p[2][2];
#pragma unroll
    for (int g = 0; g < 2; ++g)
#pragma unroll
      for (int i = 0; i < 2; ++i) p[g][i] = ex2_approx(fmaf(sc[g][i], kLog2e, -mb));
    l_part = al * l_part + ((p[0][0] + p[0][1]) + (p[1][0] + p[1][1]));
    pp0 = pack_bf16x2(p[0][0], p[0][1]);
    pp1 = pack_bf16x2(p[1][0], p[1][1]);
    palpha = al;
    prows = min(kDecBc, Lb - j * kDecBc);
    pend = true;
    ++kept;
  };
  // head hr's entry of a per-head array (head 0's for padding rows)
  auto mine = [&](const float (&x)[G]) {
    float v = x[0];
#pragma unroll
    for (int g = 1; g < G; ++g)
      if (g == hr) v = x[g];
    return v;
  };

  if constexpr (BATCH == 1) {
  for (int r = 0; r < nblk; ++r) {
    const int j = j0 + r;
    const int stage = r % C::NK;
    float sc[2][2];
    const float mx = score(r, sc);
    float* sMr = sM + (r & 1) * 32;  // [head][warp], double-buffered
    if (q4 == 0 && hr < G) sMr[hr * 4 + warp] = mx;
    if (__syncthreads_or(!ok)) { ok = false; break; }
    // every warp has read K slot `stage`: refill it
    if (tid == 0 && r + C::NK < nblk)
      load(&a.tk, sK + stage * C::TILE, &kfull[stage], j + C::NK);

    // ---- decision (the same in every thread)
    float mt[G];
    bool skip = ln_lambda > -INFINITY;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float4 w4 = *reinterpret_cast<const float4*>(sMr + g * 4);
      mt[g] = fmaxf(fmaxf(w4.x, w4.y), fmaxf(w4.z, w4.w));
      if (!(mt[g] - m_run[g] < ln_lambda)) skip = false;
    }
    record(j, skip, mt, m_run);
    if (!skip && !stats_only) {
      const float mo = mine(m_run);
      keep(j, sc, mo, fmaxf(mo, mine(mt)));
    }
#pragma unroll
    for (int g = 0; g < G; ++g) m_run[g] = fmaxf(m_run[g], mt[g]);
    if (__any_sync(FULL, !ok)) { ok = false; }
  }
  } else {
  for (int r = 0; r < nblk; r += 2) {
    const bool two = r + 1 < nblk;
    float sc0[2][2], sc1[2][2];
    float* sMp = sM + ((r >> 1) & 1) * 64;  // [block of the pair][head][warp]
    const float mx0 = score(r, sc0);
    if (q4 == 0 && hr < G) sMp[hr * 4 + warp] = mx0;
    if (two) {
      const float mx1 = score(r + 1, sc1);
      if (q4 == 0 && hr < G) sMp[32 + hr * 4 + warp] = mx1;
    }
    if (__syncthreads_or(!ok)) { ok = false; break; }
    // both K slots have been read: refill them
    if (tid == 0) {
      if (r + 2 < nblk) load(&a.tk, sK + (r % C::NK) * C::TILE, &kfull[r % C::NK], j0 + r + 2);
      if (r + 3 < nblk)
        load(&a.tk, sK + ((r + 1) % C::NK) * C::TILE, &kfull[(r + 1) % C::NK], j0 + r + 3);
    }
    float mt0[G], mt1[G], Mb[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float4 w0 = *reinterpret_cast<const float4*>(sMp + g * 4);
      mt0[g] = fmaxf(fmaxf(w0.x, w0.y), fmaxf(w0.z, w0.w));
      if (two) {
        const float4 w1 = *reinterpret_cast<const float4*>(sMp + 32 + g * 4);
        mt1[g] = fmaxf(fmaxf(w1.x, w1.y), fmaxf(w1.z, w1.w));
      } else {
        mt1[g] = -INFINITY;
      }
      Mb[g] = fmaxf(m_run[g], fmaxf(mt0[g], mt1[g]));
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (u == 1 && !two) break;
      const int j = j0 + r + u;
      bool skip = ln_lambda > -INFINITY;
#pragma unroll
      for (int g = 0; g < G; ++g)
        if (!((u ? mt1[g] : mt0[g]) - Mb[g] < ln_lambda)) skip = false;
      record(j, skip, u ? mt1 : mt0, Mb);
      if (!skip && !stats_only) {
        keep(j, u ? sc1 : sc0, mine(m_run), mine(Mb));
#pragma unroll
        for (int g = 0; g < G; ++g) m_run[g] = Mb[g];  // the new reference
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) m_run[g] = Mb[g];
    if (__any_sync(FULL, !ok)) { ok = false; }
  }
  }
  if (ok && pend && !pv(kept - 1)) ok = false;
  if (__syncthreads_or(!ok)) ok = false;

  if (!ok) {
    // outstanding copies get a bounded chance to land before the shared
    // memory is released
    if (tid == 0) {
      for (int i = 0; i < C::NK; ++i)
        mbar_wait(&kfull[i], 0, kWaitDecodeDrain, i, 0, 1000000);
      for (int i = 0; i < C::NV; ++i)
        mbar_wait(&vfull[i], 0, kWaitDecodeDrain, i, 1, 1000000);
    }
    return;
  }
  if (tid == 0 && a.counters) {
    atomicAdd(&a.counters[0], n_vis);
    atomicAdd(&a.counters[1], n_skp);
  }
  if (stats_only) return;

  // normaliser: the 4 lanes of a head in this warp, then the 4 warps
  {
    float x = l_part;
    x += __shfl_xor_sync(FULL, x, 1);
    x += __shfl_xor_sync(FULL, x, 2);
    if (q4 == 0 && hr < G) sL[warp * 8 + hr] = x;
  }
  // per-warp outputs [warp][head][dim] in the (now idle) K ring
  float* red = reinterpret_cast<float*>(sK);
  if (hr < G) {
#pragma unroll
    for (int n = 0; n < NG; ++n)
      *reinterpret_cast<float2*>(red + ((warp * 8 + hr) * D + 8 * n + 2 * q4)) =
          make_float2(o[n][0], o[n][1]);
  }
  __syncthreads();
  if (tid < D) {
    const int dd = tid;  // one thread per output column
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float sum = red[(0 * 8 + g) * D + dd] + red[(1 * 8 + g) * D + dd] +
                        red[(2 * 8 + g) * D + dd] + red[(3 * 8 + g) * D + dd];
      const float l = sL[g] + sL[8 + g] + sL[16 + g] + sL[24 + g];
      const size_t row = (size_t)b * Hq + hkv * G + g;
      a.o_part[(row * a.S + s) * D + dd] = l > 0.f ? sum / l : 0.f;
      if (dd == 0)
        a.lse_part[row * a.S + s] = l > 0.f ? m_run[g] + __logf(l) : -INFINITY;
    }
  }
}

}  // namespace blasst

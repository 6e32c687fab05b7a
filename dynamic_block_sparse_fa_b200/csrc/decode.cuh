// decode.cuh -- BLASST decode forward: one query token per sequence against a
// contiguous bf16 KV cache, split-KV, GQA head packing, V read only for kept
// blocks, then a log-sum-exp merge of the splits.
//
// Method: "BLASST: Dynamic BLocked Attention Sparsity via Softmax
// Thresholding" (gist.science summary, section 2 "Criterio de Pulo" and
// "Acoes de Otimizacao"; section 3: in the memory-bound decode the saving is
// the V blocks never loaded from HBM).  The Hindi summary (section 2, kernel
// optimisation) notes that conditional V loads cause pipeline bubbles unless
// several Q.K products are scored before deciding which V blocks to fetch;
// here K runs a fixed number of blocks ahead of the decisions and the P.V
// product of a kept block runs a fixed number of kept blocks behind its V
// load, so the loads of the decided blocks are in flight while later blocks
// are scored.  The decision for block j still uses the running max over the
// blocks before j (the order of the blockwise algorithm is unchanged).
//
// One CTA of 128 threads per (sequence b, KV head, split).  The G query
// heads of the KV head are the rows of the tile: every K and V byte fetched
// serves G heads.  K and V blocks (Bc = 64 keys x d = 128 = 16 KB) arrive
// through bulk asynchronous copies into shared memory and are read back with
// 128-bit shared loads.
//
// Two cache forms share the kernel.  Contiguous: [B, Hkv, Lkv, d], one copy
// per block.  Paged: a pool of pages of page_size tokens, page p of KV head
// h at p * page_stride + h * page_size * d, a block table per sequence and a
// length per sequence (device-resident); a block is one copy when pages hold
// 64 tokens or more, else one copy per page.
#pragma once

#include "ptx.cuh"

namespace blasst {

struct DecodeArgs {
  const __nv_bfloat16* q;  // [B, Hq, D]
  const __nv_bfloat16* k;  // [B, Hkv, Lkv, D]
  const __nv_bfloat16* v;  // [B, Hkv, Lkv, D]
  float* o_part;           // [B*Hq, S, D]  normalised split outputs
  float* lse_part;         // [B*Hq, S]
  unsigned long long* counters;  // [2] visited, skipped (may be null)
  unsigned char* mask;           // [B*Hkv, nk] (may be null)
  int Hkv, Lkv, nk, S;  // paged: Lkv = upper bound on the lengths
  float scale, ln_lambda;
  int stats_only;
  // paged cache only
  const int* block_table;  // [B, max_pages]
  const int* seq_lens;     // [B]
  long long page_stride;   // elements
  int log2_page, max_pages, num_pages;
  int per_length;  // ln_lambda is ln a; sequence b uses min(0, ln a - ln L_b)
  // paged: the sequence decoded by each slot of the grid (NULL: slot b is
  // sequence b), from decode_order_kernel
  const int* order;
  // sliding window: the token sees only the last `window` keys (0 = all);
  // the splits divide the blocks that hold them
  int window;
  // decode tiles per KV head of the cache (>= 1): with G query heads per KV
  // head above the tile's rows, the heads are cut into kv_div tiles of G /
  // kv_div heads; Hkv then counts tiles (cache heads * kv_div)
  int kv_div;
};

constexpr int kDecD = 128;       // head dimension
constexpr int kDecBc = 64;       // keys per block
constexpr int kDecThreads = 128;
// Resident CTAs per SM the kernel is sized for (shared memory: 3 for G <= 4,
// registers: 2 for G = 8).  The sequential kernel's launch bound asks for 2:
// for G <= 4 that lets the compiler use up to ~168 registers (measured 3-4%
// faster than capping it for 3 blocks), which still leaves 3 CTAs resident;
// the batched kernel (more live scores) keeps the bound of 3.
template <int G>
constexpr int dec_ctas_per_sm() { return G >= 8 ? 2 : 3; }
constexpr int kDecLaunchMinBlocks = 2;
constexpr int kDecNK = 2;        // K blocks staged (one ahead of the scoring)
constexpr int kDecNV = 2;        // V block slots
constexpr int kDecLag = 1;       // P.V of kept block n runs once n+Lag+1 are issued
static_assert(kDecNV >= kDecLag + 1, "V ring must cover the lag");
constexpr int kDecBlockBytes = kDecBc * kDecD * 2;  // 16 KB
constexpr int kDecRowBytes = kDecD * 2;             // 256 B per key

template <int G>
struct DecodeSmem {
  static constexpr int kK = 0;                                  // [NK][Bc][D] bf16
  static constexpr int kV = kK + kDecNK * kDecBlockBytes;        // [NV][Bc][D] bf16
  static constexpr int kP = kV + kDecNV * kDecBlockBytes;        // [NV][Bc][G] f32
  static constexpr int kM = kP + kDecNV * kDecBc * G * 4;        // [4][4 warps][8] f32
  static constexpr int kA = kM + 4 * 4 * 8 * 4;                  // [NV][8] f32
  static constexpr int kL = kA + kDecNV * 8 * 4;                 // [4 warps][8] f32
  static constexpr int kNV = kL + 4 * 8 * 4;                     // [NV] int
  // paged cache, 2 chunks of 32 blocks, up to 4 copies a block: element
  // offsets of each copy's source in the pool, and the page ids they are
  // computed from
  static constexpr int kOff = (kNV + kDecNV * 4 + 7) & ~7;       // [64][4] i64
  static constexpr int kPid = kOff + 64 * 4 * 8;                 // [64][4] int
  static constexpr int kBar = (kPid + 64 * 4 * 4 + 15) & ~15;    // [NK+NV] u64
  static constexpr int kTotal = kBar + (kDecNK + kDecNV) * 8;
  // The end-of-split reduction [8 key groups][G][D] f32 reuses the K and V
  // rings (all copies into them have been consumed by then).
  static_assert(8 * G * kDecD * 4 <= kP, "reduction fits in the rings");
  static_assert(dec_ctas_per_sm<G>() * (kTotal + 1024) <= 228 * 1024,
                "shared memory for the intended residency");
};

constexpr float kLog2e = 1.4426950408889634f;

// Sum over the 8 lanes that share a key (lane bits 0..2) of G partial dot
// products.  While more than one value is held, each exchange step keeps half
// of the values and sends the other half, so the lane ends up holding the
// full sum of head  head_of_lane<G>(lane).
template <int G>
__device__ __forceinline__ float reduce8_transpose(float (&v)[G], int lane) {
  float x[G];
#pragma unroll
  for (int g = 0; g < G; ++g) x[g] = v[g];
  int n = G;
#pragma unroll
  for (int msk = 4; msk >= 1; msk >>= 1) {
    if (n > 1) {
      const int h = n / 2;
      const bool upper = (lane & msk) != 0;
#pragma unroll
      for (int i = 0; i < G / 2; ++i) {
        if (i < h) {
          float send = upper ? x[i] : x[i + h];
          float keep = upper ? x[i + h] : x[i];
          x[i] = keep + __shfl_xor_sync(0xffffffffu, send, msk);
        }
      }
      n = h;
    } else {
      x[0] += __shfl_xor_sync(0xffffffffu, x[0], msk);
    }
  }
  return x[0];
}

template <int G>
__device__ __forceinline__ int head_of_lane(int lane) {
  int h = 0, n = G;
#pragma unroll
  for (int msk = 4; msk >= 1; msk >>= 1) {
    if (n > 1) {
      n /= 2;
      if (lane & msk) h += n;
    }
  }
  return h;
}

template <int G, bool PAGED, int BATCH = 1>
__global__ void __launch_bounds__(kDecThreads, BATCH == 1
                                                   ? kDecLaunchMinBlocks
                                                   : dec_ctas_per_sm<G>())
    decode_split_kernel(const DecodeArgs a) {
  using L = DecodeSmem<G>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;

  const int s = blockIdx.x % a.S;
  const int slot = blockIdx.x / a.S;  // sequence slot * Hkv + hkv (tiles)
  const int Hq = a.Hkv * G;
  const int hkv = slot % a.Hkv;
  int b = slot / a.Hkv;
  if constexpr (PAGED) {
    if (a.order) b = __ldg(a.order + b);
  }
  const int bh = b * a.Hkv + hkv;
  const int hkv_c = hkv / a.kv_div;  // the cache head of this tile
  int Lb = a.Lkv;  // keys of this sequence
  float ln_lambda = a.ln_lambda;
  if constexpr (PAGED) {
    Lb = __ldg(a.seq_lens + b);
    if (Lb < 0 || Lb > a.Lkv) {  // uniform across the CTA
      if (tid == 0) record_error(kBadSeqLen, (unsigned)b, (unsigned)Lb, 0);
      return;
    }
    // lambda = a / L with L this sequence's own context length
    if (a.per_length && ln_lambda > -INFINITY && Lb > 0)
      ln_lambda = fminf(0.f, ln_lambda - logf((float)Lb));
  }
  const int nk_b = (Lb + kDecBc - 1) / kDecBc;
  // first visible key and its block (sliding window)
  const int key_lo = (a.window > 0 && Lb > a.window) ? Lb - a.window : 0;
  const int jlo = key_lo / kDecBc;
  const int j0 = jlo + (int)(((long long)s * (nk_b - jlo)) / a.S);
  const int j1 = jlo + (int)(((long long)(s + 1) * (nk_b - jlo)) / a.S);
  const int nblk = j1 - j0;
  if (a.mask && s == 0)  // blocks left of the window are not visited
    for (int j = tid; j < jlo; j += kDecThreads) a.mask[(size_t)bh * a.nk + j] = 0;
  // Paged cache: a block of 64 keys is npb copies of 2^seg_l2 rows, each
  // from one page.  The source offsets of the copies of blocks r (relative
  // to j0) are kept in a shared ring sOff[r mod 64][copy], filled 32 blocks
  // ahead, so the thread that issues a copy reads a ready address.
  long long* sOff = reinterpret_cast<long long*>(smem + L::kOff);
  int* sPid = reinterpret_cast<int*>(smem + L::kPid);
  const int* bt_row = nullptr;
  const int seg_l2 = a.log2_page < 6 ? a.log2_page : 6;
  const int npb = 1 << (6 - seg_l2);
  // element offset of the copy of block r (relative) that starts at token
  // tok, in page id
  auto src_off = [&](int id, int tok) -> long long {
    return (long long)id * a.page_stride +
           ((long long)hkv_c << (a.log2_page + 7)) +
           (long long)(tok & ((1 << a.log2_page) - 1)) * kDecD;
  };
  if constexpr (PAGED) {
    // Every page id this split will read is checked before its first copy;
    // the copies of its first 64 blocks go into the ring.
    bt_row = a.block_table + (size_t)b * a.max_pages;
    bool bad = false;
    for (int e = tid; e < 64 * 4; e += kDecThreads) {
      const int r = e >> 2, i = e & 3;
      const int tok = (j0 + r) * kDecBc + (i << seg_l2);
      if (r < nblk && i < npb && tok < Lb) {
        const int p = tok >> a.log2_page;
        const int id = __ldg(bt_row + p);
        if (id < 0 || id >= a.num_pages) {
          bad = true;
          record_error(kBadPageId, (unsigned)b, (unsigned)p, (unsigned)id);
        }
        sOff[e] = src_off(id, tok);
      }
    }
    const int t0 = (j0 + min(nblk, 64)) * kDecBc;
    const int t1 = min(j1 * kDecBc, Lb);
    if (t1 > t0) {
      const int p1 = ((t1 - 1) >> a.log2_page) + 1;
      for (int p = (t0 >> a.log2_page) + tid; p < p1; p += kDecThreads) {
        const int id = __ldg(bt_row + p);
        if (id < 0 || id >= a.num_pages) {
          bad = true;
          record_error(kBadPageId, (unsigned)b, (unsigned)p, (unsigned)id);
        }
      }
    }
    if (__syncthreads_or(bad)) return;
  }

  uint8_t* sK = smem + L::kK;
  uint8_t* sV = smem + L::kV;
  float* sP = reinterpret_cast<float*>(smem + L::kP);
  float* sM = reinterpret_cast<float*>(smem + L::kM);
  float* sA = reinterpret_cast<float*>(smem + L::kA);
  float* sL = reinterpret_cast<float*>(smem + L::kL);
  int* sNV = reinterpret_cast<int*>(smem + L::kNV);
  uint64_t* kfull = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* vfull = kfull + kDecNK;

  // contiguous: the (b, hkv) cache; paged: the pool (the ring's offsets
  // include the head)
  const __nv_bfloat16* kbase;
  const __nv_bfloat16* vbase;
  if constexpr (PAGED) {
    kbase = a.k;
    vbase = a.v;
  } else {
    kbase = a.k + (size_t)(bh / a.kv_div) * a.Lkv * kDecD;  // (b, hkv_c)
    vbase = a.v + (size_t)(bh / a.kv_div) * a.Lkv * kDecD;
  }
  const uint64_t pol = policy_evict_first();

  if (tid == 0) {
    for (int i = 0; i < kDecNK; ++i) mbar_init(&kfull[i], 1);
    for (int i = 0; i < kDecNV; ++i) mbar_init(&vfull[i], 1);
    fence_mbar_init();
  }
  __syncthreads();

  auto rows_of = [&](int j) { return min(kDecBc, Lb - j * kDecBc); };
  // Copy the rows of block j from base (K or V) into dst; the barrier
  // expects every byte.  Issued by one thread.
  auto copy_block = [&](uint8_t* dst, const __nv_bfloat16* base, int j,
                        uint64_t* bar) {
    const int n = rows_of(j);
    mbar_arrive_expect_tx(bar, (uint32_t)n * kDecRowBytes);
    if constexpr (!PAGED) {
      bulk_load(dst, base + (size_t)j * kDecBc * kDecD,
                (uint32_t)n * kDecRowBytes, bar, pol);
    } else {
      const long long* offs = sOff + ((j - j0) & 63) * 4;
      if (npb == 1) {
        bulk_load(dst, base + offs[0], (uint32_t)n * kDecRowBytes, bar, pol);
      } else {
        const int seg = 1 << seg_l2;  // rows per copy
        for (int t = 0, i = 0; t < n; t += seg, ++i)
          bulk_load(dst + t * kDecRowBytes, base + offs[i],
                    (uint32_t)min(seg, n - t) * kDecRowBytes, bar, pol);
      }
    }
  };
  auto issue_k = [&](int r) {
    copy_block(sK + (r % kDecNK) * kDecBlockBytes, kbase, j0 + r,
               &kfull[r % kDecNK]);
  };
  if (tid == 0) {
    const int n0 = nblk < kDecNK ? nblk : kDecNK;
    for (int r = 0; r < n0; ++r) issue_k(r);
  }

  // Scoring layout: 8 lanes per key (kl = lane-in-key), 16 keys per pass,
  // 4 passes per block; warp w scores keys 4w..4w+3 (+16 per pass).
  // Lane kl holds dims [8kl, 8kl+8) and [64+8kl, 64+8kl+8) so that the 8
  // lanes of a key read 128 contiguous bytes per shared load.
  const int kl = tid & 7;
  const int ks = tid >> 3;
  float qf[G][16];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const __nv_bfloat16* qg = a.q + ((size_t)b * Hq + hkv * G + g) * kDecD;
    const uint4 w0 = *reinterpret_cast<const uint4*>(qg + 8 * kl);
    const uint4 w1 = *reinterpret_cast<const uint4*>(qg + 64 + 8 * kl);
    const uint32_t ww[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      qf[g][2 * i] = bf16lo(ww[i]);
      qf[g][2 * i + 1] = bf16hi(ww[i]);
    }
  }
  // After the 8-lane reduction a lane holds the score of one head for one
  // key; lanes that differ only in kDupMask bits hold the same value.
  const int my_head = head_of_lane<G>(lane);
  constexpr int kDupMask = G >= 8 ? 0 : (G == 4 ? 1 : (G == 2 ? 3 : 7));
  const bool writer = (lane & kDupMask) == 0;

  // P.V layout: 16 lanes cover the 128 dims of a key (8 dims each), 8 key
  // groups, keys c = kg + 8 i.
  const int dc = tid & 15;
  const int kg = tid >> 4;
  float acc[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int x = 0; x < 8; ++x) acc[g][x] = 0.f;

  float m_run[G];  // running max per head (replicated in every thread)
#pragma unroll
  for (int g = 0; g < G; ++g) m_run[g] = -INFINITY;
  float l_part = 0.f;  // writer lanes: partial normaliser of my_head

  int kept_issued = 0, kept_done = 0;
  unsigned long long n_vis = 0, n_skp = 0;

  auto pv = [&](int kidx) -> bool {
    const int slot = kidx % kDecNV;
    if (!mbar_wait(&vfull[slot], (uint32_t)(kidx / kDecNV) & 1u, kWaitDecodeV,
                   kidx, slot))
      return false;
    const float* al = sA + slot * 8;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float f = al[g];
#pragma unroll
      for (int x = 0; x < 8; ++x) acc[g][x] *= f;
    }
    const int nvalid = sNV[slot];
    const uint8_t* vst = sV + slot * kDecBlockBytes;
    const float* ps = sP + slot * kDecBc * G;
#pragma unroll 4
    for (int i = 0; i < 8; ++i) {
      const int c = kg + 8 * i;
      if (c < nvalid) {
        const uint4 vw =
            *reinterpret_cast<const uint4*>(vst + c * kDecRowBytes + dc * 16);
        const uint32_t w[4] = {vw.x, vw.y, vw.z, vw.w};
        float vf[8];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          vf[2 * t] = bf16lo(w[t]);
          vf[2 * t + 1] = bf16hi(w[t]);
        }
        float pg[G];
        if constexpr (G % 4 == 0) {
#pragma unroll
          for (int g4 = 0; g4 < G; g4 += 4) {
            const float4 p4 = *reinterpret_cast<const float4*>(ps + c * G + g4);
            pg[g4] = p4.x;
            pg[g4 + 1] = p4.y;
            pg[g4 + 2] = p4.z;
            pg[g4 + 3] = p4.w;
          }
        } else {
#pragma unroll
          for (int g = 0; g < G; ++g) pg[g] = ps[c * G + g];
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
#pragma unroll
          for (int x = 0; x < 8; x += 2) {
            float2 r = __ffma2_rn(make_float2(pg[g], pg[g]),
                                  make_float2(vf[x], vf[x + 1]),
                                  make_float2(acc[g][x], acc[g][x + 1]));
            acc[g][x] = r.x;
            acc[g][x + 1] = r.y;
          }
        }
      }
    }
    return true;
  };

  bool ok = true;
  // Scores of block r of the split (kept in registers by the caller) and
  // the per-warp head maxima, written to sMw[warp][head].
  auto score_block = [&](int r, float (&sc)[kDecBc / 16], float* sMw) {
    const int j = j0 + r;
    const int stage = r % kDecNK;
    const int nvalid = rows_of(j);
    if (ok)
      ok = mbar_wait(&kfull[stage], (uint32_t)(r / kDecNK) & 1u, kWaitDecodeK,
                     r, stage);
    if (ok) {
      const uint8_t* kst = sK + stage * kDecBlockBytes;
#pragma unroll
      for (int i = 0; i < kDecBc / 16; ++i) {
        const int c = ks + 16 * i;
        float part[G];
#pragma unroll
        for (int g = 0; g < G; ++g) part[g] = 0.f;
        if (c < nvalid) {
          const uint4 w0 =
              *reinterpret_cast<const uint4*>(kst + c * kDecRowBytes + kl * 16);
          const uint4 w1 = *reinterpret_cast<const uint4*>(
              kst + c * kDecRowBytes + 128 + kl * 16);
          const uint32_t ww[8] = {w0.x, w0.y, w0.z, w0.w,
                                  w1.x, w1.y, w1.z, w1.w};
          float kf[16];
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            kf[2 * t] = bf16lo(ww[t]);
            kf[2 * t + 1] = bf16hi(ww[t]);
          }
#pragma unroll
          for (int g = 0; g < G; ++g) {
            float2 s2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int x = 0; x < 16; x += 2)
              s2 = __ffma2_rn(make_float2(qf[g][x], qf[g][x + 1]),
                              make_float2(kf[x], kf[x + 1]), s2);
            part[g] = s2.x + s2.y;
          }
        }
        const float tot = reduce8_transpose<G>(part, lane);
        sc[i] = (c < nvalid && j * kDecBc + c >= key_lo) ? tot * a.scale
                                                         : -INFINITY;
      }
      float mx = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      if ((lane & (kDupMask | 24)) == 0) sMw[warp * 8 + my_head] = mx;
    }
  };
  if constexpr (BATCH == 1) {
  for (int r = 0; r < nblk; ++r) {
    const int j = j0 + r;
    const int nvalid = rows_of(j);

    // ---- scores of block j (kept in registers) and per-warp head maxima
    // (double-buffered by block parity: a fast warp may write block j+1's
    // while a slow one still reads block j's)
    float sc[kDecBc / 16];
    score_block(r, sc, sM + (r & 1) * 32);
    if (__syncthreads_or(!ok)) { ok = false; break; }
    if (tid == 0 && r + kDecNK < nblk) issue_k(r + kDecNK);
    if constexpr (PAGED) {
      // Ring refill, by the last warp, lane l for block 32(c+1) + l: at
      // block 32c (c >= 1) it copies the page ids of chunk c+1 into sPid
      // asynchronously; at block 32c+1 it waits for them and writes the
      // copies' offsets into the sOff slots chunk c-1 used (their last
      // reader, the V copy of block 32c-1, was issued before the barrier of
      // block 32c).  The first reader of chunk c+1 (the K copy of block
      // 32c+32, issued at block 32c+30) comes after many more barriers.
      if (warp == kDecThreads / 32 - 1 && r >= 32 && (r & 31) <= 1) {
        const int rr = (r & ~31) + 32 + lane;
        if ((r & 31) == 0) {
          if (rr < nblk) {
            for (int i = 0; i < npb; ++i) {
              const int tok = (j0 + rr) * kDecBc + (i << seg_l2);
              if (tok < Lb)
                cp_async_4(sPid + (rr & 63) * 4 + i,
                           bt_row + (tok >> a.log2_page));
            }
          }
          cp_async_commit();
        } else {
          cp_async_wait_all();
          if (rr < nblk) {
            for (int i = 0; i < npb; ++i) {
              const int tok = (j0 + rr) * kDecBc + (i << seg_l2);
              if (tok < Lb)
                sOff[(rr & 63) * 4 + i] = src_off(sPid[(rr & 63) * 4 + i], tok);
            }
          }
        }
      }
    }

    // ---- decision, identical in every thread: skip block j iff every
    // head's block max lies more than |ln lambda| below its running max.
    float mt[G];
    bool skip = ln_lambda > -INFINITY;
    const float* sMr = sM + (r & 1) * 32;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      mt[g] = fmaxf(fmaxf(sMr[g], sMr[8 + g]), fmaxf(sMr[16 + g], sMr[24 + g]));
      if (!(mt[g] - m_run[g] < ln_lambda)) skip = false;
    }
    if (tid == 0) {
      ++n_vis;
      if (skip) ++n_skp;
      if (a.mask) a.mask[(size_t)bh * a.nk + j] = skip ? 2 : 1;
    }
    if (!skip && !a.stats_only) {
      const int slot = kept_issued % kDecNV;
      if (tid == 0) {
        sNV[slot] = nvalid;
        copy_block(sV + slot * kDecBlockBytes, vbase, j, &vfull[slot]);
      }
      // new running max, rescale factor and P, per head
      float mn_mine = 0.f, al_mine = 1.f;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float mn = fmaxf(m_run[g], mt[g]);
        const float al =
            (m_run[g] == -INFINITY) ? 0.f : ex2_approx((m_run[g] - mn) * kLog2e);
        if (tid == 0) sA[slot * 8 + g] = al;
        if (g == my_head) {
          mn_mine = mn;
          al_mine = al;
        }
      }
      if (writer) {
        float* ps = sP + slot * kDecBc * G;
        float psum = 0.f;
#pragma unroll
        for (int i = 0; i < kDecBc / 16; ++i) {
          const float pv_ = ex2_approx((sc[i] - mn_mine) * kLog2e);
          ps[(ks + 16 * i) * G + my_head] = pv_;
          psum += pv_;
        }
        l_part = al_mine * l_part + psum;
      }
      ++kept_issued;
    }
#pragma unroll
    for (int g = 0; g < G; ++g) m_run[g] = fmaxf(m_run[g], mt[g]);

    while (ok && kept_issued - kept_done > kDecLag) {
      ok = pv(kept_done);
      ++kept_done;
    }
  }
  } else {
    // Batched decisions (contiguous cache): blocks r and r+1 are scored
    // before either is decided, and each is judged against
    //   Mb = max(running max over earlier blocks, maxima of both blocks);
    // kept blocks use Mb as the reference of P (m_ref, which acc and l
    // follow; it can move past m_run's old value through a skipped block).
    static_assert(BATCH == 2 && !PAGED, "batched decisions: pairs, contiguous");
    float m_ref[G];
#pragma unroll
    for (int g = 0; g < G; ++g) m_ref[g] = -INFINITY;
    for (int r = 0; r < nblk; r += 2) {
      const bool two = r + 1 < nblk;
      float sc0[kDecBc / 16], sc1[kDecBc / 16];
      // pair maxima double-buffered by pair parity
      float* sMp = sM + ((r >> 1) & 1) * 64;
      score_block(r, sc0, sMp);
      if (two) score_block(r + 1, sc1, sMp + 32);
      if (__syncthreads_or(!ok)) { ok = false; break; }
      if (tid == 0) {
        if (r + 2 < nblk) issue_k(r + 2);
        if (r + 3 < nblk) issue_k(r + 3);
      }
      float mt0[G], mt1[G], Mb[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        mt0[g] = fmaxf(fmaxf(sMp[g], sMp[8 + g]), fmaxf(sMp[16 + g], sMp[24 + g]));
        mt1[g] = two ? fmaxf(fmaxf(sMp[32 + g], sMp[40 + g]),
                             fmaxf(sMp[48 + g], sMp[56 + g]))
                     : -INFINITY;
        Mb[g] = fmaxf(m_run[g], fmaxf(mt0[g], mt1[g]));
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (u == 1 && !two) break;
        const int j = j0 + r + u;
        const int nvalid = rows_of(j);
        bool skip = ln_lambda > -INFINITY;
#pragma unroll
        for (int g = 0; g < G; ++g)
          if (!((u ? mt1[g] : mt0[g]) - Mb[g] < ln_lambda)) skip = false;
        if (tid == 0) {
          ++n_vis;
          if (skip) ++n_skp;
          if (a.mask) a.mask[(size_t)bh * a.nk + j] = skip ? 2 : 1;
        }
        if (!skip && !a.stats_only) {
          const int slot = kept_issued % kDecNV;
          if (tid == 0) {
            sNV[slot] = nvalid;
            copy_block(sV + slot * kDecBlockBytes, vbase, j, &vfull[slot]);
          }
          float mb_mine = 0.f, al_mine = 1.f;
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float al = (m_ref[g] == -INFINITY)
                                 ? 0.f
                                 : ex2_approx((m_ref[g] - Mb[g]) * kLog2e);
            if (tid == 0) sA[slot * 8 + g] = al;
            if (g == my_head) {
              mb_mine = Mb[g];
              al_mine = al;
            }
            m_ref[g] = Mb[g];
          }
          if (writer) {
            float* ps = sP + slot * kDecBc * G;
            float psum = 0.f;
#pragma unroll
            for (int i = 0; i < kDecBc / 16; ++i) {
              const float pv_ =
                  ex2_approx(((u ? sc1[i] : sc0[i]) - mb_mine) * kLog2e);
              ps[(ks + 16 * i) * G + my_head] = pv_;
              psum += pv_;
            }
            l_part = al_mine * l_part + psum;
          }
          ++kept_issued;
          // the next kept block's V slot is the one kept block n-1 used
          while (ok && kept_issued - kept_done > kDecLag) {
            ok = pv(kept_done);
            ++kept_done;
          }
        }
      }
#pragma unroll
      for (int g = 0; g < G; ++g) m_run[g] = Mb[g];
    }
#pragma unroll
    for (int g = 0; g < G; ++g) m_run[g] = m_ref[g];  // reference of l, acc
  }
  if constexpr (PAGED) {
    // no ring copy may still be landing when the CTA leaves
    if (warp == kDecThreads / 32 - 1) cp_async_wait_all();
  }
  if (__syncthreads_or(!ok)) ok = false;
  while (ok && kept_done < kept_issued) {
    ok = pv(kept_done);
    ++kept_done;
  }
  if (__syncthreads_or(!ok)) ok = false;

  if (!ok) {
    // Give outstanding copies a bounded chance to land before the CTA's
    // shared memory is released.
    if (tid == 0) {
      for (int i = 0; i < kDecNK; ++i)
        mbar_wait(&kfull[i], 0, kWaitDecodeDrain, i, 0, 1000000);
      for (int i = 0; i < kDecNV; ++i)
        mbar_wait(&vfull[i], 0, kWaitDecodeDrain, i, 1, 1000000);
    }
    return;
  }

  if (tid == 0 && a.counters) {
    atomicAdd(&a.counters[0], n_vis);
    atomicAdd(&a.counters[1], n_skp);
  }
  if (a.stats_only) return;

  // Normaliser of each head: writer lanes hold partials of their head; sum
  // over the lanes of the warp that share it, then over the 4 warps.
  {
    float x = writer ? l_part : 0.f;
    x += __shfl_xor_sync(0xffffffffu, x, 8);
    x += __shfl_xor_sync(0xffffffffu, x, 16);
#pragma unroll
    for (int msk = 1; msk <= 4; msk <<= 1)
      if (kDupMask & msk) x += __shfl_xor_sync(0xffffffffu, x, msk);
    if ((lane & (kDupMask | 24)) == 0) sL[warp * 8 + my_head] = x;
  }
  // Partial outputs of the 8 key groups -> shared (reusing the rings).
  float* red = reinterpret_cast<float*>(sK);
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float4* dst = reinterpret_cast<float4*>(red + ((kg * G + g) * kDecD + dc * 8));
    dst[0] = make_float4(acc[g][0], acc[g][1], acc[g][2], acc[g][3]);
    dst[1] = make_float4(acc[g][4], acc[g][5], acc[g][6], acc[g][7]);
  }
  __syncthreads();
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const int dd = tid;  // 128 threads = 128 dims
    float sum = 0.f;
#pragma unroll
    for (int t = 0; t < 8; ++t) sum += red[(t * G + g) * kDecD + dd];
    const float l = sL[g] + sL[8 + g] + sL[16 + g] + sL[24 + g];
    const size_t row = (size_t)b * Hq + hkv * G + g;
    // a split with no blocks (only a short paged sequence has one)
    // contributes o = 0, lse = -inf
    a.o_part[(row * a.S + s) * kDecD + dd] = l > 0.f ? sum / l : 0.f;
    if (dd == 0)
      a.lse_part[row * a.S + s] = l > 0.f ? m_run[g] + __logf(l) : -INFINITY;
  }
}

// Log-sum-exp merge of the S split partials of one (sequence, query head):
//   lse = ln sum_s exp(lse_s),  o = sum_s exp(lse_s - lse) o_s.
// Work order of a paged call: order[r] is the sequence with the r-th
// longest length (ties by index), so that the CTAs of the longest sequences
// start first and the last wave holds the shortest splits.  Which CTA runs a
// split changes nothing in what the split computes.  rank(i) counts the
// sequences before i in the strict order (length descending, index
// ascending); distinct sequences get distinct ranks in [0, B), so `order`
// is a permutation.  Grid ceil(B / 256) x 256 threads.
__global__ void __launch_bounds__(256)
    decode_order_kernel(const int* __restrict__ seq_lens, int B,
                        int* __restrict__ order) {
  __shared__ int len[256];
  const int i = blockIdx.x * 256 + threadIdx.x;
  const int li = i < B ? __ldg(seq_lens + i) : 0;
  int rank = 0;
  for (int j0 = 0; j0 < B; j0 += 256) {
    __syncthreads();
    if (j0 + (int)threadIdx.x < B) len[threadIdx.x] = __ldg(seq_lens + j0 + threadIdx.x);
    __syncthreads();
    const int n = min(256, B - j0);
    for (int jj = 0; jj < n; ++jj) {
      const int lj = len[jj];
      rank += (lj > li || (lj == li && j0 + jj < i)) ? 1 : 0;
    }
  }
  if (i < B) order[rank] = i;
}

// An empty split (lse_s = -inf, o_s = 0) gets weight 0.  One thread per
// output column: the block has d (64 or 128) threads.
__global__ void __launch_bounds__(kDecD)
    decode_combine_kernel(const float* __restrict__ o_part,
                          const float* __restrict__ lse_part,
                          __nv_bfloat16* __restrict__ o, float* __restrict__ lse,
                          int S) {
#if defined(__CUDA_ARCH__)
  asm volatile("griddepcontrol.wait;" ::: "memory");
#endif
  const int D = blockDim.x;
  const size_t row = blockIdx.x;
  const int dd = threadIdx.x;
  const float* lp = lse_part + row * S;
  float mx = -INFINITY;
  for (int s = 0; s < S; ++s) mx = fmaxf(mx, lp[s]);
  if (mx == -INFINITY) {  // no keys at all (a paged sequence of length 0)
    o[row * D + dd] = __float2bfloat16_rn(0.f);
    if (dd == 0 && lse) lse[row] = -INFINITY;
    return;
  }
  float sum = 0.f;
  for (int s = 0; s < S; ++s) sum += ex2_approx((lp[s] - mx) * kLog2e);
  const float L = mx + __logf(sum);
  float acc = 0.f;
  const float* op = o_part + row * S * D + dd;
  for (int s = 0; s < S; ++s)
    acc += ex2_approx((lp[s] - L) * kLog2e) * op[(size_t)s * D];
  o[row * D + dd] = __float2bfloat16_rn(acc);
  if (dd == 0 && lse) lse[row] = L;
}

}  // namespace blasst

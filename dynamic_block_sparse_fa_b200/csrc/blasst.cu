// blasst.cu -- the C ABI declared in include/blasst.h: argument validation,
// launch configuration, the calibration search and the error plumbing.
// Kernels live in decode.cuh / prefill.cuh; this is one translation unit so
// that the device error word is a single symbol.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "blasst.h"
#include "decode.cuh"
#include "prefill.cuh"
#include "prefill2.cuh"
#include "backward.cuh"
#include "mla.cuh"
#include "decode_wide.cuh"
#include "decode_mma.cuh"

namespace {

thread_local char g_last_error[512] = "";

blasst_status_t cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return BLASST_OK;
  snprintf(g_last_error, sizeof g_last_error, "%s: %s", what,
           cudaGetErrorString(e));
  return BLASST_ERR_CUDA;
}

bool aligned16(const void* p) {
  return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

bool valid_ln_lambda(float x) { return x <= 0.0f; }  // false for NaN, > 0

constexpr int kNumSmB200 = 148;

}  // namespace

extern "C" {

const char* blasst_version(void) { return "0.1.0"; }

const char* blasst_last_error(void) { return g_last_error; }

const char* blasst_strerror(blasst_status_t s) {
  switch (s) {
    case BLASST_OK: return "ok";
    case BLASST_ERR_INVALID_ARG: return "invalid argument";
    case BLASST_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case BLASST_ERR_MISALIGNED: return "tensor pointer not 16-byte aligned";
    case BLASST_ERR_CUDA: return "CUDA error";
    case BLASST_ERR_TIMEOUT: return "a kernel gave up a bounded wait";
    case BLASST_ERR_NO_CONVERGE: return "calibration did not reach the target";
    case BLASST_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

blasst_status_t blasst_skip_stats_reset(unsigned long long* counters,
                                        void* stream) {
  if (!counters) return BLASST_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(counters, 0, 2 * sizeof(unsigned long long),
                                     (cudaStream_t)stream),
                     "cudaMemsetAsync(counters)");
}

namespace {
// Waits on an mbarrier that nothing arrives at, with the given limit: the
// wait gives up, records kWaitSelfTest in the device error word and the
// kernel returns.  Exercises the failure path of every bounded wait of the
// library without faulting the GPU.
__global__ void selftest_wait_kernel(long long limit_cycles) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    blasst::mbar_init(&bar, 1);
    blasst::fence_mbar_init();
  }
  __syncthreads();
  blasst::mbar_wait(&bar, 0, blasst::kWaitSelfTest, 0, 0, limit_cycles);
}
}  // namespace

blasst_status_t blasst_selftest_wait_timeout(long long limit_cycles,
                                             void* stream) {
  if (limit_cycles < 1 || limit_cycles > 4000000000LL)
    return BLASST_ERR_INVALID_ARG;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      limit_cycles);
  return cuda_status(cudaGetLastError(), "selftest launch");
}

blasst_status_t blasst_check_device_error(int* where_out) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_status(e, "cudaDeviceSynchronize");
  unsigned int code = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&code, blasst::g_error_code, sizeof code);
  if (e != cudaSuccess) return cuda_status(e, "read error word");
  if (where_out) *where_out = (int)code;
  if (code == 0) return BLASST_OK;
  unsigned int info[4] = {0, 0, 0, 0}, count = 0;
  cudaMemcpyFromSymbol(info, blasst::g_error_info, sizeof info);
  cudaMemcpyFromSymbol(&count, blasst::g_error_count, sizeof count);
  cudaMemcpyToSymbol(blasst::g_error_code, &zero, sizeof zero);
  cudaMemcpyToSymbol(blasst::g_error_count, &zero, sizeof zero);
  if (code == blasst::kBadSeqLen) {
    snprintf(g_last_error, sizeof g_last_error,
             "paged decode: sequence %u has length %d, outside [0, "
             "max_seq_len]",
             info[1], (int)info[2]);
    return BLASST_ERR_INVALID_ARG;
  }
  if (code == blasst::kBadPageId) {
    snprintf(g_last_error, sizeof g_last_error,
             "paged decode: sequence %u, block-table entry %u holds page id "
             "%d, outside [0, num_pages)",
             info[1], info[2], (int)info[3]);
    return BLASST_ERR_INVALID_ARG;
  }
  snprintf(g_last_error, sizeof g_last_error,
           "wait %u gave up first (block %u, step %u, parity %u, slot %u); "
           "%u waits gave up in total",
           code, info[0], info[1], info[2], info[3], count);
  return BLASST_ERR_TIMEOUT;
}

// ---------------------------------------------------------------------------
// Decode
// ---------------------------------------------------------------------------
int blasst_decode_splits(int B, int Hkv, int Lkv, int Bc) {
  if (B < 1 || Hkv < 1 || Lkv < 1 || Bc < 1) return 1;
  const long long nk = (Lkv + (long long)Bc - 1) / Bc;
  const long long units = (long long)B * Hkv;
  // At least two waves of the split kernel on a 148-SM B200 with 3 resident
  // CTAs per SM, at least 8 blocks per split, and among the split counts up
  // to twice that minimum the one whose last wave is fullest (fewer splits
  // on ties: every split restarts the running max).
  const long long slots = (long long)kNumSmB200 * 3;
  const long long s_max = nk / 8 > 1 ? nk / 8 : 1;
  long long s_min = (2 * slots + units - 1) / units;
  if (s_min > s_max) return (int)s_max;
  if (s_min < 1) s_min = 1;
  const long long s_hi = 2 * s_min < s_max ? 2 * s_min : s_max;
  long long best = s_min;
  double best_eff = -1.0;
  for (long long s = s_min; s <= s_hi; ++s) {
    const double waves = (double)(units * s) / (double)slots;
    const double eff = waves / std::ceil(waves);
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = s;
    }
  }
  return (int)best;
}

int blasst_decode_wide_splits(int B, int Hkv, int Lkv, int Bc) {
  if (B < 1 || Hkv < 1 || Lkv < 1 || Bc < 1) return 1;
  const long long nk = (Lkv + (long long)Bc - 1) / Bc;
  const long long units = (long long)B * Hkv;
  // The tensor-core kernel of wide groups keeps 2 CTAs per SM.  Modelled
  // time of S splits: the waves of (sequence, KV head, split) items times
  // one item's time, nk / S blocks plus the fixed cost of an item (its q,
  // its partial write and merge row: about two blocks).  The S with at least
  // 8 blocks per split that minimises it, fewer splits on ties.
  const long long slots = (long long)kNumSmB200 * 2;
  const long long s_max = nk / 8 > 1 ? nk / 8 : 1;
  long long best = 1;
  double best_t = 0.0;
  for (long long s = 1; s <= s_max; ++s) {
    const double waves = std::ceil((double)(units * s) / (double)slots);
    const double t = waves * ((double)nk / (double)s + 2.0);
    if (s == 1 || t < best_t - 1e-9) {
      best_t = t;
      best = s;
    }
  }
  return (int)best;
}

int blasst_decode_group_splits(int B, int Hq, int Hkv, int Lkv, int Bc) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Lkv < 1 || Bc < 1 || Hq % Hkv != 0)
    return 1;
  const int G = Hq / Hkv;
  if (G > 8 && G <= 128 && Bc == blasst::kWideBc)
    return blasst_decode_wide_splits(B, Hkv, Lkv, Bc);
  return blasst_decode_splits(B, Hkv, Lkv, Bc);
}

size_t blasst_decode_workspace_size(int B, int Hq, int d, int num_splits) {
  if (B < 1 || Hq < 1 || d < 1 || num_splits < 1) return 0;
  const size_t rows = (size_t)B * Hq * num_splits;
  const size_t o_bytes = (rows * d * sizeof(float) + 255) & ~(size_t)255;
  const size_t l_bytes = (rows * sizeof(float) + 255) & ~(size_t)255;
  const size_t w_bytes = ((size_t)B * sizeof(int) + 255) & ~(size_t)255;
  return o_bytes + l_bytes + w_bytes;
}

}  // extern "C"

namespace {
// Query heads per KV head the decode kernel takes: 1, 2, 4 or 8 heads form
// one tile; a larger power of two is cut into tiles of 8 heads.
bool decode_group_ok(int G) {
  return G >= 1 && G <= 256 && (G & (G - 1)) == 0;
}

// Split kernel, then (unless statistics only) the merge, launched as a
// programmatic dependent of the split kernel so its launch overlaps the
// split kernel's tail (it waits on griddepcontrol).
template <int G, bool PAGED, int BATCH = 1>
cudaError_t launch_split(const blasst::DecodeArgs& a, long long grid,
                         cudaStream_t st) {
  const int smem = blasst::DecodeSmem<G>::kTotal;
  cudaError_t e = cudaFuncSetAttribute(
      blasst::decode_split_kernel<G, PAGED, BATCH>,
      cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  blasst::decode_split_kernel<G, PAGED, BATCH>
      <<<(unsigned)grid, blasst::kDecThreads, smem, st>>>(a);
  return cudaGetLastError();
}

// The warp-MMA decode (decode_mma.cuh) for the sequential rule on a
// contiguous cache with G <= 8, then the merge as for launch_decode.
template <int G, int D, bool PAGED, int BATCH = 1>
cudaError_t launch_mma_split(const blasst::DecodeMmaArgs& a, long long grid,
                             cudaStream_t st) {
  using C = blasst::DecodeMmaCfg;
  cudaError_t e = cudaFuncSetAttribute(
      blasst::decode_mma_kernel<G, D, PAGED, BATCH>,
      cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  blasst::decode_mma_kernel<G, D, PAGED, BATCH>
      <<<(unsigned)grid, blasst::kDecThreads, C::SMEM_ALLOC, st>>>(a);
  return cudaGetLastError();
}

// paged: the pool form; batch 2: the batched decision rule (contiguous)
blasst_status_t launch_decode_mma(const blasst::DecodeMmaArgs& a, int G,
                                  int d, bool paged, long long grid,
                                  bool stats_only, void* o, float* lse,
                                  int rows, cudaStream_t st, int batch = 1) {
  cudaError_t e = cudaErrorInvalidValue;
  switch (G * 1000 + d) {
#define BLASST_LAUNCH_MMA(GG, DD)                                           \
  case GG * 1000 + DD:                                                      \
    e = paged ? launch_mma_split<GG, DD, true>(a, grid, st)                 \
              : (batch == 2 ? launch_mma_split<GG, DD, false, 2>(a, grid, st) \
                            : launch_mma_split<GG, DD, false>(a, grid, st)); \
    break;
    BLASST_LAUNCH_MMA(1, 128)
    BLASST_LAUNCH_MMA(2, 128)
    BLASST_LAUNCH_MMA(4, 128)
    BLASST_LAUNCH_MMA(8, 128)
    BLASST_LAUNCH_MMA(1, 64)
    BLASST_LAUNCH_MMA(2, 64)
    BLASST_LAUNCH_MMA(4, 64)
    BLASST_LAUNCH_MMA(8, 64)
#undef BLASST_LAUNCH_MMA
  }
  if (e != cudaSuccess) return cuda_status(e, "decode split launch");
  if (stats_only) return BLASST_OK;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)rows);
  cfg.blockDim = dim3(d);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, blasst::decode_combine_kernel,
                         (const float*)a.o_part, (const float*)a.lse_part,
                         static_cast<__nv_bfloat16*>(o), lse, a.S);
  return cuda_status(e, "decode merge launch");
}

blasst_status_t launch_decode(const blasst::DecodeArgs& a, int G, bool paged,
                              long long grid, bool stats_only, void* o,
                              float* lse, int rows, cudaStream_t st,
                              int batch = 1) {
  cudaError_t e = cudaErrorInvalidValue;
  switch (G) {
#define BLASST_LAUNCH_DECODE(GG)                                             \
  case GG:                                                                   \
    e = paged ? launch_split<GG, true>(a, grid, st)                          \
              : (batch == 2 ? launch_split<GG, false, 2>(a, grid, st)        \
                            : launch_split<GG, false>(a, grid, st));         \
    break;
    BLASST_LAUNCH_DECODE(1)
    BLASST_LAUNCH_DECODE(2)
    BLASST_LAUNCH_DECODE(4)
    BLASST_LAUNCH_DECODE(8)
#undef BLASST_LAUNCH_DECODE
  }
  if (e != cudaSuccess) return cuda_status(e, "decode split launch");
  if (stats_only) return BLASST_OK;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)rows);
  cfg.blockDim = dim3(blasst::kDecD);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, blasst::decode_combine_kernel,
                         (const float*)a.o_part, (const float*)a.lse_part,
                         static_cast<__nv_bfloat16*>(o), lse, a.S);
  return cuda_status(e, "decode merge launch");
}

blasst_status_t decode_contiguous(const void* q, const void* k_cache,
                                  const void* v_cache, void* o, float* lse,
                                  int B, int Hq, int Hkv, int Lkv, int d,
                                  float scale, int window, int batch,
                                  float ln_lambda, int Bc, int num_splits,
                                  void* workspace, size_t workspace_bytes,
                                  const blasst_skip_stats_t* skip_stats,
                                  void* stream);

// Split partials inside a caller workspace (layout of
// blasst_decode_workspace_size).
blasst_status_t carve_workspace(void* workspace, size_t workspace_bytes,
                                int B, int Hq, int d, int S, float** o_part,
                                float** lse_part, int** order = nullptr) {
  const size_t need = blasst_decode_workspace_size(B, Hq, d, S);
  if (!workspace || workspace_bytes < need) return BLASST_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return BLASST_ERR_MISALIGNED;
  const size_t rows = (size_t)B * Hq * S;
  const size_t o_bytes = (rows * d * sizeof(float) + 255) & ~(size_t)255;
  const size_t l_bytes = (rows * sizeof(float) + 255) & ~(size_t)255;
  *o_part = static_cast<float*>(workspace);
  *lse_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + o_bytes);
  if (order)
    *order = reinterpret_cast<int*>(static_cast<char*>(workspace) + o_bytes +
                                    l_bytes);
  return BLASST_OK;
}

// Paged calls whose grid is more than one wave decode the longest sequences
// first: the order (a permutation of the B sequences, see
// decode_order_kernel) goes to the workspace's last region.  NULL when the
// order cannot matter (one sequence, or every CTA resident at once).
int* paged_work_order(const int* seq_lens, int B, long long ctas, int* region,
                      cudaStream_t st, blasst_status_t* rc) {
  *rc = BLASST_OK;
  if (B < 2 || ctas <= (long long)kNumSmB200 * 3) return nullptr;
  blasst::decode_order_kernel<<<(unsigned)((B + 255) / 256), 256, 0, st>>>(
      seq_lens, B, region);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    *rc = cuda_status(e, "paged decode work order");
    return nullptr;
  }
  return region;
}
}  // namespace

extern "C" {

blasst_status_t blasst_decode(const void* q, const void* k_cache,
                              const void* v_cache, void* o, float* lse, int B,
                              int Hq, int Hkv, int Lkv, int d, float scale,
                              float ln_lambda, int Bc, int num_splits,
                              void* workspace, size_t workspace_bytes,
                              const blasst_skip_stats_t* skip_stats,
                              void* stream) {
  return blasst_decode_window(q, k_cache, v_cache, o, lse, B, Hq, Hkv, Lkv, d,
                              scale, 0, ln_lambda, Bc, num_splits, workspace,
                              workspace_bytes, skip_stats, stream);
}

blasst_status_t blasst_decode_window(const void* q, const void* k_cache,
                                     const void* v_cache, void* o, float* lse,
                                     int B, int Hq, int Hkv, int Lkv, int d,
                                     float scale, int window, float ln_lambda,
                                     int Bc, int num_splits, void* workspace,
                                     size_t workspace_bytes,
                                     const blasst_skip_stats_t* skip_stats,
                                     void* stream) {
  return decode_contiguous(q, k_cache, v_cache, o, lse, B, Hq, Hkv, Lkv, d,
                           scale, window, 0, ln_lambda, Bc, num_splits,
                           workspace, workspace_bytes, skip_stats, stream);
}

blasst_status_t blasst_decode_batched(const void* q, const void* k_cache,
                                      const void* v_cache, void* o, float* lse,
                                      int B, int Hq, int Hkv, int Lkv, int d,
                                      float scale, float ln_lambda, int Bc,
                                      int num_splits, int batch,
                                      void* workspace, size_t workspace_bytes,
                                      const blasst_skip_stats_t* skip_stats,
                                      void* stream) {
  if (batch != 1 && batch != 2) return BLASST_ERR_UNSUPPORTED_SHAPE;
  return decode_contiguous(q, k_cache, v_cache, o, lse, B, Hq, Hkv, Lkv, d,
                           scale, 0, batch, ln_lambda, Bc, num_splits,
                           workspace, workspace_bytes, skip_stats, stream);
}

}  // extern "C"

namespace {
// The tensor-core decode (decode_wide.cuh) for G = Hq / Hkv <= 128 heads
// per KV head, in tiles of T heads (T = G, or 8 for G a multiple of 8);
// arguments already validated, S resolved.
blasst_status_t wide_launch(const void* q, const void* k_cache,
                            const void* v_cache, void* o, float* lse, int B,
                            int Hq, int Hkv, int Lkv, float scale, int window,
                            int T, float ln_lambda, int S, void* workspace,
                            size_t workspace_bytes,
                            const blasst_skip_stats_t* skip_stats,
                            void* stream) {
  const int d = blasst::kWideD;
  const int G = Hq / Hkv;
  const int nk = (Lkv + blasst::kWideBc - 1) / blasst::kWideBc;
  const long long grid = (long long)B * Hkv * S;
  if (grid > 0x7fffffffLL) return BLASST_ERR_UNSUPPORTED_SHAPE;
  const bool stats_only = (o == nullptr);
  blasst::WideArgs a;
  memset(&a, 0, sizeof a);
  if (!stats_only) {
    const blasst_status_t ws = carve_workspace(workspace, workspace_bytes, B,
                                               Hq, d, S, &a.o_part,
                                               &a.lse_part);
    if (ws != BLASST_OK) return ws;
  }
  if (!blasst::encode_map(&a.tk, k_cache, d, Lkv, (long long)B * Hkv, 64) ||
      !blasst::encode_map(&a.tv, v_cache, d, Lkv, (long long)B * Hkv, 64))
    return cuda_status(cudaErrorInvalidValue, "wide decode tensor maps");
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.counters = skip_stats ? skip_stats->counters : nullptr;
  a.mask = skip_stats ? skip_stats->mask : nullptr;
  a.Hkv = Hkv;
  a.G = G;
  a.T = T;
  a.window = window;
  a.Lkv = Lkv;
  a.nk = nk;
  a.S = S;
  a.scale = scale;
  a.ln_lambda = ln_lambda;
  a.stats_only = stats_only ? 1 : 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaFuncSetAttribute(blasst::decode_wide_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       blasst::WideCfg::SMEM_ALLOC);
  if (e != cudaSuccess) return cuda_status(e, "wide decode attribute");
  blasst::decode_wide_kernel<<<(unsigned)grid, blasst::kWideThreads,
                               blasst::WideCfg::SMEM_ALLOC, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess || stats_only)
    return cuda_status(e, "wide decode split launch");
  blasst::decode_combine_kernel<<<(unsigned)((long long)B * Hq), blasst::kDecD,
                                  0, st>>>(
      a.o_part, a.lse_part, static_cast<__nv_bfloat16*>(o), lse, S);
  return cuda_status(cudaGetLastError(), "wide decode merge launch");
}

// Contiguous-cache decode.  batch = 0: blasst_decode / blasst_decode_window
// (the sequential rule on the fastest kernel for the group: the warp-MMA
// kernel for G <= 8, the tensor-core tiles for 16 <= G <= 128, the
// CUDA-core kernel above); batch = 2: the batched rule (warp-MMA kernel for
// G <= 8, else the CUDA-core kernel); batch = 1: the sequential rule on the
// CUDA-core split kernel (a second, independent implementation).
blasst_status_t decode_contiguous(const void* q, const void* k_cache,
                                  const void* v_cache, void* o, float* lse,
                                  int B, int Hq, int Hkv, int Lkv, int d,
                                  float scale, int window, int batch,
                                  float ln_lambda, int Bc, int num_splits,
                                  void* workspace, size_t workspace_bytes,
                                  const blasst_skip_stats_t* skip_stats,
                                  void* stream) {
  if (!q || !k_cache || !v_cache) return BLASST_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Lkv < 1 || Hq % Hkv != 0 || window < 0)
    return BLASST_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !valid_ln_lambda(ln_lambda))
    return BLASST_ERR_INVALID_ARG;
  int G = Hq / Hkv;
  if (Bc != blasst::kDecBc || !decode_group_ok(G))
    return BLASST_ERR_UNSUPPORTED_SHAPE;
  // d = 128 everywhere; d = 64 on the warp-MMA kernel (the sequential or
  // the batched rule with at most 8 heads per KV head)
  if (!(d == blasst::kDecD || (d == 64 && batch != 1 && G <= 8)))
    return BLASST_ERR_UNSUPPORTED_SHAPE;
  const int kv_div = G > 8 ? G / 8 : 1;  // tiles of 8 heads above 8
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) ||
      (o && !aligned16(o)))
    return BLASST_ERR_MISALIGNED;
  const int nk = (Lkv + Bc - 1) / Bc;
  // blocks that hold the visible keys (all of them without a window)
  const int jlo = (window > 0 && Lkv > window) ? (Lkv - window) / Bc : 0;
  // the automatic count: the group's own policy for the sequential rule
  // (its kernel follows from G), the GQA one for the CUDA-core kernel
  const int S = num_splits != 0 ? num_splits
                : batch == 0 ? blasst_decode_group_splits(B, Hq, Hkv,
                                                          Lkv - jlo * Bc, Bc)
                             : blasst_decode_splits(B, Hkv, Lkv - jlo * Bc, Bc);
  if (S < 1 || S > nk - jlo) return BLASST_ERR_INVALID_ARG;
  // Wide groups (16 to 128 heads per KV head): the tiles of 8 run on the
  // tensor core, one CTA per (sequence, KV head, split) for all of them;
  // G x d FMAs per key would leave the CUDA-core kernel far below the
  // memory time.  Same tiles, decisions and split policy.
  if (batch == 0 && G > 8 && G <= 128)
    return wide_launch(q, k_cache, v_cache, o, lse, B, Hq, Hkv, Lkv, scale,
                       window, 8, ln_lambda, S, workspace, workspace_bytes,
                       skip_stats, stream);
  const long long grid_mma = (long long)B * Hkv * S;
  if (batch != 1 && G <= 8 && grid_mma <= 0x7fffffffLL) {
    // the sequential rule (batch 0) or the batched rule (batch 2) on the
    // warp-MMA kernel
    const bool stats_only = (o == nullptr);
    blasst::DecodeMmaArgs m;
    memset(&m, 0, sizeof m);
    if (!stats_only) {
      const blasst_status_t ws = carve_workspace(workspace, workspace_bytes, B,
                                                 Hq, d, S, &m.o_part,
                                                 &m.lse_part);
      if (ws != BLASST_OK) return ws;
    }
    if (!blasst::encode_map(&m.tk, k_cache, d, Lkv, (long long)B * Hkv, 64) ||
        !blasst::encode_map(&m.tv, v_cache, d, Lkv, (long long)B * Hkv, 64))
      return cuda_status(cudaErrorInvalidValue, "decode tensor maps");
    m.q = static_cast<const __nv_bfloat16*>(q);
    m.counters = skip_stats ? skip_stats->counters : nullptr;
    m.mask = skip_stats ? skip_stats->mask : nullptr;
    m.margin = skip_stats ? skip_stats->margin : nullptr;
    m.Hkv = Hkv;
    m.Lkv = Lkv;
    m.nk = nk;
    m.S = S;
    m.scale = scale;
    m.ln_lambda = ln_lambda;
    m.stats_only = stats_only ? 1 : 0;
    m.window = window;
    return launch_decode_mma(m, G, d, false, grid_mma, stats_only, o, lse,
                             B * Hq, static_cast<cudaStream_t>(stream),
                             batch == 2 ? 2 : 1);
  }
  G /= kv_div;
  const long long grid = (long long)B * Hkv * kv_div * S;
  if (grid > 0x7fffffffLL) return BLASST_ERR_UNSUPPORTED_SHAPE;
  const bool stats_only = (o == nullptr);
  float* o_part = nullptr;
  float* lse_part = nullptr;
  if (!stats_only) {
    const blasst_status_t ws = carve_workspace(workspace, workspace_bytes, B,
                                               Hq, d, S, &o_part, &lse_part);
    if (ws != BLASST_OK) return ws;
  }
  blasst::DecodeArgs a = {};
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k_cache);
  a.v = static_cast<const __nv_bfloat16*>(v_cache);
  a.o_part = o_part;
  a.lse_part = lse_part;
  a.counters = skip_stats ? skip_stats->counters : nullptr;
  a.mask = skip_stats ? skip_stats->mask : nullptr;
  a.Hkv = Hkv * kv_div;
  a.kv_div = kv_div;
  a.Lkv = Lkv;
  a.nk = nk;
  a.S = S;
  a.scale = scale;
  a.ln_lambda = ln_lambda;
  a.stats_only = stats_only ? 1 : 0;
  a.window = window;

  return launch_decode(a, G, false, grid, stats_only, o, lse, B * Hq,
                       static_cast<cudaStream_t>(stream), batch);
}
}  // namespace

extern "C" {

// ---------------------------------------------------------------------------
// Decode over a paged cache (block table + per-sequence lengths)
// ---------------------------------------------------------------------------
blasst_status_t blasst_decode_paged(const void* q, const void* k_pages,
                                    const void* v_pages, long long page_stride,
                                    int num_pages, int page_size,
                                    const int* block_table, int max_pages,
                                    const int* seq_lens, int max_seq_len,
                                    void* o, float* lse, int B, int Hq,
                                    int Hkv, int d, float scale,
                                    float ln_lambda, int per_length,
                                    int num_splits, void* workspace,
                                    size_t workspace_bytes,
                                    const blasst_skip_stats_t* skip_stats,
                                    void* stream) {
  if (!q || !k_pages || !v_pages || !block_table || !seq_lens)
    return BLASST_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || num_pages < 1 ||
      max_pages < 1 || max_seq_len < 1 || num_splits < 0)
    return BLASST_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return BLASST_ERR_INVALID_ARG;
  if (per_length ? (std::isnan(ln_lambda) || ln_lambda == INFINITY)
                 : !valid_ln_lambda(ln_lambda))
    return BLASST_ERR_INVALID_ARG;
  int log2_page = -1;
  for (int l2 = 4; l2 <= 8; ++l2)
    if (page_size == (1 << l2)) log2_page = l2;
  if (log2_page < 0) return BLASST_ERR_UNSUPPORTED_SHAPE;
  if ((long long)max_seq_len > (long long)max_pages * page_size)
    return BLASST_ERR_INVALID_ARG;
  int G = Hq / Hkv;
  // d 128, or 64 on the warp-MMA kernel (up to 8 heads per KV head)
  if (!(d == blasst::kDecD || (d == 64 && G <= 8)) || !decode_group_ok(G))
    return BLASST_ERR_UNSUPPORTED_SHAPE;
  const int kv_div = G > 8 ? G / 8 : 1;  // tiles of 8 heads above 8
  if (page_stride < (long long)Hkv * page_size * d || page_stride % 8 != 0)
    return BLASST_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) ||
      (o && !aligned16(o)))
    return BLASST_ERR_MISALIGNED;
  const int Bc = blasst::kDecBc;
  const int nk = (max_seq_len + Bc - 1) / Bc;
  const int S = num_splits == 0 ? blasst_decode_splits(B, Hkv, max_seq_len, Bc)
                                : num_splits;
  if (S < 1 || S > nk) return BLASST_ERR_INVALID_ARG;
  if (G <= 8 && (long long)B * Hkv * S <= 0x7fffffffLL) {
    // up to 8 heads per KV head: the warp-MMA kernel over the pool
    const bool stats_only = (o == nullptr);
    blasst::DecodeMmaArgs m;
    memset(&m, 0, sizeof m);
    int* region = nullptr;
    if (!stats_only) {
      const blasst_status_t ws = carve_workspace(workspace, workspace_bytes, B,
                                                 Hq, d, S, &m.o_part,
                                                 &m.lse_part, &region);
      if (ws != BLASST_OK) return ws;
    }
    const int box_rows = page_size < 64 ? page_size : 64;
    // d 128: whole rows per copy (5-D map); d 64: one 64-column box
    const bool maps_ok =
        d == 128
            ? blasst::encode_pool_map_rows(&m.tk, k_pages, page_size, Hkv,
                                           num_pages, page_stride, box_rows) &&
                  blasst::encode_pool_map_rows(&m.tv, v_pages, page_size, Hkv,
                                               num_pages, page_stride, box_rows)
            : blasst::encode_pool_map(&m.tk, k_pages, d, page_size, Hkv,
                                      num_pages, page_stride, box_rows) &&
                  blasst::encode_pool_map(&m.tv, v_pages, d, page_size, Hkv,
                                          num_pages, page_stride, box_rows);
    if (!maps_ok)
      return cuda_status(cudaErrorInvalidValue, "paged decode tensor maps");
    m.q = static_cast<const __nv_bfloat16*>(q);
    m.counters = skip_stats ? skip_stats->counters : nullptr;
    m.mask = skip_stats ? skip_stats->mask : nullptr;
    m.margin = skip_stats ? skip_stats->margin : nullptr;
    m.Hkv = Hkv;
    m.Lkv = max_seq_len;
    m.nk = nk;
    m.S = S;
    m.scale = scale;
    m.ln_lambda = ln_lambda;
    m.stats_only = stats_only ? 1 : 0;
    m.block_table = block_table;
    m.seq_lens = seq_lens;
    m.max_pages = max_pages;
    m.num_pages = num_pages;
    m.log2_page = log2_page;
    m.per_length = per_length ? 1 : 0;
    if (region) {
      blasst_status_t rc;
      m.order = paged_work_order(seq_lens, B, (long long)B * Hkv * S, region,
                                 static_cast<cudaStream_t>(stream), &rc);
      if (rc != BLASST_OK) return rc;
    }
    return launch_decode_mma(m, G, d, true, (long long)B * Hkv * S, stats_only,
                             o, lse, B * Hq, static_cast<cudaStream_t>(stream));
  }
  G /= kv_div;
  const long long grid = (long long)B * Hkv * kv_div * S;
  if (grid > 0x7fffffffLL) return BLASST_ERR_UNSUPPORTED_SHAPE;
  const bool stats_only = (o == nullptr);
  float* o_part = nullptr;
  float* lse_part = nullptr;
  int* region = nullptr;
  if (!stats_only) {
    const blasst_status_t ws = carve_workspace(workspace, workspace_bytes, B,
                                               Hq, d, S, &o_part, &lse_part,
                                               &region);
    if (ws != BLASST_OK) return ws;
  }
  blasst::DecodeArgs a = {};
  if (region) {
    blasst_status_t rc;
    a.order = paged_work_order(seq_lens, B, grid, region,
                               static_cast<cudaStream_t>(stream), &rc);
    if (rc != BLASST_OK) return rc;
  }
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k_pages);
  a.v = static_cast<const __nv_bfloat16*>(v_pages);
  a.o_part = o_part;
  a.lse_part = lse_part;
  a.counters = skip_stats ? skip_stats->counters : nullptr;
  a.mask = skip_stats ? skip_stats->mask : nullptr;
  a.Hkv = Hkv * kv_div;
  a.kv_div = kv_div;
  a.Lkv = max_seq_len;
  a.nk = nk;
  a.S = S;
  a.scale = scale;
  a.ln_lambda = ln_lambda;
  a.stats_only = stats_only ? 1 : 0;
  a.block_table = block_table;
  a.seq_lens = seq_lens;
  a.page_stride = page_stride;
  a.log2_page = log2_page;
  a.max_pages = max_pages;
  a.num_pages = num_pages;
  a.per_length = per_length ? 1 : 0;
  return launch_decode(a, G, true, grid, stats_only, o, lse, B * Hq,
                       static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------------------
// Decode with library-owned scratch (no allocation by anyone at call time)
// ---------------------------------------------------------------------------
// Some callers may not allocate device memory when they run the decode: an
// inference-engine plugin whose enqueue step is forbidden to allocate, or a
// latency-critical decode loop that cannot afford cudaMalloc's implicit
// device-wide synchronisation and has no workspace of its own to lend.  For
// them the split partials live in this fixed array, which the CUDA runtime
// places in device memory when the library is loaded: every GPU that loads
// the library keeps these bytes until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB per device
static __device__ __align__(256) unsigned char
    g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
// Per device: the context the address was looked up in, and the address.
// The array moves when its module is loaded again (after cudaDeviceReset,
// or in another context made current on the same device), so the address
// is looked up again whenever the current context differs.
void* g_noalloc_ctx[kMaxDevices] = {};
void* g_noalloc_ptr[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

CtxGetCurrentFn get_ctx_fn() {
  static CtxGetCurrentFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault,
                                &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(ptr);
  }
  return fn;
}

// Device address of g_noalloc_scratch on the current device.  In host code
// the array's name only stands in for the symbol; its device address must be
// asked of the runtime, with that device current: once per device and
// context (the first call after the context was created, or re-created).
blasst_status_t noalloc_scratch(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return BLASST_ERR_UNSUPPORTED_SHAPE;
  CtxGetCurrentFn ctx_fn = get_ctx_fn();
  if (!ctx_fn) {
    snprintf(g_last_error, sizeof g_last_error,
             "blasst_decode_noalloc: cuCtxGetCurrent is not available");
    return BLASST_ERR_CUDA;
  }
  CUcontext ctx = nullptr;
  if (ctx_fn(&ctx) != CUDA_SUCCESS) ctx = nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!ctx || !g_noalloc_ptr[dev] || g_noalloc_ctx[dev] != (void*)ctx) {
    // The runtime binds the device's primary context here if none is
    // current yet, so the context is read again afterwards.
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_status(e, "cudaGetSymbolAddress(scratch)");
    if (ctx_fn(&ctx) != CUDA_SUCCESS) ctx = nullptr;
    g_noalloc_ptr[dev] = p;
    g_noalloc_ctx[dev] = (void*)ctx;
  }
  *out = g_noalloc_ptr[dev];
  return BLASST_OK;
}
}  // namespace

blasst_status_t blasst_decode_noalloc(const void* q, const void* k_cache,
                                      const void* v_cache, void* o, float* lse,
                                      int B, int Hq, int Hkv, int Lkv, int d,
                                      float scale, float ln_lambda, int Bc,
                                      int num_splits,
                                      const blasst_skip_stats_t* skip_stats,
                                      void* stream) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Lkv < 1 || Bc < 1 || num_splits < 0)
    return BLASST_ERR_INVALID_ARG;
  const int S = num_splits == 0 ? blasst_decode_group_splits(B, Hq, Hkv, Lkv, Bc)
                                : num_splits;
  const size_t need = blasst_decode_workspace_size(B, Hq, d, S);
  if (o && need > kNoAllocScratchBytes) {
    snprintf(g_last_error, sizeof g_last_error,
             "blasst_decode_noalloc: these shapes need %zu bytes of split "
             "partials, the built-in scratch holds %zu (use blasst_decode with "
             "a caller workspace, or fewer splits)",
             need, kNoAllocScratchBytes);
    return BLASST_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  blasst_status_t rc = noalloc_scratch(&scratch);
  if (rc != BLASST_OK) return rc;
  // Nothing in the scratch needs clearing: the split kernel writes every
  // partial it later merges.
  return blasst_decode(q, k_cache, v_cache, o, lse, B, Hq, Hkv, Lkv, d, scale,
                       ln_lambda, Bc, S, scratch, kNoAllocScratchBytes,
                       skip_stats, stream);
}

// ---------------------------------------------------------------------------
// Prefill
// ---------------------------------------------------------------------------
blasst_status_t blasst_prefill(const void* q, const void* k, const void* v,
                               void* o, float* lse, int B, int Hq, int Hkv,
                               int Lq, int Lkv, int d, float scale, int causal,
                               float ln_lambda, int Br, int Bc,
                               const blasst_skip_stats_t* skip_stats,
                               void* stream) {
  return blasst_prefill_window(q, k, v, o, lse, B, Hq, Hkv, Lq, Lkv, d, scale,
                               causal, 0, ln_lambda, Br, Bc, skip_stats,
                               stream);
}

blasst_status_t blasst_prefill_window(const void* q, const void* k,
                                      const void* v, void* o, float* lse,
                                      int B, int Hq, int Hkv, int Lq, int Lkv,
                                      int d, float scale, int causal,
                                      int window, float ln_lambda, int Br,
                                      int Bc,
                                      const blasst_skip_stats_t* skip_stats,
                                      void* stream) {
  if (!q || !k || !v) return BLASST_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Lq < 1 || Lkv < 1 || Hq % Hkv != 0)
    return BLASST_ERR_INVALID_ARG;
  if (window < 0 || (window > 0 && !causal)) return BLASST_ERR_INVALID_ARG;
  if (window > 0 && Br != 128) return BLASST_ERR_UNSUPPORTED_SHAPE;
  if (!std::isfinite(scale) || !valid_ln_lambda(ln_lambda))
    return BLASST_ERR_INVALID_ARG;
  if (causal && Lq > Lkv) return BLASST_ERR_INVALID_ARG;
  if (!((d == 64 || d == 128) &&
        ((Br == 64 && Bc == 64) || (Br == 128 && Bc == 128))))
    return BLASST_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || (o && !aligned16(o)))
    return BLASST_ERR_MISALIGNED;
  blasst::PrefillProblem p;
  p.q = q;
  p.k = k;
  p.v = v;
  p.o = o;
  p.lse = lse;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Lq = Lq;
  p.Lkv = Lkv;
  p.d = d;
  p.scale = scale;
  p.causal = causal ? 1 : 0;
  p.ln_lambda = ln_lambda;
  p.Br = Br;
  p.Bc = Bc;
  p.counters = skip_stats ? skip_stats->counters : nullptr;
  p.mask = skip_stats ? skip_stats->mask : nullptr;
  p.margin = skip_stats ? skip_stats->margin : nullptr;
  p.window = window;
  cudaError_t e = blasst::launch_prefill(p, static_cast<cudaStream_t>(stream));
  return cuda_status(e, "prefill launch");
}

blasst_status_t blasst_decode_wide(const void* q, const void* k_cache,
                                   const void* v_cache, void* o, float* lse,
                                   int B, int Hq, int Hkv, int Lkv, int d,
                                   float scale, float ln_lambda, int Bc,
                                   int num_splits, void* workspace,
                                   size_t workspace_bytes,
                                   const blasst_skip_stats_t* skip_stats,
                                   void* stream) {
  if (!q || !k_cache || !v_cache) return BLASST_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Lkv < 1 || Hq % Hkv != 0 ||
      num_splits < 0)
    return BLASST_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !valid_ln_lambda(ln_lambda))
    return BLASST_ERR_INVALID_ARG;
  const int G = Hq / Hkv;
  if (d != blasst::kWideD || Bc != blasst::kWideBc || G > 128)
    return BLASST_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) ||
      (o && !aligned16(o)))
    return BLASST_ERR_MISALIGNED;
  const int nk = (Lkv + Bc - 1) / Bc;
  const int S = num_splits == 0 ? blasst_decode_wide_splits(B, Hkv, Lkv, Bc)
                                : num_splits;
  if (S < 1 || S > nk) return BLASST_ERR_INVALID_ARG;
  return wide_launch(q, k_cache, v_cache, o, lse, B, Hq, Hkv, Lkv, scale, 0,
                     G, ln_lambda, S, workspace, workspace_bytes, skip_stats,
                     stream);
}

int blasst_mla_decode_splits(int B, int L) {
  if (B < 1 || L < 1) return 1;
  const long long nk = (L + (long long)blasst::kMlaBc - 1) / blasst::kMlaBc;
  const long long per = 2LL * B;  // a cluster pair of CTAs per split
  // one CTA per SM: the split count with the least time in waves of SMs
  // (waves / splits), among those of at most two waves and 8 blocks or
  // more per split; the smaller on a tie (fewer partials to merge)
  const long long s_max = nk / 8 > 1 ? nk / 8 : 1;
  long long best = 1;
  double best_cost = 1e30;
  for (long long s = 1; s <= s_max && per * s <= 2LL * kNumSmB200; ++s) {
    const long long waves = (per * s + kNumSmB200 - 1) / kNumSmB200;
    const double cost = (double)waves / (double)s;
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = s;
    }
  }
  return (int)best;
}

size_t blasst_mla_decode_workspace_size(int B, int H, int num_splits) {
  if (B < 1 || H < 1 || num_splits < 1) return 0;
  const size_t rows = (size_t)B * H * num_splits;
  return ((rows * blasst::kMlaDv * 4 + 255) & ~(size_t)255) +
         ((rows * 4 + 255) & ~(size_t)255);
}

blasst_status_t blasst_mla_decode(const void* q, const void* cache, void* o,
                                  float* lse, int B, int H, int L, int d_qk,
                                  int d_v, float scale, float ln_lambda,
                                  int num_splits, void* workspace,
                                  size_t workspace_bytes,
                                  const blasst_skip_stats_t* skip_stats,
                                  void* stream) {
  if (!q || !cache) return BLASST_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || L < 1 || num_splits < 0) return BLASST_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !valid_ln_lambda(ln_lambda))
    return BLASST_ERR_INVALID_ARG;
  if (d_qk != blasst::kMlaDqk || d_v != blasst::kMlaDv ||
      H > blasst::kMlaRows)
    return BLASST_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(q) || !aligned16(cache) || (o && !aligned16(o)))
    return BLASST_ERR_MISALIGNED;
  const int nk = (L + blasst::kMlaBc - 1) / blasst::kMlaBc;
  const int S = num_splits == 0 ? blasst_mla_decode_splits(B, L) : num_splits;
  if (S < 1 || S > nk) return BLASST_ERR_INVALID_ARG;
  const long long grid = 2LL * B * S;  // cluster pairs
  if (grid > 0x7fffffffLL) return BLASST_ERR_UNSUPPORTED_SHAPE;
  const bool stats_only = (o == nullptr);
  blasst::MlaArgs a;
  memset(&a, 0, sizeof a);
  if (!stats_only) {
    const size_t need = blasst_mla_decode_workspace_size(B, H, S);
    if (!workspace || workspace_bytes < need) return BLASST_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
      return BLASST_ERR_MISALIGNED;
    const size_t rows = (size_t)B * H * S;
    a.o_part = static_cast<float*>(workspace);
    a.lse_part = reinterpret_cast<float*>(
        static_cast<char*>(workspace) +
        ((rows * blasst::kMlaDv * 4 + 255) & ~(size_t)255));
  }
  if (!blasst::encode_map(&a.tc, cache, blasst::kMlaDqk, L, B, 64))
    return cuda_status(cudaErrorInvalidValue, "mla tensor map");
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.counters = skip_stats ? skip_stats->counters : nullptr;
  a.mask = skip_stats ? skip_stats->mask : nullptr;
  a.B = B;
  a.H = H;
  a.L = L;
  a.nk = nk;
  a.S = S;
  a.scale = scale;
  a.ln_lambda = ln_lambda;
  a.stats_only = stats_only ? 1 : 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaFuncSetAttribute(blasst::mla_pair_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       blasst::MlaPairCfg::SMEM_ALLOC);
  if (e != cudaSuccess) return cuda_status(e, "mla attribute");
  blasst::mla_pair_kernel<<<(unsigned)grid, blasst::kMlaPairThreads,
                            blasst::MlaPairCfg::SMEM_ALLOC, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess || stats_only) return cuda_status(e, "mla split launch");
  blasst::mla_combine_kernel<<<(unsigned)((long long)B * H), 128, 0, st>>>(
      a.o_part, a.lse_part, static_cast<__nv_bfloat16*>(o), lse, S);
  return cuda_status(cudaGetLastError(), "mla merge launch");
}

size_t blasst_prefill_backward_workspace_size(int B, int Hq, int Lq, int d) {
  if (B < 1 || Hq < 1 || Lq < 1 || d != blasst::kBwdD) return 0;
  return blasst::bwd_workspace_bytes(B, Hq, Lq);
}

blasst_status_t blasst_prefill_backward(
    const void* q, const void* k, const void* v, const void* o,
    const void* dout, const float* lse, const unsigned char* mask, void* dq,
    void* dk, void* dv, int B, int Hq, int Hkv, int Lq, int Lkv, int d,
    float scale, int causal, int Br, int Bc, void* workspace,
    size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv)
    return BLASST_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Lq < 1 || Lkv < 1 || Hq % Hkv != 0)
    return BLASST_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return BLASST_ERR_INVALID_ARG;
  if (causal && Lq > Lkv) return BLASST_ERR_INVALID_ARG;
  if (d != blasst::kBwdD || Br != 128 || Bc != 128)
    return BLASST_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      !aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return BLASST_ERR_MISALIGNED;
  if (!workspace ||
      workspace_bytes < blasst::bwd_workspace_bytes(B, Hq, Lq))
    return BLASST_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return BLASST_ERR_MISALIGNED;
  blasst::BwdProblem p;
  p.q = q;
  p.k = k;
  p.v = v;
  p.o = o;
  p.dout = dout;
  p.lse = lse;
  p.mask = mask;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.workspace = static_cast<float*>(workspace);
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Lq = Lq;
  p.Lkv = Lkv;
  p.causal = causal ? 1 : 0;
  p.scale = scale;
  cudaError_t e = blasst::launch_backward(p, static_cast<cudaStream_t>(stream));
  return cuda_status(e, "backward launch");
}

// ---------------------------------------------------------------------------
// Calibration
// ---------------------------------------------------------------------------
namespace {

blasst_status_t sparsity_at(const blasst_calib_sample_t* s, double ln_lambda,
                            unsigned long long* counters, cudaStream_t st,
                            unsigned long long* vis, unsigned long long* skp) {
  blasst_status_t rc = blasst_skip_stats_reset(counters, st);
  if (rc != BLASST_OK) return rc;
  blasst_skip_stats_t stats = {counters, nullptr, nullptr};
  const float lnl = (float)ln_lambda;
  if (s->mode == 0) {
    rc = blasst_prefill(s->q, s->k, s->v, nullptr, nullptr, s->B, s->Hq,
                        s->Hkv, s->Lq, s->Lkv, s->d, s->scale, s->causal, lnl,
                        s->Br, s->Bc, &stats, st);
  } else {
    rc = blasst_decode(s->q, s->k, s->v, nullptr, nullptr, s->B, s->Hq, s->Hkv,
                       s->Lkv, s->d, s->scale, lnl, s->Bc, s->num_splits,
                       nullptr, 0, &stats, st);
  }
  if (rc != BLASST_OK) return rc;
  unsigned long long h[2] = {0, 0};
  cudaError_t e = cudaMemcpyAsync(h, counters, sizeof h, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_status(e, "calibration counters");
  *vis = h[0];
  *skp = h[1];
  return BLASST_OK;
}

}  // namespace

blasst_status_t blasst_calibrate(double target, const blasst_calib_sample_t* s,
                                 double tol, unsigned long long* counters_dev,
                                 blasst_calib_result_t* out, void* stream) {
  if (!s || !out || !counters_dev || !(target >= 0.0 && target < 1.0) ||
      !(tol >= 0.0) || (s->mode != 0 && s->mode != 1))
    return BLASST_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  memset(out, 0, sizeof *out);
  out->L = s->Lkv;
  // s(ln_lambda) is a non-decreasing step function.  Keep lo with s < target
  // and hi with s >= target; return hi.
  double lo = -64.0, hi = 0.0;
  unsigned long long v_hi = 0, k_hi = 0, v_lo = 0, k_lo = 0;
  blasst_status_t rc = sparsity_at(s, hi, counters_dev, st, &v_hi, &k_hi);
  int it = 1;
  if (rc != BLASST_OK) return rc;
  double s_hi = v_hi ? (double)k_hi / (double)v_hi : 0.0;
  auto fill = [&](double lnl, unsigned long long vv, unsigned long long kk) {
    out->ln_lambda = lnl;
    out->lambda = std::exp(lnl);
    out->a = out->lambda * (double)s->Lkv;
    out->visited = vv;
    out->skipped = kk;
    out->achieved = vv ? (double)kk / (double)vv : 0.0;
    out->iterations = it;
  };
  if (s_hi < target) {  // even ln(lambda) = 0 does not reach the target
    fill(hi, v_hi, k_hi);
    return BLASST_ERR_NO_CONVERGE;
  }
  rc = sparsity_at(s, lo, counters_dev, st, &v_lo, &k_lo);
  ++it;
  if (rc != BLASST_OK) return rc;
  const double s_lo = v_lo ? (double)k_lo / (double)v_lo : 0.0;
  if (s_lo >= target) {  // target reached everywhere (e.g. target 0)
    fill(lo, v_lo, k_lo);
    return BLASST_OK;
  }
  while (hi - lo > 1e-6 && s_hi - target > tol && it < 100) {
    const double mid = 0.5 * (lo + hi);
    unsigned long long vv = 0, kk = 0;
    rc = sparsity_at(s, mid, counters_dev, st, &vv, &kk);
    ++it;
    if (rc != BLASST_OK) return rc;
    const double sm = vv ? (double)kk / (double)vv : 0.0;
    if (sm >= target) {
      hi = mid;
      s_hi = sm;
      v_hi = vv;
      k_hi = kk;
    } else {
      lo = mid;
    }
  }
  fill(hi, v_hi, k_hi);
  return BLASST_OK;
}

double blasst_fit_a(int n, const double* lambdas, const int* lengths) {
  if (n < 1 || !lambdas || !lengths) return NAN;
  double acc = 0.0;
  for (int i = 0; i < n; ++i) acc += std::log(lambdas[i] * (double)lengths[i]);
  return std::exp(acc / n);
}

}  // extern "C"

/*
 * blasst.h -- C ABI of the BLASST attention forward for NVIDIA B200 (sm_100a).
 *
 * BLASST ("BLASST: Dynamic BLocked Attention Sparsity via Softmax
 * Thresholding"; gist.science summary, section 2 "Metodologia") is the
 * FlashAttention blockwise online-softmax forward in which KV block j is
 * skipped for a query tile when, for every row i of the tile,
 *
 *        m~_i(j) - m_i(j) < ln(lambda)                      (criterion)
 *
 * where m~_i(j) is the row's maximum scaled score inside block j and m_i(j)
 * the running row maximum over the blocks before j (section 2 "Criterio de
 * Pulo"; Hindi summary, section 2 "Core Insight").  A skipped block costs no
 * exp, no V load from HBM and no P.V product (section 2 "Acoes de
 * Otimizacao"); the decision is made per block for the whole tile (MLSys'26
 * reading notes, "design trade-offs": block skip vs token skip).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors are dense row-major with the head dimension innermost:
 *      prefill  q [B,Hq,Lq,d]   k, v [B,Hkv,Lkv,d]   o [B,Hq,Lq,d]
 *               lse [B,Hq,Lq]
 *      decode   q [B,Hq,d]      k, v [B,Hkv,Lkv,d]   o [B,Hq,d]  lse [B,Hq]
 *    q, k, v, o are bfloat16; lse is float32 (natural log of the kept
 *    entries' normaliser, m + ln l).  Query head hq reads KV head
 *    hq / (Hq / Hkv) (GQA; MQA is Hkv = 1, MHA is Hkv = Hq).
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never allocates device memory in these calls and never keeps a pointer
 *    after a call returns.  q, k, v, o must be 16-byte aligned.
 *  - scale multiplies q.k (usually 1/sqrt(d)); ln_lambda is in the same
 *    natural-log units as the scaled scores.  ln_lambda must be <= 0, or
 *    -INFINITY for the dense path (nothing is skipped).
 *  - Causal masking is bottom-right aligned: key c is visible to query r iff
 *    c <= r + (Lkv - Lq).  Causal calls need Lq <= Lkv.
 *  - stream is a cudaStream_t (NULL = legacy default stream).  Calls only
 *    enqueue work and return; results are ready when the stream is.
 *  - Errors are returned by value and never thrown.  Validation errors are
 *    detected before any work is enqueued; BLASST_ERR_CUDA reports a failed
 *    launch (the message of the last CUDA error is in blasst_last_error()).
 */
#ifndef BLASST_H
#define BLASST_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BLASST_OK = 0,
    BLASST_ERR_INVALID_ARG = 1,       /* null pointer, bad size, ln_lambda > 0 */
    BLASST_ERR_UNSUPPORTED_SHAPE = 2, /* d, Br/Bc or head ratio not built */
    BLASST_ERR_MISALIGNED = 3,        /* a tensor pointer not 16-byte aligned */
    BLASST_ERR_CUDA = 4,              /* a CUDA runtime call or launch failed */
    BLASST_ERR_TIMEOUT = 5,           /* a kernel gave up a bounded wait */
    BLASST_ERR_NO_CONVERGE = 6,       /* calibration bracket exhausted */
    BLASST_ERR_WORKSPACE = 7          /* workspace missing or too small */
} blasst_status_t;

/*
 * Skip statistics ("sparsity" = skipped / visited (tile, block) pairs).
 * The struct itself lives in HOST memory; its fields are DEVICE pointers.
 * Every field may be NULL (not written).
 *
 *  counters  device uint64[2]: [0] += visited pairs, [1] += skipped pairs.
 *            Kernels ADD to them (atomics), so one pair of counters can sum
 *            several calls; clear with blasst_skip_stats_reset().
 *  mask      optional device uint8 buffer (NULL = not written) receiving one
 *            decision per (tile, block): 0 not visited, 1 kept, 2 skipped.
 *            Prefill layout [B, Hq, ceil(Lq/Br), ceil(Lkv/Bc)];
 *            decode layout  [B, Hkv * T, ceil(Lkv/Bc)] with T decode tiles
 *            per KV head (1 when Hq/Hkv <= 8, else Hq/Hkv/8; a block
 *            belongs to exactly one split).  The caller allocates the whole
 *            layout: the library cannot check a device buffer's size.  Entries of pairs that are not visited are
 *            written as 0 by prefill only for tiles it runs; callers that
 *            need them zeroed clear the buffer first.
 *  margin    optional device float32 buffer, same layout as mask, receiving
 *            for every visited pair the margin of its decision
 *              max_r (m~_r - m_r) - ln_lambda
 *            (rows r of the tile with a visible key in the block; m_r the
 *            running max before the block, so the tile's first visited
 *            block gives +inf).  The pair is skipped exactly when the
 *            margin is < 0; a pair with |margin| < 1e-3 is a near-tie, whose
 *            decision a float32 rounding difference may flip.  Written by
 *            blasst_prefill / blasst_prefill_window, blasst_decode,
 *            blasst_decode_window, blasst_decode_noalloc and
 *            blasst_decode_paged with Hq/Hkv <= 8; other calls leave it
 *            untouched.  Computing it costs a max-reduction per pair, so
 *            pass NULL in timed calls.
 * A NULL blasst_skip_stats_t* disables all three.
 */
typedef struct {
    unsigned long long *counters;
    unsigned char *mask;
    float *margin;
} blasst_skip_stats_t;

/*
 * blasst_prefill -- prefill (many query tokens) forward with block skipping.
 *
 * The query rows are cut into tiles of Br rows and the keys into blocks of
 * Bc keys; each (tile, block) pair follows the online-softmax update and the
 * criterion above, blocks in ascending order.  The kernel issues the V
 * block's TMA load and the P.V tensor-core product only for kept pairs.
 *
 *  q, k, v     device bf16 inputs (layouts above)
 *  o           device bf16 output [B,Hq,Lq,d], or NULL for a statistics-only
 *              pass: decisions and counters are produced exactly as in a
 *              full call (the running max never depends on them) but no
 *              exp, V load or P.V product is executed and nothing is written
 *              to o/lse.
 *  lse         device float32 [B,Hq,Lq] or NULL
 *  d           64 or 128
 *  Br, Bc      (64, 64) or (128, 128)
 *  skip_stats  host pointer to the statistics struct, or NULL
 *
 * With 128 x 128 tiles and o given, ln_lambda = -INFINITY runs a dense
 * kernel built without the skip machinery (no vote, no decision hand-offs,
 * V loaded for every block without waiting for a decision).  Any finite
 * ln_lambda runs the skipping kernel; ln_lambda = -FLT_MAX skips nothing
 * either (no score gap reaches it), so it gives the same result through
 * the skipping kernel and measures what the vote costs on the dense path.
 */
blasst_status_t blasst_prefill(const void *q, const void *k, const void *v,
                               void *o, float *lse, int B, int Hq, int Hkv,
                               int Lq, int Lkv, int d, float scale, int causal,
                               float ln_lambda, int Br, int Bc,
                               const blasst_skip_stats_t *skip_stats,
                               void *stream);

/*
 * blasst_prefill_window -- blasst_prefill with a causal sliding window (the
 * attention variants the method is stated to support: MLSys'26 reading
 * notes, claims on sliding-window / GQA / MLA forms; gist.science summary,
 * section 3).  Query r attends to keys c with
 *     diag_r - window < c <= diag_r,   diag_r = r + Lkv - Lq
 * (the `window` keys ending at its bottom-right aligned diagonal).  A
 * (tile, block) pair none of whose entries is inside the window is not
 * visited (no load, no MMA, not counted, mask byte 0); a row with no
 * visible key in a visited block votes "skippable" there, so a block in
 * which a row sees its first keys is never skipped.
 *
 *  causal   must be 1 when window > 0
 *  window   >= 0; 0 (or >= Lkv) is blasst_prefill exactly
 *  Br, Bc   128, 128 when window > 0 (else BLASST_ERR_UNSUPPORTED_SHAPE)
 *  other arguments, layouts, ownership and errors as blasst_prefill.
 */
blasst_status_t blasst_prefill_window(const void *q, const void *k,
                                      const void *v, void *o, float *lse,
                                      int B, int Hq, int Hkv, int Lq, int Lkv,
                                      int d, float scale, int causal,
                                      int window, float ln_lambda, int Br,
                                      int Bc,
                                      const blasst_skip_stats_t *skip_stats,
                                      void *stream);

/*
 * blasst_prefill_backward -- gradients of a blasst_prefill forward with the
 * decisions that forward took held fixed (sparsity-aware fine-tuning with
 * the method active: gist.science summary, section 2, "Treinamento
 * Consciente de Esparsidade"; Hindi summary, algorithm design).  With its
 * decisions fixed the forward is softmax attention restricted, per query
 * tile, to its kept blocks; a decision is a step function, so its gradient
 * is that of the restricted attention:
 *     D_r = dO_r . O_r,  P = exp(scale q k^T - lse) on kept pairs (else 0),
 *     dV = P^T dO,  dS = P o (dO V^T - D),  dQ = scale dS K,
 *     dK = scale dS^T Q  (dK, dV summed over the G heads of a KV head).
 * Pairs the forward skipped or did not visit issue no load and no MMA.
 *
 *  q, k, v     the forward's inputs (device bf16, layouts as blasst_prefill)
 *  o, lse      the forward's outputs: o bf16 [B,Hq,Lq,d], lse float32
 *              [B,Hq,Lq] (required)
 *  dout        device bf16 [B,Hq,Lq,d], the gradient of o
 *  mask        the forward's decision bytes (skip_stats.mask layout
 *              [B,Hq,ceil(Lq/128),ceil(Lkv/128)], 1 = kept), or NULL for
 *              the dense backward (every visible pair kept)
 *  dq          device bf16 [B,Hq,Lq,d] (written; with a mask it first
 *              holds, as scratch, each key block's count of kept pairs and
 *              the order the key blocks run in: most kept pairs first; so
 *              dq must not overlap any input)
 *  dk, dv      device bf16 [B,Hkv,Lkv,d] (written)
 *  d = 128, Br = Bc = 128 (else BLASST_ERR_UNSUPPORTED_SHAPE); causal with
 *              Lq > Lkv is rejected
 *  workspace   device buffer of blasst_prefill_backward_workspace_size()
 *              bytes, 256-byte aligned, caller-owned (f32 dQ accumulator,
 *              the per-row D and lse * log2 e); contents need not be
 *              initialised
 * Asynchronous on `stream`; three kernel launches (five with a mask, for
 * the work order, unless B*Hkv*ceil(Lkv/128) exceeds 32768 or dq is too
 * small to hold 8 bytes per key block); allocates nothing.
 * Errors as blasst_prefill (BLASST_ERR_WORKSPACE for a missing or small
 * workspace).
 */
size_t blasst_prefill_backward_workspace_size(int B, int Hq, int Lq, int d);
blasst_status_t blasst_prefill_backward(
    const void *q, const void *k, const void *v, const void *o,
    const void *dout, const float *lse, const unsigned char *mask, void *dq,
    void *dk, void *dv, int B, int Hq, int Hkv, int Lq, int Lkv, int d,
    float scale, int causal, int Br, int Bc, void *workspace,
    size_t workspace_bytes, void *stream);

/*
 * blasst_decode -- one query token per sequence against a contiguous bf16
 * KV cache, split-KV with a log-sum-exp merge.
 *
 * The G = Hq/Hkv query heads sharing a KV head form the rows of one tile, so
 * every K and V byte read serves all G heads.  A tile has at most 8 rows:
 * for G = 16, 32, ... (MQA with many heads) the heads of a KV head are cut
 * into G/8 consecutive tiles of 8 heads, each with its own skip decisions.
 * For 16 <= G <= 128 one tensor-core CTA (tcgen05) scores all tiles of a
 * KV head (the V block is read when any tile keeps it; the rows of a tile
 * that skips it are left untouched); for G <= 8 a warp-level tensor-core
 * kernel (mma.sync, K and V by TMA) runs one CTA per (sequence, KV head,
 * split); for G = 256 the CUDA-core kernel runs one CTA per tile.  The
 * Lkv keys are cut into nk = ceil(Lkv/Bc) blocks and the blocks into
 * num_splits contiguous splits (split s covers blocks
 * [floor(s*nk/S), floor((s+1)*nk/S))).  Each split
 * runs the blockwise forward independently (its running max starts at
 * -inf), reading V only for kept blocks; a second kernel merges the splits:
 * lse = ln sum_s exp(lse_s), o = sum_s exp(lse_s - lse) o_s.
 *
 *  o           device bf16 [B,Hq,d], or NULL for a statistics-only pass
 *              (K is read and scored, V is never read)
 *  lse         device float32 [B,Hq] or NULL
 *  d           128, or 64 with Hq/Hkv <= 8;  Hq/Hkv a power of two up to
 *              256;  Bc = 64
 *  num_splits  >= 1, or 0 for the automatic choice
 *              blasst_decode_group_splits(B, Hq, Hkv, Lkv, 64)
 *  workspace   device buffer of at least blasst_decode_workspace_size()
 *              bytes (16-byte aligned) holding the per-split partials;
 *              caller-owned, contents need not be initialised.  May be NULL
 *              in a statistics-only pass.
 */
blasst_status_t blasst_decode(const void *q, const void *k_cache,
                              const void *v_cache, void *o, float *lse, int B,
                              int Hq, int Hkv, int Lkv, int d, float scale,
                              float ln_lambda, int Bc, int num_splits,
                              void *workspace, size_t workspace_bytes,
                              const blasst_skip_stats_t *skip_stats,
                              void *stream);

/*
 * blasst_decode_window -- blasst_decode with a sliding attention window (the
 * attention variants the method is stated to support: MLSys'26 reading
 * notes, claims on sliding-window / GQA / MLA forms; gist.science summary,
 * section 3).  The token at position Lkv - 1 attends only to keys
 * [max(0, Lkv - window), Lkv).  The 64-key blocks that hold them,
 * [jlo, nk) with jlo = floor(max(0, Lkv - window) / 64), are divided into the
 * splits as blasst_decode divides [0, nk) (split s covers
 * [jlo + floor(s (nk - jlo) / S), jlo + floor((s + 1)(nk - jlo) / S))); keys
 * of block jlo before the window are masked; blocks before jlo are neither
 * read nor counted, and their mask bytes are written 0 (not visited).
 *
 *  window       >= 0; 0 (or >= Lkv) is blasst_decode exactly
 *  num_splits   1 .. nk - jlo, or 0 = blasst_decode_group_splits(B, Hq,
 *               Hkv, Lkv - 64 jlo, 64)
 *  other arguments, layouts, ownership and errors as blasst_decode.
 */
blasst_status_t blasst_decode_window(const void *q, const void *k_cache,
                                     const void *v_cache, void *o, float *lse,
                                     int B, int Hq, int Hkv, int Lkv, int d,
                                     float scale, int window, float ln_lambda,
                                     int Bc, int num_splits, void *workspace,
                                     size_t workspace_bytes,
                                     const blasst_skip_stats_t *skip_stats,
                                     void *stream);

/*
 * blasst_decode_batched -- blasst_decode with the batched decision rule
 * (Hindi summary, section 2 "kernel optimisation": the Q.K products of
 * several blocks are formed before their V loads are decided, which keeps
 * the conditional V loads from stalling the pipeline).  With batch = 2 each
 * split's blocks are taken in pairs (j, j+1), both scored before either is
 * decided, and each is skipped iff for every head g of the tile
 *     m~_g(block) - max(m_g before the pair, m~_g(j), m~_g(j+1)) < ln lambda
 * where m_g is the max over all earlier blocks of the split.  The block
 * holding the pair's max is always kept; the rule skips every block the
 * sequential rule (blasst_decode) skips and possibly more, and each skipped
 * weight stays below lambda times the split's final max.
 *
 *  batch   1 (= blasst_decode) or 2 (else BLASST_ERR_UNSUPPORTED_SHAPE)
 *  other arguments, layouts, ownership and errors as blasst_decode.
 */
blasst_status_t blasst_decode_batched(const void *q, const void *k_cache,
                                      const void *v_cache, void *o, float *lse,
                                      int B, int Hq, int Hkv, int Lkv, int d,
                                      float scale, float ln_lambda, int Bc,
                                      int num_splits, int batch,
                                      void *workspace, size_t workspace_bytes,
                                      const blasst_skip_stats_t *skip_stats,
                                      void *stream);

/*
 * blasst_decode_noalloc -- blasst_decode for callers that may not allocate
 * device memory at call time and have no workspace to pass: for example an
 * inference-engine plugin whose enqueue step must not allocate, or a
 * latency-critical decode loop that cannot take cudaMalloc's implicit
 * device-wide synchronisation.  (No counterpart in the BLASST papers: this
 * is a deployment convenience of this library.)
 *
 * Same arguments and results as blasst_decode minus the workspace (the
 * automatic split count is blasst_decode's).  The
 * split partials go to an 8 MiB array that the library holds in device
 * memory on every GPU that loads it, until the process exits.
 *  - The first call on a device looks up that array's device address for
 *    the current device and context (once per device and context: a call
 *    made after cudaDeviceReset, or with another context current on the
 *    device, looks it up again, because the array then lives at a new
 *    address); make that first call before any stream capture.
 *  - Shapes whose partials exceed 8 MiB (B*Hq*S*(d+1) float32 values plus
 *    alignment, see blasst_decode_workspace_size) are rejected with
 *    BLASST_ERR_WORKSPACE and a message in blasst_last_error().
 *  - All calls on a device share the one array and it keeps the previous
 *    call's contents (nothing in it needs to start at zero).  Calls whose
 *    kernels may overlap on the GPU (different streams without ordering)
 *    race on it: serialise them, or use blasst_decode with one workspace per
 *    stream.
 */
blasst_status_t blasst_decode_noalloc(const void *q, const void *k_cache,
                                      const void *v_cache, void *o, float *lse,
                                      int B, int Hq, int Hkv, int Lkv, int d,
                                      float scale, float ln_lambda, int Bc,
                                      int num_splits,
                                      const blasst_skip_stats_t *skip_stats,
                                      void *stream);

/*
 * blasst_decode_paged -- blasst_decode over a paged KV cache with a block
 * table and per-sequence lengths: the cache form of serving engines.  The
 * MLSys'26 reading notes ("limitations and follow-up work") name end-to-end
 * runs on PagedAttention serving stacks as future work, and the
 * gist.science summary (section 3, "Integracao") the integration into
 * TensorRT-LLM and FlashInfer, whose decode kernels read such caches.
 *
 * Sequence b holds seq_lens[b] tokens; its token t lives in page
 * block_table[b * max_pages + t / page_size] at row t % page_size.  Pool
 * layout: page p of KV head h starts at element
 *     p * page_stride + h * page_size * d
 * of k_pages (and of v_pages), its page_size rows of d bf16 elements
 * contiguous -- [num_pages, Hkv, page_size, d] when page_stride =
 * Hkv * page_size * d; an interleaved pool [num_pages, 2, Hkv, page_size, d]
 * is v_pages = k_pages + Hkv * page_size * d with page_stride twice that.
 * Each sequence is decoded exactly as blasst_decode decodes a contiguous
 * cache of length seq_lens[b]: its ceil(L_b / 64) blocks of 64 keys (the
 * last one ragged) cut into the call's num_splits splits by the same
 * formula; a split with no blocks contributes nothing, and a sequence of
 * length 0 gives o = 0 and lse = -inf.
 *
 *  q, o, lse       as blasst_decode ([B,Hq,d] bf16, [B,Hq,d] bf16 or NULL
 *                  for statistics only, [B,Hq] float32 or NULL)
 *  k_pages,v_pages device bf16 pools, 16-byte aligned
 *  page_stride     elements between consecutive pages, >= Hkv*page_size*d,
 *                  a multiple of 8 (16 bytes)
 *  num_pages       pages in the pool (page ids must lie in [0, num_pages))
 *  page_size       tokens per page: 16, 32, 64, 128 or 256
 *  block_table     device int32 [B, max_pages]; entries past a sequence's
 *                  last page are never read
 *  seq_lens        device int32 [B], each in [0, max_seq_len]
 *  max_seq_len     host upper bound on seq_lens (1 .. max_pages*page_size):
 *                  sizes the split policy (blasst_decode_splits(B, Hkv,
 *                  max_seq_len, 64) when num_splits == 0) and the mask
 *  ln_lambda       per_length == 0: ln lambda (<= 0 or -INFINITY) for every
 *                  sequence.  per_length != 0: ln a of the law lambda = a/L
 *                  (finite or -INFINITY), and sequence b uses
 *                  ln lambda_b = min(0, ln a - ln L_b), L_b its own length
 *                  (gist.science summary, section 2 "Calibracao Automatica")
 *  d = 128, or 64 with Hq/Hkv <= 8; Hq/Hkv a power of two up to 256
 *                  (tiles as blasst_decode)
 *  num_splits      >= 1 (at most ceil(max_seq_len / 64)), or 0 = automatic
 *  workspace       as blasst_decode: blasst_decode_workspace_size(B, Hq, d,
 *                  resolved num_splits) bytes
 *  skip_stats      as blasst_decode; the mask layout is
 *                  [B, Hkv * T, ceil(max_seq_len / 64)] and blocks past a
 *                  sequence's end are not written
 * When the call has more (sequence, KV head, split) work items than the
 * GPU holds at once, a small kernel first sorts the sequences by length
 * into the workspace and the CTAs take the longest sequences' splits
 * first, so that the last wave holds the shortest splits.  Which CTA runs a
 * split changes nothing in what it computes: outputs, decisions and
 * counters are the same bits in any order.
 * The block table and the lengths live on the device, so they are checked
 * there: before any copy of a split is issued, its kernel checks its
 * sequence's length and every page id it will read.  A bad value is not
 * read through; the split is abandoned (the sequence's o and lse are then
 * undefined) and blasst_check_device_error() returns
 * BLASST_ERR_INVALID_ARG with the sequence, position and value in
 * blasst_last_error().
 */
blasst_status_t blasst_decode_paged(const void *q, const void *k_pages,
                                    const void *v_pages, long long page_stride,
                                    int num_pages, int page_size,
                                    const int *block_table, int max_pages,
                                    const int *seq_lens, int max_seq_len,
                                    void *o, float *lse, int B, int Hq,
                                    int Hkv, int d, float scale,
                                    float ln_lambda, int per_length,
                                    int num_splits, void *workspace,
                                    size_t workspace_bytes,
                                    const blasst_skip_stats_t *skip_stats,
                                    void *stream);

/* Bytes of decode workspace: B*Hq*S*(d+1) float32 values (the split
 * partials) and B int32 values (blasst_decode_paged's work order), each
 * region rounded up to 256.  num_splits must be the resolved value (>= 1). */
size_t blasst_decode_workspace_size(int B, int Hq, int d, int num_splits);

/* The automatic split count of the kernels that keep 3 CTAs per SM: every
 * blasst_decode_paged and blasst_decode_batched call, and blasst_decode
 * (window, no-alloc) for Hq/Hkv <= 8 or 256.  Pure function of its arguments
 * (so a reference can reproduce the masks, which depend on the splits): at
 * least two waves of (sequence, KV head, split) work items on a 148-SM B200
 * with 3 resident CTAs per SM, at least 8 blocks per split, and among the
 * counts up to twice that minimum the one that fills the last wave best
 * (fewest splits on ties).  Batch 32 x 8 KV heads at 32K keys gives 5;
 * batch 148 gives 1. */
int blasst_decode_splits(int B, int Hkv, int Lkv, int Bc);

/* The automatic split count of the tensor-core kernel for wide head groups
 * (2 CTAs per SM): blasst_decode_wide, and blasst_decode (window, no-alloc)
 * for 16 <= Hq/Hkv <= 128.  Pure function of its arguments: among the counts
 * with at least 8 blocks per split, the one that minimises
 * ceil(B*Hkv*S / 296) * (nk/S + 2) -- the waves of work items times one
 * item's blocks plus its fixed cost of about two blocks (q, partial write,
 * merge row) -- fewest splits on ties.  Batch 32 x 1 KV head at 32K keys
 * gives 9 (one wave). */
int blasst_decode_wide_splits(int B, int Hkv, int Lkv, int Bc);

/* The automatic split count of blasst_decode, blasst_decode_window and
 * blasst_decode_noalloc for Hq/Hkv query heads per KV head:
 * blasst_decode_wide_splits for 16 <= Hq/Hkv <= 128 with Bc = 64, else
 * blasst_decode_splits.  Returns 1 for invalid arguments. */
int blasst_decode_group_splits(int B, int Hq, int Hkv, int Lkv, int Bc);

/*
 * blasst_decode_wide -- blasst_decode on the tensor core for wide head
 * groups: all G = Hq/Hkv (1..128) query heads of a KV head form one tile
 * (the rows of 128 x 64 score and 128 x 128 P.V MMAs; G < 128 is padded),
 * with the decode criterion, V read only for kept blocks and the split/merge
 * of blasst_decode.  For MQA and large GQA ratios, where G x d FMAs per key
 * outgrow the memory time of the CUDA-core kernel.  Unlike blasst_decode
 * with G > 8 (tiles of 8 heads), the whole group votes together; the mask
 * layout is [B, Hkv, ceil(Lkv/64)].
 *
 *  d = 128, Bc = 64, 1 <= Hq/Hkv <= 128 (else UNSUPPORTED_SHAPE);
 *  num_splits 0 = blasst_decode_wide_splits(B, Hkv, Lkv, 64); other
 *  arguments, workspace (blasst_decode_workspace_size), ownership and
 *  errors as blasst_decode.
 */
blasst_status_t blasst_decode_wide(const void *q, const void *k_cache,
                                   const void *v_cache, void *o, float *lse,
                                   int B, int Hq, int Hkv, int Lkv, int d,
                                   float scale, float ln_lambda, int Bc,
                                   int num_splits, void *workspace,
                                   size_t workspace_bytes,
                                   const blasst_skip_stats_t *skip_stats,
                                   void *stream);

/*
 * blasst_mla_decode -- decode over a multi-head latent (MLA) cache: each
 * of the H query heads of a token scores the shared latent row c_t of every
 * key as scale * q_h . c_t (d_qk = 576: 512 latent + 64 rope dimensions)
 * and takes the latent part c_t[0:512] as value (the attention forms the
 * method is stated to support: MLSys'26 reading notes; gist.science
 * summary, section 3).  The H heads form one decode tile; blocks of 64 keys
 * with the decode criterion and online softmax per split (split s covers
 * blocks [floor(s*nk/S), floor((s+1)*nk/S))), merged by log-sum-exp as in
 * blasst_decode.  Only the P.V product and the exp are saved by a skip: the
 * value is part of the row the score already read.
 *
 *  q           device bf16 [B, H, 576]
 *  cache       device bf16 [B, L, 576] (one latent row per key)
 *  o           device bf16 [B, H, 512], or NULL for a statistics-only pass
 *  lse         device float32 [B, H] or NULL
 *  H           1..128;  d_qk = 576, d_v = 512 (else UNSUPPORTED_SHAPE)
 *  num_splits  >= 1 (at most ceil(L/64)), or 0 = blasst_mla_decode_splits
 *  workspace   blasst_mla_decode_workspace_size(B, H, resolved splits)
 *              bytes, 256-byte aligned, caller-owned (NULL allowed when o
 *              is NULL)
 *  skip_stats  counters as blasst_decode; mask layout [B, ceil(L/64)]
 * Asynchronous on `stream`; two kernel launches; allocates nothing.
 */
blasst_status_t blasst_mla_decode(const void *q, const void *cache, void *o,
                                  float *lse, int B, int H, int L, int d_qk,
                                  int d_v, float scale, float ln_lambda,
                                  int num_splits, void *workspace,
                                  size_t workspace_bytes,
                                  const blasst_skip_stats_t *skip_stats,
                                  void *stream);
/* Bytes of MLA decode workspace (split outputs and their lse). */
size_t blasst_mla_decode_workspace_size(int B, int H, int num_splits);
/* The automatic MLA split count.  A split runs on a pair of CTAs (a cluster
 * of 2, one CTA per SM); the count is the one with the fewest waves of SMs
 * per split among counts of at most two waves and at least 8 blocks per
 * split, the smaller on a tie. */
int blasst_mla_decode_splits(int B, int L);

/*
 * Calibration of the threshold lambda = a / L for a target sparsity
 * (gist.science summary, section 2 "Calibracao Automatica"; MLSys'26 reading
 * notes, observation 2: a is fitted on calibration data, not universal).
 *
 * The sparsity s(ln_lambda) of a fixed input is a non-decreasing step
 * function.  The routine bisects ln_lambda over [-64, 0] with
 * statistics-only passes of the chosen operation on the caller's sample and
 * returns the smallest ln_lambda found whose sparsity reaches the target
 * (within tol), together with a = lambda * L where L = Lkv of the sample.
 * It synchronises the stream once per bisection step.
 */
typedef struct {
    int mode;                   /* 0 = prefill, 1 = decode */
    const void *q, *k, *v;      /* device bf16 sample (layouts as above) */
    int B, Hq, Hkv, Lq, Lkv, d; /* Lq is ignored for decode */
    float scale;
    int causal;                 /* prefill only */
    int Br, Bc;                 /* Br ignored for decode */
    int num_splits;             /* decode only; 0 = automatic */
} blasst_calib_sample_t;

typedef struct {
    double ln_lambda;           /* calibrated threshold (natural log) */
    double lambda;              /* exp(ln_lambda) */
    double a;                   /* lambda * L */
    double achieved;            /* sparsity at ln_lambda */
    int L;                      /* the sample's Lkv */
    int iterations;             /* statistics-only passes run */
    unsigned long long visited, skipped; /* counts at ln_lambda */
} blasst_calib_result_t;

/*
 *  target        sparsity in [0, 1)
 *  tol           accepted |achieved - target| (e.g. 0.005); the search also
 *                stops when the ln_lambda bracket is narrower than 1e-6
 *  counters_dev  device uint64[2] scratch for the counters (caller-owned)
 *  out           host pointer receiving the result
 * Returns BLASST_ERR_NO_CONVERGE (with out filled with the closest value
 * reached from above) when no ln_lambda <= 0 reaches the target.
 */
blasst_status_t blasst_calibrate(double target, const blasst_calib_sample_t *sample,
                                 double tol, unsigned long long *counters_dev,
                                 blasst_calib_result_t *out, void *stream);

/* a of lambda = a / L fitted over n calibrations in log space:
 * a = exp(mean_i ln(lambda_i * L_i)). */
double blasst_fit_a(int n, const double *lambdas, const int *lengths);

/* cudaMemsetAsync of the two counters. */
blasst_status_t blasst_skip_stats_reset(unsigned long long *counters,
                                        void *stream);

/* Reads and clears the library's device error word for the current device
 * (set by a kernel that abandoned a bounded wait, or by the paged decode on
 * a bad length or page id).  Synchronises the device.  Returns BLASST_OK,
 * BLASST_ERR_TIMEOUT (a wait gave up: blasst_last_error() describes the
 * first one -- block, step, parity, slot) or BLASST_ERR_INVALID_ARG (a
 * device-resident argument was out of range: blasst_last_error() names the
 * sequence, the position and the value).  *where_out (may be NULL)
 * receives the code recorded first: 1..99 a wait, 100 a sequence length,
 * 101 a page id. */
blasst_status_t blasst_check_device_error(int *where_out);

/* Diagnostic: launches one CTA that waits on an mbarrier nothing arrives
 * at, giving up after limit_cycles (1 .. 4e9) SM clock cycles the way every
 * bounded wait of the library does.  The next blasst_check_device_error()
 * then returns BLASST_ERR_TIMEOUT with where = 99.  Nothing faults: the
 * context stays usable.  (Test support for the failure path; the BLASST
 * pages have no counterpart.) */
blasst_status_t blasst_selftest_wait_timeout(long long limit_cycles,
                                             void *stream);

const char *blasst_strerror(blasst_status_t status);

/* Text of the last CUDA error seen by this thread's calls ("" if none). */
const char *blasst_last_error(void);

/* Library version, e.g. "0.1.0". */
const char *blasst_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BLASST_H */

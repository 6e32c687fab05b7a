/*
 * CPU oracle for the BLASST attention forward -- TEST INFRASTRUCTURE ONLY.
 *
 * Only the test suite, the smoke check and the benchmark's CPU-baseline leg
 * may load or call this code.  The product library never links it and shares
 * no code with it.
 *
 * What it computes: the blockwise online-softmax attention forward with the
 * BLASST skip rule, written out step by step in float64 so that a reader can
 * check each step against the method's description:
 *
 *   - running row max m and normaliser l, rescaled when m grows
 *     ("BLASST: Dynamic BLocked Attention Sparsity via Softmax Thresholding",
 *      gist.science summary, section 2 "Estatisticas Online");
 *   - block j is negligible for row i when  m~_i(j) - m_i(j) < ln(lambda)
 *     (same page, section 2 "Criterio de Pulo"; Hindi summary, section 2
 *      "Core Insight");
 *   - a negligible block costs no exp, no V load and no P.V product
 *     (same pages, section 2 "Acoes de Otimizacao");
 *   - the decision is taken per block for the whole query tile
 *     (MLSys'26 reading notes, "design trade-offs": block skip vs token skip).
 *
 * Readings of points the pages leave open (documented in the design notes):
 *   - m is the running max over blocks before j (identical decisions to the
 *     after-update reading whenever ln(lambda) <= 0);
 *   - strict '<';
 *   - a tile skips block j only if EVERY row satisfies the criterion; a row
 *     whose entries in block j are all masked satisfies it trivially;
 *   - the first visited block (m = -inf) is never skipped;
 *   - a (tile, block) pair whose entries are all masked is not visited;
 *   - causal masking is bottom-right aligned: key c is visible to query r
 *     iff c <= r + (Lkv - Lq);
 *   - GQA: query head hq reads KV head hq / (Hq / Hkv);
 *   - decode split-KV: each split runs the algorithm independently
 *     (m restarts at -inf) over blocks [floor(s*nk/S), floor((s+1)*nk/S)),
 *     then the partials are merged by log-sum-exp;
 *   - lse is the natural-log normaliser of the kept entries, m + ln l.
 *
 * Tensors are row-major, innermost dimension last:
 *   prefill q [B,Hq,Lq,d], k/v [B,Hkv,Lkv,d]; decode q [B,Hq,d],
 *   k/v [B,Hkv,Lkv,d].  Inputs are raw bfloat16 bit patterns (uint16).
 */
#ifndef BLASST_ORACLE_H
#define BLASST_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Decision codes written to the per-(tile, block) mask. */
#define ORACLE_NOT_VISITED 0
#define ORACLE_KEPT 1
#define ORACLE_SKIPPED 2

/* bfloat16 bit pattern -> value (exact). */
double oracle_bf16_to_double(uint16_t h);

/*
 * Prefill forward for a list of query tiles.
 *
 * units:  n_units triples (b, hq, i); tile i covers query rows
 *         [i*Br, min((i+1)*Br, Lq)).
 * o:      [n_units][Br][d]   normalised output (rows past Lq are left 0)
 * lse:    [n_units][Br]      m + ln l (natural log); -inf for rows past Lq
 * mask:   [n_units][nk]      ORACLE_* decision per KV block (may be NULL)
 * margin: [n_units][nk]      max_r(m~_r - m_r) - ln_lambda for visited
 *                            pairs (+inf for the first visited block, NaN
 *                            for pairs not visited) (may be NULL)
 * counts: [2]                visited and skipped pairs, summed over units
 * ln_lambda = -INFINITY gives the dense forward.
 * Returns 0, or -1 on invalid arguments.
 */
int oracle_prefill(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                   int B, int Hq, int Hkv, int Lq, int Lkv, int d,
                   double scale, int causal, double ln_lambda, int Br, int Bc,
                   int n_units, const int32_t *units,
                   double *o, double *lse, uint8_t *mask, double *margin,
                   int64_t *counts, int n_threads);

/*
 * Prefill with a causal sliding window (the attention-variant row of the
 * method's supported forms): query r sees the `window` keys ending at its
 * diagonal, c in [diag_r - window + 1, diag_r] with diag_r = r + Lkv - Lq.
 * window = 0 is plain causal/non-causal attention (oracle_prefill); a
 * window needs causal = 1.  Blocks wholly outside every row's window are
 * not visited; a row with no visible key in a block votes "skippable" there.
 */
int oracle_prefill_window(const uint16_t *q, const uint16_t *k,
                          const uint16_t *v, int B, int Hq, int Hkv, int Lq,
                          int Lkv, int d, double scale, int causal,
                          int window, double ln_lambda, int Br, int Bc,
                          int n_units, const int32_t *units, double *o,
                          double *lse, uint8_t *mask, double *margin,
                          int64_t *counts, int n_threads);

/*
 * Decode forward: one query token per sequence, the G = Hq/Hkv query heads
 * of a KV head form the rows of one tile.
 *
 * o:        [B,Hq,d]     merged output
 * lse:      [B,Hq]       merged log-sum-exp
 * o_part:   [B,Hq,S,d]   per-split normalised output (may be NULL)
 * lse_part: [B,Hq,S]     per-split lse, -inf for an empty split (may be NULL)
 * mask:     [B,Hkv,nk]   ORACLE_* decision per block (may be NULL)
 * margin:   [B,Hkv,nk]   as for prefill (may be NULL)
 * counts:   [2]          visited and skipped (b, hkv, block) triples
 */
int oracle_decode(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                  int B, int Hq, int Hkv, int Lkv, int d, double scale,
                  double ln_lambda, int Bc, int num_splits,
                  double *o, double *lse, double *o_part, double *lse_part,
                  uint8_t *mask, double *margin, int64_t *counts,
                  int n_threads);

/*
 * Decode with a sliding window: the token (position Lkv - 1) sees keys
 * [max(0, Lkv - window), Lkv).  The blocks holding them,
 * [jlo, nk) with jlo = floor(max(0, Lkv - window) / Bc), are divided into
 * the S splits as oracle_decode divides [0, nk); blocks before jlo are not
 * visited.  window = 0 is oracle_decode.
 */
int oracle_decode_window(const uint16_t *q, const uint16_t *k,
                         const uint16_t *v, int B, int Hq, int Hkv, int Lkv,
                         int d, double scale, int window, double ln_lambda,
                         int Bc, int num_splits, double *o, double *lse,
                         double *o_part, double *lse_part, uint8_t *mask,
                         double *margin, int64_t *counts, int n_threads);

/*
 * Decode with the batched decision rule (the Hindi summary's "batched load
 * scheduling", section 2 kernel optimisation: several Q.K products are
 * formed before the V loads are decided).  Each split's blocks are taken in
 * batches of `batch` consecutive blocks; every block of a batch is judged
 * against Mb = max(max over all earlier blocks, max over the whole batch):
 *   skip(j) <=> for every head g:  mt_g(j) - Mb_g < ln_lambda.
 * Kept blocks update the online softmax as in oracle_decode.  batch = 1 is
 * oracle_decode exactly; a larger batch skips a superset of its blocks, and
 * every skipped weight stays below lambda times the split's final max.
 */
int oracle_decode_batched(const uint16_t *q, const uint16_t *k,
                          const uint16_t *v, int B, int Hq, int Hkv, int Lkv,
                          int d, double scale, double ln_lambda, int Bc,
                          int num_splits, int batch, double *o, double *lse,
                          double *o_part, double *lse_part, uint8_t *mask,
                          double *margin, int64_t *counts, int n_threads);

/*
 * Paged, variable-length decode (block-table indirection).
 *
 * Sequence b holds seq_lens[b] tokens.  Its token t lives in page
 * block_table[b * max_pages + t / page_size]; inside a page, KV head h holds
 * rows [h * page_size, (h + 1) * page_size) of d elements, and page p starts
 * p * page_stride elements into k_pool / v_pool.  The logical cache of each
 * (b, h) is gathered from the pool and decoded as oracle_decode decodes a
 * contiguous cache of length seq_lens[b]: S splits over the sequence's own
 * ceil(L_b / Bc) blocks, empty splits contribute nothing, and an empty
 * sequence gives o = 0 and lse = -inf.
 *
 * per_length != 0: ln_lambda holds ln a (any finite value, or -inf) and
 * sequence b uses
 *   ln lambda_b = min(0, ln a - ln L_b)       (lambda = a / L, L its length)
 * per_length == 0: ln_lambda <= 0 (or -inf) for every sequence.
 * mask / margin: [B,Hkv,nk_max]; blocks past a sequence's end stay
 * ORACLE_NOT_VISITED / NaN.
 * Returns -1 on invalid arguments, including a length outside
 * [0, max_pages * page_size] or a page id outside [0, num_pages).
 */
int oracle_decode_paged(const uint16_t *q, const uint16_t *k_pool,
                        const uint16_t *v_pool, int64_t page_stride,
                        int num_pages, int page_size,
                        const int32_t *block_table, int max_pages,
                        const int32_t *seq_lens, int B, int Hq, int Hkv, int d,
                        double scale, double ln_lambda, int per_length, int Bc,
                        int num_splits, int nk_max, double *o, double *lse,
                        double *o_part, double *lse_part, uint8_t *mask,
                        double *margin, int64_t *counts, int n_threads);

/*
 * Log-sum-exp merge of S partial results for n rows:
 *   lse = ln sum_s exp(lse_s),  o = sum_s exp(lse_s - lse) * o_s.
 * o_part [n][S][d], lse_part [n][S]; o [n][d], lse [n].
 */
void oracle_combine(const double *o_part, const double *lse_part, int n,
                    int S, int d, double *o, double *lse);

/* First block of split s when nk blocks are divided into S splits. */
int oracle_split_begin(int nk, int S, int s);

#ifdef __cplusplus
}
#endif

#endif

/*
 * vark.h -- C ABI of the head-scale KV-cache pruning library for next-scale
 * (VAR) transformers (HeatKV-style), B200 / sm_100a.
 *
 * Sources, cited by page title and section:
 *   [HeatKV] "HeatKV: Head-tuned KV-cache Compression for Visual
 *            Autoregressive Modeling" project page: Abstract; Method steps
 *            1-5 (calibration prompts, per-(layer, head, source scale, future
 *            scale) attention aggregation, S-CAS ranking, budget allocation
 *            with retained sink scales, static schedule at inference);
 *            Table 1 (budgets as fractions of the full cache).
 *   [Review] machine review page of the HeatKV paper (arXiv 2605.14877):
 *            Figure 3 caption (tokens of a scale in raster order), Figure 4
 *            caption (Algorithm 1, BINARY-HEATKV with GREEDYEARLYPRUNING).
 *   [AMS-KV] "AMS-KV: Adaptive KV Caching in Multi-Scale Visual
 *            Autoregressive Transformers" listing: Abstract (attending to the
 *            local scale matters most; condensed early scales).
 *   [VAR-Q]  VAR-Q summary page: Key Contributions ((block, channel)
 *            quantisation groups, bit packing), Main Findings (INT4 / INT3
 *            quality), Why This Matters (composes with eviction).
 *
 * Conventions shared by every call
 *   - bf16 tensors are passed as `const uint16_t*` holding raw bf16 bits.
 *   - "dev" pointers are CUDA device pointers, "host" pointers host memory.
 *     The caller owns all memory; the library allocates nothing, keeps no
 *     state between calls and is safe to call from several host threads.
 *   - Device calls are asynchronous on `stream` (a cudaStream_t passed as
 *     void*; NULL = the legacy default stream).  Host calls are synchronous.
 *   - Every call returns a status: VARK_OK (0) or a negative VARK_E_* code.
 *     On an argument error nothing is launched and no output is touched.
 *   - Device pointers and row strides must be 16-byte aligned (VARK_E_ALIGN).
 *   - Failure-detection test hook (attention calls only; unset in normal use):
 *     VARK_TEST_WAIT_LIMIT_MS shortens the kernels' bounded waits (default 2 s)
 *     and VARK_TEST_WITHHOLD_KV_TILE=j makes each CTA's loader stop before key
 *     tile j, so waits on it run out and the call reports VARK_E_TIMEOUT
 *     through *dev_status while the CUDA context stays usable.
 *   - Scale lists: `sides[S]` (host) gives the side of each square token map,
 *     ascending; scale s holds n_s = sides[s]^2 tokens, token maps are stored
 *     scale after scale, raster order inside a scale, so
 *     off_s = sum_{s'<s} n_s', T = sum_s n_s.  1 <= S <= VARK_MAX_SCALES.
 *   - Logit of query i and key j of head h:
 *       x_ij = tau[h] * (q_i . k_j) / sqrt(D) + bias[h][scale(j)]
 *     (bias may be NULL = 0).  Softmax over the keys a query sees; fp32
 *     accumulation on bf16 inputs; outputs rounded to bf16 (RNE).
 *
 * Memory layout of the compacted (pruned) cache, defined by this library:
 *   R[l][h]          = sum_s keep[l][h][s] * n_s       rows kept by head h
 *   R_l              = sum_h R[l][h]                   rows per batch element
 *   head_off[l][h]   = sum_{h'<h} R[l][h']
 *   seg_off[l][h][s] = sum_{s'<s} keep[l][h][s'] * n_s'  if kept, else -1
 *   past_len[l][h][k]= sum_{s<k} keep[l][h][s] * n_s
 *   layer_base[l]    = sum_{l'<l} B * R_l' * D           (elements, L+1 entries)
 *   Layer l's compacted K (and V) is a [B][R_l][D] bf16 block at element
 *   layer_base[l]; token t of kept scale s of (b, h) is row
 *   b*R_l + head_off[l][h] + seg_off[l][h][s] + t of that block.
 */
#ifndef VARK_H
#define VARK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define VARK_MAX_SCALES 32

enum vark_status {
  VARK_OK = 0,
  VARK_E_ARG = -1,      /* null pointer, negative size or otherwise bad argument */
  VARK_E_SHAPE = -2,    /* unsupported shape (e.g. D not 64/128, S out of range, size overflow) */
  VARK_E_ALIGN = -3,    /* pointer or stride not 16-byte aligned */
  VARK_E_BUDGET = -4,   /* the sink scales alone exceed the requested budget */
  VARK_E_CUDA = -5,     /* a CUDA runtime / driver call failed (launch, tensor map) */
  VARK_E_TIMEOUT = -6,  /* a bounded device wait gave up; written to *dev_status */
  VARK_E_DEVICE = -7    /* the current device is not an sm_100 part */
};

/* Human-readable name of a status code (static string, never NULL). */
const char* vark_status_string(int status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int vark_version(void);

/*
 * vark_scas_accumulate -- S-CAS calibration attention of one layer.
 * [HeatKV] Method step 2: attention probabilities aggregated for each layer,
 * head, source scale and future (query) scale.
 *
 * Block-causal multi-scale attention: a query of scale k attends to every key
 * of scales 0..k (its own scale included, [Review] Figure 3 caption).  For
 * every query row i of scale k and source scale s <= k the probability mass
 * m_i(s) = sum_{j in scale s} p_ij is reduced over the B * n_k rows of scale k
 * and their MEAN is ADDED to mass[h][s][k]:
 *     mass[h][s][k] += (1 / (B * n_k)) * sum_{b, i in scale k} m_i(s)
 * With calibration seeds folded into the batch one call already averages the
 * seeds; several calls accumulate (divide by the call count when finalising).
 *
 *   q, k, v    dev  bf16 [B][H][T][D], contiguous.
 *   B, H       batch (calibration seeds) and heads, >= 1.
 *   D          head dimension, 64 or 128.
 *   S, sides   host scale list (see conventions).
 *   tau        dev  fp32 [H] per-head temperature.
 *   bias       dev  fp32 [H][S] additive logit bias per source scale, or NULL.
 *   mass       dev  fp32 [H][S][S], indexed [h][s][k]; accumulated with fp32
 *              atomics (one per (h, s, k) per CTA): entries s > k untouched.
 *   out        dev  bf16 [B][H][T][D] attention output O, or NULL to skip it:
 *              then v is not read and no PV product is formed (S-CAS only;
 *              the mass is the same up to fp32 summation order).
 *   dev_status dev  int32, required; the caller sets it to 0 before the call;
 *              a kernel that gives up a bounded wait stores VARK_E_TIMEOUT.
 * Limits: the per-row mass partials of S scales live in shared memory, so
 *   with D = 128 at most 30 scales fit the 227 KB a CTA may use (D = 64: all
 *   VARK_MAX_SCALES); more return VARK_E_SHAPE before any device call.
 * Errors: VARK_E_ARG, VARK_E_SHAPE, VARK_E_ALIGN, VARK_E_CUDA, VARK_E_DEVICE.
 */
int vark_scas_accumulate(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                         int B, int H, int D, int S, const int32_t* sides,
                         const float* tau, const float* bias,
                         float* mass, uint16_t* out, int32_t* dev_status, void* stream);

/*
 * vark_scas_finalize -- host.  [HeatKV] Abstract / Method step 3: the
 * Scale-dependent Cumulative Attention Score of a (layer, head, source scale):
 *     scas[l][h][s] = (1 / n_calls) * sum_{k > s} mass[l][h][s][k]
 * i.e. the attention mass a head puts on scale s, summed over the future scales
 * that read it (the last scale scores 0).
 *   mass  host fp32 [L][H][S][S] as accumulated by vark_scas_accumulate
 *         (one [H][S][S] block per layer) over n_calls calls per layer.
 *   scas  host fp64 [L][H][S] output.
 * Errors: VARK_E_ARG (null, n_calls < 1), VARK_E_SHAPE.
 */
int vark_scas_finalize(const float* mass, int L, int H, int S, int n_calls, double* scas);

/*
 * vark_build_schedule -- host.  [HeatKV] Method steps 3-4 and Abstract: remove
 * the lowest-ranked head-scale pairs until a user-selected memory budget is met,
 * always retaining the early sink scales; one static schedule per budget.
 *
 *   F = L * H * T tokens (the whole cache at the end of generation).
 *   Candidates: every (l, h, s) with s >= n_sinks, in ascending order of
 *   (scas[l][h][s], l, h, s) -- ties broken by index.  Pairs are dropped in
 *   that order until kept * 10000 <= budget_bp * F (the first point where the
 *   budget holds; equality meets it).  The local scale of a query is attended
 *   from the dense cache at inference, so it is not exempt here.
 *
 *   scas       host fp64 [L][H][S] (finite).
 *   budget_bp  budget in basis points of F, 0..10000 (10000 keeps everything).
 *   n_sinks    number of leading sink scales never dropped, 0..S.
 *   keep       host uint8 [L][H][S] output, 1 = retained.
 * Limits: L * H <= 2^24 and F * 10000 < 2^63 (the budget test is exact int64
 *   arithmetic); larger shapes return VARK_E_SHAPE before scas is read.
 * Errors: VARK_E_ARG (null, non-finite scas, budget > 10000), VARK_E_SHAPE,
 *         VARK_E_BUDGET (the sinks alone exceed the budget; keep untouched).
 */
int vark_build_schedule(const double* scas, int L, int H, int S, const int32_t* sides,
                        uint32_t budget_bp, int n_sinks, uint8_t* keep);

/*
 * vark_build_offsets -- device.  Offset tables of the ragged per-head layout
 * (see the layout block above) from a keep schedule.
 *   keep        dev uint8 [L][H][S] (0 / non-zero).
 *   B, D        batch and head dimension used for layer_base.
 *   head_off    dev int32 [L][H]      out
 *   seg_off     dev int32 [L][H][S]   out (-1 for dropped scales)
 *   past_len    dev int32 [L][H][S]   out
 *   layer_base  dev int64 [L + 1]     out (elements; layer_base[L] = total)
 * Limits: L * H <= 16384, every R_l * B fits in int32.
 * Errors: VARK_E_ARG, VARK_E_SHAPE, VARK_E_ALIGN, VARK_E_CUDA.
 */
int vark_build_offsets(const uint8_t* keep, int L, int H, int S, const int32_t* sides, int B, int D,
                       int32_t* head_off, int32_t* seg_off, int32_t* past_len, int64_t* layer_base,
                       void* stream);

/*
 * vark_compact_kv -- device.  Applies a keep schedule ([HeatKV] Method step 5):
 * for every (l, b, h, s) with keep[l][h][s] the K and V rows [off_s, off_s+n_s)
 * of (l, b, h) are copied, bit for bit, to their place in the compacted layout.
 * Dropped scales are not read.  One launch covers all layers.
 *   k, v         dev bf16, layer l's dense cache is the [B][H][T][D] block at
 *                element l * layer_stride (layer_stride >= B*H*T*D).
 *   keep, head_off, seg_off, layer_base   dev tables from vark_build_offsets.
 *   kc, vc       dev bf16 outputs of layer_base[L] elements each.
 * Errors: VARK_E_ARG, VARK_E_SHAPE (D % 8 != 0), VARK_E_ALIGN, VARK_E_CUDA.
 */
int vark_compact_kv(const uint16_t* k, const uint16_t* v, int64_t layer_stride,
                    int L, int B, int H, int S, int D, const int32_t* sides,
                    const uint8_t* keep, const int32_t* head_off, const int32_t* seg_off,
                    const int64_t* layer_base, uint16_t* kc, uint16_t* vc, void* stream);

/*
 * vark_pruned_attention -- device.  Pruned-cache attention of one layer
 * ([HeatKV] Method step 5 with the head-specific schedule of the Abstract;
 * [AMS-KV] Abstract: the local scale is always attended).  A query of scale k
 * of head h attends to that head's retained past scales s < k (ascending,
 * read from the compacted cache: past_len[h][k] rows starting at row
 * b*R_l + head_off[h]) followed by all n_k rows of its own scale k (read from
 * the dense cache).  Online-softmax attention, fp32 accumulation.
 *
 *   q            dev bf16 queries: [B][H][T][D] when query_scale = -1 (every
 *                scale), or [B][H][n_k][D] for query_scale = k.
 *   kc, vc       dev bf16 this layer's compacted block, [B][R_l][D] with
 *                kc_rows = B * R_l rows (kc, vc point at layer_base[l]).
 *   k_dense, v_dense  dev bf16 [B][H][T][D] this layer's dense cache (only
 *                the local-scale rows are read).
 *   head_off     dev int32 [H]     this layer's row of the offset tables
 *   seg_off      dev int32 [H][S]  (used for the bias of compacted keys)
 *   past_len     dev int32 [H][S]
 *   tau, bias    dev fp32 [H] and [H][S] (bias may be NULL).
 *   out          dev bf16, same shape as q.
 *   dev_status   dev int32, required (see vark_scas_accumulate).
 * Errors: VARK_E_ARG, VARK_E_SHAPE, VARK_E_ALIGN, VARK_E_CUDA, VARK_E_DEVICE.
 */
int vark_pruned_attention(const uint16_t* q, const uint16_t* kc, const uint16_t* vc, int64_t kc_rows,
                          const uint16_t* k_dense, const uint16_t* v_dense,
                          int B, int H, int S, int D, const int32_t* sides, int query_scale,
                          const int32_t* head_off, const int32_t* seg_off, const int32_t* past_len,
                          const float* tau, const float* bias,
                          uint16_t* out, int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * Generation order.  [HeatKV] Method step 5: the static schedule keeps cache use
 * within budget as new scales are generated.  Scale k is generated, its queries
 * attend to the cache built so far plus scale k itself, then scale k's retained
 * blocks are appended to the compacted cache.  The compacted buffers use the
 * final layout of vark_build_offsets from the start (every segment has its
 * final place); rows that no append has written yet must hold finite values,
 * so zero-initialise kc / vc once before the first scale.
 * ------------------------------------------------------------------------- */

/*
 * vark_append_scale -- device.  Appends scale `scale` of every layer: for each
 * (l, b, h) with keep[l][h][scale], copies the n_k rows of the new scale's K and
 * V to row b*R_l + head_off[l][h] + seg_off[l][h][scale] of layer l's block.
 *   k_new, v_new  dev bf16, layer l's new-scale block [B][H][n_k][D] at element
 *                 l * layer_stride (layer_stride >= B*H*n_k*D).
 *   other arguments as vark_compact_kv.
 * Appending scales 0..S-1 in turn leaves kc / vc equal to vark_compact_kv's.
 * Errors: VARK_E_ARG, VARK_E_SHAPE, VARK_E_ALIGN, VARK_E_CUDA.
 */
int vark_append_scale(const uint16_t* k_new, const uint16_t* v_new, int64_t layer_stride,
                      int L, int B, int H, int S, int D, const int32_t* sides, int scale,
                      const uint8_t* keep, const int32_t* head_off, const int32_t* seg_off,
                      const int64_t* layer_base, uint16_t* kc, uint16_t* vc, void* stream);

/*
 * vark_pruned_attention_step -- device.  Pruned attention of one layer for the
 * queries of scale `scale` while that scale is generated: keys = the head's
 * retained past scales s < scale (compacted, past_len[h][scale] rows) followed
 * by the n_k rows of the new scale itself ([AMS-KV] Abstract: the local scale
 * is always attended).  Identical arithmetic to vark_pruned_attention with
 * query_scale = scale; only the local scale's K / V come as their own block.
 *   q            dev bf16 [B][H][n_k][D]
 *   k_local, v_local  dev bf16 [B][H][n_k][D], the new scale's keys / values
 *   out          dev bf16 [B][H][n_k][D]
 *   other arguments as vark_pruned_attention.
 * Errors: as vark_pruned_attention.
 */
int vark_pruned_attention_step(const uint16_t* q, const uint16_t* kc, const uint16_t* vc, int64_t kc_rows,
                               const uint16_t* k_local, const uint16_t* v_local,
                               int B, int H, int S, int D, const int32_t* sides, int scale,
                               const int32_t* head_off, const int32_t* seg_off, const int32_t* past_len,
                               const float* tau, const float* bias,
                               uint16_t* out, int32_t* dev_status, void* stream);

/*
 * vark_cache_size_after_layer -- host.  Cache-size accounting while scales are
 * generated ([Review] Appendix A, Algorithm 2 CACHESIZEAFTERLAYER(k, l, G_k,
 * G_k-1, E_k); its body is truncated on the page).  Reading for a static
 * schedule (G_k = G_k-1 = the dropped pairs, E_k = scale k's entries): during
 * scale k the layers run in order, so after layer l the layers 0..l hold their
 * retained scales <= k and the layers l+1.. their retained scales < k.
 *   bytes  host int64 [S][L]: bytes[k][l] = retained K + V bytes (bf16) held
 *          after layer l during scale k; bytes[S-1][L-1] = 2 * 2 * layer_base[L].
 *   keep   host uint8 [L][H][S].
 * Limits: L * H * T * B * D * 4 < 2^63.
 * Errors: VARK_E_ARG, VARK_E_SHAPE.
 */
int vark_cache_size_after_layer(const uint8_t* keep, int L, int H, int S, const int32_t* sides, int B, int D,
                                int64_t* bytes);

/*
 * vark_rank_stability -- host.  [HeatKV] Results (S-CAS rankings remain stable
 * with a small calibration set); [Review] Figure 6 caption (stability of S-CAS
 * head-scale rankings across calibration runs).  Compares the S-CAS of two
 * calibration runs on disjoint seed sets over the candidate pairs
 * (l, h, s >= n_sinks):
 *   spearman      Pearson correlation of the two vectors of average ranks
 *                 (ties share the mean of their positions); 0 if either is
 *                 constant;
 *   drop_jaccard  |D_a & D_b| / |D_a | D_b| of the pairs each run's
 *                 vark_build_schedule drops at budget_bp (1 if neither drops).
 *   scas_a, scas_b  host fp64 [L][H][S], finite.
 * Limits: as vark_build_schedule.
 * Errors: VARK_E_ARG, VARK_E_SHAPE (n_sinks >= S), VARK_E_BUDGET.
 */
int vark_rank_stability(const double* scas_a, const double* scas_b, int L, int H, int S, const int32_t* sides,
                        uint32_t budget_bp, int n_sinks, double* spearman, double* drop_jaccard);

/* ---------------------------------------------------------------------------
 * Time-varying schedule: BINARY-HEATKV with GREEDYEARLYPRUNING.  [Review]
 * Figure 4 caption (Algorithm 1): per source scale i an order O_i ranks the
 * (layer, head) squares from least to most dependent on scale i; after scale k,
 * G_k = union over i <= k of the length-N_k prefixes of O_i must be absent.
 * [HeatKV] Method step 5: cache use stays within the budget as scales are
 * generated.  The pages leave N_k undefined; this library's reading: the
 * budget is absolute (budget_bp / 10000 of the final full cache) and N_k is
 * the smallest non-decreasing prefix length under which the cache after step k
 * (sink scales of every head, non-sink scales <= k of the heads outside the
 * prefixes) fits it.  Cache held after step k:
 *     keep_k[l][h][i] = (i <= k) and (evict_step[l][h][i] > k).
 * ------------------------------------------------------------------------- */

/*
 * vark_build_early_pruning_schedule -- host.
 *   scas        host fp64 [L][H][S]; O_i = ascending (scas[l][h][i], l, h).
 *   prefix_len  host int32 [S] out: N_k (0 while no non-sink scale exists).
 *   evict_step  host uint8 [L][H][S] out: first step k >= i at which (l, h, i)
 *               must be absent, 255 if it stays to the end (always 255 for
 *               sink scales).  S <= 254, L * H <= INT32_MAX, F * 10000 < 2^63.
 * Errors: VARK_E_ARG, VARK_E_SHAPE, VARK_E_BUDGET (sinks alone over budget).
 */
int vark_build_early_pruning_schedule(const double* scas, int L, int H, int S, const int32_t* sides,
                                      uint32_t budget_bp, int n_sinks, int32_t* prefix_len, uint8_t* evict_step);

/*
 * vark_recompact_kv -- device.  Moves a compacted cache to the layout of a
 * smaller (or shifted) retained set, e.g. keep_k after evictions: for every
 * (l, b, h, s) with keep_new[l][h][s] and s < max_scale, copies the rows from
 * the old layout (old tables) to the new one (tables of vark_build_offsets on
 * keep_new).  Pairs absent from the old layout (seg_off_old < 0) are skipped.
 * Source and destination buffers must differ.
 * Errors: VARK_E_ARG, VARK_E_SHAPE, VARK_E_ALIGN, VARK_E_CUDA.
 */
int vark_recompact_kv(const uint16_t* kc_old, const uint16_t* vc_old, const int32_t* head_off_old,
                      const int32_t* seg_off_old, const int64_t* layer_base_old,
                      int L, int B, int H, int S, int D, const int32_t* sides, int max_scale,
                      const uint8_t* keep_new, const int32_t* head_off_new, const int32_t* seg_off_new,
                      const int64_t* layer_base_new, uint16_t* kc_new, uint16_t* vc_new, void* stream);

/* ---------------------------------------------------------------------------
 * Quantised retained cache (int8).  [VAR-Q] summary page: KV quantisation for
 * visual AR models with groups indexed by (block, channel), block boundaries
 * given by the generation loop, composable with eviction.  Here a block is one
 * retained scale of one (layer, batch, head) and every channel d of it has one
 * absmax a (fp32); code = rint(x / (a / 127)) clamped to [-127, 127] (IEEE fp32
 * division, round half to even; a = 0 gives code 0); x' = code * (a / 127),
 * rounded to bf16.  Codes sit at the element positions of the compacted layout
 * (one byte each); absmax tables are [L][B][H][S][D] fp32 (entries of dropped
 * scales are 0).
 * ------------------------------------------------------------------------- */

/*
 * vark_quantize_kv_int8 -- device.  Compaction with quantisation: like
 * vark_compact_kv, but writes int8 codes to kq / vq (layer_base[L] bytes each)
 * and the per-(block, channel) absmax to k_absmax / v_absmax.  Each kept block
 * is read from HBM once (blocks of more than 1024 rows are split over the CTAs
 * of a thread-block cluster, which exchange their partial maxima); the code
 * pass re-reads the rows from L2.  k, v, kq, vq, k_absmax, v_absmax 16-byte
 * aligned; layer_stride a multiple of 8.  Non-finite inputs: a NaN in a block
 * makes that channel's absmax NaN (magnitude bits compare above infinity).
 * Errors: VARK_E_ARG, VARK_E_SHAPE (D % 8 != 0, D > 512, H > 2048), VARK_E_ALIGN,
 * VARK_E_CUDA.
 */
int vark_quantize_kv_int8(const uint16_t* k, const uint16_t* v, int64_t layer_stride,
                          int L, int B, int H, int S, int D, const int32_t* sides,
                          const uint8_t* keep, const int32_t* head_off, const int32_t* seg_off,
                          const int64_t* layer_base, int8_t* kq, int8_t* vq,
                          float* k_absmax, float* v_absmax, void* stream);

/*
 * vark_dequantize_layer_int8 -- device.  Expands one layer's int8 codes back to
 * its bf16 compacted block (the input of vark_pruned_attention), e.g. into a
 * one-layer buffer just before that layer's attention.
 *   kq, vq        dev int8, the layer's codes (kq + layer_base[l]), kc_rows rows.
 *   k_absmax, v_absmax  dev fp32 [B][H][S][D], the layer's absmax tables.
 *   head_off, seg_off   dev int32 [H], [H][S]: the layer's offset tables.
 *   kc, vc        dev bf16 [kc_rows][D] out.
 * kq, vq 8-byte aligned; the absmax tables, kc and vc 16-byte aligned.
 * Errors: VARK_E_ARG, VARK_E_SHAPE (D % 8 != 0, D > 512, H > 4096, kc_rows not a
 * multiple of B), VARK_E_ALIGN, VARK_E_CUDA.
 */
int vark_dequantize_layer_int8(const int8_t* kq, const int8_t* vq, const float* k_absmax, const float* v_absmax,
                               int64_t kc_rows, int B, int H, int S, int D, const int32_t* sides,
                               const int32_t* head_off, const int32_t* seg_off,
                               uint16_t* kc, uint16_t* vc, void* stream);

/* ---------------------------------------------------------------------------
 * Quantised retained cache (4-bit).  [VAR-Q] summary page: INT4 codes on the
 * same (block, channel) groups keep BF16 quality, and bit packing turns the
 * nominal bit width into real memory savings.  Same groups as the 8-bit cache;
 * per channel:
 *   a    = max |x| over the block        s = bf16(a / 7)   (IEEE fp32 division, RNE to bf16)
 *   code = rint(x / s) in [-7, 7]        (IEEE fp32 division, half to even; s = 0 gives 0)
 *   x'   = bf16(code * s)                (the product is exact in fp32; one rounding)
 * Packing: nibble = code + 8 (1..15); the 8 channels c0..c7 of a row that
 * start at a multiple of 8 form one little-endian 32-bit word, c0, c2, c4, c6
 * in nibbles 0-3 and c1, c3, c5, c7 in nibbles 4-7.  Element e of the
 * compacted layout (see the layout block) is nibble e % 8 of word e / 8, so a
 * layer's codes start at byte layer_base[l] / 2 and a row is D / 2 bytes.
 * Scale tables are [L][B][H][S][D] bf16 bits (0 for dropped scales).
 * ------------------------------------------------------------------------- */

/*
 * vark_quantize_kv_int4 -- device.  Compaction with 4-bit quantisation: like
 * vark_quantize_kv_int8, but kq / vq receive packed nibbles (layer_base[L] / 2
 * bytes each) and k_scale / v_scale the bf16 scales s.  Each kept block is read
 * from HBM once (as vark_quantize_kv_int8).  k, v, kq, vq, k_scale, v_scale
 * 16-byte aligned; layer_stride a multiple of 8.
 * Errors: VARK_E_ARG, VARK_E_SHAPE (D % 8 != 0, D > 512, H > 2048), VARK_E_ALIGN,
 * VARK_E_CUDA.
 */
int vark_quantize_kv_int4(const uint16_t* k, const uint16_t* v, int64_t layer_stride,
                          int L, int B, int H, int S, int D, const int32_t* sides,
                          const uint8_t* keep, const int32_t* head_off, const int32_t* seg_off,
                          const int64_t* layer_base, uint8_t* kq, uint8_t* vq,
                          uint16_t* k_scale, uint16_t* v_scale, void* stream);

/*
 * vark_dequantize_layer_int4 -- device.  Expands one layer's 4-bit codes to
 * its bf16 compacted block (as vark_dequantize_layer_int8).
 *   kq, vq        dev uint8, the layer's packed codes (kq + layer_base[l] / 2),
 *                 kc_rows rows of D / 2 bytes; 4-byte aligned.
 *   k_scale, v_scale  dev bf16 bits [B][H][S][D], the layer's scale tables.
 *   other arguments as vark_dequantize_layer_int8.
 * Errors: as vark_dequantize_layer_int8.
 */
int vark_dequantize_layer_int4(const uint8_t* kq, const uint8_t* vq, const uint16_t* k_scale,
                               const uint16_t* v_scale, int64_t kc_rows, int B, int H, int S, int D,
                               const int32_t* sides, const int32_t* head_off, const int32_t* seg_off,
                               uint16_t* kc, uint16_t* vc, void* stream);

/* ---------------------------------------------------------------------------
 * Quantised retained cache (3-bit).  [VAR-Q] summary page, Main Findings: INT3
 * codes on the (block, channel) groups stay within one FID point of BF16 on
 * the next-scale image models; Key Contributions: packing turns the nominal
 * bit width into memory savings (the page reports up to 78.5%).
 * Same groups; per channel:
 *   a    = max |x| over the block        s = bf16(a / 3)   (IEEE fp32 division, RNE to bf16)
 *   code = rint(x / s) in [-3, 3]        (IEEE fp32 division, half to even; s = 0 gives 0)
 *   x'   = bf16(code * s)                (the product is exact in fp32; one rounding)
 * Packing: field = code + 4 (1..7); the 8 channels c0..c7 of a row that start
 * at a multiple of 8 form one little-endian 24-bit group (3 bytes) with cj in
 * bits 3j .. 3j + 2.  Element e of the compacted layout (e a multiple of 8)
 * starts group e / 8 at byte 3 e / 8, so a layer's codes start at byte
 * 3 layer_base[l] / 8 and a row is 3 D / 8 bytes.  Scale tables are
 * [L][B][H][S][D] bf16 bits (0 for dropped scales).
 * ------------------------------------------------------------------------- */

/*
 * vark_quantize_kv_int3 -- device.  Compaction with 3-bit quantisation: like
 * vark_quantize_kv_int4, but kq / vq receive 24-bit groups (3 layer_base[L] / 8
 * bytes each) and k_scale / v_scale the bf16 scales s = bf16(a / 3).  k, v,
 * kq, vq, k_scale, v_scale 16-byte aligned; layer_stride a multiple of 8.
 * Errors: VARK_E_ARG, VARK_E_SHAPE (D % 8 != 0, D > 512, H > 2048), VARK_E_ALIGN,
 * VARK_E_CUDA.
 */
int vark_quantize_kv_int3(const uint16_t* k, const uint16_t* v, int64_t layer_stride,
                          int L, int B, int H, int S, int D, const int32_t* sides,
                          const uint8_t* keep, const int32_t* head_off, const int32_t* seg_off,
                          const int64_t* layer_base, uint8_t* kq, uint8_t* vq,
                          uint16_t* k_scale, uint16_t* v_scale, void* stream);

/*
 * vark_dequantize_layer_int3 -- device.  Expands one layer's 3-bit codes to
 * its bf16 compacted block (as vark_dequantize_layer_int8).
 *   kq, vq        dev uint8, the layer's packed codes (kq + 3 layer_base[l] / 8),
 *                 kc_rows rows of 3 D / 8 bytes; any alignment.
 *   k_scale, v_scale  dev bf16 bits [B][H][S][D], the layer's scale tables.
 *   other arguments as vark_dequantize_layer_int8.
 * Errors: as vark_dequantize_layer_int8.
 */
int vark_dequantize_layer_int3(const uint8_t* kq, const uint8_t* vq, const uint16_t* k_scale,
                               const uint16_t* v_scale, int64_t kc_rows, int B, int H, int S, int D,
                               const int32_t* sides, const int32_t* head_off, const int32_t* seg_off,
                               uint16_t* kc, uint16_t* vc, void* stream);

/* ---------------------------------------------------------------------------
 * Pruned attention straight over a quantised retained cache.  [VAR-Q] Why This
 * Matters: quantisation composes with eviction; here the dequantisation is
 * part of the attention kernel itself, so no bf16 copy of a layer's cache is
 * written.  The past K / V tiles are expanded from the codes in shared memory
 * with exactly the arithmetic of vark_dequantize_layer_int8 / _int4 / _int3,
 * so the output equals vark_pruned_attention over the dequantised block bit
 * for bit.
 * ------------------------------------------------------------------------- */

/*
 * vark_pruned_attention_int8 -- device.  vark_pruned_attention whose past
 * comes as this layer's 8-bit codes and absmax tables.
 *   kq, vq       dev int8, the layer's codes (kq + layer_base[l]), kc_rows
 *                rows of D bytes; 16-byte aligned.
 *   k_absmax, v_absmax  dev fp32 [B][H][S][D], the layer's tables (element
 *                l*B*H*S*D of vark_quantize_kv_int8's); 16-byte aligned.
 *   other arguments as vark_pruned_attention.
 * Codes and tables must come from vark_quantize_kv_int8 with the same offset
 * tables: a past tile whose rows would lie outside [0, kc_rows) is not read
 * and sets *dev_status to VARK_E_SHAPE.
 * Errors: as vark_pruned_attention.
 */
int vark_pruned_attention_int8(const uint16_t* q, const int8_t* kq, const int8_t* vq,
                               const float* k_absmax, const float* v_absmax, int64_t kc_rows,
                               const uint16_t* k_dense, const uint16_t* v_dense,
                               int B, int H, int S, int D, const int32_t* sides, int query_scale,
                               const int32_t* head_off, const int32_t* seg_off, const int32_t* past_len,
                               const float* tau, const float* bias,
                               uint16_t* out, int32_t* dev_status, void* stream);

/*
 * vark_pruned_attention_int4 -- device.  As vark_pruned_attention_int8 over
 * 4-bit codes: kq, vq hold the layer's packed codes (kq + layer_base[l] / 2),
 * rows of D / 2 bytes; k_scale, v_scale the layer's bf16 scale tables.
 * Errors: as vark_pruned_attention.
 */
int vark_pruned_attention_int4(const uint16_t* q, const uint8_t* kq, const uint8_t* vq,
                               const uint16_t* k_scale, const uint16_t* v_scale, int64_t kc_rows,
                               const uint16_t* k_dense, const uint16_t* v_dense,
                               int B, int H, int S, int D, const int32_t* sides, int query_scale,
                               const int32_t* head_off, const int32_t* seg_off, const int32_t* past_len,
                               const float* tau, const float* bias,
                               uint16_t* out, int32_t* dev_status, void* stream);

/*
 * vark_pruned_attention_int3 -- device.  As vark_pruned_attention_int4 over
 * 3-bit codes (kq + 3 layer_base[l] / 8, rows of 3 D / 8 bytes).  A packed
 * tile is copied whole, so rows must be a multiple of 16 bytes: D = 128 only
 * (D = 64 returns VARK_E_SHAPE; use vark_dequantize_layer_int3 there).
 * Errors: as vark_pruned_attention.
 */
int vark_pruned_attention_int3(const uint16_t* q, const uint8_t* kq, const uint8_t* vq,
                               const uint16_t* k_scale, const uint16_t* v_scale, int64_t kc_rows,
                               const uint16_t* k_dense, const uint16_t* v_dense,
                               int B, int H, int S, int D, const int32_t* sides, int query_scale,
                               const int32_t* head_off, const int32_t* seg_off, const int32_t* past_len,
                               const float* tau, const float* bias,
                               uint16_t* out, int32_t* dev_status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* VARK_H */

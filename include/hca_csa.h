/*
 * hca_csa.h -- C ABI of the B200 (sm_100a) hybrid compressed attention library.
 *
 * The operation is the attention layer of DeepSeek-V4 as described in
 * "DeepSeek-V4: interleaved compressed attention with manifold-constrained
 * hyper-connections" (TL;DR and the three-tier diagram: HCA 128-to-1, CSA
 * 4-to-1 plus an indexer over a low-dimensional projection, an uncompressed
 * recent window) and "DeepSeek-V4: ... KV cache ... compressed attention"
 * (sections "CSA: compresion 4x mas recuperacion dispersa", "HCA: compresion
 * 128x mas atencion densa", "Ventana deslizante"), with every step fixed as in
 * the CSA fp32 T=2048 workload definition:
 *
 *   projections   kv = x W_kv, g = x W_g, ki = x W_ki, qi = x W_qi, w = x W_w, q = x W_q
 *   compressor    entry j pools tokens i in [m j - (width - m), m j + m) within [0, T):
 *                   c_j[c] = sum_i softmax_i(g[i,c] + B[i - m j + width - m, c]) kv[i,c]
 *                 indexer key k_j[d] = the same pool over ki[i,d], gate channel d
 *   indexer       s[t,j] = sum_h w[t,h] ReLU(qi[t,h,:] . k_j),  j visible iff m j + m <= t
 *   top-k         the min(topk, visible) best s[t,j]; equal scores -> lower j first
 *   attention     MQA over {selected entries} U {raw tokens (t - window, t]};
 *                 key = first C/2 channels, value = last C/2; one softmax, scale tau
 *   HCA           m = width = 128, every visible entry attended (no indexer)
 *   decode        one new token per sequence over a compressed cache (the pages'
 *                 problem statement: each decode step reads the past K/V)
 *
 * Conventions for every call
 *   - All tensors are row-major and live in device memory owned by the caller.
 *     The library allocates nothing and keeps one device status word per
 *     device (plus the fixed scratch array of the allocation-free entry
 *     point below).
 *   - Storage type is p->dtype: HCSA_F32 (fp32 storage; the kernels compute in
 *     fp64) or HCSA_BF16 (bf16 storage; fp32 accumulation, tensor cores).
 *   - Pointers must be 16-byte aligned; every leading dimension `ld_*` (in
 *     elements) must keep rows 16-byte aligned.  Violations return
 *     HCSA_ERR_ALIGN; wrong sizes return HCSA_ERR_SHAPE; a NULL tensor returns
 *     HCSA_ERR_NULL; too little workspace returns HCSA_ERR_WORKSPACE.  Argument
 *     errors are found on the host before anything is enqueued.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     asynchronous, stream-ordered and deterministic.  Launch failures return
 *     HCSA_ERR_CUDA.  Errors found by the kernels themselves (bounded waits
 *     that gave up, out-of-range indices) are recorded in the device status
 *     word and reported by hcsa_get_device_status().
 *   - Entry selections `sel` are int32 [rows, topk], ascending entry index,
 *     padded with -1 when fewer than topk entries are visible.
 */
#ifndef HCA_CSA_H
#define HCA_CSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    HCSA_OK = 0,
    HCSA_ERR_NULL = 1,
    HCSA_ERR_SHAPE = 2,
    HCSA_ERR_DTYPE = 3,
    HCSA_ERR_ALIGN = 4,
    HCSA_ERR_WORKSPACE = 5,
    HCSA_ERR_CUDA = 6,
    HCSA_ERR_TIMEOUT = 7,      /* a bounded device-side wait gave up */
    HCSA_ERR_UNSUPPORTED = 8,  /* valid request the library does not implement */
    HCSA_ERR_DEVICE = 9        /* a kernel's own bounds check fired */
} hcsa_status;

typedef enum { HCSA_F32 = 0, HCSA_BF16 = 1 } hcsa_dtype;

typedef enum { HCSA_KIND_CSA = 0, HCSA_KIND_HCA = 1 } hcsa_kind;

/* One struct describes a layer; each call reads the fields it needs. */
typedef struct {
    int32_t B;       /* sequences in a decode batch (prefill: 1) */
    int32_t T;       /* tokens of the prefill sequence */
    int32_t D;       /* model width */
    int32_t m;       /* compression ratio (CSA 4, HCA 128) */
    int32_t width;   /* pool width (CSA 8: overlapping; HCA = m) */
    int32_t C;       /* compressed dim: key half C/2, value half C/2 */
    int32_t di;      /* indexer key dim (CSA) */
    int32_t Hi;      /* indexer heads (CSA) */
    int32_t topk;    /* entries selected per query (CSA) */
    int32_t window;  /* raw sliding window (tokens), >= width for decode */
    int32_t H;       /* query heads */
    int32_t dh;      /* head dim, must equal C/2 */
    float scale;     /* softmax scale tau */
    int32_t dtype;   /* hcsa_dtype */
    int32_t n_cap;   /* decode: entry capacity per sequence of the cache arrays */
    /* Prefill row range (both 0: the whole sequence).  The calls keep global token positions and
     * full-length arrays, but compute only query rows [row0, row1) of the T tokens: csa_compress /
     * hca_compress form the entries whose pools end in the range (j in [row0 / m, ceil(row1 / m))), the
     * indexer + top-k and the attention compute those query rows.  Such a call reads no projection row
     * outside [row0 - max(window - 1, width - m), row1) and no entry (or indexer key) at or past
     * (row1 - 1) / m, the last one the range's last query sees; so a sequence split over ranks needs,
     * in its arrays, only its rows with that halo and the entries it gathered from the other ranks
     * between the compressor and the indexer.  row0 must be a multiple of 128; row1 a multiple of 128
     * or T; otherwise the calls return HCSA_ERR_SHAPE. */
    int32_t row0;
    int32_t row1;
    /* Storage of the compressed entries and the indexer keys ("DeepSeek-V4 ... KV cache ...", section
     * "FP8 y FP4": most of each entry in FP8, the indexer keys in FP4).  0: the layer's dtype.
     * 1 (bf16 layers, C and di multiples of 32): block-scaled FP8 / FP4, every 32 channels of a row
     * sharing a power-of-two scale 2^e, e the smallest integer that clips nothing:
     *   entries   rows x C bytes of OCP E4M3 codes, then rows x C/32 int8 exponents e
     *             (stored value = E4M3(code) x 2^e; |value| / 2^e <= 448)
     *   idx_keys  rows x di/2 bytes of OCP E2M1 code pairs (channel 2i in the low nibble, 2i + 1 in
     *             the high one), then rows x di/32 int8 exponents (|value| / 2^e <= 6)
     * rows = ceil(T / m) for prefill arrays, B * n_cap for a decode cache (row b * n_cap + j);
     * hcsa_entry_bytes / hcsa_key_bytes give the sizes.  Codes round to nearest, ties to even.
     * Every stored value is a bf16 number, so the kernels dequantize exactly and compute as in the bf16
     * path.  Supported: compressors, cache append, the CSA calls (prefill and decode, tensor-core
     * shapes: di = 64; H = 64, dh = 512 for the attention) and hca_decode_attend (same shape);
     * hca_attend and the fp32 / CUDA-core paths return HCSA_ERR_UNSUPPORTED. */
    int32_t lowprec;
    /* Entry-sharded decode (a cache too large for one GPU split by entry index over ranks; the split of
     * the decode path is that of the CSA / HCA sections of the KV-cache page).  ent_shard = 1: the decode cache holds entries [ent0, ent0 + n_cap) of
     * each sequence (row b * n_cap + j - ent0); hcsa_cache_append writes a formed entry only when it
     * falls in that range, and the *_shard calls below work on it.  0 (the default): the cache holds
     * entries [0, n_cap) and ent0 must be 0. */
    int32_t ent0;
    int32_t ent_shard;
} hcsa_params;

/* Decode cache of one layer (device pointers, caller-owned).
 * entries  [B, n_cap, C]        compressed entries, entry j of sequence b at row j
 * idx_keys [B, n_cap, di]       indexer keys (CSA; NULL for HCA)
 * win_kv   [B, window, C]       raw kv rows: token p in slot p % window
 * ring_g   [B, width, C]        gate logits g = x W_g of token p in slot p % width
 * ring_ki  [B, width, di]       indexer-key projections of token p in slot p % width (CSA)
 * The window ring also stages the kv rows of the pool that is still open, which
 * is why window >= width is required. */
typedef struct {
    void *entries;
    void *idx_keys;
    void *win_kv;
    void *ring_g;
    void *ring_ki;
} hcsa_cache;

/* Workspace queries: op selects the call. */
typedef enum {
    HCSA_OP_PROJECT = 0,
    HCSA_OP_CSA_INDEX_TOPK = 1,
    HCSA_OP_CSA_ATTEND = 2,
    HCSA_OP_HCA_ATTEND = 3,
    HCSA_OP_CSA_DECODE_INDEX_TOPK = 4,
    HCSA_OP_CSA_DECODE_ATTEND = 5,
    HCSA_OP_HCA_DECODE_ATTEND = 6,
    HCSA_OP_CSA_DECODE_INDEX_TOPK_SHARD = 7,
    HCSA_OP_CSA_DECODE_ATTEND_SHARD = 8,
    HCSA_OP_HCA_DECODE_ATTEND_SHARD = 9
} hcsa_op;

/* Library version (major * 10000 + minor * 100 + patch). */
int32_t hcsa_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char *hcsa_status_string(hcsa_status s);

/* Bytes of scratch the call `op` needs for layer p (0 if none). */
size_t hcsa_workspace_bytes(const hcsa_params *p, int32_t op);

/* Number of projected columns for a layer of `kind`:
 * CSA: C (kv) + C (g) + di (ki) + Hi*di (qi) + Hi (w) + H*dh (q);  HCA: C + C + H*dh. */
int64_t hcsa_proj_cols(const hcsa_params *p, int32_t kind);

/* Bytes of an entries array (hcsa_entry_bytes) or an indexer-key array (hcsa_key_bytes) of `rows`
 * rows in the storage p selects (dtype, lowprec); 0 for a NULL p or negative rows. */
size_t hcsa_entry_bytes(const hcsa_params *p, int64_t rows);
size_t hcsa_key_bytes(const hcsa_params *p, int64_t rows);

/* hcsa_quantize_rows: store bf16 rows in the block-scaled formats of p->lowprec = 1 (the FP8 / FP4 of
 * the "FP8 y FP4" section, layout as documented at hcsa_params.lowprec), e.g. to convert a bf16 cache.
 *   what  HCSA_STORE_ENTRIES: src [rows, C] bf16 -> dst of hcsa_entry_bytes(p, rows) bytes (E4M3)
 *         HCSA_STORE_KEYS:    src [rows, di] bf16 -> dst of hcsa_key_bytes(p, rows) bytes (E2M1)
 * The same rounding as the compressor and the cache append.  Errors: HCSA_ERR_UNSUPPORTED when
 * p->lowprec is 0 or the shape has no low-precision form; the usual checks otherwise. */
#define HCSA_STORE_ENTRIES 0
#define HCSA_STORE_KEYS 1
hcsa_status hcsa_quantize_rows(const hcsa_params *p, int32_t what, const void *src, int64_t rows, void *dst,
                               void *stream);

/* Token projections: every per-token input of the layer in one GEMM -- the compressor's kv and gate
 * logits, the indexer's "lower-dimensional projection" keys, queries and head weights, and the
 * attention queries (page "DeepSeek-V4: interleaved compressed attention ...", TL;DR and "The HCA-CSA
 * pair"; the weight list of the CSA workload definition).
 *   x     [rows, D]           (ld = D)
 *   W_cat [D, ncols]          the concatenation [W_kv | W_g | W_ki | W_qi | W_w | W_q] (HCA: [W_kv | W_g | W_q])
 *   y     [rows, ncols]       y = x W_cat rounded once to the storage type; ncols = hcsa_proj_cols(p, kind)
 * bf16: tcgen05 tensor-core GEMM, fp32 accumulate.  ws (hcsa_workspace_bytes(p, HCSA_OP_PROJECT)
 * bytes) is optional: with it, outputs with too few column tiles to fill the GPU split the contraction
 * over CTAs; with NULL every tile is one CTA (same result up to fp32 summation order).
 * f32: CUDA cores, fp64 accumulate, ws unused.  Requires D and ncols to keep rows 16-byte aligned. */
hcsa_status hcsa_project(const hcsa_params *p, int32_t kind, int64_t rows, const void *x, const void *W_cat,
                         void *y, void *ws, size_t ws_bytes, void *stream);

/* Output projection with the residual stream, for stacks whose layers are chained (the V4-style
 * schedule of page "DeepSeek-V4 ... KV cache ... atencion comprimida", section "Pila hibrida de
 * capas": two HCA layers, then CSA and HCA alternating).  The pages define no output projection or
 * normalisation; the reading is x_{l+1} = x_l + out_l W_o,l.
 *   out [rows, ld_out]   the layer's attention output (H*dh columns used); must hold rows * ld_out elements
 *   W_o [H*dh, D]        row-major, H*dh * D elements
 *   x   [rows, ld_x]     the hidden state, updated in place: x = round(x + out W_o), fp32 accumulate,
 *                        one rounding to bf16 (the tcgen05 GEMM of hcsa_project with the residual added
 *                        in its epilogue); must hold rows * ld_x elements
 * Decode parameters (p->T == 0) allow at most p->B rows (HCSA_ERR_SHAPE otherwise).
 * bf16 storage only (HCSA_ERR_UNSUPPORTED otherwise).  ws as for hcsa_project (may be NULL). */
hcsa_status hcsa_out_project(const hcsa_params *p, int64_t rows, const void *out, int64_t ld_out, const void *W_o,
                             void *x, int64_t ld_x, void *ws, size_t ws_bytes, void *stream);

/* CSA compressor: the learned compression pool over overlapping windows (page "DeepSeek-V4 ... KV
 * cache ... atencion comprimida", section "CSA: compresion 4x mas recuperacion dispersa"; the pool
 * formula of the CSA workload definition), m = 4 with width 8, prefill of one sequence of p->T tokens.
 *   kv [T, ld_kv] (C used), g [T, ld_g] (C used), ki [T, ld_ki] (di used), bias [width, C]
 *   entries [N, C], idx_keys [N, di] with N = ceil(T / m) (edge pools are truncated to [0, T)). */
hcsa_status csa_compress(const hcsa_params *p, const void *kv, int64_t ld_kv, const void *g, int64_t ld_g,
                         const void *ki, int64_t ld_ki, const void *bias, void *entries, void *idx_keys,
                         void *stream);

/* HCA compressor: 128 tokens into one entry (same page, section "HCA: compresion 128x mas atencion
 * densa"; the HCA prefill workload definition), width = m, non-overlapping pools; as csa_compress
 * without indexer keys. */
hcsa_status hca_compress(const hcsa_params *p, const void *kv, int64_t ld_kv, const void *g, int64_t ld_g,
                         const void *bias, void *entries, void *stream);

/* CSA lightning indexer + top-k, causal prefill (section "CSA: compresion 4x mas recuperacion
 * dispersa": the indexer scores the compressed entries, the query keeps the most relevant ones; the
 * score, visibility and tie rule of the CSA workload definition).
 *   qi [T, ld_qi] (Hi*di used, head-major), w [T, ld_w] (Hi used), idx_keys [N, di]
 *   sel [T, topk] int32: for query t the min(topk, t / m) best visible entries, ascending, -1 padded.
 * ws: hcsa_workspace_bytes(p, HCSA_OP_CSA_INDEX_TOPK) bytes (materialised scores). */
hcsa_status csa_index_topk(const hcsa_params *p, const void *qi, int64_t ld_qi, const void *w, int64_t ld_w,
                           const void *idx_keys, int32_t *sel, void *ws, size_t ws_bytes, void *stream);

/* CSA attention, causal prefill: one softmax over the selected entries and the uncompressed recent
 * window (sections "CSA: ..." and "Ventana deslizante: el contexto reciente conserva detalle"; MQA,
 * key / value halves and scale as in the CSA workload definition).
 *   q [T, ld_q] (H*dh used, head-major), kv [T, ld_kv] raw window rows (C used), entries [N, C], sel [T, topk]
 *   out [T, H*dh]: softmax over selected entries and raw tokens (t - window, t]. */
hcsa_status csa_attend(const hcsa_params *p, const void *q, int64_t ld_q, const void *kv, int64_t ld_kv,
                       const void *entries, const int32_t *sel, void *out, void *ws, size_t ws_bytes,
                       void *stream);

/* HCA attention, causal prefill: every visible entry (j < t / m) plus the raw window (sections "HCA:
 * compresion 128x mas atencion densa" and "Ventana deslizante"). */
hcsa_status hca_attend(const hcsa_params *p, const void *q, int64_t ld_q, const void *kv, int64_t ld_kv,
                       const void *entries, void *out, void *ws, size_t ws_bytes, void *stream);

/* Decode: append one new token per sequence to the cache.  Each decode step reads the past keys and
 * values (page "DeepSeek-V4 ... KV cache ... atencion comprimida", opening section); the cache holds the
 * compressed entries plus the uncompressed window (sections "CSA", "HCA", "Ventana deslizante").
 *   pos [B] int32 (device): position of the new token of each sequence (not modified)
 *   kv/g/ki [B, ld] the new token's projections (ki NULL for HCA), bias [width, C]
 * Writes the rings; when pos[b] = m j + m - 1 the entry j is formed from the rings
 * (and written if j < n_cap).  Callers advance pos themselves between steps. */
hcsa_status hcsa_cache_append(const hcsa_params *p, const hcsa_cache *cache, const int32_t *pos,
                              const void *kv, int64_t ld_kv, const void *g, int64_t ld_g, const void *ki,
                              int64_t ld_ki, const void *bias, void *stream);

/* Prefill: the projection with the compressor done in the GEMM's epilogue (the compressor of "CSA:
 * compresion 4x" fed straight from the projection tile).  Same results as hcsa_project followed by
 * csa_compress / hca_compress with the same params: y [T, ncols] (ld ncols), entries and idx_keys (CSA;
 * NULL for HCA) as documented for the compressors (bf16, or FP8 / FP4 with p->lowprec; a row range forms
 * the range's entries).  The fused kernel covers CSA layers (m = 4, width = 8, di = 64, C a multiple
 * of 64, bf16) over the whole sequence: pools inside a 128-token half of a 256-token tile are formed in
 * the epilogue, the one per half boundary afterwards from the stored projections; other shapes and row
 * ranges run the two calls' kernels.  ws as for hcsa_project. */
hcsa_status hcsa_project_compress(const hcsa_params *p, int32_t kind, const void *x, const void *W_cat,
                                  const void *bias, void *y, void *entries, void *idx_keys, void *ws, size_t ws_bytes,
                                  void *stream);

/* Decode: the projection of the new tokens with the cache append done in the GEMM's epilogue (the
 * compressor of "CSA: compresion 4x" / "HCA: compresion 128x" fed straight from the projection tile).
 * Same results as hcsa_project followed by hcsa_cache_append: y [B, ncols] (ld ncols) is written, the
 * rings get the new token and a closed entry is pooled into the cache (FP8 / FP4 with p->lowprec, only
 * on its shard with p->ent_shard).  x [B, D], W_cat [D, ncols], bias [width, C].  Shapes outside the
 * fused kernel (fp32 storage, B > 16, C not a multiple of 64, CSA with di != 64) run the two calls'
 * kernels instead; ws as for hcsa_project. */
hcsa_status hcsa_project_append(const hcsa_params *p, int32_t kind, const hcsa_cache *cache, const int32_t *pos,
                                const void *x, const void *W_cat, const void *bias, void *y, void *ws, size_t ws_bytes,
                                void *stream);

/* Decode: CSA indexer + top-k for the new token of each sequence over entries j < pos[b] / m.
 *   qi [B, ld_qi], w [B, ld_w]; sel [B, topk]. */
hcsa_status csa_decode_index_topk(const hcsa_params *p, const hcsa_cache *cache, const int32_t *pos,
                                  const void *qi, int64_t ld_qi, const void *w, int64_t ld_w, int32_t *sel,
                                  void *ws, size_t ws_bytes, void *stream);

/* Decode: CSA attention (split over keys, then a log-sum-exp combine).
 *   q [B, ld_q], sel [B, topk]; out [B, H*dh].  Keys: selected entries U tokens (pos - window, pos]. */
hcsa_status csa_decode_attend(const hcsa_params *p, const hcsa_cache *cache, const int32_t *pos, const void *q,
                              int64_t ld_q, const int32_t *sel, void *out, void *ws, size_t ws_bytes,
                              void *stream);

/* Decode: HCA attention over entries j < pos[b] / m and the raw window. */
hcsa_status hca_decode_attend(const hcsa_params *p, const hcsa_cache *cache, const int32_t *pos, const void *q,
                              int64_t ld_q, void *out, void *ws, size_t ws_bytes, void *stream);

/* ---- entry-sharded decode (p->ent_shard = 1; the cache is one shard: entries [ent0, ent0 + n_cap)).
 * A step: every shard runs csa_decode_index_topk_shard; the ranks all-gather (sel, sel_scores); every
 * rank runs csa_topk_merge (the exact global top-k: each global top-k entry is in its own shard's top-k),
 * then csa_decode_attend_shard (or hca_decode_attend_shard) on its shard; the ranks all-gather the
 * partials and hcsa_merge_partials combines them.  Tensor-core shapes only (di = 64; H = 64, dh = 512,
 * C = 1024, window 128), bf16 storage; others return HCSA_ERR_UNSUPPORTED.
 *
 * Partial layout (part): acc [B, H, dh] fp32 (the unnormalized softmax-weighted value sum), then
 * ml [B, H, 2] fp32 (max logit in natural units, sum of exp(logit - max)); a head with no key has
 * max = -inf and sum = 0.  B * H * (dh + 2) floats. */

/* Indexer + exact top-k over the shard's visible entries (global j < pos[b] / m); sel [B, topk] gets
 * global indices in ascending order (-1 padding), sel_scores [B, topk] their scores (-inf padding).
 * ws: hcsa_workspace_bytes(p, HCSA_OP_CSA_DECODE_INDEX_TOPK_SHARD). */
hcsa_status csa_decode_index_topk_shard(const hcsa_params *p, const hcsa_cache *cache, const int32_t *pos,
                                        const void *qi, int64_t ld_qi, const void *w, int64_t ld_w, int32_t *sel,
                                        float *sel_scores, void *ws, size_t ws_bytes, void *stream);

/* Exact top-k (p->topk) of n_cand candidates per row (B = p->B rows): cand_sel [B, n_cand] indices (-1:
 * none), cand_scores [B, n_cand]; the k best by (score desc, index asc), emitted in ascending index order
 * into sel [B, topk] (-1 padding).  n_cand <= 8192.  Candidates must be distinct per row. */
hcsa_status csa_topk_merge(const hcsa_params *p, const int32_t *cand_sel, const float *cand_scores, int32_t n_cand,
                           int32_t *sel, void *stream);

/* Attention over the entries of sel [B, topk] (global indices) that this shard holds, plus the raw window
 * when with_window != 0 (exactly one shard attends it); writes the partial (layout above).
 * ws: hcsa_workspace_bytes(p, HCSA_OP_CSA_DECODE_ATTEND_SHARD). */
hcsa_status csa_decode_attend_shard(const hcsa_params *p, const hcsa_cache *cache, const int32_t *pos, const void *q,
                                    int64_t ld_q, const int32_t *sel, int32_t with_window, float *part, void *ws,
                                    size_t ws_bytes, void *stream);

/* HCA: attention over the shard's visible entries (global j < pos[b] / m) plus the window when
 * with_window != 0; writes the partial.  ws: hcsa_workspace_bytes(p, HCSA_OP_HCA_DECODE_ATTEND_SHARD). */
hcsa_status hca_decode_attend_shard(const hcsa_params *p, const hcsa_cache *cache, const int32_t *pos, const void *q,
                                    int64_t ld_q, int32_t with_window, float *part, void *ws, size_t ws_bytes,
                                    void *stream);

/* Log-sum-exp merge of n_parts partials (consecutive blocks of B * H * (dh + 2) floats) into the output
 * out [B, ld_out] bf16 (out[b, h * dh + d]). */
hcsa_status hcsa_merge_partials(const hcsa_params *p, const float *parts, int32_t n_parts, void *out,
                                int64_t ld_out, void *stream);

/* Decode: csa_decode_index_topk without a caller workspace, for callers that cannot allocate
 * device memory (for example code inside a serving engine or host framework that owns every
 * device allocation and hands out no scratch).  The pages have no counterpart: this is an
 * interface convenience, not part of the method.
 * Arguments and results are those of csa_decode_index_topk.  Its scratch (the scores, plus 49,168
 * bytes per sequence for the multi-block selection when n_cap > 32768) goes to one fixed 8 MiB
 * device array inside the library (held by every GPU that loads the library until exit):
 * hcsa_workspace_bytes(p, HCSA_OP_CSA_DECODE_INDEX_TOPK) must be at most 8 MiB -- with bf16
 * storage B * n_cap <= 2,097,152 while n_cap <= 32768 -- or the call returns HCSA_ERR_WORKSPACE
 * and launches nothing.  Allocates nothing.
 * The first call on a device (with that device current) looks up the array's device address
 * once; make that first call before any stream capture.  All calls share the array: calls
 * that overlap on the GPU (other streams, other host threads) race on it. */
hcsa_status csa_decode_index_topk_noalloc(const hcsa_params *p, const hcsa_cache *cache, const int32_t *pos,
                                          const void *qi, int64_t ld_qi, const void *w, int64_t ld_w,
                                          int32_t *sel, void *stream);

/* Waits for `stream`, then returns and clears the device status word of the current device
 * (HCSA_OK, HCSA_ERR_TIMEOUT or HCSA_ERR_DEVICE), or HCSA_ERR_CUDA if the wait itself failed. */
hcsa_status hcsa_get_device_status(void *stream);

/* Self-test of the failure path (not part of the method; the pages have no counterpart): enqueues one
 * kernel whose bounded wait on a barrier that nothing completes gives up after its limit (about a
 * second), records HCSA_ERR_TIMEOUT in the device status word and returns.  A following
 * hcsa_get_device_status(stream) then returns HCSA_ERR_TIMEOUT (and clears it); the context stays
 * usable.  Returns HCSA_ERR_CUDA if the launch fails. */
hcsa_status hcsa_selftest_wait_timeout(void *stream);

/* Number of kernels this library enqueued on the calling host thread since the last reset.
 * For launch accounting in benchmarks. */
int64_t hcsa_launch_count(int32_t reset);

#ifdef __cplusplus
}
#endif

#endif /* HCA_CSA_H */

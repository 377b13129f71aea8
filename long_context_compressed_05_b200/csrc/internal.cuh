// Internal declarations shared by the translation units of libhcsa.so.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hca_csa.h"

namespace hcsa {

// ---------------------------------------------------------------- storage / compute types
// HCSA_F32 stores fp32 and computes in fp64; HCSA_BF16 stores bf16 and computes in fp32.
template <typename S> struct Traits;
template <> struct Traits<float> {
    using A = double;
    static constexpr int VEC = 4;  // elements per 16-byte vector
};
template <> struct Traits<__nv_bfloat16> {
    using A = float;
    static constexpr int VEC = 8;
};

__device__ __forceinline__ double to_acc(float v, double) { return (double)v; }
__device__ __forceinline__ float to_acc(__nv_bfloat16 v, float) { return __bfloat162float(v); }

__device__ __forceinline__ void store_val(float *p, double v) { *p = (float)v; }
__device__ __forceinline__ void store_val(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }

// 16-byte vector load of VEC storage elements widened to the accumulation type.
template <typename S, typename A>
__device__ __forceinline__ void load_vec(const S *p, A *out) {
    uint4 raw = __ldg(reinterpret_cast<const uint4 *>(p));
    const S *e = reinterpret_cast<const S *>(&raw);
#pragma unroll
    for (int i = 0; i < Traits<S>::VEC; ++i) out[i] = to_acc(e[i], A());
}

template <typename S, typename A>
__device__ __forceinline__ void store_vec(S *p, const A *v) {
    uint4 raw;
    S *e = reinterpret_cast<S *>(&raw);
#pragma unroll
    for (int i = 0; i < Traits<S>::VEC; ++i) store_val(&e[i], v[i]);
    *reinterpret_cast<uint4 *>(p) = raw;
}

__device__ __forceinline__ double exp_acc(double x) { return exp(x); }
__device__ __forceinline__ float exp_acc(float x) { return expf(x); }

// device status word codes (match hcsa_status)
enum : int { kStatusOk = 0, kStatusTimeout = HCSA_ERR_TIMEOUT, kStatusBounds = HCSA_ERR_DEVICE };

__device__ __forceinline__ void report(int *status, int code) {
    if (status) atomicCAS(status, 0, code);
}

// ---------------------------------------------------------------- host side helpers
int *device_status_ptr();           // lazily resolved per device; nullptr on failure
// host-side argument checks of csa_decode_index_topk (everything but the workspace)
hcsa_status check_decode_index_topk_args(const hcsa_params *p, const hcsa_cache *cache, const int32_t *pos,
                                         const void *qi, int64_t ld_qi, const void *w, int64_t ld_w,
                                         const int32_t *sel);
void count_launch(int n = 1);
hcsa_status check_launch();         // maps cudaGetLastError() to a status

// ---------------------------------------------------------------- launchers
// compressor (prefill): entries j0 .. j1 - 1 of [N, C] (+ idx_keys [N, di] when ki != nullptr); the pools
// are truncated to the sequence [0, T) and read kv / g / ki by global token index
hcsa_status launch_compress(int dtype, int64_t T, int C, int m, int width, const void *kv, int64_t ld_kv,
                            const void *g, int64_t ld_g, const void *ki, int64_t ld_ki, int di, const void *bias,
                            void *entries, void *idx_keys, int64_t j0, int64_t j1, bool lowprec, int64_t rows,
                            cudaStream_t st, int jstride = 1);

// entry-sharded decode (shard.cu)
hcsa_status launch_shift_pos(const int32_t *pos, int64_t B, int64_t delta, int32_t *out, cudaStream_t st);
hcsa_status launch_shard_finish(int32_t *sel, int64_t B, int k, const float *scores, int64_t N, int64_t ent0,
                                float *sel_scores, cudaStream_t st);
hcsa_status launch_localize_sel(const int32_t *sel, int64_t n, int64_t ent0, int64_t n_cap, int32_t *out,
                                cudaStream_t st);
bool topk_merge_supported(int n_cand, int k);
hcsa_status launch_topk_merge(const int32_t *cand_sel, const float *cand_scores, int64_t rows, int n_cand, int k,
                              int32_t *sel, cudaStream_t st);
hcsa_status launch_merge_parts(const float *acc, const float *ml, int64_t ss, int64_t sr, int64_t ms, int64_t mr,
                               int n_parts, int64_t rows, int H, int dh, void *out, float *pacc, float *pml,
                               cudaStream_t st);

// bf16 rows [rows, ch] -> block-scaled FP8 (keys = false) or FP4 (keys = true) storage
hcsa_status launch_quantize_rows(const void *src, int64_t rows, int ch, bool keys, void *dst, cudaStream_t st);

hcsa_status launch_cache_append(int dtype, const hcsa_params &p, const hcsa_cache &c, const int32_t *pos,
                                const void *kv, int64_t ld_kv, const void *g, int64_t ld_g, const void *ki,
                                int64_t ld_ki, const void *bias, cudaStream_t st);

// indexer scores + top-k.  Prefill: rows = T queries of one sequence, n_vis(t) = min(t / m, N).
// Decode: rows = B sequences, query b sees entries j < min(pos[b] / m, n_cap) of keys + b * n_cap * di.
struct IndexArgs {
    int dtype;
    int64_t rows;        // queries
    int Hi, di, topk, m;
    int64_t N;           // entries per sequence (prefill: ceil(T/m); decode: n_cap)
    const void *qi; int64_t ld_qi;
    const void *w; int64_t ld_w;
    const void *keys;    // [N, di] (prefill) or [B, n_cap, di] (decode)
    const int32_t *pos;  // decode positions (nullptr: prefill, query t at position t)
    int32_t *sel;
    void *ws; size_t ws_bytes;
    const int32_t *only_rows;   // if set: the generic select handles only rows r with only_rows[4 r + 3] != 0
    int64_t row0, row1;         // query rows computed (prefill row range; decode: 0, rows)
    bool lowprec;               // keys: E2M1 code pairs [rows][di / 2], then int8 exponents [rows][di / 32]
};
size_t index_topk_ws_bytes(int dtype, int64_t rows, int64_t N);
// multi-CTA exact top-k for long decode rows (N > 32768); scratch after the scores.  The scratch starts
// with the rows' histograms of the top 12 bits of score_order_key ([rows][4096] uint32, filled by the
// indexer), then [rows][4] int32 counters whose element 3 flags rows left to the generic select.
bool topk_rows_supported(const IndexArgs &a);
size_t topk_rows_ws_bytes(int64_t rows);
hcsa_status topk_rows_begin(const IndexArgs &a, void *scratch, cudaStream_t st);   // zero histograms + counters
const int32_t *topk_rows_flags(const IndexArgs &a, const void *scratch);
hcsa_status launch_topk_rows(const IndexArgs &a, void *scratch, cudaStream_t st);

// order-preserving key of a score: larger score -> larger key; -0.0 and +0.0 map to the same key
__device__ __forceinline__ uint32_t score_order_key(float s) {
    if (s == 0.0f) s = 0.0f;
    const uint32_t b = __float_as_uint(s);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
hcsa_status launch_index_topk(const IndexArgs &a, cudaStream_t st);
hcsa_status launch_topk_generic(const IndexArgs &a, cudaStream_t st);
// tensor-core indexer scores (bf16, di = 64) + register-resident top-k
bool index_tc_supported(const IndexArgs &a);
hcsa_status launch_index_tc(const IndexArgs &a, cudaStream_t st);


// attention.  Prefill (pos == nullptr): query t of one sequence, window rows kv[t-window+1 .. t].
// Decode: query b at position pos[b], entries of sequence b, window ring win_kv[b].
struct AttendArgs {
    int dtype;
    int64_t rows;
    int H, dh, C, window, m, topk;
    float scale;
    bool dense;              // HCA: all visible entries instead of sel
    int64_t N;               // entries per sequence (prefill: ceil(T/m); decode: n_cap)
    const void *q; int64_t ld_q;
    const void *kv; int64_t ld_kv;   // prefill raw rows [T, ld_kv] / decode ring base [B, window, C]
    const void *entries;             // [N, C] or [B, n_cap, C]
    const int32_t *sel;              // [rows, topk] (CSA)
    const int32_t *pos;              // decode positions or nullptr
    void *out;
    void *ws; size_t ws_bytes;
    int64_t row0, row1;              // query rows computed (prefill row range; decode: 0, rows)
    bool lowprec;                    // entries: E4M3 codes [rows][C], then int8 exponents [rows][C / 32]
    int64_t ent0;                    // decode shard: global index of the cache's first entry (else 0)
    bool no_window;                  // decode shard: skip the raw window (another shard attends it)
    bool partial_out;                // tensor-core decode: write per-segment partials to ws even for one segment
};
size_t attend_ws_bytes(int dtype, bool decode, bool dense, int64_t rows, int H, int dh, int topk, int window,
                       int64_t N);
hcsa_status launch_attend(const AttendArgs &a, cudaStream_t st);
// tensor-core MQA attention (H = 64, dh = 512, window 128, bf16): prefill CSA, decode CSA and HCA
bool attend_tc_supported(const AttendArgs &a);
int attend_tc_segments(const AttendArgs &a);     // key segments per query (> 1: partials + combine)
hcsa_status launch_attend_tc(const AttendArgs &a, cudaStream_t st);
// tensor-core HCA prefill attention over query blocks (dh = 128, C = 256, H | 128, window 128, bf16)
bool hca_attend_tc_supported(const AttendArgs &a);
hcsa_status launch_hca_attend_tc(const AttendArgs &a, cudaStream_t st);

// prefill projection with the CSA compressor in the GEMM epilogue (gemm_tc.cu): y [T, ncols], entries, keys
bool project_compress_supported(const hcsa_params &p, bool csa);
hcsa_status launch_project_compress(const hcsa_params &p, const void *x, const void *W, int64_t ncols, void *y,
                                    const void *bias, void *entries, void *idx_keys, cudaStream_t st);
// decode projection with the cache append in the GEMM epilogue (gemm_tc.cu): y [B, ncols] and the cache update
bool project_append_supported(const hcsa_params &p, bool csa);
hcsa_status launch_project_append(const hcsa_params &p, bool csa, const hcsa_cache &c, const int32_t *pos,
                                  const void *x, const void *W, int64_t ncols, void *y, const void *bias,
                                  cudaStream_t st);
// tcgen05 GEMM y[M, N] = x[M, K] W[K, N] (+ res), bf16 (gemm_tc.cu); ws (optional) enables split-K
size_t gemm_tc_ws_bytes();
bool gemm_tc_supported(int64_t M, int N, int K, const void *x, int64_t ld_x, const void *W, int64_t ld_w,
                       const void *y, int64_t ld_y);
hcsa_status launch_gemm_tc(int64_t M, int N, int K, const void *x, int64_t ld_x, const void *W, int64_t ld_w,
                           void *y, int64_t ld_y, const void *res, int64_t ld_res, void *ws, size_t ws_bytes,
                           cudaStream_t st);
// projection y[rows, ncols] = x[rows, D] W[D, ncols]
size_t project_ws_bytes(int dtype);
hcsa_status launch_project(int dtype, int64_t rows, int D, int64_t ncols, const void *x, const void *W, void *y,
                           void *ws, size_t ws_bytes, cudaStream_t st);
// x[rows, D] += out[rows, HD] W_o[HD, D] (bf16)
hcsa_status launch_out_project(int64_t rows, int64_t HD, int D, const void *out, int64_t ld_out, const void *W_o,
                               void *x, int64_t ld_x, void *ws, size_t ws_bytes, cudaStream_t st);

}  // namespace hcsa

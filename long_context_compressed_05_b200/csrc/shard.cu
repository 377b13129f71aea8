// Entry-sharded decode: the compressed cache of every sequence is split by entry index over the ranks
// (each rank holds entries [ent0, ent0 + n_cap)).  A decode step then takes
//   1. on every rank: the indexer and an exact top-k over its own entries, with the selected scores;
//   2. an all-gather of those (index, score) candidates and the exact global top-k of their union
//      (csa_topk_merge: a global top-k entry is in the top-k of its own shard);
//   3. on every rank: attention over the selected entries it holds (the raw window on one rank), as an
//      unnormalized partial (accumulator, max logit, sum of weights) per head;
//   4. an all-gather of the partials and their log-sum-exp merge (hcsa_merge_partials).
// Selection: the same order as everywhere (score desc, equal scores to the lower index), emitted in
// ascending index order.  The method is the decode path of the CSA / HCA layer ("DeepSeek-V4 ... KV
// cache compressed attention", sections "CSA", "HCA"), split the way its cache is split.
#include "internal.cuh"

namespace hcsa {

namespace {

// positions seen by a shard: entry j of the sequence is local entry j - ent0, so the visible count of
// the shard is the visible count at position pos - m ent0 (negative: none)
__global__ void shift_pos_kernel(const int32_t *__restrict__ pos, int64_t B, int64_t delta, int32_t *out) {
    const int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= B) return;
    const int64_t p = pos[b];
    const int64_t q = p < 0 ? -1 : p - delta;
    out[b] = (int32_t)(q < -1 ? -1 : q);
}

// local selection -> global indices, with the scores of the selected entries (-inf for padding)
__global__ void shard_finish_kernel(int32_t *sel, int64_t B, int k, const float *__restrict__ scores, int64_t N,
                                    int64_t ent0, float *sel_scores) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= B * k) return;
    const int64_t b = i / k;
    const int32_t jl = sel[i];
    if (jl >= 0) {
        sel_scores[i] = scores[b * N + jl];
        sel[i] = (int32_t)(jl + ent0);
    } else {
        sel_scores[i] = -INFINITY;
    }
}

// global selection -> the shard's local rows (-1: not held by this shard, or padding)
__global__ void localize_sel_kernel(const int32_t *__restrict__ sel, int64_t n, int64_t ent0, int64_t n_cap,
                                    int32_t *out) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const int64_t j = sel[i];
    out[i] = (j >= ent0 && j < ent0 + n_cap) ? (int32_t)(j - ent0) : -1;
}

// Exact top-k of a row of candidates (index, score): composite 64-bit keys (order key of the score,
// then the complement of the index, so that equal scores rank the lower index first) are sorted
// descending by a bitonic network in shared memory; the first k valid ones are then sorted by index.
constexpr int kMergeThreads = 512;
constexpr int kMergeCap = 8192;   // candidates per row

__device__ __forceinline__ void bitonic_desc(uint64_t *v, int n) {
    for (int size = 2; size <= n; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = threadIdx.x; i < n / 2; i += blockDim.x) {
                const int lo = 2 * i - (i & (stride - 1));
                const int hi = lo + stride;
                const bool desc = (lo & size) == 0;
                const uint64_t a = v[lo], b = v[hi];
                if ((a < b) == desc) { v[lo] = b; v[hi] = a; }
            }
            __syncthreads();
        }
    }
}

__global__ void __launch_bounds__(kMergeThreads) topk_merge_kernel(const int32_t *__restrict__ cand_sel,
                                                                    const float *__restrict__ cand_scores,
                                                                    int n_cand, int k, int32_t *sel) {
    extern __shared__ uint64_t keys[];   // pow2(n_cand) composites, then pow2(k) indices
    const int64_t r = blockIdx.x;
    int n = 1;
    while (n < n_cand) n <<= 1;
    int nk = 1;
    while (nk < k) nk <<= 1;
    uint64_t *idx = keys + n;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        uint64_t c = 0;   // below every valid candidate
        if (i < n_cand) {
            const int32_t j = cand_sel[r * n_cand + i];
            if (j >= 0) c = ((uint64_t)score_order_key(cand_scores[r * n_cand + i]) << 32) | (uint32_t)~(uint32_t)j;
        }
        keys[i] = c;
    }
    __syncthreads();
    bitonic_desc(keys, n);
    // the first k composites (or fewer valid ones), by index; invalid -> top of the 32-bit range
    for (int i = threadIdx.x; i < nk; i += blockDim.x) {
        const uint64_t c = i < k && i < n ? keys[i] : 0;
        idx[i] = c ? (uint64_t)(~(uint32_t)c) : 0xFFFFFFFFull;
    }
    __syncthreads();
    // ascending: sort the complements descending
    for (int i = threadIdx.x; i < nk; i += blockDim.x) idx[i] = 0xFFFFFFFFull - idx[i];
    __syncthreads();
    bitonic_desc(idx, nk);
    for (int i = threadIdx.x; i < k; i += blockDim.x) {
        const uint64_t v = 0xFFFFFFFFull - idx[i];
        sel[r * k + i] = v == 0xFFFFFFFFull ? -1 : (int32_t)v;
    }
}

// Log-sum-exp merge of n_parts partials per (row, head): acc(s, r, h, :) at acc + s ss + r sr + h dh,
// (max logit, sum) at ml + 2 (s ms + r mr + h).  Output: normalized bf16 (out) or a merged partial
// (pacc [rows][H][dh], pml [rows][H][2]).
struct MergeArgs {
    const float *acc, *ml;
    int64_t ss, sr, ms, mr;
    int n_parts, H, dh;
    __nv_bfloat16 *out;
    float *pacc, *pml;
};

__global__ void __launch_bounds__(256) merge_parts_kernel(MergeArgs a) {
    const int64_t r = blockIdx.x;
    const int h = blockIdx.y;
    float M = -INFINITY;
    for (int s = 0; s < a.n_parts; ++s) M = fmaxf(M, a.ml[2 * (s * a.ms + r * a.mr + h)]);
    float Z = 0.f;
    for (int s = 0; s < a.n_parts; ++s) {
        const float m = a.ml[2 * (s * a.ms + r * a.mr + h)];
        if (m != -INFINITY) Z += expf(m - M) * a.ml[2 * (s * a.ms + r * a.mr + h) + 1];
    }
    const float zi = Z > 0.f ? 1.f / Z : 0.f;
    for (int d = threadIdx.x; d < a.dh; d += blockDim.x) {
        float o = 0.f;
        for (int s = 0; s < a.n_parts; ++s) {
            const float m = a.ml[2 * (s * a.ms + r * a.mr + h)];
            if (m != -INFINITY) o += expf(m - M) * a.acc[s * a.ss + r * a.sr + (int64_t)h * a.dh + d];
        }
        if (a.out) a.out[(r * a.H + h) * (int64_t)a.dh + d] = __float2bfloat16_rn(o * zi);
        else a.pacc[(r * a.H + h) * (int64_t)a.dh + d] = o;
    }
    if (!a.out && threadIdx.x == 0) {
        a.pml[2 * (r * a.H + h)] = M;
        a.pml[2 * (r * a.H + h) + 1] = Z;
    }
}

}  // namespace

hcsa_status launch_shift_pos(const int32_t *pos, int64_t B, int64_t delta, int32_t *out, cudaStream_t st) {
    shift_pos_kernel<<<(unsigned)((B + 127) / 128), 128, 0, st>>>(pos, B, delta, out);
    count_launch();
    return check_launch();
}

hcsa_status launch_shard_finish(int32_t *sel, int64_t B, int k, const float *scores, int64_t N, int64_t ent0,
                                float *sel_scores, cudaStream_t st) {
    const int64_t n = B * k;
    shard_finish_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(sel, B, k, scores, N, ent0, sel_scores);
    count_launch();
    return check_launch();
}

hcsa_status launch_localize_sel(const int32_t *sel, int64_t n, int64_t ent0, int64_t n_cap, int32_t *out,
                                cudaStream_t st) {
    localize_sel_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(sel, n, ent0, n_cap, out);
    count_launch();
    return check_launch();
}

bool topk_merge_supported(int n_cand, int k) { return n_cand >= 1 && n_cand <= kMergeCap && k >= 1 && k <= n_cand; }

hcsa_status launch_topk_merge(const int32_t *cand_sel, const float *cand_scores, int64_t rows, int n_cand, int k,
                              int32_t *sel, cudaStream_t st) {
    int n = 1, nk = 1;
    while (n < n_cand) n <<= 1;
    while (nk < k) nk <<= 1;
    const size_t smem = sizeof(uint64_t) * (size_t)(n + nk);
    static bool configured[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return HCSA_ERR_CUDA;
    if (!configured[dev]) {
        if (cudaFuncSetAttribute(topk_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)(sizeof(uint64_t) * 2 * kMergeCap)) != cudaSuccess)
            return HCSA_ERR_CUDA;
        configured[dev] = true;
    }
    topk_merge_kernel<<<(unsigned)rows, kMergeThreads, smem, st>>>(cand_sel, cand_scores, n_cand, k, sel);
    count_launch();
    return check_launch();
}

hcsa_status launch_merge_parts(const float *acc, const float *ml, int64_t ss, int64_t sr, int64_t ms, int64_t mr,
                               int n_parts, int64_t rows, int H, int dh, void *out, float *pacc, float *pml,
                               cudaStream_t st) {
    MergeArgs a{acc, ml, ss, sr, ms, mr, n_parts, H, dh, (__nv_bfloat16 *)out, pacc, pml};
    merge_parts_kernel<<<dim3((unsigned)rows, (unsigned)H), 256, 0, st>>>(a);
    count_launch();
    return check_launch();
}

}  // namespace hcsa

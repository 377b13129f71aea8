// Exact top-k over long score rows (decode: one row of up to 2^18 scores per sequence), spread
// over many CTAs per row.
//
// Same selection as every other top-k here: the min(k, n) largest scores of the row, equal scores
// taken lowest index first, emitted in ascending index order.  Scores are compared through an
// order-preserving 32-bit key (-0.0 folded onto +0.0, score_order_key).
//
//   0. the row's histogram of the top 12 key bits is built by the indexer while it writes the
//      scores (shared-memory counts per work unit, added into the global histogram);
//   1. finish, every CTA of a row: find the bucket holding the k-th largest key from the histogram
//      (`above` = keys in higher buckets) and append (key, index) of every key of its slice in that
//      bucket or above to the row's candidate list (one atomic per warp);
//   2. finish, the CTA of the row that completes last: refine the threshold inside the bucket (two
//      10-bit histogram passes over the candidates), mark the chosen indices in a bitmap of the row
//      and emit them in ascending order with a block scan over the bitmap words.
// The candidate list holds at most kCap entries per row; a row whose candidates overflow it, or with
// more than 64 keys tied at the threshold, is flagged and finished by the generic single-CTA select.
#include "internal.cuh"

namespace hcsa {

namespace {

constexpr int kBins = 4096;
constexpr int kSlice = 8192;          // scores per CTA
constexpr int kThreads = 256;
constexpr int kCap = 4096;            // candidates per row
constexpr int kCandPerThread = kCap / kThreads;
constexpr int kMaxRow = 1 << 18;      // rows up to 262144 entries (shared-memory bitmap)
constexpr int kWords = kMaxRow / 32;
// bitmap word w lives at w + w / 32: the 32 words a thread owns in the emission are then in 32 different
// banks across the warp's lanes
__device__ __forceinline__ int bw(int w) { return w + (w >> 5); }
static_assert(kWords <= 32 * kThreads, "emission: 32 bitmap words per thread");
static_assert(kCap * 2 <= kWords, "candidate staging fits in the bitmap");

struct RowArgs {
    const float *scores;
    int64_t N;            // row stride and capacity
    int m, topk;
    const int32_t *pos;   // visible count of row r = min(pos[r] / m, N)
    int32_t *sel;
    const uint32_t *hist; // [rows][kBins]
    int32_t *meta;        // [rows][4]: candidate count, CTAs done, -, overflow flag
    uint64_t *cand;       // [rows][kCap] (key << 32 | index)
};

__device__ __forceinline__ int64_t row_n(const RowArgs &a, int64_t r) {
    const int64_t p = a.pos[r];
    if (p < 0) return 0;
    return p / a.m < a.N ? p / a.m : a.N;
}

// inclusive prefix sum over the block (kThreads), returns the block total in *total
__device__ __forceinline__ uint32_t block_incl_scan(uint32_t v, uint32_t *warp_sums, uint32_t *total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_sums[wid] = incl;
    __syncthreads();
    if (wid == 0) {
        uint32_t s = lane < kThreads / 32 ? warp_sums[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        if (lane < kThreads / 32) warp_sums[lane] = s;
    }
    __syncthreads();
    *total = warp_sums[kThreads / 32 - 1];
    const uint32_t r = incl + (wid > 0 ? warp_sums[wid - 1] : 0);
    __syncthreads();
    return r;
}

__global__ void __launch_bounds__(kThreads) rows_finish_kernel(RowArgs a) {
    __shared__ __align__(16) uint32_t bitmap[kWords + kWords / 32];   // also stages kCap candidates
    __shared__ uint32_t hist[1024];
    __shared__ uint32_t warp_sums[kThreads / 32];
    __shared__ uint32_t eq_idx[64];
    __shared__ uint32_t s_bucket, s_above, s_prefix;
    __shared__ int s_rem, s_eq_cnt, s_last, s_cnt, s_base;
    const int tid = threadIdx.x, lane = tid & 31;
    const int64_t r = blockIdx.y, s0 = (int64_t)blockIdx.x * kSlice;
    const int64_t n = row_n(a, r);
    int32_t *out = a.sel + r * a.topk;
    if (n <= a.topk) {
        if (blockIdx.x == 0)
            for (int i = tid; i < a.topk; i += kThreads) out[i] = i < n ? i : -1;
        return;
    }
    // ---- 1a. threshold bucket: thread t owns bins [16 (255 - t), +16), thread 0 the highest
    {
        constexpr int per = kBins / kThreads;
        const int b0 = per * (kThreads - 1 - tid);
        const uint4 *hv = reinterpret_cast<const uint4 *>(a.hist + r * kBins + b0);
        uint32_t c[per];
#pragma unroll
        for (int i = 0; i < per / 4; ++i) {
            const uint4 x = __ldcg(hv + i);
            c[4 * i] = x.x; c[4 * i + 1] = x.y; c[4 * i + 2] = x.z; c[4 * i + 3] = x.w;
        }
        uint32_t local = 0;
#pragma unroll
        for (int i = 0; i < per; ++i) local += c[i];
        uint32_t total;
        const uint32_t incl = block_incl_scan(local, warp_sums, &total);
        const uint32_t excl = incl - local;
        if (excl < (uint32_t)a.topk && incl >= (uint32_t)a.topk) {
            uint32_t cum = excl;
#pragma unroll
            for (int i = per - 1; i >= 0; --i) {
                if (cum + c[i] >= (uint32_t)a.topk) {
                    s_bucket = (uint32_t)(b0 + i);
                    s_above = cum;
                    break;
                }
                cum += c[i];
            }
        }
        __syncthreads();
    }
    const uint32_t bucket = s_bucket;
    // ---- 1b. candidates of this slice (every key in the threshold bucket or above), staged in shared
    //      memory (the bitmap's space, unused until the select) and appended to the row's list with one
    //      global atomic per CTA
    if (s0 < n) {
        uint64_t *stage = reinterpret_cast<uint64_t *>(bitmap);   // kCap entries
        if (tid == 0) s_cnt = 0;
        __syncthreads();
        const float *row = a.scores + r * a.N;
        const int64_t e = s0 + kSlice < n ? s0 + kSlice : n;
        auto push = [&](uint32_t k, int64_t j, bool take) {
            const uint32_t m = __ballot_sync(0xffffffffu, take);
            if (!m) return;
            int slot = 0;
            if (lane == 0) slot = atomicAdd(&s_cnt, __popc(m));
            slot = __shfl_sync(0xffffffffu, slot, 0) + __popc(m & ((1u << lane) - 1u));
            if (take && slot < kCap) stage[slot] = ((uint64_t)k << 32) | (uint32_t)j;
        };
        if ((a.N & 3) == 0 && e - s0 == kSlice) {
            const float4 *v = reinterpret_cast<const float4 *>(row + s0);
            float4 x[kSlice / 4 / kThreads];
#pragma unroll
            for (int i = 0; i < kSlice / 4 / kThreads; ++i) x[i] = __ldcs(v + tid + i * kThreads);
#pragma unroll
            for (int i = 0; i < kSlice / 4 / kThreads; ++i) {
                const int64_t j = s0 + 4 * (int64_t)(tid + i * kThreads);
                const uint32_t k0 = score_order_key(x[i].x), k1 = score_order_key(x[i].y);
                const uint32_t k2 = score_order_key(x[i].z), k3 = score_order_key(x[i].w);
                if (!__any_sync(0xffffffffu, (k0 >> 20) >= bucket || (k1 >> 20) >= bucket ||
                                                 (k2 >> 20) >= bucket || (k3 >> 20) >= bucket))
                    continue;
                push(k0, j, (k0 >> 20) >= bucket);
                push(k1, j + 1, (k1 >> 20) >= bucket);
                push(k2, j + 2, (k2 >> 20) >= bucket);
                push(k3, j + 3, (k3 >> 20) >= bucket);
            }
        } else {
            for (int64_t base = s0; base < e; base += kThreads) {
                const int64_t j = base + tid;
                uint32_t k = 0;
                bool take = false;
                if (j < e) {
                    k = score_order_key(row[j]);
                    take = (k >> 20) >= bucket;
                }
                push(k, j, take);
            }
        }
        __syncthreads();
        const int cnt = s_cnt;
        if (tid == 0) s_base = cnt ? atomicAdd(&a.meta[r * 4 + 0], cnt) : 0;
        __syncthreads();
        const int base = s_base;
        uint64_t *cand = a.cand + r * kCap;
        for (int i = tid; i < cnt && base + i < kCap; i += kThreads) cand[base + i] = stage[i];
    }
    // ---- the CTA that completes the row last selects
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(&a.meta[r * 4 + 1], 1) == (int)gridDim.x - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const int cnt = __ldcg(&a.meta[r * 4 + 0]);
    if (cnt > kCap) {   // threshold bucket too full for the list: the single-CTA select takes the row
        if (tid == 0) a.meta[r * 4 + 3] = 1;
        return;
    }
    uint32_t ck[kCandPerThread], cj[kCandPerThread];
    {
        const uint64_t *cand = a.cand + r * kCap;
#pragma unroll
        for (int i = 0; i < kCandPerThread; ++i) {
            const int q = tid + i * kThreads;
            const uint64_t c = q < cnt ? __ldcg(cand + q) : 0ull;
            ck[i] = (uint32_t)(c >> 32);
            cj[i] = (uint32_t)c;
        }
    }
    // ---- 2. refine the threshold inside the bucket: bits [10, 20), then [0, 10)
    uint32_t prefix = bucket << 20, mask = 0xFFF00000u;
    int rem = a.topk - (int)s_above;
    for (int pass = 0; pass < 2; ++pass) {
        const int sh = pass == 0 ? 10 : 0;
        for (int i = tid; i < 1024; i += kThreads) hist[i] = 0;
        __syncthreads();
#pragma unroll
        for (int i = 0; i < kCandPerThread; ++i)
            if (tid + i * kThreads < cnt && (ck[i] & mask) == prefix) atomicAdd(&hist[(ck[i] >> sh) & 1023u], 1u);
        __syncthreads();
        // thread t owns bins [4 (255 - t), +4): thread 0 the highest
        const int b0 = 4 * (kThreads - 1 - tid);
        uint32_t c[4], local = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) { c[i] = hist[b0 + i]; local += c[i]; }
        uint32_t total;
        const uint32_t incl = block_incl_scan(local, warp_sums, &total);
        const uint32_t excl = incl - local;
        if (excl < (uint32_t)rem && incl >= (uint32_t)rem) {
            uint32_t cum = excl;
#pragma unroll
            for (int i = 3; i >= 0; --i) {
                if (cum + c[i] >= (uint32_t)rem) {
                    s_prefix = prefix | ((uint32_t)(b0 + i) << sh);
                    s_rem = rem - (int)cum;
                    break;
                }
                cum += c[i];
            }
        }
        __syncthreads();
        prefix = s_prefix;
        rem = s_rem;
        mask |= 1023u << sh;
    }
    // prefix = K*: keys above are taken, plus the `rem` lowest indices among keys equal to K*
    const int nw = (int)((n + 31) / 32);
    for (int i = tid; i < bw(nw); i += kThreads) bitmap[i] = 0;
    if (tid == 0) s_eq_cnt = 0;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kCandPerThread; ++i) {
        if (tid + i * kThreads >= cnt) continue;
        if (ck[i] > prefix) atomicOr(&bitmap[bw(cj[i] >> 5)], 1u << (cj[i] & 31));
        else if (ck[i] == prefix) {
            const int e = atomicAdd(&s_eq_cnt, 1);
            if (e < 64) eq_idx[e] = cj[i];
        }
    }
    __syncthreads();
    if (s_eq_cnt > 64) {   // too many keys tie at the threshold to rank here
        if (tid == 0) a.meta[r * 4 + 3] = 1;
        return;
    }
    if (tid == 0) {
        const int ne = s_eq_cnt;
        // the `rem` lowest indices among the equal keys (repeated minimum; ne <= 64)
        for (int t = 0; t < rem && t < ne; ++t) {
            int best = t;
            for (int q = t + 1; q < ne; ++q)
                if (eq_idx[q] < eq_idx[best]) best = q;
            const uint32_t tmp = eq_idx[t];
            eq_idx[t] = eq_idx[best];
            eq_idx[best] = tmp;
            bitmap[bw(eq_idx[t] >> 5)] |= 1u << (eq_idx[t] & 31);
        }
    }
    __syncthreads();
    // ascending emission: thread t owns words [32 t, 32 t + 32) (nw <= 32 x 256; the padded layout puts
    // them in 32 different banks across a warp); one block scan of the threads' bit counts gives the
    // output positions.  The loops stay rolled: this code runs once per launch, from a cold
    // instruction cache.
    uint32_t local = 0;
#pragma unroll 1
    for (int i = 0; i < 32; ++i) {
        const int w = tid * 32 + i;
        local += w < nw ? __popc(bitmap[bw(w)]) : 0u;
    }
    uint32_t total;
    int q = (int)(block_incl_scan(local, warp_sums, &total) - local);
#pragma unroll 1
    for (int i = 0; i < 32; ++i) {
        const int w = tid * 32 + i;
        uint32_t bits = w < nw ? bitmap[bw(w)] : 0u;
        while (bits) {
            const int b = __ffs(bits) - 1;
            bits &= bits - 1;
            if (q < a.topk) out[q] = w * 32 + b;
            ++q;
        }
    }
}

}  // namespace

bool topk_rows_supported(const IndexArgs &a) {
    return a.pos != nullptr && a.dtype == HCSA_BF16 && a.topk <= kCap && a.N > 32768 && a.N <= kMaxRow;
}

size_t topk_rows_ws_bytes(int64_t rows) {
    return (size_t)rows * (kBins * sizeof(uint32_t) + 4 * sizeof(int32_t) + kCap * sizeof(uint64_t));
}

hcsa_status topk_rows_begin(const IndexArgs &ia, void *scratch, cudaStream_t st) {
    // histogram and per-row counters start at zero (they are contiguous at the start of the scratch)
    const size_t n = (size_t)ia.rows * (kBins * sizeof(uint32_t) + 4 * sizeof(int32_t));
    return cudaMemsetAsync(scratch, 0, n, st) == cudaSuccess ? HCSA_OK : HCSA_ERR_CUDA;
}

const int32_t *topk_rows_flags(const IndexArgs &ia, const void *scratch) {
    return reinterpret_cast<const int32_t *>((const uint8_t *)scratch + (size_t)ia.rows * kBins * sizeof(uint32_t));
}

hcsa_status launch_topk_rows(const IndexArgs &ia, void *scratch, cudaStream_t st) {
    RowArgs a{};
    a.scores = (const float *)ia.ws;
    a.N = ia.N;
    a.m = ia.m;
    a.topk = ia.topk;
    a.pos = ia.pos;
    a.sel = ia.sel;
    uint8_t *p = (uint8_t *)scratch;
    a.hist = (const uint32_t *)p;
    p += (size_t)ia.rows * kBins * sizeof(uint32_t);
    a.meta = (int32_t *)p;
    p += (size_t)ia.rows * 4 * sizeof(int32_t);
    a.cand = (uint64_t *)(((uintptr_t)p + 15) & ~uintptr_t(15));
    const int64_t slices = (ia.N + kSlice - 1) / kSlice;
    if (slices > 65535 || ia.rows > 65535) return HCSA_ERR_UNSUPPORTED;
    rows_finish_kernel<<<dim3((unsigned)slices, (unsigned)ia.rows), kThreads, 0, st>>>(a);
    count_launch();
    return check_launch();
}

}  // namespace hcsa

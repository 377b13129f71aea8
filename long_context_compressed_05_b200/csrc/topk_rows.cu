// Exact top-k over long score rows (decode: one row of up to 2^31 scores per sequence), spread
// over many CTAs per row.
//
// Same selection as every other top-k here: the min(k, n) largest scores of the row, equal scores
// taken lowest index first, emitted in ascending index order.  Scores are compared through an
// order-preserving 32-bit key (-0.0 folded onto +0.0).
//
//   1. hist:    each CTA histograms the top 12 key bits of its slice of the row (shared memory),
//               then adds its counts into the row's global histogram.
//   2. bucket:  one CTA per row finds the bucket holding the k-th largest key: `above` = how many
//               keys are in higher buckets.
//   3. collect: each CTA appends (key, index) of every key in that bucket or above to the row's
//               candidate list (one atomic per warp).
//   4. select:  one CTA per row sorts the candidates by (key desc, index asc) in shared memory,
//               keeps the first k and sorts their indices ascending.
// The candidate list holds at most `cap` entries per row; a row whose threshold bucket overflows
// it is finished by the generic single-CTA select instead.
#include "internal.cuh"

namespace hcsa {

namespace {

constexpr int kBins = 4096;
constexpr int kSlice = 8192;          // scores per CTA in passes 1 and 3
constexpr int kThreads = 256;
constexpr int kCap = 4096;            // candidates per row (power of two, sorted in shared memory)

__device__ __forceinline__ uint32_t okey(float s) {
    if (s == 0.0f) s = 0.0f;
    const uint32_t b = __float_as_uint(s);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

struct RowArgs {
    const float *scores;
    int64_t N;            // row stride and capacity
    int m, topk;
    const int32_t *pos;   // visible count of row r = min(pos[r] / m, N)
    int32_t *sel;
    uint32_t *hist;       // [rows][kBins]
    int32_t *meta;        // [rows][4]: bucket, above, count, overflow
    uint64_t *cand;       // [rows][kCap] (key << 32 | index)
    int64_t slices;       // CTAs per row
};

__device__ __forceinline__ int64_t row_n(const RowArgs &a, int64_t r) {
    const int64_t p = a.pos[r];
    if (p < 0) return 0;
    return p / a.m < a.N ? p / a.m : a.N;
}

__global__ void __launch_bounds__(kThreads) rows_hist_kernel(RowArgs a) {
    __shared__ uint32_t h[kBins];
    const int64_t r = blockIdx.y, s0 = (int64_t)blockIdx.x * kSlice;
    const int64_t n = row_n(a, r);
    if (n <= a.topk || s0 >= n) return;
    for (int i = threadIdx.x; i < kBins; i += kThreads) h[i] = 0;
    __syncthreads();
    const float *row = a.scores + r * a.N;
    const int64_t e = s0 + kSlice < n ? s0 + kSlice : n;
    if ((a.N & 3) == 0 && e - s0 == kSlice) {   // full slice, 16-byte aligned: vector loads
        const float4 *v = reinterpret_cast<const float4 *>(row + s0);
#pragma unroll 4
        for (int i = threadIdx.x; i < kSlice / 4; i += kThreads) {
            const float4 x = v[i];
            atomicAdd(&h[okey(x.x) >> 20], 1u);
            atomicAdd(&h[okey(x.y) >> 20], 1u);
            atomicAdd(&h[okey(x.z) >> 20], 1u);
            atomicAdd(&h[okey(x.w) >> 20], 1u);
        }
    } else {
        for (int64_t j = s0 + threadIdx.x; j < e; j += kThreads) atomicAdd(&h[okey(row[j]) >> 20], 1u);
    }
    __syncthreads();
    uint32_t *g = a.hist + r * kBins;
    for (int i = threadIdx.x; i < kBins; i += kThreads)
        if (h[i]) atomicAdd(&g[i], h[i]);
}

__global__ void __launch_bounds__(kThreads) rows_bucket_kernel(RowArgs a) {
    __shared__ uint32_t part[kThreads];
    const int64_t r = blockIdx.x;
    const int64_t n = row_n(a, r);
    if (n <= a.topk) return;
    const uint32_t *g = a.hist + r * kBins;
    // thread t owns bins [16 (255 - t), +16): thread 0 the highest
    constexpr int per = kBins / kThreads;
    const int b0 = per * (kThreads - 1 - threadIdx.x);
    uint32_t local = 0;
    for (int i = 0; i < per; ++i) local += g[b0 + i];
    part[threadIdx.x] = local;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t cum = 0;
        int t = 0;
        for (; t < kThreads; ++t) {
            if (cum + part[t] >= (uint32_t)a.topk) break;
            cum += part[t];
        }
        const int bb0 = per * (kThreads - 1 - t);
        int bucket = bb0;
        for (int i = per - 1; i >= 0; --i) {
            if (cum + g[bb0 + i] >= (uint32_t)a.topk) { bucket = bb0 + i; break; }
            cum += g[bb0 + i];
        }
        a.meta[r * 4 + 0] = bucket;
        a.meta[r * 4 + 1] = (int32_t)cum;                 // keys in higher buckets
        a.meta[r * 4 + 2] = 0;
        a.meta[r * 4 + 3] = (int32_t)(cum + g[bucket] > (uint32_t)kCap);
    }
}

__global__ void __launch_bounds__(kThreads) rows_collect_kernel(RowArgs a) {
    const int64_t r = blockIdx.y, s0 = (int64_t)blockIdx.x * kSlice;
    const int64_t n = row_n(a, r);
    if (n <= a.topk || s0 >= n || a.meta[r * 4 + 3]) return;
    const uint32_t bucket = (uint32_t)a.meta[r * 4 + 0];
    const float *row = a.scores + r * a.N;
    uint64_t *cand = a.cand + r * kCap;
    const int64_t e = s0 + kSlice < n ? s0 + kSlice : n;
    const int lane = threadIdx.x & 31;
    auto push = [&](uint32_t k, int64_t j, bool take) {
        const uint32_t m = __ballot_sync(0xffffffffu, take);
        if (!m) return;
        int slot = 0;
        if (lane == 0) slot = atomicAdd(&a.meta[r * 4 + 2], __popc(m));
        slot = __shfl_sync(0xffffffffu, slot, 0) + __popc(m & ((1u << lane) - 1u));
        if (take && slot < kCap) cand[slot] = ((uint64_t)k << 32) | (uint32_t)j;
    };
    if ((a.N & 3) == 0 && e - s0 == kSlice) {
        const float4 *v = reinterpret_cast<const float4 *>(row + s0);
        for (int i = threadIdx.x; i < kSlice / 4; i += kThreads) {
            const float4 x = v[i];
            const int64_t j = s0 + 4 * (int64_t)i;
            const uint32_t k0 = okey(x.x), k1 = okey(x.y), k2 = okey(x.z), k3 = okey(x.w);
            if (!__any_sync(0xffffffffu, (k0 >> 20) >= bucket || (k1 >> 20) >= bucket || (k2 >> 20) >= bucket ||
                                             (k3 >> 20) >= bucket))
                continue;
            push(k0, j, (k0 >> 20) >= bucket);
            push(k1, j + 1, (k1 >> 20) >= bucket);
            push(k2, j + 2, (k2 >> 20) >= bucket);
            push(k3, j + 3, (k3 >> 20) >= bucket);
        }
    } else {
        for (int64_t base = s0; base < e; base += kThreads) {
            const int64_t j = base + threadIdx.x;
            uint32_t k = 0;
            bool take = false;
            if (j < e) {
                k = okey(row[j]);
                take = (k >> 20) >= bucket;
            }
            push(k, j, take);
        }
    }
}

// bitonic sort of n (power of two) 64-bit values in shared memory, descending
__device__ void sort_desc(uint64_t *v, int n) {
    for (int size = 2; size <= n; size <<= 1)
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            __syncthreads();
            for (int i = threadIdx.x; i < n / 2; i += blockDim.x) {
                const int lo = 2 * i - (i & (stride - 1)), hi = lo + stride;
                const bool desc = (lo & size) == 0;
                const uint64_t x = v[lo], y = v[hi];
                if ((x < y) == desc) { v[lo] = y; v[hi] = x; }
            }
        }
    __syncthreads();
}

__global__ void __launch_bounds__(1024) rows_select_kernel(RowArgs a) {
    extern __shared__ uint64_t v[];   // kCap
    const int64_t r = blockIdx.x;
    const int64_t n = row_n(a, r);
    int32_t *out = a.sel + r * a.topk;
    if (n <= a.topk) {
        for (int i = threadIdx.x; i < a.topk; i += blockDim.x) out[i] = i < n ? i : -1;
        return;
    }
    if (a.meta[r * 4 + 3]) return;   // finished by the single-CTA select
    const int cnt = a.meta[r * 4 + 2];
    int n2 = 1;
    while (n2 < cnt) n2 <<= 1;
    // (key desc, index asc): store key << 32 | ~index so a descending sort puts lower indices first
    for (int i = threadIdx.x; i < n2; i += blockDim.x) {
        uint64_t x = 0;
        if (i < cnt) {
            const uint64_t c = a.cand[r * kCap + i];
            x = (c & 0xFFFFFFFF00000000ull) | (uint32_t)(~(uint32_t)c);
        }
        v[i] = x;
    }
    sort_desc(v, n2);
    // the first topk entries are the selection; re-sort their indices ascending (as descending ~index)
    int k2 = 1;
    while (k2 < a.topk) k2 <<= 1;
    __syncthreads();
    for (int i = threadIdx.x; i < k2; i += blockDim.x) v[i] = i < a.topk ? (uint64_t)(uint32_t)v[i] : 0;
    sort_desc(v, k2);   // ~index descending == index ascending
    for (int i = threadIdx.x; i < a.topk; i += blockDim.x) out[i] = (int32_t)(~(uint32_t)v[i]);
}

}  // namespace

bool topk_rows_supported(const IndexArgs &a) {
    return a.pos != nullptr && a.dtype == HCSA_BF16 && a.topk <= 2048 && a.N > 32768 && a.N <= INT32_MAX;
}

size_t topk_rows_ws_bytes(int64_t rows) {
    return (size_t)rows * (kBins * sizeof(uint32_t) + 4 * sizeof(int32_t) + kCap * sizeof(uint64_t));
}

hcsa_status launch_topk_rows(const IndexArgs &ia, void *extra, cudaStream_t st) {
    RowArgs a{};
    a.scores = (const float *)ia.ws;
    a.N = ia.N;
    a.m = ia.m;
    a.topk = ia.topk;
    a.pos = ia.pos;
    a.sel = ia.sel;
    uint8_t *p = (uint8_t *)extra;
    a.hist = (uint32_t *)p;
    p += (size_t)ia.rows * kBins * sizeof(uint32_t);
    a.meta = (int32_t *)p;
    p += (size_t)ia.rows * 4 * sizeof(int32_t);
    a.cand = (uint64_t *)(((uintptr_t)p + 15) & ~uintptr_t(15));
    a.slices = (ia.N + kSlice - 1) / kSlice;
    if (a.slices > 65535 || ia.rows > 65535) return HCSA_ERR_UNSUPPORTED;
    if (cudaMemsetAsync(a.hist, 0, (size_t)ia.rows * kBins * sizeof(uint32_t), st) != cudaSuccess)
        return HCSA_ERR_CUDA;
    dim3 g2((unsigned)a.slices, (unsigned)ia.rows);
    rows_hist_kernel<<<g2, kThreads, 0, st>>>(a);
    rows_bucket_kernel<<<(unsigned)ia.rows, kThreads, 0, st>>>(a);
    rows_collect_kernel<<<g2, kThreads, 0, st>>>(a);
    static bool configured = false;
    if (!configured) {
        if (cudaFuncSetAttribute(rows_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)(kCap * sizeof(uint64_t))) != cudaSuccess)
            return HCSA_ERR_CUDA;
        configured = true;
    }
    rows_select_kernel<<<(unsigned)ia.rows, 1024, kCap * sizeof(uint64_t), st>>>(a);
    count_launch(4);
    return check_launch();
}

}  // namespace hcsa

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
//   4. select:  one CTA per row refines the threshold inside the bucket (two 10-bit histogram passes
//               over the candidates), marks the chosen indices in a bitmap of the row and emits them in
//               ascending order with a block scan over the bitmap words.
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

constexpr int kSelThreads = 1024;
constexpr int kMaxRow = 1 << 18;   // rows up to 262144 entries use the shared-memory bitmap

// Exact selection among the candidates of one row, then the indices in ascending order:
//   two 10-bit histogram passes over the low 20 key bits of the threshold-bucket candidates give the
//   k-th largest key K* and how many keys equal to K* are taken (lowest index first); every chosen
//   index is set in a bitmap of the row, and a block scan over the bitmap words emits them in order.
__global__ void __launch_bounds__(kSelThreads) rows_select_kernel(RowArgs a) {
    extern __shared__ uint32_t sm[];
    uint32_t *bitmap = sm;                       // kMaxRow / 32 words
    uint32_t *hist = bitmap + kMaxRow / 32;      // 1024 bins
    __shared__ uint32_t s_prefix;
    __shared__ int s_rem, s_eq_cnt, s_base;
    __shared__ uint32_t eq_idx[64];
    __shared__ uint32_t warp_sums[kSelThreads / 32];
    const int64_t r = blockIdx.x;
    const int64_t n = row_n(a, r);
    int32_t *out = a.sel + r * a.topk;
    const int tid = threadIdx.x;
    if (n <= a.topk) {
        for (int i = tid; i < a.topk; i += kSelThreads) out[i] = i < n ? i : -1;
        return;
    }
    if (a.meta[r * 4 + 3]) return;   // finished by the single-CTA select
    const int cnt = a.meta[r * 4 + 2];
    const uint32_t bucket = (uint32_t)a.meta[r * 4 + 0];
    const uint64_t *cand = a.cand + r * kCap;
    // refine the threshold inside the bucket: bits [10, 20), then [0, 10)
    uint32_t prefix = bucket << 20, mask = 0xFFF00000u;
    int rem = a.topk - a.meta[r * 4 + 1];
    for (int pass = 0; pass < 2; ++pass) {
        const int sh = pass == 0 ? 10 : 0;
        for (int i = tid; i < 1024; i += kSelThreads) hist[i] = 0;
        __syncthreads();
        for (int i = tid; i < cnt; i += kSelThreads) {
            const uint32_t k = (uint32_t)(cand[i] >> 32);
            if ((k & mask) == prefix) atomicAdd(&hist[(k >> sh) & 1023u], 1u);
        }
        __syncthreads();
        if (tid < 32) {   // one warp scans the 1024 bins from the top
            uint32_t local = 0;
            for (int i = 0; i < 32; ++i) local += hist[1023 - (tid * 32 + i)];
            uint32_t incl = local;
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
                if (tid >= o) incl += y;
            }
            const uint32_t excl = incl - local;
            if (excl < (uint32_t)rem && incl >= (uint32_t)rem) {
                uint32_t cum = excl;
                for (int i = 0; i < 32; ++i) {
                    const int bin = 1023 - (tid * 32 + i);
                    if (cum + hist[bin] >= (uint32_t)rem) {
                        s_prefix = prefix | ((uint32_t)bin << sh);
                        s_rem = rem - (int)cum;
                        break;
                    }
                    cum += hist[bin];
                }
            }
        }
        __syncthreads();
        prefix = s_prefix;
        rem = s_rem;
        mask |= 1023u << sh;
        __syncthreads();
    }
    // prefix = K*: keys above are taken, plus the `rem` lowest indices among keys equal to K*
    for (int i = tid; i < (int)((n + 31) / 32); i += kSelThreads) bitmap[i] = 0;
    if (tid == 0) s_eq_cnt = 0;
    __syncthreads();
    for (int i = tid; i < cnt; i += kSelThreads) {
        const uint64_t c = cand[i];
        const uint32_t k = (uint32_t)(c >> 32), j = (uint32_t)c;
        if (k > prefix) atomicOr(&bitmap[j >> 5], 1u << (j & 31));
        else if (k == prefix) {
            const int e = atomicAdd(&s_eq_cnt, 1);
            if (e < 64) eq_idx[e] = j;
        }
    }
    __syncthreads();
    if (s_eq_cnt > 64) {
        // too many keys tie at the threshold to rank here: hand the row to the single-CTA select
        if (tid == 0) a.meta[r * 4 + 3] = 1;
        return;
    }
    if (tid == 0) {
        int ne = s_eq_cnt < 64 ? s_eq_cnt : 64;
        // take the `rem` lowest indices among the equal keys (selection by repeated minimum; ne is small)
        for (int t = 0; t < rem && t < ne; ++t) {
            int best = t;
            for (int q = t + 1; q < ne; ++q)
                if (eq_idx[q] < eq_idx[best]) best = q;
            const uint32_t tmp = eq_idx[t];
            eq_idx[t] = eq_idx[best];
            eq_idx[best] = tmp;
            bitmap[eq_idx[t] >> 5] |= 1u << (eq_idx[t] & 31);
        }
    }
    __syncthreads();
    // ascending emission: each thread owns a contiguous range of bitmap words
    const int nw = (int)((n + 31) / 32);
    const int per = (nw + kSelThreads - 1) / kSelThreads;
    const int w0 = tid * per;
    int local = 0;
    for (int w = w0; w < w0 + per && w < nw; ++w) local += __popc(bitmap[w]);
    int incl = local;
    const int lane = tid & 31, wid = tid >> 5;
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_sums[wid] = (uint32_t)incl;
    __syncthreads();
    if (wid == 0) {
        int v = lane < kSelThreads / 32 ? (int)warp_sums[lane] : 0;
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += y;
        }
        if (lane < kSelThreads / 32) warp_sums[lane] = (uint32_t)v;
    }
    __syncthreads();
    int pos = incl - local + (wid > 0 ? (int)warp_sums[wid - 1] : 0);
    for (int w = w0; w < w0 + per && w < nw; ++w) {
        uint32_t bits = bitmap[w];
        while (bits) {
            const int b = __ffs(bits) - 1;
            bits &= bits - 1;
            if (pos < a.topk) out[pos] = w * 32 + b;
            ++pos;
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
    constexpr size_t sel_smem = (kMaxRow / 32 + 1024) * sizeof(uint32_t);
    static bool configured = false;
    if (!configured) {
        if (cudaFuncSetAttribute(rows_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sel_smem) !=
            cudaSuccess)
            return HCSA_ERR_CUDA;
        configured = true;
    }
    rows_select_kernel<<<(unsigned)ia.rows, kSelThreads, sel_smem, st>>>(a);
    count_launch(4);
    return check_launch();
}

}  // namespace hcsa

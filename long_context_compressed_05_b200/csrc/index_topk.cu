// Lightning indexer + exact top-k (CUDA-core form, used for fp32 storage and
// for every decode batch).
//
// "DeepSeek-V4 ... KV cache compressed attention", section "CSA: compresion 4x":
// the query first scores the compressed blocks with the Lightning Indexer and
// keeps the top-k; the score is fixed by the CSA workload definition as
//   s[t,j] = sum_h w[t,h] ReLU(qi[t,h,:] . k_j)   (j visible iff m j + m <= t),
// and top-k keeps the min(k, visible) largest, equal scores going to the lower j.
//
// Scores are materialised in the workspace (one row per query), then one CTA per
// query runs an MSB-first radix select on order-preserving integer keys (-0.0
// folded onto +0.0 so that equal scores compare equal), and writes the chosen
// indices in ascending order with two block scans (rank among equal keys, output
// slot).  The result is the unique (score desc, index asc) top-k set.
#include <cub/block/block_scan.cuh>

#include "internal.cuh"

namespace hcsa {

// ---------------------------------------------------------------- scores
constexpr int kQT = 8;    // queries per CTA (prefill)
constexpr int kJT = 64;   // entries per CTA

template <typename S>
__global__ void __launch_bounds__(256) index_scores_kernel(IndexArgs a, int qt) {
    using A = typename Traits<S>::A;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    A *sq = reinterpret_cast<A *>(smem_raw);             // [qt][Hi*di]
    A *sw = sq + qt * a.Hi * a.di;                       // [qt][Hi]
    A *sk = sw + qt * a.Hi;                              // [kJT][di + 1]
    const int hd = a.Hi * a.di;
    const int64_t r0 = a.row0 + (int64_t)blockIdx.y * qt;   // query tile of the row range
    const int64_t j0 = (int64_t)blockIdx.x * kJT;
    // visible entries of the last query in the tile bound the whole tile
    int64_t last = r0 + qt - 1 < a.row1 ? r0 + qt - 1 : a.row1 - 1;
    int64_t pmax = a.pos ? a.pos[last] : last;
    int64_t nv_max = pmax / a.m < a.N ? pmax / a.m : a.N;
    if (a.pos) {   // decode: qt == 1, one sequence per row
        nv_max = a.pos[r0] / a.m < a.N ? a.pos[r0] / a.m : a.N;
        if (a.pos[r0] < 0) nv_max = 0;
    }
    if (j0 >= nv_max) return;
    const S *qi = reinterpret_cast<const S *>(a.qi);
    const S *w = reinterpret_cast<const S *>(a.w);
    const S *keys = reinterpret_cast<const S *>(a.keys) + (a.pos ? r0 * a.N * a.di : 0);
    for (int i = threadIdx.x; i < qt * hd; i += blockDim.x) {
        int64_t r = r0 + i / hd;
        sq[i] = r < a.row1 ? to_acc(qi[r * a.ld_qi + i % hd], A()) : A(0);
    }
    for (int i = threadIdx.x; i < qt * a.Hi; i += blockDim.x) {
        int64_t r = r0 + i / a.Hi;
        sw[i] = r < a.row1 ? to_acc(w[r * a.ld_w + i % a.Hi], A()) : A(0);
    }
    for (int i = threadIdx.x; i < kJT * a.di; i += blockDim.x) {
        int64_t j = j0 + i / a.di;
        sk[(i / a.di) * (a.di + 1) + i % a.di] = j < a.N ? to_acc(keys[j * a.di + i % a.di], A()) : A(0);
    }
    __syncthreads();
    A *scores = reinterpret_cast<A *>(a.ws);
    const int jl = threadIdx.x % kJT;
    const int64_t j = j0 + jl;
    for (int ql = threadIdx.x / kJT; ql < qt; ql += blockDim.x / kJT) {
        const int64_t r = r0 + ql;
        if (r >= a.row1) break;
        const int64_t p = a.pos ? a.pos[r] : r;
        const int64_t nv = p < 0 ? 0 : (p / a.m < a.N ? p / a.m : a.N);
        if (j >= nv) continue;
        const A *qrow = sq + ql * hd;
        const A *krow = sk + jl * (a.di + 1);
        A acc = A(0);
        for (int h = 0; h < a.Hi; ++h) {
            A dot = A(0);
            for (int d = 0; d < a.di; ++d) dot += qrow[h * a.di + d] * krow[d];
            acc += sw[ql * a.Hi + h] * (dot > A(0) ? dot : A(0));
        }
        scores[r * a.N + j] = acc;
    }
}

// ---------------------------------------------------------------- top-k
template <typename A> struct OrderKey;
template <> struct OrderKey<float> {
    using K = uint32_t;
    static constexpr int BITS = 32;
    __device__ static K of(float s) {
        if (s == 0.0f) s = 0.0f;   // fold -0 onto +0
        K b = __float_as_uint(s);
        return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
    }
};
template <> struct OrderKey<double> {
    using K = unsigned long long;
    static constexpr int BITS = 64;
    __device__ static K of(double s) {
        if (s == 0.0) s = 0.0;
        K b = (K)__double_as_longlong(s);
        return (b & 0x8000000000000000ull) ? ~b : (b | 0x8000000000000000ull);
    }
};

constexpr int kTopkThreads = 512;

template <typename A>
__global__ void __launch_bounds__(kTopkThreads) topk_kernel(IndexArgs a) {
    using OK = OrderKey<A>;
    using K = typename OK::K;
    using Scan = cub::BlockScan<int, kTopkThreads>;
    __shared__ typename Scan::TempStorage scan_tmp;
    __shared__ int hist[256];
    __shared__ int s_digit, s_rem;
    __shared__ int s_base_eq, s_base_out;

    const int64_t r = a.row0 + blockIdx.x;
    if (a.only_rows && a.only_rows[4 * r + 3] == 0) return;
    const int64_t p = a.pos ? a.pos[r] : r;
    const int64_t n = p < 0 ? 0 : (p / a.m < a.N ? p / a.m : a.N);
    const int k = a.topk;
    int32_t *out = a.sel + r * k;
    const A *s = reinterpret_cast<const A *>(a.ws) + r * a.N;

    if (n <= k) {
        for (int i = threadIdx.x; i < k; i += blockDim.x) out[i] = i < n ? i : -1;
        return;
    }
    K prefix = 0, mask = 0;
    int rem = k;
    for (int shift = OK::BITS - 8; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
        __syncthreads();
        for (int64_t j = threadIdx.x; j < n; j += blockDim.x) {
            K key = OK::of(s[j]);
            if ((key & mask) == prefix) atomicAdd(&hist[(int)((key >> shift) & 0xFF)], 1);
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            int cum = 0, d = 255;
            for (; d > 0; --d) {
                if (cum + hist[d] >= rem) break;
                cum += hist[d];
            }
            s_digit = d;
            s_rem = rem - cum;
        }
        __syncthreads();
        prefix |= (K)s_digit << shift;
        mask |= (K)0xFF << shift;
        rem = s_rem;
        __syncthreads();
    }
    // prefix is the k-th largest key; rem = how many keys equal to it are taken (lowest j first)
    if (threadIdx.x == 0) { s_base_eq = 0; s_base_out = 0; }
    __syncthreads();
    for (int64_t c0 = 0; c0 < n; c0 += blockDim.x) {
        const int64_t j = c0 + threadIdx.x;
        K key = j < n ? OK::of(s[j]) : 0;
        int gt = (j < n && key > prefix) ? 1 : 0;
        int eq = (j < n && key == prefix) ? 1 : 0;
        int eq_rank, eq_total;
        Scan(scan_tmp).ExclusiveSum(eq, eq_rank, eq_total);
        __syncthreads();
        const int base_eq = s_base_eq, base_out = s_base_out;
        int take = gt | (eq & (base_eq + eq_rank < rem ? 1 : 0));
        int slot, total;
        Scan(scan_tmp).ExclusiveSum(take, slot, total);
        if (take && base_out + slot < k) out[base_out + slot] = (int32_t)j;
        __syncthreads();
        if (threadIdx.x == 0) { s_base_eq = base_eq + eq_total; s_base_out = base_out + total; }
        __syncthreads();
    }
}

size_t index_topk_ws_bytes(int dtype, int64_t rows, int64_t N) {
    const size_t scores = (size_t)rows * (size_t)N * (dtype == HCSA_BF16 ? sizeof(float) : sizeof(double));
    if (dtype != HCSA_BF16) return scores;
    // bf16 (tensor-core indexer): after the scores, 256-byte aligned, a per-row key bound and a per-row flag
    return ((scores + 255) & ~(size_t)255) + (size_t)rows * 2 * sizeof(uint32_t);
}

hcsa_status launch_topk_generic(const IndexArgs &a, cudaStream_t st) {
    const unsigned nrows = (unsigned)(a.row1 - a.row0);
    if (nrows == 0) return HCSA_OK;
    if (a.dtype == HCSA_BF16) topk_kernel<float><<<nrows, kTopkThreads, 0, st>>>(a);
    else topk_kernel<double><<<nrows, kTopkThreads, 0, st>>>(a);
    count_launch();
    return check_launch();
}

hcsa_status launch_index_topk(const IndexArgs &a, cudaStream_t st) {
    if (a.rows == 0) return HCSA_OK;
    if (index_tc_supported(a)) return launch_index_tc(a, st);
    if (a.lowprec) return HCSA_ERR_UNSUPPORTED;   // FP4 keys: tensor-core shapes only
    // CUDA-core scores + generic select: the scores are materialised in the workspace
    if (a.ws_bytes < index_topk_ws_bytes(a.dtype, a.rows, a.N)) return HCSA_ERR_WORKSPACE;
    const int qt = a.pos ? 1 : kQT;
    const size_t esz = a.dtype == HCSA_BF16 ? sizeof(float) : sizeof(double);
    const size_t smem = esz * ((size_t)qt * a.Hi * a.di + (size_t)qt * a.Hi + (size_t)kJT * (a.di + 1));
    if (smem > 200 * 1024) return HCSA_ERR_UNSUPPORTED;
    dim3 grid((unsigned)((a.N + kJT - 1) / kJT), (unsigned)((a.row1 - a.row0 + qt - 1) / qt));
    if (grid.y > 65535 || a.rows > INT32_MAX) return HCSA_ERR_UNSUPPORTED;
    if (a.N > 0) {
        if (a.dtype == HCSA_BF16) {
            auto kern = index_scores_kernel<__nv_bfloat16>;
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            kern<<<grid, 256, smem, st>>>(a, qt);
        } else {
            auto kern = index_scores_kernel<float>;
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            kern<<<grid, 256, smem, st>>>(a, qt);
        }
        count_launch();
    }
    return launch_topk_generic(a, st);
}

}  // namespace hcsa

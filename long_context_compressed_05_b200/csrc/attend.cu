// Attention over the compressed branch united with the raw sliding window
// (CUDA-core form: fp32 storage, and every shape the tensor-core kernels do not
// take).
//
// "DeepSeek-V4 ... KV cache compressed attention", section "Ventana
// deslizante": the attention blocks concatenate the compressed long-range
// branch with sliding-window K/V.  With the operator fixed by the CSA workload
// definition: MQA, key = first C/2 channels of a row, value = last C/2; the key
// set of query t is the selected entries (CSA) or every visible entry (HCA)
// plus the raw tokens (t - window, t]; one softmax with scale tau.
//
// One warp per (query, head), online softmax over the key list.  Decode splits
// the key list into chunks (one CTA each) and merges the partial
// (max, sum, accumulator) triples with a log-sum-exp combine kernel.
#include "internal.cuh"

namespace hcsa {

constexpr int kHeadsPerCta = 8;
constexpr int kMaxEpl = 16;          // dh <= 512
constexpr int kDecodeSplit = 128;    // keys per split (decode)

// Key row kk of query r: entries first (the selection, or every visible entry), then the raw window.
// A selected index that is neither the -1 padding nor a visible entry is skipped and reported.
template <typename S>
__device__ __forceinline__ const S *key_row(const AttendArgs &a, int64_t r, int64_t p, int64_t ne, int64_t nvis,
                                            int64_t kk, int *status) {
    const S *ent = reinterpret_cast<const S *>(a.entries) + (a.pos ? r * a.N * a.C : 0);
    if (kk < ne) {
        int64_t j = a.dense ? kk : (int64_t)a.sel[r * a.topk + kk];
        if (j < 0 || j >= nvis) {
            if (j != -1) report(status, kStatusBounds);
            return nullptr;
        }
        return ent + j * a.C;
    }
    int64_t pp = p - a.window + 1 + (kk - ne);
    if (pp < 0) return nullptr;
    if (a.pos) return reinterpret_cast<const S *>(a.kv) + (r * a.window + pp % a.window) * (int64_t)a.C;
    return reinterpret_cast<const S *>(a.kv) + pp * a.ld_kv;
}

template <typename S>
__global__ void __launch_bounds__(kHeadsPerCta * 32) attend_kernel(AttendArgs a, int nsplit, int *status) {
    using A = typename Traits<S>::A;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int h = blockIdx.y * kHeadsPerCta + warp;
    const int64_t r = a.row0 + blockIdx.x;
    const int split = blockIdx.z;
    if (h >= a.H) return;
    const int64_t p = a.pos ? a.pos[r] : r;
    const int64_t nvis = p < 0 ? 0 : (p / a.m < a.N ? p / a.m : a.N);
    const int64_t ne = a.dense ? nvis : a.topk;
    const int64_t nk = ne + a.window;
    const int64_t per = (nk + nsplit - 1) / nsplit;
    const int64_t k0 = split * per, k1 = k0 + per < nk ? k0 + per : nk;
    const int epl = (a.dh + 31) / 32;
    const S *qrow = reinterpret_cast<const S *>(a.q) + r * a.ld_q + (int64_t)h * a.dh;
    A q[kMaxEpl], acc[kMaxEpl];
#pragma unroll
    for (int i = 0; i < kMaxEpl; ++i) {
        int d = lane + 32 * i;
        q[i] = (i < epl && d < a.dh) ? to_acc(qrow[d], A()) : A(0);
        acc[i] = A(0);
    }
    A mx = -INFINITY, z = A(0);
    const A scale = (A)a.scale;
    for (int64_t kk = k0; kk < k1; ++kk) {
        const S *row = key_row<S>(a, r, p, ne, nvis, kk, status);
        if (!row) continue;
        A dot = A(0);
#pragma unroll
        for (int i = 0; i < kMaxEpl; ++i) {
            int d = lane + 32 * i;
            if (i < epl && d < a.dh) dot += q[i] * to_acc(row[d], A());
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
        const A logit = dot * scale;
        const A mnew = logit > mx ? logit : mx;
        const A corr = exp_acc(mx - mnew);
        const A pr = exp_acc(logit - mnew);
        z = z * corr + pr;
        const S *v = row + a.C / 2;
#pragma unroll
        for (int i = 0; i < kMaxEpl; ++i) {
            int d = lane + 32 * i;
            if (i < epl && d < a.dh) acc[i] = acc[i] * corr + pr * to_acc(v[d], A());
        }
        mx = mnew;
    }
    if (nsplit == 1) {
        S *o = reinterpret_cast<S *>(a.out) + r * (int64_t)a.H * a.dh + (int64_t)h * a.dh;
#pragma unroll
        for (int i = 0; i < kMaxEpl; ++i) {
            int d = lane + 32 * i;
            if (i < epl && d < a.dh) store_val(&o[d], z > A(0) ? acc[i] / z : A(0));
        }
        return;
    }
    // partials: acc [rows][nsplit][H][dh], (max, sum) [rows][nsplit][H][2]
    A *pacc = reinterpret_cast<A *>(a.ws);
    A *pml = pacc + a.rows * (int64_t)nsplit * a.H * a.dh;
    const int64_t slot = (r * nsplit + split) * a.H + h;
#pragma unroll
    for (int i = 0; i < kMaxEpl; ++i) {
        int d = lane + 32 * i;
        if (i < epl && d < a.dh) pacc[slot * a.dh + d] = acc[i];
    }
    if (lane == 0) { pml[slot * 2] = mx; pml[slot * 2 + 1] = z; }
}

// Log-sum-exp merge of the per-split partials of one (row, head).  Warp 0 computes the weights
// exp(m_s - M) / Z of the splits that hold keys (compacted in split order, with warp reductions only),
// then every thread merges one output element across those splits.
template <typename S>
__global__ void __launch_bounds__(512) combine_kernel(AttendArgs a, int nsplit) {
    using A = typename Traits<S>::A;
    extern __shared__ __align__(16) unsigned char comb_smem[];
    A *wgt = reinterpret_cast<A *>(comb_smem);                 // [nsplit]
    int *idx = reinterpret_cast<int *>(wgt + nsplit);          // [nsplit]
    __shared__ int n_live;
    const int64_t r = blockIdx.x;
    const int h = blockIdx.y;
    const A *pacc = reinterpret_cast<const A *>(a.ws);
    const A *pml = pacc + a.rows * (int64_t)nsplit * a.H * a.dh;
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        A M = -INFINITY;
        for (int s = lane; s < nsplit; s += 32) {
            const A m = pml[((r * nsplit + s) * a.H + h) * 2];
            M = m > M ? m : M;
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const A y = __shfl_xor_sync(0xffffffffu, M, o);
            M = y > M ? y : M;
        }
        A zl = A(0);
        int live_total = 0;
        for (int s0 = 0; s0 < nsplit; s0 += 32) {
            const int s = s0 + lane;
            A e = A(0);
            if (s < nsplit) {
                const A m = pml[((r * nsplit + s) * a.H + h) * 2];
                e = m == -INFINITY ? A(0) : exp_acc(m - M);
                zl += e * pml[((r * nsplit + s) * a.H + h) * 2 + 1];
            }
            const bool live = e != A(0);   // an empty split's accumulator is never written
            const uint32_t b = __ballot_sync(0xffffffffu, live);
            if (live) {
                const int q = live_total + __popc(b & ((1u << lane) - 1u));
                idx[q] = s;
                wgt[q] = e;
            }
            live_total += __popc(b);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) zl += __shfl_xor_sync(0xffffffffu, zl, o);
        const A zi = zl > A(0) ? A(1) / zl : A(0);
        __syncwarp();
        for (int q = lane; q < live_total; q += 32) wgt[q] *= zi;
        if (lane == 0) n_live = live_total;
    }
    __syncthreads();
    const int nl = n_live;
    S *o = reinterpret_cast<S *>(a.out) + r * (int64_t)a.H * a.dh + (int64_t)h * a.dh;
    const A *base = pacc + ((r * nsplit) * a.H + h) * (int64_t)a.dh;
    const int64_t sstride = (int64_t)a.H * a.dh;
    for (int d = threadIdx.x; d < a.dh; d += blockDim.x) {
        A acc = A(0);
#pragma unroll 16
        for (int i = 0; i < nl; ++i) acc += wgt[i] * base[idx[i] * sstride + d];
        store_val(&o[d], acc);
    }
}

static void launch_combine(const AttendArgs &a, int ns, cudaStream_t st) {
    int threads = 32;
    while (threads < a.dh && threads < 512) threads <<= 1;
    const size_t esz = a.dtype == HCSA_BF16 ? sizeof(float) : sizeof(double);
    const size_t smem = esz * (size_t)ns + sizeof(int) * (size_t)ns;
    if (a.dtype == HCSA_BF16) {
        if (smem > 48 * 1024)
            cudaFuncSetAttribute(combine_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        combine_kernel<__nv_bfloat16><<<dim3((unsigned)a.rows, a.H), threads, smem, st>>>(a, ns);
    } else {
        if (smem > 48 * 1024)
            cudaFuncSetAttribute(combine_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        combine_kernel<float><<<dim3((unsigned)a.rows, a.H), threads, smem, st>>>(a, ns);
    }
}

static int decode_splits(bool dense, int topk, int window, int64_t N) {
    int64_t nk = (dense ? N : topk) + window;
    int64_t s = (nk + kDecodeSplit - 1) / kDecodeSplit;
    return (int)(s < 1 ? 1 : s);
}

size_t attend_ws_bytes(int dtype, bool decode, bool dense, int64_t rows, int H, int dh, int topk, int window,
                       int64_t N) {
    if (!decode) return 0;
    const int ns = decode_splits(dense, topk, window, N);
    if (ns == 1) return 0;
    const size_t esz = dtype == HCSA_BF16 ? sizeof(float) : sizeof(double);
    return esz * (size_t)rows * ns * H * ((size_t)dh + 2);
}

hcsa_status launch_attend(const AttendArgs &a, cudaStream_t st) {
    if (a.rows == 0) return HCSA_OK;
    if (a.lowprec && !attend_tc_supported(a)) return HCSA_ERR_UNSUPPORTED;   // FP8 entries: tensor-core shapes only
    if (!a.lowprec && hca_attend_tc_supported(a)) return launch_hca_attend_tc(a, st);
    if (attend_tc_supported(a)) {
        const int ns = attend_tc_segments(a);
        if (ns > 1 &&
            a.ws_bytes < attend_ws_bytes(a.dtype, true, a.dense, a.rows, a.H, a.dh, a.topk, a.window, a.N))
            return HCSA_ERR_WORKSPACE;
        hcsa_status s = launch_attend_tc(a, st);
        if (s != HCSA_OK || ns == 1) return s;
        launch_combine(a, ns, st);
        count_launch();
        return check_launch();
    }
    if ((a.dh + 31) / 32 > kMaxEpl) return HCSA_ERR_UNSUPPORTED;
    const int ns = a.pos ? decode_splits(a.dense, a.topk, a.window, a.N) : 1;
    if (ns > 1 && a.ws_bytes < attend_ws_bytes(a.dtype, true, a.dense, a.rows, a.H, a.dh, a.topk, a.window, a.N))
        return HCSA_ERR_WORKSPACE;
    if (ns > 65535) return HCSA_ERR_UNSUPPORTED;
    if (a.row1 <= a.row0) return HCSA_OK;
    dim3 grid((unsigned)(a.row1 - a.row0), (a.H + kHeadsPerCta - 1) / kHeadsPerCta, ns);
    int *status = device_status_ptr();
    if (a.dtype == HCSA_BF16) attend_kernel<__nv_bfloat16><<<grid, kHeadsPerCta * 32, 0, st>>>(a, ns, status);
    else attend_kernel<float><<<grid, kHeadsPerCta * 32, 0, st>>>(a, ns, status);
    if (ns > 1) launch_combine(a, ns, st);
    count_launch(ns > 1 ? 2 : 1);
    return check_launch();
}

}  // namespace hcsa

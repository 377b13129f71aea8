// Learned gated-pool compressor (CSA m=4 over overlapping width-8 pools, HCA
// m'=128 over non-overlapping pools), prefill and decode-append forms.
//
// Follows "DeepSeek-V4 ... KV cache compressed attention", sections "CSA:
// compresion 4x" (learned pool over overlapping windows) and "HCA: compresion
// 128x", with the pool fixed by the CSA workload definition: entry j pools
// tokens [m j - (width - m), m j + m) within [0, T), per channel
//   c_j[c] = sum_i softmax_i(g[i,c] + B[i - m j + width - m, c]) kv[i,c];
// the indexer key of entry j is the same pool over ki with gate channel d.
//
// HBM-bound.  bf16 storage: narrow pools (CSA, width 8) take one thread per
// 16-byte channel vector of one entry, which loads the whole pool first and
// runs a two-pass softmax; wide pools (HCA, 128 tokens) split each pool's
// tokens over 8 warps and merge their partial softmaxes.  Adjacent threads
// read adjacent 16-byte vectors of the same row, so every warp load is
// coalesced.  fp32 storage (computed in fp64) keeps the generic form, a
// single-pass running max per channel.
#include "internal.cuh"
#include "lowprec.cuh"

namespace hcsa {

// Store one 8-channel vector (c0 .. c0 + 7) of entry row `row`: in the storage dtype, or (lp.on) rounded to
// bf16 and then as block-scaled FP8 (entries) / FP4 (indexer keys); the 4 lanes of a 32-channel block call
// this together.
struct LowPrecOut {
    bool on;
    int64_t rows;   // rows of the whole array: the exponents follow rows x ch code bytes
    int jstride;    // entries j0, j0 + jstride, ... (1: a contiguous range)
};

__device__ __forceinline__ void store_row_vec(const float *r, bool is_key, int64_t row, int C, int di, int c0,
                                              __nv_bfloat16 *entries, __nv_bfloat16 *idx_keys, LowPrecOut lp) {
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = __bfloat162float(__float2bfloat16_rn(r[e]));
    if (lp.on) {
        if (is_key) {
            uint8_t *codes = reinterpret_cast<uint8_t *>(idx_keys);
            lp::store_fp4x8(v, codes, reinterpret_cast<int8_t *>(codes + lp.rows * (di / 2)), row, di, c0);
        } else {
            uint8_t *codes = reinterpret_cast<uint8_t *>(entries);
            lp::store_fp8x8(v, codes, reinterpret_cast<int8_t *>(codes + lp.rows * C), row, C, c0);
        }
        return;
    }
    uint4 o;
    __nv_bfloat16 *oe = reinterpret_cast<__nv_bfloat16 *>(&o);
#pragma unroll
    for (int e = 0; e < 8; ++e) oe[e] = __float2bfloat16_rn(v[e]);
    if (is_key) *reinterpret_cast<uint4 *>(idx_keys + row * di + c0) = o;
    else *reinterpret_cast<uint4 *>(entries + row * C + c0) = o;
}


template <typename A, int V>
struct PoolAcc {
    A mx[V], z[V], acc[V];
    __device__ __forceinline__ void init() {
#pragma unroll
        for (int e = 0; e < V; ++e) { mx[e] = -INFINITY; z[e] = A(0); acc[e] = A(0); }
    }
    __device__ __forceinline__ void add(const A *gate, const A *bias, const A *val) {
#pragma unroll
        for (int e = 0; e < V; ++e) {
            A l = gate[e] + bias[e];
            if (l > mx[e]) {
                A sc = exp_acc(mx[e] - l);
                acc[e] = acc[e] * sc + val[e];
                z[e] = z[e] * sc + A(1);
                mx[e] = l;
            } else {
                A p = exp_acc(l - mx[e]);
                acc[e] += p * val[e];
                z[e] += p;
            }
        }
    }
    __device__ __forceinline__ void result(A *out) const {
#pragma unroll
        for (int e = 0; e < V; ++e) out[e] = acc[e] / z[e];
    }
};

template <typename S>
__global__ void __launch_bounds__(256) compress_kernel(int64_t T, int C, int m, int width, const S *__restrict__ kv,
                                                       int64_t ld_kv, const S *__restrict__ g, int64_t ld_g,
                                                       const S *__restrict__ ki, int64_t ld_ki, int di,
                                                       const S *__restrict__ bias, S *__restrict__ entries,
                                                       S *__restrict__ idx_keys, int64_t j0, int64_t N,
                                                       LowPrecOut lp) {
    using A = typename Traits<S>::A;
    constexpr int V = Traits<S>::VEC;
    const int slots_c = C / V;
    const int slots = slots_c + (ki ? di / V : 0);
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= N * slots) return;   // entries j0 .. j0 + N - 1
    const int64_t jl = gid / slots;
    const int s = (int)(gid - jl * slots);
    const int64_t j = j0 + jl * lp.jstride;
    const bool is_key = s >= slots_c;
    const int c0 = (is_key ? s - slots_c : s) * V;   // value channel; also the gate channel
    const S *val = is_key ? ki : kv;
    const int64_t ld_val = is_key ? ld_ki : ld_kv;
    const int64_t lo = (int64_t)m * j - (width - m);
    const int64_t a = lo < 0 ? 0 : lo;
    const int64_t b = (int64_t)m * j + m < T ? (int64_t)m * j + m : T;

    PoolAcc<A, V> pa;
    pa.init();
#pragma unroll 4
    for (int64_t i = a; i < b; ++i) {
        A gv[V], bv[V], vv[V];
        load_vec(g + i * ld_g + c0, gv);
        load_vec(bias + (i - lo) * C + c0, bv);
        load_vec(val + i * ld_val + c0, vv);
        pa.add(gv, bv, vv);
    }
    A r[V];
    pa.result(r);
    if constexpr (V == 8) {   // bf16 storage
        if (lp.on) {
            store_row_vec(r, is_key, j, C, di, c0, reinterpret_cast<__nv_bfloat16 *>(entries),
                          reinterpret_cast<__nv_bfloat16 *>(idx_keys), lp);
            return;
        }
    }
    if (is_key) store_vec(idx_keys + j * di + c0, r);
    else store_vec(entries + j * C + c0, r);
}


// ---------------------------------------------------------------- bf16 prefill, faster forms
__device__ __forceinline__ float ex2_fast(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void unpack8(const uint4 &u, float *f) {
    const __nv_bfloat16 *e = reinterpret_cast<const __nv_bfloat16 *>(&u);
#pragma unroll
    for (int i = 0; i < 8; ++i) f[i] = __bfloat162float(e[i]);
}

constexpr float kLog2e = 1.4426950408889634f;

// Pools of at most WMAX tokens (CSA: width 8): one thread per 16-byte channel vector (8 channels) of one
// entry.  Every row of the pool is loaded first (up to 3 WMAX independent 16-byte loads in flight per
// thread, adjacent threads reading adjacent vectors of a row), then a two-pass softmax in fp32.
template <int WMAX>
__global__ void __launch_bounds__(256) compress_narrow_bf16_kernel(
    int T, int C, int m, int width, const __nv_bfloat16 *__restrict__ kv, int64_t ld_kv,
    const __nv_bfloat16 *__restrict__ g, int64_t ld_g, const __nv_bfloat16 *__restrict__ ki, int64_t ld_ki, int di,
    const __nv_bfloat16 *__restrict__ bias, __nv_bfloat16 *__restrict__ entries, __nv_bfloat16 *__restrict__ idx_keys,
    int j0, int N, LowPrecOut lp) {
    const int slots_c = C >> 3;
    const int slots = slots_c + (ki ? di >> 3 : 0);
    const int gid = blockIdx.x * 256 + threadIdx.x;
    if (gid >= N * slots) return;   // entries j0 .. j0 + N - 1
    const int jl = gid / slots, s = gid - jl * slots;
    const int j = j0 + jl * lp.jstride;
    const bool is_key = s >= slots_c;
    const int c0 = (is_key ? s - slots_c : s) * 8;   // value channel, also the gate channel
    const __nv_bfloat16 *val = is_key ? ki : kv;
    const int64_t ld_val = is_key ? ld_ki : ld_kv;
    const int lo = m * j - (width - m);
    uint4 gr[WMAX], br[WMAX], vr[WMAX];
    uint32_t in = 0;
#pragma unroll
    for (int r = 0; r < WMAX; ++r) {
        const int i = lo + r;
        if (r < width && i >= 0 && i < T) {
            in |= 1u << r;
            gr[r] = __ldg(reinterpret_cast<const uint4 *>(g + (int64_t)i * ld_g + c0));
            br[r] = __ldg(reinterpret_cast<const uint4 *>(bias + (int64_t)r * C + c0));
            vr[r] = __ldg(reinterpret_cast<const uint4 *>(val + (int64_t)i * ld_val + c0));
        }
    }
    float mx[8], z[8], acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) { mx[e] = -INFINITY; z[e] = 0.f; acc[e] = 0.f; }
#pragma unroll
    for (int r = 0; r < WMAX; ++r) {
        if (!(in >> r & 1u)) continue;
        float gv[8], bv[8];
        unpack8(gr[r], gv);
        unpack8(br[r], bv);
#pragma unroll
        for (int e = 0; e < 8; ++e) mx[e] = fmaxf(mx[e], gv[e] + bv[e]);
    }
#pragma unroll
    for (int r = 0; r < WMAX; ++r) {
        if (!(in >> r & 1u)) continue;
        float gv[8], bv[8], vv[8];
        unpack8(gr[r], gv);
        unpack8(br[r], bv);
        unpack8(vr[r], vv);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float p = ex2_fast((gv[e] + bv[e] - mx[e]) * kLog2e);
            z[e] += p;
            acc[e] = fmaf(p, vv[e], acc[e]);
        }
    }
    float r[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) r[e] = acc[e] / z[e];
    store_row_vec(r, is_key, j, C, di, c0, entries, idx_keys, lp);
}

// Wide pools (HCA: 128 tokens): a block of 8 warps per (entry, 32 channel vectors); lane = channel vector,
// warp w takes the pool's tokens w, w + 8, ... with a running (max, sum, weighted sum) per channel, and
// warp 0 merges the eight partial softmaxes.
constexpr int kWideWarps = 8;
__global__ void __launch_bounds__(32 * kWideWarps) compress_wide_bf16_kernel(
    int T, int C, int m, int width, const __nv_bfloat16 *__restrict__ kv, int64_t ld_kv,
    const __nv_bfloat16 *__restrict__ g, int64_t ld_g, const __nv_bfloat16 *__restrict__ ki, int64_t ld_ki, int di,
    const __nv_bfloat16 *__restrict__ bias, __nv_bfloat16 *__restrict__ entries, __nv_bfloat16 *__restrict__ idx_keys,
    int j0, LowPrecOut lp) {
    __shared__ float part[kWideWarps][3][8][32];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int slots_c = C >> 3;
    const int slots = slots_c + (ki ? di >> 3 : 0);
    const int s = blockIdx.x * 32 + lane;
    const int j = j0 + (int)blockIdx.y * lp.jstride;
    const bool active = s < slots;
    const bool is_key = s >= slots_c;
    const int c0 = (is_key ? s - slots_c : s) * 8;
    const __nv_bfloat16 *val = is_key ? ki : kv;
    const int64_t ld_val = is_key ? ld_ki : ld_kv;
    const int lo = m * j - (width - m);
    float mx[8], z[8], acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) { mx[e] = -INFINITY; z[e] = 0.f; acc[e] = 0.f; }
    if (active) {
        for (int r0 = w; r0 < width; r0 += 4 * kWideWarps) {
            uint4 gr[4], br[4], vr[4];
            uint32_t in = 0;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int r = r0 + q * kWideWarps, i = lo + r;
                if (r < width && i >= 0 && i < T) {
                    in |= 1u << q;
                    gr[q] = __ldg(reinterpret_cast<const uint4 *>(g + (int64_t)i * ld_g + c0));
                    br[q] = __ldg(reinterpret_cast<const uint4 *>(bias + (int64_t)r * C + c0));
                    vr[q] = __ldg(reinterpret_cast<const uint4 *>(val + (int64_t)i * ld_val + c0));
                }
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if (!(in >> q & 1u)) continue;
                float gv[8], bv[8], vv[8];
                unpack8(gr[q], gv);
                unpack8(br[q], bv);
                unpack8(vr[q], vv);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float l = gv[e] + bv[e];
                    const float mn = fmaxf(mx[e], l);
                    const float sc = ex2_fast((mx[e] - mn) * kLog2e);   // mx = -inf -> 0
                    const float p = ex2_fast((l - mn) * kLog2e);
                    z[e] = z[e] * sc + p;
                    acc[e] = fmaf(p, vv[e], acc[e] * sc);
                    mx[e] = mn;
                }
            }
        }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) { part[w][0][e][lane] = mx[e]; part[w][1][e][lane] = z[e]; part[w][2][e][lane] = acc[e]; }
    __syncthreads();
    if (w != 0 || !active) return;
    float res[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        float M = -INFINITY;
        for (int q = 0; q < kWideWarps; ++q) M = fmaxf(M, part[q][0][e][lane]);
        float Z = 0.f, Acc = 0.f;
        for (int q = 0; q < kWideWarps; ++q) {
            const float mq = part[q][0][e][lane];
            if (mq == -INFINITY) continue;
            const float sc = ex2_fast((mq - M) * kLog2e);
            Z = fmaf(part[q][1][e][lane], sc, Z);
            Acc = fmaf(part[q][2][e][lane], sc, Acc);
        }
        res[e] = Acc / Z;
    }
    store_row_vec(res, is_key, j, C, di, c0, entries, idx_keys, lp);
}

hcsa_status launch_compress(int dtype, int64_t T, int C, int m, int width, const void *kv, int64_t ld_kv,
                            const void *g, int64_t ld_g, const void *ki, int64_t ld_ki, int di, const void *bias,
                            void *entries, void *idx_keys, int64_t j0, int64_t j1, bool lowprec, int64_t rows,
                            cudaStream_t st, int jstride) {
    const int64_t N = (j1 - j0 + jstride - 1) / jstride;   // entries j0, j0 + jstride, ... below j1
    if (N <= 0) return HCSA_OK;
    const LowPrecOut lp{lowprec, rows, jstride};
    const int threads = 256;
    if (dtype == HCSA_BF16) {
        using S = __nv_bfloat16;
        const int64_t slots = C / 8 + (ki ? di / 8 : 0);
        if (width <= 8 && j1 * slots <= INT32_MAX && T <= INT32_MAX) {
            const int64_t blocks = (N * slots + threads - 1) / threads;
            compress_narrow_bf16_kernel<8><<<(unsigned)blocks, threads, 0, st>>>(
                (int)T, C, m, width, (const S *)kv, ld_kv, (const S *)g, ld_g, (const S *)ki, ld_ki, di,
                (const S *)bias, (S *)entries, (S *)idx_keys, (int)j0, (int)N, lp);
        } else if (N <= 65535 && T <= INT32_MAX && (int64_t)m * j1 <= INT32_MAX) {
            dim3 grid((unsigned)((slots + 31) / 32), (unsigned)N);
            compress_wide_bf16_kernel<<<grid, 32 * kWideWarps, 0, st>>>(
                (int)T, C, m, width, (const S *)kv, ld_kv, (const S *)g, ld_g, (const S *)ki, ld_ki, di,
                (const S *)bias, (S *)entries, (S *)idx_keys, (int)j0, lp);
        } else {
            const int64_t blocks = (N * slots + threads - 1) / threads;
            compress_kernel<S><<<(unsigned)blocks, threads, 0, st>>>(
                T, C, m, width, (const S *)kv, ld_kv, (const S *)g, ld_g, (const S *)ki, ld_ki, di, (const S *)bias,
                (S *)entries, (S *)idx_keys, j0, N, lp);
        }
    } else {
        const int64_t slots = C / 4 + (ki ? di / 4 : 0);
        const int64_t blocks = (N * slots + threads - 1) / threads;
        compress_kernel<float><<<(unsigned)blocks, threads, 0, st>>>(
            T, C, m, width, (const float *)kv, ld_kv, (const float *)g, ld_g, (const float *)ki, ld_ki, di,
            (const float *)bias, (float *)entries, (float *)idx_keys, j0, N, LowPrecOut{false, 0, jstride});
    }
    count_launch();
    return check_launch();
}

// ---------------------------------------------------------------- bf16 rows -> FP8 / FP4 storage
// One thread per 8-channel vector of a row (the 4 lanes of a 32-channel block are adjacent threads).
__global__ void __launch_bounds__(256) quantize_rows_kernel(const __nv_bfloat16 *__restrict__ src, int64_t rows,
                                                            int ch, bool keys, uint8_t *dst) {
    const int vpr = ch / 8;
    const int64_t gid = (int64_t)blockIdx.x * 256 + threadIdx.x;
    if (gid >= rows * vpr) return;   // rows x vpr is a multiple of 4: blocks are whole
    const int64_t r = gid / vpr;
    const int c0 = (int)(gid - r * vpr) * 8;
    const uint4 u = *reinterpret_cast<const uint4 *>(src + r * ch + c0);
    const __nv_bfloat16 *e = reinterpret_cast<const __nv_bfloat16 *>(&u);
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __bfloat162float(e[i]);
    if (keys) lp::store_fp4x8(v, dst, reinterpret_cast<int8_t *>(dst + rows * (ch / 2)), r, ch, c0);
    else lp::store_fp8x8(v, dst, reinterpret_cast<int8_t *>(dst + rows * ch), r, ch, c0);
}

hcsa_status launch_quantize_rows(const void *src, int64_t rows, int ch, bool keys, void *dst, cudaStream_t st) {
    if (rows <= 0) return HCSA_OK;
    const int64_t n = rows * (ch / 8);
    quantize_rows_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>((const __nv_bfloat16 *)src, rows, ch, keys,
                                                                        (uint8_t *)dst);
    count_launch();
    return check_launch();
}

// ---------------------------------------------------------------- decode append
// Sequence b's new token P = pos[b] is written into the rings; when P = m j + m - 1
// entry j is formed from tokens [m j - (width - m), P] (earlier tokens from the
// rings, token P straight from the inputs, so no thread waits on another's write).
template <typename S>
__global__ void __launch_bounds__(128) cache_append_kernel(
    int C, int m, int width, int window, int di, int64_t n_cap, const int32_t *__restrict__ pos,
    const S *__restrict__ kv_new, int64_t ld_kv, const S *__restrict__ g_new, int64_t ld_g,
    const S *__restrict__ ki_new, int64_t ld_ki, const S *__restrict__ bias, S *entries, S *idx_keys, S *win_kv,
    S *ring_g, S *ring_ki, int *status, LowPrecOut lp, int64_t ent0, bool shard) {
    using A = typename Traits<S>::A;
    constexpr int V = Traits<S>::VEC;
    const int b = blockIdx.y;
    const int slots_c = C / V;
    const int slots = slots_c + (ki_new ? di / V : 0);
    const int s = blockIdx.x * blockDim.x + threadIdx.x;
    if (s >= slots) return;
    const int64_t P = pos[b];
    if (P < 0) { report(status, kStatusBounds); return; }
    const bool is_key = s >= slots_c;
    const int c0 = (is_key ? s - slots_c : s) * V;
    const S *gnew = g_new + b * ld_g;
    const S *vnew = is_key ? ki_new + b * ld_ki : kv_new + b * ld_kv;
    // 1) ring writes (each thread writes its own 16-byte vector)
    if (is_key) {
        *reinterpret_cast<uint4 *>(ring_ki + ((int64_t)b * width + P % width) * di + c0) =
            *reinterpret_cast<const uint4 *>(vnew + c0);
    } else {
        *reinterpret_cast<uint4 *>(win_kv + ((int64_t)b * window + P % window) * C + c0) =
            *reinterpret_cast<const uint4 *>(vnew + c0);
        *reinterpret_cast<uint4 *>(ring_g + ((int64_t)b * width + P % width) * C + c0) =
            *reinterpret_cast<const uint4 *>(gnew + c0);
    }
    // 2) entry completion
    if ((P + 1) % m != 0) return;
    const int64_t jg = (P + 1) / m - 1;   // the entry the token closes
    if (shard && (jg < ent0 || jg >= ent0 + n_cap)) return;   // held by another shard
    const int64_t j = jg - ent0;
    if (j >= n_cap) { report(status, kStatusBounds); return; }
    const int64_t lo = (int64_t)m * jg - (width - m);
    PoolAcc<A, V> pa;
    pa.init();
    for (int64_t i = lo < 0 ? 0 : lo; i <= P; ++i) {
        A gv[V], bv[V], vv[V];
        const S *grow = (i == P) ? gnew : ring_g + ((int64_t)b * width + i % width) * C;
        const S *vrow = (i == P) ? vnew
                        : is_key ? ring_ki + ((int64_t)b * width + i % width) * di
                                 : win_kv + ((int64_t)b * window + i % window) * C;
        load_vec(grow + c0, gv);
        load_vec(bias + (i - lo) * C + c0, bv);
        load_vec(vrow + c0, vv);
        pa.add(gv, bv, vv);
    }
    A r[V];
    pa.result(r);
    if constexpr (V == 8) {   // bf16 storage
        if (lp.on) {
            store_row_vec(r, is_key, (int64_t)b * n_cap + j, C, di, c0, reinterpret_cast<__nv_bfloat16 *>(entries),
                          reinterpret_cast<__nv_bfloat16 *>(idx_keys), lp);
            return;
        }
    }
    if (is_key) store_vec(idx_keys + ((int64_t)b * n_cap + j) * di + c0, r);
    else store_vec(entries + ((int64_t)b * n_cap + j) * C + c0, r);
}

hcsa_status launch_cache_append(int dtype, const hcsa_params &p, const hcsa_cache &c, const int32_t *pos,
                                const void *kv, int64_t ld_kv, const void *g, int64_t ld_g, const void *ki,
                                int64_t ld_ki, const void *bias, cudaStream_t st) {
    const int V = dtype == HCSA_BF16 ? 8 : 4;
    const int slots = p.C / V + (ki ? p.di / V : 0);
    dim3 grid((slots + 127) / 128, p.B);
    int *status = device_status_ptr();
    if (dtype == HCSA_BF16) {
        using S = __nv_bfloat16;
        cache_append_kernel<S><<<grid, 128, 0, st>>>(
            p.C, p.m, p.width, p.window, p.di, p.n_cap, pos, (const S *)kv, ld_kv, (const S *)g, ld_g,
            (const S *)ki, ld_ki, (const S *)bias, (S *)c.entries, (S *)c.idx_keys, (S *)c.win_kv, (S *)c.ring_g,
            (S *)c.ring_ki, status, LowPrecOut{p.lowprec != 0, (int64_t)p.B * p.n_cap, 1}, (int64_t)p.ent0,
            p.ent_shard != 0);
    } else {
        using S = float;
        cache_append_kernel<S><<<grid, 128, 0, st>>>(
            p.C, p.m, p.width, p.window, p.di, p.n_cap, pos, (const S *)kv, ld_kv, (const S *)g, ld_g,
            (const S *)ki, ld_ki, (const S *)bias, (S *)c.entries, (S *)c.idx_keys, (S *)c.win_kv, (S *)c.ring_g,
            (S *)c.ring_ki, status, LowPrecOut{false, 0, 1}, (int64_t)p.ent0, p.ent_shard != 0);
    }
    count_launch();
    return check_launch();
}

}  // namespace hcsa

// CSA prefill attention on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// Operation ("DeepSeek-V4 ... KV cache compressed attention", sections "CSA" and
// "Ventana deslizante", fixed by the CSA workload definition): for query token t,
// the keys are the selected compressed entries plus the raw tokens (t - 128, t];
// key = first C/2 channels of a row, value = last C/2; every one of the H heads
// shares those keys (MQA); one softmax over the union with scale tau.
//
// Shape handled here: H = 64 heads, dh = C/2 = 512, at most 640 keys (top-k 512 +
// window 128), bf16 storage.  One CTA (4 warps) per query token.
//
// Layout choice: the MQA sharing makes the 64 heads the natural N of the MMA and
// the keys its M, so S^T[key, head] = K . Q^T lands in TMEM with one key per lane
// (5 tiles x 64 columns).  The softmax is exact and two-pass over all <= 640 keys
// (per-head max across lanes via a warp transpose-reduction), which avoids any
// rescaling of the output accumulator.  P^T is written to shared memory as a bf16
// MN-major operand and O^T[dh, head] = V^T . P^T accumulates in the TMEM columns
// the scores used (4 x 64 columns).  Gathered key / value rows stream through a
// 6-stage ring of 16 KB chunks [128 rows x 64 bf16] in the 128-byte swizzled
// layout, filled with 16-byte cp.async (8 threads per 128-byte row segment, so
// every warp request covers whole L2 sectors); the MMA of chunk c overlaps the
// loads of chunks c+1 .. c+4.
#include "tc_common.cuh"

namespace hcsa {

namespace {

constexpr int kH = 64;          // heads (MMA N)
constexpr int kDh = 512;        // head dim = C / 2
constexpr int kRowElems = 1024; // C
constexpr int kKT = 128;        // keys per tile (MMA M)
constexpr int kMaxTiles = 5;    // <= 640 keys
constexpr int kNS = 6;          // ring stages (even: V chunk pairs sit in adjacent stages)
constexpr int kStage = 16384;   // [128 rows x 128 bytes]
constexpr int kUBytes = kMaxTiles * kKT * 128;   // P^T: 640 rows x 64 heads bf16 (Q needs 64 KB of it)
constexpr int kThreads = 128;
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kIdescS = tc::idesc_bf16(128, kH, false, false);   // S^T = K . Q^T
constexpr uint32_t kIdescPV = tc::idesc_bf16(128, kH, true, true);    // O^T = V^T . P^T

struct Smem {
    uint8_t *U, *ring;
    const __nv_bfloat16 **rowptr;
    float *red, *mx, *zinv;
    uint64_t *empty, *s_done, *o_done;
    uint32_t *tmem_slot;
    int *abort_flag;
};

__device__ __forceinline__ Smem carve(uint8_t *raw) {
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    Smem s;
    s.U = base;
    s.ring = base + kUBytes;
    uint8_t *p = s.ring + kNS * kStage;
    s.rowptr = reinterpret_cast<const __nv_bfloat16 **>(p);
    p += sizeof(void *) * kMaxTiles * kKT;
    s.red = reinterpret_cast<float *>(p);
    p += sizeof(float) * 4 * kH;
    s.mx = reinterpret_cast<float *>(p);
    p += sizeof(float) * kH;
    s.zinv = reinterpret_cast<float *>(p);
    p += sizeof(float) * kH;
    s.empty = reinterpret_cast<uint64_t *>(p);
    s.s_done = s.empty + kNS;
    s.o_done = s.s_done + 1;
    p += sizeof(uint64_t) * (kNS + 2);
    s.tmem_slot = reinterpret_cast<uint32_t *>(p);
    s.abort_flag = reinterpret_cast<int *>(p + 4);
    return s;
}

constexpr size_t kSmemBytes = 1024 + kUBytes + kNS * kStage + sizeof(void *) * kMaxTiles * kKT +
                              sizeof(float) * 6 * kH + sizeof(uint64_t) * (kNS + 2) + 16;

// Per head, reduce 64 values across the 32 lanes of a warp (max or sum).  On return lane l holds
// the warp-wide results for heads 2l and 2l+1 in v[0], v[1].
template <bool kMax>
__device__ __forceinline__ void warp_transpose_reduce(float *v, int lane) {
#pragma unroll
    for (int o = 16, n = 32; o >= 1; o >>= 1, n >>= 1) {
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < n; ++i) {
            float send = upper ? v[i] : v[i + n];
            float keep = upper ? v[i + n] : v[i];
            float recv = __shfl_xor_sync(0xffffffffu, send, o);
            v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
        }
    }
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__global__ void __launch_bounds__(kThreads, 1)
csa_attend_tc_kernel(const __nv_bfloat16 *__restrict__ q, int64_t ld_q, const __nv_bfloat16 *__restrict__ kv,
                     int64_t ld_kv, const __nv_bfloat16 *__restrict__ entries, const int32_t *__restrict__ sel,
                     int topk, int window, int64_t N, float scale_log2, __nv_bfloat16 *__restrict__ out,
                     int *status) {
    extern __shared__ uint8_t smem_raw[];
    Smem sm = carve(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t t = blockIdx.x;
    const int nk = topk + window;
    const int ntiles = (nk + kKT - 1) / kKT;
    const int nS = ntiles * 8, total = 2 * nS;

    // ---- key row pointers (nullptr = masked key: zero-filled, probability 0)
    for (int kk = tid; kk < ntiles * kKT; kk += kThreads) {
        const __nv_bfloat16 *ptr = nullptr;
        if (kk < topk) {
            const int32_t j = sel[t * topk + kk];
            if (j >= 0 && j < N) ptr = entries + (int64_t)j * kRowElems;
        } else if (kk < nk) {
            const int64_t pp = t - window + 1 + (kk - topk);
            if (pp >= 0) ptr = kv + pp * ld_kv;
        }
        sm.rowptr[kk] = ptr;
    }
    if (tid == 0) {
        for (int s = 0; s < kNS; ++s) tc::mbar_init(&sm.empty[s], 1);
        tc::mbar_init(sm.s_done, 1);
        tc::mbar_init(sm.o_done, 1);
        *sm.abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 0) tc::tmem_alloc(sm.tmem_slot, kTmemCols);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *sm.tmem_slot;
    const uint32_t U = tc::smem_u32(sm.U), ring = tc::smem_u32(sm.ring);

    // ---- loaders
    auto load_q = [&]() {
        const __nv_bfloat16 *qrow = q + t * ld_q;
        for (int idx = tid; idx < kH * 64; idx += kThreads) {
            const int h = idx >> 6, dc = (idx >> 3) & 7, g = idx & 7;
            tc::cp_async16(U + dc * 8192 + tc::sw128_offset(h, g), qrow + h * kDh + dc * 64 + g * 8, true);
        }
    };
    auto load_chunk = [&](int c) {
        int kt, col;
        if (c < nS) {
            kt = c >> 3;
            col = (c & 7) * 64;
        } else {
            const int v = c - nS, u = v >> 1;
            kt = u >> 2;
            col = kDh + (u & 3) * 128 + (v & 1) * 64;
        }
        const uint32_t st = ring + (c % kNS) * kStage;
        const int g = tid & 7;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int row = i * 16 + (tid >> 3);
            const __nv_bfloat16 *p = sm.rowptr[kt * kKT + row];
            tc::cp_async16(st + tc::sw128_offset(row, g), p ? p + col + g * 8 : entries, p != nullptr);
        }
    };

    load_q();
    load_chunk(0);
    tc::cp_async_commit();
    for (int c = 1; c <= kNS - 3; ++c) {
        if (c < total) load_chunk(c);
        tc::cp_async_commit();
    }

    for (int c = 0; c < total; ++c) {
        const int cn = c + kNS - 2;
        if (cn < total) {
            if (cn >= kNS && !tc::mbar_wait(&sm.empty[cn % kNS], ((cn - kNS) / kNS) & 1, status)) *sm.abort_flag = 1;
            load_chunk(cn);
        }
        tc::cp_async_commit();
        tc::cp_async_wait<kNS - 2>();

        if (c == nS) {
            // ---- softmax over all keys: S^T tiles in TMEM -> P^T (bf16) in shared memory
            if (!tc::mbar_wait(sm.s_done, 0, status)) *sm.abort_flag = 1;
            tc::tc_fence_after();
            const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
            float m[kH];
#pragma unroll
            for (int h = 0; h < kH; ++h) m[h] = -INFINITY;
            for (int kt = 0; kt < ntiles; ++kt) {
                float s[kH];
                tc::tmem_ld32(tl + kt * kH, s);
                tc::tmem_ld32(tl + kt * kH + 32, s + 32);
                tc::tmem_ld_wait();
                if (sm.rowptr[kt * kKT + tid]) {
#pragma unroll
                    for (int h = 0; h < kH; ++h) m[h] = fmaxf(m[h], s[h]);
                }
            }
            warp_transpose_reduce<true>(m, lane);
            sm.red[warp * kH + 2 * lane] = m[0];
            sm.red[warp * kH + 2 * lane + 1] = m[1];
            __syncthreads();
            if (tid < kH) {
                float mm = fmaxf(fmaxf(sm.red[tid], sm.red[kH + tid]), fmaxf(sm.red[2 * kH + tid], sm.red[3 * kH + tid]));
                sm.mx[tid] = mm * scale_log2;
            }
            __syncthreads();
            float z[kH];
#pragma unroll
            for (int h = 0; h < kH; ++h) z[h] = 0.f;
            for (int kt = 0; kt < ntiles; ++kt) {
                float s[kH];
                tc::tmem_ld32(tl + kt * kH, s);
                tc::tmem_ld32(tl + kt * kH + 32, s + 32);
                tc::tmem_ld_wait();
                const bool valid = sm.rowptr[kt * kKT + tid] != nullptr;
                const int R = kt * kKT + tid;
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int h0 = g * 8 + 2 * e;
                        float p0 = valid ? ex2(fmaf(s[h0], scale_log2, -sm.mx[h0])) : 0.f;
                        float p1 = valid ? ex2(fmaf(s[h0 + 1], scale_log2, -sm.mx[h0 + 1])) : 0.f;
                        z[h0] += p0;
                        z[h0 + 1] += p1;
                        __nv_bfloat162 pr = __floats2bfloat162_rn(p0, p1);
                        w[e] = *reinterpret_cast<uint32_t *>(&pr);
                    }
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(U + tc::sw128_offset(R, g)),
                                 "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3])
                                 : "memory");
                }
            }
            warp_transpose_reduce<false>(z, lane);
            __syncthreads();   // everyone is done reading red[] (max pass)
            sm.red[warp * kH + 2 * lane] = z[0];
            sm.red[warp * kH + 2 * lane + 1] = z[1];
            __syncthreads();
            if (tid < kH) sm.zinv[tid] = 1.f / (sm.red[tid] + sm.red[kH + tid] + sm.red[2 * kH + tid] + sm.red[3 * kH + tid]);
            tc::tc_fence_before();
        }
        tc::fence_async_smem();
        __syncthreads();
        if (*sm.abort_flag) break;

        if (tid == 0) {
            tc::tc_fence_after();
            if (c < nS) {
                const int kt = c >> 3, dc = c & 7;
                const uint32_t a = ring + (c % kNS) * kStage, b = U + dc * 8192;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    tc::mma_bf16(tmem + kt * kH, tc::sdesc_sw128(a + 32 * k, 16, 1024),
                                 tc::sdesc_sw128(b + 32 * k, 16, 1024), kIdescS, (dc | k) != 0);
                tc::mma_commit(&sm.empty[c % kNS]);
                if (c == nS - 1) tc::mma_commit(sm.s_done);
            } else if ((c - nS) & 1) {
                const int u = (c - nS) >> 1, kt = u >> 2, dp = u & 3;
                const uint32_t a = ring + ((c - 1) % kNS) * kStage, b = U + kt * kKT * 128;
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    tc::mma_bf16(tmem + dp * kH, tc::sdesc_sw128(a + 2048 * k, kStage, 1024),
                                 tc::sdesc_sw128(b + 2048 * k, kStage, 1024), kIdescPV, (kt | k) != 0);
                tc::mma_commit(&sm.empty[(c - 1) % kNS]);
                tc::mma_commit(&sm.empty[c % kNS]);
            }
            if (c == total - 1) tc::mma_commit(sm.o_done);
        }
    }
    tc::cp_async_wait<0>();

    // ---- epilogue: O^T[dh, head] / Z[head] -> out[t, head, dh]
    if (!*sm.abort_flag) {
        if (tc::mbar_wait(sm.o_done, 0, status)) {
            tc::tc_fence_after();
            const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
            __nv_bfloat16 *orow = out + t * (int64_t)kH * kDh;
            for (int dp = 0; dp < 4; ++dp) {
                float o[kH];
                tc::tmem_ld32(tl + dp * kH, o);
                tc::tmem_ld32(tl + dp * kH + 32, o + 32);
                tc::tmem_ld_wait();
#pragma unroll
                for (int h = 0; h < kH; ++h) orow[h * kDh + dp * 128 + tid] = __float2bfloat16_rn(o[h] * sm.zinv[h]);
            }
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_free(tmem, kTmemCols);
    }
}

}  // namespace

bool csa_attend_tc_supported(const AttendArgs &a) {
    return a.dtype == HCSA_BF16 && a.pos == nullptr && !a.dense && a.H == kH && a.dh == kDh && a.C == kRowElems &&
           a.topk >= 1 && a.topk + a.window <= kMaxTiles * kKT;
}

hcsa_status launch_csa_attend_tc(const AttendArgs &a, cudaStream_t st) {
    static bool configured = false;
    if (!configured) {
        if (cudaFuncSetAttribute(csa_attend_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kSmemBytes) != cudaSuccess)
            return HCSA_ERR_CUDA;
        configured = true;
    }
    const float scale_log2 = a.scale * 1.4426950408889634f;
    csa_attend_tc_kernel<<<(unsigned)a.rows, kThreads, kSmemBytes, st>>>(
        (const __nv_bfloat16 *)a.q, a.ld_q, (const __nv_bfloat16 *)a.kv, a.ld_kv,
        (const __nv_bfloat16 *)a.entries, a.sel, a.topk, a.window, a.N, scale_log2, (__nv_bfloat16 *)a.out,
        device_status_ptr());
    count_launch();
    return check_launch();
}

}  // namespace hcsa

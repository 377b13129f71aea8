// HCA prefill attention on the tensor cores (tcgen05 + TMEM, TMA box loads), dh = 128 (C = 256), bf16.
//
// Operation ("DeepSeek-V4 ... KV cache compressed attention", section "HCA: compresion 128x mas
// atencion densa" and "Ventana deslizante", fixed by the HCA workload definition): query token t,
// every head sharing the keys (MQA), attends to every visible entry (128 j + 128 <= t) and to the raw
// tokens (t - 128, t]; key = first 128 channels of a row, value = last 128; one softmax, scale tau.
//
// HCA entries are visible to whole runs of consecutive tokens, so the kernel is flash-style over
// query blocks: 128 / H consecutive tokens x H heads = 128 query rows (the MMA's M, one row per TMEM
// lane).  Key tiles of 128 rows (entries 0 .. visible, then the raw rows t0 - 127 .. t0 + TB) are
// loaded by TMA boxes; per-row masks select what each token may see.
//   S = Q K^T          [128 rows x 128 keys] fp32 in TMEM, two buffers
//   online softmax     one thread per row; the running reference max is raised only when a row's
//                      max grows by more than 2^8 in exp2 units, and only then is that row's O rescaled
//   O += P V           P (bf16) in shared memory as the A operand, V as an MN-major B operand
// Warp roles: warp 0 TMA producer, warp 1 MMA issuer, warps 2..5 softmax + output epilogue.
#include "tc_common.cuh"

namespace hcsa {

namespace {

constexpr int kDh = 128;
constexpr int kC = 256;
constexpr int kKT = 128;          // keys per tile
constexpr int kRows = 128;        // query rows per block
constexpr int kNS = 2;            // K/V stages
constexpr int kChunk = 16384;     // 128 rows x 64 bf16
constexpr int kStage = 4 * kChunk;   // K (2 chunks) + V (2 chunks)
constexpr int kThreads = 192;
constexpr uint32_t kColO = 256;   // S buffers at columns 0 and 128, O at 256
constexpr float kRescaleLog2 = 8.f;

constexpr uint32_t kIdescS = tc::idesc_bf16(128, 128, false, false);
constexpr uint32_t kIdescPV = tc::idesc_bf16(128, 128, false, true);

struct Params {
    int64_t T, N;
    int H, m, tb;            // heads, compression ratio, tokens per block (128 / H)
    float scale_log2;
    __nv_bfloat16 *out;
    int *status;
};

struct Bars {
    uint64_t kv_full[kNS], kv_empty[kNS], s_full[2], s_free[2], p_full, o_done, q_full;
};

__device__ __forceinline__ int64_t vis_of(const Params &a, int64_t t) {
    const int64_t v = t / a.m;
    return v < a.N ? v : a.N;
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__global__ void __launch_bounds__(kThreads, 1)
hca_attend_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_ent,
                     const __grid_constant__ CUtensorMap tm_raw, Params a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = base;                       // 2 chunks
    uint8_t *sKV = sQ + 2 * kChunk;           // kNS stages
    uint8_t *sP = sKV + kNS * kStage;         // 2 chunks
    Bars *bars = reinterpret_cast<Bars *>(sP + 2 * kChunk);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t0 = (int64_t)blockIdx.x * a.tb;
    const int64_t t_last = t0 + a.tb - 1 < a.T ? t0 + a.tb - 1 : a.T - 1;
    const int n_ent_tiles = (int)((vis_of(a, t_last) + kKT - 1) / kKT);
    const int n_tiles = n_ent_tiles + 2;      // + raw rows t0 - 127 .. t0 + 128
    if (threadIdx.x == 0) {
        for (int i = 0; i < kNS; ++i) { tc::mbar_init(&bars->kv_full[i], 1); tc::mbar_init(&bars->kv_empty[i], 1); }
        for (int i = 0; i < 2; ++i) { tc::mbar_init(&bars->s_full[i], 1); tc::mbar_init(&bars->s_free[i], 4); }
        tc::mbar_init(&bars->p_full, 4);
        tc::mbar_init(&bars->o_done, 1);
        tc::mbar_init(&bars->q_full, 1);
        tc::fence_mbar_init();
    }
    if (warp == 0) tc::tmem_alloc(tmem_slot, 512);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t Qs = tc::smem_u32(sQ), KV = tc::smem_u32(sKV), Ps = tc::smem_u32(sP);
    bool ok = true;

    if (warp == 0) {
        if (lane == 0) {
            tc::mbar_arrive_expect_tx(&bars->q_full, 2 * kChunk);
            for (int dc = 0; dc < 2; ++dc)
                tc::tma_load_3d(Qs + dc * kChunk, &tm_q, dc * 64, 0, (int)t0, &bars->q_full);
            for (int i = 0; i < n_tiles && ok; ++i) {
                const int s = i % kNS;
                if (i >= kNS) ok = ok && tc::mbar_wait(&bars->kv_empty[s], ((i / kNS) - 1) & 1, a.status);
                tc::mbar_arrive_expect_tx(&bars->kv_full[s], kStage);
                const bool ent = i < n_ent_tiles;
                const int row0 = ent ? i * kKT : (int)(t0 - (kKT - 1) + (int64_t)(i - n_ent_tiles) * kKT);
                for (int c = 0; c < 4; ++c)
                    tc::tma_load_2d(KV + s * kStage + c * kChunk, ent ? &tm_ent : &tm_raw, c * 64, row0,
                                    &bars->kv_full[s]);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            ok = ok && tc::mbar_wait(&bars->q_full, 0, a.status);
            auto issue_pv = [&](int i) {
                const int s = i % kNS;
                ok = ok && tc::mbar_wait(&bars->p_full, i & 1, a.status);
                tc::fence_async_smem();
                tc::tc_fence_after();
                const uint32_t v = KV + s * kStage + 2 * kChunk;
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    tc::mma_bf16(tmem + kColO, tc::sdesc_sw128(Ps + (k >> 2) * kChunk + 32 * (k & 3), 16, 1024),
                                 tc::sdesc_sw128(v + 2048 * k, kChunk, 1024), kIdescPV, (i | k) != 0);
                tc::mma_commit(&bars->kv_empty[s]);
                tc::mma_commit(&bars->o_done);
            };
            for (int i = 0; i < n_tiles && ok; ++i) {
                const int s = i % kNS, sb = i & 1;
                ok = ok && tc::mbar_wait(&bars->kv_full[s], (i / kNS) & 1, a.status);
                if (i >= 2) ok = ok && tc::mbar_wait(&bars->s_free[sb], ((i >> 1) - 1) & 1, a.status);
                tc::tc_fence_after();
                const uint32_t k0 = KV + s * kStage;
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    tc::mma_bf16(tmem + sb * 128, tc::sdesc_sw128(Qs + (k >> 2) * kChunk + 32 * (k & 3), 16, 1024),
                                 tc::sdesc_sw128(k0 + (k >> 2) * kChunk + 32 * (k & 3), 16, 1024), kIdescS, k != 0);
                tc::mma_commit(&bars->s_full[sb]);
                if (i >= 1) issue_pv(i - 1);
            }
            if (ok) issue_pv(n_tiles - 1);
        }
    } else {
        // ---------------------------------------------------------- softmax + epilogue (4 warps, one row each)
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        const int tl = r / a.H, h = r % a.H;
        const int64_t t = t0 + tl;
        const bool row_ok = t < a.T;
        const int64_t vis = row_ok ? vis_of(a, t) : 0;
        const uint32_t tl_addr = tmem + ((uint32_t)(quad * 32) << 16);
        float m_used = -INFINITY, l = 0.f;
        for (int i = 0; i < n_tiles && ok; ++i) {
            const int sb = i & 1;
            ok = ok && tc::mbar_wait(&bars->s_full[sb], (i >> 1) & 1, a.status);
            tc::tc_fence_after();
            float sv[kKT];
#pragma unroll
            for (int c = 0; c < 4; ++c) tc::tmem_ld32(tl_addr + sb * 128 + c * 32, sv + c * 32);
            tc::tmem_ld_wait();
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bars->s_free[sb]);
            // mask: which keys of this tile the row's token may see
            const bool ent = i < n_ent_tiles;
            const int64_t key0 = ent ? (int64_t)i * kKT : t0 - (kKT - 1) + (int64_t)(i - n_ent_tiles) * kKT;
            float mt = -INFINITY;
#pragma unroll
            for (int c = 0; c < kKT; ++c) {
                const int64_t key = key0 + c;
                const bool v = row_ok && (ent ? key < vis : (key >= 0 && key <= t && key > t - kKT));
                sv[c] = v ? sv[c] * a.scale_log2 : -INFINITY;
                mt = fmaxf(mt, sv[c]);
            }
            // lazy rescale of the reference max (exp2 units)
            const bool need = mt > m_used + kRescaleLog2;
            const float m_new = need ? mt : m_used;
            const float factor = need ? ex2(m_used - m_new) : 1.f;   // m_used = -inf -> 0
            if (i >= 1) {
                // P of the previous tile must have been consumed (and O updated) before P and O change
                ok = ok && tc::mbar_wait(&bars->o_done, (i - 1) & 1, a.status);
                tc::tc_fence_after();
                if (__any_sync(0xffffffffu, need)) {
                    for (int c = 0; c < 4; ++c) {
                        float o[32];
                        tc::tmem_ld32(tl_addr + kColO + c * 32, o);
                        tc::tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] *= factor;
                        tc::tmem_st32(tl_addr + kColO + c * 32, o);
                    }
                    tc::tmem_st_wait();
                }
            }
            l *= factor;
            m_used = m_new;
            // P row (bf16) into the K-major A operand: 2 chunks of 64 keys
#pragma unroll
            for (int g = 0; g < 16; ++g) {
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int c = g * 8 + 2 * e;
                    const float p0 = sv[c] == -INFINITY ? 0.f : ex2(sv[c] - m_used);
                    const float p1 = sv[c + 1] == -INFINITY ? 0.f : ex2(sv[c + 1] - m_used);
                    l += p0 + p1;
                    __nv_bfloat162 pr = __floats2bfloat162_rn(p0, p1);
                    w[e] = *reinterpret_cast<uint32_t *>(&pr);
                }
                const uint32_t addr = Ps + (g >> 3) * kChunk + tc::sw128_offset(r, g & 7);
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w[0]), "r"(w[1]), "r"(w[2]),
                             "r"(w[3])
                             : "memory");
            }
            tc::fence_async_smem();
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bars->p_full);
        }
        // output: O / l
        if (ok) ok = ok && tc::mbar_wait(&bars->o_done, (n_tiles - 1) & 1, a.status);
        tc::tc_fence_after();
        const float li = l > 0.f ? 1.f / l : 0.f;
        for (int c = 0; c < 4; ++c) {
            float o[32];
            tc::tmem_ld32(tl_addr + kColO + c * 32, o);
            tc::tmem_ld_wait();
            if (row_ok && ok) {
                uint32_t w[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    __nv_bfloat162 pr = __floats2bfloat162_rn(o[2 * e] * li, o[2 * e + 1] * li);
                    w[e] = *reinterpret_cast<uint32_t *>(&pr);
                }
                uint4 *dst = reinterpret_cast<uint4 *>(a.out + t * (int64_t)a.H * kDh + (int64_t)h * kDh + c * 32);
#pragma unroll
                for (int q = 0; q < 4; ++q) dst[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
            }
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_free(tmem, 512);
    }
}

constexpr size_t kSmemBytes = 1024 + 2 * kChunk + kNS * kStage + 2 * kChunk + sizeof(Bars) + 16;

}  // namespace

bool hca_attend_tc_supported(const AttendArgs &a) {
    if (a.dtype != HCSA_BF16 || a.pos != nullptr || !a.dense) return false;
    if (a.dh != kDh || a.C != kC || a.window != kKT || a.H < 1 || a.H > kRows || kRows % a.H) return false;
    if (a.ld_q % 8 || a.ld_kv % 8 || a.rows > INT32_MAX || a.N > INT32_MAX) return false;
    return true;
}

hcsa_status launch_hca_attend_tc(const AttendArgs &a, cudaStream_t st) {
    static bool configured[64] = {};   // kernel attributes are set per device
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return HCSA_ERR_CUDA;
    if (!configured[dev]) {
        if (cudaFuncSetAttribute(hca_attend_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes) !=
            cudaSuccess)
            return HCSA_ERR_CUDA;
        configured[dev] = true;
    }
    const int tb = kRows / a.H;
    CUtensorMap tq, te, tr;
    // q rows of a block: (token, head) pairs, 128 dims each
    if (!make_tmap_bf16_3d(&tq, a.q, kDh, (uint64_t)a.H, (uint64_t)a.rows, kDh * 2, (uint64_t)a.ld_q * 2, 64,
                           (uint32_t)a.H, (uint32_t)tb, true))
        return HCSA_ERR_CUDA;
    if (!make_tmap_bf16_2d(&te, a.entries, kC, (uint64_t)(a.N > 0 ? a.N : 1), kC * 2, 64, kKT, true))
        return HCSA_ERR_CUDA;
    if (!make_tmap_bf16_2d(&tr, a.kv, kC, (uint64_t)a.rows, (uint64_t)a.ld_kv * 2, 64, kKT, true))
        return HCSA_ERR_CUDA;
    Params p{};
    p.T = a.rows;
    p.N = a.N;
    p.H = a.H;
    p.m = a.m;
    p.tb = tb;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.out = (__nv_bfloat16 *)a.out;
    p.status = device_status_ptr();
    const int64_t blocks = (a.rows + tb - 1) / tb;
    hca_attend_tc_kernel<<<(unsigned)blocks, kThreads, kSmemBytes, st>>>(tq, te, tr, p);
    count_launch();
    return check_launch();
}

}  // namespace hcsa

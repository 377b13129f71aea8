// HCA prefill attention on the tensor cores (tcgen05 + TMEM, TMA box loads), dh = 128 (C = 256), bf16.
//
// Operation ("DeepSeek-V4 ... KV cache compressed attention", section "HCA: compresion 128x mas
// atencion densa" and "Ventana deslizante", fixed by the HCA workload definition): query token t,
// every head sharing the keys (MQA), attends to every visible entry (128 j + 128 <= t) and to the raw
// tokens (t - 128, t]; key = first 128 channels of a row, value = last 128; one softmax, scale tau.
//
// HCA entries are visible to whole runs of consecutive tokens, so the kernel is flash-style over
// query blocks: 128 / H consecutive tokens x H heads = 128 query rows (the MMA's M, one row per TMEM
// lane).  Key tiles of 128 rows (entries 0 .. visible, then the raw rows t0 - 127 .. t0 + 128) are
// loaded by TMA boxes; per-row masks select what each token may see.
//   S = Q K^T          [128 rows x 128 keys] fp32 in TMEM, two buffers
//   online softmax     four threads per row (16 warps, each a TMEM lane quadrant and 32 of the 128 key
//                      columns; the mask is a column range per row; the four exchange their tile max
//                      and final sum through spare TMEM columns of the row's lane); the running max is
//                      raised only when a row's max grows by more than 2^8 in exp2 units, and only then
//                      is that row's O rescaled
//   O += P V           P (bf16) as the A operand, written over the tile's K half in shared memory (the
//                      S MMAs are its only readers and have completed), V as an MN-major B operand;
//                      three K/V stages, so the softmax of tile i overlaps the MMAs of its neighbours
// Persistent CTAs walk the query blocks heaviest first; the next block's Q is loaded as soon as the
// current block's last S MMA has read its Q.  Warp roles: warp 0 TMA producer, warp 1 MMA issuer,
// warps 2..17 softmax + output epilogue.
#include "tc_common.cuh"

namespace hcsa {

namespace {

constexpr int kDh = 128;
constexpr int kC = 256;
constexpr int kKT = 128;             // keys per tile
constexpr int kRows = 128;           // query rows per block
constexpr int kNS = 3;               // K/V stages (the K half of a stage then holds the tile's P)
constexpr int kChunk = 16384;        // 128 rows x 64 bf16
constexpr int kStage = 4 * kChunk;   // K (2 chunks) + V (2 chunks)
constexpr int kSoftWarps = 16;
constexpr int kParts = kSoftWarps / 4;   // threads per query row
constexpr int kPartCols = kKT / kParts;  // key columns (and output dims) per thread
constexpr int kThreads = 64 + 32 * kSoftWarps;
constexpr uint32_t kColO = 256;      // S buffers at columns 0 and 128, O at 256
constexpr uint32_t kColX = 384;      // exchange between the threads of a row: one column per part
constexpr float kRescaleLog2 = 8.f;

constexpr uint32_t kIdescS = tc::idesc_bf16(128, 128, false, false);
constexpr uint32_t kIdescPV = tc::idesc_bf16(128, 128, false, true);

struct Params {
    int64_t T, N;
    int H, m, tb;            // heads, compression ratio, tokens per block (128 / H)
    int64_t n_blocks, b_end;   // blocks of the row range: b_end - n_blocks .. b_end - 1
    float scale_log2;
    __nv_bfloat16 *out;
    int *status;
};

struct Bars {
    uint64_t kv_full[kNS], kv_empty[kNS], s_full[2], s_free[2], p_full[2], o_done[2], q_full, q_empty;
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

struct Block {
    int64_t t0;
    int n_ent_tiles, n_tiles;
};

__device__ __forceinline__ Block block_of(const Params &a, int64_t u) {
    Block b;
    b.t0 = (a.b_end - 1 - u) * a.tb;   // heaviest (latest) blocks of the row range first
    const int64_t t_last = b.t0 + a.tb - 1 < a.T ? b.t0 + a.tb - 1 : a.T - 1;
    b.n_ent_tiles = (int)((vis_of(a, t_last) + kKT - 1) / kKT);
    b.n_tiles = b.n_ent_tiles + 2;   // + raw rows t0 - 127 .. t0 + 128
    return b;
}

__global__ void __launch_bounds__(kThreads, 1)
hca_attend_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_ent,
                     const __grid_constant__ CUtensorMap tm_raw, Params a) {
    extern __shared__ uint8_t smem_raw[];
    // small state first, then the 1024-byte aligned tiles (the alignment gap follows the small state)
    Bars *bars = reinterpret_cast<Bars *>(smem_raw);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 1);
    uint8_t *base =
        reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(tmem_slot + 4) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = base;                       // 2 chunks
    uint8_t *sKV = sQ + 2 * kChunk;           // kNS stages: K (later P) | V

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kNS; ++i) { tc::mbar_init(&bars->kv_full[i], 1); tc::mbar_init(&bars->kv_empty[i], 1); }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&bars->s_full[i], 1);
            tc::mbar_init(&bars->s_free[i], kSoftWarps);
            tc::mbar_init(&bars->p_full[i], kSoftWarps);
            tc::mbar_init(&bars->o_done[i], 1);
        }
        tc::mbar_init(&bars->q_full, 1);
        tc::mbar_init(&bars->q_empty, 1);
        tc::fence_mbar_init();
    }
    if (warp == 0) tc::tmem_alloc(tmem_slot, 512);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t Qs = tc::smem_u32(sQ), KV = tc::smem_u32(sKV);
    bool ok = true;

    if (warp == 0) {
        // ---------------------------------------------------------- TMA producer
        if (lane == 0) {
            uint32_t it = 0, nb = 0;
            for (int64_t u = blockIdx.x; u < a.n_blocks && ok; u += gridDim.x, ++nb) {
                const Block b = block_of(a, u);
                if (nb >= 1) ok = ok && tc::mbar_wait(&bars->q_empty, (nb - 1) & 1, a.status);
                if (!ok) break;
                tc::mbar_arrive_expect_tx(&bars->q_full, 2 * kChunk);
                for (int dc = 0; dc < 2; ++dc)
                    tc::tma_load_3d(Qs + dc * kChunk, &tm_q, dc * 64, 0, (int)b.t0, &bars->q_full);
                for (int i = 0; i < b.n_tiles && ok; ++i, ++it) {
                    const int s = it % kNS;
                    if (it >= kNS) ok = ok && tc::mbar_wait(&bars->kv_empty[s], ((it / kNS) - 1) & 1, a.status);
                    if (!ok) break;
                    tc::mbar_arrive_expect_tx(&bars->kv_full[s], kStage);
                    const bool ent = i < b.n_ent_tiles;
                    const int row0 = ent ? i * kKT : (int)(b.t0 - (kKT - 1) + (int64_t)(i - b.n_ent_tiles) * kKT);
                    for (int c = 0; c < 4; ++c)
                        tc::tma_load_2d(KV + s * kStage + c * kChunk, ent ? &tm_ent : &tm_raw, c * 64, row0,
                                        &bars->kv_full[s]);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            uint32_t it = 0, is = 0, ip = 0, nb = 0;
            // O += P V for the tile that used K/V stage s; first tile of a block overwrites O
            auto issue_pv = [&](int s, bool first) {
                const int pb = ip & 1;
                ok = ok && tc::mbar_wait(&bars->p_full[pb], (ip >> 1) & 1, a.status);
                if (!ok) return;
                tc::tc_fence_after();
                const uint32_t v = KV + s * kStage + 2 * kChunk;
                const uint32_t p = KV + s * kStage;   // P over the K half of the stage
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    tc::mma_bf16(tmem + kColO, tc::sdesc_sw128(p + (k >> 2) * kChunk + 32 * (k & 3), 16, 1024),
                                 tc::sdesc_sw128(v + 2048 * k, kChunk, 1024), kIdescPV, (!first || k != 0) ? 1u : 0u);
                tc::mma_commit(&bars->kv_empty[s]);
                tc::mma_commit(&bars->o_done[pb]);
                ++ip;
            };
            for (int64_t u = blockIdx.x; u < a.n_blocks && ok; u += gridDim.x, ++nb) {
                const Block b = block_of(a, u);
                ok = ok && tc::mbar_wait(&bars->q_full, nb & 1, a.status);
                int prev_s = -1;
                for (int i = 0; i < b.n_tiles && ok; ++i, ++it, ++is) {
                    const int s = it % kNS, sb = is & 1;
                    ok = ok && tc::mbar_wait(&bars->kv_full[s], (it / kNS) & 1, a.status);
                    if (is >= 2) ok = ok && tc::mbar_wait(&bars->s_free[sb], ((is >> 1) - 1) & 1, a.status);
                    if (!ok) break;
                    tc::tc_fence_after();
                    const uint32_t k0 = KV + s * kStage;
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        tc::mma_bf16(tmem + sb * 128, tc::sdesc_sw128(Qs + (k >> 2) * kChunk + 32 * (k & 3), 16, 1024),
                                     tc::sdesc_sw128(k0 + (k >> 2) * kChunk + 32 * (k & 3), 16, 1024), kIdescS,
                                     k != 0 ? 1u : 0u);
                    tc::mma_commit(&bars->s_full[sb]);
                    if (i == b.n_tiles - 1) tc::mma_commit(&bars->q_empty);   // Q free once these S MMAs complete
                    if (prev_s >= 0) issue_pv(prev_s, i == 1);
                    prev_s = s;
                }
                if (ok && prev_s >= 0) issue_pv(prev_s, b.n_tiles == 1);
            }
        }
    } else {
        // ---------------------------------------------------------- softmax + output epilogue (16 warps)
        static_assert(kPartCols == 32, "one 32-column TMEM load per thread and tile");
        const int quad = warp & 3, part = (warp - 2) >> 2;
        const int r = quad * 32 + lane;
        const int tl = r / a.H, h = r % a.H;
        const uint32_t tl_addr = tmem + ((uint32_t)(quad * 32) << 16);
        const int pbar = 2 + quad;   // the four warps of this lane quadrant
        uint32_t is = 0;
        for (int64_t u = blockIdx.x; u < a.n_blocks && ok; u += gridDim.x) {
            const Block b = block_of(a, u);
            const int64_t t = b.t0 + tl;
            const bool row_ok = t < a.T;
            const int64_t vis = row_ok ? vis_of(a, t) : 0;
            float m_used = -INFINITY, l = 0.f;
            for (int i = 0; i < b.n_tiles; ++i, ++is) {
                const int sb = is & 1;
                ok = ok && tc::mbar_wait(&bars->s_full[sb], (is >> 1) & 1, a.status);
                tc::tc_fence_after();
                float sv[32];
                tc::tmem_ld32(tl_addr + sb * 128 + part * 32, sv);
                tc::tmem_ld_wait();
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&bars->s_free[sb]);
                // visible key columns of this thread: [lo, hi) of its 32
                const bool ent = i < b.n_ent_tiles;
                const int64_t kb =
                    (ent ? (int64_t)i * kKT : b.t0 - (kKT - 1) + (int64_t)(i - b.n_ent_tiles) * kKT) + part * 32;
                int64_t lo64 = 0, hi64 = 0;
                if (row_ok) {
                    if (ent) {
                        hi64 = vis - kb;
                    } else {
                        lo64 = (t - (kKT - 1) > 0 ? t - (kKT - 1) : 0) - kb;
                        hi64 = t + 1 - kb;
                    }
                }
                const int lo = (int)(lo64 < 0 ? 0 : lo64 > 32 ? 32 : lo64);
                const int hi = (int)(hi64 < 0 ? 0 : hi64 > 32 ? 32 : hi64);
                float mt = -INFINITY;
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    sv[c] = (c >= lo && c < hi) ? sv[c] * a.scale_log2 : -INFINITY;
                    mt = fmaxf(mt, sv[c]);
                }
                // the row's tile max over its four threads, through TMEM columns kColX .. kColX + 3 of its lane
                tc::tmem_st1(tl_addr + kColX + part, mt);
                tc::tmem_st_wait();
                tc::tc_fence_before();
                ok = tc::named_bar_and(pbar, 128, ok);   // the row's four threads leave together
                if (!ok) break;
                tc::tc_fence_after();
                {
                    float xv[4];
                    tc::tmem_ld4(tl_addr + kColX, xv);
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int q = 0; q < kParts; ++q) mt = fmaxf(mt, xv[q]);
                }
                tc::tc_fence_before();
                tc::named_bar_sync(pbar, 128);           // all have read before the columns are written again
                tc::tc_fence_after();
                // lazy rescale of the reference max (exp2 units)
                const bool need = mt > m_used + kRescaleLog2;
                const float m_new = need ? mt : m_used;
                const float factor = need ? ex2(m_used - m_new) : 1.f;   // m_used = -inf -> 0
                if (i >= 1 && __any_sync(0xffffffffu, need)) {
                    // O must hold the previous tile's P V before it is rescaled (and before P V of this tile)
                    const uint32_t q = is - 1;
                    ok = ok && tc::mbar_wait(&bars->o_done[q & 1], (q >> 1) & 1, a.status);
                    tc::tc_fence_after();
                    float o[32];
                    tc::tmem_ld32(tl_addr + kColO + part * 32, o);
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] *= factor;
                    tc::tmem_st32(tl_addr + kColO + part * 32, o);
                    tc::tmem_st_wait();
                }
                l *= factor;
                m_used = m_new;
                // P (bf16) into the K-major A operand over the K half of this tile's stage (its S MMAs, the only
                // readers of K, have completed): chunk part / 2, granules (part % 2) * 4 .. + 4 of row r
                const uint32_t pbase = KV + (is % kNS) * kStage + (part >> 1) * kChunk;
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int c = g * 8 + 2 * e;
                        const float p0 = ex2(sv[c] - m_used), p1 = ex2(sv[c + 1] - m_used);   // ex2(-inf) = 0
                        l += p0 + p1;
                        __nv_bfloat162 pr = __floats2bfloat162_rn(p0, p1);
                        w[e] = *reinterpret_cast<uint32_t *>(&pr);
                    }
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(pbase +
                                                                              tc::sw128_offset(r, (part & 1) * 4 + g)),
                                 "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3])
                                 : "memory");
                }
                tc::fence_async_smem();
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&bars->p_full[sb]);
            }
            if (!ok) break;
            // output: O / l (the four threads' sums), 32 dims per thread
            const uint32_t q = is - 1;
            ok = ok && tc::mbar_wait(&bars->o_done[q & 1], (q >> 1) & 1, a.status);
            tc::tc_fence_after();
            tc::tmem_st1(tl_addr + kColX + part, l);
            tc::tmem_st_wait();
            tc::tc_fence_before();
            ok = tc::named_bar_and(pbar, 128, ok);
            if (!ok) break;
            tc::tc_fence_after();
            {
                float xv[4];
                tc::tmem_ld4(tl_addr + kColX, xv);
                tc::tmem_ld_wait();
                l = xv[0] + xv[1] + xv[2] + xv[3];
            }
            tc::tc_fence_before();
            tc::named_bar_sync(pbar, 128);
            tc::tc_fence_after();
            const float li = l > 0.f ? 1.f / l : 0.f;
            float o[32];
            tc::tmem_ld32(tl_addr + kColO + part * 32, o);
            tc::tmem_ld_wait();
            if (row_ok) {
                uint32_t w[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    __nv_bfloat162 pr = __floats2bfloat162_rn(o[2 * e] * li, o[2 * e + 1] * li);
                    w[e] = *reinterpret_cast<uint32_t *>(&pr);
                }
                uint4 *dst = reinterpret_cast<uint4 *>(a.out + t * (int64_t)a.H * kDh + (int64_t)h * kDh + part * 32);
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) dst[qq] = make_uint4(w[4 * qq], w[4 * qq + 1], w[4 * qq + 2], w[4 * qq + 3]);
            }
            // the next block's first P V overwrites O only after this block's softmax warps signal its P,
            // which comes after these reads
            tc::tc_fence_before();
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_free(tmem, 512);
    }
}

constexpr size_t kSmemBytes = sizeof(Bars) + 16 + 1023 + 2 * kChunk + kNS * kStage;
static_assert(kSmemBytes <= 232448, "shared memory per CTA");

int sm_count() {
    static int n = 0;
    if (!n) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

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
    // entries end at the last one the range's last query sees: the last entry tile rounds up past it, and
    // those rows read as zeros, so a row-range caller need not have gathered them
    const int64_t last_vis = a.row1 > 0 ? (a.row1 - 1) / a.m : 0;
    const uint64_t ent_rows = (uint64_t)std::max<int64_t>(1, std::min<int64_t>(a.N, last_vis));
    if (!make_tmap_bf16_2d(&te, a.entries, kC, ent_rows, kC * 2, 64, kKT, true)) return HCSA_ERR_CUDA;
    // raw rows end at the row range's end: the second window tile of a range's last block reaches one row
    // past it, which a row-range caller need not have projected (rows past the end read as zeros and are
    // masked like any other key a query may not see)
    if (!make_tmap_bf16_2d(&tr, a.kv, kC, (uint64_t)a.row1, (uint64_t)a.ld_kv * 2, 64, kKT, true))
        return HCSA_ERR_CUDA;
    Params p{};
    p.T = a.rows;
    p.N = a.N;
    p.H = a.H;
    p.m = a.m;
    p.tb = tb;
    p.b_end = (a.row1 + tb - 1) / tb;
    p.n_blocks = p.b_end - a.row0 / tb;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.out = (__nv_bfloat16 *)a.out;
    p.status = device_status_ptr();
    if (p.n_blocks <= 0) return HCSA_OK;
    const int64_t grid = p.n_blocks < sm_count() ? p.n_blocks : sm_count();
    hca_attend_tc_kernel<<<(unsigned)grid, kThreads, kSmemBytes, st>>>(tq, te, tr, p);
    count_launch();
    return check_launch();
}

}  // namespace hcsa

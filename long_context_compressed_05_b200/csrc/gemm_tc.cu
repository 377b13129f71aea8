// Token projections on the tensor cores: y[M, N] = x[M, K] W[K, N] (+ residual), bf16 storage, fp32
// accumulation, one rounding.  This is the "lower-dimensional projection" step of the layer (the kv /
// gate / indexer-key / indexer-query / head-weight / query columns, one GEMM over the concatenated
// weights) and the output projection of residual-chained stacks.
//
// Layout.  W is row-major [K, N] (columns contiguous), x row-major [M, K].  The kernel computes the
// transposed product D[n, t] = sum_k W[k, n] x[t, k]: 128 output columns sit on the MMA's M axis (one
// TMEM lane each) and NTOK tokens on its N axis, so the same kernel streams the weights for a decode
// step (NTOK = 16 or 32 tokens) and tiles a prefill (NTOK = 256).  Both operands come in by TMA in the
// 128-byte swizzle: W as the MN-major A operand (two 64-column boxes of 64 k-rows), x as the K-major B
// operand (NTOK rows of 64 k).  Out-of-range rows / columns / k are zero-filled by TMA and masked at the
// store.
//
// Pipeline.  Warp 0 = TMA producer, warp 1 = MMA issuer (4 MMAs of K = 16 per 64-wide k step into one
// of two TMEM accumulators), the remaining warps = epilogue (TMEM -> registers -> bf16 stores, 64
// contiguous bytes per warp and token); the epilogue of one tile overlaps the MMAs of the next.
// Persistent CTAs walk the tiles in bands of 16 token tiles (every weight tile is read from HBM once
// per band, the band's activations stay in L2).
//
// Split-K.  When the output has too few column tiles to occupy the GPU (a decode step's output
// projection: 2048 columns, K = 32768), the k range is split; every split writes fp32 partials, and the
// CTA that finishes a tile last (an atomic ticket per tile, no waiting) sums them, adds the residual
// and rounds once.
#include "tc_common.cuh"

namespace hcsa {

namespace {

constexpr int kBN = 128;                 // output columns per tile (MMA M)
constexpr int kBoxW = 64 * 128;          // TMA box of W: 64 k-rows x 64 columns, bf16 (8 KB)
constexpr int kBand = 16;                // token tiles per band of the tile order

__host__ __device__ constexpr int stages_for(int ntok) { return ntok >= 256 ? 4 : ntok >= 128 ? 6 : ntok >= 64 ? 4 : 5; }
__host__ __device__ constexpr int ctas_per_sm(int ntok) { return ntok >= 128 ? 1 : 2; }
__host__ __device__ constexpr int epi_warps(int ntok) { return ntok >= 128 ? 8 : 4; }
__host__ __device__ constexpr int stage_bytes(int ntok) { return 2 * kBoxW + ntok * 128; }
__host__ __device__ constexpr uint32_t tmem_cols(int ntok) {
    return 2 * ntok <= 32 ? 32 : 2 * ntok <= 64 ? 64 : 2 * ntok <= 128 ? 128 : 2 * ntok <= 256 ? 256 : 512;
}
__host__ __device__ constexpr size_t smem_bytes(int ntok) {
    return 1024 + (size_t)stages_for(ntok) * stage_bytes(ntok) + (2 * stages_for(ntok) + 8) * sizeof(uint64_t) + 16;
}

struct GemmArgs {
    int64_t M;                 // tokens
    int N, K;                  // output columns, contraction
    int ksteps;                // ceil(K / 64)
    int S, kper;               // k splits and k steps per split
    int n_tiles, m_tiles;
    int64_t n_units;           // n_tiles * m_tiles * S
    __nv_bfloat16 *y;          // [M, ld_y]
    int64_t ld_y;
    const __nv_bfloat16 *res;  // residual [M, ld_res] added before the rounding (may alias y), or nullptr
    int64_t ld_res;
    float *part;               // S > 1: partials [S][M][N]
    int *tickets;              // S > 1: one arrival counter per (token tile, column tile), zero at launch
    int *status;
};

struct Unit {
    int n_tile, m_tile, split;
    int k0, k1;                // k steps [k0, k1)
};

// Tile order: bands of kBand token tiles; inside a band, column-tile major (consecutive units share a
// weight tile), splits of one tile adjacent.
__device__ __forceinline__ Unit unit_of(const GemmArgs &a, int64_t u) {
    Unit x;
    x.split = (int)(u % a.S);
    const int64_t p = u / a.S;
    const int64_t per_band = (int64_t)kBand * a.n_tiles;
    const int band = (int)(p / per_band);
    const int64_t r = p % per_band;
    const int rows = min(kBand, a.m_tiles - band * kBand);
    x.n_tile = (int)(r / rows);
    x.m_tile = band * kBand + (int)(r % rows);
    x.k0 = x.split * a.kper;
    x.k1 = min(a.ksteps, x.k0 + a.kper);
    return x;
}

template <int NTOK>
__global__ void __launch_bounds__(64 + 32 * epi_warps(NTOK), ctas_per_sm(NTOK))
gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x, GemmArgs a) {
    constexpr int NS = stages_for(NTOK), SB = stage_bytes(NTOK), E = epi_warps(NTOK), ET = 32 * E;
    constexpr int kColsPerWarp = NTOK / (E / 4);   // accumulator columns (tokens) each epilogue warp drains
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + NS * SB);
    uint64_t *full = bars, *empty = bars + NS, *acc_full = bars + 2 * NS, *acc_empty = acc_full + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_empty + 2);
    int *s_last = reinterpret_cast<int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; ++i) { tc::mbar_init(&full[i], 1); tc::mbar_init(&empty[i], 1); }
        for (int i = 0; i < 2; ++i) { tc::mbar_init(&acc_full[i], 1); tc::mbar_init(&acc_empty[i], E); }
        tc::fence_mbar_init();
    }
    if (warp == 0) tc::tmem_alloc(tmem_slot, tmem_cols(NTOK));
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t it = 0;
            for (int64_t u = blockIdx.x; u < a.n_units && ok; u += gridDim.x) {
                const Unit x = unit_of(a, u);
                const int n0 = x.n_tile * kBN;
                const bool two = n0 + 64 < a.N;   // the second 64-column box holds at least one column
                const uint32_t bytes = (two ? 2 : 1) * kBoxW + NTOK * 128;
                for (int ks = x.k0; ks < x.k1 && ok; ++ks, ++it) {
                    const int s = it % NS;
                    if (it >= NS) ok = ok && tc::mbar_wait(&empty[s], ((it / NS) - 1) & 1, a.status);
                    if (!ok) break;
                    uint8_t *st = base + s * SB;
                    tc::mbar_arrive_expect_tx(&full[s], bytes);
                    tc::tma_load_2d(tc::smem_u32(st), &tm_w, n0, ks * 64, &full[s]);
                    if (two) tc::tma_load_2d(tc::smem_u32(st + kBoxW), &tm_w, n0 + 64, ks * 64, &full[s]);
                    tc::tma_load_2d(tc::smem_u32(st + 2 * kBoxW), &tm_x, ks * 64, x.m_tile * NTOK, &full[s]);
                }
            }
            // after a failed wait: let the copies still in flight land before the CTA exits
            if (!ok)
                for (uint32_t i = it > (uint32_t)NS ? it - NS : 0; i < it; ++i)
                    tc::mbar_wait(&full[i % NS], (i / NS) & 1, a.status);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = tc::idesc_bf16(128, NTOK, true, false);
            uint32_t it = 0, iacc = 0;
            for (int64_t u = blockIdx.x; u < a.n_units && ok; u += gridDim.x, ++iacc) {
                const Unit x = unit_of(a, u);
                const int ab = iacc & 1;
                if (iacc >= 2) ok = ok && tc::mbar_wait(&acc_empty[ab], ((iacc >> 1) - 1) & 1, a.status);
                for (int ks = x.k0; ks < x.k1 && ok; ++ks, ++it) {
                    const int s = it % NS;
                    ok = ok && tc::mbar_wait(&full[s], (it / NS) & 1, a.status);
                    if (!ok) break;
                    tc::tc_fence_after();
                    const uint32_t wa = tc::smem_u32(base + s * SB), xa = wa + 2 * kBoxW;
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        tc::mma_bf16(tmem + ab * NTOK, tc::sdesc_sw128(wa + 2048 * k, kBoxW, 1024),
                                     tc::sdesc_sw128(xa + 32 * k, 16, 1024), idesc, (ks > x.k0 || k > 0) ? 1u : 0u);
                    tc::mma_commit(&empty[s]);
                }
                if (!ok) break;
                tc::mma_commit(&acc_full[ab]);
            }
        }
    } else {
        // ------------------------------------------------ epilogue: TMEM -> bf16 (split-K: partials, last CTA reduces)
        const int ew = warp - 2;                      // 0 .. E-1
        const int quad = warp & 3;                    // TMEM lane quadrant this warp may read
        const int c_begin = (ew >> 2) * kColsPerWarp;
        const int et = threadIdx.x - 64;
        uint32_t iacc = 0;
        for (int64_t u = blockIdx.x; u < a.n_units; u += gridDim.x, ++iacc) {
            const Unit x = unit_of(a, u);
            const int ab = iacc & 1;
            ok = ok && tc::mbar_wait(&acc_full[ab], (iacc >> 1) & 1, a.status);
            if (a.S > 1) ok = tc::named_bar_and(1, ET, ok);   // the split-K path meets at barriers below
            if (!ok) break;
            tc::tc_fence_after();
            const int n = x.n_tile * kBN + quad * 32 + lane;
            const int64_t t0 = (int64_t)x.m_tile * NTOK;
            const uint32_t tl = tmem + ab * NTOK + ((uint32_t)(quad * 32) << 16);
            constexpr int CH = kColsPerWarp < 32 ? kColsPerWarp : 32;   // columns per TMEM load
            for (int c0 = c_begin; c0 < c_begin + kColsPerWarp; c0 += CH) {
                float v[CH];
                if constexpr (CH == 32) tc::tmem_ld32(tl + c0, v);
                else tc::tmem_ld16(tl + c0, v);
                tc::tmem_ld_wait();
                if (a.S == 1) {
                    if (n < a.N) {
#pragma unroll
                        for (int i = 0; i < CH; ++i) {
                            const int64_t t = t0 + c0 + i;
                            if (t < a.M) {
                                float r = v[i];
                                if (a.res) r += __bfloat162float(a.res[t * a.ld_res + n]);
                                a.y[t * a.ld_y + n] = __float2bfloat16_rn(r);
                            }
                        }
                    }
                } else if (n < a.N) {
                    float *pp = a.part + (size_t)x.split * a.M * a.N;
#pragma unroll
                    for (int i = 0; i < CH; ++i) {
                        const int64_t t = t0 + c0 + i;
                        if (t < a.M) pp[t * a.N + n] = v[i];
                    }
                }
            }
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&acc_empty[ab]);
            if (a.S > 1) {
                // publish this split's partials; the last split of the tile to arrive reduces them
                __threadfence();
                tc::named_bar_sync(1, ET);
                if (et == 0) {
                    int *tk = &a.tickets[(int64_t)x.m_tile * a.n_tiles + x.n_tile];
                    const int prev = atomicAdd(tk, 1);
                    *s_last = prev == a.S - 1;
                    if (prev == a.S - 1) *tk = 0;   // leave the counter at zero for the next call
                }
                tc::named_bar_sync(1, ET);
                if (*s_last) {
                    __threadfence();
                    // thread -> (column, token group): the 128 columns of the tile, ET / 128 token groups
                    constexpr int G = ET / 128;
                    const int nn = x.n_tile * kBN + (et & 127);
                    if (nn < a.N) {
                        for (int64_t t = t0 + (et >> 7); t < t0 + NTOK && t < a.M; t += G) {
                            float r = 0.f;
                            for (int s = 0; s < a.S; ++s) r += __ldcg(&a.part[((size_t)s * a.M + t) * a.N + nn]);
                            if (a.res) r += __bfloat162float(a.res[t * a.ld_res + nn]);
                            a.y[t * a.ld_y + nn] = __float2bfloat16_rn(r);
                        }
                    }
                }
            }
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_free(tmem, tmem_cols(NTOK));
    }
}

int num_sms() {
    static int n = 0;
    if (!n) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

// split-K scratch: partials of at most this many fp32 values, then the tickets
constexpr size_t kPartFloats = (size_t)4 << 20;
constexpr size_t kTicketBytes = 4096;

template <int NTOK>
hcsa_status launch_ntok(const CUtensorMap &tw, const CUtensorMap &tx, GemmArgs a, cudaStream_t st) {
    constexpr size_t smem = smem_bytes(NTOK);
    static_assert(smem <= 232448, "shared memory per CTA");
    static bool configured[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return HCSA_ERR_CUDA;
    if (!configured[dev]) {
        if (cudaFuncSetAttribute(gemm_tc_kernel<NTOK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return HCSA_ERR_CUDA;
        configured[dev] = true;
    }
    const int64_t slots = (int64_t)num_sms() * ctas_per_sm(NTOK);
    const int64_t grid = a.n_units < slots ? a.n_units : slots;
    gemm_tc_kernel<NTOK><<<(unsigned)grid, 64 + 32 * epi_warps(NTOK), smem, st>>>(tw, tx, a);
    count_launch();
    return check_launch();
}

}  // namespace

size_t gemm_tc_ws_bytes() { return kPartFloats * sizeof(float) + kTicketBytes; }

bool gemm_tc_supported(int64_t M, int N, int K, const void *x, int64_t ld_x, const void *W, int64_t ld_w,
                       const void *y, int64_t ld_y) {
    if (M < 1 || N < 1 || K < 1 || M > INT32_MAX) return false;
    // TMA: 16-byte aligned bases and row strides
    if (((uintptr_t)x & 15) || ((uintptr_t)W & 15) || (ld_x * 2) % 16 || (ld_w * 2) % 16) return false;
    if (ld_x < K || ld_w < N || ld_y < N) return false;
    return y != nullptr;
}

hcsa_status launch_gemm_tc(int64_t M, int N, int K, const void *x, int64_t ld_x, const void *W, int64_t ld_w,
                           void *y, int64_t ld_y, const void *res, int64_t ld_res, void *ws, size_t ws_bytes,
                           cudaStream_t st) {
    const int ntok = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : M <= 128 ? 128 : 256;
    CUtensorMap tw, tx;
    if (!make_tmap_bf16_2d(&tw, W, (uint64_t)N, (uint64_t)K, (uint64_t)ld_w * 2, 64, 64, true)) return HCSA_ERR_CUDA;
    if (!make_tmap_bf16_2d(&tx, x, (uint64_t)K, (uint64_t)M, (uint64_t)ld_x * 2, 64, (uint32_t)ntok, true))
        return HCSA_ERR_CUDA;
    GemmArgs a{};
    a.M = M; a.N = N; a.K = K;
    a.ksteps = (K + 63) / 64;
    a.n_tiles = (N + kBN - 1) / kBN;
    a.m_tiles = (int)((M + ntok - 1) / ntok);
    a.y = (__nv_bfloat16 *)y; a.ld_y = ld_y;
    a.res = (const __nv_bfloat16 *)res; a.ld_res = ld_res;
    a.status = device_status_ptr();
    // split K only when the tiles alone leave most of the GPU idle and the partials fit the workspace
    const int64_t slots = (int64_t)num_sms() * ctas_per_sm(ntok);
    const int64_t tiles = (int64_t)a.n_tiles * a.m_tiles;
    int S = 1;
    if (tiles * 2 <= slots && ws && ws_bytes >= gemm_tc_ws_bytes() && tiles * (int64_t)sizeof(int) <= (int64_t)kTicketBytes) {
        S = (int)(slots / tiles);   // one wave: every unit gets its own CTA slot
        if (S > a.ksteps) S = a.ksteps;
        while (S > 1 && (size_t)S * M * N > kPartFloats) --S;
    }
    a.kper = (a.ksteps + S - 1) / S;
    a.S = (a.ksteps + a.kper - 1) / a.kper;   // every split has at least one k step
    a.n_units = tiles * a.S;
    if (a.S > 1) {
        a.part = (float *)ws;
        a.tickets = (int *)((uint8_t *)ws + kPartFloats * sizeof(float));
        if (cudaMemsetAsync(a.tickets, 0, (size_t)tiles * sizeof(int), st) != cudaSuccess) return HCSA_ERR_CUDA;
    }
    switch (ntok) {
        case 16: return launch_ntok<16>(tw, tx, a, st);
        case 32: return launch_ntok<32>(tw, tx, a, st);
        case 64: return launch_ntok<64>(tw, tx, a, st);
        case 128: return launch_ntok<128>(tw, tx, a, st);
        default: return launch_ntok<256>(tw, tx, a, st);
    }
}

}  // namespace hcsa

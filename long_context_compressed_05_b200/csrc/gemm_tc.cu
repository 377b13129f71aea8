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
//
// Decode step with the cache append in the epilogue (the compressor fed straight from the projection
// tile).  The pooled columns are tiled in pairs: a tile's first 64 accumulator lanes hold 64 value
// channels (kv, or the 64 indexer-key channels) and its last 64 lanes the gate channels of the same
// index.  The gate lanes pass their bf16 values through shared memory; the value lanes then write the
// new token into the rings and, when the token closes an entry, pool it from the rings and the tile
// (the same online softmax as the append kernel, so the results are identical).  The other columns
// (indexer queries, head weights, queries) are tiled as usual.
#include "lowprec.cuh"
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
__host__ __device__ constexpr size_t smem_bytes(int ntok, int pool = 0) {
    // pool 1 (decode append): gates [64][ntok]; pool 2 (prefill compressor): gates [2 halves][64][32]
    return 1024 + (size_t)stages_for(ntok) * stage_bytes(ntok) + (2 * stages_for(ntok) + 8) * sizeof(uint64_t) + 16 +
           (pool == 1 ? 64 * ntok * sizeof(float) : pool == 2 ? 2 * 64 * 32 * sizeof(float) : 0);
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

// Fused cache append (decode, S = 1): the first pool_tiles column tiles pair value and gate channels.
struct PoolArgs {
    int pool_tiles;            // 0: a plain GEMM
    int plain0;                // first column of the plain tiles
    const int32_t *pos;        // position of each row's new token
    int C, di, m, width, window;
    int64_t n_cap, ent0, rows_total;
    bool shard, lowprec;
    const __nv_bfloat16 *bias; // [width, C]
    __nv_bfloat16 *entries, *idx_keys, *win_kv, *ring_g, *ring_ki;
};

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Store one entry value e (a bf16 number) of channel c of row j, bf16 or block-scaled (the warp's 32 lanes
// are one 32-channel block; every lane of the warp calls this together).
__device__ __forceinline__ void store_entry_value(float e, bool key, int64_t j, int c, int lane, int64_t rows_total,
                                                  int C, int di, bool lowprec, __nv_bfloat16 *entries,
                                                  __nv_bfloat16 *idx_keys) {
    if (!lowprec) {
        if (key) idx_keys[j * di + c] = __float2bfloat16_rn(e);
        else entries[j * C + c] = __float2bfloat16_rn(e);
        return;
    }
    float am = fabsf(e);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
    if (key) {
        uint8_t *codes = reinterpret_cast<uint8_t *>(idx_keys);
        int8_t *ex = reinterpret_cast<int8_t *>(codes + rows_total * (di / 2));
        const int ee = lp::block_exponent(am, 1.5f, 2);
        const uint32_t cd = __nv_cvt_float_to_fp4(scalbnf(e, -ee), __NV_E2M1, cudaRoundNearest) & 0xFu;
        const uint32_t hi = __shfl_down_sync(0xffffffffu, cd, 1);
        if ((lane & 1) == 0) codes[j * (di / 2) + c / 2] = (uint8_t)(cd | (hi << 4));
        if (lane == 0) ex[j * (di / 32) + c / 32] = (int8_t)ee;
    } else {
        uint8_t *codes = reinterpret_cast<uint8_t *>(entries);
        int8_t *ex = reinterpret_cast<int8_t *>(codes + rows_total * C);
        const int ee = lp::block_exponent(am, 1.75f, 8);
        codes[j * C + c] = (uint8_t)__nv_cvt_float_to_fp8(scalbnf(e, -ee), __NV_SATFINITE, __NV_E4M3);
        if (lane == 0) ex[j * (C / 32) + c / 32] = (int8_t)ee;
    }
}

// Prefill: the CSA compressor (pools of 8 tokens at stride 4) on one 32-token chunk of a pooled tile.  The
// four warps of a 128-token half call this together: the gate lanes publish the chunk's bf16 gates, each
// value lane appends the chunk's tokens to its 8-token ring and closes the entries whose last token is in
// the chunk, with the compressor kernel's two-pass softmax in its row order (so the entries are
// identical).  Entries whose pool reaches into the previous half are left to the seam pass.
__device__ void fused_compress_chunk(const GemmArgs &g, const PoolArgs &a, const float *v, int quad, int lane,
                                     int64_t tb, int64_t hs, int nt, int ca, float *sg, int bar_id, float (&kr)[8],
                                     float (&gr)[8], const float (&b8)[8]) {
    constexpr float kLog2e = 1.4426950408889634f;
    const int l = (quad & 1) * 32 + lane;
    if (quad >= 2) {
#pragma unroll
        for (int i = 0; i < 32; ++i) sg[l * 32 + i] = __bfloat162float(__float2bfloat16_rn(v[i]));
    }
    tc::named_bar_sync(bar_id, 128);
    if (quad < 2) {
        const bool key = nt >= a.C / 64;
        const int c = key ? l : ca + l;
        const int64_t T = g.M;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int64_t t = tb + i;
            if (t < T) {
                kr[i & 7] = __bfloat162float(__float2bfloat16_rn(v[i]));
                gr[i & 7] = sg[l * 32 + i];
            }
            // entry j = t / 4 closes at its last token (4 j + 3, or the sequence's last)
            if (t < T && ((i & 3) == 3 || t == T - 1)) {
                const int64_t j = t >> 2;
                const int64_t lo = 4 * j - 4;
                if ((lo < 0 ? 0 : lo) >= hs) {
                    float mx = -INFINITY;
#pragma unroll
                    for (int r = 0; r < 8; ++r) {
                        const int64_t tok = lo + r;
                        const int sl = ((i & 7) - (i & 3) - 4 + r) & 7;   // ring slot of token lo + r
                        if (tok >= 0 && tok <= t) mx = fmaxf(mx, gr[sl] + b8[r]);
                    }
                    float z = 0.f, acc = 0.f;
#pragma unroll
                    for (int r = 0; r < 8; ++r) {
                        const int64_t tok = lo + r;
                        const int sl = ((i & 7) - (i & 3) - 4 + r) & 7;
                        if (tok >= 0 && tok <= t) {
                            const float p = ex2_approx((gr[sl] + b8[r] - mx) * kLog2e);
                            z += p;
                            acc = fmaf(p, kr[sl], acc);
                        }
                    }
                    const float e = __bfloat162float(__float2bfloat16_rn(acc / z));
                    store_entry_value(e, key, j, c, lane, a.rows_total, a.C, a.di, a.lowprec, a.entries, a.idx_keys);
                }
            }
        }
    }
    tc::named_bar_sync(bar_id, 128);   // the gate buffer is rewritten by the next chunk
}

// Columns of the two 64-column boxes of column tile nt (box 0 -> TMEM lanes 0..63, box 1 -> 64..127).
template <int POOL>
__device__ __forceinline__ void tile_cols(const PoolArgs &a, int nt, int &ca, int &cb) {
    if (!POOL) {   // a plain GEMM
        ca = nt * 128;
        cb = ca + 64;
        return;
    }
    if (nt < a.pool_tiles) {
        if (nt < a.C / 64) {
            ca = nt * 64;           // kv channels
            cb = a.C + nt * 64;     // their gate channels
        } else {
            ca = 2 * a.C;           // the indexer-key channels 0..63
            cb = a.C;               // gate channels 0..63
        }
    } else {
        ca = a.plain0 + (nt - a.pool_tiles) * 128;
        cb = ca + 64;
    }
}

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

// The cache append of one pooled tile's 64 channels for the tile's tokens (one decode sequence each).  Called
// by the four epilogue warps of the tile together (warp quad holds TMEM lanes 32 quad .. 32 quad + 31):
// the gate lanes (quads 2, 3) publish their bf16 gate values, the value lanes (quads 0, 1) append.
template <int NTOK>
__device__ void fused_append(const GemmArgs &g, const PoolArgs &a, const float *v, int quad, int lane, int64_t t0,
                             int nt, int ca, int cb, float *sgate) {
    const int l = (quad & 1) * 32 + lane;   // channel within the 64-channel pair
    if (quad >= 2) {
#pragma unroll
        for (int i = 0; i < NTOK; ++i) sgate[l * NTOK + i] = __bfloat162float(__float2bfloat16_rn(v[i]));
    }
    tc::named_bar_sync(1, 128);
    if (quad < 2) {
        const bool key = nt >= a.C / 64;                  // indexer-key channels (gates 0..63)
        const int c = key ? l : ca + l;                   // value channel (key: indexer-key channel)
        const int gc = cb - a.C + l;                      // gate channel
        for (int i = 0; i < NTOK; ++i) {
            const int64_t b = t0 + i;
            if (b >= g.M) break;
            const int64_t P = a.pos[b];
            if (P < 0) {
                if (l == 0) report(g.status, kStatusBounds);
                continue;
            }
            float vi = 0.f;   // v[i] by an unrolled select: v stays in registers
#pragma unroll
            for (int k = 0; k < NTOK; ++k) vi = k == i ? v[k] : vi;
            const float vnew = __bfloat162float(__float2bfloat16_rn(vi)), gnew = sgate[l * NTOK + i];
            if (key) {
                a.ring_ki[(b * a.width + P % a.width) * a.di + c] = __float2bfloat16_rn(vnew);
            } else {
                a.win_kv[(b * a.window + P % a.window) * a.C + c] = __float2bfloat16_rn(vnew);
                a.ring_g[(b * a.width + P % a.width) * a.C + c] = __float2bfloat16_rn(gnew);
            }
            if ((P + 1) % a.m != 0) continue;
            const int64_t jg = (P + 1) / a.m - 1;         // the entry the token closes
            if (a.shard && (jg < a.ent0 || jg >= a.ent0 + a.n_cap)) continue;
            const int64_t j = jg - a.ent0;
            if (j >= a.n_cap) {
                if (l == 0) report(g.status, kStatusBounds);
                continue;
            }
            const int64_t lo = (int64_t)a.m * jg - (a.width - a.m);
            float mx = -INFINITY, z = 0.f, acc = 0.f;
            for (int64_t t = lo < 0 ? 0 : lo; t <= P; ++t) {
                const float g = t == P ? gnew : __bfloat162float(a.ring_g[(b * a.width + t % a.width) * a.C + gc]);
                const float val = t == P ? vnew
                                  : key ? __bfloat162float(a.ring_ki[(b * a.width + t % a.width) * a.di + c])
                                        : __bfloat162float(a.win_kv[(b * a.window + t % a.window) * a.C + c]);
                const float lg = g + __bfloat162float(a.bias[(t - lo) * a.C + gc]);
                if (lg > mx) {
                    const float sc = expf(mx - lg);
                    acc = acc * sc + val;
                    z = z * sc + 1.f;
                    mx = lg;
                } else {
                    const float p = expf(lg - mx);
                    acc += p * val;
                    z += p;
                }
            }
            const float e = __bfloat162float(__float2bfloat16_rn(acc / z));
            const int64_t row = b * a.n_cap + j;
            if (!a.lowprec) {
                if (key) a.idx_keys[row * a.di + c] = __float2bfloat16_rn(e);
                else a.entries[row * a.C + c] = __float2bfloat16_rn(e);
                continue;
            }
            // block-scaled storage: the warp's 32 lanes are one 32-channel block
            float am = fabsf(e);
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
            if (key) {
                uint8_t *codes = reinterpret_cast<uint8_t *>(a.idx_keys);
                int8_t *ex = reinterpret_cast<int8_t *>(codes + a.rows_total * (a.di / 2));
                const int ee = lp::block_exponent(am, 1.5f, 2);
                const uint32_t cd = __nv_cvt_float_to_fp4(scalbnf(e, -ee), __NV_E2M1, cudaRoundNearest) & 0xFu;
                const uint32_t hi = __shfl_down_sync(0xffffffffu, cd, 1);
                if ((lane & 1) == 0) codes[row * (a.di / 2) + c / 2] = (uint8_t)(cd | (hi << 4));
                if (lane == 0) ex[row * (a.di / 32) + c / 32] = (int8_t)ee;
            } else {
                uint8_t *codes = reinterpret_cast<uint8_t *>(a.entries);
                int8_t *ex = reinterpret_cast<int8_t *>(codes + a.rows_total * a.C);
                const int ee = lp::block_exponent(am, 1.75f, 8);
                codes[row * a.C + c] = (uint8_t)__nv_cvt_float_to_fp8(scalbnf(e, -ee), __NV_SATFINITE, __NV_E4M3);
                if (lane == 0) ex[row * (a.C / 32) + c / 32] = (int8_t)ee;
            }
        }
    }
    tc::named_bar_sync(1, 128);   // the gate buffer is reused by the next tile
}

template <int NTOK, int POOL>
__global__ void __launch_bounds__(64 + 32 * epi_warps(NTOK), ctas_per_sm(NTOK))
gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x, GemmArgs a,
               const __grid_constant__ PoolArgs pa) {
    constexpr int NS = stages_for(NTOK), SB = stage_bytes(NTOK), E = epi_warps(NTOK), ET = 32 * E;
    constexpr int kColsPerWarp = NTOK / (E / 4);   // accumulator columns (tokens) each epilogue warp drains
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + NS * SB);
    uint64_t *full = bars, *empty = bars + NS, *acc_full = bars + 2 * NS, *acc_empty = acc_full + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_empty + 2);
    int *s_last = reinterpret_cast<int *>(tmem_slot + 1);
    float *sgate = reinterpret_cast<float *>(tmem_slot + 4);   // fused append / compressor: gate values

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
                int n0, n1;
                tile_cols<POOL>(pa, x.n_tile, n0, n1);
                const bool two = n1 < a.N;   // the second 64-column box holds at least one column
                const uint32_t bytes = (two ? 2 : 1) * kBoxW + NTOK * 128;
                for (int ks = x.k0; ks < x.k1 && ok; ++ks, ++it) {
                    const int s = it % NS;
                    if (it >= NS) ok = ok && tc::mbar_wait(&empty[s], ((it / NS) - 1) & 1, a.status);
                    if (!ok) break;
                    uint8_t *st = base + s * SB;
                    tc::mbar_arrive_expect_tx(&full[s], bytes);
                    tc::tma_load_2d(tc::smem_u32(st), &tm_w, n0, ks * 64, &full[s]);
                    if (two) tc::tma_load_2d(tc::smem_u32(st + kBoxW), &tm_w, n1, ks * 64, &full[s]);
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
            // the split-K path and the fused append meet at barriers below
            if (a.S > 1 || POOL != 0) ok = tc::named_bar_and(1, ET, ok);
            if (!ok) break;
            tc::tc_fence_after();
            int ca = 0, cb = 0;
            int n = x.n_tile * kBN + quad * 32 + lane;
            if constexpr (POOL != 0) {
                tile_cols<POOL>(pa, x.n_tile, ca, cb);
                n = quad < 2 ? ca + quad * 32 + lane : cb + (quad - 2) * 32 + lane;
            }
            // prefill compressor state of a value lane: the last 8 tokens (value, gate) and the 8 bias rows
            float kr[8], gr[8], b8[8];
            const bool pooled = POOL == 2 && x.n_tile < pa.pool_tiles;
            if constexpr (POOL == 2) {
                if (pooled && quad < 2) {
                    const int gc = cb - pa.C + (quad & 1) * 32 + lane;
#pragma unroll
                    for (int r = 0; r < 8; ++r) b8[r] = __bfloat162float(pa.bias[r * pa.C + gc]);
                }
            }
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
                if constexpr (POOL == 1) {
                    if (x.n_tile < pa.pool_tiles)
                        fused_append<NTOK>(a, pa, v, quad, lane, t0, x.n_tile, ca, cb, sgate);
                }
                if constexpr (POOL == 2 && CH == 32) {
                    if (pooled)
                        fused_compress_chunk(a, pa, v, quad, lane, t0 + c0, t0 + c_begin, x.n_tile, ca,
                                             sgate + (c_begin / 128) * 64 * 32, 2 + c_begin / 128, kr, gr, b8);
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
                    const int nn = x.n_tile * kBN + (et & 127);   // split-K never runs with the fused append
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

template <int NTOK, int POOL = 0>
hcsa_status launch_ntok(const CUtensorMap &tw, const CUtensorMap &tx, GemmArgs a, cudaStream_t st,
                        const PoolArgs &pa = PoolArgs{}) {
    constexpr size_t smem = smem_bytes(NTOK, POOL);
    static_assert(smem <= 232448, "shared memory per CTA");
    static bool configured[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return HCSA_ERR_CUDA;
    if (!configured[dev]) {
        if (cudaFuncSetAttribute(gemm_tc_kernel<NTOK, POOL>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return HCSA_ERR_CUDA;
        configured[dev] = true;
    }
    const int64_t slots = (int64_t)num_sms() * ctas_per_sm(NTOK);
    const int64_t grid = a.n_units < slots ? a.n_units : slots;
    gemm_tc_kernel<NTOK, POOL><<<(unsigned)grid, 64 + 32 * epi_warps(NTOK), smem, st>>>(tw, tx, a, pa);
    count_launch();
    return check_launch();
}

}  // namespace

size_t gemm_tc_ws_bytes() { return kPartFloats * sizeof(float) + kTicketBytes; }

// Fused only up to one 16-token tile: the value lanes append the tile's tokens one after another, and at
// 32 sequences that serial loop costs more than the separate append kernel (measured: 161 vs 143 us per
// CSA layer at 32 sequences, 106.5 vs 107.8 us at 4).
// Prefill: the CSA compressor (m = 4, width = 8) in the epilogue of the projection's 256-token tiles.  Pools
// inside a 128-token half of a tile are formed there; the one pool per half boundary that reaches into the
// previous half (entry 32 s) is formed afterwards from the stored projections by the compressor kernel.
// Measured at T = 131072: 18.0-19.5 ms against 17.4-18.9 ms for the projection and the compressor kernel
// (the pooled tiles' epilogue costs more than the 0.4 ms pass it replaces).
bool project_compress_supported(const hcsa_params &p, bool csa) {
    return csa && p.dtype == HCSA_BF16 && p.m == 4 && p.width == 8 && p.C % 64 == 0 && p.di == 64 &&
           p.D % 8 == 0 && p.T >= 1 && p.T <= INT32_MAX;
}

hcsa_status launch_project_compress(const hcsa_params &p, const void *x, const void *W, int64_t ncols, void *y,
                                    const void *bias, void *entries, void *idx_keys, cudaStream_t st) {
    const int64_t M = p.T;
    const int N = (int)ncols, K = p.D;
    constexpr int ntok = 256;
    CUtensorMap tw, tx;
    if (!make_tmap_bf16_2d(&tw, W, (uint64_t)N, (uint64_t)K, (uint64_t)N * 2, 64, 64, true)) return HCSA_ERR_CUDA;
    if (!make_tmap_bf16_2d(&tx, x, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2, 64, (uint32_t)ntok, true))
        return HCSA_ERR_CUDA;
    GemmArgs a{};
    a.M = M; a.N = N; a.K = K;
    a.ksteps = (K + 63) / 64;
    a.S = 1; a.kper = a.ksteps;
    PoolArgs pa{};
    pa.pool_tiles = p.C / 64 + 1;
    pa.plain0 = 2 * p.C + p.di;
    a.n_tiles = pa.pool_tiles + (N - pa.plain0 + kBN - 1) / kBN;
    a.m_tiles = (int)((M + ntok - 1) / ntok);
    a.n_units = (int64_t)a.n_tiles * a.m_tiles;
    a.y = (__nv_bfloat16 *)y; a.ld_y = N;
    a.status = device_status_ptr();
    const int64_t n_ent = (p.T + p.m - 1) / p.m;
    pa.C = p.C; pa.di = p.di; pa.m = p.m; pa.width = p.width;
    pa.rows_total = n_ent; pa.lowprec = p.lowprec != 0;
    pa.bias = (const __nv_bfloat16 *)bias;
    pa.entries = (__nv_bfloat16 *)entries; pa.idx_keys = (__nv_bfloat16 *)idx_keys;
    const hcsa_status s = launch_ntok<ntok, 2>(tw, tx, a, st, pa);
    if (s != HCSA_OK) return s;
    // seams: entries 32, 64, ... (pools across a 128-token boundary), from the stored projections
    const uint8_t *y8 = (const uint8_t *)y;
    return launch_compress(HCSA_BF16, p.T, p.C, p.m, p.width, y8, N, y8 + 2 * (int64_t)p.C, N,
                           y8 + 4 * (int64_t)p.C, N, p.di, bias, entries, idx_keys, 32, n_ent, p.lowprec != 0, n_ent,
                           st, 32);
}

bool project_append_supported(const hcsa_params &p, bool csa) {
    return p.dtype == HCSA_BF16 && p.B >= 1 && p.B <= 16 && p.C % 64 == 0 && (!csa || p.di == 64) && p.D % 8 == 0;
}

hcsa_status launch_project_append(const hcsa_params &p, bool csa, const hcsa_cache &c, const int32_t *pos,
                                  const void *x, const void *W, int64_t ncols, void *y, const void *bias,
                                  cudaStream_t st) {
    const int64_t M = p.B;
    const int N = (int)ncols, K = p.D;
    constexpr int ntok = 16;
    CUtensorMap tw, tx;
    if (!make_tmap_bf16_2d(&tw, W, (uint64_t)N, (uint64_t)K, (uint64_t)N * 2, 64, 64, true)) return HCSA_ERR_CUDA;
    if (!make_tmap_bf16_2d(&tx, x, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2, 64, (uint32_t)ntok, true))
        return HCSA_ERR_CUDA;
    GemmArgs a{};
    a.M = M; a.N = N; a.K = K;
    a.ksteps = (K + 63) / 64;
    a.S = 1; a.kper = a.ksteps;
    PoolArgs pa{};
    pa.pool_tiles = p.C / 64 + (csa ? 1 : 0);
    pa.plain0 = 2 * p.C + (csa ? p.di : 0);
    a.n_tiles = pa.pool_tiles + (N - pa.plain0 + kBN - 1) / kBN;
    a.m_tiles = (int)((M + ntok - 1) / ntok);
    a.n_units = (int64_t)a.n_tiles * a.m_tiles;
    a.y = (__nv_bfloat16 *)y; a.ld_y = N;
    a.status = device_status_ptr();
    pa.pos = pos;
    pa.C = p.C; pa.di = p.di; pa.m = p.m; pa.width = p.width; pa.window = p.window;
    pa.n_cap = p.n_cap; pa.ent0 = p.ent0; pa.rows_total = (int64_t)p.B * p.n_cap;
    pa.shard = p.ent_shard != 0; pa.lowprec = p.lowprec != 0;
    pa.bias = (const __nv_bfloat16 *)bias;
    pa.entries = (__nv_bfloat16 *)c.entries; pa.idx_keys = (__nv_bfloat16 *)c.idx_keys;
    pa.win_kv = (__nv_bfloat16 *)c.win_kv; pa.ring_g = (__nv_bfloat16 *)c.ring_g; pa.ring_ki = (__nv_bfloat16 *)c.ring_ki;
    return launch_ntok<16, 1>(tw, tx, a, st, pa);
}

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

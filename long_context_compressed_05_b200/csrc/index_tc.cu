// Lightning indexer on the tensor cores + register-resident exact top-k (bf16 storage).
//
// Operation ("DeepSeek-V4 ... KV cache compressed attention", section "CSA":
// the Lightning Indexer scores the compressed blocks, the top-k are kept; fixed
// by the CSA workload definition): s[t,j] = sum_h w[t,h] ReLU(qi[t,h,:] . k_j)
// over visible entries (m j + m <= t); top-k keeps the min(k, visible) best,
// equal scores to the lower j.
//
// Scores kernel.  The contraction has K = di = 64 only, so it is arranged to keep
// the tensor core and the ReLU-weighted head reduction both busy:
//   * A = 128 indexer keys (one TMEM lane each), B = TQ tokens x Hi heads of qi
//     (TQ * Hi = 256 columns for prefill, Hi for decode), both loaded by TMA in the
//     128-byte swizzled K-major layout (64 bf16 = one swizzle row);
//   * 4 MMAs (K = 16 each) per key tile into one of two 256-column TMEM
//     accumulators, so the epilogue of tile i overlaps the MMAs of tile i + 1;
//   * prefill: 16 epilogue warps (four per TMEM lane quadrant, each owning 64 of the
//     256 columns) read the accumulator, apply ReLU, weight by w and sum the heads in
//     registers -- no cross-lane traffic -- and store fp32 scores coalesced;
//   * decode (one token, Hi columns): two CTAs per SM; four key tiles share a
//     128-column accumulator, 8 epilogue warps in two groups each own one of the CTA's
//     two accumulators and also count the row's 12-bit key histogram for the
//     multi-CTA top-k; a tile's four MMAs form a dependent chain whose latency sets
//     the pace, so the K steps of two tiles are issued interleaved.
// Warp roles: warp 0 = TMA producer, warp 1 = MMA issuer, the rest = epilogue.
// Persistent CTAs: prefill walks query tiles (heaviest causal tiles first); decode
// gives every CTA an equal contiguous share of the (sequence, key tile) pairs.
//
// Top-k kernel.  One 512-thread CTA per query row at a time (persistent, prefetching
// its next row into L2) keeps the row's scores in registers (<= 32768) and finds the
// bucket of the k-th largest order-preserving key with a 12-bit histogram pass; a
// bucket of <= 1024 keys is ranked directly (key desc, index asc), a larger one takes
// two more 10-bit passes and an equal-key scan.  The chosen indices are marked in a
// shared-memory bitmap of the row and emitted in ascending order with one block scan
// over the bitmap words.
#include <cub/block/block_scan.cuh>

#include "lowprec.cuh"
#include "tc_common.cuh"

namespace hcsa {

namespace {

constexpr int kNS = 8;               // key-tile ring stages (prefill)
// Decode runs two CTAs per SM (two independent TMA / MMA pipelines: a tile's dependent MMA chain and
// the single producer thread each pace one pipeline), each with 4 stages and 2 accumulators of 128
// TMEM columns.
constexpr int kNSDec = 4;
constexpr int kDecCtasPerSm = 2;
constexpr int kATile = 128 * 128;    // 128 keys x 64 bf16
constexpr int kBTile = 256 * 128;    // up to 256 (token, head) rows x 64 bf16
constexpr int kBTileDec = 64 * 128;  // decode: one token, Hi <= 64 heads
// epilogue warps: prefill 16 (four per TMEM lane quadrant, 64 columns each: the ReLU-weighted head sum
// is the busy part), decode 8 (two groups taking alternate accumulators)
__host__ __device__ constexpr int epi_warps(bool dec) { return dec ? 8 : 16; }
// FP4 keys: converter warps (after the epilogue warps) rebuild each staged tile of E2M1 codes as the bf16
// operand tile, one key row per thread
__host__ __device__ constexpr int conv_warps(bool dec) { return dec ? 2 : 4; }   // decode: two CTAs per SM
constexpr int kCodeTile = 128 * 32;   // 128 keys x 64 E2M1 codes
__host__ __device__ constexpr int cta_threads(bool dec, bool lp = false) {
    return 64 + 32 * epi_warps(dec) + (lp ? 32 * conv_warps(dec) : 0);
}
// key-tile ring stages: fewer with FP4 keys, whose staging ring also takes shared memory
__host__ __device__ constexpr int ring_stages(bool dec, bool lp) { return dec ? (lp ? 3 : kNSDec) : (lp ? 6 : kNS); }

struct Args {
    int64_t rows;        // prefill: T; decode: B
    int64_t N;           // entries per sequence
    int m, tq, ncols;    // tokens per unit, MMA N = tq * Hi
    int nbuf, stride;    // TMEM accumulators (2 x 256 columns, or 4 x 128 when ncols <= 128)
    bool decode;
    const int32_t *pos;
    const __nv_bfloat16 *w;
    int64_t ld_w;
    float *scores;       // [rows, N]
    uint32_t *hist;      // decode: per-row histogram of the top 12 key bits of the scores, or nullptr
    int64_t n_units, n_qtiles;   // prefill: query tiles; decode: (sequence, key tile) pairs
    int64_t tps;         // decode: key tiles per sequence (ceil(N / 128))
    int *status;
    uint32_t *bound;     // prefill, or nullptr: per row a lower bound of the order key of its k-th best score
    // FP4 keys: code pairs [key_rows][32] then int8 exponents [key_rows][2]
    const uint8_t *codes;
    const int8_t *kexp;
    int64_t key_rows;
};

struct Unit {
    int64_t b, r0;       // sequence, first query row
    int kt0, kt1;        // key tiles [kt0, kt1)
};

__device__ __forceinline__ int64_t visible(const Args &a, int64_t row) {
    int64_t p = a.decode ? (int64_t)a.pos[row] : row;
    if (p < 0) return 0;
    int64_t v = p / a.m;
    return v < a.N ? v : a.N;
}

__device__ __forceinline__ Unit unit_of(const Args &a, int64_t u) {
    Unit x;
    const int64_t q = a.n_qtiles - 1 - u;   // heaviest first
    x.b = 0;
    x.r0 = q * a.tq;
    int64_t last = x.r0 + a.tq - 1 < a.rows ? x.r0 + a.tq - 1 : a.rows - 1;
    x.kt0 = 0;
    x.kt1 = (int)((visible(a, last) + 127) / 128);
    return x;
}

// Work iteration, the same in every warp role.  Prefill: persistent CTAs take query tiles round-robin.
// Decode: CTA c takes an equal contiguous share [g0, g1) of the (sequence, key tile) pairs in
// sequence-major order; its units are the pieces of that share inside each sequence (usually one or two).
struct Iter {
    int64_t u, g, g1;
};

__device__ __forceinline__ Iter iter_begin(const Args &a) {
    Iter it;
    it.u = blockIdx.x;
    it.g = (int64_t)blockIdx.x * a.n_units / gridDim.x;
    it.g1 = (int64_t)(blockIdx.x + 1) * a.n_units / gridDim.x;
    return it;
}

__device__ __forceinline__ bool iter_next(const Args &a, Iter &it, Unit &x) {
    if (!a.decode) {
        while (it.u < a.n_units) {
            x = unit_of(a, it.u);
            it.u += gridDim.x;
            if (x.kt0 < x.kt1) return true;
        }
        return false;
    }
    while (it.g < it.g1) {
        const int64_t b = it.g / a.tps;
        const int64_t end = it.g1 < (b + 1) * a.tps ? it.g1 : (b + 1) * a.tps;
        const int nkt = (int)((visible(a, b) + 127) / 128);
        x.b = b;
        x.r0 = b;
        x.kt0 = (int)(it.g - b * a.tps);
        x.kt1 = min(nkt, (int)(end - b * a.tps));
        it.g = end;
        if (x.kt0 < x.kt1) return true;
    }
    return false;
}

// c += a * b on two fp32 lanes at once (one packed FMA instruction)
__device__ __forceinline__ void fma2(float &c0, float &c1, float a0, float a1, float b0, float b1) {
    asm("{.reg .b64 ra, rb, rc; mov.b64 ra, {%2, %3}; mov.b64 rb, {%4, %5}; mov.b64 rc, {%0, %1};"
        " fma.rn.f32x2 rc, ra, rb, rc; mov.b64 {%0, %1}, rc;}"
        : "+f"(c0), "+f"(c1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

template <int HI, bool DEC, bool LP>
__global__ void __launch_bounds__(cta_threads(DEC, LP), DEC ? kDecCtasPerSm : 1)
index_scores_tc_kernel(const __grid_constant__ CUtensorMap tm_keys, const __grid_constant__ CUtensorMap tm_qi,
                       Args a) {
    // decode: key tiles that share one 128-column TMEM accumulator (Hi columns each)
    constexpr int kTPB = 128 / HI < 4 ? 128 / HI : 4;
    constexpr int kEpiWarps = epi_warps(DEC), kEpiThreads = 32 * kEpiWarps, kGroups = kEpiWarps / 4;
    constexpr int NS = ring_stages(DEC, LP);
    constexpr int BT = DEC ? kBTileDec : kBTile;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = base;                       // NS x 16 KB
    uint8_t *sB = sA + NS * kATile;           // 2 x BT
    float *sw = reinterpret_cast<float *>(sB + 2 * BT);   // prefill: 2 x 256 head weights
    uint8_t *sK8 = reinterpret_cast<uint8_t *>(sw + (DEC ? 0 : 512));   // FP4 keys: NS x 4 KB of staged codes
    uint64_t *bars = reinterpret_cast<uint64_t *>(sK8 + (LP ? NS * kCodeTile : 0));
    uint64_t *a_full = bars, *a_empty = bars + NS, *b_full = bars + 2 * NS, *b_empty = b_full + 2;
    uint64_t *acc_full = b_empty + 2, *acc_empty = acc_full + 4;
    uint64_t *c_full = acc_empty + 4;         // FP4 keys: codes of stage s landed
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(c_full + (LP ? NS : 0));
    uint32_t *shist = tmem_slot + 4;          // decode: [4096] key-bit histogram of the current unit

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; ++i) {
            tc::mbar_init(&a_full[i], LP ? conv_warps(DEC) : 1);
            tc::mbar_init(&a_empty[i], 1);
            if (LP) tc::mbar_init(&c_full[i], 1);
        }
        for (int i = 0; i < 2; ++i) { tc::mbar_init(&b_full[i], 1); tc::mbar_init(&b_empty[i], 1); }
        for (int i = 0; i < 4; ++i) { tc::mbar_init(&acc_full[i], 1); tc::mbar_init(&acc_empty[i], kEpiThreads / 32); }
        tc::fence_mbar_init();
    }
    constexpr uint32_t kTmemCols = DEC ? 256 : 512;
    if (warp == 0) tc::tmem_alloc(tmem_slot, kTmemCols);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t ia = 0, ib = 0;
            Unit x;
            for (Iter it = iter_begin(a); ok && iter_next(a, it, x);) {
                const int bb = ib & 1;
                if (ib >= 2) ok = ok && tc::mbar_wait(&b_empty[bb], ((ib >> 1) - 1) & 1, a.status);
                tc::mbar_arrive_expect_tx(&b_full[bb], a.ncols * 128);
                tc::tma_load_3d(tc::smem_u32(sB + bb * BT), &tm_qi, 0, 0, (int)x.r0, &b_full[bb]);
                ++ib;
                for (int kt = x.kt0; kt < x.kt1 && ok; ++kt, ++ia) {
                    const int s = ia % NS;
                    if (ia >= NS) ok = ok && tc::mbar_wait(&a_empty[s], ((ia / NS) - 1) & 1, a.status);
                    if (!ok) break;
                    if (LP) {
                        // the tile's codes: 128 consecutive key rows, cut at the end of the array
                        const int64_t r0 = x.b * a.N + (int64_t)kt * 128;
                        const int64_t nr = a.key_rows - r0 < 128 ? a.key_rows - r0 : 128;
                        tc::mbar_arrive_expect_tx(&c_full[s], (uint32_t)nr * 32);
                        tc::bulk_load(tc::smem_u32(sK8 + s * kCodeTile), a.codes + r0 * 32, (uint32_t)nr * 32,
                                      &c_full[s]);
                    } else {
                        tc::mbar_arrive_expect_tx(&a_full[s], kATile);
                        tc::tma_load_3d(tc::smem_u32(sA + s * kATile), &tm_keys, 0, kt * 128, (int)x.b, &a_full[s]);
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = tc::idesc_bf16(128, a.ncols, false, false);
            uint32_t ia = 0, ib = 0, iacc = 0;
            Unit x;
            for (Iter it = iter_begin(a); ok && iter_next(a, it, x);) {
                const int bb = ib & 1;
                ok = ok && tc::mbar_wait(&b_full[bb], (ib >> 1) & 1, a.status);
                const uint32_t bsm = tc::smem_u32(sB + bb * BT);
                if (DEC) {
                    // Decode: kTPB consecutive tiles share one accumulator (HI columns each).  Every tile is a
                    // chain of 4 dependent MMAs (K = 16 each) whose latency, not the tensor pipe, sets the pace,
                    // so the K steps of two tiles are interleaved (two independent chains in flight).
                    for (int kt = x.kt0; kt < x.kt1 && ok; kt += 2, ia += 2) {
                        const int slot = (kt - x.kt0) % kTPB;
                        const bool two = kt + 1 < x.kt1;   // pairs start at even slots: both in one accumulator
                        const int s0 = ia % NS, s1 = (ia + 1) % NS, ab = iacc % a.nbuf;
                        ok = ok && tc::mbar_wait(&a_full[s0], (ia / NS) & 1, a.status);
                        if (two) ok = ok && tc::mbar_wait(&a_full[s1], ((ia + 1) / NS) & 1, a.status);
                        if (LP) tc::fence_async_smem();   // converter writes (generic proxy) -> MMA
                        if (slot == 0 && iacc >= (uint32_t)a.nbuf)
                            ok = ok && tc::mbar_wait(&acc_empty[ab], ((iacc / a.nbuf) - 1) & 1, a.status);
                        tc::tc_fence_after();
                        const uint32_t a0 = tc::smem_u32(sA + s0 * kATile), a1 = tc::smem_u32(sA + s1 * kATile);
                        const uint32_t d0 = tmem + ab * a.stride + slot * HI;
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint64_t bd = tc::sdesc_sw128(bsm + 32 * k, 16, 1024);
                            tc::mma_bf16(d0, tc::sdesc_sw128(a0 + 32 * k, 16, 1024), bd, idesc, k > 0);
                            if (two) tc::mma_bf16(d0 + HI, tc::sdesc_sw128(a1 + 32 * k, 16, 1024), bd, idesc, k > 0);
                        }
                        tc::mma_commit(&a_empty[s0]);
                        if (two) tc::mma_commit(&a_empty[s1]);
                        const int last = kt + (two ? 1 : 0);
                        if ((slot + (two ? 1 : 0)) == kTPB - 1 || last == x.kt1 - 1) {
                            tc::mma_commit(&acc_full[ab]);
                            ++iacc;
                        }
                    }
                    if (!ok) break;
                    ia -= (uint32_t)((x.kt1 - x.kt0) & 1);   // an odd tile count used one stage, not two
                    tc::mma_commit(&b_empty[bb]);
                    ++ib;
                    continue;
                }
                for (int kt = x.kt0; kt < x.kt1 && ok; ++kt, ++ia) {
                    const int s = ia % NS, ab = iacc % a.nbuf;
                    ok = ok && tc::mbar_wait(&a_full[s], (ia / NS) & 1, a.status);
                    if (LP) tc::fence_async_smem();   // converter writes (generic proxy) -> MMA
                    if (iacc >= (uint32_t)a.nbuf)
                        ok = ok && tc::mbar_wait(&acc_empty[ab], ((iacc / a.nbuf) - 1) & 1, a.status);
                    tc::tc_fence_after();
                    const uint32_t asm_ = tc::smem_u32(sA + s * kATile);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        tc::mma_bf16(tmem + ab * a.stride, tc::sdesc_sw128(asm_ + 32 * k, 16, 1024),
                                     tc::sdesc_sw128(bsm + 32 * k, 16, 1024), idesc, k > 0);
                    tc::mma_commit(&a_empty[s]);
                    tc::mma_commit(&acc_full[ab]);
                    ++iacc;
                }
                tc::mma_commit(&b_empty[bb]);
                ++ib;
            }
        }
    } else if (LP && warp >= 2 + kEpiWarps) {
        // ------------------------------------------------ FP4 keys: staged codes -> bf16 operand tile
        // One key row per thread: 32 code bytes (64 E2M1 values) and the row's two block exponents become
        // the row's 128-byte swizzled bf16 line (exact: every stored key is a bf16 number).
        constexpr int kConvThreads = 32 * conv_warps(DEC);
        const int ct = threadIdx.x - 32 * (2 + kEpiWarps);   // 0 .. kConvThreads - 1
        uint32_t ia = 0;
        Unit x;
        for (Iter it = iter_begin(a); ok && iter_next(a, it, x);) {
            for (int kt = x.kt0; kt < x.kt1 && ok; ++kt, ++ia) {
                const int s = ia % NS;
                ok = ok && tc::mbar_wait(&c_full[s], (ia / NS) & 1, a.status);
                if (!ok) break;
                uint8_t *dst = sA + s * kATile;
#pragma unroll
                for (int kr = ct; kr < 128; kr += kConvThreads) {   // key row of the tile
                    const int64_t row = x.b * a.N + (int64_t)kt * 128 + kr;
                    int e0 = 0, e1 = 0;
                    if (row < a.key_rows) {
                        e0 = a.kexp[row * 2];
                        e1 = a.kexp[row * 2 + 1];
                    }
                    const uint4 *src = reinterpret_cast<const uint4 *>(sK8 + s * kCodeTile + kr * 32);
                    const uint4 c01 = src[0], c23 = src[1];
                    const uint32_t cw[8] = {c01.x, c01.y, c01.z, c01.w, c23.x, c23.y, c23.z, c23.w};
                    const float s0 = lp::pow2f(e0), s1 = lp::pow2f(e1);
#pragma unroll
                    for (int g = 0; g < 8; ++g) {   // 16-byte chunk g = channels 8 g .. 8 g + 7
                        const uint4 v = lp::fp4x8_to_bf16x8(cw[g], g < 4 ? s0 : s1);
                        *reinterpret_cast<uint4 *>(dst + tc::sw128_offset((uint32_t)kr, (uint32_t)g)) = v;
                    }
                }
                tc::fence_async_smem();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&a_full[s]);
            }
        }
    } else if (DEC) {
        // ------------------------------------------------ decode epilogue: one token, Hi columns per tile
        // The two warp groups take alternate accumulators; each holds up to kTPB key tiles.
        const int quad = warp & 3, grp = (warp - 2) >> 2;   // group grp takes accumulators iacc % kGroups == grp
        const int row = quad * 32 + lane;
        const int et = threadIdx.x - 64;              // 0..kEpiThreads-1
        const bool hist = a.hist != nullptr;
        if (hist)
            for (int i = et; i < 4096; i += kEpiThreads) shist[i] = 0;
        uint32_t iacc = 0;
        Unit x;
        for (Iter it = iter_begin(a); iter_next(a, it, x);) {
            // with the histogram the epilogue warps meet at barriers: they leave the loop together
            if (hist) ok = tc::named_bar_and(1, kEpiThreads, ok);
            if (!ok) break;
            float wr[HI];
#pragma unroll
            for (int h = 0; h < HI; ++h) wr[h] = __bfloat162float(a.w[x.b * a.ld_w + h]);
            const int64_t vis = visible(a, x.b);
            float *srow = a.scores + x.b * a.N;
            const int nbat = (x.kt1 - x.kt0 + kTPB - 1) / kTPB;
            for (int bi = 0; bi < nbat && ok; ++bi, ++iacc) {
                if ((int)(iacc % kGroups) != grp) continue;
                const int ab = iacc % a.nbuf;
                ok = ok && tc::mbar_wait(&acc_full[ab], (iacc / a.nbuf) & 1, a.status);
                tc::tc_fence_after();
                const int kt0 = x.kt0 + bi * kTPB;
                const int nt = min(kTPB, x.kt1 - kt0);
                const uint32_t tl = tmem + ab * a.stride + ((uint32_t)(quad * 32) << 16);
                float sc[kTPB];
#pragma unroll
                for (int t = 0; t < kTPB; ++t) sc[t] = 0.f;
#pragma unroll
                for (int c0 = 0; c0 < kTPB * HI; c0 += 32) {   // 32 columns: part of a tile, or 32 / HI tiles
                    if (c0 / HI < nt) {
                        float v[32];
                        tc::tmem_ld32(tl + c0, v);
                        tc::tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 32; ++i) sc[(c0 + i) / HI] += wr[(c0 + i) % HI] * fmaxf(v[i], 0.f);
                    }
                }
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive_cnt(&acc_empty[ab], kGroups);
#pragma unroll
                for (int t = 0; t < kTPB; ++t) {
                    const int64_t j = (int64_t)(kt0 + t) * 128 + row;
                    if (t < nt && j < vis) {
                        srow[j] = sc[t];
                        if (hist) atomicAdd(&shist[score_order_key(sc[t]) >> 20], 1u);
                    }
                }
            }
            if (hist) {   // add the unit's counts into its row's histogram
                tc::named_bar_sync(1, kEpiThreads);
                uint32_t *g = a.hist + x.b * 4096;
                for (int i = et; i < 4096; i += kEpiThreads) {
                    const uint32_t c = shist[i];
                    if (c) {
                        atomicAdd(&g[i], c);
                        shist[i] = 0;
                    }
                }
            }
        }
    } else {
        // ------------------------------------------------ epilogue: ReLU, head weights, head sum
        // The four warp groups split the 256 columns of every tile (64 each).
        const int et = threadIdx.x - 64;              // 0..kEpiThreads-1
        const int quad = warp & 3, grp = (warp - 2) >> 2;
        const int row = quad * 32 + lane;             // key within the tile (TMEM lane)
        constexpr int TPH = 64 / HI > 0 ? 64 / HI : 1;      // tokens per 64 columns
        const int tok_base = grp * TPH;
        const int col_base = grp * 64;
        uint32_t iacc = 0, iu = 0;
        Unit x;
        for (Iter it = iter_begin(a); iter_next(a, it, x);) {
            float *w_s = sw + (iu & 1) * 256;
            if (et < a.ncols) {
                const int64_t r = x.r0 + et / HI;
                w_s[et] = r < a.rows ? __bfloat162float(a.w[r * a.ld_w + et % HI]) : 0.f;
            }
            ok = tc::named_bar_and(1, kEpiThreads, ok);   // all epilogue warps leave together on a failed wait
            if (!ok) break;
            ++iu;
            const int ntok = a.ncols / HI;                       // tokens in the unit
            int64_t vis[TPH];
#pragma unroll
            for (int i = 0; i < TPH; ++i) {
                const int64_t r = x.r0 + tok_base + i;
                vis[i] = (tok_base + i < ntok && r < a.rows) ? visible(a, r) : 0;
            }
            // per token, the four largest order keys this thread sees (one key per tile: its TMEM lane)
            uint32_t t4[TPH][4];
#pragma unroll
            for (int i = 0; i < TPH; ++i)
#pragma unroll
                for (int q = 0; q < 4; ++q) t4[i][q] = 0u;
            for (int kt = x.kt0; kt < x.kt1 && ok; ++kt, ++iacc) {
                const int ab = iacc % a.nbuf;
                ok = ok && tc::mbar_wait(&acc_full[ab], (iacc / a.nbuf) & 1, a.status);
                tc::tc_fence_after();
                // two partial sums per token, updated by packed FMAs (even / odd head of each pair)
                float s[TPH], s1[TPH];
#pragma unroll
                for (int i = 0; i < TPH; ++i) { s[i] = 0.f; s1[i] = 0.f; }
                const uint32_t tl = tmem + ab * a.stride + ((uint32_t)(quad * 32) << 16);
                // the head weights are read as float4 (the same address in every lane: a broadcast)
                constexpr int LB = 1;
#pragma unroll
                for (int c0 = 0; c0 < 2; c0 += LB) {
                    float v[LB][32];
#pragma unroll
                    for (int l = 0; l < LB; ++l) tc::tmem_ld32(tl + col_base + (c0 + l) * 32, v[l]);
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int l = 0; l < LB; ++l) {
                        const float4 *wv = reinterpret_cast<const float4 *>(w_s + col_base + (c0 + l) * 32);
#pragma unroll
                        for (int i4 = 0; i4 < 8; ++i4) {
                            const float4 wq = wv[i4];
                            const float wl[4] = {wq.x, wq.y, wq.z, wq.w};
#pragma unroll
                            for (int e = 0; e < 4; e += 2) {
                                const int c = (c0 + l) * 32 + i4 * 4 + e;   // column within this group's 64
                                const int ti = c / HI < TPH ? c / HI : TPH - 1;   // c, c + 1: the same token
                                fma2(s[ti], s1[ti], wl[e], wl[e + 1], fmaxf(v[l][i4 * 4 + e], 0.f),
                                     fmaxf(v[l][i4 * 4 + e + 1], 0.f));
                            }
                        }
                    }
                }
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&acc_empty[ab]);
#pragma unroll
                for (int i = 0; i < TPH; ++i) s[i] += s1[i];
                const int64_t j = (int64_t)kt * 128 + row;
#pragma unroll
                for (int i = 0; i < TPH; ++i)
                    if (j < vis[i]) {
                        a.scores[(x.r0 + tok_base + i) * a.N + j] = s[i];
                        uint32_t key = score_order_key(s[i]);
                        if (key > t4[i][3]) {   // insert into the descending top four
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const uint32_t hi = max(t4[i][q], key), lo = min(t4[i][q], key);
                                t4[i][q] = hi;
                                key = lo;
                            }
                        }
                    }
            }
            if (a.bound) {
                // The 128 threads of this group saw every score of its tokens, four best each: at least 512
                // scores reach the smallest of their fourth-best keys, a lower bound of the k-th best (k <= 512).
                uint32_t *gmin = reinterpret_cast<uint32_t *>(tmem_slot + 4) + grp * 32;   // [token][quadrant]
#pragma unroll
                for (int i = 0; i < TPH; ++i) {
                    const uint32_t wm = __reduce_min_sync(0xffffffffu, t4[i][3]);
                    if (lane == 0) gmin[i * 4 + quad] = wm;
                }
                tc::named_bar_sync(2 + grp, 128);
                if (quad == 0 && lane < TPH) {
                    const int64_t r = x.r0 + tok_base + lane;
                    if (tok_base + lane < ntok && r < a.rows) {
                        const uint32_t *gm = gmin + lane * 4;
                        a.bound[r] = min(min(gm[0], gm[1]), min(gm[2], gm[3]));
                    }
                }
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

// ------------------------------------------------------------------ register-resident top-k
constexpr int kTkThreads = 512;
constexpr int kRankCap = 1024;   // threshold buckets up to this size are ranked directly
constexpr int kCandCap = 4096;   // bound path: candidates of a row held in shared memory


template <int VPT>   // float4 vectors per thread: row capacity = 2048 * VPT
__global__ void __launch_bounds__(kTkThreads, VPT <= 4 ? 2 : 1) topk_regs_kernel(const float *__restrict__ scores, int64_t row0,
                                                               int64_t rows,
                                                               int64_t N, int m, const int32_t *__restrict__ pos,
                                                               int topk, int32_t *__restrict__ sel,
                                                               const int32_t *__restrict__ flags) {
    using Scan = cub::BlockScan<int, kTkThreads>;
    __shared__ typename Scan::TempStorage scan_tmp;
    // histogram path: hist[4096] and cand[kRankCap]; bound path: the same bytes hold ckey[kCandCap] and
    // cj[kCandCap] (a row takes one path or the other)
    __shared__ __align__(16) uint8_t pool[4096 * sizeof(int) + kRankCap * sizeof(uint64_t)];
    int *hist = reinterpret_cast<int *>(pool);
    uint64_t *cand = reinterpret_cast<uint64_t *>(pool + 4096 * sizeof(int));  // (key << 32 | ~index)
    uint32_t *ckey = reinterpret_cast<uint32_t *>(pool);
    uint16_t *cj = reinterpret_cast<uint16_t *>(pool + kCandCap * sizeof(uint32_t));
    __shared__ uint32_t bitmap[1024];   // rows of up to 32768 entries
    __shared__ uint32_t eq_idx[64];
    __shared__ uint32_t s_red[64];      // per-warp partials (two alternating sets of 16, then min / max)
    __shared__ uint32_t s_prefix;
    __shared__ int s_rem, s_eq_total, s_bcount, s_cnt;
    const int tid = threadIdx.x;
    const bool vec_ok = (N & 3) == 0 && ((uintptr_t)scores & 15) == 0;   // rows start 16-byte aligned
    auto visible_of = [&](int64_t rr) -> int64_t {
        const int64_t pp = pos ? (int64_t)pos[rr] : rr;
        return pp < 0 ? 0 : (pp / m < N ? pp / m : N);
    };
    // Persistent CTAs walk the rows round-robin (every CTA sees short and long rows).  While a row is
    // ranked, the CTA's next row is prefetched into L2: loading a row is otherwise a bare HBM round trip
    // with nothing else to do.
    for (int64_t r = row0 + blockIdx.x; r < rows; r += gridDim.x) {
    if (flags && flags[r] == 0) continue;   // only the rows the warp kernel left to this one
    if (tid == 0 && vec_ok && !flags && r + gridDim.x < rows) {
        const int64_t nn = visible_of(r + gridDim.x);
        const uint8_t *src = reinterpret_cast<const uint8_t *>(scores + (r + gridDim.x) * N);
        const uint32_t bytes = (uint32_t)(((nn + 3) & ~int64_t(3)) * sizeof(float));
        for (uint32_t off = 0; off < bytes; off += 65536u)
            tc::bulk_prefetch_l2(src + off, bytes - off < 65536u ? bytes - off : 65536u);
    }
    const int64_t n = visible_of(r);
    int32_t *out = sel + r * topk;
    if (n <= topk) {
        for (int i = tid; i < topk; i += kTkThreads) out[i] = i < n ? i : -1;
        continue;
    }
    const float *row = scores + r * N;
    uint32_t key[VPT * 4];
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int64_t j0 = 4 * ((int64_t)tid + (int64_t)kTkThreads * i);
        if (vec_ok && j0 + 3 < n) {
            float4 v = __ldcs(reinterpret_cast<const float4 *>(row + j0));
            key[4 * i] = score_order_key(v.x); key[4 * i + 1] = score_order_key(v.y);
            key[4 * i + 2] = score_order_key(v.z); key[4 * i + 3] = score_order_key(v.w);
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) key[4 * i + e] = (j0 + e < n) ? score_order_key(row[j0 + e]) : 0u;
        }
    }
    const int nw = (int)((n + 31) / 32);
    const int lane = tid & 31, warp = tid >> 5;
    bool marked = false;
    // Bound path.  Every thread's largest key is at least tau0, the smallest of those maxima, so at least
    // kTkThreads >= k keys reach tau0 and the k best lie among the keys >= tau0 (a few per thread for random
    // scores).  They are gathered in shared memory and selected exactly: the k-th largest key bit by bit
    // from the top (a bit stays set while at least k candidates reach the prefix; the search stops when
    // exactly k do), then the lowest entry indices among the keys equal to it.
    if (topk <= kTkThreads && n >= 4 * kTkThreads) {   // k <= threads, and every thread holds a visible key
        uint32_t mymax = 0;
#pragma unroll
        for (int i = 0; i < VPT * 4; ++i) mymax = max(mymax, key[i]);
        const uint32_t wmin = __reduce_min_sync(0xffffffffu, mymax), wmax = __reduce_max_sync(0xffffffffu, mymax);
        if (lane == 0) { s_red[32 + warp] = wmin; s_red[48 + warp] = wmax; }
        __syncthreads();
        uint32_t tau0 = s_red[32], kmax = s_red[48];
#pragma unroll
        for (int w = 1; w < kTkThreads / 32; ++w) { tau0 = min(tau0, s_red[32 + w]); kmax = max(kmax, s_red[48 + w]); }
        int c = 0;
#pragma unroll
        for (int i = 0; i < VPT * 4; ++i) c += key[i] >= tau0 ? 1 : 0;
        int off, total;
        Scan(scan_tmp).ExclusiveSum(c, off, total);
        if (total <= kCandCap) {
#pragma unroll
            for (int i = 0; i < VPT; ++i)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (key[4 * i + e] >= tau0) {
                        ckey[off] = key[4 * i + e];
                        cj[off] = (uint16_t)(4 * (tid + kTkThreads * i) + e);
                        ++off;
                    }
            __syncthreads();
            constexpr int CPT = kCandCap / kTkThreads;   // candidates per thread
            uint32_t ck[CPT];
#pragma unroll
            for (int i = 0; i < CPT; ++i) {
                const int q = tid + kTkThreads * i;
                ck[i] = q < total ? ckey[q] : 0u;
            }
            int sset = 0;
            auto block_sum = [&](uint32_t v) -> uint32_t {
                v = __reduce_add_sync(0xffffffffu, v);
                if (lane == 0) s_red[sset * 16 + warp] = v;
                __syncthreads();
                uint32_t t = 0;
#pragma unroll
                for (int w = 0; w < kTkThreads / 32; ++w) t += s_red[sset * 16 + w];
                sset ^= 1;
                return t;
            };
            const uint32_t k = (uint32_t)topk;
            const int top = kmax == tau0 ? -1 : 31 - __clz(kmax ^ tau0);
            uint32_t prefix = top < 0 ? kmax : top >= 31 ? 0u : kmax & ~((2u << top) - 1u);
            bool exact = false;
            for (int bb = top; bb >= 0; --bb) {
                const uint32_t cut = prefix | (1u << bb);
                uint32_t cc = 0;
#pragma unroll
                for (int i = 0; i < CPT; ++i) cc += ck[i] >= cut ? 1u : 0u;
                const uint32_t tot = block_sum(cc);
                if (tot >= k) prefix = cut;
                if (tot == k) { exact = true; break; }
            }
            const uint32_t tau = prefix;
            uint32_t takem = 0;   // bit i: candidate tid + kTkThreads i is taken
            if (exact) {
#pragma unroll
                for (int i = 0; i < CPT; ++i) takem |= (ck[i] >= tau ? 1u : 0u) << i;
            } else {
                uint32_t gtm = 0, eqm = 0;
#pragma unroll
                for (int i = 0; i < CPT; ++i) {
                    gtm |= (ck[i] > tau ? 1u : 0u) << i;
                    eqm |= (ck[i] == tau ? 1u : 0u) << i;
                }
                const uint32_t n_gt = block_sum(__popc(gtm));
                const uint32_t n_eq = block_sum(__popc(eqm));
                const uint32_t rem = k - n_gt;
                uint32_t tm = eqm;
                if (n_eq > rem) {
                    // the rem lowest entry indices among the ties: the rem largest 32767 - j, bit by bit
                    uint32_t rk[CPT];
#pragma unroll
                    for (int i = 0; i < CPT; ++i)
                        rk[i] = (eqm >> i & 1u) ? 32768u + 32767u - (uint32_t)cj[tid + kTkThreads * i] : 0u;
                    uint32_t pj = 32768u;
                    for (int bb = 14; bb >= 0; --bb) {
                        const uint32_t cut = pj | (1u << bb);
                        uint32_t cc = 0;
#pragma unroll
                        for (int i = 0; i < CPT; ++i) cc += rk[i] >= cut ? 1u : 0u;
                        if (block_sum(cc) >= rem) pj = cut;
                    }
                    tm = 0;
#pragma unroll
                    for (int i = 0; i < CPT; ++i) tm |= (rk[i] >= pj ? 1u : 0u) << i;
                }
                takem = gtm | tm;
            }
            for (int i = tid; i < nw; i += kTkThreads) bitmap[i] = 0;
            __syncthreads();
#pragma unroll
            for (int i = 0; i < CPT; ++i)
                if (takem >> i & 1u) {
                    const uint32_t j = cj[tid + kTkThreads * i];
                    atomicOr(&bitmap[j >> 5], 1u << (j & 31));
                }
            marked = true;
        } else {
            __syncthreads();   // the scan storage is used again below
        }
    }
    if (!marked) {
        // Histogram passes over bits [20,32), then [10,20) and [0,10) inside the threshold bucket.  Usually
        // the first pass leaves a small bucket: its keys are then ranked directly instead (the two later
        // passes cost more in barriers than in work).
        uint32_t prefix = 0, mask = 0;
        int rem = topk;
        bool ranked = false;
        const int shifts[3] = {20, 10, 0};
        const int widths[3] = {12, 10, 10};
    #pragma unroll
        for (int pass = 0; pass < 3; ++pass) {
            const int sh = shifts[pass], nb = 1 << widths[pass];
            for (int i = tid; i < nb; i += kTkThreads) hist[i] = 0;
            __syncthreads();
    #pragma unroll
            for (int i = 0; i < VPT * 4; ++i)
                if ((key[i] & mask) == prefix && key[i] != 0u) atomicAdd(&hist[(key[i] >> sh) & (nb - 1)], 1);
            __syncthreads();
            // suffix scan: thread tid owns bins [(nb/512) * (511 - tid), ...) so thread 0 holds the highest bins
            const int per = nb / kTkThreads;
            const int b0 = per * (kTkThreads - 1 - tid);
            int local = 0;
            for (int i = 0; i < per; ++i) local += hist[b0 + i];
            int above, total;
            Scan(scan_tmp).ExclusiveSum(local, above, total);
            if (above < rem && above + local >= rem) {
                int cum = above;
                for (int i = per - 1; i >= 0; --i) {
                    const int c = hist[b0 + i];
                    if (cum + c >= rem) {
                        s_prefix = prefix | ((uint32_t)(b0 + i) << sh);
                        s_rem = rem - cum;
                        s_bcount = c;
                        break;
                    }
                    cum += c;
                }
            }
            __syncthreads();
            prefix = s_prefix;
            rem = s_rem;
            mask |= (uint32_t)(nb - 1) << sh;
            const bool small = s_bcount <= kRankCap;
            __syncthreads();
            if (pass == 0 && small) {
                ranked = true;
                break;
            }
        }
        for (int i = tid; i < nw; i += kTkThreads) bitmap[i] = 0;
        if (tid == 0) {
            s_eq_total = 0;
            s_cnt = 0;
        }
        __syncthreads();
        if (ranked) {
            // prefix = threshold bucket << 20: keys in higher buckets are taken; the `rem` best keys of the
            // bucket (larger key first, then lower index) are found by ranking the bucket's keys
            const uint32_t bucket = prefix >> 20;
    #pragma unroll
            for (int i = 0; i < VPT; ++i) {
    #pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const uint32_t kv = key[4 * i + e];
                    const int64_t j = 4 * ((int64_t)tid + (int64_t)kTkThreads * i) + e;
                    if ((kv >> 20) > bucket) {
                        atomicOr(&bitmap[j >> 5], 1u << (j & 31));
                    } else if ((kv >> 20) == bucket && kv != 0u) {
                        const int q = atomicAdd(&s_cnt, 1);
                        if (q < kRankCap) cand[q] = ((uint64_t)kv << 32) | (0xFFFFFFFFu - (uint32_t)j);
                    }
                }
            }
            __syncthreads();
            const int mb = s_cnt < kRankCap ? s_cnt : kRankCap;
            for (int c = tid; c < mb; c += kTkThreads) {
                const uint64_t v = cand[c];
                int rk = 0;
                for (int d = 0; d < mb; ++d) rk += cand[d] > v ? 1 : 0;
                if (rk < rem) {
                    const uint32_t j = 0xFFFFFFFFu - (uint32_t)v;
                    atomicOr(&bitmap[j >> 5], 1u << (j & 31));
                }
            }
        } else {
        // prefix = k-th largest key; rem = keys equal to it that are taken (lowest j first).
        // Mark the chosen indices in a bitmap of the row, then emit them in ascending order with one scan.
    #pragma unroll
        for (int i = 0; i < VPT; ++i) {
    #pragma unroll
            for (int e = 0; e < 4; ++e) {
                const uint32_t kv = key[4 * i + e];
                const int64_t j = 4 * ((int64_t)tid + (int64_t)kTkThreads * i) + e;
                if (kv > prefix) atomicOr(&bitmap[j >> 5], 1u << (j & 31));
                else if (kv == prefix && kv != 0u) {
                    const int q = atomicAdd(&s_eq_total, 1);
                    if (q < 64) eq_idx[q] = (uint32_t)j;
                }
            }
        }
        __syncthreads();
        if (s_eq_total > 64) {
            // many equal keys at the threshold: mark the lowest `rem` of them by scanning the row in order
            if (tid < 32) {
                int taken = 0;
                for (int64_t base = 0; base < n && taken < rem; base += 32) {
                    const int64_t j = base + tid;
                    bool eq = false;
                    if (j < n) eq = score_order_key(row[j]) == prefix;
                    const uint32_t m = __ballot_sync(0xffffffffu, eq);
                    const int before = __popc(m & ((1u << tid) - 1u));
                    if (eq && taken + before < rem) atomicOr(&bitmap[j >> 5], 1u << (j & 31));
                    taken += __popc(m);
                }
            }
        } else if (tid == 0) {
            const int ne = s_eq_total;
            for (int t = 0; t < rem && t < ne; ++t) {   // repeated minimum over the few equal keys
                int best = t;
                for (int q = t + 1; q < ne; ++q)
                    if (eq_idx[q] < eq_idx[best]) best = q;
                const uint32_t tmp = eq_idx[t];
                eq_idx[t] = eq_idx[best];
                eq_idx[best] = tmp;
                atomicOr(&bitmap[eq_idx[t] >> 5], 1u << (eq_idx[t] & 31));
            }
        }
        }
    }
    __syncthreads();
    const int per = (nw + kTkThreads - 1) / kTkThreads;
    const int w0 = tid * per;
    int local = 0;
    for (int w = w0; w < w0 + per && w < nw; ++w) local += __popc(bitmap[w]);
    int slot, total;
    Scan(scan_tmp).ExclusiveSum(local, slot, total);
    for (int w = w0; w < w0 + per && w < nw; ++w) {
        uint32_t bits = bitmap[w];
        while (bits) {
            const int bpos = __ffs(bits) - 1;
            bits &= bits - 1;
            if (slot < topk) out[slot] = w * 32 + bpos;
            ++slot;
        }
    }
    __syncthreads();   // shared state is reused by the next row
    }
}

// ------------------------------------------------------------------ warp-per-row top-k over a bounded row
// Prefill rows whose scores' lower bound (indexer epilogue) is known: one warp per row reads the row
// once and keeps the keys at or above the bound (a few percent of the row) in shared memory, then
// selects the k best exactly: the k-th largest key bit by bit from the top (the search stops when exactly
// k candidates reach the prefix), ties to the lowest entry indices, which are emitted in ascending order
// through a bitmap of the row.  A row with more than kWCap candidates is flagged for the block kernel.
constexpr int kWCap = 2048;          // candidates per row
constexpr int kWarpsPerCta = 12;
struct WarpTopk {
    uint32_t key[kWCap];
    uint16_t j[kWCap];
    uint32_t bitmap[1024];           // rows of up to 32768 entries
};
constexpr size_t kWarpTopkSmem = kWarpsPerCta * sizeof(WarpTopk);

__global__ void __launch_bounds__(32 * kWarpsPerCta) topk_warp_kernel(const float *__restrict__ scores, int64_t row0,
                                                                     int64_t rows, int64_t N, int m, int topk,
                                                                     const uint32_t *__restrict__ bound,
                                                                     int32_t *__restrict__ flags,
                                                                     int32_t *__restrict__ sel) {
    extern __shared__ __align__(16) uint8_t wsm[];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    WarpTopk &S = reinterpret_cast<WarpTopk *>(wsm)[w];
    const bool vec_ok = (N & 3) == 0 && ((uintptr_t)scores & 15) == 0;
    const int64_t nwarps = (int64_t)gridDim.x * kWarpsPerCta;
    const uint32_t k = (uint32_t)topk;
    for (int64_t r = row0 + (int64_t)blockIdx.x * kWarpsPerCta + w; r < rows; r += nwarps) {
        const int64_t n = r / m < N ? r / m : N;
        int32_t *out = sel + r * topk;
        if (n <= topk) {
            for (int c = lane; c < topk; c += 32) out[c] = c < n ? c : -1;
            if (lane == 0) flags[r] = 0;
            continue;
        }
        const uint32_t b = bound[r];
        const float *row = scores + r * N;
        uint32_t cnt = 0;
        // one pass over the row, 8 vectors of 4 scores per lane in flight
        for (int64_t base = 0; base < n; base += 32 * 4 * 8) {
            float4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int64_t j0 = base + 4 * (lane + 32 * u);
                if (vec_ok && j0 + 3 < n) {
                    v[u] = __ldcs(reinterpret_cast<const float4 *>(row + j0));
                } else {
                    v[u].x = j0 < n ? row[j0] : 0.f;
                    v[u].y = j0 + 1 < n ? row[j0 + 1] : 0.f;
                    v[u].z = j0 + 2 < n ? row[j0 + 2] : 0.f;
                    v[u].w = j0 + 3 < n ? row[j0 + 3] : 0.f;
                }
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int64_t j0 = base + 4 * (lane + 32 * u);
                const float f[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const uint32_t key = score_order_key(f[e]);
                    const bool take = j0 + e < n && key >= b;
                    const uint32_t bal = __ballot_sync(0xffffffffu, take);
                    const uint32_t q = cnt + __popc(bal & ((1u << lane) - 1u));
                    if (take && q < kWCap) {
                        S.key[q] = key;
                        S.j[q] = (uint16_t)(j0 + e);
                    }
                    cnt += __popc(bal);
                }
            }
        }
        if (cnt > kWCap || cnt < k) {   // too many candidates (or a bound that does not hold): block kernel
            if (lane == 0) flags[r] = 1;
            continue;
        }
        __syncwarp();
        constexpr int CPL = kWCap / 32;   // candidates per lane: c = lane + 32 i
        uint32_t ck[CPL];
        uint32_t kmax = 0;
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            const uint32_t c = lane + 32 * i;
            ck[i] = c < cnt ? S.key[c] : 0u;
            kmax = max(kmax, ck[i]);
        }
        kmax = __reduce_max_sync(0xffffffffu, kmax);
        const int top = kmax == b ? -1 : 31 - __clz(kmax ^ b);   // every candidate lies in [b, kmax]
        uint32_t prefix = top < 0 ? kmax : top >= 31 ? 0u : kmax & ~((2u << top) - 1u);
        bool exact = false;
        for (int bb = top; bb >= 0; --bb) {
            const uint32_t cut = prefix | (1u << bb);
            uint32_t cc = 0;
#pragma unroll
            for (int i = 0; i < CPL; ++i) cc += ck[i] >= cut ? 1u : 0u;
            const uint32_t tot = __reduce_add_sync(0xffffffffu, cc);
            if (tot >= k) prefix = cut;
            if (tot == k) { exact = true; break; }
        }
        const uint32_t tau = prefix;
        uint64_t takem = 0;   // bit i: candidate lane + 32 i is among the k best
        if (exact) {
#pragma unroll
            for (int i = 0; i < CPL; ++i) takem |= (uint64_t)(ck[i] >= tau ? 1u : 0u) << i;
        } else {
            uint64_t gtm = 0, eqm = 0;
            uint32_t ng = 0, ne = 0;
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                gtm |= (uint64_t)(ck[i] > tau ? 1u : 0u) << i;
                eqm |= (uint64_t)(ck[i] == tau ? 1u : 0u) << i;
            }
            ng = __reduce_add_sync(0xffffffffu, (uint32_t)__popcll(gtm));
            ne = __reduce_add_sync(0xffffffffu, (uint32_t)__popcll(eqm));
            const uint32_t rem = k - ng;
            uint64_t tm = eqm;
            if (ne > rem) {
                // the rem lowest entry indices among the ties: the rem largest 32767 - j, bit by bit
#pragma unroll
                for (int i = 0; i < CPL; ++i)
                    ck[i] = (eqm >> i & 1ull) ? 32768u + 32767u - (uint32_t)S.j[lane + 32 * i] : 0u;
                uint32_t pj = 32768u;
                for (int bb = 14; bb >= 0; --bb) {
                    const uint32_t cut = pj | (1u << bb);
                    uint32_t cc = 0;
#pragma unroll
                    for (int i = 0; i < CPL; ++i) cc += ck[i] >= cut ? 1u : 0u;
                    if (__reduce_add_sync(0xffffffffu, cc) >= rem) pj = cut;
                }
                tm = 0;
#pragma unroll
                for (int i = 0; i < CPL; ++i) tm |= (uint64_t)(ck[i] >= pj ? 1u : 0u) << i;
            }
            takem = gtm | tm;
        }
        const int nw = (int)((n + 31) / 32);
        for (int i = lane; i < nw; i += 32) S.bitmap[i] = 0;
        __syncwarp();
#pragma unroll
        for (int i = 0; i < CPL; ++i)
            if (takem >> i & 1ull) {
                const uint32_t jj = S.j[lane + 32 * i];
                atomicOr(&S.bitmap[jj >> 5], 1u << (jj & 31));
            }
        __syncwarp();
        const int per = (nw + 31) / 32, w0 = lane * per;
        uint32_t local = 0;
        for (int i = w0; i < w0 + per && i < nw; ++i) local += __popc(S.bitmap[i]);
        uint32_t incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        uint32_t pos = incl - local;
        for (int i = w0; i < w0 + per && i < nw; ++i) {
            uint32_t bits = S.bitmap[i];
            while (bits) {
                const int bp = __ffs(bits) - 1;
                bits &= bits - 1;
                if (pos < k) out[pos] = i * 32 + bp;
                ++pos;
            }
        }
        if (lane == 0) flags[r] = 0;
        __syncwarp();   // the warp's candidate list and bitmap are reused by its next row
    }
}

}  // namespace

bool index_tc_supported(const IndexArgs &a) {
    if (a.dtype != HCSA_BF16 || a.di != 64) return false;
    if (!(a.Hi == 8 || a.Hi == 16 || a.Hi == 32 || a.Hi == 64)) return false;
    if (a.pos && a.Hi < 16) return false;          // decode MMA N = Hi must be >= 16
    if (((uintptr_t)a.qi & 15) || ((uintptr_t)a.keys & 15) || (a.ld_qi * 2) % 16) return false;
    return a.N <= INT32_MAX && a.rows <= INT32_MAX;
}

static int num_sms() {
    static int n = 0;
    if (!n) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

template <int HI, bool DEC, bool LP>
static hcsa_status launch_scores(const IndexArgs &ia, const CUtensorMap &tk, const CUtensorMap &tq, Args a,
                                 cudaStream_t st) {
    constexpr int NS = ring_stages(DEC, LP);
    constexpr size_t smem = 1024 + NS * kATile + 2 * (DEC ? kBTileDec : kBTile) + (DEC ? 0 : 512 * sizeof(float)) +
                            (LP ? NS * kCodeTile : 0) + (3 * NS + 12) * sizeof(uint64_t) + 16 +
                            (DEC ? 4096 * sizeof(uint32_t) : 128 * sizeof(uint32_t));
    static_assert(smem <= 232448, "shared memory per CTA");
    static bool configured[64] = {};   // kernel attributes are set per device
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return HCSA_ERR_CUDA;
    if (!configured[dev]) {
        if (cudaFuncSetAttribute(index_scores_tc_kernel<HI, DEC, LP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem) != cudaSuccess)
            return HCSA_ERR_CUDA;
        configured[dev] = true;
    }
    const int64_t slots = (int64_t)num_sms() * (DEC ? kDecCtasPerSm : 1);
    const int64_t grid = a.n_units < slots ? a.n_units : slots;
    if (grid <= 0) return HCSA_OK;
    index_scores_tc_kernel<HI, DEC, LP><<<(unsigned)grid, cta_threads(DEC, LP), smem, st>>>(tk, tq, a);
    count_launch();
    return check_launch();
}

template <bool LP>
static hcsa_status dispatch_scores(const IndexArgs &ia, bool decode, const CUtensorMap &tk, const CUtensorMap &tq,
                                   const Args &a, cudaStream_t st) {
    if (decode) {
        switch (ia.Hi) {
            case 16: return launch_scores<16, true, LP>(ia, tk, tq, a, st);
            case 32: return launch_scores<32, true, LP>(ia, tk, tq, a, st);
            default: return launch_scores<64, true, LP>(ia, tk, tq, a, st);
        }
    }
    switch (ia.Hi) {
        case 8: return launch_scores<8, false, LP>(ia, tk, tq, a, st);
        case 16: return launch_scores<16, false, LP>(ia, tk, tq, a, st);
        case 32: return launch_scores<32, false, LP>(ia, tk, tq, a, st);
        default: return launch_scores<64, false, LP>(ia, tk, tq, a, st);
    }
}

hcsa_status launch_index_tc(const IndexArgs &ia, cudaStream_t st) {
    const bool decode = ia.pos != nullptr;
    const int64_t nseq = decode ? ia.rows : 1;
    const int tq = decode ? 1 : 256 / ia.Hi;
    CUtensorMap tk, tq_map;
    // prefill: keys end at the last entry the range's last query sees (the key tiles round up past it; those
    // rows read as zeros, so a row-range caller need not have gathered them)
    const int64_t last_vis = ia.row1 > 0 ? (ia.row1 - 1) / ia.m : 0;
    const uint64_t key_rows = decode ? (uint64_t)ia.N : (uint64_t)std::max<int64_t>(1, std::min<int64_t>(ia.N, last_vis));
    if (!make_tmap_bf16_3d(&tq_map, ia.qi, 64, (uint64_t)ia.Hi, (uint64_t)ia.rows, 128, (uint64_t)ia.ld_qi * 2, 64,
                           (uint32_t)ia.Hi, (uint32_t)tq, true))
        return HCSA_ERR_CUDA;
    if (ia.lowprec) {
        tk = tq_map;   // unused: FP4 key tiles are bulk copies of their code rows
    } else if (!make_tmap_bf16_3d(&tk, ia.keys, 64, key_rows, (uint64_t)nseq, 128, (uint64_t)ia.N * 128, 64, 128, 1,
                                  true)) {
        return HCSA_ERR_CUDA;
    }
    Args a{};
    a.rows = ia.rows; a.N = ia.N; a.m = ia.m; a.tq = tq; a.ncols = tq * ia.Hi; a.decode = decode; a.pos = ia.pos;
    a.nbuf = 2;                                   // prefill: 2 x 256 columns; decode: 2 x 128 columns
    a.stride = a.ncols <= 128 ? 128 : 256;
    a.w = (const __nv_bfloat16 *)ia.w; a.ld_w = ia.ld_w; a.scores = (float *)ia.ws; a.status = device_status_ptr();
    if (ia.lowprec) {
        // code rows [nseq * N][32], then their exponents; prefill loads stop at the range's last visible key
        a.codes = (const uint8_t *)ia.keys;
        a.kexp = (const int8_t *)(a.codes + nseq * ia.N * 32);
        a.key_rows = decode ? nseq * ia.N : (int64_t)key_rows;
    }
    // long decode rows: multi-CTA select, whose histogram the scores kernel fills; scratch after the scores
    const bool rows_path = ia.N > 32768 && topk_rows_supported(ia);
    uint8_t *scratch = (uint8_t *)ia.ws + (((size_t)ia.rows * ia.N * sizeof(float) + 255) & ~(size_t)255);
    a.hist = nullptr;
    a.bound = nullptr;
    if (!decode && ia.topk <= 512 && ia.N <= 32768 &&
        ia.ws_bytes >= index_topk_ws_bytes(ia.dtype, ia.rows, ia.N))   // bound + flags after the scores
        a.bound = reinterpret_cast<uint32_t *>(scratch);
    if (rows_path) {
        if (topk_rows_begin(ia, scratch, st) != HCSA_OK) return HCSA_ERR_CUDA;
        a.hist = reinterpret_cast<uint32_t *>(scratch);
    }
    if (decode) {
        a.tps = (ia.N + 127) / 128;
        a.n_units = ia.rows * a.tps;
        a.n_qtiles = 0;
    } else {
        // query tiles of the row range [row0, row1): tiles row0 / tq .. n_qtiles - 1, heaviest first
        a.n_qtiles = (ia.row1 + tq - 1) / tq;
        a.n_units = a.n_qtiles - ia.row0 / tq;
        a.tps = 0;
    }
    hcsa_status s = ia.lowprec ? dispatch_scores<true>(ia, decode, tk, tq_map, a, st)
                               : dispatch_scores<false>(ia, decode, tk, tq_map, a, st);
    if (s != HCSA_OK) return s;
    // top-k over the materialised scores
    const int64_t nrows = ia.row1 - ia.row0;
    if (nrows <= 0) return HCSA_OK;
    if (ia.N <= 32768) {
        const float *sc = (const float *)ia.ws;
        const int32_t *flags = nullptr;
        if (a.bound) {
            // warp per row over the bounded rows; the block kernel below takes only the rows it flags
            static bool configured_w[64] = {};
            int dev = 0;
            if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return HCSA_ERR_CUDA;
            if (!configured_w[dev]) {
                if (cudaFuncSetAttribute(topk_warp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kWarpTopkSmem) != cudaSuccess)
                    return HCSA_ERR_CUDA;
                configured_w[dev] = true;
            }
            int32_t *fl = reinterpret_cast<int32_t *>(a.bound + ia.rows);
            const int64_t need = (nrows + kWarpsPerCta - 1) / kWarpsPerCta;
            const int64_t g = need < num_sms() ? need : num_sms();
            topk_warp_kernel<<<(unsigned)g, 32 * kWarpsPerCta, kWarpTopkSmem, st>>>(sc, ia.row0, ia.row1, ia.N, ia.m,
                                                                                    ia.topk, a.bound, fl, ia.sel);
            count_launch();
            if (check_launch() != HCSA_OK) return HCSA_ERR_CUDA;
            flags = fl;
        }
        // persistent: as many CTAs as fit at once (one per SM at 16 vectors per thread, two at 4)
        if (ia.N <= 8192) {
            const int64_t g = nrows < 2 * num_sms() ? nrows : 2 * num_sms();
            topk_regs_kernel<4><<<(unsigned)g, kTkThreads, 0, st>>>(sc, ia.row0, ia.row1, ia.N, ia.m, ia.pos, ia.topk,
                                                                   ia.sel, flags);
        } else {
            const int64_t g = nrows < num_sms() ? nrows : num_sms();
            topk_regs_kernel<16><<<(unsigned)g, kTkThreads, 0, st>>>(sc, ia.row0, ia.row1, ia.N, ia.m, ia.pos, ia.topk,
                                                                    ia.sel, flags);
        }
        count_launch();
        return check_launch();
    }
    if (rows_path) {
        hcsa_status s2 = launch_topk_rows(ia, scratch, st);
        if (s2 != HCSA_OK) return s2;
        IndexArgs fb = ia;                       // rows flagged by the multi-CTA select
        fb.only_rows = topk_rows_flags(ia, scratch);
        return launch_topk_generic(fb, st);
    }
    return launch_topk_generic(ia, st);
}

}  // namespace hcsa

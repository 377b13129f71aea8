// MQA attention over compressed entries + the raw window on the 5th-generation tensor cores
// (tcgen05 + TMEM, TMA row gathers), for 64 heads of dh = 512 (C = 1024), bf16 storage.
//
// Operation ("DeepSeek-V4 ... KV cache compressed attention", sections "CSA", "HCA" and
// "Ventana deslizante", fixed by the CSA workload definition): the query of token t (or the
// new token of a decode sequence) attends, with every head sharing the keys, to the selected
// compressed entries (CSA) or to every visible entry (HCA) plus the raw tokens (t - 128, t];
// key = first C/2 channels of a row, value = last C/2; one softmax with scale tau.
//
// Work unit = (query, segment of its key list).  The key list is the entry part, padded to a
// multiple of 128 keys, followed by one 128-key window tile.  A unit holds at most 5 tiles
// (640 keys): prefill CSA is one unit per token (top-k 512 + window); decode splits every
// sequence into units of equal tile counts (the fewest that still fill one wave over the SMs)
// whose partials (accumulator, max, sum) are merged by the log-sum-exp combine kernel.
//
// Per unit, with 128 keys on the TMEM lanes and the 64 heads as the MMA's N:
//   S^T[key, head] = K . Q^T   tiles 0..3 in TMEM columns [0, 256), tile 4 in [256, 320)
//   exact softmax over all keys of the unit (per-head max / sum across lanes)
//   P^T (bf16) -> shared memory as an MN-major operand
//   O^T[dh, head] = V^T . P^T  4 blocks of 128 dh in columns [256, 512)
// Decode writes all of P^T, then runs P V.  Prefill writes P^T one tile at a time into two 16 KB slots,
// the window tile first (its score columns are the accumulator's), and P V of a tile starts as soon as
// that tile is written; the smaller P region leaves room for 10 ring stages instead of 6.
// Prefill streams Q in 64-dim chunks, each next to the key chunks of every tile (one pass over Q per
// unit), so the scores of the next unit accumulate while this unit's output drains; tile 4, whose
// columns the output accumulator reuses, starts once the drain is done.  Decode loads a unit's whole
// query at once into the P region, which is free until the softmax writes P.
//
// Warp roles (persistent CTAs, 16 warps): warps 0-6 load (gathered entry rows and the decode window
// ring with 16-byte cp.async whose completion arrives on the stage's mbarrier by itself; Q chunks and
// the prefill window tile -- 128 consecutive raw rows -- with TMA box loads), warp 7 issues the MMAs,
// warps 8..15 run the softmax and the output epilogue (two warps per TMEM lane quadrant, 32 heads
// each).  The producers' copy path bounds this kernel: without its MMAs, softmax arithmetic and output
// stores it keeps 82% of its time, and gathering from a few hot rows instead is no faster; its rate
// grows with the number of warps issuing the copies.
#include "lowprec.cuh"
#include "tc_common.cuh"

namespace hcsa {

namespace {

constexpr int kH = 64;
constexpr int kDh = 512;
constexpr int kC = 1024;
constexpr int kKT = 128;          // keys per tile (MMA M)
constexpr int kMaxTiles = 5;
// Key/value ring stages (even: P V pairs sit in adjacent stages).  Decode keeps all of P^T (and, until
// the softmax, the whole query) in one 80 KB region; prefill keeps two 16 KB P^T tile slots, which
// leaves room for 10 stages (6, 8 and 10 measured the same: the stage count is not what limits it).
constexpr int ring_stages(bool dec) { return dec ? 6 : 10; }
constexpr int kNSMax = 10;
constexpr int kStage = 16384;     // 128 rows x 64 bf16
constexpr int kGatherDepth = 4;   // gathered chunks in flight per producer thread
constexpr int kQStage = kH * 128; // 64 heads x 64 bf16
constexpr int p_bytes(bool dec) { return dec ? kMaxTiles * kKT * 128 : 2 * kKT * 128; }
// The gather rate of cp.async grows with the number of warps issuing it, so most of the CTA's warps are
// producers (the warps take 128 registers each either way).
constexpr int kProdWarps = 7;
constexpr int kProdThreads = 32 * kProdWarps;
constexpr int kMmaWarp = kProdWarps;
constexpr int kSoftWarp0 = kProdWarps + 1;   // 8 softmax/epilogue warps
constexpr int kThreads = 32 * (kProdWarps + 9);
constexpr int kSoftThreads = 256;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColB = 256;

constexpr uint32_t kIdescS = tc::idesc_bf16(128, kH, false, false);   // S^T = K . Q^T
constexpr uint32_t kIdescPV = tc::idesc_bf16(128, kH, true, true);    // O^T = V^T . P^T

struct Params {
    bool decode, dense;
    bool lowprec;                     // entries: E4M3 codes (ld C bytes), then int8 exponents (ld C / 32)
    const __nv_bfloat16 *ent, *raw;   // entry rows (ld C) and raw window rows
    const uint8_t *ent8;              // lowprec: code rows
    const int8_t *ent_exp;            // lowprec: exponent rows
    int64_t ld_raw;
    int64_t nq;          // queries (prefill T, decode B)
    int64_t N;           // entries per sequence (prefill ceil(T/m), decode n_cap)
    int m, topk, seg_tiles, nseg;
    int dq_split;        // decode: units per (query, segment), each taking 4 / dq_split of the 128-dh value blocks
    const int32_t *sel, *pos;
    float scale, scale_log2;
    __nv_bfloat16 *out;  // direct output [nq, H*dh] (nseg == 1)
    float *part;         // partials: acc [nq][nseg][H][dh], then (max, sum) [nq][nseg][H][2]
    int64_t n_units;
    int64_t q0;          // first query of the row range
    int64_t ent0;        // decode shard: global index of the cache's first entry
    bool no_window;      // decode shard: the raw window is attended by another shard
    int *status;
};

struct Unit {
    int64_t q, p, nvis;
    int seg, E, t0, nt;
    int dp0, dp1;        // value blocks [dp0, dp1) of 128 dh this unit accumulates and writes
};

__device__ __forceinline__ Unit unit_of(const Params &a, int64_t u) {
    Unit x;
    const int dq = (int)(u % a.dq_split);
    u /= a.dq_split;
    x.q = a.q0 + u / a.nseg;
    x.seg = (int)(u % a.nseg);
    x.dp0 = dq * (4 / a.dq_split);
    x.dp1 = x.dp0 + 4 / a.dq_split;
    x.p = a.decode ? (int64_t)a.pos[x.q] : x.q;
    {   // visible entries held here: global j < p / m, local j - ent0 in [0, N)
        int64_t v = x.p < 0 ? 0 : x.p / a.m - a.ent0;
        x.nvis = v < 0 ? 0 : (v < a.N ? v : a.N);
    }
    x.E = a.dense ? (int)((x.nvis + kKT - 1) / kKT) * kKT : a.topk;
    const int ntiles = x.E / kKT + 1;
    x.t0 = x.seg * a.seg_tiles;
    x.nt = ntiles - x.t0;
    x.nt = x.nt < 0 ? 0 : (x.nt > a.seg_tiles ? a.seg_tiles : x.nt);
    return x;
}

// Row of key kk (index into the query's key list) in the entry tensor (kk < E) or the raw tensor; -1 = masked.
__device__ __forceinline__ int key_row(const Params &a, const Unit &x, int kk) {
    if (kk < x.E) {
        const int64_t j = a.dense ? (int64_t)kk : (int64_t)a.sel[x.q * a.topk + kk];
        if (j < 0 || j >= x.nvis) return -1;
        return (int)(a.decode ? x.q * a.N + j : j);
    }
    const int64_t pp = x.p - (kKT - 1) + (kk - x.E);
    if (pp < 0 || a.no_window) return -1;
    return (int)(a.decode ? x.q * kKT + pp % kKT : pp);
}

__device__ __forceinline__ uint32_t s_col(int t) { return t < 4 ? (uint32_t)(t * kH) : kColB; }

// Tile of the i-th step of the P V phase.  Prefill hands P^T over tile by tile, and the first P V overwrites
// the output accumulator's columns, which hold tile 4's scores: so the last tile goes first there.
template <bool DEC>
__device__ __forceinline__ int pv_tile(int i, int nt) { return DEC ? i : (i == 0 ? nt - 1 : i - 1); }

template <bool kMax>
__device__ __forceinline__ float warp_transpose_reduce32(float *v, int lane) {
    // 32 values per lane -> lane l holds the warp-wide reduction of value l
#pragma unroll
    for (int o = 16, n = 16; o >= 1; o >>= 1, n >>= 1) {
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < n; ++i) {
            float send = upper ? v[i] : v[i + n];
            float keep = upper ? v[i + n] : v[i];
            float recv = __shfl_xor_sync(0xffffffffu, send, o);
            v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
        }
    }
    return v[0];
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ const __nv_bfloat16 *key_ptr(const Params &a, const Unit &x, int kk) {
    const int row = key_row(a, x, kk);
    if (row < 0) return nullptr;
    return kk < x.E ? a.ent + (int64_t)row * kC : a.raw + (int64_t)row * a.ld_raw;
}

struct Bars {
    uint64_t rf[kNSMax], re[kNSMax], qf[2], qe[2];
    uint64_t s_full, s_free, p_full, o_full, o_free, fin;
    uint64_t pt_full[2], pt_empty[2];   // prefill: P^T tile slots (written by the softmax, read by P V)
};

template <bool DEC>
__global__ void __launch_bounds__(kThreads, 1)
attend_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_ent,
                 const __grid_constant__ CUtensorMap tm_raw, Params a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int kNS = ring_stages(DEC);
    uint8_t *sP = base;                         // P^T: 640 rows x 128 B (decode), 2 x 128 rows x 128 B (prefill)
    uint8_t *sRing = sP + p_bytes(DEC);         // kNS x 16 KB
    uint8_t *sQ = sRing + kNS * kStage;         // 2 x 8 KB
    float *red = reinterpret_cast<float *>(sQ + 2 * kQStage);   // [4][64]
    float *mx = red + 4 * kH;                   // [64] scaled max
    float *zinv = mx + kH;                      // [64]
    float *znat = zinv + kH;                    // [64] sum
    float *mnat = znat + kH;                    // [64] max logit in natural units (-inf: no valid key)
    const __nv_bfloat16 **rowptr = reinterpret_cast<const __nv_bfloat16 **>(mnat + kH);   // [2][640]
    Bars *bars = reinterpret_cast<Bars *>(rowptr + 2 * kMaxTiles * kKT);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kNS; ++i) { tc::mbar_init(&bars->rf[i], kProdThreads); tc::mbar_init(&bars->re[i], 1); }
        for (int i = 0; i < 2; ++i) { tc::mbar_init(&bars->qf[i], 1); tc::mbar_init(&bars->qe[i], 1); }
        tc::mbar_init(&bars->s_full, 1);
        tc::mbar_init(&bars->o_full, 1);
        tc::mbar_init(&bars->s_free, kSoftThreads / 32);
        tc::mbar_init(&bars->p_full, kSoftThreads / 32);
        for (int i = 0; i < 2; ++i) { tc::mbar_init(&bars->pt_full[i], kSoftThreads / 32); tc::mbar_init(&bars->pt_empty[i], 1); }
        tc::mbar_init(&bars->o_free, kSoftThreads / 32);
        tc::mbar_init(&bars->fin, 1);
        tc::fence_mbar_init();
    }
    if (warp == 0) tc::tmem_alloc(tmem_slot, kTmemCols);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t P = tc::smem_u32(sP), ring = tc::smem_u32(sRing), Qs = tc::smem_u32(sQ);
    bool ok = true;

    if (warp < kProdThreads / 32) {
        // ------------------------------------------------ producers: cp.async gathers + TMA boxes
        const int pt = threadIdx.x;
        uint32_t ic = 0, iq = 0, iu = 0;
        int32_t tma_use[kNS + 2];                        // thread 0: last use index of a stage filled by TMA
        for (int i = 0; i < kNS + 2; ++i) tma_use[i] = -1;
        // After a failed wait no producer issues another copy; the producers leave the loop together at
        // the next per-unit barrier (an AND of their flags), so none is left waiting there.
        for (int64_t u = blockIdx.x; u < a.n_units; u += gridDim.x) {
            const Unit x = unit_of(a, u);
            if (x.nt <= 0) continue;
            if (a.decode && pt == 0 && ok) {
                // decode: the whole query (8 chunks of 64 dims) lands in the P region at once; P of the
                // previous unit must have been consumed by its P V first
                if (iu >= 1) ok = ok && tc::mbar_wait(&bars->o_full, (iu - 1) & 1, a.status);
                if (ok) {
                    tc::mbar_arrive_expect_tx(&bars->qf[0], 8 * kQStage);
                    for (int dc = 0; dc < 8; ++dc)
                        tc::tma_load_3d(P + dc * kQStage, &tm_q, dc * 64, 0, (int)x.q, &bars->qf[0]);
                    tma_use[kNS] = (int32_t)iu;
                }
            }
            const __nv_bfloat16 **rp = rowptr + (iu & 1) * (kMaxTiles * kKT);
            {
                // all selection indices of the unit are loaded before any is used (independent loads in flight)
                constexpr int kPer = (kMaxTiles * kKT + kProdThreads - 1) / kProdThreads;
                int32_t jsel[kPer];
#pragma unroll
                for (int i = 0; i < kPer; ++i) {
                    const int kk = x.t0 * kKT + pt + i * kProdThreads;
                    jsel[i] = (pt + i * kProdThreads < x.nt * kKT && !a.dense && kk < x.E) ? __ldg(&a.sel[x.q * a.topk + kk])
                                                                                      : 0;
                }
#pragma unroll
                for (int i = 0; i < kPer; ++i) {
                    const int loc = pt + i * kProdThreads;
                    if (loc >= x.nt * kKT) break;
                    const int kk = x.t0 * kKT + loc;
                    const __nv_bfloat16 *ptr = nullptr;
                    if (kk < x.E) {
                        const int64_t j = a.dense ? (int64_t)kk : (int64_t)jsel[i];
                        if (j >= 0 && j < x.nvis) {
                            const int64_t R = (a.decode ? x.q * a.N : 0) + j;
                            ptr = a.lowprec ? reinterpret_cast<const __nv_bfloat16 *>(a.ent8 + R * kC)
                                            : a.ent + R * (int64_t)kC;
                        }
                        else if (!a.dense && j != -1) report(a.status, kStatusBounds);   // a selected index that is
                                                                                        // neither padding nor visible
                    } else {
                        const int64_t pp = x.p - (kKT - 1) + (kk - x.E);
                        if (pp >= 0 && !a.no_window) ptr = a.raw + (a.decode ? x.q * kKT + pp % kKT : pp) * a.ld_raw;
                    }
                    rp[loc] = ptr;
                }
            }
            ok = tc::named_bar_and(2, kProdThreads, ok);
            if (!ok) break;
            ++iu;
            auto load_chunk = [&](int t, int col) {
                const int s = ic % kNS;
                const int kt = x.t0 + t;
                if (a.lowprec && kt * kKT < x.E) {
                    // FP8 entry rows: 8 codes (one 16-byte bf16 chunk) and their block exponent per thread, loaded
                    // into registers before the stage is free, then rebuilt as bf16 (exact) in the swizzled stage
                    constexpr int kIt = (kKT * 8 + kProdThreads - 1) / kProdThreads;
                    const int g = pt & 7;
                    const __nv_bfloat16 *const *rows = rp + t * kKT;
                    uint2 cv[kIt];
                    int ev[kIt];
#pragma unroll
                    for (int i = 0; i < kIt; ++i) {
                        const int row = i * (kProdThreads / 8) + (pt >> 3);
                        cv[i] = make_uint2(0u, 0u);
                        ev[i] = 0;
                        if ((kKT * 8) % kProdThreads != 0 && row >= kKT) break;
                        const uint8_t *p = reinterpret_cast<const uint8_t *>(rows[row]);
                        if (p) {
                            const int ch = col + g * 8;
                            cv[i] = __ldg(reinterpret_cast<const uint2 *>(p + ch));
                            ev[i] = __ldg(a.ent_exp + ((p - a.ent8) + ch) / lp::kBlock);
                        }
                    }
                    if (ic >= kNS) ok = ok && tc::mbar_wait(&bars->re[s], ((ic / kNS) - 1) & 1, a.status);
                    if (!ok) {
                        ++ic;
                        return;
                    }
#pragma unroll
                    for (int i = 0; i < kIt; ++i) {
                        const int row = i * (kProdThreads / 8) + (pt >> 3);
                        if ((kKT * 8) % kProdThreads != 0 && row >= kKT) break;
                        const uint4 v = lp::fp8x8_to_bf16x8(cv[i], lp::pow2f(ev[i]));
                        *reinterpret_cast<uint4 *>(sRing + s * kStage + tc::sw128_offset(row, g)) = v;
                    }
                    tc::fence_async_smem();   // generic-proxy stores -> the MMA's async proxy
                    tc::mbar_arrive(&bars->rf[s]);
                    ++ic;
                    return;
                }
                if (ic >= kNS) ok = ok && tc::mbar_wait(&bars->re[s], ((ic / kNS) - 1) & 1, a.status);
                if (!ok) {
                    ++ic;
                    return;
                }
                // 128 consecutive rows: the prefill window, or a dense (HCA) entry tile inside the visible range
                const bool win_tile = !a.decode && kt * kKT >= x.E;
                const bool ent_tile = a.dense && !a.lowprec && (int64_t)(kt + 1) * kKT <= x.nvis;
                if (win_tile || ent_tile) {
                    if (pt == 0) {
                        tc::mbar_arrive_expect_tx(&bars->rf[s], kStage);
                        if (win_tile)
                            tc::tma_load_2d(ring + s * kStage, &tm_raw, col, (int)(x.p - (kKT - 1)), &bars->rf[s]);
                        else
                            tc::tma_load_2d(ring + s * kStage, &tm_ent, col,
                                            (int)((a.decode ? x.q * a.N : 0) + (int64_t)kt * kKT), &bars->rf[s]);
                        tma_use[s] = (int32_t)(ic / kNS);
                    } else {
                        tc::mbar_arrive(&bars->rf[s]);
                    }
                } else {
                    const int g = pt & 7;
                    const __nv_bfloat16 *const *rows = rp + t * kKT;
#pragma unroll
                    for (int i = 0; i < (kKT * 8 + kProdThreads - 1) / kProdThreads; ++i) {
                        const int row = i * (kProdThreads / 8) + (pt >> 3);
                        if ((kKT * 8) % kProdThreads != 0 && row >= kKT) break;
                        const __nv_bfloat16 *p = rows[row];
                        tc::cp_async16(ring + s * kStage + tc::sw128_offset(row, g), p ? p + col + g * 8 : a.ent,
                                       p != nullptr);
                    }
                    tc::cp_async_arrive_noinc(&bars->rf[s]);
                    // At most kGatherDepth chunks of this thread in flight: a thread whose copies cannot be
                    // accepted waits here instead of holding up the shared load/store queue that the softmax
                    // warps' shuffles, shared-memory accesses and barrier polls also go through.
                    tc::cp_async_commit();
                    tc::cp_async_wait<kGatherDepth - 1>();
                }
                ++ic;
            };
            auto load_q = [&](int dc) {
                const int qb = iq & 1;
                if (pt == 0 && ok) {
                    if (iq >= 2) ok = ok && tc::mbar_wait(&bars->qe[qb], ((iq >> 1) - 1) & 1, a.status);
                    if (ok) {
                        tc::mbar_arrive_expect_tx(&bars->qf[qb], kQStage);
                        tc::tma_load_3d(Qs + qb * kQStage, &tm_q, dc * 64, 0, (int)x.q, &bars->qf[qb]);
                        tma_use[kNS + qb] = (int32_t)(iq >> 1);
                    }
                }
                ++iq;
            };
            for (int dc = 0; dc < 8; ++dc) {          // S: every tile's key chunk next to its Q chunk
                if (!a.decode) load_q(dc);
                for (int t = 0; t < x.nt; ++t) load_chunk(t, dc * 64);
            }
            for (int i = 0; i < x.nt; ++i)            // P V: value halves, 64-dh chunks in pairs
                for (int c = 2 * x.dp0; c < 2 * x.dp1; ++c) load_chunk(pv_tile<DEC>(i, x.nt), kDh + c * 64);
        }
        tc::cp_async_wait_all();
        if (!ok && pt == 0) {
            // abandoned run: let every TMA load this thread issued land before the CTA exits
            for (int i = 0; i < kNS + 2; ++i)
                if (tma_use[i] >= 0)
                    tc::mbar_wait(i < kNS ? &bars->rf[i] : &bars->qf[i - kNS], (uint32_t)tma_use[i] & 1, nullptr);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint32_t ic = 0, iq = 0, iu = 0;
            uint32_t puse[2] = {0u, 0u};   // prefill: uses of each P^T tile slot so far
            for (int64_t u = blockIdx.x; u < a.n_units && ok; u += gridDim.x) {
                const Unit x = unit_of(a, u);
                if (x.nt <= 0) continue;
                if (iu >= 1) ok = ok && tc::mbar_wait(&bars->s_free, (iu - 1) & 1, a.status);
                if (a.decode) ok = ok && tc::mbar_wait(&bars->qf[0], iu & 1, a.status);   // whole query in P
                for (int dc = 0; dc < 8; ++dc) {
                    const int qb = iq & 1;
                    if (!a.decode) ok = ok && tc::mbar_wait(&bars->qf[qb], (iq >> 1) & 1, a.status);
                    const uint32_t qsm = a.decode ? P + dc * kQStage : Qs + qb * kQStage;
                    for (int t = 0; t < x.nt; ++t, ++ic) {
                        const int s = ic % kNS;
                        // tile 4's scores share TMEM columns with the previous unit's output accumulator
                        if (t == 4 && dc == 0 && iu >= 1) ok = ok && tc::mbar_wait(&bars->o_free, (iu - 1) & 1, a.status);
                        ok = ok && tc::mbar_wait(&bars->rf[s], (ic / kNS) & 1, a.status);
                        tc::fence_async_smem();   // cp.async data (generic proxy) -> MMA (async proxy)
                        tc::tc_fence_after();
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            tc::mma_bf16(tmem + s_col(t), tc::sdesc_sw128(ring + s * kStage + 32 * k, 16, 1024),
                                         tc::sdesc_sw128(qsm + 32 * k, 16, 1024), kIdescS, (dc | k) != 0);
                        tc::mma_commit(&bars->re[s]);
                    }
                    if (!a.decode) {
                        tc::mma_commit(&bars->qe[qb]);
                        ++iq;
                    }
                }
                tc::mma_commit(&bars->s_full);
                if (DEC) {   // all of P^T at once
                    ok = ok && tc::mbar_wait(&bars->p_full, iu & 1, a.status);
                    tc::tc_fence_after();
                }
                for (int i = 0; i < x.nt; ++i) {
                    const int t = pv_tile<DEC>(i, x.nt);
                    const int ps = i & 1;   // prefill: the P^T slot of step i
                    if (!DEC) {
                        ok = ok && tc::mbar_wait(&bars->pt_full[ps], puse[ps] & 1, a.status);
                        tc::tc_fence_after();
                    }
                    for (int dp = x.dp0; dp < x.dp1; ++dp, ic += 2) {
                        const int s0 = ic % kNS, s1 = (ic + 1) % kNS;
                        ok = ok && tc::mbar_wait(&bars->rf[s0], (ic / kNS) & 1, a.status);
                        ok = ok && tc::mbar_wait(&bars->rf[s1], ((ic + 1) / kNS) & 1, a.status);
                        tc::fence_async_smem();
                        tc::tc_fence_after();
                        const uint32_t av = ring + s0 * kStage, bp = P + (DEC ? t : ps) * kKT * 128;
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            tc::mma_bf16(tmem + kColB + dp * kH, tc::sdesc_sw128(av + 2048 * k, kStage, 1024),
                                         tc::sdesc_sw128(bp + 2048 * k, kStage, 1024), kIdescPV, (i | k) != 0);
                        tc::mma_commit(&bars->re[s0]);
                        tc::mma_commit(&bars->re[s1]);
                    }
                    if (!DEC) {
                        tc::mma_commit(&bars->pt_empty[ps]);
                        ++puse[ps];
                    }
                }
                tc::mma_commit(&bars->o_full);
                ++iu;
            }
            // every MMA issued by this thread has completed before TMEM is released
            tc::mma_commit(&bars->fin);
            tc::mbar_wait(&bars->fin, 0, a.status);
        }
    } else {
        // ------------------------------------------------ softmax + output epilogue (8 warps)
        const int et = threadIdx.x - kSoftWarp0 * 32;
        const int quad = warp & 3, hh = (warp - kSoftWarp0) >> 2;
        const int r = quad * 32 + lane;                  // key row in a tile; dh row in an output block
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
        uint32_t iu = 0;
        uint32_t puse[2] = {0u, 0u};   // prefill: uses of each P^T tile slot so far
        for (int64_t u = blockIdx.x; u < a.n_units; u += gridDim.x) {
            // the softmax warps meet at named barriers within a unit: they leave the loop together
            ok = tc::named_bar_and(1, kSoftThreads, ok);
            if (!ok) break;
            const Unit x = unit_of(a, u);
            const int64_t slot = x.q * a.nseg + x.seg;
            if (x.nt <= 0) {
                if (a.part && et < kH && x.dp0 == 0) {
                    float *pml = a.part + a.nq * (int64_t)a.nseg * kH * kDh;
                    pml[(slot * kH + et) * 2] = -INFINITY;
                    pml[(slot * kH + et) * 2 + 1] = 0.f;
                }
                continue;
            }
            bool valid[kMaxTiles];
            {
                int32_t jsel[kMaxTiles];
#pragma unroll
                for (int t = 0; t < kMaxTiles; ++t) {
                    const int kk = (x.t0 + t) * kKT + r;
                    jsel[t] = (t < x.nt && !a.dense && kk < x.E) ? __ldg(&a.sel[x.q * a.topk + kk]) : 0;
                }
#pragma unroll
                for (int t = 0; t < kMaxTiles; ++t) {
                    const int kk = (x.t0 + t) * kKT + r;
                    bool v = false;
                    if (t < x.nt) {
                        if (kk < x.E) {
                            const int64_t j = a.dense ? (int64_t)kk : (int64_t)jsel[t];
                            v = j >= 0 && j < x.nvis;
                        } else {
                            v = !a.no_window && x.p - (kKT - 1) + (kk - x.E) >= 0;
                        }
                    }
                    valid[t] = v;
                }
            }
            ok = ok && tc::mbar_wait(&bars->s_full, iu & 1, a.status);
            tc::tc_fence_after();
            float v[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = -INFINITY;
            for (int t = 0; t < x.nt; ++t) {
                float s[32];
                tc::tmem_ld32(tl + s_col(t) + hh * 32, s);
                tc::tmem_ld_wait();
                if (valid[t]) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = fmaxf(v[i], s[i]);
                }
            }
            red[quad * kH + hh * 32 + lane] = warp_transpose_reduce32<true>(v, lane);
            tc::named_bar_sync(1, kSoftThreads);
            if (et < kH) {
                const float mm = fmaxf(fmaxf(red[et], red[kH + et]), fmaxf(red[2 * kH + et], red[3 * kH + et]));
                mx[et] = mm == -INFINITY ? 0.f : mm * a.scale_log2;
                mnat[et] = mm == -INFINITY ? -INFINITY : mm * a.scale;
            }
            tc::named_bar_sync(1, kSoftThreads);
            float mloc[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) { mloc[i] = mx[hh * 32 + i]; v[i] = 0.f; }
            for (int i = 0; i < x.nt; ++i) {
                const int t = pv_tile<DEC>(i, x.nt);
                const int ps = i & 1;   // prefill: step i's tile goes to slot i % 2 once P V of step i - 2 has read it
                if (!DEC && puse[ps] >= 1)
                    ok = ok && tc::mbar_wait(&bars->pt_empty[ps], (puse[ps] - 1) & 1, a.status);
                float s[32];
                tc::tmem_ld32(tl + s_col(t) + hh * 32, s);
                tc::tmem_ld_wait();
                const bool vt = valid[t];
                const uint32_t rowaddr = P + (uint32_t)((DEC ? t : ps) * kKT + r) * 128u;
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int h0 = g * 8 + 2 * e;
                        const float p0 = vt ? ex2(fmaf(s[h0], a.scale_log2, -mloc[h0])) : 0.f;
                        const float p1 = vt ? ex2(fmaf(s[h0 + 1], a.scale_log2, -mloc[h0 + 1])) : 0.f;
                        v[h0] += p0;
                        v[h0 + 1] += p1;
                        __nv_bfloat162 pr = __floats2bfloat162_rn(p0, p1);
                        w[e] = *reinterpret_cast<uint32_t *>(&pr);
                    }
                    const uint32_t gg = (uint32_t)(hh * 4 + g);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(rowaddr + ((gg ^ (uint32_t)(r & 7)) << 4)),
                                 "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3])
                                 : "memory");
                }
                if (!DEC) {   // this warp's part of the tile -> the MMA's async proxy; P V of tile t may start
                    tc::fence_async_smem();
                    tc::tc_fence_before();   // and its TMEM reads of the scores before P V writes those columns
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(&bars->pt_full[ps]);
                    ++puse[ps];
                }
            }
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bars->s_free);
            const float zsum = warp_transpose_reduce32<false>(v, lane);
            tc::named_bar_sync(1, kSoftThreads);     // everyone is done with red[] from the max pass
            red[quad * kH + hh * 32 + lane] = zsum;
            tc::named_bar_sync(1, kSoftThreads);
            if (et < kH) {
                const float Z = red[et] + red[kH + et] + red[2 * kH + et] + red[3 * kH + et];
                zinv[et] = Z > 0.f ? 1.f / Z : 0.f;
                znat[et] = Z;
            }
            tc::fence_async_smem();
            tc::named_bar_sync(1, kSoftThreads);     // zinv / znat visible to every epilogue thread
            if (DEC && lane == 0) tc::mbar_arrive(&bars->p_full);
            // ---- output
            ok = ok && tc::mbar_wait(&bars->o_full, iu & 1, a.status);
            tc::tc_fence_after();
            for (int dp = x.dp0; dp < x.dp1; ++dp) {
                float o[32];
                tc::tmem_ld32(tl + kColB + dp * kH + hh * 32, o);
                tc::tmem_ld_wait();
                const int dh = dp * 128 + r;
                if (a.part == nullptr) {
                    __nv_bfloat16 *orow = a.out + x.q * (int64_t)kH * kDh + dh;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int h = hh * 32 + i;
                        orow[(int64_t)h * kDh] = __float2bfloat16_rn(o[i] * zinv[h]);
                    }
                } else {
                    float *pacc = a.part + slot * (int64_t)kH * kDh + dh;
#pragma unroll
                    for (int i = 0; i < 32; ++i) pacc[(int64_t)(hh * 32 + i) * kDh] = o[i];
                }
            }
            if (a.part && et < kH && x.dp0 == 0) {   // the value-block units of a slot share its (max, sum)
                float *pml = a.part + a.nq * (int64_t)a.nseg * kH * kDh;
                pml[(slot * kH + et) * 2] = mnat[et];
                pml[(slot * kH + et) * 2 + 1] = znat[et];
            }
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bars->o_free);
            ++iu;
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_free(tmem, kTmemCols);
    }
}

constexpr size_t smem_bytes(bool dec) {
    return 1024 + p_bytes(dec) + (size_t)ring_stages(dec) * kStage + 2 * kQStage + sizeof(float) * 8 * kH +
           sizeof(void *) * 2 * kMaxTiles * kKT + sizeof(Bars) + 16;
}
static_assert(smem_bytes(false) <= 232448 && smem_bytes(true) <= 232448, "shared memory per CTA");

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

}  // namespace

bool attend_tc_supported(const AttendArgs &a) {
    if (a.dtype != HCSA_BF16 || a.H != kH || a.dh != kDh || a.C != kC || a.window != kKT) return false;
    if (a.ld_q % 8 || (a.pos == nullptr && a.ld_kv % 8)) return false;
    if (a.N > INT32_MAX / 2 || a.rows * (a.pos ? a.N : 1) > INT32_MAX) return false;
    if (!a.dense) {
        if (a.topk % kKT) return false;
        if (a.pos == nullptr && a.topk / kKT + 1 > kMaxTiles) return false;
    } else if (a.pos == nullptr && (a.N + kKT - 1) / kKT + 1 > kMaxTiles) {
        return false;
    }
    return true;
}

static int64_t decode_tiles(const AttendArgs &a) {
    const int64_t e = a.dense ? (a.N + kKT - 1) / kKT * kKT : a.topk;
    return e / kKT + 1;
}

// Decode splits each sequence's key list into units of equal tile counts.  Every SM streams its
// units at a rate of its own, so the step takes as long as the busiest SM: use the fewest tiles per
// unit that still fit all units in one wave over the SMs (fewer, longer units write fewer partials
// for the merge); when no split fits one wave, take the longest units.
static int decode_seg_tiles(const AttendArgs &a) {
    const int64_t tiles = decode_tiles(a);
    for (int s = 1; s <= kMaxTiles; ++s)
        if (a.rows * ((tiles + s - 1) / s) <= num_sms()) return s;
    return kMaxTiles;
}

int attend_tc_segments(const AttendArgs &a) {
    if (a.pos == nullptr) return 1;
    const int64_t tiles = decode_tiles(a);
    const int st = decode_seg_tiles(a);
    return (int)((tiles + st - 1) / st);
}

hcsa_status launch_attend_tc(const AttendArgs &a, cudaStream_t st) {
    static bool configured[64] = {};   // kernel attributes are set per device
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return HCSA_ERR_CUDA;
    if (!configured[dev]) {
        if (cudaFuncSetAttribute(attend_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem_bytes(true)) != cudaSuccess ||
            cudaFuncSetAttribute(attend_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem_bytes(false)) != cudaSuccess)
            return HCSA_ERR_CUDA;
        configured[dev] = true;
    }
    const bool decode = a.pos != nullptr;
    CUtensorMap tq, te, tr;
    // prefill: entries end at the last one the range's last query sees (the dense tiles round up past it;
    // those rows read as zeros, so a row-range caller need not have gathered them)
    const int64_t last_vis = a.row1 > 0 ? (a.row1 - 1) / a.m : 0;
    const uint64_t ent_rows = decode ? (uint64_t)a.rows * a.N
                                     : (uint64_t)std::max<int64_t>(1, std::min<int64_t>(a.N, last_vis));
    if (!make_tmap_bf16_3d(&tq, a.q, kDh, kH, (uint64_t)a.rows, kDh * 2, (uint64_t)a.ld_q * 2, 64, kH, 1, true))
        return HCSA_ERR_CUDA;
    if (!make_tmap_bf16_2d(&te, a.entries, kC, ent_rows, kC * 2, 64, kKT, true)) return HCSA_ERR_CUDA;
    if (decode) {
        tr = te;   // unused: decode window rows are gathered from the ring
    } else if (!make_tmap_bf16_2d(&tr, a.kv, kC, (uint64_t)a.rows, (uint64_t)a.ld_kv * 2, 64, kKT, true)) {
        return HCSA_ERR_CUDA;
    }
    Params p{};
    p.ent = (const __nv_bfloat16 *)a.entries;
    p.lowprec = a.lowprec;
    if (a.lowprec) {   // code rows [ent_rows][C], then exponent rows [ent_rows][C / 32]
        const int64_t rows_all = decode ? a.rows * a.N : a.N;
        p.ent8 = (const uint8_t *)a.entries;
        p.ent_exp = (const int8_t *)(p.ent8 + rows_all * kC);
    }
    p.raw = (const __nv_bfloat16 *)a.kv;
    p.ld_raw = decode ? kC : a.ld_kv;
    p.decode = decode;
    p.dense = a.dense;
    p.nq = a.rows;
    p.N = a.N;
    p.m = a.m;
    p.topk = a.topk;
    p.nseg = attend_tc_segments(a);
    p.seg_tiles = decode ? decode_seg_tiles(a) : kMaxTiles;
    // decode units that leave most SMs idle split their value blocks over 2 or 4 CTAs (each recomputes the
    // scores from the same key rows, an L2 hit after the first, and gathers and writes a part of the values)
    p.dq_split = 1;
    if (decode)
        for (int s = 4; s >= 2; s /= 2)
            if ((a.row1 - a.row0) * p.nseg * s <= num_sms()) {
                p.dq_split = s;
                break;
            }
    p.sel = a.sel;
    p.pos = a.pos;
    p.scale = a.scale;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.out = (__nv_bfloat16 *)a.out;
    p.part = (p.nseg > 1 || a.partial_out) ? (float *)a.ws : nullptr;
    p.q0 = a.row0;
    p.ent0 = a.ent0;
    p.no_window = a.no_window;
    p.n_units = (a.row1 - a.row0) * p.nseg * p.dq_split;
    p.status = device_status_ptr();
    if (p.n_units <= 0) return HCSA_OK;
    const int64_t grid = p.n_units < num_sms() ? p.n_units : num_sms();
    if (decode)
        attend_tc_kernel<true><<<(unsigned)grid, kThreads, smem_bytes(true), st>>>(tq, te, tr, p);
    else
        attend_tc_kernel<false><<<(unsigned)grid, kThreads, smem_bytes(false), st>>>(tq, te, tr, p);
    count_launch();
    return check_launch();
}

}  // namespace hcsa

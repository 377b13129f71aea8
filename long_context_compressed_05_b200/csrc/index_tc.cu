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
//   * 8 epilogue warps (two per TMEM lane quadrant, each owning half of the
//     columns) read the accumulator, apply ReLU, weight by w and sum the heads in
//     registers -- no cross-lane traffic -- and store fp32 scores coalesced.
// Warp roles: warp 0 = TMA producer, warp 1 = MMA issuer, warps 2..9 = epilogue.
// Persistent CTAs walk a list of work units (prefill: one query tile each, the
// heaviest causal tiles first; decode: (sequence, 8 key tiles)).
//
// Top-k kernel.  One CTA of 512 threads per query row keeps the row's scores in
// registers (<= 32768), and finds the k-th largest order-preserving key with three
// histogram passes (12 + 10 + 10 bits) over the registers; the chosen indices are
// marked in a shared-memory bitmap of the row (ties at the k-th value: lowest j) and
// emitted in ascending order with one block scan over the bitmap words.
#include <cub/block/block_scan.cuh>

#include "tc_common.cuh"

namespace hcsa {

namespace {

constexpr int kNS = 8;               // key-tile ring stages
constexpr int kATile = 128 * 128;    // 128 keys x 64 bf16
constexpr int kBTile = 256 * 128;    // up to 256 (token, head) rows x 64 bf16
constexpr int kThreads = 320;        // 10 warps
constexpr int kEpiThreads = 256;
constexpr int kDecodeTilesPerUnit = 32;

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
    int64_t n_units, n_qtiles;
    int64_t dec_chunks;  // decode: units per sequence
    int *status;
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
    if (!a.decode) {
        const int64_t q = a.n_qtiles - 1 - u;   // heaviest first
        x.b = 0;
        x.r0 = q * a.tq;
        int64_t last = x.r0 + a.tq - 1 < a.rows ? x.r0 + a.tq - 1 : a.rows - 1;
        x.kt0 = 0;
        x.kt1 = (int)((visible(a, last) + 127) / 128);
    } else {
        x.b = u / a.dec_chunks;
        x.r0 = x.b;
        const int c = (int)(u % a.dec_chunks);
        const int nkt = (int)((visible(a, x.b) + 127) / 128);
        x.kt0 = c * kDecodeTilesPerUnit;
        x.kt1 = min(nkt, x.kt0 + kDecodeTilesPerUnit);
    }
    return x;
}

template <int HI>
__global__ void __launch_bounds__(kThreads, 1)
index_scores_tc_kernel(const __grid_constant__ CUtensorMap tm_keys, const __grid_constant__ CUtensorMap tm_qi,
                       Args a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = base;                       // kNS x 16 KB
    uint8_t *sB = sA + kNS * kATile;          // 2 x 32 KB
    float *sw = reinterpret_cast<float *>(sB + 2 * kBTile);   // 2 x 256 head weights
    uint64_t *bars = reinterpret_cast<uint64_t *>(sw + 512);
    uint64_t *a_full = bars, *a_empty = bars + kNS, *b_full = bars + 2 * kNS, *b_empty = b_full + 2;
    uint64_t *acc_full = b_empty + 2, *acc_empty = acc_full + 4;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_empty + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kNS; ++i) { tc::mbar_init(&a_full[i], 1); tc::mbar_init(&a_empty[i], 1); }
        for (int i = 0; i < 2; ++i) { tc::mbar_init(&b_full[i], 1); tc::mbar_init(&b_empty[i], 1); }
        for (int i = 0; i < 4; ++i) { tc::mbar_init(&acc_full[i], 1); tc::mbar_init(&acc_empty[i], kEpiThreads / 32); }
        tc::fence_mbar_init();
    }
    if (warp == 0) tc::tmem_alloc(tmem_slot, 512);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t ia = 0, ib = 0;
            for (int64_t u = blockIdx.x; u < a.n_units && ok; u += gridDim.x) {
                const Unit x = unit_of(a, u);
                if (x.kt0 >= x.kt1) continue;
                const int bb = ib & 1;
                if (ib >= 2) ok &= tc::mbar_wait(&b_empty[bb], ((ib >> 1) - 1) & 1, a.status);
                tc::mbar_arrive_expect_tx(&b_full[bb], a.ncols * 128);
                tc::tma_load_3d(tc::smem_u32(sB + bb * kBTile), &tm_qi, 0, 0, (int)x.r0, &b_full[bb]);
                ++ib;
                for (int kt = x.kt0; kt < x.kt1 && ok; ++kt, ++ia) {
                    const int s = ia % kNS;
                    if (ia >= kNS) ok &= tc::mbar_wait(&a_empty[s], ((ia / kNS) - 1) & 1, a.status);
                    tc::mbar_arrive_expect_tx(&a_full[s], kATile);
                    tc::tma_load_3d(tc::smem_u32(sA + s * kATile), &tm_keys, 0, kt * 128, (int)x.b, &a_full[s]);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = tc::idesc_bf16(128, a.ncols, false, false);
            uint32_t ia = 0, ib = 0, iacc = 0;
            for (int64_t u = blockIdx.x; u < a.n_units && ok; u += gridDim.x) {
                const Unit x = unit_of(a, u);
                if (x.kt0 >= x.kt1) continue;
                const int bb = ib & 1;
                ok &= tc::mbar_wait(&b_full[bb], (ib >> 1) & 1, a.status);
                const uint32_t bsm = tc::smem_u32(sB + bb * kBTile);
                for (int kt = x.kt0; kt < x.kt1 && ok; ++kt, ++ia, ++iacc) {
                    const int s = ia % kNS, ab = iacc % a.nbuf;
                    ok &= tc::mbar_wait(&a_full[s], (ia / kNS) & 1, a.status);
                    if (iacc >= (uint32_t)a.nbuf)
                        ok &= tc::mbar_wait(&acc_empty[ab], ((iacc / a.nbuf) - 1) & 1, a.status);
                    tc::tc_fence_after();
                    const uint32_t asm_ = tc::smem_u32(sA + s * kATile);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        tc::mma_bf16(tmem + ab * a.stride, tc::sdesc_sw128(asm_ + 32 * k, 16, 1024),
                                     tc::sdesc_sw128(bsm + 32 * k, 16, 1024), idesc, k > 0);
                    tc::mma_commit(&a_empty[s]);
                    tc::mma_commit(&acc_full[ab]);
                }
                tc::mma_commit(&b_empty[bb]);
                ++ib;
            }
        }
    } else {
        // ------------------------------------------------ epilogue: ReLU, head weights, head sum
        // Prefill (256 columns): the two warp groups split the columns of every tile.  Decode (<= 128
        // columns): the groups take alternate tiles, each reading all columns.
        const int et = threadIdx.x - 64;              // 0..255
        const int quad = warp & 3, half = (warp - 2) >> 2;
        const int row = quad * 32 + lane;             // key within the tile (TMEM lane)
        const bool split = a.ncols <= 128;
        constexpr int TPH = 128 / HI > 0 ? 128 / HI : 1;   // tokens per 128 columns
        const int tok_base = split ? 0 : half * TPH;
        const int col_base = split ? 0 : half * 128;
        uint32_t iacc = 0, iu = 0;
        for (int64_t u = blockIdx.x; u < a.n_units && ok; u += gridDim.x) {
            const Unit x = unit_of(a, u);
            if (x.kt0 >= x.kt1) continue;
            float *w_s = sw + (iu & 1) * 256;
            if (et < a.ncols) {
                const int64_t r = x.r0 + et / HI;
                w_s[et] = r < a.rows ? __bfloat162float(a.w[r * a.ld_w + et % HI]) : 0.f;
            }
            tc::named_bar_sync(1, kEpiThreads);
            ++iu;
            const int ntok = a.ncols / HI;                       // tokens in the unit
            int64_t vis[TPH];
#pragma unroll
            for (int i = 0; i < TPH; ++i) {
                const int64_t r = x.r0 + tok_base + i;
                vis[i] = (tok_base + i < ntok && r < a.rows) ? visible(a, r) : 0;
            }
            for (int kt = x.kt0; kt < x.kt1 && ok; ++kt, ++iacc) {
                if (split && (int)(iacc & 1) != half) continue;
                const int ab = iacc % a.nbuf;
                ok &= tc::mbar_wait(&acc_full[ab], (iacc / a.nbuf) & 1, a.status);
                tc::tc_fence_after();
                float s[TPH];
#pragma unroll
                for (int i = 0; i < TPH; ++i) s[i] = 0.f;
                const uint32_t tl = tmem + ab * a.stride + ((uint32_t)(quad * 32) << 16);
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    const int col0 = col_base + cc * 32;
                    if (col0 < a.ncols) {
                        float v[32];
                        tc::tmem_ld32(tl + col0, v);
                        tc::tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            const int c = cc * 32 + i;                // column within this group's 128
                            s[c / HI < TPH ? c / HI : TPH - 1] += w_s[col0 + i] * fmaxf(v[i], 0.f);
                        }
                    }
                }
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive_cnt(&acc_empty[ab], split ? 2 : 1);
                const int64_t j = (int64_t)kt * 128 + row;
#pragma unroll
                for (int i = 0; i < TPH; ++i)
                    if (j < vis[i]) a.scores[(x.r0 + tok_base + i) * a.N + j] = s[i];
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

// ------------------------------------------------------------------ register-resident top-k
constexpr int kTkThreads = 512;

__device__ __forceinline__ uint32_t order_key(float s) {
    if (s == 0.0f) s = 0.0f;   // -0 and +0 compare equal
    uint32_t b = __float_as_uint(s);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

template <int VPT>   // float4 vectors per thread: row capacity = 2048 * VPT
__global__ void __launch_bounds__(kTkThreads) topk_regs_kernel(const float *__restrict__ scores, int64_t N,
                                                               int m, const int32_t *__restrict__ pos, int topk,
                                                               int32_t *__restrict__ sel) {
    using Scan = cub::BlockScan<int, kTkThreads>;
    __shared__ typename Scan::TempStorage scan_tmp;
    __shared__ int hist[4096];
    __shared__ uint32_t bitmap[1024];   // rows of up to 32768 entries
    __shared__ uint32_t eq_idx[64];
    __shared__ uint32_t s_prefix;
    __shared__ int s_rem, s_eq_total;
    const int tid = threadIdx.x;
    const int64_t r = blockIdx.x;
    int64_t p = pos ? (int64_t)pos[r] : r;
    int64_t n = p < 0 ? 0 : (p / m < N ? p / m : N);
    int32_t *out = sel + r * topk;
    if (n <= topk) {
        for (int i = tid; i < topk; i += kTkThreads) out[i] = i < n ? i : -1;
        return;
    }
    const float *row = scores + r * N;
    const bool vec_ok = (N & 3) == 0;   // rows start 16-byte aligned
    uint32_t key[VPT * 4];
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int64_t j0 = 4 * ((int64_t)tid + (int64_t)kTkThreads * i);
        if (vec_ok && j0 + 3 < n) {
            float4 v = __ldcs(reinterpret_cast<const float4 *>(row + j0));
            key[4 * i] = order_key(v.x); key[4 * i + 1] = order_key(v.y);
            key[4 * i + 2] = order_key(v.z); key[4 * i + 3] = order_key(v.w);
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) key[4 * i + e] = (j0 + e < n) ? order_key(row[j0 + e]) : 0u;
        }
    }
    // three histogram passes: bits [20,32), [10,20), [0,10)
    uint32_t prefix = 0, mask = 0;
    int rem = topk;
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
                    break;
                }
                cum += c;
            }
        }
        __syncthreads();
        prefix = s_prefix;
        rem = s_rem;
        mask |= (uint32_t)(nb - 1) << sh;
        __syncthreads();
    }
    // prefix = k-th largest key; rem = keys equal to it that are taken (lowest j first).
    // Mark the chosen indices in a bitmap of the row, then emit them in ascending order with one scan.
    const int nw = (int)((n + 31) / 32);
    for (int i = tid; i < nw; i += kTkThreads) bitmap[i] = 0;
    if (tid == 0) s_eq_total = 0;
    __syncthreads();
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
                if (j < n) eq = order_key(row[j]) == prefix;
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

template <int HI>
static hcsa_status launch_scores(const IndexArgs &ia, const CUtensorMap &tk, const CUtensorMap &tq, Args a,
                                 cudaStream_t st) {
    constexpr size_t smem = 1024 + kNS * kATile + 2 * kBTile + 512 * sizeof(float) + (2 * kNS + 12) * sizeof(uint64_t) + 16;
    static bool configured = false;
    if (!configured) {
        if (cudaFuncSetAttribute(index_scores_tc_kernel<HI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem) != cudaSuccess)
            return HCSA_ERR_CUDA;
        configured = true;
    }
    const int64_t grid = a.n_units < num_sms() ? a.n_units : num_sms();
    if (grid <= 0) return HCSA_OK;
    index_scores_tc_kernel<HI><<<(unsigned)grid, kThreads, smem, st>>>(tk, tq, a);
    count_launch();
    return check_launch();
}

hcsa_status launch_index_tc(const IndexArgs &ia, cudaStream_t st) {
    const bool decode = ia.pos != nullptr;
    const int64_t nseq = decode ? ia.rows : 1;
    const int tq = decode ? 1 : 256 / ia.Hi;
    CUtensorMap tk, tq_map;
    if (!make_tmap_bf16_3d(&tk, ia.keys, 64, (uint64_t)ia.N, (uint64_t)nseq, 128, (uint64_t)ia.N * 128, 64, 128, 1,
                           true))
        return HCSA_ERR_CUDA;
    if (!make_tmap_bf16_3d(&tq_map, ia.qi, 64, (uint64_t)ia.Hi, (uint64_t)ia.rows, 128, (uint64_t)ia.ld_qi * 2, 64,
                           (uint32_t)ia.Hi, (uint32_t)tq, true))
        return HCSA_ERR_CUDA;
    Args a{};
    a.rows = ia.rows; a.N = ia.N; a.m = ia.m; a.tq = tq; a.ncols = tq * ia.Hi; a.decode = decode; a.pos = ia.pos;
    a.nbuf = a.ncols <= 128 ? 4 : 2;
    a.stride = a.ncols <= 128 ? 128 : 256;
    a.w = (const __nv_bfloat16 *)ia.w; a.ld_w = ia.ld_w; a.scores = (float *)ia.ws; a.status = device_status_ptr();
    if (decode) {
        const int64_t ntiles = (ia.N + 127) / 128;
        a.dec_chunks = (ntiles + kDecodeTilesPerUnit - 1) / kDecodeTilesPerUnit;
        a.n_units = ia.rows * a.dec_chunks;
        a.n_qtiles = 0;
    } else {
        a.n_qtiles = (ia.rows + tq - 1) / tq;
        a.n_units = a.n_qtiles;
        a.dec_chunks = 0;
    }
    hcsa_status s;
    switch (ia.Hi) {
        case 8: s = launch_scores<8>(ia, tk, tq_map, a, st); break;
        case 16: s = launch_scores<16>(ia, tk, tq_map, a, st); break;
        case 32: s = launch_scores<32>(ia, tk, tq_map, a, st); break;
        default: s = launch_scores<64>(ia, tk, tq_map, a, st); break;
    }
    if (s != HCSA_OK) return s;
    // top-k over the materialised scores
    if (ia.N <= 32768) {
        const float *sc = (const float *)ia.ws;
        if (ia.N <= 8192)
            topk_regs_kernel<4><<<(unsigned)ia.rows, kTkThreads, 0, st>>>(sc, ia.N, ia.m, ia.pos, ia.topk, ia.sel);
        else
            topk_regs_kernel<16><<<(unsigned)ia.rows, kTkThreads, 0, st>>>(sc, ia.N, ia.m, ia.pos, ia.topk, ia.sel);
        count_launch();
        return check_launch();
    }
    if (topk_rows_supported(ia)) {
        // scratch for the multi-CTA select sits after the scores
        uint8_t *scratch = (uint8_t *)ia.ws + (((size_t)ia.rows * ia.N * sizeof(float) + 255) & ~(size_t)255);
        hcsa_status s2 = launch_topk_rows(ia, scratch, st);
        if (s2 != HCSA_OK) return s2;
        IndexArgs fb = ia;                       // rows whose threshold bucket overflowed the candidate list
        fb.only_rows = (const int32_t *)(scratch + (size_t)ia.rows * 4096 * sizeof(uint32_t));
        return launch_topk_generic(fb, st);
    }
    return launch_topk_generic(ia, st);
}

}  // namespace hcsa

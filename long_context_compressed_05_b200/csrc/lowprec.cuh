// Block-scaled FP8 entries and FP4 indexer keys ("DeepSeek-V4 ... KV cache compressed attention",
// section "FP8 y FP4": most of each compressed entry in FP8, the indexer keys in FP4).
//
// Every 32 channels of a row share a power-of-two scale 2^e, e the smallest integer with
// amax / 2^e <= top (top = 448 for OCP E4M3, 6 for OCP E2M1), so nothing clips; a value x is stored
// as the code nearest to x / 2^e (ties to even).  A stored value (code x 2^e) has at most four
// significant bits, so it is exactly a bf16 number: the readers below rebuild the bf16 operand
// without rounding and the tensor-core paths compute exactly as they do on bf16 entries.
//
// Layout of an array of `rows` rows with `ch` channels:
//   FP8: rows x ch bytes of E4M3 codes, then rows x ch / 32 int8 exponents;
//   FP4: rows x ch / 2 bytes of E2M1 code pairs (channel 2i in the low nibble), then rows x ch / 32
//        int8 exponents.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <stdint.h>

namespace hcsa {
namespace lp {

constexpr int kBlock = 32;

// Exponent of the block scale: the smallest e with amax / 2^e <= top, top = tm x 2^te (1 <= tm < 2).
__device__ __forceinline__ int block_exponent(float amax, float tm, int te) {
    if (!(amax > 0.f)) return 0;
    int k;
    const float f = frexpf(amax, &k);   // amax = f 2^k, f in [0.5, 1)
    return (2.f * f <= tm) ? (k - 1) - te : (k - 1) - te + 1;
}

// The 4 lanes of one 32-channel block (lanes 4i .. 4i + 3, all active, 8 channels each) agree on the
// block's amax.
__device__ __forceinline__ float block_amax(const float *v) {
    float a = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(v[i]));
    const unsigned grp = 0xFu << (threadIdx.x & 28);
    a = fmaxf(a, __shfl_xor_sync(grp, a, 1));
    a = fmaxf(a, __shfl_xor_sync(grp, a, 2));
    return a;
}

// Store 8 channels c0 .. c0 + 7 of row `row` (values already rounded to bf16) as E4M3 codes; called by
// the 4 lanes of a 32-channel block together.
__device__ __forceinline__ void store_fp8x8(const float *v, uint8_t *codes, int8_t *exps, int64_t row, int ch,
                                            int c0) {
    const int e = block_exponent(block_amax(v), 1.75f, 8);   // 448 = 1.75 x 2^8
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t c = __nv_cvt_float_to_fp8(scalbnf(v[i], -e), __NV_SATFINITE, __NV_E4M3);
        w[i >> 2] |= (c & 0xFFu) << (8 * (i & 3));
    }
    *reinterpret_cast<uint2 *>(codes + row * ch + c0) = make_uint2(w[0], w[1]);
    if ((c0 & (kBlock - 1)) == 0) exps[row * (ch / kBlock) + c0 / kBlock] = (int8_t)e;
}

// Store 8 channels of row `row` as E2M1 code pairs (4 bytes); called by the 4 lanes of a block together.
__device__ __forceinline__ void store_fp4x8(const float *v, uint8_t *codes, int8_t *exps, int64_t row, int ch,
                                            int c0) {
    const int e = block_exponent(block_amax(v), 1.5f, 2);    // 6 = 1.5 x 2^2
    uint32_t w = 0u;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t c = __nv_cvt_float_to_fp4(scalbnf(v[i], -e), __NV_E2M1, cudaRoundNearest);
        w |= (c & 0xFu) << (4 * i);
    }
    *reinterpret_cast<uint32_t *>(codes + row * (ch / 2) + c0 / 2) = w;
    if ((c0 & (kBlock - 1)) == 0) exps[row * (ch / kBlock) + c0 / kBlock] = (int8_t)e;
}

// 2^e as a float (e within the normal range)
__device__ __forceinline__ float pow2f(int e) { return __int_as_float((127 + e) << 23); }

// Two E4M3 codes (low byte: first channel) -> bf16x2 of code x 2^e (exact).
__device__ __forceinline__ uint32_t fp8x2_to_bf16x2(uint32_t two, float s) {
    uint32_t h;   // f16x2: E4M3 values are f16 numbers
    asm("{.reg .b16 t; cvt.u16.u32 t, %1; cvt.rn.f16x2.e4m3x2 %0, t;}" : "=r"(h) : "r"(two & 0xFFFFu));
    float lo, hi;
    asm("{.reg .b16 l, u; mov.b32 {l, u}, %2; cvt.f32.f16 %0, l; cvt.f32.f16 %1, u;}" : "=f"(lo), "=f"(hi) : "r"(h));
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi * s), "f"(lo * s));
    return r;
}

// Two E2M1 codes (low nibble: first channel) -> bf16x2 of code x 2^e (exact).
__device__ __forceinline__ uint32_t fp4x2_to_bf16x2(uint32_t two, float s) {
    uint32_t h;
    asm("{.reg .b8 t; cvt.u8.u32 t, %1; cvt.rn.f16x2.e2m1x2 %0, t;}" : "=r"(h) : "r"(two & 0xFFu));
    float lo, hi;
    asm("{.reg .b16 l, u; mov.b32 {l, u}, %2; cvt.f32.f16 %0, l; cvt.f32.f16 %1, u;}" : "=f"(lo), "=f"(hi) : "r"(h));
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi * s), "f"(lo * s));
    return r;
}

// 8 E4M3 codes (uint2, channel order by byte) -> 8 bf16 (uint4)
__device__ __forceinline__ uint4 fp8x8_to_bf16x8(uint2 c, float s) {
    return make_uint4(fp8x2_to_bf16x2(c.x, s), fp8x2_to_bf16x2(c.x >> 16, s), fp8x2_to_bf16x2(c.y, s),
                      fp8x2_to_bf16x2(c.y >> 16, s));
}

// 8 E2M1 codes (uint32, channel order by nibble) -> 8 bf16 (uint4)
__device__ __forceinline__ uint4 fp4x8_to_bf16x8(uint32_t c, float s) {
    return make_uint4(fp4x2_to_bf16x2(c, s), fp4x2_to_bf16x2(c >> 8, s), fp4x2_to_bf16x2(c >> 16, s),
                      fp4x2_to_bf16x2(c >> 24, s));
}

}  // namespace lp
}  // namespace hcsa

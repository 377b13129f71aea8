// Token projections y = x W_cat (the layer's "low-dimensional projection"
// inputs: kv, gate, indexer key / query / head weight and query columns).
//
// A plain dense GEMM.  bf16 storage runs the tcgen05 kernel of gemm_tc.cu
// (bf16 tensor cores, fp32 accumulate, one rounding to bf16); fp32 storage
// uses a tiled CUDA-core kernel that accumulates in fp64 and rounds once to
// fp32.
#include "internal.cuh"

namespace hcsa {

constexpr int kPT = 64;   // output tile (rows and cols)
constexpr int kPK = 16;   // k step

__global__ void __launch_bounds__(256) project_f64acc_kernel(int64_t rows, int D, int64_t ncols,
                                                             const float *__restrict__ x,
                                                             const float *__restrict__ W, float *__restrict__ y) {
    __shared__ double sx[kPK][kPT + 1];
    __shared__ double sw[kPK][kPT + 1];
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    const int64_t r0 = (int64_t)blockIdx.y * kPT, c0 = (int64_t)blockIdx.x * kPT;
    double acc[4][4] = {};
    for (int k0 = 0; k0 < D; k0 += kPK) {
        for (int i = threadIdx.x; i < kPK * kPT; i += 256) {
            int kk = i % kPK, rr = i / kPK;
            int64_t r = r0 + rr;
            sx[kk][rr] = (r < rows && k0 + kk < D) ? (double)x[r * D + k0 + kk] : 0.0;
            int cc = i % kPT, k2 = i / kPT;
            int64_t c = c0 + cc;
            sw[k2][cc] = (c < ncols && k0 + k2 < D) ? (double)W[(int64_t)(k0 + k2) * ncols + c] : 0.0;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < kPK; ++kk) {
            double a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) { a[i] = sx[kk][ty * 4 + i]; b[i] = sw[kk][tx * 4 + i]; }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fma(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int64_t r = r0 + ty * 4 + i;
        if (r >= rows) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            int64_t c = c0 + tx * 4 + j;
            if (c < ncols) y[r * ncols + c] = (float)acc[i][j];
        }
    }
}

size_t project_ws_bytes(int dtype) { return dtype == HCSA_BF16 ? gemm_tc_ws_bytes() : 0; }

hcsa_status launch_project(int dtype, int64_t rows, int D, int64_t ncols, const void *x, const void *W, void *y,
                           void *ws, size_t ws_bytes, cudaStream_t st) {
    if (rows == 0 || ncols == 0) return HCSA_OK;
    if (dtype == HCSA_F32) {
        dim3 grid((unsigned)((ncols + kPT - 1) / kPT), (unsigned)((rows + kPT - 1) / kPT));
        if (grid.y > 65535) return HCSA_ERR_UNSUPPORTED;
        project_f64acc_kernel<<<grid, 256, 0, st>>>(rows, D, ncols, (const float *)x, (const float *)W, (float *)y);
        count_launch();
        return check_launch();
    }
    if (ncols > INT32_MAX || !gemm_tc_supported(rows, (int)ncols, D, x, D, W, ncols, y, ncols))
        return HCSA_ERR_UNSUPPORTED;
    return launch_gemm_tc(rows, (int)ncols, D, x, D, W, ncols, y, ncols, nullptr, 0, ws, ws_bytes, st);
}

// Output projection with the residual: x[rows, D] += out[rows, HD] W_o[HD, D] (bf16 storage, fp32
// accumulate, one rounding of x + out W_o).
hcsa_status launch_out_project(int64_t rows, int64_t HD, int D, const void *out, int64_t ld_out, const void *W_o,
                               void *x, int64_t ld_x, void *ws, size_t ws_bytes, cudaStream_t st) {
    if (rows == 0) return HCSA_OK;
    if (HD > INT32_MAX || !gemm_tc_supported(rows, D, (int)HD, out, ld_out, W_o, D, x, ld_x))
        return HCSA_ERR_UNSUPPORTED;
    return launch_gemm_tc(rows, D, (int)HD, out, ld_out, W_o, D, x, ld_x, x, ld_x, ws, ws_bytes, st);
}

}  // namespace hcsa

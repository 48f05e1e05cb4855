// projection.cu -- input pre-activations P = x W_ih^T + b_ih for every step.
//
// The input projection does not depend on the state, so it is computed once
// per solve for all (b, t) as one GEMM [B*T, Din] x [Din, 3D] -> [B*T, 3D]
// (fp32 accumulate, fp32 output), and every Newton iteration reads P.
//
// This file holds the general CUDA-core kernel: shared-memory tiles of
// 128 x 64 outputs, 8 x 4 outputs per thread, fp32 FMAs.  It takes fp32 or
// bf16 operands (bf16 is widened to fp32 on the way into shared memory) and
// any Din; it keeps fp32 inputs exact to fp32 rounding, which matters because
// the fixed point of the iteration is set by P as evaluated.
#include <cuda_bf16.h>

#include "common.cuh"
#include "solver.cuh"

namespace pararnn {
namespace {

constexpr int BM = 128, BN = 64, BK = 16;

__device__ __forceinline__ float widen(float v) { return v; }
__device__ __forceinline__ float widen(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename Tin>
__global__ void __launch_bounds__(256) proj_gemm_kernel(const Tin *__restrict__ X,
                                                        const Tin *__restrict__ W,
                                                        const float *__restrict__ bias,
                                                        float *__restrict__ P, long long M, int N,
                                                        int K) {
    __shared__ float Xs[BK][BM + 4];
    __shared__ float Ws[BK][BN + 4];
    const int tid = threadIdx.x;
    const int tx = tid % 16, ty = tid / 16;  // 16 x 16 threads; thread = 8 rows x 4 cols
    const long long m0 = static_cast<long long>(blockIdx.x) * BM;
    const int n0 = blockIdx.y * BN;
    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

    for (int k0 = 0; k0 < K; k0 += BK) {
#pragma unroll
        for (int s = 0; s < (BM * BK) / 256; ++s) {
            const int i = tid + s * 256;
            const int r = i / BK, kk = i % BK;
            const long long m = m0 + r;
            const int k = k0 + kk;
            Xs[kk][r] = (m < M && k < K) ? widen(X[m * K + k]) : 0.f;
        }
#pragma unroll
        for (int s = 0; s < (BN * BK) / 256; ++s) {
            const int i = tid + s * 256;
            const int r = i / BK, kk = i % BK;
            const int n = n0 + r, k = k0 + kk;
            Ws[kk][r] = (n < N && k < K) ? widen(W[static_cast<long long>(n) * K + k]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < BK; ++kk) {
            const float4 xa = *reinterpret_cast<const float4 *>(&Xs[kk][ty * 8]);
            const float4 xb = *reinterpret_cast<const float4 *>(&Xs[kk][ty * 8 + 4]);
            const float4 wv = *reinterpret_cast<const float4 *>(&Ws[kk][tx * 4]);
            const float xr[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
            const float wr[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(xr[i], wr[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const long long m = m0 + ty * 8 + i;
        if (m >= M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx * 4 + j;
            if (n < N) P[m * N + n] = acc[i][j] + __ldg(bias + n);
        }
    }
}

}  // namespace

bool proj_tcgen05_supported(int x_dtype, int N, int K);
cudaError_t launch_proj_tcgen05(const void *x, const void *w_ih, const float *b_ih, float *P, long long M, int N,
                                int K, cudaStream_t s);

// bf16 operands with Din a multiple of 64 and 3D a multiple of 256 take the
// tcgen05 kernel (proj_tcgen05.cu); everything else this CUDA-core kernel.
// P [M, N] = x [M, K] W^T + b, W [N, K] (x and W of dtype x_dtype).
cudaError_t launch_projection_n(int x_dtype, const void *x, const void *w_ih, const float *b_ih, float *P,
                                long long M, int N, int K, cudaStream_t s) {
    if (proj_tcgen05_supported(x_dtype, N, K)) return launch_proj_tcgen05(x, w_ih, b_ih, P, M, N, K, s);
    const dim3 grid(static_cast<unsigned>((M + BM - 1) / BM), (N + BN - 1) / BN);
    if (x_dtype == PARARNN_BF16)
        proj_gemm_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
            static_cast<const __nv_bfloat16 *>(x), static_cast<const __nv_bfloat16 *>(w_ih), b_ih,
            P, M, N, K);
    else
        proj_gemm_kernel<float><<<grid, 256, 0, s>>>(static_cast<const float *>(x),
                                                     static_cast<const float *>(w_ih), b_ih, P, M,
                                                     N, K);
    return cudaGetLastError();
}

// The GRU's projection: N = 3D gate rows.
cudaError_t launch_projection(const pararnn_cell &cell, const void *x, const void *w_ih,
                              const float *b_ih, float *P, long long M, cudaStream_t s) {
    return launch_projection_n(cell.x_dtype, x, w_ih, b_ih, P, M, 3 * cell.d, cell.din, s);
}

}  // namespace pararnn

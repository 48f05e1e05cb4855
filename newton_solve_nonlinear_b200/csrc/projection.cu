// projection.cu -- input pre-activations P = x W_ih^T + b_ih for every step.
//
// The input projection does not depend on the state, so it is computed once
// per solve for all (b, t) as one GEMM [B*T, Din] x [Din, 3D] -> [B*T, 3D]
// (fp32 accumulate, fp32 output), and every Newton iteration reads P.
//
// This file holds the general CUDA-core kernel: shared-memory tiles of
// 128 x 64 outputs, 8 x 4 outputs per thread, packed fp32x2 FMAs.  It takes fp32 or
// bf16 operands (bf16 is widened to fp32 on the way into shared memory) and
// any Din; it keeps fp32 inputs exact to fp32 rounding, which matters because
// the fixed point of the iteration is set by P as evaluated.
#include <cuda_bf16.h>

#include "common.cuh"
#include "solver.cuh"

namespace pararnn {
namespace {

constexpr int BM = 128, BN = 64, BK = 16;
constexpr int XPT = BM * BK / 256, WPT = BN * BK / 256;  // staged elements per thread: 8 and 4

__device__ __forceinline__ float widen(float v) { return v; }
__device__ __forceinline__ float widen(__nv_bfloat16 v) { return __bfloat162float(v); }

// The k-slice k0 .. k0+BK-1 of the CTA's x rows and W rows, into registers
// (zero outside the matrices).  VEC: K % 4 == 0 and fp32, so a thread fetches
// 4 consecutive k of a row as one float4.
template <typename Tin, bool VEC>
__device__ __forceinline__ void fetch_slice(const Tin *__restrict__ X, const Tin *__restrict__ W, long long m0,
                                            int n0, int k0, long long M, int N, int K, float (&xr)[XPT],
                                            float (&wr)[WPT]) {
    const int tid = threadIdx.x;
    if constexpr (VEC) {
#pragma unroll
        for (int s = 0; s < XPT / 4; ++s) {  // 128 rows x 4 float4
            const int i = tid + s * 256, r = i / (BK / 4), kq = i % (BK / 4);
            const long long m = m0 + r;
            const int k = k0 + 4 * kq;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (m < M && k < K) v = __ldcs(reinterpret_cast<const float4 *>(X + m * K + k));
            xr[4 * s] = v.x, xr[4 * s + 1] = v.y, xr[4 * s + 2] = v.z, xr[4 * s + 3] = v.w;
        }
        {  // 64 rows x 4 float4: one per thread
            const int r = tid / (BK / 4), kq = tid % (BK / 4);
            const int n = n0 + r, k = k0 + 4 * kq;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (n < N && k < K) v = __ldg(reinterpret_cast<const float4 *>(W + static_cast<long long>(n) * K + k));
            wr[0] = v.x, wr[1] = v.y, wr[2] = v.z, wr[3] = v.w;
        }
    } else {
#pragma unroll
        for (int s = 0; s < XPT; ++s) {
            const int i = tid + s * 256, r = i / BK, kk = i % BK;
            const long long m = m0 + r;
            const int k = k0 + kk;
            xr[s] = (m < M && k < K) ? widen(X[m * K + k]) : 0.f;
        }
#pragma unroll
        for (int s = 0; s < WPT; ++s) {
            const int i = tid + s * 256, r = i / BK, kk = i % BK;
            const int n = n0 + r, k = k0 + kk;
            wr[s] = (n < N && k < K) ? widen(W[static_cast<long long>(n) * K + k]) : 0.f;
        }
    }
}

// Registers -> the shared tiles Xs[k][row], Ws[k][col] (transposed, so the
// inner loop reads rows and columns as float4).
template <bool VEC>
__device__ __forceinline__ void put_slice(float (*Xs)[BM + 4], float (*Ws)[BN + 4], const float (&xr)[XPT],
                                          const float (&wr)[WPT]) {
    const int tid = threadIdx.x;
    if constexpr (VEC) {
#pragma unroll
        for (int s = 0; s < XPT / 4; ++s) {
            const int i = tid + s * 256, r = i / (BK / 4), kq = i % (BK / 4);
#pragma unroll
            for (int e = 0; e < 4; ++e) Xs[4 * kq + e][r] = xr[4 * s + e];
        }
        const int r = tid / (BK / 4), kq = tid % (BK / 4);
#pragma unroll
        for (int e = 0; e < 4; ++e) Ws[4 * kq + e][r] = wr[e];
    } else {
#pragma unroll
        for (int s = 0; s < XPT; ++s) {
            const int i = tid + s * 256;
            Xs[i % BK][i / BK] = xr[s];
        }
#pragma unroll
        for (int s = 0; s < WPT; ++s) {
            const int i = tid + s * 256;
            Ws[i % BK][i / BK] = wr[s];
        }
    }
}

// 128 x 64 outputs per CTA, 8 rows x 4 columns per thread accumulated as
// row pairs on packed fp32x2 FMAs; the next k-slice is fetched into registers
// while the current one is multiplied (two shared buffers, one barrier per
// slice).
template <typename Tin, bool VEC>
__global__ void __launch_bounds__(256, VEC ? 3 : 2) proj_gemm_kernel(const Tin *__restrict__ X,
                                                        const Tin *__restrict__ W,
                                                        const float *__restrict__ bias,
                                                        float *__restrict__ P, long long M, int N,
                                                        int K) {
    __shared__ __align__(16) float Xs[2][BK][BM + 4];
    __shared__ __align__(16) float Ws[2][BK][BN + 4];
    const int tid = threadIdx.x;
    const int tx = tid % 16, ty = tid / 16;  // 16 x 16 threads; thread = 8 rows x 4 cols
    const long long m0 = static_cast<long long>(blockIdx.x) * BM;
    const int n0 = blockIdx.y * BN;
    u64 acc[4][4];  // [row pair][column]: rows (ty*8 + 2p, ty*8 + 2p + 1)
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[p][j] = 0ull;

    float xr[XPT], wr[WPT];
    fetch_slice<Tin, VEC>(X, W, m0, n0, 0, M, N, K, xr, wr);
    put_slice<VEC>(Xs[0], Ws[0], xr, wr);
    __syncthreads();
    const int nk = (K + BK - 1) / BK;
    for (int ks = 0; ks < nk; ++ks) {
        const int cur = ks & 1;
        if (ks + 1 < nk) fetch_slice<Tin, VEC>(X, W, m0, n0, (ks + 1) * BK, M, N, K, xr, wr);
#pragma unroll
        for (int kk = 0; kk < BK; ++kk) {
            const float4 xa = *reinterpret_cast<const float4 *>(&Xs[cur][kk][ty * 8]);
            const float4 xb = *reinterpret_cast<const float4 *>(&Xs[cur][kk][ty * 8 + 4]);
            const float4 wv = *reinterpret_cast<const float4 *>(&Ws[cur][kk][tx * 4]);
            const u64 xp[4] = {pk(xa.x, xa.y), pk(xa.z, xa.w), pk(xb.x, xb.y), pk(xb.z, xb.w)};
            const u64 ws[4] = {splat(wv.x), splat(wv.y), splat(wv.z), splat(wv.w)};
#pragma unroll
            for (int p = 0; p < 4; ++p)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[p][j] = fma2(xp[p], ws[j], acc[p][j]);
        }
        if (ks + 1 < nk) put_slice<VEC>(Xs[cur ^ 1], Ws[cur ^ 1], xr, wr);
        __syncthreads();
    }
    const int nb = n0 + tx * 4;
    float bv[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) bv[j] = nb + j < N ? __ldg(bias + nb + j) : 0.f;
    const bool vec_out = (N % 4 == 0) && nb + 3 < N;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        float lo[4], hi[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) upk(acc[p][j], lo[j], hi[j]);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const long long m = m0 + ty * 8 + 2 * p + h;
            if (m >= M) continue;
            const float *v = h ? hi : lo;
            if (vec_out) {
                __stcs(reinterpret_cast<float4 *>(P + m * N + nb),
                       make_float4(v[0] + bv[0], v[1] + bv[1], v[2] + bv[2], v[3] + bv[3]));
            } else {
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (nb + j < N) P[m * N + nb + j] = v[j] + bv[j];
            }
        }
    }
}

}  // namespace

bool proj_tcgen05_supported(int x_dtype, int N, int K);
bool proj_tf32_supported(int x_dtype, long long M, int N, int K, const void *x, const void *P);
cudaError_t launch_proj_tf32(const float *x, const float *w, const float *b, float *P, long long M, int N, int K,
                             cudaStream_t s);
cudaError_t launch_proj_tcgen05(const void *x, const void *w_ih, const float *b_ih, float *P, long long M, int N,
                                int K, cudaStream_t s);

// bf16 operands with Din a multiple of 64 and 3D a multiple of 256 take the
// tcgen05 kernel (proj_tcgen05.cu); everything else this CUDA-core kernel.
// P [M, N] = x [M, K] W^T + b, W [N, K] (x and W of dtype x_dtype).
cudaError_t launch_projection_n(int x_dtype, const void *x, const void *w_ih, const float *b_ih, float *P,
                                long long M, int N, int K, cudaStream_t s) {
    if (proj_tcgen05_supported(x_dtype, N, K)) return launch_proj_tcgen05(x, w_ih, b_ih, P, M, N, K, s);
    if (proj_tf32_supported(x_dtype, M, N, K, x, P))
        return launch_proj_tf32(static_cast<const float *>(x), static_cast<const float *>(w_ih), b_ih, P, M, N, K, s);
    const dim3 grid(static_cast<unsigned>((M + BM - 1) / BM), (N + BN - 1) / BN);
    const bool vec = K % 4 == 0 && reinterpret_cast<uintptr_t>(x) % 16 == 0 &&
                     reinterpret_cast<uintptr_t>(w_ih) % 16 == 0;
    if (x_dtype == PARARNN_BF16)
        proj_gemm_kernel<__nv_bfloat16, false><<<grid, 256, 0, s>>>(
            static_cast<const __nv_bfloat16 *>(x), static_cast<const __nv_bfloat16 *>(w_ih), b_ih,
            P, M, N, K);
    else if (vec)
        proj_gemm_kernel<float, true><<<grid, 256, 0, s>>>(static_cast<const float *>(x),
                                                           static_cast<const float *>(w_ih), b_ih, P, M, N, K);
    else
        proj_gemm_kernel<float, false><<<grid, 256, 0, s>>>(static_cast<const float *>(x),
                                                            static_cast<const float *>(w_ih), b_ih, P, M, N, K);
    return cudaGetLastError();
}

// The GRU's projection: N = 3D gate rows.
cudaError_t launch_projection(const pararnn_cell &cell, const void *x, const void *w_ih,
                              const float *b_ih, float *P, long long M, cudaStream_t s) {
    return launch_projection_n(cell.x_dtype, x, w_ih, b_ih, P, M, 3 * cell.d, cell.din, s);
}

}  // namespace pararnn

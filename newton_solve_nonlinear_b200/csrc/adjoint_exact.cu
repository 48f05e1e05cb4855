// adjoint_exact.cu -- the exact backward pass of the dense GRU: the reverse-time
// adjoint with the full transposed Jacobian,
//   lam_T = g_T,  lam_t = g_t + J_{t+1}^T lam_{t+1}   (g = dL/dh),
// followed by the per-step partials of f for the input pre-activations, the
// initial state and the recurrent parameters.
//
// The pages train with the Jacobian's diagonal in the backward pass ("Towards
// Scalable and Stable Parallelization of Nonlinear RNNs", atlas summary, table
// of measured effects); this pass gives the exact gradients of the evaluated
// sequence for comparison and for callers that need them.  The reverse
// recurrence is a linear recurrence with dense D x D matrices, i.e. the same
// block scan as a DEER step, run on reversed time: with s = T - 1 - t,
//   mu_s = J_{T-s}^T mu_{s-1} + g_{T-1-s},  mu_0 = g_{T-1},  lam_t = mu_{T-1-t}.
// So the pass materialises A_s = J_{T-s}^T (built from the cell's gates at the
// evaluated states and the recurrent matrices) and b_s, runs the library's
// dense affine scan, and reads lam back in reverse.  Memory: B T D^2 floats for
// the matrices (17 GB at B = 16, T = 65536, D = 64).
//
// Gates and partials follow the GRU of include/pararnn.h (rows r, z, n): with
// G = U h_{t-1} + b_hh,
//   r = sig(P_r + G_r), z = sig(P_z + G_z), n = tanh(P_n + r G_n),
//   J = diag(z) + diag((h_{t-1} - n) z (1 - z)) U_z + diag((1 - z)(1 - n^2) r) U_n
//       + diag((1 - z)(1 - n^2) G_n r (1 - r)) U_r,
//   dP_r = lam (1 - z)(1 - n^2) G_n r (1 - r), dP_z = lam (h_{t-1} - n) z (1 - z),
//   dP_n = lam (1 - z)(1 - n^2); the recurrent pre-activation gradients (dP_r,
//   dP_z, dP_n r) give dW_hh (their outer products with h_{t-1}) and db_hh.
#include "common.cuh"
#include "solver.cuh"

namespace pararnn {

cudaError_t launch_scan_dense(const float *A, const float *b, const float *h0, int B, int T, int D, float *h,
                              void *ws, cudaStream_t s);
size_t scan_dense_ws_bytes(int B, int T, int D);
cudaError_t launch_projection_n(int x_dtype, const void *x, const void *w_ih, const float *b_ih, float *P,
                                long long M, int N, int K, cudaStream_t s);
cudaError_t launch_outer_sum(const float *grow, const float *hp, long long M, int N, int K, float *part, float *out,
                             cudaStream_t s);
size_t adjoint_outer_part_bytes(long long M, int N, int K);
cudaError_t launch_sum_rows(const float *in, int rows, int n, float *out, cudaStream_t s);

namespace {

constexpr int kXT = 256;       // threads of the build and gradient kernels
constexpr int kColRows = 2048; // rows per block of the db_hh column sums

struct AdjxArgs {
    const float *P, *G, *hp, *dh, *w_hh, *mu;
    float *Arev, *brev, *dP, *grow, *dh0;
    int B, T, D;
};

// Gates of (b, t, i) at the evaluated state: r, z, n and G_n.
__device__ __forceinline__ void gates(const AdjxArgs &S, size_t row, int i, float &r, float &z, float &n,
                                      float &gn) {
    const int D = S.D;
    const float *p = S.P + row * 3 * D, *g = S.G + row * 3 * D;
    r = sigmoidf_(p[i] + g[i]);
    z = sigmoidf_(p[D + i] + g[D + i]);
    gn = g[2 * D + i];
    n = tanhf_(p[2 * D + i] + r * gn);
}

// A_s = J_{T-s}^T (zero for s = 0) and b_s = g_{T-1-s}, for every sequence and
// reversed step; U_r, U_z, U_n are staged in shared memory once per block.
__global__ void __launch_bounds__(kXT) adjx_build_kernel(AdjxArgs S) {
    extern __shared__ float us[];  // [3][D][D + 1]: U_g[i][k]
    __shared__ float cf[4][64];    // z, cz, cn, cr of the step
    const int D = S.D, T = S.T, DP = D + 1;
    for (int q = threadIdx.x; q < 3 * D * D; q += kXT) {
        const int g = q / (D * D), i = (q / D) % D, k = q % D;
        us[(g * D + i) * DP + k] = __ldg(S.w_hh + q);
    }
    __syncthreads();
    const long long n_steps = static_cast<long long>(S.B) * T;
    for (long long q = blockIdx.x; q < n_steps; q += gridDim.x) {
        const int b = static_cast<int>(q / T), s = static_cast<int>(q % T);
        const size_t out = static_cast<size_t>(q);
        for (int i = threadIdx.x; i < D; i += kXT)
            S.brev[out * D + i] = __ldg(S.dh + (static_cast<size_t>(b) * T + (T - 1 - s)) * D + i);
        float *A = S.Arev + out * D * D;
        if (s == 0) {
            for (int e = threadIdx.x; e < D * D; e += kXT) A[e] = 0.f;
            continue;  // uniform across the block
        }
        const size_t row = static_cast<size_t>(b) * T + (T - s);  // the step whose Jacobian enters
        if (threadIdx.x < D) {
            const int i = threadIdx.x;
            float r, z, n, gn;
            gates(S, row, i, r, z, n, gn);
            const float hprev = S.hp[row * D + i];
            const float omz = 1.f - z;
            const float cn = omz * (1.f - n * n) * r;
            cf[0][i] = z;
            cf[1][i] = (hprev - n) * z * omz;
            cf[2][i] = cn;
            cf[3][i] = cn * gn * (1.f - r);
        }
        __syncthreads();
        // A[k][i] = J[i][k] = z_i [i == k] + cz_i U_z[i][k] + cn_i U_n[i][k] + cr_i U_r[i][k]
        for (int e = threadIdx.x; e < D * D; e += kXT) {
            const int k = e / D, i = e % D;
            float v = cf[1][i] * us[(D + i) * DP + k];
            v = fmaf(cf[2][i], us[(2 * D + i) * DP + k], v);
            v = fmaf(cf[3][i], us[i * DP + k], v);
            if (i == k) v += cf[0][i];
            __stcs(A + e, v);
        }
        __syncthreads();  // cf is rewritten by the next step
    }
}

// dP and the recurrent pre-activation gradients of every (b, t, i), from
// lam_t = mu_{T-1-t}.
__global__ void __launch_bounds__(kXT) adjx_grads_kernel(AdjxArgs S) {
    const int D = S.D, T = S.T;
    const long long n = static_cast<long long>(S.B) * T * D;
    for (long long q = static_cast<long long>(blockIdx.x) * kXT + threadIdx.x; q < n;
         q += static_cast<long long>(gridDim.x) * kXT) {
        const int i = static_cast<int>(q % D);
        const long long row = q / D;
        const int b = static_cast<int>(row / T), t = static_cast<int>(row % T);
        const float lam = __ldcs(S.mu + (static_cast<size_t>(b) * T + (T - 1 - t)) * D + i);
        float r, z, nn, gn;
        gates(S, static_cast<size_t>(row), i, r, z, nn, gn);
        const float hprev = S.hp[row * D + i];
        const float omz = 1.f - z;
        const float dpn = lam * omz * (1.f - nn * nn);
        const float dpr = dpn * gn * r * (1.f - r);
        const float dpz = lam * (hprev - nn) * z * omz;
        float *dp = S.dP + static_cast<size_t>(row) * 3 * D, *gw = S.grow + static_cast<size_t>(row) * 3 * D;
        __stcs(dp + i, dpr);
        __stcs(dp + D + i, dpz);
        __stcs(dp + 2 * D + i, dpn);
        __stcs(gw + i, dpr);
        __stcs(gw + D + i, dpz);
        __stcs(gw + 2 * D + i, dpn * r);
    }
}

// dh0[b] = J_0^T lam_0 (the Jacobian of the first step, at h0): one block per sequence.
__global__ void __launch_bounds__(kXT) adjx_dh0_kernel(AdjxArgs S) {
    __shared__ float w[4][64];  // z lam, cz lam, cn lam, cr lam
    const int D = S.D, T = S.T, b = blockIdx.x;
    const size_t row = static_cast<size_t>(b) * T;  // step 0 of sequence b
    if (threadIdx.x < D) {
        const int i = threadIdx.x;
        const float lam = S.mu[(row + T - 1) * D + i];
        float r, z, n, gn;
        gates(S, row, i, r, z, n, gn);
        const float hprev = S.hp[row * D + i];
        const float omz = 1.f - z;
        const float cn = omz * (1.f - n * n) * r;
        w[0][i] = z * lam;
        w[1][i] = (hprev - n) * z * omz * lam;
        w[2][i] = cn * lam;
        w[3][i] = cn * gn * (1.f - r) * lam;
    }
    __syncthreads();
    if (threadIdx.x < D) {
        const int k = threadIdx.x;
        float v = w[0][k];
        for (int i = 0; i < D; ++i) {
            v = fmaf(w[1][i], __ldg(S.w_hh + (static_cast<size_t>(D) + i) * D + k), v);
            v = fmaf(w[2][i], __ldg(S.w_hh + (static_cast<size_t>(2 * D) + i) * D + k), v);
            v = fmaf(w[3][i], __ldg(S.w_hh + static_cast<size_t>(i) * D + k), v);
        }
        S.dh0[static_cast<size_t>(b) * D + k] = v;
    }
}

// Column sums of grow over a block of kColRows rows (db_hh, in a fixed order).
__global__ void __launch_bounds__(kXT) adjx_colsum_kernel(const float *grow, long long rows, int n, float *part) {
    const long long r0 = static_cast<long long>(blockIdx.x) * kColRows;
    const long long r1 = min(rows, r0 + kColRows);
    for (int c = threadIdx.x; c < n; c += kXT) {
        float acc = 0.f;
        for (long long r = r0; r < r1; ++r) acc += __ldcs(grow + r * n + c);
        part[static_cast<size_t>(blockIdx.x) * n + c] = acc;
    }
}

size_t al256x(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct AdjxLayout {
    size_t hp, G, Arev, brev, mu, h0z, scan, grow, opart, cpart, total;
};

AdjxLayout adjx_layout(int B, int T, int D) {
    AdjxLayout L{};
    const size_t st = static_cast<size_t>(B) * T * D * 4;
    const long long M = static_cast<long long>(B) * T;
    size_t off = 0;
    L.hp = off; off = al256x(off + st);
    L.G = off; off = al256x(off + 3 * st);
    L.Arev = off; off = al256x(off + st * D);
    L.brev = off; off = al256x(off + st);
    L.mu = off; off = al256x(off + st);
    L.h0z = off; off = al256x(off + static_cast<size_t>(B) * D * 4);
    L.scan = off; off = al256x(off + scan_dense_ws_bytes(B, T, D));
    L.grow = off; off = al256x(off + 3 * st);
    L.opart = off; off = al256x(off + adjoint_outer_part_bytes(M, 3 * D, D));
    L.cpart = off; off = al256x(off + static_cast<size_t>((M + kColRows - 1) / kColRows) * 3 * D * 4);
    L.total = off;
    return L;
}

}  // namespace

size_t adjoint_exact_ws_bytes(int B, int T, int D) { return adjx_layout(B, T, D).total; }

cudaError_t adjoint_exact_enqueue(const float *w_hh, const float *b_hh, const float *P, const float *h0,
                                  const float *h, const float *dh, int B, int T, int D, float *dP, float *dh0,
                                  float *dw_hh, float *db_hh, void *workspace, cudaStream_t s) {
    const AdjxLayout L = adjx_layout(B, T, D);
    char *ws = static_cast<char *>(workspace);
    AdjxArgs S;
    S.P = P; S.dh = dh; S.w_hh = w_hh;
    S.B = B; S.T = T; S.D = D;
    float *hp = reinterpret_cast<float *>(ws + L.hp), *G = reinterpret_cast<float *>(ws + L.G);
    S.hp = hp; S.G = G;
    S.Arev = reinterpret_cast<float *>(ws + L.Arev);
    S.brev = reinterpret_cast<float *>(ws + L.brev);
    float *mu = reinterpret_cast<float *>(ws + L.mu);
    S.mu = mu;
    S.dP = dP; S.grow = reinterpret_cast<float *>(ws + L.grow); S.dh0 = dh0;
    // h_{t-1} packed: h0, then the states shifted by one step
    const size_t row = static_cast<size_t>(D) * 4, seq = static_cast<size_t>(T) * D * 4;
    cudaError_t e = cudaMemcpy2DAsync(hp, seq, h0, row, row, B, cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess && T > 1)
        e = cudaMemcpy2DAsync(reinterpret_cast<char *>(hp) + row, seq, h, seq, seq - row, B, cudaMemcpyDeviceToDevice,
                              s);
    // G = U h_{t-1} + b_hh for every step: one fp32 GEMM
    const long long M = static_cast<long long>(B) * T;
    if (e == cudaSuccess) e = launch_projection_n(PARARNN_F32, hp, w_hh, b_hh, G, M, 3 * D, D, s);
    // the reversed recurrence's matrices and inputs
    const int smem = 3 * D * (D + 1) * 4;
    if (e == cudaSuccess) e = cudaFuncSetAttribute(adjx_build_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    int dev = 0, nsm = 0;
    if (e == cudaSuccess) e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const long long nb = min(M, static_cast<long long>(nsm) * 8);
    adjx_build_kernel<<<static_cast<unsigned>(nb), kXT, smem, s>>>(S);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // mu = the dense scan over reversed time from zero
    float *h0z = reinterpret_cast<float *>(ws + L.h0z);
    if ((e = cudaMemsetAsync(h0z, 0, static_cast<size_t>(B) * D * 4, s)) != cudaSuccess) return e;
    if ((e = launch_scan_dense(S.Arev, S.brev, h0z, B, T, D, mu, ws + L.scan, s)) != cudaSuccess) return e;
    // dP, the recurrent pre-activation gradients, dh0
    const long long ng = min((M * D + kXT - 1) / kXT, static_cast<long long>(nsm) * 16);
    adjx_grads_kernel<<<static_cast<unsigned>(ng), kXT, 0, s>>>(S);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    adjx_dh0_kernel<<<static_cast<unsigned>(B), kXT, 0, s>>>(S);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // dW_hh = sum of grow (outer) h_{t-1}; db_hh = sum of grow; both in a fixed order
    if ((e = launch_outer_sum(S.grow, hp, M, 3 * D, D, reinterpret_cast<float *>(ws + L.opart), dw_hh, s)) !=
        cudaSuccess)
        return e;
    const long long nc = (M + kColRows - 1) / kColRows;
    float *cpart = reinterpret_cast<float *>(ws + L.cpart);
    adjx_colsum_kernel<<<static_cast<unsigned>(nc), kXT, 0, s>>>(S.grow, M, 3 * D, cpart);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    return launch_sum_rows(cpart, static_cast<int>(nc), 3 * D, db_hh, s);
}

}  // namespace pararnn

// newton_dense_elk.cu -- ELK (full-Jacobian Levenberg-Marquardt step) on the
// dense GRU.
//
// ELK ("Towards Scalable and Stable Parallelization of Nonlinear RNNs",
// abstract and "Approach") damps each DEER step with a trust region and
// observes that the damped step is the posterior mean of a linear-Gaussian
// state-space model (a Kalman smoother).  With the linearisation at the guess
// y = h^(i) (J_t, residual r_t = y_t - f(y_{t-1}, x_t)) the step dh = h - y
// minimises
//     sum_t |dh_t - J_t dh_{t-1} + r_t|^2 + lambda sum_t |dh_t|^2,  dh_0 = 0,
// i.e. the Kalman model with unit process noise and observation noise 1/lambda.
// Its normal equations are block tridiagonal and symmetric positive definite:
//     M_t dh_t - L_t dh_{t-1} - L_{t+1}^T dh_{t+1} = c_t,
//     M_t = (1 + lambda) I + J_{t+1}^T J_{t+1}   (the J term absent at t = T),
//     L_t = J_t (L_1 = 0),   c_t = -r_t + J_{t+1}^T r_{t+1}.
// The smoother's posterior mean is the unique solution of this system, so any
// exact solver gives the same step.  The pages only ask for a parallel
// smoother; this file solves the system by block cyclic reduction, which is
// parallel over the sequence (log2 T levels, every level a batch of
// independent D x D inversions and products):
//   level l (stride s = 2^l) holds rows k = 1..n, n = floor(T / s), at the
//   0-based steps j = k s - 1.  Odd rows are eliminated:
//     F1 (odd k):  G1_j = M_j^-1 L_j,  G2_j = M_j^-1 L_{j+s}^T,  g_j = M_j^-1 c_j
//     F2 (even k): M_j -= L_j G2_{j-s} + L_{j+s}^T G1_{j+s}
//                  c_j += L_j g_{j-s} + L_{j+s}^T g_{j+s}
//                  L_j <- L_j G1_{j-s}
//   which leaves the same kind of system on the even rows.  Back-substitution
//   from the top level down: dh_j = g_j + G1_j dh_{j-s} + G2_j dh_{j+s}.
// Each step j is eliminated at exactly one level, so G1 overwrites M_j, g
// overwrites c_j and every dh_j is produced once.  The inversions are in-place
// Gauss-Jordan without pivoting, which is stable here because every M on
// every level is symmetric positive definite (a Schur complement of the
// positive definite normal matrix).
//
// One cooperative persistent launch runs every Newton iteration: linearise,
// 2 grid barriers per reduction level, one per back-substitution level, and
// the convergence test (max |dh| <= tol) on the device.  fp32 throughout; the
// D x D products are CUDA-core FMAs (this mode is the accuracy reference of
// the damped family, not a throughput path).
#include "common.cuh"
#include "solver.cuh"

namespace pararnn {

static size_t al256e(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

static int elk_dmax(int D) { return D <= 8 ? 8 : (D <= 16 ? 16 : (D <= 32 ? 32 : 64)); }

// M/G1, L, G2: 3 x [B, T, DMAX, DMAX]; c/g and dh: 2 x [B, T, DMAX].
size_t dense_elk_ws_bytes(int B, int T, int D) {
    const size_t dm = elk_dmax(D);
    const size_t rows = static_cast<size_t>(B) * T;
    return 3 * al256e(rows * dm * dm * 4) + 2 * al256e(rows * dm * 4);
}

namespace {

constexpr int kCh = 16;  // steps per linearisation work item

template <int DMAX>
struct EG {
    static constexpr int LD = DMAX + 4;  // shared-memory row stride (floats; rows stay 16-B aligned)
    static constexpr int RB = DMAX >= 32 ? DMAX / 16 : 1;  // RB x RB entries per thread
    static constexpr int TG = DMAX / RB;                   // TG x TG threads own a block
    static constexpr int NT = TG * TG;
    static constexpr int MAT = DMAX * LD;
    static constexpr size_t MM = static_cast<size_t>(DMAX) * DMAX;  // floats per global matrix
    // shared memory (floats): U_r, U_z, U_n | union(linearise, reduction) | vectors
    static constexpr int LIN = (kCh + 2) * DMAX + 5 * (kCh + 1) * DMAX + MAT;
    static constexpr int RED = 3 * MAT;
    static constexpr int WORK = LIN > RED ? LIN : RED;
    static constexpr int VEC = 4 * DMAX;
    static constexpr size_t SMEM = (3 * MAT + WORK + VEC + 32) * sizeof(float);
};

struct ElkArgs {
    DiagArgs a;
    float *Mb;   // M_j, then G1_j once j is eliminated       [B, T, DMAX, DMAX]
    float *Lb;   // coupling of row j to its left neighbour    [B, T, DMAX, DMAX]
    float *G2b;  // G2_j                                       [B, T, DMAX, DMAX]
    float *cv;   // c_j, then g_j                              [B, T, DMAX]
    float *dv;   // dh_j                                       [B, T, DMAX]
};

template <int DMAX>
__device__ __forceinline__ void blk_origin(int &i0, int &j0) {
    i0 = (threadIdx.x / EG<DMAX>::TG) * EG<DMAX>::RB;
    j0 = (threadIdx.x % EG<DMAX>::TG) * EG<DMAX>::RB;
}

// global [DMAX][DMAX] -> shared [DMAX][LD]
template <int DMAX>
__device__ __forceinline__ void stage(float *s, const float *g) {
    constexpr int V = DMAX / 4;
    for (int q = threadIdx.x; q < DMAX * V; q += kThreads) {
        const int r = q / V, c4 = q % V;
        *reinterpret_cast<float4 *>(s + r * EG<DMAX>::LD + c4 * 4) = ldcg4(g + 4 * q);
    }
}

// global [DMAX][DMAX] -> shared transposed: s[c][r] = g[r][c]
template <int DMAX>
__device__ __forceinline__ void stage_t(float *s, const float *g) {
    for (int q = threadIdx.x; q < DMAX * DMAX; q += kThreads) {
        const int r = q / DMAX, c = q % DMAX;
        s[c * EG<DMAX>::LD + r] = __ldcg(g + q);
    }
}

template <int DMAX>
__device__ __forceinline__ void zero_acc(float (&acc)[EG<DMAX>::RB][EG<DMAX>::RB]) {
#pragma unroll
    for (int a = 0; a < EG<DMAX>::RB; ++a)
#pragma unroll
        for (int c = 0; c < EG<DMAX>::RB; ++c) acc[a][c] = 0.f;
}

// acc += X Y over the thread's block (X, Y shared, row-major with stride LD).
template <int DMAX>
__device__ __forceinline__ void mm_nn(float (&acc)[EG<DMAX>::RB][EG<DMAX>::RB], const float *X,
                                      const float *Y, int i0, int j0) {
    constexpr int RB = EG<DMAX>::RB, LD = EG<DMAX>::LD;
#pragma unroll 4
    for (int k = 0; k < DMAX; ++k) {
        float xa[RB], yc[RB];
#pragma unroll
        for (int a = 0; a < RB; ++a) xa[a] = X[(i0 + a) * LD + k];
#pragma unroll
        for (int c = 0; c < RB; ++c) yc[c] = Y[k * LD + j0 + c];
#pragma unroll
        for (int a = 0; a < RB; ++a)
#pragma unroll
            for (int c = 0; c < RB; ++c) acc[a][c] = fmaf(xa[a], yc[c], acc[a][c]);
    }
}

// acc += X^T Y over the thread's block.
template <int DMAX>
__device__ __forceinline__ void mm_tn(float (&acc)[EG<DMAX>::RB][EG<DMAX>::RB], const float *X,
                                      const float *Y, int i0, int j0) {
    constexpr int RB = EG<DMAX>::RB, LD = EG<DMAX>::LD;
#pragma unroll 4
    for (int k = 0; k < DMAX; ++k) {
        float xa[RB], yc[RB];
#pragma unroll
        for (int a = 0; a < RB; ++a) xa[a] = X[k * LD + i0 + a];
#pragma unroll
        for (int c = 0; c < RB; ++c) yc[c] = Y[k * LD + j0 + c];
#pragma unroll
        for (int a = 0; a < RB; ++a)
#pragma unroll
            for (int c = 0; c < RB; ++c) acc[a][c] = fmaf(xa[a], yc[c], acc[a][c]);
    }
}

// Store the thread's block to a global [DMAX][DMAX] matrix.
template <int DMAX>
__device__ __forceinline__ void store_blk(float *g, const float (&acc)[EG<DMAX>::RB][EG<DMAX>::RB],
                                          int i0, int j0) {
    constexpr int RB = EG<DMAX>::RB;
#pragma unroll
    for (int a = 0; a < RB; ++a) {
        float *row = g + (i0 + a) * DMAX + j0;
        if constexpr (RB == 4) {
            stcg4(row, make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]));
        } else {
#pragma unroll
            for (int c = 0; c < RB; ++c) __stcg(row + c, acc[a][c]);
        }
    }
}

// In-place inverse of the shared matrix A (Gauss-Jordan, no pivoting; A is
// symmetric positive definite, so every pivot is a positive Schur complement
// diagonal).
template <int DMAX>
__device__ void gj_invert(float *A) {
    constexpr int RB = EG<DMAX>::RB, LD = EG<DMAX>::LD;
    const bool own = threadIdx.x < EG<DMAX>::NT;
    int i0 = 0, j0 = 0;
    blk_origin<DMAX>(i0, j0);
    for (int k = 0; k < DMAX; ++k) {
        float colk[RB], rowk[RB], p = 1.f;
        if (own) {
            p = A[k * LD + k];
#pragma unroll
            for (int a = 0; a < RB; ++a) colk[a] = A[(i0 + a) * LD + k];
#pragma unroll
            for (int c = 0; c < RB; ++c) rowk[c] = A[k * LD + j0 + c];
        }
        __syncthreads();
        if (own) {
            const float ip = 1.f / p;
#pragma unroll
            for (int a = 0; a < RB; ++a) {
                const int i = i0 + a;
#pragma unroll
                for (int c = 0; c < RB; ++c) {
                    const int j = j0 + c;
                    float v;
                    if (i == k)
                        v = (j == k) ? ip : rowk[c] * ip;
                    else if (j == k)
                        v = -colk[a] * ip;
                    else
                        v = fmaf(-colk[a] * ip, rowk[c], A[i * LD + j]);
                    A[i * LD + j] = v;
                }
            }
        }
        __syncthreads();
    }
}

template <int DMAX>
struct ElkSmem {
    float *U;    // U_r, U_z, U_n as [DMAX][LD] each
    float *ys;   // guess rows ts-1 .. ts+kCh          (kCh+2) x DMAX
    float *co;   // z, cz, cn, cr, r per step            5 x (kCh+1) x DMAX
    float *J;    // J_t                                  [DMAX][LD]
    float *S0, *S1, *S2;  // reduction operands (alias the linearisation buffers)
    float *v;    // 4 vectors of DMAX
    unsigned *red;
};

template <int DMAX>
__device__ ElkSmem<DMAX> elk_carve(float *p) {
    using G = EG<DMAX>;
    ElkSmem<DMAX> s;
    s.U = p; p += 3 * G::MAT;
    float *w = p;
    s.ys = w;
    s.co = w + (kCh + 2) * DMAX;
    s.J = s.co + 5 * (kCh + 1) * DMAX;
    s.S0 = w; s.S1 = w + G::MAT; s.S2 = w + 2 * G::MAT;
    p += G::WORK;
    s.v = p; p += G::VEC;
    s.red = reinterpret_cast<unsigned *>(p);
    return s;
}

// Linearise steps ts .. ts+n-1 of sequence b: L_t = J_t (0 at t = 0),
// M_t = (1+lambda) I + J_{t+1}^T J_{t+1}, c_t = -r_t + J_{t+1}^T r_{t+1}.
template <int DMAX>
__device__ void elk_linearise(const ElkArgs &S, const ElkSmem<DMAX> &sm, int b, int ts, int n,
                              const float *hold, bool zero_guess, unsigned &rmax) {
    using G = EG<DMAX>;
    constexpr int LD = G::LD, RB = G::RB;
    const DiagArgs &A = S.a;
    const int D = A.D, T = A.T;
    const float lam1 = 1.f + A.lambda;
    const int m = (ts + n < T) ? n + 1 : n;  // steps whose coefficients are needed
    // guess rows t = ts-1 .. ts+m-1 (row index t - ts + 1)
    for (int q = threadIdx.x; q < (m + 1) * DMAX; q += kThreads) {
        const int r = q / DMAX, col = q % DMAX, t = ts - 1 + r;
        float v = 0.f;
        if (col < D) {
            if (t < 0)
                v = __ldg(A.h0 + static_cast<size_t>(b) * D + col);
            else if (!zero_guess)
                v = __ldcg(hold + (static_cast<size_t>(b) * T + t) * D + col);
        }
        sm.ys[q] = v;
    }
    __syncthreads();
    // gate coefficients and residuals: thread (i, grp) for steps grp, grp+NG, ...
    {
        constexpr int NG = kThreads / DMAX;
        const int i = threadIdx.x % DMAX, grp = threadIdx.x / DMAX;
        for (int st = grp; st < m; st += NG) {
            float z = 0.f, cz = 0.f, cn = 0.f, cr = 0.f, res = 0.f;
            if (i < D) {
                const float *yp = sm.ys + st * DMAX;
                float g0 = 0.f, g1 = 0.f, g2 = 0.f;
#pragma unroll 4
                for (int k = 0; k < DMAX; k += 4) {
                    const float4 y4 = *reinterpret_cast<const float4 *>(yp + k);
                    const float4 u0 = *reinterpret_cast<const float4 *>(sm.U + 0 * G::MAT + i * LD + k);
                    const float4 u1 = *reinterpret_cast<const float4 *>(sm.U + 1 * G::MAT + i * LD + k);
                    const float4 u2 = *reinterpret_cast<const float4 *>(sm.U + 2 * G::MAT + i * LD + k);
                    g0 = fmaf(u0.x, y4.x, fmaf(u0.y, y4.y, fmaf(u0.z, y4.z, fmaf(u0.w, y4.w, g0))));
                    g1 = fmaf(u1.x, y4.x, fmaf(u1.y, y4.y, fmaf(u1.z, y4.z, fmaf(u1.w, y4.w, g1))));
                    g2 = fmaf(u2.x, y4.x, fmaf(u2.y, y4.y, fmaf(u2.z, y4.z, fmaf(u2.w, y4.w, g2))));
                }
                const int t = ts + st;
                const float *prow = A.P + (static_cast<size_t>(b) * T + t) * 3 * D + i;
                const float hp = yp[i];
                const float hc = sm.ys[(st + 1) * DMAX + i];
                const float r = sigmoidf_(__ldg(prow) + g0 + __ldg(A.b_hh + i));
                z = sigmoidf_(__ldg(prow + D) + g1 + __ldg(A.b_hh + D + i));
                const float gn = g2 + __ldg(A.b_hh + 2 * D + i);
                const float nn = tanhf_(__ldg(prow + 2 * D) + r * gn);
                const float f = nn + z * (hp - nn);
                const float omz = 1.f - z;
                cz = (hp - nn) * z * omz;
                cn = omz * (1.f - nn * nn) * r;
                cr = cn * gn * (1.f - r);
                res = hc - f;
                if (st < n) rmax = max(rmax, abs_bits(res));
            }
            sm.co[(0 * (kCh + 1) + st) * DMAX + i] = z;
            sm.co[(1 * (kCh + 1) + st) * DMAX + i] = cz;
            sm.co[(2 * (kCh + 1) + st) * DMAX + i] = cn;
            sm.co[(3 * (kCh + 1) + st) * DMAX + i] = cr;
            sm.co[(4 * (kCh + 1) + st) * DMAX + i] = res;
        }
    }
    __syncthreads();
    const bool own = threadIdx.x < G::NT;
    int i0 = 0, j0 = 0;
    blk_origin<DMAX>(i0, j0);
    const float *resv = sm.co + 4 * (kCh + 1) * DMAX;
    for (int st = 0; st < m; ++st) {
        const int t = ts + st;
        // J_t over the thread's block: z_i delta_ik + cz_i Uz_ik + cn_i Un_ik + cr_i Ur_ik
        if (own) {
#pragma unroll
            for (int a = 0; a < RB; ++a) {
                const int i = i0 + a;
                const float z = sm.co[(0 * (kCh + 1) + st) * DMAX + i];
                const float cz = sm.co[(1 * (kCh + 1) + st) * DMAX + i];
                const float cn = sm.co[(2 * (kCh + 1) + st) * DMAX + i];
                const float cr = sm.co[(3 * (kCh + 1) + st) * DMAX + i];
#pragma unroll
                for (int c = 0; c < RB; ++c) {
                    const int k = j0 + c;
                    float v = fmaf(cz, sm.U[1 * G::MAT + i * LD + k],
                                   fmaf(cn, sm.U[2 * G::MAT + i * LD + k],
                                        cr * sm.U[0 * G::MAT + i * LD + k]));
                    if (i == k) v += z;
                    sm.J[i * LD + k] = v;
                }
            }
        }
        __syncthreads();
        const size_t row = static_cast<size_t>(b) * T + t;
        if (st < n) {  // L_t = J_t (the coupling to dh_0 = 0 is dropped)
            float *dst = S.Lb + row * G::MM;
            constexpr int V = DMAX / 4;
            for (int q = threadIdx.x; q < DMAX * V; q += kThreads) {
                const int r = q / V, c4 = q % V;
                float4 v = *reinterpret_cast<const float4 *>(sm.J + r * LD + c4 * 4);
                if (t == 0) v = make_float4(0.f, 0.f, 0.f, 0.f);
                stcg4(dst + 4 * q, v);
            }
        }
        if (st >= 1) {  // M_{t-1}, c_{t-1} from J_t
            float acc[RB][RB];
            zero_acc<DMAX>(acc);
            if (own) {
                mm_tn<DMAX>(acc, sm.J, sm.J, i0, j0);
#pragma unroll
                for (int a = 0; a < RB; ++a)
#pragma unroll
                    for (int c = 0; c < RB; ++c)
                        if (i0 + a == j0 + c) acc[a][c] += lam1;
                store_blk<DMAX>(S.Mb + (row - 1) * G::MM, acc, i0, j0);
            }
            if (threadIdx.x < DMAX) {
                const int a = threadIdx.x;
                float s = -resv[(st - 1) * DMAX + a];
                for (int i = 0; i < DMAX; ++i) s = fmaf(sm.J[i * LD + a], resv[st * DMAX + i], s);
                __stcg(S.cv + (row - 1) * DMAX + a, s);
            }
        }
        if (st == n - 1 && t == T - 1) {  // last step of the sequence: no J_{t+1} term
            float acc[RB][RB];
            zero_acc<DMAX>(acc);
            if (own) {
#pragma unroll
                for (int a = 0; a < RB; ++a)
#pragma unroll
                    for (int c = 0; c < RB; ++c)
                        if (i0 + a == j0 + c) acc[a][c] = lam1;
                store_blk<DMAX>(S.Mb + row * G::MM, acc, i0, j0);
            }
            if (threadIdx.x < DMAX) __stcg(S.cv + row * DMAX + threadIdx.x, -resv[st * DMAX + threadIdx.x]);
        }
        __syncthreads();
    }
}

// F1 on step j (odd row of the level with stride s).
template <int DMAX>
__device__ void elk_eliminate(const ElkArgs &S, const ElkSmem<DMAX> &sm, size_t base, int j, int s,
                              bool right) {
    using G = EG<DMAX>;
    constexpr int RB = G::RB, LD = G::LD;
    const size_t row = base + j;
    stage<DMAX>(sm.S0, S.Mb + row * G::MM);
    stage<DMAX>(sm.S1, S.Lb + row * G::MM);
    if (right) stage_t<DMAX>(sm.S2, S.Lb + (row + s) * G::MM);
    if (threadIdx.x < DMAX) sm.v[threadIdx.x] = __ldcg(S.cv + row * DMAX + threadIdx.x);
    __syncthreads();
    gj_invert<DMAX>(sm.S0);
    int i0 = 0, j0 = 0;
    blk_origin<DMAX>(i0, j0);
    if (threadIdx.x < G::NT) {
        float acc[RB][RB];
        zero_acc<DMAX>(acc);
        mm_nn<DMAX>(acc, sm.S0, sm.S1, i0, j0);
        store_blk<DMAX>(S.Mb + row * G::MM, acc, i0, j0);  // G1 replaces M
        if (right) {
            zero_acc<DMAX>(acc);
            mm_nn<DMAX>(acc, sm.S0, sm.S2, i0, j0);
            store_blk<DMAX>(S.G2b + row * G::MM, acc, i0, j0);
        }
    }
    if (threadIdx.x < DMAX) {
        const int i = threadIdx.x;
        float g = 0.f;
        for (int k = 0; k < DMAX; ++k) g = fmaf(sm.S0[i * LD + k], sm.v[k], g);
        __stcg(S.cv + row * DMAX + i, g);  // g replaces c
    }
    __syncthreads();
}

// F2 on step j (even row of the level with stride s): fold in both neighbours.
template <int DMAX>
__device__ void elk_fold(const ElkArgs &S, const ElkSmem<DMAX> &sm, size_t base, int j, int s,
                         bool right) {
    using G = EG<DMAX>;
    constexpr int RB = G::RB, LD = G::LD;
    const size_t row = base + j, lrow = row - s, rrow = row + s;
    float *vc = sm.v, *vgl = sm.v + DMAX, *vgr = sm.v + 2 * DMAX;
    stage<DMAX>(sm.S0, S.Lb + row * G::MM);    // L_j
    stage<DMAX>(sm.S1, S.G2b + lrow * G::MM);  // G2_l
    stage<DMAX>(sm.S2, S.Mb + lrow * G::MM);   // G1_l
    if (threadIdx.x < DMAX) {
        vc[threadIdx.x] = __ldcg(S.cv + row * DMAX + threadIdx.x);
        vgl[threadIdx.x] = __ldcg(S.cv + lrow * DMAX + threadIdx.x);
        vgr[threadIdx.x] = right ? __ldcg(S.cv + rrow * DMAX + threadIdx.x) : 0.f;
    }
    __syncthreads();
    int i0 = 0, j0 = 0;
    blk_origin<DMAX>(i0, j0);
    const bool own = threadIdx.x < G::NT;
    float accM[RB][RB], accL[RB][RB];
    zero_acc<DMAX>(accM);
    zero_acc<DMAX>(accL);
    if (own) {
#pragma unroll 4
        for (int k = 0; k < DMAX; ++k) {
            float xa[RB], y1[RB], y2[RB];
#pragma unroll
            for (int a = 0; a < RB; ++a) xa[a] = sm.S0[(i0 + a) * LD + k];
#pragma unroll
            for (int c = 0; c < RB; ++c) {
                y1[c] = sm.S1[k * LD + j0 + c];
                y2[c] = sm.S2[k * LD + j0 + c];
            }
#pragma unroll
            for (int a = 0; a < RB; ++a)
#pragma unroll
                for (int c = 0; c < RB; ++c) {
                    accM[a][c] = fmaf(xa[a], y1[c], accM[a][c]);
                    accL[a][c] = fmaf(xa[a], y2[c], accL[a][c]);
                }
        }
    }
    float cnew = 0.f;
    if (threadIdx.x < DMAX) {
        const int i = threadIdx.x;
        cnew = vc[i];
        for (int k = 0; k < DMAX; ++k) cnew = fmaf(sm.S0[i * LD + k], vgl[k], cnew);
    }
    __syncthreads();
    if (right) {
        stage<DMAX>(sm.S1, S.Lb + rrow * G::MM);  // L_r
        stage<DMAX>(sm.S2, S.Mb + rrow * G::MM);  // G1_r
        __syncthreads();
        if (own) mm_tn<DMAX>(accM, sm.S1, sm.S2, i0, j0);
        if (threadIdx.x < DMAX) {
            const int i = threadIdx.x;
            for (int k = 0; k < DMAX; ++k) cnew = fmaf(sm.S1[k * LD + i], vgr[k], cnew);
        }
    }
    if (own) {
        float *Mj = S.Mb + row * G::MM;
#pragma unroll
        for (int a = 0; a < RB; ++a)
#pragma unroll
            for (int c = 0; c < RB; ++c) {
                const float mv = __ldcg(Mj + (i0 + a) * DMAX + j0 + c);
                accM[a][c] = mv - accM[a][c];
            }
        store_blk<DMAX>(Mj, accM, i0, j0);
        store_blk<DMAX>(S.Lb + row * G::MM, accL, i0, j0);
    }
    if (threadIdx.x < DMAX) __stcg(S.cv + row * DMAX + threadIdx.x, cnew);
    __syncthreads();
}

// Back-substitution of step j (odd row of the level with stride s); writes
// h^(i+1)_j = y_j + dh_j and folds max |dh| into dmax.
template <int DMAX>
__device__ void elk_backsub(const ElkArgs &S, const ElkSmem<DMAX> &sm, int b, int j, int s, bool left,
                            bool right, const float *hold, float *hnew, bool zero_guess,
                            unsigned &dmax) {
    using G = EG<DMAX>;
    const DiagArgs &A = S.a;
    const int D = A.D;
    const size_t base = static_cast<size_t>(b) * A.T, row = base + j;
    float *vl = sm.v, *vr = sm.v + DMAX, *vo = sm.v + 2 * DMAX;
    if (threadIdx.x < DMAX) {
        vl[threadIdx.x] = left ? __ldcg(S.dv + (row - s) * DMAX + threadIdx.x) : 0.f;
        vr[threadIdx.x] = right ? __ldcg(S.dv + (row + s) * DMAX + threadIdx.x) : 0.f;
    }
    __syncthreads();
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const float *G1 = S.Mb + row * G::MM, *G2 = S.G2b + row * G::MM;
    for (int i = warp; i < DMAX; i += kThreads / 32) {
        float acc = 0.f;
        for (int k = lane; k < DMAX; k += 32) {
            if (left) acc = fmaf(__ldcg(G1 + i * DMAX + k), vl[k], acc);
            if (right) acc = fmaf(__ldcg(G2 + i * DMAX + k), vr[k], acc);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) vo[i] = acc + __ldcg(S.cv + row * DMAX + i);
    }
    __syncthreads();
    if (threadIdx.x < DMAX) {
        const int i = threadIdx.x;
        const float d = vo[i];
        __stcg(S.dv + row * DMAX + i, d);
        if (i < D) {
            const size_t o = row * D + i;
            const float y = zero_guess ? 0.f : __ldcg(hold + o);
            __stcg(hnew + o, y + d);
            dmax = max(dmax, abs_bits(d));
        }
    }
    __syncthreads();
}

template <int DMAX>
__global__ void __launch_bounds__(kThreads, 2) dense_elk_kernel(ElkArgs S) {
    using G = EG<DMAX>;
    extern __shared__ float4 smem_raw[];
    const ElkSmem<DMAX> sm = elk_carve<DMAX>(reinterpret_cast<float *>(smem_raw));
    const DiagArgs &A = S.a;
    WsHeader *hdr = A.hdr;
    unsigned *status = &hdr->status;
    const unsigned nblocks = gridDim.x;
    const int D = A.D, T = A.T, B = A.B;
    // recurrent matrices U_g[i][k] = w_hh[g D + i][k], zero padded
    for (int q = threadIdx.x; q < 3 * DMAX * DMAX; q += kThreads) {
        const int g = q / (DMAX * DMAX), i = (q / DMAX) % DMAX, k = q % DMAX;
        sm.U[g * G::MAT + i * G::LD + k] =
            (i < D && k < D) ? __ldg(A.w_hh + (static_cast<size_t>(g) * D + i) * D + k) : 0.f;
    }
    __syncthreads();
    const int n_chunks = (T + kCh - 1) / kCh;
    const long long lin_items = static_cast<long long>(B) * n_chunks;
    int top = 1;
    while (2 * top <= T) top *= 2;

    int iters = 0, final_status = PARARNN_NOT_CONVERGED;
    unsigned last_delta = 0u, last_resid = 0u;
    for (int it = 0; it < A.max_iters; ++it) {
        if (blockIdx.x == 0 && threadIdx.x == 0) {
            hdr->delta_bits[(it + 1) % 3] = 0u;
            hdr->resid_bits[(it + 1) % 3] = 0u;
        }
        const float *hold = A.hbuf[it & 1];
        float *hnew = A.hbuf[(it + 1) & 1];
        const bool zero_guess = it == 0 && !A.warm;  // the first guess: zero, or the caller's
        unsigned dmax = 0u, rmax = 0u;
        for (long long w = blockIdx.x; w < lin_items; w += nblocks) {
            const int b = static_cast<int>(w / n_chunks), c = static_cast<int>(w % n_chunks);
            const int ts = c * kCh, n = min(kCh, T - ts);
            elk_linearise<DMAX>(S, sm, b, ts, n, hold, zero_guess, rmax);
        }
        grid_barrier(hdr->barrier, nblocks, status);
        // reduction levels
        for (int s = 1; s <= top; s *= 2) {
            const int n = T / s;
            const long long odd = (n + 1) / 2, even = n / 2;
            for (long long w = blockIdx.x; w < B * odd; w += nblocks) {
                const int b = static_cast<int>(w / odd);
                const int k = 2 * static_cast<int>(w % odd) + 1;
                elk_eliminate<DMAX>(S, sm, static_cast<size_t>(b) * T, k * s - 1, s, k < n);
            }
            grid_barrier(hdr->barrier, nblocks, status);
            if (even > 0) {
                for (long long w = blockIdx.x; w < B * even; w += nblocks) {
                    const int b = static_cast<int>(w / even);
                    const int k = 2 * static_cast<int>(w % even) + 2;
                    elk_fold<DMAX>(S, sm, static_cast<size_t>(b) * T, k * s - 1, s, k < n);
                }
                grid_barrier(hdr->barrier, nblocks, status);
            }
        }
        // back-substitution, top level first
        for (int s = top; s >= 1; s /= 2) {
            const int n = T / s;
            const long long odd = (n + 1) / 2;
            for (long long w = blockIdx.x; w < B * odd; w += nblocks) {
                const int b = static_cast<int>(w / odd);
                const int k = 2 * static_cast<int>(w % odd) + 1;
                elk_backsub<DMAX>(S, sm, b, k * s - 1, s, k > 1, k < n, hold, hnew, zero_guess,
                                  dmax);
            }
            grid_barrier(hdr->barrier, nblocks, status);
        }
        const unsigned bd = block_max_u32(dmax, sm.red);
        const unsigned br = block_max_u32(rmax, sm.red);
        if (threadIdx.x == 0) {
            atomicMax(&hdr->delta_bits[it % 3], bd);
            atomicMax(&hdr->resid_bits[it % 3], br);
        }
        grid_barrier(hdr->barrier, nblocks, status);
        last_delta = ld_acquire_u32(&hdr->delta_bits[it % 3]);
        last_resid = ld_acquire_u32(&hdr->resid_bits[it % 3]);
        record_trace(A, it, last_delta, last_resid);
        iters = it + 1;
        // a timeout another CTA raises may land between two threads' reads: decide once per CTA
        if (__syncthreads_or(timed_out(status))) { final_status = PARARNN_TIMEOUT; break; }
        if (last_delta >= 0x7f800000u) { final_status = PARARNN_DIVERGED; break; }
        if (__uint_as_float(last_delta) <= A.tol) { final_status = PARARNN_OK; break; }
    }
    if ((iters & 1) == 0 && iters > 0) {
        const size_t n4 = static_cast<size_t>(B) * T * D / 4;
        const float4 *src = reinterpret_cast<const float4 *>(A.hbuf[0]);
        float4 *dst = reinterpret_cast<float4 *>(A.hbuf[1]);
        for (size_t q = static_cast<size_t>(blockIdx.x) * kThreads + threadIdx.x; q < n4;
             q += static_cast<size_t>(nblocks) * kThreads)
            dst[q] = __ldcg(src + q);
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        pararnn_info info;
        info.iters = iters;
        info.status = final_status;
        info.delta = __uint_as_float(last_delta);
        info.residual = __uint_as_float(last_resid);
        *A.info_out = info;
        hdr->info = info;
    }
}

template <int DMAX>
cudaError_t launch_elk(const ElkArgs &S, cudaStream_t s) {
    auto kern = dense_elk_kernel<DMAX>;
    const size_t smem = EG<DMAX>::SMEM;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    int dev = 0, nsm = 0, per_sm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem)) !=
        cudaSuccess)
        return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    long long grid = static_cast<long long>(per_sm) * nsm;
    const long long need =
        static_cast<long long>(S.a.B) * ((S.a.T + kCh - 1) / kCh > (S.a.T + 1) / 2
                                             ? (S.a.T + kCh - 1) / kCh : (S.a.T + 1) / 2);
    if (grid > need) grid = need;
    ElkArgs args = S;
    void *params[] = {&args};
    return cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(kern),
                                       dim3(static_cast<unsigned>(grid)), dim3(kThreads), params,
                                       smem, s);
}

}  // namespace

cudaError_t launch_dense_elk(const DiagArgs &a, void *ws, cudaStream_t s) {
    const int dm = elk_dmax(a.D);
    const size_t rows = static_cast<size_t>(a.B) * a.T;
    char *p = static_cast<char *>(ws);
    ElkArgs S;
    S.a = a;
    S.Mb = reinterpret_cast<float *>(p); p += al256e(rows * dm * dm * 4);
    S.Lb = reinterpret_cast<float *>(p); p += al256e(rows * dm * dm * 4);
    S.G2b = reinterpret_cast<float *>(p); p += al256e(rows * dm * dm * 4);
    S.cv = reinterpret_cast<float *>(p); p += al256e(rows * dm * 4);
    S.dv = reinterpret_cast<float *>(p);
    switch (dm) {
        case 8: return launch_elk<8>(S, s);
        case 16: return launch_elk<16>(S, s);
        case 32: return launch_elk<32>(S, s);
        default: return launch_elk<64>(S, s);
    }
}

}  // namespace pararnn

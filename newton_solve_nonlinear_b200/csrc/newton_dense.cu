// newton_dense.cu -- dense-Jacobian DEER on the dense GRU, and the standalone
// dense affine scan h_t = A_t h_{t-1} + b_t with D x D matrices.
//
// DEER ("Towards Scalable and Stable Parallelization of Nonlinear RNNs",
// abstract; "Parallelizing non-linear sequential models over the sequence
// length", abstract) linearises the cell with its full Jacobian J_t and solves
// the block-bidiagonal system ("ParaRNN" summary, "Newton's Iteration") by a
// parallel scan whose elements are D x D matrices -- cubic in D per step, as
// the ELK abstract notes.
//
// The iteration is written in delta form: with the residual
// r_t = h^(i)_t - f(h^(i)_{t-1}, x_t), the update dh solves
//     dh_t = J_t dh_{t-1} - r_t,   dh_0 = 0,   h^(i+1) = h^(i) + dh,
// which is the same Newton step as the absolute form.  J_t is never stored:
// it is rebuilt on chip from the gate coefficients of the step and the
// recurrent matrices, J_t = diag(z) + diag(cz) U_z + diag(cn) U_n + diag(cr) U_r.
//
// One cooperative launch runs every iteration in three phases separated by
// grid barriers:
//   1. chunk aggregates: each tile (sequence b, chunk c of LC steps) forms
//      Phi_c = J_last ... J_first and the particular solution p_c (dh with a
//      zero carry-in) by sequential composition on chip;
//   2. carries: per sequence, dh_in(c+1) = Phi_c dh_in(c) + p_c over chunks;
//   3. re-sweep: each tile recomputes dh_t = J_t dh_{t-1} - r_t from its true
//      carry in fp32, writes h^(i+1) = h^(i) + dh and reduces max |dh|.
#include "common.cuh"
#include "solver.cuh"

namespace pararnn {

constexpr int kSC = 32;  // steps per sub-chunk of the coefficient pre-pass

struct DenseGeom {
    int DMAX;  // padded width (8, 16, 32 or 64)
    int LC;    // steps per chunk (multiple of kSC)
    int NC;    // chunks per sequence
    long long n_tiles;
};

DenseGeom dense_geom(int B, int T, int D) {
    DenseGeom g{};
    g.DMAX = D <= 8 ? 8 : (D <= 16 ? 16 : (D <= 32 ? 32 : 64));
    const long long bt = static_cast<long long>(B) * T;
    long long lc = (bt + 511) / 512;
    lc = ((lc + kSC - 1) / kSC) * kSC;
    if (lc < kSC) lc = kSC;
    if (lc > (1 << 20)) lc = 1 << 20;
    g.LC = static_cast<int>(lc);
    g.NC = static_cast<int>((T + lc - 1) / lc);
    g.n_tiles = static_cast<long long>(B) * g.NC;
    return g;
}

static size_t al256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

size_t dense_elk_ws_bytes(int B, int T, int D);
bool deer_mma_supported(const pararnn_cell &cell);
size_t deer_mma_ws_bytes(int B, int T);

// DEER: Phi [B][NC][D][D], p [B][NC][D], carry [B][NC][D]; ELK: the cyclic
// reduction arrays of newton_dense_elk.cu.
size_t dense_ws_bytes(const pararnn_cell &cell, int B, int T, int mode) {
    if (mode == PARARNN_ELK) return dense_elk_ws_bytes(B, T, cell.d);
    if (deer_mma_supported(cell)) return deer_mma_ws_bytes(B, T);
    const DenseGeom g = dense_geom(B, T, cell.d);
    const size_t n = static_cast<size_t>(B) * g.NC;
    const size_t D = cell.d;
    return al256(n * D * D * 4) + al256(n * D * 4) + al256(n * D * 4);
}

namespace {

template <int DMAX>
struct DenseSmem {
    float *Us;    // [k][g][i] = U_g[i][k]          3*DMAX*DMAX
    float *hs;    // guess rows ts-1 .. ts+SC-1      (kSC+1)*DMAX
    float *coef;  // z, cz, cn, cr per step and row  4*kSC*DMAX
    float *res;   // residual h_t - f_t              kSC*DMAX
    float *hcur;  // guess h_t                       kSC*DMAX
    float *Jt;    // J^T of the current step         DMAX*DMAX
    float *Phi;   // two buffers                     2*DMAX*DMAX
    float *vec;   // two buffers                     2*DMAX
    unsigned *red;
};

template <int DMAX>
constexpr size_t dense_smem_floats() {
    return 3 * DMAX * DMAX + (kSC + 1) * DMAX + 4 * kSC * DMAX + 2 * kSC * DMAX +
           3 * DMAX * DMAX + 2 * DMAX + 32;
}

template <int DMAX>
__device__ DenseSmem<DMAX> dense_carve(float *p) {
    DenseSmem<DMAX> s;
    s.Us = p; p += 3 * DMAX * DMAX;
    s.hs = p; p += (kSC + 1) * DMAX;
    s.coef = p; p += 4 * kSC * DMAX;
    s.res = p; p += kSC * DMAX;
    s.hcur = p; p += kSC * DMAX;
    s.Jt = p; p += DMAX * DMAX;
    s.Phi = p; p += 2 * DMAX * DMAX;
    s.vec = p; p += 2 * DMAX;
    s.red = reinterpret_cast<unsigned *>(p);
    return s;
}

struct DenseArgs {
    DiagArgs a;
    DenseGeom g;
    float *Phi, *pvec, *carry;
};

// Gate coefficients and residuals of steps ts .. ts+n-1 of sequence b at the
// guess `hold` (zero when zero_guess); rows >= D and steps >= n are zeroed so
// that they act as empty rows of J.
template <int DMAX>
__device__ void dense_coeffs(const DenseArgs &S, const DenseSmem<DMAX> &sm, int b, int ts, int n,
                             const float *hold, bool zero_guess, unsigned &rmax) {
    const DiagArgs &A = S.a;
    const int D = A.D, T = A.T;
    for (int q = threadIdx.x; q < (kSC + 1) * DMAX; q += kThreads) {
        const int r = q / DMAX, col = q % DMAX, t = ts - 1 + r;
        float v = 0.f;
        if (col < D && r <= n) {
            if (t < 0)
                v = __ldg(A.h0 + static_cast<size_t>(b) * D + col);
            else if (!zero_guess && t < T)
                v = __ldcg(hold + (static_cast<size_t>(b) * T + t) * D + col);
        }
        sm.hs[q] = v;
    }
    __syncthreads();
    constexpr int NG = kThreads / DMAX;  // step groups
    constexpr int SPT = kSC / NG;        // steps per thread
    const int i = threadIdx.x % DMAX, grp = threadIdx.x / DMAX;
    float acc[3][SPT];
#pragma unroll
    for (int g = 0; g < 3; ++g)
#pragma unroll
        for (int s = 0; s < SPT; ++s) acc[g][s] = 0.f;
    for (int k = 0; k < D; ++k) {
        const float u0 = sm.Us[(k * 3 + 0) * DMAX + i];
        const float u1 = sm.Us[(k * 3 + 1) * DMAX + i];
        const float u2 = sm.Us[(k * 3 + 2) * DMAX + i];
#pragma unroll
        for (int s = 0; s < SPT; ++s) {
            const float hv = sm.hs[(grp * SPT + s) * DMAX + k];
            acc[0][s] = fmaf(u0, hv, acc[0][s]);
            acc[1][s] = fmaf(u1, hv, acc[1][s]);
            acc[2][s] = fmaf(u2, hv, acc[2][s]);
        }
    }
#pragma unroll
    for (int s = 0; s < SPT; ++s) {
        const int tt = grp * SPT + s;
        float z = 0.f, cz = 0.f, cn = 0.f, cr = 0.f, res = 0.f, hc = 0.f;
        if (i < D && tt < n) {
            const int t = ts + tt;
            const float *prow = A.P + (static_cast<size_t>(b) * T + t) * 3 * D + i;
            const float hp = sm.hs[tt * DMAX + i];
            hc = sm.hs[(tt + 1) * DMAX + i];
            const float r = sigmoidf_(__ldg(prow) + acc[0][s] + __ldg(A.b_hh + i));
            z = sigmoidf_(__ldg(prow + D) + acc[1][s] + __ldg(A.b_hh + D + i));
            const float gn = acc[2][s] + __ldg(A.b_hh + 2 * D + i);
            const float nn = tanhf_(__ldg(prow + 2 * D) + r * gn);
            const float f = nn + z * (hp - nn);
            const float omz = 1.f - z;
            cz = (hp - nn) * z * omz;
            cn = omz * (1.f - nn * nn) * r;
            cr = cn * gn * (1.f - r);
            res = hc - f;
            rmax = max(rmax, abs_bits(res));
        }
        sm.coef[(0 * kSC + tt) * DMAX + i] = z;
        sm.coef[(1 * kSC + tt) * DMAX + i] = cz;
        sm.coef[(2 * kSC + tt) * DMAX + i] = cn;
        sm.coef[(3 * kSC + tt) * DMAX + i] = cr;
        sm.res[tt * DMAX + i] = res;
        sm.hcur[tt * DMAX + i] = hc;
    }
    __syncthreads();
}

// Block mapping of the D x D products: TG x TG threads, RB x RB entries each.
template <int DMAX>
struct Blk {
    static constexpr int RB = DMAX >= 32 ? DMAX / 16 : 1;
    static constexpr int TG = DMAX / RB;
};

// J_t^T of step tt into sm.Jt (rows/cols >= D are zero).
template <int DMAX>
__device__ __forceinline__ void build_jt(const DenseSmem<DMAX> &sm, int tt) {
    constexpr int RB = Blk<DMAX>::RB, TG = Blk<DMAX>::TG;
    if (threadIdx.x >= TG * TG) return;
    const int i0 = (threadIdx.x / TG) * RB, k0 = (threadIdx.x % TG) * RB;
#pragma unroll
    for (int a = 0; a < RB; ++a) {
        const int i = i0 + a;
        const float z = sm.coef[(0 * kSC + tt) * DMAX + i];
        const float cz = sm.coef[(1 * kSC + tt) * DMAX + i];
        const float cn = sm.coef[(2 * kSC + tt) * DMAX + i];
        const float cr = sm.coef[(3 * kSC + tt) * DMAX + i];
#pragma unroll
        for (int c = 0; c < RB; ++c) {
            const int k = k0 + c;
            const float ur = sm.Us[(k * 3 + 0) * DMAX + i];
            const float uz = sm.Us[(k * 3 + 1) * DMAX + i];
            const float un = sm.Us[(k * 3 + 2) * DMAX + i];
            float v = fmaf(cz, uz, fmaf(cn, un, cr * ur));
            if (i == k) v += z;
            sm.Jt[k * DMAX + i] = v;
        }
    }
}

// dst = J src (D x D, via Jt) for the thread's block; vector: vdst = J vsrc - res.
template <int DMAX>
__device__ __forceinline__ void jt_product(const DenseSmem<DMAX> &sm, const float *src, float *dst,
                                           bool matrix, const float *vsrc, float *vdst,
                                           const float *res) {
    constexpr int RB = Blk<DMAX>::RB, TG = Blk<DMAX>::TG;
    if (matrix && threadIdx.x < TG * TG) {
        const int i0 = (threadIdx.x / TG) * RB, j0 = (threadIdx.x % TG) * RB;
        float acc[RB][RB];
#pragma unroll
        for (int a = 0; a < RB; ++a)
#pragma unroll
            for (int c = 0; c < RB; ++c) acc[a][c] = 0.f;
#pragma unroll 4
        for (int k = 0; k < DMAX; ++k) {
            float jv[RB], pv[RB];
#pragma unroll
            for (int a = 0; a < RB; ++a) jv[a] = sm.Jt[k * DMAX + i0 + a];
#pragma unroll
            for (int c = 0; c < RB; ++c) pv[c] = src[k * DMAX + j0 + c];
#pragma unroll
            for (int a = 0; a < RB; ++a)
#pragma unroll
                for (int c = 0; c < RB; ++c) acc[a][c] = fmaf(jv[a], pv[c], acc[a][c]);
        }
#pragma unroll
        for (int a = 0; a < RB; ++a)
#pragma unroll
            for (int c = 0; c < RB; ++c) dst[(i0 + a) * DMAX + j0 + c] = acc[a][c];
    }
    if (threadIdx.x >= kThreads - DMAX) {
        const int i = threadIdx.x - (kThreads - DMAX);
        float s = 0.f;
#pragma unroll 8
        for (int k = 0; k < DMAX; ++k) s = fmaf(sm.Jt[k * DMAX + i], vsrc[k], s);
        vdst[i] = s - res[i];
    }
}

// Row-segment mapping for matrix-vector products: S lanes per row.
template <int DMAX>
struct Seg {
    static constexpr int S = DMAX <= 16 ? DMAX : (kThreads / DMAX);
    static constexpr int W = DMAX / S;
};

template <int DMAX>
__device__ __forceinline__ float seg_sum(float v) {
    constexpr int S = Seg<DMAX>::S;
#pragma unroll
    for (int o = S / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o, S);
    return v;
}

// Phase 1: aggregate of tile (b, c).
template <int DMAX>
__device__ void phase_aggregate(const DenseArgs &S, const DenseSmem<DMAX> &sm, long long tile,
                                const float *hold, bool zero_guess, unsigned &rmax) {
    const DiagArgs &A = S.a;
    const int D = A.D;
    const int b = static_cast<int>(tile % A.B), c = static_cast<int>(tile / A.B);
    const int t_begin = c * S.g.LC;
    const int t_end = min(A.T, t_begin + S.g.LC);
    // the first chunk's carry-in is zero and the last chunk feeds no carry:
    // their Phi is never used
    const bool need_phi = c > 0 && c < S.g.NC - 1;
    for (int q = threadIdx.x; q < DMAX * DMAX; q += kThreads)
        sm.Phi[q] = (q / DMAX == q % DMAX) ? 1.f : 0.f;
    if (threadIdx.x < DMAX) sm.vec[threadIdx.x] = 0.f;
    __syncthreads();
    int cur = 0;
    for (int ts = t_begin; ts < t_end; ts += kSC) {
        const int n = min(kSC, t_end - ts);
        dense_coeffs<DMAX>(S, sm, b, ts, n, hold, zero_guess, rmax);
        for (int tt = 0; tt < n; ++tt) {
            build_jt<DMAX>(sm, tt);
            __syncthreads();
            jt_product<DMAX>(sm, sm.Phi + cur * DMAX * DMAX, sm.Phi + (cur ^ 1) * DMAX * DMAX,
                             need_phi, sm.vec + cur * DMAX, sm.vec + (cur ^ 1) * DMAX,
                             sm.res + tt * DMAX);
            __syncthreads();
            cur ^= 1;
        }
    }
    const size_t slot = static_cast<size_t>(b) * S.g.NC + c;
    if (need_phi)
        for (int q = threadIdx.x; q < D * D; q += kThreads)
            __stcg(S.Phi + slot * D * D + q, sm.Phi[cur * DMAX * DMAX + (q / D) * DMAX + q % D]);
    if (threadIdx.x < D) __stcg(S.pvec + slot * D + threadIdx.x, sm.vec[cur * DMAX + threadIdx.x]);
    __syncthreads();
}

// Phase 2: carries of sequence b.
template <int DMAX>
__device__ void phase_carry(const DenseArgs &S, const DenseSmem<DMAX> &sm, int b) {
    constexpr int SS = Seg<DMAX>::S, W = Seg<DMAX>::W;
    const int D = S.a.D, NC = S.g.NC;
    const bool act = threadIdx.x < DMAX * SS;
    const int i = threadIdx.x / SS, seg = threadIdx.x % SS;
    if (threadIdx.x < DMAX) sm.vec[threadIdx.x] = 0.f;
    __syncthreads();
    int cur = 0;
    for (int c = 0; c < NC; ++c) {
        const size_t slot = static_cast<size_t>(b) * NC + c;
        if (threadIdx.x < D) __stcg(S.carry + slot * D + threadIdx.x, sm.vec[cur * DMAX + threadIdx.x]);
        if (c == NC - 1) break;
        float part = 0.f;
        if (act && i < D) {
            if (c == 0) {
                part = 0.f;  // zero carry-in: Phi_0 is not formed
            } else {
#pragma unroll
                for (int w = 0; w < W; ++w) {
                    const int k = seg * W + w;
                    if (k < D)
                        part = fmaf(__ldcg(S.Phi + slot * D * D + static_cast<size_t>(i) * D + k),
                                    sm.vec[cur * DMAX + k], part);
                }
            }
        }
        if (act) part = seg_sum<DMAX>(part);
        if (act && seg == 0 && i < DMAX)
            sm.vec[(cur ^ 1) * DMAX + i] = i < D ? part + __ldcg(S.pvec + slot * D + i) : 0.f;
        __syncthreads();
        cur ^= 1;
    }
    __syncthreads();
}

// Phase 3: re-sweep tile (b, c) from its carry; writes h^(i+1) and max |dh|.
template <int DMAX>
__device__ void phase_sweep(const DenseArgs &S, const DenseSmem<DMAX> &sm, long long tile,
                            const float *hold, float *hnew, bool zero_guess, unsigned &dmax,
                            const float (&ureg)[3][Seg<DMAX>::W]) {
    constexpr int SS = Seg<DMAX>::S, W = Seg<DMAX>::W;
    const DiagArgs &A = S.a;
    const int D = A.D, T = A.T;
    const int b = static_cast<int>(tile % A.B), c = static_cast<int>(tile / A.B);
    const int t_begin = c * S.g.LC;
    const int t_end = min(T, t_begin + S.g.LC);
    const bool act = threadIdx.x < DMAX * SS;
    const int i = threadIdx.x / SS, seg = threadIdx.x % SS;
    const size_t slot = static_cast<size_t>(b) * S.g.NC + c;
    if (threadIdx.x < DMAX) sm.vec[threadIdx.x] = threadIdx.x < D ? __ldcg(S.carry + slot * D + threadIdx.x) : 0.f;
    __syncthreads();
    unsigned rdummy = 0u;
    int cur = 0;
    for (int ts = t_begin; ts < t_end; ts += kSC) {
        const int n = min(kSC, t_end - ts);
        dense_coeffs<DMAX>(S, sm, b, ts, n, hold, zero_guess, rdummy);
        for (int tt = 0; tt < n; ++tt) {
            float pr = 0.f, pz = 0.f, pn = 0.f;
            if (act) {
#pragma unroll
                for (int w = 0; w < W; ++w) {
                    const float dv = sm.vec[cur * DMAX + seg * W + w];
                    pr = fmaf(ureg[0][w], dv, pr);
                    pz = fmaf(ureg[1][w], dv, pz);
                    pn = fmaf(ureg[2][w], dv, pn);
                }
                pr = seg_sum<DMAX>(pr);
                pz = seg_sum<DMAX>(pz);
                pn = seg_sum<DMAX>(pn);
            }
            if (act && seg == 0) {
                float dn = 0.f;
                if (i < D) {
                    const float z = sm.coef[(0 * kSC + tt) * DMAX + i];
                    const float cz = sm.coef[(1 * kSC + tt) * DMAX + i];
                    const float cn = sm.coef[(2 * kSC + tt) * DMAX + i];
                    const float cr = sm.coef[(3 * kSC + tt) * DMAX + i];
                    dn = z * sm.vec[cur * DMAX + i] + cz * pz + cn * pn + cr * pr -
                         sm.res[tt * DMAX + i];
                    const int t = ts + tt;
                    __stcg(hnew + (static_cast<size_t>(b) * T + t) * D + i, sm.hcur[tt * DMAX + i] + dn);
                    dmax = max(dmax, abs_bits(dn));
                }
                sm.vec[(cur ^ 1) * DMAX + i] = dn;
            }
            __syncthreads();
            cur ^= 1;
        }
    }
}

template <int DMAX>
__global__ void __launch_bounds__(kThreads, 1) dense_deer_kernel(DenseArgs S) {
    extern __shared__ float4 smem_raw[];
    const DenseSmem<DMAX> sm = dense_carve<DMAX>(reinterpret_cast<float *>(smem_raw));
    const DiagArgs &A = S.a;
    WsHeader *hdr = A.hdr;
    unsigned *status = &hdr->status;
    const unsigned nblocks = gridDim.x;
    const int D = A.D;
    for (int q = threadIdx.x; q < 3 * DMAX * DMAX; q += kThreads) {
        const int i = q % DMAX, g = (q / DMAX) % 3, k = q / (3 * DMAX);
        sm.Us[q] = (i < D && k < D) ? __ldg(A.w_hh + (static_cast<size_t>(g) * D + i) * D + k) : 0.f;
    }
    constexpr int SS = Seg<DMAX>::S, W = Seg<DMAX>::W;
    float ureg[3][W];
    {
        const int i = threadIdx.x / SS, seg = threadIdx.x % SS;
#pragma unroll
        for (int g = 0; g < 3; ++g)
#pragma unroll
            for (int w = 0; w < W; ++w) {
                const int k = seg * W + w;
                ureg[g][w] = (threadIdx.x < DMAX * SS && i < D && k < D)
                                 ? __ldg(A.w_hh + (static_cast<size_t>(g) * D + i) * D + k) : 0.f;
            }
    }
    __syncthreads();

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
        for (long long tile = blockIdx.x; tile < S.g.n_tiles; tile += nblocks)
            phase_aggregate<DMAX>(S, sm, tile, hold, zero_guess, rmax);
        grid_barrier(hdr->barrier, nblocks, status);
        for (int b = blockIdx.x; b < A.B; b += nblocks) phase_carry<DMAX>(S, sm, b);
        grid_barrier(hdr->barrier, nblocks, status);
        for (long long tile = blockIdx.x; tile < S.g.n_tiles; tile += nblocks)
            phase_sweep<DMAX>(S, sm, tile, hold, hnew, zero_guess, dmax, ureg);
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
        const size_t n4 = static_cast<size_t>(A.B) * A.T * A.D / 4;
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
cudaError_t launch_deer(const DenseArgs &S, cudaStream_t s) {
    auto kern = dense_deer_kernel<DMAX>;
    const size_t smem = dense_smem_floats<DMAX>() * sizeof(float);
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
    const long long need = S.g.n_tiles > S.a.B ? S.g.n_tiles : S.a.B;
    if (grid > need) grid = need;
    DenseArgs args = S;
    void *params[] = {&args};
    return cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(kern),
                                       dim3(static_cast<unsigned>(grid)), dim3(kThreads), params,
                                       smem, s);
}

// ---------------------------------------------------------------------------
// standalone dense scan: three launches (aggregate, carry, re-sweep)
// ---------------------------------------------------------------------------
struct DScanArgs {
    const float *A, *b, *h0;
    float *h;
    int B, T, D;
    DenseGeom g;
    float *Phi, *pvec, *carry;
};

template <int DMAX>
struct ScanSmem {
    float *Jt, *Phi, *vec;
};

// A_t^T of sequence b, step t into Jt (zero padded).
template <int DMAX>
__device__ __forceinline__ void load_at(const DScanArgs &S, float *Jt, int b, int t) {
    const int D = S.D;
    const float *At = S.A + (static_cast<size_t>(b) * S.T + t) * D * D;
    for (int q = threadIdx.x; q < DMAX * DMAX; q += kThreads) {
        const int i = q / DMAX, k = q % DMAX;  // coalesced along k
        Jt[k * DMAX + i] = (i < D && k < D) ? __ldcs(At + i * D + k) : 0.f;
    }
}

template <int DMAX>
constexpr size_t dscan_smem_floats() { return 3 * DMAX * DMAX + 3 * DMAX; }

template <int DMAX>
__global__ void __launch_bounds__(kThreads) dscan_aggregate(DScanArgs S) {
    extern __shared__ float4 dsmem_raw[];
    float *Jt = reinterpret_cast<float *>(dsmem_raw);
    float *Phi = Jt + DMAX * DMAX;
    float *vec = Phi + 2 * DMAX * DMAX;
    float *zero = vec + 2 * DMAX;
    DenseSmem<DMAX> sm{};
    sm.Jt = Jt;
    const long long tile = blockIdx.x;
    const int b = static_cast<int>(tile % S.B), c = static_cast<int>(tile / S.B);
    const int t_begin = c * S.g.LC, t_end = min(S.T, t_begin + S.g.LC);
    const bool need_phi = c < S.g.NC - 1;  // chunk 0 needs Phi too: its carry-in is h0
    for (int q = threadIdx.x; q < DMAX * DMAX; q += kThreads) Phi[q] = (q / DMAX == q % DMAX) ? 1.f : 0.f;
    if (threadIdx.x < DMAX) { vec[threadIdx.x] = 0.f; zero[threadIdx.x] = 0.f; }
    __syncthreads();
    int cur = 0;
    for (int t = t_begin; t < t_end; ++t) {
        load_at<DMAX>(S, Jt, b, t);
        __syncthreads();
        // res = -b_t so that vdst = A p + b
        if (threadIdx.x < DMAX)
            zero[threadIdx.x] = threadIdx.x < S.D ? -__ldcs(S.b + (static_cast<size_t>(b) * S.T + t) * S.D + threadIdx.x) : 0.f;
        __syncthreads();
        jt_product<DMAX>(sm, Phi + cur * DMAX * DMAX, Phi + (cur ^ 1) * DMAX * DMAX, need_phi,
                         vec + cur * DMAX, vec + (cur ^ 1) * DMAX, zero);
        __syncthreads();
        cur ^= 1;
    }
    const size_t slot = static_cast<size_t>(b) * S.g.NC + c;
    const int D = S.D;
    if (need_phi)
        for (int q = threadIdx.x; q < D * D; q += kThreads)
            S.Phi[slot * D * D + q] = Phi[cur * DMAX * DMAX + (q / D) * DMAX + q % D];
    if (threadIdx.x < D) S.pvec[slot * D + threadIdx.x] = vec[cur * DMAX + threadIdx.x];
}

template <int DMAX>
__global__ void __launch_bounds__(kThreads) dscan_carry(DScanArgs S) {
    constexpr int SS = Seg<DMAX>::S, W = Seg<DMAX>::W;
    __shared__ float vec[2 * DMAX];
    const int b = blockIdx.x, D = S.D, NC = S.g.NC;
    const bool act = threadIdx.x < DMAX * SS;
    const int i = threadIdx.x / SS, seg = threadIdx.x % SS;
    if (threadIdx.x < DMAX) vec[threadIdx.x] = threadIdx.x < D ? S.h0[static_cast<size_t>(b) * D + threadIdx.x] : 0.f;
    __syncthreads();
    int cur = 0;
    for (int c = 0; c < NC; ++c) {
        const size_t slot = static_cast<size_t>(b) * NC + c;
        if (threadIdx.x < D) S.carry[slot * D + threadIdx.x] = vec[cur * DMAX + threadIdx.x];
        if (c == NC - 1) break;
        float part = 0.f;
        if (act && i < D)
#pragma unroll
            for (int w = 0; w < W; ++w) {
                const int k = seg * W + w;
                if (k < D) part = fmaf(S.Phi[slot * D * D + static_cast<size_t>(i) * D + k], vec[cur * DMAX + k], part);
            }
        if (act) part = seg_sum<DMAX>(part);
        if (act && seg == 0 && i < DMAX) vec[(cur ^ 1) * DMAX + i] = i < D ? part + S.pvec[slot * D + i] : 0.f;
        __syncthreads();
        cur ^= 1;
    }
}

template <int DMAX>
__global__ void __launch_bounds__(kThreads) dscan_sweep(DScanArgs S) {
    constexpr int SS = Seg<DMAX>::S, W = Seg<DMAX>::W;
    __shared__ float vec[2 * DMAX];
    const long long tile = blockIdx.x;
    const int b = static_cast<int>(tile % S.B), c = static_cast<int>(tile / S.B);
    const int t_begin = c * S.g.LC, t_end = min(S.T, t_begin + S.g.LC);
    const int D = S.D;
    const bool act = threadIdx.x < DMAX * SS;
    const int i = threadIdx.x / SS, seg = threadIdx.x % SS;
    const size_t slot = static_cast<size_t>(b) * S.g.NC + c;
    if (threadIdx.x < DMAX) vec[threadIdx.x] = threadIdx.x < D ? S.carry[slot * D + threadIdx.x] : 0.f;
    __syncthreads();
    int cur = 0;
    for (int t = t_begin; t < t_end; ++t) {
        const size_t row = static_cast<size_t>(b) * S.T + t;
        float part = 0.f;
        if (act && i < D)
#pragma unroll
            for (int w = 0; w < W; ++w) {
                const int k = seg * W + w;
                if (k < D) part = fmaf(__ldcs(S.A + row * D * D + static_cast<size_t>(i) * D + k), vec[cur * DMAX + k], part);
            }
        if (act) part = seg_sum<DMAX>(part);
        if (act && seg == 0 && i < DMAX) {
            float hv = 0.f;
            if (i < D) {
                hv = part + __ldcs(S.b + row * D + i);
                S.h[row * D + i] = hv;
            }
            vec[(cur ^ 1) * DMAX + i] = hv;
        }
        __syncthreads();
        cur ^= 1;
    }
}

template <int DMAX>
cudaError_t launch_dscan(const DScanArgs &S, cudaStream_t s) {
    const unsigned tiles = static_cast<unsigned>(S.g.n_tiles);
    const size_t smem = dscan_smem_floats<DMAX>() * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(dscan_aggregate<DMAX>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    dscan_aggregate<DMAX><<<tiles, kThreads, smem, s>>>(S);
    dscan_carry<DMAX><<<S.B, kThreads, 0, s>>>(S);
    dscan_sweep<DMAX><<<tiles, kThreads, 0, s>>>(S);
    return cudaGetLastError();
}

}  // namespace

size_t dense_elk_ws_bytes(int B, int T, int D);
cudaError_t launch_dense_elk(const DiagArgs &a, void *ws, cudaStream_t s);
bool deer_mma_supported(const pararnn_cell &cell);
cudaError_t launch_deer_mma(const DiagArgs &a, void *ws, cudaStream_t s);

cudaError_t launch_dense_solver(const pararnn_cell &cell, int mode, const DiagArgs &a,
                                void *dense_ws, cudaStream_t s) {
    if (mode == PARARNN_ELK) return launch_dense_elk(a, dense_ws, s);
    if (mode == PARARNN_DEER && deer_mma_supported(cell)) return launch_deer_mma(a, dense_ws, s);
    if (mode != PARARNN_DEER) return cudaErrorNotSupported;
    DenseArgs S;
    S.a = a;
    S.g = dense_geom(a.B, a.T, a.D);
    const size_t n = static_cast<size_t>(a.B) * S.g.NC;
    char *p = static_cast<char *>(dense_ws);
    S.Phi = reinterpret_cast<float *>(p);
    p += al256(n * a.D * a.D * 4);
    S.pvec = reinterpret_cast<float *>(p);
    p += al256(n * a.D * 4);
    S.carry = reinterpret_cast<float *>(p);
    switch (S.g.DMAX) {
        case 8: return launch_deer<8>(S, s);
        case 16: return launch_deer<16>(S, s);
        case 32: return launch_deer<32>(S, s);
        default: return launch_deer<64>(S, s);
    }
}

size_t scan_dense_ws_bytes(int B, int T, int D) {
    const DenseGeom g = dense_geom(B, T, D);
    const size_t n = static_cast<size_t>(B) * g.NC;
    return 256 + al256(n * D * D * 4) + al256(n * D * 4) + al256(n * D * 4);
}

cudaError_t launch_scan_dense(const float *A, const float *b, const float *h0, int B, int T,
                              int D, float *h, void *ws, cudaStream_t s) {
    DScanArgs S;
    S.A = A; S.b = b; S.h0 = h0; S.h = h;
    S.B = B; S.T = T; S.D = D;
    S.g = dense_geom(B, T, D);
    const size_t n = static_cast<size_t>(B) * S.g.NC;
    char *p = static_cast<char *>(ws) + 256;
    cudaError_t e = cudaMemsetAsync(ws, 0, 256, s);  // status word: no bounded waits here
    if (e != cudaSuccess) return e;
    S.Phi = reinterpret_cast<float *>(p);
    p += al256(n * D * D * 4);
    S.pvec = reinterpret_cast<float *>(p);
    p += al256(n * D * 4);
    S.carry = reinterpret_cast<float *>(p);
    switch (S.g.DMAX) {
        case 8: return launch_dscan<8>(S, s);
        case 16: return launch_dscan<16>(S, s);
        case 32: return launch_dscan<32>(S, s);
        default: return launch_dscan<64>(S, s);
    }
}

}  // namespace pararnn

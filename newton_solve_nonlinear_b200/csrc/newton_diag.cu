// newton_diag.cu -- persistent solver for the diagonal-Jacobian family:
//   quasi-DEER on the dense GRU, exact Newton (DEER == quasi-DEER) on the
//   diagonal-recurrence GRU, and quasi-ELK on either cell.
//
// Method: "Towards Scalable and Stable Parallelization of Nonlinear RNNs"
// (abstract; atlas summary "Approach": diagonal Jacobian, O(TD) work and
// memory per iteration; LM damping solved as a parallel Kalman filter and
// smoother) on the unrolled system of the ParaRNN summary ("Core Idea",
// "Newton's Iteration").
//
// One cooperative launch runs the whole Newton loop.  Per iteration every CTA
// walks its share of tiles; a tile is (sequence b, a group of DG state lanes,
// a chunk of L time steps).  Inside a tile each thread owns TK consecutive
// steps of 4 adjacent lanes (float4 accesses along D, coalesced across the
// warp), so:
//   1. the cell is evaluated at the shifted guess for all of the tile's states
//      at once (the guess is known, so this part has no sequential dependence);
//      for the dense cell the recurrent product U h_{t-1} is computed from a
//      shared-memory copy of the tile's guess rows and of U, in fp32 FMAs so
//      the fixed point is the fp32 rollout's;
//   2. each thread composes its TK affine maps (a_t, b_t) per lane in
//      registers, a shared-memory pass turns these into exclusive prefixes
//      across the tile's thread rows, and one thread per lane resolves the
//      tile's carry-in with a decoupled look-back over earlier chunks of the
//      same lanes (single pass over HBM);
//   3. the states are re-swept from the carry, written once, and the max of
//      |h^(i+1) - h^(i)| (and of the residual) is reduced to one atomicMax per
//      CTA.
// A bounded grid barrier closes the iteration; every CTA reads the same
// reduced delta and stops together.  quasi-ELK runs a forward pass (scalar
// Kalman covariance as a 2x2 Mobius scan, then the filtered mean as an affine
// scan) and a backward pass (RTS smoother as a reverse affine scan), each
// single-pass with look-back, separated by a grid barrier.
#include <cstdio>

#include "common.cuh"
#include "lookback.cuh"
#include "solver.cuh"

namespace pararnn {

Tiling make_tiling(int B, int T, int D, bool dense_cell, int TK) {
    Tiling t{};
    t.DG = dense_cell ? D : (D < 64 ? D : 64);
    t.DB = t.DG / 4;
    t.NTB = kThreads / t.DB;
    t.TK = TK;
    t.L = t.NTB * t.TK;
    t.n_dgroups = (D + t.DG - 1) / t.DG;
    t.n_groups = B * t.n_dgroups;
    t.n_chunks = (T + t.L - 1) / t.L;
    t.n_tiles = static_cast<long long>(t.n_groups) * t.n_chunks;
    return t;
}

namespace {

struct TileCoord {
    long long tile;
    int chunk, b, dg, db, tb, lane0, d0, t0, tile_t0;
    bool active, dvalid;
};

template <int TK>
__device__ __forceinline__ TileCoord tile_coord(const DiagArgs &A, long long tile) {
    TileCoord c;
    const Tiling &tl = A.tl;
    c.tile = tile;
    c.chunk = static_cast<int>(tile / tl.n_groups);
    const int grp = static_cast<int>(tile % tl.n_groups);
    c.b = grp / tl.n_dgroups;
    c.dg = grp % tl.n_dgroups;
    c.db = threadIdx.x % tl.DB;
    c.tb = threadIdx.x / tl.DB;
    c.active = c.tb < tl.NTB;
    c.lane0 = c.db * 4;
    c.d0 = c.dg * tl.DG + c.lane0;
    c.dvalid = c.active && c.d0 < A.D;
    c.tile_t0 = c.chunk * tl.L;
    c.t0 = c.tile_t0 + c.tb * TK;
    return c;
}

// Shared memory carve-up (floats).
struct Smem {
    float *Us;    // dense: [D][3][DG]
    float *hs;    // dense: [L+1][D]   guess rows tile_t0-1 .. tile_t0+L-1
    float *aby;   // dense-mma: a, bb, y of the tile [3][L][D+4]
    float *s0, *s1, *s2, *s3;  // [NTB][DG] scan scratch
    float *c0, *c1;            // [DG] carries
    unsigned *red;             // [32]
};

// Cell variants of the solver kernels.
constexpr int kCellDiag = 0;      // diagonal recurrence: u_g * h, no product
constexpr int kCellDenseFma = 1;  // dense U h in fp32 FMAs (any D multiple of 4)
constexpr int kCellDenseMma = 2;  // dense U h on tensor cores, 3 x TF32 (D in 8,16,32,64)

__host__ __device__ inline int mma_stride(int D) { return D + 4; }  // padded rows: no bank conflicts

__host__ __device__ inline size_t smem_floats(const Tiling &tl, int D, int cell) {
    size_t n = 0;
    if (cell == kCellDenseFma)
        n += static_cast<size_t>(D) * 3 * tl.DG + static_cast<size_t>(tl.L + 1) * D;
    if (cell == kCellDenseMma) {
        const size_t S = mma_stride(D);
        n += static_cast<size_t>(tl.L + 1) * S + 3 * static_cast<size_t>(tl.L) * S;
    }
    n += 4 * static_cast<size_t>(tl.NTB) * tl.DG + 2 * tl.DG + 32;
    return n;
}

__device__ __forceinline__ Smem carve(float *base, const Tiling &tl, int D, int cell) {
    Smem s;
    float *p = base;
    s.Us = p;
    s.hs = p;
    s.aby = p;
    if (cell == kCellDenseFma) {
        s.Us = p;
        p += static_cast<size_t>(D) * 3 * tl.DG;
        s.hs = p;
        p += static_cast<size_t>(tl.L + 1) * D;
    } else if (cell == kCellDenseMma) {
        const size_t S = mma_stride(D);
        s.hs = p;
        p += static_cast<size_t>(tl.L + 1) * S;
        s.aby = p;
        p += 3 * static_cast<size_t>(tl.L) * S;
    }
    const size_t n = static_cast<size_t>(tl.NTB) * tl.DG;
    s.s0 = p; p += n;
    s.s1 = p; p += n;
    s.s2 = p; p += n;
    s.s3 = p; p += n;
    s.c0 = p; p += tl.DG;
    s.c1 = p; p += tl.DG;
    s.red = reinterpret_cast<unsigned *>(p);
    return s;
}

// One state of the cell and its Jacobian diagonal.  pr, pz, pn: input
// pre-activations (b_ih included); gr, gz, gnh: recurrent sums U_g h (or
// u_g * h); bh: b_hh; ud: diagonal entries of U_g; h: guess at t-1; hc: guess
// at t.  Returns a = dJ_tt and bb = f - a h, and folds |hc - f| into rmax.
__device__ __forceinline__ void cell_state(float pr, float pz, float pn, float gr, float gz,
                                           float gnh, float bhr, float bhz, float bhn, float udr,
                                           float udz, float udn, float h, float hc, float &a,
                                           float &bb, unsigned &rmax) {
    float f;
    gru_cell_diag(pr, pz, pn, gr, gz, gnh, bhr, bhz, bhn, udr, udz, udn, h, f, a, bb);
    rmax = max(rmax, abs_bits(hc - f));
}

__device__ __forceinline__ void mma_tf32(float (&c)[4], const unsigned (&a)[4], unsigned b0,
                                         unsigned b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// x = hi + lo with hi exactly representable in TF32 (top 10 mantissa bits) and
// lo the exact fp32 remainder; hi*hi + hi*lo + lo*hi then carries a product to
// ~2^-21 relative accuracy (the error-compensated 3 x TF32 split).
__device__ __forceinline__ void split_tf32(float x, unsigned &hi, unsigned &lo) {
    hi = __float_as_uint(x) & 0xffffe000u;
    lo = __float_as_uint(x - __uint_as_float(hi));
}

// Dense cell with U h on the tensor cores.  Warp w owns lane block
// lb = w % (D/8) (8 state lanes) and two 16-step row blocks of the tile; its
// mma.sync m16n8k8 fragments hold, per thread, the three gates of the same
// (step, lane) pairs, so the cell is evaluated straight from the accumulators.
// a, bb, y go through shared memory to the (thread row, float4 column) layout
// of the scan.
template <int TK>
__device__ __forceinline__ void linearise_mma(const DiagArgs &A, const TileCoord &c, const Smem &sm,
                                              const float *hold, bool zero_guess, float (&a)[TK][4],
                                              float (&bb)[TK][4], float (&y)[TK][4],
                                              unsigned &rmax) {
    const int D = A.D, T = A.T, L = A.tl.L;
    const int S = mma_stride(D);
    const int nq = D / 4, nvec = (L + 1) * nq;
    for (int i = threadIdx.x; i < nvec; i += kThreads) {
        const int r = i / nq, col = (i % nq) * 4;
        const int t = c.tile_t0 - 1 + r;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (t < 0)
            v = __ldg(reinterpret_cast<const float4 *>(A.h0 + static_cast<size_t>(c.b) * D + col));
        else if (!zero_guess && t < T)
            v = ldcg4(hold + (static_cast<size_t>(c.b) * T + t) * D + col);
        *reinterpret_cast<float4 *>(sm.hs + static_cast<size_t>(r) * S + col) = v;
    }
    __syncthreads();
    {
        const int lid = threadIdx.x & 31, w = threadIdx.x >> 5;
        const int gid = lid >> 2, tq = lid & 3;
        const int LB = D / 8;
        const int lb = w % LB;
        const int row0 = (w / LB) * 32;  // first tile step of the warp's two row blocks
        float acc[2][3][4];
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int g = 0; g < 3; ++g)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[m][g][e] = 0.f;
        // U_g rows of this warp's 8 lanes, read through L1 (48 KB, shared by all CTAs)
        const float *urow[3];
#pragma unroll
        for (int g = 0; g < 3; ++g) urow[g] = A.w_hh + static_cast<size_t>(g * D + lb * 8 + gid) * D;
        // input pre-activations of this thread's (step, lane-pair) slots, issued
        // before the products so that their latency overlaps the MMAs
        const int l0 = lb * 8 + 2 * tq;  // lanes l0, l0 + 1
        float2 pv[2][2][3];
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int t = c.tile_t0 + row0 + m * 16 + gid + hh * 8;
                const float *prow = A.P + (static_cast<size_t>(c.b) * T + (t < T ? t : T - 1)) * 3 * D + l0;
#pragma unroll
                for (int g = 0; g < 3; ++g) pv[m][hh][g] = __ldg(reinterpret_cast<const float2 *>(prow + g * D));
            }
        for (int k0 = 0; k0 < D; k0 += 8) {
            unsigned bh[3][2], bl[3][2];
#pragma unroll
            for (int g = 0; g < 3; ++g) {
                split_tf32(__ldg(urow[g] + k0 + tq), bh[g][0], bl[g][0]);
                split_tf32(__ldg(urow[g] + k0 + tq + 4), bh[g][1], bl[g][1]);
            }
            unsigned ah[2][4], al[2][4];
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                const float *r0 = sm.hs + static_cast<size_t>(row0 + m * 16 + gid) * S + k0 + tq;
                const float *r1 = r0 + 8 * S;
                split_tf32(r0[0], ah[m][0], al[m][0]);
                split_tf32(r1[0], ah[m][1], al[m][1]);
                split_tf32(r0[4], ah[m][2], al[m][2]);
                split_tf32(r1[4], ah[m][3], al[m][3]);
            }
            // small terms first; six independent accumulators between dependent MMAs
#pragma unroll
            for (int m = 0; m < 2; ++m)
#pragma unroll
                for (int g = 0; g < 3; ++g) mma_tf32(acc[m][g], al[m], bh[g][0], bh[g][1]);
#pragma unroll
            for (int m = 0; m < 2; ++m)
#pragma unroll
                for (int g = 0; g < 3; ++g) mma_tf32(acc[m][g], ah[m], bl[g][0], bl[g][1]);
#pragma unroll
            for (int m = 0; m < 2; ++m)
#pragma unroll
                for (int g = 0; g < 3; ++g) mma_tf32(acc[m][g], ah[m], bh[g][0], bh[g][1]);
        }
        // the cell for this thread's (step, lane) pairs
        float bh2[3][2], ud2[3][2];
#pragma unroll
        for (int g = 0; g < 3; ++g) {
            const float2 v = __ldg(reinterpret_cast<const float2 *>(A.b_hh + g * D + l0));
            bh2[g][0] = v.x;
            bh2[g][1] = v.y;
            ud2[g][0] = __ldg(A.w_hh + static_cast<size_t>(g * D + l0) * D + l0);
            ud2[g][1] = __ldg(A.w_hh + static_cast<size_t>(g * D + l0 + 1) * D + l0 + 1);
        }
        float *sa = sm.aby, *sb = sm.aby + static_cast<size_t>(L) * S, *sy = sb + static_cast<size_t>(L) * S;
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int tl_ = row0 + m * 16 + gid + hh * 8;  // tile-local step
                const int t = c.tile_t0 + tl_;
                float2 av = make_float2(1.f, 1.f), bv = make_float2(0.f, 0.f), yv = make_float2(0.f, 0.f);
                if (t < T) {
                    const float2 pr = pv[m][hh][0], pz = pv[m][hh][1], pn = pv[m][hh][2];
                    const float2 hp = *reinterpret_cast<const float2 *>(sm.hs + static_cast<size_t>(tl_) * S + l0);
                    yv = *reinterpret_cast<const float2 *>(sm.hs + static_cast<size_t>(tl_ + 1) * S + l0);
                    cell_state(pr.x, pz.x, pn.x, acc[m][0][hh * 2], acc[m][1][hh * 2],
                               acc[m][2][hh * 2], bh2[0][0], bh2[1][0], bh2[2][0], ud2[0][0],
                               ud2[1][0], ud2[2][0], hp.x, yv.x, av.x, bv.x, rmax);
                    cell_state(pr.y, pz.y, pn.y, acc[m][0][hh * 2 + 1], acc[m][1][hh * 2 + 1],
                               acc[m][2][hh * 2 + 1], bh2[0][1], bh2[1][1], bh2[2][1], ud2[0][1],
                               ud2[1][1], ud2[2][1], hp.y, yv.y, av.y, bv.y, rmax);
                }
                const size_t off = static_cast<size_t>(tl_) * S + l0;
                *reinterpret_cast<float2 *>(sa + off) = av;
                *reinterpret_cast<float2 *>(sb + off) = bv;
                *reinterpret_cast<float2 *>(sy + off) = yv;
            }
    }
    __syncthreads();
    if (c.active) {
        const float *sa = sm.aby, *sb = sm.aby + static_cast<size_t>(L) * S, *sy = sb + static_cast<size_t>(L) * S;
#pragma unroll
        for (int k = 0; k < TK; ++k) {
            const size_t off = static_cast<size_t>(c.tb * TK + k) * S + c.d0;
            const float4 av = *reinterpret_cast<const float4 *>(sa + off);
            const float4 bv = *reinterpret_cast<const float4 *>(sb + off);
            const float4 yv = *reinterpret_cast<const float4 *>(sy + off);
            a[k][0] = av.x; a[k][1] = av.y; a[k][2] = av.z; a[k][3] = av.w;
            bb[k][0] = bv.x; bb[k][1] = bv.y; bb[k][2] = bv.z; bb[k][3] = bv.w;
            y[k][0] = yv.x; y[k][1] = yv.y; y[k][2] = yv.z; y[k][3] = yv.w;
        }
    }
}

// ---------------------------------------------------------------------------
// 1. linearisation at the shifted guess
// ---------------------------------------------------------------------------
// Produces, for the thread's TK x 4 states: a (diag of the Jacobian), bb
// (f - a h_{t-1}) and y (the guess at t).  Steps past T or lanes past D get
// the identity map (a = 1, bb = 0).
template <int CELL, int TK>
__device__ __forceinline__ void linearise(const DiagArgs &A, const TileCoord &c, const Smem &sm,
                                          const float *hold, bool zero_guess, float (&a)[TK][4],
                                          float (&bb)[TK][4], float (&y)[TK][4], unsigned &rmax) {
    if (CELL == kCellDenseMma) {
        linearise_mma<TK>(A, c, sm, hold, zero_guess, a, bb, y, rmax);
        return;
    }
    constexpr bool DENSE = CELL == kCellDenseFma;
    const int D = A.D, T = A.T;
    const size_t rowP = 3 * static_cast<size_t>(D);
    float hp[TK + 1][4];
    float G[3][TK][4];
    if (DENSE) {
        // guess rows tile_t0-1 .. tile_t0+L-1 into shared memory (row 0 may be h0)
        const int L = A.tl.L, nq = D / 4, nvec = (L + 1) * nq;
        for (int i = threadIdx.x; i < nvec; i += kThreads) {
            const int r = i / nq, col = (i % nq) * 4;
            const int t = c.tile_t0 - 1 + r;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (t < 0)
                v = __ldg(reinterpret_cast<const float4 *>(A.h0 + static_cast<size_t>(c.b) * D + col));
            else if (!zero_guess && t < T)
                v = ldcg4(hold + (static_cast<size_t>(c.b) * T + t) * D + col);
            *reinterpret_cast<float4 *>(sm.hs + static_cast<size_t>(r) * D + col) = v;
        }
        __syncthreads();
        if (c.active) {
#pragma unroll
            for (int k = 0; k <= TK; ++k) {
                const float4 v = *reinterpret_cast<const float4 *>(sm.hs + static_cast<size_t>(c.tb * TK + k) * D + c.d0);
                hp[k][0] = v.x; hp[k][1] = v.y; hp[k][2] = v.z; hp[k][3] = v.w;
            }
#pragma unroll
            for (int g = 0; g < 3; ++g)
#pragma unroll
                for (int k = 0; k < TK; ++k)
#pragma unroll
                    for (int j = 0; j < 4; ++j) G[g][k][j] = 0.f;
            const int DG = A.tl.DG;
            for (int m = 0; m < D; m += 4) {
                float4 hv[TK];
#pragma unroll
                for (int k = 0; k < TK; ++k)
                    hv[k] = *reinterpret_cast<const float4 *>(sm.hs + static_cast<size_t>(c.tb * TK + k) * D + m);
#pragma unroll
                for (int mm = 0; mm < 4; ++mm) {
                    const float4 u0 = *reinterpret_cast<const float4 *>(sm.Us + ((m + mm) * 3 + 0) * DG + c.lane0);
                    const float4 u1 = *reinterpret_cast<const float4 *>(sm.Us + ((m + mm) * 3 + 1) * DG + c.lane0);
                    const float4 u2 = *reinterpret_cast<const float4 *>(sm.Us + ((m + mm) * 3 + 2) * DG + c.lane0);
#pragma unroll
                    for (int k = 0; k < TK; ++k) {
                        const float h = get(hv[k], mm);
                        ffma2(G[0][k][0], G[0][k][1], u0.x, u0.y, h);
                        ffma2(G[0][k][2], G[0][k][3], u0.z, u0.w, h);
                        ffma2(G[1][k][0], G[1][k][1], u1.x, u1.y, h);
                        ffma2(G[1][k][2], G[1][k][3], u1.z, u1.w, h);
                        ffma2(G[2][k][0], G[2][k][1], u2.x, u2.y, h);
                        ffma2(G[2][k][2], G[2][k][3], u2.z, u2.w, h);
                    }
                }
            }
        }
    } else if (c.dvalid) {
#pragma unroll
        for (int k = 0; k <= TK; ++k) {
            const int t = c.t0 - 1 + k;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (t < 0)
                v = __ldg(reinterpret_cast<const float4 *>(A.h0 + static_cast<size_t>(c.b) * D + c.d0));
            else if (!zero_guess && t < T)
                v = ldcg4(hold + (static_cast<size_t>(c.b) * T + t) * D + c.d0);
            hp[k][0] = v.x; hp[k][1] = v.y; hp[k][2] = v.z; hp[k][3] = v.w;
        }
    }

    // per-lane constants: recurrent biases and the diagonal of each U_g
    float bh[3][4], ud[3][4];
    if (c.dvalid) {
#pragma unroll
        for (int g = 0; g < 3; ++g) {
            const float4 v = __ldg(reinterpret_cast<const float4 *>(A.b_hh + g * D + c.d0));
            bh[g][0] = v.x; bh[g][1] = v.y; bh[g][2] = v.z; bh[g][3] = v.w;
            if (DENSE) {
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    ud[g][j] = sm.Us[((c.d0 + j) * 3 + g) * A.tl.DG + c.lane0 + j];
            } else {
                const float4 u = __ldg(reinterpret_cast<const float4 *>(A.w_hh + g * D + c.d0));
                ud[g][0] = u.x; ud[g][1] = u.y; ud[g][2] = u.z; ud[g][3] = u.w;
            }
        }
    }

#pragma unroll
    for (int k = 0; k < TK; ++k) {
        const int t = c.t0 + k;
        const bool valid = c.dvalid && t < T;
        float4 pv[3];
        if (valid) {
            const float *prow = A.P + (static_cast<size_t>(c.b) * T + t) * rowP + c.d0;
#pragma unroll
            for (int g = 0; g < 3; ++g) pv[g] = __ldg(reinterpret_cast<const float4 *>(prow + g * D));
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (!valid) {
                a[k][j] = 1.f;
                bb[k][j] = 0.f;
                y[k][j] = 0.f;
                continue;
            }
            const float h = hp[k][j];
            const float gr = DENSE ? G[0][k][j] : ud[0][j] * h;
            const float gz = DENSE ? G[1][k][j] : ud[1][j] * h;
            const float gnh = DENSE ? G[2][k][j] : ud[2][j] * h;
            float f, aa, bv;
            gru_cell_diag(get(pv[0], j), get(pv[1], j), get(pv[2], j), gr, gz, gnh, bh[0][j], bh[1][j],
                          bh[2][j], ud[0][j], ud[1][j], ud[2][j], h, f, aa, bv);
            a[k][j] = aa;
            bb[k][j] = bv;
            y[k][j] = hp[k + 1][j];
            rmax = max(rmax, abs_bits(hp[k + 1][j] - f));
        }
    }
}

// ---------------------------------------------------------------------------
// 3. tile passes
// ---------------------------------------------------------------------------
// Forward affine scan of (a, bb) with the carry from the previous chunk; writes
// out[k][j] = state at step t0+k.  All threads of the CTA must call it.
template <int TK>
__device__ __forceinline__ void scan_forward(const DiagArgs &A, const TileCoord &c, const Smem &sm,
                                             unsigned long long *desc, unsigned epoch,
                                             const float (&a)[TK][4], const float (&bb)[TK][4],
                                             const float *carry0 /*[DG] for chunk 0*/,
                                             float (&out)[TK][4]) {
    const Tiling &tl = A.tl;
    float cA[4], cB[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) { cA[j] = 1.f; cB[j] = 0.f; }
#pragma unroll
    for (int k = 0; k < TK; ++k)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            cB[j] = fmaf(a[k][j], cB[j], bb[k][j]);
            cA[j] = a[k][j] * cA[j];
        }
    if (c.active)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            sm.s0[c.tb * tl.DG + c.lane0 + j] = cA[j];
            sm.s1[c.tb * tl.DG + c.lane0 + j] = cB[j];
        }
    __syncthreads();
    if (threadIdx.x < tl.DG) {
        const int lane = threadIdx.x;
        float EA = 1.f, EB = 0.f;
        for (int q = 0; q < tl.NTB; ++q) {
            const float qa = sm.s0[q * tl.DG + lane], qb = sm.s1[q * tl.DG + lane];
            sm.s0[q * tl.DG + lane] = EA;
            sm.s1[q * tl.DG + lane] = EB;
            EB = fmaf(qa, EB, qb);
            EA = qa * EA;
        }
        sm.c0[lane] = lookback_affine(desc, c.tile, tl.n_groups, tl.DG, lane, epoch, EA, EB,
                                      c.chunk, carry0[lane], &A.hdr->status);
    }
    __syncthreads();
    if (c.active) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int l = c.lane0 + j;
            float h = fmaf(sm.s0[c.tb * tl.DG + l], sm.c0[l], sm.s1[c.tb * tl.DG + l]);
#pragma unroll
            for (int k = 0; k < TK; ++k) {
                h = fmaf(a[k][j], h, bb[k][j]);
                out[k][j] = h;
            }
        }
    }
    __syncthreads();
}

template <int TK>
__device__ __forceinline__ void store_states(const DiagArgs &A, const TileCoord &c, float *dst,
                                             const float (&v)[TK][4]) {
    if (!c.dvalid) return;
#pragma unroll
    for (int k = 0; k < TK; ++k) {
        const int t = c.t0 + k;
        if (t < A.T)
            stcg4(dst + (static_cast<size_t>(c.b) * A.T + t) * A.D + c.d0,
                  make_float4(v[k][0], v[k][1], v[k][2], v[k][3]));
    }
}

template <int TK>
__device__ __forceinline__ void load_states(const DiagArgs &A, const TileCoord &c, const float *src,
                                            int shift, float (&v)[TK][4], float fill) {
#pragma unroll
    for (int k = 0; k < TK; ++k) {
        const int t = c.t0 + k + shift;
        float4 x = make_float4(fill, fill, fill, fill);
        if (c.dvalid && t < A.T) x = ldcg4(src + (static_cast<size_t>(c.b) * A.T + t) * A.D + c.d0);
        v[k][0] = x.x; v[k][1] = x.y; v[k][2] = x.z; v[k][3] = x.w;
    }
}

// carries of chunk 0 for this tile's lanes: h0 (mean) into sm.c1
__device__ __forceinline__ void load_h0_carry(const DiagArgs &A, const TileCoord &c, const Smem &sm) {
    if (threadIdx.x < A.tl.DG) {
        const int d = c.dg * A.tl.DG + threadIdx.x;
        sm.c1[threadIdx.x] = d < A.D ? __ldg(A.h0 + static_cast<size_t>(c.b) * A.D + d) : 0.f;
    }
    __syncthreads();
}

// --- quasi-DEER tile: linearise, scan, write, reduce ------------------------
template <int CELL, int TK>
__device__ void quasi_tile(const DiagArgs &A, long long tile, const Smem &sm, const float *hold,
                           float *hnew, bool zero_guess, unsigned epoch, unsigned &dmax,
                           unsigned &rmax) {
    const TileCoord c = tile_coord<TK>(A, tile);
    float a[TK][4], bb[TK][4], y[TK][4], out[TK][4];
    load_h0_carry(A, c, sm);
    linearise<CELL, TK>(A, c, sm, hold, zero_guess, a, bb, y, rmax);
    scan_forward(A, c, sm, A.desc, epoch, a, bb, sm.c1, out);
    if (c.dvalid) {
#pragma unroll
        for (int k = 0; k < TK; ++k)
            if (c.t0 + k < A.T)
#pragma unroll
                for (int j = 0; j < 4; ++j) dmax = max(dmax, abs_bits(out[k][j] - y[k][j]));
    }
    store_states(A, c, hnew, out);
}

// --- quasi-ELK forward tile: Kalman covariance (Mobius) + filtered mean -------
template <int CELL, int TK>
__device__ void elk_forward_tile(const DiagArgs &A, long long tile, const Smem &sm,
                                 const float *hold, bool zero_guess, unsigned epoch,
                                 unsigned &rmax) {
    const Tiling &tl = A.tl;
    const TileCoord c = tile_coord<TK>(A, tile);
    const float lam = A.lambda;
    float a[TK][4], bb[TK][4], y[TK][4];
    load_h0_carry(A, c, sm);
    linearise<CELL, TK>(A, c, sm, hold, zero_guess, a, bb, y, rmax);

    unsigned long long *desc_cov = A.desc;
    unsigned long long *desc_mean = A.desc + static_cast<size_t>(tl.n_tiles) * tl.DG * 4;

    // (i) covariance: P_t = M_t * P_{t-1} with M_t = [[a^2, 1], [lam a^2, 1 + lam]], P_0 = 0
    Mob cm[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) cm[j] = Mob{1.f, 0.f, 0.f, 1.f};
#pragma unroll
    for (int k = 0; k < TK; ++k)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float a2 = a[k][j] * a[k][j];
            const bool valid = c.dvalid && c.t0 + k < A.T;
            const Mob Mk = valid ? Mob{a2, 1.f, lam * a2, 1.f + lam} : Mob{1.f, 0.f, 0.f, 1.f};
            cm[j] = mob_mul(Mk, cm[j]);
        }
    if (c.active)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int idx = c.tb * tl.DG + c.lane0 + j;
            sm.s0[idx] = cm[j].m0; sm.s1[idx] = cm[j].m1; sm.s2[idx] = cm[j].m2; sm.s3[idx] = cm[j].m3;
        }
    __syncthreads();
    if (threadIdx.x < tl.DG) {
        const int lane = threadIdx.x;
        Mob E{1.f, 0.f, 0.f, 1.f};
        for (int q = 0; q < tl.NTB; ++q) {
            const int idx = q * tl.DG + lane;
            const Mob Q{sm.s0[idx], sm.s1[idx], sm.s2[idx], sm.s3[idx]};
            sm.s0[idx] = E.m0; sm.s1[idx] = E.m1; sm.s2[idx] = E.m2; sm.s3[idx] = E.m3;
            E = mob_mul(Q, E);
        }
        sm.c0[lane] = lookback_mobius(desc_cov, c.tile, tl.n_groups, tl.DG, lane, epoch, E,
                                      c.chunk, 0.f, &A.hdr->status);
    }
    __syncthreads();
    float Pk[TK][4], al[TK][4], be[TK][4];
    if (c.active) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int idx = c.tb * tl.DG + c.lane0 + j;
            const Mob E{sm.s0[idx], sm.s1[idx], sm.s2[idx], sm.s3[idx]};
            float P = mob_apply(E, sm.c0[c.lane0 + j]);
#pragma unroll
            for (int k = 0; k < TK; ++k) {
                const float Pm = fmaf(a[k][j] * a[k][j], P, 1.f);  // P-_t
                const float K = lam * Pm / (1.f + lam * Pm);       // gain; K = lam P_t
                P = Pm / (1.f + lam * Pm);
                Pk[k][j] = P;
                const float omk = 1.f - K;
                const bool valid = c.dvalid && c.t0 + k < A.T;
                al[k][j] = valid ? omk * a[k][j] : 1.f;
                be[k][j] = valid ? fmaf(omk, bb[k][j], K * y[k][j]) : 0.f;
            }
        }
    }
    __syncthreads();
    // (ii) filtered mean: m_t = (1 - K_t)(a_t m_{t-1} + b_t) + K_t y_t, m_0 = h0
    float m[TK][4];
    scan_forward(A, c, sm, desc_mean, epoch, al, be, sm.c1, m);
    store_states(A, c, A.elk_m, m);
    store_states(A, c, A.elk_p, Pk);
    store_states(A, c, A.elk_a, a);
    store_states(A, c, A.elk_b, bb);
}

// --- quasi-ELK backward tile: RTS smoother as a reverse affine scan ----------
template <int TK>
__device__ void elk_backward_tile(const DiagArgs &A, long long tile, const Smem &sm,
                                  const float *hold, float *hnew, bool zero_guess,
                                  unsigned epoch, unsigned &dmax) {
    const Tiling &tl = A.tl;
    const TileCoord c = tile_coord<TK>(A, tile);
    unsigned long long *desc_bwd = A.desc + static_cast<size_t>(tl.n_tiles) * tl.DG * 6;
    float m[TK][4], P[TK][4], an[TK][4], bn[TK][4], y[TK][4];
    load_states(A, c, A.elk_m, 0, m, 0.f);
    load_states(A, c, A.elk_p, 0, P, 0.f);
    load_states(A, c, A.elk_a, 1, an, 0.f);
    load_states(A, c, A.elk_b, 1, bn, 0.f);
    if (zero_guess) {
#pragma unroll
        for (int k = 0; k < TK; ++k)
#pragma unroll
            for (int j = 0; j < 4; ++j) y[k][j] = 0.f;
    } else {
        load_states(A, c, hold, 0, y, 0.f);
    }
    // s_t = G_t s_{t+1} + c_t,  G_t = P_t a_{t+1} / (a_{t+1}^2 P_t + 1),
    // c_t = m_t - G_t (a_{t+1} m_t + b_{t+1});  G = 0 at t = T-1; identity past T.
    float Gk[TK][4], Ck[TK][4];
#pragma unroll
    for (int k = 0; k < TK; ++k) {
        const int t = c.t0 + k;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (!c.dvalid || t >= A.T) { Gk[k][j] = 1.f; Ck[k][j] = 0.f; continue; }
            if (t == A.T - 1) { Gk[k][j] = 0.f; Ck[k][j] = m[k][j]; continue; }
            const float an_ = an[k][j];
            const float G = P[k][j] * an_ / fmaf(an_ * an_, P[k][j], 1.f);
            Gk[k][j] = G;
            Ck[k][j] = m[k][j] - G * fmaf(an_, m[k][j], bn[k][j]);
        }
    }
    // reverse composition within the thread: maps s_{t0+TK} -> s_{t0}
    float cG[4], cC[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) { cG[j] = 1.f; cC[j] = 0.f; }
#pragma unroll
    for (int k = TK - 1; k >= 0; --k)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            cC[j] = fmaf(Gk[k][j], cC[j], Ck[k][j]);
            cG[j] = Gk[k][j] * cG[j];
        }
    if (c.active)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            sm.s0[c.tb * tl.DG + c.lane0 + j] = cG[j];
            sm.s1[c.tb * tl.DG + c.lane0 + j] = cC[j];
        }
    __syncthreads();
    if (threadIdx.x < tl.DG) {
        const int lane = threadIdx.x;
        float EG = 1.f, EC = 0.f;
        for (int q = tl.NTB - 1; q >= 0; --q) {
            const float qg = sm.s0[q * tl.DG + lane], qc = sm.s1[q * tl.DG + lane];
            sm.s0[q * tl.DG + lane] = EG;
            sm.s1[q * tl.DG + lane] = EC;
            EC = fmaf(qg, EC, qc);
            EG = qg * EG;
        }
        sm.c0[lane] = lookback_affine(desc_bwd, c.tile, -static_cast<long long>(tl.n_groups),
                                      tl.DG, lane, epoch, EG, EC, tl.n_chunks - 1 - c.chunk,
                                      0.f, &A.hdr->status);
    }
    __syncthreads();
    float out[TK][4];
    if (c.active) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int l = c.lane0 + j;
            float s = fmaf(sm.s0[c.tb * tl.DG + l], sm.c0[l], sm.s1[c.tb * tl.DG + l]);
#pragma unroll
            for (int k = TK - 1; k >= 0; --k) {
                s = fmaf(Gk[k][j], s, Ck[k][j]);
                out[k][j] = s;
            }
        }
    }
    __syncthreads();
    if (c.dvalid) {
#pragma unroll
        for (int k = 0; k < TK; ++k)
            if (c.t0 + k < A.T)
#pragma unroll
                for (int j = 0; j < 4; ++j) dmax = max(dmax, abs_bits(out[k][j] - y[k][j]));
    }
    store_states(A, c, hnew, out);
}

// ---------------------------------------------------------------------------
// 4. the persistent kernel
// ---------------------------------------------------------------------------
template <int CELL, bool ELK, int TK>
__global__ void __launch_bounds__(kThreads, ELK ? 1 : 2) diag_solver_kernel(DiagArgs A) {
    extern __shared__ float4 smem_raw[];
    const Tiling &tl = A.tl;
    const Smem sm = carve(reinterpret_cast<float *>(smem_raw), tl, A.D, CELL);
    WsHeader *hdr = A.hdr;
    unsigned *status = &hdr->status;
    const unsigned nblocks = gridDim.x;

    if (CELL == kCellDenseFma) {
        // U^T slices into shared memory, layout [m][g][lane]: Us = U_g[lane][m]
        const int D = A.D, n = D * 3 * tl.DG;
        for (int i = threadIdx.x; i < n; i += kThreads) {
            const int lane = i % tl.DG, g = (i / tl.DG) % 3, m = i / (3 * tl.DG);
            sm.Us[i] = __ldg(A.w_hh + (static_cast<size_t>(g) * D + lane) * D + m);
        }
        __syncthreads();
    }

    int it = 0;
    int iters = 0;
    int final_status = PARARNN_NOT_CONVERGED;
    unsigned last_delta = 0u, last_resid = 0u;
    for (; it < A.max_iters; ++it) {
        if (blockIdx.x == 0 && threadIdx.x == 0) {
            hdr->delta_bits[(it + 1) % 3] = 0u;
            hdr->resid_bits[(it + 1) % 3] = 0u;
        }
        const float *hold = A.hbuf[it & 1];
        float *hnew = A.hbuf[(it + 1) & 1];
        const bool zero_guess = it == 0 && !A.warm;  // the first guess: zero, or the caller's
        const unsigned epoch = static_cast<unsigned>(it + 1);
        unsigned dmax = 0u, rmax = 0u;
        if (!ELK) {
            for (long long tile = blockIdx.x; tile < tl.n_tiles; tile += nblocks)
                quasi_tile<CELL, TK>(A, tile, sm, hold, hnew, zero_guess, epoch, dmax, rmax);
        } else {
            for (long long tile = blockIdx.x; tile < tl.n_tiles; tile += nblocks)
                elk_forward_tile<CELL, TK>(A, tile, sm, hold, zero_guess, epoch, rmax);
            grid_barrier(hdr->barrier, nblocks, status);
            for (long long k = blockIdx.x; k < tl.n_tiles; k += nblocks)
                elk_backward_tile<TK>(A, tl.n_tiles - 1 - k, sm, hold, hnew, zero_guess, epoch, dmax);
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
    // the final iterate lives in hbuf[iters & 1]; hbuf[1] is the caller's array
    if ((iters & 1) == 0 && iters > 0) {
        const size_t n4 = static_cast<size_t>(A.B) * A.T * A.D / 4;
        const float4 *src = reinterpret_cast<const float4 *>(A.hbuf[0]);
        float4 *dst = reinterpret_cast<float4 *>(A.hbuf[1]);
        for (size_t i = static_cast<size_t>(blockIdx.x) * kThreads + threadIdx.x; i < n4;
             i += static_cast<size_t>(nblocks) * kThreads)
            dst[i] = __ldcg(src + i);
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

template <int CELL, bool ELK, int TK>
cudaError_t launch_one(const DiagArgs &a, cudaStream_t s) {
    auto kern = diag_solver_kernel<CELL, ELK, TK>;
    const size_t smem = smem_floats(a.tl, a.D, CELL) * sizeof(float);
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
    if (grid > a.tl.n_tiles) grid = a.tl.n_tiles;
    DiagArgs args = a;
    void *params[] = {&args};
    return cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(kern),
                                       dim3(static_cast<unsigned>(grid)), dim3(kThreads), params,
                                       smem, s);
}

}  // namespace

static int cell_variant(const pararnn_cell &cell) {
    if (cell.kind != PARARNN_GRU_DENSE) return kCellDiag;
    const int D = cell.d;
    return (D == 8 || D == 16 || D == 32 || D == 64) ? kCellDenseMma : kCellDenseFma;
}

cudaError_t launch_diag_solver(const pararnn_cell &cell, int mode, const DiagArgs &a,
                               cudaStream_t s) {
    const bool elk = mode == PARARNN_ELK || mode == PARARNN_QUASI_ELK;
    if (a.tl.TK != kSolverTK) return cudaErrorInvalidValue;
    switch (cell_variant(cell)) {
        case kCellDenseMma:
            return elk ? launch_one<kCellDenseMma, true, kSolverTK>(a, s)
                       : launch_one<kCellDenseMma, false, kSolverTK>(a, s);
        case kCellDenseFma:
            return elk ? launch_one<kCellDenseFma, true, kSolverTK>(a, s)
                       : launch_one<kCellDenseFma, false, kSolverTK>(a, s);
        default:
            return elk ? launch_one<kCellDiag, true, kSolverTK>(a, s)
                       : launch_one<kCellDiag, false, kSolverTK>(a, s);
    }
}

}  // namespace pararnn

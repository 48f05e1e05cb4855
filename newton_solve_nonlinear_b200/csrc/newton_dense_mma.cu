// newton_dense_mma.cu -- DEER (full Jacobian) on the dense GRU for D <= 32,
// with the Jacobian products on the tensor cores.
//
// DEER ("Parallelizing non-linear sequential models over the sequence
// length", abstract; "ParaRNN" summary, "Newton's Iteration") solves each
// Newton step, in delta form dh_t = J_t dh_{t-1} - r_t (dh_0 = 0,
// r_t = h^(i)_t - f(h^(i)_{t-1}, x_t)), by a parallel scan whose elements are
// D x D matrices; composing them is cubic in D per step (ELK abstract).
//
// Work unit: one warp owns one chunk of L steps of one sequence; L is chosen
// at launch so that the chunks of all sequences fill the resident warps once
// (a multiple of the 16-step staging block).  Per Newton iteration:
//   P1  chunk aggregates.  The warp walks its chunk once, evaluating the cell
//       at the old guess and forming J_t in registers, and accumulates
//       Psi = Phi_c^T = J_first^T ... J_last^T on mma.sync m16n8k8 (TF32
//       operands, fp32 accumulation) together with the particular solution
//       p_c (dh with zero carry-in) in fp32.  The product never leaves
//       registers: the accumulator fragment of one step is the A fragment of
//       the next once the K index inside each 8-wide slice is permuted
//       (slot s <-> column 2s, slot s+4 <-> column 2s+1), and J_t^T is built
//       directly in that permuted order.
//   P2a group aggregates: a warp composes G ~ sqrt(chunks) consecutive chunk
//       aggregates the same way (Phi_g, p_g).
//   P2b carries: the warp of each group runs the matrix-vector recurrence
//       over the earlier groups' aggregates for the group's carry-in, then
//       over its own chunks for theirs.  Phase 2 streams the aggregates
//       through shared memory one element ahead (cp.async).
//   P3  re-sweep: the warp walks its chunk again from its true carry-in in
//       fp32, dh_t = J_t dh_{t-1} - r_t, writes h^(i+1) = h^(i) + dh and
//       reduces max |dh| and max |r|.
// Only the carries pass through the TF32 products; every state is produced by
// the fp32 re-sweep, so the fixed point (r = 0) is exact in fp32 and a
// rounded product only perturbs the step, not where the iteration ends.
//
// Jacobian reuse (approximate Newton: the Jacobian recomputed only every few
// iterations, "ParaRNN" summary, "Newton's Iteration").  With jac_every = k > 1
// the J_t of iteration i are those of iteration k floor(i / k): a refreshing
// iteration runs as above and also stores the per-row coefficients
// (z, cz, cn, cr) of every step, 512 bytes per step; the k - 1 iterations after
// it reload them instead of taking them from the new guess.  Their chunk and
// group products Phi are then still the refreshed ones, so those iterations
// skip every matrix-matrix product: P1 and P2a shrink to the matrix-vector
// recurrences of the particular solutions, and each step of the iteration
// costs O(D^2) instead of O(D^3).  The residual r_t always comes from the
// current guess, so the fixed point is unchanged.
//
// Lane layout (lane = 4 gid + tq): rows R(nt) = 8 nt + gid, columns
// C(kt, e) = 8 kt + 2 tq + e, nt, kt in 0..3, e in 0..1.  Each lane keeps
// U_g[R(nt)][C(kt, e)] for the three gates (96 registers): they serve both
// U h^(i)_{t-1} (partial sums reduced over the 4 lanes of a quad) and the
// Jacobian entries J[R(nt)][C(kt, e)], which are exactly the lane's B
// fragment entries.  Vectors are held twice: by rows (all four quad lanes
// hold dh[R(nt)]) and by columns (dh[C(kt, e)]), one shuffle apart.
#include "common.cuh"
#include "solver.cuh"

namespace pararnn {

namespace {

constexpr int kBlk = 16;   // steps per staged block (chunk lengths are multiples)
constexpr int kMaxWarps = 4096;  // bound on resident warps used to size the workspace
constexpr int kWarps = kThreads / 32;
constexpr int kPB = kBlk * 96;        // staged P floats per block ([step][gate][32])
constexpr int kHB = (kBlk + 1) * 32;  // staged guess floats per block ([row][32])
constexpr int kCS = 164;              // coefficient step stride: [gid][z, cz, cn, cr, r][nt] (+4 pad)
constexpr int kWarpSmem = 2 * (kPB + kHB) + kBlk * kCS;
constexpr size_t kSmemBytes = (96 + kWarps * kWarpSmem + 32) * sizeof(float);

struct MmaArgs {
    DiagArgs a;
    int L, NC;   // steps per chunk, chunks per sequence
    int G, NG;   // chunks per group, groups per sequence
    float *PhiC, *pC, *PhiG, *pG, *carryC;
};

// The frozen coefficients: step t of sequence b is 128 floats, [gid][z, cz, cn,
// cr][nt] (the coefficient block's layout without the residual), one float4
// per lane.
__device__ __forceinline__ float *coef_step(const DiagArgs &A, int b, int t) {
    return A.coef + (static_cast<size_t>(b) * A.T + t) * 128;
}

// mma.sync with .tf32 operands reads the top 19 bits of each 32-bit register
// (the low 13 mantissa bits are ignored: truncation), so fp32 values are passed
// as they are wherever TF32 accuracy is the intent.
__device__ __forceinline__ unsigned bits(float x) { return __float_as_uint(x); }

// (c0, c1) += (a0, a1) * (b0, b1), one packed fp32x2 FMA.
__device__ __forceinline__ void ffma2v(float &c0, float &c1, float a0, float a1, float b0, float b1) {
    asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
        "mov.b64 ra, {%2, %3};\n\t"
        "mov.b64 rb, {%4, %5};\n\t"
        "mov.b64 rc, {%0, %1};\n\t"
        "fma.rn.f32x2 rc, ra, rb, rc;\n\t"
        "mov.b64 {%0, %1}, rc;\n\t}"
        : "+f"(c0), "+f"(c1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

__device__ __forceinline__ void mma8(float (&c)[4], unsigned a0, unsigned a1, unsigned a2,
                                     unsigned a3, unsigned b0, unsigned b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// d = A B (zero accumulator).
__device__ __forceinline__ void mma8z(float (&d)[4], unsigned a0, unsigned a1, unsigned a2,
                                      unsigned a3, unsigned b0, unsigned b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.f));
}

__device__ __forceinline__ void cp16(float *dst, const float *src) {
    const unsigned d = static_cast<unsigned>(__cvta_generic_to_shared(dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Quad reduction: every lane of the quad gets the sum over its 4 lanes.
__device__ __forceinline__ float quad_sum(float v) {
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    return v;
}

// Row layout -> column layout: col[kt][e] = x[C(kt, e)] from row[nt] = x[R(nt)].
__device__ __forceinline__ void rows_to_cols(const float (&row)[4], float (&col)[4][2], int tq) {
#pragma unroll
    for (int kt = 0; kt < 4; ++kt)
#pragma unroll
        for (int e = 0; e < 2; ++e) col[kt][e] = __shfl_sync(0xffffffffu, row[kt], (2 * tq + e) * 4);
}

struct Lane {
    int lane, gid, tq;
};

__device__ __forceinline__ Lane lane_ids() {
    Lane l;
    l.lane = threadIdx.x & 31;
    l.gid = l.lane >> 2;
    l.tq = l.lane & 3;
    return l;
}

// Per-lane copy of U_g[R(nt)][C(kt, e)] (zero outside D x D).
__device__ __forceinline__ void load_u(float (&u)[3][4][4][2], const float *w_hh, int D,
                                       const Lane &L) {
#pragma unroll
    for (int g = 0; g < 3; ++g)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int kt = 0; kt < 4; ++kt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int i = nt * 8 + L.gid, k = kt * 8 + 2 * L.tq + e;
                    u[g][nt][kt][e] =
                        (i < D && k < D) ? __ldg(w_hh + (static_cast<size_t>(g) * D + i) * D + k) : 0.f;
                }
}

// Stage steps tb .. tb+n-1 (P rows, gates padded to 32) and guess rows
// tb-1 .. tb+n-1 of sequence b into one warp buffer.  Padding entries of the
// buffers are zero from the start and never written.
__device__ void stage_block(const DiagArgs &A, float *buf, int b, int tb, int n, const float *hold,
                            bool zero_guess, int lane) {
    const int D = A.D, T = A.T, DV = D / 4;
    float *Pb = buf, *Hb = buf + kPB;
    const int g = lane >> 3, j = lane & 7;  // P: lane = (gate, float4) of one row per pass
    if (g < 3 && j < DV) {
        const float *src = A.P + (static_cast<size_t>(b) * T + tb) * 3 * D + g * D + 4 * j;
        for (int r = 0; r < n; ++r) cp16(Pb + r * 96 + g * 32 + 4 * j, src + static_cast<size_t>(r) * 3 * D);
    }
    if (j < DV) {  // guess rows tb-1 .. tb+n-1: lane = (row mod 4, float4)
        for (int r = g; r <= n; r += 4) {
            const int t = tb - 1 + r;
            float *dst = Hb + r * 32 + 4 * j;
            if (t < 0)
                cp16(dst, A.h0 + static_cast<size_t>(b) * D + 4 * j);
            else if (!zero_guess)
                cp16(dst, hold + (static_cast<size_t>(b) * T + t) * D + 4 * j);
            else
                *reinterpret_cast<float4 *>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    cp_commit();
}

// Cell at the guess for the steps of one staged block, batched: the gate
// pre-activations U_g h_{t-1} of all 16 steps are one m16 x n96 x k32 product
// on mma.sync (3 x TF32 split, fp32-accurate), with the lane's U entries as
// the B fragments (the same permuted K order as the chain).  The accumulator
// then holds, per thread, all three gates of steps s = gid, gid + 8 and rows
// i = 8 nt + 2 tq + e, so the cell is evaluated in place and its Jacobian
// coefficients z, cz, cn, cr and residual r are written to `cf`, laid out
// [s][i mod 8][coefficient][i / 8] so that a lane reads its rows R(nt) as
// five float4.
__device__ void block_coefs(const float (&u)[3][4][4][2], const float *Pb, const float *Hb,
                            const float *bh, int D, const Lane &L, float *cf, bool coefs = true) {
#pragma unroll
    for (int np = 0; np < 2; ++np) {  // row tiles in pairs: six independent accumulation chains
        float acc[2][3][4];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int g = 0; g < 3; ++g)
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[h][g][q] = 0.f;
#pragma unroll
        for (int kt = 0; kt < 4; ++kt) {
            const float2 r0 = *reinterpret_cast<const float2 *>(Hb + L.gid * 32 + kt * 8 + 2 * L.tq);
            const float2 r1 =
                *reinterpret_cast<const float2 *>(Hb + (L.gid + 8) * 32 + kt * 8 + 2 * L.tq);
            const float av[4] = {r0.x, r1.x, r0.y, r1.y};
            unsigned ah[4], al[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                ah[q] = __float_as_uint(av[q]) & 0xffffe000u;
                al[q] = __float_as_uint(av[q] - __uint_as_float(ah[q]));
            }
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int g = 0; g < 3; ++g) {
                    const int nt = 2 * np + h;
                    const unsigned bh0 = __float_as_uint(u[g][nt][kt][0]) & 0xffffe000u;
                    const unsigned bh1 = __float_as_uint(u[g][nt][kt][1]) & 0xffffe000u;
                    const unsigned bl0 = __float_as_uint(u[g][nt][kt][0] - __uint_as_float(bh0));
                    const unsigned bl1 = __float_as_uint(u[g][nt][kt][1] - __uint_as_float(bh1));
                    mma8(acc[h][g], al[0], al[1], al[2], al[3], bh0, bh1);
                    mma8(acc[h][g], ah[0], ah[1], ah[2], ah[3], bl0, bl1);
                    mma8(acc[h][g], ah[0], ah[1], ah[2], ah[3], bh0, bh1);
                }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int nt = 2 * np + h;
                const int s = L.gid + 8 * (q >> 1), i = nt * 8 + 2 * L.tq + (q & 1);
                const float *Pt = Pb + s * 96;
                const float r = sigmoidf_(Pt[i] + acc[h][0][q] + bh[i]);
                const float z = sigmoidf_(Pt[32 + i] + acc[h][1][q] + bh[32 + i]);
                const float gn = acc[h][2][q] + bh[64 + i];
                const float nn = tanhf_(Pt[64 + i] + r * gn);
                const float hprev = Hb[s * 32 + i];
                const float f = nn + z * (hprev - nn);
                const float omz = 1.f - z;
                const float cn = omz * (1.f - nn * nn) * r;
                const bool live = i < D;
                float *o = cf + s * kCS + (2 * L.tq + (q & 1)) * 20 + nt;  // row i = 8 nt + gid'
                if (coefs) {  // else they come from the frozen copy
                    o[0] = live ? z : 0.f;
                    o[4] = live ? (hprev - nn) * z * omz : 0.f;
                    o[8] = live ? cn : 0.f;
                    o[12] = live ? cn * gn * (1.f - r) : 0.f;
                }
                o[16] = live ? Hb[(s + 1) * 32 + i] - f : 0.f;
            }
    }
}

// Jacobian coefficients and residual of rows R(nt) at step s of the block.
struct Coef {
    float z[4], cz[4], cn[4], cr[4], res[4];
};

__device__ __forceinline__ void read_coefs(const float *cf, int s, const Lane &L, Coef &C) {
    const float4 *o = reinterpret_cast<const float4 *>(cf + s * kCS + L.gid * 20);
    const float4 z = o[0], cz = o[1], cn = o[2], cr = o[3], res = o[4];
    C.z[0] = z.x; C.z[1] = z.y; C.z[2] = z.z; C.z[3] = z.w;
    C.cz[0] = cz.x; C.cz[1] = cz.y; C.cz[2] = cz.z; C.cz[3] = cz.w;
    C.cn[0] = cn.x; C.cn[1] = cn.y; C.cn[2] = cn.z; C.cn[3] = cn.w;
    C.cr[0] = cr.x; C.cr[1] = cr.y; C.cr[2] = cr.z; C.cr[3] = cr.w;
    C.res[0] = res.x; C.res[1] = res.y; C.res[2] = res.z; C.res[3] = res.w;
}

// Frozen coefficients of the block's steps tb .. tb+n-1: store from, or
// fetch (cp.async, one commit group) into, the coefficient block.
__device__ __forceinline__ void coefs_store(const DiagArgs &A, const float *cf, int b, int tb, int n, const Lane &L) {
    for (int s = 0; s < n; ++s)
        __stcg(reinterpret_cast<float4 *>(coef_step(A, b, tb + s)) + L.lane,
               *reinterpret_cast<const float4 *>(cf + s * kCS + L.gid * 20 + L.tq * 4));
}
__device__ __forceinline__ void coefs_fetch(const DiagArgs &A, float *cf, int b, int tb, int n, const Lane &L) {
    for (int s = 0; s < n; ++s) cp16(cf + s * kCS + L.gid * 20 + L.tq * 4, coef_step(A, b, tb + s) + 4 * L.lane);
    cp_commit();
}

// J[R(nt)][C(kt, e)] for one kt (pairs e = 0, 1 as packed FMAs).  dz0, dz1:
// 1 where R(kt) is C(kt, 0) resp. C(kt, 1) (the diagonal of J), else 0.
__device__ __forceinline__ void jac_slice(const float (&u)[3][4][4][2], const Coef &C, int kt,
                                          float dz0, float dz1, float (&j)[4][2]) {
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
        float v0 = 0.f, v1 = 0.f;
        if (nt == kt) {
            v0 = dz0 * C.z[nt];
            v1 = dz1 * C.z[nt];
        }
        ffma2(v0, v1, u[0][nt][kt][0], u[0][nt][kt][1], C.cr[nt]);
        ffma2(v0, v1, u[2][nt][kt][0], u[2][nt][kt][1], C.cn[nt]);
        ffma2(v0, v1, u[1][nt][kt][0], u[1][nt][kt][1], C.cz[nt]);
        j[nt][0] = v0;
        j[nt][1] = v1;
    }
}

// Psi <- Psi B^T over one K slice kt (B entries in the lane layout), into
// acc; the first slice starts from a zero accumulator.
__device__ __forceinline__ void chain_slice(const float (&psi)[2][4][4], float (&acc)[2][4][4],
                                            const float (&bj)[4][2], int kt) {
    unsigned a[2][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
        a[mt][0] = bits(psi[mt][kt][0]);
        a[mt][1] = bits(psi[mt][kt][2]);
        a[mt][2] = bits(psi[mt][kt][1]);
        a[mt][3] = bits(psi[mt][kt][3]);
    }
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
        const unsigned b0 = bits(bj[nt][0]), b1 = bits(bj[nt][1]);
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            if (kt == 0)
                mma8z(acc[mt][nt], a[mt][0], a[mt][1], a[mt][2], a[mt][3], b0, b1);
            else
                mma8(acc[mt][nt], a[mt][0], a[mt][1], a[mt][2], a[mt][3], b0, b1);
        }
    }
}

__device__ __forceinline__ void psi_identity(float (&psi)[2][4][4], const Lane &L) {
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int m = mt * 16 + L.gid + 8 * (q >> 1), j = nt * 8 + 2 * L.tq + (q & 1);
                psi[mt][nt][q] = m == j ? 1.f : 0.f;
            }
}

// Store Phi = Psi^T row-major [32][32].
__device__ __forceinline__ void store_phi(float *dst, const float (&psi)[2][4][4], const Lane &L) {
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int m = mt * 16 + L.gid + 8 * (q >> 1), j = nt * 8 + 2 * L.tq + (q & 1);
                __stcg(dst + j * 32 + m, psi[mt][nt][q]);
            }
}

// y[R(nt)] = sum_k M[R(nt)][k] x[k] + add[R(nt)] from the lane's entries of M.
__device__ __forceinline__ void matvec(const float (&m)[4][4][2], const float (&xc)[4][2],
                                       const float (&add)[4], float (&row)[4]) {
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
        float s = 0.f;
#pragma unroll
        for (int kt = 0; kt < 4; ++kt) s = fmaf(m[nt][kt][0], xc[kt][0], fmaf(m[nt][kt][1], xc[kt][1], s));
        row[nt] = quad_sum(s) + add[nt];
    }
}

struct WarpCtx {
    const float *bh;
    float *buf;  // this warp's two staging buffers
    float *cf;   // this warp's coefficient block
};

// One step of the chunk chain: pout = pin J_t^T (kChain), p <- J_t p - r_t.
template <bool kChain = true>
__device__ __forceinline__ void chain_step(const float (&u)[3][4][4][2], const float *cf, int s,
                                           const Lane &L, float dz0, float dz1,
                                           const float (&pin)[2][4][4], float (&pout)[2][4][4],
                                           float (&pcol)[4][2], float (&prow)[4]) {
    Coef C;
    read_coefs(cf, s, L, C);
    float q0[4] = {}, q1[4] = {};
#pragma unroll
    for (int kt = 0; kt < 4; ++kt) {
        float bj[4][2];
        jac_slice(u, C, kt, dz0, dz1, bj);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) ffma2v(q0[nt], q1[nt], bj[nt][0], bj[nt][1], pcol[kt][0], pcol[kt][1]);
        if constexpr (kChain) chain_slice(pin, pout, bj, kt);
    }
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) prow[nt] = quad_sum(q0[nt] + q1[nt]) - C.res[nt];
    rows_to_cols(prow, pcol, L.tq);
}

// P1: aggregate (Phi_c, p_c) of chunk c of sequence b.  fresh: the Jacobian
// is taken at this guess (stored when it is to be reused); else the frozen
// one is reloaded and only p_c is formed (Phi_c is the refreshed one).
__device__ void chunk_aggregate(const MmaArgs &S, const WarpCtx &W, int b, int c, const float *hold,
                                bool zero_guess, bool fresh) {
    const bool reuse = S.a.jac_every > 1;
    const DiagArgs &A = S.a;
    const Lane L = lane_ids();
    const int t0 = c * S.L, n = min(S.L, A.T - t0), nb = (n + kBlk - 1) / kBlk;
    const float dz0 = L.gid == 2 * L.tq ? 1.f : 0.f, dz1 = L.gid == 2 * L.tq + 1 ? 1.f : 0.f;
    float u[3][4][4][2];
    load_u(u, A.w_hh, A.D, L);
    float psi[2][4][4], tmp[2][4][4];
    psi_identity(psi, L);
    float pcol[4][2] = {}, prow[4] = {};
    stage_block(A, W.buf, b, t0, min(kBlk, n), hold, zero_guess, L.lane);
    for (int blk = 0; blk < nb; ++blk) {
        const int tb = t0 + blk * kBlk, nblk = min(kBlk, n - blk * kBlk);
        if (blk + 1 < nb) {
            stage_block(A, W.buf + ((blk + 1) & 1) * (kPB + kHB), b, tb + kBlk,
                        min(kBlk, n - (blk + 1) * kBlk), hold, zero_guess, L.lane);
            cp_wait<1>();
        } else {
            cp_wait<0>();
        }
        __syncwarp();
        const float *Pb = W.buf + (blk & 1) * (kPB + kHB), *Hb = Pb + kPB;
        if (!fresh) coefs_fetch(A, W.cf, b, tb, nblk, L);
        block_coefs(u, Pb, Hb, W.bh, A.D, L, W.cf, fresh);
        if (!fresh) cp_wait<0>();
        __syncwarp();
        if (!fresh) {
            for (int s = 0; s < nblk; ++s) chain_step<false>(u, W.cf, s, L, dz0, dz1, psi, tmp, pcol, prow);
            __syncwarp();
            continue;
        }
        if (reuse) coefs_store(A, W.cf, b, tb, nblk, L);
        int s = 0;
        for (; s + 1 < nblk; s += 2) {
            chain_step(u, W.cf, s, L, dz0, dz1, psi, tmp, pcol, prow);
            chain_step(u, W.cf, s + 1, L, dz0, dz1, tmp, psi, pcol, prow);
        }
        if (s < nblk) {
            chain_step(u, W.cf, s, L, dz0, dz1, psi, tmp, pcol, prow);
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                    for (int q = 0; q < 4; ++q) psi[mt][nt][q] = tmp[mt][nt][q];
        }
        __syncwarp();
    }
    const size_t idx = static_cast<size_t>(b) * S.NC + c;
    if (fresh) store_phi(S.PhiC + idx * 1024, psi, L);
    if (L.tq == 0)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) __stcg(S.pC + idx * 32 + nt * 8 + L.gid, prow[nt]);
}

// Stream element k of an aggregate list (Phi [32][32], p [32]) into a
// shared-memory slot of 1056 floats.
__device__ __forceinline__ void stage_agg(float *slot, const float *Phi, const float *p, int lane) {
    for (int q = lane; q < 264; q += 32) cp16(slot + 4 * q, q < 256 ? Phi + 4 * q : p + 4 * (q - 256));
    cp_commit();
}

__device__ __forceinline__ void read_agg(const float *slot, const Lane &L, float (&ph)[4][4][2],
                                         float (&pv)[4]) {
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
        for (int kt = 0; kt < 4; ++kt) {
            const float2 v =
                *reinterpret_cast<const float2 *>(slot + (nt * 8 + L.gid) * 32 + kt * 8 + 2 * L.tq);
            ph[nt][kt][0] = v.x;
            ph[nt][kt][1] = v.y;
        }
        pv[nt] = slot[1024 + nt * 8 + L.gid];
    }
}

// P2a: aggregate of group g of sequence b (chunks g G .. g G + G - 1); with a
// frozen Jacobian (not fresh) only p_g: Phi_g is the refreshed one.
__device__ void group_aggregate(const MmaArgs &S, const WarpCtx &W, int b, int g, bool fresh) {
    const Lane L = lane_ids();
    const int c0 = g * S.G, c1 = min(S.NC, c0 + S.G);
    float psi[2][4][4];
    psi_identity(psi, L);
    float pcol[4][2] = {}, prow[4] = {};
    const size_t base = static_cast<size_t>(b) * S.NC;
    stage_agg(W.buf, S.PhiC + (base + c0) * 1024, S.pC + (base + c0) * 32, L.lane);
    for (int c = c0; c < c1; ++c) {
        const int slot = (c - c0) & 1;
        if (c + 1 < c1) {
            stage_agg(W.buf + (slot ^ 1) * 1056, S.PhiC + (base + c + 1) * 1024,
                      S.pC + (base + c + 1) * 32, L.lane);
            cp_wait<1>();
        } else {
            cp_wait<0>();
        }
        __syncwarp();
        float ph[4][4][2], pc[4];
        read_agg(W.buf + slot * 1056, L, ph, pc);
        if (fresh) {
            float acc[2][4][4];
#pragma unroll
            for (int kt = 0; kt < 4; ++kt) {
                float bj[4][2];
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
                    bj[nt][0] = ph[nt][kt][0];
                    bj[nt][1] = ph[nt][kt][1];
                }
                chain_slice(psi, acc, bj, kt);
            }
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                    for (int q = 0; q < 4; ++q) psi[mt][nt][q] = acc[mt][nt][q];
        }
        matvec(ph, pcol, pc, prow);
        rows_to_cols(prow, pcol, L.tq);
        __syncwarp();
    }
    const size_t idx = static_cast<size_t>(b) * S.NG + g;
    if (fresh) store_phi(S.PhiG + idx * 1024, psi, L);
    if (L.tq == 0)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) __stcg(S.pG + idx * 32 + nt * 8 + L.gid, prow[nt]);
}

// x <- Phi_k x + p_k over k = k0 .. k1-1 (aggregate lists in global memory,
// streamed through the warp's buffer); when `carry` is set, stores the
// carry-in of each k there.
__device__ void carry_chain(const WarpCtx &W, const float *Phi, const float *p, float *carry, int k0,
                            int k1, float (&xrow)[4]) {
    const Lane L = lane_ids();
    float xcol[4][2];
    rows_to_cols(xrow, xcol, L.tq);
    if (k0 < k1) stage_agg(W.buf, Phi + static_cast<size_t>(k0) * 1024, p + static_cast<size_t>(k0) * 32, L.lane);
    for (int k = k0; k < k1; ++k) {
        const int slot = (k - k0) & 1;
        if (k + 1 < k1) {
            stage_agg(W.buf + (slot ^ 1) * 1056, Phi + static_cast<size_t>(k + 1) * 1024,
                      p + static_cast<size_t>(k + 1) * 32, L.lane);
            cp_wait<1>();
        } else {
            cp_wait<0>();
        }
        __syncwarp();
        if (carry != nullptr && L.tq == 0)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) __stcg(carry + static_cast<size_t>(k) * 32 + nt * 8 + L.gid, xrow[nt]);
        float ph[4][4][2], pk[4];
        read_agg(W.buf + slot * 1056, L, ph, pk);
        matvec(ph, xcol, pk, xrow);
        rows_to_cols(xrow, xcol, L.tq);
        __syncwarp();
    }
}

// P3: re-sweep chunk c of sequence b from its carry-in.
__device__ void chunk_sweep(const MmaArgs &S, const WarpCtx &W, int b, int c, const float *hold,
                            float *hnew, bool zero_guess, bool fresh, unsigned &dmax, unsigned &rmax) {
    const DiagArgs &A = S.a;
    const Lane L = lane_ids();
    const int D = A.D, T = A.T;
    const int t0 = c * S.L, n = min(S.L, T - t0), nb = (n + kBlk - 1) / kBlk;
    const float dz0 = L.gid == 2 * L.tq ? 1.f : 0.f, dz1 = L.gid == 2 * L.tq + 1 ? 1.f : 0.f;
    float u[3][4][4][2];
    load_u(u, A.w_hh, D, L);
    float drow[4], dcol[4][2];
    const float *cin = S.carryC + (static_cast<size_t>(b) * S.NC + c) * 32;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) drow[nt] = __ldcg(cin + nt * 8 + L.gid);
    rows_to_cols(drow, dcol, L.tq);
    stage_block(A, W.buf, b, t0, min(kBlk, n), hold, zero_guess, L.lane);
    for (int blk = 0; blk < nb; ++blk) {
        const int tb = t0 + blk * kBlk, nblk = min(kBlk, n - blk * kBlk);
        if (blk + 1 < nb) {
            stage_block(A, W.buf + ((blk + 1) & 1) * (kPB + kHB), b, tb + kBlk,
                        min(kBlk, n - (blk + 1) * kBlk), hold, zero_guess, L.lane);
            cp_wait<1>();
        } else {
            cp_wait<0>();
        }
        __syncwarp();
        const float *Pb = W.buf + (blk & 1) * (kPB + kHB), *Hb = Pb + kPB;
        if (!fresh) coefs_fetch(A, W.cf, b, tb, nblk, L);
        block_coefs(u, Pb, Hb, W.bh, D, L, W.cf, fresh);
        if (!fresh) cp_wait<0>();
        __syncwarp();
        for (int s = 0; s < nblk; ++s) {
            Coef C;
            const float *hc = Hb + (s + 1) * 32;
            read_coefs(W.cf, s, L, C);
            float q0[4] = {}, q1[4] = {};
#pragma unroll
            for (int kt = 0; kt < 4; ++kt) {
                float bj[4][2];
                jac_slice(u, C, kt, dz0, dz1, bj);
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
                    ffma2v(q0[nt], q1[nt], bj[nt][0], bj[nt][1], dcol[kt][0], dcol[kt][1]);
            }
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                drow[nt] = quad_sum(q0[nt] + q1[nt]) - C.res[nt];
                rmax = max(rmax, abs_bits(C.res[nt]));
            }
            rows_to_cols(drow, dcol, L.tq);
            const size_t o = (static_cast<size_t>(b) * T + tb + s) * D;
            if (L.tq == 0)
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
                    const int i = nt * 8 + L.gid;
                    if (i < D) {
                        __stcg(hnew + o + i, hc[i] + drow[nt]);
                        dmax = max(dmax, abs_bits(drow[nt]));
                    }
                }
        }
        __syncwarp();
    }
}

__global__ void __launch_bounds__(kThreads, 1) deer_mma_kernel(MmaArgs S) {
    extern __shared__ float4 smem_raw[];
    float *smem = reinterpret_cast<float *>(smem_raw);
    const DiagArgs &A = S.a;
    WsHeader *hdr = A.hdr;
    unsigned *status = &hdr->status;
    const unsigned nblocks = gridDim.x;
    const int D = A.D, B = A.B;
    float *bh = smem, *wbase = bh + 96;
    unsigned *red = reinterpret_cast<unsigned *>(wbase + kWarps * kWarpSmem);
    for (int q = threadIdx.x; q < 96; q += kThreads) {
        const int g = q / 32, i = q % 32;
        bh[q] = i < D ? __ldg(A.b_hh + g * D + i) : 0.f;
    }
    for (int q = threadIdx.x; q < kWarps * kWarpSmem; q += kThreads) wbase[q] = 0.f;
    __syncthreads();
    const int warp = threadIdx.x / 32;
    WarpCtx W{bh, wbase + warp * kWarpSmem, wbase + warp * kWarpSmem + 2 * (kPB + kHB)};
    const long long gw = static_cast<long long>(blockIdx.x) * kWarps + warp;
    const long long nw = static_cast<long long>(nblocks) * kWarps;
    const long long n_chunks = static_cast<long long>(B) * S.NC, n_groups = static_cast<long long>(B) * S.NG;

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
        const bool fresh = A.jac_every <= 1 || it % A.jac_every == 0;  // Jacobian taken at this guess
        unsigned dmax = 0u, rmax = 0u;
        for (long long w = gw; w < n_chunks; w += nw)
            chunk_aggregate(S, W, static_cast<int>(w / S.NC), static_cast<int>(w % S.NC), hold,
                            zero_guess, fresh);
        grid_barrier(hdr->barrier, nblocks, status);
        for (long long w = gw; w < n_groups; w += nw)
            group_aggregate(S, W, static_cast<int>(w / S.NG), static_cast<int>(w % S.NG), fresh);
        grid_barrier(hdr->barrier, nblocks, status);
        for (long long w = gw; w < n_groups; w += nw) {
            const int b = static_cast<int>(w / S.NG), g = static_cast<int>(w % S.NG);
            float x[4] = {0.f, 0.f, 0.f, 0.f};
            const size_t gb = static_cast<size_t>(b) * S.NG, cb = static_cast<size_t>(b) * S.NC;
            carry_chain(W, S.PhiG + gb * 1024, S.pG + gb * 32, nullptr, 0, g, x);
            carry_chain(W, S.PhiC + cb * 1024, S.pC + cb * 32, S.carryC + cb * 32, g * S.G,
                        min(S.NC, (g + 1) * S.G), x);
        }
        grid_barrier(hdr->barrier, nblocks, status);
        for (long long w = gw; w < n_chunks; w += nw)
            chunk_sweep(S, W, static_cast<int>(w / S.NC), static_cast<int>(w % S.NC), hold, hnew,
                        zero_guess, fresh, dmax, rmax);
        const unsigned bd = block_max_u32(dmax, red);
        const unsigned br = block_max_u32(rmax, red);
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
        const size_t n4 = static_cast<size_t>(B) * A.T * D / 4;
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

size_t al256m(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

}  // namespace

bool deer_mma_supported(const pararnn_cell &cell) {
    return cell.kind == PARARNN_GRU_DENSE && cell.d <= 32;
}

// Chunk geometry for `nwarps` resident warps: chunks of a multiple of 16
// steps, as many per sequence as the warps allow (at least one), groups of
// about sqrt(chunks) chunks.
static void deer_geom(int B, int T, long long nwarps, int &L, int &NC, int &G, int &NG) {
    long long per_seq = nwarps / B;
    if (per_seq < 1) per_seq = 1;
    long long l = (T + per_seq - 1) / per_seq;
    l = ((l + kBlk - 1) / kBlk) * kBlk;
    L = static_cast<int>(l);
    NC = (T + L - 1) / L;
    G = 1;
    while (static_cast<long long>(G) * G < NC) ++G;
    NG = (NC + G - 1) / G;
}

// PhiC [B][NC][32][32], pC, carryC [B][NC][32]; PhiG [B][NG][32][32], pG [B][NG][32];
// sized for the largest geometry any device can pick (kMaxWarps resident
// warps, and NG <= NC).
size_t deer_mma_ws_bytes(int B, int T) {
    int L, NC, G, NG;
    deer_geom(B, T, kMaxWarps, L, NC, G, NG);
    const size_t nc = static_cast<size_t>(B) * NC, ng = nc;
    return al256m(nc * 1024 * 4) + 2 * al256m(nc * 32 * 4) + al256m(ng * 1024 * 4) +
           al256m(ng * 32 * 4);
}

cudaError_t launch_deer_mma(const DiagArgs &a, void *ws, cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(deer_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    int dev = 0, nsm = 0, per_sm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, deer_mma_kernel, kThreads,
                                                           kSmemBytes)) != cudaSuccess)
        return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    long long grid = static_cast<long long>(per_sm) * nsm;
    if (grid * kWarps > kMaxWarps) grid = kMaxWarps / kWarps;
    MmaArgs S;
    S.a = a;
    deer_geom(a.B, a.T, grid * kWarps, S.L, S.NC, S.G, S.NG);
    const long long need = (static_cast<long long>(a.B) * S.NC + kWarps - 1) / kWarps;
    if (grid > need) grid = need;
    const size_t nc = static_cast<size_t>(a.B) * S.NC, ng = static_cast<size_t>(a.B) * S.NG;
    char *p = static_cast<char *>(ws);
    S.PhiC = reinterpret_cast<float *>(p); p += al256m(nc * 1024 * 4);
    S.pC = reinterpret_cast<float *>(p); p += al256m(nc * 32 * 4);
    S.carryC = reinterpret_cast<float *>(p); p += al256m(nc * 32 * 4);
    S.PhiG = reinterpret_cast<float *>(p); p += al256m(ng * 1024 * 4);
    S.pG = reinterpret_cast<float *>(p);
    MmaArgs args = S;
    void *params[] = {&args};
    return cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(deer_mma_kernel),
                                       dim3(static_cast<unsigned>(grid)), dim3(kThreads), params,
                                       kSmemBytes, s);
}

}  // namespace pararnn

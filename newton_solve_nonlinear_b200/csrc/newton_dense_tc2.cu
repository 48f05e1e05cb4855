// newton_dense_tc2.cu -- quasi-DEER on the dense GRU, software-pipelined over
// tiles, with the recurrent product U h_{t-1} on the 5th-generation tensor
// cores (tcgen05, sm_100a) and the time scan in registers.
//
// Method: "Towards Scalable and Stable Parallelization of Nonlinear RNNs"
// (atlas summary, "Approach": quasi-DEER, the diagonal of the Jacobian, O(TD)
// memory and work per iteration) on the unrolled system of the ParaRNN summary
// ("Core Idea", "Newton's Iteration"), with the affine scan as a single pass
// over time (decoupled look-back between tiles).
//
// One cooperative launch runs every Newton iteration; one CTA per SM walks
// tiles of (sequence b, 128 steps, all D state lanes), chunk-major.  Each
// tile's guess rows h_{t0-1} .. h_{t0+127} arrive by TMA in one of two
// shared-memory slots.  While tile i is finished by all eight warps, the
// asynchronous units already work on the next ones:
//   * tile i+1's rows h_{t-1} are split into a TF32-exact high part and an fp32
//     remainder and written to TMEM as the A operand; one thread then issues
//     tcgen05.mma kind::tf32 (M = 128 steps, N = 3D gate rows, K = 8 per
//     instruction) for lo*U_hi + hi*U_lo + hi*U_hi (the error-compensated
//     3 x TF32 split: G = U h_{t-1} fp32-accurate) into the second of two
//     TMEM accumulators (U_hi / U_lo stay in shared memory for the solve);
//   * tile i+2's rows are in flight by TMA into the slot tile i frees.
// Tile i's epilogue reads its accumulator in the 16x256b fragment layout
// (each thread: 4 steps x 8 lanes, all three gates), evaluates the cell and
// its Jacobian diagonal (a_t, b_t = f_t - a_t h_{t-1}), and scans over time
// without leaving registers: Kogge-Stone over the 8 steps a quad column holds
// (warp shuffles), a 4-group prefix inside the thread, a 4-warp prefix through
// shared memory, and the tile's carry-in by decoupled look-back over earlier
// chunks of the sequence (one thread per lane).  Every state is then final and is stored with the
// convergence maxima max |h^(i+1) - h^(i)| and max |h_t - f_t|.
// Traffic per state and iteration: P (12 B), the guess (4 B, by TMA),
// h^(i+1) (4 B).  A bounded grid barrier ends each iteration.
#include "common.cuh"
#include "lookback.cuh"
#include "solver.cuh"
#include "tc_utils.cuh"

namespace pararnn {
namespace {
using namespace tc;

constexpr int TM = 128;        // steps per tile (MMA M)
constexpr int NTHREADS = 512;  // 16 warps: TMEM lane quarter x lane quarter
constexpr int ROWS = TM + 1;   // staged guess rows t0-1 .. t0+127

template <int D>
struct Tc2Geom {
    static constexpr int N = 3 * D;                  // MMA N: gate rows (r, z, n) x lanes
    static constexpr int HALVES = D / 32;            // 128-byte K atoms per row
    static constexpr int SLOT_HALF = 17 * 1024;      // one K atom of ROWS staged rows (1 KB aligned)
    static constexpr int SLOT_BYTES = HALVES * SLOT_HALF;
    static constexpr int SLOT_TX = HALVES * ROWS * 128;  // bytes one TMA fill delivers
    static constexpr int B_HALF = N * 128;
    static constexpr int B_BYTES = HALVES * B_HALF;
    // TMEM columns: accumulators at 0 and ACC1, A operand hi / lo after them
    static constexpr int ACC1 = (N + 63) / 64 * 64;
    static constexpr int A_HI = 2 * ACC1;
    static constexpr int A_LO = A_HI + 64;
    static constexpr int TMEM_COLS = 512;
    static constexpr int LH = D / 4;   // lanes per warp group in the epilogue
    static constexpr int NJ = LH / 8;  // 8-lane column groups per thread
    static constexpr int KW = D / 4;   // K columns of the A operand each warp writes
    static constexpr int V = 2 * NJ;   // consecutive lanes per epilogue thread
    // The MMA's N order is permuted inside each gate so that the 16x256b
    // fragment hands thread tq of lane group lh the lanes lh LH + V tq .. + V-1:
    // accumulator column c = lh LH + 8 j + 2 tq + x holds lane
    // lh LH + V tq + 2 j + x.
    static __device__ __forceinline__ int lane_of_col(int c) {
        const int lh = c / LH, w = c % LH, j = w >> 3, tq = (w >> 1) & 3, x = w & 1;
        return lh * LH + V * tq + 2 * j + x;
    }
    static constexpr int OFF_BHI = 0;
    static constexpr int OFF_BLO = B_BYTES;
    static constexpr int OFF_SLOT = 2 * B_BYTES;
    static constexpr int OFF_MISC = OFF_SLOT + 2 * SLOT_BYTES;
    // misc floats: b_hh 3D, diag U 3D, warp-quarter totals 2 x 4D, carries D, reduction 32,
    // quasi-ELK segment maps (Moebius 4 + affine 2 per thread) and two carries per lane
    static constexpr int ELK_FLOATS = 6 * NTHREADS + 2 * D;
    static constexpr int MISC_FLOATS = 6 * D + 8 * D + D + 32 + 16 + ELK_FLOATS;  // 16: barriers, TMEM slot, flag
    static constexpr int SMEM_BYTES = OFF_MISC + MISC_FLOATS * 4 + 64 + 1024;
    static_assert(D == 32 || D == 64, "tensor-core cell path takes D = 32 or 64");
    static_assert(A_LO + 64 <= TMEM_COLS, "TMEM columns");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

struct Tc2Args {
    DiagArgs a;
    int n_chunks;
    long long n_tiles;
};

// Swizzled byte offset of element (row, k) inside a K-major 128-byte-swizzle
// tile made of K atoms of `half_bytes` each (rows of 128 bytes).
__device__ __forceinline__ int sw_off(int row, int k, int half_bytes) {
    const int hf = k >> 5, j = (k & 31) >> 2;
    return hf * half_bytes + row * 128 + ((j ^ (row & 7)) << 4) + ((k & 3) << 2);
}

// V consecutive floats (V = 4 or 2; 16- resp. 8-byte aligned).
template <int V>
__device__ __forceinline__ void ldv(const float *p, float (&o)[V]) {
    if constexpr (V == 4) {
        const float4 v = *reinterpret_cast<const float4 *>(p);
        o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
    } else {
        const float2 v = *reinterpret_cast<const float2 *>(p);
        o[0] = v.x; o[1] = v.y;
    }
}
template <int V>
__device__ __forceinline__ void ldgv(const float *p, float (&o)[V]) {
    if constexpr (V == 4) {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(p));
        o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
    } else {
        const float2 v = __ldg(reinterpret_cast<const float2 *>(p));
        o[0] = v.x; o[1] = v.y;
    }
}
template <int V>
__device__ __forceinline__ void stv(float *p, const float (&v)[V]) {
    if constexpr (V == 4)
        __stcg(reinterpret_cast<float4 *>(p), make_float4(v[0], v[1], v[2], v[3]));
    else
        __stcg(reinterpret_cast<float2 *>(p), make_float2(v[0], v[1]));
}

// compose() for two lanes: (a2, b2) := (a2, b2) o (a1, b1).
__device__ __forceinline__ void compose2(u64 &a2, u64 &b2, u64 a1, u64 b1) {
    b2 = fma2(a2, b1, b2);
    a2 = mul2(a2, a1);
}
__device__ __forceinline__ u64 shfl_up2(u64 v, int delta) {
    float a, b;
    upk(v, a, b);
    return pk(__shfl_up_sync(0xffffffffu, a, delta), __shfl_up_sync(0xffffffffu, b, delta));
}

// Affine map composition: apply (a1, b1) first, then (a2, b2).
__device__ __forceinline__ void compose(float &a2, float &b2, float a1, float b1) {
    b2 = fmaf(a2, b1, b2);
    a2 = a2 * a1;
}

// 16 / 8 consecutive TMEM columns of this warp's lane quarter <- registers.
__device__ __forceinline__ void tmem_st(unsigned taddr, const unsigned (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
        "%13,%14,%15,%16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st(unsigned taddr, const unsigned (&v)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
                 "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
                 : "memory");
}

// Time step held by TMEM lane 32 qd + l of the accumulator (and A row): the
// 16x256b fragment hands thread (gid = l & 7) of a warp the lanes gid, gid + 8,
// gid + 16, gid + 24 of its quarter; they hold the four consecutive steps
// 32 qd + 4 gid .. + 3, so each thread scans its steps in registers.
__device__ __forceinline__ int step_of_lane(int qd, int l) {
    return qd * 32 + 4 * (l & 7) + 2 * (l >> 4) + ((l >> 3) & 1);
}

// A operand of the tile staged in `slot`: the row of TMEM lane L is h_{t0+s-1},
// s = step_of_lane (staged row s; h0 replaces it for a sequence's first step).
// Warp (quarter qd, column group kq) writes TMEM lanes 32 qd .. 32 qd + 31 (its
// own lane quarter), K columns kq KW .. kq KW + KW - 1, split into hi (A_HI) and
// lo (A_LO).
template <int D>
__device__ __forceinline__ void write_a(const unsigned char *slot, unsigned tmem, const float *h0row,
                                        bool first_chunk, int warp, int lane) {
    using G = Tc2Geom<D>;
    constexpr int KW = G::KW;
    const int qd = warp & 3, kq = warp >> 2;
    const int r = step_of_lane(qd, lane);
    const int k0 = kq * KW;
    float v[KW];
#pragma unroll
    for (int q = 0; q < KW / 4; ++q) {
        const float4 x = *reinterpret_cast<const float4 *>(slot + sw_off(r, k0 + 4 * q, G::SLOT_HALF));
        v[4 * q] = x.x; v[4 * q + 1] = x.y; v[4 * q + 2] = x.z; v[4 * q + 3] = x.w;
    }
    if (first_chunk && r == 0)
#pragma unroll
        for (int q = 0; q < KW; ++q) v[q] = __ldg(h0row + k0 + q);
    unsigned hi[KW], lo[KW];
#pragma unroll
    for (int q = 0; q < KW; ++q) {
        hi[q] = __float_as_uint(v[q]) & 0xffffe000u;
        lo[q] = __float_as_uint(v[q] - __uint_as_float(hi[q]));
    }
    const unsigned lane_base = static_cast<unsigned>(qd * 32) << 16;
    tmem_st(tmem + lane_base + G::A_HI + k0, hi);
    tmem_st(tmem + lane_base + G::A_LO + k0, lo);
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// One thread: G = lo*U_hi + hi*U_lo + hi*U_hi into accumulator `acc`, then
// commit to `bar`.
template <int D>
__device__ __forceinline__ void issue_mma(unsigned tmem, unsigned acc, unsigned b_hi, unsigned b_lo,
                                          unsigned idesc, unsigned bar) {
    using G = Tc2Geom<D>;
#pragma unroll
    for (int term = 0; term < 3; ++term) {
        const unsigned a_col = term == 0 ? G::A_LO : G::A_HI;
        const unsigned bs = term == 1 ? b_lo : b_hi;
#pragma unroll
        for (int ks = 0; ks < D / 8; ++ks) {
            const int hf = ks >> 2, off = (ks & 3) * 32;
            const unsigned long long db = sw128_desc(bs + hf * G::B_HALF + off);
            const unsigned en = (term > 0 || ks > 0) ? 1u : 0u;
            asm volatile(
                "{\n\t.reg .pred p;\n\t"
                "setp.ne.b32 p, %4, 0;\n\t"
                "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, {%5, %5, %5, %5}, p;\n\t}" ::"r"(
                    tmem + acc),
                "r"(tmem + a_col + ks * 8), "l"(db), "r"(idesc), "r"(en), "r"(0u));
        }
    }
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar));
}

// Pull a tile's input pre-activations (rows t0 .. t0+127 of P, contiguous,
// clamped to the sequence) into L2 ahead of use.
template <int D>
__device__ __forceinline__ void prefetch_p(const float *P, long long tile, int B, int T) {
    const int c = static_cast<int>(static_cast<unsigned>(tile) / static_cast<unsigned>(B));
    const int t0 = c * TM;
    const int n = min(TM, T - t0);
    const float *src = P + (static_cast<size_t>(static_cast<int>(tile) - c * B) * T + t0) * 3 * D;
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(n * 3 * D * 4) : "memory");
}

// ---- quasi-ELK (the damped step as a scalar Kalman filter + RTS smoother per
// lane; "Towards Scalable and Stable Parallelization of Nonlinear RNNs",
// atlas summary "Approach": quasi-ELK) ------------------------------------------
// With the linearisation a_t, b_t at the guess y = h^(i), process noise 1 and
// observation noise 1 / lambda:
//   filter   P-_t = a_t^2 P_{t-1} + 1,  K_t = lambda P-_t / (1 + lambda P-_t),
//            P_t = P-_t / (1 + lambda P-_t)  (so K_t = lambda P_t),
//            m_t = (1 - K_t)(a_t m_{t-1} + b_t) + K_t y_t,  m_0 = h0, P_0 = 0;
//   smoother s_t = G_t s_{t+1} + (m_t - G_t (a_{t+1} m_t + b_{t+1})),
//            G_t = P_t a_{t+1} / P-_{t+1},  s_T = m_T;  h^(i+1) = s.
// The covariance step is the Moebius map [[a^2, 1], [lambda a^2, 1 + lambda]].
// Inside a tile, thread (lane d, segment g) walks SLE consecutive steps; the
// segments of a lane are chained through shared memory and tiles through
// look-back (covariance, mean forward; smoother backward), one thread per lane
// (near-unstable GRU, B = 8, T = 10000, ms per solve: 8 threads per lane 3.62,
// one 3.18).

// predecessors each look-back thread reads per round trip (same workload, with
// 8 threads per lane: 1 -> 3.54 ms per solve, 2 -> 3.77, 3 -> 3.87, 5 -> 4.49, 8 -> 4.90)
constexpr int kElkWin = 1;

struct ElkSmem {
    float *mob;   // [SEGS][D][4] segment Moebius maps, then exclusive prefixes
    float *aff;   // [SEGS][D][2] segment affine maps, then exclusive prefixes
    float *cP;    // [D] covariance entering the tile
    float *cM;    // [D] mean entering the tile (smoother: state after the tile)
};

// Forward scans of one tile: a_t, b_t of the tile are in A.elk_a / elk_b
// (written by this CTA), the guess rows in `slot`.  Writes m_t and P_t.
template <int D>
__device__ void elk_forward_scans(const DiagArgs &A, const ElkSmem &E, const unsigned char *slot,
                                  long long tile, int chunk, int b, int t0, long long row0,
                                  unsigned epoch, unsigned long long *desc_cov,
                                  unsigned long long *desc_mean, unsigned *status) {
    using G = Tc2Geom<D>;
    constexpr int SEGS = NTHREADS / D, SLE = TM / SEGS;
    const int T = A.T, B = A.B;
    const float lam = A.lambda;
    const int tid = threadIdx.x, d = tid % D, g = tid / D, s0 = g * SLE;
    // (i) covariance maps of the thread's steps
    float ak[SLE];
    Mob M{1.f, 0.f, 0.f, 1.f};
#pragma unroll
    for (int i = 0; i < SLE; ++i)  // all of the segment's a_t in flight at once
        ak[i] = t0 + s0 + i < T ? __ldcg(A.elk_a + (static_cast<size_t>(row0) + s0 + i) * D + d) : 1.f;
#pragma unroll
    for (int i = 0; i < SLE; ++i) {
        if (t0 + s0 + i < T) {
            const float a2 = ak[i] * ak[i];
            M = mob_mul(Mob{a2, 1.f, lam * a2, 1.f + lam}, M);
        }
    }
    {
        float *mm = E.mob + (g * D + d) * 4;
        mm[0] = M.m0; mm[1] = M.m1; mm[2] = M.m2; mm[3] = M.m3;
    }
    __syncthreads();
    if (tid < D) {  // covariance entering the tile: one thread per lane
        const int ld = tid, lq = 0;
        Mob Ex{1.f, 0.f, 0.f, 1.f};
        for (int q = 0; q < SEGS; ++q) {
            const float *qm = E.mob + (q * D + ld) * 4;
            Ex = mob_mul(Mob{qm[0], qm[1], qm[2], qm[3]}, Ex);
        }
        const float pin = coop_lookback_mob<1, kElkWin>(desc_cov, tile, B, D, ld, lq, epoch, Ex, chunk,
                                                        0.f, status);
        if (lq == 0) E.cP[ld] = pin;
    }
    __syncthreads();
    // (ii) covariances, gains and the mean's affine maps
    float Pk[SLE], bk[SLE];
#pragma unroll
    for (int i = 0; i < SLE; ++i)  // all of the segment's b_t in flight at once
        bk[i] = t0 + s0 + i < T ? __ldcg(A.elk_b + (static_cast<size_t>(row0) + s0 + i) * D + d) : 0.f;
    {
        Mob X{1.f, 0.f, 0.f, 1.f};  // this segment's exclusive prefix
        for (int q = 0; q < g; ++q) {
            const float *qm = E.mob + (q * D + d) * 4;
            X = mob_mul(Mob{qm[0], qm[1], qm[2], qm[3]}, X);
        }
        float P = mob_apply(X, E.cP[d]);
        float SA = 1.f, SB = 0.f;
#pragma unroll
        for (int i = 0; i < SLE; ++i) {
            const int s = s0 + i;
            float alpha = 1.f, beta = 0.f;
            if (t0 + s < T) {
                const float Pm = fmaf(ak[i] * ak[i], P, 1.f);
                P = __fdividef(Pm, fmaf(lam, Pm, 1.f));
                const float K = lam * P, omk = 1.f - K;
                const float y = *reinterpret_cast<const float *>(slot + sw_off(s + 1, d, G::SLOT_HALF));
                alpha = omk * ak[i];
                beta = fmaf(omk, bk[i], K * y);
            }
            Pk[i] = P;
            SB = fmaf(alpha, SB, beta);
            SA = alpha * SA;
        }
        float *fa = E.aff + (g * D + d) * 2;
        fa[0] = SA;
        fa[1] = SB;
    }
    __syncthreads();
    if (tid < D) {  // mean entering the tile: one thread per lane
        const int ld = tid, lq = 0;
        float EA = 1.f, EB = 0.f;
        for (int q = 0; q < SEGS; ++q) {
            const float *qa = E.aff + (q * D + ld) * 2;
            EB = fmaf(qa[0], EB, qa[1]);
            EA = qa[0] * EA;
        }
        const float c0 = chunk == 0 ? __ldg(A.h0 + static_cast<size_t>(b) * D + ld) : 0.f;
        const float min_ = coop_lookback<1, kElkWin>(desc_mean, tile, B, D, ld, lq, epoch, EA, EB, chunk,
                                                     c0, status);
        if (lq == 0) E.cM[ld] = min_;
    }
    __syncthreads();
    // (iii) filtered means and covariances of the thread's steps
    {
        float m = E.cM[d];
        for (int q = 0; q < g; ++q) {
            const float *qa = E.aff + (q * D + d) * 2;
            m = fmaf(qa[0], m, qa[1]);
        }
#pragma unroll
        for (int i = 0; i < SLE; ++i) {
            const int s = s0 + i;
            if (t0 + s < T) {  // the gain-weighted map again: K_t = lambda P_t
                const size_t o = (static_cast<size_t>(row0) + s) * D + d;
                const float K = lam * Pk[i], omk = 1.f - K;
                const float y = *reinterpret_cast<const float *>(slot + sw_off(s + 1, d, G::SLOT_HALF));
                m = fmaf(omk * ak[i], m, fmaf(omk, bk[i], K * y));
                __stcg(A.elk_m + o, m);
                __stcg(A.elk_p + o, Pk[i]);
            }
        }
    }
}

// Smoother over one tile (tiles visited in reverse chunk order): h^(i+1) and
// max |h^(i+1) - h^(i)|.
template <int D>
__device__ void elk_backward_tile(const DiagArgs &A, const ElkSmem &E, long long tile, int chunk, int b,
                                  int n_chunks, unsigned epoch, unsigned long long *desc_bwd,
                                  const float *hold, float *hnew, unsigned &dmax, unsigned *status) {
    constexpr int SEGS = NTHREADS / D, SLE = TM / SEGS;
    const int T = A.T, B = A.B;
    const int tid = threadIdx.x, d = tid % D, g = tid / D, s0 = g * SLE;
    const int t0 = chunk * TM;
    const long long row0 = static_cast<long long>(b) * T + t0;
    float Gk[SLE], Ck[SLE], yk[SLE];
    // loads in batches of 4 steps, the next batch in flight while one is used
    float mv[2][4], pv[2][4], av[2][4], bv[2][4];
    auto load_batch = [&](int i0, int sl) {
#pragma unroll
        for (int i = i0; i < i0 + 4; ++i) {
            const int t = t0 + s0 + i;
            const size_t o = (static_cast<size_t>(row0) + s0 + i) * D + d;
            mv[sl][i - i0] = t < T ? __ldcg(A.elk_m + o) : 0.f;
            yk[i] = t < T ? __ldcg(hold + o) : 0.f;
            pv[sl][i - i0] = t + 1 < T ? __ldcg(A.elk_p + o) : 0.f;
            av[sl][i - i0] = t + 1 < T ? __ldcg(A.elk_a + o + D) : 0.f;
            bv[sl][i - i0] = t + 1 < T ? __ldcg(A.elk_b + o + D) : 0.f;
        }
    };
    load_batch(0, 0);
#pragma unroll
    for (int i0 = 0; i0 < SLE; i0 += 4) {
        const int sl = (i0 / 4) & 1;
        if (i0 + 4 < SLE) load_batch(i0 + 4, sl ^ 1);
#pragma unroll
        for (int i = i0; i < i0 + 4; ++i) {
            const int t = t0 + s0 + i;
            float Gv = 1.f, Cv = 0.f;
            if (t == T - 1) {
                Gv = 0.f;
                Cv = mv[sl][i - i0];
            } else if (t < T) {
                const float P = pv[sl][i - i0], an = av[sl][i - i0], m = mv[sl][i - i0];
                Gv = __fdividef(P * an, fmaf(an * an, P, 1.f));
                Cv = m - Gv * fmaf(an, m, bv[sl][i - i0]);
            }
            Gk[i] = Gv;
            Ck[i] = Cv;
        }
    }
    float cG = 1.f, cC = 0.f;  // s at the segment's first step from s after its last
#pragma unroll
    for (int i = SLE - 1; i >= 0; --i) {
        cC = fmaf(Gk[i], cC, Ck[i]);
        cG = Gk[i] * cG;
    }
    {
        float *fa = E.aff + (g * D + d) * 2;
        fa[0] = cG;
        fa[1] = cC;
    }
    __syncthreads();
    if (tid < D) {  // state after the tile (from the next chunk): one thread per lane
        const int ld = tid, lq = 0;
        float EG = 1.f, EC = 0.f;
        for (int q = SEGS - 1; q >= 0; --q) {
            const float *qa = E.aff + (q * D + ld) * 2;
            EC = fmaf(qa[0], EC, qa[1]);
            EG = qa[0] * EG;
        }
        const float sin_ = coop_lookback<1, kElkWin>(desc_bwd, tile, -static_cast<long long>(B), D, ld, lq,
                                                     epoch, EG, EC, n_chunks - 1 - chunk, 0.f, status);
        if (lq == 0) E.cM[ld] = sin_;
    }
    __syncthreads();
    float sv = E.cM[d];
    for (int q = SEGS - 1; q > g; --q) {
        const float *qa = E.aff + (q * D + d) * 2;
        sv = fmaf(qa[0], sv, qa[1]);
    }
#pragma unroll
    for (int i = SLE - 1; i >= 0; --i) {
        sv = fmaf(Gk[i], sv, Ck[i]);
        if (t0 + s0 + i < T) {
            __stcg(hnew + (static_cast<size_t>(row0) + s0 + i) * D + d, sv);
            dmax = max(dmax, abs_bits(sv - yk[i]));
        }
    }
    __syncthreads();  // the segment maps are rewritten by the next tile
}

template <int D>
__device__ __forceinline__ void issue_fill(const CUtensorMap *map, unsigned char *slot, long long row0,
                                           unsigned bar) {
    using G = Tc2Geom<D>;
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // after the slot's last reads
    mbar_expect_tx(bar, G::SLOT_TX);
#pragma unroll
    for (int hf = 0; hf < G::HALVES; ++hf)
        tma_load_2d(smem_u32(slot + hf * G::SLOT_HALF), map, hf * 32, static_cast<int>(row0 - 1), bar);
}

template <int D, bool ELK>
__global__ void __launch_bounds__(NTHREADS, 1)
quasi_tc2_kernel(const __grid_constant__ CUtensorMap map_h0, const __grid_constant__ CUtensorMap map_h1,
                 Tc2Args S) {
    using G = Tc2Geom<D>;
    constexpr int LH = G::LH, NJ = G::NJ;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    unsigned char *bhi = smem + G::OFF_BHI, *blo = smem + G::OFF_BLO;
    unsigned char *slots = smem + G::OFF_SLOT;
    float *misc = reinterpret_cast<float *>(smem + G::OFF_MISC);
    float *c_bh = misc;                   // [3D] b_hh; the r and z parts times -log2(e)
    float *c_ud = c_bh + 3 * D;           // [3D] diagonal of U_g
    float *wt_a = c_ud + 3 * D;           // [4][D] affine total of each warp quarter's 32 steps
    float *wt_b = wt_a + 4 * D;
    float *carry = wt_b + 4 * D;          // [D] tile carry-in
    unsigned *red = reinterpret_cast<unsigned *>(carry + D);  // [32]
    unsigned long long *bars = reinterpret_cast<unsigned long long *>(red + 32);  // fill[2], mma[2]
    unsigned *tmem_slot = reinterpret_cast<unsigned *>(bars + 4);
    volatile int *cta_err = reinterpret_cast<volatile int *>(tmem_slot + 1);
    ElkSmem es;
    es.mob = reinterpret_cast<float *>(tmem_slot + 4);
    es.aff = es.mob + 4 * NTHREADS;
    es.cP = es.aff + 2 * NTHREADS;
    es.cM = es.cP + D;

    const DiagArgs &A = S.a;
    const int T = A.T, B = A.B;
    WsHeader *hdr = A.hdr;
    unsigned *status = &hdr->status;
    const unsigned nblocks = gridDim.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qd = warp & 3, lh = warp >> 2, gid = lane >> 2, tq = lane & 3;
    constexpr int V = G::V;
    const int dbase = lh * LH + V * tq;  // this thread's lanes in the epilogue and scan

    // ---- once per solve: U split into TF32 hi / lo, constants, barriers, TMEM
    for (int i = tid; i < G::N * D; i += NTHREADS) {
        const int n = i / D, k = i % D;
        const int g = n / D, dl = G::lane_of_col(n % D);
        const float v = __ldg(A.w_hh + (static_cast<size_t>(g) * D + dl) * D + k);
        const float hi = __uint_as_float(__float_as_uint(v) & 0xffffe000u);
        const int off = sw_off(n, k, G::B_HALF);
        *reinterpret_cast<float *>(bhi + off) = hi;
        *reinterpret_cast<float *>(blo + off) = v - hi;
    }
    for (int i = tid; i < 3 * D; i += NTHREADS) {
        c_bh[i] = __ldg(A.b_hh + i) * (i < 2 * D ? -kLog2eF : 1.f);
        const int g = i / D, d = i % D;
        c_ud[i] = __ldg(A.w_hh + (static_cast<size_t>(g) * D + d) * D + d);
    }
    if (tid == 0) {
        for (int q = 0; q < 4; ++q) mbar_init(smem_u32(&bars[q]), 1);
        *cta_err = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(G::TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;");
    const unsigned tmem = *tmem_slot;
    constexpr unsigned idesc = make_idesc(2u, TM, G::N);  // kind::tf32, M=128, N=3D
    const unsigned b_hi = smem_u32(bhi), b_lo = smem_u32(blo);
    // quasi-ELK look-back descriptors: covariance [tile][D][4], mean and smoother [tile][D][2]
    unsigned long long *desc_cov = A.desc;
    unsigned long long *desc_mean = A.desc + static_cast<size_t>(S.n_tiles) * D * 4;
    unsigned long long *desc_bwd = A.desc + static_cast<size_t>(S.n_tiles) * D * 6;

    // bit q: mbarrier parity of fill slot q / accumulator q; an operation in flight
    unsigned fill_par = 0u, mma_par = 0u, fill_pending = 0u, mma_pending = 0u;
    const long long my_n =
        blockIdx.x < S.n_tiles ? (S.n_tiles - blockIdx.x + nblocks - 1) / nblocks : 0;
    auto tile_of = [&](long long k) { return static_cast<long long>(blockIdx.x) + k * nblocks; };
    auto row0_of = [&](long long tile) {
        const int c = static_cast<int>(static_cast<unsigned>(tile) / static_cast<unsigned>(B));
        return static_cast<long long>(static_cast<int>(tile) - c * B) * T + static_cast<long long>(c) * TM;
    };

    int iters = 0, final_status = PARARNN_NOT_CONVERGED;
    unsigned last_delta = 0u, last_resid = 0u;
    for (int it = 0; it < A.max_iters; ++it) {
        if (blockIdx.x == 0 && tid == 0) {
            hdr->delta_bits[(it + 1) % 3] = 0u;
            hdr->resid_bits[(it + 1) % 3] = 0u;
        }
        float *hnew = A.hbuf[(it + 1) & 1];
        const CUtensorMap *map = (it & 1) ? &map_h1 : &map_h0;
        const unsigned epoch = static_cast<unsigned>(it + 1);
        unsigned dmax = 0u, rmax = 0u;

        // prologue: fill slots 0 and 1, operand + products of the first tile
        if (tid == 0) {
            for (int q = 0; q < 2 && q < my_n; ++q) {
                prefetch_p<D>(A.P, tile_of(q), B, T);
                issue_fill<D>(map, slots + q * G::SLOT_BYTES, row0_of(tile_of(q)), smem_u32(&bars[q]));
            }
        }
        fill_pending = my_n > 1 ? 3u : (my_n > 0 ? 1u : 0u);
        if (my_n > 0) {
            if (!mbar_wait(smem_u32(&bars[0]), fill_par & 1u, cta_err)) *cta_err = 1;
            fill_par ^= 1u;
            fill_pending &= ~1u;
            const long long t0t = tile_of(0);
            write_a<D>(slots, tmem, A.h0 + static_cast<size_t>(static_cast<int>(t0t) % B) * D,
                       static_cast<int>(t0t) < B, warp, lane);
            asm volatile("tcgen05.fence::before_thread_sync;");
            __syncthreads();
            if (tid == 0) {
                asm volatile("tcgen05.fence::after_thread_sync;");
                issue_mma<D>(tmem, 0u, b_hi, b_lo, idesc, smem_u32(&bars[2]));
            }
            mma_pending |= 1u;
        }

        for (long long k = 0; k < my_n; ++k) {
            const long long tile = tile_of(k);
            // tile < 2^31 (B*T < 2^31 is required): 32-bit arithmetic
            const int chunk = static_cast<int>(static_cast<unsigned>(tile) / static_cast<unsigned>(B));
            const int b = static_cast<int>(tile) - chunk * B;
            const int t0 = chunk * TM;
            const long long row0 = static_cast<long long>(b) * T + t0;
            const int cur = static_cast<int>(k & 1);
            const unsigned char *slot = slots + cur * G::SLOT_BYTES;

            if (tid == 0 && k + 2 < my_n) prefetch_p<D>(A.P, tile_of(k + 2), B, T);
            // 1. this tile's input pre-activations: thread (gid, tq) of warp (qd, lh)
            // owns steps r = 32 qd + 4 gid + 2 rh + e (TMEM lanes 32 qd + 16 rh + 8 e
            // + gid) and lanes dbase .. dbase + V - 1
            float pv[2][2][3][V];
#pragma unroll
            for (int rh = 0; rh < 2; ++rh)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int r = qd * 32 + 4 * gid + 2 * rh + e;
                    const float *prow = A.P + (static_cast<size_t>(row0) + r) * 3 * D + dbase;
#pragma unroll
                    for (int g = 0; g < 3; ++g) {
                        if (t0 + r < T)
                            ldgv<V>(prow + g * D, pv[rh][e][g]);
                        else
#pragma unroll
                            for (int v = 0; v < V; ++v) pv[rh][e][g][v] = 0.f;
                    }
                }

            // 2. the products of tile k are done: refill A with tile k+1 and start its products
            if (!mbar_wait(smem_u32(&bars[2 + cur]), (mma_par >> cur) & 1u, cta_err)) *cta_err = 1;
            mma_par ^= 1u << cur;
            mma_pending &= ~(1u << cur);
            if (k + 1 < my_n) {
                const int nxt = cur ^ 1;
                if (!mbar_wait(smem_u32(&bars[nxt]), (fill_par >> nxt) & 1u, cta_err)) *cta_err = 1;
                fill_par ^= 1u << nxt;
                fill_pending &= ~(1u << nxt);
                const long long tn = tile_of(k + 1);
                write_a<D>(slots + nxt * G::SLOT_BYTES, tmem, A.h0 + static_cast<size_t>(static_cast<int>(tn) % B) * D,
                           static_cast<int>(tn) < B, warp, lane);
                asm volatile("tcgen05.fence::before_thread_sync;");
            }
            __syncthreads();
            if (*cta_err != 0) break;  // uniform: read after the barrier
            asm volatile("tcgen05.fence::after_thread_sync;");
            if (k + 1 < my_n) {
                if (tid == 0)
                    issue_mma<D>(tmem, (cur ^ 1) ? G::ACC1 : 0u, b_hi, b_lo, idesc,
                                 smem_u32(&bars[2 + (cur ^ 1)]));
                mma_pending |= 1u << (cur ^ 1);
            }

            // 3. epilogue: the cell at the guess, a_t and b_t per (step, lane);
            // element (rh, e, j, x) is step r = 32 qd + 4 gid + 2 rh + e, lane
            // dbase + 2 j + x
            float av[2][2][NJ][2], bv[2][2][NJ][2];
            const unsigned acc = cur ? G::ACC1 : 0u;
#pragma unroll
            for (int rh = 0; rh < 2; ++rh) {
                const unsigned trow = tmem + acc + (static_cast<unsigned>(qd * 32 + rh * 16) << 16);
                // staged rows r, r + 1, r + 2 of the steps r, r + 1: h_{t-1} and h_t
                float hp[2][V], y[2][V];
                {
                    const int r = qd * 32 + 4 * gid + 2 * rh;
                    ldv<V>(reinterpret_cast<const float *>(slot + sw_off(r, dbase, G::SLOT_HALF)), hp[0]);
                    if (t0 == 0 && r == 0) ldgv<V>(A.h0 + static_cast<size_t>(b) * D + dbase, hp[0]);
                    ldv<V>(reinterpret_cast<const float *>(slot + sw_off(r + 1, dbase, G::SLOT_HALF)), y[0]);
                    ldv<V>(reinterpret_cast<const float *>(slot + sw_off(r + 2, dbase, G::SLOT_HALF)), y[1]);
#pragma unroll
                    for (int v = 0; v < V; ++v) hp[1][v] = y[0][v];
                }
#pragma unroll
                for (int j = 0; j < NJ; ++j) {
                    // the lane pair's recurrent biases and U diagonals, read once
                    const int d2 = dbase + 2 * j;
                    const float2 bhr = *reinterpret_cast<const float2 *>(c_bh + d2);
                    const float2 bhz = *reinterpret_cast<const float2 *>(c_bh + D + d2);
                    const float2 bhn = *reinterpret_cast<const float2 *>(c_bh + 2 * D + d2);
                    const float2 udr = *reinterpret_cast<const float2 *>(c_ud + d2);
                    const float2 udz = *reinterpret_cast<const float2 *>(c_ud + D + d2);
                    const float2 udn = *reinterpret_cast<const float2 *>(c_ud + 2 * D + d2);
                    unsigned gv[3][4];
#pragma unroll
                    for (int g = 0; g < 3; ++g)
                        asm volatile("tcgen05.ld.sync.aligned.16x256b.x1.b32 {%0,%1,%2,%3}, [%4];"
                                     : "=r"(gv[g][0]), "=r"(gv[g][1]), "=r"(gv[g][2]), "=r"(gv[g][3])
                                     : "r"(trow + g * D + lh * LH + 8 * j));
                    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int r = qd * 32 + 4 * gid + 2 * rh + e;
                        const bool ok = t0 + r < T;
                        float a0 = 1.f, a1 = 1.f, b0 = 0.f, b1 = 0.f;
                        if (ok) {  // lanes 2j, 2j + 1 together
                            const int v = 2 * j;
                            u64 f2, a2, b2;
                            gru_cell_diag_x2(pk(pv[rh][e][0][v], pv[rh][e][0][v + 1]),
                                             pk(pv[rh][e][1][v], pv[rh][e][1][v + 1]),
                                             pk(pv[rh][e][2][v], pv[rh][e][2][v + 1]),
                                             pk(__uint_as_float(gv[0][2 * e]), __uint_as_float(gv[0][2 * e + 1])),
                                             pk(__uint_as_float(gv[1][2 * e]), __uint_as_float(gv[1][2 * e + 1])),
                                             pk(__uint_as_float(gv[2][2 * e]), __uint_as_float(gv[2][2 * e + 1])),
                                             pk(bhr.x, bhr.y), pk(bhz.x, bhz.y), pk(bhn.x, bhn.y),
                                             pk(udr.x, udr.y), pk(udz.x, udz.y), pk(udn.x, udn.y),
                                             pk(hp[e][v], hp[e][v + 1]), f2, a2, b2);
                            float r0, r1;
                            upk(sub2(pk(y[e][v], y[e][v + 1]), f2), r0, r1);
                            rmax = max(rmax, max(abs_bits(r0), abs_bits(r1)));
                            upk(a2, a0, a1);
                            upk(b2, b0, b1);
                        }
                        av[rh][e][j][0] = a0;
                        av[rh][e][j][1] = a1;
                        bv[rh][e][j][0] = b0;
                        bv[rh][e][j][1] = b1;
                    }
                }
            }
            asm volatile("tcgen05.fence::before_thread_sync;");

            if constexpr (ELK) {
                // 4'. quasi-ELK: a_t, b_t to memory (the smoother reads them too),
                // then the filter's covariance and mean scans
#pragma unroll
                for (int rh = 0; rh < 2; ++rh)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int r = qd * 32 + 4 * gid + 2 * rh + e;
                        if (t0 + r < T) {
                            float va[V], vb[V];
#pragma unroll
                            for (int j = 0; j < NJ; ++j)
#pragma unroll
                                for (int x = 0; x < 2; ++x) {
                                    va[2 * j + x] = av[rh][e][j][x];
                                    vb[2 * j + x] = bv[rh][e][j][x];
                                }
                            const size_t o = (static_cast<size_t>(row0) + r) * D + dbase;
                            stv<V>(A.elk_a + o, va);
                            stv<V>(A.elk_b + o, vb);
                        }
                    }
                __syncthreads();
                elk_forward_scans<D>(A, es, slot, tile, chunk, b, t0, row0, epoch, desc_cov, desc_mean,
                                     status);
            } else {
            // 4. scan over the tile's steps, per lane d, in registers.  Thread gid of
            // a quad column holds the consecutive steps 32 qd + 4 gid + k, k = 2 rh + e.
#pragma unroll
            for (int j = 0; j < NJ; ++j) {  // lanes 2j, 2j + 1 as fp32x2 pairs
                u64 pa_[2][2], pb_[2][2];
#pragma unroll
                for (int rh = 0; rh < 2; ++rh)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        pa_[rh][e] = pk(av[rh][e][j][0], av[rh][e][j][1]);
                        pb_[rh][e] = pk(bv[rh][e][j][0], bv[rh][e][j][1]);
                    }
                // 4a. inclusive prefix over the thread's four steps
                compose2(pa_[0][1], pb_[0][1], pa_[0][0], pb_[0][0]);
                compose2(pa_[1][0], pb_[1][0], pa_[0][1], pb_[0][1]);
                compose2(pa_[1][1], pb_[1][1], pa_[1][0], pb_[1][0]);
                // 4b. Kogge-Stone over the eight threads' totals (gid = 0 .. 7)
                u64 ta = pa_[1][1], tb = pb_[1][1];
#pragma unroll
                for (int o = 1; o < 8; o <<= 1) {
                    const u64 qa = shfl_up2(ta, 4 * o), qb = shfl_up2(tb, 4 * o);
                    if (gid >= o) compose2(ta, tb, qa, qb);
                }
                // the thread's exclusive prefix (gid - 1's inclusive) folded into its
                // steps: every (a, b) then maps the quarter's carry-in to the step
                const u64 ea = shfl_up2(ta, 4), eb = shfl_up2(tb, 4);
#pragma unroll
                for (int rh = 0; rh < 2; ++rh)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        if (gid > 0) compose2(pa_[rh][e], pb_[rh][e], ea, eb);
                        upk(pa_[rh][e], av[rh][e][j][0], av[rh][e][j][1]);
                        upk(pb_[rh][e], bv[rh][e][j][0], bv[rh][e][j][1]);
                    }
                if (gid == 7) {  // the warp quarter's total
                    const int d = dbase + 2 * j;
                    float a0, a1, b0, b1;
                    upk(ta, a0, a1);
                    upk(tb, b0, b1);
                    *reinterpret_cast<float2 *>(wt_a + qd * D + d) = make_float2(a0, a1);
                    *reinterpret_cast<float2 *>(wt_b + qd * D + d) = make_float2(b0, b1);
                }
            }
            __syncthreads();
            // 4c. the tile's carry-in per lane by look-back over earlier chunks: one
            // thread per lane (threads 0 .. D-1; the rest go on to the barrier).
            // Threads per lane, measured on the untrained workload (ms per solve):
            // 8 (all 512 threads) 7.19, 4 6.74, 2 6.68, 1 6.65 -- the wider groups'
            // shuffles and ballots cost more issue slots than their reads save
            if (tid < D) {
                constexpr int GL = 1;
                const int d = tid, q = 0;
                float EA = wt_a[d], EB = wt_b[d];
#pragma unroll
                for (int qq = 1; qq < 4; ++qq) {
                    float qa = wt_a[qq * D + d], qb = wt_b[qq * D + d];
                    compose(qa, qb, EA, EB);
                    EA = qa;
                    EB = qb;
                }
                const float c0 = chunk == 0 ? __ldg(A.h0 + static_cast<size_t>(b) * D + d) : 0.f;
                const float hin = coop_lookback<GL, 1, false>(A.desc, tile, B, D, d, q, epoch, EA, EB, chunk, c0, status,
                                                    nullptr, publishes(A, tile, epoch));
                if (q == 0) carry[d] = hin;
            }
            __syncthreads();
            // 4d. states: carry through the earlier warp quarters, then the thread's prefixes
            {
                float hin[V];
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    float h = carry[dbase + v];
                    for (int q = 0; q < qd; ++q) h = fmaf(wt_a[q * D + dbase + v], h, wt_b[q * D + dbase + v]);
                    hin[v] = h;
                }
#pragma unroll
                for (int rh = 0; rh < 2; ++rh)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int r = qd * 32 + 4 * gid + 2 * rh + e;
                        if (t0 + r < T) {
                            float y[V], h[V];
                            ldv<V>(reinterpret_cast<const float *>(slot + sw_off(r + 1, dbase, G::SLOT_HALF)), y);
#pragma unroll
                            for (int j = 0; j < NJ; ++j) {
                                const int v = 2 * j;
                                const u64 h2 = fma2(pk(av[rh][e][j][0], av[rh][e][j][1]), pk(hin[v], hin[v + 1]),
                                                    pk(bv[rh][e][j][0], bv[rh][e][j][1]));
                                float d0, d1;
                                upk(sub2(h2, pk(y[v], y[v + 1])), d0, d1);
                                dmax = max(dmax, max(abs_bits(d0), abs_bits(d1)));
                                upk(h2, h[v], h[v + 1]);
                            }
                            stv<V>(hnew + (static_cast<size_t>(row0) + r) * D + dbase, h);
                        }
                    }
            }

            }  // quasi scan

            // 5. slot `cur` and accumulator `cur` are free: refill the slot with tile k+2
            asm volatile("tcgen05.fence::before_thread_sync;");
            __syncthreads();
            if (k + 2 < my_n) {
                if (tid == 0)
                    issue_fill<D>(map, slots + cur * G::SLOT_BYTES, row0_of(tile_of(k + 2)),
                                  smem_u32(&bars[cur]));
                fill_pending |= 1u << cur;
            }
        }
        if constexpr (ELK) {
            // the smoother runs backward over time once every filter value is written
            grid_barrier(hdr->barrier, nblocks, status);
            const float *hold = A.hbuf[it & 1];
            for (long long k = 0; k < my_n; ++k) {
                // leave on an error or a timeout seen by any thread (uniform decision)
                if (__syncthreads_or(*cta_err != 0 || timed_out(status))) break;
                const long long tr = S.n_tiles - 1 - tile_of(k);
                const int c = static_cast<int>(static_cast<unsigned>(tr) / static_cast<unsigned>(B));
                elk_backward_tile<D>(A, es, tr, c, static_cast<int>(tr) - c * B, S.n_chunks, epoch,
                                     desc_bwd, hold, hnew, dmax, status);
            }
        }
        const unsigned bd = block_max_u32(dmax, red);
        const unsigned br = block_max_u32(rmax, red);
        if (tid == 0) {
            atomicMax(&hdr->delta_bits[it % 3], bd);
            atomicMax(&hdr->resid_bits[it % 3], br);
            if (*cta_err) flag_timeout(status);
            // P of the next iteration's first two tiles into L2 while the grid meets
            for (int q = 0; q < 2 && q < my_n; ++q) prefetch_p<D>(A.P, tile_of(q), B, T);
        }
        grid_barrier(hdr->barrier, nblocks, status);
        last_delta = ld_acquire_u32(&hdr->delta_bits[it % 3]);
        last_resid = ld_acquire_u32(&hdr->resid_bits[it % 3]);
        record_trace(A, it, last_delta, last_resid);
        iters = it + 1;
        // a timeout another CTA raises may land between two threads' reads: decide once per CTA
        if (__syncthreads_or(*cta_err || timed_out(status))) { final_status = PARARNN_TIMEOUT; break; }
        if (last_delta >= 0x7f800000u) { final_status = PARARNN_DIVERGED; break; }
        if (__uint_as_float(last_delta) <= A.tol) { final_status = PARARNN_OK; break; }
    }
    if ((iters & 1) == 0 && iters > 0) {
        const size_t n4 = static_cast<size_t>(A.B) * A.T * A.D / 4;
        const float4 *src = reinterpret_cast<const float4 *>(A.hbuf[0]);
        float4 *dst = reinterpret_cast<float4 *>(A.hbuf[1]);
        for (size_t q = static_cast<size_t>(blockIdx.x) * NTHREADS + tid; q < n4;
             q += static_cast<size_t>(nblocks) * NTHREADS)
            dst[q] = __ldcg(src + q);
    }
    if (blockIdx.x == 0 && tid == 0) {
        pararnn_info info;
        info.iters = iters;
        info.status = final_status;
        info.delta = __uint_as_float(last_delta);
        info.residual = __uint_as_float(last_resid);
        *A.info_out = info;
        hdr->info = info;
    }
    if (tid == 0) {  // copies and products still in flight after a failed wait finish first
        for (int q = 0; q < 2; ++q) {
            if ((fill_pending >> q) & 1u) mbar_drain(smem_u32(&bars[q]), (fill_par >> q) & 1u);
            if ((mma_pending >> q) & 1u) mbar_drain(smem_u32(&bars[2 + q]), (mma_par >> q) & 1u);
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;");
    __syncthreads();
    if (warp == 1) {
        asm volatile("tcgen05.fence::after_thread_sync;");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(G::TMEM_COLS));
    }
}

template <int D, bool ELK>
cudaError_t launch_tc2(const DiagArgs &a, cudaStream_t s) {
    using G = Tc2Geom<D>;
    Tc2Args S;
    S.a = a;
    S.n_chunks = (a.T + TM - 1) / TM;
    S.n_tiles = static_cast<long long>(a.B) * S.n_chunks;
    CUtensorMap m0, m1;
    const long long rows = static_cast<long long>(a.B) * a.T;
    if (!make_map(&m0, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.hbuf[0], rows, D, 32, ROWS) ||
        !make_map(&m1, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.hbuf[1], rows, D, 32, ROWS))
        return cudaErrorInvalidValue;
    auto kern = quasi_tc2_kernel<D, ELK>;
    // every CTA takes all 512 TMEM columns, so at most one may reside on an SM:
    // the shared-memory request alone guarantees it
    const int smem = G::SMEM_BYTES > 120 * 1024 ? G::SMEM_BYTES : 120 * 1024;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int dev = 0, nsm = 0, per_sm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, NTHREADS, smem)) != cudaSuccess)
        return e;
    if (per_sm != 1) return cudaErrorInvalidConfiguration;
    long long grid = nsm;
    if (grid > S.n_tiles) grid = S.n_tiles;
    void *params[] = {&m0, &m1, &S};
    return cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(kern),
                                       dim3(static_cast<unsigned>(grid)), dim3(NTHREADS), params, smem, s);
}

}  // namespace

// Look-back descriptors of the tensor-core path: tiles of 128 steps x D lanes, two words each.
size_t quasi_tc_desc_bytes(int B, int T, int D) {
    const long long tiles = static_cast<long long>(B) * ((T + TM - 1) / TM);
    return static_cast<size_t>(tiles) * D * 2 * 8;
}

bool quasi_tc_supported(const pararnn_cell &cell, int B, int T) {
    if (cell.kind != PARARNN_GRU_DENSE || (cell.d != 32 && cell.d != 64)) return false;
    if (static_cast<long long>(B) * T >= (1ll << 31) - 1) return false;
    return encode_fn() != nullptr;
}

cudaError_t launch_quasi_tc2(const DiagArgs &a, bool elk, cudaStream_t s) {
    if (elk) return a.D == 32 ? launch_tc2<32, true>(a, s) : launch_tc2<64, true>(a, s);
    return a.D == 32 ? launch_tc2<32, false>(a, s) : launch_tc2<64, false>(a, s);
}

}  // namespace pararnn

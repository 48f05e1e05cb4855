// adjoint_diag.cu -- the backward pass through an evaluated sequence of the
// diagonal-recurrence GRU: gradients of a loss with respect to the input
// pre-activations, the initial state and the recurrent parameters.
//
// Method: the pages train the evaluated RNN with the diagonal Jacobian in the
// backward pass ("Towards Scalable and Stable Parallelization of Nonlinear
// RNNs", atlas summary, table "Measured effects reported in the paper"); for
// the diagonal-recurrence cell (the "adapted" GRU of the ParaRNN talk page,
// "Federico Danieli", Abstract) that Jacobian is exact.  The chain rule on the
// unrolled system h_t = f(h_{t-1}, p_t) gives, backwards in time,
//     lam_t = g_t + a_{t+1} lam_{t+1},   lam_T = g_T,
// a_t = df_t/dh_{t-1} (diagonal), g_t = dL/dh_t the upstream gradient: a
// reverse affine recurrence, solved in one pass with decoupled look-back over
// the later chunks.  Then per state (lane i of step t, previous state hp):
//     dL/dp_r = lam (1-z)(1-n^2) g r (1-r),  dL/dp_z = lam (hp - n) z (1-z),
//     dL/dp_n = lam (1-z)(1-n^2),            dL/dh_0 = a_1 lam_1,
//     dL/du_r = sum lam (1-z)(1-n^2) g r(1-r) hp,  dL/du_z = sum lam (hp-n) z(1-z) hp,
//     dL/du_n = sum lam (1-z)(1-n^2) r hp,  dL/db_hh likewise without hp.
//
// One cooperative launch: CTAs of 512 threads walk tiles of (sequence, 64
// lanes, 32 steps) from the last chunk to the first.  Thread (lane d, segment
// s) evaluates the cell at its 4 steps and the next one (for a_{t+1}), folds
// its steps' maps in reverse, the eight segments of a lane chain through shared
// memory, the tile takes lam at its end from a decoupled look-back over later
// chunks (one thread per lane), and the sweep writes dL/dP and the per-tile partial sums of
// the parameter gradients.  After a grid barrier every warp reduces some of
// those partials in a fixed order.
// Traffic per state: P (12 B), h (4 B), dL/dh (4 B) read; dL/dP (12 B) written.
#include "common.cuh"
#include "lookback.cuh"
#include "solver.cuh"

namespace pararnn {
namespace {

constexpr int ATS = 32;            // steps per tile
constexpr int ADL = 64;            // lanes per tile
constexpr int ANT = 512;           // threads: lane x 8 segments
constexpr int ASEGS = ANT / ADL;   // 8 segments
constexpr int ASL = ATS / ASEGS;   // 4 steps per thread

struct AdjArgs {
    const float *P, *h0, *h, *dh, *u, *b_hh;  // u: [3D] recurrent vectors (r, z, n)
    // dense cell (quasi backward): w_hh [3D, D] (the Jacobian's diagonal is read
    // from it), G [B, T, 3D] = U h_{t-1} + b_hh, and grow [B, T, 3D] out: the
    // gradient w.r.t. the recurrent pre-activations (dP with the n gate times r)
    const float *w_hh, *G;
    float *grow;
    float *dP, *dh0, *du, *db_hh;
    WsHeader *hdr;
    unsigned long long *desc;  // [n_tiles][ADL][2] look-back words
    float *part;               // [n_tiles][6][ADL] per-tile partial sums
    int B, T, D, ndg, ngroups, n_chunks;
    long long n_tiles;
};

// One step of the diagonal cell at (hp, p): the partials of f with respect to
// the three pre-activations, r, and a = df/dh_{t-1}.
__device__ __forceinline__ void adj_cell(float pr, float pz, float pn, float hp, float ur, float uz, float un,
                                         float br, float bz, float bn, float &fr, float &fz, float &fn,
                                         float &r, float &a) {
    r = sigmoidf_(pr + ur * hp + br);
    const float z = sigmoidf_(pz + uz * hp + bz);
    const float g = un * hp + bn;
    const float n = tanhf_(pn + r * g);
    fn = (1.f - z) * (1.f - n * n);
    fr = fn * g * r * (1.f - r);
    fz = (hp - n) * z * (1.f - z);
    a = z + fz * uz + fn * r * un + fr * ur;
}

// The same for the dense cell at recurrent pre-activations q = U h_{t-1} + b_hh
// (computed beforehand), with the Jacobian's diagonal entries ud of U.
__device__ __forceinline__ void adj_cell_q(float pr, float pz, float pn, float qr, float qz, float qn, float hp,
                                           float udr, float udz, float udn, float &fr, float &fz, float &fn,
                                           float &r, float &a) {
    r = sigmoidf_(pr + qr);
    const float z = sigmoidf_(pz + qz);
    const float n = tanhf_(pn + r * qn);
    fn = (1.f - z) * (1.f - n * n);
    fr = fn * qn * r * (1.f - r);
    fz = (hp - n) * z * (1.f - z);
    a = z + fz * udz + fn * r * udn + fr * udr;
}

__device__ __forceinline__ void prefetch_l2(const float *p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }

template <bool DENSE>
__global__ void __launch_bounds__(ANT, 2) adjoint_diag_kernel(AdjArgs S) {
    static_assert(ASEGS == 8, "the per-tile partial sums below add eight segments");
    __shared__ float seg_a[ASEGS][ADL], seg_b[ASEGS][ADL];
    __shared__ float carry[ADL];
    __shared__ float red6[ASEGS][6][ADL];
    const int T = S.T, D = S.D;
    unsigned *status = &S.hdr->status;
    const int tid = threadIdx.x;
    const int d = tid & (ADL - 1), seg = tid / ADL;  // sweep role
    // look-back threads per lane (diagonal backward pass, B = 8, T = 4096, D = 2048, ms:
    // 8 -> 0.890, 1 -> 0.776)
    constexpr int ALB = 1;
    const int ld = tid / ALB, lq = tid % ALB;        // look-back role (tid < ADL * ALB)
    const unsigned nblocks = gridDim.x;
    const unsigned epoch = 1u;

    for (long long v = blockIdx.x; v < S.n_tiles; v += nblocks) {
        // processing order: last chunk first; v - ngroups is the same lanes one chunk later
        const unsigned v32 = static_cast<unsigned>(v), ng = static_cast<unsigned>(S.ngroups);
        const int cidx = static_cast<int>(v32 / ng);
        const int grp = static_cast<int>(v32 - static_cast<unsigned>(cidx) * ng);
        const int chunk = S.n_chunks - 1 - cidx;
        const int b = grp / S.ndg, dg = grp - (grp / S.ndg) * S.ndg;
        const int t0 = chunk * ATS;
        const int lane = dg * ADL + d;
        const bool lane_ok = lane < D;
        const size_t row0 = static_cast<size_t>(b) * T;

        float ur = 0.f, uz = 0.f, un = 0.f, br = 0.f, bz = 0.f, bn = 0.f;
        if (lane_ok) {
            if constexpr (DENSE) {  // the Jacobian's diagonal: U_g[lane][lane]
                const size_t dd = static_cast<size_t>(lane) * D + lane;
                ur = __ldg(S.w_hh + dd), uz = __ldg(S.w_hh + static_cast<size_t>(D) * D + dd);
                un = __ldg(S.w_hh + 2 * static_cast<size_t>(D) * D + dd);
            } else {
                ur = __ldg(S.u + lane), uz = __ldg(S.u + D + lane), un = __ldg(S.u + 2 * D + lane);
                br = __ldg(S.b_hh + lane), bz = __ldg(S.b_hh + D + lane), bn = __ldg(S.b_hh + 2 * D + lane);
            }
        }
        // 1. the cell at the thread's 8 steps and the next one
        float fr[ASL], fz[ASL], fn[ASL], rr[ASL], hp[ASL], gg[ASL], al[ASL];
        float a_first = 0.f;
        {
            float pr[ASL + 1], pz[ASL + 1], pn[ASL + 1], hv[ASL + 1];
            float qr[ASL + 1], qz[ASL + 1], qn[ASL + 1];  // dense: U h_{t-1} + b_hh
#pragma unroll
            for (int i = 0; i <= ASL; ++i) {  // all loads in flight together
                const int t = t0 + seg * ASL + i;
                const bool ok = lane_ok && t < T;
                const size_t o = (row0 + t) * 3 * D + lane;
                pr[i] = ok ? __ldcs(S.P + o) : 0.f;
                pz[i] = ok ? __ldcs(S.P + o + D) : 0.f;
                pn[i] = ok ? __ldcs(S.P + o + 2 * D) : 0.f;
                hv[i] = ok ? (t == 0 ? __ldg(S.h0 + static_cast<size_t>(b) * D + lane)
                                     : __ldcs(S.h + (row0 + t - 1) * D + lane))
                           : 0.f;
                if (i < ASL) gg[i] = ok ? __ldcs(S.dh + (row0 + t) * D + lane) : 0.f;
                if constexpr (DENSE) {
                    qr[i] = ok ? __ldcs(S.G + o) : 0.f;
                    qz[i] = ok ? __ldcs(S.G + o + D) : 0.f;
                    qn[i] = ok ? __ldcs(S.G + o + 2 * D) : 0.f;
                }
            }
            // dense cell: the CTA's next tile (its rows are whole, contiguous state
            // rows) into L2 while this one is computed; on the diagonal cell's
            // 64-lane slices of wide rows this measured slower, so it is not done there
            const long long vn = v + nblocks;
            if (DENSE && vn < S.n_tiles) {
                const unsigned vn32 = static_cast<unsigned>(vn);
                const int cn = static_cast<int>(vn32 / ng);
                const int gn = static_cast<int>(vn32 - static_cast<unsigned>(cn) * ng);
                const int tn0 = (S.n_chunks - 1 - cn) * ATS;
                const int bn = gn / S.ndg, lanen = (gn - bn * S.ndg) * ADL + d;
                const size_t rown = static_cast<size_t>(bn) * T;
                if (lanen < D)
#pragma unroll
                    for (int i = 0; i < ASL; ++i) {
                        const int t = tn0 + seg * ASL + i;
                        if (t >= T) break;
                        const size_t o = (rown + t) * 3 * D + lanen;
                        prefetch_l2(S.P + o);
                        prefetch_l2(S.P + o + D);
                        prefetch_l2(S.P + o + 2 * D);
                        if constexpr (DENSE) {
                            prefetch_l2(S.G + o);
                            prefetch_l2(S.G + o + D);
                            prefetch_l2(S.G + o + 2 * D);
                        }
                        prefetch_l2(S.dh + (rown + t) * D + lanen);
                        if (t > 0) prefetch_l2(S.h + (rown + t - 1) * D + lanen);
                    }
            }
#pragma unroll
            for (int i = 0; i <= ASL; ++i) {
                const int t = t0 + seg * ASL + i;
                float f_r, f_z, f_n, r_, a_;
                if constexpr (DENSE)
                    adj_cell_q(pr[i], pz[i], pn[i], qr[i], qz[i], qn[i], hv[i], ur, uz, un, f_r, f_z, f_n, r_, a_);
                else
                    adj_cell(pr[i], pz[i], pn[i], hv[i], ur, uz, un, br, bz, bn, f_r, f_z, f_n, r_, a_);
                if (i < ASL) {
                    fr[i] = f_r, fz[i] = f_z, fn[i] = f_n, rr[i] = r_, hp[i] = hv[i];
                    if (i == 0) a_first = a_;
                }
                // a_{t} of step i is the coefficient of lam_i in lam_{i-1}
                if (i > 0) al[i - 1] = (lane_ok && t < T) ? a_ : 0.f;
            }
        }
        // 2. this segment's reverse map: lam_i = A_i lam_after + B_i
        float Ai[ASL], Bi[ASL];
        {
            float A = 1.f, Bv = 0.f;
#pragma unroll
            for (int i = ASL - 1; i >= 0; --i) {
                Bv = fmaf(al[i], Bv, gg[i]);
                A = al[i] * A;
                Ai[i] = A;
                Bi[i] = Bv;
            }
        }
        LookbackWindow<1> lbw{};
        if (tid < ADL * ALB) lbw = coop_lookback_prefetch<ALB>(S.desc, v, S.ngroups, ADL, ld, lq, cidx);
        seg_a[seg][d] = Ai[0];
        seg_b[seg][d] = Bi[0];
        __syncthreads();
        // 3. lam at the tile's end (step t0 + 32) by look-back over later chunks
        if (tid < ADL * ALB) {
            float TA = 1.f, TB = 0.f;  // the tile: lam_{t0} = TA lam_{t0+32} + TB
#pragma unroll
            for (int q = ASEGS - 1; q >= 0; --q) {
                TB = fmaf(seg_a[q][ld], TB, seg_b[q][ld]);
                TA = seg_a[q][ld] * TA;
            }
            const float lin =
                coop_lookback<ALB, 1, true>(S.desc, v, S.ngroups, ADL, ld, lq, epoch, TA, TB, cidx, 0.f, status, &lbw);
            if (lq == 0) carry[ld] = lin;
        }
        __syncthreads();
        // 4. sweep: lam after this segment, then its steps; dL/dP and partial sums
        float s_r = 0.f, s_z = 0.f, s_n = 0.f, q_r = 0.f, q_z = 0.f, q_n = 0.f;
        {
            float lam_after = carry[d];
            for (int q = ASEGS - 1; q > seg; --q) lam_after = fmaf(seg_a[q][d], lam_after, seg_b[q][d]);
#pragma unroll
            for (int i = 0; i < ASL; ++i) {
                const int t = t0 + seg * ASL + i;
                if (lane_ok && t < T) {
                    const float lam = fmaf(Ai[i], lam_after, Bi[i]);
                    const float gr = fr[i] * lam, gz = fz[i] * lam, gn = fn[i] * lam, gnr = gn * rr[i];
                    const size_t o = (row0 + t) * 3 * D + lane;
                    __stcs(S.dP + o, gr);
                    __stcs(S.dP + o + D, gz);
                    __stcs(S.dP + o + 2 * D, gn);
                    if constexpr (DENSE) {  // for dW_hh = sum grow (outer) h_{t-1}, a GEMM after this pass
                        __stcs(S.grow + o, gr);
                        __stcs(S.grow + o + D, gz);
                        __stcs(S.grow + o + 2 * D, gnr);
                    }
                    q_r += gr, q_z += gz, q_n += gnr;
                    s_r = fmaf(gr, hp[i], s_r), s_z = fmaf(gz, hp[i], s_z), s_n = fmaf(gnr, hp[i], s_n);
                    if (t == 0) S.dh0[static_cast<size_t>(b) * D + lane] = a_first * lam;
                }
            }
        }
        red6[seg][0][d] = s_r, red6[seg][1][d] = s_z, red6[seg][2][d] = s_n;
        red6[seg][3][d] = q_r, red6[seg][4][d] = q_z, red6[seg][5][d] = q_n;
        __syncthreads();
        for (int i = tid; i < 6 * ADL; i += ANT) {  // per-tile partials, segments summed in order
            const int k = i / ADL, dd = i % ADL;
            S.part[(static_cast<size_t>(v) * 6 + k) * ADL + dd] =
                ((red6[0][k][dd] + red6[1][k][dd]) + (red6[2][k][dd] + red6[3][k][dd])) +
                ((red6[4][k][dd] + red6[5][k][dd]) + (red6[6][k][dd] + red6[7][k][dd]));
        }
        __syncthreads();  // shared arrays are rewritten by the next tile
    }

    // 5. parameter gradients: each warp sums one (quantity, lane) over the tiles
    // of that lane group, always in the same order
    grid_barrier(S.hdr->barrier, nblocks, status);
    const int warp = tid >> 5, wl = tid & 31;
    const long long nwarps = static_cast<long long>(nblocks) * (ANT / 32);
    const int per_group = S.n_chunks * S.B;  // tiles of one lane group
    for (long long o = static_cast<long long>(blockIdx.x) * (ANT / 32) + warp; o < 6ll * D; o += nwarps) {
        const int k = static_cast<int>(o / D), lane = static_cast<int>(o % D);
        const int dg = lane / ADL, dd = lane % ADL;
        float acc = 0.f;
        for (int j = wl; j < per_group; j += 32) {
            const int cidx = j / S.B, bb = j - cidx * S.B;
            const long long v = static_cast<long long>(cidx) * S.ngroups + bb * S.ndg + dg;
            acc += __ldcg(S.part + (static_cast<size_t>(v) * 6 + k) * ADL + dd);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (wl == 0 && (k >= 3 || !DENSE)) {  // dense: dW_hh comes from the GEMM after this pass
            float *dst = k < 3 ? S.du : S.db_hh;
            dst[(k % 3) * D + lane] = acc;
        }
    }
}

}  // namespace

size_t adjoint_diag_desc_bytes(int B, int T, int D) {
    const long long tiles = static_cast<long long>(B) * ((D + ADL - 1) / ADL) * ((T + ATS - 1) / ATS);
    return static_cast<size_t>(tiles) * ADL * 2 * 8;
}
size_t adjoint_diag_part_bytes(int B, int T, int D) {
    const long long tiles = static_cast<long long>(B) * ((D + ADL - 1) / ADL) * ((T + ATS - 1) / ATS);
    return static_cast<size_t>(tiles) * 6 * ADL * 4;
}

namespace {

// dW_hh [N, K] = sum over the M rows m of grow[m, :N] (outer) hp[m, :K]
// (grow [M, 3D], hp [M, D]): each CTA sums a chunk of OSR rows into its own
// partial (no atomics), a second pass adds the partials in chunk order, so the
// result does not depend on scheduling.  Rows are staged 32 at a time into
// shared memory, zero-padded to 192 x 64 columns (cp.async, double-buffered);
// each thread keeps a 6 x 8 block of the outputs in registers (n = 6 nb + i,
// k = 8 kb + j) and adds 48 products per row from five vector loads, as
// packed fp32x2 FMAs.
constexpr int OSR = 512;   // rows per chunk
constexpr int OSM = 32;    // rows per shared-memory stage
constexpr int OST = 256;   // threads: 32 row blocks x 8 column blocks
constexpr int ONI = 6, OKJ = 8;
constexpr int ONP = 32 * ONI, OKP = 8 * OKJ;  // padded widths: N <= 192, K <= 64
constexpr int OSTAGE = OSM * (ONP + OKP);     // floats per stage
constexpr size_t OS_SMEM = 2 * OSTAGE * sizeof(float);

// 4-byte asynchronous copy to shared memory; zero-fills when !ok (the source
// is then not read).
__device__ __forceinline__ void cp4z(float *dst, const float *src, bool ok) {
    const unsigned d = static_cast<unsigned>(__cvta_generic_to_shared(dst));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(d), "l"(src), "r"(ok ? 4 : 0) : "memory");
}

__device__ __forceinline__ void os_stage(float *st, const float *grow, const float *hp, long long mb, long long M,
                                         int N, int K) {
    for (int i = threadIdx.x; i < OSM * ONP; i += OST) {
        const int r = i / ONP, n = i - r * ONP;
        const bool ok = mb + r < M && n < N;
        cp4z(st + i, ok ? grow + (mb + r) * N + n : grow, ok);
    }
    for (int i = threadIdx.x; i < OSM * OKP; i += OST) {
        const int r = i / OKP, k = i - r * OKP;
        const bool ok = mb + r < M && k < K;
        cp4z(st + OSM * ONP + i, ok ? hp + (mb + r) * K + k : hp, ok);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
}

__global__ void __launch_bounds__(OST) outer_sum_partial_kernel(const float *grow, const float *hp, long long M,
                                                                int N, int K, float *part) {
    extern __shared__ float4 os_raw[];
    float *buf = reinterpret_cast<float *>(os_raw);
    const long long m0 = static_cast<long long>(blockIdx.x) * OSR;
    const long long m1 = m0 + OSR < M ? m0 + OSR : M;
    const int nst = static_cast<int>((m1 - m0 + OSM - 1) / OSM);
    const int kb = threadIdx.x % OKJ, nb = threadIdx.x / OKJ;
    u64 acc[ONI][OKJ / 2];
#pragma unroll
    for (int i = 0; i < ONI; ++i)
#pragma unroll
        for (int j = 0; j < OKJ / 2; ++j) acc[i][j] = 0ull;
    os_stage(buf, grow, hp, m0, m1, N, K);
    for (int st = 0; st < nst; ++st) {
        if (st + 1 < nst) {
            os_stage(buf + ((st + 1) & 1) * OSTAGE, grow, hp, m0 + (st + 1) * OSM, m1, N, K);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();
        const float *sg = buf + (st & 1) * OSTAGE, *sh = sg + OSM * ONP;
#pragma unroll 4
        for (int r = 0; r < OSM; ++r) {
            const float2 g0 = *reinterpret_cast<const float2 *>(sg + r * ONP + ONI * nb);
            const float2 g1 = *reinterpret_cast<const float2 *>(sg + r * ONP + ONI * nb + 2);
            const float2 g2 = *reinterpret_cast<const float2 *>(sg + r * ONP + ONI * nb + 4);
            const float4 h0 = *reinterpret_cast<const float4 *>(sh + r * OKP + OKJ * kb);
            const float4 h1 = *reinterpret_cast<const float4 *>(sh + r * OKP + OKJ * kb + 4);
            const float gv[ONI] = {g0.x, g0.y, g1.x, g1.y, g2.x, g2.y};
            const u64 hv[OKJ / 2] = {pk(h0.x, h0.y), pk(h0.z, h0.w), pk(h1.x, h1.y), pk(h1.z, h1.w)};
#pragma unroll
            for (int i = 0; i < ONI; ++i) {
                const u64 g = splat(gv[i]);
#pragma unroll
                for (int j = 0; j < OKJ / 2; ++j) acc[i][j] = fma2(g, hv[j], acc[i][j]);
            }
        }
        __syncthreads();  // the buffer is refilled next
    }
    float *dst = part + static_cast<size_t>(blockIdx.x) * N * K;
#pragma unroll
    for (int i = 0; i < ONI; ++i) {
        const int n = ONI * nb + i;
#pragma unroll
        for (int j = 0; j < OKJ / 2; ++j) {
            float a, b;
            upk(acc[i][j], a, b);
            const int k = OKJ * kb + 2 * j;
            if (n < N && k < K) dst[n * K + k] = a;
            if (n < N && k + 1 < K) dst[n * K + k + 1] = b;
        }
    }
}
// out[o] = sum over chunks of part[c][o]: a CTA owns 32 consecutive outputs
// (coalesced rows of the partials); its 8 warps take the chunks c = w, w + 8,
// ... and the 8 warp sums are added in warp order, so the order is fixed.
constexpr int ORW = 8;
__global__ void __launch_bounds__(32 * ORW) outer_sum_reduce_kernel(const float *part, int nchunks, int NK,
                                                                    float *out) {
    __shared__ float red[ORW][32];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int o = blockIdx.x * 32 + lane;
    float a = 0.f;
    if (o < NK)
        for (int c = w; c < nchunks; c += ORW) a += __ldcs(part + static_cast<size_t>(c) * NK + o);
    red[w][lane] = a;
    __syncthreads();
    if (w == 0 && o < NK) {
        float t = red[0][lane];
#pragma unroll
        for (int q = 1; q < ORW; ++q) t += red[q][lane];
        out[o] = t;
    }
}

}  // namespace

size_t adjoint_outer_part_bytes(long long M, int N, int K) {
    return static_cast<size_t>((M + OSR - 1) / OSR) * N * K * 4;
}

cudaError_t launch_outer_sum(const float *grow, const float *hp, long long M, int N, int K, float *part, float *out,
                             cudaStream_t s) {
    if (N > ONP || K > OKP) return cudaErrorInvalidValue;
    const long long nchunks = (M + OSR - 1) / OSR;
    cudaError_t e = cudaFuncSetAttribute(outer_sum_partial_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(OS_SMEM));
    if (e != cudaSuccess) return e;
    outer_sum_partial_kernel<<<static_cast<unsigned>(nchunks), OST, OS_SMEM, s>>>(grow, hp, M, N, K, part);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int NK = N * K;
    outer_sum_reduce_kernel<<<(NK + 31) / 32, 32 * ORW, 0, s>>>(part, static_cast<int>(nchunks), NK, out);
    return cudaGetLastError();
}

// out[o] = sum over r < rows of in[r][o] (o < n), added in row order.
cudaError_t launch_sum_rows(const float *in, int rows, int n, float *out, cudaStream_t s) {
    outer_sum_reduce_kernel<<<(n + 31) / 32, 32 * ORW, 0, s>>>(in, rows, n, out);
    return cudaGetLastError();
}

cudaError_t launch_adjoint_diag(const float *P, const float *h0, const float *h, const float *dh, const float *u,
                                const float *b_hh, float *dP, float *dh0, float *du, float *db_hh, int B, int T,
                                int D, void *hdr, void *desc, void *part, cudaStream_t s, const float *w_hh_dense,
                                const float *G, float *grow) {
    AdjArgs S;
    S.P = P, S.h0 = h0, S.h = h, S.dh = dh, S.u = u, S.b_hh = b_hh;
    S.w_hh = w_hh_dense, S.G = G, S.grow = grow;
    S.dP = dP, S.dh0 = dh0, S.du = du, S.db_hh = db_hh;
    S.hdr = static_cast<WsHeader *>(hdr);
    S.desc = static_cast<unsigned long long *>(desc);
    S.part = static_cast<float *>(part);
    S.B = B, S.T = T, S.D = D;
    S.ndg = (D + ADL - 1) / ADL;
    S.ngroups = B * S.ndg;
    S.n_chunks = (T + ATS - 1) / ATS;
    S.n_tiles = static_cast<long long>(S.ngroups) * S.n_chunks;
    const bool dense = G != nullptr;
    const void *kern = dense ? reinterpret_cast<const void *>(adjoint_diag_kernel<true>)
                             : reinterpret_cast<const void *>(adjoint_diag_kernel<false>);
    int dev = 0, nsm = 0, per_sm = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, ANT, 0);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    long long grid = static_cast<long long>(nsm) * per_sm;
    void *params[] = {&S};
    return cudaLaunchCooperativeKernel(kern, dim3(static_cast<unsigned>(grid)), dim3(ANT), params, 0, s);
}

}  // namespace pararnn

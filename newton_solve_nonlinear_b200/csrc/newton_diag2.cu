// newton_diag2.cu -- Newton on the diagonal-recurrence GRU (exact Newton: the
// Jacobian of u_g * h is diagonal, so the quasi-DEER step is the DEER step),
// as a software-pipelined streaming kernel.
//
// Method: the unrolled system of the ParaRNN summary ("Core Idea", "Newton's
// Iteration") with the diagonal Jacobian of "Towards Scalable and Stable
// Parallelization of Nonlinear RNNs" (atlas summary, "Approach"); the affine
// recurrence h_t = a_t h_{t-1} + b_t is solved in one pass over time with
// decoupled look-back between tiles.
//
// One cooperative launch runs every Newton iteration; CTAs of 256 threads (two
// or more per SM, so that one CTA's look-back wait overlaps another's cells)
// walk tiles of (sequence b, 64 lanes, 32 steps), chunk-major.  A tile's input
// pre-activations (3 gates) and guess rows h_{t0-1} .. h_{t0+31} arrive by TMA
// in one of two shared-memory slots while the previous tile is processed.
// Thread (lane d, segment s) owns 8 consecutive steps of one lane: it
// evaluates the cell and a_t, b_t (b_t = f_t - a_t h_{t-1}), composes its 8
// maps, the 4 segments of a lane are chained through shared memory, the
// tile's carry-in per lane comes from a decoupled look-back (one thread per
// lane), and every state is swept and stored with the convergence maxima
// max |h^(i+1) - h^(i)| and max |h_t - f_t|.
// Traffic per state and iteration: P (12 B), the guess (4 B), h^(i+1) (4 B).
#include "common.cuh"
#include "lookback.cuh"
#include "solver.cuh"
#include "tc_utils.cuh"

namespace pararnn {
namespace {
using namespace tc;

constexpr int TS = 32;          // steps per tile
constexpr int DL = 64;          // lanes per tile
constexpr int NT = 256;         // threads: lane x 4 segments
constexpr int SEGS = NT / DL;   // 4 segments of 8 steps
constexpr int SL = TS / SEGS;   // steps per thread
constexpr int HALF = 32;        // lanes per 128-byte TMA box row
constexpr int P_BOX = TS * 128;                // one (gate, half) box of P: 4 KB
constexpr int H_BOX = ((TS + 1) * 128 + 1023) / 1024 * 1024;  // one half of TS + 1 guess rows, 1 KB aligned
constexpr int SLOT = 6 * P_BOX + 2 * H_BOX;    // 34 KB
constexpr int SLOT_TX = 6 * P_BOX + 2 * (TS + 1) * 128;
constexpr int OFF_MISC = 2 * SLOT;
// misc floats: segment maps 2 x SEGS x DL, carries DL, reduction 32
constexpr int MISC_FLOATS = 2 * SEGS * DL + DL + 32;
constexpr int SMEM_BYTES = OFF_MISC + MISC_FLOATS * 4 + 64 + 1024;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");

struct Diag2Args {
    DiagArgs a;
    int ndg;            // lane groups per sequence (D / 64)
    int ngroups;        // B * ndg: tiles per chunk
    long long n_tiles;
};

__device__ __forceinline__ void issue_fill(const CUtensorMap *mp, const CUtensorMap *mh,
                                           unsigned char *slot, int D, long long row0, int lane0,
                                           unsigned bar) {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // after the slot's last reads
    mbar_expect_tx(bar, SLOT_TX);
#pragma unroll
    for (int g = 0; g < 3; ++g)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
            tma_load_2d(smem_u32(slot + (2 * g + hf) * P_BOX), mp, g * D + lane0 + hf * HALF,
                        static_cast<int>(row0), bar);
#pragma unroll
    for (int hf = 0; hf < 2; ++hf)
        tma_load_2d(smem_u32(slot + 6 * P_BOX + hf * H_BOX), mh, lane0 + hf * HALF,
                    static_cast<int>(row0 - 1), bar);
}

// Tile indices stay below 2^31 (n_tiles <= B*T*D / 2048): 32-bit arithmetic.
__device__ __forceinline__ void tile_pos(const Diag2Args &S, long long tile, int T, int &chunk, int &b,
                                         int &dg, long long &row0) {
    const unsigned t32 = static_cast<unsigned>(tile), ng = static_cast<unsigned>(S.ngroups);
    chunk = static_cast<int>(t32 / ng);
    const unsigned grp = t32 - static_cast<unsigned>(chunk) * ng;
    b = static_cast<int>(grp / static_cast<unsigned>(S.ndg));
    dg = static_cast<int>(grp) - b * S.ndg;
    row0 = static_cast<long long>(b) * T + static_cast<long long>(chunk) * TS;
}

__global__ void __launch_bounds__(NT, 3)
diag2_kernel(const __grid_constant__ CUtensorMap map_p, const __grid_constant__ CUtensorMap map_h0,
             const __grid_constant__ CUtensorMap map_h1, Diag2Args S) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    float *misc = reinterpret_cast<float *>(smem + OFF_MISC);
    float *seg_a = misc;                   // [SEGS][DL] map of each 8-step segment
    float *seg_b = seg_a + SEGS * DL;
    float *carry = seg_b + SEGS * DL;      // [DL] tile carry-in
    unsigned *red = reinterpret_cast<unsigned *>(carry + DL);  // [32]
    unsigned long long *bars = reinterpret_cast<unsigned long long *>(red + 32);  // fill[2]
    volatile int *cta_err = reinterpret_cast<volatile int *>(bars + 2);

    const DiagArgs &A = S.a;
    const int T = A.T, D = A.D;
    WsHeader *hdr = A.hdr;
    unsigned *status = &hdr->status;
    const unsigned nblocks = gridDim.x;
    const int tid = threadIdx.x;
    const int d = tid & (DL - 1), seg = tid / DL;  // sweep role: lane, segment
    // look-back threads per lane (diagonal workload, us per iteration: 4 -> 362, 2 -> 339, 1 -> 325)
    constexpr int LBG = 1;
    const int ld = tid / LBG, lq = tid % LBG;       // look-back role: lane, rank (tid < DL * LBG)
    const int jq = (d & 31) >> 2;                   // 16-byte chunk of lane d in a 128-byte row

    if (tid == 0) {
        mbar_init(smem_u32(&bars[0]), 1);
        mbar_init(smem_u32(&bars[1]), 1);
        *cta_err = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    unsigned fill_par = 0u, fill_pending = 0u;
    const long long my_n = blockIdx.x < S.n_tiles ? (S.n_tiles - blockIdx.x + nblocks - 1) / nblocks : 0;
    int iters = 0, final_status = PARARNN_NOT_CONVERGED;
    unsigned last_delta = 0u, last_resid = 0u;
    for (int it = 0; it < A.max_iters; ++it) {
        if (blockIdx.x == 0 && tid == 0) {
            hdr->delta_bits[(it + 1) % 3] = 0u;
            hdr->resid_bits[(it + 1) % 3] = 0u;
        }
        float *hnew = A.hbuf[(it + 1) & 1];
        const CUtensorMap *mh = (it & 1) ? &map_h1 : &map_h0;
        const unsigned epoch = static_cast<unsigned>(it + 1);
        unsigned dmax = 0u, rmax = 0u;

        if (tid == 0) {
            for (int q = 0; q < 2 && q < my_n; ++q) {
                int chunk, b, dg;
                long long row0;
                tile_pos(S, blockIdx.x + static_cast<long long>(q) * nblocks, T, chunk, b, dg, row0);
                issue_fill(&map_p, mh, smem + q * SLOT, D, row0, dg * DL, smem_u32(&bars[q]));
            }
        }
        fill_pending = my_n > 1 ? 3u : (my_n > 0 ? 1u : 0u);

        for (long long k = 0; k < my_n; ++k) {
            const long long tile = blockIdx.x + k * nblocks;
            int chunk, b, dg;
            long long row0;
            tile_pos(S, tile, T, chunk, b, dg, row0);
            const int t0 = chunk * TS, lane0 = dg * DL;
            const int cur = static_cast<int>(k & 1);
            const unsigned char *slot = smem + cur * SLOT;
            const unsigned char *Hs = slot + 6 * P_BOX;
            if (!mbar_wait(smem_u32(&bars[cur]), (fill_par >> cur) & 1u, cta_err)) *cta_err = 1;
            fill_par ^= 1u << cur;
            fill_pending &= ~(1u << cur);

            // 1. cells of this thread's 8 steps
            const int di = lane0 + d;
            const float ur = __ldg(A.w_hh + di), uz = __ldg(A.w_hh + D + di), un = __ldg(A.w_hh + 2 * D + di);
            // r and z biases times -log2(e), as gru_cell_diag_x2 takes them
            const float br = -kLog2eF * __ldg(A.b_hh + di), bz = -kLog2eF * __ldg(A.b_hh + D + di);
            const float bn = __ldg(A.b_hh + 2 * D + di);
            // a thread's rows start at a multiple of 8, so the swizzle of row
            // seg*SL + i is the constant i: lane offsets are hoisted out of the loop
            const unsigned char *Pt = slot + (d >> 5) * P_BOX + seg * SL * 128 + (d & 3) * 4;
            const unsigned char *Ht = Hs + (d >> 5) * H_BOX + seg * SL * 128 + (d & 3) * 4;
            const bool full = t0 + TS <= T;
            float av[SL], bv[SL];
            float EA = 1.f, EB = 0.f;
            float hp = *reinterpret_cast<const float *>(Ht + (jq << 4));
            if (t0 == 0 && seg == 0) hp = __ldg(A.h0 + static_cast<size_t>(b) * D + di);
            const u64 ur2 = splat(ur), uz2 = splat(uz), un2 = splat(un);
#pragma unroll
            for (int i = 0; i < SL; i += 2) {  // steps i, i + 1 together on fp32x2
                const int o0 = i * 128 + ((jq ^ i) << 4), o1 = (i + 1) * 128 + ((jq ^ (i + 1)) << 4);
                const int oy = (i + 2) * 128 + ((jq ^ ((i + 2) & 7)) << 4);
                const float y0 = *reinterpret_cast<const float *>(Ht + o1);  // h_{t}, then h_{t-1} of i + 1
                const float y1 = *reinterpret_cast<const float *>(Ht + oy);
                const u64 h2 = pk(hp, y0);
                u64 f2, a2, b2;
                gru_cell_diag_x2(pk(*reinterpret_cast<const float *>(Pt + 0 * P_BOX + o0),
                                    *reinterpret_cast<const float *>(Pt + 0 * P_BOX + o1)),
                                 pk(*reinterpret_cast<const float *>(Pt + 2 * P_BOX + o0),
                                    *reinterpret_cast<const float *>(Pt + 2 * P_BOX + o1)),
                                 pk(*reinterpret_cast<const float *>(Pt + 4 * P_BOX + o0),
                                    *reinterpret_cast<const float *>(Pt + 4 * P_BOX + o1)),
                                 mul2(ur2, h2), mul2(uz2, h2), mul2(un2, h2), splat(br), splat(bz), splat(bn), ur2,
                                 uz2, un2, h2, f2, a2, b2);
                float r0, r1;
                upk(sub2(pk(y0, y1), f2), r0, r1);
                upk(a2, av[i], av[i + 1]);
                upk(b2, bv[i], bv[i + 1]);
                // steps past the sequence's end (zero-filled rows) are the identity map
                if (full || t0 + seg * SL + i < T) {
                    rmax = max(rmax, abs_bits(r0));
                } else {
                    av[i] = 1.f;
                    bv[i] = 0.f;
                }
                if (full || t0 + seg * SL + i + 1 < T) {
                    rmax = max(rmax, abs_bits(r1));
                } else {
                    av[i + 1] = 1.f;
                    bv[i + 1] = 0.f;
                }
#pragma unroll
                for (int u = i; u < i + 2; ++u) {
                    EB = fmaf(av[u], EB, bv[u]);
                    EA = av[u] * EA;
                }
                hp = y1;
            }
            // the predecessors' descriptors, on their way during the barrier
            LookbackWindow<1> lbw{};
            if (tid < DL * LBG) lbw = coop_lookback_prefetch<LBG>(A.desc, tile, S.ngroups, DL, ld, lq, chunk);
            seg_a[seg * DL + d] = EA;
            seg_b[seg * DL + d] = EB;
            __syncthreads();
            if (*cta_err != 0) break;  // uniform: read after the barrier

            // 2. tile carry-in per lane (LBG threads per lane)
            if (tid < DL * LBG) {
                float TA = 1.f, TB = 0.f;
#pragma unroll
                for (int q = 0; q < SEGS; ++q) {
                    const float qa = seg_a[q * DL + ld], qb = seg_b[q * DL + ld];
                    TB = fmaf(qa, TB, qb);
                    TA = qa * TA;
                }
                const float c0 = chunk == 0 ? __ldg(A.h0 + static_cast<size_t>(b) * D + lane0 + ld) : 0.f;
                const float hin =
                    coop_lookback<LBG, 1, true>(A.desc, tile, S.ngroups, DL, ld, lq, epoch, TA, TB, chunk, c0,
                                                 status, &lbw, publishes(A, tile, epoch));
                if (lq == 0) carry[ld] = hin;
            }
            __syncthreads();

            // 3. sweep: carry through the earlier segments, then this thread's steps
            {
                float h = carry[d];
                for (int q = 0; q < seg; ++q) h = fmaf(seg_a[q * DL + d], h, seg_b[q * DL + d]);
                float *out = hnew + static_cast<size_t>(row0) * D + di;
                out += static_cast<size_t>(seg) * SL * D;
#pragma unroll
                for (int i = 0; i < SL; ++i) {
                    h = fmaf(av[i], h, bv[i]);
                    if (full || t0 + seg * SL + i < T) {
                        __stcg(out + static_cast<size_t>(i) * D, h);
                        const int oy = (i + 1) * 128 + ((jq ^ ((i + 1) & 7)) << 4);
                        const float y = *reinterpret_cast<const float *>(Ht + oy);
                        dmax = max(dmax, abs_bits(h - y));
                    }
                }
            }
            __syncthreads();  // slot, segment maps and carries are rewritten next
            if (k + 2 < my_n) {
                if (tid == 0) {
                    int c2, b2, dg2;
                    long long r2;
                    tile_pos(S, tile + 2 * static_cast<long long>(nblocks), T, c2, b2, dg2, r2);
                    issue_fill(&map_p, mh, smem + cur * SLOT, D, r2, dg2 * DL, smem_u32(&bars[cur]));
                }
                fill_pending |= 1u << cur;
            }
        }
        const unsigned bd = block_max_u32(dmax, red);
        const unsigned br = block_max_u32(rmax, red);
        if (tid == 0) {
            atomicMax(&hdr->delta_bits[it % 3], bd);
            atomicMax(&hdr->resid_bits[it % 3], br);
            if (*cta_err) flag_timeout(status);
        }
        // P of the next iteration's first two tiles into L2 while the grid meets:
        // one 256-byte row segment (gate, step) per thread
        if (tid < 2 * 3 * TS) {
            const int q = tid / (3 * TS), g = (tid / TS) % 3, r = tid % TS;
            if (q < my_n) {
                int chunk, b, dg;
                long long row0;
                tile_pos(S, blockIdx.x + static_cast<long long>(q) * nblocks, T, chunk, b, dg, row0);
                if (chunk * TS + r < T) {
                    const float *src = A.P + (row0 + r) * 3 * D + g * D + dg * DL;
                    asm volatile("cp.async.bulk.prefetch.L2.global [%0], 256;" ::"l"(src) : "memory");
                }
            }
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
        for (size_t q = static_cast<size_t>(blockIdx.x) * NT + tid; q < n4; q += static_cast<size_t>(nblocks) * NT)
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
    if (tid == 0)  // copies still in flight after a failed wait finish first
        for (int q = 0; q < 2; ++q)
            if ((fill_pending >> q) & 1u) mbar_drain(smem_u32(&bars[q]), (fill_par >> q) & 1u);
}

}  // namespace

// The streaming path takes the diagonal cell with D a multiple of 64.
bool diag2_supported(const pararnn_cell &cell, int B, int T) {
    if (cell.kind != PARARNN_GRU_DIAG || cell.d % DL != 0) return false;
    if (static_cast<long long>(B) * T >= (1ll << 31) - 1) return false;
    return encode_fn() != nullptr;
}

// Look-back descriptors: tiles of 32 steps x 64 lanes, two words each.
size_t diag2_desc_bytes(int B, int T, int D) {
    const long long tiles = static_cast<long long>(B) * (D / DL) * ((T + TS - 1) / TS);
    return static_cast<size_t>(tiles) * DL * 2 * 8;
}

cudaError_t launch_diag2(const DiagArgs &a, cudaStream_t s) {
    Diag2Args S;
    S.a = a;
    S.ndg = a.D / DL;
    S.ngroups = a.B * S.ndg;
    S.n_tiles = static_cast<long long>(S.ngroups) * ((a.T + TS - 1) / TS);
    CUtensorMap mp, m0, m1;
    const long long rows = static_cast<long long>(a.B) * a.T;
    if (!make_map(&mp, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.P, rows, 3 * a.D, HALF, TS) ||
        !make_map(&m0, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.hbuf[0], rows, a.D, HALF, TS + 1) ||
        !make_map(&m1, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.hbuf[1], rows, a.D, HALF, TS + 1))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(diag2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    int dev = 0, nsm = 0, per_sm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, diag2_kernel, NT, SMEM_BYTES)) != cudaSuccess)
        return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    long long grid = static_cast<long long>(per_sm) * nsm;
    if (grid > S.n_tiles) grid = S.n_tiles;
    void *params[] = {&mp, &m0, &m1, &S};
    return cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(diag2_kernel),
                                       dim3(static_cast<unsigned>(grid)), dim3(NT), params, SMEM_BYTES, s);
}

}  // namespace pararnn

// newton_dense_tc.cu -- quasi-DEER on the dense GRU with the recurrent product
// U h_{t-1} on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// Method: "Towards Scalable and Stable Parallelization of Nonlinear RNNs"
// (atlas summary, "Approach": quasi-DEER, the diagonal of the Jacobian, O(TD)
// memory and work per iteration) on the unrolled system of the ParaRNN summary
// ("Core Idea", "Newton's Iteration").
//
// One cooperative launch runs every Newton iteration; one CTA per SM walks
// tiles of (sequence b, 128 steps, all D state lanes).  Per tile:
//   1. TMA loads the guess rows h_{t-1} (t = t0..t0+127) into shared memory
//      with the 128-byte swizzle; the rows are split in place into a TF32-exact
//      high part and an fp32 remainder (h0 replaces row 0 of a sequence);
//   2. one thread issues tcgen05.mma kind::tf32 (M = 128 steps, N = 3D gate
//      rows, K = 8 per instruction) for hi*U_hi + hi*U_lo + lo*U_hi, the
//      error-compensated 3 x TF32 split, so G = U h_{t-1} is fp32-accurate
//      (U_hi / U_lo stay resident in shared memory for the whole solve);
//   3. the epilogue reads G rows from TMEM (thread = step), evaluates the cell
//      and its Jacobian diagonal a_t, b_t = f_t - a_t h_{t-1} for every lane,
//      and writes them transposed into shared memory (reusing the A buffers);
//   4. a thread per (lane, segment) composes the segment's affine maps, one
//      thread per lane resolves the tile's carry-in by decoupled look-back over
//      earlier chunks of the sequence, and the segment is re-swept, writing
//      h^(i+1), max |h^(i+1) - h^(i)| and the residual max.
// Traffic per state and iteration: P (12 B), the guess row read by TMA and
// again at the re-sweep (4 + 4 B, the second mostly from L2), h^(i+1) (4 B).
// A bounded grid barrier ends each iteration; every CTA reads the same
// reduced delta and stops together.
#include "common.cuh"
#include "lookback.cuh"
#include "solver.cuh"
#include "tc_utils.cuh"

namespace pararnn {
namespace {
using namespace tc;

constexpr int TM = 128;        // steps per tile (MMA M)
constexpr int NTHREADS = 256;  // 8 warps: two threads per tile row in the epilogue

template <int D>
struct TcGeom {
    static constexpr int N = 3 * D;                  // MMA N: gate rows (r, z, n) x lanes
    static constexpr int HALVES = D / 32;            // 128-byte K atoms per row
    static constexpr int A_HALF = TM * 128;          // one K atom of the A tile
    static constexpr int A_BYTES = HALVES * A_HALF;  // 16 KB per atom
    static constexpr int B_HALF = N * 128;
    static constexpr int B_BYTES = HALVES * B_HALF;
    static constexpr int TMEM_COLS = N <= 128 ? 128 : 256;
    static constexpr int OFF_BHI = 0;
    static constexpr int OFF_BLO = B_BYTES;
    static constexpr int OFF_AHI = 2 * B_BYTES;
    static constexpr int OFF_ALO = OFF_AHI + A_BYTES;
    static constexpr int OFF_MISC = OFF_ALO + A_BYTES;
    static constexpr int SEG = NTHREADS / D;  // time segments per lane in the scan
    static constexpr int LS = TM / SEG;       // steps per segment
    static constexpr int LH = D / 2;                      // lanes per warp half in the epilogue
    static constexpr int OFF_SY = OFF_MISC;               // [D][TM] guess h_t of the tile
    static constexpr int SY_BYTES = D * TM * 4;
    static constexpr int OFF_MISC2 = OFF_SY + SY_BYTES;
    // misc: consts (b_hh, diag U) 6D floats, guess before the tile D, segment
    // aggregates 2*SEG*D, prefixes 2*SEG*D, carries D, reduction 32, barriers,
    // TMEM slot, flags
    static constexpr int MISC_FLOATS = 6 * D + D + 4 * SEG * D + D + 32;
    static constexpr int SMEM_BYTES = OFF_MISC2 + MISC_FLOATS * 4 + 64 + 1024;
    static_assert(D == 32 || D == 64, "tensor-core cell path takes D = 32 or 64");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

struct TcArgs {
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

__device__ __forceinline__ void tmem_ld8(unsigned taddr, float (&v)[8]) {
    unsigned r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

template <int D>
__global__ void __launch_bounds__(NTHREADS, 1)
quasi_tc_kernel(const __grid_constant__ CUtensorMap map_h0, const __grid_constant__ CUtensorMap map_h1,
                TcArgs S) {
    using G = TcGeom<D>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    float *SY = reinterpret_cast<float *>(smem + G::OFF_SY);  // [D][TM], lane-swizzled
    float *misc = reinterpret_cast<float *>(smem + G::OFF_MISC2);
    float *c_bh = misc;                   // [3D] b_hh
    float *c_ud = c_bh + 3 * D;           // [3D] diagonal of U_g
    float *ym1 = c_ud + 3 * D;            // [D] guess at step t0 - 1 (h0 at t0 = 0)
    float *seg_a = ym1 + D;               // [SEG][D] segment aggregate A
    float *seg_b = seg_a + G::SEG * D;    // [SEG][D] segment aggregate B
    float *pre_a = seg_b + G::SEG * D;    // [SEG][D] exclusive prefix A
    float *pre_b = pre_a + G::SEG * D;    // [SEG][D] exclusive prefix B
    float *carry = pre_b + G::SEG * D;    // [D] tile carry-in
    unsigned *red = reinterpret_cast<unsigned *>(carry + D);  // [32]
    unsigned long long *bars = reinterpret_cast<unsigned long long *>(red + 32);  // tma, mma
    unsigned *tmem_slot = reinterpret_cast<unsigned *>(bars + 2);
    volatile int *cta_err = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const DiagArgs &A = S.a;
    const int T = A.T;
    WsHeader *hdr = A.hdr;
    unsigned *status = &hdr->status;
    const unsigned nblocks = gridDim.x;
    const int tid = threadIdx.x, warp = tid >> 5;
    unsigned char *bhi = smem + G::OFF_BHI, *blo = smem + G::OFF_BLO;
    unsigned char *ahi = smem + G::OFF_AHI, *alo = smem + G::OFF_ALO;
    float *SA = reinterpret_cast<float *>(ahi);  // [D][TM] a_t, swizzled by lane (aliases A)
    float *SB = reinterpret_cast<float *>(alo);  // [D][TM] b_t

    // ---- once per solve: U split into TF32 hi / lo, constants, barriers, TMEM
    for (int i = tid; i < G::N * D; i += NTHREADS) {
        const int n = i / D, k = i % D;
        const float v = __ldg(A.w_hh + i);
        const float hi = __uint_as_float(__float_as_uint(v) & 0xffffe000u);
        const int off = sw_off(n, k, G::B_HALF);
        *reinterpret_cast<float *>(bhi + off) = hi;
        *reinterpret_cast<float *>(blo + off) = v - hi;
    }
    for (int i = tid; i < 3 * D; i += NTHREADS) {
        c_bh[i] = __ldg(A.b_hh + i);
        const int g = i / D, d = i % D;
        c_ud[i] = __ldg(A.w_hh + (static_cast<size_t>(g) * D + d) * D + d);
    }
    if (tid == 0) {
        mbar_init(smem_u32(&bars[0]), 1);
        mbar_init(smem_u32(&bars[1]), 1);
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

    unsigned tile_phase = 0;  // mbarrier parity, flips every tile
    int iters = 0, final_status = PARARNN_NOT_CONVERGED;
    unsigned last_delta = 0u, last_resid = 0u;
    for (int it = 0; it < A.max_iters; ++it) {
        if (blockIdx.x == 0 && tid == 0) {
            hdr->delta_bits[(it + 1) % 3] = 0u;
            hdr->resid_bits[(it + 1) % 3] = 0u;
        }
        const float *hold = A.hbuf[it & 1];
        float *hnew = A.hbuf[(it + 1) & 1];
        const CUtensorMap *map = (it & 1) ? &map_h1 : &map_h0;
        const unsigned epoch = static_cast<unsigned>(it + 1);
        unsigned dmax = 0u, rmax = 0u;

        for (long long tile = blockIdx.x; tile < S.n_tiles; tile += nblocks) {
            const int chunk = static_cast<int>(tile / A.B);
            const int b = static_cast<int>(tile % A.B);
            const int t0 = chunk * TM;
            const long long row0 = static_cast<long long>(b) * T + t0;  // flat row of step t0

            // 1. guess rows h_{t-1}, t = t0..t0+127 (row t0-1 may be out of range: zero fill)
            if (tid == 0) {
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // after the last tile's reads
                const unsigned bar = smem_u32(&bars[0]);
                mbar_expect_tx(bar, G::A_BYTES);
#pragma unroll
                for (int hf = 0; hf < G::HALVES; ++hf)
                    tma_load_2d(smem_u32(ahi + hf * G::A_HALF), map, hf * 32,
                                static_cast<int>(row0 - 1), bar);
            }
            if (!mbar_wait(smem_u32(&bars[0]), tile_phase, cta_err)) *cta_err = 1;
            // split the tile into hi (in place) and lo, element-wise; thread =
            // (row, K atom); chunks visited in a rotated order (no bank conflicts)
            {
                const int r = tid % TM, hq = tid / TM;
                if (t0 == 0 && r == 0)  // h_{t-1} of a sequence's first step is h0
                    for (int k = 0; k < D; ++k)
                        if ((k >> 5) % (NTHREADS / TM) == hq)  // the K atom this thread splits
                            *reinterpret_cast<float *>(ahi + sw_off(0, k, G::A_HALF)) =
                                __ldg(A.h0 + static_cast<size_t>(b) * D + k);
#pragma unroll
                for (int hf = hq; hf < G::HALVES; hf += NTHREADS / TM)
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj) {
                        const int j = (jj + r) & 7;
                        const int off = hf * G::A_HALF + r * 128 + j * 16;
                        float4 v = *reinterpret_cast<float4 *>(ahi + off);
                        float4 hi, lo;
                        hi.x = __uint_as_float(__float_as_uint(v.x) & 0xffffe000u); lo.x = v.x - hi.x;
                        hi.y = __uint_as_float(__float_as_uint(v.y) & 0xffffe000u); lo.y = v.y - hi.y;
                        hi.z = __uint_as_float(__float_as_uint(v.z) & 0xffffe000u); lo.z = v.z - hi.z;
                        hi.w = __uint_as_float(__float_as_uint(v.w) & 0xffffe000u); lo.w = v.w - hi.w;
                        *reinterpret_cast<float4 *>(ahi + off) = hi;
                        *reinterpret_cast<float4 *>(alo + off) = lo;
                    }
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            asm volatile("tcgen05.fence::before_thread_sync;");
            __syncthreads();
            const bool bad = *cta_err != 0;
            if (bad) break;  // uniform: read after the barrier

            // 2. G = U h_{t-1}: lo*U_hi + hi*U_lo + hi*U_hi (small terms first)
            if (tid == 0) {
                asm volatile("tcgen05.fence::after_thread_sync;");
                const unsigned a_hi = smem_u32(ahi), a_lo = smem_u32(alo);
                const unsigned b_hi = smem_u32(bhi), b_lo = smem_u32(blo);
#pragma unroll
                for (int term = 0; term < 3; ++term) {
                    const unsigned as = term == 0 ? a_lo : a_hi;
                    const unsigned bs = term == 1 ? b_lo : b_hi;
#pragma unroll
                    for (int ks = 0; ks < D / 8; ++ks) {
                        const int hf = ks >> 2, off = (ks & 3) * 32;
                        const unsigned long long da = sw128_desc(as + hf * G::A_HALF + off);
                        const unsigned long long db = sw128_desc(bs + hf * G::B_HALF + off);
                        const unsigned acc = (term > 0 || ks > 0) ? 1u : 0u;
                        asm volatile(
                            "{\n\t.reg .pred p;\n\t"
                            "setp.ne.b32 p, %4, 0;\n\t"
                            "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem),
                            "l"(da), "l"(db), "r"(idesc), "r"(acc));
                    }
                }
                asm volatile(
                    "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                        smem_u32(&bars[1])));
            }

            // 3. epilogue in the 16x256b TMEM fragment layout: warp w reads rows of
            // its TMEM quadrant qd = w % 4 for the lane half lh = w / 4; thread
            // (gid, tq) owns rows qd*32 + rh*16 + gid + 8*e (rh, e in {0,1}) and lanes
            // lh*LH + 8*j + 2*tq + {0,1} -- all three gates of each (step, lane).
            const int qd = warp & 3, lh = warp >> 2;
            const int gid = (tid & 31) >> 2, tq = tid & 3;
            constexpr int NJ = G::LH / 8;
            // input pre-activations first: their latency overlaps the products
            float2 pv[2][2][NJ][3];
#pragma unroll
            for (int rh = 0; rh < 2; ++rh)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int r = qd * 32 + rh * 16 + gid + 8 * e;
                    const bool ok = t0 + r < T;
                    const float *prow = A.P + (static_cast<size_t>(row0) + r) * 3 * D + lh * G::LH + 2 * tq;
#pragma unroll
                    for (int j = 0; j < NJ; ++j)
#pragma unroll
                        for (int g = 0; g < 3; ++g)
                            pv[rh][e][j][g] = ok ? __ldg(reinterpret_cast<const float2 *>(prow + g * D + 8 * j))
                                                 : make_float2(0.f, 0.f);
                }
            if (!mbar_wait(smem_u32(&bars[1]), tile_phase, cta_err)) *cta_err = 1;
            asm volatile("tcgen05.fence::after_thread_sync;");
            tile_phase ^= 1u;
            // h_{t-1} of this thread's (step, lane) pairs, and the guess rows for the scan
            float2 hp[2][2][NJ];
#pragma unroll
            for (int rh = 0; rh < 2; ++rh)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int r = qd * 32 + rh * 16 + gid + 8 * e;
#pragma unroll
                    for (int j = 0; j < NJ; ++j) {
                        const int d = lh * G::LH + 8 * j + 2 * tq;
                        const int off = sw_off(r, d, G::A_HALF);
                        const float2 vh = *reinterpret_cast<const float2 *>(ahi + off);
                        const float2 vl = *reinterpret_cast<const float2 *>(alo + off);
                        hp[rh][e][j] = make_float2(vh.x + vl.x, vh.y + vl.y);
                        if (r == 0) {
                            ym1[d] = hp[rh][e][j].x;
                            ym1[d + 1] = hp[rh][e][j].y;
                        } else {
                            SY[d * TM + ((r - 1) ^ (d & 31))] = hp[rh][e][j].x;
                            SY[(d + 1) * TM + ((r - 1) ^ ((d + 1) & 31))] = hp[rh][e][j].y;
                        }
                        if (r == TM - 1) {  // h_t of the tile's last step is not in the A tile
                            float2 yl = make_float2(0.f, 0.f);
                            if (t0 + r < T)
                                yl = __ldcg(reinterpret_cast<const float2 *>(hold + (static_cast<size_t>(row0) + r) * D + d));
                            SY[d * TM + ((TM - 1) ^ (d & 31))] = yl.x;
                            SY[(d + 1) * TM + ((TM - 1) ^ ((d + 1) & 31))] = yl.y;
                        }
                    }
                }
            __syncthreads();  // A is free: SA / SB overwrite it
#pragma unroll
            for (int rh = 0; rh < 2; ++rh) {
                const unsigned trow = tmem + (static_cast<unsigned>(qd * 32 + rh * 16) << 16);
#pragma unroll
                for (int j = 0; j < NJ; ++j) {
                    const int col = lh * G::LH + 8 * j;
                    unsigned gv[3][4];
#pragma unroll
                    for (int g = 0; g < 3; ++g)
                        asm volatile("tcgen05.ld.sync.aligned.16x256b.x1.b32 {%0,%1,%2,%3}, [%4];"
                                     : "=r"(gv[g][0]), "=r"(gv[g][1]), "=r"(gv[g][2]), "=r"(gv[g][3])
                                     : "r"(trow + g * D + col));
                    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int r = qd * 32 + rh * 16 + gid + 8 * e;
                        const bool ok = t0 + r < T;
#pragma unroll
                        for (int x = 0; x < 2; ++x) {
                            const int d = col + 2 * tq + x;
                            float av = 1.f, bv = 0.f;
                            if (ok) {
                                const float2 pr = pv[rh][e][j][0], pz = pv[rh][e][j][1], pn = pv[rh][e][j][2];
                                float f;
                                gru_cell_diag(x ? pr.y : pr.x, x ? pz.y : pz.x, x ? pn.y : pn.x,
                                              __uint_as_float(gv[0][2 * e + x]),
                                              __uint_as_float(gv[1][2 * e + x]),
                                              __uint_as_float(gv[2][2 * e + x]), c_bh[d], c_bh[D + d],
                                              c_bh[2 * D + d], c_ud[d], c_ud[D + d], c_ud[2 * D + d],
                                              x ? hp[rh][e][j].y : hp[rh][e][j].x, f, av, bv);
                            }
                            const int cc = r ^ (d & 31);
                            SA[d * TM + cc] = av;
                            SB[d * TM + cc] = bv;
                        }
                    }
                }
            }
            asm volatile("tcgen05.fence::before_thread_sync;");
            __syncthreads();

            // 4. scan over the tile's steps: thread = (lane d, segment sg)
            {
                const int d = tid % D, sg = tid / D;
                const int sw = d & 31;
                const int s0 = sg * G::LS;
                int nv = T - (t0 + s0);
                nv = nv < 0 ? 0 : (nv > G::LS ? G::LS : nv);
                float ca = 1.f, cb = 0.f;
                for (int q = 0; q < G::LS; ++q) {
                    const int col = (s0 + q) ^ sw;
                    const float a_ = SA[d * TM + col], b_ = SB[d * TM + col];
                    cb = fmaf(a_, cb, b_);
                    ca = a_ * ca;
                }
                seg_a[sg * D + d] = ca;
                seg_b[sg * D + d] = cb;
                __syncthreads();
                if (sg == 0) {
                    float EA = 1.f, EB = 0.f;
#pragma unroll
                    for (int q = 0; q < G::SEG; ++q) {
                        pre_a[q * D + d] = EA;
                        pre_b[q * D + d] = EB;
                        const float qa = seg_a[q * D + d], qb = seg_b[q * D + d];
                        EB = fmaf(qa, EB, qb);
                        EA = qa * EA;
                    }
                    const float c0 = chunk == 0 ? __ldg(A.h0 + static_cast<size_t>(b) * D + d) : 0.f;
                    carry[d] = lookback_affine(A.desc, tile, A.B, D, d, epoch, EA, EB, chunk, c0, status);
                }
                __syncthreads();
                float h = fmaf(pre_a[sg * D + d], carry[d], pre_b[sg * D + d]);
                float yp = s0 == 0 ? ym1[d] : SY[d * TM + ((s0 - 1) ^ sw)];
                float* hrow = hnew + (static_cast<size_t>(b) * T + t0 + s0) * D + d;
                for (int q = 0; q < nv; ++q) {
                    const int col = (s0 + q) ^ sw;
                    const float a_ = SA[d * TM + col], b_ = SB[d * TM + col];
                    const float y = SY[d * TM + col];
                    h = fmaf(a_, h, b_);
                    __stcg(hrow + static_cast<size_t>(q) * D, h);
                    dmax = max(dmax, abs_bits(h - y));
                    rmax = max(rmax, abs_bits(y - fmaf(a_, yp, b_)));
                    yp = y;
                }
            }
            __syncthreads();  // SA / SB / SY are rewritten by the next tile
        }
        const unsigned bd = block_max_u32(dmax, red);
        const unsigned br = block_max_u32(rmax, red);
        if (tid == 0) {
            atomicMax(&hdr->delta_bits[it % 3], bd);
            atomicMax(&hdr->resid_bits[it % 3], br);
            if (*cta_err) flag_timeout(status);
        }
        grid_barrier(hdr->barrier, nblocks, status);
        last_delta = ld_acquire_u32(&hdr->delta_bits[it % 3]);
        last_resid = ld_acquire_u32(&hdr->resid_bits[it % 3]);
        iters = it + 1;
        if (timed_out(status)) { final_status = PARARNN_TIMEOUT; break; }
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
    if (*cta_err && tid == 0) {  // a wait ran out: let copies and products in flight finish
        mbar_drain(smem_u32(&bars[0]), tile_phase);
        mbar_drain(smem_u32(&bars[1]), tile_phase);
    }
    asm volatile("tcgen05.fence::before_thread_sync;");
    __syncthreads();
    if (warp == 1) {
        asm volatile("tcgen05.fence::after_thread_sync;");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(G::TMEM_COLS));
    }
}

template <int D>
cudaError_t launch_tc(const DiagArgs &a, cudaStream_t s) {
    using G = TcGeom<D>;
    TcArgs S;
    S.a = a;
    S.n_chunks = (a.T + TM - 1) / TM;
    S.n_tiles = static_cast<long long>(a.B) * S.n_chunks;
    CUtensorMap m0, m1;
    const long long rows = static_cast<long long>(a.B) * a.T;
    if (!make_map(&m0, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.hbuf[0], rows, D, 32, TM) ||
        !make_map(&m1, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.hbuf[1], rows, D, 32, TM))
        return cudaErrorInvalidValue;
    auto kern = quasi_tc_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         G::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    int dev = 0, nsm = 0, per_sm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, NTHREADS, G::SMEM_BYTES)) !=
        cudaSuccess)
        return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    long long grid = static_cast<long long>(per_sm) * nsm;
    if (grid > S.n_tiles) grid = S.n_tiles;
    void *params[] = {&m0, &m1, &S};
    return cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(kern),
                                       dim3(static_cast<unsigned>(grid)), dim3(NTHREADS), params,
                                       G::SMEM_BYTES, s);
}

}  // namespace

// Descriptors the tensor-core path needs: tiles of 128 steps x D lanes, two words each.
size_t quasi_tc_desc_bytes(int B, int T, int D) {
    const long long tiles = static_cast<long long>(B) * ((T + TM - 1) / TM);
    return static_cast<size_t>(tiles) * D * 2 * 8;
}

bool quasi_tc_supported(const pararnn_cell &cell, int B, int T) {
    if (cell.kind != PARARNN_GRU_DENSE || (cell.d != 32 && cell.d != 64)) return false;
    if (static_cast<long long>(B) * T >= (1ll << 31) - 1) return false;
    return encode_fn() != nullptr;
}

cudaError_t launch_quasi_tc(const DiagArgs &a, cudaStream_t s) {
    return a.D == 32 ? launch_tc<32>(a, s) : launch_tc<64>(a, s);
}

}  // namespace pararnn

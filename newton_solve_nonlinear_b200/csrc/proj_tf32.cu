// proj_tf32.cu -- the input projection P = x W^T + b for fp32 operands on the
// 5th-generation tensor cores (tcgen05, sm_100a), as an error-compensated
// 3 x TF32 product.
//
// The input projection does not depend on the state, so one GEMM
// [M = B*T, K = Din] x [K, N = 3D] serves every Newton iteration (and the
// dense backward pass uses the same GEMM for U h_{t-1}).  For the fp32 dense
// workloads (K = 64, N = 192) it is short and wide: 2 M N K flop against
// 4 (K + N) bytes per row, so it should run at the speed of writing P.
//
// One CTA per SM walks row tiles of 128 (persistent, no grid barrier):
//   * TMA brings a tile of x (128 rows x K fp32, 128-byte swizzle) into one
//     of two shared-memory slots;
//   * all eight warps split the tile into a TF32-exact high part and an fp32
//     remainder and write both to TMEM as the MMA's A operand (thread = row);
//   * one thread issues tcgen05.mma kind::tf32 (M = 128, N, K = 8 per
//     instruction) for lo*W_hi + hi*W_lo + hi*W_hi into one of two TMEM
//     accumulators (W_hi, W_lo stay in shared memory for the whole launch);
//   * while those products run, the warps read the other accumulator (the
//     previous tile) in the 16x256b layout, add the bias and store the rows of
//     P in whole 32-byte sectors.
// The dropped lo*lo term is below 2^-22 of each product, so P agrees with an
// fp32 FMA evaluation to within fp32 rounding of the sum.  Every wait is
// bounded; a wait that runs out makes the CTA drain what it started and write
// NaN over its rows, which a solve reports as DIVERGED.
#include "common.cuh"
#include "solver.cuh"
#include "tc_utils.cuh"

namespace pararnn {
namespace {
using namespace tc;

constexpr int PM = 128;   // rows per tile (MMA M)
constexpr int PNT = 256;  // 8 warps: TMEM lane quarter x (K half | column half)

template <int N, int K>
struct PGeom {
    static constexpr int HALVES = K / 32;           // 128-byte K atoms per row
    static constexpr int SLOT_HALF = PM * 128;      // one K atom of a tile, 16 KB
    static constexpr int SLOT_BYTES = HALVES * SLOT_HALF;
    static constexpr int B_HALF = N * 128;
    static constexpr int B_BYTES = HALVES * B_HALF;
    static constexpr int ACC1 = (N + 63) / 64 * 64;  // TMEM: accumulators at 0 and ACC1,
    static constexpr int A_HI = 2 * ACC1;            // then the A operand, hi and lo
    static constexpr int A_LO = A_HI + K;
    static constexpr int TMEM_COLS = 512;
    static constexpr int OFF_BHI = 0;
    static constexpr int OFF_BLO = B_BYTES;
    static constexpr int OFF_SLOT = 2 * B_BYTES;
    static constexpr int OFF_MISC = OFF_SLOT + 2 * SLOT_BYTES;  // bias [N], 4 barriers, TMEM slot, flag
    static constexpr int SMEM_BYTES = OFF_MISC + N * 4 + 64 + 1024;
    static_assert(K == 32 || K == 64, "K atoms");
    static_assert(N % 32 == 0 && N <= 256, "N: two column halves of 16-column loads, MMA N <= 256");
    static_assert(A_LO + K <= TMEM_COLS, "TMEM columns");
    static_assert(B_HALF % 1024 == 0, "swizzle atoms stay 1024-byte aligned");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

// Swizzled byte offset of element (row, k) in a K-major 128-byte-swizzle tile
// made of K atoms of `half_bytes` each.
__device__ __forceinline__ int swz(int row, int k, int half_bytes) {
    const int hf = k >> 5, j = (k & 31) >> 2;
    return hf * half_bytes + row * 128 + ((j ^ (row & 7)) << 4) + ((k & 3) << 2);
}

__device__ __forceinline__ void tmem_st16(unsigned taddr, const unsigned (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
        "%13,%14,%15,%16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

// A operand of the tile in `slot`: warp (quarter qd, half kq) writes TMEM
// lanes 32 qd .. 32 qd + 31 (rows of the tile), K columns kq K/2 .. + K/2 - 1.
template <int N, int K>
__device__ __forceinline__ void put_a(const unsigned char *slot, unsigned tmem, int warp, int lane) {
    using G = PGeom<N, K>;
    constexpr int KW = K / 2;
    const int qd = warp & 3, kq = warp >> 2;
    const int r = qd * 32 + lane;
    const unsigned lane_base = static_cast<unsigned>(qd * 32) << 16;
#pragma unroll
    for (int c = 0; c < KW; c += 16) {
        const int k0 = kq * KW + c;
        unsigned hi[16], lo[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 x = *reinterpret_cast<const float4 *>(slot + swz(r, k0 + 4 * q, G::SLOT_HALF));
            const float v[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                hi[4 * q + e] = __float_as_uint(v[e]) & 0xffffe000u;
                lo[4 * q + e] = __float_as_uint(v[e] - __uint_as_float(hi[4 * q + e]));
            }
        }
        tmem_st16(tmem + lane_base + G::A_HI + k0, hi);
        tmem_st16(tmem + lane_base + G::A_LO + k0, lo);
    }
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// One thread: lo*W_hi + hi*W_lo + hi*W_hi into accumulator `acc`, then commit to `bar`.
template <int N, int K>
__device__ __forceinline__ void issue_products(unsigned tmem, unsigned acc, unsigned b_hi, unsigned b_lo,
                                               unsigned bar) {
    using G = PGeom<N, K>;
    constexpr unsigned idesc = make_idesc(2u, PM, N);  // kind::tf32, fp32 accumulate
#pragma unroll
    for (int term = 0; term < 3; ++term) {
        const unsigned a_col = term == 0 ? G::A_LO : G::A_HI;
        const unsigned bs = term == 1 ? b_lo : b_hi;
#pragma unroll
        for (int ks = 0; ks < K / 8; ++ks) {
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

template <int N, int K>
__device__ __forceinline__ void issue_tile_load(const CUtensorMap *map, unsigned char *slot, long long row0,
                                                unsigned bar) {
    using G = PGeom<N, K>;
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // after the slot's last reads
    mbar_expect_tx(bar, G::SLOT_BYTES);
#pragma unroll
    for (int hf = 0; hf < G::HALVES; ++hf)
        tma_load_2d(smem_u32(slot + hf * G::SLOT_HALF), map, hf * 32, static_cast<int>(row0), bar);
}

template <int N, int K>
__global__ void __launch_bounds__(PNT, 1)
proj_tf32_kernel(const __grid_constant__ CUtensorMap map_x, const float *__restrict__ W,
                 const float *__restrict__ bias, float *__restrict__ P, long long M) {
    using G = PGeom<N, K>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    unsigned char *bhi = smem + G::OFF_BHI, *blo = smem + G::OFF_BLO, *slots = smem + G::OFF_SLOT;
    float *c_b = reinterpret_cast<float *>(smem + G::OFF_MISC);
    unsigned long long *bars = reinterpret_cast<unsigned long long *>(c_b + N);  // 0, 1: loads; 2, 3: products
    unsigned *tmem_slot = reinterpret_cast<unsigned *>(bars + 4);
    volatile int *cta_err = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qd = warp & 3, ch = warp >> 2;

    // ---- once per launch: W split into TF32 hi / lo (K-major, swizzled), bias, barriers, TMEM
    for (int i = tid; i < N * K; i += PNT) {
        const int n = i / K, k = i - n * K;
        const float v = __ldg(W + i);
        const float hi = __uint_as_float(__float_as_uint(v) & 0xffffe000u);
        const int off = swz(n, k, G::B_HALF);
        *reinterpret_cast<float *>(bhi + off) = hi;
        *reinterpret_cast<float *>(blo + off) = v - hi;
    }
    for (int i = tid; i < N; i += PNT) c_b[i] = __ldg(bias + i);
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
    const unsigned b_hi = smem_u32(bhi), b_lo = smem_u32(blo);

    const long long n_tiles = (M + PM - 1) / PM;
    const long long nb = gridDim.x;
    const long long my_n = blockIdx.x < n_tiles ? (n_tiles - blockIdx.x + nb - 1) / nb : 0;
    auto row0_of = [&](long long k) { return (static_cast<long long>(blockIdx.x) + k * nb) * PM; };

    // bit q: mbarrier parity of slot q / accumulator q; an operation in flight
    unsigned load_par = 0u, mma_par = 0u, load_pending = 0u, mma_pending = 0u;
    if (tid == 0)
        for (int q = 0; q < 2 && q < my_n; ++q)
            issue_tile_load<N, K>(&map_x, slots + q * G::SLOT_BYTES, row0_of(q), smem_u32(&bars[q]));
    load_pending = my_n > 1 ? 3u : (my_n > 0 ? 1u : 0u);
    if (my_n > 0) {
        if (!mbar_wait(smem_u32(&bars[0]), 0u, cta_err)) *cta_err = 1;
        load_par ^= 1u;
        load_pending &= ~1u;
        put_a<N, K>(slots, tmem, warp, lane);
        asm volatile("tcgen05.fence::before_thread_sync;");
        __syncthreads();
        if (!*cta_err) {
            asm volatile("tcgen05.fence::after_thread_sync;");
            if (tid == 0) {
                issue_products<N, K>(tmem, 0u, b_hi, b_lo, smem_u32(&bars[2]));
                if (my_n > 2) issue_tile_load<N, K>(&map_x, slots, row0_of(2), smem_u32(&bars[0]));
            }
            mma_pending |= 1u;
            if (my_n > 2) load_pending |= 1u;
        }
    }

    for (long long k = 0; k < my_n && !*cta_err; ++k) {
        const int cur = static_cast<int>(k & 1), nxt = cur ^ 1;
        // the products of tile k are done: the A operand is free for tile k+1
        if (!mbar_wait(smem_u32(&bars[2 + cur]), (mma_par >> cur) & 1u, cta_err)) *cta_err = 1;
        mma_par ^= 1u << cur;
        mma_pending &= ~(1u << cur);
        if (k + 1 < my_n) {
            if (!mbar_wait(smem_u32(&bars[nxt]), (load_par >> nxt) & 1u, cta_err)) *cta_err = 1;
            load_par ^= 1u << nxt;
            load_pending &= ~(1u << nxt);
            put_a<N, K>(slots + nxt * G::SLOT_BYTES, tmem, warp, lane);
        }
        asm volatile("tcgen05.fence::before_thread_sync;");
        __syncthreads();
        if (*cta_err) break;  // uniform: read after the barrier
        asm volatile("tcgen05.fence::after_thread_sync;");
        if (k + 1 < my_n) {
            if (tid == 0) {
                issue_products<N, K>(tmem, nxt ? G::ACC1 : 0u, b_hi, b_lo, smem_u32(&bars[2 + nxt]));
                if (k + 3 < my_n)  // the slot tile k+1 came from is free again
                    issue_tile_load<N, K>(&map_x, slots + nxt * G::SLOT_BYTES, row0_of(k + 3),
                                          smem_u32(&bars[nxt]));
            }
            mma_pending |= 1u << nxt;
            if (k + 3 < my_n) load_pending |= 1u << nxt;
        }
        // epilogue of tile k: warp (qd, ch) takes rows 32 qd .. + 31 and columns
        // ch N/2 .. + N/2 - 1 in the 16x256b layout (thread (gid, tq): rows gid and
        // gid + 8 of a 16-row half, columns 2 tq, 2 tq + 1 of each 8), so the four
        // threads of a row store 32 contiguous bytes: whole sectors
        const int gid = lane >> 2, tq = lane & 3;
        const unsigned tbase = tmem + (cur ? G::ACC1 : 0u) + (static_cast<unsigned>(qd * 32) << 16);
#pragma unroll
        for (int rh = 0; rh < 2; ++rh) {
            const unsigned trow = tbase + (static_cast<unsigned>(rh * 16) << 16);
            const long long ma = row0_of(k) + qd * 32 + rh * 16 + gid, mb = ma + 8;
#pragma unroll
            for (int c = 0; c < N / 2; c += 32) {
                constexpr int NQ_FULL = 4;
                const int nq = (N / 2 - c) / 8 < NQ_FULL ? (N / 2 - c) / 8 : NQ_FULL;
                unsigned v[NQ_FULL][4];
#pragma unroll
                for (int q = 0; q < NQ_FULL; ++q)
                    if (q < nq)
                        asm volatile("tcgen05.ld.sync.aligned.16x256b.x1.b32 {%0,%1,%2,%3}, [%4];"
                                     : "=r"(v[q][0]), "=r"(v[q][1]), "=r"(v[q][2]), "=r"(v[q][3])
                                     : "r"(trow + ch * (N / 2) + c + 8 * q));
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
                for (int q = 0; q < NQ_FULL; ++q) {
                    if (q >= nq) continue;
                    const int col = ch * (N / 2) + c + 8 * q + 2 * tq;
                    const float2 b2 = *reinterpret_cast<const float2 *>(c_b + col);
                    if (ma < M)
                        __stcs(reinterpret_cast<float2 *>(P + ma * N + col),
                               make_float2(__uint_as_float(v[q][0]) + b2.x, __uint_as_float(v[q][1]) + b2.y));
                    if (mb < M)
                        __stcs(reinterpret_cast<float2 *>(P + mb * N + col),
                               make_float2(__uint_as_float(v[q][2]) + b2.x, __uint_as_float(v[q][3]) + b2.y));
                }
            }
        }
    }

    const bool failed = *cta_err != 0;
    if (tid == 0) {  // copies and products still in flight finish before the CTA leaves
        for (int q = 0; q < 2; ++q) {
            if ((load_pending >> q) & 1u) mbar_drain(smem_u32(&bars[q]), (load_par >> q) & 1u);
            if ((mma_pending >> q) & 1u) mbar_drain(smem_u32(&bars[2 + q]), (mma_par >> q) & 1u);
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;");
    __syncthreads();
    if (failed)  // every row of this CTA's tiles becomes NaN
        for (long long k = 0; k < my_n; ++k)
            for (int i = tid; i < PM * N; i += PNT) {
                const long long m = row0_of(k) + i / N;
                if (m < M) P[m * N + i % N] = __int_as_float(0x7fc00000);
            }
    if (warp == 1) {
        asm volatile("tcgen05.fence::after_thread_sync;");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(G::TMEM_COLS));
    }
}

template <int N, int K>
cudaError_t launch_tf32(const float *x, const float *w, const float *b, float *P, long long M, cudaStream_t s) {
    using G = PGeom<N, K>;
    CUtensorMap mx;
    if (!make_map(&mx, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, x, M, K, 32, PM)) return cudaErrorInvalidValue;
    auto kern = proj_tf32_kernel<N, K>;
    // every CTA takes all 512 TMEM columns: its shared-memory request keeps it alone on an SM
    const int smem = G::SMEM_BYTES > 120 * 1024 ? G::SMEM_BYTES : 120 * 1024;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int dev = 0, nsm = 0, per_sm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, PNT, smem)) != cudaSuccess) return e;
    if (per_sm != 1) return cudaErrorInvalidConfiguration;
    const long long n_tiles = (M + PM - 1) / PM;
    const long long grid = n_tiles < nsm ? n_tiles : nsm;
    kern<<<static_cast<unsigned>(grid), PNT, smem, s>>>(mx, w, b, P, M);
    return cudaGetLastError();
}

}  // namespace

// fp32 x [M, K] with K = 32 or 64, N = 96 or 192 output columns, x and P
// 16-byte aligned, M < 2^31 (TMA row coordinates are 32-bit).
bool proj_tf32_supported(int x_dtype, long long M, int N, int K, const void *x, const void *P) {
    if (x_dtype != PARARNN_F32 || M < 1 || M >= (1ll << 31) - PM) return false;
    if ((N != 96 && N != 192) || (K != 32 && K != 64)) return false;
    if (reinterpret_cast<uintptr_t>(x) % 16 != 0 || reinterpret_cast<uintptr_t>(P) % 16 != 0) return false;
    return encode_fn() != nullptr;
}

cudaError_t launch_proj_tf32(const float *x, const float *w, const float *b, float *P, long long M, int N, int K,
                             cudaStream_t s) {
    if (N == 192) return K == 64 ? launch_tf32<192, 64>(x, w, b, P, M, s) : launch_tf32<192, 32>(x, w, b, P, M, s);
    return K == 64 ? launch_tf32<96, 64>(x, w, b, P, M, s) : launch_tf32<96, 32>(x, w, b, P, M, s);
}

}  // namespace pararnn

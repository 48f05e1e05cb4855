// proj_tcgen05.cu -- the input projection P = x W_ih^T + b_ih on the 5th-generation
// tensor cores (tcgen05, sm_100a), for bf16 operands.
//
// The input projection does not depend on the state, so one GEMM
// [B*T, Din] x [Din, 3D] serves every Newton iteration.  For the bf16 layer
// (Din = D = 2048) it is the one tensor-bound step of the solve (2*M*N*K flop).
//
// A persistent CTA per SM walks the 128 x 256 fp32 tiles of P (tile t: rows
// 128 (t / nN), columns 256 (t % nN), so the CTAs working at one time share
// their rows of x in L2 and every tile of W_ih stays there), with its warps
// specialised:
//   * warp 0 (one thread): TMA brings 128 x 64 tiles of x and 256 x 64 tiles of
//     W_ih (bf16, 128-byte swizzle) into a ring of STAGES shared-memory
//     stages, signalled by mbarriers;
//   * warp 1 (one thread): tcgen05.mma kind::f16 (bf16 x bf16 -> fp32, M = 128,
//     N = 256, K = 16 per instruction) into one of two 256-column TMEM
//     accumulators, freeing each stage with tcgen05.commit and handing the
//     finished accumulator to the epilogue;
//   * warps 2-5: read an accumulator's rows with tcgen05.ld (thread = row, warp
//     w reads lane quarter w % 4), add the bias, stage 32-column blocks in a
//     double-buffered shared-memory area with the 128-byte swizzle and TMA-store
//     them, then free the accumulator -- while the next tile's products run in
//     the other one.
// Every wait is bounded; a wait that runs out raises an error flag, every role
// stops issuing, the epilogue writes NaN into the tiles it has not stored
// (which the solver reports as DIVERGED), and work in flight is drained before
// TMEM is freed.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "solver.cuh"
#include "tc_utils.cuh"

namespace pararnn {
namespace {
using namespace tc;

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;        // 16 KB
constexpr int B_BYTES = BN * BK * 2;        // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int OUT_BLOCK = BM * 128;         // 32 fp32 columns of 128 rows: 16 KB
constexpr int OFF_OUT = STAGES * STAGE_BYTES;
constexpr int OFF_BARS = OFF_OUT + 2 * OUT_BLOCK;
constexpr int SMEM_BYTES = OFF_BARS + 256 + 1024;  // + barriers, flags, alignment
constexpr int NTHR = 192;                   // producer, MMA, four epilogue warps
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");

// kind::f16 instruction descriptor: fp32 accumulate, bf16 A and B, both K-major.
constexpr unsigned kIdescBf16 = make_idesc(1u, BM, BN);

__device__ __forceinline__ void mbar_arrive(unsigned bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// OR of v over the 128 epilogue threads (named barrier 1), the same in each.
__device__ __forceinline__ bool epi_any(bool v) {
    unsigned r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.cta.red.or.pred q, 1, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(static_cast<unsigned>(v))
        : "memory");
    return r != 0u;
}

__global__ void __launch_bounds__(NTHR, 1)
proj_tcgen05_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
                    const __grid_constant__ CUtensorMap map_p, const float *__restrict__ bias, int K,
                    float *__restrict__ Pout, long long M, int N) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    unsigned long long *bars = reinterpret_cast<unsigned long long *>(smem + OFF_BARS);
    // full[STAGES], empty[STAGES], acc_full[2], acc_empty[2]
    unsigned long long *full = bars, *empty = bars + STAGES, *acc_full = bars + 2 * STAGES,
                       *acc_empty = bars + 2 * STAGES + 2;
    unsigned *tmem_slot = reinterpret_cast<unsigned *>(bars + 2 * STAGES + 4);
    volatile int *err = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *issued = reinterpret_cast<volatile int *>(tmem_slot + 2);    // k-blocks loaded by TMA
    volatile int *consumed = reinterpret_cast<volatile int *>(tmem_slot + 3);  // k-blocks given to MMA

    const int warp = threadIdx.x >> 5;
    const long long nM = (M + BM - 1) / BM;
    const int nN = N / BN, nk = K / BK;
    const long long n_tiles = nM * nN;
    const long long my_n = blockIdx.x < n_tiles ? (n_tiles - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&acc_full[a]), 1);
            mbar_init(smem_u32(&acc_empty[a]), 4);  // one arrival per epilogue warp
        }
        *err = 0;
        *issued = 0;
        *consumed = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(2 * BN));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    asm volatile("tcgen05.fence::before_thread_sync;");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;");
    const unsigned tmem = *tmem_slot;

    if (threadIdx.x == 0) {
        // TMA producer: k-block q of this CTA's sequence goes to stage q % STAGES
        long long q = 0;
        bool ok = true;
        for (long long k = 0; k < my_n && ok; ++k) {
            const long long tile = blockIdx.x + k * gridDim.x;
            const int m0 = static_cast<int>(tile / nN) * BM, n0 = static_cast<int>(tile % nN) * BN;
            for (int kb = 0; kb < nk; ++kb, ++q) {
                const int s = static_cast<int>(q % STAGES);
                const unsigned ph = static_cast<unsigned>((q / STAGES) & 1);
                if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1u, err)) { ok = false; break; }
                mbar_expect_tx(smem_u32(&full[s]), STAGE_BYTES);
                unsigned char *sa = smem + s * STAGE_BYTES;
                tma_load_2d(smem_u32(sa), &map_x, kb * BK, m0, smem_u32(&full[s]));
                tma_load_2d(smem_u32(sa + A_BYTES), &map_w, kb * BK, n0, smem_u32(&full[s]));
                *issued = static_cast<int>(q + 1);
            }
        }
        if (!ok) *err = 1;
    } else if (threadIdx.x == 32) {
        // MMA issuer: tile k into accumulator k & 1
        long long q = 0;
        bool ok = true;
        for (long long k = 0; k < my_n && ok; ++k) {
            const int a = static_cast<int>(k & 1);
            const unsigned acc = tmem + static_cast<unsigned>(a * BN);
            if (!mbar_wait(smem_u32(&acc_empty[a]), static_cast<unsigned>(((k >> 1) & 1) ^ 1), err)) {
                ok = false;
                break;
            }
            asm volatile("tcgen05.fence::after_thread_sync;");
            for (int kb = 0; kb < nk; ++kb, ++q) {
                const int s = static_cast<int>(q % STAGES);
                const unsigned ph = static_cast<unsigned>((q / STAGES) & 1);
                if (!mbar_wait(smem_u32(&full[s]), ph, err)) { ok = false; break; }
                asm volatile("tcgen05.fence::after_thread_sync;");
                const unsigned sa = smem_u32(smem + s * STAGE_BYTES);
                const unsigned sb = sa + A_BYTES;
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk) {
                    const unsigned long long da = sw128_desc(sa + kk * 32);
                    const unsigned long long db = sw128_desc(sb + kk * 32);
                    const unsigned en = (kb > 0 || kk > 0) ? 1u : 0u;
                    asm volatile(
                        "{\n\t.reg .pred p;\n\t"
                        "setp.ne.b32 p, %4, 0;\n\t"
                        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(acc),
                        "l"(da), "l"(db), "r"(kIdescBf16), "r"(en));
                }
                asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                    smem_u32(&empty[s])));
                *consumed = static_cast<int>(q + 1);
            }
            if (!ok) break;
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                smem_u32(&acc_full[a])));
        }
        if (!ok) *err = 1;
    } else if (warp >= 2) {
        // epilogue: thread = accumulator row of its warp's lane quarter
        const int quarter = warp & 3, lane = threadIdx.x & 31;
        const int row = quarter * 32 + lane;
        const int et = threadIdx.x - 64;  // 0 .. 127 among the epilogue threads
        unsigned out_q = 0;               // staging blocks handed to TMA so far
        for (long long k = 0; k < my_n; ++k) {
            const long long tile = blockIdx.x + k * gridDim.x;
            const int m0 = static_cast<int>(tile / nN) * BM, n0 = static_cast<int>(tile % nN) * BN;
            const int a = static_cast<int>(k & 1);
            bool bad = !mbar_wait(smem_u32(&acc_full[a]), static_cast<unsigned>((k >> 1) & 1), err) || *err;
            bad = epi_any(bad);  // one decision for the four epilogue warps
            asm volatile("tcgen05.fence::after_thread_sync;");
            if (bad) {
                // the products of this tile (and every later one) are lost: mark them
                for (long long kk = k; kk < my_n; ++kk) {
                    const long long tl = blockIdx.x + kk * gridDim.x;
                    const long long r = (tl / nN) * BM + row;
                    if (r < M)
                        for (int n = 0; n < BN; ++n)
                            Pout[r * static_cast<long long>(N) + (tl % nN) * BN + n] = __int_as_float(0x7fc00000);
                }
                break;
            }
#pragma unroll 1
            for (int cb = 0; cb < BN / 32; ++cb, ++out_q) {
                unsigned v[32];
                const unsigned taddr = tmem + (static_cast<unsigned>(quarter * 32) << 16) +
                                       static_cast<unsigned>(a * BN + cb * 32);
                asm volatile(
                    "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
                    "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
                    : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
                      "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
                      "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),
                      "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
                      "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),
                      "=r"(v[31])
                    : "r"(taddr));
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                if (cb == BN / 32 - 1) {
                    // every column of this accumulator is read: the next tile may use it
                    asm volatile("tcgen05.fence::before_thread_sync;");
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_u32(&acc_empty[a]));
                }
                // the staging block out_q % 2 is free once the store two blocks ago has read it
                if (et == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
                asm volatile("bar.sync 1, 128;" ::: "memory");
                unsigned char *blk = smem + OFF_OUT + (out_q & 1u) * OUT_BLOCK + row * 128;
#pragma unroll
                for (int j = 0; j < 8; ++j) {  // 16-byte chunk j of this row, swizzled
                    float4 o;
                    const int n = n0 + cb * 32 + j * 4;
                    o.x = __uint_as_float(v[4 * j + 0]) + __ldg(bias + n + 0);
                    o.y = __uint_as_float(v[4 * j + 1]) + __ldg(bias + n + 1);
                    o.z = __uint_as_float(v[4 * j + 2]) + __ldg(bias + n + 2);
                    o.w = __uint_as_float(v[4 * j + 3]) + __ldg(bias + n + 3);
                    *reinterpret_cast<float4 *>(blk + ((j ^ (row & 7)) << 4)) = o;
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (et == 0) {
                    tma_store_2d(&map_p, n0 + cb * 32, m0, smem_u32(smem + OFF_OUT + (out_q & 1u) * OUT_BLOCK));
                    asm volatile("cp.async.bulk.commit_group;");
                }
            }
        }
        if (et == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x == 0 && *err) {
        // a wait ran out: the copies issued but not consumed, and the last
        // products committed (their commit covers every earlier one), land first
        const int c = *consumed, i = *issued;
        for (int q = c; q < i; ++q) mbar_drain(smem_u32(&full[q % STAGES]), static_cast<unsigned>((q / STAGES) & 1));
        if (c > 0) mbar_drain(smem_u32(&empty[(c - 1) % STAGES]), static_cast<unsigned>(((c - 1) / STAGES) & 1));
    }
    asm volatile("tcgen05.fence::before_thread_sync;");
    __syncthreads();
    if (warp == 1) {
        asm volatile("tcgen05.fence::after_thread_sync;");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * BN));
    }
}

}  // namespace

// N output columns (gate rows x lanes), K = Din.
bool proj_tcgen05_supported(int x_dtype, int N, int K) {
    return x_dtype == PARARNN_BF16 && K % BK == 0 && N % BN == 0 && encode_fn() != nullptr;
}

cudaError_t launch_proj_tcgen05(const void *x, const void *w_ih, const float *b_ih, float *P, long long M, int N,
                                int K, cudaStream_t s) {
    CUtensorMap mx, mw, mp;
    if (!make_map(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, M, K, BK, BM) ||
        !make_map(&mw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w_ih, N, K, BK, BN) ||
        !make_map(&mp, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, P, M, N, 32, BM))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(proj_tcgen05_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    int dev = 0, nsm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    const long long tiles = ((M + BM - 1) / BM) * (N / BN);
    const long long grid = tiles < nsm ? tiles : nsm;
    proj_tcgen05_kernel<<<static_cast<unsigned>(grid), NTHR, SMEM_BYTES, s>>>(mx, mw, mp, b_ih, K, P, M, N);
    return cudaGetLastError();
}

}  // namespace pararnn

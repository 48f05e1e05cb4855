// proj_tcgen05.cu -- the input projection P = x W_ih^T + b_ih on the 5th-generation
// tensor cores (tcgen05, sm_100a), for bf16 operands.
//
// The input projection does not depend on the state, so one GEMM
// [B*T, Din] x [Din, 3D] serves every Newton iteration.  For the bf16 layer
// (Din = D = 2048) it is the one tensor-bound step of the solve (2*M*N*K flop).
//
// One CTA computes a 128 x 256 fp32 tile of P:
//   * TMA brings 128 x 64 tiles of x and 256 x 64 tiles of W_ih (bf16, 128-byte
//     swizzle) into a 4-stage shared-memory ring, signalled by mbarriers;
//   * one thread issues tcgen05.mma kind::f16 (bf16 x bf16 -> fp32, M=128,
//     N=256, K=16 per instruction) into a 256-column TMEM accumulator and
//     frees each stage with tcgen05.commit;
//   * after the last k-block, the four warps read the accumulator rows with
//     tcgen05.ld (thread = row), add the bias, stage 32-column blocks in
//     shared memory with the 128-byte swizzle, and TMA stores them.
// Every wait is bounded; a wait that runs out marks the tile and the epilogue
// writes NaN, which the solver reports as DIVERGED.
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
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;  // + alignment + barriers

// kind::f16 instruction descriptor: fp32 accumulate, bf16 A and B, both K-major.
constexpr unsigned kIdescBf16 = make_idesc(1u, BM, BN);

__global__ void __launch_bounds__(128, 1)
proj_tcgen05_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
                    const __grid_constant__ CUtensorMap map_p, const float *__restrict__ bias, int K,
                    float *__restrict__ Pout, long long M, int N) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    unsigned long long *bars = reinterpret_cast<unsigned long long *>(smem + STAGES * STAGE_BYTES);
    // bars[0..3] full, bars[4..7] empty, bars[8] done; then TMEM base address and error flag
    unsigned *tmem_slot = reinterpret_cast<unsigned *>(bars + 2 * STAGES + 1);
    volatile int *err = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *issued = reinterpret_cast<volatile int *>(tmem_slot + 2);    // TMA k-blocks issued
    volatile int *consumed = reinterpret_cast<volatile int *>(tmem_slot + 3);  // k-blocks given to MMA

    const int warp = threadIdx.x >> 5;
    const int m0 = blockIdx.x * BM, n0 = blockIdx.y * BN;
    const int nk = K / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&bars[s]), 1);
            mbar_init(smem_u32(&bars[STAGES + s]), 1);
        }
        mbar_init(smem_u32(&bars[2 * STAGES]), 1);
        *err = 0;
        *issued = 0;
        *consumed = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 2) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(BN));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    asm volatile("tcgen05.fence::before_thread_sync;");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;");
    const unsigned tmem = *tmem_slot;

    if (threadIdx.x == 0) {
        // TMA producer
        for (int kb = 0; kb < nk; ++kb) {
            const int s = kb % STAGES;
            const unsigned ph = (kb / STAGES) & 1u;
            if (!mbar_wait(smem_u32(&bars[STAGES + s]), ph ^ 1u, err)) break;
            const unsigned full = smem_u32(&bars[s]);
            mbar_expect_tx(full, STAGE_BYTES);
            unsigned char *sa = smem + s * STAGE_BYTES;
            tma_load_2d(smem_u32(sa), &map_x, kb * BK, m0, full);
            tma_load_2d(smem_u32(sa + A_BYTES), &map_w, kb * BK, n0, full);
            *issued = kb + 1;
        }
    } else if (threadIdx.x == 32) {
        // MMA issuer
        for (int kb = 0; kb < nk; ++kb) {
            const int s = kb % STAGES;
            const unsigned ph = (kb / STAGES) & 1u;
            if (!mbar_wait(smem_u32(&bars[s]), ph, err)) break;
            asm volatile("tcgen05.fence::after_thread_sync;");
            const unsigned sa = smem_u32(smem + s * STAGE_BYTES);
            const unsigned sb = sa + A_BYTES;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
                const unsigned long long da = sw128_desc(sa + kk * 32);
                const unsigned long long db = sw128_desc(sb + kk * 32);
                const unsigned acc = (kb > 0 || kk > 0) ? 1u : 0u;
                asm volatile(
                    "{\n\t.reg .pred p;\n\t"
                    "setp.ne.b32 p, %4, 0;\n\t"
                    "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem),
                    "l"(da), "l"(db), "r"(kIdescBf16), "r"(acc));
            }
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                smem_u32(&bars[STAGES + s])));
            *consumed = kb + 1;
        }
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(&bars[2 * STAGES])));
    }
    __syncwarp();

    // epilogue: thread = accumulator row
    const bool ok = mbar_wait(smem_u32(&bars[2 * STAGES]), 0u, err);
    asm volatile("tcgen05.fence::after_thread_sync;");
    __syncthreads();  // every stage is free now: reuse the ring as the output staging area
    const bool good = ok && !*err;
    const int row = threadIdx.x;
    if (!good) {
        // a wait ran out: drain the copies and products still in flight, then
        // mark this tile with NaN (no TMA store from a ring that may still change)
        if (threadIdx.x == 0) {
            for (int kb = *consumed; kb < *issued; ++kb)
                mbar_drain(smem_u32(&bars[kb % STAGES]), (kb / STAGES) & 1u);
            mbar_drain(smem_u32(&bars[2 * STAGES]), 0u);
        }
        __syncthreads();
        if (m0 + row < M)
            for (int n = n0; n < n0 + BN; ++n) Pout[(m0 + row) * static_cast<long long>(N) + n] = __int_as_float(0x7fc00000);
        asm volatile("tcgen05.fence::before_thread_sync;");
        __syncthreads();
        if (warp == 2) {
            asm volatile("tcgen05.fence::after_thread_sync;");
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(BN));
        }
        return;
    }
    unsigned char *stage = smem;  // 8 blocks of [128 rows x 128 B]
#pragma unroll 1
    for (int cb = 0; cb < BN / 32; ++cb) {
        unsigned v[32];
        const unsigned taddr = tmem + (static_cast<unsigned>(warp * 32) << 16) + cb * 32;
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
        unsigned char *blk = stage + cb * (BM * 128) + row * 128;
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
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;");
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int cb = 0; cb < BN / 32; ++cb)
            tma_store_2d(&map_p, n0 + cb * 32, m0, smem_u32(stage + cb * (BM * 128)));
        asm volatile("cp.async.bulk.commit_group;");
        asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
    }
    __syncthreads();
    if (warp == 2) {
        asm volatile("tcgen05.fence::after_thread_sync;");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(BN));
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
    const dim3 grid(static_cast<unsigned>((M + BM - 1) / BM), static_cast<unsigned>(N / BN));
    proj_tcgen05_kernel<<<grid, 128, SMEM_BYTES, s>>>(mx, mw, mp, b_ih, K, P, M, N);
    return cudaGetLastError();
}

}  // namespace pararnn

// tc_utils.cuh -- helpers for the 5th-generation tensor-core path (sm_100a):
// mbarriers, TMA tensor copies, UMMA shared-memory descriptors, and host-side
// tensor-map encoding through the driver entry point (no libcuda link needed).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace pararnn {
namespace tc {

constexpr long long kWaitBudget = 1ll << 22;

__device__ __forceinline__ unsigned smem_u32(const void *p) {
    return static_cast<unsigned>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(unsigned bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(unsigned bar, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(unsigned bar, unsigned parity) {
    unsigned done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
}
// Bounded wait that ignores the error flag (used to drain work in flight).
__device__ __forceinline__ void mbar_drain(unsigned bar, unsigned parity) {
    for (long long n = 0; n < kWaitBudget && !mbar_try_wait(bar, parity); ++n) {
    }
}
// Bounded wait; returns false (and sets *err) when the budget runs out.
__device__ __forceinline__ bool mbar_wait(unsigned bar, unsigned parity, volatile int *err) {
    long long n = 0;
    while (!mbar_try_wait(bar, parity)) {
        if (*err) return false;
        if (++n > kWaitBudget) {
            *err = 1;
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ void tma_load_2d(unsigned dst, const CUtensorMap *map, int c0, int c1,
                                            unsigned bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<unsigned long long>(map)), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, int c0, int c1, unsigned src) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                     reinterpret_cast<unsigned long long>(map)),
                 "r"(c0), "r"(c1), "r"(src)
                 : "memory");
}

// K-major operand tile with 128-byte swizzle: rows of 128 bytes, 8-row groups
// 1024 bytes apart (SBO), descriptor version 1, layout type 2 (SWIZZLE_128B).
__device__ __forceinline__ unsigned long long sw128_desc(unsigned addr) {
    unsigned long long d = 0;
    d |= static_cast<unsigned long long>((addr >> 4) & 0x3fffu);
    d |= static_cast<unsigned long long>(1u) << 16;           // LBO (unused with swizzle)
    d |= static_cast<unsigned long long>(1024u >> 4) << 32;   // SBO
    d |= static_cast<unsigned long long>(1u) << 46;           // version
    d |= static_cast<unsigned long long>(2u) << 61;           // SWIZZLE_128B
    return d;
}


// Instruction descriptor of tcgen05.mma (kind::f16 / kind::tf32): fp32
// accumulate, A and B K-major.  fmt: 1 = bf16, 2 = tf32.
__host__ __device__ constexpr unsigned make_idesc(unsigned fmt, int M, int N) {
    return (1u << 4) | (fmt << 7) | (fmt << 10) | (static_cast<unsigned>(N >> 3) << 17) |
           (static_cast<unsigned>(M >> 4) << 24);
}

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (fn == nullptr) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

inline bool make_map(CUtensorMap *m, CUtensorMapDataType dt, int esize, const void *base, long long rows,
              int cols, int box_cols, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * esize};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


}  // namespace tc
}  // namespace pararnn

// common.cuh -- device helpers shared by the parallel-Newton kernels (sm_100a).
//
// * Look-back descriptors for single-pass scans (decoupled look-back, Merrill &
//   Garland 2016).  A descriptor word packs a 32-bit tag and a 32-bit float in
//   one 64-bit word, written with st.release.gpu and read with ld.acquire.gpu,
//   so a reader never sees a value without its tag.  Tags carry an epoch (the
//   Newton iteration + 1, or 1 for a standalone scan) so descriptors need no
//   reset between iterations; the solver clears them once per call.
// * A bounded grid barrier for persistent cooperative kernels.
// * Bounded spins: every wait gives up after a fixed budget, records
//   PARARNN_TIMEOUT in a device status word and returns; once that word is set
//   every other wait returns at once, so a lost publisher can never hang the GPU.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace pararnn {

constexpr int kThreads = 256;            // threads per CTA of the scan kernels
constexpr unsigned kStateAgg = 1u;       // descriptor holds a tile aggregate
constexpr unsigned kStateInc = 2u;       // descriptor holds an inclusive value
constexpr unsigned kStatusTimeout = 1u;  // bit in the device status word
constexpr long long kSpinBudget = 1ll << 24;  // ~2-4 s with the back-off below

__host__ __device__ inline unsigned make_tag(unsigned epoch, unsigned state) {
    return (epoch << 2) | state;
}

__device__ __forceinline__ unsigned long long pack_word(unsigned tag, float v) {
    return (static_cast<unsigned long long>(tag) << 32) | __float_as_uint(v);
}
__device__ __forceinline__ unsigned word_tag(unsigned long long w) {
    return static_cast<unsigned>(w >> 32);
}
__device__ __forceinline__ float word_val(unsigned long long w) {
    return __uint_as_float(static_cast<unsigned>(w & 0xffffffffull));
}

__device__ __forceinline__ void st_release(unsigned long long *p, unsigned long long v) {
    asm volatile("st.release.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ void st_relaxed(unsigned long long *p, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long ld_acquire(const unsigned long long *p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ unsigned long long ld_relaxed(const unsigned long long *p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_u32(unsigned *p, unsigned v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ bool timed_out(const unsigned *status) {
    return (ld_acquire_u32(status) & kStatusTimeout) != 0u;
}
__device__ __forceinline__ void flag_timeout(unsigned *status) {
    atomicOr(status, kStatusTimeout);
}

// Spin until the word at p carries `epoch` in state >= kStateAgg.  Returns the
// word, or 0 after recording a timeout.
__device__ __forceinline__ unsigned long long wait_word(const unsigned long long *p,
                                                        unsigned epoch, unsigned *status) {
    long long spins = 0;
    while (true) {
        unsigned long long w = ld_acquire(p);
        if ((word_tag(w) >> 2) == epoch && (word_tag(w) & 3u) != 0u) return w;
        if (++spins > 64) {
            if ((spins & 1023) == 0 && timed_out(status)) return 0ull;
            if (spins > kSpinBudget) {
                flag_timeout(status);
                return 0ull;
            }
            __nanosleep(32);
        }
    }
}

// Grid-wide barrier for a cooperative launch (all CTAs co-resident).
// bar[0] counts arrivals, bar[1] is the generation.  Bounded.
__device__ __forceinline__ void grid_barrier(unsigned *bar, unsigned nblocks, unsigned *status) {
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned gen = ld_acquire_u32(&bar[1]);
        __threadfence();
        const unsigned arrived = atomicAdd(&bar[0], 1u);
        if (arrived == nblocks - 1) {
            atomicExch(&bar[0], 0u);
            __threadfence();
            st_release_u32(&bar[1], gen + 1u);
        } else {
            long long spins = 0;
            while (ld_acquire_u32(&bar[1]) == gen) {
                if (++spins > 64) {
                    if ((spins & 1023) == 0 && timed_out(status)) break;
                    if (spins > kSpinBudget) {
                        flag_timeout(status);
                        break;
                    }
                    __nanosleep(64);
                }
            }
        }
        __threadfence();
    }
    __syncthreads();
}

// ---- math -----------------------------------------------------------------
// Logistic sigmoid and tanh from the CUDA exponential intrinsic.  Absolute
// error ~1e-7, far inside the 1e-4 state tolerance; tanh uses the identity
// tanh(v) = 1 - 2 / (exp(2v) + 1), which saturates correctly for large |v|.
__device__ __forceinline__ float sigmoidf_(float v) {
    return __fdividef(1.0f, 1.0f + __expf(-v));
}
__device__ __forceinline__ float tanhf_(float v) {
    return 1.0f - __fdividef(2.0f, __expf(2.0f * v) + 1.0f);
}

// One GRU state (gate order r, z, n; reset gate applied after the recurrent
// bias) and the diagonal of its Jacobian with respect to the previous state.
//   pr, pz, pn   input pre-activations (W x + b_ih) of the lane
//   gr, gz, gnh  recurrent sums U_g h (or u_g * h for the diagonal cell)
//   bh*          recurrent biases b_hh;  ud*: diagonal entries of U_g
//   h            the previous state h_{t-1}
// Returns f = f(h, x), a = df/dh (diagonal entry) and bb = f - a h.
//   a = z + (h - n) z (1 - z) U_z + (1 - z)(1 - n^2) r U_n
//         + (1 - z)(1 - n^2) g r (1 - r) U_r          (diagonal entries)
__device__ __forceinline__ void gru_cell_diag(float pr, float pz, float pn, float gr, float gz,
                                              float gnh, float bhr, float bhz, float bhn, float udr,
                                              float udz, float udn, float h, float &f, float &a,
                                              float &bb) {
    const float r = sigmoidf_(pr + gr + bhr);
    const float z = sigmoidf_(pz + gz + bhz);
    const float gn = gnh + bhn;
    const float n = tanhf_(pn + r * gn);
    f = n + z * (h - n);
    const float omz = 1.f - z;
    const float cz = (h - n) * z * omz;
    const float cn = omz * (1.f - n * n) * r;
    const float cr = cn * gn * (1.f - r);
    a = z + cz * udz + cn * udn + cr * udr;
    bb = f - a * h;
}

// ---- two cells at once on the fp32x2 datapath (sm_100):
// add / sub / mul / fma .f32x2 round each half exactly like the fp32
// instruction, so results equal the one-lane form bit for bit up to the
// order of operations; exp and reciprocal stay per lane (ex2.approx,
// rcp.approx, as in the one-lane form).
using u64 = unsigned long long;
__device__ __forceinline__ u64 pk(float a, float b) {
    u64 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void upk(u64 r, float &a, float &b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ u64 add2(u64 a, u64 b) {
    u64 d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ u64 sub2(u64 a, u64 b) {
    u64 d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ u64 mul2(u64 a, u64 b) {
    u64 d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ u64 fma2(u64 a, u64 b, u64 c) {
    u64 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ u64 ex2_2(u64 v) {  // 2^v per lane
    float a, b;
    upk(v, a, b);
    asm("ex2.approx.ftz.f32 %0, %0;" : "+f"(a));
    asm("ex2.approx.ftz.f32 %0, %0;" : "+f"(b));
    return pk(a, b);
}
__device__ __forceinline__ u64 rcp2(u64 v) {  // 1 / v per lane
    float a, b;
    upk(v, a, b);
    asm("rcp.approx.ftz.f32 %0, %0;" : "+f"(a));
    asm("rcp.approx.ftz.f32 %0, %0;" : "+f"(b));
    return pk(a, b);
}
__device__ __forceinline__ u64 splat(float v) { return pk(v, v); }

constexpr float kLog2eF = 1.4426950408889634f;

// gru_cell_diag for two lanes: the gates r = 1 / (1 + 2^(-v log2 e)), likewise z,
// n = tanh(u) = 1 - 2 / (2^(2 u log2 e) + 1); f = n + z (h - n); the Jacobian
// diagonal a = z + (h - n) z (1 - z) U_z + (1 - z)(1 - n^2) r U_n
// + (1 - z)(1 - n^2)(U_n h + b_hn) r (1 - r) U_r; bb = f - a h.  bhr and bhz
// come premultiplied by -log2(e): -v log2 e = (p + g) (-log2 e) + bh (-log2 e).
__device__ __forceinline__ void gru_cell_diag_x2(u64 pr, u64 pz, u64 pn, u64 gr, u64 gz, u64 gnh,
                                                 u64 bhr, u64 bhz, u64 bhn, u64 udr, u64 udz, u64 udn,
                                                 u64 h, u64 &f, u64 &a, u64 &bb) {
    const u64 one = splat(1.f);
    const u64 r = rcp2(add2(ex2_2(fma2(add2(pr, gr), splat(-kLog2eF), bhr)), one));
    const u64 z = rcp2(add2(ex2_2(fma2(add2(pz, gz), splat(-kLog2eF), bhz)), one));
    const u64 gn = add2(gnh, bhn);
    const u64 en = ex2_2(mul2(fma2(r, gn, pn), splat(2.f * kLog2eF)));
    const u64 n = fma2(splat(-2.f), rcp2(add2(en, one)), one);
    const u64 hmn = sub2(h, n);
    f = fma2(z, hmn, n);
    const u64 omz = sub2(one, z);
    const u64 cz = mul2(mul2(hmn, z), omz);
    const u64 m = mul2(mul2(omz, fma2(n, n, splat(-1.f))), r);  // -(1 - z)(1 - n^2) r
    const u64 mr = mul2(mul2(m, gn), sub2(one, r));                // -(cell's U_r coefficient)
    a = sub2(fma2(cz, udz, z), fma2(mr, udr, mul2(m, udn)));
    bb = sub2(f, mul2(a, h));
}

// |x| as an unsigned bit pattern: ordered like the float for x >= 0, and any
// NaN or Inf maps above every finite value (0x7f800000 and up), so an integer
// max over patterns both finds the largest |dh| and flags non-finite values.
__device__ __forceinline__ unsigned abs_bits(float x) {
    return __float_as_uint(fabsf(x));
}

__device__ __forceinline__ unsigned warp_max_u32(unsigned v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Block-wide max of an unsigned (kThreads threads); result valid in thread 0.
__device__ __forceinline__ unsigned block_max_u32(unsigned v, unsigned *red /*[32]*/) {
    v = warp_max_u32(v);
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    __syncthreads();
    if (lane == 0) red[wid] = v;
    __syncthreads();
    unsigned r = 0;
    if (threadIdx.x < 32) {
        r = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0u;
        r = warp_max_u32(r);
    }
    return r;
}

// (c0, c1) += (a0, a1) * h as one packed fp32x2 FMA (sm_100 f32x2 datapath:
// the same fp32 rounding as two FFMAs, half the issued instructions).
__device__ __forceinline__ void ffma2(float &c0, float &c1, float a0, float a1, float h) {
    asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
        "mov.b64 ra, {%2, %3};\n\t"
        "mov.b64 rb, {%4, %4};\n\t"
        "mov.b64 rc, {%0, %1};\n\t"
        "fma.rn.f32x2 rc, ra, rb, rc;\n\t"
        "mov.b64 {%0, %1}, rc;\n\t}"
        : "+f"(c0), "+f"(c1)
        : "f"(a0), "f"(a1), "f"(h));
}

__device__ __forceinline__ float4 ldcg4(const float *p) {
    return __ldcg(reinterpret_cast<const float4 *>(p));
}
__device__ __forceinline__ void stcg4(float *p, float4 v) {
    __stcg(reinterpret_cast<float4 *>(p), v);
}
__device__ __forceinline__ float get(const float4 &v, int j) {
    return j == 0 ? v.x : (j == 1 ? v.y : (j == 2 ? v.z : v.w));
}
__device__ __forceinline__ void set(float4 &v, int j, float x) {
    if (j == 0) v.x = x; else if (j == 1) v.y = x; else if (j == 2) v.z = x; else v.w = x;
}

}  // namespace pararnn

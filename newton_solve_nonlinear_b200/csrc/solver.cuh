// solver.cuh -- internal interface between the C ABI and the solver kernels.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/pararnn.h"

namespace pararnn {

// Device-side header at the start of every workspace (256 bytes).
struct WsHeader {
    unsigned barrier[2];     // grid barrier: arrivals, generation
    unsigned status;         // kStatusTimeout bit
    unsigned delta_bits[3];  // per-iteration max |dh| (rotating slots)
    unsigned resid_bits[3];  // per-iteration max |residual|
    unsigned pad0[7];
    pararnn_info info;       // report of the last solve
    unsigned long long ticket;  // tile ticket of standalone (non-cooperative) scans
    unsigned pad1[38];
};
static_assert(sizeof(WsHeader) <= 256, "header must fit 256 bytes");

// Tiling of the [B, T, D] state array into (sequence, lane-group, chunk) tiles.
struct Tiling {
    int DG;         // lanes (state components) per tile, multiple of 4, <= 64
    int DB;         // float4 columns per tile row = DG / 4
    int NTB;        // thread rows (t-blocks) per tile = kThreads / DB
    int TK;         // time steps per thread
    int L;          // time steps per tile = NTB * TK
    int n_dgroups;  // ceil(D / DG)
    int n_groups;   // B * n_dgroups
    int n_chunks;   // ceil(T / L)
    long long n_tiles;
};

// Tiling of the state array.  The solver kernels take two steps per thread
// (kSolverTK): that keeps the per-thread state -- 3 x TK x 4 recurrent sums for
// the dense cell, the TK x 4 scan operands -- inside the register budget of
// two CTAs per SM.  The standalone scan holds only a and b and takes four.
constexpr int kSolverTK = 2;
Tiling make_tiling(int B, int T, int D, bool dense_cell, int TK);

// Arguments of the persistent diagonal-Jacobian solver kernels.
struct DiagArgs {
    int B, T, D;
    const float *P;      // [B, T, 3D] input pre-activations (b_ih included)
    const float *w_hh;   // dense [3D, D] or diag [3D]
    const float *b_hh;   // [3D]
    const float *h0;     // [B, D]
    float *hbuf[2];      // iterate ping-pong; hbuf[1] is the caller's output
    float lambda, tol;
    int max_iters;
    Tiling tl;
    unsigned long long *desc;  // look-back descriptors
    float *elk_m, *elk_p, *elk_a, *elk_b;  // quasi-ELK forward results [B, T, D]
    WsHeader *hdr;
    pararnn_info *info_out;  // device report destination
    int warm;                // hbuf[0] holds a caller's initial guess (else the guess is zero)
    int jac_every;           // Jacobian refreshed every jac_every iterations (<= 1: every one)
    float *coef;             // frozen Jacobian coefficients while jac_every > 1
    float *trace;            // optional [trace_len][2]: max |dh| and max |r| of every iteration
    int trace_len;
    long long withhold;      // testing hook: this tile never publishes in the first iteration (-1: none)
};

// Iteration `it`'s convergence maxima into the optional trace (one thread).
__device__ __forceinline__ void record_trace(const DiagArgs &A, int it, unsigned dbits, unsigned rbits) {
    if (A.trace != nullptr && it < A.trace_len && blockIdx.x == 0 && threadIdx.x == 0) {
        A.trace[2 * it] = __uint_as_float(dbits);
        A.trace[2 * it + 1] = __uint_as_float(rbits);
    }
}

// Whether a tile publishes its look-back descriptors in iteration epoch - 1.
__device__ __forceinline__ bool publishes(const DiagArgs &A, long long tile, unsigned epoch) {
    return epoch != 1u || tile != A.withhold;
}

// Workspace carve-up shared by the size query and the solver.
struct WsLayout {
    size_t header, P, hbuf, desc, elk, dense, total;
};
WsLayout ws_layout(const pararnn_cell &cell, int B, int T, int mode);

// Kernel launchers (return a cudaError_t).
cudaError_t launch_projection_n(int x_dtype, const void *x, const void *w_ih, const float *b_ih, float *P,
                                long long M, int N, int K, cudaStream_t s);
cudaError_t launch_projection(const pararnn_cell &cell, const void *x, const void *w_ih,
                              const float *b_ih, float *P, long long M, cudaStream_t s);
cudaError_t launch_diag_solver(const pararnn_cell &cell, int mode, const DiagArgs &a,
                               cudaStream_t s);
cudaError_t launch_scan_diag(const float *A, const float *b, const float *h0, int B, int T,
                             int D, float *h, void *ws, cudaStream_t s);

}  // namespace pararnn

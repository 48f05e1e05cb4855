/*
 * pararnn.h -- C ABI of the parallel-Newton GRU evaluator for NVIDIA B200 (sm_100a).
 *
 * The library evaluates a nonlinear recurrence h_t = f(h_{t-1}, x_t) (a GRU
 * cell) over a whole sequence at once.  All T states are treated as the
 * unknowns of one system of nonlinear equations, one per step, and solved
 * with Newton iterations; each iteration solves the linearised, block
 * bidiagonal system h_t = A_t h_{t-1} + b_t with a parallel scan over t.
 *   - "ParaRNN: A Revolutionary Framework for Parallel Training of Nonlinear
 *     RNNs", sections "Core Idea" and "Newton's Iteration";
 *   - "Towards Scalable and Stable Parallelization of Nonlinear RNNs",
 *     abstract (DEER as a fixed-point problem, quasi-Newton, ELK) and the atlas
 *     summary, "Approach" (diagonal Jacobian; Levenberg-Marquardt step as a
 *     parallel Kalman filter/smoother);
 *   - "Parallelizing non-linear sequential models over the sequence length",
 *     abstract (DEER).
 *
 * Conventions for every entry point
 *   - Device pointers are CUDA device addresses of the current device; host
 *     pointers are ordinary host memory.  Each argument says which it is.
 *   - Arrays are dense, row-major and contiguous; device arrays start on a
 *     16-byte boundary.
 *   - The caller owns all memory, including the workspace.  The library
 *     allocates no device or host memory.  The host-buffer calls (the
 *     *_host entry points) keep two helper streams and their events per device
 *     (one set per call running at a time), created on first use and reused
 *     until the process exits; nothing else persists between calls.
 *   - Work is enqueued on `stream` (NULL means the legacy default stream).
 *   - Return value: a pararnn_status code; pararnn_status_string() names it.
 *     On PARARNN_INVALID_ARG nothing was enqueued.
 */
#ifndef PARARNN_H
#define PARARNN_H

#include <stddef.h>

#if defined(__GNUC__)
#define PARARNN_API __attribute__((visibility("default")))
#else
#define PARARNN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t.  Declared here so that the header needs no CUDA include. */
struct CUstream_st;
typedef struct CUstream_st *pararnn_stream;

/* Solver modes ("Towards Scalable and Stable Parallelization of Nonlinear
 * RNNs": abstract; atlas summary "Approach").
 *   DEER      Newton with the full D x D Jacobian of the cell.
 *   QUASI     quasi-DEER: the Jacobian replaced by its diagonal.
 *   ELK       Newton with a Levenberg-Marquardt trust region, the damped step
 *             computed as a Kalman filter + smoother (full Jacobian).
 *   QUASI_ELK ELK with the diagonal Jacobian. */
typedef enum {
    PARARNN_DEER = 0,
    PARARNN_QUASI = 1,
    PARARNN_ELK = 2,
    PARARNN_QUASI_ELK = 3
} pararnn_mode;

/* Cell kinds.  DENSE: the GRU with full recurrent matrices U_r, U_z, U_n.
 * DIAG: the recurrent weights are elementwise vectors u_r, u_z, u_n, so the
 * Jacobian is exactly diagonal and QUASI is exact Newton (the "adapted" GRU of
 * the ParaRNN abstract). */
typedef enum { PARARNN_GRU_DENSE = 0, PARARNN_GRU_DIAG = 1, PARARNN_LSTM_DIAG = 2 } pararnn_cell_kind;

typedef enum { PARARNN_F32 = 0, PARARNN_BF16 = 1 } pararnn_dtype;

typedef enum {
    PARARNN_OK = 0,             /* converged: max |h^(i+1) - h^(i)| <= tol        */
    PARARNN_NOT_CONVERGED = 1,  /* max_iters reached; h holds the last iterate    */
    PARARNN_DIVERGED = 2,       /* a non-finite value appeared; h holds that iterate */
    PARARNN_INVALID_ARG = 3,    /* bad pointer, size, alignment, mode or workspace */
    PARARNN_CUDA_ERROR = 4,     /* a CUDA runtime call failed                      */
    PARARNN_TIMEOUT = 5         /* a bounded device-side wait expired (h unreliable) */
} pararnn_status;

/* The GRU cell.
 *   din, d     input and state widths.  d must be a multiple of 4.
 *   x_dtype    element type of x; w_dtype that of w_ih.  Both F32, or both BF16.
 * Gates (rows of every [3D, .] array in the order r, z, n):
 *   r = sigmoid(W_r x + b_ir + U_r h + b_hr),  z = sigmoid(W_z x + b_iz + U_z h + b_hz),
 *   n = tanh(W_n x + b_in + r * (U_n h + b_hn)),  f = (1 - z) * n + z * h.          */
typedef struct {
    int kind;     /* pararnn_cell_kind */
    int din;
    int d;
    int x_dtype;  /* pararnn_dtype */
    int w_dtype;  /* pararnn_dtype */
} pararnn_cell;

/* Cell parameters, all DEVICE pointers.
 *   w_ih  [3D, Din]  of w_dtype
 *   b_ih  [3D]       float
 *   w_hh  DENSE: [3D, D] float (U_r; U_z; U_n stacked by rows)
 *         DIAG:  [3D]    float (u_r, u_z, u_n)
 *   b_hh  [3D]       float                                                    */
typedef struct {
    const void *w_ih;
    const float *b_ih;
    const float *w_hh;
    const float *b_hh;
} pararnn_params;

/* Per-solve report, written to DEVICE memory by pararnn_newton_solve_async
 * (and copied to the host by pararnn_newton_solve). */
typedef struct {
    int iters;          /* linear solves performed                                */
    int status;         /* PARARNN_OK / NOT_CONVERGED / DIVERGED / TIMEOUT        */
    float delta;        /* max |h^(iters) - h^(iters-1)|                           */
    float residual;     /* max |h_t - f(h_{t-1}, x_t)| at the last linearisation   */
} pararnn_info;

/*
 * pararnn_workspace_size -- bytes of device workspace pararnn_newton_solve needs.
 * Returns 0 for arguments pararnn_newton_solve would reject.
 */
PARARNN_API size_t pararnn_workspace_size(const pararnn_cell *cell, int B, int T, int mode);

/*
 * pararnn_newton_solve -- evaluate the GRU over B sequences of length T by
 * (quasi-)Newton / (quasi-)ELK iterations, and wait for the result.
 *
 * Method ("ParaRNN" summary, "Core Idea" and "Newton's Iteration";
 * "Towards Scalable and Stable Parallelization of Nonlinear RNNs", abstract
 * and atlas summary "Approach"):
 *   unknowns h_1..h_T per sequence, residual r_t = h_t - f(h_{t-1}, x_t),
 *   h_0 = h0 fixed; initial guess h^(0) = 0.
 *   Iteration i linearises f at the shifted guess h^(i)_{t-1}:
 *     A_t = df/dh (DEER, ELK) or its diagonal (QUASI, QUASI_ELK),
 *     b_t = f(h^(i)_{t-1}, x_t) - A_t h^(i)_{t-1};
 *   DEER / QUASI:   h^(i+1) solves h_t = A_t h_{t-1} + b_t (parallel scan);
 *   ELK / QUASI_ELK: h^(i+1) minimises
 *       sum_t |h_t - A_t h_{t-1} - b_t|^2 + lambda sum_t |h_t - h^(i)_t|^2
 *     (Kalman filter + RTS smoother with process noise I, observation noise
 *     I / lambda, observations h^(i)).  QUASI_ELK runs that smoother as
 *     scans; ELK on the DENSE cell solves the same minimiser from its
 *     block-tridiagonal normal equations by block cyclic reduction.
 *   Stop when delta = max_{b,t,d} |h^(i+1) - h^(i)| <= tol (iters = i + 1),
 *   when a value is non-finite (DIVERGED), or after max_iters iterations.
 *
 * Arguments
 *   cell, params   the GRU (host struct; params holds device pointers).
 *   x              DEVICE [B, T, Din] of cell->x_dtype; x[:, 0] is x_1.
 *   h0             DEVICE [B, D] float.
 *   B, T           batch and sequence length, B >= 1, T >= 1.
 *   mode           pararnn_mode.  The DIAG cell has a diagonal Jacobian, so
 *                  DEER equals QUASI and ELK equals QUASI_ELK for it.
 *   lambda         LM damping (> 0) for ELK / QUASI_ELK; ignored otherwise.
 *   tol            convergence threshold on max |dh| (>= 0).
 *   max_iters      iteration cap; <= 0 means T + 1 (undamped Newton is exact
 *                  after T iterations; one more observes delta = 0).
 *   h              DEVICE [B, T, D] float, output (the final iterate; h[:, t]
 *                  is h_{t+1}).  Must not alias any input or the workspace.
 *   info           HOST pararnn_info, output; may be NULL.
 *   workspace      DEVICE, at least pararnn_workspace_size(cell, B, T, mode)
 *                  bytes, 256-byte aligned, not used by anything else while the
 *                  solve runs.  Its contents on entry do not matter.
 *   stream         stream to enqueue on.  The call synchronises this stream
 *                  once, at the end, to read the report.
 * Returns pararnn_status (the solve's own status, or INVALID_ARG / CUDA_ERROR).
 * Limits: DENSE cells need d <= 64 (recurrent matrices are kept on chip).
 * ELK on the DENSE cell keeps three D x D matrices per step in the workspace
 * (D rounded up to 8, 16, 32 or 64): about 3 * B * T * D^2 * 4 bytes.
 */
PARARNN_API int pararnn_newton_solve(const pararnn_cell *cell, const pararnn_params *params,
                         const void *x, const float *h0, int B, int T, int mode,
                         float lambda, float tol, int max_iters, float *h,
                         pararnn_info *info, void *workspace, size_t ws_bytes,
                         pararnn_stream stream);

/*
 * pararnn_newton_solve_async -- the same solve without any host synchronisation.
 * The report is written to `info_dev` (DEVICE pararnn_info) when the last
 * kernel finishes.  Returns PARARNN_OK if everything was enqueued (the solve's
 * own status is info_dev->status), else INVALID_ARG / CUDA_ERROR.
 */
PARARNN_API int pararnn_newton_solve_async(const pararnn_cell *cell, const pararnn_params *params,
                               const void *x, const float *h0, int B, int T, int mode,
                               float lambda, float tol, int max_iters, float *h,
                               pararnn_info *info_dev, void *workspace, size_t ws_bytes,
                               pararnn_stream stream);

/*
 * pararnn_newton_solve_guess_async -- pararnn_newton_solve_async started from a
 * caller's initial guess instead of zero (a warm start: the previous epoch's
 * states, or a nearby solution).  The pages leave the starting guess open
 * (the zero-start solve's choice is a reading); starting elsewhere changes only
 * where the iteration begins: the fixed point, the convergence test and every
 * other argument are those of the zero-start solve.
 *   h_init  DEVICE float [B, T, D], 16-byte aligned, read once before the first
 *           iteration; it may be `h` itself (the solve then updates h in place).
 * Asynchronous; the report goes to info_dev.
 */
PARARNN_API int pararnn_newton_solve_guess_async(const pararnn_cell *cell, const pararnn_params *params,
                                                 const void *x, const float *h0, const float *h_init, int B,
                                                 int T, int mode, float lambda, float tol, int max_iters,
                                                 float *h, pararnn_info *info_dev, void *workspace,
                                                 size_t ws_bytes, pararnn_stream stream);

/*
 * pararnn_newton_solve_trace -- pararnn_newton_solve that also records every
 * iteration's convergence maxima, so a caller can follow the whole trajectory
 * of the stopping test rather than its last value: the per-iteration max|dh|
 * whose first value <= tol ends the solve ("ParaRNN" summary, "Newton's
 * Iteration"; "Towards Scalable and Stable Parallelization of Nonlinear RNNs",
 * atlas summary "Limitations": the quasi methods take more iterations).
 *   trace      DEVICE float [trace_len][2], 8-byte aligned, not overlapping h
 *              or the workspace: trace[i][0] = max_{b,t,d} |h^(i+1) - h^(i)|,
 *              trace[i][1] = max |h^(i)_t - f(h^(i)_{t-1}, x_t)| at iteration
 *              i's linearisation point, for i < min(iters, trace_len); later
 *              entries are left untouched.
 *   trace_len  >= 1.
 * Other arguments, the stopping rule and the return value as
 * pararnn_newton_solve (synchronises `stream` once).
 */
PARARNN_API int pararnn_newton_solve_trace(const pararnn_cell *cell, const pararnn_params *params,
                                           const void *x, const float *h0, int B, int T, int mode,
                                           float lambda, float tol, int max_iters, float *h,
                                           pararnn_info *info, float *trace, int trace_len,
                                           void *workspace, size_t ws_bytes, pararnn_stream stream);

/*
 * pararnn_test_withheld_publish -- a testing hook for the bounded device-side
 * waits (no counterpart on the pages).  It runs pararnn_newton_solve (tol,
 * max_iters = T + 1) with one change: in the first iteration, look-back tile
 * `tile` of the single-pass scan never publishes its descriptors, so every
 * later tile of its lanes waits for a value that never arrives.  Those waits
 * give up after their fixed spin budget (seconds), raise the workspace's
 * timeout flag, and every CTA then leaves its waits and the grid barrier: the
 * call returns PARARNN_TIMEOUT, h is unreliable, and the workspace is fit for
 * the next solve (its header is rewritten by every solve).
 * Taken by two paths only: the dense cell with d = 32 or 64 in mode QUASI (the
 * tensor-core kernel; tiles of 128 steps x all lanes, chunk-major: tile =
 * chunk * B + b), and the diagonal cell with d % 64 == 0 in mode DEER or QUASI
 * (tiles of 32 steps x 64 lanes).  Other arguments, or a tile beyond the
 * path's tile count, give PARARNN_INVALID_ARG.  Synchronises `stream`.
 */
PARARNN_API int pararnn_test_withheld_publish(const pararnn_cell *cell, const pararnn_params *params,
                                              const void *x, const float *h0, int B, int T, int mode,
                                              float tol, float *h, pararnn_info *info, long long tile,
                                              void *workspace, size_t ws_bytes, pararnn_stream stream);

/*
 * pararnn_newton_solve_reuse -- DEER on the dense cell with the Jacobian reused:
 * recomputed only every jac_every iterations, an approximate Newton strategy
 * the pages name for cost at scale ("ParaRNN" summary, "Newton's Iteration").
 * Iteration i linearises with the J_t of iteration jac_every * floor(i /
 * jac_every) and the residual of its own guess:
 *   h^(i+1)_t = J^(i0)_t h^(i+1)_{t-1} + f(h^(i)_{t-1}, x_t) - J^(i0)_t h^(i)_{t-1},
 * so the fixed point is the one of DEER, and after i iterations the first i
 * states are exact (the T + 1 cap holds); in between refreshes convergence is
 * linear instead of quadratic.  On this path an iteration that reuses the
 * Jacobian also reuses the scan's matrix products (the chunk and group
 * aggregates of J), so it costs O(D^2) per step instead of O(D^3).
 *   jac_every  >= 1 (1: plain DEER).  Other arguments as pararnn_newton_solve
 *              with mode DEER; the cell: PARARNN_GRU_DENSE, d <= 32.
 *   workspace  pararnn_reuse_workspace_size bytes (the DEER workspace plus
 *              512 bytes per step of B*T for the frozen coefficients).
 * Synchronises `stream` once; returns the solve's status, or INVALID_ARG /
 * CUDA_ERROR.
 */
PARARNN_API int pararnn_newton_solve_reuse(const pararnn_cell *cell, const pararnn_params *params,
                                           const void *x, const float *h0, int B, int T, int jac_every,
                                           float tol, int max_iters, float *h, pararnn_info *info,
                                           void *workspace, size_t ws_bytes, pararnn_stream stream);

/* pararnn_reuse_workspace_size -- bytes pararnn_newton_solve_reuse needs, or 0
 * for arguments it rejects (not the dense cell with d <= 32). */
PARARNN_API size_t pararnn_reuse_workspace_size(const pararnn_cell *cell, int B, int T);

/*
 * pararnn_newton_solve_chunked -- the solve over consecutive time chunks of at
 * most t_chunk steps, one after another, each started from the last state the
 * previous chunk reached: device memory grows with t_chunk instead of T (for
 * sequences too long for one solve's workspace; the ParaRNN summary page,
 * "Experimental Results", names chunking as the remedy for the Newton
 * iteration's hidden-state memory).  Each chunk is an independent
 * solve to `tol`; for contractive cells the joined states match the
 * one-shot solve to within the propagated tolerance.  Arguments as for
 * pararnn_newton_solve, plus t_chunk >= 1 (max_iters <= 0 caps every chunk at
 * T + 1 of the whole sequence); the workspace is
 * pararnn_chunked_workspace_size bytes.  The report: iterations summed over
 * the chunks, the worst status, the largest delta and residual.  Synchronises
 * `stream` once, at the end.
 */
PARARNN_API int pararnn_newton_solve_chunked(const pararnn_cell *cell, const pararnn_params *params,
                                             const void *x, const float *h0, int B, int T, int t_chunk,
                                             int mode, float lambda, float tol, int max_iters, float *h,
                                             pararnn_info *info, void *workspace, size_t ws_bytes,
                                             pararnn_stream stream);

/* pararnn_chunked_workspace_size -- bytes pararnn_newton_solve_chunked needs
 * (one chunk's solve workspace plus staging for one chunk), or 0. */
PARARNN_API size_t pararnn_chunked_workspace_size(const pararnn_cell *cell, int B, int T, int t_chunk,
                                                  int mode);

/*
 * pararnn_newton_solve_host -- the same evaluation from and to HOST memory,
 * with the copies overlapped with the computation.
 *
 * The B sequences are independent, so the batch is solved in `parts`
 * consecutive parts.  Their sizes ramp, because the first part's copy in and
 * the last part's copy out overlap no solve while a solve's cost per sequence
 * falls as the part grows: part p has weight min(p + 1, parts - p, 4)
 * (1, 2, 3, 4, ..., 4, 3, 2, 1), rounded by largest remainder, at least one
 * sequence each (B = 16 in 7 parts: 1, 2, 3, 4, 3, 2, 1).
 * While part p is solved on `stream`, part p+1's inputs are copied in and
 * part p-1's states copied out on two helper streams (kept per device and
 * reused by later calls);
 * the device staging holds three parts' inputs and outputs in the workspace
 * (with two, a part's input copy would wait for the output copy two parts
 * earlier, and copies slower than the solve would set the pace).  Each part is an
 * independent solve to `tol` (its own convergence test), so a part may take
 * fewer iterations than the whole batch would.
 *
 * Arguments as for pararnn_newton_solve, except:
 *   x_host     HOST [B, T, Din] of cell->x_dtype (page-locked memory lets the
 *              copies run asynchronously; pageable memory is accepted).
 *   h0_host    HOST [B, D] float.
 *   h_host     HOST [B, T, D] float, output.
 *   info       HOST, output, may be NULL: the worst part (largest iters,
 *              status, delta and residual over the parts).
 *   parts      1 <= parts <= B.
 *   workspace  DEVICE, at least pararnn_host_workspace_size(cell, B, T, mode,
 *              parts) bytes, 256-byte aligned.
 *   stream     work on `stream` queued before the call runs first; on return
 *              everything has completed (the call synchronises `stream`).
 * Returns the worst part's status, or INVALID_ARG / CUDA_ERROR.
 */
PARARNN_API int pararnn_newton_solve_host(const pararnn_cell *cell, const pararnn_params *params,
                              const void *x_host, const float *h0_host, int B, int T, int mode,
                              float lambda, float tol, int max_iters, float *h_host,
                              pararnn_info *info, int parts, void *workspace, size_t ws_bytes,
                              pararnn_stream stream);

/* Workspace bytes of pararnn_newton_solve_host; 0 if the arguments are rejected. */
PARARNN_API size_t pararnn_host_workspace_size(const pararnn_cell *cell, int B, int T, int mode,
                                               int parts);

/*
 * pararnn_newton_solve_host_streamed -- the evaluation from and to HOST memory
 * with the sequence streamed through the device in `parts` consecutive time
 * parts, every sequence of the batch in each part.  Part p starts from each
 * sequence's last state of part p-1 (h0 for the first) and is solved to `tol`
 * on its own: the solve over time chunks of pararnn_newton_solve_chunked (the
 * ParaRNN summary page, "Experimental Results", names chunking for the Newton
 * iteration's state memory), here with the copies overlapped: while part p is
 * solved on `stream`, part p+1's inputs are copied in and part p-1's states
 * out on two helper streams.  Unlike batch
 * parts, every part keeps the whole batch, so each solve keeps its full width;
 * the parts ramp (128-step units weighted min(p + 1, parts - p, 4), rounded
 * by largest remainder with at least one unit each, as in
 * pararnn_newton_solve_host; the last part gives up the steps past T) so that
 * the exposed first copy in and last copy out are short (T = 65536 in 7 parts:
 * 4096, 8192, 12288, 16384, 12288, 8192, 4096 steps).  The states differ from the single solve's within the
 * convergence tolerance (each part meets it on its own).
 *
 * Arguments as for pararnn_newton_solve_host, except:
 *   parts      1 <= parts <= ceil(T / 128).
 *   max_iters  the cap of each part's solve; <= 0 means T + 1.
 *   info       HOST, output, may be NULL: iterations summed over the parts
 *              (as pararnn_newton_solve_chunked reports them), the worst
 *              status, the largest delta and residual.
 *   workspace  DEVICE, at least pararnn_host_streamed_workspace_size(cell, B,
 *              T, mode, parts) bytes, 256-byte aligned.
 * The copies are strided (each sequence's rows of a part): x_host, h_host
 * are [B, T, .] as for pararnn_newton_solve_host.
 * Returns the worst part's status, or INVALID_ARG / CUDA_ERROR.
 */
PARARNN_API int pararnn_newton_solve_host_streamed(const pararnn_cell *cell, const pararnn_params *params,
                                                   const void *x_host, const float *h0_host, int B, int T,
                                                   int mode, float lambda, float tol, int max_iters,
                                                   float *h_host, pararnn_info *info, int parts,
                                                   void *workspace, size_t ws_bytes, pararnn_stream stream);

/* Workspace bytes of pararnn_newton_solve_host_streamed; 0 if the arguments are rejected. */
PARARNN_API size_t pararnn_host_streamed_workspace_size(const pararnn_cell *cell, int B, int T, int mode,
                                                        int parts);

/*
 * pararnn_input_projection -- P = x W_ih^T + b_ih for every (b, t): the input
 * pre-activations, which do not depend on the state and so are computed once
 * per solve (as one GEMM [B*T, Din] x [Din, 3D]).  pararnn_newton_solve runs
 * this first; calling it separately lets a caller reuse P across solves (for
 * example a sweep over the ELK damping lambda, which the quasi-ELK method
 * needs: "Towards Scalable and Stable Parallelization of Nonlinear RNNs",
 * atlas summary "Limitations").
 *   x   DEVICE [B, T, Din] of cell->x_dtype;  params->w_ih, params->b_ih used.
 *   P   DEVICE float [B, T, 3D] output, gate-major rows (r, z, n).
 * Asynchronous.  Returns PARARNN_OK, INVALID_ARG or CUDA_ERROR.
 */
PARARNN_API int pararnn_input_projection(const pararnn_cell *cell, const pararnn_params *params,
                                         const void *x, int B, int T, float *P,
                                         pararnn_stream stream);

/*
 * pararnn_newton_iterate_async -- the Newton loop of pararnn_newton_solve_async
 * on precomputed pre-activations P (from pararnn_input_projection): every
 * iteration, the cell and its Jacobian at the shifted guess, the parallel
 * linear solve, and the on-device convergence test, until it stops.
 *   P           DEVICE float [B, T, 3D]; not modified.
 *   other arguments as pararnn_newton_solve_async; params->w_ih is not read.
 *   workspace   pararnn_workspace_size(cell, B, T, mode) bytes (its
 *               projection section is left unused).
 * Asynchronous; the report goes to info_dev.
 */
PARARNN_API int pararnn_newton_iterate_async(const pararnn_cell *cell,
                                             const pararnn_params *params, const float *P,
                                             const float *h0, int B, int T, int mode,
                                             float lambda, float tol, int max_iters, float *h,
                                             pararnn_info *info_dev, void *workspace,
                                             size_t ws_bytes, pararnn_stream stream);

/*
 * pararnn_affine_scan_workspace_size -- bytes of device workspace that
 * pararnn_affine_scan needs for these sizes (0 if they would be rejected).
 */
PARARNN_API size_t pararnn_affine_scan_workspace_size(int B, int T, int D, int dense);

/*
 * pararnn_affine_scan -- solve the linear recurrence h_t = A_t h_{t-1} + b_t,
 * t = 1..T, h_0 = h0, for B independent sequences, as a single-pass parallel
 * scan over t (the linear solve inside each Newton iteration; "ParaRNN"
 * summary, "Newton's Iteration"; "Towards Scalable and Stable Parallelization
 * of Nonlinear RNNs", atlas summary "Builds on": parallel associative scan).
 *
 *   A      DEVICE float.  dense == 0: [B, T, D], A_t acts elementwise.
 *                         dense != 0: [B, T, D, D], row-major matrices.
 *   b      DEVICE float [B, T, D].
 *   h0     DEVICE float [B, D].
 *   h      DEVICE float [B, T, D], output.  May be b itself; must not
 *          overlap b otherwise, nor A or h0.
 *   workspace  DEVICE, >= pararnn_affine_scan_workspace_size(B, T, D, dense)
 *              bytes, 256-byte aligned.  Contents on entry do not matter.
 *   D must be a multiple of 4; dense needs D <= 64.
 * Fully asynchronous.  Returns PARARNN_OK, INVALID_ARG or CUDA_ERROR; a
 * bounded device wait that expired is reported through the next call of
 * pararnn_affine_scan_status().
 */
PARARNN_API int pararnn_affine_scan(const float *A, const float *b, const float *h0, int B, int T,
                        int D, int dense, float *h, void *workspace, size_t ws_bytes,
                        pararnn_stream stream);

/*
 * pararnn_affine_scan_status -- read (and wait for) the device status word the
 * last pararnn_affine_scan using `workspace` wrote: PARARNN_OK or
 * PARARNN_TIMEOUT.  Synchronises `stream`.
 */
PARARNN_API int pararnn_affine_scan_status(const void *workspace, pararnn_stream stream);

/*
 * pararnn_affine_scan_host -- the same scan from and to HOST memory, streamed
 * through the device in `parts` consecutive time parts (every sequence in
 * each): part p is scanned from each sequence's last state of part p-1 (h0 for
 * the first), which is exact, since the scan's carry across a part boundary is
 * that state (ParaRNN summary, "Newton's Iteration": forward substitution
 * over the time steps).  While part p is scanned on `stream`, part p+1's A and
 * b are copied in and part p-1's h out on two helper streams (as in
 * pararnn_newton_solve_host_streamed, with the same ramped split in 128-step
 * units).  The results equal pararnn_affine_scan's up to the association order
 * of fp32 products.
 *   A_host     HOST [B, T, D] (dense = 0) or [B, T, D, D] (dense = 1) float.
 *   b_host     HOST [B, T, D] float.   h0_host  HOST [B, D] float.
 *   h_host     HOST [B, T, D] float, output.  Page-locked host memory lets the
 *              copies overlap; pageable memory is accepted.
 *   parts      1 <= parts <= ceil(T / 128).
 *   workspace  DEVICE, >= pararnn_affine_scan_host_workspace_size(B, T, D,
 *              dense, parts) bytes, 256-byte aligned.
 *   stream     work queued on it before the call runs first; on return
 *              everything has completed (the call synchronises `stream`).
 * Returns PARARNN_OK, PARARNN_TIMEOUT (a part's bounded look-back gave up;
 * h_host unreliable), INVALID_ARG or CUDA_ERROR.
 */
PARARNN_API int pararnn_affine_scan_host(const float *A_host, const float *b_host, const float *h0_host, int B,
                                         int T, int D, int dense, float *h_host, int parts, void *workspace,
                                         size_t ws_bytes, pararnn_stream stream);

/* Workspace bytes of pararnn_affine_scan_host; 0 if the arguments are rejected. */
PARARNN_API size_t pararnn_affine_scan_host_workspace_size(int B, int T, int D, int dense, int parts);

/*
 * pararnn_affine_scan_noalloc -- the diagonal scan of pararnn_affine_scan
 * (dense == 0) for callers that cannot allocate device memory: plugins handed
 * only their input and output buffers, code running where an allocator must
 * not be entered, or paths that forbid allocation after start-up.  The pages
 * have no counterpart; this is an interface for such callers.
 *
 * The scan's scratch (status header and look-back descriptors) is a
 * file-scope device array of 16 MiB inside this library, created when the
 * library's device code is loaded and held by every GPU that loads it until
 * the process exits.  No call allocates or frees anything.
 *   A, b, h0, h   as pararnn_affine_scan with dense == 0, except that h may
 *                 also be A itself (h may equal A or b exactly; any other
 *                 overlap with A, b or h0 is rejected).
 *   status_dev    DEVICE unsigned, may be NULL: receives 0, or 1 if a bounded
 *                 device-side wait expired (result unreliable).
 * Limits: the scratch a size needs is pararnn_affine_scan_workspace_size(B, T,
 * D, 0) bytes (a 256-byte header plus 16 bytes per lane of every look-back
 * tile; a tile spans min(D, 64) lanes and 8 * 256 / (min(D, 64) / 4) steps,
 * i.e. 128 steps for D >= 64).  Sizes needing more than 16 MiB -- about 2^25
 * elements of B*T*D for D >= 64, e.g. [31, 65536, 64] is accepted and
 * [32, 65536, 64] is not -- are rejected with PARARNN_INVALID_ARG.
 * Every call made outside stream capture looks the array's device address up
 * with the current device (so a device reset, which reloads the library's
 * device code, is followed correctly); a call inside a capture reuses the
 * address the last uncaptured call on that device found, so make one call on
 * each device before capturing it (a captured first call returns CUDA_ERROR).
 * Every call shares the one array and overwrites it (the parts that must
 * start at zero are cleared on the stream first), so calls that overlap on
 * the GPU -- on different streams, or from different host threads -- race.
 * Asynchronous.  Returns PARARNN_OK, INVALID_ARG or CUDA_ERROR.
 */
PARARNN_API int pararnn_affine_scan_noalloc(const float *A, const float *b, const float *h0,
                                            int B, int T, int D, float *h,
                                            unsigned *status_dev, pararnn_stream stream);

/*
 * pararnn_adjoint -- the backward pass through an evaluated sequence of the
 * diagonal-recurrence GRU (cell->kind == PARARNN_GRU_DIAG): the gradients of
 * a loss L with respect to the input pre-activations, the initial state and
 * the recurrent parameters, given the states and the upstream gradients.
 *
 * The pages train the evaluated RNN with the diagonal Jacobian in the backward
 * pass ("Towards Scalable and Stable Parallelization of Nonlinear RNNs", atlas
 * summary, table "Measured effects reported in the paper"); for this cell that
 * Jacobian is exact, so the results are the exact gradients.  With
 * a_t = df_t/dh_{t-1} (diagonal) and g_t = dh[t], the total derivatives
 * lam_t = dL/dh_t solve lam_T = g_T, lam_t = g_t + a_{t+1} lam_{t+1} (one
 * reverse pass with decoupled look-back), and then per (b, t, i):
 *   dP[b,t,i]     = lam (1-z)(1-n^2) g r(1-r)      (reset-gate pre-activation)
 *   dP[b,t,D+i]   = lam (h_{t-1} - n) z(1-z)       (update gate)
 *   dP[b,t,2D+i]  = lam (1-z)(1-n^2)               (candidate), g = u_n h_{t-1} + b_hn
 *   dh0[b,i]      = a_1 lam_1
 *   dw_hh[k*D+i]  = sum_{b,t} (r: dP_r, z: dP_z, n: dP_n r) * h_{t-1}    (k = r, z, n)
 *   db_hh[k*D+i]  = sum_{b,t} (dP_r, dP_z, dP_n r)
 * The input projection's gradients follow from dP by plain GEMMs the caller
 * runs (dx = dP W_ih, dW_ih = dP^T x, db_ih = sum dP); they are not computed
 * here.  The parameter sums are taken in a fixed order; the reverse scan's
 * look-back composes the later chunks' maps in an order that follows timing,
 * so repeated calls agree to fp32 rounding, not necessarily bit for bit.
 *
 *   cell, params  params->w_hh (the vectors u_r, u_z, u_n, [3D]) and
 *                 params->b_hh [3D] are read; the input weights are not.
 *   P   DEVICE [B, T, 3D] fp32 input pre-activations (pararnn_input_projection).
 *   h0  DEVICE [B, D];  h DEVICE [B, T, D] the evaluated states (a converged
 *       solve or a rollout);  dh DEVICE [B, T, D] the upstream gradients dL/dh.
 *   dP  DEVICE [B, T, 3D] out;  dh0 DEVICE [B, D] out;  dw_hh, db_hh DEVICE [3D] out.
 *   workspace  DEVICE, >= pararnn_adjoint_workspace_size bytes, 256-byte aligned.
 * All device pointers 16-byte aligned; outputs must not overlap inputs or the
 * workspace.  Asynchronous: enqueues on `stream` and returns PARARNN_OK,
 * INVALID_ARG or CUDA_ERROR; pararnn_adjoint_status reports a device timeout.
 */
PARARNN_API int pararnn_adjoint(const pararnn_cell *cell, const pararnn_params *params, const float *P,
                                const float *h0, const float *h, const float *dh, int B, int T, float *dP,
                                float *dh0, float *dw_hh, float *db_hh, void *workspace, size_t ws_bytes,
                                pararnn_stream stream);

/*
 * pararnn_adjoint_exact -- the exact backward pass of the dense GRU
 * (cell->kind == PARARNN_GRU_DENSE): pararnn_adjoint with the full transposed
 * Jacobian in the reverse recurrence, lam_T = g_T, lam_t = g_t + J_{t+1}^T
 * lam_{t+1}, instead of its diagonal (the pages train with the diagonal --
 * "Towards Scalable and Stable Parallelization of Nonlinear RNNs", atlas
 * summary, table "Measured effects reported in the paper" -- so this is the
 * reference those gradients approximate).  J_t is the dense-cell Jacobian of
 * pararnn_newton_solve (mode DEER) at the evaluated states.  The recurrence is
 * solved as the library's dense affine scan over reversed time on the
 * materialised matrices J_{t+1}^T, so the workspace holds B * T * D^2 floats
 * besides the pass's vectors.  Outputs and formulas otherwise as
 * pararnn_adjoint (dw_hh [3D, D]; dh0 = J_1^T lam_1).
 *   cell      PARARNN_GRU_DENSE, d a multiple of 4, d <= 64.
 *   workspace DEVICE, >= pararnn_adjoint_exact_workspace_size bytes, 256-byte aligned.
 * All device pointers 16-byte aligned; outputs must not overlap inputs or the
 * workspace.  Asynchronous: returns PARARNN_OK, INVALID_ARG or CUDA_ERROR.
 * The parameter sums are taken in a fixed order.
 */
PARARNN_API int pararnn_adjoint_exact(const pararnn_cell *cell, const pararnn_params *params, const float *P,
                                      const float *h0, const float *h, const float *dh, int B, int T, float *dP,
                                      float *dh0, float *dw_hh, float *db_hh, void *workspace, size_t ws_bytes,
                                      pararnn_stream stream);

/* pararnn_adjoint_exact_workspace_size -- bytes pararnn_adjoint_exact needs
 * (about (D + 12) floats per state of B*T*D, plus the scan's and the sums'
 * scratch), or 0 for rejected arguments. */
PARARNN_API size_t pararnn_adjoint_exact_workspace_size(const pararnn_cell *cell, int B, int T);

/* pararnn_adjoint_workspace_size -- bytes of workspace pararnn_adjoint needs
 * (about 0.25 B + 0.02 B per state of B*T*D plus 256), or 0 when the
 * arguments are rejected (not the diagonal cell, B, T or D < 1). */
PARARNN_API size_t pararnn_adjoint_workspace_size(const pararnn_cell *cell, int B, int T);

/* pararnn_adjoint_status -- wait for `stream` and read the status the last
 * pararnn_adjoint using `workspace` left: PARARNN_OK, or PARARNN_TIMEOUT if a
 * bounded device-side wait expired (results unreliable). */
PARARNN_API int pararnn_adjoint_status(const void *workspace, pararnn_stream stream);

/*
 * pararnn_lstm_solve -- evaluate the diagonal-recurrence LSTM (cell->kind ==
 * PARARNN_LSTM_DIAG; the pages' "adapted" LSTM, ParaLSTM: the ParaRNN talk
 * page "Federico Danieli", Abstract; the ParaRNN summary page, "Experimental
 * Results") over B sequences of length T by exact Newton (DEER), and wait.
 *
 * Cell (torch.nn.LSTMCell layout, gate rows i, f, g, o; u_k the recurrent
 * vectors, p = W_ih x + b_ih, b = b_hh):
 *   i = sig(p_i + u_i h + b_i), f = sig(p_f + u_f h + b_f), g = tanh(p_g + u_g h + b_g),
 *   o = sig(p_o + u_o h + b_o), c' = f c + i g, h' = o tanh(c').
 * Lane j of the state (c, h) depends only on lane j of the previous state, so
 * the Jacobian is a 2x2 block per lane and each Newton step is the scan of
 * s_t = A_t s_{t-1} + b_t over 2x2 affine maps (exact Newton).  The guess
 * starts at zero; convergence: max |s^(i+1) - s^(i)| over c and h <= tol.
 *
 *   params  w_ih [4D, Din] of w_dtype, b_ih [4D], w_hh [4D] (u_i, u_f, u_g, u_o),
 *           b_hh [4D] (float), all DEVICE.
 *   x       DEVICE [B, T, Din];  c0, h0 DEVICE [B, D].
 *   c, h    DEVICE [B, T, D] float, outputs (c[:, t], h[:, t] = state after step t+1).
 *   info    HOST report (may be NULL);  workspace: pararnn_lstm_workspace_size bytes.
 * d % 4 == 0 (as the GRU cells), x_dtype == w_dtype.  Synchronises `stream`
 * once; returns the solve's status (OK / NOT_CONVERGED / DIVERGED / TIMEOUT)
 * or INVALID_ARG / CUDA_ERROR.
 */
PARARNN_API int pararnn_lstm_solve(const pararnn_cell *cell, const pararnn_params *params, const void *x,
                                   const float *c0, const float *h0, int B, int T, float tol, int max_iters,
                                   float *c, float *h, pararnn_info *info, void *workspace, size_t ws_bytes,
                                   pararnn_stream stream);

/* pararnn_lstm_workspace_size -- bytes pararnn_lstm_solve needs (P, one
 * iterate copy, look-back words), or 0 for rejected arguments. */
PARARNN_API size_t pararnn_lstm_workspace_size(const pararnn_cell *cell, int B, int T);

/*
 * pararnn_adjoint_host -- pararnn_adjoint from and to HOST memory, the copies
 * overlapped with the computation through the host-buffer pipeline (ramped
 * parts, three staging buffers, the helper copy streams): part p's P,
 * h and dL/dh are copied in while its neighbours are computed, its dL/dP
 * copied out.  Each part's dW_hh and db_hh partial sums stay on the device and
 * are added in part order at the end.
 *   P_host [B, T, 3D], h0_host [B, D], h_host, dh_host [B, T, D]: HOST float.
 *   dP_host [B, T, 3D], dh0_host [B, D], dw_hh_host (the cell's w_hh shape),
 *   db_hh_host [3D]: HOST float outputs.  Page-locked memory lets the copies
 *   run asynchronously.  params->w_hh, b_hh: DEVICE, as for pararnn_adjoint.
 *   parts      1 <= parts <= B.
 *   workspace  DEVICE, >= pararnn_adjoint_host_workspace_size bytes.
 * Synchronises `stream` once, at the end; returns PARARNN_OK, PARARNN_TIMEOUT
 * (a bounded device-side wait expired in some part), INVALID_ARG or CUDA_ERROR.
 */
PARARNN_API int pararnn_adjoint_host(const pararnn_cell *cell, const pararnn_params *params, const float *P_host,
                                     const float *h0_host, const float *h_host, const float *dh_host, int B, int T,
                                     float *dP_host, float *dh0_host, float *dw_hh_host, float *db_hh_host,
                                     int parts, void *workspace, size_t ws_bytes, pararnn_stream stream);

/* pararnn_adjoint_host_workspace_size -- bytes pararnn_adjoint_host needs, or 0. */
PARARNN_API size_t pararnn_adjoint_host_workspace_size(const pararnn_cell *cell, int B, int T, int parts);

/*
 * pararnn_lstm_solve_host -- pararnn_lstm_solve from and to HOST memory, with
 * the copies overlapped with the computation as in pararnn_newton_solve_host:
 * the batch in `parts` ramped parts (same sizes), three staging buffers, part
 * p's x copied in and its (c, h) copied out on the two helper streams,
 * while part p's neighbours are solved on `stream`.  Each part is an
 * independent solve to `tol`; the report is the worst part's.
 *   x_host     HOST [B, T, Din] of cell->x_dtype;  c0_host, h0_host HOST [B, D].
 *   c_host, h_host  HOST [B, T, D] float outputs.  Page-locked memory lets the
 *              copies run asynchronously.
 *   parts      1 <= parts <= B.
 *   workspace  DEVICE, >= pararnn_lstm_host_workspace_size bytes, 256-byte aligned.
 * Synchronises `stream` once, at the end; returns the worst part's status, or
 * INVALID_ARG / CUDA_ERROR.
 */
PARARNN_API int pararnn_lstm_solve_host(const pararnn_cell *cell, const pararnn_params *params, const void *x_host,
                                        const float *c0_host, const float *h0_host, int B, int T, float tol,
                                        int max_iters, float *c_host, float *h_host, pararnn_info *info, int parts,
                                        void *workspace, size_t ws_bytes, pararnn_stream stream);

/* pararnn_lstm_host_workspace_size -- bytes pararnn_lstm_solve_host needs (one
 * part's solve workspace, three parts' staging, the initial states), or 0. */
PARARNN_API size_t pararnn_lstm_host_workspace_size(const pararnn_cell *cell, int B, int T, int parts);

/*
 * pararnn_lstm_solve_host_streamed -- the LSTM solve from and to HOST memory
 * with the sequence streamed through the device in `parts` consecutive time
 * parts (every sequence in each), as pararnn_newton_solve_host_streamed: part
 * p starts from each sequence's last (c, h) of part p-1 ((c0, h0) for the
 * first) and is solved to `tol` on its own while part p+1's inputs are copied
 * in and part p-1's (c, h) out.  Same ramped split in 128-step units.
 * Arguments as for pararnn_lstm_solve_host, except 1 <= parts <= ceil(T / 128),
 * max_iters caps each part (<= 0: T + 1), the workspace is
 * pararnn_lstm_host_streamed_workspace_size bytes, and the report sums
 * iterations over the parts (worst status, largest delta and residual).
 */
PARARNN_API int pararnn_lstm_solve_host_streamed(const pararnn_cell *cell, const pararnn_params *params,
                                                 const void *x_host, const float *c0_host, const float *h0_host,
                                                 int B, int T, float tol, int max_iters, float *c_host,
                                                 float *h_host, pararnn_info *info, int parts, void *workspace,
                                                 size_t ws_bytes, pararnn_stream stream);

/* Workspace bytes of pararnn_lstm_solve_host_streamed; 0 if the arguments are rejected. */
PARARNN_API size_t pararnn_lstm_host_streamed_workspace_size(const pararnn_cell *cell, int B, int T, int parts);

/* pararnn_status_string -- a static, human-readable name of a status code. */
PARARNN_API const char *pararnn_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* PARARNN_H */

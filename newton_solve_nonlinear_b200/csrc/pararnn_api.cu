// pararnn_api.cu -- the C ABI: argument checks, workspace layout, launches.
//
// Every entry point is declared and documented in include/pararnn.h.  Nothing
// here allocates memory; the caller's workspace is carved into the sections
// below (each 256-byte aligned):
//   header  WsHeader (grid barrier, status word, delta/residual slots, report)
//   P       [B, T, 3D] fp32 input pre-activations
//   hbuf    [B, T, D]  fp32 second iterate buffer (the caller's h is the first)
//   desc    look-back descriptors: tiles x lanes x (2 words, or 8 for quasi-ELK)
//   elk     quasi-ELK forward results m, P, a, b: 4 x [B, T, D] fp32
//   dense   block-scan scratch of the dense-Jacobian modes
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "solver.cuh"

namespace pararnn {

size_t scan_diag_ws_bytes(int B, int T, int D);
size_t dense_ws_bytes(const pararnn_cell &cell, int B, int T, int mode);
cudaError_t launch_dense_solver(const pararnn_cell &cell, int mode, const DiagArgs &a,
                                void *dense_ws, cudaStream_t s);
size_t quasi_tc_desc_bytes(int B, int T, int D);
bool quasi_tc_supported(const pararnn_cell &cell, int B, int T);
cudaError_t launch_quasi_tc2(const DiagArgs &a, bool elk, cudaStream_t s);
bool diag2_supported(const pararnn_cell &cell, int B, int T);
size_t diag2_desc_bytes(int B, int T, int D);
cudaError_t launch_diag2(const DiagArgs &a, cudaStream_t s);
cudaError_t launch_scan_dense(const float *A, const float *b, const float *h0, int B, int T,
                              int D, float *h, void *ws, cudaStream_t s);
size_t scan_dense_ws_bytes(int B, int T, int D);
size_t lstm_diag_desc_bytes(int B, int T, int D);
cudaError_t launch_lstm_diag(const float *P, const float *u, const float *b_hh, const float *c0, const float *h0,
                             int B, int T, int D, float tol, int max_iters, float *c_ws, float *h_ws, float *c_out,
                             float *h_out, void *hdr, void *desc, pararnn_info *info_out, cudaStream_t s);
size_t adjoint_diag_desc_bytes(int B, int T, int D);
size_t adjoint_diag_part_bytes(int B, int T, int D);
cudaError_t launch_adjoint_diag(const float *P, const float *h0, const float *h, const float *dh, const float *u,
                                const float *b_hh, float *dP, float *dh0, float *du, float *db_hh, int B, int T,
                                int D, void *hdr, void *desc, void *part, cudaStream_t s, const float *w_hh_dense,
                                const float *G, float *grow);
size_t adjoint_outer_part_bytes(long long M, int N, int K);
bool deer_mma_supported(const pararnn_cell &cell);
cudaError_t launch_sum_rows(const float *in, int rows, int n, float *out, cudaStream_t s);
cudaError_t adjoint_enqueue(const pararnn_cell *cell, const pararnn_params *params, const float *P, const float *h0,
                            const float *h, const float *dh, int B, int T, float *dP, float *dh0, float *dw_hh,
                            float *db_hh, void *workspace, cudaStream_t s);
cudaError_t launch_outer_sum(const float *grow, const float *hp, long long M, int N, int K, float *part, float *out,
                             cudaStream_t s);
size_t adjoint_exact_ws_bytes(int B, int T, int D);
cudaError_t adjoint_exact_enqueue(const float *w_hh, const float *b_hh, const float *P, const float *h0,
                                  const float *h, const float *dh, int B, int T, int D, float *dP, float *dh0,
                                  float *dw_hh, float *db_hh, void *workspace, cudaStream_t s);

namespace {

// NVTX range around a host-side phase of a call (projection, Newton loop,
// host-buffer part, backward pass, report wait): Nsight Systems shows the
// phases and the launches they enqueue; with no tool attached a push/pop is a
// few nanoseconds.
struct Range {
    explicit Range(const char *name) { nvtxRangePushA(name); }
    ~Range() { nvtxRangePop(); }
    Range(const Range &) = delete;
    Range &operator=(const Range &) = delete;
};

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    const auto pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
    return pa < pb + nb && pb < pa + na;
}

bool diag_jacobian(const pararnn_cell &cell, int mode) {
    return cell.kind == PARARNN_GRU_DIAG || mode == PARARNN_QUASI || mode == PARARNN_QUASI_ELK;
}

bool is_elk(int mode) { return mode == PARARNN_ELK || mode == PARARNN_QUASI_ELK; }

bool cell_ok(const pararnn_cell *cell, int B, int T, int mode) {
    if (cell == nullptr || B < 1 || T < 1) return false;
    if (cell->kind != PARARNN_GRU_DENSE && cell->kind != PARARNN_GRU_DIAG) return false;
    if (cell->d < 4 || cell->d % 4 != 0 || cell->din < 1) return false;
    if (cell->x_dtype != cell->w_dtype) return false;
    if (cell->x_dtype != PARARNN_F32 && cell->x_dtype != PARARNN_BF16) return false;
    if (mode < PARARNN_DEER || mode > PARARNN_QUASI_ELK) return false;
    if (cell->kind == PARARNN_GRU_DENSE && cell->d > 64) return false;
    // the state array is indexed with 32-bit time and lane counts
    if (static_cast<long long>(T) * 3 * cell->d > (1ll << 31)) return false;
    return true;
}

}  // namespace

WsLayout ws_layout(const pararnn_cell &cell, int B, int T, int mode) {
    WsLayout L{};
    const size_t states = static_cast<size_t>(B) * T * cell.d;
    const bool diag = diag_jacobian(cell, mode);
    const Tiling tl = make_tiling(B, T, cell.d, cell.kind == PARARNN_GRU_DENSE, kSolverTK);
    size_t off = 0;
    L.header = off; off += 256;
    L.P = off; off = align256(off + states * 3 * sizeof(float));
    L.hbuf = off; off = align256(off + states * sizeof(float));
    L.desc = off;
    if (diag) {
        size_t desc = static_cast<size_t>(tl.n_tiles) * tl.DG * (is_elk(mode) ? 8 : 2) * 8;
        // the tensor-core dense-cell path tiles by 128 steps x all lanes (quasi-ELK:
        // covariance, mean and smoother descriptors, 8 words per tile and lane)
        if (cell.kind == PARARNN_GRU_DENSE && (mode == PARARNN_QUASI || mode == PARARNN_QUASI_ELK) &&
            (cell.d == 32 || cell.d == 64)) {
            const size_t tc = quasi_tc_desc_bytes(B, T, cell.d) * (is_elk(mode) ? 4 : 1);
            if (tc > desc) desc = tc;
        }
        // the streaming diagonal-cell path tiles by 32 steps x 64 lanes
        if (cell.kind == PARARNN_GRU_DIAG && !is_elk(mode) && cell.d % 64 == 0) {
            const size_t d2 = diag2_desc_bytes(B, T, cell.d);
            if (d2 > desc) desc = d2;
        }
        off = align256(off + desc);
    }
    L.elk = off;
    if (diag && is_elk(mode)) off = align256(off + 4 * states * sizeof(float));
    L.dense = off;
    if (!diag) off = align256(off + dense_ws_bytes(cell, B, T, mode));
    L.total = off;
    return L;
}

}  // namespace pararnn

using namespace pararnn;

extern "C" {

size_t pararnn_workspace_size(const pararnn_cell *cell, int B, int T, int mode) {
    if (!cell_ok(cell, B, T, mode)) return 0;
    return ws_layout(*cell, B, T, mode).total;
}

// Checks shared by every solve entry point.  `need_x`: the projection runs.
static int check_solve(const pararnn_cell *cell, const pararnn_params *params, const void *x,
                       const float *P, const float *h0, int B, int T, int mode, float lambda,
                       float tol, float *h, void *workspace, size_t ws_bytes) {
    if (!cell_ok(cell, B, T, mode) || params == nullptr) return PARARNN_INVALID_ARG;
    if ((!x && !P) || !h0 || !h || !workspace || !params->w_hh || !params->b_hh)
        return PARARNN_INVALID_ARG;
    if (x && (!params->w_ih || !params->b_ih)) return PARARNN_INVALID_ARG;
    if (!(tol >= 0.f) || !std::isfinite(tol)) return PARARNN_INVALID_ARG;
    if (is_elk(mode) && !(lambda > 0.f && std::isfinite(lambda))) return PARARNN_INVALID_ARG;
    if ((x && !aligned(x, 16)) || (P && !aligned(P, 16)) || !aligned(h0, 16) || !aligned(h, 16) ||
        !aligned(params->w_hh, 16) || !aligned(params->b_hh, 16) || !aligned(workspace, 256))
        return PARARNN_INVALID_ARG;
    if (x && (!aligned(params->b_ih, 16) || !aligned(params->w_ih, 16))) return PARARNN_INVALID_ARG;
    const WsLayout L = ws_layout(*cell, B, T, mode);
    if (ws_bytes < L.total) return PARARNN_INVALID_ARG;
    const size_t states = static_cast<size_t>(B) * T * cell->d;
    const size_t xbytes = static_cast<size_t>(B) * T * cell->din *
                          (cell->x_dtype == PARARNN_BF16 ? 2 : 4);
    if (overlaps(h, states * 4, workspace, L.total) ||
        (x && overlaps(h, states * 4, x, xbytes)) || (P && overlaps(h, states * 4, P, states * 12)) ||
        overlaps(h, states * 4, h0, static_cast<size_t>(B) * cell->d * 4))
        return PARARNN_INVALID_ARG;
    if (P && overlaps(P, states * 12, workspace, L.total)) return PARARNN_INVALID_ARG;
    return PARARNN_OK;
}

// Enqueue the Newton loop on pre-activations P (device).
static cudaError_t enqueue_iterate(const pararnn_cell *cell, const pararnn_params *params,
                                   const float *P, const float *h0, int B, int T, int mode,
                                   float lambda, float tol, int max_iters, float *h,
                                   pararnn_info *info_dev, void *workspace, cudaStream_t s,
                                   const float *h_init = nullptr, int jac_every = 1,
                                   float *trace = nullptr, int trace_len = 0, long long withhold = -1) {
    const Range range("pararnn: Newton loop");
    const WsLayout L = ws_layout(*cell, B, T, mode);
    char *ws = static_cast<char *>(workspace);
    WsHeader *hdr = reinterpret_cast<WsHeader *>(ws + L.header);
    const bool diag = diag_jacobian(*cell, mode);
    const size_t states = static_cast<size_t>(B) * T * cell->d;

    DiagArgs a{};
    a.B = B; a.T = T; a.D = cell->d;
    a.P = P;
    a.w_hh = params->w_hh;
    a.b_hh = params->b_hh;
    a.h0 = h0;
    a.hbuf[0] = reinterpret_cast<float *>(ws + L.hbuf);
    a.hbuf[1] = h;
    a.lambda = lambda;
    a.tol = tol;
    a.max_iters = max_iters <= 0 ? T + 1 : max_iters;
    a.tl = make_tiling(B, T, cell->d, cell->kind == PARARNN_GRU_DENSE, kSolverTK);
    a.desc = reinterpret_cast<unsigned long long *>(ws + L.desc);
    const size_t states4 = states * sizeof(float);
    a.elk_m = reinterpret_cast<float *>(ws + L.elk);
    a.elk_p = reinterpret_cast<float *>(ws + L.elk + states4);
    a.elk_a = reinterpret_cast<float *>(ws + L.elk + 2 * states4);
    a.elk_b = reinterpret_cast<float *>(ws + L.elk + 3 * states4);
    a.hdr = hdr;
    a.info_out = info_dev ? info_dev : &hdr->info;
    a.warm = h_init != nullptr;
    a.jac_every = jac_every;
    // the frozen Jacobian coefficients sit after the solve's own workspace
    a.coef = jac_every > 1 ? reinterpret_cast<float *>(ws + L.total) : nullptr;
    a.trace = trace;
    a.trace_len = trace ? trace_len : 0;
    a.withhold = withhold;

    cudaError_t e = cudaMemsetAsync(ws + L.header, 0, 256, s);
    if (e == cudaSuccess && diag && L.elk > L.desc) e = cudaMemsetAsync(ws + L.desc, 0, L.elk - L.desc, s);
    // the first guess: the caller's (copied first, so h_init may be h itself), else zero
    if (e == cudaSuccess && h_init)
        e = cudaMemcpyAsync(a.hbuf[0], h_init, states * sizeof(float), cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return e;
    if ((mode == PARARNN_QUASI || mode == PARARNN_QUASI_ELK) && quasi_tc_supported(*cell, B, T)) {
        // the tensor-core path reads the initial guess from memory
        if (!h_init) e = cudaMemsetAsync(a.hbuf[0], 0, states * sizeof(float), s);
        if (e != cudaSuccess) return e;
        return launch_quasi_tc2(a, mode == PARARNN_QUASI_ELK, s);
    }
    if (cell->kind == PARARNN_GRU_DIAG && !is_elk(mode) && diag2_supported(*cell, B, T)) {
        if (!h_init) e = cudaMemsetAsync(a.hbuf[0], 0, states * sizeof(float), s);
        if (e != cudaSuccess) return e;
        return launch_diag2(a, s);
    }
    return diag ? launch_diag_solver(*cell, mode, a, s)
                : launch_dense_solver(*cell, mode, a, ws + L.dense, s);
}

int pararnn_input_projection(const pararnn_cell *cell, const pararnn_params *params,
                             const void *x, int B, int T, float *P, pararnn_stream stream) {
    // the projection does not involve the recurrence: only the widths and dtypes matter
    if (!cell || B < 1 || T < 1 || cell->d < 1 || cell->din < 1) return PARARNN_INVALID_ARG;
    if (cell->x_dtype != cell->w_dtype ||
        (cell->x_dtype != PARARNN_F32 && cell->x_dtype != PARARNN_BF16))
        return PARARNN_INVALID_ARG;
    if (!params || !x || !P || !params->w_ih || !params->b_ih) return PARARNN_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(P, 16) || !aligned(params->w_ih, 16) || !aligned(params->b_ih, 16))
        return PARARNN_INVALID_ARG;
    const Range range("pararnn: input projection");
    const cudaError_t e = launch_projection(*cell, x, params->w_ih, params->b_ih, P,
                                            static_cast<long long>(B) * T,
                                            reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PARARNN_OK : PARARNN_CUDA_ERROR;
}

int pararnn_newton_iterate_async(const pararnn_cell *cell, const pararnn_params *params,
                                 const float *P, const float *h0, int B, int T, int mode,
                                 float lambda, float tol, int max_iters, float *h,
                                 pararnn_info *info_dev, void *workspace, size_t ws_bytes,
                                 pararnn_stream stream) {
    if (!P || !info_dev || !aligned(info_dev, 4)) return PARARNN_INVALID_ARG;
    int rc = check_solve(cell, params, nullptr, P, h0, B, T, mode, lambda, tol, h, workspace,
                         ws_bytes);
    if (rc != PARARNN_OK) return rc;
    const cudaError_t e = enqueue_iterate(cell, params, P, h0, B, T, mode, lambda, tol, max_iters,
                                          h, info_dev, workspace,
                                          reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PARARNN_OK : PARARNN_CUDA_ERROR;
}

static int solve_enqueue(const pararnn_cell *cell, const pararnn_params *params, const void *x,
                         const float *h0, int B, int T, int mode, float lambda, float tol,
                         int max_iters, float *h, pararnn_info *info_dev, void *workspace,
                         size_t ws_bytes, pararnn_stream stream, const float *h_init = nullptr,
                         int jac_every = 1, float *trace = nullptr, int trace_len = 0,
                         long long withhold = -1) {
    int rc = check_solve(cell, params, x, nullptr, h0, B, T, mode, lambda, tol, h, workspace,
                         ws_bytes);
    if (rc != PARARNN_OK) return rc;
    if (h_init) {  // a guess of [B, T, D]: aligned, and clear of the workspace (it may be h)
        const size_t nb = static_cast<size_t>(B) * T * cell->d * 4;
        if (!aligned(h_init, 16) || overlaps(h_init, nb, workspace, ws_layout(*cell, B, T, mode).total))
            return PARARNN_INVALID_ARG;
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const WsLayout L = ws_layout(*cell, B, T, mode);
    float *P = reinterpret_cast<float *>(static_cast<char *>(workspace) + L.P);
    cudaError_t e;
    {
        const Range range("pararnn: input projection");
        e = launch_projection(*cell, x, params->w_ih, params->b_ih, P, static_cast<long long>(B) * T, s);
    }
    if (e == cudaSuccess)
        e = enqueue_iterate(cell, params, P, h0, B, T, mode, lambda, tol, max_iters, h, info_dev,
                            workspace, s, h_init, jac_every, trace, trace_len, withhold);
    return e == cudaSuccess ? PARARNN_OK : PARARNN_CUDA_ERROR;
}

int pararnn_newton_solve_async(const pararnn_cell *cell, const pararnn_params *params,
                               const void *x, const float *h0, int B, int T, int mode,
                               float lambda, float tol, int max_iters, float *h,
                               pararnn_info *info_dev, void *workspace, size_t ws_bytes,
                               pararnn_stream stream) {
    if (info_dev == nullptr || !aligned(info_dev, 4)) return PARARNN_INVALID_ARG;
    return solve_enqueue(cell, params, x, h0, B, T, mode, lambda, tol, max_iters, h, info_dev,
                         workspace, ws_bytes, stream);
}

int pararnn_newton_solve(const pararnn_cell *cell, const pararnn_params *params, const void *x,
                         const float *h0, int B, int T, int mode, float lambda, float tol,
                         int max_iters, float *h, pararnn_info *info, void *workspace,
                         size_t ws_bytes, pararnn_stream stream) {
    const int rc = solve_enqueue(cell, params, x, h0, B, T, mode, lambda, tol, max_iters, h,
                                 nullptr, workspace, ws_bytes, stream);
    if (rc != PARARNN_OK) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const WsLayout L = ws_layout(*cell, B, T, mode);
    pararnn_info host{};
    const WsHeader *hdr = reinterpret_cast<const WsHeader *>(static_cast<char *>(workspace) + L.header);
    cudaError_t e = cudaMemcpyAsync(&host, &hdr->info, sizeof(host), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return PARARNN_CUDA_ERROR;
    if (info) *info = host;
    return host.status;
}

int pararnn_newton_solve_guess_async(const pararnn_cell *cell, const pararnn_params *params, const void *x,
                                     const float *h0, const float *h_init, int B, int T, int mode, float lambda,
                                     float tol, int max_iters, float *h, pararnn_info *info_dev,
                                     void *workspace, size_t ws_bytes, pararnn_stream stream) {
    if (info_dev == nullptr || !aligned(info_dev, 4) || h_init == nullptr) return PARARNN_INVALID_ARG;
    return solve_enqueue(cell, params, x, h0, B, T, mode, lambda, tol, max_iters, h, info_dev, workspace,
                         ws_bytes, stream, h_init);
}

// Wait for `stream` and read the report the last solve on `workspace` left.
static int read_report(const pararnn_cell *cell, int B, int T, int mode, void *workspace, cudaStream_t s,
                       pararnn_info *info) {
    const Range range("pararnn: wait for the report");
    const WsLayout L = ws_layout(*cell, B, T, mode);
    pararnn_info host{};
    const WsHeader *hdr = reinterpret_cast<const WsHeader *>(static_cast<char *>(workspace) + L.header);
    cudaError_t e = cudaMemcpyAsync(&host, &hdr->info, sizeof(host), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return PARARNN_CUDA_ERROR;
    if (info) *info = host;
    return host.status;
}

int pararnn_newton_solve_trace(const pararnn_cell *cell, const pararnn_params *params, const void *x,
                               const float *h0, int B, int T, int mode, float lambda, float tol, int max_iters,
                               float *h, pararnn_info *info, float *trace, int trace_len, void *workspace,
                               size_t ws_bytes, pararnn_stream stream) {
    if (trace == nullptr || trace_len < 1 || !aligned(trace, 8)) return PARARNN_INVALID_ARG;
    if (cell_ok(cell, B, T, mode)) {
        const size_t tb = static_cast<size_t>(trace_len) * 8;
        const size_t hb = static_cast<size_t>(B) * T * cell->d * 4;
        if (overlaps(trace, tb, workspace, ws_layout(*cell, B, T, mode).total) || overlaps(trace, tb, h, hb))
            return PARARNN_INVALID_ARG;
    }
    const int rc = solve_enqueue(cell, params, x, h0, B, T, mode, lambda, tol, max_iters, h, nullptr, workspace,
                                 ws_bytes, stream, nullptr, 1, trace, trace_len);
    if (rc != PARARNN_OK) return rc;
    return read_report(cell, B, T, mode, workspace, reinterpret_cast<cudaStream_t>(stream), info);
}

int pararnn_test_withheld_publish(const pararnn_cell *cell, const pararnn_params *params, const void *x,
                                  const float *h0, int B, int T, int mode, float tol, float *h, pararnn_info *info,
                                  long long tile, void *workspace, size_t ws_bytes, pararnn_stream stream) {
    if (!cell_ok(cell, B, T, mode) || tile < 0) return PARARNN_INVALID_ARG;
    long long tiles = 0;  // tiles of the look-back the solve will take
    if (mode == PARARNN_QUASI && quasi_tc_supported(*cell, B, T))
        tiles = static_cast<long long>(quasi_tc_desc_bytes(B, T, cell->d) / (static_cast<size_t>(cell->d) * 16));
    else if (cell->kind == PARARNN_GRU_DIAG && (mode == PARARNN_DEER || mode == PARARNN_QUASI) &&
             diag2_supported(*cell, B, T))
        tiles = static_cast<long long>(diag2_desc_bytes(B, T, cell->d) / (64 * 16));
    if (tile >= tiles) return PARARNN_INVALID_ARG;
    const int rc = solve_enqueue(cell, params, x, h0, B, T, mode, 0.f, tol, 0, h, nullptr, workspace, ws_bytes,
                                 stream, nullptr, 1, nullptr, 0, tile);
    if (rc != PARARNN_OK) return rc;
    return read_report(cell, B, T, mode, workspace, reinterpret_cast<cudaStream_t>(stream), info);
}

// ---- DEER with the Jacobian reused for several iterations ----

// Frozen coefficients: 128 floats per step (z, cz, cn, cr for 32 rows).
static size_t reuse_coef_bytes(int B, int T) { return align256(static_cast<size_t>(B) * T * 512); }

size_t pararnn_reuse_workspace_size(const pararnn_cell *cell, int B, int T) {
    if (!cell || cell->kind != PARARNN_GRU_DENSE || !cell_ok(cell, B, T, PARARNN_DEER) ||
        !deer_mma_supported(*cell))
        return 0;
    return ws_layout(*cell, B, T, PARARNN_DEER).total + reuse_coef_bytes(B, T);
}

int pararnn_newton_solve_reuse(const pararnn_cell *cell, const pararnn_params *params, const void *x,
                               const float *h0, int B, int T, int jac_every, float tol, int max_iters, float *h,
                               pararnn_info *info, void *workspace, size_t ws_bytes, pararnn_stream stream) {
    const size_t need = pararnn_reuse_workspace_size(cell, B, T);
    if (need == 0 || jac_every < 1 || ws_bytes < need || !h || !workspace) return PARARNN_INVALID_ARG;
    if (overlaps(h, static_cast<size_t>(B) * T * cell->d * 4, workspace, need)) return PARARNN_INVALID_ARG;
    const int rc = solve_enqueue(cell, params, x, h0, B, T, PARARNN_DEER, 0.f, tol, max_iters, h, nullptr,
                                 workspace, ws_bytes, stream, nullptr, jac_every);
    if (rc != PARARNN_OK) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const WsLayout L = ws_layout(*cell, B, T, PARARNN_DEER);
    pararnn_info host{};
    const WsHeader *hdr = reinterpret_cast<const WsHeader *>(static_cast<char *>(workspace) + L.header);
    cudaError_t e = cudaMemcpyAsync(&host, &hdr->info, sizeof(host), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return PARARNN_CUDA_ERROR;
    if (info) *info = host;
    return host.status;
}

// ---- T-chunked solve: consecutive time chunks solved one after another ----

namespace {
struct ChunkLayout {
    int tc, nchunks;
    size_t solve, xs, hs, h0, infos, total;
};
ChunkLayout chunk_layout(const pararnn_cell &cell, int B, int T, int t_chunk, int mode) {
    ChunkLayout C{};
    C.tc = t_chunk < T ? t_chunk : T;
    C.nchunks = (T + C.tc - 1) / C.tc;
    const size_t es = cell.x_dtype == PARARNN_BF16 ? 2 : 4;
    size_t off = 0;
    C.solve = off; off = align256(off + ws_layout(cell, B, C.tc, mode).total);
    C.xs = off; off = align256(off + static_cast<size_t>(B) * C.tc * cell.din * es);
    C.hs = off; off = align256(off + static_cast<size_t>(B) * C.tc * cell.d * 4);
    C.h0 = off; off = align256(off + static_cast<size_t>(B) * cell.d * 4);
    C.infos = off; off = align256(off + static_cast<size_t>(C.nchunks) * sizeof(pararnn_info));
    C.total = off;
    return C;
}
}  // namespace

size_t pararnn_chunked_workspace_size(const pararnn_cell *cell, int B, int T, int t_chunk, int mode) {
    if (t_chunk < 1 || !cell_ok(cell, B, T, mode)) return 0;
    const int tc = t_chunk < T ? t_chunk : T;
    if (!cell_ok(cell, B, tc, mode)) return 0;
    return chunk_layout(*cell, B, T, t_chunk, mode).total;
}

int pararnn_newton_solve_chunked(const pararnn_cell *cell, const pararnn_params *params, const void *x,
                                 const float *h0, int B, int T, int t_chunk, int mode, float lambda, float tol,
                                 int max_iters, float *h, pararnn_info *info, void *workspace, size_t ws_bytes,
                                 pararnn_stream stream) {
    const size_t need = pararnn_chunked_workspace_size(cell, B, T, t_chunk, mode);
    if (need == 0 || ws_bytes < need || !params || !x || !h0 || !h || !workspace || !aligned(workspace, 256) ||
        !aligned(x, 16) || !aligned(h0, 16) || !aligned(h, 16))
        return PARARNN_INVALID_ARG;
    const ChunkLayout C = chunk_layout(*cell, B, T, t_chunk, mode);
    const size_t es = cell->x_dtype == PARARNN_BF16 ? 2 : 4;
    const size_t xrow = static_cast<size_t>(T) * cell->din * es, hrow = static_cast<size_t>(T) * cell->d * 4;
    if (overlaps(h, B * hrow, workspace, need) || overlaps(h, B * hrow, x, B * xrow) ||
        overlaps(h, B * hrow, h0, static_cast<size_t>(B) * cell->d * 4))
        return PARARNN_INVALID_ARG;
    char *ws = static_cast<char *>(workspace);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    pararnn_info *infos = reinterpret_cast<pararnn_info *>(ws + C.infos);
    cudaError_t e = cudaSuccess;
    int rc = PARARNN_OK;
    for (int c = 0; c < C.nchunks && e == cudaSuccess && rc == PARARNN_OK; ++c) {
        const int t0 = c * C.tc, n = (T - t0) < C.tc ? (T - t0) : C.tc;
        // this chunk's inputs of every sequence, packed [B, n, Din]
        e = cudaMemcpy2DAsync(ws + C.xs, n * cell->din * es, static_cast<const char *>(x) + t0 * cell->din * es,
                              xrow, n * cell->din * es, B, cudaMemcpyDeviceToDevice, s);
        // the state entering the chunk: h0, or each sequence's last state of the previous chunk
        if (e == cudaSuccess && c > 0)
            e = cudaMemcpy2DAsync(ws + C.h0, cell->d * 4, reinterpret_cast<const char *>(h) + (t0 - 1) * cell->d * 4,
                                  hrow, cell->d * 4, B, cudaMemcpyDeviceToDevice, s);
        if (e != cudaSuccess) break;
        const float *hin = c == 0 ? h0 : reinterpret_cast<const float *>(ws + C.h0);
        // the cap of the whole sequence's solve (T + 1 by default), not of the chunk:
        // damped modes may need more iterations than a short chunk has steps
        rc = solve_enqueue(cell, params, ws + C.xs, hin, B, n, mode, lambda, tol, max_iters > 0 ? max_iters : T + 1,
                           reinterpret_cast<float *>(ws + C.hs), infos + c, ws + C.solve,
                           ws_layout(*cell, B, n, mode).total, stream);
        if (rc != PARARNN_OK) break;
        e = cudaMemcpy2DAsync(reinterpret_cast<char *>(h) + t0 * cell->d * 4, hrow, ws + C.hs, n * cell->d * 4,
                              n * cell->d * 4, B, cudaMemcpyDeviceToDevice, s);
    }
    if (e != cudaSuccess) return PARARNN_CUDA_ERROR;
    if (rc != PARARNN_OK) return rc;
    std::vector<pararnn_info> host(C.nchunks);
    e = cudaMemcpyAsync(host.data(), infos, C.nchunks * sizeof(pararnn_info), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return PARARNN_CUDA_ERROR;
    pararnn_info agg{};
    for (const pararnn_info &q : host) {  // iterations summed over the chunks; the worst of the rest
        agg.iters += q.iters;
        agg.status = q.status > agg.status ? q.status : agg.status;
        agg.delta = q.delta > agg.delta ? q.delta : agg.delta;
        agg.residual = q.residual > agg.residual ? q.residual : agg.residual;
    }
    if (info) *info = agg;
    return agg.status;
}

size_t pararnn_affine_scan_workspace_size(int B, int T, int D, int dense) {
    if (B < 1 || T < 1 || D < 4 || D % 4 != 0) return 0;
    if (static_cast<long long>(T) * D > (1ll << 31)) return 0;
    if (dense) return D <= 64 ? scan_dense_ws_bytes(B, T, D) : 0;
    return scan_diag_ws_bytes(B, T, D);
}

int pararnn_affine_scan(const float *A, const float *b, const float *h0, int B, int T, int D,
                        int dense, float *h, void *workspace, size_t ws_bytes,
                        pararnn_stream stream) {
    const size_t need = pararnn_affine_scan_workspace_size(B, T, D, dense);
    if (need == 0 || ws_bytes < need) return PARARNN_INVALID_ARG;
    if (!A || !b || !h0 || !h || !workspace) return PARARNN_INVALID_ARG;
    if (!aligned(A, 16) || !aligned(b, 16) || !aligned(h0, 16) || !aligned(h, 16) ||
        !aligned(workspace, 256))
        return PARARNN_INVALID_ARG;
    const size_t nA = static_cast<size_t>(B) * T * D * (dense ? D : 1) * 4;
    const size_t nh = static_cast<size_t>(B) * T * D * 4;
    // h may be b itself (each b_t is read before its h_t is written), not a part of it
    if (overlaps(h, nh, A, nA) || overlaps(h, nh, h0, static_cast<size_t>(B) * D * 4) ||
        overlaps(h, nh, workspace, need) || (h != b && overlaps(h, nh, b, nh)))
        return PARARNN_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const cudaError_t e = dense ? launch_scan_dense(A, b, h0, B, T, D, h, workspace, s)
                                : launch_scan_diag(A, b, h0, B, T, D, h, workspace, s);
    return e == cudaSuccess ? PARARNN_OK : PARARNN_CUDA_ERROR;
}

int pararnn_affine_scan_status(const void *workspace, pararnn_stream stream) {
    if (!workspace || !aligned(workspace, 256)) return PARARNN_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    unsigned st = 0;
    const WsHeader *hdr = static_cast<const WsHeader *>(workspace);
    cudaError_t e = cudaMemcpyAsync(&st, &hdr->status, sizeof(st), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return PARARNN_CUDA_ERROR;
    return (st & kStatusTimeout) ? PARARNN_TIMEOUT : PARARNN_OK;
}

// ---- diagonal-recurrence LSTM ------------------------------------------------

namespace {
struct LstmLayout {
    size_t header, P, cws, hws, desc, total;
};
bool lstm_cell_ok(const pararnn_cell *cell, int B, int T) {
    if (!cell || cell->kind != PARARNN_LSTM_DIAG || B < 1 || T < 1) return false;
    if (cell->d < 4 || cell->d % 4 != 0 || cell->din < 1 || cell->x_dtype != cell->w_dtype) return false;
    if (cell->x_dtype != PARARNN_F32 && cell->x_dtype != PARARNN_BF16) return false;
    return static_cast<long long>(T) * 4 * cell->d <= (1ll << 31) && static_cast<long long>(B) * T < (1ll << 31);
}
LstmLayout lstm_layout(const pararnn_cell &cell, int B, int T) {
    LstmLayout L{};
    const size_t states = static_cast<size_t>(B) * T * cell.d;
    size_t off = 0;
    L.header = off; off += 256;
    L.P = off; off = align256(off + states * 4 * sizeof(float));
    L.cws = off; off = align256(off + states * sizeof(float));
    L.hws = off; off = align256(off + states * sizeof(float));
    L.desc = off; off = align256(off + lstm_diag_desc_bytes(B, T, cell.d));
    L.total = off;
    return L;
}

// Enqueue the projection (4D gate rows) and the solve on `s`; the report goes
// to info_dev (nullptr: the workspace header).  Arguments already checked.
cudaError_t lstm_enqueue(const pararnn_cell *cell, const pararnn_params *params, const void *x, const float *c0,
                         const float *h0, int B, int T, float tol, int max_iters, float *c, float *h,
                         pararnn_info *info_dev, void *workspace, cudaStream_t s) {
    const LstmLayout L = lstm_layout(*cell, B, T);
    char *ws = static_cast<char *>(workspace);
    float *P = reinterpret_cast<float *>(ws + L.P);
    WsHeader *hdr = reinterpret_cast<WsHeader *>(ws + L.header);
    cudaError_t e = cudaMemsetAsync(ws + L.header, 0, 256, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(ws + L.desc, 0, L.total - L.desc, s);
    if (e == cudaSuccess)
        e = launch_projection_n(cell->x_dtype, x, params->w_ih, params->b_ih, P, static_cast<long long>(B) * T,
                                4 * cell->d, cell->din, s);
    if (e == cudaSuccess)
        e = launch_lstm_diag(P, params->w_hh, params->b_hh, c0, h0, B, T, cell->d, tol, max_iters,
                             reinterpret_cast<float *>(ws + L.cws), reinterpret_cast<float *>(ws + L.hws), c, h, hdr,
                             ws + L.desc, info_dev, s);
    return e;
}
}  // namespace

size_t pararnn_lstm_workspace_size(const pararnn_cell *cell, int B, int T) {
    return lstm_cell_ok(cell, B, T) ? lstm_layout(*cell, B, T).total : 0;
}

int pararnn_lstm_solve(const pararnn_cell *cell, const pararnn_params *params, const void *x, const float *c0,
                       const float *h0, int B, int T, float tol, int max_iters, float *c, float *h, pararnn_info *info,
                       void *workspace, size_t ws_bytes, pararnn_stream stream) {
    if (!lstm_cell_ok(cell, B, T) || !params || !params->w_ih || !params->b_ih || !params->w_hh || !params->b_hh)
        return PARARNN_INVALID_ARG;
    if (!x || !c0 || !h0 || !c || !h || !workspace || !(tol >= 0.f) || !std::isfinite(tol)) return PARARNN_INVALID_ARG;
    const LstmLayout L = lstm_layout(*cell, B, T);
    if (ws_bytes < L.total) return PARARNN_INVALID_ARG;
    const void *ptrs[] = {x, c0, h0, c, h, params->w_ih, params->b_ih, params->w_hh, params->b_hh};
    for (const void *q : ptrs)
        if (!aligned(q, 16)) return PARARNN_INVALID_ARG;
    if (!aligned(workspace, 256)) return PARARNN_INVALID_ARG;
    const size_t sb = static_cast<size_t>(B) * T * cell->d * 4;
    const size_t xb = static_cast<size_t>(B) * T * cell->din * (cell->x_dtype == PARARNN_BF16 ? 2 : 4);
    const size_t bd = static_cast<size_t>(B) * cell->d * 4;
    if (overlaps(c, sb, h, sb) || overlaps(c, sb, workspace, L.total) || overlaps(h, sb, workspace, L.total) ||
        overlaps(c, sb, x, xb) || overlaps(h, sb, x, xb) || overlaps(c, sb, c0, bd) || overlaps(c, sb, h0, bd) ||
        overlaps(h, sb, c0, bd) || overlaps(h, sb, h0, bd))
        return PARARNN_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const WsHeader *hdr = reinterpret_cast<const WsHeader *>(static_cast<char *>(workspace) + L.header);
    cudaError_t e = lstm_enqueue(cell, params, x, c0, h0, B, T, tol, max_iters, c, h, nullptr, workspace, s);
    pararnn_info host{};
    if (e == cudaSuccess) e = cudaMemcpyAsync(&host, &hdr->info, sizeof(host), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return PARARNN_CUDA_ERROR;
    if (info) *info = host;
    return host.status;
}

// ---- backward pass (diagonal cell) -------------------------------------------

namespace {
struct AdjLayout {
    size_t header, desc, part, hprev, G, grow, opart, total;
};
// dense: + h_{t-1} [B, T, D], U h_{t-1} + b_hh [B, T, 3D], grow [B, T, 3D] and
// the dW_hh GEMM's per-chunk partials
AdjLayout adj_layout(int B, int T, int D, bool dense) {
    AdjLayout L{};
    size_t off = 0;
    L.header = off; off += 256;
    L.desc = off; off = align256(off + adjoint_diag_desc_bytes(B, T, D));
    L.part = off; off = align256(off + adjoint_diag_part_bytes(B, T, D));
    if (dense) {
        const size_t st = static_cast<size_t>(B) * T * D * 4;
        L.hprev = off; off = align256(off + st);
        L.G = off; off = align256(off + 3 * st);
        L.grow = off; off = align256(off + 3 * st);
        L.opart = off; off = align256(off + adjoint_outer_part_bytes(static_cast<long long>(B) * T, 3 * D, D));
    }
    L.total = off;
    return L;
}
}  // namespace

size_t pararnn_adjoint_workspace_size(const pararnn_cell *cell, int B, int T) {
    if (!cell || cell->d < 1 || B < 1 || T < 1) return 0;
    if (cell->kind != PARARNN_GRU_DIAG && !(cell->kind == PARARNN_GRU_DENSE && cell->d <= 64)) return 0;
    if (static_cast<long long>(B) * T >= (1ll << 31) - 1) return 0;
    return adj_layout(B, T, cell->d, cell->kind == PARARNN_GRU_DENSE).total;
}

int pararnn_adjoint(const pararnn_cell *cell, const pararnn_params *params, const float *P, const float *h0,
                    const float *h, const float *dh, int B, int T, float *dP, float *dh0, float *dw_hh,
                    float *db_hh, void *workspace, size_t ws_bytes, pararnn_stream stream) {
    const size_t need = pararnn_adjoint_workspace_size(cell, B, T);
    if (need == 0 || ws_bytes < need || !params || !params->w_hh || !params->b_hh) return PARARNN_INVALID_ARG;
    if (!P || !h0 || !h || !dh || !dP || !dh0 || !dw_hh || !db_hh || !workspace) return PARARNN_INVALID_ARG;
    const void *ptrs[] = {P, h0, h, dh, dP, dh0, dw_hh, db_hh, params->w_hh, params->b_hh};
    for (const void *q : ptrs)
        if (!aligned(q, 16)) return PARARNN_INVALID_ARG;
    if (!aligned(workspace, 256)) return PARARNN_INVALID_ARG;
    const int D = cell->d;
    const bool dense = cell->kind == PARARNN_GRU_DENSE;
    const size_t st = static_cast<size_t>(B) * T * D * 4;
    const size_t bd = static_cast<size_t>(B) * D * 4, pd = static_cast<size_t>(3) * D * 4 * (dense ? D : 1);
    const size_t bb = static_cast<size_t>(3) * D * 4;  // b_hh and db_hh
    const struct { const void *p; size_t n; } ins[] = {{P, 3 * st}, {h0, bd}, {h, st}, {dh, st},
                                                       {params->w_hh, pd}, {params->b_hh, bb}, {workspace, need}};
    const struct { const void *p; size_t n; } outs[] = {{dP, 3 * st}, {dh0, bd}, {dw_hh, pd}, {db_hh, bb}};
    for (const auto &o : outs) {
        for (const auto &i : ins)
            if (overlaps(o.p, o.n, i.p, i.n)) return PARARNN_INVALID_ARG;
        for (const auto &o2 : outs)
            if (&o2 != &o && overlaps(o.p, o.n, o2.p, o2.n)) return PARARNN_INVALID_ARG;
    }
    const Range range("pararnn: backward pass");
    const cudaError_t e = adjoint_enqueue(cell, params, P, h0, h, dh, B, T, dP, dh0, dw_hh, db_hh, workspace,
                                          reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PARARNN_OK : PARARNN_CUDA_ERROR;
}

size_t pararnn_adjoint_exact_workspace_size(const pararnn_cell *cell, int B, int T) {
    if (!cell || cell->kind != PARARNN_GRU_DENSE || B < 1 || T < 1) return 0;
    if (cell->d < 4 || cell->d > 64 || cell->d % 4 != 0) return 0;
    if (static_cast<long long>(B) * T >= (1ll << 31) - 1) return 0;
    return adjoint_exact_ws_bytes(B, T, cell->d);
}

int pararnn_adjoint_exact(const pararnn_cell *cell, const pararnn_params *params, const float *P, const float *h0,
                          const float *h, const float *dh, int B, int T, float *dP, float *dh0, float *dw_hh,
                          float *db_hh, void *workspace, size_t ws_bytes, pararnn_stream stream) {
    const size_t need = pararnn_adjoint_exact_workspace_size(cell, B, T);
    if (need == 0 || ws_bytes < need || !params || !params->w_hh || !params->b_hh) return PARARNN_INVALID_ARG;
    if (!P || !h0 || !h || !dh || !dP || !dh0 || !dw_hh || !db_hh || !workspace) return PARARNN_INVALID_ARG;
    const void *ptrs[] = {P, h0, h, dh, dP, dh0, dw_hh, db_hh, params->w_hh, params->b_hh};
    for (const void *q : ptrs)
        if (!aligned(q, 16)) return PARARNN_INVALID_ARG;
    if (!aligned(workspace, 256)) return PARARNN_INVALID_ARG;
    const int D = cell->d;
    const size_t st = static_cast<size_t>(B) * T * D * 4;
    const size_t bd = static_cast<size_t>(B) * D * 4, pd = static_cast<size_t>(3) * D * D * 4;
    const size_t bb = static_cast<size_t>(3) * D * 4;
    const struct { const void *p; size_t n; } ins[] = {{P, 3 * st}, {h0, bd}, {h, st}, {dh, st},
                                                       {params->w_hh, pd}, {params->b_hh, bb}, {workspace, need}};
    const struct { const void *p; size_t n; } outs[] = {{dP, 3 * st}, {dh0, bd}, {dw_hh, pd}, {db_hh, bb}};
    for (const auto &o : outs) {
        for (const auto &i : ins)
            if (overlaps(o.p, o.n, i.p, i.n)) return PARARNN_INVALID_ARG;
        for (const auto &o2 : outs)
            if (&o2 != &o && overlaps(o.p, o.n, o2.p, o2.n)) return PARARNN_INVALID_ARG;
    }
    const Range range("pararnn: exact backward pass");
    const cudaError_t e = adjoint_exact_enqueue(params->w_hh, params->b_hh, P, h0, h, dh, B, T, D, dP, dh0, dw_hh,
                                                db_hh, workspace, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PARARNN_OK : PARARNN_CUDA_ERROR;
}

int pararnn_adjoint_status(const void *workspace, pararnn_stream stream) {
    return pararnn_affine_scan_status(workspace, stream);
}

}  // extern "C"

namespace pararnn {
// The backward pass enqueued on `s` (arguments already checked).
cudaError_t adjoint_enqueue(const pararnn_cell *cell, const pararnn_params *params, const float *P, const float *h0,
                            const float *h, const float *dh, int B, int T, float *dP, float *dh0, float *dw_hh,
                            float *db_hh, void *workspace, cudaStream_t s) {
    const int D = cell->d;
    const bool dense = cell->kind == PARARNN_GRU_DENSE;
    const AdjLayout L = adj_layout(B, T, D, dense);
    char *ws = static_cast<char *>(workspace);
    // header (status, grid barrier) and look-back words start at zero
    cudaError_t e = cudaMemsetAsync(ws, 0, L.part, s);
    if (!dense) {
        if (e == cudaSuccess)
            e = launch_adjoint_diag(P, h0, h, dh, params->w_hh, params->b_hh, dP, dh0, dw_hh, db_hh, B, T, D,
                                    ws + L.header, ws + L.desc, ws + L.part, s, nullptr, nullptr, nullptr);
        return e;
    }
    // dense cell: h_{t-1} packed [B, T, D] (h0, then the states shifted by one step)
    float *hp = reinterpret_cast<float *>(ws + L.hprev);
    const size_t row = static_cast<size_t>(D) * 4, seq = static_cast<size_t>(T) * D * 4;
    if (e == cudaSuccess) e = cudaMemcpy2DAsync(hp, seq, h0, row, row, B, cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess && T > 1)
        e = cudaMemcpy2DAsync(reinterpret_cast<char *>(hp) + row, seq, h, seq, seq - row, B, cudaMemcpyDeviceToDevice, s);
    // U h_{t-1} + b_hh for every step: one fp32 GEMM
    float *G = reinterpret_cast<float *>(ws + L.G);
    if (e == cudaSuccess)
        e = launch_projection_n(PARARNN_F32, hp, params->w_hh, params->b_hh, G, static_cast<long long>(B) * T, 3 * D,
                                D, s);
    // the reverse scan with the Jacobian's diagonal; dP, dh0, db_hh and grow
    float *grow = reinterpret_cast<float *>(ws + L.grow);
    if (e == cudaSuccess)
        e = launch_adjoint_diag(P, h0, h, dh, nullptr, params->b_hh, dP, dh0, nullptr, db_hh, B, T, D, ws + L.header,
                                ws + L.desc, ws + L.part, s, params->w_hh, G, grow);
    // dW_hh = sum over steps of grow (outer) h_{t-1}
    if (e == cudaSuccess)
        e = launch_outer_sum(grow, hp, static_cast<long long>(B) * T, 3 * D, D,
                             reinterpret_cast<float *>(ws + L.opart), dw_hh, s);
    return e;
}
}  // namespace pararnn

extern "C" {

const char *pararnn_status_string(int status) {
    switch (status) {
        case PARARNN_OK: return "PARARNN_OK";
        case PARARNN_NOT_CONVERGED: return "PARARNN_NOT_CONVERGED";
        case PARARNN_DIVERGED: return "PARARNN_DIVERGED";
        case PARARNN_INVALID_ARG: return "PARARNN_INVALID_ARG";
        case PARARNN_CUDA_ERROR: return "PARARNN_CUDA_ERROR";
        case PARARNN_TIMEOUT: return "PARARNN_TIMEOUT";
        default: return "PARARNN_UNKNOWN_STATUS";
    }
}


// ---- host-buffer solve: the batch in parts, copies overlapped with compute ----

namespace {

// Staging buffers for the parts' inputs and outputs.  With two, part p+2's
// input copy would wait for part p's output copy, so whenever both copies of a
// part take longer than one part's solve (PCIe: ~10 ms of copies against ~7 ms
// of solve on the dense workload) the copies would set the pace; three keep
// the solve busy.
constexpr int kHostBufs = 3;

// Sequences per part.  The first part's copy in and the last part's copy out
// overlap no solve, while a solve's cost per sequence falls as its part grows
// (fewer, shorter look-back chains per iteration), so the parts ramp up and
// down: weight min(p + 1, parts - p, 4) for part p (1, 2, 3, 4, ..., 4, 3, 2,
// 1), rounded by largest remainder with at least one sequence per part
// (parts <= B).  Each next part's copy in then fits under the solve before it.
std::vector<int> part_sizes(int B, int parts) {
    std::vector<int> w(parts);
    for (int p = 0; p < parts; ++p) w[p] = std::min(std::min(p + 1, parts - p), 4);
    long long W = 0;
    for (int v : w) W += v;
    std::vector<int> n(parts);
    std::vector<std::pair<long long, int>> rem(parts);
    int used = 0;
    for (int i = 0; i < parts; ++i) {
        const long long num = static_cast<long long>(B) * w[i];
        n[i] = static_cast<int>(num / W);
        rem[i] = {num % W, -i};
        used += n[i];
    }
    std::sort(rem.begin(), rem.end(), [](const auto &a, const auto &b) { return a > b; });
    for (int r = 0; used < B; ++r, ++used) ++n[-rem[r % parts].second];
    for (int i = 0; i < parts; ++i)  // at least one each: from the largest part
        while (n[i] == 0) {
            int j = 0;
            for (int q = 1; q < parts; ++q)
                if (n[q] > n[j]) j = q;
            --n[j];
            ++n[i];
        }
    return n;
}

struct HostLayout {
    int parts, bp, nbuf;  // number of parts, sequences of the largest part, buffers
    size_t solve, xs[kHostBufs], hs[kHostBufs], h0, infos, total;
};

HostLayout host_layout(const pararnn_cell &cell, int B, int T, int mode, int parts) {
    HostLayout H{};
    H.parts = parts;
    H.bp = 0;
    for (int v : part_sizes(B, parts)) H.bp = v > H.bp ? v : H.bp;
    H.nbuf = H.parts < kHostBufs ? H.parts : kHostBufs;
    const size_t es = cell.x_dtype == PARARNN_BF16 ? 2 : 4;
    const size_t xbytes = static_cast<size_t>(H.bp) * T * cell.din * es;
    const size_t hbytes = static_cast<size_t>(H.bp) * T * cell.d * 4;
    size_t off = 0;
    H.solve = off; off = align256(off + ws_layout(cell, H.bp, T, mode).total);
    for (int q = 0; q < H.nbuf; ++q) { H.xs[q] = off; off = align256(off + xbytes); }
    for (int q = 0; q < H.nbuf; ++q) { H.hs[q] = off; off = align256(off + hbytes); }
    H.h0 = off; off = align256(off + static_cast<size_t>(B) * cell.d * 4);
    H.infos = off; off = align256(off + static_cast<size_t>(parts) * sizeof(pararnn_info));
    H.total = off;
    return H;
}

// The host arrays one pipeline moves per part: up to three inputs and two
// outputs, [B, ...] with `row` bytes per sequence, staged in the workspace at
// off[q] for buffer q.
struct PipeIo {
    int nin = 0, nout = 0;
    const char *in[3] = {};
    char *out[2] = {};
    size_t in_row[3] = {}, out_row[2] = {};
    size_t in_off[3][kHostBufs] = {}, out_off[2][kHostBufs] = {};
};

// The pipeline's two helper streams and their events, created on a device's
// first host-buffer call and reused by later calls on that device (creating
// and destroying them cost a visible fraction of a short call).  A set is
// held by one call at a time; concurrent calls on one device take separate
// sets.  A set whose stream no longer answers (its context was reset) is
// dropped and a new one made.
struct PipeRes {
    int dev = -1;
    cudaStream_t s_in = nullptr, s_out = nullptr;
    cudaEvent_t ev[3 * kHostBufs + 1] = {};  // in[NB], comp[NB], out[NB], start / end
};
std::mutex g_pipe_mutex;
std::vector<PipeRes *> g_pipe_free;

void pipe_destroy(PipeRes *r) {
    for (cudaEvent_t &v : r->ev)
        if (v) cudaEventDestroy(v);
    if (r->s_in) cudaStreamDestroy(r->s_in);
    if (r->s_out) cudaStreamDestroy(r->s_out);
    delete r;
}

cudaError_t pipe_acquire(PipeRes **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    PipeRes *r = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_pipe_mutex);
        for (size_t i = 0; i < g_pipe_free.size(); ++i)
            if (g_pipe_free[i]->dev == dev) {
                r = g_pipe_free[i];
                g_pipe_free.erase(g_pipe_free.begin() + static_cast<long>(i));
                break;
            }
    }
    if (r != nullptr) {
        const cudaError_t q = cudaStreamQuery(r->s_in);
        if (q != cudaSuccess && q != cudaErrorNotReady) {  // stale: drop it without touching it
            cudaGetLastError();
            delete r;
            r = nullptr;
        }
    }
    if (r == nullptr) {
        r = new PipeRes;
        r->dev = dev;
        e = cudaStreamCreateWithFlags(&r->s_in, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&r->s_out, cudaStreamNonBlocking);
        for (int q = 0; q < 3 * kHostBufs + 1 && e == cudaSuccess; ++q)
            e = cudaEventCreateWithFlags(&r->ev[q], cudaEventDisableTiming);
        if (e != cudaSuccess) {
            pipe_destroy(r);
            return e;
        }
    }
    *out = r;
    return cudaSuccess;
}

void pipe_release(PipeRes *r, bool reuse) {
    if (!reuse) {
        pipe_destroy(r);
        return;
    }
    std::lock_guard<std::mutex> lock(g_pipe_mutex);
    g_pipe_free.push_back(r);
}

extern "C++" {  // templates: C++ linkage inside the exported block
// The parts of `sizes` through `nbuf` staging buffers: part p's inputs are
// copied in by cin(p, first, n, buf, s_in) on one helper stream, solved on `sc`
// by enq(p, first, n, buf) (returns a pararnn status), and its outputs copied
// out by cout(p, first, n, buf, s_out) on a second helper stream; `first` is
// the part's first sequence (batch parts) or step (time parts), n its count.
// pre(s_in) enqueues the copies made once per call (initial states).  On
// return `sc` is ordered after the last copy out.
template <class Pre, class In, class Enq, class Out>
int run_parts(const std::vector<int> &sizes, int nbuf, cudaStream_t sc, Pre pre, In cin, Enq enq, Out cout) {
    constexpr int NB = kHostBufs;
    PipeRes *res = nullptr;
    cudaError_t e = pipe_acquire(&res);
    if (e != cudaSuccess) return PARARNN_CUDA_ERROR;
    cudaStream_t s_in = res->s_in, s_out = res->s_out;
    cudaEvent_t *ev = res->ev;
    cudaEvent_t *ev_in = ev, *ev_comp = ev + NB, *ev_out = ev + 2 * NB, &ev_edge = ev[3 * NB];
    int rc = PARARNN_OK;
    if (e == cudaSuccess) {  // start only after the caller's earlier work on its stream
        e = cudaEventRecord(ev_edge, sc);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(s_in, ev_edge, 0);
        if (e == cudaSuccess) e = pre(s_in);
    }
    const int parts = static_cast<int>(sizes.size());
    int first = 0;
    for (int p = 0; p < parts && e == cudaSuccess && rc == PARARNN_OK; first += sizes[p], ++p) {
        const int buf = p % nbuf, n = sizes[p];
        if (p >= nbuf) e = cudaStreamWaitEvent(s_in, ev_out[buf], 0);  // staging of part p-nbuf free
        if (e == cudaSuccess) e = cin(p, first, n, buf, s_in);
        if (e == cudaSuccess) e = cudaEventRecord(ev_in[buf], s_in);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(sc, ev_in[buf], 0);
        if (e != cudaSuccess) break;
        {
            const Range range("pararnn: host-buffer part");
            rc = enq(p, first, n, buf);
        }
        if (rc != PARARNN_OK) break;
        e = cudaEventRecord(ev_comp[buf], sc);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(s_out, ev_comp[buf], 0);
        if (e == cudaSuccess) e = cout(p, first, n, buf, s_out);
        if (e == cudaSuccess) e = cudaEventRecord(ev_out[buf], s_out);
    }
    if (e == cudaSuccess && rc == PARARNN_OK) {  // the caller's stream continues after the last copy out
        e = cudaEventRecord(ev_edge, s_out);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(sc, ev_edge, 0);
    }
    // leave nothing in flight on the helper streams before the set is handed on
    const cudaError_t e1 = cudaStreamSynchronize(s_in);
    const cudaError_t e2 = cudaStreamSynchronize(s_out);
    pipe_release(res, e == cudaSuccess && e1 == cudaSuccess && e2 == cudaSuccess);
    if (e != cudaSuccess) return PARARNN_CUDA_ERROR;
    return rc;
}

// The batch in ramped parts (part_sizes): whole sequences of every array in `io`.
template <class Pre, class Enq>
int run_pipeline(int B, int parts, int nbuf, const PipeIo &io, char *ws, cudaStream_t sc, Pre pre, Enq enq) {
    auto cin = [&](int, int b0, int nb, int buf, cudaStream_t s) {
        cudaError_t e = cudaSuccess;
        for (int a = 0; a < io.nin && e == cudaSuccess; ++a)
            e = cudaMemcpyAsync(ws + io.in_off[a][buf], io.in[a] + b0 * io.in_row[a], nb * io.in_row[a],
                                cudaMemcpyHostToDevice, s);
        return e;
    };
    auto cout = [&](int, int b0, int nb, int buf, cudaStream_t s) {
        cudaError_t e = cudaSuccess;
        for (int a = 0; a < io.nout && e == cudaSuccess; ++a)
            e = cudaMemcpyAsync(io.out[a] + b0 * io.out_row[a], ws + io.out_off[a][buf], nb * io.out_row[a],
                                cudaMemcpyDeviceToHost, s);
        return e;
    };
    return run_parts(part_sizes(B, parts), nbuf, sc, pre, cin, enq, cout);
}
}  // extern "C++"

// Wait for `sc`, read the parts' reports and fold them: the worst part
// (statuses are ordered by severity), the largest count (or, with sum_iters,
// the total over parts), delta and residual.
int fold_reports(const pararnn_info *infos_dev, int parts, cudaStream_t sc, pararnn_info *info,
                 bool sum_iters = false) {
    std::vector<pararnn_info> host(parts);
    cudaError_t e = cudaMemcpyAsync(host.data(), infos_dev, parts * sizeof(pararnn_info), cudaMemcpyDeviceToHost, sc);
    if (e == cudaSuccess) e = cudaStreamSynchronize(sc);
    if (e != cudaSuccess) return PARARNN_CUDA_ERROR;
    pararnn_info agg{};
    for (int p = 0; p < parts; ++p) {
        agg.iters = sum_iters ? agg.iters + host[p].iters : (host[p].iters > agg.iters ? host[p].iters : agg.iters);
        agg.status = host[p].status > agg.status ? host[p].status : agg.status;
        agg.delta = host[p].delta > agg.delta ? host[p].delta : agg.delta;
        agg.residual = host[p].residual > agg.residual ? host[p].residual : agg.residual;
    }
    if (info) *info = agg;
    return agg.status;
}

struct LstmHostLayout {
    int bp, nbuf;
    size_t solve, xs[kHostBufs], cs[kHostBufs], hs[kHostBufs], c0, h0, infos, total;
};

LstmHostLayout lstm_host_layout(const pararnn_cell &cell, int B, int T, int parts) {
    LstmHostLayout H{};
    for (int v : part_sizes(B, parts)) H.bp = v > H.bp ? v : H.bp;
    H.nbuf = parts < kHostBufs ? parts : kHostBufs;
    const size_t es = cell.x_dtype == PARARNN_BF16 ? 2 : 4;
    const size_t xbytes = static_cast<size_t>(H.bp) * T * cell.din * es;
    const size_t sbytes = static_cast<size_t>(H.bp) * T * cell.d * 4;
    size_t off = 0;
    H.solve = off; off = align256(off + lstm_layout(cell, H.bp, T).total);
    for (int q = 0; q < H.nbuf; ++q) { H.xs[q] = off; off = align256(off + xbytes); }
    for (int q = 0; q < H.nbuf; ++q) { H.cs[q] = off; off = align256(off + sbytes); }
    for (int q = 0; q < H.nbuf; ++q) { H.hs[q] = off; off = align256(off + sbytes); }
    H.c0 = off; off = align256(off + static_cast<size_t>(B) * cell.d * 4);
    H.h0 = off; off = align256(off + static_cast<size_t>(B) * cell.d * 4);
    H.infos = off; off = align256(off + static_cast<size_t>(parts) * sizeof(pararnn_info));
    H.total = off;
    return H;
}

struct AdjHostLayout {
    int bp, nbuf;
    size_t solve, Ps[kHostBufs], hs[kHostBufs], dhs[kHostBufs], dPs[kHostBufs], h0, dh0, dwp, dbp, dw, db, stat,
        total;
};

// dW_hh per part: 3D (diagonal cell) or 3D x D (dense) floats.
size_t adj_param_floats(const pararnn_cell &cell) {
    return static_cast<size_t>(3) * cell.d * (cell.kind == PARARNN_GRU_DENSE ? cell.d : 1);
}

AdjHostLayout adj_host_layout(const pararnn_cell &cell, int B, int T, int parts) {
    AdjHostLayout H{};
    for (int v : part_sizes(B, parts)) H.bp = v > H.bp ? v : H.bp;
    H.nbuf = parts < kHostBufs ? parts : kHostBufs;
    const size_t st = static_cast<size_t>(H.bp) * T * cell.d * 4, bd = static_cast<size_t>(B) * cell.d * 4;
    size_t off = 0;
    H.solve = off; off = align256(off + pararnn_adjoint_workspace_size(&cell, H.bp, T));
    for (int q = 0; q < H.nbuf; ++q) { H.Ps[q] = off; off = align256(off + 3 * st); }
    for (int q = 0; q < H.nbuf; ++q) { H.hs[q] = off; off = align256(off + st); }
    for (int q = 0; q < H.nbuf; ++q) { H.dhs[q] = off; off = align256(off + st); }
    for (int q = 0; q < H.nbuf; ++q) { H.dPs[q] = off; off = align256(off + 3 * st); }
    H.h0 = off; off = align256(off + bd);
    H.dh0 = off; off = align256(off + bd);
    H.dwp = off; off = align256(off + static_cast<size_t>(parts) * adj_param_floats(cell) * 4);
    H.dbp = off; off = align256(off + static_cast<size_t>(parts) * 3 * cell.d * 4);
    H.dw = off; off = align256(off + adj_param_floats(cell) * 4);
    H.db = off; off = align256(off + static_cast<size_t>(3) * cell.d * 4);
    H.stat = off; off = align256(off + static_cast<size_t>(parts) * 4);
    H.total = off;
    return H;
}

}  // namespace

size_t pararnn_adjoint_host_workspace_size(const pararnn_cell *cell, int B, int T, int parts) {
    if (pararnn_adjoint_workspace_size(cell, B, T) == 0 || parts < 1 || parts > B) return 0;
    return adj_host_layout(*cell, B, T, parts).total;
}

int pararnn_adjoint_host(const pararnn_cell *cell, const pararnn_params *params, const float *P_host,
                         const float *h0_host, const float *h_host, const float *dh_host, int B, int T, float *dP_host,
                         float *dh0_host, float *dw_hh_host, float *db_hh_host, int parts, void *workspace,
                         size_t ws_bytes, pararnn_stream stream) {
    if (pararnn_adjoint_workspace_size(cell, B, T) == 0 || parts < 1 || parts > B || !params || !params->w_hh ||
        !params->b_hh || !P_host || !h0_host || !h_host || !dh_host || !dP_host || !dh0_host || !dw_hh_host ||
        !db_hh_host || !workspace || !aligned(workspace, 256) || !aligned(params->w_hh, 16) ||
        !aligned(params->b_hh, 16))
        return PARARNN_INVALID_ARG;
    const AdjHostLayout H = adj_host_layout(*cell, B, T, parts);
    if (ws_bytes < H.total) return PARARNN_INVALID_ARG;
    char *ws = static_cast<char *>(workspace);
    const int D = cell->d;
    const size_t srow = static_cast<size_t>(T) * D * 4, pf = adj_param_floats(*cell);
    PipeIo io;  // in: P, h, dL/dh; out: dL/dP
    io.nin = 3;
    io.nout = 1;
    io.in[0] = reinterpret_cast<const char *>(P_host);
    io.in[1] = reinterpret_cast<const char *>(h_host);
    io.in[2] = reinterpret_cast<const char *>(dh_host);
    io.in_row[0] = 3 * srow;
    io.in_row[1] = io.in_row[2] = srow;
    io.out[0] = reinterpret_cast<char *>(dP_host);
    io.out_row[0] = 3 * srow;
    for (int q = 0; q < H.nbuf; ++q)
        io.in_off[0][q] = H.Ps[q], io.in_off[1][q] = H.hs[q], io.in_off[2][q] = H.dhs[q], io.out_off[0][q] = H.dPs[q];
    cudaStream_t sc = reinterpret_cast<cudaStream_t>(stream);
    float *h0_dev = reinterpret_cast<float *>(ws + H.h0), *dh0_dev = reinterpret_cast<float *>(ws + H.dh0);
    float *dwp = reinterpret_cast<float *>(ws + H.dwp), *dbp = reinterpret_cast<float *>(ws + H.dbp);
    unsigned *stat = reinterpret_cast<unsigned *>(ws + H.stat);
    const WsHeader *shdr = reinterpret_cast<const WsHeader *>(ws + H.solve);
    const size_t bd = static_cast<size_t>(B) * D * 4;
    auto pre = [&](cudaStream_t s_in) {
        return cudaMemcpyAsync(h0_dev, h0_host, bd, cudaMemcpyHostToDevice, s_in);
    };
    auto enq = [&](int p, int b0, int nb, int buf) {
        const size_t o = static_cast<size_t>(b0) * D;
        cudaError_t e = adjoint_enqueue(cell, params, reinterpret_cast<const float *>(ws + H.Ps[buf]), h0_dev + o,
                                reinterpret_cast<const float *>(ws + H.hs[buf]),
                                reinterpret_cast<const float *>(ws + H.dhs[buf]), nb, T,
                                reinterpret_cast<float *>(ws + H.dPs[buf]), dh0_dev + o, dwp + p * pf,
                                dbp + static_cast<size_t>(p) * 3 * D, ws + H.solve, sc);
        if (e == cudaSuccess)  // the part's bounded-wait status, before the next part clears it
            e = cudaMemcpyAsync(stat + p, &shdr->status, sizeof(unsigned), cudaMemcpyDeviceToDevice, sc);
        return e == cudaSuccess ? PARARNN_OK : PARARNN_CUDA_ERROR;
    };
    int rc = run_pipeline(B, parts, H.nbuf, io, ws, sc, pre, enq);
    if (rc != PARARNN_OK) return rc;
    // the parameter gradients: the parts' sums added in part order
    float *dw = reinterpret_cast<float *>(ws + H.dw), *db = reinterpret_cast<float *>(ws + H.db);
    std::vector<unsigned> hstat(parts);
    cudaError_t e = launch_sum_rows(dwp, parts, static_cast<int>(pf), dw, sc);
    if (e == cudaSuccess) e = launch_sum_rows(dbp, parts, 3 * D, db, sc);
    if (e == cudaSuccess) e = cudaMemcpyAsync(dw_hh_host, dw, pf * 4, cudaMemcpyDeviceToHost, sc);
    if (e == cudaSuccess) e = cudaMemcpyAsync(db_hh_host, db, static_cast<size_t>(3) * D * 4, cudaMemcpyDeviceToHost, sc);
    if (e == cudaSuccess) e = cudaMemcpyAsync(dh0_host, dh0_dev, bd, cudaMemcpyDeviceToHost, sc);
    if (e == cudaSuccess) e = cudaMemcpyAsync(hstat.data(), stat, parts * sizeof(unsigned), cudaMemcpyDeviceToHost, sc);
    if (e == cudaSuccess) e = cudaStreamSynchronize(sc);
    if (e != cudaSuccess) return PARARNN_CUDA_ERROR;
    for (unsigned v : hstat)
        if (v != 0u) return PARARNN_TIMEOUT;
    return PARARNN_OK;
}

size_t pararnn_host_workspace_size(const pararnn_cell *cell, int B, int T, int mode, int parts) {
    if (!cell_ok(cell, B, T, mode) || parts < 1 || parts > B) return 0;
    return host_layout(*cell, B, T, mode, parts).total;
}

int pararnn_newton_solve_host(const pararnn_cell *cell, const pararnn_params *params, const void *x_host,
                              const float *h0_host, int B, int T, int mode, float lambda, float tol,
                              int max_iters, float *h_host, pararnn_info *info, int parts,
                              void *workspace, size_t ws_bytes, pararnn_stream stream) {
    if (!cell_ok(cell, B, T, mode) || parts < 1 || parts > B || !params || !x_host || !h0_host ||
        !h_host || !workspace || !aligned(workspace, 256))
        return PARARNN_INVALID_ARG;
    const HostLayout H = host_layout(*cell, B, T, mode, parts);
    if (ws_bytes < H.total) return PARARNN_INVALID_ARG;
    char *ws = static_cast<char *>(workspace);
    const size_t es = cell->x_dtype == PARARNN_BF16 ? 2 : 4;
    PipeIo io;
    io.nin = io.nout = 1;
    io.in[0] = static_cast<const char *>(x_host);
    io.in_row[0] = static_cast<size_t>(T) * cell->din * es;  // bytes of one sequence's input
    io.out[0] = reinterpret_cast<char *>(h_host);
    io.out_row[0] = static_cast<size_t>(T) * cell->d * 4;    // bytes of one sequence's states
    for (int q = 0; q < H.nbuf; ++q) io.in_off[0][q] = H.xs[q], io.out_off[0][q] = H.hs[q];
    cudaStream_t sc = reinterpret_cast<cudaStream_t>(stream);
    float *h0_dev = reinterpret_cast<float *>(ws + H.h0);
    pararnn_info *infos = reinterpret_cast<pararnn_info *>(ws + H.infos);
    auto pre = [&](cudaStream_t s_in) {
        return cudaMemcpyAsync(h0_dev, h0_host, static_cast<size_t>(B) * cell->d * 4, cudaMemcpyHostToDevice, s_in);
    };
    auto enq = [&](int p, int b0, int nb, int buf) {
        return solve_enqueue(cell, params, ws + H.xs[buf], h0_dev + static_cast<size_t>(b0) * cell->d, nb, T, mode,
                             lambda, tol, max_iters, reinterpret_cast<float *>(ws + H.hs[buf]), infos + p,
                             ws + H.solve, ws_layout(*cell, nb, T, mode).total, stream);
    };
    const int rc = run_pipeline(B, parts, H.nbuf, io, ws, sc, pre, enq);
    if (rc != PARARNN_OK) return rc;
    return fold_reports(infos, parts, sc, info);
}

namespace {

// Steps per time part: whole 128-step units (the solvers' tile length) with the
// ramped weights of part_sizes; the last part ends at T.  parts <= ceil(T / 128).
std::vector<int> time_part_sizes(int T, int parts) {
    const int units = (T + 127) / 128;
    std::vector<int> n = part_sizes(units, parts);
    for (int &v : n) v *= 128;
    n.back() -= units * 128 - T;
    return n;
}

struct StreamLayout {
    int tmax, nbuf;  // steps of the longest part, staging buffers
    size_t solve, xs[kHostBufs], hs[kHostBufs], h0, carry, infos, total;
};

StreamLayout stream_layout(const pararnn_cell &cell, int B, int T, int mode, int parts) {
    StreamLayout H{};
    for (int v : time_part_sizes(T, parts)) H.tmax = v > H.tmax ? v : H.tmax;
    H.nbuf = parts < kHostBufs ? parts : kHostBufs;
    const size_t es = cell.x_dtype == PARARNN_BF16 ? 2 : 4;
    const size_t xbytes = static_cast<size_t>(B) * H.tmax * cell.din * es;
    const size_t hbytes = static_cast<size_t>(B) * H.tmax * cell.d * 4;
    size_t off = 0;
    H.solve = off; off = align256(off + ws_layout(cell, B, H.tmax, mode).total);
    for (int q = 0; q < H.nbuf; ++q) { H.xs[q] = off; off = align256(off + xbytes); }
    for (int q = 0; q < H.nbuf; ++q) { H.hs[q] = off; off = align256(off + hbytes); }
    H.h0 = off; off = align256(off + static_cast<size_t>(B) * cell.d * 4);
    H.carry = off; off = align256(off + static_cast<size_t>(B) * cell.d * 4);
    H.infos = off; off = align256(off + static_cast<size_t>(parts) * sizeof(pararnn_info));
    H.total = off;
    return H;
}

}  // namespace

size_t pararnn_host_streamed_workspace_size(const pararnn_cell *cell, int B, int T, int mode, int parts) {
    if (!cell_ok(cell, B, T, mode) || parts < 1 || parts > (T + 127) / 128) return 0;
    return stream_layout(*cell, B, T, mode, parts).total;
}

int pararnn_newton_solve_host_streamed(const pararnn_cell *cell, const pararnn_params *params,
                                       const void *x_host, const float *h0_host, int B, int T, int mode,
                                       float lambda, float tol, int max_iters, float *h_host, pararnn_info *info,
                                       int parts, void *workspace, size_t ws_bytes, pararnn_stream stream) {
    if (!cell_ok(cell, B, T, mode) || parts < 1 || parts > (T + 127) / 128 || !params || !x_host ||
        !h0_host || !h_host || !workspace || !aligned(workspace, 256))
        return PARARNN_INVALID_ARG;
    const StreamLayout H = stream_layout(*cell, B, T, mode, parts);
    if (ws_bytes < H.total) return PARARNN_INVALID_ARG;
    char *ws = static_cast<char *>(workspace);
    const size_t es = cell->x_dtype == PARARNN_BF16 ? 2 : 4;
    const size_t xstep = static_cast<size_t>(cell->din) * es, hstep = static_cast<size_t>(cell->d) * 4;
    const std::vector<int> sizes = time_part_sizes(T, parts);
    cudaStream_t sc = reinterpret_cast<cudaStream_t>(stream);
    float *h0_dev = reinterpret_cast<float *>(ws + H.h0), *carry = reinterpret_cast<float *>(ws + H.carry);
    pararnn_info *infos = reinterpret_cast<pararnn_info *>(ws + H.infos);
    const char *xh = static_cast<const char *>(x_host);
    char *hh = reinterpret_cast<char *>(h_host);
    // the cap of the whole sequence's solve (T + 1 by default), as for the chunked solve
    const int cap = max_iters > 0 ? max_iters : T + 1;
    auto pre = [&](cudaStream_t s_in) {
        return cudaMemcpyAsync(h0_dev, h0_host, B * hstep, cudaMemcpyHostToDevice, s_in);
    };
    // steps [t0, t0 + n) of every sequence: rows of the host arrays, packed [B, n, .] in staging
    auto cin = [&](int, int t0, int n, int buf, cudaStream_t s) {
        return cudaMemcpy2DAsync(ws + H.xs[buf], n * xstep, xh + t0 * xstep, T * xstep, n * xstep, B,
                                 cudaMemcpyHostToDevice, s);
    };
    auto enq = [&](int p, int, int n, int buf) {
        const float *hin = h0_dev;
        if (p > 0) {  // the state entering the part: each sequence's last state of the part before
            const int pb = (p - 1) % H.nbuf, pn = sizes[p - 1];
            if (cudaMemcpy2DAsync(carry, hstep, ws + H.hs[pb] + (pn - 1) * hstep, pn * hstep, hstep, B,
                                  cudaMemcpyDeviceToDevice, sc) != cudaSuccess)
                return static_cast<int>(PARARNN_CUDA_ERROR);
            hin = carry;
        }
        return solve_enqueue(cell, params, ws + H.xs[buf], hin, B, n, mode, lambda, tol, cap,
                             reinterpret_cast<float *>(ws + H.hs[buf]), infos + p, ws + H.solve,
                             ws_layout(*cell, B, n, mode).total, stream);
    };
    auto cout = [&](int, int t0, int n, int buf, cudaStream_t s) {
        return cudaMemcpy2DAsync(hh + t0 * hstep, T * hstep, ws + H.hs[buf], n * hstep, n * hstep, B,
                                 cudaMemcpyDeviceToHost, s);
    };
    const int rc = run_parts(sizes, H.nbuf, sc, pre, cin, enq, cout);
    if (rc != PARARNN_OK) return rc;
    return fold_reports(infos, parts, sc, info, true);
}

namespace {

struct LstmStreamLayout {
    int tmax, nbuf;
    size_t solve, xs[kHostBufs], cs[kHostBufs], hs[kHostBufs], c0, h0, cc, hc, infos, total;
};

LstmStreamLayout lstm_stream_layout(const pararnn_cell &cell, int B, int T, int parts) {
    LstmStreamLayout H{};
    for (int v : time_part_sizes(T, parts)) H.tmax = v > H.tmax ? v : H.tmax;
    H.nbuf = parts < kHostBufs ? parts : kHostBufs;
    const size_t es = cell.x_dtype == PARARNN_BF16 ? 2 : 4;
    const size_t xbytes = static_cast<size_t>(B) * H.tmax * cell.din * es;
    const size_t sbytes = static_cast<size_t>(B) * H.tmax * cell.d * 4;
    const size_t bd = static_cast<size_t>(B) * cell.d * 4;
    size_t off = 0;
    H.solve = off; off = align256(off + lstm_layout(cell, B, H.tmax).total);
    for (int q = 0; q < H.nbuf; ++q) { H.xs[q] = off; off = align256(off + xbytes); }
    for (int q = 0; q < H.nbuf; ++q) { H.cs[q] = off; off = align256(off + sbytes); }
    for (int q = 0; q < H.nbuf; ++q) { H.hs[q] = off; off = align256(off + sbytes); }
    H.c0 = off; off = align256(off + bd);
    H.h0 = off; off = align256(off + bd);
    H.cc = off; off = align256(off + bd);
    H.hc = off; off = align256(off + bd);
    H.infos = off; off = align256(off + static_cast<size_t>(parts) * sizeof(pararnn_info));
    H.total = off;
    return H;
}

}  // namespace

size_t pararnn_lstm_host_streamed_workspace_size(const pararnn_cell *cell, int B, int T, int parts) {
    if (!lstm_cell_ok(cell, B, T) || parts < 1 || parts > (T + 127) / 128) return 0;
    return lstm_stream_layout(*cell, B, T, parts).total;
}

int pararnn_lstm_solve_host_streamed(const pararnn_cell *cell, const pararnn_params *params, const void *x_host,
                                     const float *c0_host, const float *h0_host, int B, int T, float tol,
                                     int max_iters, float *c_host, float *h_host, pararnn_info *info, int parts,
                                     void *workspace, size_t ws_bytes, pararnn_stream stream) {
    if (!lstm_cell_ok(cell, B, T) || parts < 1 || parts > (T + 127) / 128 || !params || !params->w_ih ||
        !params->b_ih || !params->w_hh || !params->b_hh || !x_host || !c0_host || !h0_host || !c_host || !h_host ||
        !workspace || !aligned(workspace, 256) || !(tol >= 0.f) || !std::isfinite(tol))
        return PARARNN_INVALID_ARG;
    const void *ptrs[] = {params->w_ih, params->b_ih, params->w_hh, params->b_hh};
    for (const void *q : ptrs)
        if (!aligned(q, 16)) return PARARNN_INVALID_ARG;
    const LstmStreamLayout H = lstm_stream_layout(*cell, B, T, parts);
    if (ws_bytes < H.total) return PARARNN_INVALID_ARG;
    char *ws = static_cast<char *>(workspace);
    const size_t es = cell->x_dtype == PARARNN_BF16 ? 2 : 4;
    const size_t xstep = static_cast<size_t>(cell->din) * es, sstep = static_cast<size_t>(cell->d) * 4;
    const std::vector<int> sizes = time_part_sizes(T, parts);
    cudaStream_t sc = reinterpret_cast<cudaStream_t>(stream);
    float *c0_dev = reinterpret_cast<float *>(ws + H.c0), *h0_dev = reinterpret_cast<float *>(ws + H.h0);
    float *cc = reinterpret_cast<float *>(ws + H.cc), *hc = reinterpret_cast<float *>(ws + H.hc);
    pararnn_info *infos = reinterpret_cast<pararnn_info *>(ws + H.infos);
    const char *xh = static_cast<const char *>(x_host);
    char *ch = reinterpret_cast<char *>(c_host), *hh = reinterpret_cast<char *>(h_host);
    const int cap = max_iters > 0 ? max_iters : T + 1;  // the whole sequence's cap
    auto pre = [&](cudaStream_t s_in) {
        cudaError_t e = cudaMemcpyAsync(c0_dev, c0_host, B * sstep, cudaMemcpyHostToDevice, s_in);
        if (e == cudaSuccess) e = cudaMemcpyAsync(h0_dev, h0_host, B * sstep, cudaMemcpyHostToDevice, s_in);
        return e;
    };
    auto cin = [&](int, int t0, int n, int buf, cudaStream_t s) {
        return cudaMemcpy2DAsync(ws + H.xs[buf], n * xstep, xh + t0 * xstep, T * xstep, n * xstep, B,
                                 cudaMemcpyHostToDevice, s);
    };
    auto enq = [&](int p, int, int n, int buf) {
        const float *cin0 = c0_dev, *hin0 = h0_dev;
        cudaError_t e = cudaSuccess;
        if (p > 0) {  // (c, h) entering the part: each sequence's last state of the part before
            const int pb = (p - 1) % H.nbuf, pn = sizes[p - 1];
            e = cudaMemcpy2DAsync(cc, sstep, ws + H.cs[pb] + (pn - 1) * sstep, pn * sstep, sstep, B,
                                  cudaMemcpyDeviceToDevice, sc);
            if (e == cudaSuccess)
                e = cudaMemcpy2DAsync(hc, sstep, ws + H.hs[pb] + (pn - 1) * sstep, pn * sstep, sstep, B,
                                      cudaMemcpyDeviceToDevice, sc);
            cin0 = cc;
            hin0 = hc;
        }
        if (e == cudaSuccess)
            e = lstm_enqueue(cell, params, ws + H.xs[buf], cin0, hin0, B, n, tol, cap,
                             reinterpret_cast<float *>(ws + H.cs[buf]), reinterpret_cast<float *>(ws + H.hs[buf]),
                             infos + p, ws + H.solve, sc);
        return e == cudaSuccess ? PARARNN_OK : PARARNN_CUDA_ERROR;
    };
    auto cout = [&](int, int t0, int n, int buf, cudaStream_t s) {
        cudaError_t e = cudaMemcpy2DAsync(ch + t0 * sstep, T * sstep, ws + H.cs[buf], n * sstep, n * sstep, B,
                                          cudaMemcpyDeviceToHost, s);
        if (e == cudaSuccess)
            e = cudaMemcpy2DAsync(hh + t0 * sstep, T * sstep, ws + H.hs[buf], n * sstep, n * sstep, B,
                                  cudaMemcpyDeviceToHost, s);
        return e;
    };
    const int rc = run_parts(sizes, H.nbuf, sc, pre, cin, enq, cout);
    if (rc != PARARNN_OK) return rc;
    return fold_reports(infos, parts, sc, info, true);
}

namespace {

struct ScanStreamLayout {
    int tmax, nbuf;
    size_t scan, As[kHostBufs], bs[kHostBufs], hs[kHostBufs], h0, carry, stat, total;
};

ScanStreamLayout scan_stream_layout(int B, int T, int D, int dense, int parts) {
    ScanStreamLayout H{};
    for (int v : time_part_sizes(T, parts)) H.tmax = v > H.tmax ? v : H.tmax;
    H.nbuf = parts < kHostBufs ? parts : kHostBufs;
    const size_t n = static_cast<size_t>(B) * H.tmax * D * 4;
    const size_t nA = n * (dense ? D : 1);
    const size_t bd = static_cast<size_t>(B) * D * 4;
    size_t off = 0;
    H.scan = off; off = align256(off + pararnn_affine_scan_workspace_size(B, H.tmax, D, dense));
    for (int q = 0; q < H.nbuf; ++q) { H.As[q] = off; off = align256(off + nA); }
    for (int q = 0; q < H.nbuf; ++q) { H.bs[q] = off; off = align256(off + n); }
    for (int q = 0; q < H.nbuf; ++q) { H.hs[q] = off; off = align256(off + n); }
    H.h0 = off; off = align256(off + bd);
    H.carry = off; off = align256(off + bd);
    H.stat = off; off = align256(off + static_cast<size_t>(parts) * 4);
    H.total = off;
    return H;
}

}  // namespace

size_t pararnn_affine_scan_host_workspace_size(int B, int T, int D, int dense, int parts) {
    if (pararnn_affine_scan_workspace_size(B, T, D, dense) == 0 || parts < 1 || parts > (T + 127) / 128) return 0;
    return scan_stream_layout(B, T, D, dense, parts).total;
}

int pararnn_affine_scan_host(const float *A_host, const float *b_host, const float *h0_host, int B, int T, int D,
                             int dense, float *h_host, int parts, void *workspace, size_t ws_bytes,
                             pararnn_stream stream) {
    if (pararnn_affine_scan_workspace_size(B, T, D, dense) == 0 || parts < 1 || parts > (T + 127) / 128 ||
        !A_host || !b_host || !h0_host || !h_host || !workspace || !aligned(workspace, 256))
        return PARARNN_INVALID_ARG;
    const ScanStreamLayout H = scan_stream_layout(B, T, D, dense, parts);
    if (ws_bytes < H.total) return PARARNN_INVALID_ARG;
    char *ws = static_cast<char *>(workspace);
    const size_t hstep = static_cast<size_t>(D) * 4, astep = hstep * (dense ? D : 1);
    const std::vector<int> sizes = time_part_sizes(T, parts);
    cudaStream_t sc = reinterpret_cast<cudaStream_t>(stream);
    float *h0_dev = reinterpret_cast<float *>(ws + H.h0), *carry = reinterpret_cast<float *>(ws + H.carry);
    unsigned *stat = reinterpret_cast<unsigned *>(ws + H.stat);
    const char *Ah = reinterpret_cast<const char *>(A_host), *bh = reinterpret_cast<const char *>(b_host);
    char *hh = reinterpret_cast<char *>(h_host);
    auto pre = [&](cudaStream_t s_in) {
        return cudaMemcpyAsync(h0_dev, h0_host, B * hstep, cudaMemcpyHostToDevice, s_in);
    };
    // steps [t0, t0 + n) of every sequence, packed [B, n, .] in staging
    auto cin = [&](int, int t0, int n, int buf, cudaStream_t s) {
        cudaError_t e = cudaMemcpy2DAsync(ws + H.As[buf], n * astep, Ah + t0 * astep, T * astep, n * astep, B,
                                          cudaMemcpyHostToDevice, s);
        if (e == cudaSuccess)
            e = cudaMemcpy2DAsync(ws + H.bs[buf], n * hstep, bh + t0 * hstep, T * hstep, n * hstep, B,
                                  cudaMemcpyHostToDevice, s);
        return e;
    };
    auto enq = [&](int p, int, int n, int buf) {
        const float *hin = h0_dev;
        cudaError_t e = cudaSuccess;
        if (p > 0) {  // the state entering the part: each sequence's last state of the part before
            const int pb = (p - 1) % H.nbuf, pn = sizes[p - 1];
            e = cudaMemcpy2DAsync(carry, hstep, ws + H.hs[pb] + (pn - 1) * hstep, pn * hstep, hstep, B,
                                  cudaMemcpyDeviceToDevice, sc);
            hin = carry;
        }
        const Range range("pararnn: affine scan");
        const float *Ap = reinterpret_cast<const float *>(ws + H.As[buf]);
        const float *bp = reinterpret_cast<const float *>(ws + H.bs[buf]);
        float *hp = reinterpret_cast<float *>(ws + H.hs[buf]);
        if (e == cudaSuccess)
            e = dense ? launch_scan_dense(Ap, bp, hin, B, n, D, hp, ws + H.scan, sc)
                      : launch_scan_diag(Ap, bp, hin, B, n, D, hp, ws + H.scan, sc);
        // the part's status word, kept before the next part's scan clears it
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(stat + p, &reinterpret_cast<const WsHeader *>(ws + H.scan)->status, 4,
                                cudaMemcpyDeviceToDevice, sc);
        return e == cudaSuccess ? static_cast<int>(PARARNN_OK) : static_cast<int>(PARARNN_CUDA_ERROR);
    };
    auto cout = [&](int, int t0, int n, int buf, cudaStream_t s) {
        return cudaMemcpy2DAsync(hh + t0 * hstep, T * hstep, ws + H.hs[buf], n * hstep, n * hstep, B,
                                 cudaMemcpyDeviceToHost, s);
    };
    const int rc = run_parts(sizes, H.nbuf, sc, pre, cin, enq, cout);
    if (rc != PARARNN_OK) return rc;
    std::vector<unsigned> host(parts);
    cudaError_t e = cudaMemcpyAsync(host.data(), stat, parts * 4, cudaMemcpyDeviceToHost, sc);
    if (e == cudaSuccess) e = cudaStreamSynchronize(sc);
    if (e != cudaSuccess) return PARARNN_CUDA_ERROR;
    for (unsigned v : host)
        if (v & kStatusTimeout) return PARARNN_TIMEOUT;
    return PARARNN_OK;
}

size_t pararnn_lstm_host_workspace_size(const pararnn_cell *cell, int B, int T, int parts) {
    if (!lstm_cell_ok(cell, B, T) || parts < 1 || parts > B) return 0;
    return lstm_host_layout(*cell, B, T, parts).total;
}

int pararnn_lstm_solve_host(const pararnn_cell *cell, const pararnn_params *params, const void *x_host,
                            const float *c0_host, const float *h0_host, int B, int T, float tol, int max_iters,
                            float *c_host, float *h_host, pararnn_info *info, int parts, void *workspace,
                            size_t ws_bytes, pararnn_stream stream) {
    if (!lstm_cell_ok(cell, B, T) || parts < 1 || parts > B || !params || !params->w_ih || !params->b_ih ||
        !params->w_hh || !params->b_hh || !x_host || !c0_host || !h0_host || !c_host || !h_host || !workspace ||
        !aligned(workspace, 256) || !(tol >= 0.f) || !std::isfinite(tol))
        return PARARNN_INVALID_ARG;
    const void *ptrs[] = {params->w_ih, params->b_ih, params->w_hh, params->b_hh};
    for (const void *q : ptrs)
        if (!aligned(q, 16)) return PARARNN_INVALID_ARG;
    const LstmHostLayout H = lstm_host_layout(*cell, B, T, parts);
    if (ws_bytes < H.total) return PARARNN_INVALID_ARG;
    char *ws = static_cast<char *>(workspace);
    const size_t es = cell->x_dtype == PARARNN_BF16 ? 2 : 4;
    const size_t srow = static_cast<size_t>(T) * cell->d * 4;
    PipeIo io;
    io.nin = 1;
    io.nout = 2;
    io.in[0] = static_cast<const char *>(x_host);
    io.in_row[0] = static_cast<size_t>(T) * cell->din * es;
    io.out[0] = reinterpret_cast<char *>(c_host);
    io.out[1] = reinterpret_cast<char *>(h_host);
    io.out_row[0] = io.out_row[1] = srow;
    for (int q = 0; q < H.nbuf; ++q) io.in_off[0][q] = H.xs[q], io.out_off[0][q] = H.cs[q], io.out_off[1][q] = H.hs[q];
    cudaStream_t sc = reinterpret_cast<cudaStream_t>(stream);
    float *c0_dev = reinterpret_cast<float *>(ws + H.c0), *h0_dev = reinterpret_cast<float *>(ws + H.h0);
    pararnn_info *infos = reinterpret_cast<pararnn_info *>(ws + H.infos);
    const size_t bd = static_cast<size_t>(B) * cell->d * 4;
    auto pre = [&](cudaStream_t s_in) {
        cudaError_t e = cudaMemcpyAsync(c0_dev, c0_host, bd, cudaMemcpyHostToDevice, s_in);
        if (e == cudaSuccess) e = cudaMemcpyAsync(h0_dev, h0_host, bd, cudaMemcpyHostToDevice, s_in);
        return e;
    };
    auto enq = [&](int p, int b0, int nb, int buf) {
        const size_t o = static_cast<size_t>(b0) * cell->d;
        const cudaError_t e = lstm_enqueue(cell, params, ws + H.xs[buf], c0_dev + o, h0_dev + o, nb, T, tol,
                                           max_iters, reinterpret_cast<float *>(ws + H.cs[buf]),
                                           reinterpret_cast<float *>(ws + H.hs[buf]), infos + p, ws + H.solve, sc);
        return e == cudaSuccess ? PARARNN_OK : PARARNN_CUDA_ERROR;
    };
    const int rc = run_pipeline(B, parts, H.nbuf, io, ws, sc, pre, enq);
    if (rc != PARARNN_OK) return rc;
    return fold_reports(infos, parts, sc, info);
}

}  // extern "C"

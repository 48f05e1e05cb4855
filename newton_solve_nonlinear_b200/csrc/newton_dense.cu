// newton_dense.cu -- dense-Jacobian modes (DEER, ELK on the dense cell) and the
// dense standalone affine scan.
#include "common.cuh"
#include "solver.cuh"

namespace pararnn {

size_t dense_ws_bytes(const pararnn_cell &cell, int B, int T, int mode) { return 256; }

cudaError_t launch_dense_solver(const pararnn_cell &cell, int mode, const DiagArgs &a,
                                void *dense_ws, cudaStream_t s) {
    return cudaErrorNotSupported;
}

size_t scan_dense_ws_bytes(int B, int T, int D) { return 256; }

cudaError_t launch_scan_dense(const float *A, const float *b, const float *h0, int B, int T,
                              int D, float *h, void *ws, cudaStream_t s) {
    return cudaErrorNotSupported;
}

}  // namespace pararnn

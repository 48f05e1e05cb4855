// scan_diag.cu -- standalone diagonal affine scan h_t = a_t * h_{t-1} + b_t.
//
// The linear solve inside each quasi-Newton iteration, exposed on its own
// ("Towards Scalable and Stable Parallelization of Nonlinear RNNs", atlas
// summary "Builds on": parallel associative scan; "ParaRNN" summary,
// "Newton's Iteration": forward substitution on a block lower-triangular
// system).  Single pass over HBM (12 bytes per element: a, b in, h out):
// tiles of (sequence, 64 lanes, L steps) are taken in order from a ticket
// counter, so every tile's predecessor has already started; each thread
// composes 8 steps x 4 lanes in registers, a shared-memory pass forms the
// tile-local exclusive prefixes, one thread per lane resolves the carry with a
// decoupled look-back, and the tile is re-swept and written with float4 stores.
#include <mutex>

#include "common.cuh"
#include "lookback.cuh"
#include "solver.cuh"

namespace pararnn {
namespace {

constexpr int TK = 8;  // steps per thread, 128-step tiles (measured: 4 steps 0.61 of HBM, 8 0.72, 12 0.67, 16 0.69)

struct ScanArgs {
    const float *A, *b, *h0;
    float *h;
    int B, T, D;
    Tiling tl;
    unsigned long long *desc;
    WsHeader *hdr;
};

__global__ void __launch_bounds__(kThreads) scan_diag_kernel(ScanArgs S) {
    __shared__ float sA[kThreads * 4], sB[kThreads * 4];  // [NTB][DG] (NTB*DG <= 1024)
    __shared__ float sC[64];
    __shared__ long long s_tile;
    const Tiling &tl = S.tl;
    if (threadIdx.x == 0) s_tile = static_cast<long long>(atomicAdd(&S.hdr->ticket, 1ull));
    __syncthreads();
    const long long tile = s_tile;
    const int chunk = static_cast<int>(tile / tl.n_groups);
    const int grp = static_cast<int>(tile % tl.n_groups);
    const int b = grp / tl.n_dgroups, dg = grp % tl.n_dgroups;
    const int db = threadIdx.x % tl.DB, tb = threadIdx.x / tl.DB;
    const bool active = tb < tl.NTB;
    const int lane0 = db * 4, d0 = dg * tl.DG + lane0;
    const bool dvalid = active && d0 < S.D;
    const int t0 = chunk * tl.L + tb * TK;

    float a[TK][4], bb[TK][4];
#pragma unroll
    for (int k = 0; k < TK; ++k) {
        const int t = t0 + k;
        float4 av = make_float4(1.f, 1.f, 1.f, 1.f), bv = make_float4(0.f, 0.f, 0.f, 0.f);
        if (dvalid && t < S.T) {
            const size_t off = (static_cast<size_t>(b) * S.T + t) * S.D + d0;
            av = __ldcs(reinterpret_cast<const float4 *>(S.A + off));
            bv = __ldcs(reinterpret_cast<const float4 *>(S.b + off));
        }
        a[k][0] = av.x; a[k][1] = av.y; a[k][2] = av.z; a[k][3] = av.w;
        bb[k][0] = bv.x; bb[k][1] = bv.y; bb[k][2] = bv.z; bb[k][3] = bv.w;
    }
    float cA[4], cB[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) { cA[j] = 1.f; cB[j] = 0.f; }
#pragma unroll
    for (int k = 0; k < TK; ++k)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            cB[j] = fmaf(a[k][j], cB[j], bb[k][j]);
            cA[j] = a[k][j] * cA[j];
        }
    if (active)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            sA[tb * tl.DG + lane0 + j] = cA[j];
            sB[tb * tl.DG + lane0 + j] = cB[j];
        }
    __syncthreads();
    if (threadIdx.x < tl.DG) {
        const int lane = threadIdx.x;
        float EA = 1.f, EB = 0.f;
        for (int q = 0; q < tl.NTB; ++q) {
            const float qa = sA[q * tl.DG + lane], qb = sB[q * tl.DG + lane];
            sA[q * tl.DG + lane] = EA;
            sB[q * tl.DG + lane] = EB;
            EB = fmaf(qa, EB, qb);
            EA = qa * EA;
        }
        const int d = dg * tl.DG + lane;
        const float carry0 = (chunk == 0 && d < S.D) ? __ldg(S.h0 + static_cast<size_t>(b) * S.D + d) : 0.f;
        sC[lane] = lookback_affine(S.desc, tile, tl.n_groups, tl.DG, lane, 1u, EA, EB, chunk,
                                   carry0, &S.hdr->status);
    }
    __syncthreads();
    if (!dvalid) return;
    float out[TK][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int l = lane0 + j;
        float hv = fmaf(sA[tb * tl.DG + l], sC[l], sB[tb * tl.DG + l]);
#pragma unroll
        for (int k = 0; k < TK; ++k) {
            hv = fmaf(a[k][j], hv, bb[k][j]);
            out[k][j] = hv;
        }
    }
#pragma unroll
    for (int k = 0; k < TK; ++k) {
        const int t = t0 + k;
        if (t < S.T)
            __stcs(reinterpret_cast<float4 *>(S.h + (static_cast<size_t>(b) * S.T + t) * S.D + d0),
                   make_float4(out[k][0], out[k][1], out[k][2], out[k][3]));
    }
}

}  // namespace

cudaError_t launch_scan_diag(const float *A, const float *b, const float *h0, int B, int T, int D,
                             float *h, void *ws, cudaStream_t s) {
    ScanArgs S;
    S.A = A; S.b = b; S.h0 = h0; S.h = h;
    S.B = B; S.T = T; S.D = D;
    S.tl = make_tiling(B, T, D, false, TK);
    S.hdr = static_cast<WsHeader *>(ws);
    S.desc = reinterpret_cast<unsigned long long *>(static_cast<char *>(ws) + 256);
    const size_t desc_bytes = static_cast<size_t>(S.tl.n_tiles) * S.tl.DG * 2 * 8;
    cudaError_t e = cudaMemsetAsync(ws, 0, 256 + desc_bytes, s);
    if (e != cudaSuccess) return e;
    scan_diag_kernel<<<static_cast<unsigned>(S.tl.n_tiles), kThreads, 0, s>>>(S);
    return cudaGetLastError();
}

size_t scan_diag_ws_bytes(int B, int T, int D) {
    const Tiling tl = make_tiling(B, T, D, false, TK);
    return 256 + static_cast<size_t>(tl.n_tiles) * tl.DG * 2 * 8;
}

}  // namespace pararnn

// ---------------------------------------------------------------------------
// The same scan for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they need a scan:
// code that runs while an allocator is locked or must not grow its memory
// footprint, plugins handed only input and output buffers by a host framework,
// and code paths where allocation is forbidden after start-up.  For them the
// scan's scratch (a 256-byte status header and the look-back descriptors) lives
// in the file-scope device array below, which the CUDA runtime creates when it
// loads this library's device code; every GPU that loads the library holds it
// until the process exits.
// ---------------------------------------------------------------------------
namespace pararnn {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
constexpr int kNoAllocMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mutex;
void *g_noalloc_ptr[kNoAllocMaxDevices] = {};

// Device address of the scratch array on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up with
// the device current.  It is looked up again on every call made outside stream
// capture: a device reset (or a primary context released and retained again)
// reloads the library's device code, and the array may then live elsewhere.
// Inside a capture the address the last uncaptured call on this device found
// is used (the lookup itself may load device code, which a capture forbids).
cudaError_t noalloc_scratch(cudaStream_t s, void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kNoAllocMaxDevices) return cudaErrorInvalidDevice;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if ((e = cudaStreamIsCapturing(s, &cap)) != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (cap == cudaStreamCaptureStatusNone) {
        void *p = nullptr;
        if ((e = cudaGetSymbolAddress(&p, g_noalloc_scratch)) != cudaSuccess) return e;
        g_noalloc_ptr[dev] = p;
    } else if (g_noalloc_ptr[dev] == nullptr) {
        return cudaErrorStreamCaptureUnsupported;
    }
    *out = g_noalloc_ptr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace pararnn

extern "C" PARARNN_API int pararnn_affine_scan_noalloc(const float *A, const float *b,
                                                       const float *h0, int B, int T, int D,
                                                       float *h, unsigned *status_dev,
                                                       pararnn_stream stream) {
    using namespace pararnn;
    if (B < 1 || T < 1 || D < 4 || D % 4 != 0) return PARARNN_INVALID_ARG;
    if (static_cast<long long>(T) * D > (1ll << 31)) return PARARNN_INVALID_ARG;
    if (!A || !b || !h0 || !h) return PARARNN_INVALID_ARG;
    const auto al16 = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (!al16(A) || !al16(b) || !al16(h0) || !al16(h)) return PARARNN_INVALID_ARG;
    if (status_dev && (reinterpret_cast<uintptr_t>(status_dev) & 3u) != 0) return PARARNN_INVALID_ARG;
    if (scan_diag_ws_bytes(B, T, D) > kNoAllocScratchBytes) return PARARNN_INVALID_ARG;
    const size_t nh = static_cast<size_t>(B) * T * D * 4;
    const auto over = [](const void *x, size_t nx, const void *y, size_t ny) {
        const auto px = reinterpret_cast<uintptr_t>(x), py = reinterpret_cast<uintptr_t>(y);
        return px < py + ny && py < px + nx;
    };
    // h may be A or b exactly (each element is read before the thread that owns
    // it writes h), but must not overlap them partly, nor h0
    if ((h != A && over(h, nh, A, nh)) || (h != b && over(h, nh, b, nh)) ||
        over(h, nh, h0, static_cast<size_t>(B) * D * 4))
        return PARARNN_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    void *scratch = nullptr;
    if (noalloc_scratch(s, &scratch) != cudaSuccess) return PARARNN_CUDA_ERROR;
    // launch_scan_diag first clears the header and the descriptors it will use
    cudaError_t e = launch_scan_diag(A, b, h0, B, T, D, h, scratch, s);
    if (e == cudaSuccess && status_dev)
        e = cudaMemcpyAsync(status_dev, &static_cast<WsHeader *>(scratch)->status, sizeof(unsigned),
                            cudaMemcpyDeviceToDevice, s);
    return e == cudaSuccess ? PARARNN_OK : PARARNN_CUDA_ERROR;
}

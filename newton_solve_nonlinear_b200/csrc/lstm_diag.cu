// lstm_diag.cu -- exact Newton (DEER) on the diagonal-recurrence LSTM.
//
// Method: the pages apply the parallel Newton solve to "adaptations" of LSTM
// and GRU (ParaLSTM; the ParaRNN talk page "Federico Danieli", Abstract; the
// ParaRNN summary page, "Experimental Results" and "Newton's Iteration").  The
// adapted cell replaces each recurrent matrix by a vector (u_k * h), so lane j
// of the next state (c', h') depends only on lane j of (c, h): the Jacobian is
// a 2x2 block per lane and Newton's linear step is the recurrence
//     s_t = A_t s_{t-1} + b_t,  s = (c, h),  A_t = dF/ds (2x2 per lane),
//     b_t = F(s^(i)_{t-1}) - A_t s^(i)_{t-1},
// solved exactly by a scan over 2x2 affine maps.  Cell (torch.nn.LSTMCell
// layout, gates i, f, g, o):
//     i = sig(p_i + u_i h + b_i), f = sig(p_f + u_f h + b_f),
//     g = tanh(p_g + u_g h + b_g), o = sig(p_o + u_o h + b_o),
//     c' = f c + i g,  h' = o tanh(c').
//
// One cooperative launch runs every iteration.  CTAs of 256 threads (two per SM) walk tiles
// of (sequence, 64 lanes, 32 steps), chunk-major; thread (lane d, segment s)
// owns 8 consecutive steps: it evaluates the cell and its 2x2 Jacobian at the
// shifted guess, composes its steps' affine maps, the four segments of a lane
// chain through shared memory, and a decoupled look-back over earlier
// chunks (2x2 maps, one thread per lane) gives the tile's entering state.
// The sweep writes the new iterate and the convergence maxima
// max |s^(i+1) - s^(i)| (both halves of the state) and max |s^(i) - F|.
// Traffic per lane-step and iteration: P (16 B), the guess (c, h: 8 B read,
// once as the previous state and once as the current one), the new state (8 B).
#include "common.cuh"
#include "lookback.cuh"
#include "solver.cuh"

namespace pararnn {
namespace {

constexpr int LTS = 32;            // steps per tile
constexpr int LDL = 64;            // lanes per tile
constexpr int LNT = 256;           // threads: lane x 4 segments (512 threads, 4 steps each: 8.10 ms per solve; 256: 6.78)
constexpr int LSEGS = LNT / LDL;   // 4 segments
constexpr int LSL = LTS / LSEGS;   // 8 steps per thread
constexpr int LWIN = 1;            // predecessors each look-back thread reads per round trip
constexpr int LWORDS = 8;          // look-back words per (tile, lane): aggregate 0..5, inclusive 6..7

// s -> [[a, b], [c, d]] s + (x, y)
struct M2 {
    float a, b, c, d, x, y;
};
__device__ __forceinline__ M2 m2_identity() { return M2{1.f, 0.f, 0.f, 1.f, 0.f, 0.f}; }
// Apply `first`, then `second`.
__device__ __forceinline__ M2 m2_compose(const M2 &second, const M2 &first) {
    return M2{fmaf(second.a, first.a, second.b * first.c), fmaf(second.a, first.b, second.b * first.d),
              fmaf(second.c, first.a, second.d * first.c), fmaf(second.c, first.b, second.d * first.d),
              fmaf(second.a, first.x, fmaf(second.b, first.y, second.x)),
              fmaf(second.c, first.x, fmaf(second.d, first.y, second.y))};
}
__device__ __forceinline__ float2 m2_apply(const M2 &m, float2 s) {
    return make_float2(fmaf(m.a, s.x, fmaf(m.b, s.y, m.x)), fmaf(m.c, s.x, fmaf(m.d, s.y, m.y)));
}
__device__ __forceinline__ M2 m2_shfl_down(const M2 &m, int o) {
    return M2{__shfl_down_sync(0xffffffffu, m.a, o), __shfl_down_sync(0xffffffffu, m.b, o),
              __shfl_down_sync(0xffffffffu, m.c, o), __shfl_down_sync(0xffffffffu, m.d, o),
              __shfl_down_sync(0xffffffffu, m.x, o), __shfl_down_sync(0xffffffffu, m.y, o)};
}
__device__ __forceinline__ M2 m2_shfl(const M2 &m, int src) {
    return M2{__shfl_sync(0xffffffffu, m.a, src), __shfl_sync(0xffffffffu, m.b, src),
              __shfl_sync(0xffffffffu, m.c, src), __shfl_sync(0xffffffffu, m.d, src),
              __shfl_sync(0xffffffffu, m.x, src), __shfl_sync(0xffffffffu, m.y, src)};
}

// Wait until a predecessor's inclusive words (6, 7) or aggregate words (0..5)
// carry this epoch: 2 = inclusive, 1 = aggregate, 0 = timeout (recorded).
__device__ __forceinline__ int m2_wait(const unsigned long long *pp, unsigned epoch, unsigned *status,
                                       unsigned long long &w0, unsigned long long &w6) {
    long long spins = 0;
    while (true) {
        if (word_ready(w6, epoch)) return 2;
        if (word_ready(w0, epoch)) return 1;
        if (++spins > 64) {
            if ((spins & 1023) == 0 && timed_out(status)) return 0;
            if (spins > kSpinBudget) {
                flag_timeout(status);
                return 0;
            }
            __nanosleep(32);
        }
        w6 = ld_relaxed(pp + 6);
        w0 = ld_relaxed(pp);
    }
}

// Cooperative decoupled look-back over 2x2 affine maps, G threads per lane
// (as coop_lookback: thread q reads predecessors q R + 1 .. back; the nearest
// inclusive value ends it; the maps in front of it compose by an ordered
// shuffle reduction).  Each (tile, lane) has 8 tagged words: the tile's map
// (0..5, written once as an aggregate) and the state after the tile (6, 7,
// written once as an inclusive value), so no word is ever rewritten.
// Returns the state entering the tile (carry0 for the first chunk).
template <int G, int R>
__device__ float2 coop_lookback_m2(unsigned long long *desc, long long tile, long long step, int DG, int d, int q,
                                   unsigned epoch, const M2 &E, int avail, float2 carry0, unsigned *status) {
    unsigned long long *mine = desc + (static_cast<size_t>(tile) * DG + d) * LWORDS;
    const int lane = threadIdx.x & 31;
    const int gbase = lane & ~(G - 1);
    const unsigned gmask = (((1u << G) - 1u) << gbase);
    float2 sin = carry0;
    if (avail > 0) {
        if (q == 0) {
            const unsigned tag = make_tag(epoch, kStateAgg);
            const float v[6] = {E.a, E.b, E.c, E.d, E.x, E.y};
#pragma unroll
            for (int e = 0; e < 6; ++e) st_relaxed(mine + e, pack_word(tag, v[e]));
        }
        M2 acc = m2_identity();
        bool done = false;
        for (int base = 0;; base += G * R) {
            unsigned long long w0[R], w6[R];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int p = base + q * R + r;
                w0[r] = w6[r] = 0ull;
                if (!done && p < avail) {
                    const unsigned long long *pp = desc + (static_cast<size_t>(tile - (p + 1) * step) * DG + d) * LWORDS;
                    w6[r] = ld_relaxed(pp + 6);
                    w0[r] = ld_relaxed(pp);
                }
            }
            M2 mp = m2_identity();
            float2 iv = make_float2(0.f, 0.f);
            bool inc = false;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int p = base + q * R + r;
                if (!done && !inc && p < avail) {
                    const unsigned long long *pp = desc + (static_cast<size_t>(tile - (p + 1) * step) * DG + d) * LWORDS;
                    const int kind = m2_wait(pp, epoch, status, w0[r], w6[r]);
                    if (kind == 0) {
                        inc = true;  // timed out: read as an inclusive zero state
                    } else if (kind == 2) {
                        const unsigned long long w7 = wait_tag(pp + 7, word_tag(w6[r]), status);
                        inc = true;
                        iv = make_float2(word_val(w6[r]), word_val(w7));
                    } else {
                        float v[6];
                        v[0] = word_val(w0[r]);
                        bool ok = true;
#pragma unroll
                        for (int e = 1; e < 6; ++e) {
                            const unsigned long long we = wait_tag(pp + e, word_tag(w0[r]), status);
                            ok = ok && we != 0ull;
                            v[e] = word_val(we);
                        }
                        if (!ok)
                            inc = true;
                        else  // map := map o (this predecessor's map)
                            mp = m2_compose(mp, M2{v[0], v[1], v[2], v[3], v[4], v[5]});
                    }
                }
            }
            const unsigned incm = (__ballot_sync(0xffffffffu, inc) & gmask) >> gbase;
            const int k = incm ? __ffs(incm) - 1 : G;  // nearest thread holding an inclusive value
            if (q > k) mp = m2_identity();
#pragma unroll
            for (int o = 1; o < G; o <<= 1) {  // ordered: map_q o map_{q+1} o ...
                const M2 n = m2_shfl_down(mp, o);
                if ((q & (2 * o - 1)) == 0) mp = m2_compose(mp, n);
            }
            mp = m2_shfl(mp, gbase);
            const int src = gbase + (k < G ? k : 0);
            const float2 kv = make_float2(__shfl_sync(0xffffffffu, iv.x, src), __shfl_sync(0xffffffffu, iv.y, src));
            if (!done) {
                acc = m2_compose(acc, mp);
                if (k < G) {
                    sin = m2_apply(acc, kv);
                    done = true;
                }
            }
            if (__all_sync(0xffffffffu, done)) break;
        }
    }
    if (q == 0) {
        const float2 so = m2_apply(E, sin);
        const unsigned tag = make_tag(epoch, kStateInc);
        st_relaxed(mine + 7, pack_word(tag, so.y));
        st_relaxed(mine + 6, pack_word(tag, so.x));
    }
    return sin;
}

struct LstmArgs {
    const float *P;              // [B, T, 4D] input pre-activations (b_ih included)
    const float *u, *b_hh;       // [4D] recurrent vectors and biases (gates i, f, g, o)
    const float *c0, *h0;        // [B, D]
    float *cbuf[2], *hbuf[2];    // iterate ping-pong; [1] are the caller's outputs
    float tol;
    int max_iters;
    WsHeader *hdr;
    unsigned long long *desc;    // [n_tiles][LDL][LWORDS]
    pararnn_info *info_out;
    int B, T, D, ndg, ngroups, n_chunks;
    long long n_tiles;
};

// The cell at (c, h) with pre-activations p (i, f, g, o): the next state and
// its 2x2 Jacobian (rows c', h'; columns c, h).
__device__ __forceinline__ void lstm_cell(float pi, float pf, float pg, float po, float c, float h, float ui,
                                          float uf, float ug, float uo, float bi, float bf, float bg, float bo,
                                          float &c2, float &h2, M2 &J) {
    const float i = sigmoidf_(fmaf(ui, h, pi + bi));
    const float f = sigmoidf_(fmaf(uf, h, pf + bf));
    const float g = tanhf_(fmaf(ug, h, pg + bg));
    const float o = sigmoidf_(fmaf(uo, h, po + bo));
    c2 = fmaf(f, c, i * g);
    const float tc = tanhf_(c2);
    h2 = o * tc;
    const float dch = fmaf(c * f * (1.f - f), uf, fmaf(g * i * (1.f - i), ui, i * (1.f - g * g) * ug));
    const float sech2 = 1.f - tc * tc;
    J.a = f;
    J.b = dch;
    J.c = o * sech2 * f;
    J.d = fmaf(tc * o * (1.f - o), uo, o * sech2 * dch);
}

__global__ void __launch_bounds__(LNT, 2) lstm_diag_kernel(LstmArgs S) {
    __shared__ float seg_m[LSEGS][6][LDL];  // each segment's map
    __shared__ float carry[2][LDL];         // state entering the tile
    __shared__ unsigned red[32];
    const int T = S.T, D = S.D;
    WsHeader *hdr = S.hdr;
    unsigned *status = &hdr->status;
    const int tid = threadIdx.x;
    const int d = tid & (LDL - 1), seg = tid / LDL;   // sweep role
    // look-back threads per lane (diagonal LSTM workload, ms per solve: 4 -> 6.78, 2 -> 6.53, 1 -> 6.42)
    constexpr int LLB = 1;
    const int ld = tid / LLB, lq = tid % LLB;         // look-back role (tid < LDL * LLB)
    const unsigned nblocks = gridDim.x;

    int iters = 0, final_status = PARARNN_NOT_CONVERGED;
    unsigned last_delta = 0u, last_resid = 0u;
    for (int it = 0; it < S.max_iters; ++it) {
        if (blockIdx.x == 0 && tid == 0) {
            hdr->delta_bits[(it + 1) % 3] = 0u;
            hdr->resid_bits[(it + 1) % 3] = 0u;
        }
        const float *cold = S.cbuf[it & 1], *hold = S.hbuf[it & 1];
        float *cnew = S.cbuf[(it + 1) & 1], *hnew = S.hbuf[(it + 1) & 1];
        const bool zero_guess = it == 0;
        const unsigned epoch = static_cast<unsigned>(it + 1);
        unsigned dmax = 0u, rmax = 0u;
        bool failed = false;
        for (long long v = blockIdx.x; v < S.n_tiles; v += nblocks) {
            const unsigned v32 = static_cast<unsigned>(v), ng = static_cast<unsigned>(S.ngroups);
            const int chunk = static_cast<int>(v32 / ng);
            const int grp = static_cast<int>(v32 - static_cast<unsigned>(chunk) * ng);
            const int b = grp / S.ndg, dg = grp - (grp / S.ndg) * S.ndg;
            const int t0 = chunk * LTS;
            const int lane = dg * LDL + d;
            const bool lane_ok = lane < D;
            const size_t row0 = static_cast<size_t>(b) * T;
            float u4[4] = {0.f, 0.f, 0.f, 0.f}, b4[4] = {0.f, 0.f, 0.f, 0.f};
            if (lane_ok)
#pragma unroll
                for (int k = 0; k < 4; ++k) u4[k] = __ldg(S.u + k * D + lane), b4[k] = __ldg(S.b_hh + k * D + lane);
            // 1. the cell at the thread's 4 steps: its maps s -> J s + (F - J s_guess)
            M2 pre[LSL];      // inclusive prefix of the thread's maps
            float yc[LSL], yh[LSL];  // the guess at each step
            {
                float pv[LSL][4], cp[LSL + 1], hp[LSL + 1];
#pragma unroll
                for (int i = 0; i <= LSL; ++i) {  // guess rows t-1 .. t+3 and P rows, all in flight
                    const int t = t0 + seg * LSL + i - 1;
                    const bool ok = lane_ok && t < T && !(zero_guess && t >= 0);
                    if (t < 0) {
                        cp[i] = lane_ok ? __ldg(S.c0 + static_cast<size_t>(b) * D + lane) : 0.f;
                        hp[i] = lane_ok ? __ldg(S.h0 + static_cast<size_t>(b) * D + lane) : 0.f;
                    } else {
                        cp[i] = ok ? __ldcg(cold + (row0 + t) * D + lane) : 0.f;
                        hp[i] = ok ? __ldcg(hold + (row0 + t) * D + lane) : 0.f;
                    }
                    if (i < LSL) {
                        const int tt = t + 1;
                        const bool okp = lane_ok && tt < T;
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            pv[i][k] = okp ? __ldcs(S.P + (row0 + tt) * 4 * D + k * D + lane) : 0.f;
                    }
                }
                M2 acc = m2_identity();
#pragma unroll
                for (int i = 0; i < LSL; ++i) {
                    const int t = t0 + seg * LSL + i;
                    M2 m = m2_identity();
                    yc[i] = cp[i + 1];
                    yh[i] = hp[i + 1];
                    if (lane_ok && t < T) {
                        float c2, h2;
                        M2 J;
                        lstm_cell(pv[i][0], pv[i][1], pv[i][2], pv[i][3], cp[i], hp[i], u4[0], u4[1], u4[2], u4[3],
                                  b4[0], b4[1], b4[2], b4[3], c2, h2, J);
                        m = J;
                        m.x = c2 - fmaf(J.a, cp[i], J.b * hp[i]);
                        m.y = h2 - fmaf(J.c, cp[i], J.d * hp[i]);
                        rmax = max(rmax, max(abs_bits(yc[i] - c2), abs_bits(yh[i] - h2)));
                    }
                    acc = m2_compose(m, acc);
                    pre[i] = acc;
                }
            }
            seg_m[seg][0][d] = pre[LSL - 1].a, seg_m[seg][1][d] = pre[LSL - 1].b;
            seg_m[seg][2][d] = pre[LSL - 1].c, seg_m[seg][3][d] = pre[LSL - 1].d;
            seg_m[seg][4][d] = pre[LSL - 1].x, seg_m[seg][5][d] = pre[LSL - 1].y;
            if (__syncthreads_or(timed_out(status))) {  // uniform
                failed = true;
                break;
            }
            // 2. the state entering the tile, by look-back over earlier chunks
            if (tid < LDL * LLB) {
                M2 E = m2_identity();
#pragma unroll
                for (int q = 0; q < LSEGS; ++q)
                    E = m2_compose(M2{seg_m[q][0][ld], seg_m[q][1][ld], seg_m[q][2][ld], seg_m[q][3][ld],
                                      seg_m[q][4][ld], seg_m[q][5][ld]},
                                   E);
                const int ln = dg * LDL + ld;
                float2 s0 = make_float2(0.f, 0.f);
                if (chunk == 0 && ln < D)
                    s0 = make_float2(__ldg(S.c0 + static_cast<size_t>(b) * D + ln),
                                     __ldg(S.h0 + static_cast<size_t>(b) * D + ln));
                const float2 sin = coop_lookback_m2<LLB, LWIN>(S.desc, v, S.ngroups, LDL, ld, lq, epoch, E, chunk,
                                                                 s0, status);
                if (lq == 0) carry[0][ld] = sin.x, carry[1][ld] = sin.y;
            }
            __syncthreads();
            // 3. sweep: through the earlier segments, then this thread's steps
            {
                float2 s = make_float2(carry[0][d], carry[1][d]);
                for (int q = 0; q < seg; ++q)
                    s = m2_apply(M2{seg_m[q][0][d], seg_m[q][1][d], seg_m[q][2][d], seg_m[q][3][d], seg_m[q][4][d],
                                    seg_m[q][5][d]},
                                 s);
#pragma unroll
                for (int i = 0; i < LSL; ++i) {
                    const int t = t0 + seg * LSL + i;
                    if (lane_ok && t < T) {
                        const float2 n = m2_apply(pre[i], s);
                        const size_t o = (row0 + t) * D + lane;
                        __stcg(cnew + o, n.x);
                        __stcg(hnew + o, n.y);
                        dmax = max(dmax, max(abs_bits(n.x - yc[i]), abs_bits(n.y - yh[i])));
                    }
                }
            }
            __syncthreads();  // shared maps and carries are rewritten by the next tile
        }
        const unsigned bd = block_max_u32(dmax, red);
        const unsigned br = block_max_u32(rmax, red);
        if (tid == 0) {
            atomicMax(&hdr->delta_bits[it % 3], bd);
            atomicMax(&hdr->resid_bits[it % 3], br);
            if (failed) flag_timeout(status);
        }
        grid_barrier(hdr->barrier, nblocks, status);
        last_delta = ld_acquire_u32(&hdr->delta_bits[it % 3]);
        last_resid = ld_acquire_u32(&hdr->resid_bits[it % 3]);
        iters = it + 1;
        // a timeout another CTA raises may land between two threads' reads: decide once per CTA
        if (__syncthreads_or(timed_out(status))) { final_status = PARARNN_TIMEOUT; break; }
        if (last_delta >= 0x7f800000u) { final_status = PARARNN_DIVERGED; break; }
        if (__uint_as_float(last_delta) <= S.tol) { final_status = PARARNN_OK; break; }
    }
    if ((iters & 1) == 0 && iters > 0) {  // the last iterate is in the workspace copy: move it out
        const size_t n = static_cast<size_t>(S.B) * T * D;
        for (size_t q = static_cast<size_t>(blockIdx.x) * LNT + tid; q < n; q += static_cast<size_t>(nblocks) * LNT) {
            S.cbuf[1][q] = __ldcg(S.cbuf[0] + q);
            S.hbuf[1][q] = __ldcg(S.hbuf[0] + q);
        }
    }
    if (blockIdx.x == 0 && tid == 0) {
        pararnn_info info;
        info.iters = iters;
        info.status = final_status;
        info.delta = __uint_as_float(last_delta);
        info.residual = __uint_as_float(last_resid);
        *S.info_out = info;
        hdr->info = info;
    }
}

}  // namespace

size_t lstm_diag_desc_bytes(int B, int T, int D) {
    const long long tiles = static_cast<long long>(B) * ((D + LDL - 1) / LDL) * ((T + LTS - 1) / LTS);
    return static_cast<size_t>(tiles) * LDL * LWORDS * 8;
}

cudaError_t launch_lstm_diag(const float *P, const float *u, const float *b_hh, const float *c0, const float *h0,
                             int B, int T, int D, float tol, int max_iters, float *c_ws, float *h_ws, float *c_out,
                             float *h_out, void *hdr, void *desc, pararnn_info *info_out, cudaStream_t s) {
    LstmArgs S;
    S.P = P, S.u = u, S.b_hh = b_hh, S.c0 = c0, S.h0 = h0;
    S.cbuf[0] = c_ws, S.cbuf[1] = c_out, S.hbuf[0] = h_ws, S.hbuf[1] = h_out;
    S.tol = tol;
    S.max_iters = max_iters <= 0 ? T + 1 : max_iters;
    S.hdr = static_cast<WsHeader *>(hdr);
    S.desc = static_cast<unsigned long long *>(desc);
    S.info_out = info_out ? info_out : &S.hdr->info;
    S.B = B, S.T = T, S.D = D;
    S.ndg = (D + LDL - 1) / LDL;
    S.ngroups = B * S.ndg;
    S.n_chunks = (T + LTS - 1) / LTS;
    S.n_tiles = static_cast<long long>(S.ngroups) * S.n_chunks;
    int dev = 0, nsm = 0, per_sm = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, lstm_diag_kernel, LNT, 0);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    long long grid = static_cast<long long>(nsm) * per_sm;
    if (grid > S.n_tiles) grid = S.n_tiles;
    void *params[] = {&S};
    return cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(lstm_diag_kernel),
                                       dim3(static_cast<unsigned>(grid)), dim3(LNT), params, 0, s);
}

}  // namespace pararnn

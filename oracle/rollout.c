/*
 * rollout.c -- the plain sequential evaluation of the GRU on the host:
 * h_t = f(h_{t-1}, x_t), t = 1..T, for each sequence of the batch, in fp64 and
 * in fp32.  TEST AND BASELINE INFRASTRUCTURE ONLY: it times what a CPU does
 * without the parallel Newton method (the sequential rollout the pages
 * compare against, the ParaRNN summary page, "Core Idea"), beside the GPU
 * solve.  The product path never loads it.
 *
 * Cell (the standard GRU in torch.nn.GRUCell's layout, gate rows r, z, n):
 *   p = W_ih x_t + b_ih,  q = U h + b_hh  (dense U [3D, D]; diagonal: u * h)
 *   r = sig(p_r + q_r),  z = sig(p_z + q_z),  n = tanh(p_n + r q_n),
 *   h' = (1 - z) n + z h.
 * Sequences are independent: OpenMP over the batch, `threads` of them
 * (<= 0: the runtime's default).  Row-major arrays: x [B, T, Din],
 * w_ih [3D, Din], b_ih [3D], w_hh [3D, D] or [3D], b_hh [3D], h0 [B, D],
 * h [B, T, D] out.  Returns 0, or -1 for bad sizes / allocation failure.
 */
#include <math.h>
#include <stdlib.h>

#define GRU_ROLLOUT(NAME, REAL, EXP, TANH)                                                          \
    int NAME(const REAL *x, const REAL *w_ih, const REAL *b_ih, const REAL *w_hh, const REAL *b_hh, \
             const REAL *h0, int B, int T, int Din, int D, int dense, REAL *h, int threads) {        \
        if (B < 1 || T < 1 || Din < 1 || D < 1) return -1;                                          \
        int bad = 0;                                                                                \
        _Pragma("omp parallel for schedule(static) num_threads(threads > 0 ? threads : omp_get_max_threads())") \
        for (int b = 0; b < B; ++b) {                                                               \
            REAL *p = (REAL *)malloc(sizeof(REAL) * 6 * (size_t)D);                                 \
            REAL *prev = (REAL *)malloc(sizeof(REAL) * (size_t)D);                                  \
            if (!p || !prev) {                                                                      \
                bad = 1;                                                                            \
                free(p);                                                                            \
                free(prev);                                                                         \
                continue;                                                                           \
            }                                                                                       \
            REAL *q = p + 3 * (size_t)D;                                                            \
            for (int j = 0; j < D; ++j) prev[j] = h0[(size_t)b * D + j];                            \
            for (int t = 0; t < T; ++t) {                                                           \
                const REAL *xt = x + ((size_t)b * T + t) * Din;                                     \
                for (int g = 0; g < 3 * D; ++g) {                                                   \
                    const REAL *w = w_ih + (size_t)g * Din;                                         \
                    REAL s = b_ih[g];                                                               \
                    for (int k = 0; k < Din; ++k) s += w[k] * xt[k];                                \
                    p[g] = s;                                                                       \
                    if (dense) {                                                                    \
                        const REAL *u = w_hh + (size_t)g * D;                                       \
                        REAL v = b_hh[g];                                                           \
                        for (int k = 0; k < D; ++k) v += u[k] * prev[k];                            \
                        q[g] = v;                                                                   \
                    } else {                                                                        \
                        q[g] = w_hh[g] * prev[g % D] + b_hh[g];                                     \
                    }                                                                               \
                }                                                                                   \
                REAL *ht = h + ((size_t)b * T + t) * D;                                             \
                for (int j = 0; j < D; ++j) {                                                       \
                    const REAL r = (REAL)1 / ((REAL)1 + EXP(-(p[j] + q[j])));                       \
                    const REAL z = (REAL)1 / ((REAL)1 + EXP(-(p[D + j] + q[D + j])));               \
                    const REAL n = TANH(p[2 * D + j] + r * q[2 * D + j]);                           \
                    ht[j] = ((REAL)1 - z) * n + z * prev[j];                                        \
                }                                                                                   \
                for (int j = 0; j < D; ++j) prev[j] = ht[j];                                        \
            }                                                                                       \
            free(p);                                                                                \
            free(prev);                                                                             \
        }                                                                                           \
        return bad ? -1 : 0;                                                                        \
    }

#include <omp.h>

GRU_ROLLOUT(gru_rollout_f64, double, exp, tanh)
GRU_ROLLOUT(gru_rollout_f32, float, expf, tanhf)

/*
 * The diagonal-recurrence LSTM the same way (gate rows i, f, g, o; u the
 * recurrent vectors [4D]):  p = W_ih x_t + b_ih,
 *   i = sig(p_i + u_i h + b_i), f = sig(p_f + u_f h + b_f),
 *   g = tanh(p_g + u_g h + b_g), o = sig(p_o + u_o h + b_o),
 *   c' = f c + i g,  h' = o tanh(c').
 * x [B, T, Din], w_ih [4D, Din], b_ih, u, b_hh [4D], c0, h0 [B, D];
 * c, h [B, T, D] out.
 */
#define LSTM_ROLLOUT(NAME, REAL, EXP, TANH)                                                          \
    int NAME(const REAL *x, const REAL *w_ih, const REAL *b_ih, const REAL *u, const REAL *b_hh,      \
             const REAL *c0, const REAL *h0, int B, int T, int Din, int D, REAL *c, REAL *h,          \
             int threads) {                                                                           \
        if (B < 1 || T < 1 || Din < 1 || D < 1) return -1;                                           \
        int bad = 0;                                                                                  \
        _Pragma("omp parallel for schedule(static) num_threads(threads > 0 ? threads : omp_get_max_threads())") \
        for (int b = 0; b < B; ++b) {                                                                 \
            REAL *p = (REAL *)malloc(sizeof(REAL) * 4 * (size_t)D);                                   \
            if (!p) {                                                                                 \
                bad = 1;                                                                              \
                continue;                                                                             \
            }                                                                                         \
            const REAL *cp = c0 + (size_t)b * D, *hp = h0 + (size_t)b * D;                            \
            for (int t = 0; t < T; ++t) {                                                             \
                const REAL *xt = x + ((size_t)b * T + t) * Din;                                       \
                for (int g = 0; g < 4 * D; ++g) {                                                     \
                    const REAL *w = w_ih + (size_t)g * Din;                                           \
                    REAL s = b_ih[g];                                                                 \
                    for (int k = 0; k < Din; ++k) s += w[k] * xt[k];                                  \
                    p[g] = s + u[g] * hp[g % D] + b_hh[g];                                            \
                }                                                                                     \
                REAL *ct = c + ((size_t)b * T + t) * D, *ht = h + ((size_t)b * T + t) * D;            \
                for (int j = 0; j < D; ++j) {                                                         \
                    const REAL i = (REAL)1 / ((REAL)1 + EXP(-p[j]));                                  \
                    const REAL f = (REAL)1 / ((REAL)1 + EXP(-p[D + j]));                              \
                    const REAL g = TANH(p[2 * D + j]);                                                \
                    const REAL o = (REAL)1 / ((REAL)1 + EXP(-p[3 * D + j]));                          \
                    ct[j] = f * cp[j] + i * g;                                                        \
                    ht[j] = o * TANH(ct[j]);                                                          \
                }                                                                                     \
                cp = ct;                                                                              \
                hp = ht;                                                                              \
            }                                                                                         \
            free(p);                                                                                  \
        }                                                                                             \
        return bad ? -1 : 0;                                                                          \
    }

LSTM_ROLLOUT(lstm_rollout_f64, double, exp, tanh)
LSTM_ROLLOUT(lstm_rollout_f32, float, expf, tanhf)

/* Threads the OpenMP runtime would use by default. */
int rollout_max_threads(void) { return omp_get_max_threads(); }

// lookback.cuh -- decoupled look-back for single-pass scans over time chunks.
//
// A tile (one chunk of time steps for a group of state lanes) first publishes
// its aggregate (the composition of its steps' maps), then walks back over
// earlier chunks of the same lanes, composing their aggregates until it meets
// a chunk that has published its inclusive value (the state at its last step);
// that gives the tile's carry-in, and it publishes its own inclusive value.
// Single-pass scan with decoupled look-back: Merrill & Garland (2016).  One
// thread per lane; each lane's words are independent.
#pragma once

#include "common.cuh"

namespace pararnn {

// Every descriptor word carries its own tag (epoch and state) next to its
// value in one 64-bit word, and each (epoch, state) value is written once, so a
// word whose tag matches *is* the value: no acquire/release ordering is needed
// between words.  The look-back therefore reads predecessors with relaxed
// loads, kWin tiles per L2 round trip.  One per round trip measured fastest
// (standalone scan [16, 65536, 64], us per scan: 4 -> 170, 2 -> 166, 1 -> 162):
// the predecessors in one wave publish within about a round trip of each other,
// so a wider batch rarely saves a round trip and costs instructions.
constexpr int kWin = 1;

__device__ __forceinline__ bool word_ready(unsigned long long w, unsigned epoch) {
    const unsigned t = word_tag(w);
    return (t >> 2) == epoch && (t & 3u) != 0u;
}

// Spin until the word carries this epoch in any published state; 0 on timeout.
__device__ __forceinline__ unsigned long long wait_ready(const unsigned long long *p,
                                                         unsigned epoch, unsigned *status) {
    long long spins = 0;
    while (true) {
        const unsigned long long w = ld_relaxed(p);
        if (word_ready(w, epoch)) return w;
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

// Spin until the word carries exactly `tag`; 0 on timeout.
__device__ __forceinline__ unsigned long long wait_tag(const unsigned long long *p, unsigned tag,
                                                       unsigned *status) {
    long long spins = 0;
    while (true) {
        const unsigned long long w = ld_relaxed(p);
        if (word_tag(w) == tag) return w;
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

// Affine maps x -> A x + B.  Descriptor slot = 2 words: [0] tag|A (or tag|INC
// value), [1] tag|B.  `step` is the tile distance to the predecessor
// (+n_groups forward, -n_groups for a reverse scan); `avail` is the number of
// predecessors (0: this tile's carry-in is `carry0`).
template <int W = kWin>
__device__ __forceinline__ float lookback_affine(unsigned long long *desc, long long tile,
                                                 long long step, int DG, int lane, unsigned epoch,
                                                 float EA, float EB, int avail, float carry0,
                                                 unsigned *status) {
    unsigned long long *mine = desc + (static_cast<size_t>(tile) * DG + lane) * 2;
    float hin = carry0;
    if (avail > 0) {
        const unsigned tag_agg = make_tag(epoch, kStateAgg);
        st_relaxed(mine + 1, pack_word(tag_agg, EB));
        st_relaxed(mine, pack_word(tag_agg, EA));
        float accA = 1.f, accB = 0.f;
        long long j = tile - step;
        int left = avail;
        bool done = false;
        while (!done && left > 0) {
            const int n = left < W ? left : W;
            unsigned long long w0[W], w1[W];
#pragma unroll
            for (int q = 0; q < W; ++q)
                if (q < n) {
                    const unsigned long long *p = desc + (static_cast<size_t>(j - q * step) * DG + lane) * 2;
                    w0[q] = ld_relaxed(p);
                    w1[q] = ld_relaxed(p + 1);
                }
#pragma unroll
            for (int q = 0; q < W; ++q)
                if (q < n && !done) {
                    const unsigned long long *p = desc + (static_cast<size_t>(j - q * step) * DG + lane) * 2;
                    unsigned long long a = w0[q];
                    if (!word_ready(a, epoch)) a = wait_ready(p, epoch, status);
                    if (a == 0ull) {
                        hin = 0.f;
                        done = true;
                    } else if ((word_tag(a) & 3u) == kStateInc) {
                        hin = fmaf(accA, word_val(a), accB);
                        done = true;
                    } else {
                        unsigned long long bw = w1[q];
                        if (word_tag(bw) != word_tag(a)) bw = wait_tag(p + 1, word_tag(a), status);
                        if (bw == 0ull) {
                            hin = 0.f;
                            done = true;
                        } else {
                            accB = fmaf(accA, word_val(bw), accB);
                            accA = accA * word_val(a);
                        }
                    }
                }
            j -= static_cast<long long>(n) * step;
            left -= n;
        }
    }
    st_relaxed(mine, pack_word(make_tag(epoch, kStateInc), fmaf(EA, hin, EB)));
    return hin;
}

// 2x2 Mobius maps P -> (m0 P + m1) / (m2 P + m3), kept normalised (max entry 1).
struct Mob {
    float m0, m1, m2, m3;
};
// x * y (apply y first).  A Moebius map does not change when its matrix is
// scaled, so the product is rescaled by the power of two that brings its
// largest entry into [1, 2): exact, and it keeps long products in range.
__device__ __forceinline__ Mob mob_mul(const Mob &x, const Mob &y) {
    Mob r{x.m0 * y.m0 + x.m1 * y.m2, x.m0 * y.m1 + x.m1 * y.m3,
          x.m2 * y.m0 + x.m3 * y.m2, x.m2 * y.m1 + x.m3 * y.m3};
    const float s = fmaxf(fmaxf(fabsf(r.m0), fabsf(r.m1)), fmaxf(fabsf(r.m2), fabsf(r.m3)));
    const int e = (__float_as_int(s) >> 23) & 0xff;  // biased exponent of the largest entry
    if (e > 0 && e < 255) {
        const float sc = __int_as_float((254 - e) << 23);  // 2^(127 - e)
        r.m0 *= sc; r.m1 *= sc; r.m2 *= sc; r.m3 *= sc;
    }
    return r;
}
__device__ __forceinline__ float mob_apply(const Mob &x, float P) {
    return (x.m0 * P + x.m1) / (x.m2 * P + x.m3);
}

__device__ __forceinline__ float lookback_mobius(unsigned long long *desc, long long tile,
                                                 long long step, int DG, int lane, unsigned epoch,
                                                 const Mob &E, int avail, float carry0,
                                                 unsigned *status) {
    constexpr int W = kWin;
    unsigned long long *mine = desc + (static_cast<size_t>(tile) * DG + lane) * 4;
    float pin = carry0;
    if (avail > 0) {
        const unsigned tg = make_tag(epoch, kStateAgg);
        st_relaxed(mine + 1, pack_word(tg, E.m1));
        st_relaxed(mine + 2, pack_word(tg, E.m2));
        st_relaxed(mine + 3, pack_word(tg, E.m3));
        st_relaxed(mine, pack_word(tg, E.m0));
        Mob acc{1.f, 0.f, 0.f, 1.f};
        long long j = tile - step;
        int left = avail;
        bool done = false;
        while (!done && left > 0) {
            const int n = left < W ? left : W;
            unsigned long long w[W][4];
#pragma unroll
            for (int q = 0; q < W; ++q)
                if (q < n) {
                    const unsigned long long *p = desc + (static_cast<size_t>(j - q * step) * DG + lane) * 4;
#pragma unroll
                    for (int e = 0; e < 4; ++e) w[q][e] = ld_relaxed(p + e);
                }
#pragma unroll
            for (int q = 0; q < W; ++q)
                if (q < n && !done) {
                    const unsigned long long *p = desc + (static_cast<size_t>(j - q * step) * DG + lane) * 4;
                    unsigned long long a = w[q][0];
                    if (!word_ready(a, epoch)) a = wait_ready(p, epoch, status);
                    if (a == 0ull) {
                        pin = 0.f;
                        done = true;
                    } else if ((word_tag(a) & 3u) == kStateInc) {
                        pin = mob_apply(acc, word_val(a));
                        done = true;
                    } else {
                        float m[3];
                        bool ok = true;
#pragma unroll
                        for (int e = 1; e < 4; ++e) {
                            unsigned long long v = w[q][e];
                            if (word_tag(v) != word_tag(a)) v = wait_tag(p + e, word_tag(a), status);
                            if (v == 0ull) ok = false;
                            m[e - 1] = word_val(v);
                        }
                        if (!ok) {
                            pin = 0.f;
                            done = true;
                        } else {
                            acc = mob_mul(acc, Mob{word_val(a), m[0], m[1], m[2]});
                        }
                    }
                }
            j -= static_cast<long long>(n) * step;
            left -= n;
        }
    }
    st_relaxed(mine, pack_word(make_tag(epoch, kStateInc), mob_apply(E, pin)));
    return pin;
}

// Cooperative decoupled look-back for lane d, shared by G threads of one
// lane group (G consecutive lanes of a warp, G a power of two <= 32; q = rank
// in the group; every lane of the warp calls it).  Descriptors are laid out
// [tile][DG lanes][2 words].  The group reads R x G predecessors per round
// trip (thread q: tiles q R + 1 .. q R + R back), finds the nearest one that
// holds an inclusive value, and composes the aggregates in front of it (first
// serially inside a thread, then with an ordered shuffle reduction); windows
// repeat until an inclusive value is reached (the chunk-0 tile always
// publishes one).  Thread q = 0 publishes the tile's aggregate first and its
// inclusive value last.  Returns the carry into the tile (carry0 when there
// is no predecessor).  Waits are bounded: a descriptor that never arrives
// reads as an inclusive 0 and raises the timeout flag.  `publish` false keeps
// the tile's descriptors unwritten (a testing hook for those bounded waits).
// The first window's descriptor words of coop_lookback, read ahead of time
// (relaxed loads: words that are not ready yet are polled again as usual), so
// that their round trip overlaps the caller's own work before the look-back.
template <int R>
struct LookbackWindow {
    unsigned long long a[R], b[R];
};
template <int G, int R = 1>
__device__ __forceinline__ LookbackWindow<R> coop_lookback_prefetch(const unsigned long long *desc, long long tile,
                                                                    long long step, int DG, int d, int q,
                                                                    int avail) {
    LookbackWindow<R> w;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int p = q * R + r;
        w.a[r] = w.b[r] = 0ull;
        if (p < avail) {
            const unsigned long long *pp = desc + (static_cast<size_t>(tile - (p + 1) * step) * DG + d) * 2;
            w.a[r] = ld_relaxed(pp);
            w.b[r] = ld_relaxed(pp + 1);
        }
    }
    return w;
}

template <int G, int R = 1, bool kPrefetched = false>
__device__ __forceinline__ float coop_lookback(unsigned long long *desc, long long tile, long long step,
                                               int DG, int d, int q, unsigned epoch, float EA, float EB,
                                               int avail, float carry0, unsigned *status,
                                               const LookbackWindow<R> *pre = nullptr, bool publish = true) {
    unsigned long long *mine = desc + (static_cast<size_t>(tile) * DG + d) * 2;
    const int lane = threadIdx.x & 31;
    const int gbase = lane & ~(G - 1);
    const unsigned gmask = G == 32 ? 0xffffffffu : (((1u << G) - 1u) << gbase);
    float hin = carry0;
    if (avail > 0) {  // the same for every thread of the CTA
        if (q == 0 && publish) {
            const unsigned tag = make_tag(epoch, kStateAgg);
            st_relaxed(mine + 1, pack_word(tag, EB));
            st_relaxed(mine, pack_word(tag, EA));
        }
        float accA = 1.f, accB = 0.f;
        bool done = false;
        for (int base = 0;; base += G * R) {
            // this thread's R predecessors, nearest first: map = m_0 o m_1 o ... up to
            // (not including) the first inclusive value
            unsigned long long wa[R], wb[R];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int p = base + q * R + r;
                wa[r] = wb[r] = 0ull;
                if (kPrefetched && base == 0) {
                    wa[r] = pre->a[r];
                    wb[r] = pre->b[r];
                } else if (!done && p < avail) {
                    const unsigned long long *pp = desc + (static_cast<size_t>(tile - (p + 1) * step) * DG + d) * 2;
                    wa[r] = ld_relaxed(pp);
                    wb[r] = ld_relaxed(pp + 1);
                }
            }
            float ma = 1.f, mb = 0.f, iv = 0.f;
            bool inc = false;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int p = base + q * R + r;
                if (!done && !inc && p < avail) {
                    const unsigned long long *pp = desc + (static_cast<size_t>(tile - (p + 1) * step) * DG + d) * 2;
                    unsigned long long a = wa[r];
                    if (!word_ready(a, epoch)) a = wait_ready(pp, epoch, status);
                    if (a == 0ull) {
                        inc = true;
                    } else if ((word_tag(a) & 3u) == kStateInc) {
                        inc = true;
                        iv = word_val(a);
                    } else {
                        unsigned long long bw = wb[r];
                        if (word_tag(bw) != word_tag(a)) bw = wait_tag(pp + 1, word_tag(a), status);
                        if (bw == 0ull) {
                            inc = true;
                        } else {  // map := map o (a, b)
                            mb = fmaf(ma, word_val(bw), mb);
                            ma = ma * word_val(a);
                        }
                    }
                }
            }
            const unsigned incm = (__ballot_sync(0xffffffffu, inc) & gmask) >> gbase;
            const int k = incm ? __ffs(incm) - 1 : G;  // nearest thread holding an inclusive value
            if (q > k) {
                ma = 1.f;
                mb = 0.f;
            }
#pragma unroll
            for (int o = 1; o < G; o <<= 1) {  // ordered: map_q o map_{q+1} o ...
                const float na = __shfl_down_sync(0xffffffffu, ma, o);
                const float nb = __shfl_down_sync(0xffffffffu, mb, o);
                if ((q & (2 * o - 1)) == 0) {
                    mb = fmaf(ma, nb, mb);
                    ma = ma * na;
                }
            }
            ma = __shfl_sync(0xffffffffu, ma, gbase);
            mb = __shfl_sync(0xffffffffu, mb, gbase);
            const float kv = __shfl_sync(0xffffffffu, iv, gbase + (k < G ? k : 0));
            if (!done) {
                accB = fmaf(accA, mb, accB);
                accA = accA * ma;
                if (k < G) {
                    hin = fmaf(accA, kv, accB);
                    done = true;
                }
            }
            if (__all_sync(0xffffffffu, done)) break;
        }
    }
    if (q == 0 && publish) st_relaxed(mine, pack_word(make_tag(epoch, kStateInc), fmaf(EA, hin, EB)));
    return hin;
}

// The same for Moebius maps (descriptors [tile][DG lanes][4 words]); returns
// the covariance entering the tile.
template <int G, int R = 1>
__device__ __forceinline__ float coop_lookback_mob(unsigned long long *desc, long long tile, long long step,
                                                   int DG, int d, int q, unsigned epoch, const Mob &E,
                                                   int avail, float carry0, unsigned *status) {
    unsigned long long *mine = desc + (static_cast<size_t>(tile) * DG + d) * 4;
    const int lane = threadIdx.x & 31;
    const int gbase = lane & ~(G - 1);
    const unsigned gmask = G == 32 ? 0xffffffffu : (((1u << G) - 1u) << gbase);
    float pin = carry0;
    if (avail > 0) {
        if (q == 0) {
            const unsigned tg = make_tag(epoch, kStateAgg);
            st_relaxed(mine + 1, pack_word(tg, E.m1));
            st_relaxed(mine + 2, pack_word(tg, E.m2));
            st_relaxed(mine + 3, pack_word(tg, E.m3));
            st_relaxed(mine, pack_word(tg, E.m0));
        }
        Mob acc{1.f, 0.f, 0.f, 1.f};
        bool done = false;
        for (int base = 0;; base += G * R) {
            unsigned long long w[R][4];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int p = base + q * R + r;
#pragma unroll
                for (int e = 0; e < 4; ++e) w[r][e] = 0ull;
                if (!done && p < avail) {
                    const unsigned long long *pp = desc + (static_cast<size_t>(tile - (p + 1) * step) * DG + d) * 4;
#pragma unroll
                    for (int e = 0; e < 4; ++e) w[r][e] = ld_relaxed(pp + e);
                }
            }
            Mob mm{1.f, 0.f, 0.f, 1.f};
            float iv = 0.f;
            bool inc = false;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int p = base + q * R + r;
                if (!done && !inc && p < avail) {
                    const unsigned long long *pp = desc + (static_cast<size_t>(tile - (p + 1) * step) * DG + d) * 4;
                    unsigned long long a = w[r][0];
                    if (!word_ready(a, epoch)) a = wait_ready(pp, epoch, status);
                    if (a == 0ull) {
                        inc = true;
                    } else if ((word_tag(a) & 3u) == kStateInc) {
                        inc = true;
                        iv = word_val(a);
                    } else {
                        float m[3];
                        bool ok = true;
#pragma unroll
                        for (int e = 1; e < 4; ++e) {
                            unsigned long long v = w[r][e];
                            if (word_tag(v) != word_tag(a)) v = wait_tag(pp + e, word_tag(a), status);
                            if (v == 0ull) ok = false;
                            m[e - 1] = word_val(v);
                        }
                        if (!ok)
                            inc = true;
                        else
                            mm = mob_mul(mm, Mob{word_val(a), m[0], m[1], m[2]});
                    }
                }
            }
            const unsigned incm = (__ballot_sync(0xffffffffu, inc) & gmask) >> gbase;
            const int k = incm ? __ffs(incm) - 1 : G;
            if (q > k) mm = Mob{1.f, 0.f, 0.f, 1.f};
#pragma unroll
            for (int o = 1; o < G; o <<= 1) {
                Mob n;
                n.m0 = __shfl_down_sync(0xffffffffu, mm.m0, o);
                n.m1 = __shfl_down_sync(0xffffffffu, mm.m1, o);
                n.m2 = __shfl_down_sync(0xffffffffu, mm.m2, o);
                n.m3 = __shfl_down_sync(0xffffffffu, mm.m3, o);
                if ((q & (2 * o - 1)) == 0) mm = mob_mul(mm, n);
            }
            mm.m0 = __shfl_sync(0xffffffffu, mm.m0, gbase);
            mm.m1 = __shfl_sync(0xffffffffu, mm.m1, gbase);
            mm.m2 = __shfl_sync(0xffffffffu, mm.m2, gbase);
            mm.m3 = __shfl_sync(0xffffffffu, mm.m3, gbase);
            const float kv = __shfl_sync(0xffffffffu, iv, gbase + (k < G ? k : 0));
            if (!done) {
                acc = mob_mul(acc, mm);
                if (k < G) {
                    pin = mob_apply(acc, kv);
                    done = true;
                }
            }
            if (__all_sync(0xffffffffu, done)) break;
        }
    }
    if (q == 0) st_relaxed(mine, pack_word(make_tag(epoch, kStateInc), mob_apply(E, pin)));
    return pin;
}

}  // namespace pararnn

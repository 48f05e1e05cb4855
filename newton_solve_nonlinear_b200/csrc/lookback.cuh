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

// Affine maps x -> A x + B.  Descriptor slot = 2 words: [0] tag|A (or tag|INC
// value), [1] tag|B.  `step` is the tile distance to the predecessor (+-n_groups).
__device__ __forceinline__ float lookback_affine(unsigned long long *desc, long long tile,
                                                 long long step, int DG, int lane, unsigned epoch,
                                                 float EA, float EB, bool first, float carry0,
                                                 unsigned *status) {
    unsigned long long *mine = desc + (static_cast<size_t>(tile) * DG + lane) * 2;
    float hin = carry0;
    if (!first) {
        st_relaxed(mine + 1, pack_word(make_tag(epoch, kStateAgg), EB));
        st_release(mine, pack_word(make_tag(epoch, kStateAgg), EA));
        float accA = 1.f, accB = 0.f;
        long long j = tile - step;
        while (true) {
            unsigned long long *pj = desc + (static_cast<size_t>(j) * DG + lane) * 2;
            const unsigned long long w = wait_word(pj, epoch, status);
            if (w == 0ull) { hin = 0.f; break; }
            if ((word_tag(w) & 3u) == kStateInc) {
                hin = fmaf(accA, word_val(w), accB);
                break;
            }
            const unsigned long long w1 = ld_relaxed(pj + 1);
            const float Aj = word_val(w), Bj = word_val(w1);
            accB = fmaf(accA, Bj, accB);
            accA = accA * Aj;
            j -= step;
        }
    }
    st_release(mine, pack_word(make_tag(epoch, kStateInc), fmaf(EA, hin, EB)));
    return hin;
}

// 2x2 Mobius maps P -> (m0 P + m1) / (m2 P + m3), kept normalised (max entry 1).
struct Mob {
    float m0, m1, m2, m3;
};
__device__ __forceinline__ Mob mob_mul(const Mob &x, const Mob &y) {  // x * y (apply y first)
    Mob r{x.m0 * y.m0 + x.m1 * y.m2, x.m0 * y.m1 + x.m1 * y.m3,
          x.m2 * y.m0 + x.m3 * y.m2, x.m2 * y.m1 + x.m3 * y.m3};
    const float s = fmaxf(fmaxf(fabsf(r.m0), fabsf(r.m1)), fmaxf(fabsf(r.m2), fabsf(r.m3)));
    const float inv = s > 0.f ? 1.f / s : 1.f;
    r.m0 *= inv; r.m1 *= inv; r.m2 *= inv; r.m3 *= inv;
    return r;
}
__device__ __forceinline__ float mob_apply(const Mob &x, float P) {
    return (x.m0 * P + x.m1) / (x.m2 * P + x.m3);
}

__device__ __forceinline__ float lookback_mobius(unsigned long long *desc, long long tile,
                                                 long long step, int DG, int lane, unsigned epoch,
                                                 const Mob &E, bool first, float carry0,
                                                 unsigned *status) {
    unsigned long long *mine = desc + (static_cast<size_t>(tile) * DG + lane) * 4;
    float pin = carry0;
    if (!first) {
        const unsigned tg = make_tag(epoch, kStateAgg);
        st_relaxed(mine + 1, pack_word(tg, E.m1));
        st_relaxed(mine + 2, pack_word(tg, E.m2));
        st_relaxed(mine + 3, pack_word(tg, E.m3));
        st_release(mine, pack_word(tg, E.m0));
        Mob acc{1.f, 0.f, 0.f, 1.f};
        long long j = tile - step;
        while (true) {
            unsigned long long *pj = desc + (static_cast<size_t>(j) * DG + lane) * 4;
            const unsigned long long w = wait_word(pj, epoch, status);
            if (w == 0ull) { pin = 0.f; break; }
            if ((word_tag(w) & 3u) == kStateInc) {
                pin = mob_apply(acc, word_val(w));
                break;
            }
            Mob Mj{word_val(w), word_val(ld_relaxed(pj + 1)), word_val(ld_relaxed(pj + 2)),
                   word_val(ld_relaxed(pj + 3))};
            acc = mob_mul(acc, Mj);
            j -= step;
        }
    }
    st_release(mine, pack_word(make_tag(epoch, kStateInc), mob_apply(E, pin)));
    return pin;
}

}  // namespace pararnn

// persist_sched.cuh -- the two-phase schedule of the two-tile persistent kernels: whole pairs of
// 128-row Q tiles round-robin over the CTAs for the full rounds, then the leftover pairs as one
// line of (pair, key tile) items cut evenly between the CTAs (stream-K).  Identical in every
// role of every CTA.
#pragma once
#include "attn_common.cuh"

namespace swattn {

struct Piece {
    int bh;     // stream * H + head
    int pair;   // index of the Q-tile pair within the head (rows pair * 256 ...)
    int live;   // Q tiles of the pair that hold queries (1 or 2)
    int j0, j1; // key tiles [j0, j1) of this piece
    bool sk;    // from the stream-K phase (may be split) rather than a whole-pair round
};

// The two-phase schedule, identical in every role of every CTA (and callable on the host, where
// an inspection hook enumerates its pieces for the tests).
struct Sched {
    int nqt, nt, npairs, P, G, g, rounds, p0, Gsk;
    long long Csk, c0, c1;   // stream-K line length and this CTA's range of it
    __host__ __device__ int live(int p) const { return min(2, nqt - 2 * (p % npairs)); }
    // cost position of pair p (p >= p0) on the stream-K line: 2 nt per pair, nt for the
    // single-tile last pair of a head (when nqt is odd)
    __host__ __device__ long long cstart(int p) const {
        return 2LL * nt * (p - p0) - (long long)(nqt & 1) * nt * (p / npairs - p0 / npairs);
    }
    __host__ __device__ void init(int nqt_, int nt_, int BH, int G_, int g_) {
        nqt = nqt_; nt = nt_; npairs = (nqt + 1) / 2; P = BH * npairs; G = G_; g = g_;
        rounds = P / G;
        p0 = rounds * G;
        Csk = P > p0 ? cstart(P) : 0;
        // every stream-K CTA gets at least two cost units, so a pair's pieces sit in
        // consecutive CTAs that all hold one of its key tiles
        Gsk = Csk > 0 ? (int)min((long long)G, max(1LL, Csk / 2)) : 0;
        set_range(g);
    }
    __host__ __device__ void set_range(int cta) {
        c0 = cta < Gsk ? (long long)cta * Csk / Gsk : 0;
        c1 = cta < Gsk ? (long long)(cta + 1) * Csk / Gsk : 0;
    }
    // the stream-K CTA whose range holds cost position s
    __host__ __device__ int cta_of(long long s) const { return (int)(((s + 1) * Gsk - 1) / Csk); }
};

struct PieceIt {
    int r = 0;             // whole-pair rounds done
    long long cur = -1;    // stream-K cursor (-1: not started)
    int p = 0;             // stream-K pair the cursor is in
};

__host__ __device__ __forceinline__ bool next_piece(const Sched& s, PieceIt& it, Piece& pc) {
    if (it.r < s.rounds) {
        const int p = s.g + it.r * s.G;
        ++it.r;
        pc.bh = p / s.npairs;
        pc.pair = p % s.npairs;
        pc.live = s.live(p);
        pc.j0 = 0;
        pc.j1 = s.nt;
        pc.sk = false;
        return true;
    }
    if (it.cur < 0) {
        it.cur = s.c0;
        it.p = s.p0;
    }
    while (it.cur < s.c1) {
        while (it.p + 1 < s.P && s.cstart(it.p + 1) <= it.cur) ++it.p;
        const long long ps = s.cstart(it.p);
        const int lv = s.live(it.p);
        const int j0 = (int)((it.cur - ps + lv - 1) / lv);     // first item starting at or after cur
        if (j0 >= s.nt) {
            it.cur = ps + (long long)lv * s.nt;
            continue;
        }
        const long long e = (s.c1 - ps + lv - 1) / lv;        // first item starting at or after c1
        const int j1 = (int)(e < s.nt ? e : s.nt);
        it.cur = ps + (long long)lv * j1;
        pc.bh = it.p / s.npairs;
        pc.pair = it.p % s.npairs;
        pc.live = lv;
        pc.j0 = j0;
        pc.j1 = j1;
        pc.sk = true;
        return true;
    }
    return false;
}

// All-of-group vote over the 128 threads of softmax warpgroup qt (barrier ids 3 and 4): true
// iff every thread passes true.  Taken at points every warp of the group reaches, failed or
// not, so a warp whose wait gave up never leaves its group mates blocked in a barrier.
__device__ __forceinline__ bool wg_all(int qt, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, %2, 128, q;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r) : "r"((uint32_t)v), "r"(3 + qt) : "memory");
    return r != 0;
}

// Barrier over the 128 threads of softmax warpgroup qt (ids 1 and 2; 0 is __syncthreads).
// Used only right after wg_all has found every warp of the group healthy, with no wait in
// between, so no warp can be stranded in it.
__device__ __forceinline__ void wg_bar(int qt) {
    if (qt == 0) asm volatile("bar.sync 1, 128;" ::: "memory");
    else asm volatile("bar.sync 2, 128;" ::: "memory");
}

}  // namespace swattn

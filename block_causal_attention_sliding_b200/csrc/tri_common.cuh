// tri_common.cuh -- pieces shared by the three-S-buffer attention kernels (one CTA per unit,
// attn_tri.cu, and its CTA-pair form, attn_pair.cu): the two-phase schedule over units, the
// issuer's polled counters, the reference-max exchange between the two softmax groups, and one
// softmax step over a key tile.
#pragma once
#include "attn_common.cuh"

namespace swattn {
namespace tri {

constexpr int kSBufs = 3;   // S accumulators in tensor memory: S of tile u + 3 while u + 1, u + 2 run

// The two-phase schedule over units (one Q tile of one (b, h)), identical in every role.
struct Sched {
    int nqt, nt, U, G, g, rounds, u0, Gsk;
    long long Csk, c0, c1;   // stream-K line length and this CTA's range of it
    __host__ __device__ long long cstart(int u) const { return (long long)(u - u0) * nt; }
    __host__ __device__ void init(int nqt_, int nt_, int BH, int G_, int g_) {
        nqt = nqt_; nt = nt_; U = BH * nqt; G = G_; g = g_;
        rounds = U / G;
        u0 = rounds * G;
        Csk = (long long)(U - u0) * nt;
        // at least two items per stream-K CTA
        Gsk = Csk > 0 ? (int)min((long long)G, max(1LL, Csk / 2)) : 0;
        set_range(g);
    }
    __host__ __device__ void set_range(int cta) {
        c0 = cta < Gsk ? (long long)cta * Csk / Gsk : 0;
        c1 = cta < Gsk ? (long long)(cta + 1) * Csk / Gsk : 0;
    }
    __host__ __device__ int cta_of(long long s) const { return (int)(((s + 1) * Gsk - 1) / Csk); }
};

struct Piece {
    int unit;     // bh * nqt + q tile
    int j0, j1;   // key tiles [j0, j1)
    bool sk;      // from the stream-K phase (may be split)
};

struct PieceIt {
    int r = 0;
    long long cur = -1;
};

__host__ __device__ __forceinline__ bool next_piece(const Sched& s, PieceIt& it, Piece& pc) {
    if (it.r < s.rounds) {
        pc.unit = s.g + it.r * s.G;
        ++it.r;
        pc.j0 = 0;
        pc.j1 = s.nt;
        pc.sk = false;
        return true;
    }
    if (it.cur < 0) it.cur = s.c0;
    if (it.cur >= s.c1) return false;
    const int u = s.u0 + (int)(it.cur / s.nt);
    const int j0 = (int)(it.cur % s.nt);
    const long long left = s.c1 - it.cur;
    const int j1 = (int)min((long long)s.nt, j0 + left);
    it.cur += j1 - j0;
    pc.unit = u;
    pc.j0 = j0;
    pc.j1 = j1;
    pc.sk = true;
    return true;
}

// Acquire load of a shared word.
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* a) {
    uint32_t v;
    asm volatile("ld.acquire.cta.shared.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(a)) : "memory");
    return v;
}

__device__ __forceinline__ void st_release(uint32_t* a, uint32_t v) {
    asm volatile("st.release.cta.shared.u32 [%0], %1;" ::"r"(smem_u32(a)), "r"(v) : "memory");
}

// One release increment per warp on a word of this CTA (shared::cta address), after the warp's
// lanes have finished (and fenced) their work.
__device__ __forceinline__ void warp_signal(uint32_t addr) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0)
        asm volatile("red.release.cta.shared::cta.add.u32 [%0], 1;" ::"r"(addr) : "memory");
}

// Acquire load at cluster scope (pairs with a release from the peer CTA of a pair).
__device__ __forceinline__ uint32_t ld_acquire_cluster(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.acquire.cluster.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

// The MMA issuer's wait: poll until the counter reaches target (wrap-safe), bounded like every
// other wait.  Returns false on abort or timeout (raising the abort flag on a timeout).
// kCluster: the word also receives release increments from the peer CTA of a pair.
template <bool kCluster = false>
__device__ __forceinline__ bool poll_reach(const uint32_t* a, uint32_t target, volatile int* abort_flag) {
    auto load = [&]() { return kCluster ? ld_acquire_cluster(smem_u32(a)) : ld_acquire(a); };
    if ((int32_t)(load() - target) >= 0) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 0;; ++it) {
        if ((int32_t)(load() - target) >= 0) return true;
        if ((it & 15u) == 15u) {
            if (*abort_flag) return false;
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                *abort_flag = 1;
                return false;
            }
        }
    }
}

// Publish v under tag for the other group's thread of the same row.
__device__ __forceinline__ void ref_put(unsigned long long* a, float v, uint32_t tag) {
    const unsigned long long w = ((unsigned long long)tag << 32) | __float_as_uint(v);
    asm volatile("st.relaxed.cta.shared.b64 [%0], %1;" ::"r"(smem_u32(a)), "l"(w) : "memory");
}

// Bounded wait for the value published under tag; false (warp-uniform) on abort or timeout,
// which raises the CTA abort flag like every other wait.
__device__ __forceinline__ bool ref_get(const unsigned long long* a, uint32_t tag, float& v,
                                        volatile int* abort_flag) {
    const uint32_t addr = smem_u32(a);
    bool ok = false;
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
        unsigned long long w;
        asm volatile("ld.relaxed.cta.shared.b64 %0, [%1];" : "=l"(w) : "r"(addr) : "memory");
        if ((uint32_t)(w >> 32) == tag) {
            v = __uint_as_float((uint32_t)w);
            ok = true;
            break;
        }
        if ((it & 31u) == 31u) {
            if (*abort_flag) break;
            const uint64_t t = globaltimer_ns();
            if (t0 == 0) {
                t0 = t;
            } else if (t - t0 > kWaitLimitNs) {
                *abort_flag = 1;
                break;
            }
        }
    }
    return __all_sync(0xffffffffu, ok);
}

// All-of-both-groups vote (256 softmax threads, barrier id 2): true iff every thread passes
// true.  Taken once per piece after the piece's waits, so a warp whose wait gave up never
// leaves the others blocked in a barrier.
__device__ __forceinline__ bool vote_all(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, 2, 256, q;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r) : "r"((uint32_t)v) : "memory");
    return r != 0;
}

// bar.sync over the 256 softmax threads (id 1); used only after vote_all found them healthy.
__device__ __forceinline__ void softmax_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }


// One online-softmax step of this thread's query row over key tile u (the caller has waited
// for S(u)).  `first`: u opens the piece (no previous reference, O is overwritten by PV(u)).
// ref_prev / ref_mine: the reference words of tiles u - 1 and u.  m_g, l_g: this group's
// reference of its last tile in the piece and its row sum relative to it (has_g: the group
// has had a tile in this piece).  P is published once it is written in full and O, if the
// reference moved, has been rescaled.
// Returns false on abort.
// p_sig: the shared::cta address of the P counter.
// kP8: P is written as e4m3 (four keys per 32-bit column over S columns 0..31, for an e4m3 P V on
// kind::f8f6f4), formed as 2^(s sl2 - m + kP8Offset) with the rescale threshold kP8Threshold, and
// the row sum adds the fp32 weights -- as in the two-tile kernel's softmax step.
template <int D, bool kP8 = false>
__device__ __forceinline__ bool softmax_tile(uint32_t tS, uint32_t tO, int valid, bool first, uint32_t u,
                                             const unsigned long long* ref_prev, unsigned long long* ref_mine,
                                             uint32_t o_full_prev, uint32_t o_full_prev_parity,
                                             uint32_t p_sig, float sl2, float& m_g, float& l_g,
                                             bool& has_g, volatile int* abort_flag) {
    uint32_t sr[4][32];
#pragma unroll
    for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, sr[c]);
    tmem_wait_ld_dep(sr[0]);
    reg_fence(sr[1]);
    reg_fence(sr[2]);
    reg_fence(sr[3]);
    if (valid < kBlockN) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (c * 32 + i >= valid) sr[c][i] = __float_as_uint(-INFINITY);
    }
    float mxa[8];
#pragma unroll
    for (int a = 0; a < 8; ++a) mxa[a] = -INFINITY;
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int i = 0; i < 32; i += 2)
            mxa[(i >> 1) & 7] = fmax3(mxa[(i >> 1) & 7], __uint_as_float(sr[c][i]), __uint_as_float(sr[c][i + 1]));
#pragma unroll
    for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
        for (int a = 0; a < w; ++a) mxa[a] = fmaxf(mxa[a], mxa[a + w]);
    const float m_loc = mxa[0] * sl2;
    float m_new = m_loc;
    float f_o = 1.f;          // factor taking O from the reference of tile u - 1 to m_new
    bool rescale = false;     // warp-uniform: this warp rescales O before PV(u)
    if (!first) {
        float m_prev;
        if (!ref_get(ref_prev, u, m_prev, abort_flag)) return false;
        const bool need = m_loc > m_prev + (kP8 ? kP8Threshold : kRescaleThreshold);
        m_new = need ? m_loc : m_prev;
        if (need) f_o = ex2_approx(m_prev - m_new);
        rescale = __any_sync(0xffffffffu, need);
    }
    ref_put(ref_mine, m_new, u + 1);     // as early as possible: the other group waits on it
    if (has_g) l_g *= ex2_approx(m_g - m_new);
    m_g = m_new;
    has_g = true;
    float suma[8];
#pragma unroll
    for (int a = 0; a < 8; ++a) suma[a] = 0.f;
    const float neg_m = kP8 ? kP8Offset - m_new : -m_new;
    const uint64_t sl2_2 = bcast2(sl2), neg_m2 = bcast2(neg_m);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        if constexpr (kP8) {
            uint32_t pk[16];
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int c = 2 * half + cc;
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    float x0, x1, x2, x3;
                    fma2_bcast(x0, x1, __uint_as_float(sr[c][i]), __uint_as_float(sr[c][i + 1]), sl2_2, neg_m2);
                    fma2_bcast(x2, x3, __uint_as_float(sr[c][i + 2]), __uint_as_float(sr[c][i + 3]), sl2_2, neg_m2);
                    const float p0 = ex2_approx(x0), p1 = ex2_approx(x1), p2 = ex2_approx(x2), p3 = ex2_approx(x3);
                    pk[cc * 8 + (i >> 2)] = pack_e4m3x4(p0, p1, p2, p3);
                    const int a = 4 * ((i >> 2) & 1);
                    add2_f32(suma[a], suma[a + 1], p0, p1);
                    add2_f32(suma[a + 2], suma[a + 3], p2, p3);
                }
            }
            tmem_st16(tS + half * 16, pk);   // over S columns this thread has already read
        } else {
            uint32_t pk[32];
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int c = 2 * half + cc;
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    float x0, x1;   // s * scale * log2(e) - m for two columns in one packed FMA
                    fma2_bcast(x0, x1, __uint_as_float(sr[c][i]), __uint_as_float(sr[c][i + 1]), sl2_2, neg_m2);
                    const uint32_t pp = pack_bf16x2(ex2_approx(x0), ex2_approx(x1));
                    // the row sum adds the same bf16-rounded weights the PV MMA multiplies
                    const int a = (i >> 1) & 7;
                    suma[a] = add_bf16x2_f32(pp, suma[a]);
                    pk[cc * 16 + (i >> 1)] = pp;
                }
            }
            tmem_st32(tS + half * 32, pk);   // over S columns this thread has already read
        }
    }
#pragma unroll
    for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
        for (int a = 0; a < w; ++a) suma[a] += suma[a + w];
    l_g += suma[0];
    if (rescale) {
        // O holds the sum up to PV(u - 1), relative to the reference of tile u - 1: wait for
        // PV(u - 1) to complete, scale, and only then let PV(u) start
        if (!warp_wait(o_full_prev, o_full_prev_parity, abort_flag)) return false;
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + c * 32, o);
            tmem_wait_ld_dep(o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f_o);
            tmem_st32(tO + c * 32, o);
        }
    }
    tmem_wait_st();
    tc_fence_before();
    warp_signal(p_sig);   // P(u) written and O ready for PV(u)
    return true;
}


}  // namespace tri
}  // namespace swattn

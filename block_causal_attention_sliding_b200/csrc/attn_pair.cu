// attn_pair.cu -- the three-buffer attention on CTA pairs (tcgen05 cta_group::2), d = 128, bf16.
//
// The same result as the other full-chunk kernels -- softmax(scale * Q K^T) V over the keys the
// visibility table lists (condition tokens, sink, window chunks, current chunk; agifrontier
// tutorial "JoyAI-Video-Edit：单卡720p 30帧，两步蒸馏攻克流式视频编辑", section
// "从双向编辑到分块因果架构的蜕变") -- computed by clusters of two CTAs on two SMs.
//
// Work unit: 256 query rows of one (b, h) -- Q tile 2i in the CTA of rank 0, 2i + 1 in rank 1 --
// against all their visible key tiles, or a slice of them: the two-phase schedule of the one-CTA
// three-buffer kernel (tri_common.cuh), over pairs of Q tiles and clusters.  Each key tile takes
// one 256-row S = Q K^T and one 256-row O += P V on the two SMs' tensor cores:
//   * S:  A = Q, each CTA its own 128 rows; B = K, each CTA holding 64 of the tile's 128 keys
//         (rank r: keys 64 r .. 64 r + 63); each CTA receives its 128 rows x all 128 keys.
//   * PV: A = P, from each CTA's own tensor memory; B = V, each CTA holding 64 of the 128 columns
//         for all 128 keys; each CTA receives its 128 rows x all 128 columns of O.
// Per key tile an SM so loads 32 KB of K and V instead of 64 KB, for the same tensor work: its
// ring stages are 16 KB and the loads of the next tiles have twice the lead they have in the
// one-CTA kernel, whose two 32 KB K stages leave them too little.
// Tensor memory per CTA as in the one-CTA kernel: S0 | S1 | S2 | O.
//
// Roles, 11 warps in each CTA:
//   warp 0     TMA producer: this CTA's Q tile and its halves of every K and V tile, in the
//              order the issuer consumes them.  Both CTAs' loads complete on the leader's
//              (rank 0's) barriers, which expect the bytes of both halves;
//   warp 1     rank 0: the MMA issuer for the pair.  Rank 1: the relay (below);
//   warps 2-9  two softmax groups on alternate key tiles over this CTA's 128 rows, sharing one
//              reference max per row through shared memory, as in the one-CTA kernel;
//   warp 10    rank 0: helper that publishes the leader's load barriers as polled words.
// Signals cross between the CTAs only where they must, and a release at cluster scope costs
// hundreds of cycles (measured on B200: ~330 alone, ~1,200 from a softmax warp in this loop;
// 12 at CTA scope), so none is made in a per-tile loop of the softmax warps:
//   * K, V and Q: the leader's barriers count both halves; its helper turns each completed
//     phase into a word (k_seq, v_seq, q_seq) with a CTA-scope release.
//   * P written / O read: every softmax warp signals its own CTA (p_cnt, oe_cnt, CTA-scope
//     release).  In rank 1 the relay acquires those counts tile by tile and forwards them to the
//     leader as p_peer / oe_peer, one cluster-scope release store per tile; the release is
//     cumulative, so it carries the softmax warps' tensor-memory writes with it.
// The issuer never waits on an mbarrier: it polls those words with acquire loads.  Its commits
// arrive on the barriers of both CTAs (multicast): S(u) done, PV(u) done, Q free.
// A CTA leaves only after a cluster barrier that follows the issuer's drain and the leader's
// load drain, so no MMA, copy, commit or remote write reaches a CTA that has gone.  Every other
// wait is bounded.
#include "tri_common.cuh"

namespace swattn {

namespace pairk {

constexpr int D = 128;
constexpr int kKSt = 3;                     // K ring stages, a stage released by S completion (<= 3)
constexpr int kVSt = 3;                     // V ring stages, released by PV completion (<= 3)
constexpr int kQBytes = kBlockM * D * 2;    // 32 KB: this CTA's Q tile, two 64-column boxes
constexpr int kHalfBytes = 16384;           // this CTA's half of a K or a V tile
constexpr int kKBoxBytes = 64 * kBoxCols * 2;   // 8 KB: 64 keys x 64 columns
constexpr int kCtlOffset = kQBytes + (kKSt + kVSt) * kHalfBytes;
constexpr int kThreads = 64 + 2 * 128 + 32;
constexpr int kTmemCols = 512;
constexpr int kOCol = tri::kSBufs * kBlockN;
static_assert(tri::kSBufs * kBlockN + D <= kTmemCols, "tensor memory budget");
static_assert(kKSt <= tri::kSBufs && kVSt <= tri::kSBufs, "ring stages released by S / PV completion");

struct Ext {
    uint64_t s_full[tri::kSBufs];   // S(u) in buffer u % 3 complete (commit, both CTAs)
    uint64_t o_full[tri::kSBufs];   // PV(u) complete (commit, both CTAs)
    uint64_t ep;                    // both groups' row sums are published (8 warps, this CTA)
    uint32_t k_seq, v_seq, q_seq;   // rank 0: K / V of tiles 0..u, Q of pieces 0..pi landed in both CTAs
    uint32_t p_cnt[tri::kSBufs];    // +1 per softmax warp of this CTA once P of the tile in buffer b is written
    uint32_t oe_cnt;                // +1 per softmax warp of this CTA once the piece's O has been read
    uint32_t p_peer, oe_peer;       // rank 0: the same for rank 1, by tile / by piece (the relay)
    unsigned long long ref[2][kBlockM];
    float lsum[2][2][kBlockM];
};

constexpr int kExtOffset = (kCtlOffset + (int)sizeof(SmemCtl) + 15) & ~15;
constexpr int kSmemBytes = kExtOffset + (int)sizeof(Ext) + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
// more than half an SM's shared memory: one CTA per SM, so no CTA waits on another's TMEM
static_assert(kSmemBytes > 114 * 1024, "one CTA per SM");

// A release store into a word of the leader (shared::cluster address); one thread.
__device__ __forceinline__ void st_release_cluster(uint32_t addr, uint32_t v) {
    asm volatile("st.release.cluster.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// S = Q K^T over the pair: 8 MMAs of 16 columns of d.  Q: two 16 KB boxes (128 rows x 64
// columns); this CTA's K half: two 8 KB boxes (64 keys x 64 columns); K-major, 128-byte swizzle.
// The two issue sequences are out of line: measured on B200, that keeps the issuer's code apart
// from the unrolled softmax and the forward takes 3% less time (0.829 against 0.857 ms at 720p).
__device__ __noinline__ void issue_s_pair(uint32_t tS, uint32_t q_tile, uint32_t k_half) {
    constexpr uint32_t idesc = idesc_bf16_f32(2 * kBlockM, kBlockN, false);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t col = (ks & 3) * 32;   // 16 columns = 32 bytes inside the swizzle atom
        mma_ss_pair(tS, smem_desc_sw128(q_tile + (ks >> 2) * kBoxBytes + col, 16, 1024),
                    smem_desc_sw128(k_half + (ks >> 2) * kKBoxBytes + col, 16, 1024), idesc, ks > 0 ? 1u : 0u);
    }
}

// O (+)= P V over the pair: 8 MMAs of 16 keys.  P: bf16 pairs in each CTA's tensor memory; this
// CTA's V half: one 16 KB box of 128 keys x 64 columns, MN-major (one 128-byte swizzle atom wide).
__device__ __noinline__ void issue_pv_pair(uint32_t tO, uint32_t tP, uint32_t v_half, bool accumulate) {
    constexpr uint32_t idesc = idesc_bf16_f32(2 * kBlockM, D, true);
#pragma unroll
    for (int ks = 0; ks < kBlockN / 16; ++ks)
        mma_ts_pair(tO, tP + ks * 8, smem_desc_sw128(v_half + ks * 16 * 128, kBoxBytes, 1024), idesc,
                    (accumulate || ks > 0) ? 1u : 0u);
}

// This CTA's half of K tile j: keys 64 rank .. 64 rank + 63 of the tile (rows past a segment's end
// read as zero and are masked by the softmax), as two 8 KB boxes, completing on the leader's
// barrier `bar` (a shared::cluster address).
__device__ __forceinline__ void load_k_half(const AttnParams& p, const SmemCtl* ctl, int j, int rank, int h, int b,
                                            uint32_t dst, uint32_t bar) {
    int seg, row0, valid;
    tile_of(ctl, j, seg, row0, valid);
    const int kind = ctl->seg_kind[seg];
    const int slot = ctl->seg_slot[seg];
    const int r = row0 + 64 * rank;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        const uint32_t d = dst + c * kKBoxBytes;
        if (kind == 0)
            tma_load_4d_pair(d, &p.tm_cond_kh, bar, c * kBoxCols, r, h, b);
        else if (kind == 1)
            tma_load_5d_pair(d, &p.tm_cache_kh, bar, c * kBoxCols, r, slot, h, b);
        else
            tma_load_4d_pair(d, &p.tm_kcur_h, bar, c * kBoxCols, h, r, b);
    }
}

// This CTA's half of V tile j: columns 64 rank .. 64 rank + 63 of all 128 keys, one 16 KB box.
__device__ __forceinline__ void load_v_half(const AttnParams& p, const SmemCtl* ctl, int j, int rank, int h, int b,
                                            uint32_t dst, uint32_t bar) {
    int seg, row0, valid;
    tile_of(ctl, j, seg, row0, valid);
    const int kind = ctl->seg_kind[seg];
    const int slot = ctl->seg_slot[seg];
    const int x = rank * kBoxCols;
    if (kind == 0)
        tma_load_4d_pair(dst, &p.tm_cond_v, bar, x, row0, h, b);
    else if (kind == 1)
        tma_load_5d_pair(dst, &p.tm_cache_v, bar, x, row0, slot, h, b);
    else
        tma_load_4d_pair(dst, &p.tm_vcur, bar, x, h, row0, b);
}

}  // namespace pairk

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(pairk::kThreads, 1)
attn_pair_kernel(const __grid_constant__ AttnParams p) {
    using namespace pairk;
    extern __shared__ uint8_t smem_raw[];
    // the same offsets in both CTAs: the MMAs address the peer's operands by this CTA's offsets
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* q_smem = base;
    uint8_t* kv_smem = base + kQBytes;
    SmemCtl* ctl = reinterpret_cast<SmemCtl*>(base + kCtlOffset);
    Ext* ex = reinterpret_cast<Ext*>(base + kExtOffset);
    volatile int* abort_flag = &ctl->abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int rank = (int)cluster_ctarank();
    const int g = blockIdx.x >> 1;           // cluster
    const int G = gridDim.x >> 1;

    for (int i = threadIdx.x; i < 2 * kBlockM; i += blockDim.x) (&ex->ref[0][0])[i] = 0ull;   // tags start at 1
    if (threadIdx.x == 64) {
        ex->k_seq = ex->v_seq = ex->q_seq = 0;
        for (int i = 0; i < tri::kSBufs; ++i) ex->p_cnt[i] = 0;
        ex->oe_cnt = 0;
        ex->p_peer = ex->oe_peer = 0;
    }
    if (warp == 0) {
        if (lane == 0) {
            for (int i = 0; i < tri::kSBufs; ++i) {
                mbar_init(smem_u32(&ex->s_full[i]), 1);
                mbar_init(smem_u32(&ex->o_full[i]), 1);
            }
            mbar_init(smem_u32(&ex->ep), 8);
            init_barriers(ctl, kKSt + kVSt);   // fences every init above at cluster scope
        }
        __syncwarp();
        tmem_alloc_pair(smem_u32(&ctl->tmem_base), kTmemCols);   // the same warp in both CTAs
        tmem_relinquish_pair();
    } else if (warp == 1 && lane == 0) {
        tma_prefetch_desc(&p.tm_q);
        tma_prefetch_desc(&p.tm_qc);
        tma_prefetch_desc(&p.tm_kcur_h);
        tma_prefetch_desc(&p.tm_vcur);
        tma_prefetch_desc(&p.tm_cache_kh);
        tma_prefetch_desc(&p.tm_cache_v);
    } else if (warp == 2 && lane == 0) {
        load_table(ctl, p.table, p.status);
    }
    // both CTAs' barriers, counters and tensor memory exist before any commit, remote write or MMA
    tc_fence_before();
    __syncwarp();
    cluster_sync_all();
    tc_fence_after();

    const uint32_t tmem = ctl->tmem_base;
    const int nt = ctl->n_tiles;
    const int nqt = q_tiles(p);
    const int npr = (nqt + 1) / 2;           // units per (b, h): pairs of Q tiles
    tri::Sched sched;
    sched.init(npr, nt, p.B * p.H, G, g);
    constexpr uint16_t kBoth = 3;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0 && nt > 0) {
            const uint32_t kv_base = smem_u32(kv_smem);
            // the leader's barriers, where both CTAs' loads complete; only the leader arms them
            const uint32_t qbar_l = mapa_shared(smem_u32(&ctl->q_full), 0);
            const uint32_t kvbar0_l = mapa_shared(smem_u32(&ctl->kv_full[0]), 0);
            tri::PieceIt pit;
            tri::Piece pc;
            uint32_t t = 0;
            int pi = 0;
            bool ok = true;
            while (ok && tri::next_piece(sched, pit, pc)) {
                const int bh = pc.unit / npr, pr = pc.unit % npr;
                const int b = bh / p.H, h = bh % p.H;
                // a unit with one Q tile: rank 1 runs the last tile again and stores nothing
                const int qtile = min(2 * pr + rank, nqt - 1);
                // the Q buffer is reused: every S MMA of the previous piece has completed
                if (pi > 0 && !wait_or_abort(smem_u32(&ctl->q_empty), (pi - 1) & 1, abort_flag)) break;
                if (rank == 0) mbar_arrive_expect_tx(smem_u32(&ctl->q_full), 2 * kQBytes);
                const QSrc qs = q_src(p, qtile);
                for (int c = 0; c < 2; ++c)
                    tma_load_4d_pair(smem_u32(q_smem + c * kBoxBytes), qs.tm, qbar_l, c * kBoxCols, h, qs.row0, b);
                ++pi;
                const int n = pc.j1 - pc.j0;
                // K(u): its stage last held K(u - kKSt), free once S(u - kKSt) has completed
                auto load_k = [&](int jrel) -> bool {
                    const uint32_t u = t + jrel;
                    if (u >= (uint32_t)kKSt) {
                        const uint32_t v = u - kKSt;
                        if (!wait_or_abort(smem_u32(&ex->s_full[v % tri::kSBufs]), (v / tri::kSBufs) & 1, abort_flag))
                            return false;
                    }
                    const int st = u % kKSt;
                    if (rank == 0) mbar_arrive_expect_tx(smem_u32(&ctl->kv_full[st]), 2 * kHalfBytes);
                    load_k_half(p, ctl, pc.j0 + jrel, rank, h, b, kv_base + st * kHalfBytes, kvbar0_l + st * 8);
                    return true;
                };
                // V(u): its stage last held V(u - kVSt), free once PV(u - kVSt) has completed
                auto load_v = [&](int jrel) -> bool {
                    const uint32_t u = t + jrel;
                    if (u >= (uint32_t)kVSt) {
                        const uint32_t v = u - kVSt;
                        if (!wait_or_abort(smem_u32(&ex->o_full[v % tri::kSBufs]), (v / tri::kSBufs) & 1, abort_flag))
                            return false;
                    }
                    const int st = kKSt + (int)(u % kVSt);
                    if (rank == 0) mbar_arrive_expect_tx(smem_u32(&ctl->kv_full[st]), 2 * kHalfBytes);
                    load_v_half(p, ctl, pc.j0 + jrel, rank, h, b, kv_base + st * kHalfBytes, kvbar0_l + st * 8);
                    return true;
                };
                // consumption order: K(0..2), then V(jj), K(jj + 3)
                for (int k = 0; k < min(3, n) && ok; ++k) ok = load_k(k);
                for (int jj = 0; jj < n && ok; ++jj) {
                    ok = load_v(jj);
                    if (ok && jj + 3 < n) ok = load_k(jj + 3);
                }
                t += n;
            }
            // never leave while copies are in flight: the leader's barriers count both CTAs'
            // loads, so the leader waits for the last fill of every stage (rank 1 cannot leave
            // before the final cluster barrier, which the leader reaches after this)
            if (rank == 0) {
                for (int st = 0; st < kKSt; ++st)
                    if (t > (uint32_t)st) wait_drain(smem_u32(&ctl->kv_full[st]), ((t - 1 - st) / kKSt) & 1);
                for (int st = 0; st < kVSt; ++st)
                    if (t > (uint32_t)st) wait_drain(smem_u32(&ctl->kv_full[kKSt + st]), ((t - 1 - st) / kVSt) & 1);
                if (pi > 0) wait_drain(smem_u32(&ctl->q_full), (pi - 1) & 1);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (rank 0)
        // Per key tile u: one poll point (V(u) and P(u) in both CTAs, K(u + 3) in both), PV(u),
        // commit o_full, S(u + 3) into the same buffer, commit s_full.
        if (rank == 0 && lane == 0 && nt > 0) {
            const uint32_t q_base = smem_u32(q_smem);
            const uint32_t kv_base = smem_u32(kv_smem);
            const uint32_t tO = tmem + kOCol;
            tri::PieceIt pit;
            tri::Piece pc;
            uint32_t t = 0;
            int pi = 0;
            bool ok = true;
            while (ok && tri::next_piece(sched, pit, pc)) {
                const int n = pc.j1 - pc.j0;
                if (!tri::poll_reach(&ex->q_seq, pi + 1, abort_flag)) break;
                for (int k = 0; k < min(3, n) && ok; ++k) {
                    const uint32_t u = t + k;
                    if (!tri::poll_reach(&ex->k_seq, u + 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    // buffer u % 3 last held P(u - 3), read by a PV issued before this S
                    issue_s_pair(tmem + (u % tri::kSBufs) * kBlockN, q_base, kv_base + (u % kKSt) * kHalfBytes);
                    mma_commit_pair(smem_u32(&ex->s_full[u % tri::kSBufs]), kBoth);
                    if (k == n - 1) mma_commit_pair(smem_u32(&ctl->q_empty), kBoth);   // last S of the piece
                }
                for (int jj = 0; jj < n && ok; ++jj) {
                    const uint32_t u = t + jj, bu = u % tri::kSBufs;
                    const bool more = jj + 3 < n;
                    if (!tri::poll_reach(&ex->v_seq, u + 1, abort_flag) ||
                        !tri::poll_reach(&ex->p_cnt[bu], 4 * (u / tri::kSBufs + 1), abort_flag) ||
                        !tri::poll_reach<true>(&ex->p_peer, u + 1, abort_flag) ||
                        (more && !tri::poll_reach(&ex->k_seq, u + 4, abort_flag)) ||
                        // the previous piece's O must be out of both CTAs' TMEM before PV(u) overwrites it
                        (jj == 0 && pi > 0 &&
                         (!tri::poll_reach(&ex->oe_cnt, 8 * pi, abort_flag) ||
                          !tri::poll_reach<true>(&ex->oe_peer, pi, abort_flag)))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t tP = tmem + bu * kBlockN;
                    issue_pv_pair(tO, tP, kv_base + (kKSt + u % kVSt) * kHalfBytes, jj > 0);
                    mma_commit_pair(smem_u32(&ex->o_full[bu]), kBoth);   // PV(u) done: V stage, rescale, epilogue
                    if (more) {
                        // S(u + 3) into the same buffer, in issue order after PV(u) read P(u)
                        issue_s_pair(tP, q_base, kv_base + ((u + 3) % kKSt) * kHalfBytes);
                        mma_commit_pair(smem_u32(&ex->s_full[bu]), kBoth);
                        if (jj + 3 == n - 1) mma_commit_pair(smem_u32(&ctl->q_empty), kBoth);
                    }
                }
                ++pi;
                t += n;
            }
            // every MMA issued has completed before either CTA releases its tensor memory
            mma_commit_pair(smem_u32(&ctl->drain), 1);
            wait_drain(smem_u32(&ctl->drain), 0);
        }
        if (rank == 1 && lane == 0 && nt > 0) {
            // ------------------------------------------------------------ relay (rank 1)
            // Tile by tile, in the issuer's order: once this CTA's 4 softmax warps of tile u have
            // written P (and rescaled O), tell the leader; after each piece, once all 8 warps have
            // read O, tell it that too.  Acquire here at CTA scope, release to the leader at
            // cluster scope: cumulative, so it orders the warps' tensor-memory writes as well.
            const uint32_t w_p = mapa_shared(smem_u32(&ex->p_peer), 0);
            const uint32_t w_oe = mapa_shared(smem_u32(&ex->oe_peer), 0);
            tri::PieceIt pit;
            tri::Piece pc;
            uint32_t t = 0;
            int pi = 0;
            bool ok = true;
            while (ok && tri::next_piece(sched, pit, pc)) {
                const int n = pc.j1 - pc.j0;
                for (int jj = 0; jj < n && ok; ++jj) {
                    const uint32_t u = t + jj;
                    ok = tri::poll_reach(&ex->p_cnt[u % tri::kSBufs], 4 * (u / tri::kSBufs + 1), abort_flag);
                    if (ok) st_release_cluster(w_p, u + 1);
                }
                ++pi;
                t += n;
                if (ok) ok = tri::poll_reach(&ex->oe_cnt, 8 * pi, abort_flag);
                if (ok) st_release_cluster(w_oe, pi);
            }
        }
    } else if (warp == 10) {
        // ------------------------------------------------------------ completion helper (rank 0)
        // Follows the producer's sequence on the leader's barriers (each phase = both CTAs'
        // halves) and publishes each completion as a word the issuer polls.  A stage is refilled
        // only after the issuer has consumed its previous fill, so no barrier here can be more
        // than one phase ahead.
        if (rank == 0 && lane == 0 && nt > 0) {
            tri::PieceIt pit;
            tri::Piece pc;
            uint32_t t = 0;
            int pi = 0;
            bool ok = true;
            while (ok && tri::next_piece(sched, pit, pc)) {
                if (!wait_or_abort(smem_u32(&ctl->q_full), pi & 1, abort_flag)) break;
                ++pi;
                tri::st_release(&ex->q_seq, pi);
                const int n = pc.j1 - pc.j0;
                auto done_k = [&](int jrel) -> bool {
                    const uint32_t u = t + jrel;
                    if (!wait_or_abort(smem_u32(&ctl->kv_full[u % kKSt]), (u / kKSt) & 1, abort_flag)) return false;
                    tri::st_release(&ex->k_seq, u + 1);
                    return true;
                };
                auto done_v = [&](int jrel) -> bool {
                    const uint32_t u = t + jrel;
                    if (!wait_or_abort(smem_u32(&ctl->kv_full[kKSt + u % kVSt]), (u / kVSt) & 1, abort_flag))
                        return false;
                    tri::st_release(&ex->v_seq, u + 1);
                    return true;
                };
                for (int k = 0; k < min(3, n) && ok; ++k) ok = done_k(k);
                for (int jj = 0; jj < n && ok; ++jj) {
                    ok = done_v(jj);
                    if (ok && jj + 3 < n) ok = done_k(jj + 3);
                }
                t += n;
            }
        }
    } else if (warp >= 2) {
        // ------------------------------------------------------------ softmax groups
        const int sw = warp - 2;          // 0..7
        const int gr = sw >> 2;           // group: key tiles u with u & 1 == gr
        const int wq = warp & 3;          // TMEM lane quarter (fixed by the warp's slot)
        const int row = wq * 32 + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(wq * 32) << 16);
        const uint32_t tO = lane_base + kOCol;
        tri::PieceIt pit;
        tri::Piece pc;
        int sk_pi = 0;            // stream-K pieces seen (the first and last may be split)
        uint32_t t = 0;           // key tiles of all pieces so far
        uint32_t ucnt = 0;        // pieces done (ep phases)
        bool ok = nt > 0;
        while (ok && tri::next_piece(sched, pit, pc)) {
            const bool first_sk = pc.sk && sk_pi == 0;
            if (pc.sk) ++sk_pi;
            const int n = pc.j1 - pc.j0;
            float m_g = 0.f, l_g = 0.f;
            bool has_g = false;
            for (int jj = (int)((gr + t) & 1); jj < n; jj += 2) {
                const uint32_t u = t + jj, bu = u % tri::kSBufs;
                int seg, row0, valid;
                tile_of(ctl, pc.j0 + jj, seg, row0, valid);
                ok = warp_wait(smem_u32(&ex->s_full[bu]), (u / tri::kSBufs) & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t up = u - 1;   // unused when jj == 0
                ok = tri::softmax_tile<D>(lane_base + bu * kBlockN, tO, valid, jj == 0, u, &ex->ref[up & 1][row],
                                          &ex->ref[u & 1][row], smem_u32(&ex->o_full[up % tri::kSBufs]),
                                          (up / tri::kSBufs) & 1, smem_u32(&ex->p_cnt[bu]), p.scale_log2, m_g, l_g,
                                          has_g, abort_flag);
                if (!ok) break;
            }
            // ---------------------------------------------------- epilogue of this piece
            const uint32_t tl = t + n - 1;   // the piece's last key tile
            const int par = ucnt & 1;
            float m_fin = m_g;
            if (ok && (int)(tl & 1) != gr) ok = tri::ref_get(&ex->ref[tl & 1][row], tl + 1, m_fin, abort_flag);
            float l_row = 0.f;
            if (ok) {
                ex->lsum[par][gr][row] = has_g ? l_g * ex2_approx(m_g - m_fin) : 0.f;
                warp_arrive(smem_u32(&ex->ep));
                ok = warp_wait(smem_u32(&ex->ep), par, abort_flag);
            }
            if (ok) {
                l_row = ex->lsum[par][0][row] + ex->lsum[par][1][row];
                // PV(tl - 3) has completed (S(tl) was seen before the exchange), so o_full of
                // buffer tl % 3 is at most one phase behind the one awaited
                ok = warp_wait(smem_u32(&ex->o_full[tl % tri::kSBufs]), (tl / tri::kSBufs) & 1, abort_flag);
            }
            ok = tri::vote_all(ok);
            ++ucnt;
            t += n;
            if (!ok) break;
            tc_fence_after();
            uint32_t o[D / 64][32];   // this group's half of the O columns
#pragma unroll
            for (int c = 0; c < D / 64; ++c) tmem_ld32(tO + gr * (D / 2) + c * 32, o[c]);
            tmem_wait_ld_dep(o[0]);
#pragma unroll
            for (int c = 1; c < D / 64; ++c) reg_fence(o[c]);
            tc_fence_before();
            tri::warp_signal(smem_u32(&ex->oe_cnt));   // O may now be overwritten

            const int bh = pc.unit / npr, pr = pc.unit % npr;
            const int qtile = 2 * pr + rank;
            if (qtile >= nqt) continue;   // the second tile of a one-tile unit: nothing to store
            const int b = bh / p.H, h = bh % p.H;
            const QSrc qs = q_src(p, qtile);
            const int m_row = qs.row0 + row;
            const size_t orow = ((size_t)b * qs.rows + m_row) * p.H + h;
            if (pc.j0 == 0 && pc.j1 == nt) {
                const float inv = 1.f / l_row;
                if (m_row < qs.rows) {
#pragma unroll
                    for (int c = 0; c < D / 64; ++c)
                        store_row_chunk<D>(qs.out, p.out_f32, orow, gr * (D / 64) + c, o[c], inv);
                }
                continue;
            }
            // split piece: publish the partial, then the last of the tile's pieces merges.  Slots
            // are per CTA (2 per CTA: its first and its last stream-K piece); the pieces of this
            // tile live in the CTAs of the same rank of clusters g_first .. g_last.
            const long long ps = sched.cstart(pc.unit);
            const int g_first = sched.cta_of(ps);
            const int g_last = sched.cta_of(ps + nt - 1);
            const int npieces = g_last - g_first + 1;
            const int slot = first_sk ? 2 * (int)blockIdx.x : 2 * (int)blockIdx.x + 1;
            float* so = p.sk_o + (size_t)slot * 2 * D * kBlockM;       // [D][128 rows]
            float* sml = p.sk_ml + (size_t)slot * 2 * kBlockM * 2;     // [128 rows][2]
#pragma unroll
            for (int c = 0; c < D / 64; ++c)
#pragma unroll
                for (int i = 0; i < 32; ++i) so[(gr * (D / 2) + c * 32 + i) * kBlockM + row] = __uint_as_float(o[c][i]);
            if (gr == 0) {
                sml[row * 2 + 0] = m_fin;
                sml[row * 2 + 1] = l_row;
            }
            __threadfence();
            tri::softmax_bar();
            int* cnt = p.sk_cnt + (size_t)bh * (2 * p.sk_pairs) + qtile;
            if (sw == 0 && lane == 0) ctl->merge_flag[0] = atomicAdd(cnt, 1);
            tri::softmax_bar();
            if (ctl->merge_flag[0] != npieces - 1) continue;     // another piece will merge
            __threadfence();
            // the tile's first piece is cluster g_first's first stream-K piece iff g_first's range
            // opens inside this unit; every later cluster's piece of it opens that cluster's range
            tri::Sched sf = sched;
            sf.set_range(g_first);
            const bool opens_first = sf.u0 + (int)(sf.c0 / nt) == pc.unit;
            auto slot_of = [&](int gg) {
                const int cta = 2 * gg + rank;
                return gg == g ? slot : ((gg > g_first || opens_first) ? 2 * cta : 2 * cta + 1);
            };
            float M = -INFINITY;
            for (int gg = g_first; gg <= g_last; ++gg)
                M = fmaxf(M, __ldcg(p.sk_ml + (size_t)slot_of(gg) * 2 * kBlockM * 2 + row * 2));
            float L_ = 0.f;
            for (int gg = g_first; gg <= g_last; ++gg) {
                const float* pml = p.sk_ml + (size_t)slot_of(gg) * 2 * kBlockM * 2 + row * 2;
                L_ += ex2_approx(__ldcg(pml) - M) * __ldcg(pml + 1);
            }
            const float inv = 1.f / L_;
#pragma unroll 1
            for (int c = 0; c < D / 64; ++c) {      // 32 columns at a time
                uint32_t acc[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) acc[i] = 0u;
                for (int gg = g_first; gg <= g_last; ++gg) {
                    const int sl = slot_of(gg);
                    const float w = ex2_approx(__ldcg(p.sk_ml + (size_t)sl * 2 * kBlockM * 2 + row * 2) - M);
                    const float* po = p.sk_o + (size_t)sl * 2 * D * kBlockM + (gr * (D / 2) + c * 32) * kBlockM + row;
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        acc[i] = __float_as_uint(fmaf(w, __ldcg(po + i * kBlockM), __uint_as_float(acc[i])));
                }
                if (m_row < qs.rows) store_row_chunk<D>(qs.out, p.out_f32, orow, gr * (D / 64) + c, acc, inv);
            }
            if (sw == 0 && lane == 0) atomicExch(cnt, 0);   // all pieces arrived: ready for the next launch
        }
    }

    // the issuer has drained (its warp arrives here after the drain), and every remote write and
    // commit arrival is ordered before this barrier: both CTAs may now release tensor memory
    tc_fence_before();
    __syncwarp();
    cluster_sync_all();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
    if (threadIdx.x == 0 && ctl->abort_flag) atomicOr(p.status, SW_STATUS_TIMEOUT);
}

cudaError_t launch_pair(const AttnParams& p, int clusters, cudaStream_t stream) {
    if (clusters < 1 || 2 * clusters > kMaxPersistentCtas) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(attn_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         pairk::kSmemBytes);
    if (e != cudaSuccess) return e;
    attn_pair_kernel<<<2 * clusters, pairk::kThreads, pairk::kSmemBytes, stream>>>(p);
    return cudaGetLastError();
}

int pair_max_clusters() {
    if (cudaFuncSetAttribute(attn_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, pairk::kSmemBytes) !=
        cudaSuccess)
        return 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * 74);
    cfg.blockDim = dim3(pairk::kThreads);
    cfg.dynamicSmemBytes = pairk::kSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, attn_pair_kernel, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        return 0;
    }
    return n;
}

}  // namespace swattn

// attn_persistent.cu -- the full-chunk attention as a persistent, load-balanced kernel.
//
// Same computation and warp roles as attn_fwd_kernel (TMA producer, one-thread tcgen05 MMA
// issuer, one softmax warpgroup per 128-row Q tile), but the grid is one CTA per SM and the
// work is dealt out in two phases:
//   1. whole pairs of Q tiles, round-robin (CTA g takes pairs g, g + G, ...) for as many full
//      rounds as there are -- like the one-CTA-per-pair grid, so the CTAs running together
//      share a handful of heads and their K/V stay in L2;
//   2. the leftover pairs (fewer than G) as one line of (pair, key tile) items costed by the
//      number of live Q tiles, cut evenly between the CTAs ("stream-K"), so no SM idles while
//      a partial last wave runs.
// A pair whose key tiles are cut between CTAs ("split piece") is merged without any inter-CTA
// waiting: every piece writes its unnormalised O rows and (max, sum) to a scratch slot, then
// bumps a per-pair counter; the piece that sees the counter reach npieces - 1 is last, merges
// all pieces in slot order (log-sum-exp) and writes the output, then clears the counter.
//
// Within a CTA, consecutive pieces overlap: the producer streams the next piece's Q and K/V
// while the softmax warpgroups finish the previous piece's epilogue; the first P V of a piece
// waits only until the epilogue has read the previous O out of TMEM.
#include "persist_sched.cuh"

namespace swattn {

// The MMA issuer runs as a converged warp (one lane issues each tcgen05 instruction, chosen by
// elect.sync) rather than as one thread of a divergent branch.
#ifndef SWATTN_MMA_WARP
#define SWATTN_MMA_WARP 1
#endif
constexpr bool kMmaWarp = SWATTN_MMA_WARP != 0;

// The merge of a split pair at the merging CTA's last piece is staged through idle shared memory
// by bulk copies (see the epilogue).
#ifndef SWATTN_STAGED_MERGE
#define SWATTN_STAGED_MERGE 1
#endif
constexpr bool kStagedMerge = SWATTN_STAGED_MERGE != 0;

// Half of O += P V (keys [64 half, 64 half + 64) of the tile): bf16 P and V on kind::f16, or e4m3
// P and V on kind::f8f6f4.
template <int D, bool kPV8>
__device__ __forceinline__ void pv_half(uint32_t tO, uint32_t tP, uint32_t v_tile, int half, bool accumulate) {
    if constexpr (kPV8) issue_pv_f8_half<kMmaWarp>(tO, tP, v_tile, half, accumulate);
    else issue_pv_half<D, kMmaWarp>(tO, tP, v_tile, half, accumulate);
}

// A bounded wait in the MMA issuer: warp-uniform when the whole warp runs the issuer, so that
// every lane takes the same branch before the next elect.sync.
template <bool kWarp>
__device__ __forceinline__ bool mma_wait(uint32_t bar, uint32_t parity, volatile int* flag) {
    if constexpr (kWarp) return warp_wait(bar, parity, flag);
    else return wait_or_abort(bar, parity, flag);
}

// Two waits of the issuer at once: both phases are tested in one block first (the common case,
// both long complete, then costs one round trip), and only if that fails are they waited for one
// after the other, bounded as usual.
template <bool kWarp>
__device__ __forceinline__ bool mma_wait2(uint32_t bar_a, uint32_t parity_a, uint32_t bar_b, uint32_t parity_b,
                                          volatile int* flag) {
    bool both = mbar_try_wait2(bar_a, parity_a, bar_b, parity_b);
    if constexpr (kWarp) both = __all_sync(0xffffffffu, both);
    if (both) return true;
    return mma_wait<kWarp>(bar_a, parity_a, flag) && mma_wait<kWarp>(bar_b, parity_b, flag);
}

// The TMA producer (one thread): Q tiles per piece, then the piece's K and V tiles in ring
// order.  A function of its own, not inlined: the kernel's register budget is set by the softmax
// warps, and the roles that hold little state must not have their loop state spilled for them.
template <int D, bool kCommit, bool kQK8, bool kPV8>
__device__ __noinline__ void persist_producer(const AttnParams& p, SmemCtl* ctl, uint8_t* q_smem, uint8_t* kv_smem,
                                             Sched sched, volatile int* abort_flag) {
    constexpr int NQ = 2;
    constexpr int kStages = TileCfg<D>::kStages;
    constexpr int kTileBytes = TileCfg<D>::kTileBytes;
    const uint32_t qbar = smem_u32(&ctl->q_full);
    PieceIt pit;
    Piece pc;
    uint32_t it = 0;
    int pi = 0;
    bool ok = true;
    // fused commit: the chunk's K_cur / V_cur tile j is stored by the piece of Q-tile pair
    // j mod npairs that loads it, so the stores spread over the CTAs
    const int cslot = kCommit ? ring_slot(__ldg(p.table), p.ring_R, p.sink) : -1;
    CommitQueue<D, kStages, kQK8, kPV8> cq;
    while (ok && next_piece(sched, pit, pc)) {
        const int b = pc.bh / p.H, h = pc.bh % p.H;
        // the Q buffers are reused: wait until every S MMA of the previous piece is done
        if (pi > 0 && !wait_or_abort(smem_u32(&ctl->q_empty), (pi - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(qbar, pc.live * QKTile<D, kQK8>::kBytes);
        for (int qt = 0; qt < pc.live; ++qt) {
            const QSrc qs = q_src(p, pc.pair * NQ + qt);
            for (int c = 0; c < QKTile<D, kQK8>::kBoxes; ++c)
                tma_load_4d(smem_u32(q_smem + qt * kTileBytes + c * kBoxBytes), qs.tm, qbar,
                            c * QKTile<D, kQK8>::kBoxCols, h, qs.row0, b);
        }
        ++pi;
        for (int j = pc.j0; j < pc.j1 && ok; ++j) {
            for (int kv = 0; kv < 2; ++kv, ++it) {
                const int s = it % kStages;
                const uint32_t r = it / kStages;
                if (!wait_or_abort(smem_u32(&ctl->kv_empty[s]), (r & 1) ^ 1, abort_flag)) {
                    ok = false;
                    break;
                }
                if (kCommit) cq.before_refill(s);
                const uint32_t fbar = smem_u32(&ctl->kv_full[s]);
                mbar_arrive_expect_tx(fbar, kv_tile_bytes<D, kQK8, kPV8>(kv));
                load_kv_tile<D, kQK8, kPV8>(p, ctl, j, kv, h, b, smem_u32(kv_smem + s * kTileBytes), fbar);
                if (kCommit) {
                    const bool mine = cslot >= 0 && pc.pair == j % sched.npairs &&
                                      ctl->seg_kind[tile_seg(ctl, j)] == 2;
                    if (!cq.step(p, ctl, kv_smem, cslot, it, CommitQueue<D, kStages>::pack(mine, j, kv, h, b),
                                 abort_flag)) {
                        ok = false;
                        break;
                    }
                }
            }
        }
    }
    if (kCommit) {
        if (ok) (void)cq.flush(p, ctl, kv_smem, cslot, it, abort_flag);
        bulk_wait_all();
    }
    for (int s = 0; s < kStages; ++s) {
        if (it > (uint32_t)s) {
            const uint32_t uses = (it - 1 - s) / kStages + 1;
            wait_drain(smem_u32(&ctl->kv_full[s]), (uses - 1) & 1);
        }
    }
    if (pi > 0) wait_drain(qbar, (pi - 1) & 1);
    mbar_arrive(smem_u32(&ctl->prod_done));   // no copy of this CTA reads or writes shared memory any more
}

// The MMA issuer (one thread): per piece, S of each live Q tile for the first key tile, then per
// key tile P V and the next tile's S for each live Q tile, in issue order.  Not inlined, for the
// same reason as the producer.
template <int D, bool kQK8, bool kPV8>
__device__ __noinline__ void persist_mma(SmemCtl* ctl, uint8_t* q_smem, uint8_t* kv_smem, uint32_t tmem,
                                        Sched sched, volatile int* abort_flag) {
    constexpr int NQ = 2;
    constexpr int kStages = TileCfg<D>::kStages;
    constexpr int kTileBytes = TileCfg<D>::kTileBytes;
    const uint32_t q_base = smem_u32(q_smem);
    const uint32_t kv_base = smem_u32(kv_smem);
    PieceIt pit;
    Piece pc;
    uint32_t it = 0;          // K/V tiles consumed so far (ring position)
    int pi = 0;               // pieces started
    uint32_t tcnt[2] = {0, 0};   // key tiles processed per Q tile (p_full phases)
    uint32_t ucnt[2] = {0, 0};   // pieces finished per Q tile (o_empty phases)
    bool ok = true;
    while (ok && next_piece(sched, pit, pc)) {
        const int n = pc.j1 - pc.j0;
        const int live = pc.live;
        if (!mma_wait<kMmaWarp>(smem_u32(&ctl->q_full), pi & 1, abort_flag)) break;
        ++pi;
        const int s0 = it % kStages;
        if (!mma_wait<kMmaWarp>(smem_u32(&ctl->kv_full[s0]), (it / kStages) & 1, abort_flag)) break;
        tc_fence_after();
        for (int qt = 0; qt < live; ++qt) {
            issue_s_qk<D, kQK8, kMmaWarp>(tmem + qt * kBlockN, q_base + qt * kTileBytes, kv_base + s0 * kTileBytes);
            mma_commit_any<kMmaWarp>(smem_u32(&ctl->s_full[qt]));
        }
        if (n == 1) mma_commit_any<kMmaWarp>(smem_u32(&ctl->q_empty));
        mma_commit_any<kMmaWarp>(smem_u32(&ctl->kv_empty[s0]));
        for (int jj = 0; jj < n && ok; ++jj) {
            const uint32_t itV = it + 2 * jj + 1, itK = it + 2 * jj + 2;
            const int sV = itV % kStages, sK = itK % kStages;
            const bool more = jj + 1 < n;
            for (int qt = 0; qt < live && ok; ++qt) {
                const uint32_t tO = tmem + NQ * kBlockN + qt * D, tP = tmem + qt * kBlockN;
                const uint32_t pbar = smem_u32(kSplitP ? &ctl->p_half[qt] : &ctl->p_full[qt]);
                const uint32_t fbar = smem_u32(&ctl->p_full[qt]), ppar = tcnt[qt] & 1;
                const uint32_t vbar = smem_u32(&ctl->kv_full[sV]), vpar = (itV / kStages) & 1;
                const uint32_t kbar = smem_u32(&ctl->kv_full[sK]), kpar = (itK / kStages) & 1;
                // V of this key tile is waited for together with the first Q tile's P
                if (!(qt == 0 ? mma_wait2<kMmaWarp>(vbar, vpar, pbar, ppar, abort_flag)
                              : mma_wait<kMmaWarp>(pbar, ppar, abort_flag))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (jj == 0 && ucnt[qt] > 0) {
                    // the previous piece's O must be out of TMEM before it is overwritten
                    if (!mma_wait<kMmaWarp>(smem_u32(&ctl->o_empty[qt]), (ucnt[qt] - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                }
                if (kSplitP) {
                    pv_half<D, kPV8>(tO, tP, kv_base + sV * kTileBytes, 0, jj > 0);
                    // the first Q tile's full P is waited for together with the next K tile
                    if (!(qt == 0 && more ? mma_wait2<kMmaWarp>(fbar, ppar, kbar, kpar, abort_flag)
                                          : mma_wait<kMmaWarp>(fbar, ppar, abort_flag))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    pv_half<D, kPV8>(tO, tP, kv_base + sV * kTileBytes, 1, true);
                } else {
                    pv_half<D, kPV8>(tO, tP, kv_base + sV * kTileBytes, 0, jj > 0);
                    pv_half<D, kPV8>(tO, tP, kv_base + sV * kTileBytes, 1, true);
                }
                ++tcnt[qt];
                if (!more) mma_commit_any<kMmaWarp>(smem_u32(&ctl->o_full[qt]));   // O complete: epilogue
                if (more) {
                    if (qt == 0 && !kSplitP && !mma_wait<kMmaWarp>(kbar, kpar, abort_flag)) {
                        ok = false;
                        break;
                    }
                    // in issue order after the PV that reads P_q from the same columns
                    issue_s_qk<D, kQK8, kMmaWarp>(tmem + qt * kBlockN, q_base + qt * kTileBytes, kv_base + sK * kTileBytes);
                    mma_commit_any<kMmaWarp>(smem_u32(&ctl->s_full[qt]));
                }
            }
            if (!ok) break;
            if (more && jj + 2 == n) mma_commit_any<kMmaWarp>(smem_u32(&ctl->q_empty));   // last S issued
            mma_commit_any<kMmaWarp>(smem_u32(&ctl->kv_empty[sV]));
            if (more) mma_commit_any<kMmaWarp>(smem_u32(&ctl->kv_empty[sK]));
        }
        for (int qt = 0; qt < live; ++qt) ++ucnt[qt];
        it += 2 * n;
    }
    mma_commit_any<kMmaWarp>(smem_u32(&ctl->drain));
    wait_drain(smem_u32(&ctl->drain), 0);
}

// kCommit: the launch also stores the chunk's K_cur / V_cur into the cache (fused commit); a
// separate instantiation, so the plain forward carries none of that code.
// kQK8: Q and K are e4m3 (d = 128), S = Q K^T on kind::f8f6f4; V, P and O as in the bf16 kernel.
// kPV8 (with kQK8): V is e4m3 too and O += P V runs on kind::f8f6f4 with P quantised to e4m3; the
// V scale is applied with the final normalisation.
template <int D, bool kCommit, bool kQK8, bool kPV8>
__global__ void __launch_bounds__(AttnLayout<D, 2>::kThreads, 1)
attn_persistent_kernel(const __grid_constant__ AttnParams p) {
    constexpr int NQ = 2;
    using C = TileCfg<D>;
    using L = AttnLayout<D, NQ>;
    constexpr int kStages = C::kStages;
    constexpr int kTileBytes = C::kTileBytes;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* q_smem = base;
    uint8_t* kv_smem = base + L::kQBytes;
    SmemCtl* ctl = reinterpret_cast<SmemCtl*>(base + L::kCtlOffset);
    volatile int* abort_flag = &ctl->abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (warp == 0) {
        if (lane == 0) init_barriers(ctl, kStages);
        __syncwarp();
        tmem_alloc(smem_u32(&ctl->tmem_base), L::kTmemCols);
        tmem_relinquish();
    } else if (warp == 1 && lane == 0) {
        tma_prefetch_desc(&p.tm_q);
        tma_prefetch_desc(&p.tm_qc);
        tma_prefetch_desc(&p.tm_kcur);
        tma_prefetch_desc(&p.tm_vcur);
        tma_prefetch_desc(&p.tm_cache_k);
        tma_prefetch_desc(&p.tm_cache_v);
    }
    // launched as a programmatic dependent: the set-up above (barriers, TMEM, descriptors, none
    // of it in global memory) overlaps the previous kernel's tail; the table, the inputs, the
    // cache, the partials, their counters and the output are touched only after that kernel has
    // completed with its writes visible
    grid_dependency_wait();
    if (warp == 2 && lane == 0) load_table(ctl, p.table, p.status);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem = ctl->tmem_base;
    const int g = blockIdx.x;
    const int nt = ctl->n_tiles;
    const int nqt = q_tiles(p);
    Sched sched;
    sched.init(nqt, nt, p.B * p.H, (int)gridDim.x, g);

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0 && nt > 0) persist_producer<D, kCommit, kQK8, kPV8>(p, ctl, q_smem, kv_smem, sched, abort_flag);
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if ((kMmaWarp || lane == 0) && nt > 0) persist_mma<D, kQK8, kPV8>(ctl, q_smem, kv_smem, tmem, sched, abort_flag);
    } else {
        // ------------------------------------------------------------ softmax warpgroups
        const int qt = (warp - 2) >> 2;
        const int wq = warp & 3;
        const int row = wq * 32 + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(wq * 32) << 16);
        const uint32_t tS = lane_base + qt * kBlockN;
        const uint32_t tO = lane_base + NQ * kBlockN + qt * D;
        const uint32_t o_bar = smem_u32(&ctl->o_full[qt]);
        PieceIt pit;
        Piece pc;
        int sk_pi = 0;            // stream-K pieces seen (the first and last may be split)
        uint32_t tcnt = 0;        // key tiles processed (s_full phases)
        uint32_t ucnt = 0;        // pieces processed (o_full phases: one per piece)
        uint32_t it_base = 0;     // K/V ring items of the pieces before this one
        bool ok = nt > 0;
        while (ok && next_piece(sched, pit, pc)) {
            const bool first_sk = pc.sk && sk_pi == 0;
            if (pc.sk) ++sk_pi;
            const int n = pc.j1 - pc.j0;
            const uint32_t it_piece = it_base;
            it_base += 2 * n;
            if (qt >= pc.live) continue;
            float m_ref = -INFINITY, l = 0.f;
            for (int jj = 0; jj < n; ++jj) {
                int seg, row0, valid;
                tile_of(ctl, pc.j0 + jj, seg, row0, valid);
                ok = warp_wait(smem_u32(&ctl->s_full[qt]), tcnt & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                softmax_step<D, false, kPV8>(tS, tO, valid, jj == 0, smem_u32(&ctl->p_half[qt]), p.scale_log2, m_ref, l);
                warp_arrive(smem_u32(&ctl->p_full[qt]));
                ++tcnt;
            }
            // ---------------------------------------------------- epilogue of this piece
            if (ok) ok = warp_wait(o_bar, ucnt & 1, abort_flag);
            ++ucnt;
            // every warp of the group reaches this point once per piece, failed or not, and
            // all of them go on (or leave) together
            ok = wg_all(qt, ok);
            if (!ok) break;
            tc_fence_after();
            uint32_t o[D / 32][32];
#pragma unroll
            for (int c = 0; c < D / 32; ++c) tmem_ld32(tO + c * 32, o[c]);
            tmem_wait_ld_dep(o[0]);
#pragma unroll
            for (int c = 1; c < D / 32; ++c) reg_fence(o[c]);
            tc_fence_before();
            warp_arrive(smem_u32(&ctl->o_empty[qt]));   // O may now be overwritten

            const int b = pc.bh / p.H, h = pc.bh % p.H;
            const QSrc qs = q_src(p, pc.pair * NQ + qt);
            const int m_row = qs.row0 + row;
            const size_t orow = ((size_t)b * qs.rows + m_row) * p.H + h;
            if (pc.j0 == 0 && pc.j1 == nt) {
                const float inv = kPV8 ? p.out_scale / l : 1.f / l;
                if (m_row < qs.rows) {
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) store_row_chunk<D>(qs.out, p.out_f32, orow, c, o[c], inv);
                }
                continue;
            }
            // split piece: publish the partial, then the last of the pair's pieces merges
            const int pidx = pc.bh * sched.npairs + pc.pair;
            const long long ps = sched.cstart(pidx);
            const int g_first = sched.cta_of(ps);
            const int g_last = sched.cta_of(ps + (long long)pc.live * (nt - 1));
            const int npieces = g_last - g_first + 1;
            const int slot = first_sk ? 2 * g : 2 * g + 1;
            float* so = p.sk_o + ((size_t)slot * 2 + qt) * D * kBlockM;     // [D][128 rows]
            float* sml = p.sk_ml + ((size_t)slot * 2 + qt) * kBlockM * 2;   // [128 rows][2]
#pragma unroll
            for (int c = 0; c < D / 32; ++c)
#pragma unroll
                for (int i = 0; i < 32; ++i) so[(c * 32 + i) * kBlockM + row] = __uint_as_float(o[c][i]);
            sml[row * 2 + 0] = m_ref;
            sml[row * 2 + 1] = l;
            __threadfence();
            wg_bar(qt);
            int* cnt = p.sk_cnt + ((size_t)pc.bh * p.sk_pairs + pc.pair) * 2 + qt;
            if (row == 0) ctl->merge_flag[qt] = atomicAdd(cnt, 1);
            wg_bar(qt);
            if (ctl->merge_flag[qt] != npieces - 1) continue;     // another piece will merge
            __threadfence();
            // the pair's first piece is CTA g_first's last piece unless it opens that CTA's
            // stream-K range
            bool opens_first = false;
            {
                Sched sf = sched;
                sf.g = g_first;
                sf.set_range(g_first);
                PieceIt fit;
                fit.r = sf.rounds;
                Piece fp;
                if (next_piece(sf, fit, fp)) opens_first = fp.bh == pc.bh && fp.pair == pc.pair;
            }
            // merge every piece -- this one's too, read back -- in slot order, so the result
            // does not depend on which piece happened to arrive last
            const auto slot_of = [&](int gg) {
                return gg == g ? slot : ((gg > g_first || opens_first) ? 2 * gg : 2 * gg + 1);
            };
            float M = -INFINITY;
            for (int gg = g_first; gg <= g_last; ++gg)
                M = fmaxf(M, __ldcg(p.sk_ml + ((size_t)slot_of(gg) * 2 + qt) * kBlockM * 2 + row * 2));
            float L_ = 0.f;
#pragma unroll
            for (int c = 0; c < D / 32; ++c)
#pragma unroll
                for (int i = 0; i < 32; ++i) o[c][i] = 0u;
            // At this CTA's last piece the producer is done and no MMA reads this Q tile's buffer
            // or any ring stage but the one of the piece's last V (and that one neither, once this
            // group's own last P V has completed): the partials are then staged through those
            // buffers with bulk copies, three in flight, instead of loaded by each thread -- the
            // direct loads are latency-bound at ~30 in flight per thread.  Same additions in the
            // same order either way, so the result is bit-identical.
            PieceIt after = pit;
            Piece nxt;
            // (at the last piece the producer has finished, or is about to: its fused-commit stores
            // may still read ring stages until it signals prod_done)
            bool staged = kStagedMerge && !next_piece(sched, after, nxt);   // the same in every warp
            if (staged) staged = wg_all(qt, warp_wait(smem_u32(&ctl->prod_done), 0, abort_flag));
            if (staged) {
                constexpr int kChunkCols = kTileBytes / (kBlockM * 4);   // partial columns per buffer
                constexpr int kChunksPerSlot = D / kChunkCols;
                const int s_last = (int)((it_piece + 2 * n - 1) % kStages);
                int fs0 = -1, fs1 = -1, fs2 = -1;   // the stages other than s_last, in order
                for (int st = 0; st < kStages; ++st) {
                    if (st == s_last) continue;
                    if (fs0 < 0) fs0 = st;
                    else if (fs1 < 0) fs1 = st;
                    else if (fs2 < 0) fs2 = st;
                }
                uint8_t* const b0 = q_smem + qt * kTileBytes;
                uint8_t* const b1 = kv_smem + (qt == 0 ? fs0 : fs2) * kTileBytes;
                uint8_t* const b2 = kv_smem + (qt == 0 ? fs1 : s_last) * kTileBytes;
                const auto buf = [&](int b) { return b == 0 ? b0 : (b == 1 ? b1 : b2); };
                const int nchunks = npieces * kChunksPerSlot;
                const bool issuer = row == 0;
                const auto issue = [&](int k) {
                    const int gg = g_first + k / kChunksPerSlot, part = k % kChunksPerSlot;
                    const float* src = p.sk_o + ((size_t)slot_of(gg) * 2 + qt) * D * kBlockM +
                                       (size_t)part * kChunkCols * kBlockM;
                    const uint32_t bar = smem_u32(&ctl->merge_bar[qt][k % 3]);
                    mbar_arrive_expect_tx(bar, kTileBytes);
                    bulk_load_1d(smem_u32(buf(k % 3)), src, kTileBytes, bar);
                };
                int issued = 0;
                if (issuer) {
                    fence_proxy_async_global();
                    for (; issued < 3 && issued < nchunks; ++issued) issue(issued);
                }
                int k = 0;
                for (; k < nchunks; ++k) {
                    const int gg = g_first + k / kChunksPerSlot, part = k % kChunksPerSlot;
                    bool mok = warp_wait(smem_u32(&ctl->merge_bar[qt][k % 3]), (k / 3) & 1, abort_flag);
                    if (mok) {
                        const float w = ex2_approx(__ldcg(p.sk_ml + ((size_t)slot_of(gg) * 2 + qt) * kBlockM * 2 + row * 2) - M);
                        const float* bf = reinterpret_cast<const float*>(buf(k % 3)) + row;
#pragma unroll
                        for (int c = 0; c < D / 32; ++c) {
                            if (c / (kChunkCols / 32) != part) continue;
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                o[c][i] = __float_as_uint(fmaf(w, bf[(c * 32 + i - part * kChunkCols) * kBlockM],
                                                               __uint_as_float(o[c][i])));
                        }
                    }
                    // every thread of the group is done with this buffer before it is refilled
                    if (!wg_all(qt, mok)) break;
                    if (issuer && issued < nchunks) issue(issued++);
                }
                if (issuer)   // a failed wait leaves copies in flight: let them land before leaving
                    for (int kk = k; kk < issued; ++kk) wait_drain(smem_u32(&ctl->merge_bar[qt][kk % 3]), (kk / 3) & 1);
                for (int gg = g_first; gg <= g_last; ++gg) {
                    const float* pml = p.sk_ml + ((size_t)slot_of(gg) * 2 + qt) * kBlockM * 2 + row * 2;
                    L_ += ex2_approx(__ldcg(pml) - M) * __ldcg(pml + 1);
                }
            } else {
                for (int gg = g_first; gg <= g_last; ++gg) {
                    const float* pml = p.sk_ml + ((size_t)slot_of(gg) * 2 + qt) * kBlockM * 2 + row * 2;
                    const float w = ex2_approx(__ldcg(pml) - M);
                    L_ += w * __ldcg(pml + 1);
                    const float* po = p.sk_o + ((size_t)slot_of(gg) * 2 + qt) * D * kBlockM + row;
#pragma unroll
                    for (int c = 0; c < D / 32; ++c)
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            o[c][i] = __float_as_uint(fmaf(w, __ldcg(po + (c * 32 + i) * kBlockM), __uint_as_float(o[c][i])));
                }
            }
            const float inv = kPV8 ? p.out_scale / L_ : 1.f / L_;
            if (m_row < qs.rows) {
#pragma unroll
                for (int c = 0; c < D / 32; ++c) store_row_chunk<D>(qs.out, p.out_f32, orow, c, o[c], inv);
            }
            if (row == 0) atomicExch(cnt, 0);   // all pieces have arrived: ready for the next launch
        }
    }

    tc_fence_before();
    __syncthreads();
    // the next kernel in the stream may be scheduled once every CTA is here (it waits for this
    // grid's completion itself).  Measured on B200 at 720p: triggered at the start instead, the
    // next grid's CTAs take the SMs in the order this grid's CTAs leave them, and the forward is
    // 2% slower than with a plain launch; triggered here it is 2% faster.
    grid_dependents_launch();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, L::kTmemCols);
    }
    if (threadIdx.x == 0 && ctl->abort_flag) atomicOr(p.status, SW_STATUS_TIMEOUT);
}

template <int D>
static cudaError_t launch_persistent_d(const AttnParams& p, int ctas, cudaStream_t stream) {
    using L = AttnLayout<D, 2>;
    auto kern = p.commit ? attn_persistent_kernel<D, true, false, false> : attn_persistent_kernel<D, false, false, false>;
    if constexpr (D == 128) {
        if (p.qk_fp8) {
            if (p.commit) kern = p.pv_fp8 ? attn_persistent_kernel<D, true, true, true> : attn_persistent_kernel<D, true, true, false>;
            else kern = p.pv_fp8 ? attn_persistent_kernel<D, false, true, true> : attn_persistent_kernel<D, false, true, false>;
        }
    }
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmemBytes);
    if (e != cudaSuccess) return e;
    return launch_dependent(kern, dim3(ctas), dim3(L::kThreads), L::kSmemBytes, stream, p);
}

cudaError_t launch_persistent(const AttnParams& p, int d, int ctas, cudaStream_t stream) {
    if (ctas < 1 || ctas > kMaxPersistentCtas) return cudaErrorInvalidValue;
    if (d == 128) return launch_persistent_d<128>(p, ctas, stream);
    if (d == 64) return launch_persistent_d<64>(p, ctas, stream);
    return cudaErrorInvalidValue;
}

}  // namespace swattn

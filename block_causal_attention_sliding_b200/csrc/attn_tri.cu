// attn_tri.cu -- the full-chunk attention with three S buffers per 128-row Q tile.
//
// Work unit: one 128-row Q tile of one (b, h) against all its visible key tiles (or a slice of
// them, see the schedule).  Tensor memory holds three S accumulators and O:
//     S0 | S1 | S2 | O        (3 x 128 + D <= 512 columns)
// so S of key tile u + 3 is computed while the softmax of tiles u + 1 and u + 2 runs, and the
// softmax never waits on the PV -> next-S round trip of its own tile.  P (bf16 pairs) is
// written over the first 64 columns of its S buffer; the next S into that buffer is issued
// after the PV that reads P, and one thread's MMAs complete in issue order.
//
// Warps: 0 = TMA producer, 1 = tcgen05 MMA issuer, 2..5 = softmax group A, 6..9 = group B,
// 10 = helper that turns TMA completions into words the MMA issuer can poll.
// Key tiles alternate between the groups (global tile counter u: group u & 1), so one group's
// exponentials overlap the other's tensor-memory loads and row maxima, and the two groups
// share the SM's MUFU units.  All tiles of a Q tile accumulate into one O, so the groups keep
// one reference max per row: the group of tile u reads the reference of tile u - 1 from the
// other group (a tagged shared-memory word), raises it lazily (only when the tile's max is
// more than 2^8 above it), publishes it for tile u + 1, and -- when it moved -- rescales O
// after PV(u - 1) has completed and before PV(u) may start.  Each group keeps its own row sum
// relative to the last reference it used; the epilogue brings both to the final reference.
//
// K and V tiles flow through two shared-memory rings (K: 2 stages, V: 3 at d = 128), loaded in
// the order the MMA issuer consumes them: K(0), K(1), K(2), then V(0), K(3), V(1), K(4), ...
// A K stage is refilled once S of its previous tile has completed (s_full), a V stage once PV
// of its previous tile has (o_full): with at most three stages per ring, neither barrier can
// run two phases ahead of the producer, so no separate release commits are needed.
//
// The MMA issuer never waits on an mbarrier: a wait in the thread that issues tcgen05.mma
// stalls the tensor pipe until its queued MMAs and commits have drained.  It polls shared
// words instead (acquire loads), once per key tile, and commits twice per key tile.
//
// Schedule (persistent, one CTA per SM): whole Q tiles round-robin (CTA g takes units g,
// g + G, ...) for the full rounds, so the CTAs running together cover a few heads and their
// K/V stay in L2; the leftover units are laid on one line of (unit, key tile) items cut
// evenly between the CTAs (stream-K).  A unit whose key tiles are cut between CTAs is merged
// by its last-arriving piece, reading all pieces in slot order (deterministic).
#include "tri_common.cuh"

namespace swattn {

namespace tri {

// kQK8: e4m3 Q and K (16 KB tiles, S on kind::f8f6f4); kPV8 (with kQK8): e4m3 V as well, P in
// e4m3 and O += P V on kind::f8f6f4.  Stages are sized by the operand format, so with e4m3 K
// the K ring holds three stages where bf16 at d = 128 fits two.
template <int D, bool kQK8 = false, bool kPV8 = false>
struct Cfg {
    static constexpr int kKBytes = kv_tile_bytes<D, kQK8, kPV8>(0);   // one K stage
    static constexpr int kVBytes = kv_tile_bytes<D, kQK8, kPV8>(1);   // one V stage
    static constexpr int kKSt = (D == 128 && !kQK8) ? 2 : 3;          // K ring stages (at most 3, see above)
    static constexpr int kVSt = 3;                                    // V ring stages (at most 3)
    static constexpr int kQBytes = QKTile<D, kQK8>::kBytes;
    static constexpr int kVOffset = kKSt * kKBytes;                   // V ring after the K ring
    static constexpr int kKVBytes = kVOffset + kVSt * kVBytes;
    static_assert(kKSt <= 3 && kVSt <= 3 && kKSt + kVSt <= 8, "ring stages");
    static constexpr int kCtlOffset = kQBytes + kKVBytes;
    static constexpr int kThreads = 64 + 2 * 128 + 32;   // + the load-completion helper warp
    static constexpr int kTmemCols = 512;
    static constexpr int kOCol = kSBufs * kBlockN;      // O after the three S buffers
    static_assert(kSBufs * kBlockN + D <= kTmemCols, "tensor memory budget");
};

// Barriers and exchange words of the three-buffer pipeline (the K/V ring, Q, the visibility
// table, the TMEM base and the abort flag live in the common SmemCtl).
struct Ext {
    uint64_t s_full[kSBufs];     // S(u) in buffer u % 3 complete                (1 commit)
    uint64_t o_full[kSBufs];     // PV(u) complete, on barrier u % 3              (1 commit)
    uint64_t ep;                 // both groups' row sums are published           (8 warps)
    // Signals the MMA issuer polls with plain acquire loads (an mbarrier wait in the issuing
    // thread stalls the tensor pipe until its queued MMAs and commits have drained):
    uint32_t k_seq;              // K of key tiles 0..u have landed once k_seq >= u + 1 (helper)
    uint32_t v_seq;              // V likewise                                        (helper)
    uint32_t q_seq;              // Q of piece pi has landed once q_seq == pi + 1     (helper)
    // P(u) written (and O ready for PV(u)): +1 per warp of the tile's group, so 4 (u / 3 + 1)
    // once tile u in buffer u % 3 is done
    uint32_t p_cnt[kSBufs];
    uint32_t oe_cnt;             // +1 per softmax warp once the piece's O has been read
    // reference max of tile u for tile u + 1: (tag u + 1) << 32 | float bits, slot u & 1
    unsigned long long ref[2][kBlockM];
    float lsum[2][2][kBlockM];   // [piece parity][group][row] row sums at the final reference
};

template <int D, bool kQK8 = false, bool kPV8 = false>
constexpr int smem_bytes() {
    // at least 120 KB: one CTA per SM, so no CTA waits on another's tensor memory
    constexpr int need = ((Cfg<D, kQK8, kPV8>::kCtlOffset + (int)sizeof(SmemCtl) + 15) & ~15) + (int)sizeof(Ext) + 1024;
    return need > 120 * 1024 ? need : 120 * 1024;
}

}  // namespace tri


template <int D, bool kQK8, bool kPV8>
__global__ void __launch_bounds__(tri::Cfg<D>::kThreads, 1)
attn_tri_kernel(const __grid_constant__ AttnParams p) {
    using C = tri::Cfg<D, kQK8, kPV8>;
    using QT = QKTile<D, kQK8>;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* q_smem = base;
    uint8_t* kv_smem = base + C::kQBytes;
    SmemCtl* ctl = reinterpret_cast<SmemCtl*>(base + C::kCtlOffset);
    tri::Ext* ex = reinterpret_cast<tri::Ext*>(base + ((C::kCtlOffset + (int)sizeof(SmemCtl) + 15) & ~15));
    volatile int* abort_flag = &ctl->abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    for (int i = threadIdx.x; i < 2 * kBlockM; i += blockDim.x) (&ex->ref[0][0])[i] = 0ull;   // tags start at 1
    if (threadIdx.x == 64) {
        for (int b = 0; b < tri::kSBufs; ++b) ex->p_cnt[b] = 0;
        ex->k_seq = ex->v_seq = ex->q_seq = 0;
        ex->oe_cnt = 0;
    }
    if (warp == 0) {
        if (lane == 0) {
            for (int b = 0; b < tri::kSBufs; ++b) {
                mbar_init(smem_u32(&ex->s_full[b]), 1);
                mbar_init(smem_u32(&ex->o_full[b]), 1);
            }
            mbar_init(smem_u32(&ex->ep), 8);
            init_barriers(ctl, C::kKSt + C::kVSt);   // Q, the K/V rings, drain; fences every init above
        }
        __syncwarp();
        tmem_alloc(smem_u32(&ctl->tmem_base), C::kTmemCols);
        tmem_relinquish();
    } else if (warp == 2 && lane == 0) {
        load_table(ctl, p.table, p.status);
    } else if (warp == 1 && lane == 0) {
        tma_prefetch_desc(&p.tm_q);
        tma_prefetch_desc(&p.tm_qc);
        tma_prefetch_desc(&p.tm_kcur);
        tma_prefetch_desc(&p.tm_vcur);
        tma_prefetch_desc(&p.tm_cache_k);
        tma_prefetch_desc(&p.tm_cache_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem = ctl->tmem_base;
    const int nt = ctl->n_tiles;
    const int nqt = q_tiles(p);
    tri::Sched sched;
    sched.init(nqt, nt, p.B * p.H, (int)gridDim.x, blockIdx.x);

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0 && nt > 0) {
            const uint32_t qbar = smem_u32(&ctl->q_full);
            tri::PieceIt pit;
            tri::Piece pc;
            uint32_t t = 0;    // key tiles of all pieces so far (global tile index base)
            int pi = 0;
            bool ok = true;
            while (ok && tri::next_piece(sched, pit, pc)) {
                const int bh = pc.unit / nqt, qtile = pc.unit % nqt;
                const int b = bh / p.H, h = bh % p.H;
                // the Q buffer is reused: every S MMA of the previous piece has completed
                if (pi > 0 && !wait_or_abort(smem_u32(&ctl->q_empty), (pi - 1) & 1, abort_flag)) break;
                mbar_arrive_expect_tx(qbar, QT::kBytes);
                const QSrc qs = q_src(p, qtile);
                for (int c = 0; c < QT::kBoxes; ++c)
                    tma_load_4d(smem_u32(q_smem + c * kBoxBytes), qs.tm, qbar, c * QT::kBoxCols, h, qs.row0, b);
                ++pi;
                const int n = pc.j1 - pc.j0;
                // K(u): its stage last held K(u - kKSt), free once S(u - kKSt) has completed
                auto load_k = [&](int jrel) -> bool {
                    const uint32_t u = t + jrel;
                    if (u >= (uint32_t)C::kKSt) {
                        const uint32_t v = u - C::kKSt;
                        if (!wait_or_abort(smem_u32(&ex->s_full[v % tri::kSBufs]), (v / tri::kSBufs) & 1, abort_flag))
                            return false;
                    }
                    const int st = u % C::kKSt;
                    const uint32_t fbar = smem_u32(&ctl->kv_full[st]);
                    mbar_arrive_expect_tx(fbar, C::kKBytes);
                    load_kv_tile<D, kQK8, kPV8>(p, ctl, pc.j0 + jrel, 0, h, b, smem_u32(kv_smem + st * C::kKBytes), fbar);
                    return true;
                };
                // V(u): its stage last held V(u - kVSt), free once PV(u - kVSt) has completed
                auto load_v = [&](int jrel) -> bool {
                    const uint32_t u = t + jrel;
                    if (u >= (uint32_t)C::kVSt) {
                        const uint32_t v = u - C::kVSt;
                        if (!wait_or_abort(smem_u32(&ex->o_full[v % tri::kSBufs]), (v / tri::kSBufs) & 1, abort_flag))
                            return false;
                    }
                    const int vs = (int)(u % C::kVSt);
                    const uint32_t fbar = smem_u32(&ctl->kv_full[C::kKSt + vs]);
                    mbar_arrive_expect_tx(fbar, C::kVBytes);
                    load_kv_tile<D, kQK8, kPV8>(p, ctl, pc.j0 + jrel, 1, h, b,
                                                smem_u32(kv_smem + C::kVOffset + vs * C::kVBytes), fbar);
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
            // never leave while copies are in flight: the last fill of every stage has landed
            for (int st = 0; st < C::kKSt; ++st)
                if (t > (uint32_t)st) wait_drain(smem_u32(&ctl->kv_full[st]), (((t - 1 - st) / C::kKSt) & 1));
            for (int st = 0; st < C::kVSt; ++st)
                if (t > (uint32_t)st)
                    wait_drain(smem_u32(&ctl->kv_full[C::kKSt + st]), (((t - 1 - st) / C::kVSt) & 1));
            if (pi > 0) wait_drain(qbar, (pi - 1) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // Per key tile u: one poll point (V(u), P(u), K(u + 3)), PV(u), commit o_full, S(u + 3)
        // into the same buffer, commit s_full.
        if (lane == 0 && nt > 0) {
            const uint32_t q_base = smem_u32(q_smem);
            const uint32_t kv_base = smem_u32(kv_smem);
            const uint32_t tO = tmem + C::kOCol;
            tri::PieceIt pit;
            tri::Piece pc;
            uint32_t t = 0;    // key tiles of all pieces so far (S buffer u % 3, phase u / 3)
            int pi = 0;        // pieces done
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
                    issue_s_qk<D, kQK8>(tmem + (u % tri::kSBufs) * kBlockN, q_base, kv_base + (u % C::kKSt) * C::kKBytes);
                    mma_commit(smem_u32(&ex->s_full[u % tri::kSBufs]));
                    if (k == n - 1) mma_commit(smem_u32(&ctl->q_empty));   // last S of the piece
                }
                for (int jj = 0; jj < n && ok; ++jj) {
                    const uint32_t u = t + jj, bu = u % tri::kSBufs;
                    const bool more = jj + 3 < n;
                    if (!tri::poll_reach(&ex->v_seq, u + 1, abort_flag) ||
                        !tri::poll_reach(&ex->p_cnt[bu], 4 * (u / tri::kSBufs + 1), abort_flag) ||
                        (more && !tri::poll_reach(&ex->k_seq, u + 4, abort_flag)) ||
                        // the previous piece's O must be out of TMEM before PV(u) overwrites it
                        (jj == 0 && pi > 0 && !tri::poll_reach(&ex->oe_cnt, 8 * pi, abort_flag))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t tP = tmem + bu * kBlockN;
                    const uint32_t v_tile = kv_base + C::kVOffset + (u % C::kVSt) * C::kVBytes;
                    if constexpr (kPV8) {
                        issue_pv_f8_half(tO, tP, v_tile, 0, jj > 0);
                        issue_pv_f8_half(tO, tP, v_tile, 1, true);
                    } else {
                        issue_pv<D>(tO, tP, v_tile, jj > 0);
                    }
                    mma_commit(smem_u32(&ex->o_full[bu]));   // PV(u) done: V stage, rescale, epilogue
                    if (more) {
                        // S(u + 3) into the same buffer, in issue order after PV(u) read P(u)
                        issue_s_qk<D, kQK8>(tP, q_base, kv_base + ((u + 3) % C::kKSt) * C::kKBytes);
                        mma_commit(smem_u32(&ex->s_full[bu]));
                        if (jj + 3 == n - 1) mma_commit(smem_u32(&ctl->q_empty));
                    }
                }
                ++pi;
                t += n;
            }
            // every MMA issued has completed before the CTA can release TMEM
            mma_commit(smem_u32(&ctl->drain));
            wait_drain(smem_u32(&ctl->drain), 0);
        }
    } else if (warp == 10) {
        // ------------------------------------------------------------ completion helper
        // Follows the producer's sequence: Q of each piece, then K and V of every key tile in
        // consumption order; publishes each completion as a word the MMA issuer polls.  Never
        // more than one phase behind a barrier: a stage is refilled only after the MMA issuer
        // has seen the word for its previous fill.
        if (lane == 0 && nt > 0) {
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
                    if (!wait_or_abort(smem_u32(&ctl->kv_full[u % C::kKSt]), (u / C::kKSt) & 1, abort_flag)) return false;
                    tri::st_release(&ex->k_seq, u + 1);
                    return true;
                };
                auto done_v = [&](int jrel) -> bool {
                    const uint32_t u = t + jrel;
                    if (!wait_or_abort(smem_u32(&ctl->kv_full[C::kKSt + u % C::kVSt]), (u / C::kVSt) & 1, abort_flag))
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
    } else {
        // ------------------------------------------------------------ softmax groups
        const int sw = warp - 2;          // 0..7
        const int g = sw >> 2;            // group: key tiles u with u & 1 == g
        const int wq = warp & 3;          // TMEM lane quarter (fixed by the warp's slot)
        const int row = wq * 32 + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(wq * 32) << 16);
        const uint32_t tO = lane_base + C::kOCol;
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
            for (int jj = (int)((g + t) & 1); jj < n; jj += 2) {
                const uint32_t u = t + jj, bu = u % tri::kSBufs;
                int seg, row0, valid;
                tile_of(ctl, pc.j0 + jj, seg, row0, valid);
                ok = warp_wait(smem_u32(&ex->s_full[bu]), (u / tri::kSBufs) & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t up = u - 1;   // unused when jj == 0
                ok = tri::softmax_tile<D, kPV8>(lane_base + bu * kBlockN, tO, valid, jj == 0, u, &ex->ref[up & 1][row],
                                          &ex->ref[u & 1][row], smem_u32(&ex->o_full[up % tri::kSBufs]),
                                          (up / tri::kSBufs) & 1, smem_u32(&ex->p_cnt[bu]), p.scale_log2, m_g,
                                          l_g, has_g, abort_flag);
                if (!ok) break;
            }
            // ---------------------------------------------------- epilogue of this piece
            const uint32_t tl = t + n - 1;   // the piece's last key tile
            const int par = ucnt & 1;
            float m_fin = m_g;
            if (ok && (int)(tl & 1) != g) ok = tri::ref_get(&ex->ref[tl & 1][row], tl + 1, m_fin, abort_flag);
            float l_row = 0.f;
            if (ok) {
                ex->lsum[par][g][row] = has_g ? l_g * ex2_approx(m_g - m_fin) : 0.f;
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
            for (int c = 0; c < D / 64; ++c) tmem_ld32(tO + g * (D / 2) + c * 32, o[c]);
            tmem_wait_ld_dep(o[0]);
#pragma unroll
            for (int c = 1; c < D / 64; ++c) reg_fence(o[c]);
            tc_fence_before();
            tri::warp_signal(smem_u32(&ex->oe_cnt));   // O may now be overwritten

            const int bh = pc.unit / nqt, qtile = pc.unit % nqt;
            const int b = bh / p.H, h = bh % p.H;
            const QSrc qs = q_src(p, qtile);
            const int m_row = qs.row0 + row;
            const size_t orow = ((size_t)b * qs.rows + m_row) * p.H + h;
            if (pc.j0 == 0 && pc.j1 == nt) {
                const float inv = (kPV8 ? p.out_scale : 1.f) / l_row;   // e4m3 V: its scale, once
                if (m_row < qs.rows) {
#pragma unroll
                    for (int c = 0; c < D / 64; ++c)
                        store_row_chunk<D>(qs.out, p.out_f32, orow, g * (D / 64) + c, o[c], inv);
                }
                continue;
            }
            // split piece: publish the partial, then the last of the unit's pieces merges
            const long long ps = sched.cstart(pc.unit);
            const int g_first = sched.cta_of(ps);
            const int g_last = sched.cta_of(ps + nt - 1);
            const int npieces = g_last - g_first + 1;
            const int cta = blockIdx.x;
            const int slot = first_sk ? 2 * cta : 2 * cta + 1;
            float* so = p.sk_o + (size_t)slot * 2 * D * kBlockM;       // [D][128 rows]
            float* sml = p.sk_ml + (size_t)slot * 2 * kBlockM * 2;     // [128 rows][2]
#pragma unroll
            for (int c = 0; c < D / 64; ++c)
#pragma unroll
                for (int i = 0; i < 32; ++i) so[(g * (D / 2) + c * 32 + i) * kBlockM + row] = __uint_as_float(o[c][i]);
            if (g == 0) {
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
            // the unit's first piece is CTA g_first's first stream-K piece iff g_first's range
            // opens inside this unit; every later CTA's piece of it opens that CTA's range
            tri::Sched sf = sched;
            sf.set_range(g_first);
            const bool opens_first = sf.u0 + (int)(sf.c0 / nt) == pc.unit;
            float M = -INFINITY;
            for (int gg = g_first; gg <= g_last; ++gg) {
                const int sl = gg == cta ? slot : ((gg > g_first || opens_first) ? 2 * gg : 2 * gg + 1);
                M = fmaxf(M, __ldcg(p.sk_ml + (size_t)sl * 2 * kBlockM * 2 + row * 2));
            }
            float L_ = 0.f;
            for (int gg = g_first; gg <= g_last; ++gg) {
                const int sl = gg == cta ? slot : ((gg > g_first || opens_first) ? 2 * gg : 2 * gg + 1);
                const float* pml = p.sk_ml + (size_t)sl * 2 * kBlockM * 2 + row * 2;
                L_ += ex2_approx(__ldcg(pml) - M) * __ldcg(pml + 1);
            }
            const float inv = (kPV8 ? p.out_scale : 1.f) / L_;
#pragma unroll 1
            for (int c = 0; c < D / 64; ++c) {      // 32 columns at a time
                uint32_t acc[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) acc[i] = 0u;
                for (int gg = g_first; gg <= g_last; ++gg) {
                    const int sl = gg == cta ? slot : ((gg > g_first || opens_first) ? 2 * gg : 2 * gg + 1);
                    const float w = ex2_approx(__ldcg(p.sk_ml + (size_t)sl * 2 * kBlockM * 2 + row * 2) - M);
                    const float* po = p.sk_o + (size_t)sl * 2 * D * kBlockM + (g * (D / 2) + c * 32) * kBlockM + row;
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        acc[i] = __float_as_uint(fmaf(w, __ldcg(po + i * kBlockM), __uint_as_float(acc[i])));
                }
                if (m_row < qs.rows) store_row_chunk<D>(qs.out, p.out_f32, orow, g * (D / 64) + c, acc, inv);
            }
            if (sw == 0 && lane == 0) atomicExch(cnt, 0);   // all pieces arrived: ready for the next launch
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
    if (threadIdx.x == 0 && ctl->abort_flag) atomicOr(p.status, SW_STATUS_TIMEOUT);
}

template <int D, bool kQK8, bool kPV8>
static cudaError_t launch_tri_d(const AttnParams& p, int ctas, cudaStream_t stream) {
    constexpr int smem = tri::smem_bytes<D, kQK8, kPV8>();
    static_assert(smem <= 227 * 1024, "shared memory budget");
    auto kern = attn_tri_kernel<D, kQK8, kPV8>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<ctas, tri::Cfg<D, kQK8, kPV8>::kThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_tri(const AttnParams& p, int d, int ctas, cudaStream_t stream) {
    if (ctas < 1 || ctas > kMaxPersistentCtas) return cudaErrorInvalidValue;
    if (d == 128) {
        if (p.qk_fp8) return p.pv_fp8 ? launch_tri_d<128, true, true>(p, ctas, stream)
                                      : launch_tri_d<128, true, false>(p, ctas, stream);
        return launch_tri_d<128, false, false>(p, ctas, stream);
    }
    if (d == 64 && !p.qk_fp8) return launch_tri_d<64, false, false>(p, ctas, stream);
    return cudaErrorInvalidValue;
}

}  // namespace swattn

// attn_kernel.cu -- fused attention of the active chunk over the bounded cache (sm_100a): the
// one-work-item-per-CTA kernel (grid over query-tile pairs, heads and streams).
//
// out = softmax(scale * Q K^T) V over the keys the visibility table lists: condition tokens,
// the sink, the window chunks and the current chunk (block-causal: bidirectional inside the
// chunk, causal across chunks -- agifrontier tutorial "JoyAI-Video-Edit：单卡720p 30帧，两步
// 蒸馏攻克流式视频编辑", section "从双向编辑到分块因果架构的蜕变").
//
// Design (one CTA = NQ query tiles of 128 rows of one (b, h); keys in tiles of 128):
//   warp 0      TMA producer: Q once, then K and V tiles of every visible segment, straight
//               from their own locations (condition region, ring slots, the caller's K_cur
//               and V_cur) through per-segment tensor maps; rows past a segment's end are
//               zero-filled by TMA.  A ring of kStages shared-memory tiles.
//   warp 1      MMA issuer (one thread): S_q = Q_q K^T into TMEM (tcgen05, bf16 in, fp32
//               accumulate), then O_q += P_q V with P read from TMEM.
//   warps 2..   one warpgroup per Q tile (thread = query row = TMEM lane): online softmax in
//               fp32 registers -- row max, lazy rescale of O only when the max grows by more
//               than 2^8, exp2, row sum -- writes P as bf16 into the S columns.
// The two Q tiles share every K/V tile, and while one warpgroup runs its softmax the tensor
// core works on the other tile.
#include "attn_common.cuh"

namespace swattn {

template <int D, int NQ>
__global__ void __launch_bounds__(AttnLayout<D, NQ>::kThreads, 1)
attn_fwd_kernel(const __grid_constant__ AttnParams p) {
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
    const int h = blockIdx.y;
    const int b = blockIdx.z;

    // ---------------------------------------------------------------- set-up
    if (warp == 0) {
        if (lane == 0) init_barriers(ctl, kStages);
        __syncwarp();
        tmem_alloc(smem_u32(&ctl->tmem_base), L::kTmemCols);
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
    const int n = ctl->n_tiles;                     // key tiles: every visible one
    const int u0 = blockIdx.x * NQ;                 // first Q tile of this CTA
    // Q tiles of this CTA that hold at least one query row (the last CTA of a head may own
    // a single tile); tiles past n_q are neither loaded nor computed
    const int live = min(NQ, q_tiles(p) - u0);

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0 && n > 0) {
            const uint32_t qbar = smem_u32(&ctl->q_full);
            mbar_arrive_expect_tx(qbar, live * kTileBytes);
            for (int qt = 0; qt < live; ++qt) {
                const QSrc qs = q_src(p, u0 + qt);
                for (int c = 0; c < C::kBoxes; ++c)
                    tma_load_4d(smem_u32(q_smem + qt * kTileBytes + c * kBoxBytes), qs.tm, qbar,
                                c * kBoxCols, h, qs.row0, b);
            }
            uint32_t it = 0;
            bool ok = true;
            // fused commit: the chunk's K_cur / V_cur tile j is stored by the CTA of Q-tile pair
            // j mod (pairs), so the stores spread over the CTAs of each head
            const int cslot = p.commit ? ring_slot(__ldg(p.table), p.ring_R, p.sink) : -1;
            CommitQueue<D, kStages> cq;
            for (int j = 0; j < n && ok; ++j) {
                for (int kv = 0; kv < 2; ++kv, ++it) {
                    const int s = it % kStages;
                    const uint32_t r = it / kStages;
                    if (!wait_or_abort(smem_u32(&ctl->kv_empty[s]), (r & 1) ^ 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    cq.before_refill(s);
                    const uint32_t fbar = smem_u32(&ctl->kv_full[s]);
                    mbar_arrive_expect_tx(fbar, kTileBytes);
                    load_kv_tile<D>(p, ctl, j, kv, h, b, smem_u32(kv_smem + s * kTileBytes), fbar);
                    if (cslot >= 0) {
                        const bool mine = (int)blockIdx.x == j % (int)gridDim.x && ctl->seg_kind[tile_seg(ctl, j)] == 2;
                        if (!cq.step(p, ctl, kv_smem, cslot, it, CommitQueue<D, kStages>::pack(mine, j, kv, h, b),
                                     abort_flag)) {
                            ok = false;
                            break;
                        }
                    }
                }
            }
            if (cslot >= 0) {
                if (ok) (void)cq.flush(p, ctl, kv_smem, cslot, it, abort_flag);
                bulk_wait_all();
            }
            // never leave while copies are in flight: the last fill of every stage has landed
            for (int s = 0; s < kStages; ++s) {
                if (it > (uint32_t)s) {
                    const uint32_t uses = (it - 1 - s) / kStages + 1;
                    wait_drain(smem_u32(&ctl->kv_full[s]), (uses - 1) & 1);
                }
            }
            wait_drain(qbar, 0);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && n > 0) {
            const uint32_t q_base = smem_u32(q_smem);
            const uint32_t kv_base = smem_u32(kv_smem);
            bool ok = wait_or_abort(smem_u32(&ctl->q_full), 0, abort_flag);
            if (ok) ok = wait_or_abort(smem_u32(&ctl->kv_full[0]), 0, abort_flag);
            if (ok) {
                tc_fence_after();
                for (int qt = 0; qt < live; ++qt) {
                    issue_s<D>(tmem + qt * kBlockN, q_base + qt * kTileBytes, kv_base);
                    mma_commit(smem_u32(&ctl->s_full[qt]));
                }
                mma_commit(smem_u32(&ctl->kv_empty[0]));
            }
            if (kDynamicMma) {
                // One small state machine per Q tile, polled without blocking: PV of the first
                // half of P (needs V_j and p_half), PV of the second half (p_full), then S of the
                // next tile (needs K_j+1).  Whichever tile is ready is served, so one softmax
                // warpgroup never waits behind the other.  Per tile the issue order is unchanged
                // (PV_j before S_j+1 over the same columns).  A K or V stage is released once
                // every live tile has issued the MMAs that read it.
                int jq[2] = {0, 0}, ph[2] = {0, 0};
                // per tile j mod 4: how many Q tiles have issued the MMAs reading V_j / K_j,
                // as 2-bit fields of one register each (no local memory)
                uint32_t cntV = 0, cntK = 0;
                int remaining = ok ? live : 0;
                uint32_t idle = 0;
                uint64_t t_idle = 0;
                while (remaining > 0) {
                    bool prog = false;
#pragma unroll
                    for (int qt = 0; qt < NQ; ++qt) {
                        if (qt >= live || jq[qt] >= n) continue;
                        const int j = jq[qt];
                        const uint32_t itV = 2 * j + 1, itK = 2 * j + 2;
                        const int sV = itV % kStages, sK = itK % kStages;
                        const uint32_t tO = tmem + NQ * kBlockN + qt * D, tP = tmem + qt * kBlockN;
                        if (ph[qt] == 0 && mbar_test(smem_u32(&ctl->kv_full[sV]), (itV / kStages) & 1) &&
                            mbar_test(smem_u32(&ctl->p_half[qt]), j & 1)) {
                            tc_fence_after();
                            issue_pv_half<D>(tO, tP, kv_base + sV * kTileBytes, 0, j > 0);
                            ph[qt] = 1;
                            prog = true;
                        }
                        if (ph[qt] == 1 && mbar_test(smem_u32(&ctl->p_full[qt]), j & 1)) {
                            tc_fence_after();
                            issue_pv_half<D>(tO, tP, kv_base + sV * kTileBytes, 1, true);
                            if (j + 1 == n) mma_commit(smem_u32(&ctl->o_full[qt]));   // O complete: epilogue
                            const int shV = 2 * (j & 3);
                            cntV += 1u << shV;
                            if ((int)((cntV >> shV) & 3u) == live) {
                                mma_commit(smem_u32(&ctl->kv_empty[sV]));
                                cntV &= ~(3u << shV);
                            }
                            if (j + 1 < n) {
                                ph[qt] = 2;
                            } else {
                                jq[qt] = n;
                                --remaining;
                            }
                            prog = true;
                        }
                        if (ph[qt] == 2 && mbar_test(smem_u32(&ctl->kv_full[sK]), (itK / kStages) & 1)) {
                            tc_fence_after();
                            issue_s<D>(tmem + qt * kBlockN, q_base + qt * kTileBytes, kv_base + sK * kTileBytes);
                            mma_commit(smem_u32(&ctl->s_full[qt]));
                            const int shK = 2 * ((j + 1) & 3);
                            cntK += 1u << shK;
                            if ((int)((cntK >> shK) & 3u) == live) {
                                mma_commit(smem_u32(&ctl->kv_empty[sK]));
                                cntK &= ~(3u << shK);
                            }
                            jq[qt] = j + 1;
                            ph[qt] = 0;
                            prog = true;
                        }
                    }
                    if (prog) {
                        idle = 0;
                        continue;
                    }
                    // nothing ready: back off briefly, and give up after the wait limit
                    if (*abort_flag) break;
                    if (idle++ == 0) t_idle = globaltimer_ns();
                    else if ((idle & 255) == 0 && globaltimer_ns() - t_idle > kWaitLimitNs) {
                        *abort_flag = 1;
                        break;
                    }
                    __nanosleep(20);
                }
            } else {
                for (int jj = 0; jj < n && ok; ++jj) {
                    const uint32_t itV = 2 * jj + 1, itK = 2 * jj + 2;
                    const int sV = itV % kStages, sK = itK % kStages;
                    const bool more = jj + 1 < n;
                    if (!wait_or_abort(smem_u32(&ctl->kv_full[sV]), (itV / kStages) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    for (int qt = 0; qt < live && ok; ++qt) {
                        // P arrives in two halves; the PV of the first 64 keys overlaps the softmax
                        // of the other 64
                        const uint32_t tO = tmem + NQ * kBlockN + qt * D, tP = tmem + qt * kBlockN;
                        if (kSplitP) {
                            if (!wait_or_abort(smem_u32(&ctl->p_half[qt]), jj & 1, abort_flag)) { ok = false; break; }
                            tc_fence_after();
                            issue_pv_half<D>(tO, tP, kv_base + sV * kTileBytes, 0, jj > 0);
                        }
                        if (!wait_or_abort(smem_u32(&ctl->p_full[qt]), jj & 1, abort_flag)) { ok = false; break; }
                        tc_fence_after();
                        if (kSplitP) issue_pv_half<D>(tO, tP, kv_base + sV * kTileBytes, 1, true);
                        else issue_pv<D>(tO, tP, kv_base + sV * kTileBytes, jj > 0);
                        if (!more) mma_commit(smem_u32(&ctl->o_full[qt]));   // O complete: epilogue
                        if (more) {
                            if (qt == 0 &&
                                !wait_or_abort(smem_u32(&ctl->kv_full[sK]), (itK / kStages) & 1, abort_flag)) {
                                ok = false;
                                break;
                            }
                            // P_q lives in the S_q columns.  MMAs issued by this thread run in
                            // issue order on the tensor pipe, so the PV above reads P_q before
                            // this S_q overwrites it.
                            issue_s<D>(tmem + qt * kBlockN, q_base + qt * kTileBytes, kv_base + sK * kTileBytes);
                            mma_commit(smem_u32(&ctl->s_full[qt]));
                        }
                    }
                    if (!ok) break;
                    mma_commit(smem_u32(&ctl->kv_empty[sV]));
                    if (more) mma_commit(smem_u32(&ctl->kv_empty[sK]));
                }
            }
            // every MMA issued has completed before the CTA can release TMEM
            mma_commit(smem_u32(&ctl->drain));
            wait_drain(smem_u32(&ctl->drain), 0);
        }
    } else if (warp >= 2 && ((warp - 2) >> 2) < live) {
        // ------------------------------------------------------------ softmax warpgroups
        // warps 2..5 own Q tile 0 and warps 6..9 Q tile 1; a warp may only touch the TMEM lane
        // quarter warp % 4, and each group of four consecutive warps covers all four quarters
        const int qt = (warp - 2) >> 2;
        const int wq = warp & 3;
        const int row = wq * 32 + lane;                // query row inside the tile
        const uint32_t lane_base = tmem + ((uint32_t)(wq * 32) << 16);
        const uint32_t tS = lane_base + qt * kBlockN;
        const uint32_t tO = lane_base + NQ * kBlockN + qt * D;
        const uint32_t o_bar = smem_u32(&ctl->o_full[qt]);
        float m_ref = -INFINITY;   // reference max, log2-scaled
        float l = 0.f;             // row sum of the bf16-rounded exp2(s*sl2 - m_ref)
        bool ok = true;
        for (int jj = 0; jj < n; ++jj) {
            int seg, row0, valid;
            tile_of(ctl, jj, seg, row0, valid);
            ok = warp_wait(smem_u32(&ctl->s_full[qt]), jj & 1, abort_flag);
            if (!ok) break;
            tc_fence_after();
            softmax_step<D>(tS, tO, valid, jj == 0, smem_u32(&ctl->p_half[qt]), p.scale_log2, m_ref, l);
            warp_arrive(smem_u32(&ctl->p_full[qt]));
        }
        // ------------------------------------------------------------ epilogue
        const QSrc qs = q_src(p, u0 + qt);
        const int m_row = qs.row0 + row;
        if (n > 0 && ok && warp_wait(o_bar, 0, abort_flag)) {   // o_full completes once, after the last PV
            tc_fence_after();
            const float inv = 1.f / l;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(tO + c * 32, o);
                tmem_wait_ld_dep(o);
                if (m_row < qs.rows)
                    store_row_chunk<D>(qs.out, p.out_f32, ((size_t)b * qs.rows + m_row) * p.H + h, c, o, inv);
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, L::kTmemCols);
    }
    if (threadIdx.x == 0 && ctl->abort_flag) atomicOr(p.status, SW_STATUS_TIMEOUT);
}

template <int D>
static cudaError_t launch_one(const AttnParams& p, int grid_x, cudaStream_t stream) {
    using L = AttnLayout<D, 2>;
    auto kern = attn_fwd_kernel<D, 2>;
    // per device and cheap; set on every launch so any current device is covered
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         L::kSmemBytes);
    if (e != cudaSuccess) return e;
    dim3 grid(grid_x, p.H, p.B);
    kern<<<grid, L::kThreads, L::kSmemBytes, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_attention(const AttnParams& p, int d, int grid_x, cudaStream_t stream) {
    if (d == 128) return launch_one<128>(p, grid_x, stream);
    if (d == 64) return launch_one<64>(p, grid_x, stream);
    return cudaErrorInvalidValue;
}

// ------------------------------------------------------------------ failure-detection self-test
// Waits on a barrier that nothing completes, with the kernels' own bounded wait; records the
// timeout in the status word like a stalled attention kernel would.
__global__ void selftest_timeout_kernel(int32_t* status, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        fence_mbar_init();
        flag = 0;
    }
    __syncthreads();
    if (threadIdx.x == 0 && !mbar_wait(smem_u32(&bar), 0, &flag, limit_ns)) atomicOr(status, SW_STATUS_TIMEOUT);
}

cudaError_t launch_selftest_timeout(int32_t* status, uint64_t limit_ns, cudaStream_t stream) {
    selftest_timeout_kernel<<<1, 32, 0, stream>>>(status, limit_ns);
    return cudaGetLastError();
}

}  // namespace swattn

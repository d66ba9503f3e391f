// attn_split.cu -- split-K attention for short query sets (n_q <= 128 queries of the active
// chunk over the whole visible key set), sm_100a.
//
// The same result as the chunk forward -- softmax(scale * Q K^T) V over the keys the
// visibility table lists (condition tokens, sink, window chunks, current chunk; agifrontier
// tutorial "JoyAI-Video-Edit：单卡720p 30帧，两步蒸馏攻克流式视频编辑", section
// "从双向编辑到分块因果架构的蜕变") -- for a query set too small to fill the GPU with query
// tiles.  The key tiles of each (b, h) are dealt round-robin to `splits` slices, one CTA per
// slice; each CTA writes the unnormalised partial (O, m, l) of its slice and the combine kernel
// (below; a programmatic dependent launch) merges the slices with a log-sum-exp weighting.
//
// One CTA = one 128-row Q tile (rows past n_q are TMA zero-fill) and one slice of key tiles:
//   warp 0      TMA producer: Q once, then K and V tiles of the slice through a ring of kStages
//               shared-memory stages (deeper than the chunk kernels': the slice is read from
//               HBM once and nothing else hides its latency).
//   warp 1      MMA issuer (one thread).  S is double-buffered in TMEM: S_{j+1} = Q K_{j+1}^T is
//               issued as soon as K_{j+1} lands, before the PV of tile j, so the tensor core
//               computes the next scores while the softmax warps work on this tile.  O += P_j V_j
//               follows P_j in two halves.
//   warps 2..5  softmax, thread = query row = TMEM lane.  Only warps whose 32 rows hold a query
//               take part; the others idle until the teardown.
// TMEM: S0 | S1 | O (128 + 128 + d columns of 512).  An O rescale (rare: the reference max grew
// by more than 2^8) first waits for the previous tile's PV, which may still be in flight.
//
// The split-K pattern itself (partials plus a log-sum-exp merge) is the standard way to spread
// a short query set over all SMs; the pages have no decode step of their own.
#include "attn_common.cuh"

namespace swattn {

struct SplitCtl {
    SmemCtl c;           // stage barriers, table copy, S/P/O barriers (index = S buffer)
    uint64_t pv_done;    // one phase per key tile: O += P_j V_j has completed
};

template <int D>
struct SplitLayout {
    using C = TileCfg<D>;
    static constexpr int kStages = D == 128 ? 6 : 8;   // 192 KB / 128 KB of K/V stages
    static constexpr int kTileBytes = C::kTileBytes;
    static constexpr int kQBytes = kTileBytes;
    static constexpr int kCtlOffset = kQBytes + kStages * kTileBytes;
    static constexpr int kNeed = kCtlOffset + (int)sizeof(SplitCtl) + 1024;   // + align slack
    // at least 120 KB, so that one CTA fills an SM and never waits on another's TMEM columns
    static constexpr int kSmemBytes = kNeed > 120 * 1024 ? kNeed : 120 * 1024;
    static constexpr int kThreads = 192;
    static constexpr int kTmemCols = 512;
    static constexpr int kColO = 2 * kBlockN;
    static_assert(kColO + D <= kTmemCols, "S0 | S1 | O must fit");
    static_assert(kStages <= 8, "stage barriers");
    static_assert(kNeed <= 227 * 1024, "shared memory");
};

// Half of O += P V: bf16 P and V on kind::f16, or e4m3 on kind::f8f6f4.
template <int D, bool kPV8>
__device__ __forceinline__ void split_pv_half(uint32_t tO, uint32_t tP, uint32_t v_tile, int half, bool accumulate) {
    if constexpr (kPV8) issue_pv_f8_half(tO, tP, v_tile, half, accumulate);
    else issue_pv_half<D>(tO, tP, v_tile, half, accumulate);
}

// kQK8: e4m3 Q and K (S on kind::f8f6f4); kPV8 (with kQK8): e4m3 V and P too (O += P V on
// kind::f8f6f4), the partials then carry the V scale, which the combine applies.
template <int D, bool kQK8, bool kPV8>
__global__ void __launch_bounds__(SplitLayout<D>::kThreads, 1)
attn_split_kernel(const __grid_constant__ AttnParams p) {
    using L = SplitLayout<D>;
    constexpr int kStages = L::kStages;
    constexpr int kTileBytes = L::kTileBytes;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* q_smem = base;
    uint8_t* kv_smem = base + L::kQBytes;
    SplitCtl* x = reinterpret_cast<SplitCtl*>(base + L::kCtlOffset);
    SmemCtl* ctl = &x->c;
    volatile int* abort_flag = &ctl->abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int h = blockIdx.y;
    const int b = blockIdx.z;
    const int bh = b * p.H + h;
    const int n_rows = p.n_q < kBlockM ? p.n_q : kBlockM;   // query rows of the tile
    const int n_warps = (n_rows + 31) >> 5;                  // softmax warps with a query row

    // ---------------------------------------------------------------- set-up
    if (warp == 0) {
        if (lane == 0) {
            mbar_init(smem_u32(&ctl->q_full), 1);
            for (int s = 0; s < kStages; ++s) {
                mbar_init(smem_u32(&ctl->kv_full[s]), 1);
                mbar_init(smem_u32(&ctl->kv_empty[s]), 1);
            }
            for (int q = 0; q < 2; ++q) {
                mbar_init(smem_u32(&ctl->s_full[q]), 1);
                mbar_init(smem_u32(&ctl->p_half[q]), n_warps);
                mbar_init(smem_u32(&ctl->p_full[q]), n_warps);
            }
            mbar_init(smem_u32(&ctl->o_full[0]), 1);
            mbar_init(smem_u32(&x->pv_done), 1);
            mbar_init(smem_u32(&ctl->drain), 1);
            ctl->abort_flag = 0;
            fence_mbar_init();
        }
        __syncwarp();
        tmem_alloc(smem_u32(&ctl->tmem_base), L::kTmemCols);
        tmem_relinquish();
    } else if (warp == 1 && lane == 0) {
        tma_prefetch_desc(&p.tm_q);
        tma_prefetch_desc(&p.tm_kcur);
        tma_prefetch_desc(&p.tm_vcur);
        tma_prefetch_desc(&p.tm_cache_k);
        tma_prefetch_desc(&p.tm_cache_v);
    }
    // launched as a programmatic dependent: the set-up above overlaps the previous kernel's
    // tail; nothing the previous kernel may have written (table, Q, K/V, partials) is read or
    // written before it has completed
    grid_dependency_wait();
    if (warp == 2 && lane == 0) load_table(ctl, p.table, p.status);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // the combine that follows may be scheduled now; it waits for this grid's completion itself
    grid_dependents_launch();

    const uint32_t tmem = ctl->tmem_base;
    const int n_tiles = ctl->n_tiles;
    // slice s takes key tiles s, s + splits, s + 2 splits, ...: every slice gets the same mix of
    // contiguous cache tiles and current-chunk tiles (read from the caller's [B, T, H, d] layout,
    // 128 separate rows each), so the slices finish together
    const int sl = blockIdx.x, ns = p.splits;
    const int n = sl < n_tiles ? (n_tiles - sl + ns - 1) / ns : 0;   // key tiles of this slice

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0 && n > 0) {
            const uint32_t qbar = smem_u32(&ctl->q_full);
            mbar_arrive_expect_tx(qbar, QKTile<D, kQK8>::kBytes);
            for (int c = 0; c < QKTile<D, kQK8>::kBoxes; ++c)
                tma_load_4d(smem_u32(q_smem + c * kBoxBytes), &p.tm_q, qbar, c * QKTile<D, kQK8>::kBoxCols, h, 0, b);
            uint32_t it = 0;
            bool ok = true;
            for (int jj = 0, j = sl; jj < n && ok; ++jj, j += ns) {
                for (int kv = 0; kv < 2; ++kv, ++it) {
                    const int s = it % kStages;
                    if (!wait_or_abort(smem_u32(&ctl->kv_empty[s]), ((it / kStages) & 1) ^ 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fbar = smem_u32(&ctl->kv_full[s]);
                    mbar_arrive_expect_tx(fbar, kv_tile_bytes<D, kQK8, kPV8>(kv));
                    load_kv_tile<D, kQK8, kPV8>(p, ctl, j, kv, h, b, smem_u32(kv_smem + s * kTileBytes), fbar);
                }
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
            const uint32_t tO = tmem + L::kColO;
            bool ok = wait_or_abort(smem_u32(&ctl->q_full), 0, abort_flag);
            if (ok) ok = wait_or_abort(smem_u32(&ctl->kv_full[0]), 0, abort_flag);
            if (ok) {
                tc_fence_after();
                issue_s_qk<D, kQK8>(tmem, q_base, kv_base);   // S_0 into buffer 0
                mma_commit(smem_u32(&ctl->s_full[0]));
                mma_commit(smem_u32(&ctl->kv_empty[0]));
            }
            for (int jj = 0; jj < n && ok; ++jj) {
                if (jj + 1 < n) {
                    // S_{jj+1} into the other buffer: it held P_{jj-1}, whose PV was issued in
                    // the previous iteration, and one thread's MMAs run in issue order
                    const uint32_t itK = 2 * jj + 2;
                    const int sK = itK % kStages;
                    if (!wait_or_abort(smem_u32(&ctl->kv_full[sK]), (itK / kStages) & 1, abort_flag)) break;
                    tc_fence_after();
                    const int nb = (jj + 1) & 1;
                    issue_s_qk<D, kQK8>(tmem + nb * kBlockN, q_base, kv_base + sK * kTileBytes);
                    mma_commit(smem_u32(&ctl->s_full[nb]));
                    mma_commit(smem_u32(&ctl->kv_empty[sK]));
                }
                const uint32_t itV = 2 * jj + 1;
                const int sV = itV % kStages;
                const int buf = jj & 1;
                const uint32_t ph = (jj >> 1) & 1;
                const uint32_t tP = tmem + buf * kBlockN;
                if (!wait_or_abort(smem_u32(&ctl->kv_full[sV]), (itV / kStages) & 1, abort_flag)) break;
                if (!wait_or_abort(smem_u32(&ctl->p_half[buf]), ph, abort_flag)) break;
                tc_fence_after();
                split_pv_half<D, kPV8>(tO, tP, kv_base + sV * kTileBytes, 0, jj > 0);
                if (!wait_or_abort(smem_u32(&ctl->p_full[buf]), ph, abort_flag)) break;
                tc_fence_after();
                split_pv_half<D, kPV8>(tO, tP, kv_base + sV * kTileBytes, 1, true);
                mma_commit(smem_u32(&x->pv_done));
                mma_commit(smem_u32(&ctl->kv_empty[sV]));
                if (jj + 1 == n) mma_commit(smem_u32(&ctl->o_full[0]));   // O complete: epilogue
            }
            // every MMA issued has completed before the CTA can release TMEM
            mma_commit(smem_u32(&ctl->drain));
            wait_drain(smem_u32(&ctl->drain), 0);
        }
    } else if ((warp & 3) < n_warps) {
        // ------------------------------------------------------------ softmax warps
        // warp w may only touch TMEM lane quarter w % 4
        const int wq = warp & 3;
        const int row = wq * 32 + lane;   // query row inside the tile
        const uint32_t lane_base = tmem + ((uint32_t)(wq * 32) << 16);
        const uint32_t tO = lane_base + L::kColO;
        float m_ref = -INFINITY;   // reference max, log2-scaled
        float l = 0.f;             // row sum of the weights (see softmax_step)
        bool ok = true;
        for (int jj = 0; jj < n; ++jj) {
            int seg, row0, valid;
            tile_of(ctl, sl + jj * ns, seg, row0, valid);
            const int buf = jj & 1;
            ok = warp_wait(smem_u32(&ctl->s_full[buf]), (jj >> 1) & 1, abort_flag);
            if (!ok) break;
            tc_fence_after();
            softmax_step<D, true, kPV8>(lane_base + buf * kBlockN, tO, valid, jj == 0, smem_u32(&ctl->p_half[buf]),
                                  p.scale_log2, m_ref, l, smem_u32(&x->pv_done), (uint32_t)((jj - 1) & 1),
                                  abort_flag);
            warp_arrive(smem_u32(&ctl->p_full[buf]));
        }
        // ------------------------------------------------------------ partials of the slice
        const size_t prow = ((size_t)blockIdx.x * p.B * p.H + bh) * kBlockM + row;
        if (n == 0) {
            if (row < n_rows) {   // empty slice: neutral partials
                float4* o4 = reinterpret_cast<float4*>(p.o_part + prow * D);
                for (int c = 0; c < D / 4; ++c) o4[c] = make_float4(0.f, 0.f, 0.f, 0.f);
                p.ml_part[prow * 2 + 0] = -INFINITY;
                p.ml_part[prow * 2 + 1] = 0.f;
            }
        } else if (ok && warp_wait(smem_u32(&ctl->o_full[0]), 0, abort_flag)) {
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(tO + c * 32, o);
                tmem_wait_ld_dep(o);
                if (row < n_rows) {
                    float4* dst = reinterpret_cast<float4*>(p.o_part + prow * D + c * 32);
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        dst[i] = make_float4(__uint_as_float(o[4 * i]), __uint_as_float(o[4 * i + 1]),
                                             __uint_as_float(o[4 * i + 2]), __uint_as_float(o[4 * i + 3]));
                }
            }
            if (row < n_rows) {
                p.ml_part[prow * 2 + 0] = m_ref;
                p.ml_part[prow * 2 + 1] = l;
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

template <int D, bool kQK8, bool kPV8>
static cudaError_t launch_split_d(const AttnParams& p, int splits, cudaStream_t stream) {
    using L = SplitLayout<D>;
    auto kern = attn_split_kernel<D, kQK8, kPV8>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmemBytes);
    if (e != cudaSuccess) return e;
    return launch_dependent(kern, dim3(splits, p.H, p.B), dim3(L::kThreads), L::kSmemBytes, stream, p);
}

cudaError_t launch_split(const AttnParams& p, int d, int splits, cudaStream_t stream) {
    if (p.n_q < 1 || p.n_q > kBlockM || splits < 1) return cudaErrorInvalidValue;
    if (d == 128) {
        if (p.qk_fp8) return p.pv_fp8 ? launch_split_d<128, true, true>(p, splits, stream)
                                      : launch_split_d<128, true, false>(p, splits, stream);
        return launch_split_d<128, false, false>(p, splits, stream);
    }
    if (d == 64 && !p.qk_fp8) return launch_split_d<64, false, false>(p, splits, stream);
    return cudaErrorInvalidValue;
}

// ------------------------------------------------------------------ split-K combine (K4)
// out[row] = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s, M = max_s m_s (log-sum-exp merge).
// One warp per (b, h, row); each lane owns d/32 consecutive columns.
template <int D>
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ o_part,
                                                      const float* __restrict__ ml_part, void* out,
                                                      int B, int H, int n_q, int splits, int out_f32,
                                                      float out_scale) {
    // one warp per output row; each lane owns D / 32 consecutive columns.  The splits are read
    // eight at a time with every load of a group issued before any is used (one memory round
    // trip per group), and merged with a running max like the online softmax.
    constexpr int V = D / 32;
    constexpr int G = 8;
    static_assert(V == 4 || V == 2, "d = 128 or 64");
    // the next kernel in the stream (the next split-K forward, say) may start its set-up now;
    // it waits for this grid's completion before it reads or writes anything
    grid_dependents_launch();
    // launched as a programmatic dependent of the split kernel: wait until that grid has
    // completed and its partials are visible (returns at once for a plain launch)
    grid_dependency_wait();
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int total = B * H * n_q;
    if (warp >= total) return;
    const int row = warp % n_q;
    const int bh = warp / n_q;
    const int b = bh / H, h = bh % H;
    const size_t stride_split = (size_t)B * H * kBlockM;
    const size_t row0 = (size_t)bh * kBlockM + row;
    float M = -INFINITY, den = 0.f;
    float acc[V];
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] = 0.f;
    for (int s0 = 0; s0 < splits; s0 += G) {
        float2 ml[G];
        float o[G][V];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const int s = s0 + g;
            if (s < splits) {
                const size_t prow = (size_t)s * stride_split + row0;
                ml[g] = __ldg(reinterpret_cast<const float2*>(ml_part) + prow);
                const float* src = o_part + prow * D + lane * V;
                if (V == 4) {
                    const float4 t = __ldg(reinterpret_cast<const float4*>(src));
                    o[g][0] = t.x; o[g][1] = t.y; o[g][V > 2 ? 2 : 0] = t.z; o[g][V > 3 ? 3 : 0] = t.w;
                } else {
                    const float2 t = __ldg(reinterpret_cast<const float2*>(src));
                    o[g][0] = t.x; o[g][1] = t.y;
                }
            } else {
                ml[g] = make_float2(-INFINITY, 0.f);
#pragma unroll
                for (int i = 0; i < V; ++i) o[g][i] = 0.f;
            }
        }
        float Mg = M;
#pragma unroll
        for (int g = 0; g < G; ++g) Mg = fmaxf(Mg, ml[g].x);
        if (Mg == -INFINITY) continue;                 // every slice so far is empty
        const float f = ex2_approx(M - Mg);            // 0 while nothing has been merged
        den *= f;
#pragma unroll
        for (int i = 0; i < V; ++i) acc[i] *= f;
#pragma unroll
        for (int g = 0; g < G; ++g) {
            if (ml[g].x == -INFINITY) continue;        // empty slice (or past the last split)
            const float w = ex2_approx(ml[g].x - Mg);
            den += w * ml[g].y;
#pragma unroll
            for (int i = 0; i < V; ++i) acc[i] += w * o[g][i];
        }
        M = Mg;
    }
    const float inv = out_scale / den;   // out_scale: the V scale of e4m3 V, else 1
    const size_t orow = ((size_t)b * n_q + row) * H + h;
    if (out_f32) {
        float* dst = static_cast<float*>(out) + orow * D + lane * V;
#pragma unroll
        for (int i = 0; i < V; ++i) dst[i] = acc[i] * inv;
    } else {
        uint32_t* dst = reinterpret_cast<uint32_t*>(static_cast<__nv_bfloat16*>(out) + orow * D + lane * V);
#pragma unroll
        for (int i = 0; i < V; i += 2) dst[i / 2] = pack_bf16x2(acc[i] * inv, acc[i + 1] * inv);
    }
}

cudaError_t launch_combine(const float* o_part, const float* ml_part, void* out, int B, int H,
                           int n_q, int d, int splits, int out_f32, float out_scale, cudaStream_t stream) {
    const long long warps = (long long)B * H * n_q;
    const unsigned blocks = (unsigned)((warps * 32 + 255) / 256);
    // programmatic dependent launch: the combine's blocks are scheduled while the split kernel
    // finishes, and wait on the device (griddepcontrol.wait) instead of behind a launch gap
    if (d == 128)
        return launch_dependent(combine_kernel<128>, dim3(blocks), dim3(256), 0, stream, o_part, ml_part, out, B, H,
                                n_q, splits, out_f32, out_scale);
    if (d == 64)
        return launch_dependent(combine_kernel<64>, dim3(blocks), dim3(256), 0, stream, o_part, ml_part, out, B, H,
                                n_q, splits, out_f32, out_scale);
    return cudaErrorInvalidValue;
}

}  // namespace swattn

// attn_kernel.cu -- fused attention of the active chunk over the bounded cache (sm_100a).
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
//   warps 4..   one warpgroup per Q tile (thread = query row = TMEM lane): online softmax in
//               fp32 registers -- row max, lazy rescale of O only when the max grows by more
//               than 2^8, exp2, row sum -- writes P as bf16 into the S columns.
// The two Q tiles share every K/V tile, and while one warpgroup runs its softmax the tensor
// core works on the other tile.  In split mode (short query sets) a CTA takes one Q tile and
// a slice of the key tiles, and writes unnormalised partials that a combine kernel merges.
#include "ptx.cuh"
#include "swattn_internal.h"

namespace swattn {

constexpr uint64_t kWaitLimitNs = 1000000000ull;   // 1 s: far above any legitimate wait
constexpr int kBoxCols = 64;                        // 128-byte swizzle atom = 64 bf16
constexpr int kBoxBytes = kBlockM * kBoxCols * 2;   // 16 KB: one TMA box (128 rows x 64 cols)
constexpr float kRescaleThreshold = 8.0f;           // log2 units: rescale O when max grows > 2^8

template <int D>
struct TileCfg {
    static constexpr int kBoxes = D / kBoxCols;
    static constexpr int kTileBytes = kBoxes * kBoxBytes;   // one 128-row tile of Q, K or V
    static constexpr int kStages = D == 128 ? 4 : 6;
};

struct SmemCtl {
    uint64_t q_full;
    uint64_t kv_full[8];
    uint64_t kv_empty[8];
    uint64_t s_full[2];
    uint64_t p_full[2];
    uint64_t o_full[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    int n_seg;
    int n_tiles;
    int seg_kind[kMaxW + 3];
    int seg_slot[kMaxW + 3];
    int seg_ntok[kMaxW + 3];
    int seg_tile0[kMaxW + 4];   // first tile index of each segment; [n_seg] = total
};

template <int D, int NQ>
struct AttnLayout {
    using C = TileCfg<D>;
    static constexpr int kQBytes = NQ * C::kTileBytes;
    static constexpr int kKVBytes = C::kStages * C::kTileBytes;
    static constexpr int kCtlOffset = kQBytes + kKVBytes;
    static constexpr int kSmemBytes = kCtlOffset + (int)sizeof(SmemCtl) + 1024;  // + align slack
    static constexpr int kThreads = 128 + NQ * 128;
    static constexpr int kTmemNeed = NQ * (kBlockN + D);
    static constexpr int kTmemCols = kTmemNeed <= 256 ? 256 : 512;
};

// Bounded wait that also honours the CTA abort flag; raises the flag on a timeout.
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, volatile int* flag) {
    const bool ok = mbar_wait(bar, parity, flag, kWaitLimitNs);
    if (!ok) *flag = 1;
    return ok;
}

// Bounded wait used while draining: ignores the abort flag (copies in flight always land).
__device__ __forceinline__ void wait_drain(uint32_t bar, uint32_t parity) {
    int never = 0;
    (void)mbar_wait(bar, parity, &never, kWaitLimitNs);
}

// Which segment tile j belongs to, its first key row, and how many of its 128 rows are keys.
__device__ __forceinline__ void tile_of(const SmemCtl* ctl, int j, int& seg, int& row0, int& valid) {
    int s = 0;
    while (s + 1 < ctl->n_seg && ctl->seg_tile0[s + 1] <= j) ++s;
    seg = s;
    row0 = (j - ctl->seg_tile0[s]) * kBlockN;
    const int rem = ctl->seg_ntok[s] - row0;
    valid = rem < kBlockN ? rem : kBlockN;
}

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
    const int bh = b * p.H + h;
    const bool split_mode = p.splits > 0;

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
                mbar_init(smem_u32(&ctl->p_full[q]), 128);
                mbar_init(smem_u32(&ctl->o_full[q]), 1);
            }
            mbar_init(smem_u32(&ctl->drain), 1);
            ctl->abort_flag = 0;
            fence_mbar_init();
        }
        __syncwarp();
        tmem_alloc(smem_u32(&ctl->tmem_base), L::kTmemCols);
        tmem_relinquish();
    } else if (warp == 2 && lane == 0) {
        // copy the visibility table's segment list into shared memory
        const int n_seg = p.table[1];
        int ok = n_seg >= 1 && n_seg <= kMaxW + 3;
        int tiles = 0;
        if (ok) {
            for (int s = 0; s < n_seg; ++s) {
                const int* e = p.table + 3 + 4 * s;
                const int kind = e[0], slot = e[2], ntok = e[3];
                if (kind < 0 || kind > 2 || ntok <= 0) ok = 0;
                ctl->seg_kind[s] = kind;
                ctl->seg_slot[s] = slot;
                ctl->seg_ntok[s] = ntok;
                ctl->seg_tile0[s] = tiles;
                tiles += (ntok + kBlockN - 1) / kBlockN;
            }
            ctl->seg_tile0[n_seg] = tiles;
        }
        if (!ok) {
            atomicOr(p.status, SW_STATUS_BAD_SLOT);
            ctl->n_seg = 0;
            ctl->n_tiles = 0;
        } else {
            ctl->n_seg = n_seg;
            ctl->n_tiles = tiles;
        }
    } else if (warp == 1 && lane == 0) {
        tma_prefetch_desc(&p.tm_q);
        tma_prefetch_desc(&p.tm_kcur);
        tma_prefetch_desc(&p.tm_vcur);
        tma_prefetch_desc(&p.tm_cache_k);
        tma_prefetch_desc(&p.tm_cache_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem = ctl->tmem_base;
    const int n_tiles = ctl->n_tiles;
    int t0 = 0, t1 = n_tiles;
    if (split_mode) {
        t0 = (int)((long long)blockIdx.x * n_tiles / p.splits);
        t1 = (int)((long long)(blockIdx.x + 1) * n_tiles / p.splits);
    }
    const int n = t1 - t0;                          // key tiles this CTA processes
    const int m0 = split_mode ? 0 : blockIdx.x * NQ * kBlockM;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0 && n > 0) {
            const uint32_t qbar = smem_u32(&ctl->q_full);
            mbar_arrive_expect_tx(qbar, NQ * kTileBytes);
            for (int qt = 0; qt < NQ; ++qt)
                for (int c = 0; c < C::kBoxes; ++c)
                    tma_load_4d(smem_u32(q_smem + qt * kTileBytes + c * kBoxBytes), &p.tm_q, qbar,
                                c * kBoxCols, h, m0 + qt * kBlockM, b);
            uint32_t it = 0;
            bool ok = true;
            for (int j = t0; j < t1 && ok; ++j) {
                int seg, row0, valid;
                tile_of(ctl, j, seg, row0, valid);
                const int kind = ctl->seg_kind[seg];
                const int slot = ctl->seg_slot[seg];
                for (int kv = 0; kv < 2; ++kv, ++it) {
                    const int s = it % kStages;
                    const uint32_t r = it / kStages;
                    if (!wait_or_abort(smem_u32(&ctl->kv_empty[s]), (r & 1) ^ 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fbar = smem_u32(&ctl->kv_full[s]);
                    mbar_arrive_expect_tx(fbar, kTileBytes);
                    const uint32_t dst = smem_u32(kv_smem + s * kTileBytes);
                    for (int c = 0; c < C::kBoxes; ++c) {
                        const uint32_t d = dst + c * kBoxBytes;
                        if (kind == 0)
                            tma_load_4d(d, kv ? &p.tm_cond_v : &p.tm_cond_k, fbar, c * kBoxCols, row0, h, b);
                        else if (kind == 1)
                            tma_load_5d(d, kv ? &p.tm_cache_v : &p.tm_cache_k, fbar, c * kBoxCols, row0,
                                        slot, h, b);
                        else
                            tma_load_4d(d, kv ? &p.tm_vcur : &p.tm_kcur, fbar, c * kBoxCols, h, row0, b);
                    }
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
            constexpr uint32_t idesc_s = idesc_bf16_f32(kBlockM, kBlockN, false);
            constexpr uint32_t idesc_o = idesc_bf16_f32(kBlockM, D, true);
            const uint32_t q_base = smem_u32(q_smem);
            const uint32_t kv_base = smem_u32(kv_smem);
            auto issue_s = [&](int qt, int s) {
                const uint32_t tS = tmem + qt * kBlockN;
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * kBoxBytes + (ks & 3) * 32;
                    const uint64_t a = smem_desc_sw128(q_base + qt * kTileBytes + off, 16, 1024);
                    const uint64_t bd = smem_desc_sw128(kv_base + s * kTileBytes + off, 16, 1024);
                    mma_ss(tS, a, bd, idesc_s, ks > 0 ? 1u : 0u);
                }
            };
            auto issue_pv = [&](int qt, int s, bool acc) {
                const uint32_t tS = tmem + qt * kBlockN;
                const uint32_t tO = tmem + NQ * kBlockN + qt * D;
#pragma unroll
                for (int ks = 0; ks < kBlockN / 16; ++ks) {
                    const uint64_t bd = smem_desc_sw128(kv_base + s * kTileBytes + ks * 16 * 128,
                                                        kBoxBytes, 1024);
                    mma_ts(tO, tS + ks * 8, bd, idesc_o, (acc || ks > 0) ? 1u : 0u);
                }
            };
            bool ok = wait_or_abort(smem_u32(&ctl->q_full), 0, abort_flag);
            if (ok) ok = wait_or_abort(smem_u32(&ctl->kv_full[0]), 0, abort_flag);
            if (ok) {
                tc_fence_after();
                for (int qt = 0; qt < NQ; ++qt) {
                    issue_s(qt, 0);
                    mma_commit(smem_u32(&ctl->s_full[qt]));
                }
                mma_commit(smem_u32(&ctl->kv_empty[0]));
            }
            for (int jj = 0; jj < n && ok; ++jj) {
                const uint32_t itV = 2 * jj + 1, itK = 2 * jj + 2;
                const int sV = itV % kStages, sK = itK % kStages;
                const bool more = jj + 1 < n;
                if (!wait_or_abort(smem_u32(&ctl->kv_full[sV]), (itV / kStages) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                for (int qt = 0; qt < NQ && ok; ++qt) {
                    if (!wait_or_abort(smem_u32(&ctl->p_full[qt]), jj & 1, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    issue_pv(qt, sV, jj > 0);
                    mma_commit(smem_u32(&ctl->o_full[qt]));
                    if (more) {
                        if (qt == 0 &&
                            !wait_or_abort(smem_u32(&ctl->kv_full[sK]), (itK / kStages) & 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        // P_q lives in the S_q columns: the next S_q may only be written once
                        // this tile's PV has read P.
                        if (!wait_or_abort(smem_u32(&ctl->o_full[qt]), jj & 1, abort_flag)) { ok = false; break; }
                        tc_fence_after();
                        issue_s(qt, sK);
                        mma_commit(smem_u32(&ctl->s_full[qt]));
                    }
                }
                if (!ok) break;
                mma_commit(smem_u32(&ctl->kv_empty[sV]));
                if (more) mma_commit(smem_u32(&ctl->kv_empty[sK]));
            }
            // every MMA issued has completed before the CTA can release TMEM
            mma_commit(smem_u32(&ctl->drain));
            wait_drain(smem_u32(&ctl->drain), 0);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ softmax warpgroups
        const int qt = (warp - 4) >> 2;
        const int wq = warp & 3;                       // TMEM lane quarter of this warp
        const int row = wq * 32 + lane;                // query row inside the tile
        const uint32_t lane_base = tmem + ((uint32_t)(wq * 32) << 16);
        const uint32_t tS = lane_base + qt * kBlockN;
        const uint32_t tO = lane_base + NQ * kBlockN + qt * D;
        const float sl2 = p.scale_log2;
        float m_ref = -INFINITY;   // reference max, log2-scaled
        float l = 0.f;             // row sum of exp2(s*sl2 - m_ref)
        bool ok = true;
        for (int jj = 0; jj < n; ++jj) {
            int seg, row0, valid;
            tile_of(ctl, t0 + jj, seg, row0, valid);
            ok = wait_or_abort(smem_u32(&ctl->s_full[qt]), jj & 1, abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            uint32_t sr[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, sr[c]);
            tmem_wait_ld_dep(sr[0]);
            reg_fence(sr[1]);
            reg_fence(sr[2]);
            reg_fence(sr[3]);
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    float v = __uint_as_float(sr[c][i]);
                    if (c * 32 + i >= valid) v = -INFINITY;
                    sr[c][i] = __float_as_uint(v);
                    mx = fmaxf(mx, v);
                }
            const float m_new = mx * sl2;
            if (jj == 0) {
                m_ref = m_new;
            } else {
                const bool need = m_new > m_ref + kRescaleThreshold;
                if (__any_sync(0xffffffffu, need)) {
                    float f = 1.f;
                    if (need) {
                        f = ex2_approx(m_ref - m_new);
                        m_ref = m_new;
                    }
                    l *= f;
                    ok = wait_or_abort(smem_u32(&ctl->o_full[qt]), (jj - 1) & 1, abort_flag);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32(tO + c * 32, o);
                        tmem_wait_ld_dep(o);
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
                        tmem_st32(tO + c * 32, o);
                    }
                    tmem_wait_st();
                }
            }
            float sum = 0.f;
            uint32_t pk[2][32];
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    const float p0 = ex2_approx(fmaf(__uint_as_float(sr[c][i]), sl2, -m_ref));
                    const float p1 = ex2_approx(fmaf(__uint_as_float(sr[c][i + 1]), sl2, -m_ref));
                    sum += p0 + p1;
                    pk[c >> 1][(c & 1) * 16 + (i >> 1)] = pack_bf16x2(p0, p1);
                }
            l += sum;
            tmem_st32(tS, pk[0]);
            tmem_st32(tS + 32, pk[1]);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(smem_u32(&ctl->p_full[qt]));
        }
        // ------------------------------------------------------------ epilogue
        const int m_row = m0 + qt * kBlockM + row;
        if (n == 0) {
            // split mode with an empty slice: neutral partials
            if (split_mode) {
                const size_t prow = ((size_t)blockIdx.x * p.B * p.H + bh) * kBlockM + row;
                float4* o4 = reinterpret_cast<float4*>(p.o_part + prow * D);
                for (int c = 0; c < D / 4; ++c) o4[c] = make_float4(0.f, 0.f, 0.f, 0.f);
                p.ml_part[prow * 2 + 0] = -INFINITY;
                p.ml_part[prow * 2 + 1] = 0.f;
            }
        } else if (ok) {
            ok = wait_or_abort(smem_u32(&ctl->o_full[qt]), (n - 1) & 1, abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (ok) {
                tc_fence_after();
                const float inv = 1.f / l;
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(tO + c * 32, o);
                    tmem_wait_ld_dep(o);
                    if (split_mode) {
                        const size_t prow = ((size_t)blockIdx.x * p.B * p.H + bh) * kBlockM + row;
                        float4* dst = reinterpret_cast<float4*>(p.o_part + prow * D + c * 32);
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            dst[i] = make_float4(__uint_as_float(o[4 * i]), __uint_as_float(o[4 * i + 1]),
                                                 __uint_as_float(o[4 * i + 2]), __uint_as_float(o[4 * i + 3]));
                        if (c == 0) {
                            p.ml_part[prow * 2 + 0] = m_ref;
                            p.ml_part[prow * 2 + 1] = l;
                        }
                    } else if (m_row < p.n_q) {
                        const size_t orow = ((size_t)b * p.n_q + m_row) * p.H + h;
                        if (p.out_f32) {
                            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + orow * D + c * 32);
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                dst[i] = make_float4(__uint_as_float(o[4 * i]) * inv,
                                                     __uint_as_float(o[4 * i + 1]) * inv,
                                                     __uint_as_float(o[4 * i + 2]) * inv,
                                                     __uint_as_float(o[4 * i + 3]) * inv);
                        } else {
                            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + orow * D + c * 32);
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                dst[i] = make_uint4(
                                    pack_bf16x2(__uint_as_float(o[8 * i + 0]) * inv, __uint_as_float(o[8 * i + 1]) * inv),
                                    pack_bf16x2(__uint_as_float(o[8 * i + 2]) * inv, __uint_as_float(o[8 * i + 3]) * inv),
                                    pack_bf16x2(__uint_as_float(o[8 * i + 4]) * inv, __uint_as_float(o[8 * i + 5]) * inv),
                                    pack_bf16x2(__uint_as_float(o[8 * i + 6]) * inv, __uint_as_float(o[8 * i + 7]) * inv));
                        }
                    }
                }
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

template <int D, int NQ>
static cudaError_t launch_one(const AttnParams& p, int grid_x, cudaStream_t stream) {
    using L = AttnLayout<D, NQ>;
    auto kern = attn_fwd_kernel<D, NQ>;
    // per device and cheap; set on every launch so any current device is covered
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         L::kSmemBytes);
    if (e != cudaSuccess) return e;
    dim3 grid(grid_x, p.H, p.B);
    kern<<<grid, L::kThreads, L::kSmemBytes, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_attention(const AttnParams& p, int d, int q_tiles_per_cta, int grid_x,
                             cudaStream_t stream) {
    if (d == 128) {
        return q_tiles_per_cta == 2 ? launch_one<128, 2>(p, grid_x, stream)
                                    : launch_one<128, 1>(p, grid_x, stream);
    }
    if (d == 64) {
        return q_tiles_per_cta == 2 ? launch_one<64, 2>(p, grid_x, stream)
                                    : launch_one<64, 1>(p, grid_x, stream);
    }
    return cudaErrorInvalidValue;
}

// ------------------------------------------------------------------ split-K combine (K4)
// out[row] = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s, M = max_s m_s (log-sum-exp merge).
// One warp per (b, h, row); each lane owns d/32 consecutive columns.
template <int D>
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ o_part,
                                                      const float* __restrict__ ml_part, void* out,
                                                      int B, int H, int n_q, int splits, int out_f32) {
    constexpr int V = D / 32;
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int total = B * H * n_q;
    if (warp >= total) return;
    const int row = warp % n_q;
    const int bh = warp / n_q;
    const int b = bh / H, h = bh % H;
    const size_t stride_split = (size_t)B * H * kBlockM;
    float M = -INFINITY;
    for (int s = 0; s < splits; ++s)
        M = fmaxf(M, ml_part[((size_t)s * stride_split + (size_t)bh * kBlockM + row) * 2]);
    float acc[V];
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] = 0.f;
    float den = 0.f;
    for (int s = 0; s < splits; ++s) {
        const size_t prow = (size_t)s * stride_split + (size_t)bh * kBlockM + row;
        const float ms = ml_part[prow * 2];
        if (ms == -INFINITY) continue;            // empty slice
        const float w = ex2_approx(ms - M);
        den += w * ml_part[prow * 2 + 1];
        const float* src = o_part + prow * D + lane * V;
#pragma unroll
        for (int i = 0; i < V; ++i) acc[i] += w * src[i];
    }
    const float inv = 1.f / den;
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
                           int n_q, int d, int splits, int out_f32, cudaStream_t stream) {
    const long long warps = (long long)B * H * n_q;
    const unsigned blocks = (unsigned)((warps * 32 + 255) / 256);
    if (d == 128)
        combine_kernel<128><<<blocks, 256, 0, stream>>>(o_part, ml_part, out, B, H, n_q, splits, out_f32);
    else if (d == 64)
        combine_kernel<64><<<blocks, 256, 0, stream>>>(o_part, ml_part, out, B, H, n_q, splits, out_f32);
    else
        return cudaErrorInvalidValue;
    return cudaGetLastError();
}

}  // namespace swattn

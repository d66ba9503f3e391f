// attn_common.cuh -- pieces shared by the attention kernels: tile geometry, the shared-memory
// control block, bounded waits, the tile schedule over the visibility table, the TMA loads of
// one K or V tile, the tcgen05 issue of S = Q K^T and O += P V, and one softmax step.
#pragma once
#include "ptx.cuh"
#include "swattn_internal.h"

namespace swattn {

constexpr uint64_t kWaitLimitNs = 1000000000ull;   // 1 s: far above any legitimate wait
constexpr int kBoxCols = 64;                        // 128-byte swizzle atom = 64 bf16
constexpr int kBoxBytes = kBlockM * kBoxCols * 2;   // 16 KB: one TMA box (128 rows x 64 cols)
constexpr float kRescaleThreshold = 8.0f;           // log2 units: rescale O when max grows > 2^8
// e4m3 P: weights are formed as 2^(s*sl2 - m + kP8Offset) and O is rescaled when the max grows
// by more than 2^kP8Threshold, so P <= 2^(offset + threshold) = 256 stays below the e4m3 limit
// (448) while the typical weight of a row (2^-6 .. 2^-2 of the max for Gaussian scores) lands in
// e4m3's normal range, not its subnormals.  The factor 2^kP8Offset is common to l and O of every
// partial, so it cancels in O / l and in the merge of split partials.
constexpr float kP8Offset = 4.0f;
constexpr float kP8Threshold = 4.0f;
// One in kPolyEvery pairs of exponentials runs on the FMA pipe (exp2_poly) instead of MUFU
// (0: none).  At two Q tiles per CTA the exponentials alone keep MUFU as busy as the tensor
// core, but the softmax step is bound by issue and latency first; measured, not assumed.
#ifndef SWATTN_POLY_EVERY
#define SWATTN_POLY_EVERY 0
#endif
constexpr int kPolyEvery = SWATTN_POLY_EVERY;
// Publish P in two halves (PV of the first 64 keys overlaps the exponentials of the rest).
#ifndef SWATTN_SPLIT_P
#define SWATTN_SPLIT_P 1
#endif
constexpr bool kSplitP = SWATTN_SPLIT_P != 0;
// MMA issuer serves whichever Q tile is ready (1) or strictly alternates between them (0).
// Measured on B200: polling both tiles costs the softmax warps that share the MMA warp's
// sub-partition more issue slots than it saves, so alternating is the default.
#ifndef SWATTN_DYNAMIC_MMA
#define SWATTN_DYNAMIC_MMA 0
#endif
constexpr bool kDynamicMma = SWATTN_DYNAMIC_MMA != 0;

template <int D>
struct TileCfg {
    static constexpr int kBoxes = D / kBoxCols;
    static constexpr int kTileBytes = kBoxes * kBoxBytes;   // one 128-row tile of Q, K or V
    static constexpr int kStages = D == 128 ? 4 : 6;
};

struct SmemCtl {
    uint64_t q_full;
    uint64_t q_empty;
    uint64_t kv_full[8];
    uint64_t kv_empty[8];
    uint64_t s_full[2];
    uint64_t p_half[2];         // first 64 keys of P written (PV may start on them)
    uint64_t p_full[2];
    uint64_t o_full[2];
    uint64_t o_empty[2];
    uint64_t drain;
    uint64_t merge_bar[2][3];   // staged merge of split-piece partials: per Q tile, three buffers
    uint64_t prod_done;         // the producer has issued its last copy and every copy has landed
    uint32_t tmem_base;
    int abort_flag;
    int n_seg;
    int n_tiles;
    int merge_flag[2];
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
    static constexpr int kThreads = 64 + NQ * 128;    // producer, MMA, NQ softmax warpgroups
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

// One arrival per warp: the warp's lanes finish their work (and tcgen05 fences) first.  128
// single-thread arrivals on one barrier word serialise for hundreds of cycles.
__device__ __forceinline__ void warp_arrive(uint32_t bar) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// Warp-uniform wait for the softmax warps.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* flag) {
    const bool ok = wait_or_abort(bar, parity, flag);
    return __all_sync(0xffffffffu, ok);
}

// Copy the table's segment list into shared memory (one thread).  Returns false on a table
// that cannot be right; the caller then processes nothing and the status word says why.
__device__ __forceinline__ void load_table(SmemCtl* ctl, const int32_t* table, int32_t* status) {
    const int n_seg = table[1];
    int ok = n_seg >= 1 && n_seg <= kMaxW + 3;
    int tiles = 0;
    if (ok) {
        for (int s = 0; s < n_seg; ++s) {
            const int32_t* e = table + 3 + 4 * s;
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
        atomicOr(status, SW_STATUS_BAD_SLOT);
        ctl->n_seg = 0;
        ctl->n_tiles = 0;
    } else {
        ctl->n_seg = n_seg;
        ctl->n_tiles = tiles;
    }
}

// Segment of key tile j.
__device__ __forceinline__ int tile_seg(const SmemCtl* ctl, int j) {
    int s = 0;
    while (s + 1 < ctl->n_seg && ctl->seg_tile0[s + 1] <= j) ++s;
    return s;
}

// Which segment key tile j belongs to, its first key row, and how many of its rows are keys.
__device__ __forceinline__ void tile_of(const SmemCtl* ctl, int j, int& seg, int& row0, int& valid) {
    int s = 0;
    while (s + 1 < ctl->n_seg && ctl->seg_tile0[s + 1] <= j) ++s;
    seg = s;
    row0 = (j - ctl->seg_tile0[s]) * kBlockN;
    const int rem = ctl->seg_ntok[s] - row0;
    valid = rem < kBlockN ? rem : kBlockN;
}

// Query tiles of a launch: the chunk's n_q queries in tiles 0 .. ceil(n_q / 128) - 1, then (joint
// forward) the n_qc condition-stream queries, which attend over the same visible keys.
struct QSrc {
    const CUtensorMap* tm;   // tensor map of the tile's query tensor
    int row0;                // first query row of the tile in that tensor
    int rows;                // rows of that tensor (n_q or n_qc)
    void* out;               // output tensor of the same rows
};

__device__ __forceinline__ int q_tiles(const AttnParams& p) {
    return (p.n_q + kBlockM - 1) / kBlockM + (p.n_qc + kBlockM - 1) / kBlockM;
}

__device__ __forceinline__ QSrc q_src(const AttnParams& p, int u) {
    const int nv = (p.n_q + kBlockM - 1) / kBlockM;
    if (u < nv) return QSrc{&p.tm_q, u * kBlockM, p.n_q, p.out};
    return QSrc{&p.tm_qc, (u - nv) * kBlockM, p.n_qc, p.out_c};
}

// TMA loads of one 128-row K (kv = 0) or V (kv = 1) tile of key tile j of (b, h) into dst,
// completing on bar: condition tokens, a ring slot, or the caller's current chunk.
template <int D, bool kQK8 = false, bool kPV8 = false>
__device__ __forceinline__ void load_kv_tile(const AttnParams& p, const SmemCtl* ctl, int j, int kv,
                                             int h, int b, uint32_t dst, uint32_t bar) {
    int seg, row0, valid;
    tile_of(ctl, j, seg, row0, valid);
    const int kind = ctl->seg_kind[seg];
    const int slot = ctl->seg_slot[seg];
    // an e4m3 tile (K, or V on a pv_fp8 handle) is one box of 128-byte rows; bf16 keeps its
    // 64-column boxes
    const int boxes = ((kQK8 && kv == 0) || (kPV8 && kv == 1)) ? 1 : TileCfg<D>::kBoxes;
#pragma unroll
    for (int c = 0; c < TileCfg<D>::kBoxes; ++c) {
        if (c >= boxes) break;
        const uint32_t d = dst + c * kBoxBytes;
        if (kind == 0)
            tma_load_4d(d, kv ? &p.tm_cond_v : &p.tm_cond_k, bar, c * kBoxCols, row0, h, b);
        else if (kind == 1)
            tma_load_5d(d, kv ? &p.tm_cache_v : &p.tm_cache_k, bar, c * kBoxCols, row0, slot, h, b);
        else
            tma_load_4d(d, kv ? &p.tm_vcur : &p.tm_kcur, bar, c * kBoxCols, h, row0, b);
    }
}

// Bytes one K (kv = 0) or V (kv = 1) tile occupies in its ring stage.
template <int D, bool kQK8, bool kPV8>
__host__ __device__ constexpr int kv_tile_bytes(int kv) {
    return ((kQK8 && kv == 0) || (kPV8 && kv == 1)) ? kBlockN * D : TileCfg<D>::kTileBytes;
}

// Fused commit: the producer stores the active chunk's K_cur / V_cur tiles, which it has just
// loaded into the K/V ring for the attention, from shared memory to the chunk's ring slot in
// the cache.  A tile's store is issued kStages - 1 ring items after its load (by then the load
// has landed, and the stage cannot have been refilled), and a stage is refilled only after
// every issued store has finished reading shared memory.  The last kStages - 1 items are kept
// in registers, one packed 64-bit word each (store it; j, head, stream, K or V), shifted once per item;
// the producer flushes them and waits for the stores to complete before it finishes.  The
// per-item work is kept out of line: inlined, it changed the register allocation of the whole
// kernel and cost more (measured) than the stores themselves.
// kQK8 / kPV8: K / V tiles are e4m3, one box of 128-byte rows each (bf16: kBoxes boxes).
template <int D, int kStages, bool kQK8 = false, bool kPV8 = false>
struct CommitQueue {
    static constexpr int kLag = kStages - 1;
    static_assert(kLag >= 1 && kLag <= 7, "commit history");
    uint64_t hist[kLag] = {};   // hist[0]: oldest
    uint32_t pending = 0;       // stages with a store that may still be reading them

    // bit 63: store it; bits 32..62: key tile j; 16..31: head; 1..15: stream; 0: V (1) or K (0)
    __device__ __forceinline__ static uint64_t pack(bool store, int j, int kv, int h, int b) {
        return (store ? (1ull << 63) : 0ull) | ((uint64_t)(uint32_t)j << 32) | ((uint64_t)(h & 0xffff) << 16) |
               ((uint64_t)(b & 0x7fff) << 1) | (uint64_t)(kv & 1);
    }
    // Before stage s takes a new load: its last store (if any) must have read it.
    __device__ __forceinline__ void before_refill(int s) {
        if ((pending >> s) & 1u) {
            bulk_wait_read_all();
            pending = 0;
        }
    }
    __device__ __noinline__ bool store_one(const AttnParams& p, const SmemCtl* ctl, const uint8_t* kv_smem,
                                              int slot, uint32_t i, uint64_t w, volatile int* abort_flag) {
        const int s = (int)(i % kStages);
        if (!wait_or_abort(smem_u32(&ctl->kv_full[s]), (i / kStages) & 1, abort_flag)) return false;
        const int j = (int)((w >> 32) & 0x7fffffffu), kv = (int)(w & 1u);
        const int h = (int)((w >> 16) & 0xffffu), b = (int)((w >> 1) & 0x7fffu);
        int seg, row0, valid;
        tile_of(ctl, j, seg, row0, valid);
        fence_proxy_async_smem();
        const uint32_t src = smem_u32(kv_smem + (size_t)s * TileCfg<D>::kTileBytes);
        const int boxes = ((kQK8 && kv == 0) || (kPV8 && kv == 1)) ? 1 : TileCfg<D>::kBoxes;
#pragma unroll
        for (int c = 0; c < TileCfg<D>::kBoxes; ++c) {
            if (c >= boxes) break;
            tma_store_5d(kv ? &p.tm_cache_v : &p.tm_cache_k, src + c * kBoxBytes, c * kBoxCols, row0, slot, h, b);
        }
        bulk_commit_group();
        pending |= 1u << s;
        return true;
    }
    // Item it (just loaded) enters the history; the item kLag before it leaves and is stored if
    // marked.  Returns false if a wait gave up.
    __device__ __noinline__ bool step(const AttnParams& p, const SmemCtl* ctl, const uint8_t* kv_smem, int slot,
                                         uint32_t it, uint64_t w, volatile int* abort_flag) {
        const uint64_t out = hist[0];
#pragma unroll
        for (int q = 0; q + 1 < kLag; ++q) hist[q] = hist[q + 1];
        hist[kLag - 1] = w;
        if ((out >> 63) && it >= (uint32_t)kLag) return store_one(p, ctl, kv_smem, slot, it - kLag, out, abort_flag);
        return true;
    }
    // Store every marked item still in the history (the last items of the launch).
    __device__ __noinline__ bool flush(const AttnParams& p, const SmemCtl* ctl, const uint8_t* kv_smem, int slot,
                                          uint32_t it_next, volatile int* abort_flag) {
#pragma unroll
        for (int q = 0; q < kLag; ++q) {
            const uint32_t i = it_next - kLag + q;
            if ((hist[q] >> 63) && it_next >= (uint32_t)(kLag - q) &&
                !store_one(p, ctl, kv_smem, slot, i, hist[q], abort_flag))
                return false;
        }
        return true;
    }
};

// Bytes of one 128-row Q or K tile: bf16, or e4m3 (one 128-byte swizzle row per token, d = 128).
template <int D, bool kQK8>
struct QKTile {
    static constexpr int kBytes = kQK8 ? kBlockM * D : TileCfg<D>::kTileBytes;
    static constexpr int kBoxes = kQK8 ? 1 : TileCfg<D>::kBoxes;
    static constexpr int kBoxCols = kQK8 ? D : swattn::kBoxCols;   // elements per box row
    static_assert(!kQK8 || D == 128, "e4m3 Q/K tiles need d = 128");
};

// The MMA issue helpers below come in two forms: kWarp = false for one issuing thread, kWarp =
// true for a converged warp in which one lane (elect.sync) issues and every lane computes the
// operands.
template <bool kWarp>
__device__ __forceinline__ void mma_ss_any(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    if constexpr (kWarp) mma_ss_warp(d, a, b, idesc, acc);
    else mma_ss(d, a, b, idesc, acc);
}
template <bool kWarp>
__device__ __forceinline__ void mma_ss_f8_any(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    if constexpr (kWarp) mma_ss_f8_warp(d, a, b, idesc, acc);
    else mma_ss_f8(d, a, b, idesc, acc);
}
template <bool kWarp>
__device__ __forceinline__ void mma_ts_any(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    if constexpr (kWarp) mma_ts_warp(d, a, b, idesc, acc);
    else mma_ts(d, a, b, idesc, acc);
}
// D (+)= A[tmem] * B[smem desc] with 8-bit floating-point operands (kind::f8f6f4).
template <bool kWarp>
__device__ __forceinline__ void mma_ss_f8_tmem_any(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    if constexpr (kWarp) mma_ts_f8_warp(d, a, b, idesc, acc);
    else mma_ts_f8(d, a, b, idesc, acc);
}
template <bool kWarp>
__device__ __forceinline__ void mma_commit_any(uint32_t bar) {
    if constexpr (kWarp) mma_commit_warp(bar);
    else mma_commit(bar);
}

// S = Q K^T with e4m3 Q and K tiles (d = 128, one 128-byte row per token): four K = 32 steps.
template <bool kWarp = false>
__device__ __forceinline__ void issue_s_f8(uint32_t tS, uint32_t q_tile, uint32_t k_tile) {
    constexpr uint32_t idesc = idesc_e4m3_f32(kBlockM, kBlockN);
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
        mma_ss_f8_any<kWarp>(tS, smem_desc_sw128(q_tile + ks * 32, 16, 1024), smem_desc_sw128(k_tile + ks * 32, 16, 1024),
                             idesc, ks > 0 ? 1u : 0u);
}

// S[tS] = Q(q_tile) K(k_tile)^T: M = 128 queries, N = 128 keys, K = D, bf16 -> fp32.
template <int D, bool kWarp = false>
__device__ __forceinline__ void issue_s(uint32_t tS, uint32_t q_tile, uint32_t k_tile) {
    constexpr uint32_t idesc = idesc_bf16_f32(kBlockM, kBlockN, false);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t off = (ks >> 2) * kBoxBytes + (ks & 3) * 32;   // 16 columns = 32 bytes
        mma_ss_any<kWarp>(tS, smem_desc_sw128(q_tile + off, 16, 1024), smem_desc_sw128(k_tile + off, 16, 1024),
                          idesc, ks > 0 ? 1u : 0u);
    }
}

// S = Q K^T for either operand format.
template <int D, bool kQK8, bool kWarp = false>
__device__ __forceinline__ void issue_s_qk(uint32_t tS, uint32_t q_tile, uint32_t k_tile) {
    if constexpr (kQK8) issue_s_f8<kWarp>(tS, q_tile, k_tile);
    else issue_s<D, kWarp>(tS, q_tile, k_tile);
}

// O[tO] (+)= P[tP] V(v_tile): P (bf16 pairs in TMEM) is the A operand, V is MN-major in shared
// memory (16 key rows per step = 2 KB; the two 64-column boxes are 16 KB apart).
template <int D, bool kWarp = false>
__device__ __forceinline__ void issue_pv(uint32_t tO, uint32_t tP, uint32_t v_tile, bool accumulate) {
    constexpr uint32_t idesc = idesc_bf16_f32(kBlockM, D, true);
#pragma unroll
    for (int ks = 0; ks < kBlockN / 16; ++ks)
        mma_ts_any<kWarp>(tO, tP + ks * 8, smem_desc_sw128(v_tile + ks * 16 * 128, kBoxBytes, 1024), idesc,
                          (accumulate || ks > 0) ? 1u : 0u);
}

// Half of O += P V: keys [64 half, 64 half + 64) of the tile (4 MMA steps of 16 keys).
template <int D, bool kWarp = false>
__device__ __forceinline__ void issue_pv_half(uint32_t tO, uint32_t tP, uint32_t v_tile, int half,
                                              bool accumulate) {
    constexpr uint32_t idesc = idesc_bf16_f32(kBlockM, D, true);
#pragma unroll
    for (int k = 0; k < kBlockN / 32; ++k) {
        const int ks = half * (kBlockN / 32) + k;
        mma_ts_any<kWarp>(tO, tP + ks * 8, smem_desc_sw128(v_tile + ks * 16 * 128, kBoxBytes, 1024), idesc,
                          (accumulate || ks > 0) ? 1u : 0u);
    }
}

// Half of O += P V with e4m3 P (in TMEM, four keys per 32-bit column) and an e4m3 V tile (one box
// of 128-byte rows, MN-major: d contiguous per key): keys [64 half, 64 half + 64), two kind::f8f6f4
// MMA steps of 32 keys (32 rows of V = 4 KB apart; d = 128 is one 128-byte swizzle atom wide).
template <bool kWarp = false>
__device__ __forceinline__ void issue_pv_f8_half(uint32_t tO, uint32_t tP, uint32_t v_tile, int half, bool accumulate) {
    constexpr uint32_t idesc = idesc_e4m3_f32(kBlockM, 128, true);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int ks = half * 2 + k;
        mma_ss_f8_tmem_any<kWarp>(tO, tP + ks * 8, smem_desc_sw128(v_tile + ks * 32 * 128, kBlockN * 128, 1024), idesc,
                                  (accumulate || ks > 0) ? 1u : 0u);
    }
}

// One online-softmax step for this thread's query row over one key tile:
//   read the S row from TMEM, mask keys past the segment's end, update the reference max
//   (lazily: only when it grows by more than 2^kRescaleThreshold), write P = exp2(s*sl2 - m)
//   as bf16 pairs over the S columns, add the same rounded weights to l, and rescale the
//   O row in TMEM when the reference moved.
// P is published in two halves: the warp arrives on p_half_bar once keys 0..63 are written
// (the PV of those keys may then start) and the caller arrives on p_full after the return.
// A warp that must rescale O first publishes nothing early: its O rescale has to land before
// any PV of this tile.  The caller has waited for S.
// kWaitO: S was computed ahead of the previous tile's PV (double-buffered S), so before an O
// rescale the warp waits for that PV on o_bar (phase parity o_parity).  Without it, the
// previous PV is known complete (it was issued before this tile's S).
// kP8: P is written as e4m3 (four keys per 32-bit column, over S columns 0..31, for the
// kind::f8f6f4 P V), rounded to nearest, offset by 2^kP8Offset with its own rescale threshold;
// the row sum adds the fp32 weights before rounding.  Widening the bytes back to sum exactly the
// quantised weights costs ten instructions per four keys on an issue-bound loop; the fp32 sum
// leaves a common factor sum(q(p)) / sum(p) on the row, within the same 2^-4 relative bound as
// each quantised weight and, over many keys, far inside it (the rounding errors average out).
template <int D, bool kWaitO = false, bool kP8 = false>
__device__ __forceinline__ void softmax_step(uint32_t tS, uint32_t tO, int valid, bool first,
                                             uint32_t p_half_bar, float sl2, float& m_ref, float& l,
                                             uint32_t o_bar = 0, uint32_t o_parity = 0,
                                             volatile int* flag = nullptr) {
    uint32_t sr[4][32];
#pragma unroll
    for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, sr[c]);
    tmem_wait_ld_dep(sr[0]);
    reg_fence(sr[1]);
    reg_fence(sr[2]);
    reg_fence(sr[3]);
    if (valid < kBlockN) {
        // last tile of a segment: keys past its end read as zero; mask them out
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (c * 32 + i >= valid) sr[c][i] = __float_as_uint(-INFINITY);
    }
    // row max as an 8-way tree of three-input maxes: independent accumulators keep the
    // dependent chain short, two elements per instruction
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
    const float m_new = mxa[0] * sl2;
    float f = 1.f;            // factor that takes O and l to the new reference max
    bool rescale = false;     // warp-uniform: does this warp rescale O this tile
    if (first) {
        m_ref = m_new;
    } else {
        const bool need = m_new > m_ref + (kP8 ? kP8Threshold : kRescaleThreshold);
        rescale = __any_sync(0xffffffffu, need);
        if (need) {
            f = ex2_approx(m_ref - m_new);
            m_ref = m_new;
        }
    }
    float suma[8];
#pragma unroll
    for (int a = 0; a < 8; ++a) suma[a] = 0.f;
    const float neg_m = kP8 ? kP8Offset - m_ref : -m_ref;
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
                    // the row sum adds the fp32 weights (two packed adds per four keys)
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
                    // x = s * scale * log2(e) - m for two columns in one packed FMA
                    float x0, x1;
                    fma2_bcast(x0, x1, __uint_as_float(sr[c][i]), __uint_as_float(sr[c][i + 1]), sl2_2, neg_m2);
                    const bool poly = kPolyEvery > 0 && ((i >> 1) % (kPolyEvery > 0 ? kPolyEvery : 1)) == kPolyEvery - 1;
                    const float p0 = poly ? exp2_poly(x0) : ex2_approx(x0);
                    const float p1 = poly ? exp2_poly(x1) : ex2_approx(x1);
                    const uint32_t pp = pack_bf16x2(p0, p1);
                    // the row sum adds the same bf16-rounded weights the PV MMA multiplies, so
                    // out is an exact weighted mean of V under those weights (8 accumulators)
                    const int a = (i >> 1) & 7;
                    suma[a] = add_bf16x2_f32(pp, suma[a]);
                    pk[cc * 16 + (i >> 1)] = pp;
                }
            }
            tmem_st32(tS + half * 32, pk);   // over S columns this thread has already read
        }
        if (half == 0 && !rescale && kSplitP) {
            tmem_wait_st();
            tc_fence_before();
            warp_arrive(p_half_bar);
        }
    }
#pragma unroll
    for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
        for (int a = 0; a < w; ++a) suma[a] += suma[a + w];
    l = l * f + suma[0];
    if (!rescale && !kSplitP) {
        tmem_wait_st();
        tc_fence_before();
        warp_arrive(p_half_bar);
    }
    if (rescale) {
        // done once the S row is dead (low register pressure); it must land before this
        // tile's PV, which waits for p_half (arrived below) and p_full.  The previous PV into
        // O has completed: it was issued before this tile's S, whose completion the caller
        // has waited for, and the tensor pipe completes one thread's MMAs in issue order --
        // or, with kWaitO, the wait below has seen it complete.
        if constexpr (kWaitO) (void)warp_wait(o_bar, o_parity, flag);
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
        tc_fence_before();
        warp_arrive(p_half_bar);
    }
    tmem_wait_st();
    tc_fence_before();
}

// Write one output row (32 columns at a time from registers), bf16 or fp32.
template <int D>
__device__ __forceinline__ void store_row_chunk(void* out, int out_f32, size_t orow, int c,
                                                const uint32_t (&o)[32], float scale) {
    if (out_f32) {
        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out) + orow * D + c * 32);
#pragma unroll
        for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(__uint_as_float(o[4 * i]) * scale, __uint_as_float(o[4 * i + 1]) * scale,
                                 __uint_as_float(o[4 * i + 2]) * scale, __uint_as_float(o[4 * i + 3]) * scale);
    } else {
        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out) + orow * D + c * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(
                pack_bf16x2(__uint_as_float(o[8 * i + 0]) * scale, __uint_as_float(o[8 * i + 1]) * scale),
                pack_bf16x2(__uint_as_float(o[8 * i + 2]) * scale, __uint_as_float(o[8 * i + 3]) * scale),
                pack_bf16x2(__uint_as_float(o[8 * i + 4]) * scale, __uint_as_float(o[8 * i + 5]) * scale),
                pack_bf16x2(__uint_as_float(o[8 * i + 6]) * scale, __uint_as_float(o[8 * i + 7]) * scale));
    }
}

__device__ __forceinline__ void init_barriers(SmemCtl* ctl, int stages) {
    mbar_init(smem_u32(&ctl->q_full), 1);
    mbar_init(smem_u32(&ctl->q_empty), 1);
    for (int s = 0; s < stages; ++s) {
        mbar_init(smem_u32(&ctl->kv_full[s]), 1);
        mbar_init(smem_u32(&ctl->kv_empty[s]), 1);
    }
    for (int q = 0; q < 2; ++q) {
        mbar_init(smem_u32(&ctl->s_full[q]), 1);
        mbar_init(smem_u32(&ctl->p_half[q]), 4);    // one arrival per softmax warp
        mbar_init(smem_u32(&ctl->p_full[q]), 4);
        mbar_init(smem_u32(&ctl->o_full[q]), 1);
        mbar_init(smem_u32(&ctl->o_empty[q]), 4);
    }
    mbar_init(smem_u32(&ctl->drain), 1);
    for (int q = 0; q < 2; ++q)
        for (int b = 0; b < 3; ++b) mbar_init(smem_u32(&ctl->merge_bar[q][b]), 1);
    mbar_init(smem_u32(&ctl->prod_done), 1);
    ctl->abort_flag = 0;
    fence_mbar_init();
}

}  // namespace swattn

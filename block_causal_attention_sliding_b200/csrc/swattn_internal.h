// swattn_internal.h -- shared between the C-ABI host code and the kernel launchers.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "swattn.h"

namespace swattn {

constexpr int kBlockM = 128;       // query rows per Q tile (MMA M)
constexpr int kBlockN = 128;       // keys per K/V tile (MMA N of QK^T, K of PV)
constexpr int kMaxW = 64;          // largest window supported
constexpr int kStateHeaderInts = 16;   // [0] chunks committed, [1] status bits, [2] commit blocks done
constexpr int kMaxShortQ = 128;    // split-K path handles one Q tile per (b, h)
constexpr int kMaxSplits = 64;
constexpr int kMaxPersistentCtas = 160;   // >= SMs of a B200 (148)

// The visibility table: [k, n_segments, N_vis], then 4 ints per segment for up to W + 3
// segments (unused ones -1), then the chunk bitmap row in 3 ints (table_vis_offset):
//   [vis_sink, vis_lo, vis_hi]: vis_sink = 1 iff chunk 0 is visible; bit i of the 64-bit word
//   vis_hi:vis_lo = 1 iff chunk k - 64 + i is visible (bits of chunks before 0 are 0).
// Every visible history chunk is the sink or one of the W <= 64 most recent chunks, so these
// three words fix the whole row vis[k][j], j < k, in constant space however long the stream.
constexpr int kVisWords = 3;
constexpr int kVisSpan = 64;   // chunks covered by the bitmap row's window word
__host__ __device__ inline int table_vis_offset(int W) { return 3 + 4 * (W + 3); }
__host__ __device__ inline int table_ints_for(int W) { return table_vis_offset(W) + kVisWords; }

// Ring slot of committed chunk c with R window slots: the sink (if any) owns slot 0 and window
// chunks rotate through the R slots after it, chunk c taking the slot of chunk c - R.  R = W
// is the plain ring; R = W + 1 keeps one spare slot, so chunk k can be written into the cache
// while its own forward still reads every visible chunk.  -1: the chunk is not kept (R = 0).
__host__ __device__ inline int ring_slot(int c, int R, int sink) {
    if (sink) {
        if (c == 0) return 0;
        return R > 0 ? 1 + (c - 1) % R : -1;
    }
    return R > 0 ? c % R : -1;
}

// Device-side state layout: int32 words at the start of the workspace.
//   state[0] = chunks committed (= index k of the active chunk)
//   state[1] = status bits (SW_STATUS_*)
//   state[2] = blocks of a running chunk-commit copy that have finished (0 between launches)
//   state[kStateHeaderInts ...] = visibility table (table_ints_for(W) entries)

// Everything a launch of the attention kernel needs.  Passed by value as a __grid_constant__
// parameter, so the tensor maps live in parameter space as TMA requires.
struct alignas(64) AttnParams {
    CUtensorMap tm_q;        // Q       [B, n_q, H, d]   dims {d, H, n_q, B}
    CUtensorMap tm_kcur;     // K_cur   [B, T, H, d]     dims {d, H, T, B}
    CUtensorMap tm_vcur;     // V_cur
    CUtensorMap tm_cache_k;  // K ring  [B][H][S][T][d]  dims {d, T, S, H, B}
    CUtensorMap tm_cache_v;
    CUtensorMap tm_cond_k;   // K cond  [B][H][n_cond][d] dims {d, n_cond, H, B}
    CUtensorMap tm_cond_v;
    CUtensorMap tm_qc;       // condition-stream queries [B, n_qc, H, d] (joint forward)
    // the same K maps with boxes of 64 rows (half a key tile), for the CTA-pair kernel
    CUtensorMap tm_kcur_h, tm_cache_kh, tm_cond_kh;
    void* out;               // [B, n_q, H, d] bf16 or f32 (full mode)
    void* out_c;             // [B, n_qc, H, d] (joint forward)
    float* o_part;           // split mode: [splits][B*H][kBlockM][d] unnormalised fp32
    float* ml_part;          // split mode: [splits][B*H][kBlockM][2] (row max log2-scaled, row sum)
    const int32_t* table;    // device visibility table
    int32_t* status;         // device status word
    int B, H, n_q;
    int n_qc;                // condition-stream query rows (0: none); their Q tiles follow the chunk's
    int commit;              // 1: also store K_cur / V_cur into the ring slot of the active chunk
    int qk_fp8;              // 1: Q and K (current, cache, condition) are e4m3, scales folded into scale_log2
    int pv_fp8;              // 1: V (current, cache, condition) is e4m3 and P V runs on kind::f8f6f4
    float out_scale;         // applied with the final normalisation (the e4m3 V's scale; 1 otherwise)
    int ring_R;              // window slots of the ring (for the commit slot)
    int sink;
    int out_f32;
    int splits;              // 0: full mode (normalised output); >= 1: split-K partials
    float scale_log2;        // softmax scale * log2(e)
    // persistent kernel: partials of pieces whose key tiles are cut between CTAs
    float* sk_o;             // [2 * kMaxPersistentCtas slots][2 Q tiles][d][128 rows] fp32
    float* sk_ml;            // [slots][2][128 rows][2] (row max log2-scaled, row sum)
    int32_t* sk_cnt;         // [B*H][sk_pairs][2] arrival counters, zero between launches
    int sk_pairs;            // Q-tile pairs per (b, h) the counters are sized for
};

// kernel launchers (defined in the .cu files)
// CTA-pair three-buffer kernel (d = 128, bf16): `clusters` pairs of CTAs.
cudaError_t launch_pair(const AttnParams& p, int clusters, cudaStream_t stream);
// Pairs of CTAs of that kernel that fit on the device at once (0 if none or on error).
int pair_max_clusters();
cudaError_t launch_table_build(int32_t* state, int W, int R, int sink, int n_cond, int T, int advance,
                               cudaStream_t stream);
cudaError_t launch_state_reset(int32_t* state, int W, int R, int sink, int n_cond, int T,
                               int32_t* counters, long long n_counters, cudaStream_t stream);
// What a table rebuild needs: window, ring slots, sink flag, condition tokens, chunk tokens.
struct TableAdvance {
    int W, R, sink, n_cond, T;
};
// Copy [B, N, H, d] bf16 K and V into [B][H][rows_per_bh][d] regions at row offset
// slot * N (slot from the device counter when `ring` is set, else 0).  With `advance` (ring
// only) the same launch then advances the counter and rebuilds the table (a chunk commit).
cudaError_t launch_relayout(const void* K, const void* V, void* dstK, void* dstV, int B, int N,
                            int H, int d, int rows_per_bh, int ring, int S, int32_t* state, const TableAdvance& ta,
                            int advance, cudaStream_t stream, int k_esz = 2, int v_esz = 2);
// One chunk commit for each of up to kMaxBatch handles (layers) of the same B, T, H, d, in one
// copy launch and one table launch (the per-handle window, sink, slots and counter stay apart).
constexpr int kMaxBatch = 32;
struct AppendBatch {
    const void* K[kMaxBatch];
    const void* V[kMaxBatch];
    void* dstK[kMaxBatch];       // the handle's K cache region [B][H][S * T][d]
    void* dstV[kMaxBatch];
    int32_t* state[kMaxBatch];   // the handle's device state (counter, status, table)
    int R[kMaxBatch], S[kMaxBatch], W[kMaxBatch], sink[kMaxBatch], n_cond[kMaxBatch];
    int n;                       // handles in this launch
};
cudaError_t launch_append_batch(const AppendBatch& a, int B, int T, int H, int d, int k_esz, int v_esz,
                                cudaStream_t stream);

cudaError_t launch_attention(const AttnParams& p, int d, int grid_x, cudaStream_t stream);
cudaError_t launch_persistent(const AttnParams& p, int d, int ctas, cudaStream_t stream);
cudaError_t launch_tri(const AttnParams& p, int d, int ctas, cudaStream_t stream);
cudaError_t launch_split(const AttnParams& p, int d, int splits, cudaStream_t stream);
cudaError_t launch_selftest_timeout(int32_t* status, uint64_t limit_ns, cudaStream_t stream);
cudaError_t launch_combine(const float* o_part, const float* ml_part, void* out, int B, int H,
                           int n_q, int d, int splits, int out_f32, float out_scale, cudaStream_t stream);

// A launch that may begin while the stream's previous kernel finishes (programmatic stream
// serialization).  Only kernels that call griddepcontrol.wait before they touch memory the
// previous kernel may write are launched this way.
template <typename... Params, typename... Args>
inline cudaError_t launch_dependent(void (*kern)(Params...), dim3 grid, dim3 block, size_t smem,
                                    cudaStream_t stream, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

}  // namespace swattn

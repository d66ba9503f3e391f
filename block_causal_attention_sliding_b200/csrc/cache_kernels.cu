// cache_kernels.cu -- the bounded KV cache: visibility/slot table builder and the
// append/evict copy into the ring buffer.
//
// The cache keeps the condition tokens, a pinned first chunk (global sink) and the W most
// recent chunks; a finished chunk's clean K/V are written into it right after the chunk
// completes, so memory and per-chunk work stay constant (agifrontier tutorial "JoyAI-Video-
// Edit：单卡720p 30帧，两步蒸馏攻克流式视频编辑", sections "从双向编辑到分块因果架构的蜕变" and
// "软硬件协同部署"; neurohive review "JoyAI-Video-Edit", section "Чанки и борьба с дрейфом").
#include "swattn_internal.h"

namespace swattn {

// K1: advance the counter (after an append) and write the visibility table of the active
// chunk k: [k, n_segments, N_vis, (kind, chunk_id, slot, n_tokens)...], in the order
// condition, sink, window ascending, current; slots of a ring with R window slots.  One
// thread: a few dozen integers.
__device__ void build_table(int32_t* state, int W, int R, int sink, int n_cond, int T, int advance, int reset) {
    int32_t* tab = state + kStateHeaderInts;
    if (reset) {
        state[0] = 0;
        state[1] = 0;
    }
    int k = state[0];
    if (advance) {
        if (k >= (1 << 30)) {
            state[1] |= SW_STATUS_OVERFLOW;
        } else {
            k += 1;
            state[0] = k;
        }
    }
    const int cap = table_ints_for(W);
    int pos = 3, nseg = 0, nvis = 0;
    auto put = [&](int kind, int chunk, int slot, int n) {
        tab[pos++] = kind; tab[pos++] = chunk; tab[pos++] = slot; tab[pos++] = n;
        ++nseg; nvis += n;
    };
    if (n_cond > 0) put(0, -1, -1, n_cond);
    const int first_win = k - W > 0 ? k - W : 0;
    if (sink && k >= 1 && first_win > 0) put(1, 0, 0, T);      // sink outside the window
    for (int j = first_win; j < k; ++j) put(1, j, ring_slot(j, R, sink), T);
    put(2, k, -1, T);
    tab[0] = k; tab[1] = nseg; tab[2] = nvis;
    for (int i = pos; i < cap; ++i) tab[i] = -1;
}

__global__ void table_build_kernel(int32_t* state, int W, int R, int sink, int n_cond, int T, int advance,
                                   int reset) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    build_table(state, W, R, sink, n_cond, T, advance, reset);
}

cudaError_t launch_table_build(int32_t* state, int W, int R, int sink, int n_cond, int T, int advance,
                               cudaStream_t stream) {
    table_build_kernel<<<1, 32, 0, stream>>>(state, W, R, sink, n_cond, T, advance, 0);
    return cudaGetLastError();
}

__global__ void zero_kernel(int32_t* p, long long n) {
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
        p[i] = 0;
}

cudaError_t launch_state_reset(int32_t* state, int W, int R, int sink, int n_cond, int T,
                               int32_t* counters, long long n_counters, cudaStream_t stream) {
    table_build_kernel<<<1, 32, 0, stream>>>(state, W, R, sink, n_cond, T, 0, 1);
    if (n_counters > 0) {
        const long long blocks = (n_counters + 255) / 256;
        zero_kernel<<<(unsigned)(blocks < 1024 ? blocks : 1024), 256, 0, stream>>>(counters, n_counters);
    }
    return cudaGetLastError();
}

// K2: copy K and V of one chunk from the user layout [B, N, H, d] into the head-major cache
// layout [B][H][rows_per_bh][d] at row offset slot * N.
// One block per kRelayoutRows consecutive token rows (b, t) of K or V (blockIdx.y = 0 / 1): a
// row's H x d values are contiguous in the caller's [B, N, H, d] layout, and head h's d values
// go to row slot * N + t of the (b, h) panel of the destination.  Thread k of the block moves
// 16-byte vector k of every row of its group (head k / vpr, vector k % vpr), looping when H * vpr
// exceeds the block; the group's loads are all issued before the first store, so each thread
// keeps kRelayoutRows reads in flight.  Consecutive threads read consecutive bytes and write
// whole 16-byte pieces of 2d-byte destination rows.  No division in the copy loop (vpr is a
// power of two).
constexpr int kRelayoutRows = 4;

__device__ __forceinline__ void relayout_rows(const uint4* __restrict__ srcK, const uint4* __restrict__ srcV,
                                              uint4* __restrict__ dstK, uint4* __restrict__ dstV, int N,
                                              long long rows, int H, int vpr_log2_k, int vpr_log2_v, int rows_per_bh,
                                              int ring, int R, int sink, int S, int32_t* state) {
    int slot = 0;
    if (ring) {
        slot = ring_slot(state[0], R, sink);
        if (slot < 0) return;                 // W = 0: nothing is kept for this chunk
        if (slot >= S) {                      // cannot happen; recorded, never trapped
            if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0)
                atomicOr(state + 1, SW_STATUS_BAD_SLOT);
            return;
        }
    }
    const uint4* __restrict__ src = blockIdx.y == 0 ? srcK : srcV;
    uint4* __restrict__ dst = blockIdx.y == 0 ? dstK : dstV;
    const int vpr_log2 = blockIdx.y == 0 ? vpr_log2_k : vpr_log2_v;   // K may be e4m3 (half the bytes)
    const int vpr = 1 << vpr_log2;
    const int per_row = H << vpr_log2;
    const long long row_first = (long long)blockIdx.x * kRelayoutRows;   // b * N + t of the group's first row
    size_t drow0[kRelayoutRows];   // destination row of head 0, per row of the group
    bool live[kRelayoutRows];
#pragma unroll
    for (int r = 0; r < kRelayoutRows; ++r) {
        const long long row = row_first + r;
        live[r] = row < rows;
        const int b = (int)(row / N), t = (int)(row - (long long)b * N);
        drow0[r] = (size_t)b * H * rows_per_bh + (size_t)slot * N + t;
    }
    for (int k = threadIdx.x; k < per_row; k += blockDim.x) {
        const int h = k >> vpr_log2, v = k & (vpr - 1);
        uint4 x[kRelayoutRows];
#pragma unroll
        for (int r = 0; r < kRelayoutRows; ++r)
            if (live[r]) x[r] = __ldg(src + (size_t)(row_first + r) * per_row + k);
#pragma unroll
        for (int r = 0; r < kRelayoutRows; ++r)
            if (live[r]) dst[(drow0[r] + (size_t)h * rows_per_bh) * vpr + v] = x[r];
    }
}

__global__ void __launch_bounds__(512) relayout_kernel(const uint4* __restrict__ srcK,
                                                       const uint4* __restrict__ srcV,
                                                       uint4* __restrict__ dstK,
                                                       uint4* __restrict__ dstV, int N, long long rows, int H,
                                                       int vpr_log2_k, int vpr_log2_v, int rows_per_bh, int ring,
                                                       int R, int sink, int S, int32_t* state) {
    relayout_rows(srcK, srcV, dstK, dstV, N, rows, H, vpr_log2_k, vpr_log2_v, rows_per_bh, ring, R, sink, S, state);
}

// Batched commit: blockIdx.z selects the handle; each copies into its own ring slot (from its
// own counter), exactly as relayout_kernel does for one handle.
__global__ void __launch_bounds__(512) relayout_batch_kernel(const __grid_constant__ AppendBatch a, int N,
                                                             long long rows, int H, int vpr_log2_k, int vpr_log2_v,
                                                             int T) {
    const int l = blockIdx.z;
    relayout_rows(static_cast<const uint4*>(a.K[l]), static_cast<const uint4*>(a.V[l]), static_cast<uint4*>(a.dstK[l]),
                  static_cast<uint4*>(a.dstV[l]), N, rows, H, vpr_log2_k, vpr_log2_v, a.S[l] * T, 1, a.R[l], a.sink[l],
                  a.S[l], a.state[l]);
}

// Batched table advance: block l advances handle l's counter and rebuilds its table.
__global__ void table_build_batch_kernel(const __grid_constant__ AppendBatch a, int T) {
    const int l = blockIdx.x;
    if (threadIdx.x != 0 || l >= a.n) return;
    build_table(a.state[l], a.W[l], a.R[l], a.sink[l], a.n_cond[l], T, 1, 0);
}

// 16-byte vectors per head row of d elements of esz bytes, as a power of two (-1: not one).
static int vpr_log2_of(int d, int esz) {
    const int vpr = d * esz / 16;
    int l = 0;
    while ((1 << l) < vpr) ++l;
    return (vpr >= 1 && (1 << l) == vpr) ? l : -1;
}

cudaError_t launch_append_batch(const AppendBatch& a, int B, int T, int H, int d, int k_esz, cudaStream_t stream) {
    if (a.n < 1 || a.n > kMaxBatch) return cudaErrorInvalidValue;
    const int vpr_log2 = vpr_log2_of(d, 2), vpr_log2_k = vpr_log2_of(d, k_esz);
    if (vpr_log2 < 0 || vpr_log2_k < 0) return cudaErrorInvalidValue;
    const int vpr = 1 << vpr_log2;
    const long long rows = (long long)B * T;
    if (rows < 1 || rows > 0x7fffffffLL) return cudaErrorInvalidValue;
    const int per_row = H * vpr;
    const int threads = per_row >= 512 ? 512 : ((per_row + 31) / 32) * 32;
    // handles without a ring (S = 0) return at once inside the kernel (slot -1)
    const long long groups = (rows + kRelayoutRows - 1) / kRelayoutRows;
    relayout_batch_kernel<<<dim3((unsigned)groups, 2, (unsigned)a.n), threads, 0, stream>>>(a, T, rows, H, vpr_log2_k,
                                                                                            vpr_log2, T);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    table_build_batch_kernel<<<a.n, 32, 0, stream>>>(a, T);
    return cudaGetLastError();
}

cudaError_t launch_relayout(const void* K, const void* V, void* dstK, void* dstV, int B, int N,
                            int H, int d, int rows_per_bh, int ring, int R, int sink, int S,
                            int32_t* state, cudaStream_t stream, int k_esz) {
    const int vpr_log2 = vpr_log2_of(d, 2), vpr_log2_k = vpr_log2_of(d, k_esz);   // 16-byte vectors per row
    if (vpr_log2 < 0 || vpr_log2_k < 0) return cudaErrorInvalidValue;              // d is 64 or 128
    const int vpr = 1 << vpr_log2;
    const long long rows = (long long)B * N;
    if (rows < 1) return cudaSuccess;
    if (rows > 0x7fffffffLL) return cudaErrorInvalidValue;
    const int per_row = H * vpr;
    const int threads = per_row >= 512 ? 512 : ((per_row + 31) / 32) * 32;
    dim3 grid((unsigned)((rows + kRelayoutRows - 1) / kRelayoutRows), 2);
    relayout_kernel<<<grid, threads, 0, stream>>>(
        static_cast<const uint4*>(K), static_cast<const uint4*>(V), static_cast<uint4*>(dstK),
        static_cast<uint4*>(dstV), N, rows, H, vpr_log2_k, vpr_log2, rows_per_bh, ring, R, sink, S, state);
    return cudaGetLastError();
}

}  // namespace swattn

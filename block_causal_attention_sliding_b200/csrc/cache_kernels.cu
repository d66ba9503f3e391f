// cache_kernels.cu -- the bounded KV cache: visibility/slot table builder and the
// append/evict copy into the ring buffer.
//
// The cache keeps the condition tokens, a pinned first chunk (global sink) and the W most
// recent chunks; a finished chunk's clean K/V are written into it right after the chunk
// completes, so memory and per-chunk work stay constant (agifrontier tutorial "JoyAI-Video-
// Edit：单卡720p 30帧，两步蒸馏攻克流式视频编辑", sections "从双向编辑到分块因果架构的蜕变" and
// "软硬件协同部署"; neurohive review "JoyAI-Video-Edit", section "Чанки и борьба с дрейфом").
#include "commit_copy.h"
#include "ptx.cuh"

namespace swattn {

// K1: advance the counter (after an append) and write the visibility table of the active
// chunk k: [k, n_segments, N_vis, (kind, chunk_id, slot, n_tokens)...], in the order
// condition, sink, window ascending, current; slots of a ring with R window slots; then the
// chunk bitmap row (see table_vis_offset).  One thread: a few dozen integers.  Also compiled
// for the host, where sw_attn_table_host runs it for the tests.
__host__ __device__ void build_table(int32_t* state, int W, int R, int sink, int n_cond, int T, int advance,
                                     int reset) {
    int32_t* tab = state + kStateHeaderInts;
    if (reset) {
        state[0] = 0;
        state[1] = 0;
        state[2] = 0;
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
    const int cap = table_vis_offset(W);
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
    // the chunk bitmap row vis[k][j] = [j in Hist(k)], j < k, in its constant-size form
    uint32_t w[2] = {0u, 0u};
    for (int i = 0; i < kVisSpan; ++i) {
        const int j = k - kVisSpan + i;
        if (j >= 0 && (j >= first_win || (sink && j == 0))) w[i >> 5] |= 1u << (i & 31);
    }
    tab[cap + 0] = (k >= 1 && (sink || first_win == 0)) ? 1 : 0;
    tab[cap + 1] = (int32_t)w[0];
    tab[cap + 2] = (int32_t)w[1];
}

}  // namespace swattn

// Host hook: the state header and table that build_table writes for active chunk k (after an
// advance if `advance`), run on the host with the device's own code.
extern "C" int sw_attn_table_host(int k, int W, int R, int sink, int n_cond, int T, int advance, int32_t* out,
                                  int cap) {
    if (!out || k < 0 || W < 0 || W > 64 || (R != W && R != W + 1) || (W == 0 && R != 0) ||
        (sink != 0 && sink != 1) || n_cond < 0 || T < 1 || (advance != 0 && advance != 1))
        return SW_EINVAL;
    const int n = swattn::kStateHeaderInts + swattn::table_ints_for(W);
    if (cap < n) return SW_ESHAPE;
    for (int i = 0; i < n; ++i) out[i] = 0;
    out[0] = k;
    swattn::build_table(out, W, R, sink, n_cond, T, advance, 0);
    return n;
}

namespace swattn {

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
// whole 16-byte pieces of d-element destination rows.  No division in the copy loop (vpr is a
// power of two).  Measured on B200 at 720p (78 MB moved): 20.5 us per commit; neither a single
// balanced wave of blocks nor two or eight rows per block did better.
constexpr int kRelayoutRows = 4;

// Destination slot of a chunk commit from the counter (-1: nothing to copy).  Every thread reads
// the counter itself: its data loads do not depend on the slot and are issued meanwhile (a
// block-wide broadcast of the slot would hold them back behind the counter's latency).
__device__ __forceinline__ int commit_slot(int32_t* state, int R, int sink, int S) {
    const int slot = ring_slot(state[0], R, sink);
    if (slot < 0) return -1;   // W = 0: nothing is kept for this chunk
    if (slot >= S) {           // cannot happen; recorded, never trapped
        if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) atomicOr(state + 1, SW_STATUS_BAD_SLOT);
        return -1;
    }
    return slot;
}

// The copy of one group of token rows into row offset slot * N of the destination panels; with
// state, the slot comes from the counter (a chunk commit), else it is 0 (the condition region).
__device__ __forceinline__ void relayout_rows(const uint4* __restrict__ srcK, const uint4* __restrict__ srcV,
                                              uint4* __restrict__ dstK, uint4* __restrict__ dstV, int N,
                                              long long rows, int H, int vpr_log2_k, int vpr_log2_v, int rows_per_bh,
                                              int32_t* state, int R, int sink, int S) {
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
        drow0[r] = (size_t)b * H * rows_per_bh + t;
    }
    for (int k = threadIdx.x; k < per_row; k += blockDim.x) {
        const int h = k >> vpr_log2, v = k & (vpr - 1);
        uint4 x[kRelayoutRows];
#pragma unroll
        for (int r = 0; r < kRelayoutRows; ++r)
            if (live[r]) x[r] = __ldg(src + (size_t)(row_first + r) * per_row + k);
        const int slot = state ? commit_slot(state, R, sink, S) : 0;
        if (slot < 0) return;
        const size_t off = (size_t)slot * N + (size_t)h * rows_per_bh;
#pragma unroll
        for (int r = 0; r < kRelayoutRows; ++r)
            if (live[r]) dst[(drow0[r] + off) * vpr + v] = x[r];
    }
}

// After a chunk commit's copy: the last block of the (handle's) grid to finish advances the
// counter and rebuilds the table, so one launch does both.  A thread's read of the counter is
// complete before the barrier below (its value decided the thread's stores, or its return), so
// every block has read the counter before it is counted; state[2] counts the finished blocks and
// is back at zero when the launch ends.
// blocks: the blocks of this handle's grid (all of the launch unless a batch gives each handle
// a part of it).
__device__ __forceinline__ void advance_after_commit(int32_t* state, const TableAdvance& ta, unsigned blocks = 0) {
    __syncthreads();
    if (threadIdx.x != 0) return;
    __threadfence();
    const unsigned total = blocks ? blocks : gridDim.x * gridDim.y;
    const unsigned done = atomicAdd(reinterpret_cast<unsigned*>(state + 2), 1u) + 1u;
    if (done == total) {
        __threadfence();
        build_table(state, ta.W, ta.R, ta.sink, ta.n_cond, ta.T, 1, 0);
        state[2] = 0;
    }
}

// ring = 0: the condition region (offset 0, no counter).  ring = 1: a chunk commit into the slot
// the counter names; with `advance` the launch then also advances the counter and the table.
__global__ void __launch_bounds__(512) relayout_kernel(const uint4* __restrict__ srcK,
                                                       const uint4* __restrict__ srcV,
                                                       uint4* __restrict__ dstK,
                                                       uint4* __restrict__ dstV, int N, long long rows, int H,
                                                       int vpr_log2_k, int vpr_log2_v, int rows_per_bh, int ring,
                                                       int S, int32_t* state, TableAdvance ta, int advance) {
    relayout_rows(srcK, srcV, dstK, dstV, N, rows, H, vpr_log2_k, vpr_log2_v, rows_per_bh, ring ? state : nullptr,
                  ta.R, ta.sink, S);
    if (advance) advance_after_commit(state, ta);
}

// Batched commit: blockIdx.z selects the handle; each copies into its own ring slot (from its
// own counter) and advances its own table, exactly as relayout_kernel does for one handle.
__global__ void __launch_bounds__(512) relayout_batch_kernel(const __grid_constant__ AppendBatch a, int N,
                                                             long long rows, int H, int vpr_log2_k, int vpr_log2_v,
                                                             int T) {
    const int l = blockIdx.z;
    const TableAdvance ta{a.W[l], a.R[l], a.sink[l], a.n_cond[l], T};
    if (a.S[l] > 0)
        relayout_rows(static_cast<const uint4*>(a.K[l]), static_cast<const uint4*>(a.V[l]),
                      static_cast<uint4*>(a.dstK[l]), static_cast<uint4*>(a.dstV[l]), N, rows, H, vpr_log2_k,
                      vpr_log2_v, a.S[l] * T, a.state[l], ta.R, ta.sink, a.S[l]);
    advance_after_commit(a.state[l], ta);
}

// K2 with the tensor-memory accelerator: a chunk commit as TMA bulk copies.  The source map
// reads the caller's [B, T, H, d] K (or V) with its dimensions ordered {d, t, h, b}, so one box
// of kCommitRows token rows x h_box heads x d lands in shared memory as [head][row][d] --
// exactly the layout of the same box of the head-major cache map {d, T, S, H, B}.  Each item
// (K or V, stream, row group, head group) is one TMA load and one TMA store from the same
// buffer; rows and heads past the ends read as zero and are not stored.  Both maps are
// unswizzled (no thread reads the buffers).  One thread per CTA (one CTA per SM) streams its
// contiguous share of the items through kCommitBufs buffers (up to 256 B x 4 rows x 24 heads =
// 24 KB each), refilling a buffer once the store issued from it one item earlier has read it, so
// the other loads stay in flight.  Every wait is bounded; on a timeout the status word records
// it and the thread still drains what it issued.

__device__ __forceinline__ void bulk_wait_read_1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }

struct CommitItems {
    int B, T, H, nt, nh;   // streams, rows, heads, row groups, head groups
    __device__ long long per_kv() const { return (long long)B * nt * nh; }
    __device__ long long total() const { return 2 * per_kv(); }
    // item -> (K or V, stream, first row, first head)
    __device__ void decode(long long i, int& kv, int& b, int& t0, int& h0) const {
        kv = i >= per_kv();
        if (kv) i -= per_kv();
        const int hg = (int)(i % nh);
        i /= nh;
        const int tg = (int)(i % nt);
        b = (int)(i / nt);
        t0 = tg * kCommitRows;
        h0 = hg * kCommitHeads;
    }
};

// One handle's commit: part `part` of `parts` of its items, by thread 0 of the block.
__device__ __forceinline__ void commit_tma_part(const CommitMaps& m, const CommitItems& it, int box_k, int box_v,
                                                int32_t* state, const TableAdvance& ta, int S, int part, int parts) {
    const int box_bytes = box_k > box_v ? box_k : box_v;   // buffer stride (K may be e4m3)
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t full[kCommitBufs];
    if (threadIdx.x == 0) {
        const int slot = commit_slot(state, ta.R, ta.sink, S);
        const long long total = it.total();
        const long long i0 = slot >= 0 ? (long long)part * total / parts : 0;
        const long long i1 = slot >= 0 ? (long long)(part + 1) * total / parts : 0;
        for (int q = 0; q < kCommitBufs; ++q) mbar_init(smem_u32(&full[q]), 1);
        fence_mbar_init();
        auto load = [&](long long i) {
            int kv, b, t0, h0;
            it.decode(i, kv, b, t0, h0);
            const int q = (int)((i - i0) % kCommitBufs);
            const uint32_t bar = smem_u32(&full[q]);
            mbar_arrive_expect_tx(bar, kv ? box_v : box_k);
            tma_load_4d(smem_u32(base + (size_t)q * box_bytes), kv ? &m.src_v : &m.src_k, bar, 0, t0, h0, b);
        };
        for (long long i = i0; i < i1 && i < i0 + kCommitBufs; ++i) load(i);
        int never = 0;
        long long done = i0;   // items whose load has been waited for
        for (long long i = i0; i < i1; ++i, ++done) {
            const long long k = i - i0;
            if (!mbar_wait(smem_u32(&full[k % kCommitBufs]), (uint32_t)((k / kCommitBufs) & 1), &never,
                           1000000000ull)) {
                atomicOr(state + 1, SW_STATUS_TIMEOUT);
                break;
            }
            int kv, b, t0, h0;
            it.decode(i, kv, b, t0, h0);
            fence_proxy_async_smem();
            tma_store_5d(kv ? &m.dst_v : &m.dst_k, smem_u32(base + (size_t)(k % kCommitBufs) * box_bytes), 0, t0, slot,
                         h0, b);
            bulk_commit_group();
            // the buffer of item i - 1 takes item i - 1 + kCommitBufs once that item's store has
            // read it (the store just issued may still be reading its own buffer)
            if (k >= 1 && i - 1 + kCommitBufs < i1) {
                bulk_wait_read_1();
                load(i - 1 + kCommitBufs);
            }
        }
        // loads issued but not waited for (only after a timeout): let them land, boundedly
        // (the prologue issued items i0 .. i0 + kCommitBufs - 1; iteration i, once done, issued item
        // i - 1 + kCommitBufs)
        long long issued = done == i0 ? i0 + kCommitBufs : done + kCommitBufs - 1;
        if (issued > i1) issued = i1;
        for (long long i = done; i < issued; ++i) {
            const long long k = i - i0;
            (void)mbar_wait(smem_u32(&full[k % kCommitBufs]), (uint32_t)((k / kCommitBufs) & 1), &never, 1000000000ull);
        }
        bulk_wait_all();   // every store complete before the buffers go away
    }
}

__global__ void __launch_bounds__(32, 1) commit_tma_kernel(const __grid_constant__ CommitMaps m, CommitItems it,
                                                           int box_k, int box_v, int32_t* state, TableAdvance ta,
                                                           int S) {
    // launched as a programmatic dependent: nothing the previous kernel may touch (the caller's
    // K/V, the ring, the counter, the table) is read or written before it has completed; the
    // next kernel may be scheduled at once, it waits for this grid's completion itself
    grid_dependency_wait();
    grid_dependents_launch();
    commit_tma_part(m, it, box_k, box_v, state, ta, S, blockIdx.x, gridDim.x);
    advance_after_commit(state, ta);
}

// The chunk commit of several handles (layers) in one launch: blockIdx.y selects the handle,
// whose gridDim.x blocks split its items; each handle's last block advances its own counter and
// table, exactly as commit_tma_kernel does for one handle.
__global__ void __launch_bounds__(32, 1) commit_tma_batch_kernel(const __grid_constant__ CommitBatch cb,
                                                                 CommitItems it, int box_k, int box_v) {
    grid_dependency_wait();
    grid_dependents_launch();
    const int l = blockIdx.y;
    commit_tma_part(cb.maps[l], it, box_k, box_v, cb.state[l], cb.ta[l], cb.S[l], blockIdx.x, gridDim.x);
    advance_after_commit(cb.state[l], cb.ta[l], gridDim.x);
}

// 16-byte vectors per head row of d elements of esz bytes, as a power of two (-1: not one).
static int vpr_log2_of(int d, int esz) {
    const int vpr = d * esz / 16;
    int l = 0;
    while ((1 << l) < vpr) ++l;
    return (vpr >= 1 && (1 << l) == vpr) ? l : -1;
}

cudaError_t launch_append_batch(const AppendBatch& a, int B, int T, int H, int d, int k_esz, int v_esz,
                                cudaStream_t stream) {
    if (a.n < 1 || a.n > kMaxBatch) return cudaErrorInvalidValue;
    const int vpr_log2 = vpr_log2_of(d, v_esz), vpr_log2_k = vpr_log2_of(d, k_esz);
    if (vpr_log2 < 0 || vpr_log2_k < 0) return cudaErrorInvalidValue;
    const int vpr = 1 << (vpr_log2 > vpr_log2_k ? vpr_log2 : vpr_log2_k);   // the wider of K and V rows
    const long long rows = (long long)B * T;
    if (rows < 1 || rows > 0x7fffffffLL) return cudaErrorInvalidValue;
    const int per_row = H * vpr;
    const int threads = per_row >= 512 ? 512 : ((per_row + 31) / 32) * 32;
    // handles without a ring (S = 0) copy nothing and only advance their tables
    const long long groups = (rows + kRelayoutRows - 1) / kRelayoutRows;
    relayout_batch_kernel<<<dim3((unsigned)groups, 2, (unsigned)a.n), threads, 0, stream>>>(a, T, rows, H, vpr_log2_k,
                                                                                            vpr_log2, T);
    return cudaGetLastError();
}

cudaError_t launch_relayout(const void* K, const void* V, void* dstK, void* dstV, int B, int N,
                            int H, int d, int rows_per_bh, int ring, int S, int32_t* state, const TableAdvance& ta,
                            int advance, cudaStream_t stream, int k_esz, int v_esz) {
    const int vpr_log2 = vpr_log2_of(d, v_esz), vpr_log2_k = vpr_log2_of(d, k_esz);   // 16-byte vectors per row
    if (vpr_log2 < 0 || vpr_log2_k < 0) return cudaErrorInvalidValue;                  // d is 64 or 128
    const int vpr = 1 << (vpr_log2 > vpr_log2_k ? vpr_log2 : vpr_log2_k);   // the wider of K and V rows
    const long long rows = (long long)B * N;
    if (rows < 1 || rows > 0x7fffffffLL || (advance && !ring)) return cudaErrorInvalidValue;
    const int per_row = H * vpr;
    const int threads = per_row >= 512 ? 512 : ((per_row + 31) / 32) * 32;
    dim3 grid((unsigned)((rows + kRelayoutRows - 1) / kRelayoutRows), 2);
    relayout_kernel<<<grid, threads, 0, stream>>>(
        static_cast<const uint4*>(K), static_cast<const uint4*>(V), static_cast<uint4*>(dstK),
        static_cast<uint4*>(dstV), N, rows, H, vpr_log2_k, vpr_log2, rows_per_bh, ring, S, state, ta, advance);
    return cudaGetLastError();
}

cudaError_t launch_commit_tma_batch(const CommitBatch& cb, int B, int T, int H, int d, int k_esz, int v_esz,
                                    int ctas_per_handle, cudaStream_t stream) {
    if (cb.n < 1 || cb.n > kCommitBatch || B < 1 || T < 1 || H < 1 || ctas_per_handle < 1 || (d * k_esz) % 16 != 0 ||
        (d * v_esz) % 16 != 0 || d * 2 > 256)
        return cudaErrorInvalidValue;
    CommitItems it;
    it.B = B;
    it.T = T;
    it.H = H;
    it.nt = (T + kCommitRows - 1) / kCommitRows;
    it.nh = (H + kCommitHeads - 1) / kCommitHeads;
    const int h_box = H < kCommitHeads ? H : kCommitHeads;
    const int box_k = d * k_esz * kCommitRows * h_box, box_v = d * v_esz * kCommitRows * h_box;
    const int smem = kCommitBufs * (box_k > box_v ? box_k : box_v) + 1024;
    cudaError_t e = cudaFuncSetAttribute(commit_tma_batch_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    return launch_dependent(commit_tma_batch_kernel, dim3(ctas_per_handle, cb.n), dim3(32), (size_t)smem, stream, cb,
                            it, box_k, box_v);
}

cudaError_t launch_commit_tma(const CommitMaps& maps, int B, int T, int H, int d, int k_esz, int v_esz,
                              int32_t* state, const TableAdvance& ta, int S, int ctas, cudaStream_t stream) {
    if (B < 1 || T < 1 || H < 1 || ctas < 1 || (d * k_esz) % 16 != 0 || (d * v_esz) % 16 != 0 || d * 2 > 256)
        return cudaErrorInvalidValue;
    CommitItems it;
    it.B = B;
    it.T = T;
    it.H = H;
    it.nt = (T + kCommitRows - 1) / kCommitRows;
    it.nh = (H + kCommitHeads - 1) / kCommitHeads;
    const int h_box = H < kCommitHeads ? H : kCommitHeads;
    const int box_k = d * k_esz * kCommitRows * h_box, box_v = d * v_esz * kCommitRows * h_box;
    const int smem = kCommitBufs * (box_k > box_v ? box_k : box_v) + 1024;
    cudaError_t e = cudaFuncSetAttribute(commit_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    return launch_dependent(commit_tma_kernel, dim3(ctas), dim3(32), (size_t)smem, stream, maps, it, box_k, box_v,
                            state, ta, S);
}

}  // namespace swattn

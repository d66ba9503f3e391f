/*
 * swattn.h -- C ABI of libswattn: streaming block-causal sink + sliding-window attention
 * for NVIDIA B200 (sm_100a).
 *
 * What is computed.  A chunk-wise autoregressive video diffusion transformer splits the
 * stream into aligned chunks (one latent frame = 8 video frames; source and target tokens);
 * attention is bidirectional inside a chunk and causal across chunks, and the active chunk
 * sees only a fixed window of the W most recent history chunks plus the first chunk, kept
 * permanently as a global sink (agifrontier tutorial "JoyAI-Video-Edit：单卡720p 30帧，
 * 两步蒸馏攻克流式视频编辑", section "从双向编辑到分块因果架构的蜕变"; neurohive review
 * "JoyAI-Video-Edit", section "Чанки и борьба с дрейфом").  Condition tokens from the MLLM
 * encoder are always-visible keys (neurohive, section "Архитектура JoyAI-Video-Edit").  After
 * a chunk finishes, its clean K/V are written to the cache, which keeps "global sink + sliding
 * local window" so memory and time stay flat (tutorial, section "软硬件协同部署").
 *
 * For active chunk k (= number of chunks committed so far), per stream b and head h:
 *   Hist(k) = { j : max(0, k-W) <= j <= k-1 }  U  ({0} if sink and k >= 1)
 *   keys    = [condition tokens ; chunks of Hist(k) ; the current chunk's K_cur]
 *   out[i]  = softmax_j(scale * q_i . k_j) . V        over those keys only
 * The result is exact masked softmax attention; the cache only decides which keys exist.
 *
 * Conventions for every call:
 *   - Tensors are device memory allocated by the caller (e.g. PyTorch), bf16, contiguous,
 *     in the user layout [B, N, H, d] (N = tokens), 16-byte aligned.  The library never
 *     takes ownership of them; the caller keeps them alive until the stream has run the work.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).  Calls only
 *     enqueue work on it and never synchronise, except sw_attn_get_status.
 *   - Return value 0 on success, a negative SW_E* code otherwise; sw_attn_last_error()
 *     then returns a message (thread-local, valid until the next call on that thread).
 *   - Problems found on the device (a wait that ran out, an impossible slot) set bits in a
 *     status word on the device; kernels never trap.  Read it with sw_attn_get_status.
 *   - One handle holds one layer's cache.  Calls on one handle must be ordered on one stream
 *     and made from one host thread at a time (the handle keeps host-side state: the tensor
 *     maps of the last inputs, reused while their pointers and row counts repeat).
 *   - Every call checks its handle against the library's set of live handles: a null,
 *     destroyed or never-created handle gives SW_EINVAL (0 from the size queries) and is never
 *     dereferenced.  A later create may be given a destroyed handle's address, and the check
 *     cannot tell the two apart, so a destroyed handle must still not be used.
 */
#ifndef SWATTN_H
#define SWATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SW_API __attribute__((visibility("default")))
#else
#define SW_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct sw_attn sw_attn_t;   /* opaque handle, created and destroyed by the caller */

/* return codes */
#define SW_OK       0
#define SW_EINVAL  (-1)   /* null, destroyed or unknown handle; null pointer, bad enum, bad number */
#define SW_ESHAPE  (-2)   /* unsupported or inconsistent size */
#define SW_EALIGN  (-3)   /* pointer or size not aligned as required */
#define SW_ESTATE  (-4)   /* call not valid in the handle's state (no workspace, no cond) */
#define SW_ECUDA   (-5)   /* a CUDA runtime or driver call failed */

/* device status bits (sw_attn_get_status) */
#define SW_STATUS_TIMEOUT    0x1   /* a bounded wait inside a kernel ran out; output invalid */
#define SW_STATUS_BAD_SLOT   0x2   /* slot index out of range (never expected) */
#define SW_STATUS_OVERFLOW   0x4   /* chunk counter overflow */

/* output dtypes */
#define SW_OUT_BF16 0
#define SW_OUT_F32  1

typedef struct {
    int   B;                 /* independent streams (batch), >= 1 */
    int   H;                 /* heads, >= 1 */
    int   d;                 /* head dim: 64 or 128 */
    int   tokens_per_chunk;  /* T = source + target tokens of one chunk, >= 1 */
    int   W;                 /* window: most recent history chunks kept, 0..64 */
    int   n_cond;            /* condition tokens (always visible), >= 0 */
    int   sink;              /* 1: chunk 0 is pinned as the global sink */
    int   out_dtype;         /* SW_OUT_BF16 or SW_OUT_F32 */
    float scale;             /* softmax scale; <= 0 selects 1/sqrt(d) */
    int   max_short_q;       /* n_q <= this uses the split-K path; 0 selects 128, max 128,
                                negative disables the split-K path */
    int   schedule;          /* full path: SW_SCHED_AUTO (default), SW_SCHED_PERSISTENT,
                                SW_SCHED_GRID, SW_SCHED_TRI or SW_SCHED_PAIR */
    int   commit_in_forward; /* 1: keep one spare window slot (W + 1 in all) so that
                                sw_attn_forward_commit can write the chunk's K/V into the cache
                                while its own forward runs; 0 (default): W window slots */
    int   qk_fp8;            /* 1: queries and keys are e4m3 (OCP FP8, 1 byte per element): Q,
                                Q_cond, K_cur, the appended K and K_cond are e4m3 tensors of
                                the same [B, N, H, d] shape, the K cache is kept in e4m3 (half
                                the bytes) and S = Q K^T runs on kind::f8f6f4; V stays bf16
                                unless pv_fp8 is set.
                                Requires d = 128; full path on the persistent or three-buffer
                                schedule (SW_SCHED_GRID and SW_SCHED_PAIR: SW_ESHAPE at create),
                                short queries on the split-K path */
    float q_scale, k_scale;  /* dequantisation scales of the e4m3 Q and K (per tensor; <= 0
                                selects 1): the attention uses q * q_scale and k * k_scale */
    int   commit_path;       /* chunk commits: SW_COMMIT_AUTO (default; TMA bulk copies when
                                the commit gives every SM at least a full ring of 8 items, else
                                the copy kernel), SW_COMMIT_TMA or SW_COMMIT_COPY */
    int   pv_fp8;            /* 1 (requires qk_fp8): V is e4m3 too -- V_cur, the appended V and
                                V_cond are e4m3 tensors of the usual shapes, the V cache is kept in
                                e4m3 (the whole K/V cache at half the bf16 bytes) -- and O = P V
                                runs on kind::f8f6f4 with P quantised to e4m3.  A precision mode of
                                its own: P in e4m3 carries 3 mantissa bits against bf16's 7, so
                                the output's rounding error is about 16x that of bf16 P (a
                                mean-relative error near 2.5e-2 on Gaussian inputs) */
    float v_scale;           /* dequantisation scale of the e4m3 V (per tensor; <= 0 selects 1):
                                the attention uses v * v_scale; applied once to the output */
} sw_attn_config;

/* schedules of the full path */
#define SW_SCHED_PERSISTENT 0   /* one CTA per SM, key tiles cut evenly (stream-K) */
#define SW_SCHED_GRID       1   /* one CTA per 256 query rows of each (b, h) */
#define SW_SCHED_TRI        2   /* one CTA per SM, one 128-row Q tile per unit, three S
                                   accumulators in tensor memory, stream-K leftover */
#define SW_SCHED_AUTO       3   /* per launch: SW_SCHED_TRI when the pairs of 128-row Q tiles
                                   (B * H * ceil(n_q / 256)) are fewer than the SMs, else
                                   SW_SCHED_PERSISTENT (see sw_attn_schedule_for) */
#define SW_SCHED_PAIR       4   /* clusters of two CTAs on two SMs, one 256-row tcgen05 MMA
                                   (cta_group::2) per key tile over two Q tiles, three S
                                   accumulators per SM; d = 128 and bf16 only (SW_ESHAPE
                                   otherwise at create); SW_SCHED_TRI where the device cannot
                                   hold a pair of its CTAs */

/*
 * Create a handle with B = 1, sink on, bf16 output, scale 1/sqrt(d).  Host only: allocates
 * no device memory and makes no CUDA call.  *out receives the handle.
 */
SW_API int sw_attn_create(int H, int d, int tokens_per_chunk, int W, int n_cond, sw_attn_t **out);

/* Same, with every option (see sw_attn_config).  Host only. */
SW_API int sw_attn_create_ex(const sw_attn_config *cfg, sw_attn_t **out);

/*
 * Bytes of device memory the handle needs: the K and V ring caches [B][H][S][T][d] bf16 with
 * S = W + sink slots, the condition K/V [B][H][n_cond][d] bf16, the split-K partials, the
 * chunk counter, the status word and the visibility table.  Constant for the handle's life.
 * Returns 0 for a NULL, destroyed or unknown handle.
 */
SW_API size_t sw_attn_workspace_bytes(const sw_attn_t *h);

/*
 * Give the handle its device memory (allocated and owned by the caller, >= 256-byte aligned,
 * at least sw_attn_workspace_bytes bytes, on the current device).  Enqueues on `stream`:
 * zeroing of the counter and status, and the table build for chunk 0.  Cache contents are
 * left as they are (unused slots are never read).  May be called again to move the handle
 * to new memory; that also resets the stream to chunk 0 and forgets the condition tokens.
 */
SW_API int sw_attn_bind_workspace(sw_attn_t *h, void *dev_ptr, size_t bytes, void *stream);

/*
 * Copy the condition keys and values (each [B, n_cond, H, d] bf16) into the handle's
 * condition region.  Required before the first forward when n_cond > 0; may be called
 * again between chunks (a prompt change).  K_cond/V_cond are read by the enqueued copy.
 */
SW_API int sw_attn_set_cond(sw_attn_t *h, const void *K_cond, const void *V_cond, void *stream);

/*
 * Commit the finished chunk c (c = chunks committed so far, tracked on the device): copy its
 * K and V ([B, T, H, d] bf16) into ring slot slot(c) -- slot 0 for the sink, then slots
 * rotating over the window, each new chunk evicting the one that leaves the window -- then
 * advance the counter and rebuild the visibility table.  With W = 0 the copy of chunks c >= 1
 * is skipped (only the counter advances).
 */
SW_API int sw_attn_append_chunk(sw_attn_t *h, const void *K, const void *V, void *stream);

/*
 * Attention of the active chunk: Q [B, n_q, H, d], K_cur and V_cur [B, T, H, d] (bf16) and
 * out [B, n_q, H, d] (bf16 or fp32, per the handle's out_dtype).  Keys are the condition
 * tokens, the visible cached chunks and K_cur.  n_q == T is the chunk's full query set;
 * 1 <= n_q <= max_short_q uses the split-K short-query path (queries are the first n_q rows);
 * other n_q in (max_short_q, T] use the full path.  Reads the visibility table on the device.
 */
SW_API int sw_attn_forward(sw_attn_t *h, const void *Q, const void *K_cur, const void *V_cur,
                    void *out, int n_q, void *stream);

/*
 * Commit the finished chunk of n handles at once -- typically the n layers of one model, each
 * with its own cache: the same effect as sw_attn_append_chunk(handles[l], K[l], V[l]) for every
 * l, in one launch (each handle's copy, then its counter and table) instead of one per handle.
 * The copies are TMA bulk copies (16 handles per launch, the SMs split between them) when every
 * handle has a ring and allows TMA commits (commit_path not SW_COMMIT_COPY) and either all force
 * them (SW_COMMIT_TMA) or the batch together gives every SM a full ring of copies; otherwise
 * the copy kernel (32 handles per launch)
 * (the clean-KV cache build of a chunk covers every layer: tutorial, section "软硬件协同部署";
 * neurohive review, section "Откуда берётся 30 FPS").  All handles share B, H, d and T; window,
 * sink, condition count and chunk counter are each handle's own.  K[l], V[l]: [B, T, H, d] bf16.
 * A handle may appear only once (SW_EINVAL).  Forwards of different layers depend on one
 * another through the model and stay separate launches; a whole chunk step (every layer's
 * forwards and this call) can be captured into one CUDA graph, since no call synchronises.
 */
SW_API int sw_attn_append_chunk_batched(sw_attn_t *const *handles, int n, const void *const *K,
                                        const void *const *V, void *stream);

/*
 * Forward of the chunk's last (clean) pass that also commits the chunk: the same result as
 * sw_attn_forward(Q, K_cur, V_cur, out, T) followed by sw_attn_append_chunk(K_cur, V_cur), in
 * one attention launch plus the table update.  The clean K/V of a finished chunk go straight
 * into the cache (tutorial, section "软硬件协同部署"; neurohive review, section "Откуда берётся
 * 30 FPS": the clean-KV cache build is its own 31 ms stage of a chunk).  On the persistent and
 * grid schedules the attention kernel stores the K_cur / V_cur tiles it has already loaded
 * into shared memory to the chunk's ring slot (TMA bulk stores): no second read of K_cur and
 * V_cur from HBM and no separate copy launch.  The slot written is never one this forward
 * reads, because the handle keeps a spare window slot (commit_in_forward = 1, required:
 * SW_ESTATE otherwise).  On the three-buffer schedule the forward is followed by the copy.
 * Q, K_cur, V_cur [B, T, H, d] bf16; out [B, T, H, d].
 * Speed: on B200 this call is SLOWER than sw_attn_forward followed by sw_attn_append_chunk (720p:
 * 0.743 ms against 0.585 + 0.021 ms): the producer that loads the attention's tiles also issues
 * the stores and waits for each store to read a ring stage before refilling it.  Prefer the two
 * calls unless one launch fewer matters more.
 */
SW_API int sw_attn_forward_commit(sw_attn_t *h, const void *Q, const void *K_cur, const void *V_cur,
                                  void *out, void *stream);

/*
 * Joint forward of the chunk's queries and the condition-stream queries, in one launch.
 * In the MM-DiT the condition tokens form a stream of their own next to the video stream
 * (neurohive review "JoyAI-Video-Edit", section "Архитектура JoyAI-Video-Edit": MM-DiT blocks
 * with a condition stream and an image stream); their queries are read here as attending over
 * the same keys as the active chunk's queries -- condition tokens, visible cached chunks and
 * K_cur -- the plainest reading of one joint attention per chunk.
 *   Q        [B, T, H, d] bf16   the chunk's queries (all T rows)
 *   Q_cond   [B, n_cond, H, d]   the condition tokens' queries
 *   K_cur, V_cur [B, T, H, d]    as in sw_attn_forward
 *   out      [B, T, H, d], out_cond [B, n_cond, H, d]   (bf16 or fp32, per out_dtype)
 * Both query sets run through the full path as one set of 128-row Q tiles (the chunk's first,
 * then the condition queries'), so the launch stays full even where n_cond alone would not
 * fill the GPU.  Needs n_cond >= 1 and the condition set (SW_ESHAPE / SW_ESTATE otherwise).
 * A prompt change (tutorial, section "范式重塑：视频交互从“渲染等待”迈向“即拍即得”": prompts
 * adjusted while streaming) is sw_attn_set_cond between chunks; the cached history is kept.
 */
SW_API int sw_attn_forward_joint(sw_attn_t *h, const void *Q, const void *Q_cond, const void *K_cur,
                                 const void *V_cur, void *out, void *out_cond, void *stream);

/*
 * Short-query forward that allocates nothing and uses no workspace scratch.
 *
 * Same result as sw_attn_forward for 1 <= n_q <= 128 (the split-K path), but its split-K
 * partials go to a fixed device array inside this library instead of the handle's workspace.
 * It is for callers that cannot allocate device memory at call time -- code running inside
 * another framework's memory pool or a pre-planned, fixed-footprint serving process -- and
 * want the cache-resident decode path without growing the workspace they hand over.  The
 * paper has no counterpart: this is an interface convenience of this library.
 *
 * Limits and behaviour:
 *   - The fixed array holds 4 Mi floats (16 MiB).  The call uses the same split count as
 *     sw_attn_forward (one key split per SM per (b, h)), so its output equals that call's bit
 *     for bit; the array only limits which shapes are accepted: each split needs
 *     B*H*128*(d+2) floats, and a shape whose splits do not fit is rejected with SW_ESHAPE
 *     (B*H > 252 at d = 128, > 496 at d = 64).  The clamp of the split count to what fits is
 *     a guard for GPUs with more SMs; on a 148-SM B200 it never binds.
 *   - Every GPU that loads the library holds the 16 MiB until the process exits.
 *   - The array is shared by every call in the process and keeps the last call's contents;
 *     every split writes its own partials before the merge reads them, so nothing needs
 *     clearing, but calls that overlap on the GPU (two streams, two threads) race on it.
 *   - The first call on each device looks up the array's device address (with that device
 *     current) and keeps it for the life of the process; make that first call before any
 *     stream capture.  A device reset (cudaDeviceReset) invalidates the kept address: no call
 *     may follow a reset of the device in the same process.
 *   - Calls no cudaMalloc, cudaFree or other allocating routine.  Same argument rules as
 *     sw_attn_forward; the caller's current device must be the workspace's device.
 */
SW_API int sw_attn_forward_short_noalloc(sw_attn_t *h, const void *Q, const void *K_cur,
                                         const void *V_cur, void *out, int n_q, void *stream);

/* Number of int32 entries of the visibility table (3 + 4 * (W + 3) + 3). */
SW_API int sw_attn_table_ints(const sw_attn_t *h);

/*
 * Copy the device visibility table for the active chunk into dev_table (device memory,
 * sw_attn_table_ints entries):
 *   [0..2]  k, n_segments, N_vis;
 *   [3 .. 3 + 4 (W + 3))  per segment (kind, chunk_id, slot, n_tokens), kind 0 = condition,
 *           1 = cached chunk, 2 = current chunk; order: condition, sink, window chunks
 *           ascending, current; unused entries are -1;
 *   [3 + 4 (W + 3) .. + 3)  the chunk bitmap row vis[k][j] = [chunk j is visible], j < k, in
 *           constant size: vis_sink (1 iff chunk 0 is visible), then vis_lo, vis_hi, where bit
 *           i of the 64-bit word vis_hi:vis_lo is vis[k][k - 64 + i] (0 for chunks before 0).
 *           Every other entry of the row is 0: a visible history chunk is the sink or one of
 *           the W <= 64 most recent (tutorial, section "从双向编辑到分块因果架构的蜕变").
 */
SW_API int sw_attn_get_table(const sw_attn_t *h, int32_t *dev_table, void *stream);

/*
 * Byte offsets, inside the bound workspace, of the K and V ring caches ([B][H][S][T][d] bf16,
 * S = W + sink slots; slot 0 holds the sink when it is on).  For inspection and tests.
 */
SW_API int sw_attn_cache_offsets(const sw_attn_t *h, size_t *k_offset, size_t *v_offset);

/*
 * Test hook: the pieces of the full-path schedules, enumerated on the host with the schedule code
 * the kernels run.  schedule: SW_SCHED_PERSISTENT (units are pairs of 128-row Q tiles), SW_SCHED_TRI
 * (units are Q tiles) or SW_SCHED_PAIR (units are pairs of Q tiles, ctas counts CTA pairs); nqt Q
 * tiles and nt key tiles per (b, h), bh = B * H.  Writes up to cap rows of 6 int32 -- CTA (or
 * pair) index, unit (bh-major), first and one-past-last key tile, 1 if from the stream-K phase,
 * Q tiles of the unit that hold queries -- in CTA order and, within a CTA, in processing order.
 * Returns the number of rows, SW_EINVAL for bad arguments, SW_ESHAPE if cap is too small.
 * No device memory is touched.
 */
SW_API int sw_attn_schedule_pieces(int schedule, int nqt, int nt, int bh, int ctas, int32_t *out, int cap);

/*
 * Test hook: the device state the table builder writes, computed on the host with the builder's
 * own code -- the header of 16 int32 ([0] chunks committed, [1] status bits) followed by the
 * visibility table as sw_attn_get_table returns it -- for active chunk k (k + 1 after an advance,
 * advance = 1, as a chunk commit does), a window of W <= 64 chunks kept in R = W or W + 1 window
 * slots (R = 0 when W = 0), sink 0 or 1, n_cond condition tokens and T tokens per chunk.
 * Returns the number of int32 written (16 + sw_attn_table_ints for W), SW_EINVAL for bad
 * arguments, SW_ESHAPE if cap is too small.  No device memory is touched.
 */
SW_API int sw_attn_table_host(int k, int W, int R, int sink, int n_cond, int T, int advance, int32_t *out,
                              int cap);

/*
 * Failure-detection self-test.  Enqueues one tiny kernel that waits on an mbarrier nothing
 * will ever complete, through the same bounded wait every attention kernel uses, with a limit
 * of limit_ns (1e6 .. 2e9 ns) instead of the kernels' 1 s.  When the wait gives up it sets
 * SW_STATUS_TIMEOUT in the device status word and returns; the context stays usable.  Shows
 * that a stalled pipeline ends in an error status rather than a hang.  sw_attn_reset clears it.
 */
SW_API int sw_attn_selftest_timeout(sw_attn_t *h, int64_t limit_ns, void *stream);

/*
 * The schedule a full-path forward of n_q queries runs with on this handle (SW_SCHED_PERSISTENT,
 * SW_SCHED_GRID or SW_SCHED_TRI; SW_SCHED_AUTO resolved as described above).  Host only, no
 * CUDA call.  Returns the schedule, or SW_EINVAL for a null handle or n_q < 1.
 */
SW_API int sw_attn_schedule_for(const sw_attn_t* h, int n_q);

/*
 * How this handle's chunk commits (sw_attn_append_chunk, and the copy after a committing forward
 * on the three-buffer schedule) move K and V into the ring: SW_COMMIT_TMA (TMA bulk copies, one
 * CTA per SM) or SW_COMMIT_COPY (the copy kernel).  Chosen at sw_attn_bind_workspace from the
 * config's commit_path: the copy kernel where the driver declines the TMA maps or the handle has
 * no ring, and under SW_COMMIT_AUTO also for commits too small to fill every SM's ring of 8
 * items (at 480p the copy kernel is faster; at 720p TMA is).  Host only, no CUDA call.  Returns
 * the kind, SW_EINVAL for a null handle, or SW_ESTATE before a workspace is bound.
 */
#define SW_COMMIT_AUTO 0
#define SW_COMMIT_COPY 1
#define SW_COMMIT_TMA 2
SW_API int sw_attn_commit_kind(const sw_attn_t* h);

/* Synchronise the device, then read the device status bits into *host_status. */
SW_API int sw_attn_get_status(sw_attn_t *h, int32_t *host_status);

/* Start a new stream on the same handle: counter and status to 0, table for chunk 0. */
SW_API int sw_attn_reset(sw_attn_t *h, void *stream);

/* Free the handle (host memory only; the workspace stays the caller's).  NULL, an unknown
 * handle and a second destroy of the same handle are ignored. */
SW_API void sw_attn_destroy(sw_attn_t *h);

/* Message for the last failed call on this thread ("" if none). */
SW_API const char *sw_attn_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* SWATTN_H */

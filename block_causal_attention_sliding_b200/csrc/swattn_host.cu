// swattn_host.cu -- the C ABI: argument checks, workspace layout, TMA tensor maps, launches.
//
// Calls only enqueue work on the caller's stream (no synchronisation, no allocation), so a
// chunk step can be captured in a CUDA graph; the chunk counter and the visibility table
// live on the device for the same reason.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <unordered_set>

#include <cudaTypedefs.h>

#include "commit_copy.h"
#include "swattn_internal.h"

using namespace swattn;

struct sw_attn {
    sw_attn_config cfg;
    int S = 0;                 // ring slots = W + sink
    int table_ints = 0;
    int max_splits = 1;
    int short_q = 0;           // n_q <= short_q uses the split-K path (0: never)
    size_t off_kcache = 0, off_vcache = 0, off_kcond = 0, off_vcond = 0, off_opart = 0, off_ml = 0;
    size_t off_sk_o = 0, off_sk_ml = 0, off_sk_cnt = 0;
    int sk_pairs = 0;
    int R = 0;                 // window slots of the ring (W, or W + 1 with commit_in_forward)
    long long n_counters = 0;
    size_t total = 0;
    char* ws = nullptr;
    size_t ws_bytes = 0;
    int device = -1;
    int num_sms = 148;
    bool cond_set = false;
    CUtensorMap tm_cache_k, tm_cache_v, tm_cond_k, tm_cond_v;
    CUtensorMap tm_cache_kh, tm_cond_kh;    // the K maps with 64-row boxes (CTA-pair kernel)
    bool pair_ok = false;                   // bf16, d = 128: the CTA-pair kernel can run
    int pair_clusters = -1;                 // CTA pairs that fit at once (-1: not yet queried)
    CUtensorMap tm_commit_k, tm_commit_v;   // the ring with the TMA commit's box
    bool commit_tma = false;                // chunk commits by TMA bulk copies (else the copy kernel)
    bool commit_maps_ok = false;            // the commit's ring maps exist (a batch may use them)
    // tensor maps over the caller's last Q, Q_cond, K_cur and V_cur: a map depends only on the
    // pointer and the row count (B, H, d and the element size are the handle's), so it is encoded
    // again only when one of them changes
    struct MapMemo {
        const void* ptr = nullptr;
        int rows = -1;
        CUtensorMap map;
    };
    MapMemo memo_q, memo_qc, memo_kcur, memo_vcur;
    MapMemo memo_commit_k, memo_commit_v;   // the same for a TMA commit's source K and V
    MapMemo memo_kcur_h;                    // K_cur with 64-row boxes (CTA-pair kernel)
};

namespace {

thread_local std::string g_err;

int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

int cuda_fail(cudaError_t e, const char* what) {
    return fail(SW_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

// The handles created and not yet destroyed.  Every call checks its handle against this set, so
// a destroyed (or never created) handle is refused instead of dereferenced, and a second destroy
// does nothing.  The check cannot tell a stale handle from a newer one that was given the same
// address by a later create.
std::mutex g_live_mu;
std::unordered_set<const sw_attn*> g_live;

bool live(const sw_attn* h) {
    if (!h) return false;
    std::lock_guard<std::mutex> lk(g_live_mu);
    return g_live.count(h) != 0;
}

int bad_handle(const sw_attn* h) {
    return fail(SW_EINVAL, h ? "unknown or destroyed handle" : "null handle");
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Tiled map, by default with 128-byte swizzle and 128-byte box rows (64 bf16 or 128 e4m3 columns,
// esz = 2 or 1 bytes per element); out-of-range rows read as zero.
int encode(CUtensorMap* m, const void* ptr, int rank, const uint64_t* dims, const uint64_t* strides,
           const uint32_t* box, const char* what, int esz = 2,
           CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
    auto fn = encode_fn();
    if (!fn) return fail(SW_ECUDA, "cuTensorMapEncodeTiled unavailable");
    uint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(m, esz == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank,
                    const_cast<void*>(ptr),
                    reinterpret_cast<const cuuint64_t*>(dims), reinterpret_cast<const cuuint64_t*>(strides),
                    reinterpret_cast<const cuuint32_t*>(box), estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(SW_ECUDA, "tensor map for %s: CUresult %d", what, (int)r);
    return SW_OK;
}

// user layout [B, N, H, d]: dims {d, H, N, B}; box (128 bytes) x 1 x rows x 1 (rows of one head;
// 128 by default, 64 for the CTA-pair kernel's K halves)
int encode_user(CUtensorMap* m, const void* ptr, int B, int N, int H, int d, const char* what, int esz = 2,
                int rows = kBlockN) {
    const uint64_t dims[4] = {(uint64_t)d, (uint64_t)H, (uint64_t)N, (uint64_t)B};
    const uint64_t strides[3] = {(uint64_t)d * esz, (uint64_t)H * d * esz, (uint64_t)N * H * d * esz};
    const uint32_t box[4] = {(uint32_t)(128 / esz), 1, (uint32_t)rows, 1};
    return encode(m, ptr, 4, dims, strides, box, what, esz);
}

// encode_user through a one-entry memo keyed by (pointer, rows).
int encode_user_memo(sw_attn::MapMemo& m, const void* ptr, int B, int N, int H, int d, const char* what, int esz,
                     int box_rows = kBlockN) {
    if (m.ptr == ptr && m.rows == N) return SW_OK;
    m.ptr = nullptr;
    m.rows = -1;
    const int rc = encode_user(&m.map, ptr, B, N, H, d, what, esz, box_rows);
    if (rc) return rc;
    m.ptr = ptr;
    m.rows = N;
    return SW_OK;
}

// The caller's [B, T, H, d] K or V for a TMA chunk commit: dims ordered {d, t, h, b} (strides
// T: H*d, h: d, b: T*H*d elements), box d x kCommitRows rows x min(H, kCommitHeads) heads,
// unswizzled.
int encode_commit_src(CUtensorMap* m, const void* ptr, int B, int T, int H, int d, const char* what, int esz) {
    const uint64_t dims[4] = {(uint64_t)d, (uint64_t)T, (uint64_t)H, (uint64_t)B};
    const uint64_t strides[3] = {(uint64_t)H * d * esz, (uint64_t)d * esz, (uint64_t)T * H * d * esz};
    const uint32_t box[4] = {(uint32_t)d, (uint32_t)kCommitRows, (uint32_t)(H < kCommitHeads ? H : kCommitHeads), 1};
    return encode(m, ptr, 4, dims, strides, box, what, esz, CU_TENSOR_MAP_SWIZZLE_NONE);
}

int check_cfg(const sw_attn_config& c) {
    if (c.B < 1 || c.H < 1) return fail(SW_ESHAPE, "B and H must be >= 1 (B=%d H=%d)", c.B, c.H);
    if (c.d != 64 && c.d != 128) return fail(SW_ESHAPE, "d must be 64 or 128 (d=%d)", c.d);
    if (c.tokens_per_chunk < 1) return fail(SW_ESHAPE, "tokens_per_chunk must be >= 1");
    if (c.W < 0 || c.W > kMaxW) return fail(SW_ESHAPE, "W must be in [0, %d] (W=%d)", kMaxW, c.W);
    if (c.n_cond < 0) return fail(SW_ESHAPE, "n_cond must be >= 0");
    if (c.sink != 0 && c.sink != 1) return fail(SW_EINVAL, "sink must be 0 or 1");
    if (c.out_dtype != SW_OUT_BF16 && c.out_dtype != SW_OUT_F32) return fail(SW_EINVAL, "bad out_dtype");
    if (c.max_short_q > kMaxShortQ) return fail(SW_ESHAPE, "max_short_q must be <= %d", kMaxShortQ);
    if (!std::isfinite(c.scale)) return fail(SW_EINVAL, "scale must be finite");
    if (c.schedule == SW_SCHED_PAIR && (c.d != 128 || c.qk_fp8))
        return fail(SW_ESHAPE, "the CTA-pair schedule needs d = 128 and bf16 Q/K/V");
    if (c.schedule != SW_SCHED_PERSISTENT && c.schedule != SW_SCHED_GRID && c.schedule != SW_SCHED_TRI &&
        c.schedule != SW_SCHED_PAIR &&
        c.schedule != SW_SCHED_AUTO)
        return fail(SW_EINVAL, "bad schedule");
    if (c.commit_in_forward != 0 && c.commit_in_forward != 1) return fail(SW_EINVAL, "commit_in_forward must be 0 or 1");
    if (c.qk_fp8 != 0 && c.qk_fp8 != 1) return fail(SW_EINVAL, "qk_fp8 must be 0 or 1");
    if (c.qk_fp8 && c.d != 128) return fail(SW_ESHAPE, "e4m3 Q/K need d = 128");
    if (c.qk_fp8 && c.schedule == SW_SCHED_GRID) return fail(SW_ESHAPE, "the grid schedule has no e4m3 Q/K form");
    if (!std::isfinite(c.q_scale) || !std::isfinite(c.k_scale)) return fail(SW_EINVAL, "scales must be finite");
    if (c.pv_fp8 != 0 && c.pv_fp8 != 1) return fail(SW_EINVAL, "pv_fp8 must be 0 or 1");
    if (c.pv_fp8 && !c.qk_fp8) return fail(SW_ESHAPE, "pv_fp8 requires qk_fp8 (e4m3 Q and K)");
    if (!std::isfinite(c.v_scale)) return fail(SW_EINVAL, "v_scale must be finite");
    if (c.commit_path != SW_COMMIT_AUTO && c.commit_path != SW_COMMIT_COPY && c.commit_path != SW_COMMIT_TMA)
        return fail(SW_EINVAL, "bad commit_path");
    const double elems = (double)c.B * c.H * (c.W + 2) * c.tokens_per_chunk * c.d;
    if (elems > 4.0e12 || (double)c.tokens_per_chunk * c.H * c.B > 2.0e9 ||
        (double)c.n_cond * c.H * c.B > 2.0e9)
        return fail(SW_ESHAPE, "problem too large");
    return SW_OK;
}

}  // namespace

extern "C" {

const char* sw_attn_last_error(void) { return g_err.c_str(); }

int sw_attn_create_ex(const sw_attn_config* cfg, sw_attn_t** out) {
    g_err.clear();
    if (!cfg || !out) return fail(SW_EINVAL, "null argument");
    *out = nullptr;
    int rc = check_cfg(*cfg);
    if (rc) return rc;
    sw_attn* h = new (std::nothrow) sw_attn();
    if (!h) return fail(SW_EINVAL, "out of host memory");
    h->cfg = *cfg;
    if (h->cfg.scale <= 0.f) h->cfg.scale = 1.0f / std::sqrt((float)cfg->d);
    h->short_q = cfg->max_short_q == 0 ? kMaxShortQ : (cfg->max_short_q < 0 ? 0 : cfg->max_short_q);
    if (h->cfg.q_scale <= 0.f) h->cfg.q_scale = 1.f;
    if (h->cfg.k_scale <= 0.f) h->cfg.k_scale = 1.f;
    if (h->cfg.v_scale <= 0.f) h->cfg.v_scale = 1.f;
    // window slots: W, or W + 1 to keep a spare slot for commits during the chunk's own forward
    h->R = cfg->commit_in_forward && cfg->W > 0 ? cfg->W + 1 : cfg->W;
    h->S = h->R + (cfg->sink ? 1 : 0);
    h->table_ints = table_ints_for(cfg->W);
    const int bh = cfg->B * cfg->H;
    h->max_splits = std::max(1, std::min(kMaxSplits, (148 + bh - 1) / bh));   // B200: 148 SMs
    const size_t B = cfg->B, H = cfg->H, d = cfg->d, T = cfg->tokens_per_chunk;
    size_t off = align_up(sizeof(int32_t) * (kStateHeaderInts + h->table_ints), 1024);
    const size_t ek = cfg->qk_fp8 ? 1 : 2;   // bytes per K element (e4m3 on an FP8 handle)
    const size_t ev = cfg->pv_fp8 ? 1 : 2;   // bytes per V element
    h->off_kcache = off; off = align_up(off + B * H * h->S * T * d * ek, 1024);
    h->off_vcache = off; off = align_up(off + B * H * h->S * T * d * ev, 1024);
    h->off_kcond = off;  off = align_up(off + B * H * cfg->n_cond * d * ek, 1024);
    h->off_vcond = off;  off = align_up(off + B * H * cfg->n_cond * d * ev, 1024);
    h->off_opart = off;
    if (h->short_q > 0) off = align_up(off + (size_t)h->max_splits * bh * kBlockM * d * 4, 1024);
    h->off_ml = off;
    if (h->short_q > 0) off = align_up(off + (size_t)h->max_splits * bh * kBlockM * 2 * 4, 1024);
    // persistent schedule: two partial slots per CTA and one counter per (b, h, pair, Q tile)
    // (a joint forward adds the condition queries' Q tiles after the chunk's)
    h->sk_pairs = ((cfg->tokens_per_chunk + kBlockM - 1) / kBlockM + (cfg->n_cond + kBlockM - 1) / kBlockM + 1) / 2;
    h->n_counters = (long long)bh * h->sk_pairs * 2;
    h->off_sk_o = off;   off = align_up(off + (size_t)2 * kMaxPersistentCtas * 2 * d * kBlockM * 4, 1024);
    h->off_sk_ml = off;  off = align_up(off + (size_t)2 * kMaxPersistentCtas * 2 * kBlockM * 2 * 4, 1024);
    h->off_sk_cnt = off; off = align_up(off + (size_t)h->n_counters * 4, 1024);
    h->total = off;
    {
        std::lock_guard<std::mutex> lk(g_live_mu);
        g_live.insert(h);
    }
    *out = h;
    return SW_OK;
}

int sw_attn_create(int H, int d, int tokens_per_chunk, int W, int n_cond, sw_attn_t** out) {
    sw_attn_config c;
    std::memset(&c, 0, sizeof c);
    c.B = 1; c.H = H; c.d = d; c.tokens_per_chunk = tokens_per_chunk; c.W = W; c.n_cond = n_cond;
    c.sink = 1; c.out_dtype = SW_OUT_BF16; c.scale = 0.f; c.max_short_q = 0; c.schedule = SW_SCHED_AUTO;
    c.commit_in_forward = 0;
    c.qk_fp8 = 0; c.q_scale = 0.f; c.k_scale = 0.f; c.commit_path = SW_COMMIT_AUTO;
    c.pv_fp8 = 0; c.v_scale = 0.f;
    return sw_attn_create_ex(&c, out);
}

size_t sw_attn_workspace_bytes(const sw_attn_t* h) { return live(h) ? h->total : 0; }

int sw_attn_table_ints(const sw_attn_t* h) { return live(h) ? h->table_ints : 0; }

void sw_attn_destroy(sw_attn_t* h) {
    if (!h) return;
    {
        std::lock_guard<std::mutex> lk(g_live_mu);
        if (!g_live.erase(h)) return;   // unknown or already destroyed
    }
    delete h;
}

int sw_attn_bind_workspace(sw_attn_t* h, void* dev_ptr, size_t bytes, void* stream) {
    g_err.clear();
    if (!live(h)) return bad_handle(h);
    if (!dev_ptr) return fail(SW_EINVAL, "null argument");
    if (reinterpret_cast<uintptr_t>(dev_ptr) & 255u) return fail(SW_EALIGN, "workspace must be 256-byte aligned");
    if (bytes < h->total) return fail(SW_ESHAPE, "workspace too small: %zu < %zu", bytes, h->total);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    // the CTA-pair kernel: bf16 with d = 128, and only where pairs of its CTAs fit the device
    h->pair_ok = h->cfg.d == 128 && !h->cfg.qk_fp8 && !h->cfg.pv_fp8;
    h->pair_clusters = h->pair_ok ? pair_max_clusters() : 0;
    const sw_attn_config& c = h->cfg;
    char* ws = static_cast<char*>(dev_ptr);
    int rc;
    if (h->S > 0) {
        // ring [B][H][S][T][d]: dims {d, T, S, H, B}; rows past T read as zero
        const uint64_t dims[5] = {(uint64_t)c.d, (uint64_t)c.tokens_per_chunk, (uint64_t)h->S, (uint64_t)c.H,
                                  (uint64_t)c.B};
        // boxes of 128-byte rows (64 bf16 or 128 e4m3 columns), 128-byte swizzle
        const int ek = c.qk_fp8 ? 1 : 2;   // K in e4m3 on an FP8 handle
        const uint64_t rowk = (uint64_t)c.d * ek;
        const uint64_t stridesk[4] = {rowk, rowk * c.tokens_per_chunk, rowk * c.tokens_per_chunk * h->S,
                                      rowk * c.tokens_per_chunk * h->S * c.H};
        const uint32_t boxk[5] = {(uint32_t)(128 / ek), (uint32_t)kBlockN, 1, 1, 1};
        const int ev = c.pv_fp8 ? 1 : 2;   // V in e4m3 on a pv_fp8 handle
        const uint64_t rowv = (uint64_t)c.d * ev;
        const uint64_t stridesv[4] = {rowv, rowv * c.tokens_per_chunk, rowv * c.tokens_per_chunk * h->S,
                                      rowv * c.tokens_per_chunk * h->S * c.H};
        const uint32_t boxv[5] = {(uint32_t)(128 / ev), (uint32_t)kBlockN, 1, 1, 1};
        if ((rc = encode(&h->tm_cache_k, ws + h->off_kcache, 5, dims, stridesk, boxk, "K cache", ek))) return rc;
        if (h->pair_ok) {
            const uint32_t boxkh[5] = {64u, (uint32_t)(kBlockN / 2), 1, 1, 1};
            if ((rc = encode(&h->tm_cache_kh, ws + h->off_kcache, 5, dims, stridesk, boxkh, "K cache", ek))) return rc;
        }
        if ((rc = encode(&h->tm_cache_v, ws + h->off_vcache, 5, dims, stridesv, boxv, "V cache", ev))) return rc;
        // chunk commits by TMA: the ring with a box of d x kCommitRows rows x up to kCommitHeads
        // heads (unswizzled), and a trial map of the caller side (permuted strides); where the
        // driver declines either, commits use the copy kernel
        const uint32_t hb = (uint32_t)(c.H < kCommitHeads ? c.H : kCommitHeads);
        const uint32_t cbox[5] = {(uint32_t)c.d, (uint32_t)kCommitRows, 1, hb, 1};
        CUtensorMap trial;
        // auto: TMA only when every SM gets at least a full ring of items
        const long long items = 2LL * c.B * ((c.tokens_per_chunk + kCommitRows - 1) / kCommitRows) *
                                ((c.H + kCommitHeads - 1) / kCommitHeads);
        const bool want = c.commit_path == SW_COMMIT_TMA ||
                          (c.commit_path == SW_COMMIT_AUTO && items >= (long long)kCommitBufs * sms);
        // the maps are made whenever TMA commits are allowed: a batched commit of several handles
        // may have enough items together where one handle alone has not
        h->commit_maps_ok = c.commit_path != SW_COMMIT_COPY &&
            encode(&h->tm_commit_k, ws + h->off_kcache, 5, dims, stridesk, cbox, "K cache", ek,
                   CU_TENSOR_MAP_SWIZZLE_NONE) == SW_OK &&
            encode(&h->tm_commit_v, ws + h->off_vcache, 5, dims, stridesv, cbox, "V cache", ev,
                   CU_TENSOR_MAP_SWIZZLE_NONE) == SW_OK &&
            encode_commit_src(&trial, ws + h->off_kcache, c.B, c.tokens_per_chunk, c.H, c.d, "K", ek) == SW_OK;
        h->commit_tma = want && h->commit_maps_ok;
        g_err.clear();
    }
    if (c.n_cond > 0) {
        const uint64_t dims[4] = {(uint64_t)c.d, (uint64_t)c.n_cond, (uint64_t)c.H, (uint64_t)c.B};
        const int ek = c.qk_fp8 ? 1 : 2;
        const uint64_t rowk = (uint64_t)c.d * ek;
        const uint64_t stridesk[3] = {rowk, rowk * c.n_cond, rowk * c.n_cond * c.H};
        const uint32_t boxk[4] = {(uint32_t)(128 / ek), (uint32_t)kBlockN, 1, 1};
        const int ev = c.pv_fp8 ? 1 : 2;
        const uint64_t rowv = (uint64_t)c.d * ev;
        const uint64_t stridesv[3] = {rowv, rowv * c.n_cond, rowv * c.n_cond * c.H};
        const uint32_t boxv[4] = {(uint32_t)(128 / ev), (uint32_t)kBlockN, 1, 1};
        if ((rc = encode(&h->tm_cond_k, ws + h->off_kcond, 4, dims, stridesk, boxk, "K cond", ek))) return rc;
        if (h->pair_ok) {
            const uint32_t boxkh[4] = {64u, (uint32_t)(kBlockN / 2), 1, 1};
            if ((rc = encode(&h->tm_cond_kh, ws + h->off_kcond, 4, dims, stridesk, boxkh, "K cond", ek))) return rc;
        }
        if ((rc = encode(&h->tm_cond_v, ws + h->off_vcond, 4, dims, stridesv, boxv, "V cond", ev))) return rc;
    }
    e = launch_state_reset(reinterpret_cast<int32_t*>(ws), c.W, h->R, c.sink, c.n_cond, c.tokens_per_chunk,
                           reinterpret_cast<int32_t*>(ws + h->off_sk_cnt), h->n_counters,
                           static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "state reset launch");
    h->ws = ws;
    h->ws_bytes = bytes;
    h->device = dev;
    h->num_sms = sms;
    h->cond_set = c.n_cond == 0;
    return SW_OK;
}

int sw_attn_reset(sw_attn_t* h, void* stream) {
    g_err.clear();
    if (!live(h)) return bad_handle(h);
    if (!h->ws) return fail(SW_ESTATE, "no workspace bound");
    const sw_attn_config& c = h->cfg;
    cudaError_t e = launch_state_reset(reinterpret_cast<int32_t*>(h->ws), c.W, h->R, c.sink, c.n_cond,
                                       c.tokens_per_chunk, reinterpret_cast<int32_t*>(h->ws + h->off_sk_cnt),
                                       h->n_counters, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SW_OK : cuda_fail(e, "state reset launch");
}

// The table parameters of a handle, for launches that rebuild its table.
static TableAdvance table_advance(const sw_attn_t* h) {
    const sw_attn_config& c = h->cfg;
    return TableAdvance{c.W, h->R, c.sink, c.n_cond, c.tokens_per_chunk};
}

int sw_attn_set_cond(sw_attn_t* h, const void* K_cond, const void* V_cond, void* stream) {
    g_err.clear();
    if (!live(h)) return bad_handle(h);
    if (!h->ws) return fail(SW_ESTATE, "no workspace bound");
    const sw_attn_config& c = h->cfg;
    if (c.n_cond == 0) return SW_OK;
    if (!K_cond || !V_cond) return fail(SW_EINVAL, "null condition tensor");
    if (!aligned16(K_cond) || !aligned16(V_cond)) return fail(SW_EALIGN, "condition tensors must be 16-byte aligned");
    cudaError_t e = launch_relayout(K_cond, V_cond, h->ws + h->off_kcond, h->ws + h->off_vcond, c.B, c.n_cond,
                                    c.H, c.d, c.n_cond, 0, h->S, reinterpret_cast<int32_t*>(h->ws), table_advance(h),
                                    0, static_cast<cudaStream_t>(stream), c.qk_fp8 ? 1 : 2, c.pv_fp8 ? 1 : 2);
    if (e != cudaSuccess) return cuda_fail(e, "condition copy launch");
    h->cond_set = true;
    return SW_OK;
}

// One chunk commit of K and V ([B, T, H, d]) into the ring slot the device counter names, with
// the counter advance and table rebuild in the same launch: TMA bulk copies (one CTA per SM),
// or the copy kernel where the handle's maps could not be made.
// The four maps of a TMA chunk commit of K, V into h's ring (source maps memoised by pointer).
static int commit_maps(sw_attn_t* h, const void* K, const void* V, CommitMaps& m) {
    const sw_attn_config& c = h->cfg;
    const int ek = c.qk_fp8 ? 1 : 2, ev = c.pv_fp8 ? 1 : 2;
    int rc;
    for (int kv = 0; kv < 2; ++kv) {
        sw_attn::MapMemo& mm = kv ? h->memo_commit_v : h->memo_commit_k;
        const void* src = kv ? V : K;
        if (mm.ptr != src) {
            mm.ptr = nullptr;
            if ((rc = encode_commit_src(&mm.map, src, c.B, c.tokens_per_chunk, c.H, c.d, kv ? "V" : "K", kv ? ev : ek)))
                return rc;
            mm.ptr = src;
        }
    }
    m.src_k = h->memo_commit_k.map;
    m.src_v = h->memo_commit_v.map;
    m.dst_k = h->tm_commit_k;
    m.dst_v = h->tm_commit_v;
    return SW_OK;
}

static int launch_commit(sw_attn_t* h, const void* K, const void* V, cudaStream_t st) {
    const sw_attn_config& c = h->cfg;
    const int ek = c.qk_fp8 ? 1 : 2, ev = c.pv_fp8 ? 1 : 2;
    int32_t* state = reinterpret_cast<int32_t*>(h->ws);
    cudaError_t e;
    if (h->commit_tma) {
        CommitMaps m;
        int rc;
        if ((rc = commit_maps(h, K, V, m))) return rc;
        e = launch_commit_tma(m, c.B, c.tokens_per_chunk, c.H, c.d, ek, ev, state, table_advance(h), h->S, h->num_sms,
                              st);
    } else {
        e = launch_relayout(K, V, h->ws + h->off_kcache, h->ws + h->off_vcache, c.B, c.tokens_per_chunk, c.H, c.d,
                            h->S * c.tokens_per_chunk, 1, h->S, state, table_advance(h), 1, st, ek, ev);
    }
    return e == cudaSuccess ? SW_OK : cuda_fail(e, "append launch");
}

int sw_attn_append_chunk(sw_attn_t* h, const void* K, const void* V, void* stream) {
    g_err.clear();
    if (!live(h)) return bad_handle(h);
    if (!h->ws) return fail(SW_ESTATE, "no workspace bound");
    if (!K || !V) return fail(SW_EINVAL, "null K or V");
    if (!aligned16(K) || !aligned16(V)) return fail(SW_EALIGN, "K and V must be 16-byte aligned");
    const sw_attn_config& c = h->cfg;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t* state = reinterpret_cast<int32_t*>(h->ws);
    cudaError_t e;
    if (h->S > 0) return launch_commit(h, K, V, st);
    e = launch_table_build(state, c.W, h->R, c.sink, c.n_cond, c.tokens_per_chunk, 1, st);
    return e == cudaSuccess ? SW_OK : cuda_fail(e, "table build launch");
}

// The full-path schedule of a forward over nqt Q tiles of 128 rows.  Auto: with fewer pairs of
// tiles than SMs, the three-buffer kernel (one tile per unit balances better); else persistent.
static int resolve_schedule_tiles(const sw_attn_t* h, long long nqt) {
    const sw_attn_config& c = h->cfg;
    // e4m3 handles: the persistent and three-buffer kernels have e4m3 forms (grid and pair do not,
    // refused at create), and the automatic choice below is the same as for bf16
    if (c.schedule == SW_SCHED_PAIR) return h->pair_clusters > 0 ? SW_SCHED_PAIR : SW_SCHED_TRI;
    if (c.schedule != SW_SCHED_AUTO) return c.schedule;
    const long long pairs = (long long)c.B * c.H * ((nqt + 1) / 2);
    return pairs < h->num_sms ? SW_SCHED_TRI : SW_SCHED_PERSISTENT;
}

static int resolve_schedule(const sw_attn_t* h, int n_q) {
    return resolve_schedule_tiles(h, (n_q + kBlockM - 1) / kBlockM);
}

int sw_attn_schedule_for(const sw_attn_t* h, int n_q) {
    g_err.clear();
    if (!live(h)) return bad_handle(h);
    if (n_q < 1) return fail(SW_EINVAL, "n_q < 1");
    return resolve_schedule(h, n_q);
}

int sw_attn_commit_kind(const sw_attn_t* h) {
    g_err.clear();
    if (!live(h)) return bad_handle(h);
    if (!h->ws) return fail(SW_ESTATE, "no workspace bound");
    return h->commit_tma ? SW_COMMIT_TMA : SW_COMMIT_COPY;
}

// Tensor maps, pointers and scalars every forward shares (the chunk's own n_q queries).
static int fill_params(sw_attn_t* h, AttnParams& p, const void* Q, const void* K_cur, const void* V_cur,
                       void* out, int n_q) {
    const sw_attn_config& c = h->cfg;
    std::memset(&p, 0, sizeof p);
    int rc;
    const int eqk = c.qk_fp8 ? 1 : 2;
    if ((rc = encode_user_memo(h->memo_q, Q, c.B, n_q, c.H, c.d, "Q", eqk))) return rc;
    if ((rc = encode_user_memo(h->memo_kcur, K_cur, c.B, c.tokens_per_chunk, c.H, c.d, "K_cur", eqk))) return rc;
    if ((rc = encode_user_memo(h->memo_vcur, V_cur, c.B, c.tokens_per_chunk, c.H, c.d, "V_cur", c.pv_fp8 ? 1 : 2)))
        return rc;
    p.tm_q = h->memo_q.map;
    p.tm_kcur = h->memo_kcur.map;
    p.tm_vcur = h->memo_vcur.map;
    // maps for regions this handle does not have are never read; fill them with a valid map
    p.tm_cache_k = h->S > 0 ? h->tm_cache_k : p.tm_kcur;
    p.tm_cache_v = h->S > 0 ? h->tm_cache_v : p.tm_vcur;
    p.tm_cond_k = c.n_cond > 0 ? h->tm_cond_k : p.tm_kcur;
    if (h->pair_ok) {
        if ((rc = encode_user_memo(h->memo_kcur_h, K_cur, c.B, c.tokens_per_chunk, c.H, c.d, "K_cur", 2, kBlockN / 2)))
            return rc;
        p.tm_kcur_h = h->memo_kcur_h.map;
        p.tm_cache_kh = h->S > 0 ? h->tm_cache_kh : p.tm_kcur_h;
        p.tm_cond_kh = c.n_cond > 0 ? h->tm_cond_kh : p.tm_kcur_h;
    } else {
        p.tm_kcur_h = p.tm_cache_kh = p.tm_cond_kh = p.tm_kcur;   // never read
    }
    p.tm_cond_v = c.n_cond > 0 ? h->tm_cond_v : p.tm_vcur;
    p.tm_qc = p.tm_q;   // no condition queries unless a joint forward sets them
    int32_t* state = reinterpret_cast<int32_t*>(h->ws);
    p.out = out;
    p.out_c = nullptr;
    p.table = state + kStateHeaderInts;
    p.status = state + 1;
    p.B = c.B;
    p.H = c.H;
    p.n_q = n_q;
    p.n_qc = 0;
    p.commit = 0;
    p.qk_fp8 = c.qk_fp8;
    p.pv_fp8 = c.pv_fp8;
    p.out_scale = c.pv_fp8 ? c.v_scale : 1.f;
    p.ring_R = h->R;
    p.sink = c.sink;
    p.out_f32 = c.out_dtype == SW_OUT_F32;
    // e4m3 Q and K: S = (q * q_scale) . (k * k_scale), the scales folded into the softmax scale
    p.scale_log2 = c.scale * 1.4426950408889634f * (c.qk_fp8 ? c.q_scale * c.k_scale : 1.f);
    return SW_OK;
}

// Full-path launch over all Q tiles of p (the chunk's, then any condition queries'), with the
// schedule the handle resolves for that many tiles.
static int launch_full(sw_attn_t* h, AttnParams& p, cudaStream_t st) {
    const sw_attn_config& c = h->cfg;
    const long long nqt = (p.n_q + kBlockM - 1) / kBlockM + (p.n_qc + kBlockM - 1) / kBlockM;
    const int sched = resolve_schedule_tiles(h, nqt);
    cudaError_t e;
    p.splits = 0;
    if (sched == SW_SCHED_GRID) {
        e = launch_attention(p, c.d, (int)((nqt + 1) / 2), st);
        if (e != cudaSuccess) return cuda_fail(e, "attention launch");
        return SW_OK;
    }
    p.sk_o = reinterpret_cast<float*>(h->ws + h->off_sk_o);
    p.sk_ml = reinterpret_cast<float*>(h->ws + h->off_sk_ml);
    p.sk_cnt = reinterpret_cast<int32_t*>(h->ws + h->off_sk_cnt);
    p.sk_pairs = h->sk_pairs;
    // one CTA per SM, but never so many that a CTA's share of the cost line is shorter than
    // two items at the fewest key tiles a chunk can have (condition + current only)
    const long long nt_min = (c.n_cond + kBlockN - 1) / kBlockN + (c.tokens_per_chunk + kBlockN - 1) / kBlockN;
    const long long c_min = (long long)c.B * c.H * nqt * nt_min;
    long long ctas = std::min<long long>(h->num_sms, kMaxPersistentCtas);
    ctas = std::max<long long>(1, std::min<long long>(ctas, c_min / 2));
    if (sched == SW_SCHED_TRI) {
        e = launch_tri(p, c.d, (int)ctas, st);
        if (e != cudaSuccess) return cuda_fail(e, "three-buffer attention launch");
        return SW_OK;
    }
    if (sched == SW_SCHED_PAIR) {
        // one CTA pair per two SMs, with the same floor of two items per pair
        long long pairs = std::min<long long>(h->pair_clusters, kMaxPersistentCtas / 2);
        pairs = std::max<long long>(1, std::min<long long>(pairs, c_min / 4));
        e = launch_pair(p, (int)pairs, st);
        if (e != cudaSuccess) return cuda_fail(e, "CTA-pair attention launch");
        return SW_OK;
    }
    e = launch_persistent(p, c.d, (int)ctas, st);
    if (e != cudaSuccess) return cuda_fail(e, "persistent attention launch");
    return SW_OK;
}

int sw_attn_forward(sw_attn_t* h, const void* Q, const void* K_cur, const void* V_cur, void* out, int n_q,
                    void* stream) {
    g_err.clear();
    if (!live(h)) return bad_handle(h);
    if (!h->ws) return fail(SW_ESTATE, "no workspace bound");
    if (!h->cond_set) return fail(SW_ESTATE, "condition tokens not set");
    if (!Q || !K_cur || !V_cur || !out) return fail(SW_EINVAL, "null tensor");
    const sw_attn_config& c = h->cfg;
    if (n_q < 1 || n_q > c.tokens_per_chunk)
        return fail(SW_ESHAPE, "n_q must be in [1, %d] (n_q=%d)", c.tokens_per_chunk, n_q);
    if (!aligned16(Q) || !aligned16(K_cur) || !aligned16(V_cur) || !aligned16(out))
        return fail(SW_EALIGN, "Q, K_cur, V_cur and out must be 16-byte aligned");
    AttnParams p;
    int rc;
    if ((rc = fill_params(h, p, Q, K_cur, V_cur, out, n_q))) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (n_q <= h->short_q) {
        const int bh = c.B * c.H;
        int splits = h->num_sms / bh;
        splits = std::max(1, std::min(splits, h->max_splits));
        p.splits = splits;
        p.o_part = reinterpret_cast<float*>(h->ws + h->off_opart);
        p.ml_part = reinterpret_cast<float*>(h->ws + h->off_ml);
        cudaError_t e = launch_split(p, c.d, splits, st);
        if (e != cudaSuccess) return cuda_fail(e, "split-K attention launch");
        e = launch_combine(p.o_part, p.ml_part, out, c.B, c.H, n_q, c.d, splits, p.out_f32, p.out_scale, st);
        if (e != cudaSuccess) return cuda_fail(e, "combine launch");
        return SW_OK;
    }
    return launch_full(h, p, st);
}

int sw_attn_append_chunk_batched(sw_attn_t* const* hs, int n, const void* const* K, const void* const* V,
                                 void* stream) {
    g_err.clear();
    if (!hs || !K || !V || n < 1) return fail(SW_EINVAL, "null array or n < 1");
    const sw_attn_t* h0 = hs[0];
    if (!live(h0)) return fail(SW_EINVAL, h0 ? "unknown or destroyed handle 0" : "null handle 0");
    const sw_attn_config& c0 = h0->cfg;
    for (int l = 0; l < n; ++l) {
        const sw_attn_t* h = hs[l];
        if (!live(h)) return fail(SW_EINVAL, h ? "unknown or destroyed handle %d" : "null handle %d", l);
        if (!h->ws) return fail(SW_ESTATE, "handle %d has no workspace bound", l);
        if (h->device != h0->device) return fail(SW_ESTATE, "handle %d is on another device", l);
        const sw_attn_config& c = h->cfg;
        if (c.B != c0.B || c.H != c0.H || c.d != c0.d || c.tokens_per_chunk != c0.tokens_per_chunk ||
            c.qk_fp8 != c0.qk_fp8 || c.pv_fp8 != c0.pv_fp8)
            return fail(SW_ESHAPE, "handle %d: B, H, d, T and the K and V formats must match handle 0", l);
        if (!K[l] || !V[l]) return fail(SW_EINVAL, "null K or V for handle %d", l);
        if (!aligned16(K[l]) || !aligned16(V[l])) return fail(SW_EALIGN, "K and V of handle %d must be 16-byte aligned", l);
        for (int m = 0; m < l; ++m)
            if (hs[m] == h) return fail(SW_EINVAL, "handle %d appears twice", l);
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // TMA bulk copies when every handle has its commit maps and either forces them or the batch
    // as a whole gives every SM a full ring of items (the single-commit rule, over all handles)
    bool tma = true, forced = true;
    for (int l = 0; l < n; ++l) {
        tma = tma && hs[l]->commit_maps_ok && hs[l]->S > 0;
        forced = forced && hs[l]->cfg.commit_path == SW_COMMIT_TMA;
    }
    const long long items = 2LL * c0.B * ((c0.tokens_per_chunk + kCommitRows - 1) / kCommitRows) *
                            ((c0.H + kCommitHeads - 1) / kCommitHeads) * n;
    tma = tma && (forced || items >= (long long)kCommitBufs * h0->num_sms);
    if (tma) {
        const int ek = c0.qk_fp8 ? 1 : 2, ev = c0.pv_fp8 ? 1 : 2;
        for (int l0 = 0; l0 < n; l0 += kCommitBatch) {
            CommitBatch cb;
            std::memset(&cb, 0, sizeof cb);
            cb.n = std::min(kCommitBatch, n - l0);
            for (int q = 0; q < cb.n; ++q) {
                sw_attn_t* h = hs[l0 + q];
                int rc;
                if ((rc = commit_maps(h, K[l0 + q], V[l0 + q], cb.maps[q]))) return rc;
                cb.state[q] = reinterpret_cast<int32_t*>(h->ws);
                cb.ta[q] = table_advance(h);
                cb.S[q] = h->S;
            }
            const int per = std::max(1, h0->num_sms / cb.n);
            cudaError_t e = launch_commit_tma_batch(cb, c0.B, c0.tokens_per_chunk, c0.H, c0.d, ek, ev, per, st);
            if (e != cudaSuccess) return cuda_fail(e, "batched TMA commit launch");
        }
        return SW_OK;
    }
    for (int l0 = 0; l0 < n; l0 += kMaxBatch) {
        AppendBatch a;
        std::memset(&a, 0, sizeof a);
        a.n = std::min(kMaxBatch, n - l0);
        for (int q = 0; q < a.n; ++q) {
            sw_attn_t* h = hs[l0 + q];
            a.K[q] = K[l0 + q];
            a.V[q] = V[l0 + q];
            a.dstK[q] = h->ws + h->off_kcache;
            a.dstV[q] = h->ws + h->off_vcache;
            a.state[q] = reinterpret_cast<int32_t*>(h->ws);
            a.R[q] = h->R;
            a.S[q] = h->S;
            a.W[q] = h->cfg.W;
            a.sink[q] = h->cfg.sink;
            a.n_cond[q] = h->cfg.n_cond;
        }
        cudaError_t e = launch_append_batch(a, c0.B, c0.tokens_per_chunk, c0.H, c0.d, c0.qk_fp8 ? 1 : 2,
                                            c0.pv_fp8 ? 1 : 2, st);
        if (e != cudaSuccess) return cuda_fail(e, "batched append launch");
    }
    return SW_OK;
}

int sw_attn_forward_commit(sw_attn_t* h, const void* Q, const void* K_cur, const void* V_cur, void* out,
                           void* stream) {
    g_err.clear();
    if (!live(h)) return bad_handle(h);
    if (!h->ws) return fail(SW_ESTATE, "no workspace bound");
    if (!h->cond_set) return fail(SW_ESTATE, "condition tokens not set");
    const sw_attn_config& c = h->cfg;
    if (!c.commit_in_forward) return fail(SW_ESTATE, "the handle was not created with commit_in_forward");
    if (c.B > 32767 || c.H > 65535) return fail(SW_ESHAPE, "a committing forward supports B <= 32767, H <= 65535");
    if (!Q || !K_cur || !V_cur || !out) return fail(SW_EINVAL, "null tensor");
    if (!aligned16(Q) || !aligned16(K_cur) || !aligned16(V_cur) || !aligned16(out))
        return fail(SW_EALIGN, "Q, K_cur, V_cur and out must be 16-byte aligned");
    AttnParams p;
    int rc;
    if ((rc = fill_params(h, p, Q, K_cur, V_cur, out, c.tokens_per_chunk))) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const long long nqt = (c.tokens_per_chunk + kBlockM - 1) / kBlockM;
    int32_t* state = reinterpret_cast<int32_t*>(h->ws);
    const int sched = resolve_schedule_tiles(h, nqt);
    if (sched == SW_SCHED_TRI || sched == SW_SCHED_PAIR) {
        // the three-buffer kernels do not store K/V: forward, then the copy into the same slot
        if ((rc = launch_full(h, p, st))) return rc;
        if (h->S > 0) return launch_commit(h, K_cur, V_cur, st);   // the copy launch also advances the table
    } else {
        p.commit = h->S > 0 ? 1 : 0;
        if ((rc = launch_full(h, p, st))) return rc;
    }
    cudaError_t e = launch_table_build(state, c.W, h->R, c.sink, c.n_cond, c.tokens_per_chunk, 1, st);
    if (e != cudaSuccess) return cuda_fail(e, "table launch");
    return SW_OK;
}

int sw_attn_forward_joint(sw_attn_t* h, const void* Q, const void* Q_cond, const void* K_cur, const void* V_cur,
                          void* out, void* out_cond, void* stream) {
    g_err.clear();
    if (!live(h)) return bad_handle(h);
    if (!h->ws) return fail(SW_ESTATE, "no workspace bound");
    if (!h->cond_set) return fail(SW_ESTATE, "condition tokens not set");
    const sw_attn_config& c = h->cfg;
    if (c.n_cond < 1) return fail(SW_ESHAPE, "a joint forward needs n_cond >= 1 condition tokens");
    if (!Q || !Q_cond || !K_cur || !V_cur || !out || !out_cond) return fail(SW_EINVAL, "null tensor");
    if (!aligned16(Q) || !aligned16(Q_cond) || !aligned16(K_cur) || !aligned16(V_cur) || !aligned16(out) ||
        !aligned16(out_cond))
        return fail(SW_EALIGN, "Q, Q_cond, K_cur, V_cur, out and out_cond must be 16-byte aligned");
    AttnParams p;
    int rc;
    if ((rc = fill_params(h, p, Q, K_cur, V_cur, out, c.tokens_per_chunk))) return rc;
    if ((rc = encode_user_memo(h->memo_qc, Q_cond, c.B, c.n_cond, c.H, c.d, "Q_cond", c.qk_fp8 ? 1 : 2))) return rc;
    p.tm_qc = h->memo_qc.map;
    p.out_c = out_cond;
    p.n_qc = c.n_cond;
    return launch_full(h, p, static_cast<cudaStream_t>(stream));
}

int sw_attn_get_table(const sw_attn_t* h, int32_t* dev_table, void* stream) {
    g_err.clear();
    if (!live(h)) return bad_handle(h);
    if (!dev_table) return fail(SW_EINVAL, "null argument");
    if (!h->ws) return fail(SW_ESTATE, "no workspace bound");
    cudaError_t e = cudaMemcpyAsync(dev_table, h->ws + sizeof(int32_t) * kStateHeaderInts,
                                    sizeof(int32_t) * h->table_ints, cudaMemcpyDeviceToDevice,
                                    static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SW_OK : cuda_fail(e, "table copy");
}

int sw_attn_cache_offsets(const sw_attn_t* h, size_t* k_offset, size_t* v_offset) {
    g_err.clear();
    if (!live(h)) return bad_handle(h);
    if (!k_offset || !v_offset) return fail(SW_EINVAL, "null argument");
    *k_offset = h->off_kcache;
    *v_offset = h->off_vcache;
    return SW_OK;
}

int sw_attn_selftest_timeout(sw_attn_t* h, int64_t limit_ns, void* stream) {
    g_err.clear();
    if (!live(h)) return bad_handle(h);
    if (!h->ws) return fail(SW_ESTATE, "no workspace bound");
    if (limit_ns < 1000000 || limit_ns > 2000000000LL) return fail(SW_EINVAL, "limit_ns must be in [1e6, 2e9]");
    cudaError_t e = launch_selftest_timeout(reinterpret_cast<int32_t*>(h->ws) + 1, (uint64_t)limit_ns,
                                            static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SW_OK : cuda_fail(e, "self-test launch");
}

int sw_attn_get_status(sw_attn_t* h, int32_t* host_status) {
    g_err.clear();
    if (!live(h)) return bad_handle(h);
    if (!host_status) return fail(SW_EINVAL, "null argument");
    if (!h->ws) return fail(SW_ESTATE, "no workspace bound");
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
    e = cudaMemcpy(host_status, h->ws + sizeof(int32_t), sizeof(int32_t), cudaMemcpyDeviceToHost);
    return e == cudaSuccess ? SW_OK : cuda_fail(e, "status copy");
}

}  // extern "C"

// ------------------------------------------------------------------ no-alloc short forward
// Callers that cannot allocate device memory at call time (a framework's fixed memory pool, a
// fixed-footprint server) get the split-K decode path with its partials in this file-scope
// array instead of the workspace.  Host code only ever uses the array's device address, looked
// up once per device with that device current (the array's name is a host-side stand-in).
namespace {
constexpr size_t kNoAllocScratchFloats = size_t(4) << 20;   // 16 MiB per GPU
constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
float* g_noalloc_ptr[kNoAllocMaxDevices] = {};
}  // namespace

static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

extern "C" int sw_attn_forward_short_noalloc(sw_attn_t* h, const void* Q, const void* K_cur, const void* V_cur,
                                             void* out, int n_q, void* stream) {
    g_err.clear();
    if (!live(h)) return bad_handle(h);
    if (!h->ws) return fail(SW_ESTATE, "no workspace bound");
    if (!h->cond_set) return fail(SW_ESTATE, "condition tokens not set");
    if (!Q || !K_cur || !V_cur || !out) return fail(SW_EINVAL, "null tensor");
    const sw_attn_config& c = h->cfg;
    if (n_q < 1 || n_q > kMaxShortQ || n_q > c.tokens_per_chunk)
        return fail(SW_ESHAPE, "n_q must be in [1, min(%d, T)] (n_q=%d)", kMaxShortQ, n_q);
    if (!aligned16(Q) || !aligned16(K_cur) || !aligned16(V_cur) || !aligned16(out))
        return fail(SW_EALIGN, "Q, K_cur, V_cur and out must be 16-byte aligned");
    const size_t per_split = (size_t)c.B * c.H * kBlockM * (c.d + 2);
    const size_t fit = kNoAllocScratchFloats / per_split;
    if (fit < 1)
        return fail(SW_ESHAPE, "B*H*128*(d+2) = %zu floats exceeds the fixed %zu-float scratch", per_split,
                    kNoAllocScratchFloats);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev != h->device) return fail(SW_ESTATE, "current device %d is not the workspace's device %d", dev, h->device);
    if (dev < 0 || dev >= kNoAllocMaxDevices) return fail(SW_EINVAL, "device ordinal %d not supported", dev);
    float* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_noalloc_mu);
        if (!g_noalloc_ptr[dev]) {
            void* ptr = nullptr;
            e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
            if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
            g_noalloc_ptr[dev] = static_cast<float*>(ptr);
        }
        scratch = g_noalloc_ptr[dev];
    }
    AttnParams p;
    int rc;
    if ((rc = fill_params(h, p, Q, K_cur, V_cur, out, n_q))) return rc;
    const int bh = c.B * c.H;
    long long splits = h->num_sms / bh;
    // the same split count as sw_attn_forward; the clamp to what fits the array only binds on a
    // GPU with more SMs than a B200 (there fit >= 148 / (B*H) for every accepted shape)
    splits = std::max<long long>(1, std::min<long long>(splits, std::min<long long>((long long)fit, kMaxSplits)));
    p.splits = (int)splits;
    p.o_part = scratch;
    p.ml_part = scratch + (size_t)splits * bh * kBlockM * c.d;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    e = launch_split(p, c.d, (int)splits, st);
    if (e != cudaSuccess) return cuda_fail(e, "split-K attention launch");
    e = launch_combine(p.o_part, p.ml_part, out, c.B, c.H, n_q, c.d, (int)splits, p.out_f32, p.out_scale, st);
    if (e != cudaSuccess) return cuda_fail(e, "combine launch");
    return SW_OK;
}

/*
 * swattn_oracle.c -- plain FP64 CPU oracle for block-causal sink + sliding-window attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call this file:
 * only the tests, the package's smoke check and the benchmark's CPU-baseline and reference legs
 * use it.
 * It shares no code, header or constant with the CUDA library.
 *
 * What it computes follows two pages about JoyAI-Video-Edit:
 *   [TUT]  "JoyAI-Video-Edit：单卡720p 30帧，两步蒸馏攻克流式视频编辑" (agifrontier tutorial),
 *          section "从双向编辑到分块因果架构的蜕变" (chunk-wise AR adaptation, block-causal mask,
 *          bounded window plus first-chunk global sink) and section "软硬件协同部署"
 *          (clean K/V written to the cache after each chunk; constant cache).
 *   [NH]   neurohive review "JoyAI-Video-Edit" (ru), section "Чанки и борьба с дрейфом"
 *          (bidirectional inside a chunk, causal across chunks, a fixed number of recent
 *          chunks plus the very first one), and section "Архитектура JoyAI-Video-Edit"
 *          (condition tokens from the MLLM encoder feed the MM-DiT).
 *
 * The method is exact masked softmax attention; the bounded cache only decides WHICH keys
 * are visible.  So the oracle is the plain definition with an explicit dense mask over the
 * full, never-evicted history, in double precision:
 *
 *   Hist(k)  = { j : max(0, k-W) <= j <= k-1 }  U  ({0} if sink and k >= 1)
 *   Kfull    = [Kc ; K(0) ; ... ; K(k-1) ; K_cur]            (same for V)
 *   M[j] = 1 iff key j is a condition key, a current-chunk key, or in a chunk of Hist(k);
 *            the mask is the same for every query row (bidirectional inside the chunk).
 *   out[i]   = sum_{M[j]=1} exp(s q_i.k_j - m_i) v_j / sum_{M[j]=1} exp(s q_i.k_j - m_i)
 *
 * Readings taken where the pages are silent:
 *   - W counts recent chunks only; the sink is a set union with the window, so chunk 0 is
 *     never counted twice and steady state sees W+1 history chunks.
 *   - the sink is exactly chunk 0 (all T tokens); chunk 0 as the active chunk sees the
 *     condition tokens and itself only.
 *   - masked keys are skipped (never multiplied by zero), so NaN in them cannot leak.
 *   - ring slots: with the sink, slot(0)=0 and slot(c)=1+((c-1) mod W); without it
 *     slot(c)=c mod W.  W=0 keeps no window chunk.
 *   - a ring may keep R = W + 1 window slots instead of W (the *_r functions): one slot then
 *     holds the chunk that has just left the window, so the chunk being produced can be
 *     written while its own forward still reads every visible chunk.  Which keys are visible
 *     does not change, only where they are kept.
 *
 * Inputs are float32 arrays holding bf16-rounded values (exact in float32); all arithmetic
 * is in double.  Layouts are the user layout [B][N][H][d], row-major.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC swattn_oracle.c -o libswattn_oracle.so -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- visibility */

/* 1 iff history chunk j (0 <= j < k) is visible to active chunk k ([TUT] §从双向编辑到分块因果架构的蜕变;
 * [NH] §Чанки и борьба с дрейфом: a fixed number of recent chunks plus the very first). */
int swo_visible(int k, int W, int sink, int j)
{
    if (j < 0 || j >= k) return 0;          /* causal across chunks: no future, no self here */
    if (j >= k - W) return 1;               /* the W most recent chunks */
    if (sink && j == 0) return 1;           /* the permanent global sink */
    return 0;
}

/* Number of ring slots for the bounded cache with R window slots. */
int swo_num_slots_r(int R, int sink)
{
    return R + (sink ? 1 : 0);
}

int swo_num_slots(int W, int sink)
{
    return swo_num_slots_r(W, sink);
}

/* Ring slot holding committed chunk c with R window slots; -1 if the chunk is never stored
 * (R = 0: no window chunk is kept).  Window chunks rotate through the R slots, so chunk c
 * takes the slot of chunk c - R. */
int swo_slot_r(int c, int R, int sink)
{
    if (c < 0) return -1;
    if (sink) {
        if (c == 0) return 0;
        if (R == 0) return -1;
        return 1 + (c - 1) % R;
    }
    if (R == 0) return -1;
    return c % R;
}

int swo_slot(int c, int W, int sink)
{
    return swo_slot_r(c, W, sink);
}

/*
 * Canonical visibility table for active chunk k.
 *   out[0] = k, out[1] = n_segments, out[2] = N_vis (visible keys),
 *   then per segment 4 ints: kind (0 cond, 1 cache, 2 current), chunk_id, slot, n_tokens.
 * Segment order: cond (only if n_cond > 0), sink, window chunks ascending, current.
 * For kind 0 chunk_id = slot = -1; for kind 2 chunk_id = k and slot = -1.
 * Returns the number of ints written, or -1 if cap is too small.
 */
int swo_table_r(int k, int W, int R, int sink, int n_cond, int T, int32_t *out, int cap)
{
    int nseg = 0, nvis = 0, pos = 3, j;
    if (cap < 3) return -1;
    if (n_cond > 0) {
        if (pos + 4 > cap) return -1;
        out[pos++] = 0; out[pos++] = -1; out[pos++] = -1; out[pos++] = n_cond;
        nseg++; nvis += n_cond;
    }
    for (j = 0; j < k; j++) {
        if (!swo_visible(k, W, sink, j)) continue;
        if (pos + 4 > cap) return -1;
        out[pos++] = 1; out[pos++] = j; out[pos++] = swo_slot_r(j, R, sink); out[pos++] = T;
        nseg++; nvis += T;
    }
    if (pos + 4 > cap) return -1;
    out[pos++] = 2; out[pos++] = k; out[pos++] = -1; out[pos++] = T;
    nseg++; nvis += T;
    out[0] = k; out[1] = nseg; out[2] = nvis;
    return pos;
}

int swo_table(int k, int W, int sink, int n_cond, int T, int32_t *out, int cap)
{
    return swo_table_r(k, W, W, sink, n_cond, T, out, cap);
}

/*
 * The chunk-level bitmap row of the visibility table for active chunk k: row[j] = 1 iff
 * history chunk j is in Hist(k), for every j < k (chunk k itself, the current chunk, is always
 * visible and is not part of the row).  This is the dense mask of the definition above taken
 * at chunk granularity ([TUT] §从双向编辑到分块因果架构的蜕变: recent window plus the first chunk;
 * [NH] §Чанки и борьба с дрейфом).  Writes k bytes; returns k, or -1 if cap < k.
 */
int swo_vis_row(int k, int W, int sink, unsigned char *row, int cap)
{
    if (k < 0 || cap < k) return -1;
    for (int j = 0; j < k; j++) row[j] = (unsigned char)swo_visible(k, W, sink, j);
    return k;
}

/* ---------------------------------------------------------------- dense oracle */

static double dot_f(const float *a, const float *b, int d)
{
    double s = 0.0;
    for (int c = 0; c < d; c++) s += (double)a[c] * (double)b[c];
    return s;
}

/*
 * Dense-mask full-history attention.
 *   Kc, Vc         [B][n_cond][H][d]     (may be NULL when n_cond == 0)
 *   Khist, Vhist   k pointers, chunk c -> [B][T][H][d]; an entry may be NULL only if the
 *                  mask says that chunk is invisible (otherwise the call fails with -2)
 *   Q              [B][n_q][H][d]
 *   Kcur, Vcur     [B][T][H][d]
 *   rows           query rows to compute (NULL: all n_q rows, n_rows must equal n_q)
 *   out            [B][n_rows][H][d] doubles
 * Returns 0, or -1 on bad arguments, -2 if a visible chunk has no data.
 */
int swo_attention(int B, int H, int d, int T, int n_cond, int W, int sink, int k,
                  const float *Kc, const float *Vc,
                  const float *const *Khist, const float *const *Vhist,
                  const float *Q, int n_q, const float *Kcur, const float *Vcur,
                  double scale, const int32_t *rows, int n_rows, double *out)
{
    if (B <= 0 || H <= 0 || d <= 0 || T <= 0 || n_cond < 0 || W < 0 || k < 0 || n_q <= 0)
        return -1;
    if (!rows && n_rows != n_q) return -1;
    const long nfull = (long)n_cond + (long)k * T + T;
    /* explicit dense mask over the full key list (identical for every query row) */
    unsigned char *mask = (unsigned char *)malloc((size_t)nfull);
    if (!mask) return -1;
    long p = 0;
    for (int j = 0; j < n_cond; j++) mask[p++] = 1;
    for (int c = 0; c < k; c++) {
        unsigned char vis = (unsigned char)swo_visible(k, W, sink, c);
        if (vis && (!Khist[c] || !Vhist[c])) { free(mask); return -2; }
        for (int t = 0; t < T; t++) mask[p++] = vis;
    }
    for (int t = 0; t < T; t++) mask[p++] = 1;

    const long total = (long)B * H * n_rows;
    int err = 0;
#pragma omp parallel
    {
        double *sc = (double *)malloc(sizeof(double) * (size_t)nfull);
        double *acc = (double *)malloc(sizeof(double) * (size_t)d);
        if (!sc || !acc) {
#pragma omp atomic write
            err = 1;
        }
#pragma omp for schedule(dynamic, 4)
        for (long w = 0; w < total; w++) {
            if (!sc || !acc) continue;
            const int b = (int)(w / ((long)H * n_rows));
            const int r = (int)((w / H) % n_rows);
            const int h = (int)(w % H);
            const int i = rows ? rows[r] : r;
            const float *q = Q + (((long)b * n_q + i) * H + h) * d;
            /* key j of Kfull: where its row lives */
            double mx = -INFINITY;
            long jj = 0;
            for (int j = 0; j < n_cond; j++, jj++) {
                const float *kr = Kc + (((long)b * n_cond + j) * H + h) * d;
                sc[jj] = scale * dot_f(q, kr, d);
                if (sc[jj] > mx) mx = sc[jj];
            }
            for (int c = 0; c < k; c++) {
                for (int t = 0; t < T; t++, jj++) {
                    if (!mask[jj]) continue;           /* skipped, never multiplied by 0 */
                    const float *kr = Khist[c] + (((long)b * T + t) * H + h) * d;
                    sc[jj] = scale * dot_f(q, kr, d);
                    if (sc[jj] > mx) mx = sc[jj];
                }
            }
            for (int t = 0; t < T; t++, jj++) {
                const float *kr = Kcur + (((long)b * T + t) * H + h) * d;
                sc[jj] = scale * dot_f(q, kr, d);
                if (sc[jj] > mx) mx = sc[jj];
            }
            for (int c = 0; c < d; c++) acc[c] = 0.0;
            double den = 0.0;
            jj = 0;
            for (int j = 0; j < n_cond; j++, jj++) {
                const double e = exp(sc[jj] - mx);
                const float *vr = Vc + (((long)b * n_cond + j) * H + h) * d;
                den += e;
                for (int c = 0; c < d; c++) acc[c] += e * (double)vr[c];
            }
            for (int cc = 0; cc < k; cc++) {
                for (int t = 0; t < T; t++, jj++) {
                    if (!mask[jj]) continue;
                    const double e = exp(sc[jj] - mx);
                    const float *vr = Vhist[cc] + (((long)b * T + t) * H + h) * d;
                    den += e;
                    for (int c = 0; c < d; c++) acc[c] += e * (double)vr[c];
                }
            }
            for (int t = 0; t < T; t++, jj++) {
                const double e = exp(sc[jj] - mx);
                const float *vr = Vcur + (((long)b * T + t) * H + h) * d;
                den += e;
                for (int c = 0; c < d; c++) acc[c] += e * (double)vr[c];
            }
            double *o = out + (((long)b * n_rows + r) * H + h) * d;
            for (int c = 0; c < d; c++) o[c] = acc[c] / den;
        }
        free(sc);
        free(acc);
    }
    free(mask);
    return err ? -1 : 0;
}

/* ---------------------------------------------------------------- ring-buffer oracle */
/*
 * A second, independent statement of the same attention: the bounded cache as a ring of
 * S slots with a pinned sink ([TUT] §软硬件协同部署: clean K/V committed after each chunk,
 * "global sink + sliding local window").  The visible set is whatever the ring holds.
 * It shares the definition with swo_attention, not its code, and is used to check that
 * streaming through the ring equals recomputation from the full history.
 */
typedef struct {
    int B, H, d, T, n_cond, W, R, sink, S, n_committed;
    int *slot_chunk;     /* chunk id held by each slot, -1 if empty */
    float *K, *V;        /* [S][B][T][H][d] */
    float *Kc, *Vc;      /* [B][n_cond][H][d] */
} swo_ring;

/* R window slots (R = W: the plain ring; R = W + 1: one spare slot). */
void *swo_ring_create_r(int B, int H, int d, int T, int n_cond, int W, int R, int sink,
                        const float *Kc, const float *Vc)
{
    swo_ring *r = (swo_ring *)calloc(1, sizeof(swo_ring));
    if (!r) return NULL;
    r->B = B; r->H = H; r->d = d; r->T = T; r->n_cond = n_cond; r->W = W; r->R = R; r->sink = sink;
    r->S = R + (sink ? 1 : 0);
    const size_t chunk = (size_t)B * T * H * d;
    const size_t cond = (size_t)B * n_cond * H * d;
    r->slot_chunk = (int *)malloc(sizeof(int) * (size_t)(r->S > 0 ? r->S : 1));
    r->K = (float *)malloc(sizeof(float) * chunk * (size_t)(r->S > 0 ? r->S : 1));
    r->V = (float *)malloc(sizeof(float) * chunk * (size_t)(r->S > 0 ? r->S : 1));
    r->Kc = (float *)malloc(sizeof(float) * (cond ? cond : 1));
    r->Vc = (float *)malloc(sizeof(float) * (cond ? cond : 1));
    if (!r->slot_chunk || !r->K || !r->V || !r->Kc || !r->Vc) return NULL;
    for (int s = 0; s < r->S; s++) r->slot_chunk[s] = -1;
    if (cond) {
        memcpy(r->Kc, Kc, sizeof(float) * cond);
        memcpy(r->Vc, Vc, sizeof(float) * cond);
    }
    return r;
}

void *swo_ring_create(int B, int H, int d, int T, int n_cond, int W, int sink,
                      const float *Kc, const float *Vc)
{
    return swo_ring_create_r(B, H, d, T, n_cond, W, W, sink, Kc, Vc);
}

void swo_ring_destroy(void *h)
{
    swo_ring *r = (swo_ring *)h;
    if (!r) return;
    free(r->slot_chunk); free(r->K); free(r->V); free(r->Kc); free(r->Vc); free(r);
}

/* Commit the finished chunk: the sink slot is written once; later chunks overwrite the
 * oldest window chunk, c - R (with R = W that is the chunk leaving the window now; with a
 * spare slot, the one that left it a chunk ago), or take an empty slot. */
void swo_ring_append(void *h, const float *K, const float *V)
{
    swo_ring *r = (swo_ring *)h;
    const int c = r->n_committed;
    int s = -1;
    if (r->sink && c == 0) {
        s = 0;
    } else if (r->R > 0 && r->W > 0) {
        /* choose the slot of the oldest window chunk, else the first empty slot */
        const int base = r->sink ? 1 : 0;
        for (int q = base; q < r->S; q++)
            if (r->slot_chunk[q] >= 0 && r->slot_chunk[q] == c - r->R) { s = q; break; }
        if (s < 0)
            for (int q = base; q < r->S; q++)
                if (r->slot_chunk[q] < 0) { s = q; break; }
    }
    if (s >= 0) {
        const size_t chunk = (size_t)r->B * r->T * r->H * r->d;
        memcpy(r->K + (size_t)s * chunk, K, sizeof(float) * chunk);
        memcpy(r->V + (size_t)s * chunk, V, sizeof(float) * chunk);
        r->slot_chunk[s] = c;
    }
    r->n_committed = c + 1;
}

int swo_ring_slot_chunk(void *h, int s) { return ((swo_ring *)h)->slot_chunk[s]; }

/* Attention of the active chunk over [cond ; occupied slots holding a window or sink chunk ;
 * current]; all rows.  (With a spare slot, one occupied slot holds the chunk that has already
 * left the window: it is skipped.) */
int swo_ring_forward(void *h, const float *Q, int n_q, const float *Kcur, const float *Vcur,
                     double scale, double *out)
{
    swo_ring *r = (swo_ring *)h;
    const int B = r->B, H = r->H, d = r->d, T = r->T, nc = r->n_cond;
    const size_t chunk = (size_t)B * T * H * d;
    const long total = (long)B * n_q * H;
#pragma omp parallel for schedule(dynamic, 4)
    for (long w = 0; w < total; w++) {
        const int b = (int)(w / ((long)n_q * H));
        const int i = (int)((w / H) % n_q);
        const int hh = (int)(w % H);
        const float *q = Q + (((long)b * n_q + i) * H + hh) * d;
        /* online (streaming) softmax in double, one key at a time */
        double m = -INFINITY, l = 0.0;
        double acc[512];
        for (int c = 0; c < d; c++) acc[c] = 0.0;
        for (int part = 0; part < 3; part++) {
            int nslot = part == 1 ? r->S : 1;
            for (int s = 0; s < nslot; s++) {
                const float *Kb, *Vb;
                int nrows, rstride_n;
                if (part == 0) { Kb = r->Kc; Vb = r->Vc; nrows = nc; rstride_n = nc; }
                else if (part == 1) {
                    const int held = r->slot_chunk[s];
                    if (held < 0) continue;
                    if (held < r->n_committed - r->W && !(r->sink && held == 0)) continue;
                    Kb = r->K + (size_t)s * chunk; Vb = r->V + (size_t)s * chunk;
                    nrows = T; rstride_n = T;
                } else { Kb = Kcur; Vb = Vcur; nrows = T; rstride_n = T; }
                for (int t = 0; t < nrows; t++) {
                    const float *kr = Kb + (((long)b * rstride_n + t) * H + hh) * d;
                    const float *vr = Vb + (((long)b * rstride_n + t) * H + hh) * d;
                    double x = 0.0;
                    for (int c = 0; c < d; c++) x += (double)q[c] * (double)kr[c];
                    x *= scale;
                    if (x > m) {
                        const double f = exp(m - x);   /* exp(-inf) = 0 on the first key */
                        l *= f;
                        for (int c = 0; c < d; c++) acc[c] *= f;
                        m = x;
                    }
                    const double e = exp(x - m);
                    l += e;
                    for (int c = 0; c < d; c++) acc[c] += e * (double)vr[c];
                }
            }
        }
        double *o = out + (((long)b * n_q + i) * H + hh) * d;
        for (int c = 0; c < d; c++) o[c] = acc[c] / l;
    }
    return 0;
}

int swo_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads for the calling thread's later parallel regions (a launcher may have set
 * OMP_NUM_THREADS=1 for every process of a multi-process job). */
void swo_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

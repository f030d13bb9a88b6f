/*
 * Sliding-window attention oracle: plain, slow, fp64, CPU only.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load this library.  The CUDA path never links,
 * includes or calls anything from this directory, and this file includes
 * nothing from the CUDA path.
 *
 * Every floating-point input arrives as fp64 (bf16 or fp32 values upcast
 * exactly by the caller), every sum is an fp64 sum in index order, and the
 * softmax is the textbook two-pass form: row maximum first, then exponentials
 * and their sum, then the weighted sum of value rows divided by that sum.
 *
 * Sources (page title, section):
 *  [P2]  "How sliding window attention works in Mistral and Longformer"
 *        (aivaro.ru answer 629), sections 2 (idea), 3 (Mistral: the window
 *        counts the token itself), 4.1 (symmetric W/2 left and right),
 *        4.3 (Longformer global attention), 9 (pet project: build the mask,
 *        put -inf at forbidden positions, softmax, weighted sum).
 *  [P3]  "Sliding Window Attention" (robocikowo.com), opening definition
 *        paragraph (causal window [i-W+1, i], symmetric [i-W/2, i+W/2],
 *        -inf logits before the softmax), glossary entries for the binary
 *        mask, the rolling KV buffer (FIFO) and global tokens.
 *  [P4]  "Sliding Window Attention" (Ultralytics glossary), section on how
 *        the window grows with depth (boolean mask, mask products for reach)
 *        and the ring-buffer paragraph (position i goes to slot i mod w).
 *
 * Layouts (the pages fix none): q, o [B,T,Hq,d]; k, v [B,T,Hkv,d];
 * lse [B,Hq,T]; ring caches [B,Hkv,W,d]; decode q/o [B,Hq,d].
 * Grouped-query heads: query head h reads kv head floor(h*Hkv/Hq).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_CAUSAL 0
#define ORACLE_SYMMETRIC 1
#define ORACLE_SINKS 2
#define ORACLE_VARLEN 3

/* ---------------------------------------------------------------- masks -- */

/* Window membership of key j for query i [P3 opening paragraph; P2 s.3, 4.1].
 * causal:    i-W+1 <= j <= i   (W keys including the query itself)
 * symmetric: i-W/2 <= j <= i+W/2 with W/2 rounded down
 * Positions outside [0,T) are never keys. */
int oracle_in_window(long i, long j, long T, long W, int mode)
{
    if (j < 0 || j >= T || i < 0 || i >= T) return 0;
    if (mode == ORACLE_CAUSAL) return (j <= i) && (j >= i - W + 1);
    long h = W / 2;
    return (j >= i - h) && (j <= i + h);
}

static int is_global(long x, const int32_t *gidx, long g)
{
    for (long c = 0; c < g; c++)
        if (gidx[c] == x) return 1;
    return 0;
}

/* Longformer-style visibility [P2 s.4.3; P3 glossary entry on global
 * tokens]: a global token sees every token and every token sees it; all other
 * pairs follow the symmetric window. */
int oracle_allowed(long i, long j, long T, long W, int mode, const int32_t *gidx, long g)
{
    if (j < 0 || j >= T || i < 0 || i >= T) return 0;
    if (g > 0 && (is_global(i, gidx, g) || is_global(j, gidx, g))) return 1;
    return oracle_in_window(i, j, T, W, mode);
}

/* Causal window plus attention sinks [P4 related-terms entry on attention
 * sinks: StreamingLLM keeps the first tokens of a sequence in the cache
 * beside the window]: query i sees key j <= i when j lies in the window
 * (j >= i-W+1) or is one of the first s tokens (j < s). */
int oracle_sink_allowed(long i, long j, long T, long W, long s)
{
    if (j < 0 || j >= T || i < 0 || i >= T || j > i) return 0;
    return j >= i - W + 1 || j < s;
}

/* Packed variable-length batch, one causal window per sequence [P3 opening
 * definition: query i sees keys i-W+1 .. i; P4 section on alternating local
 * and global layers: Gemma 2 used a 4,096-token window and Gemma 3 a
 * 1,024-token one, so one batch may hold sequences whose windows differ].
 * Packed rows cu[s] .. cu[s+1]-1 hold sequence s.  Row r of sequence s sees
 * packed row j when j belongs to the same sequence and r - wseq[s] + 1 <= j
 * <= r.  A row outside every sequence sees nothing. */
int oracle_varlen_allowed(long r, long j, const int32_t *cu, long nseq, const int32_t *wseq)
{
    for (long s = 0; s < nseq; s++) {
        if (r < cu[s] || r >= cu[s + 1]) continue;
        if (j < cu[s] || j >= cu[s + 1]) return 0;
        return j <= r && j >= r - (long)wseq[s] + 1;
    }
    return 0;
}

/* Pairs the packed batch allows, counted cell by cell over [total,total]. */
long long oracle_count_pairs_varlen(const int32_t *cu, long nseq, const int32_t *wseq)
{
    const long total = nseq > 0 ? cu[nseq] : 0;
    long long n = 0;
    for (long r = 0; r < total; r++)
        for (long j = 0; j < total; j++) n += oracle_varlen_allowed(r, j, cu, nseq, wseq);
    return n;
}

/* Dilated window [P2 s.4.2: instead of all W neighbours, every dil-th token
 * is taken, which widens the span without more keys].  Causal: keys
 * i - dil*m for m = 0..W-1; symmetric: keys i + dil*m for |m| <= W/2.  The
 * page's worked example is garbled (its key count and span disagree); the
 * reading taken keeps W keys (W/2 per side) and stretches the span by dil. */
int oracle_dilated_allowed(long i, long j, long T, long W, long dil, int mode)
{
    if (j < 0 || j >= T || i < 0 || i >= T || dil < 1) return 0;
    const long diff = i - j;
    if (diff % dil != 0) return 0;
    const long m = diff / dil;
    if (mode == ORACLE_CAUSAL) return m >= 0 && m <= W - 1;
    const long h = W / 2;
    return m >= -h && m <= h;
}

long long oracle_count_pairs_dilated(long T, long W, long dil, int mode)
{
    long long n = 0;
    for (long i = 0; i < T; i++)
        for (long j = 0; j < T; j++) n += oracle_dilated_allowed(i, j, T, W, dil, mode);
    return n;
}

/* Pairs a causal window with s sinks allows. */
long long oracle_count_pairs_sinks(long T, long W, long s)
{
    long long n = 0;
    for (long i = 0; i < T; i++)
        for (long j = 0; j < T; j++) n += oracle_sink_allowed(i, j, T, W, s);
    return n;
}

/* The explicit [T,T] boolean mask (the brute-force form the pages warn
 * against for large T; here it is only a checker) [P3 binary-mask entry;
 * P4 depth section]. */
void oracle_mask(uint8_t *out, long T, long W, int mode, const int32_t *gidx, long g)
{
    for (long i = 0; i < T; i++)
        for (long j = 0; j < T; j++)
            out[i * T + j] = (uint8_t)oracle_allowed(i, j, T, W, mode, gidx, g);
}

/* Number of allowed (query, key) pairs = number of scores one layer computes
 * [P4 depth section: 58 with the window against 136 fully causal, T=16, W=4]. */
long long oracle_count_pairs(long T, long W, int mode, const int32_t *gidx, long g)
{
    long long n = 0;
    for (long i = 0; i < T; i++)
        for (long j = 0; j < T; j++) n += oracle_allowed(i, j, T, W, mode, gidx, g);
    return n;
}

/* Reach of the last token through L stacked causal window layers [P4 depth
 * section]: reach_1 = mask, reach_{l+1} = (mask x reach_l) > 0 as boolean
 * matrices; out[l-1] = number of tokens the last row of reach_l touches. */
int oracle_reach(int32_t *out, long T, long W, int L)
{
    uint8_t *m = malloc((size_t)T * T), *r = malloc((size_t)T * T), *t = malloc((size_t)T * T);
    if (!m || !r || !t) { free(m); free(r); free(t); return -1; }
    oracle_mask(m, T, W, ORACLE_CAUSAL, NULL, 0);
    memcpy(r, m, (size_t)T * T);
    for (int l = 0; l < L; l++) {
        long cnt = 0;
        for (long j = 0; j < T; j++) cnt += r[(T - 1) * T + j];
        out[l] = (int32_t)cnt;
        for (long i = 0; i < T; i++)
            for (long j = 0; j < T; j++) {
                int any = 0;
                for (long k = 0; k < T && !any; k++) any = m[i * T + k] && r[k * T + j];
                t[i * T + j] = (uint8_t)any;
            }
        memcpy(r, t, (size_t)T * T);
    }
    free(m); free(r); free(t);
    return 0;
}

/* ------------------------------------------------------------ ring cache -- */

/* Ring slot of absolute position pos in a W-slot cache [P4 ring-buffer
 * paragraph: position i is stored in slot i mod w]. */
long oracle_slot(long pos, long W) { return pos % W; }

/* Append n new tokens per sequence, one after the other, oldest first; each
 * write replaces whatever the slot held (FIFO overwrite) [P3 rolling-buffer
 * entry; P4 ring-buffer paragraph].  kn/vn [B,n,Hkv,d]; caches [B,Hkv,W,d];
 * pos[b] is the absolute position of token 0 of the batch row; slot_out
 * (nullable) [B,n] receives the slot each token was written to. */
void oracle_ring_append(double *kc, double *vc, const double *kn, const double *vn,
                        const int32_t *pos, int32_t *slot_out,
                        long B, long n, long Hkv, long d, long W)
{
    for (long b = 0; b < B; b++)
        for (long t = 0; t < n; t++) {
            long s = oracle_slot((long)pos[b] + t, W);
            if (slot_out) slot_out[b * n + t] = (int32_t)s;
            for (long h = 0; h < Hkv; h++) {
                const double *ksrc = kn + ((b * n + t) * Hkv + h) * d;
                const double *vsrc = vn + ((b * n + t) * Hkv + h) * d;
                double *kdst = kc + ((b * Hkv + h) * W + s) * d;
                double *vdst = vc + ((b * Hkv + h) * W + s) * d;
                for (long e = 0; e < d; e++) { kdst[e] = ksrc[e]; vdst[e] = vsrc[e]; }
            }
        }
}

/* Paged ring: the W slots of a sequence's ring live in W/P pages of P slots
 * taken from a shared pool, in any order [P4 ring-buffer paragraph: position
 * i goes to slot i mod w, overwriting the oldest entry; P5 check-yourself
 * question 1: the cache holds only the window, so a sequence never needs more
 * than W slots].  Pool [num_pages,Hkv,P,d]; table [B, W/P]: ring slot s of
 * sequence b is row s mod P of page table[b, s / P].  Returns the address of
 * that row for kv head h, or NULL when the table names no page of the pool. */
static double *paged_row(double *pool, const int32_t *table, long b, long h, long s, long Hkv, long d, long W,
                         long P, long num_pages)
{
    const long page = table[b * (W / P) + s / P];
    if (page < 0 || page >= num_pages) return NULL;
    return pool + ((page * Hkv + h) * P + s % P) * d;
}

/* Append into a paged ring: token t of sequence b (position pos[b]+t) goes to
 * ring slot (pos[b]+t) mod W, i.e. into its page as paged_row says; tokens
 * are written one after the other, oldest first (FIFO overwrite) [P3
 * rolling-buffer entry].  Returns -1 if a slot's page is outside the pool
 * (nothing is written for that token). */
int oracle_paged_append(double *kp, double *vp, const double *kn, const double *vn, const int32_t *pos,
                        const int32_t *table, int32_t *slot_out, long B, long n, long Hkv, long d, long W, long P,
                        long num_pages)
{
    int rc = 0;
    for (long b = 0; b < B; b++)
        for (long t = 0; t < n; t++) {
            const long s = oracle_slot((long)pos[b] + t, W);
            if (slot_out) slot_out[b * n + t] = (int32_t)s;
            for (long h = 0; h < Hkv; h++) {
                double *kd = paged_row(kp, table, b, h, s, Hkv, d, W, P, num_pages);
                double *vd = paged_row(vp, table, b, h, s, Hkv, d, W, P, num_pages);
                if (!kd || !vd) { rc = -1; continue; }
                const double *ksrc = kn + ((b * n + t) * Hkv + h) * d;
                const double *vsrc = vn + ((b * n + t) * Hkv + h) * d;
                for (long e = 0; e < d; e++) { kd[e] = ksrc[e]; vd[e] = vsrc[e]; }
            }
        }
    return rc;
}

/* ------------------------------------------------------ one attention row -- */

/* Softmax-weighted sum over an explicit key list [P2 s.9: scores, forbidden
 * positions at -inf, softmax, weighted sum; P3: the -inf logits drop out of
 * the softmax, so only listed keys contribute].  krows/vrows point at the
 * key/value rows in list order.  Writes o[d] and *lse (natural log of the sum
 * of exp(score)).  An empty list gives o = 0 and lse = -inf. */
static void attend_row(const double *q, const double *const *krows, const double *const *vrows,
                       long nkeys, long d, double scale, double *o, double *lse, double *s)
{
    for (long e = 0; e < d; e++) o[e] = 0.0;
    if (nkeys == 0) { *lse = -INFINITY; return; }
    double m = -INFINITY;
    for (long c = 0; c < nkeys; c++) {
        double acc = 0.0;
        for (long e = 0; e < d; e++) acc += q[e] * krows[c][e];
        s[c] = scale * acc;
        if (s[c] > m) m = s[c];
    }
    double l = 0.0;
    for (long c = 0; c < nkeys; c++) {
        double p = exp(s[c] - m);
        l += p;
        for (long e = 0; e < d; e++) o[e] += p * vrows[c][e];
    }
    for (long e = 0; e < d; e++) o[e] /= l;
    *lse = m + log(l);
}

/* ---------------------------------------------------------------- prefill -- */

typedef struct {
    const double *q, *k, *v;
    double *o, *lse;
    long B, T, Hq, Hkv, d, W;
    int mode;
    const int32_t *gidx; /* [B,g] or NULL */
    long g;
    long sinks;          /* causal window plus the first `sinks` tokens (mode ORACLE_SINKS) */
    long dil;            /* dilation (> 1: modes ORACLE_DILATED_*) */
    double scale;
    const int64_t *rows; /* flattened (b*Hq + h)*T + i */
    long nrows;
    long next;           /* work counter */
    pthread_mutex_t mu;
    const int32_t *cu;   /* packed sequences (mode ORACLE_VARLEN): offsets [nseq+1] */
    long nseq;
    const int32_t *wseq; /* window of each sequence [nseq] */
} prefill_job;

static void prefill_one(prefill_job *J, long r, const double **kr, const double **vr, double *s)
{
    long flat = (long)J->rows[r];
    long i = flat % J->T;
    long bh = flat / J->T;
    long h = bh % J->Hq, b = bh / J->Hq;
    long hk = h * J->Hkv / J->Hq; /* grouped-query head mapping */
    const int32_t *gb = J->gidx ? J->gidx + b * J->g : NULL;
    long n = 0;
    for (long j = 0; j < J->T; j++) {
        int ok;
        if (J->mode == ORACLE_SINKS) ok = oracle_sink_allowed(i, j, J->T, J->W, J->sinks);
        else if (J->mode == ORACLE_VARLEN) ok = oracle_varlen_allowed(i, j, J->cu, J->nseq, J->wseq);
        else if (J->dil > 1) ok = oracle_dilated_allowed(i, j, J->T, J->W, J->dil, J->mode);
        else ok = oracle_allowed(i, j, J->T, J->W, J->mode, gb, gb ? J->g : 0);
        if (!ok) continue;
        kr[n] = J->k + ((b * J->T + j) * J->Hkv + hk) * J->d;
        vr[n] = J->v + ((b * J->T + j) * J->Hkv + hk) * J->d;
        n++;
    }
    const double *qrow = J->q + ((b * J->T + i) * J->Hq + h) * J->d;
    double lse;
    attend_row(qrow, kr, vr, n, J->d, J->scale, J->o + r * J->d, &lse, s);
    if (J->lse) J->lse[r] = lse;
}

static void *prefill_worker(void *arg)
{
    prefill_job *J = (prefill_job *)arg;
    const double **kr = malloc(sizeof(double *) * (size_t)J->T);
    const double **vr = malloc(sizeof(double *) * (size_t)J->T);
    double *s = malloc(sizeof(double) * (size_t)J->T);
    for (;;) {
        pthread_mutex_lock(&J->mu);
        long r = J->next;
        J->next += 16;
        pthread_mutex_unlock(&J->mu);
        if (r >= J->nrows) break;
        long e = r + 16 < J->nrows ? r + 16 : J->nrows;
        for (; r < e; r++) prefill_one(J, r, kr, vr, s);
    }
    free(kr); free(vr); free(s);
    return NULL;
}

static int run_prefill(prefill_job *J, int nthreads)
{
    if (nthreads < 1) nthreads = 1;
    J->next = 0;
    pthread_mutex_init(&J->mu, NULL);
    pthread_t *th = malloc(sizeof(pthread_t) * (size_t)nthreads);
    for (int t = 0; t < nthreads; t++) pthread_create(&th[t], NULL, prefill_worker, J);
    for (int t = 0; t < nthreads; t++) pthread_join(th[t], NULL);
    free(th);
    pthread_mutex_destroy(&J->mu);
    return 0;
}

/* Causal sliding-window prefill [P3 opening paragraph; P2 s.3]: for each
 * requested row (b, h, i) the keys j with i-W+1 <= j <= i of kv head
 * floor(h*Hkv/Hq).  o: [nrows, d]; lse (nullable): [nrows]. */
int oracle_swa_prefill(const double *q, const double *k, const double *v, double *o, double *lse,
                       long B, long T, long Hq, long Hkv, long d, long W, double scale,
                       const int64_t *rows, long nrows, int nthreads)
{
    prefill_job J = {q, k, v, o, lse, B, T, Hq, Hkv, d, W, ORACLE_CAUSAL, NULL, 0, 0, 1, scale, rows, nrows};
    return run_prefill(&J, nthreads);
}

/* Symmetric window plus global tokens [P2 s.4.1, 4.3; P3 global-token
 * entry].  gidx [B,g] lists the global positions of each sequence (g may be
 * 0: plain symmetric window). */
int oracle_swa_prefill_global(const double *q, const double *k, const double *v, double *o, double *lse,
                              const int32_t *gidx, long g,
                              long B, long T, long Hq, long Hkv, long d, long W, double scale,
                              const int64_t *rows, long nrows, int nthreads)
{
    prefill_job J = {q, k, v, o, lse, B, T, Hq, Hkv, d, W, ORACLE_SYMMETRIC, g > 0 ? gidx : NULL, g, 0, 1, scale, rows, nrows};
    return run_prefill(&J, nthreads);
}

/* Causal window plus the first s tokens as attention sinks [P4 related-terms
 * entry on attention sinks; P3 opening definition for the window]. */
int oracle_swa_prefill_sinks(const double *q, const double *k, const double *v, double *o, double *lse,
                             long B, long T, long Hq, long Hkv, long d, long W, long s, double scale,
                             const int64_t *rows, long nrows, int nthreads)
{
    prefill_job J = {q, k, v, o, lse, B, T, Hq, Hkv, d, W, ORACLE_SINKS, NULL, 0, s, 1, scale, rows, nrows};
    return run_prefill(&J, nthreads);
}

/* Dilated window, causal (mode 0) or symmetric (mode 1) [P2 s.4.2]; the
 * keys of each row are those oracle_dilated_allowed admits. */
int oracle_swa_prefill_dilated(const double *q, const double *k, const double *v, double *o, double *lse,
                               long B, long T, long Hq, long Hkv, long d, long W, long dil, int mode,
                               double scale, const int64_t *rows, long nrows, int nthreads)
{
    if (dil < 1 || (mode != ORACLE_CAUSAL && mode != ORACLE_SYMMETRIC)) return -1;
    prefill_job J = {q, k, v, o, lse, B, T, Hq, Hkv, d, W, mode, NULL, 0, 0, dil, scale, rows, nrows};
    return run_prefill(&J, nthreads);
}

/* Packed variable-length prefill with one window per sequence (see
 * oracle_varlen_allowed): q, o [total,Hq,d]; k, v [total,Hkv,d]; rows are
 * flattened h*total + r; o [nrows,d], lse (nullable) [nrows]. */
int oracle_swa_prefill_varlen(const double *q, const double *k, const double *v, double *o, double *lse,
                              const int32_t *cu, long nseq, const int32_t *wseq, long total, long Hq, long Hkv,
                              long d, double scale, const int64_t *rows, long nrows, int nthreads)
{
    if (nseq < 0 || (nseq > 0 && cu[nseq] != total)) return -1;
    for (long s = 0; s < nseq; s++)
        if (cu[s] > cu[s + 1] || wseq[s] < 1) return -1;
    prefill_job J = {q, k, v, o, lse, 1, total, Hq, Hkv, d, 0, ORACLE_VARLEN, NULL, 0, 0, 1, scale, rows, nrows};
    J.cu = cu;
    J.nseq = nseq;
    J.wseq = wseq;
    return run_prefill(&J, nthreads);
}

/* ----------------------------------------------------------------- decode -- */

/* One decode step over the ring cache [P4 ring-buffer paragraph; P5
 * "Sliding-window and hybrid attention", check-yourself question 1: only the
 * latest W tokens are kept].  The token at position pos[b] is already in the
 * cache, so the visible positions are max(0,pos-W+1)..pos, which occupy slots
 * 0..min(pos+1,W)-1 of the ring.  q/o [B,Hq,d]; caches [B,Hkv,W,d];
 * lse (nullable) [B,Hq]. */
int oracle_swa_decode(const double *q, const double *kc, const double *vc, const int32_t *pos,
                      double *o, double *lse, long B, long Hq, long Hkv, long d, long W, double scale)
{
    const double **kr = malloc(sizeof(double *) * (size_t)W);
    const double **vr = malloc(sizeof(double *) * (size_t)W);
    double *s = malloc(sizeof(double) * (size_t)W);
    for (long b = 0; b < B; b++) {
        long nvalid = (long)pos[b] + 1 < W ? (long)pos[b] + 1 : W;
        if (pos[b] < 0) nvalid = 0;
        for (long h = 0; h < Hq; h++) {
            long hk = h * Hkv / Hq;
            for (long sl = 0; sl < nvalid; sl++) {
                kr[sl] = kc + ((b * Hkv + hk) * W + sl) * d;
                vr[sl] = vc + ((b * Hkv + hk) * W + sl) * d;
            }
            double l;
            attend_row(q + (b * Hq + h) * d, kr, vr, nvalid, d, scale, o + (b * Hq + h) * d, &l, s);
            if (lse) lse[b * Hq + h] = l;
        }
    }
    free(kr); free(vr); free(s);
    return 0;
}

/* One decode step over a paged ring (see paged_row): the current token at
 * position pos[b] is already appended; the visible keys are ring slots
 * 0 .. min(pos+1,W)-1, in slot order, each read through the page table [P4
 * ring-buffer paragraph].  Returns -1 for a negative position or a page
 * outside the pool. */
int oracle_swa_decode_paged(const double *q, const double *kp, const double *vp, const int32_t *table,
                            const int32_t *pos, double *o, double *lse, long B, long Hq, long Hkv, long d, long W,
                            long P, long num_pages, double scale)
{
    for (long b = 0; b < B; b++)
        if (pos[b] < 0) return -1;
    const double **kr = malloc(sizeof(double *) * (size_t)W);
    const double **vr = malloc(sizeof(double *) * (size_t)W);
    double *sc = malloc(sizeof(double) * (size_t)W);
    int rc = 0;
    for (long b = 0; b < B && rc == 0; b++) {
        const long nvalid = (long)pos[b] + 1 < W ? (long)pos[b] + 1 : W;
        for (long h = 0; h < Hq && rc == 0; h++) {
            const long hk = h * Hkv / Hq;
            for (long sl = 0; sl < nvalid; sl++) {
                kr[sl] = paged_row((double *)kp, table, b, hk, sl, Hkv, d, W, P, num_pages);
                vr[sl] = paged_row((double *)vp, table, b, hk, sl, Hkv, d, W, P, num_pages);
                if (!kr[sl] || !vr[sl]) rc = -1;
            }
            if (rc) break;
            double l;
            attend_row(q + (b * Hq + h) * d, kr, vr, nvalid, d, scale, o + (b * Hq + h) * d, &l, sc);
            if (lse) lse[b * Hq + h] = l;
        }
    }
    free(kr); free(vr); free(sc);
    return rc;
}

/* ---------------------------------------------------------- chunk prefill -- */

/* Prefill of n new tokens at positions pos[b] .. pos[b]+n-1 that continue a
 * sequence whose earlier tokens live in the W-slot ring [P4 ring-buffer
 * paragraph: position p sits in slot p mod W and only the latest W tokens
 * are kept; P3 opening definition: query P sees the keys at positions
 * P-W+1 .. P].  Keys at positions >= pos[b] are rows of the chunk itself;
 * earlier ones are read from ring slot (position mod W), which holds them as
 * long as the chunk has not been appended yet.  Keys in list order of
 * position.  q/o [B,n,Hq,d]; k/v [B,n,Hkv,d]; caches [B,Hkv,W,d];
 * lse (nullable) [B,Hq,n].  Returns -1 for a negative position. */
int oracle_swa_prefill_chunk(const double *q, const double *k, const double *v, const double *kc,
                             const double *vc, const int32_t *pos, double *o, double *lse, long B, long n,
                             long Hq, long Hkv, long d, long W, double scale)
{
    for (long b = 0; b < B; b++)
        if (pos[b] < 0) return -1;
    const double **kr = malloc(sizeof(double *) * (size_t)W);
    const double **vr = malloc(sizeof(double *) * (size_t)W);
    double *s = malloc(sizeof(double) * (size_t)W);
    for (long b = 0; b < B; b++) {
        const long p0 = pos[b];
        for (long h = 0; h < Hq; h++) {
            const long hk = h * Hkv / Hq;
            for (long t = 0; t < n; t++) {
                const long P = p0 + t;
                const long lo = P - W + 1 > 0 ? P - W + 1 : 0;
                long nk = 0;
                for (long j = lo; j <= P; j++) {
                    if (j >= p0) {
                        kr[nk] = k + ((b * n + (j - p0)) * Hkv + hk) * d;
                        vr[nk] = v + ((b * n + (j - p0)) * Hkv + hk) * d;
                    } else {
                        const long sl = oracle_slot(j, W);
                        kr[nk] = kc + ((b * Hkv + hk) * W + sl) * d;
                        vr[nk] = vc + ((b * Hkv + hk) * W + sl) * d;
                    }
                    nk++;
                }
                double l;
                attend_row(q + ((b * n + t) * Hq + h) * d, kr, vr, nk, d, scale, o + ((b * n + t) * Hq + h) * d,
                           &l, s);
                if (lse) lse[(b * Hq + h) * n + t] = l;
            }
        }
    }
    free(kr); free(vr); free(s);
    return 0;
}

/* One decode step with attention sinks beside the ring [P4 related-terms
 * entry: StreamingLLM keeps the first tokens in the cache beside the window;
 * P4 ring-buffer paragraph].  The token at position P = pos[b] is already in
 * the ring, whose filled slots 0..min(P+1,W)-1 hold the window; the sink
 * caches [B,Hkv,s,d] hold positions 0..s-1, of which those older than the
 * window (position < P-W+1) are added; the others are still in the ring and
 * count once.  Keys in list order: sinks, then ring slots. */
int oracle_swa_decode_sinks(const double *q, const double *kc, const double *vc, const double *ks,
                            const double *vs, const int32_t *pos, double *o, double *lse, long B, long Hq,
                            long Hkv, long d, long W, long s, double scale)
{
    for (long b = 0; b < B; b++)
        if (pos[b] < 0) return -1;
    const double **kr = malloc(sizeof(double *) * (size_t)(W + s));
    const double **vr = malloc(sizeof(double *) * (size_t)(W + s));
    double *sc = malloc(sizeof(double) * (size_t)(W + s));
    for (long b = 0; b < B; b++) {
        const long P = pos[b];
        const long nvalid = P + 1 < W ? P + 1 : W;
        long nsink = P - W + 1 < s ? P - W + 1 : s;
        if (nsink < 0) nsink = 0;
        for (long h = 0; h < Hq; h++) {
            const long hk = h * Hkv / Hq;
            long n = 0;
            for (long j = 0; j < nsink; j++, n++) {
                kr[n] = ks + ((b * Hkv + hk) * s + j) * d;
                vr[n] = vs + ((b * Hkv + hk) * s + j) * d;
            }
            for (long sl = 0; sl < nvalid; sl++, n++) {
                kr[n] = kc + ((b * Hkv + hk) * W + sl) * d;
                vr[n] = vc + ((b * Hkv + hk) * W + sl) * d;
            }
            double l;
            attend_row(q + (b * Hq + h) * d, kr, vr, n, d, scale, o + (b * Hq + h) * d, &l, sc);
            if (lse) lse[b * Hq + h] = l;
        }
    }
    free(kr); free(vr); free(sc);
    return 0;
}

/* -------------------------------------------------------------- backward -- */

/* Gradient of the sliding-window prefill (the causal or symmetric window of
 * [P3 opening paragraph; P2 s.3, 4.1]) with respect to q, k and v, for an
 * upstream gradient dO.  The pages define only the forward computation; this
 * is that definition differentiated by the chain rule, row by row:
 *   s_j  = scale q_i.k_j for j in the window,  p = softmax(s),  o_i = sum p_j v_j
 *   dv_j += p_j dO_i
 *   dp_j  = dO_i . v_j,   D = sum_j p_j dp_j  (= dO_i . o_i)
 *   ds_j  = p_j (dp_j - D)
 *   dq_i  = scale sum_j ds_j k_j,   dk_j += scale ds_j q_i
 * Grouped-query heads: a kv head's dk, dv sum the rows of all its query heads.
 * Every sum is an fp64 sum in index order.  Work is split over (b, kv head)
 * so that each thread owns its dk, dv rows. */
typedef struct {
    const double *q, *k, *v, *dout;
    double *dq, *dk, *dv;
    long B, T, Hq, Hkv, d, W;
    int mode;
    double scale;
    long next;
    pthread_mutex_t mu;
} backward_job;

static void backward_group(backward_job *J, long b, long hk, long *keys, double *s, double *dp)
{
    const long T = J->T, d = J->d, Hq = J->Hq, Hkv = J->Hkv;
    for (long h = 0; h < Hq; h++) {
        if (h * Hkv / Hq != hk) continue;
        for (long i = 0; i < T; i++) {
            const double *qi = J->q + ((b * T + i) * Hq + h) * d;
            const double *gi = J->dout + ((b * T + i) * Hq + h) * d;
            double *dqi = J->dq + ((b * T + i) * Hq + h) * d;
            long n = 0;
            for (long j = 0; j < T; j++)
                if (oracle_in_window(i, j, T, J->W, J->mode)) keys[n++] = j;
            /* probabilities, two-pass */
            double m = -INFINITY;
            for (long c = 0; c < n; c++) {
                const double *kj = J->k + ((b * T + keys[c]) * Hkv + hk) * d;
                double acc = 0.0;
                for (long e = 0; e < d; e++) acc += qi[e] * kj[e];
                s[c] = J->scale * acc;
                if (s[c] > m) m = s[c];
            }
            double l = 0.0;
            for (long c = 0; c < n; c++) {
                s[c] = exp(s[c] - m);
                l += s[c];
            }
            for (long c = 0; c < n; c++) s[c] /= l;
            /* dp_j = dO_i . v_j and D = sum p_j dp_j */
            double D = 0.0;
            for (long c = 0; c < n; c++) {
                const double *vj = J->v + ((b * T + keys[c]) * Hkv + hk) * d;
                double acc = 0.0;
                for (long e = 0; e < d; e++) acc += gi[e] * vj[e];
                dp[c] = acc;
                D += s[c] * acc;
            }
            for (long e = 0; e < d; e++) dqi[e] = 0.0;
            for (long c = 0; c < n; c++) {
                const double ds = s[c] * (dp[c] - D);
                const double *kj = J->k + ((b * T + keys[c]) * Hkv + hk) * d;
                double *dkj = J->dk + ((b * T + keys[c]) * Hkv + hk) * d;
                double *dvj = J->dv + ((b * T + keys[c]) * Hkv + hk) * d;
                for (long e = 0; e < d; e++) {
                    dqi[e] += J->scale * ds * kj[e];
                    dkj[e] += J->scale * ds * qi[e];
                    dvj[e] += s[c] * gi[e];
                }
            }
        }
    }
}

static void *backward_worker(void *arg)
{
    backward_job *J = (backward_job *)arg;
    long *keys = malloc(sizeof(long) * (size_t)J->T);
    double *s = malloc(sizeof(double) * (size_t)J->T);
    double *dp = malloc(sizeof(double) * (size_t)J->T);
    for (;;) {
        pthread_mutex_lock(&J->mu);
        long u = J->next++;
        pthread_mutex_unlock(&J->mu);
        if (u >= J->B * J->Hkv) break;
        backward_group(J, u / J->Hkv, u % J->Hkv, keys, s, dp);
    }
    free(keys); free(s); free(dp);
    return NULL;
}

/* dq [B,T,Hq,d], dk and dv [B,T,Hkv,d] (all overwritten) for q, k, v, dout in
 * the prefill layouts; mode ORACLE_CAUSAL or ORACLE_SYMMETRIC. */
int oracle_swa_backward(const double *q, const double *k, const double *v, const double *dout, double *dq,
                        double *dk, double *dv, long B, long T, long Hq, long Hkv, long d, long W, int mode,
                        double scale, int nthreads)
{
    if (mode != ORACLE_CAUSAL && mode != ORACLE_SYMMETRIC) return -1;
    memset(dk, 0, sizeof(double) * (size_t)(B * T * Hkv * d));
    memset(dv, 0, sizeof(double) * (size_t)(B * T * Hkv * d));
    backward_job J = {q, k, v, dout, dq, dk, dv, B, T, Hq, Hkv, d, W, mode, scale};
    if (nthreads < 1) nthreads = 1;
    J.next = 0;
    pthread_mutex_init(&J.mu, NULL);
    pthread_t *th = malloc(sizeof(pthread_t) * (size_t)nthreads);
    for (int t = 0; t < nthreads; t++) pthread_create(&th[t], NULL, backward_worker, &J);
    for (int t = 0; t < nthreads; t++) pthread_join(th[t], NULL);
    free(th);
    pthread_mutex_destroy(&J.mu);
    return 0;
}

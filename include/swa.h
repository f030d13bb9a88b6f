/*
 * swa.h: sliding-window attention on NVIDIA B200 (sm_100a), C ABI.
 *
 * The method (as the pages define it):
 *  - A causal window lets query i see keys i-W+1 .. i: W keys, itself
 *    included ("Sliding Window Attention", robocikowo.com, opening
 *    definition; "How sliding window attention works in Mistral and
 *    Longformer", aivaro.ru, section 3).
 *  - A symmetric window lets query i see keys i-W/2 .. i+W/2 (W/2 rounded
 *    down; up to W+1 keys); Longformer adds global tokens that see every
 *    token and are seen by every token (aivaro.ru, sections 4.1 and 4.3).
 *  - Scores outside the window are -inf before the softmax, so they take no
 *    part in it, and the [T,T] score matrix is never formed (robocikowo.com,
 *    opening definition; aivaro.ru, section 9).
 *  - Decode keeps a ring of W key/value slots per sequence and head; position
 *    p lives in slot p mod W, overwriting the oldest entry ("Sliding Window
 *    Attention", Ultralytics glossary, ring-buffer paragraph).
 *
 * Conventions for every call:
 *  - Every buffer is owned by the caller and lives in device memory unless a
 *    parameter says otherwise.  The library never allocates device memory
 *    at run time; its device code holds two static arrays (a status word and
 *    the 16 MiB scratch of swa_decode_noalloc) on each GPU it is loaded on.
 *  - Tensors are dense, row-major, 16-byte aligned, with the layouts given
 *    below (innermost dimension last).  B batch, T sequence length, Hq query
 *    heads, Hkv key/value heads (Hq % Hkv == 0; query head h reads kv head
 *    h / (Hq/Hkv)), d head dimension, W window.
 *  - bf16 calls run on tcgen05 tensor cores (prefill) or as vectorised SIMT
 *    (decode); fp32 calls run as SIMT fp32 FMA.  Accumulation is fp32 in
 *    both, and bf16 outputs are rounded to nearest even.
 *  - Every compute call is asynchronous on `stream` (a cudaStream_t passed as
 *    void*; NULL is the legacy default stream).  Argument errors are detected
 *    on the host before anything is launched and return SWA_ERR_INVALID_ARG
 *    or SWA_ERR_UNSUPPORTED; launch failures return SWA_ERR_CUDA.  Errors
 *    found on the device (a bounded wait that expired, a negative position)
 *    are recorded in a per-device status word that swa_get_device_status
 *    reads.  No call aborts the process.
 */
#ifndef SWA_H
#define SWA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SWA_OK = 0,
    SWA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, Hq % Hkv != 0 ... */
    SWA_ERR_UNSUPPORTED = 2, /* valid request the library has no kernel for (e.g. d) */
    SWA_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
    SWA_ERR_TIMEOUT = 4,     /* a kernel's bounded wait expired; its outputs are invalid */
    SWA_ERR_INTERNAL = 5     /* debug build only: a device-side index check failed */
} swa_status;

typedef enum {
    SWA_DTYPE_F32 = 0,
    SWA_DTYPE_BF16 = 1
} swa_dtype;

/*
 * Causal sliding-window prefill with grouped-query heads.
 *   o[b,i,h,:] = sum over j in [max(0,i-W+1), i] of
 *                softmax_j(scale * q[b,i,h,:].k[b,j,hk,:]) * v[b,j,hk,:]
 * with hk = h / (Hq/Hkv)  (robocikowo.com opening definition; aivaro.ru s.3).
 *   q, o : [B,T,Hq,d]   k, v : [B,T,Hkv,d]   dtype dt for all four
 *   lse  : nullable, fp32 [B,Hq,T], natural-log sum of exp(score) per row
 *   W >= 1 (W >= T is plain causal attention).  scale is normally 1/sqrt(d).
 *   bf16: d in {32, 64, 128}.  fp32: d <= 128 and d % 4 == 0.
 */
swa_status swa_prefill(const void *q, const void *k, const void *v, void *o, float *lse,
                       int B, int T, int Hq, int Hkv, int d, int W, float scale,
                       swa_dtype dt, void *stream);

/*
 * Longformer-style bidirectional prefill: symmetric window plus g global
 * tokens (aivaro.ru sections 4.1 and 4.3; robocikowo.com global-token entry).
 *   Row i not global: keys j with |i-j| <= W/2, together with every global
 *   position (a global key inside the band counts once).
 *   Row i global: every key 0..T-1.
 *   global_idx : device int32 [B,g], per-sequence positions, strictly
 *                increasing, each in [0,T); g may be 0 (then global_idx may be
 *                NULL).  Unsorted or out-of-range entries are undefined.
 *   Other arguments as swa_prefill; W >= 1 (half-width W/2 rounded down).
 */
swa_status swa_prefill_global(const void *q, const void *k, const void *v, void *o, float *lse,
                              const int32_t *global_idx, int g,
                              int B, int T, int Hq, int Hkv, int d, int W, float scale,
                              swa_dtype dt, void *stream);

/*
 * Causal sliding-window prefill over packed sequences of different lengths
 * (variable-length batches), each with its own window if asked: every
 * sequence is its own causal prefill (robocikowo.com opening definition) and
 * no row sees another sequence.  Windows may differ from sequence to sequence
 * the way local layers of different models differ (Ultralytics glossary,
 * section on alternating local and global layers: 4,096 tokens in Gemma 2,
 * 1,024 in Gemma 3).
 *   q, o : [total,Hq,d]   k, v : [total,Hkv,d]   (rows of all sequences, one
 *          after the other)
 *   cu_seqlens : device int32 [nseq+1]: sequence s holds rows cu[s] ..
 *          cu[s+1]-1; cu[0] = 0, non-decreasing, cu[nseq] = total, each
 *          length <= max_seqlen (an entry breaking this makes its sequence
 *          empty and records SWA_ERR_INVALID_ARG in the device status word)
 *   windows : nullable device int32 [nseq]: sequence s uses window
 *          windows[s] >= 1 (an entry below 1 leaves that sequence's rows
 *          untouched and records SWA_ERR_INVALID_ARG in the device status
 *          word); NULL: every sequence uses W
 *   lse  : nullable fp32 [Hq,total]
 *   0 <= max_seqlen <= total; W >= 1 even when `windows` is given; other
 *   arguments as swa_prefill.
 */
swa_status swa_prefill_varlen(const void *q, const void *k, const void *v, void *o, float *lse,
                              const int32_t *cu_seqlens, const int32_t *windows, int nseq, int total,
                              int max_seqlen, int Hq, int Hkv, int d, int W, float scale, swa_dtype dt,
                              void *stream);

/*
 * Dilated sliding-window prefill (aivaro.ru section 4.2: instead of all
 * neighbours, every dil-th token, which widens the span without more keys).
 *   symmetric = 0: query i sees keys i - dil*m, m = 0 .. W-1 (j >= 0)
 *   symmetric = 1: query i sees keys i + dil*m, |m| <= W/2 (0 <= j < T)
 *   The page's worked example is inconsistent (its key count and span
 *   disagree); the window keeps W keys (W/2 per side) and its span grows by
 *   dil.  dil = 1 is swa_prefill (symmetric: swa_prefill_global without
 *   globals) and needs no workspace.
 *   Such a window only pairs positions with equal residues modulo dil, so the
 *   call permutes q, k, v into the dil strided sub-sequences, runs the plain
 *   window on them and permutes o (and lse) back.
 *   workspace : device scratch of swa_prefill_dilated_workspace_bytes(...)
 *               bytes, 256-byte aligned; calls sharing it must not overlap.
 *   Other arguments as swa_prefill.
 */
size_t swa_prefill_dilated_workspace_bytes(int B, int T, int Hq, int Hkv, int d, int dil, swa_dtype dt,
                                           int with_lse);
swa_status swa_prefill_dilated(const void *q, const void *k, const void *v, void *o, float *lse, int dil,
                               int symmetric, int B, int T, int Hq, int Hkv, int d, int W, float scale,
                               swa_dtype dt, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Causal sliding-window prefill with attention sinks: the first n_sink tokens
 * of each sequence stay visible to every later query beside its window
 * (Ultralytics glossary, related-terms entry on attention sinks: StreamingLLM
 * keeps them in the cache beside the window; robocikowo.com opening
 * definition for the window).
 *   o[b,i,h,:] = softmax-weighted sum over the keys j <= i with
 *                j >= i-W+1 or j < n_sink (a sink inside the window counts
 *                once)
 *   n_sink >= 0 (0 is swa_prefill; n_sink >= T makes every row full causal).
 *   Other arguments as swa_prefill.
 */
swa_status swa_prefill_sinks(const void *q, const void *k, const void *v, void *o, float *lse, int n_sink,
                             int B, int T, int Hq, int Hkv, int d, int W, float scale,
                             swa_dtype dt, void *stream);

/*
 * Causal prefill of a chunk of n new tokens that continues sequences whose
 * earlier tokens are already in the W-slot rings: token t of batch row b is
 * at position P = pos[b]+t and sees the keys at positions max(0,P-W+1) .. P
 * (robocikowo.com opening definition).  Keys at positions >= pos[b] are rows
 * of k/v; earlier ones are read from ring slot (position mod W) (Ultralytics
 * ring-buffer paragraph), so the rings must hold positions
 * max(0,pos[b]-W+1) .. pos[b]-1 and must not yet hold the chunk: append the
 * chunk with swa_cache_append after this call.  The pages state no chunked
 * form; it is the causal definition above with the keys split between the
 * ring and the chunk, and equals rows pos[b] .. pos[b]+n-1 of swa_prefill
 * over the whole sequence.
 *   q, o             : [B,n,Hq,d]       k, v : [B,n,Hkv,d]
 *   k_cache, v_cache : [B,Hkv,W,d], read only
 *   pos              : device int32 [B], >= 0 (a negative entry is read as 0
 *                      and records SWA_ERR_INVALID_ARG in the device status
 *                      word)
 *   lse              : nullable fp32 [B,Hq,n]
 *   Other arguments as swa_prefill (bf16: d in {32, 64, 128}; fp32: d <= 128
 *   and d % 4 == 0).
 */
swa_status swa_prefill_chunk(const void *q, const void *k, const void *v, void *o, float *lse,
                             const void *k_cache, const void *v_cache, const int32_t *pos,
                             int B, int n, int Hq, int Hkv, int d, int W, float scale,
                             swa_dtype dt, void *stream);

/*
 * Ring-cache append: token t of batch row b (absolute position pos[b]+t)
 * goes to slot (pos[b]+t) mod W of that row's ring, overwriting the oldest
 * entry (Ultralytics ring-buffer paragraph; robocikowo.com rolling-buffer
 * entry).  When n > W only the last W tokens are written, which leaves the
 * ring exactly as n one-at-a-time appends would.
 *   k_cache, v_cache : [B,Hkv,W,d], updated in place
 *   k_new, v_new     : [B,n,Hkv,d]
 *   pos              : device int32 [B], >= 0 (a negative entry leaves its row
 *                      untouched and records SWA_ERR_INVALID_ARG in the
 *                      device status word)
 *   slot_out         : nullable device int32 [B,n], receives (pos[b]+t) mod W
 *   Any d with d * sizeof(dtype) a multiple of 16.
 */
swa_status swa_cache_append(void *k_cache, void *v_cache, const void *k_new, const void *v_new,
                            const int32_t *pos, int32_t *slot_out,
                            int B, int n, int Hkv, int d, int W, swa_dtype dt, void *stream);

/*
 * Paged ring caches.  The W slots of each sequence's ring need not be one
 * contiguous [W,d] block per kv head: they can live in W/P pages of P slots
 * taken, in any order, from a pool shared by all sequences, the way a serving
 * engine hands out fixed-size cache blocks.  The ring itself is unchanged:
 * position i is ring slot i mod W (Ultralytics ring-buffer paragraph), and a
 * sequence never needs more than W slots (dupenodi.dev, check-yourself
 * question 1); the page table only says where each group of P slots is.
 *   k_pages, v_pages : pools [num_pages,Hkv,P,d] (P = page_size)
 *   page_table       : device int32 [B, W/P]: ring slot s of sequence b is
 *                      row s mod P of page page_table[b*(W/P) + s/P]; an
 *                      entry outside [0,num_pages) is recorded as
 *                      SWA_ERR_INVALID_ARG in the device status word (append:
 *                      that token is not written; decode: page 0 is read
 *                      instead and the output is invalid)
 *   page_size        : a power of two that divides W
 * Pages of different sequences must not overlap.
 */

/* swa_cache_append into a paged ring; arguments as swa_cache_append, with
 * the pools, page_table, page_size and num_pages as above. */
swa_status swa_cache_append_paged(void *k_pages, void *v_pages, const void *k_new, const void *v_new,
                                  const int32_t *pos, const int32_t *page_table, int32_t *slot_out,
                                  int B, int n, int Hkv, int d, int W, int page_size, int num_pages,
                                  swa_dtype dt, void *stream);

/* Bytes of scratch swa_decode needs for these sizes (0 means none). */
size_t swa_decode_workspace_bytes(int B, int Hq, int Hkv, int d, int W);

/*
 * One decode step per sequence over the ring (Ultralytics ring-buffer
 * paragraph; "Sliding-window and hybrid attention", dupenodi.dev, check-
 * yourself question 1).  The current token (position pos[b]) must already be
 * appended, so the visible keys are the min(pos[b]+1, W) filled slots
 * 0 .. min(pos[b]+1,W)-1.
 *   q, o     : [B,Hq,d]          k_cache, v_cache : [B,Hkv,W,d]
 *   pos      : device int32 [B], >= 0
 *   lse      : nullable fp32 [B,Hq]
 *   workspace: device scratch of at least swa_decode_workspace_bytes(...)
 *              bytes (may be NULL when that is 0); its contents on entry do
 *              not matter; calls sharing a workspace must not overlap.
 *   d in {32, 64, 128}; Hq/Hkv in {1, 2, 4, 8}.
 */
swa_status swa_decode(const void *q, const void *k_cache, const void *v_cache, void *o, float *lse,
                      const int32_t *pos, int B, int Hq, int Hkv, int d, int W, float scale,
                      swa_dtype dt, void *workspace, size_t workspace_bytes, void *stream);

/*
 * swa_decode over a paged ring (see swa_cache_append_paged): the same step,
 * the keys of ring slots 0 .. min(pos[b]+1,W)-1 read through page_table.
 * The workspace is sized by swa_decode_workspace_bytes with the same B, Hq,
 * Hkv, d, W.
 */
swa_status swa_decode_paged(const void *q, const void *k_pages, const void *v_pages, const int32_t *page_table,
                            void *o, float *lse, const int32_t *pos, int B, int Hq, int Hkv, int d, int W,
                            int page_size, int num_pages, float scale, swa_dtype dt, void *workspace,
                            size_t workspace_bytes, void *stream);

/*
 * One decode step over the ring plus attention sinks (Ultralytics glossary,
 * related-terms entry on attention sinks).  The query at position P =
 * pos[b] sees the ring's filled slots (the window, as in swa_decode) and
 * the sinks older than the window, positions 0 .. min(n_sink, P-W+1)-1; a
 * sink still inside the window is read once, from the ring.
 *   k_sink, v_sink : [B,Hkv,n_sink,d], row j holding position j (written by
 *                    the caller, e.g. swa_cache_append with W = n_sink while
 *                    the positions are below n_sink); may be NULL when
 *                    n_sink == 0
 *   n_sink >= 0; other arguments, the workspace included, as swa_decode.
 */
swa_status swa_decode_sinks(const void *q, const void *k_cache, const void *v_cache,
                            const void *k_sink, const void *v_sink, int n_sink, void *o, float *lse,
                            const int32_t *pos, int B, int Hq, int Hkv, int d, int W, float scale,
                            swa_dtype dt, void *workspace, size_t workspace_bytes, void *stream);

/*
 * swa_decode with no workspace argument, for callers that cannot allocate
 * device memory when they decode: a C host program without an allocator of
 * its own, a plugin inside a runtime that owns all device memory, or a
 * serving loop where an allocation could block on the device.  The pages
 * have no counterpart of this call; it exists only for those callers.
 *   Arguments, layouts and results as swa_decode (bit for bit: the same
 *   kernels with the same split count).
 *   Scratch: one static device array of 16 MiB.  It is part of the library's
 *   device code, so every process that loads this library holds it on every
 *   GPU the library's kernels are loaded on, until the process exits, whether
 *   or not it ever calls swa_decode_noalloc.  Sizes whose split partials
 *   (swa_decode_workspace_bytes) exceed 16 MiB are rejected with
 *   SWA_ERR_UNSUPPORTED before anything runs.  Nothing is allocated.
 *   The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current and keeps it for the
 *   life of the process; make that first call before any stream capture, and
 *   do not use this call on a device after cudaDeviceReset.
 *   All calls share the array: calls whose kernels overlap on the GPU (two
 *   streams, or two host threads on one device) race and give wrong results.
 *   Each call writes every scratch record it reads, so nothing is cleared
 *   between calls.
 */
swa_status swa_decode_noalloc(const void *q, const void *k_cache, const void *v_cache, void *o, float *lse,
                              const int32_t *pos, int B, int Hq, int Hkv, int d, int W, float scale,
                              swa_dtype dt, void *stream);

/*
 * Backward pass of the window prefill: the gradients of swa_prefill
 * (symmetric = 0) or of swa_prefill_global without globals (symmetric = 1)
 * with respect to q, k and v, for an upstream gradient dout.  The pages
 * define only the forward computation ("Sliding Window Attention",
 * robocikowo.com, opening definition); this is its chain rule, with the
 * probabilities recomputed from the forward pass's log-sum-exp:
 *   p_ij = exp(scale q_i.k_j - lse_i) in the window, D_i = dout_i . o_i,
 *   ds_ij = p_ij (dout_i.v_j - D_i), dq_i = scale sum_j ds_ij k_j,
 *   dk_j = scale sum_i ds_ij q_i, dv_j = sum_i p_ij dout_i
 * (a kv head's dk, dv sum over the query heads of its group).
 *   q, o, dout, dq : [B,T,Hq,d]   k, v, dk, dv : [B,T,Hkv,d]   bf16
 *   lse        : fp32 [B,Hq,T], the forward call's lse for the same inputs
 *   workspace  : device scratch of swa_prefill_backward_workspace_bytes(...)
 *                bytes, 16-byte aligned; calls sharing it must not overlap
 *   bf16 only (SWA_ERR_UNSUPPORTED otherwise); d in {64, 128}; W >= 1;
 *   other arguments as swa_prefill.  dq, dk, dv are overwritten.
 */
size_t swa_prefill_backward_workspace_bytes(int B, int T, int Hq);
swa_status swa_prefill_backward(const void *q, const void *k, const void *v, const void *o, const float *lse,
                                const void *dout, void *dq, void *dk, void *dv, int symmetric, int B, int T,
                                int Hq, int Hkv, int d, int W, float scale, swa_dtype dt, void *workspace,
                                size_t workspace_bytes, void *stream);

/*
 * Debug export of the visibility mask, from the same device predicate the
 * prefill kernels apply (robocikowo.com binary-mask entry).
 *   mask : device uint8 [T,T], mask[i*T+j] = 1 when query i may see key j
 *   symmetric = 0: causal window; 1: symmetric window, with global_idx
 *   (device int32 [g], sorted, may be NULL when g == 0) as global tokens.
 *   T <= 65536.
 */
swa_status swa_mask_export(uint8_t *mask, int T, int W, int symmetric,
                           const int32_t *global_idx, int g, void *stream);

/*
 * Synchronises `stream`, then reads and clears the current device's status
 * word.  Returns SWA_ERR_TIMEOUT if a kernel gave up on a bounded wait since
 * the last call, SWA_ERR_INTERNAL if (debug build, libswa_debug.so, compiled
 * with -DSWA_DEBUG) a kernel's check of its own tile, row or slot indices
 * failed, SWA_ERR_INVALID_ARG if a kernel met a bad device-side input,
 * SWA_ERR_CUDA if synchronising failed, else SWA_OK.
 */
swa_status swa_get_device_status(void *stream);

/*
 * Test hook for the failure path: launches one thread that waits on a
 * barrier nothing will ever complete, through the same bounded wait the
 * kernels use, with a limit of timeout_us microseconds.  The wait expires,
 * the kernel records SWA_ERR_TIMEOUT and returns; the context stays usable.
 */
swa_status swa_debug_expire_wait(int timeout_us, void *stream);

/* Per-wait limit (nanoseconds) the kernels use; default 2e9 (2 s). */
void swa_set_wait_limit_ns(unsigned long long ns);

/* Static text for a status code. */
const char *swa_status_string(swa_status s);

#ifdef __cplusplus
}
#endif

#endif /* SWA_H */

/*
 * tfa.h -- C ABI of the B200 (sm_100a) tiled GQA prefill attention library.
 *
 * One operation: dense prefill attention for grouped-query attention, where
 * L new query rows attend to S = prefix + L keys, under a causal mask offset by
 * the prefix, an optional sliding window and an optional length-S key mask.
 *
 * Definition (for batch b, query head h, new row i, P = S - L, p = P + i,
 * G = Hq / Hkv, g = floor(h / G)):
 *   key j is allowed iff (!causal || j <= p)
 *                     && (!causal || window <= 0 || j > p - window)
 *                     && (key_mask == NULL || key_mask[b*S + j] > 0.5f)
 *   o[b,h,i,:] = sum_j softmax_j(scale * q[b,h,i,:] . k[b,g,j,:]) v[b,g,j,:]
 *   over the allowed j; a row with no allowed key is written as zeros.
 * Sources: tiny-llm "Week 2 Day 5: Tiled Dense Prefill Attention", Task 1
 * (layouts, GQA head mapping without replicating K/V, online-softmax merge,
 * partial-tail guards, BF16 after the final FP32 normalisation) and Task 2
 * (causality aligned to the end of the cached prefix; fully masked rows are
 * finite zeros); brotensor "include/brotensor/ops/flash_attention.h"
 * (flash_attention_decode: window keeps [max(0,p-window+1), p]; key mask is
 * FP32 1 valid / 0 invalid, dropped when <= 0.5, combined multiplicatively).
 *
 * Layout: every tensor is contiguous row-major with the head dimension
 * innermost, bf16 stored as 16-bit words:
 *   q, o : [B, Hq,  L, D]        k, v : [B, Hkv, S, D]        key_mask : [B, S] fp32
 *
 * Ownership: every pointer passed to tfa_prefill is caller-owned DEVICE memory
 * on the current CUDA device; the call neither allocates nor frees the tensors
 * and never reads them on the host.  The library keeps one small status word
 * per device (allocated on the first call on that device) where the kernel
 * records a timed-out internal wait, and per stream the scratch of the split
 * schedule (2 x SMs partial slots of 128 x 128 + 256 floats, allocated on the
 * first call on that stream, kept until process exit).
 *
 * Asynchrony: tfa_prefill validates its arguments on the host, then enqueues
 * the kernel on `stream` and returns; o is fully overwritten when the stream
 * reaches that point.  Errors found by validation are returned before any
 * launch, with no side effect.  A device-side failure (a wait that gave up)
 * is reported by tfa_check_status().
 *
 * Graph capture: tfa_prefill and tfa_decode may be captured into a CUDA graph
 * on a stream that has already seen one call outside capture (that call
 * creates the device state and the stream's scratch; a first call made during
 * capture returns TFA_ERR_CAPTURE instead of allocating).  Every replay is a
 * complete, independent call on the captured pointers, sizes and scale; the
 * split schedule's synchronisation lives in device memory, not in the
 * captured arguments.  A replay uses the scratch of the stream it was
 * captured on, so it must not run concurrently with another replay or call
 * that uses that stream's scratch (replaying on that stream guarantees it).
 */
#ifndef TFA_H
#define TFA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *tfa_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
    TFA_OK = 0,
    TFA_ERR_NULL = 1,        /* q, k, v or o is NULL                                      */
    TFA_ERR_HEADS = 2,       /* Hq < 1, Hkv < 1 or Hq % Hkv != 0                         */
    TFA_ERR_SHORT_QUERY = 3, /* L < 9: the tiled operator rejects short queries          */
    TFA_ERR_SHAPE = 4,       /* B < 1, S < L, or a size whose element count overflows    */
    TFA_ERR_HEAD_DIM = 5,    /* D not 64 or 128                                          */
    TFA_ERR_WINDOW = 6,      /* window > 0 without causal (no page defines it)           */
    TFA_ERR_ALIGN = 7,       /* a tensor pointer is not 16-byte aligned, key_mask not 4  */
    TFA_ERR_CUDA = 8,        /* a CUDA runtime/driver call failed (launch, encode, ...)  */
    TFA_ERR_TIMEOUT = 9,     /* a kernel wait gave up; the output of that call is invalid */
    TFA_ERR_SCALE = 10,      /* scale is not finite                                      */
    TFA_ERR_FLAGS = 11,      /* unknown debug flag bits                                  */
    TFA_ERR_CAPTURE = 12,    /* first call on a device or stream made inside a CUDA graph
                                capture (it would allocate); call once outside capture   */
    TFA_ERR_SOFTCAP = 13,    /* softcap not finite, negative, or > 0 with scale == 0     */
    TFA_ERR_SEQLENS = 14,    /* (tfa_check_status) a variable-length call met an
                                inconsistent cu_seqlens entry; that call's output is
                                invalid                                                  */
    TFA_ERR_RING = 15        /* ring cache without a window, ring_rows not a positive
                                multiple of 64, or ring_rows < window - 1 + L            */
} tfa_status;

/* Minimum query length accepted by the tiled operator (tiny-llm Week 2 Day 5,
 * Task 1: the direct operator rejects queries shorter than nine rows). */
#define TFA_MIN_QUERY_ROWS 9

/* tfa_prefill -- tiled dense prefill attention with GQA.
 *   q        bf16 [B,Hq,L,D] device, 16-byte aligned, read only
 *   k, v     bf16 [B,Hkv,S,D] device, 16-byte aligned, read only
 *   o        bf16 [B,Hq,L,D] device, 16-byte aligned, written (every element)
 *   B        batch, >= 1
 *   Hq, Hkv  query / KV heads, Hq % Hkv == 0; query head h reads KV head h/(Hq/Hkv)
 *   L        new query rows, >= TFA_MIN_QUERY_ROWS
 *   S        keys (cached prefix + L), >= L
 *   D        head dimension, 64 or 128
 *   scale    softmax scale applied to q.k (typically 1/sqrt(D)), finite
 *   causal   nonzero: row i sees keys j <= S-L+i; zero: every key (bidirectional)
 *   window   > 0 (causal only): additionally j > S-L+i-window; <= 0: no window
 *   key_mask fp32 [B,S] device (4-byte aligned) or NULL; key j of batch b kept iff > 0.5
 *   stream   CUDA stream to enqueue on
 * Returns TFA_OK or a tfa_status code.
 * Queries of at most 128 rows run through the packed tiles described under
 * tfa_decode (floor(128 / L) query heads of a KV group per tile); longer ones
 * through pairs of 128-row tiles of one head, or, for causal calls with short
 * key ranges and an even number of query heads per KV group, the same
 * 128-row tile of two heads.  The results are the same attention either way. */
int tfa_prefill(const void *q, const void *k, const void *v, void *o,
                int B, int Hq, int Hkv, int L, int S, int D, float scale,
                int causal, int window, const float *key_mask, tfa_stream_t stream);

/* Longest query accepted by tfa_decode. */
#define TFA_MAX_DECODE_ROWS 8

/* tfa_decode -- the same attention for short queries: 1 <= L <= 8 new rows
 * (L = 1 is token-by-token decoding), which tfa_prefill rejects.  Arguments,
 * layouts, masks, ownership and errors are those of tfa_prefill, except that
 * L must lie in [1, TFA_MAX_DECODE_ROWS] (else TFA_ERR_SHAPE).  The kernel
 * packs the L rows of several query heads of one KV group into each
 * 128-row tensor-core tile and spreads the key range of every KV group over
 * all SMs, merging the pieces' softmax statistics exactly (the online-softmax
 * merge of tiny-llm "Week 2 Day 5: Tiled Dense Prefill Attention", Task 1).
 * The pages route such queries to a separate path (tiny-llm's readable
 * fallback for L <= 8; mlx-lm's sdpa_vector for at most 8 rows; brotensor's
 * flash_attention_decode for L_q == 1). */
int tfa_decode(const void *q, const void *k, const void *v, void *o,
               int B, int Hq, int Hkv, int L, int S, int D, float scale,
               int causal, int window, const float *key_mask, tfa_stream_t stream);

/* tfa_attention_ex -- the same attention with the score variants, for any
 * L >= 1 (L <= 128 takes the packed tiles, longer queries pairs of
 * 128-row tiles).  Arguments, layouts, ownership, asynchrony and
 * errors are those of tfa_prefill/tfa_decode, plus:
 *   softcap  logit soft-capping (brotensor flash_attention.h, Gemma-2
 *            extensions): after the scale and before the masks and the
 *            softmax, each score t becomes softcap * tanh(t / softcap).
 *            0 disables it; negative, NaN or infinite values, or softcap > 0
 *            with scale == 0, return TFA_ERR_SOFTCAP.
 *   sinks    NULL, or caller-owned device fp32 [Hq], 4-byte aligned (else
 *            TFA_ERR_ALIGN): attention-sink logits (named among the tested
 *            cases of mlx-lm's sliding-window SDPA PR, without a formula).
 *            Read here as one extra logit per query head that joins the
 *            softmax denominator with no value row, in the same units as the
 *            capped, scaled scores (not scaled, not capped):
 *            o = sum_j e^(t_j - m) v_j / (sum_j e^(t_j - m) + e^(sink_h - m)).
 *            A row with no allowed key is still written as zeros.
 * With softcap = 0 and sinks = NULL the result equals tfa_prefill's
 * (tfa_decode's for short queries). */
int tfa_attention_ex(const void *q, const void *k, const void *v, void *o,
                     int B, int Hq, int Hkv, int L, int S, int D, float scale,
                     int causal, int window, const float *key_mask, float softcap,
                     const float *sinks, tfa_stream_t stream);

/* Longest batch of tfa_prefill_varlen. */
#define TFA_MAX_VARLEN_SEQS 1024

/* tfa_prefill_ring -- the same attention over a rotating (ring) K/V cache
 * (TensorFold PR 3269's sliding layer: WINDOW and RING, the ring slot of a
 * key and value row; mlx-lm's RotatingKVCache).  k and v hold the last
 * ring_rows positions: [B, Hkv, ring_rows, D] bf16, where the key at absolute
 * position j (0 <= j < S, S = prefix + L) lives in row j mod ring_rows.
 * q/o are [B, Hq, L, D] as for tfa_prefill (any L >= 1; L <= 8 takes the
 * packed short-query path).  Causal with a sliding window, always:
 * window > 0, ring_rows a positive multiple of 64, and
 * ring_rows >= window - 1 + L (every key a new row may see is still in the
 * ring), else TFA_ERR_RING.  No key mask.  softcap and sinks as for
 * tfa_attention_ex.  Other arguments, ownership and errors as tfa_prefill. */
int tfa_prefill_ring(const void *q, const void *k, const void *v, void *o,
                     int B, int Hq, int Hkv, int L, int S, int ring_rows, int D, float scale,
                     int window, float softcap, const float *sinks, tfa_stream_t stream);

/* tfa_prefill_varlen -- packed variable-length batches (brotensor
 * flash_attention.h, flash_attention_varlen_forward; flash_attn_varlen_func
 * semantics, here with GQA).  q and o are [total_q, Hq, D] bf16, k and v
 * [total_k, Hkv, D] bf16, all caller-owned device memory, 16-byte aligned.
 * cu_seqlens_q / cu_seqlens_k: caller-owned DEVICE int32 [B + 1] prefix sums
 * (4-byte aligned), 1 <= B <= TFA_MAX_VARLEN_SEQS: sequence b owns query rows
 * [cu_seqlens_q[b], cu_seqlens_q[b+1]) and key/value rows
 * [cu_seqlens_k[b], cu_seqlens_k[b+1]); nothing crosses sequences.
 * max_seqlen_q bounds every sequence's query count (tiles are enumerated up
 * to it).  Within sequence b the definition of tfa_prefill holds with
 * L_b = its query count and S_b = its key count: causal rows are aligned to
 * the end of the sequence's keys (prefix S_b - L_b; for L_b == S_b this is
 * brotensor's (k - cu_k[b]) <= (q - cu_q[b])), and a causal sequence needs
 * S_b >= L_b.  Any L_b >= 0 (no short-query minimum).  window, softcap and
 * sinks as for tfa_attention_ex; no key mask.
 * The lengths live in device memory, so they are checked by the kernel: a
 * sequence whose entries are inconsistent (decreasing, past total_q/total_k,
 * L_b > max_seqlen_q, or causal with S_b < L_b) is skipped, its rows are not
 * written, and tfa_check_status() returns TFA_ERR_SEQLENS.  total_q == 0:
 * nothing to do, TFA_OK without a launch (no pointer is examined); with
 * queries, max_seqlen_q == 0 or total_k == 0 return TFA_ERR_SHAPE. */
int tfa_prefill_varlen(const void *q, const void *k, const void *v, void *o,
                       const int *cu_seqlens_q, const int *cu_seqlens_k, int B, int Hq, int Hkv,
                       int total_q, int total_k, int max_seqlen_q, int D, float scale,
                       int causal, int window, float softcap, const float *sinks,
                       tfa_stream_t stream);

/* tfa_prefill_backward -- gradients of the attention core (brotensor
 * flash_attention.h, flash_attention_backward: the backward of the bare
 * core, recompute-based, consuming no forward caches; causal- and
 * mask-excluded positions contribute nothing to any gradient).
 *   q, k, v, key_mask, sizes, scale, causal, window: as for tfa_prefill
 *            (any L >= 1; L <= 8 recomputes through tfa_decode's path)
 *   dout     upstream gradient of the output, bf16 [B, Hq, L, D]
 *   dq       bf16 [B, Hq, L, D]; dk, dv bf16 [B, Hkv, S, D] -- overwritten
 *            (dk, dv summed over the query heads of each KV group)
 * All caller-owned device memory, 16-byte aligned (else TFA_ERR_ALIGN;
 * TFA_ERR_NULL for a NULL gradient pointer).  With P the softmax weights and
 * dP = dout V^T: dS = P (dP - rowsum(dout o O)), dq = scale dS K,
 * dk = scale dS^T Q, dv = P^T dout.  The call re-runs the forward (its output
 * and per-row log-sum-exp go to a per-stream workspace of 2 B Hq L (D + 4)
 * bytes, grown on demand; growth during graph capture returns
 * TFA_ERR_CAPTURE), then three kernels, all asynchronous on `stream`: a
 * delta kernel, the dQ kernel, and the dK/dV kernel, launched with
 * programmatic stream serialisation so that its CTAs start on the SMs the dQ
 * kernel's CTAs leave (it reads nothing dQ writes).  The dK/dV kernel does
 * not complete before the dQ kernel has, so work queued on `stream` after
 * the call sees all three gradients. */
int tfa_prefill_backward(const void *q, const void *k, const void *v, const void *dout,
                         void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int L, int S,
                         int D, float scale, int causal, int window, const float *key_mask,
                         tfa_stream_t stream);

/* tfa_prefill_lse -- tfa_prefill (any L >= 1) that also writes each query
 * row's base-2 log-sum-exp of its scaled scores,
 *   lse[b, h, i] = log2( sum over allowed j of 2^(scale * log2(e) * q.k_j) )
 * (+inf for a row with no allowed key), fp32 [B, Hq, L], caller-owned device
 * memory, 4-byte aligned (TFA_ERR_NULL if NULL, TFA_ERR_ALIGN if not).  Other
 * arguments, layouts, errors and asynchrony are tfa_prefill's.  The output
 * and lse are what tfa_prefill_backward_saved takes. */
int tfa_prefill_lse(const void *q, const void *k, const void *v, void *o, float *lse,
                    int B, int Hq, int Hkv, int L, int S, int D, float scale,
                    int causal, int window, const float *key_mask, tfa_stream_t stream);

/* tfa_prefill_backward_saved -- tfa_prefill_backward given the forward's
 * output o (bf16 [B, Hq, L, D], 16-byte aligned) and lse (fp32 [B, Hq, L],
 * 4-byte aligned) as tfa_prefill_lse wrote them for the same q, k, v, mask,
 * scale, causal and window: the forward is not re-run (the usual training
 * order, the forward's statistics saved for the backward).  Gradients,
 * layouts, workspace, errors and asynchrony as for tfa_prefill_backward;
 * NULL o or lse returns TFA_ERR_NULL.  With o and lse from tfa_prefill_lse
 * the gradients are bit-identical to tfa_prefill_backward's. */
int tfa_prefill_backward_saved(const void *q, const void *k, const void *v, const void *o,
                               const float *lse, const void *dout, void *dq, void *dk, void *dv,
                               int B, int Hq, int Hkv, int L, int S, int D, float scale,
                               int causal, int window, const float *key_mask, tfa_stream_t stream);

/* Debug flags for tfa_prefill_debug. */
#define TFA_DEBUG_NO_TILE_SKIP  1u /* visit every key tile, even fully masked ones   */
#define TFA_DEBUG_MASK_ALL      2u /* apply the mask predicate on interior tiles too */
#define TFA_DEBUG_SYNC          4u /* synchronize the stream and return the device status */
#define TFA_DEBUG_NO_SPLIT      8u /* deal whole work items (snake order, longest first) instead
                                      of splitting key ranges evenly across the CTAs (no partial
                                      merges) */
#define TFA_DEBUG_FORCE_SPLIT  16u /* always split key ranges evenly across the CTAs (by
                                      default the library picks the schedule it estimates
                                      finishes first) */
#define TFA_DEBUG_SHORT_WAITS  32u /* give up every pipeline wait of the kernel after ~1000 SM
                                      cycles instead of ~4 s, to exercise the give-up path: the
                                      waits run out, the kernel drains its copies and tensor-core
                                      work, the output is invalid and tfa_check_status (or
                                      TFA_DEBUG_SYNC) returns TFA_ERR_TIMEOUT. */

/* tfa_prefill_debug -- tfa_prefill with debug flags (arguments as above).  With
 * NO_TILE_SKIP and/or MASK_ALL the result must be bit-identical to tfa_prefill's
 * (masked-tile skipping is exact: mlx-lm PR "Skip fully masked key tiles in Flint
 * sliding-window prefill" requires the banded result to equal the single call). */
int tfa_prefill_debug(const void *q, const void *k, const void *v, void *o,
                      int B, int Hq, int Hkv, int L, int S, int D, float scale,
                      int causal, int window, const float *key_mask, tfa_stream_t stream,
                      unsigned flags);

/* tfa_prefill_host -- the same operation on HOST buffers (q, k, v, key_mask
 * read, o written; plain or pinned host memory), for L >= 9 as tfa_prefill and
 * for 1 <= L <= 8 as tfa_decode.  The library copies the
 * inputs to device staging buffers it owns (one set per device, grown on
 * demand and kept until process exit), runs the attention, copies o back and
 * synchronizes before returning.  The work is pipelined over up to 4 stages
 * of KV groups (ranges of groups of one batch element, or runs of whole
 * elements when B > 4): a stage's inputs are copied in on a library-owned
 * stream while the previous stage computes on `stream` and the one before is
 * copied out on a second library-owned stream.  With pinned host memory the
 * transfers overlap the computation; with plain memory the copies are
 * synchronous to the host and the result is the same.  Not safe to call from
 * two host threads on the same device at once. */
int tfa_prefill_host(const void *q, const void *k, const void *v, void *o,
                     int B, int Hq, int Hkv, int L, int S, int D, float scale,
                     int causal, int window, const float *key_mask, tfa_stream_t stream);

/* tfa_prefill_noalloc -- tfa_prefill for callers that cannot allocate device
 * memory (a caching or arena allocator owns all of it, allocation is not
 * allowed at the point of the call, or the host runtime only hands out its own
 * buffers).  No counterpart on the pages: it exists for those callers.
 * Arguments, layout and validation are tfa_prefill's; the caller still passes
 * every input and output.  The call makes no cudaMalloc, cudaFree or other
 * allocating call: the kernel's scratch (its status word) lives in a fixed
 * 256-byte device array inside the library, which every GPU that loads the
 * library holds until the process exits.
 *   - It always runs the whole-item schedule (no query tile is cut into key
 *     ranges; the split schedule's partials would not fit the array), so its
 *     output is not bit-identical to tfa_prefill's, which may cut tiles and
 *     merge partial results in another rounding order.  Both match the fp64
 *     definition within the operator tolerance (|err| <= 0.02 + 0.02 |ref|).
 *     On large causal calls the whole-item schedule can be slower.
 *   - The first call on a device sets the array up (looks up its address and
 *     clears it with that device current); a first call made while `stream`
 *     is being captured is refused with TFA_ERR_CAPTURE.
 *   - Every call shares the one array, which keeps the last call's contents:
 *     calls that overlap on the GPU (other streams, other threads) race on it.
 *   - The kernel needs 4 bytes of the 256-byte maximum for every size
 *     tfa_prefill accepts (checked when the library is compiled), so no valid
 *     call is rejected for its size.
 *   - A timed-out kernel wait is reported by tfa_check_status, as for tfa_prefill. */
int tfa_prefill_noalloc(const void *q, const void *k, const void *v, void *o,
                        int B, int Hq, int Hkv, int L, int S, int D, float scale,
                        int causal, int window, const float *key_mask, tfa_stream_t stream);

/* tfa_check_status -- synchronizes `stream`, then reads and clears the current
 * device's status words (tfa_prefill's and, once set up, tfa_prefill_noalloc's;
 * both are read and cleared on every call).  Returns TFA_OK, TFA_ERR_TIMEOUT if
 * a kernel launched since the last check recorded a wait that gave up (in
 * either word), TFA_ERR_SEQLENS if a tfa_prefill_varlen call met inconsistent
 * cu_seqlens (and no wait gave up), or TFA_ERR_CUDA. */
int tfa_check_status(tfa_stream_t stream);

/* tfa_last_error -- for the calling host thread, a description of the last CUDA
 * runtime/driver call that failed inside the library (the call and its error
 * string), or "" if none has.  Never NULL; valid until the next library call. */
const char *tfa_last_error(void);

/* tfa_status_string -- static description of a status code (never NULL). */
const char *tfa_status_string(int status);

/* tfa_plan_qtile -- host view of the work enumeration the kernel performs for
 * one 128-row query tile (rows [128*qtile, min(128*qtile+128, L))); for
 * 1 <= L <= 8 (tfa_decode) tile 0 is the key range of every packed tile:
 *   *kt_lo, *kt_hi  first and last 128-key tile it visits (kt_hi < kt_lo: none)
 *   needs_mask      if not NULL, receives kt_hi-kt_lo+1 bytes: 1 where the tile
 *                   crosses the causal diagonal, the window edge, the key tail
 *                   or a key mask is present; 0 for interior tiles
 * Returns TFA_OK, TFA_ERR_SHAPE for an out-of-range tile, or a validation
 * error for the sizes.  No device work. */
int tfa_plan_qtile(int L, int S, int causal, int window, int has_key_mask, int qtile,
                   int *kt_lo, int *kt_hi, unsigned char *needs_mask, int needs_mask_len);

/* tfa_plan_ktile -- host view of the backward pass's enumeration for one
 * 128-key tile (keys [128*ktile, min(128*ktile+128, S))): the first and last
 * 128-row query tile holding a row that may see one of its keys under the
 * causal mask and the window (*qt_hi < *qt_lo: no row sees the tile, and its
 * key and value gradients are zero).  Returns TFA_OK, TFA_ERR_SHAPE for an
 * out-of-range tile, or a validation error for the sizes.  No device work. */
int tfa_plan_ktile(int L, int S, int causal, int window, int ktile, int *qt_lo, int *qt_hi);

/* tfa_plan_pieces -- host view of the work one CTA of a grid of `grid` CTAs
 * performs (no device work).  The work of (batch, query head, pair of 128-row
 * query tiles) is the union of the two tiles' key-tile ranges.  With split != 0
 * (tfa_prefill's schedule) the concatenated key-tile steps of all such items
 * are cut into `grid` contiguous ranges of almost equal length; a cut item is
 * finished by the piece holding a tile's first key tile, which merges the
 * others' partial softmax statistics.  Without bit 0 of split whole items are
 * dealt in snake order: CTA c takes items c, 2G-1-c, 2G+c, 4G-1-c, ... (G =
 * grid).  Bit 1 of split (value 2) selects head pairs, as tfa_prefill uses
 * when Hq / Hkv is even: an item is then one 128-row query tile of query
 * heads 2h and 2h+1 (h counting pairs, Hq must be even), its two tiles
 * visiting the same key tiles.
 *   out          10 ints per piece: item, qp (query-tile pair, or the query
 *                tile with head pairs), b, h (head, or head pair), first key tile, last key
 *                tile, role of tile 0, role of tile 1 (bit 0 active, bit 1
 *                finalizer, bit 2 complete), and for a finalizer that must
 *                merge, the last CTA contributing to tile 0 / tile 1 (else -1)
 *   *n_pieces    number of pieces of this CTA (written even when > max_pieces)
 *   total_steps  if not NULL, the total number of key-tile steps
 * Returns TFA_OK, TFA_ERR_SHAPE (bad grid/cta, or more than max_pieces), or a
 * validation error for the sizes (Hkv is taken equal to Hq, D as 128). */
int tfa_plan_pieces(int B, int Hq, int L, int S, int causal, int window, int grid, int split,
                    int cta, int *out, int max_pieces, int *n_pieces, long long *total_steps);

/* Tile sizes of the kernel: 128 query rows x 128 keys per tensor-core tile. */
#define TFA_BLOCK_Q 128
#define TFA_BLOCK_K 128

#ifdef __cplusplus
}
#endif

#endif /* TFA_H */

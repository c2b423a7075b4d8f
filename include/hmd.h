/*
 * hmd.h — C ABI of the hybrid-mixer decoding library (libhmd.so, sm_100a).
 *
 * The library runs the per-layer token-mixer step of a hybrid "supernet" decoder in which every
 * layer offers four mixers — full attention (FA), sliding-window attention (SWA), Kimi Delta
 * Attention (KDA) and Gated DeltaNet (GDN) — and a placement vector picks one mixer per layer
 * ("Super Apriel: One Checkpoint, Many Speeds", abstract; gist.science technical summary of the
 * same paper, section 2a "Supernet architecture").
 *
 * Conventions for every entry point:
 *  - Tensors are DEVICE pointers owned by the caller (the library owns only the caches it
 *    allocates through *_alloc and frees through *_free). They are dense and contiguous in the
 *    row-major layouts stated, and 16-byte aligned.
 *  - Streams: `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *    Every call is asynchronous on that stream, never synchronises, allocates nothing on the
 *    decode/prefill paths, and can be captured into a CUDA graph (cache alloc/free excepted).
 *  - Errors: no exception crosses the ABI. Argument, shape and dtype errors return a status
 *    before anything is launched and leave every output untouched. A failed launch returns
 *    HMD_ERR_CUDA. Faults detected inside a kernel (an out-of-range page id or state slot, a
 *    wait that timed out) skip the offending access and set a bit in a per-device error word,
 *    read (and cleared) by hmd_device_errors().
 *  - Precision: activations (q, k, v, o) are bf16 or fp32; gates, beta and recurrent states are
 *    fp32; attention KV caches are bf16. Outputs take the activation dtype (bf16 stores round to
 *    nearest even).
 */
#ifndef HMD_H
#define HMD_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HMD_API __attribute__((visibility("default")))
#else
#define HMD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { HMD_FA = 0, HMD_SWA = 1, HMD_KDA = 2, HMD_GDN = 3 } hmd_kind_t;
typedef enum { HMD_F32 = 0, HMD_BF16 = 1 } hmd_dtype_t;
typedef enum {
    HMD_OK = 0,
    HMD_ERR_ARG = 1,          /* null pointer, bad enum, negative size, bad layer/window */
    HMD_ERR_SHAPE = 2,        /* sizes inconsistent with each other or with a cache */
    HMD_ERR_DTYPE = 3,        /* dtype not accepted by this entry point */
    HMD_ERR_OOM = 4,          /* cache allocation failed */
    HMD_ERR_CUDA = 5,         /* a CUDA call or a kernel launch failed */
    HMD_ERR_UNSUPPORTED = 6,  /* valid but not implemented (e.g. a head size with no kernel) */
    HMD_ERR_DEVICE_CHECK = 7  /* a kernel-side check fired (see hmd_device_errors) */
} hmd_status_t;

/* Bits of the per-device error word. */
#define HMD_DEVERR_TIMEOUT   0x1u  /* a bounded wait on a copy barrier gave up */
#define HMD_DEVERR_PAGE      0x2u  /* a page-table entry was outside [0, n_pages) */
#define HMD_DEVERR_SLOT      0x4u  /* a state-slot index was outside [0, n_slots) */
#define HMD_DEVERR_SEQLEN    0x8u  /* a sequence length was < 1 or above the stated maximum */
#define HMD_DEVERR_GATE      0x10u /* reserved: no longer raised (the chunked prefill accepts
                                      every gate range) */

typedef void *hmd_stream_t;

/* ------------------------------------------------------------------------------------------ */
/* Delta-rule mixers (GDN, KDA).                                                              */
/* The pages name GDN as a recurrence with a scalar gate and KDA as one with channel-wise     */
/* gating, both O(n) with a constant-size state (gist.science summary, section 2a). The       */
/* library implements the standard definitions, with the state stored as M[d_k][d_v]:         */
/*   GDN: S_t = g_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T, o_t = S_t q_t, M = S^T       */
/*   KDA: S_t = (I - b_t k_t k_t^T) Diag(a_t) S_{t-1} + b_t k_t v_t^T, o_t = S_t^T q_t, M = S */
/* i.e. for both: M' = Diag(a) M, u = b (v - M'^T k), M <- M' + k u^T, o = scale * M^T q,      */
/* with a = exp(log_gate) broadcast over d_k for GDN.                                          */
/* ------------------------------------------------------------------------------------------ */

/* One decode token per sequence for one layer.
 *   q, k      [B][H][dk]   (dtype)        v, o  [B][H][dv] (dtype)
 *   beta      [B][H]       fp32
 *   log_gate  [B][H] fp32 (GDN) or [B][H][dk] fp32 (KDA); values <= 0
 *   state     [n_slots][H][dk][dv] fp32, updated in place; sequence b uses slot slots[b]
 *             (slots == NULL: slot b). Two sequences must not share a slot.
 *   scale     multiplies o (1.0 reproduces the definitions).
 * Supported: dk in {16, 32, 64, 128, 256}; dv a multiple of 4, 4 <= dv <= 1024.
 * Returns HMD_ERR_ARG for a bad kind / null pointer, HMD_ERR_UNSUPPORTED for other dk/dv.     */
HMD_API hmd_status_t delta_rule_decode(hmd_kind_t kind, int B, int H, int dk, int dv, hmd_dtype_t dtype,
                               const void *q, const void *k, const void *v, const float *beta,
                               const float *log_gate, float *state, int n_slots,
                               const int32_t *slots, void *o, float scale, hmd_stream_t stream);

/* delta_rule_decode that writes the updated state of sequence b to slot dst_slots[b] (device
 * int32 [B]) and leaves slot slots[b] as it was (dst_slots == NULL: in place). A speculative
 * draft of k tokens steps slot s0 -> s1 -> ... -> sk; keeping the first j accepted tokens is
 * then the choice of slot s_j, with nothing copied or recomputed. Slots must lie in
 * [0, n_slots) (else the device error word reports HMD_DEVERR_SLOT and that sequence is
 * skipped); no destination slot may be another sequence's source or destination in this call. */
HMD_API hmd_status_t delta_rule_decode_to(hmd_kind_t kind, int B, int H, int dk, int dv,
                                          hmd_dtype_t dtype, const void *q, const void *k,
                                          const void *v, const float *beta,
                                          const float *log_gate, float *state, int n_slots,
                                          const int32_t *slots, const int32_t *dst_slots,
                                          void *o, float scale, hmd_stream_t stream);

/* Input activations fused into the delta-rule kernels. The pages name GDN and KDA but not
 * how their inputs are formed; this follows the published layers: from the projections' raw
 * outputs, q and k are L2-normalised over d_k (x / sqrt(sum x^2 + l2_eps)), beta = sigmoid of
 * its logit, and the log-gate = -exp(A_log[h]) * softplus(gate_logit + dt_bias) with
 * softplus(x) = log(1 + e^x). A_log [H] fp32 (device); dt_bias [H] (GDN) or [H][dk] (KDA)
 * fp32 (device).                                                                              */
typedef struct {
    const float *A_log;
    const float *dt_bias;
    float l2_eps;
} hmd_delta_act_t;

/* delta_rule_decode_to on raw projections: q_raw, k_raw as q, k; beta_logit as beta;
 * gate_logit as log_gate (same shapes); activations as above, computed in fp32 inside the
 * kernel. HMD_ERR_ARG for a null act, A_log or dt_bias, or a negative l2_eps.                 */
HMD_API hmd_status_t delta_rule_decode_act(hmd_kind_t kind, int B, int H, int dk, int dv,
                                           hmd_dtype_t dtype, const void *q_raw,
                                           const void *k_raw, const void *v,
                                           const float *beta_logit, const float *gate_logit,
                                           const hmd_delta_act_t *act, float *state,
                                           int n_slots, const int32_t *slots,
                                           const int32_t *dst_slots, void *o, float scale,
                                           hmd_stream_t stream);

/* n_q decode tokens per sequence in one launch, along a slot chain: the state is read once
 * from slot chain[0][b] and, after token t, stored to slot chain[t + 1][b] (the state read is
 * never written back). Equal to n_q delta_rule_decode_to calls stepping chain[t] ->
 * chain[t + 1], bit for bit, while reading the state once instead of n_q times: the form a
 * speculative verifier's GDN/KDA layers take, since its k + 1 positions are all known.
 *   q, k [B][n_q][H][dk]; v, o [B][n_q][H][dv]; beta [B][n_q][H]; log_gate [B][n_q][H] (GDN)
 *   or [B][n_q][H][dk] (KDA); chain int32 [n_q + 1][B] on the device, slots in [0, n_slots)
 *   (a bad slot skips that sequence and sets HMD_DEVERR_SLOT), no slot shared between
 *   sequences; act: NULL for activated inputs, else raw projections as in delta_rule_decode_act.
 */
HMD_API hmd_status_t delta_rule_decode_chain(hmd_kind_t kind, int n_q, int B, int H, int dk,
                                             int dv, hmd_dtype_t dtype, const void *q,
                                             const void *k, const void *v, const float *beta,
                                             const float *log_gate, const hmd_delta_act_t *act,
                                             float *state, int n_slots, const int32_t *chain,
                                             void *o, float scale, hmd_stream_t stream);

/* Chunked (WY / UT-transform) prefill over T tokens per sequence for one layer: the same
 * recurrence as delta_rule_decode applied to tokens 0..T-1 in order, computed chunk by chunk.
 *   q, k [B][T][H][dk]; v, o [B][T][H][dv] (dtype); beta [B][T][H] fp32;
 *   log_gate [B][T][H] (GDN) or [B][T][H][dk] (KDA) fp32;
 *   state [n_slots][H][dk][dv] fp32: read as the initial state and overwritten with the final
 *   one (slot slots[b], or b when slots == NULL).
 *   chunk: tokens per chunk; 64 is the supported value. T need not be a multiple of it.
 * Supported: bf16 with dk = dv = 128 and chunk 64 on the tensor-core path; fp32 or other
 * sizes (dk, dv in {16..128}, multiples of 16) on the CUDA-core path. q, k, v, o, log_gate and
 * state must be 16-byte aligned (HMD_ERR_ARG otherwise).
 * The tensor-core path runs in two passes that exchange one record per chunk and head through
 * device scratch (delta_rule_prefill_workspace_size bytes for the whole input). This entry point
 * takes that scratch, up to 1 GiB per call (longer inputs run in segments), as a stream-ordered
 * allocation from a pool the library keeps per device (up to 1 GiB stays cached between calls);
 * HMD_ERR_OOM if it cannot. Under stream capture, or to own the memory, call
 * delta_rule_prefill_chunked_ws instead.
 * Gate range: any log-gate <= 0 is accepted. The chunk form splits each decay e^{G_r - G_s}
 * (G the cumulative log-gate inside a chunk) into e^{G_r} and e^{-G_s} while every |G| of the
 * chunk is at most 80 (both factors then fit fp32), so that the chunk's products are plain
 * matrix products; a chunk with stronger decay forms its decays directly, at a higher cost
 * (KDA: on the CUDA cores; GDN's scalar decay needs no split).                                  */
HMD_API hmd_status_t delta_rule_prefill_chunked(hmd_kind_t kind, int B, int T, int H, int dk, int dv,
                                        hmd_dtype_t dtype, const void *q, const void *k,
                                        const void *v, const float *beta, const float *log_gate,
                                        float *state, int n_slots, const int32_t *slots, void *o,
                                        int chunk, float scale, hmd_stream_t stream);

/* Scratch bytes for delta_rule_prefill_chunked_ws to run these sizes in one segment: one record
 * (74,240 bytes at dk = dv = 128, chunk 64) per chunk and (sequence, head). 0 when the call
 * needs no scratch (the CUDA-core path) or the sizes are empty or invalid.                    */
HMD_API size_t delta_rule_prefill_workspace_size(hmd_kind_t kind, int B, int T, int H, int dk,
                                                 int dv, hmd_dtype_t dtype, int chunk);

/* delta_rule_prefill_chunked on raw projections (activations as for delta_rule_decode_act,
 * fused into the chunk-parallel pass). Supported on the tensor-core path only: bf16 with
 * dk = dv = 128 and chunk 64 (HMD_ERR_UNSUPPORTED otherwise).                                */
HMD_API hmd_status_t delta_rule_prefill_chunked_act(hmd_kind_t kind, int B, int T, int H, int dk,
                                                    int dv, hmd_dtype_t dtype, const void *q_raw,
                                                    const void *k_raw, const void *v,
                                                    const float *beta_logit,
                                                    const float *gate_logit,
                                                    const hmd_delta_act_t *act, float *state,
                                                    int n_slots, const int32_t *slots, void *o,
                                                    int chunk, float scale, hmd_stream_t stream);

/* delta_rule_prefill_chunked with caller-owned scratch: `workspace` (device, 16-byte aligned)
 * of ws_bytes. Any size from one chunk's records for all B*H heads up works; with less than
 * delta_rule_prefill_workspace_size(...) bytes the call runs the sequence in segments of as many
 * chunks as fit (same results, bit for bit). HMD_ERR_SHAPE if not even one chunk fits. The
 * scratch must not be in use by another call while this one runs. Allocates nothing, so it
 * can be captured in a CUDA graph. Paths that need no scratch ignore workspace and ws_bytes. */
HMD_API hmd_status_t delta_rule_prefill_chunked_ws(hmd_kind_t kind, int B, int T, int H, int dk,
                                                   int dv, hmd_dtype_t dtype, const void *q,
                                                   const void *k, const void *v,
                                                   const float *beta, const float *log_gate,
                                                   float *state, int n_slots,
                                                   const int32_t *slots, void *o, int chunk,
                                                   float scale, void *workspace,
                                                   size_t ws_bytes, hmd_stream_t stream);

/* ------------------------------------------------------------------------------------------ */
/* Attention mixers (FA, SWA) over a paged bf16 KV cache.                                     */
/* FA is standard causal attention, O(n^2) over a KV cache that grows with the context; SWA   */
/* attends to a local window, O(n*w) (gist.science summary, sections 1 and 2a).               */
/* One decode step: append the new token's k, v at logical position L-1 (L = seq_lens[b],     */
/* counting the new token), then o = softmax(q K^T / sqrt(d)) V over keys j in [lo, L-1],     */
/* lo = 0 (FA) or max(0, L - window) (SWA). Query head h uses kv-head h / (Hq / Hkv).         */
/* Paged layout: k_pool, v_pool [n_pages][Hkv][page_tokens][d] bf16. FA: position p is at      */
/* (page_table[b][p / page_tokens], p % page_tokens). SWA keeps a ring of                      */
/* R = ceil(window / page_tokens) pages: position p is at ring index r = p mod (R*page_tokens),*/
/* i.e. (page_table[b][r / page_tokens], r % page_tokens).                                     */
/* ------------------------------------------------------------------------------------------ */

/* Workspace bytes attn_decode needs for these sizes (split-K partials; 0 is never returned).
 * The figure follows the launch plan for exactly these arguments and is not monotone in them
 * (a longer context may take fewer key ranges); size a shared workspace as the maximum over
 * every (kind, window, sizes) it will serve. It never exceeds 4 * B * Hq * 256 * (d + 2) + 12. */
HMD_API size_t attn_decode_workspace_size(hmd_kind_t kind, int window, int B, int Hq, int Hkv, int d,
                                  int page_tokens, int max_seq_len);

/*   q [B][Hq][d] bf16; new_k, new_v [B][Hkv][d] bf16; o [B][Hq][d] bf16.
 *   page_table [B][max_pages] int32 (device); seq_lens [B] int32 (device), each in
 *   [1, max_seq_len]; max_seq_len is a host-side upper bound that sizes the launch.
 *   workspace: device scratch of at least attn_decode_workspace_size(...) bytes.
 * Supported: d in {64, 128}; page_tokens == 64; Hq / Hkv <= 16. The pools must hold finite
 * values (freshly allocated pools from kv_cache_alloc are zero-filled).                       */
HMD_API hmd_status_t attn_decode(hmd_kind_t kind, int window, int B, int Hq, int Hkv, int d,
                         int page_tokens, const void *q, const void *new_k, const void *new_v,
                         void *k_pool, void *v_pool, int n_pages, const int32_t *page_table,
                         int max_pages, const int32_t *seq_lens, int max_seq_len, void *o,
                         void *workspace, size_t ws_bytes, hmd_stream_t stream);

/* Verification pass of speculative decoding (and multi-token decoding): n_q new tokens per
 * sequence in one pass, equal to n_q attn_decode steps in a row. Token i of sequence b sits at
 * logical position P = L - n_q + i (L = seq_lens[b] counts all n_q, each L >= n_q) and attends
 * keys j in [lo, P], lo = 0 (FA) or max(0, P + 1 - window) (SWA); all n_q tokens' k, v are
 * appended at their slots. Self-speculative decoding drafts tokens with a cheap placement of
 * the supernet and checks them with a better one ("Super Apriel: One Checkpoint, Many Speeds",
 * gist.science summary, sections 1 and 4); on a memory-bound decode step the n_q * (Hq / Hkv)
 * query rows of a kv-head share one pass over its pages, so checking n_q tokens costs about
 * one decode step. Rejected tokens need no undo: the next call's seq_lens decide what is read.
 *   q, o [B][n_q][Hq][d] bf16; new_k, new_v [B][n_q][Hkv][d] bf16; the rest as in attn_decode.
 *   ring_pages (SWA; ignored for FA): the ring's size in pages. Positions are kept at ring index
 *   p mod (ring_pages * page_tokens); it must hold window + n_q - 1 positions
 *   (ring_pages >= ceil((window + n_q - 1) / page_tokens), else HMD_ERR_SHAPE), so that the new
 *   tokens never overwrite a key an earlier row or the next step still reads. A cache verified
 *   this way must be decoded with attn_verify(n_q = 1) on the same ring_pages (attn_decode
 *   assumes ceil(window / page_tokens)).
 *   workspace: at least attn_verify_workspace_size(...) bytes.
 * Supported: d in {64, 128}; page_tokens == 64; n_q * (Hq / Hkv) <= 16 (HMD_ERR_UNSUPPORTED).
 * Allocates nothing. attn_decode is this call with n_q = 1 on the default ring.               */
HMD_API size_t attn_verify_workspace_size(hmd_kind_t kind, int window, int n_q, int B, int Hq,
                                          int Hkv, int d, int page_tokens, int max_seq_len);
HMD_API hmd_status_t attn_verify(hmd_kind_t kind, int window, int ring_pages, int n_q, int B,
                                 int Hq, int Hkv, int d, int page_tokens, const void *q,
                                 const void *new_k, const void *new_v, void *k_pool,
                                 void *v_pool, int n_pages, const int32_t *page_table,
                                 int max_pages, const int32_t *seq_lens, int max_seq_len,
                                 void *o, void *workspace, size_t ws_bytes, hmd_stream_t stream);

/* FA / SWA prefill of T prompt tokens per sequence into an empty paged cache. Token t of
 * sequence b is logical position t and attends keys j in [lo_t, t], lo_t = 0 (FA) or
 * max(0, t + 1 - window) (SWA): the attn_decode step with L = t + 1 for every t at once. The
 * prompt's K and V are written to the cache at the slots attn_decode reads (FA: every position;
 * SWA: the positions the ring keeps, t >= T - R*page_tokens), so decoding can follow directly.
 *   q, o [B][T][Hq][d] bf16; k, v [B][T][Hkv][d] bf16 (the prompt's own keys and values, which
 *   must hold finite values); k_pool, v_pool, page_table, n_pages as in attn_decode, with
 *   max_pages >= ceil(T / page_tokens) (FA) or R (SWA).
 * Supported: d in {64, 128}; page_tokens == 64; Hq / Hkv in {1, 2, 4, 8, 16}. q, k, v, o and
 * the pools must be 16-byte aligned (HMD_ERR_ARG). Allocates nothing.                          */
HMD_API hmd_status_t attn_prefill(hmd_kind_t kind, int window, int B, int T, int Hq, int Hkv,
                                  int d, int page_tokens, const void *q, const void *k,
                                  const void *v, void *k_pool, void *v_pool, int n_pages,
                                  const int32_t *page_table, int max_pages, void *o,
                                  hmd_stream_t stream);

/* attn_prefill after a cached prefix (chunked prefill): sequence b already holds positions
 * 0..prefix_lens[b]-1 in the paged cache (as attn_prefill / attn_decode wrote them); prompt
 * token t sits at position P = prefix_lens[b] + t and attends keys [lo, P], lo = 0 (FA) or
 * max(0, P + 1 - window) (SWA), reading the prefix keys from the cache and the prompt's own from
 * k, v. The prompt's K and V are then written at their slots (SWA: the positions the ring of
 * ceil(window / page_tokens) pages keeps; that write runs after every prefix key has been read).
 *   prefix_lens: device int32 [B], each a multiple of page_tokens and <= max_prefix (a host
 *   bound, itself a multiple of page_tokens); NULL is attn_prefill. FA needs
 *   max_pages >= ceil((max_prefix + T) / page_tokens).
 * Supported with a prefix: d in {64, 128}, as without one. A prefix
 * length that is not a whole number of pages sets HMD_DEVERR_SEQLEN (that sequence then runs as
 * if it had none).                                                                            */
HMD_API hmd_status_t attn_prefill_ext(hmd_kind_t kind, int window, int B, int T, int Hq, int Hkv,
                                      int d, int page_tokens, const void *q, const void *k,
                                      const void *v, const int32_t *prefix_lens, int max_prefix,
                                      void *k_pool, void *v_pool, int n_pages,
                                      const int32_t *page_table, int max_pages, void *o,
                                      hmd_stream_t stream);

/* attn_decode without a caller-provided workspace. The paper has no counterpart to this entry
 * point: it exists for callers that cannot allocate device memory, such as a plugin whose host
 * application owns all device memory through its own allocator, or a serving loop that forbids
 * device allocation after start-up. Arguments, layouts and results are those of attn_decode.
 * The split-K partials go to a fixed 16 MiB array compiled into the library (one per GPU that
 * loads it, held until the process exits); the call allocates nothing.
 *  - Returns HMD_ERR_UNSUPPORTED, before launching anything, when
 *    attn_decode_workspace_size(...) for these sizes exceeds 16 MiB (16777216 bytes).
 *  - The first call on each device looks up the array's device address (with that device
 *    current); make that first call before any stream capture.
 *  - All calls share the one array and leave it holding the last call's partials; nothing needs
 *    clearing, since each call writes every partial it reads. Calls that overlap on the GPU
 *    (different streams, or unordered host threads) race on it and must not be issued.       */
HMD_API hmd_status_t attn_decode_static_ws(hmd_kind_t kind, int window, int B, int Hq, int Hkv,
                                           int d, int page_tokens, const void *q,
                                           const void *new_k, const void *new_v, void *k_pool,
                                           void *v_pool, int n_pages, const int32_t *page_table,
                                           int max_pages, const int32_t *seq_lens,
                                           int max_seq_len, void *o, hmd_stream_t stream);

/* ------------------------------------------------------------------------------------------ */
/* Caches and the placement dispatcher.                                                       */
/* A placement selects one mixer per layer and can change between requests without reloading */
/* weights (abstract; gist.science summary, section 2d "Inference and serving"). The library  */
/* keeps every layer's caches registered for the life of the handles, so switching placements */
/* is passing a different placement array: nothing is copied or reallocated.                 */
/* ------------------------------------------------------------------------------------------ */

typedef struct hmd_state_cache hmd_state_cache_t;
typedef struct hmd_kv_cache hmd_kv_cache_t;

/* Recurrent-state cache: n_layers blocks of [slots][H][dk][dv] fp32, zero-filled.
 * Memory comes from cudaMallocAsync on `stream`; the handle is freed by state_cache_free.      */
HMD_API hmd_status_t state_cache_alloc(int n_layers, int slots, int H, int dk, int dv,
                               hmd_stream_t stream, hmd_state_cache_t **out);
HMD_API hmd_status_t state_cache_free(hmd_state_cache_t *cache, hmd_stream_t stream);
/* Device pointer of layer `layer`'s [slots][H][dk][dv] block.                                 */
HMD_API hmd_status_t state_cache_layer(hmd_state_cache_t *cache, int layer, float **out);
/* Copy n slots (host array `slot_ids`) of one layer out to `out` [n][H][dk][dv] fp32 (device),
 * asynchronously on `stream`: a request's recurrent state set aside (preemption, or a
 * checkpoint of a long prompt), to come back with state_cache_reset(..., init = out).
 * HMD_ERR_ARG for a bad layer, slot or null pointer.                                          */
HMD_API hmd_status_t state_cache_save(hmd_state_cache_t *cache, int layer, const int32_t *slot_ids,
                                      int n, float *out, hmd_stream_t stream);
/* Reset n slots (host array `slot_ids`) of one layer to zero, or to init [n][H][dk][dv] fp32
 * (device) when init is not NULL.                                                            */
HMD_API hmd_status_t state_cache_reset(hmd_state_cache_t *cache, int layer, const int32_t *slot_ids,
                               int n, const float *init, hmd_stream_t stream);

/* Paged KV cache: n_pools pairs of K and V pools [n_pages][Hkv][page_tokens][d] bf16,
 * zero-filled. layer_pool (host, n_layers entries) maps each layer to a pool, or -1 for none;
 * several layers may share a pool (aliasing, for placements whose KV exceeds memory).         */
HMD_API hmd_status_t kv_cache_alloc(int n_layers, const int32_t *layer_pool, int n_pools, int n_pages,
                            int Hkv, int d, int page_tokens, hmd_stream_t stream,
                            hmd_kv_cache_t **out);
HMD_API hmd_status_t kv_cache_free(hmd_kv_cache_t *cache, hmd_stream_t stream);
HMD_API hmd_status_t kv_cache_layer(hmd_kv_cache_t *cache, int layer, void **k_pool, void **v_pool);

/* Per-layer decode inputs. Delta layers read q, k, v with H heads and dk = dv = d, beta and
 * log_gate_scalar (GDN, [B][H]) or log_gate_channel (KDA, [B][H][d]), and the state slots.
 * Attention layers read q with H heads, k, v (the new token) with Hkv heads, page_table,
 * seq_lens, max_seq_len and window (SWA). o has H heads. A layer's io may fill only the fields
 * of the mixer kinds it can be switched to.                                                    */
typedef struct {
    int B, H, Hkv, d;
    hmd_dtype_t dtype;         /* activations; attention layers require HMD_BF16 */
    const void *q, *k, *v;
    const float *beta;
    const float *log_gate_scalar;
    const float *log_gate_channel;
    const int32_t *slots;      /* state slot per sequence (NULL: b) */
    const int32_t *page_table; /* [B][max_pages] */
    int max_pages;
    const int32_t *seq_lens;   /* [B], counting the new token */
    int max_seq_len;
    int window;                /* SWA window (keys, including the current token) */
    float scale;               /* delta layers: output scale (1.0 = the definition) */
    void *o;
} hmd_decode_io_t;

/* One decode token for layer `layer`: runs the mixer placement[layer] (host int8 array of
 * n_layers kinds) on that layer's registered caches. Attention layers need a workspace of
 * attn_decode_workspace_size(...) bytes for the chosen kind; one workspace serving layers that
 * can switch between FA and SWA takes the larger of the two sizes. Returns HMD_ERR_ARG if the chosen mixer's cache is not
 * registered for the layer (no pool for FA/SWA, no state block for GDN/KDA).                 */
HMD_API hmd_status_t mixer_decode_step(const int8_t *placement, int n_layers, int layer,
                               const hmd_decode_io_t *io, hmd_state_cache_t *state_cache,
                               hmd_kv_cache_t *kv_cache, void *workspace, size_t ws_bytes,
                               hmd_stream_t stream);

/* ------------------------------------------------------------------------------------------ */
/* Mixed placements in one batch. Placements switch between requests ("Super Apriel: One       */
/* Checkpoint, Many Speeds", abstract; gist.science summary, section 2d); here each sequence  */
/* of a batch may follow its own placement. A batch plan groups, for every layer, the          */
/* sequences by the mixer their placement picks there; one step of a layer then runs each     */
/* mixer once over its group through a device list of batch rows (no inputs are gathered or  */
/* copied: every kernel reads and writes row b of the full-batch tensors directly).            */
/* ------------------------------------------------------------------------------------------ */
typedef struct hmd_batch_plan hmd_batch_plan_t;

/* The grouping itself (host only, no device work): placements is a host int8 array
 * [n_placements][n_layers] of kinds, seq_placement [B] names each sequence's placement.
 * Writes rows [n_layers][B] (per layer: the FA rows, then SWA, KDA, GDN, each in increasing b)
 * and offsets [n_layers][5] (kind k's rows are rows[l][offsets[l][k] .. offsets[l][k+1])).
 * HMD_ERR_ARG for a bad kind, placement index or null pointer.                               */
HMD_API hmd_status_t hmd_group_sequences(int n_layers, int n_placements, const int8_t *placements,
                                         int B, const int32_t *seq_placement, int32_t *rows,
                                         int32_t *offsets);

/* Build a plan (the grouping above, with the rows uploaded to the device on `stream`; the
 * plan owns that memory until batch_plan_free). Build it outside any CUDA-graph capture; the
 * steps that use it can be captured.                                                          */
HMD_API hmd_status_t batch_plan_create(int n_layers, int n_placements, const int8_t *placements,
                                       int B, const int32_t *seq_placement, hmd_stream_t stream,
                                       hmd_batch_plan_t **out);
HMD_API hmd_status_t batch_plan_free(hmd_batch_plan_t *plan, hmd_stream_t stream);
/* Size of kind's group at a layer, and (optional) its rows on the host. */
HMD_API hmd_status_t batch_plan_group(const hmd_batch_plan_t *plan, int layer, hmd_kind_t kind,
                                      int *count, const int32_t **rows_host);
/* Attention workspace for every step of this plan: the largest attn_decode_workspace_size over
 * the plan's FA and SWA groups (the figure depends on the group size). */
HMD_API size_t batch_plan_workspace_size(const hmd_batch_plan_t *plan, int window, int Hq,
                                         int Hkv, int d, int page_tokens, int max_seq_len);

/* One decode token for layer `layer` of a mixed batch: for each kind with a non-empty group,
 * runs that mixer over the group's rows, with io[kind] (an array of 4 pointers indexed by
 * hmd_kind_t; entries of absent kinds may be NULL) describing the full-batch tensors of that
 * mixer (io[kind]->B must equal the plan's B). FA and SWA groups of a layer share its
 * registered pool (SWA on the ring of ceil(window / page_tokens) pages). The groups run in
 * turn on `stream`, sharing `workspace` (batch_plan_workspace_size bytes). Each sequence's
 * results are those of mixer_decode_step under its own placement.                              */
HMD_API hmd_status_t mixer_decode_step_batch(const hmd_batch_plan_t *plan, int layer,
                                             const hmd_decode_io_t *const *io,
                                             hmd_state_cache_t *state_cache,
                                             hmd_kv_cache_t *kv_cache, void *workspace,
                                             size_t ws_bytes, hmd_stream_t stream);

/* ------------------------------------------------------------------------------------------ */
/* Diagnostics.                                                                               */
/* ------------------------------------------------------------------------------------------ */
HMD_API const char *hmd_status_string(hmd_status_t status);
/* The status of the most recent failing call on this host thread (HMD_OK if none), cleared on
 * read.                                                                                       */
HMD_API hmd_status_t hmd_last_error(void);
/* Synchronise `stream`, then read the current device's error word (HMD_DEVERR_* bits) into
 * *bits and clear it when clear != 0.                                                         */
HMD_API hmd_status_t hmd_device_errors(hmd_stream_t stream, uint32_t *bits, int clear);
/* Library version string. */
HMD_API const char *hmd_version(void);

/* ------------------------------------------------------------------------------------------ */
/* Failure-detection testing hook. The paper has no counterpart: it exists so that the bounded */
/* waits of the kernels (every wait on a copy barrier gives up instead of hanging, reports    */
/* HMD_DEVERR_TIMEOUT and writes nothing) can be exercised without any invalid access.        */
/* ------------------------------------------------------------------------------------------ */
typedef enum { HMD_TEST_DELTA_DECODE = 0, HMD_TEST_ATTN_SPLIT = 1 } hmd_test_kernel_t;
/* Arms a one-shot fault for the next launch of `kernel` made by this host thread (the delta-rule
 * decode kernel of delta_rule_decode*, or the split kernel of attn_decode / attn_verify): CTA
 * `cta` of that launch arms its first copy barrier for the copy's bytes but issues no copy, so
 * its wait can never complete, and every bounded wait of the launch gives up after wait_ns
 * nanoseconds (1e3 .. 2e9) instead of 2 s. That CTA then reports HMD_DEVERR_TIMEOUT and leaves
 * its outputs untouched (delta decode: its state slice and its columns of o; attention: the
 * query heads of its kv-head for that sequence, whose combine is skipped); every other CTA runs
 * normally. A cta beyond the launch's grid arms nothing that fires; cta = -1 disarms.
 * HMD_ERR_ARG for a bad kernel, cta < -1 or wait_ns out of range.                             */
HMD_API hmd_status_t hmd_test_arm_copy_skip(hmd_test_kernel_t kernel, int cta, uint64_t wait_ns);

#ifdef __cplusplus
}
#endif
#endif /* HMD_H */

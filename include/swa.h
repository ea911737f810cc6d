/*
 * swa.h -- C ABI of libswa.so: the attention core of a hybrid sliding-window /
 * full-attention GQA decoder layer on NVIDIA B200 (sm_100a).
 *
 * The operation (page title, section that defines it):
 *   - "Step-3.7-Flash-oQ3e" explainer, section 2.2: sliding layers attend
 *     through a sliding-window causal mask and keep only the last W (= 512)
 *     tokens of KV cache; full layers use a plain causal mask.  Read here as:
 *     query i sees key j iff i - W < j <= i (W keys, self included);
 *     window = SWA_WINDOW_FULL means no lower bound.
 *   - same page, section 2.3: rope_theta is chosen per layer, partial rotary
 *     factors rotate only part of each head on full layers, and every head
 *     has its own sigmoid output gate.  Read here as: the first rotary_dim
 *     dims are rotated in rotate-half pairs (k, k + rotary_dim/2) by the angle
 *     p * rope_theta^(-2k/rotary_dim); the gate multiplies the normalised
 *     attention output of (token, q-head) by sigmoid(gate logit).
 *   - "Step-3.7-Flash" spec card, config dump: 64 query heads in 8 attention
 *     groups (att_impl_type GQA).  Read here as: q-head h uses kv-head
 *     h / (num_q_heads / num_kv_heads).
 *   - "Muse-Glimmer-30B-6bit" explainer, RoPE section: a layer rope theta of
 *     0 means the layer applies no rotary encoding.
 *   Scores are softmax_scale * <q_i, k_j> (default 1/sqrt(head_dim)), the
 *   masked softmax is taken over the visible keys, and the output is the
 *   softmax-weighted sum of values.
 *
 * Conventions for every call:
 *   - Tensors are device pointers to contiguous row-major arrays in the layout
 *     stated at each argument; bf16 tensors are passed as uint16_t (their bit
 *     patterns).  Every tensor pointer must be 16-byte aligned and point into
 *     the memory of the current device (the one `stream` belongs to); the
 *     calls do not check the device of a pointer.
 *   - The caller owns all memory.  No call allocates device memory; calls that
 *     need scratch take a caller-provided workspace whose size a *_size()
 *     query returns.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream) and never synchronise the host.
 *   - Errors: argument problems are reported before anything is launched
 *     (SWA_ERR_INVALID_ARG / SWA_ERR_UNSUPPORTED / SWA_ERR_WORKSPACE); a
 *     failed launch returns SWA_ERR_CUDA.  swa_last_error_detail() describes
 *     the last failure of the calling thread.  Kernels never trap: a device-
 *     side wait that runs out of time records a code that swa_device_error()
 *     reads.  No C++ exception crosses this interface.
 */
#ifndef SWA_H_
#define SWA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SWA_API __attribute__((visibility("default")))
#else
#define SWA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum swa_status {
  SWA_OK = 0,
  SWA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size or parameter */
  SWA_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. head_dim != 128) */
  SWA_ERR_WORKSPACE = 3,     /* workspace pointer missing or too small */
  SWA_ERR_CUDA = 4           /* a CUDA runtime/driver call failed */
} swa_status;

#define SWA_WINDOW_FULL (-1)

/* One attention layer's parameters. */
typedef struct swa_layer_params {
  int32_t num_q_heads;   /* Hq >= 1 */
  int32_t num_kv_heads;  /* Hkv >= 1, Hq % Hkv == 0 */
  int32_t head_dim;      /* D; 128 is the only supported value */
  int32_t window;        /* W >= 1 for a sliding layer; SWA_WINDOW_FULL for full causal */
  double rope_theta;     /* >= 0; 0 means no rotary encoding */
  int32_t rotary_dim;    /* even, 0..head_dim; 0 means no rotary encoding */
  float softmax_scale;   /* > 0, or <= 0 for 1/sqrt(head_dim) */
  /* Host pointer to rotary_dim/2 angular frequencies (each finite, >= 0)
   * that replace rope_theta^(-2k/rotary_dim), or NULL.  For a scaled RoPE
   * computed by the caller: the Step explainer's section 2.3 gives the full
   * layers a YaRN scaling (llama3 style, factor 2.0) without its other
   * parameters.  Read during the call only (copied into the launch); with a
   * table the layer rotates whenever rotary_dim > 0, whatever rope_theta is.
   * A zero-initialised struct leaves it NULL. */
  const double* inv_freq;
} swa_layer_params;

/*
 * swa_rope_qk -- rotary position encoding of q and k in place, optionally
 * appending the rotated keys and the raw values to a KV cache.
 * (Step explainer section 2.3; Muse explainer RoPE section; the cache rule is
 *  Step explainer section 2.2: a sliding layer keeps the last W tokens.)
 *
 *   q        [B, S, Hq, D] bf16, rotated in place; may be NULL.
 *   k        [B, S, Hkv, D] bf16, rotated in place; may be NULL.
 *   pos      [B, S] int32 device positions (each >= 0), or NULL: token s of
 *            every sequence is at position pos0 + s.
 *   v        [B, S, Hkv, D] bf16; required iff the caches are given.
 *   k_cache, v_cache  [B, Hkv, C, D] bf16 with C = cache_capacity, or both
 *            NULL.  Token at position p goes to slot p mod W on a sliding
 *            layer (C must equal W) and to slot p on a full layer (p < C is
 *            the caller's promise; C >= 1).  k must be given with caches.
 *            On a sliding layer with pos == NULL only the last W positions
 *            pos0 + S - W .. pos0 + S - 1 are written, so no two tokens of one
 *            call write the same slot; with explicit positions, no two tokens
 *            of one sequence in a call may map to the same slot (caller's
 *            promise).
 *   The angle is p * theta^(-2k/rotary_dim) (p * inv_freq[k] with a table),
 *   evaluated in fp64; the rotation itself runs in fp32 and the result is
 *   rounded to bf16.  With rotary_dim == 0, or theta == 0 and no table, q/k
 *   are left unchanged and the caches (if any) still receive k and v.
 */
SWA_API swa_status swa_rope_qk(const swa_layer_params* params, int32_t B, int32_t S, uint16_t* q, uint16_t* k,
                       const int32_t* pos, int32_t pos0, const uint16_t* v, uint16_t* k_cache,
                       uint16_t* v_cache, int32_t cache_capacity, void* stream);

/*
 * swa_prefill_workspace_size -- bytes of workspace swa_attn_prefill needs for
 * (params, B, S): the rotated keys [B, S, Hkv, D] bf16 plus the fp32 cos/sin
 * table of positions 0..S-1 (rounded up to a multiple of 32 positions), each
 * 256-byte aligned; 0 when the layer applies no rotary encoding.  Returns 0
 * for invalid parameters.
 */
SWA_API size_t swa_prefill_workspace_size(const swa_layer_params* params, int32_t B, int32_t S);

/*
 * swa_attn_prefill -- causal (W infinite) or banded (W finite) GQA attention
 * of S tokens at positions 0..S-1, RoPE included, with the per-head gate.
 * (Step explainer sections 2.2 and 2.3; spec card GQA groups.)
 *
 *   q      [B, S, Hq, D]  bf16, NOT rotated (RoPE is applied on the tile load)
 *   k      [B, S, Hkv, D] bf16, NOT rotated
 *   v      [B, S, Hkv, D] bf16
 *   gate   [B, S, Hq] fp32 logits, or NULL for no gate
 *   out    [B, S, Hq, D]  bf16: sigmoid(gate) * softmax(scale q k^T) v,
 *          accumulated in fp32 and rounded to nearest-even bf16
 *   workspace / workspace_bytes: at least swa_prefill_workspace_size()
 *          bytes of device memory, 256-byte aligned; overwritten.
 *   q, k, v, gate and workspace must not overlap out.
 */
SWA_API swa_status swa_attn_prefill(const swa_layer_params* params, int32_t B, int32_t S, const uint16_t* q,
                            const uint16_t* k, const uint16_t* v, const float* gate, uint16_t* out,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * swa_prefill_chunk_workspace_size -- bytes of workspace
 * swa_attn_prefill_chunk needs for (params, B, S, pos0): on a sliding layer
 * the keys and values the chunk attends to (up to W - 1 earlier tokens plus
 * the chunk) as [B, h + S, Hkv, D] bf16 each, h = min(pos0, W - 1); on a full
 * layer the rotated chunk keys [B, S, Hkv, D]; plus the cos/sin table of
 * positions pos0 .. pos0 + S - 1 when the layer rotates.  Each part 256-byte
 * aligned.  Returns 0 for invalid parameters.
 */
SWA_API size_t swa_prefill_chunk_workspace_size(const swa_layer_params* params, int32_t B, int32_t S,
                                                 int32_t pos0);

/*
 * swa_attn_prefill_chunk -- continue a prefill: S new tokens at positions
 * pos0 .. pos0 + S - 1 of each of B sequences whose tokens 0 .. pos0 - 1 are
 * already in the KV cache (rotated keys, raw values, as swa_rope_qk or an
 * earlier chunk wrote them).  Each new token attends to its visible keys --
 * cached and new -- exactly as in swa_attn_prefill over the whole sequence
 * (the same rows of the same result), and the chunk's keys and values are
 * then in the cache, so decode or the next chunk can follow.  pos0 = 0
 * is a whole prefill that also fills the cache.  (Step explainer section 2.2:
 * the sliding layers' cache keeps the last W tokens, the KV cache prefill
 * the page mentions; sections 2.3 for RoPE and the gate.)
 *
 *   q, k, v  [B, S, Hq | Hkv, D] bf16 of the new tokens, NOT rotated
 *   gate     [B, S, Hq] fp32 logits, or NULL
 *   k_cache, v_cache  [B, Hkv, C, D] bf16, C = cache_capacity: a sliding
 *            layer's ring (C must equal W; position p in slot p mod W) or a
 *            full layer's linear cache (slot p; C >= pos0 + S).  Read for
 *            positions < pos0, written for the new positions (on a ring only
 *            the last W of them).
 *   out      [B, S, Hq, D] bf16
 *   workspace / workspace_bytes: at least swa_prefill_chunk_workspace_size()
 *            bytes, 256-byte aligned; overwritten.
 *   No tensor may overlap another.  Positions pos0 + S must stay below 2^31.
 */
SWA_API swa_status swa_attn_prefill_chunk(const swa_layer_params* params, int32_t B, int32_t S, int32_t pos0,
                                          const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                          const float* gate, uint16_t* k_cache, uint16_t* v_cache,
                                          int32_t cache_capacity, uint16_t* out, void* workspace,
                                          size_t workspace_bytes, void* stream);

/*
 * swa_decode_workspace_size -- bytes of workspace swa_attn_decode needs for a
 * batch of B sequences whose lengths are at most max_len (split-K partial
 * results).  Returns 0 when no workspace is needed or parameters are invalid.
 */
SWA_API size_t swa_decode_workspace_size(const swa_layer_params* params, int32_t B, int32_t max_len);

/*
 * swa_attn_decode -- one query token per sequence against its KV cache.
 * (Step explainer section 2.2: a sliding layer's cache holds only the last W
 *  tokens; full layers see the whole history.)
 *
 *   q        [B, Hq, D] bf16, ALREADY rotated (swa_rope_qk at p = L_b - 1)
 *   gate     [B, Hq] fp32 logits, or NULL
 *   k_cache  [B, Hkv, C, D] bf16 rotated keys; v_cache same shape, raw values
 *   cache_capacity  C: must equal W on a sliding layer (ring of W slots,
 *            position p in slot p mod W); on a full layer slot p holds
 *            position p and C >= every seq_lens[b].
 *   seq_lens [B] int32 device, 1 <= L_b, counting the current token (already
 *            appended); the query sits at position L_b - 1 and sees the
 *            min(L_b, W) filled ring slots (sliding) or slots 0..L_b-1 (full).
 *   max_len  host-side upper bound of seq_lens (sizes the split grid).  A
 *            sequence longer than max_len breaks this contract: the keys
 *            past the planned splits are not read (its output is wrong) and
 *            device error 203 is recorded; no read leaves the workspace.
 *   out      [B, Hq, D] bf16
 *   workspace / workspace_bytes: at least swa_decode_workspace_size() bytes
 *            (may be NULL when that is 0); overwritten.
 *   Cache slots that are not visible are never read as values: they may
 *   hold anything, including NaN.
 */
SWA_API swa_status swa_attn_decode(const swa_layer_params* params, int32_t B, const uint16_t* q, const float* gate,
                           const uint16_t* k_cache, const uint16_t* v_cache, int32_t cache_capacity,
                           const int32_t* seq_lens, int32_t max_len, uint16_t* out, void* workspace,
                           size_t workspace_bytes, void* stream);

/*
 * swa_decode_mq_workspace_size -- bytes of workspace swa_attn_decode_mq needs
 * for B sequences of T new tokens whose lengths (new tokens included) are at
 * most max_len.  Returns 0 when no workspace is needed or parameters are
 * invalid.
 */
SWA_API size_t swa_decode_mq_workspace_size(const swa_layer_params* params, int32_t B, int32_t T,
                                            int32_t max_len);

/*
 * swa_attn_decode_mq -- T new tokens per sequence attend in one call, each
 * through its own band: the check of tokens proposed by multi-token-
 * prediction (MTP) layers ("Step-3.7-Flash" spec card, architecture notes:
 * three such layers speed up decoding) or any other speculative draft.  Band and cache rule: Step explainer section 2.2; gate:
 * section 2.3.
 *
 *   T        1 <= T <= 16 new tokens per sequence, and T * (Hq / Hkv) <= 64
 *            (SWA_ERR_UNSUPPORTED otherwise).
 *   q        [B, T, Hq, D] bf16, ALREADY rotated (positions L_b - T .. L_b - 1)
 *   gate     [B, T, Hq] fp32 logits, or NULL
 *   k_new    [B, T, Hkv, D] bf16, the new tokens' ALREADY rotated keys
 *   v_new    [B, T, Hkv, D] bf16, their values
 *   k_cache, v_cache  [B, Hkv, C, D] bf16 holding the L_b - T EARLIER tokens
 *            only: a ring of C = W slots on a sliding layer (position p in
 *            slot p mod W), slots 0 .. L_b - T - 1 on a full layer
 *            (C >= max_len - T).  The new tokens are NOT in the cache, so a
 *            rejected draft never overwrites a ring slot; append the accepted
 *            ones afterwards with swa_rope_qk (rotary_dim = 0 in a copy of the
 *            parameters appends already rotated keys unchanged).
 *   seq_lens [B] int32 device, L_b >= T, counting the T new tokens.  Query t
 *            sits at position L_b - T + t and sees the keys j with
 *            p - W < j <= p: cached ones and new tokens 0 .. t.  A sequence
 *            with L_b < T (or, full layer, L_b - T > C) records device error
 *            403 (404) and its rows are left unwritten.
 *   max_len  host-side upper bound of seq_lens (sizes the split grid).
 *   out      [B, T, Hq, D] bf16
 *   workspace / workspace_bytes: at least swa_decode_mq_workspace_size()
 *            bytes (may be NULL when that is 0); overwritten.
 *   Cache slots outside every query's band (unfilled slots, the oldest ring
 *   entry) are never read as values: they may hold anything, including NaN.
 */
SWA_API swa_status swa_attn_decode_mq(const swa_layer_params* params, int32_t B, int32_t T, const uint16_t* q,
                                      const float* gate, const uint16_t* k_new, const uint16_t* v_new,
                                      const uint16_t* k_cache, const uint16_t* v_cache, int32_t cache_capacity,
                                      const int32_t* seq_lens, int32_t max_len, uint16_t* out, void* workspace,
                                      size_t workspace_bytes, void* stream);

/*
 * swa_kv_cache_bytes -- bytes of one layer's K and V cache for `batch`
 * sequences of up to `context` tokens: batch x Hkv x C x D x 2 (K and V) x 2
 * (bf16), with C = min(context, W) on a sliding layer and C = context on a
 * full layer.  (Muse explainer, GQA section: the per-model footprint is this
 * summed over layers.)  Returns -1 for invalid arguments.
 */
SWA_API int64_t swa_kv_cache_bytes(const swa_layer_params* params, int64_t batch, int64_t context);

/* Human-readable name of a status code (static string). */
SWA_API const char* swa_status_string(swa_status status);

/* Detail of the calling thread's last failed call (static per-thread buffer;
 * "" if none). */
SWA_API const char* swa_last_error_detail(void);

/*
 * swa_device_error -- reads the device-side error word of the current device
 * (synchronises the device first).  *code = 0 means no kernel recorded an
 * error; otherwise the kernel and wait site whose bounded wait ran out
 * (decimal: kernel * 100 + site).  reset != 0 clears the word afterwards.
 */
SWA_API swa_status swa_device_error(int32_t* code, int32_t reset);

/* Library version string. */
SWA_API const char* swa_version(void);

/*
 * swa_attn_decode_no_alloc -- swa_attn_decode for callers that cannot obtain
 * device memory at call time.  The pages have no counterpart: this is an
 * interface convenience of this library, not part of the method.
 *
 * Who needs it: code that runs where cudaMalloc is unavailable or unwanted,
 * for example a plugin inside an engine that plans all device memory up
 * front and hands its plugins no allocator, a host callback in which CUDA API
 * calls are not permitted to allocate, or a latency-critical serving loop in
 * which an allocation could stall on the device.  Such callers cannot supply
 * the workspace that swa_attn_decode takes.
 *
 * Arguments and result are those of swa_attn_decode without the workspace:
 * the split-K partial results live in one statically sized device array of
 * SWA_NO_ALLOC_SCRATCH_BYTES bytes inside libswa.so, which every GPU that
 * loads the library holds until the process exits.  Each split of a
 * (sequence, q-head) row takes 520 bytes there.  When the usual split of the
 * cache would not fit, fewer, longer splits are used; when even two splits
 * per row do not fit (B * Hq * 2 * 520 bytes, plus 512 bytes of alignment,
 * above SWA_NO_ALLOC_SCRATCH_BYTES), each row's whole visible range runs as
 * one split, which writes the output directly and uses none of the array
 * (slower for long contexts and small batches, never refused for size).
 * Nothing in the array needs to start at zero: every partial a call reads was
 * written earlier in the same call.
 *
 * All calls on a device share that array, and it keeps the contents of the
 * last call: two calls whose kernels overlap on the GPU (different streams,
 * or different host threads, without ordering between them) race on it and
 * may return wrong results.  Order such calls on one stream or with events.
 *
 * The first call on each device does a one-time set-up: it looks up the
 * device address of the array with cudaGetSymbolAddress while that device is
 * current.  The call itself allocates nothing: no cudaMalloc, cudaFree or
 * allocating library routine.
 */
#define SWA_NO_ALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)

SWA_API swa_status swa_attn_decode_no_alloc(const swa_layer_params* params, int32_t B, const uint16_t* q,
                                            const float* gate, const uint16_t* k_cache, const uint16_t* v_cache,
                                            int32_t cache_capacity, const int32_t* seq_lens, int32_t max_len,
                                            uint16_t* out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SWA_H_ */

/*
 * libmimoattn — MiMo-V2.6-Flash hybrid attention forward on NVIDIA B200 (sm_100a).
 *
 * The operation is the attention layer that the model pages state
 * (radixark miles docs "MiMo-V2.6-Flash", section 1 "Key highlights" and
 * section 5.4 "Notable quirks"; "Model techniques map" page, sections
 * "Grouped-query attention", "Sliding-window attention", "Learnable attention
 * sink", "Partial RoPE"; gaudi-cookbook "MiMo-V2.6-Flash-RL", "Required fixes"):
 *
 *   64 query heads, KV heads 8 (sliding-window layers) or 4 (global layers);
 *   query head h reads KV head h / (64 / num_kv_heads);
 *   Q/K head dim 192, V head dim 128; NeoX rotate-half RoPE on dims 0..63 with
 *   frequencies base^(-2j/64), j = 0..31, angles taken from float64;
 *   query at position p sees keys t with t <= p and (window == 0 or p - t < window);
 *   z_t = softmax_scale * q.k_t; an optional per-query-head sink logit s_h joins
 *   the softmax denominator and carries no value;
 *   out = v_scale * sum_t softmax(z, s_h)_t v_t;   lse = ln(sum_t e^{z_t} + e^{s_h}).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller, 16-byte
 *     aligned, dense and row-major in the stated shape.  bf16 tensors are
 *     passed as `void*` (IEEE bfloat16 bit patterns).
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls only
 *     enqueue work: no host synchronisation, no memory allocation.
 *   - Return MIMO_OK or a MIMO_ERR_* code; mimo_last_error() gives a message
 *     (thread-local).  Arguments are validated on the host before any launch; a
 *     rejected call enqueues nothing.
 *   - Device-side problems (a bounded wait that ran out, an index outside a
 *     cache) set bits in a device status word instead of faulting; read and
 *     clear it with mimo_status_poll().
 *   - The fixed model dimensions (64 / 192 / 128 / 64) are the only ones
 *     supported; other values return MIMO_ERR_UNSUPPORTED.
 */
#ifndef MIMOATTN_H
#define MIMOATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MIMO_API __attribute__((visibility("default")))
#else
#define MIMO_API
#endif

#define MIMO_OK 0
#define MIMO_ERR_INVALID_ARG 1 /* a NULL / misaligned pointer, a bad size */
#define MIMO_ERR_UNSUPPORTED 2 /* dims or head counts other than the model's */
#define MIMO_ERR_WORKSPACE 3   /* workspace missing or smaller than required */
#define MIMO_ERR_CUDA 4        /* a CUDA runtime / driver call failed */
#define MIMO_ERR_TIMEOUT 5     /* a device wait gave up (from mimo_status_poll) */

/* Device status bits reported by mimo_status_poll(). */
#define MIMO_STATUS_TIMEOUT 1u    /* a bounded barrier / copy wait ran out */
#define MIMO_STATUS_BAD_INDEX 2u  /* a page id, slot or position outside its cache */
#define MIMO_STATUS_RANGE 4u      /* a rotated query / key component beyond fp16's range,
                                     stored saturated at +-65504 */
#define MIMO_STATUS_BAD_SCALE 8u  /* an E4M3 dequantisation scale not finite and positive */

/* The attention layer.  num_q_heads 64, head_dim_qk 192, head_dim_v 128 and
 * rope_dim 64 are required; num_kv_heads is 8 or 4. */
typedef struct {
  int num_q_heads;
  int num_kv_heads;
  int head_dim_qk;
  int head_dim_v;
  int rope_dim;
  double rope_base;    /* 1e4 (sliding-window layers) or 1e7 (global layers); > 0 */
  float softmax_scale; /* 1/sqrt(192) in the model */
  float v_scale;       /* 0.707 in the model; applied to the output (attention is linear in V) */
  int window;          /* keys in total including the query itself (128 in the model);
                          0 = global causal attention */
  const float* sink;   /* device fp32 [num_q_heads] sink logits, or NULL for no sink */
} mimo_layer;

/* The (left, right) form of the window, as the sliding-window layers are configured in
 * the SGLang / miles stack (radixark miles docs "MiMo-V2.6-Flash", section 5.4 "Notable
 * quirks", which sets the window as (128, 0) there against 128 keys in total in the HF
 * and Megatron-Bridge code): a query at position p sees the keys at positions
 * [p - left, p + right].  The layers are causal, so right must be 0; left = -1 means no
 * left bound (a global layer).  Writes the equivalent `window` of mimo_layer (keys in
 * total including the query: left + 1, or 0 for left = -1) to *window, so (128, 0)
 * gives 129 and (127, 0) gives 128.
 * Errors: MIMO_ERR_UNSUPPORTED for right != 0 (non-causal); MIMO_ERR_INVALID_ARG for
 * left < -1, left + 1 overflowing an int, or window == NULL.  Host only: touches no
 * device and launches nothing. */
MIMO_API int mimo_window_from_left_right(int left, int right, int* window);

/* KV cache layouts.  The serving pages keep window-sized KV for the sliding-window
 * layers and paged KV in blocks of 128 positions for the global layers (gaudi-cookbook
 * "MiMo-V2.6-Flash-RL", section "Launch": MIMO_SWA_KV_GROUPS=1 gives the 39 sliding
 * layers window-sized KV, --block-size 128), and their exact decode window keeps one
 * block more than the window with the oldest block masked (same page, "Fixes" table,
 * swa-decode-window).
 *   MIMO_CACHE_PAGED: [num_pages, 128, Hkv, D]; position p of sequence s sits in page
 *     block_table[s][p / 128], slot p % 128.
 *   MIMO_CACHE_RING: [num_seqs, ring_slots, Hkv, D]; position p of sequence s sits in slot
 *     p % ring_slots, so the ring holds the last ring_slots positions appended.  ring_slots
 *     (a field of the prefill, decode and append arguments; 0 means 128) is a multiple of
 *     16 in 128..512.  The model's window of 128 keys fits 128 slots.  The SGLang window of
 *     the query plus 128 previous keys (radixark miles docs "MiMo-V2.6-Flash", section 5.4)
 *     needs at least 129 slots to decode, because appending the query's own key overwrites
 *     the oldest slot: 144 is the smallest ring that serves it. */
#define MIMO_CACHE_NONE 0
#define MIMO_CACHE_PAGED 1
#define MIMO_CACHE_RING 2
#define MIMO_RING_SLOTS_DEFAULT 128
#define MIMO_RING_SLOTS_MAX 512

/* Cache element formats (mimo_decode_args.cache_dtype, mimo_append_args.cache_dtype).
 *   MIMO_DTYPE_BF16: key dims 0..63 (the rotated part) as IEEE fp16, key dims
 *     64..191 and the value as bf16 (2 bytes per element).
 *   MIMO_DTYPE_FP8_E4M3: every key and value element is one OCP E4M3 byte; it
 *     stands for code * k_dequant[g] (keys of KV head g) or code * v_dequant[g]
 *     (values).  Appends quantise x / dequant with round-to-nearest-even,
 *     saturating at +-448.  Decode only (prefill reads bf16 caches).  The vLLM
 *     recipe page for MiMo-V2.6-Flash ("Launch command", the AMD MI355X line)
 *     serves the model with an FP8 KV cache (--kv-cache-dtype fp8) without
 *     saying how it is scaled; one scale per KV head is this library's reading.
 *     It halves the bytes a decode step streams. */
#define MIMO_DTYPE_BF16 0
#define MIMO_DTYPE_FP8_E4M3 1

/*
 * Prefill (varlen, causal, window or global, sink on/off).
 *
 * Sequence s has q_len = cu_seqlens_q[s+1]-cu_seqlens_q[s] query rows and
 * k_len = cu_seqlens_k[s+1]-cu_seqlens_k[s] new (pre-RoPE) key/value rows.
 * Its context length is ctx = cache_lens[s] + k_len (cache_lens NULL = 0).
 * Queries sit at positions ctx - q_len .. ctx - 1 (bottom-right aligned), new
 * keys at positions cache_lens[s] .. ctx - 1, and positions below cache_lens[s]
 * are read from the cache, where keys are stored already rotated.
 *
 *   MIMO_CACHE_NONE : all keys are new; k, v, cu_seqlens_k required.
 *   MIMO_CACHE_RING : sliding-window chunk: the ring holds the prefix tail, positions
 *                     cache_lens[s]-ring_slots .. cache_lens[s]-1 (not yet overwritten by
 *                     this chunk), of which the last 128 are read; requires window in
 *                     1..129 (a window reaches at most 128 positions before the chunk).
 *   MIMO_CACHE_PAGED: all keys come from the paged cache (append the chunk with
 *                     mimo_kv_append first); k, v, cu_seqlens_k must be NULL and
 *                     cache_lens[s] is the full context length.
 *
 * Layouts: q [total_q, 64, 192] bf16 pre-RoPE; k [total_k, Hkv, 192] bf16
 * pre-RoPE; v [total_k, Hkv, 128] bf16; out [total_q, 64, 128] bf16;
 * lse [total_q, 64] fp32 natural-log LSE including the sink (may be NULL).
 * The workspace (size from mimo_attn_prefill_workspace_size) holds rotated
 * key copies and a per-query-row table of the rotary cos / sin values; its
 * contents need no initialisation.
 * Cache slots at or beyond a sequence's context must hold finite values
 * (e.g. zero-initialise caches): they are read and masked, not skipped.
 */
typedef struct {
  mimo_layer layer;
  int num_seqs;
  int total_q;
  int total_k;              /* rows of k / v (0 for MIMO_CACHE_PAGED) */
  const void* q;
  const void* k;
  const void* v;
  const int32_t* cu_seqlens_q; /* device int32 [num_seqs+1] */
  const int32_t* cu_seqlens_k; /* device int32 [num_seqs+1] or NULL (paged) */
  const int32_t* cache_lens;   /* device int32 [num_seqs] or NULL */
  int cache_kind;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_table; /* paged: device int32 [num_seqs, max_pages] */
  int max_pages;
  int num_pages; /* paged: pages in the pool */
  void* out;
  float* lse;
  void* workspace;
  size_t workspace_bytes;
  /* Optional timing hooks: cudaEvent_t handles or NULL.  When set, they are
   * recorded on `stream` immediately before the first and after the last
   * launch of the attention kernel itself (not the key pre-pass), so that
   * cudaEventElapsedTime gives that kernel's device time. */
  void* ev_kernel_begin;
  void* ev_kernel_end;
  int ring_slots; /* MIMO_CACHE_RING: slots per sequence of the ring (0 = 128) */
} mimo_prefill_args;

/* Bytes of workspace mimo_attn_prefill needs for these sizes. */
MIMO_API size_t mimo_attn_prefill_workspace_size(int num_seqs, int total_q, int total_k, int num_kv_heads,
                                                 int cache_kind);

MIMO_API int mimo_attn_prefill(const mimo_prefill_args* args, void* stream);

/*
 * Failure-detection test of the prefill (no counterpart in the pages: it exercises this
 * library's own bounded waits).  Validates and enqueues exactly what mimo_attn_prefill
 * would, except that the attention kernel's producer never loads a query tile, so the
 * roles waiting for one give up after wait_limit_ns (1e6..1e10 ns), set
 * MIMO_STATUS_TIMEOUT in the device status word, wait for their copies and tensor-core
 * operations already in flight, free their tensor memory and return; the outputs are
 * left unspecified.  mimo_status_poll() then returns MIMO_ERR_TIMEOUT, and later calls
 * run normally.  Nothing faults and nothing waits without a limit.
 */
MIMO_API int mimo_attn_prefill_stall_test(const mimo_prefill_args* args, void* stream,
                                          unsigned long long wait_limit_ns);

/*
 * Decode: q_len query tokens per sequence, the last q_len positions of its context
 * (q_len = 1: one decode step; 2..MIMO_MAX_DRAFTS: draft tokens of speculative decoding
 * scored in one pass, as the serving pages run it: vLLM recipe page, DFlash; SGLang
 * cookbook page; radixark miles docs section 4.2, EAGLE with 4 draft tokens).  Query
 * row s * q_len + i sits at position seq_lens[s] - q_len + i and sees the keys up to its
 * own position (and, with a window, the window before it): draft i sees the context and
 * drafts 0..i.  The cache already holds positions 0 .. seq_lens[s]-1, the drafts
 * included (append them with mimo_kv_append first).  Sliding-window layers use a ring
 * cache (the last ring_slots positions are kept: window + q_len - 1 <= ring_slots),
 * global layers a paged cache (gaudi-cookbook "MiMo-V2.6-Flash-RL", "Launch":
 * window-sized KV for the sliding layers, blocks of 128 positions).
 *
 * Layouts: q [batch * q_len, 64, 192] bf16 pre-RoPE; out [batch * q_len, 64, 128] bf16;
 * lse [batch * q_len, 64] fp32 or NULL.  max_seq_len is a host-side upper bound of
 * seq_lens (it sizes the split-KV grid and the workspace); every seq_lens[s] >= q_len.
 * A sequence whose seq_lens is below q_len sets MIMO_STATUS_BAD_INDEX; its rows are
 * undefined.  A seq_lens above max_seq_len breaks the contract: keys beyond the splits
 * that max_seq_len sizes are not attended (reported as MIMO_STATUS_BAD_INDEX whenever the
 * call has more than one split).
 *
 * Kernels: one token per sequence, a ring cache, an E4M3 cache or a window run the
 * split-KV decode kernel; draft rows (q_len >= 2) of a global layer (4 KV heads, no
 * window) on a bf16 paged cache run the tensor-core prefill kernel, whose 128-row tile
 * holds the q_len x 16 query rows of one KV head, over page-aligned splits, then the same
 * combine pass.  Either way the split-KV workspace is the one the size queries give.
 */
#define MIMO_MAX_DRAFTS 8
typedef struct {
  mimo_layer layer;
  int batch;
  int max_seq_len;
  const void* q;
  const int32_t* seq_lens; /* device int32 [batch], each >= 1 */
  int cache_kind;          /* MIMO_CACHE_PAGED or MIMO_CACHE_RING */
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_table; /* paged: device int32 [batch, max_pages] */
  int max_pages;
  int num_pages;
  void* out;
  float* lse;
  void* workspace;
  size_t workspace_bytes;
  /* Optional timing hooks: cudaEvent_t handles or NULL.  When set, they are
   * recorded on `stream` immediately before the first and after the last
   * launch of the attention kernel itself (not the split combine pass), so that
   * cudaEventElapsedTime gives that kernel's device time. */
  void* ev_kernel_begin;
  void* ev_kernel_end;
  int cache_dtype;          /* MIMO_DTYPE_BF16 (default 0) or MIMO_DTYPE_FP8_E4M3 */
  const float* k_dequant;   /* FP8: device fp32 [num_kv_heads] key scales, else NULL */
  const float* v_dequant;   /* FP8: device fp32 [num_kv_heads] value scales, else NULL */
  int ring_slots;           /* MIMO_CACHE_RING: slots per sequence of the ring (0 = 128) */
  int q_len;                /* query tokens per sequence: 0 or 1 (decode), up to MIMO_MAX_DRAFTS */
} mimo_decode_args;

/* Bytes of workspace mimo_attn_decode needs (split-KV partials) for one query token per
 * sequence. */
MIMO_API size_t mimo_attn_decode_workspace_size(int batch, int max_seq_len, int num_kv_heads, int window);

/* The same for q_len query tokens per sequence (0 for q_len outside 1..MIMO_MAX_DRAFTS). */
MIMO_API size_t mimo_attn_verify_workspace_size(int batch, int q_len, int max_seq_len, int num_kv_heads,
                                                int window);

MIMO_API int mimo_attn_decode(const mimo_decode_args* args, void* stream);

/*
 * Decode for callers that cannot allocate device memory.
 *
 * No page describes this call: it is a deployment convenience.  Some callers
 * cannot call cudaMalloc at all: code running inside a CUDA graph capture
 * region, or runtimes whose only device memory is a fixed arena handed out by
 * someone else.  For them this entry point behaves exactly like
 * mimo_attn_decode, except that `workspace` / `workspace_bytes` in the
 * arguments are ignored: the split-KV partials go to a library-owned device
 * array of MIMO_DECODE_NOALLOC_MAX_BYTES (16 MiB) that every GPU which loads the
 * library holds until the process exits.
 *   - Nothing is allocated: no cudaMalloc / cudaFree, no allocating library call.
 *   - The first call on each device looks up that device's copy of the array
 *     (cudaGetSymbolAddress, with the device current): make that first call
 *     before any stream capture.  The address is looked up again when the
 *     device's context has changed since (after a device reset).
 *   - Problems whose partials need more than MIMO_DECODE_NOALLOC_MAX_BYTES
 *     (mimo_attn_decode_workspace_size of the same sizes) are rejected with
 *     MIMO_ERR_WORKSPACE before anything is enqueued.
 *   - All calls share the one array, so calls whose kernels overlap on the GPU
 *     (different streams, or different host threads) race and corrupt each
 *     other's results; serialise them.  No part of the array needs to start at
 *     zero: each call writes every partial it later reads.
 */
#define MIMO_DECODE_NOALLOC_MAX_BYTES (16u << 20)
MIMO_API int mimo_attn_decode_noalloc(const mimo_decode_args* args, void* stream);

/*
 * KV append: rotates the first 64 dims of each new key at its position (the
 * layer's RoPE base, angles from float64) and stores key and value (value
 * unscaled) in the cache: ring slot pos % ring_slots of sequence seq_idx[t], or page
 * block_table[seq_idx[t]][pos / 128], slot pos % 128 (the cache layouts above:
 * gaudi-cookbook "MiMo-V2.6-Flash-RL", "Launch").
 *
 * Layouts: k_new [num_tokens, Hkv, 192] bf16 pre-RoPE; v_new [num_tokens, Hkv, 128];
 * pos, seq_idx: device int32 [num_tokens].  Two tokens must not target the same slot.
 * A token whose sequence, position or page lies outside the cache is skipped and sets
 * MIMO_STATUS_BAD_INDEX.  For an E4M3 cache every k_dequant / v_dequant scale must be
 * finite and positive; a token of a KV head whose scale is not is skipped and sets
 * MIMO_STATUS_BAD_SCALE.  A rotated key component beyond the fp16 range (|x| > 65504)
 * is stored as +-65504 and sets MIMO_STATUS_RANGE (bf16 caches).
 */
typedef struct {
  int num_tokens;
  int num_kv_heads;
  int head_dim_qk;
  int head_dim_v;
  int rope_dim;
  double rope_base;
  const void* k_new;
  const void* v_new;
  const int32_t* pos;
  const int32_t* seq_idx;
  int cache_kind;
  void* k_cache;
  void* v_cache;
  int num_seqs;               /* ring: sequences in the ring cache */
  const int32_t* block_table; /* paged: device int32 [num_seqs, max_pages] */
  int max_pages;
  int num_pages;
  int cache_dtype;          /* MIMO_DTYPE_BF16 (default 0) or MIMO_DTYPE_FP8_E4M3 */
  const float* k_dequant;   /* FP8: device fp32 [num_kv_heads], else NULL */
  const float* v_dequant;
  int ring_slots;           /* MIMO_CACHE_RING: slots per sequence of the ring (0 = 128) */
} mimo_append_args;

MIMO_API int mimo_kv_append(const mimo_append_args* args, void* stream);

/* Thread-local message for the last error returned on this thread. */
MIMO_API const char* mimo_last_error(void);

/* Reads and clears the device status word of the current device
 * (synchronises the device).  Returns MIMO_STATUS_* bits in *status. */
MIMO_API int mimo_status_poll(uint32_t* status);

/* Library version string. */
MIMO_API const char* mimo_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MIMOATTN_H */

/*
 * kvattn.h -- C ABI of libkvattn.so: the cached grouped-query-attention step
 * of a Llama-3.1-style decoder on NVIDIA B200 (sm_100a).
 *
 * One call of the step, as "Llama 3 8B · KV cache" (its "update" and
 * "mask" code excerpts) and "Llama 3.1 8B KV cache" (sections "RoPE has to know
 * where it is" and "The cache itself is concatenation") describe it:
 *   1. rotate the new queries and keys with RoPE at absolute positions
 *      start_pos .. start_pos+T-1                    -> kvattn_rope_append
 *   2. write the rotated keys and the values into cache rows
 *      start_pos .. start_pos+T-1                    -> kvattn_rope_append
 *   3. attend softmax(q K^T / sqrt(d)) V over rows 0 .. start_pos+t with the
 *      rectangular causal mask, query head h reading KV head floor(h/G)
 *      ("Llama 3.1 8B · Repeat heads")               -> kvattn_decode (T = 1)
 *                                                    -> kvattn_prefill_chunk (T >= 1)
 *
 * Conventions shared by every entry point
 *  - Tensors are caller-owned, contiguous DEVICE memory.  bf16 tensors are
 *    passed as uint16_t bit patterns.  Every tensor pointer must be 16-byte
 *    aligned.
 *  - Layouts follow the code layout of "Llama 3 8B · KV cache" ([B,
 *    positions, heads, d]):
 *      q, q_rot, out        [B, T, H,   d]
 *      k_new, v_new         [B, T, Hkv, d]
 *      cache_k, cache_v     [B, S, Hkv, d]   (S = max_seq_len rows, allocated up front)
 *      start_pos            int32 [B] on the device: the past length of each
 *                           sequence, i.e. the first row this call writes.
 *  - Calls are asynchronous on `stream` (NULL = legacy default stream); the
 *    library performs no host synchronisation and allocates no memory.
 *  - Return value: KVATTN_OK, or a kvattn_status for problems found on the
 *    host before anything is launched (nothing is launched then).
 *  - Problems only the device can see (a start_pos outside the cache, a
 *    sequence longer than max_kv_len_hint, an in-kernel wait that gave up)
 *    skip the affected sequence's writes and OR a KVATTN_DEV_* bit into
 *    *dev_status (a device int32 the caller zeroes; may be NULL).
 */
#ifndef KVATTN_H
#define KVATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define KVATTN_API __attribute__((visibility("default")))
#else
#define KVATTN_API
#endif

struct CUstream_st;
/* Same type as cudaStream_t. */
typedef struct CUstream_st* kvattn_stream_t;

typedef enum kvattn_status {
  KVATTN_OK = 0,
  KVATTN_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, H % Hkv != 0 */
  KVATTN_ERR_UNSUPPORTED = 2, /* head_dim != 128, group size G = H/Hkv not in {1,2,4,...,128} */
  KVATTN_ERR_OUT_OF_RANGE = 3, /* a host-visible length outside the cache */
  KVATTN_ERR_WORKSPACE = 4,    /* workspace missing or smaller than required */
  KVATTN_ERR_CUDA = 5          /* a CUDA launch or query failed */
} kvattn_status;

/* Bits OR-ed into *dev_status by the kernels. */
#define KVATTN_DEV_START_POS_RANGE 0x1 /* start_pos[b] < 0 or start_pos[b]+T > max_seq_len */
#define KVATTN_DEV_KV_LEN_HINT 0x2     /* start_pos[b]+T > max_kv_len_hint */
#define KVATTN_DEV_WAIT_TIMEOUT 0x4    /* an in-kernel pipeline wait gave up */
#define KVATTN_DEV_INTERNAL 0x8        /* an internal invariant failed (the launch did nothing) */

typedef struct kvattn_dims {
  int32_t batch;       /* B: sequences in this call (rows 0..B-1 of the caches) */
  int32_t n_heads;     /* H: query heads (32 for Llama 3.1 8B, 64 for 70B) */
  int32_t n_kv_heads;  /* Hkv: key/value heads (8); G = H / Hkv query heads share one */
  int32_t head_dim;    /* d: must be 128 */
  int32_t max_seq_len; /* S: rows the caches were allocated with */
} kvattn_dims;

/* RoPE parameters: f_i = theta^(-2i/r), i < r/2, r = rotary_dim ("Llama 3.1
 * 8B KV cache", section "RoPE has to know where it is", with r = d), with
 * optional Llama-3.1 frequency scaling (use_scaled_rope in "Llama 3.1 8B ·
 * Repeat heads", sku_list.py excerpt): wavelengths 2*pi/f_i shorter than
 * original_max_pos/high_freq_factor are kept, longer than
 * original_max_pos/low_freq_factor are divided by `factor`, and in between f
 * becomes (1-s) f/factor + s f with
 * s = (original_max_pos/wavelength - low_freq_factor) /
 *     (high_freq_factor - low_freq_factor).
 * layout selects the rotated pairs: KVATTN_ROPE_INTERLEAVED (2i, 2i+1), the
 * Meta layout, or KVATTN_ROPE_HALF_SPLIT (i, i + r/2) (both listed with
 * partial rotary for the modern decoder block, "The Modern Decoder Block",
 * module L7.3).  Elements r..d-1 pass through unchanged. */
#define KVATTN_ROPE_INTERLEAVED 0
#define KVATTN_ROPE_HALF_SPLIT 1
typedef struct kvattn_rope_params {
  double theta;            /* 500000 for Llama 3 / 3.1 */
  int32_t use_scaled;      /* 0 or 1 */
  double factor;           /* 8 */
  double low_freq_factor;  /* 1 */
  double high_freq_factor; /* 4 */
  double original_max_pos; /* 8192 */
  int32_t layout;          /* KVATTN_ROPE_INTERLEAVED (0) or KVATTN_ROPE_HALF_SPLIT (1) */
  int32_t rotary_dim;      /* even, 2..head_dim; 0 means head_dim */
} kvattn_rope_params;

/* Steps 1-2 (cache write "C_K[p] <- K_r, C_V[p] <- V" of "Llama 3 8B · KV
 * cache"; the position offset of "Llama 3.1 8B KV cache", section "RoPE has to
 * know where it is").
 * For every b < B and t < T, with p = start_pos[b] + t:
 *   q_rot[b,t,h,:]   = RoPE_p(q[b,t,h,:])      for h < H
 *   cache_k[b,p,j,:] = RoPE_p(k_new[b,t,j,:])  for j < Hkv
 *   cache_v[b,p,j,:] = v_new[b,t,j,:]          (bit copy)
 * RoPE_p rotates each pair (a, b) of the chosen layout counter-clockwise by
 * p*f_i (the complex product (x_a + i x_b) e^{i p f_i}); elements at or past
 * rotary_dim are copied.  Angles, cos/sin
 * and the rotation are computed in fp64 and rounded once to bf16 (nearest,
 * ties to even).  q_rot may equal q (in place); it must not partially overlap
 * q.  No other cache row is touched.  A sequence with start_pos[b] < 0 or
 * start_pos[b] + T > max_seq_len writes nothing and sets
 * KVATTN_DEV_START_POS_RANGE.
 * Host errors: INVALID_ARG (null/misaligned pointer, T < 1, B < 1, S < 1,
 * H % Hkv != 0, non-finite or non-positive theta, bad layout or
 * rotary_dim), UNSUPPORTED (d != 128). */
KVATTN_API int kvattn_rope_append(const kvattn_dims* dims, const kvattn_rope_params* rope, int32_t T,
                       const uint16_t* q, uint16_t* q_rot, const uint16_t* k_new,
                       const uint16_t* v_new, uint16_t* cache_k, uint16_t* cache_v,
                       const int32_t* start_pos, int32_t* dev_status, kvattn_stream_t stream);

/* Bytes of device workspace kvattn_decode needs for these dims and
 * max_kv_len_hint on the CURRENT device (the split size depends on its SM
 * count).  0 on invalid arguments. */
KVATTN_API size_t kvattn_decode_workspace_bytes(const kvattn_dims* dims, int32_t max_kv_len_hint);

/* Step 3 for one new token per sequence (T = 1; the decode step of "Llama 3 8B
 * · KV cache" at p = 1000: write row 1000, read rows 0..1000).
 *   out[b,0,h,:] = sum_{r <= start_pos[b]} softmax_r(scale * q_rot[b,0,h,:] .
 *                  cache_k[b,r,floor(h/G),:]) * cache_v[b,r,floor(h/G),:]
 * The cache rows 0..start_pos[b] must already hold the sequence (row
 * start_pos[b] written by kvattn_rope_append earlier on the same stream).
 * The rows of each (sequence, KV head) are streamed from HBM once and serve
 * all G query heads.  At G = 32 (e.g. multi-query attention with 32 heads) a
 * call with more than one split runs on the 5th-generation tensor cores: the
 * 32 heads are 32 rows of a 128-row MMA tile, and the 128-row key tiles of
 * all (sequence, KV head) pairs, laid end to end, are cut into equal
 * contiguous ranges, two per SM (one per tensor-memory accumulator); each
 * piece of a sequence within a range leaves one partial.  G = 64, 128 (and
 * masked G = 32 calls) run as G/16 groups of 16 heads over the same rows,
 * scheduled side by side so the repeat reads are served by L2.  Long rows
 * are split across CTAs and the partial (o, max, sum) triples are merged by
 * log-sum-exp in a second kernel; the tensor-core G = 32 path uses the same
 * workspace layout and merge (never more partials per sequence than the
 * plan's splits).
 * scale <= 0 selects 1/sqrt(d).  max_kv_len_hint (<= 0: max_seq_len) is a
 * host upper bound on start_pos[b] + 1; it sizes the splits and the
 * workspace.  A sequence above the hint or outside the cache leaves its
 * output untouched and sets a KVATTN_DEV_* bit.  out is bf16 [B,1,H,d].
 * workspace: device memory of kvattn_decode_workspace_bytes() bytes, 16-byte
 * aligned, owned by the caller.  Its first 16 bytes hold a work counter that
 * must be ZERO before the first call (e.g. cudaMemset once after
 * allocation); every call leaves it zero again (the merge kernel resets it,
 * also after a pipeline wait gave up), so one workspace serves calls of any
 * shape with no memset between them.  After a call that returned
 * KVATTN_ERR_CUDA, zero those 16 bytes again before the next call.
 * Calls that share a workspace must be ordered on one stream.
 * Every kernel of the library is launched with programmatic stream
 * serialization and waits for the previous kernel in the stream before it
 * reads anything, so consecutive calls may overlap their launch and tail.
 * Host errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
KVATTN_API int kvattn_decode(const kvattn_dims* dims, const uint16_t* q_rot, const uint16_t* cache_k,
                  const uint16_t* cache_v, const int32_t* start_pos, int32_t max_kv_len_hint,
                  float scale, uint16_t* out, void* workspace, size_t workspace_bytes,
                  int32_t* dev_status, kvattn_stream_t stream);

/* How kvattn_decode will split the work for these dims and max_kv_len_hint
 * on the CURRENT device: rows per split (C), the most splits a sequence can
 * have, the persistent grid (CTAs), the CTAs resident per SM, and whether the
 * tensor-core decode runs (1; G >= 8 always, G = 4 for calls of at least
 * 2^18 (row, KV head) pairs) or the CUDA-core one (0).  Any output pointer
 * may be NULL.  Returns a kvattn_status (host-side only, launches nothing). */
KVATTN_API int kvattn_decode_plan(const kvattn_dims* dims, int32_t max_kv_len_hint, int32_t* rows_per_split,
                                  int32_t* max_splits, int32_t* grid, int32_t* ctas_per_sm,
                                  int32_t* tensor_cores);

/* Optional attention masks of "The Modern Decoder Block" (modules L7.5 and
 * L7.7: sliding window, StreamingLLM attention sinks, learned sinks).  The
 * page names them without defining them; the readings taken are the plain
 * ones of the works it cites:
 *  - window W > 0: the token at position p sees cache rows p - W < r <= p
 *    (W = 0: every row 0..p);
 *  - n_sink (with a window): rows 0..n_sink-1 stay visible as well; positions
 *    stay absolute (RoPE is applied at the true position, rows are
 *    positions);
 *  - sink_logits: device fp32 [H] or NULL, one learned logit sigma_h per query
 *    head in the units of the scaled score: e^{sigma_h} joins the head's
 *    softmax denominator and carries no value,
 *    out = sum_r e^{s_r} V_r / (e^{sigma_h} + sum_r e^{s_r}).
 * A NULL mask pointer means none of these. */
typedef struct kvattn_attn_mask {
  int32_t window;
  int32_t n_sink;
  const float* sink_logits;
} kvattn_attn_mask;

/* kvattn_decode with a mask (mask may be NULL).  Only the visible rows are
 * read from HBM: the sink rows and the window rows (each rounded out to
 * 64-row boundaries).  Workspace: kvattn_decode_masked_workspace_bytes() for
 * the same mask (with learned sinks every sequence writes split partials and
 * the merge kernel adds the sink term, so a workspace is needed even when no
 * sequence is split).
 * Host errors: those of kvattn_decode, and INVALID_ARG for a negative window
 * or n_sink or a misaligned sink_logits. */
KVATTN_API size_t kvattn_decode_masked_workspace_bytes(const kvattn_dims* dims, int32_t max_kv_len_hint,
                                                       const kvattn_attn_mask* mask);
KVATTN_API int kvattn_decode_masked(const kvattn_dims* dims, const uint16_t* q_rot, const uint16_t* cache_k,
                                    const uint16_t* cache_v, const int32_t* start_pos, int32_t max_kv_len_hint,
                                    float scale, const kvattn_attn_mask* mask, uint16_t* out, void* workspace,
                                    size_t workspace_bytes, int32_t* dev_status, kvattn_stream_t stream);

/* kvattn_prefill_chunk with a mask (mask may be NULL): each token applies its
 * own window; key tiles outside every row's window and the sinks are not
 * read. */
KVATTN_API int kvattn_prefill_chunk_masked(const kvattn_dims* dims, int32_t T, const uint16_t* q_rot,
                                           const uint16_t* cache_k, const uint16_t* cache_v,
                                           const int32_t* start_pos, int32_t max_kv_len_hint, float scale,
                                           const kvattn_attn_mask* mask, uint16_t* out, void* workspace,
                                           size_t workspace_bytes, int32_t* dev_status, kvattn_stream_t stream);

/* Bytes of device workspace kvattn_decode_fused needs for these dims and
 * max_kv_len_hint on the CURRENT device (0: none needed, or invalid
 * arguments). */
KVATTN_API size_t kvattn_decode_fused_workspace_bytes(const kvattn_dims* dims, int32_t max_kv_len_hint);

/* Steps 1-3 of one decode step in a single kernel launch (T = 1): the
 * per-token work of "Llama 3 8B · KV cache" (rotate the new q and k at
 * p = start_pos[b], write cache row p, attend rows 0..p) and the log-sum-exp
 * merge of the split partials, with the results of kvattn_rope_append
 * followed by kvattn_decode:
 *   q_rot[b,0,h,:]   = RoPE_p(q[b,0,h,:])          (only if q_rot != NULL)
 *   cache_k[b,p,j,:] = RoPE_p(k_new[b,0,j,:]),  cache_v[b,p,j,:] = v_new[b,0,j,:]
 *   out[b,0,h,:]     = attention of RoPE_p(q[b,0,h,:]) over rows 0..p
 * q, k_new, v_new are bf16 [B,1,H,d] / [B,1,Hkv,d]; q_rot may be NULL and
 * must not be q (the kernel reads q until it ends).  Rows other than p are
 * not written.  A sequence with start_pos[b] outside the cache or above the
 * hint writes nothing (no cache row, no output) and sets its KVATTN_DEV_*
 * bit.  rope, scale and max_kv_len_hint are as in kvattn_rope_append and
 * kvattn_decode.
 * workspace: kvattn_decode_fused_workspace_bytes() bytes, 16-byte aligned,
 * owned by the caller (NULL allowed when that size is 0).  Unlike
 * kvattn_decode's, it holds counters that must be ZERO before the first call
 * (e.g. cudaMemset once after allocation); every call leaves them zero again
 * when it completes, so no memset is needed between calls.  After a call
 * that set KVATTN_DEV_WAIT_TIMEOUT, zero the workspace again.  Calls sharing
 * a workspace must be ordered on one stream.
 * Host errors: INVALID_ARG, UNSUPPORTED, OUT_OF_RANGE, WORKSPACE, CUDA. */
KVATTN_API int kvattn_decode_fused(const kvattn_dims* dims, const kvattn_rope_params* rope, const uint16_t* q,
                                   uint16_t* q_rot, const uint16_t* k_new, const uint16_t* v_new, uint16_t* cache_k,
                                   uint16_t* cache_v, const int32_t* start_pos, int32_t max_kv_len_hint, float scale,
                                   uint16_t* out, void* workspace, size_t workspace_bytes, int32_t* dev_status,
                                   kvattn_stream_t stream);

/* Size of the static device array behind kvattn_decode_noalloc: 64 MiB. */
#define KVATTN_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

/* Allocation-free variant of kvattn_decode.  The pages have no counterpart:
 * this exists for callers that cannot give the library device memory -- a
 * plugin whose host framework owns every allocation and offers no allocator,
 * an engine that has reserved nearly all of HBM for its caches and allows no
 * allocation on the decode path, or a latency-critical loop that cannot pay
 * for cudaMalloc/cudaFree.  Arguments and results are those of kvattn_decode
 * without the workspace: the split partials go to a file-scope device array of
 * KVATTN_NOALLOC_SCRATCH_BYTES that every GPU using this entry point keeps
 * until the process exits.  The entry point itself allocates nothing.
 *  - The array's device address is looked up on the first call on each
 *    device; make that first call before any stream capture.
 *  - Every call shares the one array: calls whose kernels overlap on the GPU
 *    (other streams, other host threads) race and must be serialised by the
 *    caller.  The array starts zeroed and each call leaves its work counter
 *    zero again, also a call that set KVATTN_DEV_WAIT_TIMEOUT (its merge
 *    kernel clears the counter after the split kernel ends) and a call whose
 *    merge launch failed (the entry point then queues the clear itself), so
 *    the caller never has to reset anything.
 *  - Shapes whose partials need more than the array (see
 *    kvattn_decode_workspace_bytes) return KVATTN_ERR_WORKSPACE and launch
 *    nothing. */
KVATTN_API int kvattn_decode_noalloc(const kvattn_dims* dims, const uint16_t* q_rot, const uint16_t* cache_k,
                                     const uint16_t* cache_v, const int32_t* start_pos, int32_t max_kv_len_hint,
                                     float scale, uint16_t* out, int32_t* dev_status, kvattn_stream_t stream);

/* KVATTN_NOALLOC_SCRATCH_BYTES, as built into the library. */
KVATTN_API size_t kvattn_decode_noalloc_scratch_bytes(void);

/* Bytes of device workspace kvattn_prefill_chunk needs (may be 0). */
KVATTN_API size_t kvattn_prefill_workspace_bytes(const kvattn_dims* dims, int32_t T, int32_t max_kv_len_hint);

/* Step 3 for a chunk of T new tokens per sequence (chunked prefill into an
 * existing cache).  Row t of the chunk sits at position start_pos[b]+t and
 * sees cache rows 0 .. start_pos[b]+t: the rectangular causal mask whose only
 * masked entries are (t, r) with r > start_pos + t (comment in the
 * "mask" code excerpt of "Llama 3 8B · KV cache").
 *   out[b,t,h,:] = sum_{r <= start_pos[b]+t} softmax_r(scale * q_rot[b,t,h,:] .
 *                  cache_k[b,r,floor(h/G),:]) * cache_v[b,r,floor(h/G),:]
 * q_rot and out are bf16 [B,T,H,d]; the chunk's rows must already be in the
 * cache (kvattn_rope_append with the same T).  max_kv_len_hint bounds
 * start_pos[b] + T.  Errors and workspace rules as kvattn_decode. */
KVATTN_API int kvattn_prefill_chunk(const kvattn_dims* dims, int32_t T, const uint16_t* q_rot,
                         const uint16_t* cache_k, const uint16_t* cache_v,
                         const int32_t* start_pos, int32_t max_kv_len_hint, float scale,
                         uint16_t* out, void* workspace, size_t workspace_bytes,
                         int32_t* dev_status, kvattn_stream_t stream);

/* Human-readable name of a kvattn_status value. */
KVATTN_API const char* kvattn_status_string(int status);

/* The cudaError_t value behind the most recent KVATTN_ERR_CUDA returned on
 * this host thread (0 if none yet), and its text. */
KVATTN_API int kvattn_last_cuda_error(void);
KVATTN_API const char* kvattn_last_cuda_error_string(void);

/* Library version, major*10000 + minor*100 + patch. */
KVATTN_API int kvattn_version(void);

/* Failure-path diagnostics (no counterpart on the pages).  Every in-kernel
 * pipeline wait of the library is bounded: when it does not complete within
 * the limit, the CTA sets KVATTN_DEV_WAIT_TIMEOUT in *dev_status, stops
 * waiting, lets the copies and tensor-core work it already issued finish,
 * frees its tensor memory and exits; the call's outputs are then undefined
 * (a fused decode may also leave its new cache row unwritten).  This sets,
 * for every launch made afterwards by this process:
 *  - limit_ns: the limit of each wait in nanoseconds (0: the default, one
 *    second);
 *  - gate: NULL, or a 4-byte aligned device int32 that the pipelined kernels
 *    (kvattn_decode, kvattn_decode_masked, kvattn_decode_fused,
 *    kvattn_decode_noalloc, kvattn_prefill_chunk(_masked)) wait on, within
 *    the limit, until it is non-zero, before they issue any copy.  A gate
 *    that stays zero makes every such launch give up after the limit, which
 *    is how the failure path is tested without breaking any kernel.
 * Recovery after a call that set KVATTN_DEV_WAIT_TIMEOUT: kvattn_decode,
 * kvattn_decode_masked and kvattn_decode_noalloc leave their work counter
 * zero and need nothing; zero a kvattn_decode_fused workspace again.
 * Process-wide; change it only while no other thread launches library work.
 * Returns KVATTN_OK, or INVALID_ARG for a misaligned gate. */
KVATTN_API int kvattn_set_wait_policy(uint64_t limit_ns, const int32_t* gate);

#ifdef __cplusplus
}
#endif

#endif /* KVATTN_H */

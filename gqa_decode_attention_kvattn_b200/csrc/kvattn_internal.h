// Internal launch interfaces between the C-ABI layer (kvattn_api.cu) and the
// kernels.  Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace kvattn {

// Launch `kernel` with programmatic stream serialization: it may be scheduled
// while the previous kernel in the stream is finishing, and waits for it
// (pdl_wait) before it touches any input.  Every kernel of the library starts
// that way, so any of them may follow any other.
template <class... KArgs, class... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// Maps a launch result to a kvattn_status (KVATTN_OK or KVATTN_ERR_CUDA) and
// remembers a failure for kvattn_last_cuda_error() on this host thread.
int launch_status(cudaError_t e);

constexpr int kMaxRopePairs = 64;  // d/2 for d = 128

struct RopeTable {
  double freq[kMaxRopePairs];  // f_i, already scaled when Llama-3.1 scaling is on
  int layout;                  // 0: pairs (2i, 2i+1); 1: pairs (i, i + r/2)
  int rotary_dim;              // r: elements 0..r-1 rotate, the rest are copied
};

struct RopeAppendArgs {
  int B, T, H, Hkv, S;
  const uint16_t* q;
  uint16_t* q_rot;
  const uint16_t* k_new;
  const uint16_t* v_new;
  uint16_t* cache_k;
  uint16_t* cache_v;
  const int32_t* start_pos;
  int32_t* dev_status;
};

cudaError_t launch_rope_append(const RopeAppendArgs& a, const RopeTable& tab, cudaStream_t stream);

// Split-K attention over the cache for Tq query tokens per sequence.  Each
// (sequence, token) pair is a "query row set" of G heads per KV head; its
// visible length is start_pos[b] + t + 1.
struct DecodeArgs {
  int B, Tq, H;
  int Hkv;       // KV-head groups the kernel walks: the KV heads, or for G > 16
                 // kv_div groups of 16 query heads per KV head
  int S;
  int kv_div;    // groups per KV head (1 unless G > 16)
  int Hkv_phys;  // KV heads in the caches and in k_new / v_new
  int kv_len_hint;     // upper bound on start_pos[b] + Tq
  int rows_per_split;  // C, a multiple of the tile rows
  int max_splits;      // ceil(kv_len_hint / C)
  float scale_log2;    // softmax scale * log2(e)
  const uint16_t* q;   // [B, Tq, H, d]: rotated, or (fused decode) as projected
  uint16_t* out;       // [B, Tq, H, d]
  const int32_t* start_pos;
  float* ws_o;   // [B*Tq, max_splits, H, d]   unnormalised partial outputs
  float* ws_ml;  // [B*Tq, max_splits, H, 2]   (running max in log2 units, sum)
  int* counter;  // work counter (split path); null: round-robin
  int32_t* dev_status;
  int grid;      // persistent CTAs
  // fused decode only (Tq = 1): the new token's K/V rows to rotate and append,
  // the optional rotated-q output, and the self-resetting counters
  const uint16_t* k_new;  // [B, 1, Hkv, d]
  const uint16_t* v_new;  // [B, 1, Hkv, d]
  uint16_t* cache_k;      // the same caches the tensor maps view
  uint16_t* cache_v;
  uint16_t* q_rot_out;    // [B, 1, H, d] or null
  int* exit_counter;      // CTAs that finished (counter reset by the last)
  int* merge_counter;     // [B, Hkv] splits finished per row set and KV head
  // multi-query decode on tcgen05 (Tq = 1): partial slots written per
  // (sequence, KV head) of the caches, read by the merge instead of
  // ceil(length / rows_per_split); null otherwise
  const int* unit_splits;
  // optional masks: window > 0 shows a token at position p the rows
  // p - window < r <= p and the first n_sink rows; sink_logits (fp32 [H],
  // score units, or null) adds e^{sink} to each head's softmax denominator
  int window;
  int n_sink;
  const float* sink_logits;
  int mma;       // 1: the tensor-core kernel (its 128B-swizzled 64-row cache view)
  // limit of each in-kernel wait (0: one second) and the diagnostics gate
  // (kvattn_set_wait_policy; null: none)
  uint64_t wait_ns;
  const int32_t* gate;
};

// Group view of the decode kernels: G <= 16 query heads per KV head run as
// one group; G = 32, 64, 128 run as G/16 groups of 16 heads that read the
// same KV head (neighbouring work items, so the second read of a row is
// normally served by L2).  (Unmasked multi-split G = 32 calls do not reach
// these kernels: the decode entry runs them on the tcgen05 multi-query
// kernel.)
inline void decode_group_view(int H, int Hkv, int* groups, int* kv_div) {
  const int G = H / Hkv;
  *kv_div = G > 16 ? G / 16 : 1;
  *groups = Hkv * *kv_div;
}

struct DecodePlan {
  int rows_per_split;
  int max_splits;
  int grid;
  int ctas_per_sm;
  bool mma;               // tensor-core decode (else the CUDA-core kernel)
  size_t ws_bytes;        // partials + work counter (unfused decode)
  size_t fused_ws_bytes;  // partials + the counters of the fused decode
};

// Split size, persistent grid and workspace for these shapes on this device.
// always_partials: every row set writes split partials for the merge kernel
// (learned sinks are applied there), so a workspace is needed even without
// splits.
DecodePlan plan_decode(int B, int Tq, int H, int Hkv, int kv_len_hint, int sm_count, bool always_partials = false);

// Whether a call of G heads per KV head over work_rows (row, KV head) pairs
// runs on the tensor-core decode, whose cache view is 128B-swizzled boxes of
// 64 elements x 64 rows (else plain boxes of 128 elements x 32 rows).
bool decode_use_mma(int G, long long work_rows);

// Points ws_o / ws_ml / counter (and, when `fused`, the fused decode's
// counters) of `a` into a workspace of plan.ws_bytes (plan.fused_ws_bytes).
void bind_decode_workspace(DecodeArgs& a, const DecodePlan& plan, void* workspace, bool fused = false);

// Unfused attention (fused == null: q already rotated, cache rows already
// appended) or the fused decode step (rope + append + attention + merge in
// one launch, Tq = 1) with the frequency table `fused`.
cudaError_t launch_decode(const DecodeArgs& a, const CUtensorMap& tmap_k, const CUtensorMap& tmap_v,
                          cudaStream_t stream, const RopeTable* fused = nullptr);

// Chunked prefill on tcgen05: one CTA per (128-row M tile, KV head, sequence).
struct PrefillArgs {
  int B, T, H, Hkv, S;
  int kv_len_hint;  // upper bound on start_pos[b] + T
  int n_mtiles;     // ceil(T / tokens per tile)
  float scale_log2; // softmax scale * log2(e)
  const int32_t* start_pos;
  uint16_t* out;    // [B, T, H, d]
  int32_t* dev_status;
  int window;       // > 0: token at position p sees keys p - window < k <= p and k < n_sink
  int n_sink;
  const float* sink_logits;  // fp32 [H] learned sink logits (score units), or null
  uint64_t wait_ns;     // limit of each in-kernel wait (0: one second)
  const int32_t* gate;  // diagnostics gate (null: none)
};

// Multi-query decode (32 query heads per KV head, one new token) on tcgen05,
// one CTA per SM: the key tiles of all (sequence, KV head) units, laid end to
// end, are cut into 2 * grid equal contiguous ranges, two per CTA; each piece
// of a unit that a range covers leaves one partial (unnormalised O and (max in
// log2 units, sum)) in part_o [B, part_splits, H, d] / part_ml [.., 2], the
// layout the decode's LSE merge reads, and unit_splits [B * Hkv] receives each
// unit's slot count.  A unit spans at most ceil(tiles / range) + 1 ranges, so
// ranges of at least min_tiles tiles, with
// min_tiles >= ceil(ceil(kv_len_hint / 128) / (part_splits - 1)), fit its slots.
struct MqaDecodeArgs {
  int B, H, Hkv, S;
  int kv_len_hint;  // upper bound on start_pos[b] + 1
  int part_splits;  // partial slots per unit (>= 2)
  int min_tiles;    // shortest range, in 128-row key tiles (>= 1)
  float scale_log2; // softmax scale * log2(e)
  const int32_t* start_pos;
  float* part_o;
  float* part_ml;
  int* unit_splits;
  int32_t* dev_status;
  uint64_t wait_ns;     // limit of each in-kernel wait (0: one second)
  const int32_t* gate;  // diagnostics gate (null: none)
};

cudaError_t launch_mqa_decode(const MqaDecodeArgs& a, const CUtensorMap& tmap_q, const CUtensorMap& tmap_k,
                              const CUtensorMap& tmap_v, int grid, cudaStream_t stream);

// The process's wait policy (kvattn_set_wait_policy) copied into launch
// arguments.
void apply_wait_policy(DecodeArgs& a);
void apply_wait_policy(PrefillArgs& a);
void apply_wait_policy(MqaDecodeArgs& a);
int set_wait_policy(uint64_t limit_ns, const int32_t* gate);

// Tokens per 128-row M tile for group size G (128 / G).
int prefill_tokens_per_tile(int G);

cudaError_t launch_prefill(const PrefillArgs& a, const CUtensorMap& tmap_q, const CUtensorMap& tmap_k,
                           const CUtensorMap& tmap_v, cudaStream_t stream);

// The decode's LSE merge of split partials (a.ws_o / a.ws_ml, a.rows_per_split
// rows per split, a.max_splits slots per row set) into a.out.
cudaError_t launch_decode_merge(const DecodeArgs& a, cudaStream_t stream);

}  // namespace kvattn

// C-ABI layer of libkvattn.so: host-side validation, the RoPE frequency
// table, TMA descriptors for the caches, and the launches.  Declared in
// include/kvattn.h, which states each call's contract.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "kvattn.h"
#include "kvattn_internal.h"

namespace kvattn {

namespace {
thread_local int t_last_cuda_error = 0;
}

int launch_status(cudaError_t e) {
  if (e == cudaSuccess) return KVATTN_OK;
  t_last_cuda_error = (int)e;
  return KVATTN_ERR_CUDA;
}

namespace {
// kvattn_set_wait_policy: in-kernel wait limit (0: the kernels' default of
// one second) and the diagnostics gate, read by every later launch
std::atomic<uint64_t> g_wait_ns{0};
std::atomic<const int32_t*> g_gate{nullptr};
}  // namespace

void apply_wait_policy(DecodeArgs& a) {
  a.wait_ns = g_wait_ns.load(std::memory_order_relaxed);
  a.gate = g_gate.load(std::memory_order_relaxed);
}

void apply_wait_policy(PrefillArgs& a) {
  a.wait_ns = g_wait_ns.load(std::memory_order_relaxed);
  a.gate = g_gate.load(std::memory_order_relaxed);
}

void apply_wait_policy(MqaDecodeArgs& a) {
  a.wait_ns = g_wait_ns.load(std::memory_order_relaxed);
  a.gate = g_gate.load(std::memory_order_relaxed);
}

int set_wait_policy(uint64_t limit_ns, const int32_t* gate) {
  if (reinterpret_cast<uintptr_t>(gate) & 3u) return KVATTN_ERR_INVALID_ARG;
  g_wait_ns.store(limit_ns, std::memory_order_relaxed);
  g_gate.store(gate, std::memory_order_relaxed);
  return KVATTN_OK;
}

}  // namespace kvattn

namespace {

using kvattn::kMaxRopePairs;

constexpr int kHeadDim = 128;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool group_supported(int G) {
  return G == 1 || G == 2 || G == 4 || G == 8 || G == 16 || G == 32 || G == 64 || G == 128;
}

// KV-head groups the decode kernels walk for these dims (see decode_group_view).
int decode_groups(const kvattn_dims* d, int* kv_div) {
  int groups = 0;
  kvattn::decode_group_view(d->n_heads, d->n_kv_heads, &groups, kv_div);
  return groups;
}

int check_dims(const kvattn_dims* d) {
  if (!d) return KVATTN_ERR_INVALID_ARG;
  if (d->batch < 1 || d->n_heads < 1 || d->n_kv_heads < 1 || d->max_seq_len < 1) return KVATTN_ERR_INVALID_ARG;
  if (d->n_heads % d->n_kv_heads != 0) return KVATTN_ERR_INVALID_ARG;
  if (d->head_dim != kHeadDim) return KVATTN_ERR_UNSUPPORTED;
  return KVATTN_OK;
}

// f_i = theta^(-2i/r), i < r/2 (r = rotary_dim), with the optional Llama-3.1
// scaling rule (stated in include/kvattn.h beside kvattn_rope_params).
int make_rope_table(const kvattn_rope_params* r, kvattn::RopeTable* tab) {
  if (!r || !std::isfinite(r->theta) || !(r->theta > 0.0)) return KVATTN_ERR_INVALID_ARG;
  if (r->use_scaled) {
    if (!(r->factor > 0.0) || !(r->low_freq_factor > 0.0) || !(r->high_freq_factor > r->low_freq_factor) ||
        !(r->original_max_pos > 0.0))
      return KVATTN_ERR_INVALID_ARG;
  }
  if (r->layout != KVATTN_ROPE_INTERLEAVED && r->layout != KVATTN_ROPE_HALF_SPLIT) return KVATTN_ERR_INVALID_ARG;
  const int rd = r->rotary_dim == 0 ? kHeadDim : r->rotary_dim;
  if (rd < 2 || rd > kHeadDim || (rd & 1)) return KVATTN_ERR_INVALID_ARG;
  const double two_pi = 6.283185307179586476925286766559;
  for (int i = 0; i < rd / 2; ++i) {
    double f = std::pow(r->theta, -(2.0 * i) / rd);
    if (r->use_scaled) {
      const double wavelength = two_pi / f;
      const double short_wl = r->original_max_pos / r->high_freq_factor;  // kept below this
      const double long_wl = r->original_max_pos / r->low_freq_factor;    // divided above this
      if (wavelength > long_wl) {
        f /= r->factor;
      } else if (wavelength >= short_wl) {
        const double s = (r->original_max_pos / wavelength - r->low_freq_factor) /
                         (r->high_freq_factor - r->low_freq_factor);
        f = (1.0 - s) * (f / r->factor) + s * f;
      }
    }
    tab->freq[i] = f;
  }
  for (int i = rd / 2; i < kMaxRopePairs; ++i) tab->freq[i] = 0.0;
  tab->layout = r->layout;
  tab->rotary_dim = rd;
  return KVATTN_OK;
}

// ------------------------------------------------------------ device queries
int current_sm_count(int* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KVATTN_ERR_CUDA;
  static std::mutex mu;
  static int cached[64] = {0};
  std::lock_guard<std::mutex> lock(mu);
  if (dev < 0 || dev >= 64) return KVATTN_ERR_CUDA;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      return KVATTN_ERR_CUDA;
    cached[dev] = n;
  }
  *out = cached[dev];
  return KVATTN_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Cache [B, S, Hkv, 128] bf16 viewed as a 4-D tensor (d, head, row, batch);
// one box is `rows` consecutive rows of one head of one sequence.
int encode_cache_map(CUtensorMap* map, const void* base, int B, int S, int Hkv, int rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return KVATTN_ERR_CUDA;
  const cuuint64_t dims[4] = {(cuuint64_t)kHeadDim, (cuuint64_t)Hkv, (cuuint64_t)S, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)Hkv * kHeadDim * 2,
                                 (cuuint64_t)S * Hkv * kHeadDim * 2};
  const cuuint32_t box[4] = {(cuuint32_t)kHeadDim, 1, (cuuint32_t)rows, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? KVATTN_OK : KVATTN_ERR_CUDA;
}

int hint_or_default(int32_t hint, int S) { return hint <= 0 ? S : hint; }

int check_mask(const kvattn_attn_mask* m) {
  if (!m) return KVATTN_OK;
  if (m->window < 0 || m->n_sink < 0) return KVATTN_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(m->sink_logits) & 3u) return KVATTN_ERR_INVALID_ARG;
  return KVATTN_OK;
}

// Rows a sequence can have visible: the hint, or with a window at most the
// window plus the 64-row-aligned sink segment and one tile of alignment.
int visible_len_bound(int hint, const kvattn_attn_mask* m) {
  if (!m || m->window <= 0) return hint;
  const long long bound = (long long)m->window + (((long long)m->n_sink + 63) & ~63ll) + 64;
  return bound < hint ? (int)bound : hint;
}

void apply_mask(kvattn::DecodeArgs& a, const kvattn_attn_mask* m) {
  a.window = m ? m->window : 0;
  a.n_sink = (m && m->window > 0) ? m->n_sink : 0;
  a.sink_logits = m ? m->sink_logits : nullptr;
}

// 4-D view (d, head, row, seq) of a [B, R, heads, 128] bf16 tensor with
// 128-byte swizzled boxes of 64 elements x box_heads x box_rows.
int encode_sw128_map(CUtensorMap* map, const void* base, int B, int R, int heads, int box_heads, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return KVATTN_ERR_CUDA;
  const cuuint64_t dims[4] = {(cuuint64_t)kHeadDim, (cuuint64_t)heads, (cuuint64_t)R, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)heads * kHeadDim * 2,
                                 (cuuint64_t)R * heads * kHeadDim * 2};
  const cuuint32_t box[4] = {64, (cuuint32_t)box_heads, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? KVATTN_OK : KVATTN_ERR_CUDA;
}


int run_attention(const kvattn_dims* dims, int32_t T, const uint16_t* q_rot, const uint16_t* cache_k,
                  const uint16_t* cache_v, const int32_t* start_pos, int32_t max_kv_len_hint, float scale,
                  const kvattn_attn_mask* mask, uint16_t* out, void* workspace, size_t workspace_bytes,
                  int32_t* dev_status, kvattn_stream_t stream) {
  int rc = check_dims(dims);
  if (rc != KVATTN_OK) return rc;
  rc = check_mask(mask);
  if (rc != KVATTN_OK) return rc;
  if (T < 1) return KVATTN_ERR_INVALID_ARG;
  if (!group_supported(dims->n_heads / dims->n_kv_heads)) return KVATTN_ERR_UNSUPPORTED;
  if (!q_rot || !cache_k || !cache_v || !start_pos || !out) return KVATTN_ERR_INVALID_ARG;
  if (!aligned16(q_rot) || !aligned16(cache_k) || !aligned16(cache_v) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(start_pos) & 3u))
    return KVATTN_ERR_INVALID_ARG;
  const int hint = hint_or_default(max_kv_len_hint, dims->max_seq_len);
  if (hint > dims->max_seq_len || hint < T) return KVATTN_ERR_OUT_OF_RANGE;
  if (!(scale > 0.f)) scale = 1.0f / std::sqrt((float)kHeadDim);
  if (!std::isfinite(scale)) return KVATTN_ERR_INVALID_ARG;
  // the merge kernel's grid is (row sets, groups of four heads): at most 2^24
  // row sets; heads are capped at 65535 (the grid's y extent would allow
  // four times more), checked before anything is launched
  if ((long long)dims->batch * T > (1LL << 24) || dims->n_heads > 65535) return KVATTN_ERR_UNSUPPORTED;

  int sms = 0;
  rc = current_sm_count(&sms);
  if (rc != KVATTN_OK) return rc;
  int kv_div = 1;
  const int groups = decode_groups(dims, &kv_div);
  const kvattn::DecodePlan plan = kvattn::plan_decode(dims->batch, T, dims->n_heads, groups,
                                                      visible_len_bound(hint, mask), sms,
                                                      mask && mask->sink_logits);
  if (plan.ws_bytes > 0) {
    if (!workspace || workspace_bytes < plan.ws_bytes || !aligned16(workspace)) return KVATTN_ERR_WORKSPACE;
  }

  CUtensorMap tk, tv;
  if (plan.mma) {
    rc = encode_sw128_map(&tk, cache_k, dims->batch, dims->max_seq_len, dims->n_kv_heads, 1, 64);
    if (rc != KVATTN_OK) return rc;
    rc = encode_sw128_map(&tv, cache_v, dims->batch, dims->max_seq_len, dims->n_kv_heads, 1, 64);
  } else {
    rc = encode_cache_map(&tk, cache_k, dims->batch, dims->max_seq_len, dims->n_kv_heads, 32);
    if (rc != KVATTN_OK) return rc;
    rc = encode_cache_map(&tv, cache_v, dims->batch, dims->max_seq_len, dims->n_kv_heads, 32);
  }
  if (rc != KVATTN_OK) return rc;

  kvattn::DecodeArgs a{};
  a.B = dims->batch;
  a.Tq = T;
  a.H = dims->n_heads;
  a.Hkv = groups;
  a.kv_div = kv_div;
  a.Hkv_phys = dims->n_kv_heads;
  a.S = dims->max_seq_len;
  a.kv_len_hint = hint;
  a.rows_per_split = plan.rows_per_split;
  a.max_splits = plan.max_splits;
  a.scale_log2 = scale * 1.4426950408889634f;
  apply_mask(a, mask);
  a.q = q_rot;
  a.out = out;
  a.start_pos = start_pos;
  kvattn::bind_decode_workspace(a, plan, workspace);
  a.dev_status = dev_status;
  a.grid = plan.grid;
  a.mma = plan.mma ? 1 : 0;
  kvattn::apply_wait_policy(a);

  // One new token per sequence with all 32 query heads on one KV head (G = 32,
  // multi-query): the 32 heads are 32 rows of a 128-row tcgen05 M tile (the
  // warp MMAs of the decode kernels top out near 100 TFLOP/s, a third of what
  // this shape needs at HBM speed).  The multi-query kernel cuts the call's
  // key tiles evenly over one CTA per SM, then the same LSE merge combines
  // the pieces.
  const bool masked = mask && (mask->window > 0 || mask->sink_logits);
  const long long units = (long long)dims->batch * dims->n_kv_heads;
  const long long tiles_per_unit = (hint + 127) / 128;
  if (dims->n_heads == 32 * dims->n_kv_heads && T == 1 && !masked && plan.mma && plan.max_splits > 1 &&
      plan.ws_bytes > 0 && units <= (1 << 16) && units * tiles_per_unit < (1ll << 30)) {
    CUtensorMap tq, tk2, tv2;
    // Q boxes: one token's 32 heads (32 rows of 128 bytes per 64-element half)
    rc = encode_sw128_map(&tq, q_rot, dims->batch, 1, dims->n_heads, 32, 1);
    if (rc != KVATTN_OK) return rc;
    rc = encode_sw128_map(&tk2, cache_k, dims->batch, dims->max_seq_len, dims->n_kv_heads, 1, 128);
    if (rc != KVATTN_OK) return rc;
    rc = encode_sw128_map(&tv2, cache_v, dims->batch, dims->max_seq_len, dims->n_kv_heads, 1, 128);
    if (rc != KVATTN_OK) return rc;
    kvattn::MqaDecodeArgs m{};
    m.B = dims->batch;
    m.H = dims->n_heads;
    m.Hkv = dims->n_kv_heads;
    m.S = dims->max_seq_len;
    m.kv_len_hint = hint;
    m.part_splits = plan.max_splits;
    // a unit of up to tiles_per_unit tiles spans at most
    // ceil(tiles_per_unit / range) + 1 ranges: keep that within its slots
    m.min_tiles = (int)std::max<long long>(1, (tiles_per_unit + plan.max_splits - 2) / (plan.max_splits - 1));
    m.scale_log2 = a.scale_log2;
    m.start_pos = start_pos;
    m.part_o = a.ws_o;
    m.part_ml = a.ws_ml;
    // the per-unit slot counts sit where the fused decode keeps its merge counters
    m.unit_splits = reinterpret_cast<int*>(static_cast<unsigned char*>(workspace) + 16);
    m.dev_status = dev_status;
    kvattn::apply_wait_policy(m);
    const int grid = (int)std::min<long long>(sms, (units * tiles_per_unit + 1) / 2);
    const cudaError_t e = kvattn::launch_mqa_decode(m, tq, tk2, tv2, grid, (cudaStream_t)stream);
    if (e != cudaSuccess) return kvattn::launch_status(e);
    a.unit_splits = m.unit_splits;
    return kvattn::launch_status(kvattn::launch_decode_merge(a, (cudaStream_t)stream));
  }
  return kvattn::launch_status(kvattn::launch_decode(a, tk, tv, (cudaStream_t)stream));
}


int run_prefill_tc(const kvattn_dims* dims, int32_t T, const uint16_t* q_rot, const uint16_t* cache_k,
                   const uint16_t* cache_v, const int32_t* start_pos, int32_t max_kv_len_hint, float scale,
                   const kvattn_attn_mask* mask, uint16_t* out, int32_t* dev_status, kvattn_stream_t stream) {
  int rc = check_dims(dims);
  if (rc != KVATTN_OK) return rc;
  rc = check_mask(mask);
  if (rc != KVATTN_OK) return rc;
  if (T < 1) return KVATTN_ERR_INVALID_ARG;
  const int G = dims->n_heads / dims->n_kv_heads;
  if (!group_supported(G)) return KVATTN_ERR_UNSUPPORTED;
  if (!q_rot || !cache_k || !cache_v || !start_pos || !out) return KVATTN_ERR_INVALID_ARG;
  if (!aligned16(q_rot) || !aligned16(cache_k) || !aligned16(cache_v) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(start_pos) & 3u))
    return KVATTN_ERR_INVALID_ARG;
  const int hint = hint_or_default(max_kv_len_hint, dims->max_seq_len);
  if (hint > dims->max_seq_len || hint < T) return KVATTN_ERR_OUT_OF_RANGE;
  if (!(scale > 0.f)) scale = 1.0f / std::sqrt((float)kHeadDim);
  if (!std::isfinite(scale)) return KVATTN_ERR_INVALID_ARG;
  const int tt = kvattn::prefill_tokens_per_tile(G);
  const long long n_mtiles = ((long long)T + tt - 1) / tt;
  if (n_mtiles * dims->n_kv_heads * dims->batch > 0x7FFFFFFFll) return KVATTN_ERR_UNSUPPORTED;

  CUtensorMap tq, tk, tv;
  rc = encode_sw128_map(&tq, q_rot, dims->batch, T, dims->n_heads, G, tt);
  if (rc != KVATTN_OK) return rc;
  rc = encode_sw128_map(&tk, cache_k, dims->batch, dims->max_seq_len, dims->n_kv_heads, 1, 128);
  if (rc != KVATTN_OK) return rc;
  rc = encode_sw128_map(&tv, cache_v, dims->batch, dims->max_seq_len, dims->n_kv_heads, 1, 128);
  if (rc != KVATTN_OK) return rc;

  kvattn::PrefillArgs a{};
  a.B = dims->batch;
  a.T = T;
  a.H = dims->n_heads;
  a.Hkv = dims->n_kv_heads;
  a.S = dims->max_seq_len;
  a.kv_len_hint = hint;
  a.n_mtiles = (int)n_mtiles;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.start_pos = start_pos;
  a.out = out;
  a.dev_status = dev_status;
  a.window = mask ? mask->window : 0;
  a.n_sink = (mask && mask->window > 0) ? mask->n_sink : 0;
  a.sink_logits = mask ? mask->sink_logits : nullptr;
  kvattn::apply_wait_policy(a);
  return kvattn::launch_status(kvattn::launch_prefill(a, tq, tk, tv, (cudaStream_t)stream));
}

}  // namespace

extern "C" {

int kvattn_rope_append(const kvattn_dims* dims, const kvattn_rope_params* rope, int32_t T, const uint16_t* q,
                       uint16_t* q_rot, const uint16_t* k_new, const uint16_t* v_new, uint16_t* cache_k,
                       uint16_t* cache_v, const int32_t* start_pos, int32_t* dev_status, kvattn_stream_t stream) {
  int rc = check_dims(dims);
  if (rc != KVATTN_OK) return rc;
  if (T < 1) return KVATTN_ERR_INVALID_ARG;
  if (!q || !q_rot || !k_new || !v_new || !cache_k || !cache_v || !start_pos) return KVATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(q_rot) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(cache_k) ||
      !aligned16(cache_v) || (reinterpret_cast<uintptr_t>(start_pos) & 3u))
    return KVATTN_ERR_INVALID_ARG;
  if (T > dims->max_seq_len) return KVATTN_ERR_OUT_OF_RANGE;
  kvattn::RopeTable tab;
  rc = make_rope_table(rope, &tab);
  if (rc != KVATTN_OK) return rc;
  kvattn::RopeAppendArgs a{};
  a.B = dims->batch;
  a.T = T;
  a.H = dims->n_heads;
  a.Hkv = dims->n_kv_heads;
  a.S = dims->max_seq_len;
  a.q = q;
  a.q_rot = q_rot;
  a.k_new = k_new;
  a.v_new = v_new;
  a.cache_k = cache_k;
  a.cache_v = cache_v;
  a.start_pos = start_pos;
  a.dev_status = dev_status;
  return kvattn::launch_status(kvattn::launch_rope_append(a, tab, (cudaStream_t)stream));
}

size_t kvattn_decode_workspace_bytes(const kvattn_dims* dims, int32_t max_kv_len_hint) {
  if (check_dims(dims) != KVATTN_OK) return 0;
  const int hint = hint_or_default(max_kv_len_hint, dims->max_seq_len);
  if (hint > dims->max_seq_len || hint < 1) return 0;
  int sms = 0;
  if (current_sm_count(&sms) != KVATTN_OK) return 0;
  int kv_div = 1;
  return kvattn::plan_decode(dims->batch, 1, dims->n_heads, decode_groups(dims, &kv_div), hint, sms).ws_bytes;
}

int kvattn_decode(const kvattn_dims* dims, const uint16_t* q_rot, const uint16_t* cache_k, const uint16_t* cache_v,
                  const int32_t* start_pos, int32_t max_kv_len_hint, float scale, uint16_t* out, void* workspace,
                  size_t workspace_bytes, int32_t* dev_status, kvattn_stream_t stream) {
  return run_attention(dims, 1, q_rot, cache_k, cache_v, start_pos, max_kv_len_hint, scale, nullptr, out, workspace,
                       workspace_bytes, dev_status, stream);
}

size_t kvattn_decode_fused_workspace_bytes(const kvattn_dims* dims, int32_t max_kv_len_hint) {
  if (check_dims(dims) != KVATTN_OK) return 0;
  const int hint = hint_or_default(max_kv_len_hint, dims->max_seq_len);
  if (hint > dims->max_seq_len || hint < 1) return 0;
  int sms = 0;
  if (current_sm_count(&sms) != KVATTN_OK) return 0;
  int kv_div = 1;
  return kvattn::plan_decode(dims->batch, 1, dims->n_heads, decode_groups(dims, &kv_div), hint, sms)
      .fused_ws_bytes;
}

int kvattn_decode_fused(const kvattn_dims* dims, const kvattn_rope_params* rope, const uint16_t* q,
                        uint16_t* q_rot, const uint16_t* k_new, const uint16_t* v_new, uint16_t* cache_k,
                        uint16_t* cache_v, const int32_t* start_pos, int32_t max_kv_len_hint, float scale,
                        uint16_t* out, void* workspace, size_t workspace_bytes, int32_t* dev_status,
                        kvattn_stream_t stream) {
  int rc = check_dims(dims);
  if (rc != KVATTN_OK) return rc;
  if (!group_supported(dims->n_heads / dims->n_kv_heads)) return KVATTN_ERR_UNSUPPORTED;
  if (!q || !k_new || !v_new || !cache_k || !cache_v || !start_pos || !out) return KVATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(cache_k) || !aligned16(cache_v) ||
      !aligned16(out) || (q_rot && !aligned16(q_rot)) || (reinterpret_cast<uintptr_t>(start_pos) & 3u))
    return KVATTN_ERR_INVALID_ARG;
  if (q_rot == q) return KVATTN_ERR_INVALID_ARG;  // other items of a sequence still read q
  kvattn::RopeTable tab;
  rc = make_rope_table(rope, &tab);
  if (rc != KVATTN_OK) return rc;
  const int hint = hint_or_default(max_kv_len_hint, dims->max_seq_len);
  if (hint > dims->max_seq_len || hint < 1) return KVATTN_ERR_OUT_OF_RANGE;
  if (!(scale > 0.f)) scale = 1.0f / std::sqrt((float)kHeadDim);
  if (!std::isfinite(scale)) return KVATTN_ERR_INVALID_ARG;
  if ((long long)dims->batch > (1LL << 24) || dims->n_heads > 65535) return KVATTN_ERR_UNSUPPORTED;

  int sms = 0;
  rc = current_sm_count(&sms);
  if (rc != KVATTN_OK) return rc;
  int kv_div = 1;
  const int groups = decode_groups(dims, &kv_div);
  const kvattn::DecodePlan plan = kvattn::plan_decode(dims->batch, 1, dims->n_heads, groups, hint, sms);
  if (plan.fused_ws_bytes > 0) {
    if (!workspace || workspace_bytes < plan.fused_ws_bytes || !aligned16(workspace)) return KVATTN_ERR_WORKSPACE;
  }
  CUtensorMap tk, tv;
  if (plan.mma) {
    rc = encode_sw128_map(&tk, cache_k, dims->batch, dims->max_seq_len, dims->n_kv_heads, 1, 64);
    if (rc != KVATTN_OK) return rc;
    rc = encode_sw128_map(&tv, cache_v, dims->batch, dims->max_seq_len, dims->n_kv_heads, 1, 64);
  } else {
    rc = encode_cache_map(&tk, cache_k, dims->batch, dims->max_seq_len, dims->n_kv_heads, 32);
    if (rc != KVATTN_OK) return rc;
    rc = encode_cache_map(&tv, cache_v, dims->batch, dims->max_seq_len, dims->n_kv_heads, 32);
  }
  if (rc != KVATTN_OK) return rc;

  kvattn::DecodeArgs a{};
  a.B = dims->batch;
  a.Tq = 1;
  a.H = dims->n_heads;
  a.Hkv = groups;
  a.kv_div = kv_div;
  a.Hkv_phys = dims->n_kv_heads;
  a.S = dims->max_seq_len;
  a.kv_len_hint = hint;
  a.rows_per_split = plan.rows_per_split;
  a.max_splits = plan.max_splits;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.q = q;
  a.out = out;
  a.start_pos = start_pos;
  kvattn::bind_decode_workspace(a, plan, workspace, true);
  a.dev_status = dev_status;
  a.grid = plan.grid;
  a.mma = plan.mma ? 1 : 0;
  a.k_new = k_new;
  a.v_new = v_new;
  a.cache_k = cache_k;
  a.cache_v = cache_v;
  a.q_rot_out = q_rot;
  kvattn::apply_wait_policy(a);
  return kvattn::launch_status(kvattn::launch_decode(a, tk, tv, (cudaStream_t)stream, &tab));
}

size_t kvattn_prefill_workspace_bytes(const kvattn_dims* dims, int32_t T, int32_t max_kv_len_hint) {
  (void)dims;
  (void)T;
  (void)max_kv_len_hint;
  return 0;  // the tensor-core prefill keeps its partial state in TMEM
}

int kvattn_prefill_chunk(const kvattn_dims* dims, int32_t T, const uint16_t* q_rot, const uint16_t* cache_k,
                         const uint16_t* cache_v, const int32_t* start_pos, int32_t max_kv_len_hint, float scale,
                         uint16_t* out, void* workspace, size_t workspace_bytes, int32_t* dev_status,
                         kvattn_stream_t stream) {
  (void)workspace;
  (void)workspace_bytes;
  return run_prefill_tc(dims, T, q_rot, cache_k, cache_v, start_pos, max_kv_len_hint, scale, nullptr, out, dev_status,
                        stream);
}

size_t kvattn_decode_masked_workspace_bytes(const kvattn_dims* dims, int32_t max_kv_len_hint,
                                            const kvattn_attn_mask* mask) {
  if (check_dims(dims) != KVATTN_OK || check_mask(mask) != KVATTN_OK) return 0;
  const int hint = hint_or_default(max_kv_len_hint, dims->max_seq_len);
  if (hint > dims->max_seq_len || hint < 1) return 0;
  int sms = 0;
  if (current_sm_count(&sms) != KVATTN_OK) return 0;
  int kv_div = 1;
  return kvattn::plan_decode(dims->batch, 1, dims->n_heads, decode_groups(dims, &kv_div),
                             visible_len_bound(hint, mask), sms, mask && mask->sink_logits)
      .ws_bytes;
}

int kvattn_decode_masked(const kvattn_dims* dims, const uint16_t* q_rot, const uint16_t* cache_k,
                         const uint16_t* cache_v, const int32_t* start_pos, int32_t max_kv_len_hint, float scale,
                         const kvattn_attn_mask* mask, uint16_t* out, void* workspace, size_t workspace_bytes,
                         int32_t* dev_status, kvattn_stream_t stream) {
  return run_attention(dims, 1, q_rot, cache_k, cache_v, start_pos, max_kv_len_hint, scale, mask, out, workspace,
                       workspace_bytes, dev_status, stream);
}

int kvattn_prefill_chunk_masked(const kvattn_dims* dims, int32_t T, const uint16_t* q_rot, const uint16_t* cache_k,
                                const uint16_t* cache_v, const int32_t* start_pos, int32_t max_kv_len_hint,
                                float scale, const kvattn_attn_mask* mask, uint16_t* out, void* workspace,
                                size_t workspace_bytes, int32_t* dev_status, kvattn_stream_t stream) {
  (void)workspace;
  (void)workspace_bytes;
  return run_prefill_tc(dims, T, q_rot, cache_k, cache_v, start_pos, max_kv_len_hint, scale, mask, out, dev_status,
                        stream);
}

int kvattn_decode_plan(const kvattn_dims* dims, int32_t max_kv_len_hint, int32_t* rows_per_split,
                       int32_t* max_splits, int32_t* grid, int32_t* ctas_per_sm, int32_t* tensor_cores) {
  int rc = check_dims(dims);
  if (rc != KVATTN_OK) return rc;
  if (!group_supported(dims->n_heads / dims->n_kv_heads)) return KVATTN_ERR_UNSUPPORTED;
  const int hint = hint_or_default(max_kv_len_hint, dims->max_seq_len);
  if (hint > dims->max_seq_len || hint < 1) return KVATTN_ERR_OUT_OF_RANGE;
  int sms = 0;
  rc = current_sm_count(&sms);
  if (rc != KVATTN_OK) return rc;
  int kv_div = 1;
  const kvattn::DecodePlan p = kvattn::plan_decode(dims->batch, 1, dims->n_heads, decode_groups(dims, &kv_div), hint, sms);
  if (rows_per_split) *rows_per_split = p.rows_per_split;
  if (max_splits) *max_splits = p.max_splits;
  if (grid) *grid = p.grid;
  if (ctas_per_sm) *ctas_per_sm = p.ctas_per_sm;
  if (tensor_cores) *tensor_cores = p.mma ? 1 : 0;
  return KVATTN_OK;
}

const char* kvattn_status_string(int status) {
  switch (status) {
    case KVATTN_OK: return "ok";
    case KVATTN_ERR_INVALID_ARG: return "invalid argument";
    case KVATTN_ERR_UNSUPPORTED: return "unsupported shape";
    case KVATTN_ERR_OUT_OF_RANGE: return "length outside the cache";
    case KVATTN_ERR_WORKSPACE: return "workspace missing or too small";
    case KVATTN_ERR_CUDA: return "CUDA error";
    default: return "unknown status";
  }
}

int kvattn_last_cuda_error(void) { return kvattn::t_last_cuda_error; }

const char* kvattn_last_cuda_error_string(void) {
  return kvattn::t_last_cuda_error ? cudaGetErrorString((cudaError_t)kvattn::t_last_cuda_error) : "no error";
}

int kvattn_version(void) { return 100; }

int kvattn_set_wait_policy(uint64_t limit_ns, const int32_t* gate) { return kvattn::set_wait_policy(limit_ns, gate); }

}  // extern "C"

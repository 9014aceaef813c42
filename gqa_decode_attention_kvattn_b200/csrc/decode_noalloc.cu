// kvattn_decode_noalloc: the split-K decode of kvattn_decode for callers
// that cannot hand the library a workspace.
//
// Some callers have no way to obtain device memory for the split partials:
// a plugin inside a host framework that owns every allocation and exposes no
// allocator, a serving engine that reserves nearly all of HBM for its KV
// caches up front and forbids allocations on the decode path, or a latency-
// critical loop where cudaMalloc / cudaFree would stall the device.  For them
// the partials live in one statically sized device array owned by this file;
// the caller passes only the inputs and the output.
//
// The array is a file-scope __device__ variable, so every GPU on which this
// code is loaded holds kScratchBytes of it until the process exits.  Host code
// cannot use the variable's name as a device address; the address is looked
// up with cudaGetSymbolAddress once per device, with that device current, the
// first time the entry point runs on it (so that first call should come
// before any stream capture).  All calls share the array: two calls whose
// kernels overlap on the GPU (different streams, or different host threads on
// one device) race on it.
//
// What the array keeps between calls.  Its first 16 bytes are the split
// kernel's work counter, which must be zero when a call starts: the array
// starts zeroed, and every call whose kernels were launched leaves the
// counter zero again (the merge kernel clears it after the split kernel has
// finished, also when a pipeline wait in that kernel gave up).  If the merge
// launch fails after the split kernel was launched, the entry point queues a
// clear of those 16 bytes itself, because the caller has no way to reach
// them.  The partials after the header are written before they are read, so
// leftovers there do no harm.
#include <cmath>
#include <cstdint>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "kvattn.h"
#include "kvattn_internal.h"

namespace {

constexpr size_t kScratchBytes = KVATTN_NOALLOC_SCRATCH_BYTES;
constexpr int kHeadDim = 128;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) float g_split_scratch[kScratchBytes / sizeof(float)];

// Device address of g_split_scratch on the current device (looked up once).
int scratch_address(void** out) {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KVATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_split_scratch) != cudaSuccess || !p) return KVATTN_ERR_CUDA;
    addr[dev] = p;
  }
  *out = addr[dev];
  return KVATTN_OK;
}

int sm_count(int* out) {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KVATTN_ERR_CUDA;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return KVATTN_ERR_CUDA;
  *out = n;
  return KVATTN_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Same cache view as kvattn_decode uses: (d, head, row, batch), boxes of 32
// rows x 128 elements of one head, or 128B-swizzled boxes of 64 rows x 64
// elements for the tensor-core decode (G >= 8).
int cache_map(CUtensorMap* map, const void* base, int B, int S, int Hkv, bool swizzled) {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  if (!fn) return KVATTN_ERR_CUDA;
  const cuuint64_t dims[4] = {(cuuint64_t)kHeadDim, (cuuint64_t)Hkv, (cuuint64_t)S, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)Hkv * kHeadDim * 2,
                                 (cuuint64_t)S * Hkv * kHeadDim * 2};
  const cuuint32_t box[4] = {swizzled ? 64u : (cuuint32_t)kHeadDim, 1, swizzled ? 64u : 32u, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzled ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS
             ? KVATTN_OK
             : KVATTN_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" KVATTN_API size_t kvattn_decode_noalloc_scratch_bytes(void) { return kScratchBytes; }

extern "C" KVATTN_API int kvattn_decode_noalloc(const kvattn_dims* dims, const uint16_t* q_rot,
                                                const uint16_t* cache_k, const uint16_t* cache_v,
                                                const int32_t* start_pos, int32_t max_kv_len_hint, float scale,
                                                uint16_t* out, int32_t* dev_status, kvattn_stream_t stream) {
  if (!dims) return KVATTN_ERR_INVALID_ARG;
  if (dims->batch < 1 || dims->n_heads < 1 || dims->n_kv_heads < 1 || dims->max_seq_len < 1 ||
      dims->n_heads % dims->n_kv_heads != 0)
    return KVATTN_ERR_INVALID_ARG;
  if (dims->head_dim != kHeadDim) return KVATTN_ERR_UNSUPPORTED;
  const int G = dims->n_heads / dims->n_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16 && G != 32 && G != 64 && G != 128)
    return KVATTN_ERR_UNSUPPORTED;
  if (!q_rot || !cache_k || !cache_v || !start_pos || !out) return KVATTN_ERR_INVALID_ARG;
  if (!aligned16(q_rot) || !aligned16(cache_k) || !aligned16(cache_v) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(start_pos) & 3u))
    return KVATTN_ERR_INVALID_ARG;
  // the merge kernel's grid is (sequences, groups of four heads); the same
  // limits as kvattn_decode
  if (dims->batch > (1 << 24) || dims->n_heads > 65535) return KVATTN_ERR_UNSUPPORTED;
  const int hint = max_kv_len_hint <= 0 ? dims->max_seq_len : max_kv_len_hint;
  if (hint > dims->max_seq_len || hint < 1) return KVATTN_ERR_OUT_OF_RANGE;
  if (!(scale > 0.f)) scale = 1.0f / std::sqrt((float)kHeadDim);
  if (!std::isfinite(scale)) return KVATTN_ERR_INVALID_ARG;

  int sms = 0;
  int rc = sm_count(&sms);
  if (rc != KVATTN_OK) return rc;
  int groups = 0, kv_div = 1;
  kvattn::decode_group_view(dims->n_heads, dims->n_kv_heads, &groups, &kv_div);
  const kvattn::DecodePlan plan = kvattn::plan_decode(dims->batch, 1, dims->n_heads, groups, hint, sms);
  if (plan.ws_bytes > kScratchBytes) return KVATTN_ERR_WORKSPACE;  // needs more than the static array

  void* scratch = nullptr;
  if (plan.ws_bytes > 0) {
    rc = scratch_address(&scratch);
    if (rc != KVATTN_OK) return rc;
  }
  CUtensorMap tk, tv;
  const bool swizzled = plan.mma;
  rc = cache_map(&tk, cache_k, dims->batch, dims->max_seq_len, dims->n_kv_heads, swizzled);
  if (rc != KVATTN_OK) return rc;
  rc = cache_map(&tv, cache_v, dims->batch, dims->max_seq_len, dims->n_kv_heads, swizzled);
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
  a.q = q_rot;
  a.out = out;
  a.start_pos = start_pos;
  kvattn::bind_decode_workspace(a, plan, scratch);
  a.dev_status = dev_status;
  a.grid = plan.grid;
  a.mma = plan.mma ? 1 : 0;
  kvattn::apply_wait_policy(a);
  const cudaError_t e = kvattn::launch_decode(a, tk, tv, (cudaStream_t)stream);
  if (e != cudaSuccess && a.counter) {
    // the split kernel may have run without the merge that clears its
    // counter: clear it here (best effort; no allocation)
    (void)cudaMemsetAsync(a.counter, 0, 16, (cudaStream_t)stream);
  }
  return kvattn::launch_status(e);
}

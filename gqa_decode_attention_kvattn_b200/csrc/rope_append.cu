// K1: RoPE with a position offset, then the KV-cache append.
//
// For token t of sequence b the position is p = start_pos[b] + t (the past
// length is the offset: "Llama 3.1 8B KV cache", section "RoPE has to know
// where it is").  Each interleaved pair (x_2i, x_2i+1) of every query head and
// every new key head is rotated by p * f_i; the rotated keys and the values go
// to cache row p ("Llama 3 8B · KV cache", cache write C_K[p] <- K_r,
// C_V[p] <- V).  Angles, sin/cos and the rotation run in fp64, which keeps the
// bf16 result within one rounding of the exact value up to p = 131071 (an fp32
// angle would already be off by ~1e-2 rad there).
//
// One CTA per (b, t); its threads first build the 64 (cos, sin) pairs of that
// position, then sweep the (H + Hkv) * 64 pairs with coalesced 4-byte
// accesses, and copy the Hkv value rows with 16-byte accesses.  The kernel
// moves B*T*(2H + 3Hkv)*256 bytes, a negligible share of a decode step.
#include "kvattn_device.cuh"
#include "kvattn_internal.h"
#include "rope_device.cuh"

namespace kvattn {
namespace {

constexpr int kRopeThreads = 256;

__global__ void __launch_bounds__(kRopeThreads) rope_append_kernel(RopeAppendArgs a, RopeTable tab) {
  const int bt = blockIdx.x;
  const int b = bt / a.T;
  const int t = bt - b * a.T;
  const int sp = a.start_pos[b];
  if (sp < 0 || (long long)sp + a.T > a.S) {
    if (t == 0 && threadIdx.x == 0) set_status(a.dev_status, KVATTN_DEV_START_POS_RANGE);
    return;
  }
  const long long pos = (long long)sp + t;

  __shared__ double s_cos[kMaxRopePairs];
  __shared__ double s_sin[kMaxRopePairs];
  const int rp = tab.rotary_dim / 2;  // rotated pairs
  for (int i = threadIdx.x; i < rp; i += blockDim.x) {
    double s, c;
    rope_cos_sin(tab, i, pos, c, s);
    s_cos[i] = c;
    s_sin[i] = s;
  }
  __syncthreads();

  constexpr int kPairs = kHeadDim / 2;
  const int q_pairs = a.H * kPairs;
  const int total = (a.H + a.Hkv) * kPairs;
  const uint32_t* q_in = reinterpret_cast<const uint32_t*>(a.q) + (size_t)bt * q_pairs;
  uint32_t* q_out = reinterpret_cast<uint32_t*>(a.q_rot) + (size_t)bt * q_pairs;
  const uint32_t* k_in = reinterpret_cast<const uint32_t*>(a.k_new) + (size_t)bt * a.Hkv * kPairs;
  uint32_t* k_out = reinterpret_cast<uint32_t*>(a.cache_k) + ((size_t)b * a.S + pos) * a.Hkv * kPairs;

  if (tab.layout == 0 && rp == kPairs) {
    // Meta layout over the whole head: each pair is one 32-bit word
    for (int idx = threadIdx.x; idx < total; idx += blockDim.x) {
      const int i = idx & (kPairs - 1);
      const bool is_q = idx < q_pairs;
      const uint32_t w = is_q ? q_in[idx] : k_in[idx - q_pairs];
      uint16_t y0, y1;
      rope_rotate_bits(true, s_cos[i], s_sin[i], (uint16_t)(w & 0xFFFFu), (uint16_t)(w >> 16), y0, y1);
      const uint32_t r = (uint32_t)y0 | ((uint32_t)y1 << 16);
      if (is_q)
        q_out[idx] = r;
      else
        k_out[idx - q_pairs] = r;
    }
  } else {
    // any layout / rotary width, one slot (pair or pass-through pair) at a time
    for (int idx = threadIdx.x; idx < total; idx += blockDim.x) {
      const int vec = idx >> 6;
      const int j = idx & (kPairs - 1);
      const bool is_q = vec < a.H;
      const uint16_t* in = is_q ? reinterpret_cast<const uint16_t*>(q_in) + (size_t)vec * kHeadDim
                                : reinterpret_cast<const uint16_t*>(k_in) + (size_t)(vec - a.H) * kHeadDim;
      uint16_t* outp = is_q ? reinterpret_cast<uint16_t*>(q_out) + (size_t)vec * kHeadDim
                            : reinterpret_cast<uint16_t*>(k_out) + (size_t)(vec - a.H) * kHeadDim;
      const RopeSlot sl = rope_slot(tab, j);
      uint16_t ya, yb;
      rope_rotate_bits(sl.rotate, sl.rotate ? s_cos[j] : 1.0, sl.rotate ? s_sin[j] : 0.0, in[sl.ea], in[sl.eb], ya,
                       yb);
      outp[sl.ea] = ya;
      outp[sl.eb] = yb;
    }
  }

  // values: bit copy of Hkv rows of 256 bytes
  const uint4* v_in = reinterpret_cast<const uint4*>(a.v_new) + (size_t)bt * a.Hkv * (kHeadDim / 8);
  uint4* v_out = reinterpret_cast<uint4*>(a.cache_v) + ((size_t)b * a.S + pos) * a.Hkv * (kHeadDim / 8);
  for (int idx = threadIdx.x; idx < a.Hkv * (kHeadDim / 8); idx += blockDim.x) v_out[idx] = v_in[idx];
}

}  // namespace

cudaError_t launch_rope_append(const RopeAppendArgs& a, const RopeTable& tab, cudaStream_t stream) {
  // every tensor argument must have been set (callers value-initialise the args)
  if (!a.q || !a.q_rot || !a.k_new || !a.v_new || !a.cache_k || !a.cache_v || !a.start_pos)
    return cudaErrorInvalidValue;
  const long long blocks = (long long)a.B * a.T;
  if (blocks > 0x7FFFFFFFll) return cudaErrorInvalidValue;
  rope_append_kernel<<<(unsigned)blocks, kRopeThreads, 0, stream>>>(a, tab);
  return cudaGetLastError();
}

}  // namespace kvattn

// K1: RoPE with a position offset, then the KV-cache append.
//
// For token t of sequence b the position is p = start_pos[b] + t (the past
// length is the offset: "Llama 3.1 8B KV cache", section "RoPE has to know
// where it is").  Each rotated pair of every query head and every new key
// head is turned by p * f_i; the rotated keys and the values go to cache row
// p ("Llama 3 8B · KV cache", cache write C_K[p] <- K_r, C_V[p] <- V).
// Angles, sin/cos and the rotation run in fp64, which keeps the bf16 result
// within one rounding of the exact value up to p = 131071 (an fp32 angle
// would already be off by ~1e-2 rad there).
//
// Work split: the H query heads and Hkv key heads of a token are H + Hkv
// head vectors; for a few tokens one CTA of 128 threads takes 8 of them for
// one (b, t), so a small decode batch still spreads over the SMs, and for
// many tokens a CTA takes a whole token.  The CTA builds the (cos,
// sin) pairs of its position in shared memory, rotates its vectors' 64 slots
// (coalesced 16-byte accesses of four pairs in the interleaved full-width
// layout, 2-byte accesses in the others), and a CTA
// holding key vectors also copies those heads' value rows (16-byte
// accesses).  The kernel moves B*T*(2H + 3Hkv)*256 bytes, a negligible share
// of a decode step.
#include "kvattn_device.cuh"
#include "kvattn_internal.h"
#include "rope_device.cuh"

namespace kvattn {
namespace {

constexpr int kRopeThreads = 128;

// vec_per_cta: head vectors (query or key heads) per CTA
__global__ void __launch_bounds__(kRopeThreads) rope_append_kernel(RopeAppendArgs a, RopeTable tab,
                                                                   int vec_per_cta) {
  pdl_wait();  // the previous kernel in the stream has finished
  pdl_launch_dependents();
  const int n_vec = a.H + a.Hkv;
  const int n_blk = (n_vec + vec_per_cta - 1) / vec_per_cta;
  const int bt = blockIdx.x / n_blk;
  const int blk = blockIdx.x - bt * n_blk;
  const int b = bt / a.T;
  const int t = bt - b * a.T;
  const int sp = a.start_pos[b];
  if (sp < 0 || (long long)sp + a.T > a.S) {
    if (t == 0 && blk == 0 && threadIdx.x == 0) set_status(a.dev_status, KVATTN_DEV_START_POS_RANGE);
    return;
  }
  const long long pos = (long long)sp + t;

  constexpr int kPairs = kHeadDim / 2;
  const int v0 = blk * vec_per_cta;
  const int nv = min(vec_per_cta, n_vec - v0);
  // vector v < H is query head v, else key head v - H
  auto vec_in = [&](int v) -> const uint16_t* {
    return v < a.H ? a.q + ((size_t)bt * a.H + v) * kHeadDim
                   : a.k_new + ((size_t)bt * a.Hkv + (v - a.H)) * kHeadDim;
  };
  auto vec_out = [&](int v) -> uint16_t* {
    return v < a.H ? a.q_rot + ((size_t)bt * a.H + v) * kHeadDim
                   : a.cache_k + (((size_t)b * a.S + pos) * a.Hkv + (v - a.H)) * kHeadDim;
  };
  const int rp = tab.rotary_dim / 2;  // rotated pairs
  const bool full_meta = tab.layout == 0 && rp == kPairs;

  // Each thread loads a batch of its chunks before it stores any: q_rot may be
  // q itself, so the compiler cannot move a load above an earlier store, and
  // one chunk at a time would pay a full memory latency per chunk.  Every
  // chunk is read and written by the same thread, so rotating in place is
  // safe.  The first batch (the whole of a decode token's share) is loaded
  // before the (cos, sin) table is built, so its latency overlaps the fp64
  // sincos.  In the interleaved full-width layout a 16-byte chunk holds four
  // whole pairs (a head vector is 16 chunks), so the addressing and the memory
  // instructions are paid once per four pairs.  Five chunks per thread cover
  // a whole token of 32 query and 8 key heads (640 chunks) in the first batch
  // (2048-token prefill rope: 19.0 us with four, 17.4 with five).
  constexpr int kBatch = 5;
  constexpr int kChunks = kHeadDim / 8;  // 16-byte chunks per head vector
  const int n_slots = nv * kPairs;
  const int n_chunks = nv * kChunks;
  auto load_batch = [&](int base_idx, uint4 (&w)[kBatch]) {
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int idx = base_idx + u * blockDim.x;
      w[u] = idx < n_chunks ? reinterpret_cast<const uint4*>(vec_in(v0 + idx / kChunks))[idx & (kChunks - 1)]
                            : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  uint4 w_first[kBatch];
  if (full_meta) load_batch(threadIdx.x, w_first);
  // values: bit copy of the 256-byte rows of this CTA's key heads, the first
  // batch of 16-byte chunks also in flight before the table
  const int k0 = max(v0, a.H) - a.H;       // first key head of this CTA
  const int k1 = max(v0 + nv, a.H) - a.H;  // one past the last
  const uint4* v_in = reinterpret_cast<const uint4*>(a.v_new) + (size_t)bt * a.Hkv * (kHeadDim / 8);
  uint4* v_out = reinterpret_cast<uint4*>(a.cache_v) + ((size_t)b * a.S + pos) * a.Hkv * (kHeadDim / 8);
  const int c_begin = k0 * (kHeadDim / 8) + threadIdx.x;
  const int c_end = k1 * (kHeadDim / 8);
  uint4 t_first[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int idx = c_begin + u * blockDim.x;
    if (idx < c_end) t_first[u] = v_in[idx];
  }

  __shared__ double s_cos[kMaxRopePairs];
  __shared__ double s_sin[kMaxRopePairs];
  for (int i = threadIdx.x; i < rp; i += blockDim.x) {
    double s, c;
    rope_cos_sin(tab, i, pos, c, s);
    s_cos[i] = c;
    s_sin[i] = s;
  }
  __syncthreads();

  if (full_meta) {
    // Meta layout over the whole head: each pair is one 32-bit word, four
    // pairs 4c .. 4c+3 per 16-byte chunk c of the head vector
    for (int base_idx = threadIdx.x; base_idx < n_chunks; base_idx += blockDim.x * kBatch) {
      uint4 w[kBatch];
      if (base_idx == (int)threadIdx.x) {
#pragma unroll
        for (int u = 0; u < kBatch; ++u) w[u] = w_first[u];
      } else {
        load_batch(base_idx, w);
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int idx = base_idx + u * blockDim.x;
        if (idx < n_chunks) {
          const int c = idx & (kChunks - 1);
          const uint32_t in[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
          uint32_t o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = 4 * c + e;
            uint16_t y0, y1;
            rope_rotate_bits(true, s_cos[i], s_sin[i], (uint16_t)(in[e] & 0xFFFFu), (uint16_t)(in[e] >> 16), y0, y1);
            o[e] = (uint32_t)y0 | ((uint32_t)y1 << 16);
          }
          reinterpret_cast<uint4*>(vec_out(v0 + idx / kChunks))[c] = make_uint4(o[0], o[1], o[2], o[3]);
        }
      }
    }
  } else {
    // any layout / rotary width, one slot (pair or pass-through pair) at a time
    for (int base_idx = threadIdx.x; base_idx < n_slots; base_idx += blockDim.x * kBatch) {
      uint16_t xa[kBatch], xb[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int idx = base_idx + u * blockDim.x;
        xa[u] = xb[u] = 0;
        if (idx < n_slots) {
          const uint16_t* in = vec_in(v0 + idx / kPairs);
          const RopeSlot sl = rope_slot(tab, idx & (kPairs - 1));
          xa[u] = in[sl.ea];
          xb[u] = in[sl.eb];
        }
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int idx = base_idx + u * blockDim.x;
        if (idx < n_slots) {
          const int j = idx & (kPairs - 1);
          uint16_t* outp = vec_out(v0 + idx / kPairs);
          const RopeSlot sl = rope_slot(tab, j);
          uint16_t ya, yb;
          rope_rotate_bits(sl.rotate, sl.rotate ? s_cos[j] : 1.0, sl.rotate ? s_sin[j] : 0.0, xa[u], xb[u], ya, yb);
          outp[sl.ea] = ya;
          outp[sl.eb] = yb;
        }
      }
    }
  }

  // the value rows: the first batch is already in registers
  for (int base_idx = c_begin; base_idx < c_end; base_idx += blockDim.x * 4) {
    uint4 t[4];
    if (base_idx == c_begin) {
#pragma unroll
      for (int u = 0; u < 4; ++u) t[u] = t_first[u];
    } else {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int idx = base_idx + u * blockDim.x;
        if (idx < c_end) t[u] = v_in[idx];
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int idx = base_idx + u * blockDim.x;
      if (idx < c_end) v_out[idx] = t[u];
    }
  }
}

}  // namespace

cudaError_t launch_rope_append(const RopeAppendArgs& a, const RopeTable& tab, cudaStream_t stream) {
  // every tensor argument must have been set (callers value-initialise the args)
  if (!a.q || !a.q_rot || !a.k_new || !a.v_new || !a.cache_k || !a.cache_v || !a.start_pos)
    return cudaErrorInvalidValue;
  // a few tokens (decode): 8 head vectors per CTA so the launch covers the
  // SMs; many tokens (prefill): whole tokens, so each CTA builds its (cos,
  // sin) table once for all of the token's heads
  const long long tokens = (long long)a.B * a.T;
  const int n_vec = a.H + a.Hkv;
  const int per_cta = tokens >= 512 ? n_vec : 8;
  const long long n_blk = (n_vec + per_cta - 1) / per_cta;
  const long long blocks = tokens * n_blk;
  if (blocks > 0x7FFFFFFFll) return cudaErrorInvalidValue;
  return launch_pdl(rope_append_kernel, dim3((unsigned)blocks), dim3(kRopeThreads), 0, stream, a, tab, per_cta);
}

}  // namespace kvattn

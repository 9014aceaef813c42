// K2 + K3: split-K grouped-query attention over the KV cache, on CUDA cores.
//
// What it computes ("Llama 3.1 8B KV cache", section "The cache itself is
// concatenation"; "Llama 3.1 8B · Repeat heads"; the comment in the "mask"
// code excerpt of "Llama 3 8B · KV cache"): for query token t of sequence b and
// query head h, with G = H / Hkv and j = floor(h / G),
//   out[b,t,h,:] = sum_{r < L} softmax_r(scale * q[b,t,h,:] . K[b,r,j,:]) V[b,r,j,:]
// over the L = start_pos[b] + t + 1 visible cache rows.
//
// Work decomposition.  An "item" is (query row set v = (b,t), split s, KV
// head j): rows [s*C, min((s+1)*C, L)) of KV head j, serving the G query
// heads of that group from the same tiles (no materialised repeat_kv).  Items
// are numbered with the KV head fastest, so CTAs that run side by side read
// the same cache rows of neighbouring heads.  A persistent grid of
// (SMs x CTAs per SM) takes the items from a per-call atomic work counter
// (full splits first, then the last splits largest first), so the tail of a
// ragged batch ends with the smallest pieces; a call with no workspace (no
// splits, no counter) hands item i to CTA i mod grid.
//
// Inside a CTA: one producer warp issues TMA tensor loads of 32-row K and V
// tiles (32 x 256 B each, row stride Hkv*256 B) into a 3-stage shared-memory
// ring; four consumer warps each take 8 rows of every tile.  Sixteen lanes
// share one cache row, each holding 8 of its 128 elements, so a half-warp
// reads a row's 256 bytes from shared memory conflict-free.  Partial dot
// products of RB rows x G heads are reduce-scattered across the 16 lanes
// (each lane ends with complete scores), the online softmax runs in log2
// units (the scale is folded into q), and the probabilities are broadcast
// through shared memory for the P.V accumulation.  FMAs use the packed
// fp32x2 form.  At the end of an item the eight half-warp states (max, sum,
// o) are merged; a single-split row set writes bf16 output directly, others
// write (o, max, sum) partials that K3 merges by log-sum-exp:
//   M = max_s m_s,  out = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s.
#include "kvattn_device.cuh"
#include "kvattn_internal.h"
#include "rope_device.cuh"

#include <algorithm>
#include <type_traits>

namespace kvattn {
namespace {

#ifndef KVATTN_DECODE_STAGES
#define KVATTN_DECODE_STAGES 3
#endif
#ifndef KVATTN_DECODE_MIN_BLOCKS
#define KVATTN_DECODE_MIN_BLOCKS 3
#endif

constexpr int kTileRows = 32;
constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kHalfWarps = kConsumerWarps * 2;
constexpr int kMaxRowSets = 512;
constexpr int kMaxBuckets = 129;  // last-split sizes in tiles: 1 .. 4096/32  // (b,t) row sets handled with a split table
constexpr uint32_t kTileBytes = kTileRows * kHeadDim * 2;

constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x / 2); }

// Shared-memory transpose buffer of the score reduction: per half-warp, 16
// rows (one per lane) of up to 16 partial sums; the 80-byte row pitch keeps
// the 16-byte stores of 8 lanes on distinct banks, and the 336-float region
// pitch puts the two half-warps of a warp on opposite bank halves.
constexpr int kRedPitch = 20;
constexpr int kRedRegion = 336;

template <int G>
struct Shape {
  static constexpr int RB = (G >= 16) ? 1 : (G >= 8) ? 2 : 4;  // rows per half-warp batch
  static constexpr int NV = G * RB;                // partial dot products per lane
  static constexpr int REP = NV >= 16 ? 1 : 16 / NV;  // lanes that end up with the same score
  static constexpr int PASSES = kTileRows / (kHalfWarps * RB);
  // pipeline depth and resident CTAs per SM: G <= 4 fits three CTAs (about
  // 124 registers a thread); G = 8 holds twice the q/o registers and fits two
  static constexpr int STAGES = (G <= 4) ? KVATTN_DECODE_STAGES : 4;
  static constexpr int MIN_BLOCKS = (G <= 4) ? KVATTN_DECODE_MIN_BLOCKS : 2;
  static_assert(kTileRows % (kHalfWarps * RB) == 0, "tile rows");
  static_assert(NV >= 4 && NV <= 16 && NV % 4 == 0, "values per lane");
};

template <int G>
struct __align__(128) Smem {
  uint16_t k[Shape<G>::STAGES][kTileRows][kHeadDim];
  uint16_t v[Shape<G>::STAGES][kTileRows][kHeadDim];
  // q of the G heads of an item, delivered with the item's first tile
  uint16_t q[Shape<G>::STAGES][G][kHeadDim];
  // the score-reduction buffer is only used inside the tile loop and the
  // merge buffer only between the named barriers of an item's epilogue
  union {
    float red[kHalfWarps * kRedRegion];
    float merge_o[kConsumerWarps][G][kHeadDim];
  } u;
  // per half-warp, double-buffered: probabilities and rescale factors, each
  // stored twice so that one 8-byte read yields a packed fp32 pair
  float2 p[2][kHalfWarps][Shape<G>::NV];
  float2 alpha[2][kHalfWarps][G];
  float merge_m[kHalfWarps][G];
  float merge_l[kHalfWarps][G];
  // work table (split path): visible rows per row set, first full-split item
  // of each row set, and the valid row sets ordered by the size of their
  // last (partial) split, largest first
  int set_len[kMaxRowSets];
  int full_start[kMaxRowSets + 1];
  int sorted_set[kMaxRowSets];
  int bucket[kMaxBuckets + 1];
  int n_full, total_items;
  int stage_item[Shape<G>::STAGES];  // item whose tile fills the stage; -1: no more work
  int abort;  // set when a pipeline wait gave up; later waits return at once
  int merge_last;  // fused decode: this CTA stored the last split of the item
  uint64_t full[Shape<G>::STAGES];
  uint64_t empty[Shape<G>::STAGES];
  uint64_t cons;  // the four consumer warps' epilogue barrier
};

// One work item: row set v = (b, t), split `split` of nsplit, KV-head group
// kvh.  Rows are counted in a compacted (virtual) index u in [0, Lv): the
// visible rows of the row set form at most two segments that start on
// 64-row boundaries, u < a_len maps to row u (attention sinks) and u >= a_len
// to row b0 + (u - a_len) (the window, ending at row L - 1).  Rows g0 <= r <
// g1 inside those segments are not visible.  Without a window: a_len = b0 =
// 0, Lv = L and no gap.
struct Item {
  int v, split, kvh, b, t, L, Lv, a_len, b0, g0, g1, r0, r1, nsplit;
};

struct RowView {
  int L, Lv, a_len, b0, g0, g1;
};

// Visible rows of row set v = (b, t) (Lv = 0 when its start position is out of
// range or above the hint).
template <bool WINDOW>
__device__ __forceinline__ RowView row_view(const DecodeArgs& a, int v) {
  RowView r{0, 0, 0, 0, 0, 0};
  const int b = v / a.Tq;
  const int sp = a.start_pos[b];
  if (sp < 0 || (long long)sp + a.Tq > a.S || (long long)sp + a.Tq > a.kv_len_hint) return r;
  r.L = sp + (v - b * a.Tq) + 1;
  r.Lv = r.L;
  if (!WINDOW || a.window <= 0 || r.L <= a.window) return r;
  const int lo = r.L - a.window;        // first row of the window
  const int ns = min(a.n_sink, lo);     // sink rows below it
  const int lo_al = lo & ~63;
  const int ns_al = (ns + 63) & ~63;
  r.g0 = ns;
  r.g1 = lo;
  if (ns == 0) {
    r.b0 = lo_al;                       // the window alone
  } else if (ns_al < lo_al) {
    r.a_len = ns_al;                    // sinks, then the window
    r.b0 = lo_al;
  }                                     // else one segment from row 0 with a short gap
  r.Lv = r.a_len + (r.L - r.b0);
  return r;
}

template <bool WINDOW>
__device__ __forceinline__ int set_length(const DecodeArgs& a, int v) { return row_view<WINDOW>(a, v).Lv; }

// the cache row of compacted index u
__device__ __forceinline__ int item_row(const Item& it, int u) { return u < it.a_len ? u : it.b0 + (u - it.a_len); }

// out = num / den, with a learned sink s2 (log2 units, -inf: none) added to
// the denominator; num and den are relative to the reference max m.
__device__ __forceinline__ float normalise_with_sink(float num, float den, float m, float s2) {
  if (s2 != -INFINITY) {
    const float mn = fmaxf(m, s2);
    const float f = (m == -INFINITY) ? 0.f : fast_exp2(m - mn);
    num *= f;
    den = den * f + fast_exp2(s2 - mn);
  }
  return num / den;
}

// Learned sink of `head` in log2 units, or -inf.
__device__ __forceinline__ float sink_log2(const DecodeArgs& a, int head) {
  return a.sink_logits ? __ldg(a.sink_logits + head) * 1.4426950408889634f : -INFINITY;
}

// Item numbering.  Without splits (max_splits == 1): item i is row set
// i / Hkv, KV head i % Hkv.  With splits: first every full split of every row
// set (row-set major, KV head fastest), then the last split of each valid row
// set in the order of sorted_set (largest first), so that work handed out
// from a counter ends with the smallest pieces.
template <bool WINDOW, class SM>
__device__ __forceinline__ Item decode_item(const DecodeArgs& a, const SM& sm, int n_sets, int i) {
  Item it;
  const int C = a.rows_per_split;
  if (a.max_splits == 1) {
    it.v = i / a.Hkv;
    it.kvh = i - it.v * a.Hkv;
    it.split = 0;
  } else if (i < sm.n_full) {
    int lo = 0, hi = n_sets;  // largest v with full_start[v] <= i
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (sm.full_start[mid] <= i) lo = mid; else hi = mid;
    }
    it.v = lo;
    const int local = i - sm.full_start[lo];
    it.split = local / a.Hkv;
    it.kvh = local - it.split * a.Hkv;
  } else {
    const int r = (i - sm.n_full) / a.Hkv;
    it.kvh = (i - sm.n_full) - r * a.Hkv;
    it.v = sm.sorted_set[r];
    it.split = -1;  // the last split, set below
  }
  if constexpr (WINDOW) {
    const RowView rv = row_view<true>(a, it.v);
    it.L = rv.L;
    it.Lv = rv.Lv;
    it.a_len = rv.a_len;
    it.b0 = rv.b0;
    it.g0 = rv.g0;
    it.g1 = rv.g1;
  } else {
    it.L = a.max_splits == 1 ? set_length<false>(a, it.v) : sm.set_len[it.v];
    it.Lv = it.L;
    it.a_len = it.b0 = it.g0 = it.g1 = 0;
  }
  it.nsplit = (it.Lv + C - 1) / C;
  if (it.split < 0) it.split = it.nsplit - 1;
  it.b = it.v / a.Tq;
  it.t = it.v - it.b * a.Tq;
  it.r0 = it.split * C;
  it.r1 = it.nsplit == 0 ? it.r0 : min(it.r0 + C, it.Lv);
  return it;
}

// Warp 0 builds the work table of the split path (deterministically, so that
// every CTA derives the same numbering).
template <bool WINDOW, class SM>
__device__ void build_work_table(const DecodeArgs& a, SM& sm, int n_sets, int lane) {
  const int C = a.rows_per_split;
  const int nb = C / kTileRows + 1;  // bucket k holds last splits of C/32 - k + ... tiles
  for (int k = lane; k <= nb; k += 32) sm.bucket[k] = 0;
  __syncwarp();
  // lengths, full-split prefix (warp scan over chunks of 32) and bucket counts
  int run = 0;
  for (int base = 0; base < n_sets; base += 32) {
    const int v = base + lane;
    int L = 0, full = 0;
    if (v < n_sets) {
      L = set_length<WINDOW>(a, v);
      sm.set_len[v] = L;
      if (L > 0) {
        const int ns = (L + C - 1) / C;
        full = (ns - 1) * a.Hkv;
        const int last_tiles = (L - (ns - 1) * C + kTileRows - 1) / kTileRows;
        atomicAdd(&sm.bucket[C / kTileRows - last_tiles], 1);  // larger pieces, smaller key
      }
    }
    int incl = full;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (v < n_sets) sm.full_start[v] = run + incl - full;
    run += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) {
    sm.full_start[n_sets] = run;
    sm.n_full = run;
  }
  __syncwarp();
  // exclusive prefix of the bucket counts (lane 0; at most 129 entries)
  if (lane == 0) {
    int acc = 0;
    for (int k = 0; k < nb; ++k) {
      const int c = sm.bucket[k];
      sm.bucket[k] = acc;
      acc += c;
    }
    sm.bucket[nb] = acc;  // valid row sets
    sm.total_items = run + acc * a.Hkv;
  }
  __syncwarp();
  // stable placement in row-set order: equal keys keep increasing v
  for (int base = 0; base < n_sets; base += 32) {
    const int v = base + lane;
    const int L = v < n_sets ? sm.set_len[v] : 0;
    int key = -1;
    if (L > 0) {
      const int ns = (L + C - 1) / C;
      key = C / kTileRows - (L - (ns - 1) * C + kTileRows - 1) / kTileRows;
    }
    const unsigned same = __match_any_sync(0xffffffffu, key);
    const int before = __popc(same & ((1u << lane) - 1u));
    if (key >= 0) sm.sorted_set[sm.bucket[key] + before] = v;
    __syncwarp();
    const int last = 31 - __clz(same);  // highest lane holding this key
    if (key >= 0 && lane == last) sm.bucket[key] += before + 1;
    __syncwarp();
  }
}

// Log-sum-exp merge of the ns split partials of (row set v, head) for output
// element c, in split order with a running maximum:
//   M = max_s m_s,  out = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s.
// The partials may come from other CTAs, so they are read from L2.
__device__ __forceinline__ float lse_merge_element(const DecodeArgs& a, int v, int head, int ns, int c) {
  const size_t base = (size_t)v * a.max_splits * a.H + head;
  float M = -INFINITY, num = 0.f, den = 0.f;
  auto step = [&](float2 ml, float o) {
    const float Mn = fmaxf(M, ml.x);
    const float f_old = (M == -INFINITY) ? 0.f : fast_exp2(M - Mn);
    const float f_new = fast_exp2(ml.x - Mn);
    num = num * f_old + o * f_new;
    den = den * f_old + ml.y * f_new;
    M = Mn;
  };
  // eight splits' loads in flight at a time; the arithmetic stays in split order
  int s = 0;
  for (; s + 8 <= ns; s += 8) {
    float2 ml[8];
    float o[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const size_t slot = base + (size_t)(s + k) * a.H;
      ml[k] = __ldcg(reinterpret_cast<const float2*>(a.ws_ml + slot * 2));
      o[k] = __ldcg(a.ws_o + slot * kHeadDim + c);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) step(ml[k], o[k]);
  }
  for (; s < ns; ++s) {
    const size_t slot = base + (size_t)s * a.H;
    step(__ldcg(reinterpret_cast<const float2*>(a.ws_ml + slot * 2)), __ldcg(a.ws_o + slot * kHeadDim + c));
  }
  return normalise_with_sink(num, den, M, sink_log2(a, head));
}

// Fused decode, after the four consumer warps stored an item's partials: the
// CTA whose item is the last of its (row set, KV head) to finish merges all
// its splits into the bf16 output and clears the counter for the next call.
// Stores, a device-scope fence, then the counter increment on one side; the
// increment that completes the count, a fence, then the loads on the other.
template <int G, class Sync>
__device__ __forceinline__ void merge_if_last(const DecodeArgs& a, const Item& it, int tid, volatile int* flag,
                                              Sync&& sync) {
  __threadfence();
  sync();
  int* cnt = a.merge_counter + (size_t)it.v * a.Hkv + it.kvh;
  if (tid == 0) {
    *flag = atomicAdd(cnt, 1) == it.nsplit - 1;
    __threadfence();
  }
  sync();
  if (*flag) {
    __threadfence();
    for (int h = 0; h < G; ++h) {
      const int head = it.kvh * G + h;
      const float r = lse_merge_element(a, it.v, head, it.nsplit, tid);
      a.out[(((size_t)it.b * a.Tq + it.t) * a.H + head) * kHeadDim + tid] = (uint16_t)f32_to_bf16_bits(r);
    }
    if (tid == 0) atomicExch(cnt, 0);
  }
}

// The producer warp of both decode kernels.  Lane 0 claims items (from the
// per-call counter when there is one, else round-robin over the grid), waits
// for free stages and issues the tile copies (`load` issues one tile's).
//
// Unfused, only lane 0 runs this and the item's (already rotated) q arrives
// by a bulk copy with its first tile.  Fused (one new token per sequence),
// the whole warp runs it: at an item's first tile each lane takes slots lane
// and lane + 32 of every head vector, computes their (cos, sin) at the new
// token's position p = L - 1, and rotates the item's G query heads into the
// stage's q slot.  The item whose rows end at p (the last split) first
// rotates the new K row and writes it, and the new V row, to cache row p,
// then fences the generic-proxy stores against the tensor copies that read
// that row back.  Only that item reads row p, so no other CTA waits on it.
template <bool FUSED, bool WINDOW, int G, int STAGES, int TILE_ROWS, class SM, class Load>
__device__ __forceinline__ void produce(const DecodeArgs& a, const RopeTable& tab, SM& sm, int n_sets,
                                        int total_items, uint32_t tile_bytes, int lane, Load&& load) {
  constexpr uint32_t kQBytes = G * kHeadDim * 2;
  const bool leader = lane == 0;
  auto bcast = [&](int x) {
    if constexpr (FUSED) return __shfl_sync(0xffffffffu, x, 0);
    else return x;
  };
  const uint64_t wlim = wait_limit(a.wait_ns);
  int stage = 0;
  uint32_t phase = 0;
  int next_static = blockIdx.x;
  // stages whose full barrier this warp has armed, and the phase parity each
  // was armed on last (to wait for copies still in flight after an abort)
  uint32_t armed = 0, armed_par = 0;
  auto arm = [&](int st) {
    armed |= 1u << st;
    armed_par = (armed_par & ~(1u << st)) | (phase << st);
  };
  if (leader && !gate_wait(a.gate, wlim)) abort_pipeline(&sm.abort, a.dev_status);
  for (;;) {
    int i = 0, stop = 0;
    if (leader) {
      i = a.counter ? atomicAdd(a.counter, 1) : next_static;
      stop = (i >= total_items || sm.abort) ? 1 : 0;
    }
    next_static += gridDim.x;
    i = bcast(i);
    stop = bcast(stop);
    if (stop) {
      // hand the consumers the end marker through the next stage
      if (leader) {
        if (mbar_wait(&sm.empty[stage], phase ^ 1, &sm.abort, wlim)) {
          sm.stage_item[stage] = -1;
          arm(stage);  // (a phase with no copy: it completes on this arrival)
          mbar_arrive(&sm.full[stage]);
        } else {
          abort_pipeline(&sm.abort, a.dev_status);
        }
      }
      if (++stage == STAGES) { stage = 0; phase ^= 1; }
      break;
    }
    const Item it = decode_item<WINDOW>(a, sm, n_sets, i);
    if (it.nsplit == 0) continue;  // invalid row set: nothing to stream
    for (int row = it.r0; row < it.r1; row += TILE_ROWS) {
      int ok = 1;
      if (leader) ok = mbar_wait(&sm.empty[stage], phase ^ 1, &sm.abort, wlim) ? 1 : 0;
      ok = bcast(ok);
      if (!ok) {
        if (leader) abort_pipeline(&sm.abort, a.dev_status);
        break;
      }
      const bool first = row == it.r0;
      if (!FUSED || !first) {
        if (leader) {
          sm.stage_item[stage] = i;
          arm(stage);
          mbar_arrive_expect_tx(&sm.full[stage], tile_bytes + (first ? kQBytes : 0u));
          if (first) {
            const uint16_t* qsrc = a.q + (((size_t)it.b * a.Tq + it.t) * a.H + (size_t)it.kvh * G) * kHeadDim;
            bulk_load(&sm.q[stage][0][0], qsrc, kQBytes, &sm.full[stage]);
          }
          load(stage, it, item_row(it, row));
        }
      } else {
        const long long pos = it.L - 1;
        RopeSlot sl[2];
        double cs[2], sn[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          sl[u] = rope_slot(tab, lane + 32 * u);
          rope_cos_sin(tab, lane + 32 * u, pos, cs[u], sn[u]);
        }
        if (it.r1 == it.Lv) {  // the last split: its last row is the new one
          // (with G > 16 every group of the KV head writes the same bits)
          const int kvp = it.kvh / a.kv_div;
          const size_t src = ((size_t)it.b * a.Hkv_phys + kvp) * kHeadDim;
          const size_t dst = (((size_t)it.b * a.S + pos) * a.Hkv_phys + kvp) * kHeadDim;
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            uint16_t ya, yb;
            rope_rotate_bits(sl[u].rotate, cs[u], sn[u], a.k_new[src + sl[u].ea], a.k_new[src + sl[u].eb], ya, yb);
            a.cache_k[dst + sl[u].ea] = ya;
            a.cache_k[dst + sl[u].eb] = yb;
          }
          if (lane < kHeadDim / 8)
            reinterpret_cast<uint4*>(a.cache_v + dst)[lane] = reinterpret_cast<const uint4*>(a.v_new + src)[lane];
          asm volatile("fence.proxy.async.global;" ::: "memory");
          __syncwarp();
        }
        if (leader) {
          sm.stage_item[stage] = i;
          arm(stage);
          mbar_expect_tx(&sm.full[stage], tile_bytes);
          load(stage, it, item_row(it, row));
        }
        const size_t qoff = ((size_t)it.b * a.H + (size_t)it.kvh * G) * kHeadDim;
        uint16_t* qout = (a.q_rot_out && it.split == 0) ? a.q_rot_out + qoff : nullptr;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const uint16_t* qin = a.q + qoff + (size_t)h * kHeadDim;
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            uint16_t ya, yb;
            rope_rotate_bits(sl[u].rotate, cs[u], sn[u], qin[sl[u].ea], qin[sl[u].eb], ya, yb);
            sm.q[stage][h][sl[u].ea] = ya;
            sm.q[stage][h][sl[u].eb] = yb;
            if (qout) {
              qout[h * kHeadDim + sl[u].ea] = ya;
              qout[h * kHeadDim + sl[u].eb] = yb;
            }
          }
        }
        __syncwarp();
        if (leader) mbar_arrive(&sm.full[stage]);  // the stage's one arrival: q is in place
      }
      if (++stage == STAGES) { stage = 0; phase ^= 1; }
    }
  }
  if (!leader) return;
  // Leave only once every copy into this CTA's shared memory has landed:
  // wait (bounded) until the consumers have released every stage.
  if (!sm.abort) {
    for (int s = 0; s < STAGES; ++s) {
      if (!mbar_wait(&sm.empty[stage], phase ^ 1, &sm.abort, wlim)) {
        abort_pipeline(&sm.abort, a.dev_status);
        break;
      }
      if (++stage == STAGES) { stage = 0; phase ^= 1; }
    }
  }
  if (sm.abort) {
    // a wait gave up and the consumers may have left without waiting for
    // their tiles: wait (bounded, regardless of the abort) for the last
    // copies issued into every stage to land before the CTA can exit
    for (int s = 0; s < STAGES; ++s)
      if ((armed >> s) & 1u) mbar_wait(&sm.full[s], (armed_par >> s) & 1u, nullptr, wlim);
  }
  if constexpr (FUSED) {
    // the last CTA to finish leaves the work counter at zero for the next call
    if (a.counter) {
      __threadfence();
      if (atomicAdd(a.exit_counter, 1) == (int)gridDim.x - 1) {
        atomicExch(a.counter, 0);
        atomicExch(a.exit_counter, 0);
      }
    }
  }
}

template <int G, bool FUSED, bool WINDOW>
__global__ void __launch_bounds__(kThreads, Shape<G>::MIN_BLOCKS) decode_splitk_kernel(
    const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
    const DecodeArgs a, const int evict_first, const __grid_constant__ RopeTable tab) {
  using Sh = Shape<G>;
  constexpr int kStages = Sh::STAGES;
  // dynamic shared memory starts 128-byte aligned (the declaration asks for
  // it); casting the array itself keeps the shared state space visible to
  // the compiler, so accesses through `sm` become LDS/STS
  extern __shared__ __align__(128) unsigned char smem_raw[];
  Smem<G>& sm = *reinterpret_cast<Smem<G>*>(smem_raw);
  pdl_wait();  // the previous kernel in the stream (rope_append, say) has finished
  pdl_launch_dependents();

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int n_sets = a.B * a.Tq;
  const uint64_t wlim = wait_limit(a.wait_ns);

  // ---- work table and barriers
  if (warp == 0) {
    if (a.max_splits == 1) {
      if (lane == 0) sm.total_items = n_sets * a.Hkv;
    } else {
      build_work_table<WINDOW>(a, sm, n_sets, lane);
    }
    if (blockIdx.x == 0) {
      for (int v = lane; v < n_sets; v += 32) {
        if (set_length<WINDOW>(a, v) == 0) {
          const int sp = a.start_pos[v / a.Tq];
          set_status(a.dev_status, (sp < 0 || (long long)sp + a.Tq > a.S) ? KVATTN_DEV_START_POS_RANGE
                                                                         : KVATTN_DEV_KV_LEN_HINT);
        }
      }
    }
  }
  if (tid == 32) {
    sm.abort = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kConsumerWarps);
    }
    mbar_init(&sm.cons, kConsumerWarps);
    fence_barrier_init();
  }
  __syncthreads();
  const int total_items = sm.total_items;

  if (warp == kConsumerWarps) {
    // ================================================================ producer
    if (FUSED || lane == 0) {
      uint64_t policy = 0;
      if (lane == 0) {
        prefetch_tensormap(&tmap_k);
        prefetch_tensormap(&tmap_v);
        if (evict_first) policy = l2_policy_evict_first();
        else asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(policy));
      }
      produce<FUSED, WINDOW, G, kStages, kTileRows>(a, tab, sm, n_sets, total_items, 2 * kTileBytes, lane,
                                            [&](int st, const Item& it, int row) {
        const int kvp = it.kvh / a.kv_div;  // the KV head in the cache
        tma_load_4d(&sm.k[st][0][0], &tmap_k, &sm.full[st], 0, kvp, row, it.b, policy);
        tma_load_4d(&sm.v[st][0][0], &tmap_v, &sm.full[st], 0, kvp, row, it.b, policy);
      });
    }
    return;
  }

  // ================================================================== consumers
  const int hw = lane >> 4;                 // half-warp within the warp
  const int l16 = lane & 15;                // 8 elements [8*l16, 8*l16+8) of every row
  const int hwg = warp * 2 + hw;            // half-warp within the CTA

  // score bookkeeping: after the reduction lane l16 holds the complete score
  // n = h*RB + j (head h, row j of the batch) with n = l16 / REP
  constexpr int LOGRB = ilog2(Sh::RB);
  constexpr int LOGREP = ilog2(Sh::REP);
  const int slot_n0 = l16 >> LOGREP;
  const int my_head = slot_n0 >> LOGRB;
  const bool writer = (l16 & (Sh::REP - 1)) == 0;
  const bool head_writer = writer && ((slot_n0 & (Sh::RB - 1)) == 0);
  float* const red = sm.u.red + hwg * kRedRegion;

  int stage = 0;
  uint32_t phase = 0;
  int pbuf = 0;

  uint32_t cons_phase = 0;
  // the four consumer warps meet here in an item's epilogue (bounded wait)
  auto cons_sync = [&]() {
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.cons);
    mbar_wait(&sm.cons, cons_phase, &sm.abort, wlim);
    cons_phase ^= 1;
    __syncwarp();
  };

  // Every consumer warp reads the same item sequence from the stages the
  // producer fills.  After an aborted wait the warps stop at their next item.
  for (;;) {
    if (!mbar_wait(&sm.full[stage], phase, &sm.abort, wlim)) abort_pipeline(&sm.abort, a.dev_status);
    const int i = sm.stage_item[stage];
    if (i < 0 || sm.abort) {
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[stage]);
      break;
    }
    const Item it = decode_item<WINDOW>(a, sm, n_sets, i);
    uint64_t q2[G][4];  // q of the G heads, scaled into log2 units (read at the first tile)
    uint64_t o2[G][4];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int k = 0; k < 4; ++k) o2[h][k] = 0;
    float m_run = -INFINITY;  // running max of my head (log2 units)
    float l_run = 0.f;        // running sum of my slots

    for (int row = it.r0; row < it.r1; row += kTileRows) {
      if (row != it.r0 && !mbar_wait(&sm.full[stage], phase, &sm.abort, wlim)) abort_pipeline(&sm.abort, a.dev_status);
      if (row == it.r0) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const uint4 w = lds128(&sm.q[stage][h][8 * l16]);
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int k = 0; k < 4; ++k)
            q2[h][k] = f2_pack(bf16lo_to_f32(ws[k]) * a.scale_log2, bf16hi_to_f32(ws[k]) * a.scale_log2);
        }
      }
      const uint16_t* Kt = &sm.k[stage][0][0];
      const uint16_t* Vt = &sm.v[stage][0][0];
      // rows of this tile that are not visible: past the item, or in the gap
      // between the attention sinks and the window
      // (the window kernels also hide the rows between the sinks and the window)
      const int act = WINDOW ? item_row(it, row) : row;
      auto hidden = [&](int k) {
        if constexpr (WINDOW) return row + k >= it.r1 || (act + k >= it.g0 && act + k < it.g1);
        else return row + k >= it.r1;
      };
      // One batch: RB rows per half-warp.  MASKED is true only on the last
      // tile of an item, where some rows may lie past the item's end.
      auto batch = [&](int pass, auto masked_tag) {
        constexpr bool MASKED = decltype(masked_tag)::value;
        const int rbase = pass * kHalfWarps * Sh::RB + hwg * Sh::RB;  // row within the tile
        // ---- partial scores for RB rows x G heads
        float part[Sh::NV];
#pragma unroll
        for (int j = 0; j < Sh::RB; ++j) {
          const uint4 kc = lds128(Kt + (rbase + j) * kHeadDim + 8 * l16);
          const uint64_t k0 = bf16x2_to_f2(kc.x), k1 = bf16x2_to_f2(kc.y);
          const uint64_t k2 = bf16x2_to_f2(kc.z), k3 = bf16x2_to_f2(kc.w);
#pragma unroll
          for (int h = 0; h < G; ++h) {
            uint64_t acc = f2_mul(q2[h][0], k0);
            acc = f2_fma(q2[h][1], k1, acc);
            acc = f2_fma(q2[h][2], k2, acc);
            acc = f2_fma(q2[h][3], k3, acc);
            float x, y;
            f2_unpack(acc, x, y);
            part[h * Sh::RB + j] = x + y;
          }
        }
        // ---- reduce over the 16 lanes through shared memory: lane l16
        // stores its NV partials as row l16, then sums column n = l16/REP
#pragma unroll
        for (int x = 0; x < Sh::NV; x += 4)
          *reinterpret_cast<float4*>(red + l16 * kRedPitch + x) =
              make_float4(part[x], part[x + 1], part[x + 2], part[x + 3]);
        __syncwarp();
        float col[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) col[k] = red[k * kRedPitch + slot_n0];
#pragma unroll
        for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
          for (int k = 0; k < w; ++k) col[k] += col[k + w];
        float sc = col[0];
        if constexpr (MASKED) {
          if (hidden(rbase + (slot_n0 & (Sh::RB - 1)))) sc = -INFINITY;
        }

        // ---- online softmax in log2 units with a lazily moved reference:
        // the reference max m_run only moves when the tile max exceeds it by
        // more than 8 (so every probability stays <= 2^8); o and l are
        // rescaled only then, and the final normalisation uses the same
        // reference, so the result is unchanged.
        float tmax = sc;
#pragma unroll
        for (int k = 0; k < LOGRB; ++k) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1 << (k + LOGREP)));
        const bool move = tmax > m_run + 8.f;  // also true while m_run is -inf
        const float m_new = move ? tmax : m_run;
        const float alpha = move ? fast_exp2(m_run - m_new) : 1.f;  // 2^-inf = 0 on the first move
        m_run = m_new;
        float2* pb = sm.p[pbuf][hwg];
        // m_new == -inf only while every row so far was masked
        const float p = (m_new == -INFINITY) ? 0.f : fast_exp2(sc - m_new);
        if (writer) pb[slot_n0] = make_float2(p, p);
        l_run = l_run * alpha + p;
        if (head_writer) sm.alpha[pbuf][hwg][my_head] = make_float2(alpha, alpha);
        const bool any_rescale = __any_sync(0xffffffffu, move);
        __syncwarp();

        // ---- rescale o (rare) and accumulate P.V
        if (any_rescale) {
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const uint64_t al = *reinterpret_cast<const uint64_t*>(&sm.alpha[pbuf][hwg][h]);
#pragma unroll
            for (int k = 0; k < 4; ++k) o2[h][k] = f2_mul(o2[h][k], al);
          }
        }
        // two rows at a time: one 16-byte read gives both rows' probability
        // of a head as packed pairs.  On a masked tile, rows past the item
        // may hold any bits (even NaN), so their V words are replaced by
        // zeros rather than multiplied by a zero probability.
#pragma unroll
        for (int j = 0; j < Sh::RB; j += 2) {
          uint4 va = lds128(Vt + (rbase + j) * kHeadDim + 8 * l16);
          uint4 vb = lds128(Vt + (rbase + j + 1) * kHeadDim + 8 * l16);
          if constexpr (MASKED) {
            const bool ok0 = !hidden(rbase + j);
            const bool ok1 = !hidden(rbase + j + 1);
            va.x = ok0 ? va.x : 0u; va.y = ok0 ? va.y : 0u; va.z = ok0 ? va.z : 0u; va.w = ok0 ? va.w : 0u;
            vb.x = ok1 ? vb.x : 0u; vb.y = ok1 ? vb.y : 0u; vb.z = ok1 ? vb.z : 0u; vb.w = ok1 ? vb.w : 0u;
          }
          const uint64_t a0 = bf16x2_to_f2(va.x), a1 = bf16x2_to_f2(va.y);
          const uint64_t a2 = bf16x2_to_f2(va.z), a3 = bf16x2_to_f2(va.w);
          const uint64_t b0 = bf16x2_to_f2(vb.x), b1 = bf16x2_to_f2(vb.y);
          const uint64_t b2 = bf16x2_to_f2(vb.z), b3 = bf16x2_to_f2(vb.w);
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const uint4 pp = lds128(&pb[h * Sh::RB + j]);
            const uint64_t pa = ((uint64_t)pp.y << 32) | pp.x;
            const uint64_t pbb = ((uint64_t)pp.w << 32) | pp.z;
            o2[h][0] = f2_fma(pbb, b0, f2_fma(pa, a0, o2[h][0]));
            o2[h][1] = f2_fma(pbb, b1, f2_fma(pa, a1, o2[h][1]));
            o2[h][2] = f2_fma(pbb, b2, f2_fma(pa, a2, o2[h][2]));
            o2[h][3] = f2_fma(pbb, b3, f2_fma(pa, a3, o2[h][3]));
          }
        }
        pbuf ^= 1;
      };
      if (row + kTileRows <= it.r1 && !(WINDOW && act < it.g1 && act + kTileRows > it.g0)) {
#pragma unroll
        for (int pass = 0; pass < Sh::PASSES; ++pass) batch(pass, std::false_type{});
      } else {
#pragma unroll
        for (int pass = 0; pass < Sh::PASSES; ++pass) batch(pass, std::true_type{});
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[stage]);
      if (++stage == kStages) { stage = 0; phase ^= 1; }
    }

    // ---- merge the eight half-warp states of this item
    // complete the running sum of my head over the lanes of its rows
    float l_head = l_run;
#pragma unroll
    for (int k = 0; k < LOGRB; ++k) l_head += __shfl_xor_sync(0xffffffffu, l_head, 1 << (k + LOGREP));
    if (head_writer) {
      sm.merge_m[hwg][my_head] = m_run;
      sm.merge_l[hwg][my_head] = l_head;
    }
    cons_sync();
    float Mh[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float mx = -INFINITY;
#pragma unroll
      for (int k = 0; k < kHalfWarps; ++k) mx = fmaxf(mx, sm.merge_m[k][h]);
      Mh[h] = mx;
      const float mine = sm.merge_m[hwg][h];
      const float f = (mine == -INFINITY) ? 0.f : fast_exp2(mine - mx);
      const uint64_t f2 = f2_pack(f, f);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        o2[h][k] = f2_mul(o2[h][k], f2);
        float x, y;
        f2_unpack(o2[h][k], x, y);
        x += __shfl_xor_sync(0xffffffffu, x, 16);
        y += __shfl_xor_sync(0xffffffffu, y, 16);
        o2[h][k] = f2_pack(x, y);
      }
    }
    if (hw == 0) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float4* dst = reinterpret_cast<float4*>(&sm.u.merge_o[warp][h][8 * l16]);
        float x0, x1, x2, x3, x4, x5, x6, x7;
        f2_unpack(o2[h][0], x0, x1);
        f2_unpack(o2[h][1], x2, x3);
        f2_unpack(o2[h][2], x4, x5);
        f2_unpack(o2[h][3], x6, x7);
        dst[0] = make_float4(x0, x1, x2, x3);
        dst[1] = make_float4(x4, x5, x6, x7);
      }
    }
    cons_sync();
    {
      const int c = tid;  // 0..127: one output element per head
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float o = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) o += sm.u.merge_o[w][h][c];
        float Ls = 0.f;
#pragma unroll
        for (int k = 0; k < kHalfWarps; ++k) {
          const float mk = sm.merge_m[k][h];
          if (mk != -INFINITY) Ls += sm.merge_l[k][h] * fast_exp2(mk - Mh[h]);
        }
        const int head = it.kvh * G + h;
        if (it.nsplit == 1 && !a.sink_logits) {
          const float r = o / Ls;
          const uint32_t bits = f32_to_bf16_bits(r);
          a.out[(((size_t)it.b * a.Tq + it.t) * a.H + head) * kHeadDim + c] = (uint16_t)bits;
        } else {
          const size_t slot = ((size_t)it.v * a.max_splits + it.split) * a.H + head;
          a.ws_o[slot * kHeadDim + c] = o;
          if (c == 0) {
            a.ws_ml[slot * 2 + 0] = Mh[h];
            a.ws_ml[slot * 2 + 1] = Ls;
          }
        }
      }
    }
    if constexpr (FUSED) {
      if (it.nsplit > 1) merge_if_last<G>(a, it, tid, &sm.merge_last, cons_sync);
    }
    cons_sync();
  }
}

// K3: log-sum-exp merge of the split partials.  One CTA per (row set, head),
// one thread per output element; one pass with a running maximum.
// query heads per merge CTA (blockDim.y), 128 threads (one per dim) each.
// Four: B=1 at 1000 rows, 32-layer graph 15.9 -> 14.5 us per layer, G = 8
// call 171.4 -> 170.9 us, the headline and multi-query steps within noise
// (one head per CTA launched 2048 CTAs for a 64 x 32-head call; eight heads
// measured slower)
#ifndef KVATTN_MERGE_HEADS_PER_CTA
#define KVATTN_MERGE_HEADS_PER_CTA 4
#endif
constexpr int kMergeHeads = KVATTN_MERGE_HEADS_PER_CTA;

__global__ void __launch_bounds__(kHeadDim * kMergeHeads) decode_merge_kernel(const DecodeArgs a) {
  pdl_wait();  // the split-K kernel has finished and its partials are visible
  pdl_launch_dependents();
  // the split-K kernel is done with the work counter: leave it zero for the next call
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0 && threadIdx.y == 0 && a.counter) *a.counter = 0;
  const int v = blockIdx.x;  // row set (up to 2^24 of them: the grid's x extent)
  const int head = blockIdx.y * kMergeHeads + (int)threadIdx.y;  // query head
  if (head >= a.H) return;
  const int L = set_length<true>(a, v);
  if (L == 0) return;  // invalid row set
  int ns;
  if (a.unit_splits) {
    // the multi-query tcgen05 decode: every unit's pieces are partials
    ns = __ldcg(a.unit_splits + (size_t)v * a.Hkv_phys + head / (a.H / a.Hkv_phys));
  } else {
    ns = (L + a.rows_per_split - 1) / a.rows_per_split;
    if (ns <= 1 && !a.sink_logits) return;  // written directly by K2
  }
  const int b = v / a.Tq, t = v - b * a.Tq;
  const int c = threadIdx.x;
  const float r = lse_merge_element(a, v, head, ns, c);
  a.out[(((size_t)b * a.Tq + t) * a.H + head) * kHeadDim + c] = (uint16_t)f32_to_bf16_bits(r);
}

// ======================================================================
// Tensor-core decode for G >= 8 (legacy warp-level mma.sync, m16n8k16).
//
// At G = 8 the decode does 16 flop per cache byte, above what the fp32 FMA
// units can sustain at HBM speed (about 74 TFLOP/s / 6.5 TB/s = 11 flop/B),
// so the contraction goes to the tensor cores: the G query heads are the M
// dimension (padded to 16), 16 cache rows per warp are K (for P.V) or N (for
// q.K^T).  Per warp and 16 rows: S = q K^T as 2 n-tiles x 8 k-steps, then
// O += P V as 16 n-tiles of 8 dims, P taken straight from the S accumulator
// registers (their layout is the A-fragment layout).  Each lane's S values and
// O values belong to the same head (lane/4, and lane/4+8 when G = 16), so the
// online softmax rescales O without any exchange between lanes.  K and V
// arrive by TMA as 128B-swizzled 64-element halves, read with ldmatrix.
//
// G = 8 runs transposed (kSwap), so no MMA row is padding: per warp and 16
// rows, S^T = K q^T with the rows as M and the 8 heads as N (8 k-steps), then
// O^T += V^T P^T with 16 head dims as M per MMA (8 MMAs), V^T read with
// ldmatrix.trans and P^T made from the S^T accumulators by one movmatrix
// transpose per 8 rows.  Half the MMAs of the padded form.  Each lane holds
// S and O for the same two heads (2(lane%4), +1), so the softmax state that
// rescales O is the lane's own after a max over the lanes that share them.
constexpr int kMmaTileRows = 64;
// G = 4 calls with at least this many (row, KV head) pairs run on the
// tensor-core decode (its 64-row tiles and 2 CTAs per SM pay off once the
// call streams tens of MB; a single short sequence is latency-bound and runs
// faster on the CUDA-core kernel's 32-row tiles and 3 CTAs per SM)
constexpr long long kMmaMinWork = 1ll << 18;
constexpr int kMmaStages = 2;
constexpr uint32_t kMmaHalfBytes = kMmaTileRows * 64 * 2;  // 8 KB

template <int G>
struct __align__(1024) SmemMma {
  uint16_t k[kMmaStages][2][kMmaTileRows * 64];  // [stage][d half][row*64 + swizzled elem]
  uint16_t v[kMmaStages][2][kMmaTileRows * 64];
  uint16_t q[kMmaStages][G][kHeadDim];
  float merge_o[kConsumerWarps][G][kHeadDim];
  float merge_m[kConsumerWarps][G];
  float merge_l[kConsumerWarps][G];
  int set_len[kMaxRowSets];
  int full_start[kMaxRowSets + 1];
  int sorted_set[kMaxRowSets];
  int bucket[kMaxBuckets + 1];
  int n_full, total_items;
  int stage_item[kMmaStages];
  int abort;
  int merge_last;
  uint64_t full[kMmaStages];
  uint64_t empty[kMmaStages];
  uint64_t cons;
};

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// Transpose of an 8x8 b16 matrix held one row pair per lane (lane l: row
// l/4, columns 2(l%4), 2(l%4)+1) into the same layout.
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t r;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(r) : "r"(x));
  return r;
}
// byte offset of the 16-byte chunk holding elements 8*chunk.. of `row` in a
// 128B-swizzled [rows][64] half tile
__device__ __forceinline__ uint32_t sw128_off(int row, int chunk) {
  return (uint32_t)(row * 128 + (((chunk ^ row) & 7) << 4));
}

template <int G, bool FUSED, bool WINDOW>
__global__ void __launch_bounds__(kThreads, 2) decode_mma_kernel(
    const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
    const DecodeArgs a, const int evict_first, const __grid_constant__ RopeTable tab) {
  static_assert(G == 1 || G == 2 || G == 4 || G == 8 || G == 16, "tensor-core decode handles G <= 16");
  // (its own name: the CUDA-core kernel in this file declares the dynamic
  // shared memory with a smaller alignment)
  extern __shared__ __align__(1024) unsigned char smem_mma_raw[];
  SmemMma<G>& sm = *reinterpret_cast<SmemMma<G>*>(smem_mma_raw);
  pdl_wait();  // the previous kernel in the stream (rope_append, say) has finished
  pdl_launch_dependents();
  // the 128B-swizzled tiles need a 1024-byte aligned base; refuse otherwise
  if ((smem_u32(smem_mma_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) set_status(a.dev_status, KVATTN_DEV_INTERNAL);
    return;
  }

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int n_sets = a.B * a.Tq;
  const uint64_t wlim = wait_limit(a.wait_ns);

  if (warp == 0) {
    if (a.max_splits == 1) {
      if (lane == 0) sm.total_items = n_sets * a.Hkv;
    } else {
      build_work_table<WINDOW>(a, sm, n_sets, lane);
    }
    if (blockIdx.x == 0) {
      for (int v = lane; v < n_sets; v += 32) {
        if (set_length<WINDOW>(a, v) == 0) {
          const int sp = a.start_pos[v / a.Tq];
          set_status(a.dev_status, (sp < 0 || (long long)sp + a.Tq > a.S) ? KVATTN_DEV_START_POS_RANGE
                                                                         : KVATTN_DEV_KV_LEN_HINT);
        }
      }
    }
  }
  if (tid == 32) {
    sm.abort = 0;
    for (int s = 0; s < kMmaStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kConsumerWarps);
    }
    mbar_init(&sm.cons, kConsumerWarps);
    fence_barrier_init();
  }
  __syncthreads();
  const int total_items = sm.total_items;

  if (warp == kConsumerWarps) {
    // ================================================================ producer
    if (FUSED || lane == 0) {
      uint64_t policy = 0;
      if (lane == 0) {
        prefetch_tensormap(&tmap_k);
        prefetch_tensormap(&tmap_v);
        if (evict_first) policy = l2_policy_evict_first();
        else asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(policy));
      }
      produce<FUSED, WINDOW, G, kMmaStages, kMmaTileRows>(a, tab, sm, n_sets, total_items, 4 * kMmaHalfBytes, lane,
                                                  [&](int st, const Item& it, int row) {
        const int kvp = it.kvh / a.kv_div;  // the KV head in the cache
        tma_load_4d(&sm.k[st][0][0], &tmap_k, &sm.full[st], 0, kvp, row, it.b, policy);
        tma_load_4d(&sm.k[st][1][0], &tmap_k, &sm.full[st], 64, kvp, row, it.b, policy);
        tma_load_4d(&sm.v[st][0][0], &tmap_v, &sm.full[st], 0, kvp, row, it.b, policy);
        tma_load_4d(&sm.v[st][1][0], &tmap_v, &sm.full[st], 64, kvp, row, it.b, policy);
      });
    }
    return;
  }

  // ================================================================== consumers
  const int g = lane >> 2;   // head of this lane's accumulator rows (and g + 8)
  const int c4 = lane & 3;   // column pair within an 8-wide fragment
  const int wrow = 16 * warp;  // this warp's 16 rows of each 64-row tile
  int stage = 0;
  uint32_t phase = 0;
  uint32_t cons_phase = 0;
  auto cons_sync = [&]() {
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.cons);
    mbar_wait(&sm.cons, cons_phase, &sm.abort, wlim);
    cons_phase ^= 1;
    __syncwarp();
  };

  for (;;) {
    if (!mbar_wait(&sm.full[stage], phase, &sm.abort, wlim)) abort_pipeline(&sm.abort, a.dev_status);
    const int i = sm.stage_item[stage];
    if (i < 0 || sm.abort) {
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[stage]);
      break;
    }
    const Item it = decode_item<WINDOW>(a, sm, n_sets, i);

    constexpr bool kSwap = (G == 8);
    // q as A fragments (rows = heads g and g+8, columns = head dims), or
    // (kSwap) as B fragments (head lane/4, dims 16kk + 2c4 .. and + 8)
    uint32_t qa[8][4];
    float o[16][4];
#pragma unroll
    for (int dt = 0; dt < 16; ++dt)
#pragma unroll
      for (int x = 0; x < 4; ++x) o[dt][x] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY};  // heads g, g+8 (log2 units)
    float l_run[2] = {0.f, 0.f};

    for (int row = it.r0; row < it.r1; row += kMmaTileRows) {
      if (row != it.r0 && !mbar_wait(&sm.full[stage], phase, &sm.abort, wlim)) abort_pipeline(&sm.abort, a.dev_status);
      if (row == it.r0) {
        const uint32_t* qw = reinterpret_cast<const uint32_t*>(&sm.q[stage][0][0]);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          if constexpr (kSwap) {
            qa[kk][0] = qw[g * 64 + 8 * kk + c4];
            qa[kk][1] = qw[g * 64 + 8 * kk + 4 + c4];
            qa[kk][2] = 0u;
            qa[kk][3] = 0u;
            continue;
          }
          const int col = 8 * kk + c4;  // word index of dims 16kk + 2*c4
          // rows g >= G pad the 16-row MMA tile with zeros
          qa[kk][0] = (G >= 8 || g < G) ? qw[g * 64 + col] : 0u;
          qa[kk][2] = (G >= 8 || g < G) ? qw[g * 64 + col + 4] : 0u;
          if constexpr (G == 16) {
            qa[kk][1] = qw[(g + 8) * 64 + col];
            qa[kk][3] = qw[(g + 8) * 64 + col + 4];
          } else {
            qa[kk][1] = 0u;
            qa[kk][3] = 0u;
          }
        }
      }
      const uint32_t kbase = smem_u32(&sm.k[stage][0][0]);
      const uint32_t vbase = smem_u32(&sm.v[stage][0][0]);
      // (the window kernels also hide the rows between the sinks and the window)
      const int act = WINDOW ? item_row(it, row) : row;
      auto hidden = [&](int k) {
        if constexpr (WINDOW) return row + k >= it.r1 || (act + k >= it.g0 && act + k < it.g1);
        else return row + k >= it.r1;
      };
      const bool masked = row + kMmaTileRows > it.r1 || (WINDOW && act < it.g1 && act + kMmaTileRows > it.g0);
      if (masked) {
        // rows of this warp past the item may hold any bits; zero their V so
        // that no 0 * NaN reaches O (the warp reads only its own 16 rows)
        for (int x = lane; x < 16 * 16; x += 32) {
          const int r = wrow + (x >> 4);
          if (hidden(r)) {
            const int half = (x >> 3) & 1, ch = x & 7;
            *reinterpret_cast<uint4*>(reinterpret_cast<unsigned char*>(&sm.v[stage][half][0]) + r * 128 + ch * 16) =
                make_uint4(0u, 0u, 0u, 0u);
          }
        }
        __syncwarp();
      }

      if constexpr (kSwap) {
        // ---- S^T = K q^T for the warp's 16 rows: lane holds rows wrow + g
        // (st[0], st[1]: heads 2c4, 2c4+1) and wrow + g + 8 (st[2], st[3])
        float st[4] = {0.f, 0.f, 0.f, 0.f};
        const int r = wrow + (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          // matrices (rows wrow..+7 | wrow+8..+15) x (dims chunk 2kk | 2kk+1)
          const int chunk = 2 * kk + (lane >> 4);
          const uint32_t addr = kbase + (uint32_t)(chunk >> 3) * kMmaHalfBytes + sw128_off(r, chunk & 7);
          uint32_t a0, a1, a2, a3;
          ldsm_x4(addr, a0, a1, a2, a3);
          mma_bf16_16816(st, a0, a1, a2, a3, qa[kk][0], qa[kk][1]);
        }
        // ---- online softmax per head: the lane's heads 2c4 (hh = 0) and
        // 2c4 + 1 (hh = 1) over its two rows, then over the 8 lanes sharing them
        float pt[4];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float s0 = st[hh] * a.scale_log2, s1 = st[2 + hh] * a.scale_log2;
          if (masked) {
            if (hidden(wrow + g)) s0 = -INFINITY;
            if (hidden(wrow + g + 8)) s1 = -INFINITY;
          }
          float tmax = fmaxf(s0, s1);
          tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 4));
          tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 8));
          tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16));
          const bool move = tmax > m_run[hh] + 8.f;
          const float m_new = move ? tmax : m_run[hh];
          const float alpha = move ? fast_exp2(m_run[hh] - m_new) : 1.f;
          m_run[hh] = m_new;
          const float p0 = (m_new == -INFINITY) ? 0.f : fast_exp2(s0 - m_new);
          const float p1 = (m_new == -INFINITY) ? 0.f : fast_exp2(s1 - m_new);
          pt[hh] = p0;
          pt[2 + hh] = p1;
          l_run[hh] = l_run[hh] * alpha + (p0 + p1);  // this lane's rows only
          if (alpha != 1.f) {
#pragma unroll
            for (int mb = 0; mb < 8; ++mb) {
              o[mb][hh] *= alpha;
              o[mb][2 + hh] *= alpha;
            }
          }
        }
        // P^T as the B fragment: rows (K) 2c4, 2c4+1 of head (N) g, from the
        // S^T layout (row g, heads 2c4, 2c4+1) by an 8x8 transpose per 8 rows
        const uint32_t pb0 = movmatrix_t(pack_bf16x2(pt[0], pt[1]));
        const uint32_t pb1 = movmatrix_t(pack_bf16x2(pt[2], pt[3]));
        // ---- O^T += V^T P^T: M block mb covers dims 16mb .. 16mb + 15
#pragma unroll
        for (int mb = 0; mb < 8; ++mb) {
          // matrices (rows wrow..+7 | wrow+8..+15) x (dims chunk 2mb | 2mb+1),
          // transposed: a0 dims 16mb.., rows 0-7; a1 dims +8, rows 0-7;
          // a2 dims 16mb.., rows 8-15; a3 dims +8, rows 8-15
          const int mi = lane >> 3;
          const int rr = wrow + 8 * (mi >> 1) + (lane & 7);
          const int chunk = 2 * mb + (mi & 1);
          const uint32_t addr = vbase + (uint32_t)(chunk >> 3) * kMmaHalfBytes + sw128_off(rr, chunk & 7);
          uint32_t a0, a1, a2, a3;
          ldsm_x4_t(addr, a0, a1, a2, a3);
          mma_bf16_16816(o[mb], a0, a1, a2, a3, pb0, pb1);
        }
      } else {
      // ---- S = q K^T for the warp's 16 rows: n-tile nt covers rows wrow+8nt..+7
      float sacc[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int x = 0; x < 4; ++x) sacc[nt][x] = 0.f;
        const int r = wrow + 8 * nt + (lane & 7);
#pragma unroll
        for (int kp = 0; kp < 4; ++kp) {
          // matrices: dims chunks 4kp + (lane>>3): k-steps 2kp (chunks 4kp, 4kp+1) and 2kp+1
          const int chunk = 4 * kp + (lane >> 3);
          const uint32_t addr = kbase + (uint32_t)(chunk >> 3) * kMmaHalfBytes + sw128_off(r, chunk & 7);
          uint32_t b0, b1, b2, b3;
          ldsm_x4(addr, b0, b1, b2, b3);
          mma_bf16_16816(sacc[nt], qa[2 * kp][0], qa[2 * kp][1], qa[2 * kp][2], qa[2 * kp][3], b0, b1);
          mma_bf16_16816(sacc[nt], qa[2 * kp + 1][0], qa[2 * kp + 1][1], qa[2 * kp + 1][2], qa[2 * kp + 1][3], b2,
                         b3);
        }
      }
      // ---- online softmax per head (lanes with the same g share a head)
      // sacc[nt][0..1]: head g, rows wrow+8nt+2c4+{0,1}; [2..3]: head g+8
      float pv[2][4];
#pragma unroll
      for (int hh = 0; hh < (G == 16 ? 2 : 1); ++hh) {
        float sv[4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int rr = row + wrow + 8 * nt + 2 * c4 + e;
            const float x = sacc[nt][2 * hh + e] * a.scale_log2;
            sv[2 * nt + e] = (masked && hidden(rr - row)) ? -INFINITY : x;
          }
        float tmax = fmaxf(fmaxf(sv[0], sv[1]), fmaxf(sv[2], sv[3]));
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
        const bool move = tmax > m_run[hh] + 8.f;
        const float m_new = move ? tmax : m_run[hh];
        const float alpha = move ? fast_exp2(m_run[hh] - m_new) : 1.f;
        m_run[hh] = m_new;
        float ps = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float p = (m_new == -INFINITY) ? 0.f : fast_exp2(sv[e] - m_new);
          pv[hh][e] = p;
          ps += p;
        }
        l_run[hh] = l_run[hh] * alpha + ps;
        if (alpha != 1.f) {
#pragma unroll
          for (int dt = 0; dt < 16; ++dt) {
            o[dt][2 * hh] *= alpha;
            o[dt][2 * hh + 1] *= alpha;
          }
        }
      }
      // P as the A fragment: a0 = head g rows 2c4..+1, a2 = rows 8+2c4..+1,
      // a1/a3 the same for head g+8 (zero when G = 8)
      uint32_t pa0 = pack_bf16x2(pv[0][0], pv[0][1]);
      uint32_t pa2 = pack_bf16x2(pv[0][2], pv[0][3]);
      uint32_t pa1 = 0u, pa3 = 0u;
      if constexpr (G == 16) {
        pa1 = pack_bf16x2(pv[1][0], pv[1][1]);
        pa3 = pack_bf16x2(pv[1][2], pv[1][3]);
      }
      // ---- O += P V: n-tile dt covers dims 8dt..8dt+7
#pragma unroll
      for (int dp = 0; dp < 8; ++dp) {
        // matrices (rows wrow..+7 | wrow+8..+15) x (dims chunk 2dp | 2dp+1)
        const int mi = lane >> 3;
        const int r = wrow + 8 * (mi & 1) + (lane & 7);
        const int chunk = 2 * dp + (mi >> 1);
        const uint32_t addr = vbase + (uint32_t)(chunk >> 3) * kMmaHalfBytes + sw128_off(r, chunk & 7);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(addr, b0, b1, b2, b3);
        mma_bf16_16816(o[2 * dp], pa0, pa1, pa2, pa3, b0, b1);
        mma_bf16_16816(o[2 * dp + 1], pa0, pa1, pa2, pa3, b2, b3);
      }
      }  // !kSwap
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[stage]);
      if (++stage == kMmaStages) { stage = 0; phase ^= 1; }
    }

    // ---- merge the four warps' states of this item
    if constexpr (kSwap) {
      // o[mb]: dims 16mb + g (0, 1) and + 8 (2, 3), heads 2c4 + (0 | 1)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        float lsum = l_run[hh];
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 4);
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 8);
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 16);
        const int h = 2 * c4 + hh;
        if (g == 0) {
          sm.merge_m[warp][h] = m_run[hh];
          sm.merge_l[warp][h] = lsum;
        }
#pragma unroll
        for (int mb = 0; mb < 8; ++mb) {
          sm.merge_o[warp][h][16 * mb + g] = o[mb][hh];
          sm.merge_o[warp][h][16 * mb + g + 8] = o[mb][2 + hh];
        }
      }
    }
#pragma unroll
    for (int hh = 0; hh < (G == 16 ? 2 : 1) && !kSwap; ++hh) {
      float lsum = l_run[hh];
      lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
      lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
      if (G >= 8 || g < G) {  // padding rows carry no head
        if (c4 == 0) {
          sm.merge_m[warp][g + 8 * hh] = m_run[hh];
          sm.merge_l[warp][g + 8 * hh] = lsum;
        }
#pragma unroll
        for (int dt = 0; dt < 16; ++dt)
          *reinterpret_cast<float2*>(&sm.merge_o[warp][g + 8 * hh][8 * dt + 2 * c4]) =
              make_float2(o[dt][2 * hh], o[dt][2 * hh + 1]);
      }
    }
    cons_sync();
    {
      const int c = tid;  // 0..127: one output element per head
#pragma unroll 1
      for (int h = 0; h < G; ++h) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, sm.merge_m[w][h]);
        float o_sum = 0.f, Ls = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
          const float mw = sm.merge_m[w][h];
          const float f = (mw == -INFINITY) ? 0.f : fast_exp2(mw - M);
          o_sum += f * sm.merge_o[w][h][c];
          Ls += f * sm.merge_l[w][h];
        }
        const int head = it.kvh * G + h;
        if (it.nsplit == 1 && !a.sink_logits) {
          a.out[(((size_t)it.b * a.Tq + it.t) * a.H + head) * kHeadDim + c] = (uint16_t)f32_to_bf16_bits(o_sum / Ls);
        } else {
          const size_t slot = ((size_t)it.v * a.max_splits + it.split) * a.H + head;
          a.ws_o[slot * kHeadDim + c] = o_sum;
          if (c == 0) {
            a.ws_ml[slot * 2 + 0] = M;
            a.ws_ml[slot * 2 + 1] = Ls;
          }
        }
      }
    }
    if constexpr (FUSED) {
      if (it.nsplit > 1) merge_if_last<G>(a, it, tid, &sm.merge_last, cons_sync);
    }
    cons_sync();
  }
}

template <int G>
size_t smem_bytes_mma() {
  return sizeof(SmemMma<G>);
}

template <int G>
size_t smem_bytes() {
  return sizeof(Smem<G>);
}

// G >= 8 always runs the tensor-core kernel; G = 4 has both (MMA when the
// call is large enough, see decode_use_mma); G <= 2 the CUDA-core kernel.
template <int G, bool FUSED, bool WINDOW, bool MMA>
auto decode_kernel() {
  if constexpr (MMA) return decode_mma_kernel<G, FUSED, WINDOW>;
  else return decode_splitk_kernel<G, FUSED, WINDOW>;
}

template <int G, bool MMA>
size_t decode_smem_bytes() {
  if constexpr (MMA) return smem_bytes_mma<G>();
  else return smem_bytes<G>();
}

template <int G, bool FUSED, bool WINDOW, bool MMA>
cudaError_t launch_g(const DecodeArgs& a, const CUtensorMap& tk, const CUtensorMap& tv, const RopeTable& tab,
                     cudaStream_t st) {
  auto kernel = decode_kernel<G, FUSED, WINDOW, MMA>();
  const size_t smem = decode_smem_bytes<G, MMA>();
  static bool configured[64] = {false};
  int dev = 0;
  cudaError_t e0 = cudaGetDevice(&dev);
  if (e0 != cudaSuccess) return e0;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  const int evict_first = a.Tq == 1 ? 1 : 0;
  // The work counter starts at zero: the merge kernel (unfused) or the last
  // CTA to finish (fused) resets it after every call.
  cudaError_t e = launch_pdl(kernel, dim3(a.grid), dim3(kThreads), smem, st, tk, tv, a, evict_first, tab);
  if (e != cudaSuccess) return e;
  if (!FUSED && (a.max_splits > 1 || a.sink_logits)) {
    e = launch_pdl(decode_merge_kernel, dim3(a.B * a.Tq, (a.H + kMergeHeads - 1) / kMergeHeads),
                   dim3(kHeadDim, kMergeHeads), 0, st, a);
  }
  return e;
}

template <int G>
cudaError_t launch_g(const DecodeArgs& a, const CUtensorMap& tk, const CUtensorMap& tv, cudaStream_t st,
                     const RopeTable* fused) {
  RopeTable unused{};
  if constexpr (G >= 8) {
    if (fused) return launch_g<G, true, false, true>(a, tk, tv, *fused, st);
    if (a.window > 0) return launch_g<G, false, true, true>(a, tk, tv, unused, st);
    return launch_g<G, false, false, true>(a, tk, tv, unused, st);
  } else if constexpr (G == 4) {
    if (a.mma) {
      if (fused) return launch_g<G, true, false, true>(a, tk, tv, *fused, st);
      if (a.window > 0) return launch_g<G, false, true, true>(a, tk, tv, unused, st);
      return launch_g<G, false, false, true>(a, tk, tv, unused, st);
    }
    if (fused) return launch_g<G, true, false, false>(a, tk, tv, *fused, st);
    if (a.window > 0) return launch_g<G, false, true, false>(a, tk, tv, unused, st);
    return launch_g<G, false, false, false>(a, tk, tv, unused, st);
  } else {
    if (fused) return launch_g<G, true, false, false>(a, tk, tv, *fused, st);
    if (a.window > 0) return launch_g<G, false, true, false>(a, tk, tv, unused, st);
    return launch_g<G, false, false, false>(a, tk, tv, unused, st);
  }
}

}  // namespace

// Resident CTAs per SM of the decode kernel for group size G (occupancy
// query: registers and shared memory both count).
template <int G, bool FUSED, bool WINDOW, bool MMA>
int resident_ctas_of() {
  auto kernel = decode_kernel<G, FUSED, WINDOW, MMA>();
  const size_t smem = decode_smem_bytes<G, MMA>();
  int n = 0;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, kThreads, smem) != cudaSuccess || n < 1)
    n = 1;
  return n;
}

// the persistent grid serves the unfused, the fused and the window kernels
template <int G, bool MMA>
int resident_ctas() {
  return std::min(std::min(resident_ctas_of<G, false, false, MMA>(), resident_ctas_of<G, true, false, MMA>()),
                  resident_ctas_of<G, false, true, MMA>());
}

int resident_ctas_for(int G, bool mma) {
  static int cached[64][6] = {};  // [device][kernel], 0 = not yet queried
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  const int gi = G == 1 ? 0 : G == 2 ? 1 : G == 4 ? (mma ? 5 : 2) : G == 8 ? 3 : 4;
  int n = __atomic_load_n(&cached[dev][gi], __ATOMIC_RELAXED);
  if (n == 0) {
    switch (gi) {
      case 0: n = resident_ctas<1, false>(); break;
      case 1: n = resident_ctas<2, false>(); break;
      case 2: n = resident_ctas<4, false>(); break;
      case 5: n = resident_ctas<4, true>(); break;
      case 3: n = resident_ctas<8, true>(); break;
      default: n = resident_ctas<16, true>(); break;
    }
    __atomic_store_n(&cached[dev][gi], n, __ATOMIC_RELAXED);
  }
  return n;
}

DecodePlan plan_decode(int B, int Tq, int H, int Hkv, int kv_len_hint, int sm_count, bool always_partials) {
  DecodePlan p;
  const int G = H / Hkv;
  p.mma = decode_use_mma(G, (long long)B * Tq * Hkv * kv_len_hint);
  const int ctas_per_sm = resident_ctas_for(G, p.mma);
  p.ctas_per_sm = ctas_per_sm;
  const int slots = sm_count * ctas_per_sm;
  const long long row_sets = (long long)B * Tq;
  // Split size: aim for a few items per resident CTA at full length (the
  // work counter hands them out, so ragged lengths still balance), as long
  // as that keeps every item long enough that its epilogue (the warps' merge
  // through shared memory and the partial writes) stays small beside its
  // rows.  Measured on 1 GB calls: the tensor-core kernel is fastest at ~4
  // items per CTA (64/8 heads: 173.7 -> 163.0 us from 16 items; 32/8 heads:
  // 168.7 -> 164.3; 131k rows: 449.7 -> 426.0), the CUDA-core kernel at ~8
  // (16/8 heads: 170.6 -> 166.8; 32/32 heads flat, 4 % slower at 4).  Never
  // split below 64 rows, and do not split at all when the (b, t, head)
  // units alone already give enough parallelism.
  const long long items_per_cta = p.mma ? 4 : 8;
  long long want = (row_sets * Hkv * (long long)kv_len_hint) / (items_per_cta * slots);
  int C = 64;
  while (C < 4096 && (long long)C * 2 <= want) C *= 2;
  if (row_sets > kMaxRowSets || row_sets * Hkv >= 16LL * slots || Tq > 1) C = kv_len_hint;
  C = ((C + kTileRows - 1) / kTileRows) * kTileRows;
  if (C >= kv_len_hint) C = ((kv_len_hint + kTileRows - 1) / kTileRows) * kTileRows;
  p.rows_per_split = std::max(C, kTileRows);
  p.max_splits = (kv_len_hint + p.rows_per_split - 1) / p.rows_per_split;
  if (p.max_splits < 1) p.max_splits = 1;
  const long long items_bound = row_sets * Hkv * p.max_splits;
  p.grid = (int)std::min<long long>(items_bound, slots);
  if (p.grid < 1) p.grid = 1;
  // the work counter's 16-byte header, one int per (row set, KV-head group)
  // padded to 16 bytes (see bind_decode_workspace), then the partial (o, max,
  // sum) per (row set, split, head)
  const size_t bytes = 16 + (((size_t)row_sets * Hkv * sizeof(int) + 15) & ~(size_t)15) +
                       (size_t)row_sets * p.max_splits * H * (kHeadDim + 2) * sizeof(float);
  p.ws_bytes = (p.max_splits > 1 || always_partials) ? bytes : 0;
  p.fused_ws_bytes = p.max_splits > 1 ? bytes : 0;
  return p;
}

// Workspace layout: a 16-byte header (work counter; exit counter of the fused
// decode), one int per row set and KV-head group padded to 16 bytes (the
// fused decode's merge counters; the multi-query tcgen05 decode's slot counts
// per unit, written before they are read), then the partial o [row sets,
// splits, H, d] and (max, sum) [row sets, splits, H, 2].  The counters sit at
// fixed offsets, so calls of any shape can share one workspace; every
// completed call leaves them zero, and they must be zero before the first
// call.
void bind_decode_workspace(DecodeArgs& a, const DecodePlan& plan, void* workspace, bool fused) {
  a.exit_counter = nullptr;
  a.merge_counter = nullptr;
  if ((fused ? plan.fused_ws_bytes : plan.ws_bytes) == 0 || !workspace) {
    a.ws_o = nullptr;
    a.ws_ml = nullptr;
    a.counter = nullptr;
    return;
  }
  const size_t n_slots = (size_t)a.B * a.Tq * plan.max_splits * a.H;
  unsigned char* base = static_cast<unsigned char*>(workspace);
  a.counter = reinterpret_cast<int*>(base);
  size_t off = 16;
  if (fused) {
    a.exit_counter = a.counter + 1;
    a.merge_counter = reinterpret_cast<int*>(base + off);
  }
  off += ((size_t)a.B * a.Tq * a.Hkv * sizeof(int) + 15) & ~(size_t)15;
  a.ws_o = reinterpret_cast<float*>(base + off);
  a.ws_ml = a.ws_o + n_slots * kHeadDim;
}

cudaError_t launch_decode(const DecodeArgs& a, const CUtensorMap& tk, const CUtensorMap& tv, cudaStream_t st,
                          const RopeTable* fused) {
  // every tensor argument the chosen kernel dereferences must have been set
  if (!a.q || !a.out || !a.start_pos) return cudaErrorInvalidValue;
  if ((a.max_splits > 1 || a.sink_logits) && (!a.ws_o || !a.ws_ml)) return cudaErrorInvalidValue;
  if (fused && a.sink_logits) return cudaErrorInvalidValue;  // the fused decode has no learned sinks
  if (fused && a.window > 0) return cudaErrorInvalidValue;  // the fused decode has no window
  if (fused && (a.Tq != 1 || !a.k_new || !a.v_new || !a.cache_k || !a.cache_v ||
                (a.counter && (!a.exit_counter || !a.merge_counter))))
    return cudaErrorInvalidValue;
  switch (a.H / a.Hkv) {
    case 1: return launch_g<1>(a, tk, tv, st, fused);
    case 2: return launch_g<2>(a, tk, tv, st, fused);
    case 4: return launch_g<4>(a, tk, tv, st, fused);
    case 8: return launch_g<8>(a, tk, tv, st, fused);
    case 16: return launch_g<16>(a, tk, tv, st, fused);
    default: return cudaErrorInvalidValue;
  }
}

bool decode_use_mma(int G, long long work_rows) { return G >= 8 || (G == 4 && work_rows >= kMmaMinWork); }

cudaError_t launch_decode_merge(const DecodeArgs& a, cudaStream_t st) {
  if (!a.ws_o || !a.ws_ml || !a.out || !a.start_pos || a.rows_per_split < 1 || a.max_splits < 1)
    return cudaErrorInvalidValue;
  return launch_pdl(decode_merge_kernel, dim3(a.B * a.Tq, (a.H + kMergeHeads - 1) / kMergeHeads),
                   dim3(kHeadDim, kMergeHeads), 0, st, a);
}

}  // namespace kvattn

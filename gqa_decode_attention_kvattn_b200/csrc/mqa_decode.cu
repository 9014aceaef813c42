// K2″: multi-query decode (32 query heads per KV head, one new token) on the
// 5th-generation tensor cores, balanced over the SMs.
//
// What it computes ("Llama 3.1 8B KV cache", section "The cache itself is
// concatenation": softmax(q K^T / sqrt(d)) V over the cached rows, with KV
// head floor(h/G) of "Llama 3.1 8B · Repeat heads"): for sequence b and query
// head h,
//   out[b,h,:] = sum_{r <= sp} softmax_r(scale * q[b,h,:] . K[b,r,j,:]) V[b,r,j,:]
// with sp = start_pos[b], j = floor(h/32).  This kernel writes unnormalised
// partials (o, max, sum) per piece of a row set; the log-sum-exp merge of the
// split decode turns them into the output.
//
// Why a kernel of its own.  At 32 heads per KV head the decode does 32 flop
// per cache byte, more than the legacy warp MMAs sustain at HBM speed, so the
// contraction runs on tcgen05: the token's 32 heads are 32 rows of a 128-row
// M tile.  Cutting each sequence into fixed-size splits left the SMs idle for
// a fifth of the kernel (sequences of very different lengths give splits of
// very different cost, and whole CTAs of work land on some SMs and not
// others).  Here the grid is one CTA per SM and the work is cut evenly
// instead (stream-K):
//   - unit u = (sequence b, KV head j) has n_u = ceil((sp + 1) / 128) key tiles;
//     the units' tiles, laid end to end, are tiles 0 .. N-1 of the call;
//   - each CTA runs two streams, stream s = 2 * cta + g takes the contiguous
//     tiles [s L, (s + 1) L) with L = max(ceil(N / streams), min_tiles);
//   - a stream walks its tiles unit by unit; the tiles of one unit within one
//     stream form a piece, and each piece leaves one partial in slot
//     s - floor(P_u / L) of its unit (P_u: the unit's first tile), so the
//     slots of a unit are 0 .. k_u - 1; the stream holding a unit's last tile
//     records k_u for the merge.
// Every CTA computes the same plan from start_pos (a block-wide scan of the
// units' tile counts), so no host round trip and no extra launch is needed.
//
// Per tile and stream g:
//   S_g = Q K^T     8 x tcgen05.mma M=128 N=128 K=16 into TMEM; one shared Q tile
//                   holds stream 0's token at rows 0-31 and stream 1's at rows
//                   32-63, so S_g's rows 32g .. 32g+31 are the ones stream g uses
//   P_g             the softmax warp of stream g reads its 32 rows of S from TMEM,
//                   exponentiates and writes bf16 P back over the S columns
//   O_g += P_g V    8 x tcgen05.mma, P from TMEM, V from shared memory
// Each stream streams its K and V tiles through a ring of three 32 KB slots
// (K(j) is load 2j, V(j) load 2j + 1), so up to 96 KB per stream are in
// flight: at one CTA per SM the loads must cover HBM latency at the SM's share
// of the bandwidth.  The producer and the MMA thread poll both streams and
// serve whichever is ready, so a late tile of one stream does not hold up the
// other.  At a piece boundary the stream's 32 rows of the Q tile are reloaded
// once the last QK of the old piece has finished (the other stream's MMAs
// read those rows too, but only into S rows it never uses), and the first PV
// of the new piece overwrites O (its softmax warp has already read the old
// piece's O out by then).
//
// Warps: 0, 1 = softmax and epilogue of streams 0, 1 (TMEM lanes 0-31 and
// 32-63, on different SM sub-partitions); 2 = TMA producer; 3 = TMEM owner
// and MMA issuer (one thread).
#include "kvattn_device.cuh"
#include "kvattn_internal.h"
#include "tc_device.cuh"

namespace kvattn {
namespace {

constexpr int kMqG = 32;             // query heads per KV head
constexpr int kBN = 128;             // key rows per tile
constexpr int kHalf = 128 * 64 * 2;  // 128 rows x 64 bf16 (16 KB)
constexpr int kSlot = 2 * kHalf;     // one K or V tile (32 KB)
constexpr int kRing = 3;             // ring slots per stream
constexpr int kMqThreads = 128;
constexpr int kWarpProducer = 2, kWarpMma = 3;
constexpr uint32_t kTmemCols = 512;  // S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512)
constexpr uint32_t kColS = 0, kColO = 256;

// shared memory (offsets from a 1024-byte aligned base)
constexpr uint32_t kOffQ = 0;                           // [half 2]: rows 0-31 stream 0, 32-63 stream 1
constexpr uint32_t kOffRing = kOffQ + 2 * kHalf;        // [stream 2][slot 3][half 2]
constexpr uint32_t kOffBar = kOffRing + 2 * kRing * kSlot;
// barriers (8 bytes each); every one exists once per buffer, so a waiter is
// never more than one phase behind
constexpr uint32_t kBarQFull = 0;                     // [stream]
constexpr uint32_t kBarQEmpty = 2;                    // [stream]
constexpr uint32_t kBarFull = 4;                      // [stream][slot]
constexpr uint32_t kBarEmpty = kBarFull + 2 * kRing;  // [stream][slot]
constexpr uint32_t kBarSFull = kBarEmpty + 2 * kRing; // [stream]
constexpr uint32_t kBarPFull = kBarSFull + 2;         // [stream]
constexpr uint32_t kBarODone = kBarPFull + 2;         // [stream]
constexpr uint32_t kBarMmaDone = kBarODone + 2;
constexpr uint32_t kNumBars = kBarMmaDone + 1;
constexpr uint32_t kOffTmemSlot = kOffBar + 8 * kNumBars;
constexpr uint32_t kOffAbort = kOffTmemSlot + 8;
constexpr uint32_t kOffPlan = kOffAbort + 8;  // int[2][4]: first unit, its first tile, range begin, end
constexpr uint32_t kOffScan = kOffPlan + 32;  // int[4]: per-warp tile sums
constexpr uint32_t kMqSmemBytes = kOffScan + 16 + 1024;  // + alignment slack
static_assert(kMqSmemBytes <= 227 * 1024, "shared memory per CTA");

// ring position of load i (K(j): i = 2j, V(j): i = 2j + 1) of a stream
__device__ __forceinline__ int ring_slot(int i) { return i % kRing; }
__device__ __forceinline__ uint32_t ring_par(int i) { return (uint32_t)(i / kRing) & 1u; }

// Tiles of unit u (0 for a start position outside the cache or above the hint).
__device__ __forceinline__ int unit_tiles(const MqaDecodeArgs& a, int u) {
  const int sp = __ldg(a.start_pos + u / a.Hkv);
  if (sp < 0 || sp >= a.S || sp >= a.kv_len_hint) return 0;
  return sp / kBN + 1;
}

// Position of a stream in its range: every role walks the same sequence.
struct Cursor {
  int u, P, n, t;  // unit, its first tile (call-wide index), its tiles, tile within it
  int x, x1;       // call-wide index of the current tile; end of the stream's range
  int pstart;      // call-wide index of the current piece's first tile
  int piece;       // pieces begun before the current one
};

__device__ __forceinline__ Cursor cursor_begin(const MqaDecodeArgs& a, const int* plan) {
  Cursor c;
  c.u = plan[0];
  c.P = plan[1];
  c.x = plan[2];
  c.x1 = plan[3];
  c.n = c.u >= 0 ? unit_tiles(a, c.u) : 0;
  c.t = c.x - c.P;
  c.pstart = c.x;
  c.piece = 0;
  return c;
}
__device__ __forceinline__ bool piece_first(const Cursor& c) { return c.x == c.pstart; }
__device__ __forceinline__ bool piece_last(const Cursor& c) { return c.t == c.n - 1 || c.x == c.x1 - 1; }
__device__ __forceinline__ void cursor_next(const MqaDecodeArgs& a, Cursor& c) {
  ++c.x;
  ++c.t;
  if (c.t == c.n && c.x < c.x1) {
    // the next unit with tiles (the plan guarantees one within the range)
    c.P += c.n;
    const int U = a.B * a.Hkv;
    do {
      ++c.u;
      c.n = c.u < U ? unit_tiles(a, c.u) : 0;
    } while (c.n == 0 && c.u < U);
    c.t = 0;
    c.pstart = c.x;
    ++c.piece;
  }
}

__global__ void __launch_bounds__(kMqThreads, 1)
    mqa_decode_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                         const __grid_constant__ CUtensorMap tmap_v, const MqaDecodeArgs a) {
  pdl_wait();  // the previous kernel in the stream (rope_append, say) has finished
  pdl_launch_dependents();
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sQ = base + kOffQ;
  auto bar = [&](uint32_t slot) { return base + kOffBar + 8u * slot; };
  const uint32_t abort_addr = base + kOffAbort;
  int* plan_sm = reinterpret_cast<int*>(smem_raw + (base - smem_u32(smem_raw)) + kOffPlan);
  int* scan_sm = reinterpret_cast<int*>(smem_raw + (base - smem_u32(smem_raw)) + kOffScan);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const uint64_t wlim = wait_limit(a.wait_ns);

  // ---------------------------------------------------------------- the plan
  // tile counts of the units, a block-wide exclusive scan over contiguous
  // chunks of units, then the thread whose chunk holds a stream's first tile
  // finds that tile's unit
  const int U = a.B * a.Hkv;
  const int chunk = (U + kMqThreads - 1) / kMqThreads;
  const int u_lo = min(U, tid * chunk), u_hi = min(U, u_lo + chunk);
  int mine = 0;
  for (int u = u_lo; u < u_hi; ++u) {
    const int n = unit_tiles(a, u);
    mine += n;
    if (n == 0 && blockIdx.x == 0 && u % a.Hkv == 0) {
      const int sp = __ldg(a.start_pos + u / a.Hkv);
      set_status(a.dev_status, (sp < 0 || sp >= a.S) ? KVATTN_DEV_START_POS_RANGE : KVATTN_DEV_KV_LEN_HINT);
    }
  }
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) scan_sm[warp] = incl;
  __syncthreads();
  int n_tiles = 0, excl = incl - mine;
#pragma unroll
  for (int w = 0; w < kMqThreads / 32; ++w) {
    const int s = scan_sm[w];
    n_tiles += s;
    if (w < warp) excl += s;
  }
  const long long n_streams = 2ll * gridDim.x;
  const int L = max(a.min_tiles, (int)((n_tiles + n_streams - 1) / n_streams));
  for (int g = 0; g < 2; ++g) {
    const long long x0 = (2ll * blockIdx.x + g) * L;
    int* p = plan_sm + 4 * g;
    if (x0 >= n_tiles) {
      if (tid == 0) p[0] = -1, p[1] = 0, p[2] = 0, p[3] = 0;
    } else if (excl <= x0 && x0 < excl + mine) {
      int P = excl;
      for (int u = u_lo; u < u_hi; ++u) {
        const int n = unit_tiles(a, u);
        if (x0 < P + n) {
          p[0] = u, p[1] = P, p[2] = (int)x0, p[3] = (int)min((long long)n_tiles, x0 + L);
          break;
        }
        P += n;
      }
    }
  }
  __syncthreads();
  const int nt0 = plan_sm[0] >= 0 ? plan_sm[3] - plan_sm[2] : 0;
  const int nt1 = plan_sm[4] >= 0 ? plan_sm[7] - plan_sm[6] : 0;
  if (nt0 + nt1 == 0) return;  // nothing left for this CTA (before anything shared)
  const int n_iter = max(nt0, nt1);
  auto n_of = [&](int g) { return g == 0 ? nt0 : nt1; };

  if (tid == 0) {
    for (int g = 0; g < 2; ++g) {
      bar_init(bar(kBarQFull + g), 1);
      bar_init(bar(kBarQEmpty + g), 1);
      for (int r = 0; r < kRing; ++r) {
        bar_init(bar(kBarFull + g * kRing + r), 1);
        bar_init(bar(kBarEmpty + g * kRing + r), 1);
      }
      bar_init(bar(kBarSFull + g), 1);
      bar_init(bar(kBarPFull + g), 1);
      bar_init(bar(kBarODone + g), 1);
    }
    bar_init(bar(kBarMmaDone), 1);
    st_shared_i32(abort_addr, 0);
    fence_barrier_init();
  }
  if (warp == kWarpMma) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(base + kOffTmemSlot),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = (uint32_t)ld_shared_i32(base + kOffTmemSlot);
  auto slot_addr = [&](int g, int i) { return base + kOffRing + (uint32_t)(g * kRing + ring_slot(i)) * kSlot; };
  auto full_bar = [&](int g, int i) { return bar(kBarFull + g * kRing + ring_slot(i)); };
  auto empty_bar = [&](int g, int i) { return bar(kBarEmpty + g * kRing + ring_slot(i)); };
  // a polling loop that made no progress for the wait limit gives up
  auto stalled = [&](uint64_t& t0, bool progress) {
    if (progress) {
      t0 = 0;
      return false;
    }
    if (ld_shared_i32(abort_addr)) return true;
    const uint64_t now = globaltimer_ns();
    if (t0 == 0) t0 = now;
    if (now - t0 > wlim) {
      st_shared_i32(abort_addr, 1);
      set_status(a.dev_status, KVATTN_DEV_WAIT_TIMEOUT);
      return true;
    }
    return false;
  };

  // producer state kept to the end: the last load issued into each ring slot
  // and the last piece whose Q rows were loaded (-1: none), to wait for copies
  // still in flight after an abort
  int last_load[2][kRing] = {{-1, -1, -1}, {-1, -1, -1}};
  int last_q[2] = {-1, -1};
  if (warp == kWarpProducer) {
    // ================================================================ producer
    if (lane == 0) {
      prefetch_tensormap(&tmap_q);
      prefetch_tensormap(&tmap_k);
      prefetch_tensormap(&tmap_v);
      bool go = gate_wait(a.gate, wlim);
      if (!go) {
        st_shared_i32(abort_addr, 1);
        set_status(a.dev_status, KVATTN_DEV_WAIT_TIMEOUT);
      }
      // stream g's token: the 32 heads of its unit, rows 32g .. 32g+31
      auto load_q = [&](int g, int u, int piece) {
        bar_expect_tx(bar(kBarQFull + g), 2u * kMqG * 128u);
        last_q[g] = piece;
        const int b = u / a.Hkv, kvh = u - b * a.Hkv;
        for (int h = 0; h < 2; ++h)
          tma_load_4d_raw(sQ + h * kHalf + g * kMqG * 128, &tmap_q, bar(kBarQFull + g), 64 * h, kvh * kMqG, 0, b);
      };
      Cursor c[2] = {cursor_begin(a, plan_sm), cursor_begin(a, plan_sm + 4)};
      int next[2] = {0, 0};                // next load of each stream
      bool q_ready[2] = {true, true};      // the current piece's Q rows are loaded
      for (int g = 0; g < 2 && go; ++g)
        if (n_of(g) > 0) load_q(g, c[g].u, 0);
      uint64_t t0 = 0;
      while (go && (next[0] < 2 * nt0 || next[1] < 2 * nt1)) {
        bool progress = false;
        for (int g = 0; g < 2; ++g) {
          const int i = next[g];
          if (i >= 2 * n_of(g)) continue;
          const bool is_k = (i & 1) == 0;
          if (is_k && !q_ready[g]) {
            // a new piece: its Q rows once the old piece's last QK has finished
            if (!bar_try_wait(bar(kBarQEmpty + g), (uint32_t)(c[g].piece - 1) & 1u, false)) continue;
            load_q(g, c[g].u, c[g].piece);
            q_ready[g] = true;
            progress = true;
          }
          if (!bar_try_wait(empty_bar(g, i), ring_par(i) ^ 1u, false)) continue;
          const int b = c[g].u / a.Hkv, kvh = c[g].u - b * a.Hkv;
          const uint32_t dst = slot_addr(g, i);
          bar_expect_tx(full_bar(g, i), kSlot);
          last_load[g][ring_slot(i)] = i;
          const CUtensorMap* map = is_k ? &tmap_k : &tmap_v;
          tma_load_4d_raw(dst, map, full_bar(g, i), 0, kvh, c[g].t * kBN, b);
          tma_load_4d_raw(dst + kHalf, map, full_bar(g, i), 64, kvh, c[g].t * kBN, b);
          next[g] = i + 1;
          progress = true;
          if (!is_k) {
            cursor_next(a, c[g]);
            if (piece_first(c[g]) && c[g].piece > 0 && next[g] < 2 * n_of(g)) q_ready[g] = false;
          }
        }
        if (stalled(t0, progress)) go = false;
      }
    }
  } else if (warp == kWarpMma) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_m128_n128(false);
      constexpr uint32_t idesc_pv = idesc_bf16_m128_n128(true);
      const uint64_t q_desc = sw128_desc(sQ, 16, 1024);
      Cursor c[2] = {cursor_begin(a, plan_sm), cursor_begin(a, plan_sm + 4)};
      int j_of[2] = {0, 0};
      bool pv_next[2] = {false, false};  // per stream the ops alternate QK(j), PV(j)
      uint64_t t0 = 0;
      bool ok = true;
      while (ok && (j_of[0] < nt0 || j_of[1] < nt1)) {
        bool progress = false;
        for (int g = 0; g < 2; ++g) {
          const int j = j_of[g];
          if (j >= n_of(g)) continue;
          const uint32_t d_s = tmem + kColS + 128u * (uint32_t)g;
          if (!pv_next[g]) {
            // S_g = Q K_j^T (QK(j) follows PV(j-1), which read P from these columns)
            if (piece_first(c[g]) && !bar_try_wait(bar(kBarQFull + g), (uint32_t)c[g].piece & 1u, false)) continue;
            if (!bar_try_wait(full_bar(g, 2 * j), ring_par(2 * j), false)) continue;
            tc_fence_after();
            const uint64_t k_desc = sw128_desc(slot_addr(g, 2 * j), 16, 1024);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t off = (uint64_t)(((kk >> 2) * kHalf + (kk & 3) * 32) >> 4);
              tc_mma(d_s, q_desc + off, k_desc + off, idesc_qk, kk > 0 ? 1u : 0u);
            }
            tc_commit(bar(kBarSFull + g));
            tc_commit(empty_bar(g, 2 * j));
            if (piece_last(c[g])) tc_commit(bar(kBarQEmpty + g));
            pv_next[g] = true;
          } else {
            // O_g += P_g V_j once the softmax has published P_g; the first PV
            // of a piece starts O afresh.  V as B = [keys x dims], dims
            // contiguous: 64-dim atoms one half apart (LBO), 8-key groups 1 KB
            // apart (SBO), 16 keys (2 KB) per step; P_g from TMEM: keys
            // 16kk .. 16kk+15 are columns 8kk .. 8kk+7 of S_g
            if (!bar_try_wait(full_bar(g, 2 * j + 1), ring_par(2 * j + 1), false)) continue;
            if (!bar_try_wait(bar(kBarPFull + g), (uint32_t)j & 1u, false)) continue;
            tc_fence_after();
            const uint64_t v_desc = sw128_desc(slot_addr(g, 2 * j + 1), kHalf, 1024);
            const uint32_t d_o = tmem + kColO + 128u * (uint32_t)g;
            const bool fresh = piece_first(c[g]);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              tc_mma_ts(d_o, d_s + 8u * kk, v_desc + (uint64_t)(kk * 2048 / 16), idesc_pv,
                        (!fresh || kk > 0) ? 1u : 0u);
            tc_commit(empty_bar(g, 2 * j + 1));
            if (piece_last(c[g])) tc_commit(bar(kBarODone + g));
            cursor_next(a, c[g]);
            pv_next[g] = false;
            j_of[g] = j + 1;
          }
          progress = true;
        }
        if (stalled(t0, progress)) ok = false;
      }
      tc_commit(bar(kBarMmaDone));
      // every MMA issued above has finished once this completes; wait for it
      // even after an abort (bounded), so TMEM and shared memory stay in use
      // until the tensor cores are done with them
      bar_wait_all(bar(kBarMmaDone), 0, wlim);
    }
  } else {
    // ================================================================ softmax / epilogue
    const int g = warp;  // stream; TMEM lanes 32g .. 32g+31 hold its rows
    const int nt = n_of(g);
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * g) << 16);
    const uint32_t col_s = kColS + 128u * (uint32_t)g;
    const uint32_t col_o = kColO + 128u * (uint32_t)g;
    const uint64_t sc2 = f2_pack(a.scale_log2, a.scale_log2);
    const int s_idx = 2 * (int)blockIdx.x + g;
    Cursor c = cursor_begin(a, plan_sm + 4 * g);
    float ref = -INFINITY;  // reference max (log2 units) of the row
    float l = 0.f;          // row sum in units of 2^ref
    for (int j = 0; j < nt; ++j) {
      const int b = c.u / a.Hkv, kvh = c.u - b * a.Hkv;
      const int sp = __ldg(a.start_pos + b);
      const int kbase = c.t * kBN;
      if (!bar_wait(bar(kBarSFull + g), (uint32_t)j & 1u, abort_addr, a.dev_status, wlim)) break;
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int c2 = 0; c2 < 4; ++c2) tmem_ld32(lane_addr + col_s + 32u * c2, sr[c2]);
      tmem_wait_ld();
      const bool need_mask = kbase + kBN - 1 > sp;
      if (need_mask) {
#pragma unroll
        for (int c2 = 0; c2 < 4; ++c2)
#pragma unroll
          for (int k = 0; k < 32; ++k)
            if (kbase + 32 * c2 + k > sp) sr[c2][k] = __float_as_uint(-INFINITY);
      }
      float mx8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx8[k] = -INFINITY;
#pragma unroll
      for (int c2 = 0; c2 < 4; ++c2)
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          mx8[k] = fmax3(mx8[k], __uint_as_float(sr[c2][k]), __uint_as_float(sr[c2][k + 8]));
          mx8[k] = fmax3(mx8[k], __uint_as_float(sr[c2][k + 16]), __uint_as_float(sr[c2][k + 24]));
        }
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]))) *
                       a.scale_log2;
      const bool move = mx > ref + 8.f;
      const float ref_new = move ? mx : ref;
      const float alpha = move ? fast_exp2(ref - ref_new) : 1.f;
      ref = ref_new;
      const float nr = (ref == -INFINITY) ? 0.f : -ref;
      const uint64_t nr2 = f2_pack(nr, nr);
      // p = 2^(s * scale_log2 - ref): one packed FMA per two scores, one pair
      // in four exponentiated on the FMA pipes, bf16 P over the S columns read
      uint64_t sum2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int c2 = 0; c2 < 4; ++c2) {
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 32; k += 2) {
          const uint64_t sv = ((uint64_t)sr[c2][k + 1] << 32) | sr[c2][k];
          float x0, x1;
          f2_unpack(f2_fma(sv, sc2, nr2), x0, x1);
          float p0, p1;
          if (((k >> 1) & 3) < 3) {
            p0 = fast_exp2(x0);
            p1 = fast_exp2(x1);
          } else {
            exp2_poly_x2(x0, x1, p0, p1);  // masked scores are -inf: 2^-inf = 0
            if (need_mask) {
              p0 = x0 == -INFINITY ? 0.f : p0;
              p1 = x1 == -INFINITY ? 0.f : p1;
            }
          }
          sum2[(k >> 1) & 3] = f2_add(sum2[(k >> 1) & 3], f2_pack(p0, p1));
          pk[k >> 1] = pack_bf16x2_p(p0, p1);
        }
        tmem_st16(lane_addr + col_s + 16u * c2, pk);
      }
      float sa, sb;
      f2_unpack(f2_add(f2_add(sum2[0], sum2[1]), f2_add(sum2[2], sum2[3])), sa, sb);
      l = l * alpha + (sa + sb);
      if (!piece_first(c) && __any_sync(0xffffffffu, move)) {
        // a row's reference moved: rescale its O (the piece's previous PV has
        // finished: this tile's QK was issued after it)
#pragma unroll
        for (int c2 = 0; c2 < 4; ++c2) {
          uint32_t r[32];
          tmem_ld32(lane_addr + col_o + 32u * c2, r);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * alpha);
          tmem_st32(lane_addr + col_o + 32u * c2, r);
        }
      }
      if (need_mask) {
        // the unit's last tile: V rows past the last key may hold any bits;
        // zero them so that 0 * (garbage) cannot reach O
        if (bar_wait(full_bar(g, 2 * j + 1), ring_par(2 * j + 1), abort_addr, a.dev_status, wlim)) {
          const uint32_t sv = slot_addr(g, 2 * j + 1);
          const int first_bad = sp + 1 - kbase;
          const int nchunks = (kBN - first_bad) * 16;  // 16-byte chunks over both halves
          for (int q = lane; q < nchunks; q += 32) {
            const int r = first_bad + (q >> 4);
            const int half = (q >> 3) & 1;
            st_shared_v4(sv + half * kHalf + r * 128 + (q & 7) * 16, 0u, 0u, 0u, 0u);
          }
        }
        // the zeroed rows, written through the generic proxy, before the
        // tensor cores read the slot (only this tile needs the fence)
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) bar_arrive(bar(kBarPFull + g));

      if (piece_last(c)) {
        // the piece's partial: unnormalised O and (max, sum), both relative to 2^ref
        if (!bar_wait(bar(kBarODone + g), (uint32_t)c.piece & 1u, abort_addr, a.dev_status, wlim)) break;
        tc_fence_after();
        const int slot = s_idx - c.P / L;
        const int head = kvh * kMqG + lane;
        const size_t row = ((size_t)b * a.part_splits + slot) * a.H + head;
        float* po = a.part_o + row * kHeadDim;
#pragma unroll
        for (int c2 = 0; c2 < 4; ++c2) {
          uint32_t r[32];
          tmem_ld32(lane_addr + col_o + 32u * c2, r);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; k += 4)
            *reinterpret_cast<float4*>(po + 32 * c2 + k) = make_float4(
                __uint_as_float(r[k]), __uint_as_float(r[k + 1]), __uint_as_float(r[k + 2]), __uint_as_float(r[k + 3]));
        }
        *reinterpret_cast<float2*>(a.part_ml + row * 2) = make_float2(ref, l);
        // the stream holding the unit's last tile records how many slots it has
        if (lane == 0 && c.P + c.n <= c.x1) a.unit_splits[c.u] = slot + 1;
        ref = -INFINITY;
        l = 0.f;
        tc_fence_before();
      }
      cursor_next(a, c);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
  if (warp == kWarpProducer && lane == 0 && ld_shared_i32(abort_addr)) {
    // a wait gave up somewhere in the CTA, so some copies may never have been
    // waited for: before the CTA exits, wait (bounded, regardless of the
    // abort) until every copy issued into its shared memory has landed
    for (int g = 0; g < 2; ++g) {
      if (last_q[g] >= 0) bar_wait_all(bar(kBarQFull + g), (uint32_t)last_q[g] & 1u, wlim);
      for (int r = 0; r < kRing; ++r)
        if (last_load[g][r] >= 0) bar_wait_all(full_bar(g, last_load[g][r]), ring_par(last_load[g][r]), wlim);
    }
  }
}

}  // namespace

cudaError_t launch_mqa_decode(const MqaDecodeArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                              const CUtensorMap& tv, int grid, cudaStream_t st) {
  if (!a.start_pos || !a.part_o || !a.part_ml || !a.unit_splits) return cudaErrorInvalidValue;
  if (a.H != kMqG * a.Hkv || a.part_splits < 2 || a.min_tiles < 1 || grid < 1) return cudaErrorInvalidValue;
  static bool configured[64] = {false};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    e = cudaFuncSetAttribute(mqa_decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMqSmemBytes);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  return launch_pdl(mqa_decode_tc_kernel, dim3((unsigned)grid), dim3(kMqThreads), kMqSmemBytes, st, tq, tk, tv, a);
}

}  // namespace kvattn

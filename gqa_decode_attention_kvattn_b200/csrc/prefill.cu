// K4: chunked-prefill attention on the 5th-generation tensor cores (tcgen05,
// accumulators in tensor memory).
//
// What it computes ("Llama 3 8B · KV cache", its "mask" code excerpt: the
// scores of T new tokens against cache_len + T keys, where entry (i, j) is
// masked iff j > cache_len + i; softmax(q K^T / sqrt(d)) V of "Llama 3.1 8B KV
// cache", section "The cache itself is concatenation"; KV head floor(h/G) of
// "Llama 3.1 8B · Repeat heads"): for token t of sequence b and query head h,
//   out[b,t,h,:] = sum_{r <= sp+t} softmax_r(scale * q[b,t,h,:] . K[b,r,j,:]) V[b,r,j,:]
// with sp = start_pos[b] and j = floor(h/G).
//
// Tiling.  The G query heads of one KV head and 128/G consecutive tokens form
// one 128-row M tile (row m = token * G + head), so the grouped heads share
// every K/V tile without a materialised repeat.  One CTA owns two consecutive
// M tiles of one (KV head, sequence) and walks the key rows in 128-row tiles
// up to the last key its last token sees; each K/V tile it loads serves both
// Q tiles, which halves the K/V bytes the SMs pull from L2 per MMA (with one
// Q tile per CTA the kernel was bound by that traffic).  Per KV tile j and Q
// tile g:
//   S_g = Q_g K_j^T      tcgen05.mma M=128 N=128 K=16 x8, bf16 -> fp32 in TMEM
//   P_g = softmax part   one thread per row reads its 128 scores from TMEM,
//                        masks, exponentiates (log2 units) and writes the
//                        bf16 P row back over the S columns it has read
//   O_g += P_g V_j       tcgen05.mma with P read from TMEM and V from shared
//                        memory as an MN-major operand, fp32 in TMEM
// TMEM holds S_0, S_1, O_0 and O_1 (512 columns).  The MMA thread ping-pongs
// between the Q tiles, QK_0(j), PV_1(j-1), QK_1(j), PV_0(j), so the tensor
// cores run one tile's MMAs while the softmax warps of the other work.
// QK_g(j+1) overwrites the columns PV_g(j) reads P_g(j) from; it is issued
// after PV_g(j) by the same thread, and one thread's MMAs run in issue order.
// The softmax publishes P in parts (the first 64 keys, then the rest), so the
// first P.V steps run while the rest of P is computed.  P never touches
// shared memory, which leaves shared-memory bandwidth to the TMA writes and
// the Q, K, V operand reads.
//
// The softmax reference.  A row's reference max only moves when a tile's max
// exceeds it by more than 8 (probabilities stay <= 2^8), so O is rescaled
// rarely; when it moves, the row's thread rescales O_g itself (PV_g(j-1) has
// finished by the time S_g(j) exists).
//
// Warps: 0 = TMA producer, 1 = TMEM owner and MMA issuer (one thread),
// 2..9 = softmax and epilogue: warp w reads TMEM lanes 32*(w%4)..+31 and
// works on Q tile (w-2)/4.
#include "kvattn_device.cuh"
#include "kvattn_internal.h"
#include "tc_device.cuh"

#include <algorithm>

namespace kvattn {
namespace {

constexpr int kBM = 128;            // query rows per tile
constexpr int kBN = 128;            // key rows per tile
constexpr int kHalf = 128 * 64 * 2; // one 128-row x 64-element bf16 half tile (16 KB)
// two softmax groups of four warps (one warp per TMEM lane quarter each), one
// per Q tile
constexpr int kGroupWarps = 4;
constexpr int kGroupThreads = 32 * kGroupWarps;
constexpr int kSoftmaxWarps = 2 * kGroupWarps;
// warp 0: TMA producer; warp 1: TMEM owner and MMA issuer; warps 2..9: softmax
constexpr int kPrefillThreads = 64 + 32 * kSoftmaxWarps;
// TMEM: S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512); bf16 P_g is
// written over the first 64 columns of S_g (two per 32-bit column)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;
constexpr uint32_t kColO = 256;

// shared memory layout (offsets from a 1024-byte aligned base)
constexpr uint32_t kOffQ = 0;                       // [Q tile 2][half 2]
constexpr uint32_t kOffK = kOffQ + 4 * kHalf;       // [stage 2][half 2]
constexpr uint32_t kOffV = kOffK + 4 * kHalf;       // [stage 2][half 2]
constexpr uint32_t kOffBar = kOffV + 4 * kHalf;
// barrier slots (8 bytes each): K/V per stage, S/P per Q tile
// (every pipeline barrier exists once per buffer, so a waiter is never more
// than one phase behind the barrier it waits on)
// (P part k of Q tile g, slot kBarPPart + 3g + k: the P columns of the first
// k+1 parts are in TMEM, the issuer may start P.V on them)
constexpr uint32_t kBarQFull = 0, kBarKFull = 1, kBarKEmpty = 3, kBarVFull = 5, kBarVEmpty = 7, kBarSFull = 9,
                   kBarPFull = 11, kBarMmaDone = 13, kBarPPart = 15,
                   kNumBars = 21;  // MMA done: one per Q tile's softmax group
constexpr uint32_t kOffTmemSlot = kOffBar + 8 * kNumBars;
constexpr uint32_t kOffAbort = kOffTmemSlot + 8;
constexpr uint32_t kPrefillSmemBytes = kOffAbort + 8 + 1024;  // + alignment slack
static_assert(kPrefillSmemBytes <= 227 * 1024, "shared memory per CTA");

// every wait of the producer and the MMA issuer polls without the suspend
// hint (1), or those waits may suspend (0); measured within noise
#ifndef KVATTN_PREFILL_SPIN_ALL
#define KVATTN_PREFILL_SPIN_ALL 1
#endif
// waits of the producer and the MMA issuers: suspend (1) or spin
#ifndef KVATTN_PREFILL_ISSUER_SUSPEND
#define KVATTN_PREFILL_ISSUER_SUSPEND 0
#endif
// of every four pairs of scores, how many are exponentiated by polynomial on
// the FMA pipes instead of the special-function unit (0..4)
#ifndef KVATTN_PREFILL_POLY_PAIRS
#define KVATTN_PREFILL_POLY_PAIRS 1
#endif
// P is published to the MMA issuer in parts, so P.V starts on the first part
// while the rest is computed: 1 (all 128 keys), 2 (64 + 64), 3 (64 + 32 + 32)
// or 4 (32 each); part h holds the 32-key chunks p_begin(h) .. p_begin(h+1)-1.
// On the 4 x 512-token prefill over 3584 cached rows: 149.0 us in one part,
// 144.5 in two, 147.0 in three, 158 in four (each signal costs the softmax a
// TMEM store wait, and four parts spill).
#ifndef KVATTN_PREFILL_P_PARTS
#define KVATTN_PREFILL_P_PARTS 2
#endif
constexpr int kPParts = KVATTN_PREFILL_P_PARTS;
static_assert(kPParts >= 1 && kPParts <= 4, "P parts");
__host__ __device__ constexpr int p_begin(int h) {
  return h >= kPParts ? 4 : kPParts == 1 ? 0 : kPParts == 2 ? 2 * h : kPParts == 3 ? (h == 0 ? 0 : h + 1) : h;
}
// row max with three-input max instructions
#ifndef KVATTN_PREFILL_MAX3
#define KVATTN_PREFILL_MAX3 1
#endif

template <int G>
__global__ void __launch_bounds__(kPrefillThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                      const __grid_constant__ CUtensorMap tmap_v, const PrefillArgs a) {
  constexpr int TT = kBM / G;  // tokens per M tile
  pdl_wait();  // the previous kernel in the stream (rope_append, say) has finished
  pdl_launch_dependents();
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sQ = base + kOffQ, sK = base + kOffK, sV = base + kOffV;
  auto bar = [&](uint32_t slot) { return base + kOffBar + 8u * slot; };
  const uint32_t abort_addr = base + kOffAbort;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const uint64_t wlim = wait_limit(a.wait_ns);

  // heaviest M tile pairs (latest tokens, most keys) first
  const int per_pair = a.Hkv * a.B;
  const int n_pairs = (a.n_mtiles + 1) / 2;
  const int unit = (int)blockIdx.x;
  const int pair = n_pairs - 1 - unit / per_pair;
  const int rem = unit % per_pair;
  const int kvh = rem % a.Hkv;
  const int b = rem / a.Hkv;
  const int sp = a.start_pos[b];
  if (sp < 0 || (long long)sp + a.T > a.S || (long long)sp + a.T > a.kv_len_hint) {
    if (pair == 0 && kvh == 0 && tid == 0)
      set_status(a.dev_status, (sp < 0 || (long long)sp + a.T > a.S) ? KVATTN_DEV_START_POS_RANGE
                                                                    : KVATTN_DEV_KV_LEN_HINT);
    return;
  }
  // Q tile g holds tokens t0 + g*TT ..; the second exists when it starts before T
  const int t0 = pair * 2 * TT;
  const int n_q = (t0 + TT < a.T) ? 2 : 1;
  const int Lmax = sp + min(t0 + n_q * TT, a.T);  // keys the pair's last token sees
  const int n_kv = (Lmax + kBN - 1) / kBN;
  // Key tiles the pair reads: all of 0..n_kv-1, or with a window the tiles
  // holding the attention sinks followed by the tiles from the one holding
  // the first token's earliest window key (the union of the rows' windows).
  int sink_tiles = 0, win_first = 0;
  if (a.window > 0) {
    win_first = max(0, sp + t0 - a.window + 1) / kBN;
    sink_tiles = min((a.n_sink + kBN - 1) / kBN, win_first);
  }
  const int n_all = sink_tiles + (n_kv - win_first);
  // Q tile g reads key tiles 0 .. nt_g - 1 of the n_all; Q tile 0 stops at
  // the key tile of its own last token (at most one short)
  const int nt0 = sink_tiles + ((sp + min(t0 + TT, a.T) + kBN - 1) / kBN - win_first);
  const int nt1 = n_q > 1 ? n_all : 0;
  const int n_iter = max(nt0, nt1);
  auto key_tile = [&](int j) { return j < sink_tiles ? j : win_first + (j - sink_tiles); };
  auto active = [&](int g, int j) { return j < (g == 0 ? nt0 : nt1); };
  // K/V stage and phase parity of key tile j (a two-stage stream)
  auto kv_stage = [&](int j) { return j & 1; };
  auto kv_par = [&](int j) { return (uint32_t)((j >> 1) & 1); };

  if (tid == 0) {
    bar_init(bar(kBarQFull), 1);
    for (int s = 0; s < 2; ++s) {
      bar_init(bar(kBarKFull + s), 1);
      bar_init(bar(kBarKEmpty + s), 1);
      bar_init(bar(kBarVFull + s), 1);
      bar_init(bar(kBarVEmpty + s), 1);
      bar_init(bar(kBarSFull + s), 1);
      bar_init(bar(kBarPFull + s), kGroupWarps);
      for (int k = 0; k < 3; ++k) bar_init(bar(kBarPPart + 3 * s + k), kGroupWarps);
      bar_init(bar(kBarMmaDone + s), 1);
    }
    st_shared_i32(abort_addr, 0);
    fence_barrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(base + kOffTmemSlot),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = (uint32_t)ld_shared_i32(base + kOffTmemSlot);

  // producer state kept to the end of the kernel: whether the gate opened
  // (the Q tiles were loaded) and the key tile last loaded into each K and V
  // stage (-1: none), to wait for copies still in flight after an abort
  bool gate_open = false;
  int last_k[2] = {-1, -1}, last_v[2] = {-1, -1};
  if (warp == 0) {
    // ================================================================ producer
    if (lane == 0) {
      prefetch_tensormap(&tmap_q);
      prefetch_tensormap(&tmap_k);
      prefetch_tensormap(&tmap_v);
      gate_open = gate_wait(a.gate, wlim);
      bool go = gate_open;
      if (!go) {
        st_shared_i32(abort_addr, 1);
        set_status(a.dev_status, KVATTN_DEV_WAIT_TIMEOUT);
      } else {
        // Q tile g: tokens t0 + g*TT .. (rows of tokens past T are the copy's
        // zero fill)
        bar_expect_tx(bar(kBarQFull), (uint32_t)n_q * 2u * kHalf);
        for (int g = 0; g < n_q; ++g) {
          const int tq0 = t0 + g * TT;
          tma_load_4d_raw(sQ + (2 * g) * kHalf, &tmap_q, bar(kBarQFull), 0, kvh * G, tq0, b);
          tma_load_4d_raw(sQ + (2 * g + 1) * kHalf, &tmap_q, bar(kBarQFull), 64, kvh * G, tq0, b);
        }
      }
      for (int j = 0; j < n_iter && go; ++j) {
        // key tile j, loaded once for both Q tiles
        {
          const int s = kv_stage(j);
          const uint32_t par = kv_par(j) ^ 1u;
          const int key0 = key_tile(j) * kBN;
          if (!bar_wait(bar(kBarKEmpty + s), par, abort_addr, a.dev_status, wlim, KVATTN_PREFILL_ISSUER_SUSPEND || !KVATTN_PREFILL_SPIN_ALL)) { go = false; break; }
          bar_expect_tx(bar(kBarKFull + s), 2 * kHalf);
          last_k[s] = j;
          tma_load_4d_raw(sK + (2 * s) * kHalf, &tmap_k, bar(kBarKFull + s), 0, kvh, key0, b);
          tma_load_4d_raw(sK + (2 * s + 1) * kHalf, &tmap_k, bar(kBarKFull + s), 64, kvh, key0, b);
          if (!bar_wait(bar(kBarVEmpty + s), par, abort_addr, a.dev_status, wlim, KVATTN_PREFILL_ISSUER_SUSPEND || !KVATTN_PREFILL_SPIN_ALL)) { go = false; break; }
          bar_expect_tx(bar(kBarVFull + s), 2 * kHalf);
          last_v[s] = j;
          tma_load_4d_raw(sV + (2 * s) * kHalf, &tmap_v, bar(kBarVFull + s), 0, kvh, key0, b);
          tma_load_4d_raw(sV + (2 * s + 1) * kHalf, &tmap_v, bar(kBarVFull + s), 64, kvh, key0, b);
        }
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    // One thread issues every MMA, in an order that keeps the two Q tiles half
    // a period apart: per key tile j,
    //   QK_0(j), PV_1(j-1), QK_1(j), PV_0(j)
    // so the tensor cores run one Q tile's MMAs while the other tile's softmax
    // works.  S_g = Q_g K_j^T goes into TMEM columns that PV_g(j-1) reads
    // P_g(j-1) from; it is issued after that PV by the same thread, and one
    // thread's MMAs run in issue order, so the PV has read its operand first.
    // (A single thread issues an MMA every ~90 cycles; a 128x128x16 MMA takes
    // 64.  Two issuing threads, one per Q tile, reach the tensor core's rate
    // but drift into lockstep: both softmaxes then share the exponential unit
    // and the tensor cores idle meanwhile, which measured slower.)
    if (lane == 0) {
      constexpr bool kSusp = KVATTN_PREFILL_ISSUER_SUSPEND || !KVATTN_PREFILL_SPIN_ALL;
      constexpr uint32_t idesc_qk = idesc_bf16_m128_n128(false);
      constexpr uint32_t idesc_pv = idesc_bf16_m128_n128(true);
      bool ok = bar_wait(bar(kBarQFull), 0, abort_addr, a.dev_status, wlim, kSusp);
      tc_fence_after();
      // operand descriptors of k-step 0; k-step kk adds (byte offset) >> 4
      auto qk = [&](int g, int j) {
        const int s = kv_stage(j);
        tc_fence_after();
        const uint64_t q_desc = sw128_desc(sQ + 2u * (uint32_t)g * kHalf, 16, 1024);
        const uint64_t k_desc = sw128_desc(sK + 2u * (uint32_t)s * kHalf, 16, 1024);
        const uint32_t d_s = tmem + kColS + 128u * (uint32_t)g;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * kHalf + (kk & 3) * 32) >> 4);
          tc_mma(d_s, q_desc + off, k_desc + off, idesc_qk, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(kBarSFull + g));
        return true;
      };
      // O_g += P_g(j) V_j, part by part as the softmax publishes P_g(j)
      auto pv = [&](int g, int j) {
        const int s = kv_stage(j);
        if (!bar_wait(bar(kBarVFull + s), kv_par(j), abort_addr, a.dev_status, wlim, kSusp)) return false;
        // V tile as B = [keys x dims], dims contiguous: 64-dim atoms one half
        // apart (LBO), 8-key groups 1 KB apart (SBO); 16 keys (2 KB) per step;
        // P_g from TMEM: keys 16kk..16kk+15 are columns 8kk..8kk+7 of S_g.
        // The steps of each part of P go out once the softmax has published
        // that part.
        const uint64_t v_desc = sw128_desc(sV + 2u * (uint32_t)s * kHalf, kHalf, 1024);
        const uint32_t d_s = tmem + kColS + 128u * (uint32_t)g;
        const uint32_t d_o = tmem + kColO + 128u * (uint32_t)g;
#pragma unroll
        for (int h = 0; h < kPParts; ++h) {
          const uint32_t pb = h + 1 < kPParts ? bar(kBarPPart + 3u * (uint32_t)g + (uint32_t)h) : bar(kBarPFull + g);
          if (!bar_wait(pb, (uint32_t)j & 1u, abort_addr, a.dev_status, wlim, kSusp)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 2 * p_begin(h); kk < 2 * p_begin(h + 1); ++kk)
            tc_mma_ts(d_o, d_s + 8u * kk, v_desc + (uint64_t)(kk * 2048 / 16), idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
        return true;
      };
      for (int j = 0; j <= n_iter && ok; ++j) {
        if (j < n_iter) {
          if (!bar_wait(bar(kBarKFull + (j & 1)), (uint32_t)(j >> 1) & 1u, abort_addr, a.dev_status, wlim, kSusp))
            break;
          if (active(0, j) && !qk(0, j)) break;
        }
        if (j > 0) {
          if (active(1, j - 1) && !pv(1, j - 1)) break;
          tc_commit(bar(kBarVEmpty + ((j - 1) & 1)));  // both PVs of tile j-1 issued
        }
        if (j < n_iter) {
          if (active(1, j) && !qk(1, j)) break;
          tc_commit(bar(kBarKEmpty + (j & 1)));  // both QKs of tile j issued
          if (active(0, j) && !pv(0, j)) break;
        }
      }
      tc_commit(bar(kBarMmaDone));
      tc_commit(bar(kBarMmaDone + 1));
      // every MMA issued above has finished once this completes; wait for it
      // even after an abort (bounded), so TMEM and shared memory stay in use
      // until the tensor cores are done with them
      bar_wait_all(bar(kBarMmaDone), 0, wlim);
    }
  } else {
    // ================================================================ softmax / epilogue
    const int quarter = warp & 3;         // TMEM lanes 32*quarter .. +31
    const int grp = (warp - 2) >> 2;      // Q tile of this warp
    const int m = 32 * quarter + lane;    // query row of this thread within its Q tile
    const int tok = t0 + grp * TT + m / G;  // token of this row
    const int head = kvh * G + (m % G);
    const int lim = sp + min(tok, a.T - 1);  // last visible key (rows past T borrow the last token's)
    // with a window: keys n_sink <= k < lo_vis are hidden as well
    const int lo_vis = a.window > 0 ? lim - a.window + 1 : 0;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * quarter) << 16);
    const uint32_t col_s = kColS + 128u * (uint32_t)grp;  // S, then P over its first 64 columns
    const uint32_t col_o = kColO + 128u * (uint32_t)grp;
    const int gt = tid - 64 - kGroupThreads * grp;  // index within the group
    const uint64_t sc2 = f2_pack(a.scale_log2, a.scale_log2);
    float ref = -INFINITY;   // reference max (log2 units) of the row
    float l = 0.f;           // row sum in units of 2^ref
    // a warp whose 32 rows are all padding (tokens before 0 or past T) only
    // keeps the barriers moving; its rows of P and O are never stored
    const bool idle = __all_sync(0xffffffffu, tok < 0 || tok >= a.T);

    for (int j = 0; active(grp, j); ++j) {
      const int jt = key_tile(j);
      if (!bar_wait(bar(kBarSFull + grp), (uint32_t)j & 1u, abort_addr, a.dev_status, wlim)) break;
      tc_fence_after();
      // the thread's whole S row, 32 columns (one TMEM load) at a time
      uint32_t sr[4][32];
      // mask (raw scores; the scale is folded into the exponent below)
      const int kbase = jt * kBN;
      const bool need_mask = kbase + kBN - 1 > lim || (kbase < lo_vis && kbase + kBN - 1 >= a.n_sink);
      auto mask_regs = [&](uint32_t (&r)[32], int c2) {
        if (need_mask) {
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int k = kbase + 32 * c2 + c;
            if (k > lim || (k < lo_vis && k >= a.n_sink)) r[c] = __float_as_uint(-INFINITY);
          }
        }
      };
      auto mask_chunk = [&](int c2) { mask_regs(sr[c2], c2); };
      // row max over eight independent accumulators
      float mx8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx8[k] = -INFINITY;
      auto max_regs = [&](const uint32_t (&r)[32]) {
#if KVATTN_PREFILL_MAX3
        // three-input max: half the instructions of a pairwise reduction
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          mx8[k] = fmax3(mx8[k], __uint_as_float(r[k]), __uint_as_float(r[k + 8]));
          mx8[k] = fmax3(mx8[k], __uint_as_float(r[k + 16]), __uint_as_float(r[k + 24]));
        }
#else
#pragma unroll
        for (int c = 0; c < 32; c += 8)
#pragma unroll
          for (int k = 0; k < 8; ++k) mx8[k] = fmaxf(mx8[k], __uint_as_float(r[c + k]));
#endif
      };
      auto max_chunk = [&](int c2) { max_regs(sr[c2]); };
      auto row_max = [&]() {
        return fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                     fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]))) *
               a.scale_log2;
      };
      // p = 2^(s * scale_log2 - ref): packed FMA for two scores, one ex2 each,
      // packed sums in four accumulators; 32 keys (16 P columns) at a time,
      // written over the S columns already read
      uint64_t sum2[4] = {0ull, 0ull, 0ull, 0ull};
      auto exp_regs = [&](uint32_t (&r)[32], int c2, uint64_t nr2) {
        // in stages over the chunk's 16 pairs, each stage's steps independent
        // of one another: the exponent arguments, the exponentials, then the
        // sums and the bf16 packing (the scores are dead after the first)
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const uint64_t sv = ((uint64_t)r[c + 1] << 32) | r[c];
          float x0, x1;
          f2_unpack(f2_fma(sv, sc2, nr2), x0, x1);
          r[c] = __float_as_uint(x0);
          r[c + 1] = __float_as_uint(x1);
        }
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float x0 = __uint_as_float(r[c]), x1 = __uint_as_float(r[c + 1]);
          float p0, p1;
          if (((c >> 1) & 3) < 4 - KVATTN_PREFILL_POLY_PAIRS) {
            p0 = fast_exp2(x0);
            p1 = fast_exp2(x1);
          } else {
            // this pair on the FMA pipes (masked scores are -inf: 2^-inf = 0)
            exp2_poly_x2(x0, x1, p0, p1);
            if (need_mask) {
              p0 = x0 == -INFINITY ? 0.f : p0;
              p1 = x1 == -INFINITY ? 0.f : p1;
            }
          }
          r[c] = __float_as_uint(p0);
          r[c + 1] = __float_as_uint(p1);
        }
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float p0 = __uint_as_float(r[c]), p1 = __uint_as_float(r[c + 1]);
          sum2[(c >> 1) & 3] = f2_add(sum2[(c >> 1) & 3], f2_pack(p0, p1));
          pk[c >> 1] = pack_bf16x2_p(p0, p1);
        }
        tmem_st16(lane_addr + col_s + 16u * c2, pk);
      };
      auto exp_chunk = [&](int c2, uint64_t nr2) { exp_regs(sr[c2], c2, nr2); };
      auto neg_ref2 = [&]() {
        const float nr = (ref == -INFINITY) ? 0.f : -ref;
        return f2_pack(nr, nr);
      };
      float alpha = 1.f;
      uint64_t nr2 = 0ull;
      if (!idle) {
        // load the row, take its max, then exponentiate
#pragma unroll
        for (int c2 = 0; c2 < 4; ++c2) tmem_ld32(lane_addr + col_s + 32u * c2, sr[c2]);
        tmem_wait_ld();
#pragma unroll
        for (int c2 = 0; c2 < 4; ++c2) {
          mask_chunk(c2);
          max_chunk(c2);
        }
        const float mx = row_max();
        const bool move = mx > ref + 8.f;
        const float ref_new = move ? mx : ref;
        alpha = move ? fast_exp2(ref - ref_new) : 1.f;
        ref = ref_new;
        nr2 = neg_ref2();
        // P of the first part's keys; then O's rescale, if the reference
        // moved, before P_g(j) V_j adds to O (PV_g(j-1) has finished: QK_g(j)
        // was issued after it)
#pragma unroll
        for (int c2 = 0; c2 < p_begin(1); ++c2) exp_chunk(c2, nr2);
        if (j > 0 && __any_sync(0xffffffffu, move)) {
#pragma unroll
          for (int c2 = 0; c2 < 4; ++c2) {
            uint32_t r[32];
            tmem_ld32(lane_addr + col_o + 32u * c2, r);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) r[c] = __float_as_uint(__uint_as_float(r[c]) * alpha);
            tmem_st32(lane_addr + col_o + 32u * c2, r);
          }
        }
      }
      if (j == n_all - 1 && Lmax < jt * kBN + kBN) {
        // rows of the last V tile past the last visible key may hold any bits;
        // zero them so that 0 * (garbage) cannot reach O (both Q tiles' groups
        // write the same zeros into the one stage before their own P goes out)
        const int s = kv_stage(j);
        bar_wait(bar(kBarVFull + s), kv_par(j), abort_addr, a.dev_status, wlim);
        const int first_bad = Lmax - jt * kBN;
        const int nchunks = (kBN - first_bad) * 16;  // 16-byte chunks over both halves
        for (int c = gt; c < nchunks; c += kGroupThreads) {
          const int r = first_bad + (c >> 4);
          const int half = (c >> 3) & 1;
          const int cc = c & 7;
          st_shared_v4(sV + (2 * s + half) * kHalf + r * 128 + cc * 16, 0u, 0u, 0u, 0u);
        }
        // the zeroed rows, written through the generic proxy, before the
        // tensor cores read the stage (only this tile needs the fence)
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      }
      // each part of P (the first with O's rescale) goes out as soon as it is
      // in TMEM: the issuer runs P.V on it while the next part is computed
#pragma unroll
      for (int h = 1; h < kPParts; ++h) {
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) bar_arrive(bar(kBarPPart + 3 * grp + (h - 1)));
        if (!idle) {
#pragma unroll
          for (int c2 = p_begin(h); c2 < p_begin(h + 1); ++c2) exp_chunk(c2, nr2);
        }
      }
      if (!idle) {
        float sa, sb;
        f2_unpack(f2_add(f2_add(sum2[0], sum2[1]), f2_add(sum2[2], sum2[3])), sa, sb);
        l = l * alpha + (sa + sb);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) bar_arrive(bar(kBarPFull + grp));
    }

    // ---- epilogue: O / l -> bf16 rows
    // (the MMA-done barrier completes once, after the last PV has finished)
    bar_wait(bar(kBarMmaDone + grp), 0, abort_addr, a.dev_status, wlim);
    tc_fence_after();
    float inv_l = 1.f / l;
    if (a.sink_logits) {
      // learned sink: e^{sink} joins the denominator (log2 units, reference ref)
      const float s2 = __ldg(a.sink_logits + head) * 1.4426950408889634f;
      const float mn = fmaxf(ref, s2);
      const float f = (ref == -INFINITY) ? 0.f : fast_exp2(ref - mn);
      inv_l = f / (l * f + fast_exp2(s2 - mn));
    }
    const bool store = grp < n_q && tok >= 0 && tok < a.T;
    uint16_t* dst = a.out + (((size_t)b * a.T + (store ? tok : 0)) * a.H + head) * kHeadDim;
#pragma unroll
    for (int c2 = 0; c2 < 4; ++c2) {
      uint32_t r[32];
      tmem_ld32(lane_addr + col_o + 32u * c2, r);
      tmem_wait_ld();
      if (store) {
#pragma unroll
        for (int c = 0; c < 32; c += 8) {
          uint4 w;
          w.x = pack_bf16x2_rn(__uint_as_float(r[c]) * inv_l, __uint_as_float(r[c + 1]) * inv_l);
          w.y = pack_bf16x2_rn(__uint_as_float(r[c + 2]) * inv_l, __uint_as_float(r[c + 3]) * inv_l);
          w.z = pack_bf16x2_rn(__uint_as_float(r[c + 4]) * inv_l, __uint_as_float(r[c + 5]) * inv_l);
          w.w = pack_bf16x2_rn(__uint_as_float(r[c + 6]) * inv_l, __uint_as_float(r[c + 7]) * inv_l);
          *reinterpret_cast<uint4*>(dst + 32 * c2 + c) = w;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
  if (tid == 0 && ld_shared_i32(abort_addr)) {
    // a wait gave up somewhere in the CTA, so some tiles may never have been
    // waited for: before the CTA exits, wait (bounded, regardless of the
    // abort) until every copy issued into its shared memory has landed
    if (gate_open) bar_wait_all(bar(kBarQFull), 0, wlim);
    for (int s = 0; s < 2; ++s) {
      if (last_k[s] >= 0) bar_wait_all(bar(kBarKFull + s), kv_par(last_k[s]), wlim);
      if (last_v[s] >= 0) bar_wait_all(bar(kBarVFull + s), kv_par(last_v[s]), wlim);
    }
  }
}

template <int G>
cudaError_t launch_prefill_g(const PrefillArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                             const CUtensorMap& tv, cudaStream_t st) {
  static bool configured[64] = {false};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    e = cudaFuncSetAttribute(prefill_tc_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kPrefillSmemBytes);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  // one CTA per M tile pair
  const long long grid = (long long)((a.n_mtiles + 1) / 2) * a.Hkv * a.B;
  if (grid <= 0 || grid > 0x7FFFFFFFll) return cudaErrorInvalidValue;
  return launch_pdl(prefill_tc_kernel<G>, dim3((unsigned)grid), dim3(kPrefillThreads), kPrefillSmemBytes, st, tq,
                    tk, tv, a);
}

}  // namespace

int prefill_tokens_per_tile(int G) { return kBM / G; }

cudaError_t launch_prefill(const PrefillArgs& a, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           cudaStream_t st) {
  switch (a.H / a.Hkv) {
    case 1: return launch_prefill_g<1>(a, tq, tk, tv, st);
    case 2: return launch_prefill_g<2>(a, tq, tk, tv, st);
    case 4: return launch_prefill_g<4>(a, tq, tk, tv, st);
    case 8: return launch_prefill_g<8>(a, tq, tk, tv, st);
    case 16: return launch_prefill_g<16>(a, tq, tk, tv, st);
    case 32: return launch_prefill_g<32>(a, tq, tk, tv, st);
    case 64: return launch_prefill_g<64>(a, tq, tk, tv, st);
    case 128: return launch_prefill_g<128>(a, tq, tk, tv, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace kvattn

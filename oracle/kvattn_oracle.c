/*
 * kvattn_oracle.c -- plain, slow, fp64 CPU oracle for the cached
 * grouped-query attention step of a Llama-3.1-style decoder.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg load this library.  It shares no code,
 * header, table or helper with the CUDA library; the two meet only through
 * the seeded inputs of kvattn_synth.
 *
 * What it computes, step by step, and where each step is stated:
 *
 *  1. Frequencies f_i = theta^(-2i/d), i < d/2, theta = 500000
 *     ("Llama 3.1 8B KV cache", section "RoPE has to know where it is",
 *     get_rope_params).  Optional Llama-3.1 frequency scaling (factor 8,
 *     low/high frequency cutoffs; named in "Llama 3.1 8B KV cache", section
 *     "Training details that matter", and as use_scaled_rope in
 *     "Llama 3.1 8B · Repeat heads", sku_list.py excerpt).  The pages name the
 *     rule without printing it; the reading taken is the public Llama-3.1
 *     definition written out as mathematics in oracle_rope_freqs.
 *  2. Positions p = start_pos[b] + t: the past length is the offset, so the
 *     token after 4096 cached ones is rotated at angle 4097*f_i (same section
 *     of "Llama 3.1 8B KV cache"; freqs_cis[start_pos:start_pos+seqlen] in the
 *     "mask" code excerpt of "Llama 3 8B · KV cache").
 *  3. Rotation of each pair of q and k by angle p*f_i, as the complex product
 *     (x_a + i x_b) e^{i p f_i}: Meta's apply_rotary_emb (the "update" code
 *     excerpt of "Llama 3 8B · KV cache"; its body is not printed;
 *     interleaved pairs (a, b) = (2i, 2i+1) and the counter-clockwise sense
 *     are the reading taken).  "The Modern Decoder Block" (module L7.3) also
 *     names the half-split layout, pairs (i, i + r/2), and partial rotary,
 *     where only the first r elements rotate (frequencies theta^(-2i/r)) and
 *     the rest pass through; both are offered.  Angle, cos/sin and rotation
 *     in fp64.
 *  4. Storage: q_rot and k_rot rounded to bf16 (round to nearest even), the
 *     cache dtype following the activations (cache.to(xq), bf16 default
 *     tensor type: "Llama 3 8B · KV cache", its "update" and
 *     "dtype" code excerpts).  cache_k[b, p] <- k_rot,
 *     cache_v[b, p] <- v_new; no other row changes (same page, KV-cache
 *     formulas and the write cache_k[:bsz, start_pos:start_pos+seqlen]).
 *  5. Attention for query token t of sequence b and query head h: KV head
 *     j = floor(h / G), G = H / Hkv ("Llama 3.1 8B · Repeat heads":
 *     K_G[h] = K_r[floor(h/4)]; "Grouped-query attention: a smaller KV cache",
 *     6:47).  Visible rows r = 0 .. start_pos[b] + t, the rectangular causal
 *     mask (entry (t, r) masked iff r > cache_len + t: comment in the
 *     "mask" code excerpt of "Llama 3 8B · KV cache").  Scores s_r = q.K_r * scale,
 *     scale = 1/sqrt(d); w = softmax(s) with the maximum subtracted;
 *     out = sum_r w_r V_r -- all in fp64 ("Llama 3.1 8B KV cache", section
 *     "The cache itself is concatenation").  The output is fp64, unrounded.
 *  6. Optional masks of "The Modern Decoder Block" (modules L7.5 and L7.7:
 *     sliding window, StreamingLLM sinks, learned sinks).  The page names
 *     them without defining them; the readings taken are the plain ones of
 *     the cited works: with a window W > 0 the query at position p sees rows
 *     p - W < r <= p; the first n_sink rows (attention sinks) stay visible as
 *     well; positions stay absolute (rows are positions in this cache).  A
 *     learned sink is one logit sigma_h per query head, in the units of the
 *     scaled scores, that joins the softmax denominator and carries no value:
 *     out = sum_r e^{s_r} V_r / (e^{sigma_h} + sum_r e^{s_r}).
 *
 * Layouts (the code layout of "Llama 3 8B · KV cache": [B, positions,
 * heads, d]): q, q_rot, out [B,T,H,d]; k_new, v_new [B,T,Hkv,d];
 * caches [B,S,Hkv,d].  bf16 tensors are passed as their uint16 bit patterns.
 *
 * Pins (tests/test_oracle_pins.py, tests/test_oracle_bruteforce.py): RoPE is
 * the identity at p = 0, preserves pair norms, the half-split layout is the
 * interleaved one conjugated by the pair permutation, partial rotary passes
 * the tail through and rotates the head like a full RoPE of that width, gives dot products that depend
 * only on the relative offset, rotates (1,0) by 90 degrees to (0,1) at angle
 * pi/2, composes additively; the unscaled frequency table has f_0 = 1,
 * f_{d/4} = 1/sqrt(theta) and a constant ratio; the scaled table keeps the
 * high frequencies, divides the low ones by the factor exactly, is
 * continuous at both cutoffs, gives the blend weights of pairs 29..34 worked
 * out by hand from the rule, and blends linearly in L0/wavelength (a pair
 * placed at wavelength L0/2.5 gets exactly 0.5625 f); attention is checked
 * against MHA with repeated KV
 * heads, MQA, single-row and uniform-weight closed forms, a planted-row
 * index test, prefill-vs-stepwise schedule equivalence, and a brute-force
 * complex-number / direct-softmax formula written separately in Python.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_RANGE 3

static const double kPi = 3.14159265358979323846;

/* bf16 bit pattern -> exact double */
static double bf16_to_f64(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* double -> bf16 bit pattern, rounding once, to nearest, ties to even.
 * bf16 carries 8 significant bits and fp32's exponent range: the spacing of
 * representable values around |x| in [2^(e-1), 2^e) is 2^(e-8), and never
 * below the smallest subnormal 2^-133. */
static uint16_t f64_to_bf16(double x) {
  if (isnan(x)) return 0x7FC0;
  if (x == 0.0) return signbit(x) ? 0x8000 : 0x0000;
  if (isinf(x)) return signbit(x) ? 0xFF80 : 0x7F80;
  int e;
  frexp(fabs(x), &e);
  int q = e - 8;
  if (q < -133) q = -133;
  double r = ldexp(nearbyint(ldexp(x, -q)), q); /* default mode: ties to even */
  if (fabs(r) > 3.3895313892515355e38)           /* (2 - 2^-7) * 2^127 */
    return signbit(x) ? 0xFF80 : 0x7F80;
  float f = (float)r; /* exact: r is a bf16 value */
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  return (uint16_t)(u >> 16);
}

uint16_t oracle_f64_to_bf16(double x) { return f64_to_bf16(x); }
double oracle_bf16_to_f64(uint16_t b) { return bf16_to_f64(b); }

/* Step 1.  freqs[i], i < head_dim/2. */
int oracle_rope_freqs(int head_dim, double theta, int use_scaled, double factor,
                      double low_freq_factor, double high_freq_factor,
                      double original_max_pos, double* freqs) {
  if (head_dim <= 0 || (head_dim & 1) || !(theta > 0.0) || !freqs) return ORACLE_ERR_ARG;
  for (int i = 0; i < head_dim / 2; ++i) {
    double f = pow(theta, -(2.0 * i) / (double)head_dim);
    if (use_scaled) {
      /* Llama-3.1 rule: wavelengths shorter than L0/high are kept, longer
       * than L0/low are divided by the factor, and in between the frequency
       * is the blend (1-s) f/factor + s f with s = (L0/wavelength - low) /
       * (high - low). */
      double wavelen = 2.0 * kPi / f;
      double short_cut = original_max_pos / high_freq_factor;
      double long_cut = original_max_pos / low_freq_factor;
      if (wavelen < short_cut) {
        /* keep f */
      } else if (wavelen > long_cut) {
        f = f / factor;
      } else {
        double s = (original_max_pos / wavelen - low_freq_factor) /
                   (high_freq_factor - low_freq_factor);
        f = (1.0 - s) * f / factor + s * f;
      }
    }
    freqs[i] = f;
  }
  return ORACLE_OK;
}

/* Step 3 on one vector of d elements at position p (fp64 in, fp64 out).
 * layout 0: pairs (2i, 2i+1); layout 1: pairs (i, i + r/2); the first
 * r = rotary_dim elements rotate, elements r..d-1 are copied. */
static void rotate_f64(const double* x, double* y, int d, const double* freqs, long p, int layout, int r) {
  for (int c = r; c < d; ++c) y[c] = x[c];
  for (int i = 0; i < r / 2; ++i) {
    const int ia = layout ? i : 2 * i;
    const int ib = layout ? i + r / 2 : 2 * i + 1;
    double a = (double)p * freqs[i];
    double c = cos(a), s = sin(a);
    double x0 = x[ia], x1 = x[ib];
    y[ia] = x0 * c - x1 * s;
    y[ib] = x0 * s + x1 * c;
  }
}

/* Exposed for the RoPE pins: rotate n_vec vectors of d doubles at position p
 * (rotary_dim 0 means d). */
int oracle_rope_rotate_f64(int n_vec, int d, const double* freqs, long p, const double* x, double* y, int layout,
                           int rotary_dim) {
  if (n_vec < 0 || d <= 0 || (d & 1) || !freqs || !x || !y) return ORACLE_ERR_ARG;
  if (rotary_dim == 0) rotary_dim = d;
  if (rotary_dim < 2 || rotary_dim > d || (rotary_dim & 1) || (layout != 0 && layout != 1)) return ORACLE_ERR_ARG;
  for (int v = 0; v < n_vec; ++v)
    rotate_f64(x + (size_t)v * d, y + (size_t)v * d, d, freqs, p, layout, rotary_dim);
  return ORACLE_OK;
}

/* Steps 2-4.  Sequences whose rows start_pos[b] .. start_pos[b]+T-1 do not fit
 * the cache (start_pos < 0 or start_pos + T > S) are left untouched and the
 * call returns ORACLE_ERR_RANGE after processing the others.
 * q_rot_exact / k_rot_exact (may be NULL) receive the fp64 rotated values
 * before rounding, laid out like q and k_new. */
int oracle_rope_append(int B, int T, int H, int Hkv, int d, int S, const double* freqs,
                       const int32_t* start_pos, const uint16_t* q, const uint16_t* k_new,
                       const uint16_t* v_new, uint16_t* q_rot, uint16_t* cache_k,
                       uint16_t* cache_v, double* q_rot_exact, double* k_rot_exact, int layout,
                       int rotary_dim) {
  if (B < 0 || T < 0 || H <= 0 || Hkv <= 0 || d <= 0 || (d & 1) || S < 0) return ORACLE_ERR_ARG;
  if (rotary_dim == 0) rotary_dim = d;
  if (rotary_dim < 2 || rotary_dim > d || (rotary_dim & 1) || (layout != 0 && layout != 1)) return ORACLE_ERR_ARG;
  if (!freqs || !start_pos || !q || !k_new || !v_new || !q_rot || !cache_k || !cache_v)
    return ORACLE_ERR_ARG;
  int rc = ORACLE_OK;
  double* x = (double*)malloc(sizeof(double) * d);
  double* y = (double*)malloc(sizeof(double) * d);
  for (int b = 0; b < B; ++b) {
    long sp = start_pos[b];
    if (sp < 0 || sp + T > S) {
      rc = ORACLE_ERR_RANGE;
      continue;
    }
    for (int t = 0; t < T; ++t) {
      long p = sp + t;
      for (int h = 0; h < H; ++h) {
        size_t off = (((size_t)b * T + t) * H + h) * d;
        for (int c = 0; c < d; ++c) x[c] = bf16_to_f64(q[off + c]);
        rotate_f64(x, y, d, freqs, p, layout, rotary_dim);
        for (int c = 0; c < d; ++c) {
          q_rot[off + c] = f64_to_bf16(y[c]);
          if (q_rot_exact) q_rot_exact[off + c] = y[c];
        }
      }
      for (int j = 0; j < Hkv; ++j) {
        size_t in = (((size_t)b * T + t) * Hkv + j) * d;
        size_t row = (((size_t)b * S + p) * Hkv + j) * d;
        for (int c = 0; c < d; ++c) x[c] = bf16_to_f64(k_new[in + c]);
        rotate_f64(x, y, d, freqs, p, layout, rotary_dim);
        for (int c = 0; c < d; ++c) {
          cache_k[row + c] = f64_to_bf16(y[c]);
          if (k_rot_exact) k_rot_exact[in + c] = y[c];
          cache_v[row + c] = v_new[in + c];
        }
      }
    }
  }
  free(x);
  free(y);
  return rc;
}

/* Step 5.  out [B,T,H,d] fp64.  Rows read: 0 .. start_pos[b]+t of the caches
 * as they stand (the caller has already appended the new rows).  Sequences
 * with start_pos < 0 or start_pos + T > S are skipped (out untouched) and the
 * call returns ORACLE_ERR_RANGE.  n_threads <= 0 uses every core. */
/* Attention with the optional masks of step 6: window <= 0 means no window,
 * n_sink rows always visible when a window is set, sink_logits (length H,
 * may be NULL) the learned sink logits. */
int oracle_attention_masked(int B, int T, int H, int Hkv, int d, int S, const int32_t* start_pos,
                            double scale, int window, int n_sink, const double* sink_logits,
                            const uint16_t* q_rot, const uint16_t* cache_k, const uint16_t* cache_v,
                            double* out, int n_threads) {
  if (B < 0 || T < 0 || H <= 0 || Hkv <= 0 || d <= 0 || S < 0) return ORACLE_ERR_ARG;
  if (H % Hkv != 0 || n_sink < 0) return ORACLE_ERR_ARG;
  if (!start_pos || !q_rot || !cache_k || !cache_v || !out) return ORACLE_ERR_ARG;
  const int G = H / Hkv;
  int rc = ORACLE_OK;
  for (int b = 0; b < B; ++b)
    if (start_pos[b] < 0 || (long)start_pos[b] + T > S) rc = ORACLE_ERR_RANGE;
  const long n_task = (long)B * T * H;
#ifdef _OPENMP
  if (n_threads <= 0) n_threads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads)
#endif
  for (long task = 0; task < n_task; ++task) {
    const int h = (int)(task % H);
    const int t = (int)((task / H) % T);
    const int b = (int)(task / ((long)H * T));
    const long sp = start_pos[b];
    if (sp < 0 || sp + T > S) continue;
    const int j = h / G;
    const long p = sp + t;          /* this token's position */
    const long L = p + 1;           /* rows 0..p */
    const size_t qoff = (((size_t)b * T + t) * H + h) * d;
    double* qv = (double*)malloc(sizeof(double) * d);
    double* s = (double*)malloc(sizeof(double) * L);
    double* acc = (double*)calloc(d, sizeof(double));
    for (int c = 0; c < d; ++c) qv[c] = bf16_to_f64(q_rot[qoff + c]);
    double m = -INFINITY;
    for (long r = 0; r < L; ++r) {
      const int visible = window <= 0 || r > p - window || r < n_sink;
      if (!visible) {
        s[r] = -INFINITY;
        continue;
      }
      const uint16_t* kr = cache_k + (((size_t)b * S + r) * Hkv + j) * d;
      double dot = 0.0;
      for (int c = 0; c < d; ++c) dot += qv[c] * bf16_to_f64(kr[c]);
      s[r] = dot * scale;
      if (s[r] > m) m = s[r];
    }
    if (sink_logits && sink_logits[h] > m) m = sink_logits[h];
    double z = sink_logits ? exp(sink_logits[h] - m) : 0.0;
    for (long r = 0; r < L; ++r) {
      if (s[r] == -INFINITY) continue;
      const double w = exp(s[r] - m);
      z += w;
      const uint16_t* vr = cache_v + (((size_t)b * S + r) * Hkv + j) * d;
      for (int c = 0; c < d; ++c) acc[c] += w * bf16_to_f64(vr[c]);
    }
    for (int c = 0; c < d; ++c) out[qoff + c] = acc[c] / z;
    free(qv);
    free(s);
    free(acc);
  }
  return rc;
}

/* Step 5: every row 0..start_pos[b]+t visible, no sink. */
int oracle_attention(int B, int T, int H, int Hkv, int d, int S, const int32_t* start_pos,
                     double scale, const uint16_t* q_rot, const uint16_t* cache_k,
                     const uint16_t* cache_v, double* out, int n_threads) {
  return oracle_attention_masked(B, T, H, Hkv, d, S, start_pos, scale, 0, 0, NULL, q_rot, cache_k, cache_v,
                                 out, n_threads);
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

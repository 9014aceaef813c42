// Device-side rotary embedding of one 128-element head vector, slot by slot.
//
// A head vector has 64 slots.  Slot j < r/2 (r = rotary width) is the pair
// of elements that frequency f_j rotates: (2j, 2j+1) in the interleaved
// layout of Meta's Llama code, (j, j + r/2) in the half-split layout of the
// GPT-NeoX / Hugging Face code ("Rotary position embeddings", section on the
// two pairing conventions).  Slots j >= r/2 carry elements r + 2(j - r/2) and
// the next one, which pass through unchanged.  The rotation by the angle
// a = p * f_j is
//   y_a = x_a cos a - x_b sin a,   y_b = x_a sin a + x_b cos a,
// evaluated in fp64 from the bf16 inputs and rounded once (RNE) to bf16.
#pragma once

#include "kvattn_device.cuh"
#include "kvattn_internal.h"

namespace kvattn {

struct RopeSlot {
  int ea, eb;   // element indices of the slot
  bool rotate;  // false: copied unchanged
};

__device__ __forceinline__ RopeSlot rope_slot(const RopeTable& tab, int j) {
  const int rp = tab.rotary_dim >> 1;
  RopeSlot s;
  s.rotate = j < rp;
  if (s.rotate) {
    s.ea = tab.layout ? j : 2 * j;
    s.eb = tab.layout ? j + rp : 2 * j + 1;
  } else {
    s.ea = 2 * rp + 2 * (j - rp);
    s.eb = s.ea + 1;
  }
  return s;
}

// (cos, sin) of the angle of slot j at position pos; (1, 0) for copied slots.
__device__ __forceinline__ void rope_cos_sin(const RopeTable& tab, int j, long long pos, double& c, double& s) {
  if (j < (tab.rotary_dim >> 1)) {
    sincos((double)pos * tab.freq[j], &s, &c);
  } else {
    c = 1.0;
    s = 0.0;
  }
}

// Rotated bf16 bits of a slot's two inputs.
__device__ __forceinline__ void rope_rotate_bits(bool rotate, double c, double s, uint16_t xa, uint16_t xb,
                                                 uint16_t& ya, uint16_t& yb) {
  if (rotate) {
    const double x0 = (double)__uint_as_float((uint32_t)xa << 16);
    const double x1 = (double)__uint_as_float((uint32_t)xb << 16);
    ya = (uint16_t)f64_to_bf16_bits(x0 * c - x1 * s);
    yb = (uint16_t)f64_to_bf16_bits(x0 * s + x1 * c);
  } else {
    ya = xa;
    yb = xb;
  }
}

}  // namespace kvattn

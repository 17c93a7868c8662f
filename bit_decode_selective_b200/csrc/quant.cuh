// quant.cuh -- the nested quantiser of one group, shared by the weight and KV
// packing kernels.
//
// "StrataFlux -- Selective precision streaming -- What does it mean?",
// nested-quantization paragraph: the resident b-bit code names a bin and the
// r fetched bits split it into 2^r equal parts.  Step s = fp16((hi-lo)/(2^b-1))
// and offset m = fp16(lo), each rounded once from fp64; the (b+r)-bit nested
// code is Q = clamp(floor((u + 1/2) * 2^r)) with u = (w - m)/s, base code
// Q >> r and refinement Q & (2^r - 1).  Every fp64 operation is explicitly
// rounded (no contraction) so the codes are bit-exact with the definition.
#pragma once

#include "common.cuh"

namespace sf {

struct Grid16 {
  uint16_t s16, m16;
  double S, M;
};

__device__ __forceinline__ Grid16 group_grid(double lo, double hi, int b) {
  Grid16 g;
  double step = __ddiv_rn(__dsub_rn(hi, lo), (double)((1 << b) - 1));
  g.s16 = __half_as_ushort(__double2half(step));  // one rounding, nearest-even
  g.m16 = __half_as_ushort(__double2half(lo));
  g.S = h2d(g.s16);
  g.M = h2d(g.m16);
  return g;
}

// (b+r)-bit nested code Q of one value: floor((u + 1/2) * 2^r), clamped.
__device__ __forceinline__ int nested_code(double w, const Grid16& g, int r, int qmax) {
  if (g.S == 0.0) return 0;
  double u = __ddiv_rn(__dsub_rn(w, g.M), g.S);
  double t = __dadd_rn(u, 0.5);
  double f = floor(__dmul_rn(t, (double)(1 << r)));
  f = fmin(fmax(f, 0.0), (double)qmax);
  return (int)f;
}

}  // namespace sf

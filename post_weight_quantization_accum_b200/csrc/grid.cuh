// The low-bit grid shared by GPTQ and round-to-nearest (GPTQ knowledge note,
// "Common Confusions": both use one fixed low-bit grid; encyclopedia "GPTQ",
// "Technical Approach": one scale per group).
//
// Asymmetric min-max grid widened to include 0; an all-zero group uses [0, 1].
// Every operation is one IEEE float32 operation with round-to-nearest-even,
// written with explicit _rn intrinsics so that no multiply-add is contracted:
// the same column gives bit-identical codes, scales and zeros on every
// implementation that follows these steps in float32.
#pragma once

#include <cuda_runtime.h>

namespace gptq {

struct GridParams {
  float scale;
  float zero;
};

// scale = (xmax - xmin) / maxq, zero = rint(-xmin / scale) over a group whose
// raw minimum and maximum are xmin_raw, xmax_raw.
__device__ __forceinline__ GridParams grid_params(float xmin_raw, float xmax_raw, float maxq) {
  float xmin = fminf(xmin_raw, 0.0f);
  float xmax = fmaxf(xmax_raw, 0.0f);
  if (xmin == 0.0f && xmax == 0.0f) xmax = 1.0f;
  GridParams p;
  p.scale = __fdiv_rn(__fsub_rn(xmax, xmin), maxq);
  p.zero = rintf(__fdiv_rn(-xmin, p.scale));
  return p;
}

// code = clamp(rint(w / scale) + zero, 0, maxq), as a float holding an integer.
__device__ __forceinline__ float grid_code(float w, GridParams p, float maxq) {
  float q = __fadd_rn(rintf(__fdiv_rn(w, p.scale)), p.zero);
  return fminf(fmaxf(q, 0.0f), maxq);
}

// grid_code with the division replaced by a product with rcp = 1 / scale
// (correctly rounded), and the quotient formed only where that could change
// the code.  rcp and the product each round once, so t = w * rcp lies within
// 3 * 2^-24 * |w / scale| of the correctly rounded quotient; rint(t) is the
// quotient's rint unless a half-integer lies within that distance of t.  The
// test below uses 2^-21 * |t| and also sends |t| >= 2^22 and non-finite t
// (a subnormal scale) to the exact quotient, so the code is grid_code's.
__device__ __forceinline__ float grid_code_rcp(float w, GridParams p, float rcp, float maxq) {
  const float t = __fmul_rn(w, rcp);
  float k = rintf(t);
  const float to_half = fabsf(__fsub_rn(fabsf(__fsub_rn(t, k)), 0.5f));
  if (!(fabsf(t) < 4194304.0f) || to_half <= 4.76837158e-7f * fabsf(t)) k = rintf(__fdiv_rn(w, p.scale));
  const float q = __fadd_rn(k, p.zero);
  return fminf(fmaxf(q, 0.0f), maxq);
}

// Dequantized value scale * (code - zero).
__device__ __forceinline__ float grid_deq(float code, GridParams p) {
  return __fmul_rn(p.scale, __fsub_rn(code, p.zero));
}

}  // namespace gptq

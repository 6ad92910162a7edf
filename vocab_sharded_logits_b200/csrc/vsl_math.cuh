// vsl_math.cuh - float arithmetic the sampler's kernels share with the test
// library's checks.
#pragma once

#include <cuda_runtime.h>

namespace vsl {

// x = fl(l / T), the IEEE round-to-nearest quotient, for T > 0, by Markstein's
// method (P. Markstein, "Computation of elementary functions on the IBM
// RISC System/6000 processor", IBM J. Res. Develop. 34(1), 1990): with
// y = RN(1 / T), q0 = RN(l y) is within one ulp of l / T, the residual
// r = l - q0 T is exact in one fused multiply-add, and RN(q0 + r y) is the
// correctly rounded quotient, provided no step overflows.  y is passed in so
// that a loop computes it once.  A zero l gives +0 (the sampler reads -0 as
// +0 everywhere).
//
// scale_x_fast is for a row whose T lies in [2^-20, 2^20] and whose nonzero
// finite logits all satisfy 2^-60 <= |l| <= 2^100 (fast_division_ok): there
// every step stays in float32's normal range.  The test library compares it
// bit for bit with __fdiv_rn over every float32 l in that domain for
// temperatures across that range.  scale_x is the IEEE division itself, for
// any l and T.
__device__ __forceinline__ float scale_x_fast(float l, float T, float y) {
  const float q0 = __fmul_rn(l, y);
  const float r = __fmaf_rn(-q0, T, l);
  return __fmaf_rn(r, y, q0);
}
__device__ __forceinline__ bool fast_division_ok(float T, float max_abs_l, float min_nonzero_abs_l) {
  return T >= 0x1p-20f && T <= 0x1p20f && max_abs_l <= 0x1p100f && min_nonzero_abs_l >= 0x1p-60f;
}
__device__ __forceinline__ float scale_x(float l, float T) { return __fdiv_rn(l, T); }
// The IEEE quotient out of line: the other side of a per-row choice of
// scale_x_fast, so that the loop's common path stays short.
static __device__ __noinline__ float div_ieee(float l, float T) { return __fdiv_rn(l, T); }

}  // namespace vsl

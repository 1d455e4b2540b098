// gdn_silu.cuh -- SiLU for the kernels whose outputs are rounded to bf16.
#pragma once
#include "gdn_common.cuh"

namespace gdn {

// SiLU through the identity sigmoid(x) = (1 + tanh(x / 2)) / 2, so silu(x) =
// h + h tanh(h) with h = x / 2: one tanh.approx.f32, a single MUFU operation,
// where silu() of gdn_common.cuh takes two (ex2 and the reciprocal).  With the
// instruction's relative error bound of 2^-11 the result is off by at most
// |h tanh(h)| 2^-11 <= |x| 2^-12: under the bf16 rounding of the output for
// x > 0, and for x < 0 (where silu is small) an absolute error of that size,
// far inside the bf16 path's tolerance relative to the largest output.  The
// kernels with bf16 outputs use it (the prefill conv was bound by the MUFU
// pipe: 0.494 -> 0.406 ms on the long prefill); fp32 outputs keep silu().
__device__ __forceinline__ float silu_tanh(float x) {
  const float h = 0.5f * x;
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(h));
  return fmaf(h, t, h);
}
template <typename IO> __device__ __forceinline__ float silu_io(float x) { return silu(x); }
template <> __device__ __forceinline__ float silu_io<__nv_bfloat16>(float x) { return silu_tanh(x); }

}  // namespace gdn

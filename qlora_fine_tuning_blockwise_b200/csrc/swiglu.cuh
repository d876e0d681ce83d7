// SwiGLU of one element, in fp32 operations that are never contracted into fused multiply-adds, so the
// standalone kernels and the GEMM epilogues that fuse it give the same bits.  The exponential and the
// divisions are CUDA's fast intrinsics (__expf, __fdividef: a few ulp, far inside the bf16 rounding of every
// result); for g below about -88 the exponential overflows to +inf and silu(g), sigma(g) come out as 0.
// ("Inside Unsloth: How the Fastest LLM Fine-Tuning Library Works", section "What You'll Learn", item "Triton
// Kernel Internals": the fused SwiGLU forward and backward).
//   h = silu(g) * up, silu(g) = g / (1 + e^-g);
//   with s = 1 / (1 + e^-g): dg = dh * up * s (1 + g (1 - s)), dup = dh * (g s).
#pragma once

#include <cuda_runtime.h>

namespace qlora {

__device__ __forceinline__ float swiglu_h(float g, float u) {
  return __fmul_rn(__fdividef(g, __fadd_rn(1.0f, __expf(-g))), u);
}

__device__ __forceinline__ void swiglu_grads(float d, float g, float u, float& dg, float& du) {
  const float s = __fdividef(1.0f, __fadd_rn(1.0f, __expf(-g)));
  const float ds = __fmul_rn(s, __fadd_rn(1.0f, __fmul_rn(g, __fsub_rn(1.0f, s))));
  dg = __fmul_rn(__fmul_rn(d, u), ds);
  du = __fmul_rn(d, __fmul_rn(g, s));
}

// The interleaved layout of a stacked gate/up projection [2F, D] (F % 16 == 0): within every 32 consecutive rows,
// 16 gate rows then the 16 up rows of the same features, so that one warp's lanes l and l + 16 hold the two
// halves of one feature.  Row (column of its output) of gate feature f, and of up feature f:
__host__ __device__ __forceinline__ long long gate_pos(long long f) { return (f >> 4) * 32 + (f & 15); }
__host__ __device__ __forceinline__ long long up_pos(long long f) { return gate_pos(f) + 16; }

}  // namespace qlora

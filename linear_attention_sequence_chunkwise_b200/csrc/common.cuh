// common.cuh -- device helpers shared by the retention kernels of libretnet.so.
//
// Notation follows "阅读笔记：RetNet" (mzeromiko blog): gamma is a head's decay, theta the
// xPos frequencies (§2.3), p an absolute 0-based token position.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "retnet.h"

namespace retnet {

constexpr int kMaxHeads = RETNET_MAX_HEADS;
constexpr int kMaxPairs = RETNET_MAX_DK / 2;

// Per-head and per-pair parameters, passed by value as a launch parameter.
struct HeadParams {
  float gamma[kMaxHeads];  // decay per head, in (0, 1)
  float log2g[kMaxHeads];  // log2(gamma), rounded from a double on the host
  float theta[kMaxPairs];  // xPos frequency per interleaved pair (2j, 2j+1)
};

struct Dims {
  int64_t batch, seqlen, heads, d_k, d_v;
};

__device__ __forceinline__ float load_f(const float* p, int64_t i) { return p[i]; }
__device__ __forceinline__ float load_f(const __nv_bfloat16* p, int64_t i) { return __bfloat162float(p[i]); }
__device__ __forceinline__ void store_f(float* p, int64_t i, float x) { p[i] = x; }
__device__ __forceinline__ void store_f(__nv_bfloat16* p, int64_t i, float x) { p[i] = __float2bfloat16_rn(x); }

// gamma^n for an integer n >= 0, from log2(gamma); relative error a few fp32 ulps for the
// exponents used here (n * |log2 gamma| stays small where the power is not negligible).
__device__ __forceinline__ float decay_pow(float log2g, int n) { return exp2f(static_cast<float>(n) * log2g); }

// cos/sin of the xPos angle p * theta.  The product and the reduction into [-pi, pi] are
// done in fp64 so that large positions keep full fp32 accuracy in the result.
__device__ __forceinline__ void xpos_sincos(int64_t p, float theta, float* s, float* c) {
  const double two_pi = 6.283185307179586476925286766559;
  double a = static_cast<double>(p) * static_cast<double>(theta);
  a -= two_pi * rint(a / two_pi);
  sincosf(static_cast<float>(a), s, c);
}

// Per-row output factor of the normalisations ("阅读笔记：RetNet" §三.3):
//   s / c_p,  s = 1/sqrt(d_k) with RETNET_F_SCALE_SQRT_D,
//   c_p = sqrt(sum_{j=0..p} gamma^j) = sqrt((1 - gamma^(p+1)) / (1 - gamma)) with RETNET_F_NORM_D.
// Evaluated in fp64 with expm1/log1p so that gamma close to 1 loses nothing to cancellation.
__device__ __forceinline__ float row_factor(float gamma, int d_k, int64_t p, uint32_t flags) {
  double f = 1.0;
  if (flags & RETNET_F_SCALE_SQRT_D) f /= sqrt(static_cast<double>(d_k));
  if (flags & RETNET_F_NORM_D) {
    double one_minus = 1.0 - static_cast<double>(gamma);
    double sum = -expm1(static_cast<double>(p + 1) * log1p(-one_minus)) / one_minus;
    f /= sqrt(sum);
  }
  return static_cast<float>(f);
}

}  // namespace retnet

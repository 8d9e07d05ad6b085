// msr_epilogue.cu -- MSR epilogue ("阅读笔记：RetNet" §三.2 Multi-Scale Retention):
//   Y = GroupNorm_h(Concat(head_1 .. head_h)),  out = swish(G) (.) Y.
// Groups are the heads: each (token, head) row of d_v values is normalised with its own
// biased mean and variance, eps inside the root, unit affine; swish(g) = g * sigmoid(g).
//
// HBM-bound (read y and g, write out).  One warp owns one row; each lane holds up to four
// 8-element groups of the row in registers (d_v <= 1024), so the row is read once, the
// mean and the centred variance come from two warp-shuffle reductions over registers, and
// the result is written once.  Accesses are 16-byte (bf16) or 32-byte (fp32) vectors.
#include "launch.h"

namespace retnet {
namespace {

constexpr int kWarpsPerBlock = 8;
constexpr int kMaxGroups = RETNET_MAX_DV / (8 * 32);  // 8-element groups per lane

__device__ __forceinline__ void load8(const float* p, float* x) {
  float4 a = *reinterpret_cast<const float4*>(p);
  float4 b = *reinterpret_cast<const float4*>(p + 4);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float* x) {
  uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void store8(float* p, const float* x) {
  *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(x[4], x[5], x[6], x[7]);
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float* x) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = u;
}

template <typename Tin, typename Tout>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    msr_epilogue_kernel(const Tin* __restrict__ y, const Tin* __restrict__ g, Tout* out, int64_t rows, int d_v,
                        float eps) {
  const int lane = threadIdx.x % 32;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kWarpsPerBlock + threadIdx.x / 32;
  if (row >= rows) return;
  const int groups = d_v / 8;
  const Tin* yr = y + row * d_v;
  const Tin* gr = g + row * d_v;
  float x[kMaxGroups][8];
  float sum = 0.f;
#pragma unroll
  for (int m = 0; m < kMaxGroups; ++m) {
    const int grp = lane + 32 * m;
    if (grp < groups) {
      load8(yr + grp * 8, x[m]);
#pragma unroll
      for (int e = 0; e < 8; ++e) sum += x[m][e];
    }
  }
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  const float mean = sum / static_cast<float>(d_v);
  float sq = 0.f;
#pragma unroll
  for (int m = 0; m < kMaxGroups; ++m) {
    const int grp = lane + 32 * m;
    if (grp < groups) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float c = x[m][e] - mean;
        sq = fmaf(c, c, sq);
      }
    }
  }
  for (int off = 16; off > 0; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
  const float inv = rsqrtf(sq / static_cast<float>(d_v) + eps);
#pragma unroll
  for (int m = 0; m < kMaxGroups; ++m) {
    const int grp = lane + 32 * m;
    if (grp < groups) {
      float gv[8], r[8];
      load8(gr + grp * 8, gv);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float sw = gv[e] / (1.f + expf(-gv[e]));  // swish(g) = g * sigmoid(g)
        r[e] = sw * ((x[m][e] - mean) * inv);
      }
      store8(out + row * d_v + grp * 8, r);
    }
  }
}

template <typename Tin, typename Tout>
cudaError_t launch_typed(const void* y, const void* g, void* out, int64_t rows, int d_v, float eps, cudaStream_t s) {
  const int64_t blocks = (rows + kWarpsPerBlock - 1) / kWarpsPerBlock;
  msr_epilogue_kernel<Tin, Tout><<<static_cast<unsigned>(blocks), kWarpsPerBlock * 32, 0, s>>>(
      static_cast<const Tin*>(y), static_cast<const Tin*>(g), static_cast<Tout*>(out), rows, d_v, eps);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_msr_epilogue(const void* y, const void* g, void* out, int64_t tokens, int64_t heads, int64_t d_v,
                                float eps, retnet_dtype_t in_dtype, retnet_dtype_t out_dtype, cudaStream_t s) {
  const int64_t rows = tokens * heads;
  if (rows == 0) return cudaSuccess;
  const int dv = static_cast<int>(d_v);
  if (in_dtype == RETNET_F32) {
    if (out_dtype == RETNET_F32) return launch_typed<float, float>(y, g, out, rows, dv, eps, s);
    return launch_typed<float, __nv_bfloat16>(y, g, out, rows, dv, eps, s);
  }
  if (out_dtype == RETNET_F32) return launch_typed<__nv_bfloat16, float>(y, g, out, rows, dv, eps, s);
  return launch_typed<__nv_bfloat16, __nv_bfloat16>(y, g, out, rows, dv, eps, s);
}

}  // namespace retnet

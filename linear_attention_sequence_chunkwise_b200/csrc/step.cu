// step.cu -- recurrent decode step ("阅读笔记：RetNet" §2.2 Recurrent Mode).
//
// For the token at absolute position p:  S <- gamma S + k'^T v (in place),  o = (q' S) * s / c_p,
// optionally divided by max(|s/c_p q'.z|, 1) with z <- gamma z + k' (§三.3), where q', k' are the
// xPos-rotated vectors.  The whole call is bound by HBM: the fp32 state (d_k x d_v per head) is
// read once and written once, everything else is a few KB.
//
// One CTA owns one (batch, head).  Its 8 warps split the d_k rows (warp w takes rows
// w, w+8, ...) and a warp's lanes cover 128 contiguous d_v columns with one 16-byte access
// each, so every state access is a fully coalesced 512-byte row segment.  Four rows are
// loaded before any is used to keep 64 bytes per thread in flight; the q'S partial sums of
// the 8 warps are combined through shared memory.  The state is accessed with streaming
// (evict-first) hints: it is far larger than L2 and is not touched again in this call.
#include "launch.h"

namespace retnet {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kColsPerPass = 128;  // 32 lanes x 4 floats
constexpr int kRowUnroll = 4;

template <typename Tin, typename Tout>
struct StepArgs {
  const Tin* q;
  const Tin* k;
  const Tin* v;
  Tout* o;
  float* state;
  float* z;
  int d_k, d_v;
  int64_t heads;
  int64_t pos;
  uint32_t flags;
};

template <typename Tin, typename Tout>
__global__ void __launch_bounds__(kThreads) step_kernel(StepArgs<Tin, Tout> a, HeadParams hp) {
  extern __shared__ float sm[];
  const int dk = a.d_k, dv = a.d_v;
  float* qs = sm;                   // [dk]   rotated q
  float* ks = qs + dk;              // [dk]   rotated k
  float* red = ks + dk;             // [kWarps][kColsPerPass] partial q'S
  float* scal = red + kWarps * kColsPerPass;  // [2]: output scale, (unused)
  const int64_t bh = blockIdx.x;
  const int h = static_cast<int>(bh % a.heads);
  const float gamma = hp.gamma[h];
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const bool xpos = (a.flags & RETNET_F_XPOS) != 0;

  // Rotated q, k of this token (§2.3 Theta applied at position p).
  for (int j = tid; j < dk / 2; j += kThreads) {
    float q0 = load_f(a.q, bh * dk + 2 * j), q1 = load_f(a.q, bh * dk + 2 * j + 1);
    float k0 = load_f(a.k, bh * dk + 2 * j), k1 = load_f(a.k, bh * dk + 2 * j + 1);
    if (xpos) {
      float s, c;
      xpos_sincos(a.pos, hp.theta[j], &s, &c);
      float t;
      t = q0 * c - q1 * s; q1 = q0 * s + q1 * c; q0 = t;
      t = k0 * c - k1 * s; k1 = k0 * s + k1 * c; k0 = t;
    }
    qs[2 * j] = q0; qs[2 * j + 1] = q1;
    ks[2 * j] = k0; ks[2 * j + 1] = k1;
  }
  if ((dk & 1) && tid == 0) {
    qs[dk - 1] = load_f(a.q, bh * dk + dk - 1);
    ks[dk - 1] = load_f(a.k, bh * dk + dk - 1);
  }
  __syncthreads();

  // Output scale s / c_p / max(|s/c_p q'.z|, 1); z <- gamma z + k' first (update, then read).
  if (warp == 0) {
    float f = row_factor(gamma, dk, a.pos, a.flags);
    float den = 1.f;
    if (a.flags & RETNET_F_NORM_R) {
      float qz = 0.f;
      for (int i = lane; i < dk; i += 32) {
        float zi = fmaf(gamma, a.z[bh * dk + i], ks[i]);
        a.z[bh * dk + i] = zi;
        qz = fmaf(qs[i], zi, qz);
      }
      for (int off = 16; off > 0; off >>= 1) qz += __shfl_xor_sync(0xffffffffu, qz, off);
      den = fmaxf(fabsf(f * qz), 1.f);
    }
    if (lane == 0) scal[0] = f / den;
  }

  float* S = a.state + bh * static_cast<int64_t>(dk) * dv;
  const bool vec = (dv % 4) == 0;
  for (int c0 = 0; c0 < dv; c0 += kColsPerPass) {
    const int col = c0 + lane * 4;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    float vv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int m = 0; m < 4; ++m)
      if (col + m < dv) vv[m] = load_f(a.v, bh * dv + col + m);
    if (vec && col < dv) {
      int i = warp;
      for (; i + (kRowUnroll - 1) * kWarps < dk; i += kRowUnroll * kWarps) {
        float4 sv[kRowUnroll];
#pragma unroll
        for (int u = 0; u < kRowUnroll; ++u)
          sv[u] = __ldcs(reinterpret_cast<const float4*>(S + static_cast<int64_t>(i + u * kWarps) * dv + col));
#pragma unroll
        for (int u = 0; u < kRowUnroll; ++u) {
          const int r = i + u * kWarps;
          const float kr = ks[r], qr = qs[r];
          float4 x = sv[u];
          x.x = fmaf(gamma, x.x, kr * vv[0]);
          x.y = fmaf(gamma, x.y, kr * vv[1]);
          x.z = fmaf(gamma, x.z, kr * vv[2]);
          x.w = fmaf(gamma, x.w, kr * vv[3]);
          __stcs(reinterpret_cast<float4*>(S + static_cast<int64_t>(r) * dv + col), x);
          acc[0] = fmaf(qr, x.x, acc[0]);
          acc[1] = fmaf(qr, x.y, acc[1]);
          acc[2] = fmaf(qr, x.z, acc[2]);
          acc[3] = fmaf(qr, x.w, acc[3]);
        }
      }
      for (; i < dk; i += kWarps) {
        float4 x = __ldcs(reinterpret_cast<const float4*>(S + static_cast<int64_t>(i) * dv + col));
        const float kr = ks[i], qr = qs[i];
        x.x = fmaf(gamma, x.x, kr * vv[0]);
        x.y = fmaf(gamma, x.y, kr * vv[1]);
        x.z = fmaf(gamma, x.z, kr * vv[2]);
        x.w = fmaf(gamma, x.w, kr * vv[3]);
        __stcs(reinterpret_cast<float4*>(S + static_cast<int64_t>(i) * dv + col), x);
        acc[0] = fmaf(qr, x.x, acc[0]);
        acc[1] = fmaf(qr, x.y, acc[1]);
        acc[2] = fmaf(qr, x.z, acc[2]);
        acc[3] = fmaf(qr, x.w, acc[3]);
      }
    } else if (!vec) {
      for (int i = warp; i < dk; i += kWarps) {
        const float kr = ks[i], qr = qs[i];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          if (col + m < dv) {
            float x = fmaf(gamma, S[static_cast<int64_t>(i) * dv + col + m], kr * vv[m]);
            S[static_cast<int64_t>(i) * dv + col + m] = x;
            acc[m] = fmaf(qr, x, acc[m]);
          }
        }
      }
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) red[warp * kColsPerPass + lane * 4 + m] = acc[m];
    __syncthreads();
    if (tid < kColsPerPass && c0 + tid < dv) {
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) s += red[w * kColsPerPass + tid];
      store_f(a.o, bh * dv + c0 + tid, s * scal[0]);
    }
    __syncthreads();
  }
}

template <typename Tin, typename Tout>
cudaError_t launch_typed(const StepCall& c, const HeadParams& hp, cudaStream_t s) {
  StepArgs<Tin, Tout> a;
  a.q = static_cast<const Tin*>(c.q);
  a.k = static_cast<const Tin*>(c.k);
  a.v = static_cast<const Tin*>(c.v);
  a.o = static_cast<Tout*>(c.o);
  a.state = c.state;
  a.z = c.z;
  a.d_k = static_cast<int>(c.d_k);
  a.d_v = static_cast<int>(c.d_v);
  a.heads = c.heads;
  a.pos = c.pos;
  a.flags = c.flags;
  // at most 4 * (2 * 512 + 8 * 128 + 2) = 8200 bytes (d_k <= RETNET_MAX_DK): within the default
  // 48 KB of dynamic shared memory, so no per-launch attribute call is needed
  const size_t smem = sizeof(float) * (size_t)(2 * c.d_k + kWarps * kColsPerPass + 2);
  static_assert(sizeof(float) * (2 * RETNET_MAX_DK + kWarps * kColsPerPass + 2) <= 48 * 1024, "step smem");
  const int64_t blocks = c.batch * c.heads;
  step_kernel<Tin, Tout><<<static_cast<unsigned>(blocks), kThreads, smem, s>>>(a, hp);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_step(const StepCall& c, const HeadParams& hp, cudaStream_t s) {
  if (c.in_dtype == RETNET_F32) {
    if (c.out_dtype == RETNET_F32) return launch_typed<float, float>(c, hp, s);
    return launch_typed<float, __nv_bfloat16>(c, hp, s);
  }
  if (c.out_dtype == RETNET_F32) return launch_typed<__nv_bfloat16, float>(c, hp, s);
  return launch_typed<__nv_bfloat16, __nv_bfloat16>(c, hp, s);
}

}  // namespace retnet

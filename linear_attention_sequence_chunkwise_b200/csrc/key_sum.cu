// key_sum.cu -- the R~ normalisation of "阅读笔记：RetNet" §三.3 for the tensor-core chunkwise
// kernel.  R~ divides output row n by max(|sum_m score_nm|, 1), the decayed, scaled scores of
// that row summed over every earlier key:
//   sum_m score_nm = f_n * q~_n . z_n,   z_n = gamma z_{n-1} + k~_n   (z_{-1} = z_in or 0),
// with q~, k~ the xPos-rotated rows and f_n = s / c_n the row factor of the other two
// normalisations.  z is the chunkwise state of §2.4 with V = 1 (a d_k vector per (batch, head)),
// so a pass over the keys alone gives every row's divisor; the tensor-core kernel folds
// 1 / max(|.|, 1) into its row factor.
//
// Parallel over the sequence as well: (batch, head) x segments of Ls tokens (a multiple of 32).
// z's recurrence is associative (a stretch of n tokens with own end value E moves any z to
// gamma^n z + E), so a first pass writes each segment's E from a zero start (keys only) and a
// second pass starts segment s from z_in carried over E_0 .. E_{s-1}, then produces the row
// factors.  One thread per rotary pair (2j, 2j+1) of d_k.  Tokens go in batches of 32: the
// next batch's q and k pairs are loaded while the current one is summed; the rotation of a
// batch is a complex recurrence from an angle reduced in fp64 at the batch's first position;
// the per-token dot products are reduced over the pairs through shared memory.  Bound by the
// reads of k (twice) and q.
#include <algorithm>

#include "launch.h"

namespace retnet {
namespace {

constexpr int kBatch = 32;
constexpr int kMaxPairsKS = 128;  // d_k <= 256

__device__ __forceinline__ uint32_t ld_pair(const __nv_bfloat16* p) { return __ldg(reinterpret_cast<const unsigned int*>(p)); }
__device__ __forceinline__ float lo_bf16(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_bf16(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// PASS1: E[bh][seg][d_k] = the segment's own end value of z.  Else: row factors of the
// segment's tokens into rden (and z_out from the last segment).
template <bool PASS1>
__global__ void __launch_bounds__(kMaxPairsKS) key_sum_kernel(const __nv_bfloat16* __restrict__ q,
                                                              const __nv_bfloat16* __restrict__ k,
                                                              const float* z_in, float* z_out, float* seg_end,
                                                              float* __restrict__ rden, int L, int heads, int d_k,
                                                              int seg_len, int64_t pos0, uint32_t flags,
                                                              HeadParams hp) {
  __shared__ float red[kBatch][kMaxPairsKS + 1];
  const int bh = blockIdx.x, seg = blockIdx.y, n_seg = gridDim.y, b = bh / heads, h = bh % heads;
  const int j = threadIdx.x, np = d_k / 2;
  const int t_lo = seg * seg_len, t_hi = min(L, t_lo + seg_len);
  const float g = hp.gamma[h];
  const bool xpos = (flags & RETNET_F_XPOS) != 0;
  const float th = xpos ? hp.theta[j] : 0.f;
  float* e_base = seg_end + static_cast<int64_t>(bh) * n_seg * d_k + 2 * j;
  float z0 = 0.f, z1 = 0.f;
  if (!PASS1) {
    if (z_in) {
      z0 = z_in[static_cast<int64_t>(bh) * d_k + 2 * j];
      z1 = z_in[static_cast<int64_t>(bh) * d_k + 2 * j + 1];
    }
    const float gl = exp2f(static_cast<float>(seg_len) * hp.log2g[h]);  // every earlier segment is full
    for (int s = 0; s < seg; ++s) {
      z0 = fmaf(gl, z0, e_base[s * d_k]);
      z1 = fmaf(gl, z1, e_base[s * d_k + 1]);
    }
  }
  float dc = 1.f, ds = 0.f;  // rotation by theta_j: one position step
  if (xpos) xpos_sincos(1, th, &ds, &dc);
  const int64_t row_stride = static_cast<int64_t>(heads) * d_k;
  const __nv_bfloat16* qp = q + (static_cast<int64_t>(b) * L * heads + h) * d_k + 2 * j;
  const __nv_bfloat16* kp = k + (static_cast<int64_t>(b) * L * heads + h) * d_k + 2 * j;
  uint32_t qv[kBatch], kv[kBatch];
  auto load = [&](int t0) {
#pragma unroll
    for (int s = 0; s < kBatch; ++s) {
      if (t0 + s < t_hi) {
        if (!PASS1) qv[s] = ld_pair(qp + (t0 + s) * row_stride);
        kv[s] = ld_pair(kp + (t0 + s) * row_stride);
      }
    }
  };
  load(t_lo);
  for (int t0 = t_lo; t0 < t_hi; t0 += kBatch) {
    uint32_t qc[kBatch], kc[kBatch];
#pragma unroll
    for (int s = 0; s < kBatch; ++s) {
      if (!PASS1) qc[s] = qv[s];
      kc[s] = kv[s];
    }
    if (t0 + kBatch < t_hi) load(t0 + kBatch);  // next batch in flight during this one
    float c = 1.f, sn = 0.f;
    if (xpos) xpos_sincos(pos0 + t0, th, &sn, &c);
    const int nt = min(kBatch, t_hi - t0);
#pragma unroll
    for (int s = 0; s < kBatch; ++s) {
      if (s < nt) {
        const float k0 = lo_bf16(kc[s]), k1 = hi_bf16(kc[s]);
        z0 = fmaf(g, z0, k0 * c - k1 * sn);
        z1 = fmaf(g, z1, fmaf(k0, sn, k1 * c));
        if (!PASS1) {
          const float q0 = lo_bf16(qc[s]), q1 = hi_bf16(qc[s]);
          red[s][j] = fmaf(q0 * c - q1 * sn, z0, fmaf(q0, sn, q1 * c) * z1);
        }
        const float nc = c * dc - sn * ds;
        sn = fmaf(c, ds, sn * dc);
        c = nc;
      }
    }
    if (!PASS1) {
      __syncthreads();
      if (j < nt) {
        float acc = 0.f;
        for (int i = 0; i < np; ++i) acc += red[j][i];
        const float f = row_factor(g, d_k, pos0 + t0 + j, flags);
        rden[(static_cast<int64_t>(b) * L + t0 + j) * heads + h] = 1.f / fmaxf(fabsf(f * acc), 1.f);
      }
      __syncthreads();
    }
  }
  if (PASS1) {
    e_base[seg * d_k] = z0;
    e_base[seg * d_k + 1] = z1;
  } else if (z_out && seg == n_seg - 1) {
    z_out[static_cast<int64_t>(bh) * d_k + 2 * j] = z0;
    z_out[static_cast<int64_t>(bh) * d_k + 2 * j + 1] = z1;
  }
}

}  // namespace

int key_sum_segments(const Dims& d) {
  // about 8 CTAs an SM's worth of (batch, head, segment) CTAs, segments of >= 64 tokens
  const int64_t bh = d.batch * d.heads;
  int64_t n = (148 * 8 + bh - 1) / bh;
  n = std::min<int64_t>(n, (d.seqlen + 63) / 64);
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(n, kMaxKeySumSegments)));
}

int key_sum_seg_len(const Dims& d, int n_seg) {
  const int64_t per = (d.seqlen + n_seg - 1) / n_seg;
  return static_cast<int>((per + kBatch - 1) / kBatch * kBatch);
}

cudaError_t launch_key_sum(const RetentionCall& c, const HeadParams& hp, cudaStream_t s) {
  const Dims& d = c.dims;
  if (d.d_k < 2 * kBatch || d.d_k > 2 * kMaxPairsKS || d.d_k % 2 != 0 || !c.rden || !c.rden_seg) return cudaErrorInvalidValue;
  int n_seg = key_sum_segments(d);
  const int seg_len = key_sum_seg_len(d, n_seg);
  n_seg = static_cast<int>((d.seqlen + seg_len - 1) / seg_len);  // no empty segment
  const dim3 grid(static_cast<unsigned>(d.batch * d.heads), static_cast<unsigned>(n_seg));
  const unsigned threads = static_cast<unsigned>(d.d_k / 2);
  const auto* q = static_cast<const __nv_bfloat16*>(c.q);
  const auto* k = static_cast<const __nv_bfloat16*>(c.k);
  if (n_seg > 1) {
    key_sum_kernel<true><<<grid, threads, 0, s>>>(q, k, nullptr, nullptr, c.rden_seg, nullptr,
                                                  static_cast<int>(d.seqlen), static_cast<int>(d.heads),
                                                  static_cast<int>(d.d_k), seg_len, c.pos0, c.flags, hp);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  key_sum_kernel<false><<<grid, threads, 0, s>>>(q, k, c.z_in, c.z_out, c.rden_seg, c.rden,
                                                 static_cast<int>(d.seqlen), static_cast<int>(d.heads),
                                                 static_cast<int>(d.d_k), seg_len, c.pos0, c.flags, hp);
  return cudaGetLastError();
}

int key_sum_launches(const Dims& d) {
  const int n_seg = key_sum_segments(d);
  const int seg_len = key_sum_seg_len(d, n_seg);
  return (d.seqlen + seg_len - 1) / seg_len > 1 ? 2 : 1;
}

}  // namespace retnet

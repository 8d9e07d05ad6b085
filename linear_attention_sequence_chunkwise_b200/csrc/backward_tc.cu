// backward_tc.cu -- the gradient of backward.cu on the tensor cores, as runs of the
// tcgen05 chunkwise forward kernel.  Each gradient sum has the shape of a retention output:
// a decayed, causal (or, read backwards, anti-causal) sum of value rows weighted by query .
// key products ("阅读笔记：RetNet" §2.3, §2.4; notation of backward.cu):
//   dq~_n / f_n = sum_{m<=n} g^(n-m) (dO_n . v_m) k~_m + g^(n+1) dO_n S0^T
//        -> retention with query dO, key v, value k~, start state S0^T (forward order);
//   dk~_m = sum_{n>=m} g^(n-m) (v_m . dO_n) (f_n q~_n)
//        -> retention over the reversed sequence (t' = L-1-t): query v, key dO, value f q~;
//   dv_m  = sum_{n>=m} g^(n-m) (q~_n . k~_m) (f_n dO_n)
//        -> reversed: query k, key q, value f dO, with the kernel's own xPos rotation at the
//           reversed positions and theta negated (the score of query t'_m and key t'_n turns
//           by (t'_n - t'_m)(-theta) = (n - m) theta, which is q~_n . k~_m);
//   dS0   = sum_n g^(n+1) (f_n q~_n)^T dO_n  (a plain reduction over the sequence).
// A prep kernel writes the operands (rotations, row factors, reversal) in bf16: exact copies
// for q, k, v, dO; k~, f q~ and f dO, which are not bf16 numbers, as two parts hi + lo (hi the
// rounded value, lo the rounded remainder, together good to about 2^-17) side by side in a
// value row of twice the width (the runs are linear in the value, so one run gives both
// parts' outputs, sharing its scores).  A post kernel adds the two halves of each output row,
// scales dq by f, turns dq and dk back (R^T) and undoes the reversal of dk and dv.
#include <algorithm>

#include "launch.h"

namespace retnet {
namespace {

__device__ __forceinline__ __nv_bfloat16 to_bf16(float x) { return __float2bfloat16_rn(x); }

// Row factor s / c_p of §三.3 in fp32 (relative error ~1e-7, far below the hi + lo split's
// 2^-17): s = 1/sqrt(d_k), c_p^2 = (1 - gamma^(p+1)) / (1 - gamma) by expm1 / log1p.
__device__ __forceinline__ float row_f(float gamma, int d_k, int64_t p, uint32_t flags) {
  float f = (flags & RETNET_F_SCALE_SQRT_D) ? rsqrtf(static_cast<float>(d_k)) : 1.f;
  if (flags & RETNET_F_NORM_D) {
    const float om = 1.f - gamma;
    f *= rsqrtf(-expm1f(static_cast<float>(p + 1) * log1pf(-om)) / om);
  }
  return f;
}


// x as bf16 hi (at i) + lo (at i + w): lo is the rounded remainder.
__device__ __forceinline__ void split_store(__nv_bfloat16* p, int64_t i, int w, float x) {
  const __nv_bfloat16 a = to_bf16(x);
  p[i] = a;
  p[i + w] = to_bf16(x - __bfloat162float(a));
}

// The elementwise kernels run one CTA per token (b, t): the rotation of pair j is the same for
// every head, and each head's row factor is computed once, into shared memory.
__device__ __forceinline__ void row_factors(float* sf, int heads, int d_k, int64_t p, uint32_t flags,
                                            const HeadParams& hp) {
  for (int h = threadIdx.x; h < heads; h += blockDim.x) sf[h] = row_f(hp.gamma[h], d_k, p, flags);
  __syncthreads();
}

// Token (b, t): k~ (forward order) and f q~ (reversed) as hi | lo rows of width 2 d_k; q, k
// copied reversed.
__global__ void __launch_bounds__(128) bwd_tc_prep_qk(const __nv_bfloat16* __restrict__ q,
                                                      const __nv_bfloat16* __restrict__ k,
                                                      __nv_bfloat16* __restrict__ ktw, __nv_bfloat16* __restrict__ qR,
                                                      __nv_bfloat16* __restrict__ kR, __nv_bfloat16* __restrict__ fqRw,
                                                      int L, int heads, int d_k, int64_t pos0, uint32_t flags,
                                                      HeadParams hp) {
  __shared__ float sf[RETNET_MAX_HEADS];
  const int64_t bt = blockIdx.x;
  const int t = static_cast<int>(bt % L);
  const int64_t rbt = bt - t + (L - 1 - t);  // the same b at t' = L-1-t
  row_factors(sf, heads, d_k, pos0 + t, flags, hp);
  const bool xpos = (flags & RETNET_F_XPOS) != 0;
  for (int j = threadIdx.x; j < d_k / 2; j += blockDim.x) {
    float c = 1.f, s = 0.f;
    if (xpos) xpos_sincos(pos0 + t, hp.theta[j], &s, &c);
    for (int h = 0; h < heads; ++h) {
      const int64_t row = bt * heads + h, rrow = rbt * heads + h;
      const int64_t o = row * d_k + 2 * j, ro = rrow * d_k + 2 * j;
      const int64_t ow = row * 2 * d_k + 2 * j, row_w = rrow * 2 * d_k + 2 * j;
      const __nv_bfloat162 q2 = *reinterpret_cast<const __nv_bfloat162*>(q + o);
      const __nv_bfloat162 k2 = *reinterpret_cast<const __nv_bfloat162*>(k + o);
      const float2 qf = __bfloat1622float2(q2), kf = __bfloat1622float2(k2);
      *reinterpret_cast<__nv_bfloat162*>(qR + ro) = q2;
      *reinterpret_cast<__nv_bfloat162*>(kR + ro) = k2;
      split_store(ktw, ow, d_k, kf.x * c - kf.y * s);
      split_store(ktw, ow + 1, d_k, kf.x * s + kf.y * c);
      const float f = sf[h];
      split_store(fqRw, row_w, d_k, f * (qf.x * c - qf.y * s));
      split_store(fqRw, row_w + 1, d_k, f * (qf.x * s + qf.y * c));
    }
  }
}

// Token (b, t): v and dO copied reversed; f dO reversed as hi | lo rows of width 2 d_v.
__global__ void __launch_bounds__(128) bwd_tc_prep_v(const __nv_bfloat16* __restrict__ v,
                                                     const __nv_bfloat16* __restrict__ dout,
                                                     __nv_bfloat16* __restrict__ vR, __nv_bfloat16* __restrict__ doR,
                                                     __nv_bfloat16* __restrict__ fdoRw, int L, int heads, int d_k,
                                                     int d_v, int64_t pos0, uint32_t flags, HeadParams hp) {
  __shared__ float sf[RETNET_MAX_HEADS];
  const int64_t bt = blockIdx.x;
  const int t = static_cast<int>(bt % L);
  const int64_t rbt = bt - t + (L - 1 - t);
  row_factors(sf, heads, d_k, pos0 + t, flags, hp);
  const int half = d_v / 2;
  for (int e = threadIdx.x; e < heads * half; e += blockDim.x) {
    const int h = e / half, j = 2 * (e % half);
    const int64_t o = (bt * heads + h) * d_v + j, ro = (rbt * heads + h) * d_v + j;
    const int64_t row_w = (rbt * heads + h) * 2 * d_v + j;
    const __nv_bfloat162 v2 = *reinterpret_cast<const __nv_bfloat162*>(v + o);
    const __nv_bfloat162 d2 = *reinterpret_cast<const __nv_bfloat162*>(dout + o);
    *reinterpret_cast<__nv_bfloat162*>(vR + ro) = v2;
    *reinterpret_cast<__nv_bfloat162*>(doR + ro) = d2;
    const float2 df = __bfloat1622float2(d2);
    split_store(fdoRw, row_w, d_v, sf[h] * df.x);
    split_store(fdoRw, row_w + 1, d_v, sf[h] * df.y);
  }
}

// S0^T per (batch, head), as the start state of the wide dq run: [d_k][d_v] -> [d_v][2 d_k],
// the lo half zero (the state term enters once).
__global__ void bwd_tc_transpose(const float* __restrict__ s, float* __restrict__ st, int64_t n, int d_k, int d_v) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = i / (static_cast<int64_t>(d_k) * d_v);
    const int r = static_cast<int>(i % (static_cast<int64_t>(d_k) * d_v));
    const int a = r / d_v, bb = r % d_v;
    float* row = st + (m * d_v + bb) * 2 * d_k;
    row[a] = s[i];
    row[d_k + a] = 0.f;
  }
}

// Token (b, t): dq = R^T (f (hi + lo halves of the dq run's row)); dk = R^T (halves of the dk
// run's reversed row).
__global__ void __launch_bounds__(128) bwd_tc_post_qk(const float* __restrict__ oq, const float* __restrict__ okR,
                                                      float* __restrict__ dq, float* __restrict__ dk, int L, int heads,
                                                      int d_k, int64_t pos0, uint32_t flags, HeadParams hp) {
  __shared__ float sf[RETNET_MAX_HEADS];
  const int64_t bt = blockIdx.x;
  const int t = static_cast<int>(bt % L);
  const int64_t rbt = bt - t + (L - 1 - t);
  row_factors(sf, heads, d_k, pos0 + t, flags, hp);
  const bool xpos = (flags & RETNET_F_XPOS) != 0;
  for (int j = threadIdx.x; j < d_k / 2; j += blockDim.x) {
    float c = 1.f, s = 0.f;
    if (xpos) xpos_sincos(pos0 + t, hp.theta[j], &s, &c);
    for (int h = 0; h < heads; ++h) {
      const int64_t row = bt * heads + h, rrow = rbt * heads + h;
      const int64_t o = row * d_k + 2 * j;
      const float* a = oq + row * 2 * d_k + 2 * j;
      const float2 ah = *reinterpret_cast<const float2*>(a), al = *reinterpret_cast<const float2*>(a + d_k);
      const float y0 = sf[h] * (ah.x + al.x), y1 = sf[h] * (ah.y + al.y);
      *reinterpret_cast<float2*>(dq + o) = make_float2(fmaf(y0, c, y1 * s), fmaf(y1, c, -y0 * s));
      const float* z = okR + rrow * 2 * d_k + 2 * j;
      const float2 zh = *reinterpret_cast<const float2*>(z), zl = *reinterpret_cast<const float2*>(z + d_k);
      const float z0 = zh.x + zl.x, z1 = zh.y + zl.y;
      *reinterpret_cast<float2*>(dk + o) = make_float2(fmaf(z0, c, z1 * s), fmaf(z1, c, -z0 * s));
    }
  }
}

// Token (b, t): dv = hi + lo halves of the dv run's reversed row (float2 a thread).
__global__ void __launch_bounds__(128) bwd_tc_post_v(const float* __restrict__ ovR, float* __restrict__ dv, int L,
                                                     int heads, int d_v) {
  const int64_t bt = blockIdx.x;
  const int t = static_cast<int>(bt % L);
  const int64_t rbt = bt - t + (L - 1 - t);
  const int half = d_v / 2;
  for (int e = threadIdx.x; e < heads * half; e += blockDim.x) {
    const int h = e / half, j = 2 * (e % half);
    const float* a = ovR + (rbt * heads + h) * 2 * d_v + j;
    const float2 ah = *reinterpret_cast<const float2*>(a), al = *reinterpret_cast<const float2*>(a + d_v);
    *reinterpret_cast<float2*>(dv + (bt * heads + h) * d_v + j) = make_float2(ah.x + al.x, ah.y + al.y);
  }
}

// dS0[i][j] = sum_t' g^(L-t') (f q~)R[t'][i] doR[t'][j]  (t' = L-1-n, so g^(n+1)), f q~ from its
// two parts: CTA = (b * h, 32-row block of d_k), thread = (row i, columns j).
__global__ void __launch_bounds__(256) bwd_tc_dstate(const __nv_bfloat16* __restrict__ fqRw,
                                                     const __nv_bfloat16* __restrict__ doR, float* __restrict__ dstate,
                                                     int L, int heads, int d_k, int d_v, HeadParams hp) {
  const int bh = blockIdx.x, b = bh / heads, h = bh % heads;
  const float lg = hp.log2g[h];
  for (int e = threadIdx.x; e < 32 * d_v; e += blockDim.x) {
    const int i = blockIdx.y * 32 + e / d_v, j = e % d_v;
    if (i >= d_k) continue;
    float s = 0.f;
    for (int tp = 0; tp < L; ++tp) {
      const int64_t r = (static_cast<int64_t>(b) * L + tp) * heads + h;
      const float fq = __bfloat162float(fqRw[r * 2 * d_k + i]) + __bfloat162float(fqRw[r * 2 * d_k + d_k + i]);
      s = fmaf(exp2f(static_cast<float>(L - tp) * lg) * fq, __bfloat162float(doR[r * d_v + j]), s);
    }
    dstate[(static_cast<int64_t>(bh) * d_k + i) * d_v + j] = s;
  }
}

constexpr int kBwdChunk = 64;

size_t a256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct TcLayout {
  size_t ktw, qR, kR, fqRw, vR, doR, fdoRw, oq, okR, ovR, s0t, fwd, total;
};
TcLayout tc_layout(const Dims& d) {
  const size_t tok = static_cast<size_t>(d.batch * d.seqlen * d.heads);
  const size_t dk = static_cast<size_t>(d.d_k), dv = static_cast<size_t>(d.d_v);
  TcLayout l{};
  size_t off = 0;
  l.ktw = off; off += a256(tok * 2 * dk * 2);
  l.qR = off; off += a256(tok * dk * 2);
  l.kR = off; off += a256(tok * dk * 2);
  l.fqRw = off; off += a256(tok * 2 * dk * 2);
  l.vR = off; off += a256(tok * dv * 2);
  l.doR = off; off += a256(tok * dv * 2);
  l.fdoRw = off; off += a256(tok * 2 * dv * 2);
  l.oq = off; off += a256(tok * 2 * dk * 4);
  l.okR = off; off += a256(tok * 2 * dk * 4);
  l.ovR = off; off += a256(tok * 2 * dv * 4);
  l.s0t = off; off += a256(static_cast<size_t>(d.batch * d.heads) * dv * 2 * dk * 4);
  l.fwd = off;
  // the forward runs' own workspace (two-pass segment states), shared by the three in turn
  off += a256(6 * 4 * static_cast<size_t>(d.batch * d.heads) * 2 * dk * dv);
  l.total = off;
  return l;
}

// The three forward runs (values of twice the width: hi | lo), described without launching.
constexpr int kRuns = 3;
void tc_calls(const BackwardCall& c, char* ws, const TcLayout& l, RetentionCall out[kRuns]) {
  const Dims& d = c.dims;
  const Dims d1{d.batch, d.seqlen, d.heads, d.d_v, 2 * d.d_k};  // key dim d_v, value dim 2 d_k
  const Dims d3{d.batch, d.seqlen, d.heads, d.d_k, 2 * d.d_v};
  auto base = [&](const void* q, const void* k, const void* v, void* o, const Dims& dd, uint32_t flags,
                  const float* s_in) {
    RetentionCall r{q, k, v, o, dd, RETNET_BF16, RETNET_F32, 0, flags, kBwdChunk, true, s_in, nullptr, nullptr,
                    nullptr};
    r.ws = ws + l.fwd;
    r.ws_bytes = l.total - l.fwd;
    return r;
  };
  out[0] = base(c.dout, c.v, ws + l.ktw, ws + l.oq, d1, 0u,
                c.state_in ? reinterpret_cast<const float*>(ws + l.s0t) : nullptr);
  out[1] = base(ws + l.vR, ws + l.doR, ws + l.fqRw, ws + l.okR, d1, 0u, nullptr);
  out[2] = base(ws + l.kR, ws + l.qR, ws + l.fdoRw, ws + l.ovR, d3, c.flags & RETNET_F_XPOS, nullptr);
}

// Head parameters of each run: the kernels rotate by whatever theta they are given (a call
// without xPos carries zeros), so the dq and dk runs get zeros and the dv run -theta.
HeadParams run_params(const HeadParams& hp, int run) {
  HeadParams r = hp;
  for (int j = 0; j < kMaxPairs; ++j) r.theta[j] = run == 2 ? -hp.theta[j] : 0.f;
  return r;
}

}  // namespace

size_t backward_tc_workspace_bytes(const Dims& d) { return tc_layout(d).total; }

bool backward_tc_applies(const BackwardCall& c, const HeadParams& hp) {
  const Dims& d = c.dims;
  if (c.in_dtype != RETNET_BF16 || !tc_driver_ready()) return false;
  auto dim_ok = [](int64_t x) { return x == 64 || x == 128 || x == 256; };
  if (!dim_ok(d.d_k) || !dim_ok(d.d_v) || d.seqlen < 1) return false;
  if (!c.ws || c.ws_bytes < backward_tc_workspace_bytes(d)) return false;
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!al16(c.q) || !al16(c.k) || !al16(c.dq) || !al16(c.dk) || !al16(c.dv) || !al16(c.ws)) return false;
  RetentionCall calls[kRuns];
  tc_calls(c, static_cast<char*>(c.ws), tc_layout(d), calls);
  for (int i = 0; i < kRuns; ++i)
    if (!tc_chunkwise_supported(calls[i]) || !tc_chunkwise_heads_ok(calls[i], run_params(hp, i))) return false;
  return true;
}

cudaError_t launch_backward_tc(const BackwardCall& c, const HeadParams& hp, cudaStream_t s) {
  const Dims& d = c.dims;
  const TcLayout l = tc_layout(d);
  char* ws = static_cast<char*>(c.ws);
  const int L = static_cast<int>(d.seqlen), H = static_cast<int>(d.heads), dk = static_cast<int>(d.d_k),
            dv = static_cast<int>(d.d_v);
  auto bf = [&](size_t off) { return reinterpret_cast<__nv_bfloat16*>(ws + off); };
  auto fp = [&](size_t off) { return reinterpret_cast<float*>(ws + off); };
  const unsigned tokens = static_cast<unsigned>(d.batch * d.seqlen);
  bwd_tc_prep_qk<<<tokens, 128, 0, s>>>(static_cast<const __nv_bfloat16*>(c.q), static_cast<const __nv_bfloat16*>(c.k),
                                         bf(l.ktw), bf(l.qR), bf(l.kR), bf(l.fqRw), L, H, dk, c.pos0, c.flags, hp);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  bwd_tc_prep_v<<<tokens, 128, 0, s>>>(static_cast<const __nv_bfloat16*>(c.v),
                                        static_cast<const __nv_bfloat16*>(c.dout), bf(l.vR), bf(l.doR), bf(l.fdoRw), L,
                                        H, dk, dv, c.pos0, c.flags, hp);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (c.state_in) {
    const int64_t n = d.batch * d.heads * d.d_k * d.d_v;
    const int blocks = static_cast<int>(std::min<int64_t>((n + 255) / 256, 148 * 16));
    bwd_tc_transpose<<<blocks, 256, 0, s>>>(c.state_in, fp(l.s0t), n, dk, dv);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  RetentionCall calls[kRuns];
  tc_calls(c, ws, l, calls);
  for (int i = 0; i < kRuns; ++i)
    if ((e = launch_tc_chunkwise(calls[i], run_params(hp, i), s)) != cudaSuccess) return e;
  bwd_tc_post_qk<<<tokens, 128, 0, s>>>(fp(l.oq), fp(l.okR), c.dq, c.dk, L, H, dk, c.pos0, c.flags, hp);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  bwd_tc_post_v<<<tokens, 128, 0, s>>>(fp(l.ovR), c.dv, L, H, dv);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (c.dstate) {
    const dim3 gs(static_cast<unsigned>(d.batch * d.heads), static_cast<unsigned>((dk + 31) / 32));
    bwd_tc_dstate<<<gs, 256, 0, s>>>(bf(l.fqRw), bf(l.doR), c.dstate, L, H, dk, dv, hp);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

int backward_tc_launches(const BackwardCall& c) {
  RetentionCall calls[kRuns];
  tc_calls(c, static_cast<char*>(c.ws), tc_layout(c.dims), calls);
  int n = 2 + 2 + (c.state_in ? 1 : 0) + (c.dstate ? 1 : 0);
  for (int i = 0; i < kRuns; ++i) n += tc_chunkwise_launches(calls[i]);
  return n;
}

}  // namespace retnet

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
// A prep kernel writes the operands (rotations, row factors, reversal): exact bf16 copies of q,
// k, v, dO for the runs' queries and keys; k~, f q~ and f dO, which are not bf16 numbers, as
// fp16 value rows (one rounding, 2^-11 relative: a bf16 rounding of the values, 2^-8, left
// 1-2e-2 max|err|/rms in the gradient), which the runs' converters take as they are.  The dv
// run writes its rows in forward order itself (reversed-output epilogue); a post kernel scales
// dq by f, turns dq and dk back (R^T) and undoes the reversal of dk.
#include <algorithm>

#include "launch.h"

namespace retnet {
namespace {

// Values rounded to fp16 that left its range (the runs would carry inf); read with the
// tensor-core kernels' own count by retnet_fp16_range_errors.
__device__ unsigned int g_bwd_fp16_overflows = 0;

__device__ __forceinline__ __half to_f16(float x, float& mx) {
  mx = fmaxf(mx, fabsf(x));
  return __float2half_rn(x);
}
__device__ __forceinline__ void report_range(float mx) {
  if (!(mx < 65520.f)) atomicAdd(&g_bwd_fp16_overflows, 1u);
}

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


// The elementwise kernels run one CTA per token (b, t): the rotation of pair j is the same for
// every head, and each head's row factor is computed once, into shared memory.
__device__ __forceinline__ void row_factors(float* sf, int heads, int d_k, int64_t p, uint32_t flags,
                                            const HeadParams& hp) {
  for (int h = threadIdx.x; h < heads; h += blockDim.x) sf[h] = row_f(hp.gamma[h], d_k, p, flags);
  __syncthreads();
}

// Rotation (cos, sin) of every pair j at position p, into shared memory (identity without
// xPos); one sincos a pair, shared by the heads.
__device__ __forceinline__ void pair_rotations(float2* rot, int d_k, int64_t p, bool xpos, const HeadParams& hp) {
  for (int j = threadIdx.x; j < d_k / 2; j += blockDim.x) {
    float c = 1.f, s = 0.f;
    if (xpos) xpos_sincos(p, hp.theta[j], &s, &c);
    rot[j] = make_float2(c, s);
  }
  __syncthreads();
}

// bf16x2 word -> two floats (element 2i at the low half).
__device__ __forceinline__ float2 bf2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
__device__ __forceinline__ uint32_t h2(float a, float b, float& mx) {
  const __half2 x = __halves2half2(to_f16(a, mx), to_f16(b, mx));
  return *reinterpret_cast<const uint32_t*>(&x);
}

// Token (b, t): k~ (forward order) and f q~ (reversed) as fp16 rows; q, k copied reversed.
// Thread = (head, 16-byte group of 8 elements = 4 rotary pairs).
__global__ void __launch_bounds__(128) bwd_tc_prep_qk(const __nv_bfloat16* __restrict__ q,
                                                      const __nv_bfloat16* __restrict__ k, __half* __restrict__ kt,
                                                      __nv_bfloat16* __restrict__ qR, __nv_bfloat16* __restrict__ kR,
                                                      __half* __restrict__ fqR, int L, int heads, int d_k, int64_t pos0,
                                                      uint32_t flags, HeadParams hp) {
  __shared__ float sf[RETNET_MAX_HEADS];
  __shared__ float2 rot[kMaxPairs];
  const int64_t bt = blockIdx.x;
  const int t = static_cast<int>(bt % L);
  const int64_t rbt = bt - t + (L - 1 - t);  // the same b at t' = L-1-t
  row_factors(sf, heads, d_k, pos0 + t, flags, hp);
  pair_rotations(rot, d_k, pos0 + t, (flags & RETNET_F_XPOS) != 0, hp);
  const int groups = d_k / 8;
  float mx = 0.f;
  for (int e = threadIdx.x; e < heads * groups; e += blockDim.x) {
    const int h = e / groups, g = e % groups;
    const int64_t o = (bt * heads + h) * d_k + 8 * g, ro = (rbt * heads + h) * d_k + 8 * g;
    const uint4 q4 = *reinterpret_cast<const uint4*>(q + o);
    const uint4 k4 = *reinterpret_cast<const uint4*>(k + o);
    *reinterpret_cast<uint4*>(qR + ro) = q4;
    *reinterpret_cast<uint4*>(kR + ro) = k4;
    const uint32_t qw[4] = {q4.x, q4.y, q4.z, q4.w}, kw[4] = {k4.x, k4.y, k4.z, k4.w};
    uint32_t ko[4], qo[4];
    const float f = sf[h];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 cs = rot[4 * g + i];
      const float2 kf = bf2(kw[i]), qf = bf2(qw[i]);
      ko[i] = h2(kf.x * cs.x - kf.y * cs.y, kf.x * cs.y + kf.y * cs.x, mx);
      qo[i] = h2(f * (qf.x * cs.x - qf.y * cs.y), f * (qf.x * cs.y + qf.y * cs.x), mx);
    }
    *reinterpret_cast<uint4*>(kt + o) = make_uint4(ko[0], ko[1], ko[2], ko[3]);
    *reinterpret_cast<uint4*>(fqR + ro) = make_uint4(qo[0], qo[1], qo[2], qo[3]);
  }
  report_range(mx);
}

// Token (b, t): v and dO copied reversed; f dO reversed as fp16 rows.  Thread = (head,
// 16-byte group of 8 elements).
__global__ void __launch_bounds__(128) bwd_tc_prep_v(const __nv_bfloat16* __restrict__ v,
                                                     const __nv_bfloat16* __restrict__ dout,
                                                     __nv_bfloat16* __restrict__ vR, __nv_bfloat16* __restrict__ doR,
                                                     __half* __restrict__ fdoR, int L, int heads, int d_k, int d_v,
                                                     int64_t pos0, uint32_t flags, HeadParams hp) {
  __shared__ float sf[RETNET_MAX_HEADS];
  const int64_t bt = blockIdx.x;
  const int t = static_cast<int>(bt % L);
  const int64_t rbt = bt - t + (L - 1 - t);
  row_factors(sf, heads, d_k, pos0 + t, flags, hp);
  const int groups = d_v / 8;
  float mx = 0.f;
  for (int e = threadIdx.x; e < heads * groups; e += blockDim.x) {
    const int h = e / groups, g = e % groups;
    const int64_t o = (bt * heads + h) * d_v + 8 * g, ro = (rbt * heads + h) * d_v + 8 * g;
    const uint4 v4 = *reinterpret_cast<const uint4*>(v + o);
    const uint4 d4 = *reinterpret_cast<const uint4*>(dout + o);
    *reinterpret_cast<uint4*>(vR + ro) = v4;
    *reinterpret_cast<uint4*>(doR + ro) = d4;
    const uint32_t dw[4] = {d4.x, d4.y, d4.z, d4.w};
    uint32_t fo[4];
    const float f = sf[h];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 df = bf2(dw[i]);
      fo[i] = h2(f * df.x, f * df.y, mx);
    }
    *reinterpret_cast<uint4*>(fdoR + ro) = make_uint4(fo[0], fo[1], fo[2], fo[3]);
  }
  report_range(mx);
}

// S0^T per (batch, head), the start state of the dq run: [d_k][d_v] -> [d_v][d_k].
__global__ void bwd_tc_transpose(const float* __restrict__ s, float* __restrict__ st, int64_t n, int d_k, int d_v) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = i / (static_cast<int64_t>(d_k) * d_v);
    const int r = static_cast<int>(i % (static_cast<int64_t>(d_k) * d_v));
    const int a = r / d_v, bb = r % d_v;
    st[(m * d_v + bb) * d_k + a] = s[i];
  }
}

// Token (b, t): dq = R^T (f (the dq run's row)); dk = R^T (the dk run's reversed row).
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
      const int64_t o = (bt * heads + h) * d_k + 2 * j, ro = (rbt * heads + h) * d_k + 2 * j;
      const float2 a = *reinterpret_cast<const float2*>(oq + o);
      const float y0 = sf[h] * a.x, y1 = sf[h] * a.y;
      *reinterpret_cast<float2*>(dq + o) = make_float2(fmaf(y0, c, y1 * s), fmaf(y1, c, -y0 * s));
      const float2 z = *reinterpret_cast<const float2*>(okR + ro);
      *reinterpret_cast<float2*>(dk + o) = make_float2(fmaf(z.x, c, z.y * s), fmaf(z.y, c, -z.x * s));
    }
  }
}

// dS0[i][j] = sum_t' g^(L-t') (f q~)R[t'][i] doR[t'][j]  (t' = L-1-n, so g^(n+1)):
// CTA = (b * h, 32-row block of d_k), thread = (row i, columns j).
__global__ void __launch_bounds__(256) bwd_tc_dstate(const __half* __restrict__ fqR,
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
      const float fq = __half2float(fqR[r * d_k + i]);
      s = fmaf(exp2f(static_cast<float>(L - tp) * lg) * fq, __bfloat162float(doR[r * d_v + j]), s);
    }
    dstate[(static_cast<int64_t>(bh) * d_k + i) * d_v + j] = s;
  }
}

constexpr int kBwdChunk = 64;

size_t a256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct TcLayout {
  size_t kt, qR, kR, fqR, vR, doR, fdoR, oq, okR, s0t, fwd, total;
};
TcLayout tc_layout(const Dims& d) {
  const size_t tok = static_cast<size_t>(d.batch * d.seqlen * d.heads);
  const size_t dk = static_cast<size_t>(d.d_k), dv = static_cast<size_t>(d.d_v);
  TcLayout l{};
  size_t off = 0;
  l.kt = off; off += a256(tok * dk * 2);
  l.qR = off; off += a256(tok * dk * 2);
  l.kR = off; off += a256(tok * dk * 2);
  l.fqR = off; off += a256(tok * dk * 2);
  l.vR = off; off += a256(tok * dv * 2);
  l.doR = off; off += a256(tok * dv * 2);
  l.fdoR = off; off += a256(tok * dv * 2);
  l.oq = off; off += a256(tok * dk * 4);
  l.okR = off; off += a256(tok * dk * 4);
  l.s0t = off; off += a256(static_cast<size_t>(d.batch * d.heads) * dv * dk * 4);
  l.fwd = off;
  // the forward runs' own workspace (two-pass segment states), shared by the three in turn
  off += a256(6 * 4 * static_cast<size_t>(d.batch * d.heads) * dk * dv);
  l.total = off;
  return l;
}

// The three forward runs (fp16 value rows), described without launching.
constexpr int kRuns = 3;
void tc_calls(const BackwardCall& c, char* ws, const TcLayout& l, RetentionCall out[kRuns]) {
  const Dims& d = c.dims;
  const Dims d1{d.batch, d.seqlen, d.heads, d.d_v, d.d_k};  // key dim d_v, value dim d_k
  const Dims d3{d.batch, d.seqlen, d.heads, d.d_k, d.d_v};
  auto base = [&](const void* q, const void* k, const void* v, void* o, const Dims& dd, uint32_t flags,
                  const float* s_in) {
    RetentionCall r{q, k, v, o, dd, RETNET_BF16, RETNET_F32, 0, flags, kBwdChunk, true, s_in, nullptr, nullptr,
                    nullptr};
    r.ws = ws + l.fwd;
    r.ws_bytes = l.total - l.fwd;
    r.v_f16 = true;
    return r;
  };
  out[0] = base(c.dout, c.v, ws + l.kt, ws + l.oq, d1, 0u,
                c.state_in ? reinterpret_cast<const float*>(ws + l.s0t) : nullptr);
  out[1] = base(ws + l.vR, ws + l.doR, ws + l.fqR, ws + l.okR, d1, 0u, nullptr);
  out[2] = base(ws + l.kR, ws + l.qR, ws + l.fdoR, c.dv, d3, c.flags & RETNET_F_XPOS, nullptr);
  out[2].o_rev = true;  // dv in forward order straight from the run
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
  if (!al16(c.q) || !al16(c.k) || !al16(c.v) || !al16(c.dout) || !al16(c.dq) || !al16(c.dk) || !al16(c.dv) ||
      !al16(c.ws))
    return false;
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
  auto hf = [&](size_t off) { return reinterpret_cast<__half*>(ws + off); };
  auto fp = [&](size_t off) { return reinterpret_cast<float*>(ws + off); };
  const unsigned tokens = static_cast<unsigned>(d.batch * d.seqlen);
  bwd_tc_prep_qk<<<tokens, 128, 0, s>>>(static_cast<const __nv_bfloat16*>(c.q), static_cast<const __nv_bfloat16*>(c.k),
                                         hf(l.kt), bf(l.qR), bf(l.kR), hf(l.fqR), L, H, dk, c.pos0, c.flags, hp);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  bwd_tc_prep_v<<<tokens, 128, 0, s>>>(static_cast<const __nv_bfloat16*>(c.v),
                                        static_cast<const __nv_bfloat16*>(c.dout), bf(l.vR), bf(l.doR), hf(l.fdoR), L,
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
  if (c.dstate) {
    const dim3 gs(static_cast<unsigned>(d.batch * d.heads), static_cast<unsigned>((dk + 31) / 32));
    bwd_tc_dstate<<<gs, 256, 0, s>>>(hf(l.fqR), bf(l.doR), c.dstate, L, H, dk, dv, hp);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t bwd_fp16_overflows(unsigned int* count, bool clear) {
  cudaError_t e = cudaMemcpyFromSymbol(count, g_bwd_fp16_overflows, sizeof(unsigned int));
  if (e != cudaSuccess || !clear || *count == 0) return e;
  const unsigned int zero = 0;
  return cudaMemcpyToSymbol(g_bwd_fp16_overflows, &zero, sizeof(unsigned int));
}

int backward_tc_launches(const BackwardCall& c) {
  RetentionCall calls[kRuns];
  tc_calls(c, static_cast<char*>(c.ws), tc_layout(c.dims), calls);
  int n = 2 + 1 + (c.state_in ? 1 : 0) + (c.dstate ? 1 : 0);
  for (int i = 0; i < kRuns; ++i) n += tc_chunkwise_launches(calls[i]);
  return n;
}

}  // namespace retnet

// backward.cu -- gradient of the retention forward for training ("阅读笔记：RetNet" §2.4: the
// chunkwise form is the training form; its output is that of the parallel form, §2.3, so the
// gradient is the derivative of that definition).  With q~, k~ the xPos-rotated rows, f_n the
// row factor of §三.3 (no R~) and S0 the state before the first token:
//   O_n   = f_n [ sum_{m<=n} g^(n-m) (q~_n . k~_m) v_m + g^(n+1) q~_n S0 ]
//   dq~_n = f_n [ sum_{m<=n} g^(n-m) (dO_n . v_m) k~_m + g^(n+1) S0 dO_n ]
//   dk~_m = sum_{n>=m} f_n g^(n-m) (dO_n . v_m) q~_n
//   dv_m  = sum_{n>=m} f_n g^(n-m) (q~_n . k~_m) dO_n
//   dS0   = sum_n f_n g^(n+1) q~_n^T dO_n,       dq = R^T dq~, dk = R^T dk~.
//
// fp32 CUDA cores: the path for fp32 inputs and other shapes (O(L^2) per (batch, head), like
// the parallel form); bf16 inputs with d_k, d_v in {64, 128, 256} take the tensor-core path of
// backward_tc.cu when the workspace holds its operands.  A prep kernel writes q~, k~ (fp32) to the workspace; the
// dq kernel gives each warp one row n and sweeps the keys m <= n in tiles of 32 staged in
// shared memory (lane = key for the dot products, lane = column for the accumulation); the
// dk/dv kernel does the same for a key row m over the queries n >= m; the state kernel
// reduces over the sequence per (d_k row, d_v column).
#include <algorithm>

#include "launch.h"

namespace retnet {
namespace {

constexpr int kBwdWarps = 32;  // rows per CTA (each CTA streams the keys once for all of them)
constexpr int kTile = 32;      // keys (or queries) staged per step
constexpr int kBwdMaxD = 256;  // d_k, d_v limit of the register layout (8 values a lane)
constexpr int kPerLane = kBwdMaxD / 32;

template <typename Tin>
__global__ void bwd_prep_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, float* __restrict__ qr,
                                float* __restrict__ kr, int64_t rows, int L, int heads, int d_k, int64_t pos0,
                                uint32_t flags, HeadParams hp) {
  const int np = d_k / 2;
  const bool xpos = (flags & RETNET_F_XPOS) != 0;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < rows * np;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = i / np;  // (b * L + t) * heads + h
    const int j = static_cast<int>(i % np);
    const int t = static_cast<int>((row / heads) % L);
    float c = 1.f, s = 0.f;
    if (xpos) xpos_sincos(pos0 + t, hp.theta[j], &s, &c);
    const int64_t o = row * d_k + 2 * j;
    const float q0 = load_f(q, o), q1 = load_f(q, o + 1), k0 = load_f(k, o), k1 = load_f(k, o + 1);
    qr[o] = q0 * c - q1 * s;
    qr[o + 1] = q0 * s + q1 * c;
    kr[o] = k0 * c - k1 * s;
    kr[o + 1] = k0 * s + k1 * c;
  }
}

// Turns a rotated-frame gradient row (d_k values in shared memory) back: x = R(p theta)^T y.
__device__ __forceinline__ void rotate_back_store(const float* y, float* out, int d_k, int64_t p, bool xpos,
                                                  const HeadParams& hp, int lane) {
  for (int j = lane; j < d_k / 2; j += 32) {
    float c = 1.f, s = 0.f;
    if (xpos) xpos_sincos(p, hp.theta[j], &s, &c);
    const float y0 = y[2 * j], y1 = y[2 * j + 1];
    out[2 * j] = fmaf(y0, c, y1 * s);
    out[2 * j + 1] = fmaf(y1, c, -y0 * s);
  }
}

// dq: CTA = (batch * head, 32 rows); warp w owns row n = n0 + w.
template <typename Tin>
__global__ void __launch_bounds__(32 * kBwdWarps) bwd_dq_kernel(const Tin* __restrict__ v, const Tin* __restrict__ dout,
                                                                const float* __restrict__ kr, const float* state_in,
                                                                float* __restrict__ dq, int L, int heads, int d_k,
                                                                int d_v, int64_t pos0, uint32_t flags, HeadParams hp) {
  extern __shared__ float sm[];
  float* sv = sm;                              // [kTile][d_v + 1]
  float* sk = sv + kTile * (d_v + 1);          // [kTile][d_k]
  float* sdo = sk + kTile * d_k;               // [kBwdWarps][d_v]
  float* srow = sdo + kBwdWarps * d_v;         // [kBwdWarps][d_k]
  const int bh = blockIdx.x, b = bh / heads, h = bh % heads;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n0 = blockIdx.y * kBwdWarps, n = n0 + warp;
  const float lg = hp.log2g[h];
  auto row = [&](int t) { return (static_cast<int64_t>(b) * L + t) * heads + h; };
  if (n < L)
    for (int j = lane; j < d_v; j += 32) sdo[warp * d_v + j] = load_f(dout, row(n) * d_v + j);
  float acc[kPerLane];
#pragma unroll
  for (int r = 0; r < kPerLane; ++r) acc[r] = 0.f;
  const int m_end = min(L, n0 + kBwdWarps);  // keys m <= the CTA's last row
  for (int m0 = 0; m0 < m_end; m0 += kTile) {
    __syncthreads();
    for (int e = threadIdx.x; e < kTile * d_v; e += blockDim.x) {
      const int mm = e / d_v, j = e % d_v;
      sv[mm * (d_v + 1) + j] = (m0 + mm < L) ? load_f(v, row(m0 + mm) * d_v + j) : 0.f;
    }
    for (int e = threadIdx.x; e < kTile * d_k; e += blockDim.x) {
      const int mm = e / d_k, i = e % d_k;
      sk[mm * d_k + i] = (m0 + mm < L) ? kr[row(m0 + mm) * d_k + i] : 0.f;
    }
    __syncthreads();
    if (n >= L) continue;
    // lane = key m0 + lane: w = g^(n-m) (dO_n . v_m)
    const int m = m0 + lane;
    float w = 0.f;
    if (m <= n) {
      float s = 0.f;
      for (int j = 0; j < d_v; ++j) s = fmaf(sdo[warp * d_v + j], sv[lane * (d_v + 1) + j], s);
      w = exp2f(static_cast<float>(n - m) * lg) * s;
    }
    // lane = column i = lane + 32 r: acc_i += sum_m w_m k~_m[i]
    for (int mm = 0; mm < kTile; ++mm) {
      const float wm = __shfl_sync(0xffffffffu, w, mm);
#pragma unroll
      for (int r = 0; r < kPerLane; ++r) {
        const int i = lane + 32 * r;
        if (i < d_k) acc[r] = fmaf(wm, sk[mm * d_k + i], acc[r]);
      }
    }
  }
  if (n >= L) return;
  const float gn = exp2f(static_cast<float>(n + 1) * lg);
  const float f = row_factor(hp.gamma[h], d_k, pos0 + n, flags);
#pragma unroll
  for (int r = 0; r < kPerLane; ++r) {
    const int i = lane + 32 * r;
    if (i >= d_k) continue;
    float x = acc[r];
    if (state_in) {  // + g^(n+1) (S0 dO_n)_i
      const float* s0 = state_in + (static_cast<int64_t>(bh) * d_k + i) * d_v;
      float s = 0.f;
      for (int j = 0; j < d_v; ++j) s = fmaf(s0[j], sdo[warp * d_v + j], s);
      x = fmaf(gn, s, x);
    }
    srow[warp * d_k + i] = f * x;
  }
  __syncwarp();
  rotate_back_store(srow + warp * d_k, dq + row(n) * d_k, d_k, pos0 + n, (flags & RETNET_F_XPOS) != 0, hp, lane);
}

// dk, dv: CTA = (batch * head, 32 rows); warp w owns key row m = m0 + w; queries n >= m.
template <typename Tin>
__global__ void __launch_bounds__(32 * kBwdWarps) bwd_dkv_kernel(const Tin* __restrict__ v, const Tin* __restrict__ dout,
                                                                 const float* __restrict__ qr,
                                                                 const float* __restrict__ kr, float* __restrict__ dk,
                                                                 float* __restrict__ dv, int L, int heads, int d_k,
                                                                 int d_v, int64_t pos0, uint32_t flags, HeadParams hp) {
  extern __shared__ float sm[];
  float* sdo = sm;                          // [kTile][d_v + 1]
  float* sq = sdo + kTile * (d_v + 1);      // [kTile][d_k + 1]
  float* sv = sq + kTile * (d_k + 1);       // [kBwdWarps][d_v]
  float* skm = sv + kBwdWarps * d_v;        // [kBwdWarps][d_k]
  float* sf = skm + kBwdWarps * d_k;        // [kTile] row factors of the staged queries
  const int bh = blockIdx.x, b = bh / heads, h = bh % heads;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int m0 = blockIdx.y * kBwdWarps, m = m0 + warp;
  const float lg = hp.log2g[h];
  auto row = [&](int t) { return (static_cast<int64_t>(b) * L + t) * heads + h; };
  if (m < L) {
    for (int j = lane; j < d_v; j += 32) sv[warp * d_v + j] = load_f(v, row(m) * d_v + j);
    for (int i = lane; i < d_k; i += 32) skm[warp * d_k + i] = kr[row(m) * d_k + i];
  }
  float ak[kPerLane], av[kPerLane];
#pragma unroll
  for (int r = 0; r < kPerLane; ++r) ak[r] = av[r] = 0.f;
  for (int t0 = m0; t0 < L; t0 += kTile) {  // queries n >= the CTA's first row
    __syncthreads();
    for (int e = threadIdx.x; e < kTile * d_v; e += blockDim.x) {
      const int nn = e / d_v, j = e % d_v;
      sdo[nn * (d_v + 1) + j] = (t0 + nn < L) ? load_f(dout, row(t0 + nn) * d_v + j) : 0.f;
    }
    for (int e = threadIdx.x; e < kTile * d_k; e += blockDim.x) {
      const int nn = e / d_k, i = e % d_k;
      sq[nn * (d_k + 1) + i] = (t0 + nn < L) ? qr[row(t0 + nn) * d_k + i] : 0.f;
    }
    for (int e = threadIdx.x; e < kTile; e += blockDim.x)
      sf[e] = (t0 + e < L) ? row_factor(hp.gamma[h], d_k, pos0 + t0 + e, flags) : 0.f;
    __syncthreads();
    if (m >= L) continue;
    // lane = query n = t0 + lane: a = f_n g^(n-m); wk = a (dO_n . v_m), wv = a (q~_n . k~_m)
    const int n = t0 + lane;
    float wk = 0.f, wv = 0.f;
    if (n >= m && n < L) {
      float s1 = 0.f, s2 = 0.f;
      for (int j = 0; j < d_v; ++j) s1 = fmaf(sdo[lane * (d_v + 1) + j], sv[warp * d_v + j], s1);
      for (int i = 0; i < d_k; ++i) s2 = fmaf(sq[lane * (d_k + 1) + i], skm[warp * d_k + i], s2);
      const float a = sf[lane] * exp2f(static_cast<float>(n - m) * lg);
      wk = a * s1;
      wv = a * s2;
    }
    for (int nn = 0; nn < kTile; ++nn) {
      const float bk = __shfl_sync(0xffffffffu, wk, nn), bv = __shfl_sync(0xffffffffu, wv, nn);
#pragma unroll
      for (int r = 0; r < kPerLane; ++r) {
        const int c = lane + 32 * r;
        if (c < d_k) ak[r] = fmaf(bk, sq[nn * (d_k + 1) + c], ak[r]);
        if (c < d_v) av[r] = fmaf(bv, sdo[nn * (d_v + 1) + c], av[r]);
      }
    }
  }
  if (m >= L) return;
  __syncwarp();
#pragma unroll
  for (int r = 0; r < kPerLane; ++r) {
    const int c = lane + 32 * r;
    if (c < d_k) skm[warp * d_k + c] = ak[r];  // this warp's own key row is no longer read
    if (c < d_v) dv[row(m) * d_v + c] = av[r];
  }
  __syncwarp();
  rotate_back_store(skm + warp * d_k, dk + row(m) * d_k, d_k, pos0 + m, (flags & RETNET_F_XPOS) != 0, hp, lane);
}

// dS0[i][j] = sum_n f_n g^(n+1) q~_n[i] dO_n[j]: CTA = (batch * head, 32-row block of d_k),
// thread = (row i, 8 columns j).
template <typename Tin>
__global__ void __launch_bounds__(256) bwd_dstate_kernel(const Tin* __restrict__ dout, const float* __restrict__ qr,
                                                         float* __restrict__ dstate, int L, int heads, int d_k,
                                                         int d_v, int64_t pos0, uint32_t flags, HeadParams hp) {
  const int bh = blockIdx.x, b = bh / heads, h = bh % heads;
  const float lg = hp.log2g[h];
  for (int e = threadIdx.x; e < 32 * d_v; e += blockDim.x) {
    const int i = blockIdx.y * 32 + e / d_v, j = e % d_v;
    if (i >= d_k) continue;
    float s = 0.f;
    for (int n = 0; n < L; ++n) {
      const int64_t r = (static_cast<int64_t>(b) * L + n) * heads + h;
      const float a = row_factor(hp.gamma[h], d_k, pos0 + n, flags) * exp2f(static_cast<float>(n + 1) * lg);
      s = fmaf(a * qr[r * d_k + i], load_f(dout, r * d_v + j), s);
    }
    dstate[(static_cast<int64_t>(bh) * d_k + i) * d_v + j] = s;
  }
}

template <typename Tin>
cudaError_t launch_backward_t(const BackwardCall& c, const HeadParams& hp, cudaStream_t s) {
  const Dims& d = c.dims;
  const int L = static_cast<int>(d.seqlen), H = static_cast<int>(d.heads), dk = static_cast<int>(d.d_k),
            dv = static_cast<int>(d.d_v);
  const int64_t rows = d.batch * d.seqlen * d.heads;
  float* qr = static_cast<float*>(c.ws);
  float* kr = qr + rows * dk;
  const auto* q = static_cast<const Tin*>(c.q);
  const auto* k = static_cast<const Tin*>(c.k);
  const auto* v = static_cast<const Tin*>(c.v);
  const auto* dout = static_cast<const Tin*>(c.dout);
  const int64_t items = rows * (dk / 2);
  const int blocks = static_cast<int>(std::min<int64_t>((items + 255) / 256, 148 * 16));
  bwd_prep_kernel<Tin><<<blocks, 256, 0, s>>>(q, k, qr, kr, rows, L, H, dk, c.pos0, c.flags, hp);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>(d.batch * d.heads), static_cast<unsigned>((L + kBwdWarps - 1) / kBwdWarps));
  const size_t smq = sizeof(float) * (kTile * (dv + 1) + kTile * dk + kBwdWarps * dv + kBwdWarps * dk);
  const size_t smkv =
      sizeof(float) * (kTile * (dv + 1) + kTile * (dk + 1) + kBwdWarps * dv + kBwdWarps * dk + kTile);
  if ((e = cudaFuncSetAttribute(bwd_dq_kernel<Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(smq))) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(bwd_dkv_kernel<Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(smkv))) != cudaSuccess)
    return e;
  bwd_dq_kernel<Tin><<<grid, 32 * kBwdWarps, smq, s>>>(v, dout, kr, c.state_in, c.dq, L, H, dk, dv, c.pos0, c.flags, hp);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  bwd_dkv_kernel<Tin><<<grid, 32 * kBwdWarps, smkv, s>>>(v, dout, qr, kr, c.dk, c.dv, L, H, dk, dv, c.pos0, c.flags, hp);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (c.dstate) {
    const dim3 gs(static_cast<unsigned>(d.batch * d.heads), static_cast<unsigned>((dk + 31) / 32));
    bwd_dstate_kernel<Tin><<<gs, 256, 0, s>>>(dout, qr, c.dstate, L, H, dk, dv, c.pos0, c.flags, hp);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

size_t backward_workspace_bytes(const Dims& d) {
  return 2 * sizeof(float) * static_cast<size_t>(d.batch * d.seqlen * d.heads * d.d_k);
}

bool backward_supported(const Dims& d) { return d.d_k <= kBwdMaxD && d.d_v <= kBwdMaxD && d.d_k % 2 == 0; }

cudaError_t launch_backward(const BackwardCall& c, const HeadParams& hp, cudaStream_t s) {
  if (backward_tc_applies(c, hp)) return launch_backward_tc(c, hp, s);
  if (c.in_dtype == RETNET_BF16) return launch_backward_t<__nv_bfloat16>(c, hp, s);
  return launch_backward_t<float>(c, hp, s);
}

}  // namespace retnet

// simt_retention.cu -- fp32 CUDA-core retention kernel (parallel form and chunkwise form).
//
// "阅读笔记：RetNet" (mzeromiko blog) §2.3 Parallel Mode and §2.4 Chunkwise Recurrent Mode,
// with the §三.3 normalisations as per-row factors.  This kernel serves fp32 inputs (whose
// tolerance rules out 16-bit tensor-core operands) and every shape the tensor-core kernel does
// not take.  One CTA owns one (batch, head, 32-wide slice of d_v); it walks the chunks in order,
// keeps its slice of the chunk state R (d_k x 32, fp32) and the key-sum z in shared memory,
// and forms the chunk's inner products in 32x32 token tiles.  The parallel form is the same
// walk with one chunk covering the whole sequence and no state.
#include "launch.h"

namespace retnet {
namespace {

constexpr int kT = 32;        // token tile
constexpr int kDVT = 32;      // d_v slice per CTA
constexpr int kThreads = 256;

template <typename Tin, typename Tout>
struct SimtArgs {
  const Tin* q;
  const Tin* k;
  const Tin* v;
  Tout* o;
  Dims d;
  int64_t pos0;
  uint32_t flags;
  int64_t chunk;
  int has_state;
  const float* state_in;
  float* state_out;
  const float* z_in;
  float* z_out;
};

// Load `rows` token rows of a head's q or k (rotated when XPOS is set) into sm[row][0..d_k)
// with row pitch `pitch`; rows past `valid` are zero.
template <typename Tin>
__device__ void load_qk_tile(float* sm, int pitch, const Tin* base, const Dims& d, int64_t b, int64_t h,
                             int64_t t_first, int valid, int64_t pos_first, bool xpos, const HeadParams& hp) {
  const int dk = static_cast<int>(d.d_k);
  const int half = dk / 2;
  for (int e = threadIdx.x; e < kT * half; e += blockDim.x) {
    int r = e / half, j = e % half;
    float x0 = 0.f, x1 = 0.f;
    if (r < valid) {
      int64_t off = ((b * d.seqlen + t_first + r) * d.heads + h) * d.d_k + 2 * j;
      x0 = load_f(base, off);
      x1 = load_f(base, off + 1);
      if (xpos) {
        float s, c;
        xpos_sincos(pos_first + r, hp.theta[j], &s, &c);
        float y0 = x0 * c - x1 * s;
        float y1 = x0 * s + x1 * c;
        x0 = y0;
        x1 = y1;
      }
    }
    sm[r * pitch + 2 * j] = x0;
    sm[r * pitch + 2 * j + 1] = x1;
  }
  if (dk & 1) {  // odd d_k (no rotation possible): last column
    for (int r = threadIdx.x; r < kT; r += blockDim.x) {
      float x = 0.f;
      if (r < valid) x = load_f(base, ((b * d.seqlen + t_first + r) * d.heads + h) * d.d_k + dk - 1);
      sm[r * pitch + dk - 1] = x;
    }
  }
}

template <typename Tin>
__device__ void load_v_tile(float* sm, const Tin* v, const Dims& d, int64_t b, int64_t h, int64_t t_first,
                            int valid, int j0) {
  for (int e = threadIdx.x; e < kT * kDVT; e += blockDim.x) {
    int r = e / kDVT, j = e % kDVT;
    float x = 0.f;
    if (r < valid && j0 + j < d.d_v) x = load_f(v, ((b * d.seqlen + t_first + r) * d.heads + h) * d.d_v + j0 + j);
    sm[r * kDVT + j] = x;
  }
}

template <typename Tin, typename Tout>
__global__ void __launch_bounds__(kThreads) simt_retention_kernel(SimtArgs<Tin, Tout> a, HeadParams hp) {
  extern __shared__ float smem[];
  const Dims d = a.d;
  const int dk = static_cast<int>(d.d_k);
  const int pitch = dk + 1;
  const int j0 = blockIdx.x * kDVT;
  const int64_t h = blockIdx.y, b = blockIdx.z;
  const bool xpos = (a.flags & RETNET_F_XPOS) != 0;
  const bool norm_r = (a.flags & RETNET_F_NORM_R) != 0;
  const float gamma = hp.gamma[h], log2g = hp.log2g[h];

  float* Qs = smem;                 // [kT][pitch]
  float* Ks = Qs + kT * pitch;      // [kT][pitch]
  float* Vs = Ks + kT * pitch;      // [kT][kDVT]
  float* Ps = Vs + kT * kDVT;       // [kT][kT + 1]
  float* Rs = Ps + kT * (kT + 1);   // [dk][kDVT]   chunk state slice R_{i-1}
  float* zs = Rs + dk * kDVT;       // [dk]         key-sum state z_{i-1}

  const int tid = threadIdx.x;
  const int64_t ssz = d.d_k * d.d_v;
  const int64_t bh = b * d.heads + h;

  // R_0 / z_0: the carried state, or zeros.
  for (int e = tid; e < dk * kDVT; e += blockDim.x) {
    int i = e / kDVT, j = e % kDVT;
    float x = 0.f;
    if (a.has_state && a.state_in && j0 + j < d.d_v) x = a.state_in[bh * ssz + i * d.d_v + j0 + j];
    Rs[e] = x;
  }
  for (int i = tid; i < dk; i += blockDim.x) zs[i] = (a.has_state && a.z_in && norm_r) ? a.z_in[bh * d.d_k + i] : 0.f;
  __syncthreads();

  // Thread roles in a 32x32 tile: row r = tid / 8, four columns c = tid % 8 + 8 m (scores)
  // and four output columns jj = (tid % 8) * 4 + m (values).
  const int tr = tid / 8, tc = tid % 8;

  for (int64_t t0 = 0; t0 < d.seqlen; t0 += a.chunk) {
    const int bl = static_cast<int>(min(a.chunk, d.seqlen - t0));  // b', the chunk's length
    for (int u0 = 0; u0 < bl; u0 += kT) {
      const int uvalid = min(kT, bl - u0);
      load_qk_tile(Qs, pitch, a.q, d, b, h, t0 + u0, uvalid, a.pos0 + t0 + u0, xpos, hp);
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      float rowsum = 0.f;  // sum of the row's unscaled inner-chunk scores
      for (int w0 = 0; w0 <= u0; w0 += kT) {
        const int wvalid = min(kT, bl - w0);
        __syncthreads();  // previous users of Ks / Vs / Ps are done
        load_qk_tile(Ks, pitch, a.k, d, b, h, t0 + w0, wvalid, a.pos0 + t0 + w0, xpos, hp);
        load_v_tile(Vs, a.v, d, b, h, t0 + w0, wvalid, j0);
        __syncthreads();
        // P_rc = (q_r . k_c) gamma^(r-c) inside the chunk, 0 above the diagonal ((Q K^T (.) D)).
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int c = tc + 8 * m;
          const int rg = u0 + tr, cg = w0 + c;
          float s = 0.f;
          if (tr < uvalid && c < wvalid && cg <= rg) {
            const float* qr = Qs + tr * pitch;
            const float* kc = Ks + c * pitch;
            for (int i = 0; i < dk; ++i) s = fmaf(qr[i], kc[i], s);
            s *= decay_pow(log2g, rg - cg);
          }
          Ps[tr * (kT + 1) + c] = s;
        }
        __syncthreads();
        const float* pr = Ps + tr * (kT + 1);
        for (int c = 0; c < kT; ++c) {
          const float p = pr[c];
          rowsum += p;
#pragma unroll
          for (int m = 0; m < 4; ++m) acc[m] = fmaf(p, Vs[c * kDVT + tc * 4 + m], acc[m]);
        }
      }
      // Cross-chunk term (Q_[i] R_{i-1}) (.) xi, xi_r = gamma^(r+1); its row sum uses z_{i-1}.
      if (tr < uvalid) {
        const int r = u0 + tr;
        const float xi = decay_pow(log2g, r + 1);
        const float* qr = Qs + tr * pitch;
        float cr[4] = {0.f, 0.f, 0.f, 0.f};
        float qz = 0.f;
        for (int i = 0; i < dk; ++i) {
          const float qi = qr[i];
#pragma unroll
          for (int m = 0; m < 4; ++m) cr[m] = fmaf(qi, Rs[i * kDVT + tc * 4 + m], cr[m]);
          qz = fmaf(qi, zs[i], qz);
        }
#pragma unroll
        for (int m = 0; m < 4; ++m) acc[m] = fmaf(xi, cr[m], acc[m]);
        rowsum = fmaf(xi, qz, rowsum);
        const int64_t p = a.pos0 + t0 + r;
        const float f = row_factor(gamma, dk, p, a.flags);
        const float den = norm_r ? fmaxf(fabsf(f * rowsum), 1.f) : 1.f;
        const float scale = f / den;
        const int64_t obase = ((b * d.seqlen + t0 + r) * d.heads + h) * d.d_v;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int j = j0 + tc * 4 + m;
          if (j < d.d_v) store_f(a.o, obase + j, acc[m] * scale);
        }
      }
      __syncthreads();  // Qs is reloaded next
    }
    if (!a.has_state) continue;  // parallel form: a single chunk, no state
    // R_i = gamma^b' R_{i-1} + K_[i]^T (V_[i] (.) zeta),  zeta_r = gamma^(b'-1-r); z_i alike.
    const float gb = decay_pow(log2g, bl);
    for (int e = tid; e < dk * kDVT; e += blockDim.x) Rs[e] *= gb;
    for (int i = tid; i < dk; i += blockDim.x) zs[i] *= gb;
    for (int w0 = 0; w0 < bl; w0 += kT) {
      const int wvalid = min(kT, bl - w0);
      __syncthreads();
      load_qk_tile(Ks, pitch, a.k, d, b, h, t0 + w0, wvalid, a.pos0 + t0 + w0, xpos, hp);
      load_v_tile(Vs, a.v, d, b, h, t0 + w0, wvalid, j0);
      if (tid < kT) Ps[tid] = (tid < wvalid) ? decay_pow(log2g, bl - 1 - (w0 + tid)) : 0.f;  // zeta
      __syncthreads();
      for (int e = tid; e < dk * kDVT; e += blockDim.x) {
        const int i = e / kDVT, j = e % kDVT;
        float s = Rs[e];
        for (int c = 0; c < wvalid; ++c) s = fmaf(Ps[c] * Ks[c * pitch + i], Vs[c * kDVT + j], s);
        Rs[e] = s;
      }
      for (int i = tid; i < dk; i += blockDim.x) {
        float s = zs[i];
        for (int c = 0; c < wvalid; ++c) s = fmaf(Ps[c], Ks[c * pitch + i], s);
        zs[i] = s;
      }
    }
    __syncthreads();
  }
  if (a.has_state) {
    if (a.state_out) {
      for (int e = tid; e < dk * kDVT; e += blockDim.x) {
        int i = e / kDVT, j = e % kDVT;
        if (j0 + j < d.d_v) a.state_out[bh * ssz + i * d.d_v + j0 + j] = Rs[e];
      }
    }
    if (a.z_out && norm_r && blockIdx.x == 0) {
      for (int i = tid; i < dk; i += blockDim.x) a.z_out[bh * d.d_k + i] = zs[i];
    }
  }
}

size_t simt_smem_bytes(int dk) {
  const int pitch = dk + 1;
  return sizeof(float) * (size_t)(2 * kT * pitch + kT * kDVT + kT * (kT + 1) + dk * kDVT + dk);
}

template <typename Tin, typename Tout>
cudaError_t launch_typed(const RetentionCall& c, const HeadParams& hp, cudaStream_t s) {
  SimtArgs<Tin, Tout> a;
  a.q = static_cast<const Tin*>(c.q);
  a.k = static_cast<const Tin*>(c.k);
  a.v = static_cast<const Tin*>(c.v);
  a.o = static_cast<Tout*>(c.o);
  a.d = c.dims;
  a.pos0 = c.pos0;
  a.flags = c.flags;
  a.chunk = c.chunk;
  a.has_state = c.has_state ? 1 : 0;
  a.state_in = c.state_in;
  a.state_out = c.state_out;
  a.z_in = c.z_in;
  a.z_out = c.z_out;
  const size_t smem = simt_smem_bytes(static_cast<int>(c.dims.d_k));
  cudaError_t e = cudaFuncSetAttribute(simt_retention_kernel<Tin, Tout>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>((c.dims.d_v + kDVT - 1) / kDVT), static_cast<unsigned>(c.dims.heads),
            static_cast<unsigned>(c.dims.batch));
  simt_retention_kernel<Tin, Tout><<<grid, kThreads, smem, s>>>(a, hp);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_simt_retention(const RetentionCall& c, const HeadParams& hp, cudaStream_t s) {
  if (c.in_dtype == RETNET_F32) {
    if (c.out_dtype == RETNET_F32) return launch_typed<float, float>(c, hp, s);
    return launch_typed<float, __nv_bfloat16>(c, hp, s);
  }
  if (c.out_dtype == RETNET_F32) return launch_typed<__nv_bfloat16, float>(c, hp, s);
  return launch_typed<__nv_bfloat16, __nv_bfloat16>(c, hp, s);
}

}  // namespace retnet

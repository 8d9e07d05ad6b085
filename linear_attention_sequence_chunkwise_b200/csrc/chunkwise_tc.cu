// chunkwise_tc.cu -- tcgen05 tensor-core kernel for the chunkwise recurrent form of retention
// ("阅读笔记：RetNet" (mzeromiko blog) §2.4 Chunkwise Recurrent Mode, with the §2.3 xPos
// rotation and the §三.3 QK^T/sqrt(d) and D~ normalisations), bf16 inputs.
//
// One CTA owns one (batch, head, 64-wide slice of d_v) and walks the chunks of B = T tokens
// in order, carrying its slice of the chunk state R (d_k x 64, fp32) in tensor memory.
//
// Scaled operands.  With xi_r = gamma^(r+1) and zeta_c = gamma^(b'-1-c) (b' the chunk's
// length), the kernel stages Qx = xi (.) rot(q) and Kz = zeta (.) rot(k) in fp16.  Then
//   Qx Kz^T = gamma^(b' + r - c) (Q K^T)         ->  P = (Qx Kz^T) * gamma^(-b') (.) causal mask
//   Qx R_{i-1} = (Q R_{i-1}) (.) xi                   (the cross-chunk term, as written)
//   Kz^T V = K^T (V (.) zeta)                         (the state increment, as written)
// so O = P V + Qx R_{i-1} accumulates in one TMEM tile and R_i = gamma^b' R_{i-1} + Kz^T V.
// All fp16 operands stay in the normal range when gamma^B >= 2^-12; the host sends other
// heads/chunk sizes to the CUDA-core kernel.
//
// Warp roles (320 threads):
//   warps 0-3  TMEM warpgroup: S -> P (mask, rescale, fp16 to smem); state update
//              (R_i from TMEM -> fp16 copy in smem for the next cross term, gamma^b' R_i back
//              to TMEM as the base of the next accumulation); epilogue (row scales, store O).
//   warps 4-7  converters: in place over each TMA-staged chunk, rotate q and k by the xPos
//              angle (pairs (2j, 2j+1)), scale by xi / zeta, convert bf16 -> fp16 (V exact).
//   warp 8     TMA producer (Q, K, V tiles, 128-byte swizzle, no multicast).
//   warp 9     TMEM allocator and single-thread tcgen05.mma issuer.
// Every mbarrier wait is bounded in time; a wait that gives up counts a timeout, and every
// role then leaves its loop, drains what it issued and the CTA frees its TMEM and returns.
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <cmath>

#include "launch.h"
#include "sm100_ptx.cuh"

namespace retnet {

namespace {
using namespace sm100;

constexpr int kThreads = 320;
constexpr int kWarpConv0 = 4;
constexpr int kWarpTma = 8;
constexpr int kWarpMma = 9;
constexpr int kDVS = 64;  // d_v slice per CTA

constexpr int kMaxSub = 6;  // pre-pass states of the two-pass form (workspace capacity)
constexpr int kMaxCluster = 4;  // d_v slices a fused GroupNorm epilogue combines (d_v <= 256)

struct TcArgs {
  void* o;
  const float* state_in;
  float* state_out;
  int L;
  int heads;
  int dv;
  int n_chunks;
  int64_t pos0;
  uint32_t flags;
  int nb;     // sub-blocks of T rows per chunk (pipelined kernel)
  int batch;
  int v_f16;  // value rows arrive as fp16 (the converters leave V alone)
  int o_rev;  // output row of token t written at token L - 1 - t (plain epilogue only)
  // Fused MSR epilogue: out = GroupNorm_h(o) * swish(gate), written to o's place.
  const void* gate;
  float eps;
  // R~ normalisation: per-row factor [batch][L][heads] folded into the output scale (or nullptr)
  const float* rden;
  // Sequence segments (pipelined kernel): CTA segment s writes the outputs of chunks
  // [seg_lo[s], seg_hi[s]) and first replays the state over chunks [0, seg_lo[s]).
  int n_seg;
  int seg_lo[4];
  int seg_hi[4];
  // Two-pass form: the pre-pass computes the state of each sub-segment j, chunks
  // [sub_lo[j], sub_hi[j]) from a zero start, into ws (fp32 [j][batch][head][d_k][d_v]);
  // output segment s starts from state_in carried over the first sub_before[s] of them.
  int n_sub;
  int sub_lo[kMaxSub];
  int sub_hi[kMaxSub];
  int sub_before[4];
  float* ws;
};

// Sequence-segment modes of the pipelined kernel.
enum : int {
  SEG_NONE = 0,     // one CTA walks the whole sequence of its slice
  SEG_REPLAY = 1,   // segment s replays the state over chunks [0, lo_s), then outputs [lo_s, hi_s)
  SEG_FROM_WS = 2,  // segment s starts from state_in and the states of segments < s (workspace)
  SEG_STATE = 3     // chunk walk of the segment-state pass (its own kernel): every chunk state-only
};

template <int DK, int T>
struct Cfg {
  static constexpr int QBYTES = T * DK * 2;  // one fp16 Qx or Kz tile
  static constexpr int VBYTES = T * kDVS * 2;
  static constexpr int STAGE = 2 * QBYTES + VBYTES;
  static constexpr int PBYTES = T * T * 2;
  static constexpr int RBYTES = DK * kDVS * 2;
  static constexpr int NBARS = 4 * 3 + 10;
  static constexpr int TABBYTES = 2 * (DK / 2) * 8;  // double-buffered per-chunk rotation base
  static constexpr int FIXED = PBYTES + RBYTES + TABBYTES + NBARS * 8 + 16;
  static constexpr int BUDGET = 227 * 1024 - 1024;
  static constexpr int NS_FIT = (BUDGET - FIXED) / STAGE;
  static constexpr int NS = NS_FIT > 4 ? 4 : NS_FIT;
  static constexpr int SMEM = NS * STAGE + FIXED + 1024;
  static constexpr int RBLK = DK > 128 ? 2 : 1;    // 128-row blocks of the state
  static constexpr int MR = DK >= 128 ? 128 : 64;  // M of the state-update MMA
  static constexpr int COL_O = 0;
  static constexpr int COL_S = kDVS;
  static constexpr int COL_R = kDVS + T;
  static constexpr int USED = kDVS + T + RBLK * kDVS;
  static constexpr int TMEM_COLS = USED <= 128 ? 128 : (USED <= 256 ? 256 : 512);
  static_assert(NS >= 1, "tile does not fit in shared memory");
  static_assert(USED <= 512, "accumulators do not fit in tensor memory");
};

// Barrier slots.
enum : int {
  B_TMA_FULL = 0,     // [4]
  B_CONV_FULL = 4,    // [4]
  B_STAGE_EMPTY = 8,  // [4]
  B_S_FULL = 12,
  B_S_FREE,
  B_P_FULL,
  B_R_DONE,
  B_R_READY,
  B_O_FULL,
  B_O_FREE,
  B_DRAIN,
  B_TAB0,  // [2]: per-chunk rotation base table written (converters)
};

__device__ __forceinline__ float2 cmul(float2 a, float2 b) {
  return make_float2(a.x * b.x - a.y * b.y, a.x * b.y + a.y * b.x);
}

// ---- converter role (shared by both kernels) ------------------------------------------------
//
// 128 threads convert each TMA-staged chunk in place.  The Q and K tiles are DK/64 boxes of
// T rows x 128 bytes; their 16-byte column slots (8 per box) are dealt out to threads, and
// each thread walks the rows of its slot: slot cs = lt % CS (CS = DK/8 slots), rows
// r0 + RS k with r0 = lt / CS and row step RS = 128 / CS.  Its four pairs j = 4 cs + jj have
// fixed frequencies, so the xPos factor e^{i p theta_j} of row r is
// base_j(chunk start) * e^{i r0 theta_j} * (e^{i RS theta_j})^k: one complex product per row.
template <int DK, int T>
struct Converter {
  static constexpr int CS = DK / 8;    // column slots (16 bytes) across the DK/64 boxes
  static constexpr int RS = 128 / CS;  // row step of one thread
  static constexpr int NR = T / RS;    // rows per thread
  static constexpr int VS = 8;         // V: one 64-wide box, 8 slots, row step 16
  float2 W[4];  // e^{i r0 theta_j}
  float2 Z[4];  // e^{i RS theta_j}
  float2 cur, stepT;  // table producer (threads lt < DK/2 own pair j = lt)
  int cs, r0, lt;

  __device__ void init(int lt_, const HeadParams& hp) {
    lt = lt_;
    cs = lt % CS;
    r0 = lt / CS;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const float th = hp.theta[4 * cs + jj];
      float sn, c;
      sincosf(static_cast<float>(r0) * th, &sn, &c);
      W[jj] = make_float2(c, sn);
      sincosf(static_cast<float>(RS) * th, &sn, &c);
      Z[jj] = make_float2(c, sn);
    }
    cur = make_float2(1.f, 0.f);
    stepT = make_float2(1.f, 0.f);
    if (lt < DK / 2) {
      float sn, c;
      xpos_sincos(T, hp.theta[lt], &sn, &c);
      stepT = make_float2(c, sn);
    }
  }

  // Rotation base e^{i p0 theta_j} of chunk i (p0 = pos0 + i T) into tab[j], for j = lt.  The
  // chunk-to-chunk step is an fp32 complex product; every 64 chunks the value is recomputed
  // from the fp64-reduced angle, which bounds the drift to ~1e-5 rad.
  __device__ void put_base(float2* tab, int i, int64_t pos0, const HeadParams& hp) {
    if (lt >= DK / 2) return;
    if ((i & 63) == 0) {
      float sn, c;
      xpos_sincos(pos0 + static_cast<int64_t>(i) * T, hp.theta[lt], &sn, &c);
      cur = make_float2(c, sn);
    } else {
      cur = cmul(cur, stepT);
    }
    tab[lt] = cur;
  }

  // In place: q -> xi (.) rot(q), k -> zeta (.) rot(k) as fp16; v -> fp16.
  __device__ void convert(uint32_t sq, uint32_t sk, uint32_t sv, const float2* base, bool xpos, float log2g,
                          int bl, float& mx) const {
    const uint32_t box = (cs / 8) * T * 128;  // this slot's 64-wide box
    const uint32_t chunk = cs % 8;
    const float xstep = decay_pow(log2g, RS), zstep = exp2f(-static_cast<float>(RS) * log2g);
    float xi = decay_pow(log2g, r0 + 1);
    float zeta = exp2f(static_cast<float>(bl - 1 - r0) * log2g);
    float2 F[4];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) F[jj] = xpos ? cmul(base[4 * cs + jj], W[jj]) : make_float2(1.f, 0.f);
    // Groups of four rows: all loads of a group are issued before its stores (the shared-memory
    // accessors are ordered asm statements, so the grouping has to be explicit).
    static_assert(NR % 4 == 0, "rows per thread must be a multiple of 4");
#pragma unroll 1
    for (int kg = 0; kg < NR; kg += 4) {
      uint32_t q4[4][4], k4[4][4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t off = box + sw128(r0 + RS * (kg + k), chunk);
        ld_shared_v4(sq + off, q4[k][0], q4[k][1], q4[k][2], q4[k][3]);
        ld_shared_v4(sk + off, k4[k][0], k4[k][1], k4[k][2], k4[k][3]);
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        uint32_t qo[4], ko[4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const float c = F[jj].x, sn = F[jj].y;
          const float q0 = __uint_as_float(q4[k][jj] << 16), q1 = __uint_as_float(q4[k][jj] & 0xffff0000u);
          const float k0 = __uint_as_float(k4[k][jj] << 16), k1 = __uint_as_float(k4[k][jj] & 0xffff0000u);
          const float x0 = xi * (q0 * c - q1 * sn), x1 = xi * (q0 * sn + q1 * c);
          const float y0 = zeta * (k0 * c - k1 * sn), y1 = zeta * (k0 * sn + k1 * c);
          mx = absmax(absmax(absmax(absmax(mx, x0), x1), y0), y1);
          qo[jj] = pack_f16x2(x0, x1);
          ko[jj] = pack_f16x2(y0, y1);
          F[jj] = cmul(F[jj], Z[jj]);
        }
        const uint32_t off = box + sw128(r0 + RS * (kg + k), chunk);
        st_shared_v4(sq + off, qo[0], qo[1], qo[2], qo[3]);
        st_shared_v4(sk + off, ko[0], ko[1], ko[2], ko[3]);
        xi *= xstep;
        zeta *= zstep;
      }
    }
    // V: one box of T rows x 64; slot lt % 8, rows lt / 8 + 16 k.
#pragma unroll 1
    for (int kg = 0; kg < T / 16; kg += 4) {
      uint32_t v4[4][4];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        ld_shared_v4(sv + sw128(lt / 8 + 16 * (kg + k), lt % 8), v4[k][0], v4[k][1], v4[k][2], v4[k][3]);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        uint32_t vo[4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const float v0 = __uint_as_float(v4[k][jj] << 16), v1 = __uint_as_float(v4[k][jj] & 0xffff0000u);
          mx = absmax(absmax(mx, v0), v1);
          vo[jj] = pack_f16x2(v0, v1);
        }
        st_shared_v4(sv + sw128(lt / 8 + 16 * (kg + k), lt % 8), vo[0], vo[1], vo[2], vo[3]);
      }
    }
  }
};

template <int DK, int T, typename Tout>
__global__ void __launch_bounds__(kThreads, 1)
    tc_chunkwise_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, TcArgs a, HeadParams hp) {
  using C = Cfg<DK, T>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - raw_addr);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int dvb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const float log2g = hp.log2g[h];
  const int n = a.n_chunks;
  // P and the fp16 state copy carry a fixed 1/sqrt(d_k) so that their fp16 magnitudes stay small;
  // the epilogue multiplies it back out.
  const float sd = rsqrtf(static_cast<float>(DK));

  const uint32_t sP = sbase + C::NS * C::STAGE;
  const uint32_t sR = sP + C::PBYTES;
  float2* tab = reinterpret_cast<float2*>(gbase + C::NS * C::STAGE + C::PBYTES + C::RBYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(gbase + C::NS * C::STAGE + C::PBYTES + C::RBYTES + C::TABBYTES);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + C::NBARS);
  auto bar = [&](int i) { return smem_addr(bars + i); };
  auto sQ = [&](int s) { return sbase + s * C::STAGE; };
  auto sK = [&](int s) { return sbase + s * C::STAGE + C::QBYTES; };
  auto sV = [&](int s) { return sbase + s * C::STAGE + 2 * C::QBYTES; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < 4; ++s) {
      mbar_init(bar(B_TMA_FULL + s), 1);
      mbar_init(bar(B_CONV_FULL + s), 128);
      mbar_init(bar(B_STAGE_EMPTY + s), 1);
    }
    mbar_init(bar(B_S_FULL), 1);
    mbar_init(bar(B_S_FREE), 128);
    mbar_init(bar(B_P_FULL), 128);
    mbar_init(bar(B_R_DONE), 1);
    mbar_init(bar(B_R_READY), 128);
    mbar_init(bar(B_O_FULL), 1);
    mbar_init(bar(B_O_FREE), 128);
    mbar_init(bar(B_DRAIN), 1);
    mbar_init(bar(B_TAB0), 128);
    mbar_init(bar(B_TAB0 + 1), 128);
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_addr(tmem_holder), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == kWarpTma && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == kWarpTma) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int issued[4] = {0, 0, 0, 0};
      for (int i = 0; i < n; ++i) {
        const int s = i % C::NS;
        if (i >= C::NS && !mbar_wait(bar(B_STAGE_EMPTY + s), ((i / C::NS) - 1) & 1)) break;
        mbar_arrive_expect_tx(bar(B_TMA_FULL + s), C::STAGE);
        const int t0 = i * T;
#pragma unroll
        for (int bx = 0; bx < DK / 64; ++bx) {
          tma_load_4d(sQ(s) + bx * T * 128, &tm_q, bar(B_TMA_FULL + s), bx * 64, h, t0, b);
          tma_load_4d(sK(s) + bx * T * 128, &tm_k, bar(B_TMA_FULL + s), bx * 64, h, t0, b);
        }
        tma_load_4d(sV(s), &tm_v, bar(B_TMA_FULL + s), dvb * kDVS, h, t0, b);
        issued[s]++;
      }
      // Every load this thread issued must have landed before the CTA may exit.
      for (int s = 0; s < C::NS; ++s)
        if (issued[s] > 0) mbar_wait(bar(B_TMA_FULL + s), (issued[s] - 1) & 1, kDrainBudget);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID_S = idesc_f16_f32(T, T, 0, 0);
      constexpr uint32_t ID_X = idesc_f16_f32(T, kDVS, 0, 1);
      constexpr uint32_t ID_R = idesc_f16_f32(C::MR, kDVS, 1, 1);
      const uint32_t tO = tmem + C::COL_O, tS = tmem + C::COL_S, tR = tmem + C::COL_R;
      bool ok = true;
      for (int i = 0; i < n && ok; ++i) {
        const int s = i % C::NS;
        ok = mbar_wait(bar(B_CONV_FULL + s), (i / C::NS) & 1);
        if (ok && i > 0) ok = mbar_wait(bar(B_S_FREE), (i - 1) & 1);
        if (!ok) break;
        tc_fence_after();
        // S'' = Qx Kz^T  (M = T rows r, N = T columns c, K = d_k)
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
          const uint32_t off = (kk / 4) * T * 128 + (kk % 4) * 32;
          mma_f16_ss(tS, sdesc_sw128(sQ(s) + off, 16, 1024), sdesc_sw128(sK(s) + off, 16, 1024), ID_S, kk > 0);
        }
        mma_commit(bar(B_S_FULL));
        ok = mbar_wait(bar(B_R_READY), i & 1);
        if (ok && i > 0) ok = mbar_wait(bar(B_O_FREE), (i - 1) & 1);
        if (!ok) break;
        tc_fence_after();
        // O = Qx R16  (cross-chunk term; K = d_k)
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
          const uint32_t off = (kk / 4) * T * 128 + (kk % 4) * 32;
          mma_f16_ss(tO, sdesc_sw128(sQ(s) + off, 16, 1024), sdesc_sw128(sR + kk * 2048, DK * 128, 1024), ID_X,
                     kk > 0);
        }
        // R += Kz^T V  (state increment; M = d_k rows in blocks of 128, K = T tokens)
#pragma unroll
        for (int blk = 0; blk < C::RBLK; ++blk) {
#pragma unroll
          for (int ks = 0; ks < T / 16; ++ks) {
            mma_f16_ss(tR + blk * kDVS, sdesc_sw128(sK(s) + blk * 2 * T * 128 + ks * 2048, T * 128, 1024),
                       sdesc_sw128(sV(s) + ks * 2048, T * 128, 1024), ID_R, 1);
          }
        }
        mma_commit(bar(B_R_DONE));
        ok = mbar_wait(bar(B_P_FULL), i & 1);
        if (!ok) break;
        tc_fence_after();
        // O += P V  (inner-chunk term; K = T tokens)
#pragma unroll
        for (int kk = 0; kk < T / 16; ++kk) {
          const uint32_t off = (kk / 4) * T * 128 + (kk % 4) * 32;
          mma_f16_ss(tO, sdesc_sw128(sP + off, 16, 1024), sdesc_sw128(sV(s) + kk * 2048, T * 128, 1024), ID_X, 1);
        }
        mma_commit(bar(B_O_FULL));
        mma_commit(bar(B_STAGE_EMPTY + s));
      }
      // Drain: every MMA issued above completes before TMEM is released.
      mma_commit(bar(B_DRAIN));
      mbar_wait(bar(B_DRAIN), 0, kDrainBudget);
    }
  } else if (warp >= kWarpConv0) {
    // ------------------------------------------------------------------ converters
    Converter<DK, T> cv;
    cv.init(threadIdx.x - 32 * kWarpConv0, hp);
    const bool xpos = (a.flags & RETNET_F_XPOS) != 0;
    bool ok = true;
    float mx = 0.f;  // largest magnitude rounded to fp16
    for (int i = 0; i < n && ok; ++i) {
      const int s = i % C::NS;
      const int bl = min(T, a.L - i * T);
      float2* base = tab + (i & 1) * (DK / 2);
      if (xpos) cv.put_base(base, i, a.pos0, hp);
      // The table buffer (i & 1) is complete once all 128 converters arrived; a thread that
      // rewrites it two chunks later has passed this wait, so every read of it is done.
      mbar_arrive(bar(B_TAB0 + (i & 1)));
      ok = mbar_wait(bar(B_TAB0 + (i & 1)), (i >> 1) & 1);
      if (ok) ok = mbar_wait(bar(B_TMA_FULL + s), (i / C::NS) & 1);
      if (!ok) break;
      cv.convert(sQ(s), sK(s), sV(s), base, xpos, log2g, bl, mx);
      fence_proxy_async_smem();
      mbar_arrive(bar(B_CONV_FULL + s));
    }
    report_fp16_range(mx);
  } else {
    // ------------------------------------------------------------------ TMEM warpgroup
    const uint32_t lane_off = static_cast<uint32_t>(32 * warp) << 16;
    const int my_row = (T == 128) ? 32 * warp + lane : (lane < 16 ? 16 * warp + lane : -1);
    // State rows (d_k) held by this thread's TMEM lane in each 128-row block.
    auto state_row = [&](int blk) -> int {
      if (DK == 64) return lane < 16 ? 16 * warp + lane : -1;
      return blk * 128 + 32 * warp + lane;
    };
    const int64_t bh = static_cast<int64_t>(b) * a.heads + h;
    const size_t srow = static_cast<size_t>(a.dv);
    float* sbase_g_out = a.state_out ? a.state_out + static_cast<size_t>(bh) * DK * a.dv + dvb * kDVS : nullptr;
    const float* sbase_g_in = a.state_in ? a.state_in + static_cast<size_t>(bh) * DK * a.dv + dvb * kDVS : nullptr;

    // Write R (64 fp32 of one state row) as fp16 into the cross-term operand (MN-major,
    // rows = d_k, 128 B = 64 d_v per row, 128-byte swizzle).
    float mx = 0.f;  // largest magnitude rounded to fp16 (P and the state copy)
    auto put_r16 = [&](int dk, const float* rv) {
#pragma unroll
      for (int c = 0; c < 64; ++c) mx = absmax(mx, sd * rv[c]);
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8)
        st_shared_v4(sR + sw128(dk, c8), pack_f16x2(sd * rv[8 * c8 + 0], sd * rv[8 * c8 + 1]),
                     pack_f16x2(sd * rv[8 * c8 + 2], sd * rv[8 * c8 + 3]),
                     pack_f16x2(sd * rv[8 * c8 + 4], sd * rv[8 * c8 + 5]),
                     pack_f16x2(sd * rv[8 * c8 + 6], sd * rv[8 * c8 + 7]));
    };

    // Initial state: master = gamma^(b'_0) R_in, fp16 copy = R_in.
    {
      const int bl0 = min(T, a.L);
      const float g0 = decay_pow(log2g, bl0);
#pragma unroll 1
      for (int blk = 0; blk < C::RBLK; ++blk) {
        const int dk = state_row(blk);
        float rv[kDVS];
#pragma unroll
        for (int c = 0; c < kDVS; ++c) rv[c] = 0.f;
        if (dk >= 0 && sbase_g_in) {
#pragma unroll
          for (int c4 = 0; c4 < kDVS / 4; ++c4) {
            const float4 x = *reinterpret_cast<const float4*>(sbase_g_in + dk * srow + 4 * c4);
            rv[4 * c4] = x.x; rv[4 * c4 + 1] = x.y; rv[4 * c4 + 2] = x.z; rv[4 * c4 + 3] = x.w;
          }
        }
        if (dk >= 0) put_r16(dk, rv);
        uint32_t w64[4][16];
#pragma unroll
        for (int e = 0; e < kDVS; ++e) w64[e / 16][e % 16] = __float_as_uint(g0 * rv[e]);
        tmem_st_wait(tmem + C::COL_R + blk * kDVS + lane_off, w64);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(B_R_READY));
    }

    bool ok = true;
    for (int i = 0; i < n && ok; ++i) {
      const int t0 = i * T;
      const int bl = min(T, a.L - t0);
      const bool last = (i == n - 1);
      // (1) P = S'' gamma^(-b') on and below the diagonal, fp16, into the K-major A tile.
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_S_FULL), i & 1));
      if (!ok) break;
      tc_fence_after();
      {
        const float ginv = exp2f(-static_cast<float>(bl) * log2g) * sd;
#pragma unroll
        for (int half = 0; half < T / 64; ++half) {
          uint32_t u[4][16];
          tmem_ld_wait(tmem + C::COL_S + half * 64 + lane_off, u);
          if (my_row >= 0) {
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8) {
              uint32_t pk[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int c0 = half * 64 + 8 * c8 + 2 * e;
                const float p0 = (c0 <= my_row) ? __uint_as_float(u[c8 / 2][(8 * c8 + 2 * e) % 16]) * ginv : 0.f;
                const float p1 = (c0 + 1 <= my_row) ? __uint_as_float(u[c8 / 2][(8 * c8 + 2 * e + 1) % 16]) * ginv : 0.f;
                mx = absmax(absmax(mx, p0), p1);
                pk[e] = pack_f16x2(p0, p1);
              }
              st_shared_v4(sP + half * T * 128 + sw128(my_row, c8), pk[0], pk[1], pk[2], pk[3]);
            }
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(B_S_FREE));
      mbar_arrive(bar(B_P_FULL));

      // (2) State: R_i (TMEM, after the increment) -> fp16 copy; gamma^(b'_{i+1}) R_i -> TMEM.
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_R_DONE), i & 1));
      if (!ok) break;
      tc_fence_after();
      {
        const int bln = last ? 0 : min(T, a.L - t0 - T);
        const float gn = decay_pow(log2g, bln);
#pragma unroll 1
        for (int blk = 0; blk < C::RBLK; ++blk) {
          const int dk = state_row(blk);
          uint32_t u[4][16];
          tmem_ld_wait(tmem + C::COL_R + blk * kDVS + lane_off, u);
          float rv[kDVS];
#pragma unroll
          for (int c = 0; c < kDVS; ++c) rv[c] = __uint_as_float(u[c / 16][c % 16]);
          if (!last) {
            if (dk >= 0) put_r16(dk, rv);
            uint32_t w64[4][16];
#pragma unroll
            for (int e = 0; e < kDVS; ++e) w64[e / 16][e % 16] = __float_as_uint(gn * rv[e]);
            tmem_st_wait(tmem + C::COL_R + blk * kDVS + lane_off, w64);
          } else if (dk >= 0 && sbase_g_out) {
#pragma unroll
            for (int c4 = 0; c4 < kDVS / 4; ++c4)
              *reinterpret_cast<float4*>(sbase_g_out + dk * srow + 4 * c4) =
                  make_float4(rv[4 * c4], rv[4 * c4 + 1], rv[4 * c4 + 2], rv[4 * c4 + 3]);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar(B_R_READY));
      }

      // (3) Epilogue: o = O * s / c_p, stored as the output dtype.
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_O_FULL), i & 1));
      if (!ok) break;
      tc_fence_after();
      {
        uint32_t u[4][16];
        tmem_ld_wait(tmem + C::COL_O + lane_off, u);
        tc_fence_before();
        mbar_arrive(bar(B_O_FREE));
        if (my_row >= 0 && my_row < bl) {
          const float f = row_factor(hp.gamma[h], DK, a.pos0 + t0 + my_row, a.flags) / sd;
          const int64_t orow = ((static_cast<int64_t>(b) * a.L + t0 + my_row) * a.heads + h) * a.dv + dvb * kDVS;
          Tout* dst = static_cast<Tout*>(a.o) + orow;
          if constexpr (sizeof(Tout) == 2) {
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8) {
              uint32_t pk[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                __nv_bfloat162 v2 = __floats2bfloat162_rn(f * __uint_as_float(u[c8 / 2][(8 * c8 + 2 * e) % 16]),
                                                          f * __uint_as_float(u[c8 / 2][(8 * c8 + 2 * e + 1) % 16]));
                pk[e] = *reinterpret_cast<uint32_t*>(&v2);
              }
              *reinterpret_cast<uint4*>(dst + 8 * c8) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
          } else {
#pragma unroll
            for (int c4 = 0; c4 < 16; ++c4)
              *reinterpret_cast<float4*>(dst + 4 * c4) =
                  make_float4(f * __uint_as_float(u[c4 / 4][(4 * c4) % 16]), f * __uint_as_float(u[c4 / 4][(4 * c4 + 1) % 16]),
                              f * __uint_as_float(u[c4 / 4][(4 * c4 + 2) % 16]), f * __uint_as_float(u[c4 / 4][(4 * c4 + 3) % 16]));
          }
        }
      }
    }
    report_fp16_range(mx);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ============================================================================================
// Pipelined kernel.  The work of a chunk of B = nb * T tokens is split into units
// (u, w): row block u (T query rows) against column block w <= u (T key/value rows).
// Sub-block-local scaled operands: rows r and columns c are local to their T-row block and
//   Qx_u = gamma^(r+1) (.) rot(q),   Kz_w = gamma^(T-1-c) (.) rot(k)   (fp16),
// so that, with S'' = Qx_u Kz_w^T = gamma^(T+r-c) (Q K^T),
//   P_{u,w} = S'' * gamma^((u-w-1) T)      (causal mask on the diagonal block only),
//   O_u = sum_{w<=u} P_{u,w} V_w,   X_u = Qx_u R16 (the chunk-start state),
//   o = (O_u + gamma^(u T) X_u) * s / c_p            (X goes straight into O when nb = 1),
//   R_i = gamma^b' R_{i-1} + sum_w gamma^(b'-(w+1)T) Kz_w^T V_w   (taken in Horner form).
// fp16 operands stay in range when gamma^T >= 2^-12.  Roles:
//   warps 0-3        P/epilogue group: S -> P for each unit; epilogue of each finished row block.
//   next 4*RBLK warps state group: the chunk state R in registers (one d_k row of the 64-wide
//                    d_v slice per thread); Horner update per column block of the last row block;
//                    fp16 copy of R for the next chunk's cross terms.
//   4 warps          converters: rotate/scale/convert each unit's Q, K, V tiles in place.
//   1 warp TMA, 1 warp MMA issuer (one unit ahead: S and dR of unit k+1 before X/PV of unit k).
// ============================================================================================

template <int DK, int T, int DVS, bool PRE = false, bool FUSE = false, bool HL = false, bool PS = false>
struct Cfg3 {
  static constexpr int NDV = DVS / 64;              // 64-column boxes of the d_v slice
  static constexpr int RBLK = DK > 128 ? 2 : 1;     // 128-row blocks of the state increment
  static constexpr int MR = DK >= 128 ? 128 : 64;
  // RTM: the fp32 state lives in tensor memory (the increment's columns) and each state
  // increment accumulates into it (four state warps, a thread per TMEM lane, all its 128-row
  // blocks); otherwise the state group holds it in registers, one thread per (d_k row, 64
  // columns).  Taken for the 128-wide slice and for d_k = 256 (where eight register warps
  // would push the CTA to 18 warps and 96 registers).
  static constexpr bool RTM = DVS == 128 || DK == 256;
  static constexpr int WARPS_S = RTM ? 4 : 4 * RBLK * NDV;
  static constexpr int BPT = RTM ? RBLK : 1;  // 128-row state blocks per state thread
  static constexpr int WARP_S0 = 4;
  static constexpr int WARP_CONV0 = WARP_S0 + WARPS_S;
  static constexpr int CONV_WARPS = PRE ? 0 : 4;  // PRE: tiles arrive converted (pre-pass)
  static constexpr int NCONV = 32 * CONV_WARPS;
  // PRE with FUSE: four epilogue warps take O (and X) out of TMEM and run the GroupNorm, so
  // that the P warps only make P (the plain epilogue is too short to pay for the warps)
  static constexpr int EPI_WARPS = (PRE && FUSE) ? 4 : 0;
  static constexpr int WARP_EPI0 = WARP_CONV0 + CONV_WARPS;
  static constexpr int WARP_TMA = WARP_EPI0 + EPI_WARPS;
  static constexpr int WARP_MMA = WARP_TMA + 1;
  static constexpr int THREADS = 32 * (WARP_MMA + 1);
  static constexpr int QBYTES = T * DK * 2;
  static constexpr int VBYTES = T * DVS * 2;
  // HL (split operands): every rounded fp16 operand -- the scaled, rotated q and k, the masked
  // scores P and the state copy -- is held as hi + lo, hi = fp16(x), lo = fp16(x - hi), so a
  // product of two of them keeps ~22 significant bits; the stage holds [Q hi][K hi][V][Q lo][K lo].
  static constexpr int QT = HL ? 2 : 1;
  static constexpr int PBYTES = T * T * 2;
  // PS (P tiles computed by the P pass): a stage holds the unit's V and P tiles, [V][P]; Q (for
  // the cross term, once a row block) and K (for the state increment, last row block) get areas
  // of their own, two slots each; there is no P buffer of the P warps.
  static constexpr int QSLOTS = 2, KSLOTS = 2;
  static constexpr int AREAS = PS ? (QSLOTS + KSLOTS) * QBYTES : 0;
  static constexpr int STAGE = PS ? VBYTES + PBYTES : 2 * QBYTES * QT + VBYTES;
  static constexpr int RBYTES = DK * DVS * 2;
  static constexpr int PB = PS ? 0 : PBYTES * QT;  // one P buffer (hi, then lo)
  static constexpr int RB = RBYTES * QT;  // one fp16 state buffer (hi, then lo)
  // TMEM: O[2] (DVS columns each), X[XBUF] (cross accumulators; none when the slice is 128
  // wide, which then runs one sub-block per chunk only), S[SBUF] (T columns), dR[DRBUF]
  // (RBLK x DVS columns).
  static constexpr int XBUF = DVS == 64 ? 2 : 0;
  static constexpr int SBUF = ((2 + XBUF) * DVS + 2 * T + RBLK * DVS <= 512) ? 2 : 1;
  static constexpr int DRBUF = ((2 + XBUF) * DVS + SBUF * T + 2 * RBLK * DVS <= 512) ? 2 : 1;
  static constexpr int COL_O = 0;
  static constexpr int COL_X = 2 * DVS;
  static constexpr int COL_S = (2 + XBUF) * DVS;
  static constexpr int COL_DR = COL_S + SBUF * T;
  static constexpr int USED = COL_DR + DRBUF * RBLK * DVS;
  static constexpr int TMEM_COLS = USED <= 128 ? 128 : (USED <= 256 ? 256 : 512);
  // shared memory: stages, P[PBUF], R16[RBUF], rotation tables (Q and K, double-buffered),
  // barriers.  A second fp16 state buffer is kept only while three stages still fit.
  static constexpr int NBARS = 3 * 6 + 2 * 10 + 1 + 2 + 2 + 4 * 2;
  // FUSE (GroupNorm + gate in the epilogue): per-row (mean, M2) of every CTA of the cluster
  // (the d_v slices of a head, at most kMaxCluster), double-buffered by row block.
  static constexpr int XBYTES = FUSE ? 2 * kMaxCluster * T * 8 : 0;
  static constexpr int TABBYTES = 2 * 2 * (DK / 2) * 8;
  static constexpr int BUDGET = 227 * 1024 - 1024;
  static constexpr int TAIL = TABBYTES + NBARS * 8 + 16 + XBYTES;
  // Buffer counts.  A second fp16 state buffer takes the cross term of chunk i off the state
  // group's path to chunk i + 1 (with one buffer the copy of R_i waits for that MMA), so it is
  // preferred as long as three stages remain, over a second P buffer.
  static constexpr int ns_for(int pbuf, int rbuf) { return (BUDGET - (pbuf * PB + rbuf * RB + AREAS + TAIL)) / STAGE; }
  static constexpr int PBUF0 = (2 * STAGE + 2 * PB + RB + TAIL <= BUDGET) ? 2 : 1;
  static constexpr int NS_R2 = ns_for(PBUF0, 2);
  static constexpr int NS_R1 = ns_for(PBUF0, 1);
  static constexpr int RBUF0 = (NS_R2 >= 3 || NS_R1 < 3) && NS_R2 >= 2 ? 2 : 1;
  static constexpr bool TRADE = RBUF0 == 1 && PBUF0 == 2 && ns_for(1, 2) >= 3;
  static constexpr int PBUF = TRADE ? 1 : PBUF0;
  static constexpr int RBUF = TRADE ? 2 : RBUF0;
  static constexpr int FIXED = PBUF * PB + RBUF * RB + AREAS + TAIL;
  static constexpr int NS_FIT = (BUDGET - FIXED) / STAGE;
  static constexpr int NS_MAX = PS ? 6 : 4;  // stage barriers exist for six
  static constexpr int NS = NS_FIT > NS_MAX ? NS_MAX : NS_FIT;
  static constexpr int SMEM = NS * STAGE + FIXED + 1024;
  // split operands at d_k = 256 leave room for one stage only (the units then run in turn)
  static constexpr bool FITS = NS >= (HL ? 1 : 2) && USED <= 512 && (DVS == 64 || DVS == 128) && (!RTM || DRBUF == 1) &&
                               (!HL || (T == 64 && DVS == 64)) && (!PS || (PRE && !HL && !FUSE));
  // Columns per TMEM load batch: 18 warps leave 96 registers a thread (five warps share one
  // sub-partition's register file), too few to hold 64 loaded columns next to the state.
  static constexpr int LDW = THREADS > 512 ? 32 : 64;
};

// Barrier slots of the pipelined kernel ([2] = indexed by buffer).
enum : int {
  Q_TMA_FULL = 0,      // [6] stage landed (TMA transaction count)
  Q_CONV_FULL = 6,     // [6] stage converted (128 converters)
  Q_STAGE_EMPTY = 12,  // [6] stage consumed (MMA commit)
  Q_S_FULL = 18,       // [2] S'' of a unit in TMEM (commit)
  Q_S_FREE = 20,       // [2] S read by the P group
  Q_P_FULL = 22,       // [2] P in shared memory
  Q_P_FREE = 24,       // [2] P consumed by the P V product (commit)
  Q_DR_FULL = 26,      // [2] state increment Kz^T V in TMEM (commit)
  Q_DR_FREE = 28,      // [2] increment read by the state group
  Q_R16_FULL = 30,     // [2] fp16 chunk-start state written (state group)
  Q_R16_FREE = 32,     // [2] every cross term of that chunk done (commit)
  Q_O_FULL = 34,       // [2] O (and X) of a row block complete (commit)
  Q_O_FREE = 36,       // [2] O/X read by the epilogue
  Q_DRAIN = 38,
  Q_TAB = 39,          // [2] rotation tables written (converters)
  Q_XFULL = 41,        // [2] FUSE: the row statistics of every CTA of the cluster have landed here
  Q_QA_FULL = 43,      // [2] PS: Q tile of a row block in its area slot (TMA)
  Q_QA_FREE = 45,      // [2] PS: that row block's cross term done (commit)
  Q_KA_FULL = 47,      // [2] PS: K tile of a last-row unit in its area slot (TMA)
  Q_KA_FREE = 49       // [2] PS: that unit's state increment done (commit)
};

__device__ __forceinline__ float2 cpow_mul(float2 base, float2 step, int n) {
  for (int i = 0; i < n; ++i) base = cmul(base, step);
  return base;
}

// s / c_p of the normalisations in fp32 (see row_factor in common.cuh; relative error a few ulp).
__device__ __forceinline__ float row_factor_f32(float gamma, float sqrt_dk_inv, int64_t p, uint32_t flags) {
  float f = (flags & RETNET_F_SCALE_SQRT_D) ? sqrt_dk_inv : 1.f;
  if (flags & RETNET_F_NORM_D) {
    const float om = 1.f - gamma;  // exact for gamma >= 1/2
    const float sum = -expm1f(static_cast<float>(p + 1) * log1pf(-om)) / om;
    f *= rsqrtf(sum);
  }
  return f;
}

// Walks the units of the CTA's part of the sequence in the order every role processes them:
// for chunk i < c_hi, for row block u < nbw_i, for column block w <= u  (nbw_i = ceil(b'_i / T)).
// Chunks below c_lo are state replay only: just their last row block (u = nbw_i - 1), whose
// units carry the state increments.
template <int T, int SM>
struct UnitIter {
  static constexpr bool SEG = SM != SEG_NONE;
  static constexpr bool PRE = SM == SEG_REPLAY || SM == SEG_STATE;  // some chunks update the state only
  int L, nb;         // sequence length, sub-blocks per full chunk
  int lo, hi;        // first output chunk (chunks below only update the state), end (SEG only)
  int i, u, w;       // current unit
  int nbw, bl;       // sub-blocks and length of chunk i
  int k;             // unit sequence number (stages, TMA, conversion)
  int kf_;           // sequence number among output units (PRE only; equals k otherwise)
  int rb;            // row-block sequence number among output units (O/X buffers)
  int dr;            // sequence number of state-increment units (u == nbw - 1)
  __device__ void start(int L_, int nb_, int first, int c_lo_, int c_hi_) {
    L = L_;
    nb = nb_;
    lo = c_lo_;
    hi = c_hi_;
    i = SEG ? first : 0;
    k = 0; kf_ = 0; rb = 0; dr = 0;
    if (valid()) set_chunk();
  }
  __device__ void set_chunk() {
    bl = min(nb * T, L - i * nb * T);
    nbw = (bl + T - 1) / T;
    u = pre() ? nbw - 1 : 0;
    w = 0;
  }
  __device__ bool valid() const { return (!SEG || i < hi) && i * nb * T < L; }
  __device__ bool pre() const { return PRE && i < lo; }     // state update only
  __device__ int kf() const { return PRE ? kf_ : k; }
  __device__ bool last_row() const { return u == nbw - 1; }  // this unit carries a state increment
  __device__ bool rb_done() const { return w == u; }         // last unit of its row block
  __device__ int t0() const { return i * nb * T; }          // chunk start (token)
  __device__ void next() {
    if (last_row()) ++dr;
    if (PRE && !pre()) ++kf_;
    ++k;
    if (w < u) { ++w; return; }
    if (!pre()) ++rb;
    w = 0;
    if (u + 1 < nbw) { ++u; return; }
    ++i;
    if (valid()) set_chunk();
  }
};

// Converter role of the pipelined kernel: like Converter, with the sub-block-local row scales
// and separate rotation bases for the unit's query rows (block u) and key rows (block w).
// NC threads; thread lt owns 16-byte column slot cs = lt % CS and rows r0 + RS k.  The row
// scale is carried inside the rotation factor: F_q(r) = gamma^(r+1) e^{i (p_r) theta_j} and
// F_k(c) = gamma^(T-1-c) e^{i (p_c) theta_j}, each advanced by one complex product per row step.
template <int DK, int T, int NC, int NDV>
struct UnitConverter {
  static constexpr int CS = DK / 8;   // 16-byte column slots across the DK/64 boxes
  static constexpr int RS = NC / CS;  // row step of one thread
  static constexpr int NR = T / RS;   // rows per thread
  static constexpr int G = NR < 4 ? NR : 4;  // rows per load batch
  static constexpr int VR = NC / 8;   // V rows per pass (8 slots of one 64-column box)
  static constexpr int VP = T / VR;   // V passes
  static constexpr int VG = VP < 4 ? VP : 4;
  static_assert(NR >= 1 && NR % G == 0 && VP >= 1 && VP % VG == 0, "converter tiling");
  float2 W[4], Z[4];                  // e^{i r0 theta_j}, e^{i RS theta_j} for the thread's pairs
  float2 cur, stepT, stepB;           // table producer (lt < DK/2): chunk base, e^{iT theta}, e^{iB theta}
  int cs, r0, lt, cur_chunk;
  bool conv_v;                        // V arrives as bf16 (converted here) rather than fp16

  __device__ void init(int lt_, int nb, const HeadParams& hp) {
    lt = lt_;
    cs = lt % CS;
    r0 = lt / CS;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const float th = hp.theta[4 * cs + jj];
      float sn, c;
      sincosf(static_cast<float>(r0) * th, &sn, &c);
      W[jj] = make_float2(c, sn);
      sincosf(static_cast<float>(RS) * th, &sn, &c);
      Z[jj] = make_float2(c, sn);
    }
    cur = stepT = stepB = make_float2(1.f, 0.f);
    cur_chunk = -1;
    conv_v = true;
    if (lt < DK / 2) {
      float sn, c;
      xpos_sincos(T, hp.theta[lt], &sn, &c);
      stepT = make_float2(c, sn);
      xpos_sincos(static_cast<int64_t>(nb) * T, hp.theta[lt], &sn, &c);
      stepB = make_float2(c, sn);
    }
  }

  // Rotation bases e^{i p theta_j} of the unit's query rows (p = pos0 + t0 + uT) and key rows
  // (p = pos0 + t0 + wT), j = lt.  The chunk base advances by an fp32 complex product and is
  // recomputed from the fp64-reduced angle every 64 chunks (drift below ~1e-5 rad).
  __device__ void put_bases(float2* tq, float2* tk, int chunk, int u, int w, int t0, int64_t pos0,
                            const HeadParams& hp) {
    if (lt >= DK / 2) return;
    if (chunk != cur_chunk) {
      if ((chunk & 63) == 0 || cur_chunk < 0) {
        float sn, c;
        xpos_sincos(pos0 + t0, hp.theta[lt], &sn, &c);
        cur = make_float2(c, sn);
      } else {
        cur = cmul(cur, stepB);
      }
      cur_chunk = chunk;
    }
    tq[lt] = cpow_mul(cur, stepT, u);
    tk[lt] = cpow_mul(cur, stepT, w);
  }

  // In place: q -> gamma^(r+1) rot(q), k -> gamma^(T-1-r) rot(k) as fp16 (r local); v -> fp16.
  // WITH_Q = false (state replay) leaves the Q tile alone.
  // zmul multiplies the K row scales (the state pre-pass decays K to its segment's end).
  // HL: the tiles take the fp16 hi parts, sql / skl (same layout) the lo parts.
  // mx: the largest magnitude rounded to fp16 so far (range check, reported at the end).
  template <bool WITH_Q, bool HL = false>
  __device__ void convert(uint32_t sq, uint32_t sk, uint32_t sv, const float2* bq, const float2* bk, bool xpos,
                          float log2g, float& mx, float zmul = 1.f, uint32_t sql = 0, uint32_t skl = 0) const {
    const uint32_t box = (cs / 8) * T * 128;
    const uint32_t chunk = cs % 8;
    const float xstep = decay_pow(log2g, RS), zstep = exp2f(-static_cast<float>(RS) * log2g);
    const float xi0 = decay_pow(log2g, r0 + 1), zeta0 = decay_pow(log2g, T - 1 - r0) * zmul;
    float2 Fq[4], Fk[4], Zq[4], Zk[4];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const float2 fq = xpos ? cmul(bq[4 * cs + jj], W[jj]) : make_float2(1.f, 0.f);
      const float2 fk = xpos ? cmul(bk[4 * cs + jj], W[jj]) : make_float2(1.f, 0.f);
      Fq[jj] = make_float2(xi0 * fq.x, xi0 * fq.y);
      Fk[jj] = make_float2(zeta0 * fk.x, zeta0 * fk.y);
      Zq[jj] = make_float2(xstep * Z[jj].x, xstep * Z[jj].y);
      Zk[jj] = make_float2(zstep * Z[jj].x, zstep * Z[jj].y);
    }
    // rows a load batch: split operands and 128-row units (more live values a row) ran faster
    // with two (1.13x and 1.05x) and the plain 64-row path the same with two or four
    constexpr int GB = (HL || T == 128) ? (NR < 2 ? NR : 2) : G;
#pragma unroll 1
    for (int kg = 0; kg < NR; kg += GB) {
      uint32_t q4[GB][4], k4[GB][4];
#pragma unroll
      for (int k = 0; k < GB; ++k) {
        const uint32_t off = box + sw128(r0 + RS * (kg + k), chunk);
        if (WITH_Q) ld_shared_v4(sq + off, q4[k][0], q4[k][1], q4[k][2], q4[k][3]);
        ld_shared_v4(sk + off, k4[k][0], k4[k][1], k4[k][2], k4[k][3]);
      }
#pragma unroll
      for (int k = 0; k < GB; ++k) {
        uint32_t qo[4], ko[4], ql[4], kl[4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          if (WITH_Q) {
            const float q0 = __uint_as_float(q4[k][jj] << 16), q1 = __uint_as_float(q4[k][jj] & 0xffff0000u);
            const float x0 = q0 * Fq[jj].x - q1 * Fq[jj].y, x1 = q0 * Fq[jj].y + q1 * Fq[jj].x;
            mx = absmax(absmax(mx, x0), x1);
            if (HL) {
              split_f16x2(x0, x1, qo[jj], ql[jj]);
            } else {
              qo[jj] = pack_f16x2(x0, x1);
            }
            Fq[jj] = cmul(Fq[jj], Zq[jj]);
          }
          const float k0 = __uint_as_float(k4[k][jj] << 16), k1 = __uint_as_float(k4[k][jj] & 0xffff0000u);
          const float y0 = k0 * Fk[jj].x - k1 * Fk[jj].y, y1 = k0 * Fk[jj].y + k1 * Fk[jj].x;
          mx = absmax(absmax(mx, y0), y1);
          if (HL) {
            split_f16x2(y0, y1, ko[jj], kl[jj]);
          } else {
            ko[jj] = pack_f16x2(y0, y1);
          }
          Fk[jj] = cmul(Fk[jj], Zk[jj]);
        }
        const uint32_t off = box + sw128(r0 + RS * (kg + k), chunk);
        if (WITH_Q) st_shared_v4(sq + off, qo[0], qo[1], qo[2], qo[3]);
        st_shared_v4(sk + off, ko[0], ko[1], ko[2], ko[3]);
        if (HL) {
          if (WITH_Q) st_shared_v4(sql + off, ql[0], ql[1], ql[2], ql[3]);
          st_shared_v4(skl + off, kl[0], kl[1], kl[2], kl[3]);
        }
      }
    }
    // V: each 64-column box, slot lt % 8, rows lt / 8 + VR k.
    if (!conv_v) return;
#pragma unroll 1
    for (int kg = 0; kg < NDV * VP; kg += VG) {
      const uint32_t vb = sv + (kg / VP) * T * 128;
      uint32_t v4[VG][4];
#pragma unroll
      for (int k = 0; k < VG; ++k)
        ld_shared_v4(vb + sw128(lt / 8 + VR * (kg % VP + k), lt % 8), v4[k][0], v4[k][1], v4[k][2], v4[k][3]);
#pragma unroll
      for (int k = 0; k < VG; ++k) {
        uint32_t vo[4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const float v0 = __uint_as_float(v4[k][jj] << 16), v1 = __uint_as_float(v4[k][jj] & 0xffff0000u);
          mx = absmax(absmax(mx, v0), v1);
          vo[jj] = pack_f16x2(v0, v1);
        }
        st_shared_v4(vb + sw128(lt / 8 + VR * (kg % VP + k), lt % 8), vo[0], vo[1], vo[2], vo[3]);
      }
    }
  }
};

template <int DK, int T, int DVS, int SM, bool PRE, bool FUSE, typename Tout, bool HL = false, bool PS = false>
__global__ void __launch_bounds__(Cfg3<DK, T, DVS, PRE, FUSE, HL, PS>::THREADS, 1)
    tc_chunkwise_pipe_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_ql,
                             const __grid_constant__ CUtensorMap tm_kl, TcArgs a, HeadParams hp) {
  // tm_ql, tm_kl: the lo parts of pre-converted split operands (HL with PRE); with PS, tm_ql is
  // the map of the P tiles ([tile][T][T] fp16, box T x T) and tm_kl is unused; unused otherwise.
  using C = Cfg3<DK, T, DVS, PRE, FUSE, HL, PS>;
  static_assert(!PS || (PRE && !HL && !FUSE && SM == SEG_NONE), "P tiles from the P pass: pre-converted, unsplit");
  static_assert(!FUSE || (SM == SEG_NONE && DVS == 64), "the fused epilogue runs unsplit, 64-column slices");
  static_assert(!HL || SM == SEG_NONE, "split operands run without sequence segments");
  // Stage ready for the MMAs: converted in place, or (PRE) landed already converted.
  constexpr int Q_READY = PRE ? Q_TMA_FULL : Q_CONV_FULL;
  constexpr bool SEG = SM != SEG_NONE;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - raw_addr);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_dvb = a.dv / DVS;
  // Grid: (slice [x segment], head, batch); the output pass of the two-pass form puts the
  // segment in z instead (segment-major), so that its segment-0 CTAs, which do not need the
  // pre-pass, are dispatched first.
  const int dvb = (SEG && SM != SEG_FROM_WS) ? blockIdx.x % n_dvb : blockIdx.x, h = blockIdx.y;
  const int b = (SM == SEG_FROM_WS) ? blockIdx.z % a.batch : blockIdx.z;
  const float log2g = hp.log2g[h];
  const int nb = a.nb;
  // The CTA visits chunks [c_first, c_hi); those below c_lo only update the state (the replay
  // of earlier segments); outputs start at c_lo.
  // Without segments the bounds are compile-time constants and every such branch folds away.
  static_assert(SM != SEG_STATE, "the segment-state pass has its own kernel");
  int seg = 0, s_lo = 0, s_hi = 0x7fffffff;
  if constexpr (SEG) {
    seg = (SM == SEG_FROM_WS) ? blockIdx.z / a.batch : blockIdx.x / n_dvb;
    s_lo = a.seg_lo[0];
    s_hi = a.seg_hi[0];
#pragma unroll
    for (int i = 1; i < 4; ++i)  // (a constant-index select keeps the kernel parameters in place)
      if (seg == i) {
        s_lo = a.seg_lo[i];
        s_hi = a.seg_hi[i];
      }
  }
  const int c_first = (SM == SEG_REPLAY) ? 0 : s_lo;
  const int c_lo = s_lo;
  const int c_hi = s_hi;
  // Start state of a two-pass output segment: state_in carried over the earlier segments,
  // R = gamma^len_j R + W_j (row dk, columns [col, col + n) of the slice, n a multiple of 32).
  // The states W_j are read two at a time with both loads in flight (they do not depend on the
  // running sum), 32 columns at a time; a loop that read one state after the other paid one
  // memory latency per state and column group.
  auto start_state = [&](int dk, int col, int n, float* R) {
    const int64_t bh = static_cast<int64_t>(b) * a.heads + h;
    for (int c = 0; c < n; ++c) R[c] = 0.f;
    if (a.state_in) {
      const float* src = a.state_in + static_cast<size_t>(bh) * DK * a.dv + col + static_cast<size_t>(dk) * a.dv;
      for (int c4 = 0; c4 < n / 4; ++c4) {
        const float4 x = *reinterpret_cast<const float4*>(src + 4 * c4);
        R[4 * c4] = x.x; R[4 * c4 + 1] = x.y; R[4 * c4 + 2] = x.z; R[4 * c4 + 3] = x.w;
      }
    }
    if constexpr (SM == SEG_FROM_WS) {
      int n_before = a.sub_before[0];
#pragma unroll
      for (int t = 1; t < 4; ++t)  // constant-index selects, as above
        if (t == seg) n_before = a.sub_before[t];
      if (n_before > 0) griddep_wait();  // the pre-pass states are complete and visible
      const size_t plane = static_cast<size_t>(a.batch) * a.heads * DK * a.dv;
      const float* w0base = a.ws + static_cast<size_t>(bh) * DK * a.dv + col + static_cast<size_t>(dk) * a.dv;
      auto factor = [&](int j) {  // gamma^len_j, len_j = the tokens of sub-segment j
        int chunks_j = 0;
#pragma unroll
        for (int t = 0; t < kMaxSub; ++t)
          if (t == j) chunks_j = a.sub_hi[t] - a.sub_lo[t];
        return exp2f(static_cast<float>(chunks_j * nb * T) * log2g);
      };
      for (int j = 0; j < n_before; j += 2) {
        const bool two = j + 1 < n_before;
        const int j1 = two ? j + 1 : j;  // a valid state either way; its terms count only if two
        const float g0 = factor(j), g1 = factor(j1);
        const float* w0 = w0base + j * plane;
        const float* w1 = w0base + j1 * plane;
        for (int c32 = 0; c32 < n; c32 += 32) {
          float4 x0[8], x1[8];
#pragma unroll
          for (int c4 = 0; c4 < 8; ++c4) {
            x0[c4] = *reinterpret_cast<const float4*>(w0 + c32 + 4 * c4);
            x1[c4] = *reinterpret_cast<const float4*>(w1 + c32 + 4 * c4);
          }
#pragma unroll
          for (int c4 = 0; c4 < 8; ++c4) {
            float* r = R + c32 + 4 * c4;
            r[0] = fmaf(g0, r[0], x0[c4].x);
            r[1] = fmaf(g0, r[1], x0[c4].y);
            r[2] = fmaf(g0, r[2], x0[c4].z);
            r[3] = fmaf(g0, r[3], x0[c4].w);
            if (two) {
              r[0] = fmaf(g1, r[0], x1[c4].x);
              r[1] = fmaf(g1, r[1], x1[c4].y);
              r[2] = fmaf(g1, r[2], x1[c4].z);
              r[3] = fmaf(g1, r[3], x1[c4].w);
            }
          }
        }
      }
    }
  };
  const float sd = rsqrtf(static_cast<float>(DK));  // carried by P and the fp16 state copy

  const uint32_t sP0 = sbase + C::NS * C::STAGE;
  const uint32_t sR0 = sP0 + C::PBUF * C::PB;
  const uint32_t sA0 = sR0 + C::RBUF * C::RB;  // PS: Q area slots, then K area slots
  const int tail_off = C::NS * C::STAGE + C::PBUF * C::PB + C::RBUF * C::RB + C::AREAS;
  float2* tab = reinterpret_cast<float2*>(gbase + tail_off);
  uint64_t* bars = reinterpret_cast<uint64_t*>(gbase + tail_off + C::TABBYTES);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + C::NBARS);
  auto bar = [&](int i) { return smem_addr(bars + i); };
  // FUSE: row statistics from the cluster, [slot][cta rank][row] of (mean, M2) over 64 columns.
  const uint32_t xbuf0 = smem_addr(tmem_holder) + 16;
  auto xaddr = [&](int slot, int rank, int row) {
    return xbuf0 + static_cast<uint32_t>(((slot * kMaxCluster + rank) * T + row) * 8);
  };
  const int n_cl = a.dv / DVS;  // cluster size under FUSE: every d_v slice of the head
  auto sQ = [&](int s) { return sbase + s * C::STAGE; };
  auto sK = [&](int s) { return sbase + s * C::STAGE + C::QBYTES; };
  auto sV = [&](int s) { return sbase + s * C::STAGE + (PS ? 0 : 2 * C::QBYTES); };
  auto sQa = [&](int slot) { return sA0 + slot * C::QBYTES; };                 // PS
  auto sKa = [&](int slot) { return sA0 + (C::QSLOTS + slot) * C::QBYTES; };   // PS
  // HL: lo parts of Q and K after V in the stage; P and the state copy keep their lo part
  // right after the hi part of the same buffer
  auto sQl = [&](int s) { return sbase + s * C::STAGE + 2 * C::QBYTES + C::VBYTES; };
  auto sKl = [&](int s) { return sbase + s * C::STAGE + 3 * C::QBYTES + C::VBYTES; };
  auto sPs = [&](int s) { return sbase + s * C::STAGE + C::VBYTES; };  // PS: the unit's P tile
  auto sP = [&](int k) { return sP0 + (k % C::PBUF) * C::PB; };
  auto sR = [&](int i) { return sR0 + (i % C::RBUF) * C::RB; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS_MAX; ++s) {
      mbar_init(bar(Q_TMA_FULL + s), 1);
      if (!PRE) mbar_init(bar(Q_CONV_FULL + s), C::NCONV);
      mbar_init(bar(Q_STAGE_EMPTY + s), 1);
    }
    for (int k = 0; k < 2; ++k) {
      if (PS) {
        mbar_init(bar(Q_QA_FULL + k), 1);
        mbar_init(bar(Q_QA_FREE + k), 1);
        mbar_init(bar(Q_KA_FULL + k), 1);
        mbar_init(bar(Q_KA_FREE + k), 1);
      }
      mbar_init(bar(Q_S_FULL + k), 1);
      mbar_init(bar(Q_S_FREE + k), 128);
      mbar_init(bar(Q_P_FULL + k), 128);
      mbar_init(bar(Q_P_FREE + k), 1);
      mbar_init(bar(Q_DR_FULL + k), 1);
      mbar_init(bar(Q_DR_FREE + k), 32 * C::WARPS_S);
      mbar_init(bar(Q_R16_FULL + k), 32 * C::WARPS_S);
      mbar_init(bar(Q_R16_FREE + k), 1);
      mbar_init(bar(Q_O_FULL + k), 1);
      mbar_init(bar(Q_O_FREE + k), 128);
      if (!PRE) mbar_init(bar(Q_TAB + k), C::NCONV);
      if (FUSE) mbar_init(bar(Q_XFULL + k), 1);  // armed once a use, the rest is transaction bytes
    }
    mbar_init(bar(Q_DRAIN), 1);
    fence_mbar_init();
  }
  if (warp == C::WARP_MMA) {
    tmem_alloc(smem_addr(tmem_holder), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == C::WARP_TMA && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    if (HL && PRE) {
      prefetch_tensormap(&tm_ql);
      prefetch_tensormap(&tm_kl);
    }
    if (PS) prefetch_tensormap(&tm_ql);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if constexpr (FUSE) cluster_sync();  // every CTA's barriers exist before any remote arrival
  const uint32_t tmem = *tmem_holder;

  if (warp == C::WARP_TMA) {
    // ------------------------------------------------------------------ TMA producer
    if (PS && lane == 0) {
      // P tiles from the P pass: every unit's stage takes V_w and P_{u,w}; the first unit of a
      // row block loads Q_u into a Q slot, a unit of the last row block K_w into a K slot.
      int issued[C::NS_MAX] = {}, q_issued[2] = {0, 0}, k_issued[2] = {0, 0};
      UnitIter<T, SM> it;
      for (it.start(a.L, nb, c_first, c_lo, c_hi); it.valid(); it.next()) {
        const int s = it.k % C::NS;
        if (it.k >= C::NS && !mbar_wait(bar(Q_STAGE_EMPTY + s), ((it.k / C::NS) - 1) & 1)) break;
        const int tq = it.t0() + it.u * T, tk = it.t0() + it.w * T;
        mbar_arrive_expect_tx(bar(Q_TMA_FULL + s), C::VBYTES + C::PBYTES);
#pragma unroll
        for (int bx = 0; bx < C::NDV; ++bx)
          tma_load_4d(sV(s) + bx * T * 128, &tm_v, bar(Q_TMA_FULL + s), dvb * DVS + 64 * bx, h, tk, b);
        // the P tile of unit (u, w) of chunk i: ((b h) n_chunks + i) U + u (u + 1) / 2 + w
        const int tile = ((b * a.heads + h) * a.n_chunks + it.i) * (nb * (nb + 1) / 2) + it.u * (it.u + 1) / 2 + it.w;
        tma_load_4d(sPs(s), &tm_ql, bar(Q_TMA_FULL + s), 0, 0, tile, 0);
        issued[s]++;
        if (it.w == 0) {
          const int qs = it.rb % 2;
          if (it.rb >= 2 && !mbar_wait(bar(Q_QA_FREE + qs), ((it.rb / 2) - 1) & 1)) break;
          mbar_arrive_expect_tx(bar(Q_QA_FULL + qs), C::QBYTES);
#pragma unroll
          for (int bx = 0; bx < DK / 64; ++bx)
            tma_load_4d(sQa(qs) + bx * T * 128, &tm_q, bar(Q_QA_FULL + qs), bx * 64, h, tq, b);
          q_issued[qs]++;
        }
        if (it.last_row()) {
          const int ks = it.dr % 2;
          if (it.dr >= 2 && !mbar_wait(bar(Q_KA_FREE + ks), ((it.dr / 2) - 1) & 1)) break;
          mbar_arrive_expect_tx(bar(Q_KA_FULL + ks), C::QBYTES);
#pragma unroll
          for (int bx = 0; bx < DK / 64; ++bx)
            tma_load_4d(sKa(ks) + bx * T * 128, &tm_k, bar(Q_KA_FULL + ks), bx * 64, h, tk, b);
          k_issued[ks]++;
        }
      }
      // Every load this thread issued must have landed before the CTA may exit.
      for (int s = 0; s < C::NS; ++s)
        if (issued[s] > 0) mbar_wait(bar(Q_TMA_FULL + s), (issued[s] - 1) & 1, kDrainBudget);
      for (int j = 0; j < 2; ++j) {
        if (q_issued[j] > 0) mbar_wait(bar(Q_QA_FULL + j), (q_issued[j] - 1) & 1, kDrainBudget);
        if (k_issued[j] > 0) mbar_wait(bar(Q_KA_FULL + j), (k_issued[j] - 1) & 1, kDrainBudget);
      }
    } else if (lane == 0) {
      int issued[4] = {0, 0, 0, 0};
      UnitIter<T, SM> it;
      for (it.start(a.L, nb, c_first, c_lo, c_hi); it.valid(); it.next()) {
        const int s = it.k % C::NS;
        if (it.k >= C::NS && !mbar_wait(bar(Q_STAGE_EMPTY + s), ((it.k / C::NS) - 1) & 1)) break;
        const bool with_q = !it.pre();  // state replay needs K and V only
        // bytes that land: Q (unless replay) and K, with their lo parts when pre-converted split
        constexpr int QK_PARTS = (HL && PRE) ? 2 : 1;
        mbar_arrive_expect_tx(bar(Q_TMA_FULL + s), (with_q ? 2 : 1) * C::QBYTES * QK_PARTS + C::VBYTES);
        const int tq = it.t0() + it.u * T, tk = it.t0() + it.w * T;
#pragma unroll
        for (int bx = 0; bx < DK / 64; ++bx) {
          if (with_q) tma_load_4d(sQ(s) + bx * T * 128, &tm_q, bar(Q_TMA_FULL + s), bx * 64, h, tq, b);
          tma_load_4d(sK(s) + bx * T * 128, &tm_k, bar(Q_TMA_FULL + s), bx * 64, h, tk, b);
          if constexpr (HL && PRE) {
            if (with_q) tma_load_4d(sQl(s) + bx * T * 128, &tm_ql, bar(Q_TMA_FULL + s), bx * 64, h, tq, b);
            tma_load_4d(sKl(s) + bx * T * 128, &tm_kl, bar(Q_TMA_FULL + s), bx * 64, h, tk, b);
          }
        }
#pragma unroll
        for (int bx = 0; bx < C::NDV; ++bx)
          tma_load_4d(sV(s) + bx * T * 128, &tm_v, bar(Q_TMA_FULL + s), dvb * DVS + 64 * bx, h, tk, b);
        issued[s]++;
      }
      // Every load this thread issued must have landed before the CTA may exit.
      for (int s = 0; s < C::NS; ++s)
        if (issued[s] > 0) mbar_wait(bar(Q_TMA_FULL + s), (issued[s] - 1) & 1, kDrainBudget);
    }
  } else if (warp == C::WARP_MMA) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID_S = idesc_f16_f32(T, T, 0, 0);
      constexpr uint32_t ID_X = idesc_f16_f32(T, DVS, 0, 1);
      constexpr uint32_t ID_R = idesc_f16_f32(C::MR, DVS, 1, 1);
      // Descriptors are built once per operand tile and advanced by constants (the start
      // address field never carries: every operand lies below 256 KB of shared memory).
      auto kstep = [](int kk) -> uint64_t { return static_cast<uint64_t>(((kk / 4) * T * 128 + (kk % 4) * 32) >> 4); };
      // The three MMA groups of a unit: F = S'' and, on the last row block, the state increment
      // Kz_w^T V_w; X = the cross term of a row block (its first unit); P = P V into O.  Each
      // has a non-blocking readiness test.  The issuer takes whichever group is ready -- X and P
      // of the oldest unit first, F at most LA units ahead -- so a late conversion of a later
      // unit never holds back the output (and the stage release) of an earlier one.
      auto f_ready = [&](const UnitIter<T, SM>& f) -> bool {
        if (!mbar_test(bar(Q_READY + f.k % C::NS), (f.k / C::NS) & 1)) return false;
        // PS: the unit's K tile in its slot (state increment of the last row block)
        if (PS && f.last_row() && !mbar_test(bar(Q_KA_FULL + f.dr % 2), (f.dr / 2) & 1)) return false;
        if (!PS && !f.pre() && f.kf() >= C::SBUF &&
            !mbar_test(bar(Q_S_FREE + (f.kf() % C::SBUF)), ((f.kf() - C::SBUF) / C::SBUF) & 1))
          return false;
        if constexpr (C::RTM) {
          // the state group has scaled the resident state for this chunk (slot dr & 1)
          if (!mbar_test(bar(Q_DR_FREE + (f.dr & 1)), (f.dr >> 1) & 1)) return false;
        } else {
          if (f.last_row() && f.dr >= C::DRBUF &&
              !mbar_test(bar(Q_DR_FREE + (f.dr % C::DRBUF)), ((f.dr - C::DRBUF) / C::DRBUF) & 1))
            return false;
        }
        return true;
      };
      auto f_issue = [&](const UnitIter<T, SM>& f) {
        const int s = f.k % C::NS;
        tc_fence_after();
        if (!PS && !f.pre()) {
          const uint32_t tS = tmem + C::COL_S + (f.kf() % C::SBUF) * T;
          const uint64_t dq = sdesc_sw128(sQ(s), 16, 1024), dk = sdesc_sw128(sK(s), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < DK / 16; ++kk) mma_f16_ss(tS, dq + kstep(kk), dk + kstep(kk), ID_S, kk > 0);
          if constexpr (HL) {  // S += Qlo Khi^T + Qhi Klo^T (the lo x lo term is below 2^-22)
            const uint64_t dql = sdesc_sw128(sQl(s), 16, 1024), dkl = sdesc_sw128(sKl(s), 16, 1024);
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk) mma_f16_ss(tS, dql + kstep(kk), dk + kstep(kk), ID_S, 1u);
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk) mma_f16_ss(tS, dq + kstep(kk), dkl + kstep(kk), ID_S, 1u);
          }
          mma_commit(bar(Q_S_FULL + (f.kf() % C::SBUF)));
        }
        if (f.last_row()) {
          const uint32_t tD = tmem + C::COL_DR + (f.dr % C::DRBUF) * C::RBLK * DVS;
          const uint64_t dkm = sdesc_sw128(PS ? sKa(f.dr % 2) : sK(s), T * 128, 1024), dv = sdesc_sw128(sV(s), T * 128, 1024);
#pragma unroll
          for (int blk = 0; blk < C::RBLK; ++blk)
#pragma unroll
            for (int ks = 0; ks < T / 16; ++ks)
              mma_f16_ss(tD + blk * DVS, dkm + static_cast<uint64_t>((blk * 2 * T * 128 + ks * 2048) >> 4),
                         dv + static_cast<uint64_t>((ks * 2048) >> 4), ID_R, (C::RTM || ks > 0) ? 1u : 0u);
          if constexpr (HL) {  // + Klo^T V (V is exact in fp16)
            const uint64_t dklm = sdesc_sw128(sKl(s), T * 128, 1024);
#pragma unroll
            for (int blk = 0; blk < C::RBLK; ++blk)
#pragma unroll
              for (int ks = 0; ks < T / 16; ++ks)
                mma_f16_ss(tD + blk * DVS, dklm + static_cast<uint64_t>((blk * 2 * T * 128 + ks * 2048) >> 4),
                           dv + static_cast<uint64_t>((ks * 2048) >> 4), ID_R, 1u);
          }
          mma_commit(bar(Q_DR_FULL + (f.dr % C::DRBUF)));
          if (PS) mma_commit(bar(Q_KA_FREE + f.dr % 2));
        }
        if (f.pre()) mma_commit(bar(Q_STAGE_EMPTY + s));  // a replay unit has no P V
      };
      auto x_ready = [&](const UnitIter<T, SM>& q) -> bool {
        const int ri = q.i - c_lo;  // fp16 state copies are written for output chunks only
        if (!mbar_test(bar(Q_R16_FULL + (ri % C::RBUF)), (ri / C::RBUF) & 1)) return false;
        if (PS && !mbar_test(bar(Q_QA_FULL + q.rb % 2), (q.rb / 2) & 1)) return false;  // the row block's Q
        return q.rb < 2 || mbar_test(bar(Q_O_FREE + (q.rb & 1)), ((q.rb - 2) >> 1) & 1);
      };
      auto x_issue = [&](const UnitIter<T, SM>& q) {
        const int s = q.k % C::NS;
        tc_fence_after();
        const uint32_t tO = tmem + C::COL_O + (q.rb & 1) * DVS;
        const uint32_t tX = (C::XBUF > 0 && nb > 1) ? tmem + C::COL_X + (q.rb & 1) * DVS : tO;
        const int ri = q.i - c_lo;
        const uint64_t dq = sdesc_sw128(PS ? sQa(q.rb % 2) : sQ(s), 16, 1024), dr = sdesc_sw128(sR(ri), DK * 128, 1024);
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk)
          mma_f16_ss(tX, dq + kstep(kk), dr + static_cast<uint64_t>((kk * 2048) >> 4), ID_X, kk > 0);
        if constexpr (HL) {  // + Qlo Rhi + Qhi Rlo
          const uint64_t dql = sdesc_sw128(sQl(s), 16, 1024), drl = sdesc_sw128(sR(ri) + C::RBYTES, DK * 128, 1024);
#pragma unroll
          for (int kk = 0; kk < DK / 16; ++kk)
            mma_f16_ss(tX, dql + kstep(kk), dr + static_cast<uint64_t>((kk * 2048) >> 4), ID_X, 1u);
#pragma unroll
          for (int kk = 0; kk < DK / 16; ++kk)
            mma_f16_ss(tX, dq + kstep(kk), drl + static_cast<uint64_t>((kk * 2048) >> 4), ID_X, 1u);
        }
        if (PS) mma_commit(bar(Q_QA_FREE + q.rb % 2));
        if (q.last_row()) mma_commit(bar(Q_R16_FREE + (ri % C::RBUF)));
      };
      auto p_ready = [&](const UnitIter<T, SM>& q) -> bool {
        if constexpr (PS) return true;  // the P tile came with the unit's stage (F issued after it landed)
        return mbar_test(bar(Q_P_FULL + (q.kf() % C::PBUF)), (q.kf() / C::PBUF) & 1);
      };
      auto p_issue = [&](const UnitIter<T, SM>& q) {
        const int s = q.k % C::NS;
        tc_fence_after();
        const uint32_t tO = tmem + C::COL_O + (q.rb & 1) * DVS;
        const uint64_t dp = sdesc_sw128(PS ? sPs(s) : sP(q.kf()), 16, 1024), dv = sdesc_sw128(sV(s), T * 128, 1024);
        const uint32_t acc0 = (q.w > 0 || nb == 1) ? 1u : 0u;
#pragma unroll
        for (int kk = 0; kk < T / 16; ++kk)
          mma_f16_ss(tO, dp + kstep(kk), dv + static_cast<uint64_t>((kk * 2048) >> 4), ID_X, kk > 0 ? 1u : acc0);
        if constexpr (HL) {  // + Plo V
          const uint64_t dpl = sdesc_sw128(sP(q.kf()) + C::PBYTES, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < T / 16; ++kk)
            mma_f16_ss(tO, dpl + kstep(kk), dv + static_cast<uint64_t>((kk * 2048) >> 4), ID_X, 1u);
        }
        if (!PS) mma_commit(bar(Q_P_FREE + (q.kf() % C::PBUF)));
        if (q.rb_done()) mma_commit(bar(Q_O_FULL + (q.rb & 1)));
        mma_commit(bar(Q_STAGE_EMPTY + s));
      };
      constexpr int LA = 2;  // F of unit f only while f <= q + LA (q = oldest unit with P pending)
      UnitIter<T, SM> f, q;
      f.start(a.L, nb, c_first, c_lo, c_hi);
      q.start(a.L, nb, c_first, c_lo, c_hi);
      while (q.valid() && q.pre()) q.next();  // q walks output units only (none in the pre-pass)
      bool x_done = false;
      long long idle_since = clock64();
      while (q.valid()) {
        bool progress = false;
        if (q.k < f.k) {  // F of unit q has been issued
          if (q.w == 0 && !x_done && x_ready(q)) {
            x_issue(q);
            x_done = true;
            progress = true;
          }
          if ((q.w != 0 || x_done) && p_ready(q)) {
            p_issue(q);
            q.next();
            x_done = false;
            progress = true;
          }
        }
        if (!progress && f.valid() && f.k <= q.k + LA && f_ready(f)) {
          f_issue(f);
          f.next();
          progress = true;
        }
        if (progress) {
          idle_since = clock64();
        } else if (clock64() - idle_since > g_wait_budget) {
          atomicAdd(&g_wait_timeouts, 1u);  // same bound and report as a blocking wait
          break;
        }
      }
      mma_commit(bar(Q_DRAIN));
      mbar_wait(bar(Q_DRAIN), 0, kDrainBudget);
    }
  } else if (warp >= C::WARP_CONV0 && warp < C::WARP_CONV0 + C::CONV_WARPS) {
    // ------------------------------------------------------------------ converters
    if constexpr (!PRE) {
    UnitConverter<DK, T, C::NCONV, C::NDV> cv;
    cv.init(threadIdx.x - 32 * C::WARP_CONV0, nb, hp);
    cv.conv_v = a.v_f16 == 0;
    const bool xpos = (a.flags & RETNET_F_XPOS) != 0;
    bool ok = true;
    float mx = 0.f;  // largest magnitude rounded to fp16
    UnitIter<T, SM> it;
    for (it.start(a.L, nb, c_first, c_lo, c_hi); ok && it.valid(); it.next()) {
      const int s = it.k % C::NS;
      float2* tq = tab + (it.k & 1) * DK;
      float2* tk = tq + DK / 2;
      if (xpos) cv.put_bases(tq, tk, it.i, it.u, it.w, it.t0(), a.pos0, hp);
      // Table buffer (k & 1) is complete once all converters arrived; a thread that
      // rewrites it two units later has passed this wait, so every read of it is done.
      mbar_arrive(bar(Q_TAB + (it.k & 1)));
      ok = mbar_wait(bar(Q_TAB + (it.k & 1)), (it.k >> 1) & 1);
      if (ok) ok = mbar_wait(bar(Q_TMA_FULL + s), (it.k / C::NS) & 1);
      if (!ok) break;
      if (SM == SEG_REPLAY && it.pre()) {
        cv.template convert<false>(sQ(s), sK(s), sV(s), tq, tk, xpos, log2g, mx);
      } else {
        cv.template convert<true, HL>(sQ(s), sK(s), sV(s), tq, tk, xpos, log2g, mx, 1.f, sQl(s), sKl(s));
      }
      fence_proxy_async_smem();
      mbar_arrive(bar(Q_CONV_FULL + s));
    }
    report_fp16_range(mx);
    }
  } else if (warp >= C::WARP_S0 && warp < C::WARP_S0 + C::WARPS_S) {
    // ------------------------------------------------------------------ state group
    if constexpr (C::RTM) {
      // The fp32 state stays in tensor memory as a master M; thread = one TMEM lane, i.e. one
      // d_k row in each of its BPT 128-row blocks, all DVS columns.  Before every increment
      // Kz_w^T V_w (the column blocks w of a chunk's last row block) accumulates into M, the
      // state group scales M by gamma^T; at w = 0 M holds R_{i-1}, whose fp16 copy (output
      // chunks only) is written first.  This is the Horner form of
      //   R_i = gamma^b' R_{i-1} + sum_w gamma^(b'-(w+1)T) Kz_w^T V_w = hh * M,
      // hh = gamma^(b' - nbw T): 1 except on the last chunk, where state_out takes it.
      const uint32_t lane_off = static_cast<uint32_t>(32 * (warp % 4)) << 16;
      const int64_t bh = static_cast<int64_t>(b) * a.heads + h;
      const size_t srow = static_cast<size_t>(a.dv);
      const float gT = decay_pow(log2g, T);
      constexpr int GW = 32;  // columns per batch
      auto row_of = [&](int blk) -> int {
        return (DK == 64) ? (lane < 16 ? 16 * (warp % 4) + lane : -1) : blk * 128 + 32 * (warp % 4) + lane;
      };
      bool ok = true;
      float smx = 0.f;  // largest state-copy magnitude rounded to fp16
      int last_dr = -1, last_bl = T, last_nbw = 1;
      UnitIter<T, SM> it;
      for (it.start(a.L, nb, c_first, c_lo, c_hi); ok && it.valid(); it.next()) {
        if (!it.last_row()) continue;
        const int d = it.dr;
        if (d > 0) {  // the previous increment has landed
          ok = __all_sync(0xffffffffu, mbar_wait(bar(Q_DR_FULL + 0), (d - 1) & 1));
          if (!ok) break;
          tc_fence_after();
        }
        const bool copy = !it.pre() && it.w == 0;  // M = R_{i-1}: write its fp16 copy
        const int ri = it.i - c_lo;
        if (copy && ri >= C::RBUF) {
          ok = __all_sync(0xffffffffu, mbar_wait(bar(Q_R16_FREE + (ri % C::RBUF)), ((ri - C::RBUF) / C::RBUF) & 1));
          if (!ok) break;
        }
        const uint32_t r16 = sR(ri);
#pragma unroll 1
        for (int bk = 0; bk < C::BPT; ++bk) {
          const int dk = row_of(bk);
          const uint32_t tR = tmem + C::COL_DR + bk * DVS + lane_off;
#pragma unroll 1
          for (int grp = 0; grp < DVS / GW; ++grp) {
            uint32_t u[GW / 16][16];
            if (d > 0) {
              tmem_ld_wait(tR + GW * grp, u);
            } else {  // first increment: M starts from state_in (carried over earlier segments)
              float r0v[GW];
              if (dk >= 0) {
                start_state(dk, dvb * DVS + GW * grp, GW, r0v);
              } else {
#pragma unroll
                for (int c = 0; c < GW; ++c) r0v[c] = 0.f;
              }
#pragma unroll
              for (int c = 0; c < GW; ++c) u[c / 16][c % 16] = __float_as_uint(r0v[c]);
            }
            if (copy && dk >= 0) {
              // fp16 copy (times 1/sqrt(d_k)) into box (column / 64), 16-byte slots of 8 columns
#pragma unroll
              for (int c8 = 0; c8 < GW / 8; ++c8) {
                const int col = GW * grp + 8 * c8;
                const uint32_t* x = &u[(8 * c8) / 16][(8 * c8) % 16];
                const uint32_t off = (col / 64) * DK * 128 + sw128(dk, (col % 64) / 8);
#pragma unroll
                for (int e = 0; e < 8; ++e) smx = absmax(smx, sd * __uint_as_float(x[e]));
                if constexpr (HL) {
                  uint32_t hi[4], lo[4];
#pragma unroll
                  for (int e = 0; e < 4; ++e)
                    split_f16x2(sd * __uint_as_float(x[2 * e]), sd * __uint_as_float(x[2 * e + 1]), hi[e], lo[e]);
                  st_shared_v4(r16 + off, hi[0], hi[1], hi[2], hi[3]);
                  st_shared_v4(r16 + C::RBYTES + off, lo[0], lo[1], lo[2], lo[3]);
                } else {
                  st_shared_v4(r16 + off, pack_f16x2(sd * __uint_as_float(x[0]), sd * __uint_as_float(x[1])),
                               pack_f16x2(sd * __uint_as_float(x[2]), sd * __uint_as_float(x[3])),
                               pack_f16x2(sd * __uint_as_float(x[4]), sd * __uint_as_float(x[5])),
                               pack_f16x2(sd * __uint_as_float(x[6]), sd * __uint_as_float(x[7])));
                }
              }
            }
#pragma unroll
            for (int c = 0; c < GW; ++c) u[c / 16][c % 16] = __float_as_uint(gT * __uint_as_float(u[c / 16][c % 16]));
            tmem_st_wait(tR + GW * grp, u);
          }
        }
        if (copy) fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar(Q_DR_FREE + (d & 1)));  // M is ready for this increment
        if (copy) mbar_arrive(bar(Q_R16_FULL + (ri % C::RBUF)));
        last_dr = d;
        last_bl = it.bl;
        last_nbw = it.nbw;
      }
      report_fp16_range(smx);
      // End of the sequence: R_last = hh * M once the last increment landed.
      if (ok && last_dr >= 0 && (!SEG || c_hi * nb * T >= a.L)) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(Q_DR_FULL + 0), last_dr & 1));
        tc_fence_after();
        if (ok && a.state_out) {
          const float hh = exp2f(static_cast<float>(last_bl - last_nbw * T) * log2g);
#pragma unroll 1
          for (int bk = 0; bk < C::BPT; ++bk) {
            const int dk = row_of(bk);
            const uint32_t tR = tmem + C::COL_DR + bk * DVS + lane_off;
#pragma unroll 1
            for (int grp = 0; grp < DVS / GW; ++grp) {
              uint32_t u[GW / 16][16];
              tmem_ld_wait(tR + GW * grp, u);
              if (dk >= 0) {
                float* dst = a.state_out + static_cast<size_t>(bh) * DK * a.dv + dvb * DVS + GW * grp + dk * srow;
#pragma unroll
                for (int c4 = 0; c4 < GW / 4; ++c4)
                  *reinterpret_cast<float4*>(dst + 4 * c4) =
                      make_float4(hh * __uint_as_float(u[(4 * c4) / 16][(4 * c4) % 16]),
                                  hh * __uint_as_float(u[(4 * c4 + 1) / 16][(4 * c4 + 1) % 16]),
                                  hh * __uint_as_float(u[(4 * c4 + 2) / 16][(4 * c4 + 2) % 16]),
                                  hh * __uint_as_float(u[(4 * c4 + 3) / 16][(4 * c4 + 3) % 16]));
              }
            }
          }
        }
      }
    } else {
      // Thread = (d_k row, 64-column box ch of the slice); warp % 4 selects its TMEM lane quarter.
      constexpr int RC = 64;
      const int ws = warp - C::WARP_S0;
      const int blk = (ws / 4) % C::RBLK;
      const int ch = ws / (4 * C::RBLK);
      const uint32_t lane_off = static_cast<uint32_t>(32 * (warp % 4)) << 16;
      const int dk = (DK == 64) ? (lane < 16 ? 16 * (warp % 4) + lane : -1) : blk * 128 + 32 * (warp % 4) + lane;
      const int64_t bh = static_cast<int64_t>(b) * a.heads + h;
      const size_t srow = static_cast<size_t>(a.dv);
      const int col0 = dvb * DVS + ch * RC;
      float R[RC];
  #pragma unroll
      for (int c = 0; c < RC; ++c) R[c] = 0.f;
      if (dk >= 0) start_state(dk, col0, RC, R);
      float smx = 0.f;  // largest state-copy magnitude rounded to fp16
      auto put_r16 = [&](uint32_t base) {
        if (dk < 0) return;
        base += ch * DK * 128;
  #pragma unroll
        for (int c = 0; c < 64; ++c) smx = absmax(smx, sd * R[c]);
  #pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          if constexpr (HL) {
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) split_f16x2(sd * R[8 * c8 + 2 * e], sd * R[8 * c8 + 2 * e + 1], hi[e], lo[e]);
            st_shared_v4(base + sw128(dk, c8), hi[0], hi[1], hi[2], hi[3]);
            st_shared_v4(base + C::RBYTES + sw128(dk, c8), lo[0], lo[1], lo[2], lo[3]);
          } else {
            st_shared_v4(base + sw128(dk, c8), pack_f16x2(sd * R[8 * c8 + 0], sd * R[8 * c8 + 1]),
                         pack_f16x2(sd * R[8 * c8 + 2], sd * R[8 * c8 + 3]),
                         pack_f16x2(sd * R[8 * c8 + 4], sd * R[8 * c8 + 5]),
                         pack_f16x2(sd * R[8 * c8 + 6], sd * R[8 * c8 + 7]));
          }
        }
      };
      if (c_first == c_lo) {  // otherwise written once the replay reaches the first output chunk
        put_r16(sR(0));
        fence_proxy_async_smem();
        mbar_arrive(bar(Q_R16_FULL + 0));
      }
      bool ok = true;
      UnitIter<T, SM> it;
      for (it.start(a.L, nb, c_first, c_lo, c_hi); ok && it.valid(); it.next()) {
        if (!it.last_row()) continue;
        ok = __all_sync(0xffffffffu, mbar_wait(bar(Q_DR_FULL + (it.dr % C::DRBUF)), (it.dr / C::DRBUF) & 1));
        if (!ok) break;
        tc_fence_after();
        // Horner form of R_i = gamma^b' R_{i-1} + sum_w gamma^(b'-(w+1)T) dR_w:
        //   w = 0: R = gamma^(b'-(nbw-1)T) R + hh dR_0;  w > 0: R = gamma^T R + hh dR_w,
        //   hh = gamma^(b' - nbw T) (1 for a full chunk).
        const float g = (it.w == 0) ? exp2f(static_cast<float>(it.bl - (it.nbw - 1) * T) * log2g)
                                    : decay_pow(log2g, T);
        const float hh = exp2f(static_cast<float>(it.bl - it.nbw * T) * log2g);
        const uint32_t tD = tmem + C::COL_DR + (it.dr % C::DRBUF) * C::RBLK * DVS + blk * DVS + ch * RC + lane_off;
        constexpr int SW = C::LDW / 2;  // columns per load next to the 64 state registers
  #pragma unroll
        for (int grp = 0; grp < RC / SW; ++grp) {
          uint32_t u[SW / 16][16];
          tmem_ld_wait(tD + SW * grp, u);
          if (grp == RC / SW - 1) {
            tc_fence_before();
            mbar_arrive(bar(Q_DR_FREE + (it.dr % C::DRBUF)));
          }
  #pragma unroll
          for (int c = 0; c < SW; ++c) R[SW * grp + c] = fmaf(g, R[SW * grp + c], hh * __uint_as_float(u[c / 16][c % 16]));
        }
        if (it.w + 1 < it.nbw) continue;  // chunk not finished
        const int nxt = it.i + 1;
        const bool seq_end = nxt * nb * T >= a.L;
        if (!seq_end && nxt < c_hi) {
          if (nxt < c_lo) continue;  // still replaying
          // fp16 copy ri of output chunk nxt; its buffer was last read by the cross terms of
          // output chunk ri - RBUF.
          const int ri = nxt - c_lo, prev = ri - C::RBUF;
          if (prev >= 0)
            ok = __all_sync(0xffffffffu, mbar_wait(bar(Q_R16_FREE + (prev % C::RBUF)), (prev / C::RBUF) & 1));
          if (!ok) break;
          put_r16(sR(ri));
          fence_proxy_async_smem();
          mbar_arrive(bar(Q_R16_FULL + (ri % C::RBUF)));
        } else if (seq_end && dk >= 0 && a.state_out) {
          float* dst = a.state_out + static_cast<size_t>(bh) * DK * a.dv + col0 + dk * srow;
  #pragma unroll
          for (int c4 = 0; c4 < RC / 4; ++c4)
            *reinterpret_cast<float4*>(dst + 4 * c4) = make_float4(R[4 * c4], R[4 * c4 + 1], R[4 * c4 + 2], R[4 * c4 + 3]);
        }
      }
      report_fp16_range(smx);
    }
  } else {
    // ------------------------------------------------------------------ P / epilogue group
    // (warps 0-3; with EPI_WARPS the epilogue runs on its own four warps, same TMEM lanes)
    static_assert(C::WARP_EPI0 % 4 == 0, "epilogue warps must cover the four TMEM lane quarters in order");
    const bool is_epi = C::EPI_WARPS > 0 && warp >= C::WARP_EPI0;
    const int gwarp = is_epi ? warp - C::WARP_EPI0 : warp;
    const uint32_t lane_off = static_cast<uint32_t>(32 * gwarp) << 16;
    const int my_row = (T == 128) ? 32 * gwarp + lane : (lane < 16 ? 16 * gwarp + lane : -1);
    // With T = 64 (rows in lanes 0-15) the scores and the plain epilogue take each row on two
    // threads: lane l and l + 16 hold row 16 gwarp + (l mod 16), columns of half phalf.
    constexpr bool HALVES = T == 64;
    const int prow = HALVES ? 16 * gwarp + (lane & 15) : my_row;
    const int phalf = HALVES ? (lane >> 4) : 0;
    const float gam = hp.gamma[h];
    // Epilogue of row block (chunk i, block u), O/X buffer rb & 1.
    auto epilogue = [&](int rb, int i, int u, int bl) -> bool {
      const int rows = min(T, bl - u * T);
      // this thread's row: with T = 64 lanes l and l + 16 share row 16 gwarp + (l mod 16)
      const int row = prow;
      const bool live = row >= 0 && row < rows;
      const int t = i * nb * T + u * T + (row < 0 ? 0 : row);
      // FUSE output rows and columns of this lane.  With T = 64 the rows sit in lanes 0-15 of
      // each warp; lane l + 16 then writes the upper half of the columns of lane l's row.
      constexpr bool SPLIT = FUSE && T == 64;
      constexpr int EC = SPLIT ? DVS / 2 : DVS;
      const int erow = SPLIT ? 16 * gwarp + (lane & 15) : my_row;
      const bool elive = erow >= 0 && erow < rows;
      const int64_t eoff = ((static_cast<int64_t>(b) * a.L + (i * nb * T + u * T + (erow < 0 ? 0 : erow))) * a.heads + h) *
                               a.dv + dvb * DVS + (SPLIT ? (lane >> 4) * EC : 0);
      const uint4* egp = nullptr;
      if constexpr (FUSE) {
        // the gate slice of this lane, into L1 now; the same row of the next row block (the
        // next T tokens: row blocks run in sequence order here) into L2
        egp = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.gate) + eoff);
        const char* cur = reinterpret_cast<const char*>(egp);
        if (elive) {
          asm volatile("prefetch.global.L1 [%0];" ::"l"(cur));
          asm volatile("prefetch.global.L1 [%0];" ::"l"(cur + EC * 2 - 1));
        }
        if (erow >= 0 && (i * nb * T + u * T + erow) + T < a.L) {
          const char* nx = cur + static_cast<int64_t>(T) * a.heads * a.dv * 2;
          asm volatile("prefetch.global.L2 [%0];" ::"l"(nx));
          asm volatile("prefetch.global.L2 [%0];" ::"l"(nx + EC * 2 - 1));
        }
      }
      if (!__all_sync(0xffffffffu, mbar_wait(bar(Q_O_FULL + (rb & 1)), (rb >> 1) & 1))) return false;
      tc_fence_after();
      float f = row_factor_f32(gam, sd, a.pos0 + t, a.flags) / sd;
      if (a.rden && live) f *= __ldg(a.rden + (static_cast<int64_t>(b) * a.L + t) * a.heads + h);
      const float gx = (nb > 1) ? exp2f(static_cast<float>(u * T) * log2g) : 0.f;
      const int t_out = a.o_rev ? a.L - 1 - t : t;
      Tout* dst = static_cast<Tout*>(a.o) + ((static_cast<int64_t>(b) * a.L + t_out) * a.heads + h) * a.dv + dvb * DVS;
      // O (and X) from TMEM, o = (O + gamma^(uT) X) * s / c_p, 16-byte stores of 16 columns.
      auto store16 = [&](int q, const float (&ov)[16]) {
        if constexpr (sizeof(Tout) == 2) {
#pragma unroll
          for (int c8 = 0; c8 < 2; ++c8) {
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __nv_bfloat162 v2 = __floats2bfloat162_rn(ov[8 * c8 + 2 * e], ov[8 * c8 + 2 * e + 1]);
              pk[e] = *reinterpret_cast<uint32_t*>(&v2);
            }
            *reinterpret_cast<uint4*>(dst + 16 * q + 8 * c8) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        } else {
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4)
            *reinterpret_cast<float4*>(dst + 16 * q + 4 * c4) =
                make_float4(ov[4 * c4], ov[4 * c4 + 1], ov[4 * c4 + 2], ov[4 * c4 + 3]);
        }
      };
      const uint32_t tO = tmem + C::COL_O + (rb & 1) * DVS + lane_off;
      const uint32_t tX = tmem + C::COL_X + (rb & 1) * DVS + lane_off;
      if constexpr (FUSE) {
        // MSR epilogue in the kernel ("阅读笔记：RetNet" §三.2): the head's d_v columns are spread
        // over the n_cl CTAs of this cluster.  Each CTA takes (mean, M2) of its 64 columns of a
        // row and stores them into every CTA's shared memory (st.async, counted in transaction
        // bytes on that CTA's barrier); the pooled statistics (Chan's combination of equal-count
        // groups) normalise the row, which is then multiplied by swish(gate).  Biased variance,
        // eps inside the root.  Slot rb & 1 is written again for row block rb + 2 only after
        // its writer has seen every CTA's statistics of row block rb + 1, which each CTA sends
        // after it has finished reading the slot for row block rb: two slots need no release
        // barrier.
        // yv: this lane's EC columns of its row (with T = 64 each lane loads its half directly
        // and the row's sum and M2 combine across lanes l and l + 16)
        float yv[EC];
        float mean_i = 0.f, m2 = 0.f;
        if constexpr (SPLIT) {
          static_assert(EC == 32, "the split epilogue takes 64-column slices");
          uint32_t uo[2][16], ux[2][16];
          if (C::XBUF > 0 && nb > 1) {
            tmem_ld16x2_wait<32>(tO, uo, tX, ux);
          } else {
            tmem_ld16x2_wait<32>(tO, uo);
          }
          tc_fence_before();
          mbar_arrive(bar(Q_O_FREE + (rb & 1)));
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float ov = __uint_as_float(uo[c / 16][c % 16]);
            yv[c] = (C::XBUF > 0 && nb > 1) ? f * fmaf(gx, __uint_as_float(ux[c / 16][c % 16]), ov) : f * ov;
            mean_i += yv[c];
          }
          mean_i += __shfl_xor_sync(0xffffffffu, mean_i, 16);
          mean_i *= 1.f / DVS;
#pragma unroll
          for (int c = 0; c < 32; ++c) m2 = fmaf(yv[c] - mean_i, yv[c] - mean_i, m2);
          m2 += __shfl_xor_sync(0xffffffffu, m2, 16);
        } else {
          float y[DVS];
#pragma unroll
          for (int grp = 0; grp < DVS / 32; ++grp) {
            uint32_t uo[2][16], ux[2][16];
            if (C::XBUF > 0 && nb > 1) {
              tmem_ld_wait(tO + 32 * grp, uo, tX + 32 * grp, ux);
            } else {
              tmem_ld_wait(tO + 32 * grp, uo);
            }
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              const float ov = __uint_as_float(uo[c / 16][c % 16]);
              y[32 * grp + c] = (C::XBUF > 0 && nb > 1) ? f * fmaf(gx, __uint_as_float(ux[c / 16][c % 16]), ov) : f * ov;
            }
          }
          tc_fence_before();
          mbar_arrive(bar(Q_O_FREE + (rb & 1)));
#pragma unroll
          for (int c = 0; c < DVS; ++c) mean_i += y[c];
          mean_i *= 1.f / DVS;
#pragma unroll
          for (int c = 0; c < DVS; ++c) m2 = fmaf(y[c] - mean_i, y[c] - mean_i, m2);
#pragma unroll
          for (int c = 0; c < EC; ++c) yv[c] = y[c];
        }
        const int slot = rb & 1;
        const uint32_t me = cluster_ctarank();
        if (gwarp == 0 && lane == 0) mbar_arrive_expect_tx(bar(Q_XFULL + slot), static_cast<uint32_t>(n_cl * T * 8));
        if (my_row >= 0) {
          for (int pr = 0; pr < n_cl; ++pr)
            st_async_v2(map_shared_rank(xaddr(slot, me, my_row), pr), mean_i, m2,
                        map_shared_rank(bar(Q_XFULL + slot), pr));
        }
        if (!__all_sync(0xffffffffu, mbar_wait_cluster(bar(Q_XFULL + slot), (rb >> 1) & 1))) return false;
        if (elive) {
          // gate loads in flight together where registers allow (half rows), else 16 columns at a time
          uint4 gv[SPLIT ? EC / 8 : 2];
          if constexpr (SPLIT) {
#pragma unroll
            for (int j = 0; j < EC / 8; ++j) gv[j] = __ldg(egp + j);
          }
          float mean = 0.f, m2t = 0.f;
          for (int pr = 0; pr < n_cl; ++pr) {
            float2 st;
            asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(st.x), "=f"(st.y) : "r"(xaddr(slot, pr, erow)));
            mean += st.x;
            m2t += st.y;
          }
          mean /= static_cast<float>(n_cl);
          for (int pr = 0; pr < n_cl; ++pr) {
            float mx;
            asm volatile("ld.shared.f32 %0, [%1];" : "=f"(mx) : "r"(xaddr(slot, pr, erow)));
            m2t = fmaf(static_cast<float>(DVS) * (mx - mean), mx - mean, m2t);
          }
          const float inv = rsqrtf(m2t / static_cast<float>(DVS * n_cl) + a.eps);
          Tout* edst = static_cast<Tout*>(a.o) + eoff;
#pragma unroll
          for (int q = 0; q < EC / 16; ++q) {
            const uint4 g0 = SPLIT ? gv[(2 * q) % (SPLIT ? EC / 8 : 2)] : __ldg(egp + 2 * q);
            const uint4 g1 = SPLIT ? gv[(2 * q + 1) % (SPLIT ? EC / 8 : 2)] : __ldg(egp + 2 * q + 1);
            const uint32_t gw[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
            float ov[16];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              // swish(g) = g / (1 + e^-g); the fast divide is exact enough here (2 ulp)
              const float ga = __uint_as_float(gw[e] << 16), gb = __uint_as_float(gw[e] & 0xffff0000u);
              ov[2 * e] = (yv[16 * q + 2 * e] - mean) * inv * __fdividef(ga, 1.f + __expf(-ga));
              ov[2 * e + 1] = (yv[16 * q + 2 * e + 1] - mean) * inv * __fdividef(gb, 1.f + __expf(-gb));
            }
            if constexpr (sizeof(Tout) == 2) {
#pragma unroll
              for (int c8 = 0; c8 < 2; ++c8) {
                uint32_t pk[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  __nv_bfloat162 v2 = __floats2bfloat162_rn(ov[8 * c8 + 2 * e], ov[8 * c8 + 2 * e + 1]);
                  pk[e] = *reinterpret_cast<uint32_t*>(&v2);
                }
                *reinterpret_cast<uint4*>(edst + 16 * q + 8 * c8) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
              }
            } else {
#pragma unroll
              for (int c4 = 0; c4 < 4; ++c4)
                *reinterpret_cast<float4*>(edst + 16 * q + 4 * c4) =
                    make_float4(ov[4 * c4], ov[4 * c4 + 1], ov[4 * c4 + 2], ov[4 * c4 + 3]);
            }
          }
        }
        return true;
      }
      if constexpr (HALVES) {
        // Each thread: half phalf of its row's DVS columns, 32 at a time (O, and X with nb > 1).
        constexpr int HC = DVS / 2;
#pragma unroll 1
        for (int grp = 0; grp < HC / 32; ++grp) {
          uint32_t uo[2][16], ux[2][16];
          if (C::XBUF > 0 && nb > 1) {
            tmem_ld16x2_wait<HC>(tO + 32 * grp, uo, tX + 32 * grp, ux);
          } else {
            tmem_ld16x2_wait<HC>(tO + 32 * grp, uo);
          }
          if (grp == HC / 32 - 1) {
            tc_fence_before();
            mbar_arrive(bar(Q_O_FREE + (rb & 1)));
          }
          if (live) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              float ov[16];
#pragma unroll
              for (int c = 0; c < 16; ++c)
                ov[c] = (C::XBUF > 0 && nb > 1) ? f * fmaf(gx, __uint_as_float(ux[e][c]), __uint_as_float(uo[e][c]))
                                                : f * __uint_as_float(uo[e][c]);
              store16((phalf * HC + 32 * grp) / 16 + e, ov);
            }
          }
        }
      } else if (C::XBUF == 0 || nb == 1) {
        // No cross accumulator: O alone, LDW columns per load.
#pragma unroll
        for (int grp = 0; grp < DVS / C::LDW; ++grp) {
          uint32_t uo[C::LDW / 16][16];
          tmem_ld_wait(tO + grp * C::LDW, uo);
          if (grp == DVS / C::LDW - 1) {
            tc_fence_before();
            mbar_arrive(bar(Q_O_FREE + (rb & 1)));
          }
          if (live) {
#pragma unroll
            for (int e = 0; e < C::LDW / 16; ++e) {
              float ov[16];
#pragma unroll
              for (int c = 0; c < 16; ++c) ov[c] = f * __uint_as_float(uo[e][c]);
              store16(grp * (C::LDW / 16) + e, ov);
            }
          }
        }
      } else {
        // O and X, LDW / 2 columns of each per load.
        constexpr int HW = C::LDW / 2;
#pragma unroll 1
        for (int grp = 0; grp < DVS / HW; ++grp) {
          uint32_t uo[HW / 16][16], ux[HW / 16][16];
          tmem_ld_wait(tO + grp * HW, uo, tX + grp * HW, ux);
          if (grp == DVS / HW - 1) {
            tc_fence_before();
            mbar_arrive(bar(Q_O_FREE + (rb & 1)));
          }
          if (live) {
#pragma unroll
            for (int e = 0; e < HW / 16; ++e) {
              float ov[16];
#pragma unroll
              for (int c = 0; c < 16; ++c) ov[c] = f * fmaf(gx, __uint_as_float(ux[e][c]), __uint_as_float(uo[e][c]));
              store16(grp * (HW / 16) + e, ov);
            }
          }
        }
      }
      return true;
    };
    bool ok = true;
    float pmx = 0.f;  // largest |P| rounded to fp16
    int pend_rb = -1, pend_i = 0, pend_u = 0, pend_bl = 0;  // a finished row block awaiting its epilogue
    UnitIter<T, SM> it;
    for (it.start(a.L, nb, c_first, c_lo, c_hi); ok && it.valid(); it.next()) {
      if (it.pre()) continue;  // replay units have no scores
      if (is_epi || PS) {  // (with P tiles from the P pass these warps only run the epilogue)
        if (it.rb_done()) ok = epilogue(it.rb, it.i, it.u, it.bl);
        continue;
      }
      const int k = it.kf();
      ok = __all_sync(0xffffffffu, mbar_wait(bar(Q_S_FULL + (k % C::SBUF)), (k / C::SBUF) & 1));
      if (ok && k >= C::PBUF)
        ok = __all_sync(0xffffffffu, mbar_wait(bar(Q_P_FREE + (k % C::PBUF)), ((k - C::PBUF) / C::PBUF) & 1));
      if (!ok) break;
      tc_fence_after();
      // P = S'' gamma^((u-w-1) T) / sqrt(d_k); causal mask on the diagonal block.
      const float pf = exp2f(static_cast<float>((it.u - it.w - 1) * T) * log2g) * sd;
      const bool diag = (it.u == it.w);
      const uint32_t tS = tmem + C::COL_S + (k % C::SBUF) * T + lane_off;
      if constexpr (HALVES) {
        // row prow, columns [32 phalf, 32 phalf + 32) of the 64-column score tile
        uint32_t u16[2][16];
        tmem_ld16x2_wait<32>(tS, u16);
        tc_fence_before();
        mbar_arrive(bar(Q_S_FREE + (k % C::SBUF)));
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          const int col = 32 * phalf + 8 * c8;
          uint32_t pk[4], pl[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c0 = col + 2 * e;
            const float p0 = (!diag || c0 <= prow) ? __uint_as_float(u16[c8 / 2][(8 * c8 + 2 * e) % 16]) * pf : 0.f;
            const float p1 = (!diag || c0 + 1 <= prow) ? __uint_as_float(u16[c8 / 2][(8 * c8 + 2 * e + 1) % 16]) * pf : 0.f;
            pmx = absmax(absmax(pmx, p0), p1);
            if (HL) {
              split_f16x2(p0, p1, pk[e], pl[e]);
            } else {
              pk[e] = pack_f16x2(p0, p1);
            }
          }
          const uint32_t poff = sw128(prow, col / 8);
          st_shared_v4(sP(k) + poff, pk[0], pk[1], pk[2], pk[3]);
          if (HL) st_shared_v4(sP(k) + C::PBYTES + poff, pl[0], pl[1], pl[2], pl[3]);
        }
      }
#pragma unroll
      for (int grp = 0; grp < (HALVES ? 0 : T / C::LDW); ++grp) {
        uint32_t u16[C::LDW / 16][16];
        tmem_ld_wait(tS + grp * C::LDW, u16);
        if (grp == T / C::LDW - 1) {
          tc_fence_before();
          mbar_arrive(bar(Q_S_FREE + (k % C::SBUF)));
        }
        if (my_row >= 0) {
#pragma unroll
          for (int c8 = 0; c8 < C::LDW / 8; ++c8) {
            const int col = grp * C::LDW + 8 * c8;
            uint32_t pk[4], pl[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c0 = col + 2 * e;
              const float p0 = (!diag || c0 <= my_row) ? __uint_as_float(u16[c8 / 2][(8 * c8 + 2 * e) % 16]) * pf : 0.f;
              const float p1 = (!diag || c0 + 1 <= my_row) ? __uint_as_float(u16[c8 / 2][(8 * c8 + 2 * e + 1) % 16]) * pf : 0.f;
              pmx = absmax(absmax(pmx, p0), p1);
              if (HL) {
                split_f16x2(p0, p1, pk[e], pl[e]);
              } else {
                pk[e] = pack_f16x2(p0, p1);
              }
            }
            const uint32_t poff = (col / 64) * T * 128 + sw128(my_row, (col % 64) / 8);
            st_shared_v4(sP(k) + poff, pk[0], pk[1], pk[2], pk[3]);
            if (HL) st_shared_v4(sP(k) + C::PBYTES + poff, pl[0], pl[1], pl[2], pl[3]);
          }
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(bar(Q_P_FULL + (k % C::PBUF)));
      if (C::EPI_WARPS > 0) continue;
      if (pend_rb >= 0) {
        ok = epilogue(pend_rb, pend_i, pend_u, pend_bl);
        pend_rb = -1;
      }
      if (it.rb_done()) {
        pend_rb = it.rb; pend_i = it.i; pend_u = it.u; pend_bl = it.bl;
      }
    }
    if (ok && pend_rb >= 0) epilogue(pend_rb, pend_i, pend_u, pend_bl);
    report_fp16_range(pmx);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  if constexpr (FUSE) cluster_sync();  // no CTA leaves while a peer may still write into it
}

// ============================================================================================
// Segment-state pass (two-pass sequence segments, and the state of a sequence shard): for each
// sub-segment j of chunks [sub_lo[j], sub_hi[j]) with end token E, from a zero start,
//   W_j = sum_t gamma^(E-1-t) k~_t^T v_t  ("阅读笔记：RetNet" §2.4: the chunk recurrence unrolled
// over the sub-segment; it is associative, R <- gamma^len R + W, which the output pass uses).
// The whole sub-segment is one contraction, so there is no per-chunk state update: the key rows
// carry the decay to E, every increment Kz^T V accumulates into one tensor-memory tile, and the
// CTA is bound by streaming and converting K and V.  Roles: eight converter warps (K rotated and
// scaled, V to fp16; they also write W out at the end), a TMA warp, an MMA warp; stages hold K
// and V only.  Output: ws fp32 [j][batch][heads][d_k][d_v] (slice columns of this CTA).
// TWO: half the shared memory, two CTAs an SM (the state of a whole sequence shard, one CTA a
// (batch, head, slice): a second resident CTA hides the fixed cost; 1663 -> 1578 us on the
// b2/L8192/h16/d256/512 shard).  The two-pass segments keep one CTA an SM, which leaves SMs to
// the first output segment.
template <int DK, int T, int DVS, bool TWO = false>
struct CfgS {
  static constexpr int NCW = 8;
  static constexpr int NCONV = 32 * NCW;
  static constexpr int WARP_TMA = NCW, WARP_MMA = NCW + 1;
  static constexpr int THREADS = 32 * (NCW + 2);
  static constexpr int NDV = DVS / 64;
  static constexpr int RBLK = DK > 128 ? 2 : 1;  // 128-row blocks of the state
  static constexpr int MR = DK >= 128 ? 128 : 64;
  static constexpr int KBYTES = T * DK * 2, VBYTES = T * DVS * 2;
  static constexpr int STAGE = KBYTES + VBYTES;
  static constexpr int TABBYTES = 2 * 2 * (DK / 2) * 8;
  static constexpr int NBARS = 3 * 6 + 2 + 2;
  static constexpr int BUDGET = (TWO ? 113 : 227) * 1024 - 1024;
  static constexpr int NS_FIT = (BUDGET - TABBYTES - NBARS * 8 - 16) / STAGE;
  static constexpr int NS = NS_FIT > 6 ? 6 : NS_FIT;
  static constexpr int SMEM = NS * STAGE + TABBYTES + NBARS * 8 + 16 + 1024;
  static constexpr int TMEM_COLS = RBLK * DVS <= 128 ? 128 : 256;
  static_assert(NS >= 2, "segment-state stages");
};

template <int DK, int T, int DVS, bool TWO = false>
__global__ void __launch_bounds__(CfgS<DK, T, DVS, TWO>::THREADS, TWO ? 2 : 1)
    tc_segment_state_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                            TcArgs a, HeadParams hp) {
  using C = CfgS<DK, T, DVS, TWO>;
  enum : int { B_FULL = 0, B_CONV = 6, B_EMPTY = 12, B_TAB = 18, B_DONE = 20, B_DRAIN = 21 };
  griddep_launch_dependents();  // the output pass may start on the SMs this grid leaves idle
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - raw_addr);
  float2* tab = reinterpret_cast<float2*>(gbase + C::NS * C::STAGE);
  uint64_t* bars = reinterpret_cast<uint64_t*>(gbase + C::NS * C::STAGE + C::TABBYTES);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + C::NBARS);
  auto bar = [&](int i) { return smem_addr(bars + i); };
  auto sK = [&](int st) { return sbase + st * C::STAGE; };
  auto sV = [&](int st) { return sbase + st * C::STAGE + C::KBYTES; };

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_dvb = a.dv / DVS;
  const int dvb = blockIdx.x % n_dvb, seg = blockIdx.x / n_dvb, h = blockIdx.y, b = blockIdx.z;
  int s_lo = a.sub_lo[0], s_hi = a.sub_hi[0];
#pragma unroll
  for (int i = 1; i < kMaxSub; ++i)  // constant-index selects keep the kernel parameters in place
    if (seg == i) {
      s_lo = a.sub_lo[i];
      s_hi = a.sub_hi[i];
    }
  const int nb = a.nb;
  const float log2g = hp.log2g[h];

  if (threadIdx.x == 0) {
    for (int st = 0; st < 6; ++st) {
      mbar_init(bar(B_FULL + st), 1);
      mbar_init(bar(B_CONV + st), C::NCONV);
      mbar_init(bar(B_EMPTY + st), 1);
    }
    mbar_init(bar(B_TAB), C::NCONV);
    mbar_init(bar(B_TAB + 1), C::NCONV);
    mbar_init(bar(B_DONE), 1);
    mbar_init(bar(B_DRAIN), 1);
    fence_mbar_init();
  }
  if (warp == C::WARP_MMA) {
    tmem_alloc(smem_addr(tmem_holder), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == C::WARP_TMA && lane == 0) {
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == C::WARP_TMA) {
    if (lane == 0) {
      int issued[6] = {0, 0, 0, 0, 0, 0};
      UnitIter<T, SEG_STATE> it;
      for (it.start(a.L, nb, s_lo, s_hi, s_hi); it.valid(); it.next()) {
        const int st = it.k % C::NS;
        if (it.k >= C::NS && !mbar_wait(bar(B_EMPTY + st), ((it.k / C::NS) - 1) & 1)) break;
        mbar_arrive_expect_tx(bar(B_FULL + st), C::KBYTES + C::VBYTES);
        const int tk = it.t0() + it.w * T;
#pragma unroll
        for (int bx = 0; bx < DK / 64; ++bx) tma_load_4d(sK(st) + bx * T * 128, &tm_k, bar(B_FULL + st), bx * 64, h, tk, b);
#pragma unroll
        for (int bx = 0; bx < C::NDV; ++bx)
          tma_load_4d(sV(st) + bx * T * 128, &tm_v, bar(B_FULL + st), dvb * DVS + 64 * bx, h, tk, b);
        issued[st]++;
      }
      // Every load this thread issued must have landed before the CTA may exit.
      for (int st = 0; st < C::NS; ++st)
        if (issued[st] > 0) mbar_wait(bar(B_FULL + st), (issued[st] - 1) & 1, kDrainBudget);
    }
  } else if (warp == C::WARP_MMA) {
    if (lane == 0) {
      constexpr uint32_t ID_R = idesc_f16_f32(C::MR, DVS, 1, 1);
      UnitIter<T, SEG_STATE> f;
      bool first = true;
      for (f.start(a.L, nb, s_lo, s_hi, s_hi); f.valid(); f.next()) {
        const int st = f.k % C::NS;
        if (!mbar_wait(bar(B_CONV + st), (f.k / C::NS) & 1)) break;
        tc_fence_after();
        const uint64_t dkm = sdesc_sw128(sK(st), T * 128, 1024), dv = sdesc_sw128(sV(st), T * 128, 1024);
#pragma unroll
        for (int blk = 0; blk < C::RBLK; ++blk)
#pragma unroll
          for (int ks = 0; ks < T / 16; ++ks)
            mma_f16_ss(tmem + blk * DVS, dkm + static_cast<uint64_t>((blk * 2 * T * 128 + ks * 2048) >> 4),
                       dv + static_cast<uint64_t>((ks * 2048) >> 4), ID_R, (first && ks == 0) ? 0u : 1u);
        first = false;
        mma_commit(bar(B_EMPTY + st));
      }
      mma_commit(bar(B_DONE));
      mma_commit(bar(B_DRAIN));
      mbar_wait(bar(B_DRAIN), 0, kDrainBudget);
    }
  } else {
    // ------------------------------------------------------------------ converters
    UnitConverter<DK, T, C::NCONV, C::NDV> cv;
    cv.init(threadIdx.x, nb, hp);
    cv.conv_v = a.v_f16 == 0;
    const bool xpos = (a.flags & RETNET_F_XPOS) != 0;
    const int e_tok = min(s_hi * nb * T, a.L);  // the sub-segment's end E
    bool ok = true;
    float mx = 0.f;
    UnitIter<T, SEG_STATE> it;
    for (it.start(a.L, nb, s_lo, s_hi, s_hi); ok && it.valid(); it.next()) {
      const int st = it.k % C::NS;
      float2* tq = tab + (it.k & 1) * DK;
      float2* tk = tq + DK / 2;
      if (xpos) cv.put_bases(tq, tk, it.i, it.u, it.w, it.t0(), a.pos0, hp);
      // table buffer (k & 1) complete once all converters arrived (as in the pipelined kernel)
      mbar_arrive(bar(B_TAB + (it.k & 1)));
      ok = mbar_wait(bar(B_TAB + (it.k & 1)), (it.k >> 1) & 1);
      if (ok) ok = mbar_wait(bar(B_FULL + st), (it.k / C::NS) & 1);
      if (!ok) break;
      // K of column block w decays to E: gamma^(E - 1 - t) in all
      const int blk_end = it.t0() + (it.w + 1) * T;
      cv.template convert<false>(0, sK(st), sV(st), tq, tk, xpos, log2g, mx,
                                 exp2f(static_cast<float>(e_tok - blk_end) * log2g));
      fence_proxy_async_smem();
      mbar_arrive(bar(B_CONV + st));
    }
    report_fp16_range(mx);
    // W out: warp w reads TMEM lane quarter w % 4 (d_k rows), column half w / 4 of the slice.
    if (__all_sync(0xffffffffu, mbar_wait(bar(B_DONE), 0))) {
      tc_fence_after();
      const uint32_t lane_off = static_cast<uint32_t>(32 * (warp % 4)) << 16;
      const size_t plane = static_cast<size_t>(a.batch) * a.heads * DK * a.dv;
      constexpr int HALF = DVS / 2;
#pragma unroll 1
      for (int blk = 0; blk < C::RBLK; ++blk) {
        const int dk = (DK == 64) ? (lane < 16 ? 16 * (warp % 4) + lane : -1) : blk * 128 + 32 * (warp % 4) + lane;
        const int col0 = (warp / 4) * HALF;
        float* dst = a.ws + seg * plane + (static_cast<size_t>(b) * a.heads + h) * DK * a.dv + dvb * DVS + col0 +
                     static_cast<size_t>(dk < 0 ? 0 : dk) * a.dv;
#pragma unroll 1
        for (int grp = 0; grp < HALF / 32; ++grp) {
          uint32_t u[2][16];
          tmem_ld_wait(tmem + blk * DVS + col0 + 32 * grp + lane_off, u);
          if (dk >= 0) {
#pragma unroll
            for (int c4 = 0; c4 < 8; ++c4)
              *reinterpret_cast<float4*>(dst + 32 * grp + 4 * c4) =
                  make_float4(__uint_as_float(u[(4 * c4) / 16][(4 * c4) % 16]),
                              __uint_as_float(u[(4 * c4 + 1) / 16][(4 * c4 + 1) % 16]),
                              __uint_as_float(u[(4 * c4 + 2) / 16][(4 * c4 + 2) % 16]),
                              __uint_as_float(u[(4 * c4 + 3) / 16][(4 * c4 + 3) % 16]));
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == C::WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Conversion pre-pass (chunks of several sub-blocks).  The pipelined kernel converts Q_u, K_w
// and V_w for every unit (u, w), i.e. (nb + 1) / 2 times per token; this kernel writes fp16
// copies that already carry its operand scaling, once per token, and the pipelined kernel then
// loads MMA-ready tiles (no converter role).  With r = t mod T the row inside its T-row
// sub-block (chunks start at multiples of B, and T divides B):
//   q~ = gamma^(r+1) rot(q),   k~ = gamma^(T-1-r) rot(k),   v~ = v   (fp16),
// the rotation by the absolute position p = pos0 + t.  Thread = (token, 8-element slot of
// d_k) across every head (the rotation factors are computed once), then (8-element slots of v).
// ============================================================================================
// HL: q~ and k~ as split operands, hi parts into qo / ko, lo parts into qlo / klo.
template <int DK, int T, bool HL = false>
__global__ void __launch_bounds__(256) tc_convert_kernel(const uint4* __restrict__ q, const uint4* __restrict__ k,
                                                         const uint4* __restrict__ v, uint4* __restrict__ qo,
                                                         uint4* __restrict__ ko, uint4* __restrict__ vo,
                                                         uint4* __restrict__ qlo, uint4* __restrict__ klo,
                                                         int64_t tokens, int L, int heads, int dv, int64_t pos0,
                                                         uint32_t flags, HeadParams hp) {
  constexpr int S = DK / 8;  // 16-byte slots of a head row of q or k
  const int64_t n_qk = tokens * S;
  const int64_t n_v = tokens * heads * (dv / 8);
  const bool xpos = (flags & RETNET_F_XPOS) != 0;
  float mx = 0.f;  // largest magnitude rounded to fp16
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_qk + n_v;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    if (i < n_qk) {
      const int64_t n = i / S;
      const int sl = static_cast<int>(i % S);
      const int t = static_cast<int>(n % L), r = t % T;
      float2 f[4];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        float sn = 0.f, c = 1.f;
        if (xpos) xpos_sincos(pos0 + t, hp.theta[4 * sl + jj], &sn, &c);
        f[jj] = make_float2(c, sn);
      }
      for (int h = 0; h < heads; ++h) {
        const int64_t off = (n * heads + h) * S + sl;
        const uint4 xq = q[off], xk = k[off];
        const float l2g = hp.log2g[h];
        const float xi = decay_pow(l2g, r + 1), zeta = decay_pow(l2g, T - 1 - r);
        const uint32_t wq[4] = {xq.x, xq.y, xq.z, xq.w}, wk[4] = {xk.x, xk.y, xk.z, xk.w};
        uint32_t oq[4], ok[4], lq[4], lk[4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const float q0 = __uint_as_float(wq[jj] << 16), q1 = __uint_as_float(wq[jj] & 0xffff0000u);
          const float k0 = __uint_as_float(wk[jj] << 16), k1 = __uint_as_float(wk[jj] & 0xffff0000u);
          const float x0 = xi * (q0 * f[jj].x - q1 * f[jj].y), x1 = xi * (q0 * f[jj].y + q1 * f[jj].x);
          const float y0 = zeta * (k0 * f[jj].x - k1 * f[jj].y), y1 = zeta * (k0 * f[jj].y + k1 * f[jj].x);
          mx = absmax(absmax(absmax(absmax(mx, x0), x1), y0), y1);
          if (HL) {
            split_f16x2(x0, x1, oq[jj], lq[jj]);
            split_f16x2(y0, y1, ok[jj], lk[jj]);
          } else {
            oq[jj] = pack_f16x2(x0, x1);
            ok[jj] = pack_f16x2(y0, y1);
          }
        }
        qo[off] = make_uint4(oq[0], oq[1], oq[2], oq[3]);
        ko[off] = make_uint4(ok[0], ok[1], ok[2], ok[3]);
        if (HL) {
          qlo[off] = make_uint4(lq[0], lq[1], lq[2], lq[3]);
          klo[off] = make_uint4(lk[0], lk[1], lk[2], lk[3]);
        }
      }
    } else {
      const int64_t j = i - n_qk;
      const uint4 x = v[j];
      const uint32_t w[4] = {x.x, x.y, x.z, x.w};
      uint32_t o[4];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const float v0 = __uint_as_float(w[jj] << 16), v1 = __uint_as_float(w[jj] & 0xffff0000u);
        mx = absmax(absmax(mx, v0), v1);
        o[jj] = pack_f16x2(v0, v1);
      }
      vo[j] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  report_fp16_range(mx);
}

// ============================================================================================
// P pass (chunks of several 64-row sub-blocks, d_k = 256).  Each d_v slice of a head needs the
// same masked scores P_{u,w} = (Qx_u Kz_w^T) gamma^((u-w-1)T) / sqrt(d_k) (causal mask on the
// diagonal block u = w) for every unit (u, w) of every chunk; the pipelined kernel computing
// them itself repeats that work for each of the d_v / 64 slices.  This kernel computes each P
// tile once, from the conversion pre-pass's copies, into the workspace: fp16, row-major
// [tile][T][T], tile = ((b heads + h) n_chunks + i) U + u (u + 1) / 2 + w, U = nb (nb + 1) / 2.
// The pipelined kernel (PS) then loads P by TMA beside V.  One CTA a tile: warp 4 loads Q_u
// and K_w (TMA, 128-byte swizzle), issues the DK / 16 MMAs into tensor memory; warps 0-3 scale,
// mask and store the rows.  The causal mask, the row scale and the rounding to fp16 are those
// of the P warps of the pipelined kernel, so the results are bit-identical.
// ============================================================================================
template <int DK, int T>
__global__ void __launch_bounds__(160, 1) tc_p_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                      const __grid_constant__ CUtensorMap tm_k, uint4* __restrict__ P,
                                                      int L, int heads, int n_chunks, int nb, HeadParams hp) {
  static_assert(T == 64, "P pass: 64-row sub-blocks");
  constexpr int QB = T * DK * 2;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - raw_addr);
  const uint32_t sQ = sbase, sK = sbase + QB;
  uint64_t* bars = reinterpret_cast<uint64_t*>(gbase + 2 * QB);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2);
  const int U = nb * (nb + 1) / 2;
  const int unit = blockIdx.x, i = blockIdx.y, bh = blockIdx.z;
  int u = 0;
  while ((u + 1) * (u + 2) / 2 <= unit) ++u;
  const int w = unit - u * (u + 1) / 2;
  const int t0 = i * nb * T;
  if (t0 + u * T >= L) return;  // a row block past the end of a short last chunk: never read
  const int h = bh % heads, b = bh / heads;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    mbar_init(smem_addr(bars), 1);
    mbar_init(smem_addr(bars + 1), 1);
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(smem_addr(tmem_holder), 64);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const float log2g = hp.log2g[h];
  if (warp == 4) {
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      mbar_arrive_expect_tx(smem_addr(bars), 2 * QB);
#pragma unroll
      for (int bx = 0; bx < DK / 64; ++bx) {
        tma_load_4d(sQ + bx * T * 128, &tm_q, smem_addr(bars), bx * 64, h, t0 + u * T, b);
        tma_load_4d(sK + bx * T * 128, &tm_k, smem_addr(bars), bx * 64, h, t0 + w * T, b);
      }
      // the loads are waited for with the full budget: they were issued and always land
      if (mbar_wait(smem_addr(bars), 0, kDrainBudget)) {
        tc_fence_after();
        constexpr uint32_t ID_S = idesc_f16_f32(T, T, 0, 0);
        const uint64_t dq = sdesc_sw128(sQ, 16, 1024), dk = sdesc_sw128(sK, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
          const uint64_t ks = static_cast<uint64_t>(((kk / 4) * T * 128 + (kk % 4) * 32) >> 4);
          mma_f16_ss(tmem, dq + ks, dk + ks, ID_S, kk > 0);
        }
      }
      mma_commit(smem_addr(bars + 1));  // (after no MMA it arrives at once)
      mbar_wait(smem_addr(bars + 1), 0, kDrainBudget);
    }
  } else {
    // rows of the M = 64 accumulator: lanes 0-15 of each warp's 32-lane quarter
    const uint32_t lane_off = static_cast<uint32_t>(32 * warp) << 16;
    const int my_row = lane < 16 ? 16 * warp + lane : -1;
    float pmx = 0.f;
    if (__all_sync(0xffffffffu, mbar_wait(smem_addr(bars + 1), 0))) {
      tc_fence_after();
      const float pf = exp2f(static_cast<float>((u - w - 1) * T) * log2g) * rsqrtf(static_cast<float>(DK));
      const bool diag = (u == w);
      uint32_t r[4][16];
      tmem_ld_wait(tmem + lane_off, r);
      if (my_row >= 0) {
        const int64_t tile = (static_cast<int64_t>(bh) * n_chunks + i) * U + unit;
        uint4* dst = P + (tile * T + my_row) * (T * 2 / 16);
#pragma unroll
        for (int c8 = 0; c8 < T / 8; ++c8) {
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c0 = 8 * c8 + 2 * e;
            const float p0 = (!diag || c0 <= my_row) ? __uint_as_float(r[c0 / 16][c0 % 16]) * pf : 0.f;
            const float p1 = (!diag || c0 + 1 <= my_row) ? __uint_as_float(r[(c0 + 1) / 16][(c0 + 1) % 16]) * pf : 0.f;
            pmx = absmax(absmax(pmx, p0), p1);
            pk[e] = pack_f16x2(p0, p1);
          }
          dst[c8] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
    }
    report_fp16_range(pmx);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
  }
}

// P pass, one CTA a (chunk, batch x head): the same tiles as tc_p_kernel, computed in turn by a
// pipeline that keeps its operands on chip -- Q_u in one of two slots for the units of row block
// u, K_w through a ring of three -- so that the launch, the tensor-memory set-up and the first
// loads' latency are paid once a chunk rather than once a tile.  Warp 4 loads (TMA), warp 5
// issues the MMAs into one of two tensor-memory score buffers, warps 0-3 scale, mask and store
// (two threads a row, each 32 columns).  Same arithmetic as tc_p_kernel: bit-identical tiles.
constexpr int kPChunkK = 3;  // K tiles in flight (two Q slots, three K slots: 160 KB at d_k 256; five ran no faster)
template <int DK, int T>
__global__ void __launch_bounds__(192, 1) tc_p_chunk_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                            const __grid_constant__ CUtensorMap tm_k,
                                                            uint4* __restrict__ P, int L, int heads, int n_chunks,
                                                            int nb, HeadParams hp) {
  static_assert(T == 64, "P pass: 64-row sub-blocks");
  constexpr int QB = T * DK * 2;
  constexpr int NQ = 2, NK = kPChunkK;
  enum : int { B_QF = 0, B_QE = 2, B_KF = 4, B_KE = 4 + NK, B_SF = 4 + 2 * NK, B_SE = 6 + 2 * NK, B_DR = 8 + 2 * NK,
               NB_ = 9 + 2 * NK };
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - raw_addr);
  auto sQ = [&](int j) { return sbase + j * QB; };
  auto sK = [&](int j) { return sbase + (NQ + j) * QB; };
  uint64_t* bars = reinterpret_cast<uint64_t*>(gbase + (NQ + NK) * QB);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + NB_);
  auto bar = [&](int j) { return smem_addr(bars + j); };
  const int U = nb * (nb + 1) / 2;
  const int i = blockIdx.x, bh = blockIdx.y;
  const int h = bh % heads, b = bh / heads;
  const int t0 = i * nb * T;
  const int nbw = min(nb, (L - t0 + T - 1) / T);  // row blocks of this chunk inside the sequence
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int j = 0; j < NB_; ++j) mbar_init(bar(j), (j == B_SE || j == B_SE + 1) ? 128 : 1);
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_addr(tmem_holder), 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const float log2g = hp.log2g[h];
  if (warp == 4) {
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      int k = 0, q_issued[NQ] = {0, 0}, k_issued[NK] = {};
      bool ok = true;
      for (int u = 0; ok && u < nbw; ++u) {
        const int qs = u % NQ;
        if (u >= NQ && !mbar_wait(bar(B_QE + qs), ((u / NQ) - 1) & 1)) break;
        mbar_arrive_expect_tx(bar(B_QF + qs), QB);
#pragma unroll
        for (int bx = 0; bx < DK / 64; ++bx) tma_load_4d(sQ(qs) + bx * T * 128, &tm_q, bar(B_QF + qs), bx * 64, h, t0 + u * T, b);
        q_issued[qs]++;
        for (int w = 0; w <= u; ++w, ++k) {
          const int ks = k % NK;
          if (k >= NK && !mbar_wait(bar(B_KE + ks), ((k / NK) - 1) & 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(B_KF + ks), QB);
#pragma unroll
          for (int bx = 0; bx < DK / 64; ++bx)
            tma_load_4d(sK(ks) + bx * T * 128, &tm_k, bar(B_KF + ks), bx * 64, h, t0 + w * T, b);
          k_issued[ks]++;
        }
      }
      // every load this thread issued lands before the CTA may exit
      for (int j = 0; j < NQ; ++j)
        if (q_issued[j] > 0) mbar_wait(bar(B_QF + j), (q_issued[j] - 1) & 1, kDrainBudget);
      for (int j = 0; j < NK; ++j)
        if (k_issued[j] > 0) mbar_wait(bar(B_KF + j), (k_issued[j] - 1) & 1, kDrainBudget);
    }
  } else if (warp == 5) {
    if (lane == 0) {
      constexpr uint32_t ID_S = idesc_f16_f32(T, T, 0, 0);
      int k = 0;
      bool ok = true;
      for (int u = 0; ok && u < nbw; ++u) {
        const int qs = u % NQ;
        if (!mbar_wait(bar(B_QF + qs), (u / NQ) & 1)) break;
        for (int w = 0; w <= u; ++w, ++k) {
          const int ks = k % NK, sb = k % 2;
          ok = mbar_wait(bar(B_KF + ks), (k / NK) & 1);
          if (ok && k >= 2) ok = mbar_wait(bar(B_SE + sb), ((k / 2) - 1) & 1);
          if (!ok) break;
          tc_fence_after();
          const uint64_t dq = sdesc_sw128(sQ(qs), 16, 1024), dk = sdesc_sw128(sK(ks), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < DK / 16; ++kk) {
            const uint64_t kst = static_cast<uint64_t>(((kk / 4) * T * 128 + (kk % 4) * 32) >> 4);
            mma_f16_ss(tmem + sb * T, dq + kst, dk + kst, ID_S, kk > 0);
          }
          mma_commit(bar(B_SF + sb));
          mma_commit(bar(B_KE + ks));
        }
        mma_commit(bar(B_QE + qs));
      }
      mma_commit(bar(B_DR));
      mbar_wait(bar(B_DR), 0, kDrainBudget);
    }
  } else {
    // rows of the M = 64 score tile: lanes 0-15 of each warp's lane quarter; lanes l and l + 16
    // take row 16 warp + (l mod 16), columns [32 (l / 16), 32 (l / 16) + 32)
    const uint32_t lane_off = static_cast<uint32_t>(32 * warp) << 16;
    const int prow = 16 * warp + (lane & 15), phalf = lane >> 4;
    const float sdk = rsqrtf(static_cast<float>(DK));
    float pmx = 0.f;
    int k = 0;
    bool ok = true;
    for (int u = 0; ok && u < nbw; ++u) {
      for (int w = 0; w <= u; ++w, ++k) {
        const int sb = k % 2;
        ok = __all_sync(0xffffffffu, mbar_wait(bar(B_SF + sb), (k / 2) & 1));
        if (!ok) break;
        tc_fence_after();
        uint32_t r[2][16];
        tmem_ld16x2_wait<32>(tmem + sb * T + lane_off, r);
        tc_fence_before();
        mbar_arrive(bar(B_SE + sb));
        const float pf = exp2f(static_cast<float>((u - w - 1) * T) * log2g) * sdk;
        const bool diag = (u == w);
        const int64_t tile = (static_cast<int64_t>(bh) * n_chunks + i) * U + u * (u + 1) / 2 + w;
        uint4* dst = P + (tile * T + prow) * (T * 2 / 16) + 4 * phalf;
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = 8 * c8 + 2 * e, c0 = 32 * phalf + c;
            const float p0 = (!diag || c0 <= prow) ? __uint_as_float(r[c / 16][c % 16]) * pf : 0.f;
            const float p1 = (!diag || c0 + 1 <= prow) ? __uint_as_float(r[(c + 1) / 16][(c + 1) % 16]) * pf : 0.f;
            pmx = absmax(absmax(pmx, p0), p1);
            pk[e] = pack_f16x2(p0, p1);
          }
          dst[c8] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
    }
    report_fp16_range(pmx);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// ---- host side -------------------------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;  // resolved once from the driver; no CUDA context state
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 4-D map over a BLHD bf16 tensor [b][L][h][d] with a (64, 1, T, 1) box, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, int64_t b, int64_t L, int64_t h, int64_t d, int T) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(h), static_cast<cuuint64_t>(L),
                        static_cast<cuuint64_t>(b)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(d * 2), static_cast<cuuint64_t>(h * d * 2),
                           static_cast<cuuint64_t>(L * h * d * 2)};
  cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(T), 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Map over P tiles [tile][T][T] fp16 (2-byte elements), box of one T x T tile, 128-byte swizzle.
bool make_map_p(CUtensorMap* m, const void* base, int64_t tiles, int T) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(tiles), 1};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(T * 2), static_cast<cuuint64_t>(T * T * 2),
                           static_cast<cuuint64_t>(tiles * T * T * 2)};
  cuuint32_t box[4] = {64, static_cast<cuuint32_t>(T), 1, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// RETNET_TC_KERNEL=serial in the environment (read once) sends every tensor-core call to the
// serial kernel, so that tests can hold both kernels to the oracle on the same shapes.
bool force_serial_kernel() {
  static const bool serial = [] {
    const char* v = getenv("RETNET_TC_KERNEL");
    return v != nullptr && strcmp(v, "serial") == 0;
  }();
  return serial;
}

// Rows per unit of the pipelined kernel: 64 for d_k = 256 (shared memory), else min(B, 128);
// split operands (precise calls) always take 64-row units.
int pipe_tile_rows(int64_t d_k, int64_t chunk) { return d_k == 256 ? 64 : static_cast<int>(chunk < 128 ? chunk : 128); }
int pipe_tile_rows(const RetentionCall& c) { return c.precise ? 64 : pipe_tile_rows(c.dims.d_k, c.chunk); }

// Segment plan of a call (see plan_segments); returns how many pre-pass states the caller's
// workspace holds (0: no workspace, single-launch replay form).
int sm_count();
void plan_segments(TcArgs& a, int64_t ctas, int sms, double rho, int max_seg);
constexpr double kReplayCost = 0.45;  // a replayed chunk, relative to an output chunk (measured)
int plan_call(const RetentionCall& c, int64_t ctas, int sms, TcArgs& as) {
  const size_t state_bytes = sizeof(float) * static_cast<size_t>(c.dims.batch * c.dims.heads * c.dims.d_k * c.dims.d_v);
  const int max_states = (c.ws && state_bytes > 0) ? static_cast<int>(std::min<size_t>(c.ws_bytes / state_bytes, kMaxSub)) : 0;
  if (max_states >= 1)
    plan_segments(as, ctas, sms, 0.0, std::min(4, max_states + 1));
  else
    plan_segments(as, ctas, sms, kReplayCost, 4);
  return max_states;
}

// fp16 copies of the conversion pre-pass in the caller's workspace (256-byte aligned parts):
// q~, k~, v, and for split operands the lo parts of q~ and k~ after them.
struct PreCopies {
  void* q;
  void* k;
  void* v;
  void* ql;
  void* kl;
};
size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
size_t pre_copy_bytes(const Dims& d, bool hl) {
  const size_t tok = static_cast<size_t>(d.batch) * static_cast<size_t>(d.seqlen) * static_cast<size_t>(d.heads);
  return (hl ? 4 : 2) * align256(tok * d.d_k * 2) + align256(tok * d.d_v * 2);
}
PreCopies pre_copies(const RetentionCall& c) {
  const size_t tok = static_cast<size_t>(c.dims.batch) * static_cast<size_t>(c.dims.seqlen) *
                     static_cast<size_t>(c.dims.heads);
  char* base = static_cast<char*>(c.ws);
  const size_t qk = align256(tok * c.dims.d_k * 2), vb = align256(tok * c.dims.d_v * 2);
  return PreCopies{base, base + qk, base + 2 * qk, base + 2 * qk + vb, base + 3 * qk + vb};
}
// The pre-pass pays one extra read and write of q, k, v; it saves the (nb + 1) / 2-fold
// reconversion of chunks of nb >= 2 sub-blocks.  Not combined with sequence segments.
bool pre_convert_applies(const RetentionCall& c, int nb, int n_seg) {
  return nb >= 2 && n_seg < 2 && !c.v_f16 && c.ws && c.ws_bytes >= pre_copy_bytes(c.dims, c.precise);
}

// P pass (d_k = 256, 64-row sub-blocks, chunks of several of them, single operands, no fused
// epilogue, no segments): the P tiles of every unit of every chunk, after the fp16 copies.
int64_t p_tiles(const Dims& d, int64_t chunk, int T) {
  const int64_t nb = chunk / T, n_chunks = (d.seqlen + chunk - 1) / chunk;
  return d.batch * d.heads * n_chunks * (nb * (nb + 1) / 2);
}
size_t p_tile_bytes(const Dims& d, int64_t chunk, int T) {
  return align256(static_cast<size_t>(p_tiles(d, chunk, T)) * T * T * 2);
}
// Which P-pass kernel: one CTA a chunk (its tiles pipelined) or one CTA a tile.
bool use_p_chunk_kernel(int nb) {
  const char* e = getenv("RETNET_P_TILE_KERNEL");  // testing aid: force the per-tile kernel
  return !(e && e[0] == '1') && nb >= 4;  // chunk 128 (two sub-blocks): the per-tile kernel was faster
}
bool p_pass_applies(const RetentionCall& c, int T, int nb, int n_seg) {
  if (c.dims.d_k != 256 || T != 64 || nb < 2 || c.precise || c.gate || n_seg >= 2 || !c.ws) return false;
  const int64_t n_chunks = (c.dims.seqlen + c.chunk - 1) / c.chunk;
  if (n_chunks > 65535 || c.dims.batch * c.dims.heads > 65535 || p_tiles(c.dims, c.chunk, T) >= (1LL << 31)) return false;
  return c.ws_bytes >= pre_copy_bytes(c.dims, false) + p_tile_bytes(c.dims, c.chunk, T);
}

// 128-column d_v slices share S and the Q/K conversion across twice the output columns
// (about 1.6x the work per SM); they need one sub-block per chunk (no cross accumulator in
// tensor memory) and d_k <= 128.  The halved CTA count is made up by sequence segments.
bool pipe_wide_slice(const RetentionCall& c, int T) {
  return !c.gate && c.dims.d_k <= 128 && T == 64 && c.chunk == 64 && c.dims.d_v % 128 == 0;
}

int sm_count() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  return sms;
}

// Sequence segments.  With fewer (batch, head, d_v slice) CTAs than SMs, the chunks are split
// into n_seg consecutive segments, one CTA each; the CTA of segment s first replays the state
// over chunks [0, lo_s) (K and V only: TMA, conversion, state increment), then produces the
// outputs of [lo_s, hi_s).  A replayed chunk costs about kReplayCost of an output chunk, and
// the boundaries equalise rho * lo_s + (hi_s - lo_s) across segments.
// With a workspace (two passes) nothing is replayed: a pre-pass launch computes each
// segment's own state in parallel and the segments split the chunks evenly (rho = 0).
void plan_segments(TcArgs& a, int64_t ctas, int sms, double rho, int max_seg) {
  const int n = a.n_chunks;
  int n_seg = (ctas > 0 && sms > 0) ? static_cast<int>(sms / ctas) : 1;
  n_seg = std::min(n_seg, max_seg);
  n_seg = std::min(n_seg, n / 4);  // at least four chunks a segment
  if (n_seg < 2) return;
  if (rho <= 0.0) {
    for (int s = 0; s < n_seg; ++s) {
      a.seg_lo[s] = static_cast<int>(static_cast<int64_t>(n) * s / n_seg);
      a.seg_hi[s] = static_cast<int>(static_cast<int64_t>(n) * (s + 1) / n_seg);
    }
    a.n_seg = n_seg;
    return;
  }
  const double keep = 1.0 - rho;
  const double cost = n * rho / (1.0 - std::pow(keep, n_seg));
  double x = 0.0;
  int prev = 0;
  for (int s = 0; s < n_seg; ++s) {
    x = keep * x + cost;
    int hi = (s == n_seg - 1) ? n : static_cast<int>(std::lround(x));
    hi = std::max(hi, prev + 1);
    hi = std::min(hi, n - (n_seg - 1 - s));
    a.seg_lo[s] = prev;
    a.seg_hi[s] = hi;
    prev = hi;
  }
  a.n_seg = n_seg;
}

TcArgs make_args(const RetentionCall& c, int n_chunks, int nb) {
  TcArgs a;
  a.ws = nullptr;
  a.o = c.o;
  a.state_in = c.state_in;
  a.state_out = c.state_out;
  a.L = static_cast<int>(c.dims.seqlen);
  a.heads = static_cast<int>(c.dims.heads);
  a.batch = static_cast<int>(c.dims.batch);
  a.gate = c.gate;
  a.eps = c.eps;
  a.rden = c.rden;
  a.dv = static_cast<int>(c.dims.d_v);
  a.n_chunks = n_chunks;
  a.pos0 = c.pos0;
  a.flags = c.flags;
  a.nb = nb;
  a.v_f16 = c.v_f16 ? 1 : 0;
  a.o_rev = c.o_rev ? 1 : 0;
  a.n_seg = 1;
  a.n_sub = 0;
  for (int s = 0; s < 4; ++s) a.seg_lo[s] = a.seg_hi[s] = a.sub_before[s] = 0;
  for (int j = 0; j < kMaxSub; ++j) a.sub_lo[j] = a.sub_hi[j] = 0;
  a.seg_hi[0] = n_chunks;
  return a;
}

bool make_maps(const RetentionCall& c, int T, CUtensorMap* mq, CUtensorMap* mk, CUtensorMap* mv) {
  const Dims& d = c.dims;
  return make_map(mq, c.q, d.batch, d.seqlen, d.heads, d.d_k, T) &&
         make_map(mk, c.k, d.batch, d.seqlen, d.heads, d.d_k, T) &&
         make_map(mv, c.v, d.batch, d.seqlen, d.heads, d.d_v, T);
}

dim3 tc_grid(const Dims& d, int dvs) {
  return dim3(static_cast<unsigned>(d.d_v / dvs), static_cast<unsigned>(d.heads), static_cast<unsigned>(d.batch));
}

// Conversion pre-pass into the workspace copies (pc), then tensor maps over them.
template <int DK, int T, bool HL>
cudaError_t run_convert(const RetentionCall& c, const HeadParams& hp, cudaStream_t s, const PreCopies& pc,
                        CUtensorMap* m) {
  const int64_t tokens = c.dims.batch * c.dims.seqlen;
  const int64_t items = tokens * (DK / 8) + tokens * c.dims.heads * (c.dims.d_v / 8);
  const int blocks = static_cast<int>(std::min<int64_t>((items + 255) / 256, static_cast<int64_t>(sm_count()) * 8));
  tc_convert_kernel<DK, T, HL><<<blocks, 256, 0, s>>>(
      static_cast<const uint4*>(c.q), static_cast<const uint4*>(c.k), static_cast<const uint4*>(c.v),
      static_cast<uint4*>(pc.q), static_cast<uint4*>(pc.k), static_cast<uint4*>(pc.v), static_cast<uint4*>(pc.ql),
      static_cast<uint4*>(pc.kl), tokens, static_cast<int>(c.dims.seqlen), static_cast<int>(c.dims.heads),
      static_cast<int>(c.dims.d_v), c.pos0, c.flags, hp);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  RetentionCall cc = c;
  cc.q = pc.q;
  cc.k = pc.k;
  cc.v = pc.v;
  if (!make_maps(cc, T, &m[0], &m[1], &m[2])) return cudaErrorInvalidValue;
  m[3] = m[0];
  m[4] = m[1];
  if (HL) {
    const Dims& d = c.dims;
    if (!make_map(&m[3], pc.ql, d.batch, d.seqlen, d.heads, d.d_k, T) ||
        !make_map(&m[4], pc.kl, d.batch, d.seqlen, d.heads, d.d_k, T))
      return cudaErrorInvalidValue;
  }
  return cudaSuccess;
}

// One launch of the pipelined kernel over the (d_v slice, head, batch) grid.  cluster > 0: the
// d_v slices of a head form one thread-block cluster of that many CTAs (the fused GroupNorm
// epilogue uses cluster-scope instructions, so it is launched as a cluster even with one CTA);
// cluster = 0: no cluster.
template <typename K>
cudaError_t launch_kernel(K kern, dim3 grid, int threads, int smem, cudaStream_t s, const CUtensorMap* m,
                          const TcArgs& a, const HeadParams& hp, int cluster) {
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  if (cluster > 0) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, kern, m[0], m[1], m[2], m[3], m[4], a, hp);
}

// Fused MSR epilogue (c.gate) and split operands (HL): one CTA per (batch, head, 64-column d_v
// slice), no sequence segments.  With the gate, the d_v slices of a head form one thread-block
// cluster (n_cl <= kMaxCluster CTAs) that pools the GroupNorm statistics in distributed shared
// memory.  With chunks of several sub-blocks and room in the workspace the conversion pre-pass
// runs first.
template <int DK, int T, typename Tout, bool HL>
cudaError_t launch_unsplit(const RetentionCall& c, const HeadParams& hp, cudaStream_t s, const CUtensorMap* maps,
                           const TcArgs& a, int nb) {
  const bool fuse = c.gate != nullptr;
  const int n_cl = fuse ? static_cast<int>(c.dims.d_v / 64) : 1;
  if (n_cl < 1 || n_cl > kMaxCluster) return cudaErrorInvalidValue;
  const dim3 grid = tc_grid(c.dims, 64);
  if constexpr (Cfg3<DK, T, 64>::XBUF > 0) {
    if (pre_convert_applies(c, nb, 1)) {
      CUtensorMap pm[5];
      cudaError_t e = run_convert<DK, T, HL>(c, hp, s, pre_copies(c), pm);
      if (e != cudaSuccess) return e;
      if (fuse) {
        using CP = Cfg3<DK, T, 64, true, true, HL>;
        static_assert(CP::FITS, "fused kernel does not fit this tile");
        return launch_kernel(tc_chunkwise_pipe_kernel<DK, T, 64, SEG_NONE, true, true, Tout, HL>, grid, CP::THREADS,
                             CP::SMEM, s, pm, a, hp, n_cl);
      }
      using CP = Cfg3<DK, T, 64, true, false, HL>;
      static_assert(CP::FITS, "pipelined kernel does not fit this tile");
      return launch_kernel(tc_chunkwise_pipe_kernel<DK, T, 64, SEG_NONE, true, false, Tout, HL>, grid, CP::THREADS,
                           CP::SMEM, s, pm, a, hp, 0);
    }
  }
  if (fuse) {
    using CF = Cfg3<DK, T, 64, false, true, HL>;
    static_assert(CF::FITS, "fused kernel does not fit this tile");
    return launch_kernel(tc_chunkwise_pipe_kernel<DK, T, 64, SEG_NONE, false, true, Tout, HL>, grid, CF::THREADS,
                         CF::SMEM, s, maps, a, hp, n_cl);
  }
  using CF = Cfg3<DK, T, 64, false, false, HL>;
  static_assert(CF::FITS, "pipelined kernel does not fit this tile");
  return launch_kernel(tc_chunkwise_pipe_kernel<DK, T, 64, SEG_NONE, false, false, Tout, HL>, grid, CF::THREADS,
                       CF::SMEM, s, maps, a, hp, 0);
}

// Split operands (precise calls: RETNET_F_PRECISE, R~ and the fused MSR epilogue): 64-row units,
// 64-column d_v slices, no sequence segments.
template <int DK, typename Tout>
cudaError_t launch_pipe_hl(const RetentionCall& c, const HeadParams& hp, cudaStream_t s) {
  CUtensorMap m[5];
  if (!make_maps(c, 64, &m[0], &m[1], &m[2])) return cudaErrorInvalidValue;
  m[3] = m[0];
  m[4] = m[1];
  const int nb = static_cast<int>(c.chunk / 64);
  const TcArgs a = make_args(c, static_cast<int>((c.dims.seqlen + c.chunk - 1) / c.chunk), nb);
  return launch_unsplit<DK, 64, Tout, true>(c, hp, s, m, a, nb);
}

// Pipelined kernel: units of T rows, nb = B / T per chunk, d_v slices of DVS columns.
template <int DK, int T, int DVS, typename Tout>
cudaError_t launch_pipe(const RetentionCall& c, const HeadParams& hp, cudaStream_t s) {
  using Cf = Cfg3<DK, T, DVS>;
  using CfP = Cfg3<DK, T, DVS, true>;
  static_assert(Cf::FITS, "pipelined kernel does not fit this tile");
  CUtensorMap mq, mk, mv;
  if (!make_maps(c, T, &mq, &mk, &mv)) return cudaErrorInvalidValue;
  const CUtensorMap m5[5] = {mq, mk, mv, mq, mk};
  const int nb = static_cast<int>(c.chunk / T);
  const TcArgs a = make_args(c, static_cast<int>((c.dims.seqlen + c.chunk - 1) / c.chunk), nb);
  if (Cf::XBUF == 0 && nb != 1) return cudaErrorInvalidValue;
  if (c.gate) {  // fused MSR epilogue: no segments, one cluster per (batch, head)
    if constexpr (DVS == 64) return launch_unsplit<DK, T, Tout, false>(c, hp, s, m5, a, nb);
    return cudaErrorInvalidValue;
  }
  TcArgs as = a;
  const dim3 grid = tc_grid(c.dims, DVS);
  const int64_t ctas = static_cast<int64_t>(grid.x) * grid.y * grid.z;
  const int sms = sm_count();
  const int max_states = plan_call(c, ctas, sms, as);
  auto run = [&](auto kern, unsigned nx) -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::SMEM);
    if (e != cudaSuccess) return e;
    kern<<<dim3(grid.x * nx, grid.y, grid.z), Cf::THREADS, Cf::SMEM, s>>>(mq, mk, mv, mq, mk, as, hp);
    return cudaGetLastError();
  };
  if (as.n_seg < 2) {
    if constexpr (Cf::XBUF > 0) {
      // Chunks of several sub-blocks, no segments, and a workspace that holds the fp16
      // copies: convert once in a pre-pass, then run the kernel without converters.
      if (pre_convert_applies(c, nb, as.n_seg)) {
        CUtensorMap pm[5];
        cudaError_t e = run_convert<DK, T, false>(c, hp, s, pre_copies(c), pm);
        if (e != cudaSuccess) return e;
        if constexpr (DK == 256 && T == 64 && DVS == 64) {
          if (p_pass_applies(c, T, nb, as.n_seg)) {
            // P tiles once per head (P pass), then the pipelined kernel loads them beside V
            void* ptiles = static_cast<char*>(c.ws) + pre_copy_bytes(c.dims, false);
            const int64_t n_chunks = (c.dims.seqlen + c.chunk - 1) / c.chunk;
            const int U = nb * (nb + 1) / 2;
            if (use_p_chunk_kernel(nb)) {  // one CTA a chunk, operands pipelined on chip
              constexpr int PCSMEM = (2 + kPChunkK) * T * DK * 2 + 1024 + (9 + 2 * kPChunkK) * 8 + 16;
              e = cudaFuncSetAttribute(tc_p_chunk_kernel<DK, T>, cudaFuncAttributeMaxDynamicSharedMemorySize, PCSMEM);
              if (e != cudaSuccess) return e;
              tc_p_chunk_kernel<DK, T><<<dim3(static_cast<unsigned>(n_chunks), static_cast<unsigned>(c.dims.batch * c.dims.heads)),
                                         192, PCSMEM, s>>>(pm[0], pm[1], static_cast<uint4*>(ptiles),
                                                           static_cast<int>(c.dims.seqlen), static_cast<int>(c.dims.heads),
                                                           static_cast<int>(n_chunks), nb, hp);
            } else {  // one CTA a tile
              constexpr int PSMEM = 2 * T * DK * 2 + 1024 + 64;
              e = cudaFuncSetAttribute(tc_p_kernel<DK, T>, cudaFuncAttributeMaxDynamicSharedMemorySize, PSMEM);
              if (e != cudaSuccess) return e;
              tc_p_kernel<DK, T><<<dim3(U, static_cast<unsigned>(n_chunks), static_cast<unsigned>(c.dims.batch * c.dims.heads)),
                                   160, PSMEM, s>>>(pm[0], pm[1], static_cast<uint4*>(ptiles),
                                                    static_cast<int>(c.dims.seqlen), static_cast<int>(c.dims.heads),
                                                    static_cast<int>(n_chunks), nb, hp);
            }
            e = cudaGetLastError();
            if (e != cudaSuccess) return e;
            if (!make_map_p(&pm[3], ptiles, p_tiles(c.dims, c.chunk, T), T)) return cudaErrorInvalidValue;
            using CPS = Cfg3<DK, T, DVS, true, false, false, true>;
            static_assert(CPS::FITS, "pipelined kernel with P tiles does not fit this tile");
            return launch_kernel(tc_chunkwise_pipe_kernel<DK, T, DVS, SEG_NONE, true, false, Tout, false, true>, grid,
                                 CPS::THREADS, CPS::SMEM, s, pm, as, hp, 0);
          }
        }
        return launch_kernel(tc_chunkwise_pipe_kernel<DK, T, DVS, SEG_NONE, true, false, Tout>, grid, CfP::THREADS,
                             CfP::SMEM, s, pm, as, hp, 0);
      }
    }
    return run(tc_chunkwise_pipe_kernel<DK, T, DVS, SEG_NONE, false, false, Tout>, 1);
  }
  if (max_states < 1) return run(tc_chunkwise_pipe_kernel<DK, T, DVS, SEG_REPLAY, false, false, Tout>, as.n_seg);
  // Pre-pass: each of the first n_seg - 1 segments split into n_split sub-segments, as many
  // as the SMs, the workspace and two chunks a sub-segment allow.
  const int n_pre = as.n_seg - 1;
  int n_split = static_cast<int>(sms / (ctas * n_pre));
  n_split = std::min(n_split, max_states / n_pre);
  n_split = std::min(n_split, (as.seg_hi[0] - as.seg_lo[0]) / 2);
  n_split = std::max(n_split, 1);
  int j = 0;
  for (int sg = 0; sg < as.n_seg; ++sg) {
    as.sub_before[sg] = j;
    if (sg == n_pre) break;
    const int lo = as.seg_lo[sg], len = as.seg_hi[sg] - lo;
    for (int p = 0; p < n_split; ++p, ++j) {
      as.sub_lo[j] = lo + len * p / n_split;
      as.sub_hi[j] = lo + len * (p + 1) / n_split;
    }
  }
  as.n_sub = j;
  as.ws = static_cast<float*>(c.ws);
  using CfS = CfgS<DK, T, DVS>;
  auto kst = tc_segment_state_kernel<DK, T, DVS>;
  cudaError_t e = cudaFuncSetAttribute(kst, cudaFuncAttributeMaxDynamicSharedMemorySize, CfS::SMEM);
  if (e != cudaSuccess) return e;
  kst<<<dim3(grid.x * as.n_sub, grid.y, grid.z), CfS::THREADS, CfS::SMEM, s>>>(mk, mv, as, hp);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // Output pass, launched as a programmatic dependent of the pre-pass (segment-major grid):
  // its segment-0 CTAs run on the SMs the pre-pass leaves idle; later segments wait on the
  // device (griddepcontrol.wait) before they read the pre-pass states.
  auto kern = tc_chunkwise_pipe_kernel<DK, T, DVS, SEG_FROM_WS, false, false, Tout>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid.x, grid.y, grid.z * as.n_seg);
  cfg.blockDim = dim3(Cf::THREADS, 1, 1);
  cfg.dynamicSmemBytes = Cf::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, mq, mk, as, hp);
}

// Serial kernel: one chunk of B = T rows per step (chunk-relative scaled operands).
template <int DK, int T, typename Tout>
cudaError_t launch_serial(const RetentionCall& c, const HeadParams& hp, cudaStream_t s) {
  using Cf = Cfg<DK, T>;
  CUtensorMap mq, mk, mv;
  if (!make_maps(c, T, &mq, &mk, &mv)) return cudaErrorInvalidValue;
  const TcArgs a = make_args(c, static_cast<int>((c.dims.seqlen + T - 1) / T), 1);
  auto kern = tc_chunkwise_kernel<DK, T, Tout>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<tc_grid(c.dims, kDVS), kThreads, Cf::SMEM, s>>>(mq, mk, mv, a, hp);
  return cudaGetLastError();
}

template <int DK, typename Tout>
cudaError_t launch_dk(const RetentionCall& c, const HeadParams& hp, cudaStream_t s) {
  if (force_serial_kernel()) {
    if (c.chunk == 64) return launch_serial<DK, 64, Tout>(c, hp, s);
    return launch_serial<DK, 128, Tout>(c, hp, s);
  }
  if (c.precise) return launch_pipe_hl<DK, Tout>(c, hp, s);
  const int T = pipe_tile_rows(DK, c.chunk);
  if constexpr (DK != 256) {
    if (pipe_wide_slice(c, T)) return launch_pipe<DK, 64, 128, Tout>(c, hp, s);
  }
  if (T == 64) return launch_pipe<DK, 64, 64, Tout>(c, hp, s);
  if constexpr (DK != 256) return launch_pipe<DK, 128, 64, Tout>(c, hp, s);
  return cudaErrorInvalidValue;
}

template <typename Tout>
cudaError_t launch_out(const RetentionCall& c, const HeadParams& hp, cudaStream_t s) {
  switch (c.dims.d_k) {
    case 64: return launch_dk<64, Tout>(c, hp, s);
    case 128: return launch_dk<128, Tout>(c, hp, s);
    default: return launch_dk<256, Tout>(c, hp, s);
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace



bool tc_chunkwise_supported(const RetentionCall& c) {
  const Dims& d = c.dims;
  if (c.in_dtype != RETNET_BF16) return false;
  // R~ needs the row factors of the key-sum pass, in the caller's workspace
  if ((c.flags & RETNET_F_NORM_R) && (!c.rden || force_serial_kernel())) return false;
  if (d.d_k != 64 && d.d_k != 128 && d.d_k != 256) return false;
  if (d.d_v % kDVS != 0) return false;
  if (c.chunk != 64 && c.chunk != 128 && c.chunk != 256 && c.chunk != 512) return false;
  if (force_serial_kernel() && (c.chunk > 128 || c.precise || c.v_f16)) return false;
  // fp16 value rows: the pipelined kernel's converters only (no pre-pass, split operands or
  // fused epilogue), values of 64 or 128 columns a CTA
  if (c.v_f16 && (c.precise || c.gate || c.rden)) return false;
  // reversed output rows: the pipelined kernel's plain epilogue only
  if (c.o_rev && (c.gate || force_serial_kernel())) return false;
  if (d.seqlen < 1 || d.seqlen > (1LL << 30) || d.heads > 65535 || d.batch > 65535) return false;
  if (!aligned16(c.q) || !aligned16(c.k) || !aligned16(c.v) || !aligned16(c.o)) return false;
  if ((c.state_in && !aligned16(c.state_in)) || (c.state_out && !aligned16(c.state_out))) return false;
  if (c.state_in && c.state_out && c.state_in != c.state_out) {
    // distinct buffers are fine; overlapping but unequal ones are not supported here
    const char* a0 = reinterpret_cast<const char*>(c.state_in);
    const char* b0 = reinterpret_cast<const char*>(c.state_out);
    const size_t bytes = sizeof(float) * static_cast<size_t>(d.batch * d.heads * d.d_k * d.d_v);
    if (a0 < b0 + bytes && b0 < a0 + bytes) return false;
  }
  return true;
}

bool tc_fused_supported(const RetentionCall& c) {
  return tc_chunkwise_supported(c) && !force_serial_kernel() && c.dims.d_v % 64 == 0 &&
         c.dims.d_v / 64 <= kMaxCluster && aligned16(c.gate);
}

bool tc_driver_ready() { return encode_fn() != nullptr; }

// Host-side part of the scaled-operand condition: every head keeps gamma^T >= 2^-12, where T
// is the scaling span (the unit rows of the pipelined kernel, the whole chunk for the serial one).
bool tc_chunkwise_heads_ok(const RetentionCall& c, const HeadParams& hp) {
  const double span = force_serial_kernel() ? static_cast<double>(c.chunk) : pipe_tile_rows(c);
  for (int64_t h = 0; h < c.dims.heads; ++h)
    if (static_cast<double>(hp.log2g[h]) * span < -12.0) return false;
  return true;
}

cudaError_t tc_set_wait_budget(long long cycles) {
  const long long v = cycles > 0 ? cycles : sm100::kDrainBudget;
  return cudaMemcpyToSymbol(sm100::g_wait_budget, &v, sizeof(long long));
}

cudaError_t tc_fp16_overflows(unsigned int* count, bool clear) {
  cudaError_t e = cudaMemcpyFromSymbol(count, sm100::g_fp16_overflows, sizeof(unsigned int));
  if (e != cudaSuccess || !clear || *count == 0) return e;
  const unsigned int zero = 0;
  return cudaMemcpyToSymbol(sm100::g_fp16_overflows, &zero, sizeof(unsigned int));
}

cudaError_t tc_wait_timeouts(unsigned int* count, bool clear) {
  cudaError_t e = cudaMemcpyFromSymbol(count, sm100::g_wait_timeouts, sizeof(unsigned int));
  if (e != cudaSuccess || !clear || *count == 0) return e;
  const unsigned int zero = 0;
  return cudaMemcpyToSymbol(sm100::g_wait_timeouts, &zero, sizeof(unsigned int));
}

namespace {
template <int DK, int T, typename Tout>
cudaError_t launch_segment_state_t(const RetentionCall& c, const HeadParams& hp, cudaStream_t s) {
  using Cf = CfgS<DK, T, 64, true>;
  CUtensorMap mq, mk, mv;
  // The state pass never loads Q: its map is built over K (a valid tensor of the same shape).
  RetentionCall cc = c;
  cc.q = c.k;
  if (!make_maps(cc, T, &mq, &mk, &mv)) return cudaErrorInvalidValue;
  const int nb = static_cast<int>(c.chunk / T);
  const int n_chunks = static_cast<int>((c.dims.seqlen + c.chunk - 1) / c.chunk);
  TcArgs a = make_args(c, n_chunks, nb);
  a.n_seg = 1;
  a.n_sub = 1;
  a.sub_lo[0] = 0;
  a.sub_hi[0] = n_chunks;
  a.ws = c.state_out;  // sub-segment 0 of the workspace layout is [batch][heads][d_k][d_v]
  auto kern = tc_segment_state_kernel<DK, T, 64, true>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<tc_grid(c.dims, 64), Cf::THREADS, Cf::SMEM, s>>>(mk, mv, a, hp);
  return cudaGetLastError();
}

template <int DK>
cudaError_t launch_segment_state_dk(const RetentionCall& c, const HeadParams& hp, cudaStream_t s) {
  if (pipe_tile_rows(DK, c.chunk) == 64) return launch_segment_state_t<DK, 64, __nv_bfloat16>(c, hp, s);
  if constexpr (DK != 256) return launch_segment_state_t<DK, 128, __nv_bfloat16>(c, hp, s);
  return cudaErrorInvalidValue;
}

// state <- gamma_h^len * state + w over [batch][heads][d_k][d_v] (fp32, float4 per thread).
__global__ void state_advance_kernel(float4* __restrict__ state, const float4* __restrict__ w, int64_t n4,
                                     int64_t per_head4, int heads, HeadParams hp) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float f = hp.gamma[static_cast<int>((i / per_head4) % heads)];
    const float4 x = state[i], y = w[i];
    state[i] = make_float4(fmaf(f, x.x, y.x), fmaf(f, x.y, y.y), fmaf(f, x.z, y.z), fmaf(f, x.w, y.w));
  }
}
}  // namespace

cudaError_t launch_tc_segment_state(const RetentionCall& c, const HeadParams& hp, cudaStream_t s) {
  switch (c.dims.d_k) {
    case 64: return launch_segment_state_dk<64>(c, hp, s);
    case 128: return launch_segment_state_dk<128>(c, hp, s);
    default: return launch_segment_state_dk<256>(c, hp, s);
  }
}

// hp.gamma carries gamma_h^len per head here (computed on the host in fp64).
cudaError_t launch_state_advance(float* state, const float* w, const Dims& d, const HeadParams& hp, cudaStream_t s) {
  const int64_t n4 = d.batch * d.heads * d.d_k * d.d_v / 4;
  if (n4 == 0) return cudaSuccess;
  const int64_t per_head4 = d.d_k * d.d_v / 4;
  const int blocks = static_cast<int>(std::min<int64_t>((n4 + 255) / 256, 148 * 8));
  state_advance_kernel<<<blocks, 256, 0, s>>>(reinterpret_cast<float4*>(state), reinterpret_cast<const float4*>(w),
                                              n4, per_head4, static_cast<int>(d.heads), hp);
  return cudaGetLastError();
}

int tc_chunkwise_launches(const RetentionCall& c) {
  if (force_serial_kernel()) return 1;
  if (c.rden) {  // key-sum pass, then the kernels of the same call without R~
    RetentionCall cc = c;
    cc.rden = nullptr;
    cc.flags &= ~static_cast<uint32_t>(RETNET_F_NORM_R);
    return key_sum_launches(c.dims) + tc_chunkwise_launches(cc);
  }
  const int T = pipe_tile_rows(c);
  const int dvs = (!c.precise && pipe_wide_slice(c, T)) ? 128 : 64;
  const int nb = static_cast<int>(c.chunk / T);
  TcArgs as = make_args(c, static_cast<int>((c.dims.seqlen + c.chunk - 1) / c.chunk), nb);
  const int64_t ctas = (c.dims.d_v / dvs) * c.dims.heads * c.dims.batch;
  // fused epilogue and split operands: never segmented
  if (c.gate || c.precise) return pre_convert_applies(c, nb, 1) ? 2 : 1;
  const int max_states = plan_call(c, ctas, sm_count(), as);
  if (dvs == 64 && pre_convert_applies(c, nb, as.n_seg))  // conversion pre-pass (+ P pass) + kernel
    return p_pass_applies(c, T, nb, as.n_seg) ? 3 : 2;
  return (as.n_seg > 1 && max_states >= 1) ? 2 : 1;
}

cudaError_t launch_tc_chunkwise(const RetentionCall& c, const HeadParams& hp, cudaStream_t s) {
  if (c.rden) {
    cudaError_t e = launch_key_sum(c, hp, s);
    if (e != cudaSuccess) return e;
  }
  if (c.out_dtype == RETNET_F32) return launch_out<float>(c, hp, s);
  return launch_out<__nv_bfloat16>(c, hp, s);
}

}  // namespace retnet

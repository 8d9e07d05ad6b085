// retnet_abi.cu -- the extern "C" entry points of libretnet.so (declared in include/retnet.h).
//
// Each entry point checks its arguments on the host, fills the per-head parameter block
// (gamma, log2 gamma, theta) from the caller's host arrays, and enqueues the kernels on the
// caller's stream.  Nothing is allocated.  Device state that outlives a call: the count of
// bounded waits that gave up (read by retnet_debug_wait_timeouts) and the static scratch of
// retnet_retention_chunkwise_static (one array per device, below).
#include <math.h>

#include <algorithm>

#include "launch.h"

using namespace retnet;

namespace {

constexpr uint32_t kAllFlags =
    RETNET_F_XPOS | RETNET_F_SCALE_SQRT_D | RETNET_F_NORM_D | RETNET_F_NORM_R | RETNET_F_PRECISE;

bool valid_dtype(retnet_dtype_t t) { return t == RETNET_F32 || t == RETNET_BF16; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The current device must be an sm_100 part (B200); the kernels are built for sm_100a only.
retnet_status_t check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return RETNET_ERR_CUDA;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return RETNET_ERR_CUDA;
  if (major != 10 || minor != 0) return RETNET_ERR_UNSUPPORTED;
  return RETNET_OK;
}

// gamma in (0, 1) per head; theta finite per pair when XPOS is set.
retnet_status_t fill_params(HeadParams* hp, const float* gamma, const float* theta, int64_t heads, int64_t d_k,
                            uint32_t flags) {
  if (!gamma) return RETNET_ERR_NULL_PTR;
  if ((flags & RETNET_F_XPOS) && !theta) return RETNET_ERR_NULL_PTR;
  for (int64_t h = 0; h < heads; ++h) {
    const float g = gamma[h];
    if (!(g > 0.f && g < 1.f)) return RETNET_ERR_BAD_PARAM;
    hp->gamma[h] = g;
    hp->log2g[h] = static_cast<float>(log2(static_cast<double>(g)));
  }
  const int64_t pairs = d_k / 2;
  for (int64_t j = 0; j < pairs; ++j) {
    float t = (flags & RETNET_F_XPOS) ? theta[j] : 0.f;
    if (!isfinite(t)) return RETNET_ERR_BAD_PARAM;
    hp->theta[j] = t;
  }
  return RETNET_OK;
}

retnet_status_t check_common(const retnet_dims_t& d, retnet_dtype_t in_dtype, retnet_dtype_t out_dtype,
                             int64_t pos0, uint32_t flags, bool allow_zero_len) {
  if (!valid_dtype(in_dtype) || !valid_dtype(out_dtype)) return RETNET_ERR_BAD_DTYPE;
  if (d.batch <= 0 || d.heads <= 0 || d.d_k <= 0 || d.d_v <= 0) return RETNET_ERR_BAD_SHAPE;
  if (d.seqlen < 0 || (!allow_zero_len && d.seqlen == 0)) return RETNET_ERR_BAD_SHAPE;
  if (d.heads > RETNET_MAX_HEADS || d.d_k > RETNET_MAX_DK || d.d_v > RETNET_MAX_DV) return RETNET_ERR_BAD_SHAPE;
  if (d.batch > 65535 || d.heads > 65535) return RETNET_ERR_BAD_SHAPE;  // grid y/z limits
  if (flags & ~kAllFlags) return RETNET_ERR_BAD_PARAM;
  if ((flags & RETNET_F_XPOS) && (d.d_k & 1)) return RETNET_ERR_BAD_PARAM;
  if (pos0 < 0) return RETNET_ERR_BAD_PARAM;
  return RETNET_OK;
}

retnet_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? RETNET_OK : RETNET_ERR_CUDA; }

}  // namespace

extern "C" {

const char* retnet_status_string(retnet_status_t status) {
  switch (status) {
    case RETNET_OK: return "ok";
    case RETNET_ERR_NULL_PTR: return "a required pointer is NULL";
    case RETNET_ERR_BAD_SHAPE: return "bad shape (non-positive size or over a limit)";
    case RETNET_ERR_BAD_DTYPE: return "bad or unsupported dtype";
    case RETNET_ERR_BAD_PARAM: return "bad parameter (gamma, theta, chunk, eps, position, flags or alignment)";
    case RETNET_ERR_UNSUPPORTED: return "unsupported (device is not sm_100, or option needs a missing buffer)";
    case RETNET_ERR_CUDA: return "CUDA call or kernel launch failed";
  }
  return "unknown status";
}

int retnet_version(void) { return 100; }

retnet_status_t retnet_retention_parallel(const void* q, const void* k, const void* v, void* o, retnet_dims_t dims,
                                          retnet_dtype_t in_dtype, retnet_dtype_t out_dtype, const float* gamma,
                                          const float* theta, int64_t pos0, uint32_t flags, void* stream) {
  retnet_status_t st = check_common(dims, in_dtype, out_dtype, pos0, flags, true);
  if (st != RETNET_OK) return st;
  if (dims.seqlen > 0 && (!q || !k || !v || !o)) return RETNET_ERR_NULL_PTR;
  HeadParams hp;
  if ((st = fill_params(&hp, gamma, theta, dims.heads, dims.d_k, flags)) != RETNET_OK) return st;
  if (dims.seqlen == 0) return RETNET_OK;
  if ((st = check_device()) != RETNET_OK) return st;
  RetentionCall c{q, k, v, o, Dims{dims.batch, dims.seqlen, dims.heads, dims.d_k, dims.d_v}, in_dtype, out_dtype,
                  pos0, flags, dims.seqlen, false, nullptr, nullptr, nullptr, nullptr};
  // bf16 inputs without R~ (whose row sums need a workspace) run on the tensor-core kernel: a
  // sequence of up to 512 tokens is one chunk of the smallest size that holds it, i.e. the
  // masked B x B product of §2.3 itself (no state: every token's history is in the tile); a
  // longer one is cut into 512-token chunks, §2.4's re-association of the same sum.
  if (in_dtype == RETNET_BF16 && !(flags & RETNET_F_NORM_R)) {
    RetentionCall t = c;
    t.chunk = dims.seqlen <= 64 ? 64 : dims.seqlen <= 128 ? 128 : dims.seqlen <= 256 ? 256 : 512;
    t.has_state = true;  // (no state_in / state_out: a zero start, nothing written)
    t.precise = (flags & RETNET_F_PRECISE) != 0;
    if (tc_chunkwise_supported(t) && tc_chunkwise_heads_ok(t, hp)) {
      if (!tc_driver_ready()) return RETNET_ERR_CUDA;
      return from_cuda(launch_tc_chunkwise(t, hp, static_cast<cudaStream_t>(stream)));
    }
  }
  return from_cuda(launch_simt_retention(c, hp, static_cast<cudaStream_t>(stream)));
}

namespace {
// R~ on the tensor-core kernel: its row factors and the key-sum pass's segment values take
// the front of the workspace, the rest serves the segment states or the conversion copies as
// without R~.
void carve_rden(RetentionCall& c) {
  const size_t rb = rden_region_bytes(c.dims);
  if (!(c.flags & RETNET_F_NORM_R) || !c.ws || c.ws_bytes < rb || c.dims.seqlen == 0) return;
  c.rden = static_cast<float*>(c.ws);
  const size_t rows = (sizeof(float) * static_cast<size_t>(c.dims.batch * c.dims.seqlen * c.dims.heads) + 255) &
                      ~static_cast<size_t>(255);
  c.rden_seg = reinterpret_cast<float*>(static_cast<char*>(c.ws) + rows);
  c.ws = c.ws_bytes > rb ? static_cast<char*>(c.ws) + rb : nullptr;
  c.ws_bytes -= rb;
}
retnet_status_t chunkwise_impl(const void* q, const void* k, const void* v, void* o, retnet_dims_t dims,
                               retnet_dtype_t in_dtype, retnet_dtype_t out_dtype, const float* gamma,
                               const float* theta, int64_t pos0, uint32_t flags, int64_t chunk,
                               const float* state_in, float* state_out, const float* z_in, float* z_out,
                               void* workspace, size_t workspace_bytes, void* stream, const void* gate = nullptr,
                               float eps = 0.f);
retnet_status_t chunkwise_impl(const void* q, const void* k, const void* v, void* o, retnet_dims_t dims,
                               retnet_dtype_t in_dtype, retnet_dtype_t out_dtype, const float* gamma,
                               const float* theta, int64_t pos0, uint32_t flags, int64_t chunk,
                               const float* state_in, float* state_out, const float* z_in, float* z_out,
                               void* workspace, size_t workspace_bytes, void* stream, const void* gate,
                               float eps) {
  retnet_status_t st = check_common(dims, in_dtype, out_dtype, pos0, flags, true);
  if (st != RETNET_OK) return st;
  if (chunk <= 0) return RETNET_ERR_BAD_PARAM;
  if (dims.seqlen > 0 && (!q || !k || !v || !o)) return RETNET_ERR_NULL_PTR;
  if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 15u) != 0) return RETNET_ERR_BAD_PARAM;
  HeadParams hp;
  if ((st = fill_params(&hp, gamma, theta, dims.heads, dims.d_k, flags)) != RETNET_OK) return st;
  if ((st = check_device()) != RETNET_OK) return st;
  RetentionCall c{q, k, v, o, Dims{dims.batch, dims.seqlen, dims.heads, dims.d_k, dims.d_v}, in_dtype, out_dtype,
                  pos0, flags, chunk, true, state_in, state_out, z_in, z_out};
  c.ws = workspace;
  c.ws_bytes = workspace ? workspace_bytes : 0;
  carve_rden(c);
  c.precise = (flags & RETNET_F_PRECISE) || c.rden || gate;
  if (gate) {
    // Fused MSR epilogue: the tensor-core kernel only, decided on the host before any launch.
    c.gate = gate;
    c.eps = eps;
    if (dims.seqlen > 0 && !(tc_fused_supported(c) && tc_chunkwise_heads_ok(c, hp))) return RETNET_ERR_UNSUPPORTED;
  }
  if (dims.seqlen == 0) {
    // No tokens: the state passes through unchanged.
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t sbytes = sizeof(float) * (size_t)(dims.batch * dims.heads * dims.d_k * dims.d_v);
    const size_t zbytes = sizeof(float) * (size_t)(dims.batch * dims.heads * dims.d_k);
    if (state_out && state_out != state_in) {
      cudaError_t e = state_in ? cudaMemcpyAsync(state_out, state_in, sbytes, cudaMemcpyDeviceToDevice, s)
                               : cudaMemsetAsync(state_out, 0, sbytes, s);
      if (e != cudaSuccess) return RETNET_ERR_CUDA;
    }
    if ((flags & RETNET_F_NORM_R) && z_out && z_out != z_in) {
      cudaError_t e = z_in ? cudaMemcpyAsync(z_out, z_in, zbytes, cudaMemcpyDeviceToDevice, s)
                           : cudaMemsetAsync(z_out, 0, zbytes, s);
      if (e != cudaSuccess) return RETNET_ERR_CUDA;
    }
    return RETNET_OK;
  }
  if (tc_chunkwise_supported(c) && tc_chunkwise_heads_ok(c, hp)) {
    if (!tc_driver_ready()) return RETNET_ERR_CUDA;
    return from_cuda(launch_tc_chunkwise(c, hp, static_cast<cudaStream_t>(stream)));
  }
  return from_cuda(launch_simt_retention(c, hp, static_cast<cudaStream_t>(stream)));
}
}  // namespace

retnet_status_t retnet_retention_chunkwise(const void* q, const void* k, const void* v, void* o, retnet_dims_t dims,
                                           retnet_dtype_t in_dtype, retnet_dtype_t out_dtype, const float* gamma,
                                           const float* theta, int64_t pos0, uint32_t flags, int64_t chunk,
                                           const float* state_in, float* state_out, const float* z_in,
                                           float* z_out, void* stream) {
  return chunkwise_impl(q, k, v, o, dims, in_dtype, out_dtype, gamma, theta, pos0, flags, chunk, state_in, state_out,
                        z_in, z_out, nullptr, 0, stream);
}

retnet_status_t retnet_retention_chunkwise_ws(const void* q, const void* k, const void* v, void* o,
                                              retnet_dims_t dims, retnet_dtype_t in_dtype, retnet_dtype_t out_dtype,
                                              const float* gamma, const float* theta, int64_t pos0, uint32_t flags,
                                              int64_t chunk, const float* state_in, float* state_out,
                                              const float* z_in, float* z_out, void* workspace,
                                              size_t workspace_bytes, void* stream) {
  return chunkwise_impl(q, k, v, o, dims, in_dtype, out_dtype, gamma, theta, pos0, flags, chunk, state_in, state_out,
                        z_in, z_out, workspace, workspace_bytes, stream);
}

retnet_status_t retnet_msr_chunkwise(const void* q, const void* k, const void* v, const void* g, void* out,
                                     retnet_dims_t dims, retnet_dtype_t in_dtype, retnet_dtype_t out_dtype,
                                     const float* gamma, const float* theta, int64_t pos0, uint32_t flags,
                                     int64_t chunk, float eps, const float* state_in, float* state_out,
                                     void* workspace, size_t workspace_bytes, void* stream) {
  if (!(eps >= 0.f) || !isfinite(eps)) return RETNET_ERR_BAD_PARAM;
  if (dims.seqlen > 0 && !g) return RETNET_ERR_NULL_PTR;
  // (without tokens nothing reads g: the call only passes the state through)
  // R~ needs its row factors in the workspace (a too small one is caught before the launch)
  if ((flags & RETNET_F_NORM_R) && dims.seqlen > 0 && !workspace) return RETNET_ERR_UNSUPPORTED;
  return chunkwise_impl(q, k, v, out, dims, in_dtype, out_dtype, gamma, theta, pos0, flags, chunk, state_in,
                        state_out, nullptr, nullptr, workspace, workspace_bytes, stream, g, eps);
}

// ---- allocation-free variant ---------------------------------------------------------------
// Segment states of the two-pass form in a file-scope device array instead of a caller's
// workspace: for callers that cannot allocate device memory -- hosts that link only this C
// library and have no device allocator of their own, and code that must not allocate on its
// hot path because cudaMalloc / cudaFree synchronise the device.  The array exists once per
// device (per context); nothing in it needs to start at zero (each call overwrites the states
// it reads).  Calls that overlap on the GPU share it and race.
static __device__ __align__(256) unsigned char g_chunkwise_scratch[RETNET_STATIC_SCRATCH_BYTES];

namespace {
// Device address of the scratch in the current device's context.  Host code cannot use the
// array's name as a device address, so every call asks the runtime (cudaGetSymbolAddress, a
// host-side query, with the calling thread's device current); nothing is cached, so a device
// reset or a recreated context never leaves a stale address behind.
retnet_status_t static_scratch(void** ptr) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_chunkwise_scratch) != cudaSuccess || !p) return RETNET_ERR_CUDA;
  *ptr = p;
  return RETNET_OK;
}
}  // namespace

retnet_status_t retnet_retention_chunkwise_static(const void* q, const void* k, const void* v, void* o,
                                                  retnet_dims_t dims, retnet_dtype_t in_dtype,
                                                  retnet_dtype_t out_dtype, const float* gamma, const float* theta,
                                                  int64_t pos0, uint32_t flags, int64_t chunk,
                                                  const float* state_in, float* state_out, const float* z_in,
                                                  float* z_out, void* stream) {
  if (dims.batch >= 0 && dims.heads >= 0 && dims.d_k >= 0 && dims.d_v >= 0) {
    // One segment state must fit the static scratch; larger calls are rejected, not degraded.
    const double state_bytes = 4.0 * static_cast<double>(dims.batch) * static_cast<double>(dims.heads) *
                               static_cast<double>(dims.d_k) * static_cast<double>(dims.d_v);
    if (state_bytes > static_cast<double>(RETNET_STATIC_SCRATCH_BYTES)) return RETNET_ERR_UNSUPPORTED;
  }
  void* scratch = nullptr;
  const retnet_status_t st = static_scratch(&scratch);
  if (st != RETNET_OK) return st;
  return chunkwise_impl(q, k, v, o, dims, in_dtype, out_dtype, gamma, theta, pos0, flags, chunk, state_in,
                        state_out, z_in, z_out, scratch, RETNET_STATIC_SCRATCH_BYTES, stream);
}

retnet_status_t retnet_chunkwise_workspace_size(retnet_dims_t dims, size_t* bytes) {
  if (!bytes) return RETNET_ERR_NULL_PTR;
  if (dims.batch < 0 || dims.seqlen < 0 || dims.heads < 0 || dims.d_k < 0 || dims.d_v < 0) return RETNET_ERR_BAD_SHAPE;
  // The larger of its two uses (never both in one call): up to six segment states, fp32
  // [6][batch][heads][d_k][d_v]; or the fp16 copies of q, k, v of the conversion pre-pass, with
  // the lo parts of q and k for split operands.
  const size_t states = 6 * sizeof(float) * static_cast<size_t>(dims.batch) * static_cast<size_t>(dims.heads) *
                        static_cast<size_t>(dims.d_k) * static_cast<size_t>(dims.d_v);
  const size_t tok = static_cast<size_t>(dims.batch) * static_cast<size_t>(dims.seqlen) * static_cast<size_t>(dims.heads);
  auto a256 = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  const size_t copies = 4 * a256(tok * static_cast<size_t>(dims.d_k) * 2) + a256(tok * static_cast<size_t>(dims.d_v) * 2);
  // with d_k = 256 the P pass's tiles after the single-operand copies, at most (chunks of 512)
  // ceil(seqlen / 512) * 36 tiles of 64 x 64 fp16 per (batch, head)
  const size_t ptiles = dims.d_k == 256 ? a256(static_cast<size_t>(dims.batch) * static_cast<size_t>(dims.heads) *
                                                static_cast<size_t>((dims.seqlen + 511) / 512) * 36 * 64 * 64 * 2)
                                        : 0;
  const size_t single = 2 * a256(tok * static_cast<size_t>(dims.d_k) * 2) + a256(tok * static_cast<size_t>(dims.d_v) * 2);
  const size_t copies_all = copies > single + ptiles ? copies : single + ptiles;
  // plus, in front, the R~ row factors (fp32 [batch][seqlen][heads]) and the key-sum pass's
  // segment values (fp32 [batch * heads][64][d_k])
  const Dims d{dims.batch, dims.seqlen, dims.heads, dims.d_k, dims.d_v};
  *bytes = rden_region_bytes(d) + (states > copies_all ? states : copies_all);
  return RETNET_OK;
}

retnet_status_t retnet_chunkwise_segment_state(const void* k, const void* v, retnet_dims_t dims,
                                               retnet_dtype_t in_dtype, const float* gamma, const float* theta,
                                               int64_t pos0, uint32_t flags, int64_t chunk, float* state_out,
                                               void* stream) {
  retnet_status_t st = check_common(dims, in_dtype, RETNET_F32, pos0, flags, true);
  if (st != RETNET_OK) return st;
  if (chunk <= 0) return RETNET_ERR_BAD_PARAM;
  if (!state_out) return RETNET_ERR_NULL_PTR;
  if (dims.seqlen > 0 && (!k || !v)) return RETNET_ERR_NULL_PTR;
  HeadParams hp;
  if ((st = fill_params(&hp, gamma, theta, dims.heads, dims.d_k, flags)) != RETNET_OK) return st;
  if ((st = check_device()) != RETNET_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dims.seqlen == 0) {
    const size_t sbytes = sizeof(float) * static_cast<size_t>(dims.batch * dims.heads * dims.d_k * dims.d_v);
    return cudaMemsetAsync(state_out, 0, sbytes, s) == cudaSuccess ? RETNET_OK : RETNET_ERR_CUDA;
  }
  // q is not read; k stands in for it so that the shape checks see three valid tensors.
  RetentionCall c{k, k, v, state_out, Dims{dims.batch, dims.seqlen, dims.heads, dims.d_k, dims.d_v}, in_dtype,
                  RETNET_F32, pos0, flags, chunk, true, nullptr, state_out, nullptr, nullptr};
  if (!tc_chunkwise_supported(c) || !tc_chunkwise_heads_ok(c, hp)) return RETNET_ERR_UNSUPPORTED;
  if (!tc_driver_ready()) return RETNET_ERR_CUDA;
  return from_cuda(launch_tc_segment_state(c, hp, s));
}

retnet_status_t retnet_state_advance(float* state, const float* w, int64_t batch, int64_t heads, int64_t d_k,
                                     int64_t d_v, const float* gamma, int64_t len, void* stream) {
  if (!state || !w || !gamma) return RETNET_ERR_NULL_PTR;
  if (batch < 0 || heads <= 0 || d_k <= 0 || d_v <= 0 || heads > RETNET_MAX_HEADS) return RETNET_ERR_BAD_SHAPE;
  if ((d_k * d_v) % 4 != 0) return RETNET_ERR_BAD_SHAPE;
  if (len < 0) return RETNET_ERR_BAD_PARAM;
  if ((reinterpret_cast<uintptr_t>(state) & 15u) || (reinterpret_cast<uintptr_t>(w) & 15u)) return RETNET_ERR_BAD_PARAM;
  HeadParams hp;
  for (int64_t h = 0; h < heads; ++h) {
    const double g = gamma[h];
    if (!(g > 0.0 && g < 1.0)) return RETNET_ERR_BAD_PARAM;
    hp.gamma[h] = static_cast<float>(exp(static_cast<double>(len) * log(g)));  // gamma^len in fp64
  }
  retnet_status_t st = check_device();
  if (st != RETNET_OK) return st;
  return from_cuda(launch_state_advance(state, w, Dims{batch, 0, heads, d_k, d_v}, hp, static_cast<cudaStream_t>(stream)));
}

int retnet_chunkwise_launches(retnet_dims_t dims, retnet_dtype_t in_dtype, uint32_t flags, int64_t chunk,
                              const float* gamma, size_t workspace_bytes) {
  // the kernel choice without R~ (R~ itself needs the workspace, below)
  const int path = retnet_chunkwise_kernel(dims, in_dtype, flags & ~static_cast<uint32_t>(RETNET_F_NORM_R), chunk,
                                           gamma);
  if (path < 0) return path;
  if (dims.seqlen == 0) return 0;
  if (path == 0) return 1;
  const retnet_status_t st = check_device();
  if (st != RETNET_OK) return -static_cast<int>(st);
  alignas(16) static const uint32_t kAligned[4] = {0, 0, 0, 0};
  RetentionCall c{kAligned, kAligned, kAligned, const_cast<uint32_t*>(kAligned),
                  Dims{dims.batch, dims.seqlen, dims.heads, dims.d_k, dims.d_v}, in_dtype, RETNET_BF16, 0, flags,
                  chunk, true, nullptr, nullptr, nullptr, nullptr};
  c.ws = workspace_bytes ? reinterpret_cast<void*>(static_cast<uintptr_t>(256)) : nullptr;  // only its size matters
  c.ws_bytes = workspace_bytes;
  carve_rden(c);
  c.precise = (flags & RETNET_F_PRECISE) || c.rden;
  if (!tc_chunkwise_supported(c)) return 1;  // R~ without room for its factors: the CUDA-core kernel
  return tc_chunkwise_launches(c);
}

int retnet_msr_chunkwise_launches(retnet_dims_t dims, retnet_dtype_t in_dtype, uint32_t flags, int64_t chunk,
                                  const float* gamma, size_t workspace_bytes) {
  const int path = retnet_chunkwise_kernel(dims, in_dtype, flags & ~static_cast<uint32_t>(RETNET_F_NORM_R), chunk,
                                           gamma);
  if (path < 0) return path;
  if (dims.seqlen == 0) return 0;
  if (path == 0) return -static_cast<int>(RETNET_ERR_UNSUPPORTED);
  const Dims dd{dims.batch, dims.seqlen, dims.heads, dims.d_k, dims.d_v};
  if ((flags & RETNET_F_NORM_R) && workspace_bytes < rden_region_bytes(dd)) return -static_cast<int>(RETNET_ERR_UNSUPPORTED);
  const retnet_status_t st = check_device();
  if (st != RETNET_OK) return -static_cast<int>(st);
  alignas(16) static const uint32_t kAligned[4] = {0, 0, 0, 0};
  RetentionCall c{kAligned, kAligned, kAligned, const_cast<uint32_t*>(kAligned),
                  Dims{dims.batch, dims.seqlen, dims.heads, dims.d_k, dims.d_v}, in_dtype, RETNET_BF16, 0, flags,
                  chunk, true, nullptr, nullptr, nullptr, nullptr};
  c.ws = workspace_bytes ? reinterpret_cast<void*>(static_cast<uintptr_t>(256)) : nullptr;  // only its size matters
  c.ws_bytes = workspace_bytes;
  carve_rden(c);
  c.gate = kAligned;
  c.precise = true;
  if (!tc_fused_supported(c)) return -static_cast<int>(RETNET_ERR_UNSUPPORTED);
  return tc_chunkwise_launches(c);
}

int retnet_chunkwise_kernel(retnet_dims_t dims, retnet_dtype_t in_dtype, uint32_t flags, int64_t chunk,
                            const float* gamma) {
  retnet_status_t st = check_common(dims, in_dtype, RETNET_F32, 0, flags, true);
  if (st != RETNET_OK) return -static_cast<int>(st);
  if (chunk <= 0) return -static_cast<int>(RETNET_ERR_BAD_PARAM);
  HeadParams hp;
  // theta is not read without XPOS, and its values do not affect the choice of kernel.
  st = fill_params(&hp, gamma, nullptr, dims.heads, dims.d_k, flags & ~static_cast<uint32_t>(RETNET_F_XPOS));
  if (st != RETNET_OK) return -static_cast<int>(st);
  alignas(16) static const uint32_t kAligned[4] = {0, 0, 0, 0};
  RetentionCall c{kAligned, kAligned, kAligned, const_cast<uint32_t*>(kAligned),
                  Dims{dims.batch, dims.seqlen, dims.heads, dims.d_k, dims.d_v}, in_dtype, RETNET_F32, 0, flags,
                  chunk, true, nullptr, nullptr, nullptr, nullptr};
  c.precise = (flags & (RETNET_F_PRECISE | RETNET_F_NORM_R)) != 0;
  return (tc_chunkwise_supported(c) && tc_chunkwise_heads_ok(c, hp)) ? 1 : 0;
}

retnet_status_t retnet_debug_wait_timeouts(unsigned int* count, int clear) {
  if (!count) return RETNET_ERR_NULL_PTR;
  if (cudaDeviceSynchronize() != cudaSuccess) return RETNET_ERR_CUDA;
  return from_cuda(tc_wait_timeouts(count, clear != 0));
}

retnet_status_t retnet_debug_set_wait_budget(long long cycles) {
  if (cycles > 0 && cycles < 100) return RETNET_ERR_BAD_PARAM;
  if (cudaDeviceSynchronize() != cudaSuccess) return RETNET_ERR_CUDA;
  return from_cuda(tc_set_wait_budget(cycles));
}

retnet_status_t retnet_fp16_range_errors(unsigned int* count, int clear) {
  if (!count) return RETNET_ERR_NULL_PTR;
  if (cudaDeviceSynchronize() != cudaSuccess) return RETNET_ERR_CUDA;
  unsigned int bwd = 0;
  const retnet_status_t st = from_cuda(tc_fp16_overflows(count, clear != 0));
  if (st != RETNET_OK) return st;
  const retnet_status_t sb = from_cuda(bwd_fp16_overflows(&bwd, clear != 0));
  *count += bwd;
  return sb;
}

retnet_status_t retnet_retention_step(const void* q, const void* k, const void* v, void* o, int64_t batch,
                                      int64_t heads, int64_t d_k, int64_t d_v, retnet_dtype_t in_dtype,
                                      retnet_dtype_t out_dtype, float* state, float* z, const float* gamma,
                                      const float* theta, int64_t pos, uint32_t flags, void* stream) {
  retnet_dims_t d{batch, 1, heads, d_k, d_v};
  retnet_status_t st = check_common(d, in_dtype, out_dtype, pos, flags, false);
  if (st != RETNET_OK) return st;
  if (batch * heads > 0x7fffffffLL) return RETNET_ERR_BAD_SHAPE;
  if (!q || !k || !v || !o || !state) return RETNET_ERR_NULL_PTR;
  if ((flags & RETNET_F_NORM_R) && !z) return RETNET_ERR_UNSUPPORTED;
  if (!aligned16(state)) return RETNET_ERR_BAD_PARAM;
  HeadParams hp;
  if ((st = fill_params(&hp, gamma, theta, heads, d_k, flags)) != RETNET_OK) return st;
  if ((st = check_device()) != RETNET_OK) return st;
  StepCall c{q, k, v, o, batch, heads, d_k, d_v, in_dtype, out_dtype, state, z, pos, flags};
  return from_cuda(launch_step(c, hp, static_cast<cudaStream_t>(stream)));
}

retnet_status_t retnet_backward_workspace_size(retnet_dims_t dims, size_t* bytes) {
  if (!bytes) return RETNET_ERR_NULL_PTR;
  if (dims.batch < 0 || dims.seqlen < 0 || dims.heads < 0 || dims.d_k < 0 || dims.d_v < 0) return RETNET_ERR_BAD_SHAPE;
  const Dims d{dims.batch, dims.seqlen, dims.heads, dims.d_k, dims.d_v};
  *bytes = std::max(backward_workspace_bytes(d), backward_tc_workspace_bytes(d));
  return RETNET_OK;
}

int retnet_backward_kernel(retnet_dims_t dims, retnet_dtype_t in_dtype, uint32_t flags, const float* gamma,
                           size_t workspace_bytes) {
  retnet_status_t st = check_common(dims, in_dtype, RETNET_F32, 0, flags, true);
  if (st != RETNET_OK) return -static_cast<int>(st);
  if (flags & RETNET_F_NORM_R) return -static_cast<int>(RETNET_ERR_UNSUPPORTED);
  HeadParams hp;
  st = fill_params(&hp, gamma, nullptr, dims.heads, dims.d_k, flags & ~static_cast<uint32_t>(RETNET_F_XPOS));
  if (st != RETNET_OK) return -static_cast<int>(st);
  alignas(16) static const uint32_t kAligned[4] = {0, 0, 0, 0};
  float* fake = const_cast<float*>(reinterpret_cast<const float*>(kAligned));
  BackwardCall c{kAligned, kAligned, kAligned, kAligned, fake, fake, fake,
                 Dims{dims.batch, dims.seqlen, dims.heads, dims.d_k, dims.d_v}, in_dtype, 0, flags, nullptr, nullptr,
                 reinterpret_cast<void*>(static_cast<uintptr_t>(256)), workspace_bytes};
  return backward_tc_applies(c, hp) ? 1 : 0;
}

int retnet_backward_launches(retnet_dims_t dims, retnet_dtype_t in_dtype, uint32_t flags, const float* gamma,
                             size_t workspace_bytes, int with_state, int with_dstate) {
  const int path = retnet_backward_kernel(dims, in_dtype, flags, gamma, workspace_bytes);
  if (path < 0) return path;
  if (dims.seqlen == 0) return with_dstate ? 1 : 0;  // a memset (no kernel of ours)
  if (path == 0) return with_dstate ? 4 : 3;
  const retnet_status_t st = check_device();
  if (st != RETNET_OK) return -static_cast<int>(st);
  HeadParams hp;
  fill_params(&hp, gamma, nullptr, dims.heads, dims.d_k, flags & ~static_cast<uint32_t>(RETNET_F_XPOS));
  alignas(16) static const uint32_t kAligned[4] = {0, 0, 0, 0};
  float* fake = const_cast<float*>(reinterpret_cast<const float*>(kAligned));
  BackwardCall c{kAligned, kAligned, kAligned, kAligned, fake, fake, fake,
                 Dims{dims.batch, dims.seqlen, dims.heads, dims.d_k, dims.d_v}, in_dtype, 0, flags,
                 with_state ? fake : nullptr, with_dstate ? fake : nullptr,
                 reinterpret_cast<void*>(static_cast<uintptr_t>(256)), workspace_bytes};
  return backward_tc_launches(c);
}

retnet_status_t retnet_retention_backward(const void* q, const void* k, const void* v, const void* dout, float* dq,
                                          float* dk, float* dv, retnet_dims_t dims, retnet_dtype_t in_dtype,
                                          const float* gamma, const float* theta, int64_t pos0, uint32_t flags,
                                          const float* state_in, float* dstate, void* workspace,
                                          size_t workspace_bytes, void* stream) {
  retnet_status_t st = check_common(dims, in_dtype, RETNET_F32, pos0, flags, true);
  if (st != RETNET_OK) return st;
  if (flags & RETNET_F_NORM_R) return RETNET_ERR_UNSUPPORTED;
  const Dims d{dims.batch, dims.seqlen, dims.heads, dims.d_k, dims.d_v};
  if (!backward_supported(d) || (dims.seqlen + 7) / 8 > 65535 || dims.batch * dims.heads > 0x7fffffffLL)
    return RETNET_ERR_UNSUPPORTED;
  if (dims.seqlen == 0) {
    if (dstate) {
      const size_t sb = sizeof(float) * static_cast<size_t>(dims.batch * dims.heads * dims.d_k * dims.d_v);
      if (cudaMemsetAsync(dstate, 0, sb, static_cast<cudaStream_t>(stream)) != cudaSuccess) return RETNET_ERR_CUDA;
    }
    return RETNET_OK;
  }
  if (!q || !k || !v || !dout || !dq || !dk || !dv || !workspace) return RETNET_ERR_NULL_PTR;
  if (workspace_bytes < backward_workspace_bytes(d) || !aligned16(workspace)) return RETNET_ERR_BAD_PARAM;
  HeadParams hp;
  if ((st = fill_params(&hp, gamma, theta, dims.heads, dims.d_k, flags)) != RETNET_OK) return st;
  if ((st = check_device()) != RETNET_OK) return st;
  BackwardCall c{q, k, v, dout, dq, dk, dv, d, in_dtype, pos0, flags, state_in, dstate, workspace, workspace_bytes};
  return from_cuda(launch_backward(c, hp, static_cast<cudaStream_t>(stream)));
}

retnet_status_t retnet_msr_epilogue(const void* y, const void* g, void* out, int64_t tokens, int64_t heads,
                                    int64_t d_v, float eps, retnet_dtype_t in_dtype, retnet_dtype_t out_dtype,
                                    void* stream) {
  if (!valid_dtype(in_dtype) || !valid_dtype(out_dtype)) return RETNET_ERR_BAD_DTYPE;
  if (tokens < 0 || heads <= 0 || d_v <= 0 || d_v > RETNET_MAX_DV || (d_v % 8) != 0) return RETNET_ERR_BAD_SHAPE;
  if (!(eps >= 0.f) || !isfinite(eps)) return RETNET_ERR_BAD_PARAM;
  if (!y || !g || !out) return RETNET_ERR_NULL_PTR;
  if (!aligned16(y) || !aligned16(g) || !aligned16(out)) return RETNET_ERR_BAD_PARAM;
  if ((tokens * heads + 7) / 8 > 0x7fffffffLL) return RETNET_ERR_BAD_SHAPE;
  if (tokens == 0) return RETNET_OK;
  retnet_status_t st = check_device();
  if (st != RETNET_OK) return st;
  return from_cuda(launch_msr_epilogue(y, g, out, tokens, heads, d_v, eps, in_dtype, out_dtype,
                                       static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

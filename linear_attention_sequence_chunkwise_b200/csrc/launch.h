// launch.h -- host-side launchers behind the C interface (internal to libretnet.so).
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"

namespace retnet {

// Arguments of one chunkwise / parallel retention call, after host validation.
struct RetentionCall {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  Dims dims;
  retnet_dtype_t in_dtype, out_dtype;
  int64_t pos0;
  uint32_t flags;
  int64_t chunk;  // == seqlen (or more) for the parallel form
  bool has_state;  // false for the parallel form: no state is read or written
  const float* state_in;
  float* state_out;
  const float* z_in;
  float* z_out;
  // Caller-owned device workspace for the two-pass sequence segments of the tensor-core
  // kernel (segment states); nullptr = single-launch segments that replay the state.
  void* ws = nullptr;
  size_t ws_bytes = 0;
  // Fused MSR epilogue (tensor-core kernel): o <- GroupNorm_h(o) * swish(gate), gate laid out
  // as o; nullptr = plain retention output.
  const void* gate = nullptr;
  float eps = 0.f;
  // R~ normalisation on the tensor-core kernel: per-row factor 1 / max(|sum of scores|, 1),
  // fp32 [batch][seqlen][heads], written by launch_key_sum (caller's workspace); nullptr = none.
  // rden_seg: the key-sum pass's segment end values, fp32 [batch * heads][<= 64][d_k].
  float* rden = nullptr;
  float* rden_seg = nullptr;
  // Split fp16 operands (hi + lo) on the tensor-core kernel: RETNET_F_PRECISE, R~ and the fused
  // MSR epilogue, whose normalisations magnify the operand rounding of a single fp16 copy.
  bool precise = false;
  // Value rows already in fp16 (in_dtype still describes q and k): the gradient's runs, whose
  // values are not bf16 numbers.  The pipelined kernel's converters leave V as it is.
  bool v_f16 = false;
  // Output row of token t written at token L - 1 - t (internal: the gradient's dv run, whose
  // sequence is reversed, writes dv in forward order).
  bool o_rev = false;
};

// Sequence segments of the key-sum pass, at most; and the workspace bytes of the R~ factors
// plus those segment values (each part rounded up to 256 bytes).
constexpr int kMaxKeySumSegments = 64;
inline size_t rden_region_bytes(const Dims& d) {
  auto a256 = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  return a256(sizeof(float) * static_cast<size_t>(d.batch * d.seqlen * d.heads)) +
         a256(sizeof(float) * static_cast<size_t>(d.batch * d.heads * d.d_k) * kMaxKeySumSegments);
}

// fp32 CUDA-core kernel: the parallel form (chunk >= seqlen, no state) and the chunkwise
// form for any shape.
cudaError_t launch_simt_retention(const RetentionCall& c, const HeadParams& hp, cudaStream_t s);

// tcgen05 tensor-core chunkwise kernel for bf16 inputs; `supported` says whether the shape
// and buffers are ones it handles, `heads_ok` whether every head keeps gamma^chunk >= 2^-12.
bool tc_chunkwise_supported(const RetentionCall& c);
bool tc_chunkwise_heads_ok(const RetentionCall& c, const HeadParams& hp);
// The tensor-core kernel with the MSR epilogue fused (c.gate set) handles this call: a
// tensor-core shape with d_v a multiple of 64 and at most 256, gate 16-byte aligned.
bool tc_fused_supported(const RetentionCall& c);
// The driver entry point that encodes TMA tensor maps could be resolved.
bool tc_driver_ready();
cudaError_t launch_tc_chunkwise(const RetentionCall& c, const HeadParams& hp, cudaStream_t s);
// Kernel launches launch_tc_chunkwise makes for this call on the current device (1 or 2).
int tc_chunkwise_launches(const RetentionCall& c);
// The state a sequence's chunks leave behind from a zero start, into c.state_out (tensor-core
// shapes only; q is not read).
cudaError_t launch_tc_segment_state(const RetentionCall& c, const HeadParams& hp, cudaStream_t s);
// state <- g_h * state + w, g_h = hp.gamma[h] (fp32 [batch][heads][d_k][d_v], d_k*d_v % 4 == 0).
cudaError_t launch_state_advance(float* state, const float* w, const Dims& d, const HeadParams& hp, cudaStream_t s);
// The R~ row factors of a chunkwise call into c.rden (and z_out from z_in): bf16 q, k, d_k in
// [64, 256], one pass over the keys.
cudaError_t launch_key_sum(const RetentionCall& c, const HeadParams& hp, cudaStream_t s);
// Kernel launches of launch_key_sum (1, or 2 when the sequence is cut into segments).
int key_sum_launches(const Dims& d);
// Reads (and optionally clears) the count of bounded waits that gave up in the tensor-core kernel.
cudaError_t tc_wait_timeouts(unsigned int* count, bool clear);
// Sets the pipeline-wait budget of the tensor-core kernels (SM cycles; <= 0 restores the default).
cudaError_t tc_set_wait_budget(long long cycles);
// Reads (and optionally clears) the count of threads that rounded a tensor-core operand outside
// the fp16 range.
cudaError_t tc_fp16_overflows(unsigned int* count, bool clear);
cudaError_t bwd_fp16_overflows(unsigned int* count, bool clear);  // the gradient's fp16 value rows

struct StepCall {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  int64_t batch, heads, d_k, d_v;
  retnet_dtype_t in_dtype, out_dtype;
  float* state;
  float* z;
  int64_t pos;
  uint32_t flags;
};
cudaError_t launch_step(const StepCall& c, const HeadParams& hp, cudaStream_t s);

// Gradient of the retention forward (dq, dk, dv, d state) on fp32 CUDA cores.
struct BackwardCall {
  const void* q;
  const void* k;
  const void* v;
  const void* dout;
  float* dq;
  float* dk;
  float* dv;
  Dims dims;
  retnet_dtype_t in_dtype;
  int64_t pos0;
  uint32_t flags;
  const float* state_in;  // S0 before the first token (or nullptr)
  float* dstate;          // gradient of S0 (or nullptr)
  void* ws;               // workspace (see backward_workspace_bytes)
  size_t ws_bytes;
};
// Bytes the CUDA-core path needs (rotated q and k in fp32); the tensor-core path needs
// backward_tc_workspace_bytes (more; it is taken when the workspace has it).
size_t backward_workspace_bytes(const Dims& d);
size_t backward_tc_workspace_bytes(const Dims& d);
bool backward_supported(const Dims& d);
// The tensor-core path (three runs of the chunkwise kernel) handles this call: bf16 inputs,
// d_k and d_v in {64, 128, 256}, room in the workspace, every run supported by the kernel.
bool backward_tc_applies(const BackwardCall& c, const HeadParams& hp);
int backward_tc_launches(const BackwardCall& c);
cudaError_t launch_backward_tc(const BackwardCall& c, const HeadParams& hp, cudaStream_t s);
cudaError_t launch_backward(const BackwardCall& c, const HeadParams& hp, cudaStream_t s);

cudaError_t launch_msr_epilogue(const void* y, const void* g, void* out, int64_t tokens, int64_t heads,
                                int64_t d_v, float eps, retnet_dtype_t in_dtype, retnet_dtype_t out_dtype,
                                cudaStream_t s);

}  // namespace retnet

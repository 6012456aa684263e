// launch.h -- host-side launchers of the library's kernels (internal).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace mixllm {

cudaError_t launch_quantize_act(const void *X, int64_t M, int64_t K, int8_t *A_q, float *s_a,
                                cudaStream_t stream);

cudaError_t launch_split_channels(const uint8_t *is8, int64_t N, int64_t N8, int32_t *idx4, int32_t *idx8,
                                  cudaStream_t stream);

cudaError_t launch_pack_w4(const float *W, int64_t N, int64_t K, const int32_t *idx4, int64_t N4, int64_t N4p,
                           uint8_t *W4, uint8_t *z4, void *s_w4, cudaStream_t stream);

cudaError_t launch_pack_w8(const float *W, int64_t N, int64_t K, const int32_t *idx8, int64_t N8, int64_t N8p,
                           int8_t *W8, void *s_w8, cudaStream_t stream);

struct GemmArgs {
  const int8_t *A_q;
  const float *s_a;
  int64_t M, K;
  const uint8_t *W4;
  const uint8_t *z4;
  const void *s_w4;
  const int32_t *idx4;
  int64_t N4;
  const int8_t *W8;
  const void *s_w8;
  const int32_t *idx8;
  int64_t N8;
  void *Y;     // fp16 [M, N4 + N8]
  int32_t *P;  // debug partials [M, N, G] or null
  const void *X = nullptr;  // fp16 [M, K] activations: the fused few-token path quantizes them itself
  bool cvt_i2f = false;     // tiled GEMM only: plain int -> float convert instead of the bias trick (measurement)
  uint32_t *qcnt = nullptr; // fused tiled layer: two counters in the workspace (pairs quantized, CTAs done)
};

// Returns a CUDA error, or cudaErrorNotSupported when the tensor-map encoder
// is unavailable.  *msg receives a static description on failure.
cudaError_t launch_gemm_w4w8a8(const GemmArgs &a, cudaStream_t stream, const char **msg);

// The tiled layer from fp16 X (M > 64) into a.A_q / a.s_a (workspace): the
// quantizer, then the GEMM; or (one_launch) the GEMM quantizing the
// activations itself and publishing them through a.qcnt (two counters, zero
// before the call and again after it; cudaErrorNotSupported for shapes that
// form does not take).
bool linear_tiled_fuses(int64_t M, int64_t K);
cudaError_t launch_linear_tiled(const GemmArgs &a, bool one_launch, cudaStream_t stream, const char **msg);
// Any M: the few-token layer (launch_linear_small_m) for M <= 64, else the
// tiled one, each with its workspace layout (linear_workspace_bytes()).
size_t linear_workspace_bytes(int64_t M, int64_t N4, int64_t N8, int64_t K);
cudaError_t launch_linear(const GemmArgs &a, void *ws, size_t ws_bytes, bool one_launch, cudaStream_t stream,
                          const char **msg);

// Few-token variant (M <= 64): split-K over the groups with a workspace of
// small_m_workspace_bytes() bytes: fp32 partial sums, then one int32 counter
// per tile (zero before the first call; every call returns them to zero).
// Y only (the debug partials: launch_small_m_debug_partials).
cudaError_t launch_gemm_small_m(const GemmArgs &a, void *ws, size_t ws_bytes, cudaStream_t stream, const char **msg);
size_t small_m_workspace_bytes(int64_t M, int64_t N4, int64_t N8, int64_t K);
// 0: tensor-core kernel, 1: split GEMV, 2: persistent GEMV (mixllm_small_m_kind)
int small_m_kernel_kind(int64_t M, int64_t N4, int64_t N8, int64_t K);
// Debug form of one named few-token kernel (kind as above, whatever the plan
// would pick): Y, and the int32 group partials into a.P [M, N, G].
bool small_m_kernel_allowed(int64_t M, int64_t N4, int64_t N8, int64_t K, int kind);
size_t small_m_debug_workspace_bytes(int64_t M, int64_t N4, int64_t N8, int64_t K, int kind);
cudaError_t launch_small_m_debug_partials(const GemmArgs &a, int kind, void *ws, size_t ws_bytes,
                                          cudaStream_t stream, const char **msg);
// The few-token layer from fp16 X (quantization included): the split GEMV
// quantizes in its prologue when its slice of X fits a ring slot; otherwise
// the quantizer writes A_q / s_a into the workspace first.  a.X is required,
// a.A_q / a.s_a are ignored.  Workspace: linear_small_m_workspace_bytes().
size_t linear_small_m_workspace_bytes(int64_t M, int64_t N4, int64_t N8, int64_t K);
bool linear_small_m_fused(int64_t M, int64_t N4, int64_t N8, int64_t K);
cudaError_t launch_linear_small_m(const GemmArgs &a, void *ws, size_t ws_bytes, cudaStream_t stream,
                                  const char **msg);
// The same with a static device scratch instead of a workspace (no allocation);
// fails with cudaErrorInvalidValue when the shape needs more than it holds.
cudaError_t launch_gemm_small_m_noalloc(const GemmArgs &a, cudaStream_t stream, const char **msg);
size_t small_m_scratch_capacity();

cudaError_t launch_selftest_wait_timeout(uint32_t limit_us, cudaStream_t stream);
cudaError_t launch_selftest_bounds(cudaStream_t stream);

// Global mixed-precision search (search.cuh).
cudaError_t launch_channel_salience(const float *W, int64_t N, int64_t K, const float *G, int64_t D, float *S,
                                    cudaStream_t stream, const char **msg);
size_t select_top_t_workspace_bytes(int64_t n);
cudaError_t launch_select_top_t(const float *S, int64_t n, int64_t T, uint8_t *is8, void *ws, cudaStream_t stream,
                                const char **msg);

int64_t padded_channels(int64_t n);  // n rounded up to a multiple of 256

}  // namespace mixllm

// mixllm.cu -- the C ABI declared in include/mixllm.h.  One translation unit:
// it includes the kernels so that they share the device status word.
//
// Host code here only validates arguments, encodes TMA descriptors and
// launches kernels; every step of the layer's arithmetic runs on the GPU.
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "../../include/mixllm.h"
#include "gemm_w4w8a8.cuh"
#include "gemm_small_m.cuh"
#include "search.cuh"
#include "launch.h"
#include "pack_host.cuh"
#include "quant.cuh"

namespace {

thread_local char g_last_error[512] = "";

mixllm_status fail(mixllm_status st, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}

mixllm_status ok() {
  g_last_error[0] = '\0';
  return MIXLLM_OK;
}

mixllm_status cuda_fail(cudaError_t e, const char *what) {
  return fail(MIXLLM_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Shape checks shared by the entry points.
mixllm_status check_k(int64_t K, int32_t group) {
  if (group != MIXLLM_GROUP) return fail(MIXLLM_ERR_UNSUPPORTED, "group size %d is not supported (only 128)", group);
  if (K <= 0 || K % MIXLLM_GROUP != 0)
    return fail(MIXLLM_ERR_UNSUPPORTED, "K = %lld must be a positive multiple of 128", static_cast<long long>(K));
  if (K > (1ll << 30)) return fail(MIXLLM_ERR_INVALID_ARG, "K = %lld is too large", static_cast<long long>(K));
  return MIXLLM_OK;
}

mixllm_status check_device() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0)
    return fail(MIXLLM_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a only", dev, major,
                minor);
  return MIXLLM_OK;
}

// Argument checks of the GEMM entry points.  Returns MIXLLM_OK with *empty
// set when there is nothing to compute.
mixllm_status check_gemm(const int8_t *A_q, const float *s_a, int64_t M, int64_t K, const uint8_t *W4,
                         const uint8_t *z4, const void *s_w4, const int32_t *idx4, int64_t N4, const int8_t *W8,
                         const void *s_w8, const int32_t *idx8, int64_t N8, void *Y, int32_t *P, bool *empty) {
  *empty = false;
  mixllm_status st = check_k(K, MIXLLM_GROUP);
  if (st != MIXLLM_OK) return st;
  if (M < 0 || N4 < 0 || N8 < 0) return fail(MIXLLM_ERR_INVALID_ARG, "negative size");
  if (M > 0x7FFFFFFF || N4 + N8 > 0x7FFFFFF0)
    return fail(MIXLLM_ERR_INVALID_ARG, "M or N beyond the supported 2^31 range");
  if (M == 0 || N4 + N8 == 0) {
    *empty = true;
    return MIXLLM_OK;
  }
  if (!A_q || !s_a || !(Y || P)) return fail(MIXLLM_ERR_INVALID_ARG, "null A_q, s_a or output");
  if (!aligned(A_q, 16)) return fail(MIXLLM_ERR_INVALID_ARG, "A_q must be 16-byte aligned");
  if (!aligned(s_a, 4)) return fail(MIXLLM_ERR_INVALID_ARG, "s_a must be 4-byte aligned");
  if (Y && !aligned(Y, 2)) return fail(MIXLLM_ERR_INVALID_ARG, "Y must be 2-byte aligned");
  if (P && !aligned(P, 4)) return fail(MIXLLM_ERR_INVALID_ARG, "P must be 4-byte aligned");
  if (N4 > 0) {
    if (!W4 || !z4 || !s_w4 || !idx4) return fail(MIXLLM_ERR_INVALID_ARG, "null 4-bit set buffer");
    if (!aligned(W4, 16) || !aligned(z4, 16) || !aligned(s_w4, 16) || !aligned(idx4, 4))
      return fail(MIXLLM_ERR_INVALID_ARG, "4-bit set buffers must be 16-byte aligned (idx4: 4)");
  }
  if (N8 > 0) {
    if (!W8 || !s_w8 || !idx8) return fail(MIXLLM_ERR_INVALID_ARG, "null 8-bit set buffer");
    if (!aligned(W8, 16) || !aligned(s_w8, 16) || !aligned(idx8, 4))
      return fail(MIXLLM_ERR_INVALID_ARG, "8-bit set buffers must be 16-byte aligned (idx8: 4)");
  }
  return check_device();
}

mixllm_status gemm_common(const int8_t *A_q, const float *s_a, int64_t M, int64_t K, const uint8_t *W4,
                          const uint8_t *z4, const void *s_w4, const int32_t *idx4, int64_t N4, const int8_t *W8,
                          const void *s_w8, const int32_t *idx8, int64_t N8, void *Y, int32_t *P, void *stream,
                          bool cvt_i2f = false) {
  bool empty = false;
  mixllm_status st = check_gemm(A_q, s_a, M, K, W4, z4, s_w4, idx4, N4, W8, s_w8, idx8, N8, Y, P, &empty);
  if (st != MIXLLM_OK) return st;
  if (empty) return ok();
  mixllm::GemmArgs a{A_q, s_a, M, K, W4, z4, s_w4, idx4, N4, W8, s_w8, idx8, N8, Y, P};
  a.cvt_i2f = cvt_i2f;
  const char *msg = "";
  cudaError_t e = mixllm::launch_gemm_w4w8a8(a, static_cast<cudaStream_t>(stream), &msg);
  if (e == cudaErrorNotSupported) return fail(MIXLLM_ERR_UNSUPPORTED, "%s", msg);
  if (e != cudaSuccess) return fail(MIXLLM_ERR_CUDA, "%s: %s", msg, cudaGetErrorString(e));
  return ok();
}

}  // namespace

extern "C" {

int mixllm_version(void) { return 100; }

const char *mixllm_last_error(void) { return g_last_error; }

mixllm_status mixllm_packed_sizes(int64_t N, int64_t K, int64_t N8, int32_t group, size_t out_bytes[7]) {
  mixllm_status st = check_k(K, group);
  if (st != MIXLLM_OK) return st;
  if (!out_bytes) return fail(MIXLLM_ERR_INVALID_ARG, "null out_bytes");
  if (N < 0 || N8 < 0 || N8 > N) return fail(MIXLLM_ERR_INVALID_ARG, "need 0 <= N8 <= N");
  const int64_t N4 = N - N8, G = K / MIXLLM_GROUP;
  const int64_t N4p = mixllm::padded_channels(N4), N8p = mixllm::padded_channels(N8);
  out_bytes[0] = static_cast<size_t>((N4 + 127) / 128 * 128 * (K / 2));  // whole 128-channel tiles
  out_bytes[1] = static_cast<size_t>(G * (N4p / 2));
  out_bytes[2] = static_cast<size_t>(G * N4p * 2);
  out_bytes[3] = static_cast<size_t>(N4 * 4);
  out_bytes[4] = static_cast<size_t>(N8 * K);
  out_bytes[5] = static_cast<size_t>(G * N8p * 2);
  out_bytes[6] = static_cast<size_t>(N8 * 4);
  return ok();
}

mixllm_status mixllm_quantize_act(const void *X_f16, int64_t M, int64_t K, int32_t group, int8_t *A_q, float *s_a,
                                  void *stream) {
  mixllm_status st = check_k(K, group);
  if (st != MIXLLM_OK) return st;
  if (M < 0) return fail(MIXLLM_ERR_INVALID_ARG, "M < 0");
  if (M == 0) return ok();
  if (!X_f16 || !A_q || !s_a) return fail(MIXLLM_ERR_INVALID_ARG, "null pointer");
  if (!aligned(X_f16, 16) || !aligned(A_q, 16) || !aligned(s_a, 4))
    return fail(MIXLLM_ERR_INVALID_ARG, "X and A_q must be 16-byte aligned, s_a 4-byte aligned");
  st = check_device();
  if (st != MIXLLM_OK) return st;
  cudaError_t e = mixllm::launch_quantize_act(X_f16, M, K, A_q, s_a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "quantize_act launch");
  return ok();
}

mixllm_status mixllm_pack_weights(const float *W, int64_t N, int64_t K, const uint8_t *is8, int64_t N8,
                                  int32_t group, uint8_t *W4, uint8_t *z4, void *s_w4_f16, int32_t *idx4,
                                  int8_t *W8, void *s_w8_f16, int32_t *idx8, void *stream) {
  mixllm_status st = check_k(K, group);
  if (st != MIXLLM_OK) return st;
  if (N < 0 || N8 < 0 || N8 > N) return fail(MIXLLM_ERR_INVALID_ARG, "need 0 <= N8 <= N");
  if (N > 0x7FFFFFF0) return fail(MIXLLM_ERR_INVALID_ARG, "N beyond the supported range");
  if (N == 0) return ok();
  const int64_t N4 = N - N8;
  if (!W || !is8) return fail(MIXLLM_ERR_INVALID_ARG, "null W or is8");
  if (!aligned(W, 16)) return fail(MIXLLM_ERR_INVALID_ARG, "W must be 16-byte aligned");
  if (N4 > 0 && (!W4 || !z4 || !s_w4_f16 || !idx4)) return fail(MIXLLM_ERR_INVALID_ARG, "null 4-bit output");
  if (N8 > 0 && (!W8 || !s_w8_f16 || !idx8)) return fail(MIXLLM_ERR_INVALID_ARG, "null 8-bit output");
  if ((W4 && !aligned(W4, 16)) || (z4 && !aligned(z4, 16)) || (s_w4_f16 && !aligned(s_w4_f16, 16)) ||
      (W8 && !aligned(W8, 16)) || (s_w8_f16 && !aligned(s_w8_f16, 16)) || (idx4 && !aligned(idx4, 4)) ||
      (idx8 && !aligned(idx8, 4)))
    return fail(MIXLLM_ERR_INVALID_ARG, "packed outputs must be 16-byte aligned (idx: 4)");
  st = check_device();
  if (st != MIXLLM_OK) return st;
  // clear any stale status first so a bad bit map is attributed to this call
  st = mixllm_sync_status(stream);
  if (st != MIXLLM_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = mixllm::launch_split_channels(is8, N, N8, idx4, idx8, s);
  if (e != cudaSuccess) return cuda_fail(e, "split_channels launch");
  if (N4 > 0) {
    e = mixllm::launch_pack_w4(W, N, K, idx4, N4, mixllm::padded_channels(N4), W4, z4, s_w4_f16, s);
    if (e != cudaSuccess) return cuda_fail(e, "pack_w4 launch");
  }
  if (N8 > 0) {
    e = mixllm::launch_pack_w8(W, N, K, idx8, N8, mixllm::padded_channels(N8), W8, s_w8_f16, s);
    if (e != cudaSuccess) return cuda_fail(e, "pack_w8 launch");
  }
  e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "pack synchronize");
  int status = 0;
  e = cudaMemcpyFromSymbol(&status, mixllm::g_status, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  if (status != 0) {
    const int zero = 0;
    cudaMemcpyToSymbol(mixllm::g_status, &zero, sizeof(int));
    if (status == mixllm::kStatusBadBitmap)
      return fail(MIXLLM_ERR_INVALID_ARG, "the bit map does not flag exactly N8 = %lld channels",
                  static_cast<long long>(N8));
    return fail(MIXLLM_ERR_TIMEOUT, "a device wait gave up during the pack");
  }
  return ok();
}

mixllm_status mixllm_pack_weights_host(const float *W, int64_t N, int64_t K, const uint8_t *is8, int64_t N8,
                                       int32_t group, uint8_t *W4, uint8_t *z4, void *s_w4_f16, int32_t *idx4,
                                       int8_t *W8, void *s_w8_f16, int32_t *idx8) {
  mixllm_status st = check_k(K, group);
  if (st != MIXLLM_OK) return st;
  if (N < 0 || N8 < 0 || N8 > N) return fail(MIXLLM_ERR_INVALID_ARG, "need 0 <= N8 <= N");
  if (N > 0x7FFFFFF0) return fail(MIXLLM_ERR_INVALID_ARG, "N beyond the supported range");
  if (N == 0) return ok();
  const int64_t N4 = N - N8;
  if (!W || !is8) return fail(MIXLLM_ERR_INVALID_ARG, "null W or is8");
  if (N4 > 0 && (!W4 || !z4 || !s_w4_f16 || !idx4)) return fail(MIXLLM_ERR_INVALID_ARG, "null 4-bit output");
  if (N8 > 0 && (!W8 || !s_w8_f16 || !idx8)) return fail(MIXLLM_ERR_INVALID_ARG, "null 8-bit output");
  // the channel lists go to the caller's buffers only once the map is known to be consistent
  int64_t n8 = 0;
  for (int64_t n = 0; n < N; ++n) n8 += is8[n] != 0;
  if (n8 != N8)
    return fail(MIXLLM_ERR_INVALID_ARG, "the bit map flags %lld channels, not N8 = %lld", static_cast<long long>(n8),
                static_cast<long long>(N8));
  (void)mixllm::host_split_channels(is8, N, N8, idx4, idx8);
  if (N4 > 0)
    mixllm::host_pack_w4(W, K, idx4, N4, mixllm::padded_channels(N4), W4, z4, static_cast<__half *>(s_w4_f16));
  if (N8 > 0) mixllm::host_pack_w8(W, K, idx8, N8, mixllm::padded_channels(N8), W8, static_cast<__half *>(s_w8_f16));
  return ok();
}

mixllm_status mixllm_gemm_w4w8a8(const int8_t *A_q, const float *s_a, int64_t M, int64_t K, const uint8_t *W4,
                                 const uint8_t *z4, const void *s_w4_f16, const int32_t *idx4, int64_t N4,
                                 const int8_t *W8, const void *s_w8_f16, const int32_t *idx8, int64_t N8,
                                 void *Y_f16, void *stream) {
  if (!Y_f16 && M > 0 && N4 + N8 > 0) return fail(MIXLLM_ERR_INVALID_ARG, "null Y");
  return gemm_common(A_q, s_a, M, K, W4, z4, s_w4_f16, idx4, N4, W8, s_w8_f16, idx8, N8, Y_f16, nullptr, stream);
}

mixllm_status mixllm_gemm_w4w8a8_plain_i2f(const int8_t *A_q, const float *s_a, int64_t M, int64_t K,
                                           const uint8_t *W4, const uint8_t *z4, const void *s_w4_f16,
                                           const int32_t *idx4, int64_t N4, const int8_t *W8, const void *s_w8_f16,
                                           const int32_t *idx8, int64_t N8, void *Y_f16, void *stream) {
  if (!Y_f16 && M > 0 && N4 + N8 > 0) return fail(MIXLLM_ERR_INVALID_ARG, "null Y");
  return gemm_common(A_q, s_a, M, K, W4, z4, s_w4_f16, idx4, N4, W8, s_w8_f16, idx8, N8, Y_f16, nullptr, stream,
                     true);
}

mixllm_status mixllm_gemm_debug_partials(const int8_t *A_q, const float *s_a, int64_t M, int64_t K,
                                         const uint8_t *W4, const uint8_t *z4, const void *s_w4_f16,
                                         const int32_t *idx4, int64_t N4, const int8_t *W8, const void *s_w8_f16,
                                         const int32_t *idx8, int64_t N8, int32_t *P, void *stream) {
  if (!P && M > 0 && N4 + N8 > 0) return fail(MIXLLM_ERR_INVALID_ARG, "null P");
  return gemm_common(A_q, s_a, M, K, W4, z4, s_w4_f16, idx4, N4, W8, s_w8_f16, idx8, N8, nullptr, P, stream);
}

mixllm_status mixllm_small_m_workspace_bytes(int64_t M, int64_t K, int64_t N4, int64_t N8, size_t *bytes) {
  mixllm_status st = check_k(K, MIXLLM_GROUP);
  if (st != MIXLLM_OK) return st;
  if (!bytes) return fail(MIXLLM_ERR_INVALID_ARG, "null bytes");
  if (M < 1 || M > 64) return fail(MIXLLM_ERR_INVALID_ARG, "the small-M path takes 1 <= M <= 64");
  if (N4 < 0 || N8 < 0 || N4 + N8 > 0x7FFFFFF0) return fail(MIXLLM_ERR_INVALID_ARG, "bad N4 / N8");
  *bytes = mixllm::small_m_workspace_bytes(M, N4, N8, K);
  return ok();
}

mixllm_status mixllm_small_m_kernel(int64_t M, int64_t K, int64_t N4, int64_t N8, int32_t *kind) {
  mixllm_status st = check_k(K, MIXLLM_GROUP);
  if (st != MIXLLM_OK) return st;
  if (!kind) return fail(MIXLLM_ERR_INVALID_ARG, "null kind");
  if (M < 1 || M > 64) return fail(MIXLLM_ERR_INVALID_ARG, "the small-M path takes 1 <= M <= 64");
  if (N4 < 0 || N8 < 0 || N4 + N8 > 0x7FFFFFF0) return fail(MIXLLM_ERR_INVALID_ARG, "bad N4 / N8");
  *kind = mixllm::small_m_kernel_kind(M, N4, N8, K);
  return ok();
}

mixllm_status mixllm_gemm_w4w8a8_small_m(const int8_t *A_q, const float *s_a, int64_t M, int64_t K,
                                         const uint8_t *W4, const uint8_t *z4, const void *s_w4_f16,
                                         const int32_t *idx4, int64_t N4, const int8_t *W8, const void *s_w8_f16,
                                         const int32_t *idx8, int64_t N8, void *Y_f16, void *workspace,
                                         size_t workspace_bytes, void *stream) {
  if (M > 64) return fail(MIXLLM_ERR_INVALID_ARG, "the small-M path takes M <= 64 (M = %lld)", static_cast<long long>(M));
  if (!Y_f16 && M > 0 && N4 + N8 > 0) return fail(MIXLLM_ERR_INVALID_ARG, "null Y");
  bool empty = false;
  mixllm_status st =
      check_gemm(A_q, s_a, M, K, W4, z4, s_w4_f16, idx4, N4, W8, s_w8_f16, idx8, N8, Y_f16, nullptr, &empty);
  if (st != MIXLLM_OK) return st;
  if (empty) return ok();
  const size_t need = mixllm::small_m_workspace_bytes(M, N4, N8, K);
  if (workspace_bytes < need)
    return fail(MIXLLM_ERR_INVALID_ARG, "workspace of %zu bytes is smaller than the %zu this shape needs",
                workspace_bytes, need);
  if (need > 0 && (!workspace || !aligned(workspace, 16)))
    return fail(MIXLLM_ERR_INVALID_ARG, "workspace must be a 16-byte aligned device buffer");
  mixllm::GemmArgs a{A_q, s_a, M, K, W4, z4, s_w4_f16, idx4, N4, W8, s_w8_f16, idx8, N8, Y_f16, nullptr};
  const char *msg = "";
  cudaError_t e = mixllm::launch_gemm_small_m(a, workspace, workspace_bytes, static_cast<cudaStream_t>(stream), &msg);
  if (e == cudaErrorNotSupported) return fail(MIXLLM_ERR_UNSUPPORTED, "%s", msg);
  if (e != cudaSuccess) return fail(MIXLLM_ERR_CUDA, "%s: %s", msg, cudaGetErrorString(e));
  return ok();
}

mixllm_status mixllm_small_m_debug_workspace_bytes(int64_t M, int64_t K, int64_t N4, int64_t N8, int32_t kind,
                                                   size_t *bytes) {
  mixllm_status st = check_k(K, MIXLLM_GROUP);
  if (st != MIXLLM_OK) return st;
  if (!bytes) return fail(MIXLLM_ERR_INVALID_ARG, "null bytes");
  if (M < 1 || M > 64) return fail(MIXLLM_ERR_INVALID_ARG, "the small-M path takes 1 <= M <= 64");
  if (N4 < 0 || N8 < 0 || N4 + N8 > 0x7FFFFFF0) return fail(MIXLLM_ERR_INVALID_ARG, "bad N4 / N8");
  if (!mixllm::small_m_kernel_allowed(M, N4, N8, K, kind))
    return fail(MIXLLM_ERR_UNSUPPORTED, "few-token kernel %d cannot take M = %lld, K = %lld", static_cast<int>(kind),
                static_cast<long long>(M), static_cast<long long>(K));
  *bytes = mixllm::small_m_debug_workspace_bytes(M, N4, N8, K, kind);
  return ok();
}

mixllm_status mixllm_small_m_debug_partials(const int8_t *A_q, const float *s_a, int64_t M, int64_t K,
                                            const uint8_t *W4, const uint8_t *z4, const void *s_w4_f16,
                                            const int32_t *idx4, int64_t N4, const int8_t *W8,
                                            const void *s_w8_f16, const int32_t *idx8, int64_t N8, int32_t kind,
                                            int32_t *P, void *Y_f16, void *workspace, size_t workspace_bytes,
                                            void *stream) {
  if (M < 1 || M > 64) return fail(MIXLLM_ERR_INVALID_ARG, "the small-M path takes 1 <= M <= 64");
  if (N4 + N8 > 0 && (!Y_f16 || !P)) return fail(MIXLLM_ERR_INVALID_ARG, "null Y or P");
  bool empty = false;
  mixllm_status st =
      check_gemm(A_q, s_a, M, K, W4, z4, s_w4_f16, idx4, N4, W8, s_w8_f16, idx8, N8, Y_f16, nullptr, &empty);
  if (st != MIXLLM_OK) return st;
  if (empty) return ok();
  if (!mixllm::small_m_kernel_allowed(M, N4, N8, K, kind))
    return fail(MIXLLM_ERR_UNSUPPORTED, "few-token kernel %d cannot take M = %lld, K = %lld", static_cast<int>(kind),
                static_cast<long long>(M), static_cast<long long>(K));
  if (!aligned(P, 4)) return fail(MIXLLM_ERR_INVALID_ARG, "P must be 4-byte aligned");
  const size_t need = mixllm::small_m_debug_workspace_bytes(M, N4, N8, K, kind);
  if (workspace_bytes < need)
    return fail(MIXLLM_ERR_INVALID_ARG, "workspace of %zu bytes is smaller than the %zu this shape needs",
                workspace_bytes, need);
  if (need > 0 && (!workspace || !aligned(workspace, 16)))
    return fail(MIXLLM_ERR_INVALID_ARG, "workspace must be a 16-byte aligned device buffer");
  mixllm::GemmArgs a{A_q, s_a, M, K, W4, z4, s_w4_f16, idx4, N4, W8, s_w8_f16, idx8, N8, Y_f16, P};
  const char *msg = "";
  cudaError_t e = mixllm::launch_small_m_debug_partials(a, kind, workspace, workspace_bytes,
                                                        static_cast<cudaStream_t>(stream), &msg);
  if (e == cudaErrorNotSupported) return fail(MIXLLM_ERR_UNSUPPORTED, "%s", msg);
  if (e != cudaSuccess) return fail(MIXLLM_ERR_CUDA, "%s: %s", msg, cudaGetErrorString(e));
  return ok();
}

mixllm_status mixllm_gemm_w4w8a8_small_m_noalloc(const int8_t *A_q, const float *s_a, int64_t M, int64_t K,
                                                 const uint8_t *W4, const uint8_t *z4, const void *s_w4_f16,
                                                 const int32_t *idx4, int64_t N4, const int8_t *W8,
                                                 const void *s_w8_f16, const int32_t *idx8, int64_t N8, void *Y_f16,
                                                 void *stream) {
  if (M > 64) return fail(MIXLLM_ERR_INVALID_ARG, "the small-M path takes M <= 64 (M = %lld)", static_cast<long long>(M));
  if (!Y_f16 && M > 0 && N4 + N8 > 0) return fail(MIXLLM_ERR_INVALID_ARG, "null Y");
  bool empty = false;
  mixllm_status st =
      check_gemm(A_q, s_a, M, K, W4, z4, s_w4_f16, idx4, N4, W8, s_w8_f16, idx8, N8, Y_f16, nullptr, &empty);
  if (st != MIXLLM_OK) return st;
  if (empty) return ok();
  const size_t need = mixllm::small_m_workspace_bytes(M, N4, N8, K);
  if (need > mixllm::small_m_scratch_capacity())
    return fail(MIXLLM_ERR_UNSUPPORTED, "this shape needs %zu bytes of scratch; the static buffer holds %zu", need,
                mixllm::small_m_scratch_capacity());
  mixllm::GemmArgs a{A_q, s_a, M, K, W4, z4, s_w4_f16, idx4, N4, W8, s_w8_f16, idx8, N8, Y_f16, nullptr};
  const char *msg = "";
  cudaError_t e = mixllm::launch_gemm_small_m_noalloc(a, static_cast<cudaStream_t>(stream), &msg);
  if (e == cudaErrorNotSupported) return fail(MIXLLM_ERR_UNSUPPORTED, "%s", msg);
  if (e != cudaSuccess) return fail(MIXLLM_ERR_CUDA, "%s: %s", msg, cudaGetErrorString(e));
  return ok();
}

mixllm_status mixllm_linear_small_m_workspace_bytes(int64_t M, int64_t K, int64_t N4, int64_t N8, size_t *bytes) {
  mixllm_status st = check_k(K, MIXLLM_GROUP);
  if (st != MIXLLM_OK) return st;
  if (!bytes) return fail(MIXLLM_ERR_INVALID_ARG, "null bytes");
  if (M < 1 || M > 64) return fail(MIXLLM_ERR_INVALID_ARG, "the small-M path takes 1 <= M <= 64");
  if (N4 < 0 || N8 < 0 || N4 + N8 > 0x7FFFFFF0) return fail(MIXLLM_ERR_INVALID_ARG, "bad N4 / N8");
  *bytes = mixllm::linear_small_m_workspace_bytes(M, N4, N8, K);
  return ok();
}

mixllm_status mixllm_linear_small_m(const void *X_f16, int64_t M, int64_t K, const uint8_t *W4, const uint8_t *z4,
                                    const void *s_w4_f16, const int32_t *idx4, int64_t N4, const int8_t *W8,
                                    const void *s_w8_f16, const int32_t *idx8, int64_t N8, void *Y_f16,
                                    void *workspace, size_t workspace_bytes, void *stream) {
  if (M > 64) return fail(MIXLLM_ERR_INVALID_ARG, "the small-M path takes M <= 64 (M = %lld)", static_cast<long long>(M));
  if (M > 0 && N4 + N8 > 0) {
    if (!X_f16 || !Y_f16) return fail(MIXLLM_ERR_INVALID_ARG, "null X or Y");
    if (!aligned(X_f16, 16)) return fail(MIXLLM_ERR_INVALID_ARG, "X must be 16-byte aligned");
  }
  bool empty = false;
  // the weight and size checks of the GEMM (X stands in for A_q / s_a, whose checks it passes)
  mixllm_status st = check_gemm(static_cast<const int8_t *>(X_f16), static_cast<const float *>(X_f16), M, K, W4, z4,
                                s_w4_f16, idx4, N4, W8, s_w8_f16, idx8, N8, Y_f16, nullptr, &empty);
  if (st != MIXLLM_OK) return st;
  if (empty) return ok();
  const size_t need = mixllm::linear_small_m_workspace_bytes(M, N4, N8, K);
  if (workspace_bytes < need)
    return fail(MIXLLM_ERR_INVALID_ARG, "workspace of %zu bytes is smaller than the %zu this shape needs",
                workspace_bytes, need);
  if (need > 0 && (!workspace || !aligned(workspace, 256)))
    return fail(MIXLLM_ERR_INVALID_ARG, "workspace must be a 256-byte aligned device buffer");
  mixllm::GemmArgs a{nullptr, nullptr, M, K, W4, z4, s_w4_f16, idx4, N4, W8, s_w8_f16, idx8, N8, Y_f16, nullptr};
  a.X = X_f16;
  const char *msg = "";
  cudaError_t e = mixllm::launch_linear_small_m(a, workspace, workspace_bytes, static_cast<cudaStream_t>(stream), &msg);
  if (e == cudaErrorNotSupported) return fail(MIXLLM_ERR_UNSUPPORTED, "%s", msg);
  if (e != cudaSuccess) return fail(MIXLLM_ERR_CUDA, "%s: %s", msg, cudaGetErrorString(e));
  return ok();
}

mixllm_status mixllm_linear_workspace_bytes(int64_t M, int64_t K, int64_t N4, int64_t N8, size_t *bytes) {
  mixllm_status st = check_k(K, MIXLLM_GROUP);
  if (st != MIXLLM_OK) return st;
  if (!bytes) return fail(MIXLLM_ERR_INVALID_ARG, "null bytes");
  if (M < 0) return fail(MIXLLM_ERR_INVALID_ARG, "M < 0");
  if (N4 < 0 || N8 < 0 || N4 + N8 > 0x7FFFFFF0) return fail(MIXLLM_ERR_INVALID_ARG, "bad N4 / N8");
  *bytes = M == 0 ? 0 : mixllm::linear_workspace_bytes(M, N4, N8, K);
  return ok();
}

static mixllm_status linear_entry(const void *X_f16, int64_t M, int64_t K, const uint8_t *W4, const uint8_t *z4,
                                  const void *s_w4_f16, const int32_t *idx4, int64_t N4, const int8_t *W8,
                                  const void *s_w8_f16, const int32_t *idx8, int64_t N8, void *Y_f16,
                                  void *workspace, size_t workspace_bytes, void *stream, bool one_launch) {
  if (one_launch && M > 0 && M <= 64)
    return fail(MIXLLM_ERR_INVALID_ARG, "the one-launch tiled form takes M > 64 (M = %lld)", static_cast<long long>(M));
  if (M > 0 && M <= 64)
    return mixllm_linear_small_m(X_f16, M, K, W4, z4, s_w4_f16, idx4, N4, W8, s_w8_f16, idx8, N8, Y_f16, workspace,
                                 workspace_bytes, stream);
  if (M > 0 && N4 + N8 > 0) {
    if (!X_f16 || !Y_f16) return fail(MIXLLM_ERR_INVALID_ARG, "null X or Y");
    if (!aligned(X_f16, 16)) return fail(MIXLLM_ERR_INVALID_ARG, "X must be 16-byte aligned");
  }
  bool empty = false;
  // the weight and size checks of the GEMM (X stands in for A_q / s_a, whose checks it passes)
  mixllm_status st = check_gemm(static_cast<const int8_t *>(X_f16), static_cast<const float *>(X_f16), M, K, W4, z4,
                                s_w4_f16, idx4, N4, W8, s_w8_f16, idx8, N8, Y_f16, nullptr, &empty);
  if (st != MIXLLM_OK) return st;
  if (empty) return ok();
  const size_t need = mixllm::linear_workspace_bytes(M, N4, N8, K);
  if (workspace_bytes < need)
    return fail(MIXLLM_ERR_INVALID_ARG, "workspace of %zu bytes is smaller than the %zu this shape needs",
                workspace_bytes, need);
  if (!workspace || !aligned(workspace, 256))
    return fail(MIXLLM_ERR_INVALID_ARG, "workspace must be a 256-byte aligned device buffer");
  mixllm::GemmArgs a{nullptr, nullptr, M, K, W4, z4, s_w4_f16, idx4, N4, W8, s_w8_f16, idx8, N8, Y_f16, nullptr};
  a.X = X_f16;
  const char *msg = "";
  cudaError_t e =
      mixllm::launch_linear(a, workspace, workspace_bytes, one_launch, static_cast<cudaStream_t>(stream), &msg);
  if (e == cudaErrorNotSupported) return fail(MIXLLM_ERR_UNSUPPORTED, "%s", msg);
  if (e != cudaSuccess) return fail(MIXLLM_ERR_CUDA, "%s: %s", msg, cudaGetErrorString(e));
  return ok();
}

mixllm_status mixllm_linear(const void *X_f16, int64_t M, int64_t K, const uint8_t *W4, const uint8_t *z4,
                            const void *s_w4_f16, const int32_t *idx4, int64_t N4, const int8_t *W8,
                            const void *s_w8_f16, const int32_t *idx8, int64_t N8, void *Y_f16, void *workspace,
                            size_t workspace_bytes, void *stream) {
  return linear_entry(X_f16, M, K, W4, z4, s_w4_f16, idx4, N4, W8, s_w8_f16, idx8, N8, Y_f16, workspace,
                      workspace_bytes, stream, false);
}

mixllm_status mixllm_linear_one_launch(const void *X_f16, int64_t M, int64_t K, const uint8_t *W4, const uint8_t *z4,
                                       const void *s_w4_f16, const int32_t *idx4, int64_t N4, const int8_t *W8,
                                       const void *s_w8_f16, const int32_t *idx8, int64_t N8, void *Y_f16,
                                       void *workspace, size_t workspace_bytes, void *stream) {
  return linear_entry(X_f16, M, K, W4, z4, s_w4_f16, idx4, N4, W8, s_w8_f16, idx8, N8, Y_f16, workspace,
                      workspace_bytes, stream, true);
}

mixllm_status mixllm_channel_salience(const float *W, int64_t N, int64_t K, const float *G, int64_t D, float *S,
                                      void *stream) {
  mixllm_status st = check_k(K, MIXLLM_GROUP);
  if (st != MIXLLM_OK) return st;
  if (K > 56832) return fail(MIXLLM_ERR_UNSUPPORTED, "K = %lld is beyond 56832", static_cast<long long>(K));
  if (N < 0 || D < 1) return fail(MIXLLM_ERR_INVALID_ARG, "need N >= 0 and D >= 1");
  if (N > 0x7FFFFFFF) return fail(MIXLLM_ERR_INVALID_ARG, "N beyond the supported 2^31 range");
  if (N == 0) return ok();
  if (!W || !G || !S) return fail(MIXLLM_ERR_INVALID_ARG, "null pointer");
  if (!aligned(W, 16) || !aligned(G, 16) || !aligned(S, 4))
    return fail(MIXLLM_ERR_INVALID_ARG, "W and G must be 16-byte aligned, S 4-byte aligned");
  st = check_device();
  if (st != MIXLLM_OK) return st;
  const char *msg = "";
  cudaError_t e = mixllm::launch_channel_salience(W, N, K, G, D, S, static_cast<cudaStream_t>(stream), &msg);
  if (e != cudaSuccess) return fail(MIXLLM_ERR_CUDA, "%s: %s", msg, cudaGetErrorString(e));
  return ok();
}

mixllm_status mixllm_select_top_t_workspace_bytes(int64_t n, size_t *bytes) {
  if (!bytes) return fail(MIXLLM_ERR_INVALID_ARG, "null bytes");
  if (n < 0 || n > (1ll << 40)) return fail(MIXLLM_ERR_INVALID_ARG, "bad n");
  *bytes = mixllm::select_top_t_workspace_bytes(n);
  return ok();
}

mixllm_status mixllm_select_top_t(const float *S, int64_t n, int64_t T, uint8_t *is8, void *workspace,
                                  size_t workspace_bytes, void *stream) {
  if (n < 0 || n > (1ll << 40)) return fail(MIXLLM_ERR_INVALID_ARG, "bad n");
  if (T < 0 || T > n) return fail(MIXLLM_ERR_INVALID_ARG, "need 0 <= T <= n");
  if (n == 0) return ok();
  if (!S || !is8) return fail(MIXLLM_ERR_INVALID_ARG, "null pointer");
  if (!aligned(S, 4)) return fail(MIXLLM_ERR_INVALID_ARG, "S must be 4-byte aligned");
  const size_t need = mixllm::select_top_t_workspace_bytes(n);
  if (workspace_bytes < need || !workspace || !aligned(workspace, 16))
    return fail(MIXLLM_ERR_INVALID_ARG, "workspace must be a 16-byte aligned device buffer of %zu bytes", need);
  mixllm_status st = check_device();
  if (st != MIXLLM_OK) return st;
  const char *msg = "";
  cudaError_t e = mixllm::launch_select_top_t(S, n, T, is8, workspace, static_cast<cudaStream_t>(stream), &msg);
  if (e != cudaSuccess) return fail(MIXLLM_ERR_CUDA, "%s: %s", msg, cudaGetErrorString(e));
  return ok();
}

mixllm_status mixllm_sync_status(void *stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  int status = 0;
  e = cudaMemcpyFromSymbol(&status, mixllm::g_status, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  if (status != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(mixllm::g_status, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "status clear");
    if (status == mixllm::kStatusTimeout) return fail(MIXLLM_ERR_TIMEOUT, "a device-side wait gave up");
    if (status == mixllm::kStatusBounds)
      return fail(MIXLLM_ERR_BOUNDS, "a range check of the checked build failed (the access was skipped)");
    return fail(MIXLLM_ERR_INVALID_ARG, "device reported status %d", status);
  }
  return ok();
}

int mixllm_checked_build(void) { return MIXLLM_CHECKED ? 1 : 0; }

mixllm_status mixllm_selftest_bounds(void *stream) {
  if (!MIXLLM_CHECKED) return fail(MIXLLM_ERR_UNSUPPORTED, "the release build has no range checks");
  mixllm_status st = check_device();
  if (st != MIXLLM_OK) return st;
  cudaError_t e = mixllm::launch_selftest_bounds(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "selftest launch");
  return ok();
}

mixllm_status mixllm_selftest_wait_timeout(uint32_t limit_us, void *stream) {
  if (limit_us < 1 || limit_us > 1000000) return fail(MIXLLM_ERR_INVALID_ARG, "limit_us must be in 1..1000000");
  mixllm_status st = check_device();
  if (st != MIXLLM_OK) return st;
  cudaError_t e = mixllm::launch_selftest_wait_timeout(limit_us, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "selftest launch");
  return ok();
}

}  // extern "C"

/*
 * mixllm.h -- C ABI of the B200 (sm_100a) W4.4A8 linear layer of MixLLM.
 *
 * The layer computes Y[M, N] = X[M, K] . W[N, K]^T with
 *   - activations quantized per token to int8, symmetric, in groups of 128
 *     along K (MLSys 2026 talk notes on MixLLM, notes.yuuk.io,
 *     §設計判断の概要; awesome-system-papers page "MixLLM (MLSys 2026)",
 *     核心方法),
 *   - output channels split into a 4-bit asymmetric set (uint4 codes, uint4
 *     zero point and fp16 scale per group of 128) and an 8-bit symmetric set
 *     (int8 codes, fp16 scale per group) by a global channel bit map
 *     (talk notes §設計判断の概要, §グローバル混合精度探索),
 *   - both sets multiplied on int8 tensor cores with two-step dequantization:
 *     P = sum over a group of (W_q - z) * A_q in int32, then
 *     acc += float(P) * s_w * s_a in fp32, with the int32-to-float step done
 *     by the 0x4b400000 bias trick (talk notes §二段階逆量子化による int8
 *     Tensor Core 活用, §高速 I2F 変換),
 *   - each channel's fp16 result written to its own column of one Y
 *     (talk notes §並列実行, fused scatter epilogue).
 *
 * Conventions for every entry point:
 *   - The caller owns every buffer and every stream; the library allocates
 *     nothing on the call path.  Device pointers are plain CUDA device
 *     addresses on the current device.  `stream` is a cudaStream_t (NULL =
 *     the legacy default stream).
 *   - Calls are asynchronous on `stream` unless stated otherwise.  Argument
 *     errors are found on the host and returned at once, with nothing
 *     launched.  A device-side wait that gives up (a hang guard, which never
 *     fires in correct operation) is recorded in a device status word and
 *     reported by mixllm_sync_status().
 *   - No call aborts the process or throws; the message of the last error
 *     of the calling thread is available from mixllm_last_error().
 *   - The group size is fixed at 128 (talk notes §設計判断の概要); any other
 *     value returns MIXLLM_ERR_UNSUPPORTED.  K must be a positive multiple
 *     of 128.
 */
#ifndef MIXLLM_H_
#define MIXLLM_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MIXLLM_API __attribute__((visibility("default")))
#else
#define MIXLLM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MIXLLM_OK = 0,
    MIXLLM_ERR_INVALID_ARG = 1, /* null / misaligned pointer, bad size      */
    MIXLLM_ERR_UNSUPPORTED = 2, /* group != 128, K % 128 != 0, no sm_100a  */
    MIXLLM_ERR_CUDA = 3,        /* a CUDA runtime call failed              */
    MIXLLM_ERR_TIMEOUT = 4,     /* a device-side wait gave up              */
    MIXLLM_ERR_BOUNDS = 5       /* checked build: a kernel's range check of
                                   a tensor- or shared-memory access failed
                                   (the access was skipped)                */
} mixllm_status;

#define MIXLLM_GROUP 128

/* Library version (major*10000 + minor*100 + patch). */
MIXLLM_API int mixllm_version(void);

/* Message of the last error returned to the calling thread ("" if none). */
MIXLLM_API const char *mixllm_last_error(void);

/*
 * Byte sizes of the seven packed-weight buffers for N output channels, of
 * which N8 are 8-bit, and inner size K:
 *   out_bytes[0] W4    uint8 [T4, G, 128, 64]  4-bit codes, two per byte,
 *                      T4 = ceil(N4/128) tiles of 128 rows
 *   out_bytes[1] z4    uint8 [G, N4p/2]  4-bit zero points, two per byte
 *   out_bytes[2] s_w4  fp16  [G, N4p]    4-bit set scales
 *   out_bytes[3] idx4  int32 [N4]        output column of each 4-bit row
 *   out_bytes[4] W8    int8  [N8, K]     8-bit codes
 *   out_bytes[5] s_w8  fp16  [G, N8p]    8-bit set scales
 *   out_bytes[6] idx8  int32 [N8]        output column of each 8-bit row
 * with N4 = N - N8, G = K/128 and Np = N rounded up to a multiple of 256.
 * The 4-bit set's footprint is 0.5 + 2.5/G bytes per weight and the 8-bit
 * set's 1 + 2/G (talk notes §ルーフラインモデルによる性能分析), plus the
 * padding of the scale/zero arrays to 256 channels.
 * Host-only; touches no device.
 */
MIXLLM_API mixllm_status mixllm_packed_sizes(int64_t N, int64_t K, int64_t N8, int32_t group,
                                  size_t out_bytes[7]);

/*
 * Activation quantization (one kernel): for every token m and group g of
 * 128 columns, amax = max |x|, s_a = amax / 127 (fp32, IEEE division),
 * A_q = clamp(round_half_even(x / s_a), -127, 127) with x / s_a the IEEE fp32
 * quotient; a group whose amax is 0 gets s_a = 0 and A_q = 0.  (Talk notes
 * §設計判断の概要: activations 8-bit symmetric, group-wise RTN; the rounding
 * mode and the fp32 scale are this library's reading -- the pages give
 * neither.)
 *   X_f16  device, fp16 [M, K] row-major, 16-byte aligned, read only
 *   A_q    device, int8 [M, K] row-major, 16-byte aligned, written
 *   s_a    device, fp32 [M, K/128] row-major, 4-byte aligned, written
 * M = 0 is a no-op.  Asynchronous on `stream`.
 */
MIXLLM_API mixllm_status mixllm_quantize_act(const void *X_f16, int64_t M, int64_t K, int32_t group,
                                  int8_t *A_q, float *s_a, void *stream);

/*
 * Offline weight quantization and pre-pack (device kernels).  The channels
 * with is8[n] != 0 form the 8-bit symmetric set, the rest the 4-bit
 * asymmetric set; each set is listed in ascending channel order (the pages
 * leave the order open; it does not change Y).
 *   4-bit, per (channel, group): lo = min(0, min w), hi = max(0, max w),
 *     s = fp16(min((hi - lo)/15, 65504)), z = clamp(rne(-lo/s), 0, 15),
 *     q = clamp(rne(w/s) + z, 0, 15); s == 0 gives z = q = 0.
 *   8-bit, per (channel, group): s = fp16(min(amax/127, 65504)),
 *     q = clamp(rne(w/s), -127, 127); s == 0 gives q = 0.
 * Packed layout (the buffers of mixllm_packed_sizes):
 *   W4: row r (channel idx4[r]) of group g is the 64 bytes at
 *       ((r/128)*G + g)*8192 + (r%128)*64, so that each 128-channel tile's
 *       group is one contiguous 8 KiB block; in each run c of 32 consecutive
 *       k, byte 16c+i (i = 0..15) holds code k = 32c+i in its low nibble and
 *       k = 32c+16+i in its high nibble; rows past N4 are 0.
 *   z4: zero point of row r, group g in byte g*N4p/2 + r/2, low nibble for
 *       even r, high for odd r; padding rows are 0.
 *   s_w4 / s_w8: scale of row r, group g at g*Np + r; padding rows are 0.
 *   W8: row r holds channel idx8[r], int8 codes in k order.
 * Arguments:
 *   W     device, fp32 [N, K] row-major, 16-byte aligned, read only
 *   is8   device, uint8 [N], the global channel bit map, read only
 *   N8    number of nonzero is8 entries (checked on the device)
 *   outputs: device buffers of the sizes given by mixllm_packed_sizes, each
 *     16-byte aligned (a buffer of size 0 may be NULL).
 * SYNCHRONOUS: waits for `stream` and returns MIXLLM_ERR_INVALID_ARG if the
 * bit map holds a number of 8-bit channels other than N8 (then the outputs
 * are unspecified).
 */
MIXLLM_API mixllm_status mixllm_pack_weights(const float *W, int64_t N, int64_t K, const uint8_t *is8,
                                  int64_t N8, int32_t group,
                                  uint8_t *W4, uint8_t *z4, void *s_w4_f16, int32_t *idx4,
                                  int8_t *W8, void *s_w8_f16, int32_t *idx8, void *stream);

/*
 * The same offline quantization and pre-pack on the host CPU, for weights in
 * host memory (converting a checkpoint without a GPU): the quantizers,
 * rounding (IEEE fp32 division, round half to even, fp16 round to nearest)
 * and packed layout of mixllm_pack_weights, byte for byte.  Every pointer is
 * HOST memory (W fp32 [N, K] row-major; is8 uint8 [N]; the outputs sized by
 * mixllm_packed_sizes); nothing touches a device, nothing runs on the layer's
 * hot path.  SYNCHRONOUS.  Returns MIXLLM_ERR_INVALID_ARG (outputs
 * untouched) when the bit map flags a number of channels other than N8.
 */
MIXLLM_API mixllm_status mixllm_pack_weights_host(const float *W, int64_t N, int64_t K, const uint8_t *is8,
                                       int64_t N8, int32_t group,
                                       uint8_t *W4, uint8_t *z4, void *s_w4_f16, int32_t *idx4,
                                       int8_t *W8, void *s_w8_f16, int32_t *idx8);

/*
 * The fused W4.4A8 GEMM: one launch covers both channel sets.  For each
 * output channel n of a set and token m,
 *   P_g = sum_{k in group g} (W_q[n,k] - z[n,g]) * A_q[m,k]   (int32 exact,
 *         z = 0 for the 8-bit set; int8 tensor cores, tcgen05 kind::i8),
 *   acc = sum_g float(P_g) * s_w[n,g] * s_a[m,g]  (fp32, groups in K order;
 *         float(P_g) by the 0x4b400000 bias trick, exact for |P_g| <= 2^22,
 *         and folded into one FMA that rounds P_g * s_w once; that product
 *         is then accumulated with an FMA by s_a),
 *   Y[m, idx[n]] = fp16_rn(acc).
 * Arguments:
 *   A_q, s_a   device, as written by mixllm_quantize_act (A_q 16-byte
 *              aligned, K a multiple of 128)
 *   W4, z4, s_w4, idx4, N4   the 4-bit set as written by mixllm_pack_weights
 *   W8, s_w8, idx8, N8       the 8-bit set as written by mixllm_pack_weights
 *              (N4 = 0 or N8 = 0 is allowed; that set's pointers may be NULL)
 *   Y          device, fp16 [M, N4 + N8] row-major, 2-byte aligned, written;
 *              column idx[n] receives channel n.  idx4 and idx8 together must
 *              list every column exactly once (not checked here).
 * The weights' packed rows are padded by the caller-provided layout only in
 * the scale and zero arrays; nothing is read outside the buffers sized by
 * mixllm_packed_sizes.  The launch picks its token tile (128, or 64 when the
 * layer's tiles would leave SMs idle); Y's bits do not depend on it.
 * Asynchronous on `stream`.
 */
MIXLLM_API mixllm_status mixllm_gemm_w4w8a8(const int8_t *A_q, const float *s_a, int64_t M, int64_t K,
                                 const uint8_t *W4, const uint8_t *z4, const void *s_w4_f16,
                                 const int32_t *idx4, int64_t N4,
                                 const int8_t *W8, const void *s_w8_f16,
                                 const int32_t *idx8, int64_t N8,
                                 void *Y_f16, void *stream);

/*
 * Debug path of the same kernel: writes the per-group int32 partials
 *   P[m, idx[n], g] = sum_{k in g} (W_q[n,k] - z[n,g]) * A_q[m,k]
 * (step 2 of the two-step dequantization, without the bias) into
 *   P   device, int32 [M, N4 + N8, K/128], 4-byte aligned,
 * instead of Y.  Same arguments and rules otherwise.  Slow (uncoalesced
 * stores); for parity tests only.
 */
MIXLLM_API mixllm_status mixllm_gemm_debug_partials(const int8_t *A_q, const float *s_a, int64_t M, int64_t K,
                                         const uint8_t *W4, const uint8_t *z4, const void *s_w4_f16,
                                         const int32_t *idx4, int64_t N4,
                                         const int8_t *W8, const void *s_w8_f16,
                                         const int32_t *idx8, int64_t N8,
                                         int32_t *P, void *stream);

/*
 * The same GEMM as mixllm_gemm_w4w8a8 with one step done the plain way: the
 * int32 partials are converted to float by the int -> float convert
 * instruction, and the tensor-memory accumulator is not preset to the
 * 0x4b400000 bias.  MLSys 2026 talk notes on MixLLM, §高速 I2F 変換, measure
 * what the bias trick gains over this (on A100); this entry point exists to
 * measure the same on B200.  The converted value is exact (|P_g| < 2^24), so
 * fl(float(P_g) * s_w) equals the bias-trick FMA and Y is bit-identical to
 * mixllm_gemm_w4w8a8's.  Same arguments, rules and errors.
 */
MIXLLM_API mixllm_status mixllm_gemm_w4w8a8_plain_i2f(const int8_t *A_q, const float *s_a, int64_t M, int64_t K,
                                 const uint8_t *W4, const uint8_t *z4, const void *s_w4_f16,
                                 const int32_t *idx4, int64_t N4,
                                 const int8_t *W8, const void *s_w8_f16,
                                 const int32_t *idx8, int64_t N8,
                                 void *Y_f16, void *stream);

/*
 * Bytes of workspace mixllm_gemm_w4w8a8_small_m needs for this shape (0 when
 * the shape is not split along K), in *bytes.  Pure host function.
 * Requires 1 <= M <= 64 and K a positive multiple of 128.
 */
MIXLLM_API mixllm_status mixllm_small_m_workspace_bytes(int64_t M, int64_t K, int64_t N4, int64_t N8,
                                             size_t *bytes);

/*
 * Which kernel mixllm_gemm_w4w8a8_small_m (and its _noalloc form) runs for a
 * shape, in *kind:
 *   MIXLLM_SMALL_M_TENSOR_CORE     9 <= M <= 64: int8 tensor-core tiles, split-K;
 *   MIXLLM_SMALL_M_GEMV_SPLIT      M <= 8: the GEMV, split-K over each tile's groups;
 *   MIXLLM_SMALL_M_GEMV_PERSISTENT M <= 4 with M*K <= 32768 and at least
 *                                  8 x 296 units of 32 KiB of weights: the
 *                                  GEMV with an even share of units per CTA.
 * Pure host function, with the arguments and errors of
 * mixllm_small_m_workspace_bytes (kind must not be NULL).  The pages have no
 * counterpart: it reports the library's own choice, for logs and benchmarks.
 */
typedef enum {
  MIXLLM_SMALL_M_TENSOR_CORE = 0,
  MIXLLM_SMALL_M_GEMV_SPLIT = 1,
  MIXLLM_SMALL_M_GEMV_PERSISTENT = 2
} mixllm_small_m_kind;
MIXLLM_API mixllm_status mixllm_small_m_kernel(int64_t M, int64_t K, int64_t N4, int64_t N8, int32_t *kind);

/*
 * The same layer and the same result rule as mixllm_gemm_w4w8a8, laid out
 * for few tokens (1 <= M <= 64, the decode regime, where the packed weights
 * are nearly all the bytes and HBM bandwidth bounds the layer).  For
 * 9 <= M <= 64 the weight tile is the tensor core's 128-row side and the
 * tokens its 16/32/64-column side; for M <= 8 a GEMV streams the packed
 * weights through shared memory and forms the exact int32 group partials
 * with dp4a (mixllm_small_m_kernel says which).  Either way the groups of
 * every 128-channel tile are split among several CTAs so the grid fills the
 * GPU: each part writes fp32 partial sums to the workspace, and the last one
 * of a tile to finish adds them in K order (the result does not depend on
 * timing) and writes Y.  The rounding differs from
 * mixllm_gemm_w4w8a8 only in the order of the fp32 operations (Y is within
 * the same tolerance of the reference definition).
 * Arguments: as mixllm_gemm_w4w8a8, plus
 *   workspace        device, at least mixllm_small_m_workspace_bytes() bytes,
 *                    16-byte aligned, owned by the caller: fp32 partial sums
 *                    followed by one int32 counter per 128-channel tile.  It
 *                    must be zero-filled before its first use; every call
 *                    returns the counters to zero (the partial sums are
 *                    scratch), so it stays ready for the next call.  Two calls
 *                    that run at the same time must not share one.  After a
 *                    MIXLLM_ERR_TIMEOUT zero it again.  May be NULL when the
 *                    size is 0.
 *   workspace_bytes  its size.
 * Asynchronous on `stream`.  Returns MIXLLM_ERR_INVALID_ARG for M > 64 or a
 * workspace that is too small.
 */
MIXLLM_API mixllm_status mixllm_gemm_w4w8a8_small_m(const int8_t *A_q, const float *s_a, int64_t M, int64_t K,
                                         const uint8_t *W4, const uint8_t *z4, const void *s_w4_f16,
                                         const int32_t *idx4, int64_t N4,
                                         const int8_t *W8, const void *s_w8_f16,
                                         const int32_t *idx8, int64_t N8,
                                         void *Y_f16, void *workspace, size_t workspace_bytes,
                                         void *stream);

/*
 * The whole few-token layer from fp16 activations: quantize_act and
 * mixllm_gemm_w4w8a8_small_m in one call, with the same result (the same
 * codes, scales and kernel arithmetic, so Y is bit-identical to the two calls).
 * For one token, where the plan runs the split GEMV and a CTA's slice of X
 * (groups x 256 bytes) fits one 32 KiB slot of its weight ring, the GEMV
 * quantizes that slice itself in its prologue (no A_q in HBM, one launch);
 * otherwise the activations are quantized into the workspace first (two
 * launches; with more tokens every CTA quantizing its own slice costs more
 * than the separate pass).
 * This fuses the activation quantization into the GEMM prologue for decode
 * (MLSys 2026 talk notes on MixLLM, notes.yuuk.io, §設計判断の概要 and
 * §二段階逆量子化による int8 Tensor Core 活用: the same two steps, without the
 * A_q round trip).
 *   X_f16      device fp16 [M, K] row-major, 16-byte aligned.
 *   workspace  device, at least mixllm_linear_small_m_workspace_bytes() bytes,
 *              256-byte aligned, zero-filled before its first use; calls
 *              leave its counters at zero (the rest is scratch); not shared by
 *              calls that run at the same time.
 * Other arguments, the M <= 64 bound and the errors: as
 * mixllm_gemm_w4w8a8_small_m.  Asynchronous on `stream`.
 */
MIXLLM_API mixllm_status mixllm_linear_small_m_workspace_bytes(int64_t M, int64_t K, int64_t N4, int64_t N8,
                                                               size_t *bytes);
MIXLLM_API mixllm_status mixllm_linear_small_m(const void *X_f16, int64_t M, int64_t K, const uint8_t *W4,
                                               const uint8_t *z4, const void *s_w4_f16, const int32_t *idx4,
                                               int64_t N4, const int8_t *W8, const void *s_w8_f16,
                                               const int32_t *idx8, int64_t N8, void *Y_f16, void *workspace,
                                               size_t workspace_bytes, void *stream);

/*
 * The whole layer from fp16 activations for any number of tokens: the
 * activation quantization and the fused W4.4A8 GEMM of the MLSys 2026 talk
 * notes on MixLLM (notes.yuuk.io, §設計判断の概要 for the quantizers,
 * §二段階逆量子化による int8 Tensor Core 活用 for the two-step GEMM).  The
 * codes, scales and Y are bit-identical to mixllm_quantize_act followed by
 * mixllm_gemm_w4w8a8 (M > 64) or mixllm_gemm_w4w8a8_small_m (M <= 64).
 * For M <= 64 this is mixllm_linear_small_m.  For M > 64 the quantizer
 * writes A_q and s_a into the workspace and the tiled GEMM runs as its
 * programmatic dependent (its prologue and weight copies overlap the
 * quantizer): two launches.
 *   X_f16      device fp16 [M, K] row-major, 16-byte aligned.
 *   workspace  device, at least mixllm_linear_workspace_bytes() bytes,
 *              256-byte aligned, owned by the caller.  For M > 64 it holds
 *              A_q [M, K] int8, then s_a [M, K/128] fp32, then two uint32
 *              counters (each part 256-byte aligned).  It must be zero-filled
 *              before its first use; every call returns the counters to zero
 *              (A_q and s_a are scratch, left holding this call's codes), so
 *              it stays ready.  Two calls that run at the same time must not
 *              share one.  After MIXLLM_ERR_TIMEOUT zero it again.
 *   workspace_bytes  its size.
 * Other arguments: as mixllm_gemm_w4w8a8.  Asynchronous on `stream`.
 * Errors: MIXLLM_ERR_INVALID_ARG for bad sizes, pointers or alignment, or a
 * workspace that is too small; MIXLLM_ERR_TIMEOUT (reported by
 * mixllm_sync_status) if a device-side wait gave up.
 */
MIXLLM_API mixllm_status mixllm_linear_workspace_bytes(int64_t M, int64_t K, int64_t N4, int64_t N8, size_t *bytes);
MIXLLM_API mixllm_status mixllm_linear(const void *X_f16, int64_t M, int64_t K, const uint8_t *W4, const uint8_t *z4,
                                       const void *s_w4_f16, const int32_t *idx4, int64_t N4, const int8_t *W8,
                                       const void *s_w8_f16, const int32_t *idx8, int64_t N8, void *Y_f16,
                                       void *workspace, size_t workspace_bytes, void *stream);

/*
 * mixllm_linear for M > 64 as ONE launch: the tiled GEMM quantizes X itself
 * (the pages' two steps with no A_q pass between kernels: MLSys 2026 talk
 * notes on MixLLM, §二段階逆量子化による int8 Tensor Core 活用; the
 * awesome-system-papers summary, 核心方法).  Every CTA first quantizes an even
 * share of the (token, group) pairs into the workspace, with all of its
 * threads and the quantizer's own arithmetic, and adds its count to a
 * counter there; each CTA loads A_q and s_a only once the count is
 * complete, and the last CTA to finish returns the counters to zero.
 * Same result, bit for bit, as mixllm_linear.  The quantization then runs
 * at one CTA per SM on the GEMM's critical path, which on B200 costs more
 * than the separate quantizer whose tail the GEMM's prologue overlaps; the
 * entry point is kept to measure that choice.
 * Arguments, workspace and errors: as mixllm_linear, plus
 * MIXLLM_ERR_INVALID_ARG for 1 <= M <= 64 and MIXLLM_ERR_UNSUPPORTED when
 * K / 128 is not a multiple of 4 or M * K / 128 reaches 2^31.  All of the
 * grid's CTAs must be resident at once (one per SM, at most one per SM of
 * the device); a device-side wait that gives up is reported by
 * mixllm_sync_status as MIXLLM_ERR_TIMEOUT.
 */
MIXLLM_API mixllm_status mixllm_linear_one_launch(const void *X_f16, int64_t M, int64_t K, const uint8_t *W4,
                                                  const uint8_t *z4, const void *s_w4_f16, const int32_t *idx4,
                                                  int64_t N4, const int8_t *W8, const void *s_w8_f16,
                                                  const int32_t *idx8, int64_t N8, void *Y_f16, void *workspace,
                                                  size_t workspace_bytes, void *stream);

/*
 * mixllm_gemm_w4w8a8_small_m without a workspace argument and without any
 * allocation: the split partial sums and tile counters live in a fixed 8 MiB
 * scratch array in the library's static device memory (one per device,
 * created with the module).  An engineering variant for callers that cannot
 * hand over device memory; the paper has no counterpart.  Same arguments,
 * result and rounding as mixllm_gemm_w4w8a8_small_m otherwise.
 *   * The tile counters are cleared on `stream` before every launch (an
 *     asynchronous memset of the scratch, no allocation).
 *   * Calls that overlap in time on one device share the scratch and race:
 *     issue them to one stream, or order them with events.
 *   * The scratch used is the current device's (cudaGetDevice at the call):
 *     `stream` must belong to that device (or be NULL, its legacy default
 *     stream); a stream of another device is not detected and the kernel
 *     would read another device's memory.
 *   * Returns MIXLLM_ERR_UNSUPPORTED when the shape needs more scratch than
 *     the array holds (see mixllm_small_m_workspace_bytes), and
 *     MIXLLM_ERR_INVALID_ARG for M > 64.
 * Asynchronous on `stream`.
 */
MIXLLM_API mixllm_status mixllm_gemm_w4w8a8_small_m_noalloc(const int8_t *A_q, const float *s_a, int64_t M,
                                                 int64_t K, const uint8_t *W4, const uint8_t *z4,
                                                 const void *s_w4_f16, const int32_t *idx4, int64_t N4,
                                                 const int8_t *W8, const void *s_w8_f16,
                                                 const int32_t *idx8, int64_t N8,
                                                 void *Y_f16, void *stream);

/*
 * Debug form of one named few-token kernel, for parity tests: runs the kernel
 * `kind` (a mixllm_small_m_kind) whatever mixllm_small_m_kernel would pick,
 * and writes both Y (as mixllm_gemm_w4w8a8_small_m would with that kernel)
 * and the per-group int32 partials of step 2 of the two-step dequantization
 * (MLSys 2026 talk notes on MixLLM, §二段階逆量子化)
 *   P[m, idx[n], g] = sum_{k in g} (W_q[n,k] - z[n,g]) * A_q[m,k]
 * into
 *   P          device, int32 [M, N4 + N8, K/128], 4-byte aligned, written
 *              for every m < M and every listed column.
 *   workspace  device, 16-byte aligned, at least
 *              mixllm_small_m_debug_workspace_bytes(.., kind, ..) bytes,
 *              zero-filled before its first use (calls leave it so).
 * Which kinds a shape allows: the tensor-core kernel any 1 <= M <= 64; the
 * split GEMV M <= 8; the persistent GEMV M <= 4 with M*K <= 32768 (rounded
 * up to 1, 2, 4 tokens).  Other kinds return MIXLLM_ERR_UNSUPPORTED.  Other
 * arguments and errors: as mixllm_gemm_w4w8a8_small_m.  Slow (uncoalesced
 * stores of P); asynchronous on `stream`.
 */
MIXLLM_API mixllm_status mixllm_small_m_debug_workspace_bytes(int64_t M, int64_t K, int64_t N4, int64_t N8,
                                                   int32_t kind, size_t *bytes);
MIXLLM_API mixllm_status mixllm_small_m_debug_partials(const int8_t *A_q, const float *s_a, int64_t M, int64_t K,
                                            const uint8_t *W4, const uint8_t *z4, const void *s_w4_f16,
                                            const int32_t *idx4, int64_t N4, const int8_t *W8,
                                            const void *s_w8_f16, const int32_t *idx8, int64_t N8,
                                            int32_t kind, int32_t *P, void *Y_f16, void *workspace,
                                            size_t workspace_bytes, void *stream);

/*
 * Global mixed-precision search, step 1 (MLSys 2026 talk notes on MixLLM,
 * notes.yuuk.io, §グローバル混合精度探索): the salience of every output channel
 * n of one linear layer,
 *   S[n] = (1/D) sum_d | t_d + t_d^2 / 2 |,  t_d = sum_k G[d, n, k] (c_q - c_0)[n, k],
 * the loss change of quantizing channel n alone to second order, with the
 * Hessian approximated by the Fisher matrix.  c_0 is the channel's weights and
 * c_q their 4-bit asymmetric group quantization (the one
 * mixllm_pack_weights applies), dequantized as s * (q - z).
 *   W   device fp32 [N, K] row-major, 16-byte aligned (the layer's weights).
 *   G   device fp32 [D, N, K], 16-byte aligned: G[d, n, :] is the gradient of
 *       the loss on calibration sample d with respect to channel n's weights.
 *   S   device fp32 [N], written.
 * K a positive multiple of 128 up to 56832 (the row of c_q - c_0 is held in
 * shared memory); D >= 1.  fp32 arithmetic in a fixed order: the result is
 * deterministic and within the rounding of an fp32 dot product of the exact
 * value.  Asynchronous on `stream`; the caller owns every buffer.
 */
MIXLLM_API mixllm_status mixllm_channel_salience(const float *W, int64_t N, int64_t K, const float *G, int64_t D,
                                                 float *S, void *stream);

/* Workspace bytes of mixllm_select_top_t for n scores.  Pure host function. */
MIXLLM_API mixllm_status mixllm_select_top_t_workspace_bytes(int64_t n, size_t *bytes);

/*
 * Global mixed-precision search, step 2 (Algorithm 1 of the same notes): the
 * scores of all channels of all layers in one list S (device fp32 [n], no
 * NaN; the concatenation order is the caller's); is8[i] = 1 for the T
 * largest, 0 for the rest (device uint8 [n], written).  Equal scores are
 * taken in list order (the lower index first), so the result is unique; -0
 * and +0 are equal.  0 <= T <= n.  workspace: device, at least
 * mixllm_select_top_t_workspace_bytes(n) bytes, 16-byte aligned, no
 * initialisation needed; not shared by calls that run at the same time.
 * Asynchronous on `stream` (a radix select on the device, no host round trip).
 */
MIXLLM_API mixllm_status mixllm_select_top_t(const float *S, int64_t n, int64_t T, uint8_t *is8, void *workspace,
                                             size_t workspace_bytes, void *stream);

/*
 * Waits for `stream`, then reads and clears the device status word of the
 * current device.  Returns MIXLLM_ERR_TIMEOUT if a kernel of this library
 * gave up a wait since the last call, MIXLLM_ERR_BOUNDS if (checked build
 * only) a range check failed, MIXLLM_ERR_CUDA if the stream reports a CUDA
 * error, MIXLLM_OK otherwise.  SYNCHRONOUS.
 */
MIXLLM_API mixllm_status mixllm_sync_status(void *stream);

/*
 * Self-test of the hang guard: launches one small kernel whose wait on a
 * shared-memory barrier that nothing signals gives up after `limit_us`
 * microseconds (1..1000000) and records MIXLLM_ERR_TIMEOUT in the device
 * status word, leaving the context usable.  Asynchronous; read the result
 * with mixllm_sync_status().
 */
MIXLLM_API mixllm_status mixllm_selftest_wait_timeout(uint32_t limit_us, void *stream);

/*
 * 1 if this is the checked build of the library (every tensor- and
 * shared-memory access of the GEMM kernels is range-checked first; a failed
 * check skips the access and records MIXLLM_ERR_BOUNDS), 0 for the release
 * build.  Pure host function.
 */
MIXLLM_API int mixllm_checked_build(void);

/*
 * Self-test of the checked build's range checks: launches one small kernel
 * that checks a tensor-memory column range and a shared-memory range which
 * both lie outside their windows (no access is made), so a checked build
 * records MIXLLM_ERR_BOUNDS in the device status word.  The release build
 * returns MIXLLM_ERR_UNSUPPORTED and launches nothing.  Asynchronous; read
 * the result with mixllm_sync_status().
 */
MIXLLM_API mixllm_status mixllm_selftest_bounds(void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MIXLLM_H_ */

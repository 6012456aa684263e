// quant.cuh -- activation quantization, offline weight pack, and the
// hang-guard self-test kernel.
//
// Sources: MLSys 2026 talk notes on MixLLM (notes.yuuk.io), §設計判断の概要
// (activations 8-bit symmetric group-wise RTN; weights 4-bit asymmetric with
// group 128, salient channels 8-bit symmetric) and §ソフトウェアパイプライン
// (weights packed and interleaved offline so no permutation runs at run time).
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

#include "launch.h"
#include "ptx_sm100.cuh"

namespace mixllm {

// ---------------------------------------------------------------------------
// Activation quantization.  One half-warp per (token m, group g): 16 lanes x
// 8 fp16 = the 128 values of the group, loaded as one 16-byte vector per lane.
// amax over the group, s_a = amax / 127 (IEEE division in fp32, kept as fp32),
// q = clamp(round_half_even(x / s_a), -127, 127) with x / s_a the IEEE fp32
// quotient; amax == 0 gives s_a = q = 0.
//
// The codes are those of rint(fl(x / s)), the plain CPU evaluation of the
// definition, with an IEEE division only for the rare element that needs it:
//   * q0 = rint(x * (1/s)) is within one of rint(x/s): the product is off
//     from the quotient by at most ~2^-23 of it (below 2^-16 for |x/s| < 128);
//   * e = fma(-q0, s, x) = x - q0*s exactly: x is an fp16 value and q0*s has
//     at most 8 + 24 significant bits; when q0 != 0, |x| >= s/2 puts x's last
//     place above s's, so e is a multiple of s's last place and below s in
//     magnitude -- 24 bits suffice;
//   * the exact quotient is q0 + e/s.  fl(x/s) differs from it by at most half
//     an ulp, 2^-18 for quotients below 128, so rint(fl(x/s)) = rint(x/s)
//     unless the quotient lies within 2^-18 of a half-integer.  Away from
//     those (| |e| - s/2 | > 2^-14 s, a wide margin) the code is q0, or q0
//     moved one step toward e when |e| > s/2; within the margin (rare for real
//     data, every tie case of the tests) the element takes the IEEE division.
// ---------------------------------------------------------------------------
// One group of 128 activations held eight per lane by the 16 lanes of `mask`
// (MLSys 2026 talk notes on MixLLM, notes.yuuk.io, §設計判断の概要: 8-bit
// symmetric, group-wise RTN): s_a = amax / 127 (IEEE division), codes
// rne(x / s_a) clamped to +-127 (an all-zero group gives s_a = 0 and zero
// codes), computed as described above.  `raw`: the lane's eight fp16 values;
// the codes are returned packed, lowest k first; returns s_a.  Shared by
// quantize_act_kernel and the fused decode GEMV.
__device__ __forceinline__ float quant_act_8x16(const uint4 raw, unsigned mask, uint32_t (&packed)[2]) {
  // the eight values stay packed as fp16 pairs and are widened where used
  const __half2 *h2 = reinterpret_cast<const __half2 *>(&raw);
  auto xval = [&](int i) {
    const float2 f = __half22float2(h2[i >> 1]);
    return (i & 1) ? f.y : f.x;
  };
  __half2 m2 = __habs2(h2[0]);
#pragma unroll
  for (int i = 1; i < 4; ++i) m2 = __hmax2(m2, __habs2(h2[i]));
  float amax = fmaxf(__low2float(m2), __high2float(m2));
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(mask, amax, o));
  const float s = __fdiv_rn(amax, 127.0f);
  packed[0] = packed[1] = 0u;
  if (s != 0.0f) {
    // Integers below 2^22 in magnitude are rounded and converted with the
    // 1.5*2^23 offset: fl(t + 1.5*2^23) - 1.5*2^23 is rint(t) (ties to even,
    // the default rounding of the add), and the bits of fl(q + 1.5*2^23) are
    // 0x4b400000 + q.  The explicit _rn intrinsics keep the compiler from
    // fusing the multiply into the add.
    constexpr float kMagic = 12582912.0f;
    const float r = __frcp_rn(s);
    const float half_s = 0.5f * s;
    const float margin = s * 0x1p-14f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float xi = xval(i);
      const float q0 = __fadd_rn(__fadd_rn(__fmul_rn(xi, r), kMagic), -kMagic);  // rint(fl(x * (1/s)))
      const float e = __fmaf_rn(-q0, s, xi);  // exact remainder x - q0*s
      const float d = fabsf(e) - half_s;
      float qf;
      if (fabsf(d) > margin) {
        qf = d > 0.0f ? q0 + (e > 0.0f ? 1.0f : -1.0f) : q0;
      } else {
        // near a half-integer: the IEEE quotient, rounded
        qf = __fadd_rn(__fadd_rn(__fdiv_rn(xi, s), kMagic), -kMagic);
      }
      qf = fminf(127.0f, fmaxf(-127.0f, qf));
      const uint32_t qi = static_cast<uint32_t>(__float_as_int(__fadd_rn(qf, kMagic)) - 0x4b400000);
      packed[i >> 2] |= (qi & 0xFFu) << ((i & 3) * 8);
    }
  }
  return s;
}

// One half-warp per (token, group): 16 lanes x one 16-byte load.  The grid
// is one wave of 8 blocks per SM where the layer allows (the register bound
// below), so every load of a layer's activations is in flight at once and
// the kernel costs about one load round trip.  I: the index type (32-bit
// when M*K fits, which keeps the kernel within that bound).
constexpr int kQuantThreads = 256;

template <typename I>
__global__ void __launch_bounds__(kQuantThreads, sizeof(I) == 4 ? 8 : 1) quantize_act_kernel(const __half *__restrict__ X, I M, I K,
                                                                        int8_t *__restrict__ A_q,
                                                                        float *__restrict__ s_a) {
  // the GEMM that consumes A_q and s_a may start its prologue now; it reads
  // them only after this grid has completed
  pdl_launch_dependents();
  const I G = K >> 7;
  const I total = M * G;
  const int lane16 = threadIdx.x & 15;
  const unsigned mask = 0xFFFFu << (threadIdx.x & 16);
  const I stride = (static_cast<I>(gridDim.x) * blockDim.x) >> 4;
  for (I hw = (static_cast<I>(blockIdx.x) * blockDim.x + threadIdx.x) >> 4; hw < total; hw += stride) {
    const I m = hw / G, g = hw - m * G;
    const I off = m * K + (g << 7) + lane16 * 8;
    const uint4 raw = *reinterpret_cast<const uint4 *>(X + off);
    uint32_t packed[2];
    const float s = quant_act_8x16(raw, mask, packed);
    *reinterpret_cast<uint2 *>(A_q + off) = make_uint2(packed[0], packed[1]);
    if (lane16 == 0) s_a[hw] = s;  // s_a[m, g] is element m*G + g = hw
  }
}

// ---------------------------------------------------------------------------
// Channel split: one block scans the bit map and lists the 8-bit channels and
// the 4-bit channels, each in ascending order.  Writes stay inside idx8[N8]
// and idx4[N - N8] even if the map holds a different count, which is then
// recorded in the status word.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) split_channels_kernel(const uint8_t *__restrict__ is8, int64_t N, int64_t N8,
                                                              int32_t *__restrict__ idx4, int32_t *__restrict__ idx8) {
  __shared__ int warp_cnt[32];
  __shared__ int warp_off[32];
  __shared__ int64_t seen8;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) seen8 = 0;
  __syncthreads();
  for (int64_t start = 0; start < N; start += 1024) {
    const int64_t n = start + tid;
    const int f = (n < N && is8[n] != 0) ? 1 : 0;
    const unsigned b = __ballot_sync(0xFFFFFFFFu, f);
    const int before_in_warp = __popc(b & ((1u << lane) - 1u));
    if (lane == 0) warp_cnt[warp] = __popc(b);
    __syncthreads();
    if (warp == 0) {
      const int c = warp_cnt[lane];
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += v;
      }
      warp_off[lane] = incl - c;
    }
    __syncthreads();
    const int64_t pre8 = seen8 + warp_off[warp] + before_in_warp;  // 8-bit channels before n
    if (n < N) {
      if (f) {
        if (pre8 < N8) idx8[pre8] = static_cast<int32_t>(n);
      } else {
        const int64_t pre4 = n - pre8;
        if (pre4 < N - N8) idx4[pre4] = static_cast<int32_t>(n);
      }
    }
    __syncthreads();
    if (tid == 0) seen8 += warp_off[31] + warp_cnt[31];
    __syncthreads();
  }
  if (tid == 0 && seen8 != N8) record_status(kStatusBadBitmap);
}

__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

// ---------------------------------------------------------------------------
// The 4-bit asymmetric quantizer of one group (MLSys 2026 talk notes on MixLLM,
// notes.yuuk.io, §設計判断の概要: 4-bit asymmetric, group 128), given the
// group's range lo = min(0, min w), hi = max(0, max w): scale
// fp16(min((hi - lo) / 15, 65504)) (IEEE division), zero point
// clamp(rne(-lo / s), 0, 15), code clamp(rne(w / s) + z, 0, 15); a zero scale
// gives z = q = 0.  Shared by the packer and the channel-salience search.
// ---------------------------------------------------------------------------
struct W4Params {
  __half sh;  // the scale as stored
  float sf;   // the same as fp32
  int z;
};
__device__ __forceinline__ W4Params w4_params(float lo, float hi) {
  W4Params p;
  const float sc = fminf(__fdiv_rn(__fsub_rn(hi, lo), 15.0f), 65504.0f);
  p.sh = __float2half_rn(sc);
  p.sf = __half2float(p.sh);
  p.z = p.sf != 0.0f ? max(0, min(15, __float2int_rn(__fdiv_rn(-lo, p.sf)))) : 0;
  return p;
}
__device__ __forceinline__ int w4_code(float v, const W4Params &p) {
  return p.sf != 0.0f ? max(0, min(15, __float2int_rn(__fdiv_rn(v, p.sf)) + p.z)) : 0;
}

// ---------------------------------------------------------------------------
// 4-bit asymmetric pack.  One warp per (pair of packed rows, group): the two
// rows share the zero-point byte.  The codes of row r, group g go to the
// 64-byte row r % 128 of block (r / 128, g) -- each 128-channel tile's group
// is one contiguous 8 KB block, loaded by the GEMM with a single bulk copy --
// and lane l writes bytes 2l and 2l+1 of it: byte b = 16c + i of a 32-k run c
// holds codes k = 32c + i (low nibble) and k = 32c + 16 + i (high nibble).
// Rows of the last tile past N4 are written as zeros.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) pack_w4_kernel(const float *__restrict__ W, int64_t N, int64_t K,
                                                      const int32_t *__restrict__ idx4, int64_t N4, int64_t N4p,
                                                      uint8_t *__restrict__ W4, uint8_t *__restrict__ z4,
                                                      __half *__restrict__ s_w4) {
  const int64_t G = K >> 7;
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= (N4p >> 1) * G) return;
  const int64_t p = wid / G, g = wid - p * G;
  uint32_t zpair = 0;
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int64_t r = 2 * p + e;
    // a channel index outside [0, N) (a bit map that disagrees with N8) packs as zeros
    const int64_t n = r < N4 ? static_cast<int64_t>(idx4[r]) : -1;
    if (r < N4) {
      const float *w = W + (n >= 0 && n < N ? n : 0) * K + (g << 7);
      const float keep = (n >= 0 && n < N) ? 1.0f : 0.0f;
      const int c = lane >> 3, i0 = (2 * lane) & 15;
      const float v[4] = {keep * w[32 * c + i0], keep * w[32 * c + 16 + i0], keep * w[32 * c + i0 + 1],
                          keep * w[32 * c + 16 + i0 + 1]};
      float lo = 0.0f, hi = 0.0f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        lo = fminf(lo, v[i]);
        hi = fmaxf(hi, v[i]);
      }
      lo = warp_min(lo);
      hi = warp_max(hi);
      const W4Params wp = w4_params(lo, hi);
      const __half sh = wp.sh;
      const int z = wp.z;
      uint32_t q[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) q[i] = static_cast<uint32_t>(w4_code(v[i], wp));
      const uint32_t two = (q[0] | (q[1] << 4)) | ((q[2] | (q[3] << 4)) << 8);
      *reinterpret_cast<uint16_t *>(W4 + (((r >> 7) * G + g) * 128 + (r & 127)) * 64 + 2 * lane) =
          static_cast<uint16_t>(two);
      if (lane == 0) s_w4[g * N4p + r] = sh;
      zpair |= static_cast<uint32_t>(z) << (4 * e);
    } else {
      if (r < ((N4 + 127) & ~int64_t(127)))  // padding row of the last tile
        *reinterpret_cast<uint16_t *>(W4 + (((r >> 7) * G + g) * 128 + (r & 127)) * 64 + 2 * lane) = 0;
      if (lane == 0) s_w4[g * N4p + r] = __float2half_rn(0.0f);
    }
  }
  if (lane == 0) z4[g * (N4p >> 1) + p] = static_cast<uint8_t>(zpair);
}

// ---------------------------------------------------------------------------
// 8-bit symmetric pack.  One warp per (row, group); lane l quantizes k = 4l..4l+3.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) pack_w8_kernel(const float *__restrict__ W, int64_t N, int64_t K,
                                                      const int32_t *__restrict__ idx8, int64_t N8, int64_t N8p,
                                                      int8_t *__restrict__ W8, __half *__restrict__ s_w8) {
  const int64_t G = K >> 7;
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= N8p * G) return;
  const int64_t r = wid / G, g = wid - r * G;
  if (r >= N8) {
    if (lane == 0) s_w8[g * N8p + r] = __float2half_rn(0.0f);
    return;
  }
  const int64_t n = idx8[r];
  const bool n_ok = n >= 0 && n < N;  // an index outside [0, N) packs as zeros
  const float4 v4 = n_ok ? *reinterpret_cast<const float4 *>(W + n * K + (g << 7) + 4 * lane)
                         : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  const float v[4] = {v4.x, v4.y, v4.z, v4.w};
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) amax = fmaxf(amax, fabsf(v[i]));
  amax = warp_max(amax);
  const float sc = fminf(__fdiv_rn(amax, 127.0f), 65504.0f);
  const __half sh = __float2half_rn(sc);
  const float sf = __half2float(sh);
  uint32_t packed = 0;
  if (sf != 0.0f) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int q = max(-127, min(127, __float2int_rn(__fdiv_rn(v[i], sf))));
      packed |= (static_cast<uint32_t>(q) & 0xFFu) << (8 * i);
    }
  }
  *reinterpret_cast<uint32_t *>(W8 + r * K + (g << 7) + 4 * lane) = packed;
  if (lane == 0) s_w8[g * N8p + r] = sh;
}

// ---------------------------------------------------------------------------
// Hang-guard self-test: thread 0 waits on a barrier that nothing signals; the
// bounded wait gives up and records a timeout.  No copy or MMA is in flight.
// ---------------------------------------------------------------------------
__global__ void selftest_wait_kernel(long long limit_cycles) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, &abort_flag, limit_cycles);
  __syncthreads();
}

int64_t padded_channels(int64_t n) { return (n + 255) / 256 * 256; }

static int grid_for(int64_t threads_needed, int block) {
  const int64_t b = (threads_needed + block - 1) / block;
  return static_cast<int>(b < 1 ? 1 : (b > (1ll << 30) ? (1ll << 30) : b));
}

cudaError_t launch_quantize_act(const void *X, int64_t M, int64_t K, int8_t *A_q, float *s_a, cudaStream_t stream) {
  const int64_t groups = M * (K >> 7);
  constexpr int kPerBlock = kQuantThreads / 16;  // groups per block and pass
  const int64_t blocks = (groups + kPerBlock - 1) / kPerBlock;
  const int grid = static_cast<int>(blocks < 148 * 64 ? blocks : 148 * 64);
  if (M * K < (int64_t{1} << 31))
    quantize_act_kernel<uint32_t><<<grid, kQuantThreads, 0, stream>>>(
        static_cast<const __half *>(X), static_cast<uint32_t>(M), static_cast<uint32_t>(K), A_q, s_a);
  else
    quantize_act_kernel<int64_t><<<grid, kQuantThreads, 0, stream>>>(static_cast<const __half *>(X), M, K, A_q, s_a);
  return cudaGetLastError();
}

cudaError_t launch_split_channels(const uint8_t *is8, int64_t N, int64_t N8, int32_t *idx4, int32_t *idx8,
                                  cudaStream_t stream) {
  split_channels_kernel<<<1, 1024, 0, stream>>>(is8, N, N8, idx4, idx8);
  return cudaGetLastError();
}

cudaError_t launch_pack_w4(const float *W, int64_t N, int64_t K, const int32_t *idx4, int64_t N4, int64_t N4p,
                           uint8_t *W4, uint8_t *z4, void *s_w4, cudaStream_t stream) {
  const int64_t warps = (N4p / 2) * (K >> 7);
  pack_w4_kernel<<<grid_for(warps * 32, 256), 256, 0, stream>>>(W, N, K, idx4, N4, N4p, W4, z4,
                                                                 static_cast<__half *>(s_w4));
  return cudaGetLastError();
}

cudaError_t launch_pack_w8(const float *W, int64_t N, int64_t K, const int32_t *idx8, int64_t N8, int64_t N8p,
                           int8_t *W8, void *s_w8, cudaStream_t stream) {
  const int64_t warps = N8p * (K >> 7);
  pack_w8_kernel<<<grid_for(warps * 32, 256), 256, 0, stream>>>(W, N, K, idx8, N8, N8p, W8,
                                                                 static_cast<__half *>(s_w8));
  return cudaGetLastError();
}

// The checked build's range checks on ranges that lie outside their windows:
// one column past a 32-column allocation, lanes 112..143, and 16 bytes that
// straddle the end of the dynamic shared memory.  Nothing is accessed.
__global__ void selftest_bounds_kernel(uint32_t tmem_base) {
  extern __shared__ uint8_t dyn[];
  const uint32_t lo = smem_u32(dyn), hi = lo + 256;
  bool ok = chk_tmem(tmem_base + 1, tmem_base, 32, 32);
  ok = chk_tmem(tmem_base + (112u << 16), tmem_base, 32, 1) && ok;
  ok = chk_smem(hi - 8, 16, lo, hi) && ok;
  if (ok && threadIdx.x == 0) record_status(kStatusBadBitmap);  // unreachable in a checked build
}

cudaError_t launch_selftest_bounds(cudaStream_t stream) {
  selftest_bounds_kernel<<<1, 32, 256, stream>>>(0u);
  return cudaGetLastError();
}

cudaError_t launch_selftest_wait_timeout(uint32_t limit_us, cudaStream_t stream) {
  // SM clocks stay below 2.1 GHz, so 2100 cycles per microsecond is an upper bound.
  selftest_wait_kernel<<<1, 32, 0, stream>>>(static_cast<long long>(limit_us) * 2100ll);
  return cudaGetLastError();
}

}  // namespace mixllm

// search.cuh -- the global mixed-precision search of MixLLM on sm_100a.
//
// MLSys 2026 talk notes on MixLLM (notes.yuuk.io), §グローバル混合精度探索 and
// its Algorithm 1: the salience of output channel c is the loss change of
// quantizing that channel alone, expanded to second order with the Fisher
// approximation of the Hessian,
//     S_c = (1/|D|) sum_d | g_d^T (c_q - c_0) + 1/2 (g_d^T (c_q - c_0))^2 |,
// with g_d the gradient of the loss on calibration sample d with respect to the
// channel's weights; the channels of all layers are then sorted by S in
// descending order and the first T get 8 bits.  c_q is the channel's 4-bit
// asymmetric group quantization (the packer's quantizer, dequantized as
// s * (q - z)).
//
// channel_salience_kernel: one CTA per output channel.  It forms c_q - c_0 for
// the whole row in shared memory (one warp per group of 128), then streams
// the channel's D gradient rows from HBM -- nearly all the bytes -- four or
// eight rows at a time with 16-byte loads, each thread summing its slice of every row in
// a fixed order and the block reducing the rows by a fixed tree, so the
// result is deterministic.
//
// Top-T: a radix select on order-preserving integer keys of the scores (four
// passes of 8 bits, most significant first, each a histogram over the keys
// that match the digits chosen so far and a one-block pick of the next
// digit) finds the key tau of the T-th largest score and how many of the
// scores equal to tau are taken; those are the first in index order (a
// per-chunk count, a one-block scan of the counts, and a marking pass).
// Everything stays on the device: no host round trip between the passes.
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

#include "launch.h"
#include "ptx_sm100.cuh"
#include "quant.cuh"

namespace mixllm {

// Two shapes, picked by K (measured on B200, 16 gradient rows per channel):
// 256 threads reducing 4 rows at a time for K <= 8192 (4.8-5.2 TB/s at
// K = 4096), 512 threads and 8 rows for longer rows, whose shared-memory
// copy of c_q - c_0 leaves fewer CTAs per SM (5.6 TB/s at K = 14336 against 3.5).
constexpr int kSalKSmall = 8192;

__device__ __forceinline__ float4 ld_stream_f4(const float *p) {
  float4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// W fp32 [N, K], G fp32 [D, N, K] (16-byte aligned), S fp32 [N].
// Dynamic shared memory: K floats (c_q - c_0 of the channel).
template <int kSalThreads, int kSalRows>
__global__ void __launch_bounds__(kSalThreads) channel_salience_kernel(const float *__restrict__ W, int64_t N,
                                                                       int64_t K, const float *__restrict__ G,
                                                                       int64_t D, float *__restrict__ S) {
  extern __shared__ float4 delta4[];  // [K / 4]
  __shared__ float red[kSalRows][kSalThreads / 32];
  const int64_t n = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int groups = static_cast<int>(K >> 7);
  const float *w = W + n * K;

  // c_q - c_0 of every group: one warp per group, four weights per lane
  for (int g = warp; g < groups; g += kSalThreads / 32) {
    const float4 v4 = *reinterpret_cast<const float4 *>(w + g * 128 + lane * 4);
    const float v[4] = {v4.x, v4.y, v4.z, v4.w};
    float lo = 0.0f, hi = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      lo = fminf(lo, v[i]);
      hi = fmaxf(hi, v[i]);
    }
    const W4Params p = w4_params(warp_min(lo), warp_max(hi));
    float d[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)  // s * (q - z) is exact in fp32 (11 x 5 bits); one rounding in the difference
      d[i] = __fsub_rn(__fmul_rn(p.sf, static_cast<float>(w4_code(v[i], p) - p.z)), v[i]);
    delta4[g * 32 + lane] = make_float4(d[0], d[1], d[2], d[3]);
  }
  __syncthreads();

  // t_d = sum_k G[d, n, k] (c_q - c_0)[k], kSalRows rows at a time
  const int K4 = static_cast<int>(K >> 2);
  float acc = 0.0f;  // thread 0: sum_d |t_d + t_d^2 / 2|, d ascending
  for (int64_t d0 = 0; d0 < D; d0 += kSalRows) {
    float part[kSalRows];
#pragma unroll
    for (int r = 0; r < kSalRows; ++r) part[r] = 0.0f;
#pragma unroll 2
    for (int j = threadIdx.x; j < K4; j += kSalThreads) {
      const float4 dl = delta4[j];
      float4 gv[kSalRows];
#pragma unroll
      for (int r = 0; r < kSalRows; ++r)
        gv[r] = d0 + r < D ? ld_stream_f4(G + ((d0 + r) * N + n) * K + 4 * j) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int r = 0; r < kSalRows; ++r) {
        part[r] = __fmaf_rn(gv[r].x, dl.x, part[r]);
        part[r] = __fmaf_rn(gv[r].y, dl.y, part[r]);
        part[r] = __fmaf_rn(gv[r].z, dl.z, part[r]);
        part[r] = __fmaf_rn(gv[r].w, dl.w, part[r]);
      }
    }
#pragma unroll
    for (int r = 0; r < kSalRows; ++r) {
      const float v = warp_sum_f(part[r]);
      if (lane == 0) red[r][warp] = v;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      for (int r = 0; r < kSalRows && d0 + r < D; ++r) {
        float t = 0.0f;
#pragma unroll
        for (int q = 0; q < kSalThreads / 32; ++q) t += red[r][q];
        acc += fabsf(__fmaf_rn(0.5f * t, t, t));
      }
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) S[n] = __fdiv_rn(acc, static_cast<float>(D));
}

// ---------------------------------------------------------------------------
// top-T selection
// ---------------------------------------------------------------------------

// Order-preserving key of a score: a larger float gives a larger key; -0 and
// +0 give the same key (they compare equal).  NaN scores are not supported.
__device__ __forceinline__ uint32_t score_key(float s) {
  uint32_t u = __float_as_uint(s);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct SelState {
  uint32_t prefix, mask;       // the digits of tau chosen so far
  long long remaining;         // how many keys matching them are still to take
  unsigned long long hist[256];
};

constexpr int kSelChunk = 1024;  // scores per marking block (256 threads x 4)

__global__ void select_init_kernel(SelState *st, long long T) {
  st->hist[threadIdx.x] = 0;
  if (threadIdx.x == 0) {
    st->prefix = 0;
    st->mask = 0;
    st->remaining = T;
  }
}

// histogram of the digit at `shift` over the keys that match the chosen digits
__global__ void __launch_bounds__(256) select_hist_kernel(const float *__restrict__ S, int64_t n, SelState *st,
                                                          int shift) {
  __shared__ unsigned int h[256];
  h[threadIdx.x] = 0;
  __syncthreads();
  const uint32_t prefix = st->prefix, mask = st->mask;
  for (int64_t i = blockIdx.x * 256ll + threadIdx.x; i < n; i += static_cast<int64_t>(gridDim.x) * 256) {
    const uint32_t u = score_key(S[i]);
    if ((u & mask) == prefix) atomicAdd(&h[(u >> shift) & 255u], 1u);
  }
  __syncthreads();
  if (h[threadIdx.x]) atomicAdd(&st->hist[threadIdx.x], static_cast<unsigned long long>(h[threadIdx.x]));
}

// the digit of tau at `shift`: scanning the bins from the top, the bin where
// the count of larger keys first reaches `remaining` (the bins are read into
// shared memory by all threads first, then scanned by one)
__global__ void select_pick_kernel(SelState *st, int shift) {
  __shared__ unsigned long long h[256];
  h[threadIdx.x] = st->hist[threadIdx.x];
  st->hist[threadIdx.x] = 0;  // ready for the next pass
  __syncthreads();
  if (threadIdx.x == 0) {
    long long above = 0;
    int b = 255;
    for (; b > 0; --b) {
      const long long c = static_cast<long long>(h[b]);
      if (above + c >= st->remaining) break;
      above += c;
    }
    st->prefix |= static_cast<uint32_t>(b) << shift;
    st->mask |= 255u << shift;
    st->remaining -= above;
  }
}

// per chunk: how many keys equal tau
__global__ void __launch_bounds__(256) select_count_kernel(const float *__restrict__ S, int64_t n,
                                                           const SelState *st, unsigned int *cnt) {
  __shared__ unsigned int c;
  if (threadIdx.x == 0) c = 0;
  __syncthreads();
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kSelChunk;
  unsigned int mine = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int64_t i = base + threadIdx.x * 4 + e;
    if (i < n && score_key(S[i]) == st->prefix) ++mine;
  }
  if (mine) atomicAdd(&c, mine);
  __syncthreads();
  if (threadIdx.x == 0) cnt[blockIdx.x] = c;
}

// exclusive prefix sums of the chunk counts, one block of 1024 threads
__global__ void __launch_bounds__(1024) select_scan_kernel(const unsigned int *cnt, int64_t chunks,
                                                           unsigned long long *off) {
  __shared__ unsigned long long part[1024];
  const int64_t per = (chunks + 1023) / 1024;
  const int64_t b0 = threadIdx.x * per, b1 = b0 + per < chunks ? b0 + per : chunks;
  unsigned long long s = 0;
  for (int64_t b = b0; b < b1; ++b) s += cnt[b];
  part[threadIdx.x] = s;
  __syncthreads();
  if (threadIdx.x == 0) {  // 1024 sums, in order
    unsigned long long run = 0;
    for (int t = 0; t < 1024; ++t) {
      const unsigned long long v = part[t];
      part[t] = run;
      run += v;
    }
  }
  __syncthreads();
  unsigned long long run = part[threadIdx.x];
  for (int64_t b = b0; b < b1; ++b) {
    off[b] = run;
    run += cnt[b];
  }
}

// is8[i] = key > tau, or key == tau and fewer than `remaining` equal keys come before it
__global__ void __launch_bounds__(256) select_mark_kernel(const float *__restrict__ S, int64_t n,
                                                          const SelState *st, const unsigned long long *off,
                                                          uint8_t *__restrict__ is8) {
  __shared__ unsigned int warp_tot[8];
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kSelChunk;
  const uint32_t tau = st->prefix;
  const long long need = st->remaining;
  uint32_t key[4];
  unsigned int eq = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int64_t i = base + threadIdx.x * 4 + e;
    key[e] = i < n ? score_key(S[i]) : 0u;
    eq += (i < n && key[e] == tau) ? 1u : 0u;
  }
  // exclusive count of equal keys before this thread's four, in index order
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned int incl = eq;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  unsigned int before = incl - eq;
  for (int q = 0; q < warp; ++q) before += warp_tot[q];
  unsigned long long rank = off[blockIdx.x] + before;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int64_t i = base + threadIdx.x * 4 + e;
    if (i < n) {
      uint8_t sel = key[e] > tau ? 1 : 0;
      if (key[e] == tau) {
        sel = rank < static_cast<unsigned long long>(need) ? 1 : 0;
        ++rank;
      }
      is8[i] = sel;
    }
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

template <int THREADS, int ROWS>
static cudaError_t launch_salience_shape(const float *W, int64_t N, int64_t K, const float *G, int64_t D, float *S,
                                         size_t smem, cudaStream_t stream, const char **msg) {
  auto kern = channel_salience_kernel<THREADS, ROWS>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) {
      *msg = "cudaFuncSetAttribute(MaxDynamicSharedMemorySize) failed";
      return e;
    }
  }
  kern<<<static_cast<unsigned>(N), THREADS, smem, stream>>>(W, N, K, G, D, S);
  return cudaSuccess;
}

cudaError_t launch_channel_salience(const float *W, int64_t N, int64_t K, const float *G, int64_t D, float *S,
                                    cudaStream_t stream, const char **msg) {
  if (N == 0) return cudaSuccess;
  const size_t smem = static_cast<size_t>(K) * sizeof(float);
  if (smem > 227 * 1024) {
    *msg = "K too large for the channel's row in shared memory";
    return cudaErrorInvalidValue;
  }
  if (N > 0x7FFFFFFF) {
    *msg = "too many channels";
    return cudaErrorInvalidValue;
  }
  cudaError_t e = K <= kSalKSmall ? launch_salience_shape<256, 4>(W, N, K, G, D, S, smem, stream, msg)
                                  : launch_salience_shape<512, 8>(W, N, K, G, D, S, smem, stream, msg);
  if (e != cudaSuccess) return e;
  e = cudaGetLastError();
  if (e != cudaSuccess) *msg = "launch of the salience kernel failed";
  return e;
}

size_t select_top_t_workspace_bytes(int64_t n) {
  const int64_t chunks = (n + kSelChunk - 1) / kSelChunk;
  return (sizeof(SelState) + 15) / 16 * 16 + static_cast<size_t>(chunks) * (4 + 8) + 16;
}

cudaError_t launch_select_top_t(const float *S, int64_t n, int64_t T, uint8_t *is8, void *ws, cudaStream_t stream,
                                const char **msg) {
  if (n == 0) return cudaSuccess;
  if (T <= 0 || T >= n) {
    cudaError_t e = cudaMemsetAsync(is8, T <= 0 ? 0 : 1, static_cast<size_t>(n), stream);
    if (e != cudaSuccess) *msg = "cudaMemsetAsync of the bit map failed";
    return e;
  }
  const int64_t chunks = (n + kSelChunk - 1) / kSelChunk;
  if (chunks > 0x7FFFFFFF) {
    *msg = "too many scores";
    return cudaErrorInvalidValue;
  }
  SelState *st = static_cast<SelState *>(ws);
  unsigned long long *off =
      reinterpret_cast<unsigned long long *>(static_cast<char *>(ws) + (sizeof(SelState) + 15) / 16 * 16);
  unsigned int *cnt = reinterpret_cast<unsigned int *>(off + chunks);
  select_init_kernel<<<1, 256, 0, stream>>>(st, T);
  const int hist_grid = static_cast<int>(chunks < 148 * 8 ? chunks : 148 * 8);
  for (int shift = 24; shift >= 0; shift -= 8) {
    select_hist_kernel<<<hist_grid, 256, 0, stream>>>(S, n, st, shift);
    select_pick_kernel<<<1, 256, 0, stream>>>(st, shift);
  }
  select_count_kernel<<<static_cast<unsigned>(chunks), 256, 0, stream>>>(S, n, st, cnt);
  select_scan_kernel<<<1, 1024, 0, stream>>>(cnt, chunks, off);
  select_mark_kernel<<<static_cast<unsigned>(chunks), 256, 0, stream>>>(S, n, st, off, is8);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) *msg = "launch of the top-T selection failed";
  return e;
}

}  // namespace mixllm

// gemv_w4w8a8.cuh -- the W4.4A8 layer for one to eight tokens (decode), sm_100a.
//
// Same arithmetic as the tensor-core kernels (MLSys 2026 talk notes on MixLLM,
// notes.yuuk.io, §二段階逆量子化による int8 Tensor Core 活用, §高速 I2F 変換):
// per group g of 128 along K the int32 partial
//     P_g = sum_{k in g} (W_q - z) * A_q        (exact)
// becomes a float by the 0x4b400000 bias trick and is accumulated,
//     acc += float(P_g) * s_w[n,g] * s_a[m,g]   (fp32),
// and Y[m, idx[n]] = fp16(acc).  With so few tokens a tensor-core tile does
// almost no useful work per weight byte and its issue and drain cost more
// than the bytes, so the layer runs as a GEMV over the packed weights, which
// are nearly all of the bytes it reads:
//   * a CTA covers one 128-channel tile of one set and a range of groups
//     (split-K, so that several CTAs per SM keep HBM busy); two threads per
//     channel row, one for the even and one for the odd groups, so a thread
//     forms whole group partials (no exchange per group) and the two fp32
//     sums meet once, at the end;
//   * the weights stream through two 32 KiB shared-memory slots filled by
//     asynchronous copies that complete on mbarriers.  A CTA's bulk-copy
//     throughput grows with the bytes of each copy (measured on B200: 8 KiB
//     copies hold a CTA near 12 GB/s however many are queued, 32 KiB copies
//     with two in flight near 40 GB/s), so every copy moves 32 KiB: four
//     4-bit groups (a tile's groups are contiguous 8 KiB blocks, so one bulk
//     copy) or two 8-bit groups (one 3-D TMA box: 128 k x 128 rows x 2
//     groups, 128-byte swizzled).  8-bit tiles have twice the bytes per group
//     and get twice the splits, so every CTA moves about the same bytes;
//   * the tile's zero points and channel scales for the CTA's groups are
//     staged once, with the tokens' codes, by ordinary loads;
//   * 4-bit: sum_k (W_q - z) A_q = sum_k W_q A_q - z * sum_k A_q; the first sum
//     takes dp4a on the unsigned nibbles (four u8 x s8 products into int32 per
//     instruction), the per-(token, group) sum of the codes is formed once
//     while they are staged in shared memory.  8-bit: dp4a on s8 x s8.  Both
//     are exact in int32 (|P| < 2^22);
//   * then v = bits(P + 0x4b400000), u = fma(v, s_w, -1.5*2^23*s_w) = fl(P*s_w)
//     (exact: s_w is fp16, so the constant is exact and the fma rounds once),
//     acc = fma(u, s_a, acc); at the end y = acc_even + acc_odd;
//   * with several splits, each writes its partial sums to the workspace and
//     the last CTA of a tile adds them in split order (fixed, so repeated
//     calls are bit-identical) and returns the tile's counter to zero.
// Every mbarrier wait is bounded: on a timeout the kernel records the status,
// stops computing, drains the copies it has in flight and returns.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "gemm_w4w8a8.cuh"  // kI2FBias, kI2FBiasBits
#include "launch.h"
#include "ptx_sm100.cuh"

namespace mixllm {

constexpr int kGvThreads = 256;  // 128 channel rows x 2 (even / odd groups)

// Per token bound: the ring (slots x bytes per copy) and the groups a CTA may
// take (bounds the staged tables), sized so that two CTAs fit on an SM.
// Measured on B200 (decode layers of Llama 3.1 8B / 70B): two 32 KiB slots
// match four 16 KiB ones; a cap of 16 groups is slower, since it forces
// extra splits and more CTAs than are resident at once.
template <int MT>
struct GvCfg {
  static constexpr int kSlots = 2;
  static constexpr int kSlotBytes = 32768;
  static constexpr int kGroupsMax = 32;
  static constexpr int kChunk4 = kSlotBytes / 8192;   // 4-bit groups per copy (8 KiB each)
  static constexpr int kChunk8 = kSlotBytes / 16384;  // 8-bit groups per copy (16 KiB each)
};
// resident CTAs per SM (the shared memory of gemv_smem_bytes allows it)
constexpr int gemv_min_blocks(int) { return 2; }

template <int MT>
struct GvShared {
  using C = GvCfg<MT>;
  int8_t a[MT][C::kGroupsMax * 128];  // the tokens' codes over this CTA's groups
  float sa[MT][C::kGroupsMax];        // their scales
  int asum[MT][C::kGroupsMax];        // sum of the 128 codes of each (token, group)
  __align__(16) uint8_t z[C::kGroupsMax][64];   // the tile's packed zero points (4-bit)
  __align__(16) __half sw[C::kGroupsMax][128];  // the tile's channel scales
  __align__(8) uint64_t full[C::kSlots];
  int abort_flag;
  int last;
};

template <int MT>
constexpr int gemv_smem_bytes() {
  // 1024: alignment slack of the ring
  return 1024 + GvCfg<MT>::kSlots * GvCfg<MT>::kSlotBytes + static_cast<int>(sizeof(GvShared<MT>));
}

// four u8 x s8 products added to c
__device__ __forceinline__ int dp4a_u8s8(uint32_t a, int b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ uint4 lds_u4(const uint8_t *p) { return *reinterpret_cast<const uint4 *>(p); }
__device__ __forceinline__ int4 lds_i4(const int8_t *p) { return *reinterpret_cast<const int4 *>(p); }

// MT: the token bound of this instantiation (1, 2, 4 or 8), M <= MT.
// Grid: nt4 4-bit tiles x S4 splits, then nt8 8-bit tiles x S8 splits; split
// s of S takes groups [s*G/S, (s+1)*G/S), 1 to GvCfg<MT>::kGroupsMax of them.
// tmW8: the 8-bit weights as a 3-D tensor (k within a group, row, group)
// with boxes of GvCfg<MT>::kChunk8 groups.
template <int MT>
__global__ void __launch_bounds__(kGvThreads, gemv_min_blocks(MT))
    gemv_w4w8a8_kernel(const __grid_constant__ CUtensorMap tmW8, const int8_t *__restrict__ A_q,
                       const float *__restrict__ s_a, const uint8_t *__restrict__ W4, const uint8_t *__restrict__ z4,
                       const __half *__restrict__ s_w4, const int32_t *__restrict__ idx4,
                       const __half *__restrict__ s_w8, const int32_t *__restrict__ idx8, int M, int K, int N4,
                       int N8, int N4p, int N8p, int nt4, int ntiles, int S4, int S8, __half *__restrict__ Y,
                       float *__restrict__ ws_part, int *__restrict__ ws_cnt) {
  using C = GvCfg<MT>;
  constexpr int kGvSlots = C::kSlots, kGvSlotBytes = C::kSlotBytes, kGvChunk4 = C::kChunk4, kGvChunk8 = C::kChunk8;
  extern __shared__ uint8_t gv_dyn[];
  uint8_t *ring = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(gv_dyn) + 1023) & ~uintptr_t(1023));
  GvShared<MT> &S = *reinterpret_cast<GvShared<MT> *>(ring + kGvSlots * kGvSlotBytes);

  const int b4 = nt4 * S4;
  const bool is4 = static_cast<int>(blockIdx.x) < b4;
  const int nsplit = is4 ? S4 : S8;
  const int bl = is4 ? static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.x) - b4;
  const int t_in_set = bl / nsplit, split = bl - t_in_set * nsplit;
  const int tile = is4 ? t_in_set : nt4 + t_in_set;
  const int n0 = t_in_set * 128;
  const int G = K >> 7;
  const int g0 = static_cast<int>((static_cast<int64_t>(split) * G) / nsplit);
  const int g1 = static_cast<int>((static_cast<int64_t>(split + 1) * G) / nsplit);
  const int ng = g1 - g0;
  const int Nset = is4 ? N4 : N8;
  const int N = N4 + N8;
  const int r = threadIdx.x & 127, par = threadIdx.x >> 7;  // channel row; the parity of its groups
  const bool row_ok = n0 + r < Nset;
  const int chunk = is4 ? kGvChunk4 : kGvChunk8;
  const int nch = (ng + chunk - 1) / chunk;
  const uint8_t *w4_tile = is4 ? W4 + (static_cast<int64_t>(t_in_set) * G + g0) * 8192 : nullptr;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGvSlots; ++s) mbar_init(&S.full[s], 1);
    S.abort_flag = 0;
    fence_mbar_init();
    if (!is4) prefetch_tmap(&tmW8);
  }
  // every global read of this grid comes after this wait (the tokens' codes
  // and scales are written by the kernel before this one)
  pdl_wait();
  __syncthreads();  // barriers initialized

  // chunk c of this CTA's groups into slot c % 2
  auto issue = [&](int c) {
    const int sl = c % kGvSlots;
    uint64_t *bar = &S.full[sl];
    if (is4) {
      const int n = min(kGvChunk4, ng - c * kGvChunk4);
      const uint32_t bytes = static_cast<uint32_t>(n) * 8192u;
      mbar_arrive_expect_tx(bar, bytes);
      bulk_load(ring + sl * kGvSlotBytes, w4_tile + static_cast<int64_t>(c) * kGvChunk4 * 8192, bytes, bar);
    } else {
      // the whole box always lands (groups past the CTA's last come from the
      // next split or are filled with zeros past K) and is never read
      mbar_arrive_expect_tx(bar, kGvSlotBytes);
      tma_load_3d(ring + sl * kGvSlotBytes, &tmW8, bar, 0, n0, g0 + c * kGvChunk8);
    }
  };
  int issued = 0;
  if (threadIdx.x == 0) {
    for (; issued < kGvSlots && issued < nch; ++issued) issue(issued);
  }

  // stage the tokens' codes of groups [g0, g1), their sums and scales, and
  // the tile's zero points and channel scales of those groups
  {
    const int pieces = MT * ng * 8;  // 16-byte pieces, 8 per (token, group)
    for (int e0 = 0; e0 < pieces; e0 += kGvThreads) {  // the same trip count in every thread
      const int e = e0 + static_cast<int>(threadIdx.x);
      const bool ok = e < pieces;
      const int m = ok ? e / (ng * 8) : 0, q = ok ? e - m * (ng * 8) : 0;
      int4 v = make_int4(0, 0, 0, 0);
      if (ok && m < M) v = *reinterpret_cast<const int4 *>(A_q + static_cast<int64_t>(m) * K + g0 * 128 + q * 16);
      if (ok) *reinterpret_cast<int4 *>(&S.a[m][q * 16]) = v;
      int sum = __dp4a(v.x, 0x01010101, 0);
      sum = __dp4a(v.y, 0x01010101, sum);
      sum = __dp4a(v.z, 0x01010101, sum);
      sum = __dp4a(v.w, 0x01010101, sum);
      sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 1);
      sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 2);
      sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 4);
      if (ok && (q & 7) == 0) S.asum[m][q >> 3] = sum;
    }
    for (int e = threadIdx.x; e < MT * ng; e += kGvThreads) {
      const int m = e / ng, i = e - m * ng;
      S.sa[m][i] = m < M ? s_a[static_cast<int64_t>(m) * G + g0 + i] : 0.0f;
    }
    const __half *swp = is4 ? s_w4 + static_cast<int64_t>(g0) * N4p + n0 : s_w8 + static_cast<int64_t>(g0) * N8p + n0;
    const int64_t sws = is4 ? N4p : N8p;
    for (int e = threadIdx.x; e < ng * 16; e += kGvThreads) {  // 16 pieces of 8 scales per group
      const int i = e >> 4, q = e & 15;
      *reinterpret_cast<uint4 *>(&S.sw[i][q * 8]) = *reinterpret_cast<const uint4 *>(swp + i * sws + q * 8);
    }
    if (is4) {
      for (int e = threadIdx.x; e < ng * 4; e += kGvThreads) {  // 4 pieces of 16 bytes per group
        const int i = e >> 2, q = e & 3;
        *reinterpret_cast<uint4 *>(&S.z[i][q * 16]) =
            *reinterpret_cast<const uint4 *>(z4 + static_cast<int64_t>(g0 + i) * (N4p >> 1) + (n0 >> 1) + q * 16);
      }
    }
  }
  __syncthreads();

  float acc[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
  int drain_from = -1;  // thread 0: first chunk whose copy was not seen to complete
  for (int c = 0; c < nch; ++c) {
    const int sl = c % kGvSlots;
    const bool ok = warp_wait(&S.full[sl], static_cast<uint32_t>((c / kGvSlots) & 1), &S.abort_flag);
    if (ok) {
      const uint8_t *slot = ring + sl * kGvSlotBytes;
      const int i_end = min(ng, (c + 1) * chunk);
      for (int i = c * chunk + par; i < i_end; i += 2) {
        const int j = i - c * chunk;  // group within the slot
        // four independent int32 chains per token, added at the end (exact)
        int p[MT][4];
#pragma unroll
        for (int m = 0; m < MT; ++m) p[m][0] = p[m][1] = p[m][2] = p[m][3] = 0;
        if (is4) {
          // the row's 64 bytes are runs c = 0..3 of 16 bytes; byte b of run c holds
          // k = 32c + b (low nibble) and k = 32c + 16 + b (high nibble).  Runs are
          // taken in an order rotated by r / 2 so that the 8 rows of a quarter
          // warp read 8 different bank groups.
          const uint8_t *wr = slot + j * 8192 + r * 64;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int rc = (u + (r >> 1)) & 3;
            const uint4 w = lds_u4(wr + 16 * rc);
            const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
            uint32_t lo[4], hi[4];
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              lo[v] = wd[v] & 0x0F0F0F0Fu;
              hi[v] = (wd[v] >> 4) & 0x0F0F0F0Fu;
            }
            const int kr = i * 128 + rc * 32;
#pragma unroll
            for (int m = 0; m < MT; ++m) {
              const int4 al = lds_i4(&S.a[m][kr]);
              const int4 ah = lds_i4(&S.a[m][kr + 16]);
              p[m][0] = dp4a_u8s8(lo[0], al.x, p[m][0]);
              p[m][1] = dp4a_u8s8(lo[1], al.y, p[m][1]);
              p[m][2] = dp4a_u8s8(lo[2], al.z, p[m][2]);
              p[m][3] = dp4a_u8s8(lo[3], al.w, p[m][3]);
              p[m][0] = dp4a_u8s8(hi[0], ah.x, p[m][0]);
              p[m][1] = dp4a_u8s8(hi[1], ah.y, p[m][1]);
              p[m][2] = dp4a_u8s8(hi[2], ah.z, p[m][2]);
              p[m][3] = dp4a_u8s8(hi[3], ah.w, p[m][3]);
            }
          }
          // the zero point's term
          const int z = (S.z[i][r >> 1] >> ((r & 1) * 4)) & 0xF;
#pragma unroll
          for (int m = 0; m < MT; ++m) p[m][0] -= z * S.asum[m][i];
        } else {
          // 128-byte swizzled rows: 16-byte chunk q of row r sits at chunk q ^ (r & 7)
          const uint8_t *wr = slot + j * 16384 + r * 128;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint4 w = lds_u4(wr + ((q ^ (r & 7)) << 4));
            const int kr = i * 128 + q * 16;
#pragma unroll
            for (int m = 0; m < MT; ++m) {
              const int4 a = lds_i4(&S.a[m][kr]);
              p[m][0] = __dp4a(static_cast<int>(w.x), a.x, p[m][0]);
              p[m][1] = __dp4a(static_cast<int>(w.y), a.y, p[m][1]);
              p[m][2] = __dp4a(static_cast<int>(w.z), a.z, p[m][2]);
              p[m][3] = __dp4a(static_cast<int>(w.w), a.w, p[m][3]);
            }
          }
        }
        const float swf = __half2float(S.sw[i][r]);
        const float cb = -kI2FBias * swf;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const int P = (p[m][0] + p[m][1]) + (p[m][2] + p[m][3]);
          const float v = __uint_as_float(static_cast<uint32_t>(P) + kI2FBiasBits);
          acc[m] = __fmaf_rn(__fmaf_rn(v, swf, cb), S.sa[m][i], acc[m]);
        }
      }
    } else if (threadIdx.x == 0 && drain_from < 0) {
      drain_from = c;
    }
    __syncthreads();  // slot sl is free
    if (threadIdx.x == 0 && issued < nch && !S.abort_flag) issue(issued++);
  }
  if (threadIdx.x == 0 && drain_from >= 0) {
    // gave up: wait (bounded) for the copies still in flight before the CTA exits
    for (int c = drain_from; c < issued; ++c)
      (void)mbar_wait_drain(&S.full[c % kGvSlots], static_cast<uint32_t>((c / kGvSlots) & 1), 1ll << 30);
  }
  const bool aborted = S.abort_flag != 0;  // uniform: set before the last barrier or never
  // y = acc(even groups) + acc(odd groups): the odd-group threads hand theirs
  // over through the tokens' code area, which the loop's last barrier freed
  float(*odd)[128] = reinterpret_cast<float(*)[128]>(&S.a[0][0]);
  static_assert(sizeof(S.a) >= MT * 128 * sizeof(float), "room for the odd-group sums");
  if (par == 1) {
#pragma unroll
    for (int m = 0; m < MT; ++m) odd[m][r] = acc[m];
  }
  __syncthreads();
  if (par == 0) {
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] += odd[m][r];
  }

  const int mt = M < MT ? M : MT;
  const int col_out = row_ok ? __ldg((is4 ? idx4 : idx8) + n0 + r) : 0;
  if (nsplit == 1) {
    if (row_ok && par == 0 && !aborted) {
#pragma unroll
      for (int m = 0; m < MT; ++m)
        if (m < mt) Y[static_cast<int64_t>(m) * N + col_out] = __float2half_rn(acc[m]);
    }
    return;
  }
  // this split's partial sums: [split][tile][MT][128]
  if (par == 0) {
    float *part = ws_part + (static_cast<size_t>(split) * ntiles + tile) * (MT * 128) + r;
#pragma unroll
    for (int m = 0; m < MT; ++m)
      if (m < mt) part[m * 128] = acc[m];
  }
  // The barrier orders every thread's partial stores before thread 0's
  // counter update, whose release at GPU scope publishes them (cumulativity);
  // the last CTA's acquire on the same counter makes all splits' partials
  // visible to it, and its barrier passes that on to the other threads.
  __syncthreads();
  if (threadIdx.x == 0) {
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;" : "=r"(old) : "l"(ws_cnt + tile) : "memory");
    S.last = old == nsplit - 1;
  }
  __syncthreads();
  if (!S.last) return;
  if (par == 0 && row_ok && !aborted) {
    const float *p0 = ws_part + static_cast<size_t>(tile) * (MT * 128) + r;
    const size_t split_stride = static_cast<size_t>(ntiles) * (MT * 128);
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      if (m < mt) {
        float y = __ldcg(p0 + m * 128);
        for (int sp = 1; sp < nsplit; ++sp) y += __ldcg(p0 + sp * split_stride + m * 128);
        Y[static_cast<int64_t>(m) * N + col_out] = __float2half_rn(y);
      }
    }
  }
  if (threadIdx.x == 0) ws_cnt[tile] = 0;  // leave the counter as it was found
}

}  // namespace mixllm

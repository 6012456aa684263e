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
#include "quant.cuh"  // quant_act_8x16

namespace mixllm {

constexpr int kGvThreads = 256;  // 128 channel rows x 2 (even / odd groups)
constexpr int kGvSlotBytesSplit = 32768;  // the split kernel's slot (its fused form stages X in one)

// Per token bound: the ring (slots x bytes per copy) and the groups a CTA may
// take (bounds the staged tables), sized so that two CTAs fit on an SM.
// Measured on B200 (decode layers of Llama 3.1 8B / 70B): two 32 KiB slots
// match four 16 KiB ones; a cap of 16 groups is slower, since it forces
// extra splits and more CTAs than are resident at once.
template <int MT>
struct GvCfg {
  static constexpr int kSlots = 2;
  static constexpr int kSlotBytes = kGvSlotBytesSplit;
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
  __align__(8) uint64_t a_full;  // the tokens' codes landed
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

// One 4-bit group of two channel rows (rp and rp + 64), all tokens:
// acc[h][m] += fl(fl(P*s_w)*s_a[m]) with P = sum_k W_q*A_q - z*sum_k A_q
// (exact).  blk: the group's 8 KiB block in shared memory (row r at 64*r; byte
// b of its 16-byte run c holds k = 32c+b in the low nibble and k = 32c+16+b in
// the high one); a: token 0's 128 codes of the group, the next token a_stride
// bytes on; asum, sa: token 0's code sum and scale of the group, the next
// token t_stride elements on.  The high nibbles stay in place (16x their
// value, still a u8), so their dp4a sum is 16x exact and >> 4 recovers it; the
// codes a thread loads serve both rows; the runs are taken in an order
// rotated by rp / 2 so that the 8 rows of a quarter warp read 8 different
// bank groups.
// DBG: P of row h, token m < mt also goes to pd[h][m * pd_tstride] (rows
// whose pointer is null are skipped).
template <int MT, bool DBG = false>
__device__ __forceinline__ void gv_group4x2(const uint8_t *blk, int rp, const int8_t *a, int a_stride,
                                            const int *asum, const float *sa, int t_stride, const int (&z)[2],
                                            const float (&sw)[2], float (&acc)[2][MT], int32_t *pd0 = nullptr,
                                            int32_t *pd1 = nullptr, int64_t pd_tstride = 0, int mt = 0) {
  int plo[2][MT][2], phi[2][MT][2];
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int m = 0; m < MT; ++m) plo[h][m][0] = plo[h][m][1] = phi[h][m][0] = phi[h][m][1] = 0;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int rc = (u + (rp >> 1)) & 3;
    uint4 w[2];
    w[0] = lds_u4(blk + rp * 64 + 16 * rc);
    w[1] = lds_u4(blk + (rp + 64) * 64 + 16 * rc);
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const int4 al = lds_i4(a + m * a_stride + rc * 32);
      const int4 ah = lds_i4(a + m * a_stride + rc * 32 + 16);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        plo[h][m][0] = dp4a_u8s8(w[h].x & 0x0F0F0F0Fu, al.x, plo[h][m][0]);
        plo[h][m][1] = dp4a_u8s8(w[h].y & 0x0F0F0F0Fu, al.y, plo[h][m][1]);
        plo[h][m][0] = dp4a_u8s8(w[h].z & 0x0F0F0F0Fu, al.z, plo[h][m][0]);
        plo[h][m][1] = dp4a_u8s8(w[h].w & 0x0F0F0F0Fu, al.w, plo[h][m][1]);
        phi[h][m][0] = dp4a_u8s8(w[h].x & 0xF0F0F0F0u, ah.x, phi[h][m][0]);
        phi[h][m][1] = dp4a_u8s8(w[h].y & 0xF0F0F0F0u, ah.y, phi[h][m][1]);
        phi[h][m][0] = dp4a_u8s8(w[h].z & 0xF0F0F0F0u, ah.z, phi[h][m][0]);
        phi[h][m][1] = dp4a_u8s8(w[h].w & 0xF0F0F0F0u, ah.w, phi[h][m][1]);
      }
    }
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const float cb = -kI2FBias * sw[h];
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const int P = (plo[h][m][0] + plo[h][m][1]) + ((phi[h][m][0] + phi[h][m][1]) >> 4) - z[h] * asum[m * t_stride];
      if constexpr (DBG) {
        int32_t *pd = h == 0 ? pd0 : pd1;
        if (pd != nullptr && m < mt) pd[m * pd_tstride] = P;
      }
      const float v = __uint_as_float(static_cast<uint32_t>(P) + kI2FBiasBits);
      acc[h][m] = __fmaf_rn(__fmaf_rn(v, sw[h], cb), sa[m * t_stride], acc[h][m]);
    }
  }
}

// One 8-bit group of one channel row, all tokens (P = sum_k W_q*A_q, exact).
// wrow: the row's 128 bytes of a 128-byte swizzled TMA box in shared memory
// (16-byte chunk q of row r at chunk q ^ (r & 7)).  DBG: as gv_group4x2.
template <int MT, bool DBG = false>
__device__ __forceinline__ void gv_group8(const uint8_t *wrow, int r, const int8_t *a, int a_stride,
                                          const float *sa, int t_stride, float sw, float (&acc)[MT],
                                          int32_t *pd = nullptr, int64_t pd_tstride = 0, int mt = 0) {
  int p[MT][4];
#pragma unroll
  for (int m = 0; m < MT; ++m) p[m][0] = p[m][1] = p[m][2] = p[m][3] = 0;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const uint4 w = lds_u4(wrow + ((q ^ (r & 7)) << 4));
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const int4 av = lds_i4(a + m * a_stride + q * 16);
      p[m][0] = __dp4a(static_cast<int>(w.x), av.x, p[m][0]);
      p[m][1] = __dp4a(static_cast<int>(w.y), av.y, p[m][1]);
      p[m][2] = __dp4a(static_cast<int>(w.z), av.z, p[m][2]);
      p[m][3] = __dp4a(static_cast<int>(w.w), av.w, p[m][3]);
    }
  }
  const float cb = -kI2FBias * sw;
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    const int P = (p[m][0] + p[m][1]) + (p[m][2] + p[m][3]);
    if constexpr (DBG) {
      if (pd != nullptr && m < mt) pd[m * pd_tstride] = P;
    }
    const float v = __uint_as_float(static_cast<uint32_t>(P) + kI2FBiasBits);
    acc[m] = __fmaf_rn(__fmaf_rn(v, sw, cb), sa[m * t_stride], acc[m]);
  }
}

// MT: the token bound of this instantiation (1, 2, 4 or 8), M <= MT.
// Grid: nt4 4-bit tiles x S4 splits, then nt8 8-bit tiles x S8 splits; split
// s of S takes groups [s*G/S, (s+1)*G/S), 1 to GvCfg<MT>::kGroupsMax of them.
// FUSE: the activations come in as fp16 X [M, K] and each CTA quantizes the
// slice it needs itself (the same quantizer as quantize_act_kernel, so the
// same codes): its slice of X is bulk-copied into the second ring slot while
// the first weight chunk streams into the first (the host launches this form
// only when the slice fits in a slot), then the slot is refilled with weights.
// tmW8: the 8-bit weights as a 3-D tensor (k within a group, row, group)
// with boxes of GvCfg<MT>::kChunk8 groups.
// DBG: the int32 group partials also go to Pd [M, N, G] (output column order).
template <int MT, bool FUSE, bool DBG = false>
__global__ void __launch_bounds__(kGvThreads, gemv_min_blocks(MT))
    gemv_w4w8a8_kernel(const __grid_constant__ CUtensorMap tmW8, const __half *__restrict__ X,
                       const int8_t *__restrict__ A_q,
                       const float *__restrict__ s_a, const uint8_t *__restrict__ W4, const uint8_t *__restrict__ z4,
                       const __half *__restrict__ s_w4, const int32_t *__restrict__ idx4,
                       const __half *__restrict__ s_w8, const int32_t *__restrict__ idx8, int M, int K, int N4,
                       int N8, int N4p, int N8p, int nt4, int ntiles, int S4, int S8, __half *__restrict__ Y,
                       float *__restrict__ ws_part, int *__restrict__ ws_cnt, int32_t *__restrict__ Pd) {
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

  // the next kernel of the stream may launch now: it reads nothing this one
  // writes before its own dependency wait
  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kGvSlots; ++s) mbar_init(&S.full[s], 1);
    mbar_init(&S.a_full, 1);
    S.abort_flag = 0;
    fence_mbar_init();
    if (!is4) prefetch_tmap(&tmW8);
  }
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
  const int mt = M < MT ? M : MT;
  // s_a rows as bulk copies too when they are 16-byte pieces (the CTAs of a
  // split read the same few lines: one request per token instead of a warp's loads)
  const bool sa_bulk = !FUSE && ((g0 | ng | G) & 3) == 0 && (reinterpret_cast<uintptr_t>(s_a) & 15) == 0;
  // The first weight chunks stream in while the kernel before this one
  // finishes (the packed layer is constant); the tokens' codes, scales or
  // activations, which that kernel writes, are read only after pdl_wait.
  int issued = 0;
  if (threadIdx.x == 0) {
    if (FUSE)
      issue(issued++);  // the first chunk into the first slot (the second takes the activations)
    else
      for (; issued < kGvSlots && issued < nch; ++issued) issue(issued);
  }
  {  // the tile's channel scales and zero points of groups [g0, g1): constant too
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
  pdl_wait();
  if (FUSE && threadIdx.x == 0) {
    // the tokens' fp16 activations of groups [g0, g1) into the second slot, one
    // bulk copy per token
    mbar_arrive_expect_tx(&S.a_full, static_cast<uint32_t>(mt * ng * 256));
    for (int m = 0; m < mt; ++m)
      bulk_load(ring + kGvSlotBytes + m * ng * 256, X + static_cast<int64_t>(m) * K + g0 * 128,
                static_cast<uint32_t>(ng * 256), &S.a_full);
  }
  if (!FUSE && threadIdx.x == 0) {
    // the tokens' codes (and scales) of groups [g0, g1): one bulk copy per token
    mbar_arrive_expect_tx(&S.a_full, static_cast<uint32_t>(mt * ng * (128 + (sa_bulk ? 4 : 0))));
    for (int m = 0; m < mt; ++m) {
      bulk_load(&S.a[m][0], A_q + static_cast<int64_t>(m) * K + g0 * 128, static_cast<uint32_t>(ng * 128), &S.a_full);
      if (sa_bulk)
        bulk_load(&S.sa[m][0], s_a + static_cast<int64_t>(m) * G + g0, static_cast<uint32_t>(ng * 4), &S.a_full);
    }
  }

  // stage the tokens' scales while the codes and weights are on their way
  {
    for (int e = threadIdx.x; e < (MT - mt) * ng * 8; e += kGvThreads)  // tokens past M: zero codes
      *reinterpret_cast<int4 *>(&S.a[mt + e / (ng * 8)][(e % (ng * 8)) * 16]) = make_int4(0, 0, 0, 0);
    for (int e = threadIdx.x; e < MT * ng; e += kGvThreads) {
      const int m = e / ng, i = e - m * ng;
      if (m >= mt) {
        S.sa[m][i] = 0.0f;
        if (FUSE) S.asum[m][i] = 0;
      } else if (!FUSE && !sa_bulk) {
        S.sa[m][i] = s_a[static_cast<int64_t>(m) * G + g0 + i];
      }
    }
    if (FUSE) {
      // quantize: a half warp per (token, group), eight activations per lane
      (void)warp_wait(&S.a_full, 0, &S.abort_flag);
      const int lane16 = threadIdx.x & 15, hw = threadIdx.x >> 4;
      const unsigned mask = 0xFFFFu << (threadIdx.x & 16);
      for (int pr = hw; pr < mt * ng; pr += kGvThreads / 16) {  // uniform within a half warp (its shuffle mask)
        const int m = pr / ng, i = pr - m * ng;
        const uint4 raw = lds_u4(ring + kGvSlotBytes + pr * 256 + lane16 * 16);
        uint32_t packed[2];
        const float sa = quant_act_8x16(raw, mask, packed);
        *reinterpret_cast<uint2 *>(&S.a[m][i * 128 + lane16 * 8]) = make_uint2(packed[0], packed[1]);
        int sum = __dp4a(static_cast<int>(packed[0]), 0x01010101, __dp4a(static_cast<int>(packed[1]), 0x01010101, 0));
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) sum += __shfl_xor_sync(mask, sum, o);
        if (lane16 == 0) {
          S.sa[m][i] = sa;
          S.asum[m][i] = sum;
        }
      }
    } else {
      // the sum of each (token, group)'s 128 codes, once they have landed:
      // 8 threads per (token, group), one 16-byte piece each
      (void)warp_wait(&S.a_full, 0, &S.abort_flag);
      const int pieces = MT * ng * 8;
      for (int e0 = 0; e0 < pieces; e0 += kGvThreads) {  // the same trip count in every thread
        const int e = e0 + static_cast<int>(threadIdx.x);
        const bool ok = e < pieces;
        const int m = ok ? (e >> 3) / ng : 0, i = ok ? (e >> 3) - m * ng : 0;
        const int4 v = ok ? lds_i4(&S.a[m][i * 128 + (e & 7) * 16]) : make_int4(0, 0, 0, 0);
        int sum = __dp4a(v.x, 0x01010101, 0);
        sum = __dp4a(v.y, 0x01010101, sum);
        sum = __dp4a(v.z, 0x01010101, sum);
        sum = __dp4a(v.w, 0x01010101, sum);
        sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 1);
        sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 2);
        sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 4);
        if (ok && (e & 7) == 0) S.asum[m][i] = sum;
      }
    }
  }
  __syncthreads();
  if (FUSE && threadIdx.x == 0 && issued < nch) issue(issued++);  // the second slot is free again

  // 4-bit: rows rp and rp + 64, group j4 of every chunk; 8-bit: row r8, group j8
  const int rp = threadIdx.x & 63, j4 = threadIdx.x >> 6;
  const int r8 = threadIdx.x & 127, j8 = threadIdx.x >> 7;
  float acc[2][MT];
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[h][m] = 0.0f;
  int drain_from = -1;  // thread 0: first chunk whose copy was not seen to complete
  for (int c = 0; c < nch; ++c) {
    const int sl = c % kGvSlots;
    const bool ok = warp_wait(&S.full[sl], static_cast<uint32_t>((c / kGvSlots) & 1), &S.abort_flag);
    if (ok) {
      const uint8_t *slot = ring + sl * kGvSlotBytes;
      if (is4) {
        const int i = c * chunk + j4;
        if (i < ng) {
          const int z[2] = {(S.z[i][rp >> 1] >> ((rp & 1) * 4)) & 0xF, (S.z[i][(rp + 64) >> 1] >> ((rp & 1) * 4)) & 0xF};
          const float sw[2] = {__half2float(S.sw[i][rp]), __half2float(S.sw[i][rp + 64])};
          int32_t *pd0 = nullptr, *pd1 = nullptr;
          if constexpr (DBG) {
            if (n0 + rp < Nset) pd0 = Pd + static_cast<int64_t>(__ldg(idx4 + n0 + rp)) * G + g0 + i;
            if (n0 + rp + 64 < Nset) pd1 = Pd + static_cast<int64_t>(__ldg(idx4 + n0 + rp + 64)) * G + g0 + i;
          }
          gv_group4x2<MT, DBG>(slot + j4 * 8192, rp, &S.a[0][i * 128], C::kGroupsMax * 128, &S.asum[0][i],
                               &S.sa[0][i], C::kGroupsMax, z, sw, acc, pd0, pd1, static_cast<int64_t>(N) * G, mt);
        }
      } else {
        const int i = c * chunk + j8;
        if (i < ng) {
          int32_t *pd = nullptr;
          if constexpr (DBG) {
            if (n0 + r8 < Nset) pd = Pd + static_cast<int64_t>(__ldg(idx8 + n0 + r8)) * G + g0 + i;
          }
          gv_group8<MT, DBG>(slot + j8 * 16384 + r8 * 128, r8, &S.a[0][i * 128], C::kGroupsMax * 128, &S.sa[0][i],
                             C::kGroupsMax, __half2float(S.sw[i][r8]), acc[0], pd, static_cast<int64_t>(N) * G, mt);
        }
      }
    } else if (threadIdx.x == 0 && drain_from < 0) {
      drain_from = c;
    }
    __syncthreads();  // slot sl is free
    if (threadIdx.x == 0 && issued < nch && !S.abort_flag) issue(issued++);
  }
  if (threadIdx.x == 0 && S.abort_flag) {
    // gave up: wait (bounded) for the copies still in flight before the CTA exits
    (void)mbar_wait_drain(&S.a_full, 0, 1ll << 30);
    for (int c = drain_from < 0 ? issued : drain_from; c < issued; ++c)
      (void)mbar_wait_drain(&S.full[c % kGvSlots], static_cast<uint32_t>((c / kGvSlots) & 1), 1ll << 30);
  }
  const bool aborted = S.abort_flag != 0;  // uniform: set before the last barrier or never
  // every row's sum over the threads that hold its groups, in group order j,
  // through the tokens' code area (the loop's last barrier freed it)
  float(*red)[128][MT] = reinterpret_cast<float(*)[128][MT]>(&S.a[0][0]);
  static_assert(sizeof(S.a) >= 4 * 128 * MT * sizeof(float), "room for the row sums");
  if (is4) {
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      red[j4][rp][m] = acc[0][m];
      red[j4][rp + 64][m] = acc[1][m];
    }
  } else {
#pragma unroll
    for (int m = 0; m < MT; ++m) red[j8][r8][m] = acc[0][m];
  }
  __syncthreads();
  float y[MT];  // row r's sums (threads r < 128)
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    y[m] = red[0][r][m];
    for (int jj = 1; jj < chunk; ++jj) y[m] += red[jj][r][m];
  }

  const int col_out = row_ok ? __ldg((is4 ? idx4 : idx8) + n0 + r) : 0;
  if (nsplit == 1) {
    if (row_ok && par == 0 && !aborted) {
#pragma unroll
      for (int m = 0; m < MT; ++m)
        if (m < mt) Y[static_cast<int64_t>(m) * N + col_out] = __float2half_rn(y[m]);
    }
    return;
  }
  // this split's partial sums: [split][tile][MT][128]
  if (par == 0) {
    float *part = ws_part + (static_cast<size_t>(split) * ntiles + tile) * (MT * 128) + r;
#pragma unroll
    for (int m = 0; m < MT; ++m)
      if (m < mt) part[m * 128] = y[m];
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
    float z[MT];
    for (int base = 0; base < nsplit; base += 8) {  // eight partials in flight at a time, added in split order
      float v[8][MT];
#pragma unroll
      for (int q = 0; q < 8; ++q)
#pragma unroll
        for (int m = 0; m < MT; ++m)
          v[q][m] = (base + q < nsplit && m < mt) ? __ldcg(p0 + (base + q) * split_stride + m * 128) : 0.0f;
#pragma unroll
      for (int q = 0; q < 8; ++q)
#pragma unroll
        for (int m = 0; m < MT; ++m)
          if (base + q < nsplit) z[m] = base + q == 0 ? v[q][m] : z[m] + v[q][m];
    }
#pragma unroll
    for (int m = 0; m < MT; ++m)
      if (m < mt) Y[static_cast<int64_t>(m) * N + col_out] = __float2half_rn(z[m]);
  }
  if (threadIdx.x == 0) ws_cnt[tile] = 0;  // leave the counter as it was found
}

// ---------------------------------------------------------------------------
// Persistent variant: one even share of the layer per CTA.
//
// The layer's weights are a sequence of U units of 32 KiB, tile-major: the
// ceil(G/4) chunks of four groups of every 4-bit tile, then the ceil(G/2)
// chunks of two groups of every 8-bit tile.  CTA b of P takes units
// [b*U/P, (b+1)*U/P) and streams them through its two-slot ring without a
// pause at tile boundaries; the zero points and channel scales of a unit
// follow it as 16-byte cp.async copies on a second mbarrier (they do not use
// the copy engine, whose rate per CTA is set by the bytes per copy), and the
// tokens' codes of all K stay in shared memory (M <= 4, M*K <= kGvpMaxTokenBytes).
// A tile whose units one CTA holds entirely is written directly; a tile
// shared by several CTAs gets one fp32 partial from each, which the last of
// them to finish adds in K order.  At most two partials per CTA (its first
// and its last tile): workspace [P][2][MT][128] fp32, then one counter per tile.
// ---------------------------------------------------------------------------

constexpr int kGvpSlotBytes = 32768;
constexpr int kGvpMetaBytes = 4 * 64 + 4 * 256;  // zero points and scales of up to four groups
constexpr int kGvpMaxTokenBytes = 32768;          // M*K bound of the resident tokens' codes
constexpr int kGvpMaxTokens = 4;                  // token bound (its row sums must fit beside them)

struct GvpLayout {  // byte offsets from the 1024-aligned base of the dynamic shared memory
  int meta, bars, a, sa, asum, red, total;
};
__host__ __device__ constexpr GvpLayout gvp_layout(int mt, int K) {
  GvpLayout L{};
  L.meta = 2 * kGvpSlotBytes;
  L.bars = L.meta + 2 * kGvpMetaBytes;
  L.a = L.bars + 64;  // full[2], meta_full[2], a_full, abort, last[2]
  L.sa = L.a + mt * K;
  L.asum = L.sa + mt * (K / 128) * 4;
  L.red = L.asum + mt * (K / 128) * 4;
  L.total = L.red + 4 * 128 * mt * 4;  // row sums [4][128][mt]
  return L;
}
template <int MT>
constexpr int gvp_smem_bytes_max() {
  return 1024 + gvp_layout(MT, kGvpMaxTokenBytes / MT).total;
}

struct GvpGeom {  // the unit sequence
  int nt4, C4, C8, U, P;
  __device__ __forceinline__ int64_t start(int b) const { return static_cast<int64_t>(b) * U / P; }
  __device__ __forceinline__ int owner(int64_t u) const { return static_cast<int>(((u + 1) * P - 1) / U); }
  __device__ __forceinline__ int64_t first_unit(int t) const {
    return t < nt4 ? static_cast<int64_t>(t) * C4 : static_cast<int64_t>(nt4) * C4 + static_cast<int64_t>(t - nt4) * C8;
  }
  __device__ __forceinline__ int chunks(int t) const { return t < nt4 ? C4 : C8; }
  __device__ __forceinline__ void locate(int64_t u, int &t, int &c) const {
    const int64_t u4 = static_cast<int64_t>(nt4) * C4;
    if (u < u4) {
      t = static_cast<int>(u / C4);
      c = static_cast<int>(u - static_cast<int64_t>(t) * C4);
    } else {
      const int64_t v = u - u4;
      t = nt4 + static_cast<int>(v / C8);
      c = static_cast<int>(v - static_cast<int64_t>(t - nt4) * C8);
    }
  }
};

// DBG: the int32 group partials also go to Pd [M, N, G] (output column order).
template <int MT, bool DBG = false>
__global__ void __launch_bounds__(kGvThreads, 2)
    gemv_w4w8a8_persistent_kernel(const __grid_constant__ CUtensorMap tmW8, const int8_t *__restrict__ A_q,
                                  const float *__restrict__ s_a, const uint8_t *__restrict__ W4,
                                  const uint8_t *__restrict__ z4, const __half *__restrict__ s_w4,
                                  const int32_t *__restrict__ idx4, const __half *__restrict__ s_w8,
                                  const int32_t *__restrict__ idx8, int M, int K, int N4, int N8, int N4p, int N8p,
                                  GvpGeom geo, __half *__restrict__ Y, float *__restrict__ ws_part,
                                  int *__restrict__ ws_cnt, int32_t *__restrict__ Pd) {
  extern __shared__ uint8_t gv_dyn[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(gv_dyn) + 1023) & ~uintptr_t(1023));
  const int G = K >> 7;
  const GvpLayout L = gvp_layout(MT, K);
  uint8_t *ring = base;
  uint8_t *meta = base + L.meta;
  uint64_t *full = reinterpret_cast<uint64_t *>(base + L.bars);
  uint64_t *meta_full = full + 2;
  uint64_t *a_full = full + 4;
  int *abort_flag = reinterpret_cast<int *>(full + 5);
  int *last_flag = abort_flag + 1;  // two flags
  int8_t *sA = reinterpret_cast<int8_t *>(base + L.a);      // [MT][K]
  float *sSa = reinterpret_cast<float *>(base + L.sa);      // [MT][G]
  int *sAsum = reinterpret_cast<int *>(base + L.asum);      // [MT][G]
  float(*red)[128][MT] = reinterpret_cast<float(*)[128][MT]>(base + L.red);

  const int b = blockIdx.x;
  const int64_t u0 = geo.start(b), u1 = geo.start(b + 1);
  const int nk = static_cast<int>(u1 - u0);
  const int N = N4 + N8;
  const int r = threadIdx.x & 127;                             // the row this thread writes (threads < 128)
  const int rp = threadIdx.x & 63, j4 = threadIdx.x >> 6;     // 4-bit units: rows rp, rp + 64; group j4
  const int r8 = threadIdx.x & 127, j8 = threadIdx.x >> 7;    // 8-bit units: row r8; group j8

  if (threadIdx.x == 0) {
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    mbar_init(&meta_full[0], kGvThreads);
    mbar_init(&meta_full[1], kGvThreads);
    mbar_init(a_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
    if (geo.nt4 * static_cast<int64_t>(geo.C4) < u1) prefetch_tmap(&tmW8);
  }
  // the next kernel of the stream may launch now: it reads nothing this one
  // writes before its own dependency wait
  pdl_launch_dependents();
  __syncthreads();  // barriers initialized

  // The next unit to issue, as (tile, chunk): advanced one unit per issue.
  int it, ic;
  geo.locate(u0, it, ic);
  int issued = 0;
  // Unit `issued` of this CTA into slot issued % 2: weights (thread 0), then
  // zero points and scales (16-byte cp.async, at most one piece per thread)
  // and every thread's arrival.  Called by every thread.
  auto issue = [&]() {
    const int sl = issued & 1;
    const bool four = it < geo.nt4;
    const int tin = four ? it : it - geo.nt4;
    const int n0 = tin * 128;
    const int g0 = ic * (four ? 4 : 2);
    const int ng = min(four ? 4 : 2, G - g0);
    if (threadIdx.x == 0) {
      if (four) {
        mbar_arrive_expect_tx(&full[sl], static_cast<uint32_t>(ng) * 8192u);
        bulk_load(ring + sl * kGvpSlotBytes, W4 + (static_cast<int64_t>(tin) * G + g0) * 8192,
                  static_cast<uint32_t>(ng) * 8192u, &full[sl]);
      } else {
        // the whole box always lands (a group past K is filled with zeros) and is never read
        mbar_arrive_expect_tx(&full[sl], kGvpSlotBytes);
        tma_load_3d(ring + sl * kGvpSlotBytes, &tmW8, &full[sl], 0, n0, g0);
      }
    }
    uint8_t *ms = meta + sl * kGvpMetaBytes;  // z [4][64], then s_w [4][128] fp16
    const int e = threadIdx.x;
    if (e < ng * 16) {  // scales: 16 pieces per group
      const int j = e >> 4, q = e & 15;
      const __half *src = four ? s_w4 + static_cast<int64_t>(g0 + j) * N4p : s_w8 + static_cast<int64_t>(g0 + j) * N8p;
      cp_async_16(ms + 256 + j * 256 + q * 16, src + n0 + q * 8);
    } else if (four && e >= 64 && e < 64 + ng * 4) {  // zero points: 4 pieces per group
      const int j = (e - 64) >> 2, q = (e - 64) & 3;
      cp_async_16(ms + j * 64 + q * 16, z4 + static_cast<int64_t>(g0 + j) * (N4p >> 1) + (n0 >> 1) + q * 16);
    }
    cp_async_mbar_arrive(&meta_full[sl]);
    ++issued;
    if (++ic == geo.chunks(it)) {
      ++it;
      ic = 0;
    }
  };
  const int mt = M < MT ? M : MT;
  // s_a rows as bulk copies too when they are 16-byte pieces (every CTA reads
  // the same few lines: one request per token instead of a warp's loads)
  const bool sa_bulk = (G & 3) == 0 && (reinterpret_cast<uintptr_t>(s_a) & 15) == 0;
  // The first two units (weights, zero points, scales: the constant packed
  // layer) stream in while the kernel before this one finishes; the tokens'
  // codes and scales, which that kernel writes, are read after pdl_wait.
  for (int k = 0; k < 2 && k < nk; ++k) issue();
  pdl_wait();
  if (threadIdx.x == 0) {
    // the tokens' codes (and scales) of all K: one bulk copy per token
    mbar_arrive_expect_tx(a_full, static_cast<uint32_t>(mt * K + (sa_bulk ? mt * G * 4 : 0)));
    for (int m = 0; m < mt; ++m) {
      bulk_load(sA + m * K, A_q + static_cast<int64_t>(m) * K, static_cast<uint32_t>(K), a_full);
      if (sa_bulk) bulk_load(sSa + m * G, s_a + static_cast<int64_t>(m) * G, static_cast<uint32_t>(G * 4), a_full);
    }
  }

  // the tokens' scales, zero codes for tokens past M, then the sum of each
  // (token, group)'s 128 codes once they have landed
  {
    for (int e = threadIdx.x; e < (MT - mt) * (K >> 4); e += kGvThreads)
      *reinterpret_cast<int4 *>(sA + mt * K + e * 16) = make_int4(0, 0, 0, 0);
    for (int e = threadIdx.x; e < MT * G; e += kGvThreads) {
      const int m = e / G, g = e - m * G;
      if (m >= mt || !sa_bulk) sSa[e] = m < M ? s_a[static_cast<int64_t>(m) * G + g] : 0.0f;
    }
    (void)warp_wait(a_full, 0, abort_flag);
    // 8 threads per (token, group), one 16-byte piece each
    const int pieces = MT * G * 8;
    for (int e0 = 0; e0 < pieces; e0 += kGvThreads) {  // the same trip count in every thread
      const int e = e0 + static_cast<int>(threadIdx.x);
      const bool ok = e < pieces;
      const int4 v = ok ? lds_i4(sA + (e >> 3) * 128 + (e & 7) * 16) : make_int4(0, 0, 0, 0);
      int sum = __dp4a(v.x, 0x01010101, 0);
      sum = __dp4a(v.y, 0x01010101, sum);
      sum = __dp4a(v.z, 0x01010101, sum);
      sum = __dp4a(v.w, 0x01010101, sum);
      sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 1);
      sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 2);
      sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 4);
      if (ok && (e & 7) == 0) sAsum[e >> 3] = sum;  // (token, group) e / 8 = m * G + g
    }
  }
  __syncthreads();

  float acc[2][MT];
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[h][m] = 0.0f;
  int t, c;
  geo.locate(u0, t, c);
  int c_first = c;        // first chunk of the current tile segment
  bool first_seg = true;  // the CTA's first segment (its partial goes to slot 0)
  int drain_from = -1;    // thread 0: first unit whose weights were not seen to land
  for (int k = 0; k < nk; ++k) {
    const int sl = k & 1;
    const uint32_t ph = static_cast<uint32_t>((k >> 1) & 1);
    const bool four = t < geo.nt4;
    const int gpc = four ? 4 : 2;
    const int g0 = c * gpc;
    const int ng = min(gpc, G - g0);
    bool ok = warp_wait(&full[sl], ph, abort_flag);
    ok = warp_wait(&meta_full[sl], ph, abort_flag) && ok;
    if (ok) {
      const uint8_t *slot = ring + sl * kGvpSlotBytes;
      const uint8_t *ms = meta + sl * kGvpMetaBytes;
      const __half *msw = reinterpret_cast<const __half *>(ms + 256);
      if (four) {
        if (j4 < ng) {
          const int g = g0 + j4;
          const int z[2] = {(ms[j4 * 64 + (rp >> 1)] >> ((rp & 1) * 4)) & 0xF,
                            (ms[j4 * 64 + ((rp + 64) >> 1)] >> ((rp & 1) * 4)) & 0xF};
          const float sw[2] = {__half2float(msw[j4 * 128 + rp]), __half2float(msw[j4 * 128 + rp + 64])};
          int32_t *pd0 = nullptr, *pd1 = nullptr;
          if constexpr (DBG) {
            const int n0 = t * 128;
            if (n0 + rp < N4) pd0 = Pd + static_cast<int64_t>(__ldg(idx4 + n0 + rp)) * G + g;
            if (n0 + rp + 64 < N4) pd1 = Pd + static_cast<int64_t>(__ldg(idx4 + n0 + rp + 64)) * G + g;
          }
          gv_group4x2<MT, DBG>(slot + j4 * 8192, rp, sA + g * 128, K, sAsum + g, sSa + g, G, z, sw, acc, pd0, pd1,
                               static_cast<int64_t>(N) * G, M < MT ? M : MT);
        }
      } else if (j8 < ng) {
        const int g = g0 + j8;
        int32_t *pd = nullptr;
        if constexpr (DBG) {
          const int n0 = (t - geo.nt4) * 128;
          if (n0 + r8 < N8) pd = Pd + static_cast<int64_t>(__ldg(idx8 + n0 + r8)) * G + g;
        }
        gv_group8<MT, DBG>(slot + j8 * 16384 + r8 * 128, r8, sA + g * 128, K, sSa + g, G,
                           __half2float(msw[j8 * 128 + r8]), acc[0], pd, static_cast<int64_t>(N) * G, M < MT ? M : MT);
      }
    } else if (threadIdx.x == 0 && drain_from < 0) {
      drain_from = k;
    }
    __syncthreads();  // slot sl is free
    if (k + 2 < nk && !*static_cast<volatile int *>(abort_flag)) issue();

    // end of a tile segment: the unit after this one belongs to another tile, or there is none
    const bool seg_end = (k == nk - 1) || (c + 1 == geo.chunks(t));
    if (seg_end) {
      // every row's sum over the threads that hold its groups, in group order
      if (four) {
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          red[j4][rp][m] = acc[0][m];
          red[j4][rp + 64][m] = acc[1][m];
        }
      } else {
#pragma unroll
        for (int m = 0; m < MT; ++m) red[j8][r8][m] = acc[0][m];
      }
      __syncthreads();
      float y[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        y[m] = red[0][r][m];
        for (int jj = 1; jj < gpc; ++jj) y[m] += red[jj][r][m];
      }
      const bool aborted = *static_cast<volatile int *>(abort_flag) != 0;
      const int tin = four ? t : t - geo.nt4;
      const int n0 = tin * 128;
      const bool row_ok = threadIdx.x < 128 && n0 + r < (four ? N4 : N8);
      const int col_out = row_ok ? __ldg((four ? idx4 : idx8) + n0 + r) : 0;
      const bool whole = c_first == 0 && c == geo.chunks(t) - 1;
      if (whole) {
        if (row_ok && !aborted) {
#pragma unroll
          for (int m = 0; m < MT; ++m)
            if (m < mt) Y[static_cast<int64_t>(m) * N + col_out] = __float2half_rn(y[m]);
        }
      } else {
        const int slot_id = first_seg ? 0 : 1;
        if (threadIdx.x < 128) {
          float *part = ws_part + (static_cast<size_t>(b) * 2 + slot_id) * (MT * 128) + r;
#pragma unroll
          for (int m = 0; m < MT; ++m)
            if (m < mt) part[m * 128] = y[m];
        }
        const int64_t tu0 = geo.first_unit(t);
        const int b_first = geo.owner(tu0), b_last = geo.owner(tu0 + geo.chunks(t) - 1);
        // The barrier orders every thread's partial stores before thread 0's
        // counter update, whose release at GPU scope publishes them; the last
        // CTA's acquire on the same counter makes every contributor's partial
        // visible to it, and its barrier passes that on to its threads.
        __syncthreads();
        if (threadIdx.x == 0) {
          int old;
          asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;" : "=r"(old) : "l"(ws_cnt + t) : "memory");
          *last_flag = old == b_last - b_first;
        }
        __syncthreads();
        if (*last_flag) {
          if (row_ok && !aborted) {
            // contributors b_first .. b_last in K order; only b_first can hold the
            // tile as its last segment (slot 1), every later one as its first (slot 0)
            const int nb = b_last - b_first + 1;
            const bool first_in_slot1 = geo.start(b_first) < tu0;
            float z[MT];
            for (int base = 0; base < nb; base += 8) {  // eight partials in flight at a time
              float v[8][MT];
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const int bb = b_first + base + q;
                const int ps = (base + q == 0 && first_in_slot1) ? 1 : 0;
                const float *pp = ws_part + (static_cast<size_t>(bb) * 2 + ps) * (MT * 128) + r;
#pragma unroll
                for (int m = 0; m < MT; ++m) v[q][m] = (base + q < nb && m < mt) ? __ldcg(pp + m * 128) : 0.0f;
              }
#pragma unroll
              for (int q = 0; q < 8; ++q)
#pragma unroll
                for (int m = 0; m < MT; ++m)
                  if (base + q < nb) z[m] = base + q == 0 ? v[q][m] : z[m] + v[q][m];
            }
#pragma unroll
            for (int m = 0; m < MT; ++m)
              if (m < mt) Y[static_cast<int64_t>(m) * N + col_out] = __float2half_rn(z[m]);
          }
          if (threadIdx.x == 0) ws_cnt[t] = 0;  // leave the counter as it was found
        }
      }
      __syncthreads();  // the row sums are read before the next segment writes them
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[h][m] = 0.0f;
      first_seg = false;
      if (k + 1 < nk) {
        ++t;
        c = 0;
        c_first = 0;
      }
    } else {
      ++c;
    }
  }
  if (threadIdx.x == 0 && *static_cast<volatile int *>(abort_flag)) {
    // gave up: wait (bounded) for the copies still in flight
    (void)mbar_wait_drain(a_full, 0, 1ll << 30);
    for (int k = drain_from < 0 ? issued : drain_from; k < issued; ++k)
      (void)mbar_wait_drain(&full[k & 1], static_cast<uint32_t>((k >> 1) & 1), 1ll << 30);
  }
  cp_async_wait_all();  // no cp.async of this thread still in flight
}

}  // namespace mixllm

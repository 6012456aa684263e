// gemm_w4w8a8.cuh -- the fused W4.4A8 GEMM for sm_100a.
//
// What it computes (MLSys 2026 talk notes on MixLLM, notes.yuuk.io,
// §二段階逆量子化による int8 Tensor Core 活用, §高速 I2F 変換, §並列実行):
//   for every output tile of one channel set (4-bit asymmetric or 8-bit
//   symmetric) and every quantization group g of 128 along K,
//     P_g  = sum_{k in g} (W_q - z) * A_q          int8 MMA, int32 exact
//     acc += float(P_g) * s_w[n,g] * s_a[m,g]      fp32
//   then Y[m, idx[n]] = fp16(acc).
//
// How it runs on B200 (one CTA per 128 x BN output tile, both channel sets in
// the same launch, warp-specialized):
//   warp 0      TMA producer: A_q tile [128 x 128] (128-byte swizzle) and the
//               weight tile of group g -- int8 [BN x 128] for the 8-bit set,
//               packed uint4 [BN x 64 B] plus the group's zero points for the
//               4-bit set -- into a ring of kStages shared-memory stages.
//   warps 2-3   4-bit set only: unpack nibbles and subtract the zero point in
//               SWAR form (four bytes per 32-bit op, no borrow between bytes)
//               into an int8 tile in the 128-byte swizzled K-major layout the
//               tensor core reads -- the B200 counterpart of the pages' vsub4
//               pre-dequantization step (§ソフトウェアパイプライン).
//   warp 1      one thread issues 4 x tcgen05.mma.kind::i8 (K = 32 each) per
//               group into one of kAccBufs int32 accumulators in tensor memory
//               (TMEM), so the MMA of later groups overlaps the SIMT work on
//               earlier ones.
//   warps 4-11  epilogue: tcgen05.ld a group's int32 partials, convert with the
//               bias trick (bits of P + 0x4b400000 read as float equal
//               1.5*2^23 + P exactly for |P| <= 2^22) and fold the bias into an
//               exact FMA: u = fma(v, s_w, -1.5*2^23*s_w) = fl(P*s_w), since
//               1.5*2^23*s_w is exact for an fp16 s_w; then acc = fma(u, s_a,
//               acc), two f32x2 FMAs per pair of elements.  After the last
//               group, fp16 results are staged in shared memory and scattered
//               row-wise to Y[:, idx] so each warp store covers a short run of
//               one output row.
// Every wait is bounded; on a timeout the CTA records an error in the status
// word, drains its own copies and MMAs, frees TMEM and exits.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>
#include <cstdint>

#include "launch.h"
#include "ptx_sm100.cuh"

namespace mixllm {

constexpr int kBM = 128;         // tile rows (tokens) = TMEM lanes
constexpr int kKG = 128;         // K per group = K per pipeline stage
constexpr int kThreads = 384;    // 12 warps
constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr float kI2FBias = 12582912.0f;     // 1.5 * 2^23, the float with bits 0x4b400000
constexpr uint32_t kI2FBiasBits = 0x4B400000u;

template <int BN>
struct GemmCfg {
  static_assert(BN % 32 == 0 && BN >= 64 && BN <= 256, "BN");
  static constexpr int kStages = 5;
  static constexpr int kAccBufs = (4 * BN <= 512) ? 4 : 2;
  static constexpr int kTmemCols = kAccBufs * BN;  // power of two for BN in {64, 128, 256}
  static constexpr int kABytes = kBM * kKG;        // 16 KB
  static constexpr int kWBytes = BN * kKG;         // int8 weight tile
  static constexpr int kStageBytes = kABytes + kWBytes;
  static constexpr int kTBufBytes = BN * kKG;      // unpacked 4-bit tile
  static constexpr int kZBytes = 128;              // zero points of one group (BN/2 used)
  static constexpr int kColsPerThread = BN * kBM / kEpiThreads;  // BN / 2
  // shared-memory layout (offsets from a 1024-byte aligned base)
  static constexpr int kOffStages = 0;
  static constexpr int kOffTBuf = kStages * kStageBytes;
  static constexpr int kOffZ = kOffTBuf + 2 * kTBufBytes;
  static constexpr int kOffTab = kOffZ + kStages * kZBytes;  // [2][BN/2] float4
  static constexpr int kOffBar = kOffTab + 2 * (BN / 2) * 16;
  static constexpr int kNumBars = 2 * kStages + 2 + 2 + 2 * kAccBufs + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16;
  static constexpr int kSmemAlloc = kSmemBytes + 1024;
  static constexpr int kStagingStride = (BN + 2) * 2;  // bytes per staged fp16 row
  static_assert(kBM * kStagingStride <= kOffTBuf, "staging must fit in the stage ring");
  static_assert(kSmemAlloc <= 227 * 1024, "shared memory");
};

// bytes of w with 0x80 set, minus z in every byte, then back to two's complement:
// byte i of the result is (w_i - z) as int8 for w_i, z in [0, 15].
__device__ __forceinline__ uint32_t sub_zero_bytes(uint32_t w, uint32_t zz) {
  return ((w | 0x80808080u) - zz) ^ 0x80808080u;
}

template <int BN, bool kDebugP>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_w4w8a8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW4,
                       const __grid_constant__ CUtensorMap tmW8, const float *__restrict__ s_a,
                       const uint8_t *__restrict__ z4, const __half *__restrict__ s_w4,
                       const int32_t *__restrict__ idx4, const __half *__restrict__ s_w8,
                       const int32_t *__restrict__ idx8, int M, int K, int N4, int N8, int N4p, int N8p, int mt,
                       int nt4, __half *__restrict__ Y, int32_t *__restrict__ P) {
  using C = GemmCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
  uint64_t *full = bars;
  uint64_t *empty = bars + C::kStages;
  uint64_t *tfull = bars + 2 * C::kStages;
  uint64_t *tempty = tfull + 2;
  uint64_t *accfull = tempty + 2;
  uint64_t *accempty = accfull + C::kAccBufs;
  uint64_t *drain = accempty + C::kAccBufs;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kOffMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x;
  const bool is4 = tile < mt * nt4;
  const int t = is4 ? tile : tile - mt * nt4;
  const int m0 = (t % mt) * kBM;
  const int n0 = (t / mt) * BN;
  const int G = K >> 7;
  const int Nset = is4 ? N4 : N8;
  const int Np = is4 ? N4p : N8p;
  const int N = N4 + N8;
  const __half *s_w = is4 ? s_w4 : s_w8;
  const int32_t *idx = is4 ? idx4 : idx8;

  auto stage_a = [&](int s) { return smem + C::kOffStages + s * C::kStageBytes; };
  auto stage_w = [&](int s) { return smem + C::kOffStages + s * C::kStageBytes + C::kABytes; };
  auto tbuf = [&](int b) { return smem + C::kOffTBuf + b * C::kTBufBytes; };
  auto zmeta = [&](int s) { return smem + C::kOffZ + s * C::kZBytes; };
  float4 *table = reinterpret_cast<float4 *>(smem + C::kOffTab);  // [2][BN/2]

  if (threadIdx.x == 0) {
    prefetch_tmap(&tmA);
    if (is4) prefetch_tmap(&tmW4); else prefetch_tmap(&tmW8);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 2);
      mbar_init(&tempty[b], 1);
    }
    for (int a = 0; a < C::kAccBufs; ++a) {
      mbar_init(&accfull[a], 1);
      mbar_init(&accempty[a], kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0;
      const uint32_t bytes = C::kABytes + (is4 ? BN * 64 + BN / 2 : BN * kKG);
      for (int g = 0; g < G; ++g) {
        const int s = g % C::kStages;
        if (!mbar_wait(&empty[s], ((g / C::kStages) & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(&full[s], bytes);
        tma_load_2d(stage_a(s), &tmA, &full[s], g * kKG, m0);
        if (is4) {
          tma_load_2d(stage_w(s), &tmW4, &full[s], g * (kKG / 2), n0);
          bulk_load(zmeta(s), z4 + static_cast<int64_t>(g) * (N4p >> 1) + (n0 >> 1), BN / 2, &full[s]);
        } else {
          tma_load_2d(stage_w(s), &tmW8, &full[s], g * kKG, n0);
        }
        issued = g + 1;
      }
      // Let every copy this thread issued land before the CTA can exit.
      for (int g = (issued > C::kStages ? issued - C::kStages : 0); g < issued; ++g) {
        volatile int never = 0;
        (void)mbar_wait(&full[g % C::kStages], (g / C::kStages) & 1, &never, 1ll << 26);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(kBM, BN);
      for (int g = 0; g < G; ++g) {
        const int s = g % C::kStages, b = g & 1, a = g % C::kAccBufs;
        if (!mbar_wait(&full[s], (g / C::kStages) & 1, abort_flag)) break;
        if (is4 && !mbar_wait(&tfull[b], (g >> 1) & 1, abort_flag)) break;
        if (!mbar_wait(&accempty[a], ((g / C::kAccBufs) & 1) ^ 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(stage_a(s));
        const uint32_t b_addr = smem_u32(is4 ? tbuf(b) : stage_w(s));
        const uint32_t d = tmem_base + static_cast<uint32_t>(a * BN);
#pragma unroll
        for (int kk = 0; kk < kKG / 32; ++kk)
          mma_i8(d, sw128_kmajor_desc(a_addr + 32 * kk), sw128_kmajor_desc(b_addr + 32 * kk), idesc, kk > 0);
        mma_commit(&empty[s]);
        if (is4) mma_commit(&tempty[b]);
        mma_commit(&accfull[a]);
      }
      mma_commit(drain);
      volatile int never = 0;
      (void)mbar_wait(drain, 0, &never, 1ll << 28);
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ 4-bit unpack
    if (is4) {
      const int tt = threadIdx.x - 64;
      for (int g = 0; g < G; ++g) {
        const int s = g % C::kStages, b = g & 1;
        if (!mbar_wait(&full[s], (g / C::kStages) & 1, abort_flag)) break;
        if (!mbar_wait(&tempty[b], ((g >> 1) & 1) ^ 1, abort_flag)) break;
        const uint8_t *raw = stage_w(s);
        const uint8_t *zb = zmeta(s);
        uint8_t *dst = tbuf(b);
#pragma unroll 2
        for (int it = tt; it < BN * 4; it += 64) {
          const int r = it >> 2, c = it & 3;
          const uint4 x = *reinterpret_cast<const uint4 *>(raw + r * 64 + c * 16);
          const uint32_t zz = ((zb[r >> 1] >> ((r & 1) * 4)) & 0xFu) * 0x01010101u;
          uint4 lo, hi;
          lo.x = sub_zero_bytes(x.x & 0x0F0F0F0Fu, zz);
          lo.y = sub_zero_bytes(x.y & 0x0F0F0F0Fu, zz);
          lo.z = sub_zero_bytes(x.z & 0x0F0F0F0Fu, zz);
          lo.w = sub_zero_bytes(x.w & 0x0F0F0F0Fu, zz);
          hi.x = sub_zero_bytes((x.x >> 4) & 0x0F0F0F0Fu, zz);
          hi.y = sub_zero_bytes((x.y >> 4) & 0x0F0F0F0Fu, zz);
          hi.z = sub_zero_bytes((x.z >> 4) & 0x0F0F0F0Fu, zz);
          hi.w = sub_zero_bytes((x.w >> 4) & 0x0F0F0F0Fu, zz);
          const int sw = r & 7;
          *reinterpret_cast<uint4 *>(dst + r * 128 + (((2 * c) ^ sw) << 4)) = lo;
          *reinterpret_cast<uint4 *>(dst + r * 128 + (((2 * c + 1) ^ sw) << 4)) = hi;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tfull[b]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    constexpr int CPT = C::kColsPerThread;  // columns per thread
    const int e = warp - 4;                 // 0..7
    const int quad = warp & 3;              // TMEM lane quadrant of this warp
    const int half = e >> 2;                // column half
    const int row = quad * 32 + lane;
    const int m = m0 + row;
    const int et = threadIdx.x - 128;       // 0..255
    const bool row_ok = m < M;

    float acc[CPT];
#pragma unroll
    for (int j = 0; j < CPT; ++j) acc[j] = 0.0f;

    float sa_q[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) sa_q[i] = (row_ok && i < G) ? __ldg(s_a + static_cast<int64_t>(m) * G + i) : 0.0f;
    __half sw_q[2];
#pragma unroll
    for (int i = 0; i < 2; ++i)
      sw_q[i] = (et < BN && i < G) ? s_w[static_cast<int64_t>(i) * Np + n0 + et] : __float2half_rn(0.0f);

    for (int g = 0; g < G; ++g) {
      const int a = g % C::kAccBufs;
      // column scales of group g, and the exact bias term -1.5*2^23*s_w
      if (et < BN) {
        const float sw = __half2float((g & 1) ? sw_q[1] : sw_q[0]);
        float *tab = reinterpret_cast<float *>(table + (g & 1) * (BN / 2));
        tab[(et >> 1) * 4 + (et & 1)] = sw;
        tab[(et >> 1) * 4 + 2 + (et & 1)] = -kI2FBias * sw;
        const __half nxt = (g + 2 < G) ? s_w[static_cast<int64_t>(g + 2) * Np + n0 + et] : __float2half_rn(0.0f);
        if (g & 1) sw_q[1] = nxt; else sw_q[0] = nxt;
      }
      named_bar_sync(1, kEpiThreads);
      const float sa = sa_q[0];
      sa_q[0] = sa_q[1];
      sa_q[1] = sa_q[2];
      sa_q[2] = sa_q[3];
      sa_q[3] = (row_ok && g + 4 < G) ? __ldg(s_a + static_cast<int64_t>(m) * G + g + 4) : 0.0f;

      (void)mbar_wait(&accfull[a], (g / C::kAccBufs) & 1, abort_flag);
      tc_fence_after();
      const uint32_t tcol = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                            static_cast<uint32_t>(a * BN + half * CPT);
      const float4 *tab = table + (g & 1) * (BN / 2) + half * (CPT / 2);
#pragma unroll
      for (int c = 0; c < CPT / 32; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tcol + c * 32, r);
        tmem_ld_wait();
        if constexpr (kDebugP) {
          if (row_ok) {
#pragma unroll 4
            for (int j = 0; j < 32; ++j) {
              const int col = half * CPT + c * 32 + j;
              if (n0 + col < Nset)
                P[(static_cast<int64_t>(m) * N + idx[n0 + col]) * G + g] = static_cast<int32_t>(r[j]);
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float4 tv = tab[c * 16 + j];
            const float2 v = make_float2(__uint_as_float(r[2 * j] + kI2FBiasBits),
                                         __uint_as_float(r[2 * j + 1] + kI2FBiasBits));
            const float2 u = __ffma2_rn(v, make_float2(tv.x, tv.y), make_float2(tv.z, tv.w));
            const float2 o = __ffma2_rn(u, make_float2(sa, sa), make_float2(acc[c * 32 + 2 * j], acc[c * 32 + 2 * j + 1]));
            acc[c * 32 + 2 * j] = o.x;
            acc[c * 32 + 2 * j + 1] = o.y;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[a]);
    }

    if constexpr (!kDebugP) {
      // stage fp16 results: row `row`, columns half*CPT .. +CPT
      uint8_t *st = smem + C::kOffStages;
      __half2 *dst = reinterpret_cast<__half2 *>(st + row * C::kStagingStride + half * CPT * 2);
#pragma unroll
      for (int j = 0; j < CPT / 2; ++j) dst[j] = __floats2half2_rn(acc[2 * j], acc[2 * j + 1]);
      named_bar_sync(1, kEpiThreads);
      if (!*abort_flag) {
        constexpr int CPL = BN / 32;  // columns per lane
        int col_out[CPL];
        bool col_ok[CPL];
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
          const int col = lane + 32 * i;
          col_ok[i] = n0 + col < Nset;
          col_out[i] = col_ok[i] ? __ldg(idx + n0 + col) : 0;
        }
        for (int rr = e; rr < kBM; rr += kEpiWarps) {
          const int mm = m0 + rr;
          if (mm >= M) break;
          const __half *srow = reinterpret_cast<const __half *>(st + rr * C::kStagingStride);
          __half *yrow = Y + static_cast<int64_t>(mm) * N;
#pragma unroll
          for (int i = 0; i < CPL; ++i)
            if (col_ok[i]) yrow[col_out[i]] = srow[lane + 32 * i];
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

static PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

static bool encode_2d_u8(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap *map, const void *base, uint64_t inner,
                         uint64_t outer, uint32_t box_inner, uint32_t box_outer, bool swizzle128) {
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE,
                         swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int BN, bool kDebugP>
static cudaError_t launch_gemm_bn(const GemmArgs &a, cudaStream_t stream, const char **msg) {
  using C = GemmCfg<BN>;
  auto enc = get_encode_fn();
  if (!enc) {
    *msg = "cuTensorMapEncodeTiled is not available from the driver";
    return cudaErrorNotSupported;
  }
  CUtensorMap tmA, tmW4, tmW8;
  memset(&tmA, 0, sizeof(tmA));
  memset(&tmW4, 0, sizeof(tmW4));
  memset(&tmW8, 0, sizeof(tmW8));
  if (!encode_2d_u8(enc, &tmA, a.A_q, a.K, a.M, kKG, kBM, true)) {
    *msg = "tensor map encoding of A_q failed";
    return cudaErrorInvalidValue;
  }
  if (a.N4 > 0 && !encode_2d_u8(enc, &tmW4, a.W4, a.K / 2, a.N4, kKG / 2, BN, false)) {
    *msg = "tensor map encoding of W4 failed";
    return cudaErrorInvalidValue;
  }
  if (a.N8 > 0 && !encode_2d_u8(enc, &tmW8, a.W8, a.K, a.N8, kKG, BN, true)) {
    *msg = "tensor map encoding of W8 failed";
    return cudaErrorInvalidValue;
  }
  const int mt = static_cast<int>((a.M + kBM - 1) / kBM);
  const int nt4 = static_cast<int>((a.N4 + BN - 1) / BN);
  const int nt8 = static_cast<int>((a.N8 + BN - 1) / BN);
  const int64_t grid = static_cast<int64_t>(mt) * (nt4 + nt8);
  if (grid > 0x7FFFFFFF) {
    *msg = "too many tiles";
    return cudaErrorInvalidValue;
  }
  auto kern = gemm_w4w8a8_kernel<BN, kDebugP>;
  int dev = 0;
  cudaGetDevice(&dev);
  static unsigned long long configured = 0;  // one bit per device ordinal
  if (dev < 64 && !(configured & (1ull << dev))) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemAlloc);
    if (e != cudaSuccess) {
      *msg = "cudaFuncSetAttribute(MaxDynamicSharedMemorySize) failed";
      return e;
    }
    configured |= 1ull << dev;
  }
  kern<<<static_cast<unsigned>(grid), kThreads, C::kSmemAlloc, stream>>>(
      tmA, tmW4, tmW8, a.s_a, a.z4, static_cast<const __half *>(a.s_w4), a.idx4,
      static_cast<const __half *>(a.s_w8), a.idx8, static_cast<int>(a.M), static_cast<int>(a.K),
      static_cast<int>(a.N4), static_cast<int>(a.N8), static_cast<int>(padded_channels(a.N4)),
      static_cast<int>(padded_channels(a.N8)), mt, nt4, static_cast<__half *>(a.Y), a.P);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) *msg = "launch of the fused GEMM failed";
  return e;
}

cudaError_t launch_gemm_w4w8a8(const GemmArgs &a, cudaStream_t stream, const char **msg) {
  if (a.P) return launch_gemm_bn<128, true>(a, stream, msg);
  return launch_gemm_bn<128, false>(a, stream, msg);
}

}  // namespace mixllm

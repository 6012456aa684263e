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
// How it runs on B200 (one CTA of 16 warps per 128 x BN output tile, both
// channel sets in the same launch, warp-specialized, registers rebalanced
// with setmaxnreg toward the epilogue):
// The weights are the MMA's A operand (the tile's BN channels are the TMEM
// lanes of the accumulator) and the activations its B operand (kBM tokens are
// the accumulator's columns).
//   warp 0      TMA producer: the A_q tile [128 x 128] (128-byte swizzle) of
//               every group -- together with the int8 weight tile [BN x 128]
//               on 8-bit tiles -- into a ring of stages, and on 4-bit tiles
//               the packed uint4 weight tile [BN x 64 B] (one contiguous 8 KB
//               block per tile and group: a single bulk copy) and the group's
//               zero points into a ring of their own.
//   warps 1, 3  one thread each issues the MMAs of alternate groups: 4 x
//               tcgen05.mma.kind::i8 (K = 32 each) into one of kAccBufs int32
//               accumulators in tensor memory (TMEM), then one commit to the
//               group's `done` barrier, which frees the A_q stage and unpacked
//               buffer it read and hands the accumulator to the epilogue.  The
//               MMA of later groups overlaps the SIMT work on earlier ones.
//   warp 2      stages, per group, the channel scales s_w (fp32) and the token
//               scales s_a of the tile in a small ring the epilogue reads.
//   warps 12-15 4-bit set only: unpack nibbles and subtract the zero point in
//               SWAR form (four bytes per 32-bit op, no borrow between bytes)
//               -- the B200 counterpart of the pages' vsub4 pre-dequantization
//               step (§ソフトウェアパイプライン) -- and store the int8 rows
//               with tcgen05.st into a TMEM buffer, from which the MMA reads
//               its A operand: the unpacked tile never touches shared memory,
//               so the tensor core's shared-memory reads per group halve.
//   warps 4-11  epilogue: tcgen05.ld a group's int32 partials, which the
//               accumulator already holds biased by 0x4b400000 (TMEM is preset
//               to the bias), so their bits read as float are 1.5*2^23 + P
//               exactly for |P| <= 2^22 -- the bias trick with no integer add.
//               The bias is folded into one FMA with the channel scale:
//               u = fma(v, s_w, -1.5*2^23*s_w) = fl(P*s_w), one rounding,
//               because 1.5*2^23*s_w is exact for an fp16-valued s_w; then
//               acc = fma(u, s_a, acc): two f32x2 FMAs per pair of elements,
//               one shared-memory load per four.  After the last group, fp16
//               results are staged in shared memory and scattered row-wise to
//               Y[:, idx] so each warp store covers a short run of one output
//               row.
// Every ring slot is refilled as soon as its own consumer is done with it (the
// A stages and unpacked buffers through the group's `done` barrier, the packed
// tiles through the unpack warps), and the rings are deep enough to cover the
// load latency of HBM.  Every wait is bounded; on a timeout the CTA records
// an error in the status word, drains its own copies and MMAs, frees TMEM and
// exits.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>
#include <cstdint>
#include <mutex>

#include "launch.h"
#include "ptx_sm100.cuh"

namespace mixllm {

constexpr int kBM = 128;         // tile rows (tokens) = TMEM lanes
constexpr int kKG = 128;         // K per group = K per pipeline stage
constexpr int kThreads = 512;    // 16 warps = 4 warpgroups
constexpr int kEpiWarps = 8;     // warps 4..11
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kXformWarps = 4;   // warps 12..15
constexpr float kI2FBias = 12582912.0f;     // 1.5 * 2^23, the float with bits 0x4b400000
constexpr uint32_t kI2FBiasBits = 0x4B400000u;
// register split (all four warpgroups together must stay within 65536):
// 128 * (kRegsCtl + kRegsXform) + 256 * kRegsEpi <= 512 * 128 (the launch's registers)
constexpr int kRegsCtl = 88, kRegsXform = 72, kRegsEpi = 176;
static_assert(128 * (kRegsCtl + kRegsXform) + 256 * kRegsEpi <= 65536, "register split");

template <int BN>
struct GemmCfg {
  static_assert(BN == 128, "the warp roles below are laid out for BN = 128");
  static constexpr int kABytes = kBM * kKG;        // 16 KB A_q tile of one group
  static constexpr int kW8Bytes = BN * kKG;        // 16 KB int8 weight tile
  static constexpr int kW4Bytes = BN * kKG / 2;    //  8 KB packed uint4 weight tile
  static constexpr int kZBytes = BN / 2;           // zero points of one group, two per byte
  // The ring region is laid out one of two ways, chosen per CTA:
  //   8-bit tile: kStages8 stages of [A | W8]                      (32 KB each)
  //   4-bit tile: kStagesA4 A stages and kRaw packed tiles          (16/8 KB)
  // The unpacked 4-bit tiles live in tensor memory (kTBufs buffers of 32
  // columns), where the MMA reads its weight operand: they take no shared
  // memory and no shared-memory bandwidth.
  static constexpr int kStages8 = 6;
  static constexpr int kStagesA4 = 8;
  static constexpr int kTBufs = 8;
  static constexpr int kRaw = 8;
  static constexpr int kMaxStages = kStages8 > kStagesA4 ? kStages8 : kStagesA4;
  // Two threads issue the MMAs of alternate groups.  Every barrier an issuer
  // waits on must belong to one issuer only, or a parity wait could see a
  // phase meant for the other one: the slot counts of those rings are even.
  static_assert(kStages8 % 2 == 0 && kStagesA4 % 2 == 0 && kTBufs % 2 == 0, "rings the issuers wait on");
  // One commit per group, to done[g % kDone]; a waiter never falls a full ring
  // behind as long as kDone covers every ring that is released through it.
  static constexpr int kDone = kMaxStages > kTBufs ? kMaxStages : kTBufs;
  static constexpr int kRing8 = kStages8 * (kABytes + kW8Bytes);
  static constexpr int kRing4 = kStagesA4 * kABytes + kRaw * kW4Bytes;
  static constexpr int kRingBytes = kRing8 > kRing4 ? kRing8 : kRing4;
  static constexpr int kAccBufs = 2;
  static_assert(kAccBufs % 2 == 0, "accumulators alternate between the issuers");
  static_assert(kDone >= kStages8 && kDone >= kStagesA4 && kDone >= kTBufs && kDone >= kAccBufs, "done ring");
  static constexpr int kTabSlots = 4;
  // tensor memory: kAccBufs int32 accumulators of kBM (token) columns, then
  // the unpacked weight tiles, 128 bytes of K per lane = 32 columns each
  static constexpr int kTmemABase = kAccBufs * kBM;
  static constexpr int kTmemABufCols = kKG / 4;
  static constexpr int kTmemCols = 512;
  static_assert(kTmemABase + kTBufs * kTmemABufCols <= kTmemCols, "tensor memory");
  static constexpr int kColsPerThread = BN * kBM / kEpiThreads;  // 64
  static constexpr int kTabSwBytes = BN * 4;                   // s_w of the tile's columns (fp32)
  static constexpr int kTabBytes = kTabSwBytes + kBM * 4;      // + s_a of the tile's rows
  static constexpr int kStgSlots = 12;                         // raw scale staging ring
  static constexpr int kStgDist = 10;                          // groups prefetched ahead
  static constexpr int kStgBytes = BN * 2 + kBM * 4;           // raw fp16 s_w + fp32 s_a
  // shared-memory layout (offsets from a 1024-byte aligned base)
  static constexpr int kOffRing = 0;
  static constexpr int kOffZ = kOffRing + kRingBytes;
  static constexpr int kOffTab = kOffZ + kRaw * kZBytes;
  static constexpr int kOffStg = kOffTab + kTabSlots * kTabBytes;
  static constexpr int kOffIdx = kOffStg + kStgSlots * kStgBytes;  // output channel of each tile column
  static constexpr int kOffBar = kOffIdx + BN * 4;
  // full per stage, done per group ring, full/empty per packed tile, full per unpacked buffer,
  // empty per accumulator, full/empty per table slot, one drain per issuer
  static constexpr int kNumBars = kMaxStages + kDone + 2 * kRaw + kTBufs + kAccBufs + 2 * kTabSlots + 2;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16;
  static constexpr int kSmemAlloc = kSmemBytes + 1024;
  static constexpr int kStagingStride = (BN + 2) * 2;  // bytes per staged fp16 row
  static_assert(kBM * kStagingStride <= kRingBytes, "staging must fit in the ring region");
  static_assert(kABytes % 1024 == 0 && kW8Bytes % 1024 == 0, "swizzled tiles need 1024-byte alignment");
  static_assert(kSmemAlloc <= 227 * 1024, "shared memory");
};

// bytes of w with 0x80 set, minus z in every byte, then back to two's complement:
// byte i of the result is (w_i - z) as int8 for w_i, z in [0, 15].
__device__ __forceinline__ uint32_t sub_zero_bytes(uint32_t w, uint32_t zz) {
  return ((w | 0x80808080u) - zz) ^ 0x80808080u;
}

template <int BN, bool kDebugP>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_w4w8a8_kernel(const __grid_constant__ CUtensorMap tmA, const uint8_t *__restrict__ W4,
                       const __grid_constant__ CUtensorMap tmW8, const float *__restrict__ s_a,
                       const uint8_t *__restrict__ z4, const __half *__restrict__ s_w4,
                       const int32_t *__restrict__ idx4, const __half *__restrict__ s_w8,
                       const int32_t *__restrict__ idx8, int M, int K, int N4, int N8, int N4p, int N8p, int mt,
                       int nt4, __half *__restrict__ Y, int32_t *__restrict__ P) {
  using C = GemmCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
  uint64_t *full = bars;                          // TMA -> MMA              (per stage)
  uint64_t *done = full + C::kMaxStages;          // MMA commit of group g   (ring of kDone): frees the
                                                  // group's A stage and unpacked buffer, fills its accumulator
  uint64_t *rfull = done + C::kDone;              // TMA -> unpack           (per packed tile)
  uint64_t *rempty = rfull + C::kRaw;             // unpack -> TMA           (per packed tile)
  uint64_t *tfull = rempty + C::kRaw;             // unpack -> MMA           (per unpacked buffer)
  uint64_t *accempty = tfull + C::kTBufs;         // epilogue -> MMA         (per TMEM accumulator)
  uint64_t *tabfull = accempty + C::kAccBufs;     // scale warp -> epilogue  (per table slot)
  uint64_t *tabempty = tabfull + C::kTabSlots;    // epilogue -> scale warp
  uint64_t *drain = tabempty + C::kTabSlots;      // [2]: each MMA issuer's final commit
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
  const int S = is4 ? C::kStagesA4 : C::kStages8;  // A stages of this tile

  // ring region: 8-bit tiles [A | W8] x kStages8; 4-bit tiles A x kStagesA4, then the packed tiles
  const int stage_bytes = is4 ? C::kABytes : C::kABytes + C::kW8Bytes;
  auto stage_a = [&](int s) { return smem + C::kOffRing + s * stage_bytes; };
  auto stage_w8 = [&](int s) { return smem + C::kOffRing + s * stage_bytes + C::kABytes; };
  auto raw_w4 = [&](int r) { return smem + C::kOffRing + C::kStagesA4 * C::kABytes + r * C::kW4Bytes; };
  auto zmeta = [&](int r) { return smem + C::kOffZ + r * C::kZBytes; };
  auto table = [&](int slot) { return reinterpret_cast<float4 *>(smem + C::kOffTab + slot * C::kTabBytes); };
  auto table_sw = [&](int slot) { return reinterpret_cast<const float *>(smem + C::kOffTab + slot * C::kTabBytes); };
  auto table_sa = [&](int slot) {
    return reinterpret_cast<float *>(smem + C::kOffTab + slot * C::kTabBytes + C::kTabSwBytes);
  };
  auto stg_sw = [&](int i) { return smem + C::kOffStg + i * C::kStgBytes; };
  auto stg_sa = [&](int i) { return reinterpret_cast<float *>(smem + C::kOffStg + i * C::kStgBytes + BN * 2); };
  int32_t *col_idx = reinterpret_cast<int32_t *>(smem + C::kOffIdx);

  // Loads of the A ring (and of W8 on 8-bit tiles) for group g into stage g % S.
  const uint32_t a_bytes = static_cast<uint32_t>(is4 ? C::kABytes : C::kABytes + C::kW8Bytes);
  auto load_a = [&](int g) {
    const int s = g % S;
    mbar_arrive_expect_tx(&full[s], a_bytes);
    tma_load_2d(stage_a(s), &tmA, &full[s], g * kKG, m0);
    if (!is4) tma_load_2d(stage_w8(s), &tmW8, &full[s], g * kKG, n0);
  };
  // Loads of the packed 4-bit tile and zero points of group g into slot g % kRaw.
  auto load_raw = [&](int g) {
    const int r = g % C::kRaw;
    mbar_arrive_expect_tx(&rfull[r], static_cast<uint32_t>(C::kW4Bytes + C::kZBytes));
    // the tile's packed group is one contiguous block: one bulk copy
    bulk_load(raw_w4(r), W4 + (static_cast<int64_t>(n0 >> 7) * G + g) * C::kW4Bytes, C::kW4Bytes, &rfull[r]);
    bulk_load(zmeta(r), z4 + static_cast<int64_t>(g) * (N4p >> 1) + (n0 >> 1), C::kZBytes, &rfull[r]);
  };

  if (threadIdx.x == 0) {
    prefetch_tmap(&tmA);
    if (!is4) prefetch_tmap(&tmW8);
    for (int s = 0; s < C::kMaxStages; ++s) mbar_init(&full[s], 1);
    for (int i = 0; i < C::kDone; ++i) mbar_init(&done[i], 1);
    for (int r = 0; r < C::kRaw; ++r) {
      mbar_init(&rfull[r], 1);
      mbar_init(&rempty[r], kXformWarps);
    }
    for (int b = 0; b < C::kTBufs; ++b) mbar_init(&tfull[b], kXformWarps);
    for (int a = 0; a < C::kAccBufs; ++a) mbar_init(&accempty[a], kEpiWarps);
    for (int i = 0; i < C::kTabSlots; ++i) {
      mbar_init(&tabfull[i], 1);
      mbar_init(&tabempty[i], kEpiWarps);
    }
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
    // Every global read of this grid comes after this wait: here, in the
    // table warp, and in the roles ordered after these loads by barriers.
    pdl_wait();
    // the first stages need nothing but their barriers: start them before the CTA-wide sync
    for (int g = 0; g < S && g < G; ++g) load_a(g);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < 4) {
    regs_dec<kRegsCtl>();
    if (warp == 0) {
      // ---------------------------------------------------------- TMA producer
      // One thread feeds both rings: the A stages (with W8 on 8-bit tiles),
      // each refilled once the MMAs of the group that held it are done, and on
      // 4-bit tiles the packed W4 tiles, each refilled once unpacked.  It
      // polls both, so neither ring waits on the other.  (L2 prefetch hints
      // ahead of the rings measured slower: they compete with the loads for
      // the TMA unit's requests.)
      if (lane == 0) {
        int ga = S < G ? S : G;  // next A group; the prologue issued groups 0 .. S-1
        int gw = is4 ? 0 : G;    // next packed W4 group
        long long idle_since = -1;
        while (ga < G || gw < G) {
          bool progressed = false;
          // packed slot gw % kRaw last held group gw - kRaw; the unpack warps released it
          if (gw < G &&
              (gw < C::kRaw || mbar_try_wait(smem_u32(&rempty[gw % C::kRaw]), ((gw / C::kRaw) - 1) & 1))) {
            load_raw(gw);
            ++gw;
            progressed = true;
          }
          // A stage ga % S last held group ga - S; it is free once that group is done
          if (ga < G && mbar_try_wait(smem_u32(&done[(ga - S) % C::kDone]), ((ga - S) / C::kDone) & 1)) {
            load_a(ga);
            ++ga;
            progressed = true;
          }
          if (progressed) {
            idle_since = -1;
            continue;
          }
          if (*abort_flag) break;
          const long long now = clock64();
          if (idle_since < 0) {
            idle_since = now;
          } else if (now - idle_since > (1ll << 32)) {
            *abort_flag = 1;
            record_status(kStatusTimeout);
            break;
          }
          __nanosleep(64);
        }
        // let every copy this thread issued land before the CTA can exit
        for (int g = (ga > S ? ga - S : 0); g < ga; ++g) (void)mbar_wait_drain(&full[g % S], (g / S) & 1, 1ll << 26);
        if (is4)
          for (int g = (gw > C::kRaw ? gw - C::kRaw : 0); g < gw; ++g)
            (void)mbar_wait_drain(&rfull[g % C::kRaw], (g / C::kRaw) & 1, 1ll << 26);
      }
    } else if (warp == 1 || warp == 3) {
      // ---------------------------------------------------------- MMA issuers
      // Two threads issue alternate groups (warp 1 the even ones, warp 3 the
      // odd ones): one thread pays for every tcgen05.mma and commit it issues
      // and leaves the tensor pipe idle between groups, two keep it busy.
      // The weights are the MMA's A operand (BN channels = the TMEM lanes of
      // the accumulator), the activations its B operand (kBM token columns):
      // on 4-bit tiles A comes from the unpacked buffer in tensor memory.
      if (lane == 0) {
        constexpr uint32_t idesc = idesc_i8(BN, kBM);
        const int who = warp == 1 ? 0 : 1;
        for (int g = who; g < G; g += 2) {
          const int s = g % S, b = g % C::kTBufs, a = g % C::kAccBufs;
          if (!mbar_wait(&full[s], (g / S) & 1, abort_flag)) break;
          if (is4 && !mbar_wait(&tfull[b], (g / C::kTBufs) & 1, abort_flag)) break;
          // phase 0 of accempty[a] is the epilogue's bias fill; phase u+1 its drain of use u
          if (!mbar_wait(&accempty[a], (g / C::kAccBufs) & 1, abort_flag)) break;
          tc_fence_after();
          const uint32_t x_addr = smem_u32(stage_a(s));
          const uint32_t d = tmem_base + static_cast<uint32_t>(a * kBM);
          if (is4) {
            const uint32_t wt = tmem_base + static_cast<uint32_t>(C::kTmemABase + b * C::kTmemABufCols);
#pragma unroll
            for (int kk = 0; kk < kKG / 32; ++kk)
              mma_i8_ts(d, wt + 8 * kk, sw128_kmajor_desc(x_addr + 32 * kk), idesc, 1u);
          } else {
            const uint32_t w_addr = smem_u32(stage_w8(s));
#pragma unroll
            for (int kk = 0; kk < kKG / 32; ++kk)
              mma_i8(d, sw128_kmajor_desc(w_addr + 32 * kk), sw128_kmajor_desc(x_addr + 32 * kk), idesc, 1u);
          }
          mma_commit(&done[g % C::kDone]);
        }
        mma_commit(&drain[who]);
        (void)mbar_wait_drain(&drain[who], 0, 1ll << 28);
      }
    } else {
      // ---------------------------------------------------------- scale table
      // Slot `slot` of group g holds s_w of the tile's BN columns as fp32,
      // followed by s_a of the tile's 128 rows.  Raw scales are prefetched
      // kStgDist groups ahead with cp.async into a staging ring, so no load
      // latency sits on the epilogue's path.
      auto issue = [&](int g) {
        if (g < G) {
          const int i = g % C::kStgSlots;
          cp_async_8(stg_sw(i) + 8 * lane, s_w + static_cast<int64_t>(g) * Np + n0 + 4 * lane);
#pragma unroll
          for (int j = 0; j < kBM / 32; ++j) {
            const int row = lane + 32 * j;
            const bool in = m0 + row < M;
            cp_async_4(stg_sa(i) + row, s_a + (in ? static_cast<int64_t>(m0 + row) * G + g : 0), in ? 4u : 0u);
          }
        }
        cp_async_commit();
      };
      pdl_wait();
      // The row scales of this tile are whole rows of s_a [M, G] (one
      // contiguous range) and its column scales one 2*BN-byte piece per group:
      // bring both into L2 first, so the scattered 4-byte reads below hit there.
      if (lane == 0) {
        const int rows = M - m0 < kBM ? M - m0 : kBM;
        const uint32_t sa_bytes = static_cast<uint32_t>(rows) * static_cast<uint32_t>(G) * 4u;
        const float *sa_rows = s_a + static_cast<int64_t>(m0) * G;  // s_a is only 4-byte aligned
        if (sa_bytes >= 16 && (reinterpret_cast<uintptr_t>(sa_rows) & 15u) == 0) bulk_prefetch_l2(sa_rows, sa_bytes & ~15u);
      }
      for (int g = lane; g < G; g += 32) bulk_prefetch_l2(s_w + static_cast<int64_t>(g) * Np + n0, BN * 2);
      for (int g = 0; g < C::kStgDist; ++g) issue(g);
      // output channel of every tile column (-1 past the set), published to
      // the epilogue by the first tabfull arrival
#pragma unroll
      for (int i = 0; i < BN / 32; ++i) {
        const int col = lane + 32 * i;
        col_idx[col] = n0 + col < Nset ? __ldg(idx + n0 + col) : -1;
      }
      for (int g = 0; g < G; ++g) {
        const int slot = g % C::kTabSlots, i = g % C::kStgSlots;
        cp_async_wait<C::kStgDist - 1>();
        __syncwarp();
        if (!warp_wait(&tabempty[slot], ((g / C::kTabSlots) & 1) ^ 1, abort_flag)) break;
        const uint2 raw = *reinterpret_cast<const uint2 *>(stg_sw(i) + 8 * lane);
        const float2 a = __half22float2(*reinterpret_cast<const __half2 *>(&raw.x));
        const float2 b = __half22float2(*reinterpret_cast<const __half2 *>(&raw.y));
        table(slot)[lane] = make_float4(a.x, a.y, b.x, b.y);
        float *tsa = table_sa(slot);
        const float *ssa = stg_sa(i);
#pragma unroll
        for (int j = 0; j < kBM / 32; ++j) tsa[lane + 32 * j] = ssa[lane + 32 * j];
        __syncwarp();
        if (lane == 0) mbar_arrive(&tabfull[slot]);
        issue(g + C::kStgDist);
      }
      cp_async_wait<0>();
    }
  } else if (warp >= 12) {
    regs_dec<kRegsXform>();
    // ------------------------------------------------------------ 4-bit unpack
    if (is4) {
      // Warp 12 + q writes TMEM lane quadrant q: thread `lane` unpacks weight
      // row rr = 32q + lane of the tile (64 packed bytes -> 128 int8 values)
      // and stores it as the 32 columns of its lane in the group's buffer.
      // The packed rows are 64 bytes apart, so lanes read their four 16-byte
      // chunks in a rotated order (8 distinct bank groups per load) and the
      // rotation is undone in registers.
      const int q = warp & 3;
      const int rr = q * 32 + lane;
      const int rot = (lane >> 1) & 3;
      const int zshift = (rr & 1) * 4;
      const uint32_t trow = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + C::kTmemABase;
      for (int g = 0; g < G; ++g) {
        const int r = g % C::kRaw, b = g % C::kTBufs;
        if (!warp_wait(&rfull[r], (g / C::kRaw) & 1, abort_flag)) break;
        // buffer b last held group g - kTBufs: free once that group's MMAs are done
        if (g >= C::kTBufs) {
          const int gp = g - C::kTBufs;
          if (!warp_wait(&done[gp % C::kDone], (gp / C::kDone) & 1, abort_flag)) break;
          tc_fence_after();
        }
        const uint8_t *src = raw_w4(r) + rr * 64;
        uint4 x[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) x[c] = *reinterpret_cast<const uint4 *>(src + (((c + rot) & 3) << 4));
        const uint32_t zz = ((static_cast<uint32_t>(zmeta(r)[rr >> 1]) >> zshift) & 0xFu) * 0x01010101u;
        // x[c] holds chunk (c + rot) & 3: rotate back by rot = (rot & 1) + (rot & 2)
        if (rot & 1) {
          const uint4 t3 = x[3];
          x[3] = x[2];
          x[2] = x[1];
          x[1] = x[0];
          x[0] = t3;
        }
        if (rot & 2) {
          const uint4 t0 = x[0], t1 = x[1];
          x[0] = x[2];
          x[1] = x[3];
          x[2] = t0;
          x[3] = t1;
        }
        // chunk c: low nibbles are k = 32c .. 32c+15 (columns 8c .. 8c+3),
        // high nibbles k = 32c+16 .. 32c+31 (columns 8c+4 .. 8c+7)
        uint32_t o[32];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          o[8 * c + 0] = sub_zero_bytes(x[c].x & 0x0F0F0F0Fu, zz);
          o[8 * c + 1] = sub_zero_bytes(x[c].y & 0x0F0F0F0Fu, zz);
          o[8 * c + 2] = sub_zero_bytes(x[c].z & 0x0F0F0F0Fu, zz);
          o[8 * c + 3] = sub_zero_bytes(x[c].w & 0x0F0F0F0Fu, zz);
          o[8 * c + 4] = sub_zero_bytes((x[c].x >> 4) & 0x0F0F0F0Fu, zz);
          o[8 * c + 5] = sub_zero_bytes((x[c].y >> 4) & 0x0F0F0F0Fu, zz);
          o[8 * c + 6] = sub_zero_bytes((x[c].z >> 4) & 0x0F0F0F0Fu, zz);
          o[8 * c + 7] = sub_zero_bytes((x[c].w >> 4) & 0x0F0F0F0Fu, zz);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&rempty[r]);  // the packed tile is in registers
        tmem_st_32x32b_x32(trow + static_cast<uint32_t>(b * C::kTmemABufCols), o);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tfull[b]);
      }
    }
  } else {
    regs_inc<kRegsEpi>();
    // ------------------------------------------------------------ epilogue
    // The accumulator is D[channel, token]: this thread owns channel `ch` of
    // the tile (its TMEM lane) and the tokens half*CPT .. half*CPT+CPT-1.
    constexpr int CPT = C::kColsPerThread;  // 64 token columns per thread
    const int e = warp - 4;                 // 0..7
    const int quad = warp & 3;              // TMEM lane quadrant of this warp
    const int half = e >> 2;                // column half
    const int ch = quad * 32 + lane;

    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + half * CPT;
    // Every accumulator starts at the bias 0x4b400000 (and is reset to it after
    // each drain), so the int32 sum the MMAs leave there, read as a float, is
    // 1.5*2^23 + P exactly: the bias trick with no per-element integer add.
#pragma unroll
    for (int a = 0; a < C::kAccBufs; ++a)
#pragma unroll
      for (int c = 0; c < CPT; c += 32) tmem_st_32x32b_x32_fill(lane_base + a * kBM + c, kI2FBiasBits);
    tmem_st_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0)
      for (int a = 0; a < C::kAccBufs; ++a) mbar_arrive(&accempty[a]);

    float acc[CPT];
#pragma unroll
    for (int j = 0; j < CPT; ++j) acc[j] = 0.0f;

    // Software pipeline over 16-column chunks: while one chunk is converted
    // and accumulated, the tcgen05.ld of the next one (this group's next
    // chunk, or the next group's first) is in flight.
    constexpr int CW = 16, NCH = CPT / CW;
    uint32_t rbuf[2][CW];
    // v = bits of (1.5*2^23 + P) as float; u = fma(v, s_w, -1.5*2^23*s_w) is
    // exactly fl(P * s_w): the bias term 1.5*2^23*s_w is exact for an
    // fp16-valued s_w and the fma rounds v*s_w - 1.5*2^23*s_w = P*s_w once.
    // Then acc += u * s_a.  tab holds the s_a of 4 consecutive tokens per float4.
    auto convert = [&](uint32_t(&r)[CW], const float4 *tab, float2 sw2, float2 cb2, int c0) {
#pragma unroll
      for (int j = 0; j < CW / 4; ++j) {
        const float4 sa = tab[j];
        const float2 v0 = make_float2(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]));
        const float2 v1 = make_float2(__uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
        const float2 u0 = __ffma2_rn(v0, sw2, cb2);
        const float2 u1 = __ffma2_rn(v1, sw2, cb2);
        const float2 o0 = __ffma2_rn(u0, make_float2(sa.x, sa.y), make_float2(acc[c0 + 4 * j], acc[c0 + 4 * j + 1]));
        const float2 o1 =
            __ffma2_rn(u1, make_float2(sa.z, sa.w), make_float2(acc[c0 + 4 * j + 2], acc[c0 + 4 * j + 3]));
        acc[c0 + 4 * j] = o0.x;
        acc[c0 + 4 * j + 1] = o0.y;
        acc[c0 + 4 * j + 2] = o1.x;
        acc[c0 + 4 * j + 3] = o1.y;
      }
    };
    auto dump = [&](uint32_t(&r)[CW], int g, int c0) {
      if (n0 + ch < Nset) {
        const int64_t nout = idx[n0 + ch];
#pragma unroll 4
        for (int j = 0; j < CW; ++j) {
          const int m = m0 + half * CPT + c0 + j;
          if (m < M) P[(static_cast<int64_t>(m) * N + nout) * G + g] = static_cast<int32_t>(r[j] - kI2FBiasBits);
        }
      }
    };

    bool live = warp_wait(&done[0], 0, abort_flag);
    if (live) {
      tc_fence_after();
      tmem_ld_32x32b_x16(lane_base, rbuf[0]);
    }
    for (int g = 0; live && g < G; ++g) {
      const int a = g % C::kAccBufs, slot = g % C::kTabSlots;
      const uint32_t col = lane_base + static_cast<uint32_t>(a * kBM);
      if (!warp_wait(&tabfull[slot], (g / C::kTabSlots) & 1, abort_flag)) break;
      const float sw = table_sw(slot)[ch];
      const float2 sw2 = make_float2(sw, sw);
      const float2 cb2 = make_float2(-kI2FBias * sw, -kI2FBias * sw);
      const float4 *tab = reinterpret_cast<const float4 *>(table_sa(slot)) + half * (CPT / 4);
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        tmem_ld_wait();
        reg_fence(rbuf[c & 1]);
        if (c + 1 < NCH) tmem_ld_32x32b_x16(col + CW * (c + 1), rbuf[(c + 1) & 1]);
        tmem_st_32x32b_x16_fill(col + CW * c, kI2FBiasBits);  // hand the chunk back preset to the bias
        if (c + 1 == NCH) {
          // Every partial of group g is in registers and its accumulator is
          // reset: release the accumulator before waiting for group g+1, so
          // the MMAs can run kAccBufs groups ahead of this warp.
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&accempty[a]);
          if (g + 1 < G) {
            const int a1 = (g + 1) % C::kAccBufs;
            live = warp_wait(&done[(g + 1) % C::kDone], ((g + 1) / C::kDone) & 1, abort_flag);
            if (live) {
              tc_fence_after();
              tmem_ld_32x32b_x16(lane_base + static_cast<uint32_t>(a1 * kBM), rbuf[(c + 1) & 1]);
            }
          }
        }
        if constexpr (kDebugP) {
          dump(rbuf[c & 1], g, CW * c);
        } else {
          convert(rbuf[c & 1], tab + (CW / 4) * c, sw2, cb2, CW * c);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&tabempty[slot]);  // table slot read for the last time
    }
    tmem_ld_wait();

    if constexpr (!kDebugP) {
      // stage fp16 results as [token][channel]: column `ch`, token rows
      // half*CPT .. +CPT (a warp's stores cover 64 contiguous bytes of a row)
      uint8_t *st = smem + C::kOffRing;
      __half *dst = reinterpret_cast<__half *>(st + half * CPT * C::kStagingStride) + ch;
#pragma unroll
      for (int j = 0; j < CPT; ++j) dst[j * (C::kStagingStride / 2)] = __float2half_rn(acc[j]);
      named_bar_sync(1, kEpiThreads);
      if (!*abort_flag) {
        constexpr int CPL = BN / 32;  // columns per lane
        int col_out[CPL];
#pragma unroll
        for (int i = 0; i < CPL; ++i) col_out[i] = col_idx[lane + 32 * i];
        for (int rr = e; rr < kBM; rr += kEpiWarps) {
          const int mm = m0 + rr;
          if (mm >= M) break;
          const __half *srow = reinterpret_cast<const __half *>(st + rr * C::kStagingStride);
          __half *yrow = Y + static_cast<int64_t>(mm) * N;
#pragma unroll
          for (int i = 0; i < CPL; ++i)
            if (col_out[i] >= 0) yrow[col_out[i]] = srow[lane + 32 * i];
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

static bool encode_2d_u8_uncached(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap *map, const void *base,
                                  uint64_t inner, uint64_t outer, uint32_t box_inner, uint32_t box_outer,
                                  bool swizzle128) {
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

// The descriptor is a pure function of its arguments, so encoded ones are
// kept (a small round-robin table) and reused: a layer called again with the
// same buffers skips the host-side encoding.
static bool encode_2d_u8(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap *map, const void *base, uint64_t inner,
                         uint64_t outer, uint32_t box_inner, uint32_t box_outer, bool swizzle128) {
  struct Entry {
    const void *base;
    uint64_t inner, outer;
    uint32_t box_inner, box_outer;
    bool swizzle;
    bool valid;
    CUtensorMap map;
  };
  static Entry table[64];
  static int next = 0;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  for (const Entry &e : table)
    if (e.valid && e.base == base && e.inner == inner && e.outer == outer && e.box_inner == box_inner &&
        e.box_outer == box_outer && e.swizzle == swizzle128) {
      *map = e.map;
      return true;
    }
  if (!encode_2d_u8_uncached(enc, map, base, inner, outer, box_inner, box_outer, swizzle128)) return false;
  table[next] = Entry{base, inner, outer, box_inner, box_outer, swizzle128, true, *map};
  next = (next + 1) % 64;
  return true;
}

template <int BN, bool kDebugP>
static cudaError_t launch_gemm_bn(const GemmArgs &a, cudaStream_t stream, const char **msg) {
  using C = GemmCfg<BN>;
  auto enc = get_encode_fn();
  if (!enc) {
    *msg = "cuTensorMapEncodeTiled is not available from the driver";
    return cudaErrorNotSupported;
  }
  CUtensorMap tmA, tmW8;
  memset(&tmA, 0, sizeof(tmA));
  memset(&tmW8, 0, sizeof(tmW8));
  if (!encode_2d_u8(enc, &tmA, a.A_q, a.K, a.M, kKG, kBM, true)) {
    *msg = "tensor map encoding of A_q failed";
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
  // Launched as a programmatic dependent of the previous kernel in the stream:
  // the CTAs set up barriers and TMEM while that kernel finishes, and wait for
  // it (griddepcontrol.wait) before their first global read.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::kSmemAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(
      &cfg, kern, tmA, a.W4, tmW8, a.s_a, a.z4, static_cast<const __half *>(a.s_w4), a.idx4,
      static_cast<const __half *>(a.s_w8), a.idx8, static_cast<int>(a.M), static_cast<int>(a.K),
      static_cast<int>(a.N4), static_cast<int>(a.N8), static_cast<int>(padded_channels(a.N4)),
      static_cast<int>(padded_channels(a.N8)), mt, nt4, static_cast<__half *>(a.Y), a.P);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) *msg = "launch of the fused GEMM failed";
  return e;
}

cudaError_t launch_gemm_w4w8a8(const GemmArgs &a, cudaStream_t stream, const char **msg) {
  if (a.P) return launch_gemm_bn<128, true>(a, stream, msg);
  return launch_gemm_bn<128, false>(a, stream, msg);
}

}  // namespace mixllm

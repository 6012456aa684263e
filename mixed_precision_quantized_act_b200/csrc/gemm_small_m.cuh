// gemm_small_m.cuh -- the W4.4A8 layer for few tokens (M <= 64) on sm_100a.
//
// Same arithmetic as the tiled kernel (MLSys 2026 talk notes on MixLLM,
// notes.yuuk.io, §二段階逆量子化による int8 Tensor Core 活用, §高速 I2F 変換,
// §並列実行): per quantization group g of 128 along K,
//     P_g  = sum_{k in g} (W_q - z) * A_q          int8 MMA, int32 exact
//     acc += float(P_g) * s_w[n,g] * s_a[m,g]      fp32
// and Y[m, idx[n]] = fp16(acc).  With a handful of tokens the layer is bound
// by HBM (the packed weights are nearly all the bytes), so the work is laid
// out for bandwidth rather than for the tensor pipe:
//   * operands swapped: the weight tile is the MMA's M = 128 side (TMEM lane =
//     output channel) and the tokens its N side (Mp = 16, 32 or 64 columns), so
//     the per-group drain is 128 x Mp values instead of 128 x 128, and the
//     channel scale is a per-thread constant (the bias fold uses s_w:
//     u = fma(v, s_w, -1.5*2^23*s_w) = fl(P*s_w), exact because s_w is fp16);
//   * split-K: the groups of every 128-channel tile are divided among S CTAs
//     so that the grid fills the SMs; each CTA writes its fp32 partial sums to
//     a workspace and the last CTA of a tile to finish (an atomic counter, no
//     waiting) adds the S partials in split order -- the result does not
//     depend on which CTA finishes last -- and writes the fp16 outputs.  The
//     counter is reset by that CTA, so the counters are zero between calls.
// Roles (512 threads, registers rebalanced per warpgroup with setmaxnreg):
// warp 0 TMA producer (weight tile, zero points and the token tile of each
// group into a ring of stages), warps 1 and 3 MMA issuers (alternate groups,
// one commit per group),
// warp 2 scale tables (this CTA's groups, loaded once), warps 4-11 4-bit
// unpack (with few tokens it is the longest per-group step) -- for 16 and 32
// tokens into tensor memory, where the MMA reads its weight operand, for 64
// tokens into the swizzled int8 operand in shared memory -- warps 12-15
// epilogue (one TMEM lane quadrant each).  Every wait is bounded as in the
// tiled kernel.
// Up to kGemvMaxM tokens the entry points below run the GEMV kernel instead
// (gemv_w4w8a8.cuh): the same plan, workspace layout and split reduction.
#pragma once

#include <atomic>
#include <cuda.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>
#include <cstdint>

#include "gemm_w4w8a8.cuh"
#include "gemv_w4w8a8.cuh"
#include "launch.h"
#include "ptx_sm100.cuh"

namespace mixllm {

constexpr int kSmThreads = 512;
constexpr int kSmUnpackWarps = 8;  // warps 4..11
// registers per thread after setmaxnreg, per warpgroup: control, unpack (two), epilogue;
// 128 * kSmRegsCtl + 256 * kSmRegsUnpack + 128 * kSmRegsEpi <= 512 * 128
constexpr int kSmRegsCtl = 88, kSmRegsUnpack = 72, kSmRegsEpi = 200;
static_assert(128 * kSmRegsCtl + 256 * kSmRegsUnpack + 128 * kSmRegsEpi <= 65536, "register split");
constexpr int kSmGroupsMax = 32;  // groups per CTA (bounds the scale tables)

// DUO (16 tokens only): two CTAs per SM -- a two-stage ring and 64
// registers a thread -- so that on layers with a wave of tiles or more
// (every CTA resident at once) one CTA's copy and drain latencies overlap
// the other's.  One CTA per SM with the deeper ring is faster for the
// smaller layers, which the plan gives more splits instead.
template <int MP, bool DUO = false>
struct SmallMCfg {
  static_assert(MP == 16 || MP == 32 || MP == 64, "token tile");
  static_assert(!DUO || MP == 16, "two CTAs per SM: 16 tokens only");
  static constexpr int kMinBlocks = DUO ? 2 : 1;
  // The ring holds stages of several groups each (four 4-bit groups, or two
  // 8-bit ones: 32 KiB of weights), loaded with one copy per operand: a CTA's
  // copy rate grows with the bytes per copy, so per-group copies of 8 KiB
  // would bound it far below HBM speed.  A stage is the chunk's weights, then
  // its token tiles (one 3-D box, group after group).
  // Where the unpacked 4-bit tiles live: tensor memory for 16 and 32 tokens
  // (the MMA reads its weight operand there, and the 64 KiB of shared memory
  // they would take doubles the ring: 4 stages instead of 2); shared memory
  // for 64 tokens, whose stages are too large for a third one to fit.
  static constexpr bool kTmemW = MP <= 32;
  static constexpr int kRingBytes = DUO ? 80 * 1024 : (kTmemW ? 192 * 1024 : 128 * 1024);
  static constexpr int kRegsCtl = DUO ? 40 : kSmRegsCtl;
  static constexpr int kRegsUnpack = DUO ? 56 : kSmRegsUnpack;
  static constexpr int kRegsEpi = DUO ? 88 : kSmRegsEpi;
  static_assert(128 * kRegsCtl + 256 * kRegsUnpack + 128 * kRegsEpi <= 65536 / kMinBlocks, "register split");
  static constexpr int kGpc4 = 4, kGpc8 = 2;                // groups per chunk
  static constexpr int kChunkWBytes = 32768;
  static constexpr int kMaxStages = 16;
  // Unpacked 4-bit tiles (32 TMEM columns or 16 KiB of shared memory each):
  // buffer i % kTBufs is free again only when the MMAs of group i - kTBufs
  // have completed, so the unpack needs several in flight.
  static constexpr int kTBufs = 4;
  static constexpr int kAccBufs = 4;
  static constexpr int kDone = kMaxStages;              // >= every ring released through it
  static_assert(kDone >= kTBufs && kDone >= kAccBufs, "done ring");
  static constexpr int kWBytes = 128 * 128;             // int8 weight tile (W8), or the unpacked 4-bit tile
  static constexpr int kW4Bytes = 128 * 64;             // packed 4-bit tile
  static constexpr int kXBytes = MP * 128;              // token tile of one group
  // tensor memory: kAccBufs accumulators of MP columns, then the unpacked
  // weight buffers; the allocation is a power of two
  static constexpr int kTmemABase = kAccBufs * MP;
  static constexpr int kTmemUsed = kTmemABase + (kTmemW ? kTBufs * 32 : 0);
  static constexpr int kTmemCols = kTmemUsed <= 32 ? 32 : kTmemUsed <= 64 ? 64 : kTmemUsed <= 128 ? 128 : kTmemUsed <= 256 ? 256 : 512;
  static_assert(kTmemUsed <= 512, "tensor memory");
  // shared-memory layout (offsets from a 1024-byte aligned base)
  static constexpr int kOffStages = 0;
  static constexpr int kOffTBuf = kOffStages + kRingBytes;
  static constexpr int kOffZ = kOffTBuf + (kTmemW ? 0 : kTBufs * kWBytes);
  static constexpr int kOffSw = kOffZ + kMaxStages * kGpc4 * 64;      // fp16 s_w [groups][128]
  static constexpr int kOffSa = kOffSw + kSmGroupsMax * 128 * 4;       // fp32 s_a [groups][MP]
  static constexpr int kOffBar = kOffSa + kSmGroupsMax * MP * 4;
  static constexpr int kNumBars = kMaxStages + kDone + kTBufs + kAccBufs + 3;  // + table ready, 2 drains
  // Two threads issue the MMAs of alternate groups; a ring they wait on must
  // give each slot to one of them (even slot counts), or a parity wait could
  // see a phase meant for the other one.
  static_assert(kTBufs % 2 == 0 && kAccBufs % 2 == 0 && kMaxStages % 2 == 0, "rings the issuers wait on");
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16;
  static constexpr int kSmemAlloc = kSmemBytes + 1024;
  static_assert(kXBytes % 1024 == 0 && kRingBytes % 1024 == 0, "swizzled tiles need 1024-byte alignment");
  static_assert(2 * (kChunkWBytes + kGpc4 * kXBytes) <= kRingBytes, "two stages must fit");
  // each stage's zero points are a 2-D TMA box: 128-byte aligned destinations
  static_assert(kOffZ % 128 == 0 && (kGpc4 * 64) % 128 == 0, "zero-point stages are TMA destinations");
  static_assert(kSmemAlloc <= 227 * 1024, "shared memory");
};

// Workspace of one call: S x tiles x MP x 128 fp32 partial sums (scratch),
// then one int32 counter per tile (zero between calls).  gemv: the call runs
// the GEMV kernel (M <= kGemvMaxM) with a token bound of MP in 1, 2, 4, 8,
// `splits` splits per 4-bit tile and `splits8` per 8-bit tile (S above is
// the larger); the tensor-core kernel uses `splits` for both sets.
struct SmallMPlan {
  int mp, nt4, nt8, splits, splits8, groups;
  bool gemv;
  // persistent GEMV (M <= kGemvMaxM and M*K within its resident-token bound):
  // `ctas` CTAs share `units` 32 KiB units evenly; workspace [ctas][2][MP][128]
  bool persistent;
  bool duo;  // 16 tokens, two CTAs per SM (SmallMCfg DUO)
  int units, ctas, chunks4, chunks8;
  size_t part_floats, counters;
  size_t bytes() const { return part_floats * 4 + counters * 4; }
};

// Atomic add at GPU scope with acquire-release semantics; returns the old value.
__device__ __forceinline__ int atom_add_acq_rel_gpu(int *p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// bytes of w with 0x80 set, minus z in every byte, then back to two's complement:
// byte i of the result is (w_i - z) as int8 for w_i, z in [0, 15].
__device__ __forceinline__ uint32_t sm_sub_zero_bytes(uint32_t w, uint32_t zz) {
  return ((w | 0x80808080u) - zz) ^ 0x80808080u;
}

// MP consecutive TMEM columns of this warp's 32 lanes into r (x16 / x32 loads).
template <int MP>
__device__ __forceinline__ void sm_tmem_ld(uint32_t taddr, uint32_t (&r)[MP]) {
  if constexpr (MP == 16) {
    tmem_ld_32x32b_x16(taddr, r);
  } else {
#pragma unroll
    for (int c = 0; c < MP / 32; ++c) tmem_ld_32x32b_x32(taddr + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(r + 32 * c));
  }
}
template <int MP>
__device__ __forceinline__ void sm_tmem_fill(uint32_t taddr, uint32_t v) {
  if constexpr (MP == 16) {
    tmem_st_32x32b_x16_fill(taddr, v);
  } else {
#pragma unroll
    for (int c = 0; c < MP / 32; ++c) tmem_st_32x32b_x32_fill(taddr + 32 * c, v);
  }
}
template <int MP>
__device__ __forceinline__ void sm_reg_fence(uint32_t (&r)[MP]) {
  if constexpr (MP == 16) {
    reg_fence(r);
  } else {
#pragma unroll
    for (int c = 0; c < MP / 32; ++c) reg_fence(*reinterpret_cast<uint32_t(*)[32]>(r + 32 * c));
  }
}

// DBG: the int32 group partials also go to Pd [M, N, G] (output column order).
template <int MP, bool DBG = false, bool DUO = false>
__global__ void __launch_bounds__(kSmThreads, SmallMCfg<MP, DUO>::kMinBlocks)
    gemm_small_m_kernel(const __grid_constant__ CUtensorMap tmX, const uint8_t *__restrict__ W4,
                        const __grid_constant__ CUtensorMap tmW8, const __grid_constant__ CUtensorMap tmZ,
                        const float *__restrict__ s_a,
                        const uint8_t *__restrict__ z4, const __half *__restrict__ s_w4,
                        const int32_t *__restrict__ idx4, const __half *__restrict__ s_w8,
                        const int32_t *__restrict__ idx8, int M, int K, int N4, int N8, int N4p, int N8p, int nt4,
                        int ntiles, int S, __half *__restrict__ Y, float *__restrict__ ws_part,
                        int *__restrict__ ws_cnt, int32_t *__restrict__ Pd) {
  using C = SmallMCfg<MP, DUO>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
  uint64_t *full = bars;                      // TMA -> unpack / MMA   (per stage)
  uint64_t *done = full + C::kMaxStages;      // MMA commit of local group i (ring of kDone)
  uint64_t *tfull = done + C::kDone;          // unpack -> MMA         (per unpacked buffer)
  uint64_t *accempty = tfull + C::kTBufs;     // epilogue -> MMA       (per accumulator)
  uint64_t *tabready = accempty + C::kAccBufs;  // scale tables loaded
  uint64_t *drain = tabready + 1;             // [2]: each MMA issuer's final commit
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kOffMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kOffMisc + 4);
  volatile int *last_flag = reinterpret_cast<volatile int *>(smem + C::kOffMisc + 8);
  float *tab_sw = reinterpret_cast<float *>(smem + C::kOffSw);
  float *tab_sa = reinterpret_cast<float *>(smem + C::kOffSa);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x / S, split = blockIdx.x - tile * S;
  const bool is4 = tile < nt4;
  const int n0 = (is4 ? tile : tile - nt4) * 128;
  const int G = K >> 7;
  const int g0 = static_cast<int>((static_cast<int64_t>(split) * G) / S);
  const int g1 = static_cast<int>((static_cast<int64_t>(split + 1) * G) / S);
  const int ng = g1 - g0;  // 1 .. kSmGroupsMax (the host sizes S so)
  const int Nset = is4 ? N4 : N8;
  const int Np = is4 ? N4p : N8p;
  const int N = N4 + N8;
  const __half *s_w = is4 ? s_w4 : s_w8;
  const int32_t *idx = is4 ? idx4 : idx8;

  // stage = one chunk: its weights (32 KiB), then the token tiles of four
  // groups (one box of the token tensor map serves both sets; an 8-bit chunk
  // of two groups leaves two of them unread); as many stages as fit, even
  const int gpc = is4 ? C::kGpc4 : C::kGpc8;
  const int nch = (ng + gpc - 1) / gpc;
  const int stage_sz = C::kChunkWBytes + C::kGpc4 * C::kXBytes;  // a multiple of 1024
  int nst = C::kRingBytes / stage_sz < C::kMaxStages ? C::kRingBytes / stage_sz : C::kMaxStages;
  nst &= ~1;  // even
  auto stage_w = [&](int s) { return smem + C::kOffStages + s * stage_sz; };
  auto stage_x = [&](int s) { return smem + C::kOffStages + s * stage_sz + C::kChunkWBytes; };
  auto tbuf = [&](int b) { return smem + C::kOffTBuf + b * C::kWBytes; };  // shared-memory unpacked tiles
  auto zmeta = [&](int s) { return smem + C::kOffZ + s * C::kGpc4 * 64; };
  // where local group i lives: its chunk's stage, its offset in the chunk, the phase of the stage
  auto gstage = [&](int i) { return (i / gpc) % nst; };
  auto gphase = [&](int i) { return static_cast<uint32_t>(((i / gpc) / nst) & 1); };
  // checked builds: the shared-memory window every access must stay in
  const uint32_t smem_lo = smem_u32(smem), smem_hi = smem_lo + static_cast<uint32_t>(C::kSmemBytes);
  (void)smem_lo, (void)smem_hi;
  // chunk c (local groups c*gpc ..) into stage c % nst: `weights` arms the
  // stage's barrier for the whole round and issues the weight copies (the
  // packed layer: constant, so they may run before the grid dependency
  // resolves); `tokens` issues the token box (written by the kernel before
  // this one: only after pdl_wait)
  auto load = [&](int c, bool weights, bool tokens) {
    const int s = c % nst, i0 = c * gpc, g = g0 + i0;
    const int n = min(gpc, ng - i0);
    // boxes always land whole (groups past the CTA's last come from the next
    // split or are zero past K; tokens past M are zero) and are never read
    const uint32_t wb = is4 ? static_cast<uint32_t>(n) * C::kW4Bytes : static_cast<uint32_t>(C::kChunkWBytes);
    if (!(chk_smem(smem_u32(stage_x(s)), C::kGpc4 * C::kXBytes, smem_lo, smem_hi) &&
          chk_smem(smem_u32(stage_w(s)), wb, smem_lo, smem_hi) &&
          (!is4 || chk_smem(smem_u32(zmeta(s)), C::kGpc4 * 64u, smem_lo, smem_hi)))) {
      if (weights) mbar_arrive_expect_tx(&full[s], 0u);  // checked build: no copy, the phase completes empty
      return;
    }
    if (weights) {
      mbar_arrive_expect_tx(&full[s], wb + static_cast<uint32_t>(C::kGpc4 * C::kXBytes) + (is4 ? C::kGpc4 * 64u : 0u));
      if (is4) {
        // the tile's packed groups are contiguous 8 KB blocks: one bulk copy
        bulk_load(stage_w(s), W4 + (static_cast<int64_t>(n0 >> 7) * G + g) * C::kW4Bytes, wb, &full[s]);
        tma_load_2d(zmeta(s), &tmZ, &full[s], n0 >> 1, g);
      } else {
        tma_load_3d(stage_w(s), &tmW8, &full[s], 0, n0, g);
      }
    }
    if (tokens) tma_load_3d(stage_x(s), &tmX, &full[s], 0, 0, g);
  };

  // the next kernel of the stream may launch now: it reads nothing this one
  // writes before its own dependency wait
  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    prefetch_tmap(&tmX);
    prefetch_tmap(is4 ? &tmZ : &tmW8);
    for (int s = 0; s < C::kMaxStages; ++s) mbar_init(&full[s], 1);
    for (int i = 0; i < C::kDone; ++i) mbar_init(&done[i], 1);
    for (int b = 0; b < C::kTBufs; ++b) mbar_init(&tfull[b], C::kTmemW ? kSmUnpackWarps / 2 : kSmUnpackWarps);
    for (int a = 0; a < C::kAccBufs; ++a) mbar_init(&accempty[a], 4);
    mbar_init(tabready, 1);
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    *abort_flag = 0;
    *last_flag = 0;
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

  if (warp < 4) {
    regs_dec<C::kRegsCtl>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // The first stages' weights stream in while the kernel before this
      // one (the quantizer, or the previous layer) finishes; every read of
      // data that kernel writes comes after this pdl_wait (here, in the
      // scale warp, or in roles ordered after these loads by barriers).
      int issued = nch < nst ? nch : nst;
      for (int c = 0; c < issued; ++c) load(c, true, false);
      pdl_wait();
      for (int c = 0; c < issued; ++c) load(c, false, true);
      for (int c = nst; c < nch; ++c) {
        // the stage last held chunk c - nst: free once both issuers' MMAs of it are done
        // (each issuer commits in its own order; there is none between the two)
        const int cp = c - nst;
        const int last = cp * gpc + gpc - 1;  // a full chunk: its last even and last odd group
        bool ok = mbar_wait(&done[last % C::kDone], (last / C::kDone) & 1, abort_flag);
        ok = ok && mbar_wait(&done[(last - 1) % C::kDone], ((last - 1) / C::kDone) & 1, abort_flag);
        if (!ok) break;
        load(c, true, true);
        issued = c + 1;
      }
      for (int c = (issued > nst ? issued - nst : 0); c < issued; ++c)
        (void)mbar_wait_drain(&full[c % nst], (c / nst) & 1, 1ll << 26);
    }
  } else if (warp == 1 || warp == 3) {
    // ------------------------------------------------------------ MMA issuers
    // warp 1 the even local groups, warp 3 the odd ones: one thread pays for
    // every tcgen05.mma and commit it issues, two keep the tensor pipe fed.
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(128, MP);
      const int who = warp == 1 ? 0 : 1;
      for (int i = who; i < ng; i += 2) {
        const int s = gstage(i), j = i % gpc, b = i % C::kTBufs, a = i % C::kAccBufs;
        if (!mbar_wait(&full[s], gphase(i), abort_flag)) break;
        if (is4 && !mbar_wait(&tfull[b], (i / C::kTBufs) & 1, abort_flag)) break;
        // phase 0 of accempty[a] is the epilogue's bias fill, phase u+1 its drain of use u
        if (!mbar_wait(&accempty[a], (i / C::kAccBufs) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t b_addr = smem_u32(stage_x(s) + j * C::kXBytes);  // tokens: MP rows x 128 k
        const uint32_t d = tmem_base + static_cast<uint32_t>(a * MP);
        bool in_range = chk_tmem(d, tmem_base, C::kTmemCols, MP, 128) && chk_smem(b_addr, C::kXBytes, smem_lo, smem_hi);
        if (is4 && C::kTmemW)
          in_range = in_range && chk_tmem(tmem_base + static_cast<uint32_t>(C::kTmemABase + b * 32), tmem_base,
                                          C::kTmemCols, 32, 128);
        else
          in_range = in_range && chk_smem(smem_u32(is4 ? tbuf(b) : stage_w(s) + j * C::kWBytes), 16384, smem_lo, smem_hi);
        if (!in_range) {
          // checked build: the group's MMAs are skipped, its commit still signals
        } else if (is4 && C::kTmemW) {  // weights: 128 channels x 128 k, unpacked into tensor memory
          const uint32_t wt = tmem_base + static_cast<uint32_t>(C::kTmemABase + b * 32);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) mma_i8_ts(d, wt + 8 * kk, sw128_kmajor_desc(b_addr + 32 * kk), idesc, 1u);
        } else {  // weights in shared memory: the unpacked tile, or the int8 tile of the stage
          const uint32_t a_addr = smem_u32(is4 ? tbuf(b) : stage_w(s) + j * C::kWBytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_i8(d, sw128_kmajor_desc(a_addr + 32 * kk), sw128_kmajor_desc(b_addr + 32 * kk), idesc, 1u);
        }
        mma_commit(&done[i % C::kDone]);
      }
      mma_commit(&drain[who]);
      (void)mbar_wait_drain(&drain[who], 0, 1ll << 28);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ scale tables
    // One batch of asynchronous copies for all of this CTA's groups, then a
    // single wait: s_w (fp16, 8 bytes per lane per group, contiguous per
    // group) and s_a (4 bytes per token per group; zero for padding tokens).
    __half *tsw = reinterpret_cast<__half *>(tab_sw);
    for (int i = 0; i < ng; ++i)  // the layer's scales: constant, before the dependency wait
      cp_async_8(tsw + i * 128 + 4 * lane, s_w + static_cast<int64_t>(g0 + i) * Np + n0 + 4 * lane);
    pdl_wait();  // s_a is written by the kernel before this one
    for (int e = lane; e < ng * MP; e += 32) {
      const int i = e / MP, t = e - i * MP;
      const bool in = t < M;
      cp_async_4(tab_sa + e, s_a + (in ? static_cast<int64_t>(t) * G + g0 + i : 0), in ? 4u : 0u);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncwarp();
    if (lane == 0) mbar_arrive(tabready);
  }
  } else if (warp < 12) {
    regs_dec<C::kRegsUnpack>();
    // ------------------------------------------------------------ 4-bit unpack
    // Warps 4 + q and 8 + q both write TMEM lane quadrant q and take alternate
    // groups.  Thread `lane` unpacks weight row rr = 32q + lane of the tile
    // (64 packed bytes -> 128 int8 values) and stores it as the 32 columns of
    // its lane in the group's buffer.  The packed rows are 64 bytes apart, so
    // lanes read their four 16-byte chunks in a rotated order (8 distinct bank
    // groups per load) and the rotation is undone in registers.
    if (C::kTmemW && is4) {
      const int q = warp & 3, h = (warp - 4) >> 2;
      const int rr = q * 32 + lane;
      const int rot = (lane >> 1) & 3;
      const int zshift = (rr & 1) * 4;
      const uint32_t trow = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + C::kTmemABase;
      for (int i = h; i < ng; i += 2) {
        const int s = gstage(i), j = i % gpc, b = i % C::kTBufs;
        if (!warp_wait(&full[s], gphase(i), abort_flag)) break;
        if (i >= C::kTBufs) {  // buffer b last held local group i - kTBufs
          const int ip = i - C::kTBufs;
          if (!warp_wait(&done[ip % C::kDone], (ip / C::kDone) & 1, abort_flag)) break;
          tc_fence_after();
        }
        const uint8_t *src = stage_w(s) + j * C::kW4Bytes + rr * 64;
        uint4 x[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) x[k] = *reinterpret_cast<const uint4 *>(src + (((k + rot) & 3) << 4));
        const uint32_t zz = ((static_cast<uint32_t>(zmeta(s)[j * 64 + (rr >> 1)]) >> zshift) & 0xFu) * 0x01010101u;
        // x[k] holds chunk (k + rot) & 3: rotate back by rot = (rot & 1) + (rot & 2)
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
        // chunk k: low nibbles are k-slice 32k .. 32k+15 (columns 8k .. 8k+3),
        // high nibbles 32k+16 .. 32k+31 (columns 8k+4 .. 8k+7)
        uint32_t o[32];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          o[8 * k + 0] = sm_sub_zero_bytes(x[k].x & 0x0F0F0F0Fu, zz);
          o[8 * k + 1] = sm_sub_zero_bytes(x[k].y & 0x0F0F0F0Fu, zz);
          o[8 * k + 2] = sm_sub_zero_bytes(x[k].z & 0x0F0F0F0Fu, zz);
          o[8 * k + 3] = sm_sub_zero_bytes(x[k].w & 0x0F0F0F0Fu, zz);
          o[8 * k + 4] = sm_sub_zero_bytes((x[k].x >> 4) & 0x0F0F0F0Fu, zz);
          o[8 * k + 5] = sm_sub_zero_bytes((x[k].y >> 4) & 0x0F0F0F0Fu, zz);
          o[8 * k + 6] = sm_sub_zero_bytes((x[k].z >> 4) & 0x0F0F0F0Fu, zz);
          o[8 * k + 7] = sm_sub_zero_bytes((x[k].w >> 4) & 0x0F0F0F0Fu, zz);
        }
        if (chk_tmem(trow + static_cast<uint32_t>(b * 32), tmem_base, C::kTmemCols, 32))
          tmem_st_32x32b_x32(trow + static_cast<uint32_t>(b * 32), o);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tfull[b]);
      }
    }
    // 64 tokens: the unpacked tile goes to shared memory in the 128-byte
    // swizzled K-major layout.
    // Thread tt owns the 16-byte column chunk c = tt % 4 (32 weights) of rows
    // r0 and r0 + 64 (r0 = tt / 4).
    if (!C::kTmemW && is4) {
      const int tt = threadIdx.x - 128;  // 0..255
      const int c = tt & 3, r0 = tt >> 2;
      const int zshift = (r0 & 1) * 4;
      const int sw = r0 & 7;
      for (int i = 0; i < ng; ++i) {
        const int s = gstage(i), j = i % gpc, b = i % C::kTBufs;
        if (!warp_wait(&full[s], gphase(i), abort_flag)) break;
        if (i >= C::kTBufs) {  // buffer b last held local group i - kTBufs
          const int ip = i - C::kTBufs;
          if (!warp_wait(&done[ip % C::kDone], (ip / C::kDone) & 1, abort_flag)) break;
        }
        const uint8_t *raw = stage_w(s) + j * C::kW4Bytes;
        const uint8_t *zb = zmeta(s) + j * 64;
        uint8_t *dst = tbuf(b);
        uint4 x[2];
        uint32_t zz[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int rr = r0 + 64 * k;
          x[k] = *reinterpret_cast<const uint4 *>(raw + rr * 64 + c * 16);
          zz[k] = ((static_cast<uint32_t>(zb[rr >> 1]) >> zshift) & 0xFu) * 0x01010101u;
        }
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int rr = r0 + 64 * k;
          uint4 lo, hi;
          lo.x = sm_sub_zero_bytes(x[k].x & 0x0F0F0F0Fu, zz[k]);
          lo.y = sm_sub_zero_bytes(x[k].y & 0x0F0F0F0Fu, zz[k]);
          lo.z = sm_sub_zero_bytes(x[k].z & 0x0F0F0F0Fu, zz[k]);
          lo.w = sm_sub_zero_bytes(x[k].w & 0x0F0F0F0Fu, zz[k]);
          hi.x = sm_sub_zero_bytes((x[k].x >> 4) & 0x0F0F0F0Fu, zz[k]);
          hi.y = sm_sub_zero_bytes((x[k].y >> 4) & 0x0F0F0F0Fu, zz[k]);
          hi.z = sm_sub_zero_bytes((x[k].z >> 4) & 0x0F0F0F0Fu, zz[k]);
          hi.w = sm_sub_zero_bytes((x[k].w >> 4) & 0x0F0F0F0Fu, zz[k]);
          *reinterpret_cast<uint4 *>(dst + rr * 128 + (((2 * c) ^ sw) << 4)) = lo;
          *reinterpret_cast<uint4 *>(dst + rr * 128 + (((2 * c + 1) ^ sw) << 4)) = hi;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tfull[b]);
      }
    }
  } else {
    regs_inc<C::kRegsEpi>();
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;        // TMEM lane quadrant: channels q*32 .. q*32+31 of the tile
    const int c = q * 32 + lane;   // this thread's channel in the tile
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    // Every accumulator starts at the bias 0x4b400000 and is reset to it after
    // each drain, so the int32 sum read as a float is 1.5*2^23 + P exactly.
#pragma unroll
    for (int a = 0; a < C::kAccBufs; ++a)
      if (chk_tmem(lane_base + static_cast<uint32_t>(a * MP), tmem_base, C::kTmemCols, MP))
        sm_tmem_fill<MP>(lane_base + static_cast<uint32_t>(a * MP), kI2FBiasBits);
    tmem_st_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0)
      for (int a = 0; a < C::kAccBufs; ++a) mbar_arrive(&accempty[a]);

    float acc[MP];
#pragma unroll
    for (int t = 0; t < MP; ++t) acc[t] = 0.0f;
    int32_t *pd = nullptr;  // DBG: this channel's partials of token 0, group g0
    if constexpr (DBG) {
      if (n0 + c < Nset) pd = Pd + static_cast<int64_t>(__ldg(idx + n0 + c)) * G + g0;
    }
    bool live = warp_wait(tabready, 0, abort_flag);
    for (int i = 0; live && i < ng; ++i) {
      const int a = i % C::kAccBufs;
      if (!warp_wait(&done[i % C::kDone], (i / C::kDone) & 1, abort_flag)) {
        live = false;
        break;
      }
      tc_fence_after();
      // v = bits of (1.5*2^23 + P) as float; u = fma(v, s_w, -1.5*2^23*s_w) is
      // exactly fl(P * s_w) (the bias term is exact for an fp16-valued s_w);
      // then acc[t] += u * s_a[t] for every token t.
      const float sw = __half2float(reinterpret_cast<const __half *>(tab_sw)[i * 128 + c]);
      const float2 sw2 = make_float2(sw, sw);
      const float2 cb2 = make_float2(-kI2FBias * sw, -kI2FBias * sw);
      const float2 *sa2 = reinterpret_cast<const float2 *>(tab_sa + i * MP);
      constexpr int CH = 16;  // columns per tcgen05.ld
#pragma unroll
      for (int h = 0; h < MP / CH; ++h) {
        uint32_t r[CH];
        const uint32_t col = lane_base + static_cast<uint32_t>(a * MP + h * CH);
        const bool col_ok = chk_tmem(col, tmem_base, C::kTmemCols, CH);
        if (col_ok) sm_tmem_ld<CH>(col, r);
        tmem_ld_wait();
        sm_reg_fence<CH>(r);
        if (col_ok) sm_tmem_fill<CH>(col, kI2FBiasBits);  // hand the columns back preset to the bias
        if constexpr (DBG) {
          if (pd != nullptr)
            for (int t = 0; t < CH; ++t)
              if (h * CH + t < M) pd[static_cast<int64_t>(h * CH + t) * N * G + i] = static_cast<int32_t>(r[t] - kI2FBiasBits);
        }
#pragma unroll
        for (int t = 0; t < CH; t += 2) {
          const int tt = h * CH + t;
          const float2 v = make_float2(__uint_as_float(r[t]), __uint_as_float(r[t + 1]));
          const float2 u = __ffma2_rn(v, sw2, cb2);
          const float2 o = __ffma2_rn(u, sa2[tt >> 1], make_float2(acc[tt], acc[tt + 1]));
          acc[tt] = o.x;
          acc[tt + 1] = o.y;
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[a]);
    }
    tmem_ld_wait();

    // Stage the sums in shared memory (the stage ring is idle now: every load
    // was consumed by an MMA that has completed), so the stores below run in a
    // plain loop over the tokens.
    float *stg = reinterpret_cast<float *>(smem + C::kOffStages) + c;
#pragma unroll
    for (int t = 0; t < MP; ++t) stg[t * 128] = acc[t];
    // One decision for all four epilogue warps (the barriers below need all
    // of them): a failed wait anywhere in the CTA has set the abort flag.
    (void)live;
    named_bar_sync(1, 128);
    if (threadIdx.x == 384) *last_flag = *abort_flag ? 2 : 0;
    named_bar_sync(1, 128);
    if (*last_flag == 0) {
      const bool ch_ok = n0 + c < Nset;
      const int col_out = ch_ok ? __ldg(idx + n0 + c) : 0;
      const int mt = M < MP ? M : MP;
      if (S == 1) {
        if (ch_ok)
          for (int t = 0; t < mt; ++t) Y[static_cast<int64_t>(t) * N + col_out] = __float2half_rn(stg[t * 128]);
      } else {
        // this split's partial sums; the last of the tile's S CTAs adds them
        float *part = ws_part + (static_cast<size_t>(split) * ntiles + tile) * (MP * 128) + c;
        for (int t = 0; t < mt; ++t) part[t * 128] = stg[t * 128];
        // The barrier orders the four warps' partial stores before the
        // counter update, whose release (GPU scope, cumulative) publishes
        // them; its acquire makes the other splits' partials visible to this
        // thread, and the second barrier to the other three warps.
        named_bar_sync(1, 128);
        if (threadIdx.x == 384) *last_flag = atom_add_acq_rel_gpu(ws_cnt + tile, 1) == S - 1 ? 1 : 0;
        named_bar_sync(1, 128);
        if (*last_flag) {
          const float *p0 = ws_part + static_cast<size_t>(tile) * (MP * 128) + c;
          const size_t split_stride = static_cast<size_t>(ntiles) * (MP * 128);
          // eight tokens at a time, so that many loads are in flight at once
          for (int t0 = 0; t0 < mt; t0 += 8) {
            float y[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) y[j] = t0 + j < mt ? __ldcg(p0 + (t0 + j) * 128) : 0.0f;
            for (int sp = 1; sp < S; ++sp) {
              const float *ps = p0 + sp * split_stride;
#pragma unroll
              for (int j = 0; j < 8; ++j)
                if (t0 + j < mt) y[j] += __ldcg(ps + (t0 + j) * 128);
            }
            if (ch_ok)
#pragma unroll
              for (int j = 0; j < 8; ++j)
                if (t0 + j < mt) Y[static_cast<int64_t>(t0 + j) * N + col_out] = __float2half_rn(y[j]);
          }
          if (threadIdx.x == 384) ws_cnt[tile] = 0;  // leave the workspace as it was found
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

constexpr int kSmWave = 148;      // SMs of a B200: split-K fills one wave of CTAs
constexpr int kGemvMaxM = 8;      // up to this many tokens the GEMV kernel runs
constexpr int kSmallMMaxM = 64;   // the few-token path takes up to this many tokens
// GEMV grid target: the CTAs that are resident at once on the 148 SMs
constexpr int gemv_cta_target(int mt) { return kSmWave * gemv_min_blocks(mt); }
constexpr int kGvpMinUnitsPerCta = 8;  // the persistent GEMV from this many 32 KiB units per CTA
constexpr int gemv_groups_max(int mt) {
  return mt == 1 ? GvCfg<1>::kGroupsMax
                 : (mt == 2 ? GvCfg<2>::kGroupsMax : (mt == 4 ? GvCfg<4>::kGroupsMax : GvCfg<8>::kGroupsMax));
}

// force: -1 plans by shape; 0, 1, 2 ask for the tensor-core kernel, the split
// GEMV or the persistent GEMV (the caller checks that the shape allows it:
// small_m_kernel_allowed).
SmallMPlan plan_small_m(int64_t M, int64_t N4, int64_t N8, int64_t K, int force = -1) {
  SmallMPlan p{};
  p.gemv = force < 0 ? M <= kGemvMaxM : force != 0;
  if (p.gemv)
    p.mp = M <= 1 ? 1 : (M <= 2 ? 2 : (M <= 4 ? 4 : 8));
  else
    p.mp = M <= 16 ? 16 : (M <= 32 ? 32 : 64);
  p.nt4 = static_cast<int>((N4 + 127) / 128);
  p.nt8 = static_cast<int>((N8 + 127) / 128);
  p.groups = static_cast<int>(K / 128);
  const int tiles = p.nt4 + p.nt8;
  // groups per CTA <= the kernel's cap
  const int gmax = p.gemv ? gemv_groups_max(p.mp) : kSmGroupsMax;
  const int s_min = (p.groups + gmax - 1) / gmax;
  auto clamp_s = [&](int S) { return S < s_min ? s_min : (S > p.groups ? p.groups : S); };
  // The persistent GEMV pays for its even shares with a reduction for every
  // tile that two CTAs share; measured on B200 it wins from about 8 units per
  // CTA (Llama 3.1 70B gate_up, down at M=1: 27 and 14 units per CTA, 19 % and
  // 16 % faster) and loses below (8B gate_up, 6 units: 8 % slower).
  const int chunks4 = (p.groups + 3) / 4, chunks8 = (p.groups + 1) / 2;
  const int64_t U = static_cast<int64_t>(p.nt4) * chunks4 + static_cast<int64_t>(p.nt8) * chunks8;
  const bool want_persistent =
      force < 0 ? U >= static_cast<int64_t>(kGvpMinUnitsPerCta) * gemv_cta_target(p.mp) : force == 2;
  if (p.gemv && p.mp <= kGvpMaxTokens && static_cast<int64_t>(p.mp) * K <= kGvpMaxTokenBytes && want_persistent) {
    p.persistent = true;
    p.chunks4 = chunks4;
    p.chunks8 = chunks8;
    p.units = static_cast<int>(U);
    p.ctas = static_cast<int>(U < gemv_cta_target(p.mp) ? U : gemv_cta_target(p.mp));
    p.splits = p.splits8 = 1;
    p.part_floats = static_cast<size_t>(p.ctas) * 2 * p.mp * 128;
    p.counters = static_cast<size_t>(tiles);
    return p;
  }
  if (p.gemv) {
    // an 8-bit tile has twice the bytes of a 4-bit one: it counts twice and gets twice the splits
    const int units = p.nt4 + 2 * p.nt8;
    int base = units > 0 ? gemv_cta_target(p.mp) / units : 1;
    if (base < 1) base = 1;
    p.splits = clamp_s(base);
    p.splits8 = clamp_s(2 * base);
  } else {
    int S = tiles > 0 ? kSmWave / tiles : 1;
    if (S < 1) S = 1;
    p.splits = p.splits8 = clamp_s(S);
    // 16 tokens with CTAs for most of two per SM: two CTAs per SM (measured
    // on B200: 8B gate_up 30.9 -> 25.1 us, 70B gate_up 112 -> 84 us; with
    // one CTA per SM, on q_proj and 8B down, the shallower ring lost 20-50 %)
    p.duo = p.mp == 16 && static_cast<int64_t>(tiles) * p.splits >= 3 * kSmWave / 2;
  }
  const int smax = p.splits > p.splits8 ? p.splits : p.splits8;
  p.part_floats = smax > 1 ? static_cast<size_t>(smax) * tiles * p.mp * 128 : 0;
  p.counters = smax > 1 ? static_cast<size_t>(tiles) : 0;
  return p;
}

template <int MP, bool DBG = false, bool DUO = false>
static cudaError_t launch_small_m_mp(const GemmArgs &a, const SmallMPlan &p, void *ws, cudaStream_t stream,
                                     const char **msg) {
  using C = SmallMCfg<MP, DUO>;
  auto enc = get_encode_fn();
  if (!enc) {
    *msg = "cuTensorMapEncodeTiled is not available from the driver";
    return cudaErrorNotSupported;
  }
  CUtensorMap tmX, tmW8, tmZ;
  memset(&tmX, 0, sizeof(tmX));
  memset(&tmW8, 0, sizeof(tmW8));
  memset(&tmZ, 0, sizeof(tmZ));
  // token tiles of four groups, 8-bit weights of two, zero points of four groups (one box each)
  if (!encode_groups_3d(enc, &tmX, a.A_q, a.K, a.M, MP, C::kGpc4)) {
    *msg = "tensor map encoding of A_q failed";
    return cudaErrorInvalidValue;
  }
  if (a.N8 > 0 && !encode_groups_3d(enc, &tmW8, a.W8, a.K, a.N8, 128, C::kGpc8)) {
    *msg = "tensor map encoding of W8 failed";
    return cudaErrorInvalidValue;
  }
  if (a.N4 > 0 && !encode_2d_u8(enc, &tmZ, a.z4, padded_channels(a.N4) / 2, a.K / 128, 64, C::kGpc4, false)) {
    *msg = "tensor map encoding of z4 failed";
    return cudaErrorInvalidValue;
  }
  const int tiles = p.nt4 + p.nt8;
  const int64_t grid = static_cast<int64_t>(tiles) * p.splits;
  if (grid > 0x7FFFFFFF) {
    *msg = "too many tiles";
    return cudaErrorInvalidValue;
  }
  auto kern = gemm_small_m_kernel<MP, DBG, DUO>;
  int dev = 0;
  cudaGetDevice(&dev);
  static std::atomic<unsigned long long> configured{0};  // one bit per device ordinal
  if (dev < 64 && !(configured.load() & (1ull << dev))) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemAlloc);
    if (e != cudaSuccess) {
      *msg = "cudaFuncSetAttribute(MaxDynamicSharedMemorySize) failed";
      return e;
    }
    configured.fetch_or(1ull << dev);
  }
  float *ws_part = static_cast<float *>(ws);
  int *ws_cnt = p.splits > 1 ? reinterpret_cast<int *>(ws_part + p.part_floats) : nullptr;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kSmThreads);
  cfg.dynamicSmemBytes = C::kSmemAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(
      &cfg, kern, tmX, a.W4, tmW8, tmZ, a.s_a, a.z4, static_cast<const __half *>(a.s_w4), a.idx4,
      static_cast<const __half *>(a.s_w8), a.idx8, static_cast<int>(a.M), static_cast<int>(a.K),
      static_cast<int>(a.N4), static_cast<int>(a.N8), static_cast<int>(padded_channels(a.N4)),
      static_cast<int>(padded_channels(a.N8)), p.nt4, tiles, p.splits, static_cast<__half *>(a.Y), ws_part, ws_cnt,
      DBG ? a.P : nullptr);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) *msg = "launch of the small-M GEMM failed";
  return e;
}

template <int MT, bool FUSE = false, bool DBG = false>
static cudaError_t launch_gemv_mt(const GemmArgs &a, const SmallMPlan &p, void *ws, cudaStream_t stream,
                                  const char **msg) {
  static_assert(gemv_min_blocks(MT) * (gemv_smem_bytes<MT>() + 1024) <= 228 * 1024, "resident CTAs per SM");
  CUtensorMap tmW8;
  memset(&tmW8, 0, sizeof(tmW8));
  if (a.N8 > 0) {
    auto enc = get_encode_fn();
    if (!enc) {
      *msg = "cuTensorMapEncodeTiled is not available from the driver";
      return cudaErrorNotSupported;
    }
    if (!encode_groups_3d(enc, &tmW8, a.W8, a.K, a.N8, 128, GvCfg<MT>::kChunk8)) {
      *msg = "tensor map encoding of W8 failed";
      return cudaErrorInvalidValue;
    }
  }
  const int tiles = p.nt4 + p.nt8;
  const int64_t grid = static_cast<int64_t>(p.nt4) * p.splits + static_cast<int64_t>(p.nt8) * p.splits8;
  if (grid > 0x7FFFFFFF) {
    *msg = "too many tiles";
    return cudaErrorInvalidValue;
  }
  auto kern = gemv_w4w8a8_kernel<MT, FUSE, DBG>;
  int dev = 0;
  cudaGetDevice(&dev);
  static std::atomic<unsigned long long> configured{0};  // one bit per device ordinal
  if (dev < 64 && !(configured.load() & (1ull << dev))) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, gemv_smem_bytes<MT>());
    if (e != cudaSuccess) {
      *msg = "cudaFuncSetAttribute(MaxDynamicSharedMemorySize) failed";
      return e;
    }
    configured.fetch_or(1ull << dev);
  }
  float *ws_part = static_cast<float *>(ws);
  int *ws_cnt = p.counters > 0 ? reinterpret_cast<int *>(ws_part + p.part_floats) : nullptr;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kGvThreads);
  cfg.dynamicSmemBytes = gemv_smem_bytes<MT>();
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(
      &cfg, kern, tmW8, static_cast<const __half *>(a.X), a.A_q, a.s_a, a.W4, a.z4,
      static_cast<const __half *>(a.s_w4), a.idx4,
      static_cast<const __half *>(a.s_w8), a.idx8, static_cast<int>(a.M), static_cast<int>(a.K),
      static_cast<int>(a.N4), static_cast<int>(a.N8), static_cast<int>(padded_channels(a.N4)),
      static_cast<int>(padded_channels(a.N8)), p.nt4, tiles, p.splits, p.splits8, static_cast<__half *>(a.Y), ws_part,
      ws_cnt, DBG ? a.P : nullptr);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) *msg = "launch of the GEMV failed";
  return e;
}

template <int MT, bool DBG = false>
static cudaError_t launch_gemv_persistent_mt(const GemmArgs &a, const SmallMPlan &p, void *ws, cudaStream_t stream,
                                             const char **msg) {
  static_assert(2 * (gvp_smem_bytes_max<MT>() + 1024) <= 228 * 1024, "two CTAs per SM");
  CUtensorMap tmW8;
  memset(&tmW8, 0, sizeof(tmW8));
  if (a.N8 > 0) {
    auto enc = get_encode_fn();
    if (!enc) {
      *msg = "cuTensorMapEncodeTiled is not available from the driver";
      return cudaErrorNotSupported;
    }
    if (!encode_groups_3d(enc, &tmW8, a.W8, a.K, a.N8, 128, 2)) {
      *msg = "tensor map encoding of W8 failed";
      return cudaErrorInvalidValue;
    }
  }
  auto kern = gemv_w4w8a8_persistent_kernel<MT, DBG>;
  int dev = 0;
  cudaGetDevice(&dev);
  static std::atomic<unsigned long long> configured{0};  // one bit per device ordinal
  if (dev < 64 && !(configured.load() & (1ull << dev))) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, gvp_smem_bytes_max<MT>());
    if (e != cudaSuccess) {
      *msg = "cudaFuncSetAttribute(MaxDynamicSharedMemorySize) failed";
      return e;
    }
    configured.fetch_or(1ull << dev);
  }
  GvpGeom geo{p.nt4, p.chunks4, p.chunks8, p.units, p.ctas};
  float *ws_part = static_cast<float *>(ws);
  int *ws_cnt = reinterpret_cast<int *>(ws_part + p.part_floats);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(p.ctas));
  cfg.blockDim = dim3(kGvThreads);
  cfg.dynamicSmemBytes = 1024 + gvp_layout(MT, static_cast<int>(a.K)).total;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(
      &cfg, kern, tmW8, a.A_q, a.s_a, a.W4, a.z4, static_cast<const __half *>(a.s_w4), a.idx4,
      static_cast<const __half *>(a.s_w8), a.idx8, static_cast<int>(a.M), static_cast<int>(a.K),
      static_cast<int>(a.N4), static_cast<int>(a.N8), static_cast<int>(padded_channels(a.N4)),
      static_cast<int>(padded_channels(a.N8)), geo, static_cast<__half *>(a.Y), ws_part, ws_cnt, DBG ? a.P : nullptr);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) *msg = "launch of the persistent GEMV failed";
  return e;
}

size_t small_m_workspace_bytes(int64_t M, int64_t N4, int64_t N8, int64_t K) {
  return plan_small_m(M, N4, N8, K).bytes();
}

// The split GEMV's fused form needs a CTA's slice of X (tokens x groups x
// 256 bytes) to fit the second 32 KiB ring slot; 4-bit CTAs hold the most
// groups.  Measured on B200 (the 8B decoder layer's four linears, rotating
// weights): one token 50.8 -> 46.9 us fused; four and eight tokens 2-3 %
// slower, each CTA quantizing its slice on the critical path -- so one token only.
static bool plan_fuses(const SmallMPlan &p) {
  if (!p.gemv || p.persistent || p.mp != 1) return false;
  const int ng_max = (p.groups + p.splits - 1) / p.splits;
  return static_cast<int64_t>(p.mp) * ng_max * 256 <= kGvSlotBytesSplit;
}

bool linear_small_m_fused(int64_t M, int64_t N4, int64_t N8, int64_t K) {
  return plan_fuses(plan_small_m(M, N4, N8, K));
}

static size_t round256(size_t b) { return (b + 255) / 256 * 256; }

size_t linear_small_m_workspace_bytes(int64_t M, int64_t N4, int64_t N8, int64_t K) {
  const SmallMPlan p = plan_small_m(M, N4, N8, K);
  if (plan_fuses(p)) return p.bytes();
  return round256(p.bytes()) + round256(static_cast<size_t>(M * K)) + static_cast<size_t>(M * (K / 128)) * 4;
}

cudaError_t launch_linear_small_m(const GemmArgs &a, void *ws, size_t ws_bytes, cudaStream_t stream,
                                  const char **msg) {
  const SmallMPlan p = plan_small_m(a.M, a.N4, a.N8, a.K);
  if (ws_bytes < linear_small_m_workspace_bytes(a.M, a.N4, a.N8, a.K) || (ws_bytes > 0 && !ws)) {
    *msg = "workspace too small for this shape";
    return cudaErrorInvalidValue;
  }
  if (plan_fuses(p)) {
    if (p.mp == 1) return launch_gemv_mt<1, true>(a, p, ws, stream, msg);
    if (p.mp == 2) return launch_gemv_mt<2, true>(a, p, ws, stream, msg);
    if (p.mp == 4) return launch_gemv_mt<4, true>(a, p, ws, stream, msg);
    return launch_gemv_mt<8, true>(a, p, ws, stream, msg);
  }
  // quantize into the workspace, then the planned kernel
  GemmArgs q = a;
  unsigned char *base = static_cast<unsigned char *>(ws);
  int8_t *A_q = reinterpret_cast<int8_t *>(base + round256(p.bytes()));
  float *s_a = reinterpret_cast<float *>(base + round256(p.bytes()) + round256(static_cast<size_t>(a.M * a.K)));
  cudaError_t e = launch_quantize_act(a.X, a.M, a.K, A_q, s_a, stream);
  if (e != cudaSuccess) {
    *msg = "launch of the activation quantizer failed";
    return e;
  }
  q.A_q = A_q;
  q.s_a = s_a;
  q.X = nullptr;
  return launch_gemm_small_m(q, ws, p.bytes(), stream, msg);
}

// Tiled layer workspace: A_q [M, K], s_a [M, G] fp32, then the two counters
// of the fused quantization (each part 256-byte aligned).
size_t linear_workspace_bytes(int64_t M, int64_t N4, int64_t N8, int64_t K) {
  if (M <= kSmallMMaxM) return linear_small_m_workspace_bytes(M, N4, N8, K);
  return round256(static_cast<size_t>(M * K)) + round256(static_cast<size_t>(M * (K / 128)) * 4) + 256;
}

cudaError_t launch_linear(const GemmArgs &a, void *ws, size_t ws_bytes, bool one_launch, cudaStream_t stream,
                          const char **msg) {
  if (a.M <= kSmallMMaxM) return launch_linear_small_m(a, ws, ws_bytes, stream, msg);
  if (ws_bytes < linear_workspace_bytes(a.M, a.N4, a.N8, a.K) || !ws) {
    *msg = "workspace too small for this shape";
    return cudaErrorInvalidValue;
  }
  unsigned char *base = static_cast<unsigned char *>(ws);
  const size_t aq_bytes = round256(static_cast<size_t>(a.M * a.K));
  const size_t sa_bytes = round256(static_cast<size_t>(a.M * (a.K / 128)) * 4);
  GemmArgs q = a;
  q.A_q = reinterpret_cast<int8_t *>(base);
  q.s_a = reinterpret_cast<float *>(base + aq_bytes);
  q.qcnt = reinterpret_cast<uint32_t *>(base + aq_bytes + sa_bytes);
  return launch_linear_tiled(q, one_launch, stream, msg);
}

bool small_m_kernel_allowed(int64_t M, int64_t N4, int64_t N8, int64_t K, int kind) {
  if (M < 1 || M > kSmallMMaxM || kind < 0 || kind > 2) return false;
  if (kind == 0) return true;
  if (M > kGemvMaxM) return false;
  const SmallMPlan p = plan_small_m(M, N4, N8, K, kind);
  return kind == 2 ? p.persistent : !p.persistent;
}

size_t small_m_debug_workspace_bytes(int64_t M, int64_t N4, int64_t N8, int64_t K, int kind) {
  return plan_small_m(M, N4, N8, K, kind).bytes();
}

cudaError_t launch_small_m_debug_partials(const GemmArgs &a, int kind, void *ws, size_t ws_bytes,
                                          cudaStream_t stream, const char **msg) {
  if (!small_m_kernel_allowed(a.M, a.N4, a.N8, a.K, kind)) {
    *msg = "the requested few-token kernel cannot take this shape";
    return cudaErrorInvalidValue;
  }
  const SmallMPlan p = plan_small_m(a.M, a.N4, a.N8, a.K, kind);
  if (ws_bytes < p.bytes() || (p.bytes() > 0 && ws == nullptr)) {
    *msg = "workspace too small for this shape";
    return cudaErrorInvalidValue;
  }
  if (a.P == nullptr) {
    *msg = "no partials buffer";
    return cudaErrorInvalidValue;
  }
  if (kind == 2) {
    if (p.mp == 1) return launch_gemv_persistent_mt<1, true>(a, p, ws, stream, msg);
    if (p.mp == 2) return launch_gemv_persistent_mt<2, true>(a, p, ws, stream, msg);
    return launch_gemv_persistent_mt<4, true>(a, p, ws, stream, msg);
  }
  if (kind == 1) {
    if (p.mp == 1) return launch_gemv_mt<1, false, true>(a, p, ws, stream, msg);
    if (p.mp == 2) return launch_gemv_mt<2, false, true>(a, p, ws, stream, msg);
    if (p.mp == 4) return launch_gemv_mt<4, false, true>(a, p, ws, stream, msg);
    return launch_gemv_mt<8, false, true>(a, p, ws, stream, msg);
  }
  if (p.mp == 16)
    return p.duo ? launch_small_m_mp<16, true, true>(a, p, ws, stream, msg) : launch_small_m_mp<16, true>(a, p, ws, stream, msg);
  if (p.mp == 32) return launch_small_m_mp<32, true>(a, p, ws, stream, msg);
  return launch_small_m_mp<64, true>(a, p, ws, stream, msg);
}

int small_m_kernel_kind(int64_t M, int64_t N4, int64_t N8, int64_t K) {
  const SmallMPlan p = plan_small_m(M, N4, N8, K);
  return p.persistent ? 2 : (p.gemv ? 1 : 0);
}

cudaError_t launch_gemm_small_m(const GemmArgs &a, void *ws, size_t ws_bytes, cudaStream_t stream, const char **msg) {
  const SmallMPlan p = plan_small_m(a.M, a.N4, a.N8, a.K);
  if (ws_bytes < p.bytes() || (p.bytes() > 0 && !ws)) {
    *msg = "workspace too small for this shape";
    return cudaErrorInvalidValue;
  }
  if (p.persistent) {
    static_assert(kGvpMaxTokens == 4, "token bounds of the persistent GEMV");
    if (p.mp == 1) return launch_gemv_persistent_mt<1>(a, p, ws, stream, msg);
    if (p.mp == 2) return launch_gemv_persistent_mt<2>(a, p, ws, stream, msg);
    return launch_gemv_persistent_mt<4>(a, p, ws, stream, msg);
  }
  if (p.gemv) {
    if (p.mp == 1) return launch_gemv_mt<1>(a, p, ws, stream, msg);
    if (p.mp == 2) return launch_gemv_mt<2>(a, p, ws, stream, msg);
    if (p.mp == 4) return launch_gemv_mt<4>(a, p, ws, stream, msg);
    return launch_gemv_mt<8>(a, p, ws, stream, msg);
  }
  if (p.mp == 16)
    return p.duo ? launch_small_m_mp<16, false, true>(a, p, ws, stream, msg) : launch_small_m_mp<16>(a, p, ws, stream, msg);
  if (p.mp == 32) return launch_small_m_mp<32>(a, p, ws, stream, msg);
  return launch_small_m_mp<64>(a, p, ws, stream, msg);
}

// ---------------------------------------------------------------------------
// The same path with no caller workspace and no allocation: a fixed scratch
// array in the module's static device memory (one copy per device, created
// when the module loads and zero-initialized).  Calls that run at the same
// time on one device (different streams or host threads) would share it, so
// they must be ordered, e.g. issued to one stream.
// ---------------------------------------------------------------------------

constexpr size_t kSmallMScratchBytes = size_t(8) << 20;
static __device__ __align__(256) unsigned char g_small_m_scratch[kSmallMScratchBytes];

size_t small_m_scratch_capacity() { return kSmallMScratchBytes; }

cudaError_t launch_gemm_small_m_noalloc(const GemmArgs &a, cudaStream_t stream, const char **msg) {
  const SmallMPlan p = plan_small_m(a.M, a.N4, a.N8, a.K);
  if (p.bytes() > kSmallMScratchBytes) {
    *msg = "shape needs more scratch than the static buffer holds";
    return cudaErrorInvalidValue;
  }
  void *ws = nullptr;
  if (p.bytes() > 0) {
    // the device's own copy of the array
    cudaError_t e = cudaGetSymbolAddress(&ws, g_small_m_scratch);
    if (e != cudaSuccess) {
      *msg = "cudaGetSymbolAddress of the static scratch failed";
      return e;
    }
    // The tile counters must start at zero.  Every call returns them to zero,
    // but one that gave up (a timeout) may not have: clear them each time.
    e = cudaMemsetAsync(static_cast<unsigned char *>(ws) + p.part_floats * sizeof(float), 0,
                        p.counters * sizeof(int), stream);
    if (e != cudaSuccess) {
      *msg = "clearing the tile counters failed";
      return e;
    }
  }
  return launch_gemm_small_m(a, ws, kSmallMScratchBytes, stream, msg);
}

}  // namespace mixllm

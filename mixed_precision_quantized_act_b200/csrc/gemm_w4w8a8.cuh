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
// How it runs on B200.  A tile is 128 output channels x 128 tokens (x 64
// tokens, with four accumulators instead of two, when the layer has so few
// tiles that even 64-token ones leave SMs idle).  The
// weights are the MMA's A operand (the tile's channels are the TMEM lanes of
// the accumulator) and the activations its B operand (the tokens are the
// accumulator's columns).  The grid is persistent: CTA c of a channel set
// takes that set's tiles c, c + C, c + 2C, ... (C = the set's CTA count), and
// every role walks one running group index gi = (tile of this CTA) * G + g,
// so the rings run on across tile boundaries and the next tile's first
// groups are loaded and multiplied while the epilogue still drains the last
// tile.  Both channel sets share the launch: the first CTAs take the 4-bit
// tiles, the others the 8-bit ones (the rings are laid out per set).
// 16 warps (the default build: 8 epilogue warps; MIXLLM_EPI_WARPS=16 builds
// 24 with 16 epilogue warps of half the columns, and the unpack warps move
// up by 8), warp-specialized, registers rebalanced with setmaxnreg toward the
// epilogue:
//   warp 0      TMA producer: the A_q tile [BM x 128] (128-byte swizzle) of
//               every group -- with the int8 weight tile on 8-bit tiles --
//               into a ring of stages; on 4-bit tiles the packed uint4 weight
//               tile (one contiguous 8 KiB block per tile and group) and the
//               group's zero points into a ring of their own.
//   warps 1, 3  one thread each issues the MMAs of alternate groups: 4 x
//               tcgen05.mma.kind::i8 (K = 32 each) into one of two int32
//               accumulators in tensor memory (TMEM; four of 64 columns with
//               64-token tiles), then one commit to the
//               group's `done` barrier, which frees the A_q stage and the
//               unpacked weight buffer and hands the accumulator over.
//   warp 2      stages per group the channel scales ({s_w, s_w, -1.5*2^23*s_w,
//               same} per channel, fp32) and the token scales s_a of the tile
//               in a small ring the epilogue reads.
//   warps 4-11  epilogue, two warps per TMEM lane quadrant (so two per SM
//               sub-partition: while one waits on a TMEM load the other keeps
//               the FMA pipe busy), BM/2 token columns each: tcgen05.ld of the
//               group's int32 partials, which the accumulator holds biased by
//               0x4b400000 (TMEM is preset to the bias and refilled with it
//               after every drain), so their bits read as float are
//               1.5*2^23 + P exactly for |P| <= 2^22 -- the bias trick with no
//               integer add.  The bias is folded into one FMA with the channel
//               scale: u = fma(v, s_w, -1.5*2^23*s_w) = fl(P*s_w), one
//               rounding, since 1.5*2^23*s_w is exact for an fp16-valued s_w;
//               then acc = fma(u, s_a, acc); both as f32x2 FMAs.  The running
//               sums stay in registers; after the tile's last group each
//               thread writes its BM/2 fp16 outputs straight to Y[m, idx[n]]
//               (a warp store covers 32 channels of one token row).
//   warps 12-15 4-bit set only: unpack the nibbles and subtract the zero
//               point in SWAR form (four bytes per 32-bit op, no borrow
//               between bytes) -- the B200 counterpart of the pages' vsub4
//               pre-dequantization (§ソフトウェアパイプライン) -- and store the
//               int8 rows with tcgen05.st into a TMEM buffer, from which the
//               MMA reads its A operand.
// Every ring slot is refilled as soon as its own consumer is done with it.
// Every wait is bounded; on a timeout the CTA records an error in the status
// word, drains its own copies and MMAs, frees TMEM and exits.
//
// kCvtI2F (measurement only): the same kernel with the int32 partials
// converted by the plain int -> float instruction: the accumulator is preset
// to 0 instead of the bias (the same refill after every drain), so the two
// variants differ in the conversion alone; fl(float(P)*s_w) is the same
// value as the bias-trick FMA, so both give identical Y.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>
#include <atomic>
#include <cstdint>
#include <mutex>

#include "launch.h"
#include "ptx_sm100.cuh"
#include "quant.cuh"  // quant_act_8x16: the fused form quantizes with the quantizer's own arithmetic

namespace mixllm {

// Tile tokens = accumulator columns: 128, or 64 when even 64-token tiles
// leave SMs idle (see gemm_tile_m).
constexpr int kBM = 128;
constexpr int kKG = 128;          // K per group = K per pipeline stage
// Epilogue warps: 16 (32 token columns each, 24 warps in all) or, with
// MIXLLM_EPI_WARPS=8, 8 (64 columns each, 16 warps, twice the registers).
#ifndef MIXLLM_EPI_WARPS
#define MIXLLM_EPI_WARPS 8
#endif
constexpr int kEpiWarps = MIXLLM_EPI_WARPS;  // warps 4 .. 3 + kEpiWarps
static_assert(kEpiWarps == 8 || kEpiWarps == 16, "epilogue warps");
constexpr int kThreads = 32 * (8 + kEpiWarps);
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kXformWarp0 = 4 + kEpiWarps;  // the four unpack warps
constexpr int kXformWarps = 4;
constexpr float kI2FBias = 12582912.0f;     // 1.5 * 2^23, the float with bits 0x4b400000
constexpr uint32_t kI2FBiasBits = 0x4B400000u;
// Registers: the launch gets kRegsLaunch per thread (768 x 80 = 61440); the
// warpgroups then rebalance with setmaxnreg within that pool.
constexpr int kRegsLaunch = kEpiWarps == 16 ? 80 : 128;
constexpr int kRegsCtl = kEpiWarps == 16 ? 40 : 56, kRegsXform = kEpiWarps == 16 ? 56 : 80;
constexpr int kRegsEpi = kEpiWarps == 16 ? 96 : 184;
static_assert(128 * (kRegsCtl + kRegsXform) + kEpiThreads * kRegsEpi <= kThreads * kRegsLaunch, "register split");
static_assert(kThreads * kRegsLaunch <= 65536, "register file");

template <int BN, int BM = kBM>
struct GemmCfg {
  static_assert(BN == 128, "the warp roles below are laid out for BN = 128");
  static_assert(BM == 128 || BM == 64, "token tile");
  static constexpr int kABytes = BM * kKG;         // 16 (8) KB A_q tile of one group
  static constexpr int kW8Bytes = BN * kKG;        // 16 KB int8 weight tile of one group
  static constexpr int kW4Bytes = BN * kKG / 2;    //  8 KB packed uint4 weight tile of one group
  static constexpr int kZBytes = BN / 2;           // zero points of one group, two per byte
  // Operands arrive in chunks of several groups: a stage holds a chunk's
  // A_q tiles (one 3-D box: k, token, group) and its weights (4-bit: the
  // packed tiles of consecutive groups, contiguous, one bulk copy, and their
  // zero points, one 2-D box; 8-bit: one 3-D box), all on one barrier.  On
  // B200 a thread that issues copies completes about one such round every
  // ~350-450 ns whatever its size, and stalls meanwhile, so one dedicated
  // thread issues one round per chunk: per-group rounds of 8-16 KiB would
  // bound a group at that time.
  static constexpr int kC4 = 4, kC8 = 3;  // groups per chunk: 4-bit, 8-bit tiles
  static constexpr int kStages = 2;
  static constexpr int kStage4 = kC4 * (kABytes + kW4Bytes);  // 96 KiB (64 KiB at BM = 64)
  static constexpr int kStage8 = kC8 * (kABytes + kW8Bytes);  // 96 KiB (72 KiB at BM = 64)
  static constexpr int kRingBytes = kStages * (kStage4 > kStage8 ? kStage4 : kStage8);
  static constexpr int kTBufs = 8;   // unpacked 4-bit tiles in TMEM, 32 columns each
  // Two threads issue the MMAs of alternate groups.  A barrier waited by one
  // issuer only must have an even slot count (the unpacked buffers, the
  // accumulators); the chunk barriers are waited by both, which is safe
  // because a chunk's slot is refilled only after the MMAs of all its groups,
  // by both issuers, have completed.
  static_assert(kTBufs % 2 == 0, "rings one issuer waits on");
  // One commit per group, to done[gi % kDone]: no waiter can fall a whole
  // ring behind as long as kDone covers every ring released through it.
  static constexpr int kDone = 8;
  static_assert(kDone >= kStages * kC4 && kDone >= kStages * kC8 && kDone >= kTBufs, "done ring");
  // TMEM accumulators: two of 128 columns, or four of 64 (the same columns)
  static constexpr int kAccBufs = BM == 128 ? 2 : 4;
  // The scale table: a slot holds kTabG consecutive groups, so the epilogue
  // waits for it, and releases it, once per kTabG groups.
  static constexpr int kTabG = 4, kTabSlots = 2;
  // tensor memory: kAccBufs int32 accumulators of BM (token) columns, then
  // the unpacked weight tiles, 128 bytes of K per lane = 32 columns each
  static constexpr int kTmemABase = kAccBufs * BM;
  static constexpr int kTmemABufCols = kKG / 4;
  static constexpr int kTmemCols = 512;
  static_assert(kTmemABase + kTBufs * kTmemABufCols <= kTmemCols, "tensor memory");
  static constexpr int kColsPerThread = BN * BM / kEpiThreads;  // token columns per epilogue thread
  static_assert(kColsPerThread % 32 == 0, "the preset fills 32 columns at a time, the drain loads 16");
  static constexpr int kTabWBytes = BN * 16;                      // {s_w, s_w, cb, cb} per channel
  static constexpr int kTabBytes = kTabWBytes + BM * 4;           // + s_a of the tile's tokens (one group)
  static constexpr int kTabSlotBytes = kTabG * kTabBytes;
  // Raw scales.  Vector path (G % 4 == 0, s_a 16-byte aligned): per chunk of
  // kScG groups one 2-D box of s_w [kScG][BN] fp16 and one of s_a [BM][kScG]
  // fp32, into kScStages stages.  Fallback: a staging ring of kStgSlots
  // single groups filled with cp.async, kStgDist groups ahead.
  static constexpr int kScG = 4, kScStages = 3;
  static constexpr int kScSwBytes = kScG * BN * 2, kScBytes = kScSwBytes + BM * kScG * 4;
  static constexpr int kStgSlots = 12;                            // raw scale staging ring
  static constexpr int kStgDist = 10;                             // groups prefetched ahead
  static constexpr int kStgBytes = BN * 2 + BM * 4;               // raw fp16 s_w + fp32 s_a
  static constexpr int kStgArea = kScStages * kScBytes > kStgSlots * kStgBytes ? kScStages * kScBytes
                                                                                : kStgSlots * kStgBytes;
  // shared-memory layout (offsets from a 1024-byte aligned base)
  static constexpr int kOffRing = 0;
  static constexpr int kOffZ = kOffRing + kRingBytes;
  static constexpr int kOffTab = kOffZ + kStages * kC4 * kZBytes;
  static constexpr int kOffStg = kOffTab + kTabSlots * kTabSlotBytes;
  static constexpr int kOffBar = kOffStg + kStgArea;
  // full per stage, done per group ring, full per unpacked buffer, empty
  // per accumulator, full/empty per table slot, one drain per issuer, full
  // per raw scale stage
  static constexpr int kNumBars = kStages + kDone + kTBufs + kAccBufs + 2 * kTabSlots + 2 + kScStages;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16;
  static constexpr int kSmemAlloc = kSmemBytes + 1024;
  static_assert(kABytes % 1024 == 0 && kW8Bytes % 1024 == 0 && kW4Bytes % 1024 == 0, "1024-byte aligned tiles");
  static_assert(kTabBytes % 16 == 0 && kStgBytes % 16 == 0 && kOffTab % 16 == 0 && kOffStg % 128 == 0, "alignment");
  static_assert(kScBytes % 128 == 0 && kScSwBytes % 128 == 0, "TMA destinations");
  // each stage's zero points are a 2-D TMA box: 128-byte aligned destinations
  static_assert(kOffZ % 128 == 0 && (kC4 * kZBytes) % 128 == 0, "zero-point stages are TMA destinations");
  static_assert(kSmemAlloc <= 227 * 1024, "shared memory");
};

// bytes of w with 0x80 set, minus z in every byte, then back to two's complement:
// byte i of the result is (w_i - z) as int8 for w_i, z in [0, 15].
__device__ __forceinline__ uint32_t sub_zero_bytes(uint32_t w, uint32_t zz) {
  return ((w | 0x80808080u) - zz) ^ 0x80808080u;
}

// The persistent schedule of one CTA: which channel set, and which tiles.
struct TileSched {
  bool is4;
  int first, stride, count;  // tiles first, first + stride, ... of the set (count of them)
  __device__ __forceinline__ TileSched(int cta, int c4, int c8, int T4, int T8) {
    is4 = cta < c4;
    first = is4 ? cta : cta - c4;
    stride = is4 ? c4 : c8;
    const int T = is4 ? T4 : T8;
    count = first < T ? (T - first + stride - 1) / stride : 0;
  }
  __device__ __forceinline__ int tile(int tl) const { return first + tl * stride; }
};

// Walks a CTA's chunks in order without dividing per step (a runtime
// division compiles to a dozen instructions, several on the XU pipe; every
// role advances its cursors once per group or chunk).  Chunk: up to CH
// consecutive groups of one tile, starting at group g0 of the tile and at
// running group index gi0.
template <int BM>
struct ChunkCursorT {
  int tl, c, g0, ng, gi0, m0, n0;
  __device__ __forceinline__ void start(const TileSched &sc, int G, int CH, int mt, int BN) {
    tl = c = g0 = gi0 = 0;
    ng = G < CH ? G : CH;
    tile(sc, mt, BN);
  }
  __device__ __forceinline__ void tile(const TileSched &sc, int mt, int BN) {
    if (tl < sc.count) {
      const int t = sc.tile(tl);
      m0 = (t % mt) * BM;
      n0 = (t / mt) * BN;
    }
  }
  __device__ __forceinline__ void next(const TileSched &sc, int G, int CH, int nch, int mt, int BN) {
    gi0 += ng;
    g0 += CH;
    if (++c == nch) {
      c = 0;
      g0 = 0;
      ++tl;
      tile(sc, mt, BN);
    }
    ng = G - g0 < CH ? G - g0 : CH;
  }
};

// Walks groups: running index gi, group g of tile tl, chunk ci (running) and
// position j inside the chunk.
struct GroupCursor {
  int gi, g, tl, ci, j;
  __device__ __forceinline__ void start() { gi = g = tl = ci = j = 0; }
  __device__ __forceinline__ void next(int G, int CH) {
    ++gi;
    ++j;
    if (++g == G) {
      g = 0;
      j = 0;
      ++tl;
      ++ci;
    } else if (j == CH) {
      j = 0;
      ++ci;
    }
  }
};

template <int BN, int BM, bool kDebugP, bool kCvtI2F, bool kFuseQ>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_w4w8a8_kernel(const __grid_constant__ CUtensorMap tmA4, const __grid_constant__ CUtensorMap tmA8,
                       const uint8_t *__restrict__ W4, const __grid_constant__ CUtensorMap tmW8,
                       const __grid_constant__ CUtensorMap tmZ, const __grid_constant__ CUtensorMap tmSa,
                       const __grid_constant__ CUtensorMap tmSw4, const __grid_constant__ CUtensorMap tmSw8, int vec_scales,
                       const float *__restrict__ s_a, const __half *__restrict__ s_w4,
                       const int32_t *__restrict__ idx4, const __half *__restrict__ s_w8,
                       const int32_t *__restrict__ idx8, int M, int K, int N4, int N8, int N4p, int N8p, int mt,
                       int T4, int T8, int c4, int c8, __half *__restrict__ Y, int32_t *__restrict__ P,
                       const __half *__restrict__ X, int8_t *__restrict__ Aq_w, float *__restrict__ sa_w,
                       uint32_t *__restrict__ qcnt) {
  using C = GemmCfg<BN, BM>;
  using ChunkCursor = ChunkCursorT<BM>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
  uint64_t *full = bars;                          // chunk landed                (per stage)
  uint64_t *done = full + C::kStages;             // MMA commit of group gi      (ring of kDone): frees the
                                                  // group's stages and unpacked buffer, fills its accumulator
  uint64_t *tfull = done + C::kDone;              // unpack -> MMA               (per unpacked buffer)
  uint64_t *accempty = tfull + C::kTBufs;         // epilogue -> MMA             (per TMEM accumulator)
  uint64_t *tabfull = accempty + C::kAccBufs;     // scale warp -> epilogue      (per table slot)
  uint64_t *tabempty = tabfull + C::kTabSlots;    // epilogue -> scale warp
  uint64_t *drain = tabempty + C::kTabSlots;      // [2]: each MMA issuer's final commit
  uint64_t *scfull = drain + 2;                   // raw scale chunk landed  (per raw scale stage)
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kOffMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const TileSched sched(static_cast<int>(blockIdx.x), c4, c8, T4, T8);
  const bool is4 = sched.is4;
  const int G = K >> 7;
  const int total = sched.count * G;  // groups this CTA runs
  const int Nset = is4 ? N4 : N8;
  const int Np = is4 ? N4p : N8p;
  const int N = N4 + N8;
  const __half *s_w = is4 ? s_w4 : s_w8;
  const int32_t *idx = is4 ? idx4 : idx8;
  // chunking of this CTA's set: CH groups per chunk, kStages stages of [A_q tiles | weights]
  const int CH = is4 ? C::kC4 : C::kC8;
  constexpr int S = C::kStages;
  const int nch = (G + CH - 1) / CH;       // chunks per tile (the last may hold fewer groups)
  const int nchunks = sched.count * nch;   // chunks this CTA loads
  const int a_bytes = CH * C::kABytes;
  const int w8_bytes = CH * C::kW8Bytes;  // an 8-bit chunk's weight tiles (the A_q box's size only when BM = BN)
  const int stage_bytes = is4 ? C::kStage4 : C::kStage8;
  // checked builds: the shared-memory window every access must stay in
  const uint32_t smem_lo = smem_u32(smem), smem_hi = smem_lo + static_cast<uint32_t>(C::kSmemBytes);
  (void)smem_lo, (void)smem_hi;
  auto stage_a = [&](int s) { return smem + C::kOffRing + s * stage_bytes; };
  auto stage_w = [&](int s) { return smem + C::kOffRing + s * stage_bytes + a_bytes; };
  auto zmeta = [&](int s) { return smem + C::kOffZ + s * C::kC4 * C::kZBytes; };
  // table entry of running group gi: slot (gi / kTabG) % kTabSlots, place gi % kTabG
  auto table_w = [&](int gi) {
    return reinterpret_cast<float4 *>(smem + C::kOffTab + ((gi / C::kTabG) % C::kTabSlots) * C::kTabSlotBytes +
                                      (gi % C::kTabG) * C::kTabBytes);
  };
  auto table_sa = [&](int gi) { return reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(table_w(gi)) + C::kTabWBytes); };
  auto stg_sw = [&](int i) { return smem + C::kOffStg + i * C::kStgBytes; };
  auto stg_sa = [&](int i) { return reinterpret_cast<float *>(smem + C::kOffStg + i * C::kStgBytes + BN * 2); };
  // Chunk `k` (a cursor) into stage k.c_run % S, one round on full[]: the
  // A_q tiles (one 3-D box: 128 k x 128 tokens x CH groups; groups past G
  // read as zeros and are never multiplied), then the packed 4-bit tiles of
  // its ng groups (one contiguous bulk copy) and their zero points (one 2-D
  // box), or the 8-bit tiles (one 3-D box).
  const CUtensorMap *tmA = is4 ? &tmA4 : &tmA8;
  // weights: arm the stage's barrier for the whole round and issue the
  // weight copies (the packed layer is constant: they may run before the
  // grid dependency resolves); tokens: the A_q box (written by the quantizer
  // before this kernel: only after pdl_wait)
  auto load_chunk = [&](const ChunkCursor &k, int ci, bool weights = true, bool tokens = true) {
    const int s = ci % S;
    if (is4) {
      const uint32_t wb = static_cast<uint32_t>(k.ng * C::kW4Bytes);
      if (!(chk_smem(smem_u32(stage_a(s)), a_bytes, smem_lo, smem_hi) &&
            chk_smem(smem_u32(stage_w(s)), wb, smem_lo, smem_hi) &&
            chk_smem(smem_u32(zmeta(s)), C::kC4 * C::kZBytes, smem_lo, smem_hi))) {
        if (weights) mbar_arrive_expect_tx(&full[s], 0u);  // checked build: no copy, the phase completes empty
        return;
      }
      if (weights) {
        mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(a_bytes) + wb + static_cast<uint32_t>(C::kC4 * C::kZBytes));
        bulk_load(stage_w(s), W4 + (static_cast<int64_t>(k.n0 >> 7) * G + k.g0) * C::kW4Bytes, wb, &full[s]);
        tma_load_2d(zmeta(s), &tmZ, &full[s], k.n0 >> 1, k.g0);
      }
      if (tokens) tma_load_3d(stage_a(s), tmA, &full[s], 0, k.m0, k.g0);
    } else {
      if (!(chk_smem(smem_u32(stage_a(s)), a_bytes, smem_lo, smem_hi) &&
            chk_smem(smem_u32(stage_w(s)), w8_bytes, smem_lo, smem_hi))) {
        if (weights) mbar_arrive_expect_tx(&full[s], 0u);
        return;
      }
      if (weights) {
        mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(a_bytes + w8_bytes));
        tma_load_3d(stage_w(s), &tmW8, &full[s], 0, k.n0, k.g0);
      }
      if (tokens) tma_load_3d(stage_a(s), tmA, &full[s], 0, k.m0, k.g0);
    }
  };
  // The producer: stage ci % S is refilled with chunk ci once the MMAs of
  // chunk ci - S are done -- the commits of its last two groups (one per
  // issuer) cover all of them.  Blocking (suspending) waits, so the thread
  // takes no issue slots from the warps of its SM sub-partition meanwhile.
  auto produce = [&](ChunkCursor &k, int first) {
    ChunkCursor rel;
    rel.start(sched, G, CH, mt, BN);
    int ci = first;
    for (; ci < nchunks; ++ci) {
      const int gl = rel.gi0 + rel.ng - 1;
      if (!mbar_wait(&done[gl % C::kDone], (gl / C::kDone) & 1, abort_flag)) break;
      if (rel.ng > 1 && !mbar_wait(&done[(gl - 1) % C::kDone], ((gl - 1) / C::kDone) & 1, abort_flag)) break;
      load_chunk(k, ci);
      k.next(sched, G, CH, nch, mt, BN);
      rel.next(sched, G, CH, nch, mt, BN);
    }
    return ci;
  };
  // let the copies of the last stages land before the CTA can exit
  auto drain_ring = [&](int issued) {
    for (int ci = (issued > S ? issued - S : 0); ci < issued; ++ci)
      (void)mbar_wait_drain(&full[ci % S], (ci / S) & 1, 1ll << 26);
  };
  ChunkCursor pk;  // the producer's next chunk (thread 0)

  if (threadIdx.x == 0) {
    prefetch_tmap(tmA);
    prefetch_tmap(is4 ? &tmZ : &tmW8);
    for (int s = 0; s < C::kStages; ++s) mbar_init(&full[s], 1);
    for (int i = 0; i < C::kDone; ++i) mbar_init(&done[i], 1);
    for (int b = 0; b < C::kTBufs; ++b) mbar_init(&tfull[b], kXformWarps);
    for (int a = 0; a < C::kAccBufs; ++a) mbar_init(&accempty[a], kEpiWarps);
    for (int i = 0; i < C::kTabSlots; ++i) {
      mbar_init(&tabfull[i], 1);
      mbar_init(&tabempty[i], kEpiWarps);
    }
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    for (int s = 0; s < C::kScStages; ++s) mbar_init(&scfull[s], 1);
    *abort_flag = 0;
    fence_mbar_init();
    // The first stages need nothing but their barriers: start them before
    // the CTA-wide sync.  Their weights stream in while the quantizer before
    // this kernel finishes; every read of data it writes comes after this
    // pdl_wait (here, in the scale warp and the epilogue, and in the roles
    // ordered after these loads by barriers).
    pk.start(sched, G, CH, mt, BN);
    {
      ChunkCursor wk = pk;
      for (int ci = 0; ci < S && ci < nchunks; ++ci) {
        load_chunk(wk, ci, true, false);
        wk.next(sched, G, CH, nch, mt, BN);
      }
    }
    pdl_wait();
    if constexpr (!kFuseQ) {
      for (int ci = 0; ci < S && ci < nchunks; ++ci) {
        load_chunk(pk, ci, false, true);
        pk.next(sched, G, CH, nch, mt, BN);
      }
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if constexpr (kFuseQ) {
    // The fused form quantizes the layer's activations first, with every
    // thread of the CTA (no role has anything else to do until the A_q tiles
    // exist; only the first stages' weight copies are in flight).  The M*G
    // (token, group) pairs are split evenly over the grid in token-major
    // order; a half-warp takes one pair with quant_act_8x16 -- the
    // stand-alone quantizer's arithmetic, so A_q and s_a are bit-identical
    // to it -- with kQB pairs' loads in flight per half-warp.  The CTA then
    // adds its pair count to qcnt[0] (release); every CTA's producer and
    // scale warp wait for the full count (acquire) before their first A_q or
    // s_a load.
    pdl_wait();  // X may be the previous kernel's output
    const int npairs = M * G;
    const int p0 = static_cast<int>(static_cast<int64_t>(npairs) * blockIdx.x / gridDim.x);
    const int p1 = static_cast<int>(static_cast<int64_t>(npairs) * (blockIdx.x + 1) / gridDim.x);
    const int hw = static_cast<int>(threadIdx.x) >> 4, lane16 = threadIdx.x & 15;
    const unsigned qmask = 0xFFFFu << (threadIdx.x & 16);
    constexpr int kHW = kThreads / 16, kQB = 4;
    for (int pb = p0 + hw; pb < p1; pb += kHW * kQB) {
      uint4 raw[kQB];
#pragma unroll
      for (int j = 0; j < kQB; ++j) {
        const int p = pb + j * kHW;
        if (p < p1) {
          const int m = p / G, g = p - m * G;
          raw[j] = __ldg(reinterpret_cast<const uint4 *>(X + static_cast<int64_t>(m) * K + g * kKG + lane16 * 8));
        }
      }
#pragma unroll
      for (int j = 0; j < kQB; ++j) {
        const int p = pb + j * kHW;
        if (p < p1) {
          const int m = p / G, g = p - m * G;
          uint32_t packed[2];
          const float sq = quant_act_8x16(raw[j], qmask, packed);
          *reinterpret_cast<uint2 *>(Aq_w + static_cast<int64_t>(m) * K + g * kKG + lane16 * 8) =
              make_uint2(packed[0], packed[1]);
          if (lane16 == 0) sa_w[p] = sq;  // s_a[m, g] is element m*G + g = p
        }
      }
    }
    fence_proxy_async_global();  // the codes are read by other CTAs' TMA
    __syncthreads();
    // the first epilogue thread publishes, and later counts the CTA done:
    // one thread, so the publication is ordered before that count
    if (threadIdx.x == 128 && p1 > p0) {
      __threadfence();
      red_release_gpu_u32(qcnt, static_cast<uint32_t>(p1 - p0));
    }
  }

  if (warp < 4) {
    regs_dec<kRegsCtl>();
    if (warp == 0) {
      // ---------------------------------------------------------- producer
      if (lane == 0) {
        const int first = S < nchunks ? S : nchunks;
        if constexpr (kFuseQ) {
          // the A_q tiles exist once every CTA has quantized its share
          if (first == 0) {
            // no tiles: nothing to load, nothing to wait for
          } else if (wait_count_gpu(qcnt, static_cast<uint32_t>(M * G), abort_flag)) {
            fence_proxy_async_global();
            for (int ci = 0; ci < first; ++ci) {
              load_chunk(pk, ci, false, true);
              pk.next(sched, G, CH, nch, mt, BN);
            }
            drain_ring(produce(pk, first));
          } else {
            drain_ring(first);  // bounded: the token boxes of these stages were never issued
          }
        } else {
          drain_ring(produce(pk, first));
        }
      }
    } else if (warp == 1 || warp == 3) {
      // ---------------------------------------------------------- MMA issuers
      // Two threads issue alternate groups (warp 1 the even ones, warp 3 the
      // odd ones): one thread pays for every tcgen05.mma and commit it issues
      // and leaves the tensor pipe idle between groups, two keep it busy.
      // The weights are the MMA's A operand (BN channels = the TMEM lanes of
      // the accumulator), the activations its B operand (BM token columns):
      // on 4-bit tiles A comes from the unpacked buffer in tensor memory.
      if (lane == 0) {
        constexpr uint32_t idesc = idesc_i8(BN, BM);
        const int who = warp == 1 ? 0 : 1;
        GroupCursor gc;
        gc.start();
        if (who) gc.next(G, CH);
        for (; gc.gi < total; gc.next(G, CH), gc.next(G, CH)) {
          const int gi = gc.gi, ci = gc.ci, j = gc.j;
          const int st = ci % S, b = gi % C::kTBufs, a = gi % C::kAccBufs;
          if (!mbar_wait(&full[st], (ci / S) & 1, abort_flag)) break;
          if (is4 && !mbar_wait(&tfull[b], (gi / C::kTBufs) & 1, abort_flag)) break;
          // phase 0 of accempty[a] is the epilogue's initial fill; phase u+1 its drain of use u
          if (!mbar_wait(&accempty[a], (gi / C::kAccBufs) & 1, abort_flag)) break;
          tc_fence_after();
          const uint32_t x_addr = smem_u32(stage_a(st) + j * C::kABytes);
          const uint32_t d = tmem_base + static_cast<uint32_t>(a * BM);
          bool in_range = chk_tmem(d, tmem_base, C::kTmemCols, BM, 128) && chk_smem(x_addr, C::kABytes, smem_lo, smem_hi);
          if (is4)
            in_range = in_range && chk_tmem(tmem_base + static_cast<uint32_t>(C::kTmemABase + b * C::kTmemABufCols),
                                            tmem_base, C::kTmemCols, C::kTmemABufCols, 128);
          else
            in_range = in_range && chk_smem(smem_u32(stage_w(st) + j * C::kW8Bytes), C::kW8Bytes, smem_lo, smem_hi);
          if (!in_range) {
            // checked build: the group's MMAs are skipped, its commit still signals
          } else if (is4) {
            const uint32_t wt = tmem_base + static_cast<uint32_t>(C::kTmemABase + b * C::kTmemABufCols);
#pragma unroll
            for (int kk = 0; kk < kKG / 32; ++kk)
              mma_i8_ts(d, wt + 8 * kk, sw128_kmajor_desc(x_addr + 32 * kk), idesc, 1u);
          } else {
            const uint32_t w_addr = smem_u32(stage_w(st) + j * C::kW8Bytes);
#pragma unroll
            for (int kk = 0; kk < kKG / 32; ++kk)
              mma_i8(d, sw128_kmajor_desc(w_addr + 32 * kk), sw128_kmajor_desc(x_addr + 32 * kk), idesc,
                     1u);
          }
          mma_commit(&done[gi % C::kDone]);
        }
        mma_commit(&drain[who]);
        (void)mbar_wait_drain(&drain[who], 0, 1ll << 28);
      }
    } else {
      // ---------------------------------------------------------- scale table
      // The entry of group gi holds, per channel of the tile, the float4
      // {s_w, s_w, -1.5*2^23*s_w, -1.5*2^23*s_w} (the f32x2 operands of the
      // bias-folding FMA), then s_a of the tile's 128 tokens.  A slot of
      // kTabG groups is waited free before its first group and published
      // after its last (or after the CTA's last group).
      auto slot_free = [&](int gi) {
        return gi % C::kTabG != 0 ||
               warp_wait(&tabempty[(gi / C::kTabG) % C::kTabSlots], ((gi / (C::kTabG * C::kTabSlots)) & 1) ^ 1,
                         abort_flag);
      };
      auto slot_done = [&](int gi) {
        if (gi % C::kTabG == C::kTabG - 1 || gi == total - 1) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&tabfull[(gi / C::kTabG) % C::kTabSlots]);
        }
      };
      auto publish = [&](int gi, const uint8_t *raw_sw, const float *sa_src, int sa_stride) {
        // raw_sw: the tile's BN fp16 s_w of this group; sa_src[t * sa_stride]: s_a of token t
        if (!(chk_smem(smem_u32(table_w(gi)), C::kTabBytes, smem_lo, smem_hi) &&
              chk_smem(smem_u32(raw_sw), BN * 2, smem_lo, smem_hi) &&
              chk_smem(smem_u32(sa_src), static_cast<uint32_t>(((BM - 1) * sa_stride + 1) * 4), smem_lo, smem_hi)))
          return;  // checked build: the entry is left as it was
        const uint2 raw = *reinterpret_cast<const uint2 *>(raw_sw + 8 * lane);
        const float2 a = __half22float2(*reinterpret_cast<const __half2 *>(&raw.x));
        const float2 b = __half22float2(*reinterpret_cast<const __half2 *>(&raw.y));
        float4 *tw = table_w(gi) + 4 * lane;
        const float sws[4] = {a.x, a.y, b.x, b.y};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float cb = kCvtI2F ? 0.0f : -kI2FBias * sws[c];
          tw[c] = make_float4(sws[c], sws[c], cb, cb);
        }
        float *tsa = table_sa(gi);
#pragma unroll
        for (int j = 0; j < BM / 32; ++j) tsa[lane + 32 * j] = sa_src[(lane + 32 * j) * sa_stride];
      };
      if (vec_scales) {
        // Vector path: per chunk of kScG groups of a tile, one 2-D box of s_w
        // and one of s_a land in a raw stage (one copy round for both), then
        // each group is converted into its table slot.  G % kScG == 0, so the
        // chunks never straddle a tile and gi = chunk * kScG + group.
        const int nsc = total / C::kScG;
        const CUtensorMap *tmSw = is4 ? &tmSw4 : &tmSw8;
        auto sc_raw = [&](int st) { return smem + C::kOffStg + st * C::kScBytes; };
        const int nscc = G / C::kScG;  // raw chunks per tile
        auto load_sc = [&](const ChunkCursor &k, int c) {
          const int st = c % C::kScStages;
          if (!chk_smem(smem_u32(sc_raw(st)), C::kScBytes, smem_lo, smem_hi)) {
            mbar_arrive_expect_tx(&scfull[st], 0u);  // checked build: no copy
            return;
          }
          mbar_arrive_expect_tx(&scfull[st], static_cast<uint32_t>(C::kScBytes));
          tma_load_2d(sc_raw(st), tmSw, &scfull[st], k.n0, k.g0);
          tma_load_2d(sc_raw(st) + C::kScSwBytes, &tmSa, &scfull[st], k.g0, k.m0);
        };
        ChunkCursor sk;  // next raw chunk to load (lane 0)
        int q_ok = 1;    // fused form: s_a exists (lane 0 waited for it)
        if (lane == 0) {
          prefetch_tmap(&tmSa);
          prefetch_tmap(tmSw);
          pdl_wait();
          if constexpr (kFuseQ) {
            if (nsc > 0) {
              q_ok = wait_count_gpu(qcnt, static_cast<uint32_t>(M * G), abort_flag) ? 1 : 0;
              if (q_ok) fence_proxy_async_global();
            }
          }
          sk.start(sched, G, C::kScG, mt, BN);
          for (int c = 0; q_ok && c < C::kScStages && c < nsc; ++c) {
            load_sc(sk, c);
            sk.next(sched, G, C::kScG, nscc, mt, BN);
          }
        }
        q_ok = __shfl_sync(0xFFFFFFFFu, q_ok, 0);
        __syncwarp();
        int c = 0;
        for (; c < nsc; ++c) {
          const int st = c % C::kScStages;
          if (!warp_wait(&scfull[st], (c / C::kScStages) & 1, abort_flag)) break;
          bool ok = true;
          for (int jg = 0; jg < C::kScG; ++jg) {
            const int gi = c * C::kScG + jg;
            if (!slot_free(gi)) {
              ok = false;
              break;
            }
            publish(gi, sc_raw(st) + jg * BN * 2,
                    reinterpret_cast<const float *>(sc_raw(st) + C::kScSwBytes) + jg, C::kScG);
            slot_done(gi);
          }
          if (!ok) break;
          __syncwarp();
          if (lane == 0 && c + C::kScStages < nsc) {  // the stage is read: refill it
            load_sc(sk, c + C::kScStages);
            sk.next(sched, G, C::kScG, nscc, mt, BN);
          }
        }
        // let the raw copies still in flight land before the CTA can exit
        if (lane == 0 && q_ok) {
          const int issued = nsc < c + C::kScStages ? nsc : c + C::kScStages;
          for (int cc = (issued > C::kScStages ? issued - C::kScStages : 0); cc < issued; ++cc)
            (void)mbar_wait_drain(&scfull[cc % C::kScStages], (cc / C::kScStages) & 1, 1ll << 26);
        }
      } else {
        // Fallback: raw scales prefetched kStgDist groups ahead with cp.async
        // into a staging ring, one group per slot.
        ChunkCursor ik;  // group gi of the lookahead, as a chunk of one group
        ik.start(sched, G, 1, mt, BN);
        auto issue = [&](int gi) {
          if (gi < total) {
            const int g = ik.g0, m0 = ik.m0, n0 = ik.n0;
            ik.next(sched, G, 1, G, mt, BN);
            const int i = gi % C::kStgSlots;
            cp_async_8(stg_sw(i) + 8 * lane, s_w + static_cast<int64_t>(g) * Np + n0 + 4 * lane);
#pragma unroll
            for (int j = 0; j < BM / 32; ++j) {
              const int row = lane + 32 * j;
              const bool in = m0 + row < M;
              cp_async_4(stg_sa(i) + row, s_a + (in ? static_cast<int64_t>(m0 + row) * G + g : 0), in ? 4u : 0u);
            }
          }
          cp_async_commit();
        };
        pdl_wait();
        // fused form: every lane acquires the published s_a itself
        const bool q_ok = !kFuseQ || total == 0 || wait_count_gpu(qcnt, static_cast<uint32_t>(M * G), abort_flag);
        for (int gi = 0; q_ok && gi < C::kStgDist; ++gi) issue(gi);
        for (int gi = 0; q_ok && gi < total; ++gi) {
          const int i = gi % C::kStgSlots;
          cp_async_wait<C::kStgDist - 1>();
          __syncwarp();
          if (!slot_free(gi)) break;
          publish(gi, stg_sw(i), stg_sa(i), 1);
          slot_done(gi);
          issue(gi + C::kStgDist);
        }
        cp_async_wait<0>();
      }
    }
  } else if (warp >= kXformWarp0) {
    regs_dec<kRegsXform>();
    if (is4) {
      // ---------------------------------------------------------- 4-bit unpack
      // Warp 20 + q writes TMEM lane quadrant q: thread `lane` unpacks weight
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
      GroupCursor gc;
      gc.start();
      for (; gc.gi < total; gc.next(G, CH)) {
        const int gi = gc.gi, ci = gc.ci, j = gc.j;
        const int r = ci % S, b = gi % C::kTBufs;
        if (j == 0 && !warp_wait(&full[r], (ci / S) & 1, abort_flag)) break;
        // buffer b last held group gi - kTBufs: free once that group's MMAs are done
        if (gi >= C::kTBufs) {
          const int gp = gi - C::kTBufs;
          if (!warp_wait(&done[gp % C::kDone], (gp / C::kDone) & 1, abort_flag)) break;
          tc_fence_after();
        }
        const uint8_t *src = stage_w(r) + j * C::kW4Bytes + rr * 64;
        const bool in_range =
            warp_all_checked(chk_smem(smem_u32(src), 64, smem_lo, smem_hi) &&
                             chk_smem(smem_u32(zmeta(r) + j * C::kZBytes + (rr >> 1)), 1, smem_lo, smem_hi)) &&
            chk_tmem(trow + static_cast<uint32_t>(b * C::kTmemABufCols), tmem_base, C::kTmemCols, C::kTmemABufCols);
        uint4 x[4];
#pragma unroll
        for (int c = 0; c < 4; ++c)
          x[c] = in_range ? *reinterpret_cast<const uint4 *>(src + (((c + rot) & 3) << 4)) : make_uint4(0, 0, 0, 0);
        const uint32_t zz =
            in_range ? ((static_cast<uint32_t>(zmeta(r)[j * C::kZBytes + (rr >> 1)]) >> zshift) & 0xFu) * 0x01010101u
                     : 0u;
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
        if (in_range) tmem_st_32x32b_x32(trow + static_cast<uint32_t>(b * C::kTmemABufCols), o);
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
    // the tile (its TMEM lane) and the tokens part*32 .. part*32+31.
    constexpr int CPT = C::kColsPerThread;
    const int e = warp - 4;                 // 0 .. kEpiWarps - 1
    const int quad = warp & 3;              // TMEM lane quadrant of this warp (= its SM sub-partition)
    const int part = e >> 2;                // which CPT-column part of the tile's BM tokens
    const int ch = quad * 32 + lane;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + part * CPT;

    // Every accumulator starts at the bias 0x4b400000 (and is reset to it
    // after each drain), so the int32 sum the MMAs leave there, read as a
    // float, is 1.5*2^23 + P exactly (kCvtI2F: at 0, so it is P).
    constexpr uint32_t kPreset = kCvtI2F ? 0u : kI2FBiasBits;
#pragma unroll
    for (int a = 0; a < C::kAccBufs; ++a)
#pragma unroll
      for (int c = 0; c < CPT; c += 32)
        if (chk_tmem(lane_base + a * BM + c, tmem_base, C::kTmemCols, 32)) tmem_st_32x32b_x32_fill(lane_base + a * BM + c, kPreset);
    tmem_st_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0)
      for (int a = 0; a < C::kAccBufs; ++a) mbar_arrive(&accempty[a]);
    pdl_wait();  // before the idx reads below
    float2 acc[CPT / 2];
#pragma unroll
    for (int j = 0; j < CPT / 2; ++j) acc[j] = make_float2(0.0f, 0.0f);
    // 32-bit shared addresses of the barriers and tables this role touches
    const uint32_t a_done = smem_u32(done);
    const uint32_t a_accempty = smem_u32(accempty);
    const uint32_t a_tabfull = smem_u32(tabfull);
    const uint32_t a_tabempty = smem_u32(tabempty);
    const uint32_t a_tab = smem_u32(smem + C::kOffTab);
    bool live = true;
    int gi = 0;  // running group index
    for (int tl = 0; live && tl < sched.count; ++tl) {
      const int t = sched.tile(tl);
      const int m0 = (t % mt) * BM;
      const int n0 = (t / mt) * BN;
      const int nout = n0 + ch < Nset ? __ldg(idx + n0 + ch) : -1;  // output column of this thread's channel
      for (int g = 0; g < G; ++g, ++gi) {
        const int a = gi % C::kAccBufs, tslot = (gi / C::kTabG) % C::kTabSlots;
        const uint32_t col = lane_base + static_cast<uint32_t>(a * BM);
        if (!warp_wait_u32(a_done + 8 * (gi % C::kDone), (gi / C::kDone) & 1, abort_flag)) {
          live = false;
          break;
        }
        tc_fence_after();
        // The group is drained in CPT/16 chunks of 16 columns.  With 8
        // epilogue warps (registers to spare) the next chunk's TMEM load is
        // in flight while the current one is converted; with 16, one chunk's
        // registers at a time.
#ifndef MIXLLM_EPI_CW
#define MIXLLM_EPI_CW 16
#endif
        constexpr int CW = CPT > 32 ? MIXLLM_EPI_CW : 16, NCH = CPT / CW;
        constexpr bool kDB = CPT > 32;
        uint32_t rb[kDB ? 2 : 1][CW];
        // checked build: this warp's CPT accumulator columns (uniform over the warp)
        const bool acc_ok = chk_tmem(col, tmem_base, C::kTmemCols, CPT);
        if (acc_ok) tmem_ld_cols(col, rb[0]);
        if (gi % C::kTabG == 0 &&
            !warp_wait_u32(a_tabfull + 8 * tslot, (gi / (C::kTabG * C::kTabSlots)) & 1, abort_flag)) {
          tmem_ld_wait();
          live = false;
          break;
        }
        const uint32_t tab = a_tab + tslot * C::kTabSlotBytes + (gi % C::kTabG) * C::kTabBytes;
        const uint32_t tsa = tab + C::kTabWBytes + part * CPT * 4;
        const bool tab_ok = warp_all_checked(chk_smem(tab + 16 * ch, 16, smem_lo, smem_hi) &&
                                             chk_smem(tsa, CPT * 4, smem_lo, smem_hi));
        const float4 w = tab_ok ? lds_f4(tab + 16 * ch) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        const float2 sw2 = make_float2(w.x, w.y);
        const float2 cb2 = make_float2(w.z, w.w);
#pragma unroll
        for (int h = 0; h < NCH; ++h) {
          uint32_t(&r)[CW] = rb[kDB ? (h & 1) : 0];
          if (acc_ok && !kDB && h > 0) tmem_ld_cols(col + CW * h, r);
          tmem_ld_wait();
          reg_fence(r);
          if (acc_ok && kDB && h + 1 < NCH) tmem_ld_cols(col + CW * (h + 1), rb[(h + 1) & 1]);
          // hand the columns back preset (its wait is after the math)
          if (acc_ok) tmem_fill_cols<CW>(col + CW * h, kPreset);
          if constexpr (kDebugP) {
            if (nout >= 0) {
#pragma unroll 4
              for (int j = 0; j < CW; ++j) {
                const int m = m0 + part * CPT + CW * h + j;
                const int32_t pv =
                    kCvtI2F ? static_cast<int32_t>(r[j]) : static_cast<int32_t>(r[j] - kI2FBiasBits);
                if (m < M) P[(static_cast<int64_t>(m) * N + nout) * G + g] = pv;
              }
            }
          } else {
            // u = fma(v, s_w, -1.5*2^23*s_w) = fl(P*s_w): the bias term is
            // exact for an fp16-valued s_w and the fma rounds
            // v*s_w - 1.5*2^23*s_w once (kCvtI2F: v = float(P), u = fl(v*s_w),
            // the same value); then acc += u * s_a.  The table holds the s_a
            // of 4 consecutive tokens per 16 bytes.
#pragma unroll
            for (int j = 0; j < CW / 4; ++j) {
              const float4 sa = tab_ok ? lds_f4(tsa + 16 * ((CW / 4) * h + j)) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
              float2 v0, v1;
              if constexpr (kCvtI2F) {
                v0 = make_float2(__int2float_rn(static_cast<int>(r[4 * j])),
                                 __int2float_rn(static_cast<int>(r[4 * j + 1])));
                v1 = make_float2(__int2float_rn(static_cast<int>(r[4 * j + 2])),
                                 __int2float_rn(static_cast<int>(r[4 * j + 3])));
              } else {
                v0 = make_float2(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]));
                v1 = make_float2(__uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
              }
              const float2 u0 = __ffma2_rn(v0, sw2, cb2);
              const float2 u1 = __ffma2_rn(v1, sw2, cb2);
              const int k = (CW / 2) * h + 2 * j;  // acc[k] holds tokens 2k, 2k+1
              acc[k] = __ffma2_rn(u0, make_float2(sa.x, sa.y), acc[k]);
              acc[k + 1] = __ffma2_rn(u1, make_float2(sa.z, sa.w), acc[k + 1]);
            }
          }
        }
        if (gi % C::kTabG == C::kTabG - 1 || gi == total - 1) {
          __syncwarp();
          if (lane == 0) mbar_arrive_u32(a_tabempty + 8 * tslot);  // the table slot is read
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_u32(a_accempty + 8 * a);  // the accumulator is drained (and refilled)
      }
      if constexpr (!kDebugP) {
        // the tile's outputs, straight from the running sums: a warp store
        // covers 32 channels of one token row (adjacent output columns for
        // most of a sorted channel set)
        const int mbase = m0 + part * CPT;
        if (live && nout >= 0) {
          // one running pointer down the column (not 32 precomputed addresses)
          __half *yp = Y + static_cast<int64_t>(mbase) * N + nout;
          const int rows = M - mbase;
#pragma unroll
          for (int j = 0; j < CPT / 2; ++j) {
            if (2 * j < rows) *yp = __float2half_rn(acc[j].x);
            yp += N;
            if (2 * j + 1 < rows) *yp = __float2half_rn(acc[j].y);
            yp += N;
          }
        }
#pragma unroll
        for (int j = 0; j < CPT / 2; ++j) acc[j] = make_float2(0.0f, 0.0f);
      }
    }
    tmem_ld_wait();
    tmem_st_wait();
    if constexpr (kFuseQ) {
      // This CTA's producer and scale warp are past their waits on qcnt[0]
      // (its last tile drained: their loads came after those waits; a CTA
      // without tiles does not wait), and this thread published the CTA's
      // pairs before, so the CTA counts itself done, and the last one
      // returns both counters to zero for the next call.
      if (threadIdx.x == 128 && atom_add_acq_rel_gpu_u32(qcnt + 1, 1u) == gridDim.x - 1) {
        qcnt[0] = 0u;
        qcnt[1] = 0u;
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
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
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

// An int8 [rows, K] matrix (W8 [N8, K], or A_q [M, K]) as a 3-D tensor (k
// within a group, row, group) with 128 x box_rows x groups_per_box boxes:
// whole groups of a block of rows, each 128-byte row swizzled.  Encodings are
// cached by (base, K, rows, box).
static bool encode_groups_3d(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap *map, const void *W8, int64_t K,
                             int64_t N8, int box_rows, int groups_per_box) {
  struct Entry {
    const void *base;
    int64_t K, N8;
    int rows, gpb;
    bool valid;
    CUtensorMap map;
  };
  static Entry table[32];
  static int next = 0;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  for (const Entry &e : table)
    if (e.valid && e.base == W8 && e.K == K && e.N8 == N8 && e.rows == box_rows && e.gpb == groups_per_box) {
      *map = e.map;
      return true;
    }
  const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(N8), static_cast<cuuint64_t>(K / 128)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(K), 128};  // bytes, dims 1 and 2
  const cuuint32_t box[3] = {128, static_cast<cuuint32_t>(box_rows), static_cast<cuuint32_t>(groups_per_box)};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(W8), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  table[next] = Entry{W8, K, N8, box_rows, groups_per_box, true, *map};
  next = (next + 1) % 32;
  return true;
}

// A 2-D tensor of `dtype` elements (dims inner x outer, row stride in bytes)
// with box_inner x box_outer boxes, no swizzle.  Encodings are cached.
static bool encode_2d(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap *map, CUtensorMapDataType dtype,
                      const void *base, int64_t inner, int64_t outer, int64_t row_bytes, int box_inner, int box_outer) {
  struct Entry {
    const void *base;
    int64_t inner, outer, row_bytes;
    int dtype, bi, bo;
    bool valid;
    CUtensorMap map;
  };
  static Entry table[32];
  static int next = 0;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  for (const Entry &e : table)
    if (e.valid && e.base == base && e.inner == inner && e.outer == outer && e.row_bytes == row_bytes &&
        e.dtype == static_cast<int>(dtype) && e.bi == box_inner && e.bo == box_outer) {
      *map = e.map;
      return true;
    }
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_outer)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, dtype, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  table[next] = Entry{base, inner, outer, row_bytes, static_cast<int>(dtype), box_inner, box_outer, true, *map};
  next = (next + 1) % 32;
  return true;
}

// Number of SMs of the current device (cached per device ordinal).
static int device_sm_count() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

// How many CTAs of the persistent grid take 4-bit and 8-bit tiles: one CTA
// per tile while the tiles fit on the SMs, otherwise the SMs split in
// proportion to each set's work (an 8-bit tile costs about as much as a
// 4-bit one here: no unpack, but twice the shared-memory operand traffic).
static void split_ctas(int64_t T4, int64_t T8, int sms, int *c4, int *c8) {
  if (T4 + T8 <= sms) {
    *c4 = static_cast<int>(T4);
    *c8 = static_cast<int>(T8);
    return;
  }
  int a = static_cast<int>((static_cast<double>(sms) * T4) / static_cast<double>(T4 + T8) + 0.5);
  if (T4 > 0 && a < 1) a = 1;
  if (T8 > 0 && a > sms - 1) a = sms - 1;
  if (T8 == 0) a = sms;
  if (T4 == 0) a = 0;
  *c4 = static_cast<int>(a < T4 ? a : T4);
  *c8 = static_cast<int>((sms - a) < T8 ? (sms - a) : T8);
}

template <int BN, int BM, bool kDebugP, bool kCvtI2F, bool kFuseQ = false>
static cudaError_t launch_gemm_bm(const GemmArgs &a, cudaStream_t stream, const char **msg) {
  using C = GemmCfg<BN, BM>;
  auto enc = get_encode_fn();
  if (!enc) {
    *msg = "cuTensorMapEncodeTiled is not available from the driver";
    return cudaErrorNotSupported;
  }
  CUtensorMap tmA4, tmA8, tmW8, tmZ;
  memset(&tmA4, 0, sizeof(tmA4));
  memset(&tmA8, 0, sizeof(tmA8));
  memset(&tmW8, 0, sizeof(tmW8));
  memset(&tmZ, 0, sizeof(tmZ));
  // A_q in chunks of groups (one box per chunk and set), W8 likewise, the
  // zero points of a 4-bit chunk as one 2-D box
  if ((a.N4 > 0 && !encode_groups_3d(enc, &tmA4, a.A_q, a.K, a.M, BM, C::kC4)) ||
      (a.N8 > 0 && !encode_groups_3d(enc, &tmA8, a.A_q, a.K, a.M, BM, C::kC8))) {
    *msg = "tensor map encoding of A_q failed";
    return cudaErrorInvalidValue;
  }
  if (a.N8 > 0 && !encode_groups_3d(enc, &tmW8, a.W8, a.K, a.N8, BN, C::kC8)) {
    *msg = "tensor map encoding of W8 failed";
    return cudaErrorInvalidValue;
  }
  if (a.N4 > 0 && !encode_2d_u8(enc, &tmZ, a.z4, padded_channels(a.N4) / 2, a.K / kKG, BN / 2, C::kC4, false)) {
    *msg = "tensor map encoding of z4 failed";
    return cudaErrorInvalidValue;
  }
  // The scales by TMA (4 groups of a tile per box) when s_a's rows are
  // 16-byte multiples on a 16-byte aligned base; otherwise cp.async.
  CUtensorMap tmSa, tmSw4, tmSw8;
  memset(&tmSa, 0, sizeof(tmSa));
  memset(&tmSw4, 0, sizeof(tmSw4));
  memset(&tmSw8, 0, sizeof(tmSw8));
  const int64_t G = a.K / kKG;
  int vec = (G % C::kScG == 0 && (reinterpret_cast<uintptr_t>(a.s_a) & 15u) == 0) ? 1 : 0;
  if (vec) {
    const bool ok = encode_2d(enc, &tmSa, CU_TENSOR_MAP_DATA_TYPE_UINT32, a.s_a, G, a.M, G * 4, C::kScG, BM) &&
                    (a.N4 == 0 || encode_2d(enc, &tmSw4, CU_TENSOR_MAP_DATA_TYPE_UINT16, a.s_w4, padded_channels(a.N4),
                                            G, padded_channels(a.N4) * 2, BN, C::kScG)) &&
                    (a.N8 == 0 || encode_2d(enc, &tmSw8, CU_TENSOR_MAP_DATA_TYPE_UINT16, a.s_w8, padded_channels(a.N8),
                                            G, padded_channels(a.N8) * 2, BN, C::kScG));
    if (!ok) vec = 0;
  }
  const int64_t mt = (a.M + BM - 1) / BM;
  const int64_t T4 = mt * ((a.N4 + BN - 1) / BN);
  const int64_t T8 = mt * ((a.N8 + BN - 1) / BN);
  if (T4 + T8 > 0x7FFFFFFF || (T4 + T8) * (a.K / kKG) > 0x7FFFFFFF) {
    *msg = "too many tiles";
    return cudaErrorInvalidValue;
  }
  int c4 = 0, c8 = 0;
  split_ctas(T4, T8, device_sm_count(), &c4, &c8);
  auto kern = gemm_w4w8a8_kernel<BN, BM, kDebugP, kCvtI2F, kFuseQ>;
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
  // Launched as a programmatic dependent of the previous kernel in the stream:
  // the CTAs set up barriers and TMEM while that kernel finishes, and wait for
  // it (griddepcontrol.wait) before their first global read.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(c4 + c8));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::kSmemAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(
      &cfg, kern, tmA4, tmA8, a.W4, tmW8, tmZ, tmSa, tmSw4, tmSw8, vec, a.s_a, static_cast<const __half *>(a.s_w4), a.idx4,
      static_cast<const __half *>(a.s_w8), a.idx8, static_cast<int>(a.M), static_cast<int>(a.K),
      static_cast<int>(a.N4), static_cast<int>(a.N8), static_cast<int>(padded_channels(a.N4)),
      static_cast<int>(padded_channels(a.N8)), static_cast<int>(mt), static_cast<int>(T4), static_cast<int>(T8), c4,
      c8, static_cast<__half *>(a.Y), a.P, static_cast<const __half *>(kFuseQ ? a.X : nullptr),
      kFuseQ ? const_cast<int8_t *>(a.A_q) : nullptr, kFuseQ ? const_cast<float *>(a.s_a) : nullptr,
      kFuseQ ? a.qcnt : nullptr);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) *msg = "launch of the fused GEMM failed";
  return e;
}

// The token tile: 64 when even the 64-token tiles fit one wave (at most one
// per SM), else 128.  A group of a 128 x 64 tile costs nearly as much time
// as one of a 128 x 128 tile (the per-group chain of barriers, MMA issue and
// TMEM drain dominates; measured on B200: ~0.65 against ~0.69 us), so
// halving the tile pays only where it fills SMs that would otherwise idle
// (M = 256 at N = 4096: 66 tiles of 128 tokens, 32.5 -> 27.2 us) and costs
// up to a third elsewhere.  MIXLLM_TILE_M (a build macro: 64 or 128) fixes
// it instead.
#ifndef MIXLLM_TILE_M
#define MIXLLM_TILE_M 0
#endif
int gemm_tile_m(int64_t M, int64_t N4, int64_t N8) {
  if (MIXLLM_TILE_M == 64 || MIXLLM_TILE_M == 128) return MIXLLM_TILE_M;
  const int64_t mt = (M + kBM - 1) / kBM;
  const int64_t tiles = mt * ((N4 + 127) / 128 + (N8 + 127) / 128);
  return 2 * tiles <= static_cast<int64_t>(device_sm_count()) ? 64 : 128;
}

template <int BN, bool kDebugP, bool kCvtI2F, bool kFuseQ = false>
static cudaError_t launch_gemm_bn(const GemmArgs &a, cudaStream_t stream, const char **msg) {
  if (gemm_tile_m(a.M, a.N4, a.N8) == 64) return launch_gemm_bm<BN, 64, kDebugP, kCvtI2F, kFuseQ>(a, stream, msg);
  return launch_gemm_bm<BN, 128, kDebugP, kCvtI2F, kFuseQ>(a, stream, msg);
}

cudaError_t launch_gemm_w4w8a8(const GemmArgs &a, cudaStream_t stream, const char **msg) {
  if (a.cvt_i2f) {
    if (a.P) return launch_gemm_bn<128, true, true>(a, stream, msg);
    return launch_gemm_bn<128, false, true>(a, stream, msg);
  }
  if (a.P) return launch_gemm_bn<128, true, false>(a, stream, msg);
  return launch_gemm_bn<128, false, false>(a, stream, msg);
}

// The layer from fp16 X: a.X is the input; a.A_q, a.s_a and a.qcnt point
// into the caller's workspace (A_q [M, K], s_a [M, G] 16-byte aligned, two
// zeroed counters).  Two launches: the stand-alone quantizer into the
// workspace, then the GEMM as its programmatic dependent.  one_launch: the
// GEMM quantizes X itself (the scales must take the TMA path, G % 4 == 0,
// and M*G must fit 32 bits).
bool linear_tiled_fuses(int64_t M, int64_t K) {
  const int64_t G = K / kKG;
  return G % GemmCfg<128>::kScG == 0 && M * G <= 0x7FFFFFFF;
}

cudaError_t launch_linear_tiled(const GemmArgs &a, bool one_launch, cudaStream_t stream, const char **msg) {
  if (one_launch) {
    if (!linear_tiled_fuses(a.M, a.K) || (reinterpret_cast<uintptr_t>(a.s_a) & 15u) != 0) {
      *msg = "the one-launch form takes K / 128 a multiple of 4 and M * K / 128 below 2^31";
      return cudaErrorNotSupported;
    }
    return launch_gemm_bn<128, false, false, true>(a, stream, msg);
  }
  cudaError_t e = launch_quantize_act(a.X, a.M, a.K, const_cast<int8_t *>(a.A_q), const_cast<float *>(a.s_a), stream);
  if (e != cudaSuccess) {
    *msg = "launch of the activation quantizer failed";
    return e;
  }
  GemmArgs q = a;
  q.X = nullptr;
  q.qcnt = nullptr;
  return launch_gemm_bn<128, false, false>(q, stream, msg);
}

}  // namespace mixllm

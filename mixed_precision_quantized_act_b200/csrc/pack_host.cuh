// pack_host.cuh -- the offline weight quantization and pre-pack on the host
// CPU, for callers whose weights are in host memory (a checkpoint being
// converted).  The same quantizers, rounding and packed layout as the device
// pack kernels of quant.cuh (MLSys 2026 talk notes on MixLLM, notes.yuuk.io,
// §設計判断の概要: 4-bit asymmetric and 8-bit symmetric weights in groups of
// 128; §ソフトウェアパイプライン: the layout is fixed offline), written for
// the host: IEEE fp32 division and round-half-even conversions, fp16 through
// the round-to-nearest host conversion of cuda_fp16.h.  Plain loops, one
// (channel, group) at a time.
#pragma once

#include <cuda_fp16.h>
#include <cmath>
#include <cstdint>
#include <cstring>

namespace mixllm {

namespace host_pack {

// round half to even, as __float2int_rn (the default rounding mode)
inline int rne(float x) { return static_cast<int>(std::nearbyint(x)); }
inline int clampi(int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); }

// 4-bit asymmetric parameters of one (channel, group) from its range [lo, hi]
// (lo <= 0 <= hi): the fp16 scale, its fp32 value and the zero point.
inline void w4_params(float lo, float hi, __half &sh, float &sf, int &z) {
  const float sc = std::fmin((hi - lo) / 15.0f, 65504.0f);
  sh = __float2half_rn(sc);
  sf = __half2float(sh);
  z = sf != 0.0f ? clampi(rne(-lo / sf), 0, 15) : 0;
}

}  // namespace host_pack

// idx4 / idx8: ascending channel lists of the bit map; returns the number of
// 8-bit channels found (the caller checks it against N8 before packing).
inline int64_t host_split_channels(const uint8_t *is8, int64_t N, int64_t N8, int32_t *idx4, int32_t *idx8) {
  int64_t n8 = 0, n4 = 0;
  for (int64_t n = 0; n < N; ++n) {
    if (is8[n]) {
      if (n8 < N8) idx8[n8] = static_cast<int32_t>(n);
      ++n8;
    } else {
      if (n4 < N - N8) idx4[n4] = static_cast<int32_t>(n);
      ++n4;
    }
  }
  return n8;
}

// The 4-bit set: W4 [ceil(N4/128), G, 128, 64], z4 [G, N4p/2], s_w4 [G, N4p].
inline void host_pack_w4(const float *W, int64_t K, const int32_t *idx4, int64_t N4, int64_t N4p, uint8_t *W4,
                         uint8_t *z4, __half *s_w4) {
  const int64_t G = K >> 7, T4 = (N4 + 127) / 128;
  std::memset(W4, 0, static_cast<size_t>(T4 * G * 8192));
  std::memset(z4, 0, static_cast<size_t>(G * (N4p / 2)));
  for (int64_t i = 0; i < G * N4p; ++i) s_w4[i] = __float2half_rn(0.0f);
  for (int64_t r = 0; r < N4; ++r) {
    const float *wr = W + static_cast<int64_t>(idx4[r]) * K;
    for (int64_t g = 0; g < G; ++g) {
      const float *w = wr + (g << 7);
      float lo = 0.0f, hi = 0.0f;
      for (int k = 0; k < 128; ++k) {
        lo = std::fmin(lo, w[k]);
        hi = std::fmax(hi, w[k]);
      }
      __half sh;
      float sf;
      int z;
      host_pack::w4_params(lo, hi, sh, sf, z);
      uint8_t *row = W4 + (((r >> 7) * G + g) * 128 + (r & 127)) * 64;
      for (int k = 0; k < 128; ++k) {
        const int q = sf != 0.0f ? host_pack::clampi(host_pack::rne(w[k] / sf) + z, 0, 15) : 0;
        // run c = k / 32: byte 16c + i holds k = 32c + i (low) and 32c + 16 + i (high)
        const int c = k >> 5, j = k & 31;
        const int byte = 16 * c + (j & 15);
        row[byte] = static_cast<uint8_t>(row[byte] | (q << ((j >> 4) * 4)));
      }
      s_w4[g * N4p + r] = sh;
      z4[g * (N4p / 2) + (r >> 1)] = static_cast<uint8_t>(z4[g * (N4p / 2) + (r >> 1)] | (z << ((r & 1) * 4)));
    }
  }
}

// The 8-bit set: W8 [N8, K], s_w8 [G, N8p].
inline void host_pack_w8(const float *W, int64_t K, const int32_t *idx8, int64_t N8, int64_t N8p, int8_t *W8,
                         __half *s_w8) {
  const int64_t G = K >> 7;
  for (int64_t i = 0; i < G * N8p; ++i) s_w8[i] = __float2half_rn(0.0f);
  for (int64_t r = 0; r < N8; ++r) {
    const float *wr = W + static_cast<int64_t>(idx8[r]) * K;
    for (int64_t g = 0; g < G; ++g) {
      const float *w = wr + (g << 7);
      float amax = 0.0f;
      for (int k = 0; k < 128; ++k) amax = std::fmax(amax, std::fabs(w[k]));
      const __half sh = __float2half_rn(std::fmin(amax / 127.0f, 65504.0f));
      const float sf = __half2float(sh);
      for (int k = 0; k < 128; ++k)
        W8[r * K + (g << 7) + k] =
            static_cast<int8_t>(sf != 0.0f ? host_pack::clampi(host_pack::rne(w[k] / sf), -127, 127) : 0);
      s_w8[g * N8p + r] = sh;
    }
  }
}

}  // namespace mixllm

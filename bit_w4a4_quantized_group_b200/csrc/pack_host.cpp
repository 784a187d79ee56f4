// Host-side pack of an already-decomposed SVDQuant layer (svdq_pack_weight).
//
// "SVDQuant 阅读笔记：用少量高精度计算保护 4-bit 扩散模型", §5 "算法 1"
// steps 5 and 9: the residual R is quantized with the deployment format and
// saved together with the low-rank factors.  Formats follow §2.2 and §8 of
// the same page: INT4 groups of 64 with a 16-bit scale (eq.(1), s = max|Z|/7),
// NVFP4 groups of 16 with an FP8 (E4M3) scale; the 8-bit setting of §8 (appendix D)
// quantizes each output channel of the weight with one scale (W8A8).  The rounding rules are the
// ones stated in svdq.h; every conversion below is written from the format
// definition (IEEE binary16, bfloat16, OCP E4M3 "fn", E2M1).
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#include "svdq.h"
#include "svdq_internal.h"

namespace svdq {

uint16_t f32_to_bf16_rn(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return static_cast<uint16_t>(u >> 16);
}

float bf16_to_f32(uint16_t h) {
  uint32_t u = static_cast<uint32_t>(h) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// IEEE binary16, round to nearest even; values that would round to infinity
// saturate to 65504 (inputs here are non-negative scales).
uint16_t f32_to_f16_rn_sat(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  uint32_t sign = (u >> 16) & 0x8000u;
  float a = std::fabs(f);
  if (!(a < 65520.0f)) return static_cast<uint16_t>(sign | 0x7BFFu);  // 65504
  if (a == 0.0f) return static_cast<uint16_t>(sign);
  int e;
  float m = std::frexp(a, &e);          // a = m * 2^e, m in [0.5, 1)
  // binary16 normal: value = (1 + f/1024) * 2^(E-15), E in 1..30; subnormal: f * 2^-24
  int E = e - 1;                        // a = (2m) * 2^E, 2m in [1, 2)
  if (E < -14) {                        // subnormal range: multiple of 2^-24
    float q = std::nearbyint(std::ldexp(a, 24));   // exact scaling, then RNE
    uint32_t qi = static_cast<uint32_t>(q);        // may reach 1024 = smallest normal
    return static_cast<uint16_t>(sign | qi);
  }
  float frac = std::nearbyint((2.0f * m - 1.0f) * 1024.0f);  // exact operands, RNE
  uint32_t fi = static_cast<uint32_t>(frac);
  uint32_t Eb = static_cast<uint32_t>(E + 15);
  if (fi == 1024u) { fi = 0; Eb += 1; }
  return static_cast<uint16_t>(sign | (Eb << 10) | fi);
}

float f16_to_f32(uint16_t h) {
  uint32_t e = (h >> 10) & 0x1Fu, f = h & 0x3FFu;
  float v;
  if (e == 0) v = std::ldexp(static_cast<float>(f), -24);
  else v = std::ldexp(1.0f + static_cast<float>(f) / 1024.0f, static_cast<int>(e) - 15);
  return (h & 0x8000u) ? -v : v;
}

// OCP E4M3 (bias 7, 3 mantissa bits, no infinity, max 448), round to nearest
// even, saturating to 448.  Input is >= 0 (group scales).
uint8_t f32_to_e4m3_rn_sat(float x) {
  if (!(x > 0.0f)) return 0;
  if (x >= 448.0f) return 0x7E;
  if (x < 0.015625f) {                  // below 2^-6: subnormal grid m * 2^-9
    float q = std::nearbyint(std::ldexp(x, 9));
    return static_cast<uint8_t>(q);     // q == 8 is the smallest normal, code 0x08
  }
  int e;
  float m = std::frexp(x, &e);          // x = (2m) * 2^(e-1)
  int E = e - 1;                        // -6 .. 8
  float frac = std::nearbyint((2.0f * m - 1.0f) * 8.0f);
  int fi = static_cast<int>(frac);
  if (fi == 8) { fi = 0; E += 1; }
  int code = ((E + 7) << 3) | fi;
  if (code > 0x7E) code = 0x7E;
  return static_cast<uint8_t>(code);
}

float e4m3_to_f32(uint8_t c) {
  int e = (c >> 3) & 0xF, m = c & 7;
  float v = (e == 0) ? std::ldexp(static_cast<float>(m), -9)
                     : std::ldexp(1.0f + m / 8.0f, e - 7);
  return (c & 0x80) ? -v : v;
}

// E2M1 magnitude grid {0, .5, 1, 1.5, 2, 3, 4, 6}, nearest with ties to the
// even code, saturating at 6; the sign of v is kept (so -0.1 -> 0x8).
uint8_t f32_to_e2m1_rn_sat(float v) {
  float a = std::fabs(v);
  uint8_t c;
  if (a <= 0.25f) c = 0;
  else if (a < 0.75f) c = 1;
  else if (a <= 1.25f) c = 2;
  else if (a < 1.75f) c = 3;
  else if (a <= 2.5f) c = 4;
  else if (a < 3.5f) c = 5;
  else if (a <= 5.0f) c = 6;
  else c = 7;
  return static_cast<uint8_t>(c | (std::signbit(v) ? 8 : 0));
}

// Smallest power of two g with amax <= 6 * 448 * g (1 when amax == 0).
float pow2_gscale(float amax) {
  if (!(amax > 0.0f)) return 1.0f;
  const double lim = 6.0 * 448.0;
  int e;
  std::frexp(static_cast<double>(amax) / lim, &e);
  // start at the estimate and correct with exact comparisons
  while (lim * std::ldexp(1.0, e - 1) >= amax) --e;
  while (lim * std::ldexp(1.0, e) < amax) ++e;
  return static_cast<float>(std::ldexp(1.0, e));
}

bool is_pow2_positive(float g) {
  if (!(g > 0.0f) || !std::isfinite(g)) return false;
  int e;
  float m = std::frexp(g, &e);
  return m == 0.5f;
}

size_t blocked_sf_offset(int64_t row, int64_t grp, int64_t K, int g) {
  return static_cast<size_t>(((row / 128) * (K / (4 * g)) + grp / 4) * 512 + (row % 32) * 16 +
                             ((row % 128) / 32) * 4 + (grp % 4));
}

}  // namespace svdq

using namespace svdq;

extern "C" svdq_status svdq_pack_weight(svdq_format fmt, int64_t N, int64_t K, int rank,
                                        float act_gscale, const float* R, const float* L1,
                                        const float* L2, void* w_codes, void* w_scales,
                                        float* w_gscale, uint16_t* L1_bf16, uint16_t* L2_bf16) {
  svdq_status st = check_dims(fmt, 1, N, K, rank);
  if (st != SVDQ_OK) return st;
  if (!R || !w_codes || !w_scales || !w_gscale) return SVDQ_ERR_INVALID_ARG;
  if (rank > 0 && (!L1 || !L2 || !L1_bf16 || !L2_bf16)) return SVDQ_ERR_INVALID_ARG;
  if (!is_pow2_positive(act_gscale)) return SVDQ_ERR_INVALID_ARG;
  if (fmt != SVDQ_FMT_NVFP4_G16 && act_gscale != 1.0f) return SVDQ_ERR_INVALID_ARG;

  uint8_t* codes = static_cast<uint8_t*>(w_codes);
  std::memset(codes, 0, code_bytes(fmt, N, K));
  const int64_t Np = (N + 127) / 128 * 128;

  float gw = 1.0f;
  if (fmt == SVDQ_FMT_W8A8) {
    // one scale per output channel: s = fp32(a / 127), q = clamp(rint(fp32(x / s)), -127, 127)
    float* sf = static_cast<float*>(w_scales);
    std::memset(sf, 0, static_cast<size_t>(Np) * sizeof(float));
    for (int64_t n = 0; n < N; ++n) {
      const float* row = R + n * K;
      float a = 0.0f;
      for (int64_t k = 0; k < K; ++k) a = std::fmax(a, std::fabs(row[k]));
      const float s = a / 127.0f;
      sf[n] = s;
      for (int64_t k = 0; k < K; ++k) {
        int q = 0;
        if (s > 0.0f) q = static_cast<int>(std::fmax(-127.0f, std::fmin(127.0f, std::nearbyint(row[k] / s))));
        codes[n * K + k] = static_cast<uint8_t>(q & 0xFF);
      }
    }
  } else if (fmt == SVDQ_FMT_NVFP4_G16) {
    float amax = 0.0f;
    for (int64_t i = 0; i < N * K; ++i) amax = std::fmax(amax, std::fabs(R[i]));
    gw = pow2_gscale(amax);
    uint8_t* sf = static_cast<uint8_t*>(w_scales);
    std::memset(sf, 0, static_cast<size_t>(Np) * static_cast<size_t>(K / 16));
    for (int64_t n = 0; n < N; ++n) {
      const float* row = R + n * K;
      for (int64_t g = 0; g < K / 16; ++g) {
        float a = 0.0f;
        for (int j = 0; j < 16; ++j) a = std::fmax(a, std::fabs(row[g * 16 + j]));
        float t = (a / 6.0f) / gw;
        uint8_t sc = f32_to_e4m3_rn_sat(t);
        sf[blocked_sf_offset(n, g, K, 16)] = sc;
        float den = e4m3_to_f32(sc) * gw;
        for (int j = 0; j < 16; ++j) {
          int64_t k = g * 16 + j;
          uint8_t c = 0;
          if (den > 0.0f) c = f32_to_e2m1_rn_sat(row[k] / den);
          codes[n * (K / 2) + k / 2] |= static_cast<uint8_t>((k & 1) ? (c << 4) : c);
        }
      }
    }
  } else if (fmt == SVDQ_FMT_MXFP4_G32) {
    // MX shared scale: X = 2^clamp(floor(log2 a) - 2, -127, 127), byte log2(X) + 127
    uint8_t* sf = static_cast<uint8_t*>(w_scales);
    std::memset(sf, 0, static_cast<size_t>(Np) * static_cast<size_t>(K / 32));
    for (int64_t n = 0; n < N; ++n) {
      const float* row = R + n * K;
      for (int64_t g = 0; g < K / 32; ++g) {
        float a = 0.0f;
        for (int j = 0; j < 32; ++j) a = std::fmax(a, std::fabs(row[g * 32 + j]));
        int e = -127;
        if (a > 0.0f) {
          int ex = 0;
          std::frexp(a, &ex);            // a = m 2^ex, m in [0.5, 1): floor(log2 a) = ex - 1
          e = std::min(127, std::max(-127, ex - 1 - 2));
        }
        sf[blocked_sf_offset(n, g, K, 32)] = static_cast<uint8_t>(e + 127);
        for (int j = 0; j < 32; ++j) {
          const int64_t k = g * 32 + j;
          const uint8_t c = f32_to_e2m1_rn_sat(std::ldexp(row[k], -e));   // exact: x / 2^e
          codes[n * (K / 2) + k / 2] |= static_cast<uint8_t>((k & 1) ? (c << 4) : c);
        }
      }
    }
  } else {
    uint16_t* sf = static_cast<uint16_t*>(w_scales);
    std::memset(sf, 0, static_cast<size_t>(Np) * static_cast<size_t>(K / 64) * 2);
    for (int64_t n = 0; n < N; ++n) {
      const float* row = R + n * K;
      for (int64_t g = 0; g < K / 64; ++g) {
        float a = 0.0f;
        for (int j = 0; j < 64; ++j) a = std::fmax(a, std::fabs(row[g * 64 + j]));
        uint16_t s16 = f32_to_f16_rn_sat(a / 7.0f);
        sf[g * Np + n] = s16;
        float s = f16_to_f32(s16);
        for (int j = 0; j < 64; ++j) {
          int64_t k = g * 64 + j;
          int q = 0;
          if (s > 0.0f) {
            float v = std::nearbyint(row[k] / s);
            q = static_cast<int>(std::fmax(-7.0f, std::fmin(7.0f, v)));
          }
          uint8_t c = static_cast<uint8_t>(q & 0xF);
          codes[n * (K / 2) + k / 2] |= static_cast<uint8_t>((k & 1) ? (c << 4) : c);
        }
      }
    }
  }
  *w_gscale = gw;

  if (rank > 0) {
    for (int64_t i = 0; i < static_cast<int64_t>(rank) * K; ++i) L1_bf16[i] = f32_to_bf16_rn(L1[i]);
    const float inv = 1.0f / (act_gscale * gw);   // exact: power of two
    for (int64_t i = 0; i < N * rank; ++i) {
      float l2 = bf16_to_f32(f32_to_bf16_rn(L2[i]));
      float s = l2 * inv;
      uint16_t b = f32_to_bf16_rn(s);
      if (bf16_to_f32(b) != s || (l2 != 0.0f && !std::isnormal(s))) return SVDQ_ERR_UNSUPPORTED;
      L2_bf16[i] = b;
    }
  }
  return SVDQ_OK;
}

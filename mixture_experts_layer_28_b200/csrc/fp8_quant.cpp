// fp8_quant.cpp -- host-side FP8 (E4M3) block quantisation of expert weights.
//
// LongCat-Flash write-up ("Meituan's large model goes viral for its speed",
// section "System-level optimisation", its quantisation paragraph): the model
// quantises at fine-grained block level, as DeepSeek-V3 does, and keeps some
// layers (the down projection among them) in higher precision.  The page
// gives no format or block shape; two readings are offered, both with E4M3
// elements (sign, 4 exponent bits with bias 7, 3 mantissa bits, no
// infinities, largest finite magnitude 448, subnormals m/8 * 2^-6):
//
//   MOE_ZC_FP8_BLOCK128  128 x 128 blocks, one fp32 scale = amax / 448 each
//                        (formed in fp32), elements w / scale in fp32;
//   MOE_ZC_FP8_MX32      1 x 32 blocks along a row, one power-of-two scale
//                        each: the smallest with amax / scale <= 448, the
//                        form the tensor cores' block-scaled FP8 MMA applies.
//
// Elements round to the nearest E4M3 value, ties to the even code, and
// saturate at +-448; an all-zero block, or one holding a NaN or an infinity,
// gets scale 1.  Weights are quantised
// once, off the forward's path, so this is plain host code: arithmetic in
// float where the reading fixes float, exact power-of-two steps elsewhere.
#include <cmath>
#include <cstdint>
#include <cstring>

#include "../../include/moe_zc.h"

namespace {

constexpr float kE4M3Max = 448.0f;

float bf16_to_float(uint16_t h) {
  const uint32_t bits = static_cast<uint32_t>(h) << 16;
  float f;
  std::memcpy(&f, &bits, sizeof f);
  return f;
}

// E4M3 code of v: nearest value, ties to even, saturating at 448; NaN -> 0x7F.
uint8_t e4m3_code(float v) {
  if (std::isnan(v)) return 0x7F;
  const uint8_t sign = std::signbit(v) ? 0x80 : 0x00;
  const double a = std::fabs(static_cast<double>(v));
  if (a >= kE4M3Max) return sign | 0x7E;
  if (a < 0x1p-6) {
    // subnormal range: multiples of 2^-9; a count of 8 is the smallest
    // normal, whose code is 8 as well
    const double q = std::nearbyint(a * 512.0);   // exact scaling, rounds half to even
    return sign | static_cast<uint8_t>(q);
  }
  int ex;
  std::frexp(a, &ex);            // a = f 2^ex, f in [0.5, 1): binade exponent ex - 1
  int e = ex - 1;
  double q = std::nearbyint(std::ldexp(a, 3 - e));   // in [8, 16]: 1.mmm scaled by 8
  if (q == 16.0) {
    q = 8.0;
    ++e;
  }
  // a < 448 keeps e <= 8 and, at e = 8, q <= 14 (448 = 14 * 2^5)
  return sign | static_cast<uint8_t>(((e + 7) << 3) | (static_cast<int>(q) - 8));
}

// The smallest power of two s with amax / s <= 448 (amax > 0), exactly.
float pow2_scale(float amax) {
  int ex;
  std::frexp(static_cast<double>(amax), &ex);
  int k = ex - 9;                                   // 448 * 2^k = 0.875 * 2^ex
  while (static_cast<double>(amax) > std::ldexp(448.0, k)) ++k;
  while (static_cast<double>(amax) <= std::ldexp(448.0, k - 1)) --k;
  return static_cast<float>(std::ldexp(1.0, k));
}

}  // namespace

extern "C" int moe_zc_fp8_quantize(const void* W, int64_t rows, int64_t cols, int32_t mode,
                                   uint8_t* codes, float* scales) {
  if (!W || !codes || !scales || rows < 1 || cols < 1) return MOE_ZC_ERR_INVALID_ARG;
  if (mode != MOE_ZC_FP8_BLOCK128 && mode != MOE_ZC_FP8_MX32) return MOE_ZC_ERR_INVALID_ARG;
  const uint16_t* w = static_cast<const uint16_t*>(W);
  const int64_t br = mode == MOE_ZC_FP8_BLOCK128 ? 128 : 1;
  const int64_t bc = mode == MOE_ZC_FP8_BLOCK128 ? 128 : 32;
  const int64_t nbr = (rows + br - 1) / br;
  const int64_t nbc = (cols + bc - 1) / bc;
  for (int64_t i = 0; i < nbr; ++i) {
    const int64_t r0 = i * br, r1 = r0 + br < rows ? r0 + br : rows;
    for (int64_t j = 0; j < nbc; ++j) {
      const int64_t c0 = j * bc, c1 = c0 + bc < cols ? c0 + bc : cols;
      float amax = 0.f;
      bool finite = true;
      for (int64_t r = r0; r < r1; ++r)
        for (int64_t c = c0; c < c1; ++c) {
          const float a = std::fabs(bf16_to_float(w[r * cols + c]));
          if (!std::isfinite(a)) finite = false;
          else if (a > amax) amax = a;
        }
      // scale 1 for an all-zero block, and for one holding a NaN or an infinity
      float s = 1.0f;
      if (amax > 0.f && finite)
        s = mode == MOE_ZC_FP8_BLOCK128 ? amax / kE4M3Max : pow2_scale(amax);
      scales[i * nbc + j] = s;
      for (int64_t r = r0; r < r1; ++r)
        for (int64_t c = c0; c < c1; ++c) codes[r * cols + c] = e4m3_code(bf16_to_float(w[r * cols + c]) / s);
    }
  }
  return MOE_ZC_OK;
}

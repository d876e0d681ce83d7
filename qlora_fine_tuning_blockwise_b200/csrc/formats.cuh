// Per-element arithmetic of the weight-format conversions: double-quantized NF4 block constants and NVFP4.
//
// Every function here is one work item of a kernel in formats.cu (one group of block constants, one
// 16-weight block, one element).  They are plain __host__ __device__ code so that the kernels are thin
// grid-stride loops over them.  Every rounding is an explicit IEEE operation (never contracted into a
// fused multiply-add), so each result is a single fixed number.
//
// Double quantization ("Unsloth v0.1.463-beta: Fixes Studio Crash and llama-server Permission Issue",
// section "About the Unsloth Project", paragraph "How LoRA and QLoRA work": the quantization constants are
// themselves quantized).
//   - The fp32 absmax values c (flat order) are centred on their mean mu.
//   - They are cut into groups of 256, and each group keeps c1 = max |fl32(c - mu)|.
//   - Each constant keeps the E4M3 bit pattern of the level nearest to n = fl32(d / c1), a tie going to
//     the lower level.  The levels are the finite E4M3 values / 448, each rounded to fp32.
//   - mu is computed in one fixed order: fp64 sums per group in index order, then over the groups in
//     order, divided by the count in fp64, rounded to fp32.
//   - Dequantized: c' = fl32(fl32(L[code] * c1) + mu).
//
// NVFP4 ("Major Unsloth Update: NVFP4 Quantization Export and DeepSeek-V4 Training Support", section
// "NVFP4: A Quantization Format for the Next Generation of Hardware": E2M1 weights, range about +-6, one
// FP8 scale per small group).
//   - The tensor scale is S = fl32(amax / 2688).
//   - Per block of 16: t = fl32(a / fl32(6 S)), sb = E4M3(t) (nearest even, saturating), and
//     D = fl32(value(sb) * S).
//   - Each weight is E2M1(fl32(w / D)) (nearest even, saturating at 6, sign kept), or +0 when D = 0.
//   - Packing puts element 2j in the low nibble.
//   - Dequantized: w' = fl32(value(code) * D).
#pragma once

#include <cstdint>
#include <cstring>

#ifdef __CUDACC__
#define QF_HD __host__ __device__ __forceinline__
#else
#include <cmath>
#define QF_HD inline
#endif

namespace qfmt {

constexpr int kDqGroup = 256;    // block constants per second-level group
constexpr int kFp4Block = 16;    // weights per NVFP4 block scale
constexpr int kDqLevels = 253;   // distinct finite E4M3 values (+-0 counted once)

// ------------------------------------------------------------------------ single IEEE operations

QF_HD float mul_rn(float a, float b) {
#ifdef __CUDA_ARCH__
  return __fmul_rn(a, b);
#else
  return a * b;
#endif
}

QF_HD float add_rn(float a, float b) {
#ifdef __CUDA_ARCH__
  return __fadd_rn(a, b);
#else
  return a + b;
#endif
}

QF_HD float sub_rn(float a, float b) {
#ifdef __CUDA_ARCH__
  return __fsub_rn(a, b);
#else
  return a - b;
#endif
}

QF_HD float div_rn(float a, float b) {
#ifdef __CUDA_ARCH__
  return __fdiv_rn(a, b);
#else
  return a / b;
#endif
}

QF_HD double dadd_rn(double a, double b) {
#ifdef __CUDA_ARCH__
  return __dadd_rn(a, b);
#else
  return a + b;
#endif
}

QF_HD float f32_of_f64_rn(double a) {
#ifdef __CUDA_ARCH__
  return __double2float_rn(a);
#else
  return static_cast<float>(a);
#endif
}

QF_HD double ddiv_rn(double a, double b) {
#ifdef __CUDA_ARCH__
  return __ddiv_rn(a, b);
#else
  return a / b;
#endif
}

QF_HD uint32_t bits_of(float f) {
#ifdef __CUDA_ARCH__
  return __float_as_uint(f);
#else
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return u;
#endif
}

QF_HD float float_of(uint32_t u) {
#ifdef __CUDA_ARCH__
  return __uint_as_float(u);
#else
  float f;
  std::memcpy(&f, &u, 4);
  return f;
#endif
}

QF_HD float abs_f(float a) { return float_of(bits_of(a) & 0x7FFFFFFFu); }

// a (0 <= a < 2^23) rounded to the nearest integer, ties to even
QF_HD uint32_t rint_even_small(float a) {
#ifdef __CUDA_ARCH__
  return static_cast<uint32_t>(__float2int_rn(a));
#else
  return static_cast<uint32_t>(std::nearbyint(a));  // the default rounding mode: nearest, ties to even
#endif
}

// ------------------------------------------------------------------------ E4M3 and E2M1 values

// Value of a finite E4M3 pattern (0x7F and 0xFF, the NaNs, are never passed): sign bit 7, exponent field
// bits 6..3 with bias 7, mantissa bits 2..0; exponent field 0 is subnormal, m * 2^-9.
QF_HD float e4m3_value(uint32_t code) {
  const uint32_t e = (code >> 3) & 15u, m = code & 7u;
  const float mag = e == 0 ? mul_rn(static_cast<float>(m), 0.001953125f)   // m * 2^-9, exact
                           : float_of(((e + 120u) << 23) | (m << 20));    // (1 + m/8) 2^(e-7), built exactly
  return (code & 0x80u) ? -mag : mag;
}

// E4M3 pattern of a finite t >= 0: nearest value, ties to the even mantissa, saturating at 448.
QF_HD uint32_t e4m3_code_rne_sat(float t) {
  if (t >= 464.0f) return 0x7Eu;  // 464 is the tie between 448 and 480 (not a finite value): 448
  if (t < 0.015625f) {            // below 2^-6: the subnormal grid of step 2^-9 (its top, 8 * 2^-9, is 0x08)
    return rint_even_small(mul_rn(t, 512.0f));
  }
  const uint32_t b = bits_of(t);
  // keep 3 of the 23 mantissa bits, rounding the dropped 20 to nearest even; a carry moves into the exponent
  const uint32_t r = (b + 0x7FFFFu + ((b >> 20) & 1u)) >> 20;
  const uint32_t code = (((r >> 3) - 120u) << 3) | (r & 7u);
  return code > 0x7Eu ? 0x7Eu : code;
}

// Value of an E2M1 pattern: sign bit 3, exponent field bits 2..1 with bias 1, mantissa bit 0.
QF_HD float e2m1_value(uint32_t code) {
  const uint32_t e = (code >> 1) & 3u, m = code & 1u;
  const float mag = e == 0 ? 0.5f * static_cast<float>(m)
                           : static_cast<float>((2u + m) << (e - 1)) * 0.5f;  // (1 + m/2) 2^(e-1)
  return (code & 8u) ? -mag : mag;
}

// E2M1 pattern of n: nearest of 0, .5, 1, 1.5, 2, 3, 4, 6 in magnitude, ties to the even mantissa bit
// (0.25 -> 0, 0.75 -> 1, 1.25 -> 1, 1.75 -> 2, 2.5 -> 2, 3.5 -> 4, 5 -> 4), saturating at 6; n's sign bit.
QF_HD uint32_t e2m1_code_rne_sat(float n) {
  const float a = abs_f(n);
  const uint32_t c = static_cast<uint32_t>(a > 0.25f) + static_cast<uint32_t>(a >= 0.75f) +
                     static_cast<uint32_t>(a > 1.25f) + static_cast<uint32_t>(a >= 1.75f) +
                     static_cast<uint32_t>(a > 2.5f) + static_cast<uint32_t>(a >= 3.5f) +
                     static_cast<uint32_t>(a > 5.0f);
  return c | ((bits_of(n) >> 31) << 3);
}

// ------------------------------------------------------------------------ double quantization

// L[code] = fl32(value(code) / 448) for a finite code.
QF_HD float dq_level(uint32_t code) { return div_rn(e4m3_value(code), 448.0f); }

// Code of the i-th level in ascending order (i = 0 .. 252): negatives 0xFE .. 0x81, then 0x00, then 0x01 .. 0x7E.
QF_HD uint32_t dq_code_of_sorted(int i) {
  return i < 126 ? (0x80u | static_cast<uint32_t>(126 - i)) : static_cast<uint32_t>(i - 126);
}

// Nearest level to n (|n| <= 1) in the ascending table `lv` [253]: the number of midpoints strictly below
// n, each midpoint of two fp32 levels exact in fp64 (a tie stays on the lower level).
QF_HD uint32_t dq_code_of(float n, const float* lv) {
  const double x = static_cast<double>(n);
  int lo = 0, hi = kDqLevels - 1;  // search over the 252 midpoints
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    const double m = (static_cast<double>(lv[mid]) + static_cast<double>(lv[mid + 1])) * 0.5;
    if (m < x)
      lo = mid + 1;
    else
      hi = mid;
  }
  return dq_code_of_sorted(lo);
}

// fp64 sum of group g's constants in index order.
QF_HD double dq_group_sum(const float* c, long long nb, long long g) {
  const long long i0 = g * kDqGroup;
  const long long i1 = i0 + kDqGroup < nb ? i0 + kDqGroup : nb;
  double s = 0.0;
  for (long long i = i0; i < i1; ++i) s = dadd_rn(s, static_cast<double>(c[i]));
  return s;
}

// mu from the group sums: added in group order, divided by the count, rounded to fp32.
QF_HD float dq_offset(const double* sums, long long ng, long long nb) {
  double t = 0.0;
  for (long long g = 0; g < ng; ++g) t = dadd_rn(t, sums[g]);
  return f32_of_f64_rn(ddiv_rn(t, static_cast<double>(nb)));
}

// Codes and scale of group g.
QF_HD void dq_quantize_group(const float* c, long long nb, float mu, const float* lv, long long g, uint8_t* code8,
                             float* c1) {
  const long long i0 = g * kDqGroup;
  const long long i1 = i0 + kDqGroup < nb ? i0 + kDqGroup : nb;
  float m = 0.0f;
  for (long long i = i0; i < i1; ++i) {
    const float d = abs_f(sub_rn(c[i], mu));
    m = d > m ? d : m;
  }
  for (long long i = i0; i < i1; ++i) {
    const float n = m > 0.0f ? div_rn(sub_rn(c[i], mu), m) : 0.0f;
    code8[i] = static_cast<uint8_t>(dq_code_of(n, lv));
  }
  c1[g] = m;
}

// One dequantized constant; `lv256` is L indexed by code.
QF_HD float dq_dequantize_one(uint32_t code, float c1g, float mu, const float* lv256) {
  return add_rn(mul_rn(lv256[code], c1g), mu);
}

// ------------------------------------------------------------------------ NVFP4

QF_HD float nvfp4_tensor_scale(float amax) { return div_rn(amax, 2688.0f); }

// Quantize block b (weights w[16 b .. 16 b + 15]) given the tensor's largest magnitude: eight packed bytes
// (element 2j in the low nibble of byte j) and the E4M3 scale pattern.
QF_HD void nvfp4_quantize_block(const float* w, long long b, float amax, uint8_t* codes, uint8_t* scales) {
  const float* x = w + b * kFp4Block;
  const float S = nvfp4_tensor_scale(amax);
  float a = 0.0f;
  for (int j = 0; j < kFp4Block; ++j) {
    const float v = abs_f(x[j]);
    a = v > a ? v : a;
  }
  const float t = S > 0.0f ? div_rn(a, mul_rn(6.0f, S)) : 0.0f;
  const uint32_t sb = e4m3_code_rne_sat(t);
  const float D = mul_rn(e4m3_value(sb), S);
  for (int j = 0; j < kFp4Block; j += 2) {
    const uint32_t lo = D > 0.0f ? e2m1_code_rne_sat(div_rn(x[j], D)) : 0u;
    const uint32_t hi = D > 0.0f ? e2m1_code_rne_sat(div_rn(x[j + 1], D)) : 0u;
    codes[b * (kFp4Block / 2) + j / 2] = static_cast<uint8_t>(lo | (hi << 4));
  }
  scales[b] = static_cast<uint8_t>(sb);
}

// Decoded block scale D = fl32(value(sb) * S).
QF_HD float nvfp4_block_scale(uint32_t sb, float S) { return mul_rn(e4m3_value(sb), S); }

QF_HD float nvfp4_dequantize_one(uint32_t code, float D) { return mul_rn(e2m1_value(code), D); }

}  // namespace qfmt

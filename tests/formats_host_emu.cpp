// Test-only host build of the format conversions' per-element arithmetic (csrc/formats.cuh).
//
// The CUDA kernels in csrc/formats.cu are grid-stride loops over these same work items.  Compiled here for the
// host (IEEE single and double precision, no contraction into fused multiply-adds), they let a CPU test compare
// the kernels' exact arithmetic -- every rounding decision -- with the oracle, element by element, without a
// GPU.  The loops below visit the work items in the kernels' order where the order matters (the group sums
// and the mean); elsewhere each item is independent of the others.
#include <cstdint>

#include "../qlora_fine_tuning_blockwise_b200/csrc/formats.cuh"

using namespace qfmt;

extern "C" {

uint32_t emu_e4m3_code(float t) { return e4m3_code_rne_sat(t); }
float emu_e4m3_value(uint32_t c) { return e4m3_value(c); }
uint32_t emu_e2m1_code(float n) { return e2m1_code_rne_sat(n); }
float emu_e2m1_value(uint32_t c) { return e2m1_value(c); }
float emu_dq_level(uint32_t c) { return dq_level(c); }

void emu_dq_quantize(const float* c, long long nb, uint8_t* code8, float* c1, float* mu_out) {
  const long long ng = (nb + kDqGroup - 1) / kDqGroup;
  double* sums = new double[ng];
  for (long long g = 0; g < ng; ++g) sums[g] = dq_group_sum(c, nb, g);   // dq_group_sums_kernel
  const float mu = dq_offset(sums, ng, nb);                               // dq_offset_kernel
  float lv[kDqLevels];
  for (int i = 0; i < kDqLevels; ++i) lv[i] = dq_level(dq_code_of_sorted(i));
  for (long long g = 0; g < ng; ++g) dq_quantize_group(c, nb, mu, lv, g, code8, c1);  // dq_codes_kernel
  *mu_out = mu;
  delete[] sums;
}

void emu_dq_dequantize(const uint8_t* code8, const float* c1, float mu, long long nb, float* out) {
  float lv[256];
  for (int i = 0; i < 256; ++i) lv[i] = (i & 0x7F) == 0x7F ? 0.0f : dq_level(static_cast<uint32_t>(i));
  for (long long i = 0; i < nb; ++i) out[i] = dq_dequantize_one(code8[i], c1[i / kDqGroup], mu, lv);
}

void emu_nvfp4_quantize(const float* w, long long numel, uint8_t* codes, uint8_t* scales, float* S_out) {
  float amax = 0.0f;
  for (long long i = 0; i < numel; ++i) {
    const float v = abs_f(w[i]);
    amax = v > amax ? v : amax;
  }
  for (long long b = 0; b < numel / kFp4Block; ++b) nvfp4_quantize_block(w, b, amax, codes, scales);
  *S_out = nvfp4_tensor_scale(amax);
}

void emu_nvfp4_dequantize(const uint8_t* codes, const uint8_t* scales, float S, long long numel, float* out) {
  for (long long i = 0; i < numel; ++i) {
    const uint32_t byte = codes[i / 2];
    const uint32_t code = (i & 1) ? (byte >> 4) : (byte & 15u);
    out[i] = nvfp4_dequantize_one(code, nvfp4_block_scale(scales[i / kFp4Block], S));
  }
}

}  // extern "C"

// Weight-format conversions: double-quantized NF4 block constants and NVFP4 (the C ABI in include/qlora.h).
//
// A translation unit of its own: the layer's GEMM kernels (qlora.cu) do not depend on it.  Each kernel is a
// grid-stride loop over one work item of formats.cuh, where all of the arithmetic lives.  These are one-time
// conversions of a frozen weight, so the kernels favour a fixed, plainly checkable order over speed where
// the two conflict: the mean of the block constants is one sequential fp64 sum.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>

#include "../../include/qlora.h"
#include "formats.cuh"

namespace qfmt {

// Device error word of the format conversions (value 2: a non-finite input), read by ql_formats_get_device_error.
__device__ unsigned int g_fmt_error = 0;
constexpr unsigned int kFmtErrNonFinite = 2;

namespace {

std::atomic<uint64_t> g_fmt_launches{0};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }
long long cdiv(long long a, long long b) { return (a + b - 1) / b; }

int sm_count() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      sms <= 0) {
    cudaGetLastError();
    return 148;
  }
  return sms;
}

// CTAs for `items` work items at `per_cta` items per CTA pass: at most 16 resident CTAs' worth per SM.
unsigned grid_for(long long items, int per_cta) {
  const long long want = std::max<long long>(1, cdiv(items, per_cta));
  return static_cast<unsigned>(std::min<long long>(want, static_cast<long long>(sm_count()) * 16));
}

ql_status launched() {
  g_fmt_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}

// ------------------------------------------------------------------------ double quantization

__global__ void dq_group_sums_kernel(const float* __restrict__ c, long long nb, long long ng, double* __restrict__ sums) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; g < ng; g += stride) {
    const long long i0 = g * kDqGroup;
    const long long i1 = std::min<long long>(i0 + kDqGroup, nb);
    bool bad = false;
    for (long long i = i0; i < i1; ++i) bad |= !isfinite(c[i]) || c[i] < 0.0f;
    if (bad) atomicOr(&g_fmt_error, kFmtErrNonFinite);
    sums[g] = dq_group_sum(c, nb, g);
  }
}

__global__ void dq_offset_kernel(const double* __restrict__ sums, long long ng, long long nb, float* __restrict__ mu) {
  if (blockIdx.x == 0 && threadIdx.x == 0) *mu = dq_offset(sums, ng, nb);
}

// The 253 levels in ascending order, built by each CTA in shared memory.
__device__ __forceinline__ void build_sorted_levels(float* lv) {
  for (int i = threadIdx.x; i < kDqLevels; i += blockDim.x) lv[i] = dq_level(dq_code_of_sorted(i));
  __syncthreads();
}

__global__ void dq_codes_kernel(const float* __restrict__ c, long long nb, long long ng, const float* __restrict__ mu_p,
                                uint8_t* __restrict__ code8, float* __restrict__ c1) {
  __shared__ float lv[kDqLevels];
  build_sorted_levels(lv);
  const float mu = *mu_p;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; g < ng; g += stride)
    dq_quantize_group(c, nb, mu, lv, g, code8, c1);
}

__global__ void dq_dequantize_kernel(const uint8_t* __restrict__ code8, const float* __restrict__ c1,
                                     const float* __restrict__ mu_p, long long nb, float* __restrict__ out) {
  __shared__ float lv[256];  // L by code (the NaN codes 0x7F and 0xFF give NaN)
  for (int i = threadIdx.x; i < 256; i += blockDim.x)
    lv[i] = (i & 0x7F) == 0x7F ? __uint_as_float(0x7FC00000u) : dq_level(static_cast<uint32_t>(i));
  __syncthreads();
  const float mu = *mu_p;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < nb; i += stride) {
    const uint32_t code = code8[i];
    if ((code & 0x7Fu) == 0x7Fu) atomicOr(&g_fmt_error, kFmtErrNonFinite);
    out[i] = dq_dequantize_one(code, c1[i / kDqGroup], mu, lv);
  }
}

// ------------------------------------------------------------------------ NVFP4

// Largest |w| as the bits of a non-negative float (their integer order is their value order).
__global__ void nvfp4_amax_kernel(const float* __restrict__ w, long long numel, unsigned int* __restrict__ amax_bits) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  float m = 0.0f;
  bool bad = false;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < numel; i += stride) {
    const float v = w[i];
    bad |= !isfinite(v);
    m = fmaxf(m, fabsf(v));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(&g_fmt_error, kFmtErrNonFinite);
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, __float_as_uint(m));
}

__global__ void nvfp4_quantize_kernel(const float* __restrict__ w, long long nblk, const unsigned int* __restrict__ amax_bits,
                                      uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  const float amax = __uint_as_float(*amax_bits);
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long b = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; b < nblk; b += stride)
    nvfp4_quantize_block(w, b, amax, codes, scales);
}

// Replaces the largest magnitude held in the tensor-scale word by the tensor scale itself.
__global__ void nvfp4_finalize_kernel(float* tensor_scale) {
  if (blockIdx.x == 0 && threadIdx.x == 0) *tensor_scale = nvfp4_tensor_scale(*tensor_scale);
}

template <bool kBf16>
__global__ void nvfp4_dequantize_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                                        const float* __restrict__ tensor_scale, long long nblk, void* __restrict__ out) {
  const float S = *tensor_scale;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long b = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; b < nblk; b += stride) {
    const uint2 q = reinterpret_cast<const uint2*>(codes)[b];  // 16 codes, element 2j in the low nibble of byte j
    const float D = nvfp4_block_scale(scales[b], S);
    float f[16];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t byte = ((j < 4 ? q.x : q.y) >> (8 * (j & 3))) & 0xFFu;
      f[2 * j] = nvfp4_dequantize_one(byte & 15u, D);
      f[2 * j + 1] = nvfp4_dequantize_one(byte >> 4, D);
    }
    if constexpr (kBf16) {
      uint4 o[2];
      uint32_t* op = reinterpret_cast<uint32_t*>(o);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * j], f[2 * j + 1]);
        op[j] = *reinterpret_cast<const uint32_t*>(&h);
      }
      uint4* dst = reinterpret_cast<uint4*>(out) + 2 * b;
      dst[0] = o[0];
      dst[1] = o[1];
    } else {
      float4* dst = reinterpret_cast<float4*>(out) + 4 * b;
#pragma unroll
      for (int j = 0; j < 4; ++j) dst[j] = make_float4(f[4 * j], f[4 * j + 1], f[4 * j + 2], f[4 * j + 3]);
    }
  }
}

}  // namespace
}  // namespace qfmt

using namespace qfmt;

extern "C" {

uint64_t ql_formats_launch_count(void) { return g_fmt_launches.load(std::memory_order_relaxed); }

ql_status ql_formats_get_device_error(void* stream) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_fmt_error) != cudaSuccess) return QL_ERR_CUDA;
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return QL_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpy(&v, p, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return QL_ERR_CUDA;
  const unsigned int zero = 0;
  if (cudaMemcpy(p, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return QL_ERR_CUDA;
  return (v & kFmtErrNonFinite) ? QL_ERR_INVALID_ARG : QL_OK;
}

size_t nf4_double_quantize_scratch_bytes(int64_t nb) {
  return nb > 0 ? static_cast<size_t>(cdiv(nb, kDqGroup)) * sizeof(double) : 0;
}

ql_status nf4_double_quantize(const float* absmax, int64_t nb, uint8_t* code8, float* c1, float* mu, void* scratch,
                              size_t scratch_bytes, void* stream) {
  if (nb <= 0 || !absmax || !code8 || !c1 || !mu || !scratch) return QL_ERR_INVALID_ARG;
  if (!aligned16(absmax) || !aligned16(code8) || !aligned16(c1) || !aligned16(mu) || !aligned16(scratch))
    return QL_ERR_INVALID_ARG;
  if (scratch_bytes < nf4_double_quantize_scratch_bytes(nb)) return QL_ERR_INVALID_ARG;
  const long long ng = cdiv(nb, kDqGroup);
  double* sums = static_cast<double*>(scratch);
  cudaStream_t s = as_stream(stream);
  const int threads = 128;
  dq_group_sums_kernel<<<grid_for(ng, threads), threads, 0, s>>>(absmax, nb, ng, sums);
  if (launched() != QL_OK) return QL_ERR_CUDA;
  dq_offset_kernel<<<1, 32, 0, s>>>(sums, ng, nb, mu);
  if (launched() != QL_OK) return QL_ERR_CUDA;
  dq_codes_kernel<<<grid_for(ng, threads), threads, 0, s>>>(absmax, nb, ng, mu, code8, c1);
  return launched();
}

ql_status nf4_double_dequantize(const uint8_t* code8, const float* c1, const float* mu, int64_t nb, float* absmax_out,
                                void* stream) {
  if (nb <= 0 || !code8 || !c1 || !mu || !absmax_out) return QL_ERR_INVALID_ARG;
  if (!aligned16(code8) || !aligned16(c1) || !aligned16(mu) || !aligned16(absmax_out)) return QL_ERR_INVALID_ARG;
  const int threads = 256;
  dq_dequantize_kernel<<<grid_for(nb, threads), threads, 0, as_stream(stream)>>>(code8, c1, mu, nb, absmax_out);
  return launched();
}

ql_status nvfp4_quantize(const float* w, int64_t numel, uint8_t* codes, uint8_t* scales, float* tensor_scale,
                         void* stream) {
  if (numel <= 0 || numel % kFp4Block != 0 || !w || !codes || !scales || !tensor_scale) return QL_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(codes) || !aligned16(scales) || !aligned16(tensor_scale)) return QL_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  if (cudaMemsetAsync(tensor_scale, 0, sizeof(float), s) != cudaSuccess) return QL_ERR_CUDA;
  unsigned int* amax_bits = reinterpret_cast<unsigned int*>(tensor_scale);
  const int threads = 256;
  nvfp4_amax_kernel<<<grid_for(numel, threads * 8), threads, 0, s>>>(w, numel, amax_bits);
  if (launched() != QL_OK) return QL_ERR_CUDA;
  const long long nblk = numel / kFp4Block;
  nvfp4_quantize_kernel<<<grid_for(nblk, threads), threads, 0, s>>>(w, nblk, amax_bits, codes, scales);
  if (launched() != QL_OK) return QL_ERR_CUDA;
  nvfp4_finalize_kernel<<<1, 32, 0, s>>>(tensor_scale);
  return launched();
}

ql_status nvfp4_dequantize(const uint8_t* codes, const uint8_t* scales, const float* tensor_scale, int64_t numel,
                           ql_dtype out_dtype, void* out, void* stream) {
  if (numel <= 0 || numel % kFp4Block != 0 || !codes || !scales || !tensor_scale || !out) return QL_ERR_INVALID_ARG;
  if (!aligned16(codes) || !aligned16(scales) || !aligned16(tensor_scale) || !aligned16(out)) return QL_ERR_INVALID_ARG;
  if (out_dtype != QL_F32 && out_dtype != QL_BF16) return QL_ERR_INVALID_ARG;
  const long long nblk = numel / kFp4Block;
  const int threads = 256;
  if (out_dtype == QL_BF16)
    nvfp4_dequantize_kernel<true><<<grid_for(nblk, threads), threads, 0, as_stream(stream)>>>(codes, scales, tensor_scale,
                                                                                             nblk, out);
  else
    nvfp4_dequantize_kernel<false><<<grid_for(nblk, threads), threads, 0, as_stream(stream)>>>(codes, scales,
                                                                                              tensor_scale, nblk, out);
  return launched();
}

}  // extern "C"

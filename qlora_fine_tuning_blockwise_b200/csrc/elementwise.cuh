// Memory-bound kernels of the QLoRA layer: NF4 quantize / dequantize, split-K reduction, SwiGLU.
#pragma once

#include <cuda_bf16.h>

#include "nf4_table.cuh"
#include "ptx.cuh"
#include "swiglu.cuh"

namespace qlora {

// Code of a normalised value n: the number of midpoints m_i = (L_i + L_{i+1}) / 2 (exact in fp64) strictly below
// n, so a value equal to a midpoint takes the lower code.  For an fp32 n, "n > m_i" is the same test as
// "n >= t_i" with t_i the least fp32 value above m_i (m_i rounded up to fp32, stepped once more when m_i is
// itself an fp32 value), so the fifteen comparisons run in fp32 against per-thread register thresholds, and a
// four-level branch-free search (each level picks the next threshold by select) finds the count.  A NaN fails
// every comparison and takes code 0, as it fails every "n > m_i".
struct Nf4Thresholds {
  float t[15];
  __device__ __forceinline__ Nf4Thresholds() {
#pragma unroll
    for (int i = 0; i < 15; ++i) {
      const double m = (static_cast<double>(kNF4LevelsDev[i]) + static_cast<double>(kNF4LevelsDev[i + 1])) * 0.5;
      const float up = __double2float_ru(m);
      t[i] = static_cast<double>(up) == m ? nextafterf(up, INFINITY) : up;
    }
  }
  __device__ __forceinline__ uint32_t code(float n) const {
    const bool b3 = n >= t[7];
    const bool b2 = n >= (b3 ? t[11] : t[3]);
    const bool b1 = n >= (b3 ? (b2 ? t[13] : t[9]) : (b2 ? t[5] : t[1]));
    const float t0 = b3 ? (b2 ? (b1 ? t[14] : t[12]) : (b1 ? t[10] : t[8]))
                        : (b2 ? (b1 ? t[6] : t[4]) : (b1 ? t[2] : t[0]));
    const bool b0 = n >= t0;
    return (static_cast<uint32_t>(b3) << 3) | (static_cast<uint32_t>(b2) << 2) | (static_cast<uint32_t>(b1) << 1) |
           static_cast<uint32_t>(b0);
  }
};

// One warp per 64-element block: lane l owns elements 2l, 2l+1 (one packed byte).  A warp takes four consecutive
// blocks per step and issues their loads before it works on any of them, so four 8-byte loads per lane are in
// flight instead of one.
constexpr int kQuantBlocksPerStep = 4;

__global__ void nf4_quantize_kernel(const float* __restrict__ w, long long nblocks, uint8_t* __restrict__ codes,
                                    float* __restrict__ absmax, unsigned int* err) {
  const int lane = threadIdx.x & 31;
  const Nf4Thresholds thr;
  const long long warps_total = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  const long long warp_id = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  for (long long b0 = warp_id * kQuantBlocksPerStep; b0 < nblocks; b0 += warps_total * kQuantBlocksPerStep) {
    float2 v[kQuantBlocksPerStep];
#pragma unroll
    for (int i = 0; i < kQuantBlocksPerStep; ++i)
      v[i] = b0 + i < nblocks ? __ldg(reinterpret_cast<const float2*>(w) + (b0 + i) * 32 + lane) : make_float2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < kQuantBlocksPerStep; ++i) {
      const long long b = b0 + i;
      if (b >= nblocks) break;  // warp-uniform
      float m = fmaxf(fabsf(v[i].x), fabsf(v[i].y));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      const bool bad = !isfinite(v[i].x) || !isfinite(v[i].y);
      if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(err, kDevErrNonFinite);
      uint32_t c0 = 7, c1 = 7;
      if (m > 0.0f) {
        c0 = thr.code(__fdiv_rn(v[i].x, m));
        c1 = thr.code(__fdiv_rn(v[i].y, m));
      }
      codes[b * 32 + lane] = static_cast<uint8_t>((c0 << 4) | c1);
      if (lane == 0) absmax[b] = m;
    }
  }
}

// LoRA merge W' = deq(W) + s B A ("unsloth" (pyshine.com), section "Why You Need This": merged saves fold
// the adapters into the base layer by layer).  One warp per 64-element block of W' (row n of W, columns
// k0 .. k0 + 63); lane l owns elements 2l, 2l+1.  Every step is one IEEE fp32 operation, never fused, in a
// fixed order -- d = level * absmax; acc = sum over j of B[n,j] A[j,k], left to right from 0; w' = d + s acc --
// so that the requantization below is decided on a value any implementation of that order reproduces.
//   kOut = 0: W' as fp32;  1: W' as bf16 (round-to-nearest-even);  2: W' requantized to NF4 (codes_out,
//   absmax_out), by the same rule as nf4_quantize_kernel.  In mode 2 the outputs may alias the inputs: a
//   block is read in full before it is written.
template <int kOut>
__global__ void lora_merge_kernel(const uint8_t* __restrict__ codes, const float* __restrict__ absmax,
                                  const uint16_t* __restrict__ A, const uint16_t* __restrict__ B, float s,
                                  long long nblocks, int K, int r, void* __restrict__ out, uint8_t* codes_out,
                                  float* absmax_out, unsigned int* err) {
  __shared__ float lv[16];
  if (threadIdx.x < 16) lv[threadIdx.x] = kNF4LevelsDev[threadIdx.x];
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int kb = K / 64;
  const Nf4Thresholds thr;
  const long long warps_total = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  for (long long b = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); b < nblocks;
       b += warps_total) {
    const long long n = b / kb;
    const int k0 = static_cast<int>(b % kb) * 64;
    const uint32_t byte = codes[b * 32 + lane];
    const float sc = absmax[b];
    const float d0 = __fmul_rn(lv[byte >> 4], sc);
    const float d1 = __fmul_rn(lv[byte & 15u], sc);
    float acc0 = 0.0f, acc1 = 0.0f;
    const uint16_t* brow = B + n * r;
    const uint32_t* apair = reinterpret_cast<const uint32_t*>(A + k0) + lane;  // A[j, k0 + 2l .. k0 + 2l + 1]
    // eight ranks at a time: their loads are issued together (one 16-byte load of B's row when r is a multiple
    // of 8, so the row is 16-byte aligned), then summed in the same order, one rank after the other
    const int r8 = r & ~7;
    int j = 0;
    for (; j < r8; j += 8) {
      uint32_t bw[4];
      if ((r & 7) == 0) {
        const uint4 b8 = __ldg(reinterpret_cast<const uint4*>(brow + j));
        bw[0] = b8.x;
        bw[1] = b8.y;
        bw[2] = b8.z;
        bw[3] = b8.w;
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q)
          bw[q] = static_cast<uint32_t>(__ldg(brow + j + 2 * q)) | (static_cast<uint32_t>(__ldg(brow + j + 2 * q + 1)) << 16);
      }
      uint32_t a8[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) a8[q] = __ldg(apair + static_cast<long long>(j + q) * (K / 2));
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float bj = __uint_as_float((q & 1) ? (bw[q >> 1] & 0xFFFF0000u) : (bw[q >> 1] << 16));
        acc0 = __fadd_rn(acc0, __fmul_rn(bj, __uint_as_float(a8[q] << 16)));
        acc1 = __fadd_rn(acc1, __fmul_rn(bj, __uint_as_float(a8[q] & 0xFFFF0000u)));
      }
    }
    for (; j < r; ++j) {
      const float bj = __uint_as_float(static_cast<uint32_t>(__ldg(brow + j)) << 16);
      const uint32_t a = __ldg(apair + static_cast<long long>(j) * (K / 2));
      acc0 = __fadd_rn(acc0, __fmul_rn(bj, __uint_as_float(a << 16)));
      acc1 = __fadd_rn(acc1, __fmul_rn(bj, __uint_as_float(a & 0xFFFF0000u)));
    }
    const float w0 = __fadd_rn(d0, __fmul_rn(s, acc0));
    const float w1 = __fadd_rn(d1, __fmul_rn(s, acc1));
    if constexpr (kOut == 0) {
      reinterpret_cast<float2*>(out)[b * 32 + lane] = make_float2(w0, w1);
    } else if constexpr (kOut == 1) {
      reinterpret_cast<__nv_bfloat162*>(out)[b * 32 + lane] = __floats2bfloat162_rn(w0, w1);
    } else {
      float m = fmaxf(fabsf(w0), fabsf(w1));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      const bool bad = !isfinite(w0) || !isfinite(w1);
      if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(err, kDevErrNonFinite);
      uint32_t c0 = 7, c1 = 7;
      if (m > 0.0f) {
        c0 = thr.code(__fdiv_rn(w0, m));
        c1 = thr.code(__fdiv_rn(w1, m));
      }
      codes_out[b * 32 + lane] = static_cast<uint8_t>((c0 << 4) | c1);
      if (lane == 0) absmax_out[b] = m;
    }
  }
}

// Each thread expands 32 elements (16 code bytes, half a block) with one absmax: one 16-byte load of codes and
// 64 (bf16) or 128 (fp32) bytes of 16-byte stores, so every thread keeps a whole vector of HBM reads in flight.
template <bool kBf16>
__global__ void nf4_dequantize_kernel(const uint8_t* __restrict__ codes, const float* __restrict__ absmax,
                                      long long nhalves, void* __restrict__ out) {
  __shared__ float lv[16];
  if (threadIdx.x < 16) lv[threadIdx.x] = kNF4LevelsDev[threadIdx.x];
  __syncthreads();
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long q = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; q < nhalves; q += stride) {
    const uint4 cw = __ldg(reinterpret_cast<const uint4*>(codes) + q);
    const float sc = __ldg(absmax + (q >> 1));
    const uint32_t w4[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      float f[8];
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const uint32_t byte = (w4[v] >> (8 * b)) & 0xFFu;
        f[2 * b] = __fmul_rn(lv[byte >> 4], sc);
        f[2 * b + 1] = __fmul_rn(lv[byte & 15u], sc);
      }
      if (kBf16) {
        uint4 o;
        uint32_t* op = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * b], f[2 * b + 1]);
          op[b] = *reinterpret_cast<uint32_t*>(&h);
        }
        reinterpret_cast<uint4*>(out)[4 * q + v] = o;
      } else {
        float4* o = reinterpret_cast<float4*>(out) + 8 * q + 2 * v;
        o[0] = make_float4(f[0], f[1], f[2], f[3]);
        o[1] = make_float4(f[4], f[5], f[6], f[7]);
      }
    }
  }
}

// su[m, j] = bf16(s * sum_k x[m, k] A[j, k]) for token-light layers (few outputs): one warp per output; lane l
// accumulates in fp32 the products of its 8-element chunks 8 (l + 32 i) .. in order, then the lanes' sums combine
// by a fixed butterfly.  Small CTAs with no shared memory fit beside a running fused GEMM; the GEMM that consumes su
// may start at once (griddep_launch_dependents) and waits for this kernel before reading it.
__global__ void su_small_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ A, int M, int K, int r,
                                float s, uint16_t* __restrict__ su) {
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const long long w = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (w >= static_cast<long long>(M) * r) return;
  const int m = static_cast<int>(w / r), j = static_cast<int>(w % r);
  const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<long long>(m) * K);
  const uint4* ar = reinterpret_cast<const uint4*>(A + static_cast<long long>(j) * K);
  float acc = 0.0f;
  for (int c = lane; c < K / 8; c += 32) {
    const uint4 xv = __ldg(xr + c), av = __ldg(ar + c);
    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w}, aw[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      acc = __fmaf_rn(__uint_as_float(xw[q] << 16), __uint_as_float(aw[q] << 16), acc);
      acc = __fmaf_rn(__uint_as_float(xw[q] & 0xFFFF0000u), __uint_as_float(aw[q] & 0xFFFF0000u), acc);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, o));
  if (lane == 0) {
    const __nv_bfloat16 v = __float2bfloat16_rn(__fmul_rn(s, acc));
    su[static_cast<long long>(m) * r + j] = *reinterpret_cast<const uint16_t*>(&v);
  }
}

// out[e] = alpha * sum_s ws[s * slab + e]  (fp32 sum in split order: deterministic)
__global__ void reduce_splits_kernel(const float* __restrict__ ws, long long slab, int nsplit, long long count,
                                     float alpha, void* __restrict__ out, int out_bf16) {
  griddep_launch_dependents();
  griddep_wait();  // the partials are the GEMM's output
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < count; e += stride) {
    float acc = 0.0f;
    for (int s = 0; s < nsplit; ++s) acc += ws[s * slab + e];
    acc *= alpha;
    if (out_bf16)
      reinterpret_cast<__nv_bfloat16*>(out)[e] = __float2bfloat16_rn(acc);
    else
      reinterpret_cast<float*>(out)[e] = acc;
  }
}


__global__ void swiglu_fwd_kernel(const __nv_bfloat16* __restrict__ g, const __nv_bfloat16* __restrict__ u,
                                  __nv_bfloat16* __restrict__ h, long long numel) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < numel; e += stride) {
    const float gv = __bfloat162float(g[e]);
    const float uv = __bfloat162float(u[e]);
    h[e] = __float2bfloat16_rn(swiglu_h(gv, uv));
  }
}

__global__ void swiglu_bwd_kernel(const __nv_bfloat16* dh, const __nv_bfloat16* __restrict__ g,
                                  const __nv_bfloat16* __restrict__ u, __nv_bfloat16* dg, __nv_bfloat16* du,
                                  long long numel) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < numel; e += stride) {
    const float gv = __bfloat162float(g[e]);
    const float uv = __bfloat162float(u[e]);
    const float dv = __bfloat162float(dh[e]);
    float dgv, duv;
    swiglu_grads(dv, gv, uv, dgv, duv);
    dg[e] = __float2bfloat16_rn(dgv);
    du[e] = __float2bfloat16_rn(duv);
  }
}

// Gated form over the fused gate/up output gu [M, 2F] (row m: g in columns [0, F), up in [F, 2F)):
//   h[m, f] = silu(g) * up.  Each thread handles 8 consecutive f (F % 8 == 0) with 16-byte accesses.
__global__ void swiglu_gated_fwd_kernel(const __nv_bfloat16* __restrict__ gu, __nv_bfloat16* __restrict__ h,
                                        long long M, long long F) {
  const long long groups = M * (F / 8);
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < groups; e += stride) {
    const long long m = e / (F / 8), f = (e % (F / 8)) * 8;
    const uint4 gv = *reinterpret_cast<const uint4*>(gu + m * 2 * F + f);
    const uint4 uv = *reinterpret_cast<const uint4*>(gu + m * 2 * F + F + f);
    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gv);
    const __nv_bfloat162* u2 = reinterpret_cast<const __nv_bfloat162*>(&uv);
    uint4 out;
    __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(&out);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 g = __bfloat1622float2(g2[i]);
      const float2 u = __bfloat1622float2(u2[i]);
      o2[i] = __floats2bfloat162_rn(swiglu_h(g.x, u.x), swiglu_h(g.y, u.y));
    }
    *reinterpret_cast<uint4*>(h + m * F + f) = out;
  }
}

//   dgu[m, f] = dh * up * silu'(g),  dgu[m, F + f] = dh * silu(g)  -- the upstream gradient of the fused
//   gate/up layer.
__global__ void swiglu_gated_bwd_kernel(const __nv_bfloat16* __restrict__ dh, const __nv_bfloat16* __restrict__ gu,
                                        __nv_bfloat16* __restrict__ dgu, long long M, long long F) {
  const long long groups = M * (F / 8);
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < groups; e += stride) {
    const long long m = e / (F / 8), f = (e % (F / 8)) * 8;
    const uint4 dv = *reinterpret_cast<const uint4*>(dh + m * F + f);
    const uint4 gv = *reinterpret_cast<const uint4*>(gu + m * 2 * F + f);
    const uint4 uv = *reinterpret_cast<const uint4*>(gu + m * 2 * F + F + f);
    const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv);
    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gv);
    const __nv_bfloat162* u2 = reinterpret_cast<const __nv_bfloat162*>(&uv);
    uint4 og, ou;
    __nv_bfloat162* og2 = reinterpret_cast<__nv_bfloat162*>(&og);
    __nv_bfloat162* ou2 = reinterpret_cast<__nv_bfloat162*>(&ou);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 d = __bfloat1622float2(d2[i]);
      const float2 g = __bfloat1622float2(g2[i]);
      const float2 u = __bfloat1622float2(u2[i]);
      float gx, ux, gy, uy;
      swiglu_grads(d.x, g.x, u.x, gx, ux);
      swiglu_grads(d.y, g.y, u.y, gy, uy);
      og2[i] = __floats2bfloat162_rn(gx, gy);
      ou2[i] = __floats2bfloat162_rn(ux, uy);
    }
    *reinterpret_cast<uint4*>(dgu + m * 2 * F + f) = og;
    *reinterpret_cast<uint4*>(dgu + m * 2 * F + F + f) = ou;
  }
}

// The same two steps over the interleaved gate/up layout (gate_pos / up_pos), for the calls whose GEMM splits
// its contraction (the fused epilogues need the whole sum in one place).  8 consecutive features per thread.
__global__ void swiglu_interleaved_fwd_kernel(const __nv_bfloat16* __restrict__ gu, __nv_bfloat16* __restrict__ h,
                                              long long M, long long F) {
  const long long groups = M * (F / 8);
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < groups; e += stride) {
    const long long m = e / (F / 8), f = (e % (F / 8)) * 8;
    const uint4 gv = *reinterpret_cast<const uint4*>(gu + m * 2 * F + gate_pos(f));
    const uint4 uv = *reinterpret_cast<const uint4*>(gu + m * 2 * F + up_pos(f));
    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gv);
    const __nv_bfloat162* u2 = reinterpret_cast<const __nv_bfloat162*>(&uv);
    uint4 out;
    __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(&out);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 g = __bfloat1622float2(g2[i]);
      const float2 u = __bfloat1622float2(u2[i]);
      o2[i] = __floats2bfloat162_rn(swiglu_h(g.x, u.x), swiglu_h(g.y, u.y));
    }
    *reinterpret_cast<uint4*>(h + m * F + f) = out;
  }
}

__global__ void swiglu_interleaved_bwd_kernel(const __nv_bfloat16* __restrict__ dh, const __nv_bfloat16* __restrict__ gu,
                                              __nv_bfloat16* __restrict__ dgu, long long M, long long F) {
  const long long groups = M * (F / 8);
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < groups; e += stride) {
    const long long m = e / (F / 8), f = (e % (F / 8)) * 8;
    const uint4 dv = *reinterpret_cast<const uint4*>(dh + m * F + f);
    const uint4 gv = *reinterpret_cast<const uint4*>(gu + m * 2 * F + gate_pos(f));
    const uint4 uv = *reinterpret_cast<const uint4*>(gu + m * 2 * F + up_pos(f));
    const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv);
    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gv);
    const __nv_bfloat162* u2 = reinterpret_cast<const __nv_bfloat162*>(&uv);
    uint4 og, ou;
    __nv_bfloat162* og2 = reinterpret_cast<__nv_bfloat162*>(&og);
    __nv_bfloat162* ou2 = reinterpret_cast<__nv_bfloat162*>(&ou);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 d = __bfloat1622float2(d2[i]);
      const float2 g = __bfloat1622float2(g2[i]);
      const float2 u = __bfloat1622float2(u2[i]);
      float gx, ux, gy, uy;
      swiglu_grads(d.x, g.x, u.x, gx, ux);
      swiglu_grads(d.y, g.y, u.y, gy, uy);
      og2[i] = __floats2bfloat162_rn(gx, gy);
      ou2[i] = __floats2bfloat162_rn(ux, uy);
    }
    *reinterpret_cast<uint4*>(dgu + m * 2 * F + gate_pos(f)) = og;
    *reinterpret_cast<uint4*>(dgu + m * 2 * F + up_pos(f)) = ou;
  }
}

// Waits on a barrier that expects one arrival nobody makes; the bounded wait must give up and latch the
// timeout bit.  Used only by ql_selftest_wait_timeout.
__global__ void selftest_wait_kernel(long long limit, unsigned int* err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, err, limit);
  __syncthreads();
}

}  // namespace qlora

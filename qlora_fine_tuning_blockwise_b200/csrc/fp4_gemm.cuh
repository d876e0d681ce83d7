// The NVFP4 form of the QLoRA forward on the block-scaled FP4 tensor core (sm_100a):
//   y = (Sw Sx) * sum_k e2m1(x)[m,k] sbx[m,k/16] e2m1(W)[n,k] sbw[n,k/16]  +  s (x A^T) B^T
// ("Major Unsloth Update: NVFP4 Quantization Export and DeepSeek-V4 Training Support" (kongchang.com), section
// "NVFP4: A Quantization Format for the Next Generation of Hardware": E2M1 values sharing an FP8 scale per
// group, multiplied directly by Blackwell's FP4 tensor cores).  Both operands are NVFP4: the frozen weight is
// quantized once; the activations are quantized by the same rule, with their own tensor scale, on every call.
// The base product runs as tcgen05.mma kind::mxf4nvf4 with 16-element scale blocks; the rank-r term keeps the
// unquantized activations (bf16 s x A^T) and runs as bf16 MMAs into a second accumulator, because the tensor
// scales Sw, Sx multiply the base product only.
//
// Scale factors live in the tensor core's layout ("MMA scale layout"): the operand's rows in blocks of 128, its
// contraction in steps of 64 elements (4 groups of 16); one 512-byte atom per (row block, step), the atoms of a
// row block consecutive along the contraction (padded to a multiple of 4 steps, zero-filled), row blocks
// consecutive.  Inside an atom the scale of group g (0..3) of row 32 r1 + r0 sits at byte 16 r0 + 4 r1 + g.  A
// tcgen05.cp of 32 rows x 16 bytes then puts row r0's 16 bytes -- the scales of rows r0, r0 + 32, r0 + 64,
// r0 + 96 -- in 4 consecutive TMEM columns of lane r0 (and of lanes r0 + 32, r0 + 64, r0 + 96), where the MMA
// reads the scales of row m in column m / 32 of its own lane.
#pragma once

#include <cuda_bf16.h>

#include "formats.cuh"
#include "ptx.cuh"
#include "umma_gemm.cuh"

namespace qlora {

__host__ __device__ inline long long fp4_sf_steps(long long K) { return ((K + 255) / 256) * 4; }
__host__ __device__ inline long long fp4_sf_rowblock_bytes(long long K) { return fp4_sf_steps(K) * 512; }
__host__ __device__ inline long long fp4_sf_bytes(long long rows, long long K) {
  return ((rows + 127) / 128) * fp4_sf_rowblock_bytes(K);
}
// Byte of the scale of group `group` (= k / 16) of row `row`.
__host__ __device__ inline long long fp4_sf_offset(long long row, long long group, long long K) {
  const long long r = row & 127;
  return (row >> 7) * fp4_sf_rowblock_bytes(K) + (group >> 2) * 512 + (r & 31) * 16 + (r >> 5) * 4 + (group & 3);
}

// ------------------------------------------------------------------------------------------ conversions

// Row-major scales [rows, K / 16] -> the MMA scale layout (out zero-filled beforehand).
__global__ void fp4_sf_to_mma_kernel(const uint8_t* __restrict__ scales, long long rows, long long K,
                                     uint8_t* __restrict__ out) {
  const long long groups = K / 16, n = rows * groups;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < n; e += stride)
    out[fp4_sf_offset(e / groups, e % groups, K)] = scales[e];
}

// Largest |x| of bf16 activations, as the bits of a non-negative float.
__global__ void fp4_act_amax_kernel(const __nv_bfloat16* __restrict__ x, long long numel,
                                    unsigned int* __restrict__ amax_bits, unsigned int* err) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  float m = 0.0f;
  bool bad = false;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < numel; i += stride) {
    const float v = __bfloat162float(x[i]);
    bad |= !isfinite(v);
    m = fmaxf(m, fabsf(v));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(err, kDevErrNonFinite);
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, __float_as_uint(m));
}

// One 16-element block of bf16 activations per thread: the NVFP4 rule of the weight (the same per-block
// arithmetic), codes row-major [M, K/2] (element 2j in the low nibble), scale into the MMA layout.
__global__ void fp4_act_quantize_kernel(const __nv_bfloat16* __restrict__ x, long long M, long long K,
                                        const unsigned int* __restrict__ amax_bits, uint8_t* __restrict__ codes,
                                        uint8_t* __restrict__ sf) {
  const float amax = __uint_as_float(*amax_bits);
  const long long groups = K / 16, nblk = M * groups;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long b = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; b < nblk; b += stride) {
    const uint4 v0 = *reinterpret_cast<const uint4*>(x + b * 16);
    const uint4 v1 = *reinterpret_cast<const uint4*>(x + b * 16 + 8);
    const uint32_t wv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    float w[16];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      w[2 * j] = __uint_as_float(wv[j] << 16);
      w[2 * j + 1] = __uint_as_float(wv[j] & 0xFFFF0000u);
    }
    uint8_t q[8], sb;
    qfmt::nvfp4_quantize_block(w, 0, amax, q, &sb);
    *reinterpret_cast<uint2*>(codes + b * 8) =
        make_uint2(q[0] | (q[1] << 8) | (q[2] << 16) | (static_cast<uint32_t>(q[3]) << 24),
                   q[4] | (q[5] << 8) | (q[6] << 16) | (static_cast<uint32_t>(q[7]) << 24));
    sf[fp4_sf_offset(b / groups, b % groups, K)] = sb;
  }
}

// Replaces the largest magnitude in the tensor-scale word by the tensor scale amax / 2688.
__global__ void fp4_act_finalize_kernel(float* tensor_scale) {
  if (blockIdx.x == 0 && threadIdx.x == 0) *tensor_scale = qfmt::nvfp4_tensor_scale(*tensor_scale);
}

// ------------------------------------------------------------------------------------------ the GEMM

struct Fp4Args {
  int rows, cols;           // D extent: i over weight rows (N), j over tokens (M)
  int tiles_i, tiles_j;     // ceil(rows / 128), ceil(cols / BN)
  int group_i;              // unit order: groups of weight tiles (0: tokens fastest)
  int k_stages;             // stages of 256 contraction elements (one 128-byte code row per operand row)
  int n_extra;              // LoRA stages of 64 bf16 contraction elements, after the base stages
  const uint8_t* sfa;       // weight scales, MMA layout
  const uint8_t* sfb;       // activation scales, MMA layout
  long long sf_rb_bytes;    // bytes of one row block of either scale buffer (same contraction length)
  const float* Sa;          // weight tensor scale
  const float* Sb;          // activation tensor scale
  __nv_bfloat16* out;       // y[j * ld + i]
  long long ld;
  int rows_lim, cols_lim;
  unsigned int* err;
};

template <int BN>
struct Fp4Cfg {
  static constexpr int kStages = 5;
  static constexpr int kABytes = 128 * 128;       // 128 weight rows x 128 bytes (256 E2M1, or 64 bf16 LoRA)
  static constexpr int kBBytes = BN * 128;        // BN token rows x 128 bytes
  static constexpr int kSfBytes = 4 * 512;        // one stage's 4 scale atoms of one 128-row block
  static constexpr int kSlot = kABytes + kBBytes + 2 * kSfBytes;
  static constexpr int kSmemBytes = 1024 + kStages * kSlot + 256;
  static constexpr int kAcc1 = BN;                // LoRA accumulator column
  static constexpr int kSfCol = 2 * BN;           // scale slots: 32 columns per stage (16 weight, 16 activation)
  static constexpr int kTmemCols = 512;
  static_assert(BN == 128, "one 128-row scale block per token tile");
  static_assert(kSfCol + kStages * 32 <= kTmemCols, "tensor memory");
  static_assert(kSlot % 1024 == 0 && kSmemBytes <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ void fp4_unit(const Fp4Args& a, int u, int BN, int& i0, int& j0) {
  int ti, tj;
  if (a.group_i > 0) {
    const int grp = u / (a.group_i * a.tiles_j);
    const int gi0 = grp * a.group_i;
    const int gsz = a.tiles_i - gi0 < a.group_i ? a.tiles_i - gi0 : a.group_i;
    const int local = u - gi0 * a.tiles_j;
    ti = gi0 + local % gsz;
    tj = local / gsz;
  } else {
    tj = u % a.tiles_j;
    ti = u / a.tiles_j;
  }
  i0 = ti * 128;
  j0 = tj * BN;
}

// Warp 0: TMA / bulk-copy producer; warp 1: TMEM allocation, scale copies into TMEM and the MMAs (one elected
// lane); warps 2..5: epilogue.  Persistent over units; every wait is bounded as in umma_gemm_kernel.
template <int BN>
__global__ void __launch_bounds__(192, 1)
    fp4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmLA, const __grid_constant__ CUtensorMap tmLB,
                    const Fp4Args args) {
  using C = Fp4Cfg<BN>;
  constexpr int S = C::kStages;
  constexpr uint32_t kFull = 0xffffffffu;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * C::kSlot);
  uint64_t* empty = full + S;
  uint64_t* tmem_full = empty + S;
  uint64_t* tmem_empty = tmem_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tmem_empty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_units = args.tiles_i * args.tiles_j;
  const int n_total = args.k_stages + args.n_extra;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tmem_full, 1);
    mbar_init(tmem_empty, 4);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (args.n_extra > 0) {
      tma_prefetch_desc(&tmLA);
      tma_prefetch_desc(&tmLB);
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

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    Armed armed;
    int g = 0;
    bool stop = false;
    for (int u = blockIdx.x; u < num_units && !stop; u += gridDim.x) {
      int i0, j0;
      fp4_unit(args, u, BN, i0, j0);
      for (int it = 0; it < n_total; ++it, ++g) {
        const int s = g % S;
        const uint32_t ph = static_cast<uint32_t>(g / S) & 1u;
        const bool ok = mbar_wait_idle(&empty[s], ph ^ 1u, abort_flag, args.err);
        if (!__all_sync(kFull, ok)) {
          stop = true;
          break;
        }
        if (lane == 0) {
          armed.set(s, ph);
          uint8_t* slot = smem + s * C::kSlot;
          if (it < args.k_stages) {
            mbar_arrive_expect_tx(&full[s], C::kABytes + C::kBBytes + 2 * C::kSfBytes);
            tma_load_2d(slot, &tmA, it * 128, i0, &full[s]);
            tma_load_2d(slot + C::kABytes, &tmB, it * 128, j0, &full[s]);
            bulk_load(slot + C::kABytes + C::kBBytes, args.sfa + (i0 >> 7) * args.sf_rb_bytes + it * C::kSfBytes,
                      C::kSfBytes, &full[s]);
            bulk_load(slot + C::kABytes + C::kBBytes + C::kSfBytes,
                      args.sfb + (j0 >> 7) * args.sf_rb_bytes + it * C::kSfBytes, C::kSfBytes, &full[s]);
          } else {
            const int e = it - args.k_stages;
            mbar_arrive_expect_tx(&full[s], C::kABytes + C::kBBytes);
            tma_load_2d(slot, &tmLA, e * 64, i0, &full[s]);
            tma_load_2d(slot + C::kABytes, &tmLB, e * 64, j0, &full[s]);
          }
        }
        __syncwarp();
      }
    }
    if (lane == 0 && *abort_flag) armed.drain(full, S, args.err);
  } else if (warp == 1) {
    // ------------------------------------------------------------------ scale copies + MMAs
    constexpr uint32_t idesc4 = idesc_fp4_block16(128, BN);
    constexpr uint32_t idesc16 = idesc_bf16_f32(128, BN, false, false);
    int g = 0, lu = 0;
    bool stop = false;
    for (int u = blockIdx.x; u < num_units && !stop; u += gridDim.x, ++lu) {
      if (!__all_sync(kFull, mbar_wait(tmem_empty, (static_cast<uint32_t>(lu) & 1u) ^ 1u, abort_flag, args.err)))
        break;
      tc_fence_after();
      for (int it = 0; it < n_total; ++it, ++g) {
        const int s = g % S;
        if (!__all_sync(kFull, mbar_wait(&full[s], static_cast<uint32_t>(g / S) & 1u, abort_flag, args.err))) {
          stop = true;
          break;
        }
        tc_fence_after();
        if (elect_one()) {
          const uint32_t a0 = smem_u32(smem + s * C::kSlot);
          const uint32_t b0 = a0 + C::kABytes;
          if (it < args.k_stages) {
            const uint32_t sfa0 = b0 + C::kBBytes, sfb0 = sfa0 + C::kSfBytes;
            const uint32_t tsf = tmem_base + static_cast<uint32_t>(C::kSfCol + s * 32);
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
              tmem_cp_32x128b_warpx4(tsf + kb * 4, sdesc_noswizzle(sfa0 + kb * 512, 128));
              tmem_cp_32x128b_warpx4(tsf + 16 + kb * 4, sdesc_noswizzle(sfb0 + kb * 512, 128));
            }
#pragma unroll
            for (int kb = 0; kb < 4; ++kb)
              umma_fp4_block16(tmem_base, sdesc_sw128(a0 + kb * 32, 16, 1024), sdesc_sw128(b0 + kb * 32, 16, 1024),
                               idesc4, tsf + kb * 4, tsf + 16 + kb * 4, (it > 0 || kb > 0) ? 1u : 0u);
          } else {
            const int e = it - args.k_stages;
#pragma unroll
            for (int k = 0; k < 4; ++k)
              umma_bf16_ss(tmem_base + C::kAcc1, sdesc_sw128(a0 + k * 32, 16, 1024), sdesc_sw128(b0 + k * 32, 16, 1024),
                           idesc16, (e > 0 || k > 0) ? 1u : 0u);
          }
          umma_commit(&empty[s]);
        }
        __syncwarp();
      }
      if (elect_one()) umma_commit(tmem_full);  // also on abort, so the MMAs issued can be waited for
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------------ epilogue (warps 2..5)
    const int qw = warp & 3;
    const float alpha = __fmul_rn(*args.Sa, *args.Sb);
    int lu = 0;
    for (int u = blockIdx.x; u < num_units; u += gridDim.x, ++lu) {
      int i0, j0;
      fp4_unit(args, u, BN, i0, j0);
      int ok = mbar_wait_idle(tmem_full, static_cast<uint32_t>(lu) & 1u, abort_flag, args.err) ? 1 : 0;
      tc_fence_after();
      ok = __shfl_sync(kFull, ok && !*abort_flag, 0);
      if (!ok) break;
      const int i = i0 + qw * 32 + lane;
      const uint32_t t0 = tmem_base + (static_cast<uint32_t>(qw * 32) << 16);
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 16) {
        uint32_t rb[16], rl[16];
        __syncwarp();
        tmem_ld_32x32b_x16(t0 + static_cast<uint32_t>(c0), rb);
        if (args.n_extra > 0) tmem_ld_32x32b_x16(t0 + static_cast<uint32_t>(C::kAcc1 + c0), rl);
        tmem_ld_wait();
        if (i < args.rows_lim) {
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            const int j = j0 + c0 + jj;
            if (j < args.cols_lim) {
              float v = __fmul_rn(alpha, __uint_as_float(rb[jj]));
              if (args.n_extra > 0) v = __fadd_rn(v, __uint_as_float(rl[jj]));
              args.out[static_cast<long long>(j) * args.ld + i] = __float2bfloat16_rn(v);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tmem_empty);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

}  // namespace qlora

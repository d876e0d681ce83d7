// tcgen05 GEMM tile kernel for the QLoRA layer (sm_100a).
//
// One CTA computes a 128 x BN fp32 tile of D[i, j] = sum_kk Aop[i, kk] * Bop[j, kk] in TMEM, over a range
// of 64-wide contraction stages, optionally preceded by "extra" stages that append the rank-r LoRA
// columns to the contraction ([x | s u] . [deq(W) | B]^T in the forward, [dY | v] . [deq(W); A] in the
// backward), so base and LoRA products land in one accumulator.
//
// The weight is always the 128-row (M-side) operand: the kernel computes the transposed product
// (y^T = deq(W) x^T, dX^T = deq(W)^T dY^T), so one dequantized weight element feeds BN tokens.
//
// Operand A, per stage (128 rows x 64 contraction elements, bf16, 128-byte swizzled canonical layout):
//   A_TMA_K / A_TMA_MN   loaded by TMA from a bf16 matrix (K-major or MN-major),
//   A_DEQ_K              dequantized from NF4 codes by producer warps (forward: rows = W rows n, K-major),
//   A_DEQ_MN             dequantized the same way into the MN-major layout (backward: rows = W columns k,
//                        contraction over W rows n) -- the transpose of deq(W) costs nothing extra.
//   The codes arrive by TMA into a shared-memory ring; absmax is read with __ldg one stage ahead.
// Operand B (BN x 64): always by TMA (K-major or MN-major).
//
// Warp roles: warp 0 = TMA producer (one thread), warp 1 = TMEM allocator + MMA issuer (one thread),
// warps 2..9 = dequantizers (A_DEQ_* only, two groups of 4 alternating over stages), warps 2..5 = epilogue
// (TMEM -> registers -> global).
//
// Shared-memory tiles: for the 128B swizzle every tile starts on a 1024-byte boundary; row r of a tile is
// 128 bytes at r*128 and its 16-byte chunk c sits at chunk position c ^ (r & 7).  TMA writes that layout;
// the dequantizers write it with plain 16-byte stores followed by fence.proxy.async.
#pragma once

#include <cuda_bf16.h>

#include "nf4_table.cuh"
#include "ptx.cuh"

namespace qlora {

enum AMode : int { A_TMA_K = 0, A_TMA_MN = 1, A_DEQ_K = 2, A_DEQ_MN = 3 };

struct UmmaArgs {
  int rows, cols;         // D extent: i in [0, rows), j in [0, cols)
  int k_stages;           // main contraction stages (64 elements each) in total
  int stages_per_split;   // main stages per blockIdx.z
  int n_extra;            // extra (LoRA) stages, run by split 0 only, before the main stages
  // dequantization (A_DEQ_*): W is [w_rows, w_cols] with absmax [w_rows, w_cols / 64]
  const float* absmax;
  int w_rows, w_cols, w_kb;
  // epilogue: out[z * split_stride + i * ls + j * cs] = alpha * D[i, j] for i < rows_lim, j < cols_lim
  void* out;
  int out_bf16;
  float alpha;
  long long ls, cs, split_stride;
  int rows_lim, cols_lim;
  unsigned int* err;
};

template <int BN, int AM, bool B_MN>
struct UmmaCfg {
  static constexpr bool kDeq = (AM == A_DEQ_K || AM == A_DEQ_MN);
  static constexpr bool kAMN = (AM == A_TMA_MN || AM == A_DEQ_MN);
  static constexpr int kABytes = 128 * 64 * 2;
  static constexpr int kBBytes = BN * 64 * 2;
  static constexpr int kCBytes = kDeq ? 4096 : 0;
  static constexpr int kStageBytes = kABytes + kBBytes + kCBytes;
  static constexpr int kStagesRaw = (210 * 1024) / kStageBytes;
  static constexpr int kStagesCap = kStagesRaw > 8 ? 8 : kStagesRaw;
  // the two dequantizer groups alternate over main stages; with an even ring every slot keeps one group
  static constexpr int kStages = kDeq ? (kStagesCap & ~1) : kStagesCap;
  static constexpr int kDeqWarpsPerGroup = 4;
  static constexpr int kThreads = 64 + (kDeq ? 256 : 128);
  static constexpr int kTmemCols = BN <= 32 ? 32 : BN <= 64 ? 64 : BN <= 128 ? 128 : 256;
  static constexpr int kBarBytes = 512;  // 4 barrier arrays x 8 stages + accumulator barrier + TMEM slot + abort flag
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kBarBytes;
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N for M=128 is a multiple of 16 in [16, 256]");
  static_assert(!B_MN || BN % 64 == 0, "MN-major B tiles are whole 64-element swizzle atoms");
  static_assert(kStages >= 2, "pipeline needs two stages");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
  static_assert((4 * kStages + 1) * 8 + 8 <= kBarBytes, "barrier area");
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// The 16 levels of one block scaled by its absmax and rounded to bf16 -- exactly the values
// nf4_dequantize(..., bf16) produces -- held in registers as byte planes for byte-permute lookups:
// lo[j] holds the low bytes of entries 4j..4j+3, hi[j] their high bytes.
struct Nf4RegTable {
  uint32_t lo[4], hi[4];
};

__device__ __forceinline__ Nf4RegTable nf4_reg_table(float sc) {
  const float lv[16] = {QLORA_NF4_LEVELS};
  uint32_t p[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    __nv_bfloat162 h = __floats2bfloat162_rn(__fmul_rn(lv[2 * i], sc), __fmul_rn(lv[2 * i + 1], sc));
    p[i] = *reinterpret_cast<uint32_t*>(&h);
  }
  Nf4RegTable t;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    t.lo[j] = prmt(p[2 * j], p[2 * j + 1], 0x6420u);
    t.hi[j] = prmt(p[2 * j], p[2 * j + 1], 0x7531u);
  }
  return t;
}

// Eight codes (one 32-bit word: byte j = element 2j in the high nibble, 2j+1 in the low nibble) ->
// eight bf16 values in element order (four bf16 pairs, first element in the low half).
// Each nibble v selects byte (v & 7) of the table half v >> 3; a byte mask from bit 3 picks the half.
__device__ __forceinline__ void nf4_lookup8(const Nf4RegTable& t, uint32_t q, uint32_t (&o)[4]) {
  const uint32_t s0 = q & 0x77777777u;
  const uint32_t b0 = (q >> 3) & 0x11111111u;
  const uint32_t s1 = s0 >> 16;
  const uint32_t b1 = b0 >> 16;
  const uint32_t m0 = prmt(0x0000FF00u, 0u, b0);  // byte i: 0xFF when code (i ^ 1) of the low half is >= 8
  const uint32_t m1 = prmt(0x0000FF00u, 0u, b1);
  const uint32_t L0 = (prmt(t.lo[0], t.lo[1], s0) & ~m0) | (prmt(t.lo[2], t.lo[3], s0) & m0);
  const uint32_t H0 = (prmt(t.hi[0], t.hi[1], s0) & ~m0) | (prmt(t.hi[2], t.hi[3], s0) & m0);
  const uint32_t L1 = (prmt(t.lo[0], t.lo[1], s1) & ~m1) | (prmt(t.lo[2], t.lo[3], s1) & m1);
  const uint32_t H1 = (prmt(t.hi[0], t.hi[1], s1) & ~m1) | (prmt(t.hi[2], t.hi[3], s1) & m1);
  // L0/H0 hold elements in the order (1, 0, 3, 2); interleave low and high bytes back into element order
  o[0] = prmt(L0, H0, 0x4051u);
  o[1] = prmt(L0, H0, 0x6273u);
  o[2] = prmt(L1, H1, 0x4051u);
  o[3] = prmt(L1, H1, 0x6273u);
}

__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity, unsigned int* err) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitTimeoutCycles) {
      atomicOr(err, kDevErrTimeout);
      return false;
    }
  }
  return true;
}

template <int BN, int AM, bool B_MN>
__global__ void __launch_bounds__(UmmaCfg<BN, AM, B_MN>::kThreads, 1)
    umma_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmBx, const __grid_constant__ CUtensorMap tmC,
                     const UmmaArgs args) {
  using C = UmmaCfg<BN, AM, B_MN>;
  constexpr int ST = C::kStages;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + ST * C::kABytes;
  uint8_t* sC = sB + ST * C::kBBytes;
  // Barrier phases: full_tma[s] and empty[s] advance once per use of slot s (every stage); full_codes[s]
  // and full_deq[s] once per MAIN-stage use of slot s (the LoRA stages carry no codes).  Each waiter visits
  // every phase of the barriers it waits on, so a parity wait never aliases an older phase.
  uint64_t* full_tma = reinterpret_cast<uint64_t*>(sC + ST * C::kCBytes);
  uint64_t* full_codes = full_tma + ST;
  uint64_t* full_deq = full_codes + ST;
  uint64_t* empty = full_deq + ST;
  uint64_t* accum_full = empty + ST;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int j0 = blockIdx.x * BN;
  const int i0 = blockIdx.y * 128;
  const int z = blockIdx.z;

  const int main_begin = z * args.stages_per_split;
  int main_end = main_begin + args.stages_per_split;
  if (main_end > args.k_stages) main_end = args.k_stages;
  const int n_main = main_end > main_begin ? main_end - main_begin : 0;
  const int n_extra = (z == 0) ? args.n_extra : 0;
  const int n_total = n_extra + n_main;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full_tma[s], 1);
      mbar_init(&full_codes[s], 1);
      mbar_init(&full_deq[s], C::kDeqWarpsPerGroup);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accum_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmB);
    if (C::kDeq) tma_prefetch_desc(&tmC);
    if (!C::kDeq || args.n_extra > 0) tma_prefetch_desc(&tmA);
    if (args.n_extra > 0) tma_prefetch_desc(&tmBx);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t armed_tma = 0, armed_codes = 0;  // bit s: slot s has an armed phase whose copies may be in flight
      uint32_t tma_par = 0, codes_par = 0;      // bit s: parity of that armed phase
      for (int it = 0; it < n_total; ++it) {
        const int s = it % ST;
        const uint32_t round = static_cast<uint32_t>(it / ST);
        if (!mbar_wait(&empty[s], (round & 1u) ^ 1u, abort_flag, args.err)) break;
        uint8_t* a_dst = sA + s * C::kABytes;
        uint8_t* b_dst = sB + s * C::kBBytes;
        armed_tma |= 1u << s;
        tma_par = (tma_par & ~(1u << s)) | ((round & 1u) << s);
        if (it < n_extra) {
          const int e = it;
          mbar_arrive_expect_tx(&full_tma[s], C::kABytes + C::kBBytes);
          if (C::kAMN) {
            tma_load_2d(a_dst, &tmA, i0, 64 * e, &full_tma[s]);
            tma_load_2d(a_dst + 8192, &tmA, i0 + 64, 64 * e, &full_tma[s]);
          } else {
            tma_load_2d(a_dst, &tmA, 64 * e, i0, &full_tma[s]);
          }
          tma_load_2d(b_dst, &tmBx, 64 * e, j0, &full_tma[s]);
        } else {
          const int kk0 = (main_begin + it - n_extra) * 64;
          mbar_arrive_expect_tx(&full_tma[s], C::kBBytes + (C::kDeq ? 0 : C::kABytes));
          if (B_MN) {
#pragma unroll
            for (int c = 0; c < BN / 64; ++c) tma_load_2d(b_dst + c * 8192, &tmB, j0 + 64 * c, kk0, &full_tma[s]);
          } else {
            tma_load_2d(b_dst, &tmB, kk0, j0, &full_tma[s]);
          }
          if constexpr (C::kDeq) {
            // codes of this stage on their own barrier; waiting on empty[s] above made A[s] free to overwrite
            const uint32_t cpar = ((codes_par >> s) & 1u) ^ ((armed_codes >> s) & 1u);
            armed_codes |= 1u << s;
            codes_par = (codes_par & ~(1u << s)) | (cpar << s);
            mbar_arrive_expect_tx(&full_codes[s], C::kCBytes);
            if constexpr (AM == A_DEQ_K)
              tma_load_2d(sC + s * C::kCBytes, &tmC, kk0 / 2, i0, &full_codes[s]);
            else
              tma_load_2d(sC + s * C::kCBytes, &tmC, i0 / 2, kk0, &full_codes[s]);
          } else if constexpr (AM == A_TMA_MN) {
            tma_load_2d(a_dst, &tmA, i0, kk0, &full_tma[s]);
            tma_load_2d(a_dst + 8192, &tmA, i0 + 64, kk0, &full_tma[s]);
          } else {
            tma_load_2d(a_dst, &tmA, kk0, i0, &full_tma[s]);
          }
        }
      }
      if (*abort_flag) {
        // copies still in flight must land before the CTA's shared memory is released: wait for the last
        // armed phase of every slot (already complete ones return at once)
        for (int s = 0; s < ST; ++s) {
          if ((armed_tma >> s) & 1u) mbar_wait_drain(&full_tma[s], (tma_par >> s) & 1u, args.err);
          if ((armed_codes >> s) & 1u) mbar_wait_drain(&full_codes[s], (codes_par >> s) & 1u, args.err);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, BN, C::kAMN, B_MN);
      // The dequantizers arrive on full_deq[s] for main stages only, so its phases count the main-stage
      // uses of slot s, not the rounds of the ring: bit s holds the parity of the next phase to wait for.
      uint32_t deq_phase = 0;
      for (int it = 0; it < n_total; ++it) {
        const int s = it % ST;
        const uint32_t par = static_cast<uint32_t>(it / ST) & 1u;
        if (!mbar_wait(&full_tma[s], par, abort_flag, args.err)) break;
        if (C::kDeq && it >= n_extra) {
          if (!mbar_wait(&full_deq[s], (deq_phase >> s) & 1u, abort_flag, args.err)) break;
          deq_phase ^= 1u << s;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA + s * C::kABytes);
        const uint32_t b0 = smem_u32(sB + s * C::kBBytes);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint64_t adesc = C::kAMN ? sdesc_sw128(a0 + k * 2048, 8192, 1024) : sdesc_sw128(a0 + k * 32, 16, 1024);
          const uint64_t bdesc = B_MN ? sdesc_sw128(b0 + k * 2048, 8192, 1024) : sdesc_sw128(b0 + k * 32, 16, 1024);
          umma_bf16_ss(tmem_d, adesc, bdesc, idesc, (it > 0 || k > 0) ? 1u : 0u);
        }
        umma_commit(&empty[s]);
      }
      umma_commit(accum_full);  // also on abort, so the MMAs already issued can be waited for
    }
  } else {
    // ------------------------------------------------------------------ dequantizers (warps 2..9)
    if constexpr (C::kDeq) {
      // Two groups of 4 warps take alternate main stages; a thread expands one 64-element block row:
      //   A_DEQ_K : thread = W row n of the stage (128 rows x 64 k), K-major tile,
      //   A_DEQ_MN: thread = (W row n of the stage, half h of the 128-wide k range), MN-major tile;
      //             rows map so that the 8 lanes of a store phase hit 8 distinct 16-byte bank groups.
      const int t = threadIdx.x - 64;  // 0..255
      const int grp = t >> 7;
      const int tg = t & 127;
      const int row = (AM == A_DEQ_K) ? tg : ((tg & 7) + 8 * (tg >> 4));
      const int h = (AM == A_DEQ_K) ? 0 : ((tg >> 3) & 1);
      const int c_off = (AM == A_DEQ_K) ? row * 32 : (row * 64 + h * 32);
      const int a_off = (AM == A_DEQ_K) ? row * 128 : (h * 8192 + row * 128);

      auto scale_of = [&](int it) -> float {
        const int kk0 = (main_begin + it - n_extra) * 64;
        const int n = (AM == A_DEQ_K) ? (i0 + row) : (kk0 + row);
        const int k = (AM == A_DEQ_K) ? kk0 : (i0 + 64 * h);
        if (n < args.w_rows && k < args.w_cols) return __ldg(args.absmax + static_cast<long long>(n) * args.w_kb + (k >> 6));
        return 0.0f;
      };

      const int first = n_extra + grp;
      float sc_next = (first < n_total) ? scale_of(first) : 0.0f;
      uint32_t codes_phase = 0;  // bit s: parity of the next full_codes[s] phase this group waits for
      for (int it = first; it < n_total; it += 2) {
        const int s = it % ST;
        const float sc = sc_next;
        if (it + 2 < n_total) sc_next = scale_of(it + 2);
        const Nf4RegTable tab = nf4_reg_table(sc);
        if (!mbar_wait(&full_codes[s], (codes_phase >> s) & 1u, abort_flag, args.err)) break;
        codes_phase ^= 1u << s;
        const uint4 c01 = *reinterpret_cast<const uint4*>(sC + s * C::kCBytes + c_off);
        const uint4 c23 = *reinterpret_cast<const uint4*>(sC + s * C::kCBytes + c_off + 16);
        const uint32_t words[8] = {c01.x, c01.y, c01.z, c01.w, c23.x, c23.y, c23.z, c23.w};
        uint8_t* a_row = sA + s * C::kABytes + a_off;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          uint32_t o[4];
          nf4_lookup8(tab, words[w], o);
          *reinterpret_cast<uint4*>(a_row + ((w ^ (row & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&full_deq[s]);
      }
    }
    // ------------------------------------------------------------------ epilogue (warps 2..5)
    if (warp < 6) {
      const int qw = warp & 3;
      const int i = i0 + qw * 32 + lane;
      int ok = mbar_wait(accum_full, 0, abort_flag, args.err) ? 1 : 0;
      tc_fence_after();
      ok = __shfl_sync(0xffffffffu, ok && !*abort_flag, 0);
      if (ok) {
        const long long base = static_cast<long long>(z) * args.split_stride + static_cast<long long>(i) * args.ls;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 16) {
          uint32_t r[16];
          tmem_ld_32x32b_x16(tmem_d + (static_cast<uint32_t>(qw * 32) << 16) + static_cast<uint32_t>(c0), r);
          tmem_ld_wait();
          if (i < args.rows_lim) {
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
              const int j = j0 + c0 + jj;
              if (j < args.cols_lim) {
                const float v = n_total > 0 ? args.alpha * __uint_as_float(r[jj]) : 0.0f;
                const long long off = base + static_cast<long long>(j) * args.cs;
                if (args.out_bf16)
                  reinterpret_cast<__nv_bfloat16*>(args.out)[off] = __float2bfloat16_rn(v);
                else
                  reinterpret_cast<float*>(args.out)[off] = v;
              }
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_d, C::kTmemCols);
  }
}

}  // namespace qlora

// tcgen05 GEMM kernel for the QLoRA layer (sm_100a), persistent over work units.
//
// A work unit is a 128 x BN fp32 tile of D[i, j] = sum_kk Aop[i, kk] * Bop[j, kk] accumulated in TMEM over
// one split of the contraction (64-element stages), optionally preceded by "extra" stages that append the
// rank-r LoRA columns to the contraction ([x | s u] . [deq(W) | B]^T in the forward, [dY | v] . [deq(W); A]
// in the backward), so base and LoRA products land in one accumulator.  Each CTA walks units
// blockIdx.x, blockIdx.x + gridDim.x, ...; its shared-memory stage ring runs on across units, and the two
// TMEM accumulators alternate between units so the epilogue of one overlaps the mainloop of the next.
//
// The weight is always the 128-row (M-side) operand: the kernel computes the transposed product
// (y^T = deq(W) x^T, dX^T = deq(W)^T dY^T), so one dequantized weight element feeds BN tokens.
//
// Operand A, per stage (128 rows x 64 contraction elements, bf16, 128-byte swizzled canonical layout):
//   A_TMA_K / A_TMA_MN   loaded by TMA from a bf16 matrix (K-major or MN-major),
//   A_DEQ_K              dequantized from NF4 codes by the dequantizer warps (forward: rows = W rows n),
//   A_DEQ_MN             dequantized the same way into the MN-major layout (backward: rows = W columns k,
//                        contraction over W rows n) -- the transpose of deq(W) costs nothing extra.
//   A_DEQ_TMEM           forward: dequantized rows go from registers straight into tensor memory
//                        (tcgen05.st) and the MMA reads A there, so A never touches shared memory; the
//                        LoRA rows of B for the extra stages are copied the same way from global memory.
//                        Codes are expanded through a lane-replicated table of bf16 level pairs and one
//                        bf16x2 multiply by the block scale (about two instructions per element).
//   The codes arrive by TMA and the stage's absmax values by cp.async, both on the stage's codes barrier.
// Operand B (BN x 64): always by TMA (K-major or MN-major).
//
// Warp roles: warp 0 = producer (lane 0 issues TMA; all lanes copy absmax), warp 1 = TMEM allocator + MMA
// issuer (one thread), warps 2..5 = epilogue (TMEM -> registers -> global), warps 6..13 = dequantizers
// (A_DEQ_* only; two groups of 4 warps, group g takes the stages of even/odd global index).
//
// Shared-memory tiles: for the 128B swizzle every tile starts on a 1024-byte boundary; row r of a tile is
// 128 bytes at r*128 and its 16-byte chunk c sits at chunk position c ^ (r & 7).  TMA writes that layout;
// the dequantizers write it with plain 16-byte stores followed by fence.proxy.async.
#pragma once

#include <cuda_bf16.h>

#include "nf4_table.cuh"
#include "ptx.cuh"

namespace qlora {

enum AMode : int { A_TMA_K = 0, A_TMA_MN = 1, A_DEQ_K = 2, A_DEQ_MN = 3, A_DEQ_TMEM = 4 };

struct UmmaArgs {
  int rows, cols;         // D extent: i in [0, rows), j in [0, cols)
  int tiles_i, tiles_j;   // ceil(rows / 128), ceil(cols / BN)
  int splits;             // contraction splits; units = splits * tiles_i * tiles_j
  int k_stages;           // main contraction stages (64 elements each) in total
  int stages_per_split;   // main stages per split
  int n_extra;            // extra (LoRA) stages, run by split 0 only, before its main stages
  // dequantization (A_DEQ_*): W is [w_rows, w_cols] with absmax [w_rows, w_cols / 64]
  const float* absmax;
  int w_rows, w_cols, w_kb;
  // A_DEQ_TMEM extra stages: rows of the LoRA matrix appended to A ([w_rows, lora_cols], row stride lora_ld)
  const uint16_t* lora;
  int lora_ld, lora_cols;
  // epilogue: out[z * split_stride + i * ls + j * cs] = alpha * D[i, j] for i < rows_lim, j < cols_lim
  void* out;
  int out_bf16;
  float alpha;
  long long ls, cs, split_stride;
  int rows_lim, cols_lim;
  unsigned int* err;
};


struct Unit {
  int i0, j0, z;
  int main_begin, n_main, n_extra, n_total;
};

// Unit u -> (split z, tile row ti, tile column tj), tj fastest: neighbouring units share the weight tile.
__device__ __forceinline__ Unit unit_of(const UmmaArgs& a, int u, int BN) {
  Unit U;
  const int tj = u % a.tiles_j;
  const int t = u / a.tiles_j;
  const int ti = t % a.tiles_i;
  U.z = t / a.tiles_i;
  U.i0 = ti * 128;
  U.j0 = tj * BN;
  U.main_begin = U.z * a.stages_per_split;
  int end = U.main_begin + a.stages_per_split;
  if (end > a.k_stages) end = a.k_stages;
  U.n_main = end > U.main_begin ? end - U.main_begin : 0;
  U.n_extra = (U.z == 0) ? a.n_extra : 0;
  U.n_total = U.n_extra + U.n_main;
  return U;
}

template <int BN, int AM, bool B_MN>
struct UmmaCfg {
  static constexpr bool kATmem = (AM == A_DEQ_TMEM);
  static constexpr bool kDeq = (AM == A_DEQ_K || AM == A_DEQ_MN || kATmem);
  static constexpr bool kAMN = (AM == A_TMA_MN || AM == A_DEQ_MN);
  static constexpr int kABytes = kATmem ? 0 : 128 * 64 * 2;
  static constexpr int kBBytes = BN * 64 * 2;
  static constexpr int kCBytes = kDeq ? 4096 : 0;
  static constexpr int kSBytes = kDeq ? 512 : 0;  // 128 absmax values per stage
  static constexpr int kStageBytes = kABytes + kBBytes + kCBytes + kSBytes;
  // A_DEQ_TMEM looks codes up in a shared-memory table of bf16 level pairs, one copy per lane (32 KB)
  static constexpr int kLutBytes = kATmem ? 256 * 32 * 4 : 0;
  static constexpr int kStagesRaw = ((kATmem ? 222 : 212) * 1024 - kLutBytes) / kStageBytes;
  static constexpr int kStagesCap = kStagesRaw > 8 ? 8 : kStagesRaw;
  // the two dequantizer groups split the stages by index parity; with an even ring every slot keeps one group
  static constexpr int kStages = kDeq ? (kStagesCap & ~1) : kStagesCap;
  static constexpr int kDeqWarpsPerGroup = 4;
  static constexpr int kThreads = 64 + 128 + (kDeq ? 256 : 0);
  static constexpr int kAccCols = BN;  // fp32 accumulator columns per buffer
  static constexpr int kACols = kATmem ? kStages * 32 : 0;  // A stages in TMEM: 64 bf16 = 32 columns each
  static constexpr int kAccBufs = (2 * BN + kACols <= 512) ? 2 : 1;
  static constexpr int kAColBase = kAccBufs * BN;
  static constexpr int kTmemNeed = kAccBufs * BN + kACols;
  static constexpr int kTmemCols = kTmemNeed <= 32 ? 32 : kTmemNeed <= 64 ? 64 : kTmemNeed <= 128 ? 128 : kTmemNeed <= 256 ? 256 : 512;
  static_assert(kTmemNeed <= 512, "tensor memory");
  static constexpr int kBarBytes = 512;
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kLutBytes + kBarBytes;
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N for M=128 is a multiple of 16 in [16, 256]");
  static_assert(!B_MN || BN % 64 == 0, "MN-major B tiles are whole 64-element swizzle atoms");
  static_assert(kStages >= 2, "pipeline needs two stages");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
  static_assert((4 * kStages + 4) * 8 + 8 <= kBarBytes, "barrier area");
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
  constexpr uint32_t kFull = 0xffffffffu;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + ST * C::kABytes;
  uint8_t* sC = sB + ST * C::kBBytes;
  float* sS = reinterpret_cast<float*>(sC + ST * C::kCBytes);
  uint32_t* sLut = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(sS) + ST * C::kSBytes);
  // Barrier phases: full_tma[s] and empty[s] advance once per use of slot s (every stage); full_codes[s]
  // and full_deq[s] once per MAIN-stage use of slot s (the LoRA stages carry no codes); tmem_full[b] and
  // tmem_empty[b] once per unit accumulated in buffer b.  Every waiter visits every phase of the barriers
  // it waits on, so a parity wait never aliases an older phase.
  uint64_t* full_tma = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(sLut) + C::kLutBytes);
  uint64_t* full_codes = full_tma + ST;
  uint64_t* full_deq = full_codes + ST;
  uint64_t* empty = full_deq + ST;
  uint64_t* tmem_full = empty + ST;
  uint64_t* tmem_empty = tmem_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tmem_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_units = args.splits * args.tiles_i * args.tiles_j;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full_tma[s], 1);
      mbar_init(&full_codes[s], 1 + 32);  // the TMA arrive + one cp.async arrive per producer lane
      mbar_init(&full_deq[s], C::kDeqWarpsPerGroup);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tmem_full[b], 1);
      mbar_init(&tmem_empty[b], 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if constexpr (C::kLutBytes > 0) {
    // entry (byte b, lane l) at word 32 b + l: the bf16 pair (level[b >> 4], level[b & 15]) -- a code byte
    // holds element 2j in its high nibble, and the first element goes to the low half
    for (int idx = threadIdx.x; idx < 256 * 32; idx += blockDim.x) {
      const int b = idx >> 5;
      __nv_bfloat162 h = __floats2bfloat162_rn(kNF4LevelsDev[b >> 4], kNF4LevelsDev[b & 15]);
      sLut[idx] = *reinterpret_cast<uint32_t*>(&h);
    }
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmB);
    if (C::kDeq) tma_prefetch_desc(&tmC);
    if (!C::kDeq || (args.n_extra > 0 && !C::kATmem)) tma_prefetch_desc(&tmA);
    if (args.n_extra > 0) tma_prefetch_desc(&tmBx);
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
    uint32_t armed_tma = 0, armed_codes = 0;  // bit s: slot s has an armed phase whose copies may be in flight
    uint32_t tma_par = 0, codes_par = 0;      // bit s: parity of that armed phase
    int g = 0;
    bool stop = false;
    for (int u = blockIdx.x; u < num_units && !stop; u += gridDim.x) {
      const Unit U = unit_of(args, u, BN);
      for (int it = 0; it < U.n_total; ++it, ++g) {
        const int s = g % ST;
        const uint32_t round = static_cast<uint32_t>(g / ST);
        const bool ok = mbar_wait(&empty[s], (round & 1u) ^ 1u, abort_flag, args.err);
        if (!__all_sync(kFull, ok)) {
          stop = true;
          break;
        }
        uint8_t* a_dst = sA + s * C::kABytes;
        uint8_t* b_dst = sB + s * C::kBBytes;
        if (lane == 0) {
          armed_tma |= 1u << s;
          tma_par = (tma_par & ~(1u << s)) | ((round & 1u) << s);
        }
        if (it < U.n_extra && C::kATmem) {
          // LoRA stage of the TMEM forward: B extra by TMA; the dequantizers copy A's LoRA rows themselves,
          // so the codes barrier only counts its 33 arrivals (no bytes)
          if (lane == 0) {
            mbar_arrive_expect_tx(&full_tma[s], C::kBBytes);
            tma_load_2d(b_dst, &tmBx, 64 * it, U.j0, &full_tma[s]);
            const uint32_t cpar = ((codes_par >> s) & 1u) ^ ((armed_codes >> s) & 1u);
            armed_codes |= 1u << s;
            codes_par = (codes_par & ~(1u << s)) | (cpar << s);
            mbar_arrive(&full_codes[s]);
          }
          mbar_arrive(&full_codes[s]);
        } else if (it < U.n_extra) {
          if (lane == 0) {
            const int e = it;
            mbar_arrive_expect_tx(&full_tma[s], C::kABytes + C::kBBytes);
            if (C::kAMN) {
              tma_load_2d(a_dst, &tmA, U.i0, 64 * e, &full_tma[s]);
              tma_load_2d(a_dst + 8192, &tmA, U.i0 + 64, 64 * e, &full_tma[s]);
            } else {
              tma_load_2d(a_dst, &tmA, 64 * e, U.i0, &full_tma[s]);
            }
            tma_load_2d(b_dst, &tmBx, 64 * e, U.j0, &full_tma[s]);
          }
        } else {
          const int kk0 = (U.main_begin + it - U.n_extra) * 64;
          if (lane == 0) {
            mbar_arrive_expect_tx(&full_tma[s], C::kBBytes + (C::kDeq ? 0 : C::kABytes));
            if (B_MN) {
#pragma unroll
              for (int c = 0; c < BN / 64; ++c) tma_load_2d(b_dst + c * 8192, &tmB, U.j0 + 64 * c, kk0, &full_tma[s]);
            } else {
              tma_load_2d(b_dst, &tmB, kk0, U.j0, &full_tma[s]);
            }
          }
          if constexpr (C::kDeq) {
            // codes by TMA and the stage's 128 absmax values by cp.async, all on full_codes[s]; waiting on
            // empty[s] above made this slot's A tile, codes and scales free to overwrite
            if (lane == 0) {
              const uint32_t cpar = ((codes_par >> s) & 1u) ^ ((armed_codes >> s) & 1u);
              armed_codes |= 1u << s;
              codes_par = (codes_par & ~(1u << s)) | (cpar << s);
              mbar_arrive_expect_tx(&full_codes[s], C::kCBytes);
              if constexpr (AM == A_DEQ_K || AM == A_DEQ_TMEM)
                tma_load_2d(sC + s * C::kCBytes, &tmC, kk0 / 2, U.i0, &full_codes[s]);
              else
                tma_load_2d(sC + s * C::kCBytes, &tmC, U.i0 / 2, kk0, &full_codes[s]);
            }
            float* sdst = sS + s * 128;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int idx = lane + 32 * q;
              int n, k;
              if (AM != A_DEQ_MN) {  // value for tile row idx (W row i0 + idx) in k-block kk0 / 64
                n = U.i0 + idx;
                k = kk0;
              } else {              // value for W row kk0 + idx / 2 in k-block (i0 + 64 (idx & 1)) / 64
                n = kk0 + (idx >> 1);
                k = U.i0 + 64 * (idx & 1);
              }
              const bool valid = n < args.w_rows && k < args.w_cols;
              const float* src = valid ? args.absmax + static_cast<long long>(n) * args.w_kb + (k >> 6) : args.absmax;
              cp_async_4_zfill(sdst + idx, src, valid);
            }
            cp_async_mbar_arrive_noinc(&full_codes[s]);
          } else {
            if (lane == 0) {
              if constexpr (AM == A_TMA_MN) {
                tma_load_2d(a_dst, &tmA, U.i0, kk0, &full_tma[s]);
                tma_load_2d(a_dst + 8192, &tmA, U.i0 + 64, kk0, &full_tma[s]);
              } else {
                tma_load_2d(a_dst, &tmA, kk0, U.i0, &full_tma[s]);
              }
            }
          }
        }
      }
    }
    if (lane == 0 && *abort_flag) {
      // copies still in flight must land before the CTA's shared memory is released: wait for the last
      // armed phase of every slot (already complete ones return at once)
      for (int s = 0; s < ST; ++s) {
        if ((armed_tma >> s) & 1u) mbar_wait_drain(&full_tma[s], (tma_par >> s) & 1u, args.err);
        if ((armed_codes >> s) & 1u) mbar_wait_drain(&full_codes[s], (codes_par >> s) & 1u, args.err);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, BN, C::kAMN, B_MN);
      // full_deq[s] phases count the main-stage uses of slot s: bit s = parity of the next one
      uint32_t deq_phase = 0;
      int g = 0, lu = 0;
      bool stop = false;
      for (int u = blockIdx.x; u < num_units && !stop; u += gridDim.x, ++lu) {
        const Unit U = unit_of(args, u, BN);
        const int acc = lu % C::kAccBufs;
        if (!mbar_wait(&tmem_empty[acc], (static_cast<uint32_t>(lu / C::kAccBufs) & 1u) ^ 1u, abort_flag, args.err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::kAccCols);
        for (int it = 0; it < U.n_total; ++it, ++g) {
          const int s = g % ST;
          const uint32_t par = static_cast<uint32_t>(g / ST) & 1u;
          if (!mbar_wait(&full_tma[s], par, abort_flag, args.err)) {
            stop = true;
            break;
          }
          if (C::kDeq && (C::kATmem || it >= U.n_extra)) {
            if (!mbar_wait(&full_deq[s], (deq_phase >> s) & 1u, abort_flag, args.err)) {
              stop = true;
              break;
            }
            deq_phase ^= 1u << s;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * C::kABytes);
          const uint32_t b0 = smem_u32(sB + s * C::kBBytes);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t bdesc = B_MN ? sdesc_sw128(b0 + k * 2048, 8192, 1024) : sdesc_sw128(b0 + k * 32, 16, 1024);
            if constexpr (C::kATmem) {
              const uint32_t a_tmem = tmem_base + static_cast<uint32_t>(C::kAColBase + s * 32 + k * 8);
              umma_bf16_ts(d_tmem, a_tmem, bdesc, idesc, (it > 0 || k > 0) ? 1u : 0u);
            } else {
              const uint64_t adesc =
                  C::kAMN ? sdesc_sw128(a0 + k * 2048, 8192, 1024) : sdesc_sw128(a0 + k * 32, 16, 1024);
              umma_bf16_ss(d_tmem, adesc, bdesc, idesc, (it > 0 || k > 0) ? 1u : 0u);
            }
          }
          umma_commit(&empty[s]);
        }
        umma_commit(&tmem_full[acc]);  // also on abort, so the MMAs already issued can be waited for
      }
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------------ epilogue (warps 2..5)
    const int qw = warp & 3;  // TMEM lane quarter this warp may access
    int lu = 0;
    for (int u = blockIdx.x; u < num_units; u += gridDim.x, ++lu) {
      const Unit U = unit_of(args, u, BN);
      const int acc = lu % C::kAccBufs;
      int ok = mbar_wait(&tmem_full[acc], static_cast<uint32_t>(lu / C::kAccBufs) & 1u, abort_flag, args.err) ? 1 : 0;
      tc_fence_after();
      ok = __shfl_sync(kFull, ok && !*abort_flag, 0);
      if (!ok) break;
      const int i = U.i0 + qw * 32 + lane;
      const long long base = static_cast<long long>(U.z) * args.split_stride + static_cast<long long>(i) * args.ls;
      const uint32_t t_acc = tmem_base + (static_cast<uint32_t>(qw * 32) << 16) + static_cast<uint32_t>(acc * C::kAccCols);
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 16) {
        uint32_t r[16];
        tmem_ld_32x32b_x16(t_acc + static_cast<uint32_t>(c0), r);
        tmem_ld_wait();
        if (i < args.rows_lim) {
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            const int j = U.j0 + c0 + jj;
            if (j < args.cols_lim) {
              const float v = U.n_total > 0 ? args.alpha * __uint_as_float(r[jj]) : 0.0f;
              const long long off = base + static_cast<long long>(j) * args.cs;
              if (args.out_bf16)
                reinterpret_cast<__nv_bfloat16*>(args.out)[off] = __float2bfloat16_rn(v);
              else
                reinterpret_cast<float*>(args.out)[off] = v;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tmem_empty[acc]);
    }
  } else {
    // ------------------------------------------------------------------ dequantizers (warps 6..13)
    if constexpr (C::kATmem) {
      // A thread owns TMEM lane 32 * (warp % 4) + lane = tile row i (W row i0 + i) and, per stage of its
      // group, writes that row's 64 bf16 (32 columns) into the stage's A columns of tensor memory.
      const int grp = (warp - 6) >> 2;
      const int row = 32 * (warp & 3) + lane;
      const uint32_t t_lane = static_cast<uint32_t>(32 * (warp & 3)) << 16;
      const uint8_t* lut_lane = reinterpret_cast<const uint8_t*>(sLut) + lane * 4;
      uint32_t codes_phase = 0;  // bit s: parity of the next full_codes[s] phase (every stage of slot s)
      int g = 0;
      bool stop = false;
      for (int u = blockIdx.x; u < num_units && !stop; u += gridDim.x) {
        const Unit U = unit_of(args, u, BN);
        for (int it = 0; it < U.n_total; ++it, ++g) {
          if ((g & 1) != grp) continue;
          const int s = g % ST;
          if (!mbar_wait(&full_codes[s], (codes_phase >> s) & 1u, abort_flag, args.err)) {
            stop = true;
            break;
          }
          codes_phase ^= 1u << s;
          tc_fence_after();  // the MMAs that read this slot's A columns have completed (empty -> producer)
          uint32_t r[32];
          if (it < U.n_extra) {
            const int n = U.i0 + row;
            const int c0 = 64 * it;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              uint4 v = make_uint4(0, 0, 0, 0);
              if (n < args.w_rows && c0 + 8 * c < args.lora_cols)
                v = __ldg(reinterpret_cast<const uint4*>(args.lora + static_cast<long long>(n) * args.lora_ld + c0 + 8 * c));
              r[4 * c] = v.x;
              r[4 * c + 1] = v.y;
              r[4 * c + 2] = v.z;
              r[4 * c + 3] = v.w;
            }
          } else {
            // level pair from this lane's copy of the table, times the block scale in bf16x2
            const __nv_bfloat162 sc2 = __float2bfloat162_rn(sS[s * 128 + row]);
            const uint4 c01 = *reinterpret_cast<const uint4*>(sC + s * C::kCBytes + row * 32);
            const uint4 c23 = *reinterpret_cast<const uint4*>(sC + s * C::kCBytes + row * 32 + 16);
            const uint32_t words[8] = {c01.x, c01.y, c01.z, c01.w, c23.x, c23.y, c23.z, c23.w};
#pragma unroll
            for (int w = 0; w < 8; ++w) {
              const uint32_t q = words[w];
              const uint32_t offs[4] = {(q << 7) & 0x7F80u, (q >> 1) & 0x7F80u, (q >> 9) & 0x7F80u, (q >> 17) & 0x7F80u};
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                uint32_t v = *reinterpret_cast<const uint32_t*>(lut_lane + offs[j]);
                __nv_bfloat162 p = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&v), sc2);
                r[4 * w + j] = *reinterpret_cast<uint32_t*>(&p);
              }
            }
          }
          tmem_st_32x32b_x32(tmem_base + t_lane + static_cast<uint32_t>(C::kAColBase + s * 32), r);
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&full_deq[s]);
        }
      }
    } else if constexpr (C::kDeq) {
      // A thread expands one 64-element block row per stage:
      //   A_DEQ_K : thread = W row n of the stage (128 rows x 64 k), K-major tile,
      //   A_DEQ_MN: thread = (W row n of the stage, half h of the 128-wide k range), MN-major tile;
      //             rows map so that the 8 lanes of a store phase hit 8 distinct 16-byte bank groups.
      const int t = threadIdx.x - 192;  // 0..255
      const int grp = t >> 7;
      const int tg = t & 127;
      const int row = (AM == A_DEQ_K) ? tg : ((tg & 7) + 8 * (tg >> 4));
      const int h = (AM == A_DEQ_K) ? 0 : ((tg >> 3) & 1);
      const int c_off = (AM == A_DEQ_K) ? row * 32 : (row * 64 + h * 32);
      const int a_off = (AM == A_DEQ_K) ? row * 128 : (h * 8192 + row * 128);
      const int s_idx = (AM == A_DEQ_K) ? row : (row * 2 + h);
      uint32_t codes_phase = 0;  // bit s: parity of the next full_codes[s] phase (this group owns slot s)
      int g = 0;
      bool stop = false;
      for (int u = blockIdx.x; u < num_units && !stop; u += gridDim.x) {
        const Unit U = unit_of(args, u, BN);
        for (int it = 0; it < U.n_total; ++it, ++g) {
          if (it < U.n_extra || (g & 1) != grp) continue;
          const int s = g % ST;
          if (!mbar_wait(&full_codes[s], (codes_phase >> s) & 1u, abort_flag, args.err)) {
            stop = true;
            break;
          }
          codes_phase ^= 1u << s;
          const Nf4RegTable tab = nf4_reg_table(sS[s * 128 + s_idx]);
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

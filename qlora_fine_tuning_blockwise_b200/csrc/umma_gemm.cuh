// tcgen05 GEMM kernel for the QLoRA layer (sm_100a), persistent over work units.
//
// A work unit is a 128 x BN fp32 tile of D[i, j] = sum_kk Aop[i, kk] * Bop[j, kk] accumulated in TMEM over
// one split of the contraction (stages of KB blocks of 64 elements), optionally preceded by "extra" stages
// that append the
// rank-r LoRA columns to the contraction ([x | s u] . [deq(W) | B]^T in the forward, [dY | v] . [deq(W); A]
// in the backward), so base and LoRA products land in one accumulator.  Each CTA walks units
// blockIdx.x, blockIdx.x + gridDim.x, ...; its rings run on across units, and where tensor memory allows
// two accumulators alternate between units so the epilogue of one overlaps the mainloop of the next.
//
// The weight is always the 128-row (M-side) operand: the kernel computes the transposed product
// (y^T = deq(W) x^T, dX^T = deq(W)^T dY^T), so one dequantized weight element feeds BN tokens.
//
// Operand A, per 64-element block (128 rows x 64 contraction elements, bf16):
//   A_TMA_K / A_TMA_MN   loaded by TMA from a bf16 matrix (K-major or MN-major) together with B,
//   A_DEQ_MN             backward: dequantized from NF4 codes into the MN-major 128B-swizzled shared-memory
//                        layout (rows = W columns k, contraction over W rows n) -- the transpose of deq(W)
//                        costs nothing extra; the LoRA stages copy rows of A the same way,
//   A_DEQ_TMEM           forward: dequantized rows go from registers straight into tensor memory
//                        (tcgen05.st) and the MMA reads A there, so A never touches shared memory; the
//                        LoRA stages copy rows of B the same way.
// The dequantizers expand a code byte (two elements) through a lane-replicated shared table of bf16 level
// pairs and multiply by the block scale in bf16x2.
// Operand B (BN x 64 per block): always by TMA.
//
// Three rings decouple the latencies of the dequantizing kernels:
//   Q ring (deep):  packed codes (TMA) + the stage's absmax values (one cp.async per row, or one TMA box in
//                   4-block stages), filled by the Q producer as far ahead as its depth allows, emptied as
//                   soon as a dequantizer has the stage in registers -- so HBM latency overlaps many stages;
//   A ring:         dequantized A tiles (TMEM columns or shared memory), filled by the dequantizers,
//                   emptied by the MMAs (tcgen05.commit);
//   B ring:         B tiles (and A tiles in the TMA modes), filled by the B producer, emptied by the MMAs.
// The MMA waits on both the A ring (dequantized tile ready) and the B ring (B tile landed) of each stage.
//
// Warp roles: warp 0 = B producer (lane 0 issues TMA), warp 1 = TMEM allocator + MMA issuer, warps 2..5 =
// epilogue (TMEM -> registers -> global), warps 6 .. 6 + 4G - 1 = dequantizers (G groups of 4 warps; group
// g % G takes stage g), warp 6 + 4G = Q producer (lane 0 issues the codes TMA, all lanes copy absmax).  The
// dequantizer and Q-producer warps exist in the dequantizing modes only.
//
// Shared-memory tiles: for the 128B swizzle every tile starts on a 1024-byte boundary; row r of a tile is
// 128 bytes at r*128 and its 16-byte chunk c sits at chunk position c ^ (r & 7).  TMA writes that layout;
// the dequantizers write it with plain 16-byte stores.  Slots change hands between the generic proxy
// (thread loads and stores) and the async proxy (TMA, MMA), so each handoff carries a fence.proxy.async:
// before a codes slot is released for a TMA refill, and before an A slot the MMAs read is overwritten.
//
// Every wait is bounded; on expiry the waiting thread raises the CTA's abort flag and the device error word,
// every role leaves its loop, and the producers wait (bounded) for their copies in flight before the CTA
// releases its shared and tensor memory.
#pragma once

#include <cuda_bf16.h>

#include "nf4_table.cuh"
#include "ptx.cuh"

namespace qlora {

enum AMode : int { A_TMA_K = 0, A_TMA_MN = 1, A_DEQ_MN = 3, A_DEQ_TMEM = 4 };

struct UmmaArgs {
  int rows, cols;         // D extent: i in [0, rows), j in [0, cols)
  int tiles_i, tiles_j;   // ceil(rows / 128), ceil(cols / BN)
  int splits;             // contraction splits; units = splits * tiles_i * tiles_j
  int k_stages;           // main contraction stages (64 KB elements each) in total
  int stages_per_split;   // main stages per split
  int n_extra;            // extra (LoRA) stages, run by split 0 only, before its main stages
  // dequantization (A_DEQ_*): W is [w_rows, w_cols] with absmax [w_rows, w_cols / 64]
  const float* absmax;
  int w_rows, w_cols, w_kb;
  // LoRA matrix copied into the extra stages of A, row stride lora_ld, lora_r valid contraction entries:
  //   A_DEQ_TMEM: B [w_rows, lora_r] (tile row i = W row i0 + i, contraction along the row),
  //   A_DEQ_MN  : A [lora_r, w_cols] (contraction index = row of A, tile row i = column i0 + i).
  const uint16_t* lora;
  int lora_ld, lora_r;
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

// KB = NF4 blocks (64 contraction elements each) per pipeline stage.  Every stage costs each role a few
// barrier round trips of fixed latency, so token-light layers -- whose MMAs are short -- run 4 blocks a stage
// (A_DEQ_TMEM only): codes then arrive as one 128B-swizzled TMA box of 128 rows x 128 bytes and the absmax
// values as one TMA box of 128 rows x 4 floats.
template <int BN, int AM, bool B_MN, int KB = 1>
struct UmmaCfg {
  static constexpr bool kATmem = (AM == A_DEQ_TMEM);
  static constexpr bool kDeq = (AM == A_DEQ_MN || kATmem);
  static constexpr bool kAMN = (AM == A_TMA_MN || AM == A_DEQ_MN);
  static constexpr bool kAbsTma = (KB == 4);  // absmax by TMA (else one cp.async per row)
  static constexpr int kTileA = 128 * 64 * 2;  // one bf16 A block in shared memory
  static constexpr int kBBytes = BN * 64 * 2 * KB;
  static constexpr int kBSlot = kBBytes + (kDeq ? 0 : kTileA);  // the TMA modes load A beside B
  static constexpr int kASlot = (AM == A_DEQ_MN) ? kTileA : 0;   // A ring in shared memory
  static constexpr int kCBytes = 4096 * KB;                       // 128 rows x 64 KB codes
  static constexpr int kSBytes = 512 * KB;                        // 128 rows x KB absmax values
  static constexpr int kQSlot = kDeq ? kCBytes + kSBytes : 0;
  // the dequantizers look codes up in a shared-memory table of bf16 level pairs, one copy per lane (32 KB)
  static constexpr int kLutBytes = kDeq ? 256 * 32 * 4 : 0;
  static constexpr int kBarBytes = 1024;
  static constexpr int kBudget = 226 * 1024 - 1024 - kLutBytes - kBarBytes;

  // tensor memory: accumulators (BN fp32 columns each), then the A ring of the TMEM mode (32 columns a stage)
  static constexpr int kAccBufs = (!kATmem || 2 * BN + 4 * 32 <= 512) ? 2 : 1;
  static constexpr int kAccCols = BN;
  static constexpr int kAColBase = kAccBufs * BN;
  static constexpr int kAColsStage = 32 * KB;
  static constexpr int kAStagesTmem = (512 - kAColBase) / kAColsStage > 8 ? 8 : (512 - kAColBase) / kAColsStage;

  // ring depths: deep B rings when B tiles are small (token-light layers), 4 stages of 16-32 KB otherwise;
  // the A ring as deep as tensor memory (or shared memory, for A_DEQ_MN) allows.
  static constexpr int kBStagesWant = kDeq ? (BN <= 64 ? 8 : (AM == A_DEQ_MN && BN >= 256 ? 3 : 4)) : 8;
  static constexpr int kAStagesWant = kATmem ? kAStagesTmem : (AM == A_DEQ_MN ? (BN >= 256 ? 3 : 4) : 0);
  static constexpr int kQWant = KB == 4 ? 6 : (BN >= 128 ? 10 : 16);
  static constexpr int kBFit = (kBudget - kAStagesWant * kASlot - (kDeq ? kQWant * kQSlot : 0)) / kBSlot;
  static constexpr int kBStages = kBFit < kBStagesWant ? (kBFit < 2 ? 2 : kBFit) : kBStagesWant;
  static constexpr int kAStages = kAStagesWant;
  static constexpr int kQFit = kDeq ? (kBudget - kAStages * kASlot - kBStages * kBSlot) / kQSlot : 0;
  static constexpr int kQStages = kQFit > 16 ? 16 : kQFit;

  // Dequantizer groups of 4 warps (one per TMEM lane quarter); group g % kDeqGroups takes stage g.  A warp
  // spends most of a stage waiting on its own instruction latencies, so stage throughput grows with the
  // number of groups in flight, up to the A ring's depth: 4 in the TMEM kernel, 3 in the MN-major one.
  static constexpr int kDeqWarpsPerGroup = 4;
  static constexpr int kDeqGroups = kDeq ? (kAStages < (kATmem ? 4 : 3) ? kAStages : (kATmem ? 4 : 3)) : 0;
  static constexpr int kQWarp = 6 + 4 * kDeqGroups;
  static constexpr int kThreads = kDeq ? 32 * (kQWarp + 1) : 64 + 128;
  static constexpr int kTmemNeed = kAColBase + (kATmem ? kAStages * kAColsStage : 0);
  static constexpr int kTmemCols = kTmemNeed <= 32 ? 32 : kTmemNeed <= 64 ? 64 : kTmemNeed <= 128 ? 128 : kTmemNeed <= 256 ? 256 : 512;
  static constexpr int kSmemBytes =
      1024 + kBStages * kBSlot + kAStages * kASlot + kQStages * kQSlot + kLutBytes + kBarBytes;

  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N for M=128 is a multiple of 16 in [16, 256]");
  static_assert(!B_MN || BN % 64 == 0, "MN-major B tiles are whole 64-element swizzle atoms");
  static_assert(!(kDeq && B_MN), "the dequantizing modes take B K-major");
  static_assert(KB == 1 || (kATmem && KB == 4), "4-block stages exist for the TMEM forward only");
  static_assert(kTmemNeed <= 512, "tensor memory");
  static_assert(kBStages >= 2 && (!kDeq || (kAStages >= 2 && kQStages >= 4)), "ring depths");
  // parity safety (see the kernel): Q ring deeper than the A ring by at least the number of dequantizer
  // groups, and no more groups than A slots
  static_assert(!kDeq || (kQStages >= kAStages + kDeqGroups && kDeqGroups <= kAStages),
                "ring depth relations");
  static_assert(kBStages <= 32 && kAStages <= 32 && kQStages <= 32, "armed-slot bit masks");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
  static_assert((2 * (kBStages + kAStages + kQStages) + 4) * 8 + 8 <= kBarBytes, "barrier area");
};

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

// Slot bookkeeping of a producer: which slots hold an armed phase whose copies may still be in flight, and
// that phase's parity -- on abort the producer waits for exactly those before the CTA exits.
struct Armed {
  uint32_t mask = 0, par = 0;
  __device__ __forceinline__ void set(int s, uint32_t p) {
    mask |= 1u << s;
    par = (par & ~(1u << s)) | (p << s);
  }
  __device__ __forceinline__ void drain(uint64_t* full, int n, unsigned int* err) const {
    for (int s = 0; s < n; ++s)
      if ((mask >> s) & 1u) mbar_wait_drain(&full[s], (par >> s) & 1u, err);
  }
};

// tmA: A for the TMA modes; the absmax matrix [w_rows, w_cols / 64] (fp32) for 4-block TMEM stages.
template <int BN, int AM, bool B_MN, int KB = 1>
__global__ void __launch_bounds__(UmmaCfg<BN, AM, B_MN, KB>::kThreads, 1)
    umma_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmBx, const __grid_constant__ CUtensorMap tmC,
                     const UmmaArgs args) {
  using C = UmmaCfg<BN, AM, B_MN, KB>;
  constexpr int BS = C::kBStages;
  constexpr int AS = C::kAStages;
  constexpr int QS = C::kQStages;
  constexpr uint32_t kFull = 0xffffffffu;

  extern __shared__ uint8_t smem_raw[];
  // align by pointer arithmetic on the shared array itself (not through an integer), so every pointer derived
  // from it stays a known shared-memory pointer and compiles to shared loads and stores
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* sB = smem;                          // B ring (B, then A in the TMA modes), 1024-aligned slots
  uint8_t* sA = sB + BS * C::kBSlot;           // A ring of A_DEQ_MN, 1024-aligned slots
  uint8_t* sQ = sA + AS * C::kASlot;           // Q ring: codes, then absmax
  uint32_t* sLut = reinterpret_cast<uint32_t*>(sQ + QS * C::kQSlot);
  // Phases: b_* advance once per stage (every stage uses the B ring), a_* once per stage in the dequantizing
  // modes, q_* once per MAIN stage, tmem_* once per unit accumulated in that buffer.  Each waiter derives
  // the parity from its running count of the ring's uses, which is sound only while the barrier's previous
  // phase has completed when the wait starts and its next one cannot complete before the waiter releases:
  //   - a barrier cannot run ahead: each refill needs the consumer's release of the slot first;
  //   - a dequantizer at stage g has seen the MMAs of stage g - G - AS complete (its own previous stage's
  //     a_empty wait, G = dequantizer groups), so with G <= AS its a_empty wait for stage g - AS cannot see
  //     an older phase, and with QS >= AS + G the Q stage QS before its own has been consumed;
  //   - the MMA and the producers visit every phase of the barriers they wait on, in order.
  uint64_t* b_full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(sLut) + C::kLutBytes);
  uint64_t* b_empty = b_full + BS;
  uint64_t* a_full = b_empty + BS;
  uint64_t* a_empty = a_full + AS;
  uint64_t* q_full = a_empty + AS;
  uint64_t* q_empty = q_full + QS;
  uint64_t* tmem_full = q_empty + QS;
  uint64_t* tmem_empty = tmem_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tmem_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_units = args.splits * args.tiles_i * args.tiles_j;

  if (threadIdx.x == 0) {
    for (int s = 0; s < BS; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], 1);
    }
    for (int s = 0; s < AS; ++s) {
      mbar_init(&a_full[s], C::kDeqWarpsPerGroup);
      mbar_init(&a_empty[s], 1);
    }
    for (int s = 0; s < QS; ++s) {
      mbar_init(&q_full[s], C::kAbsTma ? 1 : 1 + 32);  // the TMA arrive (+ one cp.async arrive per producer lane)
      mbar_init(&q_empty[s], C::kDeqWarpsPerGroup * 32);  // every lane of the consuming group
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
    if (!C::kDeq) tma_prefetch_desc(&tmA);
    if (args.n_extra > 0) tma_prefetch_desc(&tmBx);
  }
  if (C::kDeq && warp == C::kQWarp && lane == 0) {
    tma_prefetch_desc(&tmC);
    if (C::kAbsTma) tma_prefetch_desc(&tmA);
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
    // ------------------------------------------------------------------ B producer
    Armed armed;
    int g = 0;
    bool stop = false;
    for (int u = blockIdx.x; u < num_units && !stop; u += gridDim.x) {
      const Unit U = unit_of(args, u, BN);
      for (int it = 0; it < U.n_total; ++it, ++g) {
        const int s = g % BS;
        const uint32_t ph = static_cast<uint32_t>(g / BS) & 1u;
        const bool ok = mbar_wait_idle(&b_empty[s], ph ^ 1u, abort_flag, args.err);
        if (!__all_sync(kFull, ok)) {
          stop = true;
          break;
        }
        if (lane == 0) {
          armed.set(s, ph);
          uint8_t* b_dst = sB + s * C::kBSlot;
          if constexpr (C::kDeq) {
            // KB blocks of BN x 64, each a 128B-swizzled K-major sub-tile
            mbar_arrive_expect_tx(&b_full[s], C::kBBytes);
#pragma unroll
            for (int kb = 0; kb < KB; ++kb) {
              if (it < U.n_extra)
                tma_load_2d(b_dst + kb * BN * 128, &tmBx, 64 * (KB * it + kb), U.j0, &b_full[s]);
              else
                tma_load_2d(b_dst + kb * BN * 128, &tmB, ((U.main_begin + it - U.n_extra) * KB + kb) * 64, U.j0,
                            &b_full[s]);
            }
          } else {
            // the TMA modes have no extra stages
            const int kk0 = (U.main_begin + it) * 64;
            uint8_t* a_dst = b_dst + C::kBBytes;
            mbar_arrive_expect_tx(&b_full[s], C::kBBytes + C::kTileA);
            if constexpr (B_MN) {
#pragma unroll
              for (int c = 0; c < BN / 64; ++c) tma_load_2d(b_dst + c * 8192, &tmB, U.j0 + 64 * c, kk0, &b_full[s]);
            } else {
              tma_load_2d(b_dst, &tmB, kk0, U.j0, &b_full[s]);
            }
            if constexpr (AM == A_TMA_MN) {
              tma_load_2d(a_dst, &tmA, U.i0, kk0, &b_full[s]);
              tma_load_2d(a_dst + 8192, &tmA, U.i0 + 64, kk0, &b_full[s]);
            } else {
              tma_load_2d(a_dst, &tmA, kk0, U.i0, &b_full[s]);
            }
          }
        }
      }
    }
    // copies still in flight must land before the CTA's shared memory is released
    if (lane == 0 && *abort_flag) armed.drain(b_full, BS, args.err);
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (whole warp waits,
    // one elected lane issues)
    constexpr uint32_t idesc = idesc_bf16_f32(128, BN, C::kAMN, B_MN);
    int g = 0, lu = 0;
    bool stop = false;
    for (int u = blockIdx.x; u < num_units && !stop; u += gridDim.x, ++lu) {
      const Unit U = unit_of(args, u, BN);
      const int acc = lu % C::kAccBufs;
      const uint32_t eph = (static_cast<uint32_t>(lu / C::kAccBufs) & 1u) ^ 1u;
      if (!__all_sync(kFull, mbar_wait(&tmem_empty[acc], eph, abort_flag, args.err))) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::kAccCols);
      for (int it = 0; it < U.n_total; ++it, ++g) {
        const int bs = g % BS;
        int as = 0;
        bool ok;
        if constexpr (C::kDeq) {
          as = g % AS;
          ok = mbar_wait(&a_full[as], static_cast<uint32_t>(g / AS) & 1u, abort_flag, args.err) &&
               mbar_wait(&b_full[bs], static_cast<uint32_t>(g / BS) & 1u, abort_flag, args.err);
        } else {
          ok = mbar_wait(&b_full[bs], static_cast<uint32_t>(g / BS) & 1u, abort_flag, args.err);
        }
        if (!__all_sync(kFull, ok)) {
          stop = true;
          break;
        }
        tc_fence_after();
        if (elect_one()) {
          const uint32_t b0 = smem_u32(sB + bs * C::kBSlot);
          const uint32_t a0 = C::kDeq ? smem_u32(sA + as * C::kASlot) : b0 + C::kBBytes;
#pragma unroll
          for (int kk = 0; kk < 4 * KB; ++kk) {
            const int kb = kk >> 2, k = kk & 3;
            const uint32_t bk = b0 + static_cast<uint32_t>(kb * BN * 128);
            const uint64_t bdesc = B_MN ? sdesc_sw128(bk + k * 2048, 8192, 1024) : sdesc_sw128(bk + k * 32, 16, 1024);
            const uint32_t accum = (it > 0 || kk > 0) ? 1u : 0u;
            if constexpr (C::kATmem) {
              const uint32_t a_tmem =
                  tmem_base + static_cast<uint32_t>(C::kAColBase + as * C::kAColsStage + kb * 32 + k * 8);
              umma_bf16_ts(d_tmem, a_tmem, bdesc, idesc, accum);
            } else {
              const uint64_t adesc =
                  C::kAMN ? sdesc_sw128(a0 + k * 2048, 8192, 1024) : sdesc_sw128(a0 + k * 32, 16, 1024);
              umma_bf16_ss(d_tmem, adesc, bdesc, idesc, accum);
            }
          }
          umma_commit(&b_empty[bs]);
          if constexpr (C::kDeq) umma_commit(&a_empty[as]);
        }
        __syncwarp();
      }
      if (elect_one()) umma_commit(&tmem_full[acc]);  // also on abort, so the MMAs issued can be waited for
      __syncwarp();
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------------ epilogue (warps 2..5)
    const int qw = warp & 3;  // TMEM lane quarter this warp may access
    int lu = 0;
    for (int u = blockIdx.x; u < num_units; u += gridDim.x, ++lu) {
      const Unit U = unit_of(args, u, BN);
      const int acc = lu % C::kAccBufs;
      int ok = mbar_wait_idle(&tmem_full[acc], static_cast<uint32_t>(lu / C::kAccBufs) & 1u, abort_flag, args.err) ? 1 : 0;
      tc_fence_after();
      ok = __shfl_sync(kFull, ok && !*abort_flag, 0);
      if (!ok) break;
      const int i = U.i0 + qw * 32 + lane;
      const long long base = static_cast<long long>(U.z) * args.split_stride + static_cast<long long>(i) * args.ls;
      const uint32_t t_acc = tmem_base + (static_cast<uint32_t>(qw * 32) << 16) + static_cast<uint32_t>(acc * C::kAccCols);
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 16) {
        uint32_t r[16];
        __syncwarp();  // tcgen05.ld is warp-aligned: reconverge after the guarded stores
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
  } else if (warp == C::kQWarp) {
    // ------------------------------------------------------------------ Q producer (dequantizing modes)
    if constexpr (C::kDeq) {
      Armed armed;
      int q = 0;
      bool stop = false;
      for (int u = blockIdx.x; u < num_units && !stop; u += gridDim.x) {
        const Unit U = unit_of(args, u, BN);
        for (int it = U.n_extra; it < U.n_total; ++it, ++q) {
          const int s = q % QS;
          const uint32_t ph = static_cast<uint32_t>(q / QS) & 1u;
          const bool ok = mbar_wait_idle(&q_empty[s], ph ^ 1u, abort_flag, args.err);
          if (!__all_sync(kFull, ok)) {
            stop = true;
            break;
          }
          const int kk0 = (U.main_begin + it - U.n_extra) * 64 * KB;
          uint8_t* q_dst = sQ + s * C::kQSlot;
          if (lane == 0) {
            armed.set(s, ph);
            if constexpr (C::kAbsTma) {
              // 128 W rows x 128 bytes of codes (swizzled) and 128 rows x 4 absmax values
              mbar_arrive_expect_tx(&q_full[s], C::kCBytes + C::kSBytes);
              tma_load_2d(q_dst, &tmC, kk0 / 2, U.i0, &q_full[s]);
              tma_load_2d(q_dst + C::kCBytes, &tmA, kk0 / 64, U.i0, &q_full[s]);
            } else {
              mbar_arrive_expect_tx(&q_full[s], C::kCBytes);
              if constexpr (AM == A_DEQ_TMEM)
                tma_load_2d(q_dst, &tmC, kk0 / 2, U.i0, &q_full[s]);  // 128 W rows x 32 bytes
              else
                tma_load_2d(q_dst, &tmC, U.i0 / 2, kk0, &q_full[s]);  // 64 W rows x 64 bytes
            }
          }
          if constexpr (C::kAbsTma) continue;
          float* sdst = reinterpret_cast<float*>(q_dst + C::kCBytes);
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            const int idx = lane + 32 * qq;
            int n, k;
            if constexpr (AM == A_DEQ_TMEM) {  // value for tile row idx (W row i0 + idx) in k-block kk0 / 64
              n = U.i0 + idx;
              k = kk0;
            } else {                           // value for W row kk0 + idx / 2 in k-block (i0 + 64 (idx & 1)) / 64
              n = kk0 + (idx >> 1);
              k = U.i0 + 64 * (idx & 1);
            }
            const bool valid = n < args.w_rows && k < args.w_cols;
            const float* src = valid ? args.absmax + static_cast<long long>(n) * args.w_kb + (k >> 6) : args.absmax;
            cp_async_4_zfill(sdst + idx, src, valid);
          }
          cp_async_mbar_arrive_noinc(&q_full[s]);
        }
      }
      if (lane == 0 && *abort_flag) armed.drain(q_full, QS, args.err);
    }
  } else {
    // ------------------------------------------------------------------ dequantizers (warps 6 .. 6 + 4G - 1)
    if constexpr (C::kDeq) {
      const int t = threadIdx.x - 192;  // 0 .. 128 kDeqGroups - 1
      const int grp = t >> 7;
      const int tg = t & 127;
      // A_DEQ_TMEM: thread = TMEM lane 32 (warp % 4) + lane = tile row (W row i0 + row), 64 elements a stage.
      // A_DEQ_MN  : thread = (contraction row `row` = W row kk0 + row, half h of the 128-wide k range); rows
      //             map so that the 8 lanes of a store phase hit 8 distinct 16-byte bank groups.
      const int row = C::kATmem ? 32 * (warp & 3) + lane : ((tg & 7) + 8 * (tg >> 4));
      const int h = C::kATmem ? 0 : ((tg >> 3) & 1);
      const int c_off = C::kATmem ? row * 32 : (row * 64 + h * 32);
      const int s_idx = C::kATmem ? row : (row * 2 + h);
      const uint32_t t_lane = static_cast<uint32_t>(32 * (warp & 3)) << 16;
      const uint8_t* lut_lane = reinterpret_cast<const uint8_t*>(sLut) + lane * 4;
      int g = 0, q = 0;
      bool stop = false;
      for (int u = blockIdx.x; u < num_units && !stop; u += gridDim.x) {
        const Unit U = unit_of(args, u, BN);
        for (int it = 0; it < U.n_total; ++it, ++g) {
          const bool extra = it < U.n_extra;
          const int qi = q;
          if (!extra) ++q;
          if (g % C::kDeqGroups != grp) continue;
          // The stage's codes and scales, held in registers: block p of the stage is words[8p .. 8p + 7]
          // (64 codes) with scale sc[p].
          uint32_t words[8 * KB];
          float sc[KB];
          if (!extra) {
            const int qs = qi % QS;
            const bool okq = mbar_wait_idle(&q_full[qs], static_cast<uint32_t>(qi / QS) & 1u, abort_flag, args.err);
            if (!__all_sync(kFull, okq)) {
              stop = true;
              break;
            }
            const uint8_t* q_src = sQ + qs * C::kQSlot;
            if constexpr (C::kAbsTma) {
              // row `row` is 128 bytes; its 16-byte chunk c sits at chunk position c ^ (row & 7)
              const uint8_t* q_row = q_src + row * 128;
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                const uint4 v = *reinterpret_cast<const uint4*>(q_row + ((c ^ (row & 7)) << 4));
                words[4 * c] = v.x;
                words[4 * c + 1] = v.y;
                words[4 * c + 2] = v.z;
                words[4 * c + 3] = v.w;
              }
              const float4 s4 = *reinterpret_cast<const float4*>(q_src + C::kCBytes + row * 16);
              sc[0] = s4.x;
              if constexpr (KB == 4) {
                sc[1] = s4.y;
                sc[2] = s4.z;
                sc[3] = s4.w;
              }
            } else {
              sc[0] = reinterpret_cast<const float*>(q_src + C::kCBytes)[s_idx];
              const uint4 c01 = *reinterpret_cast<const uint4*>(q_src + c_off);
              const uint4 c23 = *reinterpret_cast<const uint4*>(q_src + c_off + 16);
              words[0] = c01.x;
              words[1] = c01.y;
              words[2] = c01.z;
              words[3] = c01.w;
              words[4] = c23.x;
              words[5] = c23.y;
              words[6] = c23.z;
              words[7] = c23.w;
            }
            // the stage is in registers: the slot may refill.  Every lane arrives for itself after a proxy
            // fence, so its own generic reads of the slot are ordered before the refill's TMA (async-proxy)
            // writes
            fence_proxy_async_smem();
            mbar_arrive(&q_empty[qs]);
          }
          // 64 bf16 values (32 registers) of block p: dequantized codes, or the LoRA rows in the extra stages
          auto block_values = [&](int p, uint32_t (&r)[32]) {
            if (extra) {
              // LoRA rows: 64 contraction entries of this thread's tile row (TMEM) or its row/half (MN)
              const uint16_t* src;
              bool valid;
              int c0 = 0;
              if constexpr (C::kATmem) {
                const int n = U.i0 + row;
                c0 = 64 * (KB * it + p);
                valid = n < args.w_rows;
                src = args.lora + static_cast<long long>(n) * args.lora_ld + c0;
              } else {
                const int jr = 64 * it + row;
                valid = jr < args.lora_r && U.i0 + 64 * h < args.w_cols;
                src = args.lora + static_cast<long long>(jr) * args.lora_ld + U.i0 + 64 * h;
              }
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                uint4 v = make_uint4(0, 0, 0, 0);
                if (valid && (!C::kATmem || c0 + 8 * c < args.lora_r))
                  v = __ldg(reinterpret_cast<const uint4*>(src + 8 * c));
                r[4 * c] = v.x;
                r[4 * c + 1] = v.y;
                r[4 * c + 2] = v.z;
                r[4 * c + 3] = v.w;
              }
            } else {
              // level pair from this lane's copy of the table, times the block scale in bf16x2
              const __nv_bfloat162 sc2 = __float2bfloat162_rn(sc[p]);
#pragma unroll
              for (int w = 0; w < 8; ++w) {
                const uint32_t qw8 = words[8 * p + w];
                const uint32_t offs[4] = {(qw8 << 7) & 0x7F80u, (qw8 >> 1) & 0x7F80u, (qw8 >> 9) & 0x7F80u,
                                          (qw8 >> 17) & 0x7F80u};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  uint32_t v = *reinterpret_cast<const uint32_t*>(lut_lane + offs[j]);
                  __nv_bfloat162 pr = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&v), sc2);
                  r[4 * w + j] = *reinterpret_cast<uint32_t*>(&pr);
                }
              }
            }
          };
          uint32_t r[32];
          block_values(0, r);
          // the A slot is free once the MMAs of its previous stage have completed
          const int as = g % AS;
          const bool oka = mbar_wait_idle(&a_empty[as], (static_cast<uint32_t>(g / AS) & 1u) ^ 1u, abort_flag, args.err);
          if (!__all_sync(kFull, oka)) {
            stop = true;
            break;
          }
          tc_fence_after();
          // the MMAs of the slot's previous stage read it through the async proxy; order those reads before
          // this thread's generic writes
          if constexpr (!C::kATmem) fence_proxy_async_smem();
          if constexpr (C::kATmem) {
            const uint32_t a_col = tmem_base + t_lane + static_cast<uint32_t>(C::kAColBase + as * C::kAColsStage);
            tmem_st_32x32b_x32(a_col, r);
#pragma unroll
            for (int p = 1; p < KB; ++p) {
              block_values(p, r);
              tmem_st_32x32b_x32(a_col + static_cast<uint32_t>(32 * p), r);
            }
            tmem_st_wait();
            tc_fence_before();
          } else {
            uint8_t* a_row = sA + as * C::kASlot + h * 8192 + row * 128;
#pragma unroll
            for (int w = 0; w < 8; ++w)
              *reinterpret_cast<uint4*>(a_row + ((w ^ (row & 7)) << 4)) =
                  make_uint4(r[4 * w], r[4 * w + 1], r[4 * w + 2], r[4 * w + 3]);
            fence_proxy_async_smem();
          }
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&a_full[as]);  // the warp's quarter of the A stage is in place
          }
          stop = __shfl_sync(kFull, stop ? 1 : 0, 0) != 0;
          if (stop) break;
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

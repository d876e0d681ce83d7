// tcgen05 GEMM kernel for the QLoRA layer (sm_100a), persistent over work units.
//
// A work unit is a 128 x BN fp32 tile of D[i, j] = sum_kk Aop[i, kk] * Bop[j, kk] accumulated in TMEM over
// one split of the contraction (stages of KB blocks of 64 elements), optionally followed by "extra" stages that
// append the rank-r LoRA columns to the contraction ([x | s u] . [deq(W) | B]^T in the forward, [dY | v] .
// [deq(W); A] in the backward), so base and LoRA products land in one accumulator.  The LoRA stages come last so
// that a kernel launched as a dependent of the one computing s u (or v) needs that operand only at the end of
// its first unit.  Each CTA walks units
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
// g % G takes stage g), warp 6 + 4G = Q producer (lane 0 issues the codes TMA, all lanes copy absmax), and in
// the tensor-memory forward at BN >= 128 four more epilogue warps after it (each epilogue warp then drains
// half the columns of its lane quarter).  The dequantizer and Q-producer warps exist in the dequantizing modes only.
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
#include "swiglu.cuh"

namespace qlora {

// A_DEQ_TMEM_T (backward dX): the transposed weight tile, dequantized straight into tensor memory -- each TMEM lane
// (tile row = a column k of W) gathers its 64 contraction values from 64 rows of codes -- so the dX operand
// needs no shared-memory round trip.  Codes and scales arrive as in A_DEQ_MN.
enum AMode : int { A_TMA_K = 0, A_TMA_MN = 1, A_DEQ_MN = 3, A_DEQ_TMEM = 4, A_DEQ_TMEM_T = 5 };
enum WFormat : int { WF_NF4 = 0, WF_NF4_DQ = 1, WF_NVFP4 = 2 };

// E4M3 value of a finite pattern (sign bit 7, exponent bits 6..3 with bias 7, mantissa bits 2..0).
__device__ __forceinline__ float e4m3_value_dev(uint32_t code) {
  const uint32_t e = (code >> 3) & 15u, m = code & 7u;
  const float mag = e == 0 ? __fmul_rn(static_cast<float>(m), 0.001953125f) : __uint_as_float(((e + 120u) << 23) | (m << 20));
  return (code & 0x80u) ? -mag : mag;
}

// E2M1 value (sign bit 3, exponent bits 2..1 with bias 1, mantissa bit 0).
__device__ __forceinline__ float e2m1_value_dev(uint32_t code) {
  const uint32_t e = (code >> 1) & 3u, m = code & 1u;
  const float mag = e == 0 ? 0.5f * static_cast<float>(m) : static_cast<float>((2u + m) << (e - 1)) * 0.5f;
  return (code & 8u) ? -mag : mag;
}
// Epilogue modes.  EPI_SWIGLU_FWD: the GEMM is the gate/up projection in the interleaved layout (gate_pos /
// up_pos): besides gu = D it writes h = silu(g) * up to out2.  EPI_DSWIGLU: D is dh of a gated MLP's down
// projection (rows = features): it reads g, up from aux (the saved gu) and writes dgu to out2 instead of dh.
// Both need the whole contraction in one unit (no split) and bf16 outputs.
enum Epi : int { EPI_PLAIN = 0, EPI_SWIGLU_FWD = 1, EPI_DSWIGLU = 2 };

struct UmmaArgs {
  int rows, cols;         // D extent: i in [0, rows), j in [0, cols)
  int tiles_i, tiles_j;   // ceil(rows / 128), ceil(cols / BN)
  int splits;             // contraction splits; units = splits * tiles_i * tiles_j
  int k_stages;           // main contraction stages (64 KB elements each) in total
  int stages_per_split;   // main stages per split
  int n_extra;            // extra (LoRA) stages, run by split 0 only, after its main stages
  // dequantization (A_DEQ_*): W is [w_rows, w_cols] of packed 4-bit codes in format `wfmt` with one 4-byte
  // scale word per 64-element block, `scale_words` [w_rows, w_cols / 64]:
  //   WF_NF4    : the fp32 absmax of the block (codes: NF4 levels, element 2j in the high nibble);
  //   WF_NF4_DQ : `scale_words` is the byte array of 8-bit double-quantized constants (one byte per block;
  //               absmax = fl32(fl32(L[code] * dq_c1[block / 256]) + *dq_mu));
  //   WF_NVFP4  : four E4M3 patterns, the scales of the block's four 16-element groups (decoded scale =
  //               fl32(value * *fp4_S); codes: E2M1, element 2j in the low nibble).
  const void* scale_words;
  int wfmt;
  const float* dq_c1;
  const float* dq_mu;
  const float* fp4_S;
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
  // fused epilogues (Epi): h [cols, rows / 2] at out2 + (row feature) * ls2 + j * cs2, or dgu at out2 with g, up
  // read from aux, both [cols, 2 * rows] bf16 with row stride aux_ld
  // cluster split-K (TMA modes): cred = S > 1 runs the S splits of one tile as the S CTAs of a cluster, which
  // sum their fp32 partial tiles through distributed shared memory instead of writing slabs (0: off)
  int cred;
  // failure-path test only (0 in every real launch): test_stall = 1, 2 or 3 makes the MMA issuer, the B producer
  // or the codes producer leave before doing anything -- none of them then has a copy or an MMA in flight -- so
  // that every other role's wait expires; wait_limit (cycles, > 0) replaces the ~2 s bound of every wait
  int test_stall;
  long long wait_limit;
  // unit order: group_i > 0 walks the tiles in groups of group_i tile rows (weight tiles), tile rows fastest
  // within a group, so that one wave of CTAs shares a few activation tiles and a group of weight tiles and
  // both stay in L2; 0 keeps tile columns fastest
  int group_i;
  // stream-K (token-light forward, tiles_j == 1): sk_stages > 0 is the number of stages of one tile; CTA c of the
  // P in the grid takes stages [T c / P, T (c + 1) / P) of the sequence tile 0's stages, tile 1's, ... (T =
  // tiles_i sk_stages), one unit per tile it touches, and writes each unit's fp32 partial to slab z = the unit's
  // place among the CTAs sharing that tile (splits and group_i unused)
  int sk_stages;
  int epi;
  void* out2;
  long long ls2, cs2;
  const uint16_t* aux;
  long long aux_ld;
  unsigned int* err;
};

struct Unit {
  int i0, j0, z;
  int main_begin, n_main, n_extra, n_total;
};

// Stream-K: the CTA whose share holds stage x of the sequence, max{c : floor(c T / P) <= x}.
__host__ __device__ __forceinline__ long long sk_cta_of(long long x, long long T, long long P) {
  return ((x + 1) * P - 1) / T;
}

// Stream-K: units (tiles touched) of CTA c of P.
__host__ __device__ __forceinline__ int sk_units(const UmmaArgs& a, long long c, long long P) {
  const long long S = a.sk_stages, T = static_cast<long long>(a.tiles_i) * S;
  const long long s0 = T * c / P, s1 = T * (c + 1) / P;
  return s1 > s0 ? static_cast<int>((s1 - 1) / S - s0 / S + 1) : 0;
}

// Stream-K: unit u of CTA c of P -- the part of tile s0 / S + u inside the CTA's share, its slab z (the CTA's
// place among those sharing the tile) and, for the part that starts the tile, the LoRA stages (that part is the
// last unit of its CTA, so the LoRA operand is needed only at the end of the CTA's work).
__host__ __device__ __forceinline__ Unit sk_unit(const UmmaArgs& a, long long c, long long P, int u) {
  Unit U;
  const long long S = a.sk_stages, T = static_cast<long long>(a.tiles_i) * S;
  const long long s0 = T * c / P, s1 = T * (c + 1) / P;
  const long long t = s0 / S + u;
  const long long b = (s0 > t * S ? s0 : t * S) - t * S, e = (s1 < (t + 1) * S ? s1 : (t + 1) * S) - t * S;
  U.z = static_cast<int>(c - sk_cta_of(t * S, T, P));
  U.i0 = static_cast<int>(t) * 128;
  U.j0 = 0;
  U.main_begin = static_cast<int>(b);
  U.n_main = static_cast<int>(e - b);
  U.n_extra = b == 0 ? a.n_extra : 0;
  U.n_total = U.n_extra + U.n_main;
  return U;
}

// Stream-K reduction: out[e] = alpha * (sum over the n(t) partial slabs of the tile t holding e, in slab order),
// with e = j * cs + i (i the D row, fastest), t = i / 128 and n(t) the number of CTAs whose share of the stage
// sequence (S stages per tile, T in all, P CTAs) touches tile t.  Slabs past n(t) are never read.
__global__ void reduce_streamk_kernel(const float* __restrict__ ws, long long slab, long long count, long long cs,
                                      long long S, long long T, long long P, float alpha, void* __restrict__ out,
                                      int out_bf16) {
  griddep_launch_dependents();
  griddep_wait();  // the slabs are the GEMM's output
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < count; e += stride) {
    const long long t = (e % cs) / 128;
    const int n = static_cast<int>(sk_cta_of(t * S + S - 1, T, P) - sk_cta_of(t * S, T, P) + 1);
    float acc = 0.0f;
    for (int z = 0; z < n; ++z) acc += ws[z * slab + e];
    acc *= alpha;
    if (out_bf16)
      reinterpret_cast<__nv_bfloat16*>(out)[e] = __float2bfloat16_rn(acc);
    else
      reinterpret_cast<float*>(out)[e] = acc;
  }
}

// Unit u -> (split z, tile row ti, tile column tj).  Splits are outermost.  Within a split, either tile columns
// run fastest (neighbouring units share the weight tile), or -- with group_i > 0 -- the tile rows come in groups
// of group_i (the last group may be smaller) and within a group the rows run fastest: a wave of consecutive
// units then covers group_i weight tiles and only a few activation tiles, so each is fetched from DRAM about
// once per wave instead of the whole activation matrix being streamed again by every wave.
// With CTA pairs a tile row is 256 weight rows and CTA `rank` of the pair owns rows 128 rank .. 128 rank + 127.
__device__ __forceinline__ Unit unit_of(const UmmaArgs& a, int u, int BN, int pair = 1, int rank = 0) {
  if (a.sk_stages > 0) return sk_unit(a, blockIdx.x, gridDim.x, u);  // unit u of this CTA's stream-K share
  Unit U;
  int tj, ti;
  if (a.cred > 1) {  // the S consecutive units of a cluster are the S splits of one tile
    U.z = u % a.cred;
    const int t = u / a.cred;
    tj = t % a.tiles_j;
    ti = t / a.tiles_j;
  } else if (a.group_i > 0) {
    const int per_split = a.tiles_i * a.tiles_j;
    U.z = u / per_split;
    const int rem = u - U.z * per_split;
    const int grp = rem / (a.group_i * a.tiles_j);
    const int gi0 = grp * a.group_i;
    const int gsz = a.tiles_i - gi0 < a.group_i ? a.tiles_i - gi0 : a.group_i;
    const int local = rem - gi0 * a.tiles_j;
    ti = gi0 + local % gsz;
    tj = local / gsz;
  } else {
    tj = u % a.tiles_j;
    const int t = u / a.tiles_j;
    ti = t % a.tiles_i;
    U.z = t / a.tiles_i;
  }
  U.i0 = ti * 128 * pair + 128 * rank;
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
template <int BN, int AM, bool B_MN, int KB = 1, bool PAIR = false, int EPI = EPI_PLAIN, int WF = WF_NF4>
struct UmmaCfg {
  static constexpr int kPair = PAIR ? 2 : 1;   // CTAs per MMA (cta_group::2: M = 256)
  static constexpr int kBRows = BN / kPair;    // B rows (tokens) held by each CTA
  static constexpr bool kTrans = (AM == A_DEQ_TMEM_T);
  static constexpr bool kATmem = (AM == A_DEQ_TMEM || kTrans);
  static constexpr bool kQmn = (AM == A_DEQ_MN || kTrans);  // codes and scales in the MN-major slot layout
  static constexpr bool kDeq = (AM == A_DEQ_MN || kATmem);
  static constexpr bool kAMN = (AM == A_TMA_MN || AM == A_DEQ_MN);
  static constexpr bool kAbsTma = (KB == 4);  // absmax by TMA (else one cp.async per row)
  static constexpr int kTileA = 128 * 64 * 2;  // one bf16 A block in shared memory
  static constexpr int kBBytes = kBRows * 64 * 2 * KB;  // this CTA's share of a B stage
  static constexpr int kBSlot = kBBytes + (kDeq ? 0 : kTileA);  // the TMA modes load A beside B
  static constexpr int kASlot = (AM == A_DEQ_MN) ? kTileA : 0;   // A ring in shared memory
  static constexpr int kCBytes = 4096 * KB;                       // 128 rows x 64 KB codes
  static constexpr int kSBytes = 512 * KB;                        // 128 rows x KB absmax values
  static constexpr int kQSlot = kDeq ? kCBytes + kSBytes : 0;
  // the dequantizers look codes up in a shared-memory table of bf16 level pairs, one copy per lane, placed at
  // the start of the dynamic shared memory (a fixed address the compiler folds into the loads): entry stride
  // 128 bytes (32 KB), or -- in the token-light 4-block kernels at BN <= 32, whose dequantizers bound the
  // kernel -- entry stride 256 bytes (64 KB, half of it padding), so that one byte permute of (code byte, lane)
  // is the whole offset
  static constexpr bool kWideLut = kDeq && KB == 4 && BN <= 32;
  // (the MN-major dequantizer of NF4 codes looks levels up in registers and needs no table)
  static constexpr bool kRegTable = AM == A_DEQ_MN && WF != WF_NVFP4;
  static constexpr int kLutBytes = (kDeq && !kRegTable) ? (kWideLut ? 256 * 64 * 4 : 256 * 32 * 4) : 0;
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
  static constexpr int kBStagesWant =
      kDeq ? (kWideLut ? 4 : BN <= 64 ? 8 : (AM == A_DEQ_MN && BN >= 256 ? (kRegTable ? 4 : 3) : 4)) : 8;
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
  // The forward at BN >= 128 keeps A in tensor memory, which leaves room for one accumulator only, so its
  // epilogue (the fused SwiGLU one above all) is not overlapped with the next unit's MMAs: it runs on 8 epilogue
  // warps (two per lane quarter, each draining half the columns), and the CTA has one dequantizer group fewer
  // to stay within the register file.
  static constexpr int kEpiWarps = (AM == A_DEQ_TMEM && BN >= 128) ? 8 : 4;
  static constexpr int kDeqCap = kATmem ? (kEpiWarps == 8 ? 3 : 4) : 3;
  static constexpr int kDeqGroups = kDeq ? (kAStages < kDeqCap ? kAStages : kDeqCap) : 0;
  static constexpr int kQWarp = 6 + 4 * kDeqGroups;
  // warps: producers and MMA (0, 1), epilogue (2..5), dequantizers, the Q producer, extra epilogue warps
  static constexpr int kThreads = kDeq ? 32 * (kQWarp + 1 + kEpiWarps - 4) : 64 + 128;
  static constexpr int kTmemNeed = kAColBase + (kATmem ? kAStages * kAColsStage : 0);
  static constexpr int kTmemCols = kTmemNeed <= 32 ? 32 : kTmemNeed <= 64 ? 64 : kTmemNeed <= 128 ? 128 : kTmemNeed <= 256 ? 256 : 512;
  static constexpr int kSmemBytes =
      1024 + kBStages * kBSlot + kAStages * kASlot + kQStages * kQSlot + kLutBytes + kBarBytes;

  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N for M=128 is a multiple of 16 in [16, 256]");
  static_assert(!B_MN || BN % 64 == 0, "MN-major B tiles are whole 64-element swizzle atoms");
  static_assert(!(kDeq && B_MN), "the dequantizing modes take B K-major");
  static_assert(KB == 1 || (AM == A_DEQ_TMEM && KB == 4), "4-block stages exist for the TMEM forward only");
  static_assert(!PAIR || (kDeq && BN % 16 == 0), "CTA pairs: dequantizing modes, 8-row-aligned B halves");
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
template <int BN, int AM, bool B_MN, int KB = 1, bool PAIR = false, int WF = WF_NF4, int EPI = EPI_PLAIN>
__global__ void __launch_bounds__(UmmaCfg<BN, AM, B_MN, KB, PAIR, EPI, WF>::kThreads, 1)
    umma_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmBx, const __grid_constant__ CUtensorMap tmC,
                     const UmmaArgs args) {
  using C = UmmaCfg<BN, AM, B_MN, KB, PAIR, EPI, WF>;
  static_assert(AM != A_DEQ_TMEM_T || WF == WF_NF4, "the transposed TMEM dequantizer reads NF4 weights");
  constexpr int BS = C::kBStages;
  constexpr int AS = C::kAStages;
  constexpr int QS = C::kQStages;
  constexpr uint32_t kFull = 0xffffffffu;

  extern __shared__ uint8_t smem_raw[];
  // the level-pair table first (at the array's own address), then the rings from the next 1024-byte boundary;
  // align by pointer arithmetic on the shared array itself (not through an integer), so every pointer derived
  // from it stays a known shared-memory pointer and compiles to shared loads and stores
  uint32_t* sLut = reinterpret_cast<uint32_t*>(smem_raw);
  uint8_t* ring_raw = smem_raw + C::kLutBytes;
  const uint32_t raw_addr = smem_u32(ring_raw);
  uint8_t* smem = ring_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* sB = smem;                          // B ring (B, then A in the TMA modes), 1024-aligned slots
  uint8_t* sA = sB + BS * C::kBSlot;           // A ring of A_DEQ_MN, 1024-aligned slots
  uint8_t* sQ = sA + AS * C::kASlot;           // Q ring: codes, then absmax
  // Phases: b_* advance once per stage (every stage uses the B ring), a_* once per stage in the dequantizing
  // modes, q_* once per MAIN stage, tmem_* once per unit accumulated in that buffer.  Each waiter derives
  // the parity from its running count of the ring's uses, which is sound only while the barrier's previous
  // phase has completed when the wait starts and its next one cannot complete before the waiter releases:
  //   - a barrier cannot run ahead: each refill needs the consumer's release of the slot first;
  //   - a dequantizer at stage g has seen the MMAs of stage g - G - AS complete (its own previous stage's
  //     a_empty wait, G = dequantizer groups), so with G <= AS its a_empty wait for stage g - AS cannot see
  //     an older phase, and with QS >= AS + G the Q stage QS before its own has been consumed;
  //   - the MMA and the producers visit every phase of the barriers they wait on, in order.
  uint64_t* b_full = reinterpret_cast<uint64_t*>(sQ + QS * C::kQSlot);
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
  const bool streamk = args.sk_stages > 0;
  const long long lim = args.wait_limit > 0 ? args.wait_limit : kWaitTimeoutCycles;
  // CTA pairs: the even CTA of the cluster (rank 0) is the leader -- it issues the pair's MMAs, and its barriers
  // gather both CTAs' arrivals; each pair walks the units together
  const int rank = PAIR ? static_cast<int>(cluster_ctarank()) : 0;
  const int first_unit = streamk ? 0 : PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int unit_step = streamk ? 1 : PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  const int num_units = streamk ? sk_units(args, blockIdx.x, gridDim.x) : args.splits * args.tiles_i * args.tiles_j;

  if (threadIdx.x == 0) {
    for (int s = 0; s < BS; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], 1);
    }
    for (int s = 0; s < AS; ++s) {
      mbar_init(&a_full[s], C::kDeqWarpsPerGroup * C::kPair);
      mbar_init(&a_empty[s], 1);
    }
    for (int s = 0; s < QS; ++s) {
      // the TMA arrive (+ one cp.async arrive per producer lane when the scale words come by cp.async)
      mbar_init(&q_full[s], C::kAbsTma && WF != WF_NF4_DQ ? 1 : 1 + 32);
      mbar_init(&q_empty[s], C::kDeqWarpsPerGroup * 32);  // every lane of the consuming group
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tmem_full[b], 1);
      mbar_init(&tmem_empty[b], C::kEpiWarps * C::kPair);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if constexpr (C::kLutBytes > 0) {
    // entry (byte b, lane l) at word 32 b + l (64 b + l in the wide table): the bf16 pair of the byte's two
    // elements, element 2j in the low half.  NF4 bytes hold element 2j in the high nibble, NVFP4 bytes in the
    // low nibble.
    constexpr bool fp4 = WF == WF_NVFP4;
    for (int idx = threadIdx.x; idx < 256 * 32; idx += blockDim.x) {
      const int b = idx >> 5;
      __nv_bfloat162 h = fp4 ? __floats2bfloat162_rn(e2m1_value_dev(b & 15), e2m1_value_dev(b >> 4))
                             : __floats2bfloat162_rn(kNF4LevelsDev[b >> 4], kNF4LevelsDev[b & 15]);
      sLut[C::kWideLut ? 64 * b + (idx & 31) : idx] = *reinterpret_cast<uint32_t*>(&h);
    }
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmB);
    if (!C::kDeq) tma_prefetch_desc(&tmA);
    if (args.n_extra > 0) tma_prefetch_desc(&tmBx);
  }
  if (C::kDeq && warp == C::kQWarp && lane == 0) {
    tma_prefetch_desc(&tmC);
    if (C::kAbsTma && WF != WF_NF4_DQ) tma_prefetch_desc(&tmA);
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, C::kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, C::kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync_all();  // the peer arrives on our barriers only once they exist
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Launched as a dependent of the kernel before it, this kernel reads nothing that kernel writes before the
  // producer's griddep_wait (B of the LoRA stages in the dequantizing modes, every operand in the TMA modes), and
  // writes nothing before the epilogue's; the weight codes and scales, the activations of the main stages and the
  // LoRA rows come from before that kernel.
  if (threadIdx.x == 0) griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------------ B producer
    Armed armed;
    int g = 0;
    bool stop = args.test_stall == 2;
    bool dep_done = false;  // griddep_wait issued
    for (int u = first_unit; u < num_units && !stop; u += unit_step) {
      const Unit U = unit_of(args, u, BN, C::kPair, rank);
      for (int it = 0; it < U.n_total; ++it, ++g) {
        const int s = g % BS;
        const uint32_t ph = static_cast<uint32_t>(g / BS) & 1u;
        const bool ok = mbar_wait_idle(&b_empty[s], ph ^ 1u, abort_flag, args.err, lim);
        if (!__all_sync(kFull, ok)) {
          stop = true;
          break;
        }
        if (lane == 0) {
          if (!dep_done && (!C::kDeq || it >= U.n_main)) {
            griddep_wait();
            dep_done = true;
          }
          armed.set(s, ph);
          uint8_t* b_dst = sB + s * C::kBSlot;
          if constexpr (C::kDeq) {
            // KB blocks of kBRows x 64 (this CTA's share of the BN tokens), each a 128B-swizzled K-major
            // sub-tile; with CTA pairs both halves complete on the leader's barrier, which expects both
            if (rank == 0) mbar_arrive_expect_tx(&b_full[s], C::kPair * C::kBBytes);
            const int jb = U.j0 + rank * C::kBRows;
#pragma unroll
            for (int kb = 0; kb < KB; ++kb) {
              uint8_t* dst = b_dst + kb * C::kBRows * 128;
              const bool ex = it >= U.n_main;  // the LoRA stages follow the unit's main stages
              const int x = ex ? 64 * (KB * (it - U.n_main) + kb) : ((U.main_begin + it) * KB + kb) * 64;
              const CUtensorMap* tm = ex ? &tmBx : &tmB;
              if constexpr (PAIR)
                tma_load_2d_pair(dst, tm, x, jb, &b_full[s]);
              else
                tma_load_2d(dst, tm, x, jb, &b_full[s]);
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
    // copies still in flight must land before the CTA's shared memory is released (a pair's copies complete
    // on the leader's barriers: the leader drains them, and the closing cluster barrier holds the follower)
    if (lane == 0 && *abort_flag && rank == 0) armed.drain(b_full, BS, args.err);
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (whole warp waits,
    // one elected lane issues)
    constexpr uint32_t idesc = idesc_bf16_f32(PAIR ? 256 : 128, BN, C::kAMN, B_MN);
    // barriers the peer CTA also arrives on are waited with acquire at cluster scope
    auto wait_mma = [&](uint64_t* bar, uint32_t par) {
      if constexpr (PAIR)
        return mbar_wait_cluster(bar, par, abort_flag, args.err, lim);
      else
        return mbar_wait(bar, par, abort_flag, args.err, lim);
    };
    int g = 0, lu = 0;
    bool stop = rank != 0 || args.test_stall == 1;  // the pair's follower issues nothing
    for (int u = first_unit; u < num_units && !stop; u += unit_step, ++lu) {
      const Unit U = unit_of(args, u, BN, C::kPair, rank);
      const int acc = lu % C::kAccBufs;
      const uint32_t eph = (static_cast<uint32_t>(lu / C::kAccBufs) & 1u) ^ 1u;
      if (!__all_sync(kFull, wait_mma(&tmem_empty[acc], eph))) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::kAccCols);
      for (int it = 0; it < U.n_total; ++it, ++g) {
        const int bs = g % BS;
        int as = 0;
        bool ok;
        if constexpr (C::kDeq) {
          as = g % AS;
          ok = wait_mma(&a_full[as], static_cast<uint32_t>(g / AS) & 1u) &&
               wait_mma(&b_full[bs], static_cast<uint32_t>(g / BS) & 1u);
        } else {
          ok = mbar_wait(&b_full[bs], static_cast<uint32_t>(g / BS) & 1u, abort_flag, args.err, lim);
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
            const uint32_t bk = b0 + static_cast<uint32_t>(kb * C::kBRows * 128);
            const uint64_t bdesc = B_MN ? sdesc_sw128(bk + k * 2048, 8192, 1024) : sdesc_sw128(bk + k * 32, 16, 1024);
            const uint32_t accum = (it > 0 || kk > 0) ? 1u : 0u;
            if constexpr (C::kATmem) {
              const uint32_t a_tmem =
                  tmem_base + static_cast<uint32_t>(C::kAColBase + as * C::kAColsStage + kb * 32 + k * 8);
              if constexpr (PAIR)
                umma_bf16_ts_pair(d_tmem, a_tmem, bdesc, idesc, accum);
              else
                umma_bf16_ts(d_tmem, a_tmem, bdesc, idesc, accum);
            } else {
              const uint64_t adesc =
                  C::kAMN ? sdesc_sw128(a0 + k * 2048, 8192, 1024) : sdesc_sw128(a0 + k * 32, 16, 1024);
              if constexpr (PAIR)
                umma_bf16_ss_pair(d_tmem, adesc, bdesc, idesc, accum);
              else
                umma_bf16_ss(d_tmem, adesc, bdesc, idesc, accum);
            }
          }
          if constexpr (PAIR) {  // the commits arrive on the barrier at this offset in both CTAs
            umma_commit_pair(&b_empty[bs]);
            umma_commit_pair(&a_empty[as]);
          } else {
            umma_commit(&b_empty[bs]);
            if constexpr (C::kDeq) umma_commit(&a_empty[as]);
          }
        }
        __syncwarp();
      }
      if (elect_one()) {  // also on abort, so the MMAs issued can be waited for
        if constexpr (PAIR)
          umma_commit_pair(&tmem_full[acc]);
        else
          umma_commit(&tmem_full[acc]);
      }
      __syncwarp();
    }
  } else if (warp < 6 || warp > C::kQWarp) {
    // ------------------------------------------------------------------ epilogue (warps 2..5, and with 8
    // epilogue warps also the last four: those drain the second half of the columns)
    const int qw = warp & 3;  // TMEM lane quarter this warp may access
    constexpr int kCols = BN * 4 / C::kEpiWarps;
    const int c_begin = warp < 6 ? 0 : kCols, c_end = c_begin + kCols;
    int lu = 0;
    for (int u = first_unit; u < num_units; u += unit_step, ++lu) {
      const Unit U = unit_of(args, u, BN, C::kPair, rank);
      const int acc = lu % C::kAccBufs;
      int ok = mbar_wait_idle(&tmem_full[acc], static_cast<uint32_t>(lu / C::kAccBufs) & 1u, abort_flag, args.err, lim) ? 1 : 0;
      tc_fence_after();
      ok = __shfl_sync(kFull, ok && !*abort_flag, 0);
      if (!ok) break;
      if (lu == 0) griddep_wait();  // before the first global access of the epilogue
      const int i = U.i0 + qw * 32 + lane;
      const long long base = static_cast<long long>(U.z) * args.split_stride + static_cast<long long>(i) * args.ls;
      const uint32_t t_acc = tmem_base + (static_cast<uint32_t>(qw * 32) << 16) + static_cast<uint32_t>(acc * C::kAccCols);
      // EPI_DSWIGLU: g (low half) and up (high half) of this row's feature for the 16 tokens of the next chunk
      // (tokens past the count read the last token's row: in bounds, never stored)
      uint32_t gunext[EPI == EPI_DSWIGLU ? 16 : 1];
      auto load_gu = [&](int cc, long long pg) {
        if constexpr (EPI == EPI_DSWIGLU) {
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            const int j = min(U.j0 + cc + jj, args.cols_lim - 1);
            const uint16_t* row = args.aux + static_cast<long long>(j) * args.aux_ld;
            gunext[jj] = static_cast<uint32_t>(__ldg(row + pg)) | (static_cast<uint32_t>(__ldg(row + pg + 16)) << 16);
          }
        }
      };
      if constexpr (EPI == EPI_DSWIGLU) load_gu(c_begin, gate_pos(i < args.rows_lim ? i : 0));
#pragma unroll 1
      for (int c0 = c_begin; c0 < c_end; c0 += 16) {
        uint32_t r[16];
        __syncwarp();  // tcgen05.ld is warp-aligned: reconverge after the guarded stores
        tmem_ld_32x32b_x16(t_acc + static_cast<uint32_t>(c0), r);
        tmem_ld_wait();
        if (!C::kDeq && args.cred > 1) {
          // this split's raw fp32 partial of the tile, row i - i0, parked in the (drained) B ring
          float* prow = reinterpret_cast<float*>(sB) + (qw * 32 + lane) * (BN + 4) + c0;
#pragma unroll
          for (int jj = 0; jj < 16; jj += 4)
            *reinterpret_cast<float4*>(prow + jj) =
                U.n_total > 0 ? make_float4(__uint_as_float(r[jj]), __uint_as_float(r[jj + 1]),
                                            __uint_as_float(r[jj + 2]), __uint_as_float(r[jj + 3]))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
          continue;
        }
        if constexpr (EPI == EPI_SWIGLU_FWD) {
          // gu as stored (bf16); lanes l and l ^ 16 hold g and up of one feature.  Each lane of the pair forms
          // h for half of the chunk's tokens -- the gate lane the even ones, the up lane the odd ones -- so all
          // lanes do the same work
          const bool gate = (lane & 16) == 0;
          const long long feat = static_cast<long long>(i >> 5) * 16 + (lane & 15);
          float v[16], pv[16];
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            const int j = U.j0 + c0 + jj;
            const __nv_bfloat16 b = __float2bfloat16_rn(U.n_total > 0 ? args.alpha * __uint_as_float(r[jj]) : 0.0f);
            v[jj] = __bfloat162float(b);
            if (i < args.rows_lim && j < args.cols_lim)
              reinterpret_cast<__nv_bfloat16*>(args.out)[base + static_cast<long long>(j) * args.cs] = b;
          }
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) pv[jj] = __shfl_xor_sync(kFull, v[jj], 16);
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            const float g = gate ? v[2 * t] : pv[2 * t + 1];
            const float u = gate ? pv[2 * t] : v[2 * t + 1];
            const int j = U.j0 + c0 + 2 * t + (gate ? 0 : 1);
            if (i < args.rows_lim && j < args.cols_lim)
              reinterpret_cast<__nv_bfloat16*>(args.out2)[feat * args.ls2 + static_cast<long long>(j) * args.cs2] =
                  __float2bfloat16_rn(swiglu_h(g, u));
          }
          continue;
        }
        if constexpr (EPI == EPI_DSWIGLU) {
          // dh as stored (bf16), with g and up of feature i from the saved gu, gives the two halves of dgu.  The
          // chunk's g and up were loaded one chunk ahead (dgu stores may alias gu as far as the compiler knows,
          // so it would not hoist the loads itself)
          const long long pg = gate_pos(i < args.rows_lim ? i : 0), pu = pg + 16;
          uint32_t gucur[16];
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) gucur[jj] = gunext[jj];
          if (c0 + 16 < c_end) load_gu(c0 + 16, pg);
          if (i < args.rows_lim) {
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
              const int j = U.j0 + c0 + jj;
              if (j < args.cols_lim) {
                const float d = __bfloat162float(
                    __float2bfloat16_rn(U.n_total > 0 ? args.alpha * __uint_as_float(r[jj]) : 0.0f));
                float dg, du;
                swiglu_grads(d, __uint_as_float(gucur[jj] << 16), __uint_as_float(gucur[jj] & 0xFFFF0000u), dg, du);
                __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(args.out2) + static_cast<long long>(j) * args.aux_ld;
                o[pg] = __float2bfloat16_rn(dg);
                o[pu] = __float2bfloat16_rn(du);
              }
            }
          }
          continue;
        }
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
      if (lane == 0) {
        if constexpr (PAIR)
          mbar_arrive_leader(&tmem_empty[acc]);
        else
          mbar_arrive(&tmem_empty[acc]);
      }
    }
  } else if (warp == C::kQWarp) {
    // ------------------------------------------------------------------ Q producer (dequantizing modes)
    if constexpr (C::kDeq) {
      Armed armed;
      int q = 0;
      bool stop = args.test_stall == 3;
      for (int u = first_unit; u < num_units && !stop; u += unit_step) {
        const Unit U = unit_of(args, u, BN, C::kPair, rank);
        for (int it = 0; it < U.n_main; ++it, ++q) {
          const int s = q % QS;
          const uint32_t ph = static_cast<uint32_t>(q / QS) & 1u;
          const bool ok = mbar_wait_idle(&q_empty[s], ph ^ 1u, abort_flag, args.err, lim);
          if (!__all_sync(kFull, ok)) {
            stop = true;
            break;
          }
          const int kk0 = (U.main_begin + it) * 64 * KB;
          uint8_t* q_dst = sQ + s * C::kQSlot;
          // 4-block stages take their scale words by TMA, except the double-quantized constants (4 bytes a row,
          // below the 16-byte minimum of a TMA box row)
          constexpr bool scale_tma = C::kAbsTma && WF != WF_NF4_DQ;
          if (lane == 0) {
            armed.set(s, ph);
            if constexpr (scale_tma) {
              // 128 W rows x 128 bytes of codes (swizzled) and 128 rows x 4 scale words
              mbar_arrive_expect_tx(&q_full[s], C::kCBytes + C::kSBytes);
              tma_load_2d(q_dst, &tmC, kk0 / 2, U.i0, &q_full[s]);
              tma_load_2d(q_dst + C::kCBytes, &tmA, WF == WF_NVFP4 ? kk0 / 16 : kk0 / 64, U.i0, &q_full[s]);
            } else if constexpr (C::kAbsTma) {
              mbar_arrive_expect_tx(&q_full[s], C::kCBytes);
              tma_load_2d(q_dst, &tmC, kk0 / 2, U.i0, &q_full[s]);
            } else {
              mbar_arrive_expect_tx(&q_full[s], C::kCBytes);
              if constexpr (!C::kQmn)
                tma_load_2d(q_dst, &tmC, kk0 / 2, U.i0, &q_full[s]);  // 128 W rows x 32 bytes
              else
                tma_load_2d(q_dst, &tmC, U.i0 / 2, kk0, &q_full[s]);  // 64 W rows x 64 bytes
            }
          }
          if constexpr (scale_tma) continue;
          // one 4-byte word per (row, block): the fp32 absmax or the four NVFP4 group scales of the block; for
          // the double-quantized constants the aligned word holding the block's byte (with 4-block stages, the
          // word of the stage's four bytes, stored at the row's 16-byte scale slot)
          uint32_t* sdst = reinterpret_cast<uint32_t*>(q_dst + C::kCBytes);
          const uint8_t* words8 = static_cast<const uint8_t*>(args.scale_words);
          constexpr bool dq = WF == WF_NF4_DQ;
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            const int idx = lane + 32 * qq;
            int n, k;
            if constexpr (!C::kQmn) {  // word for tile row idx (W row i0 + idx) in k-block kk0 / 64
              n = U.i0 + idx;
              k = kk0;
            } else {                           // word for W row kk0 + idx / 2 in k-block (i0 + 64 (idx & 1)) / 64
              n = kk0 + (idx >> 1);
              k = U.i0 + 64 * (idx & 1);
            }
            const bool valid = n < args.w_rows && k < args.w_cols;
            const long long blk = static_cast<long long>(n) * args.w_kb + (k >> 6);
            const uint8_t* src = !valid ? words8 : dq ? words8 + (blk & ~3ll) : words8 + 4 * blk;
            cp_async_4_zfill(sdst + (C::kAbsTma ? 4 * idx : idx), src, valid);
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
      const int s_idx = C::kATmem ? row : (row * 2 + h);
      const uint32_t t_lane = static_cast<uint32_t>(32 * (warp & 3)) << 16;
      const uint8_t* lut_lane = reinterpret_cast<const uint8_t*>(sLut) + lane * 4;
      const uint32_t lane4 = static_cast<uint32_t>(lane) * 4u;
      // The MN-major (dX) dequantizer of NF4 codes looks levels up in registers instead of the shared table, which
      // takes the table's 16 KB per stage off the shared-memory pipe that bounds dX: tl[q] / th[q] hold the low
      // / high bytes of the bf16 levels 4q .. 4q + 3.
      uint32_t tl[4] = {}, th[4] = {};
      if constexpr (C::kRegTable) {
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat16 hv = __float2bfloat16_rn(kNF4LevelsDev[4 * q4 + e]);
            const uint32_t bits = *reinterpret_cast<const uint16_t*>(&hv);
            tl[q4] |= (bits & 0xFFu) << (8 * e);
            th[q4] |= (bits >> 8) << (8 * e);
          }
        }
      }
      const float dq_mu = WF == WF_NF4_DQ ? *args.dq_mu : 0.0f;
      const float fp4_S = WF == WF_NVFP4 ? *args.fp4_S : 0.0f;
      int g = 0, q = 0;
      bool stop = false;
      for (int u = first_unit; u < num_units && !stop; u += unit_step) {
        const Unit U = unit_of(args, u, BN, C::kPair, rank);
        for (int it = 0; it < U.n_total; ++it, ++g) {
          const bool extra = it >= U.n_main;
          const int xe = it - U.n_main;  // LoRA stage index within the unit
          const int qi = q;
          if (!extra) ++q;
          if (g % C::kDeqGroups != grp) continue;
          // The stage's codes and scales, held in registers: block p of the stage is words[8p .. 8p + 7]
          // (64 codes) with scale word sw[p] (for the double-quantized constants: the aligned word that holds
          // the block's byte, or with 4-block stages the stage's four bytes, in sw[0]).
          uint32_t words[8 * KB];
          uint32_t sw[KB] = {};  // (the transposing dequantizer reads its scales straight from the slot)
          uint32_t r[32];  // the stage's 64 bf16 values (the first block's), packed in pairs
          if (!extra) {
            const int qs = qi % QS;
            const bool okq = mbar_wait_idle(&q_full[qs], static_cast<uint32_t>(qi / QS) & 1u, abort_flag, args.err, lim);
            if (!__all_sync(kFull, okq)) {
              stop = true;
              break;
            }
            const uint8_t* q_src = sQ + qs * C::kQSlot;
            if constexpr (C::kTrans) {
              // tile row `row` = column k = i0 + row of W: its code in each of the stage's 64 W rows is byte
              // row / 2 of the row's 64 (the high nibble for even k), its scale that of the row's k-block
              // (i0 + 64 (row / 64)) / 64; two rows per pair lookup, two scales per bf16x2 product
              const uint8_t* cb = q_src + (row >> 1);
              const float* sb = reinterpret_cast<const float*>(q_src + C::kCBytes) + (row >> 6);
              const uint32_t sh = (row & 1) ? 0u : 4u;
#pragma unroll
              for (int pp = 0; pp < 32; ++pp) {
                const uint32_t c0 = (static_cast<uint32_t>(cb[(2 * pp) * 64]) >> sh) & 15u;
                const uint32_t c1 = (static_cast<uint32_t>(cb[(2 * pp + 1) * 64]) >> sh) & 15u;
                uint32_t v = *reinterpret_cast<const uint32_t*>(lut_lane + (((c0 << 4) | c1) << 7));
                const __nv_bfloat162 s2 = __floats2bfloat162_rn(sb[(2 * pp) * 2], sb[(2 * pp + 1) * 2]);
                const __nv_bfloat162 pr = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&v), s2);
                r[pp] = *reinterpret_cast<const uint32_t*>(&pr);
              }
            } else if constexpr (C::kAbsTma) {
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
              const uint4 s4 = *reinterpret_cast<const uint4*>(q_src + C::kCBytes + row * 16);
              sw[0] = s4.x;
              if constexpr (KB == 4) {
                sw[1] = s4.y;
                sw[2] = s4.z;
                sw[3] = s4.w;
              }
            } else {
              sw[0] = reinterpret_cast<const uint32_t*>(q_src + C::kCBytes)[s_idx];
              // the thread's two 16-byte chunks (c0, c0 + 1) of its codes row, each at its swizzled position:
              // 32-byte rows (forward) XOR bit 7 of the address, 64-byte rows (dX) XOR bits 7..8
              const int c0 = C::kATmem ? 0 : 2 * h;
              const int sx = C::kATmem ? ((row >> 2) & 1) : ((row >> 1) & 3);
              const uint8_t* q_row = q_src + (C::kATmem ? row * 32 : row * 64);
              const uint4 c01 = *reinterpret_cast<const uint4*>(q_row + ((c0 ^ sx) << 4));
              const uint4 c23 = *reinterpret_cast<const uint4*>(q_row + (((c0 + 1) ^ sx) << 4));
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
                c0 = 64 * (KB * xe + p);
                valid = n < args.w_rows;
                src = args.lora + static_cast<long long>(n) * args.lora_ld + c0;
              } else {
                const int jr = 64 * xe + row;
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
              // level pair from this lane's copy of the table, times the scale of its 16-element group in bf16x2
              __nv_bfloat162 sc2q[4];
              if constexpr (WF == WF_NVFP4) {
#pragma unroll
                for (int gq = 0; gq < 4; ++gq)
                  sc2q[gq] = __float2bfloat162_rn(__fmul_rn(e4m3_value_dev((sw[p] >> (8 * gq)) & 0xFFu), fp4_S));
              } else {
                float a;
                if constexpr (WF == WF_NF4_DQ) {
                  // this thread's W row and k-block of block p (the producer's word holds its byte)
                  int n, kb;
                  if constexpr (C::kATmem) {
                    n = U.i0 + row;
                    kb = (U.main_begin + it) * KB + p;
                  } else {
                    n = (U.main_begin + it) * 64 + row;
                    kb = (U.i0 >> 6) + h;
                  }
                  const long long blk = static_cast<long long>(n) * args.w_kb + kb;
                  const uint32_t code = (sw[KB == 4 ? 0 : p] >> (8 * static_cast<int>(blk & 3))) & 0xFFu;
                  a = (n < args.w_rows && kb < args.w_kb)
                          ? __fadd_rn(__fmul_rn(__fdiv_rn(e4m3_value_dev(code), 448.0f), __ldg(args.dq_c1 + (blk >> 8))),
                                      dq_mu)
                          : 0.0f;
                } else {
                  a = __uint_as_float(sw[p]);
                }
                sc2q[0] = sc2q[1] = sc2q[2] = sc2q[3] = __float2bfloat162_rn(a);
              }
              if constexpr (C::kRegTable) {
                // Per code word (8 elements; byte j holds element 2j in its high nibble): swap the nibbles of each
                // byte so that nibble k is element k's code, select the level bytes of four codes at a time from
                // the register table (codes 0..7 from tl[0..1], 8..15 from tl[2..3], chosen per byte by a mask of
                // the codes' top bits, which prmt's sign mode spreads over their bytes), interleave low and high
                // bytes into bf16 pairs, then scale.  Equal to the table lookup bit for bit.
#pragma unroll
                for (int w = 0; w < 8; ++w) {
                  const __nv_bfloat162 sc2 = sc2q[w >> 1];
                  const uint32_t qw8 = words[8 * p + w];
                  const uint32_t qs = ((qw8 >> 4) & 0x0F0F0F0Fu) | ((qw8 << 4) & 0xF0F0F0F0u);
                  const uint32_t s7 = qs & 0x77777777u, t4 = qs << 4;
#pragma unroll
                  for (int hf = 0; hf < 2; ++hf) {
                    const uint32_t sel = hf ? (s7 >> 16) : s7;
                    const uint32_t m = prmt_sign(t4, qs, hf ? 0xFBEAu : 0xD9C8u);
                    const uint32_t lo = (__byte_perm(tl[0], tl[1], sel) & ~m) | (__byte_perm(tl[2], tl[3], sel) & m);
                    const uint32_t hi = (__byte_perm(th[0], th[1], sel) & ~m) | (__byte_perm(th[2], th[3], sel) & m);
                    uint32_t v0 = __byte_perm(lo, hi, 0x5140u), v1 = __byte_perm(lo, hi, 0x7362u);
                    const __nv_bfloat162 p0 = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&v0), sc2);
                    const __nv_bfloat162 p1 = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&v1), sc2);
                    r[4 * w + 2 * hf] = *reinterpret_cast<const uint32_t*>(&p0);
                    r[4 * w + 2 * hf + 1] = *reinterpret_cast<const uint32_t*>(&p1);
                  }
                }
              } else {
#pragma unroll
                for (int w = 0; w < 8; ++w) {
                  const __nv_bfloat162 sc2 = sc2q[w >> 1];
                  const uint32_t qw8 = words[8 * p + w];
#pragma unroll
                  for (int j = 0; j < 4; ++j) {
                    // byte offset of (code byte j, lane) in the table: one byte permute into (byte << 8) | 4 lane for
                    // the wide table, a permute and a shift-add for the narrow one
                    const uint32_t off =
                        C::kWideLut ? __byte_perm(qw8, lane4, 0x5504u | (static_cast<uint32_t>(j) << 4))
                                    : (__byte_perm(qw8, 0u, 0x4440u + static_cast<uint32_t>(j)) << 7) + lane4;
                    uint32_t v = *reinterpret_cast<const uint32_t*>(smem_raw + off);
                    __nv_bfloat162 pr = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&v), sc2);
                    r[4 * w + j] = *reinterpret_cast<uint32_t*>(&pr);
                  }
                }
              }
            }
          };
          if constexpr (C::kTrans) {
            if (extra) {
              // LoRA rows of A [lora_r, w_cols]: tile row k = i0 + row takes column k of the stage's 64 rows
              const int k = U.i0 + row;
              const bool vk = k < args.w_cols;
#pragma unroll
              for (int pp = 0; pp < 32; ++pp) {
                const int j = 64 * xe + 2 * pp;
                const uint32_t lo = (vk && j < args.lora_r)
                                        ? __ldg(args.lora + static_cast<long long>(j) * args.lora_ld + k) : 0u;
                const uint32_t hi = (vk && j + 1 < args.lora_r)
                                        ? __ldg(args.lora + static_cast<long long>(j + 1) * args.lora_ld + k) : 0u;
                r[pp] = lo | (hi << 16);
              }
            }
          } else {
            block_values(0, r);
          }
          // the A slot is free once the MMAs of its previous stage have completed
          const int as = g % AS;
          const bool oka = mbar_wait_idle(&a_empty[as], (static_cast<uint32_t>(g / AS) & 1u) ^ 1u, abort_flag, args.err, lim);
          if (!__all_sync(kFull, oka)) {
            stop = true;
            break;
          }
          tc_fence_after();
          // the MMAs of the slot's previous stage read it through the async proxy; order those reads before
          // this thread's generic writes
          if constexpr (!C::kATmem) {
            if constexpr (PAIR)
              fence_proxy_async_smem_cluster();
            else
              fence_proxy_async_smem();
          }
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
            // visible to the async proxy -- with CTA pairs, to the leader's MMA reading this CTA's tile
            if constexpr (PAIR)
              fence_proxy_async_smem_cluster();
            else
              fence_proxy_async_smem();
          }
          __syncwarp();
          if (lane == 0) {  // this warp's quarter of the A stage is in place (with pairs: on the leader's barrier)
            if constexpr (PAIR)
              mbar_arrive_leader(&a_full[as]);
            else
              mbar_arrive(&a_full[as]);
          }
          stop = __shfl_sync(kFull, stop ? 1 : 0, 0) != 0;
          if (stop) break;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  // a pair stays together to the end: the peer may still arrive on our barriers or have copies in flight
  // counted on the leader's, and tensor memory is released by both CTAs together
  if constexpr (PAIR) cluster_sync_all();
  if constexpr (!C::kDeq && !PAIR) {
    if (args.cred > 1) {
      // cluster split-K: every CTA holds one split's partial tile (one unit each); CTA c sums rows
      // [c R, (c + 1) R) of the tile over the S partials in split order -- the order of the slab reduction --
      // then scales and stores them.  The second barrier keeps every CTA's shared memory alive until read.
      cluster_sync_all();
      const int S = args.cred;
      const int c = static_cast<int>(cluster_ctarank());
      const Unit U = unit_of(args, static_cast<int>(blockIdx.x), BN);
      const int R = 128 / S;
      const int per_row = BN / 4;
      const uint32_t base_addr = smem_u32(sB);
      if (warp >= 2 && warp < 6) {
        for (int e = threadIdx.x - 64; e < R * per_row; e += 128) {
          const int row = c * R + e / per_row, col = (e % per_row) * 4;
          const uint32_t off = static_cast<uint32_t>((row * (BN + 4) + col) * 4);
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int src = 0; src < S; ++src) {
            const float4 v = ld_dsmem_f32x4(mapa_cluster(base_addr + off, static_cast<uint32_t>(src)));
            acc.x = __fadd_rn(acc.x, v.x);
            acc.y = __fadd_rn(acc.y, v.y);
            acc.z = __fadd_rn(acc.z, v.z);
            acc.w = __fadd_rn(acc.w, v.w);
          }
          const int i = U.i0 + row;
          if (i < args.rows_lim) {
            const float o[4] = {__fmul_rn(acc.x, args.alpha), __fmul_rn(acc.y, args.alpha),
                                __fmul_rn(acc.z, args.alpha), __fmul_rn(acc.w, args.alpha)};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int j = U.j0 + col + q;
              if (j < args.cols_lim) {
                const long long at = static_cast<long long>(i) * args.ls + static_cast<long long>(j) * args.cs;
                if (args.out_bf16)
                  reinterpret_cast<__nv_bfloat16*>(args.out)[at] = __float2bfloat16_rn(o[q]);
                else
                  reinterpret_cast<float*>(args.out)[at] = o[q];
              }
            }
          }
        }
      }
      cluster_sync_all();
    }
  }
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if constexpr (PAIR)
      tmem_dealloc_pair(tmem_base, C::kTmemCols);
    else
      tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

}  // namespace qlora

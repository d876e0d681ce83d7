// libqlora: host side of the C ABI declared in include/qlora.h -- argument checks, TMA tensor maps,
// tile/split planning and kernel launches for the QLoRA NF4 linear layer on sm_100a.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/qlora.h"
#include "elementwise.cuh"
#include "umma_gemm.cuh"

namespace qlora {

// Device error word: bits from ptx.cuh (kDevErr*), read and cleared by ql_get_device_error.
__device__ unsigned int g_dev_error = 0;

namespace {

constexpr int kMaxDevices = 64;

// ------------------------------------------------------------------------------------------ helpers

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct DeviceInfo {
  int sms = 148;
  unsigned int* err = nullptr;
};

std::atomic<uint64_t> g_launches{0};
std::atomic<void*> g_prof_events[2][2] = {};  // [which][start, stop]

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

// Records the caller's profiling event `which` (0 = fused forward GEMM, 1 = fused dX GEMM) if set.
void prof_record(int which, int edge, cudaStream_t stream) {
  void* ev = g_prof_events[which][edge].load(std::memory_order_relaxed);
  if (ev) cudaEventRecord(reinterpret_cast<cudaEvent_t>(ev), stream);
}

DeviceInfo g_dev[kMaxDevices];
bool g_dev_ready[kMaxDevices] = {};
std::mutex g_dev_mu;

// Per-device constants, created on first use on that device (the current one).
bool device_info(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (!g_dev_ready[dev]) {
    DeviceInfo d;
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dev_error) != cudaSuccess) return false;
    d.err = static_cast<unsigned int*>(p);
    g_dev[dev] = d;
    g_dev_ready[dev] = true;
  }
  *out = g_dev[dev];
  return true;
}

// SM count for planning; 148 (B200) when no device is visible (host-only workspace queries).
int plan_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) == cudaSuccess && cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
      sms > 0)
    return sms;
  cudaGetLastError();
  return 148;
}

// ------------------------------------------------------------------------------------------ tensor maps

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Row-major matrix [rows, cols] of 1-, 2- or 4-byte elements; box = box_cols x box_rows.
bool make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int elem_bytes, int box_cols,
              int box_rows, bool swizzle128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t gstride[1] = {static_cast<cuuint64_t>(cols * elem_bytes)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt = elem_bytes == 4   ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                 : elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                   : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  CUresult r = fn(m, dt, 2,
                  const_cast<void*>(base), gdim, gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------------------------------------ GEMM launch

struct Operand {  // a bf16 row-major matrix used through TMA
  const void* ptr = nullptr;
  int64_t rows = 0, cols = 0;
};

struct GemmCall {
  int am = A_TMA_K;
  bool b_mn = false;
  int bn = 64;
  Operand a, b, bx;       // A (TMA modes, or the LoRA extra A), B main, B extra
  const uint8_t* codes = nullptr;
  int64_t rows = 0, cols = 0, k_total = 0;
  int n_extra = 0;
  int kb = 1;             // NF4 blocks per pipeline stage (4 only for token-light A_DEQ_TMEM)
  int splits = 1;
  int prof = -1;          // profiling-event slot recorded around this launch (-1: none)
  int ctas = 148;         // persistent CTAs: at most one per SM
  UmmaArgs args{};
};

template <int BN, int AM, bool BMN, int KB = 1>
cudaError_t launch_umma(const GemmCall& g, cudaStream_t stream) {
  using C = UmmaCfg<BN, AM, BMN, KB>;
  CUtensorMap tmA, tmB, tmBx, tmC;
  std::memset(&tmA, 0, sizeof(tmA));
  std::memset(&tmBx, 0, sizeof(tmBx));
  std::memset(&tmC, 0, sizeof(tmC));
  const bool a_mn = C::kAMN;
  // B main
  if (BMN) {
    if (!make_map(&tmB, g.b.ptr, g.b.rows, g.b.cols, 2, 64, 64, true)) return cudaErrorInvalidValue;
  } else {
    if (!make_map(&tmB, g.b.ptr, g.b.rows, g.b.cols, 2, 64, BN, true)) return cudaErrorInvalidValue;
  }
  // A (TMA modes or LoRA extra)
  if (g.a.ptr) {
    if (a_mn) {
      if (!make_map(&tmA, g.a.ptr, g.a.rows, g.a.cols, 2, 64, 64, true)) return cudaErrorInvalidValue;
    } else {
      if (!make_map(&tmA, g.a.ptr, g.a.rows, g.a.cols, 2, 64, 128, true)) return cudaErrorInvalidValue;
    }
  }
  if (g.bx.ptr) {
    if (!make_map(&tmBx, g.bx.ptr, g.bx.rows, g.bx.cols, 2, 64, BN, true)) return cudaErrorInvalidValue;
  }
  if (C::kAbsTma) {
    // 4-block stages: codes 128 rows x 128 bytes (swizzled), absmax 128 rows x 4 values into tmA
    const int64_t N = g.args.w_rows, K = g.args.w_cols;
    if (!make_map(&tmC, g.codes, N, K / 2, 1, 128, 128, true)) return cudaErrorInvalidValue;
    if (!make_map(&tmA, g.args.absmax, N, K / 64, 4, 4, 128, false)) return cudaErrorInvalidValue;
  } else if (C::kDeq) {
    const int64_t N = g.args.w_rows, K = g.args.w_cols;
    if (AM == A_DEQ_TMEM) {
      if (!make_map(&tmC, g.codes, N, K / 2, 1, 32, 128, false)) return cudaErrorInvalidValue;
    } else {
      if (!make_map(&tmC, g.codes, N, K / 2, 1, 64, 64, false)) return cudaErrorInvalidValue;
    }
  }
  auto kern = umma_gemm_kernel<BN, AM, BMN, KB>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int64_t units = static_cast<int64_t>(g.args.splits) * g.args.tiles_i * g.args.tiles_j;
  dim3 grid(static_cast<unsigned>(std::min<int64_t>(units, g.ctas)));
  if (g.prof >= 0) prof_record(g.prof, 0, stream);
  kern<<<grid, C::kThreads, C::kSmemBytes, stream>>>(tmA, tmB, tmBx, tmC, g.args);
  count_launch();
  if (g.prof >= 0) prof_record(g.prof, 1, stream);
  return cudaGetLastError();
}

template <int AM, bool BMN>
cudaError_t launch_bn(const GemmCall& g, cudaStream_t stream) {
  if constexpr (BMN) {
    switch (g.bn) {
      case 64: return launch_umma<64, AM, BMN>(g, stream);
      case 128: return launch_umma<128, AM, BMN>(g, stream);
      case 256: return launch_umma<256, AM, BMN>(g, stream);
      default: return cudaErrorInvalidValue;
    }
  } else {
    switch (g.bn) {
      case 16: return launch_umma<16, AM, BMN>(g, stream);
      case 32: return launch_umma<32, AM, BMN>(g, stream);
      case 64: return launch_umma<64, AM, BMN>(g, stream);
      case 128: return launch_umma<128, AM, BMN>(g, stream);
      case 256: return launch_umma<256, AM, BMN>(g, stream);
      default: return cudaErrorInvalidValue;
    }
  }
}

cudaError_t launch_gemm(const GemmCall& g, cudaStream_t stream) {
  if (g.am == A_DEQ_TMEM && !g.b_mn && g.kb == 4) {
    switch (g.bn) {
      case 16: return launch_umma<16, A_DEQ_TMEM, false, 4>(g, stream);
      case 32: return launch_umma<32, A_DEQ_TMEM, false, 4>(g, stream);
      case 64: return launch_umma<64, A_DEQ_TMEM, false, 4>(g, stream);
      default: return cudaErrorInvalidValue;
    }
  }
  if (g.kb != 1) return cudaErrorInvalidValue;
  if (g.am == A_DEQ_TMEM && !g.b_mn) return launch_bn<A_DEQ_TMEM, false>(g, stream);
  if (g.am == A_DEQ_MN && !g.b_mn) return launch_bn<A_DEQ_MN, false>(g, stream);
  if (g.am == A_TMA_K && !g.b_mn) return launch_bn<A_TMA_K, false>(g, stream);
  if (g.am == A_TMA_K && g.b_mn) return launch_bn<A_TMA_K, true>(g, stream);
  if (g.am == A_TMA_MN && g.b_mn) return launch_bn<A_TMA_MN, true>(g, stream);
  return cudaErrorInvalidValue;
}

// ------------------------------------------------------------------------------------------ planning

// Rank padded to whole 64-element swizzle atoms: the N of the skinny rank-r products.
int rank_pad(int64_t r) { return r <= 64 ? 64 : r <= 128 ? 128 : 256; }

// Token-tile width of the dequantizing kernels.
int main_bn(int64_t cols) {
  if (cols > 128) return 256;
  if (cols > 64) return 128;
  if (cols > 32) return 64;
  if (cols > 16) return 32;
  return 16;
}

// Split the contraction only while the grid is below one wave; keep >= 4 stages per split.
int plan_splits(int64_t tiles, int64_t kstages, int sms) {
  int s = 1;
  while (tiles * s * 2 <= sms && kstages >= static_cast<int64_t>(s) * 2 * 4 && s < 64) s *= 2;
  return s;
}

// Token-light layers (decode-like, at most 64 tokens) stream the weight once; split the contraction so the
// persistent grid's makespan -- waves of units times stages per unit -- is smallest (at least 8 stages per
// split, at most 8 splits: the fp32 partial sums cost extra traffic).
int plan_splits_streaming(int64_t tiles, int64_t kstages, int sms) {
  int best = 1;
  int64_t best_cost = cdiv(tiles, sms) * kstages;
  for (int s = 2; s <= 8; s *= 2) {
    if (kstages < 8 * s) break;
    const int64_t cost = cdiv(tiles * s, sms) * cdiv(kstages, s);
    if (cost < best_cost) {
      best = s;
      best_cost = cost;
    }
  }
  return best;
}

// NF4 blocks per stage of the fused forward: 4 for token-light layers (short MMAs, so per-stage sync costs
// dominate) when the absmax rows are whole 16-byte TMA boxes (K a multiple of 256), else 1.
int fwd_stage_blocks(int64_t M, int64_t K) { return (main_bn(M) <= 64 && K % 256 == 0) ? 4 : 1; }

struct LinearPlan {
  int bn_main = 16, s_main = 1;      // forward y / backward dX
  int s_su = 1, s_v = 1, s_da = 1, s_db = 1;
  size_t off_su = 0, off_v = 0, off_part = 0, total = 0;
};

// Workspace layout: [su bf16 M x r][v bf16 M x r][fp32 partials (largest user)].
LinearPlan plan_linear(int64_t M, int64_t N, int64_t K, int64_t r, ql_pass pass) {
  LinearPlan p;
  const int sms = plan_sms();
  const int rp = rank_pad(r);
  p.bn_main = main_bn(M);
  const int64_t main_tiles = cdiv(M, p.bn_main) * (pass == QL_PASS_FWD ? cdiv(N, 128) : cdiv(K, 128));
  const int64_t main_kst = pass == QL_PASS_FWD ? cdiv(K, 64 * fwd_stage_blocks(M, K)) : cdiv(N, 64);
  p.s_main = M <= 64 ? plan_splits_streaming(main_tiles, main_kst, sms) : plan_splits(main_tiles, main_kst, sms);
  size_t part = 0;
  if (p.s_main > 1) part = std::max(part, static_cast<size_t>(p.s_main) * M * (pass == QL_PASS_FWD ? N : K) * 4);
  if (r > 0) {
    p.s_su = plan_splits(cdiv(M, 128) * (rp / rp), cdiv(K, 64), sms);
    if (p.s_su > 1) part = std::max(part, static_cast<size_t>(p.s_su) * M * r * 4);
    if (pass == QL_PASS_BWD) {
      p.s_v = plan_splits(cdiv(M, 128), cdiv(N, 64), sms);
      if (p.s_v > 1) part = std::max(part, static_cast<size_t>(p.s_v) * M * r * 4);
      p.s_da = plan_splits(cdiv(K, 128), cdiv(M, 64), sms);
      if (p.s_da > 1) part = std::max(part, static_cast<size_t>(p.s_da) * r * K * 4);
      p.s_db = plan_splits(cdiv(N, 128), cdiv(M, 64), sms);
      if (p.s_db > 1) part = std::max(part, static_cast<size_t>(p.s_db) * N * r * 4);
    }
  }
  size_t off = 0;
  if (r > 0) {
    p.off_su = off;
    off += align256(static_cast<size_t>(M) * r * 2);
    if (pass == QL_PASS_BWD) {
      p.off_v = off;
      off += align256(static_cast<size_t>(M) * r * 2);
    }
  }
  p.off_part = off;
  off += align256(part);
  p.total = (off == 0 || (r == 0 && part == 0)) ? 0 : off;
  return p;
}

cudaError_t launch_reduce(const float* ws, int64_t slab, int nsplit, int64_t count, float alpha, void* out,
                          bool out_bf16, cudaStream_t stream) {
  if (count <= 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = std::min<int64_t>(cdiv(count, threads), 148 * 16);
  reduce_splits_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(ws, slab, nsplit, count, alpha, out,
                                                                              out_bf16 ? 1 : 0);
  count_launch();
  return cudaGetLastError();
}

// Run a GEMM whose output is dense [count] in the final layout: direct when unsplit, else fp32 partials in
// `part` then one reduction.
cudaError_t run_gemm(GemmCall g, void* out, bool out_bf16, float alpha, int64_t ls, int64_t cs, int64_t rows_lim,
                     int64_t cols_lim, int64_t count, float* part, unsigned int* err, cudaStream_t stream) {
  g.ctas = plan_sms();
  g.args.rows = static_cast<int>(g.rows);
  g.args.cols = static_cast<int>(g.cols);
  g.args.tiles_i = static_cast<int>(cdiv(g.rows, 128));
  g.args.tiles_j = static_cast<int>(cdiv(g.cols, g.bn));
  g.args.k_stages = static_cast<int>(cdiv(g.k_total, 64 * g.kb));
  g.args.stages_per_split = static_cast<int>(cdiv(g.args.k_stages, g.splits));
  g.splits = static_cast<int>(cdiv(g.args.k_stages, g.args.stages_per_split));  // no empty splits
  g.args.splits = g.splits;
  g.args.n_extra = g.n_extra;
  g.args.ls = ls;
  g.args.cs = cs;
  g.args.rows_lim = static_cast<int>(rows_lim);
  g.args.cols_lim = static_cast<int>(cols_lim);
  g.args.err = err;
  if (g.splits == 1) {
    g.args.out = out;
    g.args.out_bf16 = out_bf16 ? 1 : 0;
    g.args.alpha = alpha;
    g.args.split_stride = 0;
    return launch_gemm(g, stream);
  }
  g.args.out = part;
  g.args.out_bf16 = 0;
  g.args.alpha = 1.0f;
  g.args.split_stride = count;
  cudaError_t e = launch_gemm(g, stream);
  if (e != cudaSuccess) return e;
  return launch_reduce(part, count, g.splits, count, alpha, out, out_bf16, stream);
}

// su = bf16(s * x A^T) [M, r]
cudaError_t run_su(int64_t M, int64_t K, int64_t r, const uint16_t* x, const uint16_t* A, float s, uint16_t* su,
                   int splits, float* part, unsigned int* err, cudaStream_t stream) {
  GemmCall g;
  g.am = A_TMA_K;
  g.b_mn = false;
  g.bn = rank_pad(r);
  g.a = {x, M, K};
  g.b = {A, r, K};
  g.rows = M;
  g.cols = g.bn;
  g.k_total = K;
  g.splits = splits;
  return run_gemm(g, su, true, s, r, 1, M, r, M * r, part, err, stream);
}

ql_status status_of(cudaError_t e) { return e == cudaSuccess ? QL_OK : QL_ERR_CUDA; }

ql_status check_linear(int64_t M, int64_t N, int64_t K, int64_t r) {
  if (M < 0 || N < 1 || K < 64 || K % 64 != 0 || N % 8 != 0 || r < 0 || r > 256 || r % 8 != 0)
    return QL_ERR_INVALID_ARG;
  if (M > (int64_t(1) << 31) - 1 || N > (int64_t(1) << 31) - 1 || K > (int64_t(1) << 31) - 1) return QL_ERR_INVALID_ARG;
  return QL_OK;
}

}  // namespace
ql_status merge_checks(int64_t N, int64_t K, int64_t r, const uint8_t* codes, const float* absmax, const uint16_t* A,
                       const uint16_t* B) {
  if (N < 1 || K < 64 || K % 64 != 0 || r < 0 || r > 256) return QL_ERR_INVALID_ARG;
  if (N > (int64_t(1) << 31) - 1 || K > (int64_t(1) << 31) - 1) return QL_ERR_INVALID_ARG;
  if (!codes || !absmax || !aligned16(codes) || !aligned16(absmax)) return QL_ERR_INVALID_ARG;
  if (r > 0 && (!A || !B || !aligned16(A) || !aligned16(B))) return QL_ERR_INVALID_ARG;
  return QL_OK;
}

template <int kOut>
ql_status launch_merge(int64_t N, int64_t K, int64_t r, const uint8_t* codes, const float* absmax, const uint16_t* A,
                       const uint16_t* B, float s, void* out, uint8_t* codes_out, float* absmax_out, void* stream) {
  DeviceInfo d;
  if (!device_info(&d)) return QL_ERR_CUDA;
  const long long nblocks = N * K / 64;
  const int threads = 256;  // 8 warps = 8 blocks per CTA iteration
  const long long ctas = std::min<long long>(cdiv(nblocks, 8), static_cast<long long>(d.sms) * 32);
  lora_merge_kernel<kOut><<<static_cast<unsigned>(ctas), threads, 0, as_stream(stream)>>>(
      codes, absmax, A, B, s, nblocks, static_cast<int>(K), static_cast<int>(r), out, codes_out, absmax_out, d.err);
  count_launch();
  return status_of(cudaGetLastError());
}

}  // namespace qlora

using namespace qlora;

extern "C" {

const char* ql_status_string(int status) {
  switch (status) {
    case QL_OK: return "QL_OK";
    case QL_ERR_INVALID_ARG: return "QL_ERR_INVALID_ARG";
    case QL_ERR_UNSUPPORTED: return "QL_ERR_UNSUPPORTED";
    case QL_ERR_CUDA: return "QL_ERR_CUDA";
    case QL_ERR_TIMEOUT: return "QL_ERR_TIMEOUT";
    default: return "QL_ERR_UNKNOWN";
  }
}

int ql_abi_version(void) { return 1; }

uint64_t ql_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

ql_status ql_set_profile_events(int which, void* start, void* stop) {
  if (which < 0 || which > 1) return QL_ERR_INVALID_ARG;
  g_prof_events[which][0].store(start);
  g_prof_events[which][1].store(stop);
  return QL_OK;
}

ql_status ql_selftest_wait_timeout(int64_t wait_cycles, void* stream) {
  if (wait_cycles < 1 || wait_cycles > (int64_t(1) << 32)) return QL_ERR_INVALID_ARG;
  DeviceInfo d;
  if (!device_info(&d)) return QL_ERR_CUDA;
  selftest_wait_kernel<<<1, 32, 0, as_stream(stream)>>>(static_cast<long long>(wait_cycles), d.err);
  count_launch();
  return status_of(cudaGetLastError());
}

void ql_nf4_codebook(float out[16]) {
  for (int i = 0; i < 16; ++i) out[i] = kNF4Levels[i];
}

ql_status ql_get_device_error(void* stream) {
  DeviceInfo d;
  if (!device_info(&d)) return QL_ERR_CUDA;
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return QL_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpy(&v, d.err, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return QL_ERR_CUDA;
  const unsigned int zero = 0;
  if (cudaMemcpy(d.err, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return QL_ERR_CUDA;
  if (v & kDevErrTimeout) return QL_ERR_TIMEOUT;
  if (v & kDevErrNonFinite) return QL_ERR_INVALID_ARG;
  return QL_OK;
}

ql_status nf4_quantize(const float* w, int64_t numel, int blocksize, uint8_t* codes, float* absmax, void* stream) {
  if (numel <= 0 || blocksize <= 0 || numel % blocksize != 0) return QL_ERR_INVALID_ARG;
  if (!w || !codes || !absmax || !aligned16(w) || !aligned16(codes) || !aligned16(absmax)) return QL_ERR_INVALID_ARG;
  if (blocksize != 64) return QL_ERR_UNSUPPORTED;
  DeviceInfo d;
  if (!device_info(&d)) return QL_ERR_CUDA;
  const long long nblocks = numel / 64;
  const int threads = 256;  // 8 warps = 8 blocks per CTA iteration
  const long long ctas = std::min<long long>(cdiv(nblocks, 8), static_cast<long long>(d.sms) * 32);
  nf4_quantize_kernel<<<static_cast<unsigned>(ctas), threads, 0, as_stream(stream)>>>(w, nblocks, codes, absmax, d.err);
  count_launch();
  return status_of(cudaGetLastError());
}

ql_status nf4_dequantize(const uint8_t* codes, const float* absmax, int64_t numel, int blocksize, ql_dtype out_dtype,
                         void* out, void* stream) {
  if (numel <= 0 || blocksize <= 0 || numel % blocksize != 0) return QL_ERR_INVALID_ARG;
  if (!codes || !absmax || !out || !aligned16(codes) || !aligned16(absmax) || !aligned16(out)) return QL_ERR_INVALID_ARG;
  if (out_dtype != QL_F32 && out_dtype != QL_BF16) return QL_ERR_INVALID_ARG;
  if (blocksize != 64) return QL_ERR_UNSUPPORTED;
  DeviceInfo d;
  if (!device_info(&d)) return QL_ERR_CUDA;
  const long long ngroups = numel / 8;
  const int threads = 256;
  const long long ctas = std::min<long long>(cdiv(ngroups, threads), static_cast<long long>(d.sms) * 16);
  if (out_dtype == QL_BF16)
    nf4_dequantize_kernel<true><<<static_cast<unsigned>(ctas), threads, 0, as_stream(stream)>>>(codes, absmax, ngroups, out);
  else
    nf4_dequantize_kernel<false><<<static_cast<unsigned>(ctas), threads, 0, as_stream(stream)>>>(codes, absmax, ngroups, out);
  count_launch();
  return status_of(cudaGetLastError());
}

size_t qlora_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t r, ql_pass pass) {
  if (check_linear(M, N, K, r) != QL_OK || (pass != QL_PASS_FWD && pass != QL_PASS_BWD)) return 0;
  if (M == 0) return 0;
  return plan_linear(M, N, K, r, pass).total;
}

ql_status qlora_linear_fwd(int64_t M, int64_t N, int64_t K, int64_t r, const uint16_t* x, const uint8_t* codes,
                           const float* absmax, const uint16_t* A, const uint16_t* B, float s, uint16_t* y,
                           uint16_t* su_out, void* workspace, size_t ws_bytes, void* stream) {
  ql_status st = check_linear(M, N, K, r);
  if (st != QL_OK) return st;
  if (M == 0) return QL_OK;
  if (!x || !codes || !absmax || !y || !aligned16(x) || !aligned16(codes) || !aligned16(absmax) || !aligned16(y))
    return QL_ERR_INVALID_ARG;
  if (r > 0 && (!A || !B || !aligned16(A) || !aligned16(B))) return QL_ERR_INVALID_ARG;
  if (su_out && !aligned16(su_out)) return QL_ERR_INVALID_ARG;
  const LinearPlan p = plan_linear(M, N, K, r, QL_PASS_FWD);
  if (ws_bytes < p.total || (p.total > 0 && (!workspace || !aligned16(workspace)))) return QL_ERR_INVALID_ARG;
  DeviceInfo d;
  if (!device_info(&d)) return QL_ERR_CUDA;
  cudaStream_t cs = as_stream(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* part = ws ? reinterpret_cast<float*>(ws + p.off_part) : nullptr;

  uint16_t* su = su_out;
  if (r > 0) {
    if (!su) su = reinterpret_cast<uint16_t*>(ws + p.off_su);
    cudaError_t e = run_su(M, K, r, x, A, s, su, p.s_su, part, d.err, cs);
    if (e != cudaSuccess) return QL_ERR_CUDA;
  }
  GemmCall g;
  g.am = A_DEQ_TMEM;
  g.b_mn = false;
  g.bn = p.bn_main;
  g.b = {x, M, K};
  if (r > 0) {
    // the LoRA columns: A extra = rows of B (copied into tensor memory by the kernel), B extra = s x A^T
    g.args.lora = B;
    g.args.lora_ld = static_cast<int>(r);
    g.args.lora_r = static_cast<int>(r);
    g.bx = {su, M, r};
  }
  g.kb = fwd_stage_blocks(M, K);
  if (r > 0) g.n_extra = static_cast<int>(cdiv(r, 64 * g.kb));
  g.codes = codes;
  g.args.absmax = absmax;
  g.args.w_rows = static_cast<int>(N);
  g.args.w_cols = static_cast<int>(K);
  g.args.w_kb = static_cast<int>(K / 64);
  g.rows = N;
  g.cols = M;
  g.k_total = K;
  g.splits = p.s_main;
  g.prof = 0;
  // D[i = n, j = m] -> y[m, n]
  return status_of(run_gemm(g, y, true, 1.0f, 1, N, N, M, M * N, part, d.err, cs));
}

ql_status qlora_linear_bwd(int64_t M, int64_t N, int64_t K, int64_t r, const uint16_t* dy, const uint16_t* x,
                           const uint8_t* codes, const float* absmax, const uint16_t* A, const uint16_t* B, float s,
                           const uint16_t* su_in, uint16_t* dx, float* dA, float* dB, void* workspace, size_t ws_bytes,
                           void* stream) {
  ql_status st = check_linear(M, N, K, r);
  if (st != QL_OK) return st;
  if (!codes || !absmax || !aligned16(codes) || !aligned16(absmax)) return QL_ERR_INVALID_ARG;
  const bool want_da = r > 0 && dA, want_db = r > 0 && dB;
  if ((dx && !aligned16(dx)) || (want_da && !aligned16(dA)) || (want_db && !aligned16(dB))) return QL_ERR_INVALID_ARG;
  if (r > 0 && (!A || !B || !aligned16(A) || !aligned16(B))) return QL_ERR_INVALID_ARG;
  if (su_in && !aligned16(su_in)) return QL_ERR_INVALID_ARG;
  cudaStream_t cs = as_stream(stream);
  if (M == 0) {
    if (want_da && cudaMemsetAsync(dA, 0, static_cast<size_t>(r) * K * 4, cs) != cudaSuccess) return QL_ERR_CUDA;
    if (want_db && cudaMemsetAsync(dB, 0, static_cast<size_t>(N) * r * 4, cs) != cudaSuccess) return QL_ERR_CUDA;
    return QL_OK;
  }
  if (!dy || !aligned16(dy)) return QL_ERR_INVALID_ARG;
  if ((want_da || want_db || (r > 0 && !su_in)) && (!x || !aligned16(x))) return QL_ERR_INVALID_ARG;
  const LinearPlan p = plan_linear(M, N, K, r, QL_PASS_BWD);
  if (ws_bytes < p.total || (p.total > 0 && (!workspace || !aligned16(workspace)))) return QL_ERR_INVALID_ARG;
  DeviceInfo d;
  if (!device_info(&d)) return QL_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* part = ws ? reinterpret_cast<float*>(ws + p.off_part) : nullptr;
  const int rp = rank_pad(r);

  uint16_t* v = nullptr;
  const uint16_t* su = su_in;
  if (r > 0) {
    // su = bf16(s x A^T), recomputed when the forward's copy is not supplied (needed by dB)
    if (!su && want_db) {
      uint16_t* su_ws = reinterpret_cast<uint16_t*>(ws + p.off_su);
      if (run_su(M, K, r, x, A, s, su_ws, p.s_su, part, d.err, cs) != cudaSuccess) return QL_ERR_CUDA;
      su = su_ws;
    }
    // v = bf16(s dY B) [M, r]: D[i = m, j] = sum_n dY[m, n] B[n, j]
    v = reinterpret_cast<uint16_t*>(ws + p.off_v);
    GemmCall g;
    g.am = A_TMA_K;
    g.b_mn = true;
    g.bn = rp;
    g.a = {dy, M, N};
    g.b = {B, N, r};
    g.rows = M;
    g.cols = rp;
    g.k_total = N;
    g.splits = p.s_v;
    if (run_gemm(g, v, true, s, r, 1, M, r, M * r, part, d.err, cs) != cudaSuccess) return QL_ERR_CUDA;
  }
  if (dx) {
    // dX^T: D[i = k, j = m] = sum_n deq(W)[n, k] dY[m, n]  (+ sum_j A[j, k] v[m, j])
    GemmCall g;
    g.am = A_DEQ_MN;
    g.b_mn = false;
    g.bn = p.bn_main;
    g.b = {dy, M, N};
    if (r > 0) {
      // the LoRA rows: A extra = A [r, K] (copied into the MN-major tiles by the kernel), B extra = v
      g.args.lora = A;
      g.args.lora_ld = static_cast<int>(K);
      g.args.lora_r = static_cast<int>(r);
      g.bx = {v, M, r};
      g.n_extra = static_cast<int>(cdiv(r, 64));
    }
    g.codes = codes;
    g.args.absmax = absmax;
    g.args.w_rows = static_cast<int>(N);
    g.args.w_cols = static_cast<int>(K);
    g.args.w_kb = static_cast<int>(K / 64);
    g.rows = K;
    g.cols = M;
    g.k_total = N;
    g.splits = p.s_main;
    g.prof = 1;
    if (run_gemm(g, dx, true, 1.0f, 1, K, K, M, M * K, part, d.err, cs) != cudaSuccess) return QL_ERR_CUDA;
  }
  if (want_da) {
    // dA^T: D[i = k, j] = sum_m x[m, k] v[m, j]  -> dA[j, k]
    GemmCall g;
    g.am = A_TMA_MN;
    g.b_mn = true;
    g.bn = rp;
    g.a = {x, M, K};
    g.b = {v, M, r};
    g.rows = K;
    g.cols = rp;
    g.k_total = M;
    g.splits = p.s_da;
    if (run_gemm(g, dA, false, 1.0f, 1, K, K, r, r * K, part, d.err, cs) != cudaSuccess) return QL_ERR_CUDA;
  }
  if (want_db) {
    // dB: D[i = n, j] = sum_m dY[m, n] su[m, j]
    GemmCall g;
    g.am = A_TMA_MN;
    g.b_mn = true;
    g.bn = rp;
    g.a = {dy, M, N};
    g.b = {su, M, r};
    g.rows = N;
    g.cols = rp;
    g.k_total = M;
    g.splits = p.s_db;
    if (run_gemm(g, dB, false, 1.0f, r, 1, N, r, N * r, part, d.err, cs) != cudaSuccess) return QL_ERR_CUDA;
  }
  return QL_OK;
}

ql_status qlora_merge_lora(int64_t N, int64_t K, int64_t r, const uint8_t* codes, const float* absmax,
                           const uint16_t* A, const uint16_t* B, float s, ql_dtype out_dtype, void* out, void* stream) {
  ql_status st = merge_checks(N, K, r, codes, absmax, A, B);
  if (st != QL_OK) return st;
  if (!out || !aligned16(out)) return QL_ERR_INVALID_ARG;
  if (out_dtype == QL_F32) return launch_merge<0>(N, K, r, codes, absmax, A, B, s, out, nullptr, nullptr, stream);
  if (out_dtype == QL_BF16) return launch_merge<1>(N, K, r, codes, absmax, A, B, s, out, nullptr, nullptr, stream);
  return QL_ERR_INVALID_ARG;
}

ql_status qlora_merge_lora_nf4(int64_t N, int64_t K, int64_t r, const uint8_t* codes, const float* absmax,
                               const uint16_t* A, const uint16_t* B, float s, uint8_t* codes_out, float* absmax_out,
                               void* stream) {
  ql_status st = merge_checks(N, K, r, codes, absmax, A, B);
  if (st != QL_OK) return st;
  if (!codes_out || !absmax_out || !aligned16(codes_out) || !aligned16(absmax_out)) return QL_ERR_INVALID_ARG;
  return launch_merge<2>(N, K, r, codes, absmax, A, B, s, nullptr, codes_out, absmax_out, stream);
}

ql_status qlora_swiglu_fwd(int64_t numel, const uint16_t* g, const uint16_t* u, uint16_t* h, void* stream) {
  if (numel < 0) return QL_ERR_INVALID_ARG;
  if (numel == 0) return QL_OK;
  if (!g || !u || !h) return QL_ERR_INVALID_ARG;
  const int threads = 256;
  const long long ctas = std::min<long long>(cdiv(numel, threads), 148LL * 32);
  swiglu_fwd_kernel<<<static_cast<unsigned>(ctas), threads, 0, as_stream(stream)>>>(
      reinterpret_cast<const __nv_bfloat16*>(g), reinterpret_cast<const __nv_bfloat16*>(u),
      reinterpret_cast<__nv_bfloat16*>(h), numel);
  count_launch();
  return status_of(cudaGetLastError());
}

ql_status qlora_swiglu_bwd(int64_t numel, const uint16_t* dh, const uint16_t* g, const uint16_t* u, uint16_t* dg,
                           uint16_t* du, void* stream) {
  if (numel < 0) return QL_ERR_INVALID_ARG;
  if (numel == 0) return QL_OK;
  if (!dh || !g || !u || !dg || !du) return QL_ERR_INVALID_ARG;
  const int threads = 256;
  const long long ctas = std::min<long long>(cdiv(numel, threads), 148LL * 32);
  swiglu_bwd_kernel<<<static_cast<unsigned>(ctas), threads, 0, as_stream(stream)>>>(
      reinterpret_cast<const __nv_bfloat16*>(dh), reinterpret_cast<const __nv_bfloat16*>(g),
      reinterpret_cast<const __nv_bfloat16*>(u), reinterpret_cast<__nv_bfloat16*>(dg),
      reinterpret_cast<__nv_bfloat16*>(du), numel);
  count_launch();
  return status_of(cudaGetLastError());
}

ql_status qlora_swiglu_gated_fwd(int64_t M, int64_t F, const uint16_t* gu, uint16_t* h, void* stream) {
  if (M < 0 || F < 0 || F % 8 != 0) return QL_ERR_INVALID_ARG;
  if (M == 0 || F == 0) return QL_OK;
  if (!gu || !h || !aligned16(gu) || !aligned16(h)) return QL_ERR_INVALID_ARG;
  const int threads = 256;
  const long long ctas = std::min<long long>(cdiv(M * (F / 8), threads), 148LL * 32);
  swiglu_gated_fwd_kernel<<<static_cast<unsigned>(ctas), threads, 0, as_stream(stream)>>>(
      reinterpret_cast<const __nv_bfloat16*>(gu), reinterpret_cast<__nv_bfloat16*>(h), M, F);
  count_launch();
  return status_of(cudaGetLastError());
}

ql_status qlora_swiglu_gated_bwd(int64_t M, int64_t F, const uint16_t* dh, const uint16_t* gu, uint16_t* dgu,
                                 void* stream) {
  if (M < 0 || F < 0 || F % 8 != 0) return QL_ERR_INVALID_ARG;
  if (M == 0 || F == 0) return QL_OK;
  if (!dh || !gu || !dgu || !aligned16(dh) || !aligned16(gu) || !aligned16(dgu)) return QL_ERR_INVALID_ARG;
  const int threads = 256;
  const long long ctas = std::min<long long>(cdiv(M * (F / 8), threads), 148LL * 32);
  swiglu_gated_bwd_kernel<<<static_cast<unsigned>(ctas), threads, 0, as_stream(stream)>>>(
      reinterpret_cast<const __nv_bfloat16*>(dh), reinterpret_cast<const __nv_bfloat16*>(gu),
      reinterpret_cast<__nv_bfloat16*>(dgu), M, F);
  count_launch();
  return status_of(cudaGetLastError());
}

}  // extern "C"

// ------------------------------------------------------------------------------------------ no-allocation forward
//
// Some callers cannot allocate device memory at all, not even a workspace to lend the library: code that
// runs while a stream is being captured in global mode (where cudaMalloc is an error), or a plug-in hosted
// by a program that owns all device memory and forbids allocations once it has started.  For them
// qlora_linear_fwd_noalloc runs the forward with its scratch in a fixed array compiled into the library.

namespace qlora {
namespace {

constexpr size_t kNoallocScratchBytes = size_t(8) << 20;  // 8 MiB on every device that loads the library

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

// Device address of g_noalloc_scratch per device.  In host code the array's name is only a host-side
// stand-in, so the address is looked up once per device, with that device current.
void* g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

bool noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return false;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return true;
}

}  // namespace
}  // namespace qlora

extern "C" ql_status qlora_linear_fwd_noalloc(int64_t M, int64_t N, int64_t K, int64_t r, const uint16_t* x,
                                              const uint8_t* codes, const float* absmax, const uint16_t* A,
                                              const uint16_t* B, float s, uint16_t* y, uint16_t* su_out,
                                              void* stream) {
  const ql_status st = check_linear(M, N, K, r);
  if (st != QL_OK) return st;
  if (qlora_workspace_bytes(M, N, K, r, QL_PASS_FWD) > kNoallocScratchBytes) return QL_ERR_INVALID_ARG;
  void* scratch = nullptr;
  if (!noalloc_scratch(&scratch)) return QL_ERR_CUDA;
  return qlora_linear_fwd(M, N, K, r, x, codes, absmax, A, B, s, y, su_out, scratch, kNoallocScratchBytes, stream);
}

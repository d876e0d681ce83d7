// libqlora: host side of the C ABI declared in include/qlora.h -- argument checks, TMA tensor maps,
// tile/split planning and kernel launches for the QLoRA NF4 linear layer on sm_100a.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/qlora.h"
#include "elementwise.cuh"
#include "fp4_gemm.cuh"
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
  cudaStream_t side = nullptr;  // second stream for work that runs beside a GEMM (nullptr: none)
};

std::atomic<uint64_t> g_launches{0};
std::atomic<void*> g_prof_events[2][2] = {};  // [which][start, stop]

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

// Records the caller's profiling event `which` (0 = fused forward GEMM, 1 = fused dX GEMM) if set.
void prof_record(int which, int edge, cudaStream_t stream) {
  void* ev = g_prof_events[which][edge].load(std::memory_order_relaxed);
  if (ev) cudaEventRecord(reinterpret_cast<cudaEvent_t>(ev), stream);
}

// Whether events are set for slot `which` (a kernel timed alone is launched the ordinary way).
bool prof_active(int which) {
  return which >= 0 && g_prof_events[which][0].load(std::memory_order_relaxed) != nullptr;
}

int g_dev_sms[kMaxDevices] = {};
cudaStream_t g_dev_side[kMaxDevices] = {};
std::mutex g_dev_mu;

// The current device's SM count (cached per device: a property of the hardware) and the device address of
// the error word.  That address belongs to the current context -- it changes after cudaDeviceReset, and a
// non-primary context has its own copy -- so it is looked up on every call; once the library's module is
// loaded in the context, the lookup allocates nothing.
bool device_info(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (g_dev_sms[dev] <= 0) {
      int sms = 0;
      if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) return false;
      // the side stream takes the lowest priority: the GEMM it runs beside keeps its SMs
      int lowest = 0, highest = 0;
      if (cudaDeviceGetStreamPriorityRange(&lowest, &highest) != cudaSuccess ||
          cudaStreamCreateWithPriority(&g_dev_side[dev], cudaStreamNonBlocking, lowest) != cudaSuccess) {
        g_dev_side[dev] = nullptr;
        cudaGetLastError();
      }
      g_dev_sms[dev] = sms;
    }
    out->sms = g_dev_sms[dev];
    out->side = g_dev_side[dev];
  }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_dev_error) != cudaSuccess || p == nullptr) return false;
  out->err = static_cast<unsigned int*>(p);
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

// Row-major matrix [rows, cols] of 1-, 2- or 4-byte elements; box = box_cols x box_rows, written to shared
// memory with the given swizzle (a box row of 32, 64 or 128 bytes has its 16-byte chunk c at c XOR bits 7.. of its
// shared-memory address).
bool make_map_sw(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int elem_bytes, int box_cols,
                 int box_rows, CUtensorMapSwizzle swizzle) {
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
                  const_cast<void*>(base), gdim, gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int elem_bytes, int box_cols,
              int box_rows, bool swizzle128) {
  return make_map_sw(m, base, rows, cols, elem_bytes, box_cols, box_rows,
                     swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE);
}

// ------------------------------------------------------------------------------------------ GEMM launch

struct Operand {  // a bf16 row-major matrix used through TMA
  const void* ptr = nullptr;
  int64_t rows = 0, cols = 0;
};

// dX through the transposing tensor-memory dequantizer (QLORA_DX_TMEM=1; off by default until measured)
bool dx_tmem_enabled() {
  static const bool on = [] {
    const char* v = std::getenv("QLORA_DX_TMEM");
    return v && v[0] == '1';
  }();
  return on;
}

// Cluster split-K for the skinny rank-r GEMMs (QLORA_CLUSTER_SPLITK=1; off by default until measured)
bool cluster_splitk_enabled() {
  static const bool on = [] {
    const char* v = std::getenv("QLORA_CLUSTER_SPLITK");
    return v && v[0] == '1';
  }();
  return on;
}

// CTA pairs for the 256-token fused GEMMs (QLORA_PAIRS=1; off by default until measured)
bool pairs_enabled() {
  static const bool on = [] {
    const char* v = std::getenv("QLORA_PAIRS");
    return v && v[0] == '1';
  }();
  return on;
}

// Grouped unit order (QLORA_GROUPED=0 turns it off, for comparison)
bool grouped_enabled() {
  static const bool on = [] {
    const char* v = std::getenv("QLORA_GROUPED");
    return !(v && v[0] == '0');
  }();
  return on;
}

struct GemmCall {
  int am = A_TMA_K;
  bool b_mn = false;
  int bn = 64;
  Operand a, b, bx;       // A (TMA modes, or the LoRA extra A), B main, B extra
  const uint8_t* codes = nullptr;
  int64_t rows = 0, cols = 0, k_total = 0;
  int n_extra = 0;
  int kb = 1;             // NF4 blocks per pipeline stage (4 only for token-light A_DEQ_TMEM)
  bool pair = false;      // 2-SM MMA by CTA pairs (256-row tiles, each CTA holding half of the B tile)
  int splits = 1;
  int prof = -1;          // profiling-event slot recorded around this launch (-1: none)
  int ctas = 0;           // persistent CTAs: at most one per SM (0: as many as the GPU has SMs)
  bool streamk = false;   // stream-K schedule (one tile column; fp32 partial slabs reduced afterwards)
  // launched as a programmatic dependent of the kernel before it in the stream: only where that kernel is this
  // library's own and writes only what the GEMM reads after griddep_wait (the LoRA B operand)
  bool pdl = false;
  UmmaArgs args{};
};

// Launch with programmatic stream serialization: the kernel may start while the one before it in the stream runs,
// and waits for it (griddep_wait) before touching its outputs.
template <typename Kern, typename... Args>
cudaError_t launch_dependent(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

template <int BN, int AM, bool BMN, int KB = 1, bool PAIR = false, int WF = WF_NF4, int EPI = EPI_PLAIN>
cudaError_t launch_umma(const GemmCall& g, cudaStream_t stream) {
  using C = UmmaCfg<BN, AM, BMN, KB, PAIR, EPI, WF>;
  CUtensorMap tmA, tmB, tmBx, tmC;
  std::memset(&tmA, 0, sizeof(tmA));
  std::memset(&tmBx, 0, sizeof(tmBx));
  std::memset(&tmC, 0, sizeof(tmC));
  const bool a_mn = C::kAMN;
  // B main
  if (BMN) {
    if (!make_map(&tmB, g.b.ptr, g.b.rows, g.b.cols, 2, 64, 64, true)) return cudaErrorInvalidValue;
  } else {
    if (!make_map(&tmB, g.b.ptr, g.b.rows, g.b.cols, 2, 64, C::kBRows, true)) return cudaErrorInvalidValue;
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
    if (!make_map(&tmBx, g.bx.ptr, g.bx.rows, g.bx.cols, 2, 64, C::kBRows, true)) return cudaErrorInvalidValue;
  }
  if (C::kAbsTma) {
    // 4-block stages: codes 128 rows x 128 bytes (swizzled), absmax 128 rows x 4 values into tmA
    const int64_t N = g.args.w_rows, K = g.args.w_cols;
    if (!make_map(&tmC, g.codes, N, K / 2, 1, 128, 128, true)) return cudaErrorInvalidValue;
    // the stage's scale words (128 rows x 16 bytes) into tmA: the fp32 absmax values or the NVFP4 group scales;
    // the double-quantized constants come by cp.async instead
    if constexpr (WF == WF_NF4) {
      if (!make_map(&tmA, g.args.scale_words, N, K / 64, 4, 4, 128, false)) return cudaErrorInvalidValue;
    } else if constexpr (WF == WF_NVFP4) {
      if (!make_map(&tmA, g.args.scale_words, N, K / 16, 1, 16, 128, false)) return cudaErrorInvalidValue;
    }
  } else if (C::kDeq) {
    const int64_t N = g.args.w_rows, K = g.args.w_cols;
    // codes rows of 32 bytes (forward) or 64 bytes (dX) swizzled so that the dequantizers' 16-byte loads of
    // eight consecutive rows hit eight distinct bank groups; the transposing dequantizer reads single bytes
    if (AM == A_DEQ_TMEM) {
      if (!make_map_sw(&tmC, g.codes, N, K / 2, 1, 32, 128, CU_TENSOR_MAP_SWIZZLE_32B)) return cudaErrorInvalidValue;
    } else if (AM == A_DEQ_MN) {
      if (!make_map_sw(&tmC, g.codes, N, K / 2, 1, 64, 64, CU_TENSOR_MAP_SWIZZLE_64B)) return cudaErrorInvalidValue;
    } else {
      if (!make_map(&tmC, g.codes, N, K / 2, 1, 64, 64, false)) return cudaErrorInvalidValue;
    }
  }
  auto kern = umma_gemm_kernel<BN, AM, BMN, KB, PAIR, WF, EPI>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  // work items that size the grid: units, or with stream-K the stages of the whole sequence
  const int64_t units = g.args.sk_stages > 0 ? static_cast<int64_t>(g.args.tiles_i) * g.args.sk_stages
                                             : static_cast<int64_t>(g.args.splits) * g.args.tiles_i * g.args.tiles_j;
  if constexpr (PAIR) {
    // clusters of two CTAs, each pair walking the units; no more pairs than can be resident at once (a GPC with
    // an odd number of free SMs leaves one idle), so no unit waits for a pair to retire
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(C::kThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(g.ctas & ~1));
    int resident = 0;
    if (cudaOccupancyMaxActiveClusters(&resident, kern, &cfg) != cudaSuccess || resident <= 0) {
      cudaGetLastError();
      resident = g.ctas / 2;
    }
    const int64_t pairs = std::min<int64_t>(units, std::min(resident, g.ctas / 2));
    cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
    if (g.prof >= 0) prof_record(g.prof, 0, stream);
    e = cudaLaunchKernelEx(&cfg, kern, tmA, tmB, tmBx, tmC, g.args);
    if (e != cudaSuccess) return e;
  } else if (!C::kDeq && g.args.cred > 1) {
    // cluster split-K: one CTA per unit, the S splits of a tile in one cluster; every unit must be resident at
    // once (the clusters reduce at the end), else the caller falls back to partial slabs
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(C::kThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(g.args.cred);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(units));
    int resident = 0;
    if (cudaOccupancyMaxActiveClusters(&resident, kern, &cfg) != cudaSuccess || resident <= 0 ||
        static_cast<int64_t>(resident) * g.args.cred < units) {
      cudaGetLastError();
      return cudaErrorCooperativeLaunchTooLarge;
    }
    if (g.prof >= 0) prof_record(g.prof, 0, stream);
    e = cudaLaunchKernelEx(&cfg, kern, tmA, tmB, tmBx, tmC, g.args);
    if (e != cudaSuccess) return e;
  } else {
    dim3 grid(static_cast<unsigned>(std::min<int64_t>(units, g.ctas)));
    if (g.prof >= 0) prof_record(g.prof, 0, stream);
    if (g.pdl && !prof_active(g.prof)) {
      e = launch_dependent(kern, grid, dim3(C::kThreads), C::kSmemBytes, stream, tmA, tmB, tmBx, tmC, g.args);
      if (e != cudaSuccess) return e;
    } else {
      kern<<<grid, C::kThreads, C::kSmemBytes, stream>>>(tmA, tmB, tmBx, tmC, g.args);
    }
  }
  count_launch();
  if (g.prof >= 0) prof_record(g.prof, 1, stream);
  return cudaGetLastError();
}

template <int AM, bool BMN, int WF = WF_NF4>
cudaError_t launch_bn(const GemmCall& g, cudaStream_t stream) {
  if constexpr (BMN) {
    switch (g.bn) {
      case 64: return launch_umma<64, AM, BMN, 1, false, WF>(g, stream);
      case 128: return launch_umma<128, AM, BMN, 1, false, WF>(g, stream);
      case 256: return launch_umma<256, AM, BMN, 1, false, WF>(g, stream);
      default: return cudaErrorInvalidValue;
    }
  } else {
    switch (g.bn) {
      case 16: return launch_umma<16, AM, BMN, 1, false, WF>(g, stream);
      case 32: return launch_umma<32, AM, BMN, 1, false, WF>(g, stream);
      case 64: return launch_umma<64, AM, BMN, 1, false, WF>(g, stream);
      case 128: return launch_umma<128, AM, BMN, 1, false, WF>(g, stream);
      case 256: return launch_umma<256, AM, BMN, 1, false, WF>(g, stream);
      default: return cudaErrorInvalidValue;
    }
  }
}

// The dequantizing GEMMs, by weight format.
template <int WF>
cudaError_t launch_deq(const GemmCall& g, cudaStream_t stream) {
  if (g.pair) {
    if (g.bn != 256 || g.b_mn || g.kb != 1) return cudaErrorInvalidValue;
    if (g.am == A_DEQ_TMEM) return launch_umma<256, A_DEQ_TMEM, false, 1, true, WF>(g, stream);
    if (g.am == A_DEQ_MN) return launch_umma<256, A_DEQ_MN, false, 1, true, WF>(g, stream);
    if constexpr (WF == WF_NF4) {
      if (g.am == A_DEQ_TMEM_T) return launch_umma<256, A_DEQ_TMEM_T, false, 1, true, WF>(g, stream);
    }
    return cudaErrorInvalidValue;
  }
  if (g.am == A_DEQ_TMEM && !g.b_mn && g.kb == 4) {
    switch (g.bn) {
      case 16: return launch_umma<16, A_DEQ_TMEM, false, 4, false, WF>(g, stream);
      case 32: return launch_umma<32, A_DEQ_TMEM, false, 4, false, WF>(g, stream);
      case 64: return launch_umma<64, A_DEQ_TMEM, false, 4, false, WF>(g, stream);
      default: return cudaErrorInvalidValue;
    }
  }
  if (g.kb != 1) return cudaErrorInvalidValue;
  if (g.am == A_DEQ_TMEM && !g.b_mn) return launch_bn<A_DEQ_TMEM, false, WF>(g, stream);
  if (g.am == A_DEQ_MN && !g.b_mn) return launch_bn<A_DEQ_MN, false, WF>(g, stream);
  if constexpr (WF == WF_NF4) {
    if (g.am == A_DEQ_TMEM_T && !g.b_mn) return launch_bn<A_DEQ_TMEM_T, false, WF>(g, stream);
  }
  return cudaErrorInvalidValue;
}

// The fused gated-MLP epilogues (NF4 weights): the gate/up forward (TMEM A) and the down projection's dX (MN A).
template <int AM, int EPI>
cudaError_t launch_epi(const GemmCall& g, cudaStream_t stream) {
  switch (g.bn) {
    case 16: return launch_umma<16, AM, false, 1, false, WF_NF4, EPI>(g, stream);
    case 32: return launch_umma<32, AM, false, 1, false, WF_NF4, EPI>(g, stream);
    case 64: return launch_umma<64, AM, false, 1, false, WF_NF4, EPI>(g, stream);
    case 128: return launch_umma<128, AM, false, 1, false, WF_NF4, EPI>(g, stream);
    case 256: return launch_umma<256, AM, false, 1, false, WF_NF4, EPI>(g, stream);
    default: return cudaErrorInvalidValue;
  }
}

// One-shot failure-path test (ql_selftest_arm_gemm_stall): the next dequantizing GEMM launch carries it.
std::atomic<int> g_test_stall{0};
std::atomic<long long> g_test_wait{0};

cudaError_t launch_gemm_impl(const GemmCall& g, cudaStream_t stream);

cudaError_t launch_gemm(const GemmCall& g, cudaStream_t stream) {
  if ((g.am == A_DEQ_TMEM || g.am == A_DEQ_MN || g.am == A_DEQ_TMEM_T) && g_test_stall.load() != 0) {
    const int role = g_test_stall.exchange(0);
    if (role != 0) {
      GemmCall t = g;
      t.args.test_stall = role;
      t.args.wait_limit = g_test_wait.load();
      return launch_gemm_impl(t, stream);
    }
  }
  return launch_gemm_impl(g, stream);
}

cudaError_t launch_gemm_impl(const GemmCall& g, cudaStream_t stream) {
  if (g.args.epi != EPI_PLAIN) {
    if (g.args.splits != 1 || g.kb != 1 || g.b_mn || g.pair || g.args.wfmt != WF_NF4) return cudaErrorInvalidValue;
    if (g.args.epi == EPI_SWIGLU_FWD && g.am == A_DEQ_TMEM) return launch_epi<A_DEQ_TMEM, EPI_SWIGLU_FWD>(g, stream);
    if (g.args.epi == EPI_DSWIGLU && g.am == A_DEQ_MN) return launch_epi<A_DEQ_MN, EPI_DSWIGLU>(g, stream);
    return cudaErrorInvalidValue;
  }
  if (g.am == A_DEQ_TMEM || g.am == A_DEQ_MN || g.am == A_DEQ_TMEM_T) {
    switch (g.args.wfmt) {
      case WF_NF4: return launch_deq<WF_NF4>(g, stream);
      case WF_NF4_DQ: return launch_deq<WF_NF4_DQ>(g, stream);
      case WF_NVFP4: return launch_deq<WF_NVFP4>(g, stream);
      default: return cudaErrorInvalidValue;
    }
  }
  if (g.kb != 1) return cudaErrorInvalidValue;
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

// Token-light layers with few s x A^T outputs take them from CUDA cores (su_small_kernel).
bool su_on_cores(int64_t M, int64_t r) { return M <= 64 && M * r <= 512; }

struct LinearPlan {
  int bn_main = 16, s_main = 1;      // forward y / backward dX
  int sk_ctas = 0, sk_slabs = 0;     // stream-K forward: CTAs and partial slabs (0: split plan)
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
  if (pass == QL_PASS_FWD && M <= 64) {
    // token-light forward: a stream-K schedule balances the stages exactly (each CTA gets T / P of them, at
    // least 4) where whole split units would leave the last wave partly empty
    const int64_t T = main_tiles * main_kst;
    const int64_t P = std::min<int64_t>(sms, cdiv(T, 4));
    const int64_t split_cost = cdiv(main_tiles * p.s_main, sms) * cdiv(main_kst, p.s_main);
    if (main_kst >= 8 && cdiv(T, P) < split_cost) {
      p.sk_ctas = static_cast<int>(P);
      for (int64_t t = 0; t < main_tiles; ++t)
        p.sk_slabs = std::max<int>(p.sk_slabs, static_cast<int>(sk_cta_of(t * main_kst + main_kst - 1, T, P) -
                                                                 sk_cta_of(t * main_kst, T, P) + 1));
      p.s_main = 1;
      part = std::max(part, static_cast<size_t>(p.sk_slabs) * M * N * 4);
    }
  }
  if (p.s_main > 1) part = std::max(part, static_cast<size_t>(p.s_main) * M * (pass == QL_PASS_FWD ? N : K) * 4);
  if (r > 0) {
    p.s_su = su_on_cores(M, r) ? 1 : plan_splits(cdiv(M, 128) * (rp / rp), cdiv(K, 64), sms);
    if (pass == QL_PASS_FWD && !su_on_cores(M, r) && p.sk_slabs == 0) {
      // The fused GEMM starts while s x A^T runs; its CTAs on the SMs that s x A^T holds start late.  When the
      // unsplit s x A^T needs no more CTAs than the fused GEMM has CTAs with one unit fewer than the rest, those
      // late CTAs are exactly the short ones and the fused GEMM ends no later: run s x A^T unsplit.
      const int64_t units = main_tiles * p.s_main;
      const int64_t short_ctas = units % sms == 0 ? 0 : sms - units % sms;
      if (units > sms && cdiv(M, 128) <= short_ctas) p.s_su = 1;
    }
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

// The split-K reduction of a GEMM's partials, launched as a dependent of that GEMM (it waits for it first).
cudaError_t launch_reduce(const float* ws, int64_t slab, int nsplit, int64_t count, float alpha, void* out,
                          bool out_bf16, cudaStream_t stream) {
  if (count <= 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = std::min<int64_t>(cdiv(count, threads), 148 * 16);
  const cudaError_t e = launch_dependent(reduce_splits_kernel, dim3(static_cast<unsigned>(blocks)), dim3(threads), 0,
                                         stream, ws, static_cast<long long>(slab), nsplit,
                                         static_cast<long long>(count), alpha, out, out_bf16 ? 1 : 0);
  if (e != cudaSuccess) return e;
  count_launch();
  return cudaGetLastError();
}

// CTAs that give a persistent GEMM of `units` work units (`per_unit` CTAs each) the makespan it has on the whole
// GPU: it takes ceil(units * per_unit / sms) waves either way, and with ceil(units / waves) units in flight its
// last wave is as full as the others.  The SMs this leaves free can run other work in the meantime.
int wave_exact_ctas(int64_t units, int per_unit, int sms) {
  const int64_t slots = std::max<int64_t>(1, sms / per_unit);
  const int64_t waves = cdiv(units, slots);
  return static_cast<int>(cdiv(units, waves) * per_unit);
}

// Run a GEMM whose output is dense [count] in the final layout: direct when unsplit, else fp32 partials in
// `part` then one reduction.
// Tile rows per group of the unit order (0: tile columns fastest).  A wave of C concurrent units covering g tile
// rows and C / g tile columns fetches about g weight tiles and C / g activation tiles; with w and a the bytes of
// one of each (both proportional to the contraction length), g w + (C / g) a is smallest at g = sqrt(C a / w).
// Grids of one wave, and outputs one tile column wide, keep the plain order.
int unit_group(const GemmCall& g) {
  if (!grouped_enabled() || g.args.tiles_j <= 1) return 0;
  const int64_t concurrent = g.pair ? g.ctas / 2 : g.ctas;
  const int64_t units = static_cast<int64_t>(g.args.splits) * g.args.tiles_i * g.args.tiles_j;
  if (units <= concurrent) return 0;
  const bool deq = g.am == A_DEQ_TMEM || g.am == A_DEQ_MN || g.am == A_DEQ_TMEM_T;
  const double w_row_bytes = deq ? 0.5625 : 2.0;  // one weight row element: 4-bit code + its share of the scale
  const double ratio = (g.bn * 2.0) / ((g.pair ? 256.0 : 128.0) * w_row_bytes);
  int gi = static_cast<int>(std::lround(std::sqrt(static_cast<double>(concurrent) * ratio)));
  if (gi < 1) gi = 1;
  if (gi > g.args.tiles_i) gi = g.args.tiles_i;
  return gi;
}

cudaError_t run_gemm(GemmCall g, void* out, bool out_bf16, float alpha, int64_t ls, int64_t cs, int64_t rows_lim,
                     int64_t cols_lim, int64_t count, float* part, unsigned int* err, cudaStream_t stream) {
  if (g.ctas <= 0) g.ctas = plan_sms();
  g.args.rows = static_cast<int>(g.rows);
  g.args.cols = static_cast<int>(g.cols);
  g.args.tiles_i = static_cast<int>(cdiv(g.rows, g.pair ? 256 : 128));
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
  g.args.group_i = unit_group(g);
  if (g.streamk) {
    // stream-K: every unit writes its fp32 partial to the slab of its place among the CTAs sharing its tile,
    // then one reduction sums each tile's slabs in that order (D rows must be the fastest output index)
    if (ls != 1 || g.args.tiles_j != 1 || !part) return cudaErrorInvalidValue;
    const int64_t T = static_cast<int64_t>(g.args.tiles_i) * g.args.k_stages;
    g.ctas = static_cast<int>(std::min<int64_t>(g.ctas, T));
    g.args.sk_stages = g.args.k_stages;
    g.args.group_i = 0;
    g.args.out = part;
    g.args.out_bf16 = 0;
    g.args.alpha = 1.0f;
    g.args.split_stride = count;
    cudaError_t e = launch_gemm(g, stream);
    if (e != cudaSuccess) return e;
    const int threads = 256;
    const int64_t blocks = std::min<int64_t>(cdiv(count, threads), 148 * 16);
    e = launch_dependent(reduce_streamk_kernel, dim3(static_cast<unsigned>(blocks)), dim3(threads), 0, stream,
                         static_cast<const float*>(part), static_cast<long long>(count), static_cast<long long>(count),
                         static_cast<long long>(cs), static_cast<long long>(g.args.k_stages),
                         static_cast<long long>(T), static_cast<long long>(g.ctas), alpha, out, out_bf16 ? 1 : 0);
    if (e != cudaSuccess) return e;
    count_launch();
    return cudaGetLastError();
  }
  if (g.splits == 1) {
    g.args.out = out;
    g.args.out_bf16 = out_bf16 ? 1 : 0;
    g.args.alpha = alpha;
    g.args.split_stride = 0;
    return launch_gemm(g, stream);
  }
  const bool tma_mode = g.am == A_TMA_K || g.am == A_TMA_MN;
  if (tma_mode && g.splits <= 8 && 128 % g.splits == 0 && cluster_splitk_enabled() &&
      static_cast<int64_t>(g.splits) * g.args.tiles_i * g.args.tiles_j <= g.ctas) {
    // the splits of a tile reduce inside their cluster: no slabs, no second launch
    GemmCall c = g;
    c.args.cred = g.splits;
    c.args.out = out;
    c.args.out_bf16 = out_bf16 ? 1 : 0;
    c.args.alpha = alpha;
    c.args.split_stride = 0;
    const cudaError_t e = launch_gemm(c, stream);
    if (e != cudaErrorCooperativeLaunchTooLarge) return e;
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
  if (su_on_cores(M, r)) {
    const int64_t warps = M * r;
    su_small_kernel<<<static_cast<unsigned>(cdiv(warps, 2)), 64, 0, stream>>>(x, A, static_cast<int>(M),
                                                                             static_cast<int>(K), static_cast<int>(r),
                                                                             s, su);
    count_launch();
    return cudaGetLastError();
  }
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

// The kernel's view of a weight descriptor: its format and the pointers that format uses.
void set_weight(UmmaArgs& a, const ql_weight& w) {
  a.wfmt = w.format == QL_W_NF4_DQ ? WF_NF4_DQ : w.format == QL_W_NVFP4 ? WF_NVFP4 : WF_NF4;
  a.scale_words = w.format == QL_W_NF4_DQ ? static_cast<const void*>(w.code8)
                  : w.format == QL_W_NVFP4 ? static_cast<const void*>(w.scales)
                                           : static_cast<const void*>(w.absmax);
  a.dq_c1 = w.c1;
  a.dq_mu = w.mu;
  a.fp4_S = w.tensor_scale;
}

ql_status check_weight(const ql_weight* w) {
  if (!w || !w->codes || !aligned16(w->codes)) return QL_ERR_INVALID_ARG;
  switch (w->format) {
    case QL_W_NF4:
      return w->absmax && aligned16(w->absmax) ? QL_OK : QL_ERR_INVALID_ARG;
    case QL_W_NF4_DQ:
      return w->code8 && w->c1 && w->mu && aligned16(w->code8) && aligned16(w->c1) && aligned16(w->mu)
                 ? QL_OK
                 : QL_ERR_INVALID_ARG;
    case QL_W_NVFP4:
      return w->scales && w->tensor_scale && aligned16(w->scales) && aligned16(w->tensor_scale) ? QL_OK
                                                                                               : QL_ERR_INVALID_ARG;
    default:
      return QL_ERR_INVALID_ARG;
  }
}

ql_weight nf4_weight(const uint8_t* codes, const float* absmax) {
  ql_weight w = {};
  w.format = QL_W_NF4;
  w.codes = codes;
  w.absmax = absmax;
  return w;
}

// A fused epilogue for the main GEMM of a layer call (Epi in umma_gemm.cuh).
struct EpiArgs {
  int mode = EPI_PLAIN;
  void* out2 = nullptr;
  int64_t ls2 = 0, cs2 = 0;
  const uint16_t* aux = nullptr;
  int64_t aux_ld = 0;
};

ql_status linear_fwd_impl(int64_t M, int64_t N, int64_t K, int64_t r, const uint16_t* x, const ql_weight* w,
                          const uint16_t* A, const uint16_t* B, float s, uint16_t* y, uint16_t* su_out,
                          void* workspace, size_t ws_bytes, void* stream, const EpiArgs* epi) {
  ql_status st = check_linear(M, N, K, r);
  if (st != QL_OK) return st;
  if (check_weight(w) != QL_OK) return QL_ERR_INVALID_ARG;
  const ql_weight& wt = *w;
  if (M == 0) return QL_OK;
  if (!x || !y || !aligned16(x) || !aligned16(y)) return QL_ERR_INVALID_ARG;
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
  g.pair = g.bn == 256 && g.kb == 1 && !epi && pairs_enabled();
  if (r > 0) g.n_extra = static_cast<int>(cdiv(r, 64 * g.kb));
  g.codes = wt.codes;
  set_weight(g.args, wt);
  g.args.w_rows = static_cast<int>(N);
  g.args.w_cols = static_cast<int>(K);
  g.args.w_kb = static_cast<int>(K / 64);
  g.rows = N;
  g.cols = M;
  g.k_total = K;
  g.splits = p.s_main;
  if (p.sk_slabs > 0 && !epi) {
    g.streamk = true;
    g.ctas = p.sk_ctas;
  }
  // after this library's s x A^T kernels, the fused GEMM starts early: it reads their output (its LoRA B operand)
  // and writes its own (which may share the workspace with their partials) only after griddep_wait
  g.pdl = r > 0;
  g.prof = 0;
  if (epi) {
    g.args.epi = epi->mode;
    g.args.out2 = epi->out2;
    g.args.ls2 = epi->ls2;
    g.args.cs2 = epi->cs2;
  }
  // D[i = n, j = m] -> y[m, n]
  return status_of(run_gemm(g, y, true, 1.0f, 1, N, N, M, M * N, part, d.err, cs));
}

ql_status linear_bwd_impl(int64_t M, int64_t N, int64_t K, int64_t r, const uint16_t* dy, const uint16_t* x,
                          const ql_weight* w, const uint16_t* A, const uint16_t* B, float s, const uint16_t* su_in,
                          uint16_t* dx, float* dA, float* dB, void* workspace, size_t ws_bytes, void* stream,
                          const EpiArgs* epi) {
  ql_status st = check_linear(M, N, K, r);
  if (st != QL_OK) return st;
  if (check_weight(w) != QL_OK) return QL_ERR_INVALID_ARG;
  const ql_weight& wt = *w;
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
  // dA and dB do not depend on dX: when the dX GEMM (unsplit) would leave its last wave partly empty, it runs
  // on the fewest CTAs that keep its makespan, and dA, dB run beside it on the SMs it leaves free, on the
  // device's side stream (forked from and joined back into the caller's stream).
  const bool dx_pair = p.bn_main == 256 && !epi && pairs_enabled();
  int dx_ctas = 0, side_sms = 0;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
  if (dx && (want_da || want_db) && p.s_main == 1 && d.side) {
    const int64_t units = cdiv(K, dx_pair ? 256 : 128) * cdiv(M, p.bn_main);
    dx_ctas = wave_exact_ctas(units, dx_pair ? 2 : 1, d.sms);
    side_sms = d.sms - dx_ctas;
    if (side_sms >= 8 && cudaEventCreateWithFlags(&ev_fork, cudaEventDisableTiming) == cudaSuccess &&
        cudaEventCreateWithFlags(&ev_join, cudaEventDisableTiming) == cudaSuccess &&
        cudaEventRecord(ev_fork, cs) == cudaSuccess && cudaStreamWaitEvent(d.side, ev_fork, 0) == cudaSuccess) {
      // forked
    } else {
      if (ev_fork) cudaEventDestroy(ev_fork);
      if (ev_join) cudaEventDestroy(ev_join);
      ev_fork = ev_join = nullptr;
      dx_ctas = side_sms = 0;
      cudaGetLastError();
    }
  }
  // on an error after the fork: release the events (they go once their work has run) and report
  auto unfork = [&]() {
    if (ev_fork) cudaEventDestroy(ev_fork);
    if (ev_join) cudaEventDestroy(ev_join);
    return QL_ERR_CUDA;
  };
  const bool beside = side_sms > 0;
  cudaStream_t gs = beside ? d.side : cs;  // the stream of dA and dB
  if (dx) {
    // dX^T: D[i = k, j = m] = sum_n deq(W)[n, k] dY[m, n]  (+ sum_j A[j, k] v[m, j])
    GemmCall g;
    // the transposing TMEM dequantizer when enabled (NF4 weights, plain epilogue, single CTAs)
    g.am = dx_tmem_enabled() && !epi && wt.format == QL_W_NF4 ? A_DEQ_TMEM_T : A_DEQ_MN;
    g.b_mn = false;
    g.bn = p.bn_main;
    g.pair = dx_pair;
    g.ctas = dx_ctas;
    g.b = {dy, M, N};
    if (r > 0) {
      // the LoRA rows: A extra = A [r, K] (copied into the MN-major tiles by the kernel), B extra = v
      g.args.lora = A;
      g.args.lora_ld = static_cast<int>(K);
      g.args.lora_r = static_cast<int>(r);
      g.bx = {v, M, r};
      g.n_extra = static_cast<int>(cdiv(r, 64));
    }
    g.codes = wt.codes;
    set_weight(g.args, wt);
    g.args.w_rows = static_cast<int>(N);
    g.args.w_cols = static_cast<int>(K);
    g.args.w_kb = static_cast<int>(K / 64);
    g.rows = K;
    g.cols = M;
    g.k_total = N;
    g.splits = p.s_main;
    g.prof = 1;
    // after this library's v kernels, dX starts early: it reads v (its LoRA B operand, in the stages after its
    // first unit's main stages) and writes its output only after griddep_wait
    g.pdl = r > 0;
    if (epi) {
      g.args.epi = epi->mode;
      g.args.out2 = epi->out2;
      g.args.aux = epi->aux;
      g.args.aux_ld = epi->aux_ld;
    }
    if (run_gemm(g, dx, true, 1.0f, 1, K, K, M, M * K, part, d.err, cs) != cudaSuccess) return unfork();
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
    g.splits = beside ? plan_splits(cdiv(K, 128), cdiv(M, 64), side_sms) : p.s_da;
    g.ctas = side_sms;
    if (run_gemm(g, dA, false, 1.0f, 1, K, K, r, r * K, part, d.err, gs) != cudaSuccess) return unfork();
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
    g.splits = beside ? plan_splits(cdiv(N, 128), cdiv(M, 64), side_sms) : p.s_db;
    g.ctas = side_sms;
    if (run_gemm(g, dB, false, 1.0f, r, 1, N, r, N * r, part, d.err, gs) != cudaSuccess) return unfork();
  }
  if (beside) {
    // join: the caller's stream continues once dA and dB are done; the events go once they have fired
    const bool ok = cudaEventRecord(ev_join, gs) == cudaSuccess && cudaStreamWaitEvent(cs, ev_join, 0) == cudaSuccess;
    cudaEventDestroy(ev_fork);
    cudaEventDestroy(ev_join);
    if (!ok) return QL_ERR_CUDA;
  }
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

ql_status ql_selftest_arm_gemm_stall(int role, int64_t wait_cycles) {
  if (role < 1 || role > 3 || wait_cycles < 100000 || wait_cycles > (int64_t(1) << 32)) return QL_ERR_INVALID_ARG;
  g_test_wait.store(wait_cycles);
  g_test_stall.store(role);
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
  const int threads = 256;  // 8 warps, each taking kQuantBlocksPerStep blocks per step
  const long long ctas =
      std::min<long long>(cdiv(nblocks, 8 * kQuantBlocksPerStep), static_cast<long long>(d.sms) * 16);
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
  const long long nhalves = numel / 32;  // 32 elements (16 code bytes) per thread
  const int threads = 256;
  const long long ctas = std::min<long long>(cdiv(nhalves, threads), static_cast<long long>(d.sms) * 8);
  if (out_dtype == QL_BF16)
    nf4_dequantize_kernel<true><<<static_cast<unsigned>(ctas), threads, 0, as_stream(stream)>>>(codes, absmax, nhalves, out);
  else
    nf4_dequantize_kernel<false><<<static_cast<unsigned>(ctas), threads, 0, as_stream(stream)>>>(codes, absmax, nhalves, out);
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
  const ql_weight w = nf4_weight(codes, absmax);
  return linear_fwd_impl(M, N, K, r, x, &w, A, B, s, y, su_out, workspace, ws_bytes, stream, nullptr);
}

ql_status qlora_linear_fwd_w(int64_t M, int64_t N, int64_t K, int64_t r, const uint16_t* x, const ql_weight* w,
                             const uint16_t* A, const uint16_t* B, float s, uint16_t* y, uint16_t* su_out,
                             void* workspace, size_t ws_bytes, void* stream) {
  return linear_fwd_impl(M, N, K, r, x, w, A, B, s, y, su_out, workspace, ws_bytes, stream, nullptr);
}

ql_status qlora_linear_bwd(int64_t M, int64_t N, int64_t K, int64_t r, const uint16_t* dy, const uint16_t* x,
                           const uint8_t* codes, const float* absmax, const uint16_t* A, const uint16_t* B, float s,
                           const uint16_t* su_in, uint16_t* dx, float* dA, float* dB, void* workspace, size_t ws_bytes,
                           void* stream) {
  const ql_weight w = nf4_weight(codes, absmax);
  return linear_bwd_impl(M, N, K, r, dy, x, &w, A, B, s, su_in, dx, dA, dB, workspace, ws_bytes, stream, nullptr);
}

ql_status qlora_linear_bwd_w(int64_t M, int64_t N, int64_t K, int64_t r, const uint16_t* dy, const uint16_t* x,
                             const ql_weight* w, const uint16_t* A, const uint16_t* B, float s, const uint16_t* su_in,
                             uint16_t* dx, float* dA, float* dB, void* workspace, size_t ws_bytes, void* stream) {
  return linear_bwd_impl(M, N, K, r, dy, x, w, A, B, s, su_in, dx, dA, dB, workspace, ws_bytes, stream, nullptr);
}

// Extra workspace of the gated calls: a dh buffer [M, F] bf16 when the down projection's dX GEMM splits its
// contraction (the fused epilogue then cannot run, and dSwiGLU follows as its own kernel).
size_t gated_dh_bytes(int64_t M, int64_t N, int64_t F, int64_t r) {
  return plan_linear(M, N, F, r, QL_PASS_BWD).s_main > 1 ? align256(static_cast<size_t>(M) * F * 2) : 0;
}

size_t qlora_gated_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t r, ql_pass pass) {
  if (pass == QL_PASS_FWD) return qlora_workspace_bytes(M, N, K, r, pass);
  const size_t base = align256(qlora_workspace_bytes(M, N, K, r, pass));
  return M > 0 && check_linear(M, N, K, r) == QL_OK ? base + gated_dh_bytes(M, N, K, r) : 0;
}

ql_status qlora_gate_up_fwd_swiglu(int64_t M, int64_t F, int64_t K, int64_t r, const uint16_t* x, const uint8_t* codes,
                                   const float* absmax, const uint16_t* A, const uint16_t* B, float s, uint16_t* gu,
                                   uint16_t* h, uint16_t* su_out, void* workspace, size_t ws_bytes, void* stream) {
  if (F <= 0 || F % 16 != 0 || !h || !aligned16(h)) return QL_ERR_INVALID_ARG;
  const int64_t N = 2 * F;
  const ql_weight w = nf4_weight(codes, absmax);
  if (check_linear(M, N, K, r) != QL_OK) return QL_ERR_INVALID_ARG;
  // the fused epilogue runs in unsplit GEMMs with one-block stages; token-light layers (4-block stages or a
  // stream-K schedule) and split contractions write gu first and run the SwiGLU as its own kernel
  const LinearPlan pl = M > 0 ? plan_linear(M, N, K, r, QL_PASS_FWD) : LinearPlan{};
  if (M > 0 && pl.s_main == 1 && pl.sk_slabs == 0 && fwd_stage_blocks(M, K) == 1) {
    EpiArgs e;
    e.mode = EPI_SWIGLU_FWD;
    e.out2 = h;
    e.ls2 = 1;
    e.cs2 = F;
    return linear_fwd_impl(M, N, K, r, x, &w, A, B, s, gu, su_out, workspace, ws_bytes, stream, &e);
  }
  ql_status st = linear_fwd_impl(M, N, K, r, x, &w, A, B, s, gu, su_out, workspace, ws_bytes, stream, nullptr);
  if (st != QL_OK || M == 0) return st;
  DeviceInfo d;
  if (!device_info(&d)) return QL_ERR_CUDA;
  const long long groups = M * (F / 8);
  const long long ctas = std::min<long long>(cdiv(groups, 256), static_cast<long long>(d.sms) * 16);
  swiglu_interleaved_fwd_kernel<<<static_cast<unsigned>(ctas), 256, 0, as_stream(stream)>>>(
      reinterpret_cast<const __nv_bfloat16*>(gu), reinterpret_cast<__nv_bfloat16*>(h), M, F);
  count_launch();
  return status_of(cudaGetLastError());
}

ql_status qlora_down_bwd_dswiglu(int64_t M, int64_t N, int64_t F, int64_t r, const uint16_t* dy, const uint16_t* h,
                                 const uint8_t* codes, const float* absmax, const uint16_t* A, const uint16_t* B,
                                 float s, const uint16_t* su, const uint16_t* gu, uint16_t* dgu, float* dA, float* dB,
                                 void* workspace, size_t ws_bytes, void* stream) {
  if (F <= 0 || F % 16 != 0 || !gu || !dgu || !aligned16(gu) || !aligned16(dgu)) return QL_ERR_INVALID_ARG;
  const ql_weight w = nf4_weight(codes, absmax);
  if (check_linear(M, N, F, r) != QL_OK) return QL_ERR_INVALID_ARG;
  if (ws_bytes < qlora_gated_workspace_bytes(M, N, F, r, QL_PASS_BWD)) return QL_ERR_INVALID_ARG;
  const size_t dh_bytes = M > 0 ? gated_dh_bytes(M, N, F, r) : 0;
  if (dh_bytes == 0) {
    EpiArgs e;
    e.mode = EPI_DSWIGLU;
    e.out2 = dgu;
    e.aux = gu;
    e.aux_ld = 2 * F;
    // dx is only the switch that runs the dX GEMM: its epilogue writes dgu and never dx
    return linear_bwd_impl(M, N, F, r, dy, h, &w, A, B, s, su, dgu, dA, dB, workspace, ws_bytes, stream, &e);
  }
  // the layer's own workspace first, then the dh buffer (ws_bytes covers both, checked above)
  if (!workspace || !aligned16(workspace)) return QL_ERR_INVALID_ARG;
  const size_t base = align256(qlora_workspace_bytes(M, N, F, r, QL_PASS_BWD));
  uint16_t* dh = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(workspace) + base);
  ql_status st = linear_bwd_impl(M, N, F, r, dy, h, &w, A, B, s, su, dh, dA, dB, workspace, base, stream, nullptr);
  if (st != QL_OK) return st;
  DeviceInfo d;
  if (!device_info(&d)) return QL_ERR_CUDA;
  const long long groups = M * (F / 8);
  const long long ctas = std::min<long long>(cdiv(groups, 256), static_cast<long long>(d.sms) * 16);
  swiglu_interleaved_bwd_kernel<<<static_cast<unsigned>(ctas), 256, 0, as_stream(stream)>>>(
      reinterpret_cast<const __nv_bfloat16*>(dh), reinterpret_cast<const __nv_bfloat16*>(gu),
      reinterpret_cast<__nv_bfloat16*>(dgu), M, F);
  count_launch();
  return status_of(cudaGetLastError());
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

// ------------------------------------------------------------------------------------------ NVFP4 forward

namespace qlora {
namespace {

// Workspace of qlora_linear_fwd_fp4: [x codes M x K/2][x scales, MMA layout][x tensor scale][su bf16 M x r]
// [fp32 partials of the split s x A^T product].
struct Fp4Plan {
  size_t off_codes = 0, off_sf = 0, off_S = 0, off_su = 0, off_part = 0, total = 0;
  int s_su = 1;
};

Fp4Plan plan_fp4(int64_t M, int64_t N, int64_t K, int64_t r) {
  Fp4Plan p;
  const LinearPlan lp = plan_linear(M, N, K, r, QL_PASS_FWD);
  size_t off = 0;
  p.off_codes = off;
  off += align256(static_cast<size_t>(M) * K / 2);
  p.off_sf = off;
  off += align256(static_cast<size_t>(fp4_sf_bytes(M, K)));
  p.off_S = off;
  off += 256;
  if (r > 0) {
    p.off_su = off;
    off += align256(static_cast<size_t>(M) * r * 2);
    p.s_su = lp.s_su;
    p.off_part = off;
    if (lp.s_su > 1) off += align256(static_cast<size_t>(lp.s_su) * M * r * 4);
  }
  p.total = off;
  return p;
}

cudaError_t launch_fp4_gemm(int64_t M, int64_t N, int64_t K, int64_t r, const uint8_t* w_codes, const uint8_t* w_sf,
                            const float* w_S, const uint8_t* x_codes, const uint8_t* x_sf, const float* x_S,
                            const uint16_t* B, const uint16_t* su, uint16_t* y, unsigned int* err, int sms,
                            cudaStream_t stream) {
  constexpr int BN = 128;
  using C = Fp4Cfg<BN>;
  CUtensorMap tmA, tmB, tmLA, tmLB;
  std::memset(&tmLA, 0, sizeof(tmLA));
  std::memset(&tmLB, 0, sizeof(tmLB));
  if (!make_map(&tmA, w_codes, N, K / 2, 1, 128, 128, true)) return cudaErrorInvalidValue;
  if (!make_map(&tmB, x_codes, M, K / 2, 1, 128, BN, true)) return cudaErrorInvalidValue;
  if (r > 0) {
    if (!make_map(&tmLA, B, N, r, 2, 64, 128, true)) return cudaErrorInvalidValue;
    if (!make_map(&tmLB, su, M, r, 2, 64, BN, true)) return cudaErrorInvalidValue;
  }
  Fp4Args a{};
  a.rows = static_cast<int>(N);
  a.cols = static_cast<int>(M);
  a.tiles_i = static_cast<int>(cdiv(N, 128));
  a.tiles_j = static_cast<int>(cdiv(M, BN));
  a.k_stages = static_cast<int>(cdiv(K, 256));
  a.n_extra = r > 0 ? static_cast<int>(cdiv(r, 64)) : 0;
  a.sfa = w_sf;
  a.sfb = x_sf;
  a.sf_rb_bytes = fp4_sf_rowblock_bytes(K);
  a.Sa = w_S;
  a.Sb = x_S;
  a.out = reinterpret_cast<__nv_bfloat16*>(y);
  a.ld = N;
  a.rows_lim = static_cast<int>(N);
  a.cols_lim = static_cast<int>(M);
  a.err = err;
  const int64_t units = static_cast<int64_t>(a.tiles_i) * a.tiles_j;
  // both operands are 0.5625 bytes per element, so the balanced group is about sqrt(C) weight tiles (see
  // unit_group)
  a.group_i = 0;
  if (grouped_enabled() && a.tiles_j > 1 && units > sms) {
    int gi = static_cast<int>(std::lround(std::sqrt(static_cast<double>(sms) * BN / 128.0)));
    a.group_i = std::max(1, std::min(gi, a.tiles_i));
  }
  auto kern = fp4_gemm_kernel<BN>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>(std::min<int64_t>(units, sms)));
  prof_record(0, 0, stream);
  kern<<<grid, 192, C::kSmemBytes, stream>>>(tmA, tmB, tmLA, tmLB, a);
  count_launch();
  prof_record(0, 1, stream);
  return cudaGetLastError();
}

}  // namespace
}  // namespace qlora

extern "C" size_t nvfp4_mma_scales_bytes(int64_t rows, int64_t K) {
  if (rows < 1 || K < 64 || K % 64 != 0) return 0;
  return static_cast<size_t>(fp4_sf_bytes(rows, K));
}

extern "C" ql_status nvfp4_scales_to_mma(const uint8_t* scales, int64_t rows, int64_t K, uint8_t* out, void* stream) {
  if (rows < 1 || K < 64 || K % 64 != 0 || !scales || !out || !aligned16(out)) return QL_ERR_INVALID_ARG;
  if (rows > (int64_t(1) << 31) - 1 || K > (int64_t(1) << 31) - 1) return QL_ERR_INVALID_ARG;
  DeviceInfo d;
  if (!device_info(&d)) return QL_ERR_CUDA;
  cudaStream_t cs = as_stream(stream);
  if (cudaMemsetAsync(out, 0, static_cast<size_t>(fp4_sf_bytes(rows, K)), cs) != cudaSuccess) return QL_ERR_CUDA;
  const long long n = rows * (K / 16);
  fp4_sf_to_mma_kernel<<<static_cast<unsigned>(std::min<long long>(cdiv(n, 256), d.sms * 16LL)), 256, 0, cs>>>(
      scales, rows, K, out);
  count_launch();
  return status_of(cudaGetLastError());
}

extern "C" size_t qlora_fp4_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t r) {
  if (check_linear(M, N, K, r) != QL_OK || M == 0) return 0;
  return plan_fp4(M, N, K, r).total;
}

extern "C" ql_status qlora_linear_fwd_fp4(int64_t M, int64_t N, int64_t K, int64_t r, const uint16_t* x,
                                          const uint8_t* w_codes, const uint8_t* w_sf_mma, const float* w_S,
                                          const uint16_t* A, const uint16_t* B, float s, uint16_t* y,
                                          uint16_t* su_out, void* workspace, size_t ws_bytes, void* stream) {
  ql_status st = check_linear(M, N, K, r);
  if (st != QL_OK) return st;
  if (M == 0) return QL_OK;
  if (!x || !w_codes || !w_sf_mma || !w_S || !y || !aligned16(x) || !aligned16(w_codes) || !aligned16(w_sf_mma) ||
      !aligned16(y))
    return QL_ERR_INVALID_ARG;
  if (r > 0 && (!A || !B || !aligned16(A) || !aligned16(B))) return QL_ERR_INVALID_ARG;
  if (su_out && !aligned16(su_out)) return QL_ERR_INVALID_ARG;
  const Fp4Plan p = plan_fp4(M, N, K, r);
  if (ws_bytes < p.total || !workspace || !aligned16(workspace)) return QL_ERR_INVALID_ARG;
  DeviceInfo d;
  if (!device_info(&d)) return QL_ERR_CUDA;
  cudaStream_t cs = as_stream(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* x_codes = ws + p.off_codes;
  uint8_t* x_sf = ws + p.off_sf;
  float* x_S = reinterpret_cast<float*>(ws + p.off_S);
  // the activations in NVFP4: largest magnitude, blocks (scales straight into the MMA layout), tensor scale
  if (cudaMemsetAsync(x_sf, 0, static_cast<size_t>(fp4_sf_bytes(M, K)), cs) != cudaSuccess) return QL_ERR_CUDA;
  if (cudaMemsetAsync(x_S, 0, sizeof(float), cs) != cudaSuccess) return QL_ERR_CUDA;
  const long long numel = M * K, nblk = numel / 16;
  const auto* xb = reinterpret_cast<const __nv_bfloat16*>(x);
  fp4_act_amax_kernel<<<static_cast<unsigned>(std::min<long long>(cdiv(numel, 256 * 8), d.sms * 16LL)), 256, 0, cs>>>(
      xb, numel, reinterpret_cast<unsigned int*>(x_S), d.err);
  count_launch();
  fp4_act_quantize_kernel<<<static_cast<unsigned>(std::min<long long>(cdiv(nblk, 256), d.sms * 16LL)), 256, 0, cs>>>(
      xb, M, K, reinterpret_cast<const unsigned int*>(x_S), x_codes, x_sf);
  count_launch();
  fp4_act_finalize_kernel<<<1, 32, 0, cs>>>(x_S);
  count_launch();
  if (cudaGetLastError() != cudaSuccess) return QL_ERR_CUDA;
  uint16_t* su = nullptr;
  if (r > 0) {
    su = su_out ? su_out : reinterpret_cast<uint16_t*>(ws + p.off_su);
    float* part = reinterpret_cast<float*>(ws + p.off_part);
    if (run_su(M, K, r, x, A, s, su, p.s_su, part, d.err, cs) != cudaSuccess) return QL_ERR_CUDA;
  }
  return status_of(launch_fp4_gemm(M, N, K, r, w_codes, w_sf_mma, w_S, x_codes, x_sf, x_S, B, su, y, d.err, d.sms,
                                   cs));
}

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

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

// The calling thread's current context (driver entry point reached through the runtime), or nullptr.
CUcontext current_context() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  CUcontext c = nullptr;
  if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Loads every kernel the forward can launch, so that no later call in this context loads one lazily (a
// module load may allocate).  cudaFuncGetAttributes forces the load and allocates nothing itself.
template <int BN, int AM, bool BMN, int KB = 1, bool PAIR = false>
bool load_umma() {
  cudaFuncAttributes a;
  return cudaFuncGetAttributes(&a, umma_gemm_kernel<BN, AM, BMN, KB, PAIR>) == cudaSuccess;
}

bool load_forward_kernels() {
  cudaFuncAttributes a;
  return load_umma<16, A_DEQ_TMEM, false>() && load_umma<32, A_DEQ_TMEM, false>() &&
         load_umma<64, A_DEQ_TMEM, false>() && load_umma<128, A_DEQ_TMEM, false>() &&
         load_umma<256, A_DEQ_TMEM, false>() && load_umma<256, A_DEQ_TMEM, false, 1, true>() &&
         load_umma<16, A_DEQ_TMEM, false, 4>() &&
         load_umma<32, A_DEQ_TMEM, false, 4>() && load_umma<64, A_DEQ_TMEM, false, 4>() &&
         load_umma<64, A_TMA_K, false>() && load_umma<128, A_TMA_K, false>() && load_umma<256, A_TMA_K, false>() &&
         cudaFuncGetAttributes(&a, reduce_splits_kernel) == cudaSuccess &&
         cudaFuncGetAttributes(&a, reduce_streamk_kernel) == cudaSuccess &&
         cudaFuncGetAttributes(&a, su_small_kernel) == cudaSuccess;
}

// Contexts in which the forward's kernels have been loaded (set-up runs once per context, with the device
// current).
CUcontext g_noalloc_ready[kMaxDevices * 4] = {};
int g_noalloc_nready = 0;
std::mutex g_noalloc_mu;

// Device address of g_noalloc_scratch in the current context.  In host code the array's name is only a
// host-side stand-in, so its address is looked up with the device current -- on every call, since it
// belongs to the context (cudaDeviceReset or a non-primary context gives another one) and the lookup
// allocates nothing once the module is loaded.  The first call in a context also loads the forward's
// kernels.
bool noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return false;
  const CUcontext ctx = current_context();
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  bool ready = false;
  for (int i = 0; i < g_noalloc_nready && !ready; ++i) ready = (g_noalloc_ready[i] == ctx);
  if (!ready) {
    if (!load_forward_kernels()) return false;
    if (ctx && g_noalloc_nready < kMaxDevices * 4) g_noalloc_ready[g_noalloc_nready++] = ctx;
  }
  *out = p;
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

"""Python binding of libqlora (the C ABI in include/qlora.h): argument marshalling only.

Every function here allocates its outputs with PyTorch on the inputs' CUDA device, passes raw pointers
and the current CUDA stream to the library, and raises ``QLoRAError`` on a non-OK status.  All arithmetic
runs in the library's kernels; there is no fallback: if libqlora.so is missing, the first call raises.
"""

from __future__ import annotations

import ctypes
import os
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqlora.so")

QL_OK, QL_ERR_INVALID_ARG, QL_ERR_UNSUPPORTED, QL_ERR_CUDA, QL_ERR_TIMEOUT = range(5)
QL_F32, QL_BF16 = 0, 1
QL_PASS_FWD, QL_PASS_BWD = 0, 1

_lib = None
_lock = threading.Lock()

_c_i64 = ctypes.c_int64
_c_p = ctypes.c_void_p

QL_W_NF4, QL_W_NF4_DQ, QL_W_NVFP4 = 0, 1, 2


class QlWeight(ctypes.Structure):
    """Mirror of include/qlora.h's ql_weight."""
    _fields_ = [("format", ctypes.c_int), ("codes", ctypes.c_void_p), ("absmax", ctypes.c_void_p),
                ("code8", ctypes.c_void_p), ("c1", ctypes.c_void_p), ("mu", ctypes.c_void_p),
                ("scales", ctypes.c_void_p), ("tensor_scale", ctypes.c_void_p)]


# name -> (restype, argtypes): mirrors include/qlora.h
SIGNATURES = {
    "ql_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "ql_abi_version": (ctypes.c_int, []),
    "ql_nf4_codebook": (None, [ctypes.POINTER(ctypes.c_float)]),
    "ql_get_device_error": (ctypes.c_int, [_c_p]),
    "ql_launch_count": (ctypes.c_uint64, []),
    "ql_set_profile_events": (ctypes.c_int, [ctypes.c_int, _c_p, _c_p]),
    "ql_selftest_wait_timeout": (ctypes.c_int, [_c_i64, _c_p]),
    "ql_selftest_arm_gemm_stall": (ctypes.c_int, [ctypes.c_int, _c_i64]),
    "nf4_quantize": (ctypes.c_int, [_c_p, _c_i64, ctypes.c_int, _c_p, _c_p, _c_p]),
    "nf4_dequantize": (ctypes.c_int, [_c_p, _c_p, _c_i64, ctypes.c_int, ctypes.c_int, _c_p, _c_p]),
    "qlora_merge_lora": (ctypes.c_int, [_c_i64, _c_i64, _c_i64, _c_p, _c_p, _c_p, _c_p, ctypes.c_float, ctypes.c_int,
                                        _c_p, _c_p]),
    "qlora_merge_lora_nf4": (ctypes.c_int, [_c_i64, _c_i64, _c_i64, _c_p, _c_p, _c_p, _c_p, ctypes.c_float, _c_p,
                                            _c_p, _c_p]),
    "qlora_workspace_bytes": (ctypes.c_size_t, [_c_i64, _c_i64, _c_i64, _c_i64, ctypes.c_int]),
    "qlora_linear_fwd": (ctypes.c_int, [_c_i64, _c_i64, _c_i64, _c_i64, _c_p, _c_p, _c_p, _c_p, _c_p, ctypes.c_float,
                                        _c_p, _c_p, _c_p, ctypes.c_size_t, _c_p]),
    "qlora_linear_bwd": (ctypes.c_int, [_c_i64, _c_i64, _c_i64, _c_i64, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p,
                                        ctypes.c_float, _c_p, _c_p, _c_p, _c_p, _c_p, ctypes.c_size_t, _c_p]),
    "qlora_linear_fwd_noalloc": (ctypes.c_int, [_c_i64, _c_i64, _c_i64, _c_i64, _c_p, _c_p, _c_p, _c_p, _c_p,
                                                ctypes.c_float, _c_p, _c_p, _c_p]),
    "qlora_swiglu_fwd": (ctypes.c_int, [_c_i64, _c_p, _c_p, _c_p, _c_p]),
    "qlora_swiglu_bwd": (ctypes.c_int, [_c_i64, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p]),
    "qlora_swiglu_gated_fwd": (ctypes.c_int, [_c_i64, _c_i64, _c_p, _c_p, _c_p]),
    "qlora_swiglu_gated_bwd": (ctypes.c_int, [_c_i64, _c_i64, _c_p, _c_p, _c_p, _c_p]),
    "qlora_linear_fwd_w": (ctypes.c_int, [_c_i64, _c_i64, _c_i64, _c_i64, _c_p, ctypes.POINTER(QlWeight), _c_p, _c_p,
                                          ctypes.c_float, _c_p, _c_p, _c_p, ctypes.c_size_t, _c_p]),
    "qlora_linear_bwd_w": (ctypes.c_int, [_c_i64, _c_i64, _c_i64, _c_i64, _c_p, _c_p, ctypes.POINTER(QlWeight), _c_p,
                                          _c_p, ctypes.c_float, _c_p, _c_p, _c_p, _c_p, _c_p, ctypes.c_size_t, _c_p]),
    "qlora_gated_workspace_bytes": (ctypes.c_size_t, [_c_i64, _c_i64, _c_i64, _c_i64, ctypes.c_int]),
    "qlora_gate_up_fwd_swiglu": (ctypes.c_int, [_c_i64, _c_i64, _c_i64, _c_i64, _c_p, _c_p, _c_p, _c_p, _c_p,
                                                ctypes.c_float, _c_p, _c_p, _c_p, _c_p, ctypes.c_size_t, _c_p]),
    "qlora_down_bwd_dswiglu": (ctypes.c_int, [_c_i64, _c_i64, _c_i64, _c_i64, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p,
                                              ctypes.c_float, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, ctypes.c_size_t,
                                              _c_p]),
    "ql_formats_launch_count": (ctypes.c_uint64, []),
    "ql_formats_get_device_error": (ctypes.c_int, [_c_p]),
    "nf4_double_quantize_scratch_bytes": (ctypes.c_size_t, [_c_i64]),
    "nf4_double_quantize": (ctypes.c_int, [_c_p, _c_i64, _c_p, _c_p, _c_p, _c_p, ctypes.c_size_t, _c_p]),
    "nf4_double_dequantize": (ctypes.c_int, [_c_p, _c_p, _c_p, _c_i64, _c_p, _c_p]),
    "nvfp4_quantize": (ctypes.c_int, [_c_p, _c_i64, _c_p, _c_p, _c_p, _c_p]),
    "nvfp4_dequantize": (ctypes.c_int, [_c_p, _c_p, _c_p, _c_i64, ctypes.c_int, _c_p, _c_p]),
    "nvfp4_mma_scales_bytes": (ctypes.c_size_t, [_c_i64, _c_i64]),
    "nvfp4_scales_to_mma": (ctypes.c_int, [_c_p, _c_i64, _c_i64, _c_p, _c_p]),
    "qlora_fp4_workspace_bytes": (ctypes.c_size_t, [_c_i64, _c_i64, _c_i64, _c_i64]),
    "qlora_linear_fwd_fp4": (ctypes.c_int, [_c_i64, _c_i64, _c_i64, _c_i64, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p,
                                            ctypes.c_float, _c_p, _c_p, _c_p, ctypes.c_size_t, _c_p]),
}


class QLoRAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built (no fallback exists)."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise RuntimeError(f"libqlora.so is not built ({LIB_PATH}); run "
                                       "`python -m qlora_fine_tuning_blockwise_b200.build`")
                L = ctypes.CDLL(LIB_PATH)
                for name, (res, args) in SIGNATURES.items():
                    f = getattr(L, name)
                    f.restype = res
                    f.argtypes = args
                _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().ql_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != QL_OK:
        raise QLoRAError(status, where)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device | None = None):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _bits(t: torch.Tensor) -> torch.Tensor:
    """bf16 tensors travel as their bit patterns; the library reads them as uint16."""
    assert t.dtype == torch.bfloat16 and t.is_cuda and t.is_contiguous(), (t.dtype, t.device, t.is_contiguous())
    return t


# ------------------------------------------------------------------------------------------ host-only


def abi_version() -> int:
    return int(lib().ql_abi_version())


def codebook() -> np.ndarray:
    """The library's NF4 table (fp32, ascending)."""
    out = (ctypes.c_float * 16)()
    lib().ql_nf4_codebook(out)
    return np.array(out[:], dtype=np.float32)


def workspace_bytes(M: int, N: int, K: int, r: int, pass_: int) -> int:
    return int(lib().qlora_workspace_bytes(M, N, K, r, pass_))


def device_error(device: torch.device | None = None) -> int:
    """Status from the device error word (synchronizes the current stream)."""
    return int(lib().ql_get_device_error(_stream(device)))


def launch_count() -> int:
    """Kernels this library has launched in this process."""
    return int(lib().ql_launch_count())


def set_profile_events(which: int, start=None, stop=None) -> None:
    """Record torch.cuda.Event ``start``/``stop`` around the fused forward (0) or dX (1) GEMM; None disables."""
    def handle(ev):
        if ev is None:
            return None
        if ev.cuda_event == 0:  # torch creates the event on first record
            ev.record()
        return ctypes.c_void_p(ev.cuda_event)
    _check(lib().ql_set_profile_events(which, handle(start), handle(stop)), "ql_set_profile_events")


def selftest_arm_gemm_stall(role: int, wait_cycles: int) -> None:
    """Arm the next fused GEMM launch to stall one warp role (1 MMA, 2 B producer, 3 codes producer) with every
    wait bounded by ``wait_cycles``: a test of the kernels' abort path."""
    _check(lib().ql_selftest_arm_gemm_stall(int(role), int(wait_cycles)), "ql_selftest_arm_gemm_stall")


def selftest_wait_timeout(wait_cycles: int) -> None:
    _check(lib().ql_selftest_wait_timeout(int(wait_cycles), _stream()), "ql_selftest_wait_timeout")


# ------------------------------------------------------------------------------------------ NF4


def nf4_quantize(w: torch.Tensor, blocksize: int = 64):
    """w: CUDA fp32 (any shape, row-major contiguous) -> (codes uint8 [numel/2], absmax fp32 [numel/blocksize])."""
    assert w.is_cuda and w.dtype == torch.float32 and w.is_contiguous()
    n = w.numel()
    codes = torch.empty(n // 2, dtype=torch.uint8, device=w.device)
    absmax = torch.empty(max(n // max(blocksize, 1), 0), dtype=torch.float32, device=w.device)
    _check(lib().nf4_quantize(_ptr(w), n, blocksize, _ptr(codes), _ptr(absmax), _stream(w.device)), "nf4_quantize")
    return codes, absmax


def nf4_dequantize(codes: torch.Tensor, absmax: torch.Tensor, numel: int, blocksize: int = 64,
                   dtype: torch.dtype = torch.float32) -> torch.Tensor:
    assert codes.is_cuda and codes.dtype == torch.uint8 and absmax.dtype == torch.float32
    out = torch.empty(numel, dtype=dtype, device=codes.device)
    code = QL_BF16 if dtype == torch.bfloat16 else QL_F32
    _check(lib().nf4_dequantize(_ptr(codes), _ptr(absmax), numel, blocksize, code, _ptr(out), _stream(codes.device)),
           "nf4_dequantize")
    return out


def merge_lora(codes: torch.Tensor, absmax: torch.Tensor, A, B, s: float, N: int, K: int,
               dtype: torch.dtype = torch.float32) -> torch.Tensor:
    """W' = deq(W) + s B A  [N,K] (fp32 or bf16); A [r,K] and B [N,r] bf16, or None for r = 0."""
    assert codes.is_cuda and codes.dtype == torch.uint8 and absmax.dtype == torch.float32
    r = 0 if A is None else A.shape[0]
    out = torch.empty(N, K, dtype=dtype, device=codes.device)
    code = QL_BF16 if dtype == torch.bfloat16 else QL_F32
    _check(lib().qlora_merge_lora(N, K, r, _ptr(codes), _ptr(absmax), _ptr(_bits(A) if r else None),
                                  _ptr(_bits(B) if r else None), float(s), code, _ptr(out), _stream(codes.device)),
           "qlora_merge_lora")
    return out


def merge_lora_nf4(codes: torch.Tensor, absmax: torch.Tensor, A, B, s: float, N: int, K: int,
                   codes_out: torch.Tensor | None = None, absmax_out: torch.Tensor | None = None):
    """(codes', absmax'): W' = deq(W) + s B A requantized to NF4 in one pass.  Passing the input tensors as the
    outputs merges in place."""
    assert codes.is_cuda and codes.dtype == torch.uint8 and absmax.dtype == torch.float32
    r = 0 if A is None else A.shape[0]
    if codes_out is None:
        codes_out = torch.empty_like(codes)
    if absmax_out is None:
        absmax_out = torch.empty_like(absmax)
    _check(lib().qlora_merge_lora_nf4(N, K, r, _ptr(codes), _ptr(absmax), _ptr(_bits(A) if r else None),
                                      _ptr(_bits(B) if r else None), float(s), _ptr(codes_out), _ptr(absmax_out),
                                      _stream(codes.device)), "qlora_merge_lora_nf4")
    return codes_out, absmax_out


# ------------------------------------------------------------------------------------------ weight formats


def formats_device_error(device: torch.device | None = None) -> int:
    """Status from the format conversions' device error word (synchronizes the current stream)."""
    return int(lib().ql_formats_get_device_error(_stream(device)))


def formats_launch_count() -> int:
    """Format-conversion kernels this library has launched in this process."""
    return int(lib().ql_formats_launch_count())


def nf4_double_quantize(absmax: torch.Tensor):
    """Double quantization of the NF4 block constants: (code8 uint8 [nb], c1 fp32 [ceil(nb/256)], mu fp32 [1])."""
    assert absmax.is_cuda and absmax.dtype == torch.float32 and absmax.is_contiguous()
    nb = absmax.numel()
    code8 = torch.empty(nb, dtype=torch.uint8, device=absmax.device)
    c1 = torch.empty((nb + 255) // 256, dtype=torch.float32, device=absmax.device)
    mu = torch.empty(1, dtype=torch.float32, device=absmax.device)
    need = int(lib().nf4_double_quantize_scratch_bytes(nb))
    scratch = torch.empty(max(need, 16), dtype=torch.uint8, device=absmax.device)
    _check(lib().nf4_double_quantize(_ptr(absmax), nb, _ptr(code8), _ptr(c1), _ptr(mu), _ptr(scratch), need,
                                     _stream(absmax.device)), "nf4_double_quantize")
    return code8, c1, mu


def nf4_double_dequantize(code8: torch.Tensor, c1: torch.Tensor, mu: torch.Tensor) -> torch.Tensor:
    """absmax' fp32 [nb] from the outputs of nf4_double_quantize."""
    assert code8.is_cuda and code8.dtype == torch.uint8 and c1.dtype == torch.float32 and mu.dtype == torch.float32
    out = torch.empty(code8.numel(), dtype=torch.float32, device=code8.device)
    _check(lib().nf4_double_dequantize(_ptr(code8), _ptr(c1), _ptr(mu), code8.numel(), _ptr(out),
                                       _stream(code8.device)), "nf4_double_dequantize")
    return out


def nvfp4_quantize(w: torch.Tensor):
    """w: CUDA fp32 contiguous -> (codes uint8 [numel/2], scales uint8 [numel/16] (E4M3), S fp32 [1])."""
    assert w.is_cuda and w.dtype == torch.float32 and w.is_contiguous()
    n = w.numel()
    codes = torch.empty(n // 2, dtype=torch.uint8, device=w.device)
    scales = torch.empty(n // 16, dtype=torch.uint8, device=w.device)
    S = torch.empty(1, dtype=torch.float32, device=w.device)
    _check(lib().nvfp4_quantize(_ptr(w), n, _ptr(codes), _ptr(scales), _ptr(S), _stream(w.device)), "nvfp4_quantize")
    return codes, scales, S


def nvfp4_dequantize(codes: torch.Tensor, scales: torch.Tensor, S: torch.Tensor, numel: int,
                     dtype: torch.dtype = torch.float32) -> torch.Tensor:
    assert codes.is_cuda and codes.dtype == torch.uint8 and scales.dtype == torch.uint8 and S.dtype == torch.float32
    out = torch.empty(numel, dtype=dtype, device=codes.device)
    code = QL_BF16 if dtype == torch.bfloat16 else QL_F32
    _check(lib().nvfp4_dequantize(_ptr(codes), _ptr(scales), _ptr(S), numel, code, _ptr(out), _stream(codes.device)),
           "nvfp4_dequantize")
    return out


# ------------------------------------------------------------------------------------------ weights in any format


class Weight:
    """A frozen base weight [N, K] in one of the formats, with the device tensors it points to kept alive."""

    def __init__(self, N, K, fmt, **t):
        self.N, self.K, self.format, self.t = N, K, fmt, t
        self.c = QlWeight(fmt, *(t[k].data_ptr() if t.get(k) is not None else None
                                 for k in ("codes", "absmax", "code8", "c1", "mu", "scales", "tensor_scale")))

    @staticmethod
    def nf4(W):
        codes, absmax = nf4_quantize(W.contiguous())
        return Weight(W.shape[0], W.shape[1], QL_W_NF4, codes=codes, absmax=absmax)

    @staticmethod
    def nf4_dq(W):
        codes, absmax = nf4_quantize(W.contiguous())
        code8, c1, mu = nf4_double_quantize(absmax)
        return Weight(W.shape[0], W.shape[1], QL_W_NF4_DQ, codes=codes, code8=code8, c1=c1, mu=mu)

    @staticmethod
    def nvfp4(W):
        codes, scales, S = nvfp4_quantize(W.contiguous())
        return Weight(W.shape[0], W.shape[1], QL_W_NVFP4, codes=codes, scales=scales, tensor_scale=S)


def linear_fwd_w(x, w: Weight, A, B, s: float, want_su: bool = True):
    M, K = x.shape
    r = 0 if A is None else A.shape[0]
    y = torch.empty(M, w.N, dtype=torch.bfloat16, device=x.device)
    su = torch.empty(M, r, dtype=torch.bfloat16, device=x.device) if (r and want_su) else None
    need = workspace_bytes(M, w.N, K, r, QL_PASS_FWD)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=x.device)
    _check(lib().qlora_linear_fwd_w(M, w.N, K, r, _ptr(_bits(x)), ctypes.byref(w.c), _ptr(A), _ptr(B), float(s),
                                    _ptr(y), _ptr(su), _ptr(ws), need, _stream(x.device)), "qlora_linear_fwd_w")
    return y, su


def linear_bwd_w(dy, x, w: Weight, A, B, s: float, su=None):
    M, N = dy.shape
    K = w.K
    r = 0 if A is None else A.shape[0]
    dx = torch.empty(M, K, dtype=torch.bfloat16, device=dy.device)
    dA = torch.empty(r, K, dtype=torch.float32, device=dy.device) if r else None
    dB = torch.empty(N, r, dtype=torch.float32, device=dy.device) if r else None
    need = workspace_bytes(M, N, K, r, QL_PASS_BWD)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dy.device)
    _check(lib().qlora_linear_bwd_w(M, N, K, r, _ptr(_bits(dy)), _ptr(_bits(x)), ctypes.byref(w.c), _ptr(A), _ptr(B),
                                    float(s), _ptr(su), _ptr(dx), _ptr(dA), _ptr(dB), _ptr(ws), need,
                                    _stream(dy.device)), "qlora_linear_bwd_w")
    return dx, dA, dB


# ------------------------------------------------------------------------------------------ gated MLP (fused SwiGLU)


def gate_up_fwd_swiglu(x, layer, h):
    """(gu [M, 2F] interleaved, h [M, F], su) for the interleaved gate/up QLoRALinear ``layer``; h is written."""
    M, K = x.shape
    N, r = layer.N, layer.r
    F = N // 2
    gu = torch.empty(M, N, dtype=torch.bfloat16, device=x.device)
    su = torch.empty(M, r, dtype=torch.bfloat16, device=x.device) if r else None
    need = int(lib().qlora_gated_workspace_bytes(M, N, K, r, QL_PASS_FWD))
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=x.device)
    _check(lib().qlora_gate_up_fwd_swiglu(M, F, K, r, _ptr(_bits(x)), _ptr(layer.codes), _ptr(layer.absmax),
                                          _ptr(layer.A if r else None), _ptr(layer.B if r else None), layer.s,
                                          _ptr(gu), _ptr(h), _ptr(su), _ptr(ws), need, _stream(x.device)),
           "qlora_gate_up_fwd_swiglu")
    return gu, h, su


def down_bwd_dswiglu(dy, h, layer, su, gu, dgu):
    """(dgu [M, 2F] interleaved, dA, dB) for the down QLoRALinear ``layer`` (input h, output dy)."""
    M, N = dy.shape
    F, r = layer.K, layer.r
    dA = torch.empty(r, F, dtype=torch.float32, device=dy.device) if r else None
    dB = torch.empty(N, r, dtype=torch.float32, device=dy.device) if r else None
    need = int(lib().qlora_gated_workspace_bytes(M, N, F, r, QL_PASS_BWD))
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dy.device)
    _check(lib().qlora_down_bwd_dswiglu(M, N, F, r, _ptr(_bits(dy)), _ptr(_bits(h)), _ptr(layer.codes),
                                        _ptr(layer.absmax), _ptr(layer.A if r else None), _ptr(layer.B if r else None),
                                        layer.s, _ptr(su), _ptr(gu), _ptr(dgu), _ptr(dA), _ptr(dB), _ptr(ws), need,
                                        _stream(dy.device)), "qlora_down_bwd_dswiglu")
    return dgu, dA, dB


def nvfp4_scales_to_mma(scales: torch.Tensor, rows: int, K: int) -> torch.Tensor:
    """An NVFP4 weight's row-major scales [rows, K/16] laid out as the FP4 tensor core reads them (uint8)."""
    assert scales.is_cuda and scales.dtype == torch.uint8
    out = torch.empty(int(lib().nvfp4_mma_scales_bytes(rows, K)), dtype=torch.uint8, device=scales.device)
    _check(lib().nvfp4_scales_to_mma(_ptr(scales), rows, K, _ptr(out), _stream(scales.device)), "nvfp4_scales_to_mma")
    return out


class FP4Linear:
    """A frozen base weight in NVFP4 with its bf16 LoRA pair, for the forward on the block-scaled FP4 tensor core
    (qlora_linear_fwd_fp4): the weight is quantized once and its scales laid out for the MMA."""

    def __init__(self, W: torch.Tensor, A, B, s: float):
        assert W.dim() == 2 and W.is_cuda
        self.N, self.K = W.shape
        self.codes, scales, self.S = nvfp4_quantize(W.contiguous())
        self.sf = nvfp4_scales_to_mma(scales, self.N, self.K)
        self.A, self.B, self.s = A, B, float(s)
        self.r = 0 if A is None else A.shape[0]
        self._ws = {}

    def forward(self, x: torch.Tensor, y: torch.Tensor | None = None, su: torch.Tensor | None = None,
                want_su: bool = False):
        M = x.shape[0]
        N, K, r = self.N, self.K, self.r
        y = torch.empty(M, N, dtype=torch.bfloat16, device=x.device) if y is None else y
        if want_su and r and su is None:
            su = torch.empty(M, r, dtype=torch.bfloat16, device=x.device)
        ws = self._ws.get(M)
        if ws is None:
            ws = self._ws[M] = torch.empty(max(int(lib().qlora_fp4_workspace_bytes(M, N, K, r)), 16),
                                           dtype=torch.uint8, device=x.device)
        _check(lib().qlora_linear_fwd_fp4(M, N, K, r, _ptr(_bits(x)), _ptr(self.codes), _ptr(self.sf), _ptr(self.S),
                                          _ptr(self.A if r else None), _ptr(self.B if r else None), self.s, _ptr(y),
                                          _ptr(su), _ptr(ws), ws.numel(), _stream(x.device)), "qlora_linear_fwd_fp4")
        return y, su

    def quantized_activations(self, M: int):
        """(codes [M, K/2], scales in the MMA layout, tensor scale) of the last forward's activations, views of the
        workspace (the layout of qlora_linear_fwd_fp4's workspace: codes, then scales, then the tensor scale)."""
        ws = self._ws[M]
        K = self.K
        ncodes = M * K // 2
        a256 = lambda n: (n + 255) // 256 * 256  # noqa: E731
        nsf = int(lib().nvfp4_mma_scales_bytes(M, K))
        codes = ws[:ncodes]
        sf = ws[a256(ncodes):a256(ncodes) + nsf]
        S = ws[a256(ncodes) + a256(nsf):a256(ncodes) + a256(nsf) + 4].view(torch.float32)
        return codes, sf, S


# ------------------------------------------------------------------------------------------ linear layer


def _workspace(M, N, K, r, pass_, device, workspace):
    need = workspace_bytes(M, N, K, r, pass_)
    if workspace is not None and workspace.numel() >= need:
        return workspace, need
    return (torch.empty(need, dtype=torch.uint8, device=device) if need else None), need


def qlora_linear_fwd(x, codes, absmax, A, B, s: float, N: int, K: int, want_su: bool = True, workspace=None,
                     y=None, su=None):
    """(y [M,N] bf16, su [M,r] bf16 or None) for y = x deq(W)^T + s (x A^T) B^T."""
    M = x.shape[0]
    r = 0 if A is None else A.shape[0]
    dev = x.device
    y = torch.empty(M, N, dtype=torch.bfloat16, device=dev) if y is None else y
    if want_su and r > 0 and su is None:
        su = torch.empty(M, r, dtype=torch.bfloat16, device=dev)
    if not want_su:
        su = None
    ws, need = _workspace(M, N, K, r, QL_PASS_FWD, dev, workspace)
    _check(lib().qlora_linear_fwd(M, N, K, r, _ptr(_bits(x)), _ptr(codes), _ptr(absmax),
                                  _ptr(A if r else None), _ptr(B if r else None), float(s), _ptr(y), _ptr(su),
                                  _ptr(ws), need, _stream(dev)), "qlora_linear_fwd")
    return y, su


def qlora_linear_fwd_noalloc(x, codes, absmax, A, B, s: float, N: int, K: int, y, su=None):
    """The forward with the library's built-in scratch instead of a workspace (for callers that cannot
    allocate device memory); ``y`` (and ``su`` when wanted) are the caller's buffers.  Returns (y, su)."""
    M = x.shape[0]
    r = 0 if A is None else A.shape[0]
    _check(lib().qlora_linear_fwd_noalloc(M, N, K, r, _ptr(_bits(x)), _ptr(codes), _ptr(absmax),
                                          _ptr(A if r else None), _ptr(B if r else None), float(s), _ptr(y),
                                          _ptr(su), _stream(x.device)), "qlora_linear_fwd_noalloc")
    return y, su


def qlora_linear_bwd(dy, x, codes, absmax, A, B, s: float, N: int, K: int, su=None, need_dx=True, need_dA=True,
                     need_dB=True, workspace=None, dx=None, dA=None, dB=None):
    """(dX [M,K] bf16, dA [r,K] fp32, dB [N,r] fp32); entries not requested are None."""
    M = dy.shape[0]
    r = 0 if A is None else A.shape[0]
    dev = dy.device
    if need_dx and dx is None:
        dx = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    if need_dA and r > 0 and dA is None:
        dA = torch.empty(r, K, dtype=torch.float32, device=dev)
    if need_dB and r > 0 and dB is None:
        dB = torch.empty(N, r, dtype=torch.float32, device=dev)
    dx = dx if need_dx else None
    dA = dA if (need_dA and r > 0) else None
    dB = dB if (need_dB and r > 0) else None
    ws, need = _workspace(M, N, K, r, QL_PASS_BWD, dev, workspace)
    _check(lib().qlora_linear_bwd(M, N, K, r, _ptr(dy), _ptr(x), _ptr(codes), _ptr(absmax),
                                  _ptr(A if r else None), _ptr(B if r else None), float(s), _ptr(su), _ptr(dx),
                                  _ptr(dA), _ptr(dB), _ptr(ws), need, _stream(dev)), "qlora_linear_bwd")
    return dx, dA, dB


# ------------------------------------------------------------------------------------------ SwiGLU


def swiglu_fwd(g: torch.Tensor, u: torch.Tensor, h: torch.Tensor | None = None) -> torch.Tensor:
    h = torch.empty_like(g) if h is None else h
    _check(lib().qlora_swiglu_fwd(g.numel(), _ptr(_bits(g)), _ptr(_bits(u)), _ptr(h), _stream(g.device)),
           "qlora_swiglu_fwd")
    return h


def swiglu_bwd(dh: torch.Tensor, g: torch.Tensor, u: torch.Tensor, dg=None, du=None):
    dg = torch.empty_like(g) if dg is None else dg
    du = torch.empty_like(u) if du is None else du
    _check(lib().qlora_swiglu_bwd(g.numel(), _ptr(_bits(dh)), _ptr(g), _ptr(u), _ptr(dg), _ptr(du),
                                  _stream(g.device)), "qlora_swiglu_bwd")
    return dg, du


def swiglu_gated_fwd(gu: torch.Tensor, h: torch.Tensor | None = None) -> torch.Tensor:
    """gu bf16 [M, 2F] (gate | up) -> h bf16 [M, F]."""
    M, F2 = gu.shape
    h = torch.empty(M, F2 // 2, dtype=torch.bfloat16, device=gu.device) if h is None else h
    _check(lib().qlora_swiglu_gated_fwd(M, F2 // 2, _ptr(_bits(gu)), _ptr(h), _stream(gu.device)),
           "qlora_swiglu_gated_fwd")
    return h


def swiglu_gated_bwd(dh: torch.Tensor, gu: torch.Tensor, dgu: torch.Tensor | None = None) -> torch.Tensor:
    """(dh [M, F], gu [M, 2F]) -> dgu [M, 2F] bf16."""
    M, F2 = gu.shape
    dgu = torch.empty_like(gu) if dgu is None else dgu
    _check(lib().qlora_swiglu_gated_bwd(M, F2 // 2, _ptr(_bits(dh)), _ptr(gu), _ptr(dgu), _stream(gu.device)),
           "qlora_swiglu_gated_bwd")
    return dgu


# ------------------------------------------------------------------------------------------ a layer object


class QLoRALinear:
    """A frozen NF4 base weight with its bf16 LoRA pair and preallocated buffers for repeated steps.

    ``forward`` / ``backward`` reuse the output and workspace buffers of the last call with the same M, so a
    training loop allocates nothing per step.
    """

    def __init__(self, W: torch.Tensor, A: torch.Tensor, B: torch.Tensor, s: float):
        assert W.dim() == 2 and W.is_cuda
        self.N, self.K = W.shape
        self.codes, self.absmax = nf4_quantize(W.contiguous())
        self.A, self.B, self.s = A, B, float(s)
        self.r = 0 if A is None else A.shape[0]
        self._bufs = {}

    @classmethod
    def from_quantized(cls, codes, absmax, N, K, A, B, s):
        self = cls.__new__(cls)
        self.N, self.K = N, K
        self.codes, self.absmax = codes, absmax
        self.A, self.B, self.s = A, B, float(s)
        self.r = 0 if A is None else A.shape[0]
        self._bufs = {}
        return self

    def _buffers(self, M: int, device):
        b = self._bufs.get(M)
        if b is None:
            N, K, r = self.N, self.K, self.r
            b = dict(
                y=torch.empty(M, N, dtype=torch.bfloat16, device=device),
                su=torch.empty(M, r, dtype=torch.bfloat16, device=device) if r else None,
                dx=torch.empty(M, K, dtype=torch.bfloat16, device=device),
                dA=torch.empty(r, K, dtype=torch.float32, device=device) if r else None,
                dB=torch.empty(N, r, dtype=torch.float32, device=device) if r else None,
                ws_f=torch.empty(max(workspace_bytes(M, N, K, r, QL_PASS_FWD), 1), dtype=torch.uint8, device=device),
                ws_b=torch.empty(max(workspace_bytes(M, N, K, r, QL_PASS_BWD), 1), dtype=torch.uint8, device=device),
            )
            self._bufs[M] = b
        return b

    def forward(self, x: torch.Tensor):
        b = self._buffers(x.shape[0], x.device)
        return qlora_linear_fwd(x, self.codes, self.absmax, self.A, self.B, self.s, self.N, self.K, want_su=True,
                                workspace=b["ws_f"], y=b["y"], su=b["su"])

    def backward(self, dy: torch.Tensor, x: torch.Tensor, su: torch.Tensor | None = None, need_dx: bool = True):
        b = self._buffers(dy.shape[0], dy.device)
        return qlora_linear_bwd(dy, x, self.codes, self.absmax, self.A, self.B, self.s, self.N, self.K, su=su,
                                need_dx=need_dx, workspace=b["ws_b"], dx=b["dx"], dA=b["dA"], dB=b["dB"])

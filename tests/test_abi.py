"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every symbol include/qlora.h
declares, carries the oracle's NF4 table bit for bit, and rejects bad arguments on the host before any
launch.  No compute call is made here."""

import ctypes
import os
import re

import numpy as np
import pytest

from oracle import nf4 as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qlora.h")


@pytest.fixture(scope="module")
def L():
    from qlora_fine_tuning_blockwise_b200 import build, ops
    build.build()
    return ops


def header_functions():
    text = open(HEADER).read()
    return re.findall(r"^QL_API\s+[\w\s\*]+?\b(\w+)\s*\(", text, flags=re.M)


def test_header_declares_the_boundary():
    names = header_functions()
    for required in ("nf4_quantize", "nf4_dequantize", "qlora_linear_fwd", "qlora_linear_bwd", "qlora_workspace_bytes"):
        assert required in names


def test_library_exports_every_declared_symbol(L):
    lib = L.lib()
    names = header_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(lib, n), n
        assert n in L.SIGNATURES, f"binding lacks {n}"


def test_abi_version_and_status_strings(L):
    assert L.abi_version() >= 1
    assert L.status_string(0) == "QL_OK"
    assert L.status_string(1) == "QL_ERR_INVALID_ARG"
    assert L.status_string(4) == "QL_ERR_TIMEOUT"


def test_library_codebook_is_bitwise_the_oracle_table(L):
    ours = L.codebook()
    assert np.array_equal(ours.view(np.uint32), O.nf4_codebook().view(np.uint32))


FAKE = 0x10000  # an aligned host address; validation must fail before anything dereferences it


def test_quantize_rejects_bad_arguments_on_host(L):
    lib = L.lib()
    p = ctypes.c_void_p(FAKE)
    assert lib.nf4_quantize(p, 0, 64, p, p, None) == L.QL_ERR_INVALID_ARG          # empty
    assert lib.nf4_quantize(p, 100, 64, p, p, None) == L.QL_ERR_INVALID_ARG        # not a multiple
    assert lib.nf4_quantize(p, 128, 32, p, p, None) == L.QL_ERR_UNSUPPORTED        # block 32 not built
    assert lib.nf4_quantize(None, 128, 64, p, p, None) == L.QL_ERR_INVALID_ARG     # null
    assert lib.nf4_quantize(ctypes.c_void_p(FAKE + 4), 128, 64, p, p, None) == L.QL_ERR_INVALID_ARG  # misaligned
    assert lib.nf4_dequantize(p, p, 128, 64, 7, p, None) == L.QL_ERR_INVALID_ARG   # bad dtype


@pytest.mark.parametrize("M,N,K,r", [(16, 12, 64, 8), (16, 16, 100, 8), (16, 16, 0, 8), (16, 16, 64, 12),
                                     (16, 16, 64, 264), (-1, 16, 64, 8), (16, 0, 64, 8)])
def test_linear_rejects_bad_shapes_on_host(L, M, N, K, r):
    lib = L.lib()
    p = ctypes.c_void_p(FAKE)
    assert lib.qlora_linear_fwd(M, N, K, r, p, p, p, p, p, 2.0, p, None, p, 1 << 30, None) == L.QL_ERR_INVALID_ARG
    assert lib.qlora_linear_bwd(M, N, K, r, p, p, p, p, p, p, 2.0, None, p, p, p, p, 1 << 30, None) == \
        L.QL_ERR_INVALID_ARG
    assert L.workspace_bytes(M, N, K, r, 0) == 0


def test_linear_rejects_small_workspace_and_misalignment_on_host(L):
    lib = L.lib()
    p = ctypes.c_void_p(FAKE)
    need = L.workspace_bytes(2048, 4096, 4096, 16, L.QL_PASS_FWD)
    assert need > 0
    assert lib.qlora_linear_fwd(2048, 4096, 4096, 16, p, p, p, p, p, 2.0, p, None, p, need - 1, None) == \
        L.QL_ERR_INVALID_ARG
    bad = ctypes.c_void_p(FAKE + 2)
    assert lib.qlora_linear_fwd(64, 256, 256, 8, bad, p, p, p, p, 2.0, p, None, p, 1 << 30, None) == \
        L.QL_ERR_INVALID_ARG


def test_workspace_plan_is_host_only_and_sane(L):
    # plain layer with many tokens needs no scratch; the rank-r intermediates need M*r*2 bytes each at least
    assert L.workspace_bytes(4096, 4096, 4096, 0, L.QL_PASS_FWD) == 0
    f = L.workspace_bytes(2048, 4096, 4096, 16, L.QL_PASS_FWD)
    b = L.workspace_bytes(2048, 4096, 4096, 16, L.QL_PASS_BWD)
    assert f >= 2048 * 16 * 2 and b >= 2 * 2048 * 16 * 2
    # small M splits the contraction: fp32 partial sums of y appear in the plan
    assert L.workspace_bytes(16, 28672, 8192, 16, L.QL_PASS_FWD) >= 16 * 16 * 2
    assert L.workspace_bytes(0, 4096, 4096, 16, L.QL_PASS_FWD) == 0


def test_forward_splits_s_x_at_only_where_the_fused_gemm_cannot_absorb_it(L):
    """The forward plan (for 148 SMs, the host-side default) runs s x A^T unsplit -- no fp32 partial sums in the
    workspace -- when its CTAs fit on the fused GEMM's CTAs that own one unit fewer (the attention layer: 256 units,
    40 short CTAs, 16 s x A^T CTAs; the MLP down projection: 512 units, 80 short, 32), and splits it where every CTA
    of the fused GEMM carries the same load (the block's layers)."""
    assert L.workspace_bytes(2048, 4096, 4096, 16, L.QL_PASS_FWD) == 2048 * 16 * 2
    assert L.workspace_bytes(4096, 4096, 11008, 64, L.QL_PASS_FWD) == 4096 * 64 * 2
    assert L.workspace_bytes(8192, 57344, 8192, 128, L.QL_PASS_FWD) > 8192 * 128 * 2
    assert L.workspace_bytes(8192, 8192, 28672, 64, L.QL_PASS_FWD) > 8192 * 64 * 2


def test_swiglu_rejects_bad_arguments_on_host(L):
    lib = L.lib()
    p = ctypes.c_void_p(FAKE)
    assert lib.qlora_swiglu_fwd(-1, p, p, p, None) == L.QL_ERR_INVALID_ARG
    assert lib.qlora_swiglu_fwd(0, None, None, None, None) == L.QL_OK
    assert lib.qlora_swiglu_bwd(8, p, None, p, p, p, None) == L.QL_ERR_INVALID_ARG


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    from qlora_fine_tuning_blockwise_b200 import ops
    monkeypatch.setattr(ops, "_lib", None)
    monkeypatch.setattr(ops, "LIB_PATH", str(tmp_path / "nope.so"))
    with pytest.raises(RuntimeError, match="not built"):
        ops.lib()


def test_merge_rejects_bad_arguments_on_host(L):
    lib = L.lib()
    p = ctypes.c_void_p(FAKE)
    for N, K, r in [(0, 64, 8), (4, 100, 8), (4, 32, 8), (4, 64, -1), (4, 64, 300)]:
        assert lib.qlora_merge_lora(N, K, r, p, p, p, p, 2.0, 0, p, None) == L.QL_ERR_INVALID_ARG
        assert lib.qlora_merge_lora_nf4(N, K, r, p, p, p, p, 2.0, p, p, None) == L.QL_ERR_INVALID_ARG
    assert lib.qlora_merge_lora(4, 64, 8, p, p, None, p, 2.0, 0, p, None) == L.QL_ERR_INVALID_ARG   # A missing
    assert lib.qlora_merge_lora(4, 64, 8, p, p, p, p, 2.0, 5, p, None) == L.QL_ERR_INVALID_ARG      # bad dtype
    assert lib.qlora_merge_lora_nf4(4, 64, 8, p, p, p, p, 2.0, None, p, None) == L.QL_ERR_INVALID_ARG
    assert lib.qlora_merge_lora(4, 64, 8, ctypes.c_void_p(FAKE + 2), p, p, p, 2.0, 0, p, None) == \
        L.QL_ERR_INVALID_ARG  # misaligned codes


def test_format_conversions_reject_bad_arguments_on_host(L):
    lib = L.lib()
    p = ctypes.c_void_p(FAKE)
    bad = ctypes.c_void_p(FAKE + 4)
    # double quantization: empty, null, misaligned, too little scratch
    need = lib.nf4_double_quantize_scratch_bytes(1000)
    assert need == 4 * 8 and lib.nf4_double_quantize_scratch_bytes(0) == 0
    assert lib.nf4_double_quantize(p, 0, p, p, p, p, need, None) == L.QL_ERR_INVALID_ARG
    assert lib.nf4_double_quantize(None, 1000, p, p, p, p, need, None) == L.QL_ERR_INVALID_ARG
    assert lib.nf4_double_quantize(p, 1000, p, p, bad, p, need, None) == L.QL_ERR_INVALID_ARG
    assert lib.nf4_double_quantize(p, 1000, p, p, p, p, need - 1, None) == L.QL_ERR_INVALID_ARG
    assert lib.nf4_double_dequantize(p, p, None, 1000, p, None) == L.QL_ERR_INVALID_ARG
    assert lib.nf4_double_dequantize(p, p, p, -5, p, None) == L.QL_ERR_INVALID_ARG
    # NVFP4: numel not a multiple of 16, null, misaligned, bad dtype
    assert lib.nvfp4_quantize(p, 24, p, p, p, None) == L.QL_ERR_INVALID_ARG
    assert lib.nvfp4_quantize(p, 32, p, None, p, None) == L.QL_ERR_INVALID_ARG
    assert lib.nvfp4_quantize(bad, 32, p, p, p, None) == L.QL_ERR_INVALID_ARG
    assert lib.nvfp4_dequantize(p, p, p, 32, 9, p, None) == L.QL_ERR_INVALID_ARG
    assert lib.nvfp4_dequantize(p, p, p, 0, 0, p, None) == L.QL_ERR_INVALID_ARG
    assert L.formats_launch_count() == 0  # nothing above reached a launch


def test_weight_descriptor_calls_reject_bad_weights_on_host(L):
    lib = L.lib()
    p = ctypes.c_void_p(FAKE)
    bad = FAKE + 4

    def call(w):
        return lib.qlora_linear_fwd_w(64, 256, 256, 8, p, ctypes.byref(w) if w is not None else None, p, p, 2.0, p,
                                      None, p, 1 << 30, None)
    assert call(None) == L.QL_ERR_INVALID_ARG
    assert call(L.QlWeight(7, FAKE, FAKE)) == L.QL_ERR_INVALID_ARG                       # unknown format
    assert call(L.QlWeight(L.QL_W_NF4, FAKE, None)) == L.QL_ERR_INVALID_ARG              # absmax missing
    assert call(L.QlWeight(L.QL_W_NF4_DQ, FAKE, None, FAKE, None, FAKE)) == L.QL_ERR_INVALID_ARG  # c1 missing
    assert call(L.QlWeight(L.QL_W_NVFP4, FAKE, None, None, None, None, bad, FAKE)) == L.QL_ERR_INVALID_ARG
    w = L.QlWeight(L.QL_W_NVFP4, FAKE, None, None, None, None, FAKE, FAKE)
    assert lib.qlora_linear_bwd_w(16, 12, 64, 8, p, p, ctypes.byref(w), p, p, 2.0, None, p, p, p, p, 1 << 30,
                                  None) == L.QL_ERR_INVALID_ARG                           # N % 8 != 0
    assert L.formats_launch_count() == 0 and L.launch_count() == 0


def test_gated_calls_reject_bad_arguments_on_host(L):
    lib = L.lib()
    p = ctypes.c_void_p(FAKE)
    assert lib.qlora_gate_up_fwd_swiglu(64, 24, 256, 8, p, p, p, p, p, 2.0, p, p, None, p, 1 << 30, None) == \
        L.QL_ERR_INVALID_ARG                                                               # F % 16 != 0
    assert lib.qlora_gate_up_fwd_swiglu(64, 32, 256, 8, p, p, p, p, p, 2.0, p, None, None, p, 1 << 30, None) == \
        L.QL_ERR_INVALID_ARG                                                               # h missing
    assert lib.qlora_down_bwd_dswiglu(64, 256, 32, 8, p, p, p, p, p, p, 2.0, None, None, p, p, p, p, 1 << 30,
                                      None) == L.QL_ERR_INVALID_ARG                        # gu missing
    need = lib.qlora_gated_workspace_bytes(64, 256, 32, 8, L.QL_PASS_BWD)
    assert lib.qlora_down_bwd_dswiglu(64, 256, 32, 8, p, p, p, p, p, p, 2.0, None, p, p, p, p, p, max(need, 1) - 1,
                                      None) == L.QL_ERR_INVALID_ARG                        # workspace short
    assert lib.qlora_gated_workspace_bytes(2048, 57344, 8192, 128, L.QL_PASS_FWD) == \
        L.workspace_bytes(2048, 57344, 8192, 128, L.QL_PASS_FWD)
    assert L.launch_count() == 0

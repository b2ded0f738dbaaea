"""The C-ABI library loads, exports every entry point include/fp4.h declares, and
rejects bad arguments on the host before touching a device (no GPU needed: every
call below fails validation, so nothing is launched)."""
import ctypes

import numpy as np
import pytest

import fp4_block_scaled_deterministic_b200 as fp4

OK, INVALID, SHAPE, ALIGN, CUDA, WORKSPACE = 0, 1, 2, 3, 5, 7
A16 = 1 << 20          # a 16-byte aligned fake pointer value (never dereferenced)
MIS = A16 + 8          # misaligned


@pytest.fixture(scope="module", autouse=True)
def built():
    from fp4_block_scaled_deterministic_b200 import build
    build.build()


def test_every_header_symbol_is_exported():
    syms = fp4.header_symbols()
    assert len(syms) >= 13
    L = ctypes.CDLL(fp4.LIB_PATH)
    for s in syms:
        assert hasattr(L, s), s
    assert fp4.lib().fp4_abi_version() == 2


def test_status_strings():
    for code in range(9):
        assert fp4.status_string(code)
    assert fp4.status_string(99) == "unknown status"


@pytest.mark.parametrize("rows,cols", [(32, 32), (160, 224), (128, 4096), (8192, 14336)])
@pytest.mark.parametrize("fmt", [0, 1, 2])
def test_size_queries_match_layout(orc, rows, cols, fmt):
    assert fp4.fp4_codes_bytes(rows, cols) == rows * cols // 2
    L = fp4.lib()
    assert L.fp4_codes_bytes_fmt(rows, cols, fmt) == rows * cols // (1 if fmt == 2 else 2)
    assert fp4.fp4_scales_bytes(rows, cols, fmt) == orc.scale_layout_bytes(rows, cols // orc.BLOCK[fmt])


def test_workspace_size_covers_operands():
    for p, (ra, rb, kc) in {0: (64, 96, 128), 1: (64, 128, 96), 2: (96, 128, 64)}.items():
        need = fp4.fp4_linear_workspace_size(p, 64, 96, 128, 0)
        assert need >= ra * kc // 2 + rb * kc // 2
    assert fp4.fp4_linear_workspace_size(7, 64, 96, 128, 0) == 0


def q(x=A16, codes=A16, scales=A16, ts=None, rows=64, cols=64, fmt=0, hn=16, axis=0):
    return fp4.lib().fp4_quantize(x, codes, scales, ts, rows, cols, fmt, hn, axis, None)


def test_quantize_validation():
    assert q(fmt=3) == INVALID
    assert q(hn=8) == INVALID
    assert q(axis=3) == INVALID
    assert q(rows=48) == SHAPE
    assert q(cols=40) == SHAPE
    assert q(rows=-32) == SHAPE
    assert q(x=MIS) == ALIGN
    assert q(codes=MIS) == ALIGN
    assert q(x=None) == INVALID
    assert q(scales=None) == INVALID
    assert q(ts=A16) == INVALID            # MXFP4 takes no tensor scale
    assert q(fmt=1, ts=None) == INVALID    # NVFP4 needs one
    assert q(fmt=2, ts=A16) == INVALID     # nor does the MXFP8 comparator
    assert q(rows=0) == OK and q(cols=0) == OK  # empty: nothing to do


def test_quantize_dual_validation():
    L = fp4.lib()
    assert L.fp4_quantize_dual(A16, A16, A16, None, A16, None, 64, 64, 0, 16, None) == INVALID
    assert L.fp4_quantize_dual(A16, A16, A16, A16, MIS, None, 64, 64, 0, 16, None) == ALIGN
    assert L.fp4_quantize_dual(A16, A16, A16, A16, A16, None, 64, 80, 0, 16, None) == SHAPE


def qo(opts, fmt=0, ts=None, x=A16):
    return fp4.lib().fp4_quantize_opts(x, A16, A16, ts, 64, 64, fmt, 16, 0, opts, None)


def test_quantize_opts_validation():
    L = fp4.lib()
    amax_mx = fp4.QuantOpts(A16, 0, 0, 0, 0)
    assert qo(ctypes.byref(amax_mx)) == INVALID               # a tensor amax is NVFP4 only
    mis = fp4.QuantOpts(A16 + 2, 0, 0, 0, 0)
    assert qo(ctypes.byref(mis), fmt=1, ts=A16) == ALIGN      # amax must be 4-byte aligned
    sr = fp4.QuantOpts(None, 1, 1, 5, 6)
    assert qo(ctypes.byref(sr), x=MIS) == ALIGN               # the plain checks still apply
    assert qo(ctypes.byref(sr), fmt=1, ts=None) == INVALID
    assert L.fp4_quantize_dual_opts(A16, A16, A16, None, A16, None, 64, 64, 0, 16,
                                    ctypes.byref(sr), None) == INVALID
    assert L.fp4_quantize_opts(A16, A16, A16, None, 0, 64, 0, 16, 0, ctypes.byref(sr), None) == OK
    assert qo(ctypes.byref(sr), fmt=2) == INVALID              # no variants for MXFP8


def g(A=A16, As=A16, Ats=None, B=A16, Bs=A16, Bts=None, C=A16, M=128, N=128, K=128, fmt=0, od=0):
    return fp4.lib().fp4_gemm(A, As, Ats, B, Bs, Bts, C, M, N, K, fmt, od, None)


def test_gemm_validation():
    assert g(fmt=5) == INVALID
    assert g(fmt=2, Ats=A16) == INVALID    # the MXFP8 comparator takes no tensor scales
    assert g(od=2) == INVALID
    assert g(M=100) == SHAPE
    assert g(K=48) == SHAPE
    assert g(Ats=A16) == INVALID
    assert g(fmt=1) == INVALID
    assert g(C=None) == INVALID
    assert g(B=MIS) == ALIGN
    assert g(K=0) == SHAPE
    assert g(M=0) == OK


def gq(C=A16, Qc=A16, Qs=A16, M=128, N=128, K=128, fmt=0, qhn=16):
    return fp4.lib().fp4_gemm_quant(A16, A16, None, A16, A16, None, C, Qc, Qs, M, N, K, fmt, qhn,
                                    None)


def test_gemm_quant_validation():
    assert gq(qhn=8) == INVALID
    assert gq(fmt=2) == INVALID           # the MXFP8 comparator has no fused output
    assert gq(Qc=None) == INVALID and gq(Qs=None) == INVALID
    assert gq(Qc=MIS) == ALIGN and gq(C=MIS) == ALIGN
    assert gq(N=100) == SHAPE
    assert gq(M=0) == OK


def test_gemm_group_validation():
    L = fp4.lib()
    def d(M=128, N=128, K=128, C=A16, od=0, Ats=None):
        return fp4.GemmDesc(A16, A16, Ats, A16, A16, None, C, M, N, K, od)
    arr = lambda *ds: (fp4.GemmDesc * len(ds))(*ds)
    assert L.fp4_gemm_group(None, 1, 0, None) == INVALID
    assert L.fp4_gemm_group(arr(d()), 0, 0, None) == INVALID
    assert L.fp4_gemm_group(arr(d(), d(), d(), d()), 4, 0, None) == INVALID  # above the maximum
    assert L.fp4_gemm_group(arr(d(), d(N=100)), 2, 0, None) == SHAPE
    assert L.fp4_gemm_group(arr(d(C=MIS), d()), 2, 0, None) == ALIGN
    assert L.fp4_gemm_group(arr(d(od=3)), 1, 0, None) == INVALID
    assert L.fp4_gemm_group(arr(d(Ats=A16)), 1, 0, None) == INVALID  # MXFP4 takes no scale
    assert L.fp4_gemm_group(arr(d(M=0), d(N=0)), 2, 0, None) == OK   # nothing to launch


def test_gemm_group_quant_validation():
    """The quantised member is checked as fp4_gemm_quant checks its call; the rest as
    fp4_gemm_group. Every case returns before anything is launched."""
    L = fp4.lib()
    def d(M=128, N=128, K=128, C=A16, od=1):
        return fp4.GemmDesc(A16, A16, None, A16, A16, None, C, M, N, K, od)
    arr = lambda *ds: (fp4.GemmDesc * len(ds))(*ds)
    g = lambda ds, qi=0, Qc=A16, Qs=A16, qhn=16, fmt=0: L.fp4_gemm_group_quant(
        arr(*ds), len(ds), fmt, qi, Qc, Qs, qhn, None)
    assert g([d()], qi=1) == INVALID and g([d()], qi=-1) == INVALID  # no such member
    assert g([d()], qhn=8) == INVALID
    assert g([d()], fmt=2) == INVALID                  # MXFP8 has no fused output
    assert g([d(od=0)]) == INVALID                     # the quantised member writes bf16
    assert g([d(), d(od=0)], qi=0, Qc=None) == INVALID
    assert g([d(), d(od=0)], qi=0, Qc=MIS) == ALIGN
    assert g([d(), d(N=100)], qi=0) == SHAPE           # another member's shape
    assert L.fp4_gemm_group_quant(None, 1, 0, 0, A16, A16, 16, None) == INVALID
    assert g([d(M=0), d(N=0, od=0)], qi=0) == OK       # nothing to launch


def test_linear_step_validation():
    L = fp4.lib()
    need = L.fp4_linear_step_workspace_size(64, 96, 128, 0)
    per_pass = sum(fp4.fp4_linear_workspace_size(p, 64, 96, 128, 0) for p in range(3))
    assert need >= per_pass // 2 > 0
    assert L.fp4_linear_step_workspace_size(64, 96, 128, 7) == 0
    args = lambda M=64, N=96, K=128, ws=A16, wsb=need, fmt=0, hn=16: (
        A16, A16, A16, A16, A16, A16, M, N, K, fmt, hn, ws, wsb, None)
    assert L.fp4_linear_step(*args(wsb=need - 1)) == WORKSPACE
    assert L.fp4_linear_step(*args(ws=None)) == WORKSPACE
    assert L.fp4_linear_step(*args(ws=MIS)) == ALIGN
    assert L.fp4_linear_step(*args(N=100)) == SHAPE
    assert L.fp4_linear_step(*args(fmt=9)) == INVALID
    assert L.fp4_linear_step(*args(hn=12)) == INVALID
    assert L.fp4_linear_step(*args(M=0)) == OK  # nothing to do


def test_quantize_batch_validation():
    L = fp4.lib()
    item = fp4.QuantItem(A16, A16, A16, A16, A16, None, 64, 64)
    bad_shape = fp4.QuantItem(A16, A16, A16, A16, A16, None, 64, 40)
    misaligned = fp4.QuantItem(MIS, A16, A16, A16, A16, None, 64, 64)
    arr = lambda *its: (fp4.QuantItem * len(its))(*its)
    assert L.fp4_quantize_dual_batch(None, -1, 0, 16, None) == INVALID
    assert L.fp4_quantize_dual_batch(None, 2, 0, 16, None) == INVALID
    assert L.fp4_quantize_dual_batch(None, 0, 0, 16, None) == OK
    assert L.fp4_quantize_dual_batch(arr(item, bad_shape), 2, 0, 16, None) == SHAPE
    assert L.fp4_quantize_dual_batch(arr(item, misaligned), 2, 0, 16, None) == ALIGN
    assert L.fp4_quantize_dual_batch(arr(item), 1, 0, 12, None) == INVALID
    assert L.fp4_quantize_dual_batch(arr(item), 1, 1, 16, None) == INVALID  # NVFP4 needs scales


def test_linear_validation():
    L = fp4.lib()
    need = fp4.fp4_linear_workspace_size(0, 64, 64, 64, 0)
    assert L.fp4_linear_fprop(A16, A16, A16, 64, 64, 64, 0, 16, 1, A16, need - 1, None) == WORKSPACE
    assert L.fp4_linear_fprop(A16, A16, A16, 64, 64, 64, 0, 16, 1, None, need, None) == WORKSPACE
    assert L.fp4_linear_dgrad(A16, A16, A16, 64, 64, 64, 0, 12, 1, A16, need, None) == INVALID
    assert L.fp4_linear_wgrad(A16, A16, A16, 64, 40, 64, 0, 16, 1, A16, need, None) == SHAPE
    assert L.fp4_linear_wgrad(A16, A16, A16, 64, 64, 64, 0, 16, 1, MIS, need, None) == ALIGN


def test_valid_call_without_gpu_reports_cuda_or_device_error():
    """With valid arguments and no usable device the call fails cleanly (no crash)."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert q() in (CUDA, 4)

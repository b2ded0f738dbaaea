"""Python binding of libfp4, the B200 (sm_100a) library for the 4-bit linear layer of
FP4 LLM pre-training: deterministic block Hadamard rotation (H16/H32) along the
contraction axis, MXFP4/NVFP4 microscaled quantisation, and the block-scaled FP4
GEMM for the Fprop, Dgrad and Wgrad passes.

This module only marshals arguments: torch provides device memory and the current
CUDA stream, every step of the computation runs in the library's kernels (see
``include/fp4.h`` for the C ABI). If ``libfp4.so`` is missing or cannot be loaded
every call raises; there is no fallback path.

The functions named ``fp4_*`` mirror the C entry points one for one (pointers as
ints); the lower-case helpers allocate outputs with torch and call them.
"""
from __future__ import annotations

import ctypes
import os
import re
from dataclasses import dataclass

import torch

MXFP4, NVFP4, MXFP8 = 0, 1, 2  # MXFP8: the FP8 comparator (E4M3 codes, one byte each)
ROW, COL = 0, 1
OUT_F32, OUT_BF16 = 0, 1
FPROP, DGRAD, WGRAD = 0, 1, 2
BLOCK = {MXFP4: 32, NVFP4: 16, MXFP8: 32}

_PKG = os.path.dirname(os.path.abspath(__file__))
# FP4_DEBUG_BOUNDS=1 in the environment selects the debug build (device-side range
# checks; fp4_check_status reports FP4_ERR_BOUNDS), same ABI and results.
LIB_PATH = os.path.join(_PKG, "libfp4_debug.so" if os.environ.get("FP4_DEBUG_BOUNDS") == "1"
                        else "libfp4.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "fp4.h")

STATUS = {0: "FP4_OK", 1: "FP4_ERR_INVALID_ARG", 2: "FP4_ERR_SHAPE", 3: "FP4_ERR_ALIGN",
          4: "FP4_ERR_UNSUPPORTED_DEVICE", 5: "FP4_ERR_CUDA", 6: "FP4_ERR_TIMEOUT",
          7: "FP4_ERR_WORKSPACE", 8: "FP4_ERR_BOUNDS"}


class Fp4Error(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)} ({status_string(code)})")


class QuantItem(ctypes.Structure):
    """fp4_quant_item of include/fp4.h (one tensor of fp4_quantize_dual_batch)."""
    _fields_ = [("x_bf16", ctypes.c_void_p), ("row_codes", ctypes.c_void_p),
                ("row_scales", ctypes.c_void_p), ("col_codes", ctypes.c_void_p),
                ("col_scales", ctypes.c_void_p), ("tensor_scale", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64)]


class GemmDesc(ctypes.Structure):
    """fp4_gemm_desc of include/fp4.h (one GEMM of fp4_gemm_group)."""
    _fields_ = [("A_codes", ctypes.c_void_p), ("A_scales", ctypes.c_void_p),
                ("A_tensor_scale", ctypes.c_void_p), ("B_codes", ctypes.c_void_p),
                ("B_scales", ctypes.c_void_p), ("B_tensor_scale", ctypes.c_void_p),
                ("C", ctypes.c_void_p), ("M", ctypes.c_int64), ("N", ctypes.c_int64),
                ("K", ctypes.c_int64), ("out_dtype", ctypes.c_int)]


GEMM_GROUP_MAX = 3


class QuantOpts(ctypes.Structure):
    """fp4_quant_opts of include/fp4.h (host struct passed by pointer)."""
    _fields_ = [("amax", ctypes.c_void_p), ("stochastic", ctypes.c_int),
                ("random_signs", ctypes.c_int), ("sr_seed", ctypes.c_uint64),
                ("sign_seed", ctypes.c_uint64)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libfp4.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{os.path.basename(LIB_PATH)} not built at {LIB_PATH}; run "
                               "python -m fp4_block_scaled_deterministic_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, I32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        sig = {
            "fp4_abi_version": (I32, []),
            "fp4_codes_bytes": (SZ, [I64, I64]),
            "fp4_codes_bytes_fmt": (SZ, [I64, I64, I32]),
            "fp4_scales_bytes": (SZ, [I64, I64, I32]),
            "fp4_quantize": (I32, [P, P, P, P, I64, I64, I32, I32, I32, P]),
            "fp4_quantize_dual": (I32, [P, P, P, P, P, P, I64, I64, I32, I32, P]),
            "fp4_quantize_opts": (I32, [P, P, P, P, I64, I64, I32, I32, I32,
                                        ctypes.POINTER(QuantOpts), P]),
            "fp4_quantize_dual_opts": (I32, [P, P, P, P, P, P, I64, I64, I32, I32,
                                             ctypes.POINTER(QuantOpts), P]),
            "fp4_quantize_dual_batch": (I32, [ctypes.POINTER(QuantItem), I32, I32, I32, P]),
            "fp4_gemm": (I32, [P, P, P, P, P, P, P, I64, I64, I64, I32, I32, P]),
            "fp4_gemm_quant": (I32, [P, P, P, P, P, P, P, P, P, I64, I64, I64, I32, I32, P]),
            "fp4_gemm_group": (I32, [ctypes.POINTER(GemmDesc), I32, I32, P]),
            "fp4_gemm_group_quant": (I32, [ctypes.POINTER(GemmDesc), I32, I32, I32, P, P, I32, P]),
            "fp4_linear_workspace_size": (SZ, [I32, I64, I64, I64, I32]),
            "fp4_linear_fprop": (I32, [P, P, P, I64, I64, I64, I32, I32, I32, P, SZ, P]),
            "fp4_linear_dgrad": (I32, [P, P, P, I64, I64, I64, I32, I32, I32, P, SZ, P]),
            "fp4_linear_wgrad": (I32, [P, P, P, I64, I64, I64, I32, I32, I32, P, SZ, P]),
            "fp4_linear_fprop_noalloc": (I32, [P, P, P, I64, I64, I64, I32, I32, I32, P]),
            "fp4_linear_step_workspace_size": (SZ, [I64, I64, I64, I32]),
            "fp4_linear_step": (I32, [P, P, P, P, P, P, I64, I64, I64, I32, I32, P, SZ, P]),
            "fp4_check_status": (I32, [P]),
            "fp4_selftest_timeout": (I32, [ctypes.c_uint64, P]),
            "fp4_status_string": (ctypes.c_char_p, [I32]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def header_symbols() -> list[str]:
    """Entry points declared in include/fp4.h."""
    text = open(HEADER_PATH).read()
    return re.findall(r"^FP4_API\s+[\w\s\*]*?\b(fp4_\w+)\s*\(", text, flags=re.M)


def status_string(code: int) -> str:
    return lib().fp4_status_string(code).decode()


def _check(code: int, where: str):
    if code != 0:
        raise Fp4Error(code, where)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream=None) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


# ---------------------------------------------------------------- C entry points

def fp4_codes_bytes(rows: int, cols: int) -> int:
    return lib().fp4_codes_bytes(rows, cols)


def fp4_scales_bytes(rows: int, cols: int, fmt: int) -> int:
    return lib().fp4_scales_bytes(rows, cols, fmt)


def fp4_linear_workspace_size(pass_: int, M: int, N: int, K: int, fmt: int) -> int:
    return lib().fp4_linear_workspace_size(pass_, M, N, K, fmt)


def fp4_quantize(x, codes, scales, tensor_scale, rows, cols, fmt, hadamard_n, axis, stream=None):
    return lib().fp4_quantize(_ptr(x), _ptr(codes), _ptr(scales), _ptr(tensor_scale), rows, cols,
                              fmt, hadamard_n, axis, _stream(stream))


def fp4_quantize_dual(x, row_codes, row_scales, col_codes, col_scales, tensor_scale, rows, cols,
                      fmt, hadamard_n, stream=None):
    return lib().fp4_quantize_dual(_ptr(x), _ptr(row_codes), _ptr(row_scales), _ptr(col_codes),
                                   _ptr(col_scales), _ptr(tensor_scale), rows, cols, fmt,
                                   hadamard_n, _stream(stream))


def fp4_quantize_dual_batch(items, fmt, hadamard_n, stream=None):
    """items: a sequence of (x, row_codes, row_scales, col_codes, col_scales, tensor_scale,
    rows, cols) -- tensors or pointers as for fp4_quantize_dual."""
    arr = (QuantItem * len(items))(*[QuantItem(*[_ptr(v) for v in it[:6]], it[6], it[7])
                                     for it in items])
    return lib().fp4_quantize_dual_batch(arr, len(items), fmt, hadamard_n, _stream(stream))


def fp4_gemm_group(descs, fmt, stream=None):
    """descs: a sequence of (A_codes, A_scales, A_tensor_scale, B_codes, B_scales,
    B_tensor_scale, C, M, N, K, out_dtype) -- tensors or pointers as for fp4_gemm."""
    arr = (GemmDesc * max(1, len(descs)))(*[GemmDesc(*[_ptr(v) for v in d[:7]], *d[7:11])
                                            for d in descs])
    return lib().fp4_gemm_group(arr, len(descs), fmt, _stream(stream))


def fp4_gemm_group_quant(descs, fmt, q_index, Q_codes, Q_scales, q_hadamard_n, stream=None):
    """fp4_gemm_group whose member q_index also quantises its bf16 output (as
    fp4_gemm_quant) into Q_codes / Q_scales."""
    arr = (GemmDesc * max(1, len(descs)))(*[GemmDesc(*[_ptr(v) for v in d[:7]], *d[7:11])
                                            for d in descs])
    return lib().fp4_gemm_group_quant(arr, len(descs), fmt, q_index, _ptr(Q_codes),
                                      _ptr(Q_scales), q_hadamard_n, _stream(stream))


def _opts(opts):
    return None if opts is None else ctypes.byref(opts)


def fp4_quantize_opts(x, codes, scales, tensor_scale, rows, cols, fmt, hadamard_n, axis, opts,
                      stream=None):
    return lib().fp4_quantize_opts(_ptr(x), _ptr(codes), _ptr(scales), _ptr(tensor_scale), rows,
                                   cols, fmt, hadamard_n, axis, _opts(opts), _stream(stream))


def fp4_quantize_dual_opts(x, row_codes, row_scales, col_codes, col_scales, tensor_scale, rows,
                           cols, fmt, hadamard_n, opts, stream=None):
    return lib().fp4_quantize_dual_opts(_ptr(x), _ptr(row_codes), _ptr(row_scales),
                                        _ptr(col_codes), _ptr(col_scales), _ptr(tensor_scale),
                                        rows, cols, fmt, hadamard_n, _opts(opts), _stream(stream))


def fp4_gemm(A, As, Ats, B, Bs, Bts, C, M, N, K, fmt, out_dtype, stream=None):
    return lib().fp4_gemm(_ptr(A), _ptr(As), _ptr(Ats), _ptr(B), _ptr(Bs), _ptr(Bts), _ptr(C), M,
                          N, K, fmt, out_dtype, _stream(stream))


def fp4_gemm_quant(A, As, Ats, B, Bs, Bts, C, Qc, Qs, M, N, K, fmt, q_hn, stream=None):
    return lib().fp4_gemm_quant(_ptr(A), _ptr(As), _ptr(Ats), _ptr(B), _ptr(Bs), _ptr(Bts),
                                _ptr(C), _ptr(Qc), _ptr(Qs), M, N, K, fmt, q_hn, _stream(stream))


def fp4_linear_fprop(X, W, Y, M, N, K, fmt, hn, out_dtype, ws, ws_bytes, stream=None):
    return lib().fp4_linear_fprop(_ptr(X), _ptr(W), _ptr(Y), M, N, K, fmt, hn, out_dtype, _ptr(ws),
                                  ws_bytes, _stream(stream))


def fp4_linear_dgrad(dY, W, dX, M, N, K, fmt, hn, out_dtype, ws, ws_bytes, stream=None):
    return lib().fp4_linear_dgrad(_ptr(dY), _ptr(W), _ptr(dX), M, N, K, fmt, hn, out_dtype,
                                  _ptr(ws), ws_bytes, _stream(stream))


def fp4_linear_wgrad(dY, X, dW, M, N, K, fmt, hn, out_dtype, ws, ws_bytes, stream=None):
    return lib().fp4_linear_wgrad(_ptr(dY), _ptr(X), _ptr(dW), M, N, K, fmt, hn, out_dtype,
                                  _ptr(ws), ws_bytes, _stream(stream))


def fp4_linear_fprop_noalloc(X, W, Y, M, N, K, fmt, hn, out_dtype, stream=None):
    """fp4_linear_fprop on the library's static scratch (no workspace argument), for
    callers that cannot allocate device memory; see include/fp4.h for its limit."""
    return lib().fp4_linear_fprop_noalloc(_ptr(X), _ptr(W), _ptr(Y), M, N, K, fmt, hn, out_dtype,
                                          _stream(stream))


def fp4_check_status(stream=None) -> int:
    return lib().fp4_check_status(_stream(stream))


def fp4_selftest_timeout(timeout_ns: int, stream=None) -> int:
    return lib().fp4_selftest_timeout(timeout_ns, _stream(stream))


# ---------------------------------------------------------------- torch helpers

@dataclass
class QTensor:
    """A quantised [rows][cols] matrix (cols = contraction axis)."""
    codes: torch.Tensor          # uint8 [rows][cols/2]
    scales: torch.Tensor         # uint8, atom layout
    tensor_scale: torch.Tensor | None  # float32 view of S (NVFP4), else None
    fmt: int
    rows: int
    cols: int


def _alloc_q(rows, cols, fmt, device):
    codes = torch.empty(rows, cols if fmt == MXFP8 else cols // 2, dtype=torch.uint8,
                        device=device)
    scales = torch.empty(max(1, fp4_scales_bytes(rows, cols, fmt)), dtype=torch.uint8, device=device)
    return codes, scales


def quant_opts(amax: torch.Tensor | None = None, sr_seed: int | None = None,
               sign_seed: int | None = None) -> QuantOpts | None:
    """Options of the quantiser variants (None when none is asked for): a device fp32
    tensor amax per layout, stochastic rounding keyed by sr_seed, random Hadamard signs
    keyed by sign_seed."""
    if amax is None and sr_seed is None and sign_seed is None:
        return None
    if amax is not None:
        assert amax.dtype == torch.float32 and amax.is_cuda
    return QuantOpts(None if amax is None else amax.data_ptr(), int(sr_seed is not None),
                     int(sign_seed is not None), sr_seed or 0, sign_seed or 0)


def quantize(x: torch.Tensor, fmt: int = MXFP4, hadamard_n: int = 16, axis: int = ROW,
             ts_buf: torch.Tensor | None = None, amax: torch.Tensor | None = None,
             sr_seed: int | None = None, sign_seed: int | None = None) -> QTensor:
    """Rotate and quantise a bf16 CUDA matrix along `axis` (COL returns the transposed
    layout [cols][rows/2]). amax / sr_seed / sign_seed select the variants of
    fp4_quantize_opts."""
    assert x.dtype == torch.bfloat16 and x.is_cuda and x.dim() == 2
    x = x.contiguous()
    rows, cols = x.shape
    R, C = (rows, cols) if axis == ROW else (cols, rows)
    codes, scales = _alloc_q(R, C, fmt, x.device)
    ts = None
    if fmt == NVFP4:
        ts = ts_buf if ts_buf is not None else torch.zeros(2, dtype=torch.float32, device=x.device)
    opts = quant_opts(amax, sr_seed, sign_seed)
    if opts is None:
        _check(fp4_quantize(x, codes, scales, ts, rows, cols, fmt, hadamard_n, axis),
               "fp4_quantize")
    else:
        _check(fp4_quantize_opts(x, codes, scales, ts, rows, cols, fmt, hadamard_n, axis, opts),
               "fp4_quantize_opts")
    return QTensor(codes, scales, None if ts is None else ts[0:1], fmt, R, C)


def quantize_dual(x: torch.Tensor, fmt: int = MXFP4, hadamard_n: int = 16,
                  amax: torch.Tensor | None = None, sr_seed: int | None = None,
                  sign_seed: int | None = None):
    """Row-wise and column-wise (transposed) quantisation from one read of x."""
    assert x.dtype == torch.bfloat16 and x.is_cuda and x.dim() == 2
    x = x.contiguous()
    rows, cols = x.shape
    rc, rs = _alloc_q(rows, cols, fmt, x.device)
    cc, cs = _alloc_q(cols, rows, fmt, x.device)
    ts = torch.zeros(4, dtype=torch.float32, device=x.device) if fmt == NVFP4 else None
    opts = quant_opts(amax, sr_seed, sign_seed)
    if opts is None:
        _check(fp4_quantize_dual(x, rc, rs, cc, cs, ts, rows, cols, fmt, hadamard_n),
               "fp4_quantize_dual")
    else:
        _check(fp4_quantize_dual_opts(x, rc, rs, cc, cs, ts, rows, cols, fmt, hadamard_n, opts),
               "fp4_quantize_dual_opts")
    return (QTensor(rc, rs, None if ts is None else ts[0:1], fmt, rows, cols),
            QTensor(cc, cs, None if ts is None else ts[1:2], fmt, cols, rows))


def quantize_dual_batch(xs, fmt: int = MXFP4, hadamard_n: int = 16):
    """quantize_dual of every bf16 CUDA matrix in xs, in as few launches as possible.
    Returns [(row QTensor, column QTensor), ...] in the order of xs."""
    items, outs = [], []
    for x in xs:
        assert x.dtype == torch.bfloat16 and x.is_cuda and x.dim() == 2
        x = x.contiguous()
        rows, cols = x.shape
        rc, rs = _alloc_q(rows, cols, fmt, x.device)
        cc, cs = _alloc_q(cols, rows, fmt, x.device)
        ts = torch.zeros(4, dtype=torch.float32, device=x.device) if fmt == NVFP4 else None
        items.append((x, rc, rs, cc, cs, ts, rows, cols))
        outs.append((QTensor(rc, rs, None if ts is None else ts[0:1], fmt, rows, cols),
                     QTensor(cc, cs, None if ts is None else ts[1:2], fmt, cols, rows)))
    _check(fp4_quantize_dual_batch(items, fmt, hadamard_n), "fp4_quantize_dual_batch")
    return outs


def gemm(a: QTensor, b: QTensor, out_dtype: int = OUT_F32, out: torch.Tensor | None = None):
    """C[M][N] = deq(a) @ deq(b)^T on the FP4 tensor cores."""
    assert a.fmt == b.fmt and a.cols == b.cols
    M, N, K = a.rows, b.rows, a.cols
    if out is None:
        dt = torch.float32 if out_dtype == OUT_F32 else torch.bfloat16
        out = torch.empty(M, N, dtype=dt, device=a.codes.device)
    _check(fp4_gemm(a.codes, a.scales, a.tensor_scale, b.codes, b.scales, b.tensor_scale, out, M,
                    N, K, a.fmt, out_dtype), "fp4_gemm")
    return out


def linear_step(X: torch.Tensor, W: torch.Tensor, dY: torch.Tensor, fmt: int = MXFP4,
                hadamard_n: int = 16, ws: torch.Tensor | None = None):
    """Fprop, Dgrad and Wgrad of one linear layer (fp4_linear_step): returns
    (Y bf16 [M][N], dX bf16 [M][K], dW fp32 [N][K])."""
    M, K = X.shape
    N = W.shape[0]
    assert W.shape == (N, K) and dY.shape == (M, N)
    dev = X.device
    need = lib().fp4_linear_step_workspace_size(M, N, K, fmt)
    if ws is None:
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    dX = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    dW = torch.empty(N, K, dtype=torch.float32, device=dev)
    _check(lib().fp4_linear_step(_ptr(X.contiguous()), _ptr(W.contiguous()),
                                 _ptr(dY.contiguous()), _ptr(Y), _ptr(dX), _ptr(dW), M, N, K,
                                 fmt, hadamard_n, _ptr(ws), ws.numel(), _stream(None)),
           "fp4_linear_step")
    return Y, dX, dW


def gemm_group(problems, out_dtypes=None):
    """Several GEMMs of one format in one launch: problems is a sequence of (a, b) QTensor
    pairs (or (a, b, out) with out a preallocated output); returns the outputs, each equal
    bit for bit to gemm(a, b, out_dtype)."""
    assert 1 <= len(problems) <= GEMM_GROUP_MAX
    fmt = problems[0][0].fmt
    outs, descs = [], []
    for i, pr in enumerate(problems):
        a, b = pr[0], pr[1]
        assert a.fmt == b.fmt == fmt and a.cols == b.cols
        od = OUT_F32 if out_dtypes is None else out_dtypes[i]
        out = pr[2] if len(pr) > 2 else torch.empty(
            a.rows, b.rows, dtype=torch.float32 if od == OUT_F32 else torch.bfloat16,
            device=a.codes.device)
        outs.append(out)
        descs.append((a.codes, a.scales, a.tensor_scale, b.codes, b.scales, b.tensor_scale,
                      out, a.rows, b.rows, a.cols, od))
    _check(fp4_gemm_group(descs, fmt), "fp4_gemm_group")
    return outs


def gemm_group_quant(problems, out_dtypes, q_index, q_hn=16):
    """gemm_group in one launch whose member q_index (a bf16 output) also has its output
    quantised row-wise as gemm_quant does. Returns (outputs, QTensor of that output)."""
    assert 1 <= len(problems) <= GEMM_GROUP_MAX and 0 <= q_index < len(problems)
    fmt = problems[0][0].fmt
    outs, descs = [], []
    for i, (a, b) in enumerate(problems):
        assert a.fmt == b.fmt == fmt and a.cols == b.cols
        od = out_dtypes[i]
        out = torch.empty(a.rows, b.rows, dtype=torch.float32 if od == OUT_F32 else torch.bfloat16,
                          device=a.codes.device)
        outs.append(out)
        descs.append((a.codes, a.scales, a.tensor_scale, b.codes, b.scales, b.tensor_scale,
                      out, a.rows, b.rows, a.cols, od))
    M, N = problems[q_index][0].rows, problems[q_index][1].rows
    codes, scales = _alloc_q(M, N, MXFP4, problems[q_index][0].codes.device)
    _check(fp4_gemm_group_quant(descs, fmt, q_index, codes, scales, q_hn), "fp4_gemm_group_quant")
    return outs, QTensor(codes, scales, None, MXFP4, M, N)


def gemm_quant(a: QTensor, b: QTensor, q_hn: int = 16, with_output: bool = True):
    """Y = RN_bf16(deq(a) @ deq(b)^T) and its row-wise MXFP4 quantisation (rotation q_hn
    along N) from the same epilogue. Returns (Y or None, QTensor of Y)."""
    assert a.fmt == b.fmt and a.cols == b.cols
    M, N, K = a.rows, b.rows, a.cols
    dev = a.codes.device
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev) if with_output else None
    codes, scales = _alloc_q(M, N, MXFP4, dev)
    _check(fp4_gemm_quant(a.codes, a.scales, a.tensor_scale, b.codes, b.scales, b.tensor_scale,
                          Y, codes, scales, M, N, K, a.fmt, q_hn), "fp4_gemm_quant")
    return Y, QTensor(codes, scales, None, MXFP4, M, N)


def _linear(pass_, P, Q, out_shape, M, N, K, fmt, hn, out_dtype, ws, out):
    dt = torch.float32 if out_dtype == OUT_F32 else torch.bfloat16
    if out is None:
        out = torch.empty(*out_shape, dtype=dt, device=P.device)
    need = fp4_linear_workspace_size(pass_, M, N, K, fmt)
    if ws is None:
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device=P.device)
    fn = {FPROP: fp4_linear_fprop, DGRAD: fp4_linear_dgrad, WGRAD: fp4_linear_wgrad}[pass_]
    _check(fn(P.contiguous(), Q.contiguous(), out, M, N, K, fmt, hn, out_dtype, ws, ws.numel()),
           fn.__name__)
    return out


def linear_fprop(X, W, fmt=MXFP4, hn=16, out_dtype=OUT_BF16, ws=None, out=None):
    """Y [M][N] = Q(X) Q(W)^T, contraction over K."""
    (M, K), N = X.shape, W.shape[0]
    return _linear(FPROP, X, W, (M, N), M, N, K, fmt, hn, out_dtype, ws, out)


def linear_dgrad(dY, W, fmt=MXFP4, hn=16, out_dtype=OUT_BF16, ws=None, out=None):
    """dX [M][K] = Q(dY) Q(W along N)^T, contraction over N."""
    (M, N), K = dY.shape, W.shape[1]
    return _linear(DGRAD, dY, W, (M, K), M, N, K, fmt, hn, out_dtype, ws, out)


def linear_wgrad(dY, X, fmt=MXFP4, hn=16, out_dtype=OUT_F32, ws=None, out=None):
    """dW [N][K] = Q(dY along M)^T-layout . Q(X along M), contraction over the tokens."""
    (M, N), K = dY.shape, X.shape[1]
    return _linear(WGRAD, dY, X, (N, K), M, N, K, fmt, hn, out_dtype, ws, out)


def check_status(stream=None):
    _check(fp4_check_status(stream), "fp4_check_status")

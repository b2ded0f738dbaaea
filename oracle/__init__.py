"""CPU oracle for the rotate -> FP4-quantise -> block-scaled GEMM path.

TEST INFRASTRUCTURE. Only the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. It shares no code with
the CUDA library (``fp4_block_scaled_deterministic_b200``) and never imports it.

The arithmetic lives in ``fp4_oracle.c`` (plain scalar C, fp32 where the method
computes in fp32, fp64 for the GEMM reference); this module only compiles it with
gcc and marshals numpy arrays. See the header of ``fp4_oracle.c`` for the pages
each step follows and for every reading taken where the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

MXFP4, NVFP4, MXFP8 = 0, 1, 2
ROW, COL = 0, 1
BLOCK = {MXFP4: 32, NVFP4: 16, MXFP8: 32}

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp4_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_LIB_OMP = os.path.join(_HERE, "liboracle_omp.so")
_lib = None
_libs = {}
_threads = 1


def _compile(out: str, extra) -> None:
    if os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(_SRC):
        return
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
           "-shared", *extra, _SRC, "-o", out + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)


def build(force: bool = False) -> str:
    """Compile fp4_oracle.c with gcc, twice: serial (liboracle.so, the default) and
    with OpenMP (liboracle_omp.so, for the all-core CPU baseline; its pragmas only
    split independent rows or entries). No fast-math and no FP contraction, so every
    fp32 operation rounds once, as IEEE 754 prescribes."""
    if force:
        for f in (_LIB, _LIB_OMP):
            if os.path.exists(f):
                os.remove(f)
    _compile(_LIB, [])
    _compile(_LIB_OMP, ["-fopenmp"])
    return _LIB


def set_threads(n: int) -> int:
    """Run the oracle on n host threads from now on (1 = the serial build, the
    default; n > 1 = the OpenMP build). Returns the thread count in use."""
    global _lib, _threads
    _threads = max(1, int(n))
    _lib = None
    return _L().fp4o_set_threads(_threads)


def _L():
    global _lib
    if _lib is None:
        build()
        path = _LIB if _threads == 1 else _LIB_OMP
        if path in _libs:
            _lib = _libs[path]
            _lib.fp4o_set_threads(_threads)
            return _lib
        lib = ctypes.CDLL(path)
        lib.fp4o_set_threads.restype = ctypes.c_int
        lib.fp4o_set_threads.argtypes = [ctypes.c_int]
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        lib.fp4o_e2m1_decode.restype = ctypes.c_double
        lib.fp4o_e2m1_decode.argtypes = [ctypes.c_uint8]
        lib.fp4o_e2m1_encode.restype = ctypes.c_uint8
        lib.fp4o_e2m1_encode.argtypes = [ctypes.c_float]
        lib.fp4o_mx_scale_exponent.restype = ctypes.c_int
        lib.fp4o_mx_scale_exponent.argtypes = [ctypes.c_float]
        lib.fp4o_e4m3_decode.restype = ctypes.c_double
        lib.fp4o_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.fp4o_e4m3_encode.restype = ctypes.c_uint8
        lib.fp4o_e4m3_encode.argtypes = [ctypes.c_float]
        lib.fp4o_hadamard_scale.restype = ctypes.c_float
        lib.fp4o_hadamard_scale.argtypes = [ctypes.c_int]
        lib.fp4o_fwht_f32.restype = None
        lib.fp4o_fwht_f32.argtypes = [P, ctypes.c_int]
        lib.fp4o_rotate.restype = ctypes.c_int
        lib.fp4o_rotate.argtypes = [P, i64, i64, ctypes.c_int, ctypes.c_int, P]
        lib.fp4o_scale_layout_bytes.restype = i64
        lib.fp4o_scale_layout_bytes.argtypes = [i64, i64]
        lib.fp4o_scale_offset.restype = i64
        lib.fp4o_scale_offset.argtypes = [i64, i64, i64]
        lib.fp4o_quantize_block_mx.restype = None
        lib.fp4o_quantize_block_mx.argtypes = [P, ctypes.c_int, P, P]
        lib.fp4o_quantize_block_nv.restype = None
        lib.fp4o_quantize_block_nv.argtypes = [P, ctypes.c_int, ctypes.c_float, P, P]
        lib.fp4o_nv_tensor_scale.restype = ctypes.c_float
        lib.fp4o_nv_tensor_scale.argtypes = [ctypes.c_float]
        lib.fp4o_quantize.restype = ctypes.c_int
        lib.fp4o_quantize.argtypes = [P, i64, i64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                      P, P, P, P]
        lib.fp4o_quantize_ex.restype = ctypes.c_int
        lib.fp4o_quantize_ex.argtypes = [P, i64, i64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         P, P, P, P, P]
        lib.fp4o_quantize_mxfp8.restype = ctypes.c_int
        lib.fp4o_quantize_mxfp8.argtypes = [P, i64, i64, ctypes.c_int, ctypes.c_int, P, P]
        lib.fp4o_rotated_amax.restype = ctypes.c_float
        lib.fp4o_rotated_amax.argtypes = [P, i64, i64, ctypes.c_int, ctypes.c_int]
        u64, u32 = ctypes.c_uint64, ctypes.c_uint32
        lib.fp4o_rotated_amax_opt.restype = ctypes.c_float
        lib.fp4o_rotated_amax_opt.argtypes = [P, i64, i64, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int, u64]
        lib.fp4o_rotate_opt.restype = ctypes.c_int
        lib.fp4o_rotate_opt.argtypes = [P, i64, i64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        u64, P]
        lib.fp4o_quantize_opt.restype = ctypes.c_int
        lib.fp4o_quantize_opt.argtypes = [P, i64, i64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          P, ctypes.c_int, u64, ctypes.c_int, u64, P, P, P, P]
        lib.fp4o_philox4x32_10.restype = None
        lib.fp4o_philox4x32_10.argtypes = [P, P, P]
        lib.fp4o_philox_word.restype = u32
        lib.fp4o_philox_word.argtypes = [u64, u64, u32]
        lib.fp4o_e2m1_encode_sr.restype = ctypes.c_uint8
        lib.fp4o_e2m1_encode_sr.argtypes = [ctypes.c_float, u32]
        lib.fp4o_rht_negate.restype = ctypes.c_int
        lib.fp4o_rht_negate.argtypes = [u64, i64]
        lib.fp4o_dequantize.restype = None
        lib.fp4o_dequantize.argtypes = [P, P, ctypes.c_float, i64, i64, ctypes.c_int, P]
        lib.fp4o_gemm_f64.restype = None
        lib.fp4o_gemm_f64.argtypes = [P, P, P, i64, i64, i64]
        lib.fp4o_gemm_entries.restype = None
        lib.fp4o_gemm_entries.argtypes = [P, P, ctypes.c_float, P, P, ctypes.c_float, i64,
                                          ctypes.c_int, P, P, i64, P]
        for name, t_in, t_out in (("fp4o_e2m1_encode_array", P, P),
                                  ("fp4o_e4m3_encode_array", P, P),
                                  ("fp4o_mx_scale_exponent_array", P, P)):
            f = getattr(lib, name)
            f.restype = None
            f.argtypes = [t_in, t_out, i64]
        lib.fp4o_set_threads(_threads)
        _libs[path] = lib
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


# ----------------------------------------------------------------- scalar codecs

def e2m1_decode(nibble: int) -> float:
    return _L().fp4o_e2m1_decode(nibble)


def e2m1_encode(q) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.float32)
    out = np.empty(q.shape, np.uint8)
    _L().fp4o_e2m1_encode_array(_ptr(q), _ptr(out), q.size)
    return out


def e4m3_decode(code: int) -> float:
    return _L().fp4o_e4m3_decode(code)


def e4m3_encode(t) -> np.ndarray:
    t = np.ascontiguousarray(t, dtype=np.float32)
    out = np.empty(t.shape, np.uint8)
    _L().fp4o_e4m3_encode_array(_ptr(t), _ptr(out), t.size)
    return out


def mx_scale_exponent(amax) -> np.ndarray:
    a = np.ascontiguousarray(amax, dtype=np.float32)
    out = np.empty(a.shape, np.int32)
    _L().fp4o_mx_scale_exponent_array(_ptr(a), _ptr(out), a.size)
    return out


def hadamard_scale(n: int) -> float:
    return _L().fp4o_hadamard_scale(n)


def fwht(v) -> np.ndarray:
    """Normalised in-place FWHT of one fp32 group (length a power of two)."""
    v = np.array(v, dtype=np.float32, copy=True)
    _L().fp4o_fwht_f32(_ptr(v), v.size)
    return v


def scale_offset(r: int, kb: int, kblocks: int) -> int:
    return _L().fp4o_scale_offset(r, kb, kblocks)


def scale_layout_bytes(rows: int, kblocks: int) -> int:
    return _L().fp4o_scale_layout_bytes(rows, kblocks)


def quantize_block_mx(v, bs=None):
    v = np.ascontiguousarray(v, dtype=np.float32)
    bs = v.size if bs is None else bs
    codes = np.empty(bs, np.uint8)
    sb = np.zeros(1, np.uint8)
    _L().fp4o_quantize_block_mx(_ptr(v), bs, _ptr(codes), _ptr(sb))
    return codes, int(sb[0])


def quantize_block_nv(v, S: float, bs=None):
    v = np.ascontiguousarray(v, dtype=np.float32)
    bs = v.size if bs is None else bs
    codes = np.empty(bs, np.uint8)
    sb = np.zeros(1, np.uint8)
    _L().fp4o_quantize_block_nv(_ptr(v), bs, S, _ptr(codes), _ptr(sb))
    return codes, int(sb[0])


def nv_tensor_scale(amax: float) -> float:
    return _L().fp4o_nv_tensor_scale(amax)


# ----------------------------------------------------------------- tensors

def _bf16_bits(x) -> np.ndarray:
    """Accept a uint16 array of bf16 bit patterns or a torch bf16 CPU tensor."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch  # plumbing only: reinterpret bits
    assert x.dtype == torch.bfloat16 and x.device.type == "cpu"
    return np.ascontiguousarray(x.contiguous().view(torch.int16).numpy().view(np.uint16))


def rotate(x, hn: int, axis: int = ROW, rht_seed: int | None = None) -> np.ndarray:
    """Widened and rotated matrix ([R][C], transposed for COL); with rht_seed the random
    signs of the randomised Hadamard variant are applied before the rotation."""
    xb = _bf16_bits(x)
    rows, cols = xb.shape
    R, C = (rows, cols) if axis == ROW else (cols, rows)
    out = np.empty((R, C), np.float32)
    if _L().fp4o_rotate_opt(_ptr(xb), rows, cols, hn, axis, rht_seed is not None,
                            rht_seed or 0, _ptr(out)) != 0:
        raise ValueError("rotation group does not divide the axis")
    return out


def rotated_amax(x, hn: int, axis: int = ROW, rht_seed: int | None = None) -> float:
    """max |v| over the rotated matrix (NVFP4 tensor amax), computed row by row."""
    xb = _bf16_bits(x)
    rows, cols = xb.shape
    return float(_L().fp4o_rotated_amax_opt(_ptr(xb), rows, cols, hn, axis,
                                            rht_seed is not None, rht_seed or 0))


# ----------------------------------------------------------------- random words

def philox4x32_10(ctr, key) -> np.ndarray:
    """The four output words of Philox4x32-10 for a 4-word counter and 2-word key."""
    c = np.ascontiguousarray(ctr, dtype=np.uint32)
    k = np.ascontiguousarray(key, dtype=np.uint32)
    out = np.empty(4, np.uint32)
    _L().fp4o_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def philox_word(seed: int, index: int, stream: int) -> int:
    return int(_L().fp4o_philox_word(seed, index, stream))


def e2m1_encode_sr(q: float, w: int) -> int:
    return int(_L().fp4o_e2m1_encode_sr(q, w))


def rht_negate(seed: int, j: int) -> bool:
    return bool(_L().fp4o_rht_negate(seed, j))


def quantize(x, fmt: int, hn: int, axis: int = ROW, amax: float | None = None,
             sr_seed: int | None = None, rht_seed: int | None = None):
    """Returns (codes [R][C/2] uint8, scales (layout R7) uint8, S, amax) where
    (R, C) = x.shape for ROW and x.shape[::-1] for COL. S and amax are None for MXFP4.
    For NVFP4, `amax` supplies the tensor amax when x is a slice of the tensor (rows of a
    ROW quantisation or columns of a COL one), or when the caller fixes it.
    sr_seed: stochastic rounding of the codes; rht_seed: randomised Hadamard signs
    (both keyed by the given seed; None = off)."""
    xb = _bf16_bits(x)
    rows, cols = xb.shape
    R, C = (rows, cols) if axis == ROW else (cols, rows)
    bs = BLOCK[fmt]
    if fmt == MXFP8:
        assert amax is None and sr_seed is None and rht_seed is None
        codes = np.zeros((R, C), np.uint8)
        scales = np.zeros(scale_layout_bytes(R, C // bs), np.uint8)
        if _L().fp4o_quantize_mxfp8(_ptr(xb), rows, cols, hn, axis, _ptr(codes), _ptr(scales)):
            raise ValueError(f"oracle quantize rejected shape {xb.shape} fmt={fmt} hn={hn}")
        return codes, scales, None, None
    codes = np.zeros((R, C // 2), np.uint8)
    scales = np.zeros(scale_layout_bytes(R, C // bs), np.uint8)
    s = np.zeros(1, np.float32)
    t = np.zeros(1, np.float32)
    a_in = None if amax is None else np.array([amax], np.float32)
    rc = _L().fp4o_quantize_opt(_ptr(xb), rows, cols, fmt, hn, axis,
                                None if a_in is None else _ptr(a_in), sr_seed is not None,
                                sr_seed or 0, rht_seed is not None, rht_seed or 0,
                                _ptr(codes), _ptr(scales), _ptr(s), _ptr(t))
    if rc != 0:
        raise ValueError(f"oracle quantize rejected shape {xb.shape} fmt={fmt} hn={hn} axis={axis}")
    if fmt == NVFP4:
        return codes, scales, float(s[0]), float(t[0])
    return codes, scales, None, None


def dequantize(codes: np.ndarray, scales: np.ndarray, tensor_scale, fmt: int) -> np.ndarray:
    R, W = codes.shape
    C = W if fmt == MXFP8 else 2 * W  # MXFP8: one code byte per element
    out = np.empty((R, C), np.float64)
    ts = 1.0 if tensor_scale is None else float(tensor_scale)
    _L().fp4o_dequantize(_ptr(np.ascontiguousarray(codes)), _ptr(np.ascontiguousarray(scales)),
                         ts, R, C, fmt, _ptr(out))
    return out


def gemm_f64(A: np.ndarray, B: np.ndarray) -> np.ndarray:
    """C = A @ B.T in fp64 by the plain triple loop (A [M][K], B [N][K])."""
    A = np.ascontiguousarray(A, dtype=np.float64)
    B = np.ascontiguousarray(B, dtype=np.float64)
    M, K = A.shape
    N = B.shape[0]
    C = np.empty((M, N), np.float64)
    _L().fp4o_gemm_f64(_ptr(A), _ptr(B), _ptr(C), M, N, K)
    return C


def gemm_entries(a_q, b_q, fmt: int, ms, ns) -> np.ndarray:
    """Entries (ms[i], ns[i]) of deq(A) @ deq(B).T from quantised operands
    a_q = (codes, scales, S) of A [M][K] and b_q likewise of B [N][K]."""
    ac, asc, ats = a_q
    bc, bsc, bts = b_q
    K = ac.shape[1] if fmt == MXFP8 else ac.shape[1] * 2
    ms = np.ascontiguousarray(ms, dtype=np.int64)
    ns = np.ascontiguousarray(ns, dtype=np.int64)
    out = np.empty(ms.size, np.float64)
    _L().fp4o_gemm_entries(_ptr(np.ascontiguousarray(ac)), _ptr(np.ascontiguousarray(asc)),
                           1.0 if ats is None else float(ats),
                           _ptr(np.ascontiguousarray(bc)), _ptr(np.ascontiguousarray(bsc)),
                           1.0 if bts is None else float(bts), K, fmt, _ptr(ms), _ptr(ns),
                           ms.size, _ptr(out))
    return out

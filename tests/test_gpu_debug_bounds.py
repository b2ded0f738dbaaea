"""The range-checked debug build (libfp4_debug.so, -DFP4_DEBUG_BOUNDS): every kernel
checks its computed shared-memory offsets, TMEM columns, tile coordinates and global
indices before use and reports a failure as FP4_ERR_BOUNDS through fp4_check_status
(the access is skipped, nothing traps). The small- and ragged-shape parity suites run
against it in a child process (FP4_DEBUG_BOUNDS=1 selects the library); they assert
bit-exact results and a clean status after their calls. A direct check then compares
the debug library's outputs with the release library's bit for bit."""
import ctypes
import os
import subprocess
import sys

import pytest
import torch

import fp4_block_scaled_deterministic_b200 as fp4
from fp4_block_scaled_deterministic_b200 import build, synthetic
from gpu_util import need_gpu

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_ragged_parity_suites_under_the_debug_build():
    need_gpu()
    build.build(debug=True)
    env = dict(os.environ, FP4_DEBUG_BOUNDS="1")
    files = ["tests/test_gpu_quantize.py", "tests/test_gpu_gemm.py",
             "tests/test_gpu_fused_epilogue.py", "tests/test_gpu_variants.py",
             "tests/test_gpu_nvfp4_golden.py"]
    r = subprocess.run([sys.executable, "-m", "pytest", "-m", "gpu", "-q", "-x", "-p",
                        "no:cacheprovider", "-k", "not full and not llama", *files],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1500)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
    assert " passed" in r.stdout


def test_debug_build_matches_release_bit_for_bit():
    need_gpu()
    dbg = ctypes.CDLL(build.build(debug=True))
    P, I64, I32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    dbg.fp4_quantize_dual.argtypes = [P, P, P, P, P, P, I64, I64, I32, I32, P]
    dbg.fp4_gemm.argtypes = [P, P, P, P, P, P, P, I64, I64, I64, I32, I32, P]
    dbg.fp4_check_status.argtypes = [P]
    s = torch.cuda.current_stream().cuda_stream
    for fmt in (fp4.MXFP4, fp4.NVFP4):
        for rows, cols in ((160, 224), (288, 4096)):
            x = synthetic.normal(rows, cols, 1.0, seed=rows, outlier_frac=0.01,
                                 outlier_mult=50.0).cuda()
            rq, cq = fp4.quantize_dual(x, fmt, 16)
            mine = [torch.empty_like(t) for t in (rq.codes, rq.scales, cq.codes, cq.scales)]
            ts = torch.zeros(4, dtype=torch.float32, device="cuda") if fmt == fp4.NVFP4 else None
            st = dbg.fp4_quantize_dual(x.data_ptr(), *[t.data_ptr() for t in mine],
                                       None if ts is None else ts.data_ptr(), rows, cols, fmt, 16,
                                       s)
            assert st == 0
            for a, b in zip(mine, (rq.codes, rq.scales, cq.codes, cq.scales)):
                assert torch.equal(a, b)
            W = synthetic.normal(96, cols, 0.02, seed=5).cuda()
            qw = fp4.quantize(W, fmt, 16)
            C = fp4.gemm(rq, qw, fp4.OUT_F32)
            Cd = torch.empty_like(C)
            st = dbg.fp4_gemm(rq.codes.data_ptr(), rq.scales.data_ptr(),
                              None if ts is None else rq.tensor_scale.data_ptr(),
                              qw.codes.data_ptr(), qw.scales.data_ptr(),
                              None if ts is None else qw.tensor_scale.data_ptr(),
                              Cd.data_ptr(), rows, 96, cols, fmt, fp4.OUT_F32, s)
            assert st == 0
            torch.cuda.synchronize()
            assert torch.equal(Cd.view(torch.int32), C.view(torch.int32))
    assert dbg.fp4_check_status(s) == 0
    assert fp4.fp4_check_status() == 0

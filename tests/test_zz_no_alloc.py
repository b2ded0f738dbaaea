"""fp4_linear_fprop_noalloc: the Fprop pass on the library's static scratch, for
callers that cannot allocate device memory (a host framework that has reserved the
GPU's memory for its own allocator, plug-ins handed tensors but no allocator, loops
that must not call cudaMalloc because it can synchronise the device).

Both entry points run the same deterministic kernels, so the no-allocation output
must equal fp4_linear_fprop's (caller-allocated workspace) bit for bit, on
consecutive calls that share the scratch: the second NVFP4 call has a smaller tensor
amax than the first, so a scratch cell left over from the first call would change its
result. The first call is also checked against the CPU oracle. This file is
collected last."""
import numpy as np
import pytest
import torch

import fp4_block_scaled_deterministic_b200 as fp4
from fp4_block_scaled_deterministic_b200 import synthetic
from gpu_util import need_gpu, rel_fro

pytestmark = pytest.mark.gpu
TOL = 1e-4  # relative Frobenius error of an fp32-output GEMM against the fp64 oracle


def _noalloc(X, W, fmt, hn, out_dtype):
    (M, K), N = X.shape, W.shape[0]
    dt = torch.float32 if out_dtype == fp4.OUT_F32 else torch.bfloat16
    Y = torch.empty(M, N, dtype=dt, device="cuda")
    st = fp4.fp4_linear_fprop_noalloc(X, W, Y, M, N, K, fmt, hn, out_dtype)
    assert st == 0, fp4.status_string(st)
    return Y


def test_noalloc_fprop_matches_workspace_fprop(orc):
    need_gpu()
    calls = [  # (M, N, K, fmt, outlier multiplier): consecutive calls share the scratch
        (256, 384, 512, fp4.NVFP4, 50.0),
        (160, 96, 224, fp4.NVFP4, 1.0),
        (512, 256, 1024, fp4.MXFP4, 50.0),
        (512, 256, 1024, fp4.MXFP4, 50.0),
    ]
    for i, (M, N, K, fmt, mult) in enumerate(calls):
        X = synthetic.normal(M, K, 1.0, seed=40 + i, outlier_frac=0.01, outlier_mult=mult)
        W = synthetic.normal(N, K, 0.02, seed=50 + i)
        Xd, Wd = X.cuda(), W.cuda()
        Y = _noalloc(Xd, Wd, fmt, 16, fp4.OUT_F32)
        Y_ref = fp4.linear_fprop(Xd, Wd, fmt, 16, fp4.OUT_F32)
        torch.cuda.synchronize()
        assert fp4.fp4_check_status() == 0
        assert torch.equal(Y.view(torch.int32), Y_ref.view(torch.int32)), (
            i, rel_fro(Y.cpu().numpy(), Y_ref.cpu().numpy()))
        if i == 0:
            oa = orc.quantize(X, fmt, 16)[:3]
            ob = orc.quantize(W, fmt, 16)[:3]
            ref = orc.gemm_f64(orc.dequantize(*oa, fmt), orc.dequantize(*ob, fmt))
            err = rel_fro(Y.cpu().numpy(), ref)
            assert err <= TOL, err


def test_noalloc_rejects_sizes_beyond_its_scratch():
    need_gpu()
    M = N = K = 8192  # needs ~66 MB of scratch, more than the 32 MiB array
    assert fp4.fp4_linear_workspace_size(fp4.FPROP, M, N, K, fp4.MXFP4) > 32 << 20
    st = fp4.fp4_linear_fprop_noalloc(None, None, None, M, N, K, fp4.MXFP4, 16, fp4.OUT_BF16)
    assert st == 7  # FP4_ERR_WORKSPACE, nothing launched

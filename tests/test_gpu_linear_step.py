"""fp4_linear_step: a layer's Fprop, Dgrad and Wgrad as one batched dual quantisation
and one grouped GEMM launch. Its outputs must equal the three separate passes
(fp4_linear_fprop / _dgrad with bf16 outputs, fp4_linear_wgrad with fp32 output) bit
for bit: the dual quantiser's layouts are those of the single-layout passes, and a
grouped GEMM those of single GEMMs. The passes themselves are checked against the
oracle in test_gpu_linear.py; one small step is also checked against the oracle here."""
import numpy as np
import pytest
import torch

import fp4_block_scaled_deterministic_b200 as fp4
from fp4_block_scaled_deterministic_b200 import synthetic
from gpu_util import need_gpu, rel_fro

pytestmark = pytest.mark.gpu


def _same_bits(a, b):
    if a.dtype == torch.bfloat16:
        return torch.equal(a.view(torch.int16), b.view(torch.int16))
    return torch.equal(a.view(torch.int32), b.view(torch.int32))


def _inputs(M, N, K, seed):
    X = synthetic.normal(M, K, 1.0, seed=seed, outlier_frac=0.01, outlier_mult=30.0).cuda()
    W = synthetic.normal(N, K, 0.02, seed=seed + 1).cuda()
    dY = synthetic.heavy_tailed_grad(M, N, 1e-3, seed=seed + 2).cuda()
    return X, W, dY


@pytest.mark.parametrize("fmt", [fp4.MXFP4, fp4.NVFP4, fp4.MXFP8])
@pytest.mark.parametrize("shape", [(256, 512, 1024), (160, 288, 640), (96, 256, 512)])
def test_step_equals_the_three_passes(fmt, shape):
    need_gpu()
    M, N, K = shape
    X, W, dY = _inputs(M, N, K, seed=M + N + K)
    Y, dX, dW = fp4.linear_step(X, W, dY, fmt, 16)
    Yr = fp4.linear_fprop(X, W, fmt, 16, fp4.OUT_BF16)
    dXr = fp4.linear_dgrad(dY, W, fmt, 16, fp4.OUT_BF16)
    dWr = fp4.linear_wgrad(dY, X, fmt, 16, fp4.OUT_F32)
    torch.cuda.synchronize()
    assert _same_bits(Y, Yr) and _same_bits(dX, dXr) and _same_bits(dW, dWr)
    assert fp4.fp4_check_status() == 0


def test_step_matches_oracle(orc):
    """Small step against the oracle: the fp64 products of the oracle's quantised and
    dequantised operands of each pass."""
    need_gpu()
    M, N, K, fmt = 256, 288, 512, fp4.MXFP4
    X, W, dY = _inputs(M, N, K, seed=3)
    Y, dX, dW = fp4.linear_step(X, W, dY, fmt, 16)
    Xc, Wc, dYc = X.cpu(), W.cpu(), dY.cpu()
    ROW, COL = fp4.ROW, fp4.COL

    def deq(t, axis):
        q = orc.quantize(t, fmt, 16, axis)
        return orc.dequantize(*q[:3], fmt)

    refs = [orc.gemm_f64(deq(Xc, ROW), deq(Wc, ROW)),        # Y  = X W^T
            orc.gemm_f64(deq(dYc, ROW), deq(Wc, COL)),       # dX = dY W
            orc.gemm_f64(deq(dYc, COL), deq(Xc, COL))]       # dW = dY^T X
    for out, ref in zip((Y, dX, dW), refs):
        assert rel_fro(out.float().cpu().numpy(), ref) <= 2e-3 if out.dtype == torch.bfloat16 \
            else rel_fro(out.cpu().numpy(), ref) <= 1e-4

"""GPU parity of the three linear-layer passes (C entry points fp4_linear_fprop,
_dgrad, _wgrad) against the oracle: each pass quantises its operands along its own
contraction axis (Wgrad along the tokens) and multiplies them."""
import numpy as np
import pytest
import torch

import fp4_block_scaled_deterministic_b200 as fp4
from fp4_block_scaled_deterministic_b200 import synthetic
from gpu_util import need_gpu, rel_fro

pytestmark = pytest.mark.gpu
TOL = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def _inputs(M, N, K, seed):
    X = synthetic.normal(M, K, 1.0, seed=seed, outlier_frac=0.01, outlier_mult=50.0)
    W = synthetic.normal(N, K, 0.02, seed=seed + 1)
    dY = synthetic.heavy_tailed_grad(M, N, seed=seed + 2)
    return X, W, dY


def _deq(orc, q, fmt):
    return orc.dequantize(q[0], q[1], q[2], fmt)


@pytest.mark.parametrize("shape", [(256, 384, 512), (160, 96, 224), (1024, 768, 256)])
@pytest.mark.parametrize("hn", [16, 32])
@pytest.mark.parametrize("fmt", [0, 1, 2])  # MXFP4, NVFP4, the MXFP8 comparator
def test_three_passes(orc, fmt, hn, shape):
    M, N, K = shape
    X, W, dY = _inputs(M, N, K, seed=M + K)
    Xg, Wg, dYg = X.cuda(), W.cuda(), dY.cuda()
    Y = fp4.linear_fprop(Xg, Wg, fmt, hn, fp4.OUT_F32)
    dX = fp4.linear_dgrad(dYg, Wg, fmt, hn, fp4.OUT_F32)
    dW = fp4.linear_wgrad(dYg, Xg, fmt, hn, fp4.OUT_F32)
    Yb = fp4.linear_fprop(Xg, Wg, fmt, hn, fp4.OUT_BF16)
    torch.cuda.synchronize()
    assert fp4.fp4_check_status() == 0
    assert Y.shape == (M, N) and dX.shape == (M, K) and dW.shape == (N, K)
    ref_y = _deq(orc, orc.quantize(X, fmt, hn, orc.ROW), fmt) @ _deq(orc, orc.quantize(W, fmt, hn, orc.ROW), fmt).T
    ref_dx = _deq(orc, orc.quantize(dY, fmt, hn, orc.ROW), fmt) @ _deq(orc, orc.quantize(W, fmt, hn, orc.COL), fmt).T
    ref_dw = _deq(orc, orc.quantize(dY, fmt, hn, orc.COL), fmt) @ _deq(orc, orc.quantize(X, fmt, hn, orc.COL), fmt).T
    assert rel_fro(Y.cpu().numpy(), ref_y) <= TOL
    assert rel_fro(dX.cpu().numpy(), ref_dx) <= TOL
    assert rel_fro(dW.cpu().numpy(), ref_dw) <= TOL
    assert torch.equal(Yb.cpu().view(torch.int16), Y.cpu().to(torch.bfloat16).view(torch.int16))
    # information only: distance to the unquantised product stays moderate
    un = X.double().numpy() @ W.double().numpy().T
    assert rel_fro(Y.cpu().numpy(), un) < 0.5


def test_workspace_too_small_is_rejected():
    X, W, _ = _inputs(64, 64, 64, seed=1)
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(fp4.Fp4Error) as e:
        fp4.linear_fprop(X.cuda(), W.cuda(), ws=ws)
    assert e.value.code == 7

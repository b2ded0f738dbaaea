"""fp4_quantize_dual_batch: several tensors' dual quantisation in as few launches as
possible. Each item must equal a separate fp4_quantize_dual of the same tensor bit for
bit (codes, scales and NVFP4 tensor scales of both layouts), and through it the oracle
(test_gpu_quantize.py checks fp4_quantize_dual against the oracle). Covered: every
format and rotation, items of different ragged shapes, an empty item, more items than
one launch takes, and the Llama-3.1-8B gate projection's X, W and dY."""
import pytest
import torch

import fp4_block_scaled_deterministic_b200 as fp4
from fp4_block_scaled_deterministic_b200 import synthetic
from gpu_util import need_gpu

pytestmark = pytest.mark.gpu
SHAPES = [(256, 384), (160, 224), (32, 4096), (1024, 128), (96, 96), (0, 64)]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def _same(a, b):
    assert torch.equal(a.codes, b.codes) and torch.equal(a.scales, b.scales)
    if a.tensor_scale is not None:
        assert torch.equal(a.tensor_scale.view(torch.int32), b.tensor_scale.view(torch.int32))


@pytest.mark.parametrize("hn", [0, 16, 32])
@pytest.mark.parametrize("fmt", [0, 1, 2])
def test_batch_equals_single_calls(fmt, hn):
    xs = [synthetic.normal(r, c, 1.0, seed=r + c + fmt, outlier_frac=0.01, outlier_mult=50.0).cuda()
          for r, c in SHAPES]
    got = fp4.quantize_dual_batch(xs, fmt, hn)
    torch.cuda.synchronize()
    assert fp4.fp4_check_status() == 0
    for x, (gr, gc) in zip(xs, got):
        if x.numel() == 0:
            continue
        rr, rc = fp4.quantize_dual(x, fmt, hn)
        torch.cuda.synchronize()
        _same(gr, rr)
        _same(gc, rc)


@pytest.mark.parametrize("fmt", [0, 1])
def test_batch_llama_gate_operands(fmt):
    X, W, dY = (t.cuda() for t in synthetic.llama_layer("gate"))
    got = fp4.quantize_dual_batch([X, W, dY], fmt, 16)
    for x, (gr, gc) in zip((X, W, dY), got):
        rr, rc = fp4.quantize_dual(x, fmt, 16)
        torch.cuda.synchronize()
        _same(gr, rr)
        _same(gc, rc)
    assert fp4.fp4_check_status() == 0

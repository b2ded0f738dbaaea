"""GPU parity of the quantiser variants of fp4_quantize_opts / fp4_quantize_dual_opts
against the oracle, bit for bit: stochastic rounding (Philox words keyed by seed and
element index), randomised Hadamard signs, both together, and a caller-supplied NVFP4
tensor amax; plus the GEMM on randomised-Hadamard operands."""
import numpy as np
import pytest
import torch

import fp4_block_scaled_deterministic_b200 as fp4
from fp4_block_scaled_deterministic_b200 import synthetic
from gpu_util import f32_bits, need_gpu, np_u8, rel_fro

pytestmark = pytest.mark.gpu
ROW, COL = fp4.ROW, fp4.COL


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def _x(rows, cols, seed):
    return synthetic.normal(rows, cols, 1.0, seed=seed, outlier_frac=0.01, outlier_mult=30.0)


def _same(q, o, fmt):
    assert np.array_equal(np_u8(q.codes), o[0]), "codes differ"
    assert np.array_equal(np_u8(q.scales), o[1]), "scales differ"
    if fmt == fp4.NVFP4:
        assert f32_bits(q.tensor_scale.item()) == f32_bits(o[2])


VARIANTS = {"sr": dict(sr_seed=0x1234_5678_9ABC), "rht": dict(sign_seed=42),
            "sr+rht": dict(sr_seed=7, sign_seed=0xFFFF_FFFF_0000_0001)}


@pytest.mark.parametrize("variant", list(VARIANTS))
@pytest.mark.parametrize("hn", [0, 16, 32])
@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("shape", [(160, 224), (512, 1024)])
def test_variant_single_layouts(orc, shape, fmt, hn, variant):
    x = _x(*shape, seed=shape[0] + hn)
    kw = VARIANTS[variant]
    for axis in (ROW, COL):
        q = fp4.quantize(x.cuda(), fmt, hn, axis, **kw)
        torch.cuda.synchronize()
        assert fp4.fp4_check_status() == 0
        o = orc.quantize(x, fmt, hn, axis, sr_seed=kw.get("sr_seed"), rht_seed=kw.get("sign_seed"))
        _same(q, o, fmt)


@pytest.mark.parametrize("variant", list(VARIANTS))
@pytest.mark.parametrize("hn", [0, 16, 32])
@pytest.mark.parametrize("fmt", [0, 1])
def test_variant_dual(orc, fmt, hn, variant):
    x = _x(384, 640, seed=11 + hn)
    kw = VARIANTS[variant]
    rq, cq = fp4.quantize_dual(x.cuda(), fmt, hn, **kw)
    torch.cuda.synchronize()
    assert fp4.fp4_check_status() == 0
    for q, axis in ((rq, ROW), (cq, COL)):
        o = orc.quantize(x, fmt, hn, axis, sr_seed=kw.get("sr_seed"), rht_seed=kw.get("sign_seed"))
        _same(q, o, fmt)


def test_variant_large_dual_mx_h16(orc):
    """A Llama-sized row length (4096) and many row tiles, both layouts, SR + RHT."""
    x = _x(1024, 4096, seed=5)
    rq, cq = fp4.quantize_dual(x.cuda(), 0, 16, sr_seed=99, sign_seed=98)
    torch.cuda.synchronize()
    for q, axis in ((rq, ROW), (cq, COL)):
        _same(q, orc.quantize(x, 0, 16, axis, sr_seed=99, rht_seed=98), 0)


def test_sr_draws_differ_by_seed_and_average_out():
    x = _x(256, 512, seed=3).cuda()
    a = fp4.quantize(x, 0, 16, ROW, sr_seed=1)
    b = fp4.quantize(x, 0, 16, ROW, sr_seed=1)
    c = fp4.quantize(x, 0, 16, ROW, sr_seed=2)
    torch.cuda.synchronize()
    assert torch.equal(a.codes, b.codes) and not torch.equal(a.codes, c.codes)
    assert torch.equal(a.scales, c.scales)


@pytest.mark.parametrize("mode", ["row", "col", "dual"])
@pytest.mark.parametrize("hn", [0, 16])
def test_supplied_amax_nvfp4(orc, hn, mode):
    """A supplied amax equal to the computed one reproduces the plain quantisation; a
    different one follows the oracle given that amax; tensor_scale holds {S, T}."""
    x = _x(256, 384, seed=21)
    xs = x.cuda()
    if mode == "dual":
        plain = fp4.quantize_dual(xs, 1, hn)
        torch.cuda.synchronize()
        T = [orc.rotated_amax(x, hn, ROW), orc.rotated_amax(x, hn, COL)]
        for scale in (1.0, 3.0):
            amax = torch.tensor([scale * T[0], scale * T[1]], dtype=torch.float32, device="cuda")
            rq, cq = fp4.quantize_dual(xs, 1, hn, amax=amax)
            torch.cuda.synchronize()
            assert fp4.fp4_check_status() == 0
            for q, axis, t in ((rq, ROW, amax[0].item()), (cq, COL, amax[1].item())):
                _same(q, orc.quantize(x, 1, hn, axis, amax=t), 1)
            if scale == 1.0:
                assert torch.equal(rq.codes, plain[0].codes) and torch.equal(cq.codes, plain[1].codes)
        return
    axis = ROW if mode == "row" else COL
    plain = fp4.quantize(xs, 1, hn, axis)
    T = orc.rotated_amax(x, hn, axis)
    for scale in (1.0, 0.5, 3.0):
        amax = torch.tensor([scale * T], dtype=torch.float32, device="cuda")
        ts = torch.zeros(2, dtype=torch.float32, device="cuda")
        q = fp4.quantize(xs, 1, hn, axis, ts_buf=ts, amax=amax)
        torch.cuda.synchronize()
        assert fp4.fp4_check_status() == 0
        o = orc.quantize(x, 1, hn, axis, amax=amax.item())
        _same(q, o, 1)
        assert f32_bits(ts[1].item()) == f32_bits(amax.item())
        if scale == 1.0:
            assert torch.equal(q.codes, plain.codes) and torch.equal(q.scales, plain.scales)


@pytest.mark.parametrize("fmt", [0, 1])
def test_gemm_on_randomised_hadamard_operands(orc, fmt):
    """Fprop with both operands under the same random signs: the GEMM of the quantised
    operands matches the oracle, and the product stays close to X W^T."""
    M, N, K = 256, 384, 1024
    X = _x(M, K, seed=31)
    W = synthetic.normal(N, K, 0.02, seed=32)
    qa = fp4.quantize(X.cuda(), fmt, 16, ROW, sign_seed=5)
    qb = fp4.quantize(W.cuda(), fmt, 16, ROW, sign_seed=5)
    C = fp4.gemm(qa, qb, fp4.OUT_F32)
    torch.cuda.synchronize()
    oa = orc.quantize(X, fmt, 16, ROW, rht_seed=5)[:3]
    ob = orc.quantize(W, fmt, 16, ROW, rht_seed=5)[:3]
    ref = orc.gemm_f64(orc.dequantize(*oa, fmt), orc.dequantize(*ob, fmt))
    assert rel_fro(C.cpu().numpy(), ref) <= 1e-4
    exact = X.double().numpy() @ W.double().numpy().T
    assert rel_fro(C.cpu().numpy(), exact) < 0.2

"""fp4_gemm_group: several GEMMs in one launch of the pair kernel. Every output must equal
the same fp4_gemm call bit for bit (same kernel, same per-tile K order), so the oracle
parity of fp4_gemm carries over; a small group is also checked against the oracle
directly. Shapes mix output types, ragged M and N, formats, an empty member and every
full-size Llama-3.1-8B projection (the bench's launches)."""
import numpy as np
import pytest
import torch

import fp4_block_scaled_deterministic_b200 as fp4
from fp4_block_scaled_deterministic_b200 import synthetic
from gpu_util import need_gpu, np_u8, rel_fro

pytestmark = pytest.mark.gpu
TOL = 1e-4


def _q(rows, cols, fmt, seed, hn=16):
    x = synthetic.normal(rows, cols, 1.0, seed=seed, outlier_frac=0.01, outlier_mult=30.0).cuda()
    return fp4.quantize(x, fmt, hn)


def _same_bits(a, b):
    if a.dtype == torch.bfloat16:
        return torch.equal(a.view(torch.int16), b.view(torch.int16))
    return torch.equal(a.view(torch.int32), b.view(torch.int32))


@pytest.mark.parametrize("fmt", [fp4.MXFP4, fp4.NVFP4, fp4.MXFP8])
def test_group_equals_single_calls(fmt):
    need_gpu()
    shapes = [(256, 768, 1024, fp4.OUT_BF16), (384, 512, 2048, fp4.OUT_F32),
              (160, 800, 512, fp4.OUT_BF16)]
    probs, ods = [], []
    for i, (M, N, K, od) in enumerate(shapes):
        probs.append((_q(M, K, fmt, seed=10 + i), _q(N, K, fmt, seed=20 + i)))
        ods.append(od)
    outs = fp4.gemm_group(probs, ods)
    for (a, b), od, out in zip(probs, ods, outs):
        ref = fp4.gemm(a, b, od)
        torch.cuda.synchronize()
        assert _same_bits(out, ref)
    assert fp4.fp4_check_status() == 0


def test_group_matches_oracle(orc):
    need_gpu()
    fmt = fp4.MXFP4
    shapes = [(288, 544, 768), (256, 256, 512)]
    probs, oracle = [], []
    for i, (M, N, K) in enumerate(shapes):
        X = synthetic.normal(M, K, 1.0, seed=30 + i, outlier_frac=0.01, outlier_mult=30.0)
        W = synthetic.normal(N, K, 0.02, seed=40 + i)
        qa, qb = fp4.quantize(X.cuda(), fmt, 16), fp4.quantize(W.cuda(), fmt, 16)
        oa, ob = orc.quantize(X, fmt, 16)[:3], orc.quantize(W, fmt, 16)[:3]
        torch.cuda.synchronize()
        assert np.array_equal(np_u8(qa.codes), oa[0]) and np.array_equal(np_u8(qb.codes), ob[0])
        probs.append((qa, qb))
        oracle.append(orc.gemm_f64(orc.dequantize(*oa, fmt), orc.dequantize(*ob, fmt)))
    outs = fp4.gemm_group(probs, [fp4.OUT_F32, fp4.OUT_F32])
    for out, ref in zip(outs, oracle):
        assert rel_fro(out.cpu().numpy(), ref) <= TOL


def test_group_with_small_m_and_empty_member(orc):
    """An M <= 128 problem runs in the pair kernel (one zero-filled 256-row band) inside a
    group; a member with M = 0 is skipped."""
    need_gpu()
    fmt = fp4.MXFP4
    M, N, K = 96, 512, 1024
    X = synthetic.normal(M, K, 1.0, seed=50)
    W = synthetic.normal(N, K, 0.02, seed=51)
    qa, qb = fp4.quantize(X.cuda(), fmt, 16), fp4.quantize(W.cuda(), fmt, 16)
    big = (_q(512, K, fmt, seed=52), qb)
    empty_a = fp4.QTensor(qa.codes[:0], qa.scales, None, fmt, 0, K)
    out_small, out_big, out_empty = fp4.gemm_group([(qa, qb), big, (empty_a, qb)],
                                                   [fp4.OUT_F32, fp4.OUT_F32, fp4.OUT_F32])
    torch.cuda.synchronize()
    assert out_empty.shape == (0, N)
    oa, ob = orc.quantize(X, fmt, 16)[:3], orc.quantize(W, fmt, 16)[:3]
    ref = orc.gemm_f64(orc.dequantize(*oa, fmt), orc.dequantize(*ob, fmt))
    assert rel_fro(out_small.cpu().numpy(), ref) <= TOL
    assert _same_bits(out_big, fp4.gemm(big[0], big[1], fp4.OUT_F32))
    assert fp4.fp4_check_status() == 0


@pytest.mark.parametrize("name", [n for n, _, _ in synthetic.LLAMA_LAYERS])
def test_group_llama_three_passes_full_size(name):
    """Fprop, Dgrad and Wgrad of each Llama-3.1-8B projection (8192 tokens, MXFP4 +
    H16) in one launch, as the bench runs them: each output equals the separate
    fp4_gemm call (whose full-size parity against the oracle is tested elsewhere) bit
    for bit."""
    need_gpu()
    fmt = fp4.MXFP4
    X, W, dY = synthetic.llama_layer(name)
    xr, xc = fp4.quantize_dual(X.cuda(), fmt, 16)
    wr, wc = fp4.quantize_dual(W.cuda(), fmt, 16)
    yr, yc = fp4.quantize_dual(dY.cuda(), fmt, 16)
    probs = [(xr, wr), (yr, wc), (yc, xc)]       # Fprop, Dgrad, Wgrad
    ods = [fp4.OUT_BF16, fp4.OUT_BF16, fp4.OUT_F32]
    outs = fp4.gemm_group(probs, ods)
    for (a, b), od, out in zip(probs, ods, outs):
        ref = fp4.gemm(a, b, od)
        torch.cuda.synchronize()
        assert _same_bits(out, ref)
        del ref
    assert fp4.fp4_check_status() == 0

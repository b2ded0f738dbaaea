"""Full-size parity of every GEMM of the Llama-3.1-8B layer step, in the benchmark's
launch configuration: 8192 tokens; projections qkv 6144x4096, o 4096x4096, gate and
up 14336x4096, down 4096x14336; MXFP4 + H16; X N(0,1) with 0.1% outlier channels
x50, W N(0, 0.02^2), dY N(0, 1e-3^2) with 0.5% heavy-tailed entries (Student-t
nu=3, x20). Operands come from the dual-layout quantiser, as in the benchmark.

For each projection and pass (Fprop Y = X W^T, Dgrad dX = dY W, Wgrad dW = dY^T X
over the 8192-token axis):
* both operands' codes and scales equal the oracle's, whole tensors, bit for bit;
* the fp32-output GEMM is within 1e-4 relative Frobenius error of the fp64 product
  of the oracle-dequantised operands (a library fp64 matmul on the device), over the
  whole output, and 256 sampled entries are within it against the oracle's own sums;
* the bf16-output GEMM equals RN_bf16 of the fp32 one bit for bit.
(The gate Fprop is also covered in test_gpu_gemm.py.)"""
import numpy as np
import pytest
import torch

import fp4_block_scaled_deterministic_b200 as fp4
from fp4_block_scaled_deterministic_b200 import synthetic
from gpu_util import need_gpu, np_u8, rel_fro

pytestmark = pytest.mark.gpu
TOL = 1e-4
FMT, HN = fp4.MXFP4, 16
PROJS = [n for n, _, _ in synthetic.LLAMA_LAYERS]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


_cache = {}


def _layer(orc, name):
    """GPU dual quantisation of X, W, dY of one projection and the oracle's
    quantisation of the same tensors (the COL layout as the ROW layout of the
    transpose, which is its definition)."""
    if name in _cache:
        return _cache[name]
    _cache.clear()
    X, W, dY = synthetic.llama_layer(name)
    g, o = {}, {}
    for key, t in (("X", X), ("W", W), ("dY", dY)):
        g[key] = fp4.quantize_dual(t.cuda(), FMT, HN)
        o[key] = (orc.quantize(t, FMT, HN, orc.ROW)[:3],
                  orc.quantize(t.t().contiguous(), FMT, HN, orc.ROW)[:3])
    torch.cuda.synchronize()
    assert fp4.fp4_check_status() == 0
    _cache[name] = (g, o)
    return g, o


def _check_operand(q, o):
    assert np.array_equal(np_u8(q.codes), o[0]), "codes differ from the oracle"
    assert np.array_equal(np_u8(q.scales), o[1]), "scales differ from the oracle"


@pytest.mark.parametrize("pass_", ["fprop", "dgrad", "wgrad"])
@pytest.mark.parametrize("name", PROJS)
def test_llama_layer_gemm_full(orc, name, pass_):
    g, o = _layer(orc, name)
    # (A, B) = (quantised along the contraction axis) pairs of each pass, [rows][K]
    A, B = {"fprop": (("X", 0), ("W", 0)), "dgrad": (("dY", 0), ("W", 1)),
            "wgrad": (("dY", 1), ("X", 1))}[pass_]
    qa, qb = g[A[0]][A[1]], g[B[0]][B[1]]
    oa, ob = o[A[0]][A[1]], o[B[0]][B[1]]
    _check_operand(qa, oa)
    _check_operand(qb, ob)
    C = fp4.gemm(qa, qb, fp4.OUT_F32)
    Cb = fp4.gemm(qa, qb, fp4.OUT_BF16)
    torch.cuda.synchronize()
    assert fp4.fp4_check_status() == 0
    assert torch.equal(Cb.view(torch.int16), C.to(torch.bfloat16).view(torch.int16))
    rng = np.random.default_rng(3 * PROJS.index(name) + ["fprop", "dgrad", "wgrad"].index(pass_))
    ms = rng.integers(0, qa.rows, 256)
    ns = rng.integers(0, qb.rows, 256)
    ref = orc.gemm_entries(oa, ob, FMT, ms, ns)
    got = C[torch.from_numpy(ms).cuda(), torch.from_numpy(ns).cuda()].cpu().numpy()
    assert rel_fro(got, ref) <= TOL
    da = torch.from_numpy(orc.dequantize(*oa, FMT)).cuda()
    db = torch.from_numpy(orc.dequantize(*ob, FMT)).cuda()
    full = da @ db.T
    del da, db
    err = float((C.double() - full).norm() / full.norm())
    del full
    assert err <= TOL, err

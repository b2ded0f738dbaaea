"""GPU parity of the fused rotate + quantise kernel against the CPU oracle: codes,
scale bytes and NVFP4 tensor scales must be bit-identical, for every format,
rotation size and layout, on shapes spanning several 128x128 tiles with ragged
tails, on crafted edge values, and at a full Llama-3.1-8B activation size."""
import numpy as np
import pytest
import torch

import fp4_block_scaled_deterministic_b200 as fp4
from fp4_block_scaled_deterministic_b200 import synthetic
from gpu_util import f32_bits, gpu_quantize_raw, need_gpu, np_u8

pytestmark = pytest.mark.gpu

SHAPES = [(256, 384), (160, 224), (32, 32), (96, 4096), (1024, 1024), (4096, 64)]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def _check_same(orc_out, gpu_out, fmt):
    oc, os_, ots, oamax = orc_out
    gc, gs, gts = gpu_out
    assert gc.shape == oc.shape
    bad = np.argwhere(gc != oc)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first at {bad[:5].tolist()}"
    bad = np.nonzero(gs != os_)[0]
    assert bad.size == 0, f"{len(bad)} scale bytes differ, first at {bad[:5].tolist()}"
    if fmt == fp4.NVFP4:
        assert f32_bits(gts[0]) == f32_bits(ots) and f32_bits(gts[1]) == f32_bits(oamax)


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("axis", [0, 1])
@pytest.mark.parametrize("hn", [0, 16, 32])
@pytest.mark.parametrize("fmt", [0, 1])
def test_quantize_bit_exact(orc, fmt, hn, axis, shape):
    x = synthetic.normal(*shape, std=1.0, seed=shape[0] * 7 + shape[1], outlier_frac=0.01,
                         outlier_mult=50.0)
    _check_same(orc.quantize(x, fmt, hn, axis), gpu_quantize_raw(x, fmt, hn, axis), fmt)


@pytest.mark.parametrize("shape", [(256, 384), (160, 224), (32, 4096)])
@pytest.mark.parametrize("hn", [0, 16, 32])
@pytest.mark.parametrize("fmt", [0, 1])
def test_quantize_dual_equals_two_single_passes(orc, fmt, hn, shape):
    x = synthetic.heavy_tailed_grad(*shape, seed=shape[1])
    rq, cq = fp4.quantize_dual(x.cuda(), fmt, hn)
    torch.cuda.synchronize()
    o_r = orc.quantize(x, fmt, hn, orc.ROW)
    o_c = orc.quantize(x, fmt, hn, orc.COL)
    assert np.array_equal(np_u8(rq.codes), o_r[0]) and np.array_equal(np_u8(rq.scales), o_r[1])
    assert np.array_equal(np_u8(cq.codes), o_c[0]) and np.array_equal(np_u8(cq.scales), o_c[1])
    if fmt == fp4.NVFP4:
        assert f32_bits(rq.tensor_scale.item()) == f32_bits(o_r[2])
        assert f32_bits(cq.tensor_scale.item()) == f32_bits(o_c[2])


def _edge_tensor():
    """32 rows x 256 cols of bf16 edge values: E2M1 midpoints and their bf16
    neighbours under a block max of 6*2^k, signed zeros, tiny negatives that round
    to zero, subnormals, all-zero blocks, subnormal-only blocks, huge values."""
    bf = lambda a: torch.tensor(np.asarray(a, np.float32)).to(torch.bfloat16)
    rows = []
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    one_ulp_up = bf(mids * (1 + 2 ** -7)).float().numpy()
    one_ulp_dn = bf(mids * (1 - 2 ** -8)).float().numpy()
    for r in range(32):
        k = (r % 16) - 8
        blk = []
        for b in range(8):
            v = np.zeros(32, np.float32)
            v[0] = 6.0
            if b == 0:
                v[1:8], v[8:15], v[15:22] = mids, one_ulp_up, one_ulp_dn
                v[22:29] = -mids
                v[29], v[30], v[31] = -0.0, -0.01, 0.01
            elif b == 1:
                v[:] = 0.0
                v[5] = -0.0
            elif b == 2:
                v[:] = np.float32(2.0 ** -130) * np.arange(-16, 16)
            elif b == 3:
                v[:] = np.linspace(-7.5, 7.5, 32)
            elif b == 4:
                v[1:] = -np.float32(2.0 ** -20) * np.arange(1, 32)
            elif b == 5:
                v[:] = np.float32(1.0e37) * np.sign(np.arange(-16, 16) + 0.5)  # no fp32 overflow under H16
            elif b == 6:
                v[:] = np.float32(2.0 ** -126)
            else:
                v[:] = -np.float32(1e-3) * (np.arange(32) % 7)
            if b not in (1, 2, 5, 6):
                v = v * np.float32(2.0 ** k)
            blk.append(v)
        rows.append(np.concatenate(blk))
    return bf(np.stack(rows))


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("hn", [0, 16])
def test_quantize_edge_values(orc, fmt, hn):
    x = _edge_tensor()
    for axis in (0, 1):
        _check_same(orc.quantize(x, fmt, hn, axis), gpu_quantize_raw(x, fmt, hn, axis), fmt)


def _cancellation_tensor(rows, cols, seed):
    """Every 16x16 block holds one 2x2 corner of four equal values (+-2^k, k in
    [-4, 4)) among bf16 subnormals. Along either axis the two equal leading inputs
    cancel in the first butterfly, so under H16 a block's rotated values of normal size
    sit beside sums of subnormals (some below 2^-124) while the tensor scale is set by
    the normal values: the NVFP4 blocks take the fast quotient path with tiny elements
    in it, and the blocks of subnormals alone get a zero scale."""
    rng = np.random.default_rng(seed)
    x = (rng.integers(-127, 128, size=(rows, cols)) * 2.0 ** -133).astype(np.float32)
    big = (rng.choice([-1.0, 1.0], size=(rows // 16, cols // 16)) *
           2.0 ** rng.integers(-4, 4, size=(rows // 16, cols // 16))).astype(np.float32)
    for a in range(rows // 16):
        for b in range(cols // 16):
            x[16 * a:16 * a + 2, 16 * b:16 * b + 2] = big[a, b]
    return torch.tensor(x).to(torch.bfloat16)


@pytest.mark.parametrize("fmt", [0, 1])
def test_quantize_cancellation_blocks(orc, fmt):
    x = _cancellation_tensor(256, 384, seed=5 + fmt)
    assert torch.equal(x.float(), torch.tensor(x.float().numpy()))  # bf16-exact inputs
    for axis in (0, 1):
        _check_same(orc.quantize(x, fmt, 16, axis), gpu_quantize_raw(x, fmt, 16, axis), fmt)
    rq, cq = fp4.quantize_dual(x.cuda(), fmt, 16)
    bq = fp4.quantize_dual_batch([x.cuda(), x[:128].cuda().contiguous()], fmt, 16)
    torch.cuda.synchronize()
    for axis, q in ((orc.ROW, rq), (orc.COL, cq)):
        o = orc.quantize(x, fmt, 16, axis)
        assert np.array_equal(np_u8(q.codes), o[0]) and np.array_equal(np_u8(q.scales), o[1])
    for got, ref in zip(bq[0], (rq, cq)):
        assert torch.equal(got.codes, ref.codes) and torch.equal(got.scales, ref.scales)


def test_quantize_is_deterministic():
    x = synthetic.normal(512, 1024, seed=3, outlier_frac=0.001, outlier_mult=50.0)
    a = gpu_quantize_raw(x, 1, 16, 0)
    b = gpu_quantize_raw(x, 1, 16, 0)
    assert all(np.array_equal(p, q) for p, q in zip(a, b))


def test_quantize_full_llama_activation_dual(orc):
    """X of the Llama-3.1-8B down projection, 8192 x 14336, MXFP4 + H16, both layouts
    in one pass: the launch configuration of the benchmark."""
    X = synthetic.normal(8192, 14336, 1.0, seed=0, outlier_frac=0.001, outlier_mult=50.0)
    rq, cq = fp4.quantize_dual(X.cuda(), fp4.MXFP4, 16)
    torch.cuda.synchronize()
    o_r = orc.quantize(X, orc.MXFP4, 16, orc.ROW)
    assert np.array_equal(np_u8(rq.codes), o_r[0]) and np.array_equal(np_u8(rq.scales), o_r[1])
    del o_r
    o_c = orc.quantize(X, orc.MXFP4, 16, orc.COL)
    assert np.array_equal(np_u8(cq.codes), o_c[0]) and np.array_equal(np_u8(cq.scales), o_c[1])


def test_empty_input_is_a_noop():
    assert fp4.fp4_quantize(None, None, None, None, 0, 64, 0, 16, 0) == 0

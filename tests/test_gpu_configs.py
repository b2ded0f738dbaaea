"""Parity on the full-size workload configurations that the benchmark does not time:

* GPT-3 175B-shaped layers (hidden 12288, FFN 49152, 4096 tokens), MXFP4/NVFP4 x
  H16/H32/none, Fprop, Dgrad and Wgrad. Full-size operands are quantised on the GPU;
  the oracle quantises only the sampled rows (a row-wise quantisation is row-local, a
  column-wise one column-local; NVFP4 gets the tensor amax the oracle computes over
  the whole rotated tensor). Sampled rows must match bit for bit (codes, scales, tensor
  scale) and the sampled outputs must be within the GEMM tolerance.
* The quantise-only sweep (2^p elements, rows of 4096 / 14336 / 49152): bit-exact on
  whole tensors at 2^20 for every format, rotation and layout, and on sampled rows of
  2^28-element (MXFP4) and 2^26-element (NVFP4) tensors.
"""
import numpy as np
import pytest
import torch

import fp4_block_scaled_deterministic_b200 as fp4
from fp4_block_scaled_deterministic_b200 import synthetic
from gpu_util import f32_bits, need_gpu, np_u8, rel_fro

pytestmark = pytest.mark.gpu
TOL = 1e-4
ROW, COL = fp4.ROW, fp4.COL


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def _oracle_rows(orc, src_cpu, axis, idx, fmt, hn):
    """Oracle quantisation of rows `idx` of the quantised matrix Q(src) (rows of src for
    ROW, columns of src for COL)."""
    sub = src_cpu[idx] if axis == ROW else src_cpu[:, idx]
    T = None
    if fmt == fp4.NVFP4:
        # a COL quantisation of x is the ROW quantisation of x^T (same rotated values);
        # the transpose is a plain copy that keeps the oracle's row walk cache-friendly
        full = src_cpu if axis == ROW else src_cpu.t().contiguous()
        T = orc.rotated_amax(full, hn, ROW)
    return orc.quantize(sub.contiguous(), fmt, hn, axis, amax=T)


def _check_rows(orc, q, o, idx, fmt):
    """GPU QTensor rows idx against the oracle's quantisation of those rows."""
    codes = np_u8(q.codes[torch.from_numpy(idx).to(q.codes.device)])
    assert np.array_equal(codes, o[0]), "sampled code rows differ"
    kb = q.cols // fp4.BLOCK[fmt]
    gs = np_u8(q.scales)
    g_sc = np.array([[gs[orc.scale_offset(int(r), k, kb)] for k in range(kb)] for r in idx])
    o_sc = np.array([[o[1][orc.scale_offset(i, k, kb)] for k in range(kb)] for i in range(len(idx))])
    assert np.array_equal(g_sc, o_sc), "sampled scale rows differ"
    if fmt == fp4.NVFP4:
        assert f32_bits(q.tensor_scale.item()) == f32_bits(o[2])


def _sampled_gemm_check(orc, A_src, a_axis, B_src, b_axis, fmt, hn, n_rows=24, seed=0):
    dev_a, dev_b = A_src.cuda(), B_src.cuda()
    qa = fp4.quantize(dev_a, fmt, hn, a_axis)
    qb = fp4.quantize(dev_b, fmt, hn, b_axis)
    C = fp4.gemm(qa, qb, fp4.OUT_F32)
    Cb = fp4.gemm(qa, qb, fp4.OUT_BF16)
    torch.cuda.synchronize()
    assert fp4.fp4_check_status() == 0
    rng = np.random.default_rng(seed)
    ms = np.sort(rng.choice(qa.rows, n_rows, replace=False))
    ns = np.sort(rng.choice(qb.rows, n_rows, replace=False))
    oa = _oracle_rows(orc, A_src, a_axis, ms, fmt, hn)
    ob = _oracle_rows(orc, B_src, b_axis, ns, fmt, hn)
    _check_rows(orc, qa, oa, ms, fmt)
    _check_rows(orc, qb, ob, ns, fmt)
    mi, ni = np.meshgrid(np.arange(n_rows), np.arange(n_rows), indexing="ij")
    ref = orc.gemm_entries(oa[:3], ob[:3], fmt, mi.ravel(), ni.ravel()).reshape(n_rows, n_rows)
    sel = C[torch.from_numpy(ms).cuda()][:, torch.from_numpy(ns).cuda()]
    assert rel_fro(sel.cpu().numpy(), ref) <= TOL
    selb = Cb[torch.from_numpy(ms).cuda()][:, torch.from_numpy(ns).cuda()]
    assert torch.equal(selb.cpu().view(torch.int16), sel.cpu().to(torch.bfloat16).view(torch.int16))


def _gpt3(name):
    X, W, dY = synthetic.gpt3_layer(name)
    return X, W, dY


@pytest.mark.parametrize("fmt", [0, 1])
def test_gpt3_qkv_three_passes_h16(orc, fmt):
    X, W, dY = _gpt3("qkv")  # X 4096x12288, W 36864x12288, dY 4096x36864
    _sampled_gemm_check(orc, X, ROW, W, ROW, fmt, 16, seed=1)    # Fprop: X W^T
    _sampled_gemm_check(orc, dY, ROW, W, COL, fmt, 16, seed=2)   # Dgrad: dY W
    _sampled_gemm_check(orc, dY, COL, X, COL, fmt, 16, seed=3)   # Wgrad: dY^T X


@pytest.mark.parametrize("hn", [0, 32])
@pytest.mark.parametrize("fmt", [0, 1])
def test_gpt3_o_proj_rotation_grid(orc, fmt, hn):
    X, W, dY = _gpt3("o")  # 4096x12288, 12288x12288, 4096x12288
    _sampled_gemm_check(orc, X, ROW, W, ROW, fmt, hn, seed=4)
    _sampled_gemm_check(orc, dY, COL, X, COL, fmt, hn, seed=5)


def test_gpt3_fc2_fprop_mx_h16(orc):
    X, W, _ = _gpt3("fc2")  # X 4096x49152, W 12288x49152
    _sampled_gemm_check(orc, X, ROW, W, ROW, fp4.MXFP4, 16, seed=6)


# ------------------------------------------------------------------ sweep

def _whole_tensor_check(orc, x, fmt, hn, mode):
    if mode == "dual":
        rq, cq = fp4.quantize_dual(x.cuda(), fmt, hn)
        pairs = ((rq, ROW), (cq, COL))
    else:
        axis = ROW if mode == "row" else COL
        pairs = ((fp4.quantize(x.cuda(), fmt, hn, axis), axis),)
    torch.cuda.synchronize()
    for q, axis in pairs:
        o = orc.quantize(x, fmt, hn, axis)
        assert np.array_equal(np_u8(q.codes), o[0]) and np.array_equal(np_u8(q.scales), o[1])
        if fmt == fp4.NVFP4:
            assert f32_bits(q.tensor_scale.item()) == f32_bits(o[2])


@pytest.mark.parametrize("mode", ["row", "col", "dual"])
@pytest.mark.parametrize("hn", [0, 16, 32])
@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("row_len", [4096, 14336, 49152])
def test_sweep_2p20_whole_tensor(orc, row_len, fmt, hn, mode):
    x = synthetic.sweep_tensor(20, row_len, seed=row_len)
    _whole_tensor_check(orc, x, fmt, hn, mode)


@pytest.mark.parametrize("p,fmt,hn", [(28, 0, 16), (26, 1, 32)])
@pytest.mark.parametrize("row_len", [4096, 49152])
def test_sweep_large_sampled_rows(orc, row_len, p, fmt, hn):
    x = synthetic.sweep_tensor(p, row_len, seed=7, device="cuda")
    rq, cq = fp4.quantize_dual(x, fmt, hn)
    torch.cuda.synchronize()
    xc = x.cpu()
    rng = np.random.default_rng(8)
    rows = np.sort(rng.choice(rq.rows, 16, replace=False))
    cols = np.sort(rng.choice(cq.rows, 16, replace=False))
    _check_rows(orc, rq, _oracle_rows(orc, xc, ROW, rows, fmt, hn), rows, fmt)
    _check_rows(orc, cq, _oracle_rows(orc, xc, COL, cols, fmt, hn), cols, fmt)


@pytest.mark.parametrize("fmt,row_len", [(0, 14336), (0, 49152), (1, 49152)])
def test_sweep_2p30_banded_tile_order_sampled_rows(orc, fmt, row_len):
    """2^30-element tensors whose column-layout codes exceed 256 MB take the banded tile
    order (bands of 32 tile columns): sampled rows of both layouts bit-exact, tensor
    scales of both layouts bit-exact for NVFP4."""
    x = synthetic.sweep_tensor(30, row_len, seed=9, device="cuda")
    assert x.shape[1] // 128 > 32 and x.numel() // 2 > (256 << 20)
    rq, cq = fp4.quantize_dual(x, fmt, 16)
    torch.cuda.synchronize()
    assert fp4.fp4_check_status() == 0
    xc = x.cpu()
    del x
    rng = np.random.default_rng(10)
    rows = np.sort(rng.choice(rq.rows, 12, replace=False))
    cols = np.sort(rng.choice(cq.rows, 12, replace=False))
    _check_rows(orc, rq, _oracle_rows(orc, xc, ROW, rows, fmt, 16), rows, fmt)
    _check_rows(orc, cq, _oracle_rows(orc, xc, COL, cols, fmt, 16), cols, fmt)


@pytest.mark.parametrize("fmt,row_len", [(0, 4096), (0, 49152), (1, 14336)])
def test_sweep_2p30_column_layout_banded_sampled_rows(orc, fmt, row_len):
    """The column layout alone of a 2^30-element tensor takes the banded tile order:
    bands of 16 tile columns for MXFP4 (also for 4096-column tensors, which bands of 32
    leave unbanded), 32 for NVFP4: sampled rows of the transposed layout bit-exact."""
    x = synthetic.sweep_tensor(30, row_len, seed=12, device="cuda")
    assert x.shape[1] // 128 > 16 and x.numel() // 2 > (256 << 20)
    cq = fp4.quantize(x, fmt, 16, COL)
    torch.cuda.synchronize()
    assert fp4.fp4_check_status() == 0
    xc = x.cpu()
    del x
    rng = np.random.default_rng(13)
    cols = np.sort(rng.choice(cq.rows, 12, replace=False))
    _check_rows(orc, cq, _oracle_rows(orc, xc, COL, cols, fmt, 16), cols, fmt)

"""GPU parity of the MXFP8 comparator (E4M3 elements, E8M0 scale per 32 elements): the
quantiser bit for bit against the oracle in both layouts and the dual pass, and the
tcgen05 kind::mxf8f6f4 GEMM within the GEMM tolerance of the fp64 oracle, exactly on
integer-valued operands, with the bf16 output equal to RN(fp32 output)."""
import numpy as np
import pytest
import torch

import fp4_block_scaled_deterministic_b200 as fp4
from fp4_block_scaled_deterministic_b200 import synthetic
from gpu_util import need_gpu, np_u8, rel_fro

pytestmark = pytest.mark.gpu
MX8 = fp4.MXFP8
TOL = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def _x(rows, cols, seed):
    return synthetic.normal(rows, cols, 1.0, seed=seed, outlier_frac=0.01, outlier_mult=30.0)


@pytest.mark.parametrize("hn", [0, 16, 32])
@pytest.mark.parametrize("shape", [(160, 224), (384, 640), (1024, 4096)])
def test_mxfp8_quantize_matches_oracle(orc, shape, hn):
    x = _x(*shape, seed=shape[1] + hn)
    xs = x.cuda()
    rq, cq = fp4.quantize_dual(xs, MX8, hn)
    singles = [fp4.quantize(xs, MX8, hn, ax) for ax in (fp4.ROW, fp4.COL)]
    torch.cuda.synchronize()
    assert fp4.fp4_check_status() == 0
    for axis, dual, single in ((fp4.ROW, rq, singles[0]), (fp4.COL, cq, singles[1])):
        o = orc.quantize(x, MX8, hn, axis)
        for q in (dual, single):
            assert q.codes.shape == o[0].shape
            assert np.array_equal(np_u8(q.codes), o[0]), "codes differ"
            assert np.array_equal(np_u8(q.scales), o[1]), "scales differ"


@pytest.mark.parametrize("shape", [(128, 256, 256), (256, 256, 256), (160, 96, 224),
                                   (384, 512, 1024), (32, 32, 32), (256, 640, 4096)])
def test_mxfp8_gemm_matches_oracle(orc, shape):
    M, N, K = shape
    X = _x(M, K, seed=M + N + K)
    W = synthetic.normal(N, K, 0.02, seed=M + N + K + 1)
    qa, qb = fp4.quantize(X.cuda(), MX8, 16), fp4.quantize(W.cuda(), MX8, 16)
    C = fp4.gemm(qa, qb, fp4.OUT_F32)
    Cb = fp4.gemm(qa, qb, fp4.OUT_BF16)
    torch.cuda.synchronize()
    assert fp4.fp4_check_status() == 0
    oa, ob = orc.quantize(X, MX8, 16)[:3], orc.quantize(W, MX8, 16)[:3]
    assert np.array_equal(np_u8(qa.codes), oa[0]) and np.array_equal(np_u8(qb.codes), ob[0])
    ref = orc.gemm_f64(orc.dequantize(*oa, MX8), orc.dequantize(*ob, MX8))
    assert rel_fro(C.cpu().numpy(), ref) <= TOL
    assert torch.equal(Cb.cpu().view(torch.int16), C.cpu().to(torch.bfloat16).view(torch.int16))


def test_mxfp8_gemm_integer_operands_exact(orc):
    """E4M3 codes of the integers -16..16 under unit scales: every product and partial sum
    is an integer below 2^24, so fp32 accumulation in any order is exact."""
    M, N, K = 256, 512, 1024
    ints = np.arange(-16, 17, dtype=np.float32)
    import ml_dtypes
    table = ints.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(table.view(ml_dtypes.float8_e4m3fn).astype(np.float32), ints)
    rng = np.random.default_rng(9)
    a_codes = table[rng.integers(0, ints.size, (M, K))]
    b_codes = table[rng.integers(0, ints.size, (N, K))]
    a_sc = np.full(fp4.fp4_scales_bytes(M, K, MX8), 127, np.uint8)
    b_sc = np.full(fp4.fp4_scales_bytes(N, K, MX8), 127, np.uint8)
    qa = fp4.QTensor(torch.from_numpy(a_codes).cuda(), torch.from_numpy(a_sc).cuda(), None, MX8, M, K)
    qb = fp4.QTensor(torch.from_numpy(b_codes).cuda(), torch.from_numpy(b_sc).cuda(), None, MX8, N, K)
    C = fp4.gemm(qa, qb, fp4.OUT_F32)
    torch.cuda.synchronize()
    A = a_codes.view(ml_dtypes.float8_e4m3fn).astype(np.int64)
    B = b_codes.view(ml_dtypes.float8_e4m3fn).astype(np.int64)
    assert np.array_equal(C.cpu().numpy().astype(np.int64), A @ B.T)


def test_mxfp8_gemm_large_sampled(orc):
    """A Llama-sized contraction (K = 4096) over many tiles, sampled outputs."""
    M, N, K = 2048, 1024, 4096
    X = _x(M, K, seed=41)
    W = synthetic.normal(N, K, 0.02, seed=42)
    qa, qb = fp4.quantize(X.cuda(), MX8, 16), fp4.quantize(W.cuda(), MX8, 16)
    C = fp4.gemm(qa, qb, fp4.OUT_F32)
    torch.cuda.synchronize()
    oa, ob = orc.quantize(X, MX8, 16)[:3], orc.quantize(W, MX8, 16)[:3]
    rng = np.random.default_rng(3)
    ms, ns = rng.integers(0, M, 400), rng.integers(0, N, 400)
    ref = orc.gemm_entries(oa, ob, MX8, ms, ns)
    got = C.cpu().numpy()[ms, ns]
    assert np.linalg.norm(got - ref) <= TOL * np.linalg.norm(ref)


def test_mxfp8_rejects_fp4_only_options():
    x = torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fp4.Fp4Error):
        fp4.quantize(x, MX8, 16, sr_seed=1)

"""GPU parity of the block-scaled FP4 GEMM (tcgen05) against the fp64 oracle:
relative Frobenius error <= 1e-4 on the same quantised operands, exact results on
integer-valued operands, the bf16 epilogue equal to RN(fp32 epilogue), bitwise
determinism, and sampled entries at a full Llama-3.1-8B GEMM size."""
import numpy as np
import pytest
import torch

import fp4_block_scaled_deterministic_b200 as fp4
from fp4_block_scaled_deterministic_b200 import synthetic
from gpu_util import need_gpu, np_u8, rel_fro

pytestmark = pytest.mark.gpu
TOL = 1e-4  # relative Frobenius error of the fp32-output GEMM vs the fp64 oracle


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def _operands(orc, M, N, K, fmt, hn, seed):
    X = synthetic.normal(M, K, 1.0, seed=seed, outlier_frac=0.01, outlier_mult=30.0)
    W = synthetic.normal(N, K, 0.02, seed=seed + 1)
    qa = fp4.quantize(X.cuda(), fmt, hn)
    qb = fp4.quantize(W.cuda(), fmt, hn)
    oa = orc.quantize(X, fmt, hn)[:3]
    ob = orc.quantize(W, fmt, hn)[:3]
    torch.cuda.synchronize()
    assert np.array_equal(np_u8(qa.codes), oa[0]) and np.array_equal(np_u8(qb.codes), ob[0])
    return qa, qb, oa, ob


@pytest.mark.parametrize("shape", [(128, 256, 256), (256, 256, 256), (160, 96, 224),
                                   (384, 512, 1024), (32, 32, 32), (256, 640, 4096),
                                   (416, 800, 512)])
@pytest.mark.parametrize("fmt", [0, 1])
def test_gemm_matches_oracle(orc, fmt, shape):
    M, N, K = shape
    qa, qb, oa, ob = _operands(orc, M, N, K, fmt, 16, seed=M + N + K)
    C = fp4.gemm(qa, qb, fp4.OUT_F32)
    Cb = fp4.gemm(qa, qb, fp4.OUT_BF16)
    torch.cuda.synchronize()
    assert fp4.fp4_check_status() == 0
    ref = orc.gemm_f64(orc.dequantize(*oa, fmt), orc.dequantize(*ob, fmt))
    err = rel_fro(C.cpu().numpy(), ref)
    assert err <= TOL, err
    # the bf16 epilogue is the round-to-nearest-even of the fp32 one
    assert torch.equal(Cb.cpu().view(torch.int16), C.cpu().to(torch.bfloat16).view(torch.int16))


@pytest.mark.parametrize("fmt", [0, 1])
def test_gemm_integer_operands_exact(orc, fmt):
    """Random codes under unit scales: every product is a multiple of 1/4 and every
    partial sum stays below 2^22, so fp32 accumulation in any order is exact."""
    M, N, K = 256, 512, 1024
    g = torch.Generator().manual_seed(5)
    a_codes = torch.randint(0, 256, (M, K // 2), generator=g, dtype=torch.uint8)
    b_codes = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.uint8)
    one = 127 if fmt == fp4.MXFP4 else 0x38  # E8M0 2^0 / E4M3 1.0
    a_sc = torch.full((fp4.fp4_scales_bytes(M, K, fmt),), one, dtype=torch.uint8)
    b_sc = torch.full((fp4.fp4_scales_bytes(N, K, fmt),), one, dtype=torch.uint8)
    ts = torch.ones(1, dtype=torch.float32).cuda() if fmt == fp4.NVFP4 else None
    qa = fp4.QTensor(a_codes.cuda(), a_sc.cuda(), ts, fmt, M, K)
    qb = fp4.QTensor(b_codes.cuda(), b_sc.cuda(), ts, fmt, N, K)
    C = fp4.gemm(qa, qb, fp4.OUT_F32).cpu().numpy()
    ref = orc.gemm_f64(orc.dequantize(a_codes.numpy(), a_sc.numpy(), 1.0, fmt),
                       orc.dequantize(b_codes.numpy(), b_sc.numpy(), 1.0, fmt))
    assert np.array_equal(C.astype(np.float64), ref)


@pytest.mark.parametrize("N", [256, 896])
def test_gemm_per_block_scales_exact(orc, N):
    """Integer codes under varied power-of-two block scales (MXFP4): each 32-block
    product is exact, and scales are chosen so all partial sums stay exact, which
    checks that every scale byte reaches the right rows and K blocks. N = 896 takes
    256 x 384 tiles (two full, one of 128 columns)."""
    M, K = 256, 384  # 1.5 K-slabs: also covers the zero-filled K tail
    g = torch.Generator().manual_seed(6)
    a_codes = torch.randint(0, 256, (M, K // 2), generator=g, dtype=torch.uint8)
    b_codes = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.uint8)
    # scales 2^-1..2^1: products are multiples of 2^-4 below 144, sums below 2^16
    a_sc = torch.randint(126, 129, (fp4.fp4_scales_bytes(M, K, 0),), generator=g, dtype=torch.uint8)
    b_sc = torch.randint(126, 129, (fp4.fp4_scales_bytes(N, K, 0),), generator=g, dtype=torch.uint8)
    qa = fp4.QTensor(a_codes.cuda(), a_sc.cuda(), None, 0, M, K)
    qb = fp4.QTensor(b_codes.cuda(), b_sc.cuda(), None, 0, N, K)
    C = fp4.gemm(qa, qb, fp4.OUT_F32).cpu().numpy()
    ref = orc.gemm_f64(orc.dequantize(a_codes.numpy(), a_sc.numpy(), None, 0),
                       orc.dequantize(b_codes.numpy(), b_sc.numpy(), None, 0))
    assert np.array_equal(C.astype(np.float64), ref)


def test_gemm_is_deterministic(orc):
    qa, qb, _, _ = _operands(orc, 512, 768, 2048, 0, 16, seed=9)
    C1 = fp4.gemm(qa, qb, fp4.OUT_F32)
    C2 = fp4.gemm(qa, qb, fp4.OUT_F32)
    torch.cuda.synchronize()
    assert torch.equal(C1.view(torch.int32), C2.view(torch.int32))


@pytest.mark.parametrize("fmt", [0, 1])
def test_gemm_full_llama_gate_sampled(orc, fmt):
    """Fprop of the Llama-3.1-8B gate projection at full size (M=8192, N=14336,
    K=4096, H16), the benchmark's launch configuration: operands bit-exact against
    the oracle, 512 sampled outputs within the tolerance against the oracle's own
    sums, the whole output within the tolerance against an fp64 library matmul of the
    oracle-dequantised operands, bf16 = RN(fp32)."""
    X, W, _ = synthetic.llama_layer("gate")
    qa = fp4.quantize(X.cuda(), fmt, 16)
    qb = fp4.quantize(W.cuda(), fmt, 16)
    C = fp4.gemm(qa, qb, fp4.OUT_F32)
    Cb = fp4.gemm(qa, qb, fp4.OUT_BF16)
    torch.cuda.synchronize()
    oa = orc.quantize(X, fmt, 16)[:3]
    ob = orc.quantize(W, fmt, 16)[:3]
    assert np.array_equal(np_u8(qa.codes), oa[0]) and np.array_equal(np_u8(qa.scales), oa[1])
    assert np.array_equal(np_u8(qb.codes), ob[0]) and np.array_equal(np_u8(qb.scales), ob[1])
    rng = np.random.default_rng(2)
    ms = rng.integers(0, 8192, 512)
    ns = rng.integers(0, 14336, 512)
    ref = orc.gemm_entries(oa, ob, fmt, ms, ns)
    got = C[torch.from_numpy(ms).cuda(), torch.from_numpy(ns).cuda()].cpu().numpy()
    assert rel_fro(got, ref) <= TOL
    assert torch.equal(Cb.view(torch.int16), C.to(torch.bfloat16).view(torch.int16))
    # Whole output: deq(A) deq(B)^T in fp64 (operands dequantised by the oracle).
    da = torch.from_numpy(orc.dequantize(*oa, fmt)).cuda()
    db = torch.from_numpy(orc.dequantize(*ob, fmt)).cuda()
    full = da @ db.T
    del da, db
    err = float((C.double() - full).norm() / full.norm())
    assert err <= TOL, err


@pytest.mark.parametrize("shape", [(160, 96, 224), (384, 512, 1024), (96, 320, 256)])
@pytest.mark.parametrize("fmt", [0, 1])
def test_gemm_16byte_aligned_output(orc, fmt, shape):
    """An output that is 16- but not 32-byte aligned takes the 16-byte store path and
    holds the same bits as the 32-byte-aligned one."""
    M, N, K = shape
    qa, qb, _, _ = _operands(orc, M, N, K, fmt, 16, seed=7 * M + N)
    for od, dt, off in ((fp4.OUT_F32, torch.float32, 4), (fp4.OUT_BF16, torch.bfloat16, 8)):
        ref = fp4.gemm(qa, qb, od)
        buf = torch.full((M * N + off,), float("nan"), dtype=dt, device="cuda")
        out = buf[off:].view(M, N)
        assert out.data_ptr() % 32 == 16
        fp4.gemm(qa, qb, od, out=out)
        torch.cuda.synchronize()
        assert fp4.fp4_check_status() == 0
        assert torch.equal(out.view(torch.int16 if od == fp4.OUT_BF16 else torch.int32),
                           ref.view(torch.int16 if od == fp4.OUT_BF16 else torch.int32))

"""fp4_gemm_quant: the GEMM epilogue that also quantises its bf16 output for the next
layer (row-wise MXFP4, rotation along N). Its bf16 output must equal fp4_gemm's bit
for bit, and its codes and scales must equal the oracle's row-wise quantisation of
that bf16 output, whole tensors (padding bytes included), for MXFP4 and NVFP4
operands, every rotation size, ragged shapes (M <= 128, M and N not multiples of
128) and the full Llama-3.1-8B QKV Fprop."""
import numpy as np
import pytest
import torch

import fp4_block_scaled_deterministic_b200 as fp4
from fp4_block_scaled_deterministic_b200 import synthetic
from gpu_util import need_gpu, np_u8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def _operands(M, N, K, fmt, seed):
    X = synthetic.normal(M, K, 1.0, seed=seed, outlier_frac=0.01, outlier_mult=30.0).cuda()
    W = synthetic.normal(N, K, 0.02, seed=seed + 1).cuda()
    return fp4.quantize(X, fmt, 16), fp4.quantize(W, fmt, 16)


def _check(orc, qa, qb, q_hn):
    Y_ref = fp4.gemm(qa, qb, fp4.OUT_BF16)
    Y, Q = fp4.gemm_quant(qa, qb, q_hn)
    _, Q2 = fp4.gemm_quant(qa, qb, q_hn, with_output=False)
    torch.cuda.synchronize()
    assert fp4.fp4_check_status() == 0
    assert torch.equal(Y.view(torch.int16), Y_ref.view(torch.int16))
    oc, os_, _, _ = orc.quantize(Y.cpu(), orc.MXFP4, q_hn, orc.ROW)
    assert np.array_equal(np_u8(Q.codes), oc), "fused codes differ from the oracle"
    assert np.array_equal(np_u8(Q.scales), os_), "fused scales differ from the oracle"
    assert torch.equal(Q2.codes, Q.codes) and torch.equal(Q2.scales, Q.scales)


@pytest.mark.parametrize("shape", [(256, 384, 512), (160, 96, 224), (96, 320, 256),
                                   (512, 640, 1024), (288, 4096, 256)])
@pytest.mark.parametrize("q_hn", [0, 16, 32])
@pytest.mark.parametrize("fmt", [0, 1])
def test_fused_output_quantisation(orc, fmt, q_hn, shape):
    M, N, K = shape
    qa, qb = _operands(M, N, K, fmt, seed=M + 3 * N + K)
    _check(orc, qa, qb, q_hn)


def test_fused_output_quantisation_llama_qkv(orc):
    """The full Llama-3.1-8B QKV Fprop (8192 x 6144 x 4096), MXFP4 + H16 in and out."""
    X, W, _ = synthetic.llama_layer("qkv")
    qa = fp4.quantize(X.cuda(), fp4.MXFP4, 16)
    qb = fp4.quantize(W.cuda(), fp4.MXFP4, 16)
    _check(orc, qa, qb, 16)


def test_fused_output_rejects_bad_arguments():
    qa, qb = _operands(128, 128, 128, 0, seed=1)
    Y = torch.empty(128, 128, dtype=torch.bfloat16, device="cuda")
    codes = torch.empty(128, 64, dtype=torch.uint8, device="cuda")
    scales = torch.empty(fp4.fp4_scales_bytes(128, 128, 0), dtype=torch.uint8, device="cuda")
    args = (qa.codes, qa.scales, None, qb.codes, qb.scales, None)
    assert fp4.fp4_gemm_quant(*args, Y, codes, scales, 128, 128, 128, 0, 8) == 1
    assert fp4.fp4_gemm_quant(*args, Y, None, scales, 128, 128, 128, 0, 16) == 1
    assert fp4.fp4_gemm_quant(*args, Y, codes, scales, 128, 128, 128, 2, 16) == 1
    assert fp4.fp4_gemm_quant(*args, Y, codes, scales, 128, 128, 128, 0, 16) == 0
    torch.cuda.synchronize()


def _same_bits(a, b):
    if a.dtype == torch.bfloat16:
        return torch.equal(a.view(torch.int16), b.view(torch.int16))
    return torch.equal(a.view(torch.int32), b.view(torch.int32))


@pytest.mark.parametrize("fmt", [fp4.MXFP4, fp4.NVFP4])
@pytest.mark.parametrize("shape,q_index", [((256, 512, 1024), 0), ((160, 288, 640), 1),
                                           ((8192, 6144, 4096), 0)])
def test_group_with_fused_output_quantisation(orc, fmt, shape, q_index):
    """fp4_gemm_group_quant: a layer's Fprop, Dgrad and Wgrad in one launch, the member
    q_index (a bf16 output) also quantised in its epilogue. Its output and codes equal
    fp4_gemm_quant's bit for bit, the other members equal fp4_gemm's, and the codes
    equal the oracle's row-wise quantisation of that bf16 output."""
    M, N, K = shape
    X = synthetic.normal(M, K, 1.0, seed=M + 3, outlier_frac=0.01, outlier_mult=30.0).cuda()
    W = synthetic.normal(N, K, 0.02, seed=N + 5).cuda()
    dY = synthetic.heavy_tailed_grad(M, N, 1e-3, seed=K + 7).cuda()
    xr, xc = fp4.quantize_dual(X, fmt, 16)
    wr, wc = fp4.quantize_dual(W, fmt, 16)
    yr, yc = fp4.quantize_dual(dY, fmt, 16)
    probs = [(xr, wr), (yr, wc), (yc, xc)]              # Fprop, Dgrad, Wgrad
    ods = [fp4.OUT_BF16, fp4.OUT_BF16, fp4.OUT_F32]
    outs, Q = fp4.gemm_group_quant(probs, ods, q_index, 16)
    a, b = probs[q_index]
    Y_ref, Q_ref = fp4.gemm_quant(a, b, 16)
    refs = [fp4.gemm(pa, pb, od) for (pa, pb), od in zip(probs, ods)]
    torch.cuda.synchronize()
    assert fp4.fp4_check_status() == 0
    for out, ref in zip(outs, refs):
        assert _same_bits(out, ref)
    assert _same_bits(outs[q_index], Y_ref)
    assert torch.equal(Q.codes, Q_ref.codes) and torch.equal(Q.scales, Q_ref.scales)
    if M * N <= 1 << 20:  # the oracle on the smaller shapes (the full one equals gemm_quant)
        oc, os_, _, _ = orc.quantize(outs[q_index].cpu(), orc.MXFP4, 16, orc.ROW)
        assert np.array_equal(np_u8(Q.codes), oc) and np.array_equal(np_u8(Q.scales), os_)

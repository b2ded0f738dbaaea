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

"""Cross-check of the block-scaled MXFP4 GEMM against an independent implementation:
cuBLASLt's MXFP4 GEMM as torch exposes it (torch.nn.functional.scaled_mm with
BlockWise1x32 E8M0 scales in the 32x4x4 swizzled layout, which is also this library's
scale-atom layout). Both accumulate the same block-scaled products in fp32 on the
tensor cores, so their bf16 outputs (round-to-nearest of the fp32 accumulator) agree
bit for bit on every shape checked. This supplements the oracle parity tests (the
product against the oracle is checked in test_gpu_gemm.py and test_gpu_llama_full.py);
it is skipped where torch does not offer the library path."""
import pytest
import torch

import fp4_block_scaled_deterministic_b200 as fp4
from fp4_block_scaled_deterministic_b200 import synthetic
from gpu_util import need_gpu

pytestmark = pytest.mark.gpu


def _library_mxfp4(a: "fp4.QTensor", b: "fp4.QTensor"):
    """C = A B^T in bf16 through torch's cuBLASLt MXFP4 path, or None if unavailable."""
    F = torch.nn.functional
    if not (hasattr(F, "scaled_mm") and hasattr(F, "ScalingType") and hasattr(torch, "float4_e2m1fn_x2")):
        return None
    try:
        return F.scaled_mm(a.codes.view(torch.float4_e2m1fn_x2),
                           b.codes.view(torch.float4_e2m1fn_x2).t(),
                           a.scales.view(torch.float8_e8m0fnu), F.ScalingType.BlockWise1x32,
                           b.scales.view(torch.float8_e8m0fnu), F.ScalingType.BlockWise1x32,
                           swizzle_a=F.SwizzleType.SWIZZLE_32_4_4,
                           swizzle_b=F.SwizzleType.SWIZZLE_32_4_4,
                           output_dtype=torch.bfloat16)
    except (RuntimeError, TypeError, AttributeError):
        return None


@pytest.mark.parametrize("shape", [(256, 256, 256), (512, 768, 1024), (1024, 2048, 4096),
                                   (8192, 14336, 4096)])
def test_bf16_output_equals_library(shape):
    need_gpu()
    M, N, K = shape
    X = synthetic.normal(M, K, 1.0, seed=M + K, outlier_frac=0.01, outlier_mult=30.0).cuda()
    W = synthetic.normal(N, K, 0.02, seed=N + K).cuda()
    qa, qb = fp4.quantize(X, fp4.MXFP4, 16), fp4.quantize(W, fp4.MXFP4, 16)
    ours = fp4.gemm(qa, qb, fp4.OUT_BF16)
    ref = _library_mxfp4(qa, qb)
    if ref is None:
        pytest.skip("torch offers no cuBLASLt MXFP4 GEMM here")
    torch.cuda.synchronize()
    assert ours.shape == ref.shape
    assert torch.equal(ours.view(torch.int16), ref.contiguous().view(torch.int16))
    assert fp4.fp4_check_status() == 0

"""Cross-check of the block-scaled GEMMs against an independent implementation:
cuBLASLt's MXFP4, NVFP4 and MXFP8 GEMMs as torch exposes them
(torch.nn.functional.scaled_mm: E8M0 scales per 32 for MX, E4M3 scales per 16 under
an fp32 tensor scale for NVFP4, in the 32x4x4 swizzled layout, which is also this
library's scale-atom layout). Both accumulate the same block-scaled products in fp32
on the tensor cores, so their bf16 outputs (round-to-nearest of the fp32 accumulator,
times S_A*S_B for NVFP4) agree bit for bit on every shape checked. This supplements
the oracle parity tests (the product against the oracle is checked in test_gpu_gemm.py
and test_gpu_llama_full.py); it is skipped where torch does not offer the library
path."""
import pytest
import torch

import fp4_block_scaled_deterministic_b200 as fp4
from fp4_block_scaled_deterministic_b200 import synthetic
from gpu_util import need_gpu

pytestmark = pytest.mark.gpu


def _library_gemm(a: "fp4.QTensor", b: "fp4.QTensor", fmt: int):
    """C = A B^T in bf16 through torch's cuBLASLt path for fmt, or None if unavailable."""
    F = torch.nn.functional
    if not (hasattr(F, "scaled_mm") and hasattr(F, "ScalingType") and hasattr(torch, "float4_e2m1fn_x2")):
        return None
    ST, SW = F.ScalingType, F.SwizzleType
    try:
        if fmt == fp4.NVFP4:  # two levels: E4M3 blocks, then the fp32 tensor scale S
            for sw in ([SW.SWIZZLE_32_4_4, SW.NO_SWIZZLE], [SW.SWIZZLE_32_4_4]):
                try:
                    return F.scaled_mm(a.codes.view(torch.float4_e2m1fn_x2),
                                       b.codes.view(torch.float4_e2m1fn_x2).t(),
                                       [a.scales.view(torch.float8_e4m3fn), a.tensor_scale],
                                       [ST.BlockWise1x16, ST.TensorWise],
                                       [b.scales.view(torch.float8_e4m3fn), b.tensor_scale],
                                       [ST.BlockWise1x16, ST.TensorWise],
                                       swizzle_a=sw, swizzle_b=sw, output_dtype=torch.bfloat16)
                except (RuntimeError, TypeError, ValueError):
                    continue
            return None
        dt = torch.float8_e4m3fn if fmt == fp4.MXFP8 else torch.float4_e2m1fn_x2
        return F.scaled_mm(a.codes.view(dt), b.codes.view(dt).t(),
                           a.scales.view(torch.float8_e8m0fnu), ST.BlockWise1x32,
                           b.scales.view(torch.float8_e8m0fnu), ST.BlockWise1x32,
                           swizzle_a=SW.SWIZZLE_32_4_4, swizzle_b=SW.SWIZZLE_32_4_4,
                           output_dtype=torch.bfloat16)
    except (RuntimeError, TypeError, AttributeError, ValueError):
        return None


@pytest.mark.parametrize("fmt", [fp4.MXFP4, fp4.NVFP4, fp4.MXFP8])
@pytest.mark.parametrize("shape", [(256, 256, 256), (512, 768, 1024), (1024, 2048, 4096),
                                   (8192, 14336, 4096)])
def test_bf16_output_equals_library(shape, fmt):
    need_gpu()
    M, N, K = shape
    X = synthetic.normal(M, K, 1.0, seed=M + K, outlier_frac=0.01, outlier_mult=30.0).cuda()
    W = synthetic.normal(N, K, 0.02, seed=N + K).cuda()
    qa, qb = fp4.quantize(X, fmt, 16), fp4.quantize(W, fmt, 16)
    ours = fp4.gemm(qa, qb, fp4.OUT_BF16)
    ref = _library_gemm(qa, qb, fmt)
    if ref is None:
        pytest.skip("torch offers no cuBLASLt GEMM for this format here")
    torch.cuda.synchronize()
    assert ours.shape == ref.shape
    assert torch.equal(ours.view(torch.int16), ref.contiguous().view(torch.int16))
    assert fp4.fp4_check_status() == 0

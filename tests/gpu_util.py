"""Shared helpers of the GPU parity tests (test plumbing only)."""
import numpy as np
import pytest
import torch

import fp4_block_scaled_deterministic_b200 as fp4


def need_gpu():
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    from fp4_block_scaled_deterministic_b200 import build
    build.build()
    fp4.lib()


def np_u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def f32_bits(x: float) -> int:
    return int(np.array([x], np.float32).view(np.uint32)[0])


def rel_fro(a: np.ndarray, b: np.ndarray) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def gpu_quantize_raw(x_cpu: torch.Tensor, fmt: int, hn: int, axis: int):
    """Quantise through the C entry point; returns numpy codes, scales and (NVFP4)
    the two tensor-scale cells {S, amax}."""
    x = x_cpu.cuda().contiguous()
    rows, cols = x.shape
    R, C = (rows, cols) if axis == fp4.ROW else (cols, rows)
    codes = torch.full((R, C // 2), 0xAB, dtype=torch.uint8, device="cuda")
    scales = torch.full((max(1, fp4.fp4_scales_bytes(R, C, fmt)),), 0xCD, dtype=torch.uint8,
                        device="cuda")
    ts = torch.full((2,), -1.0, dtype=torch.float32, device="cuda") if fmt == fp4.NVFP4 else None
    st = fp4.fp4_quantize(x, codes, scales, ts, rows, cols, fmt, hn, axis)
    assert st == 0, fp4.status_string(st)
    torch.cuda.synchronize()
    assert fp4.fp4_check_status() == 0
    return np_u8(codes), np_u8(scales), (None if ts is None else ts.cpu().numpy())

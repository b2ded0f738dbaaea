"""The CUDA quantiser on the hand-worked NVFP4 examples of
tests/golden/nvfp4_block_rounding.json: the tensor scale, the block-scale byte, the
pinned nibbles, and every other code and scale byte, bit for bit against the golden
file and the oracle, in the single-layout and the dual-layout kernels. The examples
put the block-scale quotient one unit below an E4M3 tie and the element quotient
one unit below an E2M1 tie, where a reciprocal multiply or another operation order
lands on the tie and rounds the other way."""
import numpy as np
import pytest
import torch

import fp4_block_scaled_deterministic_b200 as fp4
from golden_util import load, nibble, nv_case_tensor
from gpu_util import f32_bits, gpu_quantize_raw, need_gpu, np_u8

pytestmark = pytest.mark.gpu
CASES = load("nvfp4_block_rounding.json")["cases"]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def _check_golden(codes, scales, S, amax, case, KB):
    exp = case["expect"]
    assert format(f32_bits(S), "08x") == exp["S_f32_hex"]
    assert format(f32_bits(amax), "08x") == exp["amax_f32_hex"]
    r, kb, byte = exp["scale"]
    off = (r // 128 * ((KB + 3) // 4) + kb // 4) * 512 + (r % 32) * 16 + (r % 128) // 32 * 4 + kb % 4
    assert scales[off] == int(byte, 16)
    for r, c, want in exp["nibbles"]:
        assert nibble(codes, r, c) == want, (r, c)


@pytest.mark.parametrize("case", CASES, ids=[c["name"] for c in CASES])
def test_nvfp4_golden_single_layout(orc, case):
    x = nv_case_tensor(case)
    codes, scales, ts = gpu_quantize_raw(x, fp4.NVFP4, 0, fp4.ROW)
    _check_golden(codes, scales, ts[0], ts[1], case, x.shape[1] // 16)
    oc, os_, oS, oT = orc.quantize(x, orc.NVFP4, 0, orc.ROW)
    assert np.array_equal(codes, oc) and np.array_equal(scales, os_)


@pytest.mark.parametrize("case", CASES, ids=[c["name"] for c in CASES])
def test_nvfp4_golden_dual_layout(orc, case):
    x = nv_case_tensor(case).cuda()
    rows, cols = x.shape
    rc = torch.empty(rows, cols // 2, dtype=torch.uint8, device="cuda")
    cc = torch.empty(cols, rows // 2, dtype=torch.uint8, device="cuda")
    rs = torch.empty(fp4.fp4_scales_bytes(rows, cols, fp4.NVFP4), dtype=torch.uint8, device="cuda")
    cs = torch.empty(fp4.fp4_scales_bytes(cols, rows, fp4.NVFP4), dtype=torch.uint8, device="cuda")
    ts = torch.full((4,), -1.0, dtype=torch.float32, device="cuda")  # {S_row, S_col, amax_row, amax_col}
    st = fp4.fp4_quantize_dual(x, rc, rs, cc, cs, ts, rows, cols, fp4.NVFP4, 0)
    assert st == 0, fp4.status_string(st)
    torch.cuda.synchronize()
    assert fp4.fp4_check_status() == 0
    t = ts.cpu().numpy()
    _check_golden(np_u8(rc), np_u8(rs), t[0], t[2], case, cols // 16)
    oc, os_, oS, oT = orc.quantize(x.cpu(), orc.NVFP4, 0, orc.COL)
    assert np.array_equal(np_u8(cc), oc) and np.array_equal(np_u8(cs), os_)
    assert f32_bits(t[1]) == f32_bits(oS) and f32_bits(t[3]) == f32_bits(oT)

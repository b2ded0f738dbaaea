"""Pins of the oracle's NVFP4 block path against hand-worked examples
(tests/golden/nvfp4_block_rounding.json): the rounding order of the block-scale
quotient t = RN(B / RN(6 S)), the element quotient q = RN(v / d) as an IEEE division
by d = RN(e4m3(sb) S), and signed zero codes under a zero block scale. Each example
was chosen so that the other plausible orders (6 S kept exact, B/6 before /S, a
reciprocal multiply, d kept exact, v/S before /e4m3(sb)) give a different byte."""
import numpy as np
import pytest

from golden_util import load, nibble, nv_case_tensor

CASES = load("nvfp4_block_rounding.json")["cases"]


def _f32_hex(x) -> str:
    return format(int(np.array([x], np.float32).view(np.uint32)[0]), "08x")


@pytest.mark.parametrize("case", CASES, ids=[c["name"] for c in CASES])
def test_nvfp4_block_rounding_golden(orc, case):
    x = nv_case_tensor(case)
    codes, scales, S, amax = orc.quantize(x, orc.NVFP4, 0, orc.ROW)
    exp = case["expect"]
    assert _f32_hex(S) == exp["S_f32_hex"]
    assert _f32_hex(amax) == exp["amax_f32_hex"]
    r, kb, byte = exp["scale"]
    assert scales[orc.scale_offset(r, kb, x.shape[1] // 16)] == int(byte, 16)
    for r, c, want in exp["nibbles"]:
        assert nibble(codes, r, c) == want, (r, c)


def test_nvfp4_block_scale_alone(orc):
    """The block quantiser on its own, given S, reproduces the first case's scale byte."""
    case = CASES[0]
    S = np.frombuffer(bytes.fromhex(case["expect"]["S_f32_hex"])[::-1], np.float32)[0]
    B = np.float32(19 * 2.0 ** -16)
    _, sb = orc.quantize_block_nv(np.array([B] + [0.0] * 15, np.float32), float(S))
    assert sb == 0x03

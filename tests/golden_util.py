"""Loading of the hand-worked golden files under tests/golden/ (test plumbing only)."""
import json
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load(name: str) -> dict:
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def nv_case_tensor(case: dict, rows: int = 32, cols: int = 32) -> torch.Tensor:
    """The case's bf16 tensor: zeros except the listed (row, col, bf16 hex) elements."""
    bits = np.zeros((rows, cols), np.uint16)
    for r, c, h in case["elements"]:
        bits[r, c] = int(h, 16)
    return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16)


def nibble(codes: np.ndarray, r: int, c: int) -> int:
    """Code of element (r, c) of a packed [R][C/2] code matrix (element 2i low nibble)."""
    b = int(codes[r, c // 2])
    return (b >> 4) & 15 if c & 1 else b & 15

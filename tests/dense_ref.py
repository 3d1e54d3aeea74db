"""Independent numpy decoding of the generator's interchange form, used by the
oracle's pin tests (dense reductions and brute force).  Tests only."""
import numpy as np

OFFSET = {0: 1.0, 1: 1.5, 2: 3.5}


def codes_int(codes: np.ndarray, hi) -> np.ndarray:
    """int [rows][K] full code values from the interchange form."""
    rows, kb = codes.shape
    c = np.empty((rows, kb * 4), dtype=np.int64)
    for i in range(4):
        c[:, i::4] = (codes >> (2 * i)) & 3
    if hi is not None:
        h = np.empty((rows, hi.shape[1] * 8), dtype=np.int64)
        for i in range(8):
            h[:, i::8] = (hi >> i) & 1
        c += 4 * h
    return c


def dequant(fmt: int, mat) -> np.ndarray:
    codes, hi, scales = mat
    c = codes_int(codes, hi).astype(np.float64)
    s = np.repeat(scales.view(np.float16).astype(np.float64), 64, axis=1)
    return (c - OFFSET[fmt]) * s


def silu(a):
    return a / (1.0 + np.exp(-a))


def expert_dense(fmt: int, mats: dict, x64: np.ndarray) -> np.ndarray:
    """[n][H] outputs of one expert for fp64 inputs x64 [n][H]."""
    Wg, Wu, Wd = (dequant(fmt, mats[m]) for m in ("gate", "up", "down"))
    return (silu(x64 @ Wg.T) * (x64 @ Wu.T)) @ Wd.T

"""Empirical conditional entropy of BF16 words, H(s) + H(f | s), in bits per weight.

This is a measurement used by the size gates. s = w >> 7 is the sign+exponent
symbol and f = w & 0x7F the fraction, as in the NVLC model card's field split.
"""
import numpy as np


def conditional_entropy_bits(words: np.ndarray) -> float:
    """Total bits n * (H(s) + H(f|s)) of the empirical distribution of ``words``."""
    w = np.asarray(words).reshape(-1).astype(np.int64)
    n = w.size
    if n == 0:
        return 0.0
    joint = np.bincount(w & 0xFFFF, minlength=65536).astype(np.float64).reshape(512, 128)
    cs = joint.sum(axis=1)
    # n*H(s) + n*H(f|s) = -sum_s c_s log2(c_s/n) - sum_{s,f} c_sf log2(c_sf/c_s) = -sum c_sf log2(c_sf/n)
    nz = joint > 0
    return float(-(joint[nz] * np.log2(joint[nz] / n)).sum())


def split_entropy_bits(words: np.ndarray):
    """(n*H(s), n*H(f|s)) separately."""
    w = np.asarray(words).reshape(-1).astype(np.int64)
    n = w.size
    joint = np.bincount(w & 0xFFFF, minlength=65536).astype(np.float64).reshape(512, 128)
    cs = joint.sum(axis=1)
    nzs = cs > 0
    hs = float(-(cs[nzs] * np.log2(cs[nzs] / n)).sum())
    return hs, conditional_entropy_bits(words) - hs

"""Comparison rules between the CUDA path and the CPU oracle.

Tolerances (derived from the arithmetic; the method states none beyond 1e-3 relative):
* S, S1 (fp32 on the GPU vs float64 in the oracle): |gpu - ora| <= 1e-3 |ora| wherever
  ora >= 1e-20 * (row max). Below that floor the GPU's fp32 exponentials may underflow
  or flush to zero, so there the GPU value only has to be <= 1e-17 * (row max).
* S2 is the absolute value of a bf16 number: bit-exact.
* Kept positions: identical to the oracle's, except positions whose oracle score lies
  within 1e-3 relative of the oracle's (B - w)-th candidate score (near ties, where the
  fp32 and float64 orders may differ).
* The selection itself, given the same fp32 scores, must match exactly.
* Compacted K/V given the indices: bit-exact.
"""
import numpy as np
import torch

REL = 1e-3
FLOOR = 1e-20
TINY = 1e-17


def to_dev(bits: np.ndarray) -> torch.Tensor:
    """bf16 bit patterns (uint16) -> bf16 CUDA tensor with the same bits."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def to_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def check_scores(gpu: np.ndarray, ora: np.ndarray, what: str):
    gpu = gpu.astype(np.float64)
    mx = ora.max(-1, keepdims=True)
    big = ora >= FLOOR * mx
    err = np.abs(gpu - ora)
    bad = big & (err > REL * ora)
    if bad.any():
        pos = np.argwhere(bad)[:5]
        raise AssertionError(f"{what}: {bad.sum()} values off by more than {REL} relative; first "
                             f"{[(tuple(p), gpu[tuple(p)], ora[tuple(p)]) for p in pos]}")
    small_bad = (~big) & (gpu > TINY * np.broadcast_to(mx, gpu.shape))
    assert not small_bad.any(), f"{what}: {small_bad.sum()} underflowed values too large"
    assert np.isfinite(gpu).all(), f"{what}: non-finite values"


def check_idx_valid(idx: np.ndarray, L: int, w: int, B: int):
    assert idx.shape[-1] == B
    rows = idx.reshape(-1, B)
    assert (rows >= 0).all() and (rows < L).all()
    if B > 1:
        assert (np.diff(rows, axis=1) > 0).all(), "kept positions not strictly ascending"
    assert (rows[:, B - w:] == np.arange(L - w, L)).all(), "window not kept"


def check_idx_near_ties(gpu_idx: np.ndarray, ora_idx: np.ndarray, ora_score: np.ndarray, w: int, B: int):
    L = ora_score.shape[-1]
    n, k = L - w, B - w
    g = gpu_idx.reshape(-1, B)
    o = ora_idx.reshape(-1, B)
    s = ora_score.reshape(-1, L)
    mismatched = 0
    for r in range(g.shape[0]):
        if np.array_equal(g[r], o[r]):
            continue
        kth = np.sort(s[r, :n])[::-1][k - 1]
        diff = np.setxor1d(g[r], o[r])
        far = diff[np.abs(s[r, diff] - kth) > REL * kth]
        assert far.size == 0, (f"row {r}: kept sets differ at positions {far[:10]} whose oracle "
                               f"scores {s[r, far[:10]]} are not near the threshold {kth}")
        mismatched += diff.size
    return mismatched

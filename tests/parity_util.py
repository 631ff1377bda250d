"""Helpers shared by the GPU parity tests: tolerances, row sampling, lazy
fp64 views of bf16 tensors for the oracle, and the comparison itself."""

from __future__ import annotations

import numpy as np
import torch

# Output tolerances (bf16 O against the fp64 oracle; LSE relative, with the
# denominator floored at 1 so rows whose LSE is near 0 are held to 1e-3 absolute).
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_REL = 1e-3


class F64View:
    """Index a (CPU) bf16/fp32 torch tensor and get float64 numpy back."""

    def __init__(self, t: torch.Tensor):
        self.t = t
        self.shape = tuple(t.shape)

    def __getitem__(self, idx):
        return self.t[idx].to(torch.float64).numpy()


def sample_rows(L: int, s: int, c: int, n_random: int = 256, seed: int = 0):
    """Rows that stress the index rule: first/last row of every chunk, rows at
    i mod s in {w-1, w, w+1}, the last 8 rows, plus seeded random rows."""
    w = c - s
    rows = set()
    for start in range(0, L, s):
        rows.update({start, min(start + s, L) - 1})
        for im in (w - 1, w, w + 1):
            if 0 <= im < s and start + im < L:
                rows.add(start + im)
    rows.update(range(max(0, L - 8), L))
    rng = np.random.default_rng(seed)
    rows.update(int(x) for x in rng.integers(0, L, size=min(n_random, L)))
    return sorted(rows)


def sample_heads(Hq: int, Hkv: int):
    G = Hq // Hkv
    return sorted({0, G - 1, min(G, Hq - 1), Hq - 1})


def compare_rows(O_gpu: torch.Tensor, LSE_gpu: torch.Tensor, ref: dict):
    """O_gpu [B, L, Hq, D] (bf16, CPU), LSE_gpu [B, Hq, L]; ref from the oracle
    {(b, h, i): (O, LSE)}.  Returns (max_abs, mean_abs, max_lse_rel)."""
    keys = sorted(ref)
    o_ref = np.stack([ref[k][0] for k in keys])
    l_ref = np.array([ref[k][1] for k in keys])
    o_got = np.stack([O_gpu[b, i, h].to(torch.float64).numpy() for b, h, i in keys])
    l_got = np.array([float(LSE_gpu[b, h, i]) for b, h, i in keys])
    err = np.abs(o_got - o_ref)
    return float(err.max()), float(err.mean()), float(np.max(np.abs(l_got - l_ref) /
                                                              np.maximum(np.abs(l_ref), 1.0)))


def assert_close(max_abs, mean_abs, lse_rel, what=""):
    assert np.isfinite(max_abs) and max_abs <= O_MAX_ABS, f"{what}: O max-abs {max_abs}"
    assert mean_abs <= O_MEAN_ABS, f"{what}: O mean-abs {mean_abs}"
    assert lse_rel <= LSE_REL, f"{what}: LSE rel {lse_rel}"

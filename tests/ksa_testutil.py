"""Helpers shared by the tests: tolerances, comparisons, and the mapping
between the library's augmented layout (documented in include/ksa.h) and
(sequence, text index) / (sequence, summary index)."""
from __future__ import annotations

import numpy as np
import torch

# Accuracy bar for bf16 inputs against the fp64 oracle.
MAX_ABS = 2e-2
REL_FROB = 5e-3
# LSE: scores carry the same bf16 rounding of rotated q/k; same absolute bar.
LSE_ABS = 2e-2


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def assert_close(gpu: np.ndarray, ref: np.ndarray, what: str, max_abs=MAX_ABS, rel_frob=REL_FROB):
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite values"
    err = np.abs(gpu - ref)
    ma = float(err.max()) if err.size else 0.0
    rf = float(np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-30)) if err.size else 0.0
    assert ma <= max_abs, f"{what}: max-abs {ma:.3e} > {max_abs}"
    if rel_frob is not None:
        assert rf <= rel_frob, f"{what}: rel-Frobenius {rf:.3e} > {rel_frob}"
    return ma, rf


class RowSet:
    """Output rows of one test compared with the oracle: max-abs on every row
    as it is added, relative Frobenius over all added rows together (the bar
    applies to the test's outputs as one set, so a row whose reference is
    small does not decide it alone)."""

    def __init__(self, what: str, max_abs=MAX_ABS, rel_frob=REL_FROB):
        self.what, self.max_abs, self.rel_frob = what, max_abs, rel_frob
        self.got, self.want = [], []

    def add(self, gpu: np.ndarray, ref: np.ndarray, what: str):
        assert_close(gpu, ref, what, max_abs=self.max_abs, rel_frob=None)
        self.got.append(np.asarray(gpu, np.float64).ravel())
        self.want.append(np.asarray(ref, np.float64).ravel())

    def check(self):
        assert self.got, f"{self.what}: no rows were checked"
        return assert_close(np.concatenate(self.got), np.concatenate(self.want), self.what,
                            max_abs=self.max_abs, rel_frob=self.rel_frob)


def chunk_offsets(seqlens, k):
    off = [0]
    for n in seqlens:
        off.append(off[-1] + (n + k - 1) // k)
    return off


def text_rows(seqlens, k, b, idx):
    """Augmented row of text tokens idx (array) of sequence b."""
    off = chunk_offsets(seqlens, k)[b]
    idx = np.asarray(idx, dtype=np.int64)
    return (off + idx // k) * (k + 1) + idx % k


def summary_rows(seqlens, k, b, idx):
    off = chunk_offsets(seqlens, k)[b]
    idx = np.asarray(idx, dtype=np.int64)
    return (off + idx) * (k + 1) + k


def sample_rows(n, count, seed):
    """A deterministic spread of indices in [0, n): evenly spaced, plus the
    first and last rows and random picks."""
    if n <= count:
        return np.arange(n)
    rng = np.random.default_rng(seed)
    base = np.linspace(0, n - 1, count // 2).astype(np.int64)
    extra = rng.choice(n, count - len(base), replace=False)
    return np.unique(np.concatenate([base, extra, [0, n - 1]]))

"""Comparison helpers for GPU-vs-oracle parity (used by the -m gpu tests)."""

import numpy as np
import torch

# Tolerances (bf16 paths): rel_l2 <= 5e-3 and per-head cosine >= 0.99999 -- the
# decode page's per-head cosine criterion, and an L2 budget that bf16 rounding
# of P (~2^-9 relative per probability) and of the output sits well inside.
BF16_REL_L2 = 5e-3
BF16_HEAD_COS = 0.99999
# FP8-KV path: rel_l2 <= 3e-2 (K/V quantisation is in the stored cache, so the
# oracle reads the same values; the budget covers the kernel's own roundings).
FP8_REL_L2 = 3e-2


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").double().numpy()


def rel_l2(got: np.ndarray, ref: np.ndarray) -> float:
    den = np.linalg.norm(ref.ravel())
    return float(np.linalg.norm((got - ref).ravel()) / (den if den > 0 else 1.0))


def head_cosines(got: np.ndarray, ref: np.ndarray, head_axes: int) -> np.ndarray:
    """Cosine similarity per head: the leading `head_axes` axes index heads."""
    g = got.reshape(int(np.prod(got.shape[:head_axes])), -1)
    r = ref.reshape(g.shape)
    num = (g * r).sum(1)
    den = np.linalg.norm(g, axis=1) * np.linalg.norm(r, axis=1)
    out = np.ones(len(num))
    nz = den > 0
    out[nz] = num[nz] / den[nz]
    # an all-zero head on both sides counts as a match
    both0 = (np.linalg.norm(g, axis=1) == 0) & (np.linalg.norm(r, axis=1) == 0)
    out[both0] = 1.0
    return out


# Per output row (one query of one head: the last axis): relative L2 error. The bf16 roundings
# give ~2e-3 per row; 2e-2 leaves room for unlucky rows and still fails a row that is wrong
# (a misplaced ragged tail or a skipped key gives errors of order 1).
BF16_ROW_REL_L2 = 2e-2
FP8_ROW_REL_L2 = 6e-2


def worst_row(got: np.ndarray, ref: np.ndarray):
    """(max per-row relative L2 error, its row index); rows = every axis but the last. A row
    that is zero in the oracle (every key masked) must be exactly zero."""
    g = got.reshape(-1, got.shape[-1])
    r = ref.reshape(g.shape)
    num = np.linalg.norm(g - r, axis=1)
    den = np.linalg.norm(r, axis=1)
    err = np.where(den > 0, num / np.where(den > 0, den, 1.0), np.where(num > 0, np.inf, 0.0))
    i = int(np.argmax(err))
    return float(err[i]), i


def assert_rows_close(got: np.ndarray, ref: np.ndarray, bound: float, what: str = ""):
    e, i = worst_row(got, ref)
    assert e <= bound, f"{what}: row {i} rel_l2 {e:.3e} > {bound}"
    return e


def assert_bf16_parity(got_t: torch.Tensor, ref: np.ndarray, head_axes: int, what: str = ""):
    got = to_f64(got_t)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    e = rel_l2(got, ref)
    c = head_cosines(got, ref, head_axes).min()
    assert e <= BF16_REL_L2, f"{what}: rel_l2 {e:.3e} > {BF16_REL_L2}"
    assert c >= BF16_HEAD_COS, f"{what}: min per-head cosine {c:.7f} < {BF16_HEAD_COS}"
    assert_rows_close(got, ref, BF16_ROW_REL_L2, what)
    return e, c

"""Comparison helpers for GPU-vs-oracle parity tests.

Tolerances (bf16 inputs and output, unit-variance data):
  O    max-abs <= 2e-2 and mean-abs <= 2e-3 against the fp64 oracle;
  LSE  abs <= 1e-3 (finite rows), identical -inf on rows with no visited block;
  masks / skip bits: bit-exact except bits whose decision margin lies within
  1e-3 of the cut (flagged by the oracle); flagged mismatches are counted,
  printed and bounded (at most 0.1 % of the compared bits), not failed;
  gradients: relative to the reference's size (check_grad below).
"""
import numpy as np
import torch

from oracle.lite import skip_flags  # noqa: F401  (the skip bits' margin rule, for the parity tests)

O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_ABS = 1e-3


def as_np(t):
    if isinstance(t, torch.Tensor):
        return t.detach().float().cpu().numpy() if t.is_floating_point() else t.detach().cpu().numpy()
    return np.asarray(t)


def check_o(o_gpu, o_ref, what=""):
    g = as_np(o_gpu).astype(np.float64)
    r = np.asarray(o_ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    err = np.abs(g - r)
    assert err.max() <= O_MAX_ABS, f"{what}: O max-abs {err.max():.3e}"
    assert err.mean() <= O_MEAN_ABS, f"{what}: O mean-abs {err.mean():.3e}"
    return float(err.max()), float(err.mean())


def check_lse(l_gpu, l_ref, what=""):
    g = as_np(l_gpu).astype(np.float64)
    r = np.asarray(l_ref, dtype=np.float64)
    fin = np.isfinite(r)
    assert np.array_equal(np.isfinite(g), fin), f"{what}: -inf rows differ"
    assert np.all(g[~fin] == -np.inf)
    if fin.any():
        err = np.abs(g[fin] - r[fin]).max()
        assert err <= LSE_ABS, f"{what}: LSE abs {err:.3e}"


# Flagged mismatches allowed per comparison: a decision only flips between
# fp32 and fp64 when its margin is within rounding of the cut, so flagged
# bits that do differ must stay rare.  Bound: 0.1 % of the compared bits, and
# at least 2 (small masks with one near-tie).
FLAG_MAX_FRAC = 1e-3
FLAG_MIN_ALLOWED = 2


def check_bits(b_gpu, b_ref, flags=None, what="", max_frac=FLAG_MAX_FRAC):
    """Bit-exact compare; mismatches on flagged positions are counted, bounded
    and reported (printed), any other mismatch fails.  Returns the count."""
    g = as_np(b_gpu).astype(np.int64)
    r = np.asarray(b_ref).astype(np.int64)
    assert g.shape == r.shape, (g.shape, r.shape)
    bad = g != r
    if flags is None:
        assert not bad.any(), f"{what}: {int(bad.sum())} mismatches"
        return 0
    f = np.asarray(flags, dtype=bool)
    unflagged = bad & ~f
    assert not unflagged.any(), f"{what}: {int(unflagged.sum())} unflagged mismatches"
    n = int((bad & f).sum())
    allowed = max(FLAG_MIN_ALLOWED, int(max_frac * g.size))
    print(f"[flagged] {what}: {n} flagged mismatches of {g.size} bits ({int(f.sum())} flagged)")
    assert n <= allowed, f"{what}: {n} flagged mismatches, more than the {allowed} allowed"
    return n


# Gradients (attention backward): their scale shrinks like 1/sqrt(kept keys),
# so the bar is relative to the reference.  The kernel rounds P and dS to bf16
# for the MMAs (relative 2^-9 each), takes D_r from the bf16 forward output and
# rounds the result to bf16: about 0.5 % per element.  Bar: max-abs error
# <= 2e-2 x max |ref| and mean-abs error <= 1e-2 x mean |ref|.
GRAD_MAX_REL = 2e-2
GRAD_MEAN_REL = 1e-2


def check_grad(g_gpu, g_ref, what=""):
    g = as_np(g_gpu).astype(np.float64)
    r = np.asarray(g_ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite gradient"
    err = np.abs(g - r)
    ref_max, ref_mean = np.abs(r).max(), np.abs(r).mean()
    if ref_max == 0.0:
        assert err.max() == 0.0, f"{what}: nonzero where the gradient is zero"
        return 0.0, 0.0
    assert err.max() <= GRAD_MAX_REL * ref_max, f"{what}: max-abs {err.max():.3e} vs max|ref| {ref_max:.3e}"
    assert err.mean() <= GRAD_MEAN_REL * ref_mean, f"{what}: mean-abs {err.mean():.3e} vs mean|ref| {ref_mean:.3e}"
    return float(err.max() / ref_max), float(err.mean() / ref_mean)

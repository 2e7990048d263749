"""Shared test helpers: tensor conversion, oracle loops over heads, error metrics."""

from __future__ import annotations

import math

import numpy as np
import torch

import oracle as orc

MAX_ABS_TOL = 2e-2   # bf16 outputs vs the fp64 oracle (max |error|)
REL_FROB_TOL = 1e-2  # ||gpu - oracle||_F / ||oracle||_F


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()


def err(gpu: torch.Tensor, ref: np.ndarray, norm_ref=None):
    g = to64(gpu)
    d = g - ref
    nr = np.linalg.norm(ref if norm_ref is None else norm_ref)
    return float(np.abs(d).max()), float(np.linalg.norm(d) / max(nr, 1e-300))


def assert_close(gpu, ref, what="", norm_ref=None):
    """max-abs and relative Frobenius bars.  For the residual R, which tends to 0 as the
    density tends to 1, pass norm_ref=O_full: an error in R moves O_hat = O_s + R by the same
    amount, so it is measured against the output it corrects."""
    mx, rf = err(gpu, ref, norm_ref)
    assert mx <= MAX_ABS_TOL and rf <= REL_FROB_TOL, f"{what}: max-abs {mx:.3e}, rel-Frob {rf:.3e}"
    return mx, rf


def oracle_heads(fn, *arrays, **kw):
    """Run a per-head oracle function over [B, H, ...] arrays; stacks array results."""
    B, H = arrays[0].shape[:2]
    out = [[fn(*(a[b, h] for a in arrays), **kw) for h in range(H)] for b in range(B)]
    return out


def scale_of(d):
    return 1.0 / math.sqrt(d)


def oracle_anchor(Q, K, V, C, k):
    """fp64 anchor for every head: dict of stacked arrays."""
    q, kk, v = to64(Q), to64(K), to64(V)
    B, H, N, d = q.shape
    res = oracle_heads(lambda a, b, c: orc.anchor(a, b, c, C, k, scale_of(d)), q, kk, v)
    keys = res[0][0].keys()
    return {key: np.stack([np.stack([res[b][h][key] for h in range(H)]) for b in range(B)]) for key in keys}


def selection_band(q, kmat, perm, C, k, lse, scale):
    """Per group: oracle scores, the k-th largest score tau and a certified rounding band eps.

    The CUDA path computes logits with exact bf16 products accumulated in fp32 (error at most
    d * 2^-24 * sum_c |q_c k_c| in sequential order), gets LSE from the same fp32 logits,
    exponentiates in fp32 (relative error <= 2^-22) and sums C terms in fp32.  eps bounds the
    resulting difference from the fp64 score, with a factor-2 margin.
    """
    scores = orc.group_scores(q, kmat, perm, C, lse, scale)
    G = scores.shape[0]
    taus = np.empty(G)
    eps = np.empty(G)
    absk = np.abs(kmat)
    for g in range(G):
        rows = perm[g * C:(g + 1) * C]
        s = np.sort(scores[g])[::-1]
        taus[g] = s[k - 1]
        d = q.shape[1]
        dot_abs = (np.abs(q[rows]) @ absk.T).max() * scale
        delta = 2 * d * 2.0 ** -24 * dot_abs + 2.0 ** -20  # logit + LSE error (natural-log units)
        eps[g] = taus[g] * 2 * (delta + (C + 4) * 2.0 ** -22)
    return scores, taus, eps


def check_selection(gpu_idx: np.ndarray, scores, taus, eps, k):
    """Exact outside the band; returns the number of keys whose membership differs."""
    swaps = 0
    G = scores.shape[0]
    for g in range(G):
        sel = gpu_idx[g]
        assert len(sel) == k
        assert np.all(np.diff(sel) > 0), "indices must ascend"
        assert sel[0] >= 0 and sel[-1] < scores.shape[1]
        chosen = np.zeros(scores.shape[1], dtype=bool)
        chosen[sel] = True
        s = scores[g]
        must = s > taus[g] + eps[g]
        never = s < taus[g] - eps[g]
        assert np.all(chosen[must]), f"group {g}: a key clearly above the cut was dropped"
        assert not np.any(chosen[never]), f"group {g}: a key clearly below the cut was chosen"
        ref = orc.select_topk(s[None, :], k)[0]
        swaps += int(np.setdiff1d(sel, ref).size)
    return swaps

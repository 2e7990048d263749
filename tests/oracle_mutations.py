"""Plausible mistakes planted in the oracle (CPU, test infrastructure): each replaces one
oracle function with a subtly wrong version, so that tests/test_oracle_mutations.py can check
that the oracle's pins catch it.  Applied only when MCS_ORACLE_MUTATION names one of them."""

from __future__ import annotations

import numpy as np

import oracle
import oracle.mcs_oracle as mo


def _uncentered_split(q, members, m, C, iters=mo.POWER_ITERS):
    x = q[members]
    v = mo.principal_direction(x, iters)  # mistake: the node is not centred
    p = (x * v[None, :]).sum(axis=1)
    order = np.lexsort((members, p))
    n_left = (m // 2) * C
    return np.sort(members[order[:n_left]]), np.sort(members[order[n_left:]]), v, p


def _ceil_half_split(q, members, m, C, iters=mo.POWER_ITERS):
    x = q[members]
    xc = x - x.mean(axis=0)
    v = mo.principal_direction(xc, iters)
    p = (xc * v[None, :]).sum(axis=1)
    order = np.lexsort((members, p))
    n_left = ((m + 1) // 2) * C  # mistake: ceil instead of floor
    return np.sort(members[order[:n_left]]), np.sort(members[order[n_left:]]), v, p


def _flipped_sign(xc, iters=mo.POWER_ITERS):
    return -_ORIG["principal_direction"](xc, iters)  # mistake: largest component negative


def _no_lse_scores(q, k, perm, C, lse, scale):
    G = q.shape[0] // C
    out = np.empty((G, k.shape[0]))
    for g in range(G):
        rows = perm[g * C:(g + 1) * C]
        out[g] = np.exp(scale * (q[rows] @ k.T)).sum(axis=0)  # mistake: LSE not subtracted
    return out


def _reversed_ties(scores, k):
    out = np.empty((scores.shape[0], k), dtype=np.int64)
    n = scores.shape[1]
    for g in range(scores.shape[0]):
        order = n - 1 - np.argsort(-scores[g][::-1], kind="stable")  # mistake: ties to the higher key
        out[g] = np.sort(order[:k])
    return out


def _unsorted_topk(scores, k):
    out = np.empty((scores.shape[0], k), dtype=np.int64)
    for g in range(scores.shape[0]):
        out[g] = np.argsort(-scores[g], kind="stable")[:k]  # mistake: not emitted ascending
    return out


def _block_max(q, k, perm, C, BK, kb, lse, scale):
    s = mo.group_scores(q, k, perm, C, lse, scale)
    bs = s.reshape(s.shape[0], k.shape[0] // BK, BK).max(axis=2)  # mistake: max, not the block mass
    return mo.expand_blocks(mo.select_topk(bs, kb), BK), bs


def _bsa_first_key(q, k, perm, C, BK, kb):
    G = q.shape[0] // C
    qbar = np.stack([q[perm[g * C:(g + 1) * C]].mean(axis=0) for g in range(G)])
    kbar = k[::BK]  # mistake: the block's first key instead of its mean
    bs = qbar @ kbar.T
    return mo.expand_blocks(mo.select_topk(bs, kb), BK), bs


def _perquery_unrenormalised(q, k, v, kk, scale):
    out = np.empty((q.shape[0], v.shape[1]))
    for i in range(q.shape[0]):
        L = scale * (k @ q[i])
        cols = np.sort(np.argsort(-L, kind="stable")[:kk])
        e = np.exp(L - L.max())
        out[i] = (e[cols] @ v[cols]) / e.sum()  # mistake: normalised over all keys
    return out


_ORIG = {n: getattr(mo, n) for n in ("principal_direction", "split_node", "group_scores", "select_topk")}

MUTATIONS = {
    "uncentered_pddp": ("split_node", _uncentered_split),
    "ceil_half_split": ("split_node", _ceil_half_split),
    "flipped_sign": ("principal_direction", _flipped_sign),
    "missing_lse": ("group_scores", _no_lse_scores),
    "reversed_ties": ("select_topk", _reversed_ties),
    "unsorted_topk": ("select_topk", _unsorted_topk),
    "block_max": ("block_oracle_select", _block_max),
    "bsa_first_key": ("bsa_select", _bsa_first_key),
    "perquery_unrenormalised": ("perquery", _perquery_unrenormalised),
}

# the pin module each planted mistake is checked against
PINS = {name: "test_oracle.py" for name in MUTATIONS}
PINS.update({"block_max": "test_oracle_variants.py", "bsa_first_key": "test_oracle_variants.py",
             "perquery_unrenormalised": "test_oracle_variants.py"})


def apply(name: str):
    fn_name, fn = MUTATIONS[name]
    setattr(mo, fn_name, fn)       # callers inside the oracle module
    setattr(oracle, fn_name, fn)   # callers through the package

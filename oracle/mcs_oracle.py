"""Plain fp64 CPU oracle for MC-Sparse's token-sparse attention path.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports, links or runs this module:
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its ``cpu_baseline`` leg and
its ``--impl reference`` arm) may use it. It shares no code with the CUDA library.

Every function works on one attention head, with NumPy float64 arrays (bf16 inputs upcast
exactly), and follows a definition on the pages:

* "MC-Sparse가 확산 트랜스포머 희소 어텐션의 품질 격차를 좁힌다" (abbreviated P4 below),
  section 무엇과 다른가 ("How it differs"): anchor steps run dense attention, build query
  groups, select KV tokens by exact probabilities and record R = O_full - O_sparse; reuse
  steps compute O_t = SparseAttn(Q_t, K_t, V_t; G, S) + R.
* P4, section 어떻게 쓰나 ("How to use"): token-level KV selection gathered by index; equal-
  size query groups of exactly the kernel's query tile C, formed by median-split PDDP
  (project onto the principal direction, split recursively at the median); a two-pass
  exact selection because an online-softmax kernel exposes no logits.
* P4, section 어떻게 동작하나 ("How it works"): the token oracle shares one query block's
  selection across its queries and picks individual KV tokens by exact dense probabilities;
  the block oracle picks KV blocks per query block and the per-query oracle picks KV tokens
  per query, by the same probabilities; vanilla BSA scores blocks from mean-pooled queries
  and keys (section 무엇인가).

Readings where the pages are silent:

* group score of key j = sum over the group's queries of the exact softmax probability;
* top-k ties go to the lower key index; indices are stored ascending;
* k = floor(s * N) is passed in directly;
* PDDP: centered data; power iteration from v0 = 1/sqrt(d) for exactly T = 20 steps; if
  X_c^T X_c v is zero, v is kept; v's sign makes its largest-magnitude component (lowest
  index on a tie) positive; a node holding m groups sends its floor(m/2)*C smallest
  projections (ties to the lower query index) to the left child; leaves are numbered left to
  right and each leaf lists its queries in ascending index order;
* sparse attention renormalises over the selected set (the residual carries the tail);
* R is kept in fp64 here; the CUDA path stores it in bf16.

Parity pins for each function are in ``tests/test_oracle.py``; none is "parity unpinned".
"""

from __future__ import annotations

import numpy as np

POWER_ITERS = 20


def default_scale(d: int) -> float:
    return 1.0 / np.sqrt(d)


# ---------------------------------------------------------------------------------------
# Dense attention and the pass-1 statistic (P4, 무엇과 다른가: anchors run dense attention;
# 어떻게 쓰나: the first of the two selection passes computes softmax statistics).
# ---------------------------------------------------------------------------------------
def dense(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float, block: int = 512):
    """O = softmax(scale * q k^T) v and LSE_i = log sum_j exp(scale * q_i . k_j).

    q [N, d], k [Nk, d], v [Nk, dv] -> (O [N, dv], lse [N]).  Row blocks only bound memory.
    """
    N = q.shape[0]
    out = np.empty((N, v.shape[1]))
    lse = np.empty(N)
    for r0 in range(0, N, block):
        r1 = min(N, r0 + block)
        L = scale * (q[r0:r1] @ k.T)
        m = L.max(axis=1, keepdims=True)
        e = np.exp(L - m)
        s = e.sum(axis=1, keepdims=True)
        lse[r0:r1] = (m + np.log(s))[:, 0]
        out[r0:r1] = (e @ v) / s
    return out, lse


# ---------------------------------------------------------------------------------------
# Median-split PDDP (P4, 어떻게 쓰나).  Fast PDDP on the GPU batches this same recursion by
# tree depth, so the partition it must produce is the one defined here.
# ---------------------------------------------------------------------------------------
def principal_direction(xc: np.ndarray, iters: int = POWER_ITERS) -> np.ndarray:
    """Top principal direction of centered rows ``xc`` by power iteration, sign-fixed."""
    d = xc.shape[1]
    v = np.full(d, 1.0 / np.sqrt(d))
    for _ in range(iters):
        w = xc.T @ (xc @ v)
        nrm = np.sqrt(np.dot(w, w))
        if nrm == 0.0:
            break  # X_c^T X_c v = 0: v is kept (and stays kept)
        v = w / nrm
    j = int(np.argmax(np.abs(v)))  # first maximum: lowest index on a tie
    if v[j] < 0:
        v = -v
    return v


def split_node(q: np.ndarray, members: np.ndarray, m: int, C: int, iters: int = POWER_ITERS):
    """One median split of a node holding ``m`` groups (``members`` ascending query ids).

    Returns (left members, right members, v, projections), children ascending.
    """
    x = q[members]
    mu = x.mean(axis=0)
    xc = x - mu
    v = principal_direction(xc, iters)
    p = (xc * v[None, :]).sum(axis=1)  # row-independent, so equal rows give equal values
    order = np.lexsort((members, p))  # by projection, then by query index
    n_left = (m // 2) * C
    left = np.sort(members[order[:n_left]])
    right = np.sort(members[order[n_left:]])
    return left, right, v, p


def pddp_groups(q: np.ndarray, C: int, iters: int = POWER_ITERS) -> np.ndarray:
    """perm [N] int64: group g is perm[g*C:(g+1)*C] (ascending query ids)."""
    N = q.shape[0]
    if N % C:
        raise ValueError("N must be a multiple of C")
    leaves = []

    def rec(members, m):
        if m == 1:
            leaves.append(members)
            return
        left, right, _, _ = split_node(q, members, m, C, iters)
        rec(left, m // 2)
        rec(right, m - m // 2)

    rec(np.arange(N), N // C)
    return np.concatenate(leaves)


# ---------------------------------------------------------------------------------------
# Exact selection, pass 2 (P4, 어떻게 쓰나 and 어떻게 동작하나): exact probabilities
# P_ij = exp(scale * q_i . k_j - LSE_i), group score = sum over the group's queries.
# ---------------------------------------------------------------------------------------
def group_scores(q: np.ndarray, k: np.ndarray, perm: np.ndarray, C: int, lse: np.ndarray,
                 scale: float) -> np.ndarray:
    """scores [G, Nk]: score[g, j] = sum_{i in group g} exp(scale q_i . k_j - lse_i)."""
    G = q.shape[0] // C
    out = np.empty((G, k.shape[0]))
    for g in range(G):
        rows = perm[g * C:(g + 1) * C]
        L = scale * (q[rows] @ k.T)
        out[g] = np.exp(L - lse[rows][:, None]).sum(axis=0)
    return out


def select_topk(scores: np.ndarray, k: int) -> np.ndarray:
    """idx [G, k]: per row the k largest scores, ties to the lower key index, ascending."""
    out = np.empty((scores.shape[0], k), dtype=np.int64)
    for g in range(scores.shape[0]):
        order = np.argsort(-scores[g], kind="stable")  # stable: equal scores keep index order
        out[g] = np.sort(order[:k])
    return out


# ---------------------------------------------------------------------------------------
# Sparse attention over cached indices (P4, 무엇과 다른가 and 어떻게 쓰나).
# ---------------------------------------------------------------------------------------
def sparse(q, k, v, perm, idx, C: int, scale: float) -> np.ndarray:
    """O_s[i] for i in group g: softmax over idx[g] of scale q_i . k_j, times v_j."""
    out = np.empty((q.shape[0], v.shape[1]))
    for g in range(idx.shape[0]):
        rows = perm[g * C:(g + 1) * C]
        cols = idx[g]
        L = scale * (q[rows] @ k[cols].T)
        e = np.exp(L - L.max(axis=1, keepdims=True))
        out[rows] = (e @ v[cols]) / e.sum(axis=1, keepdims=True)
    return out


# ---------------------------------------------------------------------------------------
# Anchor and reuse steps (P4, 무엇과 다른가).
# ---------------------------------------------------------------------------------------
def anchor(q, k, v, C: int, kk: int, scale: float, iters: int = POWER_ITERS):
    """Returns dict(O_full, lse, perm, idx, O_sparse, R) for one head."""
    o_full, lse = dense(q, k, v, scale)
    perm = pddp_groups(q, C, iters)
    idx = select_topk(group_scores(q, k, perm, C, lse, scale), kk)
    o_s = sparse(q, k, v, perm, idx, C, scale)
    return dict(O_full=o_full, lse=lse, perm=perm, idx=idx, O_sparse=o_s, R=o_full - o_s)


def reuse(q, k, v, perm, idx, R, C: int, scale: float) -> np.ndarray:
    """O_hat = SparseAttn(q, k, v; perm, idx) + R."""
    return sparse(q, k, v, perm, idx, C, scale) + R


# ---------------------------------------------------------------------------------------
# Selection variants of the controlled oracle comparison (P4, 어떻게 동작하나: block oracle,
# token oracle, per-query oracle by exact dense probabilities, against vanilla BSA, which
# scores blocks from mean-pooled queries and keys; P4, 무엇인가).
# ---------------------------------------------------------------------------------------
def expand_blocks(blocks: np.ndarray, BK: int) -> np.ndarray:
    """[G, kb] ascending block ids -> [G, kb*BK] ascending key ids (whole blocks)."""
    return (blocks[:, :, None] * BK + np.arange(BK)[None, None, :]).reshape(blocks.shape[0], -1)


def block_oracle_select(q, k, perm, C: int, BK: int, kb: int, lse, scale: float):
    """Block oracle: block score = exact probability mass of the block summed over the group's
    queries; the kb largest blocks (ties to the lower block).  Returns (idx, block_scores)."""
    s = group_scores(q, k, perm, C, lse, scale)
    bs = s.reshape(s.shape[0], k.shape[0] // BK, BK).sum(axis=2)
    return expand_blocks(select_topk(bs, kb), BK), bs


def bsa_select(q, k, perm, C: int, BK: int, kb: int):
    """Vanilla BSA: block score = (mean of the group's queries) . (mean of the block's keys);
    the kb largest blocks (ties to the lower block).  Returns (idx, block_scores)."""
    G = q.shape[0] // C
    qbar = np.stack([q[perm[g * C:(g + 1) * C]].mean(axis=0) for g in range(G)])
    kbar = k.reshape(k.shape[0] // BK, BK, k.shape[1]).mean(axis=1)
    bs = qbar @ kbar.T
    return expand_blocks(select_topk(bs, kb), BK), bs


def perquery(q, k, v, kk: int, scale: float) -> np.ndarray:
    """Per-query oracle: each query's own kk keys of largest logit (ties to the lower key),
    softmax renormalised over them."""
    out = np.empty((q.shape[0], v.shape[1]))
    for i in range(q.shape[0]):
        L = scale * (k @ q[i])
        cols = np.sort(np.argsort(-L, kind="stable")[:kk])
        e = np.exp(L[cols] - L[cols].max())
        out[i] = (e @ v[cols]) / e.sum()
    return out


def kept_mass(q, k, perm, idx, C: int, lse, scale: float) -> float:
    """Mean over queries of the exact softmax probability mass on the selected keys."""
    tot = 0.0
    for g in range(idx.shape[0]):
        rows = perm[g * C:(g + 1) * C]
        L = scale * (q[rows] @ k[idx[g]].T)
        tot += np.exp(L - lse[rows][:, None]).sum()
    return tot / q.shape[0]


# ---------------------------------------------------------------------------------------
# Grouping-cost baseline (P4, 전제와 한계: Fast PDDP's grouping cost is set against a k-means
# clustering).  The pages name the comparison but give no algorithm for an equal-size
# k-means, so this is a reading: Lloyd's k-means on the queries, then one capacity-constrained
# assignment that gives every cluster exactly C queries.
#   * G = N / C centroids, initialised as the means of the contiguous query blocks
#     [g*C, (g+1)*C) (neighbouring tokens of the flattened grid);
#   * `iters` Lloyd steps: every query goes to its nearest centroid (squared Euclidean
#     distance, summed over the d coordinates in order; ties to the lower centroid), then
#     every centroid becomes the mean of its queries (summed in query order; an empty cluster
#     keeps its centroid);
#   * equal sizes: the clusters in order 0, 1, ..., G-1 each take the C not yet taken queries
#     nearest to their final centroid (ties to the lower query index).
# Group g of the output is cluster g's queries in ascending order.
# ---------------------------------------------------------------------------------------
KMEANS_ITERS = 10


def sq_distances(q: np.ndarray, cent: np.ndarray) -> np.ndarray:
    """dist [N, G]: sum over c = 0..d-1, in that order, of (q[i, c] - cent[g, c])^2, each term
    rounded before it is added."""
    dist = np.zeros((q.shape[0], cent.shape[0]))
    for c in range(q.shape[1]):
        diff = q[:, c][:, None] - cent[:, c][None, :]
        dist += diff * diff
    return dist


def kmeans_groups(q: np.ndarray, C: int, iters: int = KMEANS_ITERS) -> np.ndarray:
    """perm [N] int64: group g is perm[g*C:(g+1)*C] (ascending query ids)."""
    N, d = q.shape
    if N % C:
        raise ValueError("N must be a multiple of C")
    G = N // C
    cent = np.empty((G, d))
    for g in range(G):
        acc = np.zeros(d)
        for i in range(g * C, (g + 1) * C):  # query order
            acc += q[i]
        cent[g] = acc / C
    for _ in range(iters):
        assign = np.argmin(sq_distances(q, cent), axis=1)  # first minimum: the lower centroid
        for g in range(G):
            members = np.nonzero(assign == g)[0]
            if members.size:
                acc = np.zeros(d)
                for i in members:  # query order
                    acc += q[i]
                cent[g] = acc / members.size
    dist = sq_distances(q, cent)
    taken = np.zeros(N, dtype=bool)
    out = []
    for g in range(G):
        cand = np.nonzero(~taken)[0]
        order = np.lexsort((cand, dist[cand, g]))  # by distance, then by query index
        pick = np.sort(cand[order[:C]])
        taken[pick] = True
        out.append(pick)
    return np.concatenate(out)


# ---------------------------------------------------------------------------------------
# Helpers over [B, H, N, d] arrays.
# ---------------------------------------------------------------------------------------
def per_head(fn, *arrays, **kw):
    """Apply a per-head function over leading [B, H] axes; returns a list of results."""
    B, H = arrays[0].shape[:2]
    return [[fn(*(a[b, h] for a in arrays), **kw) for h in range(H)] for b in range(B)]

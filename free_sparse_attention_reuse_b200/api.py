"""Public Python API: thin wrappers over the C ABI (include/mcs.h), plus the anchor/reuse
schedule of MC-Sparse ("MC-Sparse가 확산 트랜스포머 희소 어텐션의 품질 격차를 좁힌다", section
무엇과 다른가: anchors are the last step of the dense warm-up or of a refresh interval; reuse
steps attend with the cached groups and indices and add the cached residual).

Tensors: Q, K, V bf16 [B, H, N, d] contiguous on a CUDA device; perm int32 [B, H, N];
idx int32 [B, H, N // C, k]; R bf16 [B, H, N, d].  Output tensors are allocated here with
torch when not given (the C library itself never allocates).
"""

from __future__ import annotations

from dataclasses import dataclass

import torch

from . import _lib
from ._lib import Shape, check, ptr, stream_ptr


def _shape(Q: torch.Tensor, scale=None) -> Shape:
    if Q.dim() != 4:
        raise ValueError("expected [B, H, N, d]")
    B, H, N, d = Q.shape
    return Shape(B, H, N, d, 0.0 if scale is None else float(scale))


def _spec(t, name: str, dtype, shape=None):
    """dtype, shape and layout of one tensor argument (where it lives is checked apart, so that
    a wrong shape is reported as such whatever the device)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _on_device(**tensors):
    """Every given tensor on the same CUDA device, the current one (the library launches there
    and the kernels dereference these pointers)."""
    dev = None
    for name, t in tensors.items():
        if t is None:
            continue
        if t.device.type != "cuda":
            raise ValueError(f"{name} must be a CUDA tensor")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{name} is on {t.device}, other arguments on {dev}")
    if dev is not None and dev.index != torch.cuda.current_device():
        raise ValueError(f"tensors are on {dev} but the current device is cuda:{torch.cuda.current_device()}")


def _req(t: torch.Tensor, dtype, name: str):
    _spec(t, name, dtype)
    _on_device(**{name: t})


def _qkv(Q, K, V=None, names=("Q", "K", "V")):
    """Q, K (and V) bf16 [B, H, N, d] of one shape; returns that shape."""
    if not isinstance(Q, torch.Tensor) or Q.dim() != 4:
        raise ValueError(f"{names[0]} must be a 4-d tensor [B, H, N, d]")
    shape = tuple(Q.shape)
    _spec(Q, names[0], torch.bfloat16, shape)
    _spec(K, names[1], torch.bfloat16, shape)
    if V is not None:
        _spec(V, names[2], torch.bfloat16, shape)
    return shape


def _groups(shape, C: int):
    """G = N // C, or None when C does not divide N (the library reports that as a shape error)."""
    N = shape[2]
    return N // C if isinstance(C, int) and C > 0 and N % C == 0 else None


def _meta(shape, C: int, perm=None, idx=None, R=None):
    """perm int32 [B, H, N], idx int32 [B, H, N // C, k], R bf16 like Q (each if given)."""
    B, H, N, _ = shape
    if perm is not None:
        _spec(perm, "perm", torch.int32, (B, H, N))
    G = _groups(shape, C)
    if idx is not None:
        if not isinstance(idx, torch.Tensor):
            raise TypeError("idx must be a torch.Tensor")
        if idx.dim() != 4 or (G is not None and tuple(idx.shape[:3]) != (B, H, G)):
            raise ValueError(f"idx must have shape {(B, H, G, 'k')}, got {tuple(idx.shape)}")
        _spec(idx, "idx", torch.int32)
    if R is not None:
        _spec(R, "R", torch.bfloat16, shape)


def workspace_size(Q: torch.Tensor, C: int, k: int, scale=None) -> int:
    return int(_lib.load().mcs_workspace_size(_shape(Q, scale), C, k))


def workspace(Q: torch.Tensor, C: int, k: int, scale=None) -> torch.Tensor:
    n = workspace_size(Q, C, k, scale)
    if n == 0:
        raise _lib.MCSError(2, "workspace_size: invalid shape")
    return torch.empty(n, dtype=torch.uint8, device=Q.device)


def dense_attn(Q, K, V, O=None, lse=None, want_out: bool = True, want_lse: bool = True, scale=None):
    """Dense attention; returns (O, lse).  want_out=False computes only the LSE; want_lse=False
    computes only O (lse is then None)."""
    B, H, N, d = shape = _qkv(Q, K, V)
    if want_out and O is None:
        O = torch.empty_like(Q)
    if want_lse and lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=Q.device)
    if not want_lse:
        lse = None
    if want_out:
        _spec(O, "O", torch.bfloat16, shape)
    if lse is not None:
        _spec(lse, "lse", torch.float32, (B, H, N))
    _on_device(Q=Q, K=K, V=V, O=O if want_out else None, lse=lse)
    check(_lib.load().mcs_dense_attn(_shape(Q, scale), ptr(Q), ptr(K), ptr(V), ptr(O if want_out else None),
                                     ptr(lse), stream_ptr()), "mcs_dense_attn")
    return O, lse


def group(Q, C: int, perm=None, ws=None, scale=None):
    """Fast PDDP grouping; returns perm int32 [B, H, N]."""
    if not isinstance(Q, torch.Tensor) or Q.dim() != 4:
        raise ValueError("Q must be a 4-d tensor [B, H, N, d]")
    _spec(Q, "Q", torch.bfloat16)
    B, H, N, d = shape = tuple(Q.shape)
    if perm is None:
        perm = torch.empty((B, H, N), dtype=torch.int32, device=Q.device)
    _meta(shape, C, perm=perm)
    _on_device(Q=Q, perm=perm)
    if ws is None:
        ws = workspace(Q, C, 1, scale)
    _spec(ws, "ws", torch.uint8)
    _on_device(Q=Q, ws=ws)
    check(_lib.load().mcs_group(_shape(Q, scale), ptr(Q), C, ptr(perm), ptr(ws), ws.numel(), stream_ptr()),
          "mcs_group")
    return perm


def select(Q, K, perm, C: int, k: int, lse=None, idx=None, ws=None, scale=None):
    """Exact two-pass top-k selection; returns idx int32 [B, H, N // C, k]."""
    B, H, N, d = shape = _qkv(Q, K)
    _meta(shape, C, perm=perm)
    if lse is not None:
        _spec(lse, "lse", torch.float32, (B, H, N))
    if idx is None:
        idx = torch.empty((B, H, N // C, k), dtype=torch.int32, device=Q.device)
    _meta(shape, C, idx=idx)
    if idx.shape[-1] != k:
        raise ValueError(f"idx must hold k = {k} indices per group, got {idx.shape[-1]}")
    _on_device(Q=Q, K=K, perm=perm, lse=lse, idx=idx)
    if ws is None:
        ws = workspace(Q, C, k, scale)
    _spec(ws, "ws", torch.uint8)
    _on_device(Q=Q, ws=ws)
    check(_lib.load().mcs_select(_shape(Q, scale), ptr(Q), ptr(K), ptr(perm), C, k, ptr(lse), ptr(idx), ptr(ws),
                                 ws.numel(), stream_ptr()), "mcs_select")
    return idx


def select_noalloc(Q, K, perm, C: int, k: int, lse, idx, scale=None):
    """mcs_select_noalloc: the same selection with no workspace and no device allocation in
    the library (its scratch is a fixed array inside libmcs.so); lse and idx must be given."""
    B, H, N, d = shape = _qkv(Q, K)
    _meta(shape, C, perm=perm, idx=idx)
    _spec(lse, "lse", torch.float32, (B, H, N))
    if idx.shape[-1] != k:
        raise ValueError(f"idx must hold k = {k} indices per group, got {idx.shape[-1]}")
    _on_device(Q=Q, K=K, perm=perm, lse=lse, idx=idx)
    check(_lib.load().mcs_select_noalloc(_shape(Q, scale), ptr(Q), ptr(K), ptr(perm), C, k, ptr(lse), ptr(idx),
                                         stream_ptr()), "mcs_select_noalloc")
    return idx


def sparse_attn(Q, K, V, perm, C: int, idx, R=None, out=None, scale=None):
    """Reuse step: SparseAttn(Q, K, V; perm, idx) + R."""
    shape = _qkv(Q, K, V)
    _meta(shape, C, perm=perm, idx=idx, R=R)
    k = idx.shape[-1]
    if out is None:
        out = torch.empty_like(Q)
    _spec(out, "out", torch.bfloat16, shape)
    _on_device(Q=Q, K=K, V=V, perm=perm, idx=idx, R=R, out=out)
    check(_lib.load().mcs_sparse_attn(_shape(Q, scale), ptr(Q), ptr(K), ptr(V), ptr(perm), C, ptr(idx), k, ptr(R),
                                      ptr(out), stream_ptr()), "mcs_sparse_attn")
    return out


def _req_host(t: torch.Tensor, name: str):
    if t.device.type != "cpu":
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if t.dtype != torch.bfloat16:
        raise ValueError(f"{name} must be torch.bfloat16")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def host_staging(shape, heads_per_chunk: int = 2, device=None) -> torch.Tensor:
    """Device staging buffer for sparse_attn_host on [B, H, N, d] tensors of `shape`."""
    B, H, N, d = shape
    n = int(_lib.load().mcs_host_staging_size(Shape(B, H, N, d, 0.0), heads_per_chunk))
    if n == 0:
        raise _lib.MCSError(2, "host_staging_size: invalid shape or heads_per_chunk")
    return torch.empty(n, dtype=torch.uint8, device="cuda" if device is None else device)


def sparse_attn_host(hQ, hK, hV, perm, C: int, idx, R=None, out=None, heads_per_chunk: int = 2, staging=None,
                     scale=None):
    """Reuse step with Q, K, V and the output in host memory (pinned for overlap) and the
    cached perm, idx and R on the device; chunks of heads are copied in, computed and copied
    out on overlapping streams.  Returns `out` (a host tensor); it is complete once the
    current CUDA stream is synchronised, and the host tensors must stay alive until then."""
    shape = _qkv(hQ, hK, hV, names=("hQ", "hK", "hV"))
    _meta(shape, C, perm=perm, idx=idx, R=R)
    if out is not None:
        _spec(out, "out", torch.bfloat16, shape)
    for t, n in ((hQ, "hQ"), (hK, "hK"), (hV, "hV"), (out, "out")):
        if t is not None:
            _req_host(t, n)
    _on_device(perm=perm, idx=idx, R=R)
    if out is None:
        out = torch.empty(shape, dtype=torch.bfloat16, pin_memory=True)
    if staging is None:
        staging = host_staging(shape, heads_per_chunk, perm.device)
    _spec(staging, "staging", torch.uint8)
    _on_device(perm=perm, staging=staging)
    k = idx.shape[-1]
    check(_lib.load().mcs_sparse_attn_host(_shape(hQ, scale), ptr(hQ), ptr(hK), ptr(hV), ptr(perm), C, ptr(idx), k,
                                           ptr(R), ptr(out), heads_per_chunk, ptr(staging), staging.numel(),
                                           stream_ptr()), "mcs_sparse_attn_host")
    return out


def residual(Q, K, V, perm, C: int, idx, O_full, R=None, scale=None):
    """Anchor residual record: R = O_full - SparseAttn(Q, K, V; perm, idx)."""
    shape = _qkv(Q, K, V)
    _meta(shape, C, perm=perm, idx=idx)
    _spec(O_full, "O_full", torch.bfloat16, shape)
    k = idx.shape[-1]
    if R is None:
        R = torch.empty_like(Q)
    _meta(shape, C, R=R)
    _on_device(Q=Q, K=K, V=V, perm=perm, idx=idx, O_full=O_full, R=R)
    check(_lib.load().mcs_residual(_shape(Q, scale), ptr(Q), ptr(K), ptr(V), ptr(perm), C, ptr(idx), k,
                                   ptr(O_full), ptr(R), stream_ptr()), "mcs_residual")
    return R


def anchor(Q, K, V, C: int, k: int, ws=None, out=None, scale=None):
    """Whole anchor step; returns (O_full, perm, idx, R)."""
    B, H, N, d = shape = _qkv(Q, K, V)
    if out is None:
        O_full = torch.empty_like(Q)
        perm = torch.empty((B, H, N), dtype=torch.int32, device=Q.device)
        idx = torch.empty((B, H, N // C, k), dtype=torch.int32, device=Q.device)
        R = torch.empty_like(Q)
    else:
        O_full, perm, idx, R = out
    _spec(O_full, "O_full", torch.bfloat16, shape)
    _meta(shape, C, perm=perm, idx=idx, R=R)
    if idx.shape[-1] != k:
        raise ValueError(f"idx must hold k = {k} indices per group, got {idx.shape[-1]}")
    _on_device(Q=Q, K=K, V=V, O_full=O_full, perm=perm, idx=idx, R=R)
    if ws is None:
        ws = workspace(Q, C, k, scale)
    _spec(ws, "ws", torch.uint8)
    _on_device(Q=Q, ws=ws)
    check(_lib.load().mcs_anchor(_shape(Q, scale), ptr(Q), ptr(K), ptr(V), C, k, ptr(O_full), ptr(perm), ptr(idx),
                                 ptr(R), ptr(ws), ws.numel(), stream_ptr()), "mcs_anchor")
    return O_full, perm, idx, R


def select_blocks(Q, K, perm, C: int, BK: int, kb: int, method: str = "oracle", lse=None, idx=None, ws=None,
                  scale=None):
    """KV-block selection per group as token indices [B, H, N//C, kb*BK] (kb whole blocks of BK
    keys, ascending).  method "oracle": exact probability mass of each block (summed group
    scores); "bsa": mean-pooled query against mean-pooled block keys (vanilla BSA)."""
    if method not in ("oracle", "bsa"):
        raise ValueError(f"method must be 'oracle' or 'bsa', got {method!r}")
    B, H, N, d = shape = _qkv(Q, K)
    _meta(shape, C, perm=perm)
    if lse is not None:
        _spec(lse, "lse", torch.float32, (B, H, N))
    if idx is None:
        idx = torch.empty((B, H, N // C, kb * BK), dtype=torch.int32, device=Q.device)
    _meta(shape, C, idx=idx)
    if idx.shape[-1] != kb * BK:
        raise ValueError(f"idx must hold kb*BK = {kb * BK} indices per group, got {idx.shape[-1]}")
    _on_device(Q=Q, K=K, perm=perm, lse=lse, idx=idx)
    if ws is None:
        ws = workspace(Q, C, kb * BK, scale)
    _spec(ws, "ws", torch.uint8)
    _on_device(Q=Q, ws=ws)
    m = {"oracle": 0, "bsa": 1}[method]
    check(_lib.load().mcs_select_blocks(_shape(Q, scale), ptr(Q), ptr(K), ptr(perm), C, BK, kb, m, ptr(lse),
                                        ptr(idx), ptr(ws), ws.numel(), stream_ptr()), "mcs_select_blocks")
    return idx


def perquery_attn(Q, K, V, k: int, out=None, ws=None, scale=None):
    """Per-query oracle: each query attends to its own k keys of largest logit (renormalised)."""
    shape = _qkv(Q, K, V)
    if out is None:
        out = torch.empty_like(Q)
    _spec(out, "out", torch.bfloat16, shape)
    _on_device(Q=Q, K=K, V=V, out=out)
    if ws is None:
        n = int(_lib.load().mcs_perquery_workspace_size(_shape(Q, scale)))
        if n == 0:
            raise _lib.MCSError(2, "mcs_perquery_workspace_size: invalid shape")
        ws = torch.empty(n, dtype=torch.uint8, device=Q.device)
    _spec(ws, "ws", torch.uint8)
    _on_device(Q=Q, ws=ws)
    check(_lib.load().mcs_perquery_attn(_shape(Q, scale), ptr(Q), ptr(K), ptr(V), k, ptr(out), ptr(ws), ws.numel(),
                                        stream_ptr()), "mcs_perquery_attn")
    return out


def group_kmeans(Q, C: int, iters: int = 10, perm=None, ws=None, scale=None):
    """Grouping-cost baseline: equal-size groups from Lloyd's k-means (fp64); returns perm int32
    [B, H, N] laid out as group() lays it out."""
    if not isinstance(Q, torch.Tensor) or Q.dim() != 4:
        raise ValueError("Q must be a 4-d tensor [B, H, N, d]")
    _spec(Q, "Q", torch.bfloat16)
    B, H, N, d = shape = tuple(Q.shape)
    if perm is None:
        perm = torch.empty((B, H, N), dtype=torch.int32, device=Q.device)
    _meta(shape, C, perm=perm)
    _on_device(Q=Q, perm=perm)
    if ws is None:
        n = int(_lib.load().mcs_kmeans_workspace_size(_shape(Q, scale), C))
        if n == 0:
            raise _lib.MCSError(2, "mcs_kmeans_workspace_size: invalid shape")
        ws = torch.empty(n, dtype=torch.uint8, device=Q.device)
    _spec(ws, "ws", torch.uint8)
    _on_device(Q=Q, ws=ws)
    check(_lib.load().mcs_group_kmeans(_shape(Q, scale), ptr(Q), C, iters, ptr(perm), ptr(ws), ws.numel(),
                                       stream_ptr()), "mcs_group_kmeans")
    return perm


def head_shard(n_heads: int, rank: int, world: int):
    """[lo, hi): the contiguous share of a layer's B*H heads that rank `rank` of `world`
    processes.  Every step of the path (grouping, selection, dense and sparse attention, the
    residual) works head by head, so a layer splits across GPUs by heads with no exchange; the
    first n_heads % world ranks take one head more."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    base, extra = divmod(n_heads, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def sync_status():
    """Synchronise the current stream and raise if a kernel reported an error."""
    check(_lib.load().mcs_sync_status(stream_ptr()), "mcs_sync_status")


@dataclass
class Metadata:
    """The per-layer metadata cache: query groups, KV indices and the dense-sparse residual."""

    perm: torch.Tensor
    idx: torch.Tensor
    R: torch.Tensor


class Schedule:
    """Anchor/reuse schedule for one attention layer.

    Steps 0..warmup-2 run dense attention; step warmup-1 and every `period` steps after it are
    anchors (dense output, fresh metadata); all other steps reuse the cached metadata.
    """

    def __init__(self, C: int, k: int, warmup: int = 5, period: int = 10, scale=None):
        self.C, self.k, self.warmup, self.period, self.scale = C, k, warmup, period, scale
        self.meta: Metadata | None = None
        self.ws: torch.Tensor | None = None

    def kind(self, step: int) -> str:
        if step < self.warmup - 1:
            return "dense"
        if (step - (self.warmup - 1)) % self.period == 0:
            return "anchor"
        return "reuse"

    def __call__(self, step: int, Q, K, V):
        kind = self.kind(step)
        if kind == "dense":
            return dense_attn(Q, K, V, want_lse=False, scale=self.scale)[0]
        if kind == "anchor":
            if self.ws is None:
                self.ws = workspace(Q, self.C, self.k, self.scale)
            if self.meta is None:
                out = None
            else:
                out = (torch.empty_like(Q), self.meta.perm, self.meta.idx, self.meta.R)
            O_full, perm, idx, R = anchor(Q, K, V, self.C, self.k, ws=self.ws, out=out, scale=self.scale)
            self.meta = Metadata(perm, idx, R)
            return O_full
        return sparse_attn(Q, K, V, self.meta.perm, self.C, self.meta.idx, R=self.meta.R, scale=self.scale)

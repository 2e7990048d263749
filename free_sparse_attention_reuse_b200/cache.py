"""Multi-layer anchor/reuse schedule with a bounded device-resident metadata cache.

"MC-Sparse가 확산 트랜스포머 희소 어텐션의 품질 격차를 좁힌다", section 어떻게 쓰나: when GPU memory
is short, inactive cache entries (a layer's query groups, KV indices and residual) are
offloaded to CPU memory and prefetched one layer ahead; section 전제와 한계 lists CPU offloading
and prefetch as a premise in that situation.

Two parts:

* `plan()` — pure Python, no device: walks the layer invocations of a denoising run in order
  (step t, layer l for l = 0..L-1, then t+1) and decides, for every invocation that uses
  metadata (anchor or reuse), which device slot holds that layer's metadata, whether the slot
  must be loaded from host memory (a reuse whose metadata is not in the slot) and whether the
  slot is written back to host memory after the invocation (an anchor, which produces new
  metadata).  Slots are assigned round-robin, so with two slots the next invocation's slot is
  never the current one's and its load can run while the current invocation computes.
* `LayeredSchedule` — executes that plan on one CUDA device: per-slot device tensors, pinned
  host copies of every layer's metadata, one side stream for the host<->device copies and
  events between the streams.  The prefetch of invocation i+1 is enqueued before invocation
  i's kernels; a slot is reloaded only after the kernels that last read it have finished, and
  an anchor's write-back is ordered before any later load into its slot (same copy stream).
  With `device_slots=None` every layer keeps its own device metadata and nothing is copied;
  the outputs of the two modes are bit-identical (the same kernels on the same data).
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, List, Optional

import torch

from .api import Metadata, anchor, dense_attn, sparse_attn, workspace


def schedule_kind(step: int, warmup: int = 5, period: int = 10) -> str:
    """'dense' for the warm-up steps before the first anchor, 'anchor' at the last warm-up step
    and every `period` steps after it, else 'reuse' (the single-layer Schedule's rule)."""
    if step < warmup - 1:
        return "dense"
    if (step - (warmup - 1)) % period == 0:
        return "anchor"
    return "reuse"


@dataclass
class Action:
    """What one layer invocation does with the metadata cache."""

    step: int
    layer: int
    kind: str               # dense | anchor | reuse
    slot: int = -1          # device slot (metadata-using invocations), -1 for dense
    load: bool = False      # copy the layer's metadata host -> slot before computing
    writeback: bool = False  # copy slot -> host after computing (a new anchor version)
    version: int = -1       # anchor version of the layer's metadata this invocation uses or writes


def plan(num_steps: int, layers: int, kind: Callable[[int], str], slots: int) -> List[Action]:
    """The cache actions of `num_steps` steps of a `layers`-layer model with `slots` device
    slots (slots >= 2).  Raises ValueError if a layer reuses metadata before its first anchor."""
    if slots < 2:
        raise ValueError("need at least two device slots (one computing, one loading)")
    acts: List[Action] = []
    content = [(-1, -1)] * slots          # (layer, version) held by each slot
    version = [-1] * layers               # latest anchor version per layer
    rr = 0                                # round-robin slot counter over metadata invocations
    for t in range(num_steps):
        kd = kind(t)
        for l in range(layers):
            if kd == "dense":
                acts.append(Action(t, l, kd))
                continue
            s = rr % slots
            rr += 1
            if kd == "anchor":
                version[l] += 1
                content[s] = (l, version[l])
                acts.append(Action(t, l, kd, slot=s, writeback=True, version=version[l]))
            else:
                if version[l] < 0:
                    raise ValueError(f"layer {l} reuses metadata at step {t} before any anchor")
                need = (l, version[l])
                load = content[s] != need
                content[s] = need
                acts.append(Action(t, l, kd, slot=s, load=load, version=version[l]))
    return acts


class LayeredSchedule:
    """The anchor/reuse schedule of an `layers`-layer model on one device.

    Call `sched(step, layer, Q, K, V)` for every layer of every step in order (layer 0..L-1 of
    step t, then step t+1, for `num_steps` steps); it returns the layer's attention output.
    `device_slots=None` keeps every layer's metadata on the device; an integer >= 2 bounds the
    device-resident metadata to that many layers and keeps the rest in pinned host memory.
    """

    def __init__(self, layers: int, shape, C: int, k: int, num_steps: int = 50, warmup: int = 5,
                 period: int = 10, device_slots: Optional[int] = None, device=None, scale=None):
        B, H, N, d = shape
        if N % C:
            raise ValueError("N must be a multiple of C")
        self.L, self.C, self.k, self.scale = layers, C, k, scale
        self.warmup, self.period = warmup, period
        self.device = torch.device("cuda") if device is None else torch.device(device)
        self.shape = (B, H, N, d)
        self.offload = device_slots is not None and device_slots < layers
        nslots = device_slots if self.offload else layers

        def meta(dev, pin=False):
            kw = dict(device=dev, pin_memory=pin) if pin else dict(device=dev)
            return Metadata(torch.empty((B, H, N), dtype=torch.int32, **kw),
                            torch.empty((B, H, N // C, k), dtype=torch.int32, **kw),
                            torch.empty((B, H, N, d), dtype=torch.bfloat16, **kw))

        self.slots = [meta(self.device) for _ in range(nslots)]
        self.host = [meta("cpu", pin=True) for _ in range(layers)] if self.offload else None
        self.ws = None
        self.num_steps = num_steps
        if self.offload:
            self.copy_stream = torch.cuda.Stream(device=self.device)
            self.loaded = [None] * nslots   # event: last load into the slot done (copy stream)
            self.freed = [None] * nslots    # event: last kernels reading/writing the slot done
            self.written = [None] * nslots  # event: last write-back out of the slot done (copy stream)
            self.plan = plan(num_steps, layers, self.kind, nslots)
            self._issued = set()            # invocations whose load is already enqueued
        self.bytes_h2d = 0
        self.bytes_d2h = 0

    def kind(self, step: int) -> str:
        return schedule_kind(step, self.warmup, self.period)

    def _action(self, i: int) -> Optional[Action]:
        return self.plan[i] if i < len(self.plan) else None

    @staticmethod
    def _bytes(m: Metadata) -> int:
        return sum(t.numel() * t.element_size() for t in (m.perm, m.idx, m.R))

    def _load(self, i: int, a: Action):
        """Enqueue the host -> slot copy of invocation i (action a) on the copy stream."""
        s = a.slot
        self._issued.add(i)
        with torch.cuda.stream(self.copy_stream):
            if self.freed[s] is not None:
                self.copy_stream.wait_event(self.freed[s])
            dst, src = self.slots[s], self.host[a.layer]
            for dt, st in ((dst.perm, src.perm), (dst.idx, src.idx), (dst.R, src.R)):
                dt.copy_(st, non_blocking=True)
            ev = torch.cuda.Event()
            ev.record(self.copy_stream)
            self.loaded[s] = ev
        self.bytes_h2d += self._bytes(self.slots[s])

    def __call__(self, step: int, layer: int, Q, K, V):
        kd = self.kind(step)
        if kd == "dense":
            return dense_attn(Q, K, V, want_lse=False, scale=self.scale)[0]
        cs = torch.cuda.current_stream(self.device)
        if not self.offload:
            m = self.slots[layer]
        else:
            i = step * self.L + layer
            a = self._action(i)
            if a is None or a.step != step or a.layer != layer:
                raise ValueError("invocations must come in (step, layer) order within num_steps")
            if a.load and i not in self._issued:
                self._load(i, a)  # not prefetched (the first use)
            # prefetch one invocation ahead, into another slot, while this one computes
            nxt = self._action(i + 1)
            if nxt is not None and nxt.load and i + 1 not in self._issued:
                self._load(i + 1, nxt)
            m = self.slots[a.slot]
            if a.load:
                cs.wait_event(self.loaded[a.slot])
            else:
                # an anchor overwrites the slot: the copies still reading it must be done
                if self.loaded[a.slot] is not None:
                    cs.wait_event(self.loaded[a.slot])
                if self.written[a.slot] is not None:
                    cs.wait_event(self.written[a.slot])
        if kd == "anchor":
            if self.ws is None:
                self.ws = workspace(Q, self.C, self.k, self.scale)
            O = anchor(Q, K, V, self.C, self.k, ws=self.ws, out=(torch.empty_like(Q), m.perm, m.idx, m.R),
                       scale=self.scale)[0]
        else:
            O = sparse_attn(Q, K, V, m.perm, self.C, m.idx, R=m.R, scale=self.scale)
        if self.offload:
            ev = torch.cuda.Event()
            ev.record(cs)
            self.freed[a.slot] = ev
            if a.writeback:
                with torch.cuda.stream(self.copy_stream):
                    self.copy_stream.wait_event(ev)
                    h = self.host[layer]
                    for ht, dt in ((h.perm, m.perm), (h.idx, m.idx), (h.R, m.R)):
                        ht.copy_(dt, non_blocking=True)
                    wb = torch.cuda.Event()
                    wb.record(self.copy_stream)
                    self.written[a.slot] = wb
                self.bytes_d2h += self._bytes(m)
        return O

    def synchronize(self):
        torch.cuda.synchronize(self.device)

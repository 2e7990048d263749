"""Benchmark of the MC-Sparse hot path on B200: reuse-step ms/layer and % of the ideal
1/density speedup over the library's own dense attention.

A step is one pass of the whole path on one attention layer (default: the 480p-shaped layer,
B=1, H=24, N=32256, d=128, C=128, density 0.15, k=4838): the anchor (dense attention + LSE,
Fast PDDP grouping, two-pass selection, residual record) followed by 9 reuse steps, each on
freshly perturbed Q, K, V.  Every kernel is called through the C ABI.

Output: one JSON line per measured (config, density) on rank 0 (one line by default).
`value` is the reuse step's mean device time per attention layer (max over ranks, divided by
the number of GPUs, since every rank processes its own layer).  Besides the timed steps the
line carries the dense baseline, a timed 50-step anchor/reuse schedule, the end-to-end call
with host buffers and the fp64 oracle's time for the same reuse step on the host cores.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mcs|reference]
                       [--config 480p|720p|3d|sweep|tiny] [--density s | --sweep]
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from free_sparse_attention_reuse_b200 import api, workload  # noqa: E402

REUSE_PER_STEP = 9
E2E_HEADS_PER_CHUNK = 2  # heads per host<->device chunk of the end-to-end measurement
METRIC = "reuse-step ms/layer & % of ideal 1/density speedup vs own dense attn @15%"


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, path=None):
        import tempfile
        self.gpu = gpu_index
        self.proc = None
        self.path = path or os.path.join(tempfile.gettempdir(), f"mcs_clocks_gpu{gpu_index}.csv")

    def start(self):
        try:
            if os.path.dirname(self.path):
                os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        # the timed region starts once the sampler is producing (its start-up takes a while)
        t0 = time.time()
        while time.time() - t0 < 3.0 and self.proc.poll() is None and os.path.getsize(self.path) == 0:
            time.sleep(0.02)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, smax, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                clk, mx, pw = float(parts[1]), float(parts[2]), float(parts[3])
            except ValueError:
                continue
            smax = max(smax, mx)
            if pw > 200:  # under load
                sm.append(clk)
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax or None, "reasons": sorted(reasons), "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def measured_traffic(name="480p", k=4838):
    """Bytes per launch of the reuse kernel from the committed ncu summary of this workload and
    k, if that capture was taken on the kernel sources as they are now (else None)."""
    import hashlib
    import re
    try:
        text = open(os.path.join(ROOT, "profiles", f"attn_kernel_{name}.md")).read()
        csrc = os.path.join(ROOT, "free_sparse_attention_reuse_b200", "csrc")
        src = b"".join(open(os.path.join(csrc, f), "rb").read() for f in ("attn.cuh", "sm100.cuh"))
    except OSError:
        return None
    sha = re.search(r"`([0-9a-f]{64})`", text)
    val = re.search(r"traffic_bytes_per_launch \(reuse\): (\d+)", text)
    kk = re.search(r"k=(\d+)\)", text.splitlines()[0])
    if not sha or not val or not kk or int(kk.group(1)) != k or sha.group(1) != hashlib.sha256(src).hexdigest():
        return None
    return int(val.group(1))


def max_over_ranks(values, dist=None, device=None):
    """Element-wise maximum of a list of floats over all ranks (identity without a group)."""
    if dist is None:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_reuse_heads(q, kk, v, perm, idx, R, C, heads, seconds_cap):
    """Time the fp64 oracle's reuse step (sparse attention + residual) head by head on the host
    cores.  q, kk, v, R: [H, N, d] tensors (any dtype; each head is upcast to fp64 outside the
    timed region); perm [H, N], idx [H, G, k] integer arrays.  Stops after `seconds_cap` of
    oracle time; returns (seconds per head, heads done)."""
    import numpy as np

    import oracle as orc

    d = q.shape[-1]
    scale = 1.0 / np.sqrt(d)
    f64 = lambda t: t.double().numpy() if isinstance(t, torch.Tensor) else np.asarray(t, dtype=np.float64)  # noqa: E731
    spent, done = 0.0, 0
    for h in heads:
        a, b, c, r = f64(q[h]), f64(kk[h]), f64(v[h]), f64(R[h])
        p_h, i_h = np.asarray(perm[h]), np.asarray(idx[h])
        t0 = time.perf_counter()
        orc.reuse(a, b, c, p_h, i_h, r, C, scale)
        spent += time.perf_counter() - t0
        done += 1
        if spent > seconds_cap:
            break
    return spent / done, done


def run_reference(args, wl, k):
    """The reference arm: the fp64 oracle (the only reference this method has: the pages carry
    no code) timed on the host cores.  Each step is a bounded sample of the workload, the reuse
    step of one head (heads in turn), with contiguous query groups and random ascending index
    sets (the oracle's cost does not depend on which keys are chosen).  `ms_per_step` is the
    measured time of one such step; `value` scales it to the whole layer (x B*H)."""
    import numpy as np

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    Q, K, V = workload.Generator(wl).current()
    B, H, N, d, C = wl.B, wl.H, wl.N, wl.d, wl.C
    q, kk, v = (t.reshape(B * H, N, d) for t in (Q, K, V))
    rng = np.random.default_rng(0)
    perm = np.tile(np.arange(N), (B * H, 1))
    idx = np.stack([np.sort(rng.choice(N, k, replace=False)) for _ in range(N // C)])[None].repeat(B * H, 0)
    R = torch.zeros((B * H, N, d), dtype=torch.bfloat16)
    step_s = []
    for s in range(args.steps + args.warmup):
        h = s % (B * H)
        sec, _ = oracle_reuse_heads(q, kk, v, perm, idx, R, C, [h], seconds_cap=1e9)
        if s >= args.warmup:
            step_s.append(sec)
    ms_step = 1000.0 * statistics.mean(step_s)
    value = ms_step * B * H
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "ms/layer", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded DiT-shaped generator, host)",
        "config": {"workload": f"{wl.name}: B={B} H={H} N={N} d={d} C={C} s={args.density} k={k}",
                   "global_batch": B, "seq_len": N, "parallelism": "replicas"},
        "cpu_baseline": {"value": value, "unit": "ms/layer", "cores": cpu_cores(), "kind": "oracle",
                         "sample": f"each step: the fp64 NumPy oracle's reuse step on 1 of {B * H} heads "
                                   f"(heads in turn), measured {ms_step:.1f} ms per step; value = that x {B * H}"},
        "e2e": {"value": value, "unit": "ms/layer", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_layers(args, wl, k, steps=50):
    """The 50-step anchor/reuse schedule (dense warm-up 0-3, anchors at 4, 14, 24, 34, 44) of
    `args.layers` layers on one GPU, all metadata resident vs at most `args.device_slots` layers
    resident (the rest in pinned host memory, prefetched one invocation ahead).  One JSON line:
    value = amortized ms per layer-step with offloading."""
    from free_sparse_attention_reuse_b200.cache import LayeredSchedule

    torch.cuda.set_device(0)
    L = args.layers
    B, H, N, d, C = wl.B, wl.H, wl.N, wl.d, wl.C
    gens = [workload.Generator(workload.custom(f"{wl.name}-layer{l}", B, H, d, wl.grid, C, index=40 + l),
                               device="cuda") for l in range(L)]
    inputs = [g.current() for g in gens]  # fixed per layer: the kernels recompute every call
    results = {}
    for mode, slots in (("resident", None), ("offload", args.device_slots)):
        sched = LayeredSchedule(L, (B, H, N, d), C, k, num_steps=steps, device_slots=slots)
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record()
        for t in range(steps):
            for l in range(L):
                sched(t, l, *inputs[l])
        t1.record()
        torch.cuda.synchronize()
        api.sync_status()
        ms = t0.elapsed_time(t1)
        results[mode] = {"ms_total": ms, "ms_per_layer_step": ms / (steps * L),
                         "h2d_bytes": sched.bytes_h2d, "d2h_bytes": sched.bytes_d2h}
        del sched
        torch.cuda.empty_cache()
    off, res = results["offload"], results["resident"]
    copy_bytes = off["h2d_bytes"] + off["d2h_bytes"]
    line = {
        "metric": f"schedule ms per layer-step ({L} layers, {steps} steps, {args.device_slots} device slots)",
        "value": off["ms_per_layer_step"], "unit": "ms/layer-step", "n_gpus": 1, "steps": steps, "warmup": 0,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded DiT-shaped generator, on device)",
        "config": {"workload": f"{wl.name}: B={B} H={H} N={N} d={d} C={C} s={args.density} k={k}; {L} layers",
                   "metadata_bytes_per_layer": (B * H * N * 4 + B * H * (N // C) * k * 4 + B * H * N * d * 2)},
        "resident": res, "offload": off,
        "offload_overhead": off["ms_total"] / res["ms_total"] - 1.0,
        "copy_gbs": copy_bytes / (off["ms_total"] * 1e-3) / 1e9,
    }
    print(json.dumps(line), flush=True)


def run_study(args, wl, k):
    """Error decomposition at equal attention density on the GPU ("MC-Sparse가 확산 트랜스포머 희소
    어텐션의 품질 격차를 좁힌다", section 어떻게 동작하나: block oracle, token oracle and per-query
    oracle by exact probabilities against mean-pooled vanilla BSA): relative Frobenius error of
    each variant's output against dense attention on the same inputs, and the reuse setting
    (metadata of this step applied to the next denoising step, with and without the residual).
    One JSON line; value = the MC-Sparse reuse-step error."""
    torch.cuda.set_device(0)
    B, H, N, d, C = wl.B, wl.H, wl.N, wl.d, wl.C
    BK = C
    kb = max(1, k // BK)
    kt = kb * BK  # the same number of keys per query for every variant
    gen = workload.Generator(wl, device="cuda")
    Q, K, V = gen.current()
    Q2, K2, V2 = gen.advance()
    O_full, lse = api.dense_attn(Q, K, V)
    ident = torch.arange(N, dtype=torch.int32, device="cuda").repeat(B, H, 1).contiguous()

    def rel(a, b):
        return float(((a.float() - b.float()).norm() / b.float().norm()).item())

    def timed(fn):
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        r = fn()
        t1.record()
        torch.cuda.synchronize()
        return r, t0.elapsed_time(t1)

    perm, _ = timed(lambda: api.group(Q, C))
    out = {}
    sel = {
        "block_oracle": lambda: api.select_blocks(Q, K, ident, C, BK, kb, "oracle", lse=lse),
        "bsa_mean_pooled": lambda: api.select_blocks(Q, K, ident, C, BK, kb, "bsa"),
        "token_oracle_contiguous": lambda: api.select(Q, K, ident, C, kt, lse=lse),
        "token_oracle_pddp_groups": lambda: api.select(Q, K, perm, C, kt, lse=lse),
    }
    idx_mcs = None
    for name, fn in sel.items():
        idx, ms = timed(fn)
        p = perm if name == "token_oracle_pddp_groups" else ident
        O = api.sparse_attn(Q, K, V, p, C, idx)
        out[name] = {"rel_frob_err": rel(O, O_full), "select_ms": ms}
        if name == "token_oracle_pddp_groups":
            idx_mcs, O_mcs = idx, O
    Opq, ms = timed(lambda: api.perquery_attn(Q, K, V, kt))
    out["per_query_oracle"] = {"rel_frob_err": rel(Opq, O_full), "ms": ms}
    # reuse setting: this step's metadata on the next step's inputs
    R = (O_full.float() - O_mcs.float()).to(torch.bfloat16)
    O_full2, _ = api.dense_attn(Q2, K2, V2, want_lse=False)
    no_res = api.sparse_attn(Q2, K2, V2, perm, C, idx_mcs)
    with_res = api.sparse_attn(Q2, K2, V2, perm, C, idx_mcs, R=R)
    api.sync_status()
    reuse = {"without_residual": rel(no_res, O_full2), "with_residual": rel(with_res, O_full2)}
    line = {
        "metric": "relative Frobenius error vs dense attention at equal density (MC-Sparse reuse step)",
        "value": reuse["with_residual"], "unit": "ratio", "n_gpus": 1, "steps": 1, "warmup": 0,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded DiT-shaped generator, on device)",
        "config": {"workload": f"{wl.name}: B={B} H={H} N={N} d={d} C={C} BK={BK} keys/query={kt} "
                               f"(s={kt / N:.4f})"},
        "variants": out, "reuse_next_step": reuse,
    }
    print(json.dumps(line), flush=True)


def run_kmeans(args, wl):
    """Grouping cost: Fast PDDP (mcs_group) against the equal-size k-means baseline
    (mcs_group_kmeans, 10 Lloyd steps) on the same queries; one JSON line, value = the Fast
    PDDP time, with the k-means time and their ratio."""
    torch.cuda.set_device(0)
    gen = workload.Generator(wl, device="cuda")
    Q, _, _ = gen.current()
    del gen
    C = wl.C
    ws = api.workspace(Q, C, 1)
    perm = torch.empty(Q.shape[:3], dtype=torch.int32, device="cuda")
    kws = torch.empty(int(api._lib.load().mcs_kmeans_workspace_size(api._shape(Q), C)), dtype=torch.uint8,
                      device="cuda")

    def timed(fn, n):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        evs = []
        for _ in range(n):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            evs.append((a, b))
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(b) for a, b in evs)

    pddp = timed(lambda: api.group(Q, C, perm=perm, ws=ws), args.steps)
    km = timed(lambda: api.group_kmeans(Q, C, 10, perm=perm, ws=kws), max(1, args.steps // 2))
    api.sync_status()
    B, H, N, d = Q.shape
    print(json.dumps({
        "metric": "grouping ms/layer: Fast PDDP against the equal-size k-means baseline (10 Lloyd steps)",
        "value": pddp, "unit": "ms/layer", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded DiT-shaped generator, on device)",
        "config": {"workload": f"{wl.name}: B={B} H={H} N={N} d={d} C={C}"},
        "kmeans_ms": km, "kmeans_over_pddp": km / pddp,
    }), flush=True)


def launches_per_step(N, C, n_reuse):
    """Kernels one bench step launches: dense (1), grouping (1 + 4 per tree level), selection
    (1), residual (1), reuse (1 each)."""
    return 1 + (1 + 4 * max(0, (N // C - 1).bit_length())) + 1 + 1 + n_reuse


def timed_schedule(steps_qkv, C, k, num_steps=50):
    """The 50-step anchor/reuse schedule of one layer (dense warm-up steps 0-3, anchors at 4,
    14, 24, 34, 44, reuse on the other 41 steps; step t attends over the t-th perturbed inputs,
    cycling through the resident copies), run once to warm up and once timed with a CUDA event
    per step.  Returns per-step kinds and milliseconds."""
    sched = api.Schedule(C, k)
    n = len(steps_qkv)
    for _ in range(2):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(num_steps + 1)]
        evs[0].record()
        for t in range(num_steps):
            sched(t, *steps_qkv[t % n])
            evs[t + 1].record()
        torch.cuda.synchronize()
    api.sync_status()
    kinds = [sched.kind(t) for t in range(num_steps)]
    ms = [evs[t].elapsed_time(evs[t + 1]) for t in range(num_steps)]
    return kinds, ms


def measure(args, wl, density, steps_qkv, ctx):
    """Time K steps (anchor + reuse steps) of `density` on the resident inputs, then the dense
    baseline, the 50-step schedule, the host-buffer call and the CPU oracle; returns the JSON
    line (rank 0) or None."""
    dist, dev, world, rank, local = ctx["dist"], ctx["dev"], ctx["world"], ctx["rank"], ctx["local"]
    k = wl.k(density)
    n_reuse = len(steps_qkv) - 1
    C = wl.C
    Q0, K0, V0 = steps_qkv[0]
    B, H, N, d = Q0.shape
    ws = api.workspace(Q0, C, k)
    O_full = torch.empty_like(Q0)
    perm = torch.empty((B, H, N), dtype=torch.int32, device=dev)
    idx = torch.empty((B, H, N // C, k), dtype=torch.int32, device=dev)
    R = torch.empty_like(Q0)
    out = torch.empty_like(Q0)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731

    def one_step(rec):
        Q, K, V = steps_qkv[0]
        e = [ev() for _ in range(5)]
        e[0].record()
        api.dense_attn(Q, K, V, O=O_full, lse=lse)
        e[1].record()
        api.group(Q, C, perm=perm, ws=ws)
        e[2].record()
        api.select(Q, K, perm, C, k, lse=lse, idx=idx, ws=ws)
        e[3].record()
        api.residual(Q, K, V, perm, C, idx, O_full, R=R)
        e[4].record()
        re = []
        for s in range(1, n_reuse + 1):
            Qs, Ks, Vs = steps_qkv[s]
            a, b = ev(), ev()
            a.record()
            api.sparse_attn(Qs, Ks, Vs, perm, C, idx, R=R, out=out)
            b.record()
            re.append((a, b))
        rec.append((e, re))

    warm = []
    for _ in range(args.warmup):
        one_step(warm)
    api.sync_status()

    sampler = ClockSampler(local, args.clocks_csv)
    if rank == 0:
        sampler.start()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t_start, t_end = ev(), ev()
    rec = []
    t_start.record()
    for _ in range(args.steps):
        one_step(rec)
    t_end.record()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clocks = sampler.stop() if rank == 0 else None
    api.sync_status()

    # the dense baseline for the ideal-speedup ratio: the same dense kernel producing only O
    # (the anchor's call above also emits the LSE the selection needs)
    Qb, Kb, Vb = steps_qkv[1 % len(steps_qkv)]
    base_ev = []
    for it in range(args.warmup + args.steps):
        a, b = ev(), ev()
        a.record()
        api.dense_attn(Qb, Kb, Vb, O=out, want_lse=False)
        b.record()
        if it >= args.warmup:
            base_ev.append((a, b))
    torch.cuda.synchronize()
    base_ms = [a.elapsed_time(b) for a, b in base_ev]

    total_ms = t_start.elapsed_time(t_end)
    dense_ms = [r[0][0].elapsed_time(r[0][1]) for r in rec]
    group_ms = [r[0][1].elapsed_time(r[0][2]) for r in rec]
    select_ms = [r[0][2].elapsed_time(r[0][3]) for r in rec]
    resid_ms = [r[0][3].elapsed_time(r[0][4]) for r in rec]
    reuse_ms = [a.elapsed_time(b) for r in rec for (a, b) in r[1]]

    # the whole 50-step schedule, timed step by step
    kinds, sched_ms = timed_schedule(steps_qkv, C, k)
    by_kind = {kd: [m for kk_, m in zip(kinds, sched_ms) if kk_ == kd] for kd in ("dense", "anchor", "reuse")}
    sched_total = sum(sched_ms)
    after_warm = sched_ms[4:]

    (total_ms, reuse_mean, dense_mean, dense_base, group_mean, select_mean, resid_mean, sched_total,
     sched_after, sched_dense, sched_anchor, sched_reuse) = max_over_ranks(
        [total_ms, statistics.mean(reuse_ms), statistics.mean(dense_ms), statistics.mean(base_ms),
         statistics.mean(group_ms), statistics.mean(select_ms), statistics.mean(resid_ms), sched_total,
         statistics.mean(after_warm), statistics.mean(by_kind["dense"]), statistics.mean(by_kind["anchor"]),
         statistics.mean(by_kind["reuse"])], dist, dev)

    # end to end through the public API with host buffers: pinned Q, K, V in, O_hat out.  The
    # host call pipelines chunks of heads (copy in / compute / copy out on three streams).
    e2e = None
    if not args.no_e2e:
        hq, hk, hv = (t.cpu().pin_memory() for t in steps_qkv[1 % len(steps_qkv)])
        hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        staging = api.host_staging(tuple(hq.shape), E2E_HEADS_PER_CHUNK)
        for it in range(2 + args.steps):
            if it == 2:
                torch.cuda.synchronize()
                a, b = ev(), ev()
                a.record()
            api.sparse_attn_host(hq, hk, hv, perm, C, idx, R=R, out=hout, heads_per_chunk=E2E_HEADS_PER_CHUNK,
                                 staging=staging)
        b.record()
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks([a.elapsed_time(b) / args.steps], dist, dev)[0]
        # the host path's result is the device path's, bit for bit
        api.sparse_attn(*steps_qkv[1 % len(steps_qkv)], perm, C, idx, R=R, out=out)
        if not torch.equal(hout, out.cpu()):
            raise RuntimeError("host-buffer reuse step differs from the device-resident one")
        del staging
        e2e = {"value": e2e_ms / world, "unit": "ms/layer",
               "h2d_bytes_per_step": 3 * hq.numel() * hq.element_size(),
               "d2h_bytes_per_step": hout.numel() * hout.element_size(),
               "heads_per_chunk": E2E_HEADS_PER_CHUNK}

    # the fp64 oracle's reuse step on the same inputs and the same cached metadata (rank 0 at
    # one GPU only), head by head up to about 45 s of host time
    cpu = None
    if not args.no_cpu_baseline and world == 1 and rank == 0:
        Qs, Ks, Vs = (t.cpu().reshape(B * H, N, d) for t in steps_qkv[1 % len(steps_qkv)])
        p_h = perm.cpu().reshape(B * H, N).numpy()
        i_h = idx.cpu().reshape(B * H, N // C, k).numpy()
        r_h = R.cpu().reshape(B * H, N, d)
        sec, done = oracle_reuse_heads(Qs, Ks, Vs, p_h, i_h, r_h, C, range(B * H), seconds_cap=45.0)
        what = "all" if done == B * H else f"{done} of"
        cpu = {"value": sec * B * H * 1000.0, "unit": "ms/layer", "cores": cpu_cores(), "kind": "oracle",
               "sample": f"fp64 NumPy oracle reuse step (sparse attention + residual) on {what} {B * H} heads of "
                         f"the timed layer with its cached metadata, {sec * done:.1f} s"
                         + ("" if done == B * H else f", scaled x{B * H}/{done}")}
        del Qs, Ks, Vs, r_h

    if rank != 0:
        return None

    pk, pk_kind = peaks()
    flops = 4.0 * B * H * N * k * d
    achieved = flops / (reuse_mean * 1e-3) / 1e12
    peak = pk["bf16_tflops"]
    ideal_frac = (dense_base / reuse_mean) * (k / N)
    anchor_ms = dense_mean + group_mean + select_mean + resid_mean
    formula = (4 * dense_base + 5 * anchor_ms + 41 * reuse_mean) / 50.0
    amortized = sched_total / 50.0
    n_anchor = len(by_kind["anchor"])
    heads_split = ctx.get("split") == "heads" and world > 1
    return {
        "metric": METRIC,
        # replicas: N layers in the time of one, so the time per layer is the time / N; heads:
        # one layer split N ways, so its time is the slowest rank's
        "value": reuse_mean if heads_split else reuse_mean / world,
        "unit": "ms/layer",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps,
        "higher_is_better": False,
        "scaling": "strong" if heads_split else "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded DiT-shaped generator, on device)",
        "config": {"workload": f"{wl.name}: B={B} H={H * world if heads_split else H} N={N} d={d} C={C} s={density} "
                               f"k={k}; step = anchor + {n_reuse} reuse steps",
                   "global_batch": B if heads_split else B * world, "seq_len": N,
                   "parallelism": f"heads x{world}" if heads_split else f"replicas x{world}",
                   "l2": f"inputs larger than L2 (Q,K,V {3 * Q0.numel() * 2 / 1e6:.0f} MB per step), no flush"},
        "pct_of_ideal_1_over_s": 100.0 * ideal_frac,
        "reuse_tflops": achieved,
        "pct_of_bf16_peak": 100.0 * achieved / peak,
        "pct_of_bf16_peak_sustained": 100.0 * achieved / pk["bf16_tflops_sustained"],
        "dense_baseline_ms": dense_base,
        "dense_tflops": 4.0 * B * H * N * N * d / (dense_base * 1e-3) / 1e12,
        "schedule_50": {
            "amortized_ms_per_step": amortized,
            "timed": "50 steps of api.Schedule (dense 0-3, anchors 4, 14, 24, 34, 44), CUDA events per step",
            "dense_step_ms": sched_dense, "anchor_step_ms": sched_anchor, "reuse_step_ms": sched_reuse,
            "formula_ms_per_step": formula,
            "delta_s_all_steps": (amortized - sched_reuse) / dense_base,
            "delta_s_after_warmup": (sched_after - sched_reuse) / dense_base,
            "delta_s_anchor_extras": n_anchor * (sched_anchor - dense_base) / (50.0 * dense_base),
            "speedup_vs_dense": dense_base / amortized,
        },
        "breakdown_ms": {"dense": dense_mean, "group": group_mean, "select": select_mean,
                         "residual": resid_mean, "reuse": reuse_mean, "anchor": anchor_ms},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": measured_traffic(wl.name, k),
                     "kernel": f"attn_kernel<{d},kReuse>",
                     "peak_kind": f"bf16_tflops burst ({pk_kind}): the kernel is timed launch by launch"},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches_per_step(N, C, n_reuse) * args.steps,
        "clocks": clocks,
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="mcs", choices=["mcs", "reference"])
    ap.add_argument("--config", default="480p", choices=sorted(workload.WORKLOADS))
    ap.add_argument("--density", type=float, default=0.15)
    ap.add_argument("--sweep", action="store_true",
                    help="one line per density of the config (--densities, default the config's own list)")
    ap.add_argument("--densities", default=None, help="comma-separated densities for --sweep")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--reuse-steps", type=int, default=REUSE_PER_STEP,
                    help="reuse steps per step (fewer keeps profiling captures small)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--layers", type=int, default=0,
                    help="time the 50-step schedule of this many layers instead (metadata cache mode)")
    ap.add_argument("--clocks-csv", default=None,
                    help="where the nvidia-smi samples of the timed region are written (default: a temp file)")
    ap.add_argument("--study", action="store_true",
                    help="error decomposition of the selection variants at equal density instead")
    ap.add_argument("--split", default="replicas", choices=["replicas", "heads"],
                    help="with N > 1 GPUs: one layer per rank (weak scaling) or one layer split by heads")
    ap.add_argument("--kmeans", action="store_true",
                    help="time Fast PDDP against the equal-size k-means grouping baseline instead")
    ap.add_argument("--device-slots", type=int, default=2,
                    help="with --layers: layers whose metadata stays on the device (the rest offloaded)")
    args = ap.parse_args()

    wl = workload.WORKLOADS[args.config]
    k = wl.k(args.density)
    if args.impl == "reference":
        run_reference(args, wl, k)
        return
    if args.layers > 0:
        run_layers(args, wl, k)
        return
    if args.study:
        run_study(args, wl, k)
        return
    if args.kmeans:
        run_kmeans(args, wl)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)

    # inputs: reuse_steps + 1 perturbed copies of Q, K, V resident in HBM (each ~594 MB at
    # 480p, far larger than L2, so no flush is needed between iterations)
    gen = workload.Generator(wl, device=str(dev))
    steps_qkv = [gen.current()]
    for _ in range(args.reuse_steps):
        steps_qkv.append(gen.advance())
    del gen
    if args.split == "heads" and world > 1:
        # one layer split by heads: every step of the path works head by head, so each rank
        # takes its share of the heads and nothing is exchanged (B = 1 here)
        lo, hi = api.head_shard(wl.B * wl.H, rank, world)
        steps_qkv = [tuple(t[:, lo:hi].contiguous() for t in qkv) for qkv in steps_qkv]
    torch.cuda.synchronize()

    if args.sweep:
        dens = [float(x) for x in args.densities.split(",")] if args.densities else list(wl.densities)
    else:
        dens = [args.density]
    ctx = dict(dist=dist, dev=dev, world=world, rank=rank, local=local, split=args.split)
    for s in dens:
        line = measure(args, wl, s, steps_qkv, ctx)
        if line is not None:
            print(json.dumps(line), flush=True)
        torch.cuda.empty_cache()

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

"""Benchmark of the block-sparse global-attention layer on B200.

One step = one whole layer on one GPU, on seeded synthetic inputs already resident in HBM.
bf16 layers (default): packing + pooling -> mask -> special queries -> fused patch rows
(block-sparse attention, special keys and the merge in one pass). `--path five`: pool ->
mask -> pack -> special dense -> block-sparse attention -> merge.
Default workload: 100 frames x (777 patch + 5 special) tokens, 16 heads, d = 64, b = 128,
layer budget rho = 0.75 split across heads by capped water-filling of LogNormal(0, 1)
scores, tau = 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Prints one JSON line (rank 0). With N > 1 (torchrun), every rank runs its own replica of
the layer (the layer has no exchange step); time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from view_transformers_b200 import configs, synth  # noqa: E402

METRIC = "global-attn ms/layer & effective TFLOPS vs dense at 100 frames, rho=0.75"
UNIT = "ms/layer"


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p["bf16_tflops_sustained"], "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            self.proc.wait(timeout=10)

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        try:
            for line in open(self.path):
                f = [x.strip() for x in line.split(",")]
                if len(f) < 9:
                    continue
                try:
                    sm.append(float(f[1]))
                    mx.append(float(f[2]))
                except ValueError:
                    continue
                for n, v in zip(names, f[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        finally:
            os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------- helpers
def kernel_source_hash() -> str:
    """sha256 of the attention kernel's sources with comments and whitespace removed, so that
    the stored traffic record stays valid across comment edits and goes stale on any code
    change."""
    import hashlib
    import re
    text = "".join(open(os.path.join(ROOT, "view_transformers_b200", "csrc", f)).read()
                   for f in ("attn_tc.cu", "sm100.cuh", "tc_layout.cuh"))
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return hashlib.sha256(re.sub(r"\s+", "", text).encode()).hexdigest()


def measured_traffic(w, path):
    """DRAM bytes per launch of the fused kernel from the committed ncu record, scaled to this
    workload by patch tokens x heads; None when the kernel code changed since the capture."""
    if path != "fused":
        return None
    try:
        rec = json.load(open(os.path.join(ROOT, "profiles", "fused_traffic.json")))
        src_hash = kernel_source_hash()
    except (OSError, ValueError):
        return None
    if src_hash != rec.get("source_sha256"):
        return None
    return rec["dram_bytes_per_launch"] * (w.n_patch * w.heads) / (rec["patch_tokens"] * rec["heads"])



def xu_roofline(f_kernel, kernel_ms, w, clocks) -> dict:
    """The attention kernel's other bound: one ex2 per computed score entry (f_kernel / 4d
    entries) on the special-function unit, 16 ex2 per clock per SM (measured on this B200 by a
    back-to-back ex2.approx.f32 microbenchmark), 148 SMs, at the median SM clock sampled during
    the timed region."""
    entries = f_kernel / (4.0 * w.head_dim)
    achieved = entries / (kernel_ms * 1e-3)
    mhz = clocks.get("sm_mhz") or 1965.0
    peak = 16.0 * 148 * mhz * 1e6
    return {"bound": "xu", "achieved": achieved, "peak": peak, "unit": "ex2/s", "frac": achieved / peak,
            "peak_kind": "16 ex2/clock/SM x 148 SMs x sampled SM clock"}


def sparse_flops(kv_cnt, kv_idx, w) -> float:
    """4 d sum_h sum_(i, j kept) |I_i| |J_j| over patch query/key blocks."""
    B, b, Np = w.n_blocks, w.block, w.n_patch
    sizes = np.minimum(b, Np - np.arange(B) * b).astype(np.float64)       # |I_j|
    valid = np.arange(B)[None, None, :] < kv_cnt[:, :, None]
    keys = np.where(valid, sizes[np.minimum(kv_idx.astype(np.int64), B - 1)], 0.0).sum(axis=2)   # [H, B]
    return float(4 * w.head_dim * (keys * sizes[None, :]).sum())


def special_flops(w) -> float:
    return float(4 * w.head_dim * w.heads * (w.n_special * w.n_tokens + w.n_patch * w.n_special))


def stage_bytes(w) -> dict:
    e = 2 if w.dtype == "bf16" else 4
    row = w.heads * w.head_dim
    B = w.n_blocks
    pooled = 2 * w.heads * B * w.head_dim * 4
    return {
        "pool": 2 * w.n_patch * row * e + pooled,
        "pack": 3 * w.n_tokens * row * e + 3 * w.n_tokens * row * 2,
        "pack_pool": 3 * w.n_tokens * row * e + 3 * w.n_tokens * row * 2 + pooled,
        "merge": 2 * w.n_patch * row * 4 + 2 * w.heads * w.n_patch * 4 + w.n_patch * row * e,
    }


def step_calls(L, q, k, v, path: str):
    """The library calls of one layer, as (stage name, callable, our kernel launches)."""
    from view_transformers_b200 import _lib
    import torch
    b = L.buf if path == "fused" else L.partials()
    sp = torch.cuda.current_stream().cuda_stream
    status = b.status.data_ptr()
    lay = L.layout
    qp, kp, vp = q.data_ptr(), k.data_ptr(), v.data_ptr()
    mask = ("mask", lambda: L._select(sp, v), 2 if L.selector == "ress" else 1)
    if path == "fused" and L.selector in ("random", "uniform"):   # no pooled means needed
        calls = [("pack", lambda: _lib.bsa_pack_qkv(lay, qp, kp, vp, L.ws_ptr, L.ws_bytes, status, sp), 1), mask]
    elif path == "fused":
        calls = [
            ("pack_pool", lambda: _lib.bsa_pack_pool_qkv(lay, qp, kp, vp, L.ws_ptr, L.ws_bytes, b.pq.data_ptr(),
                                                         b.pk.data_ptr(), status, sp), 1),
            mask,
        ]
    else:
        calls = [
            ("pool", lambda: _lib.bsa_pool_qk(lay, qp, kp, b.pq.data_ptr(), b.pk.data_ptr(), status, sp), 1),
            mask,
            ("pack", lambda: _lib.bsa_pack_qkv(lay, qp, kp, vp, L.ws_ptr, L.ws_bytes, status, sp), 1),
        ]
    if path == "fused":
        calls += [
            ("special", lambda: _lib.bsa_special_dense(lay, qp, kp, vp, L.ws_ptr, L.ws_bytes, b.out.data_ptr(),
                                                       None, None, status, sp), 2),
            ("sparse", lambda: _lib.bsa_block_sparse_attn_fused(lay, qp, kp, vp, L.ws_ptr, L.ws_bytes,
                                                                b.kv_idx.data_ptr(), b.kv_cnt.data_ptr(),
                                                                b.out.data_ptr(), status, sp), 1),
        ]
    else:
        calls += [
            ("special", lambda: _lib.bsa_special_dense(lay, qp, kp, vp, L.ws_ptr, L.ws_bytes, b.out.data_ptr(),
                                                       b.o_ps.data_ptr(), b.lse_ps.data_ptr(), status, sp), 3),
            ("sparse", lambda: _lib.bsa_block_sparse_attn(lay, qp, kp, vp, L.ws_ptr, L.ws_bytes, b.kv_idx.data_ptr(),
                                                          b.kv_cnt.data_ptr(), b.o_pp.data_ptr(),
                                                          b.lse_pp.data_ptr(), status, sp), 1),
            ("merge", lambda: _lib.bsa_merge(lay, b.o_pp.data_ptr(), b.lse_pp.data_ptr(), b.o_ps.data_ptr(),
                                             b.lse_ps.data_ptr(), b.out.data_ptr(), status, sp), 1),
        ]
    return calls


def run_forward(torch, L, q, k, v, steps, path="fused", kernel_ms=None):
    """Runs `steps` layers through the public L.forward; returns the total device time in ms.
    With a list
    `kernel_ms` (fused path), appends the in-place duration of each patch-row attention launch,
    timed by CUDA events on the stream it is launched on."""
    st = torch.cuda.current_stream()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    evs = []
    start.record(st)
    for _ in range(steps):
        pair = None
        if kernel_ms is not None and path == "fused":
            pair = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            evs.append(pair)
        L.forward(q, k, v, fused=(path == "fused"), kernel_events=pair)
    end.record(st)
    end.synchronize()
    if kernel_ms is not None:
        kernel_ms.extend(a.elapsed_time(b_) for a, b_ in evs)
    return start.elapsed_time(end)


def run_steps(torch, L, q, k, v, steps, path="fused"):
    """Runs `steps` layers; returns per-stage durations (ms, per step) and the total (ms)."""
    st = torch.cuda.current_stream()
    calls = step_calls(L, q, k, v, path)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)] for _ in range(steps)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(st)
    for s in range(steps):
        e = evs[s]
        e[0].record(st)
        for i, (_, fn, _) in enumerate(calls):
            fn()
            e[i + 1].record(st)
    end.record(st)
    end.synchronize()
    per_stage = {name: [evs[s][i].elapsed_time(evs[s][i + 1]) for s in range(steps)]
                 for i, (name, _, _) in enumerate(calls)}
    return per_stage, start.elapsed_time(end), sum(c[2] for c in calls)


# ---------------------------------------------------------------------------- CPU oracle
def oracle_layer_sample(w, x, budget_s: float, seed: int = 7, keep: dict | None = None):
    """Times the fp64 oracle on a bounded sample of one layer and scales it to ms/layer.

    Full pooling and mask prediction; attention for a seeded sample of (head, query block)
    pairs plus a seeded sample of special query rows, scaled by the sampled fraction. When
    `keep` is a dict it receives the oracle's mask result and the outputs of the first
    sampled pairs and special rows, for a parity check of the same run."""
    import oracle
    from threadpoolctl import threadpool_info, threadpool_limits
    host_cpus = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    with threadpool_limits(limits=host_cpus):           # the BLAS pools use every host CPU
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
        est, sample = _oracle_layer_sample(oracle, w, x, budget_s, seed, keep)
    return est, threads, host_cpus, sample


def sample_parity(torch, L, w, keep: dict) -> dict:
    """The benchmarked run's output and mask against the oracle on the CPU leg's sample:
    relative L2 and max-abs over the kept rows (oracle run with its own mask), and the mask
    of every row under the near-tie rule (the dual-threshold selector only)."""
    from oracle.compare import compare_mask, max_abs, rel_l2
    got, ref = [], []
    out = L.buf.out
    for rows, h, o in keep["rows"]:
        idx = torch.as_tensor(rows, device=out.device)
        got.append(out[idx, h].float().cpu().numpy())
        ref.append(o)
    got, ref = np.concatenate(got), np.concatenate(ref)
    r = rel_l2(got, ref)
    rep = {"rows": int(len(ref)), "rel_l2": r, "nmse": r * r, "max_abs": max_abs(got, ref),
           "against": "the oracle's own mask, rows of the first sampled (head, query block) pairs and special rows"}
    if keep.get("mask") is not None:
        m = compare_mask(keep["mask"], L.selected(), w.tau)
        rep["mask"] = {"rows": m.rows, "exact": m.exact, "near_tie_exempt": m.exempt, "failed": m.failed}
    return rep


def _oracle_layer_sample(oracle, w, x, budget_s, seed, keep=None):
    from oracle import selectors
    lay = oracle.Layout(w.frames, w.tokens_per_frame, w.layer_special, w.heads, w.head_dim, w.block)
    t0 = time.perf_counter()
    Q, K = oracle.to_f64(x.q, w.dtype), oracle.to_f64(x.k, w.dtype)
    dens = None if x.scores is None else oracle.water_fill(x.scores, w.heads * (1 - w.rho), 1.0)
    kh = oracle.head_k(lay, w.rho, dens)
    if w.selector == "predict":
        mres = oracle.predict_mask(oracle.pool(Q, lay), oracle.pool(K, lay), lay.head_dim, kh, w.tau)
        selected = mres.selected
        if keep is not None:
            keep["mask"] = mres
    elif w.selector == "random":
        selected = selectors.random_mask(lay, kh, w.seed)
    elif w.selector == "uniform":
        selected = selectors.uniform_mask(lay, w.stride)
    elif w.selector == "probe":
        selected = selectors.probe_mask(Q, K, lay, kh)[1]
    else:
        selected = None          # drift-score rows: selected per sampled pair below
        from oracle import ress
        PQ, PK = oracle.pool(Q, lay), oracle.pool(K, lay)
        PV = oracle.pool(oracle.to_f64(x.v, w.dtype), lay)
        probs = oracle.pooled_probs(PQ, PK, lay.head_dim)
    t_mask = time.perf_counter() - t0
    V = oracle.to_f64(x.v, w.dtype)
    g = np.random.default_rng(seed)
    pairs = [(int(g.integers(0, lay.heads)), int(g.integers(0, lay.B))) for _ in range(100000)]
    t1 = time.perf_counter()
    done = 0
    sr = oracle.special_rows(lay)
    for h, i in pairs:
        rows = oracle.patch_rows(lay)[slice(*oracle.block_bounds(lay, i))]
        kept = selected[h, i] if selected is not None else ress.select_row(probs[h, i], PV[h], int(kh[h]),
                                                                          w.rounds)[0]
        keys = np.concatenate([sr, oracle.patch_keys_of(lay, kept)])
        o = oracle.attend(Q[rows, h], K[keys, h], V[keys, h])[0]
        if keep is not None and done < 16:
            keep.setdefault("rows", []).append((rows, h, o))
        done += 1
        if time.perf_counter() - t1 > budget_s * 0.8:
            break
    t_patch = time.perf_counter() - t1
    t2 = time.perf_counter()
    n_spec_rows = 0
    if lay.Ns:
        for h in range(lay.heads):
            rows = sr[g.choice(len(sr), size=min(8, len(sr)), replace=False)]
            o = oracle.attend(Q[rows, h], K[:, h], V[:, h])[0]
            if keep is not None:
                keep.setdefault("rows", []).append((rows, h, o))
            n_spec_rows += len(rows)
    t_spec = time.perf_counter() - t2
    total_pairs = lay.heads * lay.B
    est = t_mask + t_patch * total_pairs / done + (t_spec * (lay.heads * lay.Ns) / n_spec_rows if n_spec_rows else 0)
    sample = (f"sampled estimate: full pool+mask ({t_mask:.1f} s) measured; attention of {done}/{total_pairs} "
              f"(head, query-block) pairs ({t_patch:.1f} s) and {n_spec_rows}/{lay.heads * lay.Ns} special "
              f"(row, head) pairs ({t_spec:.1f} s) measured, each scaled by its sampled fraction to one layer")
    return est * 1e3, sample


def reference_arm(args, w):
    x = synth.make_inputs(w) if w.kind == "global" else None
    times, walls = [], []
    for s in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        if w.kind == "global":
            ms, threads, host_cpus, sample = oracle_layer_sample(w, x, budget_s=args.ref_budget, seed=s)
        else:
            ms, threads, host_cpus, sample = oracle_block_sample(w, budget_s=args.ref_budget, seed=s)
        if s >= args.warmup:
            times.append(ms)
            walls.append(time.perf_counter() - t0)
    v = float(np.mean(times))
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": v, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": threads, "host_cpus": host_cpus, "kind": "oracle",
                             "extrapolated": True, "sample": sample},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            # each step runs a bounded sample of the layer and scales it to one layer: the value is
            # an estimate of the oracle's time per layer, not the wall time of the step
            "extrapolated": True, "sampled_wall_s_per_step": float(np.mean(walls))}
    print(json.dumps(line), flush=True)


SELECTOR_TEXT = {
    "predict": "",
    "random": ", random blocks (k_h per row, Philox4x32-10 keys, seed {seed})",
    "uniform": ", fixed-stride uniform sampling (every {stride}th block)",
    "probe": ", query-probe Top-K (mean-query scores, k_h per head)",
    "ress": ", drift-score selection (k_h per head, up to {rounds} restoration rounds)",
}


KIND_TEXT = {
    "global": "",
    "frame": "; frame-wise dense attention over each frame's {T} tokens (no mask: rho, tau, b unused)",
    "block": "; QKV projection (C = {C} -> 3C) + this global layer + output projection, random-init weights",
    "frame_block": "; QKV projection (C = {C} -> 3C) + frame-wise dense attention + output projection, "
                   "random-init weights",
}


def workload_config(w):
    return {"workload": f"{w.name}: {w.frames} frames x ({w.patch_per_frame} patch + {w.special_per_frame} special)"
                        f" tokens, {w.heads} heads, d={w.head_dim}, b={w.block}, rho={w.rho}, tau={w.tau}"
                        + (", per-head budgets (LogNormal(0,1) scores, capped water-filling, cap 1)"
                           if w.head_budgets else "")
                        + SELECTOR_TEXT[w.selector].format(seed=w.seed, stride=w.stride, rounds=w.rounds)
                        + (", special tokens read as patch tokens (no dense special path)"
                           if w.sparse_specials else "")
                        + KIND_TEXT[w.kind].format(T=w.tokens_per_frame, C=w.heads * w.head_dim),
            "frames": w.frames, "tokens_per_frame": w.tokens_per_frame, "heads": w.heads, "head_dim": w.head_dim,
            "block": w.block, "rho": w.rho, "tau": w.tau, "global_batch": 1, "seq_len": w.n_tokens,
            "parallelism": "replicas",
            "l2": "inputs larger than L2 (Q, K, V and the packed workspace: about 1 GB touched per step)"}


# ---------------------------------------------------------------------------- end to end
def e2e_pipelined(torch, L, q, k, v, steps: int, path: str) -> float:
    """ms per layer through L.forward with every step's inputs copied from pinned host memory
    and its output copied back. Two device slots: the copy stream fills slot s+1 while the
    compute stream runs step s (it waits until step s-1 released that slot); the output of
    each step goes back on a third stream. Timed from the first host-to-device copy to the
    last device-to-host copy, on the device."""
    hq, hk, hv = (t_.cpu().pin_memory() for t_ in (q, k, v))
    hout = torch.empty(L.buf.out.shape, dtype=L.buf.out.dtype).pin_memory()
    slots = [tuple(torch.empty_like(t_) for t_ in (q, k, v, L.buf.out)) for _ in range(2)]
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    loaded = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    saved = [torch.cuda.Event() for _ in range(2)]

    def upload(s):
        d = slots[s % 2]
        with torch.cuda.stream(up):
            if s >= 2:
                up.wait_event(computed[s % 2])   # step s-2 is done with this slot's inputs
            for dst, src in zip(d[:3], (hq, hk, hv)):
                dst.copy_(src, non_blocking=True)
            loaded[s % 2].record(up)

    def run(n, t0=None, t1=None):
        if t0 is not None:
            t0.record(up)
        upload(0)
        for s in range(n):
            if s + 1 < n:
                upload(s + 1)
            d = slots[s % 2]
            comp.wait_event(loaded[s % 2])
            if s >= 2:
                comp.wait_event(saved[s % 2])    # the output of step s-2 has left this slot
            L.forward(d[0], d[1], d[2], fused=(path == "fused"), out=d[3])
            computed[s % 2].record(comp)
            with torch.cuda.stream(down):
                down.wait_event(computed[s % 2])
                hout.copy_(d[3], non_blocking=True)
                saved[s % 2].record(down)
        if t1 is not None:
            t1.record(down)
        torch.cuda.synchronize()

    run(2)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    run(steps, t0, t1)
    return t0.elapsed_time(t1) / steps


def e2e_pipelined_calls(torch, t, ins, outk, calls, steps: int) -> float:
    """e2e_pipelined for a list of library calls that read the tensors t[k] for k in `ins`
    and write t[outk] (the calls look the tensors up when they run): two device slots of those
    tensors, filled and drained on their own streams while the compute stream runs the calls
    on the other slot. ms per step, timed on the device."""
    keys = list(ins) + [outk]
    orig = {k_: t[k_] for k_ in keys}
    host_in = {k_: t[k_].cpu().pin_memory() for k_ in ins}
    hout = torch.empty(t[outk].shape, dtype=t[outk].dtype).pin_memory()
    slots = [{k_: torch.empty_like(t[k_]) for k_ in keys} for _ in range(2)]
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    loaded = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    saved = [torch.cuda.Event() for _ in range(2)]

    def upload(s):
        d = slots[s % 2]
        with torch.cuda.stream(up):
            if s >= 2:
                up.wait_event(computed[s % 2])   # step s-2 is done with this slot's inputs
            for k_ in ins:
                d[k_].copy_(host_in[k_], non_blocking=True)
            loaded[s % 2].record(up)

    def run(n, t0=None, t1=None):
        if t0 is not None:
            t0.record(up)
        upload(0)
        for s in range(n):
            if s + 1 < n:
                upload(s + 1)
            d = slots[s % 2]
            comp.wait_event(loaded[s % 2])
            if s >= 2:
                comp.wait_event(saved[s % 2])    # the output of step s-2 has left this slot
            t.update(d)
            for _, fn, _ in calls:
                fn()
            computed[s % 2].record(comp)
            with torch.cuda.stream(down):
                down.wait_event(computed[s % 2])
                hout.copy_(d[outk], non_blocking=True)
                saved[s % 2].record(down)
        if t1 is not None:
            t1.record(down)
        torch.cuda.synchronize()

    try:
        run(2)
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        run(steps, t0, t1)
    finally:
        t.update(orig)
    return t0.elapsed_time(t1) / steps


# ---------------------------------------------------------------------------- frame / block steps
def oracle_block_sample(w, budget_s: float, seed: int = 7):
    """Times the fp64 oracle of a frame-attention or projection-block step on bounded samples
    and scales each part to one step: the projections on seeded token rows, the frame attention
    on seeded (row, head) pairs, the global layer through oracle_layer_sample."""
    import oracle  # noqa: F401
    from oracle import layer_io
    from threadpoolctl import threadpool_info, threadpool_limits
    host_cpus = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    g = np.random.default_rng(seed)
    N, H, d = w.n_tokens, w.heads, w.head_dim
    C = H * d
    parts, est = [], 0.0
    with threadpool_limits(limits=host_cpus):
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
        if w.kind in ("block", "frame_block"):
            bi = synth.make_block_inputs(w.with_(frames=1))          # weights do not depend on F
            rows = min(N, 4096)
            X = g.standard_normal((rows, C))
            t0 = time.perf_counter()
            layer_io.qkv_project(X, synth.decode(bi.w_qkv, "bf16"), bi.b_qkv, H, d)
            layer_io.out_project(X.reshape(rows, H, d), synth.decode(bi.w_o, "bf16"), bi.b_o)
            t = time.perf_counter() - t0
            est += t * N / rows
            parts.append(f"projections of {rows}/{N} token rows ({t:.1f} s)")
        if w.kind in ("frame", "frame_block"):
            x = synth.make_inputs(w.with_(frames=min(w.frames, 4)))
            Q, K, V = (synth.decode(a, "bf16") for a in (x.q, x.k, x.v))
            t0, done = time.perf_counter(), 0
            while time.perf_counter() - t0 < budget_s * 0.5:
                rows = g.integers(0, len(Q), 256)
                heads = g.integers(0, H, 256)
                layer_io.frame_attention_rows(Q, K, V, w.tokens_per_frame, rows, heads)
                done += 256
            t = time.perf_counter() - t0
            est += t * N * H / done
            parts.append(f"frame attention of {done}/{N * H} (row, head) pairs ({t:.1f} s)")
        if w.kind == "block":
            ms, _, _, sample = oracle_layer_sample(w.with_(kind="global"), synth.make_inputs(w), budget_s * 0.5, seed)
            est += ms / 1e3
            parts.append("global layer: " + sample)
    return est * 1e3, threads, host_cpus, "sampled estimate: " + "; ".join(parts) + "; each scaled to one step"


def block_stage_calls(w, L, tensors, status, sp):
    """(stage, callable, launches) of one frame-attention or projection-block step."""
    from view_transformers_b200 import _lib
    lay = _lib.layout_of(w)
    t = tensors
    ptr = (lambda a: 0 if a is None else a.data_ptr())
    calls = []
    if w.kind in ("block", "frame_block"):
        calls.append(("qkv", lambda: _lib.bsa_qkv_project(lay, t["x"].data_ptr(), t["w_qkv"].data_ptr(),
                                                          ptr(t["b_qkv"]), t["q"].data_ptr(), t["k"].data_ptr(),
                                                          t["v"].data_ptr(), status, sp), 1))
    if w.kind in ("frame", "frame_block"):
        calls.append(("pack_frames", lambda: _lib.bsa_pack_frames(lay, t["q"].data_ptr(), t["k"].data_ptr(),
                                                                  t["v"].data_ptr(), t["ws"], t["ws_bytes"], status,
                                                                  sp), 1))
        calls.append(("frame_attn", lambda: _lib.bsa_frame_attention(lay, t["ws"], t["ws_bytes"], t["o"].data_ptr(),
                                                                     status, sp), 1))
    else:
        calls.append(("global_layer", lambda: L.forward(t["q"], t["k"], t["v"], stream=sp, out=t["o"]), 5))
    if w.kind in ("block", "frame_block"):
        calls.append(("out", lambda: _lib.bsa_out_project(lay, t["o"].data_ptr(), t["w_o"].data_ptr(), ptr(t["b_o"]),
                                                          t["y"].data_ptr(), status, sp), 1))
    return calls


def block_parity_sample(torch, w, t, seed: int = 11) -> dict:
    """The benchmarked frame-wise step against the oracle on sampled rows of two frames, each
    stage on the device's own input to it: the QKV projection from x (block workloads), the
    frame attention from the device's Q, K, V, the output projection from the device's
    attention output. Relative L2 and max-abs per stage."""
    from oracle import layer_io
    from oracle.compare import max_abs, rel_l2
    g = np.random.default_rng(seed)
    T, H = w.tokens_per_frame, w.heads
    frames = [int(f) for f in g.choice(w.frames, size=min(2, w.frames), replace=False)]
    dev = t["o"].device
    host = lambda a: a.float().cpu().numpy().astype(np.float64)
    rep = {}

    def stage(got, ref):
        got, ref = np.concatenate(got), np.concatenate(ref)
        return {"values": int(ref.size), "rel_l2": rel_l2(got, ref), "max_abs": max_abs(got, ref)}

    if "y" in t:
        rows = torch.as_tensor([f * T + int(r) for f in frames for r in g.integers(0, T, 16)], device=dev)
        want = layer_io.qkv_project(host(t["x"][rows]), host(t["w_qkv"]), t["b_qkv"].cpu().numpy(), H, w.head_dim)
        rep["qkv_projection"] = stage([host(t[k_][rows]) for k_ in ("q", "k", "v")], list(want))
    got, ref = [], []
    for f in frames:
        sl = slice(f * T, (f + 1) * T)
        Q, K, V = (host(t[k_][sl]) for k_ in ("q", "k", "v"))
        rows, heads = g.integers(0, T, 64), g.integers(0, H, 64)
        ref.append(layer_io.frame_attention_rows(Q, K, V, T, rows, heads))
        o = t["o"][sl]
        got.append(host(o[torch.as_tensor(rows, device=dev), torch.as_tensor(heads, device=dev)]))
    rep["frame_attention"] = stage(got, ref)
    if "y" in t:
        rows = torch.as_tensor([f * T + int(r) for f in frames for r in g.integers(0, T, 16)], device=dev)
        want = layer_io.out_project(host(t["o"][rows]), host(t["w_o"]), t["b_o"].cpu().numpy())
        rep["out_projection"] = stage([host(t["y"][rows])], [want])
    return rep


def bench_block(args, w, world, rank, local, dist):
    """One step = the frame-wise attention layer, or a whole block (QKV projection, attention,
    output projection), on synthetic tokens and random-init weights resident in HBM."""
    import torch
    from view_transformers_b200 import _lib, layer
    N, H, d = w.n_tokens, w.heads, w.head_dim
    C = H * d
    dev = torch.device("cuda", local)
    x = synth.make_inputs(w)
    t = {k_: layer.to_device(a, "bf16") for k_, a in (("q", x.q), ("k", x.k), ("v", x.v))}
    t["o"] = torch.empty_like(t["q"])
    L = None
    if w.kind in ("block", "frame_block"):
        bi = synth.make_block_inputs(w)
        t["x"] = layer.to_device(bi.x, "bf16")
        t["w_qkv"], t["w_o"] = layer.to_device(bi.w_qkv, "bf16"), layer.to_device(bi.w_o, "bf16")
        t["b_qkv"], t["b_o"] = torch.from_numpy(bi.b_qkv).to(dev), torch.from_numpy(bi.b_o).to(dev)
        t["y"] = torch.empty((N, C), dtype=torch.bfloat16, device=dev)
    if w.kind in ("frame", "frame_block"):
        nbytes = _lib.bsa_frame_workspace_size(_lib.layout_of(w))
        t["ws_buf"] = torch.empty(nbytes + 1024, dtype=torch.uint8, device=dev)
        t["ws"], t["ws_bytes"] = (t["ws_buf"].data_ptr() + 1023) // 1024 * 1024, nbytes
    else:
        dens = _lib.bsa_head_budgets(x.scores, w.rho, 1.0) if x.scores is not None else None
        L = layer.BlockSparseLayer.for_workload(w.with_(kind="global"), head_density=dens)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    sp = torch.cuda.current_stream().cuda_stream
    calls = block_stage_calls(w, L, t, status.data_ptr(), sp)

    def run(steps, stage_ms=None):
        st = torch.cuda.current_stream()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)] for _ in range(steps)]
        for s in range(steps):
            evs[s][0].record(st)
            for i, (_, fn, _) in enumerate(calls):
                fn()
                evs[s][i + 1].record(st)
        torch.cuda.synchronize()
        if stage_ms is not None:
            for i, (name, _, _) in enumerate(calls):
                stage_ms[name] = float(np.mean([evs[s][i].elapsed_time(evs[s][i + 1]) for s in range(steps)]))
        return evs[0][0].elapsed_time(evs[-1][-1])

    run(args.warmup)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    stage_ms = {}
    with ClockSampler(local) as clk:
        total_ms = run(args.steps, stage_ms)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    code = _lib.bsa_check_status(status.data_ptr(), sp) or (L.check_status() if L is not None else 0)
    clocks = clk.summary()
    total_ms = max_over_ranks(total_ms, dist, "cuda")
    ms_per_step = total_ms / args.steps
    value = job_ms_per_layer(total_ms, args.steps, world)

    # algorithmic work per stage
    flops = {"qkv": 2.0 * N * C * 3 * C, "out": 2.0 * N * C * C,
             "frame_attn": 4.0 * d * H * w.frames * float(w.tokens_per_frame) ** 2}
    if L is not None:
        kv_cnt = L.buf.kv_cnt.cpu().numpy()
        kv_idx = L.buf.kv_idx.cpu().numpy().view(np.uint16)
        flops["global_layer"] = sparse_flops(kv_cnt, kv_idx, w) + special_flops(w)
    hbm, tf_burst, tf_sus, peak_src = peaks()
    tflops = {k_: flops[k_] / (stage_ms[k_] * 1e-3) / 1e12 for k_ in stage_ms if k_ in flops}
    dom = max((k_ for k_ in stage_ms if k_ in flops), key=lambda k_: stage_ms[k_])
    kernel_name = {"qkv": "bsa_qkv_project (tcgen05 GEMM)", "out": "bsa_out_project (tcgen05 GEMM)",
                   "frame_attn": "bsa_frame_attention (tcgen05 attention)",
                   "global_layer": "global layer (five launches, fused tcgen05 attention dominant)"}[dom]

    # end to end: the step's inputs from pinned host memory, its output back, every step
    ins = ["x"] if "x" in t else ["q", "k", "v"]
    outk = "y" if "y" in t else "o"
    e2e_ms = float("nan")
    if args.e2e_steps > 0:
        e2e_ms = e2e_pipelined_calls(torch, t, ins, outk, calls, args.e2e_steps)
    e2e_value = max_over_ranks(e2e_ms, dist, "cuda") / world
    h2d = sum(t[k_].numel() * t[k_].element_size() for k_ in ins)
    d2h = t[outk].numel() * t[outk].element_size()
    achieved = tflops[dom]
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded N(0,1) tokens / Q, K, V; random-init projection weights N(0, 1/C))",
        "config": workload_config(w),
        "stage_ms": stage_ms, "stage_tflops": tflops, "step_flops": sum(flops[k_] for k_ in stage_ms if k_ in flops),
        "roofline": {"kernel": kernel_name, "bound": "tensor", "achieved": achieved, "peak": tf_burst,
                     "unit": "TFLOP/s", "frac": achieved / tf_burst,
                     "peak_kind": f"{peak_src} burst bf16", "frac_of_sustained": achieved / tf_sus,
                     "flops_per_launch": flops[dom], "launch_ms": stage_ms[dom], "traffic": None},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": args.e2e_steps,
                "copies": "pinned host buffers; inputs of step s+1 and output of step s-1 copied on "
                          "their own streams while step s computes (two device slots)"},
        "gpu_launches": sum(c[2] for c in calls) * args.steps,
        "clocks": clocks, "device_status": code,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        ms, threads, host_cpus, sample = oracle_block_sample(w, budget_s=args.cpu_budget)
        line["cpu_baseline"] = {"value": ms, "unit": UNIT, "cores": threads, "host_cpus": host_cpus,
                                "kind": "oracle", "extrapolated": True, "sample": sample}
        if w.kind in ("frame", "frame_block"):
            line["parity_sample"] = block_parity_sample(torch, w, t)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.destroy_process_group()


# ---------------------------------------------------------------------------- ranks
def max_over_ranks(value: float, dist, device) -> float:
    """The job's time is its slowest rank's: max of a per-rank value over all ranks."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_ms_per_layer(total_ms_max: float, steps: int, world: int) -> float:
    """Whole-job ms per layer: every rank runs `steps` layers (replicas, weak scaling)."""
    return total_ms_max / (steps * world)


# ---------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="perhead100", choices=sorted(configs.ALL))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=20.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--ref-budget", type=float, default=3.0, help="seconds of oracle work per reference step")
    ap.add_argument("--dense-steps", type=int, default=3)
    ap.add_argument("--e2e-steps", type=int, default=30)
    ap.add_argument("--frames", type=int, default=None,
                    help="override the workload's frame count (smaller cases for profiling)")
    ap.add_argument("--path", default=None, choices=["fused", "five"],
                    help="fused: special dense + one fused patch-row pass (bf16 default); "
                         "five: the five-step path with fp32 partials and the merge")
    args = ap.parse_args()
    w = configs.ALL[args.workload]
    if args.frames:
        w = w.with_(name=f"{w.name}_f{args.frames}", frames=args.frames)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            reference_arm(args, w)
        return
    if args.warmup < 3:
        args.warmup = 3

    import torch
    from view_transformers_b200 import _lib, layer
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))

    if w.kind != "global":
        return bench_block(args, w, world, rank, local, dist)
    path = args.path or ("fused" if w.dtype == "bf16" else "five")
    x = synth.make_inputs(w)
    density = _lib.bsa_head_budgets(x.scores, w.rho, 1.0) if x.scores is not None else None
    L = layer.BlockSparseLayer.for_workload(w, head_density=density)
    q, k, v = (layer.to_device(a, w.dtype) for a in (x.q, x.k, x.v))

    run_forward(torch, L, q, k, v, args.warmup, path)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        fused_kernel_ms = []
        total_ms = run_forward(torch, L, q, k, v, args.steps, path, fused_kernel_ms)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    status = L.check_status()
    clocks = clk.summary()
    total_ms = max_over_ranks(total_ms, dist, "cuda")
    ms_per_step = total_ms / args.steps
    value = job_ms_per_layer(total_ms, args.steps, world)   # whole job: layers of all ranks
    # per-stage split (diagnostic, outside the timed region): the same calls one after the
    # other on one stream, a CUDA event between stages
    per_stage, _, launches = run_steps(torch, L, q, k, v, min(args.steps, 10), path)

    kv_cnt = L.buf.kv_cnt.cpu().numpy()
    kv_idx = L.buf.kv_idx.cpu().numpy().view(np.uint16)
    wl = w.layer_view()     # token split as the layer reads it
    f_sparse = sparse_flops(kv_cnt, kv_idx, wl)
    f_special = special_flops(wl)
    density_real = f_sparse / (4 * wl.head_dim * wl.heads * float(wl.n_patch) ** 2)
    stage_ms = {k_: float(np.mean(vs)) for k_, vs in per_stage.items()}

    # dense comparator: the same kernels with every block kept
    dense_ms, dense_stage = None, {}
    if args.dense_steps > 0:
        Ld = layer.BlockSparseLayer.for_workload(w.with_(rho=0.0, tau=0.0, head_budgets=False, selector="predict"))
        run_forward(torch, Ld, q, k, v, 2, path)
        dense_ms = run_forward(torch, Ld, q, k, v, args.dense_steps, path) / args.dense_steps
        dense_stage, _, _ = run_steps(torch, Ld, q, k, v, args.dense_steps, path)
        del Ld

    # end to end through the public API: pinned host inputs in, output back to the host,
    # every step. Copies run on their own streams, double-buffered, so that the inputs of
    # step s+1 and the output of step s-1 cross the host link while step s computes.
    e2e_ms = float("nan")
    h2d = 3 * q.numel() * q.element_size()
    d2h = L.buf.out.numel() * L.buf.out.element_size()
    if args.e2e_steps > 0:
        e2e_ms = e2e_pipelined(torch, L, q, k, v, args.e2e_steps, path)
    e2e_value = max_over_ranks(e2e_ms, dist, "cuda") / world

    hbm, tf_burst, tf_sus, peak_src = peaks()
    # the dominant kernel's duration inside the timed region (events on its stream around each
    # launch); the stage split's number when not available
    sparse_ms = float(np.mean(fused_kernel_ms)) if fused_kernel_ms else stage_ms["sparse"]
    # algorithmic work of the timed sparse kernel: kept patch-patch entries, plus the
    # patch-to-special entries when the special keys are fused into it
    f_kernel = f_sparse + (4.0 * wl.head_dim * wl.heads * wl.n_patch * wl.n_special if path == "fused" else 0.0)
    achieved = f_kernel / (sparse_ms * 1e-3) / 1e12
    sb = stage_bytes(wl)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded N(0,1) Q/K/V, 5% planted correspondences)",
        "config": workload_config(w),
        "effective_tflops": (f_sparse + f_special) / (ms_per_step * 1e-3) / 1e12,
        "sparse_kernel_tflops": achieved,
        "dense_ms_per_layer": dense_ms, "speedup_vs_dense": dense_ms / ms_per_step if dense_ms else None,
        "density": density_real, "sparsity": 1 - density_real,
        "stage_ms": stage_ms, "dense_stage_ms": {k_: float(np.mean(vs)) for k_, vs in dense_stage.items()},
        "stage_gbs": {k_: sb[k_] / (stage_ms[k_] * 1e-3) / 1e9 for k_ in ("pool", "pack", "pack_pool", "merge")
                      if k_ in stage_ms},
        "path": path,
        "roofline": {"kernel": ("bsa_block_sparse_attn_fused" if path == "fused" else "bsa_block_sparse_attn")
                               + " (tcgen05 attention)", "bound": "tensor",
                     "achieved": achieved, "peak": tf_burst, "unit": "TFLOP/s", "frac": achieved / tf_burst,
                     "peak_kind": f"{peak_src} burst bf16 (the timed region is {total_ms / 1e3:.2f} s of "
                                  f"back-to-back layers, well short of the seconds-long sustained measurement)",
                     "frac_of_sustained": achieved / tf_sus, "frac_of_nominal_2250": achieved / 2250.0,
                     "flops_per_launch": f_kernel, "launch_ms": sparse_ms,
                     "launch_ms_alone": stage_ms["sparse"], "traffic": measured_traffic(w, path),
                     "traffic_unit": "bytes per launch (ncu dram read+write, scaled by patch tokens x heads)",
                     "xu": xu_roofline(f_kernel, sparse_ms, w, clocks)},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": args.e2e_steps,
                "copies": "pinned host buffers; inputs of step s+1 and output of step s-1 copied on "
                          "their own streams while step s computes (two device slots)"},
        "gpu_launches": launches * args.steps,
        "clocks": clocks, "device_status": status,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        keep = {}
        ms, threads, host_cpus, sample = oracle_layer_sample(w, x, budget_s=args.cpu_budget, keep=keep)
        if keep.get("rows"):
            line["parity_sample"] = sample_parity(torch, L, w, keep)
        line["cpu_baseline"] = {"value": ms, "unit": UNIT, "cores": threads, "host_cpus": host_cpus,
                                "kind": "oracle", "extrapolated": True, "sample": sample}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""Benchmark of the Orthrus dual-view decode step on B200.

Workload (default): the Qwen3-8B-shaped decoder (36 layers, hidden 4096, 32/8
heads, head_dim 128, QK-RMSNorm, RoPE theta 1e6, SwiGLU 12288, vocab 151936)
with a same-shaped draft attention module per layer, random N(0, 0.02) bf16
weights; batch 1, a 512-token uniform prompt, block K = 32. Drafts are planted
per step: the accept length a ~ Geometric with mean 6 (capped at K), the first
a drafts equal the greedy stream and the next one differs from it. The greedy
stream is produced beforehand on the GPU by plain AR decoding (verify with
K = 0) and the timed run must reproduce it exactly.

One step = orthrus_decode_step (draft view, planted-draft copy, verify view,
accept/commit). The weights (30.3 GB streamed per step) are far larger than
L2, so no L2 flush is needed between steps. Prints ONE JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import dataclasses
import ctypes as C
import glob
import hashlib
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

import synth  # noqa: E402

WEIGHT_BYTES_PER_FORWARD = None  # computed from the shape
KV_BYTES_PER_POSITION = None


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "forward_kernel_traffic.json")


# CUDA sources that hold no code of the persistent forward kernel (its traffic record stays valid
# when only these change)
NOT_FORWARD_SOURCES = {"sampling.cuh"}


def kernel_sources_sha256():
    """sha256 over the CUDA sources the persistent forward kernel is built from (file name +
    contents, sorted by path): every file of csrc/ except NOT_FORWARD_SOURCES."""
    csrc = os.path.join(ROOT, "shared_kv_draft_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(csrc, "*.cuh")) + glob.glob(os.path.join(csrc, "*.cu"))):
        if os.path.basename(f) in NOT_FORWARD_SOURCES:
            continue
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def captured_traffic(kernel, algo_bytes):
    """DRAM bytes per launch of the persistent kernel from the committed ncu capture
    (profiles/forward_kernel_traffic.json), scaled to this launch by its algorithmic bytes.
    None when the kernel sources changed since the capture, or for another kernel."""
    if kernel != "forward" or not algo_bytes or not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as fh:
        cap = json.load(fh)
    if cap.get("sources_sha256") != kernel_sources_sha256():
        return None
    dram = cap["dram_bytes_per_launch"]
    ratio = (sum(dram.values()) / len(dram)) / cap["algorithmic_bytes_per_launch"]
    return round(algo_bytes * ratio)


def rank_reduce(x, op, world, dev):
    """x reduced over the ranks with op ("max", "min" or "sum"); x itself on a single rank.
    Every rank must call it, in the same order (it is a collective)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op={"max": dist.ReduceOp.MAX, "min": dist.ReduceOp.MIN, "sum": dist.ReduceOp.SUM}[op])
    return int(round(t.item())) if isinstance(x, int) else float(t.item())


def raise_on_any_rank(err, world, dev):
    """A collective every rank takes after its checks: all ranks raise if any rank found an
    error, so that no rank is left waiting in a later collective."""
    if rank_reduce(1 if err else 0, "max", world, dev):
        raise RuntimeError(err or "another rank failed its checks")


def shape_bytes(shape):
    """Weight bytes streamed by one forward and KV bytes per cached position (all layers)."""
    D, H, Hkv, d, F, V, L = (shape.d_model, shape.n_heads, shape.n_kv_heads, shape.head_dim, shape.d_ff, shape.vocab,
                             shape.n_layers)
    per_layer = ((H + 2 * Hkv) * d * D + D * H * d + 2 * F * D + D * F) * 2
    return L * per_layer + V * D * 2, L * Hkv * d * 2 * 2


WORKLOADS = {
    "qwen3_8b_b1_k32": dict(shape=synth.QWEN3_8B, batch=1, prompt=512, gen=1024, K=32, mean_accept=6.0,
                            steps=147),
    "tiny_b1_k8": dict(shape=synth.TINY, batch=1, prompt=64, gen=128, K=8, mean_accept=3.0, steps=32),
    # two layers of the Qwen3-8B shape (same kernels, about 2 GB of weights): the small case for profiling
    "qwen3_8b_2layer_b1_k32": dict(shape=dataclasses.replace(synth.QWEN3_8B, n_layers=2, name="qwen3_8b_2layer"),
                                   batch=1, prompt=512, gen=1024, K=32, mean_accept=6.0, steps=40),
}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d.get("bf16_tflops_sustained", d.get("bf16_tflops"))), "measured"
    return 6650.0, 1590.0, "fallback"


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    def __init__(self, gpu_id):
        self.file = tempfile.NamedTemporaryFile(mode="w+", suffix=".csv", delete=False)
        cmd = ["nvidia-smi", f"--query-gpu={CLOCK_FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if gpu_id:
            cmd += ["-i", gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r.split(",") for r in self.file.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                smax.append(float(r[2]))
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def run_ours(args, wl, rank, world, local_rank):
    import torch

    from shared_kv_draft_b200 import orthrus

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    shape, B, P, K = wl["shape"], wl["batch"], wl["prompt"], wl["K"]
    W, Ksteps = args.warmup, args.steps
    total_steps = W + Ksteps

    accepts = synth.planted_accepts(total_steps, wl["mean_accept"], K, seed=1000 + rank)
    need = 1 + int(np.sum(accepts[:total_steps] + 1)) + K + 2  # greedy tokens the schedule reads
    cap = ((P + need + K + 2 + 127) // 128) * 128

    t0 = time.time()
    w = synth.make_weights(shape, 1, 2)
    t_gen = time.time() - t0
    m = orthrus.DeviceModel(shape, w, batch=B, capacity=cap, max_block=K, max_rows=max(B * (K + 1), 512),
                            device=dev)
    prompt = synth.make_prompt(shape, P, 3 + rank)
    tok = torch.from_numpy(prompt.astype(np.int32)).view(1, P).to(dev)
    i32 = lambda *s: torch.zeros(s, dtype=torch.int32, device=dev)
    pending = i32(B)
    m.prefill(tok, [P], pending)

    # greedy AR stream on the GPU (verify with K = 0); the timed run must reproduce it
    # (also the plain-AR baseline: one token per forward through the same kernel, timed with CUDA events)
    stream_dev = i32(need)
    ar1, acc1 = i32(B, 1), i32(B)
    stream_dev[0] = pending[0]
    ar_e0, ar_e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ar_w = min(3, need - 1)
    for j in range(1, need):
        if j == ar_w + 1:
            ar_e0.record()
        m.verify_block(pending, None, 0, ar1)
        m.accept_commit(pending, None, ar1, 0, acc1, stream_dev[j:j + 1])
    ar_e1.record()
    torch.cuda.synchronize(dev)
    ar_tokens = need - 1 - ar_w
    ar_ms = ar_e0.elapsed_time(ar_e1) if ar_tokens > 0 else float("nan")
    if m.read_status() != 0:
        raise RuntimeError(f"device status {m.read_status()} while building the greedy stream")
    stream = stream_dev.cpu().numpy()

    rng = np.random.default_rng(2000 + rank)
    planted = np.zeros((total_steps, B, K), dtype=np.int32)
    j = 0
    for t in range(total_steps):
        planted[t, 0] = synth.planted_drafts(stream, j, int(accepts[t]), K, shape.vocab, rng)
        j += int(accepts[t]) + 1
    planted_dev = torch.from_numpy(planted).to(dev)
    acc_all = i32(total_steps, B)
    com_all = i32(total_steps, B, K + 1)
    launches_per_step = m.launches_per_step(K)

    def reset():
        m.lens.fill_(P)
        pending.fill_(int(stream[0]))

    def run_steps(lo, hi):
        for t in range(lo, hi):
            m.decode_step(pending, K, planted_dev[t], acc_all[t], com_all[t])

    # ---- warm-up, then exactly K timed steps --------------------------------------------------
    reset()
    run_steps(0, W)
    torch.cuda.synchronize(dev)
    props = torch.cuda.get_device_properties(dev)
    gpu_uuid = getattr(props, "uuid", None)
    sampler = ClockSampler(f"GPU-{gpu_uuid}" if gpu_uuid else None)
    time.sleep(0.3)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.profiler.start()  # ncu --profile-from-start off captures the timed steps only
    ev0.record()
    run_steps(W, total_steps)
    ev1.record()
    torch.cuda.synchronize(dev)
    torch.cuda.profiler.stop()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    ms = rank_reduce(ev0.elapsed_time(ev1), "max", world, dev)

    # ---- checks: accept lengths as planted, committed stream == greedy stream -----------------
    err = None
    acc = acc_all.cpu().numpy()[:, 0]
    com = com_all.cpu().numpy()[:, 0]
    out = [int(stream[0])]
    for t in range(total_steps):
        out.extend(int(x) for x in com[t, :max(acc[t], 0) + 1])
    if m.read_status() != 0:
        err = f"device status {m.read_status()} after the timed run"
    elif not np.array_equal(acc, accepts[:total_steps]):
        err = "accept lengths differ from the planted schedule"
    elif out != [int(x) for x in stream[:len(out)]]:
        err = "committed stream differs from the greedy stream"
    raise_on_any_rank(err, world, dev)
    tokens = rank_reduce(int(np.sum(acc[W:] + 1)), "sum", world, dev)  # all ranks' committed tokens
    # algorithmic HBM bytes of the timed steps
    wbytes, kvpos = shape_bytes(shape)
    n0 = P + int(np.sum(acc[:W] + 1))
    bytes_total = 0
    n = n0
    for t in range(W, total_steps):
        bytes_total += 2 * wbytes + kvpos * (2 * n + B * (2 * K + 1))
        n += int(acc[t]) + 1
    hbm_peak, tf_peak, peak_src = load_peaks()

    # ---- traced pass: duration of every launch inside the same decode steps ------------------
    reset()
    run_steps(0, W)
    trace_steps = min(4, Ksteps)
    n_ev = trace_steps * (launches_per_step + 8) + 8
    events = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    for e in events:
        e.record()
    torch.cuda.synchronize(dev)
    handles = (C.c_void_p * n_ev)(*[e.cuda_event for e in events])
    kinds = (C.c_int32 * n_ev)()
    count = (C.c_int32 * 1)(0)
    m.trace(handles, kinds, count)
    run_steps(W, W + trace_steps)
    m.trace(None, None, None)
    torch.cuda.synchronize(dev)
    per_kind = {}
    for i in range(count[0] - 1):
        k = kinds[i]
        if k == 11:
            continue
        dt = events[i].elapsed_time(events[i + 1])
        per_kind.setdefault(orthrus.KIND_NAMES[k], []).append(dt)
    traced_ms = sum(sum(v) for v in per_kind.values())
    kernels = {}
    for name, v in per_kind.items():
        kernels[name] = {"launches_per_step": len(v) // trace_steps, "ms_per_step": sum(v) / trace_steps,
                         "share": sum(v) / traced_ms if traced_ms else None}
    n_mean = P + int(np.sum(acc[:W] + 1))
    M_tok = {"draft": B * K, "verify": B * (K + 1)}
    D, F, V = shape.d_model, shape.d_ff, shape.vocab
    Hd = shape.n_heads * shape.head_dim
    qkv_rows = shape.qkv_rows
    mm = (M_tok["draft"] + M_tok["verify"]) / 2.0
    algo = {  # algorithmic bytes of one launch (mean of the draft and verify launches)
        "gemm_qkv": qkv_rows * D * 2 + mm * (D * 2 + qkv_rows * 2),
        "gemm_o": D * Hd * 2 + mm * (Hd * 2 + 2 * D * 4),
        "gemm_gate_up": 2 * F * D * 2 + mm * (D * 2 + F * 2),
        "gemm_down": D * F * 2 + mm * (F * 2 + 2 * D * 4),
        "lm_head": V * D * 2 + mm * D * 2,
        "attention": shape.n_kv_heads * shape.head_dim * 2 * 2 * (n_mean + K) + mm * Hd * 2 * 2,
        # persistent kernel: one whole forward (draft or verify) per launch, two per step
        "forward": bytes_total / Ksteps / 2.0,
    }
    for name, b in algo.items():
        if name in kernels:
            avg_ms = kernels[name]["ms_per_step"] / kernels[name]["launches_per_step"]
            kernels[name]["bytes_per_launch"] = b
            kernels[name]["gbs"] = b / (avg_ms * 1e-3) / 1e9
    dom = max((k for k in kernels if k in algo), key=lambda k: kernels[k]["ms_per_step"])
    roof = {"kernel": dom, "bound": "hbm", "achieved": round(kernels[dom]["gbs"], 1), "peak": hbm_peak,
            "unit": "GB/s", "frac": round(kernels[dom]["gbs"] / hbm_peak, 4),
            "traffic": captured_traffic(dom, kernels[dom].get("bytes_per_launch")), "peak_source": peak_src}

    # ---- end to end through the public API: pinned host inputs/outputs every step ------------
    reset()
    run_steps(0, W)
    torch.cuda.synchronize(dev)
    h_planted = torch.from_numpy(planted).pin_memory()
    h_acc = torch.zeros((total_steps, B), dtype=torch.int32).pin_memory()
    h_com = torch.zeros((total_steps, B, K + 1), dtype=torch.int32).pin_memory()
    d_in = i32(B, K)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    e0.record()
    for t in range(W, total_steps):
        d_in.copy_(h_planted[t], non_blocking=True)
        m.decode_step(pending, K, d_in, acc_all[t], com_all[t])
        h_acc[t].copy_(acc_all[t], non_blocking=True)
        h_com[t].copy_(com_all[t], non_blocking=True)
    e1.record()
    torch.cuda.synchronize(dev)
    e2e_ms = rank_reduce(e0.elapsed_time(e1), "max", world, dev)
    raise_on_any_rank(None if np.array_equal(h_acc.numpy()[W:, 0], accepts[W:total_steps])
                      else "end-to-end pass: accept lengths differ from the planted schedule", world, dev)

    try:  # measured after the main line's numbers; a failure here must not cost the main line
        variants = measure_variants(m, orthrus, dev, wl, W, Ksteps, planted_dev, accepts, reset, pending, cap,
                                    rank)
    except RuntimeError as e:
        variants = {"variants_error": str(e)}

    res = {
        "variants": variants,
        "ms": ms, "tokens": tokens, "bytes": bytes_total, "roofline": roof, "kernels": kernels, "clocks": clocks,
        "launches": launches_per_step * Ksteps, "e2e_ms": e2e_ms,
        "h2d": B * K * 4, "d2h": B * 4 + B * (K + 1) * 4, "hbm_peak": hbm_peak, "tf_peak": tf_peak,
        "peak_src": peak_src, "t_gen": t_gen, "weights": w, "stream": stream, "accepts": acc,
        "mean_committed": float(np.mean(acc[W:] + 1)), "cap": cap, "n_mean": n0 + int(np.sum(acc[W:] + 1)) // 2,
        "ar_ms": ar_ms, "ar_tokens": ar_tokens,
    }
    return res


def measure_variants(m, orthrus, dev, wl, W, Ksteps, planted_dev, accepts, reset, pending, cap, rank):
    """Two decoding variants on the same model, timed with CUDA events after W warm-up steps:
    - the 2-step iterative draft (orthrus_decode_step_ex, draft_steps = 2) on the planted
      drafts of the main run (accept lengths must match the schedule);
    - sampling at T = 1 (orthrus_decode_step_sampled): drafts drawn from the draft view,
      rejection-sampling consensus with seeded uniforms; acceptance is whatever these
      random-weight views give. The per-kernel split of one sampled step comes from the
      library's event trace."""
    import torch

    shape, B, P, K = wl["shape"], wl["batch"], wl["prompt"], wl["K"]
    V = shape.vocab
    i32 = lambda *s: torch.zeros(s, dtype=torch.int32, device=dev)
    out = {}
    n = min(Ksteps, 24)
    acc, com = i32(W + n, B), i32(W + n, B, K + 1)
    reset()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for t in range(W + n):
        if t == W:
            e0.record()
        m.decode_step_ex(pending, K, 2, planted_dev[t], acc[t], com[t])
    e1.record()
    torch.cuda.synchronize(dev)
    if m.read_status() != 0 or not np.array_equal(acc.cpu().numpy()[:, 0], accepts[:W + n]):
        raise RuntimeError("2-step draft run: accept lengths differ from the planted schedule")
    ms = e0.elapsed_time(e1)
    tok = int(np.sum(accepts[W:W + n] + 1)) * B
    out["two_step_draft"] = {"value": round(tok / (ms * 1e-3), 2), "unit": "tok/s", "steps": n,
                             "ms_per_step": round(ms / n, 4), "forwards_per_step": 3,
                             "path": "orthrus_decode_step_ex(draft_steps=2), planted drafts"}

    # sampling at T = 1: at most (K + 1) tokens per step must fit the cache
    T = 1.0
    n = max(0, min(Ksteps, 24, (cap - P - K - 2) // (K + 1) - W))
    if n == 0:
        return out
    rng = np.random.default_rng(3000 + rank)
    ud = torch.from_numpy(rng.random((W + n, B, K), dtype=np.float32)).to(dev)
    ua = torch.from_numpy(rng.random((W + n, B, K), dtype=np.float32)).to(dev)
    uf = torch.from_numpy(rng.random((W + n, B), dtype=np.float32)).to(dev)
    dl = torch.empty((B, K, V), dtype=torch.float32, device=dev)
    vl = torch.empty((B, K + 1, V), dtype=torch.float32, device=dev)
    acc, com = i32(W + n, B), i32(W + n, B, K + 1)
    reset()
    for t in range(W + n):
        if t == W:
            e0.record()
        m.decode_step_sampled(pending, K, T, ud[t], ua[t], uf[t], dl, vl, acc[t], com[t])
    e1.record()
    torch.cuda.synchronize(dev)
    if m.read_status() != 0:
        raise RuntimeError(f"sampled run: device status {m.read_status()}")
    ms = e0.elapsed_time(e1)
    a = acc.cpu().numpy()[W:, :]
    tok = int(np.sum(a + 1))
    # per-kernel split of sampled steps (event trace, same steps replayed from the same state)
    reset()
    for t in range(W):
        m.decode_step_sampled(pending, K, T, ud[t], ua[t], uf[t], dl, vl, acc[t], com[t])
    n_tr = min(n, 4)
    n_ev = n_tr * 12 + 8
    events = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    for e in events:
        e.record()
    torch.cuda.synchronize(dev)
    handles = (C.c_void_p * n_ev)(*[e.cuda_event for e in events])
    kinds = (C.c_int32 * n_ev)()
    count = (C.c_int32 * 1)(0)
    m.trace(handles, kinds, count)
    for t in range(W, W + n_tr):
        m.decode_step_sampled(pending, K, T, ud[t], ua[t], uf[t], dl, vl, acc[t], com[t])
    m.trace(None, None, None)
    torch.cuda.synchronize(dev)
    split = {}
    for i in range(count[0] - 1):
        if kinds[i] == 11:
            continue
        name = orthrus.KIND_NAMES[kinds[i]]
        split[name] = split.get(name, 0.0) + events[i].elapsed_time(events[i + 1]) / n_tr
    out["sampled_t1"] = {"value": round(tok / (ms * 1e-3), 2), "unit": "tok/s", "steps": n, "temperature": T,
                         "ms_per_step": round(ms / n, 4), "mean_accept": round(float(np.mean(a)), 3),
                         "ms_per_step_by_kind": {k: round(v, 4) for k, v in split.items()},
                         "path": "orthrus_decode_step_sampled (draft view + draws, verify view, "
                                 "rejection-sampling consensus)",
                         "note": "acceptance of random-weight views, not of a trained draft module"}
    return out


# ---------------------------------------------------------------------------
# the oracle on the host cores
# ---------------------------------------------------------------------------
def oracle_step_time(shape, weights, K, planted_a, stream, n_ctx=16):
    """Time one oracle Orthrus step (draft K + verify K+1 + accept) with an n_ctx-token cache."""
    import torch

    from oracle import Oracle
    o = Oracle(shape, weights, capacity=n_ctx + K + 2)
    st = o.new_state()
    o.prefill(st, stream[:n_ctx])
    t0 = time.time()
    o.draft_block(st, K)
    drafts = [int(x) for x in stream[n_ctx + 1:n_ctx + 1 + K]]
    if planted_a < K:
        drafts[planted_a] = (drafts[planted_a] + 1) % shape.vocab
    g, _ = o.verify_block(st, drafts)
    o.accept_commit(st, drafts, g)
    return time.time() - t0, torch.get_num_threads()


def run_reference(args, wl):
    """The oracle as it stands, timed on the host cores. Each of the K timed steps is a
    bounded sample of one decode step: one (layer, draft+verify) unit of the
    Qwen3-8B-shaped model, round-robin over the 36 layers, or, every 37th step, the
    two LM heads; a full step's time is 36 x (mean layer unit) + (mean head unit)."""
    import torch

    from oracle import Oracle
    shape, K = wl["shape"], wl["K"]
    w = synth.make_weights(shape, 1, 2)
    n_ctx = 16
    prompt = synth.make_prompt(shape, n_ctx, 3)
    L = shape.n_layers
    V_slice = 128

    def layer_model(l):
        from dataclasses import replace
        s1 = replace(shape, n_layers=1, vocab=V_slice)
        wl1 = {"embed": w["embed"][:V_slice], "final_norm": w["final_norm"], "lm_head": w["lm_head"][:V_slice]}
        for k, v in w.items():
            if k.startswith(f"l{l}."):
                wl1["l0." + k.split(".", 1)[1]] = v
        return Oracle(s1, wl1, capacity=n_ctx + K + 2), s1

    def head_model():
        from dataclasses import replace
        s0 = replace(shape, n_layers=0)
        return Oracle(s0, {"embed": w["embed"], "final_norm": w["final_norm"], "lm_head": w["lm_head"]},
                      capacity=n_ctx + K + 2), s0

    def unit(t):
        if t % (L + 1) == L:
            o, s = head_model()
            ids = prompt
        else:
            o, s = layer_model(t % (L + 1))
            ids = [int(x) % V_slice for x in prompt]
        st = o.new_state()
        o.prefill(st, ids)
        t0 = time.time()
        o.draft_block(st, K)
        o.verify_block(st, [int(x) % s.vocab for x in range(1, K + 1)])
        return (t % (L + 1) == L), time.time() - t0

    for t in range(args.warmup):
        unit(t)
    layer_t, head_t = [], []
    t_start = time.time()
    for t in range(args.steps):
        is_head, dt = unit(t)
        (head_t if is_head else layer_t).append(dt)
    if not head_t:
        head_t.append(unit(L)[1])
    if not layer_t:
        layer_t.append(unit(0)[1])
    step_s = L * statistics.mean(layer_t) + statistics.mean(head_t)
    mean_committed = wl["mean_accept"] + 1.0
    value = mean_committed / step_s
    cores = torch.get_num_threads()
    sample = (f"{args.steps} timed units of the fp64 oracle: {len(layer_t)} single-layer draft+verify "
              f"units and {len(head_t)} LM-head units (draft K={K}, verify K+1, {n_ctx}-token cache); "
              f"full step = {L} x layer + head = {step_s:.2f} s; tok/s = (mean planted accept {wl['mean_accept']} "
              f"+ 1) / step")
    return {"metric": "committed_tokens_per_s", "value": round(value, 4), "unit": "tok/s", "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_s * 1e3, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "batch": wl["batch"], "prompt": wl["prompt"], "K": K},
            "cpu_baseline": {"value": round(value, 4), "unit": "tok/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "wall_s": round(time.time() - t_start, 1)}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="qwen3_8b_b1_k32")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    wl = WORKLOADS[args.workload]
    if args.steps is None:
        args.steps = wl["steps"]
    args.warmup = max(3, args.warmup)
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, wl)), flush=True)
        return

    import torch
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                             device_id=torch.device("cuda", local_rank))
    r = run_ours(args, wl, rank, world, local_rank)
    ms_per_step = r["ms"] / args.steps
    value = r["tokens"] / (r["ms"] * 1e-3)
    step_gbs = r["bytes"] / (r["ms"] * 1e-3) / 1e9
    line = {
        "metric": "committed_tokens_per_s", "value": round(value, 2), "unit": "tok/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": args.workload, "batch": wl["batch"], "prompt": wl["prompt"], "K": wl["K"],
                   "planted_mean_accept": wl["mean_accept"], "capacity": r["cap"],
                   "parallelism": "replicas" if world > 1 else "single",
                   "l2": "inputs larger than L2 (30.3 GB of weights streamed per step)"},
        "decode_step_hbm": {"achieved_gbs": round(step_gbs, 1), "peak_gbs": r["hbm_peak"],
                            "frac": round(step_gbs / r["hbm_peak"], 4), "algorithmic_bytes_per_step":
                                int(r["bytes"] / args.steps), "peak_source": r["peak_src"]},
        "tokens_per_step": round(r["mean_committed"], 3),
        "roofline": r["roofline"],
        "kernels": {k: {kk: (round(vv, 4) if isinstance(vv, float) else vv) for kk, vv in v.items()}
                    for k, v in r["kernels"].items()},
        "clocks": r["clocks"],
        "gpu_launches": r["launches"],
        "e2e": {"value": round(r["tokens"] / (r["e2e_ms"] * 1e-3), 2), "unit": "tok/s",
                "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"]},
    }
    if r["ar_tokens"] > 0:
        # plain greedy AR (one verify forward with K = 0 plus the commit per token) through the
        # same kernels, on the same model and prompt: the like-for-like baseline of the speedup
        ar_tps = r["ar_tokens"] / (r["ar_ms"] * 1e-3)
        line["ar_baseline"] = {"value": round(ar_tps, 2), "unit": "tok/s", "tokens": r["ar_tokens"],
                               "ms_per_token": round(r["ar_ms"] / r["ar_tokens"], 4),
                               "speedup": round(value / ar_tps, 3),
                               "path": "orthrus_verify_block(K=0) + orthrus_accept_commit per token"}
    line.update(r["variants"])  # the 2-step draft and sampling at T = 1, outside the timed region
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        t_cpu, cores = oracle_step_time(wl["shape"], r["weights"], wl["K"], int(round(wl["mean_accept"])),
                                        r["stream"])
        line["cpu_baseline"] = {
            "value": round(r["mean_committed"] / t_cpu, 4), "unit": "tok/s", "cores": cores, "kind": "oracle",
            "sample": (f"1 Orthrus step of the fp64 oracle (draft K={wl['K']} + verify + accept) at the full shape "
                       f"with a 16-token cache: {t_cpu:.1f} s; tok/s = mean committed tokens per step of the GPU "
                       f"run ({r['mean_committed']:.2f}) / that time")}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()

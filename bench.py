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
NOT_FORWARD_SOURCES = {"sampling.cuh", "policy.cuh"}


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
    # config 3 (the headline): batch 1, 512-token prompt, K = 32, planted accept mean 6
    "qwen3_8b_b1_k32": dict(shape=synth.QWEN3_8B, batch=1, prompt=512, gen=1024, K=32, mean_accept=6.0,
                            steps=147),
    # config 4: batch 16, cache lengths uniform in [1024, 8192], K = 32, planted accept mean 6
    "qwen3_8b_b16_ragged_k32": dict(shape=synth.QWEN3_8B, batch=16, lens=("uniform", 1024, 8192, 41), K=32,
                                    mean_accept=6.0, steps=20),
    # config 5: batch 4 at a 32768-token cache, K in {8, 16, 32, 64}, planted accept mean K / 5
    **{f"qwen3_8b_b4_32k_k{k}": dict(shape=synth.QWEN3_8B, batch=4, lens=("fixed", 32768), K=k,
                                     mean_accept=k / 5.0, steps=16) for k in (8, 16, 32, 64)},
    # config 5 with the block size chosen per step among {8, 16, 32, 64}
    "qwen3_8b_b4_32k_dynamic": dict(shape=synth.QWEN3_8B, batch=4, lens=("fixed", 32768), K=64, mean_accept=6.0,
                                    steps=24, runner="dynamic"),
    # config 2: block attention alone, Qwen3-8B attention shape, 4096 cached keys, K = 32
    "qwen3_8b_attn_n4096": dict(shape=synth.QWEN3_8B, batch=1, n=4096, K=32, mean_accept=6.0, steps=20,
                                runner="attention"),
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
def prompt_lengths(wl, rank):
    """Per-sequence prompt (= cache) lengths of a workload."""
    B = wl["batch"]
    if "lens" in wl:
        kind = wl["lens"][0]
        if kind == "uniform":
            _, lo, hi, seed = wl["lens"]
            g = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed + rank, spawn_key=(0x1E5,))))
            return [int(x) for x in g.integers(lo, hi + 1, size=B)]
        return [int(wl["lens"][1])] * B
    return [int(wl["prompt"])] * B


def step_flops(shape, B, K, n_list):
    """Algorithmic flops of one decode step (draft K rows + verify K + 1 rows per sequence):
    2 per weight and token row, plus q.K and P.V over the visible keys (4 H d per key)."""
    wbytes, _ = shape_bytes(shape)
    params = wbytes / 2
    H, d, L = shape.n_heads, shape.head_dim, shape.n_layers
    att = sum(4 * H * d * L * (K * (n + K) + sum(n + i + 1 for i in range(K + 1))) for n in n_list)
    return 2.0 * params * B * (2 * K + 1) + att


def greedy_streams(m, pending, n, dev):
    """The next n greedy tokens of every sequence from the current device state, by K = 0 steps
    (the verify view on the pending token, then its commit): [B][n], column 0 the pending token.
    Advances the cache lengths and pending tokens; callers restore them."""
    import torch
    B = pending.numel()
    sd = torch.zeros((n, B), dtype=torch.int32, device=dev)
    sd[0] = pending
    ar1 = torch.zeros((B, 1), dtype=torch.int32, device=dev)
    acc1 = torch.zeros((B,), dtype=torch.int32, device=dev)
    for j in range(1, n):
        m.verify_block(pending, None, 0, ar1)
        m.accept_commit(pending, None, ar1, 0, acc1, sd[j])
    if torch.device(dev).type == "cuda":
        torch.cuda.synchronize(dev)
    if m.read_status() != 0:
        raise RuntimeError(f"device status {m.read_status()} while building the greedy streams")
    return sd.cpu().numpy().T.copy()


def planted_step(m, pending, dev, stream, jpos, a_plan, K, V, rng, acc, com):
    """One untimed decode step on drafts planted from the greedy streams (accept lengths a_plan),
    read back on the host. The streams come from the K = 0 path; a verify block of more than 128
    token rows runs on the per-op kernels, whose sums run in another order, so at a near tie its
    argmax can leave the stream. The committed tokens then replace the stream there and the rest
    of every stream is rebuilt from the new state. Returns (drafts, accept lengths, committed ids,
    rebuilt); jpos advances by each sequence's committed count."""
    import torch
    B = len(jpos)
    d = np.stack([synth.planted_drafts(stream[b], jpos[b], int(a_plan[b]), K, V, rng)
                  for b in range(B)]).astype(np.int32)
    m.decode_step(pending, K, torch.from_numpy(d).to(dev), acc, com)
    a = acc.cpu().numpy().astype(np.int64)
    c = com.cpu().numpy()
    if m.read_status() != 0 or np.any(a < 0):
        raise RuntimeError(f"device status {m.read_status()} in a planted step")
    left = False
    for b in range(B):
        got = c[b, :a[b] + 1]
        if a[b] != a_plan[b] or not np.array_equal(got, stream[b, jpos[b] + 1:jpos[b] + a[b] + 2]):
            left = True
        stream[b, jpos[b] + 1:jpos[b] + a[b] + 2] = got
        jpos[b] += int(a[b]) + 1
    if left:
        lens0, pend0 = m.lens.clone(), pending.clone()
        # as many tokens as the longest cache has room for (a later rebuild extends the rest)
        n = min(stream.shape[1] - min(jpos), m.capacity - int(lens0.max()) - 2)
        fresh = greedy_streams(m, pending, n, dev)
        m.lens.copy_(lens0)
        pending.copy_(pend0)
        for b in range(B):
            w = min(n, stream.shape[1] - jpos[b])
            stream[b, jpos[b]:jpos[b] + w] = fresh[b, :w]
    return d, a, c, left


def run_ours(args, wl, rank, world, local_rank):
    import torch

    from shared_kv_draft_b200 import orthrus

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    shape, B, K = wl["shape"], wl["batch"], wl["K"]
    V = shape.vocab
    W, Ksteps = args.warmup, args.steps
    total_steps = W + Ksteps
    lens = prompt_lengths(wl, rank)

    # planted accept lengths per sequence: stratified draws of the capped geometric law, warm-up
    # and timed window separately, so the timed window commits the law's mean tokens per step
    accepts = np.stack([np.concatenate([
        synth.planted_accepts_stratified(W, wl["mean_accept"], K, seed=1000 + 37 * rank + b),
        synth.planted_accepts_stratified(Ksteps, wl["mean_accept"], K, seed=1100 + 37 * rank + b)])
        for b in range(B)], axis=1)  # [total_steps, B]
    need = 1 + int(np.max(np.sum(accepts + 1, axis=0))) + K + 2  # greedy tokens the schedule reads
    need += 4 * (K + 1)  # room for steps that leave the stream (see planted_step)
    n_var = min(Ksteps, 24) if B == 1 else 0  # the variants (batch 1) commit up to K + 1 per step
    cap = ((max(max(lens) + need + K + 2, max(lens) + (W + n_var) * (K + 1) + K + 2) + 127) // 128) * 128

    t0 = time.time()
    w = synth.make_weights(shape, 1, 2)
    t_gen = time.time() - t0
    m = orthrus.DeviceModel(shape, w, batch=B, capacity=cap, max_block=K, max_rows=max(B * (K + 1), 512),
                            device=dev)
    toks = np.zeros((B, max(lens)), dtype=np.int32)
    for b, n in enumerate(lens):
        toks[b, :n] = synth.make_prompt(shape, n, 3 + rank * 101 + b)
    tok = torch.from_numpy(toks).to(dev)
    i32 = lambda *s: torch.zeros(s, dtype=torch.int32, device=dev)
    pending = i32(B)
    # prefill (the step before the decode path), timed with CUDA events
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    p0.record()
    m.prefill(tok, lens, pending)
    p1.record()
    torch.cuda.synchronize(dev)
    prefill_ms = p0.elapsed_time(p1)
    if m.read_status() != 0:
        raise RuntimeError(f"device status {m.read_status()} after the prefill")

    # greedy AR streams on the GPU (verify with K = 0: B rows per forward); the timed run must
    # reproduce them (also the plain-AR baseline through the same kernel, timed with CUDA events)
    stream_dev = i32(need, B)
    ar1, acc1 = i32(B, 1), i32(B)
    stream_dev[0] = pending
    ar_e0, ar_e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ar_w = min(3, need - 1)
    for j in range(1, need):
        if j == ar_w + 1:
            ar_e0.record()
        m.verify_block(pending, None, 0, ar1)
        m.accept_commit(pending, None, ar1, 0, acc1, stream_dev[j])
    ar_e1.record()
    torch.cuda.synchronize(dev)
    ar_tokens = (need - 1 - ar_w) * B
    ar_ms = ar_e0.elapsed_time(ar_e1) if ar_tokens > 0 else float("nan")
    if m.read_status() != 0:
        raise RuntimeError(f"device status {m.read_status()} while building the greedy stream")
    stream = stream_dev.cpu().numpy().T.copy()  # [B, need]

    acc_all = i32(total_steps, B)
    com_all = i32(total_steps, B, K + 1)
    launches_per_step = m.launches_per_step(K)
    lens_dev = torch.tensor(lens, dtype=torch.int32, device=dev)
    pend0 = torch.from_numpy(stream[:, 0].astype(np.int32)).to(dev)

    def reset():
        m.lens.copy_(lens_dev)
        pending.copy_(pend0)

    # untimed rehearsal: plant every step's drafts from the greedy streams and check it on the host;
    # the timed runs replay the same drafts from the same state and must give the same results
    rng = np.random.default_rng(2000 + rank)
    planted = np.zeros((total_steps, B, K), dtype=np.int32)
    acc_ref = np.zeros((total_steps, B), dtype=np.int64)
    com_ref = np.zeros((total_steps, B, K + 1), dtype=np.int32)
    jpos, rebuilt = [0] * B, 0
    stream0 = stream[:, 0].copy()
    reset()
    for t in range(total_steps):
        if max(jpos) + K + 2 > stream.shape[1]:
            raise RuntimeError("the greedy streams are too short for the planted schedule")
        planted[t], acc_ref[t], com_ref[t], left = planted_step(m, pending, dev, stream, jpos, accepts[t], K, V, rng,
                                                                acc_all[t], com_all[t])
        rebuilt += int(left)
    planted_dev = torch.from_numpy(planted).to(dev)

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

    # ---- checks: accept lengths as planted, committed streams == greedy streams ---------------
    err = None
    acc = acc_all.cpu().numpy()
    com = com_all.cpu().numpy()
    if m.read_status() != 0:
        err = f"device status {m.read_status()} after the timed run"
    elif not np.array_equal(acc, acc_ref) or not np.array_equal(com, com_ref):
        err = "the timed steps differ from the rehearsal on the same drafts"
    else:
        for b in range(B):
            out = [int(stream0[b])]
            for t in range(total_steps):
                out.extend(int(x) for x in com[t, b, :max(acc[t, b], 0) + 1])
            if out != [int(x) for x in stream[b, :len(out)]]:
                err = f"committed stream of sequence {b} differs from its greedy stream"
                break
    raise_on_any_rank(err, world, dev)
    tokens = rank_reduce(int(np.sum(acc[W:] + 1)), "sum", world, dev)  # all ranks' committed tokens
    # algorithmic HBM bytes and flops of the timed steps
    wbytes, kvpos = shape_bytes(shape)
    n = [lens[b] + int(np.sum(acc[:W, b] + 1)) for b in range(B)]
    bytes_total, flops_total = 0, 0.0
    for t in range(W, total_steps):
        bytes_total += 2 * wbytes + kvpos * (2 * sum(n) + B * (2 * K + 1))
        flops_total += step_flops(shape, B, K, n)
        n = [n[b] + int(acc[t, b]) + 1 for b in range(B)]
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
    n_mean = [lens[b] + int(np.sum(acc[:W, b] + 1)) for b in range(B)]
    D, F = shape.d_model, shape.d_ff
    Hd = shape.n_heads * shape.head_dim
    qkv_rows = shape.qkv_rows
    mm = B * (2 * K + 1) / 2.0  # token rows of a launch, mean of the draft and verify launches
    kv_rows = sum(x + K for x in n_mean)
    # algorithmic (bytes, flops) of one launch, mean of the draft and verify launches. Activations
    # that feed a projection are read as two bf16 planes (hi, lo).
    algo = {
        "gemm_qkv": (qkv_rows * D * 2 + mm * (2 * D * 2 + qkv_rows * 2), 2 * mm * qkv_rows * D),
        "gemm_o": (D * Hd * 2 + mm * (2 * Hd * 2 + 2 * D * 4), 2 * mm * D * Hd),
        "gemm_gate_up": (2 * F * D * 2 + mm * (2 * D * 2 + 2 * F * 2), 2 * mm * 2 * F * D),
        "gemm_down": (D * F * 2 + mm * (2 * F * 2 + 2 * D * 4), 2 * mm * D * F),
        "lm_head": (V * D * 2 + mm * D * 2, 2 * mm * V * D),
        "attention": (shape.n_kv_heads * shape.head_dim * 2 * 2 * kv_rows + mm * Hd * 2 * 3,
                      4 * shape.n_heads * shape.head_dim * (K + 0.5) * kv_rows),
        # persistent kernel: one whole forward (draft or verify) per launch, two per step
        "forward": (bytes_total / Ksteps / 2.0, flops_total / Ksteps / 2.0),
    }
    for name, (b, f) in algo.items():
        if name in kernels:
            avg_s = kernels[name]["ms_per_step"] / kernels[name]["launches_per_step"] * 1e-3
            kernels[name]["bytes_per_launch"] = b
            kernels[name]["gbs"] = b / avg_s / 1e9
            kernels[name]["tflops"] = f / avg_s / 1e12
    dom = max((k for k in kernels if k in algo), key=lambda k: kernels[k]["ms_per_step"])
    b_dom, f_dom = algo[dom]
    tensor_bound = f_dom / (tf_peak * 1e12) > b_dom / (hbm_peak * 1e9)
    if tensor_bound:
        roof = {"kernel": dom, "bound": "tensor", "achieved": round(kernels[dom]["tflops"], 1), "peak": tf_peak,
                "unit": "TFLOP/s", "frac": round(kernels[dom]["tflops"] / tf_peak, 4), "traffic": None,
                "hbm_frac": round(kernels[dom]["gbs"] / hbm_peak, 4), "peak_source": peak_src}
    else:
        roof = {"kernel": dom, "bound": "hbm", "achieved": round(kernels[dom]["gbs"], 1), "peak": hbm_peak,
                "unit": "GB/s", "frac": round(kernels[dom]["gbs"] / hbm_peak, 4),
                "traffic": captured_traffic(dom, b_dom), "peak_source": peak_src}

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
    raise_on_any_rank(None if np.array_equal(h_acc.numpy()[W:], acc_ref[W:total_steps])
                      else "end-to-end pass: accept lengths differ from the planted schedule", world, dev)

    variants = {}
    if B == 1:
        try:  # measured after the main line's numbers; a failure here must not cost the main line
            variants = measure_variants(m, orthrus, dev, wl, W, Ksteps, planted_dev, acc_ref[:, 0], reset,
                                        pending, cap, rank)
        except RuntimeError as e:
            variants = {"variants_error": str(e)}

    # prefill: 2 flops per weight and prompt token (the LM head for each sequence's last row only)
    # plus causal attention; tensor-bound at hundreds of rows
    params = wbytes / 2
    lm = V * D
    H, d, L = shape.n_heads, shape.head_dim, shape.n_layers
    pf_flops = sum(2.0 * (params - lm) * x + 2.0 * lm + 2.0 * H * d * L * x * (x + 1) for x in lens)
    prefill = {"ms": round(prefill_ms, 3), "tokens": int(sum(lens)),
               "tok_per_s": round(sum(lens) / (prefill_ms * 1e-3), 1),
               "tflops": round(pf_flops / (prefill_ms * 1e-3) / 1e12, 1),
               "tensor_frac": round(pf_flops / (prefill_ms * 1e-3) / 1e12 / tf_peak, 4),
               "path": "orthrus_prefill: per-op kernels, causal chunks"}

    res = {
        "variants": variants, "prefill": prefill,
        "ms": ms, "tokens": tokens, "bytes": bytes_total, "flops": flops_total, "roofline": roof,
        "kernels": kernels, "clocks": clocks,
        "launches": launches_per_step * Ksteps, "e2e_ms": e2e_ms,
        "h2d": B * K * 4, "d2h": B * 4 + B * (K + 1) * 4, "hbm_peak": hbm_peak, "tf_peak": tf_peak,
        "peak_src": peak_src, "t_gen": t_gen, "weights": w, "stream": stream[0], "accepts": acc,
        "mean_committed": float(np.mean(acc[W:] + 1)), "cap": cap, "lens": lens, "rebuilt": rebuilt,
        "ar_ms": ar_ms, "ar_tokens": ar_tokens,
    }
    return res


def run_attention_bench(args, wl, rank, world, local_rank):
    """Config 2: block attention alone at the Qwen3-8B attention shape (32 q / 8 kv heads,
    head_dim 128), a 4096-key cache, K = 32 (draft, bidirectional block) and K + 1 = 33
    (verify, causal), batch 1, through orthrus_attention (the per-op kernel). A step is one
    pass over 36 distinct layer caches (N(0, 1) values, 600 MB together, far above L2), so
    every call streams its cache from HBM. Metric: HBM GB/s of the algorithmic bytes."""
    import torch

    from shared_kv_draft_b200 import orthrus
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    L, Hkv, G, d, n = 36, 8, 4, 128, wl["n"]
    H = Hkv * G
    cap = n + 64
    g = torch.Generator(device=dev)
    g.manual_seed(5 + rank)
    f16 = lambda *s: torch.randn(s, generator=g, device=dev).to(torch.bfloat16).to(torch.float16)
    kc, vc = f16(L, 1, Hkv, cap, d), f16(L, 1, Hkv, cap, d)
    hbm_peak, tf_peak, peak_src = load_peaks()
    lens = torch.tensor([n], dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    modes = {}
    W, Ks = args.warmup, args.steps
    sampler = None
    total_ms, total_bytes = 0.0, 0.0
    for mode, Q in ((0, wl["K"]), (1, wl["K"] + 1)):
        q = f16(L, 1, Hkv, Q * G, d)
        kb, vb = f16(L, 1, Hkv, Q, d), f16(L, 1, Hkv, Q, d)
        out = torch.empty((2, Q, H * d), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(orthrus.attention_workspace_bytes(1, Hkv, G, Q, d, cap), dtype=torch.uint8, device=dev)
        keys = n + Q
        call_bytes = Hkv * d * 2 * 2 * keys + Q * G * Hkv * d * 2 + 2 * Q * H * d * 2
        call_flops = 4.0 * H * d * Q * keys

        def one_pass():
            for l in range(L):
                orthrus.attention(q[l], kc[l], vc[l], kb[l], vb[l], lens, 1, Hkv, G, Q, d, cap, Q, mode, out, ws,
                                  status)
        for _ in range(W):
            one_pass()
        torch.cuda.synchronize(dev)
        if mode == 1:
            props = torch.cuda.get_device_properties(dev)
            gpu_uuid = getattr(props, "uuid", None)
            sampler = ClockSampler(f"GPU-{gpu_uuid}" if gpu_uuid else None)
            time.sleep(0.3)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(Ks):
            one_pass()
        e1.record()
        torch.cuda.synchronize(dev)
        eager_call = e0.elapsed_time(e1) / (Ks * L)
        # the 36 calls of a pass as one CUDA graph: each call's host work (five tensor maps, the
        # counter reset, the launch) is paid at capture, so the replay times the device work
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            one_pass()
        torch.cuda.current_stream(dev).wait_stream(side)
        with torch.cuda.graph(graph):
            one_pass()
        for _ in range(W):
            graph.replay()
        torch.cuda.synchronize(dev)
        e0.record()
        for _ in range(Ks):
            graph.replay()
        e1.record()
        torch.cuda.synchronize(dev)
        if int(status.item()) != 0:
            raise RuntimeError(f"attention status {int(status.item())}")
        ms = e0.elapsed_time(e1)
        per_call = ms / (Ks * L)
        modes["draft" if mode == 0 else "verify"] = {
            "Q": Q, "keys": keys, "us_per_call": round(per_call * 1e3, 3),
            "us_per_call_eager": round(eager_call * 1e3, 3), "bytes_per_call": call_bytes,
            "gbs": round(call_bytes / (per_call * 1e-3) / 1e9, 1),
            "hbm_frac": round(call_bytes / (per_call * 1e-3) / 1e9 / hbm_peak, 4),
            "tflops": round(call_flops / (per_call * 1e-3) / 1e12, 2)}
        total_ms += ms
        total_bytes += call_bytes * Ks * L
    clocks = sampler.stop() if sampler else None
    gbs = total_bytes / (total_ms * 1e-3) / 1e9
    return {"metric": "attention_hbm_gbs", "value": round(gbs, 1), "unit": "GB/s", "n_gpus": world,
            "steps": Ks, "warmup": W, "ms_per_step": round(total_ms / Ks, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
            "config": {"workload": args.workload, "layers_rotated": L, "cache_keys": n, "K": wl["K"],
                       "heads": H, "kv_heads": Hkv, "head_dim": d,
                       "l2": "36 distinct layer caches per step (600 MB), larger than L2",
                       "launch": "one CUDA graph per step: 36 orthrus_attention calls (counter reset + kernel)"},
            "modes": modes,
            "roofline": {"kernel": "attention", "bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_peak,
                         "unit": "GB/s", "frac": round(gbs / hbm_peak, 4), "traffic": None, "peak_source": peak_src},
            "clocks": clocks, "gpu_launches": 2 * Ks * L}


def run_dynamic_k(args, wl, rank, world, local_rank):
    """Config 5 with the block size chosen per step (news article, "Future Directions:
    Larger K and Higher Acceptance", item 1). Batch 4 at a 32768-token cache:
      1. each K of the sweep {8, 16, 32, 64} is timed on its own planted schedule (accept
         mean K / 5), which gives the step-time table and the sweep's tok/s;
      2. an acceptance process whose per-position rate alternates between a predictable
         phase (0.95) and an open-ended one (0.6), every 8 steps, is run with each fixed K
         and with the policy (orthrus_choose_block_size, fed every step by the host copy of
         the accept lengths), on the same seeded draws. Drafts are planted from each
         sequence's greedy stream (rebuilt where a verify block on the per-op kernels breaks a
         near tie differently, see planted_step); every timed run must reproduce its rehearsal."""
    import torch

    from shared_kv_draft_b200 import orthrus
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    shape, B = wl["shape"], wl["batch"]
    V = shape.vocab
    ks = [8, 16, 32, 64]
    Kmax = max(ks)
    n_dyn = args.steps
    W = args.warmup
    need = (W + n_dyn + 4) * (Kmax + 1) + Kmax + 3  # the sweep's warm-up steps, and room for rebuilt streams
    lens = prompt_lengths(wl, rank)
    cap = ((max(lens) + need + Kmax + 2 + 127) // 128) * 128
    w = synth.make_weights(shape, 1, 2)
    m = orthrus.DeviceModel(shape, w, batch=B, capacity=cap, max_block=Kmax, max_rows=max(B * (Kmax + 1), 512),
                            device=dev)
    toks = np.zeros((B, max(lens)), dtype=np.int32)
    for b, n in enumerate(lens):
        toks[b, :n] = synth.make_prompt(shape, n, 3 + rank * 101 + b)
    i32 = lambda *s: torch.zeros(s, dtype=torch.int32, device=dev)
    pending = i32(B)
    m.prefill(torch.from_numpy(toks).to(dev), lens, pending)
    stream = greedy_streams(m, pending, need, dev)
    lens_dev = torch.tensor(lens, dtype=torch.int32, device=dev)
    pend0 = torch.from_numpy(stream[:, 0].astype(np.int32)).to(dev)
    acc = i32(B)
    coms = {K: i32(B, K + 1) for K in ks}  # committed ids [B][K + 1], one buffer per block size

    def run(schedule, choose, n_steps, timed_from):
        """schedule(t, K, rng) -> accept lengths [B]; choose(stats) -> K. An untimed rehearsal plants
        every step's drafts (planted_step); the timed pass replays them from the same state, reading
        every step's accept lengths on the host for the policy, and must reproduce the rehearsal.
        Returns (ms of the steps from timed_from on, committed tokens there, Ks used)."""
        st = stream.copy()
        m.lens.copy_(lens_dev)
        pending.copy_(pend0)
        rng = np.random.default_rng(7000 + rank)
        stats = orthrus.accept_stats(B)
        jpos, rec = [0] * B, []
        for t in range(n_steps):
            K = choose(stats)
            a_plan = schedule(t, K, rng)
            if max(jpos) + K + 2 > st.shape[1]:
                raise RuntimeError("the greedy streams are too short for the planted schedule")
            d, a, _, _ = planted_step(m, pending, dev, st, jpos, a_plan, K, V, rng, acc, coms[K])
            orthrus.accept_stats_update(stats, a.tolist(), K, 0.7)
            rec.append((K, torch.from_numpy(d).to(dev), a))
        m.lens.copy_(lens_dev)
        pending.copy_(pend0)
        stats = orthrus.accept_stats(B)
        used, tokens = [], 0
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        for t in range(n_steps):
            if t == timed_from:
                torch.cuda.synchronize(dev)
                e0.record()
            K = choose(stats)
            if K != rec[t][0]:
                raise RuntimeError(f"step {t}: the policy chose K = {K}, the rehearsal {rec[t][0]}")
            m.decode_step(pending, K, rec[t][1], acc, coms[K])
            a = acc.cpu().numpy()  # the policy reads every step's accept lengths on the host
            if not np.array_equal(a, rec[t][2]):
                raise RuntimeError(f"step {t}, K = {K}: accept lengths {a} differ from the rehearsal {rec[t][2]}")
            orthrus.accept_stats_update(stats, a.tolist(), K, 0.7)
            if t >= timed_from:
                tokens += int(np.sum(a + 1))
                used.append(K)
        e1.record()
        torch.cuda.synchronize(dev)
        if m.read_status() != 0:
            raise RuntimeError(f"device status {m.read_status()}")
        return e0.elapsed_time(e1), tokens, used

    # 1. the sweep: step time and tok/s of each K on its own planted schedule (accept mean K / 5)
    sweep, step_ms = {}, []
    for K in ks:
        mean = K / 5.0
        per = [synth.planted_accepts_stratified(W + n_dyn, mean, K, seed=900 + b) for b in range(B)]
        ms, tok, _ = run(lambda t, K_, rng, per=per: np.array([per[b][t] for b in range(B)]), lambda s, K=K: K,
                         W + n_dyn, W)
        sweep[f"k{K}"] = {"ms_per_step": round(ms / n_dyn, 3), "tok_per_s": round(tok / (ms * 1e-3), 1),
                          "planted_mean_accept": mean}
        step_ms.append(ms / n_dyn)

    # 2. phases of certainty: each fixed K and the policy on the same seeded draws
    def phase_alpha(t):
        return 0.95 if (t // 8) % 2 == 0 else 0.6

    def trunc_geometric(t, K, rng):
        al = phase_alpha(t)
        u = rng.random((B, Kmax))
        out = np.zeros(B, dtype=np.int64)
        for b in range(B):
            a = 0
            while a < K and u[b, a] < al:
                a += 1
            out[b] = a
        return out

    fixed = {}
    for K in ks:
        ms, tok, _ = run(trunc_geometric, lambda s, K=K: K, n_dyn, 0)
        fixed[f"k{K}"] = round(tok / (ms * 1e-3), 1)
    ms, tok, used = run(trunc_geometric, lambda s: orthrus.choose_block_size(s, ks, step_ms), n_dyn, 0)
    dyn = tok / (ms * 1e-3)
    by_phase = {}
    for t, K in enumerate(used):
        by_phase.setdefault(str(phase_alpha(t)), []).append(K)
    best_fixed = max(fixed.values())
    return {"metric": "committed_tokens_per_s", "value": round(dyn, 2), "unit": "tok/s", "n_gpus": world,
            "steps": n_dyn, "warmup": W, "ms_per_step": round(ms / n_dyn, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": args.workload, "batch": B, "cache": lens[0], "K_options": ks,
                       "acceptance": "per-position rate 0.95 and 0.6 in alternating phases of 8 steps",
                       "policy": "orthrus_choose_block_size, decay 0.7, step times from the sweep"},
            "k_sweep": sweep, "fixed_k_same_schedule": fixed,
            "dynamic_vs_best_fixed": round(dyn / best_fixed, 4),
            "chosen_k_by_phase_rate": {k: round(float(np.mean(v)), 2) for k, v in by_phase.items()},
            "gpu_launches": 2 * n_dyn}


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
    n = max(0, min(Ksteps, 24, (cap - P - K - 2) // (K + 1) - W))  # the capacity is sized for 24 steps
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


def cpu_model():
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


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
    mean_committed = synth.capped_geometric_mean(wl["mean_accept"], K) + 1.0
    value = mean_committed / step_s
    unit_ms = 1e3 * (sum(layer_t) + sum(head_t)) / args.steps  # what each timed step actually took
    cores = torch.get_num_threads()
    sample = (f"{args.steps} timed units of the fp64 oracle: {len(layer_t)} single-layer draft+verify "
              f"units and {len(head_t)} LM-head units (draft K={K}, verify K+1, {n_ctx}-token cache); "
              f"full step scaled from the units = {L} x layer + head = {step_s:.2f} s; tok/s = expected "
              f"committed tokens per step ({mean_committed:.3f}) / scaled step")
    return {"metric": "committed_tokens_per_s", "value": round(value, 4), "unit": "tok/s", "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(unit_ms, 1),
            "ms_per_step_is": "mean time of one timed unit (a bounded sample of a step), not of a full step",
            "full_step_ms_scaled": round(step_s * 1e3, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "batch": wl["batch"], "prompt": wl.get("prompt"), "K": K},
            "cpu_baseline": {"value": round(value, 4), "unit": "tok/s", "cores": cores, "kind": "oracle",
                             "cpu_model": cpu_model(), "sample": sample},
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
    if wl.get("runner") in ("attention", "dynamic"):
        fn = run_attention_bench if wl["runner"] == "attention" else run_dynamic_k
        line = fn(args, wl, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(line), flush=True)
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    r = run_ours(args, wl, rank, world, local_rank)
    ms_per_step = r["ms"] / args.steps
    value = r["tokens"] / (r["ms"] * 1e-3)
    step_gbs = r["bytes"] / (r["ms"] * 1e-3) / 1e9
    line = {
        "metric": "committed_tokens_per_s", "value": round(value, 2), "unit": "tok/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": args.workload, "batch": wl["batch"],
                   "prompt": wl["prompt"] if "prompt" in wl else f"{min(r['lens'])}..{max(r['lens'])} tokens",
                   "K": wl["K"], "planted_mean_accept": wl["mean_accept"], "capacity": r["cap"],
                   "planted_schedule": "stratified quantiles of the capped geometric law, seeded order",
                   "streams_rebuilt": r["rebuilt"],
                   "tokens_per_step_expected": round(synth.capped_geometric_mean(wl["mean_accept"], wl["K"]) + 1, 4),
                   "parallelism": "replicas" if world > 1 else "single",
                   "l2": "inputs larger than L2 (30.3 GB of weights streamed per step)"},
        "decode_step_hbm": {"achieved_gbs": round(step_gbs, 1), "peak_gbs": r["hbm_peak"],
                            "frac": round(step_gbs / r["hbm_peak"], 4), "algorithmic_bytes_per_step":
                                int(r["bytes"] / args.steps), "peak_source": r["peak_src"]},
        "tokens_per_step": round(r["mean_committed"] * wl["batch"], 3),
        "decode_step_tensor": {"achieved_tflops": round(r["flops"] / (r["ms"] * 1e-3) / 1e12, 1),
                               "peak_tflops": r["tf_peak"],
                               "frac": round(r["flops"] / (r["ms"] * 1e-3) / 1e12 / r["tf_peak"], 4),
                               "note": "algorithmic flops; the layer projections run on both activation planes "
                                       "(hi and lo rows in one MMA), twice these flops on the tensor pipe"},
        "prefill": r["prefill"],
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
            "cpu_model": cpu_model(),
            "sample": (f"1 Orthrus step of the fp64 oracle (draft K={wl['K']} + verify + accept) at the full shape "
                       f"with a 16-token cache: {t_cpu:.1f} s; tok/s = mean committed tokens per step of the GPU "
                       f"run ({r['mean_committed']:.2f}) / that time")}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()

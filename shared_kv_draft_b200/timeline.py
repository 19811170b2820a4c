"""Phase timeline of the persistent forward kernel (profiling tool).

    python -m shared_kv_draft_b200.timeline [--layers L] [--K 32] [--prompt 512] [--capacity 1792] [--reps 3]

Builds a Qwen3-8B-shaped model (optionally with fewer layers) with seeded N(0, 0.02) bf16 weights drawn on the
device, prefills a seeded uniform prompt, times the draft and verify forwards with CUDA events, and then runs one
draft and one verify forward with the orthrus_timeline hook. For every phase kind it prints:
- the mean time from the previous phase's end to this phase's end (max over CTAs);
- the streaming part (first activation load to last MMA issued);
- the tail (last MMA to the phase's last completion).
Everything runs in the library's kernels; this script only allocates and reads the timestamps.
"""
from __future__ import annotations

import argparse
import dataclasses
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402
from shared_kv_draft_b200 import orthrus  # noqa: E402

EVENTS = 16  # timestamps per (CTA, phase), see orthrus_timeline in include/orthrus.h
KINDS = ["QKV", "ATTN", "COMBINE", "O", "GU", "DOWN"]


def device_weights(shape, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    w = {}
    for name, dims, kind in synth.tensor_specs(shape):
        if kind == "gain":
            w[name] = torch.ones(dims, dtype=torch.float32, device="cuda")
        else:
            w[name] = (torch.randn(dims, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    return w


def phase_names(L):
    names = ["EMBED"] + [f"{k}{l}" for l in range(L) for k in KINDS] + ["LM"]
    return names


def summarize(raw, L, sms, weight_bytes):
    nph = 2 + 6 * L
    t = raw.reshape(sms, nph, EVENTS)[:, :, :8].astype(np.float64)
    valid = t > 0
    t = np.where(valid, (t - t[valid].min()) / 1000.0, np.nan)  # microseconds
    names = phase_names(L)
    ends = np.full(nph, np.nan)
    for p in range(nph):
        col = t[:, p, 7]
        if np.any(~np.isnan(col)):
            ends[p] = np.nanmax(col)
    rows = {}
    prev = ends[0] if not np.isnan(ends[0]) else np.nanmin(t)
    for p in range(1, nph):
        if np.isnan(ends[p]):
            continue
        kind = names[p].rstrip("0123456789")
        x0 = np.nanmin(t[:, p, 2]) if np.any(~np.isnan(t[:, p, 2])) else np.nan
        m1 = np.nanmax(t[:, p, 5]) if np.any(~np.isnan(t[:, p, 5])) else np.nan
        r = rows.setdefault(kind, {"phase": [], "stream": [], "tail": []})
        r["phase"].append(ends[p] - prev)
        if not np.isnan(x0):
            r["stream"].append(m1 - x0)
            r["tail"].append(ends[p] - m1)
        prev = ends[p]
    span = np.nanmax(t)
    lines = [f"  span {span:.1f} us"]
    for kind, r in rows.items():
        s = f"  {kind:8s} n={len(r['phase']):3d}  phase {np.mean(r['phase']):7.1f} us"
        if r["stream"]:
            s += f"  stream {np.mean(r['stream']):6.1f} us  tail {np.mean(r['tail']):6.1f} us"
            if kind in weight_bytes:
                s += f"  ({weight_bytes[kind] / (np.mean(r['stream']) * 1e-6) / 1e12:.2f} TB/s while streaming)"
        lines.append(s)
    return "\n".join(lines)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--layers", type=int, default=36)
    ap.add_argument("--K", type=int, default=32)
    ap.add_argument("--prompt", type=int, default=512)
    ap.add_argument("--capacity", type=int, default=1792)
    ap.add_argument("--reps", type=int, default=3)
    args = ap.parse_args()
    shape = dataclasses.replace(synth.QWEN3_8B, n_layers=args.layers)
    K = args.K
    w = device_weights(shape, 1)
    dev = orthrus.DeviceModel(shape, w, batch=1, capacity=args.capacity, max_block=K, max_rows=max(K + 1, 512))
    g = torch.Generator(device="cuda")
    g.manual_seed(3)
    prompt = torch.randint(0, shape.vocab, (1, args.prompt), generator=g, device="cuda", dtype=torch.int32)
    pend = torch.zeros(1, dtype=torch.int32, device="cuda")
    dev.prefill(prompt, [args.prompt], pend)
    draft = torch.zeros(1, K, dtype=torch.int32, device="cuda")
    ar = torch.zeros(1, K + 1, dtype=torch.int32, device="cuda")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(args.reps):
        e0.record()
        dev.draft_block(pend, K, draft)
        e1.record()
        torch.cuda.synchronize()
        td = e0.elapsed_time(e1)
        e0.record()
        dev.verify_block(pend, draft, K, ar)
        e1.record()
        torch.cuda.synchronize()
        print(f"draft forward {td:.3f} ms   verify forward {e0.elapsed_time(e1):.3f} ms", flush=True)
    D, H, Hkv, d, F, V = shape.d_model, shape.n_heads, shape.n_kv_heads, shape.head_dim, shape.d_ff, shape.vocab
    wb = {"QKV": (H + 2 * Hkv) * d * D * 2, "O": D * H * d * 2, "GU": 2 * F * D * 2, "DOWN": D * F * 2, "LM": V * D * 2}
    buf = torch.zeros(dev.timeline_bytes() // 8, dtype=torch.int64, device="cuda")
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for view in ("draft", "verify"):
        buf.zero_()
        dev.timeline(buf)
        if view == "draft":
            dev.draft_block(pend, K, draft)
        else:
            dev.verify_block(pend, draft, K, ar)
        torch.cuda.synchronize()
        dev.timeline(None)
        print(f"{view} view (status {dev.read_status()}):")
        print(summarize(buf.cpu().numpy(), shape.n_layers, sms, wb))


if __name__ == "__main__":
    main()

"""GPU parity of the single kernels, called through the C ABI, against the oracle.

* GEMM (tcgen05, stream-K, fp32 store epilogue) vs the oracle's float64
  product of the same bf16 operands: fp32 accumulation over Kd terms bounds
  the error far below the stated tolerance.
* Block attention, draft (bidirectional block) and verify (causal) modes, vs
  the oracle's row-by-row softmax attention: relative L2 <= 1e-2 per sequence.
  Covers ragged cache lengths, tile and chunk boundaries, an empty cache, one
  query, two row tiles (Q*G > 128), every supported group size, both head
  dims, NaN-poisoned cache rows past the live range, and the Qwen3-8B-shaped
  attention microbenchmark (4096 cached keys, K = 32).
"""
import numpy as np
import pytest
import torch

import synth
from oracle import attention as oracle_attention
from oracle import linear as oracle_linear

pytestmark = pytest.mark.gpu


def lib():
    from shared_kv_draft_b200 import orthrus
    return orthrus


def bf16_tensor(shape, seed, std=1.0):
    bits = synth.normal_bf16(shape, seed, std)
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)


@pytest.mark.parametrize("M,N,Kd", [(1, 128, 64), (9, 256, 256), (16, 512, 768), (33, 512, 4096), (48, 1024, 512),
                                    (130, 384, 256), (300, 256, 1024), (33, 6144, 4096), (528, 256, 512)])
def test_linear_matches_oracle(M, N, Kd):
    o = lib()
    X = bf16_tensor((M, Kd), M * 7 + Kd)
    W = bf16_tensor((N, Kd), N * 13 + Kd, std=0.05)
    ref = oracle_linear(X.to(torch.float64), W, rowwise=False).numpy()
    Y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(o.linear_workspace_bytes(M, N, Kd), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o.linear(X.cuda(), W.cuda(), Y, ws, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    got = Y.cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    err = np.abs(got - ref).max()
    assert err <= 1e-5 * np.sqrt(Kd) * max(1.0, np.abs(ref).max()), err
    # a second call reuses the zeroed tile counters and gives identical bits
    Y2 = torch.empty_like(Y)
    o.linear(X.cuda(), W.cuda(), Y2, ws, status)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y2)


def run_attention(B, Hkv, G, Q, d, cap, lens, mode, seed, poison=False, blk_stride=None):
    """Block attention through orthrus_attention against the oracle. q, K and V are bf16
    values (N(0, 1) from a seed); the kernel takes them in the fp16 encoding, which holds
    every such value of magnitude >= 2^-17 exactly, and writes the output as two bf16
    planes (hi, lo) whose sum is compared."""
    o = lib()
    H = Hkv * G
    blk_stride = blk_stride or Q
    q = bf16_tensor((B, Hkv, Q * G, d), seed)
    kc = bf16_tensor((B, Hkv, cap, d), seed + 1)
    vc = bf16_tensor((B, Hkv, cap, d), seed + 2)
    kb = bf16_tensor((B, Hkv, blk_stride, d), seed + 3)
    vb = bf16_tensor((B, Hkv, blk_stride, d), seed + 4)
    if poison:
        nan = torch.tensor(float("nan")).to(torch.bfloat16)
        for b in range(B):
            live = lens[b] + (Q if mode == 1 else 0)
            kc[b, :, live:] = nan
            vc[b, :, live:] = nan
            kb[b, :, Q:] = nan
            vb[b, :, Q:] = nan
    f16 = lambda t: t.to(torch.float16).cuda()
    out = torch.full((2, B, Q, H * d), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(o.attention_workspace_bytes(B, Hkv, G, Q, d, cap), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ln = torch.tensor(lens, dtype=torch.int32, device="cuda")
    o.attention(f16(q), f16(kc), f16(vc), f16(kb), f16(vb), ln, B, Hkv, G, Q, d, cap, blk_stride, mode, out,
                ws, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    got = (out[0].double() + out[1].double()).cpu().numpy()
    for b in range(B):
        n = lens[b]
        qo = q[b].to(torch.float64).reshape(Hkv, Q, G, d).permute(1, 0, 2, 3).reshape(Q, H, d)
        if mode == 0:
            keys = torch.cat([kc[b, :, :n], kb[b, :, :Q]], dim=1).to(torch.float64)
            vals = torch.cat([vc[b, :, :n], vb[b, :, :Q]], dim=1).to(torch.float64)
            nv = [n + Q] * Q
        else:
            keys = kc[b, :, :n + Q].to(torch.float64)
            vals = vc[b, :, :n + Q].to(torch.float64)
            nv = [n + i + 1 for i in range(Q)]
        ref = oracle_attention(qo, keys, vals, nv).numpy()
        g = got[b]
        assert np.isfinite(g).all(), f"non-finite output for sequence {b}"
        rel = np.linalg.norm(g - ref) / np.linalg.norm(ref)
        assert rel <= 1e-2, (b, rel)
    return got


@pytest.mark.parametrize("mode", [0, 1], ids=["draft", "verify"])
@pytest.mark.parametrize("n", [0, 1, 100, 127, 128, 129, 300])
def test_attention_lengths(mode, n):
    run_attention(1, 2, 4, 8, 128, 512, [n], mode, seed=11 + n)


@pytest.mark.parametrize("mode", [0, 1], ids=["draft", "verify"])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_attention_groups(mode, G):
    run_attention(2, 2, G, 8, 64, 384, [37, 250], mode, seed=100 + G)


@pytest.mark.parametrize("mode", [0, 1], ids=["draft", "verify"])
def test_attention_single_query(mode):
    run_attention(1, 4, 4, 1, 128, 256, [200], mode, seed=5)


def test_attention_two_row_tiles_verify():
    # Q*G = 132 rows: the last block position falls into a second 128-row tile
    run_attention(1, 2, 4, 33, 128, 1024, [700], 1, seed=6)


def test_attention_two_row_tiles_draft():
    run_attention(1, 2, 4, 64, 128, 1024, [513], 0, seed=7)


@pytest.mark.parametrize("mode", [0, 1], ids=["draft", "verify"])
def test_attention_ragged_batch_many_chunks(mode):
    run_attention(3, 2, 4, 8, 128, 4096, [3000, 17, 1029], mode, seed=8)


@pytest.mark.parametrize("mode", [0, 1], ids=["draft", "verify"])
def test_attention_ignores_poisoned_rows(mode):
    run_attention(2, 2, 4, 8, 128, 640, [130, 257], mode, seed=9, poison=True, blk_stride=16)


@pytest.mark.parametrize("mode,Q", [(0, 32), (1, 33)], ids=["draft", "verify"])
def test_attention_qwen_microbench_shape(mode, Q):
    # one layer at the Qwen3-8B attention shape: 32 q / 8 kv heads, d = 128, 4096 cached keys
    run_attention(1, 8, 4, Q, 128, 4096 + 64, [4096], mode, seed=12)

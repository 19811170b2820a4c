"""Pins for the oracle's building blocks against definitions written independently
(pure-Python loops, complex arithmetic) and against closed-form properties."""
import cmath
import math

import numpy as np
import pytest
import torch

from oracle import attention, attention_by_head, linear, rms_norm, rope, silu

F64 = torch.float64


def brute_attention(q, keys, vals, n_visible):
    """Triple loop with an explicit max-subtracted softmax; q [Q][H][d], keys [Hkv][N][d]."""
    Q, H, d = len(q), len(q[0]), len(q[0][0])
    Hkv = len(keys)
    G = H // Hkv
    out = []
    for i in range(Q):
        row = []
        for h in range(H):
            kv = h // G
            s = [sum(q[i][h][t] * keys[kv][j][t] for t in range(d)) / math.sqrt(d) for j in range(n_visible[i])]
            m = max(s)
            e = [math.exp(x - m) for x in s]
            z = sum(e)
            row.extend(sum(e[j] / z * vals[kv][j][t] for j in range(len(e))) for t in range(d))
        out.append(row)
    return out


ATTENTION_FORMS = [attention, attention_by_head]


@pytest.mark.parametrize("attention", ATTENTION_FORMS, ids=["by_row", "by_head"])
@pytest.mark.parametrize("H,Hkv", [(1, 1), (2, 1), (4, 2), (4, 1), (2, 2)])
@pytest.mark.parametrize("mode", ["all", "causal"])
def test_attention_matches_brute_force(H, Hkv, mode, attention):
    rng = np.random.default_rng(H * 10 + Hkv)
    d, n, Q = 4, 5, 3
    q = rng.standard_normal((Q, H, d))
    keys = rng.standard_normal((Hkv, n + Q, d))
    vals = rng.standard_normal((Hkv, n + Q, d))
    nv = [n + Q] * Q if mode == "all" else [n + i + 1 for i in range(Q)]
    got = attention(torch.tensor(q), torch.tensor(keys), torch.tensor(vals), nv).numpy()
    ref = np.array(brute_attention(q.tolist(), keys.tolist(), vals.tolist(), nv))
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("attention", ATTENTION_FORMS, ids=["by_row", "by_head"])
def test_attention_special_cases(attention):
    rng = np.random.default_rng(5)
    d = 8
    q = torch.tensor(rng.standard_normal((1, 2, d)))
    k = torch.tensor(rng.standard_normal((1, 1, d)))
    v = torch.tensor(rng.standard_normal((1, 1, d)))
    # a single visible key returns its value
    out = attention(q, k, v, [1]).reshape(2, d)
    np.testing.assert_allclose(out[0].numpy(), v[0, 0].numpy(), rtol=1e-14)
    np.testing.assert_allclose(out[1].numpy(), v[0, 0].numpy(), rtol=1e-14)
    # identical keys give the mean of the values
    k2 = k.repeat(1, 6, 1)
    v2 = torch.tensor(rng.standard_normal((1, 6, d)))
    out = attention(q, k2, v2, [6]).reshape(2, d)
    np.testing.assert_allclose(out[0].numpy(), v2[0].mean(0).numpy(), rtol=1e-12)
    # keys beyond n_visible are ignored, whatever they hold
    k3 = torch.tensor(rng.standard_normal((1, 4, d)))
    v3 = torch.tensor(rng.standard_normal((1, 4, d)))
    a = attention(q, k3, v3, [2])
    k3[:, 2:] = float("nan")
    v3[:, 2:] = float("nan")
    b = attention(q, k3, v3, [2])
    assert torch.equal(a, b)


@pytest.mark.parametrize("attention", ATTENTION_FORMS, ids=["by_row", "by_head"])
def test_gqa_group_reads_its_kv_head(attention):
    # G = 2: query heads 0,1 read kv head 0, heads 2,3 read kv head 1
    rng = np.random.default_rng(9)
    q = torch.tensor(rng.standard_normal((2, 4, 4)))
    k = torch.tensor(rng.standard_normal((2, 3, 4)))
    v = torch.tensor(rng.standard_normal((2, 3, 4)))
    full = attention(q, k, v, [3, 3]).reshape(2, 4, 4)
    for h in range(4):
        single = attention(q[:, h:h + 1], k[h // 2:h // 2 + 1], v[h // 2:h // 2 + 1], [3, 3])
        np.testing.assert_allclose(full[:, h].numpy(), single.numpy(), rtol=1e-14)


def test_rmsnorm_definition():
    rng = np.random.default_rng(1)
    x = rng.standard_normal(7)
    g = rng.standard_normal(7)
    eps = 1e-6
    ms = sum(t * t for t in x) / len(x)
    ref = [x[i] / math.sqrt(ms + eps) * g[i] for i in range(7)]
    np.testing.assert_allclose(rms_norm(torch.tensor(x), torch.tensor(g), eps).numpy(), ref, rtol=1e-13)
    # a constant vector c maps to sign(c) * gain (up to eps)
    c = torch.full((16,), -3.0, dtype=F64)
    out = rms_norm(c, torch.ones(16, dtype=F64), 1e-6)
    np.testing.assert_allclose(out.numpy(), -1.0, rtol=1e-6)
    # scale invariance
    np.testing.assert_allclose(rms_norm(torch.tensor(x) * 100, torch.tensor(g), 0.0).numpy(),
                               rms_norm(torch.tensor(x), torch.tensor(g), 0.0).numpy(), rtol=1e-13)


def test_silu_definition():
    xs = [-5.0, -1.0, 0.0, 0.5, 3.0]
    ref = [x / (1.0 + math.exp(-x)) for x in xs]
    np.testing.assert_allclose(silu(torch.tensor(xs, dtype=F64)).numpy(), ref, rtol=1e-14)
    assert float(silu(torch.tensor(0.0, dtype=F64))) == 0.0
    x = torch.tensor(xs, dtype=F64)
    np.testing.assert_allclose((silu(x) - silu(-x)).numpy(), x.numpy(), rtol=1e-13)


def test_rope_matches_complex_rotation():
    rng = np.random.default_rng(2)
    d, theta = 8, 10000.0
    x = rng.standard_normal((3, 2, d))
    pos = [0, 5, 1234]
    got = rope(torch.tensor(x), torch.tensor(pos), theta).numpy()
    for i, p in enumerate(pos):
        for h in range(2):
            for j in range(d // 2):
                z = complex(x[i, h, j], x[i, h, j + d // 2]) * cmath.exp(1j * p * theta ** (-2.0 * j / d))
                assert abs(got[i, h, j] - z.real) < 1e-12
                assert abs(got[i, h, j + d // 2] - z.imag) < 1e-12


def test_rope_properties():
    rng = np.random.default_rng(3)
    d, theta = 16, 1e6
    q = torch.tensor(rng.standard_normal((1, 1, d)))
    k = torch.tensor(rng.standard_normal((1, 1, d)))
    # position 0 is the identity and rotation preserves the norm
    assert torch.allclose(rope(q, torch.tensor([0]), theta), q, rtol=0, atol=0)
    assert abs(float(rope(q, torch.tensor([77]), theta).norm() - q.norm())) < 1e-12
    # q(p) . k(p') depends only on p - p'
    def dot(p, pp):
        return float((rope(q, torch.tensor([p]), theta) * rope(k, torch.tensor([pp]), theta)).sum())
    assert abs(dot(10, 3) - dot(107, 100)) < 1e-10
    assert abs(dot(3, 10) - dot(1000, 1007)) < 1e-10


def test_linear_orientation():
    # y = W x with W [out, in], checked with loops on a non-square W (a transposed operand fails)
    rng = np.random.default_rng(4)
    W = rng.standard_normal((3, 5)).astype(np.float32)
    x = rng.standard_normal((2, 5))
    wb = torch.tensor(W).to(torch.bfloat16)
    Wv = wb.to(F64).numpy()
    ref = [[sum(Wv[o][i] * x[r][i] for i in range(5)) for o in range(3)] for r in range(2)]
    for rowwise in (False, True):
        np.testing.assert_allclose(linear(torch.tensor(x), wb, rowwise).numpy(), ref, rtol=1e-12)


def test_attention_forms_agree_on_long_ragged_rows():
    rng = np.random.default_rng(21)
    Q, H, Hkv, d, n = 9, 8, 2, 16, 700
    q = torch.tensor(rng.standard_normal((Q, H, d)))
    keys = torch.tensor(rng.standard_normal((Hkv, n + Q, d)))
    vals = torch.tensor(rng.standard_normal((Hkv, n + Q, d)))
    nv = [n + i + 1 for i in range(Q)]
    np.testing.assert_allclose(attention_by_head(q, keys, vals, nv).numpy(), attention(q, keys, vals, nv).numpy(),
                               rtol=1e-12, atol=1e-13)

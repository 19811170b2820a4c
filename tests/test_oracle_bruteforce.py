"""Pin the oracle's whole decoder against a second, independent implementation in
pure-Python loops on a micro shape: every term of the layer (pre-norms, q/k/v
split, per-head q/k RMSNorm, rotate-half RoPE, grouped attention, output
projection, residuals, SwiGLU MLP, final norm, LM head) is restated here from
the model definition, so a dropped term, a wrong sign or index or a transposed
operand in either implementation makes the two disagree."""
import math
from dataclasses import dataclass

import numpy as np
import pytest

import synth
from oracle import Oracle


@dataclass(frozen=True)
class Micro:
    name: str = "micro"
    n_layers: int = 2
    d_model: int = 8
    n_heads: int = 4
    n_kv_heads: int = 2
    head_dim: int = 4
    d_ff: int = 6
    vocab: int = 13
    qk_norm: bool = True
    rope_theta: float = 100.0
    rms_eps: float = 1e-6

    @property
    def mask_id(self):
        return self.vocab - 1

    @property
    def qkv_rows(self):
        return (self.n_heads + 2 * self.n_kv_heads) * self.head_dim


def mat(w, name):
    a = w[name]
    if a.dtype == np.uint16:
        a = synth.bf16_bits_to_f32(a)
    return a.astype(np.float64).tolist()


def vec(w, name):
    return np.asarray(w[name], dtype=np.float64).tolist()


def bf16_round(x):
    return float(synth.bf16_bits_to_f32(synth.round_to_bf16_bits(np.array([x], dtype=np.float32)))[0])


def norm(x, g, eps):
    r = math.sqrt(sum(t * t for t in x) / len(x) + eps)
    return [x[i] / r * g[i] for i in range(len(x))]


def matvec(W, x):
    return [sum(W[o][i] * x[i] for i in range(len(x))) for o in range(len(W))]


def rot(x, p, theta):
    d = len(x)
    h = d // 2
    out = [0.0] * d
    for j in range(h):
        a = p * theta ** (-2.0 * j / d)
        out[j] = x[j] * math.cos(a) - x[j + h] * math.sin(a)
        out[j + h] = x[j + h] * math.cos(a) + x[j] * math.sin(a)
    return out


def layer_qkv(s, w, l, x, p, draft):
    pre = "wd_" if draft else "w_"
    H, Hkv, d = s.n_heads, s.n_kv_heads, s.head_dim
    xn = norm(x, vec(w, f"l{l}.attn_norm"), s.rms_eps)
    y = matvec(mat(w, f"l{l}.{pre}qkv"), xn)
    qs = [y[h * d:(h + 1) * d] for h in range(H)]
    ks = [y[(H + j) * d:(H + j + 1) * d] for j in range(Hkv)]
    vs = [y[(H + Hkv + j) * d:(H + Hkv + j + 1) * d] for j in range(Hkv)]
    gq = vec(w, f"l{l}.{'wd_q_norm' if draft else 'q_norm'}")
    gk = vec(w, f"l{l}.{'wd_k_norm' if draft else 'k_norm'}")
    qs = [rot(norm(q, gq, s.rms_eps), p, s.rope_theta) for q in qs]
    ks = [[bf16_round(t) for t in rot(norm(k, gk, s.rms_eps), p, s.rope_theta)] for k in ks]
    vs = [[bf16_round(t) for t in v] for v in vs]
    return qs, ks, vs


def attend(s, q, keys, vals):
    d = len(q)
    sc = [sum(q[t] * k[t] for t in range(d)) / math.sqrt(d) for k in keys]
    m = max(sc)
    e = [math.exp(t - m) for t in sc]
    z = sum(e)
    return [sum(e[j] * vals[j][t] for j in range(len(e))) / z for t in range(d)]


def finish_layer(s, w, l, x, heads_out, draft):
    pre = "wd_" if draft else "w_"
    o = [t for h in heads_out for t in h]
    x = [a + b for a, b in zip(x, matvec(mat(w, f"l{l}.{pre}o"), o))]
    xn = norm(x, vec(w, f"l{l}.mlp_norm"), s.rms_eps)
    gu = matvec(mat(w, f"l{l}.w_gate_up"), xn)
    F = s.d_ff
    act = [gu[i] / (1 + math.exp(-gu[i])) * gu[F + i] for i in range(F)]
    return [a + b for a, b in zip(x, matvec(mat(w, f"l{l}.w_down"), act))]


def logits_of(s, w, x):
    return matvec(mat(w, "lm_head"), norm(x, vec(w, "final_norm"), s.rms_eps))


def brute_run(s, w, prompt, block, draft):
    """Causal pass over the prompt (building the cache), then one block at
    positions P.. either causal over the frozen weights (draft=False) or with the
    draft module and all block positions visible to each other (draft=True)."""
    G = s.n_heads // s.n_kv_heads
    E = mat(w, "embed")
    cache = [[[] for _ in range(s.n_kv_heads)] for _ in range(s.n_layers)]
    cachev = [[[] for _ in range(s.n_kv_heads)] for _ in range(s.n_layers)]
    for p, tok in enumerate(prompt):  # one token at a time, causal by construction
        x = list(E[tok])
        for l in range(s.n_layers):
            qs, ks, vs = layer_qkv(s, w, l, x, p, False)
            for j in range(s.n_kv_heads):
                cache[l][j].append(ks[j])
                cachev[l][j].append(vs[j])
            outs = [attend(s, qs[h], cache[l][h // G], cachev[l][h // G]) for h in range(s.n_heads)]
            x = finish_layer(s, w, l, x, outs, False)
    P = len(prompt)
    xs = [list(E[t]) for t in block]
    for l in range(s.n_layers):
        per = [layer_qkv(s, w, l, xs[i], P + i, draft) for i in range(len(block))]
        new = []
        for i in range(len(block)):
            outs = []
            for h in range(s.n_heads):
                j = h // G
                upto = len(block) if draft else i + 1
                keys = cache[l][j] + [per[b][1][j] for b in range(upto)]
                vals = cachev[l][j] + [per[b][2][j] for b in range(upto)]
                outs.append(attend(s, per[i][0][h], keys, vals))
            new.append(finish_layer(s, w, l, xs[i], outs, draft))
        xs = new
    return [logits_of(s, w, x) for x in xs]


@pytest.mark.parametrize("gain_std", [0.0, 0.3])
def test_decoder_matches_pure_python(gain_std):
    s = Micro()
    w = synth.make_weights(s, 11, 12, std=0.3, gain_std=gain_std, threads=1)
    prompt = [3, 1, 4, 1, 5, 9]
    m = Oracle(s, w, capacity=32, rowwise=True)
    st = m.new_state()
    m.prefill(st, prompt)
    # verify view: block [y, d1, d2, d3], causal
    drafts = [2, 6, 5]
    block = [st.y] + drafts
    _, lg = m.verify_block(st, drafts)
    ref = brute_run(s, w, prompt, block, draft=False)
    np.testing.assert_allclose(lg.numpy(), np.array(ref), rtol=1e-9, atol=1e-11)
    # draft view: block [y, MASK, MASK, MASK], all visible, draft weights
    st2 = m.new_state()
    m.prefill(st2, prompt)
    _, lgd = m.draft_block(st2, 4)
    refd = brute_run(s, w, prompt, [st2.y] + [s.mask_id] * 3, draft=True)
    np.testing.assert_allclose(lgd.numpy(), np.array(refd), rtol=1e-9, atol=1e-11)
    # the prefill's first generated token is the argmax at the last prompt row
    full = brute_run(s, w, prompt[:-1], [prompt[-1]], draft=False)
    assert st.y == int(np.argmax(full[0]))


def test_views_read_their_own_weights():
    s = synth.TINY_QK
    w = synth.make_weights(s, 21, 22, threads=2)
    prompt = synth.make_prompt(s, 12, 21)

    def run(weights):
        m = Oracle(s, weights, capacity=64, rowwise=True)
        st = m.new_state()
        m.prefill(st, prompt)
        _, ld = m.draft_block(st, 4)
        _, lv = m.verify_block(st, [1, 2, 3])
        return ld, lv

    ld0, lv0 = run(w)
    w2 = dict(w)
    w2["l1.wd_o"] = synth.round_to_bf16_bits(synth.bf16_bits_to_f32(w["l1.wd_o"]) * 2.0)
    ld1, lv1 = run(w2)
    assert not np.allclose(ld0.numpy(), ld1.numpy()) and np.array_equal(lv0.numpy(), lv1.numpy())
    w3 = dict(w)
    w3["l1.w_o"] = synth.round_to_bf16_bits(synth.bf16_bits_to_f32(w["l1.w_o"]) * 2.0)
    ld2, lv2 = run(w3)
    assert not np.allclose(lv0.numpy(), lv2.numpy())

"""Pins for the oracle's decoder and Orthrus loop.

* Losslessness: the Orthrus loop's output equals plain greedy AR decoding token
  for token, whatever the drafts (Hacker News summary, 'Idea'; atlas.scime.ai
  summary, 'Approach': output matches greedy AR decoding exactly; opentrain.ai
  abstract: exact consensus).
* All-correct drafts are accepted in full; a wrong first draft advances one token.
* Incremental decoding through the cache equals a one-shot causal forward.
* Closed-form sizes against the figures the pages print (tests/golden).
"""
import json
import os

import numpy as np
import pytest
import torch

import synth
from oracle import (Oracle, attention, draft_param_fraction, greedy_ar, orthrus_generate,
                    scratch_bytes, tokens_per_forward, top2_margin)

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_figures.json")))


def tiny(shape, seed=1, rowwise=True, gain_std=0.0):
    w = synth.make_weights(shape, seed, seed + 100, gain_std=gain_std, threads=2)
    return Oracle(shape, w, capacity=512, rowwise=rowwise), w


def drafter_random(seed):
    rng = np.random.default_rng(seed)
    return lambda m, st, K: rng.integers(0, m.s.vocab, K)


def drafter_from_stream(stream, prompt_len, kind):
    """Drafts built from the known greedy stream (generated tokens; stream[0] sits at
    position prompt_len): all correct, first wrong, or last wrong."""
    def f(m, st, K):
        j = st.n - prompt_len  # generated index of the pending token
        d = [stream[j + 1 + i] for i in range(K)]
        if kind == "first_wrong":
            d[0] = (d[0] + 1) % m.s.vocab
        elif kind == "last_wrong":
            d[-1] = (d[-1] + 1) % m.s.vocab
        return d
    return f


@pytest.mark.parametrize("shape", [synth.TINY, synth.TINY_QK], ids=["tiny", "tiny_qk"])
@pytest.mark.parametrize("seed", [1, 2])
def test_orthrus_equals_greedy_ar(shape, seed):
    m, _ = tiny(shape, seed, gain_std=0.1)
    prompt = synth.make_prompt(shape, 24, seed)
    N, K = 40, 6
    ref = greedy_ar(m, prompt, N + K + 2)
    for name, drafter in [("draft_view", None), ("random", drafter_random(seed)),
                          ("all_correct", drafter_from_stream(ref, len(prompt), "all")),
                          ("first_wrong", drafter_from_stream(ref, len(prompt), "first_wrong")),
                          ("last_wrong", drafter_from_stream(ref, len(prompt), "last_wrong"))]:
        out, acc = orthrus_generate(m, prompt, N, K, drafter)
        assert out == ref[:N], name
        # cache bookkeeping: each step adds a + 1 tokens; the first came from prefill
        assert 1 + sum(a + 1 for a in acc) >= N
        assert 1 + sum(a + 1 for a in acc[:-1]) < N
        if name == "all_correct":
            assert all(a == K for a in acc)
        if name == "first_wrong":
            assert all(a == 0 for a in acc)
        if name == "last_wrong":
            assert all(a == K - 1 for a in acc)


def test_orthrus_equals_greedy_ar_batched_linear():
    # the same invariant with whole-block matrix products: fp64 rounding differences
    # between block shapes stay far below every top-2 margin met on the way
    m, _ = tiny(synth.TINY_QK, 3, rowwise=False)
    prompt = synth.make_prompt(synth.TINY_QK, 16, 3)
    ref = greedy_ar(m, prompt, 30)
    out, _ = orthrus_generate(m, prompt, 30, 5, drafter_random(3))
    assert out == ref


def test_step_accounting_all_correct_and_first_wrong():
    m, _ = tiny(synth.TINY, 4)
    prompt = synth.make_prompt(synth.TINY, 20, 4)
    K = 5
    ref = greedy_ar(m, prompt, 20)
    st = m.new_state()
    m.prefill(st, prompt)
    n0 = st.n
    d = ref[1:1 + K]
    g, _ = m.verify_block(st, d)
    a, toks = m.accept_commit(st, d, g)
    assert a == K and st.n == n0 + K + 1 and toks == ref[1:K + 2] and st.y == ref[K + 1]
    d = [(ref[K + 2] + 1) % 1024] + ref[K + 3:K + 2 + K]
    g, _ = m.verify_block(st, d)
    a, toks = m.accept_commit(st, d, g)
    assert a == 0 and toks == [ref[K + 2]] and st.n == n0 + K + 2


def test_incremental_equals_one_shot_causal_forward():
    # prefill of the whole prompt vs. prefill of a prefix and a teacher-forced verify block
    m, _ = tiny(synth.TINY_QK, 5, gain_std=0.1)
    prompt = synth.make_prompt(synth.TINY_QK, 30, 5)
    full = m.new_state()
    lg_full = m.forward(full, prompt, "verify")
    part = m.new_state()
    m.forward(part, prompt[:22], "verify")
    part.n = 22
    part.y = int(prompt[22])
    _, lg_tail = m.verify_block(part, prompt[23:30])
    np.testing.assert_allclose(lg_tail.numpy(), lg_full[22:30].numpy(), rtol=0, atol=1e-10)
    for l in range(m.s.n_layers):
        np.testing.assert_allclose(part.k[l][:, :30].double().numpy(), full.k[l][:, :30].double().numpy(), atol=1e-12)


def test_single_position_draft_equals_ar_step_with_shared_weights():
    # K = 1: the draft block is [y] alone, so with draft weights set to the base
    # weights the draft view and the AR step compute the same thing
    m, w = tiny(synth.TINY_QK, 6, gain_std=0.1)
    w2 = dict(w)
    for l in range(m.s.n_layers):
        for a, b in [("wd_qkv", "w_qkv"), ("wd_o", "w_o"), ("wd_q_norm", "q_norm"), ("wd_k_norm", "k_norm")]:
            w2[f"l{l}.{a}"] = w[f"l{l}.{b}"]
    m2 = Oracle(m.s, w2, capacity=512, rowwise=True)
    prompt = synth.make_prompt(m.s, 20, 6)
    st = m2.new_state()
    m2.prefill(st, prompt)
    d, lg_d = m2.draft_block(st, 1)
    g, lg_v = m2.verify_block(st, [])
    assert torch.equal(lg_d, lg_v) and d == g
    # K > 1: block row 0 sees the later (mask) positions in the draft view, so it differs
    d4, lg_d4 = m2.draft_block(st, 4)
    assert not torch.allclose(lg_d4[0], lg_v[0])


def test_draft_attention_is_bidirectional_in_block():
    m, _ = tiny(synth.TINY_QK, 7)
    prompt = synth.make_prompt(m.s, 12, 7)
    st = m.new_state()
    m.prefill(st, prompt)
    K = 4
    ids = [st.y] + [m.s.mask_id] * (K - 1)
    _, trace = m.forward(st, ids, "draft", return_qkv=True)
    t0 = trace[0]
    keys = torch.cat([st.k[0][:, :st.n], t0["k"].permute(1, 0, 2)], dim=1)
    vals = torch.cat([st.v[0][:, :st.n], t0["v"].permute(1, 0, 2)], dim=1)
    np.testing.assert_allclose(attention(t0["q"], keys, vals, [st.n + K] * K).numpy(), t0["o"].numpy())
    causal = attention(t0["q"], keys, vals, [st.n + i + 1 for i in range(K)])
    assert not torch.allclose(causal[0], t0["o"][0])
    # the draft pass leaves the cache untouched
    assert st.n == len(prompt)


def test_verify_writes_only_block_slots():
    m, _ = tiny(synth.TINY, 8)
    prompt = synth.make_prompt(m.s, 10, 8)
    st = m.new_state()
    m.prefill(st, prompt)
    before = [k.clone() for k in st.k]
    m.verify_block(st, [1, 2, 3])
    for l in range(m.s.n_layers):
        assert torch.equal(before[l][:, :10], st.k[l][:, :10])
        assert torch.equal(before[l][:, 14:], st.k[l][:, 14:])
        assert not torch.equal(before[l][:, 10:14], st.k[l][:, 10:14])


def test_closed_forms_against_pages():
    g = GOLDEN
    assert g["block_size"]["K"] == 32
    assert scratch_bytes(synth.QWEN3_8B, g["block_size"]["K"]) == 4_718_592
    assert scratch_bytes(synth.QWEN3_8B, 32) / 2 ** 20 == g["scratch_mib_qwen3_8b_k32"]["value"]
    frac = draft_param_fraction(synth.QWEN3_8B)
    assert abs(frac - g["trained_param_fraction"]["value"]) < g["trained_param_fraction"]["tol"]
    t = g["tpf_vs_accept_math500"]
    assert abs(tokens_per_forward(t["accept"]) - t["tpf"]) < 1e-9


def test_margin_helper():
    assert top2_margin(torch.tensor([1.0, 3.0, 2.5], dtype=torch.float64)) == 0.5


@pytest.mark.parametrize("shape", [synth.TINY, synth.TINY_QK], ids=["tiny", "tiny_qk"])
def test_row_by_row_and_batched_evaluation_agree(shape):
    """rowwise=False (matrix products per layer, attention one head at a time) against the
    row-by-row evaluation pinned above: equal up to float64 rounding order, both views."""
    _, w = tiny(shape, 5, gain_std=0.1)
    prompt = synth.make_prompt(shape, 40, 5)
    outs = []
    for rowwise in (True, False):
        m = Oracle(shape, w, capacity=128, rowwise=rowwise)
        st = m.new_state()
        m.prefill(st, prompt)
        d, dl = m.draft_block(st, 6)
        g, vl = m.verify_block(st, d)
        outs.append((dl.numpy(), vl.numpy()))
    for a, b in zip(outs[0], outs[1]):
        np.testing.assert_allclose(a, b, rtol=1e-9, atol=1e-11)

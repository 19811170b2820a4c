"""Pins for the 2-step iterative draft (atlas summary "Surprising findings": a second
denoising step of the draft view, compared there with the single-step projection).

Reading: the second step re-runs the draft view over [y, d_1..d_{K-1}], the first
step's predictions in place of the masks, at the same positions.
* against the pure-Python brute-force decoder (an independent definition);
* with all-mask inputs the refinement is the single step itself;
* d_K has no input slot; every other draft reaches every row (bidirectional);
* the Orthrus loop with 2-step drafts is still lossless.
"""
import numpy as np
import pytest
import torch

import oracle.model as om
import synth
from oracle import Oracle, greedy_ar, orthrus_generate
from test_oracle_bruteforce import Micro, brute_run


def micro_model(seed=21):
    s = Micro()
    w = synth.make_weights(s, seed, seed + 1, std=0.3, gain_std=0.3, threads=1)
    return s, w, Oracle(s, w, capacity=32, rowwise=True)


def test_refine_matches_brute_force():
    s, w, m = micro_model()
    prompt = [3, 1, 4, 1, 5, 9]
    st = m.new_state()
    m.prefill(st, prompt)
    prev = [7, 2, 11, 0]
    new, lg = m.draft_refine(st, prev)
    ref = np.array(brute_run(s, w, prompt, [st.y, 7, 2, 11], True))
    np.testing.assert_allclose(lg.numpy(), ref, rtol=1e-9, atol=1e-11)
    assert new == [int(np.argmax(r)) for r in ref]
    # a draft pass leaves the cache length and the pending token as they were
    y = st.y
    m.draft_refine(st, prev)
    assert st.n == len(prompt) and st.y == y


def test_refine_of_masks_is_the_single_step():
    s, w, m = micro_model(22)
    st = m.new_state()
    m.prefill(st, [2, 7, 1, 8, 2, 8])
    for K in (1, 2, 5):
        d1, lg1 = m.draft_block(st, K)
        d2, lg2 = m.draft_refine(st, [s.mask_id] * K)
        assert torch.equal(lg1, lg2) and d1 == d2


def test_last_draft_is_not_read_and_others_reach_every_row():
    s, w, m = micro_model(23)
    st = m.new_state()
    m.prefill(st, [1, 2, 3, 4, 5])
    base = [4, 9, 6, 3]
    _, lg = m.draft_refine(st, base)
    _, lg_last = m.draft_refine(st, base[:3] + [10])
    assert torch.equal(lg, lg_last)
    for j in range(3):
        alt = list(base)
        alt[j] = (alt[j] + 5) % (s.vocab - 1)
        _, lg_j = m.draft_refine(st, alt)
        for i in range(4):  # rows before and after slot j + 1 both see the change
            assert not torch.allclose(lg_j[i], lg[i]), (j, i)


@pytest.mark.parametrize("shape", [synth.TINY, synth.TINY_QK], ids=["tiny", "tiny_qk"])
def test_two_step_loop_is_lossless(shape):
    w = synth.make_weights(shape, 3, 103, gain_std=0.1, threads=2)
    m = Oracle(shape, w, capacity=256, rowwise=True)
    prompt = synth.make_prompt(shape, 16, 3)
    N, K = 24, 4
    ref = greedy_ar(m, prompt, N)
    out, acc = orthrus_generate(m, prompt, N, K, draft_steps=2)
    assert out == ref
    assert all(0 <= a <= K for a in acc)


def test_draft_steps_counts_passes(monkeypatch):
    _, _, m = micro_model(24)
    st = m.new_state()
    m.prefill(st, [5, 6, 7])
    first, _ = m.draft_block(st, 3)
    calls = []
    orig = om.Oracle.forward

    def counting(self, st_, ids, view, **kw):
        calls.append((view, list(ids)))
        return orig(self, st_, ids, view, **kw)

    monkeypatch.setattr(om.Oracle, "forward", counting)
    m.draft_steps(st, 3, 2)
    assert [v for v, _ in calls] == ["draft", "draft"]
    assert calls[0][1] == [st.y, m.s.mask_id, m.s.mask_id]
    assert calls[1][1] == [st.y] + first[:2]


# ---- planted mistakes in the refinement -------------------------------------------------

def refine_shifted(self, st, drafts):  # d_2..d_K in the slots instead of d_1..d_{K-1}
    K = len(drafts)
    logits = self.forward(st, [st.y] + [int(t) for t in drafts[1:K]], "draft")
    return [int(torch.argmax(logits[i])) for i in range(K)], logits


def refine_without_pending(self, st, drafts):  # the block starts at d_1: y dropped
    K = len(drafts)
    logits = self.forward(st, [int(t) for t in drafts[:K]], "draft")
    return [int(torch.argmax(logits[i])) for i in range(K)], logits


def refine_verify_view(self, st, drafts):  # the frozen causal view instead of the draft view
    K = len(drafts)
    saved = (st.n, [k.clone() for k in st.k], [v.clone() for v in st.v])
    logits = self.forward(st, [st.y] + [int(t) for t in drafts[:K - 1]], "verify")
    st.n, st.k, st.v = saved
    return [int(torch.argmax(logits[i])) for i in range(K)], logits


def brute_pin_holds(m, s, w):
    prompt = [3, 1, 4, 1, 5, 9]
    st = m.new_state()
    m.prefill(st, prompt)
    prev = [7, 2, 11, 0]
    _, lg = m.draft_refine(st, prev)
    ref = np.array(brute_run(s, w, prompt, [st.y, 7, 2, 11], True))
    return bool(np.allclose(lg.numpy(), ref, rtol=1e-9, atol=1e-11))


@pytest.mark.parametrize("mistake", [refine_shifted, refine_without_pending, refine_verify_view],
                         ids=lambda f: f.__name__)
def test_planted_refinement_mistake_is_caught(mistake, monkeypatch):
    s, w, m = micro_model()
    assert brute_pin_holds(m, s, w)
    monkeypatch.setattr(om.Oracle, "draft_refine", mistake)
    assert not brute_pin_holds(m, s, w)

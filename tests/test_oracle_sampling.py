"""Pins for the oracle of decoding at temperature T > 0 (rejection sampling; atlas
summary "Limitations", Hacker News summary "Limitations"), against what the
mathematics fixes rather than the oracle's own formulas:

* the inverse-CDF draw on hand-computed cases and, over a stratified grid of
  uniforms, with frequencies equal to the weights;
* softmax at temperature T: closed forms, shift invariance, the T -> 0 and
  T -> infinity limits;
* the speculative-sampling theorem: the first committed token is distributed as
  the target p whatever the draft distribution q (exact integration over grids of
  the uniforms), and a whole sampled decode of a toy prefix-dependent model has the
  joint distribution of plain sampling (seeded Monte Carlo, chi-square bound);
* special cases: T -> 0 is the greedy consensus; q == p accepts every draft; a
  draft the target gives zero probability is always rejected;
* plausible mistakes planted in the consensus are caught by the exact pin.
"""
import math

import numpy as np
import pytest
import torch

import oracle.sampling as osamp
from oracle import accept_length, committed_tokens, inverse_cdf, speculative_accept, tempered_probs

F64 = torch.float64


def test_inverse_cdf_hand_values():
    w = [1.0, 2.0, 3.0]  # C = 1, 3, 6
    assert inverse_cdf(w, 0.0) == 0
    assert inverse_cdf(w, 0.1) == 0        # 0.6 < 1
    assert inverse_cdf(w, 1 / 6) == 1      # 1.0 is not > 1.0
    assert inverse_cdf(w, 0.2) == 1        # 1.2
    assert inverse_cdf(w, 0.5) == 2        # 3.0 is not > 3.0
    assert inverse_cdf(w, 0.999) == 2
    z = [0.0, 1.0, 0.0, 1.0, 0.0]          # zero weights are never drawn
    assert inverse_cdf(z, 0.0) == 1
    assert inverse_cdf(z, 0.5) == 3
    assert inverse_cdf(z, 0.9999) == 3
    assert inverse_cdf([0.0, 0.0, 5.0], 0.3) == 2
    with pytest.raises(ValueError):
        inverse_cdf([0.0, 0.0], 0.5)
    with pytest.raises(ValueError):
        inverse_cdf([1.0, -1.0, 1.0], 0.5)


def test_inverse_cdf_frequencies_on_a_stratified_grid():
    rng = np.random.default_rng(3)
    w = rng.random(9)
    w[[2, 5]] = 0.0
    N = 3000
    counts = np.zeros(9)
    for k in range(N):
        counts[inverse_cdf(w, (k + 0.5) / N)] += 1
    assert counts[2] == 0 and counts[5] == 0
    np.testing.assert_allclose(counts / N, w / w.sum(), atol=1.0 / N + 1e-12)


def test_tempered_probs_closed_forms():
    z = [0.3, -1.2, 2.0, 0.0, 1.1]
    for T in (0.5, 1.0, 2.5):
        e = [math.exp(x / T) for x in z]
        ref = [x / sum(e) for x in e]
        np.testing.assert_allclose(tempered_probs(z, T).numpy(), ref, rtol=1e-13)
        p = tempered_probs(z, T)
        assert abs(float(p[2] / p[1]) - math.exp((2.0 + 1.2) / T)) < 1e-9 * math.exp(3.2 / T)
        shifted = tempered_probs([x + 37.5 for x in z], T)
        np.testing.assert_allclose(shifted.numpy(), p.numpy(), rtol=1e-12)
    np.testing.assert_allclose(tempered_probs(z, 1e6).numpy(), [0.2] * 5, atol=1e-5)
    cold = tempered_probs(z, 1e-3).numpy()
    assert cold[2] == pytest.approx(1.0) and cold.sum() == pytest.approx(1.0)
    with pytest.raises(FloatingPointError):
        tempered_probs([0.0, float("nan")], 1.0)
    with pytest.raises(ValueError):
        tempered_probs([0.0, 1.0], 0.0)


def first_token_distribution(p0, q0, p1, N=2000):
    """Exact distribution of the first committed token of a K = 1 block, integrating
    the consensus over its inputs: the draft d ~ q0 (its weight), the accept uniform
    u and the last-token uniform v (independent, midpoints of an N-point grid)."""
    V = len(p0)
    grid = [(k + 0.5) / N for k in range(N)]
    out = np.zeros(V)
    p = [p0, p1]
    for d in range(V):
        if q0[d] == 0:
            continue
        acc = 0
        rej_u = None
        for u in grid:
            a, _ = speculative_accept([d], [q0], p, [u], 0.5)
            if a == 1:
                acc += 1
            else:
                rej_u = u
        out[d] += q0[d] * acc / N
        if rej_u is not None:
            resid = np.zeros(V)
            for v in grid:
                _, toks = speculative_accept([d], [q0], p, [rej_u], v)
                resid[toks[0]] += 1
            out += q0[d] * (N - acc) / N * resid / N
    return out


def random_pair(seed, V=6):
    rng = np.random.default_rng(seed)
    p = rng.random(V) ** 2
    q = rng.random(V) ** 2
    p[1] = 0.0   # the target never emits token 1 ...
    q[4] = 0.0   # ... and the drafter never proposes token 4
    return p / p.sum(), q / q.sum(), np.full(V, 1.0 / V)


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_first_token_is_distributed_as_the_target(seed):
    p0, q0, p1 = random_pair(seed)
    got = first_token_distribution(p0, q0, p1)
    np.testing.assert_allclose(got, p0, atol=3.0 / 2000)
    assert got[1] == 0.0


def test_bonus_token_is_drawn_from_the_last_verify_row():
    p0 = np.array([0.5, 0.5, 0.0])
    q0 = np.array([0.5, 0.5, 0.0])    # p == q: every draft accepted
    p1 = np.array([0.1, 0.3, 0.6])
    N = 1000
    counts = np.zeros(3)
    for k in range(N):
        a, toks = speculative_accept([1], [q0], [p0, p1], [0.999], (k + 0.5) / N)
        assert a == 1 and toks[0] == 1
        counts[toks[1]] += 1
    np.testing.assert_allclose(counts / N, p1, atol=1.0 / N + 1e-12)


# ---- the joint distribution of a whole sampled decode (toy model) -----------

class Toy:
    """Target p(.|prefix) depends on the last two tokens; the drafter's row i
    distribution q_i(.|prefix at the step's start) on the last token and i (drafts
    drawn independently, as in a one-pass block projection)."""

    def __init__(self, V=3, K=2, seed=7):
        rng = np.random.default_rng(seed)
        self.V, self.K = V, K
        self.pt = {key: rng.normal(0, 1.0, V) for key in self.keys2()}
        self.qd = {(i, t): rng.normal(0, 1.0, V) for i in range(K) for t in range(-1, V)}

    def keys2(self):
        return [(a, b) for a in range(-1, self.V) for b in range(-1, self.V)]

    def p(self, s):
        key = ((s[-2] if len(s) > 1 else -1), (s[-1] if s else -1))
        return tempered_probs(self.pt[key], 1.0).numpy()

    def q(self, i, s):
        return tempered_probs(self.qd[(i, s[-1] if s else -1)], 1.0).numpy()

    def decode(self, n, rng, accept=speculative_accept):
        s = []
        while len(s) < n:
            q = [self.q(i, s) for i in range(self.K)]
            d = [inverse_cdf(q[i], rng.random()) for i in range(self.K)]
            p = [self.p(s + d[:j]) for j in range(self.K + 1)]
            _, toks = accept(d, q, p, rng.random(self.K), rng.random())
            s += toks
        return tuple(s[:n])

    def exact(self, n):
        out = {}
        def rec(s, pr):
            if len(s) == n:
                out[tuple(s)] = pr
                return
            p = self.p(s)
            for t in range(self.V):
                rec(s + [t], pr * p[t])
        rec([], 1.0)
        return out


def chi_square(toy, n_tok, samples, seed, accept=speculative_accept):
    rng = np.random.default_rng(seed)
    exp = toy.exact(n_tok)
    counts = dict.fromkeys(exp, 0)
    for _ in range(samples):
        counts[toy.decode(n_tok, rng, accept)] += 1
    return sum((counts[k] - samples * e) ** 2 / (samples * e) for k, e in exp.items()), len(exp) - 1


@pytest.mark.parametrize("K", [2, 3])
def test_sampled_decode_has_the_joint_distribution_of_plain_sampling(K):
    toy = Toy(V=3, K=K, seed=7 + K)
    chi2, df = chi_square(toy, 3, 12000, seed=11 + K)
    # 26 degrees of freedom: P(chi2 > 80) < 1e-6 under the null hypothesis
    assert df == 26 and chi2 < 80.0, chi2


# ---- special cases ----------------------------------------------------------

def test_cold_temperature_reduces_to_greedy_consensus():
    rng = np.random.default_rng(5)
    V, K, T = 50, 6, 1e-3
    for trial in range(40):
        dl = rng.normal(0, 1, (K, V))
        vl = rng.normal(0, 1, (K + 1, V))
        g = [int(np.argmax(r)) for r in vl]
        d = [g[i] if i < trial % (K + 1) else int(np.argmax(dl[i])) for i in range(K)]
        # the draft view's row i prefers d_{i+1} by a clear margin
        for i in range(K):
            dl[i, d[i]] = dl[i].max() + 1.0
        drafts = osamp.sample_tokens(dl, T, rng.random(K))
        assert drafts == d
        a, toks = osamp.accept_sample_logits(drafts, dl, vl, T, rng.random(K), float(rng.random()))
        ag = accept_length(drafts, g)
        assert a == ag and toks == committed_tokens(drafts, g, ag)


def test_equal_distributions_accept_every_draft():
    rng = np.random.default_rng(6)
    V, K = 20, 5
    logits = rng.normal(0, 2, (K + 1, V))
    for _ in range(20):
        drafts = [int(t) for t in rng.integers(0, V, K)]
        a, toks = osamp.accept_sample_logits(drafts, logits[:K], logits, 0.8, rng.random(K), float(rng.random()))
        assert a == K and toks[:K] == drafts


def test_draft_of_zero_target_probability_is_rejected():
    q = [np.array([0.25, 0.25, 0.25, 0.25])]
    p = [np.array([0.0, 0.5, 0.5, 0.0]), np.array([1.0, 0.0, 0.0, 0.0])]
    for u in (0.0, 0.3, 0.999):
        for v in (0.0, 0.4, 0.7, 0.999):
            a, toks = speculative_accept([0], q, p, [u], v)
            # residual max(0, p - q) = [0, .25, .25, 0]: token 1 or 2, never 0 or 3
            assert a == 0 and toks[0] in (1, 2)
            assert toks[0] == (1 if v < 0.5 else 2)


# ---- planted mistakes -------------------------------------------------------

def resid_reversed(drafts, q, p, u_accept, v_final):
    K = len(drafts)
    a = 0
    while a < K and u_accept[a] * q[a][drafts[a]] < p[a][drafts[a]]:
        a += 1
    if a == K:
        return a, list(drafts) + [inverse_cdf(p[K], v_final)]
    return a, list(drafts[:a]) + [inverse_cdf(np.maximum(np.asarray(q[a]) - p[a], 0.0), v_final)]


def ratio_inverted(drafts, q, p, u_accept, v_final):
    K = len(drafts)
    a = 0
    while a < K and u_accept[a] * p[a][drafts[a]] < q[a][drafts[a]]:
        a += 1
    if a == K:
        return a, list(drafts) + [inverse_cdf(p[K], v_final)]
    return a, list(drafts[:a]) + [inverse_cdf(np.maximum(np.asarray(p[a]) - q[a], 0.0), v_final)]


def resample_from_target(drafts, q, p, u_accept, v_final):
    K = len(drafts)
    a = 0
    while a < K and u_accept[a] * q[a][drafts[a]] < p[a][drafts[a]]:
        a += 1
    return a, list(drafts[:a]) + [inverse_cdf(p[a], v_final)]


@pytest.mark.parametrize("mistake", [resid_reversed, ratio_inverted, resample_from_target],
                         ids=lambda f: f.__name__)
def test_planted_mistake_is_caught(mistake, monkeypatch):
    monkeypatch.setattr(osamp, "speculative_accept", mistake)
    monkeypatch.setattr(__import__(__name__), "speculative_accept", mistake)
    p0, q0, p1 = random_pair(1)
    got = first_token_distribution(p0, q0, p1, N=400)
    assert np.abs(got - p0).max() > 0.02


def test_sampled_step_on_the_decoder_reduces_to_the_greedy_step_when_cold():
    """The oracle's whole sampled step on a tiny decoder: at T -> 0 the draws are the
    argmaxes and the consensus is the greedy one, so the step commits what the greedy step
    commits; the cache bookkeeping is the greedy step's."""
    import synth
    from oracle import Oracle
    from test_oracle_bruteforce import Micro
    s = Micro()
    w = synth.make_weights(s, 31, 32, std=0.3, gain_std=0.3, threads=1)
    m = Oracle(s, w, capacity=64, rowwise=True)
    rng = np.random.default_rng(8)
    cold, greedy = m.new_state(), m.new_state()
    prompt = [3, 1, 4, 1, 5, 9, 2, 6]
    m.prefill(cold, prompt)
    m.prefill(greedy, prompt)
    K = 4
    for _ in range(5):
        ud, ua, uf = osamp.step_uniforms(rng, 1, K)
        d_ref, _ = m.draft_block(greedy, K)
        g, _ = m.verify_block(greedy, d_ref)
        a_ref, toks_ref = m.accept_commit(greedy, d_ref, g)
        drafts, a, toks = osamp.sampled_step(m, cold, K, 1e-4, ud[0], ua[0], float(uf[0]))
        assert drafts == d_ref and a == a_ref and toks == toks_ref
        assert cold.n == greedy.n and cold.y == greedy.y


def test_empty_residual_draws_from_the_target():
    # p_0 == q_0 and a draft outside q_0's support: u * q(d) = 0 is not < p(d) = 0, so the draft
    # is rejected and max(0, p_0 - q_0) is zero everywhere. The committed token must still be
    # distributed as p_0 (the frozen model's sampling distribution): one-hot p_0 forces its
    # token, a spread p_0 gives p_0's frequencies on a stratified grid of v.
    one_hot = np.array([0.0, 0.0, 1.0, 0.0])
    for u in (0.0, 0.5, 0.999):
        for v in (0.0, 0.5, 0.999):
            a, toks = speculative_accept([1], [one_hot], [one_hot, one_hot], [u], v)
            assert a == 0 and toks == [2]
    p0 = np.array([0.1, 0.0, 0.6, 0.3])
    N = 1000
    counts = np.zeros(4)
    for i in range(N):
        a, toks = speculative_accept([1], [p0], [p0, one_hot], [0.5], (i + 0.5) / N)
        assert a == 0
        counts[toks[0]] += 1
    assert np.allclose(counts / N, p0, atol=1.5 / N)

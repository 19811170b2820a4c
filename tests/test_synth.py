"""The seeded input generators (`synth/`), which both the oracle and the GPU path read:

* bfloat16 rounding is round-to-nearest-even, checked against PyTorch's own conversion
  on random values, exact ties and the special values;
* weights are deterministic in their seeds and independent of the thread count;
* the planted schedule: accept lengths are Geometric on {0, 1, ...} with the requested
  mean, capped at K (the capped mean has the closed form m (1 - (m/(m+1))^K)); planted
  drafts reproduce exactly the planted accept length under the accept rule, with
  d_{a+1} never the greedy token.
"""
import numpy as np
import torch

import synth
from oracle import accept_length


def test_bf16_rounding_is_round_to_nearest_even():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(100000).astype(np.float32) * np.float32(3.0),
        rng.standard_normal(1000).astype(np.float32) * np.float32(1e-30),  # subnormal range of bf16
        np.array([0.0, -0.0, np.inf, -np.inf, 1.0, -2.5, 3.3895314e38], dtype=np.float32),
    ])
    # exact ties: the low 16 bits are 0x8000, with both parities of the kept part
    ties = (np.arange(2000, dtype=np.uint32) << np.uint32(16)) | np.uint32(0x3F800000 | 0x8000)
    x = np.concatenate([x, ties.view(np.float32)])
    got = synth.round_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)
    back = synth.bf16_bits_to_f32(got)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy())


def test_weights_are_deterministic_and_thread_independent():
    a = synth.make_weights(synth.TINY, 5, 6, threads=1)
    b = synth.make_weights(synth.TINY, 5, 6, threads=4)
    c = synth.make_weights(synth.TINY, 5, 7, threads=2)
    assert a.keys() == b.keys()
    for k in a:
        assert np.array_equal(a[k], b[k]), k
    # the draft seed moves only the draft module's tensors
    for k in a:
        same = np.array_equal(a[k], c[k])
        assert same == (".wd_" not in k or k.endswith("_norm")), k
    w = synth.bf16_bits_to_f32(a["l0.w_qkv"]).astype(np.float64)
    assert abs(w.std() - 0.02) < 5e-4 and abs(w.mean()) < 5e-4


def test_planted_accepts_are_capped_geometric():
    for mean, K in [(6.0, 32), (1.6, 8), (12.8, 64), (3.0, 4)]:
        a = synth.planted_accepts(200000, mean, K, seed=3)
        assert a.min() == 0 and a.max() <= K
        capped = mean * (1.0 - (mean / (mean + 1.0)) ** K)
        assert abs(a.mean() - capped) < 0.03 * max(1.0, capped) ** 0.5, (mean, K, a.mean(), capped)
        p = 1.0 / (mean + 1.0)
        assert abs(np.mean(a == 0) - p) < 0.005
    assert np.array_equal(synth.planted_accepts(50, 6.0, 32, seed=9), synth.planted_accepts(50, 6.0, 32, seed=9))


def test_planted_drafts_reproduce_the_planted_accept_length():
    rng = np.random.default_rng(4)
    V, K = 1000, 16
    stream = rng.integers(0, V, 400).astype(np.int32)
    for trial in range(500):
        n = int(rng.integers(0, 300))
        a = int(rng.integers(0, K + 1))
        d = synth.planted_drafts(stream, n, a, K, V, rng)
        greedy = stream[n + 1:n + K + 2]  # g_0..g_K of this step
        assert d.shape == (K,) and d.min() >= 0 and d.max() < V
        assert np.array_equal(d[:a], stream[n + 1:n + 1 + a])
        if a < K:
            assert d[a] != stream[n + a + 1]
        assert accept_length(d.tolist(), greedy.tolist()) == a


def test_stratified_accepts_follow_the_capped_geometric_law():
    for mean, K in [(6.0, 32), (1.6, 8), (12.8, 64), (3.0, 4)]:
        capped = synth.capped_geometric_mean(mean, K)
        # the closed form against a direct sum of the capped law
        p = 1.0 / (mean + 1.0)
        pk = p * (1.0 - p) ** np.arange(K)
        direct = float(np.sum(np.arange(K) * pk) + K * (1.0 - p) ** K)
        assert abs(capped - direct) < 1e-9
        a = synth.planted_accepts_stratified(4000, mean, K, seed=5)
        assert a.min() == 0 and a.max() <= K
        assert abs(a.mean() - capped) < 0.01 * max(1.0, capped)
        assert abs(np.mean(a == 0) - p) < 1e-3  # the quantiles put a fraction p at zero
        # a short window keeps its mean near the law's (stratified, not i.i.d.)
        assert abs(synth.planted_accepts_stratified(147, mean, K, seed=6).mean() - capped) < 0.1 * max(1.0, capped)
    a = synth.planted_accepts_stratified(64, 6.0, 32, seed=9)
    assert np.array_equal(a, synth.planted_accepts_stratified(64, 6.0, 32, seed=9))
    assert not np.array_equal(a, np.sort(a))  # seeded order, not sorted

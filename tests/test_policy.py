"""Dynamic block size (news article, "Future Directions: Larger K and Higher Acceptance",
item 1: choose K by how certain the generation is).

Pins of the oracle's definitions (oracle/policy.py) against things other than
themselves:
  - E[a + 1 | K] against a seeded simulation of the acceptance process it models
    (each draft accepted with probability alpha until the first rejection), and its
    limits: 1 at alpha = 0, K + 1 at alpha = 1;
  - the rate estimate against the true alpha of simulated accept lengths, censored at
    K (a mistake that counts a full block as a rejection is caught);
  - block-size choices computed by hand;
  - planted mistakes in the oracle are caught.
Then the library's host-only calls (orthrus_accept_stats_update, orthrus_accept_rate,
orthrus_choose_block_size) against the oracle on the same inputs. No GPU is needed:
the calls touch no device memory.
"""
import numpy as np
import pytest

from oracle import policy as P


def simulate_accepts(alpha, K, n, seed):
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        a = 0
        while a < K and rng.random() < alpha:
            a += 1
        out.append(a)
    return np.array(out)


@pytest.mark.parametrize("alpha,K", [(0.3, 8), (0.8, 8), (0.9, 32), (0.97, 64)])
def test_expected_committed_matches_simulated_process(alpha, K):
    a = simulate_accepts(alpha, K, 40000, seed=int(alpha * 100) + K)
    mc = float(np.mean(a + 1))
    se = float(np.std(a + 1)) / np.sqrt(len(a))
    assert abs(P.expected_committed(alpha, K) - mc) < 5 * se


def test_expected_committed_limits():
    assert P.expected_committed(0.0, 16) == 1.0
    assert P.expected_committed(1.0, 16) == 17.0
    assert P.expected_committed(0.5, 0) == 1.0


@pytest.mark.parametrize("alpha,K", [(0.6, 8), (0.85, 16), (0.5, 4), (0.9, 8)])
def test_rate_estimate_recovers_alpha_from_censored_lengths(alpha, K):
    a = simulate_accepts(alpha, K, 20000, seed=7 + K)
    stats = [[0.0, 0.0]]
    for x in a:
        P.update_stats(stats, [int(x)], K)
    est = P.accept_rate(*stats[0])
    assert abs(est - alpha) < 0.01, (est, alpha)


def test_hand_computed_choices():
    ks, t = [8, 16, 32, 64], [10.0, 11.0, 14.0, 20.0]
    # alpha 0.9: E = 6.126, 8.332, 9.690, 9.988 -> per ms 0.613, 0.757, 0.692, 0.499
    assert P.choose_block_size([[89.0, 9.0]], ks, t) == 16  # rate (89+1)/(98+2) = 0.9
    # alpha 0.99: per ms 0.865, 1.426, 2.013, 2.378
    assert P.choose_block_size([[97.0, 0.0]], ks, t) == 64  # (97+1)/(97+2) = 0.98989...
    # alpha 0.25: E is 1.33 for every K: the fastest step wins
    assert P.choose_block_size([[2.0, 8.0]], ks, t) == 8
    # equal step times: larger K never commits fewer tokens; equal rates go to the smaller K
    assert P.choose_block_size([[0.0, 0.0]], [4, 8], [5.0, 5.0]) == 8
    assert P.choose_block_size([[0.0, 1e9]], [4, 8], [5.0, 5.0]) == 4
    # a batch sums its sequences: one certain and one uncertain sequence
    assert P.choose_block_size([[97.0, 0.0], [2.0, 8.0]], ks, t) == 64


def wrong_expected_linear(alpha, K):
    return 1.0 + alpha * K


def wrong_update_counts_full_blocks(stats, accept_lens, K, decay=1.0):
    for b, a in enumerate(accept_lens):
        stats[b][0] = decay * stats[b][0] + a
        stats[b][1] = decay * stats[b][1] + 1.0
    return stats


def pins_hold():
    try:
        test_expected_committed_matches_simulated_process(0.9, 32)
        test_rate_estimate_recovers_alpha_from_censored_lengths(0.9, 8)  # 43% of blocks end full
        test_hand_computed_choices()
    except AssertionError:
        return False
    return True


@pytest.mark.parametrize("name,fn", [("expected_committed", wrong_expected_linear),
                                     ("update_stats", wrong_update_counts_full_blocks)])
def test_planted_policy_mistake_is_caught(name, fn, monkeypatch):
    assert pins_hold()
    monkeypatch.setattr(P, name, fn)
    assert not pins_hold()


# ---- the library's host-only calls against the oracle --------------------------------------------
def lib():
    from shared_kv_draft_b200 import orthrus
    orthrus.load()
    return orthrus


def test_library_policy_matches_oracle():
    o = lib()
    rng = np.random.default_rng(11)
    checked = 0
    for trial in range(300):
        B = int(rng.integers(1, 6))
        K = int(rng.choice([4, 8, 16, 32, 64]))
        decay = float(rng.choice([1.0, 0.9, 0.5]))
        stats_c = o.accept_stats(B)
        stats_p = [[0.0, 0.0] for _ in range(B)]
        for _ in range(int(rng.integers(0, 12))):
            al = [int(x) for x in rng.integers(-1, K + 1, size=B)]
            o.accept_stats_update(stats_c, al, K, decay)
            P.update_stats(stats_p, al, K, decay)
        for b in range(B):
            assert abs(stats_c[b].accepted - stats_p[b][0]) <= 1e-4 * max(1.0, stats_p[b][0])
            assert abs(stats_c[b].rejected - stats_p[b][1]) <= 1e-4 * max(1.0, stats_p[b][1])
            assert abs(o.accept_rate(stats_c, b) - P.accept_rate(*stats_p[b])) < 1e-5
        n = int(rng.integers(1, 6))
        ks = sorted(set(int(k) for k in rng.integers(1, 65, size=n)))
        t = [float(x) for x in rng.uniform(1.0, 20.0, size=len(ks))]
        # compare where the oracle's best rate beats the runner-up clearly (float32 counts)
        stats_f = [[float(stats_c[b].accepted), float(stats_c[b].rejected)] for b in range(B)]
        rates = sorted((sum(P.expected_committed(P.accept_rate(a, r), k) for a, r in stats_f) / tt)
                       for k, tt in zip(ks, t))
        if len(rates) > 1 and rates[-1] - rates[-2] < 1e-6 * rates[-1]:
            continue
        assert o.choose_block_size(stats_c, ks, t) == P.choose_block_size(stats_f, ks, t)
        checked += 1
    assert checked > 250


def test_library_policy_rejects_bad_arguments():
    o = lib()
    st = o.accept_stats(1)
    with pytest.raises(o.OrthrusError):
        o.accept_stats_update(st, [9], 8)  # a > K
    with pytest.raises(o.OrthrusError):
        o.accept_stats_update(st, [1], 8, decay=0.0)
    with pytest.raises(o.OrthrusError):
        o.choose_block_size(st, [0, 8], [1.0, 1.0])
    with pytest.raises(o.OrthrusError):
        o.choose_block_size(st, [8], [0.0])
    o.accept_stats_update(st, [-1], 8)  # a failed step changes nothing
    assert st[0].accepted == 0.0 and st[0].rejected == 0.0
    assert abs(o.accept_rate(st, 0) - 0.5) < 1e-7

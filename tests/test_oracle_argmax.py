"""Pins for the oracle's argmax, reading R8 of the build: the pages do not say how an
exact tie between logits is broken, and the reading taken is the lowest vocabulary
index among the maximal values; a NaN logit anywhere in the row is an error. The
greedy consensus (HN summary "Idea": longest draft prefix equal to the AR argmax)
compares integer ids, so the tie rule decides committed tokens whenever two logits
are equal.

The pin is a pure-Python scan, independent of the oracle's torch call: keep the
first index whose value is strictly larger than every earlier one. Two planted
mistakes must fail it: the highest index on ties, and a NaN that is skipped.
"""
import math

import numpy as np
import pytest
import torch

import oracle.model as om
import synth
from oracle import Oracle, argmax_checked


def first_max_index(values):
    best = 0
    for i in range(1, len(values)):
        if values[i] > values[best]:
            best = i
    return best


def tie_rows():
    """Rows with exact ties among their maxima, small and vocabulary-sized."""
    rows = [
        [1.0, 3.0, 3.0, 2.0],
        [5.0, 5.0, 5.0],
        [-math.inf, -1.0, -1.0],
        [-0.0, 0.0, -0.0],            # -0 and +0 are equal numbers: index 0
        [0.0, -0.0],
        [-2.0, -0.0, 0.0, -1.0],      # max is the {-0, +0} tie at 1, 2
        [7.0],
    ]
    rng = np.random.default_rng(5)
    for V, n_ties in [(1024, 2), (1024, 5), (151936, 2), (151936, 4)]:
        r = rng.standard_normal(V)
        pos = np.sort(rng.choice(V, n_ties, replace=False))
        r[pos] = r.max() + 1.0
        rows.append(r.tolist())
    r = np.zeros(151936)
    r[[150000, 151935]] = 0.5        # ties near the end of the vocabulary
    rows.append(r.tolist())
    return rows


def nan_rows():
    rows = []
    for V in (4, 1024):
        for at in (0, V // 2, V - 1):
            r = np.linspace(-1.0, 1.0, V)
            r[at] = math.nan
            rows.append(r)
    r = np.full(16, -math.inf)
    r[3] = math.nan
    rows.append(r)
    r = np.array([math.inf, math.nan])
    rows.append(r)
    return rows


def pins_hold(argmax_fn) -> bool:
    for r in tie_rows():
        if argmax_fn(torch.tensor(r, dtype=torch.float64)) != first_max_index(r):
            return False
    for r in nan_rows():
        try:
            argmax_fn(torch.tensor(r, dtype=torch.float64))
        except FloatingPointError:
            continue
        return False
    return True


def test_oracle_argmax_takes_lowest_index_and_rejects_nan():
    assert pins_hold(argmax_checked)


def test_pure_python_scan_reading():
    # the scan itself, on rows whose answer is plain by eye
    assert first_max_index([1.0, 3.0, 3.0, 2.0]) == 1
    assert first_max_index([-0.0, 0.0]) == 0
    assert first_max_index([0.0, 2.0, 1.0, 2.0]) == 1


def highest_index_on_ties(row):
    if torch.isnan(row).any():
        raise FloatingPointError("NaN logit")
    return int(len(row) - 1 - torch.argmax(row.flip(0)))


def nan_skipped(row):
    return int(torch.argmax(torch.nan_to_num(row, nan=-math.inf)))


@pytest.mark.parametrize("bad", [highest_index_on_ties, nan_skipped], ids=["highest_index", "nan_skipped"])
def test_planted_argmax_mistake_is_caught(bad):
    assert not pins_hold(bad)


def tie_head_weights(shape, seed, j1, j2, col):
    """Weights whose LM head is zero except rows j1 < j2, both equal to a unit vector
    at column ``col``: every logit is exactly 0 except logits j1 and j2, which are
    equal (one product each). The maximum is therefore always an exact tie: {j1, j2}
    when their shared value is positive, else every zero logit."""
    w = synth.make_weights(shape, seed, seed + 1, threads=2)
    lm = np.zeros_like(w["lm_head"])
    one = synth.round_to_bf16_bits(np.ones(1, dtype=np.float32))[0]
    lm[j1, col] = one
    lm[j2, col] = one
    w["lm_head"] = lm
    return w


def test_decoder_level_tie_goes_to_lowest_index():
    """The oracle's decoder resolves a planted exact logit tie through argmax_checked:
    tokens are j1 where the tied value is positive, else the lowest index with a zero
    logit (0 here, since j1 > 0)."""
    shape = synth.TINY
    j1, j2, col = 37, 101, 5
    w = tie_head_weights(shape, 3, j1, j2, col)
    m = Oracle(shape, w, capacity=64, rowwise=True)
    st = m.new_state()
    m.prefill(st, synth.make_prompt(shape, 12, 3))
    g, lg = m.verify_block(st, [5, 9, 200, 1000])
    seen = set()
    for j, tok in enumerate(g):
        row = lg[j]
        assert float(row[j1]) == float(row[j2])
        expect = j1 if float(row[j1]) > 0 else 0
        assert tok == expect
        seen.add(expect)
    assert seen  # at least one row checked

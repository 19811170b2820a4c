"""Pins for greedy consensus: the longest draft prefix equal to the AR argmax is
accepted and the AR token at the first mismatch is committed (Hacker News
summary, 'Idea'; atlas.scime.ai summary, 'Approach')."""
import itertools

import pytest

from oracle import accept_length, committed_tokens


def leading_ones(mask_bits: int, K: int) -> int:
    # count of trailing set bits of the match mask, capped at K (bit i = match of d_{i+1})
    return min(K, ((~mask_bits) & (mask_bits + 1)).bit_length() - 1)


@pytest.mark.parametrize("K", range(1, 9))
def test_accept_exhaustive(K):
    ar = [100 + j for j in range(K + 1)]
    for pattern in itertools.product([0, 1], repeat=K):
        drafts = [ar[i] if pattern[i] else 7 for i in range(K)]
        bits = sum(1 << i for i in range(K) if pattern[i])
        a = accept_length(drafts, ar)
        assert a == leading_ones(bits, K)
        toks = committed_tokens(drafts, ar, a)
        assert len(toks) == a + 1
        assert toks[:a] == ar[:a] and toks[-1] == ar[a]


def test_accept_hand_cases():
    g = [5, 6, 7, 8]
    assert accept_length([5, 6, 7], g) == 3 and committed_tokens([5, 6, 7], g, 3) == [5, 6, 7, 8]
    assert accept_length([9, 6, 7], g) == 0 and committed_tokens([9, 6, 7], g, 0) == [5]
    assert accept_length([5, 9, 7], g) == 1 and committed_tokens([5, 9, 7], g, 1) == [5, 6]
    assert accept_length([5, 6, 9], g) == 2
    assert accept_length([], [4]) == 0 and committed_tokens([], [4], 0) == [4]

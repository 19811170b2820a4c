"""Dynamic block size: the plain definitions the library's policy is checked against.

TEST INFRASTRUCTURE ONLY. Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import this module. The
library never calls it and shares no code with it.

The pages leave the block size to future work: choose K by how certain the
generation is, larger for predictable text such as code completion, smaller for
open-ended text (news article, "Future Directions: Larger K and Higher
Acceptance", item 1). Readings taken here, since the pages give no formula:

* certainty is the per-position acceptance rate alpha: each draft is accepted
  with probability alpha, independently, until the first rejection, so the accept
  length of a block of K drafts has P(a >= j) = alpha^j for j <= K, and the step
  commits a + 1 tokens;
* alpha of a sequence is estimated from its accept lengths: a step with a < K
  shows a accepted positions and one rejection, a step with a = K shows K accepted
  positions and no rejection (the block ended first). The counts are forgotten
  exponentially (factor ``decay`` per step) and read with Laplace's rule of
  succession, (accepted + 1) / (accepted + rejected + 2);
* among candidate block sizes with measured step times, the policy takes the one
  that commits the most tokens per unit time, summed over the batch; ties go to
  the smaller K.
"""
from __future__ import annotations


def expected_committed(alpha: float, K: int) -> float:
    """E[a + 1] for a block of K drafts: sum over j = 0..K of P(a >= j) = alpha^j."""
    return sum(alpha ** j for j in range(K + 1))


def accept_rate(accepted: float, rejected: float) -> float:
    return (accepted + 1.0) / (accepted + rejected + 2.0)


def update_stats(stats, accept_lens, K: int, decay: float = 1.0):
    """stats: list of [accepted, rejected] per sequence, updated in place."""
    for b, a in enumerate(accept_lens):
        if a < 0:
            continue
        stats[b][0] = decay * stats[b][0] + a
        stats[b][1] = decay * stats[b][1] + (1.0 if a < K else 0.0)
    return stats


def choose_block_size(stats, ks, step_ms) -> int:
    best_k, best = None, None
    for k, t in zip(ks, step_ms):
        rate = sum(expected_committed(accept_rate(acc, rej), k) for acc, rej in stats) / t
        if best is None or rate > best or (rate == best and k < best_k):
            best_k, best = k, rate
    return best_k

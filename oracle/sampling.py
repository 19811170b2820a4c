"""CPU oracle of Orthrus decoding at temperature T > 0 (speculative rejection sampling).

TEST INFRASTRUCTURE ONLY. Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import this module. The
CUDA library never calls it and shares no code with it.

The pages name the mode and no more: sampling at T > 0 goes through rejection
sampling, described only briefly (atlas summary "Limitations"; Hacker News
summary "Limitations": greedy and rejection sampling are the two modes). The
reading taken here is standard speculative sampling (Leviathan, Kalman and
Matias, "Fast Inference from Transformers via Speculative Decoding", 2023;
Chen et al., "Accelerating Large Language Model Decoding with Speculative
Sampling", 2023), applied to the Orthrus block:

* draft-view row i (i = 0..K-1) gives q_i = softmax(z^d_i / T); the drafts are
  drawn independently, d_{i+1} ~ q_i (the block is projected in one pass, so
  no draft is conditioned on another);
* verify-view row j (j = 0..K) gives p_j = softmax(z^v_j / T), the frozen
  model's next-token distribution after [y, d_1..d_j];
* for i = 1..K in order: accept d_i iff u_i * q_{i-1}(d_i) < p_{i-1}(d_i)
  (i.e. u_i < min(1, p/q) with u_i uniform on [0, 1)), stop at the first
  rejection; a = number accepted;
* the last committed token is drawn with a further uniform v: from the
  residual max(0, p_a - q_a) (normalised) when d_{a+1} was rejected, else
  from p_K (the bonus token). The pages leave open a residual that is zero
  everywhere, which needs p_a == q_a and a draft of zero draft probability;
  the reading here draws from p_a then, the target distribution itself;
* committed = d_1..d_a and that token; the cache and pending-token bookkeeping
  is the greedy step's (n += a + 1, y = last committed).

Every random number is an input (a uniform on [0, 1)), so the step is a
deterministic function that the GPU path can be compared with. A categorical
draw from unnormalised weights w with a uniform v is the inverse CDF: the
smallest index j with C_j > v * Z, where C_j = w_0 + .. + w_j and Z = C_{V-1};
an index of zero weight is never chosen. With these definitions the committed
tokens are distributed as sampling from the frozen model at temperature T,
whatever the drafts' distribution (the cited papers' theorem; pinned here by
exact and statistical tests).
Arithmetic is float64.
"""
from __future__ import annotations

import numpy as np
import torch

F64 = torch.float64


def _f64(x) -> torch.Tensor:
    """A row as float64 (exact for float32 inputs; lists are read as float64)."""
    if isinstance(x, torch.Tensor):
        return x.to(F64)
    return torch.from_numpy(np.asarray(x, dtype=np.float64))


def tempered_weights(logits_row, T: float) -> torch.Tensor:
    """Unnormalised softmax weights exp((z - max z) / T) of one logits row, float64."""
    z = _f64(logits_row)
    if torch.isnan(z).any():
        raise FloatingPointError("NaN logit")
    if not T > 0:
        raise ValueError("temperature must be positive")
    return torch.exp((z - z.max()) / T)


def tempered_probs(logits_row, T: float) -> torch.Tensor:
    """softmax(z / T) of one logits row, float64."""
    w = tempered_weights(logits_row, T)
    return w / w.sum()


def inverse_cdf(weights, v: float) -> int:
    """Categorical draw from non-negative weights with the uniform v in [0, 1):
    the smallest j with C_j > v * Z (C = cumulative sum, Z = total). If rounding
    leaves no such j (v * Z >= Z), the last index of positive weight."""
    w = _f64(weights)
    if (w < 0).any() or not (0.0 <= v < 1.0):
        raise ValueError("weights must be >= 0 and v in [0, 1)")
    c = torch.cumsum(w, 0)
    Z = float(c[-1])
    if not Z > 0:
        raise ValueError("all weights are zero")
    above = torch.nonzero(c > v * Z)
    if len(above):
        return int(above[0, 0])
    return int(torch.nonzero(w > 0)[-1, 0])


def sample_tokens(logits, T: float, uniforms):
    """One categorical draw per row of ``logits`` [R][V] from softmax(row / T),
    with uniforms [R]."""
    return [inverse_cdf(tempered_weights(logits[r], T), float(uniforms[r])) for r in range(len(uniforms))]


def speculative_accept(drafts, q, p, u_accept, v_final):
    """Rejection-sampling consensus of one block.

    drafts [K] = d_1..d_K; q [K][V] = draft distributions q_0..q_{K-1};
    p [K+1][V] = verify distributions p_0..p_K (rows of probabilities);
    u_accept [K], v_final: uniforms on [0, 1).
    Returns (a, committed) with committed = d_1..d_a, last token.
    """
    K = len(drafts)
    a = 0
    while a < K:
        d = int(drafts[a])
        if float(u_accept[a]) * float(q[a][d]) < float(p[a][d]):
            a += 1
        else:
            break
    if a < K:
        resid = torch.clamp(_f64(p[a]) - _f64(q[a]), min=0.0)
        # The residual is empty only when p_a == q_a and d_{a+1} lies outside q_a's support
        # (a draft the draft view gives probability zero, so never one drawn from it): the
        # rejection then says nothing and the last token is drawn from p_a itself.
        last = inverse_cdf(resid if float(resid.sum()) > 0 else _f64(p[a]), float(v_final))
    else:
        last = inverse_cdf(_f64(p[K]), float(v_final))
    return a, [int(t) for t in drafts[:a]] + [last]


def accept_sample_logits(drafts, draft_logits, verify_logits, T: float, u_accept, v_final):
    """``speculative_accept`` on logits: q_i = softmax(draft row i / T),
    p_j = softmax(verify row j / T)."""
    K = len(drafts)
    q = [tempered_probs(draft_logits[i], T) for i in range(K)]
    p = [tempered_probs(verify_logits[j], T) for j in range(K + 1)]
    return speculative_accept(drafts, q, p, u_accept, v_final)


def sampled_step(model, st, K: int, T: float, u_draft, u_accept, v_final):
    """One Orthrus step at temperature T on the oracle decoder: draft view,
    drafts drawn from it, verify view, rejection-sampling consensus, commit.
    Returns (drafts, a, committed)."""
    _, dlog = model.draft_block(st, K)
    drafts = sample_tokens(dlog, T, u_draft)
    _, vlog = model.verify_block(st, drafts)
    a, toks = accept_sample_logits(drafts, dlog, vlog, T, u_accept, v_final)
    st.n += a + 1
    st.y = toks[-1]
    st.out.extend(toks)
    return drafts, a, toks


def step_uniforms(rng: np.random.Generator, B: int, K: int):
    """The uniforms one sampled step draws, as float32 (the GPU's input type):
    drafts [B][K], accept tests [B][K], last token [B]."""
    f = lambda *s: rng.random(s, dtype=np.float32)
    return f(B, K), f(B, K), f(B)

"""CPU oracle of the Orthrus dual-view decode step.

TEST INFRASTRUCTURE ONLY. Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import this module. The
CUDA library never calls it and shares no code with it.

Plain float64 PyTorch CPU arithmetic, written from the method's description:

* Orthrus (abstract; atlas summary "Approach"): a frozen autoregressive (AR)
  decoder builds the KV cache; a trainable attention path per layer (the
  "diffusion view") predicts a block of K tokens in one forward pass over the
  same cache; the frozen AR view then verifies the block, and greedy consensus
  keeps the longest draft prefix that matches the AR argmax, so the output
  equals greedy AR decoding (HN summary "Idea"; atlas "Approach").
* Only base-view K/V of committed tokens ever enters the one shared cache; the
  draft view's in-block K/V is per-step scratch (HN summary "Results": O(1)
  KV overhead; news article "KV Cache Overhead").

Readings where the pages are silent (each is stated where it is used):

* State: the cache holds positions [0, n); the pending token y sits at
  position n and has no K/V yet.
* Draft block = [y, MASK x (K-1)] at positions n..n+K-1; block row i predicts
  position n+1+i with the frozen LM head. Draft keys = cache[0, n) plus the
  block's draft-view K/V, all visible to every block row (bidirectional).
* Verify block = [y, d_1..d_K] at positions n..n+K with the frozen weights,
  causal; its base K/V is written into cache slots n..n+K, of which n..n+a
  become live after acceptance.
* Draft module = its own q/k/v/o projections (and q/k norm gains) with the
  shapes of the base attention; norms, MLP and LM head are the frozen ones.
* Accept: a = number of leading i with d_i == g_{i-1}; commit d_1..d_a, g_a.
* 2-step draft (atlas "Surprising findings"): a second draft-view pass over
  [y, d_1..d_{K-1}], the first pass's predictions in place of the masks.
* Decoder layer (Qwen3 style): pre-RMSNorm attention with optional per-head
  q/k RMSNorm and rotate-half RoPE, SwiGLU MLP, untied LM head.
* K/V are rounded to bfloat16 when stored (the model's cache dtype); weights
  are the given bfloat16 values; everything else is float64.
* Argmax ties resolve to the lowest index; a NaN logit is an error.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

F64 = torch.float64


def _bf16(arr: np.ndarray) -> torch.Tensor:
    """uint16 bfloat16 bit patterns -> a bfloat16 CPU tensor sharing the memory."""
    return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16)


def round_bf16(x: torch.Tensor) -> torch.Tensor:
    """Round to bfloat16 (the cache's storage type) and return as float64."""
    return x.to(torch.float32).to(torch.bfloat16).to(F64)


# ---------------------------------------------------------------------------
# Building blocks (each one a direct definition)
# ---------------------------------------------------------------------------

def rms_norm(x: torch.Tensor, gain: torch.Tensor, eps: float) -> torch.Tensor:
    """RMSNorm over the last axis: x * gain / sqrt(mean(x^2) + eps)."""
    return x / torch.sqrt((x * x).mean(dim=-1, keepdim=True) + eps) * gain


def silu(x: torch.Tensor) -> torch.Tensor:
    return x / (1.0 + torch.exp(-x))


def rope(x: torch.Tensor, positions: torch.Tensor, theta: float) -> torch.Tensor:
    """Rotate-half rotary embedding of x[..., Q, heads, d] at absolute positions[Q].

    Pairs (j, j + d/2) are rotated by angle pos * theta^(-2j/d).
    """
    d = x.shape[-1]
    half = d // 2
    j = torch.arange(half, dtype=F64)
    inv_freq = theta ** (-2.0 * j / d)
    ang = positions.to(F64)[:, None] * inv_freq[None, :]           # [Q, d/2]
    cos = torch.cos(ang)[:, None, :]
    sin = torch.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return torch.cat([x1 * cos - x2 * sin, x2 * cos + x1 * sin], dim=-1)


def linear(x: torch.Tensor, w: torch.Tensor, rowwise: bool) -> torch.Tensor:
    """y[i] = W x[i] for each row i; W is [out, in] (bf16 values)."""
    w64 = w.to(F64)
    if rowwise:
        return torch.stack([w64 @ x[i] for i in range(x.shape[0])]) if x.shape[0] else x.new_zeros((0, w.shape[0]))
    return x @ w64.T


def attention(q: torch.Tensor, keys: torch.Tensor, vals: torch.Tensor, n_visible) -> torch.Tensor:
    """Grouped-query attention, one query row and one head at a time.

    q: [Q, H, d]; keys/vals: [Hkv, N, d]; row i sees keys [0, n_visible[i]).
    Query head h reads KV head h // (H / Hkv). Returns [Q, H * d].
    """
    Q, H, d = q.shape
    Hkv = keys.shape[0]
    G = H // Hkv
    out = torch.empty((Q, H, d), dtype=F64)
    scale = 1.0 / math.sqrt(d)
    for i in range(Q):
        nv = int(n_visible[i])
        for h in range(H):
            kv = h // G
            s = (keys[kv, :nv] @ q[i, h]) * scale
            p = torch.exp(s - s.max())
            p = p / p.sum()
            out[i, h] = p @ vals[kv, :nv]
    return out.reshape(Q, H * d)


def attention_by_head(q: torch.Tensor, keys: torch.Tensor, vals: torch.Tensor, n_visible) -> torch.Tensor:
    """The same grouped-query attention, one head at a time over all query rows:
    scores of row i against keys [0, n_visible[i]) with the others masked to -inf, then
    the softmax and the weighted sum of the values. Keys past max(n_visible) are never
    read. Used when the rows need not be evaluated one at a time (long caches)."""
    Q, H, d = q.shape
    Hkv = keys.shape[0]
    G = H // Hkv
    nmax = int(max(n_visible)) if Q else 0
    out = torch.empty((Q, H, d), dtype=F64)
    mask = torch.arange(nmax)[None, :] < torch.as_tensor([int(x) for x in n_visible])[:, None]  # [Q, nmax]
    scale = 1.0 / math.sqrt(d)
    for h in range(H):
        kv = h // G
        s = (q[:, h] @ keys[kv, :nmax].T) * scale
        s = s.masked_fill(~mask, -math.inf)
        p = torch.exp(s - s.max(dim=1, keepdim=True).values)
        p = p / p.sum(dim=1, keepdim=True)
        out[:, h] = p @ vals[kv, :nmax]
    return out.reshape(Q, H * d)


def argmax_checked(logits_row: torch.Tensor) -> int:
    if torch.isnan(logits_row).any():
        raise FloatingPointError("NaN logit")
    return int(torch.argmax(logits_row))  # first maximal index on ties


def top2_margin(logits_row: torch.Tensor) -> float:
    v = torch.topk(logits_row, 2).values
    return float(v[0] - v[1])


# ---------------------------------------------------------------------------
# Accept rule (pure integer logic)
# ---------------------------------------------------------------------------

def accept_length(drafts, ar) -> int:
    """Number of leading draft tokens d_i (i = 1..K) equal to the AR token g_{i-1}.

    ``drafts`` = [d_1..d_K], ``ar`` = [g_0..g_K] (g_j is the verifier's argmax at
    block row j, i.e. its prediction for position n + j + 1).
    """
    a = 0
    while a < len(drafts) and int(drafts[a]) == int(ar[a]):
        a += 1
    return a


def committed_tokens(drafts, ar, a: int):
    """Greedy consensus: the accepted drafts d_1..d_a and the AR token g_a."""
    return [int(t) for t in drafts[:a]] + [int(ar[a])]


# ---------------------------------------------------------------------------
# The model
# ---------------------------------------------------------------------------

@dataclass
class SeqState:
    """One sequence: cache slots [0, n) are live; ``y`` is the pending token at position n."""

    k: list
    v: list
    n: int = 0
    y: int = -1
    out: list = field(default_factory=list)


class Oracle:
    """The decoder, its draft module and the Orthrus step, in float64.

    ``shape`` is any object with the attributes n_layers, d_model, n_heads,
    n_kv_heads, head_dim, d_ff, vocab, qk_norm, rope_theta, rms_eps, mask_id.
    ``weights`` maps tensor names to uint16 bfloat16 bits (matrices) or float32
    gains, with the row layouts: w_qkv rows = q heads | k heads | v heads;
    w_gate_up rows = gate | up.
    ``rowwise=True`` evaluates every linear layer and the attention one row at a
    time, so that a row's result never depends on which other rows share the block;
    otherwise rows are evaluated together (a matrix product per layer, attention one
    head at a time), which is faster and equal up to float64 rounding order.
    """

    def __init__(self, shape, weights: dict, capacity: int, rowwise: bool = False):
        self.s = shape
        self.cap = capacity
        self.rowwise = rowwise
        self.w = {}
        for name, arr in weights.items():
            if arr.dtype == np.uint16:
                self.w[name] = _bf16(arr)
            else:
                self.w[name] = torch.from_numpy(np.asarray(arr, dtype=np.float64))

    # -- state ------------------------------------------------------------
    def new_state(self) -> SeqState:
        """Cache slots hold bf16 values (K and V are rounded to bf16 when stored), so they
        are kept as bfloat16: lossless, and a quarter of the float64 footprint."""
        s = self.s
        k = [torch.zeros((s.n_kv_heads, self.cap, s.head_dim), dtype=torch.bfloat16) for _ in range(s.n_layers)]
        v = [torch.zeros((s.n_kv_heads, self.cap, s.head_dim), dtype=torch.bfloat16) for _ in range(s.n_layers)]
        return SeqState(k=k, v=v)

    # -- one forward over a block of positions n .. n+Q-1 -------------------
    def forward(self, st: SeqState, ids, view: str, last_only: bool = False,
                return_qkv: bool = False):
        """Run the block ``ids`` at positions st.n .. st.n+Q-1.

        view = "draft": draft q/k/v/o and norm gains; keys = cache[0, n) plus the
        block's own draft K/V, all visible to every block row.
        view = "verify": frozen weights, causal over cache[0, n) plus the block;
        the block's K/V is written to cache slots n .. n+Q-1 (n is not advanced).
        Returns logits [Q, V] (or [1, V] with last_only).
        """
        s = self.s
        w = self.w
        Q = len(ids)
        n = st.n
        if n + Q > self.cap:
            raise ValueError("cache capacity exceeded")
        H, Hkv, d, F = s.n_heads, s.n_kv_heads, s.head_dim, s.d_ff
        pos = torch.arange(n, n + Q)
        ids_t = torch.as_tensor(np.asarray(ids, dtype=np.int64))
        h = w["embed"][ids_t].to(F64)
        if view == "draft":
            n_visible = [n + Q] * Q
        elif view == "verify":
            n_visible = [n + i + 1 for i in range(Q)]
        else:
            raise ValueError(view)
        trace = []
        for l in range(s.n_layers):
            p = f"l{l}."
            pre = "wd_" if view == "draft" else "w_"
            gq = w[p + ("wd_q_norm" if view == "draft" else "q_norm")]
            gk = w[p + ("wd_k_norm" if view == "draft" else "k_norm")]
            x = rms_norm(h, w[p + "attn_norm"], s.rms_eps)
            qkv = linear(x, w[p + pre + "qkv"], self.rowwise)
            q = qkv[:, : H * d].reshape(Q, H, d)
            k = qkv[:, H * d:(H + Hkv) * d].reshape(Q, Hkv, d)
            v = qkv[:, (H + Hkv) * d:].reshape(Q, Hkv, d)
            if s.qk_norm:
                q = rms_norm(q, gq, s.rms_eps)
                k = rms_norm(k, gk, s.rms_eps)
            q = rope(q, pos, s.rope_theta)
            k = rope(k, pos, s.rope_theta)
            k = round_bf16(k)
            v = round_bf16(v)
            keys = torch.cat([st.k[l][:, :n].to(F64), k.permute(1, 0, 2)], dim=1)
            vals = torch.cat([st.v[l][:, :n].to(F64), v.permute(1, 0, 2)], dim=1)
            if view == "verify":  # bf16 values: stored exactly
                st.k[l][:, n:n + Q] = k.permute(1, 0, 2).to(torch.bfloat16)
                st.v[l][:, n:n + Q] = v.permute(1, 0, 2).to(torch.bfloat16)
            o = attention(q, keys, vals, n_visible) if self.rowwise else attention_by_head(q, keys, vals, n_visible)
            if return_qkv:
                trace.append({"q": q.clone(), "k": k.clone(), "v": v.clone(), "o": o.clone()})
            h = h + linear(o, w[p + pre + "o"], self.rowwise)
            x2 = rms_norm(h, w[p + "mlp_norm"], s.rms_eps)
            gu = linear(x2, w[p + "w_gate_up"], self.rowwise)
            act = silu(gu[:, :F]) * gu[:, F:]
            h = h + linear(act, w[p + "w_down"], self.rowwise)
        hf = rms_norm(h[-1:] if last_only else h, w["final_norm"], s.rms_eps)
        logits = linear(hf, w["lm_head"], self.rowwise)
        if return_qkv:
            return logits, trace
        return logits

    # -- the Orthrus calls --------------------------------------------------
    def prefill(self, st: SeqState, prompt) -> int:
        """AR prefill: cache slots [0, P) get the prompt's base K/V; the argmax at
        the last prompt row is the first generated token (it counts as token 1)."""
        assert st.n == 0
        logits = self.forward(st, prompt, "verify", last_only=True)
        st.n = len(prompt)
        st.y = argmax_checked(logits[0])
        st.out = [st.y]
        return st.y

    def draft_block(self, st: SeqState, K: int):
        """Draft view over [y, MASK x (K-1)]; d_{i+1} = argmax of block row i."""
        ids = [st.y] + [self.s.mask_id] * (K - 1)
        logits = self.forward(st, ids, "draft")
        return [argmax_checked(logits[i]) for i in range(K)], logits

    def draft_refine(self, st: SeqState, drafts):
        """Second denoising step of the draft view (atlas summary "Surprising findings":
        the 2-step iterative variant the single-step projection is compared with).

        The pages leave its mechanism open; the reading taken here is the plainest one:
        the masks of the first step are replaced by that step's predictions, i.e. the
        draft view runs again over [y, d_1..d_{K-1}] at positions n..n+K-1 (block row i
        still predicts position n+1+i, so d_K has no input slot and is not read), and
        the new argmaxes d'_1..d'_K replace the drafts."""
        K = len(drafts)
        ids = [st.y] + [int(t) for t in drafts[:K - 1]]
        logits = self.forward(st, ids, "draft")
        return [argmax_checked(logits[i]) for i in range(K)], logits

    def draft_steps(self, st: SeqState, K: int, steps: int):
        """``steps`` denoising steps of the draft view: the single-step block
        projection (steps = 1) followed by steps - 1 refinements."""
        drafts, logits = self.draft_block(st, K)
        for _ in range(steps - 1):
            drafts, logits = self.draft_refine(st, drafts)
        return drafts, logits

    def verify_block(self, st: SeqState, drafts):
        """Verify view over [y, d_1..d_K]; g_j = argmax of block row j (j = 0..K)."""
        ids = [st.y] + [int(t) for t in drafts]
        logits = self.forward(st, ids, "verify")
        return [argmax_checked(logits[j]) for j in range(len(ids))], logits

    def accept_commit(self, st: SeqState, drafts, ar):
        """Commit d_1..d_a, g_a: slots n..n+a become live, n += a+1, y = g_a."""
        a = accept_length(drafts, ar)
        toks = committed_tokens(drafts, ar, a)
        st.n += a + 1
        st.y = toks[-1]
        st.out.extend(toks)
        return a, toks

    def ar_step(self, st: SeqState) -> int:
        """Plain greedy AR: verify with K = 0, commit g_0."""
        g, _ = self.verify_block(st, [])
        self.accept_commit(st, [], g)
        return g[0]


def greedy_ar(model: Oracle, prompt, n_tokens: int):
    """Plain greedy decoding: the reference stream the Orthrus loop must reproduce."""
    st = model.new_state()
    model.prefill(st, prompt)
    while len(st.out) < n_tokens:
        model.ar_step(st)
    return st.out[:n_tokens]


def orthrus_generate(model: Oracle, prompt, n_tokens: int, K: int, drafter=None, draft_steps: int = 1):
    """The Orthrus loop. ``drafter(model, st, K)`` returns d_1..d_K; by default the
    draft view's argmax after ``draft_steps`` denoising steps. Returns
    (tokens[:n_tokens], accept lengths)."""
    st = model.new_state()
    model.prefill(st, prompt)
    accepts = []
    while len(st.out) < n_tokens:
        if drafter is None:
            drafts, _ = model.draft_steps(st, K, draft_steps)
        else:
            drafts = [int(t) for t in drafter(model, st, K)]
        g, _ = model.verify_block(st, drafts)
        a, _ = model.accept_commit(st, drafts, g)
        accepts.append(a)
    return st.out[:n_tokens], accepts

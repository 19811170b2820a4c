"""Closed-form sizes of the Orthrus decode step (test infrastructure only).

* Block scratch: the draft view's in-block K/V for every layer,
  2 (K and V) * L * B * K * Hkv * d elements of 2 bytes. The pages give the
  Orthrus KV overhead as about 4.5 MiB, flat (HN summary "Results"; news
  article "KV Cache Overhead").
* Draft-module share of parameters: the pages say about 16% of parameters are
  trained (HN summary "Results"; atlas "Key results").
* Tokens per forward: each decode step runs two forwards (draft and verify)
  and commits a + 1 tokens, so TPF = (a + 1) / 2.
"""


def scratch_bytes(shape, K: int, batch: int = 1) -> int:
    return 2 * shape.n_layers * batch * K * shape.n_kv_heads * shape.head_dim * 2


def param_counts(shape):
    """(base, draft) parameter counts; norm gains included, embedding and LM head untied."""
    D, H, Hkv, d, F, V, L = (shape.d_model, shape.n_heads, shape.n_kv_heads, shape.head_dim,
                             shape.d_ff, shape.vocab, shape.n_layers)
    attn = (H + 2 * Hkv) * d * D + D * H * d
    qk = 2 * d if shape.qk_norm else 0
    per_layer_base = attn + qk + 2 * F * D + D * F + 2 * D
    base = L * per_layer_base + 2 * V * D + D
    draft = L * (attn + qk)
    return base, draft


def draft_param_fraction(shape) -> float:
    base, draft = param_counts(shape)
    return draft / (base + draft)


def tokens_per_forward(mean_accept: float) -> float:
    return (mean_accept + 1.0) / 2.0

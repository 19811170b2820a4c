"""CPU oracle for the Orthrus dual-view decode step (test infrastructure only).

Imported only by the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline / reference leg. The CUDA library shares no code with it.
"""
from .model import (Oracle, SeqState, accept_length, argmax_checked, attention, attention_by_head, committed_tokens,
                    greedy_ar, linear, orthrus_generate, rms_norm, rope, round_bf16, silu, top2_margin)
from .sampling import (accept_sample_logits, inverse_cdf, sample_tokens, sampled_step, speculative_accept,
                       step_uniforms, tempered_probs, tempered_weights)
from .sizes import draft_param_fraction, param_counts, scratch_bytes, tokens_per_forward
from . import policy

__all__ = ["Oracle", "SeqState", "accept_length", "argmax_checked", "attention", "attention_by_head", "committed_tokens",
           "greedy_ar", "linear", "orthrus_generate", "rms_norm", "rope", "round_bf16", "silu",
           "top2_margin", "draft_param_fraction", "param_counts", "scratch_bytes", "tokens_per_forward",
           "accept_sample_logits", "inverse_cdf", "sample_tokens", "sampled_step", "speculative_accept",
           "step_uniforms", "tempered_probs", "tempered_weights", "policy"]

"""Plant plausible mistakes in the oracle (on the CPU, by patching its functions)
and check that the pins catch each of them."""
import numpy as np
import pytest
import torch

import oracle.model as om
import synth
from test_oracle_bruteforce import Micro, brute_run


def pinned_decoder_agrees() -> bool:
    s = Micro()
    w = synth.make_weights(s, 11, 12, std=0.3, gain_std=0.3, threads=1)
    prompt = [3, 1, 4, 1, 5, 9]
    m = om.Oracle(s, w, capacity=32, rowwise=True)
    st = m.new_state()
    m.prefill(st, prompt)
    _, lg = m.verify_block(st, [2, 6, 5])
    ref = brute_run(s, w, prompt, [st.y, 2, 6, 5], False)  # verify leaves st.y unchanged
    if not np.allclose(lg.numpy(), np.array(ref), rtol=1e-9, atol=1e-11):
        return False
    st2 = m.new_state()
    m.prefill(st2, prompt)
    _, lgd = m.draft_block(st2, 4)
    refd = brute_run(s, w, prompt, [st2.y] + [s.mask_id] * 3, True)
    return bool(np.allclose(lgd.numpy(), np.array(refd), rtol=1e-9, atol=1e-11))


def rope_wrong_sign(x, positions, theta):
    return om.__dict__["_orig_rope"](x, -positions, theta)


def rope_wrong_pairs(x, positions, theta):
    # interleaved (2j, 2j+1) pairing instead of rotate-half
    d = x.shape[-1]
    perm = torch.cat([torch.arange(0, d, 2), torch.arange(1, d, 2)])
    inv = torch.argsort(perm)
    return om.__dict__["_orig_rope"](x[..., perm], positions, theta)[..., inv]


def norm_without_gain(x, gain, eps):
    return om.__dict__["_orig_rms_norm"](x, torch.ones_like(gain), eps)


def silu_wrong(x):
    return x / (1.0 + torch.exp(x))


def attention_wrong_group(q, keys, vals, n_visible):
    Hkv = keys.shape[0]
    H = q.shape[1]
    G = H // Hkv
    order = torch.tensor([(h % Hkv) * G + h // Hkv for h in range(H)])  # head h reads kv head h % Hkv
    return om.__dict__["_orig_attention"](q[:, order], keys, vals, n_visible).reshape(q.shape[0], H, -1)[:, torch.argsort(order)].reshape(q.shape[0], -1)


def attention_off_by_one(q, keys, vals, n_visible):
    return om.__dict__["_orig_attention"](q, keys, vals, [max(1, v - 1) for v in n_visible])


def no_kv_rounding(x):
    return x


MUTATIONS = {
    "rope_sign": ("rope", rope_wrong_sign),
    "rope_pairs": ("rope", rope_wrong_pairs),
    "norm_gain_dropped": ("rms_norm", norm_without_gain),
    "silu_sign": ("silu", silu_wrong),
    "gqa_mapping": ("attention", attention_wrong_group),
    "mask_off_by_one": ("attention", attention_off_by_one),
    "kv_not_rounded": ("round_bf16", no_kv_rounding),
}


def test_unmutated_oracle_agrees():
    assert pinned_decoder_agrees()


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name, monkeypatch):
    fn_name, bad = MUTATIONS[name]
    monkeypatch.setitem(om.__dict__, "_orig_" + fn_name, getattr(om, fn_name))
    monkeypatch.setattr(om, fn_name, bad)
    assert not pinned_decoder_agrees()


def test_accept_off_by_one_is_caught(monkeypatch):
    from test_oracle_accept import leading_ones
    def bad(drafts, ar):
        a = 0
        while a < len(drafts) and int(drafts[a]) == int(ar[a + 1 if a + 1 < len(ar) else a]):
            a += 1
        return a
    ar = [100 + j for j in range(5)]
    drafts = ar[:4]
    assert om.accept_length(drafts, ar) == leading_ones(0b1111, 4)
    assert bad(drafts, ar) != leading_ones(0b1111, 4)

"""GPU parity of the greedy consensus against the oracle, through the C ABI.

- The fused step (orthrus_decode_step: draft forward, verify forward with the
  consensus in its last CTA) on the tiny decoder with drafts planted from the
  oracle's own greedy AR stream, so that long accepted prefixes occur: accept
  lengths, committed ids, cache length and pending token are compared with the
  oracle's accept_commit on its own verify argmaxes, bit-exact.
- Plain greedy AR on the GPU (verify with K = 0, then accept) against the
  oracle's greedy_ar, token for token.
- Exact logit ties: reading R8 (lowest index among equal maxima) on the
  persistent kernel and on the per-op kernels.

The losslessness these check is the pages' claim that the output equals greedy
AR decoding (HN summary "Idea"; atlas.scime.ai summary "Approach").

Where the oracle's top-2 logit margin is at most 0.1 the GPU may pick any token
within 0.1 of the maximum; the oracle then adopts the GPU's token (the follow
rule), and the tests count such rows.
"""
import copy

import numpy as np
import pytest
import torch

import synth
from oracle import Oracle, accept_length, greedy_ar, top2_margin
from test_oracle_argmax import tie_head_weights

pytestmark = pytest.mark.gpu

MARGIN = 0.1


def lib():
    from shared_kv_draft_b200 import orthrus
    return orthrus


def greedy_continuation(o, st, n_tokens):
    """st.out followed by the oracle's greedy AR tokens from state st (a copy is stepped)."""
    s2 = copy.deepcopy(st)
    while len(s2.out) < n_tokens:
        o.ar_step(s2)
    return s2.out


def adopt(tok, row):
    """Margin rule on one row: returns (token the oracle continues with, ambiguous?)."""
    best = int(torch.argmax(row))
    if top2_margin(row) > MARGIN:
        assert tok == best, (tok, best)
        return tok, False
    assert float(row[tok]) >= float(row[best]) - MARGIN, (tok, best)
    return tok, True


@pytest.mark.parametrize("shape", [synth.TINY, synth.TINY_QK], ids=["tiny", "tiny_qk"])
def test_fused_decode_step_matches_oracle_with_planted_greedy_drafts(shape):
    """Tiny config (64-token prompt, K = 8, 128 tokens). Each step's drafts are the
    oracle's greedy tokens for a planted prefix a ~ Geometric(mean 3), then a wrong
    token, then random ids; the step runs through orthrus_decode_step."""
    K, P, N = 8, 64, 128
    cap = P + N + K + 2
    w = synth.make_weights(shape, 21, 22, gain_std=0.1 if shape.qk_norm else 0.0)
    dev = lib().DeviceModel(shape, w, batch=1, capacity=cap, max_block=K, max_rows=64)
    o = Oracle(shape, w, capacity=cap)
    prompt = synth.make_prompt(shape, P, 23)
    stream = greedy_ar(o, prompt, N + K + 2)

    z = lambda *s: torch.zeros(s, dtype=torch.int32, device="cuda")
    pending, acc, com = z(1), z(1), z(1, K + 1)
    dev.prefill(torch.from_numpy(prompt).view(1, P).cuda(), [P], pending)
    torch.cuda.synchronize()
    st = o.new_state()
    o.prefill(st, prompt)
    assert int(pending.item()) == st.y == stream[0]

    accepts = synth.planted_accepts(200, 3.0, K, seed=24)
    rng = np.random.default_rng(25)
    n_ambiguous, a_seen = 0, []
    step = 0
    while len(st.out) < N:
        j = len(st.out) - 1  # generated index of the pending token
        if st.out != stream[:len(st.out)]:  # a near tie was followed: plant from the new greedy path
            stream = greedy_continuation(o, st, N + K + 2)
        d = synth.planted_drafts(np.array(stream), j, int(accepts[step]), K, shape.vocab, rng)
        dev.decode_step(pending, K, torch.from_numpy(d).view(1, K).cuda(), acc, com)
        torch.cuda.synchronize()
        assert dev.read_status() == 0
        a_gpu = int(acc.item())
        c_gpu = com[0].cpu().tolist()
        # the oracle's verify of the same drafts decides every token it can
        g_ref, vl = o.verify_block(st, d.tolist())
        # The GPU's verify argmaxes at rows 0..a are implied by its result: g_r = d_{r+1}
        # below a, g_a = the committed AR token. Where one differs from the oracle's, the
        # margin rule must allow it, and the oracle adopts it (follow rule).
        assert 0 <= a_gpu <= K
        g = list(g_ref)
        for r in range(a_gpu + 1):
            tok = int(d[r]) if r < a_gpu else int(c_gpu[a_gpu])
            if tok != g_ref[r]:
                g[r], amb = adopt(tok, vl[r])
                n_ambiguous += int(amb)
        a_ref, toks = o.accept_commit(st, d.tolist(), g)
        assert a_gpu == a_ref, (step, a_gpu, a_ref)
        assert c_gpu[:a_ref + 1] == toks and all(x == -1 for x in c_gpu[a_ref + 1:]), step
        assert int(dev.lens[0].item()) == st.n
        assert int(pending.item()) == st.y
        a_seen.append(a_gpu)
        step += 1
    assert max(a_seen) >= 4 and sum(a > 0 for a in a_seen) >= len(a_seen) // 3, a_seen
    if n_ambiguous == 0:
        assert st.out[:N] == greedy_ar(o, prompt, N)
    print(f"\n{shape.name}: {step} fused steps, accept lengths {a_seen}, {n_ambiguous} rows within the margin")


@pytest.mark.parametrize("shape", [synth.TINY, synth.TINY_QK], ids=["tiny", "tiny_qk"])
def test_gpu_greedy_ar_equals_oracle_greedy_ar(shape):
    """K = 0: one verify row per token through the persistent kernel, then the
    standalone accept; the stream equals the oracle's greedy AR stream."""
    P, N = 64, 96
    cap = P + N + 4
    w = synth.make_weights(shape, 31, 32, gain_std=0.1 if shape.qk_norm else 0.0)
    dev = lib().DeviceModel(shape, w, batch=1, capacity=cap, max_block=8, max_rows=64)
    o = Oracle(shape, w, capacity=cap)
    prompt = synth.make_prompt(shape, P, 33)
    z = lambda *s: torch.zeros(s, dtype=torch.int32, device="cuda")
    pending, acc, ar1, com1 = z(1), z(1), z(1, 1), z(1, 1)
    dev.prefill(torch.from_numpy(prompt).view(1, P).cuda(), [P], pending)
    gpu = [int(pending.item())]
    while len(gpu) < N:
        dev.verify_block(pending, None, 0, ar1)
        dev.accept_commit(pending, None, ar1, 0, acc, com1)
        gpu.append(int(com1.item()))
    torch.cuda.synchronize()
    assert dev.read_status() == 0
    assert int(dev.lens[0].item()) == P + N - 1
    # follow rule: the oracle steps along the GPU's stream, checking each token's row
    st = o.new_state()
    last = o.forward(o.new_state(), prompt, "verify", last_only=True)
    y, amb = adopt(gpu[0], last[0])
    n_amb = int(amb)
    o.prefill(st, prompt)
    st.y, st.out = y, [y]
    for tok in gpu[1:]:
        _, lg = o.verify_block(st, [])
        t, amb = adopt(tok, lg[0])
        n_amb += int(amb)
        o.accept_commit(st, [], [t])
    assert st.out == gpu
    if n_amb == 0:
        assert gpu == greedy_ar(o, prompt, N)
    print(f"\n{shape.name}: {N} greedy tokens, {n_amb} within the margin")


def test_exact_logit_tie_goes_to_lowest_index():
    """LM head zero except two equal rows j1 < j2 in one 128-row vocabulary tile: every
    logit row's maximum is an exact tie, {j1, j2} (value > 0) or all the zeros (value
    < 0, lowest index 0). Signed zeros are equal numbers, so they tie as well. Checked
    on the persistent kernel (draft and verify blocks, the fused step) and the per-op
    kernels (prefill, and a batch of 16 x 9 verify rows)."""
    shape = synth.TINY
    j1, j2, col = 37, 101, 5
    w = tie_head_weights(shape, 3, j1, j2, col)
    K, P = 8, 12
    cap = 64
    o = Oracle(shape, w, capacity=cap)

    def expected(row):
        assert float(row[j1]) == float(row[j2])
        v = float(row[j1])
        return None if abs(v) < 1e-3 else (j1 if v > 0 else 0)

    checked = {"persistent": 0, "per_op": 0}
    for B, path in [(1, "persistent"), (16, "per_op")]:
        dev = lib().DeviceModel(shape, w, batch=B, capacity=cap, max_block=K, max_rows=max(64, B * (K + 1)))
        toks = np.stack([synth.make_prompt(shape, P, 40 + b) for b in range(B)]).astype(np.int32)
        z = lambda *s: torch.zeros(s, dtype=torch.int32, device="cuda")
        pending, draft, ar = z(B), z(B, K), z(B, K + 1)
        dev.prefill(torch.from_numpy(toks).cuda(), [P] * B, pending)
        dev.draft_block(pending, K, draft)
        dev.verify_block(pending, draft, K, ar)
        torch.cuda.synchronize()
        assert dev.read_status() == 0
        for b in range(B):
            st = o.new_state()
            last = o.forward(o.new_state(), toks[b], "verify", last_only=True)
            e = expected(last[0])
            if e is not None:
                assert int(pending[b].item()) == e
                checked["per_op"] += 1
            o.prefill(st, toks[b])
            st.y = int(pending[b].item())
            _, dl = o.draft_block(st, K)
            for i in range(K):
                e = expected(dl[i])
                if e is not None:
                    assert int(draft[b, i].item()) == e, (b, i)
                    checked[path] += 1
            _, vl = o.verify_block(st, draft[b].cpu().tolist())
            for i in range(K + 1):
                e = expected(vl[i])
                if e is not None:
                    assert int(ar[b, i].item()) == e, (b, i)
                    checked[path] += 1
        if B == 1:
            # the fused consensus decodes the same keys
            acc, com = z(1), z(1, K + 1)
            st = o.new_state()
            o.prefill(st, toks[0])
            st.y = int(pending.item())
            dev.lens.fill_(P)
            planted = torch.full((1, K), j1, dtype=torch.int32, device="cuda")
            dev.decode_step(pending, K, planted, acc, com)
            torch.cuda.synchronize()
            assert dev.read_status() == 0
            g, vl = o.verify_block(st, [j1] * K)
            if all(expected(vl[i]) is not None for i in range(K + 1)):
                a_ref = accept_length([j1] * K, g)
                assert int(acc.item()) == a_ref
                assert com[0, a_ref].item() == g[a_ref]
                checked[path] += 1
    assert checked["persistent"] > 0 and checked["per_op"] > 0, checked
    print(f"\ntie rows checked: {checked}")

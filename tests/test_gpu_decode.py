"""End-to-end GPU parity of the Orthrus decode step on the tiny decoder, through
the C ABI, against the oracle.

Tolerances: logits max-abs <= 5e-2; token ids bit-exact wherever the oracle's
top-2 logit margin exceeds 0.1 (elsewhere the GPU's choice must lie within 0.1
of the oracle's maximum, and the oracle then adopts it so later steps stay
comparable); accept lengths, committed ids and cache lengths bit-exact.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import Oracle, top2_margin

pytestmark = pytest.mark.gpu

MARGIN = 0.1
LOGIT_TOL = 5e-2


def lib():
    from shared_kv_draft_b200 import orthrus
    return orthrus


class Stats:
    def __init__(self):
        self.checked = 0
        self.ambiguous = 0
        self.differed = 0
        self.max_logit_err = 0.0


def check_tokens(gpu_ids, ref_logits, stats):
    """Apply the margin rule row by row; return the ids the oracle adopts."""
    out = []
    for j, t in enumerate(gpu_ids):
        row = ref_logits[j]
        best = int(torch.argmax(row))
        stats.checked += 1
        if top2_margin(row) > MARGIN:
            assert t == best, (j, t, best)
        else:
            stats.ambiguous += 1
            assert float(row[t]) >= float(row[best]) - MARGIN, (j, t, best)
        stats.differed += int(t != best)
        out.append(int(t))
    return out


def check_logits(gpu, ref, stats):
    err = float(np.abs(gpu - ref.numpy()).max())
    stats.max_logit_err = max(stats.max_logit_err, err)
    assert err <= LOGIT_TOL, err


def make_pair(shape, K, P, cap, seed=1, gain_std=0.0, batch=1):
    w = synth.make_weights(shape, seed, seed + 1, gain_std=gain_std)
    dev = lib().DeviceModel(shape, w, batch=batch, capacity=cap, max_block=K, max_rows=max(batch * (K + 1), 64))
    return w, dev


def gpu_tensors(B, K, V):
    z = lambda *s: torch.zeros(s, dtype=torch.int32, device="cuda")
    return dict(pending=z(B), draft=z(B, K), ar=z(B, K + 1), acc=z(B), com=z(B, K + 1),
                dlog=torch.zeros((B, K, V), device="cuda"), vlog=torch.zeros((B, K + 1, V), device="cuda"))


@pytest.mark.parametrize("shape", [synth.TINY, synth.TINY_QK], ids=["tiny", "tiny_qk"])
def test_tiny_config_orthrus_loop_matches_oracle(shape):
    """Tiny config: prompt of 64 uniform ids, K = 8, 128 generated tokens, drafts
    from the draft view; every step's draft and verify logits are checked."""
    K, P, N = 8, 64, 128
    cap = P + N + K + 2
    w, dev = make_pair(shape, K, P, cap, gain_std=0.1 if shape.qk_norm else 0.0)
    o = Oracle(shape, w, capacity=cap)
    prompt = synth.make_prompt(shape, P, 3)
    t = gpu_tensors(1, K, shape.vocab)
    dev.prefill(torch.from_numpy(prompt).view(1, P).cuda(), [P], t["pending"])
    st = o.new_state()
    o.prefill(st, prompt)
    stats = Stats()
    y = int(t["pending"].item())
    # the prefill's argmax is checked like any other token
    ref_last = o.forward(o.new_state(), prompt, "verify", last_only=True)
    assert check_tokens([y], ref_last, stats) == [y]
    st.y = y
    st.out = [y]
    gpu_out = [y]
    while len(gpu_out) < N:
        dev.draft_block(t["pending"], K, t["draft"], t["dlog"])
        dev.verify_block(t["pending"], t["draft"], K, t["ar"], t["vlog"])
        dev.accept_commit(t["pending"], t["draft"], t["ar"], K, t["acc"], t["com"])
        torch.cuda.synchronize()
        assert dev.read_status() == 0
        drafts = t["draft"][0].cpu().tolist()
        d_ref, dl_ref = o.draft_block(st, K)
        check_logits(t["dlog"][0].cpu().numpy(), dl_ref, stats)
        check_tokens(drafts, dl_ref, stats)
        g_ref, vl_ref = o.verify_block(st, drafts)
        check_logits(t["vlog"][0].cpu().numpy(), vl_ref, stats)
        g = check_tokens(t["ar"][0].cpu().tolist(), vl_ref, stats)
        a_ref, toks = o.accept_commit(st, drafts, g)
        a = int(t["acc"].item())
        assert a == a_ref
        com = t["com"][0].cpu().tolist()
        assert com[:a + 1] == toks and all(c == -1 for c in com[a + 1:])
        assert int(dev.lens[0].item()) == st.n
        assert int(t["pending"].item()) == st.y
        gpu_out.extend(toks)
    print(f"\n{shape.name}: {stats.checked} tokens checked, {stats.ambiguous} within margin, "
          f"{stats.differed} differing, max logit err {stats.max_logit_err:.3g}")


def test_planted_drafts_accept_exactly_and_match_greedy_ar():
    """All-correct drafts are accepted in full (a = K, K+1 tokens), a wrong first
    draft advances one token, and the committed stream equals greedy AR."""
    shape = synth.TINY_QK
    K, P, N = 6, 20, 60
    cap = P + N + 2 * K + 4
    w, dev = make_pair(shape, K, P, cap, seed=4)
    prompt = synth.make_prompt(shape, P, 4)
    # greedy AR on the GPU itself (verify with K = 0)
    t = gpu_tensors(1, K, shape.vocab)
    dev.prefill(torch.from_numpy(prompt).view(1, P).cuda(), [P], t["pending"])
    stream = [int(t["pending"].item())]
    ar1 = torch.zeros((1, 1), dtype=torch.int32, device="cuda")
    com1 = torch.zeros((1, 1), dtype=torch.int32, device="cuda")
    while len(stream) < N + K + 2:
        dev.verify_block(t["pending"], None, 0, ar1)
        dev.accept_commit(t["pending"], None, ar1, 0, t["acc"], com1)
        stream.append(int(com1.item()))
    assert dev.read_status() == 0
    # restart the same model from the prompt and decode with planted drafts
    dev.lens.zero_()
    dev.prefill(torch.from_numpy(prompt).view(1, P).cuda(), [P], t["pending"])
    out = [int(t["pending"].item())]
    step = 0
    while len(out) < N:
        j = len(out) - 1  # generated index of the pending token
        drafts = stream[j + 1:j + 1 + K]
        if step % 3 == 1:
            drafts = [(drafts[0] + 1) % shape.vocab] + drafts[1:]
        t["draft"].copy_(torch.tensor([drafts], dtype=torch.int32))
        dev.verify_block(t["pending"], t["draft"], K, t["ar"])
        dev.accept_commit(t["pending"], t["draft"], t["ar"], K, t["acc"], t["com"])
        a = int(t["acc"].item())
        assert a == (0 if step % 3 == 1 else K)
        com = t["com"][0].cpu().tolist()
        out.extend(com[:a + 1])
        step += 1
    assert out[:N] == stream[:N]


def test_decode_step_with_planted_drafts_and_poisoned_dead_slots():
    """orthrus_decode_step with planted drafts reproduces the GPU's own greedy
    stream; NaN-poisoning the dead verify slots after every commit changes nothing."""
    shape = synth.TINY
    K, P, N = 8, 32, 80
    cap = P + N + 2 * K + 4
    w, dev = make_pair(shape, K, P, cap, seed=9)
    prompt = synth.make_prompt(shape, P, 9)
    tok = torch.from_numpy(prompt).view(1, P).cuda()
    t = gpu_tensors(1, K, shape.vocab)
    dev.prefill(tok, [P], t["pending"])
    stream = [int(t["pending"].item())]
    ar1 = torch.zeros((1, 1), dtype=torch.int32, device="cuda")
    com1 = torch.zeros((1, 1), dtype=torch.int32, device="cuda")
    while len(stream) < N + K + 2:
        dev.verify_block(t["pending"], None, 0, ar1)
        dev.accept_commit(t["pending"], None, ar1, 0, t["acc"], com1, poison_dead=True)
        stream.append(int(com1.item()))
    accepts = synth.planted_accepts(64, 3.0, K, seed=5)
    rng = np.random.default_rng(5)
    for poison in (False, True):
        dev.lens.zero_()
        dev.prefill(tok, [P], t["pending"])
        out = [int(t["pending"].item())]
        s = 0
        while len(out) < N:
            j = len(out) - 1
            a_plan = int(accepts[s])
            d = synth.planted_drafts(np.array(stream), j, a_plan, K, shape.vocab, rng)
            planted = torch.from_numpy(d).view(1, K).cuda()
            if poison:
                dev.draft_block(t["pending"], K, t["draft"])
                t["draft"].copy_(planted)
                dev.verify_block(t["pending"], t["draft"], K, t["ar"])
                dev.accept_commit(t["pending"], t["draft"], t["ar"], K, t["acc"], t["com"], poison_dead=True)
            else:
                dev.decode_step(t["pending"], K, planted, t["acc"], t["com"])
            a = int(t["acc"].item())
            assert a == a_plan
            out.extend(t["com"][0].cpu().tolist()[:a + 1])
            s += 1
        assert out[:N] == stream[:N], poison
        assert dev.read_status() == 0


def test_capacity_overrun_is_reported_and_nothing_commits():
    shape = synth.TINY
    K, P = 8, 16
    cap = P + K  # one slot short for a verify block of K + 1 rows
    w, dev = make_pair(shape, K, P, cap, seed=3)
    prompt = synth.make_prompt(shape, P, 3)
    t = gpu_tensors(1, K, shape.vocab)
    dev.prefill(torch.from_numpy(prompt).view(1, P).cuda(), [P], t["pending"])
    pend0 = int(t["pending"].item())
    dev.draft_block(t["pending"], K, t["draft"])
    dev.verify_block(t["pending"], t["draft"], K, t["ar"])
    dev.accept_commit(t["pending"], t["draft"], t["ar"], K, t["acc"], t["com"])
    torch.cuda.synchronize()
    assert dev.read_status() == lib().ERR_CAPACITY
    assert int(t["acc"].item()) == -1
    assert int(dev.lens[0].item()) == P and int(t["pending"].item()) == pend0
    dev.clear_status()
    torch.cuda.synchronize()
    assert dev.read_status() == 0


def test_batched_ragged_prefill_and_step():
    """Batch of 3 with different prompt lengths: each sequence's verify logits
    match the oracle run on that sequence alone."""
    shape = synth.TINY_QK
    K = 4
    lens = [20, 45, 33]
    cap = 64
    w, dev = make_pair(shape, K, max(lens), cap, seed=6, batch=3)
    o = Oracle(shape, w, capacity=cap)
    toks = np.zeros((3, max(lens)), dtype=np.int32)
    for b, L in enumerate(lens):
        toks[b, :L] = synth.make_prompt(shape, L, 20 + b)
    t = gpu_tensors(3, K, shape.vocab)
    dev.prefill(torch.from_numpy(toks).cuda(), lens, t["pending"])
    dev.draft_block(t["pending"], K, t["draft"], t["dlog"])
    dev.verify_block(t["pending"], t["draft"], K, t["ar"], t["vlog"])
    torch.cuda.synchronize()
    assert dev.read_status() == 0
    stats = Stats()
    for b, L in enumerate(lens):
        st = o.new_state()
        o.prefill(st, toks[b, :L])
        last = o.forward(o.new_state(), toks[b, :L], "verify", last_only=True)
        st.y = check_tokens([int(t["pending"][b].item())], last, stats)[0]
        _, dl = o.draft_block(st, K)
        check_logits(t["dlog"][b].cpu().numpy(), dl, stats)
        g, vl = o.verify_block(st, t["draft"][b].cpu().tolist())
        check_logits(t["vlog"][b].cpu().numpy(), vl, stats)
        check_tokens(t["ar"][b].cpu().tolist(), vl, stats)



def test_large_batch_per_op_path_matches_oracle():
    """Batch 16 with K = 8: 144 verify rows exceed the persistent kernel's 128, so draft and
    verify run through the per-op kernels. Every sequence's draft and verify logits and
    argmaxes match the oracle run on that sequence alone, and the accept/commit that
    follows is consistent with the drafts and the AR argmax (bit-exact)."""
    shape = synth.TINY_QK
    K, B = 8, 16
    rng = np.random.default_rng(77)
    lens = rng.integers(5, 60, size=B).tolist()
    cap = 80
    w, dev = make_pair(shape, K, max(lens), cap, seed=12, batch=B)
    o = Oracle(shape, w, capacity=cap)
    toks = np.zeros((B, max(lens)), dtype=np.int32)
    for b, L in enumerate(lens):
        toks[b, :L] = synth.make_prompt(shape, L, 300 + b)
    t = gpu_tensors(B, K, shape.vocab)
    dev.prefill(torch.from_numpy(toks).cuda(), lens, t["pending"])
    pend = t["pending"].cpu().numpy().copy()
    dev.draft_block(t["pending"], K, t["draft"], t["dlog"])
    dev.verify_block(t["pending"], t["draft"], K, t["ar"], t["vlog"])
    dev.accept_commit(t["pending"], t["draft"], t["ar"], K, t["acc"], t["com"])
    torch.cuda.synchronize()
    assert dev.read_status() == 0
    stats = Stats()
    drafts, ar = t["draft"].cpu().numpy(), t["ar"].cpu().numpy()
    acc, com = t["acc"].cpu().numpy(), t["com"].cpu().numpy()
    new_lens, new_pend = dev.lens.cpu().numpy(), t["pending"].cpu().numpy()
    for b, L in enumerate(lens):
        st = o.new_state()
        o.prefill(st, toks[b, :L])
        last = o.forward(o.new_state(), toks[b, :L], "verify", last_only=True)
        st.y = check_tokens([int(pend[b])], last, stats)[0]
        _, dl = o.draft_block(st, K)
        check_logits(t["dlog"][b].cpu().numpy(), dl, stats)
        check_tokens(drafts[b].tolist(), dl, stats)
        _, vl = o.verify_block(st, drafts[b].tolist())
        check_logits(t["vlog"][b].cpu().numpy(), vl, stats)
        check_tokens(ar[b].tolist(), vl, stats)
        # the consensus on the GPU's own drafts and AR argmax, bit-exact
        a = 0
        while a < K and drafts[b, a] == ar[b, a]:
            a += 1
        assert acc[b] == a, (b, acc[b], a)
        assert com[b, :a].tolist() == drafts[b, :a].tolist() and com[b, a] == ar[b, a], b
        assert (com[b, a + 1:] == -1).all(), b
        assert new_lens[b] == L + a + 1 and new_pend[b] == ar[b, a], b
    print(stats)


@pytest.mark.parametrize("B,K", [(1, 33), (4, 8), (2, 17), (2, 32), (3, 24), (4, 16), (1, 64)],
                         ids=["rows34", "rows36", "rows36_b2", "rows66", "rows75", "rows68", "rows65"])
def test_token_rows_past_32_match_oracle(B, K):
    """Blocks of 34-96 token rows on the persistent kernel: the projections' epilogues handle
    a second group of token columns past the first 32 (the 33rd row of a K = 32 verify
    block) and further 32-row groups, including split tiles with several rounds of
    contributors (the tiny model's down projection splits each tile over six CTAs). Draft
    and verify logits and argmaxes of every sequence match the oracle."""
    shape = synth.TINY_QK
    rng = np.random.default_rng(90 + B)
    lens = rng.integers(10, 40, size=B).tolist()
    cap = 40 + K + 8
    w, dev = make_pair(shape, K, max(lens), cap, seed=13 + B, batch=B)
    o = Oracle(shape, w, capacity=cap)
    toks = np.zeros((B, max(lens)), dtype=np.int32)
    for b, L in enumerate(lens):
        toks[b, :L] = synth.make_prompt(shape, L, 400 + b)
    t = gpu_tensors(B, K, shape.vocab)
    dev.prefill(torch.from_numpy(toks).cuda(), lens, t["pending"])
    pend = t["pending"].cpu().numpy().copy()
    dev.draft_block(t["pending"], K, t["draft"], t["dlog"])
    dev.verify_block(t["pending"], t["draft"], K, t["ar"], t["vlog"])
    torch.cuda.synchronize()
    assert dev.read_status() == 0
    stats = Stats()
    drafts = t["draft"].cpu().numpy()
    for b, L in enumerate(lens):
        st = o.new_state()
        o.prefill(st, toks[b, :L])
        last = o.forward(o.new_state(), toks[b, :L], "verify", last_only=True)
        st.y = check_tokens([int(pend[b])], last, stats)[0]
        _, dl = o.draft_block(st, K)
        check_logits(t["dlog"][b].cpu().numpy(), dl, stats)
        check_tokens(drafts[b].tolist(), dl, stats)
        _, vl = o.verify_block(st, drafts[b].tolist())
        check_logits(t["vlog"][b].cpu().numpy(), vl, stats)
        check_tokens(t["ar"][b].cpu().tolist(), vl, stats)

"""Dynamic block size on the GPU: the policy (orthrus_choose_block_size, fed by
orthrus_accept_stats_update) picks K for every step of an Orthrus loop on the tiny
decoder, and the committed stream still equals the oracle's greedy AR decoding
(HN summary "Idea": the output equals greedy AR decoding, whatever the drafts).

Drafts are planted from the oracle's greedy stream: the accept length of each step is
drawn from the acceptance process the policy models, with a per-position rate that
alternates between a predictable phase (0.9) and an open-ended one (0.3). The test
checks that the chosen K follows the phases (larger in the predictable phase), that
every step's accept length, committed ids, cache length and pending token equal the
oracle's consensus on its own verify argmaxes (bit-exact, with the 0.1 margin rule),
and that the stream equals greedy AR.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import Oracle, greedy_ar, top2_margin
from test_gpu_consensus import greedy_continuation

pytestmark = pytest.mark.gpu

MARGIN = 0.1


def planted_length(alpha, K, rng):
    a = 0
    while a < K and rng.random() < alpha:
        a += 1
    return a


def test_dynamic_block_size_loop_equals_greedy_ar():
    from shared_kv_draft_b200 import orthrus
    shape = synth.TINY_QK
    P, N, KMAX = 64, 160, 8
    ks, step_ms = [2, 4, 8], [1.1, 1.2, 1.4]  # a step-time table with a per-K cost
    cap = P + N + KMAX + 2
    w = synth.make_weights(shape, 41, 42, gain_std=0.1)
    dev = orthrus.DeviceModel(shape, w, batch=1, capacity=cap, max_block=KMAX, max_rows=64)
    o = Oracle(shape, w, capacity=cap)
    prompt = synth.make_prompt(shape, P, 43)
    stream = greedy_ar(o, prompt, N + KMAX + 2)

    z = lambda *s: torch.zeros(s, dtype=torch.int32, device="cuda")
    pending, acc, com = z(1), z(1), z(1, KMAX + 1)
    dev.prefill(torch.from_numpy(prompt).view(1, P).cuda(), [P], pending)
    st = o.new_state()
    o.prefill(st, prompt)
    torch.cuda.synchronize()
    assert int(pending.item()) == st.y == stream[0]

    stats = orthrus.accept_stats(1)
    rng = np.random.default_rng(44)
    chosen = {0.9: [], 0.3: []}
    step, followed = 0, 0
    while len(st.out) < N:
        alpha = 0.9 if (step // 8) % 2 == 0 else 0.3
        K = orthrus.choose_block_size(stats, ks, step_ms)
        chosen[alpha].append(K)
        a_plan = planted_length(alpha, K, rng)
        j = len(st.out) - 1
        if st.out != stream[:len(st.out)]:  # a near tie was followed: plant from the new greedy path
            stream = greedy_continuation(o, st, N + KMAX + 2)
        d = synth.planted_drafts(np.array(stream), j, a_plan, K, shape.vocab, rng)
        dev.decode_step(pending, K, torch.from_numpy(d).view(1, K).cuda(), acc, com[:, :K + 1])
        torch.cuda.synchronize()
        assert dev.read_status() == 0
        a_gpu = int(acc.item())
        c_gpu = com[0, :K + 1].cpu().tolist()
        g_ref, vl = o.verify_block(st, d.tolist())
        g = list(g_ref)
        for r in range(a_gpu + 1):
            tok = int(d[r]) if r < a_gpu else int(c_gpu[a_gpu])
            if tok != g_ref[r]:  # allowed only within the margin; the oracle then follows
                best = int(torch.argmax(vl[r]))
                assert top2_margin(vl[r]) <= MARGIN and float(vl[r][tok]) >= float(vl[r][best]) - MARGIN
                g[r] = tok
                followed += 1
        a_ref, toks = o.accept_commit(st, d.tolist(), g)
        assert a_gpu == a_ref
        assert c_gpu[:a_ref + 1] == toks and all(x == -1 for x in c_gpu[a_ref + 1:])
        assert int(dev.lens[0].item()) == st.n and int(pending.item()) == st.y
        orthrus.accept_stats_update(stats, [a_gpu], K, decay=0.7)
        step += 1
    if followed == 0:  # the GPU took no near-tie token differently: the stream is greedy AR itself
        assert st.out[:N] == greedy_ar(o, prompt, N)
    hi, lo = np.mean(chosen[0.9][2:]), np.mean(chosen[0.3][2:])
    print(f"\n{step} steps; mean K chosen: {hi:.2f} in the predictable phase, {lo:.2f} in the open-ended one")
    assert hi > lo

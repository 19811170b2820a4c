"""GPU parity, through the C ABI, of the two decoding variants around the greedy step:

* the 2-step iterative draft (atlas summary "Surprising findings"): orthrus_draft_refine
  against the oracle's refinement on the GPU's own first-step drafts, in place and out of
  place, on the persistent kernel and the per-op kernels, and orthrus_decode_step_ex with
  two draft steps against the same calls made one by one (bit-exact);
* decoding at temperature T > 0 by rejection sampling (atlas summary "Limitations"):
  orthrus_sample_tokens, orthrus_accept_sample and orthrus_decode_step_sampled against
  the oracle fed the same fp32 logits and the same uniforms.

Tolerances. Logits max-abs <= 5e-2 and tokens by the 0.1 margin rule, as for the greedy
step. A sampling decision is taken in fp32 on the GPU and in fp64 by the oracle on the
same inputs; the two must agree exactly unless the oracle's value lies within a band of
the decision boundary that the fp32 arithmetic can cross:
- an inverse-CDF draw: the GPU's index j must have positive weight and satisfy
  C_{j-1} - TOL <= v <= C_j + TOL on the oracle's normalised fp64 CDF C, and must equal
  the oracle's index when no boundary lies within TOL of v. TOL = 5e-5: each fp32 weight
  carries a relative error below 3e-6 (an exp of an argument of magnitude < 30, rounded
  differences and products), and the fp32 running sum adds at most (5 + 5 + 256) roundings
  of 2^-24 each, 1.6e-5 relative; 5e-5 is three times that. For the residual
  max(0, p - q) the error is relative to p + q, so the band is TOL / Z_r on its
  normalised CDF (Z_r = sum of the residual);
- an accept test u q < p: the two sides agree unless |u q - p| <= 1e-4 max(u q, p).
Bookkeeping (accept length, committed ids, cache length, pending token) is then bit-exact.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

import synth
from oracle import Oracle, accept_sample_logits, inverse_cdf, tempered_probs, tempered_weights, top2_margin

pytestmark = pytest.mark.gpu

MARGIN = 0.1
LOGIT_TOL = 5e-2
TOL_CDF = 5e-5
TOL_ACCEPT = 1e-4


def lib():
    from shared_kv_draft_b200 import orthrus
    return orthrus


def i32(*s):
    return torch.zeros(s, dtype=torch.int32, device="cuda")


def check_tokens(gpu_ids, ref_logits):
    for j, t in enumerate(gpu_ids):
        row = ref_logits[j]
        best = int(torch.argmax(row))
        if top2_margin(row) > MARGIN:
            assert t == best, (j, t, best)
        else:
            assert float(row[t]) >= float(row[best]) - MARGIN, (j, t, best)


def check_logits(gpu, ref):
    err = float(np.abs(gpu - ref.numpy()).max())
    assert err <= LOGIT_TOL, err


# ---- the 2-step iterative draft ------------------------------------------------------------

@pytest.mark.parametrize("shape,B,K", [(synth.TINY, 1, 8), (synth.TINY_QK, 2, 16), (synth.TINY_QK, 16, 8)],
                         ids=["tiny_b1", "tiny_qk_b2", "tiny_qk_b16_per_op"])
def test_draft_refine_matches_oracle(shape, B, K):
    rng = np.random.default_rng(5 + B)
    lens = rng.integers(8, 40, size=B).tolist()
    cap = 48 + 2 * K
    w = synth.make_weights(shape, 31 + B, 32 + B, gain_std=0.1 if shape.qk_norm else 0.0)
    dev = lib().DeviceModel(shape, w, batch=B, capacity=cap, max_block=K, max_rows=max(B * (K + 1), 64))
    o = Oracle(shape, w, capacity=cap)
    toks = np.zeros((B, max(lens)), dtype=np.int32)
    for b, L in enumerate(lens):
        toks[b, :L] = synth.make_prompt(shape, L, 500 + b)
    V = shape.vocab
    pending, d1, d2 = i32(B), i32(B, K), i32(B, K)
    dl2 = torch.zeros((B, K, V), device="cuda")
    dev.prefill(torch.from_numpy(toks).cuda(), lens, pending)
    dev.draft_block(pending, K, d1)
    dev.draft_refine(pending, d1, K, d2, dl2)
    inplace = d1.clone()
    dev.draft_refine(pending, inplace, K, inplace)
    torch.cuda.synchronize()
    assert dev.read_status() == 0
    assert torch.equal(inplace, d2)  # in place: every id is read before any is written
    assert dev.lens.cpu().tolist() == lens  # the draft view leaves the cache alone
    first, second, pend = d1.cpu().tolist(), d2.cpu().tolist(), pending.cpu().tolist()
    for b, L in enumerate(lens):
        st = o.new_state()
        o.prefill(st, toks[b, :L])
        st.y = pend[b]  # the prefill's own token is checked by the greedy tests
        _, lg = o.draft_refine(st, first[b])
        check_logits(dl2[b].cpu().numpy(), lg)
        check_tokens(second[b], lg)


def test_two_step_decode_step_equals_the_calls_one_by_one():
    shape, B, K = synth.TINY_QK, 2, 8
    cap = 96
    w = synth.make_weights(shape, 41, 42, gain_std=0.1)
    dev = lib().DeviceModel(shape, w, batch=B, capacity=cap, max_block=K, max_rows=64)
    lens = [20, 33]
    toks = np.stack([synth.make_prompt(shape, 33, 600 + b) for b in range(B)]).astype(np.int32)
    pending = i32(B)
    dev.prefill(torch.from_numpy(toks).cuda(), lens, pending)
    lens0, pend0 = dev.lens.clone(), pending.clone()
    d, ar, acc, com = i32(B, K), i32(B, K + 1), i32(B), i32(B, K + 1)
    for step in range(3):
        dev.draft_block(pending, K, d)
        dev.draft_refine(pending, d, K, d)
        dev.verify_block(pending, d, K, ar)
        dev.accept_commit(pending, d, ar, K, acc, com)
    torch.cuda.synchronize()
    ref = (dev.lens.clone(), pending.clone(), acc.clone(), com.clone())
    dev.lens.copy_(lens0)
    pending.copy_(pend0)
    acc2, com2 = i32(B), i32(B, K + 1)
    for step in range(3):
        dev.decode_step_ex(pending, K, 2, None, acc2, com2)
    torch.cuda.synchronize()
    assert dev.read_status() == 0
    assert torch.equal(dev.lens, ref[0]) and torch.equal(pending, ref[1])
    assert torch.equal(acc2, ref[2]) and torch.equal(com2, ref[3])


# ---- categorical draws ---------------------------------------------------------------------

def cdf_band_ok(weights, v, j, j_ref, tol):
    """The GPU's draw j against the oracle's j_ref: equal, or inside the rounding band."""
    w = np.asarray(weights, dtype=np.float64)
    if j == j_ref:
        return True, False
    if not (0 <= j < len(w)) or w[j] <= 0:
        return False, True
    C = np.cumsum(w) / w.sum()
    lo = C[j - 1] if j > 0 else 0.0
    return bool(lo - tol <= v <= C[j] + tol), True


def logits_rows(rng, R, V):
    x = rng.normal(0.0, 2.5, (R, V)).astype(np.float32)
    x[0, rng.integers(0, V, V // 3)] = -np.inf     # masked tokens: weight zero
    if R > 1:
        x[1, rng.integers(0, V)] += 40.0           # one dominant token
    if R > 2:
        x[2] = rng.normal(0.0, 0.01, V)            # near uniform
    return x


@pytest.mark.parametrize("V", [1000, 3149, 151936], ids=["v1000", "v3149", "v151936"])
@pytest.mark.parametrize("T", [0.6, 1.0, 1.7])
def test_sample_tokens_matches_oracle(V, T):
    rng = np.random.default_rng(V + int(10 * T))
    R = 12
    x = logits_rows(rng, R, V)
    u = rng.random(R, dtype=np.float32)
    u[3], u[4] = 0.0, np.float32(1.0 - 2.0 ** -24)  # both ends of [0, 1)
    out, status = i32(R), i32(1)
    lib().sample_tokens(torch.from_numpy(x).cuda(), T, torch.from_numpy(u).cuda(), out, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    got = out.cpu().tolist()
    near = 0
    for r in range(R):
        w = tempered_weights(torch.from_numpy(x[r]), T)
        ref = inverse_cdf(w, float(u[r]))
        ok, amb = cdf_band_ok(w.numpy(), float(u[r]), got[r], ref, TOL_CDF)
        assert ok, (r, got[r], ref)
        near += amb
    assert got[1] == int(np.argmax(x[1]))
    assert near <= 1, near


def test_sample_tokens_flags_nan_rows():
    x = np.zeros((3, 2048), dtype=np.float32)
    x[1, 77] = np.nan
    x[2, :] = -np.inf
    out, status = i32(3), i32(1)
    lib().sample_tokens(torch.from_numpy(x).cuda(), 1.0, torch.full((3,), 0.5, device="cuda"), out, status)
    torch.cuda.synchronize()
    assert int(status.item()) == lib().ERR_NAN
    o = out.cpu().tolist()
    assert o[1] == -1 and o[2] == -1 and o[0] == 1024  # uniform row, v = 0.5: index 1024 (C = 1025/2048)


# ---- the rejection-sampling consensus ------------------------------------------------------

def check_consensus(drafts, dl, vl, T, ua, uf, a_gpu, com_gpu):
    """The GPU's accept length and committed ids for one sequence against the oracle on the
    same fp32 logits and uniforms; returns 1 if a decision fell inside a rounding band."""
    K = len(drafts)
    q = [tempered_probs(torch.from_numpy(dl[i]), T).numpy() for i in range(K)]
    p = [tempered_probs(torch.from_numpy(vl[j]), T).numpy() for j in range(K + 1)]
    a_ref, toks_ref = accept_sample_logits(drafts, torch.from_numpy(dl), torch.from_numpy(vl), T, ua, uf)
    near = 0
    for i in range(min(a_gpu, a_ref) + 1):
        if i < K:
            lhs, rhs = float(ua[i]) * q[i][drafts[i]], p[i][drafts[i]]
            near |= abs(lhs - rhs) <= TOL_ACCEPT * max(lhs, rhs)
    if not near:
        assert a_gpu == a_ref, (a_gpu, a_ref)
    else:
        for i in range(a_gpu):  # the GPU's accepted drafts pass the test within the band
            lhs, rhs = float(ua[i]) * q[i][drafts[i]], p[i][drafts[i]]
            assert lhs < rhs * (1 + TOL_ACCEPT), i
    a = a_gpu
    assert com_gpu[:a] == list(drafts[:a]) and all(c == -1 for c in com_gpu[a + 1:])
    if a < K:
        w = np.maximum(p[a] - q[a], 0.0)
        tol = TOL_CDF / w.sum()
    else:
        w = p[K]
        tol = TOL_CDF
    ref_last = inverse_cdf(w, float(uf)) if a == a_ref else -1
    ok, amb = cdf_band_ok(w, float(uf), com_gpu[a], ref_last, tol)
    if a == a_ref and not amb:
        assert com_gpu[a] == toks_ref[-1]
    assert ok, (a, com_gpu[a], ref_last)
    return int(near or amb)


@pytest.mark.parametrize("V,B,K", [(1024, 4, 8), (3200, 3, 16), (3200, 2, 1), (1024, 4, 0)],
                         ids=["v1024_b4_k8", "v3200_b3_k16", "v3200_b2_k1", "v1024_b4_k0_ar"])
@pytest.mark.parametrize("T", [0.7, 1.3])
def test_accept_sample_matches_oracle(V, B, K, T):
    shape = replace(synth.TINY, name=f"tiny_v{V}", n_layers=1, vocab=V)
    w = synth.make_weights(shape, 71, 72)
    Km = max(K, 1)
    dev = lib().DeviceModel(shape, w, batch=B, capacity=64, max_block=Km, max_rows=max(B * (Km + 1), 64))
    rng = np.random.default_rng(V + 10 * B + K + int(10 * T))
    dl = rng.normal(0.0, 2.0, (B, K, V)).astype(np.float32)
    vl = rng.normal(0.0, 2.0, (B, K + 1, V)).astype(np.float32)
    for b in range(B):  # verify rows near the draft rows, by a different amount per sequence
        vl[b, :K] = dl[b] + rng.normal(0.0, [0.02, 0.2, 0.6, 2.0][b % 4], (K, V)).astype(np.float32)
    ud, ua, uf = (rng.random(s, dtype=np.float32) for s in ((B, K), (B, K), (B,)))
    dl_d, vl_d = torch.from_numpy(dl).cuda(), torch.from_numpy(vl).cuda()
    drafts = i32(B, K)
    pending, acc, com = i32(B), i32(B), i32(B, K + 1)
    dev.lens.copy_(torch.arange(10, 10 + B, dtype=torch.int32))
    if K:
        lib().sample_tokens(dl_d.view(B * K, V), T, torch.from_numpy(ud).cuda(), drafts.view(-1), dev.status)
    dev.accept_sample(pending, drafts if K else None, dl_d if K else None, vl_d, K, T,
                      torch.from_numpy(ua).cuda() if K else None, torch.from_numpy(uf).cuda(), acc, com)
    torch.cuda.synchronize()
    assert dev.read_status() == 0
    D, A, Cm = drafts.cpu().numpy(), acc.cpu().numpy(), com.cpu().numpy()
    near = 0
    for b in range(B):
        for i in range(K):  # the drafts: draws from q_i
            wq = tempered_weights(torch.from_numpy(dl[b, i]), T)
            ok, amb = cdf_band_ok(wq.numpy(), float(ud[b, i]), int(D[b, i]), inverse_cdf(wq, float(ud[b, i])),
                                  TOL_CDF)
            assert ok
            near += amb
        near += check_consensus([int(t) for t in D[b]], dl[b], vl[b], T, ua[b], uf[b], int(A[b]), Cm[b].tolist())
        assert int(dev.lens[b]) == 10 + b + int(A[b]) + 1
        assert int(pending[b]) == Cm[b, A[b]]
    assert near <= 1, near
    if K >= 8:  # the spread of agreement between the views gives a spread of accept lengths
        assert len(set(A.tolist())) > 1


def test_accept_sample_with_nan_logit_commits_nothing():
    shape = replace(synth.TINY, name="tiny_v1024", n_layers=1)
    w = synth.make_weights(shape, 73, 74)
    B, K, V = 2, 4, 1024
    dev = lib().DeviceModel(shape, w, batch=B, capacity=64, max_block=K, max_rows=64)
    dl = torch.zeros((B, K, V), device="cuda")
    vl = torch.zeros((B, K + 1, V), device="cuda")
    vl[1, 2, 5] = float("nan")
    pending, acc, com = i32(B), i32(B), i32(B, K + 1)
    dev.lens.fill_(7)
    dev.accept_sample(pending, i32(B, K), dl, vl, K, 1.0, torch.full((B, K), 0.5, device="cuda"),
                      torch.full((B,), 0.5, device="cuda"), acc, com)
    torch.cuda.synchronize()
    assert dev.read_status() == lib().ERR_NAN
    assert acc.cpu().tolist() == [-1, -1] and (com == -1).all()
    assert dev.lens.cpu().tolist() == [7, 7]


# ---- the whole sampled step on the tiny decoder ----------------------------------------------

@pytest.mark.parametrize("shape", [synth.TINY, synth.TINY_QK], ids=["tiny", "tiny_qk"])
def test_sampled_decode_matches_oracle(shape):
    """Several sampled steps through the pieces (draft view, draws, verify view, consensus):
    logits against the oracle's forwards, every decision against the oracle on the GPU's
    logits, the oracle's state advanced by the GPU's commits. Then the same steps through
    orthrus_decode_step_sampled from the same state: bit-identical."""
    K, P, B, T = 8, 40, 2, 1.0
    cap = P + 8 * (K + 1) + 4
    w = synth.make_weights(shape, 81, 82, gain_std=0.1 if shape.qk_norm else 0.0)
    dev = lib().DeviceModel(shape, w, batch=B, capacity=cap, max_block=K, max_rows=64)
    o = Oracle(shape, w, capacity=cap)
    V = shape.vocab
    toks = np.stack([synth.make_prompt(shape, P, 700 + b) for b in range(B)]).astype(np.int32)
    pending = i32(B)
    dev.prefill(torch.from_numpy(toks).cuda(), [P] * B, pending)
    torch.cuda.synchronize()
    lens0, pend0 = dev.lens.clone(), pending.clone()
    states = []
    for b in range(B):
        st = o.new_state()
        o.prefill(st, toks[b])
        st.y = int(pend0[b])
        states.append(st)
    rng = np.random.default_rng(99)
    steps = [tuple(torch.from_numpy(a).cuda() for a in (rng.random((B, K), dtype=np.float32),
                                                         rng.random((B, K), dtype=np.float32),
                                                         rng.random(B, dtype=np.float32))) for _ in range(4)]
    d, ar, acc, com = i32(B, K), i32(B, K + 1), i32(B), i32(B, K + 1)
    dl, vl = torch.zeros((B, K, V), device="cuda"), torch.zeros((B, K + 1, V), device="cuda")
    record = []
    near = 0
    for ud, ua, uf in steps:
        dev.draft_block(pending, K, d, dl)
        lib().sample_tokens(dl.view(B * K, V), T, ud, d.view(-1), dev.status)
        dev.verify_block(pending, d, K, ar, vl)
        dev.accept_sample(pending, d, dl, vl, K, T, ua, uf, acc, com)
        torch.cuda.synchronize()
        assert dev.read_status() == 0
        D, DL, VL = d.cpu().numpy(), dl.cpu().numpy(), vl.cpu().numpy()
        A, Cm = acc.cpu().numpy(), com.cpu().numpy()
        record.append((A.copy(), Cm.copy()))
        for b, st in enumerate(states):
            _, dl_ref = o.draft_block(st, K)
            check_logits(DL[b], dl_ref)
            for i in range(K):
                wq = tempered_weights(torch.from_numpy(DL[b, i]), T)
                ok, amb = cdf_band_ok(wq.numpy(), float(ud[b, i]), int(D[b, i]),
                                      inverse_cdf(wq, float(ud[b, i])), TOL_CDF)
                assert ok
                near += amb
            _, vl_ref = o.verify_block(st, D[b].tolist())
            check_logits(VL[b], vl_ref)
            near += check_consensus(D[b].tolist(), DL[b], VL[b], T, ua[b].cpu().numpy(), float(uf[b]), int(A[b]),
                                    Cm[b].tolist())
            a = int(A[b])
            st.n += a + 1
            st.y = int(Cm[b, a])
            assert int(dev.lens[b]) == st.n and int(pending[b]) == st.y
    assert near <= 2, near
    # the fused entry point from the same starting state, with the same uniforms
    dev.lens.copy_(lens0)
    pending.copy_(pend0)
    for (ud, ua, uf), (A, Cm) in zip(steps, record):
        dev.decode_step_sampled(pending, K, T, ud, ua, uf, dl, vl, acc, com)
        torch.cuda.synchronize()
        assert np.array_equal(acc.cpu().numpy(), A) and np.array_equal(com.cpu().numpy(), Cm)
    assert dev.read_status() == 0
    assert [int(x) for x in dev.lens] == [st.n for st in states]


# ---- edges of the inverse CDF and of the residual ------------------------------------------

V_BELOW_ONE = np.float32(1.0 - 2.0 ** -24)  # the largest fp32 uniform below 1


def test_sample_tokens_edges_of_the_cdf():
    # Rows whose draw is the same index in any precision, at the top end of [0, 1): v * Z lies
    # within 6e-8 of the total, where the kernel's fallbacks decide the token when its running
    # sums round past the target, or reach it only at zero-weight elements.
    V = 3149  # four CDF tiles, the last one ragged
    rng = np.random.default_rng(91)
    x = np.full((4, V), -np.inf, dtype=np.float32)
    x[0, :1500] = rng.normal(-30.0, 1.0, 1500)  # tiny weights before one dominant token,
    x[0, 1500] = 0.0                             # nothing after it
    x[1, 0] = 3.0                                # one token, the first
    x[2, :1000] = rng.normal(0.0, 1.0, 1000)     # the first tile only: the last positive index
    x[3, 2048:V] = rng.normal(0.0, 1.0, V - 2048)  # the last two tiles only, v = 0: the first of them
    u = np.array([V_BELOW_ONE, V_BELOW_ONE, V_BELOW_ONE, 0.0], dtype=np.float32)
    out, status = i32(4), i32(1)
    lib().sample_tokens(torch.from_numpy(x).cuda(), 1.0, torch.from_numpy(u).cuda(), out, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = [inverse_cdf(tempered_weights(torch.from_numpy(x[r]), 1.0), float(u[r])) for r in range(4)]
    assert ref == [1500, 0, 999, 2048]
    assert out.cpu().tolist() == ref


def test_accept_sample_edges_of_the_residual():
    # Three sequences, K = 2, uniforms at the top end of [0, 1):
    #  b = 0: verify row 0 equals draft row 0 except one raised logit j, so p_0 < q_0 everywhere
    #         but at j: d_1 is rejected (p/q = Z_d / Z_v well below u) and the residual is
    #         positive only at j, the last token for any v;
    #  b = 1: p_0 == q_0 exactly and d_1 outside their support: rejected, the residual is zero
    #         everywhere, and the last token is drawn from p_0 (one-hot: its token);
    #  b = 2: p == q exactly on rows 0 and 1 with each draft the row's top token (q = 1 after the
    #         max shift): both accepted for u just below 1, and the bonus token drawn from p_2
    #         with v just below 1 is its dominant token (nothing after it has weight).
    shape = replace(synth.TINY, name="tiny_v1024", n_layers=1)
    w = synth.make_weights(shape, 75, 76)
    B, K, V = 3, 2, 1024
    dev = lib().DeviceModel(shape, w, batch=B, capacity=64, max_block=K, max_rows=64)
    rng = np.random.default_rng(92)
    dl = rng.normal(0.0, 1.0, (B, K, V)).astype(np.float32)
    vl = dl.copy()
    vl = np.concatenate([vl, rng.normal(0.0, 1.0, (B, 1, V)).astype(np.float32)], axis=1)
    drafts = np.zeros((B, K), dtype=np.int32)
    # b = 0
    top = int(np.argmax(dl[0, 0]))
    j = int(np.argsort(dl[0, 0])[-3])            # third largest: stays below the max once raised
    vl[0, 0, j] = dl[0, 0, j] + np.float32(0.9 * (dl[0, 0, top] - dl[0, 0, j]))
    drafts[0] = [(j + 1) % V if (j + 1) % V != top else (j + 2) % V, 5]
    # b = 1
    dl[1, 0] = -np.inf
    dl[1, 0, 321] = 0.5
    vl[1, 0] = dl[1, 0]
    drafts[1] = [100, 7]
    # b = 2
    for i in range(K):
        vl[2, i] = dl[2, i]
        drafts[2, i] = int(np.argmax(dl[2, i]))
    vl[2, K, :] = -np.inf
    vl[2, K, :600] = rng.normal(-30.0, 1.0, 600)
    vl[2, K, 600] = 1.0
    ua = np.full((B, K), V_BELOW_ONE, dtype=np.float32)
    uf = np.full((B,), V_BELOW_ONE, dtype=np.float32)
    pending, acc, com = i32(B), i32(B), i32(B, K + 1)
    dev.lens.fill_(10)
    dev.accept_sample(pending, torch.from_numpy(drafts).cuda(), torch.from_numpy(dl).cuda(),
                      torch.from_numpy(vl).cuda(), K, 1.0, torch.from_numpy(ua).cuda(), torch.from_numpy(uf).cuda(),
                      acc, com)
    torch.cuda.synchronize()
    assert dev.read_status() == 0
    expect = [(0, [j]), (0, [321]), (2, [int(drafts[2, 0]), int(drafts[2, 1]), 600])]
    for b in range(B):
        a_ref, toks = accept_sample_logits([int(t) for t in drafts[b]], torch.from_numpy(dl[b]),
                                           torch.from_numpy(vl[b]), 1.0, ua[b], uf[b])
        assert (a_ref, toks) == expect[b], b
        assert int(acc[b]) == a_ref
        assert com[b].cpu().tolist() == toks + [-1] * (K + 1 - len(toks))
        assert int(pending[b]) == toks[-1] and int(dev.lens[b]) == 10 + a_ref + 1


def test_accept_sample_with_a_row_of_no_finite_logit_commits_nothing():
    # A verify row whose logits are all -inf has no distribution: the status word takes
    # ORTHRUS_ERR_NAN and no sequence commits anything.
    shape = replace(synth.TINY, name="tiny_v1024", n_layers=1)
    w = synth.make_weights(shape, 77, 78)
    B, K, V = 2, 3, 1024
    dev = lib().DeviceModel(shape, w, batch=B, capacity=64, max_block=K, max_rows=64)
    dl = torch.zeros((B, K, V), device="cuda")
    vl = torch.zeros((B, K + 1, V), device="cuda")
    vl[0, K] = float("-inf")
    pending, acc, com = i32(B), i32(B), i32(B, K + 1)
    dev.lens.fill_(9)
    dev.accept_sample(pending, i32(B, K), dl, vl, K, 1.0, torch.full((B, K), 0.5, device="cuda"),
                      torch.full((B,), 0.5, device="cuda"), acc, com)
    torch.cuda.synchronize()
    assert dev.read_status() == lib().ERR_NAN
    assert acc.cpu().tolist() == [-1, -1] and (com == -1).all()
    assert dev.lens.cpu().tolist() == [9, 9]

"""Host logic of the bench's planted-draft rehearsal (bench.greedy_streams, bench.planted_step),
on the CPU with a stand-in decoder.

The stand-in keeps a token cache and a pending token per sequence like the library does, and
takes its next-token function from the context. Its verify view agrees with its K = 0 view
everywhere but at one position of sequence 0, where it picks another token: the situation of
a near tie that per-op kernels and the persistent kernel round differently. The rehearsal must
detect that step, adopt the verify view's tokens, rebuild the greedy streams from the new
state, and every later step must then commit exactly its planted accept length; the committed
stream must equal the (rebuilt) greedy stream, as the bench checks after timing.
"""
import numpy as np
import torch

import bench
import synth

V, B, K = 97, 2, 6
SPECIAL = (0, 23)  # (sequence, context length) where the verify view leaves the K = 0 view


def next_token(ctx):
    h = 0
    for t in ctx[-4:]:
        h = (h * 1000003 + int(t) * 7919 + 17) % 2147483647
    return (h + 31 * len(ctx)) % V


class StandIn:
    def __init__(self, prompts, capacity):
        self.capacity = capacity
        self.cache = [list(p[:-1]) + [0] * (capacity - len(p) + 1) for p in prompts]
        self.lens = torch.tensor([len(p) - 1 for p in prompts], dtype=torch.int32)
        self.first = [int(p[-1]) for p in prompts]

    def ctx(self, b, pending, extra=()):
        return self.cache[b][:int(self.lens[b])] + [pending] + list(extra)

    def _commit(self, b, toks):
        n = int(self.lens[b])
        for i, t in enumerate(toks):
            self.cache[b][n + i] = int(t)
        self.lens[b] = n + len(toks)

    def verify_next(self, b, ctx):
        t = next_token(ctx)
        return (t + 1) % V if (b, len(ctx)) == SPECIAL else t

    # K = 0 path: the view the greedy streams come from
    def verify_block(self, pending, drafts, k, ar):
        assert k == 0 and drafts is None
        for b in range(B):
            ar[b, 0] = next_token(self.ctx(b, int(pending[b])))

    def accept_commit(self, pending, drafts, ar, k, acc, out):
        for b in range(B):
            self._commit(b, [int(pending[b])])
            pending[b] = int(ar[b, 0])
            out[b] = int(ar[b, 0])
            acc[b] = 0

    def decode_step(self, pending, k, drafts, acc, com):
        for b in range(B):
            d = [int(x) for x in drafts[b]]
            p = int(pending[b])
            a = 0
            while a < k and d[a] == self.verify_next(b, self.ctx(b, p, d[:a])):
                a += 1
            last = self.verify_next(b, self.ctx(b, p, d[:a]))
            self._commit(b, [p] + d[:a])
            pending[b] = last
            acc[b] = a
            com[b, :] = -1
            com[b, :a] = torch.tensor(d[:a], dtype=torch.int32)
            com[b, a] = last

    def read_status(self):
        return 0


def test_rehearsal_rebuilds_the_stream_where_the_verify_view_leaves_it():
    rng = np.random.default_rng(5)
    prompts = [list(rng.integers(0, V, 9)), list(rng.integers(0, V, 12))]
    steps = 12
    accepts = np.stack([synth.planted_accepts_stratified(steps, 3.0, K, seed=40 + b) for b in range(B)], axis=1)
    need = 1 + int(np.max(np.sum(accepts + 1, axis=0))) + K + 2 + 4 * (K + 1)
    m = StandIn(prompts, capacity=max(len(p) for p in prompts) + 3 * need)
    pending = torch.tensor([m.first[0], m.first[1]], dtype=torch.int32)
    lens0, pend0 = m.lens.clone(), pending.clone()
    stream = bench.greedy_streams(m, pending, need, "cpu")
    assert stream.shape == (B, need)
    m.lens.copy_(lens0)
    pending.copy_(pend0)
    stream0 = stream[:, 0].copy()

    acc = torch.zeros(B, dtype=torch.int32)
    com = torch.zeros((B, K + 1), dtype=torch.int32)
    jpos, left_at, got = [0] * B, [], []
    drng = np.random.default_rng(6)
    for t in range(steps):
        _, a, c, left = bench.planted_step(m, pending, "cpu", stream, jpos, accepts[t], K, V, drng, acc, com)
        got.append((a.copy(), c.copy()))
        if left:
            left_at.append(t)
        else:
            assert np.array_equal(a, accepts[t])  # every step away from the tie commits its plan
    assert len(left_at) == 1  # the tie is met once, then the rebuilt stream holds
    for b in range(B):  # the committed stream is the (rebuilt) greedy stream
        out = [int(stream0[b])]
        for a, c in got:
            out.extend(int(x) for x in c[b, :a[b] + 1])
        assert out == [int(x) for x in stream[b, :len(out)]]

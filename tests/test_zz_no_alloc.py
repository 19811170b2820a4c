"""GPU test of orthrus_linear_noalloc, the GEMM entry point for callers that
cannot allocate device memory (for example a plugin interface that receives
only its input and output buffers): its scratch is a static device array inside
the library.

Calls in a row, each checked against orthrus_linear (the workspace-taking entry
point) and against the oracle's linear layer on the same inputs, within the GEMM
tolerance of the other kernel tests. The shapes are chosen so that the stream-K
split of the 32-CTA grid cuts weight tiles between CTAs: (33, 1152, 4096) gives
each CTA 18 of a tile's 64 k-chunks, so CTA ranges straddle tiles and both of a
CTA's partial slots are used; (17, 256, 4096) gives each tile 16 contributors.
Each later call has a different shape, so it would see any arrival counter an
earlier call left behind in the shared array. The file is named to be collected
last; it passes alone in a fresh process and after the other tests.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import linear as oracle_linear

pytestmark = pytest.mark.gpu


def bf16_tensor(shape, seed, std=1.0):
    bits = synth.normal_bf16(shape, seed, std)
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def with_workspace(o, X, W):
    M, Kd = X.shape
    N = W.shape[0]
    Y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(o.linear_workspace_bytes(M, N, Kd), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o.linear(X, W, Y, ws, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return Y.cpu().numpy().astype(np.float64)


def test_noalloc_linear_matches_workspace_linear_and_oracle():
    from shared_kv_draft_b200 import orthrus as o
    for M, N, Kd in [(33, 1152, 4096), (17, 256, 4096), (33, 4096, 4096), (130, 1024, 768), (33, 1152, 4096)]:
        X = bf16_tensor((M, Kd), M * 5 + Kd)
        W = bf16_tensor((N, Kd), N * 3 + Kd, std=0.05)
        ref = with_workspace(o, X, W)
        exact = oracle_linear(X.cpu().to(torch.float64), W.cpu(), rowwise=False).numpy()
        tol = 1e-5 * np.sqrt(Kd) * max(1.0, np.abs(exact).max())
        assert np.abs(ref - exact).max() <= tol
        Y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        o.linear_noalloc(X, W, Y, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        got = Y.cpu().numpy().astype(np.float64)
        assert np.isfinite(got).all()
        assert np.abs(got - ref).max() <= tol, (M, N, Kd)
        assert np.abs(got - exact).max() <= tol, (M, N, Kd)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from shared_kv_draft_b200 import orthrus as o
    X = torch.zeros((129, 64), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((128 * 8193, 64), dtype=torch.bfloat16, device="cuda")
    Y = torch.zeros((1, 1), dtype=torch.float32, device="cuda")
    with pytest.raises(o.OrthrusError) as e:
        o.linear_noalloc(X, W, Y)
    assert e.value.code == o.ERR_WORKSPACE

"""Routing (k-means) attention with quota execution on the GPU against the oracle
(PaperTrace 2.1.1 §3.1).  The quotas are integer decisions taken in fp32 in the same
order on both sides: JQ, JK and the per-query key counts are compared exactly; outputs
and lse within the bf16-input tolerance 2e-3 max(1, |oracle|)."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu
TOL = 2e-3


def _case(B, H, n, C, seed, dev, d=64):
    g = torch.Generator(device="cpu").manual_seed(seed)
    Q = torch.randn(B, H, n, d, generator=g).to(torch.bfloat16)
    K = torch.randn(B, H, n, d, generator=g).to(torch.bfloat16)
    V = torch.randn(B, H, n, d, generator=g).to(torch.bfloat16)
    M = torch.randn(H, C, d, generator=g)
    M = M / M.norm(dim=-1, keepdim=True)                   # equal-norm centres
    return Q.to(dev), K.to(dev), V.to(dev), M.to(dev)


@pytest.mark.parametrize("B,H,n,C,m,causal,no_self", [
    (1, 2, 300, 8, 48, True, False),
    (2, 2, 1000, 16, 100, True, True),
    (1, 1, 777, 12, 256, False, False),        # quota larger than n / C: heavy overlap
    (1, 2, 4096, 64, 64, True, False),
])
def test_route_matches_oracle(crs, cuda_dev, B, H, n, C, m, causal, no_self):
    Q, K, V, M = _case(B, H, n, C, seed=n + C, dev=cuda_dev)
    JQ, JK, O, lse, cnt = crs.route_attn(Q, K, V, M, m, causal=causal, no_self=no_self)
    torch.cuda.synchronize()
    assert crs.get_device_error() == 0
    oJQ, oJK, oO, olse, ocnt = oracle.kmeans_route(Q.float().cpu().numpy(), K.float().cpu().numpy(),
                                                   V.float().cpu().numpy(), M.cpu().numpy(), m,
                                                   causal=causal, no_self=no_self)
    assert np.array_equal(JQ.cpu().numpy(), oJQ)
    assert np.array_equal(JK.cpu().numpy(), oJK)
    assert np.array_equal(cnt.cpu().numpy(), ocnt)
    err = np.abs(O.cpu().numpy() - oO) / np.maximum(1.0, np.abs(oO))
    assert err.max() <= TOL, f"max rel err {err.max():.3e}"
    gl, fin = lse.cpu().numpy(), np.isfinite(olse)
    assert np.array_equal(np.isfinite(gl), fin)
    assert np.abs(gl[fin] - olse[fin]).max() <= TOL * max(1.0, np.abs(olse[fin]).max())

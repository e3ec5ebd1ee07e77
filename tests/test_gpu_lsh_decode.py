"""LSH attention in decode on the GPU (paged K/V behind a shuffled block table, bucket
lists appended per token) against the oracle's decode step (PaperTrace 2.1.1 §5.2).
Bucket ids are bit-exact, so the candidate counts are compared exactly; outputs and lse
within the bf16-input tolerance |gpu - oracle| <= 2e-3 max(1, |oracle|)."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu
TOL = 2e-3


def _inputs(S, n, H, d, b, R, seed, dev):
    g = torch.Generator(device="cpu").manual_seed(seed)
    x = torch.randn(S, n, H, d, generator=g).to(torch.bfloat16)
    v = torch.randn(S, n, H, d, generator=g).to(torch.bfloat16)
    rot = torch.randn(H, R, d, b // 2, generator=g)
    return x.to(dev), v.to(dev), rot.to(dev)


def _oracle(x, v, rot, b, lengths, no_self):
    X = x.float().cpu().numpy().transpose(0, 2, 1, 3)       # [S, H, n, d]
    V = v.float().cpu().numpy().transpose(0, 2, 1, 3)
    return oracle.lsh_decode(X, V, rot.cpu().numpy(), b, lengths, no_self=no_self)


def _compare(O, lse, cnt, o_O, o_lse, o_cnt):
    assert np.array_equal(cnt.cpu().numpy(), o_cnt)
    g = O.cpu().numpy()
    err = np.abs(g - o_O) / np.maximum(1.0, np.abs(o_O))
    assert err.max() <= TOL, f"max rel err {err.max():.3e}"
    gl, fin = lse.cpu().numpy(), np.isfinite(o_lse)
    assert np.array_equal(np.isfinite(gl), fin)
    assert np.abs(gl[fin] - o_lse[fin]).max() <= TOL * max(1.0, np.abs(o_lse[fin]).max())


@pytest.mark.parametrize("no_self", [True, False])
def test_prefill_then_two_steps(crs, cuda_dev, no_self):
    S, n, H, d, b, R = 3, 301, 2, 64, 16, 3
    x, v, rot = _inputs(S, n + 2, H, d, b, R, seed=51, dev=cuda_dev)
    cache = crs.LshDecodeCache(S, H, b, R, max_len=400, page_size=16, list_page=8, list_cap=400,
                               no_self=no_self, device=cuda_dev)
    cache.prefill(x[:, :n].contiguous(), v[:, :n].contiguous(), rot)
    for step in range(2):
        t = n + step
        O, lse, cnt = cache.step(x[:, t: t + 1].contiguous(), v[:, t: t + 1].contiguous(), rot)
        torch.cuda.synchronize()
        assert crs.get_device_error() == 0
        o_O, o_lse, o_cnt = _oracle(x[:, : t + 1], v[:, : t + 1], rot, b, np.full(S, t + 1), no_self)
        _compare(O, lse, cnt, o_O, o_lse, o_cnt)
    assert (cache.seq_len.cpu().numpy() == n + 2).all()


def test_long_rows_64_buckets_4_rounds(crs, cuda_dev):
    """Rows of 4096 tokens, 64 buckets, 4 rounds, 64-token KV pages, 64-entry list pages."""
    S, n, H, d, b, R = 2, 4096, 4, 64, 64, 4
    x, v, rot = _inputs(S, n + 1, H, d, b, R, seed=52, dev=cuda_dev)
    cache = crs.LshDecodeCache(S, H, b, R, max_len=n + 64, device=cuda_dev)
    cache.prefill(x[:, :n].contiguous(), v[:, :n].contiguous(), rot)
    O, lse, cnt = cache.step(x[:, n:].contiguous(), v[:, n:].contiguous(), rot)
    torch.cuda.synchronize()
    assert crs.get_device_error() == 0
    o_O, o_lse, o_cnt = _oracle(x, v, rot, b, np.full(S, n + 1), True)
    _compare(O, lse, cnt, o_O, o_lse, o_cnt)


def test_full_list_flags_capacity_and_keeps_running(crs, cuda_dev):
    """Two buckets and an 8-entry list: the lists overflow; the overflow is flagged, the
    step still returns finite outputs over the entries that fit."""
    S, n, H, d, b, R = 1, 100, 1, 64, 2, 1
    x, v, rot = _inputs(S, n + 1, H, d, b, R, seed=53, dev=cuda_dev)
    cache = crs.LshDecodeCache(S, H, b, R, max_len=128, page_size=16, list_page=8, list_cap=8, device=cuda_dev)
    crs.get_device_error()
    cache.prefill(x[:, :n].contiguous(), v[:, :n].contiguous(), rot)
    O, lse, cnt = cache.step(x[:, n:].contiguous(), v[:, n:].contiguous(), rot)
    torch.cuda.synchronize()
    assert crs.get_device_error() & 0x8
    assert torch.isfinite(O).all() and (cnt.cpu().numpy() <= 8).all()


def test_many_candidates_per_row(crs, cuda_dev):
    """Two buckets, two rounds, 3000-token rows: about 2250 candidates per (row, head),
    more than the attend kernel buffers at once, so it scores them in several batches."""
    S, n, H, d, b, R = 2, 3000, 2, 64, 2, 2
    x, v, rot = _inputs(S, n + 1, H, d, b, R, seed=54, dev=cuda_dev)
    cache = crs.LshDecodeCache(S, H, b, R, max_len=n + 64, device=cuda_dev)
    cache.prefill(x[:, :n].contiguous(), v[:, :n].contiguous(), rot)
    O, lse, cnt = cache.step(x[:, n:].contiguous(), v[:, n:].contiguous(), rot)
    torch.cuda.synchronize()
    assert crs.get_device_error() == 0
    o_O, o_lse, o_cnt = _oracle(x, v, rot, b, np.full(S, n + 1), True)
    assert o_cnt.min() > 2048
    _compare(O, lse, cnt, o_O, o_lse, o_cnt)

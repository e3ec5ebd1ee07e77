"""The allocation-free block selection (crs_block_select_noalloc).

Some callers cannot allocate device memory when they call the library (an
engine whose memory pool owns the device, a plugin host that passes only
input and output buffers, a loop that must not pay for cudaMalloc).  For them
crs_block_select_noalloc keeps its scratch in a static device array inside
libcrs.  This file runs last so that a failure here leaves every other test
already run; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


def _case(crs, dev, n_seq, T, top, win, seed):
    c = workloads.block_decode_case(n_seq=n_seq, T=T, seed=seed, device=dev)
    p = c["params"]
    mu, xi = crs.block_describe(c["K"], p["L"], p["rank"])
    return c, p, mu, xi, top, win


def test_noalloc_matches_block_select_twice(crs, cuda_dev):
    """Two calls in a row, different problems: each equals crs_block_select's
    result exactly (same kernels; the token lists are integers)."""
    for n_seq, T, top, win, seed in ((2, 4096, 16, 256, 11), (3, 2048, 8, 128, 12)):
        c, p, mu, xi, top, win = _case(crs, cuda_dev, n_seq, T, top, win, seed)
        ref_tok, ref_cnt = crs.block_select(c["Q"], mu, xi, p["T"], p["L"], top, win)
        cap = top * p["L"] + win
        tok = torch.full((n_seq, p["n_kv_heads"], cap), -7, dtype=torch.int32, device=cuda_dev)
        cnt = torch.full((n_seq, p["n_kv_heads"]), -7, dtype=torch.int32, device=cuda_dev)
        crs.block_select_noalloc(c["Q"], mu, xi, p["T"], p["L"], top, win, tok=tok, count=cnt)
        torch.cuda.synchronize()
        assert torch.equal(cnt, ref_cnt)
        assert torch.equal(tok, ref_tok)
    assert crs.get_device_error() == 0


def test_noalloc_rejects_problems_beyond_the_scratch(crs, cuda_dev):
    """n_seq * n_q * (T/L) scores must fit the 16 MiB array: 17 * 32 * 8192 > 4,194,304.
    The call is refused on the host, before any launch."""
    n_seq, T = 17, 32 * 8192
    Q = torch.zeros(n_seq, 32, 128, dtype=torch.bfloat16, device=cuda_dev)
    mu = torch.zeros(n_seq, 4, T // 32, 128, dtype=torch.float32, device=cuda_dev)
    xi = torch.zeros(n_seq, 4, T // 32, 1, 128, dtype=torch.float32, device=cuda_dev)
    with pytest.raises(crs.CrsError) as e:
        crs.block_select_noalloc(Q, mu, xi, T, 32, 4, 0)
    assert e.value.status == 6   # CRS_ERR_WORKSPACE

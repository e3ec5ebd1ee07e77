"""GPU parity: lightning-indexer token top-k (prefill and decode) vs the oracle."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import check_topk_row, indexer_abs_bound

pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().cpu().float().numpy().astype(np.float64)


def _check_rows(g_idx, g_cnt, qd, wd, Kd, key_base, n_vis, rows, topk, what):
    o_idx, o_cnt, o_cut, _ = oracle.indexer_topk(qd[rows], wd[rows], Kd, key_base[rows],
                                                 n_vis[rows], topk)
    ndiff, worst = 0, 0.0
    for j, r in enumerate(rows):
        kb, nv = int(key_base[r]), int(n_vis[r])
        Kr = Kd[kb:kb + nv]
        sc = lambda pos: oracle.indexer_score(qd[r], wd[r], Kr[pos])
        bd = lambda pos: indexer_abs_bound(qd[r], wd[r], Kr[pos])
        nd, wg = check_topk_row(g_idx[r], g_cnt[r], o_idx[j], o_cnt[j], o_cut[j], sc, bd,
                                what=f"{what} row {r}")
        ndiff += nd
        worst = max(worst, wg)
    print(f"{what}: {len(rows)} rows, {ndiff} differing positions, largest relative gap to the "
          f"cutoff {worst:.3e}")
    return ndiff


@pytest.mark.parametrize("n,topk", [(700, 64), (3000, 256), (17000, 2048)])
def test_prefill_small(crs, cuda_dev, n, topk):
    case = workloads.indexer_prefill_case(n=n, topk=topk, seed=n, device=cuda_dev)
    idx, cnt = crs.indexer_topk(case["q_idx"], case["w"], case["k_idx"], topk,
                                crs.CRS_IDX_PREFILL)
    torch.cuda.synchronize()
    assert crs.get_device_error() == 0
    g_idx, g_cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    assert (g_cnt == np.minimum(topk, np.arange(n) + 1)).all()
    qd, wd, Kd = _np(case["q_idx"]), _np(case["w"]), _np(case["k_idx"])
    rng = np.random.default_rng(n)
    rows = np.unique(np.concatenate([[0, 1, topk - 1, topk, topk + 1, n - 1],
                                     [min(n - 1, 16383), min(n - 1, 16384)],
                                     rng.choice(n, min(n, 120), replace=False)]))
    _check_rows(g_idx, g_cnt, qd, wd, Kd, np.zeros(n, np.int64), np.arange(1, n + 1, dtype=np.int32),
                rows, topk, "prefill")


def test_prefill_tensor_core_path_traced(crs, cuda_dev):
    """4 index heads of dim 64 run on the tcgen05 kernel (sample, threshold, filter, select)."""
    n, topk = 5000, 512
    case = workloads.indexer_prefill_case(n=n, topk=topk, seed=11, device=cuda_dev)
    crs.profile_collect()
    idx, cnt = crs.indexer_topk(case["q_idx"], case["w"], case["k_idx"], topk,
                                crs.CRS_IDX_PREFILL)
    torch.cuda.synchronize()
    names = crs.profile_collect()
    assert "idx_prefill_tc" in names
    assert crs.get_device_error() == 0
    g_idx, g_cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    assert (g_cnt == np.minimum(topk, np.arange(n) + 1)).all()
    rows = np.unique(np.concatenate([np.arange(0, n, 37), [topk - 1, topk, 1279, 1280, n - 1]]))
    _check_rows(g_idx, g_cnt, _np(case["q_idx"]), _np(case["w"]), _np(case["k_idx"]),
                np.zeros(n, np.int64), np.arange(1, n + 1, dtype=np.int32), rows, topk,
                "prefill-tc")


@pytest.mark.parametrize("n_idx_heads", [2, 8])
def test_prefill_cuda_core_path(crs, cuda_dev, n_idx_heads):
    """Index-head counts other than 4 take the CUDA-core slice path."""
    n, topk = 2500, 256
    case = workloads.indexer_prefill_case(n=n, topk=topk, n_idx_heads=n_idx_heads, seed=5,
                                          device=cuda_dev)
    crs.profile_collect()
    idx, cnt = crs.indexer_topk(case["q_idx"], case["w"], case["k_idx"], topk,
                                crs.CRS_IDX_PREFILL)
    torch.cuda.synchronize()
    assert "idx_prefill_tc" not in crs.profile_collect()
    assert crs.get_device_error() == 0
    g_idx, g_cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    rows = np.unique(np.concatenate([np.arange(0, n, 41), [topk - 1, topk, n - 1]]))
    _check_rows(g_idx, g_cnt, _np(case["q_idx"]), _np(case["w"]), _np(case["k_idx"]),
                np.zeros(n, np.int64), np.arange(1, n + 1, dtype=np.int32), rows, topk,
                "prefill-cc")


def test_prefill_all_tied_rows_take_exact_fallback(crs, cuda_dev):
    """Every key identical: each row's scores tie and the sampled threshold lets all
    keys through.  Rows up to ~8k keys select among the ties (smallest positions
    first); longer rows overflow their candidate lists and are recomputed by the
    exact slice path."""
    n, topk = 10000, 1024
    g = torch.Generator(device=cuda_dev).manual_seed(3)
    q = torch.randn(n, 4, 64, generator=g, device=cuda_dev).to(torch.bfloat16)
    w = torch.randn(n, 4, generator=g, device=cuda_dev)
    k = torch.randn(1, 64, generator=g, device=cuda_dev).to(torch.bfloat16).expand(n, 64).contiguous()
    crs.profile_collect()
    idx, cnt = crs.indexer_topk(q, w, k, topk, crs.CRS_IDX_PREFILL)
    torch.cuda.synchronize()
    names = crs.profile_collect()
    assert "idx_prefill_tc" in names and "idx_slice_topk" in names
    assert crs.get_device_error() == 0
    g_idx, g_cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    assert (g_cnt == np.minimum(topk, np.arange(n) + 1)).all()
    for r in (0, 100, topk, 4095, 4096, 4097, 8191, 8192, 8193, 9000, n - 1):
        m = min(topk, r + 1)
        assert (g_idx[r, :m] == np.arange(m)).all(), f"row {r}"
        assert (g_idx[r, m:] == -1).all()


def test_prefill_nan_score_flags_device_error(crs, cuda_dev):
    g = torch.Generator(device=cuda_dev).manual_seed(4)
    q = torch.randn(600, 4, 64, generator=g, device=cuda_dev).to(torch.bfloat16)
    w = torch.randn(600, 4, generator=g, device=cuda_dev)
    k = torch.randn(600, 64, generator=g, device=cuda_dev).to(torch.bfloat16)
    k[300, 5] = float("nan")
    crs.get_device_error()
    crs.indexer_topk(q, w, k, 64, crs.CRS_IDX_PREFILL)
    torch.cuda.synchronize()
    assert crs.get_device_error() & crs.DEVERR_NONFINITE


@pytest.mark.parametrize("lens,topk", [([100, 2048, 2049, 5000], 2048), ([40000, 17, 16384, 16385, 33000], 512)])
def test_decode_small(crs, cuda_dev, lens, topk):
    g = torch.Generator(device=cuda_dev).manual_seed(len(lens))
    n_seq = len(lens)
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    k_idx = torch.randn(int(off[-1]), 64, generator=g, device=cuda_dev).to(torch.bfloat16)
    q_idx = torch.randn(n_seq, 4, 64, generator=g, device=cuda_dev).to(torch.bfloat16)
    w = torch.randn(n_seq, 4, generator=g, device=cuda_dev)
    # exact ties: duplicate some keys
    k_idx[5:9] = k_idx[1]
    offs = torch.from_numpy(off).to(cuda_dev)
    idx, cnt = crs.indexer_topk(q_idx, w, k_idx, topk, crs.CRS_IDX_DECODE, k_offsets=offs,
                                max_keys=max(lens))
    torch.cuda.synchronize()
    assert crs.get_device_error() == 0
    _check_rows(idx.cpu().numpy(), cnt.cpu().numpy(), _np(q_idx), _np(w), _np(k_idx), off[:-1],
                np.array(lens, np.int32), np.arange(n_seq), topk, "decode")


def test_decode_full_config(crs, cuda_dev):
    """64 sequences, ctx ~ U{8192..131072}, top-2048: every row compared."""
    case = workloads.indexer_decode_case(device=cuda_dev)
    p = case["params"]
    idx, cnt = crs.indexer_topk(case["q_idx"], case["w"], case["k_idx"], p["topk"],
                                crs.CRS_IDX_DECODE, k_offsets=case["offsets"], max_keys=131072)
    torch.cuda.synchronize()
    assert crs.get_device_error() == 0
    off = case["offsets"].cpu().numpy()
    _check_rows(idx.cpu().numpy(), cnt.cpu().numpy(), _np(case["q_idx"]), _np(case["w"]),
                _np(case["k_idx"]), off[:-1], np.diff(off).astype(np.int32),
                np.arange(p["n_seq"]), p["topk"], "decode-full")


def test_prefill_full_config_sampled(crs, cuda_dev):
    """n = 32768 causal, top-2048: all rows on the GPU, 64 sampled rows vs the oracle."""
    case = workloads.indexer_prefill_case(device=cuda_dev)
    n, topk = case["params"]["n"], case["params"]["topk"]
    idx, cnt = crs.indexer_topk(case["q_idx"], case["w"], case["k_idx"], topk,
                                crs.CRS_IDX_PREFILL)
    torch.cuda.synchronize()
    assert crs.get_device_error() == 0
    g_cnt = cnt.cpu().numpy()
    assert (g_cnt == np.minimum(topk, np.arange(n) + 1)).all()
    rng = np.random.default_rng(1)
    rows = np.unique(np.concatenate([[0, 2046, 2047, 2048, 16383, 16384, n - 1],
                                     rng.choice(n, 57, replace=False)]))
    _check_rows(idx.cpu().numpy(), g_cnt, _np(case["q_idx"]), _np(case["w"]), _np(case["k_idx"]),
                np.zeros(n, np.int64), np.arange(1, n + 1, dtype=np.int32), rows, topk,
                "prefill-full")


def test_decode_all_tied_row_selects_whole_row(crs, cuda_dev):
    """Every cached index key equal: one histogram bucket holds the whole row (more than the
    bucket list holds), so the select runs over the whole row; ties go to the smallest
    positions.  A second, ordinary row shares the launch."""
    g = torch.Generator(device=cuda_dev).manual_seed(21)
    lens = [40000, 9000]
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    k_idx = torch.randn(int(off[-1]), 64, generator=g, device=cuda_dev).to(torch.bfloat16)
    k_idx[:lens[0]] = k_idx[0]
    q_idx = torch.randn(2, 4, 64, generator=g, device=cuda_dev).to(torch.bfloat16)
    w = torch.randn(2, 4, generator=g, device=cuda_dev)
    topk = 1024
    idx, cnt = crs.indexer_topk(q_idx, w, k_idx, topk, crs.CRS_IDX_DECODE,
                                k_offsets=torch.from_numpy(off).to(cuda_dev), max_keys=max(lens))
    torch.cuda.synchronize()
    assert crs.get_device_error() == 0
    g_idx, g_cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    assert g_cnt[0] == topk and (g_idx[0] == np.arange(topk)).all()
    _check_rows(g_idx, g_cnt, _np(q_idx), _np(w), _np(k_idx), off[:-1], np.array(lens, np.int32),
                np.array([1]), topk, "decode-tied")


def test_nan_score_flags_device_error(crs, cuda_dev):
    q = torch.randn(1, 4, 64, device=cuda_dev).to(torch.bfloat16)
    w = torch.randn(1, 4, device=cuda_dev)
    k = torch.randn(300, 64, device=cuda_dev).to(torch.bfloat16)
    k[7, 3] = float("nan")
    offs = torch.tensor([0, 300], dtype=torch.int64, device=cuda_dev)
    crs.get_device_error()
    crs.indexer_topk(q, w, k, 16, crs.CRS_IDX_DECODE, k_offsets=offs, max_keys=300)
    assert crs.get_device_error() & crs.DEVERR_NONFINITE

"""HISA (hierarchical indexer) on the GPU against the oracle ("细粒度索引" page, HISA and
§2.2 Eq.(7)).  The coarse level is checked on the kept block set (a difference must
sit at the coarse cutoff), the fine level against the oracle's fine stage run on the
GPU's own kept blocks (a difference must sit at the fine cutoff)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import cutoff_gaps, indexer_abs_bound

pytestmark = pytest.mark.gpu


def _cutoff_ok(scores, chosen_gpu, chosen_ref, k, what, floor_of=None):
    """Differences between the two chosen sets sit within 1e-5 relative of the cutoff
    (within the fp32 bound floor_of(d) only at an exact-0 cutoff)."""
    d = np.setxor1d(chosen_gpu, chosen_ref)
    if d.size == 0:
        return 0.0
    order = np.sort(scores)[::-1]
    cut = float(order[min(k, len(order)) - 1])
    return cutoff_gaps(scores[d], cut, None if (floor_of is None or cut != 0.0) else floor_of(d),
                       what=what)


def _run(crs, cuda_dev, case, blk, top_blocks, topk, max_keys):
    ko = case["offsets"].to(cuda_dev)
    rep, bo = crs.hisa_describe(case["k_idx"].to(cuda_dev), ko, blk, max_keys)
    blocks, idx, cnt = crs.hisa_topk(case["q_idx"].to(cuda_dev), case["w"].to(cuda_dev),
                                     case["k_idx"].to(cuda_dev), ko, rep, bo, topk, blk, top_blocks, max_keys)
    torch.cuda.synchronize()
    assert crs.get_device_error() == 0
    return rep, bo, blocks.cpu().numpy(), idx.cpu().numpy(), cnt.cpu().numpy()


def _check(case, rep, bo, blocks, idx, cnt, blk, top_blocks, topk, rows=None):
    K = case["k_idx"].float().cpu().numpy()
    q = case["q_idx"].float().cpu().numpy()
    w = case["w"].cpu().numpy()
    ko = case["offsets"].cpu().numpy()
    bo_np = bo.cpu().numpy()
    rep_np = rep.double().cpu().numpy()
    rows = range(len(ko) - 1) if rows is None else rows
    for t in rows:
        qk = q[t: t + 1]
        wk = w[t: t + 1]
        ko_t = np.array([ko[t], ko[t + 1]])
        bo_t = np.array([0, bo_np[t + 1] - bo_np[t]])
        rep_t = rep_np[bo_np[t]: bo_np[t + 1]]
        o_blocks, _, _, coarse = oracle.hisa_topk(qk, wk, K, ko_t, rep_t, bo_t, topk, blk, top_blocks)
        gb = blocks[t][blocks[t] >= 0]
        assert (np.diff(gb) > 0).all()
        _cutoff_ok(coarse, gb, o_blocks[0][o_blocks[0] >= 0], top_blocks, f"row {t} blocks")
        # fine level on the GPU's kept blocks
        _, o_idx, o_cnt, _ = oracle.hisa_topk(qk, wk, K, ko_t, rep_t, bo_t, topk, blk, top_blocks,
                                              given_blocks=blocks[t: t + 1])
        assert cnt[t] == o_cnt[0]
        gi = idx[t, : cnt[t]]
        assert (np.diff(gi) > 0).all() and (idx[t, cnt[t]:] == -1).all()
        ctx = ko[t + 1] - ko[t]
        nb = ctx // blk
        cand = np.concatenate([np.arange(b * blk, b * blk + blk) for b in gb] + [np.arange(nb * blk, ctx)])
        fine = oracle.indexer_score(qk[0], wk[0], K[ko[t] + cand])
        pos_score = dict(zip(cand.tolist(), fine.tolist()))
        # positions -> their slot in cand, to score a difference and bound it at an exact-0 cutoff
        slot = {int(p): i for i, p in enumerate(cand)}
        gsl = np.array([slot[int(p)] for p in gi], np.int64)
        osl = np.array([slot[int(p)] for p in o_idx[0, : o_cnt[0]]], np.int64)
        _cutoff_ok(fine, gsl, osl, topk, f"row {t} tokens",
                   floor_of=lambda d: indexer_abs_bound(qk[0].astype(np.float64), wk[0].astype(np.float64),
                                                        K[ko[t] + cand[d]].astype(np.float64)))


def test_representatives_match_oracle(crs, cuda_dev):
    case = workloads.indexer_decode_case(n_seq=5, ctx_lo=100, ctx_hi=3000, seed=31, device=cuda_dev)
    ko = case["offsets"]
    rep, bo = crs.hisa_describe(case["k_idx"], ko, 64, 3000)
    torch.cuda.synchronize()
    o_rep, o_bo = oracle.hisa_describe(case["k_idx"].float().cpu().numpy(), ko.cpu().numpy(), 64)
    assert np.array_equal(bo.cpu().numpy(), o_bo)
    np.testing.assert_allclose(rep.cpu().numpy()[: o_rep.shape[0]], o_rep, rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("blk,top_blocks,topk", [(64, 16, 256), (32, 40, 100), (64, 128, 2048)])
def test_hisa_small_rows(crs, cuda_dev, blk, top_blocks, topk):
    """Ragged rows: shorter than one block, fewer blocks than top_blocks, open blocks."""
    case = workloads.indexer_decode_case(n_seq=8, ctx_lo=20, ctx_hi=12000, seed=blk + top_blocks,
                                         device=cuda_dev)
    rep, bo, blocks, idx, cnt = _run(crs, cuda_dev, case, blk, top_blocks, topk, 12000)
    _check(case, rep, bo, blocks, idx, cnt, blk, top_blocks, topk)


def test_hisa_full_decode_config_sampled(crs, cuda_dev):
    """The indexer decode workload (64 rows, ctx up to 131072, top-2048) with 64-key blocks
    and 128 kept blocks; 4 rows checked against the oracle."""
    case = workloads.indexer_decode_case(device=cuda_dev)
    rep, bo, blocks, idx, cnt = _run(crs, cuda_dev, case, 64, 128, 2048, 131072)
    _check(case, rep, bo, blocks, idx, cnt, 64, 128, 2048, rows=[0, 17, 40, 63])


def test_hisa_row_beyond_max_keys_flags_device_error(crs, cuda_dev):
    case = workloads.indexer_decode_case(n_seq=3, ctx_lo=500, ctx_hi=900, seed=33, device=cuda_dev)
    ko = case["offsets"]
    rep, bo = crs.hisa_describe(case["k_idx"], ko, 64, 1000)
    crs.get_device_error()       # clear
    _, idx, cnt = crs.hisa_topk(case["q_idx"], case["w"], case["k_idx"], ko, rep, bo, 16, 64, 4, 400)
    torch.cuda.synchronize()
    assert crs.get_device_error() != 0
    assert (cnt.cpu().numpy() == 0).all() and (idx.cpu().numpy() == -1).all()

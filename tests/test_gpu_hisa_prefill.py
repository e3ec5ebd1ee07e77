"""HISA prefill (causal) form on the GPU against the oracle ("细粒度索引" page, HISA and
§2.2 Eq.(7); query t of one sequence is a decode row with ctx = t + 1 over the same keys).
Checked stage by stage on sampled rows: the kept blocks against the oracle's coarse
level on the GPU's representatives (a difference must sit at the coarse cutoff), the
tokens against the oracle's token level on the GPU's kept blocks (a difference must sit
at the token cutoff); counts and ordering exactly."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import cutoff_gaps, indexer_abs_bound

pytestmark = pytest.mark.gpu


def _run(crs, case, blk, top_blocks, topk):
    n = case["q_idx"].shape[0]
    dev = case["q_idx"].device
    ko = torch.tensor([0, n], dtype=torch.int64, device=dev)
    rep, _ = crs.hisa_describe(case["k_idx"], ko, blk, n)
    blocks, idx, cnt = crs.hisa_topk_prefill(case["q_idx"], case["w"], case["k_idx"], rep, topk, blk, top_blocks)
    torch.cuda.synchronize()
    assert crs.get_device_error() == 0
    return rep, blocks.cpu().numpy(), idx.cpu().numpy(), cnt.cpu().numpy()


def _check_rows(case, rep, blocks, idx, cnt, blk, top_blocks, topk, rows):
    K = case["k_idx"].double().cpu().numpy()
    q = case["q_idx"].double().cpu().numpy()
    w = case["w"].double().cpu().numpy()
    rep_np = rep.double().cpu().numpy()
    worst_b, worst_t, nd_b, nd_t = 0.0, 0.0, 0, 0
    for t in rows:
        ctx = t + 1
        nb = ctx // blk
        ko_t = np.array([0, ctx], np.int64)
        bo_t = np.array([0, nb], np.int64)
        rep_t = rep_np[:nb] if nb else np.zeros((1, 64))
        o_blocks, _, _, coarse = oracle.hisa_topk(q[t:t + 1], w[t:t + 1], K[:ctx], ko_t, rep_t, bo_t, topk, blk,
                                                  top_blocks)
        gb = blocks[t][blocks[t] >= 0]
        assert (np.diff(gb) > 0).all() and len(gb) == min(nb, top_blocks), f"row {t}"
        assert (blocks[t][len(gb):] == -1).all()
        d = np.setxor1d(gb, o_blocks[0][o_blocks[0] >= 0])
        if d.size:
            cut = float(np.sort(coarse[:nb])[::-1][top_blocks - 1])
            worst_b = max(worst_b, cutoff_gaps(coarse[d], cut, what=f"row {t} blocks"))
            nd_b += d.size
        # token level on the GPU's kept blocks
        _, o_idx, o_cnt, _ = oracle.hisa_topk(q[t:t + 1], w[t:t + 1], K[:ctx], ko_t, rep_t, bo_t, topk, blk,
                                              top_blocks, given_blocks=blocks[t:t + 1])
        assert cnt[t] == o_cnt[0], f"row {t}: count {cnt[t]} vs {o_cnt[0]}"
        gi = idx[t, : cnt[t]]
        assert (np.diff(gi) > 0).all() and (idx[t, cnt[t]:] == -1).all()
        cand = np.concatenate([np.arange(b * blk, b * blk + blk) for b in gb] + [np.arange(nb * blk, ctx)])
        d = np.setxor1d(gi, o_idx[0, : o_cnt[0]])
        if d.size:
            assert np.isin(d, cand).all(), f"row {t}: a token outside the kept blocks"
            fine = oracle.indexer_score(q[t], w[t], K[cand])
            cut = float(np.sort(fine)[::-1][min(topk, len(fine)) - 1])
            sd = oracle.indexer_score(q[t], w[t], K[d])
            worst_t = max(worst_t, cutoff_gaps(sd, cut, indexer_abs_bound(q[t], w[t], K[d]) if cut == 0.0 else None,
                                               what=f"row {t} tokens"))
            nd_t += d.size
    print(f"hisa prefill: {len(rows)} rows, {nd_b} differing blocks (gap {worst_b:.2e}), {nd_t} differing "
          f"tokens (gap {worst_t:.2e})")


@pytest.mark.parametrize("n,top_blocks,topk", [(3000, 32, 256), (5000, 16, 1024), (17000, 128, 2048)])
def test_hisa_prefill_small(crs, cuda_dev, n, top_blocks, topk):
    case = workloads.indexer_prefill_case(n=n, topk=topk, seed=n + top_blocks, device=cuda_dev)
    rep, blocks, idx, cnt = _run(crs, case, 64, top_blocks, topk)
    assert (cnt == np.minimum(topk, np.minimum(np.arange(n) + 1,
                                               np.minimum((np.arange(n) + 1) // 64, top_blocks) * 64
                                               + (np.arange(n) + 1) % 64))).all()
    rng = np.random.default_rng(n)
    edge = [0, 62, 63, 64, top_blocks * 64 - 1, top_blocks * 64, top_blocks * 64 + 63, top_blocks * 64 + 64,
            topk - 1, topk, n - 1]
    rows = np.unique(np.concatenate([[r for r in edge if 0 <= r < n], rng.choice(n, 60, replace=False)]))
    _check_rows(case, rep, blocks, idx, cnt, 64, top_blocks, topk, rows)


def test_hisa_prefill_matches_whole_oracle_on_a_small_sequence(crs, cuda_dev):
    """Every row of a 2500-token sequence against the oracle's prefill form run whole
    (its own representatives): equal counts, sets equal up to cutoff ties."""
    n, top_blocks, topk, blk = 2500, 12, 512, 64
    case = workloads.indexer_prefill_case(n=n, topk=topk, seed=99, device=cuda_dev)
    rep, blocks, idx, cnt = _run(crs, case, blk, top_blocks, topk)
    K = case["k_idx"].double().cpu().numpy()
    o_rep, _ = oracle.hisa_describe(K, np.array([0, n], np.int64), blk)
    np.testing.assert_allclose(rep.cpu().numpy()[: o_rep.shape[0]], o_rep, rtol=1e-5, atol=1e-6)
    o_blocks, o_idx, o_cnt = oracle.hisa_topk_prefill(case["q_idx"].double().cpu().numpy(),
                                                      case["w"].double().cpu().numpy(), K, o_rep, topk, blk,
                                                      top_blocks)
    assert np.array_equal(cnt, o_cnt)
    same_b = np.mean([np.array_equal(blocks[t], o_blocks[t]) for t in range(n)])
    same_t = np.mean([np.array_equal(idx[t], o_idx[t]) for t in range(n)])
    print(f"whole-oracle agreement: blocks {same_b:.4f}, tokens {same_t:.4f} of rows")
    # rows that differ anywhere are re-checked stage by stage (differences at cutoffs only)
    diff_rows = [t for t in range(n) if not (np.array_equal(blocks[t], o_blocks[t]) and
                                             np.array_equal(idx[t], o_idx[t]))]
    _check_rows(case, rep, blocks, idx, cnt, blk, top_blocks, topk, np.array(diff_rows[:200], np.int64))


def test_hisa_prefill_full_size_sampled(crs, cuda_dev):
    """The indexer prefill workload (n = 32768, needles) with 64-key blocks, 128 kept,
    top-2048: every row on the GPU, 48 sampled rows against the oracle."""
    case = workloads.indexer_prefill_case(device=cuda_dev)
    n, topk = case["params"]["n"], case["params"]["topk"]
    rep, blocks, idx, cnt = _run(crs, case, 64, 128, topk)
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([[0, 2047, 2048, 8191, 8192, 8255, 8256, 16383, n - 1],
                                     rng.choice(n, 40, replace=False)]))
    _check_rows(case, rep, blocks, idx, cnt, 64, 128, topk, rows)


def test_hisa_prefill_rejects_unsupported_shapes(crs, cuda_dev):
    case = workloads.indexer_prefill_case(n=1000, topk=256, seed=1, device=cuda_dev)
    ko = torch.tensor([0, 1000], dtype=torch.int64, device=cuda_dev)
    rep, _ = crs.hisa_describe(case["k_idx"], ko, 32, 1000)
    with pytest.raises(crs.CrsError):       # blocks of 32: not one key tile
        crs.hisa_topk_prefill(case["q_idx"], case["w"], case["k_idx"], rep, 256, 32, 16)
    rep, _ = crs.hisa_describe(case["k_idx"], ko, 64, 1000)
    with pytest.raises(crs.CrsError):       # top_blocks * blk < topk
        crs.hisa_topk_prefill(case["q_idx"], case["w"], case["k_idx"], rep, 256, 64, 2)

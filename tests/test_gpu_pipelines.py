"""Full-size pipelines against the oracle, in the launch configuration bench.py times.

Each workload runs its whole step on the GPU (selector -> index lists -> gather
attention); the oracle then recomputes, on sampled rows or on every row, first
the selection (the set rule: a difference must lie within 1e-5 relative of the
oracle's cutoff) and then the attention on the GPU's own index lists, element by
element within 2e-3 max(1, |oracle|) ([P1] PaperTrace 2.1.1 "最小正确性测试": the
same candidate set first, then the whole path).  The oracle reads compacted K/V
(the rows a list names, gathered by torch indexing and re-numbered): the same
arithmetic on fewer bytes of host memory.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import check_topk_row, cutoff_gaps, indexer_abs_bound, rel_err

pytestmark = pytest.mark.gpu
TOL = 2e-3


def _np(t):
    return t.detach().cpu().double().numpy()


def _attn_on_lists(Q, K, V, lists, kv_head, G):
    """Oracle attention of query heads [kv_head*G, +G) of one row over the keys `lists`
    (ascending positions into K/V [tokens, n_kv, D] on the device), re-numbered 0..c-1."""
    pos = torch.as_tensor(lists, dtype=torch.int64, device=K.device)
    Kc = K[pos, kv_head][:, None, :]
    Vc = V[pos, kv_head][:, None, :]
    Qr = Q[kv_head * G:(kv_head + 1) * G][None]
    I = np.arange(len(lists), dtype=np.int32)[None, None]
    O, lse = oracle.sparse_attn(_np(Qr), _np(Kc), _np(Vc), I)
    return O[0], lse[0]


def _check_o(g, o, what):
    err = rel_err(g, o)
    assert err.max() <= TOL, f"{what}: max rel err {err.max():.3e}"
    return float(err.max())


def test_indexer_prefill_then_attention_full_size(crs, cuda_dev):
    """n = 32768 causal, top-2048, 16 query heads over one K/V head: the bench's step
    (indexer_topk then sparse_attn with the causal limit q_pos = t), 40 sampled rows
    checked for the selected set and for every output element."""
    c = workloads.indexer_prefill_case(device=cuda_dev)
    p = c["params"]
    n, k = p["n"], p["topk"]
    idx, cnt = crs.indexer_topk(c["q_idx"], c["w"], c["k_idx"], k, crs.CRS_IDX_PREFILL)
    q_pos = torch.arange(n, dtype=torch.int32, device=cuda_dev)
    O, _ = crs.sparse_attn(c["Q"], c["K"], c["V"], idx.view(n, 1, k), q_pos=q_pos)
    torch.cuda.synchronize()
    assert crs.get_device_error() == 0
    rng = np.random.default_rng(3)
    rows = np.unique(np.concatenate([[0, 1, 2047, 2048, 16383, 16384, n - 1],
                                     rng.choice(n, 33, replace=False)]))
    g_idx, g_cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    qd, wd, Kd = _np(c["q_idx"]), _np(c["w"]), _np(c["k_idx"])
    o_idx, o_cnt, o_cut, _ = oracle.indexer_topk(qd[rows], wd[rows], Kd, np.zeros(len(rows), np.int64),
                                                 (rows + 1).astype(np.int32), k)
    worst_gap, worst_err = 0.0, 0.0
    for j, t in enumerate(rows):
        Kr = Kd[: t + 1]
        _, gap = check_topk_row(g_idx[t], g_cnt[t], o_idx[j], o_cnt[j], o_cut[j],
                                lambda pos: oracle.indexer_score(qd[t], wd[t], Kr[pos]),
                                lambda pos: indexer_abs_bound(qd[t], wd[t], Kr[pos]), what=f"row {t}")
        worst_gap = max(worst_gap, gap)
        lst = g_idx[t, : g_cnt[t]]
        oO, _ = _attn_on_lists(c["Q"][t], c["K"], c["V"], lst, 0, p["n_q_heads"])
        worst_err = max(worst_err, _check_o(O[t].cpu().double().numpy(), oO, f"row {t}"))
    print(f"prefill n={n}: {len(rows)} rows, largest cutoff gap {worst_gap:.3e}, largest rel err "
          f"{worst_err:.3e}")


def test_indexer_decode_then_attention_full_size(crs, cuda_dev):
    """64 sequences with ctx ~ U{8192..131072} (4.5 M cached tokens x 8 KV heads: K/V
    element offsets reach past 2^31), top-2048, 32 query heads over 8 KV heads: the
    bench's step; every row checked (set rule, then every output element)."""
    c = workloads.indexer_decode_case(device=cuda_dev)
    p = c["params"]
    ns, k, G = p["n_seq"], p["topk"], p["n_q_heads"] // p["n_kv_heads"]
    assert c["K"].numel() > 2 ** 31
    idx, cnt = crs.indexer_topk(c["q_idx"], c["w"], c["k_idx"], k, crs.CRS_IDX_DECODE,
                                k_offsets=c["offsets"], max_keys=131072)
    kv_base = c["offsets"][:-1].contiguous()
    q_pos = (c["ctx"] - 1).to(torch.int32).contiguous()
    O, _ = crs.sparse_attn(c["Q"], c["K"], c["V"], idx.view(ns, 1, k), kv_base=kv_base, q_pos=q_pos)
    torch.cuda.synchronize()
    assert crs.get_device_error() == 0
    g_idx, g_cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    off = c["offsets"].cpu().numpy()
    qd, wd = _np(c["q_idx"]), _np(c["w"])
    Og = O.cpu().double().numpy()
    worst_gap, worst_err = 0.0, 0.0
    for s in range(ns):
        Kr = _np(c["k_idx"][off[s]:off[s + 1]])
        o_idx, o_cnt, o_cut, _ = oracle.indexer_topk(qd[s:s + 1], wd[s:s + 1], Kr, np.zeros(1, np.int64),
                                                     np.array([Kr.shape[0]], np.int32), k)
        _, gap = check_topk_row(g_idx[s], g_cnt[s], o_idx[0], o_cnt[0], o_cut[0],
                                lambda pos: oracle.indexer_score(qd[s], wd[s], Kr[pos]),
                                lambda pos: indexer_abs_bound(qd[s], wd[s], Kr[pos]), what=f"seq {s}")
        worst_gap = max(worst_gap, gap)
        lst = off[s] + g_idx[s, : g_cnt[s]]
        for h in range(p["n_kv_heads"]):
            oO, _ = _attn_on_lists(c["Q"][s], c["K"], c["V"], lst, h, G)
            worst_err = max(worst_err, _check_o(Og[s, h * G:(h + 1) * G], oO, f"seq {s} kv {h}"))
    print(f"decode: {ns} rows, largest cutoff gap {worst_gap:.3e}, largest rel err {worst_err:.3e}")


def _block_pipeline(crs, c, fp4):
    p = c["params"]
    T, L, r, top, win = p["T"], p["L"], p["rank"], p["top_blocks"], p["window"]
    mu, xi = crs.block_describe(c["K"], L, r)
    if fp4:
        mu16, xi4, xs = crs.block_quantize(mu, xi, T, L)
        tok, cnt = crs.block_select_fp4(c["Q"], mu16, xi4, xs, T, L, top, win)
        desc = (mu16, xi4, xs)
    else:
        tok, cnt = crs.block_select(c["Q"], mu, xi, T, L, top, win)
        desc = (mu, xi)
    ns, nkv, D = p["n_seq"], p["n_kv_heads"], p["D"]
    Kf = c["K"].view(ns * T, nkv, D)
    Vf = c["V"].view(ns * T, nkv, D)
    kv_base = torch.arange(ns, dtype=torch.int64, device=c["K"].device) * T
    q_pos = torch.full((ns,), T - 1, dtype=torch.int32, device=c["K"].device)
    O, _ = crs.sparse_attn(c["Q"], Kf, Vf, tok, kv_base=kv_base, q_pos=q_pos)
    torch.cuda.synchronize()
    assert crs.get_device_error() == 0
    return desc, tok, cnt, O, Kf, Vf


@pytest.mark.parametrize("fp4", [False, True])
def test_block_select_then_attention_full_size(crs, cuda_dev, fp4):
    """Block-sparse decode, batch 32, T = 32768, 32 query heads over 4 KV heads, top-64
    blocks of 32 plus a 512-token window: describe, select (fp32 descriptors, or bf16
    means + FP4 eigenvectors), gather attention with its split-KV merge.  Selection
    checked on 8 sequences against the oracle on the GPU's descriptors (set rule);
    attention checked on every (sequence, KV head) list."""
    c = workloads.block_decode_case(device=cuda_dev)
    p = c["params"]
    T, L, top, win = p["T"], p["L"], p["top_blocks"], p["window"]
    G = p["n_q_heads"] // p["n_kv_heads"]
    desc, tok, cnt, O, Kf, Vf = _block_pipeline(crs, c, fp4)
    seqs = [0, 3, 9, 14, 20, 25, 30, 31]
    if fp4:
        omu = _np(desc[0])[seqs]
        oxi = oracle.fp4_dequantize(desc[1].cpu().numpy()[seqs], desc[2].cpu().numpy()[seqs])
    else:
        omu, oxi = _np(desc[0])[seqs], _np(desc[1])[seqs]
    o_tok, o_cnt, o_blk, o_bs = oracle.block_select(_np(c["Q"])[seqs], omu, oxi, T, L, top, win)
    g_tok, g_cnt = tok.cpu().numpy(), cnt.cpu().numpy()
    worst_gap, ndiff = 0.0, 0
    for j, s in enumerate(seqs):
        for h in range(p["n_kv_heads"]):
            gt = g_tok[s, h, : g_cnt[s, h]]
            assert (np.diff(gt) > 0).all() and (g_tok[s, h, g_cnt[s, h]:] == -1).all()
            gb = np.unique(gt[gt < T - win] // L)
            ob = np.unique(o_tok[j, h, : o_cnt[j, h]][o_tok[j, h, : o_cnt[j, h]] < T - win] // L)
            d = np.setxor1d(gb, ob)
            if d.size:
                cut = float(np.sort(o_bs[j, h])[::-1][top - 1])
                worst_gap = max(worst_gap, cutoff_gaps(o_bs[j, h][d], cut, what=f"seq {s} kv {h}"))
                ndiff += d.size
            else:
                assert g_cnt[s, h] == o_cnt[j, h]
    Og = O.cpu().double().numpy()
    worst_err = 0.0
    for s in range(p["n_seq"]):
        for h in range(p["n_kv_heads"]):
            lst = s * T + g_tok[s, h, : g_cnt[s, h]]
            oO, _ = _attn_on_lists(c["Q"][s], Kf, Vf, lst, h, G)
            worst_err = max(worst_err, _check_o(Og[s, h * G:(h + 1) * G], oO, f"seq {s} kv {h}"))
    print(f"block fp4={fp4}: {ndiff} differing blocks, largest cutoff gap {worst_gap:.3e}, largest "
          f"rel err {worst_err:.3e}")


def test_route_full_size_sampled_segments(crs, cuda_dev):
    """Routing with quotas at the bench's size (B = 2, H = 8, n = 16384, C = 128 unit
    centres, m = 128, causal): the GPU runs the whole batch; two (batch, head)
    segments are recomputed by the oracle (quotas and counts exactly, outputs within
    2e-3)."""
    B, H, n, d, C, m = 2, 8, 16384, 64, 128, 128
    g = torch.Generator(device="cpu").manual_seed(81)
    Q = torch.randn(B, H, n, d, generator=g).to(torch.bfloat16)
    K = torch.randn(B, H, n, d, generator=g).to(torch.bfloat16)
    V = torch.randn(B, H, n, d, generator=g).to(torch.bfloat16)
    M = torch.randn(H, C, d, generator=g)
    M = M / M.norm(dim=-1, keepdim=True)
    JQ, JK, O, lse, cnt = crs.route_attn(Q.to(cuda_dev), K.to(cuda_dev), V.to(cuda_dev), M.to(cuda_dev), m,
                                         causal=True)
    torch.cuda.synchronize()
    assert crs.get_device_error() == 0
    for b, h in [(0, 0), (1, 5)]:
        sl = (slice(b, b + 1), slice(h, h + 1))
        oJQ, oJK, oO, olse, ocnt = oracle.kmeans_route(Q[sl].float().numpy(), K[sl].float().numpy(),
                                                       V[sl].float().numpy(), M[h:h + 1].numpy(), m,
                                                       causal=True)
        assert np.array_equal(JQ[sl].cpu().numpy(), oJQ)
        assert np.array_equal(JK[sl].cpu().numpy(), oJK)
        assert np.array_equal(cnt[sl].cpu().numpy(), ocnt)
        _check_o(O[sl].cpu().double().numpy(), oO, f"route ({b},{h})")
        gl, fin = lse[sl].cpu().numpy(), np.isfinite(olse)
        assert np.array_equal(np.isfinite(gl), fin)
        assert np.abs(gl[fin] - olse[fin]).max() <= TOL * max(1.0, np.abs(olse[fin]).max())

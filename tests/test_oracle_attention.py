"""Pins for the oracle's attention over a given index set."""
import math

import numpy as np
import pytest
import torch

import oracle
from conftest import golden


def test_kmeans_example_weights_and_output():
    """PaperTrace 2.1.1 §3.2 worked example, as 1-D attention with raw scores."""
    g = golden("p1_kmeans_example.json")
    pr = g["printed"]
    s = np.array(pr["scores"])
    v = np.array(pr["values"])
    Q = np.ones((1, 1, 1))
    K = s[:, None, None]
    V = v[:, None, None]
    I = np.arange(3, dtype=np.int32)[None, None]
    O, lse = oracle.sparse_attn(Q, K, V, I, scale=1.0)
    wts = np.exp(s - lse[0, 0])
    assert wts == pytest.approx(pr["weights"], abs=5e-4)
    assert O[0, 0, 0] == pytest.approx(g["derived"]["output"], abs=5e-4)


def _dense_sdpa(Q, K, V, mask, scale):
    """torch SDPA in fp64; Q [rows, n_q, D], K/V [tokens, n_kv, D]."""
    n_q, n_kv = Q.shape[1], K.shape[1]
    G = n_q // n_kv
    q = torch.from_numpy(Q).permute(1, 0, 2)                        # [n_q, rows, D]
    k = torch.from_numpy(K).permute(1, 0, 2).repeat_interleave(G, 0)
    v = torch.from_numpy(V).permute(1, 0, 2).repeat_interleave(G, 0)
    o = torch.nn.functional.scaled_dot_product_attention(
        q, k, v, attn_mask=torch.from_numpy(mask)[None], scale=scale)
    return o.permute(1, 0, 2).numpy()


@pytest.mark.parametrize("n_q,n_kv", [(4, 1), (4, 2), (3, 3)])
def test_all_visible_is_dense_causal(n_q, n_kv):
    """PaperTrace 2.1.1 "最小正确性测试": full candidate set -> dense causal attention."""
    rng = np.random.default_rng(n_q * 10 + n_kv)
    n, D = 37, 16
    Q = rng.standard_normal((n, n_q, D))
    K = rng.standard_normal((n, n_kv, D))
    V = rng.standard_normal((n, n_kv, D))
    I = np.full((n, 1, n), -1, np.int32)
    for t in range(n):
        I[t, 0, : t + 1] = np.arange(t + 1)
    O, lse = oracle.sparse_attn(Q, K, V, I)
    mask = np.tril(np.ones((n, n), bool))
    ref = _dense_sdpa(Q, K, V, mask, 1.0 / math.sqrt(D))
    assert np.abs(O - ref).max() < 1e-12


@pytest.mark.parametrize("n_q,n_kv", [(4, 1), (6, 2)])
def test_masks_on_full_lists_are_dense_causal_with_padding(n_q, n_kv):
    """PaperTrace 2.1.1 §1.1 Eq.(2): the allowed set is cut by the causal and the padding
    masks.  Every row lists every key; q_pos and key_valid alone must then give dense
    attention under the mask (j <= i) & valid(j) (torch SDPA, fp64), on two sequences
    packed behind kv_base."""
    rng = np.random.default_rng(n_q + 7 * n_kv)
    lens, D = [23, 31], 16
    base = np.array([0, lens[0]], np.int64)
    tokens = sum(lens)
    K = rng.standard_normal((tokens, n_kv, D))
    V = rng.standard_normal((tokens, n_kv, D))
    valid = rng.random(tokens) > 0.3
    valid[[0, lens[0]]] = True                      # every row keeps at least one key
    rows_q, rows_b, rows_p = [], [], []
    for s_, n in enumerate(lens):
        for t in range(n):
            rows_b.append(base[s_])
            rows_p.append(t)
    rows = len(rows_b)
    Q = rng.standard_normal((rows, n_q, D))
    nmax = max(lens)
    I = np.full((rows, 1, nmax), -1, np.int32)
    for r in range(rows):
        n = lens[0] if rows_b[r] == 0 else lens[1]
        I[r, 0, :n] = rng.permutation(n)            # list order does not matter
    O, lse = oracle.sparse_attn(Q, K, V, I, kv_base=np.array(rows_b), key_valid=valid,
                                q_pos=np.array(rows_p, np.int32))
    scale = 1.0 / math.sqrt(D)
    r0 = 0
    for s_, n in enumerate(lens):
        b = int(base[s_])
        i = np.arange(n)[:, None]
        j = np.arange(n)[None]
        mask = (j <= i) & valid[b:b + n][None]
        ref = _dense_sdpa(Q[r0:r0 + n], K[b:b + n], V[b:b + n], mask, scale)
        assert np.abs(O[r0:r0 + n] - ref).max() < 1e-12
        r0 += n
    # the unmasked call attends to every listed key
    O2, _ = oracle.sparse_attn(Q[:lens[0]], K[:lens[0]], V[:lens[0]], I[:lens[0], :, :lens[0]])
    ref2 = _dense_sdpa(Q[:lens[0]], K[:lens[0]], V[:lens[0]], np.ones((lens[0], lens[0]), bool), scale)
    assert np.abs(O2 - ref2).max() < 1e-12


def test_masks_that_remove_every_entry_give_zero():
    rng = np.random.default_rng(9)
    Q = rng.standard_normal((2, 2, 8))
    K = rng.standard_normal((10, 1, 8))
    V = rng.standard_normal((10, 1, 8))
    I = np.array([[[5, 6, 7]], [[1, 2, -1]]], np.int32)
    valid = np.ones(10, bool)
    valid[[1, 2]] = False
    O, lse = oracle.sparse_attn(Q, K, V, I, key_valid=valid, q_pos=np.array([4, 9], np.int32))
    assert (O == 0).all() and (lse == -np.inf).all()


def test_window_is_sliding_window_attention():
    rng = np.random.default_rng(1)
    n, D, W = 50, 8, 6
    Q = rng.standard_normal((n, 2, D))
    K = rng.standard_normal((n, 1, D))
    V = rng.standard_normal((n, 1, D))
    I = np.full((n, 1, W), -1, np.int32)
    for t in range(n):
        lo = max(0, t - W + 1)
        I[t, 0, : t - lo + 1] = np.arange(lo, t + 1)
    O, _ = oracle.sparse_attn(Q, K, V, I)
    i = np.arange(n)[:, None]
    j = np.arange(n)[None]
    ref = _dense_sdpa(Q, K, V, (j <= i) & (j > i - W), 1.0 / math.sqrt(D))
    assert np.abs(O - ref).max() < 1e-12


def test_per_kv_lists_and_empty_rows():
    rng = np.random.default_rng(2)
    n, D = 20, 8
    Q = rng.standard_normal((2, 4, D))
    K = rng.standard_normal((n, 2, D))
    V = rng.standard_normal((n, 2, D))
    I = np.full((2, 2, 5), -1, np.int32)
    I[0, 0, :3] = [1, 4, 9]
    I[0, 1, :2] = [0, 19]
    # row 1, kv head 0: empty list -> 0 and lse = -inf
    I[1, 1, :5] = [3, 5, 7, 11, 13]
    O, lse = oracle.sparse_attn(Q, K, V, I)
    assert (O[1, :2] == 0).all() and (lse[1, :2] == -np.inf).all()
    for g in range(4):
        h = g // 2
        lst = [x for x in I[0, h] if x >= 0]
        s = K[lst, h] @ Q[0, g] / math.sqrt(D)
        p = np.exp(s - s.max())
        p /= p.sum()
        assert np.abs(O[0, g] - p @ V[lst, h]).max() < 1e-12


def test_drop_error_identity_block_partition():
    """COBS notes Eq.(3): o* - o_S = 1/(1-tau) sum_{b not in S} P_b (v_b^c - o*),
    with P_b, v_b^c from per-block attention (Eq.(1), (P3))."""
    rng = np.random.default_rng(3)
    nb, L, D = 6, 5, 4
    n = nb * L
    Q = rng.standard_normal((1, 1, D))
    K = rng.standard_normal((n, 1, D))
    V = rng.standard_normal((n, 1, D))
    all_idx = np.arange(n, dtype=np.int32)[None, None]
    o_star, lse_all = oracle.sparse_attn(Q, K, V, all_idx)
    P, vc = [], []
    for b in range(nb):
        ob, lb = oracle.sparse_attn(Q, K, V, np.arange(b * L, b * L + L, dtype=np.int32)[None, None])
        P.append(math.exp(lb[0, 0] - lse_all[0, 0]))
        vc.append(ob[0, 0])
    assert sum(P) == pytest.approx(1.0)
    assert np.abs(sum(P[b] * vc[b] for b in range(nb)) - o_star[0, 0]).max() < 1e-12  # Eq.(P3)
    S = [0, 2, 3]
    keep = np.concatenate([np.arange(b * L, b * L + L) for b in S]).astype(np.int32)
    o_S, _ = oracle.sparse_attn(Q, K, V, keep[None, None])
    tau = sum(P[b] for b in range(nb) if b not in S)
    rhs = sum(P[b] * (vc[b] - o_star[0, 0]) for b in range(nb) if b not in S) / (1 - tau)
    assert np.abs((o_star[0, 0] - o_S[0, 0]) - rhs).max() < 1e-12

"""GPU parity: block descriptors and block selection vs the oracle."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import cutoff_gaps, rel_err

pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().cpu().float().numpy().astype(np.float64)


def _blocks(K, L):
    """[n_seq, T, n_kv, D] -> [n_seq, n_kv, n_full, L, D] (full blocks only)."""
    n_seq, T, n_kv, D = K.shape
    nf = T // L
    return K[:, : nf * L].reshape(n_seq, nf, L, n_kv, D).transpose(0, 3, 1, 2, 4)


def _oracle_describe(Kd, L, rank):
    kb = _blocks(Kd, L)
    s, h, nf = kb.shape[:3]
    mu, xi, lam = oracle.block_describe(kb.reshape(-1, L, kb.shape[-1]), rank + 1)
    return (mu.reshape(s, h, nf, -1), xi.reshape(s, h, nf, rank + 1, -1),
            lam.reshape(s, h, nf, rank + 1))


def test_describe_small(crs, cuda_dev):
    case = workloads.block_decode_case(n_seq=2, T=32 * 40 + 7, seed=3, device=cuda_dev)
    p = case["params"]
    L, r = p["L"], p["rank"]
    mu, xi = crs.block_describe(case["K"], L, r)
    torch.cuda.synchronize()
    Kd = _np(case["K"])
    omu, oxi, olam = _oracle_describe(Kd, L, r)
    assert rel_err(_np(mu), omu).max() < 1e-5
    g = _np(xi)
    glam = (g ** 2).sum(-1)                          # |xi_i|^2 = lambda_i
    assert np.abs(glam - olam[..., :r]).max() <= 1e-4 * olam[..., 0].max()
    # the rank-r factor sum xi xi^T where the r-th eigengap is clear of fp32 noise
    gap = (olam[..., r - 1] - olam[..., r]) / olam[..., 0]
    P = np.einsum("shbrd,shbre->shbde", g, g)
    Po = np.einsum("shbrd,shbre->shbde", oxi[..., :r, :], oxi[..., :r, :])
    err = np.abs(P - Po).max(axis=(-1, -2)) / olam[..., 0]
    ok = gap > 1e-3
    assert ok.mean() > 0.9
    assert (err[ok] <= 1e-4 / gap[ok]).all()


def _check_select(tok, cnt, o_tok, o_cnt, o_blk, o_bs, L, T, window, top, what):
    """Token lists ascending and -1 padded; kept blocks equal to the oracle's except
    blocks whose oracle score lies within 1e-5 relative of the cutoff."""
    n_seq, n_kv = cnt.shape
    ndiff, worst = 0, 0.0
    for s in range(n_seq):
        for h in range(n_kv):
            gt = tok[s, h, : cnt[s, h]]
            ot = o_tok[s, h, : o_cnt[s, h]]
            assert (np.diff(gt) > 0).all() and (tok[s, h, cnt[s, h]:] == -1).all()
            gb = np.unique(gt[gt < max(0, T - window)] // L)
            ob = np.unique(ot[ot < max(0, T - window)] // L)
            diff = np.setxor1d(gb, ob)
            if diff.size:
                sc = o_bs[s, h]
                cut = float(np.sort(sc)[::-1][top - 1])
                worst = max(worst, cutoff_gaps(sc[diff], cut, what=f"{what} ({s},{h}) blocks {diff}"))
                ndiff += diff.size
            else:
                assert cnt[s, h] == o_cnt[s, h]
    print(f"{what}: {n_seq * n_kv} (sequence, KV head) sets, {ndiff} differing blocks, largest "
          f"relative gap to the cutoff {worst:.3e}")
    return ndiff


def test_select_on_oracle_descriptors(crs, cuda_dev):
    """Selection alone: the GPU reads the oracle's descriptors (rounded to fp32)."""
    case = workloads.block_decode_case(n_seq=3, T=4096, seed=5, device=cuda_dev)
    p = case["params"]
    L, r, top, win = p["L"], p["rank"], 16, 256
    omu, oxi, _ = _oracle_describe(_np(case["K"]), L, r)
    oxi = oxi[..., :r, :]
    mu32 = torch.from_numpy(omu.astype(np.float32)).to(cuda_dev)
    xi32 = torch.from_numpy(oxi.astype(np.float32)).to(cuda_dev)
    tok, cnt = crs.block_select(case["Q"], mu32, xi32, p["T"], L, top, win)
    torch.cuda.synchronize()
    o_tok, o_cnt, o_blk, o_bs = oracle.block_select(
        _np(case["Q"]), mu32.double().cpu().numpy(), xi32.double().cpu().numpy(), p["T"], L, top, win)
    _check_select(tok.cpu().numpy(), cnt.cpu().numpy(), o_tok, o_cnt, o_blk, o_bs, L, p["T"], win,
                  top, "select")


def test_select_ragged_block_count(crs, cuda_dev):
    """50 complete blocks (a partial last chunk of the streamed descriptors) and a partial
    last block of tokens: selection alone on the oracle's descriptors."""
    T = 32 * 50 + 13
    case = workloads.block_decode_case(n_seq=2, T=T, seed=17, device=cuda_dev)
    p = case["params"]
    L, r, top, win = p["L"], p["rank"], 9, 100
    omu, oxi, _ = _oracle_describe(_np(case["K"]), L, r)
    mu32 = torch.from_numpy(omu.astype(np.float32)).to(cuda_dev)
    xi32 = torch.from_numpy(oxi[..., :r, :].astype(np.float32)).to(cuda_dev)
    tok, cnt = crs.block_select(case["Q"], mu32, xi32, T, L, top, win)
    torch.cuda.synchronize()
    o_tok, o_cnt, o_blk, o_bs = oracle.block_select(
        _np(case["Q"]), mu32.double().cpu().numpy(), xi32.double().cpu().numpy(), T, L, top, win)
    _check_select(tok.cpu().numpy(), cnt.cpu().numpy(), o_tok, o_cnt, o_blk, o_bs, L, T, win, top,
                  "select-ragged")


def test_describe_select_end_to_end_small(crs, cuda_dev):
    """Describe then select, checked stage by stage ([P1] "最小正确性测试": the same
    inputs first).  The fp32 descriptors against the fp64 oracle within the fp32
    Jacobi bounds of test_describe_small; the selection against the oracle run on
    those GPU descriptors under the 1e-5 cutoff rule.  (The oracle's own fp64
    descriptors move a block score by up to ~1e-4 relative when the fp32 eigen
    decomposition differs at that level, which no cutoff rule on the selection
    alone can separate from a selection fault.)"""
    case = workloads.block_decode_case(n_seq=2, T=2048, seed=6, device=cuda_dev)
    p = case["params"]
    L, r, top, win = p["L"], p["rank"], 8, 128
    mu, xi = crs.block_describe(case["K"], L, r)
    tok, cnt = crs.block_select(case["Q"], mu, xi, p["T"], L, top, win)
    torch.cuda.synchronize()
    omu, oxi, olam = _oracle_describe(_np(case["K"]), L, r)
    assert rel_err(_np(mu), omu).max() < 1e-5
    glam = (_np(xi) ** 2).sum(-1)
    assert np.abs(glam - olam[..., :r]).max() <= 1e-4 * olam[..., 0].max()
    o_tok, o_cnt, o_blk, o_bs = oracle.block_select(_np(case["Q"]), _np(mu), _np(xi), p["T"], L,
                                                    top, win)
    _check_select(tok.cpu().numpy(), cnt.cpu().numpy(), o_tok, o_cnt, o_blk, o_bs, L, p["T"], win,
                  top, "describe+select")


def test_quantize_matches_oracle_bit_exact(crs, cuda_dev):
    """FP4 codes and scales equal the oracle's (integers decided in fp32), the bf16 mean is
    round-to-nearest-even ([P5] §5.5)."""
    case = workloads.block_decode_case(n_seq=2, T=32 * 37, seed=8, device=cuda_dev)
    p = case["params"]
    mu, xi = crs.block_describe(case["K"], p["L"], p["rank"])
    # a few planted values on the rounding midpoints and an all-zero vector
    xi[0, 0, 0, 0] = 0.0
    xi[0, 0, 1, 0, :8] = torch.tensor([6.0, 2.5, 0.25, 0.75, 1.25, 1.75, 3.5, 5.0], device=cuda_dev)
    xi[0, 0, 1, 0, 8:] = 0.1
    mu16, xi4, xs = crs.block_quantize(mu, xi, p["T"], p["L"])
    torch.cuda.synchronize()
    o_codes, o_scale = oracle.fp4_quantize(xi.cpu().numpy())
    assert np.array_equal(xi4.cpu().numpy(), o_codes)
    assert np.array_equal(xs.cpu().numpy(), o_scale)
    assert torch.equal(mu16.cpu(), mu.cpu().to(torch.bfloat16))
    assert xs[0, 0, 0, 0].item() == 0.0 and (xi4[0, 0, 0, 0] == 0).all()


@pytest.mark.parametrize("n_seq,T,top,win", [(3, 4096, 16, 256), (2, 32 * 50 + 13, 9, 100)])
def test_select_fp4_on_its_own_descriptors(crs, cuda_dev, n_seq, T, top, win):
    """Selection over compressed descriptors equals the oracle's selection over the same
    dequantised descriptors (set rule at the cutoff)."""
    case = workloads.block_decode_case(n_seq=n_seq, T=T, seed=T, device=cuda_dev)
    p = case["params"]
    L, r = p["L"], p["rank"]
    mu, xi = crs.block_describe(case["K"], L, r)
    mu16, xi4, xs = crs.block_quantize(mu, xi, T, L)
    tok, cnt = crs.block_select_fp4(case["Q"], mu16, xi4, xs, T, L, top, win)
    torch.cuda.synchronize()
    omu = _np(mu16)
    oxi = oracle.fp4_dequantize(xi4.cpu().numpy(), xs.cpu().numpy())
    o_tok, o_cnt, o_blk, o_bs = oracle.block_select(_np(case["Q"]), omu, oxi, T, L, top, win)
    _check_select(tok.cpu().numpy(), cnt.cpu().numpy(), o_tok, o_cnt, o_blk, o_bs, L, T, win,
                  top, "select-fp4")


def test_select_fp4_full_config_sampled(crs, cuda_dev):
    """The block-sparse decode workload (32 seqs, T = 32768) on FP4 descriptors: every
    (sequence, KV head) set checked against the oracle on the dequantised descriptors for
    4 sampled sequences."""
    case = workloads.block_decode_case(device=cuda_dev)
    p = case["params"]
    T, L, r, top, win = p["T"], p["L"], p["rank"], p["top_blocks"], p["window"]
    mu, xi = crs.block_describe(case["K"], L, r)
    mu16, xi4, xs = crs.block_quantize(mu, xi, T, L)
    tok, cnt = crs.block_select_fp4(case["Q"], mu16, xi4, xs, T, L, top, win)
    torch.cuda.synchronize()
    assert crs.get_device_error() == 0
    seqs = [0, 7, 19, 31]
    omu = _np(mu16)[seqs]
    oxi = oracle.fp4_dequantize(xi4.cpu().numpy()[seqs], xs.cpu().numpy()[seqs])
    o_tok, o_cnt, o_blk, o_bs = oracle.block_select(_np(case["Q"])[seqs], omu, oxi, T, L, top, win)
    _check_select(tok.cpu().numpy()[seqs], cnt.cpu().numpy()[seqs], o_tok, o_cnt, o_blk, o_bs, L, T,
                  win, top, "select-fp4-full")


@pytest.mark.parametrize("n_q,n_kv,rank,T,top,win", [
    (16, 4, 2, 32 * 300 + 5, 20, 64),     # G = 4, three tiles of 128 blocks, ragged last tile
    (64, 4, 1, 32 * 130, 7, 0),           # G = 16 (every column of the MMA), rank 1
    (8, 2, 3, 32 * 257, 31, 300),         # G = 4, rank 3, one block past two full tiles
])
def test_select_fp4_head_and_rank_shapes(crs, cuda_dev, n_q, n_kv, rank, T, top, win):
    """Compressed-descriptor selection for other query-group sizes and ranks, several
    (sequence, KV head) pairs per CTA, against the oracle on the dequantised descriptors."""
    case = workloads.block_decode_case(n_seq=3, T=T, n_kv_heads=n_kv, n_q_heads=n_q, rank=rank,
                                       seed=T + n_q, device=cuda_dev)
    p = case["params"]
    L = p["L"]
    mu, xi = crs.block_describe(case["K"], L, rank)
    mu16, xi4, xs = crs.block_quantize(mu, xi, T, L)
    tok, cnt = crs.block_select_fp4(case["Q"], mu16, xi4, xs, T, L, top, win)
    torch.cuda.synchronize()
    assert crs.get_device_error() == 0
    omu = _np(mu16)
    oxi = oracle.fp4_dequantize(xi4.cpu().numpy(), xs.cpu().numpy())
    o_tok, o_cnt, o_blk, o_bs = oracle.block_select(_np(case["Q"]), omu, oxi, T, L, top, win)
    _check_select(tok.cpu().numpy(), cnt.cpu().numpy(), o_tok, o_cnt, o_blk, o_bs, L, T, win,
                  top, f"select-fp4-G{n_q // n_kv}-r{rank}")


@pytest.mark.parametrize("n_full,n_q,n_kv,top", [(1500, 16, 2, 40), (3000, 8, 2, 100), (5000, 16, 2, 64),
                                                 (8192, 4, 2, 300)])
def test_select_many_blocks(crs, cuda_dev, n_full, n_q, n_kv, top):
    """More than 1024 blocks per (sequence, KV head): several blocks per thread in the
    pick kernel.  Random descriptors with planted exact ties at the cutoff."""
    rng = np.random.default_rng(n_full)
    L, D, rank, win = 32, 128, 2, 200
    T = n_full * L + 7
    mu = rng.standard_normal((1, n_kv, n_full, D)).astype(np.float32)
    xi = (0.3 * rng.standard_normal((1, n_kv, n_full, rank, D))).astype(np.float32)
    mu[0, 0, 7] = mu[0, 0, 3]            # identical descriptors -> identical block scores
    xi[0, 0, 7] = xi[0, 0, 3]
    Q = torch.from_numpy(rng.standard_normal((1, n_q, D)).astype(np.float32)).to(torch.bfloat16)
    tok, cnt = crs.block_select(Q.to(cuda_dev), torch.from_numpy(mu).to(cuda_dev),
                                torch.from_numpy(xi).to(cuda_dev), T, L, top, win)
    torch.cuda.synchronize()
    assert crs.get_device_error() == 0
    o_tok, o_cnt, o_blk, o_bs = oracle.block_select(Q.float().numpy(), mu, xi, T, L, top, win)
    _check_select(tok.cpu().numpy(), cnt.cpu().numpy(), o_tok, o_cnt, o_blk, o_bs, L, T, win, top,
                  f"select-{n_full}")


# ---------------------------------------------------------------- Quest / mean-pool --
def test_quest_describe_matches_oracle_bit_exact(crs, cuda_dev):
    """kmin / kmax are key values: bf16 on the GPU, equal to the oracle's min / max."""
    case = workloads.block_decode_case(n_seq=2, T=32 * 37 + 5, seed=9, device=cuda_dev)
    p = case["params"]
    kmin, kmax = crs.quest_describe(case["K"], p["L"])
    torch.cuda.synchronize()
    o_min, o_max = oracle.quest_describe(_np(case["K"]), p["L"])
    assert np.array_equal(kmin.double().cpu().numpy(), o_min)
    assert np.array_equal(kmax.double().cpu().numpy(), o_max)


@pytest.mark.parametrize("n_q,n_kv,T,top,win", [
    (32, 4, 4096, 16, 256),          # G = 8
    (16, 4, 32 * 300 + 5, 20, 64),   # G = 4, ragged
    (64, 4, 32 * 130, 7, 0),         # G = 16
    (4, 4, 32 * 77, 9, 100),         # G = 1
])
def test_select_quest_matches_oracle(crs, cuda_dev, n_q, n_kv, T, top, win):
    case = workloads.block_decode_case(n_seq=3, T=T, n_kv_heads=n_kv, n_q_heads=n_q, seed=T + n_q,
                                       device=cuda_dev)
    L = case["params"]["L"]
    kmin, kmax = crs.quest_describe(case["K"], L)
    tok, cnt = crs.block_select_quest(case["Q"], kmin, kmax, T, L, top, win)
    torch.cuda.synchronize()
    assert crs.get_device_error() == 0
    o_tok, o_cnt, o_blk, o_bs = oracle.quest_select(_np(case["Q"]), kmin.double().cpu().numpy(),
                                                    kmax.double().cpu().numpy(), T, L, top, win)
    _check_select(tok.cpu().numpy(), cnt.cpu().numpy(), o_tok, o_cnt, o_blk, o_bs, L, T, win, top,
                  f"quest-G{n_q // n_kv}")


@pytest.mark.parametrize("n_q,n_kv,T,top,win", [(32, 4, 4096, 16, 256), (16, 4, 32 * 300 + 5, 20, 64),
                                                (64, 4, 32 * 130, 7, 0)])
def test_select_meanpool_matches_oracle(crs, cuda_dev, n_q, n_kv, T, top, win):
    """Rank 0 (xi = None): the first-order score q . mu alone."""
    case = workloads.block_decode_case(n_seq=3, T=T, n_kv_heads=n_kv, n_q_heads=n_q, seed=T + 1,
                                       device=cuda_dev)
    L = case["params"]["L"]
    mu, _ = crs.block_describe(case["K"], L, 1)
    tok, cnt = crs.block_select(case["Q"], mu, None, T, L, top, win)
    torch.cuda.synchronize()
    assert crs.get_device_error() == 0
    omu = mu.double().cpu().numpy()
    oxi = np.zeros(omu.shape[:3] + (0, omu.shape[3]))
    o_tok, o_cnt, o_blk, o_bs = oracle.block_select(_np(case["Q"]), omu, oxi, T, L, top, win)
    _check_select(tok.cpu().numpy(), cnt.cpu().numpy(), o_tok, o_cnt, o_blk, o_bs, L, T, win, top,
                  f"meanpool-G{n_q // n_kv}")


def test_select_quest_full_config_sampled(crs, cuda_dev):
    """The block-sparse decode workload (32 seqs, T = 32768) with the Quest selector; 4
    sampled sequences checked against the oracle."""
    case = workloads.block_decode_case(device=cuda_dev)
    p = case["params"]
    T, L, top, win = p["T"], p["L"], p["top_blocks"], p["window"]
    kmin, kmax = crs.quest_describe(case["K"], L)
    tok, cnt = crs.block_select_quest(case["Q"], kmin, kmax, T, L, top, win)
    torch.cuda.synchronize()
    assert crs.get_device_error() == 0
    seqs = [0, 11, 22, 31]
    o_tok, o_cnt, o_blk, o_bs = oracle.quest_select(_np(case["Q"])[seqs], kmin.double().cpu().numpy()[seqs],
                                                    kmax.double().cpu().numpy()[seqs], T, L, top, win)
    _check_select(tok.cpu().numpy()[seqs], cnt.cpu().numpy()[seqs], o_tok, o_cnt, o_blk, o_bs, L, T,
                  win, top, "quest-full")


# ---------------------------------------------------------------- query subspace --
def test_describe_ss_matches_oracle(crs, cuda_dev):
    """Subspace descriptors (s = 85 of D = 128): the mean, the eigenvalues of U^T Sigma U and
    the rank-r factor sum xi xi^T (where the r-th eigengap is clear of fp32 noise)."""
    case = workloads.block_decode_case(n_seq=2, T=32 * 40 + 7, seed=14, device=cuda_dev)
    p = case["params"]
    L, r = p["L"], p["rank"]
    U = workloads.query_subspace(128, 85, device=cuda_dev)
    mu, xi = crs.block_describe_ss(case["K"], L, r, U)
    torch.cuda.synchronize()
    kb = _blocks(_np(case["K"]), L)
    s_, h_, nf = kb.shape[:3]
    omu, oxi, olam = oracle.block_describe_ss(kb.reshape(-1, L, 128), U.double().cpu().numpy(), r + 1)
    omu, oxi, olam = omu.reshape(s_, h_, nf, -1), oxi.reshape(s_, h_, nf, r + 1, -1), olam.reshape(s_, h_, nf, r + 1)
    assert rel_err(_np(mu), omu).max() < 1e-5
    g = _np(xi)
    assert np.abs((g ** 2).sum(-1) - olam[..., :r]).max() <= 1e-4 * olam[..., 0].max()
    gap = (olam[..., r - 1] - olam[..., r]) / olam[..., 0]
    P = np.einsum("shbrd,shbre->shbde", g, g)
    Po = np.einsum("shbrd,shbre->shbde", oxi[..., :r, :], oxi[..., :r, :])
    err = np.abs(P - Po).max(axis=(-1, -2)) / olam[..., 0]
    ok = gap > 1e-3
    assert ok.mean() > 0.9
    assert (err[ok] <= 1e-4 / gap[ok]).all()


@pytest.mark.parametrize("n_q,n_kv,T,top,win,sd", [(32, 4, 4096, 16, 256, 85), (16, 4, 32 * 300 + 5, 20, 64, 48),
                                                   (4, 4, 32 * 90, 9, 100, 128)])
def test_select_ss_matches_oracle(crs, cuda_dev, n_q, n_kv, T, top, win, sd):
    case = workloads.block_decode_case(n_seq=3, T=T, n_kv_heads=n_kv, n_q_heads=n_q, seed=T + sd,
                                       device=cuda_dev)
    p = case["params"]
    L, r = p["L"], p["rank"]
    U = workloads.query_subspace(128, sd, seed=sd, device=cuda_dev)
    mu, xi = crs.block_describe_ss(case["K"], L, r, U)
    tok, cnt = crs.block_select_ss(case["Q"], U, mu, xi, T, L, top, win)
    torch.cuda.synchronize()
    assert crs.get_device_error() == 0
    o_tok, o_cnt, o_blk, o_bs = oracle.block_select_ss(_np(case["Q"]), U.double().cpu().numpy(),
                                                       mu.double().cpu().numpy(), xi.double().cpu().numpy(),
                                                       T, L, top, win)
    _check_select(tok.cpu().numpy(), cnt.cpu().numpy(), o_tok, o_cnt, o_blk, o_bs, L, T, win, top,
                  f"ss{sd}-G{n_q // n_kv}")


def test_select_one_query_head_per_kv_head(crs, cuda_dev):
    """G = 1 with rank 4 on the generic scorer (a tile of 32 blocks per CTA)."""
    case = workloads.block_decode_case(n_seq=2, T=32 * 200, n_kv_heads=4, n_q_heads=4, seed=15,
                                       device=cuda_dev)
    p = case["params"]
    L, r = p["L"], p["rank"]
    mu, xi = crs.block_describe(case["K"], L, r)
    tok, cnt = crs.block_select(case["Q"], mu, xi, p["T"], L, 12, 64)
    torch.cuda.synchronize()
    o_tok, o_cnt, o_blk, o_bs = oracle.block_select(_np(case["Q"]), mu.double().cpu().numpy(),
                                                    xi.double().cpu().numpy(), p["T"], L, 12, 64)
    _check_select(tok.cpu().numpy(), cnt.cpu().numpy(), o_tok, o_cnt, o_blk, o_bs, L, p["T"], 64, 12, "G1")


def _pad96(x):
    out = np.zeros(x.shape[:-1] + (96,), dtype=np.float32)
    out[..., : x.shape[-1]] = x
    return out


def test_quantize_ss_matches_oracle_bit_exact(crs, cuda_dev):
    """The deployed descriptor's codes ([P5] "量化" on the subspace eigenvectors): the
    codes and scales of each s = 85 vector equal the oracle's for the same vector padded
    with zeros to the 96 stored dims (zeros change neither the scale nor any code);
    the mean is bf16 round-to-nearest-even."""
    case = workloads.block_decode_case(n_seq=2, T=32 * 41, seed=44, device=cuda_dev)
    p = case["params"]
    U = workloads.query_subspace(128, 85, device=cuda_dev)
    mu, xi = crs.block_describe_ss(case["K"], p["L"], p["rank"], U)
    mu16, xi4, xs = crs.block_quantize_ss(mu, xi, p["T"], p["L"])
    torch.cuda.synchronize()
    o_codes, o_scale = oracle.fp4_quantize(_pad96(xi.cpu().numpy()))
    assert np.array_equal(xi4.cpu().numpy(), o_codes)
    assert np.array_equal(xs.cpu().numpy(), o_scale)
    assert torch.equal(mu16.cpu(), mu.cpu().to(torch.bfloat16))


def _select_fp4_ss_and_check(crs, case, U, top, win, seqs=None, what=""):
    p = case["params"]
    T, L, r = p["T"], p["L"], p["rank"]
    sd = U.shape[1]
    mu, xi = crs.block_describe_ss(case["K"], L, r, U)
    mu16, xi4, xs = crs.block_quantize_ss(mu, xi, T, L)
    tok, cnt = crs.block_select_fp4_ss(case["Q"], U, mu16, xi4, xs, T, L, top, win)
    torch.cuda.synchronize()
    assert crs.get_device_error() == 0
    seqs = list(range(p["n_seq"])) if seqs is None else seqs
    omu = _np(mu16)[seqs]
    oxi = oracle.fp4_dequantize(xi4.cpu().numpy()[seqs], xs.cpu().numpy()[seqs])[..., :sd]
    o_tok, o_cnt, o_blk, o_bs = oracle.block_select_ss(_np(case["Q"])[seqs], U.double().cpu().numpy(), omu, oxi,
                                                       T, L, top, win)
    _check_select(tok.cpu().numpy()[seqs], cnt.cpu().numpy()[seqs], o_tok, o_cnt, o_blk, o_bs, L, T, win, top,
                  what)


@pytest.mark.parametrize("n_q,n_kv,T,top,win,sd", [(32, 4, 4096, 16, 256, 85), (16, 4, 32 * 300 + 5, 20, 64, 48),
                                                   (4, 4, 32 * 90, 9, 100, 96), (8, 8, 32 * 129, 7, 0, 85)])
def test_select_fp4_ss_matches_oracle(crs, cuda_dev, n_q, n_kv, T, top, win, sd):
    """The deployed descriptor scored on the tensor cores equals the oracle's subspace
    selection over the same dequantised descriptors (set rule at the cutoff)."""
    case = workloads.block_decode_case(n_seq=3, T=T, n_kv_heads=n_kv, n_q_heads=n_q, seed=T + sd + 1,
                                       device=cuda_dev)
    U = workloads.query_subspace(128, sd, seed=sd, device=cuda_dev)
    _select_fp4_ss_and_check(crs, case, U, top, win, what=f"fp4-ss{sd}-G{n_q // n_kv}")


def test_select_fp4_ss_full_config_sampled(crs, cuda_dev):
    """The block-sparse decode workload (32 sequences, T = 32768, 32 query heads over 4
    KV heads) on the deployed descriptor (s = 85, r = 4, FP4): 6 sequences checked."""
    case = workloads.block_decode_case(device=cuda_dev)
    U = workloads.query_subspace(128, 85, device=cuda_dev)
    p = case["params"]
    _select_fp4_ss_and_check(crs, case, U, p["top_blocks"], p["window"], seqs=[0, 5, 11, 17, 26, 31],
                             what="fp4-ss85-full")


def test_select_fp4_ss_rejects_wide_groups(crs, cuda_dev):
    """More than 8 query heads per KV head leave no room for the split query columns."""
    case = workloads.block_decode_case(n_seq=1, T=32 * 64, n_kv_heads=2, n_q_heads=32, seed=3, device=cuda_dev)
    p = case["params"]
    U = workloads.query_subspace(128, 85, device=cuda_dev)
    mu, xi = crs.block_describe_ss(case["K"], p["L"], p["rank"], U)
    mu16, xi4, xs = crs.block_quantize_ss(mu, xi, p["T"], p["L"])
    with pytest.raises(crs.CrsError):
        crs.block_select_fp4_ss(case["Q"], U, mu16, xi4, xs, p["T"], p["L"], 8, 64)

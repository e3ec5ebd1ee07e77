"""GPU parity: LSH routing (bit-exact) and LSH attention (float tolerance) vs the oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

# |gpu - oracle| <= TOL * max(1, |oracle|): 1e-5 for fp32 inputs, 2e-3 for bf16
# inputs with fp32 accumulation (the tolerances the workloads state).
TOL = {"f32": 1e-5, "bf16": 2e-3}


def _host(x):
    return x.detach().cpu()


def _route_and_check(crs, case):
    p = case["params"]
    X = case["QK"]
    bucket, perm, inv = crs.lsh_route(X, case["R"], p["n_buckets"], p["chunk"])
    torch.cuda.synchronize()
    Xh = _host(X).float().numpy()
    Rh = _host(case["R"]).numpy()
    ob = oracle.lsh_hash(Xh, Rh, p["n_buckets"])
    op, oi = oracle.lsh_sort(ob)
    gb, gp, gi = (_host(t).numpy() for t in (bucket, perm, inv))
    assert (gb == ob).all(), f"bucket mismatch at {np.argwhere(gb != ob)[:5]}"
    assert (gp == op).all()
    assert (gi == oi).all()
    return bucket, perm, inv, ob, op, oi


def _attn_and_check(crs, case, bucket, perm, inv, ob, op, oi, rows=None, unit=None):
    p = case["params"]
    O, lse = crs.lsh_attn(case["QK"], case["V"], bucket, perm, inv, case["valid_len"],
                          n_buckets=p["n_buckets"], chunk=p["chunk"], causal=p["causal"],
                          no_self=p["no_self"], key_norm=p["key_norm"], scale=p["scale"],
                          lse=torch.empty(bucket.shape[0], bucket.shape[1], bucket.shape[3],
                                          device=bucket.device))
    torch.cuda.synchronize()
    assert crs.get_device_error() == 0
    Qh = _host(case["QK"]).double().numpy()
    Vh = _host(case["V"]).double().numpy()
    vl = _host(case["valid_len"]).numpy()
    oO, olse, ocnt = oracle.lsh_attn(Qh, Vh, ob, op, oi, vl, p["chunk"], p["causal"],
                                     p["no_self"], p["key_norm"], p["scale"], rows=rows)
    gO = _host(O).double().numpy()
    gl = _host(lse).double().numpy()
    if rows is not None:
        gO = gO[:, :, rows]
        gl = gl[:, :, rows]
    tol = TOL[p["dtype"]]
    # `unit`: per (b, h) scale of V (the output is linear in V, so a head whose V is
    # multiplied by 2^k is compared in units of 2^k)
    u = 1.0 if unit is None else np.asarray(unit, dtype=np.float64)[:, :, None, None]
    err = np.abs(gO - oO) / np.maximum(u, np.abs(oO))
    assert err.max() <= tol, f"max rel err {err.max():.3e} > {tol}"
    fin = np.isfinite(olse)
    assert (np.isfinite(gl) == fin).all()
    assert np.abs(gl[fin] - olse[fin]).max() <= tol * max(1.0, np.abs(olse[fin]).max())
    return ocnt


def test_lsh_fp32_full_config(crs, cuda_dev):
    """n=1024 fp32, one round, b=16, m=64, causal, no self (the fp32 LSH workload)."""
    case = workloads.lsh_fp32_case(device=cuda_dev)
    r = _route_and_check(crs, case)
    cnt = _attn_and_check(crs, case, *r)
    assert (cnt[0, 0, 0] == 0)  # position 0 has no legal key (causal + no self)


@pytest.mark.parametrize("n,chunk,rounds,nb,vl_frac", [
    (1000, 64, 2, 16, 0.05),    # ragged last chunk, padding
    (2048, 128, 4, 64, 0.05),   # the bf16 workload's shape per head, 4 rounds
    (77, 128, 3, 8, 0.0),       # n < chunk: one chunk, no previous
    (333, 32, 8, 4, 0.3),       # many rounds, heavy duplication
])
def test_lsh_bf16_small(crs, cuda_dev, n, chunk, rounds, nb, vl_frac):
    case = workloads.lsh_clustered_case(B=2, H=2, n=n, n_buckets=nb, n_rounds=rounds, chunk=chunk,
                                        n_centres=16, pad_frac=vl_frac, seed=n, device=cuda_dev)
    r = _route_and_check(crs, case)
    _attn_and_check(crs, case, *r)


@pytest.mark.parametrize("n,rounds,nb,causal,no_self,key_norm,vl_frac", [
    (1000, 2, 16, 1, 0, 1, 0.05),   # ragged last chunk (n % 128 != 0)
    (1280, 8, 4, 1, 1, 1, 0.2),     # 8 rounds: dedup against 7 earlier rounds
    (640, 3, 8, 0, 0, 0, 0.0),      # no causal mask, raw keys
    (129, 1, 2, 1, 1, 1, 0.0),      # two chunks, the second of one slot
    (2200, 4, 16, 1, 0, 1, 0.1),    # 18 chunks: work units of 8, 8 and 2 chunks in the ring kernel
    (3000, 4, 32, 0, 1, 1, 0.0),    # no causal mask, self excluded, 24 chunks
])
def test_lsh_bf16_tensor_core_path(crs, cuda_dev, n, rounds, nb, causal, no_self, key_norm, vl_frac):
    """bf16, d = 64, chunk = 128 runs on the tcgen05 kernel."""
    case = workloads.lsh_clustered_case(B=1, H=3, n=n, n_buckets=nb, n_rounds=rounds, chunk=128,
                                        n_centres=8, pad_frac=vl_frac, causal=causal,
                                        no_self=no_self, seed=n + rounds, device=cuda_dev)
    case["params"]["key_norm"] = key_norm
    crs.profile_collect()
    r = _route_and_check(crs, case)
    _attn_and_check(crs, case, *r)
    prof = crs.profile_collect()
    # normalised keys and at most four rounds: the persistent kernel; otherwise the per-item one
    assert ("lsh_chunk_attn_ring" if key_norm and rounds <= 4 else "lsh_chunk_attn_tc") in prof


@pytest.mark.parametrize("variant", ["v_large_head", "v_large_one", "bound_mid", "bound_two_pass", "bound_big"])
def test_lsh_bf16_tc_precision_paths(crs, cuda_dev, variant):
    """The tensor-core kernel's P formats: fp16 P (bounds <= 14 and V below 2^16 in
    magnitude), the bf16 value + residual single pass (V not fp16-representable, or a row
    bound in (14, 48]) and the two-pass path (bound > 48).  Each CTA picks its path alone:
    one large V entry moves only the CTAs whose window holds it.  Rows with a bound up to
    63 sum the rounds with a fixed shift; larger bounds keep the per-round form."""
    case = workloads.lsh_clustered_case(B=1, H=2, n=1024, n_buckets=16, n_rounds=3, chunk=128,
                                        n_centres=8, pad_frac=0.05, seed=77, device=cuda_dev)
    V = case["V"].float()
    unit = np.ones((1, 2))
    if variant == "v_large_head":        # exact scaling: bf16(2^17 v) = 2^17 bf16(v)
        V[0, 1] *= 2.0 ** 17
        unit[0, 1] = 2.0 ** 17
    elif variant == "v_large_one":
        V[0, 0, 500, 3] = 1.0e6
    elif variant == "bound_mid":          # |q| ~ 1.3: bound ~ 18.5 (log2 units)
        case["params"]["scale"] = 10.0
    elif variant == "bound_two_pass":     # bound ~ 55: two passes, rows around 63 take either
        case["params"]["scale"] = 29.0    # the fixed-shift sums or the per-round form
    else:                                 # bound ~ 370
        case["params"]["scale"] = 200.0
    case["V"] = V.to(torch.bfloat16)
    r = _route_and_check(crs, case)
    _attn_and_check(crs, case, *r, unit=unit)


def test_lsh_fp32_variants(crs, cuda_dev):
    """fp32, causal off / self allowed / raw keys."""
    case = workloads.lsh_fp32_case(n=300, n_rounds=3, chunk=16, causal=0, no_self=0, seed=9,
                                   device=cuda_dev)
    case["params"]["key_norm"] = 0
    r = _route_and_check(crs, case)
    _attn_and_check(crs, case, *r)


def test_lsh_bf16_full_config_sampled(crs, cuda_dev):
    """The full bf16 multi-round workload (B=2, H=8, n=16384, 4 rounds); routing is
    compared everywhere, attention on 96 sampled query rows per (b, h)."""
    case = workloads.lsh_clustered_case(device=cuda_dev)
    r = _route_and_check(crs, case)
    n = case["params"]["n"]
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([rng.choice(n, 90, replace=False),
                                     [0, 1, 127, 128, n - 1, int(case["valid_len"][0]) - 1]]))
    _attn_and_check(crs, case, *r, rows=rows.astype(np.int32))


def test_lsh_rejects_bad_args(crs, cuda_dev):
    case = workloads.lsh_fp32_case(n=64, device=cuda_dev)
    with pytest.raises(ValueError):
        crs.lsh_route(case["QK"], case["R"][:, :, :, :4], 16)   # R shape mismatch
    X = case["QK"][..., :7].contiguous()                        # d not a multiple of 8
    R = torch.zeros(1, 1, 7, 8, device=cuda_dev)
    with pytest.raises(crs.CrsError):
        crs.lsh_route(X, R, 16)


@pytest.mark.parametrize("n,chunk,rounds,nb,causal,no_self,vl_frac", [
    (700, 64, 3, 16, 1, 0, 0.9),
    (333, 128, 1, 8, 1, 1, 1.0),      # n < 3 chunks, ragged last chunk
    (1024, 32, 8, 64, 0, 1, 0.95),    # 8 rounds, not causal
])
def test_lsh_candidates_csr_matches_oracle(crs, cuda_dev, n, chunk, rounds, nb, causal, no_self, vl_frac):
    """The CSR export of U(i) (PaperTrace 2.1.1 §4 index tensors) equals the oracle's
    candidate set for every row, bit for bit."""
    case = workloads.lsh_clustered_case(B=2, H=2, n=n, n_rounds=rounds, n_buckets=nb, chunk=chunk,
                                        pad_frac=1.0 - vl_frac, seed=n + rounds, device=cuda_dev)
    bucket, perm, inv, ob, op, oi = _route_and_check(crs, case)
    row_ptr, col = crs.lsh_candidates_csr(bucket, perm, inv, case["valid_len"], chunk=chunk,
                                          causal=causal, no_self=no_self)
    torch.cuda.synchronize()
    assert crs.get_device_error() == 0
    rp, cl = row_ptr.cpu().numpy(), col.cpu().numpy()
    vl = case["valid_len"].cpu().numpy()
    B, H = 2, 2
    assert rp[0] == 0 and (np.diff(rp) >= 0).all()
    for b in range(B):
        for h in range(H):
            for i in range(n):
                row = (b * H + h) * n + i
                want = oracle.lsh_candidates(ob[b, h], op[b, h], oi[b, h], i, chunk, causal, no_self,
                                             int(vl[b]))
                got = cl[rp[row]:rp[row + 1]]
                assert np.array_equal(got, want), f"(b={b}, h={h}, i={i}): {got[:8]} vs {want[:8]}"


def test_lsh_hash_tensor_core_near_ties(crs, cuda_dev):
    """bf16, d = 64, b = 64: the tensor-core hash decides a bucket only when the winner
    leads by more than its error bound, else recomputes the fp32 chain.  Exact ties
    (duplicated rotation columns: the first maximum wins), near ties (columns 1e-6
    apart), zero rows and rows of mixed magnitude must all give the oracle's ids."""
    case = workloads.lsh_clustered_case(B=2, H=2, n=3000, n_rounds=4, n_buckets=64, chunk=128,
                                        seed=5, device=cuda_dev)
    R = case["R"].clone()
    R[:, :, :, 5] = R[:, :, :, 3]
    R[:, :, :, 7] = R[:, :, :, 6] + 1e-6 * torch.randn_like(R[:, :, :, 6])
    R[:, 1, :, 20] = -R[:, 1, :, 19]
    X = case["QK"].clone()
    X[0, 0, 100:140] = 0
    X[1, 1, :50] *= 1000.0
    case["R"], case["QK"] = R, X.contiguous()
    crs.profile_collect()
    _route_and_check(crs, case)
    assert "lsh_hash" in crs.profile_collect()


def test_lsh_bf16_unaligned_inputs_take_the_cuda_core_kernel(crs, cuda_dev):
    """QK and V that do not start on a 16-byte boundary cannot feed the tensor-core
    kernels' 16-byte row reads: the call takes the CUDA-core kernel, same results."""
    case = workloads.lsh_clustered_case(B=1, H=2, n=700, n_buckets=16, n_rounds=2, chunk=128,
                                        n_centres=8, pad_frac=0.1, seed=31, device=cuda_dev)
    r = _route_and_check(crs, case)
    for k in ("QK", "V"):                      # same values, storage shifted by one element (2 bytes)
        t = case[k]
        buf = torch.empty(t.numel() + 1, dtype=t.dtype, device=t.device)
        case[k] = buf[1:].view(t.shape)
        case[k].copy_(t)
        assert case[k].data_ptr() % 16 != 0
    crs.profile_collect()
    _attn_and_check(crs, case, *r)
    prof = crs.profile_collect()
    assert "lsh_chunk_attn" in prof and "lsh_chunk_attn_ring" not in prof and "lsh_chunk_attn_tc" not in prof

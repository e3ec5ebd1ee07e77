"""The failure path of the bounded waits, driven on the GPU without a stuck barrier.

crs_debug_force_wait_timeout makes the first mbarrier wait of the tensor-core LSH
kernels give up at once, exactly as a wait that ran out does: the kernel raises
CRS_DEVERR_TIMEOUT, records (kernel, site) in the diagnostic record, drains the
tensor-core work it issued, frees its tensor memory and returns.  Nothing faults,
traps or hangs; afterwards the context must be fully usable (the same calls match
the oracle)."""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

K_LSH_HASH, K_LSH_ATTN_TC = 0, 11     # kernel ids of the diagnostic record (id + 1 is stored)


def _attn(crs, case, b, pm, ip):
    p = case["params"]
    return crs.lsh_attn(case["QK"], case["V"], b, pm, ip, case["valid_len"], n_buckets=p["n_buckets"],
                        chunk=p["chunk"], causal=p["causal"], no_self=p["no_self"], key_norm=p["key_norm"],
                        scale=p["scale"])


def test_forced_wait_timeout_is_reported_and_the_next_call_is_correct(crs, cuda_dev):
    case = workloads.lsh_clustered_case(B=1, H=2, n=1000, n_rounds=2, n_buckets=64, chunk=128, seed=13,
                                        device=cuda_dev)
    p = case["params"]
    crs.get_device_error()
    crs.get_device_diag()
    b, pm, ip = crs.lsh_route(case["QK"], case["R"], p["n_buckets"], p["chunk"])
    assert crs.get_device_error() == 0

    # chunk attention: the wait for S = Q K^T gives up in every CTA
    try:
        crs.debug_force_wait_timeout(True)
        _attn(crs, case, b, pm, ip)
        flags = crs.get_device_error()
        diag = crs.get_device_diag()
    finally:
        crs.debug_force_wait_timeout(False)
    assert flags & crs.DEVERR_TIMEOUT
    assert diag[0] == K_LSH_ATTN_TC + 1 and diag[1] == 1

    # routing: the hash's first wait gives up (its bucket ids are not written)
    bad = tuple(torch.full_like(b, -1) for _ in range(3))
    try:
        crs.debug_force_wait_timeout(True)
        crs.lsh_route(case["QK"], case["R"], p["n_buckets"], p["chunk"], out=bad)
        flags = crs.get_device_error()
        diag = crs.get_device_diag()
    finally:
        crs.debug_force_wait_timeout(False)
    assert flags & crs.DEVERR_TIMEOUT
    assert diag[0] == K_LSH_HASH + 1 and diag[1] == 1

    # the same calls, switch off: bit-exact routing and attention within 2e-3 of the oracle
    b, pm, ip = crs.lsh_route(case["QK"], case["R"], p["n_buckets"], p["chunk"])
    O, _ = _attn(crs, case, b, pm, ip)
    torch.cuda.synchronize()
    assert crs.get_device_error() == 0
    assert crs.get_device_diag()[0] == 0
    Xh = case["QK"].float().cpu().numpy()
    ob = oracle.lsh_hash(Xh, case["R"].cpu().numpy(), p["n_buckets"])
    op, oi = oracle.lsh_sort(ob)
    assert (b.cpu().numpy() == ob).all() and (pm.cpu().numpy() == op).all() and (ip.cpu().numpy() == oi).all()
    oO, _, _ = oracle.lsh_attn(Xh.astype(np.float64), case["V"].double().cpu().numpy(), ob, op, oi,
                               case["valid_len"].cpu().numpy(), p["chunk"], p["causal"], p["no_self"],
                               p["key_norm"], p["scale"])
    err = np.abs(O.double().cpu().numpy() - oO) / np.maximum(1.0, np.abs(oO))
    assert err.max() <= 2e-3

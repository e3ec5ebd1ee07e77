"""The seeded input recipes: determinism, shapes, and the planted needles."""
import math

import torch

import workloads


def test_lsh_cases_deterministic_and_shaped():
    a = workloads.lsh_clustered_case(B=1, H=2, n=512, seed=3)
    b = workloads.lsh_clustered_case(B=1, H=2, n=512, seed=3)
    assert torch.equal(a["QK"].view(torch.int16), b["QK"].view(torch.int16))
    assert a["QK"].dtype == torch.bfloat16 and a["QK"].shape == (1, 2, 512, 64)
    assert a["R"].shape == (2, 4, 64, 32)
    assert int(a["valid_len"][0]) == 512 - math.floor(0.05 * 512)
    c = workloads.lsh_fp32_case(n=256)
    assert c["QK"].dtype == torch.float32 and c["R"].shape == (1, 1, 64, 8)


def test_prefill_needles_align_with_targets():
    c = workloads.indexer_prefill_case(n=2000, seed=5)
    k = c["k_idx"].float()
    q = c["q_idx"].float()
    # at least one planted key has cosine ~0.9 with some later query head
    cos = (torch.nn.functional.normalize(k, dim=-1) @
           torch.nn.functional.normalize(q.reshape(-1, 64), dim=-1).T)
    assert (cos > 0.85).sum() >= 10


def test_decode_and_block_cases_small():
    d = workloads.indexer_decode_case(n_seq=3, ctx_lo=100, ctx_hi=300, seed=1)
    assert int(d["offsets"][-1]) == int(d["ctx"].sum())
    assert d["K"].shape == (int(d["offsets"][-1]), 8, 128)
    b = workloads.block_decode_case(n_seq=2, T=256, seed=2)
    assert b["K"].shape == (2, 256, 4, 128) and b["Q"].shape == (2, 32, 128)

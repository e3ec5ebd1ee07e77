"""Input recipes for the five workloads.

Every function is deterministic for a given (seed, device): it draws from a
``torch.Generator`` seeded with ``seed`` on ``device``.  Values stored as bf16
are rounded (round-to-nearest-even) once, here; every consumer sees the same
rounded numbers.  Large caches are generated on the device in slices so the
host never holds them.

The recipes follow the workload descriptions that accompany the pages (LSH
sizes from PaperTrace 2.1.1 "哈希与聚类" §2; the k=2048 token budget from
PaperTrace 2.2 "细粒度索引" §1.1; the L=32 / D=128 / GQA shapes from the COBS
reading notes).  Where the pages give no generator (cluster structure,
planted "needle" keys, anisotropic block covariance) the recipe below is this
library's own reading.
"""
from __future__ import annotations

import math
from typing import Dict

import torch


def _generator(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(int(seed))
    return g


def _unit(x: torch.Tensor, dim: int = -1) -> torch.Tensor:
    return x / x.norm(dim=dim, keepdim=True).clamp_min(1e-30)


def _perp_unit(u: torch.Tensor, e: torch.Tensor) -> torch.Tensor:
    """Unit vector along the part of ``e`` orthogonal to the unit vector ``u`` (rows)."""
    e = e - (e * u).sum(-1, keepdim=True) * u
    return _unit(e)


# --------------------------------------------------------------------------
# LSH workloads
# --------------------------------------------------------------------------
def lsh_fp32_case(B=1, H=1, n=1024, d=64, n_buckets=16, n_rounds=1, chunk=64,
                  causal=1, no_self=1, seed=0, device="cpu") -> Dict:
    """fp32 shared-QK LSH attention: Q, V ~ N(0,1), one rotation R ~ N(0,1) of d x b/2."""
    g = _generator(seed, device)
    QK = torch.randn(B, H, n, d, generator=g, device=device, dtype=torch.float32)
    V = torch.randn(B, H, n, d, generator=g, device=device, dtype=torch.float32)
    R = torch.randn(H, n_rounds, d, n_buckets // 2, generator=g, device=device, dtype=torch.float32)
    valid_len = torch.full((B,), n, dtype=torch.int32, device=device)
    params = dict(B=B, H=H, n=n, d=d, n_buckets=n_buckets, n_rounds=n_rounds, chunk=chunk,
                  causal=causal, no_self=no_self, key_norm=1, dtype="f32",
                  scale=1.0 / math.sqrt(d))
    return dict(QK=QK, V=V, R=R, valid_len=valid_len, params=params,
                workload=f"lsh_fp32_B{B}_H{H}_n{n}_d{d}_b{n_buckets}_r{n_rounds}_m{chunk}")


def lsh_clustered_case(B=2, H=8, n=16384, d=64, n_buckets=64, n_rounds=4, chunk=128,
                       n_centres=256, noise=0.1, pad_frac=0.05, causal=1, no_self=0,
                       seed=1, device="cpu") -> Dict:
    """bf16 multi-round LSH attention on clustered shared-QK vectors.

    Per (batch, head): ``n_centres`` centres ~ N(0, I) scaled to unit norm; each
    token picks a centre uniformly; q = centre + N(0, noise^2 I).  V ~ N(0, 1).
    One independent rotation per head and round.  The last ``pad_frac`` of every
    sequence is padding: valid_len = n - floor(pad_frac * n).
    """
    g = _generator(seed, device)
    centres = _unit(torch.randn(B, H, n_centres, d, generator=g, device=device))
    pick = torch.randint(0, n_centres, (B, H, n), generator=g, device=device)
    q = torch.gather(centres, 2, pick[..., None].expand(B, H, n, d))
    q = q + noise * torch.randn(B, H, n, d, generator=g, device=device)
    V = torch.randn(B, H, n, d, generator=g, device=device)
    R = torch.randn(H, n_rounds, d, n_buckets // 2, generator=g, device=device, dtype=torch.float32)
    vl = n - int(math.floor(pad_frac * n))
    valid_len = torch.full((B,), vl, dtype=torch.int32, device=device)
    params = dict(B=B, H=H, n=n, d=d, n_buckets=n_buckets, n_rounds=n_rounds, chunk=chunk,
                  causal=causal, no_self=no_self, key_norm=1, dtype="bf16",
                  scale=1.0 / math.sqrt(d))
    return dict(QK=q.to(torch.bfloat16), V=V.to(torch.bfloat16), R=R, valid_len=valid_len,
                params=params,
                workload=f"lsh_bf16_B{B}_H{H}_n{n}_d{d}_b{n_buckets}_r{n_rounds}_m{chunk}_pad{vl}")


# --------------------------------------------------------------------------
# Indexer workloads
# --------------------------------------------------------------------------
def indexer_prefill_case(n=32768, n_q_heads=16, D=128, n_idx_heads=4, d_idx=64, topk=2048,
                         needle_frac=0.01, seed=2, device="cpu") -> Dict:
    """Causal prefill: MQA main attention (one K/V head) plus a 4-head index.

    Q ~ N(0,1) [n,Hq,D]; K, V ~ N(0,1) [n,1,D]; q_idx ~ N(0,1) [n,4,64];
    k_idx ~ N(0,1) [n,64]; w ~ N(0,1) fp32 [n,4].  Needles: floor(needle_frac*n)
    positions p drawn without replacement from [0, n-2]; each gets a target
    query t ~ U(p, n-1]; k_idx[p] keeps its norm but turns to cosine 0.9 with
    q_idx[t, h*] (h* = argmax_h w[t, h]); K[p] likewise with the mean of Q[t, :].
    """
    g = _generator(seed, device)
    Q = torch.randn(n, n_q_heads, D, generator=g, device=device)
    K = torch.randn(n, 1, D, generator=g, device=device)
    V = torch.randn(n, 1, D, generator=g, device=device)
    q_idx = torch.randn(n, n_idx_heads, d_idx, generator=g, device=device)
    k_idx = torch.randn(n, d_idx, generator=g, device=device)
    w = torch.randn(n, n_idx_heads, generator=g, device=device)
    # round the query side first: needles align with the stored (rounded) queries
    Q = Q.to(torch.bfloat16)
    q_idx = q_idx.to(torch.bfloat16)
    n_needle = int(math.floor(needle_frac * n))
    if n_needle > 0 and n >= 2:
        p = torch.randperm(n - 1, generator=g, device=device)[:n_needle]
        u = torch.rand(n_needle, generator=g, device=device, dtype=torch.float64)
        t = p + 1 + torch.floor(u * (n - 1 - p).to(torch.float64)).to(p.dtype)
        t = torch.minimum(t, torch.full_like(t, n - 1))
        hstar = w[t].argmax(dim=1)
        qh = _unit(q_idx[t, hstar].float())
        e = _perp_unit(qh, torch.randn(n_needle, d_idx, generator=g, device=device))
        kn = k_idx[p].norm(dim=-1, keepdim=True)
        k_idx[p] = kn * (0.9 * qh + math.sqrt(0.19) * e)
        qm = _unit(Q[t].float().mean(dim=1))
        e2 = _perp_unit(qm, torch.randn(n_needle, D, generator=g, device=device))
        kn2 = K[p, 0].norm(dim=-1, keepdim=True)
        K[p, 0] = kn2 * (0.9 * qm + math.sqrt(0.19) * e2)
    params = dict(n=n, n_q_heads=n_q_heads, n_kv_heads=1, D=D, n_idx_heads=n_idx_heads,
                  d_idx=d_idx, topk=topk, scale=1.0 / math.sqrt(D))
    return dict(Q=Q, K=K.to(torch.bfloat16), V=V.to(torch.bfloat16), q_idx=q_idx,
                k_idx=k_idx.to(torch.bfloat16), w=w.float().contiguous(), params=params,
                workload=f"indexer_prefill_n{n}_Hq{n_q_heads}_D{D}_Hi{n_idx_heads}_dI{d_idx}_k{topk}")


def indexer_decode_case(n_seq=64, ctx_lo=8192, ctx_hi=131072, n_idx_heads=4, d_idx=64,
                        n_q_heads=32, n_kv_heads=8, D=128, topk=2048, needle_frac=0.01,
                        seed=3, device="cpu", slice_tokens=1 << 20) -> Dict:
    """One decode step for ``n_seq`` sequences of ragged context.

    ctx ~ U{ctx_lo..ctx_hi}; caches are packed by sequence with int64 offsets.
    The current token is already in the cache: its query sees positions
    [0, ctx).  Needles: floor(needle_frac*ctx) positions per sequence (without
    replacement) turned to cosine 0.9 with that sequence's query (index key with
    q_idx[h*], main key of KV head h with the mean of its query-head group).
    """
    g = _generator(seed, device)
    ctx = torch.randint(ctx_lo, ctx_hi + 1, (n_seq,), generator=g, device=device)
    offsets = torch.zeros(n_seq + 1, dtype=torch.int64, device=device)
    offsets[1:] = torch.cumsum(ctx, 0)
    total = int(offsets[-1].item())
    q_idx = torch.randn(n_seq, n_idx_heads, d_idx, generator=g, device=device).to(torch.bfloat16)
    w = torch.randn(n_seq, n_idx_heads, generator=g, device=device).float()
    Q = torch.randn(n_seq, n_q_heads, D, generator=g, device=device).to(torch.bfloat16)
    k_idx = torch.empty(total, d_idx, dtype=torch.bfloat16, device=device)
    K = torch.empty(total, n_kv_heads, D, dtype=torch.bfloat16, device=device)
    V = torch.empty(total, n_kv_heads, D, dtype=torch.bfloat16, device=device)
    for s0 in range(0, total, slice_tokens):
        s1 = min(total, s0 + slice_tokens)
        k_idx[s0:s1] = torch.randn(s1 - s0, d_idx, generator=g, device=device).to(torch.bfloat16)
        K[s0:s1] = torch.randn(s1 - s0, n_kv_heads, D, generator=g, device=device).to(torch.bfloat16)
        V[s0:s1] = torch.randn(s1 - s0, n_kv_heads, D, generator=g, device=device).to(torch.bfloat16)
    G = n_q_heads // n_kv_heads
    hstar = w.argmax(dim=1)
    for s in range(n_seq):
        c = int(ctx[s].item())
        P = int(math.floor(needle_frac * c))
        if P == 0:
            continue
        base = int(offsets[s].item())
        p = base + torch.randperm(c, generator=g, device=device)[:P]
        qh = _unit(q_idx[s, hstar[s]].float())[None, :].expand(P, d_idx)
        e = _perp_unit(qh, torch.randn(P, d_idx, generator=g, device=device))
        kn = k_idx[p].float().norm(dim=-1, keepdim=True)
        k_idx[p] = (kn * (0.9 * qh + math.sqrt(0.19) * e)).to(torch.bfloat16)
        qm = _unit(Q[s].float().view(n_kv_heads, G, D).mean(dim=1))  # [Hkv, D]
        qm = qm[None].expand(P, n_kv_heads, D)
        e2 = _perp_unit(qm, torch.randn(P, n_kv_heads, D, generator=g, device=device))
        kn2 = K[p].float().norm(dim=-1, keepdim=True)
        K[p] = (kn2 * (0.9 * qm + math.sqrt(0.19) * e2)).to(torch.bfloat16)
    params = dict(n_seq=n_seq, n_idx_heads=n_idx_heads, d_idx=d_idx, n_q_heads=n_q_heads,
                  n_kv_heads=n_kv_heads, D=D, topk=topk, scale=1.0 / math.sqrt(D))
    return dict(ctx=ctx.to(torch.int32), offsets=offsets, q_idx=q_idx, w=w, Q=Q, k_idx=k_idx,
                K=K, V=V, params=params,
                workload=(f"indexer_decode_seq{n_seq}_ctx{ctx_lo}-{ctx_hi}_Hq{n_q_heads}"
                          f"_Hkv{n_kv_heads}_D{D}_k{topk}"))


# --------------------------------------------------------------------------
# Block-mass selector workload
# --------------------------------------------------------------------------
def block_decode_case(n_seq=32, T=32768, n_kv_heads=4, n_q_heads=32, D=128, L=32,
                      top_blocks=64, window=512, rank=4, n_centres=64, seed=4,
                      device="cpu") -> Dict:
    """One decode step over a clustered, anisotropic key cache.

    Per (sequence, KV head): ``n_centres`` centres ~ N(0, 0.5 I); each block of
    L keys picks a centre c and a mixing matrix A_b = N(0,1)^{D x 8} diag(sigma)/sqrt(8)
    with sigma_j ~ U(0.2, 1.5); key r = c + A_b eps_r + 0.3 eta_r, eps ~ N(0, I_8),
    eta ~ N(0, I_D).  V ~ N(0,1), Q ~ N(0,1).  Layout K, V: [n_seq, T, Hkv, D] bf16.
    """
    g = _generator(seed, device)
    nb_all = (T + L - 1) // L
    K = torch.empty(n_seq, T, n_kv_heads, D, dtype=torch.bfloat16, device=device)
    for s in range(n_seq):
        for h in range(n_kv_heads):
            cen = math.sqrt(0.5) * torch.randn(n_centres, D, generator=g, device=device)
            pick = torch.randint(0, n_centres, (nb_all,), generator=g, device=device)
            sigma = 0.2 + 1.3 * torch.rand(nb_all, 8, generator=g, device=device)
            A = torch.randn(nb_all, D, 8, generator=g, device=device) * sigma[:, None, :] / math.sqrt(8.0)
            eps = torch.randn(nb_all, L, 8, generator=g, device=device)
            eta = torch.randn(nb_all, L, D, generator=g, device=device)
            k = cen[pick][:, None, :] + torch.einsum("bdk,blk->bld", A, eps) + 0.3 * eta
            K[s, :, h, :] = k.reshape(nb_all * L, D)[:T].to(torch.bfloat16)
    V = torch.randn(n_seq, T, n_kv_heads, D, generator=g, device=device).to(torch.bfloat16)
    Q = torch.randn(n_seq, n_q_heads, D, generator=g, device=device).to(torch.bfloat16)
    params = dict(n_seq=n_seq, T=T, n_kv_heads=n_kv_heads, n_q_heads=n_q_heads, D=D, L=L,
                  top_blocks=top_blocks, window=window, rank=rank, scale=1.0 / math.sqrt(D))
    return dict(K=K, V=V, Q=Q, params=params,
                workload=(f"block_decode_seq{n_seq}_T{T}_Hq{n_q_heads}_Hkv{n_kv_heads}_D{D}"
                          f"_L{L}_top{top_blocks}_win{window}_r{rank}"))


CONFIGS = {
    1: lambda device="cpu": lsh_fp32_case(seed=0, device=device),
    2: lambda device="cpu": lsh_clustered_case(seed=1, device=device),
    3: lambda device="cpu": indexer_prefill_case(seed=2, device=device),
    4: lambda device="cpu": indexer_decode_case(seed=3, device=device),
    5: lambda device="cpu": block_decode_case(seed=4, device=device),
}


def query_subspace(D=128, s=85, seed=21, device="cpu") -> "torch.Tensor":
    """An orthonormal basis U [D, s] (fp32) of a query subspace.  The synthetic
    queries are isotropic N(0, I), so no subspace captures more of their second
    moment than another: U is the Q factor of a seeded Gaussian D x s matrix."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    A = torch.randn(D, s, generator=g, dtype=torch.float64)
    Uq, _ = torch.linalg.qr(A)
    return Uq.to(torch.float32).contiguous().to(device)


def make_config(i: int, device="cpu") -> Dict:
    """Full-size workload ``i`` (1..5); seed = i - 1."""
    return CONFIGS[int(i)](device=device)

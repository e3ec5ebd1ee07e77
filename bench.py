"""Throughput of content-routed sparse attention on B200 (one JSON line).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl product|reference]
                  [--workload lsh|lsh_fp32|lsh_decode|route|prefill|prefill_hisa|decode|decode_hisa|block|block_fp4|
                              block_ss|block_fp4_ss|block_quest|block_meanpool] [--no-extras]

A step is one pass of the hot path over one batch of the workload:
  lsh      (headline) multi-round bf16 LSH attention, B=2, H=8, n=16384, d=64,
           b=64 buckets, 4 rounds, chunk 128, causal, last 5% padding:
           hash -> sort -> chunked attention -> round merge.  Metric: tokens/s.
  lsh_fp32 fp32 LSH attention, n=1024, b=16, 1 round, chunk 64.
  route    routing (k-means) attention with quotas, B=2, H=8, n=16384, C=128, m=128.
  lsh_decode  LSH attention in decode: 64 rows x 8 heads, 16384-token prompts in bucket
           lists (64 buckets x 4 rounds) and paged K/V; a step appends one token per row
           and attends with it.
  prefill  indexer prefill n=32768 (top-2048) + MQA gather attention (16 heads).
  prefill_hisa  the same with the hierarchical indexer's prefill form (64-key blocks, 128 kept).
  decode   indexer decode, 64 sequences of ragged context + GQA gather attention.
  decode_hisa  the same with the hierarchical indexer (64-key blocks, 128 kept).
  block    block-mass decode: block select (top-64 + 512 window) + GQA attention;
           the descriptor build is timed separately (it runs once per filled block).
  block_fp4 the same on bf16 means + FP4 (E2M1) eigenvectors (528 B per block).
  block_ss  the same on descriptors in a query subspace of 85 dims (fp32).
  block_fp4_ss  the deployed descriptor: bf16 means + FP4 eigenvectors in the 85-dim query
           subspace, scored on the tensor cores.
  block_quest / block_meanpool  the same step with the baseline selectors (Quest boxes;
           block means alone).
Timing: W untimed warm-up steps, then K steps each bracketed by CUDA events on
the launching stream; a 256 MiB buffer (2x L2) is written between steps,
outside the events.  Multi-GPU: one process per GPU (torchrun), each rank runs
its own batch (weak scaling); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "sparse-attn prefill tokens/s & decode steps/s on 1 B200; % of HBM/TC roofline"
FP32_ALU_TFLOPS_NOMINAL = 148 * 128 * 2 * 1.965e9 / 1e12   # SMs x FP32 lanes x 2 x max clock


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def l2_gather_gbs(crs, dev, reps=5):
    """The L2 read ceiling of 512-byte row gathers on this GPU, measured now: random rows
    of a 16 MiB table (inside L2), one row per warp load, through crs_probe_l2_gather;
    CUDA events around `reps` launches of 2^21 rows each, after two warm-up launches."""
    table = torch.zeros(32768 * 128, dtype=torch.float32, device=dev)          # 32768 rows x 512 B
    gen = torch.Generator(device=dev).manual_seed(7)
    idx = torch.randint(0, 32768, (1 << 21,), dtype=torch.int32, device=dev, generator=gen)
    sink = torch.zeros(4, dtype=torch.int32, device=dev)
    for _ in range(2):
        crs.probe_l2_gather(table, idx, sink)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        crs.probe_l2_gather(table, idx, sink)
    b.record()
    torch.cuda.synchronize()
    return 512.0 * idx.numel() * reps / (a.elapsed_time(b) * 1e6)


# ------------------------------------------------------------------ workloads --
class Workload:
    name = ""
    unit = "tokens/s"
    units_per_step = 1.0
    dtype = "bf16"

    def step(self):
        raise NotImplementedError

    def e2e_step(self):
        raise NotImplementedError

    def roofline_spec(self):
        """{kernel: (bound, amount per launch, unit)} for kernels we can account."""
        return {}


class LshWorkload(Workload):
    def __init__(self, crs, dev, fp32=False):
        import workloads
        self.crs = crs
        case = workloads.lsh_fp32_case(device=dev) if fp32 else workloads.lsh_clustered_case(device=dev)
        self.case = case
        p = case["params"]
        self.p = p
        self.name = case["workload"]
        self.dtype = "f32" if fp32 else "bf16"
        self.units_per_step = p["B"] * p["n"]
        B, H, n, d, R = p["B"], p["H"], p["n"], p["d"], p["n_rounds"]
        self.route_out = tuple(torch.empty((B, H, R, n), dtype=torch.int32, device=dev) for _ in range(3))
        self.O = torch.empty(case["QK"].shape, dtype=torch.float32, device=dev)
        a = crs.LshAttnParams(crs.lsh_params(case["QK"], p["n_buckets"], R, p["chunk"]),
                              p["causal"], p["no_self"], p["key_norm"], p["scale"])
        import ctypes
        ws = int(crs.lib().crs_lsh_attn_workspace_size(ctypes.byref(a)))
        self.ws = torch.empty(ws, dtype=torch.uint8, device=dev)
        # host copies for the end-to-end pass
        self.h_in = {k: case[k].cpu().pin_memory() for k in ("QK", "V", "R", "valid_len")}
        self.h_out = torch.empty(self.O.shape, dtype=self.O.dtype).pin_memory()
        self.d_in = {k: torch.empty_like(case[k]) for k in self.h_in}
        self.h2d = sum(t.numel() * t.element_size() for t in self.h_in.values())
        self.d2h = self.h_out.numel() * self.h_out.element_size()

    def _run(self, src):
        p = self.p
        b, pm, ip = self.crs.lsh_route(src["QK"], src["R"], p["n_buckets"], p["chunk"],
                                       out=self.route_out)
        self.crs.lsh_attn(src["QK"], src["V"], b, pm, ip, src["valid_len"],
                          n_buckets=p["n_buckets"], chunk=p["chunk"], causal=p["causal"],
                          no_self=p["no_self"], key_norm=p["key_norm"], scale=p["scale"],
                          out=self.O, workspace=self.ws)

    def step(self):
        self._run(self.case)

    def e2e_step(self):
        for k, h in self.h_in.items():
            self.d_in[k].copy_(h, non_blocking=True)
        self._run(self.d_in)
        self.h_out.copy_(self.O, non_blocking=True)

    def step_bytes(self):
        """Algorithmic bytes of a whole step: per (batch, head) Q and V once per round,
        O once and the routing integers of every round."""
        p = self.p
        B, H, n, d, R = p["B"], p["H"], p["n"], p["d"], p["n_rounds"]
        esz = 2 if self.dtype == "bf16" else 4
        return B * H * (R * n * d * esz * 2 + n * d * esz + R * n * 4 * 3)

    def cpu_sample(self, frac):
        p = self.p
        segs = max(1, int(round(p["B"] * p["H"] * frac)))
        return cpu_sample_lsh(self.case, segs)

    def roofline_spec(self):
        p = self.p
        B, H, n, d, R, m = p["B"], p["H"], p["n"], p["d"], p["n_rounds"], p["chunk"]
        rect_flops = B * H * R * n * (2 * m) * d * 4          # QK^T and P.V over own+previous chunk
        esz = 2 if self.dtype == "bf16" else 4
        # algorithmic bytes of the attention: Q (= K) and V read once per round, and the
        # three int32 routing arrays (bucket, perm, inv_perm) of every round
        attn_bytes = B * H * R * n * d * esz * 2 + B * H * R * n * 4 * 3
        return {
            "lsh_chunk_attn": [("alu", rect_flops / 1e12, "TFLOP/s"),
                               ("hbm", attn_bytes / 1e9, "GB/s")],
            "lsh_chunk_attn_tc": [("tensor", rect_flops / 1e12, "TFLOP/s"),
                                  ("hbm", attn_bytes / 1e9, "GB/s")],
            # the persistent kernel; the per-item kernel then runs over the items it left
            # (normally none) and its time is counted with it
            "lsh_chunk_attn_ring": [("tensor", rect_flops / 1e12, "TFLOP/s"),
                                    ("hbm", attn_bytes / 1e9, "GB/s")],
            "_with": {"lsh_chunk_attn_ring": ["lsh_chunk_attn_tc"]},
            "lsh_hash": [("alu", B * H * R * n * d * (p["n_buckets"] // 2) * 2 / 1e12, "TFLOP/s")],
        }


class RouteWorkload(Workload):
    """Routing (k-means) attention with quota execution: B = 2, H = 8, n = 16384, d = 64,
    C = 128 frozen unit centres, quota m = 128 (C m = n), causal.  A step = routing
    scores -> quotas -> per-centre attention -> merge.  Metric: tokens/s."""

    def __init__(self, crs, dev):
        self.crs = crs
        B, H, n, d, C, m = 2, 8, 16384, 64, 128, 128
        self.p = dict(B=B, H=H, n=n, d=d, C=C, m=m, causal=1)
        self.name = f"route_B{B}_H{H}_n{n}_d{d}_C{C}_m{m}_causal"
        self.units_per_step = B * n
        g = torch.Generator(device="cpu").manual_seed(81)
        self.Q = torch.randn(B, H, n, d, generator=g).to(torch.bfloat16).to(dev)
        self.K = torch.randn(B, H, n, d, generator=g).to(torch.bfloat16).to(dev)
        self.V = torch.randn(B, H, n, d, generator=g).to(torch.bfloat16).to(dev)
        M = torch.randn(H, C, d, generator=g)
        self.M = (M / M.norm(dim=-1, keepdim=True)).to(dev)
        self.JQ = torch.empty((B, H, C, m), dtype=torch.int32, device=dev)
        self.JK = torch.empty_like(self.JQ)
        self.O = torch.empty((B, H, n, d), dtype=torch.float32, device=dev)
        self.lse = torch.empty((B, H, n), dtype=torch.float32, device=dev)
        self.cnt = torch.empty((B, H, n), dtype=torch.int32, device=dev)
        import ctypes
        rp = crs.RouteParams(B, H, n, d, C, m, 1, 0, 1.0 / math.sqrt(d))
        self.ws = torch.empty(int(crs.lib().crs_route_attn_workspace_size(ctypes.byref(rp))), dtype=torch.uint8,
                              device=dev)
        self.h_in = {k: getattr(self, k).cpu().pin_memory() for k in ("Q", "K", "V")}
        self.d_in = {k: torch.empty_like(getattr(self, k)) for k in self.h_in}
        self.h_out = torch.empty(self.O.shape, dtype=self.O.dtype).pin_memory()
        self.h2d = sum(t.numel() * t.element_size() for t in self.h_in.values())
        self.d2h = self.h_out.numel() * self.h_out.element_size()

    def _run(self, Q, K, V):
        self.crs.route_attn(Q, K, V, self.M, self.p["m"], causal=True, out=self.O, lse=self.lse, count=self.cnt,
                            JQ=self.JQ, JK=self.JK, workspace=self.ws)

    def step(self):
        self._run(self.Q, self.K, self.V)

    def e2e_step(self):
        for k, h in self.h_in.items():
            self.d_in[k].copy_(h, non_blocking=True)
        self._run(self.d_in["Q"], self.d_in["K"], self.d_in["V"])
        self.h_out.copy_(self.O, non_blocking=True)

    def roofline_spec(self):
        p = self.p
        BH = p["B"] * p["H"]
        # scores n C d per role (ALU) vs the bytes: Q, K read for the scores, Q, K, V gathered
        # per centre, O written
        flops = BH * 2 * p["n"] * p["C"] * p["d"] * 2 + BH * p["C"] * p["m"] * p["m"] * p["d"] * 4
        byts = BH * (2 * p["n"] * p["d"] * 2 + p["C"] * p["m"] * p["d"] * 2 * 3 + p["n"] * p["d"] * 4)
        return {"route": [("alu", flops / 1e12, "TFLOP/s"), ("hbm", byts / 1e9, "GB/s")]}


class LshDecodeWorkload(Workload):
    """LSH attention in decode: 64 rows x 8 heads (d = 64) whose 16384-token prompts were
    hashed into 64 buckets x 4 rounds (bucket lists, paged K/V behind a shuffled block
    table); a step appends one token per row and attends with it."""
    unit = "steps/s"

    def __init__(self, crs, dev):
        self.crs = crs
        S, H, d, b, R, n = 64, 8, 64, 64, 4, 16384
        self.p = dict(n_seq=S, n_heads=H, d=d, n_buckets=b, n_rounds=R, prompt=n, page_size=64, list_page=64)
        self.name = f"lsh_decode_seq{S}_H{H}_d{d}_b{b}_r{R}_ctx{n}"
        self.units_per_step = 1
        g = torch.Generator(device="cpu").manual_seed(61)
        self.rot = torch.randn(H, R, d, b // 2, generator=g).to(dev)
        self.cache = crs.LshDecodeCache(S, H, b, R, max_len=n + 256, device=dev)
        for c0 in range(0, n, 4096):              # the prompt, in pieces (device memory for inputs)
            x = torch.randn(S, 4096, H, d, generator=g).to(torch.bfloat16).to(dev)
            v = torch.randn(S, 4096, H, d, generator=g).to(torch.bfloat16).to(dev)
            self.cache.prefill(x, v, self.rot)
        self.x = torch.randn(S, 1, H, d, generator=g).to(torch.bfloat16).to(dev)
        self.v = torch.randn(S, 1, H, d, generator=g).to(torch.bfloat16).to(dev)
        self.O = torch.empty((S, H, d), dtype=torch.float32, device=dev)
        self.lse = torch.empty((S, H), dtype=torch.float32, device=dev)
        self.cnt = torch.empty((S, H), dtype=torch.int32, device=dev)
        self.cache.step(self.x, self.v, self.rot, out=self.O, lse=self.lse, count=self.cnt)
        torch.cuda.synchronize()
        self.cand = int(self.cnt.sum())            # candidates of a step (K + V rows read)
        self.h_in = {"x": self.x.cpu().pin_memory(), "v": self.v.cpu().pin_memory()}
        self.d_in = {k: torch.empty_like(t, device=dev) for k, t in self.h_in.items()}
        self.h_out = torch.empty(self.O.shape, dtype=self.O.dtype).pin_memory()
        self.h2d = sum(t.numel() * t.element_size() for t in self.h_in.values())
        self.d2h = self.h_out.numel() * self.h_out.element_size()

    def step(self):
        self.cache.step(self.x, self.v, self.rot, out=self.O, lse=self.lse, count=self.cnt)

    def e2e_step(self):
        for k, h in self.h_in.items():
            self.d_in[k].copy_(h, non_blocking=True)
        self.cache.step(self.d_in["x"], self.d_in["v"], self.rot, out=self.O, lse=self.lse, count=self.cnt)
        self.h_out.copy_(self.O, non_blocking=True)

    def roofline_spec(self):
        # per candidate: its key and value rows (2 x 128 B), its list entry (4 B) and the
        # earlier rounds' bucket bytes; per step and (row, head): the new rows written
        return {"lsh_decode": [("hbm", self.cand * (256 + 4 + self.p["n_rounds"]) / 1e9, "GB/s")]}


class PrefillWorkload(Workload):
    unit = "tokens/s"

    def __init__(self, crs, dev):
        import workloads
        self.crs = crs
        c = workloads.indexer_prefill_case(device=dev)
        self.c = c
        self.p = c["params"]
        self.name = c["workload"]
        n, k = self.p["n"], self.p["topk"]
        self.units_per_step = n
        self.idx = torch.empty((n, k), dtype=torch.int32, device=dev)
        self.cnt = torch.empty((n,), dtype=torch.int32, device=dev)
        self.O = torch.empty(c["Q"].shape, dtype=torch.float32, device=dev)
        self.q_pos = torch.arange(n, dtype=torch.int32, device=dev)     # causal limit of row t
        import ctypes
        ip = crs.IndexerParams(crs.CRS_IDX_PREFILL, n, 4, 64, k, 0)
        self.ws = torch.empty(max(1, int(crs.lib().crs_indexer_topk_workspace_size(ctypes.byref(ip)))),
                              dtype=torch.uint8, device=dev)
        self.h_in = {k2: c[k2].cpu().pin_memory() for k2 in ("Q", "K", "V", "q_idx", "k_idx", "w")}
        self.d_in = {k2: torch.empty_like(c[k2]) for k2 in self.h_in}
        self.h_out = torch.empty(self.O.shape, dtype=self.O.dtype).pin_memory()
        self.h2d = sum(t.numel() * t.element_size() for t in self.h_in.values())
        self.d2h = self.h_out.numel() * self.h_out.element_size()

    def _run(self, src):
        k = self.p["topk"]
        self.crs.indexer_topk(src["q_idx"], src["w"], src["k_idx"], k, self.crs.CRS_IDX_PREFILL,
                              out=self.idx, count=self.cnt, workspace=self.ws)
        self.crs.sparse_attn(src["Q"], src["K"], src["V"], self.idx.view(-1, 1, k), q_pos=self.q_pos,
                             out=self.O)

    def step(self):
        self._run(self.c)

    def e2e_step(self):
        for k2, h in self.h_in.items():
            self.d_in[k2].copy_(h, non_blocking=True)
        self._run(self.d_in)
        self.h_out.copy_(self.O, non_blocking=True)

    def cpu_sample(self, frac):
        return cpu_sample_prefill(self.c, max(16, int(512 * frac)))

    def roofline_spec(self):
        n, k = self.p["n"], self.p["topk"]
        pairs = n * (n + 1) // 2
        rows = sum(min(k, t + 1) for t in range(n))
        return {
            "idx_slice_topk": [("alu", pairs * 4 * 64 * 2 / 1e12, "TFLOP/s")],
            # two launches per step (sampled threshold pass + filter pass): the
            # step's causal score FLOPs split evenly over them
            "idx_prefill_tc": [("tensor", pairs * 4 * 64 * 2 / 2 / 1e12, "TFLOP/s")],
            # the K/V cache (n x 512 B = 16.8 MB) stays in L2: its gathers are bound by the
            # L2 read ceiling, measured by crs_probe_l2_gather in the same run
            "sparse_attn": [("l2", rows * 128 * 2 * 2 / 1e9, "GB/s"),
                            ("tensor", rows * 16 * 128 * 4 / 1e12, "TFLOP/s")],
        }


class PrefillHisaWorkload(PrefillWorkload):
    """The indexer prefill workload with the hierarchical indexer in its prefill form:
    mean representatives of 64-key blocks (built once per filled block, untimed), 128
    kept blocks per query (all of them for the first 8192 + 64 queries), the token
    top-2048 on the tensor cores over the kept blocks and the open block, then the
    same gather attention."""
    BLK, TOP_BLOCKS = 64, 128
    cpu_sample = None

    def __init__(self, crs, dev):
        super().__init__(crs, dev)
        n = self.p["n"]
        self.name = self.c["workload"].replace("indexer_prefill_", f"hisa_b{self.BLK}_kb{self.TOP_BLOCKS}_prefill_", 1)
        ko = torch.tensor([0, n], dtype=torch.int64, device=dev)
        self.rep, _ = crs.hisa_describe(self.c["k_idx"], ko, self.BLK, n)
        self.blocks = torch.empty((n, self.TOP_BLOCKS), dtype=torch.int32, device=dev)
        import ctypes
        hp = crs.HisaParams(n, 4, 64, self.p["topk"], self.BLK, self.TOP_BLOCKS, n)
        self.ws = torch.empty(int(crs.lib().crs_hisa_topk_prefill_workspace_size(ctypes.byref(hp))),
                              dtype=torch.uint8, device=dev)
        torch.cuda.synchronize()

    def _run(self, src):
        k = self.p["topk"]
        self.crs.hisa_topk_prefill(src["q_idx"], src["w"], src["k_idx"], self.rep, k, self.BLK, self.TOP_BLOCKS,
                                   out_blocks=self.blocks, out=self.idx, count=self.cnt, workspace=self.ws)
        self.crs.sparse_attn(src["Q"], src["K"], src["V"], self.idx.view(-1, 1, k), q_pos=self.q_pos,
                             out=self.O)

    def roofline_spec(self):
        spec = super().roofline_spec()
        n = self.p["n"]
        nb = n // self.BLK
        # coarse scores of the rows with more than TOP_BLOCKS complete blocks (CUDA cores)
        coarse = sum(max(0, (t + 1) // self.BLK) for t in range(n) if (t + 1) // self.BLK > self.TOP_BLOCKS)
        spec["hisa"] = [("alu", coarse * 4 * 64 * 2 / 1e12, "TFLOP/s")]
        return spec


class DecodeWorkload(Workload):
    unit = "steps/s"

    def __init__(self, crs, dev):
        import workloads
        self.crs = crs
        c = workloads.indexer_decode_case(device=dev)
        self.c = c
        self.p = c["params"]
        self.name = c["workload"]
        ns, k = self.p["n_seq"], self.p["topk"]
        self.units_per_step = 1
        self.idx = torch.empty((ns, k), dtype=torch.int32, device=dev)
        self.cnt = torch.empty((ns,), dtype=torch.int32, device=dev)
        self.O = torch.empty(c["Q"].shape, dtype=torch.float32, device=dev)
        self.kv_base = c["offsets"][:-1].contiguous()
        self.q_pos = (c["ctx"] - 1).to(torch.int32).contiguous()     # row s sees [0, ctx_s)
        import ctypes
        ip = crs.IndexerParams(crs.CRS_IDX_DECODE, ns, 4, 64, k, 131072)
        self.ws = torch.empty(int(crs.lib().crs_indexer_topk_workspace_size(ctypes.byref(ip))),
                              dtype=torch.uint8, device=dev)
        ap = crs.AttnParams(ns, 32, 8, 128, k, 1, int(c["offsets"][-1]), 0.0)
        self.ws2 = torch.empty(max(1, int(crs.lib().crs_sparse_attn_workspace_size(ctypes.byref(ap)))),
                               dtype=torch.uint8, device=dev)
        # end to end: the per-step inputs are the new queries (caches stay resident)
        self.h_in = {k2: c[k2].cpu().pin_memory() for k2 in ("q_idx", "w", "Q")}
        self.d_in = {k2: torch.empty_like(c[k2]) for k2 in self.h_in}
        self.h_out = torch.empty(self.O.shape, dtype=self.O.dtype).pin_memory()
        self.h2d = sum(t.numel() * t.element_size() for t in self.h_in.values())
        self.d2h = self.h_out.numel() * self.h_out.element_size()
        self.total_ctx = int(c["offsets"][-1])

    def _run(self, q_idx, w, Q):
        k = self.p["topk"]
        self.crs.indexer_topk(q_idx, w, self.c["k_idx"], k, self.crs.CRS_IDX_DECODE,
                              k_offsets=self.c["offsets"], max_keys=131072, out=self.idx,
                              count=self.cnt, workspace=self.ws)
        self.crs.sparse_attn(Q, self.c["K"], self.c["V"], self.idx.view(-1, 1, k),
                             kv_base=self.kv_base, q_pos=self.q_pos, out=self.O, workspace=self.ws2)

    def step(self):
        self._run(self.c["q_idx"], self.c["w"], self.c["Q"])

    def e2e_step(self):
        for k2, h in self.h_in.items():
            self.d_in[k2].copy_(h, non_blocking=True)
        self._run(self.d_in["q_idx"], self.d_in["w"], self.d_in["Q"])
        self.h_out.copy_(self.O, non_blocking=True)

    def cpu_sample(self, frac):
        return cpu_sample_decode(self.c, max(1, int(self.p["n_seq"] * frac)))

    def roofline_spec(self):
        ns, k = self.p["n_seq"], self.p["topk"]
        return {
            "idx_slice_topk": [("hbm", self.total_ctx * 64 * 2 / 1e9, "GB/s")],
            # the select reads each row's score keys (4 B per cached token)
            "idx_select": [("hbm", self.total_ctx * 4 / 1e9, "GB/s")],
            "sparse_attn": [("hbm", ns * k * 8 * 128 * 2 * 2 / 1e9, "GB/s")],
        }


class DecodeHisaWorkload(DecodeWorkload):
    """The indexer decode step with the hierarchical indexer: mean representatives of
    64-key blocks (a cache, built once per filled block), 128 kept blocks per row, the
    token indexer on their keys and the open block, then the gather attention."""
    BLK, TOP_BLOCKS = 64, 128
    cpu_sample = None

    def __init__(self, crs, dev):
        super().__init__(crs, dev)
        self.name = self.c["workload"].replace("indexer_decode_", f"hisa_b{self.BLK}_kb{self.TOP_BLOCKS}_decode_", 1)
        self.rep, self.bo = crs.hisa_describe(self.c["k_idx"], self.c["offsets"], self.BLK, 131072)
        torch.cuda.synchronize()
        import ctypes
        hp = crs.HisaParams(self.p["n_seq"], 4, 64, self.p["topk"], self.BLK, self.TOP_BLOCKS, 131072)
        self.ws = torch.empty(int(crs.lib().crs_hisa_topk_workspace_size(ctypes.byref(hp))),
                              dtype=torch.uint8, device=dev)
        self.blocks = torch.empty((self.p["n_seq"], self.TOP_BLOCKS), dtype=torch.int32, device=dev)

    def _run(self, q_idx, w, Q):
        k = self.p["topk"]
        self.crs.hisa_topk(q_idx, w, self.c["k_idx"], self.c["offsets"], self.rep, self.bo, k, self.BLK,
                           self.TOP_BLOCKS, 131072, out_blocks=self.blocks, out=self.idx, count=self.cnt,
                           workspace=self.ws)
        self.crs.sparse_attn(Q, self.c["K"], self.c["V"], self.idx.view(-1, 1, k),
                             kv_base=self.kv_base, q_pos=self.q_pos, out=self.O, workspace=self.ws2)

    def roofline_spec(self):
        ns, k = self.p["n_seq"], self.p["topk"]
        n_blocks = int(self.bo[-1])
        cand = ns * (self.TOP_BLOCKS * self.BLK + self.BLK // 2)
        return {
            # representatives (256 B each) + the candidates' index keys (128 B each)
            "hisa": [("hbm", (n_blocks * 256 + cand * 128) / 1e9, "GB/s")],
            "sparse_attn": [("hbm", ns * k * 8 * 128 * 2 * 2 / 1e9, "GB/s")],
        }


class BlockWorkload(Workload):
    unit = "steps/s"

    def __init__(self, crs, dev):
        import workloads
        self.crs = crs
        c = workloads.block_decode_case(device=dev)
        self.c = c
        self.p = c["params"]
        self.name = c["workload"]
        p = self.p
        self.units_per_step = 1
        self._build_cache()                     # descriptor cache build (once, untimed)
        torch.cuda.synchronize()
        cap = p["top_blocks"] * p["L"] + p["window"]
        self.tok = torch.empty((p["n_seq"], p["n_kv_heads"], cap), dtype=torch.int32, device=dev)
        self.cnt = torch.empty((p["n_seq"], p["n_kv_heads"]), dtype=torch.int32, device=dev)
        self.O = torch.empty(c["Q"].shape, dtype=torch.float32, device=dev)
        self.Kf = c["K"].view(p["n_seq"] * p["T"], p["n_kv_heads"], p["D"])
        self.Vf = c["V"].view(p["n_seq"] * p["T"], p["n_kv_heads"], p["D"])
        self.kv_base = torch.arange(p["n_seq"], device=dev, dtype=torch.int64) * p["T"]
        self.q_pos = torch.full((p["n_seq"],), p["T"] - 1, dtype=torch.int32, device=dev)
        import ctypes
        bp = crs.BlockSelParams(crs.BlockParams(p["n_seq"], p["n_kv_heads"], p["T"], p["D"], p["L"],
                                                p["rank"], 0, p["T"] // p["L"]),
                                p["n_q_heads"], p["top_blocks"], p["window"], p["scale"])
        self.ws = torch.empty(int(crs.lib().crs_block_select_workspace_size(ctypes.byref(bp))),
                              dtype=torch.uint8, device=dev)
        ap = crs.AttnParams(p["n_seq"], p["n_q_heads"], p["n_kv_heads"], p["D"], cap,
                            p["n_kv_heads"], p["n_seq"] * p["T"], 0.0)
        self.ws2 = torch.empty(max(1, int(crs.lib().crs_sparse_attn_workspace_size(ctypes.byref(ap)))),
                               dtype=torch.uint8, device=dev)
        self.h_in = {"Q": c["Q"].cpu().pin_memory()}
        self.d_in = {"Q": torch.empty_like(c["Q"])}
        self.h_out = torch.empty(self.O.shape, dtype=self.O.dtype).pin_memory()
        self.h2d = self.h_in["Q"].numel() * 2
        self.d2h = self.h_out.numel() * 2

    def _build_cache(self):
        self.mu, self.xi = self.crs.block_describe(self.c["K"], self.p["L"], self.p["rank"])

    def cpu_sample(self, frac):
        return cpu_sample_block(self, max(1, int(self.p["n_seq"] * frac)))

    def _run(self, Q):
        p = self.p
        self.crs.block_select(Q, self.mu, self.xi, p["T"], p["L"], p["top_blocks"], p["window"],
                              tok=self.tok, count=self.cnt, workspace=self.ws)
        self.crs.sparse_attn(Q, self.Kf, self.Vf, self.tok, kv_base=self.kv_base, q_pos=self.q_pos,
                             out=self.O, workspace=self.ws2)

    def step(self):
        self._run(self.c["Q"])

    def e2e_step(self):
        self.d_in["Q"].copy_(self.h_in["Q"], non_blocking=True)
        self._run(self.d_in["Q"])
        self.h_out.copy_(self.O, non_blocking=True)

    def roofline_spec(self):
        p = self.p
        nf = p["T"] // p["L"]
        desc = p["n_seq"] * p["n_kv_heads"] * nf * (1 + p["rank"]) * p["D"] * 4
        cap = p["top_blocks"] * p["L"] + p["window"]
        return {
            "block_score": [("hbm", desc / 1e9, "GB/s")],
            "sparse_attn": [("hbm", p["n_seq"] * p["n_kv_heads"] * cap * p["D"] * 2 * 2 / 1e9, "GB/s")],
        }


class BlockFp4Workload(BlockWorkload):
    """The block workload on the deployed descriptor format: bf16 block means and
    FP4 (E2M1) eigenvectors with one fp32 scale per vector (528 B per block of
    D=128, rank 4, against 2560 B in fp32).  Cache build: describe + quantise."""

    def __init__(self, crs, dev):
        super().__init__(crs, dev)
        p = self.p
        self.name = self.c["workload"].replace("block_", "block_fp4_", 1)
        self.mu16, self.xi4, self.xs = crs.block_quantize(self.mu, self.xi, p["T"], p["L"])
        torch.cuda.synchronize()
        del self.mu, self.xi
        torch.cuda.empty_cache()

    def _run(self, Q):
        p = self.p
        self.crs.block_select_fp4(Q, self.mu16, self.xi4, self.xs, p["T"], p["L"], p["top_blocks"],
                                  p["window"], tok=self.tok, count=self.cnt, workspace=self.ws)
        self.crs.sparse_attn(Q, self.Kf, self.Vf, self.tok, kv_base=self.kv_base, q_pos=self.q_pos,
                             out=self.O, workspace=self.ws2)

    def roofline_spec(self):
        p = self.p
        nf = p["T"] // p["L"]
        per_block = p["D"] * 2 + p["rank"] * (p["D"] // 2 + 4)
        cap = p["top_blocks"] * p["L"] + p["window"]
        return {
            "block_score": [("hbm", p["n_seq"] * p["n_kv_heads"] * nf * per_block / 1e9, "GB/s")],
            "sparse_attn": [("hbm", p["n_seq"] * p["n_kv_heads"] * cap * p["D"] * 2 * 2 / 1e9, "GB/s")],
        }


class BlockQuestWorkload(BlockWorkload):
    """Baseline selector: Quest boxes (element-wise key min / max per block, bf16, 512 B
    per block) under the same selection rule, then the gather attention."""
    cpu_sample = None

    def __init__(self, crs, dev):
        super().__init__(crs, dev)
        self.name = self.c["workload"].replace("block_", "block_quest_", 1)

    def _build_cache(self):
        self.kmin, self.kmax = self.crs.quest_describe(self.c["K"], self.p["L"])

    def _run(self, Q):
        p = self.p
        self.crs.block_select_quest(Q, self.kmin, self.kmax, p["T"], p["L"], p["top_blocks"], p["window"],
                                    tok=self.tok, count=self.cnt, workspace=self.ws)
        self.crs.sparse_attn(Q, self.Kf, self.Vf, self.tok, kv_base=self.kv_base, q_pos=self.q_pos,
                             out=self.O, workspace=self.ws2)

    def roofline_spec(self):
        p = self.p
        spec = super().roofline_spec()
        spec["block_score"] = [("hbm", p["n_seq"] * p["n_kv_heads"] * (p["T"] // p["L"]) * p["D"] * 4 / 1e9,
                                "GB/s")]
        return spec


class BlockSubspaceWorkload(BlockWorkload):
    """COBS descriptors in a query subspace of s = 85 dims: fp32 mean (512 B) and four
    scaled eigenvectors of U^T Sigma U (4 x 85 x 4 B) per block."""
    cpu_sample = None
    SD = 85

    def __init__(self, crs, dev):
        import workloads
        self.U = workloads.query_subspace(128, self.SD, device=dev)
        super().__init__(crs, dev)
        self.name = self.c["workload"].replace("block_", f"block_ss{self.SD}_", 1)
        import ctypes
        p = self.p
        bp = crs.BlockSelParams(crs.BlockParams(p["n_seq"], p["n_kv_heads"], p["T"], p["D"], p["L"],
                                                p["rank"], 0, p["T"] // p["L"]),
                                p["n_q_heads"], p["top_blocks"], p["window"], p["scale"])
        self.ws = torch.empty(int(crs.lib().crs_block_select_ss_workspace_size(ctypes.byref(bp), self.SD)),
                              dtype=torch.uint8, device=dev)

    def _build_cache(self):
        self.mu, self.xi = self.crs.block_describe_ss(self.c["K"], self.p["L"], self.p["rank"], self.U)

    def _run(self, Q):
        p = self.p
        self.crs.block_select_ss(Q, self.U, self.mu, self.xi, p["T"], p["L"], p["top_blocks"], p["window"],
                                 tok=self.tok, count=self.cnt, workspace=self.ws)
        self.crs.sparse_attn(Q, self.Kf, self.Vf, self.tok, kv_base=self.kv_base, q_pos=self.q_pos,
                             out=self.O, workspace=self.ws2)

    def roofline_spec(self):
        p = self.p
        spec = super().roofline_spec()
        per_block = p["D"] * 4 + p["rank"] * self.SD * 4
        spec["block_score"] = [("hbm", p["n_seq"] * p["n_kv_heads"] * (p["T"] // p["L"]) * per_block / 1e9,
                                "GB/s")]
        return spec


class BlockFp4SubspaceWorkload(BlockWorkload):
    """The pages' deployed descriptor (the delivered row of the COBS notes' Table 3):
    bf16 block means and four FP4 (E2M1) scaled eigenvectors of the query-subspace
    covariance (s = 85), scored on the tensor cores with the projected query.  Cache
    build: subspace describe + quantise (untimed)."""
    SD = 85
    cpu_sample = None

    def __init__(self, crs, dev):
        import workloads
        self.U = workloads.query_subspace(128, self.SD, device=dev)
        super().__init__(crs, dev)
        p = self.p
        self.name = self.c["workload"].replace("block_", f"block_fp4_ss{self.SD}_", 1)
        import ctypes
        bp = crs.BlockSelParams(crs.BlockParams(p["n_seq"], p["n_kv_heads"], p["T"], p["D"], p["L"],
                                                p["rank"], 0, p["T"] // p["L"]),
                                p["n_q_heads"], p["top_blocks"], p["window"], p["scale"])
        self.ws = torch.empty(int(crs.lib().crs_block_select_fp4_ss_workspace_size(ctypes.byref(bp), self.SD)),
                              dtype=torch.uint8, device=dev)

    def _build_cache(self):
        mu, xi = self.crs.block_describe_ss(self.c["K"], self.p["L"], self.p["rank"], self.U)
        self.mu16, self.xi4, self.xs = self.crs.block_quantize_ss(mu, xi, self.p["T"], self.p["L"])
        torch.cuda.synchronize()
        del mu, xi

    def _run(self, Q):
        p = self.p
        self.crs.block_select_fp4_ss(Q, self.U, self.mu16, self.xi4, self.xs, p["T"], p["L"], p["top_blocks"],
                                     p["window"], tok=self.tok, count=self.cnt, workspace=self.ws)
        self.crs.sparse_attn(Q, self.Kf, self.Vf, self.tok, kv_base=self.kv_base, q_pos=self.q_pos,
                             out=self.O, workspace=self.ws2)

    def summary_bytes(self):
        """Summary-key bytes of one sequence's step (4 KV heads x T/L blocks): the pages'
        accounting (bf16 mean + 4 x (s/2 code bytes + a 4-byte scale)) and what is stored
        (codes padded to 48 bytes per vector)."""
        p = self.p
        blocks = p["n_kv_heads"] * (p["T"] // p["L"])
        alg = blocks * (p["D"] * 2 + p["rank"] * (self.SD / 2 + 4))
        stored = blocks * (p["D"] * 2 + p["rank"] * (48 + 4))
        return alg, stored

    def roofline_spec(self):
        p = self.p
        spec = super().roofline_spec()
        _, stored = self.summary_bytes()
        spec["block_score"] = [("hbm", p["n_seq"] * stored / 1e9, "GB/s")]
        return spec


class BlockMeanPoolWorkload(BlockWorkload):
    """Baseline selector: the block mean alone (first-order score, fp32, 512 B per block)."""
    cpu_sample = None

    def __init__(self, crs, dev):
        super().__init__(crs, dev)
        self.name = self.c["workload"].replace("block_", "block_meanpool_", 1)

    def _build_cache(self):
        self.mu, _ = self.crs.block_describe(self.c["K"], self.p["L"], 1)
        self.xi = None

    def roofline_spec(self):
        p = self.p
        spec = super().roofline_spec()
        spec["block_score"] = [("hbm", p["n_seq"] * p["n_kv_heads"] * (p["T"] // p["L"]) * p["D"] * 4 / 1e9,
                                "GB/s")]
        return spec


WORKLOADS = {"lsh": lambda crs, dev: LshWorkload(crs, dev),
             "lsh_fp32": lambda crs, dev: LshWorkload(crs, dev, fp32=True),
             "prefill": PrefillWorkload, "prefill_hisa": PrefillHisaWorkload, "decode": DecodeWorkload,
             "decode_hisa": DecodeHisaWorkload,
             "lsh_decode": LshDecodeWorkload, "route": RouteWorkload,
             "block": BlockWorkload,
             "block_fp4": BlockFp4Workload, "block_quest": BlockQuestWorkload,
             "block_meanpool": BlockMeanPoolWorkload, "block_ss": BlockSubspaceWorkload,
             "block_fp4_ss": BlockFp4SubspaceWorkload}


# ------------------------------------------------------------------- timing --
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(gpu_index)], stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.flush()
        self.f.seek(0)
        rows = [r.split(",") for r in self.f.read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        sm, mx, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
                power.append(float(r[3]))
                for k, v in zip(names, r[5:9]):
                    if v.strip().lower() == "active":
                        reasons.add(k)
            except (ValueError, IndexError):
                continue
        loaded = [s for s, p in zip(sm, power) if p > 200] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm), "samples_under_load": len([p for p in power if p > 200])}


def _flush_l2(buf):
    buf.add_(1)


def time_steps(fn, steps, warmup, flush_buf, dist_on):
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        fn()
        _flush_l2(flush_buf)
    torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for a, b in ev:
        a.record(stream)
        fn()
        b.record(stream)
        _flush_l2(flush_buf)
    torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def _traffic(kernel, workload):
    """DRAM bytes per launch of `kernel` on `workload` from profiles/traffic.json,
    only while the kernel's source file is unchanged since the capture (else None)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f).get(f"{kernel}@{workload}")
    if not t:
        return None
    src = os.path.join(ROOT, t["source"])
    if not os.path.exists(src):
        return None
    with open(src, "rb") as f:
        if hashlib.sha256(f.read()).hexdigest()[:16] != t["sha256_16"]:
            return None
    return t["bytes_per_launch"]


def roofline(wl, prof, peaks, traffic=None):
    """The dominant kernel (largest summed device time) with its algorithmic work."""
    spec = dict(wl.roofline_spec())
    companions = spec.pop("_with", {})
    timed = {k: v for k, v in prof.items() if v["timed_launches"] > 0}
    if not timed:
        return None, {}
    stages = {k: round(v["total_ms"] / v["timed_launches"], 5) for k, v in timed.items()}
    top = max(timed, key=lambda k: timed[k]["total_ms"])
    if top not in spec:
        return {"kernel": top, "bound": None, "achieved": None, "peak": None, "unit": None,
                "frac": None, "traffic": None}, stages
    # kernels that always run right after the top one, on its leftovers, count with it
    with_ms = sum(timed[c]["total_ms"] for c in companions.get(top, []) if c in timed)
    per_launch_s = (timed[top]["total_ms"] + with_ms) / timed[top]["timed_launches"] / 1e3

    def peak_of(bound):
        if bound == "hbm":
            return peaks["hbm_gbs"], f"hbm_gbs ({peaks['source']})"
        if bound == "tensor":
            return peaks["bf16_tflops"], f"bf16_tflops ({peaks['source']})"
        if bound == "l2":
            return peaks["l2_gather_gbs"], "l2_gather_gbs (crs_probe_l2_gather on this GPU, this run)"
        return FP32_ALU_TFLOPS_NOMINAL, "fp32 FMA: 148 SM x 128 lanes x 2 x 1.965 GHz"

    # the binding roofline: the resource whose algorithmic work takes longest at its peak
    entries = sorted(spec[top], key=lambda e: -e[1] / peak_of(e[0])[0])
    bound, amount, unit = entries[0]
    peak, src = peak_of(bound)
    achieved = amount / per_launch_s
    out = {"kernel": top, "bound": bound, "achieved": round(achieved, 3), "peak": round(peak, 1),
           "unit": unit, "frac": round(achieved / peak, 4), "traffic": _traffic(top, wl.name),
           "peak_source": src,
           "per_launch_ms": round(per_launch_s * 1e3, 5)}
    if companions.get(top):
        out["includes"] = [c for c in companions[top] if c in timed]
    if len(entries) > 1:
        b2, a2, u2 = entries[1]
        p2 = peak_of(b2)[0]
        out["secondary"] = {"bound": b2, "achieved": round(a2 / per_launch_s, 3), "peak": round(p2, 1),
                            "unit": u2, "frac": round(a2 / per_launch_s / p2, 4)}
    return out, stages


def measure(crs, wl, steps, warmup, flush_buf, dist_on, peaks, e2e=True):
    crs.profile_collect()
    times = time_steps(wl.step, steps, warmup, flush_buf, dist_on)
    launched = crs.profile_collect()
    launches_timed = sum(v["launches"] for v in launched.values())
    # launches per step, counted over the timed steps only (warm-up excluded by a separate count)
    crs.profile_collect()
    for _ in range(1):
        wl.step()
    torch.cuda.synchronize()
    per_step = sum(v["launches"] for v in crs.profile_collect().values())
    crs.profile_set(True)
    time_steps(wl.step, steps, 1, flush_buf, False)
    crs.profile_set(False)
    prof = crs.profile_collect()
    rl, stages = roofline(wl, prof, peaks)
    out = {"times_ms": times, "gpu_launches": per_step * steps, "roofline": rl, "stages_ms": stages,
           "launches_in_timed_region_incl_warmup": launches_timed}
    if e2e:
        out["e2e_times_ms"] = time_steps(wl.e2e_step, steps, warmup, flush_buf, dist_on)
    return out


# ------------------------------------------------------------- CPU baseline --
# The oracle (plain C, fp64, OpenMP over rows), timed as it stands on the host
# cores on a bounded sample of the same workload.  Only the oracle calls are
# timed; copying inputs to the host (and, for the gather stages, collecting the
# K/V rows a list names) happens outside the timed spans.  Each function returns
# (units of the workload's metric covered by the sample, seconds, sample text).
def _tnp(t):
    import numpy as np
    return t.detach().cpu().double().numpy().astype(np.float64)


class _Clock:
    def __init__(self):
        self.s = 0.0

    def __call__(self, fn, *a, **k):
        t0 = time.perf_counter()
        r = fn(*a, **k)
        self.s += time.perf_counter() - t0
        return r


def cpu_sample_lsh(case, n_segments=16):
    """n_segments of the B*H (batch, head) segments, each routed (hash + sort, all
    rounds) and attended for all n query rows."""
    import numpy as np

    import oracle
    p = case["params"]
    B, H, n = p["B"], p["H"], p["n"]
    QK = case["QK"].float().cpu().numpy()
    V = case["V"].float().cpu().numpy().astype(np.float64)
    R = case["R"].cpu().numpy()
    vl = case["valid_len"].cpu().numpy()
    segs = [(s // H, s % H) for s in range(min(n_segments, B * H))]
    clk = _Clock()
    for b, h in segs:
        x = QK[b:b + 1, h:h + 1]
        bk = clk(oracle.lsh_hash, x, R[h:h + 1], p["n_buckets"])
        pm, ip = clk(oracle.lsh_sort, bk)
        clk(oracle.lsh_attn, x.astype(np.float64), V[b:b + 1, h:h + 1], bk, pm, ip, vl[b:b + 1],
            p["chunk"], p["causal"], p["no_self"], p["key_norm"], p["scale"])
    tokens = B * n * len(segs) / (B * H)      # a (b, h) segment is 1/(B*H) of a step's work
    sample = (f"{len(segs)} of {B*H} (batch, head) segments: hash + sort + LSH attention for all "
              f"{n} query rows and {p['n_rounds']} rounds, scaled by segments/(B*H)")
    return tokens, clk.s, sample


def cpu_baseline_lsh(case, n_segments=16):
    tokens, dt, sample = cpu_sample_lsh(case, n_segments)
    return tokens / dt, dt, sample


def cpu_sample_prefill(c, n_rows=512):
    """n_rows query rows spread evenly over the sequence (row t scores its t + 1 keys),
    each: indexer top-k, then gather attention of the 16 heads over the oracle's own
    list.  Tokens covered = rows."""
    import numpy as np

    import oracle
    p = c["params"]
    n, k = p["n"], p["topk"]
    rows = ((np.arange(n_rows) + 0.5) * n / n_rows).astype(np.int64)
    qd, wd, Kd = _tnp(c["q_idx"][rows]), _tnp(c["w"][rows]), _tnp(c["k_idx"])
    Q, K, V = _tnp(c["Q"][rows]), _tnp(c["K"]), _tnp(c["V"])
    clk = _Clock()
    idx, cnt, _, _ = clk(oracle.indexer_topk, qd, wd, Kd, np.zeros(n_rows, np.int64),
                         (rows + 1).astype(np.int32), k)
    clk(oracle.sparse_attn, Q, K, V, idx[:, None, :], q_pos=rows.astype(np.int32))
    return float(n_rows), clk.s, (f"{n_rows} of {n} query rows evenly spaced (indexer top-{k} over "
                                  f"keys 0..t, then {p['n_q_heads']}-head attention over the list)")


def cpu_sample_decode(c, n_seq=64):
    """n_seq of the sequences: indexer top-k over the whole context, then the GQA
    attention over the oracle's list (the listed K/V rows collected on the device,
    untimed).  Steps covered = n_seq / sequences."""
    import numpy as np

    import oracle
    p = c["params"]
    S, k = p["n_seq"], p["topk"]
    off = c["offsets"].cpu().numpy()
    clk = _Clock()
    for s in range(min(n_seq, S)):
        Kr = _tnp(c["k_idx"][off[s]:off[s + 1]])
        idx, cnt, _, _ = clk(oracle.indexer_topk, _tnp(c["q_idx"][s:s + 1]), _tnp(c["w"][s:s + 1]), Kr,
                             np.zeros(1, np.int64), np.array([Kr.shape[0]], np.int32), k)
        lst = torch.as_tensor(off[s] + idx[0, : cnt[0]], dtype=torch.int64, device=c["K"].device)
        Kc, Vc = _tnp(c["K"][lst]), _tnp(c["V"][lst])
        I = np.arange(int(cnt[0]), dtype=np.int32)[None, None]
        clk(oracle.sparse_attn, _tnp(c["Q"][s:s + 1]), Kc, Vc, I)
    m = min(n_seq, S)
    return m / S, clk.s, (f"{m} of {S} sequences (indexer top-{k} over the context, then "
                          f"{p['n_q_heads']}/{p['n_kv_heads']} GQA attention), scaled by sequences/{S}")


def cpu_sample_block(wl, n_seq=32):
    """n_seq of the sequences: block selection on the step's descriptors (fp32, or the
    dequantised FP4 ones), then the attention over each KV head's token list (the listed
    rows collected on the device, untimed).  Steps covered = n_seq / sequences."""
    import numpy as np

    import oracle
    c, p = wl.c, wl.p
    S, T, L, nkv = p["n_seq"], p["T"], p["L"], p["n_kv_heads"]
    G = p["n_q_heads"] // nkv
    clk = _Clock()
    m = min(n_seq, S)
    for s in range(m):
        if hasattr(wl, "xi4"):
            mu = _tnp(wl.mu16[s:s + 1])
            xi = oracle.fp4_dequantize(wl.xi4[s:s + 1].cpu().numpy(), wl.xs[s:s + 1].cpu().numpy())
        else:
            mu, xi = _tnp(wl.mu[s:s + 1]), _tnp(wl.xi[s:s + 1])
        Qs = _tnp(c["Q"][s:s + 1])
        tok, cnt, _, _ = clk(oracle.block_select, Qs, mu, xi, T, L, p["top_blocks"], p["window"])
        for h in range(nkv):
            lst = torch.as_tensor(tok[0, h, : cnt[0, h]], dtype=torch.int64, device=c["K"].device)
            Kc = _tnp(c["K"][s, lst, h])[:, None, :]
            Vc = _tnp(c["V"][s, lst, h])[:, None, :]
            I = np.arange(int(cnt[0, h]), dtype=np.int32)[None, None]
            clk(oracle.sparse_attn, Qs[:, h * G:(h + 1) * G], Kc, Vc, I)
    kind = "FP4 (dequantised)" if hasattr(wl, "xi4") else "fp32"
    return m / S, clk.s, (f"{m} of {S} sequences (block selection on {kind} descriptors, then "
                          f"attention over each KV head's list), scaled by sequences/{S}")


def cpu_baseline(wl, single_thread_fraction):
    """The oracle on all host cores (the workload's default sample) and on one core
    (a smaller sample): value in the workload's unit, cores, per-core value."""
    import oracle
    fn = getattr(wl, "cpu_sample", None)
    if fn is None:
        return None
    cores = os.cpu_count() or 1
    oracle.set_threads(cores)
    units, dt, sample = fn(1.0)
    oracle.set_threads(1)
    u1, dt1, sample1 = fn(single_thread_fraction)
    oracle.set_threads(cores)
    return {"value": round(units / dt, 3), "unit": wl.unit, "cores": cores, "kind": "oracle",
            "sample": sample, "seconds": round(dt, 3),
            "per_core": {"value": round(u1 / dt1, 3), "unit": wl.unit, "cores": 1, "sample": sample1,
                         "seconds": round(dt1, 3)}}


def _omp_threads():
    v = os.environ.get("OMP_NUM_THREADS")
    return int(v) if v and v.isdigit() else (os.cpu_count() or 1)


# --------------------------------------------------------------------- main --
def reduce_max_over_ranks(values, device):
    """Each entry's maximum over the ranks of the default process group: the job
    takes as long as its slowest rank."""
    t = torch.tensor(values, device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(x) for x in t]


def job_throughput(units_per_step, steps, world, total_ms):
    """Whole-job units per second: every rank processes its own batch (weak
    scaling), timed as the slowest rank's total."""
    return units_per_step * steps * world / (total_ms / 1e3)


def run_reference(args, rank):
    """Oracle arm: the CPU oracle on the host cores, bounded sample per step."""
    if rank != 0:
        return 0
    import workloads
    case = workloads.lsh_clustered_case(device="cpu")
    p = case["params"]
    for _ in range(args.warmup):
        cpu_baseline_lsh(case, n_segments=1)
    total = 0.0
    for _ in range(args.steps):
        _, dt, sample = cpu_baseline_lsh(case, n_segments=1)
        total += dt
    tokens = p["B"] * p["n"] / (p["B"] * p["H"]) * args.steps
    val = tokens / total
    line = {"impl": "reference", "metric": METRIC, "value": round(val, 3), "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(total / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": case["workload"], "sample": "1 (batch, head) segment per step"},
            "cpu_baseline": {"value": round(val, 3), "unit": "tokens/s", "cores": _omp_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(val, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="product", choices=["product", "reference"])
    ap.add_argument("--workload", default="lsh", choices=sorted(WORKLOADS))
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank)

    dist_on = world > 1
    if dist_on:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    import content_routed_sparse_b200 as crs

    peaks = _peaks()
    peaks["l2_gather_gbs"] = l2_gather_gbs(crs, dev)
    flush_buf = torch.zeros(64 * 1024 * 1024, dtype=torch.float32, device=dev)   # 256 MiB
    wl = WORKLOADS[args.workload](crs, dev)
    sampler = ClockSampler(local)
    time.sleep(0.3)
    res = measure(crs, wl, args.steps, args.warmup, flush_buf, dist_on, peaks)
    clocks = sampler.stop()
    assert crs.get_device_error() == 0, "device error word set during the bench"

    tot_ms = sum(res["times_ms"])
    e2e_ms = sum(res["e2e_times_ms"])
    if dist_on:
        tot_ms, e2e_ms = reduce_max_over_ranks([tot_ms, e2e_ms], dev)
    value = job_throughput(wl.units_per_step, args.steps, world, tot_ms)
    e2e_value = job_throughput(wl.units_per_step, args.steps, world, e2e_ms)

    extras = {}
    if not args.no_extras and not dist_on:
        for name in [w for w in ("lsh_fp32", "lsh_decode", "route", "prefill", "prefill_hisa", "decode", "decode_hisa",
                                  "block", "block_fp4", "block_fp4_ss", "block_ss",
                                  "block_quest", "block_meanpool") if w != args.workload]:
            try:
                w2 = WORKLOADS[name](crs, dev)
                r2 = measure(crs, w2, 5, 3, flush_buf, False, peaks)
                t2 = sum(r2["times_ms"])
                extras[name] = {"workload": w2.name, "value": round(w2.units_per_step * 5 / (t2 / 1e3), 3),
                                "unit": w2.unit, "ms_per_step": round(t2 / 5, 4),
                                "roofline": r2["roofline"], "stages_ms": r2["stages_ms"],
                                "e2e": {"value": round(w2.units_per_step * 5 / (sum(r2["e2e_times_ms"]) / 1e3), 3),
                                        "unit": w2.unit, "h2d_bytes_per_step": w2.h2d,
                                        "d2h_bytes_per_step": w2.d2h},
                                "gpu_launches": r2["gpu_launches"]}
                if not args.no_cpu_baseline:
                    extras[name]["cpu_baseline"] = cpu_baseline(w2, 1.0 / 8)
                if hasattr(w2, "summary_bytes"):
                    alg, stored = w2.summary_bytes()
                    extras[name]["summary_key_kib_per_seq"] = {"algorithmic": round(alg / 1024, 1),
                                                               "stored": round(stored / 1024, 1),
                                                               "pages_table3": 1767}
                if name == "block":
                    torch.cuda.synchronize()
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record()
                    crs.block_describe(w2.c["K"], w2.p["L"], w2.p["rank"], mu=w2.mu, xi=w2.xi)
                    e1.record()
                    torch.cuda.synchronize()
                    extras[name]["cache_build_ms"] = round(e0.elapsed_time(e1), 4)
                    e0.record()
                    crs.block_quantize(w2.mu, w2.xi, w2.p["T"], w2.p["L"])
                    e1.record()
                    torch.cuda.synchronize()
                    extras[name]["fp4_quantize_ms"] = round(e0.elapsed_time(e1), 4)
                del w2
                torch.cuda.empty_cache()
            except Exception as e:   # an extra section must not hide the headline
                extras[name] = {"error": f"{type(e).__name__}: {e}"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, 1.0 / 16)
    step_rl = None
    if hasattr(wl, "step_bytes"):
        gbs = wl.step_bytes() / (tot_ms / args.steps / 1e3) / 1e9
        step_rl = {"bound": "hbm", "bytes_per_step": wl.step_bytes(), "achieved": round(gbs, 3),
                   "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4)}

    if rank == 0:
        p = getattr(wl, "p", {})
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": wl.unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(tot_ms / args.steps, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype,
            "data": "synthetic",
            "config": {"workload": wl.name, **{k: v for k, v in p.items() if not callable(v)},
                       "l2": "256 MiB buffer written between timed steps (outside the events)",
                       "parallelism": f"replica per GPU x{world}"},
            "e2e": {"value": round(e2e_value, 3), "unit": wl.unit, "h2d_bytes_per_step": wl.h2d,
                    "d2h_bytes_per_step": wl.d2h},
            "gpu_launches": res["gpu_launches"],
            "roofline": res["roofline"],
            "step_roofline": step_rl,
            "stages_ms": res["stages_ms"],
            "cpu_baseline": cpu,
            "clocks": clocks,
            "extras": extras,
        }
        print(json.dumps(line), flush=True)
    if dist_on:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

#!/usr/bin/env python3
"""Benchmark of the hybrid CSA/HCA attention layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Default workload: hybrid_decode_b8_1m -- a CSA layer and an HCA layer decoded
back to back for 8 requests at 1,048,576 tokens of context (CSA: 262,144
compressed entries x 512 + indexer keys x 128, 64 indexer heads, top-1024;
HCA: 8,192 entries; 128-row windows; 64 query heads x 512).  Metric: decode
queries per second (one query = one request's step through both layers).
Other workloads: csa_prefill_64k (tokens/s), csa_decode_b32_128k and
hca_decode_b16_1m (queries/s).

One process per GPU; under torchrun every rank runs the same per-GPU
workload on its own requests (weak scaling, no collective on the data path),
timing is the max over ranks.  Prints one JSON line on rank 0.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from long_context_attention_compress_b200 import workloads as wl  # noqa: E402

L2_FLUSH_BYTES = 256 << 20
MIB = 1 << 20
DEFAULT_WORKLOAD = "hybrid_decode_b8_1m"
# the headline region is repeated until it has run this long (>= ~10 clock samples at 50 ms)
HEADLINE_MIN_S = 0.75


# ----------------------------------------------------------------------------
# distributed plumbing
# ----------------------------------------------------------------------------
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, local, ws


def init_dist(backend):
    import datetime
    import torch.distributed as dist
    rank, local, ws = dist_env()
    if ws > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return rank, local, ws


def reduce_max(x: float, ws: int, device) -> float:
    if ws == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(ws: int):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def shard_seed(seed: int, rank: int) -> int:
    """Each rank draws its own requests: disjoint seeds, same distribution."""
    return seed + 1_000_000 * rank


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None

    def __enter__(self):
        self.first = ""
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            # the timed region starts only once the sampler is producing samples
            # (that first sample is kept with the others)
            self.first = self.proc.stdout.readline()
        except (FileNotFoundError, OSError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.rows = []
        if self.proc is None:
            return False
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.rows = parse_clock_rows(self.first + out)
        return False

    def summary(self):
        if not getattr(self, "rows", None):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(self.rows)}


def parse_clock_rows(text: str):
    """nvidia-smi CSV rows (index, sm MHz, max MHz, power, reasons...) as lists of fields."""
    rows = []
    for line in text.splitlines():
        parts = [p.strip() for p in line.split(",")]
        if len(parts) >= 9:
            rows.append(parts)
    return rows


def clock_rejected(c) -> bool:
    """A timed region whose clocks saw a hardware or thermal slowdown, or an SM clock
    well below its maximum with no reason reported (a leftover clock lock)."""
    if set(c.get("reasons", [])) & {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}:
        return True
    sm, smax = c.get("sm_mhz"), c.get("sm_max_mhz")
    return bool(sm and smax and sm < 0.8 * smax and not c.get("reasons"))


# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------
# B200 datasheet figures, reported beside the measured peaks (the stricter denominators):
# ~8 TB/s of HBM3e and 2.25 PFLOP/s dense bf16.
DATASHEET = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def traffic_table():
    """ncu DRAM bytes per launch, keyed by kernel, valid only for the source hash it was taken on."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return {}
    try:
        return json.load(open(p))
    except ValueError:
        return {}


def source_hash(files):
    import hashlib
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(ROOT, "long_context_attention_compress_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


class DecodeBench:
    """Hybrid / CSA / HCA decode.  Per step: one hybrid_attn_decode call."""

    def __init__(self, name, spec, seed, device, qk_norm=False, indexer="bf16", paged=False, kv_fp8=False):
        import long_context_attention_compress_b200 as hca
        self.hca = hca
        self.name = name
        self.spec = spec
        self.indexer = indexer
        self.kv_fp8 = kv_fp8
        s = self.shape = spec["shape"]
        B, ctx = spec["B"], spec["ctx"]
        # Q/KV normalisation + partial RoPE: synthetic weights per layer
        self.norm_kw = {}
        if qk_norm:
            self.norm_kw = {"csa_norm": wl.norm_weights(s, seed=seed, device=device),
                            "hca_norm": wl.norm_weights(s, seed=seed + 1, device=device)}
        self.B, self.ctx = B, ctx
        kind = spec["kind"]
        std = spec["cache_std"]
        self.csa = self.hcad = None
        if kind == "hybrid_decode":
            d = wl.hybrid_decode_inputs(s, B, ctx, seed=seed, cache_std=std, device=device)
            self.csa, self.hcad = d["csa"], d["hca"]
        elif kind == "csa_decode":
            self.csa = wl.csa_decode_inputs(s, B, ctx, seed=seed, cache_std=std, device=device)
        else:
            self.hcad = wl.hca_decode_inputs(s, B, ctx, seed=seed, cache_std=std, device=device)
        self.cfg = hca.make_cfg(s)
        dev = device
        self.q_pos = (self.csa or self.hcad)["q_pos"]
        self.idx = torch.empty((B, s.topk), dtype=torch.int32, device=dev) if self.csa else None
        self.csa_out = torch.empty((B, s.n_heads, s.c), dtype=torch.bfloat16, device=dev) if self.csa else None
        self.hca_out = torch.empty((B, s.n_heads, s.c), dtype=torch.bfloat16, device=dev) if self.hcad else None
        self.phases = []
        if self.hcad is not None and "block_cand" in self.hcad:
            self.phases.append("hca_compress")
        if self.csa is not None:
            self.phases += ["indexer_scores", "topk_select", "csa_attention"]
        if self.hcad is not None:
            self.phases.append("hca_attention")
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(len(self.phases) + 1)]
        self.norm_kw = {k: v for k, v in self.norm_kw.items()
                        if (k == "csa_norm" and self.csa is not None) or (k == "hca_norm" and self.hcad is not None)}
        if indexer == "fp4":
            # the cache form of the indexer keys: MXFP4 codes + scales (64 + 4 B per key)
            K = self.csa.pop("K_I")
            N = K.shape[1]
            codes = torch.empty((B, N, s.d_idx // 2), dtype=torch.uint8, device=dev)
            scales = torch.empty((B, N, s.d_idx // 32), dtype=torch.uint8, device=dev)
            for b in range(B):
                hca.mxfp4_quantize(K[b], codes=codes[b], scales=scales[b])
            del K
            self.norm_kw["csa_k4"] = (codes, scales)
        self.n_entries = {"csa": self.csa["E"].shape[1] if self.csa is not None else 0,
                          "hca": self.hcad["E_h"].shape[1] if self.hcad is not None else 0}
        self.paged = None
        if paged:
            self._make_paged(seed, dev)
        if kv_fp8:
            # FP8 cache form of both layers' entries (E4M3 + f32 group scales, bf16 rotary part)
            for key, d, arg in (("E", self.csa, "csa_kv8"), ("E_h", self.hcad, "hca_kv8")):
                if d is not None:
                    self.norm_kw[arg] = hca.kv_fp8_quantize(d.pop(key), self.cfg)
            torch.cuda.empty_cache()
        self.args, self._keep = hca.make_decode_args(B, self.q_pos, csa=self.csa, hca=self.hcad,
                                                     csa_topk_idx=self.idx, csa_out=self.csa_out,
                                                     hca_out=self.hca_out, events=self.events, **self.norm_kw)
        self._apply_paged(self.args)
        self.ws = torch.empty(max(1, hca.hybrid_attn_decode_workspace(self.cfg, self.args)), dtype=torch.uint8,
                              device=dev)
        self.units = B
        self.metric = "hybrid CSA+HCA decode queries/s at 1M ctx"
        self.unit = "queries/s"

    def _make_paged(self, seed, dev):
        """The caches in paged form: blocks of lcm(m, m') = 128 raw tokens (32 CSA entries
        and keys, 1 HCA entry per block) in pools, reached through a shuffled block table."""
        s, B = self.shape, self.B
        L = s.m * s.m_hca // math.gcd(s.m, s.m_hca)
        rc, rh = L // s.m, L // s.m_hca
        N = self.csa["E"].shape[1] if self.csa is not None else 0
        Nh = self.hcad["E_h"].shape[1] if self.hcad is not None else 0
        nblk = max((N + rc - 1) // rc, (Nh + rh - 1) // rh)
        P = B * nblk
        g = torch.Generator(device="cpu").manual_seed(seed + 99)
        perm = torch.randperm(P, generator=g).to(torch.int32)
        bt = perm.view(B, nblk).to(dev)
        # physical block perm[b * nblk + j] holds request b's logical block j
        inv = torch.empty_like(perm)
        inv[perm.long()] = torch.arange(P, dtype=torch.int32)
        inv = inv.long().to(dev)

        def pool(flat, rpb):  # [B, n, w] -> [P, rpb, w] in shuffled block order
            Bn, n, w = flat.shape
            fb = flat.new_zeros((Bn, nblk * rpb, w))
            fb[:, :n] = flat
            return fb.view(Bn * nblk, rpb, w)[inv].contiguous()
        if self.csa is not None:
            self.csa["E"] = pool(self.csa["E"], rc)
            if "K_I" in self.csa:
                self.csa["K_I"] = pool(self.csa["K_I"], rc)
        if self.hcad is not None:
            self.hcad["E_h"] = pool(self.hcad["E_h"], rh)
        torch.cuda.empty_cache()
        self.paged = {"bt": bt, "nblk": nblk, "P": P, "N": N, "Nh": Nh}

    def _apply_paged(self, args):
        if self.paged is None:
            return
        pg = self.paged
        args.csa_N, args.hca_N = pg["N"], pg["Nh"]
        args.block_table, args.bt_stride, args.n_pool_blocks = pg["bt"].data_ptr(), pg["nblk"], pg["P"]
        args.csa_kv_stride = args.csa_k_stride = args.hca_kv_stride = 0

    def step(self, record=True):
        self.args.n_events = len(self.events) if record else 0
        self.hca.hybrid_attn_decode(self.cfg, self.args, ws=self.ws)

    def launches_per_step(self):
        return int(self.hca.lib.hca_last_launch_count())

    # algorithmic HBM bytes per phase (what the method must move)
    def phase_bytes(self):
        s, B = self.shape, self.B
        out = {}
        if "hca_compress" in self.phases:
            out["hca_compress"] = B * (2 * s.m_hca * s.c * 2 + s.c * 2)
        if self.csa is not None:
            N = self.n_entries["csa"]
            key_bytes = s.d_idx // 2 + s.d_idx // 32 if self.indexer == "fp4" else s.d_idx * 2
            out["indexer_scores"] = B * (N * key_bytes + s.n_idx_heads * (s.d_idx * 2 + 4))
            out["topk_select"] = B * s.topk * 4
            row = (s.c - s.rope_dims) + 4 * (s.c - s.rope_dims) // 64 + 2 * s.rope_dims if self.kv_fp8 else s.c * 2
            out["csa_attention"] = B * (min(s.topk, N) * row + s.n_win * s.c * 2 + 2 * s.n_heads * s.c * 2 + s.topk * 4)
        if self.hcad is not None:
            Nh = self.n_entries["hca"]
            row = (s.c - s.rope_dims) + 4 * (s.c - s.rope_dims) // 64 + 2 * s.rope_dims if self.kv_fp8 else s.c * 2
            out["hca_attention"] = B * (Nh * row + s.n_win * s.c * 2 + 2 * s.n_heads * s.c * 2)
        return out

    def config(self):
        s = self.shape
        c = {"workload": self.name, "batch": self.B, "context": self.ctx, "c": s.c, "heads": s.n_heads,
             "topk": s.topk, "indexer": f"{s.n_idx_heads}x{s.d_idx}" + (" MXFP4 keys, BF16 scores"
                                                                         if self.indexer == "fp4" else ""),
             "n_win": s.n_win}
        if self.csa is not None:
            c["csa_entries"] = int(self.n_entries["csa"])
        if self.hcad is not None:
            c["hca_entries"] = int(self.n_entries["hca"])
        if self.kv_fp8:
            c["kv_cache"] = "FP8 E4M3 (448 channels, f32 scale per 64) + bf16 rotary 64 channels"
        if self.paged:
            c["cache"] = (f"paged: blocks of 128 raw tokens (32 CSA entries + keys, 1 HCA entry), "
                          f"{self.paged['P']} blocks, shuffled block table")
        return c

    # --- end to end: per-step inputs from pinned host memory, outputs back ---
    def e2e_setup(self):
        """Two device buffer sets of the per-step inputs and outputs (set 0 is the
        bench's own), so that one step's copies overlap the neighbouring steps'
        compute; the caches and the workspace are shared (compute is serial)."""
        in_keys = ("q", "q_idx", "w_idx", "win", "block_cand", "block_logits")
        self.h_in = []
        for d in (self.csa, self.hcad):
            if d is None:
                continue
            for k in in_keys:
                if k in d:
                    self.h_in.append(torch.empty(d[k].shape, dtype=d[k].dtype, pin_memory=True).copy_(d[k].cpu()))
        self.sets = []
        for b in range(2):
            csa = dict(self.csa) if self.csa is not None else None
            hcad = dict(self.hcad) if self.hcad is not None else None
            if b == 0:
                outs = (self.idx, self.csa_out, self.hca_out)
            else:
                for d in (csa, hcad):
                    if d is not None:
                        for k in in_keys:
                            if k in d:
                                d[k] = d[k].clone()
                outs = tuple(None if t is None else torch.empty_like(t) for t in (self.idx, self.csa_out, self.hca_out))
            d_in = [d[k] for d in (csa, hcad) if d is not None for k in in_keys if k in d]
            d_out = [t for t in outs if t is not None]
            args, keep = self.hca.make_decode_args(self.B, self.q_pos, csa=csa, hca=hcad, csa_topk_idx=outs[0],
                                                   csa_out=outs[1], hca_out=outs[2], **self.norm_kw)
            self._apply_paged(args)
            h_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in d_out]
            self.sets.append({"args": args, "keep": (keep, csa, hcad, outs), "d_in": d_in, "d_out": d_out,
                              "h_out": h_out})
        self.h2d = sum(t.numel() * t.element_size() for t in self.h_in)
        self.d2h = sum(t.numel() * t.element_size() for t in self.sets[0]["h_out"])

    def run_set(self, b):
        self.hca.hybrid_attn_decode(self.cfg, self.sets[b]["args"], ws=self.ws)

    # --- CPU oracle on a bounded sample of requests ---
    def oracle_sample(self, n_req):
        import oracle
        s = self.shape
        t = self.ctx - 1
        spec = self.spec
        t0 = time.perf_counter()
        for b in range(n_req):
            if self.csa is not None:
                d = wl.csa_decode_inputs(s, 1, self.ctx, seed=900 + b, cache_std=spec["cache_std"])
                f = lambda x: x[0].float().numpy().astype(np.float64)  # noqa: E731
                if getattr(self, "indexer", "bf16") == "fp4":
                    nv = oracle.n_visible(t, s.m, d["E"].shape[1])
                    sc = oracle.indexer_scores_fp4(f(d["q_idx"]), d["w_idx"][0].double().numpy(), f(d["K_I"])[:nv])
                    sel = oracle.topk_select(sc, s.topk)
                    oracle.mqa_attend(f(d["q"]), np.concatenate([f(d["E"])[sel], f(d["win"])]), s.scale)
                else:
                    oracle.csa_layer_decode(f(d["E"]), f(d["K_I"]), f(d["win"]), f(d["q"]), f(d["q_idx"]),
                                            d["w_idx"][0].double().numpy(), t, m=s.m, topk=s.topk, n_win=s.n_win,
                                            scale=s.scale)
            if self.hcad is not None:
                wb = "block_cand" in self.hcad
                d = wl.hca_decode_inputs(s, 1, self.ctx, seed=900 + b, cache_std=spec["cache_std"], with_block=wb)
                f = lambda x: x[0].float().numpy().astype(np.float64)  # noqa: E731
                if wb:
                    oracle.hca_layer_decode(f(d["E_h"]), f(d["block_cand"]), f(d["block_logits"]),
                                            d["bias_hca"].double().numpy(), f(d["win"]), f(d["q"]), t,
                                            m_hca=s.m_hca, n_win=s.n_win, scale=s.scale)
                else:
                    oracle.mqa_attend(f(d["q"]), np.concatenate([f(d["E_h"]), f(d["win"])]), s.scale)
        return time.perf_counter() - t0


class PrefillBench:
    """CSA prefill of one 65,536-token sequence (compress, indexer + top-k, sparse MQA)."""

    def __init__(self, name, spec, seed, device, qk_norm=False):
        import long_context_attention_compress_b200 as hca
        self.hca = hca
        self.name = name
        s = self.shape = spec["shape"]
        T = self.T = spec["T"]
        self.norm_kw = {"csa_norm": wl.norm_weights(s, seed=seed, device=device)} if qk_norm else {}
        self.inp = wl.prefill_inputs(s, T, seed=seed, device=device, with_hca=False)
        dev = device
        Nc = T // s.m
        self.csa_kv = torch.empty((Nc, s.c), dtype=torch.bfloat16, device=dev)
        self.csa_k = torch.empty((Nc, s.d_idx), dtype=torch.bfloat16, device=dev)
        self.topk = torch.empty((T, s.topk), dtype=torch.int32, device=dev)
        self.out = torch.empty((T, s.n_heads, s.c), dtype=torch.bfloat16, device=dev)
        self.cfg = hca.make_cfg(s)
        self.phases = ["compress", "indexer_scores", "topk_select", "csa_attention"]
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(len(self.phases) + 1)]
        self.args, self._keep = hca.make_prefill_args(self.inp, self.csa_kv, self.csa_k, self.topk, self.out,
                                                      events=self.events, **self.norm_kw)
        self.ws = torch.empty(max(1, hca.hybrid_attn_prefill_workspace(self.cfg, self.args)), dtype=torch.uint8,
                              device=dev)
        self.units = T
        self.metric = "CSA prefill tokens/s at 64K"
        self.unit = "tokens/s"

    def step(self, record=True):
        self.args.n_events = len(self.events) if record else 0
        self.hca.hybrid_attn_prefill(self.cfg, self.args, ws=self.ws)

    def launches_per_step(self):
        return int(self.hca.lib.hca_last_launch_count())

    def flops(self):
        s, T = self.shape, self.T
        pairs = sum(min(s.topk, (t + 1) // s.m) + min(s.n_win, t + 1) for t in range(T))
        vis = sum((t + 1) // s.m for t in range(T))
        return {"indexer_scores": 2.0 * vis * s.n_idx_heads * s.d_idx,
                "csa_attention": 4.0 * pairs * s.n_heads * s.c}

    def phase_bytes(self):
        s, T = self.shape, self.T
        return {"compress": T * (2 * s.c + s.d_idx) * 2 + (T // s.m) * (s.c + s.d_idx) * 2}

    def config(self):
        s = self.shape
        return {"workload": self.name, "tokens": self.T, "c": s.c, "heads": s.n_heads, "topk": s.topk,
                "indexer": f"{s.n_idx_heads}x{s.d_idx}", "n_win": s.n_win}

    def e2e_setup(self):
        """Two device buffer sets of the per-step inputs and outputs (see DecodeBench)."""
        keys = ("cand", "logits", "kidx_cand", "q_idx", "w_idx", "q")
        self.h_in = [torch.empty(self.inp[k].shape, dtype=self.inp[k].dtype, pin_memory=True).copy_(self.inp[k].cpu())
                     for k in keys]
        self.sets = []
        for b in range(2):
            inp = dict(self.inp) if b == 0 else {k: (v.clone() if k in keys else v) for k, v in self.inp.items()}
            topk, out = (self.topk, self.out) if b == 0 else (torch.empty_like(self.topk), torch.empty_like(self.out))
            args, keep = self.hca.make_prefill_args(inp, self.csa_kv, self.csa_k, topk, out, **self.norm_kw)
            d_out = [topk, out]
            self.sets.append({"args": args, "keep": (keep, inp), "d_in": [inp[k] for k in keys], "d_out": d_out,
                              "h_out": [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in d_out]})
        self.h2d = sum(t.numel() * t.element_size() for t in self.h_in)
        self.d2h = sum(t.numel() * t.element_size() for t in self.sets[0]["h_out"])

    def run_set(self, b):
        self.hca.hybrid_attn_prefill(self.cfg, self.sets[b]["args"], ws=self.ws)

    def oracle_sample(self, n_q):
        import oracle
        s = self.shape
        T = self.T
        d = wl.prefill_inputs(s, T, seed=0, with_hca=False)
        f = lambda x: x.float().numpy().astype(np.float64)  # noqa: E731

        class Rows:  # float64 rows of a bf16 tensor, converted one query at a time
            def __init__(self, t):
                self.t = t

            def __getitem__(self, i):
                return self.t[i].float().numpy().astype(np.float64)
        qs = np.linspace(T // 2, T - 1, n_q).astype(int).tolist()
        t0 = time.perf_counter()
        oracle.csa_layer_prefill(f(d["cand"]), f(d["logits"]), f(d["kidx_cand"]), f(d["bias_csa"]),
                                 Rows(d["q_idx"]), d["w_idx"].double().numpy(), Rows(d["q"]), m=s.m, topk=s.topk,
                                 d_idx=s.d_idx, n_win=s.n_win, scale=s.scale, queries=qs)
        return time.perf_counter() - t0


def make_bench(name, seed, device, tokens=None, qk_norm=False, indexer="bf16", paged=False, kv_fp8=False):
    spec = wl.WORKLOADS[name]
    if qk_norm:
        name = f"{name}+qk_norm"  # the layer with Q/KV RMSNorm + partial RoPE (not the headline workload)
    if spec["kind"] == "prefill":
        if indexer != "bf16":
            raise SystemExit("--indexer fp4 is a decode variant")
        if tokens:
            # a shorter sequence of the same shape (profiling captures): not the headline workload
            spec = dict(spec, T=int(tokens))
            name = f"{name}_T{int(tokens)}"
        return PrefillBench(name, spec, seed, device, qk_norm)
    if indexer != "bf16":
        if spec["kind"] == "hca_decode":
            raise SystemExit("--indexer fp4 needs a CSA layer")
        name = f"{name}+fp4_indexer"  # the FP4 indexer variant (not the headline workload)
    if paged:
        if indexer != "bf16" or kv_fp8:
            raise SystemExit("--paged takes the bf16 indexer and bf16 caches")
        name = f"{name}+paged"  # the paged-cache variant (not the headline workload)
    if kv_fp8:
        name = f"{name}+kv_fp8"  # the FP8 KV-cache variant (not the headline workload)
    return DecodeBench(name, spec, seed, device, qk_norm, indexer=indexer, paged=paged, kv_fp8=kv_fp8)


def norm_prologue_roofline(bench, flush, pk, reps=20):
    """The Q/KV normaliser timed alone on the prefill's queries [T, H, c] (its
    largest launch): algorithmic bytes = one bf16 read and one bf16 write per element."""
    q = bench.inp["q"]
    w = bench.norm_kw["csa_norm"][0]
    out = torch.empty_like(q)
    st = torch.cuda.current_stream()
    ms = []
    for i in range(reps + 3):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        bench.hca.rms_norm_rope(q, w, bench.cfg, pos=bench.inp["q_pos"], out=out)
        e1.record(st)
        torch.cuda.synchronize()
        if i >= 3:
            ms.append(e0.elapsed_time(e1))
    avg = sum(ms) / len(ms)
    nbytes = 2 * q.numel() * 2
    ach = nbytes / (avg / 1e3) / 1e9
    return {"kernel": "norm_rope_kernel", "rows": int(q.shape[0] * q.shape[1]), "ms": round(avg, 4),
            "bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": round(ach / pk["hbm_gbs"], 4)}


# ----------------------------------------------------------------------------
# timing
# ----------------------------------------------------------------------------
def timed_steps(bench, K, flush, rank, ws, device, record=True):
    """Run K steps, each preceded by an L2 flush outside its events.
    Returns (total device ms, per-phase mean ms)."""
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    phase_ms = {p: 0.0 for p in bench.phases} if record else {}
    barrier(ws)
    torch.cuda.synchronize()
    for i in range(K):
        flush.zero_()
        starts[i].record()
        bench.step(record=record)
        ends[i].record()
        if record:
            torch.cuda.synchronize()
            for j, p in enumerate(bench.phases):
                phase_ms[p] += bench.events[j].elapsed_time(bench.events[j + 1])
    torch.cuda.synchronize()
    barrier(ws)
    total = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
    return total, {p: v / K for p, v in phase_ms.items()}


def e2e_pipelined(bench, K, device):
    """K steps through the C ABI, each with the host->device copy of its inputs
    from pinned memory and the device->host copy of its results, as a serving
    loop runs them: copies on their own streams (one per direction), two device
    buffer sets, so that step s+1's inputs arrive and step s-1's results leave
    while step s computes.  Returns device ms per step (first copy to last copy,
    CUDA events).  No L2 flush between steps: a step streams far more than the
    L2 holds (the indexer keys alone are 512 MiB at 1M context)."""
    main = torch.cuda.current_stream(device)
    h2d, d2h = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_ready, done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def load(s):
        b = s % 2
        with torch.cuda.stream(h2d):
            if s >= 2:
                h2d.wait_event(done[b])  # step s-2 has consumed this set's inputs
            for h, d in zip(bench.h_in, bench.sets[b]["d_in"]):
                d.copy_(h, non_blocking=True)
            in_ready[b].record(h2d)

    torch.cuda.synchronize(device)
    start.record(main)
    h2d.wait_event(start)
    load(0)
    for s in range(K):
        b = s % 2
        if s + 1 < K:
            load(s + 1)
        main.wait_event(in_ready[b])
        if s >= 2:
            main.wait_event(out_done[b])  # step s-2's results have left this set's outputs
        bench.run_set(b)
        done[b].record(main)
        with torch.cuda.stream(d2h):
            d2h.wait_event(done[b])
            for h, d in zip(bench.sets[b]["h_out"], bench.sets[b]["d_out"]):
                h.copy_(d, non_blocking=True)
            out_done[b].record(d2h)
    main.wait_stream(d2h)
    main.wait_stream(h2d)
    end.record(main)
    torch.cuda.synchronize(device)
    return start.elapsed_time(end) / K


def headline_region(bench, K, flush, rank, ws, device, local):
    """The headline timing: the K-step region (no host syncs inside), repeated
    until it has covered at least HEADLINE_MIN_S of wall time so that the clock
    sampler holds at least ~10 samples under load; the median repeat is the
    number.  A run whose clock record shows a hardware/thermal slowdown (or SM
    clocks stuck low with no reason) is taken once more, on every rank alike."""
    def once():
        totals = []
        with ClockSampler(local) as clk:
            t0 = time.perf_counter()
            while True:
                t, _ = timed_steps(bench, K, flush, rank, ws, device, record=False)
                totals.append(t)
                # every rank repeats the same number of times
                more = 1.0 if time.perf_counter() - t0 < HEADLINE_MIN_S else 0.0
                if reduce_max(more, ws, device) == 0.0:
                    break
        med = float(np.median(totals))
        return reduce_max(med, ws, device), dict(clk.summary(), region_repeats=len(totals))

    total_ms, clocks = once()
    if reduce_max(1.0 if clock_rejected(clocks) else 0.0, ws, device) > 0.0:
        first = clocks["reasons"] or ["sm clock %s of %s MHz" % (clocks["sm_mhz"], clocks["sm_max_mhz"])]
        total_ms, clocks = once()
        clocks = dict(clocks, remeasured_after=first)
    return total_ms, clocks


def roofline_of(bench, phase_ms, pk, sustained):
    """Roofline of the dominant phase: algorithmic bytes (or FLOPs) per launch over
    its event time, against the measured peak (and the datasheet's)."""
    dom = max(phase_ms, key=phase_ms.get) if phase_ms else None
    if dom is None:
        return None
    flops = bench.flops() if hasattr(bench, "flops") else {}
    bytes_ = bench.phase_bytes()
    dur_s = phase_ms[dom] / 1e3
    tt = traffic_table().get(dom)
    traffic = None
    if tt and tt.get("source_hash") == source_hash(tt.get("files", [])) and tt.get("workload") == bench.name:
        traffic = tt["dram_bytes_per_launch"]
    if dom in flops:
        ach = flops[dom] / dur_s / 1e12
        peak = pk["bf16_tflops_sustained"] if sustained else pk["bf16_tflops"]
        return {"bound": "tensor", "kernel": dom, "achieved": round(ach, 2), "peak": peak, "unit": "TFLOP/s",
                "frac": round(ach / peak, 4), "traffic": traffic, "peak_source": pk["source"],
                "peak_kind": "sustained" if sustained else "burst",
                "datasheet_peak": DATASHEET["bf16_tflops"], "frac_datasheet": round(ach / DATASHEET["bf16_tflops"], 4)}
    if dom in bytes_:
        ach = bytes_[dom] / dur_s / 1e9
        return {"bound": "hbm", "kernel": dom, "achieved": round(ach, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": round(ach / pk["hbm_gbs"], 4), "traffic": traffic, "peak_source": pk["source"],
                "datasheet_peak": DATASHEET["hbm_gbs"], "frac_datasheet": round(ach / DATASHEET["hbm_gbs"], 4)}
    return {"bound": "alu", "kernel": dom, "achieved": None, "peak": None, "unit": None, "frac": None,
            "traffic": traffic, "note": "selection kernel; no algorithmic HBM bytes"}


def whole_step_roofline(bench, ms, pk):
    """The whole step against the roofline its bound names: all algorithmic FLOPs
    (prefill) or bytes (decode) of the step over the step's time."""
    flops = bench.flops() if hasattr(bench, "flops") else {}
    if flops:
        ach = sum(flops.values()) / (ms / 1e3) / 1e12
        return {"bound": "tensor", "achieved": round(ach, 2), "unit": "TFLOP/s",
                "frac_burst": round(ach / pk["bf16_tflops"], 4),
                "frac_sustained": round(ach / pk["bf16_tflops_sustained"], 4),
                "frac_datasheet": round(ach / DATASHEET["bf16_tflops"], 4)}
    b = sum(bench.phase_bytes().values())
    ach = b / (ms / 1e3) / 1e9
    return {"bound": "hbm", "bytes": int(b), "achieved": round(ach, 1), "unit": "GB/s",
            "frac": round(ach / pk["hbm_gbs"], 4), "frac_datasheet": round(ach / DATASHEET["hbm_gbs"], 4)}


def measure(bench, a, steps, warmup, flush, rank, ws, device, local, cpu_sample):
    """Everything one workload reports: headline value, phases, rooflines, e2e,
    launches, clocks and (rank 0, one GPU) the CPU oracle baseline."""
    for _ in range(warmup):
        bench.step()
    torch.cuda.synchronize()
    launches = bench.launches_per_step()
    if steps is None:
        # default K: a timed region of about 2 s
        t0 = time.perf_counter()
        for _ in range(3):
            flush.zero_()
            bench.step(record=False)
        torch.cuda.synchronize()
        per = (time.perf_counter() - t0) / 3
        steps = int(min(20000, max(20, math.ceil(2.0 / max(per, 1e-6)))))
        steps = int(reduce_max(float(steps), ws, device))
    # phase breakdown pass (events between kernels, one sync per step)
    _, phase_ms = timed_steps(bench, min(steps, 50), flush, rank, ws, device, record=True)
    total_ms, clocks = headline_region(bench, steps, flush, rank, ws, device, local)
    ms = total_ms / steps
    value = bench.units * ws / (ms / 1e3)

    # end to end through the C ABI with host buffers
    bench.e2e_setup()
    e2e_pipelined(bench, 2, device)  # warm-up
    e2e_ms = reduce_max(e2e_pipelined(bench, steps, device), ws, device)
    e2e_value = bench.units * ws / (e2e_ms / 1e3)

    pk = peaks()
    prefill = isinstance(bench, PrefillBench)
    out = {"metric": bench.metric, "value": round(value, 2), "unit": bench.unit, "n_gpus": ws, "steps": steps,
           "warmup": warmup, "ms_per_step": round(ms, 4),
           "config": dict(bench.config(), parallelism=f"replicas x{ws} (requests sharded, no collective)",
                          l2="flushed before every timed step (256 MiB write, outside the step's events)"),
           "e2e": {"value": round(e2e_value, 2), "unit": bench.unit, "h2d_bytes_per_step": bench.h2d,
                   "d2h_bytes_per_step": bench.d2h, "ms_per_step": round(e2e_ms, 4),
                   "note": "every step copies its inputs from pinned host memory and its outputs back, on copy "
                           "streams that overlap the neighbouring steps' compute (two device buffer sets; no L2 "
                           "flush: a step streams more than the L2 holds); KV caches resident on the device"},
           "gpu_launches": launches * steps,
           "phase_ms": {k: round(v, 4) for k, v in phase_ms.items()},
           # a prefill step is long: its attention runs at the sustained (power-capped) rate
           "roofline": roofline_of(bench, phase_ms, pk, sustained=prefill),
           "step_roofline": whole_step_roofline(bench, ms, pk),
           "clocks": clocks}
    if a.qk_norm and prefill:
        out["qk_norm_prologue"] = norm_prologue_roofline(bench, flush, pk)
    if rank == 0 and ws == 1 and not a.no_cpu_baseline:
        import oracle  # noqa: F401  (timed baseline only)
        cores = len(os.sched_getaffinity(0))
        secs = bench.oracle_sample(cpu_sample)
        out["cpu_baseline"] = {"value": round(cpu_sample / secs, 4), "unit": bench.unit, "cores": cores,
                               "kind": "oracle",
                               "sample": f"{cpu_sample} {'queries' if bench.unit == 'tokens/s' else 'requests'} of "
                                         f"the same workload recipe through the float64 NumPy oracle ({secs:.1f} s)"}
    return out


def run_ours(a):
    rank, local, ws = init_dist("nccl")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    bench = make_bench(a.workload, shard_seed(a.seed, rank), device, tokens=a.tokens, qk_norm=a.qk_norm,
                       indexer=a.indexer, paged=a.paged, kv_fp8=a.kv_fp8)
    m = measure(bench, a, a.steps, a.warmup, flush, rank, ws, device, local, a.cpu_sample)
    out = {"metric": bench.metric, "value": m.pop("value"), "unit": m.pop("unit"), "n_gpus": ws,
           "steps": m.pop("steps"), "warmup": a.warmup, "ms_per_step": m.pop("ms_per_step"),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
           "data": "synthetic (seeded N(0,1)/U(0,1) tensors of the workload's shapes; caches drawn on the device)"}
    m.pop("metric")
    m.pop("n_gpus")
    m.pop("warmup")
    out.update(m)
    # The metric has two halves: decode queries/s (the headline) and prefill tokens/s.
    # The default run measures the 64K CSA prefill as well, in the same line.
    if (a.workload == DEFAULT_WORKLOAD and not a.no_prefill and a.tokens is None and a.indexer == "bf16"
            and not a.paged and not a.kv_fp8):
        del bench
        torch.cuda.empty_cache()
        pb = make_bench("csa_prefill_64k", shard_seed(a.seed, rank), device, qk_norm=a.qk_norm)
        # the prefill step is ~200x longer than a decode step: fewer steps cover as long a region
        psteps = a.prefill_steps if a.prefill_steps else max(3, min(20, a.steps or 20))
        pm = measure(pb, a, psteps, max(3, min(a.warmup, 5)), flush, rank, ws, device, local,
                     4 * a.cpu_sample)
        pm["workload"] = "csa_prefill_64k"
        out["prefill"] = pm
    if rank == 0:
        print(json.dumps(out), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def free_port() -> int:
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as so:
        so.bind(("127.0.0.1", 0))
        return so.getsockname()[1]


def spawn_ranks(n: int) -> int:
    """Re-run this command under torch.distributed.run with n ranks on this node
    (rendezvous on 127.0.0.1); returns the launcher's exit status."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={free_port()}", os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd)


def check_launch():
    """Start the process group (gloo without a GPU), agree on the world size with one
    collective, and print it from rank 0."""
    import datetime
    import torch.distributed as dist
    rank, local, ws = dist_env()
    if ws > 1:
        dist.init_process_group(backend="nccl" if torch.cuda.is_available() else "gloo",
                                timeout=datetime.timedelta(seconds=60))
        dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
        if dev.type == "cuda":
            torch.cuda.set_device(local)
        t = torch.ones(1, device=dev)
        dist.all_reduce(t)
        agreed = int(t.item())
        dist.destroy_process_group()
    else:
        agreed = 1
    if rank == 0:
        print(json.dumps({"check_launch": True, "world_size": ws, "ranks_agreed": agreed}), flush=True)


def run_reference(a):
    """Reference arm: the CPU oracle as it stands, on rank 0, bounded samples per step."""
    rank, local, ws = dist_env()
    if rank != 0:
        return
    os.environ.setdefault("OMP_NUM_THREADS", str(len(os.sched_getaffinity(0))))
    spec = wl.WORKLOADS[a.workload]
    cores = len(os.sched_getaffinity(0))

    class _Stub:
        pass
    if spec["kind"] == "prefill":
        b = PrefillBench.__new__(PrefillBench)
        b.shape, b.T, b.name = spec["shape"], spec["T"], a.workload
        unit, metric, per = "tokens/s", "CSA prefill tokens/s at 64K", 16
        conf = {"workload": a.workload, "tokens": b.T}
    else:
        b = DecodeBench.__new__(DecodeBench)
        b.shape, b.B, b.ctx, b.spec, b.name = spec["shape"], spec["B"], spec["ctx"], spec, a.workload
        b.csa = {} if spec["kind"] in ("hybrid_decode", "csa_decode") else None
        b.hcad = ({"block_cand": 1} if spec["kind"] == "hca_decode" else {}) if spec["kind"] in (
            "hybrid_decode", "hca_decode") else None
        unit, metric, per = "queries/s", "hybrid CSA+HCA decode queries/s at 1M ctx", 1
        conf = {"workload": a.workload, "batch": b.B, "context": b.ctx}
    for _ in range(a.warmup):
        b.oracle_sample(per)
    tot = 0.0
    for _ in range(a.steps):
        tot += b.oracle_sample(per)
    v = per * a.steps / tot
    out = {"impl": "reference", "metric": metric, "value": round(v, 4), "unit": unit, "n_gpus": ws, "steps": a.steps,
           "warmup": a.warmup, "ms_per_step": round(1e3 * tot / a.steps, 2), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": conf,
           "cpu_baseline": {"value": round(v, 4), "unit": unit, "cores": cores, "kind": "oracle",
                            "sample": f"{per} {'queries' if unit == 'tokens/s' else 'requests'} per step"},
           "e2e": {"value": round(v, 4), "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: enough for a ~2 s timed region)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="hybrid_decode_b8_1m", choices=[k for k in wl.WORKLOADS
                                                                          if k != "tiny_prefill_1k"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-sample", type=int, default=10,
                    help="requests (decode; the 64K prefill in the same line takes 4x as many queries) for the oracle")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--qk-norm", action="store_true",
                    help="the layer with Q/KV RMSNorm + partial RoPE (synthetic weights)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="prefill workloads: a shorter sequence of the same shape (for profiler captures)")
    ap.add_argument("--indexer", default="bf16", choices=["bf16", "fp4"],
                    help="fp4: the decode indexer over MXFP4 keys with BF16 scores (a variant, not the headline)")
    ap.add_argument("--kv-fp8", action="store_true",
                    help="decode workloads: the KV caches in FP8 form (E4M3 + bf16 rotary channels)")
    ap.add_argument("--paged", action="store_true",
                    help="decode workloads: the caches in paged form (blocks of 128 raw tokens, shuffled block table)")
    ap.add_argument("--no-prefill", action="store_true",
                    help="default workload only: skip the 64K prefill measured in the same line")
    ap.add_argument("--prefill-steps", type=int, default=None,
                    help="timed steps of the 64K prefill in the default run (default: min(20, --steps))")
    ap.add_argument("--check-launch", action="store_true",
                    help="start the ranks and report the world size only (tests of the launcher, no GPU work)")
    a = ap.parse_args()
    if a.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU: start the ranks here when not already under torchrun
        sys.exit(spawn_ranks(a.gpus))
    if a.check_launch:
        check_launch()
        return
    if a.warmup < 3:
        print("warning: fewer than 3 warm-up steps; the number is not a valid measurement", file=sys.stderr)
    if a.impl == "reference":
        a.steps = a.steps or 3
        run_reference(a)
    else:
        run_ours(a)


if __name__ == "__main__":
    main()

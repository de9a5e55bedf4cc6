#!/usr/bin/env python
"""Benchmark of quantized paged-KV attention on B200.

Headline (one JSON line on rank 0): decode at 131,072 context -- 16 layers x 4 KV heads x
head_dim 256, 24 query heads, 1 query token, Q8_0 K / Q4_0 V pages in a seeded shuffled page
table.  One step = for every layer: quantize-append the new token's K/V, then split-KV decode
(with its split-merge grid).  value = algorithmic KV bytes read per step (416 B per token, KV
head and layer) / device time per step, in GB/s.  The other workloads (the Q8_0/Q8_0,
Q4_0/Q4_0 and Q5_1/Q4_0 decodes, MTP verify at 262K with block selection, chunked prefill at
524K, host-streamed decode with and without resident-page reuse) are measured in the same run
and reported under "extra".

--impl reference times the CPU oracle (float64 NumPy) on the host cores on the same workload
and metric, each step a bounded sample of it.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from synth import WORKLOADS, derived_seed, np_rng, page_permutation, torch_normal, workload_layer_kv  # noqa: E402

METRIC = "quantized paged KV attention: decode HBM GB/s & prefill TFLOP/s vs roofline"
PAGE_BYTES = {("k", "q8_0"): 34816, ("k", "q4_0"): 18432, ("k", "q5_1"): 24576, ("k", "q5_0"): 22528,
              ("v", "q4_0"): 18432, ("v", "q8_0"): 34816, ("v", "q4_1"): 20480}


def bytes_per_token_head(k_fmt: str, v_fmt: str) -> int:
    """K + V bytes of one token of one KV head: 416 (Q8_0/Q4_0), 544 (Q8_0/Q8_0), 288 (Q4_0/Q4_0),
    416 (Q4_0/Q8_0), 336 (Q5_1/Q4_0), 464 (Q5_1/Q8_0), 336 (Q5_0/Q4_1)."""
    return (PAGE_BYTES[("k", k_fmt)] + PAGE_BYTES[("v", v_fmt)]) // 128


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extra", action="store_true", help="only the headline workload")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--extra-steps", type=int, default=100)
    ap.add_argument("--stream-steps", type=int, default=0,
                    help="decode steps of the host-streamed generation to time (0 = the workload's 512)")
    ap.add_argument("--prefill-layers", type=int, default=0, help="layers of the prefill workload (0 = 16)")
    ap.add_argument("--profile", choices=["none", "decode", "prefill", "prefill_f16", "verify", "stream"], default="none",
                    help="profiling only: run just this workload's steps (no JSON bench line)")
    ap.add_argument("--context", type=int, default=0, help="profiling only: prior-context override")
    ap.add_argument("--layers", type=int, default=0,
                    help="profiling only: override the layer count of the headline workload")
    return ap.parse_args()


# --------------------------------------------------------------------------- plumbing
KERNEL_SOURCES = {
    "decode_kernel_decode131k.md": ["common.cuh", "decode.cuh", "quantize.cu", "decode.cu"],
    "prefill_kernel_prefill65k.md": ["common.cuh", "tcgen05.cuh", "decode.cuh", "prefill.cu"],
}


def kernel_source_hash(files):
    import hashlib

    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "quantized_paged_kv_q4_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def profiled_traffic(summary):
    """DRAM bytes (read + write) per launch from the committed ncu summary, or None when the
    kernel's sources changed since those counters were taken."""
    try:
        vals = {}
        with open(os.path.join(ROOT, "profiles", summary)) as f:
            for line in f:
                if ":" in line and line.startswith(("traffic_bytes_per_launch", "source_sha256")):
                    k, v = line.split(":", 1)
                    vals[k.strip()] = v.strip().strip("`")
        if vals.get("source_sha256") != kernel_source_hash(KERNEL_SOURCES[summary]):
            return None
        return float(vals["traffic_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        # raw samples: $KVATTN_CLOCKS_DIR if set, else the temp directory; the summary goes into
        # the JSON line
        out_dir = os.environ.get("KVATTN_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out_dir, f"clocks_bench_{os.getpid()}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_init(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_step_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job rate: the units all ranks processed / the slowest rank's time per step."""
    return units_per_step_per_rank * world / (ms_max * 1e-3)


# --------------------------------------------------------------------------- caches
class DecodeCache:
    """All layers of one workload in device page pools, filled through quantize-append."""

    def __init__(self, kv, w, n_blocks_per_unit, tokens, device, with_needles=False, q_for_needles=None):
        import torch

        self.kv, self.w = kv, w
        L, H = w.layers, w.kv_heads
        self.L, self.H, self.nb = L, H, n_blocks_per_unit
        n_phys = L * H * n_blocks_per_unit
        kb = kv.kvattn_page_bytes(kv.ROLE_K, kv.FMT[w.k_fmt])
        vb = kv.kvattn_page_bytes(kv.ROLE_V, kv.FMT[w.v_fmt])
        self.k_pool = torch.empty((n_phys, kb), dtype=torch.uint8, device=device)
        self.v_pool = torch.empty((n_phys, vb), dtype=torch.uint8, device=device)
        self.k_pool.zero_()
        self.v_pool.zero_()
        rng = np_rng(w.seed, 1)
        perm = page_permutation(rng, n_phys).reshape(L, H, n_blocks_per_unit)
        self.page_table = torch.from_numpy(perm).to(device)        # [L][H][nb]
        self.desc = kv.make_desc(H, w.q_heads, self.k_pool, self.v_pool, n_phys, v_fmt=w.v_fmt, k_fmt=w.k_fmt)
        self.needles = {}
        for l in range(L):
            k, v, nd = workload_layer_kv(w, l, tokens, device, q_for_needles[l] if with_needles else None)
            for h, blocks in nd.items():
                self.needles[(l, h)] = blocks
            kv.kvattn_quantize_append(self.desc, k, v, tokens, 0, self.page_table[l], n_blocks_per_unit)
            del k, v
        torch.cuda.synchronize()


def event_pair():
    import torch

    return torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)


# --------------------------------------------------------------------------- decode workloads
class GraphStep:
    """One step's launches through the C ABI, optionally captured once as a CUDA graph and
    replayed: the same kernels on the same buffers, without the host's per-launch cost (a
    decode step is ~50 launches of ~50 us each)."""

    graph = None

    def launch_step(self):
        for l in range(self.w.layers):
            self.layer(l)

    def capture(self):
        import torch

        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self.launch_step()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.launch_step()
        torch.cuda.synchronize()
        self.graph = g

    def step(self):
        if self.graph is not None:
            self.graph.replay()
        else:
            self.launch_step()


class DecodeBench(GraphStep):
    def __init__(self, kv, wname, device, layers=0):
        import dataclasses

        import torch

        w = WORKLOADS[wname]
        if layers:
            w = dataclasses.replace(w, layers=layers)
        self.kv, self.w, self.device = kv, w, device
        self.ctx = w.context
        self.nb = (self.ctx + 127) // 128
        self.cache = DecodeCache(kv, w, self.nb, self.ctx, device)
        L, Hq, H = w.layers, w.q_heads, w.kv_heads
        self.q = torch_normal(derived_seed(w.seed, 20), (L, 1, Hq, 256), device)
        self.k_new = torch_normal(derived_seed(w.seed, 21), (L, 1, H, 256), device)
        self.v_new = torch_normal(derived_seed(w.seed, 22), (L, 1, H, 256), device)
        self.pos = self.ctx - 1                                   # the new token takes the last slot
        self.q_pos = torch.tensor([self.pos], dtype=torch.int32, device=device)
        self.out = torch.empty((L, 1, Hq, 256), device=device)
        self.lse = torch.empty((L, 1, Hq), device=device)
        self.ws_bytes = kv.kvattn_decode_workspace_size(self.cache.desc, 1, self.nb)
        self.ws = torch.zeros((L, max(self.ws_bytes, 256)), dtype=torch.uint8, device=device)
        self.bytes_per_layer = self.ctx * H * bytes_per_token_head(w.k_fmt, w.v_fmt)
        self.bytes_per_step = self.bytes_per_layer * L
        self.launches_per_step = 2 * L  # decode with the append fused in, split merge

    def layer(self, l):
        """One layer: append the new token and attend, as one kvattn_append_decode (its split
        grid, then the merge grid)."""
        kv, c = self.kv, self.cache
        kv.kvattn_append_decode(c.desc, self.k_new[l], self.v_new[l], 1, self.pos, c.page_table[l], self.nb,
                                self.q[l], 1, self.q_pos, c.page_table[l], None, None, self.nb, self.out[l],
                                self.lse[l], self.ws[l], self.ws_bytes)

    def split_grid(self, l):
        """The layer's decode split grid alone (the token already appended)."""
        c = self.cache
        self.kv.kvattn_decode_splits(c.desc, self.q[l], 1, self.q_pos, c.page_table[l], None, None, self.nb,
                                     self.out[l], self.lse[l], self.ws[l], self.ws_bytes)

    def merge_grid(self, l):
        self.kv.kvattn_decode_merge_splits(self.cache.desc, 1, self.nb, self.out[l], self.lse[l], self.ws[l],
                                           self.ws_bytes)


class VerifyBench(GraphStep):
    """MTP verify at 262,144 context: per layer, select 256 + 128 recent blocks (+ the tail
    page) with the block summaries, append the 4 verify tokens, decode n_q = 4 over the
    selected pages."""

    def __init__(self, kv, device, layers=0):
        import dataclasses

        import torch

        w = WORKLOADS["verify262k"]
        if layers:
            w = dataclasses.replace(w, layers=layers)
        self.kv, self.w = kv, w
        L, H, Hq, g = w.layers, w.kv_heads, w.q_heads, w.group
        self.n_full = w.context // 128
        self.nb = self.n_full + 1                                 # + the tail page of the new tokens
        self.q = torch_normal(derived_seed(w.seed, 20), (L, w.n_q, Hq, 256), device)
        self.cache = DecodeCache(kv, w, self.nb, w.context, device, with_needles=True, q_for_needles=self.q)
        c = self.cache
        self.summ = torch.zeros((L * H, self.nb, 256), device=device)
        kv.kvattn_block_summaries(c.desc, c.page_table.view(L * H, self.nb), L * H, self.nb, 0, self.n_full, self.summ)
        # retrieval query rows: the last verify token's query heads, grouped per KV head
        self.q_group = self.q[:, -1].reshape(L, H, g, 256).contiguous()
        self.cap = w.budget_blocks + w.recent_blocks + 1
        self.sel_l = torch.zeros((L, H, self.cap), dtype=torch.int32, device=device)
        self.sel_p = torch.zeros((L, H, self.cap), dtype=torch.int32, device=device)
        self.n_sel = torch.zeros((L, H), dtype=torch.int32, device=device)
        self.sws_bytes = kv.kvattn_select_workspace_size(H, self.nb)
        self.sws = torch.zeros(self.sws_bytes, dtype=torch.uint8, device=device)
        self.k_new = torch_normal(derived_seed(w.seed, 21), (L, w.n_q, H, 256), device)
        self.v_new = torch_normal(derived_seed(w.seed, 22), (L, w.n_q, H, 256), device)
        self.pos0 = w.context
        self.q_pos = torch.arange(self.pos0, self.pos0 + w.n_q, dtype=torch.int32, device=device)
        self.out = torch.empty((L, w.n_q, Hq, 256), device=device)
        self.lse = torch.empty((L, w.n_q, Hq), device=device)
        self.ws_bytes = kv.kvattn_decode_workspace_size(c.desc, w.n_q, self.cap)
        self.ws = torch.zeros((L, max(self.ws_bytes, 256)), dtype=torch.uint8, device=device)
        tokens = (w.budget_blocks + w.recent_blocks) * 128 + w.n_q
        self.bytes_per_layer = tokens * H * bytes_per_token_head(w.k_fmt, w.v_fmt)
        self.bytes_per_step = self.bytes_per_layer * L
        self.select_bytes_per_layer = H * (self.n_full - w.recent_blocks) * 256 * 4
        self.launches_per_step = 4 * L  # block scores, top-k, decode with the append fused in, split merge

    def layer(self, l):
        kv, c, w = self.kv, self.cache, self.w
        kv.kvattn_select_blocks(self.summ[l * w.kv_heads:(l + 1) * w.kv_heads], self.q_group[l], w.kv_heads, w.group,
                                self.nb, self.n_full, self.nb, w.budget_blocks, w.recent_blocks, c.page_table[l],
                                self.sel_l[l], self.sel_p[l], self.n_sel[l], self.cap, self.sws, self.sws_bytes)
        kv.kvattn_append_decode(c.desc, self.k_new[l], self.v_new[l], w.n_q, self.pos0, c.page_table[l], self.nb,
                                self.q[l], w.n_q, self.q_pos, self.sel_p[l], self.sel_l[l], self.n_sel[l],
                                self.cap, self.out[l], self.lse[l], self.ws[l], self.ws_bytes)

    def split_grid(self, l):
        """The layer's decode split grid alone, over the selection of the last step."""
        c, w = self.cache, self.w
        self.kv.kvattn_decode_splits(c.desc, self.q[l], w.n_q, self.q_pos, self.sel_p[l], self.sel_l[l],
                                     self.n_sel[l], self.cap, self.out[l], self.lse[l], self.ws[l], self.ws_bytes)

    def merge_grid(self, l):
        self.kv.kvattn_decode_merge_splits(self.cache.desc, self.w.n_q, self.cap, self.out[l], self.lse[l],
                                           self.ws[l], self.ws_bytes)


class PrefillBench:
    """Chunked prefill: a 2,048-token bf16 chunk (4 ubatches of 512) over 524,288 prior tokens,
    16 layers x 4 KV heads, 4,096-token KV splits.  One step = for every layer: append the
    chunk's K/V, then the four ubatch prefill calls."""

    def __init__(self, kv, device, layers=0, context=0, wname="prefill524k", f16=False):
        import dataclasses

        import torch

        w = WORKLOADS[wname]
        if layers:
            w = dataclasses.replace(w, layers=layers)
        if context:
            w = dataclasses.replace(w, context=context)
        self.kv, self.w = kv, w
        L, H, Hq = w.layers, w.kv_heads, w.q_heads
        self.total = w.context + w.n_q
        self.nb = (self.total + 127) // 128
        self.cache = DecodeCache(kv, w, self.nb, w.context, device)
        self.k_new = torch_normal(derived_seed(w.seed, 21), (L, w.n_q, H, 256), device)
        self.v_new = torch_normal(derived_seed(w.seed, 22), (L, w.n_q, H, 256), device)
        self.q = torch_normal(derived_seed(w.seed, 20), (L, w.n_q, Hq, 256), device).to(torch.bfloat16)
        self.q_bits = self.q.view(torch.int16)
        self.q_pos = torch.arange(w.context, self.total, dtype=torch.int32, device=device)
        self.out = torch.empty((L, w.n_q, Hq, 256), device=device)
        self.lse = torch.empty((L, w.n_q, Hq), device=device)
        self.ws_bytes = kv.kvattn_prefill_workspace_size(self.cache.desc, w.ubatch, self.nb, w.kv_split_tokens)
        self.ws = torch.zeros(max(self.ws_bytes, 256), dtype=torch.uint8, device=device)
        g = w.group
        self.flops_per_layer = 4.0 * Hq * 256 * (w.n_q * w.context + w.n_q * (w.n_q + 1) / 2)
        # tensor-core work per algorithmic flop: QK^T as two MMAs (K^ high and low parts) and PV
        # as three (P_hi V^_hi, P_lo V^_hi, P_hi V^_lo); one each with operands rounded once
        self.f16 = f16
        self.call = kv.kvattn_prefill_chunk_f16 if f16 else kv.kvattn_prefill_chunk
        self.mma_work_factor = 1.0 if f16 else (2 + 3) / 2
        self.flops_per_step = self.flops_per_layer * L
        self.launches_per_step = L * (1 + 2 * (w.n_q // w.ubatch))

    def layer(self, l, timed=None):
        kv, c, w = self.kv, self.cache, self.w
        kv.kvattn_quantize_append(c.desc, self.k_new[l], self.v_new[l], w.n_q, w.context, c.page_table[l], self.nb)
        if timed is not None:
            timed[0].record()
        for u in range(w.n_q // w.ubatch):
            a, b = u * w.ubatch, (u + 1) * w.ubatch
            self.call(c.desc, self.q_bits[l, a:b], w.ubatch, self.q_pos[a:b], c.page_table[l], None, None, self.nb,
                      w.kv_split_tokens, self.out[l, a:b], self.lse[l, a:b], self.ws, self.ws_bytes)
        if timed is not None:
            timed[1].record()

    def step(self):
        for l in range(self.w.layers):
            self.layer(l)


class StreamBench:
    """Host-streamed decode: the full 524,288-token cache of 16 layers x 4 KV heads sits in
    pinned host RAM (K|V interleaved per page).  A generation is `steps` decode steps (512)
    whose position advances by one each step.  Per step and layer the step's retrieval query
    selects 256 blocks per KV head among the prompt's full blocks, a copy kernel brings those
    pages into device slots on a side stream (layer L+1 while layer L decodes), the step's new
    token is quantize-appended into the generated-token pages (resident on the device: the
    generation reserve) and that page is written back to host RAM, and decode attends over the
    256 selected pages plus the generated-token pages so far."""

    PAGE = 34816 + 18432

    def __init__(self, kv, device, layers=0, context=0, steps=0):
        import dataclasses

        import torch

        w = WORKLOADS["stream524k"]
        if layers:
            w = dataclasses.replace(w, layers=layers)
        if context:
            w = dataclasses.replace(w, context=context)
        if steps:
            w = dataclasses.replace(w, steps=steps)
        self.kv, self.w, self.device = kv, w, device
        L, H, Hq, g = w.layers, w.kv_heads, w.q_heads, w.group
        self.n_full = w.context // 128
        self.n_tail = (w.context % 128 + w.steps + 127) // 128     # pages the generated tokens fill
        self.nb = self.n_full + self.n_tail
        self.budget = w.budget_blocks
        self.cap = self.budget + self.n_tail
        P = self.PAGE
        # ---- build: per layer on the device, then into pinned host RAM ----
        self.host = torch.empty((L * H * self.nb, P), dtype=torch.uint8).pin_memory()
        self.summ = torch.zeros((L * H, self.nb, 256), device=device)
        tmp = torch.zeros((H * self.nb, P), dtype=torch.uint8, device=device)
        tdesc = kv.make_desc(H, Hq, tmp, tmp.data_ptr() + 34816, H * self.nb, k_page_stride=P, v_page_stride=P)
        ttab = torch.arange(H * self.nb, dtype=torch.int32, device=device).view(H, self.nb)
        for l in range(L):
            k, v, _ = workload_layer_kv(w, l, w.context, device)
            tmp.zero_()
            kv.kvattn_quantize_append(tdesc, k, v, w.context, 0, ttab, self.nb)
            del k, v
            kv.kvattn_block_summaries(tdesc, ttab, H, self.nb, 0, self.n_full, self.summ[l * H:(l + 1) * H])
            self.host[l * H * self.nb:(l + 1) * H * self.nb].copy_(tmp)
        del tmp
        torch.cuda.synchronize()
        # host page ids per (layer, head, block)
        self.host_table = torch.arange(L * H * self.nb, dtype=torch.int32, device=device).view(L, H, self.nb)
        # ---- device slots: 2 buffers x H x budget streamed pages + L x H x n_tail resident pages
        # of the generated tokens ----
        self.n_stream_slots = 2 * H * self.budget
        self.n_slots = self.n_stream_slots + L * H * self.n_tail
        self.slots = torch.zeros((self.n_slots, P), dtype=torch.uint8, device=device)
        self.tail_slots = torch.tensor([[[self.n_stream_slots + (l * H + h) * self.n_tail + k for k in range(self.n_tail)]
                                         for h in range(H)] for l in range(L)], dtype=torch.int32, device=device)
        self.tail_hosts = self.host_table[:, :, self.n_full:].contiguous()
        # per (layer, generated-token page): the H host pages and device slots, contiguous
        self.tail_hosts_k = self.tail_hosts.permute(0, 2, 1).contiguous()
        self.tail_slots_k = self.tail_slots.permute(0, 2, 1).contiguous()
        self.reset()
        # the page copy runs on gather_ctas SMs beside the decode: the decode grid leaves them free
        self.gather_ctas = 16
        sms = torch.cuda.get_device_properties(device).multi_processor_count
        self.desc = kv.make_desc(H, Hq, self.slots, self.slots.data_ptr() + 34816, self.n_slots, k_page_stride=P,
                                 v_page_stride=P, sm_budget=sms - self.gather_ctas)
        # per buffer: gather destinations (-1 for the generated-token entries) and the decode page lists
        self.dst = []
        self.plist = []
        for b in range(2):
            base = b * H * self.budget
            self.dst.append(torch.tensor([[base + h * self.budget + i if i < self.budget else -1 for i in range(self.cap)]
                                          for h in range(H)], dtype=torch.int32, device=device))
        for l in range(L):
            b = l % 2
            base = b * H * self.budget
            self.plist.append(torch.tensor([[base + h * self.budget + i if i < self.budget
                                             else int(self.tail_slots[l, h, i - self.budget]) for i in range(self.cap)]
                                            for h in range(H)], dtype=torch.int32, device=device))
        # append page table: logical block n_full + k -> generated-token slot k of the unit
        self.tail_tab = torch.zeros((L, H, self.nb), dtype=torch.int32, device=device)
        self.tail_tab[:, :, self.n_full:] = self.tail_slots
        # selection outputs and workspaces
        self.sel_l = torch.zeros((L, H, self.cap), dtype=torch.int32, device=device)
        self.sel_p = torch.zeros((L, H, self.cap), dtype=torch.int32, device=device)
        self.n_sel = torch.zeros((L, H), dtype=torch.int32, device=device)
        self.sws_bytes = kv.kvattn_select_workspace_size(H, self.nb)
        self.sws = torch.zeros((L, self.sws_bytes), dtype=torch.uint8, device=device)
        self.ws_bytes = kv.kvattn_decode_workspace_size(self.desc, 1, self.cap)
        self.ws = torch.zeros((L, max(self.ws_bytes, 256)), dtype=torch.uint8, device=device)
        # per-step inputs of the whole generation: query, new K and V of every step and layer
        S = w.steps
        self.q_all = torch_normal(derived_seed(w.seed, 20), (S, L, 1, Hq, 256), device)
        self.qg_all = self.q_all[:, :, 0].reshape(S, L, H, g, 256).contiguous()
        self.k_all = torch_normal(derived_seed(w.seed, 21), (S, L, 1, H, 256), device)
        self.v_all = torch_normal(derived_seed(w.seed, 22), (S, L, 1, H, 256), device)
        self.pos_all = torch.arange(w.context, w.context + S, dtype=torch.int32, device=device)
        # step 0's views, kept for the fixed-position subclass
        self.q, self.q_group, self.k_new, self.v_new = self.q_all[0], self.qg_all[0], self.k_all[0], self.v_all[0]
        self.pos = w.context
        self.q_pos = self.pos_all[:1]
        self.out = torch.empty((L, 1, Hq, 256), device=device)
        self.lse = torch.empty((L, 1, Hq), device=device)
        self.copy_stream = torch.cuda.Stream(device=device)
        self.ev_sel = [torch.cuda.Event() for _ in range(L)]
        self.ev_copy = [torch.cuda.Event() for _ in range(L)]
        self.ev_dec = [torch.cuda.Event() for _ in range(L)]
        self.copy_bytes_per_step = L * H * self.budget * P
        self.launches_per_step = 6 * L  # scores, top-k, copy, decode with the append (+ merge), write-back

    def reset(self):
        """Back to the first step of the generation: the generated-token pages hold the prompt's
        partial tail (if any), as in host RAM before the generation."""
        L, H = self.w.layers, self.w.kv_heads
        self.gen_t = 0
        self.slots[self.n_stream_slots:].zero_()
        if self.w.context % 128:
            for l in range(L):
                for h in range(H):
                    self.slots[int(self.tail_slots[l, h, 0])].copy_(self.host[(l * H + h) * self.nb + self.n_full])

    def attn_bytes(self, t):
        """Quantized KV bytes the decode launches of step t read (all layers)."""
        w = self.w
        tokens = self.budget * 128 + w.context % 128 + t + 1
        return w.layers * w.kv_heads * tokens * bytes_per_token_head(w.k_fmt, w.v_fmt)

    def _n_total(self):
        """Blocks of the unit so far: the prompt's full blocks and the generated-token pages."""
        return self.n_full + (self.w.context % 128 + self.gen_t) // 128 + 1

    def _select(self, l):
        w, t = self.w, self.gen_t
        self.kv.kvattn_select_blocks(self.summ[l * w.kv_heads:(l + 1) * w.kv_heads], self.qg_all[t, l], w.kv_heads,
                                     w.group, self.nb, self.n_full, self._n_total(), self.budget, 0,
                                     self.host_table[l], self.sel_l[l], self.sel_p[l], self.n_sel[l], self.cap,
                                     self.sws[l], self.sws_bytes)

    def _gather(self, l, stream):
        H = self.w.kv_heads
        self.kv.kvattn_gather_pages(self.host, self.PAGE, self.host.shape[0], self.slots, self.PAGE, self.n_slots,
                                    self.PAGE, self.sel_p[l], self.dst[l % 2], H * self.cap, self.gather_ctas,
                                    stream)

    def _attend(self, l, timed=None):
        kv, w, t = self.kv, self.w, self.gen_t
        pos = w.context + t
        if timed is None:
            kv.kvattn_append_decode(self.desc, self.k_all[t, l], self.v_all[t, l], 1, pos, self.tail_tab[l], self.nb,
                                    self.q_all[t, l], 1, self.pos_all[t:t + 1], self.plist[l], self.sel_l[l],
                                    self.n_sel[l], self.cap, self.out[l], self.lse[l], self.ws[l], self.ws_bytes)
        else:
            kv.kvattn_quantize_append(self.desc, self.k_all[t, l], self.v_all[t, l], 1, pos, self.tail_tab[l],
                                      self.nb)
            timed[0].record()
            kv.kvattn_decode(self.desc, self.q_all[t, l], 1, self.pos_all[t:t + 1], self.plist[l], self.sel_l[l],
                             self.n_sel[l], self.cap, self.out[l], self.lse[l], self.ws[l], self.ws_bytes)
            timed[1].record()
        k = (w.context % 128 + t) // 128     # the generated-token page the token went to
        kv.kvattn_scatter_pages(self.host, self.PAGE, self.host.shape[0], self.slots, self.PAGE, self.n_slots,
                                self.PAGE, self.tail_hosts_k[l, k], self.tail_slots_k[l, k], w.kv_heads, 4)

    def step(self, stream_pages=True, timed=None):
        """One decode step of all layers at the current position; the position then advances
        (after the last step of the generation it stays there)."""
        import torch

        L = self.w.layers
        main = torch.cuda.current_stream()
        cs = self.copy_stream
        self._select(0)
        self.ev_sel[0].record(main)
        if stream_pages:
            cs.wait_event(self.ev_sel[0])
            self._gather(0, cs)
            self.ev_copy[0].record(cs)
        for l in range(L):
            if l + 1 < L:
                self._select(l + 1)
                self.ev_sel[l + 1].record(main)
                if stream_pages:
                    cs.wait_event(self.ev_sel[l + 1])
                    if l >= 1:
                        cs.wait_event(self.ev_dec[l - 1])  # buffer (l+1)%2 was read by layer l-1
                    self._gather(l + 1, cs)
                    self.ev_copy[l + 1].record(cs)
            if stream_pages:
                main.wait_event(self.ev_copy[l])
            self._attend(l, timed[l] if timed is not None else None)
            self.ev_dec[l].record(main)
        self.gen_t = min(self.gen_t + 1, self.w.steps - 1)

    def copies_only(self):
        import torch

        cs = torch.cuda.current_stream()
        for l in range(self.w.layers):
            self._gather(l, cs)


class ResidentStreamBench(StreamBench):
    """The streamed step with resident-page reuse: every (layer, KV head) keeps a pool of 256
    device slots across steps; per layer, kvattn_resident_update maps the new selection onto
    the pool and only the misses cross PCIe (layer L+1's on the side stream while layer L
    decodes).  `queries` per-step retrieval queries are cycled: 1 = the per-turn query KVMem
    uses (the working set is fixed during a turn), more = a drifting query."""

    def __init__(self, kv, device, queries=1, drift=0.0, layers=0, context=0):
        import torch

        super().__init__(kv, device, layers=layers, context=context, steps=1)
        w, L, H = self.w, self.w.layers, self.w.kv_heads
        self.units = L * H
        self.n_res = self.units * self.budget                 # resident pool pages, then the tails
        P = self.PAGE
        self.slots = torch.zeros((self.n_res + self.units, P), dtype=torch.uint8, device=device)
        for l in range(L):
            for h in range(H):
                self.slots[self.n_res + l * H + h].copy_(self.host[(l * H + h) * self.nb + self.n_full])
        self.n_slots = self.slots.shape[0]
        sms = torch.cuda.get_device_properties(device).multi_processor_count
        self.desc = kv.make_desc(H, w.q_heads, self.slots, self.slots.data_ptr() + 34816, self.n_slots,
                                 k_page_stride=P, v_page_stride=P, sm_budget=sms - self.gather_ctas)
        self.tail_slot = torch.tensor([[self.n_res + l * H + h for h in range(H)] for l in range(L)],
                                      dtype=torch.int32, device=device)
        self.tail_tab = self.tail_slot[:, :, None].expand(L, H, self.nb).contiguous()
        self.tail_host = self.tail_hosts[:, :, 0].contiguous()
        self.sob = torch.full((self.units, self.nb), -1, dtype=torch.int32, device=device)
        self.bos = torch.full((self.units, self.budget), -1, dtype=torch.int32, device=device)
        self.plist_r = torch.zeros((L, H, self.cap), dtype=torch.int32, device=device)
        self.copy_host = torch.zeros((L, H, self.cap), dtype=torch.int32, device=device)
        self.copy_dst = torch.full((L, H, self.cap), -1, dtype=torch.int32, device=device)
        self.n_copies = torch.zeros((L, H), dtype=torch.int32, device=device)
        # per-step retrieval queries: q_0 = the workload's, q_t = q_{t-1} + drift * N(0, 1)
        qs = [self.q]
        for t in range(1, queries):
            qs.append(qs[-1] + drift * torch_normal(derived_seed(w.seed, 30, t), tuple(self.q.shape), device))
        self.qs = [q.contiguous() for q in qs]
        self.qgs = [q[:, 0].reshape(L, H, w.group, 256).contiguous() for q in qs]
        self.t = 0

    def _select(self, l):
        w, H = self.w, self.w.kv_heads
        qg = self.qgs[self.t % len(self.qgs)]
        self.kv.kvattn_select_blocks(self.summ[l * H:(l + 1) * H], qg[l], H, w.group, self.nb, self.n_full, self.nb,
                                     self.budget, 0, self.host_table[l], self.sel_l[l], self.sel_p[l], self.n_sel[l],
                                     self.cap, self.sws[l], self.sws_bytes)
        self.kv.kvattn_resident_update(self.sel_l[l], self.n_sel[l], self.cap, H, self.nb, self.n_full,
                                       self.sob[l * H:(l + 1) * H], self.bos[l * H:(l + 1) * H], self.budget,
                                       self.host_table[l], l * H * self.budget, self.tail_slot[l], self.plist_r[l],
                                       self.copy_host[l], self.copy_dst[l], self.n_copies[l])

    def _gather(self, l, stream):
        H = self.w.kv_heads
        self.kv.kvattn_gather_pages(self.host, self.PAGE, self.host.shape[0], self.slots, self.PAGE, self.n_slots,
                                    self.PAGE, self.copy_host[l], self.copy_dst[l], H * self.cap, self.gather_ctas,
                                    stream)

    def _attend(self, l, timed=None):
        kv, w = self.kv, self.w
        q = self.qs[self.t % len(self.qs)]
        kv.kvattn_quantize_append(self.desc, self.k_new[l], self.v_new[l], 1, self.pos, self.tail_tab[l], self.nb)
        kv.kvattn_decode(self.desc, q[l], 1, self.q_pos, self.plist_r[l], self.sel_l[l], self.n_sel[l], self.cap,
                         self.out[l], self.lse[l], self.ws[l], self.ws_bytes)
        kv.kvattn_scatter_pages(self.host, self.PAGE, self.host.shape[0], self.slots, self.PAGE, self.n_slots,
                                self.PAGE, self.tail_host[l], self.tail_slot[l], w.kv_heads, 4)

    def step(self, stream_pages=True, timed=None):
        super().step(stream_pages, timed)
        self.t += 1

    def copies_per_step(self, steps):
        """Pages copied per step over `steps` steps (read back after each; untimed)."""
        import torch

        n = []
        for _ in range(steps):
            self.step()
            torch.cuda.synchronize()
            n.append(int(self.n_copies.sum()))
        return n


def time_stream(b, steps, warmup):
    """A generation of `steps` advancing decode steps, pipelined (T_stream per step); the same
    steps without page copies (T_resident), the copies alone (T_copy), and the decode launches
    of one step.  Warm-up steps run first and the generation then restarts at its first step."""
    import torch

    def timed(fn, n):
        torch.cuda.synchronize()
        e0, e1 = event_pair()
        e0.record()
        for _ in range(n):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    b.reset()
    for _ in range(warmup):
        b.step(True)
    b.reset()
    t_stream = timed(lambda: b.step(True), steps)
    short = min(steps, 32)
    b.reset()
    t_res = timed(lambda: b.step(False), short)
    t_copy = timed(b.copies_only, short)
    b.reset()
    pairs = [event_pair() for _ in range(b.w.layers)]
    b.step(True, timed=pairs)
    torch.cuda.synchronize()
    t_dec = sum(a.elapsed_time(c) for a, c in pairs)
    b.reset()
    return t_stream, t_res, t_copy, t_dec


def time_memcpy_route(b):
    """The same step's page copies through kvattn_stream_pages (one cudaMemcpyAsync per run of
    consecutive pages, page ids on the host): device time of the copies and host enqueue time."""
    import torch

    L, H = b.w.layers, b.w.kv_heads
    for l in range(L):
        b._select(l)
    sel = b.sel_p.cpu().numpy()
    cs = b.copy_stream
    e0, e1 = event_pair()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    e0.record(cs)
    n_copies = 0
    for l in range(L):
        base = (l % 2) * H * b.budget
        hid = sel[l, :, :b.budget].reshape(-1)
        slots = base + np.arange(H * b.budget, dtype=np.int32)
        n_copies += b.kv.kvattn_stream_pages(b.host, b.PAGE, b.slots, b.PAGE, b.PAGE, hid, slots, copy_stream=cs)
    e1.record(cs)
    t_enq = time.perf_counter() - t0
    torch.cuda.synchronize()
    return e0.elapsed_time(e1), t_enq * 1e3, n_copies


def time_steps(bench, steps, warmup, world):
    import torch

    for _ in range(warmup):
        bench.step()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = event_pair()
    torch.cuda.nvtx.range_push(f"timed_steps_{bench.w.name}")  # lets ncu select exactly these launches
    e0.record()
    for _ in range(steps):
        bench.step()
    e1.record()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    barrier(world)
    ms = e0.elapsed_time(e1) / steps
    return max_over_ranks(ms, world)


def time_kernel(bench, steps):
    """Average device duration of one launch of the decode split grid and of its merge grid.
    Each kind is captured as a CUDA graph of its launches for every layer, back to back on one
    stream (programmatic dependent launch, as in the step), and replayed `steps` times between
    two events on that stream; the duration is the elapsed time / launches.  The grids run on
    the state the preceding full steps left (pages with the token appended, selections)."""
    import torch

    out = []
    for grid in (bench.split_grid, bench.merge_grid):
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for l in range(bench.w.layers):
                grid(l)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for l in range(bench.w.layers):
                grid(l)
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = event_pair()
        e0.record()
        for _ in range(steps):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        out.append(e0.elapsed_time(e1) / (steps * bench.w.layers))
        del g
    return out[0], out[1]


def time_layers(bench, steps):
    """Average device duration of one layer's prefill calls (events before and after them)."""
    import torch

    pairs = []
    for _ in range(steps):
        for l in range(bench.w.layers):
            p = event_pair()
            bench.layer(l, timed=p)
            pairs.append(p)
    torch.cuda.synchronize()
    return statistics.mean(a.elapsed_time(b) for a, b in pairs)


def time_e2e(bench, steps, warmup):
    """Same step with the per-step inputs in pinned host memory: H2D copies of q and the new
    K/V and a D2H copy of the outputs are inside the timed region."""
    import torch

    hq = bench.q.cpu().pin_memory()
    hk = bench.k_new.cpu().pin_memory()
    hv = bench.v_new.cpu().pin_memory()
    ho = torch.empty(bench.out.shape, dtype=torch.float32).pin_memory()
    hl = torch.empty(bench.lse.shape, dtype=torch.float32).pin_memory()

    def one():
        bench.q.copy_(hq, non_blocking=True)
        bench.k_new.copy_(hk, non_blocking=True)
        bench.v_new.copy_(hv, non_blocking=True)
        bench.launch_step()  # the C-ABI calls themselves, no graph
        ho.copy_(bench.out, non_blocking=True)
        hl.copy_(bench.lse, non_blocking=True)

    for _ in range(warmup):
        one()
    torch.cuda.synchronize()
    e0, e1 = event_pair()
    e0.record()
    for _ in range(steps):
        one()
    e1.record()
    torch.cuda.synchronize()
    h2d = (hq.numel() + hk.numel() + hv.numel()) * 4
    d2h = (ho.numel() + hl.numel()) * 4
    return e0.elapsed_time(e1) / steps, h2d, d2h


# --------------------------------------------------------------------------- CPU oracle
_ORACLE_INPUTS = {}


def _oracle_inputs(wname, n_tokens):
    """Seeded codes for one (layer, KV head) unit, quantised by the oracle (untimed setup)."""
    from oracle import quant as oq

    key = (wname, n_tokens)
    if key not in _ORACLE_INPUTS:
        w = WORKLOADS[wname]
        rng = np_rng(w.seed, 99)
        k = rng.standard_normal((n_tokens, 256), dtype=np.float32)
        v = rng.standard_normal((n_tokens, 256), dtype=np.float32)
        q = rng.standard_normal((w.group, 256), dtype=np.float32)
        _ORACLE_INPUTS.clear()
        _ORACLE_INPUTS[key] = (q, oq.quantize(k, w.k_fmt), oq.quantize(v, w.v_fmt))
    return _ORACLE_INPUTS[key]


def _blas_threads():
    """Threads the oracle can use: numpy's BLAS pool runs the contractions; the elementwise
    steps run on one thread."""
    try:
        from threadpoolctl import threadpool_info

        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def oracle_decode_sample(wname, n_tokens, reps_min_s=10.0, max_reps=200):
    """Times the oracle (dequantise + float64 attention) on one (layer, KV head) unit and
    the last n_tokens of the workload's context, repeated until reps_min_s seconds of CPU
    work have been timed.  Returns (GB/s, seconds per repetition, threads, sample)."""
    from oracle import attention as oatt
    from oracle import quant as oq

    w = WORKLOADS[wname]
    q, (kc, kd), (vc, vd) = _oracle_inputs(wname, n_tokens)
    pos = np.arange(w.context - n_tokens, w.context)
    t_total, reps = 0.0, 0
    while reps < max_reps and (reps == 0 or t_total < reps_min_s):
        t0 = time.perf_counter()
        kh = oq.dequantize(kc, kd, w.k_fmt)
        vh = oq.dequantize(vc, vd, w.v_fmt)
        oatt.attend(q, kh, vh, pos, np.full(w.group, w.context - 1), 1.0 / 16)
        t_total += time.perf_counter() - t0
        reps += 1
    secs = t_total / reps
    gbs = n_tokens * bytes_per_token_head(w.k_fmt, w.v_fmt) / secs / 1e9
    threads = _blas_threads()
    sample = (f"1 of {w.layers * w.kv_heads} (layer, KV head) units, {n_tokens} of {w.context} tokens, "
              f"{w.group} query heads, timed {reps} times ({t_total:.1f} s of CPU work)")
    return gbs, secs, threads, sample


def reference_arm(args, world, rank):
    if world > 1 and rank != 0:
        return
    w = WORKLOADS["decode131k"]
    # size the per-step sample so that warmup + steps take about two minutes
    probe_tokens = 8192
    gbs, secs, threads, _ = oracle_decode_sample("decode131k", probe_tokens, 0.0, 1)
    budget_s = 120.0 / max(1, args.steps + args.warmup)
    n_tok = int(max(1024, min(w.context, probe_tokens * budget_s / max(secs, 1e-6))) // 128 * 128)
    times = []
    for i in range(args.warmup + args.steps):
        g, s, threads, sample = oracle_decode_sample("decode131k", n_tok, 0.0, 1)
        if i >= args.warmup:
            times.append(s)
    secs = statistics.mean(times)
    value = n_tok * bytes_per_token_head(w.k_fmt, w.v_fmt) / secs / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "decode131k", "layers": w.layers, "kv_heads": w.kv_heads, "q_heads": w.q_heads,
                   "context": w.context, "n_q": 1, "k_fmt": w.k_fmt, "v_fmt": w.v_fmt},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": len(os.sched_getaffinity(0)), "blas_threads": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- main
def main():
    args = parse_args()
    world, rank, local = dist_init(args)
    if args.impl == "reference":
        reference_arm(args, world, rank)
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()
        return

    import torch

    from quantized_paged_kv_q4_b200 import build, kvattn

    build.build()
    torch.cuda.set_device(local)
    kvattn.kvattn_init(local)
    device = torch.device("cuda", local)
    hbm, bf16, bf16_sus, peak_kind = peaks()

    if args.profile != "none":
        # a short run of one workload for ncu captures; prints no bench line
        if args.profile == "decode":
            b = DecodeBench(kvattn, "decode131k", device, layers=args.layers or 2)
        elif args.profile == "verify":
            b = VerifyBench(kvattn, device, layers=args.layers or 2)
        elif args.profile == "stream":
            b = StreamBench(kvattn, device, layers=args.layers or 2, context=args.context)
        else:
            b = PrefillBench(kvattn, device, layers=args.layers or 1, context=args.context,
                             f16=args.profile == "prefill_f16")
        for _ in range(args.warmup + args.steps):
            b.step()
        torch.cuda.synchronize()
        assert kvattn.kvattn_device_error() == 0
        print(json.dumps({"profiling_run": args.profile, "steps": args.steps, "warmup": args.warmup}))
        return

    # ---------------- headline: decode at 131K ----------------
    b = DecodeBench(kvattn, "decode131k", device, layers=args.layers)
    launch_mode = "one CUDA graph per step (2 launches per layer: kvattn_append_decode's two grids, programmatic dependent launch)"
    try:
        b.capture()
    except Exception as exc:  # report and time the direct launches instead
        launch_mode = f"direct launches (graph capture failed: {exc!r})"
    # clocks are sampled over the whole headline section: warm-up, timed steps, the per-grid
    # timing and the end-to-end steps
    clocks = ClockSampler(local)
    clocks.start()
    ms = time_steps(b, args.steps, args.warmup, world)
    kern_ms, merge_ms = time_kernel(b, max(3, min(args.steps, 50)))
    e2e_ms, h2d, d2h = time_e2e(b, max(3, min(args.steps, 200)), 3)
    clk = clocks.stop()
    assert kvattn.kvattn_device_error() == 0
    value = job_throughput(b.bytes_per_step, world, ms) / 1e9
    achieved = b.bytes_per_layer / (kern_ms * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16 MMA (exact hi+lo f16 operands), f32 accumulate", "data": "synthetic",
        "config": {"workload": "decode131k", "layers": b.w.layers, "kv_heads": b.w.kv_heads,
                   "q_heads": b.w.q_heads, "context": b.ctx, "n_q": 1, "k_fmt": "q8_0", "v_fmt": "q4_0",
                   "outliers": "1% of channels x8", "parallelism": f"{world} independent decodes (one per GPU)",
                   "l2": "inputs larger than L2 (218 MB of KV per layer launch, 3.49 GB per step)",
                   "launch": launch_mode},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                     "traffic": profiled_traffic("decode_kernel_decode131k.md"),
                     "kernel": ("decode_kernel<Q8_0 K, Q4_0 V, 8 rows>: the split grid alone, one launch per "
                                "layer back to back in a CUDA graph"),
                     "peak_kind": f"{peak_kind} copy bandwidth (hbm_gbs)",
                     "algorithmic_bytes_per_launch": b.bytes_per_layer, "avg_launch_ms": kern_ms,
                     "merge_grid_ms": merge_ms, "step_ms_per_layer": ms / b.w.layers,
                     "step_frac": value / world / hbm},
        "e2e": {"value": b.bytes_per_step * world / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": b.launches_per_step * args.steps,
        "clocks": clk,
    }
    if args.layers:
        line["profiling_run"] = f"layers overridden to {args.layers}: not a bench value"
    del b
    torch.cuda.empty_cache()

    # ---------------- the other workloads ----------------
    extra = {}
    if not args.no_extra:
        try:
            # the same decode step over the other KV format pairs
            for wn in ("decode131k_q8q8", "decode131k_q4q4", "decode131k_q4q8", "decode131k_q51q4",
                       "decode131k_q51q8", "decode131k_q50q41"):
                b2 = DecodeBench(kvattn, wn, device)
                b2.capture()
                ms2 = time_steps(b2, args.extra_steps, 5, world)
                k2, m2 = time_kernel(b2, 10)
                extra[wn] = {"GB/s": b2.bytes_per_step / (ms2 * 1e-3) / 1e9, "ms_per_step": ms2,
                             "kernel_GB/s": b2.bytes_per_layer / (k2 * 1e-3) / 1e9,
                             "kernel_frac_hbm": b2.bytes_per_layer / (k2 * 1e-3) / 1e9 / hbm,
                             "kernel_ms": k2, "merge_ms": m2, "k_fmt": b2.w.k_fmt, "v_fmt": b2.w.v_fmt,
                             "bytes_per_token_head": bytes_per_token_head(b2.w.k_fmt, b2.w.v_fmt)}
                del b2
                torch.cuda.empty_cache()
            b3 = VerifyBench(kvattn, device)
            b3.capture()
            ms3 = time_steps(b3, args.extra_steps, 5, world)
            k3, m3 = time_kernel(b3, 10)
            extra["verify262k"] = {"GB/s": b3.bytes_per_step / (ms3 * 1e-3) / 1e9, "ms_per_step": ms3,
                                   "decode_kernel_GB/s": b3.bytes_per_layer / (k3 * 1e-3) / 1e9,
                                   "decode_kernel_frac_hbm": b3.bytes_per_layer / (k3 * 1e-3) / 1e9 / hbm,
                                   "decode_kernel_ms": k3, "merge_ms": m3,
                                   "selected_tokens_per_unit": (b3.w.budget_blocks + b3.w.recent_blocks) * 128 + 4}
            del b3
            torch.cuda.empty_cache()
            b4 = PrefillBench(kvattn, device, layers=args.prefill_layers)
            ms4 = time_steps(b4, max(1, args.extra_steps // 50), 1, world)
            k4 = time_layers(b4, 1)
            tf = b4.flops_per_layer / (k4 * 1e-3) / 1e12
            extra["prefill524k"] = {"TFLOP/s": b4.flops_per_step / (ms4 * 1e-3) / 1e12, "ms_per_step": ms4,
                                    "layers": b4.w.layers, "kernel_TFLOP/s": tf, "kernel_frac_bf16": tf / bf16,
                                    "kernel_frac_bf16_sustained": tf / bf16_sus,
                                    "layer_ms": k4, "flop_per_layer": b4.flops_per_layer,
                                    "executed_TFLOP/s": tf * b4.mma_work_factor,
                                    "executed_frac_bf16": tf * b4.mma_work_factor / bf16,
                                    "mma_work_factor": b4.mma_work_factor,
                                    "peak": f"{peak_kind} dense bf16, burst and sustained (f16 operands run at "
                                            "the same rate; the 16-layer step keeps the GPU at its power cap)"}
            del b4
            torch.cuda.empty_cache()
            # the same prefill layer over the other format pairs, and with operands rounded once to f16
            # (kvattn_prefill_chunk_f16); one layer each: kernel rate only
            for wn, f16 in (("prefill524k_q4q4", False), ("prefill524k_q51q4", False), ("prefill524k_q50q41", False),
                            ("prefill524k_q8q8", False), ("prefill524k", True)):
                b6 = PrefillBench(kvattn, device, layers=1, wname=wn, f16=f16)
                b6.layer(0)
                k6 = time_layers(b6, 2)
                tf6 = b6.flops_per_layer / (k6 * 1e-3) / 1e12
                extra[wn + ("_f16" if f16 else "")] = {
                    "kernel_TFLOP/s": tf6, "kernel_frac_bf16": tf6 / bf16, "kernel_frac_bf16_sustained": tf6 / bf16_sus,
                    "layer_ms": k6,
                    "executed_frac_bf16": tf6 * b6.mma_work_factor / bf16, "k_fmt": b6.w.k_fmt, "v_fmt": b6.w.v_fmt,
                    "operands": "f16, rounded once" if f16 else "f16 high + low parts (about 22 bits)"}
                del b6
                torch.cuda.empty_cache()
            b5 = StreamBench(kvattn, device)
            n_gen = args.stream_steps or b5.w.steps
            ts, tr, tcp, td = time_stream(b5, n_gen, 2)
            tm, tenq, ncp = time_memcpy_route(b5)
            extra["stream524k"] = {
                "ms_per_step": ts, "ms_per_step_resident": tr, "ms_copies_only": tcp, "ms_decode": td,
                "pcie_GB/s": b5.copy_bytes_per_step / (tcp * 1e-3) / 1e9,
                "hbm_GB/s_decode": b5.attn_bytes(0) / (td * 1e-3) / 1e9,
                "generation_steps_timed": n_gen, "positions": [b5.w.context, b5.w.context + n_gen - 1],
                "hidden_copy_fraction": max(0.0, 1.0 - (ts - tr) / tcp) if tcp > 0 else None,
                "copy_bytes_per_step": b5.copy_bytes_per_step,
                "memcpy_route": {"ms_device": tm, "ms_host_enqueue": tenq, "copies": ncp,
                                 "pcie_GB/s": b5.copy_bytes_per_step / (max(tm, tenq) * 1e-3) / 1e9},
                "host_pool_GB": b5.host.numel() / 1e9}
            del b5
            torch.cuda.empty_cache()
            res = {}
            for name, nq, drift in (("per_turn_query", 1, 0.0), ("drifting_query", 16, 0.05)):
                b6 = ResidentStreamBench(kvattn, device, queries=nq, drift=drift)
                first = b6.copies_per_step(1)[0]          # the cold step copies the whole working set
                warm = b6.copies_per_step(max(2 * nq, 4))
                full = b6.w.layers * b6.w.kv_heads * b6.budget
                ms6 = time_steps(b6, max(8, args.extra_steps // 5), 2, world)
                res[name] = {"ms_per_step": ms6, "pages_copied_first_step": first,
                             "pages_copied_per_step": statistics.mean(warm), "hit_rate": 1.0 - statistics.mean(warm) / full,
                             "queries_cycled": nq, "drift": drift}
                del b6
                torch.cuda.empty_cache()
            extra["stream524k"]["resident_reuse"] = res
        except Exception as exc:  # report, do not hide
            extra["error"] = repr(exc)
        assert kvattn.kvattn_device_error() == 0
    line["extra"] = extra

    if rank == 0 and not args.no_cpu_baseline:
        gbs, secs, threads, sample = oracle_decode_sample("decode131k", 131072)
        line["cpu_baseline"] = {"value": gbs, "unit": "GB/s", "cores": len(os.sched_getaffinity(0)),
                                "blas_threads": threads, "kind": "oracle", "sample": sample,
                                "seconds_per_sample": secs}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        barrier(world)
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""Benchmark of the DSA hot path on B200: indexer -> top-k -> sparse attention (+ gate).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config c5] [--impl reference]

One step is one pass of the whole path over one batch of the workload, with inputs resident
in HBM.  The default workload is c5, the largest single-GPU configuration: the hybrid
DSA-SWA-SWA block at S = 65536 (one DSA layer -- indexer, top-k, sparse attention, gate --
and two sliding-window layers).  Times are CUDA events on the launching stream around each
library call; L2 is flushed (a 512 MB write) between steps, outside the timed events.
Prints one JSON line.

Multi-GPU: one process per GPU (torchrun); each rank runs its own copy of the workload
(the path has no exchange step: weak scaling), the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from workloads import dsa_inputs, get_config, swa_inputs  # noqa: E402
from workloads.gen import latent_inputs  # noqa: E402

METRIC = "query-tokens/s (indexer+top-k+sparse attn) and % of tensor/HBM roofline"
UNIT = "query-tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# float32 FMA peak of the CUDA cores: 148 SMs x 128 FMA/clk x 2 flop x 1.965 GHz.
F32_SIMT_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12

# DRAM traffic per launch from committed ncu captures: (kernel, config) -> (bytes,
# sha256 of the kernel source when captured).  Reported as null when the source changed.
NCU_TRAFFIC = {
    # masked_attn_tc_kernel, c5 full size (the DSA layer): 15.426 GB read + 0.532 GB written
    ("masked_attn", "c5"): (15957929728, "ddd03e9b88d66548"),
    # masked_attn_tc_kernel, c2 full size: 64.40 MB read + 3.63 MB written
    ("masked_attn", "c2"): (68023808, "ddd03e9b88d66548"),
    # gather_attn_kernel, c4: captured at B = 32 (same per-row work: 9 splits x 228 keys),
    # 1.3429 GB read + 5.37 MB written, scaled by the rows (x2) to the full B = 64 launch
    ("gather_attn", "c4"): (2696538112, "8652b3612fcab04a"),
}


# ----------------------------------------------------------------------------- helpers
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS if k in d}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def src_sha(name):
    """Hash of a kernel source's code: comments and blank lines do not count, so that a
    stored ncu figure stays attached to the code it was taken on."""
    p = os.path.join(ROOT, "sparse_attention_15_b200", "csrc", name)
    with open(p, encoding="utf-8") as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    code = "\n".join(line.rstrip() for line in text.splitlines() if line.strip())
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def causal_pairs(S, T, B, q_off):
    # number of (query, key) pairs with t <= s + q_off, over all batch rows
    n = np.minimum(np.arange(S, dtype=np.int64) + q_off + 1, T)
    return int(B * n.sum())


def selected_pairs(S, T, B, q_off, K):
    n = np.minimum(np.arange(S, dtype=np.int64) + q_off + 1, T)
    return int(B * np.minimum(n, K).sum())


class ClockSampler:
    """nvidia-smi sampling (every 20 ms) of the GPU this process uses, during the timed
    region (samples inside it; the nearest ones within 0.2 s when the region is shorter than
    the sampling interval)."""

    FIELDS = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.samples = []
        self.proc = None
        self.t_start = self.t_stop = None
        try:
            pci = torch.cuda.get_device_properties(device).pci_bus_id.lower()
        except Exception:
            pci = None
        self.pci = pci

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), [x.strip() for x in line.split(",")]))

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = [(t, f) for t, f in self.samples if len(f) >= 9 and
                (self.pci is None or self.pci.endswith(f[0].lower()[-12:]) or
                 f[0].lower().endswith(self.pci[-12:]))]
        if not rows:
            return None
        inside = [f for t, f in rows if self.t_start and self.t_stop and
                  self.t_start <= t <= self.t_stop]
        win = inside or [f for t, f in rows if self.t_start and self.t_stop and
                         self.t_start - 0.2 <= t <= self.t_stop + 0.2] or [f for _, f in rows]

        def num(x):
            try:
                return float(x)
            except ValueError:
                return float("nan")

        sm = [num(f[1]) for f in win]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for f in win:
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": num(win[0][2]),
                "reasons": sorted(reasons), "samples": len(win),
                "samples_inside_timed_region": len(inside),
                "power_w_max": max(num(f[3]) for f in win)}


def reduce_max(value, dist=None, device="cpu"):
    """Max of a float over all ranks (identity without a process group)."""
    if dist is None:
        return float(value)
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(units_per_rank, world, step_ms_max):
    """Whole-job throughput: every rank's units over the slowest rank's step time."""
    return units_per_rank * world / (step_ms_max / 1e3)


# ----------------------------------------------------------------------------- workloads
class Workload:
    """Device buffers and the library calls of one step of config `name`."""

    def __init__(self, name, device, seed_offset=0, S=None, T=None, B=None, indexer="per_head",
                 index_dtype="as_dtype", nsink=0, hadamard=False, attn_form="expanded",
                 latent_heads=128, score_rows=0):
        import dataclasses

        import sparse_attention_15_b200 as dsa

        self.dsa = dsa
        cfg = get_config(name)
        if S is not None or T is not None or B is not None:  # a reduced case (profiling)
            S = cfg.S if S is None else S
            T = cfg.T if T is None else T
            B = cfg.B if B is None else B
            cfg = dataclasses.replace(
                cfg, S=S, T=T, B=B,
                description=f"{cfg.description} [reduced: B={B}, S={S}, T={T}]")
        self.cfg = cfg
        self.device = device
        B = cfg.B
        self.attn_form = attn_form
        latent = attn_form == "latent"
        # latent (MQA-form) attention: one 512 + 64 latent row per token shared by the heads
        self.H = latent_heads if latent else cfg.H
        self.dqk, self.dv = (576, 512) if latent else (cfg.dqk, cfg.dv)
        if name == "c4":  # 174 GB of expanded K/V cache: shrink the batch only if it cannot fit
            free, _ = torch.cuda.mem_get_info(device)
            per_row = cfg.T * (cfg.DI + (self.dqk if latent else cfg.H * (cfg.dqk + cfg.dv))) * 2
            B = min(cfg.B, int((free - (6 << 30)) // per_row))
            if B < 1:
                raise RuntimeError("not enough device memory for one decode batch row")
        self.B = B
        if latent:
            x = dsa_inputs(cfg, device=device, B=B, seed=cfg.seed + seed_offset,
                           need=("q_idx", "k_idx", "w"))
            lt = latent_inputs(cfg, H=self.H, device=device, B=B, seed=cfg.seed + seed_offset,
                               nsink=nsink)
            # the attention tensors: q [B,S,H,576], k = the latent cache [B,T,576], no v
            x.update({"q": lt["q"], "k": lt["kv"], "v": None, "gate": lt["gate"]})
        else:
            x = dsa_inputs(cfg, device=device, B=B, seed=cfg.seed + seed_offset)
        self.index_dtype = index_dtype
        if index_dtype == "e4m3":  # indexer inputs handed over as e4m3 (exact for the integers)
            x["q_idx"] = x["q_idx"].to(torch.float8_e4m3fn)
            x["k_idx"] = x["k_idx"].to(torch.float8_e4m3fn)
        self.x = x
        self.nsink = nsink
        self.sink_k = self.sink_v = None
        if nsink and latent:  # latent sink rows [nsink, 576]
            self.sink_k = lt["sink_kv"]
        elif nsink:  # attention sinks (PAS): synthetic per-head sink rows, N(0,1)
            g = torch.Generator(device="cpu").manual_seed(cfg.seed + 7919)
            self.sink_k = torch.randn(nsink, cfg.H, cfg.dqk, generator=g).to(
                x["q"].dtype).to(device)
            self.sink_v = torch.randn(nsink, cfg.H, cfg.dv, generator=g).to(
                x["q"].dtype).to(device)
        self.K = cfg.k_eff
        self.idx = torch.empty((B, cfg.S, self.K), dtype=torch.int32, device=device)
        self.out = torch.empty((B, cfg.S, self.H, self.dv), dtype=x["q"].dtype, device=device)
        self.indexer = indexer
        self.args = dsa._forward_args(x["q_idx"], x["k_idx"], x["w"], cfg.scale, cfg.K, x["q"],
                                      x["k"], x["v"], x["gate"], None, "none", 0.0, "auto",
                                      self.out, None, self.idx,
                                      indexer, self.sink_k, self.sink_v, attn_form, self.dv)
        self.ws_bytes = dsa.dsa_forward_workspace_bytes(self.args)
        self.score_rows = 0
        if score_rows and cfg.S > score_rows:
            # a score buffer of `score_rows` rows: dsa_forward then runs the indexer and the
            # top-k block by block, and a block's scores stay in L2 between the two
            small = dsa.dsa_forward_workspace_bytes(self.args, minimum=True)
            self.ws_bytes = small + (score_rows - 1) * cfg.T * 4
            self.score_rows = score_rows
        self.ws = torch.empty(max(self.ws_bytes, 16), dtype=torch.uint8, device=device)
        dt = dsa.DTYPE[x["q"].dtype]
        if latent:
            self.algo = "latent"
            split_ws = dsa.lib().dsa_sparse_attn_latent_workspace_bytes(B, cfg.S, self.H, self.K,
                                                                        nsink)
        else:
            self.algo = dsa.dsa_sparse_attn_algo(dt, B, cfg.S, cfg.T, cfg.H, cfg.dqk, cfg.dv,
                                                 self.K)
            split_ws = dsa.dsa_sparse_attn_workspace_bytes(dt, B, cfg.S, cfg.T, cfg.H, cfg.dqk,
                                                           cfg.dv, self.K, "gather")
        self.swa = []
        for layer in range(1, cfg.swa_layers + 1):
            s = swa_inputs(cfg, layer, device=device, seed=cfg.seed + seed_offset)
            s["out"] = torch.empty((B, cfg.S, cfg.H, cfg.dv), dtype=x["q"].dtype, device=device)
            s["sink_k"] = s["sink_v"] = None
            if nsink:  # every layer has its own sinks, one row per KV head
                g = torch.Generator(device="cpu").manual_seed(cfg.seed + 7919 + layer)
                hkv = s["k"].shape[2]
                s["sink_k"] = torch.randn(nsink, hkv, cfg.dqk, generator=g).to(
                    x["q"].dtype).to(device)
                s["sink_v"] = torch.randn(nsink, hkv, cfg.dv, generator=g).to(
                    x["q"].dtype).to(device)
            self.swa.append(s)
        # optional Hadamard rotation of the indexer inputs (prefill), a stage of its own
        self.hadamard = hadamard and cfg.S > 1
        if self.hadamard:
            self.q_rot = torch.empty_like(x["q_idx"])
            self.k_rot = torch.empty_like(x["k_idx"])
        self.stages = (["hadamard"] if self.hadamard else []) + \
            ["indexer", "topk", "attention"] + [f"swa{i + 1}" for i in range(len(self.swa))]
        # our kernels per step: indexer (+ the query collapse), top-k, attention (+ combine for
        # split gathers), SWA.  The fused indexer launches six: the sampled indexer, the
        # thresholds, the filtering indexer, the candidate select and the two fallback
        # kernels (which return at once when the filter held)
        self.launches_per_step = 3 + \
            (1 if self.algo in ("gather", "latent") and split_ws > 0 else 0) + \
            (1 if indexer == "collapsed" else 0) + (4 if indexer == "fused" else 0) + \
            (2 if self.hadamard else 0) + len(self.swa)

    def _forward(self, x, events=None):
        """The DSA layer through the public whole-step call."""
        c = self.cfg
        self.dsa.dsa_forward(x["q_idx"], x["k_idx"], x["w"], c.scale, c.K, x["q"], x["k"],
                             x["v"], gate=x["gate"], out=self.out, idx_out=self.idx,
                             ws=self.ws, ws_bytes=self.ws_bytes, events=events,
                             indexer=self.indexer, sink_k=self.sink_k, sink_v=self.sink_v,
                             attn_form=self.attn_form, dv=self.dv)

    def step(self, ev):
        """Run one step; ev is a list of len(stages)+1 CUDA events (stage boundaries)."""
        c, x, d = self.cfg, self.x, self.dsa
        qi, ki, e0 = x["q_idx"], x["k_idx"], 0
        if self.hadamard:
            ev[0].record()
            qi = d.dsa_hadamard_rotate(x["q_idx"], out=self.q_rot)
            ki = d.dsa_hadamard_rotate(x["k_idx"], out=self.k_rot)
            e0 = 1
        self._forward(dict(x, q_idx=qi, k_idx=ki), events=ev[e0:e0 + 4])
        for i, s in enumerate(self.swa):
            d.dsa_window_attn(s["q"], s["k"], s["v"], c.window, gate=s["gate"], out=s["out"],
                              sink_k=s["sink_k"], sink_v=s["sink_v"])
            ev[e0 + 4 + i].record()

    # algorithmic work per launch of each stage
    def work(self):
        c, B = self.cfg, self.B
        es = 4 if c.dtype == "f32" else 2
        pairs = causal_pairs(c.S, c.T, B, c.q_off)
        sel = selected_pairs(c.S, c.T, B, c.q_off, self.K)
        rows = B * c.S
        ies = 1 if self.index_dtype == "e4m3" else es  # bytes per indexer input element
        if c.S == 1:
            # decode: one query per batch row streams the whole k_I cache once; HBM-bound
            # (k_I, the row's q_I and w, the score row written)
            idx_work = ("hbm", B * c.T * c.DI * ies + rows * c.HI * (c.DI * ies + 4) +
                        4.0 * pairs, "GB/s")
        elif self.indexer == "collapsed":
            # the head-collapsed form is not held to the per-head flop count: it is bound by
            # the score writes (4 B per causal pair) plus its reads of q_I, w and k_I
            idx_work = ("hbm", 4.0 * pairs + rows * c.HI * (c.DI * es + 4) +
                        B * c.T * c.DI * es, "GB/s")
        else:
            idx_work = ("tensor" if c.dtype == "bf16" else "alu", 2.0 * c.HI * c.DI * pairs,
                        "TFLOP/s")
        w = {}
        if self.hadamard:  # read and write q_I and k_I once each
            w["hadamard"] = ("hbm", 2.0 * (rows * c.HI * c.DI + B * c.T * c.DI) * es, "GB/s")
        w.update({
            "indexer": idx_work,
            "topk": ("hbm", 4.0 * pairs + 4.0 * rows * self.K, "GB/s"),
        })
        if self.algo == "latent":
            # every selected (query, key) pair, all heads: S = q . kv (2*H*576 flops) and
            # O += p kv[:512] (2*H*512); + every query against the sinks
            w["attention"] = ("tensor", 2.0 * self.H * (self.dqk + self.dv) *
                              (sel + rows * self.nsink), "TFLOP/s")
        elif self.algo == "masked_tile":
            # the method's work: QK^T and PV over every SELECTED pair, all heads (+ every
            # query against the sinks).  The kernel executes dense 128 x 128 tiles over every
            # causal pair under the selection mask; that executed work is reported beside it
            w["attention"] = ("tensor", 2.0 * c.H * (c.dqk + c.dv) * (sel + rows * self.nsink),
                              "TFLOP/s")
        else:
            w["attention"] = ("hbm", (sel + rows * self.nsink) * c.H * (c.dqk + c.dv) * es +
                              rows * c.H * (c.dqk + c.dv) * es, "GB/s")
        for i in range(len(self.swa)):
            band = selected_pairs(c.S, c.T, B, c.q_off, c.window)
            w[f"swa{i + 1}"] = ("tensor", 2.0 * c.H * (c.dqk + c.dv) * (band + rows * self.nsink),
                                "TFLOP/s")
        return w

    def executed_work(self):
        """Work the kernels execute where it differs from the method's: the masked-tile
        attention computes every causal (query, key) pair of every head under the mask."""
        c, B = self.cfg, self.B
        if self.algo != "masked_tile":
            return {}
        pairs = causal_pairs(c.S, c.T, B, c.q_off)
        return {"attention": 2.0 * c.H * (c.dqk + c.dv) * (pairs + B * c.S * self.nsink)}

    def host_copy(self):
        """Pinned host copies of what one step takes from the host.  Prefill: every input of
        the DSA layer (and of the SWA layers).  Decode: the new queries and the new token's
        cache rows (the caches themselves stay resident in HBM)."""
        x = self.x
        if self.cfg.S == 1:
            sel = {"q_idx": x["q_idx"], "w": x["w"], "q": x["q"], "gate": x["gate"],
                   "k_idx_row": x["k_idx"][:, -1:], "k_row": x["k"][:, -1:]}
            if x["v"] is not None:
                sel["v_row"] = x["v"][:, -1:]
        else:
            sel = dict(x)
            for i, layer in enumerate(self.swa):
                for k in ("q", "k", "v", "gate"):
                    sel[f"swa{i}_{k}"] = layer[k]
        return {k: (None if v is None else v.contiguous().cpu().pin_memory())
                for k, v in sel.items()}

    def result(self):
        """The step's result: the output of its last attention layer (the block's output)."""
        return self.swa[-1]["out"] if self.swa else self.out

    def forward_from(self, bufs):
        """One step on device buffers `bufs` (names as in host_copy)."""
        c = self.cfg
        x = dict(self.x)
        x.update({k: v for k, v in bufs.items() if not k.startswith("swa")})
        self._forward(x)
        for i, layer in enumerate(self.swa):
            g = {k: bufs.get(f"swa{i}_{k}", layer[k]) for k in ("q", "k", "v", "gate")}
            self.dsa.dsa_window_attn(g["q"], g["k"], g["v"], c.window, gate=g["gate"],
                                     out=layer["out"], sink_k=layer["sink_k"],
                                     sink_v=layer["sink_v"])

    def e2e_pipelined(self, host, n):
        """Prefill end to end over n steps: every step copies all its inputs from pinned host
        memory and reads its result back; the copies of step i+1 (a second stream, double
        buffers) overlap the compute of step i.  Nothing else runs in the timed region (no L2
        flush: every step's inputs are fresh copies from the host).  Returns ms per step
        (device events)."""
        dev = self.device
        bufs = [{k: torch.empty_like(v, device=dev) for k, v in host.items() if v is not None}
                for _ in range(2)]
        out_host = torch.empty(self.result().shape, dtype=self.result().dtype).pin_memory()
        main = torch.cuda.current_stream(dev)
        cs = torch.cuda.Stream(device=dev)
        ready = [torch.cuda.Event() for _ in range(2)]
        free = [torch.cuda.Event() for _ in range(2)]
        used = [False, False]

        def copy_in(slot):
            with torch.cuda.stream(cs):
                if used[slot]:
                    cs.wait_event(free[slot])  # the compute that read this buffer is done
                for k, v in host.items():
                    if v is not None:
                        bufs[slot][k].copy_(v, non_blocking=True)
                ready[slot].record(cs)

        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(main)
        cs.wait_stream(main)  # no copy starts before the timed region
        copy_in(0)
        for i in range(n):
            slot = i & 1
            if i + 1 < n:
                copy_in(1 - slot)
            main.wait_event(ready[slot])
            self.forward_from(bufs[slot])
            out_host.copy_(self.result(), non_blocking=True)
            free[slot].record(main)
            used[slot] = True
        t1.record(main)
        torch.cuda.synchronize(dev)
        return t0.elapsed_time(t1) / n, out_host.numel() * out_host.element_size()

    def e2e_step(self, host, dev_bufs, out_host):
        """Host inputs -> device -> dsa_forward -> result back to the host."""
        x = dict(self.x)
        for k, v in host.items():
            if v is None:
                continue
            if k.endswith("_row"):
                name = k[:-4]
                x[name][:, -1:].copy_(v, non_blocking=True)
            else:
                dev_bufs[k].copy_(v, non_blocking=True)
                x[k] = dev_bufs[k]
        self._forward(x)
        out_host.copy_(self.out, non_blocking=True)


# ----------------------------------------------------------------------------- oracle timing
def oracle_rows_per_s(cfg, x_host, rows, budget_s, sink_kv=None):
    """The CPU oracle as it stands, on sampled query rows of batch row 0: returns
    (rows done, seconds).  Each row runs scores -> top-k -> dense masked attention (over
    the shared latent rows when x_host has no v: the latent form)."""
    from oracle import dsa_oracle as O

    q_off = cfg.q_off
    done = 0
    t0 = time.perf_counter()
    for s in rows:
        sl = slice(s, s + 1)
        sc = O.index_scores(x_host["q_idx"][:1, sl], x_host["k_idx"][:1], x_host["w"][:1, sl],
                            cfg.scale, q_off=s + q_off)
        idx = O.topk_indices(sc, cfg.k_eff, q_off=s + q_off)
        g = None if x_host["gate"] is None else x_host["gate"][:1, sl]
        if x_host["v"] is None:
            O.sparse_attention_latent(x_host["q"][:1, sl], x_host["k"][:1], idx, 512, gate=g,
                                      gate_mode=cfg.gate, q_off=s + q_off, sink_kv=sink_kv)
        else:
            O.sparse_attention(x_host["q"][:1, sl], x_host["k"][:1], x_host["v"][:1], idx,
                               gate=g, gate_mode=cfg.gate, q_off=s + q_off)
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    return done, time.perf_counter() - t0


def blas_threads():
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


def sample_rows(S, n):
    return sorted(set(int(r) for r in np.linspace(0, S - 1, n)))


def host_inputs(cfg, x, B_rows=1):
    return {k: (None if v is None else v[:B_rows].cpu()) for k, v in x.items()}


# ----------------------------------------------------------------------------- main
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            sys.exit("bench.py --gpus N>1 must be launched with torchrun (one process per GPU)")
    return world, rank, local


def run_reference(args, world, rank):
    """The reference arm: the CPU oracle, timed on bounded samples of the workload."""
    if rank != 0:
        return
    cfg = get_config(args.config)
    latent = getattr(args, "attn", "expanded") == "latent"
    if latent:  # the latent form: shared 512+64 rows, the oracle's latent attention
        x = dsa_inputs(cfg, device="cpu", B=1, need=("q_idx", "k_idx", "w"))
        lt = latent_inputs(cfg, H=args.latent_heads, device="cpu", B=1)
        x.update({"q": lt["q"], "k": lt["kv"], "v": None, "gate": lt["gate"]})
    else:
        x = dsa_inputs(cfg, device="cpu", B=1)
    per_step = {"c1": 16, "c2": 4, "c3": 1, "c4": 1, "c5": 1}[cfg.name]
    rows_all = sample_rows(cfg.S, max(per_step * (args.steps + args.warmup), 1))
    rng = np.random.default_rng(0)
    rng.shuffle(rows_all)
    it = iter(rows_all * 2)
    for _ in range(args.warmup):
        oracle_rows_per_s(cfg, x, [next(it) for _ in range(per_step)], 1e9)
    total_rows, total_s = 0, 0.0
    for _ in range(args.steps):
        n, dt = oracle_rows_per_s(cfg, x, [next(it) for _ in range(per_step)], 1e9)
        total_rows += n
        total_s += dt
    value = total_rows / total_s
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total_s / max(args.steps, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(cfg, cfg.B, args),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{per_step} query row(s) per step of batch row 0, spread "
                                   f"over the {cfg.S} queries; float64 numpy oracle"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(cfg, B):
    return {"workload": f"{cfg.name}: {cfg.description}", "B": B, "S": cfg.S, "T": cfg.T,
            "indexer": f"{cfg.HI}x{cfg.DI}", "top_k": cfg.K, "heads": cfg.H,
            "qk_dim": f"{cfg.d_nope}+{cfg.d_rope}", "v_dim": cfg.dv, "gate": cfg.gate,
            "swa_layers": cfg.swa_layers, "window": cfg.window,
            "l2": "flushed between steps (512 MB write outside the timed events); the e2e "
                  "steps copy fresh inputs from the host instead"}


def bench_config(cfg, B, args, hadamard=None, score_rows=None):
    """The `config` object of a JSON line: the same keys and values for both arms."""
    latent = args.attn == "latent"
    d = dict(workload_config(cfg, B), indexer_form=args.indexer,
             indexer_dtype=args.index_dtype, sinks=args.sinks,
             hadamard=bool(args.hadamard and cfg.S > 1) if hadamard is None else hadamard,
             attention_form=args.attn,
             score_block_rows=(args.score_rows if args.score_rows and cfg.S > args.score_rows
                               else None) if score_rows is None else score_rows)
    if latent:
        d.update({"heads": args.latent_heads, "qk_dim": "512+64 (latent, shared by all heads)",
                  "v_dim": 512})
    return d


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="c5", choices=["c1", "c2", "c3", "c4", "c5"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work")
    ap.add_argument("--S", type=int, default=None, help="reduced query count (profiling cases)")
    ap.add_argument("--T", type=int, default=None, help="reduced key count (profiling cases)")
    ap.add_argument("--B", type=int, default=None, help="reduced batch (profiling cases)")
    ap.add_argument("--indexer", default="per_head", choices=["per_head", "collapsed", "fused"],
                    help="indexer form: the pages' per-head work (default), head-collapsed, or "
                         "per-head with the top-k candidates filtered inside the indexer")
    ap.add_argument("--index-dtype", default="as_dtype", choices=["as_dtype", "e4m3"],
                    help="indexer input type (the workload's dtype by default)")
    ap.add_argument("--sinks", type=int, default=0,
                    help="attention sinks (PAS virtual KV entries) per layer, 0..128")
    ap.add_argument("--hadamard", action="store_true",
                    help="rotate the indexer inputs (Hadamard) every prefill step")
    ap.add_argument("--attn", default="expanded", choices=["expanded", "latent"],
                    help="attention over the expanded per-head K/V (the workloads' form) or "
                         "over a shared 512+64 latent cache (MQA form)")
    ap.add_argument("--latent-heads", type=int, default=128,
                    help="query heads of the latent form (<= 128)")
    ap.add_argument("--score-rows", type=int, default=0,
                    help="score buffer of this many query rows (indexer and top-k run block "
                         "by block, the scores staying in L2); 0 = the whole matrix")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    world, rank, local = dist_setup(args)

    if args.impl == "reference":
        run_reference(args, world, rank)
        return

    from sparse_attention_15_b200 import build as _build

    _build.build_if_needed()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist

    wl = Workload(args.config, dev, seed_offset=rank, S=args.S, T=args.T, B=args.B,
                  indexer=args.indexer, index_dtype=args.index_dtype, nsink=args.sinks,
                  hadamard=args.hadamard, attn_form=args.attn, latent_heads=args.latent_heads,
                  score_rows=args.score_rows)
    cfg = wl.cfg
    nst = len(wl.stages)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if pg is not None:
            pg.barrier()
        torch.cuda.synchronize(dev)

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nst + 1)]
          for _ in range(args.steps)]
    wev = [torch.cuda.Event(enable_timing=True) for _ in range(nst + 1)]
    for _ in range(args.warmup):
        flush.zero_()
        wl.step(wev)
    torch.cuda.synchronize(dev)
    wl.dsa.dsa_device_status(reset=True)

    clocks = ClockSampler(dev)
    clocks.start()
    time.sleep(0.3)
    barrier()
    clocks.mark("t_start")
    t_wall = time.perf_counter()
    for i in range(args.steps):
        flush.zero_()
        wl.step(ev[i])
    barrier()
    t_wall = time.perf_counter() - t_wall
    clocks.mark("t_stop")
    clk = clocks.stop()
    wl.dsa.dsa_device_status(reset=True)  # raises if any wait timed out

    stage_ms = np.zeros(nst)
    for i in range(args.steps):
        for j in range(nst):
            stage_ms[j] += ev[i][j].elapsed_time(ev[i][j + 1])
    stage_ms /= args.steps
    step_ms = reduce_max(float(stage_ms.sum()), pg, dev)
    units = wl.B * cfg.S * world
    value = job_value(wl.B * cfg.S, world, step_ms)

    # roofline of the dominant stage
    peaks, peak_src = load_peaks()
    work = wl.work()
    executed = wl.executed_work()
    kernels = {}
    # tensor-bound kernels are held to the burst bf16 figure: every step here is far shorter
    # than the seconds-long loop the sustained figure comes from (that one is quoted beside it)
    tensor_peak = peaks["bf16_tflops"]
    sustained = peaks.get("bf16_tflops_sustained")
    for j, name in enumerate(wl.stages):
        bound, amount, unit = work[name]
        sec = stage_ms[j] / 1e3
        if bound == "tensor":
            # e4m3 indexer operands: the bf16 figure times the nominal fp8:bf16 ratio of 2
            scale = 2.0 if (name == "indexer" and wl.index_dtype == "e4m3") else 1.0
            ach, peak = amount / sec / 1e12, tensor_peak * scale
        elif bound == "alu":
            ach, peak = amount / sec / 1e12, F32_SIMT_TFLOPS
        else:
            ach, peak = amount / sec / 1e9, peaks["hbm_gbs"]
        kernels[name] = {"ms": round(float(stage_ms[j]), 5), "bound": bound,
                         "achieved": round(ach, 2), "peak": peak, "unit": unit,
                         "frac": round(ach / peak, 4),
                         "share": round(float(stage_ms[j]) / float(stage_ms.sum()), 4)}
        if bound == "tensor" and sustained:
            kernels[name]["frac_of_sustained"] = round(ach / (sustained * scale), 4)
        if name in executed:  # the dense tiles the kernel actually computes
            ex = executed[name] / sec / 1e12
            kernels[name]["executed_achieved"] = round(ex, 2)
            kernels[name]["executed_frac"] = round(ex / peak, 4)
    if wl.score_rows:
        # row blocks interleave the indexer and the top-k: the first event pair spans both
        kernels["indexer_and_topk"] = dict(kernels.pop("indexer"), bound="mixed",
                                           achieved=None, frac=None)
        kernels.pop("topk")
    elif wl.indexer == "fused":
        # one fused stage: the sampled pass, the filtering indexer and the candidate select
        # (+ the fallback check), held to the per-head indexer's flops over both event spans
        ki, kt = kernels.pop("indexer"), kernels.pop("topk")
        ms = ki["ms"] + kt["ms"]
        ach = ki["achieved"] * ki["ms"] / ms
        kernels["indexer_and_topk"] = dict(
            ki, ms=round(ms, 5), achieved=round(ach, 2), frac=round(ach / ki["peak"], 4),
            share=round(ki["share"] + kt["share"], 4),
            split_ms={"sample_and_filter": ki["ms"], "select": kt["ms"]})
        if "frac_of_sustained" in ki:
            kernels["indexer_and_topk"]["frac_of_sustained"] = round(
                ki["frac_of_sustained"] * ki["ms"] / ms, 4)
    dom = max(kernels, key=lambda k: kernels[k]["ms"])
    attn_k = {"masked_tile": "masked_attn", "latent": "latent_attn"}.get(wl.algo, "gather_attn")
    kname = {"indexer": "index_scores", "topk": "topk", "attention": attn_k,
             "indexer_and_topk": "index_scores"}.get(dom, "masked_attn")
    tr = NCU_TRAFFIC.get((kname, cfg.name))
    srcfile = {"index_scores": "indexer_tc.cu", "topk": "topk.cu", "gather_attn": "gather_attn.cu",
               "masked_attn": "attn_tc.cu", "latent_attn": "latent_attn.cu"}[kname]
    traffic = tr[0] if tr and tr[1] == src_sha(srcfile) else None
    roof = dict(kernels[dom])
    roof.pop("ms")
    roof.pop("share")
    roof.update({"kernel": dom, "attention_algo": wl.algo, "traffic": traffic,
                 "tensor_peak_kind": "burst",
                 "work": "the method's algorithmic work (attention: selected pairs only)",
                 "peak_source": "measured (MEASURED_PEAKS.json)" if peak_src == "measured" else
                                "fallback (6.65 TB/s HBM, 1.59 / 1.40 PFLOP/s bf16 burst / sustained)"})

    # end-to-end through the public call with host buffers
    e2e = None
    if not args.no_e2e and cfg.S > 1:
        host = wl.host_copy()
        for _ in range(max(1, args.warmup // 2)):
            wl.e2e_pipelined(host, 2)
        n_e2e = max(3, min(args.steps, 50))
        barrier()
        e2e_ms, d2h = wl.e2e_pipelined(host, n_e2e)
        barrier()
        e2e_ms = reduce_max(e2e_ms, pg, dev)
        h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
        e2e = {"value": units / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "ms_per_step": round(e2e_ms, 4),
               "steps": n_e2e, "overlap": "step i+1's copies run during step i's compute"}
        wl.dsa.dsa_device_status(reset=True)
    elif not args.no_e2e:
        host = wl.host_copy()
        dev_bufs = {k: (None if v is None else torch.empty_like(v, device=dev))
                    for k, v in host.items() if not k.endswith("_row")}
        out_host = torch.empty(wl.out.shape, dtype=wl.out.dtype).pin_memory()
        for _ in range(args.warmup):
            wl.e2e_step(host, dev_bufs, out_host)
        torch.cuda.synchronize(dev)
        n_e2e = max(3, min(args.steps, 50))
        e0 = [torch.cuda.Event(enable_timing=True) for _ in range(n_e2e)]
        e1 = [torch.cuda.Event(enable_timing=True) for _ in range(n_e2e)]
        barrier()
        for i in range(n_e2e):
            flush.zero_()
            e0[i].record()
            wl.e2e_step(host, dev_bufs, out_host)
            e1[i].record()
        barrier()
        e2e_ms = reduce_max(sum(e0[i].elapsed_time(e1[i]) for i in range(n_e2e)) / n_e2e, pg,
                            dev)
        h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
        e2e = {"value": units / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(out_host.numel() * out_host.element_size()),
               "ms_per_step": round(e2e_ms, 4), "steps": n_e2e}
        wl.dsa.dsa_device_status(reset=True)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        xh = host_inputs(cfg, wl.x, 1)
        rows = sample_rows(cfg.S, 4096)
        rng = np.random.default_rng(0)
        rng.shuffle(rows)
        skv = None if wl.sink_k is None or wl.attn_form != "latent" else wl.sink_k.cpu()
        n, sec = oracle_rows_per_s(cfg, xh, rows, args.cpu_budget, sink_kv=skv)
        cpu = {"value": n / sec, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": f"{n} query rows of batch row 0 drawn evenly over the {cfg.S} "
                         f"queries, {sec:.1f} s of float64 numpy oracle work "
                         f"(scores -> top-k -> dense masked attention per row)"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32" if cfg.dtype == "f32" else "bf16", "data": "synthetic",
            "config": bench_config(cfg, wl.B, args, hadamard=wl.hadamard,
                                   score_rows=wl.score_rows or None),
            "roofline": roof, "kernels": kernels, "cpu_baseline": cpu, "e2e": e2e,
            "clocks": clk, "gpu_launches": wl.launches_per_step * args.steps,
            "wall_ms_per_step_incl_flush": round(1e3 * t_wall / args.steps, 4),
        }
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""Benchmark of the LSA layer hot path on B200 (one process per GPU).

Default workload (N=1 headline): decode, 32 sequences x 131072 cached tokens, one query each,
indexer H_I=64 d_I=128, K = 2048 = 16 sink + 1024 window + 1008 dynamic, 128 MLA heads over
576-dim latent rows, two layers forming a Cross-Layer-Indexing pair (N=2).  One step =
  append the step's token (indexer key + sub-block mean + latent row, both layers)
  -> lsa_index (owner layer) -> lsa_attend (owner) -> lsa_attend (reuse layer, owner's indices).
Metric: LSA layer decode tokens/s = sequences x layers / step time (per-layer throughput).

Other workloads (--workload): decode_1m_hi / decode_1m_flat (B=4, L=1M, HI with P=128, B=8,
M=1024 vs flat on the same inputs) and prefill_32k (B=1, L=32768 causal, chunks of 4096
queries, tokens/s = L / step time).

--impl reference times the CPU oracle (the slow fp64 restatement of the method) on a bounded
sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# DRAM bytes per launch of the dominant kernel (the tcgen05 scorer of lsa_index), from one ncu
# capture of that kernel on 4 of the 32 sequences: dram__bytes_read.sum + dram__bytes_write.sum,
# the mean of two consecutive launches (133.355 + 2.130 MB), scaled by the 8x more keys of the
# full launch.  A figure is valid only for the scorer source it was measured on: `source_sha` is
# the sha256 prefix of csrc/score_tc.cu at the capture, and on any other source the bench reports
# the traffic as null.
SCORER_TRAFFIC = {"decode_b32_128k_cli2": {"bytes": (133.355008e6 + 2.129536e6) * 8,
                                           "source_sha": "a2adafef6315fca9",
                                           "how": "ncu capture of score_tc_kernel at 4 sequences "
                                                  "(mean of 2 launches), scaled x8"}}


def scorer_source_sha() -> str:
    import hashlib
    p = os.path.join(ROOT, "lightning_indexer_top_score_b200", "csrc", "score_tc.cu")
    with open(p, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def scorer_traffic(name: str):
    """(bytes, how) of the stored capture for this workload, or (None, why not)."""
    ent = SCORER_TRAFFIC.get(name)
    if ent is None:
        return None, None
    if ent["source_sha"] != scorer_source_sha():
        return None, "the scorer changed since its last ncu capture"
    return ent["bytes"], ent["how"]


L2_BYTES = 126 * 2 ** 20


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples the SM clock, its maximum and the throttle reasons of one GPU every ~1 ms through
    NVML (read-only queries) while the timed region runs.  Without NVML (pynvml missing or its
    initialisation failing) there is no sampling and stop() returns None."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self._stop = None
        self._thread = None
        self.max_mhz = None

    def start(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._thread = None
            return
        self._stop = threading.Event()

        def run():
            while not self._stop.is_set():
                try:
                    sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                    rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.samples.append((sm, rs))
                except Exception:
                    pass
                self._stop.wait(0.001)

        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()

    def stop(self):
        if self._thread is None:
            return None
        self._stop.set()
        self._thread.join(timeout=2)
        if not self.samples:
            return None
        sm = [a for a, _ in self.samples]
        reasons = sorted({k for _, r in self.samples for k, bit in self.REASONS.items() if r & bit})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(sm), "source": "nvml"}


# ----------------------------------------------------------------------------- replicas

def replica_seed(base: int, rank: int) -> int:
    """Seed of a replica's synthetic inputs: every rank works on its own sequences."""
    return base + 7919 * rank


def max_over_ranks(x: float, world: int, device) -> float:
    """Largest per-rank value (a device-timed duration); every rank calls it in the same order."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank_step: int, world: int, steps: int, total_ms: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return units_per_rank_step * world * steps / (total_ms / 1000.0)


# ----------------------------------------------------------------------------- workloads

def workload_config(name):
    from lightning_indexer_top_score_b200 import workloads as W
    from dataclasses import replace
    if name == "decode_128k":
        return W.DECODE_128K
    if name == "decode_128k_fp8":
        # the same decode step with the FP8 (E4M3) indexer; attention stays bf16
        return replace(W.DECODE_128K, name="decode_b32_128k_cli2_fp8_indexer")
    if name == "decode_1m_hi":
        return W.DECODE_1M_HI
    if name == "decode_1m_flat":
        return replace(W.DECODE_1M_HI, name="decode_b4_1m_flat", M=0)
    if name == "prefill_32k":
        return W.PREFILL_32K
    if name.startswith("index_chunk_"):
        # one 2048-query prefill chunk's indexer: index_chunk_<hi|flat>_<L>
        parts = name.split("_")
        if len(parts) == 4 and parts[2] in ("hi", "flat") and parts[3].isdigit():
            return W.index_chunk_config(int(parts[3]), parts[2])
    if name.startswith("train_"):
        # core attention of one training step (forward + backward): train_<L>
        parts = name.split("_")
        if len(parts) == 2 and parts[1].isdigit():
            return W.train_config(int(parts[1]))
    if name.startswith("table11_"):
        # the pooling ablation's setting (Table 11): decode at 128K, M = 128 recalled pages,
        # table11_<mean|minmax>_<sub-block size>
        parts = name.split("_")
        if len(parts) == 3 and parts[1] in ("mean", "minmax") and parts[2].isdigit():
            return replace(W.DECODE_128K, name=f"decode_b32_128k_hi_m128_{parts[1]}_sb{parts[2]}",
                           M=128, sub_block=int(parts[2]))
    if name.startswith("sweep_"):
        # decode sweep point of the length table: sweep_<dsa|lsa>_<L>
        parts = name.split("_")
        if len(parts) == 3 and parts[1] in ("dsa", "lsa") and parts[2].isdigit():
            return W.sweep_config(int(parts[2]), parts[1])
    raise SystemExit(f"unknown workload {name}")


class DecodeStep:
    """One decode step of a CLI pair through the public API (liblsa via the binding)."""

    def __init__(self, cfg, device, rank=0, fp8=False, minmax=False):
        import torch
        from lightning_indexer_top_score_b200 import lsa
        from lightning_indexer_top_score_b200.workloads import DeviceInputs
        self.cfg, self.lsa, self.torch, self.fp8, self.minmax = cfg, lsa, torch, fp8, minmax
        self.inp = DeviceInputs(cfg, device=device, seed=replica_seed(cfg.seed, rank))
        B, L, cap = cfg.B, cfg.L, cfg.cap
        inp = self.inp
        # mean cache of the whole prefix through the library's own append
        zero = torch.zeros(B, dtype=torch.int32, device=device)
        lsa.lsa_kv_append(zero, k_I_new=inp.k_I[:, :L].contiguous(), k_I=inp.k_I,
                          k_mean=inp.k_mean, sub_block=cfg.sub_block)
        if minmax:
            # MinMax pooling rows (k_max | k_min) of the whole prefix for the HI stage 1
            nb = (cap + cfg.sub_block - 1) // cfg.sub_block
            self.k_minmax = torch.zeros(B, nb, 2 * cfg.D_I, dtype=torch.bfloat16, device=device)
            lsa.lsa_kv_minmax(zero, L, inp.k_I, self.k_minmax, sub_block=cfg.sub_block)
        # the step's token: re-appended at position L-1 every step (state stays fixed)
        self.kv_old = torch.full((B,), L - 1, dtype=torch.int32, device=device)
        self.k_new = inp.k_I[:, L - 1:L].contiguous()
        self.c_new = [c[:, L - 1:L].contiguous() for c in inp.c_kv]
        self.idx = torch.empty(B, cfg.T, cfg.K_sparse, dtype=torch.int32, device=device)
        self.ws_i = torch.empty(lsa.lsa_index_workspace_bytes(
            B, cfg.T, cfg.H_I, cfg.D_I, cap, cfg.K_sparse, cfg.page, cfg.sub_block, cfg.M),
            dtype=torch.uint8, device=device)
        self.ws_a = torch.empty(max(256, lsa.lsa_attend_workspace_bytes(
            B, cfg.T, cfg.H, 512, cfg.K_sparse, cfg.sink, cfg.swa)), dtype=torch.uint8,
            device=device)
        self.out = [torch.empty(B, cfg.T, cfg.H, 512, dtype=torch.bfloat16, device=device)
                    for _ in inp.q]
        self.lse = [torch.empty(B, cfg.T, cfg.H, dtype=torch.float32, device=device)
                    for _ in inp.q]
        self.devw = torch.zeros(1, dtype=torch.int32, device=device)
        self.events = None
        if fp8:
            # FP8 key cache (codes + per-token scales) quantised once from the bf16 prefix; each
            # step writes its token's key into slot L-1 and quantises its queries
            inp = self.inp
            self.k8, self.ks = lsa.lsa_quantize_fp8(inp.k_I)
            self.q8 = torch.empty(inp.q_I.shape, dtype=torch.uint8, device=device)
            self.qs = torch.empty(inp.q_I.shape[:-1], dtype=torch.float32, device=device)

    def run(self, ev=None):
        lsa, inp, cfg = self.lsa, self.inp, self.cfg
        if ev is not None:
            ev[0].record()
        if self.fp8:
            L = cfg.L
            lsa.lsa_quantize_fp8(self.k_new, codes=self.k8[:, L - 1], scales=self.ks[:, L - 1],
                                 device_error=self.devw)
            for layer in range(len(inp.c_kv)):
                lsa.lsa_kv_append(self.kv_old, c_new=self.c_new[layer], c_kv=inp.c_kv[layer],
                                  device_error=self.devw)
        else:
            lsa.lsa_kv_append(self.kv_old, k_I_new=self.k_new, k_I=inp.k_I,
                              k_mean=None if self.minmax else inp.k_mean, c_new=self.c_new[0],
                              c_kv=inp.c_kv[0], sub_block=cfg.sub_block, device_error=self.devw)
            if self.minmax:
                lsa.lsa_kv_minmax(self.kv_old, 1, inp.k_I, self.k_minmax,
                                  sub_block=cfg.sub_block, device_error=self.devw)
            for layer in range(1, len(inp.c_kv)):
                lsa.lsa_kv_append(self.kv_old, c_new=self.c_new[layer], c_kv=inp.c_kv[layer],
                                  device_error=self.devw)
        if ev is not None:
            ev[1].record()
        if self.fp8:
            lsa.lsa_quantize_fp8(inp.q_I, codes=self.q8, scales=self.qs, device_error=self.devw)
            lsa.lsa_index_fp8(self.q8, self.qs, inp.w_I, self.k8, self.ks, inp.kv_len, inp.q_pos,
                              cfg.K_sparse, cfg.sink, cfg.swa, indices=self.idx, ws=self.ws_i)
        elif self.minmax:
            lsa.lsa_index_minmax(inp.q_I, inp.w_I, inp.k_I, self.k_minmax, inp.kv_len,
                                 inp.q_pos, cfg.K_sparse, cfg.sink, cfg.swa, cfg.page,
                                 cfg.sub_block, cfg.M, indices=self.idx, ws=self.ws_i)
        else:
            lsa.lsa_index(inp.q_I, inp.w_I, inp.k_I, inp.k_mean if cfg.M else None, inp.kv_len,
                          inp.q_pos, cfg.K_sparse, cfg.sink, cfg.swa, cfg.page, cfg.sub_block,
                          cfg.M, indices=self.idx, ws=self.ws_i)
        if ev is not None:
            ev[2].record()
        for layer in range(len(inp.q)):
            lsa.lsa_attend(inp.q[layer], inp.c_kv[layer], self.idx, inp.kv_len, inp.q_pos,
                           cfg.sink, cfg.swa, cfg.scale, out=self.out[layer], lse=self.lse[layer],
                           ws=self.ws_a)
            if ev is not None:
                ev[3 + layer].record()

    def tokens_per_step(self):
        return self.cfg.B * self.cfg.T * len(self.inp.q)

    def check_errors(self):
        return self.lsa.lsa_get_error(self.ws_i) | self.lsa.lsa_get_error(self.ws_a) | int(
            self.devw.item())

    def index_bytes(self):
        """Algorithmic bytes of the flat decode scoring pass: every dynamic key read once."""
        cfg = self.cfg
        dyn = cfg.L - cfg.sink - cfg.swa
        if self.fp8:
            # one E4M3 code per dim plus one fp32 scale per key
            return cfg.B * cfg.T * dyn * (cfg.D_I + 4)
        if cfg.M == 0:
            return cfg.B * cfg.T * dyn * cfg.D_I * 2
        pages = math.ceil(dyn / cfg.page)
        means = pages * (cfg.page // cfg.sub_block)
        # a MinMax row holds two keys' worth of dims (k_max | k_min)
        pooled = means * (2 if self.minmax else 1)
        return cfg.B * cfg.T * (pooled + cfg.M * cfg.page) * cfg.D_I * 2

    def step_bytes(self):
        """Bytes one step reads at least once: the scored keys (or means and recalled pages) and
        every layer's attended latent rows."""
        cfg = self.cfg
        keys = attended_keys(np.array([cfg.L - 1]), cfg.sink, cfg.swa, cfg.K_sparse)[0]
        return self.index_bytes() + len(self.inp.q) * cfg.B * cfg.T * int(keys) * 1152

    # ---- end-to-end through host buffers
    def e2e_setup(self):
        """Pinned host copies of each step's inputs (indexer q / w, the new key and latent rows,
        the MLA queries) and outputs (out, lse), and a second device slot of the step's inputs
        and outputs, so that one step's copies overlap the other slot's compute."""
        torch = self.torch
        inp = self.inp
        self.h_in = {"q_I": inp.q_I.cpu().pin_memory(), "w_I": inp.w_I.cpu().pin_memory(),
                     "k_new": self.k_new.cpu().pin_memory(),
                     "c_new": [c.cpu().pin_memory() for c in self.c_new],
                     "q": [q.cpu().pin_memory() for q in inp.q]}
        self.h_out = [{"out": [torch.empty_like(o, device="cpu").pin_memory() for o in self.out],
                       "lse": [torch.empty_like(l, device="cpu").pin_memory() for l in self.lse]}
                      for _ in range(2)]
        self.slots = [{"q_I": inp.q_I, "w_I": inp.w_I, "k_new": self.k_new,
                       "c_new": list(self.c_new), "q": list(inp.q), "out": list(self.out),
                       "lse": list(self.lse)}]
        self.slots.append({k: ([torch.empty_like(t) for t in v] if isinstance(v, list)
                               else torch.empty_like(v)) for k, v in self.slots[0].items()})
        self.s_in, self.s_out = torch.cuda.Stream(), torch.cuda.Stream()
        # one CUDA graph of the step per slot (the graph keeps the slot's buffer addresses)
        self.graphs = []
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for k in range(2):
                self._use_slot(k)
                self.run()
                side.synchronize()
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=side):
                    self.run()
                self.graphs.append(g)
        torch.cuda.synchronize()
        self._use_slot(0)
        bi = sum(t.numel() * t.element_size() for t in (self.h_in["q_I"], self.h_in["w_I"],
                                                        self.h_in["k_new"]))
        bi += sum(t.numel() * t.element_size() for t in self.h_in["c_new"] + self.h_in["q"])
        bo = sum(t.numel() * t.element_size() for t in self.h_out[0]["out"] + self.h_out[0]["lse"])
        return bi, bo

    def _use_slot(self, k):
        sl = self.slots[k]
        self.inp.q_I, self.inp.w_I, self.k_new = sl["q_I"], sl["w_I"], sl["k_new"]
        self.c_new, self.inp.q = sl["c_new"], sl["q"]
        self.out, self.lse = sl["out"], sl["lse"]

    def e2e_run(self, steps):
        """`steps` decode steps through host buffers, pipelined over two slots: the inputs of
        step i+1 go up (stream s_in) and the outputs of step i-1 come down (stream s_out) while
        step i (the slot's captured graph) computes on the current stream.  Every step's copies
        lie between the returned events."""
        torch = self.torch
        comp = torch.cuda.current_stream()
        ev_in = [torch.cuda.Event() for _ in range(2)]    # the slot's inputs landed
        ev_comp = [torch.cuda.Event() for _ in range(2)]  # the slot's step finished
        ev_out = [torch.cuda.Event() for _ in range(2)]   # the slot's outputs were read back
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(comp)
        self.s_in.wait_event(start)
        self.s_out.wait_event(start)
        h = self.h_in

        def upload(i):
            k = i & 1
            sl = self.slots[k]
            with torch.cuda.stream(self.s_in):
                if i >= 2:
                    self.s_in.wait_event(ev_comp[k])  # step i-2 has read this slot
                sl["q_I"].copy_(h["q_I"], non_blocking=True)
                sl["w_I"].copy_(h["w_I"], non_blocking=True)
                sl["k_new"].copy_(h["k_new"], non_blocking=True)
                for layer in range(len(sl["q"])):
                    sl["c_new"][layer].copy_(h["c_new"][layer], non_blocking=True)
                    sl["q"][layer].copy_(h["q"][layer], non_blocking=True)
                ev_in[k].record(self.s_in)

        upload(0)
        for i in range(steps):
            k = i & 1
            if i + 1 < steps:
                upload(i + 1)
            comp.wait_event(ev_in[k])
            if i >= 2:
                comp.wait_event(ev_out[k])  # step i-2's outputs have left this slot
            self.graphs[k].replay()
            ev_comp[k].record(comp)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(ev_comp[k])
                ho, sl = self.h_out[k], self.slots[k]
                for layer in range(len(sl["out"])):
                    ho["out"][layer].copy_(sl["out"][layer], non_blocking=True)
                    ho["lse"][layer].copy_(sl["lse"][layer], non_blocking=True)
                ev_out[k].record(self.s_out)
        comp.wait_stream(self.s_out)
        end.record(comp)
        return start, end


class PrefillStep:
    """Chunked causal prefill of one sequence: for each chunk of C queries, lsa_index over the
    chunk's rows, then lsa_attend.  tokens/s = L / step time."""

    def __init__(self, cfg, device, rank=0):
        import torch
        from lightning_indexer_top_score_b200 import lsa
        from lightning_indexer_top_score_b200.workloads import DeviceInputs
        self.cfg, self.lsa, self.torch = cfg, lsa, torch
        self.inp = DeviceInputs(cfg, device=device, seed=replica_seed(cfg.seed, rank))
        inp = self.inp
        C = cfg.chunk
        self.chunks = []
        for c0 in range(0, cfg.L, C):
            self.chunks.append((c0, min(cfg.L, c0 + C)))
        self.idx = torch.empty(cfg.B, C, cfg.K_sparse, dtype=torch.int32, device=device)
        self.qpos = [torch.arange(a, b, dtype=torch.int32, device=device).view(1, -1).repeat(
            cfg.B, 1).contiguous() for a, b in self.chunks]
        self.ws_i = torch.empty(lsa.lsa_index_workspace_bytes(
            cfg.B, C, cfg.H_I, cfg.D_I, cfg.cap, cfg.K_sparse, cfg.page, cfg.sub_block, 0),
            dtype=torch.uint8, device=device)
        self.ws_a = torch.empty(max(256, lsa.lsa_attend_workspace_bytes(
            cfg.B, C, cfg.H, 512, cfg.K_sparse, cfg.sink, cfg.swa)), dtype=torch.uint8,
            device=device)
        self.out = torch.empty(cfg.B, cfg.L, cfg.H, 512, dtype=torch.bfloat16, device=device)
        self.lse = torch.empty(cfg.B, cfg.L, cfg.H, dtype=torch.float32, device=device)
        self.devw = torch.zeros(1, dtype=torch.int32, device=device)

    def run(self, ev=None):
        """ev: None, or events for the phase split -- one (index start, index end = attend
        start, attend end) triple per chunk, recorded around each call."""
        lsa, inp, cfg = self.lsa, self.inp, self.cfg
        for j, ((a, b), qp) in enumerate(zip(self.chunks, self.qpos)):
            n = b - a
            if ev is not None:
                ev[3 * j].record()
            lsa.lsa_index(inp.q_I[:, a:b], inp.w_I[:, a:b], inp.k_I, None, inp.kv_len, qp,
                          cfg.K_sparse, cfg.sink, cfg.swa, indices=self.idx[:, :n], ws=self.ws_i)
            if ev is not None:
                ev[3 * j + 1].record()
            lsa.lsa_attend(inp.q[0][:, a:b], inp.c_kv[0], self.idx[:, :n], inp.kv_len, qp,
                           cfg.sink, cfg.swa, cfg.scale, out=self.out[:, a:b],
                           lse=self.lse[:, a:b], ws=self.ws_a)
            if ev is not None:
                ev[3 * j + 2].record()

    def n_events(self):
        return 3 * len(self.chunks)

    def phases(self, evs):
        """Mean per-step milliseconds of the index calls and of the attend calls."""
        ix = [sum(e[3 * j].elapsed_time(e[3 * j + 1]) for j in range(len(self.chunks)))
              for e in evs]
        at = [sum(e[3 * j + 1].elapsed_time(e[3 * j + 2]) for j in range(len(self.chunks)))
              for e in evs]
        return {"index": statistics.mean(ix), "attend": statistics.mean(at)}

    def tokens_per_step(self):
        return self.cfg.B * self.cfg.L

    def check_errors(self):
        return self.lsa.lsa_get_error(self.ws_i) | self.lsa.lsa_get_error(self.ws_a)

    def index_bytes(self):
        return None

    def index_flops(self):
        """2 * H_I * d_I flop per (query, dynamic key): every query t scores its whole dyn."""
        cfg = self.cfg
        t = np.arange(cfg.L, dtype=np.int64)
        dyn = np.maximum(0, t - cfg.swa + 1 - cfg.sink)
        return float(2 * cfg.H_I * cfg.D_I * dyn.sum() * cfg.B)

    def attend_flops(self):
        """2 * H * (576 + 512) flop per (query, attended key): S = q.c over 576 dims, O += p v
        over 512."""
        cfg = self.cfg
        keys = attended_keys(np.arange(cfg.L), cfg.sink, cfg.swa, cfg.K_sparse)
        return float(2 * cfg.H * (576 + 512) * keys.sum() * cfg.B)

    def step_bytes(self):
        """Queries in, outputs out and the fp32 score rows written and read back: each far
        larger than L2 on its own."""
        cfg = self.cfg
        q = cfg.B * cfg.L * (cfg.H_I * cfg.D_I * 2 + cfg.H * 576 * 2)
        out = cfg.B * cfg.L * cfg.H * 512 * 2
        return q + out


class IndexChunkStep:
    """The indexer of one prefill chunk (the paper's Table 4 setting): lsa_index over the last T
    queries of one L-token sequence, hierarchical (M > 0, means built once by lsa_kv_append) or
    flat.  tokens/s = T / step time."""

    def __init__(self, cfg, device, rank=0):
        import torch
        from lightning_indexer_top_score_b200 import lsa
        from lightning_indexer_top_score_b200.workloads import DeviceInputs
        self.cfg, self.lsa, self.torch = cfg, lsa, torch
        self.inp = DeviceInputs(cfg, device=device, seed=replica_seed(cfg.seed, rank),
                                with_attention=False)
        inp = self.inp
        if cfg.M:
            zero = torch.zeros(cfg.B, dtype=torch.int32, device=device)
            lsa.lsa_kv_append(zero, k_I_new=inp.k_I[:, :cfg.L].contiguous(), k_I=inp.k_I,
                              k_mean=inp.k_mean, sub_block=cfg.sub_block)
        self.idx = torch.empty(cfg.B, cfg.T, cfg.K_sparse, dtype=torch.int32, device=device)
        self.ws_i = torch.empty(lsa.lsa_index_workspace_bytes(
            cfg.B, cfg.T, cfg.H_I, cfg.D_I, cfg.cap, cfg.K_sparse, cfg.page, cfg.sub_block, cfg.M),
            dtype=torch.uint8, device=device)

    def run(self, ev=None):
        lsa, inp, cfg = self.lsa, self.inp, self.cfg
        if ev is not None:
            ev[0].record()
        lsa.lsa_index(inp.q_I, inp.w_I, inp.k_I, inp.k_mean if cfg.M else None, inp.kv_len,
                      inp.q_pos, cfg.K_sparse, cfg.sink, cfg.swa, cfg.page, cfg.sub_block, cfg.M,
                      indices=self.idx, ws=self.ws_i)
        if ev is not None:
            ev[1].record()

    def tokens_per_step(self):
        return self.cfg.B * self.cfg.T

    def check_errors(self):
        return self.lsa.lsa_get_error(self.ws_i)

    def index_bytes(self):
        return None

    def step_bytes(self):
        """The chunk's queries, the keys (or means and pages) it scores, and one fp32 score per
        scored (query, key) written and read back."""
        cfg = self.cfg
        per = 2 * cfg.H_I * cfg.D_I
        return int(cfg.B * cfg.T * cfg.H_I * cfg.D_I * 2 + cfg.B * cfg.L * cfg.D_I * 2
                   + 8 * self.index_flops() / per)

    def index_flops(self):
        """Algorithmic flop of the scoring: 2 * H_I * d_I per (query, scored key); flat scores
        each query's dyn, HI scores every mean of its dyn pages plus M pages of tokens."""
        cfg = self.cfg
        per = 2 * cfg.H_I * cfg.D_I
        q_pos = np.arange(cfg.L - cfg.T, cfg.L)
        dyn = np.maximum(0, q_pos - cfg.swa + 1 - cfg.sink)
        if cfg.M == 0:
            return float(per * dyn.sum() * cfg.B)
        means = np.ceil((q_pos - cfg.swa + 1) / cfg.page) * (cfg.page // cfg.sub_block)
        stage2 = np.minimum(dyn, cfg.M * cfg.page)
        return float(per * (means.sum() + stage2.sum()) * cfg.B)


def attended_keys(q_pos, sink, swa, K_sparse):
    """|S_t| of every query position: the sink and window keys that exist at t plus the dynamic
    picks, min(K_sparse, size of the region between them)."""
    t = np.asarray(q_pos, np.int64)
    n_sink = np.minimum(sink, t + 1)
    swa_lo = np.maximum(sink, t - swa + 1)
    n_swa = np.maximum(0, t + 1 - swa_lo)
    n_dyn = np.minimum(K_sparse, np.maximum(0, swa_lo - sink))
    return n_sink + n_swa + n_dyn


class TrainStep:
    """Core attention of one training step (the paper's Table 2 setting): lsa_attend forward,
    then lsa_attend_bwd over the same index sets (taking the forward's out and lse) into a zeroed
    latent-row gradient buffer.  The
    index sets are built once by lsa_index outside the timed region (the table times core
    attention alone).  tokens/s = T / step time."""

    # contraction widths per (head, attended key): S = q.c (576), dP = dO.v (512),
    # dQ += dZ c (576), dC += dZ q (576) + P dO (512)
    BWD_WIDTH = 576 + 512 + 576 + 576 + 512

    def __init__(self, cfg, device, rank=0):
        import torch
        from lightning_indexer_top_score_b200 import lsa
        from lightning_indexer_top_score_b200.workloads import DeviceInputs
        self.cfg, self.lsa, self.torch = cfg, lsa, torch
        self.inp = inp = DeviceInputs(cfg, device=device, seed=replica_seed(cfg.seed, rank))
        B, T, H = cfg.B, cfg.T, cfg.H
        self.idx = torch.empty(B, T, cfg.K_sparse, dtype=torch.int32, device=device)
        C = 512
        ws_i = torch.empty(lsa.lsa_index_workspace_bytes(
            B, C, cfg.H_I, cfg.D_I, cfg.cap, cfg.K_sparse, cfg.page, cfg.sub_block, 0),
            dtype=torch.uint8, device=device)
        for a in range(0, T, C):
            b = min(T, a + C)
            lsa.lsa_index(inp.q_I[:, a:b], inp.w_I[:, a:b], inp.k_I, None, inp.kv_len,
                          inp.q_pos[:, a:b], cfg.K_sparse, cfg.sink, cfg.swa,
                          indices=self.idx[:, a:b], ws=ws_i)
        if lsa.lsa_get_error(ws_i):
            raise SystemExit("device error while building the index sets")
        del ws_i
        g = torch.Generator(device=device)
        g.manual_seed(replica_seed(cfg.seed + 11, rank))
        self.dout = torch.randn(B, T, H, 512, generator=g, device=device).to(torch.bfloat16)
        self.ws_a = torch.empty(max(256, lsa.lsa_attend_workspace_bytes(
            B, T, H, 512, cfg.K_sparse, cfg.sink, cfg.swa)), dtype=torch.uint8, device=device)
        self.out = torch.empty(B, T, H, 512, dtype=torch.bfloat16, device=device)
        self.lse = torch.empty(B, T, H, dtype=torch.float32, device=device)
        self.dq = torch.empty(B, T, H, 576, dtype=torch.float32, device=device)
        self.dc = torch.empty(B, cfg.cap, 576, dtype=torch.float32, device=device)
        self.devw = torch.zeros(1, dtype=torch.int32, device=device)

    def run(self, ev=None):
        lsa, inp, cfg = self.lsa, self.inp, self.cfg
        if ev is not None:
            ev[0].record()
        lsa.lsa_attend(inp.q[0], inp.c_kv[0], self.idx, inp.kv_len, inp.q_pos, cfg.sink,
                       cfg.swa, cfg.scale, out=self.out, lse=self.lse, ws=self.ws_a)
        if ev is not None:
            ev[1].record()
        self.dc.zero_()
        lsa.lsa_attend_bwd(inp.q[0], inp.c_kv[0], self.idx, inp.kv_len, inp.q_pos, cfg.sink,
                           cfg.swa, cfg.scale, self.dout, out=self.out, lse=self.lse, dq=self.dq,
                           dc_kv=self.dc, device_error=self.devw)
        if ev is not None:
            ev[2].record()

    def tokens_per_step(self):
        return self.cfg.B * self.cfg.T

    def step_bytes(self):
        """Queries, output gradients and dq: each far larger than L2."""
        cfg = self.cfg
        return cfg.B * cfg.T * cfg.H * (576 * 2 + 512 * 2 + 576 * 4)

    def check_errors(self):
        return self.lsa.lsa_get_error(self.ws_a) | int(self.devw.item())

    def index_bytes(self):
        return None

    def bwd_flops(self):
        """Algorithmic flop of the backward: 2 x BWD_WIDTH per (query, head, attended key)."""
        cfg = self.cfg
        n = attended_keys(self.inp.q_pos.cpu().numpy(), cfg.sink, cfg.swa, cfg.K_sparse)
        return float(2 * self.BWD_WIDTH * cfg.H * n.sum())


# ----------------------------------------------------------------------------- CPU oracle arm

def _bits(t) -> np.ndarray:
    import torch
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def cpu_units(cfg, step=None, n_distinct=8, seed=0):
    """Host copies of a few work units of the workload for the CPU oracle.  Decode: one unit =
    one sequence with its query (copied from the device inputs the GPU timed).  Prefill: one
    unit = one query row at a random position of the sequence (host-generated, same recipe)."""
    rng = np.random.default_rng(seed)
    units = []
    if step is not None and hasattr(step, "e2e_setup"):
        inp = step.inp
        for b in rng.permutation(cfg.B)[:n_distinct]:
            b = int(b)
            units.append(dict(q_I=_bits(inp.q_I[b:b + 1]), w_I=_bits(inp.w_I[b:b + 1]),
                              k_I=_bits(inp.k_I[b:b + 1]), q=[_bits(q[b:b + 1]) for q in inp.q],
                              c=[_bits(c[b:b + 1]) for c in inp.c_kv],
                              kv=inp.kv_len[b:b + 1].cpu().numpy(),
                              qp=inp.q_pos[b:b + 1].cpu().numpy(),
                              km=(_bits(step.k_minmax[b:b + 1]) if getattr(step, "minmax", False)
                                  else _bits(inp.k_mean[b:b + 1]) if cfg.M else None),
                              pooling="minmax" if getattr(step, "minmax", False) else "mean"))
        return units, "decode"
    from dataclasses import replace
    from lightning_indexer_top_score_b200.workloads import make_host_inputs
    if cfg.name.startswith("hfa_train"):
        # one unit = one query row's core attention, forward + backward.  Its cost depends only
        # on |S_t|, so the rows come from a 16384-token host sequence at positions with the same
        # |S_t| as the workload's rows; the index sets are built here, outside the timing.
        import oracle
        from lightning_indexer_top_score_b200.workloads import bf16_bits_to_f32, to_bf16_bits
        oracle.build()
        Ls = min(cfg.L, 16384)
        small = replace(cfg, B=1, T=1, L=Ls, n_needles=0)
        h = make_host_inputs(small, q_pos=np.array([[Ls - 1]], np.int32))
        for _ in range(n_distinct):
            t = int(rng.integers(max(0, Ls - cfg.T), Ls)) if cfg.L <= Ls else Ls - 1
            qp = np.array([[t]], np.int32)
            idx = oracle.index(h.q_I, h.w_I, h.k_I, None, h.kv_len, qp, cfg.K_sparse, cfg.sink,
                               cfg.swa)
            dout = bf16_bits_to_f32(to_bf16_bits(
                rng.standard_normal((1, 1, cfg.H, 512)).astype(np.float32))).astype(np.float64)
            units.append(dict(q=h.q, c=h.c_kv, qp=qp, idx=idx, dout=dout))
        return units, "training"
    small = replace(cfg, B=1, T=1, n_needles=0)
    h = make_host_inputs(small, q_pos=np.array([[cfg.L - 1]], np.int32))
    km = None
    if cfg.M:
        # the stored means the GPU path keeps (bf16 of the fp64 sub-block means)
        import oracle
        from lightning_indexer_top_score_b200.workloads import to_bf16_bits
        oracle.build()
        km = to_bf16_bits(oracle.block_means(h.k_I[0], cfg.L, cfg.sub_block))[None]
    if cfg.T > 1:
        # prefill rows differ in cost (query t scores its whole prefix): stratified positions,
        # one per stratum of [0, L), visited in random order
        n = max(n_distinct, 256)
        ts = [int((i + rng.random()) * cfg.L / n) for i in rng.permutation(n)]
    else:
        ts = [cfg.L - 1] * n_distinct
    for t in ts:
        units.append(dict(q_I=h.q_I, w_I=h.w_I, k_I=h.k_I, q=h.q, c=h.c_kv, kv=h.kv_len,
                          qp=np.array([[t]], np.int32), km=km))
    return units, "prefill" if cfg.T > 1 else "decode"


def _unit_work(kind):
    return ("core attention forward + backward" if kind == "training"
            else "indexer + attention of every layer")


def cpu_oracle_sample(cfg, units, budget_s=15.0):
    """Time the fp64 CPU oracle on the sampled units (the whole layer path of each: indexer +
    attention of every layer).  One single-threaded oracle call per host core at a time (threads
    share the units' arrays), waves until budget_s of wall time is used."""
    import concurrent.futures as cf
    import oracle
    oracle.build()
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    layers = max(1, len(units[0]["q"]))

    def work(u):
        oracle.set_num_threads(1)
        if "dout" in u:
            oracle.attend(u["q"][0], u["c"][0], u["idx"], u["qp"], cfg.sink, cfg.swa, 512,
                          cfg.scale)
            oracle.attend_bwd(u["q"][0], u["c"][0], u["idx"], u["qp"], cfg.sink, cfg.swa, 512,
                              cfg.scale, u["dout"])
            return 1
        idx = oracle.index(u["q_I"], u["w_I"], u["k_I"], u["km"], u["kv"], u["qp"], cfg.K_sparse,
                           cfg.sink, cfg.swa, cfg.page, cfg.sub_block, cfg.M,
                           pooling=u.get("pooling", "mean"))
        for l in range(layers):
            oracle.attend(u["q"][l], u["c"][l], idx, u["qp"], cfg.sink, cfg.swa, 512, cfg.scale)
        return 1

    done, pos = 0, 0
    t0 = time.perf_counter()
    with cf.ThreadPoolExecutor(max_workers=cores) as ex:
        while True:
            wave = [units[(pos + i) % len(units)] for i in range(cores)]
            pos += cores
            done += sum(ex.map(work, wave))
            if time.perf_counter() - t0 >= budget_s:
                break
    wall = time.perf_counter() - t0
    return {"rows": done, "seconds": wall, "cores": cores, "layers": layers,
            "tokens_per_s": done * layers / wall}


# ----------------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode_128k")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch size")
    ap.add_argument("--queries", type=int, default=0,
                    help="override the workload's queries per sequence (small profiling cases)")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch every call eagerly instead of replaying a captured CUDA graph")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    cfg = workload_config(args.workload)
    if args.batch:
        from dataclasses import replace
        cfg = replace(cfg, B=args.batch, name=f"{cfg.name}_b{args.batch}")
    if args.queries:
        from dataclasses import replace
        cfg = replace(cfg, T=args.queries, name=f"{cfg.name}_q{args.queries}")
    metric = ("LSA layer prefill tokens/s" if args.workload.startswith("prefill")
              else "LSA indexer prefill-chunk tokens/s" if args.workload.startswith("index_chunk_")
              else "HFA core-attention training (fwd+bwd) tokens/s"
              if args.workload.startswith("train_")
              else "LSA layer decode tokens/s")
    config = {"workload": cfg.name, "B": cfg.B, "L": cfg.L, "T": cfg.T, "H_I": cfg.H_I,
              "d_I": cfg.D_I, "H": cfg.H, "K": cfg.K, "sink": cfg.sink, "swa": cfg.swa,
              "K_sparse": cfg.K_sparse, "page": cfg.page, "sub_block": cfg.sub_block, "M": cfg.M,
              "layers": cfg.layers, "chunk": cfg.chunk}

    if args.impl == "reference":
        if rank != 0:
            return
        units, kind = cpu_units(cfg, None, n_distinct=2)
        # one step = one wave of query rows, one row per host core (the smallest sample that
        # keeps every core busy), so that the run's length grows only with K + W
        times = []
        for i in range(args.warmup + args.steps):
            res = cpu_oracle_sample(cfg, units, budget_s=0.0)
            if i >= args.warmup:
                times.append(res)
        tok = sum(r["rows"] * r["layers"] for r in times)
        sec = sum(r["seconds"] for r in times)
        v = tok / sec
        line = {"impl": "reference", "metric": metric, "value": v, "unit": "tokens/s",
                "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": 1000 * sec / len(times), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": config,
                "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": times[0]["cores"],
                                 "kind": "oracle",
                                 "sample": f"{times[0]['rows']} {kind} query rows per step, one "
                                           f"per core ({_unit_work(kind)} of each), same "
                                           f"shapes"},
                "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    import torch
    import torch.distributed as dist
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    device = f"cuda:{local}"
    torch.cuda.set_device(local)
    from lightning_indexer_top_score_b200 import build as lsa_build
    if not os.path.exists(lsa_build.LIB):
        lsa_build.build()

    if args.workload.startswith("prefill"):
        step = PrefillStep(cfg, device, rank)
    elif args.workload.startswith("index_chunk_"):
        step = IndexChunkStep(cfg, device, rank)
    elif args.workload.startswith("train_"):
        step = TrainStep(cfg, device, rank)
    else:
        step = DecodeStep(cfg, device, rank, fp8=args.workload.endswith("_fp8"),
                          minmax=args.workload.startswith("table11_minmax"))
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step.run()
    barrier()
    err = step.check_errors()
    if err:
        raise SystemExit(f"device error word {err:#x} after warm-up")

    # L2 policy: a step that reads less than twice the L2 capacity is timed one step at a time
    # with a write of a buffer larger than L2 between steps (outside the timed events); larger
    # steps run back to back, their inputs evicting each other
    sb = int(step.step_bytes())
    flush = sb < 2 * L2_BYTES
    flush_buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=device) if flush else None
    config["l2"] = (f"L2 flushed between timed steps (a step reads {sb / 1e6:.1f} MB, L2 "
                    f"{L2_BYTES / 2 ** 20:.0f} MiB)" if flush else
                    f"no flush: a step reads {sb / 1e6:.1f} MB, more than twice the "
                    f"{L2_BYTES / 2 ** 20:.0f} MiB L2")

    n_layers = len(step.inp.q)
    n_ev = (3 + n_layers if isinstance(step, DecodeStep) else 3 if isinstance(step, TrainStep)
            else step.n_events() if isinstance(step, PrefillStep) else 2)
    # The decode step (about a dozen short kernels) is captured once into a CUDA graph and
    # replayed, which removes host launch gaps; phase events are recorded in the eager run.
    graph = None
    if isinstance(step, DecodeStep) and not args.no_graph:
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            step.run()  # warm the capture stream
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=side):
                step.run()
        torch.cuda.synchronize()
        for _ in range(args.warmup):
            graph.replay()
        barrier()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    # phases (eager launches, same kernels), timed outside the headline region; the library's
    # own launch counter gives the kernels one step launches
    n0 = step.lsa.lsa_launch_count()
    for i in range(args.steps):
        step.run(evs[i])
    barrier()
    launches_per_step = (step.lsa.lsa_launch_count() - n0) // args.steps
    end = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    barrier()
    start = torch.cuda.Event(enable_timing=True)
    if flush:
        # per-step events; the L2 flush between steps lies outside them
        marks = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in range(args.steps)]
        for i in range(args.steps):
            flush_buf.fill_(i & 0xFF)
            marks[i][0].record(stream)
            if graph is not None:
                graph.replay()
            else:
                step.run()
            marks[i][1].record(stream)
        barrier()
        local_ms = sum(a_.elapsed_time(b_) for a_, b_ in marks)
    else:
        start.record(stream)
        for i in range(args.steps):
            if graph is not None:
                graph.replay()
            else:
                step.run()
        end.record(stream)
        barrier()
        local_ms = start.elapsed_time(end)
    clk = clocks.stop()
    total_ms = max_over_ranks(local_ms, world, device)
    ms_step = total_ms / args.steps
    phases = {}
    names = (["append", "index"] + (["attend_owner", "attend_reuse"] if n_layers == 2 else
                                    [f"attend_{i}" for i in range(n_layers)])
             if isinstance(step, DecodeStep) else
             ["index"] if isinstance(step, IndexChunkStep) else
             ["fwd", "bwd"] if isinstance(step, TrainStep) else ["step"])
    if isinstance(step, PrefillStep):
        phases = step.phases(evs)
    else:
        for j, nm in enumerate(names):
            phases[nm] = statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs)
    value = job_rate(step.tokens_per_step(), world, args.steps, total_ms)

    # ---- end-to-end through host buffers
    e2e = None
    if isinstance(step, DecodeStep):
        bi, bo = step.e2e_setup()
        step.e2e_run(3)
        barrier()
        s0, s1 = step.e2e_run(args.steps)
        barrier()
        te = max_over_ranks(s0.elapsed_time(s1), world, device)
        # every step had the same inputs: both slots must have read back the same bytes
        for a_, b_ in zip(step.h_out[0]["out"] + step.h_out[0]["lse"],
                          step.h_out[1]["out"] + step.h_out[1]["lse"]):
            if not torch.equal(a_, b_):
                raise SystemExit("end-to-end slots disagree")
        e2e = {"value": job_rate(step.tokens_per_step(), world, args.steps, te),
               "unit": "tokens/s", "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo}

    peaks, peak_kind = load_peaks()
    roofline = None
    if isinstance(step, IndexChunkStep):
        # the scoring contraction of a whole chunk is tensor-bound; each lsa_index call is an
        # isolated launch group of a few milliseconds, so the burst bf16 peak is the denominator
        fl = step.index_flops()
        achieved = fl / (phases["index"] / 1000.0) / 1e12
        peak = float(peaks["bf16_tflops"])
        roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "traffic": None,
                    "kernel": "lsa_index over the chunk (timed as the whole call)",
                    "peak_kind": peak_kind + " (burst)", "algorithmic_flops": fl}
    if isinstance(step, PrefillStep):
        # both passes are bf16 contractions; the roofline object describes the one that takes
        # longer, and the other pass's rate is reported beside it.  The step runs for tens of
        # milliseconds, so the sustained bf16 peak is the denominator
        peak = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
        rates = {"index": step.index_flops(), "attend": step.attend_flops()}
        dom = max(rates, key=lambda k: phases[k])
        other = "attend" if dom == "index" else "index"
        achieved = rates[dom] / (phases[dom] / 1000.0) / 1e12
        roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "traffic": None,
                    "kernel": (f"lsa_{dom} over the 8 chunks (timed as whole calls)"),
                    "peak_kind": peak_kind + " (sustained)", "algorithmic_flops": rates[dom],
                    "other_pass": {"pass": f"lsa_{other}",
                                   "achieved": rates[other] / (phases[other] / 1000.0) / 1e12,
                                   "algorithmic_flops": rates[other]}}
    if isinstance(step, TrainStep):
        # the backward dominates: bf16 tensor-core contractions inside a step of 100+ ms, so the
        # sustained bf16 peak is the denominator
        fl = step.bwd_flops()
        achieved = fl / (phases["bwd"] / 1000.0) / 1e12
        peak = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
        roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "traffic": None,
                    "kernel": "hfa_bwd_kernel (timed with the gradient zeroing before it)",
                    "peak_kind": peak_kind + " (sustained)", "algorithmic_flops": fl}
    ib = step.index_bytes()
    if ib is not None and "index" in phases:
        achieved = ib / (phases["index"] / 1000.0) / 1e9
        peak = float(peaks["hbm_gbs"])
        traffic, how = scorer_traffic(cfg.name)
        roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                    "frac": achieved / peak, "traffic": traffic,
                    "kernel": "lsa_index decode scoring pass (timed as the whole lsa_index call)",
                    "traffic_source": how, "peak_kind": peak_kind, "algorithmic_bytes": ib}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not isinstance(step,
                                                                          IndexChunkStep):
        try:
            units, kind = cpu_units(cfg, step)
            res = cpu_oracle_sample(cfg, units, budget_s=args.cpu_budget)
            cpu = {"value": res["tokens_per_s"], "unit": "tokens/s", "cores": res["cores"],
                   "kind": "oracle",
                   "sample": f"{res['rows']} {kind} query rows ({_unit_work(kind)}, drawn "
                             f"from {len(units)} sequences/positions of this workload), "
                             f"{res['seconds']:.1f} s of CPU time"}
            if kind == "prefill":
                cpu["extrapolated"] = ("rows/s over stratified query positions of the prefill; "
                                       "each row is one prefill token, so tokens/s = rows/s")
        except Exception as ex:  # the baseline is reported, never required
            cpu = {"value": None, "unit": "tokens/s", "cores": None, "kind": "oracle",
                   "sample": f"failed: {ex!r}"}

    if rank == 0:
        line = {"metric": metric, "value": value, "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": ("e4m3 indexer, bf16 attention" if getattr(step, "fp8", False)
                          else "bf16"),
                "data": "synthetic (seeded; no dataset)", "config": config,
                "parallelism": f"replicas x{world} (independent sequences per GPU)",
                "phases_ms": phases, "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": launches_per_step * args.steps, "clocks": clk}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

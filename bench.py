#!/usr/bin/env python
"""Throughput of the compressed-KV hot path on B200, as one JSON line.

Default workload (one step): the write path of an 8B-dense-shaped layer --
B=8 sequences x 8 KV heads x 32,768 tokens x d=128, bf16 K/V compressed to
K = 4-bit Lloyd-Max + 1-bit QJL and V = 4-bit -- followed by one GQA decode
step (32 query heads) over the cache it just wrote.  Metric: KV vectors
encoded plus (query-head, key) pairs scored, per second; the encode and
decode parts and their HBM roofline fractions are reported alongside.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload step|decode32k|longctx|search]

Multi-GPU runs are replicas (the path has no exchange step): each rank
repeats the same per-GPU work, value = all ranks' units / max rank time.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "KV vectors encoded/s + decode-attn keys scored/s; % HBM roofline (1 B200)"
EXTRA_METRICS = {"decode32k": "decode-attn keys scored/s", "longctx": "decode + prefill (query-head, key) pairs/s",
                 "search": "database vectors scored per query per second (top-10 search)"}
UNIT_NOTES = {"step": "units = KV vectors encoded + (query-head, key) pairs scored",
              "decode32k": "units = (query-head, key) pairs scored",
              "longctx": "units = (query-head, key) pairs scored in the decode step and the prefill chunk",
              "search": "units = (query, database vector) pairs scored"}
FALLBACK_HBM_GBS = 6650.0


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), float(j.get("bf16_tflops", 1631.1)), float(j.get("bf16_tflops_sustained", 1375.3)), "measured"
    return FALLBACK_HBM_GBS, 1590.0, 1400.0, "fallback"


# --------------------------------------------------------------------------
# distributed plumbing (replicas)
# --------------------------------------------------------------------------
def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def reduce_max(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"      # gloo: host tensors
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(units_per_rank: float, times_s: list[float]) -> tuple[float, float]:
    """Whole-job throughput of replicas: all ranks' units over the slowest rank's time."""
    t = max(times_s)
    return units_per_rank * len(times_s) / t, t


# --------------------------------------------------------------------------
# clocks sampled during the timed region
# --------------------------------------------------------------------------
class ClockSampler:
    """SM clock, power and throttle reasons while the timed region runs.

    NVML (read-only queries) is polled from a thread about every millisecond,
    so even a region of a few milliseconds yields samples; without NVML,
    nvidia-smi at its 200 ms rate.  Nothing here changes a GPU setting."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.path = None
        self.thread = None
        self.nvml = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.sel = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        except Exception:
            self.sel = str(device_index)
        try:
            import pynvml
            pynvml.nvmlInit()
            try:
                h = pynvml.nvmlDeviceGetHandleByUUID(self.sel)
            except Exception:
                h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nvml, self.handle = pynvml, h
            self.bits = {"hw_slowdown": pynvml.nvmlClocksEventReasonHwSlowdown,
                         "hw_thermal_slowdown": pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                         "sw_thermal_slowdown": pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                         "sw_power_cap": pynvml.nvmlClocksEventReasonSwPowerCap}
        except Exception:
            self.nvml = None

    def _poll(self):
        nv, h = self.nvml, self.handle
        while not self.done.is_set():
            try:
                self.sm.append(float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)))
                self.power.append(nv.nvmlDeviceGetPowerUsage(h) / 1000.0)
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                for n, b in self.bits.items():
                    if r & b:
                        self.reasons.add(n)
            except Exception:
                pass
            self.done.wait(0.001)

    def start(self):
        import threading
        self.sm, self.power, self.reasons = [], [], set()
        if self.nvml is not None:
            try:
                self.smax = float(self.nvml.nvmlDeviceGetMaxClockInfo(self.handle, self.nvml.NVML_CLOCK_SM))
            except Exception:
                self.smax = None
            self.done = threading.Event()
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.sel, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200", "-f", self.path],
                                         stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def _result(self, sm, smax, power, source):
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(self.reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None, "source": source}

    def stop(self) -> dict:
        if self.thread is not None:
            self.done.set()
            self.thread.join(timeout=5)
            return self._result(self.sm, self.smax, self.power, "nvml, 1 ms polling")
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, power = [], [], []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                    power.append(float(parts[3]))
                except ValueError:
                    continue
                for n, v in zip(self.NAMES, parts[5:9]):
                    if v.lower().startswith("active"):
                        self.reasons.add(n)
        os.unlink(self.path)
        return self._result(sm, max(smax) if smax else None, power, "nvidia-smi, 200 ms")


# --------------------------------------------------------------------------
# workloads
# --------------------------------------------------------------------------
class StepWorkload:
    """Write path (B=8, Hkv=8, 32,768 tokens, d=128; K 4-bit + QJL, V 4-bit)
    plus one GQA decode step (Hq=32) over the written cache."""
    name = ("write path B=8 x Hkv=8 x 32768 tokens x d=128 bf16 (K 4-bit Lloyd-Max + 1-bit QJL, V 4-bit) "
            "+ one GQA decode step Hq=32 over the written cache")

    def __init__(self, dev, batch=8, **_):
        from kv_cache_vector_07_b200 import synth, tqkv
        self.tq = tqkv
        B, L, H, Hq, d, P = batch, 32768, 8, 32, 128, 64
        if batch != 8:
            self.name = self.name.replace("B=8", f"B={batch}")
        self.B, self.L, self.H, self.Hq, self.d, self.P = B, L, H, Hq, d, P
        n = B * L
        self.n_vec = 2 * n * H
        self.n_pairs = B * Hq * L
        self.units = self.n_vec + self.n_pairs
        self.desc = tqkv.cache_desc(d, 4, True, 4, page_tokens=P, n_kv_heads=H)
        self.kp = tqkv.make_params(d, 4, 1001)
        self.vp = tqkv.make_params(d, 4, 2001)
        self.K = synth.lognormal_channels(n, H, d, seed=1, device=dev)
        self.V = synth.lognormal_channels(n, H, d, seed=10001, device=dev)
        self.Q = synth.normal((B, Hq, d), seed=12, device=dev)
        self.bt, self.slots, nblk = synth.contiguous_block_table(B, L, P, device=dev, shuffle_seed=11)
        self.seq = torch.full((B,), L, dtype=torch.int32, device=dev)
        self.cache = tqkv.alloc_cache(self.desc, nblk, device=dev)
        self.ws_e = torch.zeros(tqkv.encode_workspace_bytes(self.desc, n), dtype=torch.uint8, device=dev)
        self.ws_d = torch.zeros(tqkv.decode_workspace_bytes(self.desc, B, Hq, L), dtype=torch.uint8, device=dev)
        self.out = torch.empty_like(self.Q)
        page = tqkv.cache_bytes(self.desc)
        per_tok = page // P
        self.enc_bytes = 2 * n * H * d * 2 + n * H * per_tok
        self.dec_bytes = B * H * L * per_tok + 2 * self.Q.numel() * 2
        self.launches = {"encode": 1, "decode": 3}       # decode: fused query prep, dec128, combine

    def ops(self):
        tq = self.tq
        return [("encode", lambda: tq.encode(self.kp, self.vp, self.desc, self.K, self.V, self.slots, self.cache,
                                              workspace=self.ws_e)),
                ("decode", lambda: tq.decode_attn(self.kp, self.vp, self.desc, self.Q, self.bt, self.seq, self.L,
                                                  self.cache, out=self.out, workspace=self.ws_d))]

    def host_io(self):
        """Pinned host copies of the per-step inputs and output, for e2e."""
        h = {name: t.cpu().pin_memory() for name, t in
             (("K", self.K), ("V", self.V), ("Q", self.Q), ("slots", self.slots), ("bt", self.bt),
              ("seq", self.seq))}
        out_h = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in h.values())
        d2h = out_h.numel() * out_h.element_size()

        def step():
            self.K.copy_(h["K"], non_blocking=True)
            self.V.copy_(h["V"], non_blocking=True)
            self.Q.copy_(h["Q"], non_blocking=True)
            self.slots.copy_(h["slots"], non_blocking=True)
            self.bt.copy_(h["bt"], non_blocking=True)
            self.seq.copy_(h["seq"], non_blocking=True)
            for _, f in self.ops():
                f()
            out_h.copy_(self.out, non_blocking=True)
        return step, h2d, d2h

    def roofline(self, op_ms: dict, hbm_peak: float):
        enc_gbs = self.enc_bytes / (op_ms["encode"] * 1e-3) / 1e9
        dec_gbs = self.dec_bytes / (op_ms["decode"] * 1e-3) / 1e9
        return ({"bound": "hbm", "achieved": round(enc_gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                 "frac": round(enc_gbs / hbm_peak, 4), "traffic": traffic_for("step/encode") if self.default_size else None,
                 "kernel": "tq_encode (encode128_kernel: TMA + tcgen05 rotation + quantize + tcgen05 QJL)",
                 "algorithmic_bytes": self.enc_bytes},
                {"encode": {"vectors_per_s": self.n_vec / (op_ms["encode"] * 1e-3), "ms": op_ms["encode"],
                            "gbs": enc_gbs, "frac": enc_gbs / hbm_peak, "algorithmic_bytes": self.enc_bytes},
                 "decode": {"keys_scored_per_s": self.n_pairs / (op_ms["decode"] * 1e-3), "ms": op_ms["decode"],
                            "gbs": dec_gbs, "frac": dec_gbs / hbm_peak, "algorithmic_bytes": self.dec_bytes,
                            "traffic": traffic_for("step/decode") if self.default_size else None}})

    def config(self):
        return {"workload": self.name, "batch": self.B, "seq_len": self.L, "n_kv_heads": self.H,
                "n_q_heads": self.Hq, "head_dim": self.d, "page_tokens": self.P, "preset": "K4+QJL/V4",
                "l2": "inputs larger than L2 (1.07 GB of bf16 K/V per step)", "parallelism": "replicas"}


class Decode32kWorkload:
    """One GQA decode step: B=32, Hq=32 over Hkv=8, L=32,768, K 2-bit + QJL, V 4-bit."""
    name = "decode B=32 x Hq=32/Hkv=8 x 32768 tokens x d=128, K 2-bit Lloyd-Max + 1-bit QJL, V 4-bit (k3v4)"

    def __init__(self, dev, batch=32, seq_len=32768, **_):
        from kv_cache_vector_07_b200 import synth, tqkv
        self.tq = tqkv
        B, L, H, Hq, d, P = batch, seq_len, 8, 32, 128, 64
        if (batch, seq_len) != (32, 32768):
            self.name = self.name.replace("B=32", f"B={batch}").replace("32768 tokens", f"{seq_len} tokens")
        self.B, self.L, self.H, self.Hq, self.d, self.P = B, L, H, Hq, d, P
        n = B * L
        self.desc = tqkv.cache_desc(d, 2, True, 4, page_tokens=P, n_kv_heads=H)
        self.kp = tqkv.make_params(d, 2, 1002)
        self.vp = tqkv.make_params(d, 4, 2002)
        self.bt, slots, nblk = synth.contiguous_block_table(B, L, P, device=dev, shuffle_seed=22)
        self.cache = tqkv.alloc_cache(self.desc, nblk, device=dev)
        step = 1 << 17
        for t0 in range(0, n, step):        # pre-encode the cache in chunks
            K = synth.outlier_normal((min(step, n - t0), H, d), seed=2 + t0, device=dev)
            V = synth.outlier_normal((min(step, n - t0), H, d), seed=20002 + t0, device=dev)
            tqkv.encode(self.kp, self.vp, self.desc, K, V, slots[t0:t0 + step].contiguous(), self.cache)
        torch.cuda.synchronize()
        self.Q = synth.normal((B, Hq, d), seed=21, device=dev)
        self.seq = torch.full((B,), L, dtype=torch.int32, device=dev)
        self.out = torch.empty_like(self.Q)
        self.ws_d = torch.zeros(tqkv.decode_workspace_bytes(self.desc, B, Hq, L), dtype=torch.uint8, device=dev)
        self.units = B * Hq * L
        self.dec_bytes = B * H * L * (tqkv.cache_bytes(self.desc) // P) + 2 * self.Q.numel() * 2
        self.launches = {"decode": 3}                    # fused query prep, dec128, combine

    def ops(self):
        tq = self.tq
        return [("decode", lambda: tq.decode_attn(self.kp, self.vp, self.desc, self.Q, self.bt, self.seq, self.L,
                                                  self.cache, out=self.out, workspace=self.ws_d))]

    def host_io(self):
        h = {"Q": self.Q.cpu().pin_memory(), "bt": self.bt.cpu().pin_memory(), "seq": self.seq.cpu().pin_memory()}
        out_h = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()

        def step():
            self.Q.copy_(h["Q"], non_blocking=True)
            self.bt.copy_(h["bt"], non_blocking=True)
            self.seq.copy_(h["seq"], non_blocking=True)
            self.ops()[0][1]()
            out_h.copy_(self.out, non_blocking=True)
        return step, sum(t.numel() * t.element_size() for t in h.values()), out_h.numel() * out_h.element_size()

    def roofline(self, op_ms, hbm_peak):
        gbs = self.dec_bytes / (op_ms["decode"] * 1e-3) / 1e9
        return ({"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                 "frac": round(gbs / hbm_peak, 4), "traffic": traffic_for("decode32k/decode") if self.default_size else None,
                 "kernel": "tq_decode_attn (prep + attn + combine)", "algorithmic_bytes": self.dec_bytes},
                {"decode": {"keys_scored_per_s": self.units / (op_ms["decode"] * 1e-3), "ms": op_ms["decode"],
                            "gbs": gbs, "frac": gbs / hbm_peak}})

    def config(self):
        return {"workload": self.name, "batch": self.B, "seq_len": self.L, "n_kv_heads": self.H,
                "n_q_heads": self.Hq, "head_dim": self.d, "page_tokens": self.P, "preset": "k3v4",
                "l2": "cache (0.99 GB) larger than L2", "parallelism": "replicas"}


class LongCtxWorkload:
    """Long-context GQA: B=1, Hq=32 over Hkv=4, L=262,144, K 2-bit + QJL, V
    3-bit; one decode step plus one 2,048-query prefill chunk (causal inside)."""
    name = ("long context B=1 x Hq=32/Hkv=4 x 262144 tokens x d=128 (K 2-bit + QJL, V 3-bit): "
            "one decode step + one 2048-query prefill chunk")

    def __init__(self, dev, seq_len=262144, chunk=2048, **_):
        from kv_cache_vector_07_b200 import synth, tqkv
        self.tq = tqkv
        L, H, Hq, d, P, C = seq_len, 4, 32, 128, 64, chunk
        self.L, self.H, self.Hq, self.d, self.P, self.C = L, H, Hq, d, P, C
        self.desc = tqkv.cache_desc(d, 2, True, 3, page_tokens=P, n_kv_heads=H)
        self.kp = tqkv.make_params(d, 2, 1003)
        self.vp = tqkv.make_params(d, 3, 2003)
        self.bt, slots, nblk = synth.contiguous_block_table(1, L, P, device=dev, shuffle_seed=33)
        self.cache = tqkv.alloc_cache(self.desc, nblk, device=dev)
        step = 1 << 16
        for t0 in range(0, L, step):
            K = synth.outlier_normal((min(step, L - t0), H, d), seed=3 + t0, device=dev)
            V = synth.outlier_normal((min(step, L - t0), H, d), seed=30003 + t0, device=dev)
            tqkv.encode(self.kp, self.vp, self.desc, K, V, slots[t0:t0 + step].contiguous(), self.cache)
        torch.cuda.synchronize()
        self.Qd = synth.normal((1, Hq, d), seed=31, device=dev)
        self.Qp = synth.normal((C, Hq, d), seed=32, device=dev)
        self.seq = torch.full((1,), L, dtype=torch.int32, device=dev)
        self.out_d = torch.empty_like(self.Qd)
        self.out_p = torch.empty_like(self.Qp)
        self.ws_d = torch.zeros(tqkv.decode_workspace_bytes(self.desc, 1, Hq, L), dtype=torch.uint8, device=dev)
        self.ws_p = torch.zeros(tqkv.prefill_workspace_bytes(self.desc, C, Hq, L), dtype=torch.uint8, device=dev)
        per_tok = tqkv.cache_bytes(self.desc) // P
        self.dec_pairs = Hq * L
        self.pre_pairs = Hq * sum(L - C + j + 1 for j in range(C))
        self.units = self.dec_pairs + self.pre_pairs
        self.dec_bytes = H * L * per_tok
        self.pre_flops = self.pre_pairs * 2 * (2 * d + d)       # QK^T over 256 features + PV over 128
        self.launches = {"decode": 3, "prefill": 3}      # each: fused query prep, dec128 / pf128, combine

    def ops(self):
        tq = self.tq
        return [("decode", lambda: tq.decode_attn(self.kp, self.vp, self.desc, self.Qd, self.bt, self.seq, self.L,
                                                  self.cache, out=self.out_d, workspace=self.ws_d)),
                ("prefill", lambda: tq.prefill_attn(self.kp, self.vp, self.desc, self.Qp, self.bt.view(-1), self.L,
                                                    self.cache, out=self.out_p, workspace=self.ws_p))]

    def host_io(self):
        h = {"Qd": self.Qd.cpu().pin_memory(), "Qp": self.Qp.cpu().pin_memory()}
        od = torch.empty(self.out_d.shape, dtype=self.out_d.dtype).pin_memory()
        op = torch.empty(self.out_p.shape, dtype=self.out_p.dtype).pin_memory()

        def step():
            self.Qd.copy_(h["Qd"], non_blocking=True)
            self.Qp.copy_(h["Qp"], non_blocking=True)
            for _, f in self.ops():
                f()
            od.copy_(self.out_d, non_blocking=True)
            op.copy_(self.out_p, non_blocking=True)
        return step, sum(t.numel() * t.element_size() for t in h.values()), (od.numel() + op.numel()) * 2

    def roofline(self, op_ms, hbm_peak):
        _, tfl, tfl_s, _ = _peaks()
        tf = self.pre_flops / (op_ms["prefill"] * 1e-3) / 1e12
        gbs = self.dec_bytes / (op_ms["decode"] * 1e-3) / 1e9
        return ({"bound": "tensor", "achieved": round(tf, 2), "peak": tfl_s, "unit": "TFLOP/s",
                 "frac": round(tf / tfl_s, 4), "traffic": traffic_for("longctx/prefill") if self.default_size else None,
                 "kernel": "tq_prefill_attn", "algorithmic_flops": self.pre_flops,
                 "peak_note": "sustained fp16/bf16 dense (MEASURED_PEAKS.json bf16_tflops_sustained)"},
                {"decode": {"keys_scored_per_s": self.dec_pairs / (op_ms["decode"] * 1e-3), "ms": op_ms["decode"],
                            "gbs": gbs, "frac": gbs / hbm_peak, "algorithmic_bytes": self.dec_bytes},
                 "prefill": {"pairs_per_s": self.pre_pairs / (op_ms["prefill"] * 1e-3), "ms": op_ms["prefill"],
                             "tflops": tf, "frac": tf / tfl_s}})

    def config(self):
        return {"workload": self.name, "batch": 1, "seq_len": self.L, "n_kv_heads": self.H, "n_q_heads": self.Hq,
                "head_dim": self.d, "chunk": self.C, "preset": "K2+QJL/V3", "parallelism": "replicas",
                "l2": "cache (107 MB) read once per decode; prefill re-reads it per query tile"}


class SearchWorkload:
    """Top-10 inner-product search: 1,000,000 x 1024 unit vectors (4-bit +
    QJL), 1,024 queries."""
    name = "search 1,000,000 x d=1024 (4-bit Lloyd-Max + 1-bit QJL) x 1024 queries, top-10"

    def __init__(self, dev, n_db=1_000_000, n_q=1024, **_):
        from kv_cache_vector_07_b200 import synth, tqkv
        self.tq = tqkv
        d = 1024
        self.n_db, self.n_q, self.k, self.d = n_db, n_q, 10, d
        self.desc = tqkv.cache_desc(d, 4, True, 0, page_tokens=64, n_kv_heads=1)
        self.p = tqkv.make_params(d, 4, 1004)
        X = synth.unit_normal(n_db, d, seed=4, device=dev)
        self.cache = tqkv.alloc_cache(self.desc, -(-n_db // 64), device=dev)
        slots = torch.arange(n_db, dtype=torch.int32, device=dev)
        ws = torch.zeros(tqkv.encode_workspace_bytes(self.desc, n_db), dtype=torch.uint8, device=dev)
        s0, e0 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        tqkv.encode(self.p, None, self.desc, X, None, slots, self.cache, workspace=ws)
        s0.record()
        tqkv.encode(self.p, None, self.desc, X, None, slots, self.cache, workspace=ws)
        e0.record()
        torch.cuda.synchronize()
        self.db_encode_ms = s0.elapsed_time(e0)
        del X, ws
        self.Q = synth.unit_normal(n_q, d, seed=5, device=dev)
        self.ws = torch.zeros(tqkv.score_workspace_bytes(self.desc, n_db, n_q, 10), dtype=torch.uint8, device=dev)
        self.sc = torch.empty((n_q, 10), device=dev)
        self.ix = torch.empty((n_q, 10), dtype=torch.int64, device=dev)
        self.units = n_db * n_q
        self.flops = 2 * n_q * n_db * 2 * d
        self.launches = {"score": 5}

    def ops(self):
        tq = self.tq
        return [("score", lambda: tq.score(self.p, self.desc, self.cache, self.n_db, self.Q, self.k,
                                           top_scores=self.sc, top_idx=self.ix, workspace=self.ws))]

    def host_io(self):
        h = self.Q.cpu().pin_memory()
        o1 = torch.empty(self.sc.shape).pin_memory()
        o2 = torch.empty(self.ix.shape, dtype=torch.int64).pin_memory()

        def step():
            self.Q.copy_(h, non_blocking=True)
            self.ops()[0][1]()
            o1.copy_(self.sc, non_blocking=True)
            o2.copy_(self.ix, non_blocking=True)
        return step, h.numel() * 4, o1.numel() * 4 + o2.numel() * 8

    def roofline(self, op_ms, hbm_peak):
        _, tfl, tfl_s, _ = _peaks()
        tf = self.flops / (op_ms["score"] * 1e-3) / 1e12
        # a search of tens of milliseconds timed on its own: the burst figure
        return ({"bound": "tensor", "achieved": round(tf, 2), "peak": tfl, "unit": "TFLOP/s",
                 "frac": round(tf / tfl, 4), "traffic": traffic_for("search/score") if self.default_size else None, "kernel": "tq_score",
                 "algorithmic_flops": self.flops,
                 "peak_note": "burst fp16/bf16 dense (MEASURED_PEAKS.json bf16_tflops; fp16 nominal = bf16 nominal)"},
                {"score": {"scores_per_s": self.units / (op_ms["score"] * 1e-3), "ms": op_ms["score"], "tflops": tf},
                 "db_encode": {"ms": self.db_encode_ms, "vectors_per_s": self.n_db / (self.db_encode_ms * 1e-3)}})

    def config(self):
        return {"workload": self.name, "n_db": self.n_db, "n_queries": self.n_q, "head_dim": self.d, "k": self.k,
                "preset": "4-bit + QJL", "parallelism": "replicas"}


WORKLOADS = {"step": StepWorkload, "decode32k": Decode32kWorkload, "longctx": LongCtxWorkload,
             "search": SearchWorkload}


def traffic_for(key: str):
    """DRAM bytes per launch ("workload/op") from the committed ncu summary,
    scaled to the workload; None unless the kernel's source is unchanged
    since the capture (matching sha256)."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as f:
            e = json.load(f).get("entries", {}).get(key)
        if not e:
            return None
        with open(os.path.join(ROOT, e["source"]), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest() != e["sha256"]:
                return None
        return int(e["bytes_per_launch"])
    except Exception:
        return None


# --------------------------------------------------------------------------
# our implementation
# --------------------------------------------------------------------------
def run_ours(args):
    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local if world > 1 else 0)
    from kv_cache_vector_07_b200 import build as b
    b.build()
    sizes = {k: v for k, v in (("batch", args.batch), ("seq_len", args.seq_len), ("n_db", args.n_db),
                               ("n_q", args.n_q)) if v}
    wl = WORKLOADS[args.workload](dev, **sizes)
    wl.default_size = not sizes           # committed traffic counts refer to the default sizes
    ops = wl.ops()
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        for _, f in ops:
            f()
    torch.cuda.synchronize()
    barrier(world)

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(ops) + 1)] for _ in range(args.steps)]
    clocks = ClockSampler(dev.index)
    clocks.start()
    if clocks.thread is None:
        time.sleep(0.3)                   # nvidia-smi needs a moment to start sampling
    torch.cuda.synchronize()
    barrier(world)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for s in range(args.steps):
        for i, (_, f) in enumerate(ops):
            ev[s][i].record(stream)
            f()
        ev[s][len(ops)].record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    total_ms = start.elapsed_time(end)
    op_ms = {name: statistics.mean(ev[s][i].elapsed_time(ev[s][i + 1]) for s in range(args.steps))
             for i, (name, _) in enumerate(ops)}
    t_max = reduce_max(total_ms / 1e3, world)
    value, _ = aggregate(wl.units * args.steps, [t_max] * world)

    # end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        step_fn, h2d, d2h = wl.host_io()
        for _ in range(2):
            step_fn()
        torch.cuda.synchronize()
        barrier(world)
        e_s, e_e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e = max(1, min(args.steps, 5))
        e_s.record(stream)
        for _ in range(n_e):
            step_fn()
        e_e.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        te = reduce_max(e_s.elapsed_time(e_e) / 1e3, world)
        e2e = {"value": wl.units * n_e * world / te, "unit": "units/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": n_e}

    hbm, bf16, bf16s, src = _peaks()
    roof, parts = wl.roofline(op_ms, hbm)
    if src != "measured":
        roof["peak_source"] = "fallback"
    else:
        roof["peak_source"] = "measured" + ("" if "peak_note" in roof else " (MEASURED_PEAKS.json hbm_gbs)")
    line = {"metric": METRIC if args.workload == "step" else EXTRA_METRICS[args.workload], "value": value,
            "unit": "units/s", "unit_note": UNIT_NOTES[args.workload],
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t_max * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded)", "config": wl.config(),
            "roofline": roof, "parts": parts, "clocks": clk, "e2e": e2e,
            "gpu_launches": sum(wl.launches.values()) * args.steps, "impl": "ours"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.workload, budget_s=args.cpu_budget)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# --------------------------------------------------------------------------
# the oracle on the host cores (CPU baseline and the reference arm)
# --------------------------------------------------------------------------
def _oracle_slice(seed_slice: int, L: int = 32768, d: int = 128, G: int = 4, kbits: int = 4, vbits: int = 4):
    """One (sequence, KV head) slice of the step workload on the oracle:
    encode L keys (+QJL) and L values, then one decode step for G query heads.
    Returns units processed (vectors encoded + pairs scored)."""
    from kv_cache_vector_07_b200 import synth
    from oracle import oracle as O
    K = synth.lognormal_channels(L, 1, d, seed=100 + seed_slice).float().numpy()[:, 0].astype(np.float64)
    V = synth.lognormal_channels(L, 1, d, seed=200 + seed_slice).float().numpy()[:, 0].astype(np.float64)
    Q = synth.normal((G, d), seed=300 + seed_slice).float().numpy().astype(np.float64)
    Pk, Pv = O.make_params(d, kbits, 1001), O.make_params(d, vbits, 2001, with_S=False)
    Ek = O.encode(K, Pk, qjl=True, margins=False)
    Ev = O.encode(V, Pv, qjl=False, margins=False)
    O.attend(Q, Pk, Ek, Pv, Ev)
    return 2 * L + G * L


def _attend_slice(kind: str, n: int):
    """Oracle attention or search on an oracle-encoded slice; returns
    (seconds spent in the timed part, units)."""
    from kv_cache_vector_07_b200 import synth
    from oracle import oracle as O
    d = 1024 if kind == "search" else 128
    if kind == "search":
        n_db, n_q = 20000, 4
        X = synth.unit_normal(n_db, d, seed=40 + n).numpy().astype(np.float64)
        Q = synth.unit_normal(n_q, d, seed=50 + n).numpy().astype(np.float64)
        P = O.make_params(d, 4, 1004)
        E = O.encode(X, P, qjl=True, margins=False)
        t0 = time.perf_counter()
        O.search(Q, P, E, 10)
        return time.perf_counter() - t0, n_db * n_q
    L, G, kb, vb = (32768, 4, 2, 4) if kind == "decode32k" else (65536, 8, 2, 3)
    K = synth.outlier_normal((L, d), seed=60 + n, dtype=torch.float32).numpy().astype(np.float64)
    V = synth.outlier_normal((L, d), seed=70 + n, dtype=torch.float32).numpy().astype(np.float64)
    Q = synth.normal((G, d), seed=80 + n, dtype=torch.float32).numpy().astype(np.float64)
    Pk, Pv = O.make_params(d, kb, 1002), O.make_params(d, vb, 2002, with_S=False)
    Ek, Ev = O.encode(K, Pk, qjl=True, margins=False), O.encode(V, Pv, qjl=False, margins=False)
    t0 = time.perf_counter()
    O.attend(Q, Pk, Ek, Pv, Ev)
    return time.perf_counter() - t0, G * L


def cpu_baseline(workload: str, budget_s: float = 15.0):
    from oracle import oracle as O
    O.build()
    cores = len(os.sched_getaffinity(0))
    os.environ.setdefault("OMP_NUM_THREADS", str(cores))
    units, spent, n = 0, 0.0, 0
    wall0 = time.perf_counter()
    if workload == "step":
        O.codebook(128, 4)
        while spent < budget_s or n == 0:
            t0 = time.perf_counter()
            units += _oracle_slice(n)
            spent += time.perf_counter() - t0
            n += 1
        sample = (f"{n} (sequence, KV head) slices of the step workload: each encodes 32,768 keys (4-bit + QJL) "
                  f"and 32,768 values (4-bit) and scores them for 4 query heads (float64 oracle, OpenMP)")
    else:
        while (spent < budget_s and time.perf_counter() - wall0 < 4 * budget_s) or n == 0:
            dt, u = _attend_slice(workload, n)
            spent += dt
            units += u
            n += 1
        what = {"decode32k": "one KV head (4 query heads) over 32,768 oracle-encoded tokens",
                "longctx": "one KV head (8 query heads) over 65,536 oracle-encoded tokens",
                "search": "4 queries over 20,000 oracle-encoded d=1024 vectors"}[workload]
        sample = f"{n} slices, each {what}; only the scoring is timed (float64 oracle, OpenMP)"
    return {"value": units / spent, "unit": "units/s", "cores": cores, "kind": "oracle", "sample": sample,
            "seconds": spent}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from oracle import oracle as O
    O.build()
    O.codebook(128, 4)
    cores = len(os.sched_getaffinity(0))
    for i in range(args.warmup):
        _oracle_slice(1000 + i, L=4096)
    t0 = time.perf_counter()
    units = 0
    for s in range(args.steps):
        units += _oracle_slice(s, L=4096)
    dt = time.perf_counter() - t0
    value = units / dt
    wl_name = StepWorkload.name
    line = {"metric": METRIC if args.workload == "step" else EXTRA_METRICS[args.workload], "value": value,
            "unit": "units/s", "unit_note": UNIT_NOTES[args.workload],
            "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3 / max(1, args.steps), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
            "config": {"workload": wl_name, "parallelism": "host cores"}, "impl": "reference",
            "cpu_baseline": {"kind": "oracle", "cores": cores, "value": value, "unit": "units/s",
                             "sample": "per step one (sequence, KV head) slice of 4,096 tokens: encode 4,096 keys "
                                       "(4-bit + QJL) and 4,096 values, score them for 4 query heads"},
            "e2e": {"value": value, "unit": "units/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="step")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch (smaller profiling cases)")
    ap.add_argument("--seq-len", type=int, default=0, help="override the workload's sequence length")
    ap.add_argument("--n-db", type=int, default=0, help="override the search database size")
    ap.add_argument("--n-q", type=int, default=0, help="override the number of search queries")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

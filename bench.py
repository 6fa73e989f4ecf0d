#!/usr/bin/env python
"""Throughput of the compressed-KV hot path on B200, as one JSON line.

Default workload (one step), every op on inputs already resident in HBM:
  * the write path of an 8B-dense-shaped layer (B=8 x 8 KV heads x 32,768
    tokens x d=128, bf16 K and V with lognormal channel scales and outlier
    channels), compressed twice: preset k8v4 (FP8 keys, 4-bit values) and
    K = 4-bit Lloyd-Max + 1-bit QJL with 4-bit values;
  * one GQA decode step over a pre-encoded k3v4 cache (B=32, 32 query heads
    over 8 KV heads, 32,768 tokens: K = 2-bit Lloyd-Max + 1-bit QJL, V = 4-bit).
Metric: KV vectors encoded plus (query-head, key) pairs scored, per second.
The same run also times, as separate parts with their own roofline fractions,
the long-context workload (B=1, 32 query heads over 4 KV heads, 262,144
tokens, 3-bit keys incl. QJL and 3-bit values: one decode step and one
2,048-query prefill chunk) and the compressed search (1,000,000 x 1024 unit
vectors, 4-bit + QJL, 1,024 queries, top-10, with recall@10 against exact
fp32 search).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload step|encode|decode32k|longctx|search] [--no-parts]

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
WORKLOAD_METRICS = {"step": METRIC, "encode": "KV vectors encoded/s", "decode32k": "decode-attn keys scored/s",
                    "decode_k8v4": "decode-attn keys scored/s", "decode_step": "decode-attn keys scored/s",
                    "dense": "KV vectors encoded/s + decode-attn keys scored/s",
                    "frac35": "KV vectors encoded/s + decode-attn keys scored/s",
                    "polar": "KV vectors encoded/s + decode-attn keys scored/s",
                    "longctx": "decode + prefill (query-head, key) pairs/s",
                    "search": "(query, database vector) pairs scored/s (top-10 search)"}
UNIT_NOTES = {"step": "units = KV vectors encoded (two presets) + (query-head, key) pairs scored",
              "encode": "units = KV vectors encoded (two presets)",
              "decode32k": "units = (query-head, key) pairs scored",
              "decode_k8v4": "units = (query-head, key) pairs scored",
              "decode_step": "units = (query-head, key) pairs scored (the new tokens' write included in the time)",
              "dense": "units = KV vectors encoded + (query-head, key) pairs scored",
              "frac35": "units = KV vectors encoded + (query-head, key) pairs scored",
              "polar": "units = KV vectors encoded + (query-head, key) pairs scored",
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
# ops and workloads
# --------------------------------------------------------------------------
class Op:
    """One timed call of the public API with its algorithmic work.

    bound "hbm": work = compressed algorithmic bytes that must cross HBM once;
    bound "tensor": work = the method's own flops (not the hi/lo passes).
    peak: which measured peak the fraction is taken against."""

    def __init__(self, name, fn, units, unit_name, bound, work, kernel, launches, peak="hbm", traffic_key=None,
                 flush=False, extra=None):
        self.name, self.fn, self.units, self.unit_name = name, fn, units, unit_name
        self.bound, self.work, self.kernel, self.launches = bound, work, kernel, launches
        self.peak, self.traffic_key, self.flush = peak, traffic_key, flush
        self.extra = extra or {}


class WritePath:
    """Config: the write path of an 8B-dense-shaped layer, B x 8 KV heads x
    32,768 tokens x d=128 bf16 (lognormal channel scales, 4 outlier channels
    per head x15), compressed with preset k8v4 and with K 4-bit + QJL / V 4-bit."""
    PRESETS = (("k8v4", 8, False, 4, 1001, 2001), ("k4qjl_v4", 4, True, 4, 1011, 2011))

    def __init__(self, dev, batch=8, seq_len=32768, **_):
        from kv_cache_vector_07_b200 import synth, tqkv
        self.tq = tqkv
        B, L, H, d, P = batch, seq_len, 8, 128, 64
        self.B, self.L, self.H, self.d, self.P = B, L, H, d, P
        n = B * L
        self.n = n
        self.K = synth.lognormal_channels(n, H, d, seed=1, device=dev)
        self.V = synth.lognormal_channels(n, H, d, seed=10001, device=dev)
        _, self.slots, self.nblk = synth.contiguous_block_table(B, L, P, device=dev, shuffle_seed=11)
        self.codecs = {}
        for name, kb, kq, vb, ks, vs in self.PRESETS:
            desc = tqkv.cache_desc(d, kb, kq, vb, page_tokens=P, n_kv_heads=H)
            kp, vp = tqkv.make_params(d, kb, ks), tqkv.make_params(d, vb, vs)
            cache = tqkv.alloc_cache(desc, self.nblk, device=dev)
            ws = torch.zeros(tqkv.encode_workspace_bytes(desc, n), dtype=torch.uint8, device=dev)
            per_tok = tqkv.cache_bytes(desc) // P
            self.codecs[name] = (desc, kp, vp, cache, ws, per_tok)

    def ops(self):
        tq, out = self.tq, []
        for name, (desc, kp, vp, cache, ws, per_tok) in self.codecs.items():
            def f(desc=desc, kp=kp, vp=vp, cache=cache, ws=ws):
                tq.encode(kp, vp, desc, self.K, self.V, self.slots, cache, workspace=ws)
            work = 2 * self.n * self.H * self.d * 2 + self.n * self.H * per_tok
            out.append(Op(f"encode_{name}", f, 2 * self.n * self.H, "vectors encoded", "hbm", work,
                          "tq_encode (encode128_kernel: TMA + tcgen05 rotation + quantize"
                          + (" + tcgen05 QJL)" if name != "k8v4" else ", E4M3 keys)"), 1,
                          traffic_key=f"step/encode_{name}" if (self.B, self.L) == (8, 32768) else None,
                          extra={"preset": name, "bytes_per_token_and_head": per_tok}))
        return out

    def host_inputs(self):
        return {"K": self.K, "V": self.V, "slots": self.slots}

    def host_outputs(self):
        return {}

    @staticmethod
    def config(batch=8, seq_len=32768, **_):
        return {"write_path": {"what": f"B={batch} x Hkv=8 x {seq_len} tokens x d=128 bf16, presets k8v4 and "
                                       "K 4-bit Lloyd-Max + 1-bit QJL / V 4-bit",
                               "batch": batch, "seq_len": seq_len, "n_kv_heads": 8, "head_dim": 128,
                               "page_tokens": 64}}


class Decode32k:
    """Config: one GQA decode step, B=32, Hq=32 over Hkv=8, 32,768 tokens,
    cache pre-encoded with k3v4 (K 2-bit + QJL, V 4-bit) from N(0,1) data
    with channels 5 and 77 scaled x20."""
    preset, kbits, kqjl = "k3v4", 2, True

    def __init__(self, dev, batch=32, seq_len=32768, **_):
        from kv_cache_vector_07_b200 import synth, tqkv
        self.tq = tqkv
        B, L, H, Hq, d, P = batch, seq_len, 8, 32, 128, 64
        self.B, self.L, self.H, self.Hq, self.d, self.P = B, L, H, Hq, d, P
        n = B * L
        self.desc = tqkv.cache_desc(d, self.kbits, self.kqjl, 4, page_tokens=P, n_kv_heads=H)
        self.kp = tqkv.make_params(d, self.kbits, 1002)
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
        self.ws = torch.zeros(tqkv.decode_workspace_bytes(self.desc, B, Hq, L), dtype=torch.uint8, device=dev)
        self.per_tok = tqkv.cache_bytes(self.desc) // P

    def ops(self):
        tq = self.tq

        def f():
            tq.decode_attn(self.kp, self.vp, self.desc, self.Q, self.bt, self.seq, self.L, self.cache, out=self.out,
                           workspace=self.ws)
        work = self.B * self.H * self.L * self.per_tok + 2 * self.Q.numel() * 2
        return [Op(f"decode_{self.preset}", f, self.B * self.Hq * self.L, "(query-head, key) pairs scored", "hbm",
                   work, "tq_decode_attn (" + ("prep_proj128" if self.kqjl else "prep") +
                   " + dec128 tensor-core decode + combine)", 3,
                   traffic_key=f"decode32k/decode_{self.preset}" if (self.B, self.L) == (32, 32768) else None,
                   extra={"bytes_per_token_and_head": self.per_tok})]

    def host_inputs(self):
        return {"Q": self.Q, "bt": self.bt, "seq": self.seq}

    def host_outputs(self):
        return {"out": self.out}

    @staticmethod
    def config(batch=32, seq_len=32768, **_):
        return {"decode": {"what": f"B={batch} x Hq=32/Hkv=8 x {seq_len} tokens x d=128, k3v4 "
                                   "(K 2-bit Lloyd-Max + 1-bit QJL, V 4-bit), one step",
                           "batch": batch, "seq_len": seq_len, "n_q_heads": 32, "n_kv_heads": 8, "head_dim": 128,
                           "page_tokens": 64}}


class Decode32kK8V4(Decode32k):
    """The same decode step over a cache written with preset k8v4 (FP8 E4M3
    keys, 4-bit values): the read side of the k8v4 write path."""
    preset, kbits, kqjl = "k8v4", 8, False

    @staticmethod
    def config(batch=32, seq_len=32768, **_):
        return {"decode_k8v4": {"what": f"B={batch} x Hq=32/Hkv=8 x {seq_len} tokens x d=128, k8v4 "
                                        "(FP8 E4M3 keys, V 4-bit), one step",
                                "batch": batch, "seq_len": seq_len, "n_q_heads": 32, "n_kv_heads": 8}}


class Decode32kStep(Decode32k):
    """The k3v4 decode step with the new token's write fused in (tq_decode_step):
    each sequence's token at position 32,767 is compressed into the cache and
    all 32 query heads attend over the 32,768 tokens."""

    def __init__(self, dev, batch=32, seq_len=32768, **kw):
        super().__init__(dev, batch=batch, seq_len=seq_len, **kw)
        from kv_cache_vector_07_b200 import synth
        self.Kn = synth.outlier_normal((self.B, self.H, self.d), seed=23, device=dev)
        self.Vn = synth.outlier_normal((self.B, self.H, self.d), seed=24, device=dev)
        self.new_slots = (self.bt[:, -1].to(torch.int64) * self.P + (self.L - 1) % self.P).to(torch.int32)

    def ops(self):
        tq = self.tq

        def f():
            tq.decode_step(self.kp, self.vp, self.desc, self.Kn, self.Vn, self.new_slots, self.Q, self.bt, self.seq,
                           self.L, self.cache, out=self.out, workspace=self.ws)
        work = self.B * self.H * self.L * self.per_tok + 2 * self.Q.numel() * 2 + 2 * 2 * self.Kn.numel()
        return [Op("decode_step_k3v4", f, self.B * self.Hq * self.L, "(query-head, key) pairs scored", "hbm", work,
                   "tq_decode_step (new-token encode + query prep in one launch, dec128 tensor-core decode, combine)",
                   3, extra={"new_tokens_written": self.B * self.H * 2})]

    @staticmethod
    def config(batch=32, seq_len=32768, **_):
        return {"decode_step": {"what": f"B={batch} x Hq=32/Hkv=8 x {seq_len} tokens x d=128, k3v4: write the new "
                                        "token's K/V, then attend (fused decode step)",
                                "batch": batch, "seq_len": seq_len}}


class PresetPart:
    """A write path and a GQA decode over it under an alternative codec: B=8
    sequences x 8 KV heads x 8,192 tokens x d=128 bf16 (N(0,1), channels 5
    and 77 x20), 32 query heads."""
    kbits, kqjl, vbits, rotation, tag, what = 2, True, 4, 0, "", ""
    enc_kernel, enc_launches = "tq_encode (encode_kernel: warp per vector, + qjl_gemm_kernel)", 2
    dec_kernel = "tq_decode_attn (prep + dec128 tensor-core decode + combine)"

    def __init__(self, dev, batch=8, seq_len=8192, **_):
        from kv_cache_vector_07_b200 import synth, tqkv
        self.tq = tqkv
        B, L, H, Hq, d, P = batch, seq_len, 8, 32, 128, 64
        self.B, self.L, self.H, self.Hq, self.d, self.P = B, L, H, Hq, d, P
        n = B * L
        self.n = n
        self.desc = tqkv.cache_desc(d, self.kbits, self.kqjl, self.vbits, page_tokens=P, n_kv_heads=H)
        self.kp = tqkv.make_params(d, self.kbits, 1005, self.rotation)
        self.vp = tqkv.make_params(d, self.vbits, 2005, self.rotation)
        self.K = synth.outlier_normal((n, H, d), seed=51, device=dev)
        self.V = synth.outlier_normal((n, H, d), seed=52, device=dev)
        self.bt, self.slots, nblk = synth.contiguous_block_table(B, L, P, device=dev, shuffle_seed=53)
        self.cache = tqkv.alloc_cache(self.desc, nblk, device=dev)
        self.ws_e = torch.zeros(tqkv.encode_workspace_bytes(self.desc, n), dtype=torch.uint8, device=dev)
        tqkv.encode(self.kp, self.vp, self.desc, self.K, self.V, self.slots, self.cache, workspace=self.ws_e)
        self.Q = synth.normal((B, Hq, d), seed=54, device=dev)
        self.seq = torch.full((B,), L, dtype=torch.int32, device=dev)
        self.out = torch.empty_like(self.Q)
        self.ws_d = torch.zeros(tqkv.decode_workspace_bytes(self.desc, B, Hq, L), dtype=torch.uint8, device=dev)
        self.per_tok = tqkv.cache_bytes(self.desc) // P
        torch.cuda.synchronize()

    def ops(self):
        tq = self.tq

        def fe():
            tq.encode(self.kp, self.vp, self.desc, self.K, self.V, self.slots, self.cache, workspace=self.ws_e)

        def fd():
            tq.decode_attn(self.kp, self.vp, self.desc, self.Q, self.bt, self.seq, self.L, self.cache, out=self.out,
                           workspace=self.ws_d)
        ex = {"bytes_per_token_and_head": self.per_tok, "codec": self.what}
        return [Op(f"{self.tag}_encode", fe, 2 * self.n * self.H, "vectors encoded", "hbm",
                   2 * self.n * self.H * self.d * 2 + self.n * self.H * self.per_tok,
                   self.enc_kernel, self.enc_launches, flush=True, extra=ex),
                Op(f"{self.tag}_decode", fd, self.B * self.Hq * self.L, "(query-head, key) pairs scored", "hbm",
                   self.B * self.H * self.L * self.per_tok, self.dec_kernel, 3, flush=True, extra=ex)]

    def host_inputs(self):
        return {"K": self.K, "V": self.V, "Q": self.Q}

    def host_outputs(self):
        return {"out": self.out}

    @classmethod
    def config(cls, batch=8, seq_len=8192, **_):
        return {cls.tag: {"what": f"B={batch} x Hkv=8 x {seq_len} tokens x d=128 bf16, 32 query heads: " + cls.what,
                          "batch": batch, "seq_len": seq_len}}


class DenseRotation(PresetPart):
    kbits, kqjl, vbits, rotation, tag = 2, True, 4, 1, "dense_k3v4"
    what = "k3v4 under the dense random rotation (encode: dense 128 x 128 product, four vectors per warp)"
    enc_kernel = "tq_encode (encode_dense_kernel: dense rotation of four vectors per warp, + qjl_gemm_kernel)"


class Fractional35(PresetPart):
    kbits, kqjl, vbits, rotation, tag = 16 | 2, True, 16 | 3, 0, "frac35"
    what = "3.5-bit keys incl. QJL (2.5-bit Lloyd-Max + QJL) and 3.5-bit values (fractional rates)"
    enc_kernel, enc_launches = "tq_encode (encode128_kernel: fused, one codebook per coordinate half)", 1
    dec_kernel = "tq_decode_attn (prep + dec128 fractional-rate decode + combine)"


class PolarCodes(PresetPart):
    kbits, kqjl, vbits, rotation, tag = 32, True, 32, 0, "polar"
    what = "PolarQuant angle codes (4-bit level-1 angles, 2-bit higher levels) for keys with QJL and for values"
    enc_kernel = "tq_encode (encode_kernel: warp per vector, polar transform by half-plane tests, + qjl_gemm_kernel)"
    dec_kernel = "tq_decode_attn (prep + dec128 polar decode, angle tree rebuilt per token + combine)"


class LongCtx:
    """Config: B=1, Hq=32 over Hkv=4, 262,144 tokens, K 2-bit + QJL, V 3-bit;
    one decode step plus one 2,048-query prefill chunk (causal inside)."""

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
        self.per_tok = tqkv.cache_bytes(self.desc) // P

    def ops(self):
        tq = self.tq
        dec_pairs = self.Hq * self.L
        pre_pairs = self.Hq * sum(self.L - self.C + j + 1 for j in range(self.C))
        full = (self.L, self.C) == (262144, 2048)

        def fd():
            tq.decode_attn(self.kp, self.vp, self.desc, self.Qd, self.bt, self.seq, self.L, self.cache,
                           out=self.out_d, workspace=self.ws_d)

        def fp():
            tq.prefill_attn(self.kp, self.vp, self.desc, self.Qp, self.bt.view(-1), self.L, self.cache,
                            out=self.out_p, workspace=self.ws_p)
        return [Op("longctx_decode", fd, dec_pairs, "(query-head, key) pairs scored", "hbm",
                   self.H * self.L * self.per_tok, "tq_decode_attn (prep_proj128 + dec128 + combine)", 3,
                   traffic_key="longctx/decode" if full else None, flush=True,
                   extra={"bytes_per_token_and_head": self.per_tok}),
                Op("longctx_prefill", fp, pre_pairs, "(query-head, key) pairs scored", "tensor",
                   pre_pairs * 2 * (2 * self.d + self.d), "tq_prefill_attn (prep_proj128 + pf128 tcgen05 + combine)",
                   3, peak="sustained", traffic_key="longctx/prefill" if full else None, flush=True,
                   extra={"flop_note": "768 flop per (query head, visible key): 2 x 256 for [q_r | w] against "
                                       "[nhat c | rho sqrt(pi/2)/m s], 2 x 128 for P V"})]

    def host_inputs(self):
        return {"Qd": self.Qd, "Qp": self.Qp}

    def host_outputs(self):
        return {"out_d": self.out_d, "out_p": self.out_p}

    @staticmethod
    def config(seq_len=262144, **_):
        return {"longctx": {"what": f"B=1 x Hq=32/Hkv=4 x {seq_len} tokens x d=128 (K 2-bit + QJL, V 3-bit): "
                                    "one decode step + one 2048-query prefill chunk, causal inside the chunk",
                            "batch": 1, "seq_len": seq_len, "chunk": 2048, "n_q_heads": 32, "n_kv_heads": 4}}


class Search:
    """Config: top-10 inner-product search over 1,000,000 x 1024 unit vectors
    (4-bit Lloyd-Max + 1-bit QJL), 1,024 queries; recall@10 against exact fp32."""

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
        tqkv.encode(self.p, None, self.desc, X, None, slots, self.cache, workspace=ws)
        times = []
        for _ in range(3):                         # the database encode, timed on its own
            s0, e0 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0.record()
            tqkv.encode(self.p, None, self.desc, X, None, slots, self.cache, workspace=ws)
            e0.record()
            torch.cuda.synchronize()
            times.append(s0.elapsed_time(e0))
        self.db_encode_ms = statistics.median(times)
        self.Q = synth.unit_normal(n_q, d, seed=5, device=dev)
        # exact fp32 top-10 (the recall reference): fp32 products, no TF32
        prev = torch.backends.cuda.matmul.allow_tf32
        torch.backends.cuda.matmul.allow_tf32 = False
        best_v = torch.full((n_q, self.k), -float("inf"), device=dev)
        best_i = torch.zeros((n_q, self.k), dtype=torch.int64, device=dev)
        for r0 in range(0, n_db, 1 << 17):
            r1 = min(n_db, r0 + (1 << 17))
            s = self.Q @ X[r0:r1].T
            v, i = torch.topk(s, min(self.k, r1 - r0), dim=1)
            cv, ci = torch.cat([best_v, v], 1), torch.cat([best_i, i + r0], 1)
            best_v, sel = torch.topk(cv, self.k, dim=1)
            best_i = torch.gather(ci, 1, sel)
        torch.backends.cuda.matmul.allow_tf32 = prev
        self.exact_idx = best_i
        self.X_cpu_slice = X[:131072].cpu()          # for the CPU exact-search baseline
        del X, ws
        self.ws = torch.zeros(tqkv.score_workspace_bytes(self.desc, n_db, n_q, 10), dtype=torch.uint8, device=dev)
        self.sc = torch.empty((n_q, 10), device=dev)
        self.ix = torch.empty((n_q, 10), dtype=torch.int64, device=dev)

    def recall_at_10(self):
        a, b = self.ix.cpu().numpy(), self.exact_idx.cpu().numpy()
        return float(np.mean([len(set(a[q]) & set(b[q])) / 10.0 for q in range(a.shape[0])]))

    def cpu_exact_search(self, n_queries=64):
        """Exact fp32 search with torch on the host cores over a 131,072-row
        slice of the database: (query, vector) pairs per second."""
        X = self.X_cpu_slice
        Q = self.Q[:n_queries].cpu()
        torch.topk(Q[:4] @ X[:4096].T, 10, dim=1)
        t0 = time.perf_counter()
        s = Q @ X.T
        torch.topk(s, 10, dim=1)
        dt = time.perf_counter() - t0
        return {"value": n_queries * X.shape[0] / dt, "unit": "(query, vector) pairs/s", "cores": torch.get_num_threads(),
                "kind": "exact fp32 search (torch CPU matmul + topk)",
                "sample": f"{n_queries} queries x {X.shape[0]} database rows", "seconds": dt}

    def ops(self):
        tq = self.tq

        def f():
            tq.score(self.p, self.desc, self.cache, self.n_db, self.Q, self.k, top_scores=self.sc, top_idx=self.ix,
                     workspace=self.ws)
        return [Op("search", f, self.n_db * self.n_q, "(query, database vector) pairs scored", "tensor",
                   2 * self.n_q * self.n_db * 2 * self.d, "tq_score (prep + qproj + qfeat + score_tc tcgen05 + merge)",
                   5, peak="burst", traffic_key="search/score" if (self.n_db, self.n_q) == (1_000_000, 1024) else None,
                   extra={"db_encode_ms": self.db_encode_ms, "db_encode_vectors_per_s": self.n_db / (self.db_encode_ms * 1e-3),
                          "db_bytes": self.n_db * (tq.cache_bytes(self.desc) // 64)})]

    def host_inputs(self):
        return {"Q": self.Q}

    def host_outputs(self):
        return {"sc": self.sc, "ix": self.ix}

    @staticmethod
    def config(n_db=1_000_000, n_q=1024, **_):
        return {"search": {"what": f"{n_db} x d=1024 unit vectors (4-bit Lloyd-Max + 1-bit QJL) x {n_q} "
                                   "queries, top-10",
                           "n_db": n_db, "n_queries": n_q, "head_dim": 1024, "k": 10}}


# workload -> (classes in the timed step, classes timed as parts)
WORKLOADS = {"step": ((WritePath, Decode32k), (Decode32kK8V4, Decode32kStep, LongCtx, Search, DenseRotation,
                                                Fractional35, PolarCodes)),
             "encode": ((WritePath,), ()),
             "decode32k": ((Decode32k,), ()),
             "decode_k8v4": ((Decode32kK8V4,), ()),
             "decode_step": ((Decode32kStep,), ()),
             "dense": ((DenseRotation,), ()),
             "frac35": ((Fractional35,), ()),
             "polar": ((PolarCodes,), ()),
             "longctx": ((LongCtx,), ()),
             "search": ((Search,), ())}
WORKLOAD_NAMES = {"step": "write path (k8v4 and K4+QJL/V4, 8 x 8 x 32768 x 128 bf16) + k3v4 GQA decode "
                          "(32 x 32/8 heads x 32768)",
                  "encode": "write path 8 x 8 x 32768 x 128 bf16, presets k8v4 and K4+QJL/V4",
                  "decode32k": "k3v4 GQA decode 32 x 32/8 heads x 32768 x 128",
                  "decode_k8v4": "k8v4 GQA decode 32 x 32/8 heads x 32768 x 128 (FP8 keys)",
                  "decode_step": "fused k3v4 decode step (write the new token, attend) 32 x 32/8 heads x 32768",
                  "dense": "k3v4 write path + decode under the dense rotation, 8 x 8 x 8192",
                  "frac35": "3.5-bit fractional-rate write path + decode, 8 x 8 x 8192",
                  "polar": "PolarQuant-coded write path + decode, 8 x 8 x 8192",
                  "longctx": "long-context 1 x 32/4 heads x 262144: decode + 2048-query prefill",
                  "search": "search 1,000,000 x 1024, 1024 queries, top-10"}


def workload_config(workload: str, sizes: dict) -> dict:
    step_cls, part_cls = WORKLOADS[workload]
    cfg = {"workload": WORKLOAD_NAMES[workload]}
    for c in step_cls:
        cfg.update(c.config(**sizes))
    if part_cls:
        cfg["parts_outside_the_step"] = {k: v for c in part_cls for k, v in c.config().items()}
    cfg["parallelism"] = "replicas"
    cfg["l2"] = ("every op of the step reads more than L2 (126 MB); parts whose inputs fit in L2 "
                 "(the 107 MB long-context cache) are timed after a 512 MB L2 flush")
    return cfg


def traffic_for(key: str):
    """DRAM bytes per launch ("workload/op") from the committed ncu summary,
    scaled to the workload; None unless the kernel's source is unchanged
    since the capture (matching sha256)."""
    import hashlib
    if key is None:
        return None
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


def roofline_of(op: Op, ms: float) -> dict:
    hbm, bf16, bf16s, src = _peaks()
    if op.bound == "hbm":
        ach, peak, unit = op.work / (ms * 1e-3) / 1e9, hbm, "GB/s"
        note = "HBM copy bandwidth"
    else:
        ach, unit = op.work / (ms * 1e-3) / 1e12, "TFLOP/s"
        peak = bf16s if op.peak == "sustained" else bf16
        note = ("sustained" if op.peak == "sustained" else "burst") + " bf16/fp16 dense (fp16 nominal = bf16 nominal)"
    r = {"bound": op.bound, "achieved": round(ach, 2), "peak": peak, "unit": unit, "frac": round(ach / peak, 4),
         "traffic": traffic_for(op.traffic_key), "kernel": op.kernel,
         ("algorithmic_bytes" if op.bound == "hbm" else "algorithmic_flops"): op.work,
         "peak_source": f"{src} ({note}{', MEASURED_PEAKS.json' if src == 'measured' else ''})"}
    return r


def _flush_l2(buf):
    if buf is not None:
        buf.add_(1)


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
    step_cls, part_cls = WORKLOADS[args.workload]
    if args.no_parts or world > 1:
        part_cls = ()
    step_objs = [c(dev, **sizes) for c in step_cls]
    ops = [op for o in step_objs for op in o.ops()]
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        for op in ops:
            op.fn()
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
        for i, op in enumerate(ops):
            ev[s][i].record(stream)
            op.fn()
        ev[s][len(ops)].record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    total_ms = start.elapsed_time(end)
    op_ms = {op.name: statistics.mean(ev[s][i].elapsed_time(ev[s][i + 1]) for s in range(args.steps))
             for i, op in enumerate(ops)}
    t_max = reduce_max(total_ms / 1e3, world)
    units = sum(op.units for op in ops)
    value, _ = aggregate(units * args.steps, [t_max] * world)

    # end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        h_in = {}
        for o in step_objs:
            for name, t in o.host_inputs().items():
                h_in[(id(o), name)] = (t, t.cpu().pin_memory())
        h_out = {}
        for o in step_objs:
            for name, t in o.host_outputs().items():
                h_out[(id(o), name)] = (t, torch.empty(t.shape, dtype=t.dtype).pin_memory())
        seen, h2d = set(), 0
        for dtn, host in h_in.values():
            if dtn.data_ptr() not in seen:
                seen.add(dtn.data_ptr())
                h2d += host.numel() * host.element_size()
        d2h = sum(h.numel() * h.element_size() for _, h in h_out.values())

        def e2e_step():
            done = set()
            for dtn, host in h_in.values():
                if dtn.data_ptr() not in done:
                    done.add(dtn.data_ptr())
                    dtn.copy_(host, non_blocking=True)
            for op in ops:
                op.fn()
            for dtn, host in h_out.values():
                host.copy_(dtn, non_blocking=True)
        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        barrier(world)
        e_s, e_e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e = max(1, min(args.steps, 5))
        e_s.record(stream)
        for _ in range(n_e):
            e2e_step()
        e_e.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        te = reduce_max(e_s.elapsed_time(e_e) / 1e3, world)
        e2e = {"value": units * n_e * world / te, "unit": "units/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": n_e}

    parts = {}
    for op in ops:
        ms = op_ms[op.name]
        parts[op.name] = {"in_step": True, "ms": ms, op.unit_name.replace(" ", "_") + "_per_s": op.units / (ms * 1e-3),
                          "roofline": roofline_of(op, ms), **op.extra}
    dominant = max(ops, key=lambda o: op_ms[o.name])
    roof = dict(parts[dominant.name]["roofline"])
    roof["op"] = dominant.name

    # parts outside the step: each op timed on its own (CUDA events on this stream)
    part_clk = None
    if part_cls:
        flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
        pclocks = ClockSampler(dev.index)
        pobjs = []
        for c in part_cls:
            o = c(dev)
            pobjs.append(o)
            pops = o.ops()
            for op in pops:
                for _ in range(2):
                    op.fn()
            torch.cuda.synchronize()
            pclocks.start() if not pobjs[:-1] else None
            for op in pops:
                n_rep = max(3, min(args.steps, 10))
                times = []
                for _ in range(n_rep):
                    if op.flush:
                        _flush_l2(flush)
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                    op.fn()
                    e1.record(stream)
                    times.append((e0, e1))
                torch.cuda.synchronize()
                ms = statistics.mean(a.elapsed_time(b2) for a, b2 in times)
                parts[op.name] = {"in_step": False, "ms": ms, "reps": n_rep,
                                  op.unit_name.replace(" ", "_") + "_per_s": op.units / (ms * 1e-3),
                                  "roofline": roofline_of(op, ms), "l2_flushed": op.flush, **op.extra}
            if isinstance(o, Search):
                parts["search"]["recall_at_10"] = o.recall_at_10()
                if rank == 0 and world == 1 and not args.no_cpu_baseline:
                    parts["search"]["cpu_exact_search"] = o.cpu_exact_search()
            del o
        part_clk = pclocks.stop()
        del flush

    line = {"metric": WORKLOAD_METRICS[args.workload], "value": value, "unit": "units/s",
            "unit_note": UNIT_NOTES[args.workload], "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t_max * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded)",
            "config": workload_config(args.workload, sizes),
            "roofline": roof, "parts": parts, "clocks": clk, "e2e": e2e,
            "gpu_launches": sum(op.launches for op in ops) * args.steps, "impl": "ours"}
    if part_clk is not None:
        line["parts_clocks"] = part_clk
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.workload, budget_s=args.cpu_budget)
        if part_cls:
            for name in ("decode_k8v4", "longctx", "search", "dense", "frac35", "polar"):
                cb = cpu_baseline(name, budget_s=min(4.0, args.cpu_budget))
                for k in [k for k in parts if k.startswith(name)]:
                    parts[k]["cpu_baseline"] = cb
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# --------------------------------------------------------------------------
# the oracle on the host cores (CPU baseline and the reference arm)
# --------------------------------------------------------------------------
def _f64(t):
    return t.float().numpy().astype(np.float64)


def _oracle_encode_slice(n: int, L: int):
    """One (sequence, KV head) slice of the write path on the oracle: L keys
    and L values, compressed with k8v4 and with K 4-bit + QJL / V 4-bit.
    Returns (seconds, vectors encoded)."""
    from kv_cache_vector_07_b200 import synth
    from oracle import oracle as O
    K = _f64(synth.lognormal_channels(L, 1, 128, seed=100 + n)[:, 0])
    V = _f64(synth.lognormal_channels(L, 1, 128, seed=200 + n)[:, 0])
    Pk8, Pk4 = O.make_params(128, 8, 1001, with_S=False), O.make_params(128, 4, 1011)
    Pv = O.make_params(128, 4, 2001, with_S=False)
    t0 = time.perf_counter()
    O.encode(K, Pk8, qjl=False, margins=False)
    O.encode(V, Pv, qjl=False, margins=False)
    O.encode(K, Pk4, qjl=True, margins=False)
    O.encode(V, Pv, qjl=False, margins=False)
    return time.perf_counter() - t0, 4 * L


def _oracle_attend_slice(kind: str, n: int, L: int | None = None):
    """Oracle attention or search on an oracle-encoded slice (encode untimed).
    Returns (seconds in the timed part, units)."""
    from kv_cache_vector_07_b200 import synth
    from oracle import oracle as O
    d = 1024 if kind == "search" else 128
    if kind == "search":
        n_db, n_q = L or 20000, 4
        X = synth.unit_normal(n_db, d, seed=40 + n).numpy().astype(np.float64)
        Q = synth.unit_normal(n_q, d, seed=50 + n).numpy().astype(np.float64)
        P = O.make_params(d, 4, 1004)
        E = O.encode(X, P, qjl=True, margins=False)
        t0 = time.perf_counter()
        O.search(Q, P, E, 10)
        return time.perf_counter() - t0, n_db * n_q
    if kind == "decode32k":
        L, G, kb, vb = L or 32768, 4, 2, 4
    elif kind == "decode_k8v4":
        L, G, kb, vb = L or 32768, 4, 8, 4
    else:
        L, G, kb, vb = L or 65536, 8, 2, 3
    K = synth.outlier_normal((L, d), seed=60 + n, dtype=torch.float32).numpy().astype(np.float64)
    V = synth.outlier_normal((L, d), seed=70 + n, dtype=torch.float32).numpy().astype(np.float64)
    Q = synth.normal((G, d), seed=80 + n, dtype=torch.float32).numpy().astype(np.float64)
    Pk, Pv = O.make_params(d, kb, 1002, with_S=kb != 8), O.make_params(d, vb, 2002, with_S=False)
    Ek, Ev = O.encode(K, Pk, qjl=kb != 8, margins=False), O.encode(V, Pv, qjl=False, margins=False)
    t0 = time.perf_counter()
    O.attend(Q, Pk, Ek, Pv, Ev)
    return time.perf_counter() - t0, G * L


def _oracle_codec_slice(kind: str, n: int, L: int):
    """One KV head of the alternative-codec parts on the oracle: encode L keys
    and L values, then score them for 4 query heads.  (seconds, units)."""
    from kv_cache_vector_07_b200 import synth
    from oracle import oracle as O
    d = 128
    K = synth.outlier_normal((L, d), seed=90 + n, dtype=torch.float32).numpy().astype(np.float64)
    V = synth.outlier_normal((L, d), seed=91 + n, dtype=torch.float32).numpy().astype(np.float64)
    Q = synth.normal((4, d), seed=92 + n, dtype=torch.float32).numpy().astype(np.float64)
    if kind == "dense":
        Pk, Pv = O.make_params(d, 2, 1005, rotation="dense"), O.make_params(d, 4, 2005, False, rotation="dense")
    elif kind == "polar":
        Pk, Pv = O.polar_params(d, 1005), O.polar_params(d, 2005, with_S=False)
    else:
        Pk, Pv = O.make_params(d, 2.5, 1005), O.make_params(d, 3.5, 2005, with_S=False)
    t0 = time.perf_counter()
    if kind == "polar":
        Ek, Ev = O.encode_polar(K, Pk, qjl=True), O.encode_polar(V, Pv, qjl=False)
    else:
        Ek, Ev = O.encode(K, Pk, qjl=True, margins=False), O.encode(V, Pv, qjl=False, margins=False)
    O.attend(Q, Pk, Ek, Pv, Ev)
    return time.perf_counter() - t0, 2 * L + 4 * L


def _oracle_sample(workload: str, n: int, small: bool):
    """One bounded sample of the workload on the oracle: (seconds, units)."""
    if workload in ("dense", "frac35", "polar"):
        return _oracle_codec_slice(workload, n, 2048 if small else 8192)
    if workload == "encode":
        return _oracle_encode_slice(n, 4096 if small else 32768)
    if workload == "step":
        t1, u1 = _oracle_encode_slice(n, 4096 if small else 32768)
        t2, u2 = _oracle_attend_slice("decode32k", n, 4096 if small else 32768)
        return t1 + t2, u1 + u2
    if workload in ("decode32k", "decode_k8v4", "decode_step"):
        return _oracle_attend_slice("decode32k" if workload == "decode_step" else workload, n,
                                    8192 if small else 32768)
    if workload == "longctx":
        return _oracle_attend_slice("longctx", n, 8192 if small else 65536)
    return _oracle_attend_slice("search", n, 5000 if small else 20000)


SAMPLE_TEXT = {
    "encode": "(sequence, KV head) slices of the write path: {L} keys and {L} values, compressed with k8v4 and "
              "with K 4-bit + QJL / V 4-bit",
    "step": "(sequence, KV head) slices of the step: the write-path slice ({L} keys and {L} values under both "
            "presets) plus 4 query heads scored over {L} k3v4 keys (encode of the decode slice untimed)",
    "decode32k": "slices of one KV head: 4 query heads over {L} k3v4 keys (encode untimed)",
    "decode_k8v4": "slices of one KV head: 4 query heads over {L} k8v4 keys (encode untimed)",
    "decode_step": "slices of one KV head: 4 query heads over {L} k3v4 keys (encode untimed)",
    "dense": "slices of one KV head: encode {L} keys and {L} values (k3v4, dense rotation), score 4 query heads",
    "frac35": "slices of one KV head: encode {L} keys and {L} values (3.5-bit rates), score 4 query heads",
    "polar": "slices of one KV head: encode {L} keys and {L} values (PolarQuant codes), score 4 query heads",
    "longctx": "slices of one KV head: 8 query heads over {L} keys (K 2-bit + QJL, V 3-bit; encode untimed)",
    "search": "slices: 4 queries over {L} oracle-encoded d=1024 vectors (encode untimed)",
}
SAMPLE_L = {"encode": (4096, 32768), "step": (4096, 32768), "decode32k": (8192, 32768),
            "decode_k8v4": (8192, 32768), "decode_step": (8192, 32768), "longctx": (8192, 65536),
            "dense": (2048, 8192), "frac35": (2048, 8192), "polar": (2048, 8192),
            "search": (5000, 20000)}


def cpu_baseline(workload: str, budget_s: float = 15.0):
    from oracle import oracle as O
    O.build()
    cores = len(os.sched_getaffinity(0))
    os.environ.setdefault("OMP_NUM_THREADS", str(cores))
    O.codebook(128, 4)
    units, spent, n = 0, 0.0, 0
    wall0 = time.perf_counter()
    while (spent < budget_s and time.perf_counter() - wall0 < 4 * budget_s) or n == 0:
        dt, u = _oracle_sample(workload, n, small=False)
        spent += dt
        units += u
        n += 1
    sample = f"{n} " + SAMPLE_TEXT[workload].format(L=SAMPLE_L[workload][1]) + " (float64 oracle, OpenMP)"
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
    os.environ.setdefault("OMP_NUM_THREADS", str(cores))
    for i in range(args.warmup):
        _oracle_sample(args.workload, 1000 + i, small=True)
    spent, units = 0.0, 0
    for s in range(args.steps):
        dt, u = _oracle_sample(args.workload, s, small=True)
        spent += dt
        units += u
    value = units / spent
    sizes = {k: v for k, v in (("batch", args.batch), ("seq_len", args.seq_len), ("n_db", args.n_db),
                               ("n_q", args.n_q)) if v}
    sample = "per step one " + SAMPLE_TEXT[args.workload].format(L=SAMPLE_L[args.workload][0]).replace("slices", "slice")
    line = {"metric": WORKLOAD_METRICS[args.workload], "value": value, "unit": "units/s",
            "unit_note": UNIT_NOTES[args.workload], "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": spent * 1e3 / max(1, args.steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)", "config": workload_config(args.workload, sizes), "impl": "reference",
            "cpu_baseline": {"kind": "oracle", "cores": cores, "value": value, "unit": "units/s", "sample": sample},
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
    ap.add_argument("--no-parts", action="store_true", help="skip the parts timed outside the step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=10.0)
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

#!/usr/bin/env python
"""Benchmark of the online-softmax attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Default workload ("vitl"): V-JEPA2 ViT-L encoder attention, B=1, H=16, S=2048,
D=64, bf16, scale 1/8; one step = the 24 layers' worth of independent calls
(24 distinct seeded input sets, 384 MiB per step, so every call's inputs come
from HBM: the inputs are larger than the 126 MB L2). The default run (one GPU)
also measures the other configurations of the metric -- "tiny", "dinov3",
"decode" (GQA decode, HBM bound, 4 rotating input sets) and "paged" (history-only
attention over the FP8 paged cache) -- each with its own roofline, clocks and
CPU-oracle sample, under the "configs" key of the same JSON line. Further
workloads (--workload): "vitl8k", "enc_d128", "gte", "decode_g8", "decode_d512",
"decode_window", "paged_prefill", "rope_vitl", "vitl_block" (the whole attention
block of a ViT-L layer: QKV projection with RoPE, attention, output projection).

Output: ONE JSON line on rank 0. `value` is whole-job throughput over all ranks
(attention TFLOP/s, or GB/s for decode) with inputs resident in HBM, timed with
CUDA events on the launching stream between barriers, max over ranks. `e2e` is
the same metric through the public API with pinned host buffers (host->device
copies of the step's inputs and device->host copies of its outputs inside the
timed region; for the multi-set encoder workloads the copies of one set overlap
the compute of the previous one, on streams of their own). `roofline` relates the dominant kernel to the measured peak in
MEASURED_PEAKS.json. `cpu_baseline` times the fp64 CPU oracle on a bounded
sample (rank 0, N=1 only).

Multi-GPU: launched by torchrun, one process per GPU; every rank runs the same
workload on its own GPU (independent problems, no data-path collective), so
scaling is weak.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention TFLOP/s (encoder/prefill) & KV GB/s (decode) vs B200 roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

WORKLOADS = {
    "vitl": dict(kind="encoder", B=1, H=16, S=2048, D=64, scale=0.125, sets=24, seed0=2000,
                 name="vitl_b1_h16_s2048_d64_x24layers"),
    "tiny": dict(kind="encoder", B=1, H=4, S=256, D=64, scale=0.125, sets=1, seed0=1001,
                 name="tiny_mha_b1_h4_s256_d64"),
    "dinov3": dict(kind="encoder", B=8, H=16, S=201, D=64, scale=0.125, sets=1, seed0=1003,
                   name="dinov3_b8_h16_s201_d64"),
    "decode": dict(kind="decode", B=8, Hq=16, Hkv=8, S=4096, D=256, scale=1.0, sets=4,
                   seed0=1004, name="gqa_decode_b8_16q_8kv_d256_ctx4096"),
    "paged": dict(kind="paged", Hq=32, Hkv=2, Sq=4096, D=256, NB=256, BS=512, L=100000,
                  scale=1.0 / 16, sets=1, seed0=1005,
                  name="paged_history_32q_2kv_d256_q4096_hist100000_fp8"),
    # wider shapes the pages name beyond the five headline configurations
    "vitl8k": dict(kind="encoder", B=1, H=16, S=8192, D=64, scale=0.125, sets=4, seed0=2100,
                   name="vitl_native_b1_h16_s8192_d64"),
    "enc_d128": dict(kind="encoder", B=1, H=16, S=2048, D=128, scale=128 ** -0.5, sets=12,
                     seed0=2200, name="encoder_b1_h16_s2048_d128_x12"),
    "gte": dict(kind="encoder", B=16, H=12, S=512, D=64, scale=0.125, sets=4, seed0=2300,
                pad=(128, 512), name="gte_b16_h12_s512_d64_rightpad_128_512"),
    # the headline decode with 8 query heads per kv head (same K/V bytes, 4x the heads)
    "decode_g8": dict(kind="decode", B=8, Hq=64, Hkv=8, S=4096, D=256, scale=1.0, sets=4,
                      seed0=2900, name="gqa_decode_b8_64q_8kv_d256_ctx4096"),
    "decode_d512": dict(kind="decode", B=8, Hq=16, Hkv=8, S=4096, D=512, scale=512 ** -0.5,
                        sets=4, seed0=2400, name="gqa_decode_b8_16q_8kv_d512_ctx4096"),
    "decode_window": dict(kind="decode", B=8, Hq=16, Hkv=8, S=4096, D=256, scale=1.0, sets=4,
                          seed0=2500, window=1024,
                          name="gqa_decode_b8_16q_8kv_d256_ctx4096_window1024"),
    # chunked prefill over the paged FP8 cache: 8 sequences, history + causal current tokens
    "paged_prefill": dict(kind="prefill", Hq=32, Hkv=2, D=256, BS=512, n_seqs=8,
                          hist=(4096, 16384), qlen=(512, 2048), scale=1.0 / 16, sets=1,
                          seed0=2700, name="paged_prefill_8seq_32q_2kv_d256_hist4k_16k_q512_2k_fp8"),
    # the whole attention block of a ViT-L layer: QKV projection with RoPE in its epilogue,
    # attention, output projection (random-init Linear weights), 24 layers
    "vitl_block": dict(kind="block", B=1, H=16, S=2048, D=64, C=1024, scale=0.125, sets=24,
                       seed0=2800, interleaved=True,
                       name="vitl_attention_block_b1_s2048_c1024_h16_d64_x24layers"),
    # the RoPE prologue of the ViT-L encoder (V-JEPA2 pairs lanes 2j, 2j+1), 24 layers
    "rope_vitl": dict(kind="rope", B=1, H=16, S=2048, D=64, sets=24, seed0=2600, interleaved=True,
                      name="rope_qk_vitl_b1_h16_s2048_d64_interleaved_x24layers"),
}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def profiled_traffic(kernel_regex: str, workload: str):
    """DRAM bytes per launch from profiles/dram_traffic.txt, if captured on a build whose
    sources for this kernel are the current ones (per-kernel digest)."""
    from online_softmax_attention_flash_b200.build import KERNEL_SOURCES, source_digest
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path) or kernel_regex not in KERNEL_SOURCES:
        return None
    digest = source_digest(kernel_regex)
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) == 4 and not line.startswith("#"):
                if parts[0] == kernel_regex and parts[1] == workload and parts[3] == digest:
                    return int(parts[2])
    return None


# --------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.12)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self._t.join(timeout=2)
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = max(mx, float(parts[1]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[3:7]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def gpu_smi_id(device) -> str:
    """nvidia-smi -i accepts a GPU UUID; CUDA_VISIBLE_DEVICES may renumber indices."""
    import torch
    try:
        return "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
    except Exception:
        return str(device.index or 0)


# ------------------------------------------------------------------ workloads
class CopyPipeline:
    """End-to-end step over independent input sets with the copies overlapped: each set's
    host->device copy runs on its own stream, the attention on the launching stream, the
    device->host copy on a third, so set i's input copy overlaps set i-1's compute and set
    i-2's output copy (PCIe carries both directions at once). Events keep a set's device
    buffers from being overwritten while a previous step still reads them."""

    def __init__(self, device, n):
        import torch
        self.s_in = torch.cuda.Stream(device)
        self.s_out = torch.cuda.Stream(device)
        ev = lambda: [torch.cuda.Event() for _ in range(n)]
        self.in_done, self.comp_done, self.out_done = ev(), ev(), ev()
        self.n = n
        self.first = True

    def run(self, stream, h2d, compute, d2h):
        import torch
        start = torch.cuda.Event()
        start.record(stream)
        self.s_in.wait_event(start)
        self.s_out.wait_event(start)
        for i in range(self.n):
            with torch.cuda.stream(self.s_in):
                if not self.first:   # the previous step's compute has read set i's inputs
                    self.s_in.wait_event(self.comp_done[i])
                h2d(i)
                self.in_done[i].record(self.s_in)
            stream.wait_event(self.in_done[i])
            if not self.first:       # the previous step's output copy of set i is done
                stream.wait_event(self.out_done[i])
            compute(i, stream)
            self.comp_done[i].record(stream)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(self.comp_done[i])
                d2h(i)
                self.out_done[i].record(self.s_out)
        end = torch.cuda.Event()
        end.record(self.s_out)
        stream.wait_event(end)
        self.first = False


class EncoderWork:
    def __init__(self, cfg, device):
        import torch
        from online_softmax_attention_flash_b200 import inputs as syn
        self.cfg = cfg
        self.sets = []
        self.host = []
        for i in range(cfg["sets"]):
            c = encoder_host_case(cfg, i)
            self.host.append(c)
            self.sets.append(tuple(t.to(device) for t in (c.q, c.k, c.v)))
        self.bias = [c.key_bias.to(device) if c.key_bias is not None else None for c in self.host]
        self.out = [torch.empty_like(s[0]) for s in self.sets]
        B, H, S, D = cfg["B"], cfg["H"], cfg["S"], cfg["D"]
        self.flops_per_launch = 4.0 * B * H * S * S * D
        self.launches_per_step = cfg["sets"]
        self.work_per_step = self.flops_per_launch * cfg["sets"]
        self.unit, self.bound = "TFLOP/s", "tensor"
        # head dim 64 (with or without a key bias) runs the one-query-tile kernel
        self.kernel_regex = "encoder_1q_kernel" if D == 64 else "encoder_fwd_kernel"
        self.peak_ratio = 1.0
        self.dtype = "bf16"

    def step(self, stream=None):
        from online_softmax_attention_flash_b200 import binding as Bd
        for (q, k, v), kb, o in zip(self.sets, self.bias, self.out):
            Bd.attn_encoder_fwd(q, k, v, self.cfg["scale"], key_bias=kb, out=o, stream=stream)

    def rate(self, work, seconds):
        return work / seconds / 1e12

    # end-to-end through the public API with pinned host buffers
    def e2e_setup(self):
        import torch
        self.h_in = [tuple(t.pin_memory() for t in (c.q, c.k, c.v)) for c in self.host]
        self.h_bias = [c.key_bias.pin_memory() if c.key_bias is not None else None for c in self.host]
        self.h_out = [torch.empty_like(c.q).pin_memory() for c in self.host]
        self.h2d = sum(t.numel() * t.element_size() for s in self.h_in for t in s)
        self.h2d += sum(t.numel() * t.element_size() for t in self.h_bias if t is not None)
        self.d2h = sum(t.numel() * t.element_size() for t in self.h_out)

    def e2e_step(self, stream):
        from online_softmax_attention_flash_b200 import binding as Bd
        if getattr(self, "pipe", None) is None:
            self.pipe = CopyPipeline(stream.device, len(self.sets))

        def h2d(i):
            if self.h_bias[i] is not None:
                self.bias[i].copy_(self.h_bias[i], non_blocking=True)
            for d, h in zip(self.sets[i], self.h_in[i]):
                d.copy_(h, non_blocking=True)

        def compute(i, st):
            q, k, v = self.sets[i]
            Bd.attn_encoder_fwd(q, k, v, self.cfg["scale"], key_bias=self.bias[i], out=self.out[i],
                                stream=st)

        def d2h(i):
            self.h_out[i].copy_(self.out[i], non_blocking=True)

        self.pipe.run(stream, h2d, compute, d2h)

    # CPU oracle on a bounded sample of the same workload
    def oracle_sample(self, step_idx, rows=256):
        import oracle
        c = self.host[step_idx % len(self.host)]
        S = self.cfg["S"]
        h = step_idx % self.cfg["H"]
        r0 = (step_idx * rows) % max(1, S - rows + 1) if S > rows else 0
        rr = np.arange(r0, min(S, r0 + rows))
        b = step_idx % self.cfg["B"]
        q = c.q[b:b + 1, h:h + 1].double().numpy()
        k = c.k[b:b + 1, h:h + 1].double().numpy()
        v = c.v[b:b + 1, h:h + 1].double().numpy()
        kb = c.key_bias[b:b + 1].double().numpy() if c.key_bias is not None else None
        oracle.encoder_attention(q, k, v, self.cfg["scale"], key_bias=kb, rows=rr)
        return 4.0 * len(rr) * S * self.cfg["D"], f"{len(rr)} query rows x {S} keys of one head"


def encoder_host_case(cfg, i):
    """Seeded encoder inputs; with cfg["pad"] = (lo, hi) every batch entry gets a right-padding
    length drawn from U{lo..hi} (gte-style 0/1 attention mask as an additive key bias)."""
    from online_softmax_attention_flash_b200 import inputs as syn
    pads = None
    if "pad" in cfg:
        g = np.random.default_rng(cfg["seed0"] + 7919 * i)
        pads = g.integers(cfg["pad"][0], cfg["pad"][1] + 1, size=cfg["B"]).tolist()
    return syn.encoder_case(cfg["B"], cfg["H"], cfg["S"], cfg["D"], seed=cfg["seed0"] + i,
                            softmax_scale=cfg["scale"], pad_lengths=pads)


def decode_host_case(cfg, i):
    """Seeded decode inputs; with cfg["window"] = W only the last W positions before each
    length stay unmasked (sliding-window layers)."""
    from online_softmax_attention_flash_b200 import inputs as syn
    c = syn.decode_case(cfg["B"], cfg["Hq"], cfg["Hkv"], cfg["S"], cfg["D"],
                        seed=cfg["seed0"] + 100 * i, softmax_scale=cfg["scale"])
    if "window" in cfg:
        for b in range(cfg["B"]):
            L = int(c.lengths[b])
            c.attn_mask[b, ..., :max(0, L - cfg["window"])] = float("-inf")
    return c


def live_lengths(cfg, c):
    """Keys each batch entry actually attends to (the bytes decode must read)."""
    lens = [int(x) for x in c.lengths]
    return [min(L, cfg["window"]) for L in lens] if "window" in cfg else lens


class DecodeWork:
    def __init__(self, cfg, device):
        import torch
        from online_softmax_attention_flash_b200 import binding as Bd
        from online_softmax_attention_flash_b200 import inputs as syn
        import oracle
        self.cfg = cfg
        self.host, self.sets = [], []
        for i in range(cfg["sets"]):
            c = decode_host_case(cfg, i)
            self.host.append(c)
            self.sets.append(tuple(t.to(device) for t in (c.q, c.k, c.v, c.attn_mask)))
        self.out = [torch.empty_like(s[0]) for s in self.sets]
        ws = Bd.attn_gqa_decode_workspace_size(cfg["B"], cfg["Hq"], cfg["Hkv"], cfg["S"], cfg["D"])
        self.ws = torch.empty(ws, dtype=torch.uint8, device=device)
        self.bytes = [oracle.decode_algorithmic_bytes(live_lengths(cfg, c), cfg["Hkv"], cfg["D"],
                                                      cfg["Hq"], cfg["S"]) for c in self.host]
        self.launches_per_step = 3   # scan + stream + combine
        self.work_per_step = float(np.mean(self.bytes))
        self.flops_per_launch = self.work_per_step
        self.unit, self.bound = "GB/s", "hbm"
        # 4 or more query heads per kv head (D <= 256) stream on the tensor cores
        G = cfg["Hq"] // cfg["Hkv"]
        self.kernel_regex = ("decode_stream_mma_kernel" if G >= 4 and cfg["D"] <= 256
                             else "decode_stream_kernel")
        self.peak_ratio = 1.0
        self.dtype = "bf16"
        self.i = 0

    def step(self, stream=None):
        from online_softmax_attention_flash_b200 import binding as Bd
        j = self.i % len(self.sets)
        self.i += 1
        q, k, v, m = self.sets[j]
        Bd.attn_gqa_decode(q, k, v, m, self.cfg["scale"], self.cfg["Hq"] // self.cfg["Hkv"],
                           out=self.out[j], workspace=self.ws, stream=stream)

    def rate(self, work, seconds):
        return work / seconds / 1e9

    def e2e_setup(self):
        import torch
        c = self.host[0]
        self.h_in = tuple(t.pin_memory() for t in (c.q, c.k, c.v, c.attn_mask))
        self.h_out = torch.empty_like(c.q).pin_memory()
        self.h2d = sum(t.numel() * t.element_size() for t in self.h_in)
        self.d2h = self.h_out.numel() * self.h_out.element_size()

    def e2e_step(self, stream):
        from online_softmax_attention_flash_b200 import binding as Bd
        q, k, v, m = self.sets[0]
        for d, h in zip((q, k, v, m), self.h_in):
            d.copy_(h, non_blocking=True)
        Bd.attn_gqa_decode(q, k, v, m, self.cfg["scale"], self.cfg["Hq"] // self.cfg["Hkv"],
                           out=self.out[0], workspace=self.ws, stream=stream)
        self.h_out.copy_(self.out[0], non_blocking=True)

    def e2e_work(self):
        return self.bytes[0]

    def oracle_sample(self, step_idx):
        import oracle
        c = self.host[step_idx % len(self.host)]
        b = step_idx % self.cfg["B"]
        oracle.gqa_decode_attention(c.q[b:b + 1].double().numpy(), c.k[b:b + 1].double().numpy(),
                                    c.v[b:b + 1].double().numpy(),
                                    c.attn_mask[b:b + 1].double().numpy(), self.cfg["scale"],
                                    self.cfg["Hq"] // self.cfg["Hkv"])
        L = live_lengths(self.cfg, c)[b]
        byt = L * self.cfg["Hkv"] * self.cfg["D"] * 4 + 2 * self.cfg["Hq"] * self.cfg["D"] * 2
        return float(byt), "one batch entry (all heads) of the decode step"


class RopeWork:
    """attn_rope_qk over 24 distinct (q, k) sets; HBM bound: each call reads and writes q and k
    and reads the [S, D/2] cos / sin tables."""

    def __init__(self, cfg, device):
        import torch
        from online_softmax_attention_flash_b200 import inputs as syn
        self.cfg = cfg
        self.host = [rope_host_case(cfg, i) for i in range(cfg["sets"])]
        self.sets = [tuple(t.to(device) for t in (q, k)) for q, k in self.host]
        cos, sin = syn.rope_tables(cfg["S"], cfg["D"])
        self.tables = (cos.to(device), sin.to(device))
        self.h_tables = (cos, sin)
        self.out = [(torch.empty_like(q), torch.empty_like(k)) for q, k in self.sets]
        B, H, S, D = cfg["B"], cfg["H"], cfg["S"], cfg["D"]
        self.bytes_per_call = 4.0 * B * H * S * D * 2 + 2.0 * S * (D // 2) * 4
        self.launches_per_step = cfg["sets"]
        self.work_per_step = self.bytes_per_call * cfg["sets"]
        self.flops_per_launch = self.bytes_per_call
        self.unit, self.bound = "GB/s", "hbm"
        self.kernel_regex = "rope_qk_kernel"
        self.peak_ratio = 1.0
        self.dtype = "f32 (bf16 in / out)"

    def step(self, stream=None):
        from online_softmax_attention_flash_b200 import binding as Bd
        for (q, k), (qo, ko) in zip(self.sets, self.out):
            Bd.attn_rope_qk(q, k, *self.tables, interleaved=self.cfg["interleaved"], q_out=qo,
                            k_out=ko, stream=stream)

    def rate(self, work, seconds):
        return work / seconds / 1e9

    def e2e_setup(self):
        import torch
        self.h_in = [tuple(t.pin_memory() for t in s) for s in self.host]
        self.h_out = [tuple(torch.empty_like(t).pin_memory() for t in s) for s in self.host]
        self.h2d = sum(t.numel() * t.element_size() for s in self.h_in for t in s)
        self.d2h = sum(t.numel() * t.element_size() for s in self.h_out for t in s)

    def e2e_step(self, stream):
        from online_softmax_attention_flash_b200 import binding as Bd
        for (hq, hk), (q, k), (qo, ko), (hqo, hko) in zip(self.h_in, self.sets, self.out, self.h_out):
            q.copy_(hq, non_blocking=True)
            k.copy_(hk, non_blocking=True)
            Bd.attn_rope_qk(q, k, *self.tables, interleaved=self.cfg["interleaved"], q_out=qo,
                            k_out=ko, stream=stream)
            hqo.copy_(qo, non_blocking=True)
            hko.copy_(ko, non_blocking=True)

    def e2e_work(self):
        return self.work_per_step

    def oracle_sample(self, step_idx):
        import oracle
        q, k = self.host[step_idx % len(self.host)]
        h = step_idx % self.cfg["H"]
        c, s = (t.double().numpy() for t in self.h_tables)
        mode = "interleaved" if self.cfg["interleaved"] else "half"
        for x in (q, k):
            oracle.rope_apply(x[0, h].double().numpy(), c, s, mode)
        S, D = self.cfg["S"], self.cfg["D"]
        return 4.0 * S * D * 2 + 2.0 * S * (D // 2) * 4, "the q and k rows of one head"


class BlockWork:
    """attn_qkv_rope_proj -> attn_encoder_fwd -> attn_out_proj for 24 layers (distinct inputs
    and random-init weights per layer). All three kernels are bf16 tensor-core work: the
    roofline is the block's algorithmic flops over its time against the bf16 peak."""

    def __init__(self, cfg, device):
        import torch
        from online_softmax_attention_flash_b200 import inputs as syn
        self.cfg = cfg
        B, S, C, H, D = cfg["B"], cfg["S"], cfg["C"], cfg["H"], cfg["D"]
        self.host = [syn.projection_case(B, S, C, H, D, seed=cfg["seed0"] + i)
                     for i in range(cfg["sets"])]
        self.h_tables = syn.rope_tables(S, D)
        self.tables = tuple(t.to(device) for t in self.h_tables)
        self.dev = [dict(x=c.x.to(device), w_qkv=c.w_qkv.to(device), b_qkv=c.b_qkv.to(device),
                         w_o=c.w_o.to(device), b_o=c.b_o.to(device)) for c in self.host]
        shp = (B, H, S, D)
        self.bufs = [dict(q=torch.empty(shp, dtype=torch.bfloat16, device=device),
                          k=torch.empty(shp, dtype=torch.bfloat16, device=device),
                          v=torch.empty(shp, dtype=torch.bfloat16, device=device),
                          o=torch.empty(shp, dtype=torch.bfloat16, device=device),
                          y=torch.empty((B, S, C), dtype=torch.float32, device=device))
                     for _ in self.host]
        HD = H * D
        self.flops_qkv = 2.0 * B * S * C * 3 * HD
        self.flops_attn = 4.0 * B * H * S * S * D
        self.flops_out = 2.0 * B * S * HD * C
        self.flops_per_launch = (self.flops_qkv + self.flops_attn + self.flops_out) / 3
        self.launches_per_step = 3 * cfg["sets"]
        self.work_per_step = (self.flops_qkv + self.flops_attn + self.flops_out) * cfg["sets"]
        self.unit, self.bound = "TFLOP/s", "tensor"
        self.kernel_regex = "proj_gemm_kernel|" + ("encoder_1q_kernel" if D == 64 else "encoder_fwd_kernel")
        self.peak_ratio = 1.0
        self.dtype = "bf16"

    def _layer(self, d, bf, stream):
        from online_softmax_attention_flash_b200 import binding as Bd
        c = self.cfg
        Bd.attn_qkv_rope_proj(d["x"], d["w_qkv"], d["b_qkv"], c["H"], c["D"], *self.tables,
                              interleaved=c["interleaved"], q=bf["q"], k=bf["k"], v=bf["v"],
                              stream=stream)
        Bd.attn_encoder_fwd(bf["q"], bf["k"], bf["v"], c["scale"], out=bf["o"], stream=stream)
        Bd.attn_out_proj(bf["o"], d["w_o"], d["b_o"], y=bf["y"], stream=stream)

    def step(self, stream=None):
        for d, bf in zip(self.dev, self.bufs):
            self._layer(d, bf, stream)

    def rate(self, work, seconds):
        return work / seconds / 1e12

    def e2e_setup(self):
        import torch
        self.h_x = [c.x.pin_memory() for c in self.host]
        self.h_y = [torch.empty_like(bf["y"], device="cpu").pin_memory() for bf in self.bufs]
        self.h2d = sum(t.numel() * t.element_size() for t in self.h_x)
        self.d2h = sum(t.numel() * t.element_size() for t in self.h_y)

    def e2e_step(self, stream):
        if getattr(self, "pipe", None) is None:
            self.pipe = CopyPipeline(stream.device, len(self.dev))
        self.pipe.run(stream,
                      lambda i: self.dev[i]["x"].copy_(self.h_x[i], non_blocking=True),
                      lambda i, st: self._layer(self.dev[i], self.bufs[i], st),
                      lambda i: self.h_y[i].copy_(self.bufs[i]["y"], non_blocking=True))

    def oracle_sample(self, step_idx, rows=256):
        import oracle
        c = self.host[step_idx % len(self.host)]
        cfg = self.cfg
        S, C, H, D = cfg["S"], cfg["C"], cfg["H"], cfg["D"]
        h = step_idx % H
        # one head's q, k, v for every token, its attention for `rows` queries, and the
        # out-projection of those rows (this head's share of the sum)
        sel = np.concatenate([np.arange(w * H * D + h * D, w * H * D + (h + 1) * D) for w in range(3)])
        x = c.x.double().numpy()
        q, k, v = oracle.qkv_rope_projection(x, c.w_qkv.double().numpy()[sel],
                                             c.b_qkv.double().numpy()[sel], 1, D,
                                             *(t.double().numpy() for t in self.h_tables),
                                             "interleaved" if cfg["interleaved"] else "half")
        r0 = (step_idx * rows) % (S - rows + 1)
        rr = np.arange(r0, r0 + rows)
        o = oracle.encoder_attention(q, k, v, cfg["scale"], rows=rr)
        oracle.out_projection(o, c.w_o.double().numpy()[:, h * D:(h + 1) * D], None)
        flops = 2.0 * S * C * 3 * D + 4.0 * rows * S * D + 2.0 * rows * D * C
        return flops, f"one head of one layer: q/k/v of all {S} tokens, {rows} query rows"


def rope_host_case(cfg, i):
    from online_softmax_attention_flash_b200 import inputs as syn
    import torch
    g = torch.Generator().manual_seed(cfg["seed0"] + i)
    shape = (cfg["B"], cfg["H"], cfg["S"], cfg["D"])
    return syn.randn_bf16(shape, g), syn.randn_bf16(shape, g)


class PagedWork:
    def __init__(self, cfg, device):
        import torch
        from online_softmax_attention_flash_b200 import inputs as syn
        self.cfg = cfg
        c = syn.paged_case(cfg["Hq"], cfg["Hkv"], cfg["Sq"], cfg["D"], cfg["NB"], cfg["BS"],
                           cfg["L"], seed=cfg["seed0"], softmax_scale=cfg["scale"])
        self.host = [c]
        self.dev = tuple(t.to(device) for t in (c.q, c.k_cache, c.v_cache, c.block_table))
        self.out = torch.empty_like(self.dev[0])
        self.flops_per_launch = 4.0 * cfg["Sq"] * cfg["Hq"] * cfg["L"] * cfg["D"]
        self.launches_per_step = 1
        self.work_per_step = self.flops_per_launch
        self.unit, self.bound = "TFLOP/s", "tensor"
        self.kernel_regex = "paged_history_kernel"
        # both matmuls are kind::f8f6f4 MMAs: the peak is the fp8 one (2x bf16 nominal)
        self.peak_ratio = 2.0
        self.dtype = "e4m3 (q and p as hi+lo e4m3 pairs), fp32 accumulate"

    def _call(self, stream):
        from online_softmax_attention_flash_b200 import binding as Bd
        c = self.host[0]
        q, kc, vc, bt = self.dev
        Bd.attn_paged_history(q, kc, vc, bt, c.block_size, c.actual_history_len, c.k_scale,
                              c.v_scale, c.softmax_scale, c.num_kv_groups, out=self.out,
                              stream=stream)

    def step(self, stream=None):
        self._call(stream)

    def rate(self, work, seconds):
        return work / seconds / 1e12

    def e2e_setup(self):
        import torch
        c = self.host[0]
        self.h_in = tuple(t.pin_memory() for t in (c.q, c.k_cache, c.v_cache, c.block_table))
        self.h_out = torch.empty_like(c.q).pin_memory()
        self.h2d = sum(t.numel() * t.element_size() for t in self.h_in)
        self.d2h = self.h_out.numel() * self.h_out.element_size()

    def e2e_step(self, stream):
        for d, h in zip(self.dev, self.h_in):
            d.copy_(h, non_blocking=True)
        self._call(stream)
        self.h_out.copy_(self.out, non_blocking=True)

    def oracle_sample(self, step_idx, rows=16):
        import oracle
        c = self.host[0]
        h = step_idx % self.cfg["Hq"]
        r0 = (step_idx * rows) % self.cfg["Sq"]
        rr = np.arange(r0, min(self.cfg["Sq"], r0 + rows))
        # one query head against its kv head only
        g = h // c.num_kv_groups
        oracle.paged_history_attention(c.q[h:h + 1].double().numpy(),
                                       c.k_cache[:, g:g + 1].numpy(), c.v_cache[:, g:g + 1].numpy(),
                                       c.k_scale, c.v_scale, c.block_table.numpy(), c.block_size,
                                       c.actual_history_len, c.softmax_scale, 1, rows=rr)
        return 4.0 * len(rr) * self.cfg["L"] * self.cfg["D"], f"{len(rr)} query rows of one head"


def prefill_host_case(cfg):
    from online_softmax_attention_flash_b200 import inputs as syn
    g = np.random.default_rng(cfg["seed0"])
    hist = g.integers(cfg["hist"][0], cfg["hist"][1] + 1, size=cfg["n_seqs"]).tolist()
    qlen = g.integers(cfg["qlen"][0], cfg["qlen"][1] + 1, size=cfg["n_seqs"]).tolist()
    return syn.paged_prefill_case(cfg["Hq"], cfg["Hkv"], cfg["D"], cfg["BS"], hist, qlen,
                                  seed=cfg["seed0"], softmax_scale=cfg["scale"])


def prefill_flops(c, Hq, D):
    """4 * Hq * D per (query, visible key) pair: query i of a sequence sees hist + i + 1 keys."""
    tot = 0
    for s in range(len(c.hist_lens)):
        n = int(c.q_start[s + 1] - c.q_start[s])
        h = int(c.hist_lens[s])
        tot += n * h + n * (n + 1) // 2
    return 4.0 * Hq * D * tot


class PrefillWork(PagedWork):
    """attn_paged_prefill on several sequences (fp8 MMAs, like the history kernel)."""

    def __init__(self, cfg, device):
        import torch
        self.cfg = cfg
        c = prefill_host_case(cfg)
        self.host = [c]
        self.dev = tuple(t.to(device) for t in (c.q, c.k_cache, c.v_cache, c.block_tables,
                                                c.q_start, c.hist_lens))
        self.max_q = int((c.q_start[1:] - c.q_start[:-1]).max())
        self.out = torch.empty_like(self.dev[0])
        self.flops_per_launch = prefill_flops(c, cfg["Hq"], cfg["D"])
        self.launches_per_step = 1
        self.work_per_step = self.flops_per_launch
        self.unit, self.bound = "TFLOP/s", "tensor"
        self.kernel_regex = "paged_history_kernel"
        self.peak_ratio = 2.0
        self.dtype = "e4m3 (q and p as hi+lo e4m3 pairs), fp32 accumulate"

    def _call(self, stream):
        from online_softmax_attention_flash_b200 import binding as Bd
        c = self.host[0]
        q, kc, vc, bt, qs, hl = self.dev
        Bd.attn_paged_prefill(q, kc, vc, bt, qs, hl, c.k_scale, c.v_scale, c.softmax_scale,
                              c.num_kv_groups, max_q_len=self.max_q, out=self.out, stream=stream)

    def e2e_setup(self):
        import torch
        c = self.host[0]
        self.h_in = tuple(t.pin_memory() for t in (c.q, c.k_cache, c.v_cache, c.block_tables,
                                                   c.q_start, c.hist_lens))
        self.h_out = torch.empty_like(c.q).pin_memory()
        self.h2d = sum(t.numel() * t.element_size() for t in self.h_in)
        self.d2h = self.h_out.numel() * self.h_out.element_size()

    def oracle_sample(self, step_idx, rows=16):
        import oracle
        import torch
        c = self.host[0]
        s = step_idx % len(c.hist_lens)
        h = step_idx % self.cfg["Hq"]
        g = h // c.num_kv_groups
        a, b = int(c.q_start[s]), int(c.q_start[s + 1])
        r0 = (step_idx * rows) % (b - a)
        rr = np.arange(r0, min(b - a, r0 + rows))
        oracle.paged_prefill_attention(c.q[h:h + 1, a:b].double().numpy(), c.k_cache[:, g:g + 1].numpy(),
                                       c.v_cache[:, g:g + 1].numpy(), c.k_scale, c.v_scale,
                                       c.block_tables[s:s + 1].numpy(), c.block_size,
                                       np.array([0, b - a]), c.hist_lens[s:s + 1].numpy(),
                                       c.softmax_scale, 1, rows=rr)
        hist = int(c.hist_lens[s])
        pairs = sum(hist + int(i) + 1 for i in rr)
        return 4.0 * pairs * self.cfg["D"], f"{len(rr)} query rows of one head of one sequence"


# steps captured per CUDA graph for the timed region (decode rotates 4 input sets)
GRAPH_STEPS = {"vitl": 1, "tiny": 20, "dinov3": 20, "decode": 4, "paged": 1, "vitl8k": 1,
               "enc_d128": 1, "gte": 4, "decode_d512": 4, "decode_window": 4, "rope_vitl": 1,
               "paged_prefill": 1, "vitl_block": 1, "decode_g8": 4}


def make_work(name, device):
    cfg = WORKLOADS[name]
    return {"encoder": EncoderWork, "decode": DecodeWork, "paged": PagedWork,
            "rope": RopeWork, "prefill": PrefillWork, "block": BlockWork}[cfg["kind"]](cfg, device)


# --------------------------------------------------------------------- oracle
def cpu_oracle_run(work, budget_s: float, max_steps=None, start=0):
    """Time the oracle (as it stands) on a bounded sample; returns (rate, secs, sample, steps)."""
    done, total, n, sample = 0.0, 0.0, 0, ""
    t_end = time.perf_counter() + budget_s
    while True:
        t0 = time.perf_counter()
        w, sample = work.oracle_sample(start + n)
        total += time.perf_counter() - t0
        done += w
        n += 1
        if (max_steps is not None and n >= max_steps) or (max_steps is None and time.perf_counter() > t_end):
            break
    return work.rate(done, total), total, sample, n


def cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ------------------------------------------------------------------- arms
def run_reference(args, info):
    """The reference arm: the fp64 CPU oracle timed on the host cores (rank 0 only)."""
    if not info.is_main:
        return 0
    cfg = WORKLOADS[args.workload]
    work = make_work_host_only(args.workload)
    for i in range(args.warmup):
        work.oracle_sample(i)
    rate, secs, sample, n = cpu_oracle_run(work, 0, max_steps=args.steps, start=args.warmup)
    line = {
        "impl": "reference", "metric": METRIC, "value": rate, "unit": work.unit,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * secs / max(1, n), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg["name"], "sample_per_step": sample},
        "cpu_baseline": {"value": rate, "unit": work.unit, "cores": cores(), "kind": "oracle",
                         "sample": f"each step: {sample}"},
        "e2e": {"value": rate, "unit": work.unit, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def make_work_host_only(name):
    """Host-side inputs only (the oracle arm never touches a GPU)."""
    cfg = WORKLOADS[name]
    cls = {"encoder": EncoderWork, "decode": DecodeWork, "paged": PagedWork,
           "rope": RopeWork, "prefill": PrefillWork, "block": BlockWork}[cfg["kind"]]
    obj = cls.__new__(cls)
    obj.cfg = cfg
    from online_softmax_attention_flash_b200 import inputs as syn
    if cfg["kind"] == "encoder":
        obj.host = [encoder_host_case(cfg, i) for i in range(cfg["sets"])]
        obj.unit = "TFLOP/s"
    elif cfg["kind"] == "decode":
        obj.host = [decode_host_case(cfg, i) for i in range(cfg["sets"])]
        obj.unit = "GB/s"
    elif cfg["kind"] == "prefill":
        obj.host = [prefill_host_case(cfg)]
        obj.unit = "TFLOP/s"
    elif cfg["kind"] == "block":
        obj.host = [syn.projection_case(cfg["B"], cfg["S"], cfg["C"], cfg["H"], cfg["D"],
                                        seed=cfg["seed0"] + i) for i in range(cfg["sets"])]
        obj.h_tables = syn.rope_tables(cfg["S"], cfg["D"])
        obj.unit = "TFLOP/s"
    elif cfg["kind"] == "rope":
        obj.host = [rope_host_case(cfg, i) for i in range(cfg["sets"])]
        obj.h_tables = syn.rope_tables(cfg["S"], cfg["D"])
        obj.unit = "GB/s"
    else:
        obj.host = [syn.paged_case(cfg["Hq"], cfg["Hkv"], cfg["Sq"], cfg["D"], cfg["NB"], cfg["BS"],
                                   cfg["L"], seed=cfg["seed0"], softmax_scale=cfg["scale"])]
        obj.unit = "TFLOP/s"
    return obj


# the other configurations the headline metric is quoted on, measured in the same default run
# (1 GPU): steps per config, chosen so each timed region is about a tenth of a second or more
CONFIG_STEPS = {"tiny": 2000, "dinov3": 2000, "decode": 2000, "paged": 60}


def time_work(work, workload, steps, warmup, info, device, stream, use_graph):
    """Warm up, then time `steps` steps (CUDA-graph replays of the same C-ABI launches) with
    CUDA events on the launching stream between barriers; clocks sampled meanwhile."""
    import torch
    from online_softmax_attention_flash_b200 import binding as Bd
    from online_softmax_attention_flash_b200 import dist as D
    for _ in range(warmup):
        work.step(stream)
    torch.cuda.synchronize(device)
    st = Bd.attn_check(stream)
    if st != 0:
        raise RuntimeError(f"{workload}: device status after warm-up: {Bd.STATUS.get(st, st)}")
    # The timed region replays CUDA graphs that capture the same C-ABI launches (n steps per
    # graph), so per-call host overhead (Python, ctypes, tensor-map encoding) is not timed.
    n_graph = math.gcd(GRAPH_STEPS[workload], steps) if use_graph else 1
    graph = None
    if use_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for _ in range(n_graph):
                work.step(None)
        for _ in range(2):
            graph.replay()
        torch.cuda.synchronize(device)
    replays = steps // n_graph
    sampler = ClockSampler(gpu_smi_id(device))
    sampler.start()
    time.sleep(0.2)
    D.barrier(info)
    torch.cuda.synchronize(device)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(replays + 1)]
    ev[0].record(stream)
    for i in range(replays):
        if graph is not None:
            graph.replay()
        else:
            work.step(stream)
        ev[i + 1].record(stream)
    torch.cuda.synchronize(device)
    D.barrier(info)
    clocks = sampler.stop()
    step_ms = [ev[i].elapsed_time(ev[i + 1]) / n_graph for i in range(replays)]
    total_ms = ev[0].elapsed_time(ev[-1])
    launch_mode = f"cuda_graph ({n_graph} steps per graph)" if graph is not None else "eager"
    del graph
    st = Bd.attn_check(stream)
    if st != 0:
        raise RuntimeError(f"{workload}: device status after timing: {Bd.STATUS.get(st, st)}")
    return total_ms, step_ms, clocks, launch_mode


def roofline_of(work, workload, total_ms, steps, clocks=None):
    """Dominant kernel: algorithmic work per launch / mean launch time against the peak.
    Tensor-bound kernels are held against the burst GEMM peak when timed alone, and against
    the sustained one when the timed region is long (over a second) or the 1 kW power cap
    held the SM clock down meanwhile (sw_power_cap active and a median clock more than 5%
    below the maximum; a cap that leaves the clock at its maximum changes nothing)."""
    peaks, peak_src = load_peaks()
    per_launch_ms = total_ms / (steps * work.launches_per_step)
    if work.bound == "hbm":
        # decode: one call = scan + stream + combine; achieved counts the whole call's time
        per_call_ms = total_ms / steps
        achieved = work.work_per_step / (per_call_ms / 1e3) / 1e9
        peak = float(peaks["hbm_gbs"])
        peak_name = "hbm_gbs"
    else:
        achieved = work.flops_per_launch / (per_launch_ms / 1e3) / 1e12
        capped = (bool(clocks) and "sw_power_cap" in clocks.get("reasons", [])
                  and clocks.get("sm_mhz") is not None and clocks.get("sm_max_mhz")
                  and clocks["sm_mhz"] < 0.95 * clocks["sm_max_mhz"])
        sustained = total_ms > 1000.0 or capped
        peak_name = "bf16_tflops_sustained" if sustained else "bf16_tflops"
        peak = float(peaks[peak_name]) * work.peak_ratio
        if work.peak_ratio != 1.0:
            peak_name += f" x {work.peak_ratio:g} (fp8/bf16 nominal ratio)"
    return {"bound": work.bound, "achieved": achieved, "peak": peak, "unit": work.unit,
            "frac": achieved / peak, "traffic": profiled_traffic(work.kernel_regex, workload),
            "peak_source": f"{peak_src} ({peak_name})", "kernel": work.kernel_regex}


def step_stats(step_ms):
    s_sorted = sorted(step_ms)
    return {"min": s_sorted[0], "median": statistics.median(step_ms),
            "mean": statistics.fmean(step_ms),
            "p90": s_sorted[min(len(s_sorted) - 1, int(0.9 * len(s_sorted)))],
            "max": s_sorted[-1]}


def measure_config(name, args, info, device, stream):
    """One more configuration, measured like the headline (own clocks, own roofline), with a
    short oracle sample on the host cores beside it."""
    import torch
    work = make_work(name, device)
    steps = CONFIG_STEPS[name]
    total_ms, step_ms, clocks, mode = time_work(work, name, steps, 5, info, device, stream,
                                                args.graph)
    entry = {"workload": WORKLOADS[name]["name"],
             "value": work.rate(work.work_per_step * steps, total_ms / 1e3), "unit": work.unit,
             "ms_per_step": total_ms / steps, "steps": steps, "launch": mode,
             "step_ms": step_stats(step_ms),
             "roofline": roofline_of(work, name, total_ms, steps, clocks),
             "clocks": clocks, "dtype": work.dtype,
             "gpu_launches": steps * work.launches_per_step}
    if not args.no_cpu_baseline:
        rate, secs, sample, n = cpu_oracle_run(work, args.config_cpu_budget)
        entry["cpu_baseline"] = {"value": rate, "unit": work.unit, "cores": cores(),
                                 "kind": "oracle",
                                 "sample": f"{n} samples of {sample} ({secs:.1f} s of fp64 NumPy)"}
    del work
    torch.cuda.empty_cache()
    return entry


def run_product(args, info):
    import torch
    from online_softmax_attention_flash_b200 import binding as Bd
    from online_softmax_attention_flash_b200 import dist as D

    torch.cuda.set_device(info.local_rank)
    device = torch.device("cuda", info.local_rank)
    Bd.load_library()
    work = make_work(args.workload, device)
    stream = torch.cuda.current_stream(device)

    total_ms, step_ms, clocks, launch_mode = time_work(work, args.workload, args.steps, args.warmup,
                                                       info, device, stream, args.graph)
    max_ms = D.max_over_ranks(total_ms, info, device)
    work_all = work.work_per_step * args.steps * info.world_size
    value = work.rate(work_all, max_ms / 1e3)
    roofline = roofline_of(work, args.workload, total_ms, args.steps, clocks)

    # end to end through the public API with host buffers
    work.e2e_setup()
    e2e_steps = max(1, min(args.steps, 10))
    work.e2e_step(stream)
    torch.cuda.synchronize(device)
    D.barrier(info)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        work.e2e_step(stream)
    e1.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = D.max_over_ranks(e0.elapsed_time(e1), info, device)
    e2e_work = getattr(work, "e2e_work", lambda: work.work_per_step)()
    e2e = {"value": work.rate(e2e_work * e2e_steps * info.world_size, e2e_ms / 1e3),
           "unit": work.unit, "h2d_bytes_per_step": int(work.h2d),
           "d2h_bytes_per_step": int(work.d2h), "steps": e2e_steps}

    dtype, launches = work.dtype, args.steps * work.launches_per_step
    # the remaining configurations of the metric, 1 GPU, same run (default workload only)
    configs = None
    if info.world_size == 1 and args.workload == "vitl" and args.configs:
        configs = {n: measure_config(n, args, info, device, stream) for n in CONFIG_STEPS}

    if not info.is_main:
        return 0
    cpu = None
    if info.world_size == 1 and not args.no_cpu_baseline:
        rate, secs, sample, n = cpu_oracle_run(work, args.cpu_budget)
        cpu = {"value": rate, "unit": work.unit, "cores": cores(), "kind": "oracle",
               "sample": f"{n} samples of {sample} ({secs:.1f} s of fp64 NumPy)"}
    cfg = WORKLOADS[args.workload]
    line = {
        "metric": METRIC, "value": value, "unit": work.unit, "n_gpus": info.world_size,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": max_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": dtype, "data": "synthetic",
        "config": {"workload": cfg["name"],
                   **{k: v for k, v in cfg.items() if k not in ("kind", "name", "seed0")},
                   "l2": ("inputs larger than L2: distinct input sets rotate across calls"
                          if cfg["sets"] > 1 or cfg["kind"] in ("paged", "prefill") else "inputs fit in L2"),
                   "parallelism": f"replicas x{info.world_size}", "launch": launch_mode},
        "step_ms": step_stats(step_ms),
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if configs is not None:
        line["configs"] = configs
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=None)
    p.add_argument("--warmup", type=int, default=None)
    p.add_argument("--workload", default="vitl", choices=sorted(WORKLOADS))
    p.add_argument("--impl", default="product", choices=["product", "reference"])
    p.add_argument("--cpu-budget", type=float, default=12.0,
                   help="seconds of oracle work for cpu_baseline")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-graph", dest="graph", action="store_false",
                   help="time eager calls instead of CUDA-graph replays")
    p.add_argument("--no-configs", dest="configs", action="store_false",
                   help="skip the other configurations of the default run")
    p.add_argument("--config-cpu-budget", type=float, default=3.0,
                   help="seconds of oracle work per additional configuration")
    args = p.parse_args(argv)
    defaults = {"vitl": (1000, 20), "tiny": (2000, 20), "dinov3": (2000, 20),
                "decode": (2000, 20), "paged": (100, 5), "vitl8k": (400, 10),
                "enc_d128": (1000, 20), "gte": (2000, 20), "decode_d512": (2000, 20),
                "decode_window": (2000, 20), "rope_vitl": (1000, 20),
                "paged_prefill": (30, 5), "vitl_block": (300, 10),
                "decode_g8": (2000, 20)}[args.workload]
    if args.steps is None:
        args.steps = defaults[0]
    if args.warmup is None:
        args.warmup = defaults[1]
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    from online_softmax_attention_flash_b200 import dist as D
    info = D.rank_info_from_env()
    if args.impl == "reference":
        # the oracle arm runs on rank 0 only; other ranks exit without work
        return run_reference(args, info)
    info = D.init("nccl" if info.world_size > 1 else "gloo")
    if info.world_size != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={info.world_size}")
    try:
        return run_product(args, info)
    finally:
        D.shutdown(info)


if __name__ == "__main__":
    sys.exit(main())

"""Benchmark plumbing: algorithmic cost of a decode step, peaks, the clock
sampler, L2 flush and the max-over-ranks reduction.
"""

from __future__ import annotations

import json
import os
import statistics
import subprocess
import threading
import time

import numpy as np

FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
L2_BYTES = 126 * 1024 * 1024


def kv_bytes_per_token(shape) -> int:
    """Cache bytes one context token contributes (the whole row is read once:
    latent row, the tied vectors of GTA, or K and V of every KV head)."""
    if shape.latent or shape.tied:
        return 2 * shape.row_elems
    elem = 1 if getattr(shape, "cache_dtype", "bf16") == "fp8" else 2
    return elem * 2 * shape.num_kv * shape.d_nope


def flops_per_token(shape) -> int:
    """2 flops per multiply-add of q.k and p.v over every head (and branch)."""
    per_head = 2 * (shape.key_dim + shape.value_dim)
    units = shape.num_kv if shape.variant == "mlra" else 1
    return shape.num_q_heads * units * per_head


def step_cost(shape, seq_lens) -> dict:
    """Algorithmic bytes and flops of one decode call over the whole batch."""
    n_tok = int(np.sum(seq_lens))
    q_rows = shape.batch * shape.num_q_heads * (shape.num_kv if shape.variant == "mlra" else 1)
    q_bytes = 2 * q_rows * shape.key_dim
    out_bytes = shape.batch * shape.num_q_heads * shape.d_nope * (4 if shape.out_dtype == "fp32" else 2)
    lse_bytes = 4 * shape.batch * shape.lse_rows
    pages = int(sum((int(x) + shape.page_size - 1) // shape.page_size for x in seq_lens))
    meta_bytes = 4 * pages + 4 * shape.batch
    kv = n_tok * kv_bytes_per_token(shape)
    return {
        "tokens": n_tok,
        "kv_bytes": kv,
        "decode_bytes": kv + q_bytes + meta_bytes,
        "bytes": kv + q_bytes + meta_bytes + out_bytes + lse_bytes,
        "flops": n_tok * flops_per_token(shape),
    }


def read_peaks(root: str) -> dict:
    """Measured peaks from MEASURED_PEAKS.json, else the machine's fallback figures."""
    path = os.path.join(root, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": 1400.0, "source": "fallback"}


_SMI_FIELDS = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
               "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
               "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled in a background process."""

    def __init__(self, bus_id: str | None = None, period_ms: int = 50):
        self.bus_id = (bus_id or "").lower()
        self.period_ms = period_ms
        self.samples = []          # (host time, sm_mhz, max_mhz, power, {reason: active})
        self._proc = None
        self._thread = None

    def start(self):
        try:
            self._proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={_SMI_FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(self.period_ms)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
        except OSError:
            self._proc = None
            return self
        self._thread = threading.Thread(target=self._read, daemon=True)
        self._thread.start()
        return self

    def _read(self):
        for line in self._proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            bus = parts[0].lower()
            if self.bus_id and not (bus.endswith(self.bus_id) or self.bus_id.endswith(bus)):
                continue
            try:
                sm, mx = float(parts[1]), float(parts[2])
                pw = float(parts[3]) if parts[3] not in ("[N/A]", "N/A") else float("nan")
            except ValueError:
                continue
            reasons = {r: parts[5 + i].lower() == "active" for i, r in enumerate(_REASONS)}
            self.samples.append((time.time(), sm, mx, pw, reasons))

    def stop(self):
        if self._proc is not None:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self._proc.kill()
        if self._thread is not None:
            self._thread.join(timeout=5)

    def summary(self, t0: float, t1: float) -> dict:
        return self.summary_windows([(t0, t1)])

    def summary_windows(self, windows) -> dict:
        """Median SM clock, max clock and active throttle reasons over the
        samples inside any of the (t0, t1) windows."""
        inside = [s for s in self.samples if any(t0 <= s[0] <= t1 for t0, t1 in windows)]
        window = "timed"
        t0, t1 = min(w[0] for w in windows), max(w[1] for w in windows)
        if len(inside) < 2:
            # the timed region was shorter than the sampling period: take the
            # samples nearest to it
            inside = sorted(self.samples, key=lambda s: min(abs(s[0] - t0), abs(s[0] - t1)))[:5]
            window = "nearest"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "window": "none"}
        reasons = sorted({r for s in inside for r, a in s[4].items() if a})
        pw = [s[3] for s in inside if s[3] == s[3]]
        return {"sm_mhz": statistics.median(s[1] for s in inside), "sm_max_mhz": max(s[2] for s in inside),
                "reasons": reasons, "samples": len(inside), "window": window,
                "power_w_max": max(pw) if pw else None}


def max_over_ranks(x: float, device=None) -> float:
    """Max of a float over the ranks of the default process group (or x)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank draws its own batch (data parallel over sequences)."""
    return int(base_seed) + 1000 * int(rank)

#!/usr/bin/env python
"""Decode-attention benchmark on B200.

    python bench.py --gpus N --steps K --warmup W [--workload NAME] [--impl reference]

The default workload is the whole suite: every decode problem of the
benchmark (``shared_kv_caches_b200.workloads.WORKLOADS`` minus the tiny parity
case) is timed in turn, each with its own warm-up and K timed steps.  The
headline (``value``, ``ms_per_step``, ``roofline``, ``e2e``) is absorbed MLA
at the DeepSeek-V3 shape (batch 64, 128 query heads, latent 512 + rope 64,
ragged contexts drawn uniformly from [4096, 32768] on a paged 64-token bf16
cache with a permuted block table), the largest problem that fits one GPU;
``suite`` carries the same figures for GQA, MFA, GLA-2 and the four MLRA-4
shapes, and GTA and MFA-KR (the GQA and MFA shapes with tied keys and
values).  ``--workload NAME`` times one problem (or ``gqa+mfa``, the GQA and
MFA layers together as one step); ``--workload steps`` only the steps either
side of attention.

A step is one decode call of a problem (split pass + combine pass) over one
batch of seeded synthetic input that is already resident in HBM.

Timing: W untimed warm-up steps, then exactly K steps, each bracketed by CUDA
events on the launching stream, with a 252 MiB write between steps (outside
the events) so every step starts with a cold L2; a barrier and a device
synchronisation on both sides of each timed loop; the max over ranks is
taken.  The per-pass split (``kernels_us``: decode and combine) comes from up
to 50 further steps with an event between the passes.  With N GPUs every rank runs its own batch (data parallel over
sequences, no collective on the data path; weak scaling).

The JSON line also carries: the roofline of each problem's decode kernel
(algorithmic bytes or flops per launch / its event-timed duration against the
measured peak), the end-to-end number through the public API with host
buffers, the oracle timed on the host cores for the headline problem (rank 0,
N = 1), SM clocks sampled during the timed regions, and how many of the
library's kernels ran in the headline's timed region.

``steps`` times the steps either side of attention at the benchmark shapes
(query absorption and up-projection per head, the query RoPE, the cache
append): calls back to back over input replicas larger than L2, against each
op's algorithmic HBM bytes.

``--impl reference`` times the fp64 CPU oracle (the reference arm) on the
headline problem, each step a bounded sample of it, and prints the same line
with ``"impl": "reference"``.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WORKLOAD_SETS = {"gqa+mfa": ("gqa", "mfa")}
SUITE = ("mla", "gqa", "mfa", "gla", "mlra_128k", "mlra_512k", "mlra_1m", "mlra_b8_128k", "gta", "mfa_kr",
         "gqa_fp8")
DEFAULT_WORKLOAD = "suite"
METRIC = "decode_attn_tokens_per_s"
UNIT = "tokens/s"


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--splits", type=int, default=0, help="force parts per context (0: library choice)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-steps", action="store_true", help="skip the steps either side of attention")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU seconds of the oracle sample")
    a = ap.parse_args(argv)
    if a.warmup < 3:
        ap.error("--warmup must be at least 3")
    if a.steps < 1:
        ap.error("--steps must be at least 1")
    return a


def problem_names(workload):
    """Problems timed together as one step (the suite's headline is its first)."""
    if workload == "suite":
        return SUITE[:1]
    if workload in WORKLOAD_SETS:
        return WORKLOAD_SETS[workload]
    from shared_kv_caches_b200.workloads import WORKLOADS
    if workload not in WORKLOADS:
        raise SystemExit(f"unknown workload {workload}")
    return (workload,)


def describe(names):
    from shared_kv_caches_b200.workloads import WORKLOADS
    parts = []
    for n in names:
        s = WORKLOADS[n]
        lo, hi = s.ctx
        ctx = f"{lo}" if lo == hi else f"U[{lo},{hi}]"
        if s.latent:
            kvdesc = {"mla": f"latent {s.d_nope}+rope {s.d_rope}",
                      "gla": f"{s.num_kv} latent heads x {s.d_nope} + shared rope {s.d_rope}",
                      "mlra": f"{s.num_kv} branches x {s.d_nope} + shared rope {s.d_rope}"}[s.variant]
        else:
            kvdesc = f"{s.num_kv} kv heads x {s.d_nope}"
        if s.cache_dtype != "bf16":
            kvdesc += f" {s.cache_dtype} e4m3 cache (k_scale {s.k_scale}, v_scale {s.v_scale})"
        parts.append(f"{s.variant} B={s.batch} H={s.num_q_heads} {kvdesc} ctx {ctx}")
    return "; ".join(parts)


KERNEL_SOURCES = {
    "gqa": ["decode_gqa.cu"],
    "gqa_fp8": ["decode_gqa_fp8.cu"],
    "mqa_tc": ["decode_mqa_mma.cu"],
    "latent_tc": ["decode_latent_tc.cu", "latent_common.cuh"],
    "latent_pair": ["decode_mla_pair.cu", "latent_common.cuh"],
    "generic": ["decode_generic.cu"],
}
SHARED_SOURCES = ["kvattn_internal.cuh", "sm100.cuh"]


def source_digest(kernel):
    """sha256 prefix over a decode kernel's sources and the shared headers, to
    tell whether a stored ncu traffic figure still describes that kernel."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "shared_kv_caches_b200", "csrc")
    for f in KERNEL_SOURCES.get(kernel, []) + SHARED_SOURCES:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def stored_traffic(workload, problem, digest):
    """DRAM bytes per launch of the decode kernel from the committed ncu
    summary, if it was captured on the current sources."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.md")
    if not os.path.exists(path):
        return None
    for line in open(path):
        cells = [c.strip() for c in line.strip().strip("|").split("|")]
        if len(cells) >= 5 and cells[0] == workload and cells[1] == problem and cells[4] == digest:
            try:
                return float(cells[3])
            except ValueError:
                return None
    return None


# --------------------------------------------------------------------- ours

def measure(names, args, dev, world, peaks, flush, workload_label, want_inputs=False):
    """Time one step (a decode call of every problem in ``names``): W warm-up
    steps, K event-timed steps with an L2 flush between them, then the same
    step end to end through the public API.  Returns the figures of the step
    and of its dominant decode kernel."""
    import numpy as np
    import torch

    from shared_kv_caches_b200 import benchutil as BU
    from shared_kv_caches_b200 import workloads as W
    from shared_kv_caches_b200.device import DeviceProblem

    rank = dist_rank()
    seed = BU.rank_seed(args.seed, rank)
    inputs = [W.make_inputs(W.WORKLOADS[n], seed=seed) for n in names]
    probs = [DeviceProblem(x, dev, num_splits=args.splits) for x in inputs]
    costs = [BU.step_cost(x["shape"], x["seq_lens"]) for x in inputs]
    batch = inputs[0]["shape"].batch
    Ev = torch.cuda.Event

    def step(evs=None):
        for i, p in enumerate(probs):
            p.run(events=None if evs is None else evs[i])

    for _ in range(args.warmup):
        step()
        flush.zero_()
    torch.cuda.synchronize()
    for p, n in zip(probs, names):
        if p.device_error():
            raise SystemExit(f"device error {p.device_error()} during warm-up of {n}")

    # The timed steps are plain calls: events only around the step, so the
    # combine pass keeps its programmatic dependent launch (its launch
    # overlaps the decode pass's tail, as in any caller's stream).
    K = args.steps
    step_ev = [(Ev(enable_timing=True), Ev(enable_timing=True)) for _ in range(K)]
    barrier(world)
    torch.cuda.synchronize()
    t0 = time.time()
    for k in range(K):
        step_ev[k][0].record()
        step()
        step_ev[k][1].record()
        flush.zero_()
    torch.cuda.synchronize()
    barrier(world)
    t1 = time.time()
    for p, n in zip(probs, names):
        if p.device_error():
            raise SystemExit(f"device error {p.device_error()} in the timed steps of {n}")

    step_ms = [a.elapsed_time(b) for a, b in step_ev]
    total_ms = BU.max_over_ranks(sum(step_ms), dev)
    ms_per_step = total_ms / K
    value = world * batch / (ms_per_step / 1e3)

    # Per-pass breakdown in separate steps: an event recorded between the
    # passes (kvattn_decode_timed) makes them run strictly one after the
    # other, so these times add up to a little more than a plain step.
    KB = min(K, 50)
    kern_ev = [[[Ev(enable_timing=True) for _ in range(3)] for _ in probs] for _ in range(KB)]
    # torch creates a CUDA event on its first record(); do that here so the
    # handles the library records exist
    for per_step in kern_ev:
        for trio in per_step:
            for e in trio:
                e.record()
    torch.cuda.synchronize()
    for k in range(KB):
        step(kern_ev[k])
        flush.zero_()
    torch.cuda.synchronize()
    decode_ms = [float(np.mean([kern_ev[k][i][0].elapsed_time(kern_ev[k][i][1]) for k in range(KB)]))
                 for i in range(len(probs))]
    combine_ms = [float(np.mean([kern_ev[k][i][1].elapsed_time(kern_ev[k][i][2]) for k in range(KB)]))
                  for i in range(len(probs))]

    # end to end through the public API with host buffers
    e2e = run_e2e(probs, K, flush, dev, world, batch)

    # roofline of the dominant kernel (the decode pass with the largest time)
    dom = int(np.argmax(decode_ms))
    c = costs[dom]
    t_s = decode_ms[dom] / 1e3
    t_mem = c["decode_bytes"] / (peaks["hbm_gbs"] * 1e9)
    t_tc = c["flops"] / (peaks["bf16_tflops"] * 1e12)
    digest = source_digest(probs[dom].plan_kernel_name())
    traffic = stored_traffic(workload_label, names[dom], digest)
    if t_tc > t_mem:
        achieved = c["flops"] / t_s / 1e12
        roof = {"bound": "tensor", "achieved": round(achieved, 2), "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops"], 4),
                "frac_hbm": round(c["decode_bytes"] / t_s / 1e9 / peaks["hbm_gbs"], 4)}
    else:
        achieved = c["decode_bytes"] / t_s / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4)}
    # the same launch against the sustained bf16 figure (a kernel timed inside
    # a long step): max(memory time, tensor time at the sustained peak) / time
    t_tc_sus = c["flops"] / (peaks["bf16_tflops_sustained"] * 1e12)
    roof["frac_sustained"] = round(max(t_mem, t_tc_sus) / t_s, 4)
    # the whole call (a plain step of a one-problem workload) against the binding roof
    call_s = ms_per_step / 1e3 if len(probs) == 1 else (decode_ms[dom] + combine_ms[dom]) / 1e3
    roof["frac_call"] = round(max(t_mem, t_tc) / call_s, 4)
    roof.update({"traffic": traffic, "kernel": f"{names[dom]} decode pass ({probs[dom].plan_kernel_name()})",
                 "algorithmic_bytes": c["decode_bytes"], "algorithmic_flops": c["flops"],
                 "launch_us": round(decode_ms[dom] * 1e3, 2),
                 "peak_source": peaks["source"] + " (burst)", "source_digest": digest})
    if traffic is not None:
        roof["traffic_per_algorithmic_byte"] = round(traffic / c["decode_bytes"], 3)

    total_bytes = sum(x["bytes"] for x in costs)
    total_tokens = sum(x["tokens"] for x in costs) // len(costs)
    out = {
        "names": list(names), "value": round(value, 1), "ms_per_step": round(ms_per_step, 5),
        "us_per_step": round(ms_per_step * 1e3, 2),
        "ctx_tokens_per_s": round(world * total_tokens / (ms_per_step / 1e3), 1),
        "hbm_gbs": round(total_bytes / (ms_per_step / 1e3) / 1e9, 1),
        "batch": batch, "ctx_tokens": total_tokens, "workload": describe(names),
        "kernels_us": {n: {"decode": round(d * 1e3, 2), "combine": round(cb * 1e3, 2),
                           "kernel": p.plan_kernel_name(), "splits": int(p.plan.num_splits),
                           "ctas": int(p.plan.ctas)}
                       for n, d, cb, p in zip(names, decode_ms, combine_ms, probs)},
        "roofline": roof, "e2e": e2e, "gpu_launches": K * sum(int(p.plan.launches) for p in probs),
        "window": (t0, t1),
    }
    if want_inputs:
        out["inputs"] = inputs
    del probs
    torch.cuda.empty_cache()
    return out


# The steps either side of attention at the benchmark shapes (rows = the
# problem's batch x query tokens, H = 128 heads): query absorption
# (W_UK, d_h = 128 -> the latent columns a head reads), the up-projection
# (W_UV, those columns -> d_v = 128; MLRA with its four branch blocks
# stacked), the query RoPE and the cache append of the newest tokens.
STEP_OPS = {
    "mla_absorb": ("proj", 64, 128, 128, 512),
    "mla_up": ("proj", 64, 128, 512, 128),
    "gla_absorb": ("proj", 64, 128, 128, 256),
    "gla_up": ("proj", 64, 128, 256, 128),
    "mlra_b8_absorb": ("proj", 8, 128, 128, 512),
    "mlra_b8_up": ("proj", 8, 128, 512, 128),
    "mla_rope_q": ("rope", 64 * 128, 64),
    "mla_append": ("append", "mla"),
}


def measure_steps(args, dev, peaks, flush):
    """Throughput of each step op as a model issues them, back to back on one
    stream: K calls cycle through enough replicas of the op's inputs (and
    outputs) to hold over 300 MB, so no call finds its operands in the 126 MB
    L2; one event pair around the K calls.  Against the op's algorithmic HBM
    bytes; all of them are bound by HBM."""
    import numpy as np
    import torch

    from shared_kv_caches_b200 import kvattn as K
    from shared_kv_caches_b200 import workloads as W
    from shared_kv_caches_b200.device import DeviceProblem

    gen = torch.Generator(device=dev).manual_seed(args.seed)
    st = torch.cuda.current_stream(dev).cuda_stream
    span = 300 << 20
    out = {}
    for name, spec in STEP_OPS.items():
        kind = spec[0]
        if kind == "proj":
            _, rows, heads, k, n = spec
            nbytes = 2 * (rows * heads * k + heads * k * n + rows * heads * n)
            reps = max(2, -(-span // nbytes))
            xs = [torch.randn((rows, heads, k), generator=gen, device=dev).to(torch.bfloat16) for _ in range(reps)]
            ws = [(torch.randn((heads, k, n), generator=gen, device=dev) / k ** 0.5).to(torch.bfloat16)
                  for _ in range(reps)]
            ys = [torch.empty((rows, heads, n), dtype=torch.bfloat16, device=dev) for _ in range(reps)]
            call = lambda i: K.kvattn_head_proj(xs[i].data_ptr(), ws[i].data_ptr(), ys[i].data_ptr(),
                                                K.KVATTN_OUT_BF16, rows, heads, k, n, None, st)
            what = f"y[{rows}][{heads}][{n}] = x[{rows}][{heads}][{k}] W[{heads}][{k}][{n}]"
        elif kind == "rope":
            _, rows, rd = spec
            nbytes = 2 * 2 * rows * rd + 4 * (rows // 128)
            reps = max(2, -(-span // nbytes))
            qs = [torch.randn((rows, rd), generator=gen, device=dev).to(torch.bfloat16) for _ in range(reps)]
            pos = torch.randint(0, 1 << 15, (rows // 128,), generator=gen, device=dev, dtype=torch.int32)
            call = lambda i: K.kvattn_rope(qs[i].data_ptr(), rows, rd, 0, rd, 128, pos.data_ptr(), W.ROPE_BASE, st)
            what = f"q_rope[{rows // 128}][128][{rd}] turned in place"
        else:
            s = W.WORKLOADS[spec[1]].replace(ctx=(4096, 4096))
            xin = W.make_step_inputs(s, seed=args.seed)
            prob = DeviceProblem(xin, dev)
            new = torch.from_numpy(np.ascontiguousarray(xin["new_kv"]).view(np.int16)).view(torch.bfloat16).to(dev)
            nbytes = 2 * 2 * new.numel() + 4 * s.batch + 4 * s.batch
            # replicas: the same rows written at 4096 different positions of
            # every sequence (each call writes other cache lines)
            reps = 4096
            pos = [torch.full((s.batch, 1), i, dtype=torch.int32, device=dev) for i in range(reps)]
            call = lambda i: K.kvattn_append_kv(prob.variant, prob.params, new.data_ptr(), pos[i].data_ptr(),
                                                prob.block_table.data_ptr(), prob.kv.data_ptr(), W.ROPE_BASE,
                                                None, st)
            what = f"{s.batch} new [{s.row_elems}] rows into the paged cache, k^R turned"
        for i in range(max(args.warmup, 3)):
            if call(i % reps):
                raise SystemExit(f"step op {name} refused")
        flush.zero_()
        n_t = max(args.steps, reps)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record()
        for i in range(n_t):
            call(i % reps)
        b.record()
        torch.cuda.synchronize()
        us = a.elapsed_time(b) * 1e3 / n_t
        gbs = nbytes / (us * 1e-6) / 1e9
        out[name] = {"op": what, "us": round(us, 2), "bytes": int(nbytes), "achieved_gbs": round(gbs, 1),
                     "frac_hbm": round(gbs / peaks["hbm_gbs"], 4), "calls": n_t, "replicas": reps}
        torch.cuda.empty_cache()
    return out


def dist_rank():
    return int(os.environ.get("RANK", "0"))


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def run_ours(args, rank, world, local):
    import torch
    import torch.distributed as dist

    from shared_kv_caches_b200 import benchutil as BU
    from shared_kv_caches_b200 import build as libbuild

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    if rank == 0:
        libbuild.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=dev)
        dist.barrier()
        if rank != 0:
            libbuild.build()

    flush = torch.empty(252 * 1024 * 1024, dtype=torch.uint8, device=dev)
    peaks = BU.read_peaks(ROOT)
    props = torch.cuda.get_device_properties(dev)
    bus = None
    if all(hasattr(props, a) for a in ("pci_domain_id", "pci_bus_id", "pci_device_id")):
        bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
    sampler = BU.ClockSampler(bus_id=bus).start()
    time.sleep(0.3)

    if args.workload == "steps":
        # the steps either side of attention alone (for profiling them)
        line = {"metric": "step_ops_us", "impl": "ours", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "steps_ops": measure_steps(args, dev, peaks, flush)}
        sampler.stop()
        if world > 1:
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps(line), flush=True)
        return 0
    groups = [(n,) for n in SUITE] if args.workload == "suite" else [problem_names(args.workload)]
    label = (lambda g: g[0]) if args.workload == "suite" else (lambda g: args.workload)
    cpu = None
    results = []
    for gi, g in enumerate(groups):
        want = gi == 0 and rank == 0 and world == 1 and not args.no_cpu_baseline
        r = measure(g, args, dev, world, peaks, flush, label(g), want_inputs=want)
        if want:
            cpu = cpu_baseline(r.pop("inputs"), args.cpu_seconds, r["batch"])
        results.append(r)
    sampler.stop()

    head = results[0]
    windows = [r["window"] for r in results]
    line = {
        "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": head["workload"], "name": "+".join(head["names"]),
                   "batch_per_gpu": head["batch"], "ctx_tokens_per_gpu": head["ctx_tokens"], "page_size": 64,
                   "seed": args.seed,
                   "l2": "flushed between timed steps (252 MiB write outside the events)",
                   "parallelism": f"dp{world} (independent batches per GPU)"},
        "us_per_step": head["us_per_step"],
        "ctx_tokens_per_s": head["ctx_tokens_per_s"],
        "hbm_gbs": head["hbm_gbs"],
        "kernels_us": head["kernels_us"],
        "roofline": head["roofline"],
        "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"],
        "clocks": sampler.summary_windows(windows),
        "clocks_headline": sampler.summary(*head["window"]),
    }
    if len(results) > 1:
        line["suite"] = {
            "+".join(r["names"]): {k: r[k] for k in ("workload", "value", "us_per_step", "ctx_tokens_per_s",
                                                     "hbm_gbs", "kernels_us", "roofline", "e2e",
                                                     "gpu_launches")}
            for r in results}
    if args.workload == "suite" and world == 1 and not args.no_steps:
        line["steps_ops"] = measure_steps(args, dev, peaks, flush)
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_e2e(probs, K, flush, dev, world, batch):
    """Same step through the public API with inputs copied from pinned host
    memory and results read back, every step, inside the timed region."""
    import torch

    from shared_kv_caches_b200 import benchutil as BU

    host_in, dev_in, host_out = [], [], []
    h2d = d2h = 0
    for p in probs:
        srcs = {"q_nope": p.q_nope, "q_rope": p.q_rope, "seq_lens": p.seq_lens, "block_table": p.block_table}
        hi, di = {}, {}
        for k, t in srcs.items():
            if t is None:
                continue
            hi[k] = t.cpu().pin_memory()
            di[k] = torch.empty_like(t)
            h2d += t.numel() * t.element_size()
        ho = {"out": torch.empty(p.out.shape, dtype=p.out.dtype).pin_memory(),
              "lse": torch.empty(p.lse.shape, dtype=p.lse.dtype).pin_memory()}
        d2h += sum(t.numel() * t.element_size() for t in (p.out, p.lse))
        host_in.append(hi)
        dev_in.append(di)
        host_out.append(ho)
    Ev = torch.cuda.Event
    evs = [(Ev(enable_timing=True), Ev(enable_timing=True)) for _ in range(K)]

    def one(k):
        evs[k][0].record()
        for p, hi, di, ho in zip(probs, host_in, dev_in, host_out):
            for key, t in hi.items():
                di[key].copy_(t, non_blocking=True)
            p.run(q_nope=di["q_nope"], q_rope=di.get("q_rope"), seq_lens=di["seq_lens"],
                  block_table=di.get("block_table"))
            ho["out"].copy_(p.out, non_blocking=True)
            ho["lse"].copy_(p.lse, non_blocking=True)
        evs[k][1].record()
        flush.zero_()

    for k in range(min(3, K)):
        one(k)
    torch.cuda.synchronize()
    for k in range(K):
        one(k)
    torch.cuda.synchronize()
    ms = BU.max_over_ranks(sum(a.elapsed_time(b) for a, b in evs), dev) / K
    return {"value": round(world * batch / (ms / 1e3), 1), "unit": UNIT, "ms_per_step": round(ms, 5),
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}


def _oracle_sample(inputs, target_s, seq_offset=0):
    """Pick a prefix of sequences (rotating from seq_offset) whose oracle run
    should take about target_s; returns the list of (problem index, b_list)."""
    import numpy as np

    from oracle import oracle
    # calibrate on the shortest sequence of the first problem
    x0 = inputs[0]
    lens = np.asarray(x0["seq_lens"])
    b_cal = int(np.argmin(lens))
    t = time.perf_counter()
    oracle.decode(x0, b_list=[b_cal])
    dt = max(time.perf_counter() - t, 1e-4)
    rate = max(int(lens[b_cal]), 1) / dt           # context tokens per second, problem 0
    batch = x0["shape"].batch
    per_tok = sum(max(1, _work_per_token(x)) for x in inputs) / max(1, _work_per_token(x0))
    budget_tokens = target_s * rate / per_tok
    chosen, acc = [], 0
    for i in range(batch):
        b = (seq_offset + i) % batch
        chosen.append(b)
        acc += int(lens[b])
        if acc >= budget_tokens:
            break
    return chosen


def _work_per_token(x):
    s = x["shape"]
    units = s.num_kv if s.variant == "mlra" else 1
    return s.num_q_heads * units * (s.key_dim + s.value_dim)


def cpu_baseline(inputs, target_s, batch):
    """The oracle as it stands, timed on this host's cores on a bounded sample
    of the same workload, scaled to the whole batch by context tokens."""
    import numpy as np

    from oracle import oracle
    oracle.build()
    chosen = _oracle_sample(inputs, target_s)
    t = time.perf_counter()
    for x in inputs:
        oracle.decode(x, b_list=chosen)
    dt = time.perf_counter() - t
    lens = np.asarray(inputs[0]["seq_lens"])
    frac = float(lens[chosen].sum()) / float(lens.sum())
    full_s = dt / frac
    return {"value": round(batch / full_s, 3), "unit": UNIT, "cores": oracle.default_threads(),
            "kind": "oracle",
            "sample": f"{len(chosen)} of {batch} sequences ({int(lens[chosen].sum())} of {int(lens.sum())} "
                      f"context tokens), all heads, every problem of the step; {dt:.2f} s measured, "
                      f"scaled by context tokens to {full_s:.2f} s per step"}


# ---------------------------------------------------------------- reference

def run_reference(args):
    """Reference arm: the fp64 oracle on the host cores, same workload."""
    import numpy as np

    from oracle import oracle
    from shared_kv_caches_b200 import benchutil as BU
    from shared_kv_caches_b200 import workloads as W

    oracle.build()
    names = problem_names(args.workload)
    inputs = [W.make_inputs(W.WORKLOADS[n], seed=BU.rank_seed(args.seed, 0)) for n in names]
    batch = inputs[0]["shape"].batch
    lens = np.asarray(inputs[0]["seq_lens"])
    per_step = max(0.2, min(20.0, 150.0 / (args.steps + args.warmup)))
    chosen0 = _oracle_sample(inputs, per_step)
    n = len(chosen0)
    times, fracs = [], []
    for k in range(args.warmup + args.steps):
        chosen = [(i + k * n) % batch for i in range(n)]
        t = time.perf_counter()
        for x in inputs:
            oracle.decode(x, b_list=chosen)
        dt = time.perf_counter() - t
        if k >= args.warmup:
            times.append(dt)
            fracs.append(float(lens[chosen].sum()) / float(lens.sum()))
    full_s = float(np.sum(times) / np.sum(fracs))       # seconds for the whole batch
    value = batch / full_s
    sample = (f"{n} of {batch} sequences per step (rotating), all heads, every problem; "
              f"{np.mean(times):.3f} s per sampled step, scaled by context tokens")
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(full_s * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": describe(names), "name": "+".join(names), "batch_per_gpu": batch,
                   "page_size": 64, "seed": args.seed},
        "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": oracle.default_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus and rank == 0:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    if args.impl == "reference":
        if rank != 0:
            return 0
        return run_reference(args)
    return run_ours(args, rank, world, local)


if __name__ == "__main__":
    sys.exit(main())

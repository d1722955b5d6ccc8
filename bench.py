#!/usr/bin/env python
"""Throughput of the gated-retention mixer on B200 through libgret.

One step = one gret_prefill call (gate, chunk decay sums, intra-chunk scores
and mask, intra and inter-chunk outputs, state carry, GroupNorm + swish
epilogue, final state) over one batch of a long-context prefill workload, bf16
I/O with fp32 state and gate logits -- the chunkwise prefill of "YOCO 深度技术分析"
(head dimension 128, contexts of 4K-64K tokens).  ``--config`` picks the
headline workload:

  c3  B1 H32 N65536, d_k = d_v = 128, chunk 128, gate logits ~ N(4, 1)  (default)
  c2  B4 H16 N4096,  d_k 128, d_v 256, chunk 64, gate logits ~ N(3, 1.5)
  c5  B2 H16 N32768, d_k 128, d_v 256, chunk 64, half the heads fast-decaying

Inputs are seeded synthetic tensors already resident in HBM (0.55-2.7 GB,
larger than the 126 MB L2, so no flush is needed between steps).  The other two
prefill workloads ride in the same JSON line under ``prefill_configs``, each
with its own roofline object.

The line also carries the recurrent decode step (256 sequences x 16 heads,
128 x 256 fp32 states, 64 consecutive launches) as ``decode``; the c2 tokens
packed as a ragged batch of sequences (gret_prefill_varlen) as ``varlen``;
one rank's computing steps of the sequence-parallel prefill (two slices of
2048 tokens of c2) as ``seqpar``; the c2 prefill with its gate logits
computed from z = X W_gamma in the gate prologue (gret_prefill_projected) as
``projected``; and the gradients of the c2 prefill (gret_prefill_backward) as
``backward``.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config c3|c2|c5] [--impl ours|reference]

Multi-GPU (weak scaling): one process per GPU, each runs its own batch; no
collective is on the data path.  ``--impl reference`` times the fp64 CPU
oracle on the host cores instead (rank 0 only).
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

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
METRIC = "gRet prefill Mtok/s & % bf16 TC peak; decode-step state GB/s & % HBM peak"
# ncu summaries (under profiles/) that carry the DRAM traffic of the timed kernels
DECODE_PROFILE = "decode_step_kernel_S256_H16_dk128_dv256.md"
PREFILL_SOURCE = "gated_retention_sequence_b200/csrc/gret_prefill_tc.cu"
# the prefill workloads a --config may name (c1 is the small fp32 parity case,
# c4 the decode workload)
PREFILL_CONFIGS = ("c3", "c2", "c5")


def fused_kernel_name(cfg):
    """The fused chunk-loop kernel that runs this workload (uniform batches):
    128-token chunks with d_v = 128 and every d_v = 256 request (as a CTA pair in
    128-token tiles) take the output-rows kernel, the others prefill_tc_kernel."""
    if cfg.io == "bf16" and ((cfg.dv == 128 and cfg.chunk == 128) or cfg.dv == 256):
        return "prefill_rows_kernel_pair" if cfg.dv == 256 else "prefill_rows_kernel"
    return "prefill_tc_kernel"


def prefill_profile(cfg):
    """Name of the ncu summary of the fused kernel on this workload."""
    return (f"{fused_kernel_name(cfg)}_B{cfg.B}_H{cfg.H}_N{cfg.N}_dk{cfg.dk}_dv{cfg.dv}_C{cfg.chunk}.md")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return dict(FALLBACK_PEAKS, source="fallback")


def prefill_alg(cfg):
    """Algorithmic bytes and flops of one prefill (per token and head:
    bytes e(2 dk + 3 dv) + 4 for Q, K, V, G, O and the fp32 gate logit;
    flops C(dk + dv) + 4 dk dv for the causal half of the intra-chunk products
    plus Q S and K^T V; plus the fp32 final state, 4 dk dv bytes per unit)."""
    e = 2 if cfg.io == "bf16" else 4
    th = cfg.B * cfg.N * cfg.H
    units = cfg.B * cfg.H
    bytes_ = th * (e * (2 * cfg.dk + 3 * cfg.dv) + 4) + units * 4 * cfg.dk * cfg.dv
    flops = th * (cfg.chunk * (cfg.dk + cfg.dv) + 4 * cfg.dk * cfg.dv)
    return bytes_, flops


def decode_alg(cfg):
    """Bytes of one decode step: the fp32 state read and written once, plus
    q, k, v, g, o and the gate logit."""
    e = 2 if cfg.io == "bf16" else 4
    units = cfg.num_seqs * cfg.H
    return units * (8 * cfg.dk * cfg.dv + e * (2 * cfg.dk + 3 * cfg.dv) + 4)


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the GPU works."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.tmp = None

    def start(self):
        try:
            self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50",
                 "-i", str(self.gpu)], stdout=self.tmp, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.tmp.flush()
        self.tmp.seek(0)
        rows = [r.strip().split(", ") for r in self.tmp.read().splitlines() if r.strip()]
        os.unlink(self.tmp.name)
        load, maxc, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm, mx, util = float(r[1]), float(r[2]), float(r[4])
            except (ValueError, IndexError):
                continue
            maxc = mx
            if util > 0:
                load.append(sm)
                for n, v in zip(names, r[6:10]):
                    if v.strip() == "Active":
                        reasons.add(n)
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": maxc,
                "reasons": sorted(reasons), "samples_under_load": len(load)}


def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    """Largest value of x over all ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, units_per_rank: float, steps: int, max_ms: float) -> float:
    """Whole-job rate (units per second) of `world` ranks that each processed
    `units_per_rank` per step for `steps` steps, timed by the slowest rank."""
    return world * units_per_rank * steps / (max_ms / 1e3)


def barrier(world):
    import torch
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


# The output-rows kernel's text within its source file (from the first marker
# up to the second): its ncu summary records the sha256 of this text only.
ROWS_KERNEL_TEXT = ("// Fused chunk loop for 128-token chunks with d_v = 128, output held as rows.",
                    "// ---------------------------------------------------------------- host side")


def kernel_digest(source, markers=None):
    """sha256 of a kernel source file, or of the text between two markers in it."""
    import hashlib
    with open(os.path.join(ROOT, source), "rb") as f:
        data = f.read()
    if markers:
        a = data.index(markers[0].encode())
        b = data.index(markers[1].encode(), a)
        data = data[a:b]
    return hashlib.sha256(data).hexdigest()


def profiled_traffic(kernel_file, source, markers=None):
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) that
    an ncu capture recorded in profiles/<kernel_file>, provided the capture was
    taken of the kernel source as it is now (its sha256 prefix is written next
    to the figure); None otherwise."""
    import re
    try:
        with open(os.path.join(ROOT, "profiles", kernel_file)) as f:
            text = f.read()
        digest = kernel_digest(source, markers)
    except (OSError, ValueError):
        return None
    m = re.search(r"^traffic_bytes_per_launch: (\d+) .*sha256 ([0-9a-f]{16})", text, re.M)
    if not m or not digest.startswith(m.group(2)):
        return None
    return int(m.group(1))


def oracle_sample_inputs(cfg, units, tokens):
    """Per-unit inputs of the first `tokens` tokens of `units` (batch, head)
    units of cfg, drawn on their own (element-identical to the full tensors),
    stacked as a [1, tokens, units, d] batch for the oracle."""
    import gret_inputs as gi
    import torch
    per = []
    for u in range(units):
        b, h = divmod(u % (cfg.B * cfg.H), cfg.H)
        per.append(gi.prefill_unit_inputs(cfg, b, h, tokens=tokens))
    return {n: torch.stack([p[n] for p in per], 1)[None] for n in ("Q", "K", "V", "G", "z")}


def oracle_sample_tokens(cfg, seconds):
    """Tokens per unit of a bounded oracle sample: each unit runs on its own
    host thread, and the fp64 recurrence costs about 4 dk dv flops per token
    at roughly 1 GFLOP/s per core."""
    return int(min(cfg.N, max(cfg.chunk, seconds * 1e9 / (4.0 * cfg.dk * cfg.dv))))


def cpu_oracle_sample(cfg, units, threads, min_seconds=0.0, tokens=None, inputs=None):
    """Time the fp64 oracle (as it stands) on the first `tokens` tokens of
    `units` (batch, head) units of cfg, repeating the call until at least
    `min_seconds` have passed.  Returns (Mtok/s, seconds, passes, tokens);
    one token is one position of the sequence with all H heads."""
    import oracle
    tokens = cfg.N if tokens is None else min(tokens, cfg.N)
    x = inputs if inputs is not None else oracle_sample_inputs(cfg, units, tokens)
    t0 = time.perf_counter()
    passes = 0
    while True:
        oracle.prefill(x["Q"], x["K"], x["V"], x["z"], x["G"], cfg.tau, cfg.eps, threads=threads)
        passes += 1
        dt = time.perf_counter() - t0
        if dt >= min_seconds:
            break
    token_heads = passes * units * tokens
    return token_heads / cfg.H / dt / 1e6, dt, passes, tokens


def config_of(name, seq_len=0):
    import gret_inputs as gi
    cfg = gi.CONFIGS[name]
    if seq_len:
        cfg = cfg.scaled(N=seq_len, name=cfg.name.replace(f"N{cfg.N}", f"N{seq_len}"))
    return cfg


def config_dict(cfg, **extra):
    d = {"workload": cfg.name, "B": cfg.B, "H": cfg.H, "N": cfg.N, "dk": cfg.dk, "dv": cfg.dv,
         "chunk": cfg.chunk, "io": "bf16 (fp32 state, fp32 gate logits)"}
    if cfg.io == "bf16" and cfg.dv == 256:
        # the chunkwise form is the same function for every chunk; d_v = 256 runs
        # 128-token tiles on the CTA-pair output-rows kernel
        d["tile"] = 128
    d.update(extra)
    return d


# tokens per (batch, head) unit of one step of the reference arm: a bounded
# prefix of the workload's sequences, so that a step is a fraction of a second
REFERENCE_TOKENS = 4096


def run_reference(args, world, rank):
    """Reference arm: the fp64 CPU oracle on a bounded sample of the workload."""
    import oracle
    if rank != 0:
        return 0
    cfg = config_of(args.config, args.seq_len)
    threads = oracle.default_threads()
    units = min(cfg.B * cfg.H, threads)
    tokens = min(cfg.N, REFERENCE_TOKENS)
    x = oracle_sample_inputs(cfg, units, tokens)
    vals = []
    for i in range(args.warmup + args.steps):
        v, dt, _, _ = cpu_oracle_sample(cfg, units, threads, tokens=tokens, inputs=x)
        if i >= args.warmup:
            vals.append((v, dt))
    value = statistics.mean(v for v, _ in vals)
    sample = (f"{units} of {cfg.B * cfg.H} (batch, head) units x the first {tokens} of {cfg.N} tokens per step, "
              f"fp64 recurrent form + GroupNorm/swish, {threads} threads")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "Mtok/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * statistics.mean(dt for _, dt in vals), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(cfg),
            "cpu_baseline": {"value": value, "unit": "Mtok/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "Mtok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def time_prefill(args, world, dev, stream, cfg, d):
    """Warm up, then time args.steps prefill calls of cfg on inputs `d` already
    in HBM: the whole call (events around the loop, max over ranks) and the
    fused kernel alone (events the library records around its launch).
    Returns (ms for all steps, mean fused-kernel ms, O, S, step function)."""
    import torch
    import gated_retention_sequence_b200 as gret
    io = gret.Dtype.BF16
    O = torch.empty_like(d["V"])
    S = torch.empty((cfg.B, cfg.H, cfg.dk, cfg.dv), dtype=torch.float32, device=dev)
    ws_bytes = gret.gret_prefill_workspace_size(cfg.B, cfg.H, cfg.N, cfg.dk, cfg.dv, cfg.chunk, io)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)

    def step():
        gret.prefill(d["Q"], d["K"], d["V"], d["z"], d["G"], cfg.tau, cfg.chunk, eps=cfg.eps, O=O,
                     S_final=S, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    gret.check_device_status()
    barrier(world)
    ks = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ke = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for e in ks + ke:
        e.record(stream)          # materialise the CUDA events
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    barrier(world)
    t_start.record(stream)
    for i in range(args.steps):
        gret.gret_set_profile_events(ks[i].cuda_event, ke[i].cuda_event)
        step()
    t_end.record(stream)
    gret.gret_set_profile_events(None, None)
    barrier(world)
    ms = max_over_ranks(t_start.elapsed_time(t_end), world)
    gret.check_device_status()
    kern_ms = statistics.mean(ks[i].elapsed_time(ke[i]) for i in range(args.steps))
    return ms, kern_ms, O, S, step


def prefill_summary(cfg, world, steps, ms, kern_ms, peaks):
    """Throughput, tensor and HBM fractions and the fused kernel's roofline
    object of `steps` prefill calls of cfg that took `ms` (whole calls, max
    over ranks) with the fused kernel taking `kern_ms` per launch."""
    alg_bytes, alg_flops = prefill_alg(cfg)
    step_s = ms / 1e3 / steps
    achieved = alg_bytes / (kern_ms / 1e3) / 1e9
    return {
        "value": job_throughput(world, cfg.B * cfg.N, steps, ms) / 1e6, "unit": "Mtok/s",
        "ms_per_step": ms / steps,
        "tc": {"alg_tflops": alg_flops / step_s / 1e12,
               "frac_of_bf16_peak": alg_flops / step_s / 1e12 / peaks["bf16_tflops"],
               "peak_tflops": peaks["bf16_tflops"], "peak_source": peaks["source"] + " burst"},
        "path_hbm": {"alg_gbs": alg_bytes / step_s / 1e9, "frac": alg_bytes / step_s / 1e9 / peaks["hbm_gbs"]},
        "roofline": {"kernel": {"prefill_tc_kernel": f"prefill_tc_kernel<{cfg.dv}, {cfg.chunk}> (fused chunk loop)",
                                "prefill_rows_kernel": "prefill_rows_kernel<false> (fused chunk loop, output rows)",
                                "prefill_rows_kernel_pair": "prefill_rows_kernel<true> (fused chunk loop, output rows, "
                                                            "CTA pair, 128-token tiles)"}[fused_kernel_name(cfg)],
                     "bound": "hbm",
                     "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"],
                     "traffic": profiled_traffic(prefill_profile(cfg), PREFILL_SOURCE,
                                                 ROWS_KERNEL_TEXT if fused_kernel_name(cfg).startswith("prefill_rows")
                                                 else None),
                     "alg_bytes_per_launch": alg_bytes, "launch_ms": kern_ms, "peak_source": peaks["source"]},
    }


def run_ours(args, world, rank, local):
    import torch
    import gated_retention_sequence_b200 as gret
    import gret_inputs as gi

    gret.load()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    cfg = config_of(args.config, args.seq_len)
    io = gret.Dtype.BF16
    path, segs = gret.prefill_path(cfg.B, cfg.H, cfg.N, cfg.dk, cfg.dv, cfg.chunk, io)
    host = gi.prefill_inputs(cfg)
    d = {k: v.to(dev) for k, v in host.items()}
    stream = torch.cuda.current_stream(dev)

    clocks = ClockSampler(local)
    clocks.start()
    ms, kern_ms, O, S, step = time_prefill(args, world, dev, stream, cfg, d)
    head = prefill_summary(cfg, world, args.steps, ms, kern_ms, peaks)
    launches_per_step = gret.gret_prefill_launches(cfg.B, cfg.H, cfg.N, cfg.dk, cfg.dv, cfg.chunk, io)

    # end to end through the public call: pinned host inputs in, O and S out
    pin = {k: v.pin_memory() for k, v in host.items()}
    del host
    O_h = torch.empty(O.shape, dtype=O.dtype, pin_memory=True)
    S_h = torch.empty(S.shape, dtype=S.dtype, pin_memory=True)
    e2e_steps = max(1, min(args.steps, 10))
    h2d = sum(v.numel() * v.element_size() for v in pin.values())
    d2h = O_h.numel() * O_h.element_size() + S_h.numel() * S_h.element_size()

    def e2e_step():
        for k, v in pin.items():
            d[k].copy_(v, non_blocking=True)
        step()
        O_h.copy_(O, non_blocking=True)
        S_h.copy_(S, non_blocking=True)

    e2e_value = None
    if not args.no_e2e:
        e2e_step()
        barrier(world)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e1.record(stream)
        barrier(world)
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
        e2e_value = job_throughput(world, cfg.B * cfg.N, e2e_steps, e2e_ms) / 1e6
    gret.check_device_status()
    del pin, O_h, S_h
    # the fp64 oracle's sample reads the headline inputs back from the device
    # (bounded: the first tokens of as many units as there are host threads)
    sample_x = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        threads = oracle.default_threads()
        units = min(cfg.B * cfg.H, threads)
        tokens = oracle_sample_tokens(cfg, seconds=10.0)
        sel = [divmod(u, cfg.H) for u in range(units)]
        sample_x = {k: torch.stack([d[k][b, :tokens, h].cpu() for b, h in sel], 1)[None]
                    for k in ("Q", "K", "V", "G", "z")}
    del d, O, S

    others = {}
    if not args.no_other_configs:
        for name in PREFILL_CONFIGS:
            if name == args.config:
                continue
            c = config_of(name)
            dd = {k: v.to(dev) for k, v in gi.prefill_inputs(c).items()}
            o_ms, o_kern, *_ = time_prefill(args, world, dev, stream, c, dd)
            p_, s_ = gret.prefill_path(c.B, c.H, c.N, c.dk, c.dv, c.chunk, io)
            others[name] = dict(config_dict(c, segments=s_, path=p_.name),
                                **prefill_summary(c, world, args.steps, o_ms, o_kern, peaks))
            del dd

    c2 = gi.C2
    d2 = None
    if not (args.no_varlen and args.no_seqpar and args.no_backward and args.no_projected):
        d2 = {k: v.to(dev) for k, v in gi.prefill_inputs(c2).items()}
    decode = None if args.no_decode else run_decode(args, world, dev, stream, peaks)
    varlen = None if args.no_varlen else run_varlen(args, world, dev, stream, d2, c2, peaks)
    seqpar = None
    if not args.no_seqpar:
        try:
            seqpar = run_seqpar(args, world, dev, stream, d2, c2, peaks)
        except Exception as exc:          # a failed sub-measurement must not cost the line
            seqpar = {"error": f"{type(exc).__name__}: {exc}"}
    projected = None
    if not args.no_projected:
        try:
            projected = run_projected(args, world, dev, stream, d2, c2, peaks)
        except Exception as exc:          # a failed sub-measurement must not cost the line
            projected = {"error": f"{type(exc).__name__}: {exc}"}
    backward = None
    if not args.no_backward:
        O2 = torch.empty_like(d2["V"])
        gret.prefill(d2["Q"], d2["K"], d2["V"], d2["z"], d2["G"], c2.tau, c2.chunk, eps=c2.eps, O=O2)
        backward = run_backward(args, world, dev, stream, d2, O2, c2, peaks)
    clk = clocks.stop()

    line = None
    if rank == 0:
        in_bytes = prefill_alg(cfg)[0]
        line = {
            "metric": METRIC, "value": head["value"], "unit": "Mtok/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_dict(cfg, segments=segs, path=path.name,
                                  l2=f"inputs and outputs {in_bytes / 1e6:.0f} MB > 126 MB L2 per step, no flush",
                                  parallelism=f"dp{world} (independent batches)"),
            "tc": head["tc"], "path_hbm": head["path_hbm"], "roofline": head["roofline"],
            "e2e": {"value": e2e_value, "unit": "Mtok/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk,
            "prefill_configs": others,
            "decode": decode,
            "varlen": varlen,
            "seqpar": seqpar,
            "projected": projected,
            "backward": backward,
        }
        if sample_x is not None:
            import oracle
            threads = oracle.default_threads()
            units = sample_x["Q"].shape[2]
            v, dt, passes, tokens = cpu_oracle_sample(cfg, units, threads, min_seconds=10.0,
                                                      tokens=sample_x["Q"].shape[1], inputs=sample_x)
            line["cpu_baseline"] = {"value": v, "unit": "Mtok/s", "cores": threads, "kind": "oracle",
                                    "sample": f"{passes} passes over {units} of {cfg.B * cfg.H} (batch, head) "
                                              f"units x the first {tokens} of {cfg.N} tokens of {cfg.name}, "
                                              f"fp64 recurrent form + GroupNorm/swish, {dt:.1f} s"}
        print(json.dumps(line), flush=True)
    return 0


def varlen_lengths(total: int, max_len: int, seed: int):
    """A ragged mix of sequence lengths summing to `total`: log-uniform draws in
    [1, max_len] (short prompts next to long documents), with a one-token
    sequence and lengths that are no multiple of the chunk."""
    import numpy as np
    rng = np.random.default_rng(seed)
    lengths = [1]
    while sum(lengths) < total:
        lengths.append(int(np.exp(rng.uniform(0.0, np.log(max_len)))))
    lengths[-1] -= sum(lengths) - total
    if lengths[-1] == 0:
        lengths.pop()
    return lengths


def run_varlen(args, world, dev, stream, d, cfg, peaks):
    """gret_prefill_varlen over the benchmark's own tokens (B*N of them, same
    heads and head sizes) packed as a ragged batch of sequences."""
    import numpy as np
    import torch
    import gated_retention_sequence_b200 as gret
    T = cfg.B * cfg.N
    lengths = varlen_lengths(T, cfg.N, seed=17)
    cu = torch.from_numpy(np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)).to(dev)
    flat = {k: v.view((T,) + tuple(v.shape[2:])) for k, v in d.items()}
    S_n, max_len = len(lengths), max(lengths)
    O = torch.empty_like(flat["V"])
    S = torch.empty((S_n, cfg.H, cfg.dk, cfg.dv), dtype=torch.float32, device=dev)
    io = gret.Dtype.BF16
    ws_bytes = gret.gret_prefill_varlen_workspace_size(S_n, T, max_len, cfg.H, cfg.dk, cfg.dv, cfg.chunk, io)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)

    def step():
        gret.prefill_varlen(flat["Q"], flat["K"], flat["V"], flat["z"], flat["G"], cu, max_len, cfg.tau,
                            cfg.chunk, eps=cfg.eps, O=O, S_final=S, workspace=ws, stream=stream)

    for _ in range(max(3, args.warmup)):
        step()
    gret.check_device_status()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    barrier(world)
    gret.check_device_status()
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    path, segs = gret.prefill_path(S_n, cfg.H, max_len, cfg.dk, cfg.dv, cfg.chunk, io)
    bytes_, _ = prefill_alg(cfg)
    bytes_ += (S_n - cfg.B) * cfg.H * 4 * cfg.dk * cfg.dv       # one final state per sequence
    step_s = ms / 1e3 / args.steps
    return {"workload": f"{cfg.name} tokens packed as {S_n} sequences of 1..{max_len} tokens",
            "sequences": S_n, "tokens": T, "steps": args.steps, "ms_per_step": ms / args.steps,
            "value": job_throughput(world, T, args.steps, ms) / 1e6, "unit": "Mtok/s",
            "path": path.name, "split": "long sequences cut on the device, longest segments first",
            "path_hbm": {"alg_gbs": bytes_ / step_s / 1e9, "frac": bytes_ / step_s / 1e9 / peaks["hbm_gbs"]},
            "gpu_launches": gret.gret_prefill_varlen_launches(S_n, T, max_len, cfg.H, cfg.dk, cfg.dv, cfg.chunk, io)
            * args.steps}


def run_seqpar(args, world, dev, stream, d, cfg, peaks):
    """Chunk Parallelism ("YOCO 深度技术分析", section 5.3.3) on one GPU: the
    benchmark's sequences cut into two slices of N/2 tokens.  Timed: one rank's
    computing steps for the second slice (the state pass of its slice, the fold
    of the first slice's increment -- what the all-gather delivers -- and the
    prefill of its slice resumed from the state pass's workspace and the folded
    state), and a plain prefill of the same slice from the zero state.  The all-gather itself (d_k d_v + 1 floats per
    (batch, head) and rank) is not timed."""
    import torch
    import gated_retention_sequence_b200 as gret
    half = cfg.N // 2
    io = gret.Dtype.BF16
    sl = [{k: v[:, a:a + half].contiguous() for k, v in d.items()} for a in (0, half)]
    s = sl[1]
    st_bytes = gret.gret_prefill_state_workspace_size(cfg.B, cfg.H, half, cfg.dk, cfg.dv, cfg.chunk, io)
    st_ws = torch.empty(max(st_bytes, 256), dtype=torch.uint8, device=dev)
    parts = [gret.prefill_state(p["K"], p["V"], p["z"], cfg.tau, cfg.chunk, workspace=st_ws, stream=stream)
             for p in sl]
    dS_all = torch.stack([p[0] for p in parts])
    decay_all = torch.stack([p[1] for p in parts])
    S_in = torch.empty((cfg.B, cfg.H, cfg.dk, cfg.dv), dtype=torch.float32, device=dev)
    O = torch.empty_like(s["V"])
    S_out = torch.empty_like(S_in)
    ws_bytes = gret.gret_prefill_workspace_size(cfg.B, cfg.H, half, cfg.dk, cfg.dv, cfg.chunk, io)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)

    def rank_step():
        gret.prefill_state(s["K"], s["V"], s["z"], cfg.tau, cfg.chunk, workspace=st_ws, stream=stream)
        gret.state_fold(dS_all, decay_all, 1, out=S_in, stream=stream)
        gret.prefill(s["Q"], s["K"], s["V"], s["z"], s["G"], cfg.tau, cfg.chunk, eps=cfg.eps, O=O,
                     S_final=S_out, workspace=st_ws, stream=stream, S0=S_in, resume=True)

    def plain_step():
        gret.prefill(s["Q"], s["K"], s["V"], s["z"], s["G"], cfg.tau, cfg.chunk, eps=cfg.eps, O=O,
                     S_final=S_out, workspace=ws, stream=stream)

    def timed(fn):
        for _ in range(max(3, args.warmup)):
            fn()
        gret.check_device_status()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            fn()
        e1.record(stream)
        barrier(world)
        gret.check_device_status()
        return max_over_ranks(e0.elapsed_time(e1), world) / args.steps

    rank_ms = timed(rank_step)
    plain_ms = timed(plain_step)
    return {"workload": f"{cfg.name} cut into 2 slices of {half} tokens; one rank's steps for the second slice",
            "rank_ms": rank_ms, "plain_slice_ms": plain_ms, "overhead": rank_ms / plain_ms - 1.0,
            "two_rank_mtoks_without_exchange": cfg.B * cfg.N / (rank_ms / 1e3) / 1e6, "steps": args.steps}


def backward_alg(cfg):
    """Algorithmic bytes of one backward: Q, K, V, G and dO read, dQ, dK, dV, dG
    written (io dtype), z read and dz written (fp32)."""
    e = 2 if cfg.io == "bf16" else 4
    return cfg.B * cfg.N * cfg.H * (e * (4 * cfg.dk + 5 * cfg.dv) + 8)


# chunk length of the backward (bf16 inputs); the flop count below depends on it
BACKWARD_CHUNK = 128


def backward_alg_flops(cfg, chunk=BACKWARD_CHUNK):
    """Algorithmic flops of one backward, per (token, head): six state-sized
    products (the state increment, Q S, G_c, dy S^T, V dS'^T, K dS'), 2 dk dv
    flops each, and the causal halves of the intra-chunk products (Q K^T twice,
    A V, dy V^T, A^T dy, D K, D^T Q), chunk (4 dk + 3 dv) flops together."""
    return cfg.B * cfg.N * cfg.H * (12 * cfg.dk * cfg.dv + chunk * (4 * cfg.dk + 3 * cfg.dv))


def backward_summary(cfg, steps, ms, world, peaks, launches_per_call, warmup=3):
    """The ``backward`` object of the JSON line for `steps` calls, after
    `warmup` untimed ones, that took `ms` (max over ranks) on each of `world`
    ranks."""
    bytes_ = backward_alg(cfg)
    flops = backward_alg_flops(cfg)
    step_s = ms / 1e3 / steps
    tflops = flops / step_s / 1e12
    peak = peaks["bf16_tflops"]
    return {"workload": cfg.name, "steps": steps, "warmup": warmup, "ms_per_step": ms / steps,
            "value": job_throughput(world, cfg.B * cfg.N, steps, ms) / 1e6, "unit": "Mtok/s",
            "kernels": "bwd_inc_tc, bwd_scan_fwd, bwd_dyq_tc, bwd_scan_rev, bwd_kv_tc, bwd_dz "
                       "(tcgen05 kind::f16, states and dy as bf16 pairs, fp32 accumulation in tensor memory)",
            "roofline": {"kernel": "whole backward (6 launches)", "bound": "tensor", "achieved": tflops,
                         "peak": peak, "unit": "TFLOP/s", "frac": tflops / peak, "traffic": None,
                         "alg_flops_per_call": flops,
                         "peak_source": peaks["source"] + " bf16 burst"},
            "path_hbm": {"alg_bytes": bytes_, "alg_gbs": bytes_ / step_s / 1e9,
                         "frac": bytes_ / step_s / 1e9 / peaks["hbm_gbs"]},
            "gpu_launches": launches_per_call * steps}


def run_backward(args, world, dev, stream, d, O, cfg, peaks):
    """gret_prefill_backward on the benchmark workload, or on its first
    --backward-batch sequences.  The upstream gradient dO is the
    forward's own output O (any tensor of O's shape and dtype serves; the cost
    does not depend on its values)."""
    import torch
    import gated_retention_sequence_b200 as gret
    if args.backward_batch and args.backward_batch < cfg.B:
        nb = args.backward_batch
        cfg = cfg.scaled(B=nb, name=f"{cfg.name} (first {nb} sequences)")
        d = {k: v[:nb] for k, v in d.items()}
        O = O[:nb]
    steps = max(1, min(args.steps, 5))
    warmup = max(3, min(args.warmup, 5))
    dO = O.clone()
    io = gret.Dtype.BF16
    ws_bytes = gret.gret_prefill_backward_workspace_size(cfg.B, cfg.H, cfg.N, cfg.dk, cfg.dv, io)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)

    def step():
        return gret.prefill_backward(d["Q"], d["K"], d["V"], d["z"], d["G"], dO, cfg.tau, eps=cfg.eps,
                                     workspace=ws, stream=stream)

    for _ in range(warmup):
        step()
    gret.check_device_status()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    barrier(world)
    gret.check_device_status()
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    return backward_summary(cfg, steps, ms, world, peaks,
                            gret.gret_prefill_backward_launches(cfg.B, cfg.H, cfg.N, cfg.dk, cfg.dv, io), warmup)


def projection_alg(cfg, d_model):
    """Algorithmic bytes of the fused gate prologue of a projected prefill: X
    read once (bf16), W_gamma read (fp32), and the decay sums and P-block
    factors written (2 fp32 per token and head); flops 2 d_model per token and
    head (z = X W_gamma; the two bf16 halves of W are an implementation detail)."""
    units = cfg.B * cfg.H
    npad = -(-cfg.N // cfg.chunk) * cfg.chunk
    bytes_ = cfg.B * cfg.N * d_model * 2 + d_model * cfg.H * 4 + 2 * units * npad * 4
    return bytes_, 2 * cfg.B * cfg.N * cfg.H * d_model


def run_projected(args, world, dev, stream, d, cfg, peaks):
    """gret_prefill_projected on the c2 tokens with X of d_model = H d_k
    channels (67 MB of bf16 rows): the gate logits come from z = X W_gamma
    inside the gate prologue.  Timed: the whole call, and the fused
    projection-and-scan kernel alone (events around its launch)."""
    import torch
    import gated_retention_sequence_b200 as gret
    import gret_inputs as gi
    d_model = cfg.H * cfg.dk
    X = gi.random_unit(cfg.seed, 41, (cfg.B, cfg.N, d_model), 0.0, 1.0 / d_model, "bf16").to(dev)
    W = gi.random_unit(cfg.seed, 42, (d_model, cfg.H), 3.0, 1.5, "f32").to(dev)
    O = torch.empty_like(d["V"])
    S = torch.empty((cfg.B, cfg.H, cfg.dk, cfg.dv), dtype=torch.float32, device=dev)
    io = gret.Dtype.BF16
    ws_bytes = gret.gret_prefill_projected_workspace_size(cfg.B, cfg.H, cfg.N, cfg.dk, cfg.dv, cfg.chunk, d_model, io)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)

    def step():
        gret.prefill_projected(d["Q"], d["K"], d["V"], X, W, d["G"], cfg.tau, cfg.chunk, eps=cfg.eps, O=O,
                               S_final=S, workspace=ws, stream=stream)

    for _ in range(max(3, args.warmup)):
        step()
    gret.check_device_status()
    barrier(world)
    ks = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ke = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for e in ks + ke:
        e.record(stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    e0.record(stream)
    for i in range(args.steps):
        gret.gret_set_gate_profile_events(ks[i].cuda_event, ke[i].cuda_event)
        step()
    e1.record(stream)
    gret.gret_set_gate_profile_events(None, None)
    barrier(world)
    gret.check_device_status()
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    kern_ms = statistics.mean(ks[i].elapsed_time(ke[i]) for i in range(args.steps))
    bytes_, flops = projection_alg(cfg, d_model)
    achieved = bytes_ / (kern_ms / 1e3) / 1e9
    return {"workload": f"{cfg.name} with gate logits z = X W_gamma, X [{cfg.B}, {cfg.N}, {d_model}] bf16",
            "steps": args.steps, "ms_per_step": ms / args.steps,
            "value": job_throughput(world, cfg.B * cfg.N, args.steps, ms) / 1e6, "unit": "Mtok/s",
            "roofline": {"kernel": "gate_project_scan_kernel (z = X W_gamma fused with the decay scan)",
                         "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"], "traffic": None, "alg_bytes_per_launch": bytes_,
                         "alg_flops_per_launch": flops, "launch_ms": kern_ms, "peak_source": peaks["source"]},
            "gpu_launches": (1 + gret.gret_prefill_launches(cfg.B, cfg.H, cfg.N, cfg.dk, cfg.dv, cfg.chunk, io))
            * args.steps}


def run_decode(args, world, dev, stream, peaks):
    """Recurrent decode: 64 consecutive single-token steps over 256 x 16 states."""
    import torch
    import gated_retention_sequence_b200 as gret
    import gret_inputs as gi
    cfg = gi.C4
    p = cfg.prior_prefill()
    prior = {k: v.to(dev) for k, v in gi.prefill_inputs(p).items()}
    _, S = gret.prefill(prior["Q"], prior["K"], prior["V"], prior["z"], prior["G"], p.tau, p.chunk)
    del prior
    st = {k: v.to(dev) for k, v in gi.decode_step_inputs(cfg).items()}
    o = torch.empty_like(st["v"][0])
    T = cfg.steps
    for t in range(min(3, T)):       # warm-up steps on a copy of the state
        S_w = S.clone()
        gret.decode_step(st["q"][t], st["k"][t], st["v"][t], st["z"][t], st["g"][t], S_w, cfg.tau, o=o)
    del S_w
    barrier(world)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(T + 1)]
    ev[0].record(stream)
    for t in range(T):
        gret.decode_step(st["q"][t], st["k"][t], st["v"][t], st["z"][t], st["g"][t], S, cfg.tau, o=o)
        ev[t + 1].record(stream)
    barrier(world)
    gret.check_device_status()
    per = [ev[t].elapsed_time(ev[t + 1]) for t in range(T)]
    mean_ms = max_over_ranks(statistics.mean(per), world)
    med_ms = statistics.median(per)
    bytes_ = decode_alg(cfg)
    gbs = bytes_ / (mean_ms / 1e3) / 1e9
    return {"workload": cfg.name, "steps": T, "ms_per_step_mean": mean_ms, "ms_per_step_median": med_ms,
            "state_gbs": world * bytes_ / (mean_ms / 1e3) / 1e9, "unit": "GB/s",
            "roofline": {"kernel": "decode_step_kernel", "bound": "hbm", "achieved": gbs,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                         "traffic": profiled_traffic(DECODE_PROFILE, "gated_retention_sequence_b200/csrc/gret_decode.cu"),
                         "alg_bytes_per_launch": bytes_,
                         "peak_source": peaks["source"]},
            "gpu_launches": T}


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", choices=list(PREFILL_CONFIGS), default="c3",
                    help="headline prefill workload (c3: B1 H32 N65536 d 128 chunk 128)")
    ap.add_argument("--no-other-configs", action="store_true",
                    help="skip the other prefill workloads' sub-measurements")
    ap.add_argument("--seq-len", type=int, default=0,
                    help="profiling aid: run the headline workload with this many tokens per sequence "
                         "(the JSON line then names the reduced workload)")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-varlen", action="store_true")
    ap.add_argument("--no-seqpar", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--no-projected", action="store_true")
    ap.add_argument("--backward-batch", type=int, default=0,
                    help="run the backward sub-measurement on this many of the batch's sequences")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        return run_reference(args, world, rank)
    world, rank, local = dist_setup()
    try:
        return run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())

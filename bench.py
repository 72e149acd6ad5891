#!/usr/bin/env python
"""Benchmark of the draft lm_head sweep + argmax (µs per draft, HBM GB/s, roofline).

One step = one draft's lm_head sweep fused with argmax (mtp_lm_head_argmax) over the
154,880 x 4,096 BF16 draft head at M = 1 (the table size of the GLM draft head on the
metrale_model_arch/glm5next_mtp_head/init.rs page). The table is 1.27 GB, ten times
the 126 MB L2, so every step streams it from HBM; no flush is needed. FP8 and NVFP4
sweeps at M = 1 are measured the same way and reported under "rows".

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--full]

N > 1 (under torchrun): every rank sweeps its own replica (the sweep has no
exchange step on one table), timed on the device, max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "lm_head+argmax µs/draft and HBM GB/s (fraction of B200 peak) at M=1"
FALLBACK_HBM_GBS = 6650.0

# DRAM traffic per launch from ncu (dram__bytes_read.sum + dram__bytes_write.sum) and
# the sha256 of sweep.cu when it was captured; reported as null once the source changed.
# bf16_M1: a full-size capture (one-pass metrics) of the headline sweep, the mean of two
# launches: 1,268,870,144 + 128,256 and 1,268,873,728 + 133,632 B.
NCU_TRAFFIC = {"bf16_M1": (1269123712, "5ffd0495da62c93b")}


def sweep_source_hash() -> str:
    p = os.path.join(ROOT, "mtp_speculative_draft_lm_b200", "csrc", "sweep.cu")
    with open(p, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


FALLBACK_TFLOPS_SUSTAINED = 1400.0
FALLBACK_TFLOPS_BURST = 1590.0
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, nominal (context beside the measured copy peak)


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def measured_tflops(key="bf16_tflops"):
    """Dense bf16 peak: the burst figure (a call of a few ms timed on its own) unless asked
    for the sustained one."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d.get(key, d.get("bf16_tflops"))), f"measured {key}"
    return (FALLBACK_TFLOPS_BURST if key == "bf16_tflops" else FALLBACK_TFLOPS_SUSTAINED), \
        f"fallback {key}"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, torch_dev):
        import torch

        self.proc = None
        self.sel = []
        try:
            pr = torch.cuda.get_device_properties(torch_dev)
            self.sel = ["-i", f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"]
        except Exception:
            self.sel = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", *self.sel, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(args):
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
    else:
        torch.cuda.set_device(local)
        if getattr(args, "sharded", False):  # a one-rank group, so the exchange runs as-is
            import torch.distributed as dist

            dist.init_process_group("nccl", store=dist.HashStore(), rank=0, world_size=1,
                                    device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch
    import torch.distributed as dist

    t = torch.tensor([v], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def build_table(fmt: str, dev, rows: int = 0):
    """Seeded synthetic table for one format (quantized on the device)."""
    import torch

    from mtp_speculative_draft_lm_b200 import api, synth

    cfg = dict({"bf16": synth.BF16_HEAD, "fp8": synth.FP8_HEAD, "nvfp4": synth.NVFP4_HEAD}[fmt])
    if rows:
        cfg["N"] = rows
    # the mask is drawn after the table and the inputs, so they do not depend on it
    d = synth.head_table(cfg["seed"], cfg["N"], cfg["K"], max(cfg["Ms"]),
                         mask_keep=cfg.get("mask_keep", 0.1))
    w = d["W"].to(dev)
    qinfo = None
    if fmt == "bf16":
        table = api.bf16_table(w)
    else:
        from mtp_speculative_draft_lm_b200 import _lib as L

        table = api.quantize_fp8(w) if fmt == "fp8" else api.quantize_nvfp4(w)
        n, k = w.shape
        if fmt == "fp8":
            def quant():
                L.mtp_quantize_fp8(w, n, k, table.data, table.row_scale)
        else:
            ws = torch.zeros((L.mtp_quantize_nvfp4_ws_bytes(n, k),), dtype=torch.uint8, device=dev)

            def quant():
                L.mtp_quantize_nvfp4(w, n, k, table.data, table.block_scale, table.global_scale,
                                     ws, ws.numel())
        quant()
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 5
        s.record()
        for _ in range(reps):
            quant()
        e.record()
        torch.cuda.synchronize()
        ms = s.elapsed_time(e) / reps
        rd = w.numel() * 2
        wr = table.nbytes()
        # NVFP4 reads the table twice (global absmax pass, then the encode pass)
        qinfo = {"ms": ms, "GB/s": (rd * (2 if fmt == "nvfp4" else 1) + wr) / ms / 1e6,
                 "bytes": rd * (2 if fmt == "nvfp4" else 1) + wr}
        del w
    return cfg, d, table, qinfo


def time_sweep(head, x, steps, warmup, world, stream, mask=None, mask_words=0):
    """Device time of `steps` back-to-back sweeps between two events (nothing else on
    the stream in between: the mean launch duration), then a shorter pass with an event
    pair around each launch (the per-launch median and p10/p90; those events add a gap
    between launches, which also ends the programmatic overlap of one launch's tail
    with the next one's start)."""
    import numpy as np
    import torch

    M = x.shape[0]
    dev = x.device
    idx = torch.empty((M,), dtype=torch.int32, device=dev)
    val = torch.empty((M,), dtype=torch.float32, device=dev)
    kw = dict(mask=mask, mask_words=mask_words, mask_stride_words=mask_words)
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            head(x, idx, val, stream=stream, **kw)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record(stream)
        for _ in range(steps):
            head(x, idx, val, stream=stream, **kw)
        t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    total_ms = t0.elapsed_time(t1)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(min(steps, 200))]
    with torch.cuda.stream(stream):
        for s, e in ev:
            s.record(stream)
            head(x, idx, val, stream=stream, **kw)
            e.record(stream)
    torch.cuda.synchronize()
    per = np.array([s.elapsed_time(e) for s, e in ev])
    return {"mean_ms": total_ms / steps, "median_ms": float(np.median(per)),
            "p10_ms": float(np.percentile(per, 10)), "p90_ms": float(np.percentile(per, 90)),
            "idx": idx.cpu().numpy()}


def time_e2e(head, x_host, steps, warmup, world, stream):
    """The same metric end to end through mtp_lm_head_argmax_host, one draft at a time as
    the pages run it: each step the call reads its input from pinned host memory and
    writes the index and value to pinned host memory, the host waits for the stream and
    reads the token before the next step. Timed with events on the stream around the K
    steps (the device is idle while the host waits, so this is the per-draft latency a
    caller sees). Also the pipelined figure: K calls enqueued back to back, no host wait."""
    import torch

    M, K = x_host.shape
    out_h = torch.empty((2 * M,), dtype=torch.int32).pin_memory()

    def step():
        head.argmax_host(x_host, out_h, stream=stream)

    for _ in range(warmup):
        step()
        stream.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    toks = 0
    with torch.cuda.stream(stream):
        t0.record(stream)
        for _ in range(steps):
            step()
            stream.synchronize()
            toks += int(out_h[0])  # the host reads the draft token
        t1.record(stream)
    torch.cuda.synchronize()
    sync_ms = t0.elapsed_time(t1) / steps
    with torch.cuda.stream(stream):
        t0.record(stream)
        for _ in range(steps):
            step()
        t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    pipe_ms = t0.elapsed_time(t1) / steps
    return sync_ms, pipe_ms, M * K * 2, M * 8, out_h[:M].numpy().copy()


def bench_tiny_draft(dev, steps, warmup):
    """The tiny draft step (hidden 256, vocab 4096), M = 1: everything is L2-resident, so
    this is latency (reported warm). The fused step (mtp_draft_step, one cluster launch)
    is the headline; the two-launch path (mtp_combine + mtp_lm_head_argmax) beside it.
    Each is timed eager (one call after another) and as a 16-draft device-side chain
    (the argmax index and y of one step feed the next) replayed from a CUDA graph."""
    import torch

    from mtp_speculative_draft_lm_b200 import api, synth

    d = synth.tiny_draft(M=1)
    dd = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    fc = api.bf16_table(dd["fc"])
    head = api.LmHead(api.bf16_table(dd["lm_head"]))
    chain = 16
    ys = [torch.empty((1, d["h"]), dtype=torch.bfloat16, device=dev) for _ in range(chain)]
    ids = [torch.empty((1,), dtype=torch.int32, device=dev) for _ in range(chain)]
    vals = [torch.empty((1,), dtype=torch.float32, device=dev) for _ in range(chain)]

    def fused(tok, hid, j):
        api.draft_step(dd["embed"], tok, hid, dd["w_norm_embed"], dd["w_norm_hidden"], d["eps"],
                       dd["fc"], dd["lm_head"],
                       out_y=ys[j], out_idx=ids[j], out_val=vals[j])

    def two_launch(tok, hid, j):
        api.combine(dd["embed"], tok, hid, dd["w_norm_embed"], dd["w_norm_hidden"], d["eps"], fc,
                    out=ys[j])
        head(ys[j], ids[j])

    def timed(step_fn):
        for _ in range(warmup):
            step_fn(dd["tokens"], dd["hidden"], 0)
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(steps):
            step_fn(dd["tokens"], dd["hidden"], 0)
        e.record()
        torch.cuda.synchronize()
        eager_us = s.elapsed_time(e) / steps * 1e3

        def run_chain():
            tok, hid = dd["tokens"], dd["hidden"]
            for j in range(chain):
                step_fn(tok, hid, j)
                tok, hid = ids[j], ys[j]

        cs = torch.cuda.Stream(device=dev)
        cs.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(cs):
            run_chain()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cs):
                run_chain()
        torch.cuda.synchronize()
        reps = max(10, steps // chain)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        s.record()
        for _ in range(reps):
            g.replay()
        e.record()
        torch.cuda.synchronize()
        graph_us = s.elapsed_time(e) / (reps * chain) * 1e3
        del g
        return eager_us, graph_us

    f_eager, f_graph = timed(fused)
    t_eager, t_graph = timed(two_launch)
    return {"us_per_draft": f_eager, "chain_graph_us_per_draft": f_graph, "launches_per_draft": 1,
            "two_launch_us_per_draft": t_eager, "two_launch_chain_graph_us_per_draft": t_graph,
            "chain_length": chain,
            "note": "hidden 256, vocab 4096, M=1, warm (L2-resident); fused: mtp_draft_step, one "
                    "cluster launch; two-launch: mtp_combine + mtp_lm_head_argmax; chain: 16 "
                    "drafts fed device-side (argmax index and y -> next step) replayed from a "
                    "CUDA graph"}


def bench_prefill(dev, reps, tflops_peak, peak_src, rows=0):
    """Drafter-context prefill: 32,768 prompt rows, hidden 5,120, chunks of 2,048."""
    import torch

    from mtp_speculative_draft_lm_b200 import api, synth

    d = synth.prefill_inputs(R=rows, vocab=4096) if rows else synth.prefill_inputs()
    dd = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    kc = torch.zeros((d["num_blocks"], d["block_size"], d["nkv"], d["hd"]), dtype=torch.uint8,
                     device=dev)
    vc = torch.zeros_like(kc)
    import numpy as np

    ws = api.prefill_kv(dd, kc, vc, chunk_rows=synth.PREFILL["chunk"])
    for _ in range(3):
        api.prefill_kv(dd, kc, vc, chunk_rows=synth.PREFILL["chunk"], ws=ws)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(reps)]
    clocks = ClockSampler(dev)
    clocks.start()
    for s, e in ev:  # one call per event pair (each call is ~3 ms: the pair's gap is noise)
        s.record()
        api.prefill_kv(dd, kc, vc, chunk_rows=synth.PREFILL["chunk"], ws=ws)
        e.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    per = np.array([s.elapsed_time(e) for s, e in ev])
    ms = float(np.median(per))
    R, h, kvd = d["R"], d["h"], d["nkv"] * d["hd"]
    flops = 2.0 * R * (2 * h) * h + 2.0 * R * h * (2 * kvd)
    tf = flops / (ms * 1e-3) / 1e12
    sus, _ = measured_tflops("bf16_tflops_sustained")
    return {"ms": ms, "statistic": f"median of {reps} calls", "ms_min_max": [float(per.min()), float(per.max())],
            "TFLOP/s": tf, "frac_of_peak": tf / tflops_peak,
            "peak_source": peak_src, "frac_of_sustained_peak": tf / sus, "flops": flops,
            "rows": R, "hidden": h, "chunk": synth.PREFILL["chunk"], "clocks": clk}


def bench_attn(dev, steps, warmup, seq=32768, nq=64, nkv=8, hd=128):
    """Single-token decode attention over a paged E4M3 cache of seq rows (the prefill
    workload's 8 KV heads x 128; 64 query heads, a reading: the pages give no head count):
    every cached K and V byte is read once, so HBM GB/s is the figure."""
    import torch

    from mtp_speculative_draft_lm_b200 import api, synth

    g = synth._gen(1006)
    nb = seq // 16 + 1
    kc = torch.randint(0, 0x7E, (nb, 16, nkv, hd), generator=g, dtype=torch.uint8).to(dev)
    vc = torch.randint(0, 0x7E, (nb, 16, nkv, hd), generator=g, dtype=torch.uint8).to(dev)
    bt = torch.randperm(nb, generator=g).to(torch.int32).to(dev)
    q = synth.normal_bf16(g, (nq, hd), 1.0).to(dev)
    out, ws = api.paged_decode_attn(q, nkv, kc, vc, bt, seq)
    for _ in range(warmup):
        api.paged_decode_attn(q, nkv, kc, vc, bt, seq, out=out, ws=ws)
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        api.paged_decode_attn(q, nkv, kc, vc, bt, seq, out=out, ws=ws)
    e.record()
    torch.cuda.synchronize()
    us = s.elapsed_time(e) / steps * 1e3
    nbytes = 2 * seq * nkv * hd + 2 * 2 * nq * hd + bt.numel() * 4
    return {"us_per_draft_position": us, "GB/s": nbytes / (us * 1e-6) / 1e9,
            "bytes_per_step": nbytes, "seq_len": seq, "nq": nq, "nkv": nkv, "hd": hd,
            "note": "K and V rows of every cached position read once; launches: 2"}


def _median_runs(fn, budget_s, max_runs=3):
    """Median wall time of up to max_runs calls of fn, stopping once budget_s is spent."""
    times = []
    t_start = time.perf_counter()
    while len(times) < max_runs:
        t = time.perf_counter()
        out = fn()
        times.append(time.perf_counter() - t)
        if time.perf_counter() - t_start > budget_s:
            break
    return statistics.median(times), len(times), out


def cpu_baseline_sweep(fmt, d, cfg, budget_s=12.0):
    """The oracle, as it stands, on the same table at M = 1 (all of its rows; quantized by
    the oracle's own quantizer, not timed). Median of up to 3 runs."""
    import oracle
    from mtp_speculative_draft_lm_b200 import synth

    W = synth.as_u16(d["W"])
    x = synth.as_u16(d["x"][:1])
    K = cfg["K"]
    kw = {}
    if fmt == "bf16":
        data, nbytes = W, W.nbytes
    elif fmt == "fp8":
        data, rs = oracle.quantize_fp8(W)
        kw = dict(row_scale=rs)
        nbytes = data.nbytes + rs.nbytes
    else:
        data, bs, g = oracle.quantize_nvfp4(W)
        kw = dict(block_scale=bs, global_scale=g)
        nbytes = data.nbytes + bs.nbytes + 4
    nbytes += x.nbytes + 8
    fid = {"bf16": 0, "fp8": 1, "nvfp4": 2}[fmt]
    med, runs, out = _median_runs(
        lambda: oracle.lm_head_argmax(fid, data, K, x, want_logits=False, **kw), budget_s)
    assert out[1][0] == d["top"][0]
    return {"value": nbytes / med / 1e9, "unit": "GB/s", "cores": oracle.num_threads(),
            "kind": "oracle", "ms_per_draft": med * 1e3,
            "sample": f"full {cfg['N']}x{K} {fmt} table, M=1, median of {runs} runs "
                      f"(fp64 accumulation, OpenMP over rows)"}


def cpu_baseline_tiny(budget_s=5.0):
    """The oracle's tiny draft step (combine + lm_head sweep + argmax), M = 1."""
    import oracle
    from mtp_speculative_draft_lm_b200 import synth

    d = synth.tiny_draft(M=1)
    u = synth.as_u16

    def run():
        y, _, _ = oracle.combine(u(d["embed"]), d["tokens"].numpy(), u(d["hidden"]),
                                 u(d["w_norm_embed"]), u(d["w_norm_hidden"]), d["eps"], u(d["fc"]))
        return oracle.lm_head_argmax(0, u(d["lm_head"]), d["h"], y, want_logits=False)

    med, runs, _ = _median_runs(run, budget_s, max_runs=20)
    return {"value": med * 1e6, "unit": "us/draft", "cores": oracle.num_threads(),
            "kind": "oracle", "sample": f"hidden 256, vocab 4096, M=1, median of {runs} runs"}


def cpu_baseline_prefill(rows=256):
    """The oracle's drafter-context prefill on `rows` prompt rows spread evenly over the
    whole prompt (every chunk), extrapolated to all rows (labelled as such)."""
    import numpy as np

    import oracle
    from mtp_speculative_draft_lm_b200 import synth

    d = synth.prefill_inputs()
    u = synth.as_u16
    R = d["R"]
    pick = np.linspace(0, R - 1, rows).astype(np.int64)
    t = time.perf_counter()
    oracle.prefill_rows(u(d["embed"]), d["tokens"].numpy(), u(d["hidden"]), u(d["w_norm_embed"]),
                        u(d["w_norm_hidden"]), d["eps"], u(d["fc"]), u(d["wk"]), u(d["wv"]),
                        d["nkv"], d["hd"], d["rope_base"], d["rope_pos"].numpy(), 0,
                        d["block_table"].numpy(), d["block_size"], d["num_blocks"], 1.0, 1.0,
                        pick)
    dt = time.perf_counter() - t
    h, kvd = d["h"], d["nkv"] * d["hd"]
    flops_row = 2.0 * (2 * h) * h + 2.0 * h * (2 * kvd)
    return {"value": flops_row * rows / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle", "ms_extrapolated": dt / rows * R * 1e3,
            "sample": f"{rows} of {R} prompt rows spread over every chunk, {dt:.2f} s; the "
                      f"32,768-row time is extrapolated per row"}


def run_reference(args):
    """--impl reference: the CPU oracle on bounded row samples of the same workload."""
    import numpy as np

    import oracle
    from mtp_speculative_draft_lm_b200 import synth

    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    cfg = synth.BF16_HEAD
    d = synth.head_table(cfg["seed"], cfg["N"], cfg["K"], 1)
    W = synth.as_u16(d["W"])
    x = synth.as_u16(d["x"][:1])
    K = cfg["K"]
    # size one step's row sample so that warmup + steps stay within about a minute
    rows = 1024
    t = time.perf_counter()
    oracle.lm_head_argmax(0, W[:rows], K, x, want_logits=False)
    per_row = (time.perf_counter() - t) / rows
    total = args.steps + args.warmup
    rows = int(max(16, min(cfg["N"], 60.0 / total / max(per_row, 1e-9))))
    starts = [(i * rows) % (cfg["N"] - rows + 1) for i in range(total)]
    for i in range(args.warmup):
        oracle.lm_head_argmax(0, W[starts[i]: starts[i] + rows], K, x, want_logits=False)
    t0 = time.perf_counter()
    for i in range(args.warmup, total):
        oracle.lm_head_argmax(0, W[starts[i]: starts[i] + rows], K, x, want_logits=False)
    dt = (time.perf_counter() - t0) / args.steps
    nbytes = rows * K * 2 + x.nbytes + 8
    value = nbytes / dt / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"bf16 lm_head sweep + argmax, table [{cfg['N']}, {K}], M=1",
                   "sample_rows_per_step": rows},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": f"{rows} of {cfg['N']} table rows per step (cycling), M=1"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_sharded(args, world, rank, dev, peak, peak_src):
    """The BF16 sweep split by vocab over the ranks: every step each rank sweeps its rows,
    the 16-byte partials are all-gathered (NCCL) and merged on every rank. One step covers
    the whole table once, so value = table bytes / max-over-ranks time (strong scaling)."""
    import numpy as np
    import torch

    from mtp_speculative_draft_lm_b200 import api

    cfg, d, table, _ = build_table("bf16", dev)
    off, cnt = api.shard_range(cfg["N"], world, rank)
    head = api.ShardedLmHead(api.table_rows(table, off, off + cnt) if cnt else None, off)
    x = d["x"][:1].to(dev)
    for _ in range(args.warmup):
        out = head.argmax(x)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    clocks = ClockSampler(dev)
    clocks.start()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(args.steps):
        out = head.argmax(x)
    e.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier(world)
    ms = max_over_ranks(s.elapsed_time(e) / args.steps, world)
    ok = int(out[0].item()) == int(d["top"][0])
    nbytes = cfg["N"] * cfg["K"] * 2 + cfg["K"] * 2 + 8
    if rank == 0:
        print(json.dumps({
            "metric": METRIC, "value": nbytes / (ms * 1e-3) / 1e9, "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "us_per_draft": ms * 1e3, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic: seeded N(0, 0.02) bf16 table with planted maximum rows",
            "config": {"workload": f"bf16 lm_head sweep + argmax, table [{cfg['N']}, {cfg['K']}], "
                                   f"M=1, split by vocab", "table_bytes": cfg["N"] * cfg["K"] * 2,
                       "M": 1, "l2": "table (1.27 GB) larger than L2 (126 MB): no flush",
                       "parallelism": f"vocab-sharded x{world} (one all-gather of 16 B per rank "
                                      f"per step)"},
            "roofline": {"bound": "hbm", "achieved": nbytes / world / (ms * 1e-3) / 1e9,
                         "peak": peak, "unit": "GB/s",
                         "frac": nbytes / world / (ms * 1e-3) / 1e9 / peak, "traffic": None,
                         "peak_source": f"{peak_src} hbm_gbs (copy), per GPU"},
            "gpu_launches": 2 * args.steps, "clocks": clk, "argmax_ok": ok}), flush=True)
    import torch.distributed as dist

    dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--full", action="store_true", help="also M>1 and masked rows")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--formats", default="bf16,fp8,nvfp4")
    ap.add_argument("--rows", type=int, default=0,
                    help="sweep a smaller table of this many rows (profiling cases)")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the tiny-draft and prefill rows")
    ap.add_argument("--only", default="",
                    help="profiling: run only 'prefill', 'tiny', 'attn' or 'masked'")
    ap.add_argument("--ms", default="",
                    help="profiling: time only these input counts (comma list, e.g. 16,32), "
                         "seeded N(0, 1) inputs")
    ap.add_argument("--sharded", action="store_true",
                    help="N > 1: split the BF16 table by vocab over the ranks (strong scaling) "
                         "instead of one replica per rank")
    ap.add_argument("--prefill-rows", type=int, default=0,
                    help="profiling: prefill prompt rows (default: the 32,768-row workload)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.impl == "reference":
        return run_reference(args)

    import numpy as np
    import torch

    from mtp_speculative_draft_lm_b200 import api

    world, rank, local = dist_setup(args)
    dev = torch.device("cuda", local)
    stream = torch.cuda.Stream(device=dev)
    peak, peak_src = measured_peaks()
    if args.only:
        tpk, tsrc = measured_tflops()
        if args.only == "prefill":
            out = bench_prefill(dev, 10, tpk, tsrc, args.prefill_rows)
        elif args.only == "attn":
            out = bench_attn(dev, args.steps, args.warmup)
        elif args.only == "masked":  # profiling: the masked M = 1 sweep alone
            out = {}
            for fmt in args.formats.split(","):
                cfg, d, table, _ = build_table(fmt, dev, args.rows)
                head = api.LmHead(table)
                words = d["mask"].shape[1]
                m = torch.from_numpy(d["mask"][:1].reshape(-1)).to(dev)
                tm = time_sweep(head, d["x"][:1].to(dev), args.steps, args.warmup, 1, stream,
                                mask=m, mask_words=words)
                out[f"{fmt}_M1_masked"] = {"us_per_draft": tm["mean_ms"] * 1e3,
                                           "argmax_ok": int(tm["idx"][0]) == int(d["second"][0])}
                del head, table, d
                torch.cuda.empty_cache()
        else:
            out = bench_tiny_draft(dev, args.steps, args.warmup)
        print(json.dumps({"only": args.only, **out}), flush=True)
        return 0
    if args.sharded:
        return run_sharded(args, world, rank, dev, peak, peak_src)
    rows = {}
    main_line = None
    cpu_base = None
    cpu_rows = rank == 0 and world == 1 and not args.no_cpu and not args.rows and not args.ms
    for fmt in args.formats.split(","):
        cfg, d, table, qinfo = build_table(fmt, dev, args.rows)
        head = api.LmHead(table)
        Ms = () if args.ms else (cfg["Ms"] if args.full else (1,))
        for M in Ms:
            x = d["x"][:M].to(dev)
            clocks = ClockSampler(dev)
            clocks.start()
            t = time_sweep(head, x, args.steps, args.warmup, world, stream)
            clk = clocks.stop()
            ok = bool(np.array_equal(t["idx"], d["top"][:M]))
            ms_max = max_over_ranks(t["mean_ms"], world)
            nbytes = head.bytes_per_call(M)
            e2e_ms, pipe_ms, h2d, d2h, e2e_idx = time_e2e(
                head, d["x"][:M].contiguous().pin_memory(), max(100, min(2000, args.steps // 5)),
                args.warmup, world, stream)
            e2e_max = max_over_ranks(e2e_ms, world)
            rec = {
                "us_per_draft": ms_max * 1e3,
                "statistic": "mean of back-to-back launches between two events",
                "median_launch_us": t["median_ms"] * 1e3,
                "p10_p90_launch_us": [t["p10_ms"] * 1e3, t["p90_ms"] * 1e3],
                "GB/s": nbytes * world / (ms_max * 1e-3) / 1e9,
                "frac_of_peak": nbytes / (ms_max * 1e-3) / 1e9 / peak,
                "frac_of_nominal_8TBps": nbytes / (ms_max * 1e-3) / 1e9 / NOMINAL_HBM_GBS,
                "bytes_per_step": nbytes,
                "e2e_us": e2e_max * 1e3,
                "e2e_pipelined_us": pipe_ms * 1e3,
                "argmax_ok": ok and bool(np.array_equal(e2e_idx, d["top"][:M])),
                "clocks": clk,
            }
            if qinfo and M == Ms[0]:
                rec["quantizer"] = qinfo
            rows[f"{fmt}_M{M}"] = rec
            if fmt == "bf16" and M == 1:
                main_line = (rec, nbytes, ms_max, e2e_max, pipe_ms, h2d, d2h, clk, cfg)
        wide = [int(v) for v in args.ms.split(",")] if args.ms else ((16, 32) if args.full else ())
        for Mw in wide:  # wide batches: 16 and 32 inputs (seeded N(0, 1) rows; timing only)
            gen = torch.Generator().manual_seed(Mw)
            xw = torch.randn((Mw, cfg["K"]), generator=gen).to(torch.bfloat16).to(dev)
            tw = time_sweep(head, xw, max(1, args.steps // 4), args.warmup, world, stream)
            us = tw["mean_ms"] * 1e3
            rows.setdefault(f"{fmt}_M{Mw}", {"us_per_draft": us,
                                             "median_launch_us": tw["median_ms"] * 1e3,
                                             "GB/s": head.bytes_per_call(Mw) / (us * 1e-6) / 1e9,
                                             "frac_of_peak": head.bytes_per_call(Mw) / (us * 1e-6) / 1e9 / peak,
                                             "note": "timing only (random inputs)"})
        if args.ms:  # profiling run: only the requested input counts
            del head, table, d
            torch.cuda.empty_cache()
            continue
        # the same sweep with the top-1 log-probability (mtp_lm_head_argmax_lp), M = 1
        x = d["x"][:1].to(dev)
        idx = torch.empty((1,), dtype=torch.int32, device=dev)
        lp = torch.empty((1,), dtype=torch.float32, device=dev)
        for _ in range(args.warmup):
            head(x, idx, None, stream=stream, out_logprob=lp)
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            s.record(stream)
            for _ in range(args.steps):
                head(x, idx, None, stream=stream, out_logprob=lp)
            e.record(stream)
        torch.cuda.synchronize()
        us = s.elapsed_time(e) / args.steps * 1e3
        rows[f"{fmt}_M1_logprob"] = {"us_per_draft": us,
                                     "GB/s": head.bytes_per_call(1) / (us * 1e-6) / 1e9,
                                     "argmax_ok": int(idx.item()) == int(d["top"][0]),
                                     "logprob": float(lp.item())}
        # a grammar mask keeping a seeded 10% of the tokens (always the planted second row,
        # never the larger planted top row): the sweep reads only the allowed rows
        words = d["mask"].shape[1]
        for M in ((1, 4) if args.full else (1,)):
            m = torch.from_numpy(d["mask"][:M].reshape(-1)).to(dev)
            x = d["x"][:M].to(dev)
            tm = time_sweep(head, x, args.steps, args.warmup, world, stream, mask=m,
                            mask_words=words)
            union = int(np.any(d["allowed"][:M], axis=0).sum())
            mbytes = head.bytes_per_call(M, rows=union) + M * words * 4
            us = tm["mean_ms"] * 1e3
            rows[f"{fmt}_M{M}_masked"] = {
                "us_per_draft": us, "median_launch_us": tm["median_ms"] * 1e3,
                "p10_p90_launch_us": [tm["p10_ms"] * 1e3, tm["p90_ms"] * 1e3],
                "allowed_rows": union, "bytes_per_step": mbytes,
                "GB/s": mbytes / (us * 1e-6) / 1e9,
                "frac_of_peak": mbytes / (us * 1e-6) / 1e9 / peak,
                "argmax_ok": bool(np.array_equal(tm["idx"], d["second"][:M])),
                "note": "bytes = allowed rows (union over inputs) + mask words + x + outputs"}
        if cpu_rows:
            cb = cpu_baseline_sweep(fmt, d, cfg)
            rows[f"{fmt}_M1"]["cpu_baseline"] = cb
            if fmt == "bf16":
                cpu_base = cb
        del head, table, d
        torch.cuda.empty_cache()

    if world == 1 and not args.no_extra and not args.rows and not args.ms:
        rows["tiny_draft_M1"] = bench_tiny_draft(dev, max(200, args.steps // 10), args.warmup)
        tpk, tsrc = measured_tflops()
        rows["prefill_32k"] = bench_prefill(dev, 10, tpk, tsrc)
        rows["decode_attn_32k"] = bench_attn(dev, max(100, args.steps // 10), args.warmup)
        torch.cuda.empty_cache()
        if cpu_rows:
            rows["tiny_draft_M1"]["cpu_baseline"] = cpu_baseline_tiny()
            rows["prefill_32k"]["cpu_baseline"] = cpu_baseline_prefill()

    if rank == 0 and main_line is not None:
        rec, nbytes, ms_max, e2e_max, pipe_ms, h2d, d2h, clk, cfg = main_line
        achieved = nbytes / (ms_max * 1e-3) / 1e9
        tr = NCU_TRAFFIC.get("bf16_M1")
        traffic = tr[0] if tr and tr[1] == sweep_source_hash() else None
        line = {
            "metric": METRIC,
            "value": nbytes * world / (ms_max * 1e-3) / 1e9,
            "unit": "GB/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms_max,
            "us_per_draft": ms_max * 1e3,
            "value_statistic": "mean over K back-to-back launches between two device events",
            "median_launch_us": rec["median_launch_us"],
            "p10_p90_launch_us": rec["p10_p90_launch_us"],
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic: seeded N(0, 0.02) bf16 table with planted maximum rows",
            "config": {"workload": f"bf16 lm_head sweep + argmax, table [{cfg['N']}, {cfg['K']}], M=1",
                       "table_bytes": cfg["N"] * cfg["K"] * 2, "M": 1,
                       "l2": "table (1.27 GB) larger than L2 (126 MB): no flush",
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "peak_source": f"{peak_src} hbm_gbs (a read+write copy; a pure read "
                                        f"stream can exceed it)",
                         "frac_of_nominal_8TBps": achieved / NOMINAL_HBM_GBS,
                         "kernel": "sweep_kernel<bf16, M<=8, argmax>"},
            "cpu_baseline": cpu_base,
            "e2e": {"value": nbytes * world / (e2e_max * 1e-3) / 1e9, "unit": "GB/s",
                    "us_per_draft": e2e_max * 1e3, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h,
                    "how": "mtp_lm_head_argmax_host per draft: x from pinned host memory, "
                           "result to pinned host memory, stream synchronised and the token "
                           "read by the host every step",
                    "pipelined_us_per_draft": pipe_ms * 1e3},
            "gpu_launches": args.steps,
            "clocks": clk,
            "rows": rows,
        }
        print(json.dumps(line), flush=True)
    elif rank == 0:  # a profiling run without the M = 1 BF16 row
        print(json.dumps({"rows": rows}), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

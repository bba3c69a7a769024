#!/usr/bin/env python3
"""Benchmark of the SAS gated block-sparse attention hot path on B200.

One step is one pass of the training hot path over the Qwen3-4B-shaped
workload: batch 1, 32 query / 8 KV heads, d 128, 32768 tokens, block 64,
Top-K 32. It runs Top-K selection + LSE(s), the gated forward, and the
backward with dq/dk/dv and the score gradient ds. The headline value is
selected-token TFLOP/s for fwd+bwd. The FLOP rule, per query head and query
block, is fwd = 4·d·64·(64·n_t + 32) and bwd = 2.5·fwd, where n_t = min(K, t)
and the causal current block counts as half.

The same JSON line also reports the single-token decode workload (16
sequences with 32768-token caches, Top-K 16 plus the current block, split-K +
merge) as tokens/s and gathered-KV GB/s.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

With N > 1 the script runs under torch.distributed.run, one rank per GPU.
Every rank processes its own replica of the workload (independent sequences,
no collective on the data path). value = total FLOPs of all ranks ÷ the
slowest rank's device time.
"""
from __future__ import annotations

import argparse
import hashlib
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

METRIC = "gated block-sparse attn TFLOP/s fwd+bwd and decode tok/s; % of roofline"
TRAIN = "qwen3_4b_train_32k"
DECODE = "decode_b16_32k"
L2_BYTES = 126 * 1024 * 1024


# ---------------------------------------------------------------------------
# work counts
# ---------------------------------------------------------------------------
def fwd_flops(n_q_heads, head_dim, n_blocks, top_k, batch=1, block=64, t_list=None):
    ts = range(n_blocks) if t_list is None else t_list
    per_head = sum(4.0 * head_dim * block * (block * min(top_k, t) + block / 2) for t in ts)
    return per_head * n_q_heads * batch


def decode_kv_bytes(w, cache_len):
    n_blocks = 0
    for L in cache_len:
        c = (int(L) - 1) // w.block
        n_blocks += min(w.top_k, c) * w.block + (int(L) - c * w.block)
    return n_blocks * w.n_kv_heads * w.head_dim * 2 * 2  # K and V, bf16


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            m = json.load(f)
        return dict(bf16=m["bf16_tflops"], bf16_sustained=m.get("bf16_tflops_sustained", m["bf16_tflops"]),
                    hbm=m["hbm_gbs"], source="measured")
    return dict(bf16=1590.0, bf16_sustained=1400.0, hbm=6650.0, source="fallback")


def traffic_record(kernel_key, src_files):
    """DRAM bytes per launch from a committed ncu summary, if taken on the current source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(kernel_key)
    if not rec:
        return None
    h = hashlib.sha256()
    for s in src_files:
        with open(os.path.join(ROOT, s), "rb") as f:
            h.update(f.read())
    return rec["bytes_per_launch"] if rec.get("source_sha256") == h.hexdigest() else None


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def wait_first(self, timeout=5.0):
        t0 = time.time()
        while self.proc is not None and not self.lines and time.time() - t0 < timeout:
            time.sleep(0.05)

    def mark(self, name):
        setattr(self, name, time.time())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        t0, t1 = getattr(self, "t_begin", 0.0), getattr(self, "t_end", float("inf"))
        inside = [ln for ts, ln in self.lines if t0 - 0.1 <= ts <= t1 + 0.1]
        for ln in (inside or [ln for _, ln in self.lines[-3:]]):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm),
                "window": "timed region" if inside else "just after the timed region"}


# ---------------------------------------------------------------------------
# CPU baseline: the fp64 oracle on a bounded sample
# ---------------------------------------------------------------------------
_ORACLE_CACHE = {}


def oracle_baseline(w, budget_s=15.0):
    """Times the oracle's fwd+bwd on one KV head over a growing set of query blocks.

    The sample's inputs and index sets are prepared once, outside the timing."""
    import oracle.sas_oracle as O
    from synth import workloads as W
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count()
    if w.name not in _ORACLE_CACHE:
        x0 = {k: v.astype(np.float64) for k, v in W.prefill_inputs(w, kv_heads=[0]).items()}
        _ORACLE_CACHE[w.name] = (x0, O.prefill_select(x0["s"], w.top_k)[0])
    x, idx = _ORACLE_CACHE[w.name]
    NB = w.n_blocks
    order = list(range(NB - 1, -1, -max(1, NB // 64)))  # spread over the sequence, long rows first
    done, t_used, flops = [], 0.0, 0.0
    t0 = time.perf_counter()
    for t in order:
        a = time.perf_counter()
        O.backward(x["q"], x["k"], x["v"], x["s"], idx, x["do"], t_list=[t])  # recomputes P and o itself
        O.forward(x["q"], x["k"], x["v"], x["s"], idx, t_list=[t])
        t_used += time.perf_counter() - a
        done.append(t)
        if time.perf_counter() - t0 > budget_s:
            break
    flops = 3.5 * fwd_flops(w.group, w.head_dim, NB, w.top_k, t_list=done)
    return {"value": flops / t_used / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"KV head 0 ({w.group} query heads), {len(done)} of {NB} query blocks spread over the "
                      f"sequence, fwd+bwd in NumPy fp64; {t_used:.1f} s"}


# ---------------------------------------------------------------------------
# ranks: one process per GPU, replicas of the workload, no collective on the data path
# ---------------------------------------------------------------------------
def rank_env(env=None):
    """(rank, world, local_rank) from the torch.distributed.run environment (one rank without it)."""
    env = os.environ if env is None else env
    return int(env.get("RANK", 0)), int(env.get("WORLD_SIZE", 1)), int(env.get("LOCAL_RANK", 0))


def relaunch_command(gpus: int, argv, port: int):
    """The torch.distributed.run command that runs this script with one rank per GPU."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={gpus}",
            "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__)] + list(argv)


def init_ranks(world: int, backend: str, device=None, timeout_s: float = 120.0):
    """The process group for the barrier and the max-over-ranks timing, or None for one rank."""
    if world <= 1:
        return None
    import datetime
    import torch.distributed as dist
    kw = {"device_id": device} if backend == "nccl" and device is not None else {}
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return dist


def barrier(dist) -> None:
    if dist is not None:
        dist.barrier()


def max_over_ranks(dist, x: float, device="cpu") -> float:
    """The slowest rank's value: every rank takes the same all-reduce, in the same order."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput of weak-scaled replicas: all ranks' units over the slowest rank's time."""
    return world * units_per_rank / max_seconds


def all_ranks_ok(dist, ok: bool, device="cpu") -> bool:
    """True when every rank reports ok; every rank takes this same all-reduce."""
    if dist is None:
        return ok
    import torch
    t = torch.tensor([1 if ok else 0], dtype=torch.int32, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MIN)
    return bool(t.item())


def is_device_failure(e: BaseException) -> bool:
    """A CUDA failure leaves the context unusable for the legs after it: such errors end the run."""
    msg = str(e)
    return "CUDA" in msg or "cuda" in type(e).__name__.lower() or "device error" in msg or "SAS_ERR_CUDA" in msg


def sig3(x):
    """x rounded to three significant digits (compact summary fields)."""
    if x is None or not isinstance(x, (int, float)) or x == 0 or not math.isfinite(x):
        return x
    return float(f"{x:.3g}")


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def run_gpu(args, rank, world, local_rank):
    import torch
    import learned_block_sparse_warp_b200 as sas
    from synth import workloads as W
    from synth.device import decode_to_device, prefill_to_device

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = init_ranks(world, "nccl", dev)

    stream = torch.cuda.Stream(device=dev)
    pk = peaks()
    line = {}

    # ---------------- training step: select + LSE, forward, backward with ds ----------------
    if args.only in ("all", "train"):
        w = W.WORKLOADS[TRAIN]
        p = sas.Params(batch=w.batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, head_dim=w.head_dim,
                       seq_len=w.seq_len, top_k=w.top_k, gate_mode=sas.SAS_GATE_LOG_SOFTMAX)
        x = prefill_to_device(w, device=dev)
        out = sas.empty_prefill_outputs(p, device=dev)
        in_bytes = sum(t.numel() * t.element_size() for t in x.values())

        def step(q, k, v, s, dO, o):
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            ev[0].record(stream)
            sas.sas_topk_select(p, s, o["idx"], o["lse_s"], stream=stream)
            ev[1].record(stream)
            sas.sas_fwd(p, q, k, v, s, o["idx"], o["lse_s"], o["o"], o["lse_o"], stream=stream)
            ev[2].record(stream)
            sas.sas_bwd(p, q, k, v, o["o"], dO, s, o["idx"], o["lse_s"], o["lse_o"], o["dq"], o["dk"], o["dv"],
                        o["ds"], o["ws"], stream=stream)
            ev[3].record(stream)
            return ev

        evs = []
        with ClockSampler(local_rank) as clk:
            clk.wait_first()
            with torch.cuda.stream(stream):
                for _ in range(args.warmup):
                    step(x["q"], x["k"], x["v"], x["s"], x["do"], out)
            torch.cuda.synchronize()
            if sas.sas_get_device_error(stream) != 0:
                raise RuntimeError("device error during warm-up")
            barrier(dist)
            torch.cuda.synchronize()
            clk.mark("t_begin")
            t_start = torch.cuda.Event(enable_timing=True)
            t_end = torch.cuda.Event(enable_timing=True)
            t_start.record(stream)
            for _ in range(args.steps):
                evs.append(step(x["q"], x["k"], x["v"], x["s"], x["do"], out))
            t_end.record(stream)
            torch.cuda.synchronize()
            clk.mark("t_end")
            time.sleep(0.25)
        barrier(dist)
        total_ms = max_over_ranks(dist, t_start.elapsed_time(t_end), dev)
        sel_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
        fwd_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
        bwd_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
        if sas.sas_get_device_error(stream) != 0:
            raise RuntimeError("device error during the timed steps")

        F = fwd_flops(w.n_q_heads, w.head_dim, w.n_blocks, w.top_k, batch=w.batch)
        step_flops = 3.5 * F

        # end to end through the C ABI with host buffers: every step's inputs go up from pinned host
        # memory and every output comes back, inside the timed region (sas_train_steps_host)
        e2e = None
        if not args.no_e2e:
            # Every rank takes the same collectives whatever happens: a host-side failure is
            # recorded and agreed on with all_ranks_ok; a device failure ends the run.
            err, e2e_local, n_e2e = None, None, max(3, min(args.steps, 8))
            h_in = h_out = slots = host_steps = None
            try:
                h_in = {k_: t.cpu().pin_memory() for k_, t in x.items()}
                outs = ["o", "lse_o", "dq", "dk", "dv", "ds"]
                h_out = {k_: torch.empty(out[k_].shape, dtype=out[k_].dtype, pin_memory=True) for k_ in outs}
                h2d = sum(t.numel() * t.element_size() for t in h_in.values())
                d2h = sum(t.numel() * t.element_size() for t in h_out.values())
                slots = [sas.empty_device_slot(p, device=dev) for _ in range(2)]
                host_steps = [{**h_in, **h_out} for _ in range(n_e2e)]
                sas.sas_train_steps_host(p, host_steps[:2], slots, stream=stream)  # untimed: first launches
                torch.cuda.synchronize()
            except Exception as e:
                if is_device_failure(e):
                    raise
                err = e
            if all_ranks_ok(dist, err is None, dev):
                barrier(dist)
                torch.cuda.synchronize()
                try:
                    a = torch.cuda.Event(enable_timing=True)
                    b = torch.cuda.Event(enable_timing=True)
                    a.record(stream)
                    sas.sas_train_steps_host(p, host_steps, slots, stream=stream)
                    b.record(stream)
                    torch.cuda.synchronize()
                    if sas.sas_get_device_error(stream) != 0:
                        raise RuntimeError("device error during the end-to-end steps")
                    e2e_local = a.elapsed_time(b)
                except Exception as e:
                    if is_device_failure(e):
                        raise
                    err = e
                if all_ranks_ok(dist, err is None, dev):
                    e2e_ms = max_over_ranks(dist, e2e_local, dev) / n_e2e
                    e2e = {"value": job_rate(step_flops, world, e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                           "steps": n_e2e,
                           "api": "sas_train_steps_host: two device slots; the next step's upload and the previous "
                                  "step's download overlap each step's kernels"}
            if e2e is None:
                e2e = {"error": (f"{type(err).__name__}: {err}" if err is not None else "failed on another rank")[:300]}
            h_in = h_out = slots = host_steps = None  # noqa: F841  (frees the pinned and device buffers)
            torch.cuda.empty_cache()

        bwd_flops = 2.5 * F
        achieved = bwd_flops / (bwd_ms * 1e-3) / 1e12
        line.update({
            "metric": METRIC, "value": job_rate(step_flops * args.steps, world, total_ms * 1e-3) / 1e12,
            "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": TRAIN, "batch": w.batch, "q_heads": w.n_q_heads, "kv_heads": w.n_kv_heads,
                       "head_dim": w.head_dim, "seq_len": w.seq_len, "block": w.block, "top_k": w.top_k,
                       "gate": "log_softmax (training form)", "flops_per_step": step_flops,
                       "parallelism": f"dp{world} (independent replicas)",
                       "l2": f"inputs {in_bytes / 1e9:.2f} GB per step > 126 MB L2 (no flush)"},
            "breakdown_ms": {"select": sel_ms, "fwd": fwd_ms, "bwd": bwd_ms},
            "fwd_tflops": F / (fwd_ms * 1e-3) / 1e12,
            "bwd_tflops": achieved,
            # fractions of the measured burst bf16 peak: the kernels run back to back for well under a
            # second at full clock, which is the burst measurement's condition
            "frac_of_peak": {"step": step_flops / (total_ms / args.steps * 1e-3) / 1e12 / pk["bf16"],
                             "fwd": F / (fwd_ms * 1e-3) / 1e12 / pk["bf16"], "bwd": achieved / pk["bf16"],
                             "peak": pk["bf16"], "peak_source": pk["source"] + " burst bf16"},
            "roofline": {"bound": "tensor",
                         "kernel": "sas_bwd call (tcgen05 KV pass storing dZ, dQ gather-GEMM pass, prep, "
                                   "reverse index, ds chain)",
                         "achieved": achieved, "peak": pk["bf16"], "unit": "TFLOP/s",
                         "frac": achieved / pk["bf16"], "peak_source": pk["source"] + " burst bf16",
                         "frac_of_sustained": achieved / pk["bf16_sustained"],
                         "flops_per_launch": bwd_flops,
                         "traffic": traffic_record("bwd_call", ["learned_block_sparse_warp_b200/csrc/bwd_mma.cu",
                                                                "learned_block_sparse_warp_b200/csrc/bwd_sm100.cu"])},
            "e2e": e2e,
            "gpu_launches": args.steps * 10,
            "clocks": clk.summary(),
        })
        del x, out
        torch.cuda.empty_cache()

    # ---------------- decode: select, split-K, merge, over rotating selections ----------------
    if args.only in ("all", "decode") and not args.no_decode:
        wd = W.WORKLOADS[DECODE]
        pd = sas.Params(batch=wd.batch, n_q_heads=wd.n_q_heads, n_kv_heads=wd.n_kv_heads, head_dim=wd.head_dim,
                        seq_len=wd.seq_len, top_k=wd.top_k, gate_mode=sas.SAS_GATE_NONE)
        xd = decode_to_device(wd, device=dev)
        n_split = args.n_split if args.n_split > 0 else wd.top_k + 1
        od = sas.empty_decode_outputs(pd, n_split, device=dev)
        # a read-only sweep of 2x the L2 evicts the previous step's lines without leaving dirty ones,
        # whose write-back would otherwise land inside the next timed step
        flush = torch.ones(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
        flush_sink = torch.empty((), dtype=torch.float32, device=dev)

        # Timing. A serving loop replays the captured step. Each figure below is one captured
        # graph of R back-to-back launches, timed by one event pair and divided by R, so no
        # launch or event floor enters it. The launches rotate over N_ROT score sets with
        # different selections, so consecutive steps gather different blocks and K/V is read
        # from HBM (only the current block, the same in every set, can stay in L2).
        N_ROT, R = 4, 32
        gen = torch.Generator(device=dev)
        gen.manual_seed(4242)
        s_rot = [xd["s"]] + [torch.randn(xd["s"].shape, generator=gen, device=dev) * 2 ** 0.5
                             for _ in range(N_ROT - 1)]
        o_rot = [od] + [sas.empty_decode_outputs(pd, n_split, device=dev) for _ in range(N_ROT - 1)]
        cl = xd["cache_len"]
        with torch.cuda.stream(stream):
            for k_ in range(N_ROT):  # each set's index lists and partials exist before any timing
                sas.decode_step(pd, xd["q"], xd["k"], xd["v"], cl, s_rot[k_], n_split, o_rot[k_], stream=stream)
        kernels = {
            "select": lambda k_: sas.sas_topk_select(pd, s_rot[k_], o_rot[k_]["idx"], o_rot[k_]["lse_s"],
                                                     cache_len=cl, stream=stream),
            "split": lambda k_: sas.sas_decode(pd, xd["q"], xd["k"], xd["v"], cl, s_rot[k_], o_rot[k_]["idx"],
                                               o_rot[k_]["lse_s"], n_split, o_rot[k_]["o_part"],
                                               o_rot[k_]["lse_part"], stream=stream),
            "combine": lambda k_: sas.sas_decode_combine(pd, n_split, o_rot[k_]["o_part"], o_rot[k_]["lse_part"],
                                                         o_rot[k_]["o"], o_rot[k_]["lse_o"], stream=stream),
            "step": lambda k_: sas.decode_step(pd, xd["q"], xd["k"], xd["v"], cl, s_rot[k_], n_split, o_rot[k_],
                                               stream=stream),
            # the one-launch step: select, attention and merge; a serving loop takes o and lse_o
            "fused": lambda k_: sas.sas_decode_fused(pd, xd["q"], xd["k"], xd["v"], cl, s_rot[k_], o_rot[k_]["o"],
                                                     lse_o=o_rot[k_]["lse_o"], stream=stream)}

        def capture_r(fn):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream, capture_error_mode="thread_local"):
                for r_ in range(R):
                    fn(r_ % N_ROT)
            return g

        with torch.cuda.stream(stream):  # the fused kernel's attributes are set outside the captures
            kernels["fused"](0)
        graphs = {key: capture_r(fn) for key, fn in kernels.items()}
        step_graph = sas.DecodeGraph(pd, xd["q"], xd["k"], xd["v"], cl, xd["s"], n_split, od, stream=stream,
                                     fused=True)

        def replay_timed(g):
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            ev[0].record(stream)
            g.replay()
            ev[1].record(stream)
            return ev

        n_rep = max(5, args.steps // 2)
        timings = {key: [] for key in graphs}
        flushed = []
        with torch.cuda.stream(stream):
            for _ in range(max(3, args.warmup)):
                for g in graphs.values():
                    g.replay()
                step_graph.replay()
            for _ in range(n_rep):
                for key, g in graphs.items():
                    timings[key].append(replay_timed(g))
            # the conservative view: one step after an L2 flush (includes one graph launch)
            for _ in range(max(20, args.steps)):
                torch.sum(flush, dim=0, out=flush_sink)
                flushed.append(replay_timed(step_graph.graph))
        torch.cuda.synchronize()
        med = {key: statistics.median(e[0].elapsed_time(e[1]) for e in evs) / R for key, evs in timings.items()}
        med["flushed"] = statistics.median(e[0].elapsed_time(e[1]) for e in flushed)
        step_ms = max_over_ranks(dist, med["fused"], dev)
        split_ms = med["split"]
        kv = decode_kv_bytes(wd, xd["cache_len"].cpu().numpy())
        gbs = kv / (step_ms * 1e-3) / 1e9
        split_gbs = kv / (split_ms * 1e-3) / 1e9
        line["decode"] = {
            "workload": DECODE, "tok_per_s": job_rate(wd.batch, world, step_ms * 1e-3), "ms_per_step": step_ms,
            "path": "sas_decode_fused: Top-K select, attention and LSE merge in one launch (outputs o, lse_o)",
            "launch": f"{R} steps back to back in one CUDA graph, rotating over {N_ROT} score sets with "
                      f"different selections",
            "three_kernel_ms_per_step": med["step"],
            "three_kernel": "sas_topk_select, sas_decode and sas_decode_combine chained by programmatic dependent "
                            "launch (outputs idx, lse_s, o, lse_o)",
            "select_ms": med["select"], "split_ms": split_ms, "combine_ms": med["combine"], "n_split": n_split,
            "breakdown": f"the three-kernel path, each kernel as {R} back-to-back launches in one graph over the "
                         f"rotating sets, / {R}",
            "flushed_ms_per_step": med["flushed"],
            "flushed": "one captured fused step replayed after a 252 MB read that flushes the L2 (one graph "
                       "launch included)",
            "gate": "none (inference form)",
            "l2": "no flush: consecutive steps gather different blocks (rotating selections)",
            "roofline": {"bound": "hbm", "kernel": "decode_fused_kernel (sas_decode_fused), the whole step",
                         "achieved": gbs, "peak": pk["hbm"], "unit": "GB/s", "frac": gbs / pk["hbm"],
                         "algorithmic_bytes": kv,
                         "traffic": traffic_record("decode_fused",
                                                   ["learned_block_sparse_warp_b200/csrc/decode.cu"])},
            "split_roofline": {"kernel": "decode_split_kernel (sas_decode)", "achieved": split_gbs,
                               "frac": split_gbs / pk["hbm"],
                               "traffic": traffic_record("decode_split",
                                                         ["learned_block_sparse_warp_b200/csrc/decode.cu"])},
            "gpu_launches_per_step": 1}
        del step_graph, kernels, graphs, o_rot, s_rot
        if sas.sas_get_device_error(stream) != 0:
            raise RuntimeError("device error during decode")
        # the captured step at other split counts, for the choice of the default (the headline stays
        # at n_split above); each is the same graph replay with the L2 flushed before it
        sweep = {}
        try:
            for ns in (1, 2, 3, 5, 9):
                if ns == n_split or (wd.top_k + ns) // ns > 64:
                    continue
                o_ns = sas.empty_decode_outputs(pd, ns, device=dev)
                g_ns = sas.DecodeGraph(pd, xd["q"], xd["k"], xd["v"], xd["cache_len"], xd["s"], ns, o_ns,
                                       stream=stream)
                evs = []
                with torch.cuda.stream(stream):
                    for i in range(3 + max(10, args.steps)):
                        torch.sum(flush, dim=0, out=flush_sink)
                        ev = replay_timed(g_ns.graph)
                        if i >= 3:
                            evs.append(ev)
                torch.cuda.synchronize()
                sweep[str(ns)] = statistics.median(e[0].elapsed_time(e[1]) for e in evs)
                del g_ns, o_ns
            if sas.sas_get_device_error(stream) != 0:
                raise RuntimeError("device error in the split-count sweep")
        except Exception as e:  # diagnostic only: a host-side failure is reported, a device failure raised
            if is_device_failure(e):
                raise
            sweep["error"] = f"{type(e).__name__}: {e}"[:300]
        line["decode"]["n_split_sweep_ms_per_step"] = sweep

    # ---------------- the 128K forward and the budget x length sweep ----------------
    if args.only in ("all", "sweep"):
        try:
            line["sweep"] = sweep_section(args, sas, stream, dev, pk, dist, world)
        except Exception as e:  # a supplementary section: a host-side failure is reported in the line
            if args.only == "sweep" or world > 1 or is_device_failure(e):
                raise
            line["sweep"] = {"error": f"{type(e).__name__}: {e}"[:400]}

    # ---------------- long-context decode that scores its own history ----------------
    if args.only in ("all", "long_decode") and not args.no_decode:
        try:
            line["long_decode"] = long_decode_section(args, sas, stream, dev, pk, dist, world)
        except Exception as e:  # a supplementary section: a host-side failure is reported in the line
            if args.only == "long_decode" or world > 1 or is_device_failure(e):
                raise
            line["long_decode"] = {"error": f"{type(e).__name__}: {e}"[:400]}

    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.only in ("all", "train"):
        line["cpu_baseline"] = oracle_baseline(W.WORKLOADS[TRAIN], budget_s=args.cpu_budget)
    line["summary"] = compact_summary(line)  # last: a reader that keeps only the line's tail still sees it
    if dist is not None:
        dist.destroy_process_group()
    return line


def compact_summary(line: dict) -> dict:
    """Every workload's headline in a few hundred characters, three significant digits.

    train: [ms per step, TFLOP/s, fraction of burst bf16 peak]; fwd/bwd: [TFLOP/s, fraction];
    decode: [tokens/s, µs per step, GB/s of the one-launch step, its fraction of HBM]; sweep: one
    [top_k, seq_len, ms, TFLOP/s, fraction] per point (the 128K forward first);
    long_decode: [batch, cache tokens, µs per step, the selection's share of the kernels' time]."""
    out = {}
    if "ms_per_step" in line and "frac_of_peak" in line:
        f = line["frac_of_peak"]
        out["train"] = [sig3(line["ms_per_step"]), sig3(line["value"]), sig3(f["step"])]
        out["fwd"] = [sig3(line["fwd_tflops"]), sig3(f["fwd"])]
        out["bwd"] = [sig3(line["bwd_tflops"]), sig3(f["bwd"])]
    dec = line.get("decode")
    if isinstance(dec, dict) and "tok_per_s" in dec:
        r = dec["roofline"]
        out["decode"] = [sig3(dec["tok_per_s"]), sig3(dec["ms_per_step"] * 1e3), sig3(r["achieved"]),
                         sig3(r["frac"])]
    sw = line.get("sweep")
    if isinstance(sw, dict):
        if "points" in sw:
            out["sweep"] = [[p_["top_k"], p_["seq_len"], sig3(p_["ms_per_step"]), sig3(p_["tflops"]),
                             sig3(p_["frac"])] for p_ in sw["points"]]
        elif "error" in sw:
            out["sweep"] = sw["error"][:120]
    ld = line.get("long_decode")
    if isinstance(ld, dict):
        if "workloads" in ld:
            out["long_decode"] = [[r_["batch"], r_["cache_len"], sig3(r_["ms_per_step"] * 1e3), sig3(r_["select_share"])]
                                  for r_ in ld["workloads"]]
        elif "error" in ld:
            out["long_decode"] = ld["error"][:120]
    return out


# ---------------------------------------------------------------------------
# the Llama-3.1-8B 128K forward and the Qwen3-14B budget x length sweep
# ---------------------------------------------------------------------------
SWEEP = ["llama31_8b_fwd_128k"] + [f"qwen3_14b_k{k}_n{n}" for k in (16, 32, 64) for n in (8192, 32768, 65536)]


def sweep_inputs(w, dev, torch):
    """Seeded device-side inputs with the workload's recipe: q, k, v, dO ~ N(0, 1) bf16, and s ~ N(0, 2),
    or, with heavy hitters, s = block-mean(k) . block-and-group-mean(q) / sqrt(d) + N(0, 0.5) after
    1% of the keys and every query of the group get 4 u_h."""
    B, Hq, Hkv, N, d, NB, G = w.batch, w.n_q_heads, w.n_kv_heads, w.seq_len, w.head_dim, w.n_blocks, w.group
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.seed)
    bf = torch.bfloat16
    q = torch.randn((B, Hq, N, d), generator=gen, device=dev, dtype=torch.float32)
    k = torch.randn((B, Hkv, N, d), generator=gen, device=dev, dtype=torch.float32)
    if w.heavy_hitters:
        u = torch.randn((B, Hkv, d), generator=gen, device=dev)
        u = u / u.norm(dim=-1, keepdim=True)
        n_hh = max(1, round(0.01 * N))
        for b in range(B):
            for h in range(Hkv):
                pos = torch.randperm(N, generator=gen, device=dev)[:n_hh]
                k[b, h, pos] += 4 * u[b, h]
        q += 4 * u.repeat_interleave(G, dim=1)[:, :, None, :]
    q, k = q.to(bf), k.to(bf)
    v = torch.randn((B, Hkv, N, d), generator=gen, device=dev, dtype=torch.float32).to(bf)
    if w.heavy_hitters:
        kbar = k.float().view(B, Hkv, NB, 64, d).mean(3)
        qbar = q.float().view(B, Hkv, G, NB, 64, d).mean((2, 4))
        s = qbar @ kbar.transpose(-1, -2) / math.sqrt(d)
        s += math.sqrt(0.5) * torch.randn(s.shape, generator=gen, device=dev)
    else:
        s = math.sqrt(w.s_var) * torch.randn((B, Hkv, NB, NB), generator=gen, device=dev)
    x = dict(q=q, k=k, v=v, s=s.contiguous())
    if w.backward:
        x["do"] = torch.randn((B, Hq, N, d), generator=gen, device=dev, dtype=torch.float32).to(bf)
    return x


def sweep_section(args, sas, stream, dev, pk, dist, world):
    import torch
    from synth import workloads as W
    points = []
    for name in SWEEP:
        if args.sweep_point and name != args.sweep_point:
            continue
        w = W.WORKLOADS[name]
        p = sas.Params(batch=w.batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, head_dim=w.head_dim,
                       seq_len=w.seq_len, top_k=w.top_k, gate_mode=sas.SAS_GATE_LOG_SOFTMAX)
        with torch.cuda.stream(stream):
            x = sweep_inputs(w, dev, torch)
        torch.cuda.synchronize()
        out = sas.empty_prefill_outputs(p, device=dev, backward=w.backward)
        if w.backward and args.min_workspace:  # the smallest workspace: dQ recomputes S and dP
            out["ws"] = torch.empty((sas.sas_bwd_workspace_size_min(p),), dtype=torch.uint8, device=dev)

        def run(evs=None):
            # select + LSE, forward, backward; with evs, an event after each call
            sas.sas_topk_select(p, x["s"], out["idx"], out["lse_s"], stream=stream)
            if evs is not None:
                evs[0].record(stream)
            sas.sas_fwd(p, x["q"], x["k"], x["v"], x["s"], out["idx"], out["lse_s"], out["o"], out["lse_o"],
                        stream=stream)
            if evs is not None:
                evs[1].record(stream)
            if w.backward:
                sas.sas_bwd(p, x["q"], x["k"], x["v"], out["o"], x["do"], x["s"], out["idx"], out["lse_s"],
                            out["lse_o"], out["dq"], out["dk"], out["dv"], out["ds"], out["ws"], stream=stream)
            if evs is not None:
                evs[2].record(stream)

        n = max(5, min(args.steps, 10))
        with torch.cuda.stream(stream):
            for _ in range(max(3, args.warmup)):
                run()
        torch.cuda.synchronize()
        barrier(dist)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        marks = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n)]
        a.record(stream)
        with torch.cuda.stream(stream):
            for i in range(n):
                run(marks[i])
        b.record(stream)
        torch.cuda.synchronize()
        starts = [a] + [m[2] for m in marks[:-1]]
        split_ms = {"select": statistics.mean(st.elapsed_time(m[0]) for st, m in zip(starts, marks)),
                    "fwd": statistics.mean(m[0].elapsed_time(m[1]) for m in marks),
                    "bwd": statistics.mean(m[1].elapsed_time(m[2]) for m in marks) if w.backward else 0.0}
        if sas.sas_get_device_error(stream) != 0:
            raise RuntimeError(f"device error in {name}")
        ms = max_over_ranks(dist, a.elapsed_time(b), dev) / n
        F = fwd_flops(w.n_q_heads, w.head_dim, w.n_blocks, w.top_k, batch=w.batch)
        flops = (3.5 if w.backward else 1.0) * F
        tf = job_rate(flops, world, ms * 1e-3) / 1e12
        points.append({"workload": name, "q_heads": w.n_q_heads, "kv_heads": w.n_kv_heads, "seq_len": w.seq_len,
                       "top_k": w.top_k, "pass": "fwd+bwd" if w.backward else "fwd", "tflop_per_step": flops / 1e12,
                       "ms_per_step": ms, "tflops": tf, "frac": tf / (pk["bf16"] * world),
                       "breakdown_ms": split_ms,
                       "fwd_tflops": F / (split_ms["fwd"] * 1e-3) / 1e12,
                       "bwd_tflops": 2.5 * F / (split_ms["bwd"] * 1e-3) / 1e12 if w.backward else None,
                       "bwd_workspace": ("minimal" if args.min_workspace else "full") if w.backward else None})
        del x, out
        torch.cuda.empty_cache()
    return {"points": points, "peak": pk["bf16"], "peak_source": pk["source"] + " burst bf16",
            "gate": "log_softmax (training form)",
            "data": "synthetic, from a seeded device generator with each workload's recipe",
            "l2": "inputs larger than L2 at every point (no flush)"}


# ---------------------------------------------------------------------------
# long-context decode: block-mean update, fused scoring + Top-K, split-K, merge
# ---------------------------------------------------------------------------
LONG_DECODE = [  # (batch, cache tokens): the context lengths and batch sizes of the pages' decode measurements
    (1, 65536), (1, 262144), (1, 524288), (8, 65536)]


def long_decode_section(args, sas, stream, dev, pk, dist, world):
    import torch
    out_rows = []
    Hq, Hkv, d, K = 32, 8, 128, 16

    def timed(g):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        ev[0].record(stream)
        g.replay()
        ev[1].record(stream)
        return ev

    for B, L in LONG_DECODE:
        NB = L // 64
        p = sas.Params(batch=B, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, seq_len=L, top_k=K,
                       gate_mode=sas.SAS_GATE_NONE)
        gen = torch.Generator(device=dev)
        gen.manual_seed(1000 + B * 7 + NB)
        with torch.cuda.stream(stream):
            kc = torch.randn((B, Hkv, L, d), generator=gen, device=dev, dtype=torch.bfloat16)
            vc = torch.randn((B, Hkv, L, d), generator=gen, device=dev, dtype=torch.bfloat16)
            q = torch.randn((B, Hq, d), generator=gen, device=dev, dtype=torch.bfloat16)
            cl = torch.full((B,), L, dtype=torch.int32, device=dev)
            km = torch.empty((B, Hkv, NB, d), dtype=torch.bfloat16, device=dev)
            sas.sas_block_mean_keys(p, kc, km, stream=stream)  # after the prefill: every block
            s = torch.empty((B, Hkv, NB), dtype=torch.float32, device=dev)
        n_split = K + 1
        # N_ROT query sets with their own outputs: consecutive steps select different blocks
        N_ROT, R = 4, 32
        q_rot = [q] + [torch.randn((B, Hq, d), generator=gen, device=dev, dtype=torch.bfloat16)
                       for _ in range(N_ROT - 1)]
        s_rot = [s] + [torch.empty_like(s) for _ in range(N_ROT - 1)]
        o_rot = [sas.empty_decode_outputs(p, n_split, device=dev) for _ in range(N_ROT)]
        with torch.cuda.stream(stream):
            for k_ in range(N_ROT):
                sas.decode_step_scored(p, q_rot[k_], kc, vc, km, cl, s_rot[k_], n_split, o_rot[k_], stream=stream)
        kernels = {
            "mean_update": lambda k_: sas.sas_block_mean_keys(p, kc, km, cache_len=cl, stream=stream),
            "select": lambda k_: sas.sas_decode_select_scored(p, q_rot[k_], km, cl, s_rot[k_], o_rot[k_]["idx"],
                                                              o_rot[k_]["lse_s"], stream=stream),
            "split": lambda k_: sas.sas_decode(p, q_rot[k_], kc, vc, cl, s_rot[k_], o_rot[k_]["idx"],
                                               o_rot[k_]["lse_s"], n_split, o_rot[k_]["o_part"],
                                               o_rot[k_]["lse_part"], stream=stream),
            "combine": lambda k_: sas.sas_decode_combine(p, n_split, o_rot[k_]["o_part"], o_rot[k_]["lse_part"],
                                                         o_rot[k_]["o"], o_rot[k_]["lse_o"], stream=stream),
            "step": lambda k_: sas.decode_step_scored(p, q_rot[k_], kc, vc, km, cl, s_rot[k_], n_split, o_rot[k_],
                                                      stream=stream)}
        # unfused comparison: the scores by a library batched matmul, then the separate Top-K kernel
        qbar = torch.empty((B * Hkv, d, 1), dtype=torch.bfloat16, device=dev)
        s_mm = torch.empty((B * Hkv, NB, 1), dtype=torch.bfloat16, device=dev)
        s_un = torch.empty((B, Hkv, NB), dtype=torch.float32, device=dev)

        def unfused(k_):
            qbar.copy_(q_rot[k_].view(B * Hkv, Hq // Hkv, d).float().mean(dim=1).mul_(d ** -0.5).unsqueeze(-1))
            torch.bmm(km.view(B * Hkv, NB, d), qbar, out=s_mm)
            s_un.view(B * Hkv, NB).copy_(s_mm.view(B * Hkv, NB))
            sas.sas_topk_select(p, s_un, o_rot[k_]["idx"], o_rot[k_]["lse_s"], cache_len=cl, stream=stream)

        with torch.cuda.stream(stream):
            unfused(0)  # first call outside capture: the library GEMM's handle is created here
        kernels["select_unfused"] = unfused

        # each figure: one graph of R back-to-back launches over the rotating sets, / R
        def capture_r(fn):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream, capture_error_mode="thread_local"):
                for r_ in range(R):
                    fn(r_ % N_ROT)
            return g

        graphs = {key: capture_r(fn) for key, fn in kernels.items()}
        times = {k: [] for k in graphs}
        with torch.cuda.stream(stream):
            for _ in range(max(3, args.warmup)):
                for g in graphs.values():
                    g.replay()
            for _ in range(max(5, args.steps // 2)):
                for key, g in graphs.items():
                    times[key].append(timed(g))
        torch.cuda.synchronize()
        med = {k: statistics.median(e[0].elapsed_time(e[1]) for e in evs) / R for k, evs in times.items()}
        if sas.sas_get_device_error(stream) != 0:
            raise RuntimeError("device error during long-context decode")
        step_ms = max_over_ranks(dist, med["step"], dev)
        c = (L - 1) // 64
        sel_bytes = B * Hkv * c * (d * 2 + 4) + B * Hq * d * 2 + B * Hkv * (K + 1) * 4
        gbs = sel_bytes / (med["select"] * 1e-3) / 1e9
        out_rows.append({
            "batch": B, "cache_len": L, "top_k": K, "heads": f"{Hq}/{Hkv}", "head_dim": d,
            "ms_per_step": step_ms, "tok_per_s": job_rate(B, world, step_ms * 1e-3),
            "breakdown_ms": {k: med[k] for k in ("mean_update", "select", "split", "combine")},
            "select_share": med["select"] / (med["mean_update"] + med["select"] + med["split"] + med["combine"]),
            "select_unfused_ms": med["select_unfused"],
            "select_roofline": {"bound": "hbm", "kernel": "select_scored_kernel (sas_decode_select_scored)",
                                "achieved": gbs, "peak": pk["hbm"], "unit": "GB/s", "frac": gbs / pk["hbm"],
                                "algorithmic_bytes": sel_bytes}})
        del kernels, graphs, kc, vc, km, s, s_rot, q_rot, o_rot
        torch.cuda.empty_cache()
    return {"workloads": out_rows, "gate": "none (inference form)", "n_split": K + 1,
            "data": "synthetic: q, k, v ~ N(0, 1) bf16 from a seeded device generator",
            "launch": "steps of four PDL-chained kernels (block-mean update, fused scoring + Top-K, split-K, merge); "
                      "every figure is one graph of 32 back-to-back launches / 32",
            "l2": "no flush: the launches rotate over 4 query sets, so consecutive steps select different blocks",
            "gpu_launches_per_step": 4}


# ---------------------------------------------------------------------------
# reference arm: the fp64 oracle on the host cores
# ---------------------------------------------------------------------------
def run_reference(args, rank, world):
    if rank != 0:
        return None
    from synth import workloads as W
    w = W.WORKLOADS[TRAIN]
    budget = max(2.0, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_baseline(w, budget_s=budget)
    vals = []
    cb = None
    for _ in range(args.steps):
        cb = oracle_baseline(w, budget_s=budget)
        vals.append(cb["value"])
    value = statistics.mean(vals)
    F = fwd_flops(w.n_q_heads, w.head_dim, w.n_blocks, w.top_k)
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 3.5 * F / (value * 1e12) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": TRAIN, "batch": w.batch, "q_heads": w.n_q_heads, "kv_heads": w.n_kv_heads,
                       "head_dim": w.head_dim, "seq_len": w.seq_len, "block": w.block, "top_k": w.top_k,
                       "gate": "log_softmax (training form)"},
            "cpu_baseline": dict(cb, value=value),
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["sas", "reference"], default="sas")
    ap.add_argument("--only", choices=["all", "train", "decode", "long_decode", "sweep"], default="all",
                    help="run only one workload (for profiling); the JSON line needs 'all'")
    ap.add_argument("--n-split", type=int, default=0, help="decode splits (0: K + 1)")
    ap.add_argument("--sweep-point", default="", help="with --only sweep: run this sweep workload alone (profiling)")
    ap.add_argument("--min-workspace", action="store_true",
                    help="with --only sweep: give sas_bwd its smallest workspace (the recomputing dQ pass)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for cpu_baseline")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:  # one rank per GPU under torch.distributed.run
        import socket
        with socket.socket() as sock:
            sock.bind(("127.0.0.1", 0))
            port = sock.getsockname()[1]
        sys.exit(subprocess.call(relaunch_command(args.gpus, sys.argv[1:], port)))
    rank, world, local_rank = rank_env()
    if args.impl == "reference":
        line = run_reference(args, rank, world)
    else:
        line = run_gpu(args, rank, world, local_rank)
    if rank == 0 and line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""Benchmark: EAGLE-3 tree-verification step on B200.

Default workload (one GPU): Llama-3.1-8B-shaped bf16 random-init target,
batch 1, prefix 2048 tokens, a 60-draft tree of depth 8 (per-level widths
10,10,10,8,8,6,4,4, top-k 10 expansion) whose tokens are planted with
acceptance probability 0.8.  A step is one whole verification: one target
forward over the 61 tree nodes on top of the cache, argmax acceptance, bonus
token, K/V compaction.  Every step replays the same step from the same cached
state (the sequence is rolled back between steps, outside the timed region).

Prints ONE JSON line (rank 0).  `--impl reference` times the float64 CPU
oracle on a bounded sample of the same workload instead.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""

from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "verify steps/s and accepted tokens/s at Llama-3.1-8B shape; % HBM roofline"
UNIT = "verify steps/s"


def workload_config(P=2048, layers=32):
    return {"workload": "llama3.1-8b-shape bf16, batch 1, prefix %d, 60-draft depth-8 tree (widths 10,10,10,8,8,6,4,4),"
                        " planted acceptance p=0.8%s" % (P, "" if layers == 32 else
                                                          " [PROFILING CASE: %d of 32 layers]" % layers),
            "model_shape": "%d layers, d 4096, 32/8 heads x 128, ffn 14336, vocab 128256" % layers,
            "batch": 1, "prefix": P, "tree_nodes": 61, "depth": 8, "accept_p": 0.8,
            "l2": "inputs larger than L2 (15 GB of weights streamed per step)",
            "parallelism": "replicas (one independent verifier per GPU)"}


def measured_traffic(cls, bytes_per_launch):
    """DRAM bytes per launch of kernel class `cls` from the committed ncu record, scaled from the captured
    (smaller) launch to this workload's launch by algorithmic bytes; None when the kernel source changed
    since the capture or there is no record."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get(cls)
    if not rec:
        return None
    src = os.path.join(ROOT, rec["source"])
    if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest()[:16] != rec["source_sha256_prefix"]:
        return None
    return bytes_per_launch * rec["dram_bytes_per_launch_small"] / rec["algorithmic_bytes_small"]


def measured_peaks(sustained=False):
    """(HBM GB/s, bf16 TF/s, source).  The bf16 figure is the burst one for work
    timed in short bursts, the sustained (power-capped) one for long steps."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        tf = j.get("bf16_tflops_sustained") if sustained else None
        return float(j["hbm_gbs"]), float(tf if tf else j["bf16_tflops"]), "measured"
    return 6650.0, 1400.0 if sustained else 1590.0, "fallback"


def step_bytes(d, P, n):
    """Algorithmic bytes of one verification step (bf16): every weight once, the prefix K/V, the tree K/V."""
    per_layer = 2 * (d.q_dim * d.hidden + 2 * d.kv_dim * d.hidden + d.hidden * d.q_dim + 3 * d.ffn * d.hidden)
    weights = d.n_layers * per_layer + 2 * d.vocab * d.hidden
    kv_tok = d.n_layers * 2 * d.kv_dim * 2
    return weights + P * kv_tok + n * kv_tok + n * d.hidden * 2


def class_bytes(d, M, P, n):
    """Algorithmic bytes per step of each kernel class: weights + activations in + outputs.

    gemm_layer is the per-layer launch that runs O, gate/up, down and then the
    next layer's QKV (the LM head after the last layer); gemm_qkv is the first
    layer's QKV.  Activations count once per GEMM: bf16 in, fp32 or bf16 out.
    """
    a = 2  # bf16
    qkv = a * (d.q_dim + 2 * d.kv_dim) * d.hidden + a * M * d.hidden + a * M * (d.q_dim + 2 * d.kv_dim)
    o = a * d.hidden * d.q_dim + a * M * d.q_dim + 4 * M * d.hidden
    gu = a * 2 * d.ffn * d.hidden + a * M * d.hidden + a * M * d.ffn
    down = a * d.hidden * d.ffn + a * M * d.ffn + 4 * M * d.hidden
    lm = a * d.vocab * d.hidden + a * M * d.hidden
    L = d.n_layers
    return {
        "gemm_qkv": qkv,
        "gemm_layer": L * (o + gu + down) + (L - 1) * qkv + lm,
        "attention": L * ((P + n) * d.kv_dim * 2 * a + M * d.q_dim * a * 2),
    }


class ClockSampler:
    """nvidia-smi clock / throttle sampling around the timed region.

    Start it before the warm-up (nvidia-smi needs a moment to come up), mark the
    timed region with begin() / end(); stop() keeps the samples whose timestamp
    falls inside the region (50 ms apart), or the nearest one when the region
    is shorter than the sampling interval."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str, interval_ms: int = 50):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.t0 = self.t1 = None
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", gpu_id, "--query-gpu=" + self.FIELDS,
                                       "--format=csv,noheader,nounits", "-lms", str(interval_ms)],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None
        # a short run can end before nvidia-smi's first sample: wait (at most 5 s) for it
        t_end = time.time() + 5.0
        while self.p is not None and time.time() < t_end and self.p.poll() is None:
            if os.path.getsize(self.f.name) > 0:
                break
            time.sleep(0.02)

    def begin(self):
        self.t0 = time.time()

    def end(self):
        self.t1 = time.time()

    @staticmethod
    def _when(stamp):
        import datetime
        for fmt in ("%Y/%m/%d %H:%M:%S.%f", "%Y/%m/%d %H:%M:%S"):
            try:
                return datetime.datetime.strptime(stamp, fmt).timestamp()
            except ValueError:
                pass
        return None

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except Exception:
            self.p.kill()
        self.f.flush()
        rows = []
        for ln in open(self.f.name):
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) >= 10 and parts[2].replace(".", "").isdigit():
                rows.append((self._when(parts[0]), parts))
        os.unlink(self.f.name)
        if not rows:
            return None
        t0 = self.t0 if self.t0 is not None else -float("inf")
        t1 = self.t1 if self.t1 is not None else float("inf")
        inside = [r for w, r in rows if w is not None and t0 <= w <= t1]
        picked = inside
        if not picked:  # region shorter than the interval: the sample nearest to it
            mid = 0.5 * (t0 + t1) if self.t0 is not None and self.t1 is not None else None
            timed = [(abs(w - mid), r) for w, r in rows if w is not None and mid is not None]
            picked = [min(timed, key=lambda x: x[0])[1]] if timed else [rows[-1][1]]
        sm = [float(r[2]) for r in picked]
        mx = [float(r[3]) for r in picked if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in picked for i in range(4) if r[6 + i].lower().startswith("active")})
        out = {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
               "samples": len(inside)}
        if self.t0 is not None and self.t1 is not None:
            out["window_ms"] = round(1000.0 * (self.t1 - self.t0), 1)
        return out


def gpu_uuid(dev):
    import torch
    try:
        return "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        return str(dev)


# ---------------------------------------------------------------------------
# CPU oracle timing (bounded sample)
# ---------------------------------------------------------------------------

def oracle_step_sample(dims, host_w, P, tokens, parents, n_layers_sample=2, seed=0):
    """Time the float64 oracle's verification step on a bounded sample.

    Sample: `n_layers_sample` of the decoder layers (each over the full tree and
    a P-token prefix cache) plus the LM head over all tree nodes, timed with the
    oracle's own layer and LM-head functions; a full step is extrapolated as
    n_layers x (mean layer time) + LM-head time.  The prefix K/V values are
    seeded random (the oracle's work does not depend on them).
    """
    import oracle
    from oracle.model import OracleModel
    from oracle.tree import tree_meta, ancestor_matrix
    rng = np.random.default_rng(seed)
    om = OracleModel(dims, host_w, cache_limit_bytes=0)
    depth, _ = tree_meta(parents)
    vis = ancestor_matrix(parents)
    x = om.embed(tokens)
    pos = P + depth
    t_layers = []
    t_all0 = time.perf_counter()
    for l in range(n_layers_sample):
        pk = rng.standard_normal((P, dims.n_kv_heads, dims.head_dim))
        pv = rng.standard_normal((P, dims.n_kv_heads, dims.head_dim))
        t0 = time.perf_counter()
        x, _, _ = om.layer_forward(l, x, pos, pk, pv, vis)
        t_layers.append(time.perf_counter() - t0)
    t0 = time.perf_counter()
    logits = om.lm_logits(x)
    amax = np.argmax(logits, axis=1)
    oracle.accept_walk(tokens, parents, amax)
    t_lm = time.perf_counter() - t0
    wall = time.perf_counter() - t_all0
    per_step = dims.n_layers * float(np.mean(t_layers)) + t_lm
    return per_step, wall


def threads_used():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return len(os.sched_getaffinity(0))


def host_sample_weights(wdev, n_layers_sample):
    sub = {"embed": wdev["embed"], "lm_head": wdev["lm_head"], "final_norm": wdev["final_norm"],
           "layers": wdev["layers"][:n_layers_sample]}
    return synth.weights_to_host(sub)


# ---------------------------------------------------------------------------
# reference arm: the oracle
# ---------------------------------------------------------------------------

def run_reference(args, rank, world):
    """The oracle, timed step by step on the host cores: each step is one whole float64 verification
    (32 decoder layers over the 61-node tree on the 2048-token cache, LM head, walk, K/V update) from the
    same cached state, exactly the step our arm times.  Set-up (weights, the oracle's own prefill of the
    prefix, planting the tree with the oracle's argmax) is untimed and reported separately."""
    if rank != 0:
        return 0
    import torch
    import oracle
    from oracle.model import OracleModel
    dims = synth.LLAMA8B
    P = args.prefix
    t_setup = time.perf_counter()
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    w = synth.model_weights(dims, seed=0, device=dev)  # the same seeded weights as our arm
    host = synth.weights_to_host(w)
    del w
    om = OracleModel(dims, host)
    prefix = synth.prefix_tokens(dims.vocab, P, seed=1)
    t0 = time.perf_counter()
    seq, _ = oracle.oracle_prefill(om, prefix)
    prefill_s = time.perf_counter() - t0
    shape = synth.tree_from_widths(synth.TREE60_WIDTHS, stream=0)
    draws = synth.plant_draws(shape.n, dims.vocab, stream=0)
    tokens = synth.plant_tree(shape, seq.pending, 0.8, draws, oracle.argmax_fn_for_planting(om, seq))
    setup_s = time.perf_counter() - t_setup

    def one_step():
        work = dataclasses.replace(seq, k=list(seq.k), v=list(seq.v), tokens=list(seq.tokens))
        return oracle.oracle_verify(om, work, tokens, shape.parents)

    for _ in range(args.warmup):
        one_step()
    times, acc = [], 0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        r = one_step()
        times.append(time.perf_counter() - t0)
        acc = r["accepted_len"]
    ms = 1000.0 * float(np.mean(times))
    v = 1000.0 / ms
    cores = len(os.sched_getaffinity(0))
    sample = ("every step is the whole float64 verification step (32 layers, 61 tree nodes, prefix %d, LM head "
              "over vocab 128256, walk, K/V update) from the same cached state; set-up untimed: %.0f s, of which the "
              "oracle's prefill of the %d-token prefix %.0f s" % (P, setup_s, P, prefill_s))
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(P), "tau": acc + 1, "accepted_tokens_per_s": v * (acc + 1),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores, "threads": threads_used(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

HOLD_NS = 300_000


def hold_stream(stream, ns: int = HOLD_NS):
    """Keep `stream` busy for ~ns (a GPU sleep) before a timed step, so that the step's host-side
    enqueue (argument checks, the parameter block's copy, the graph launch) happens while the
    GPU is still busy: the start event then fires right before the step's first device work,
    and the event pair measures device time only."""
    import torch
    with torch.cuda.stream(stream):
        torch.cuda._sleep(int(ns * 2.0))  # cycles at up to 2 GHz: at least ns


def replica_command(n: int, script: str, argv, port: int):
    """torchrun command for n ranks on one node, one per GPU, over 127.0.0.1."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", str(n),
            "--master-addr", "127.0.0.1", "--master-port", str(port), script] + list(argv)


def run_replicas(n: int, argv, script: str = None, timeout_s: int = 1800) -> int:
    """Launch n ranks of `script` (default: this file) with the same arguments and return the
    launcher's exit status; rank 0's JSON line passes through on stdout."""
    import socket
    sk = socket.socket()
    sk.bind(("127.0.0.1", 0))
    port = sk.getsockname()[1]
    sk.close()
    cmd = replica_command(n, script or os.path.abspath(__file__), argv, port)
    env = dict(os.environ)
    env.setdefault("NCCL_NVLS_ENABLE", "0")  # the replicas exchange one float per job: no switch reductions
    return subprocess.run(cmd, env=env, timeout=timeout_s).returncode


def max_over_ranks(value: float, dist=None, device=None) -> float:
    """The largest `value` over all ranks (every rank calls it, in the same order)."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, steps: int, t_total_ms: float) -> float:
    """Whole-job steps per second: every rank ran `steps` steps; the job took the slowest rank's time."""
    return world * steps / (t_total_ms / 1000.0)


def run_ours(args, rank, world, local_rank):
    import torch
    from speculative_decoding_06_b200.engine import SpecEngine, pack_trees
    from speculative_decoding_06_b200 import spec as S

    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local_rank))
    dims = dataclasses.replace(synth.LLAMA8B, n_layers=args.layers)
    P = args.prefix
    w = synth.model_weights(dims, seed=0, device="cuda")
    eng = SpecEngine(dims, w, max_batch=1, max_seq=P + 256, max_nodes=64)
    if args.temperature > 0:
        eng.set_sampling(args.temperature, 1)  # tokens are draws at temperature T (planting included)
    prefix = synth.prefix_tokens(dims.vocab, P, seed=1)
    pend = eng.prefill(0, prefix)
    shape = synth.tree_from_widths(synth.TREE60_WIDTHS, stream=0)
    draws = synth.plant_draws(shape.n, dims.vocab, stream=0)

    def gpu_argmax(tokens, parents):
        return eng.score([0], [(tokens, parents)])[0]

    tokens = synth.plant_tree(shape, pend, 0.8, draws, gpu_argmax)
    tk, pr, off = pack_trees([(tokens, shape.parents)])
    ids = np.array([0], np.int32)
    acc_dev = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = eng.stream  # the library's stream: events must be recorded where its kernels run

    def one_step():
        eng.verify_batch_device(ids, tk, pr, off, outputs=(acc_dev, None, None, None))

    # warm-up (also captures the CUDA graph)
    clk = ClockSampler(gpu_uuid(local_rank))
    for _ in range(max(3, args.warmup)):
        one_step()
        eng.sync()
        eng.truncate(0, P)
    a_len, _, _ = eng.verify(0, tokens, shape.parents)
    eng.truncate(0, P)
    launches = eng.step_launches()

    # ---- timed region: K steps, device time from CUDA events on the launching stream
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    clk.begin()
    times = []
    for _ in range(args.steps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        torch.cuda.nvtx.range_push("timed_step")
        hold_stream(stream)
        e0.record(stream)
        one_step()
        e1.record(stream)
        torch.cuda.nvtx.range_pop()
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
        eng.sync()
        eng.truncate(0, P)
    torch.cuda.synchronize()
    clk.end()
    if dist:
        dist.barrier()
    clocks = clk.stop()
    t_total = max_over_ranks(float(sum(times)), dist, "cuda")
    ms = t_total / args.steps
    value = job_throughput(world, args.steps, t_total)

    # ---- end to end through the public API with host buffers (H2D + D2H inside)
    e2e_times = []
    for _ in range(args.steps):
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        eng.verify(0, tokens, shape.parents)
        e2e_times.append(time.perf_counter() - t0)
        eng.truncate(0, P)
    h2d, d2h = eng.io_bytes()
    e2e_value = world / max_over_ranks(float(np.mean(e2e_times)), dist, "cuda")

    # ---- per-kernel-class device time (event pair per launch, launch by launch)
    eng.profile(True)
    nprof = 3
    for _ in range(nprof):
        eng.verify_batch_device(ids, tk, pr, off)
        eng.sync()
        eng.truncate(0, P)
    prof = eng.profile_read()
    eng.profile(False)
    hbm, tflops, peak_kind = measured_peaks()
    M = shape.n
    cb = class_bytes(dims, M, P, shape.n)
    dom = max(cb, key=lambda k: prof[k][0])
    dom_ms, dom_n = prof[dom]
    dom_ms /= nprof  # per step
    dom_n = max(1, dom_n // nprof)
    achieved = cb[dom] / (dom_ms / 1000.0) / 1e9
    sb = step_bytes(dims, P, shape.n)
    step_gbs = sb / (ms / 1000.0) / 1e9
    kernel_share = {k: round(v[0] / nprof, 4) for k, v in prof.items()}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (random-init weights, uniform prefix, planted tree)",
        "config": dict(workload_config(P, args.layers), **({"temperature": args.temperature}
                                                           if args.temperature > 0 else {})),
        "accepted_tokens_per_s": value * (a_len + 1), "tau": a_len + 1,
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "traffic": measured_traffic(dom, cb[dom] / dom_n),
                     "traffic_source": "profiles/traffic.json (ncu dram__bytes_read+write, scaled by algorithmic bytes)",
                     "peak_source": peak_kind,
                     "bytes_per_launch": cb[dom] / dom_n, "launches_per_step": dom_n,
                     "ms_per_launch": dom_ms / dom_n},
        "step_roofline": {"bound": "hbm", "bytes_per_step": sb, "achieved": step_gbs, "peak": hbm, "unit": "GB/s",
                          "frac": step_gbs / hbm, "roofline_ms": sb / hbm / 1e6},
        "kernel_ms_per_step": kernel_share,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches * args.steps,
        "plan": eng.info(1, shape.n, P),
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.layers == 32:
        hostw = host_sample_weights(w, args.sample_layers)
        # repeat the bounded sample until about 10 s of CPU work have run (at most 12 repeats)
        per, wall, reps = [], 0.0, 0
        while (wall < 10.0 and reps < 12) or reps == 0:
            p_, w_ = oracle_step_sample(dims, hostw, P, tokens, shape.parents, args.sample_layers, seed=reps)
            per.append(p_)
            wall += w_
            reps += 1
        per_step = float(np.mean(per))
        line["cpu_baseline"] = {"value": 1.0 / per_step, "unit": UNIT, "cores": len(os.sched_getaffinity(0)),
                                "threads": threads_used(), "kind": "oracle",
                                "sample": "%d of 32 decoder layers (61-node tree, prefix %d) + LM head, extrapolated"
                                          " to 32 layers, repeated %d times; %.1f s of CPU work"
                                          % (args.sample_layers, P, reps, wall)}
    if rank == 0:
        print(json.dumps(line))
    eng.close()
    if dist:
        dist.destroy_process_group()
    return 0


# ---------------------------------------------------------------------------
# the other configurations of the pages' workload list (one JSON line each;
# the default line above stays the batch-1 verification step)
# ---------------------------------------------------------------------------

def flops_per_token(d):
    """Dense multiply-adds x 2 per token through every weight matrix (attention scores excluded)."""
    per_layer = d.q_dim * d.hidden + 2 * d.kv_dim * d.hidden + d.hidden * d.q_dim + 3 * d.ffn * d.hidden
    return 2 * (d.n_layers * per_layer + d.vocab * d.hidden)


def attn_flops(d, rows_keys, layers):
    """QK and PV: 4 * head_dim flops per (query head, node, visible key) per layer; rows_keys = sum over
    nodes of their visible keys."""
    return 4 * d.head_dim * d.n_q_heads * rows_keys * layers


def _timed(stream, fn, steps, reset):
    import torch
    times = []
    for _ in range(steps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        torch.cuda.nvtx.range_push("timed_step")
        hold_stream(stream)
        e0.record(stream)
        fn()
        e1.record(stream)
        torch.cuda.nvtx.range_pop()
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
        reset()
    return float(np.mean(times))


def _roofline(bytes_, flops, ms, sustained=False):
    hbm, tflops, kind = measured_peaks(sustained)
    t_mem = bytes_ / hbm / 1e6
    t_fl = flops / tflops / 1e9
    bound = "hbm" if t_mem >= t_fl else "tensor"
    return {"bound": bound, "bytes": bytes_, "flops": flops, "roofline_ms": max(t_mem, t_fl),
            "frac": max(t_mem, t_fl) / ms, "hbm_gbs": hbm, "bf16_tflops": tflops, "peak_source": kind}


def run_batch64(args):
    """64 sequences, prefixes uniform in [512, 4096], each with its own 60-draft tree, p uniform in [0.6, 0.9]."""
    import torch
    from speculative_decoding_06_b200.engine import SpecEngine, pack_trees
    dims = dataclasses.replace(synth.LLAMA8B, n_layers=args.layers)
    B = 64
    lens, ps = synth.batch_prefix_lengths_and_p(B)
    w = synth.model_weights(dims, seed=0, device="cuda")
    eng = SpecEngine(dims, w, max_batch=B, max_seq=int(lens.max()) + 64, max_nodes=64)
    trees = []
    for b in range(B):
        pend = eng.prefill(b, synth.prefix_tokens(dims.vocab, int(lens[b]), stream=b))
        sh = synth.tree_from_widths(synth.TREE60_WIDTHS, stream=b)
        draws = synth.plant_draws(sh.n, dims.vocab, stream=b)
        toks = synth.plant_tree(sh, pend, float(ps[b]), draws,
                                lambda t, p_, b=b: eng.score([b], [(t, p_)])[0])
        trees.append((toks, sh.parents))
    tk, pr, off = pack_trees(trees)
    ids = np.arange(B, dtype=np.int32)
    acc = torch.zeros(B, dtype=torch.int32, device="cuda")

    def reset():
        eng.sync()
        for b in range(B):
            eng.truncate(b, int(lens[b]))

    clk = ClockSampler(gpu_uuid(0))
    for _ in range(max(3, args.warmup)):
        eng.verify_batch_device(ids, tk, pr, off, outputs=(acc, None, None, None))
        reset()
    a_len = eng.verify_batch(list(range(B)), trees)[0]
    reset()
    clk.begin()
    ms = _timed(eng.stream, lambda: eng.verify_batch_device(ids, tk, pr, off, outputs=(acc, None, None, None)),
                args.steps, reset)
    clk.end()
    clocks = clk.stop()
    eng.profile(True)
    eng.verify_batch_device(ids, tk, pr, off)
    reset()
    prof = {k: round(v[0], 3) for k, v in eng.profile_read().items() if v[1]}
    eng.profile(False)
    M = int(off[-1])
    kv_tok = dims.n_layers * 2 * dims.kv_dim * 2
    bytes_ = step_bytes(dims, 0, 0) + int(lens.sum() + M) * kv_tok
    rk = sum(int(lens[b]) * 61 + 61 * 5 for b in range(B))  # prefix keys per node + ~ancestors
    fl = flops_per_token(dims) * M + attn_flops(dims, rk, dims.n_layers)
    tau = float(np.mean(a_len + 1))
    print(json.dumps({"layers": dims.n_layers,
                      "workload": "llama3.1-8b-shape bf16, batch 64, prefixes U[512,4096], own 60-draft trees,"
                                  " planted p U[0.6,0.9]", "tokens_per_step": M, "ms_per_step": ms,
                      "verify_steps_per_s": 1000.0 / ms, "accepted_tokens_per_s": float(np.sum(a_len + 1)) * 1000.0 / ms,
                      "tau_mean": tau, "roofline": _roofline(bytes_, fl, ms, sustained=True), "kernel_ms_per_step": prof,
                      "plan": eng.info(B, 61, int(lens.max())),
                      "clocks": clocks, "data": "synthetic"}))
    eng.close()
    return 0


def run_sweep(args):
    """Chain-vs-tree sweep at prefix 8192, batch 1, planted p = 0.85."""
    import torch
    from speculative_decoding_06_b200.engine import SpecEngine, pack_trees
    dims = synth.LLAMA8B
    P = 8192
    w = synth.model_weights(dims, seed=0, device="cuda")
    eng = SpecEngine(dims, w, max_batch=1, max_seq=P + 128, max_nodes=128)
    pend = eng.prefill(0, synth.prefix_tokens(dims.vocab, P, seed=1))
    shapes = [("chain5", synth.chain(5)), ("chain8", synth.chain(8))]
    shapes += [("tree%d" % n, synth.tree_from_widths(synth.SWEEP_WIDTHS[n], stream=0)) for n in (16, 32, 60, 80)]
    kv_tok = dims.n_layers * 2 * dims.kv_dim * 2
    out = []
    clk = ClockSampler(gpu_uuid(0))
    time.sleep(0.2)
    clk.begin()
    for name, sh in shapes:
        draws = synth.plant_draws(sh.n, dims.vocab, stream=0)
        toks = synth.plant_tree(sh, pend, 0.85, draws, lambda t, p_: eng.score([0], [(t, p_)])[0])
        tk, pr, off = pack_trees([(toks, sh.parents)])
        ids = np.zeros(1, np.int32)

        def reset():
            eng.sync()
            eng.truncate(0, P)

        for _ in range(max(3, args.warmup)):
            eng.verify_batch_device(ids, tk, pr, off)
            reset()
        a, _, _ = eng.verify(0, toks, sh.parents)
        reset()
        ms = _timed(eng.stream, lambda: eng.verify_batch_device(ids, tk, pr, off), args.steps, reset)
        # per-kernel time of one step (launches serialised by the profiler's events)
        eng.profile(True)
        eng.verify_batch_device(ids, tk, pr, off)
        reset()
        prof = {k: round(v[0], 3) for k, v in eng.profile_read().items() if v[1]}
        eng.profile(False)
        bytes_ = step_bytes(dims, P, sh.n)
        fl = flops_per_token(dims) * sh.n + attn_flops(dims, P * sh.n, dims.n_layers)
        out.append({"draft": name, "nodes": sh.n, "ms_per_step": ms, "tau": a + 1,
                    "accepted_tokens_per_s": (a + 1) * 1000.0 / ms, "roofline_frac": _roofline(bytes_, fl, ms)["frac"],
                    "kernel_ms_per_step": prof})
    clk.end()
    clocks = clk.stop()
    print(json.dumps({"workload": "llama3.1-8b-shape bf16, batch 1, prefix 8192, chains 5/8 and trees 16/32/60/80"
                                  " at depth 8, planted p=0.85", "results": out, "clocks": clocks, "data": "synthetic"}))
    eng.close()
    return 0


def reduce_draft_vocab(dw, w, vocab, n):
    """Give the draft head a reduced vocabulary of n seeded token ids (the target's LM-head rows of them)."""
    import torch
    if n:
        dw["vocab_ids"] = torch.as_tensor(synth.draft_vocab_ids(vocab, n), device="cuda")
        dw["lm_head"] = w["lm_head"][dw["vocab_ids"].long()].contiguous()
    return dw


def run_draft(args):
    """Draft-head step: batch 16, 60-draft trees, draft prefixes of 2048 rows, N(0,1) features."""
    import torch
    from speculative_decoding_06_b200.engine import SpecEngine, pack_trees
    dims = synth.LLAMA8B
    B, P = 16, 2048
    w = synth.model_weights(dims, seed=0, device="cuda")
    dw = reduce_draft_vocab(synth.draft_head_weights(dims, seed=6, device="cuda"), w, dims.vocab, args.draft_vocab)
    eng = SpecEngine(dims, w, max_batch=B, max_seq=P + 64, max_nodes=64, draft=dw)
    rng = np.random.default_rng(5)
    for b in range(B):
        f = synth.draft_features(P, dims.hidden, seed=100 + b, device="cuda")
        eng.draft_prefill(b, f, rng.integers(0, dims.vocab, size=P).astype(np.int32))
    trees = []
    for b in range(B):
        sh = synth.tree_from_widths(synth.TREE60_WIDTHS, stream=b)
        trees.append((rng.integers(0, dims.vocab, size=sh.n).astype(np.int32), sh.parents))
    tk, pr, off = pack_trees(trees)
    M = int(off[-1])
    feats = synth.draft_features(M, dims.hidden, seed=5, device="cuda")
    ids = np.arange(B, dtype=np.int32)
    ti = torch.zeros(M, 10, dtype=torch.int32, device="cuda")
    tv = torch.zeros(M, 10, dtype=torch.float32, device="cuda")
    step = lambda: eng.draft_step_device(ids, feats, tk, pr, off, outputs=(ti, tv))
    clk = ClockSampler(gpu_uuid(0))
    for _ in range(max(3, args.warmup)):
        step()
        eng.sync()
    clk.begin()
    ms = _timed(eng.stream, step, args.steps, lambda: None)
    clk.end()
    clocks = clk.stop()
    eng.profile(True)
    step()
    eng.sync()
    prof = {k: round(v[0], 3) for k, v in eng.profile_read().items() if v[1]}
    eng.profile(False)
    d = dims
    Vd = args.draft_vocab or d.vocab
    layer = d.q_dim * d.hidden + 2 * d.kv_dim * d.hidden + d.hidden * d.q_dim + 3 * d.ffn * d.hidden
    params = 3 * d.hidden * d.hidden + 2 * d.hidden * d.hidden + layer + Vd * d.hidden
    kv_tok = 2 * d.kv_dim * 2
    bytes_ = 2 * params + B * (P + 61) * kv_tok + M * 3 * d.hidden * 2
    fl = 2 * params * M + attn_flops(d, P * M, 1)
    print(json.dumps({"workload": "EAGLE-3 draft head at 8B shape bf16: batch 16, 60-draft trees, draft prefix 2048,"
                                  " N(0,1) low/mid/high features, fusion FC + input FC + one tree-masked decoder layer"
                                  " + LM head + top-10" + (" over a reduced draft vocabulary of %d tokens" % Vd
                                                           if args.draft_vocab else ""), "tokens_per_step": M, "ms_per_step": ms,
                      "draft_steps_per_s": 1000.0 / ms, "roofline": _roofline(bytes_, fl, ms),
                      "kernel_ms_per_step": prof, "plan": eng.info(B, 61, P), "clocks": clocks,
                      "data": "synthetic"}))
    eng.close()
    return 0


def run_draft_tree(args):
    """Dynamic draft tree: batch 16, draft prefixes of 2048 rows, 8 drafting steps, top-10, 60 nodes."""
    import torch
    from speculative_decoding_06_b200.engine import SpecEngine
    dims = synth.LLAMA8B
    B, P, steps, K, total = 16, 2048, 8, 10, 60
    w = synth.model_weights(dims, seed=0, device="cuda")
    dw = reduce_draft_vocab(synth.draft_head_weights(dims, seed=6, device="cuda"), w, dims.vocab, args.draft_vocab)
    eng = SpecEngine(dims, w, max_batch=B, max_seq=P + 128, max_nodes=128, draft=dw)
    rng = np.random.default_rng(5)
    for b in range(B):
        f = synth.draft_features(P, dims.hidden, seed=100 + b, device="cuda")
        eng.draft_prefill(b, f, rng.integers(0, dims.vocab, size=P).astype(np.int32))
    root_feats = synth.draft_features(B, dims.hidden, seed=7, device="cuda")
    roots = rng.integers(0, dims.vocab, size=B).astype(np.int32)
    ids = list(range(B))
    step = lambda: eng.draft_tree(ids, root_feats, roots, steps=steps, topk=K, total=total)
    clk = ClockSampler(gpu_uuid(0))
    for _ in range(max(3, args.warmup)):
        step()
    clk.begin()
    ms = _timed(eng.stream, step, args.steps, lambda: None)
    clk.end()
    clocks = clk.stop()
    eng.profile(True)
    step()
    prof = {k: round(v[0], 3) for k, v in eng.profile_read().items() if v[1]}
    eng.profile(False)
    d = dims
    layer = d.q_dim * d.hidden + 2 * d.kv_dim * d.hidden + d.hidden * d.q_dim + 3 * d.ffn * d.hidden
    per_step = 2 * d.hidden * d.hidden + layer + (args.draft_vocab or d.vocab) * d.hidden  # input FC, layer, LM head
    hbm, tflops, kind = measured_peaks()
    roof = 0.0
    fl_all = 0.0
    for t in range(steps):
        M = B * (1 + t * K)  # every step recomputes the tree built so far
        fl = 2.0 * per_step * M + (2.0 * 3 * d.hidden * d.hidden * B if t == 0 else 0.0) + attn_flops(d, P * M, 1)
        by = 2.0 * per_step + B * (P + M // B) * 2 * d.kv_dim * 2
        roof += max(by / hbm / 1e6, fl / tflops / 1e9)
        fl_all += fl
    print(json.dumps({"workload": "EAGLE-3 dynamic draft tree at 8B shape bf16: batch 16, draft prefix 2048, "
                                  "8 drafting steps, top-10 offers, 60 nodes (every step recomputes the tree so far)"
                                  + (", reduced draft vocabulary of %d tokens" % args.draft_vocab
                                     if args.draft_vocab else ""),
                      "ms_per_tree_batch": ms, "trees_per_s": B * 1000.0 / ms,
                      "roofline": {"bound": "per step: max(hbm, tensor)", "roofline_ms": roof, "frac": roof / ms,
                                   "flops": fl_all, "hbm_gbs": hbm, "bf16_tflops": tflops, "peak_source": kind},
                      "kernel_ms_per_tree_batch": prof, "clocks": clocks, "data": "synthetic"}))
    eng.close()
    return 0


def run_decode(args):
    """The closed loop at the 8B shape, prefix 2048, `--batch` sequences: per step one dynamic
    draft tree per sequence (8 steps of top-10, 60 nodes), their verification with features,
    the draft-prefix updates."""
    import torch
    from speculative_decoding_06_b200.engine import SpecEngine
    dims = synth.LLAMA8B
    P, steps, K, total = 2048, 8, 10, 60
    n_steps = args.steps + max(3, args.warmup)
    w = synth.model_weights(dims, seed=0, device="cuda")
    dw = synth.draft_head_weights(dims, seed=6, device="cuda")
    L = dims.n_layers
    B = args.batch
    eng = SpecEngine(dims, w, max_batch=B, max_seq=P + 64 * (n_steps + 2), max_nodes=128, draft=dw,
                     feature_layers=(2, L // 2, L - 3))
    ids = list(range(B))
    pend, last = [], []
    for b in ids:
        prompt = synth.prefix_tokens(dims.vocab, P, seed=1, stream=b)
        pb, feats = eng.prefill_features(b, prompt)
        eng.draft_prefill(b, feats[:P - 1], prompt[1:])
        pend.append(pb)
        last.append(feats[P - 1:P].clone())
    times, accs = [], []
    clk = ClockSampler(gpu_uuid(0))
    for i in range(n_steps):
        if i == max(3, args.warmup):
            clk.begin()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        timed = i >= max(3, args.warmup)
        if timed:
            torch.cuda.nvtx.range_push("timed_step")
        e0.record(eng.stream)
        tok, par, _ = eng.draft_tree(ids, torch.cat(last, dim=0), pend, steps=steps, topk=K, total=total)
        acc_len, _, acc_tok, bonus, F = eng.verify_batch(ids, [(tok[b], par[b]) for b in ids], features=True)
        for b in ids:
            a = int(acc_len[b])
            acc = [int(x) for x in acc_tok[b, :a]]
            eng.draft_append(b, torch.cat([last[b], F[b, :a]], dim=0), [pend[b]] + acc)
            last[b] = F[b, a:a + 1].clone()
            pend[b] = int(bonus[b])
        a = float(np.mean(acc_len[:B]))
        e1.record(eng.stream)
        if timed:
            torch.cuda.nvtx.range_pop()
        e1.synchronize()
        if timed:
            times.append(e0.elapsed_time(e1))
            accs.append(a)
    clk.end()
    clocks = clk.stop()
    ms = float(np.mean(times))
    tau = float(np.mean(accs)) + 1.0
    print(json.dumps({"workload": "EAGLE-3 greedy decoding loop at 8B shape bf16, batch %d, prefix 2048: dynamic "
                                  "draft tree (8 steps, top-10, 60 nodes) per sequence + verification with features + "
                                  "draft-prefix update per step; random-init draft head, so few drafts are "
                                  "accepted" % B,
                      "batch": B, "ms_per_decode_step": ms, "tau": tau, "tokens_per_s": B * tau * 1000.0 / ms,
                      "steps": len(times), "clocks": clocks,
                      "data": "synthetic"}))
    eng.close()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--prefix", type=int, default=2048)
    ap.add_argument("--sample-layers", type=int, default=2)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=1, help="sequences decoded together (--workload decode)")
    ap.add_argument("--draft-vocab", type=int, default=0,
                    help="draft / draft_tree workloads: a reduced draft vocabulary of this many seeded token ids")
    ap.add_argument("--temperature", type=float, default=0.0,
                    help="verify workload: sample at this temperature instead of greedy choices (0: greedy)")
    ap.add_argument("--layers", type=int, default=32, help="decoder layers (32 = the 8B shape; fewer only for profiling)")
    ap.add_argument("--workload", default="verify", choices=["verify", "batch64", "sweep", "draft", "draft_tree", "decode"],
                    help="verify: the default line (batch 1, prefix 2048); the others measure the remaining"
                         " configurations (one GPU, one JSON line each)")
    args = ap.parse_args()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # N GPUs without a launcher: start N ranks (one replica per GPU) through torchrun
        return run_replicas(args.gpus, sys.argv[1:])
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.workload != "verify":
        import torch
        torch.cuda.set_device(local_rank)
        return {"batch64": run_batch64, "sweep": run_sweep, "draft": run_draft,
                "draft_tree": run_draft_tree, "decode": run_decode}[args.workload](args)
    return run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    sys.exit(main())

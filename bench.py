#!/usr/bin/env python
"""Throughput of the block-diffusion draft step + greedy verification.

One step = the whole hot path over one batch of seeded synthetic inputs:
fusion of the target states of every context row for every draft layer,
context K/V projection into the caches, D draft layers over the block(s),
final norm, LM-head argmax and acceptance against planted target tokens
(for the D2SD workload: first draft, lowest-confidence cuts, batched
re-anchored second draft over K candidates, acceptance).

    python bench.py [--gpus N --steps K --warmup W] [--config qwen3_4b]
                    [--mode full|steady] [--impl ours|reference]

Prints one JSON line (rank 0).  Under torchrun every rank runs an
independent replica of the workload (requests are independent units, so
there is no data-path collective); time is the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
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

METRIC = "draft blocks/s and accepted tok/s per B200; HBM GB/s / tensor util vs peak"
ACCEPT_DRAWS = 32          # planted target draws averaged for accepted tok/s
# DRAM bytes (read + write) of one LM-head launch from an ncu capture of
# `bench.py --op lmhead` (summarised under profiles/), valid only for the
# GEMM code it was taken with (digest of gemm.cu without comments); any
# later change of that code nulls it.
LMHEAD_TRAFFIC = {         # workload -> {"bytes": int, "gemm_cu_sha256": str}
    "qwen3_4b": {"bytes": 785283584, "gemm_cu_sha256": "c631e555a25cd81b"},
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="qwen3_4b")
    ap.add_argument("--mode", choices=["full", "steady"], default="full")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch the step eagerly instead of replaying a CUDA graph")
    ap.add_argument("--profile", action="store_true",
                    help="eager steps inside an NVTX range 'dflash_step' (for ncu launch lists)")
    ap.add_argument("--op", choices=["lmhead", "mlp", "ctxproj", "attn", "fuse"],
                    help="time one entry point alone at the workload's shapes")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), \
            d.get("bf16_tflops_sustained", 1400.0), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------- clocks
class Clocks:
    """nvidia-smi sampling in the background (read-only queries)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None
        self.t_marks = {}

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu=timestamp,{self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def mark(self, name):
        self.t_marks[name] = time.time()

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(parts[2]), float(parts[3]), parts[5:10]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        t0 = self.t_marks.get("timed_start", 0)
        t1 = self.t_marks.get("timed_end", 1e30)
        inside = [r for r in rows if t0 - 0.05 <= r[0] <= t1 + 0.05]
        window = "timed"
        if len(inside) < 3:
            w0 = self.t_marks.get("warm_start", t0)
            inside = [r for r in rows if w0 - 0.05 <= r[0] <= t1 + 0.05]
            window = "warmup+timed"
        if not inside:
            inside = rows
            window = "run"
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in inside for i, v in enumerate(r[3][1:])
                          if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in inside),
                "sm_max_mhz": max(r[2] for r in inside), "reasons": reasons,
                "samples": len(inside), "window": window}


# ---------------------------------------------------------------- distributed
def dist_init(backend: str = "nccl"):
    """One process per GPU (torchrun env).  Returns (rank, world, local_rank)."""
    import torch
    import torch.distributed as dist
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws > 1:
        lr = int(os.environ.get("LOCAL_RANK", "0"))
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(lr)
            kw["device_id"] = torch.device("cuda", lr)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
        return dist.get_rank(), ws, lr
    return 0, 1, 0


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """Every rank gets the maximum of x over ranks (one all-reduce)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------- oracle timing
def oracle_sample(cfg, seed, max_seconds=30.0):
    """Time the CPU oracle on one block of the workload (the request with the
    median context length): one full draft step plus acceptance."""
    from block_diffusion_speculative_softmax_b200 import synth
    from oracle import dflash_oracle as O
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:   # pragma: no cover
        threads = os.cpu_count() or 1
    w = synth.make_weights(cfg, seed)
    lens = synth.ctx_lengths(cfg, seed)
    r = int(np.argsort(lens)[len(lens) // 2])
    st = synth.make_states(cfg, seed, r, lens[r])
    anchor = int(synth.make_anchors(cfg, seed)[r])
    blk = O.Block(r, [anchor] + [0] * (cfg.block - 1), 1)
    times = []
    t_start = time.perf_counter()
    while True:
        t0 = time.perf_counter()
        tok, _ = O.draft_step(cfg, w, {r: st}, [blk], bf16_storage=(cfg.dtype == "bf16"))
        rng = np.random.default_rng(1)
        n = synth.geometric_lengths(cfg.accept_p, 1, cfg.block - 1, rng)
        t = synth.plant_targets(tok, n, cfg.vocab, rng)
        O.accept(tok[:, None, :], t[:, None, :])
        times.append(time.perf_counter() - t0)
        if time.perf_counter() - t_start > max_seconds * 0.5 or len(times) >= 3:
            break
    sec = statistics.median(times)
    return {"value": 1.0 / sec, "unit": "blocks/s", "cores": threads, "kind": "oracle",
            "sample": f"{len(times)} oracle step(s) on 1 block (request {r}, L={lens[r]}) of "
                      f"{cfg.name}: fuse + ctx K/V projection + {cfg.n_draft_layers} layers + "
                      f"LM head argmax + accept, NumPy float64; median {sec:.2f} s/step",
            "host_cpus": os.cpu_count()}


def run_reference(args):
    """The oracle as the reference arm (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from block_diffusion_speculative_softmax_b200 import synth
    cfg = synth.get_config(args.config)
    budget = 150.0
    first = oracle_sample(cfg, args.seed, max_seconds=0.0)       # one step (+ warm-up)
    per = 1.0 / first["value"]
    k = max(1, min(args.steps, int(budget / max(per, 1e-3))))
    t0 = time.perf_counter()
    vals = []
    for _ in range(k):
        vals.append(oracle_sample(cfg, args.seed, max_seconds=0.0)["value"])
    el = time.perf_counter() - t0
    v = statistics.median(vals)
    line = {"metric": METRIC, "value": v, "unit": "blocks/s", "n_gpus": args.gpus,
            "steps": k, "warmup": 1, "ms_per_step": 1000.0 / v, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": cfg.name, "mode": args.mode, "batch_blocks": 1,
                       "note": "CPU oracle on one block per step"},
            "cpu_baseline": {"value": v, "unit": "blocks/s", "cores": first["cores"],
                             "kind": "oracle", "sample": first["sample"] +
                             f"; {k} steps in {el:.1f} s"},
            "e2e": {"value": v, "unit": "blocks/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- our arm
def run_ours(args):
    import torch
    rank, world, lr = dist_init("nccl")
    from block_diffusion_speculative_softmax_b200 import build as B
    if rank == 0:
        B.build()
    barrier(world)
    from block_diffusion_speculative_softmax_b200 import dflash as DF
    from block_diffusion_speculative_softmax_b200 import synth, workload
    DF.load()
    cfg = synth.get_config(args.config)
    hbm_peak, tf_burst, tf_sust, peak_src = load_peaks()

    wl = workload.Workload(cfg, seed=args.seed + rank, mode=args.mode)
    # pass once, plant target tokens against the drafted blocks
    wl.step(verify=False)
    torch.cuda.synchronize()
    n_plant = wl.plant_targets()
    stream = torch.cuda.Stream()
    clocks = Clocks(torch.cuda.current_device())
    clocks.start()
    clocks.mark("warm_start")
    with torch.cuda.stream(stream):
        wl.step(verify=True)
    stream.synchronize()
    wl.check()
    c0 = DF.dflash_launch_count()
    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            wl.step(verify=True)
    else:
        with torch.cuda.stream(stream):
            wl.step(verify=True)
    launches_per_step = DF.dflash_launch_count() - c0

    def one_step():
        if graph is not None:
            graph.replay()
        else:
            wl.step(verify=True)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            one_step()
    stream.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    clocks.mark("timed_start")
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for _ in range(args.steps):
            one_step()
        ev1.record(stream)
    ev1.synchronize()
    clocks.mark("timed_end")
    torch.cuda.synchronize()
    barrier(world)
    ms = ev0.elapsed_time(ev1) / args.steps
    ms = max_over_ranks(ms, world)
    wl.check()
    fb = wl.final_buf
    n_acc = fb.n_acc.cpu().numpy()
    assert (n_acc == n_plant).all() or wl.K > 1, "accept lengths differ from the planted ones"
    blocks_per_step = fb.nb
    # The step's work does not depend on the targets, so the accepted tokens
    # per step are averaged over several planted draws (each run through
    # verification on the GPU, and checked) rather than the single draw the
    # timed steps used.
    tok_draws = [int((n_acc + 1).sum())]
    for draw in range(1, ACCEPT_DRAWS):
        n_pl = wl.plant_targets(seed_offset=draw)
        with torch.cuda.stream(stream):
            wl.step(verify=True)
        stream.synchronize()
        wl.check()
        na = fb.n_acc.cpu().numpy()
        assert (na == n_pl).all() or wl.K > 1, "accept lengths differ from the planted ones"
        tok_draws.append(int((na + 1).sum()))
    tok_per_step = float(np.mean(tok_draws))
    value = blocks_per_step * world / (ms / 1e3)
    acc_tok_s = tok_per_step * world / (ms / 1e3)
    # accepted draft tokens only (sum of n, without the bonus token)
    acc_draft_tok_s = (tok_per_step - wl.R) * world / (ms / 1e3)

    # ---- roofline of the dominant kernel, timed alone on its own stream
    roof = roofline(args, wl, cfg, DF, hbm_peak, tf_burst, peak_src, stream)
    clk = clocks.stop()

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        e2e = end_to_end(args, wl, DF, stream, world, blocks_per_step)

    used_graph = graph is not None
    if graph is not None:
        del graph
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_sample(cfg, args.seed)
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "blocks/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if cfg.dtype == "bf16" else "fp32", "data": "synthetic",
            "accepted_tok_s": acc_tok_s, "accepted_draft_tok_s": acc_draft_tok_s,
            "mean_accept_tau": tok_per_step / wl.R,
            "accept_draws": len(tok_draws),
            "config": {"workload": cfg.name, "mode": args.mode, "n_req": cfg.n_req,
                       "blocks_per_step": blocks_per_step, "block": cfg.block,
                       "ctx_len": cfg.ctx_len if cfg.ctx_len_min == 0 else
                       f"U[{cfg.ctx_len_min},{cfg.ctx_len}]",
                       "draft_layers": cfg.n_draft_layers, "target_layers": cfg.n_target_layers,
                       "hidden": cfg.hidden, "vocab": cfg.vocab,
                       "parallelism": f"replicas{world}",
                       "cuda_graph": used_graph,
                       "l2": "inputs larger than L2 (weights %.2f GB streamed per step)"
                             % (wl.w.nbytes() / 1e9)},
            "gpu_launches": launches_per_step * args.steps,
            "launches_per_step": launches_per_step,
            "roofline": roof,
            "clocks": clk,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def code_digest(text):
    """sha256 of C/C++ source with comments removed and whitespace collapsed,
    so only a change of the code itself changes it."""
    import hashlib
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return hashlib.sha256(" ".join(text.split()).encode()).hexdigest()


def gemm_source_digest():
    src = os.path.join(ROOT, "block_diffusion_speculative_softmax_b200", "csrc", "gemm.cu")
    with open(src) as f:
        return code_digest(f.read())


def lmhead_traffic(workload):
    """Measured DRAM bytes per LM-head launch, or None when there is no
    capture for this workload or the GEMM code changed since."""
    ent = LMHEAD_TRAFFIC.get(workload)
    if ent is None:
        return None
    return ent["bytes"] if gemm_source_digest().startswith(ent["gemm_cu_sha256"]) else None


def roofline(args, wl, cfg, DF, hbm_peak, tf_burst, peak_src, stream):
    """LM-head argmax (weight streaming, the largest single launch of the
    step), timed alone with CUDA events on its launch stream."""
    import torch
    M = wl.final_buf.nb * cfg.block
    H, V = cfg.hidden, cfg.vocab
    x = torch.randn(M, H, device="cuda").to(wl.dt)
    tok = torch.empty(M, dtype=torch.int32, device="cuda")
    ws = DF.alloc_workspace(DF.dflash_workspace_size(wl.ccfg, 1, wl.final_buf.nb, 0, 0))
    reps = max(10, min(200, args.steps))
    with torch.cuda.stream(stream):
        for _ in range(3):
            DF.dflash_lmhead_argmax(wl.ccfg, x, wl.w.lm_head, tok, None, ws, stream=stream)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            DF.dflash_lmhead_argmax(wl.ccfg, x, wl.w.lm_head, tok, None, ws, stream=stream)
        e1.record(stream)
    e1.synchronize()
    DF.dflash_check(ws, stream=stream)
    sec = e0.elapsed_time(e1) / reps / 1e3
    esz = 2 if cfg.dtype == "bf16" else 4
    algo = V * H * esz + M * H * esz + M * 8 + M * 4
    flops = 2.0 * M * V * H
    common = {"kernel": "lmhead_argmax (tcgen05 GEMM, argmax epilogue)",
              "peak_source": peak_src, "traffic": lmhead_traffic(cfg.name),
              "algorithmic_bytes_per_launch": algo, "algorithmic_flops_per_launch": flops,
              "us_per_launch": sec * 1e6,
              "note": "time includes the argmax-key reset and finish launches"}
    # bf16 with enough tokens per weight byte to pass the ridge point is
    # bounded by the tensor pipe (burst peak: the kernel is timed alone)
    if cfg.dtype == "bf16" and flops / algo > tf_burst * 1e12 / (hbm_peak * 1e9):
        tf = flops / sec / 1e12
        return dict(common, bound="tensor", achieved=tf, peak=tf_burst, unit="TFLOP/s",
                    frac=tf / tf_burst)
    gbs = algo / sec / 1e9
    return dict(common, bound="hbm", achieved=gbs, peak=hbm_peak, unit="GB/s",
                frac=gbs / hbm_peak)


def end_to_end(args, wl, DF, stream, world, blocks_per_step):
    """Per step: pinned host -> device copy of the step's inputs (the target
    states of the new context rows, the block tokens and the target tokens),
    the draft step + verification through the public API, and a device ->
    host read of the accepted tokens and lengths."""
    import torch
    fb = wl.final_buf
    dev_in = [t for t in (wl.new_states, wl.buf.block_tokens, fb.target_tokens) if t is not None]
    host_in = [t.cpu().pin_memory() for t in dev_in]
    host_out = [torch.empty_like(fb.out_tok, device="cpu").pin_memory(),
                torch.empty_like(fb.n_acc, device="cpu").pin_memory()]
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    steps = max(3, min(args.steps, 50))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for i in range(steps + 2):
            if i == 2:
                e0.record(stream)
            for d, h in zip(dev_in, host_in):
                d.copy_(h, non_blocking=True)
            wl.step(verify=True, stream=stream)
            host_out[0].copy_(fb.out_tok, non_blocking=True)
            host_out[1].copy_(fb.n_acc, non_blocking=True)
        e1.record(stream)
    e1.synchronize()
    ms = e0.elapsed_time(e1) / steps
    ms = max_over_ranks(ms, world)
    return {"value": blocks_per_step * world / (ms / 1e3), "unit": "blocks/s",
            "ms_per_step": ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "api": "dflash_draft_step via the Python binding, eager launches"}


# ---------------------------------------------------------------- profiling modes
def run_profile(args):
    """Setup, W eager warm-up steps, then K eager steps inside the NVTX range
    'dflash_step' (ncu --nvtx --nvtx-include dflash_step/ captures exactly
    the kernels of those K steps)."""
    import torch
    from block_diffusion_speculative_softmax_b200 import build as B
    B.build()
    from block_diffusion_speculative_softmax_b200 import dflash as DF
    from block_diffusion_speculative_softmax_b200 import synth, workload
    cfg = synth.get_config(args.config)
    wl = workload.Workload(cfg, seed=args.seed, mode=args.mode)
    wl.step(verify=False)
    torch.cuda.synchronize()
    wl.plant_targets()
    for _ in range(args.warmup):
        wl.step(verify=True)
    torch.cuda.synchronize()
    c0 = DF.dflash_launch_count()
    torch.cuda.nvtx.range_push("dflash_step")
    for _ in range(args.steps):
        wl.step(verify=True)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    wl.check()
    print(json.dumps({"mode": "profile", "workload": cfg.name, "steps": args.steps,
                      "launches": DF.dflash_launch_count() - c0}), flush=True)


def run_op(args):
    """One entry point alone at the workload's shapes: W warm-up + K timed
    calls between CUDA events on the launching stream; achieved bandwidth
    (or FLOP rate) from the algorithmic bytes (FLOPs) of one call."""
    import torch
    from block_diffusion_speculative_softmax_b200 import build as B
    B.build()
    from block_diffusion_speculative_softmax_b200 import dflash as DF
    from block_diffusion_speculative_softmax_b200 import synth
    cfg = synth.get_config(args.config)
    cc = DF.config_from(cfg)
    dt = DF.torch_dtype(cc)
    e = 2 if cfg.dtype == "bf16" else 4
    hbm, tfb, tfs, src = load_peaks()
    H, F, V, T, D = cfg.hidden, cfg.ffn, cfg.vocab, cfg.n_target_layers, cfg.n_draft_layers
    kvd, qd = cfg.kv_dim, cfg.q_dim
    nb = cfg.n_req * cfg.n_cand
    M = nb * cfg.block
    lens = synth.ctx_lengths(cfg, args.seed)
    N = int(sum(lens))
    g = torch.Generator(device="cuda").manual_seed(args.seed)

    def rnd(*shape, scale=1.0, dtype=dt):
        return (torch.randn(*shape, device="cuda", generator=g) * scale).to(dtype)

    ws = DF.alloc_workspace(DF.dflash_workspace_size(cc, cfg.n_req, nb, N, max(lens)))
    flops = 0.0
    if args.op == "lmhead":
        x, w = rnd(M, H), rnd(V, H, scale=0.02)
        tok = torch.empty(M, dtype=torch.int32, device="cuda")
        call = lambda: DF.dflash_lmhead_argmax(cc, x, w, tok, None, ws)
        algo = V * H * e + M * H * e + M * 4
        kernel = "gemm_sk_kernel<ARGMAX> (<= 64 tokens) / gemm_tok_kernel<ARGMAX> (LM head)"
    elif args.op == "mlp":
        h = rnd(M, H, dtype=torch.float32)
        gm = torch.ones(H, device="cuda")
        wg, wu, wd = rnd(F, H, scale=0.02), rnd(F, H, scale=0.02), rnd(H, F, scale=0.02)
        call = lambda: DF.dflash_mlp(cc, h, gm, wg, wu, wd, ws)
        algo = 3 * F * H * e + 2 * M * H * 4
        kernel = "rmsnorm + gemm_kernel x2 (split-K, SwiGLU and residual epilogues)"
    elif args.op == "ctxproj":
        x = rnd(N, H)
        pos = torch.arange(N, dtype=torch.int32, device="cuda")
        wk, wv = rnd(kvd, H, scale=0.02), rnd(kvd, H, scale=0.02)
        ko, vo = torch.empty(N, kvd, dtype=dt, device="cuda"), torch.empty(N, kvd, dtype=dt,
                                                                           device="cuda")
        call = lambda: DF.dflash_kv_project(cc, x, pos, None, wk, wv, ko, vo, ws)
        algo = N * H * e + 2 * kvd * H * e + 2 * N * kvd * e
        flops = 2.0 * N * H * 2 * kvd
        kernel = "gemm_tok_kernel<256,4> (context K/V projection, RoPE epilogue)"
    elif args.op == "attn":
        q, kb, vb = rnd(M, qd), rnd(M, kvd), rnd(M, kvd)
        kc, vc = rnd(N, kvd), rnd(N, kvd)
        off = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int64,
                           device="cuda")
        req = torch.arange(nb, dtype=torch.int32, device="cuda") // cfg.n_cand
        out = torch.empty(M, qd, dtype=dt, device="cuda")
        call = lambda: DF.dflash_block_attn(cc, nb, q, kb, vb, kc, vc, off, req, max(lens), out,
                                            ws)
        algo = 2 * N * kvd * e + 2 * M * qd * e + 2 * M * kvd * e
        flops = 4.0 * cfg.n_cand * N * cfg.block * qd
        kernel = "attn_mma_kernel<d, CS> (split-KV block attention, cluster merge)"
    else:  # fuse
        st = rnd(N, T, H)
        wf = torch.randn(D, T, device="cuda", generator=g)
        gl = [torch.ones(H, device="cuda") for _ in range(D)]
        fused = torch.empty(D, N, H, dtype=dt, device="cuda")
        call = lambda: DF.dflash_fuse_ctx(cc, st, wf, gl, fused)
        algo = N * T * H * e + D * N * H * e
        kernel = "fuse_rows_kernel (fusion + RMSNorm, all draft layers)"
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        call()
    e1.record()
    e1.synchronize()
    DF.dflash_check(ws)
    sec = e0.elapsed_time(e1) / args.steps / 1e3
    line = {"mode": "op", "op": args.op, "kernel": kernel, "workload": cfg.name,
            "us_per_call": sec * 1e6, "algorithmic_bytes": algo,
            "achieved_gbs": algo / sec / 1e9, "hbm_peak_gbs": hbm, "hbm_frac": algo / sec / 1e9 / hbm,
            "peak_source": src, "steps": args.steps, "warmup": args.warmup}
    if flops:
        line.update({"flops": flops, "achieved_tflops": flops / sec / 1e12,
                     "tensor_peak_tflops": tfb, "tensor_frac": flops / sec / 1e12 / tfb})
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    elif args.op:
        run_op(args)
    elif args.profile:
        run_profile(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""Throughput of the block-diffusion draft step + greedy verification.

One step = the whole hot path over one batch of seeded synthetic inputs:
fusion of the target states of every context row for every draft layer,
context K/V projection into the caches, D draft layers over the block(s),
final norm, LM-head argmax and acceptance against planted target tokens
(for the D2SD workload: first draft, lowest-confidence cuts, batched
re-anchored second draft over K candidates, acceptance).

    python bench.py [--gpus N --steps K --warmup W] [--config serving32]
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
# DRAM bytes (read + write) of one launch of a kernel from an ncu capture
# (summarised under profiles/), valid only for the source file it was taken
# with (digest of the file without comments); any later change of that code
# nulls it.  Key: (workload, mode, kernel-table name).
TRAFFIC = {
    # one serving32 context K/V projection (1 pass: dram__bytes_read.sum +
    # dram__bytes_write.sum of gemm_tokp_kernel, profiles/gemm_tokp_ctxproj_serving32.md)
    ("serving32", "full", "ctx_kv_proj"): {"bytes": 1192218112 + 533901312, "file": "gemm.cu",
                                          "sha256": "17615a7f2c849ec7"},
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="serving32")
    ap.add_argument("--mode", choices=["full", "steady"], default="full")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the step time and kernel table of the other workloads")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch the step eagerly instead of replaying a CUDA graph")
    ap.add_argument("--profile", action="store_true",
                    help="eager steps inside an NVTX range 'dflash_step' (for ncu launch lists)")
    ap.add_argument("--op", choices=["lmhead", "mlp", "ctxproj", "attn", "fuse", "fusenorm",
                                     "fcfuse", "sample"],
                    help="time one entry point alone at the workload's shapes")
    ap.add_argument("--rows", type=int, default=0,
                    help="--op: context rows (default: the workload's own sum of lengths)")
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
def _ev():
    import torch
    return torch.cuda.Event(enable_timing=True)


def time_calls(call, stream, reps, warm=2):
    """Mean device time (s) of ``call()`` over ``reps`` calls, CUDA events on
    the launching stream, after ``warm`` untimed calls."""
    import torch
    with torch.cuda.stream(stream):
        for _ in range(warm):
            call()
        e0, e1 = _ev(), _ev()
        e0.record(stream)
        for _ in range(reps):
            call()
        e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1) / reps / 1e3


def measure_step(wl, args, stream, steps, warmup, world, clocks=None):
    """Graph-captured step replayed ``steps`` times between CUDA events on its
    stream (after ``warmup`` replays), max over ranks.  Returns (ms, graph,
    launches per step)."""
    import torch
    from block_diffusion_speculative_softmax_b200 import dflash as DF
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
    launches = DF.dflash_launch_count() - c0

    def one_step():
        if graph is not None:
            graph.replay()
        else:
            wl.step(verify=True)

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            one_step()
    stream.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = _ev(), _ev()
    if clocks:
        clocks.mark("timed_start")
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(steps):
            one_step()
        e1.record(stream)
    e1.synchronize()
    if clocks:
        clocks.mark("timed_end")
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, world)
    wl.check()
    return ms, graph, launches


def accepted_tokens(wl, stream, n_plant, draws):
    """Mean emitted tokens per step over ``draws`` planted target draws, each
    run through verification on the GPU (and checked for K = 1).  The step's
    work does not depend on the targets."""
    import torch
    fb = wl.final_buf
    n_acc = fb.n_acc.cpu().numpy()
    assert (n_acc == n_plant).all() or wl.K > 1, "accept lengths differ from the planted ones"
    tok_draws = [int((n_acc + 1).sum())]
    for draw in range(1, draws):
        n_pl = wl.plant_targets(seed_offset=draw)
        with torch.cuda.stream(stream):
            wl.step(verify=True)
        stream.synchronize()
        wl.check()
        na = fb.n_acc.cpu().numpy()
        assert (na == n_pl).all() or wl.K > 1, "accept lengths differ from the planted ones"
        tok_draws.append(int((na + 1).sum()))
    return float(np.mean(tok_draws)), len(tok_draws)


def _entry(name, kernel, sec, count, algo_bytes, flops, peaks, ms_step):
    """One row of the kernel table: bound and roofline fraction from the
    algorithmic bytes / FLOPs of one call and its measured duration."""
    hbm, tf_burst, _, src = peaks
    ridge = tf_burst * 1e12 / (hbm * 1e9)
    tensor = flops > 0 and flops / max(algo_bytes, 1) > ridge
    row = {"kernel": name, "impl": kernel, "us_per_call": sec * 1e6, "calls_per_step": count,
           "algorithmic_bytes_per_call": int(algo_bytes), "algorithmic_flops_per_call": flops,
           "step_share_est": sec * count * 1e3 / ms_step if ms_step else None,
           "peak_source": src}
    if tensor:
        a = flops / sec / 1e12
        row.update(bound="tensor", achieved=a, peak=tf_burst, unit="TFLOP/s", frac=a / tf_burst)
    else:
        a = algo_bytes / sec / 1e9
        row.update(bound="hbm", achieved=a, peak=hbm, unit="GB/s", frac=a / hbm)
    return row


def kernel_table(wl, cfg, DF, peaks, stream, reps, ms_step):
    """Every entry point of the step timed alone on the workload's own device
    buffers (weights, states, KV caches) with CUDA events on its launch
    stream; algorithmic bytes / FLOPs per call from the path's formulas:
    fusion reads the new rows' T states once and writes D fused rows; the
    context K/V projection reads its rows and both weight matrices and
    writes K and V; attention reads every request's context K/V once (its
    candidates share it) plus Q, block K/V and the output; the MLP streams
    its three weight matrices; the LM head streams the vocabulary."""
    import torch
    e = 2 if cfg.dtype == "bf16" else 4
    H, F, V, T, D = cfg.hidden, cfg.ffn, cfg.vocab, cfg.n_target_layers, cfg.n_draft_layers
    kvd, qd = cfg.kv_dim, cfg.q_dim
    fb = wl.final_buf
    nb = fb.nb
    M = nb * cfg.block
    cc = wl.ccfg
    dt = wl.dt
    rows = []
    g = torch.Generator(device="cuda").manual_seed(1234)

    def rnd(*shape, scale=1.0, dtype=dt):
        return (torch.randn(*shape, device="cuda", generator=g) * scale).to(dtype)

    n_new = wl.n_new
    ws = DF.alloc_workspace(DF.dflash_workspace_size(cc, wl.R, nb, max(n_new, 1),
                                                     max(wl.ctx_lens)))
    if n_new > 0 and wl.w.w_fc is None:
        fused = torch.empty(D, n_new, H, dtype=dt, device="cuda")
        gl = [l["g_fuse"] for l in wl.w.layers]
        if cfg.dtype == "bf16":
            # the step's form: unnormalised rows + per-row partial sums of
            # squares (the norm is applied in the context projection)
            P = DF.dflash_fuse_rss_parts(H)
            rss = torch.empty(D, n_new, P, device="cuda")
            sec = time_calls(lambda: DF.dflash_fuse_ctx_rss(cc, wl.new_states, wl.w.w_fuse, gl,
                                                            fused, rss, ws), stream, reps)
            rows.append(_entry("fuse", "fuse_rows_unnorm_kernel", sec, 1,
                               n_new * T * H * e + D * n_new * H * e + D * n_new * P * 4, 0.0,
                               peaks, ms_step))
            del rss
        else:
            sec = time_calls(lambda: DF.dflash_fuse_ctx(cc, wl.new_states, wl.w.w_fuse, gl,
                                                        fused), stream, reps)
            rows.append(_entry("fuse", "fuse_rows_kernel", sec, 1,
                               n_new * T * H * e + D * n_new * H * e, 0.0, peaks, ms_step))
        pos = torch.arange(n_new, dtype=torch.int32, device="cuda")
        lay = wl.w.layers[0]
        kc, vc = fb.k_cache[0], fb.v_cache[0]
        sec = time_calls(lambda: DF.dflash_kv_project(cc, fused[0], pos, None, lay["w_kt"],
                                                      lay["w_vt"], kc, vc, ws), stream, reps)
        rows.append(_entry("ctx_kv_proj", "gemm_tokp_kernel / gemm_tok_kernel (RoPE epilogue)",
                           sec, D,
                           n_new * H * e + 2 * kvd * H * e + 2 * n_new * kvd * e,
                           2.0 * n_new * H * 2 * kvd, peaks, ms_step))
        del fused
    sum_L = int(sum(wl.ctx_lens))
    q, kb, vb = rnd(M, qd), rnd(M, kvd), rnd(M, kvd)
    out = torch.empty(M, qd, dtype=dt, device="cuda")
    sec = time_calls(lambda: DF.dflash_block_attn(cc, nb, q, kb, vb, fb.k_cache[0],
                                                  fb.v_cache[0], fb.ctx_off, fb.block_req,
                                                  fb.max_L, out, ws), stream, reps)
    rows.append(_entry("block_attn", "attn_mma_kernel (split-KV, cluster merge)", sec, D,
                       2 * sum_L * kvd * e + 2 * M * qd * e + 2 * M * kvd * e,
                       4.0 * cfg.n_cand * sum_L * cfg.block * qd + 4.0 * M * cfg.block * qd,
                       peaks, ms_step))
    h = torch.randn(M, H, device="cuda", generator=g)
    lay = wl.w.layers[0]
    sec = time_calls(lambda: DF.dflash_mlp(cc, h, lay["g_mlp"], lay["w_gate"], lay["w_up"],
                                           lay["w_down"], ws), stream, reps)
    rows.append(_entry("mlp", "rmsnorm + SwiGLU GEMM + down GEMM", sec, D,
                       3 * F * H * e + M * H * 4 * 2 + M * F * e * 2, 6.0 * M * H * F,
                       peaks, ms_step))
    x = rnd(M, H)
    tok = torch.empty(M, dtype=torch.int32, device="cuda")
    sec = time_calls(lambda: DF.dflash_lmhead_argmax(cc, x, wl.w.lm_head, tok, None, ws),
                     stream, reps)
    rows.append(_entry("lmhead_argmax", "LM-head GEMM with argmax epilogue", sec, 1,
                       V * H * e + M * H * e + M * 12, 2.0 * M * V * H, peaks, ms_step))
    DF.dflash_check(ws, stream=stream)
    del ws
    torch.cuda.empty_cache()
    return rows


def dominant(rows):
    return max(rows, key=lambda r: r["us_per_call"] * r["calls_per_step"])


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
    peaks = load_peaks()
    stream = torch.cuda.Stream()

    wl = workload.Workload(cfg, seed=args.seed + rank, mode=args.mode)
    # pass once, plant target tokens against the drafted blocks
    wl.step(verify=False)
    torch.cuda.synchronize()
    n_plant = wl.plant_targets()
    clocks = Clocks(torch.cuda.current_device())
    clocks.start()
    clocks.mark("warm_start")
    ms, graph, launches_per_step = measure_step(wl, args, stream, args.steps, args.warmup,
                                                world, clocks)
    tok_per_step, n_draws = accepted_tokens(wl, stream, n_plant, ACCEPT_DRAWS)
    blocks_per_step = wl.final_buf.nb
    value = blocks_per_step * world / (ms / 1e3)
    acc_tok_s = tok_per_step * world / (ms / 1e3)
    acc_draft_tok_s = (tok_per_step - wl.R) * world / (ms / 1e3)

    # ---- every kernel against its roofline; the dominant one is `roofline`
    rows = kernel_table(wl, cfg, DF, peaks, stream, max(5, min(50, args.steps)), ms)
    dom = dominant(rows)
    roof = dict(dom)
    roof["traffic"] = recorded_traffic(cfg.name, dom["kernel"], args.mode)
    clk = clocks.stop()

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        e2e = end_to_end(args, wl, DF, stream, world, blocks_per_step, graph)
    used_graph = graph is not None
    if graph is not None:
        del graph
    cfg_line = {"workload": cfg.name, "mode": args.mode, "n_req": cfg.n_req,
                "blocks_per_step": blocks_per_step, "block": cfg.block,
                "ctx_len": cfg.ctx_len if cfg.ctx_len_min == 0 else
                f"U[{cfg.ctx_len_min},{cfg.ctx_len}] (sum {int(sum(wl.ctx_lens))})",
                "draft_layers": cfg.n_draft_layers, "target_layers": cfg.n_target_layers,
                "hidden": cfg.hidden, "vocab": cfg.vocab, "parallelism": f"replicas{world}",
                "cuda_graph": used_graph,
                "l2": "inputs larger than L2 (weights %.2f GB streamed per step)"
                      % (wl.w.nbytes() / 1e9)}
    del wl
    torch.cuda.empty_cache()

    # ---- the other workloads (rank-local, no collectives): step time and
    # dominant-kernel roofline of each
    per_config = {}
    if world == 1 and not args.no_per_config:
        # every other workload in this mode, and the main workload in the
        # other mode (steady: only the newly accepted rows fused/projected)
        other = "steady" if args.mode == "full" else "full"
        runs = [(n, args.mode) for n in synth.CONFIG_ORDER if n != cfg.name]
        runs.append((cfg.name, other))
        for name, mode2 in runs:
            c2 = synth.get_config(name)
            w2 = workload.Workload(c2, seed=args.seed, mode=mode2)
            w2.step(verify=False)
            torch.cuda.synchronize()
            n2 = w2.plant_targets()
            steps2 = max(5, min(args.steps, 30))
            ms2, g2, _ = measure_step(w2, args, stream, steps2, max(3, args.warmup), 1)
            del g2
            t2, _ = accepted_tokens(w2, stream, n2, 16)
            r2 = kernel_table(w2, c2, DF, peaks, stream, 10, ms2)
            d2 = dominant(r2)
            key = name if mode2 == args.mode else f"{name}/{mode2}"
            per_config[key] = {"ms_per_step": ms2, "blocks_s": w2.final_buf.nb / (ms2 / 1e3),
                                "accepted_tok_s": t2 / (ms2 / 1e3), "steps": steps2,
                                "dominant_kernel": d2["kernel"], "dominant_bound": d2["bound"],
                                "dominant_frac": d2["frac"],
                                "kernels": {r["kernel"]: round(r["frac"], 4) for r in r2}}
            del w2
            torch.cuda.empty_cache()
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
            "mean_accept_tau": tok_per_step / cfg.n_req,
            "accept_draws": n_draws,
            "config": cfg_line,
            "gpu_launches": launches_per_step * args.steps,
            "launches_per_step": launches_per_step,
            "roofline": roof,
            "kernels": rows,
            "per_config": per_config or None,
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


def source_digest(fname):
    src = os.path.join(ROOT, "block_diffusion_speculative_softmax_b200", "csrc", fname)
    with open(src) as f:
        return code_digest(f.read())


def recorded_traffic(workload, kernel, mode="full"):
    """Measured DRAM bytes (read + write) per launch of ``kernel`` on
    ``workload``, or None when there is no capture for it or its source file
    changed since the capture."""
    ent = TRAFFIC.get((workload, mode, kernel))
    if ent is None:
        return None
    return ent["bytes"] if source_digest(ent["file"]).startswith(ent["sha256"]) else None


def end_to_end(args, wl, DF, stream, world, blocks_per_step, graph=None):
    """Per step: pinned host -> device copy of the step's inputs (the target
    states of the new context rows, the block tokens and the target tokens),
    the draft step + verification (the captured graph of the public API's
    calls when there is one, else the calls themselves), and a device -> host
    read of the accepted tokens and lengths."""
    import torch
    fb = wl.final_buf
    dev_in = [t for t in (wl.new_states, wl.buf.block_tokens, fb.target_tokens) if t is not None]
    host_in = [t.cpu().pin_memory() for t in dev_in]
    host_out = [torch.empty_like(fb.out_tok, device="cpu").pin_memory(),
                torch.empty_like(fb.n_acc, device="cpu").pin_memory()]
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    steps = max(3, min(args.steps, 20))
    e0, e1 = _ev(), _ev()
    with torch.cuda.stream(stream):
        for i in range(steps + 2):
            if i == 2:
                e0.record(stream)
            for d, h in zip(dev_in, host_in):
                d.copy_(h, non_blocking=True)
            if graph is not None:
                graph.replay()
            else:
                wl.step(verify=True, stream=stream)
            host_out[0].copy_(fb.out_tok, non_blocking=True)
            host_out[1].copy_(fb.n_acc, non_blocking=True)
        e1.record(stream)
    e1.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, world)
    return {"value": blocks_per_step * world / (ms / 1e3), "unit": "blocks/s",
            "ms_per_step": ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "api": "dflash_draft_step (graph-replayed) with pinned host copies in and out"
                   if graph is not None else "dflash_draft_step via the Python binding"}


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
    if args.rows > 0:   # same shapes, fewer rows (small ncu captures)
        lens = [max(1, args.rows // len(lens))] * len(lens)
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
        kernel = "gemm_tokp_kernel / gemm_tok_kernel (context K/V projection, RoPE epilogue)"
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
    elif args.op == "fcfuse":
        st = rnd(N, T, H)
        wfc = rnd(H, T * H, scale=0.02)
        gfc = torch.ones(H, device="cuda")
        fused = torch.empty(N, H, dtype=dt, device="cuda")
        ws = DF.alloc_workspace(DF.dflash_workspace_size(cc, cfg.n_req, nb, N, max(lens)))
        call = lambda: DF.dflash_fc_fuse_ctx(cc, st, wfc, gfc, fused, ws)
        algo = N * T * H * e + H * T * H * e + N * H * (e + 8)
        flops = 2.0 * N * T * H * H
        kernel = "FC fusion GEMM (fp32 epilogue) + rmsnorm_kernel"
    elif args.op == "sample":
        z = torch.randn(M, V, device="cuda", generator=g)
        tok = torch.empty(M, dtype=torch.int32, device="cuda")
        lq = torch.empty(M, device="cuda")
        call = lambda: DF.dflash_sample(cc, z, 1, 0, tok, lq, None)
        algo = M * V * 4 + M * 8
        kernel = "sample_rows_kernel (Gumbel-max over stored logits)"
    else:  # fuse (the step's split form for bf16), fusenorm (normalised output)
        st = rnd(N, T, H)
        wf = torch.randn(D, T, device="cuda", generator=g)
        gl = [torch.ones(H, device="cuda") for _ in range(D)]
        fused = torch.empty(D, N, H, dtype=dt, device="cuda")
        if args.op == "fuse" and cfg.dtype == "bf16":
            P = DF.dflash_fuse_rss_parts(H)
            rss = torch.empty(D, N, P, device="cuda")
            call = lambda: DF.dflash_fuse_ctx_rss(cc, st, wf, gl, fused, rss, ws)
            algo = N * T * H * e + D * N * H * e + D * N * P * 4
            kernel = "fuse_rows_unnorm_kernel (fusion, row sums of squares, all draft layers)"
        else:
            call = lambda: DF.dflash_fuse_ctx(cc, st, wf, gl, fused)
            algo = N * T * H * e + D * N * H * e
            kernel = "fuse_rows_kernel (fusion + RMSNorm, all draft layers)"

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            fn()
        e1.record()
        e1.synchronize()
        return e0.elapsed_time(e1) / args.steps / 1e3

    sec = timed(call)
    DF.dflash_check(ws)
    extra = {}
    if args.op == "lmhead" and M <= 4096:
        # the allocation-free entry point on the same inputs (<= 64 tokens it
        # takes the one-CTA-per-tile kernel instead of stream-K)
        s2 = timed(lambda: DF.dflash_lmhead_argmax_noalloc(cc, x, w, tok))
        extra = {"noalloc_us_per_call": s2 * 1e6, "noalloc_hbm_frac": algo / s2 / 1e9 / hbm}
    line = {"mode": "op", "op": args.op, "kernel": kernel, "workload": cfg.name,
            "us_per_call": sec * 1e6, "algorithmic_bytes": algo,
            "achieved_gbs": algo / sec / 1e9, "hbm_peak_gbs": hbm, "hbm_frac": algo / sec / 1e9 / hbm,
            "peak_source": src, "steps": args.steps, "warmup": args.warmup}
    if flops:
        line.update({"flops": flops, "achieved_tflops": flops / sec / 1e12,
                     "tensor_peak_tflops": tfb, "tensor_frac": flops / sec / 1e12 / tfb})
    line.update(extra)
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

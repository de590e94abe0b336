"""Throughput of the APB per-host prefill path on B200.

One step = one whole prefill of one sequence: retaining-head scoring and top-k
compression (apb_score_compress), the passing block (apb_build_passing) and
block attention (apb_block_attention), with Q/K/V already resident in HBM.
Default workload: Llama-3.1-8B attention shapes at 128K (32 q / 8 kv heads,
d = 128, 8 virtual hosts x 16384 tokens, anchor 2048, keep 2048).

  python bench.py [--gpus N --steps K --warmup W --workload NAME]
  python bench.py --impl reference ...     # the CPU oracle, bounded sample

N > 1 (one process per GPU under torch.distributed.run): every rank prefills
its own independent sequence (weak scaling, no collective on the data path);
the step time is the max over ranks.
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

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from long_context_sparse_apb_b200 import inputs  # noqa: E402

METRIC = "APB prefill tokens/s at 128K (Llama-8B attn shapes); % bf16 peak; % HBM BW"
UNIT = "tokens/s"


def visible_pairs(cfg) -> int:
    """(query, key) pairs one q head attends: per host n(n+1)/2 causal, n*A
    anchor (hosts >= 1), n*h*keep passing."""
    n, A, keep = cfg.block_len, cfg.anchor_len, cfg.keep
    return sum(n * (n + 1) // 2 + (n * A if h else 0) + n * h * keep for h in range(cfg.n_hosts))


def visited_tile_pairs(cfg) -> int:
    """Pairs the kernel computes: whole 128x128 tiles (mask applied inside)."""
    n, A, keep, T = cfg.block_len, cfg.anchor_len, cfg.keep, 128
    nq = -(-n // T)
    tot = 0
    for h in range(cfg.n_hosts):
        na = -(-A // T) if (h and A) else 0
        np_ = -(-(h * keep) // T)
        for t in range(nq):
            tot += (na + np_ + t + 1) * T * T
    return tot


def attention_flops(cfg, pairs) -> float:
    return 4.0 * cfg.head_dim * cfg.n_q_heads * pairs


def hbm_bytes_compress(cfg) -> int:
    """Algorithmic bytes of score + top-k + gather (bytes each must move once)."""
    N, d, hq, hkv = cfg.seq_len, cfg.head_dim, cfg.n_q_heads, cfg.n_kv_heads
    H, keep = cfg.n_hosts, cfg.keep
    return (N * hq * d * 2 + 2 * N * hkv * d * 2 + 2 * N * hkv * 4 + H * hkv * keep * 4
            + 2 * (2 * H * hkv * keep * d * 2))


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained", j["bf16_tflops"]),
                "sustained_mhz": j.get("clocks_under_load", {}).get("sm_mhz_median"),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while running."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append((float(f[1]), float(f[2]), float(f[3]), f[4], f[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        load = [r for r in rows if r[2] > 300.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        seen = set()
        for r in load:
            for nm, val in zip(names, r[4]):
                if val.lower().startswith("active"):
                    seen.add(nm)
        return {"sm_mhz": statistics.median(r[0] for r in load), "sm_max_mhz": load[0][1],
                "power_w_max": max(r[2] for r in load), "samples": len(load),
                "reasons": sorted(seen)}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_config(cfg, rank):
    """Each rank prefills its own sequence: same workload, its own seed."""
    return cfg.replace(seed=cfg.seed + 1000 * rank)


def config_dict(cfg, world, mode="replicas"):
    if mode == "heads":
        par = (f"kv-head-sharded: one sequence, {world} GPU(s) x {cfg.n_kv_heads // world} kv "
               f"head(s) and their q heads, no collective")
    else:
        par = f"{world} independent sequence(s), one per GPU"
    return {"workload": cfg.name, "seq_len": cfg.seq_len, "n_hosts": cfg.n_hosts,
            "block_len": cfg.block_len, "anchor_len": cfg.anchor_len, "keep": cfg.keep,
            "n_q_heads": cfg.n_q_heads, "n_kv_heads": cfg.n_kv_heads,
            "head_dim": cfg.head_dim, "parallelism": par,
            "l2": "no flush: each step reads Q/K/V far larger than the 126 MB L2"}


# ---------------------------------------------------------------- CPU oracle

def oracle_sample(cfg, x, attn_rows_per_host: int):
    """Times the oracle on a bounded sample of one prefill and extrapolates to
    the whole prefill.  Sample: scoring and top-k of host 0's block, the
    passing block of every host, and attention of `attn_rows_per_host` rows
    per host on all q heads (rows spread over the block)."""
    import numpy as np
    import oracle

    f = lambda t: t.float().numpy()
    n, H = cfg.block_len, cfg.n_hosts
    w = [x[k].numpy() for k in ("w1", "b1", "w2", "b2")]
    t0 = time.perf_counter()
    s0 = oracle.retaining_scores(f(x["q"][:n]), f(x["k"][:n]), f(x["v"][:n]), *w)
    t1 = time.perf_counter()
    idx0 = oracle.compress_indices(s0, 1, n, cfg.keep)
    t2 = time.perf_counter()
    idx = np.concatenate([idx0 + h * n for h in range(H)], axis=0)   # stand-in positions
    k, v = f(x["k"]), f(x["v"])
    pk, pv = oracle.passing_blocks(k, v, idx)
    t3 = time.perf_counter()
    rows = np.linspace(0, n - 1, attn_rows_per_host).astype(np.int64)
    for h in range(H):
        oracle.host_attention(f(x["q"][h * n + torch.as_tensor(rows)]), rows, h, k, v, pk, pv, n,
                              cfg.anchor_len, cfg.keep)
    t4 = time.perf_counter()
    total = (t1 - t0) * H + (t2 - t1) * H + (t3 - t2) + (t4 - t3) * (n / attn_rows_per_host)
    measured = t4 - t0
    return cfg.seq_len / total, measured


def cpu_cores() -> int:
    try:
        from threadpoolctl import threadpool_info
        nth = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if nth:
            return int(max(nth))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def run_reference(args, cfg):
    world, rank, _ = dist_setup(args.gpus)
    if rank != 0:
        return
    x = inputs.generate(cfg)
    rows = args.oracle_rows
    vals, secs = [], []
    for i in range(args.warmup + args.steps):
        v, meas = oracle_sample(cfg, x, rows)
        if i >= args.warmup:
            vals.append(v)
            secs.append(meas)
    value = statistics.median(vals)
    # one step = one bounded sample, timed as it ran; `value` is the tokens of
    # the whole sequence over the sample's time extrapolated to the sequence,
    # so a step stands for value * step-seconds tokens of work
    ms_per_step = statistics.median(secs) * 1e3
    sample = (f"per step: scoring+top-k of host 0 (x{cfg.n_hosts} hosts), passing block of every "
              f"host, attention of {rows} rows/host on all {cfg.n_q_heads} q heads "
              f"(x{cfg.block_len // rows}); NumPy float64; a step is this sample "
              f"({ms_per_step / 1e3:.1f} s measured), worth {value * ms_per_step / 1e3:.0f} of "
              f"the sequence's {cfg.seq_len} tokens at the extrapolated rate")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "tokens_equiv_per_step": value * ms_per_step / 1e3,
            "higher_is_better": True, "scaling": "weak" if args.mode == "replicas" else "strong",
            "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_dict(cfg, args.gpus, args.mode),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU path

def local_work(cfg, mode, rank, world):
    """(config of this rank's work, its inputs).  heads: kv heads [gb, ge) of
    the one sequence and their q heads (every (host, kv head) unit is
    independent, so the ranks need no collective); replicas: an independent
    sequence per rank (its own seed)."""
    if mode == "heads":
        from long_context_sparse_apb_b200.sharded import head_slice, kv_head_range
        gb, ge = kv_head_range(cfg.n_kv_heads, rank, world)
        lcfg = cfg.replace(n_q_heads=(ge - gb) * cfg.group, n_kv_heads=ge - gb)
        x = inputs.generate(cfg)
        x = head_slice(x, cfg.n_q_heads, cfg.n_kv_heads, gb, ge)
        return lcfg, x
    rcfg = rank_config(cfg, rank)
    return rcfg, inputs.generate(rcfg)


def run_gpu(args, cfg):
    from long_context_sparse_apb_b200 import _lib as apb

    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    mode = args.mode
    # sequences prefilled per timed step by the whole job
    seqs = world if mode == "replicas" else 1
    full_cfg = cfg
    cfg, x = local_work(full_cfg, mode, rank, world)      # this rank's share
    xd = {k: v.to(dev) for k, v in x.items() if k != "needles"}
    c = apb.make_config(cfg)
    run = apb.Prefill(c, device=dev)
    stream = torch.cuda.current_stream(dev)
    w = (xd["w1"], xd["b1"], xd["w2"], xd["b2"])

    n_ev = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_ev)]
    # the timed step: the whole path in one C call (apb_prefill)
    pws = torch.zeros(apb.prefill_workspace_bytes(c), dtype=torch.uint8, device=dev)
    pout = torch.empty_like(run.out)

    def step():
        apb.prefill(c, xd["q"], xd["k"], xd["v"], *w, out=pout, workspace=pws, stream=stream)

    # the same path as three calls, for the per-stage breakdown
    def staged(e):
        e[0].record(stream)
        apb.score_compress(c, xd["q"], xd["k"], xd["v"], *w, idx=run.idx,
                           workspace=run.workspace, stream=stream)
        e[1].record(stream)
        apb.build_passing(c, xd["k"], xd["v"], run.idx, run.pass_k, run.pass_v, stream=stream)
        e[2].record(stream)
        apb.block_attention(c, xd["q"], xd["k"], xd["v"], run.pass_k, run.pass_v, out=run.out,
                            workspace=run.workspace, stream=stream)
        e[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if apb.device_status(pws) != apb.APB_OK:
        raise RuntimeError("device status not OK after warm-up")

    clocks = ClockSampler(local)
    clocks.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    t_start.record(stream)
    for i in range(args.steps):
        step()
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    clk = clocks.stop()
    elapsed_ms = t_start.elapsed_time(t_end)
    status = apb.device_status(pws)
    if status != apb.APB_OK:
        raise RuntimeError(f"device status {apb.status_string(status)} after timed steps")
    for i in range(n_ev):
        staged(ev[i])
    # the compression as the one-call step runs it: score, then top-k with the
    # passing-block gather in the same launch
    evf = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n_ev)]
    for e in evf:
        e[0].record(stream)
        apb.score_compress_pass(c, xd["q"], xd["k"], xd["v"], *w, run.pass_k, run.pass_v,
                                idx=run.idx, workspace=run.workspace, stream=stream)
        e[1].record(stream)
    torch.cuda.synchronize(dev)
    fused_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evf)

    score_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    gather_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    attn_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in ev)
    max_ms = max_over_ranks(elapsed_ms, world)
    ms_per_step = max_ms / args.steps
    value = seqs * cfg.seq_len / (max_ms / 1e3 / args.steps)

    # ---- end to end through the public API with pinned host buffers: every
    # step copies its inputs in and its output back; StreamedPrefill streams
    # each step host by host, so its copies overlap its own compute and the
    # other step's
    hx = {k: v.pin_memory() for k, v in x.items() if k != "needles"}
    hout = [torch.empty(run.out.shape, dtype=run.out.dtype).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in hx.values())
    d2h = hout[0].numel() * hout[0].element_size()
    del run, xd, pws, pout
    torch.cuda.empty_cache()
    # host-by-host streaming pays per-host launches; for short blocks the
    # whole-step pipeline (one apb_prefill per step) is the faster public path
    streamed = cfg.block_len >= 4096
    pipe = (apb.StreamedPrefill if streamed else apb.PrefillPipeline)(c, device=dev, depth=2)
    for i in range(max(2, args.warmup)):
        pipe.submit(hx, hout[i % 2])
    pipe.synchronize()
    barrier(world)
    torch.cuda.synchronize(dev)
    e2e_steps = max(4, args.steps)
    t0 = time.perf_counter()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(pipe.h2d)
    for i in range(e2e_steps):
        pipe.submit(hx, hout[i % 2])
    for s in [pipe.comp] + (pipe.att if streamed else []):
        pipe.d2h.wait_stream(s)
    e1.record(pipe.d2h)
    pipe.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    wall_ms = (time.perf_counter() - t0) * 1e3
    barrier(world)
    e2e_value = seqs * cfg.seq_len / (e2e_ms / 1e3 / e2e_steps)
    wss = pipe.workspaces() if streamed else [sl["ws"] for sl in pipe.slots]
    if any(apb.device_status(w) != apb.APB_OK for w in wss):
        raise RuntimeError("device status not OK after the end-to-end steps")
    del pipe
    torch.cuda.empty_cache()
    xd = {k: v.to(dev) for k, v in x.items() if k != "needles"}

    variants = None
    if not args.no_variants:
        variants = attention_variants(apb, cfg, xd, dev, stream, attn_ms)

    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    peaks = load_peaks()
    pairs = visible_pairs(cfg)
    tiles = visited_tile_pairs(cfg)
    fl_alg = attention_flops(cfg, pairs)
    fl_vis = attention_flops(cfg, tiles)
    ach = fl_alg / (attn_ms / 1e3) / 1e12
    # the attention kernel is timed alone (one ~33 ms launch per step), so the
    # roofline uses the measured burst GEMM peak; the sustained figure was
    # measured at a lower clock (see MEASURED_PEAKS.json), so a fraction of it
    # mixes two clocks and is reported only as such.  The per-cycle figure
    # compares with the tensor core's 8192 bf16 FLOP per SM and cycle (one
    # 128x128x16 UMMA per 64 cycles) at the SM clock sampled during the run.
    peak = peaks["bf16_tflops"]
    sm_mhz = clk["sm_mhz"] if clk else None
    n_sms = torch.cuda.get_device_properties(dev).multi_processor_count
    per_cycle_peak = 8192 * n_sms * sm_mhz * 1e6 / 1e12 if sm_mhz else None
    hbm = hbm_bytes_compress(cfg)
    hbm_ach = hbm / (fused_ms / 1e3) / 1e9
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        v, meas = oracle_sample(cfg, x, args.oracle_rows)
        cpu = {"value": v, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
               "sample": (f"scoring+top-k of host 0 extrapolated x{cfg.n_hosts}, passing block of "
                          f"all hosts, attention of {args.oracle_rows} rows/host on all heads "
                          f"extrapolated x{cfg.block_len // args.oracle_rows}; NumPy float64; "
                          f"{meas:.1f} s measured")}
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "attention_traffic.json")
    if os.path.exists(tpath):
        tj = json.load(open(tpath))
        if (world == 1 and tj.get("workload") == cfg.name
                and tj.get("kernel_rev") == apb_kernel_rev()):
            traffic = tj.get("bytes_per_launch")
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak" if mode == "replicas" else "strong", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": config_dict(full_cfg, world, mode),
        "stages_ms": {"score_topk": score_ms, "passing": gather_ms, "attention": attn_ms,
                      "compress_fused": fused_ms},
        "attention": {"tflops_algorithmic": ach, "tflops_visited_tiles": fl_vis / (attn_ms / 1e3) / 1e12,
                      "frac_visited_of_peak": fl_vis / (attn_ms / 1e3) / 1e12 / peak,
                      "frac_of_sustained_peak_other_clock": ach / peaks["bf16_tflops_sustained"],
                      "sustained_peak_clock_mhz": peaks.get("sustained_mhz"),
                      "frac_of_per_cycle_peak": (ach / per_cycle_peak) if per_cycle_peak else None,
                      "per_cycle_peak_tflops": per_cycle_peak, "sm_mhz": sm_mhz},
        "compress_stages": {"bytes": hbm, "gbs": hbm_ach, "frac_of_hbm_peak": hbm_ach / peaks["hbm_gbs"],
                            "how": "score + top-k with the gather in its launch (the one-call path)",
                            "two_call_gbs": hbm / ((score_ms + gather_ms) / 1e3) / 1e9},
        "roofline": {"bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                     "frac": ach / peak, "traffic": traffic,
                     "frac_per_cycle": (ach / per_cycle_peak) if per_cycle_peak else None,
                     "sm_mhz": sm_mhz,
                     "peak_source": f"{peaks['source']} bf16_tflops (burst; the kernel is one "
                                    f"{attn_ms:.1f} ms launch per step); frac_per_cycle: against "
                                    f"8192 FLOP/SM/cycle x {n_sms} SMs at the run's median "
                                    f"SM clock"},
        "cpu_baseline": cpu,
        "variants": variants,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps, "ms": e2e_ms,
                "host_wall_ms": wall_ms,
                "how": ("StreamedPrefill: pinned host buffers; per step the H2D copies, the "
                        "compression, the attention (two streams) and the D2H copies run host by "
                        "host on their own streams, two slots; copy-in of host h+1 overlaps host "
                        "h's compute, and host h's output goes back as soon as it is attended"
                        if streamed else
                        "PrefillPipeline (blocks shorter than 4096 rows): pinned H2D copies, one "
                        "apb_prefill call and the D2H copy of the output on three streams, two "
                        "slots, copies of one step overlapping another step's compute")},
        # per apb_prefill: weight split, score, top-k with the gather, attention
        "gpu_launches": args.steps * (4 if cfg.keep > 0 and cfg.n_hosts > 1 else 1),
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def attention_variants(apb, cfg, xd, dev, stream, apb_ms, reps=3):
    """The same attention kernel on the same Q/K/V with the two masks the
    pages compare APB against: dense causal attention over the whole
    sequence (one host), and a Star-Attention-style pattern (anchor = a whole
    block, no passing block).  Reports the APB mask's speed-up over each, and
    the score + top-k time of the query-aware compression variant."""
    out = {"apb_ms": apb_ms}
    other_anchor = cfg.block_len // 4 if cfg.anchor_len * 8 == cfg.block_len else cfg.block_len // 8
    shapes = {"dense_causal": dict(n_hosts=1, block_len=cfg.seq_len, anchor_len=0, query_len=0,
                                   keep=0),
              "star": dict(anchor_len=cfg.block_len, keep=0),
              # the pages' other anchor size (1/4 <-> 1/8 of a block), same keep
              f"anchor_{other_anchor}": dict(anchor_len=other_anchor,
                                             query_len=min(cfg.query_len, other_anchor))}
    for name, kw in shapes.items():
        c = apb.make_config(cfg, **kw)
        pk = pv = None
        if c.keep > 0 and c.n_hosts > 1:
            # the same compressed blocks as the APB step (the anchor size does not enter them)
            run = apb.Prefill(c, device=dev)
            apb.score_compress(c, xd["q"], xd["k"], xd["v"], xd["w1"], xd["b1"], xd["w2"],
                               xd["b2"], idx=run.idx, workspace=run.workspace, stream=stream)
            pk, pv = apb.build_passing(c, xd["k"], xd["v"], run.idx, run.pass_k, run.pass_v,
                                       stream=stream)
        apb.block_attention(c, xd["q"], xd["k"], xd["v"], pk, pv, out=None, stream=stream)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        o = torch.empty_like(xd["q"])
        e0.record(stream)
        for _ in range(reps):
            apb.block_attention(c, xd["q"], xd["k"], xd["v"], pk, pv, out=o, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms = e0.elapsed_time(e1) / reps
        out[f"{name}_ms"] = ms
        out[f"apb_speedup_vs_{name}"] = ms / apb_ms
        del o, pk, pv
    # query-aware compression (q input = query-segment mean): score + top-k time
    c = apb.make_config(cfg)
    ws = apb.new_workspace(c)
    w = (xd["w1"], xd["b1"], xd["w2"], xd["b2"])
    apb.score_compress(c, xd["q"], xd["k"], xd["v"], *w, workspace=ws, stream=stream,
                       query_aware=True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        apb.score_compress(c, xd["q"], xd["k"], xd["v"], *w, workspace=ws, stream=stream,
                           query_aware=True)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    out["query_aware_score_topk_ms"] = e0.elapsed_time(e1) / reps
    return out


def run_sharded(args, cfg):
    """One sequence prefilled by N GPUs, hosts split evenly and round-robin
    (the pages' distributed form; round-robin balances the per-host work):
    per step each rank compresses its hosts, the compressed blocks are
    all-gathered over NCCL, each rank attends its hosts.  Strong scaling:
    value = tokens of the one sequence / max-over-ranks step time."""
    from long_context_sparse_apb_b200 import _lib as apb
    from long_context_sparse_apb_b200.sharded import ShardedPrefill, tensor_all_gather

    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    c = apb.make_config(cfg)
    sp = ShardedPrefill(c, rank, world, device=dev,
                        all_gather=tensor_all_gather() if world > 1 else None)
    loc = {k: v.to(dev) for k, v in inputs.generate_local(
        cfg, sp.first, sp.first + sp.count * sp.stride, sp.stride).items()}
    w = (loc["w1"], loc["b1"], loc["w2"], loc["b2"])
    stream = torch.cuda.current_stream(dev)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]

    def step(e=None):
        if e is not None:
            e[0].record(stream)
        sp.compress(loc["q"], loc["k"], loc["v"], *w)
        if e is not None:
            e[1].record(stream)
        sp.exchange()
        if e is not None:
            e[2].record(stream)
        sp.attend(loc["q"], loc["k"], loc["v"])
        if e is not None:
            e[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize(dev)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        step(ev[i])
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    clk = clocks.stop()
    if apb.device_status(sp.workspace) != apb.APB_OK:
        raise RuntimeError("device status not OK after timed steps")
    max_ms = max_over_ranks(t0.elapsed_time(t1), world)
    stages = {name: max_over_ranks(statistics.mean(e[a].elapsed_time(e[b]) for e in ev), world)
              for name, a, b in (("compress", 0, 1), ("exchange", 1, 2), ("attention", 2, 3))}
    if rank == 0:
        cdict = config_dict(cfg, world)
        cdict["parallelism"] = (f"host-sharded: {world} GPU(s) x {cfg.n_hosts // world} host(s) "
                                f"({sp.order}), NCCL all-gather of the compressed blocks")
        line = {"metric": METRIC, "value": cfg.seq_len / (max_ms / 1e3 / args.steps),
                "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": max_ms / args.steps, "higher_is_better": True,
                "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": cdict, "stages_ms_max_over_ranks": stages,
                "exchange_bytes_per_rank": 2 * sp.count * cfg.keep * cfg.n_kv_heads
                * cfg.head_dim * 2,
                "e2e": None, "e2e_note": "host-buffer end-to-end is measured in the default mode",
                # per owned host: weight split, score, top-k (with the gather
                # when keep > 0); one attention launch per step
                "gpu_launches": args.steps * (cfg.n_hosts // world) * (3 if cfg.keep else 2)
                + args.steps, "clocks": clk}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def source_rev(src: str) -> str:
    """Hash of C++ source with comments, blank lines and trailing blanks
    removed."""
    import hashlib
    import re
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    code = "\n".join(line.rstrip() for line in src.splitlines() if line.strip())
    return hashlib.sha1(code.encode()).hexdigest()[:12]


def apb_kernel_rev() -> str:
    """Revision of the attention kernel's code: ncu traffic counters only
    apply to the code they were taken on (a comment edit does not change it)."""
    p = os.path.join(ROOT, "long_context_sparse_apb_b200", "csrc", "attention.cu")
    return source_rev(open(p, encoding="utf-8").read())


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--mode", default="heads", choices=["heads", "sharded", "replicas"],
                    help="heads (default): one sequence with its kv heads split over the GPUs, "
                         "no collective (strong scaling; at one GPU the whole sequence); "
                         "sharded: one sequence with its hosts split over the GPUs and an "
                         "NCCL all-gather of the compressed blocks (strong scaling); "
                         "replicas: one independent sequence per GPU (weak scaling)")
    ap.add_argument("--workload", default="llama8b_128k", choices=sorted(inputs.CONFIGS))
    ap.add_argument("--oracle-rows", type=int, default=64)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the dense-causal and Star-style timings of the same kernel")
    args = ap.parse_args()
    cfg = inputs.CONFIGS[args.workload]
    if args.impl == "reference":
        run_reference(args, cfg)
    elif args.mode == "sharded":
        run_sharded(args, cfg)
    else:
        run_gpu(args, cfg)


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""Throughput of the SPIN-4DGS per-Gaussian attribute decoder on B200.

Metric: decoded spatiotemporal positions/s.  One step = one fused decode
(normalise -> 4D hash encode -> trunk + heads -> activations -> Sigma) of one
synthetic sports frame (300k positions, 16-level fp16 hash grid with 2^19
entries per level, 32-64-64-11 fp16 network).  With N GPUs every rank
decodes its own frame (weak scaling, no collective on the data path); the
time is the max over ranks.  A second measurement covers fwd+bwd: one
1M-position training launch (forward, then backward with the scatter-add into
the tables and the weight gradients).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
import argparse
import dataclasses
import ctypes
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from spatiotemporal_neural_field_b200 import synthetic as S  # noqa: E402

WORKLOAD = "sports_frame_fp16"
OUT_WIDTHS = S.DECODE_OUT_WIDTHS
METRIC = "decoded spatiotemporal positions/s (fwd)"
UNIT = "positions/s"
KERNEL_SRC = os.path.join(ROOT, "spatiotemporal_neural_field_b200", "csrc")


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-fwd-bwd", action="store_true")
    p.add_argument("--cpu-sample", type=int, default=100_000,
                   help="positions the oracle decodes on one core for cpu_baseline (~4 s); every core's process "
                        "decodes a quarter of that for the all-cores figure")
    p.add_argument("--no-probe", action="store_true", help="skip the random-gather ceiling measurement")
    p.add_argument("--workloads", action="store_true",
                   help="time every workload (fwd, and fwd+bwd where trained) and the device ceilings; "
                        "one JSON line each")
    p.add_argument("--l2-window", action="store_true",
                   help="time the 45-launch training step without and with an L2 access-policy window over the "
                        "fp16 tables and over the fp32 table gradients; one JSON line each")
    p.add_argument("--cpu-workloads", action="store_true",
                   help="time the oracle on every workload (1 thread and all cores); one JSON line each")
    p.add_argument("--ncu-case", default=None,
                   help="profiling driver: run a few untimed launches of one workload and exit "
                        "(sports_frame_fp16, stress_fp16_gate, sports_train_fp16, hexplane_fp32, tiny_fp32, "
                        "render_sports_frame, paper_heads_fp16, hexplane_fwd_fp32)")
    return p.parse_args()


def workload_config(n_gpus):
    w = S.WORKLOADS[WORKLOAD]
    g, m = w["grid"], w["mlp"]
    return {
        "workload": "%s: one frame of %d positions per GPU (80%% static, 20%% in 8 fast blobs), "
                    "L=%d F=%d T=2^%d fp16 tables, spatial res %d-%d, temporal %d-%d, "
                    "%d-%dx%d-11 fp16 trunk+heads" % (WORKLOAD, w["N"], g.L, g.F, g.log2_T, g.nmin_s, g.nmax_s,
                                                       g.nmin_t, g.nmax_t, m.in_dim, m.n_hidden, m.hidden),
        "positions_per_gpu": w["N"],
        "l2": "flushed before every timed step (256 MiB write, outside the events)",
        "parallelism": "dp%d (independent frames per rank, no collective)" % n_gpus,
    }


def algorithmic_bytes_per_position():
    """Useful table bytes a position needs: 16 levels x 16 corners x F fp16
    features (its 16-byte input and 17 fp32 outputs come on top)."""
    g = S.WORKLOADS[WORKLOAD]["grid"]
    return g.L * 16 * g.F * 2


IO_BYTES_PER_POSITION = 16 + 17 * 4


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


DECODE_SOURCES = ("decode_tc.cu", "common.cuh", "tc.cuh")


def kernel_source_hash(files=DECODE_SOURCES):
    """Hash of the sources the timed decode kernel is built from."""
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(KERNEL_SRC, f), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per launch of the decode kernel from the committed ncu
    summary, if it was taken on the current kernel sources."""
    p = os.path.join(ROOT, "profiles", "decode_fwd_sports_frame.traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    if d.get("source_hash") != kernel_source_hash():
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.proc = None
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", uuid, "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except Exception:
            self.proc.kill()
            out = ""
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                smax.append(float(f[1]))
            except ValueError:
                continue
            for nm, v in zip(names, f[4:8]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def table_sectors_per_position(sp, g, pos_dev, F, elem_bytes, sample=20_000):
    """Distinct 32-byte table sectors one position touches (all levels), from
    the kernel's own corner indices: the minimum sector traffic of a position
    when no other position shares its sectors."""
    idx, _ = sp.debug_corners(g, pos_dev[:sample].contiguous())
    idx = idx.cpu().numpy().view(np.uint32).astype(np.int64)
    sec = np.sort((idx * F * elem_bytes) >> 5, axis=2)
    distinct = 1 + np.count_nonzero(np.diff(sec, axis=2), axis=2)
    return float(distinct.sum(axis=1).mean())


def probe_sector_rates(sp, torch, dev):
    """Random 16-byte loads (one sector each) from a 32 MiB L2-resident buffer
    and from a 4 GiB buffer (HBM): the gather ceilings, sectors/s."""
    from spatiotemporal_neural_field_b200 import probe as pr
    out = {}
    blocks = 4 * torch.cuda.get_device_properties(dev).multi_processor_count
    for name, nbytes, lpt in (("l2", 32 << 20, 4096), ("hbm", 4 << 30, 1024)):
        buf = torch.ones(nbytes // 4, dtype=torch.int32, device=dev)
        best = None
        for it in range(4):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            n = pr.probe_gather(buf, 16, lpt, blocks, seed=it + 1)
            b.record()
            torch.cuda.synchronize()
            if it:
                rate = n / (a.elapsed_time(b) * 1e-3)
                best = rate if best is None else max(best, rate)
        out[name] = best
        del buf
    return out


def train_step_measurement(args, sp, torch, dist, dev, world, rank, scene, tables16, weights16, grid, mlp, g, m,
                           flush, stream, l2_window=None):
    """One training step over the whole 150-frame sequence (45M positions):
    45 launches of 1M positions, each decode_fwd (saving z) + decode_bwd
    (gradients accumulate), then fused Adam on the fp32 master tables and
    weights, which also rewrites the fp16 working copies and clears the
    gradients.  With N ranks every rank does this on its own upstream
    gradients and the gradients are summed over ranks before Adam."""
    from spatiotemporal_neural_field_b200 import dp
    wt = S.WORKLOADS["sports_train_fp16"]
    nb, total = wt["batch"], wt["N"]
    n_batches = total // nb
    pos_all = torch.from_numpy(scene.frames(range(S.N_FRAMES))).to(dev)
    gen = torch.Generator(device=dev).manual_seed(1234 + rank)
    grads = {k: torch.randn((total, wd), device=dev, generator=gen) * wt["grad_std"] for k, wd in OUT_WIDTHS.items()}
    tab32 = tables16.float().contiguous()
    w32 = weights16.float().contiguous()
    tab16, w16 = tables16.clone(), weights16.clone()
    gtab, gw = torch.zeros_like(tab32), torch.zeros_like(w32)
    mt, vt, mw, vw = (torch.zeros_like(tab32), torch.zeros_like(tab32), torch.zeros_like(w32),
                      torch.zeros_like(w32))
    out = sp.alloc_outputs(nb, dev, latent_dim=grid.L * grid.F)
    ws = torch.empty(max(sp.decode_bwd_workspace(g, m, nb), 1), dtype=torch.uint8, device=dev)
    b1, b2 = wt["betas"]
    state = {"step": 0}
    window = None
    if l2_window is not None:
        # opt-in L2 residency over the fp16 tables or the fp32 table gradients
        window = sp.l2_window_set(stream, {"tables": tab16, "grads": gtab}[l2_window])

    def step():
        for b in range(n_batches):
            a, e = b * nb, (b + 1) * nb
            p = pos_all[a:e]
            sp.decode_fwd(g, m, p, tab16, w16, out=out, stream=stream)
            sp.decode_bwd(g, m, p, tab16, w16, {k: v[a:e] for k, v in grads.items()}, gtab, gw, workspace=ws,
                          latent=out["latent"], stream=stream)
        state["step"] += 1
        dp.allreduce_gradients([gtab, gw])     # the step's one exchange (a no-op on one GPU)
        sp.adam_step(tab32, gtab, mt, vt, state["step"], wt["lr"], b1, b2, wt["eps"], params_work=tab16,
                     zero_grad=True, stream=stream)
        sp.adam_step(w32, gw, mw, vw, state["step"], wt["lr"], b1, b2, wt["eps"], params_work=w16,
                     zero_grad=True, stream=stream)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    k = 3
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(k)]
    for i in range(k):
        flush.zero_()
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    ms = dp.max_over_ranks(sum(a.elapsed_time(b) for a, b in evs), device=dev) / k
    if window is not None:
        sp.l2_window_clear(stream)
    return {"metric": "decoded spatiotemporal positions/s (training step: fwd+bwd+Adam)",
            "l2_window": None if window is None else {"over": l2_window, "bytes": window},
            "value": total * world / (ms * 1e-3), "unit": UNIT, "ms_per_step": ms, "launches_per_step": 2 * n_batches + 2,
            "workload": "sports_train_fp16: 150 frames x 300k = 45M positions, 45 launches of 1M (decode_fwd saving z "
                        "+ decode_bwd), then fused Adam (lr 1e-3, betas (0.9, 0.99), eps 1e-15) on 16.8M table and "
                        "6987 weight parameters (fp32 master, fp16 working copy)"}


def _cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


_WORKER = {}


def _init_oracle_worker():
    """Builds the frame, tables and weights once per spawned worker."""
    sys.path.insert(0, ROOT)
    w = S.WORKLOADS[WORKLOAD]
    _WORKER["frame"] = S.sports_scene(w["N"]).frame(w["frame"])
    _WORKER["tables"] = S.hash_tables(w["grid"])
    _WORKER["weights"] = S.mlp_weights(w["mlp"])


def _frame_decode_chunk(task):
    """One worker's share of the oracle's frame decode: (seed, n) -> seconds
    for n positions of the frame, single-threaded (0.2 s of sleep for n = 0,
    which lines every worker up)."""
    seed, n = task
    if n == 0:
        time.sleep(0.2)
        return 0.0
    if not _WORKER:
        _init_oracle_worker()
    from threadpoolctl import threadpool_limits
    from oracle import decoder as dec
    w = S.WORKLOADS[WORKLOAD]
    frame = _WORKER["frame"]
    rows = np.random.default_rng(seed).choice(len(frame), n, replace=False)
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        dec.decode_forward(frame[rows], _WORKER["tables"], _WORKER["weights"], w["grid"], w["mlp"])
        return time.perf_counter() - t0


class OraclePool:
    """Spawned single-threaded worker processes, one per host core (spawn:
    safe after the GPU work of the parent); each builds the workload's inputs
    once, before anything is timed."""

    def __init__(self):
        import multiprocessing as mp
        self.procs = os.cpu_count() or 1
        self.pool = mp.get_context("spawn").Pool(self.procs, initializer=_init_oracle_worker)
        for _ in range(2):   # every worker initialised and busy at once
            self.pool.map(_frame_decode_chunk, [(i, 0) for i in range(self.procs)], chunksize=1)
        self.pool.map(_frame_decode_chunk, [(i, 64) for i in range(self.procs)], chunksize=1)

    def rate(self, per_proc, seed0=100):
        """Positions/s of all workers decoding per_proc positions each."""
        t0 = time.perf_counter()
        self.pool.map(_frame_decode_chunk, [(seed0 + i, per_proc) for i in range(self.procs)], chunksize=1)
        return per_proc * self.procs / (time.perf_counter() - t0)

    def close(self):
        self.pool.close()
        self.pool.join()


def cpu_baseline(n_sample):
    """The oracle, as it stands, on bounded samples of the same workload: one
    thread, and one single-threaded spawned process per host core, each
    decoding an equal share."""
    one = _frame_decode_chunk((7, n_sample))
    pool = OraclePool()
    try:
        per = max(n_sample // 4, 1000)
        all_rate = pool.rate(per)
    finally:
        pool.close()
    return {"value": all_rate, "unit": UNIT, "cores": pool.procs, "kind": "oracle",
            "sample": "%d processes x %d positions of the same frame (numpy fp64, one thread each)" % (pool.procs, per),
            "host_cores": os.cpu_count(), "cpu_model": _cpu_model(),
            "single_core": {"value": n_sample / one, "unit": UNIT, "cores": 1,
                            "sample": "%d positions of the same frame (numpy fp64, BLAS limited to 1 thread)"
                                      % n_sample, "seconds": one}}


def run_reference(args):
    """The reference arm: the oracle, as it stands, on the host's cores (one
    single-threaded spawned process per core, each decoding its own sample of
    the frame every step)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    per = 10_000   # the oracle widens every table column per call: larger samples amortise that
    pool = OraclePool()
    try:
        for i in range(args.warmup):
            pool.rate(per, seed0=1000 * (i + 1))
        t0 = time.perf_counter()
        for i in range(args.steps):
            pool.rate(per, seed0=1000 * (args.warmup + i + 1))
        dt = time.perf_counter() - t0
    finally:
        pool.close()
    value = per * pool.procs * args.steps / dt
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(args.gpus),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": pool.procs, "kind": "oracle",
                             "sample": "%d processes x %d positions of the frame per step" % (pool.procs, per),
                             "cpu_model": _cpu_model()},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from spatiotemporal_neural_field_b200 import build as _b
    if rank == 0:
        _b.build()
    if world > 1:
        dist.barrier()
    from spatiotemporal_neural_field_b200 import spin4d as sp
    from spatiotemporal_neural_field_b200 import dp

    w = S.WORKLOADS[WORKLOAD]
    grid, mlp, N = w["grid"], w["mlp"], w["N"]
    scene = S.sports_scene(N)
    frame_idx = dp.rank_frame(w["frame"], rank, S.N_FRAMES)
    pos_h = scene.frame(frame_idx)
    tables = torch.from_numpy(S.hash_tables(grid)).to(dev)
    weights = torch.from_numpy(S.mlp_weights(mlp)).to(dev)
    pos = torch.from_numpy(pos_h).to(dev)
    g, m = sp.grid_from_spec(grid), sp.mlp_from_spec(mlp)
    out = sp.alloc_outputs(N, dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        sp.decode_fwd(g, m, pos, tables, weights, out=out, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    clocks = ClockSampler(uuid)
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    ms_max = dp.max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), device=dev)
    ms_per_step = ms_max / args.steps
    value = N * world * args.steps / (ms_max * 1e-3)

    # ---- end to end: pinned host input -> decode -> pinned host outputs ----
    # The frame is decoded in chunks on three streams (copy in, compute, copy
    # out) so the host<->device copies of one chunk overlap the decode of the
    # next; every byte of input and output still crosses the host link.  Each
    # chunk costs six copies with a fixed per-copy overhead, so few chunks win:
    # 2-3 chunks 0.47 ms a step, 6 chunks 0.56, 12 chunks 1.10 (the copy-out of
    # 20.4 MB then runs at ~43 GB/s).
    pos_pin = torch.from_numpy(pos_h).pin_memory()
    out_pin = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in out.items()}
    pos_d = torch.empty_like(pos)
    n_chunks = 3
    bounds = [N * c // n_chunks for c in range(n_chunks + 1)]
    s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(n_chunks)]
    ev_cmp = [torch.cuda.Event() for _ in range(n_chunks)]
    ev_out = [torch.cuda.Event() for _ in range(n_chunks)]
    for e in ev_cmp + ev_out:
        e.record(stream)

    def e2e_step():
        for c in range(n_chunks):
            a, b = bounds[c], bounds[c + 1]
            s_in.wait_event(ev_cmp[c])            # previous step's decode of this chunk read pos_d
            with torch.cuda.stream(s_in):
                pos_d[a:b].copy_(pos_pin[a:b], non_blocking=True)
            ev_in[c].record(s_in)
            s_cmp.wait_event(ev_in[c])
            s_cmp.wait_event(ev_out[c])           # previous step's copy-out of this chunk
            sp.decode_fwd(g, m, pos_d[a:b], tables, weights, out={k: v[a:b] for k, v in out.items()}, stream=s_cmp)
            ev_cmp[c].record(s_cmp)
            s_out.wait_event(ev_cmp[c])
            with torch.cuda.stream(s_out):
                for k in out:
                    out_pin[k][a:b].copy_(out[k][a:b], non_blocking=True)
            ev_out[c].record(s_out)

    for _ in range(args.warmup):
        e2e_step()
    torch.cuda.synchronize()
    e_s, e_e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e_s.record(s_in)
    for _ in range(args.steps):
        e2e_step()
    e_e.record(s_out)
    torch.cuda.synchronize()
    te = dp.max_over_ranks(e_s.elapsed_time(e_e), device=dev)
    e2e_value = N * world * args.steps / (te * 1e-3)
    h2d = pos_h.nbytes
    d2h = sum(v.numel() * v.element_size() for v in out.values())

    # ---- fwd+bwd: one 1M-position training launch ----
    fwd_bwd = None
    if not args.no_fwd_bwd:
        wt = S.WORKLOADS["sports_train_fp16"]
        nb = wt["batch"]
        pb = torch.from_numpy(scene.frames(range(0, 4))[:nb]).to(dev)
        gb = {k: torch.randn((nb, wd), device=dev, generator=torch.Generator(device=dev).manual_seed(rank))
              * wt["grad_std"] for k, wd in OUT_WIDTHS.items()}
        outb = sp.alloc_outputs(nb, dev, latent_dim=grid.L * grid.F)
        gtab = torch.zeros((grid.L, 1 << grid.log2_T, grid.F), dtype=torch.float32, device=dev)
        gwt = torch.zeros(mlp.n_params(), dtype=torch.float32, device=dev)
        ws = torch.empty(max(sp.decode_bwd_workspace(g, m, nb), 1), dtype=torch.uint8, device=dev)

        def fb():
            sp.decode_fwd(g, m, pb, tables, weights, out=outb, stream=stream)
            sp.decode_bwd(g, m, pb, tables, weights, gb, gtab, gwt, workspace=ws, latent=outb["latent"], stream=stream)

        for _ in range(max(3, args.warmup // 2)):
            fb()
        torch.cuda.synchronize()
        k = max(3, args.steps // 4)
        evb = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(k)]
        for i in range(k):
            flush.zero_()
            evb[i][0].record(stream)
            fb()
            evb[i][1].record(stream)
        torch.cuda.synchronize()
        tb = dp.max_over_ranks(sum(a.elapsed_time(b) for a, b in evb), device=dev)
        fwd_bwd = {"metric": "decoded spatiotemporal positions/s (fwd+bwd)", "value": nb * world * k /
                   (tb * 1e-3), "unit": UNIT, "ms_per_step": tb / k,
                   "workload": "sports_train_fp16: one 1M-position launch (frames 0-3), decode_fwd (saving z) + decode_bwd (reading z)"}

    # ---- full training step over the 150-frame sequence ----
    train = None
    if not args.no_fwd_bwd:
        train = train_step_measurement(args, sp, torch, dist, dev, world, rank, scene, tables, weights, grid, mlp,
                                       g, m, flush, stream)

    # ---- the same frame decoded in Z-order (spin4d_morton_order + spin4d_permute_rows) ----
    morton = None
    if not args.no_fwd_bwd:
        ws_sort = torch.empty(max(sp.lib.spin4d_morton_order_workspace(N), 1), dtype=torch.uint8, device=dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for _ in range(2):
            flush.zero_()
            a.record(stream)
            _, perm = sp.morton_order(g, pos, workspace=ws_sort, stream=stream)
            pos_sorted = sp.permute_rows(pos, perm, stream=stream)
            b.record(stream)
            torch.cuda.synchronize()
        sort_ms = a.elapsed_time(b)

        def step_sorted():
            sp.decode_fwd(g, m, pos_sorted, tables, weights, out=out, stream=stream)

        for _ in range(args.warmup):
            step_sorted()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for i in range(args.steps):
            flush.zero_()
            evs[i][0].record(stream)
            step_sorted()
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        ms_s = dp.max_over_ranks(sum(x.elapsed_time(y) for x, y in evs), device=dev) / args.steps
        morton = {"value": N * world / (ms_s * 1e-3), "unit": UNIT, "ms_per_step": ms_s,
                  "sort_ms": sort_ms,
                  "note": "the same frame with the Gaussians in Z-order of their normalised positions (sorted once, "
                          "outside the timed steps: the order is per scene, every frame reuses it); "
                          "sort_ms = spin4d_morton_order + spin4d_permute_rows of the positions"}

    gather = None
    if not args.no_probe:
        rates = probe_sector_rates(sp, torch, dev)
        spp = table_sectors_per_position(sp, g, pos, grid.F, 2)
        dec_rate = spp * value / world
        gather = {"table_sectors_per_position": spp,
                  "decoder_sector_rate": dec_rate,
                  "l2_random_sector_rate": rates["l2"], "hbm_random_sector_rate": rates["hbm"],
                  "frac_of_l2_random": dec_rate / rates["l2"], "unit": "sectors/s per GPU",
                  "note": "tables (32 MiB) are L2-resident: the gather ceiling is the measured random "
                          "32-byte-sector rate of an L2-resident buffer (spin4d_probe_gather)"}

    if rank == 0:
        peak, peak_kind = measured_peaks()
        bpp = algorithmic_bytes_per_position()
        achieved = bpp * N / (ms_per_step * 1e-3) / 1e9
        traffic = profiled_traffic()
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f16", "data": "synthetic", "config": workload_config(world),
            "roofline": {"bound": "l2_random_sector", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic, "peak_source": peak_kind,
                         "bytes_per_position": bpp, "io_bytes_per_position": IO_BYTES_PER_POSITION,
                         "kernel": "decode_fwd_tc_kernel<2,32,64>",
                         "note": "achieved = useful table bytes (16 levels x 16 corners x 2 fp16) per position x "
                                 "positions / event time, against the driver's HBM copy peak; the tables (32 MiB) "
                                 "are L2-resident, so the bound is the random 32-byte-sector rate of L2: see frac_l2"},
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": args.steps,
            "clocks": clk,
        }
        if fwd_bwd:
            line["fwd_bwd"] = fwd_bwd
        if gather:
            line["gather_roofline"] = gather
            line["roofline"]["frac_l2"] = gather["frac_of_l2_random"]
            line["roofline"]["l2_probe"] = (
                "spin4d_probe_gather: 4 x SMs blocks of random 16-byte loads (one 32-byte sector each) over a "
                "32 MiB L2-resident buffer, best of 3 timed runs; frac_l2 = the decoder's distinct table sectors "
                "per position (from its own corner indices) x positions/s / that rate")
        if train:
            line["train_step"] = train
        if morton:
            line["morton_sorted"] = morton
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(args.cpu_sample)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def device_ceilings(sp, torch, dev):
    """Measured ceilings of one GPU: random 32-byte-sector and random 128-byte
    line gather rates and sequential read bandwidth for an L2-resident
    (32 MiB) and an HBM-resident (4 GiB) buffer, the random-sector rate of a
    256 MiB buffer, and the fp32 FMA rate."""
    from spatiotemporal_neural_field_b200 import probe as pr
    sms = torch.cuda.get_device_properties(dev).multi_processor_count

    def best(fn, reps=4):
        rate = 0.0
        for it in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            units = fn(it)
            b.record()
            torch.cuda.synchronize()
            if it:
                rate = max(rate, units / (a.elapsed_time(b) * 1e-3))
        return rate

    out = {}
    for name, nbytes, lpt in (("l2", 32 << 20, 4096), ("hbm", 4 << 30, 1024)):
        buf = torch.ones(nbytes // 4, dtype=torch.int32, device=dev)
        out[name + "_random_sector_per_s"] = best(lambda it: pr.probe_gather(buf, 16, lpt, 4 * sms, seed=it + 1))
        out[name + "_random_line128_per_s"] = best(lambda it: pr.probe_gather(buf, 128, lpt, 4 * sms, seed=it + 1))
        passes = 64 if name == "l2" else 2
        out[name + "_sequential_bytes_per_s"] = best(lambda it: pr.probe_stream(buf, passes, 4 * sms))
        ops = 512 if name == "l2" else 128
        for wdt in (8, 16):
            out["%s_random_red%d_per_s" % (name, wdt)] = best(
                lambda it: pr.probe_atomic(buf, wdt, ops, 4 * sms, seed=it + 1))
        for rb in (128, 256):
            out["%s_random_bulk_red%d_rows_per_s" % (name, rb)] = best(
                lambda it: pr.probe_bulk_reduce(buf, ops // 4, 8 * sms, seed=it + 1, row_bytes=rb))
        del buf
    # random sectors of a buffer the size of the paper's tables (256 MiB: about
    # twice the L2, so part of the reads hit it as they do in the decoder)
    buf = torch.ones((256 << 20) // 4, dtype=torch.int32, device=dev)
    out["tables256_random_sector_per_s"] = best(lambda it: pr.probe_gather(buf, 16, 1024, 4 * sms, seed=it + 1))
    del buf
    out["fp32_fma_flop_per_s"] = best(lambda it: pr.probe_fma(1 << 16, 8 * sms, dev))
    return out


def run_l2_window(args):
    """The training step on a created stream: no window, a persisting window
    over the fp16 tables, one over the fp32 table gradients."""
    import torch
    import torch.distributed as dist
    from spatiotemporal_neural_field_b200 import build as _b
    _b.build()
    from spatiotemporal_neural_field_b200 import spin4d as sp
    dev = torch.device("cuda", 0)
    w = S.WORKLOADS[WORKLOAD]
    grid, mlp = w["grid"], w["mlp"]
    g, m = sp.grid_from_spec(grid), sp.mlp_from_spec(mlp)
    scene = S.sports_scene(w["N"])
    tables = torch.from_numpy(S.hash_tables(grid)).to(dev)
    weights = torch.from_numpy(S.mlp_weights(mlp)).to(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    s = torch.cuda.Stream(dev)
    with torch.cuda.stream(s):
        for which in (None, "tables", "grads", None):
            r = train_step_measurement(args, sp, torch, dist, dev, 1, 0, scene, tables, weights, grid, mlp, g, m,
                                       flush, s, l2_window=which)
            print(json.dumps({"workload": "sports_train_fp16 training step", "l2_window": r["l2_window"],
                              "ms_per_step": r["ms_per_step"], "positions_per_s": r["value"]}), flush=True)


def run_workloads(args):
    """Every workload of the build on one GPU: events around each launch (or
    launch pair), L2 flushed before each, median of the timed reps."""
    import torch
    from spatiotemporal_neural_field_b200 import build as _b
    _b.build()
    from spatiotemporal_neural_field_b200 import spin4d as sp
    dev = torch.device("cuda", 0)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    ceil = device_ceilings(sp, torch, dev)
    print(json.dumps({"ceilings": ceil}), flush=True)

    def timed(fn, reps):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    def emit(name, what, n, ms, **extra):
        line = {"workload": name, "pass": what, "positions": n, "ms": ms, "positions_per_s": n / (ms * 1e-3)}
        line.update(extra)
        print(json.dumps(line), flush=True)

    # decoder workloads
    for name in ("tiny_fp32", "sports_frame_fp16", "sports_train_fp16", "stress_fp16_gate"):
        w = S.WORKLOADS[name]
        grid, mlp = w["grid"], w["mlp"]
        g, m = sp.grid_from_spec(grid), sp.mlp_from_spec(mlp)
        if name == "tiny_fp32":
            n, pos = w["N"], S.uniform_positions(w["N"])
        elif name == "sports_frame_fp16":
            n, pos = w["N"], S.sports_scene(w["N"]).frame(w["frame"])
        elif name == "sports_train_fp16":
            n = w["batch"]
            pos = S.sports_scene(300_000).frames(range(4))[:n]
        else:
            n, pos = w["N"], S.stress_positions(w["N"])
        P = torch.from_numpy(pos).to(dev)
        T = torch.from_numpy(S.hash_tables(grid)).to(dev)
        W = torch.from_numpy(S.mlp_weights(mlp)).to(dev)
        cr = torch.from_numpy(S.gate_params(n)).to(dev) if mlp.gate else None
        out = sp.alloc_outputs(n, dev, latent_dim=grid.L * grid.F)
        fwd_out = {k: v for k, v in out.items() if k != "latent"}
        reps = 20 if n <= 1_000_000 else 7
        ms = timed(lambda: sp.decode_fwd(g, m, P, T, W, cr, out=fwd_out), reps)
        spp = table_sectors_per_position(sp, g, P, grid.F, 2 if grid.dtype == "f16" else 4)
        rate = spp * n / (ms * 1e-3)
        where = "hbm" if name == "stress_fp16_gate" else "l2"
        emit(name, "fwd", n, ms, table_sectors_per_position=spp, sector_rate=rate,
             frac_of_random_sector_ceiling=rate / ceil[where + "_random_sector_per_s"], ceiling=where)
        if name in ("sports_frame_fp16", "stress_fp16_gate"):
            ws_sort = torch.empty(max(sp.lib.spin4d_morton_order_workspace(n), 1), dtype=torch.uint8, device=dev)
            for _ in range(2):   # the first call allocates the outputs; time the second
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                flush.zero_()
                a.record()
                _, perm = sp.morton_order(g, P, workspace=ws_sort)
                Ps = sp.permute_rows(P, perm)
                crs = sp.permute_rows(cr, perm) if cr is not None else None
                b.record()
                torch.cuda.synchronize()
            ms_s = timed(lambda: sp.decode_fwd(g, m, Ps, T, W, crs, out=fwd_out), reps)
            emit(name, "fwd (Z-order sorted)", n, ms_s, sort_and_permute_ms=a.elapsed_time(b),
                 table_sectors_per_position=spp, sector_rate=spp * n / (ms_s * 1e-3))
            del Ps, crs, perm, ws_sort
        if name == "sports_frame_fp16":
            continue
        grads = {k: torch.randn((n, wd), device=dev) * (1e-2 if grid.dtype == "f16" else 1.0)
                 for k, wd in OUT_WIDTHS.items()}
        gt = torch.zeros((grid.L, 1 << grid.log2_T, grid.F), dtype=torch.float32, device=dev)
        gw = torch.zeros(mlp.n_params(), dtype=torch.float32, device=dev)
        ws = torch.empty(max(sp.decode_bwd_workspace(g, m, n), 1), dtype=torch.uint8, device=dev)

        def fb():
            sp.decode_fwd(g, m, P, T, W, cr, out=out)
            sp.decode_bwd(g, m, P, T, W, grads, gt, gw, gate_cr=cr, workspace=ws, latent=out["latent"])

        emit(name, "fwd+bwd (saved latent)", n, timed(fb, reps))
        gpos = torch.zeros((n, 3), device=dev)

        def fbp():
            sp.decode_fwd(g, m, P, T, W, cr, out=out)
            sp.decode_bwd(g, m, P, T, W, grads, gt, gw, gate_cr=cr, workspace=ws, latent=out["latent"], grad_pos=gpos)

        emit(name, "fwd+bwd+position gradient (saved latent)", n, timed(fbp, reps))
        del P, T, W, out, fwd_out, grads, gt, gw, ws, gpos
        torch.cuda.empty_cache()

    # the paper's four-head GELU decoder, one 1M-position training launch, at
    # the measured table size 2^21 and at 2^23 (SPIN-4DGS section 4, Table 5)
    for log2_T in (21, 23):
        paper_heads_workload(sp, torch, dev, timed, emit, ceil, log2_T)

    # HexPlane
    w = S.WORKLOADS["hexplane_fp32"]
    hx, n = w["hex"], w["N"]
    h = sp.hex_from_spec(hx)
    inp = {k: torch.from_numpy(v).to(dev) for k, v in S.hexplane_inputs(n).items()}
    planes = torch.from_numpy(S.hexplane_planes(hx)).to(dev)
    weights = torch.from_numpy(S.hexplane_weights(hx)).to(dev)
    out = {k: torch.empty((n, wd), device=dev) for k, wd in sp.HEX_KEYS}
    lat = torch.empty((n, hx.in_dim), device=dev)
    grads = {k: torch.randn((n, wd), device=dev) for k, wd in S.HEX_OUT_WIDTHS.items()}
    gp = torch.zeros(hx.n_plane_floats(), device=dev)
    gw = torch.zeros(hx.n_params(), device=dev)
    ws = torch.empty(max(sp.hexplane_bwd_workspace(h, n), 1), dtype=torch.uint8, device=dev)
    lines = len(hx.scales) * 6 * 4   # 128-byte plane rows per Gaussian
    ms = timed(lambda: sp.hexplane_fwd(h, inp, planes, weights, out=out), 20)
    emit("hexplane_fp32", "fwd", n, ms, plane_lines_per_gaussian=lines,
         frac_of_l2_random_line_ceiling=lines * n / (ms * 1e-3) / ceil["l2_random_line128_per_s"])
    out_l = dict(out, latent=lat)
    hid = torch.empty((n, hx.hidden), device=dev)
    out_h = dict(out_l, hidden=hid)

    def hfb():
        sp.hexplane_fwd(h, inp, planes, weights, out=out_l)
        sp.hexplane_bwd(h, inp, planes, weights, grads, gp, gw, workspace=ws, latent=lat)

    def hfb_h1():
        sp.hexplane_fwd(h, inp, planes, weights, out=out_h)
        sp.hexplane_bwd(h, inp, planes, weights, grads, gp, gw, workspace=ws, latent=lat, hidden=hid)

    emit("hexplane_fp32", "fwd+bwd (saved latent)", n, timed(hfb, 10))
    emit("hexplane_fp32", "fwd+bwd (saved latent and h1)", n, timed(hfb_h1, 10))
    emit("hexplane_fp32", "bwd (saved latent and h1)", n,
         timed(lambda: sp.hexplane_bwd(h, inp, planes, weights, grads, gp, gw, workspace=ws, latent=lat, hidden=hid),
               10))
    emit("hexplane_fp32", "bwd (gathering again)", n,
         timed(lambda: sp.hexplane_bwd(h, inp, planes, weights, grads, gp, gw, workspace=ws), 10))
    del inp, planes, weights, out, lat, grads, gp, gw, ws, out_l, hid, out_h
    torch.cuda.empty_cache()
    render_workloads(sp, torch, dev, timed)
    sp.check_device_errors()


def paper_heads_workload(sp, torch, dev, timed, emit, ceil, log2_T):
    """Times the paper decoder's 1M-position launch at table size 2^log2_T."""
    w = S.WORKLOADS["paper_heads_fp16"]
    grid, spec, n = dataclasses.replace(w["grid"], log2_T=log2_T), w["heads"], w["N"]
    name = "paper_heads_fp16" if log2_T == 21 else "paper_heads_fp16_T2^%d" % log2_T
    g, h = sp.grid_from_spec(grid), sp.heads_from_spec(spec)
    P = torch.from_numpy(S.sports_scene(300_000).frames(range(4))[:n]).to(dev)
    T = torch.from_numpy(S.hash_tables(grid)).to(dev)
    W = torch.from_numpy(S.heads_weights(spec)).to(dev)
    out = sp.heads_fwd(g, h, P, T, W, latent=True, raw=True)
    fwd_out = {k: v for k, v in out.items() if k not in ("latent", "raw")}
    ms = timed(lambda: sp.heads_fwd(g, h, P, T, W, out=fwd_out), 10)
    spp = table_sectors_per_position(sp, g, P, grid.F, 2)
    emit(name, "fwd", n, ms, table_sectors_per_position=spp, sector_rate=spp * n / (ms * 1e-3),
         frac_of_256mib_random_sector_ceiling=spp * n / (ms * 1e-3) / ceil["tables256_random_sector_per_s"],
         mlp_flop_per_position=2 * sum(o * i for hd_ in range(4) for o, i in spec.layer_shapes(hd_)))
    # the same launch decoded in Z-order (sorted once per scene; outputs in sorted order)
    ws_sort = torch.empty(max(sp.lib.spin4d_morton_order_workspace(n), 1), dtype=torch.uint8, device=dev)
    _, perm = sp.morton_order(g, P, workspace=ws_sort)
    Ps = sp.permute_rows(P, perm)
    ms_s = timed(lambda: sp.heads_fwd(g, h, Ps, T, W, out=fwd_out), 10)
    emit(name, "fwd (Z-order sorted)", n, ms_s, table_sectors_per_position=spp,
         sector_rate=spp * n / (ms_s * 1e-3),
         frac_of_256mib_random_sector_ceiling=spp * n / (ms_s * 1e-3) / ceil["tables256_random_sector_per_s"])
    del Ps, perm, ws_sort
    grads = {k: torch.randn((n, wd), device=dev) * w["grad_std"]
             for k, wd in dict(S.HEADS_OUT_WIDTHS, sh=spec.sh_dim).items()}
    gt = torch.zeros((grid.L, 1 << grid.log2_T, grid.F), device=dev)
    gw = torch.zeros(spec.n_params(), device=dev)
    ws = torch.empty(max(sp.lib.spin4d_heads_bwd_workspace(ctypes.byref(g), ctypes.byref(h), n), 1),
                     dtype=torch.uint8, device=dev)

    def hfb():
        sp.heads_fwd(g, h, P, T, W, out=out)
        sp.heads_bwd(g, h, P, T, W, grads, gt, gw, latent=out["latent"], raw=out["raw"], workspace=ws)

    emit(name, "fwd (saving z and raw head outputs) + bwd", n, timed(hfb, 5))
    sp.heads_fwd(g, h, P, T, W, out=out)
    emit(name, "bwd (saved z and raw head outputs)", n,
         timed(lambda: sp.heads_bwd(g, h, P, T, W, grads, gt, gw, latent=out["latent"], raw=out["raw"], workspace=ws),
               5))
    del P, T, W, out, fwd_out, grads, gt, gw, ws
    torch.cuda.empty_cache()


def render_workloads(sp, torch, dev, timed):
    """EWA projection + tile compositing of one sports frame (300k Gaussians,
    SH degree 3) at the Panoptic Sports resolution 640 x 360: forward as
    separate launches and as one CUDA graph, forward+backward, and the
    paper's decoder followed by the render (a whole decoded frame)."""
    spec = S.orbit_camera(640, 360)
    sc = S.render_scene(300_000, seed=0)
    n = sc["mu"].shape[0]
    cam, desc = sp.camera_from_spec(spec), sp.render_desc(sh_degree=3)
    args = [torch.from_numpy(sc[k]).to(dev) for k in ("mu", "cov", "opacity", "colours")]
    img, st = sp.render(cam, desc, *args)
    T = torch.empty((360, 640), device=dev)
    pairs = st.pairs_needed()

    def fwd():
        sp.render_fwd(cam, desc, *args, image=img, final_T=T, state=st)

    def line(what, ms, **extra):
        d = {"workload": "render_sports_frame", "pass": what, "gaussians": n, "width": 640, "height": 360,
             "ms": ms, "frames_per_s": 1e3 / ms, "gaussians_per_s": n / (ms * 1e-3), "tile_pairs": pairs}
        d.update(extra)
        print(json.dumps(d), flush=True)

    line("fwd (separate launches)", timed(fwd, 20))
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fwd()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            fwd()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    line("fwd (one CUDA graph)", timed(graph.replay, 20))
    G = torch.from_numpy(S.image_grads(spec)).to(dev)
    grads = [torch.zeros((n, 3), device=dev), torch.zeros((n, 6), device=dev), torch.zeros(n, device=dev),
             torch.zeros((n, 48), device=dev)]

    def fb():
        fwd()
        sp.render_bwd(cam, desc, *args, G, st, *grads)

    line("fwd+bwd (separate launches)", timed(fb, 20))
    del graph

    # the paper's decoder on the same frame, then the render of its output
    grid, spec_h = S.GRID_PAPER, S.HEADS_PAPER
    g, h = sp.grid_from_spec(grid), sp.heads_from_spec(spec_h)
    P = torch.from_numpy(S.sports_scene(n).frame(75)).to(dev)
    Tb = torch.from_numpy(S.hash_tables(grid)).to(dev)
    W = torch.from_numpy(S.heads_weights(spec_h)).to(dev)
    out = sp.heads_fwd(g, h, P, Tb, W)
    desc4 = sp.render_desc(sh_degree=3, mean_stride=4)
    dimg, dst = sp.render(cam, desc4, P, out["cov"], out["opacity"], out["sh"])

    def dr():
        sp.heads_fwd(g, h, P, Tb, W, out=out)
        sp.render_fwd(cam, desc4, P, out["cov"], out["opacity"], out["sh"], image=dimg, state=dst)

    ms = timed(dr, 10)
    print(json.dumps({"workload": "decode_and_render_frame", "pass": "paper decoder fwd + render fwd",
                      "gaussians": n, "width": 640, "height": 360, "ms": ms, "frames_per_s": 1e3 / ms,
                      "tile_pairs": dst.pairs_needed(),
                      "note": "decoder at its initial state (scale e^-5, opacity 0.1, SH 0)"}), flush=True)


def _oracle_chunk(task):
    """One worker's share of an oracle timing (runs in a spawned process)."""
    name, what, rows_seed, n = task
    from threadpoolctl import threadpool_limits
    sys.path.insert(0, ROOT)
    with threadpool_limits(limits=1):
        fn = _oracle_job(name, what, n, rows_seed)
        t0 = time.perf_counter()
        fn()
        return time.perf_counter() - t0


def _oracle_job(name, what, n, seed):
    """The oracle's forward (or forward+backward) on n positions of a workload
    (for the render: n sampled pixels of the frame)."""
    from oracle import decoder as dec, hexplane as hxo, render as rdo
    rng = np.random.default_rng(seed)
    if name == "render_sports_frame":
        spec = S.orbit_camera(640, 360)
        sc = S.render_scene(300_000, seed=0)
        cam = rdo.Camera(view=np.array(spec.view, np.float64), fx=spec.fx, fy=spec.fy, cx=spec.cx, cy=spec.cy,
                         width=spec.width, height=spec.height, z_near=spec.z_near)
        pix = np.stack([rng.integers(0, 640, n), rng.integers(0, 360, n)], axis=1)
        return lambda: rdo.render_pixels(cam, rdo.Settings(sh_degree=3), sc["mu"], sc["cov"], sc["opacity"],
                                         sc["colours"], pix)
    if name == "hexplane_fp32":
        hx = S.WORKLOADS[name]["hex"]
        inp = S.hexplane_inputs(n, seed)
        planes, weights = S.hexplane_planes(hx), S.hexplane_weights(hx)
        if what == "fwd":
            return lambda: hxo.forward(inp, planes, weights, hx)
        grads = S.upstream_grads(n, S.HEX_OUT_WIDTHS, 1.0, seed)
        return lambda: (hxo.forward(inp, planes, weights, hx), hxo.backward(inp, planes, weights, hx, grads))
    w = S.WORKLOADS[name]
    grid, mlp = w["grid"], w["mlp"]
    if name == "tiny_fp32":
        pos = S.uniform_positions(w["N"])
    elif name == "stress_fp16_gate":
        pos = S.stress_positions(1_000_000)
    else:
        pos = S.sports_scene(300_000).frame(w.get("frame", 75))
    pos = pos[rng.choice(len(pos), min(n, len(pos)), replace=False)]
    tables, weights = S.hash_tables(grid), S.mlp_weights(mlp)
    cr = S.gate_params(len(pos), seed) if mlp.gate else None
    if what == "fwd":
        return lambda: dec.decode_forward(pos, tables, weights, grid, mlp, gate_cr=cr)
    grads = S.upstream_grads(len(pos), S.DECODE_OUT_WIDTHS, 1e-2, seed)
    return lambda: (dec.decode_forward(pos, tables, weights, grid, mlp, gate_cr=cr),
                    dec.decode_backward(pos, tables, weights, grid, mlp, grads, gate_cr=cr))


def run_cpu_workloads(args):
    """The oracle, as it stands, on a bounded sample of every workload: one
    thread, and a pool of spawned single-threaded processes (one per core, at
    most 32) over equal shares of a larger sample.  The stress workload gets
    the single-thread timing only: the oracle widens its 512 MiB of tables to
    fp64 per call, too much memory to hold once per process."""
    import multiprocessing as mp
    procs = min(os.cpu_count() or 1, 32)
    jobs = [("tiny_fp32", "fwd", 4096), ("tiny_fp32", "fwd+bwd", 4096), ("sports_frame_fp16", "fwd", 20_000),
            ("sports_train_fp16", "fwd+bwd", 10_000), ("stress_fp16_gate", "fwd", 10_000),
            ("hexplane_fp32", "fwd", 2_000), ("hexplane_fp32", "fwd+bwd", 1_000),
            ("render_sports_frame", "fwd", 64)]
    ctx = mp.get_context("spawn")
    with ctx.Pool(procs) as pool:
        pool.map(_oracle_chunk, [("tiny_fp32", "fwd", i, 64) for i in range(procs)])   # start every worker
        for name, what, n in jobs:
            one = _oracle_chunk((name, what, 1, n))
            line = {"workload": name, "pass": what, "kind": "oracle", "sample": n,
                    "positions_per_s_1_thread": n / one, "host_cores": os.cpu_count()}
            if name == "render_sports_frame":
                # the projection of all 300k Gaussians is paid once per frame, the blend per pixel
                proj = _oracle_chunk((name, what, 1, 0))
                frame = proj + (one - proj) * 640 * 360 / n
                line = {"workload": name, "pass": what, "kind": "oracle", "sample_pixels": n,
                        "sample_s": one, "projection_s": proj, "frame_s_1_thread_extrapolated": frame,
                        "host_cores": os.cpu_count()}
                print(json.dumps(line), flush=True)
                continue
            if name != "stress_fp16_gate":
                t0 = time.perf_counter()
                pool.map(_oracle_chunk, [(name, what, 100 + i, n) for i in range(procs)])
                line["positions_per_s_pool"] = n * procs / (time.perf_counter() - t0)
                line["pool_processes"] = procs
            print(json.dumps(line), flush=True)


def run_ncu_case(name):
    """A few untimed launches of one workload, for an ncu capture."""
    import torch
    from spatiotemporal_neural_field_b200 import build as _b
    _b.build()
    from spatiotemporal_neural_field_b200 import spin4d as sp
    dev = torch.device("cuda", 0)
    w = S.WORKLOADS.get(name)
    if name == "paper_heads_fp16":
        # 200k positions (a small case of the 1M launch): forward saving z, then the backward
        grid, spec_h = w["grid"], w["heads"]
        n = 200_000
        g, h = sp.grid_from_spec(grid), sp.heads_from_spec(spec_h)
        P = torch.from_numpy(S.sports_scene(300_000).frames(range(4))[:n]).to(dev)
        T = torch.from_numpy(S.hash_tables(grid)).to(dev)
        W = torch.from_numpy(S.heads_weights(spec_h)).to(dev)
        grads = {k: torch.randn((n, wd), device=dev) * w["grad_std"]
                 for k, wd in dict(S.HEADS_OUT_WIDTHS, sh=spec_h.sh_dim).items()}
        gt = torch.zeros((grid.L, 1 << grid.log2_T, grid.F), device=dev)
        gw = torch.zeros(spec_h.n_params(), device=dev)
        for _ in range(2):
            out = sp.heads_fwd(g, h, P, T, W, latent=True, raw=True)
            sp.heads_bwd(g, h, P, T, W, grads, gt, gw, latent=out["latent"], raw=out["raw"])
        torch.cuda.synchronize()
        sp.check_device_errors()
        print("ncu case done:", name)
        return
    if name == "render_sports_frame":
        spec = S.orbit_camera(640, 360)
        sc = S.render_scene(300_000, seed=0)
        cam, desc = sp.camera_from_spec(spec), sp.render_desc(sh_degree=3)
        args = [torch.from_numpy(sc[k]).to(dev) for k in ("mu", "cov", "opacity", "colours")]
        G = torch.from_numpy(S.image_grads(spec)).to(dev)
        img, st = sp.render(cam, desc, *args)
        for _ in range(3):
            sp.render_fwd(cam, desc, *args, image=img, state=st)
            sp.render_bwd(cam, desc, *args, G, st)
        torch.cuda.synchronize()
        sp.check_device_errors()
        print("ncu case done:", name)
        return
    if name == "hexplane_fwd_fp32":
        # the forward alone (no saved latent), as the timed forward line runs it
        w = S.WORKLOADS["hexplane_fp32"]
        hx, n = w["hex"], w["N"]
        inp = {k: torch.from_numpy(v).to(dev) for k, v in S.hexplane_inputs(n).items()}
        planes = torch.from_numpy(S.hexplane_planes(hx)).to(dev)
        weights = torch.from_numpy(S.hexplane_weights(hx)).to(dev)
        h = sp.hex_from_spec(hx)
        out = {k: torch.empty((n, wd), device=dev) for k, wd in sp.HEX_KEYS}
        for _ in range(3):
            sp.hexplane_fwd(h, inp, planes, weights, out=out)
        torch.cuda.synchronize()
        sp.check_device_errors()
        print("ncu case done:", name)
        return
    if name == "hexplane_fp32":
        hx = w["hex"]
        n = w["N"]
        inp = {k: torch.from_numpy(v).to(dev) for k, v in S.hexplane_inputs(n).items()}
        planes = torch.from_numpy(S.hexplane_planes(hx)).to(dev)
        weights = torch.from_numpy(S.hexplane_weights(hx)).to(dev)
        h = sp.hex_from_spec(hx)
        grads = {k: torch.randn((n, wd), device=dev) for k, wd in S.HEX_OUT_WIDTHS.items()}
        gp = torch.zeros(hx.n_plane_floats(), device=dev)
        gw = torch.zeros(hx.n_params(), device=dev)
        out = {k: torch.empty((n, wd), device=dev) for k, wd in sp.HEX_KEYS}
        out["latent"] = torch.empty((n, hx.in_dim), device=dev)
        out["hidden"] = torch.empty((n, hx.hidden), device=dev)
        for _ in range(3):   # a training step: forward saving the latent and h1, backward reading them
            sp.hexplane_fwd(h, inp, planes, weights, out=out)
            sp.hexplane_bwd(h, inp, planes, weights, grads, gp, gw, latent=out["latent"], hidden=out["hidden"])
    else:
        grid, mlp = w["grid"], w["mlp"]
        g, m = sp.grid_from_spec(grid), sp.mlp_from_spec(mlp)
        if name == "stress_fp16_gate":
            n = w["N"]
            pos = S.stress_positions(n)
        elif name == "sports_train_fp16":
            n = w["batch"]
            pos = S.sports_scene(300_000).frames(range(4))[:n]
        elif name == "tiny_fp32":
            n = w["N"]
            pos = S.uniform_positions(n)
        else:
            n = w["N"]
            pos = S.sports_scene(n).frame(w["frame"])
        P = torch.from_numpy(pos).to(dev)
        T = torch.from_numpy(S.hash_tables(grid)).to(dev)
        W = torch.from_numpy(S.mlp_weights(mlp)).to(dev)
        cr = torch.from_numpy(S.gate_params(n)).to(dev) if mlp.gate else None
        out = sp.alloc_outputs(n, dev, latent_dim=grid.L * grid.F)
        bwd = name in ("sports_train_fp16", "tiny_fp32")
        if bwd:
            grads = {k: torch.randn((n, wd), device=dev) * 1e-2 for k, wd in OUT_WIDTHS.items()}
            gt = torch.zeros((grid.L, 1 << grid.log2_T, grid.F), device=dev)
            gw = torch.zeros(mlp.n_params(), device=dev)
        for _ in range(3):
            sp.decode_fwd(g, m, P, T, W, cr, out=out)
            if bwd:
                sp.decode_bwd(g, m, P, T, W, grads, gt, gw, gate_cr=cr, latent=out["latent"])
    torch.cuda.synchronize()
    sp.check_device_errors()
    print("ncu case done:", name)


def main():
    args = parse()
    if args.ncu_case:
        run_ncu_case(args.ncu_case)
        return
    if args.l2_window:
        return run_l2_window(args)
    if args.cpu_workloads:
        run_cpu_workloads(args)
        return
    if args.workloads:
        run_workloads(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

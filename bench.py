#!/usr/bin/env python
"""Benchmark of the lightning vecset decoder hot path on B200.

One step = the whole hot path for one shape per rank: K/V projection of a
3072-token vecset, then hierarchical volume decoding 96^3 -> 192^3 -> 384^3
with adaptive KV selection on the fine levels (boundary marking, dilation,
compaction, sub-volume packing, probe scoring, Top-K, gathered decode,
inherit fill).  Inputs are seeded synthetic arrays with the workload's shapes
(latents N(0,1), weights N(0,0.02^2) rounded to bf16, a union of 16 spheres
plus 0.01 tanh(decoder)); the real Hunyuan3D-2 latents and weights are not
available.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl vdm|reference] [--config 4]

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle on
a bounded sample of the same workload (rank 0 only).
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

import numpy as np  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "SDF query points/sec & ms/shape (384³ hierarchical); % of bf16 TC / HBM peak"
UNIT = "points/s"
L2_FLUSH_BYTES = 512 << 20     # > 126 MB L2


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16": d["bf16_tflops"], "bf16_sust": d["bf16_tflops_sustained"],
                "sm_max_mhz": d.get("sm_max_mhz", 1965.0), "src": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sust": 1400.0, "sm_max_mhz": 1965.0,
                "src": "fallback"}


# dram__bytes_read.sum + dram__bytes_write.sum per decode launch, mean over the five
# launches of one config-4 shape, captured with ncu on the bench's own launches
# (profiles/launches_config4_hierarchical_384.md); re-capture when the kernel changes.
DECODE_DRAM_BYTES_PER_LAUNCH = {4: 40.18e6}


def decode_flops_per_query(spec: W.DecoderSpec, n_tokens: int) -> float:
    """Algorithmic FLOPs of one decoded query: 2 x multiply-adds of the Q
    projection (51 embedding lanes), attention (QK^T and PV over n_tokens), output
    projection, MLP and head."""
    C, H, F = spec.C, spec.H, spec.F
    macs = 51 * C + 2 * H * n_tokens * 64 + C * C + 2 * C * F + C
    return 2.0 * macs


def select_flops_per_probe(spec: W.DecoderSpec) -> float:
    """Scoring pass per probe: Q projection + QK^T over all tokens, twice
    (normaliser, then weights)."""
    return 2.0 * (51 * spec.C + 2 * spec.H * spec.N * 64)


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu: int):
        self.gpu = gpu
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) >= 9:
                rows.append(f)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def _dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def run_vdm(args, world, rank, local):
    import datetime

    import torch
    import torch.distributed as dist

    import neural_sdf_volume_b200 as vdm
    from neural_sdf_volume_b200 import shard

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    cfg = W.CONFIGS[args.config]
    assert cfg.mode == "hier"
    # each rank decodes its own shape(s): weak scaling, no data-path collective
    my_shapes = shard.shapes_for_rank(cfg.B * world, rank, world)
    inp = W.make_decoder(cfg.dec, seed=0, key=cfg.seed_key, B=cfg.B * world)
    spheres_all = W.make_spheres(cfg.n_spheres, 0, cfg.sphere_key, cfg.B * world)
    z_np = np.ascontiguousarray(inp["z"][my_shapes])
    sp_np = np.ascontiguousarray(spheres_all[my_shapes])
    B = len(my_shapes)
    dec = vdm.Decoder.from_numpy(inp["weights"], cfg.dec.C, cfg.dec.H, cfg.dec.F, cfg.dec.query_ln,
                                 cfg.dec.dtype, device=dev)
    z = torch.from_numpy(z_np).to(dev)
    spheres = torch.from_numpy(sp_np).to(dev)
    params = vdm.hier_params(cfg.r0, cfg.n_levels, cfg.adaptive, cfg.tile, cfg.n_probe, cfg.top_k, 0)
    ws = torch.empty((vdm.vdm_hierarchical_workspace_size(dec, params, cfg.dec.N),), device=dev,
                     dtype=torch.uint8)
    Rf = cfg.r_final
    out = torch.empty((B, Rf, Rf, Rf), device=dev, dtype=torch.float32)
    flush = torch.empty((L2_FLUSH_BYTES // 4,), device=dev, dtype=torch.float32)
    stream = torch.cuda.current_stream(dev)

    def step(zin):
        K, V = vdm.vdm_precompute_kv(dec, zin)
        _, st = vdm.vdm_decode_hierarchical(dec, K, V, params, spheres, cfg.dec_scale, workspace=ws, out=out)
        return st

    for _ in range(args.warmup):
        stats = step(z)
    torch.cuda.synchronize(dev)

    # ---------------- device-timed region: inputs resident in HBM
    clocks = ClockSampler(local)
    shard.barrier(dev)
    torch.cuda.synchronize(dev)
    clocks.start()
    vdm.vdm_profile_begin()
    evs = []
    for _ in range(args.steps):
        flush.zero_()                       # L2 flush between timed steps (outside the events)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        stats = step(z)
        e1.record(stream)
        evs.append((e0, e1))
    torch.cuda.synchronize(dev)
    prof = vdm.vdm_profile_end()
    clk = clocks.stop()
    shard.barrier(dev)
    torch.cuda.synchronize(dev)
    step_ms = [a.elapsed_time(b) for a, b in evs]
    my_ms = sum(step_ms) / len(step_ms)
    ms = shard.max_over_ranks(my_ms, dev)

    # decoded queries and algorithmic work per step (this rank's shapes)
    dense_q, sparse_q = 0, 0
    for s in stats:
        dense_q += s["decoded"][0]
        for l in range(1, cfg.n_levels):
            if cfg.adaptive:
                dense_q += s["probes"][l]
                sparse_q += s["decoded"][l] - s["probes"][l]
            else:
                dense_q += s["decoded"][l]
    decoded = dense_q + sparse_q
    k = min(cfg.top_k, cfg.dec.N)
    dec_flops = dense_q * decode_flops_per_query(cfg.dec, cfg.dec.N) + \
        sparse_q * decode_flops_per_query(cfg.dec, k)
    total_decoded = shard.sum_over_ranks(decoded, dev)
    value = total_decoded / (ms / 1e3)

    # ---------------- end to end: host latents in, host volume out (pinned)
    z_host = torch.from_numpy(z_np).pin_memory()
    out_host = torch.empty(out.shape, dtype=torch.float32).pin_memory()
    z_dev = torch.empty_like(z)
    for _ in range(2):
        z_dev.copy_(z_host, non_blocking=True)
        step(z_dev)
        out_host.copy_(out, non_blocking=True)
    torch.cuda.synchronize(dev)
    shard.barrier(dev)
    e2e = []
    for _ in range(args.steps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        z_dev.copy_(z_host, non_blocking=True)
        step(z_dev)
        out_host.copy_(out, non_blocking=True)
        e1.record(stream)
        e2e.append((e0, e1))
    torch.cuda.synchronize(dev)
    e2e_ms = shard.max_over_ranks(sum(a.elapsed_time(b) for a, b in e2e) / len(e2e), dev)

    peaks = _peaks()
    dec_prof = prof["decode"]
    decode_ms_step = dec_prof["ms"] / args.steps
    achieved_tflops = dec_flops / (decode_ms_step / 1e3) / 1e12 if decode_ms_step > 0 else 0.0
    # the fused decoder runs on the bf16 tensor cores; it is timed inside a long
    # step, so the sustained (power-capped) bf16 matmul peak is the denominator
    tc_peak = peaks["bf16_sust"]
    launches = sum(v["launches"] for v in prof.values())
    sel_flops = sum(s["selected_tiles"][l] for s in stats for l in range(cfg.n_levels)) * \
        cfg.n_probe * select_flops_per_probe(cfg.dec) / 2.0   # one scoring pass
    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"config {cfg.cid}: {cfg.name}, N={cfg.dec.N}, C={cfg.dec.C}, "
                               f"H={cfg.dec.H}, F={cfg.dec.F}, top_k={cfg.top_k}, {cfg.n_spheres} spheres",
                   "shapes_per_gpu": B, "final_resolution": Rf, "l2": "flushed between timed steps",
                   "parallelism": f"shape-sharded x{world}"},
        "ms_per_shape": ms / B,
        "decoded_points_per_shape": decoded / B,
        "queries_saved_vs_dense": 1.0 - decoded / (B * Rf ** 3),
        "effective_voxels_per_s": B * world * Rf ** 3 / (ms / 1e3),
        "e2e": {"value": total_decoded / (e2e_ms / 1e3), "unit": UNIT, "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": int(z_host.numel() * 4),
                "d2h_bytes_per_step": int(out_host.numel() * 4)},
        "roofline": {"kernel": "decode_tc_kernel", "bound": "tensor", "achieved": achieved_tflops,
                     "peak": tc_peak, "unit": "TFLOP/s", "frac": achieved_tflops / tc_peak,
                     "traffic": DECODE_DRAM_BYTES_PER_LAUNCH.get(cfg.cid),
                     "traffic_note": "DRAM bytes read + written per decode launch (mean of the step's "
                                     "launches) from ncu on this workload's own launches; null where "
                                     "not captured for the current kernel",
                     "peak_note": "measured sustained bf16 matmul peak (MEASURED_PEAKS.json), "
                                  f"{peaks['src']}; algorithmic FLOPs: {dec_flops / 1e12:.2f} TFLOP/step"},
        "select_roofline": {"kernel": "select_tc_kernel", "achieved":
                            (sel_flops / (prof["select"]["ms"] / args.steps / 1e3) / 1e12)
                            if prof["select"]["ms"] > 0 else 0.0, "unit": "TFLOP/s"},
        "kernels": {k2: {"launches": v["launches"], "ms_per_step": v["ms"] / args.steps}
                    for k2, v in prof.items()},
        "gpu_launches": launches,
        "stats": {"decoded_per_level": stats[0]["decoded"][:cfg.n_levels],
                  "probes_per_level": stats[0]["probes"][:cfg.n_levels],
                  "tiles_per_level": stats[0]["tiles"][:cfg.n_levels],
                  "selected_tiles_per_level": stats[0]["selected_tiles"][:cfg.n_levels]},
        "clocks": clk,
        "peaks": peaks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(cfg, seconds=args.cpu_seconds)
    if world > 1:
        dist.destroy_process_group()
    return res


def run_dense(args, world, rank, local):
    """Dense decoding on one GPU: the full grid of a dense workload (``--config 1``:
    32^3 fp32, ``--config 2``: 128^3 bf16), or ``--dense-queries M`` uniform random
    points with the workload-2 decoder (N=3072, C=512, 8 heads, F=2048)."""
    import torch

    import neural_sdf_volume_b200 as vdm
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    cfg = W.CONFIGS[args.config if args.config in (1, 2) else 2]
    inp = W.make_decoder(cfg.dec, seed=0, key=cfg.seed_key, B=1)
    dec = vdm.Decoder.from_numpy(inp["weights"], cfg.dec.C, cfg.dec.H, cfg.dec.F, cfg.dec.query_ln,
                                 cfg.dec.dtype, device=dev)
    K, V = vdm.vdm_precompute_kv(dec, torch.from_numpy(inp["z"]).to(dev))
    if args.dense_queries > 0:
        M = args.dense_queries
        pts = torch.from_numpy(W.make_points(M, seed=1, key=2)).to(dev)
        call = lambda out: vdm.vdm_decode_dense(dec, K, V, xyz=pts, out=out)
        workload = f"dense decode of {M} uniform points, config 2 decoder"
    else:
        M = cfg.grid_R ** 3
        pts = None
        call = lambda out: vdm.vdm_decode_dense(dec, K, V, grid_R=cfg.grid_R, out=out)
        workload = f"config {cfg.cid}: {cfg.name}"
    out = torch.empty((1, M), device=dev)
    flush = torch.empty((L2_FLUSH_BYTES // 4,), device=dev, dtype=torch.float32)
    for _ in range(args.warmup):
        call(out)
    torch.cuda.synchronize(dev)
    evs = []
    for _ in range(args.steps):
        flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        call(out)
        e1.record()
        evs.append((e0, e1))
    torch.cuda.synchronize(dev)
    ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
    flops = M * decode_flops_per_query(cfg.dec, cfg.dec.N)
    peaks = _peaks()
    tf = flops / (ms / 1e3) / 1e12
    return {"metric": f"dense decode points/sec ({cfg.dec.dtype}, N={cfg.dec.N}, C={cfg.dec.C})",
            "value": M / (ms / 1e3), "unit": UNIT, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "dtype": cfg.dec.dtype, "data": "synthetic",
            "config": {"workload": workload, "queries": M, "l2": "flushed between timed steps"},
            "tflops": tf, "frac_of_bf16_burst": tf / peaks["bf16"] if cfg.dec.dtype == "bf16" else None}


def _oracle_sample_points(cfg, n: int, seed: int = 0) -> np.ndarray:
    """A bounded, seeded sample of the workload's query points: coarse voxels and
    fine voxels near the spheres' surfaces (where the fine levels decode)."""
    from oracle import decoder as OD
    rng = np.random.default_rng(seed)
    if cfg.mode != "hier":   # dense workloads: voxels of the grid
        return OD.grid_points(cfg.grid_R, rng.integers(0, cfg.grid_R ** 3, n))
    half = n // 2
    coarse = OD.grid_points(cfg.r0, rng.integers(0, cfg.r0 ** 3, half))
    sp = W.make_spheres(cfg.n_spheres, 0, cfg.sphere_key, 1)[0]
    s_idx = rng.integers(0, cfg.n_spheres, n - half)
    d = rng.standard_normal((n - half, 3))
    d /= np.linalg.norm(d, axis=1, keepdims=True)
    fine = sp[s_idx, :3] + d * (sp[s_idx, 3:4] + rng.uniform(-0.02, 0.02, (n - half, 1)))
    return np.concatenate([coarse, np.clip(fine, -1, 1)])


def _oracle_rate(cfg, n_points: int):
    from threadpoolctl import threadpool_info

    from oracle import decoder as OD
    inp = W.make_decoder(cfg.dec, seed=0, key=cfg.seed_key, B=1)
    K, V = OD.precompute_kv(inp["z"][0], inp["weights"])
    pts = _oracle_sample_points(cfg, n_points)
    t0 = time.perf_counter()
    OD.decode_points(pts, K, V, inp["weights"], cfg.dec.query_ln)
    dt = time.perf_counter() - t0
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    return n_points / dt, dt, threads


def cpu_baseline(cfg, seconds: float = 15.0):
    """The oracle (float64 numpy) on a bounded sample of the workload's query
    points, dense attention over all tokens; ~``seconds`` of CPU work."""
    rate, dt, threads = _oracle_rate(cfg, 256)
    n = int(max(256, min(65536, rate * seconds)))
    rate, dt, threads = _oracle_rate(cfg, n)
    return {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{n} query points of the workload (half coarse voxels, half near-surface), "
                      f"float64 dense decode, {dt:.1f} s"}


def run_reference(args, world, rank):
    cfg = W.CONFIGS[args.config]
    if rank != 0:
        return None
    rate, dt, threads = _oracle_rate(cfg, 128)
    n = int(max(64, min(8192, rate * 4.0)))          # ~4 s per step
    for _ in range(args.warmup):
        _oracle_rate(cfg, max(32, n // 8))
    times = []
    for _ in range(args.steps):
        r, dt, threads = _oracle_rate(cfg, n)
        times.append(dt)
    ms = 1e3 * sum(times) / len(times)
    value = n / (ms / 1e3)
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"config {cfg.cid}: {cfg.name}", "sample_points_per_step": n},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": f"{n} query points per step, float64 dense decode"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="vdm", choices=["vdm", "reference"])
    ap.add_argument("--config", type=int, default=4, choices=[1, 2, 3, 4, 5],
                    help="3-5: hierarchical workloads (the step of the headline metric); 1-2: dense grids")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--dense-queries", type=int, default=0,
                    help="time dense decoding of this many points instead (config 2 decoder)")
    args = ap.parse_args()
    world, rank, local = _dist_init()
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        res = run_reference(args, world, rank)
    elif args.dense_queries > 0 or args.config in (1, 2):
        res = run_dense(args, world, rank, local)
    else:
        res = run_vdm(args, world, rank, local)
    if rank == 0 and res is not None:
        print(json.dumps(res))


if __name__ == "__main__":
    main()

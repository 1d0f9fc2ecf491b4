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


# dram__bytes_read.sum + dram__bytes_write.sum per decode launch of one shape of a
# workload (mean over the shape's decode launches), from ncu's one-pass DRAM counters on
# this script's own launches; None until captured for the current decoder kernel.
DECODE_DRAM_BYTES_PER_LAUNCH = {4: 39.48e6}


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


def level_kernel_bytes(cfg, stats) -> dict:
    """Algorithmic DRAM bytes of the level kernels for one shape, summed over the
    level steps R -> 2R (R the parent resolution, Mp its refined voxels):
    mark+dilate reads the level grid (4 R^3) and writes the mask (R^3 / 8);
    scan + parent list read the mask twice and write the word offsets
    (4 (R/4)^3), sub-volume ids and offsets (8 (R/4)^3 at most) and the parent
    list (4 Mp); the inherit fill reads the level grid and the mask and writes
    the fine voxels that are not decoded (4 (8 R^3 - 8 Mp))."""
    out = {"mark": 0.0, "scan_list": 0.0, "fill": 0.0}
    for s in stats:
        for l in range(cfg.n_levels - 1):
            R = cfg.r0 << l
            mp = s["active_parents"][l + 1]
            out["mark"] += 4 * R ** 3 + R ** 3 / 8
            out["scan_list"] += 2 * R ** 3 / 8 + 12 * (R // 4) ** 3 + 4 * mp
            out["fill"] += 4 * R ** 3 + R ** 3 / 8 + 4 * (8 * R ** 3 - 8 * mp)
    return out


def pick_tc_peak(peaks, clk):
    """Burst bf16 peak when the timed region ran at the maximum SM clock with no
    power cap (the kernel then runs as fast as in the burst measurement), else
    the sustained (power-capped) one."""
    sm, mx = clk.get("sm_mhz"), clk.get("sm_max_mhz") or peaks["sm_max_mhz"]
    at_max = sm is not None and sm >= 0.97 * mx and "sw_power_cap" not in clk.get("reasons", [])
    return (peaks["bf16"], "burst") if at_max else (peaks["bf16_sust"], "sustained")


def _decode_counts(cfg, stats):
    dense_q, sparse_q = 0, 0
    for s in stats:
        dense_q += s["decoded"][0]
        for l in range(1, cfg.n_levels):
            if cfg.adaptive:
                dense_q += s["probes"][l]
                sparse_q += s["decoded"][l] - s["probes"][l]
            else:
                dense_q += s["decoded"][l]
    return dense_q, sparse_q


def _timed(fn, steps, warmup, stream, flush):
    """Mean CUDA-event ms of ``fn`` over ``steps`` calls after ``warmup`` calls,
    L2 flushed before each timed call (outside the events)."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    evs = []
    for _ in range(steps):
        flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        evs.append((e0, e1))
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in evs) / steps


def accuracy_vs_dense(vdm, dec, K, V, cfg, spheres, params, ws, out_adaptive, p=None, vol_d=None):
    """Error of the lightning decoder against dense decoding, on shape 0.

    * same points: every voxel the adaptive hierarchical run decoded, decoded
      again with full attention over all tokens (vdm_decode_dense at the same
      xyz): max and mean |dec difference| and sign agreement of the field;
    * volumes: V-IoU and sign agreement of the adaptive hierarchical volume
      against the hierarchical volume without adaptive KV (same schedule) and
      against the dense decode of the whole final grid."""
    import torch
    Rf = cfg.r_final
    dbg = {"dec": [torch.full((1, (cfg.r0 << l) ** 3), float("nan"), device=K.device)
                   for l in range(cfg.n_levels)]}
    if p is None:
        p = vdm.hier_params(cfg.r0, cfg.n_levels, cfg.adaptive, cfg.tile, cfg.n_probe, cfg.top_k, 0)
    vol_a, _ = vdm.vdm_decode_hierarchical(dec, K[:1], V[:1], p, spheres[:1], cfg.dec_scale,
                                           workspace=ws, debug=dbg)
    res = {}
    worst, total, count, agree = 0.0, 0.0, 0, 0
    for l in range(cfg.n_levels):
        R = cfg.r0 << l
        d = dbg["dec"][l][0]
        idx = torch.nonzero(torch.isfinite(d)).flatten()
        i = idx // (R * R)
        j = (idx // R) % R
        k = idx % R
        xyz = (torch.stack([i, j, k], 1).float() * 2.0 + 1.0) / R - 1.0
        dense = vdm.vdm_decode_dense(dec, K[:1], V[:1], xyz=xyz[None].contiguous())[0]
        diff = (d[idx] - dense).abs()
        worst = max(worst, float(diff.max()))
        total += float(diff.double().sum())
        count += int(idx.numel())
        # field = sphere term + scale tanh(dec): the sphere term is shared, so the field's
        # sign is compared through the same vdm call with the analytic term on both sides
        fa = vdm.vdm_decode_dense(dec, K[:1], V[:1], xyz=xyz[None].contiguous(), spheres=spheres[:1],
                                  dec_scale=cfg.dec_scale)[0]
        fv = vol_a.reshape(-1)[idx] if l == cfg.n_levels - 1 else None
        if fv is not None:
            agree += int(((fv < 0) == (fa < 0)).sum())
        res[f"decoded_level_{l}"] = int(idx.numel())
    n_last = res[f"decoded_level_{cfg.n_levels - 1}"]
    res["same_points"] = {"points": count, "max_abs_dec_diff": worst, "mean_abs_dec_diff": total / count,
                          "final_level_sign_agreement": agree / n_last if n_last else 1.0}
    p_dense_kv = vdm.hier_params(cfg.r0, cfg.n_levels, False, cfg.tile, cfg.n_probe, cfg.top_k, 0)
    vol_h, _ = vdm.vdm_decode_hierarchical(dec, K[:1], V[:1], p_dense_kv, spheres[:1], cfg.dec_scale,
                                           workspace=ws)
    if vol_d is None:
        vol_d = vdm.vdm_decode_dense(dec, K[:1], V[:1], grid_R=Rf, spheres=spheres[:1],
                                     dec_scale=cfg.dec_scale).reshape(vol_h.shape)
    for name, other in (("vs_hierarchical_dense_kv", vol_h), ("vs_dense_grid", vol_d)):
        c = vdm.vdm_compare_volumes(vol_a, other)
        res[name] = {"v_iou": c["v_iou"], "sign_agreement": c["sign_agreement"],
                     "max_abs_field_diff": c["max_abs_diff"]}
    c = vdm.vdm_compare_volumes(vol_h, vol_d)
    res["hierarchical_dense_kv_vs_dense_grid"] = {"v_iou": c["v_iou"], "sign_agreement": c["sign_agreement"]}
    res["_vol_d"] = vol_d
    return res


def run_sweep(args, local):
    """Adaptive-KV settings against their cost: for each (probes per sub-volume,
    kept tokens k), the step time of one shape, the decoder's algorithmic FLOPs
    and the error against dense decoding (same points and V-IoU).  One JSON line
    per setting (sub-volumes are the 8^3 tiles the kernels are built for)."""
    import torch

    import neural_sdf_volume_b200 as vdm
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    cfg = W.CONFIGS[args.config]
    inp = W.make_decoder(cfg.dec, seed=0, key=cfg.seed_key, B=1)
    dec = vdm.Decoder.from_numpy(inp["weights"], cfg.dec.C, cfg.dec.H, cfg.dec.F, cfg.dec.query_ln,
                                 cfg.dec.dtype, device=dev)
    z = torch.from_numpy(inp["z"]).to(dev)
    spheres = torch.from_numpy(W.make_spheres(cfg.n_spheres, 0, cfg.sphere_key, 1)).to(dev)
    K, V = vdm.vdm_precompute_kv(dec, z)
    flush = torch.empty((L2_FLUSH_BYTES // 4,), device=dev, dtype=torch.float32)
    stream = torch.cuda.current_stream(dev)
    vol_d = None
    rows = []
    settings = [(0, 0)] + [(np_, k) for np_ in (32, 64, 128) for k in (256, 512, 1024, 2048)]
    for n_probe, k in settings:
        adaptive = n_probe > 0
        p = vdm.hier_params(cfg.r0, cfg.n_levels, adaptive, 8, n_probe or 64, k or cfg.top_k, 0)
        ws = torch.empty((vdm.vdm_hierarchical_workspace_size(dec, p, cfg.dec.N),), device=dev, dtype=torch.uint8)
        out = torch.empty((1,) + (cfg.r_final,) * 3, device=dev)
        holder = {}

        def one():
            holder["st"] = vdm.vdm_decode_hierarchical(dec, K, V, p, spheres, cfg.dec_scale, workspace=ws, out=out)[1]
        ms = _timed(one, args.steps, 3, stream, flush)
        st = holder["st"]
        c2 = cfg.with_(adaptive=adaptive, n_probe=n_probe or 64, top_k=k or cfg.top_k)
        dq, sq = _decode_counts(c2, st)
        kk = min(k or cfg.dec.N, cfg.dec.N)
        flops = dq * decode_flops_per_query(cfg.dec, cfg.dec.N) + sq * decode_flops_per_query(cfg.dec, kk)
        row = {"n_probe": n_probe, "top_k": k, "adaptive": adaptive, "ms_per_shape": ms,
               "decoder_tflop_per_shape": flops / 1e12, "decoded_points": dq + sq}
        if adaptive:
            acc = accuracy_vs_dense(vdm, dec, K, V, cfg, spheres, p, ws, out, p=p, vol_d=vol_d)
            vol_d = acc.pop("_vol_d")
            row["same_points"] = acc["same_points"]
            row["vs_dense_grid"] = acc["vs_dense_grid"]
        rows.append(row)
        print(json.dumps({"sweep": f"config {cfg.cid}", **row}), flush=True)
    return None


def level_kernels_large(vdm, cfg, dev, flush, steps, peaks, sizes=(384, 512)):
    """The level kernels (vdm_refine_level: mark + dilation, compaction, inherit
    fill) timed alone on level grids larger than the 126 MB L2 (L2 flushed
    before every call): a union of the workload's spheres sampled at R^3, the
    fine grid (2R)^3.  Algorithmic bytes as in ``level_kernel_bytes``."""
    import torch
    sp = torch.from_numpy(W.make_spheres(cfg.n_spheres, 0, cfg.sphere_key, 1)[0]).to(dev).double()
    out = {}
    for R in sizes:
        x = -1.0 + (2.0 * torch.arange(R, device=dev, dtype=torch.float64) + 1.0) / R
        f = torch.empty((R, R, R), device=dev, dtype=torch.float32)
        for i in range(R):   # one slab at a time keeps the temporaries small
            d = torch.sqrt((x[i] - sp[:, 0]).view(-1, 1, 1) ** 2 + (x.view(1, -1, 1) - sp[:, 1].view(-1, 1, 1)) ** 2 +
                           (x.view(1, 1, -1) - sp[:, 2].view(-1, 1, 1)) ** 2) - sp[:, 3].view(-1, 1, 1)
            f[i] = d.min(dim=0).values.float()
        fine = torch.empty((2 * R,) * 3, device=dev, dtype=torch.float32)
        parents = torch.empty((R ** 3,), device=dev, dtype=torch.int32)
        ws = torch.empty((vdm.vdm_refine_workspace_size(R),), device=dev, dtype=torch.uint8)
        for _ in range(3):
            _, counts = vdm.vdm_refine_level(f, fine, parents, ws)
        torch.cuda.synchronize(dev)
        vdm.vdm_profile_begin()
        for _ in range(steps):
            flush.zero_()
            vdm.vdm_refine_level(f, fine, parents, ws)
        torch.cuda.synchronize(dev)
        prof = vdm.vdm_profile_end()
        mp = int(counts[0].item())
        nbytes = {"mark_dilate": 4 * R ** 3 + R ** 3 / 8,
                  "compaction": 2 * R ** 3 / 8 + 12 * (R // 4) ** 3 + 4 * mp,
                  "fill": 4 * R ** 3 + 32 * R ** 3}
        ms = {"mark_dilate": prof["mark"]["ms"] / steps,
              "compaction": (prof["scan"]["ms"] + prof["list"]["ms"]) / steps,
              "fill": prof["fill"]["ms"] / steps}
        out[f"R{R}"] = {k: {"bytes": nbytes[k], "ms": ms[k], "GB/s": nbytes[k] / (ms[k] / 1e3) / 1e9,
                            "frac_of_measured_hbm": nbytes[k] / (ms[k] / 1e3) / 1e9 / peaks["hbm_gbs"],
                            "frac_of_8TBs_spec": nbytes[k] / (ms[k] / 1e3) / 1e9 / 8000.0}
                        for k in nbytes}
        out[f"R{R}"]["refined_voxels"] = mp
        del f, fine, parents, ws
        torch.cuda.empty_cache()
    return out


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

    def step(zin, prm=params):
        K, V = vdm.vdm_precompute_kv(dec, zin)
        _, st = vdm.vdm_decode_hierarchical(dec, K, V, prm, spheres, cfg.dec_scale, workspace=ws, out=out)
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
    dense_q, sparse_q = _decode_counts(cfg, stats)
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
    tc_peak, peak_kind = pick_tc_peak(peaks, clk)
    launches = sum(v["launches"] for v in prof.values())
    sel_flops = sum(s["selected_tiles"][l] for s in stats for l in range(cfg.n_levels)) * \
        cfg.n_probe * select_flops_per_probe(cfg.dec) / 2.0   # one scoring pass
    # memory-bound level kernels: algorithmic bytes / live CUDA-event time
    lbytes = level_kernel_bytes(cfg, stats)
    mem = {}
    for name, classes in (("mark_dilate_kernel", ("mark",)), ("scan_and_list_kernels", ("scan", "list")),
                          ("fill_kernel", ("fill",))):
        t = sum(prof[c]["ms"] for c in classes) / args.steps
        key = {"mark_dilate_kernel": "mark", "scan_and_list_kernels": "scan_list", "fill_kernel": "fill"}[name]
        gbs = lbytes[key] / (t / 1e3) / 1e9 if t > 0 else 0.0
        mem[name] = {"bytes_per_step": lbytes[key], "ms_per_step": t, "GB/s": gbs,
                     "frac_of_measured_hbm": gbs / peaks["hbm_gbs"], "frac_of_8TBs_spec": gbs / 8000.0}
    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": hier_config(cfg, world),
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
                     "peak_note": f"measured {peak_kind} bf16 matmul peak (MEASURED_PEAKS.json, "
                                  f"{peaks['src']}): burst when the timed region held the maximum SM "
                                  f"clock without a power cap, else sustained; algorithmic FLOPs: "
                                  f"{dec_flops / 1e12:.2f} TFLOP/step"},
        "select_roofline": {"kernel": "select_tc_kernel", "achieved":
                            (sel_flops / (prof["select"]["ms"] / args.steps / 1e3) / 1e12)
                            if prof["select"]["ms"] > 0 else 0.0, "unit": "TFLOP/s"},
        "memory_kernels": mem,
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
    if world == 1 and not args.no_extras:
        # companions of the headline on the same box, outside its timed region
        K, V = vdm.vdm_precompute_kv(dec, z)
        if cfg.adaptive:   # the same schedule with dense attention (config 3 for config 4)
            p3 = vdm.hier_params(cfg.r0, cfg.n_levels, False, cfg.tile, cfg.n_probe, cfg.top_k, 0)
            t3 = _timed(lambda: step(z, p3), args.steps, 3, stream, flush)
            res["without_adaptive_kv"] = {"ms_per_shape": t3 / B,
                                          "adaptive_kv_saves": 1.0 - (ms / B) / (t3 / B)}
        if cfg.cid == 4:   # the dense 128^3 grid of config 2 (same decoder)
            R2 = W.CONFIGS[2].grid_R
            g2 = torch.empty((1, R2 ** 3), device=dev)
            t2 = _timed(lambda: vdm.vdm_decode_dense(dec, K[:1], V[:1], grid_R=R2, out=g2), args.steps, 3,
                        stream, flush)
            tf2 = R2 ** 3 * decode_flops_per_query(cfg.dec, cfg.dec.N) / (t2 / 1e3) / 1e12
            res["dense_grid_128"] = {"workload": "config 2: dense 128^3 grid, same decoder",
                                     "ms": t2, "points_per_s": R2 ** 3 / (t2 / 1e3), "TFLOP/s": tf2,
                                     "frac_of_bf16_burst": tf2 / peaks["bf16"]}
        if cfg.cid == 4:   # the same pipeline with the quarter-width efficient decoder (config 6)
            c6 = W.CONFIGS[6]
            i6 = W.make_decoder(c6.dec, seed=0, key=c6.seed_key, B=1)
            d6 = vdm.Decoder.from_numpy(i6["weights"], c6.dec.C, c6.dec.H, c6.dec.F, c6.dec.query_ln,
                                        c6.dec.dtype, device=dev)
            sp6 = torch.from_numpy(W.make_spheres(c6.n_spheres, 0, c6.sphere_key, 1)).to(dev)
            p6 = vdm.hier_params(c6.r0, c6.n_levels, True, c6.tile, c6.n_probe, c6.top_k, 0)
            ws6 = torch.empty((vdm.vdm_hierarchical_workspace_size(d6, p6, c6.dec.N),), device=dev,
                              dtype=torch.uint8)
            z6 = torch.from_numpy(i6["z"]).to(dev)
            h6 = {}

            def step6():
                K6, V6 = vdm.vdm_precompute_kv(d6, z6)
                h6["st"] = vdm.vdm_decode_hierarchical(d6, K6, V6, p6, sp6, c6.dec_scale, workspace=ws6)[1]
            t6 = _timed(step6, args.steps, 3, stream, flush)
            dq6, sq6 = _decode_counts(c6, h6["st"])
            f6 = dq6 * decode_flops_per_query(c6.dec, c6.dec.N) + sq6 * decode_flops_per_query(c6.dec, c6.top_k)
            res["quarter_width_decoder"] = {
                "workload": f"config 6: {c6.name}, C={c6.dec.C}, H={c6.dec.H}, F={c6.dec.F}",
                "ms_per_shape": t6, "points_per_s": (dq6 + sq6) / (t6 / 1e3),
                "flops_per_query_vs_full_width": decode_flops_per_query(c6.dec, c6.dec.N) /
                decode_flops_per_query(cfg.dec, cfg.dec.N),
                "decoder_tflop_per_shape": f6 / 1e12}
        if cfg.cid == 4:   # vecset encoding of a surface point cloud with a full-width block
            M_pts, N_tok = 8192, cfg.dec.N
            cloud = W.make_point_cloud(sp_np[0], M_pts, N_tok, seed=0, key=7)
            proj = W.make_encoder_input_proj(cfg.dec.C, seed=0, key=7)
            blk_w = W.make_decoder(cfg.dec, seed=0, key=7)["weights"]
            blk = vdm.Decoder.from_numpy(blk_w, cfg.dec.C, cfg.dec.H, cfg.dec.F, cfg.dec.query_ln, cfg.dec.dtype,
                                         device=dev)
            W_in = torch.from_numpy(proj["W_in"]).to(dev).bfloat16()
            b_in = torch.from_numpy(proj["b_in"]).to(dev)
            pts = torch.from_numpy(cloud["points"][None]).to(dev)
            qs = torch.from_numpy(cloud["queries"][None]).to(dev)
            tenc = _timed(lambda: vdm.vdm_encode(blk, W_in, b_in, pts, qs), args.steps, 3, stream, flush)
            C_, H_, F_ = cfg.dec.C, cfg.dec.H, cfg.dec.F
            enc_flops = 2.0 * (M_pts * (51 * C_ + 2 * C_ * C_) +
                               N_tok * (51 * C_ + 2 * H_ * M_pts * 64 + C_ * C_ + 2 * C_ * F_))
            res["vecset_encoder"] = {"workload": f"{M_pts}-point surface cloud -> {N_tok} tokens, C={C_}",
                                     "ms_per_shape": tenc, "TFLOP/s": enc_flops / (tenc / 1e3) / 1e12}
        if cfg.cid == 4:   # the local (MSVS-style) decoder query at the MSVS page's 200K-query batch
            res["local_decoder_200k"] = local_decoder_200k(vdm, sp_np[0], dev, args.steps, stream, flush)
        if cfg.adaptive:
            res["accuracy_vs_dense"] = accuracy_vs_dense(vdm, dec, K, V, cfg, spheres, params, ws, out)
            res["accuracy_vs_dense"].pop("_vol_d", None)
        # surface extraction of the shape's final volume (the pipeline's next stage)
        step(z)
        sws = torch.empty((vdm.vdm_surface_workspace_size(Rf),), device=dev, dtype=torch.uint8)
        verts, tris = vdm.vdm_extract_surface(out[0], workspace=sws)
        tmc = _timed(lambda: vdm.vdm_extract_surface(out[0], workspace=sws), args.steps, 3, stream, flush)
        res["surface_extraction"] = {"ms_per_shape": tmc, "vertices": int(verts.shape[0]),
                                     "triangles": int(tris.shape[0]),
                                     "note": "sparse marching cubes of the final volume, L2 flushed"}
        res["memory_kernels_large"] = level_kernels_large(vdm, cfg, dev, flush, args.steps, peaks)
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


def hier_config(cfg, world):
    """The `config` object of a hierarchical workload's line (both arms print the same one)."""
    return {"workload": f"config {cfg.cid}: {cfg.name}, N={cfg.dec.N}, C={cfg.dec.C}, "
                        f"H={cfg.dec.H}, F={cfg.dec.F}, top_k={cfg.top_k}, {cfg.n_spheres} spheres",
            "shapes_per_gpu": cfg.B, "final_resolution": cfg.r_final, "l2": "flushed between timed steps",
            "parallelism": f"shape-sharded x{world}"}


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
            "config": hier_config(cfg, world) if cfg.mode == "hier" else {"workload": f"config {cfg.cid}: {cfg.name}"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": f"{n} query points per step, float64 dense decode"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def local_decoder_200k(vdm, spheres, dev, steps, stream, flush):
    """The local (MSVS-style) decoder query on the MSVS page's 200K-query batch."""
    import torch
    ldw = W.make_local_decoder(spheres, seed=0, key=9)
    ld = vdm.LocalDecoder.from_numpy(ldw, 8, device=dev)
    q200 = torch.from_numpy(W.make_points(200_000, seed=0, key=9)[0]).to(dev)
    tloc = _timed(lambda: vdm.vdm_decode_local(ld, q200), steps, 3, stream, flush)
    return {"workload": "200,000 uniform queries, 2 scales (4096 + 16384 surface anchors, C 64 + 32), K = 8",
            "ms": tloc, "points_per_s": 200_000 / (tloc / 1e3),
            "context": "MSVS page, 3.3: 213 ms (MSVS) vs 3068 ms (Lattice) for 200K queries, hardware not stated"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="vdm", choices=["vdm", "reference"])
    ap.add_argument("--config", type=int, default=4, choices=[1, 2, 3, 4, 5, 6],
                    help="3-6: hierarchical workloads (the step of the headline metric); 1-2: dense grids")
    ap.add_argument("--level-only", type=int, default=0, metavar="R",
                    help="only time the level kernels (vdm_refine_level) on an R^3 grid of the workload's spheres")
    ap.add_argument("--local-only", action="store_true",
                    help="only time the local (MSVS-style) decoder query on 200,000 points")
    ap.add_argument("--sweep", action="store_true",
                    help="adaptive-KV settings (probes, kept tokens) against time and error, one line each")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the companion measurements (dense-KV schedule, dense grid, accuracy)")
    ap.add_argument("--dense-queries", type=int, default=0,
                    help="time dense decoding of this many points instead (config 2 decoder)")
    args = ap.parse_args()
    world, rank, local = _dist_init()
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        res = run_reference(args, world, rank)
    elif args.sweep:
        res = run_sweep(args, local)
    elif args.level_only:
        import torch

        import neural_sdf_volume_b200 as vdm
        torch.cuda.set_device(local)
        dev = torch.device("cuda", local)
        flush = torch.empty((L2_FLUSH_BYTES // 4,), device=dev, dtype=torch.float32)
        res = {"level_kernels": level_kernels_large(vdm, W.CONFIGS[args.config], dev, flush, args.steps, _peaks(),
                                                    sizes=(args.level_only,))}
    elif args.local_only:
        import torch

        import neural_sdf_volume_b200 as vdm
        torch.cuda.set_device(local)
        dev = torch.device("cuda", local)
        flush = torch.empty((L2_FLUSH_BYTES // 4,), device=dev, dtype=torch.float32)
        sp = W.make_spheres(W.CONFIGS[args.config].n_spheres, seed=0, key=W.CONFIGS[args.config].sphere_key)[0]
        res = {"local_decoder_200k": local_decoder_200k(vdm, sp, dev, args.steps, torch.cuda.current_stream(dev),
                                                        flush)}
    elif args.dense_queries > 0 or args.config in (1, 2):
        res = run_dense(args, world, rank, local)
    else:
        res = run_vdm(args, world, rank, local)
    if rank == 0 and res is not None:
        print(json.dumps(res))


if __name__ == "__main__":
    main()

"""Throughput of the mesh rasterizer hot path on B200: pixel-face samples/s and Mpix/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config C]

One step is the whole hot path over one batch: stage one (face setup, coarse binning,
fine rasterization with the fused soft silhouette) followed by the fused silhouette +
rasterizer backward to the vertex positions, with dL/dalpha ~ N(0, 1).  The default
workload is the 64-image 512x512 heterogeneous batch (32 icospheres of levels 3-6 and
32 tori, K=4, sigma=1e-4).  Under torchrun every rank renders its own batch (seed offset
by rank: weak scaling; no collective on the data path) and the reported time is the
maximum over ranks; with --split the ranks share ONE batch, split by whole meshes balanced
by their pixel-face samples (strong scaling; still no collective on the data path).

A pixel-face sample is a (pixel, face) pair of the same image whose pixel centre lies in
the face's 2-D box grown by sqrt(blur_radius): the tests the method must make.  It is
counted exactly on the host from the inputs.
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

METRIC = "pixel-face samples/s and Mpix/s (fwd+bwd) at 1 B200; % of rasterizer roofline"
UNIT = "pixel-face samples/s"
C_TEST = 38                 # FP32 instructions per pixel-face test in this formulation (frozen)
FP32_LANES_PER_SM = 128
L2_FLUSH_BYTES = 256 << 20
KERNELS_PER_STAGE = {"silhouette_raster_bwd": 2,   # main kernel + (x, y) -> (x, y, z) copy
                     "bin_scan": 6}                # tile scans, tile totals, tile prefixes added; the bins'
                                                   # length histogram and longest-first order; and right
                                                   # after the stage the one-thread read-back of the list
                                                   # total, error word and empty-bin count (k_post_counts)


# ----------------------------------------------------------------------------- counting
def face_boxes(batch):
    """Per (image, face) pixel boxes grown by sqrt(blur) (exact, float64), degenerate faces dropped."""
    from differentiable_mesh_rasterization_b200.sharding import face_pixel_boxes
    w = batch.workload
    out = []
    for n in range(batch.N):
        f0, nf = int(batch.mesh_to_face_first_idx[n]), int(batch.num_faces_per_mesh[n])
        out.append(face_pixel_boxes(batch.verts, batch.faces[f0:f0 + nf], w.H, w.W, w.blur_radius))
    return out


def count_samples(batch, rows=None):
    """Pixel-face samples of the batch; with ``rows`` only those image rows count."""
    total = 0
    for jl, jh, il, ih in face_boxes(batch):
        width = jh - jl + 1
        if rows is None:
            total += int(np.sum(width * (ih - il + 1)))
        else:
            rr = np.asarray(rows)
            inr = (rr[None, :] >= il[:, None]) & (rr[None, :] <= ih[:, None])
            total += int(np.sum(width * inr.sum(1)))
    return total


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"mr_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50"]
            if self.uuid:
                cmd += ["-i", self.uuid]
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(cmd, stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None
        time.sleep(1.5)     # let nvidia-smi start sampling before the timed region
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        top = max(sm)
        loaded = [x for x in sm if x >= 0.5 * top] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- oracle leg
def oracle_sample(batch, ga, seconds=15.0):
    """A bounded sample of the workload for the CPU oracle: R evenly spaced rows of every
    image, R chosen from a one-row calibration run so the sample takes about ``seconds``."""
    w = batch.workload
    t1 = run_oracle(batch, ga, np.array([w.H // 2]))
    R = int(max(1, min(w.H, round(seconds / max(t1, 1e-3)))))
    rows = np.unique(np.linspace(0, w.H - 1, R).round().astype(np.int64))
    what = "fwd" if w.sigma is None else "fwd + silhouette fwd/bwd + raster bwd"
    return rows, f"{len(rows)} evenly spaced rows of each of the {batch.N} images ({what} on those pixels)"


def run_oracle(batch, ga, rows):
    """Oracle fwd (no exemption diagnostics) + silhouette fwd/bwd + raster bwd on the sampled rows."""
    import oracle
    w = batch.workload
    H, W, K = w.H, w.W, w.K
    pix = ((np.arange(batch.N)[:, None, None] * H + rows[None, :, None]) * W +
           np.arange(W)[None, None, :]).reshape(-1)
    t0 = time.perf_counter()
    p2f, zbuf, bary, dists, _ = oracle.rasterize_fwd(batch.verts, batch.faces, batch.mesh_to_face_first_idx,
                                                     batch.num_faces_per_mesh, H, W, np.float32(w.blur_radius), K,
                                                     w.perspective_correct, pixels=pix, exempt=False)
    if w.sigma is None:                   # forward-only (hard) workload
        return time.perf_counter() - t0
    sig = np.float32(w.sigma)
    oracle.silhouette_fwd(p2f, dists, sig)
    gd = oracle.silhouette_bwd(ga.reshape(-1)[pix], p2f, dists, sig)
    P2F = np.full((batch.N * H * W, K), -1, np.int64)
    GD = np.zeros((batch.N * H * W, K))
    P2F[pix] = p2f
    GD[pix] = gd
    oracle.rasterize_bwd(batch.verts, batch.faces, P2F.reshape(batch.N, H, W, K), w.perspective_correct,
                         grad_dists=GD.reshape(batch.N, H, W, K))
    return time.perf_counter() - t0


def reference_arm(args, rank):
    """`--impl reference`: the float64 CPU oracle on the host cores, bounded samples per step."""
    if rank != 0:
        return
    from differentiable_mesh_rasterization_b200 import synthetic as syn
    import oracle
    oracle.build()
    batch = syn.make_batch(args.config)
    ga = syn.grad_alpha(batch)
    budget = max(1.0, min(10.0, 150.0 / max(1, args.steps + args.warmup)))
    rows, desc = oracle_sample(batch, ga, seconds=budget)
    samples = count_samples(batch, rows)
    for _ in range(args.warmup):
        run_oracle(batch, ga, rows[:1])
    times = [run_oracle(batch, ga, rows) for _ in range(args.steps)]
    t = sum(times)
    w = batch.workload
    value = samples * args.steps / t
    cores = oracle.default_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(w, args),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_config(w, args):
    return {"workload": w.name, "description": w.description, "batch": w.N, "H": w.H, "W": w.W, "K": w.K,
            "blur_radius": w.blur_radius, "sigma": w.sigma, "perspective_correct": w.perspective_correct,
            "passes": "fwd+bwd" if w.backward else "fwd", "l2": "flushed (256 MiB write) between timed steps",
            "parallelism": (f"one batch split by whole meshes over {args.gpus} GPUs" if args.split else
                            f"independent batch per GPU x{args.gpus}")}


# ----------------------------------------------------------------------------- ncu traffic
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic_batch5_512px.json")
KERNEL_SOURCE = os.path.join(ROOT, "differentiable_mesh_rasterization_b200", "csrc", "mr_forward_kernels.cuh")


def measured_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu capture (a smaller case of
    this workload, scaled to it by the units the kernel processes), or None when there is
    none or the kernel source changed since it was taken."""
    import hashlib
    try:
        rec = json.load(open(TRAFFIC_FILE))
        sha = hashlib.sha256(open(KERNEL_SOURCE, "rb").read()).hexdigest()
    except (OSError, ValueError):
        return None
    if rec.get("source_sha256") != sha:
        return None
    k = rec.get("kernels", {}).get(kernel)
    return None if k is None else (k["dram_read_bytes"] + k["dram_write_bytes"]) * k.get("scale", 1.0)


# ----------------------------------------------------------------------------- ranks
def rank_seed(config: int, rank: int) -> int:
    """Weak scaling: every rank renders its own batch of the same workload."""
    return 1000 + config + 1000 * rank


def combine_ranks(dev_ms: float, samples: float, pixels: float, device=None):
    """(max over ranks of the device time, sum of samples, sum of pixels)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([dev_ms, samples, pixels], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        tmax = t[:1].clone()
        dist.all_reduce(tmax, op=dist.ReduceOp.MAX)
        tsum = t[1:].clone()
        dist.all_reduce(tsum, op=dist.ReduceOp.SUM)
        return float(tmax[0]), float(tsum[0]), float(tsum[1])
    return float(t[0]), float(t[1]), float(t[2])


# ----------------------------------------------------------------------------- shading row
def shading_step_timing(mr, torch, dev, stream, batch, verts, faces, first, num, flush, args, hbm_peak, hbm_note):
    """The two stage-two RGB steps on the same batch, each timed like the main step (L2
    flushed, CUDA events, stage timing):

    gouraud_rgb: stage one (no silhouette), Phong lighting at the vertices, interpolation
        of the lit colours, soft RGB blend; backward of all of it to the world positions,
        normals and albedo of the vertices and to the screen-space vertices.
    phong_rgb: stage one, per-fragment Phong shading (interpolation of position, normal and
        albedo fused with the lighting), soft RGB blend; backward likewise.
    """
    from differentiable_mesh_rasterization_b200 import synthetic as syn
    w = batch.workload
    V = batch.verts.shape[0]
    P = torch.from_numpy(batch.world).to(dev)
    N = torch.from_numpy(batch.normals).to(dev)
    alb = torch.from_numpy(syn.random_grads((V, 3), 11)).abs().clamp(max=1.0).to(dev)
    prm = mr.phong_params([1.0, 1.5, 3.0], [0.0, 0.0, 2.7], [0.1, 0.1, 0.15], [0.6, 0.55, 0.5], [0.3, 0.3, 0.3],
                          32.0)
    bg = [1.0, 1.0, 1.0]
    kw = dict(sigma=w.sigma, gamma=1e-2, znear=1.0, zfar=10.0)
    g = torch.from_numpy(syn.random_grads((batch.N, w.H, w.W, 4), 12)).to(dev)

    def frags():
        return mr.rasterize_fwd(verts, faces, first, num, w.H, w.W, w.blur_radius, w.K, w.perspective_correct)

    def gouraud():
        p2f, zbuf, bary, dists = frags()
        vcol = mr.phong_fwd(P, N, alb, prm)
        col = mr.interpolate_fwd(p2f, bary, faces, vcol)
        mr.blend_fwd(p2f, col, dists, zbuf, bg, **kw)
        gcol, gd, gz = mr.blend_bwd(p2f, col, dists, zbuf, bg, grad_rgba=g, **kw)
        gvcol, gbary = mr.interpolate_bwd(p2f, bary, faces, vcol, gcol)
        mr.phong_bwd(P, N, alb, prm, gvcol)
        mr.rasterize_bwd(verts, faces, p2f, w.perspective_correct, grad_zbuf=gz, grad_bary=gbary, grad_dists=gd)

    def phong():
        p2f, zbuf, bary, dists = frags()
        col = mr.phong_shade_fwd(p2f, bary, faces, P, N, alb, prm)
        mr.blend_fwd(p2f, col, dists, zbuf, bg, **kw)
        gcol, gd, gz = mr.blend_bwd(p2f, col, dists, zbuf, bg, grad_rgba=g, **kw)
        _, _, _, gbary = mr.phong_shade_bwd(p2f, bary, faces, P, N, alb, prm, gcol)
        mr.rasterize_bwd(verts, faces, p2f, w.perspective_correct, grad_zbuf=gz, grad_bary=gbary, grad_dists=gd)

    npix = batch.N * w.H * w.W
    K = w.K
    # algorithmic bytes of the stage-two kernels (slot = K per pixel; colours D = 3): each
    # per-slot input read once, each output written once; vertex gathers hit L2 and are
    # not counted
    algo = {"interpolate_fwd": npix * K * (8 + 12 + 12), "blend_fwd": npix * (K * (8 + 12 + 4 + 4) + 16),
            "blend_bwd": npix * (K * (8 + 12 + 4 + 4) + 16 + K * (12 + 4 + 4)),
            "interpolate_bwd": npix * K * (8 + 12 + 12 + 12),
            "phong_shade_fwd": npix * K * (8 + 12 + 12), "phong_shade_bwd": npix * K * (8 + 12 + 12 + 12)}

    def timed(step, note):
        for _ in range(3):
            step()
        torch.cuda.synchronize(dev)
        steps = max(3, args.steps // 5)
        ms, st = _timed_and_staged(mr, torch, dev, stream, flush, steps, step)
        stages = {}
        for name, (t, n) in st.items():
            if n:
                ent = {"ms_per_step": t / steps}
                if name in algo:
                    ent["hbm_frac"] = algo[name] / (t / steps / 1e3) / 1e9 / hbm_peak
                stages[name] = ent
        return {"ms_per_step": ms, "samples_per_s": float(count_samples(batch)) / (ms / 1e3),
                "mpix_per_s": npix / (ms / 1e3) / 1e6, "steps": steps, "stages": stages,
                "hbm_peak_note": hbm_note, "note": note + "; same workload, L2 flushed per step"}

    out = {}
    if "gouraud" in args.rows:
        out["gouraud_rgb"] = timed(gouraud, "Gouraud: stage one + Phong lighting at the vertices + colour "
                                            "interpolation + soft RGB blend (gamma 1e-2), fwd+bwd")
    if "phong" in args.rows:
        out["phong_rgb"] = timed(phong, "Phong: stage one + per-fragment interpolation and lighting (fused) + "
                                        "soft RGB blend (gamma 1e-2), fwd+bwd")
    return out


def _timed_and_staged(mr, torch, dev, stream, flush, steps, step):
    """``steps`` timed calls of ``step`` (L2 flushed before each, CUDA events on the launching
    stream), then the same number again with the library's stage events on: (ms per step,
    {stage: (ms, launches)} of the second pass)."""
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for k in range(steps):
        flush.zero_()
        starts[k].record(stream)
        step()
        ends[k].record(stream)
    torch.cuda.synchronize(dev)
    ms = sum(a.elapsed_time(b) for a, b in zip(starts, ends)) / steps
    mr.profile_read()
    mr.profile_enable(True)
    for k in range(steps):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    mr.profile_enable(False)
    return ms, mr.profile_read()


def _timed_steps(mr, torch, dev, stream, flush, steps, step):
    """Warm-up, then ``steps`` timed calls of ``step`` and a second pass for the library's
    stage times (see _timed_and_staged): (ms per step, stage dict)."""
    for _ in range(3):
        step()
    torch.cuda.synchronize(dev)
    ms, st = _timed_and_staged(mr, torch, dev, stream, flush, steps, step)
    return ms, {name: t / steps for name, (t, n) in st.items() if n}


def point_box_samples(pb, rows=None):
    """Pixel-point samples of a point batch: (pixel, point) pairs of the same image whose pixel
    centre lies in the point's box of half-width radius (exact host count; points behind the
    camera excluded); with ``rows`` only those image rows count."""
    w = pb.workload
    p = pb.points.astype(np.float64)
    r = float(np.float32(w.radius))
    ok = p[:, 2] >= 0
    jl = np.maximum(np.ceil((p[:, 0] - r + 1) * w.W / 2 - 0.5), 0)
    jh = np.minimum(np.floor((p[:, 0] + r + 1) * w.W / 2 - 0.5), w.W - 1)
    il = np.maximum(np.ceil((1 - p[:, 1] - r) * w.H / 2 - 0.5), 0)
    ih = np.minimum(np.floor((1 - p[:, 1] + r) * w.H / 2 - 0.5), w.H - 1)
    if rows is None:
        n = np.clip(jh - jl + 1, 0, None) * np.clip(ih - il + 1, 0, None)
    else:
        rr = np.asarray(rows)
        n = np.clip(jh - jl + 1, 0, None) * ((rr[None, :] >= il[:, None]) & (rr[None, :] <= ih[:, None])).sum(1)
    return int(np.sum(n[ok]))


def points_step_timing(mr, torch, dev, stream, flush, args, hbm_peak, hbm_note):
    """Point-cloud render step: 64 clouds (1.18 M points) -> K=8 nearest per pixel at 512x512
    -> alpha compositing of RGB features -> backward to the points and features."""
    from differentiable_mesh_rasterization_b200 import synthetic as syn
    pb = syn.make_point_batch(5, n_clouds=args.images)
    w = pb.workload
    P = torch.from_numpy(pb.points).to(dev)
    F = torch.from_numpy(pb.features).to(dev)
    r = float(np.float32(w.radius))
    g = torch.from_numpy(syn.random_grads((pb.N, w.H, w.W, w.C), 13)).to(dev)

    def step():
        idx, zbuf, dists = mr.rasterize_points_fwd(P, pb.cloud_first_idx, pb.num_points_per_cloud, w.H, w.W, r, w.K)
        mr.composite_points_fwd(idx, dists, F, r, "alpha")
        _, gd = mr.composite_points_bwd(idx, dists, F, r, g, "alpha")
        mr.rasterize_points_bwd(P, idx, grad_dists=gd)

    steps = max(3, args.steps // 5)
    ms, stages = _timed_steps(mr, torch, dev, stream, flush, steps, step)
    npix = pb.N * w.H * w.W
    slot = npix * w.K
    # algorithmic bytes: each per-slot array read or written once
    algo = {"points_fine": slot * (8 + 4 + 4), "composite_fwd": slot * (8 + 4) + npix * w.C * 4,
            "composite_bwd": slot * (8 + 4 + 4) + npix * w.C * 4, "points_bwd": slot * (8 + 4)}
    out = {s: {"ms_per_step": t} for s, t in stages.items()}
    for s, b in algo.items():
        if s in out:
            out[s]["hbm_frac"] = b / (out[s]["ms_per_step"] / 1e3) / 1e9 / hbm_peak
    samples = point_box_samples(pb)
    return {"workload": w.name, "ms_per_step": ms, "pixel_point_samples_per_s": samples / (ms / 1e3),
            "mpix_per_s": npix / (ms / 1e3) / 1e6, "points": int(pb.points.shape[0]), "steps": steps,
            "stages": out, "hbm_peak_note": hbm_note,
            "note": w.description + "; alpha compositing fwd+bwd; L2 flushed per step"}


def next_row_oracle_baselines(batch, rows_wanted):
    """The oracle, as it stands, on a bounded sample of each next row's workload (rank 0,
    host cores): the same fwd+bwd chain as the timed step on a few whole image rows (one
    query subset for KNN).  Returns {row: cpu_baseline dict}."""
    import oracle
    from differentiable_mesh_rasterization_b200 import synthetic as syn
    out = {}
    w = batch.workload
    H, W, K = w.H, w.W, w.K
    cores = oracle.default_threads()
    kw = dict(sigma=w.sigma, gamma=1e-2, znear=1.0, zfar=10.0)
    bg = np.ones(3)
    prm = oracle.phong_params([1.0, 1.5, 3.0], [0.0, 0.0, 2.7], [0.1, 0.1, 0.15], [0.6, 0.55, 0.5],
                              [0.3, 0.3, 0.3], 32.0)
    alb = np.abs(syn.random_grads((batch.verts.shape[0], 3), 11)).clip(max=1.0)
    rows = np.unique(np.linspace(0, H - 1, 4).round().astype(np.int64))
    pix = ((np.arange(batch.N)[:, None, None] * H + rows[None, :, None]) * W + np.arange(W)[None, None, :]).reshape(-1)
    full = batch.N * H * W

    def scatter(a, fill):
        z = np.full((full,) + a.shape[1:], fill, a.dtype)
        z[pix] = a
        return z.reshape((batch.N, H, W) + a.shape[1:])

    for shading in ("gouraud", "phong"):
        if shading not in rows_wanted:
            continue
        t0 = time.perf_counter()
        p2f, zb, ba, di, _ = oracle.rasterize_fwd(batch.verts, batch.faces, batch.mesh_to_face_first_idx,
                                                  batch.num_faces_per_mesh, H, W, np.float32(w.blur_radius), K,
                                                  False, pixels=pix, exempt=False)
        g = np.ones((len(pix), 4))
        if shading == "gouraud":
            vcol, _ = oracle.phong_fwd(batch.world, batch.normals, alb, prm)
            col = oracle.interpolate_fwd(p2f, ba, batch.faces, vcol)
        else:
            col, _ = oracle.phong_shade_fwd(p2f, ba, batch.faces, batch.world, batch.normals, alb, prm)
        oracle.blend_fwd(p2f, col, di, zb, bg, **kw)
        gc, gd, gz = oracle.blend_bwd(p2f, col, di, zb, bg, grad_rgba=g, **kw)
        if shading == "gouraud":
            gv, gb = oracle.interpolate_bwd(p2f, ba, batch.faces, vcol, gc)
            oracle.phong_bwd(batch.world, batch.normals, alb, prm, gv)
        else:
            gb = oracle.phong_shade_bwd(p2f, ba, batch.faces, batch.world, batch.normals, alb, prm, gc)[3]
        oracle.rasterize_bwd(batch.verts, batch.faces, scatter(p2f, -1), False, grad_zbuf=scatter(gz, 0.0),
                             grad_bary=scatter(gb, 0.0), grad_dists=scatter(gd, 0.0))
        dt = time.perf_counter() - t0
        out[shading + "_rgb"] = {"value": count_samples(batch, rows) / dt, "unit": "pixel-face samples/s",
                                 "cores": cores, "kind": "oracle", "seconds": dt,
                                 "sample": f"{len(rows)} evenly spaced rows of each of the {batch.N} images"}
    if "points" in rows_wanted:
        pb = syn.make_point_batch(5, n_clouds=batch.N)
        pw = pb.workload
        r = np.float32(pw.radius)
        prow = np.array([pw.H // 2])
        ppix = ((np.arange(pb.N)[:, None, None] * pw.H + prow[None, :, None]) * pw.W +
                np.arange(pw.W)[None, None, :]).reshape(-1)
        t0 = time.perf_counter()
        idx, _, pd, _ = oracle.rasterize_points(pb.points, pb.cloud_first_idx, pb.num_points_per_cloud, pw.H, pw.W,
                                                r, pw.K, pixels=ppix)
        oracle.composite_points(idx, pd, pb.features, r)
        _, gdd = oracle.composite_points_bwd(idx, pd, pb.features, r, np.ones((len(ppix), pw.C)))
        fi = np.full((pb.N * pw.H * pw.W, pw.K), -1, np.int64)
        fd = np.zeros((pb.N * pw.H * pw.W, pw.K))
        fi[ppix] = idx
        fd[ppix] = gdd
        oracle.rasterize_points_bwd(pb.points, fi.reshape(pb.N, pw.H, pw.W, pw.K),
                                    grad_dists=fd.reshape(pb.N, pw.H, pw.W, pw.K))
        dt = time.perf_counter() - t0
        out["points_rgb"] = {"value": point_box_samples(pb, prow) / dt, "unit": "pixel-point samples/s",
                             "cores": 1, "kind": "oracle", "seconds": dt,
                             "sample": f"the middle row of each of the {pb.N} images"}
    if "knn" in rows_wanted:
        kb = syn.make_knn_batch(5, n_clouds=batch.N)
        sel = np.concatenate([kb.first1[n] + np.arange(min(50, kb.num1[n])) for n in range(kb.N)])
        n1 = np.array([min(50, kb.num1[n]) for n in range(kb.N)], np.int64)
        f1 = np.cumsum(np.r_[0, n1[:-1]])
        t0 = time.perf_counter()
        ki, kd, _ = oracle.knn(kb.p1[sel], f1, n1, kb.p2, kb.first2, kb.num2, kb.workload.K)
        oracle.knn_bwd(kb.p1[sel], kb.p2, ki, np.ones(kd.shape))
        dt = time.perf_counter() - t0
        out["knn"] = {"value": float(np.sum(n1 * kb.num2)) / dt, "unit": "pairs/s", "cores": 1, "kind": "oracle",
                      "seconds": dt, "sample": f"the first 50 queries of each of the {kb.N} clouds"}
    if "subpixel" in rows_wanted:
        sb = syn.make_batch(4)
        sw = sb.workload
        srow = np.array([sw.H // 2])
        spix = (srow[:, None] * sw.W + np.arange(sw.W)[None, :]).reshape(-1)
        t0 = time.perf_counter()
        oracle.rasterize_fwd(sb.verts, sb.faces, sb.mesh_to_face_first_idx, sb.num_faces_per_mesh, sw.H, sw.W,
                             np.float32(sw.blur_radius), sw.K, sw.perspective_correct, pixels=spix, exempt=False)
        dt = time.perf_counter() - t0
        out["subpixel_1024px"] = {"value": count_samples(sb, srow) / dt, "unit": "pixel-face samples/s",
                                  "cores": cores, "kind": "oracle", "seconds": dt,
                                  "sample": "the middle row of the image (forward)"}
    return out


KNN_C_PAIR = 7       # FP32 instructions per (query, reference) pair for D=3: 3 FADD, 3 FFMA, 1 compare


def subpixel_step_timing(mr, torch, dev, stream, flush, args, peak_alu, hbm_peak, hbm_note):
    """The single-image sub-pixel workload (one 1024x1024 image of an icosphere of level 7:
    327,680 faces, most smaller than a pixel; K=8, blur 1e-5, perspective-correct; hard
    rasterization, so a step is the forward): step time, and the fine pass and the fine pass
    with its epilogue against the same rooflines as the main workload."""
    from differentiable_mesh_rasterization_b200 import synthetic as syn
    batch = syn.make_batch(4)
    w = batch.workload
    verts = torch.from_numpy(batch.verts).to(dev)
    faces = torch.from_numpy(batch.faces).to(dev)
    first, num = batch.mesh_to_face_first_idx, batch.num_faces_per_mesh

    def step():
        mr.rasterize_fwd(verts, faces, first, num, w.H, w.W, w.blur_radius, w.K, w.perspective_correct)

    steps = max(3, args.steps // 5)
    ms, stages = _timed_steps(mr, torch, dev, stream, flush, steps, step)
    samples = float(count_samples(batch))
    npix = batch.N * w.H * w.W
    fine_s, epi_s = stages["fine"] / 1e3, stages["epilogue"] / 1e3
    achieved = samples * C_TEST / fine_s / 1e12
    return {"workload": w.name, "ms_per_step": ms, "samples_per_s": samples / (ms / 1e3),
            "mpix_per_s": npix / (ms / 1e3) / 1e6, "samples_per_step": samples, "steps": steps,
            "stages": {s: {"ms_per_step": t} for s, t in stages.items()},
            "roofline": {"bound": "alu", "kernel": "k_fine", "achieved": achieved, "peak": peak_alu,
                         "unit": "T FP32-inst/s", "frac": achieved / peak_alu, "c_test": C_TEST,
                         "a3a4": a3a4_roofline(samples, fine_s, epi_s, npix * 28 * w.K, peak_alu, hbm_peak,
                                               hbm_note)},
            "note": w.description + "; forward (hard rasterization); L2 flushed per step"}


def knn_step_timing(mr, torch, dev, stream, flush, args, peak_alu):
    """Batched KNN step: 64 heterogeneous clouds (1.18 M queries against 1.18 M references,
    D=3, K=8) forward and backward."""
    from differentiable_mesh_rasterization_b200 import synthetic as syn
    kb = syn.make_knn_batch(5, n_clouds=args.images)
    K = kb.workload.K
    A = torch.from_numpy(kb.p1).to(dev)
    B = torch.from_numpy(kb.p2).to(dev)
    g = torch.from_numpy(syn.random_grads((kb.p1.shape[0], K), 14)).to(dev)

    def step():
        idx, _ = mr.knn_fwd(A, kb.first1, kb.num1, B, kb.first2, kb.num2, K)
        mr.knn_bwd(A, B, idx, g)

    steps = max(3, args.steps // 10)
    ms, stages = _timed_steps(mr, torch, dev, stream, flush, steps, step)
    pairs = int(np.sum(kb.num1.astype(np.int64) * kb.num2.astype(np.int64)))
    # the pairs the pruned search really evaluates (a counting build of the same search, run
    # once outside the timed region): the work of the roofline
    with torch.cuda.stream(stream):
        evaluated, _, _ = mr.knn_count_pairs(A, kb.first1, kb.num1, B, kb.first2, kb.num2, K)
    out = {s: {"ms_per_step": t} for s, t in stages.items()}
    knn_ms = out.get("knn", {}).get("ms_per_step")
    roof = None
    if knn_ms:
        achieved = evaluated * KNN_C_PAIR / (knn_ms / 1e3) / 1e12
        roof = {"bound": "alu", "kernel": "k_knn (pruned exact search, register top-K; the stage includes the "
                                          "ordering passes)",
                "achieved": achieved, "peak": peak_alu, "unit": "T FP32-inst/s", "frac": achieved / peak_alu,
                "c_pair": KNN_C_PAIR, "evaluated_pairs_per_step": evaluated,
                "work_note": "evaluated (query, reference) pairs counted by mr_knn_count_pairs; the exhaustive "
                             "count is reported as throughput only"}
    return {"workload": kb.workload.name, "ms_per_step": ms, "pairs_per_s": pairs / (ms / 1e3), "pairs": pairs,
            "evaluated_pairs": evaluated, "evaluated_fraction": evaluated / max(pairs, 1),
            "queries": int(kb.p1.shape[0]), "steps": steps, "stages": out, "roofline": roof,
            "note": kb.workload.description + "; fwd+bwd; L2 flushed per step"}


def a3a4_roofline(samples, fine_s, epi_s, epi_bytes, peak_alu, hbm_peak, hbm_note):
    """The fine pass as the target states it: the pixel-face tests (k_fine) and the per-slot
    outputs (k_epilogue) together.  Its roofline is the slower of the tests at the FP32 peak
    and the epilogue's bytes at the HBM peak; the two kernels run one after the other, so the
    sum of the two bounds (the serial floor) is given beside it."""
    t = fine_s + epi_s
    t_alu = samples * C_TEST / (peak_alu * 1e12)
    t_hbm = epi_bytes / (hbm_peak * 1e9)
    return {"kernels": "k_fine + k_epilogue", "bound": "alu" if t_alu >= t_hbm else "hbm",
            "ms_per_step": t * 1e3, "roof_ms": max(t_alu, t_hbm) * 1e3, "frac": max(t_alu, t_hbm) / t,
            "achieved": samples * C_TEST / t / 1e12, "peak": peak_alu, "unit": "T FP32-inst/s",
            "serial_floor_ms": (t_alu + t_hbm) * 1e3, "frac_of_serial_floor": (t_alu + t_hbm) / t,
            "hbm_peak_note": hbm_note}


# ----------------------------------------------------------------------------- our arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=5)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-shading", action="store_true", help="skip the Gouraud, Phong, point-cloud and KNN measurements")
    ap.add_argument("--rows", default="gouraud,phong,points,knn,subpixel",
                    help="comma-separated next-row measurements after the main step (gouraud, phong, points, knn, "
                         "subpixel: the one-image 1024x1024 workload of sub-pixel faces)")
    ap.add_argument("--split", action="store_true",
                    help="under torchrun, split ONE batch over the ranks by whole meshes, balanced by their "
                         "pixel-face samples (strong scaling), instead of one batch per rank (weak scaling)")
    ap.add_argument("--images", type=int, default=None,
                    help="render only the first N meshes of the batch, clouds of the point and KNN batches "
                         "(small profiling case)")
    args = ap.parse_args()

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        reference_arm(args, rank)
        return

    import torch
    import torch.distributed as dist

    import differentiable_mesh_rasterization_b200 as mr
    from differentiable_mesh_rasterization_b200 import synthetic as syn

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    batch = syn.make_batch(args.config, seed=rank_seed(args.config, 0 if args.split else rank),
                           n_meshes=args.images)
    w = batch.workload
    hard = w.sigma is None            # batch 4: hard rasterization, forward only
    ga_host = syn.grad_alpha(batch)
    h_v, h_f = batch.verts, batch.faces
    first, num = batch.mesh_to_face_first_idx, batch.num_faces_per_mesh
    n_img = batch.N
    if args.split:
        # this rank's meshes of the one batch: every rank computes the same split from the
        # same inputs, so nothing is exchanged
        from differentiable_mesh_rasterization_b200 import sharding
        costs = sharding.mesh_sample_counts(h_v, h_f, first, num, w.H, w.W, w.blur_radius)
        mine = sharding.partition_meshes(costs, world)[rank]
        sh = sharding.Shard(h_f, first, num, mine)
        h_v, h_f, first, num = np.ascontiguousarray(h_v[sh.vert_ids]), sh.faces, sh.first, sh.num
        ga_host = np.ascontiguousarray(ga_host[mine])
        n_img = len(mine)
        samples = int(costs[mine].sum())
    else:
        samples = count_samples(batch)
    verts = torch.from_numpy(h_v).to(dev)
    faces = torch.from_numpy(h_f).to(dev)
    ga = torch.from_numpy(ga_host).to(dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def run(v, f, g, before_backward=None):
        """One step on device inputs; returns the results a caller reads back: alpha and
        grad_verts, or the depth buffer of a forward-only (hard) workload."""
        if hard:
            return (mr.rasterize_fwd(v, f, first, num, w.H, w.W, w.blur_radius, w.K, w.perspective_correct)[1],)
        p2f, zbuf, bary, dists, alpha = mr.rasterize_fwd(v, f, first, num, w.H, w.W, w.blur_radius, w.K,
                                                         w.perspective_correct, sigma=w.sigma)
        if before_backward is not None:
            before_backward()
        return alpha, mr.silhouette_rasterize_bwd(v, f, p2f, dists, w.sigma, g)

    def step():
        return run(verts, faces, ga)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    mr.device_status(dev)

    props = torch.cuda.get_device_properties(dev)
    uuid = str(getattr(props, "uuid", "") or "")
    uuid = ("GPU-" + uuid) if uuid and not uuid.startswith("GPU-") else uuid
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    torch.cuda.reset_peak_memory_stats(dev)
    mr.scratch_peak(dev, reset=True)
    mr.profile_enable(False)
    with ClockSampler(uuid or None) as clocks:
        for k in range(args.steps):
            flush.zero_()
            starts[k].record(stream)
            step()
            ends[k].record(stream)
        torch.cuda.synchronize(dev)
    memory = {"scratch_peak_bytes": mr.scratch_peak(dev), "torch_peak_bytes": int(torch.cuda.max_memory_allocated(dev)),
              "l2_flush_bytes": L2_FLUSH_BYTES,
              "note": "over the timed steps: the library's scratch (high-water mark of the device's default "
                      "memory pool) and torch's allocations (inputs, the outputs of each step, the L2-flush buffer)"}
    # Per-stage times (and from them the kernels' rooflines and the launch count): a second
    # pass of the same steps with the library's stage events on.  They are kept out of the
    # timed steps above, where their 14 event records per step would add about 0.04 ms.
    mr.profile_read()
    mr.profile_enable(True)
    for k in range(args.steps):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    mr.profile_enable(False)
    if world > 1:
        dist.barrier()
    stages = mr.profile_read()
    dev_ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
    dev_ms, tot_samples, tot_pix = combine_ranks(dev_ms, float(samples), float(n_img * w.H * w.W), dev)
    sec = dev_ms / 1e3
    value = tot_samples * args.steps / sec
    mpix = tot_pix * args.steps / sec / 1e6

    # end to end through the public API: pinned host inputs in, alpha + grad_verts out
    h_verts = torch.from_numpy(h_v).pin_memory()
    h_faces = torch.from_numpy(h_f).pin_memory()
    h_ga = torch.from_numpy(np.zeros(0, np.float32) if hard else ga_host).pin_memory()   # nothing to upload when hard
    h_res = ([torch.empty((n_img, w.H, w.W, w.K), dtype=torch.float32).pin_memory()] if hard else
             [torch.empty((n_img, w.H, w.W), dtype=torch.float32).pin_memory(),
              torch.empty(h_v.shape, dtype=torch.float32).pin_memory()])

    def e2e_step():
        dv = h_verts.to(dev, non_blocking=True)
        df = h_faces.to(dev, non_blocking=True)
        dg = h_ga.to(dev, non_blocking=True)
        for h, d in zip(h_res, run(dv, df, dg)):
            h.copy_(d, non_blocking=True)

    def e2e_serial(n):
        """Copies and compute of every step one after the other on the compute stream."""
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            flush.zero_()
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1)

    def e2e_pipelined(n):
        """The same steps with the host-to-device copy of step k+1 on one copy stream and the
        device-to-host copy of step k on another (one copy engine each way), overlapping the
        compute of step k (triple-buffered device inputs; events order every copy against
        the compute that uses it: a step's forward waits for its verts and faces, its
        backward also for its dL/dalpha, which is copied last).  Timed from before the first
        input copy to after the last result copy."""
        cs = torch.cuda.Stream(device=dev)
        ds = torch.cuda.Stream(device=dev)
        NBUF = 3
        # device inputs allocated once (three sets, so a step's upload never waits for the
        # compute just before it), so no allocation sits between the streams
        bufs = [(torch.empty_like(h_verts, device=dev), torch.empty_like(h_faces, device=dev),
                 torch.empty_like(h_ga, device=dev)) for _ in range(NBUF)]
        torch.cuda.synchronize(dev)
        geo_done = [torch.cuda.Event() for _ in range(NBUF)]     # verts and faces of a step arrived
        h2d_done = [torch.cuda.Event() for _ in range(NBUF)]     # and its dL/dalpha
        freed = [None] * NBUF
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)

        def upload(k):
            i = k % NBUF
            with torch.cuda.stream(cs):
                if freed[i] is not None:
                    cs.wait_event(freed[i])
                for dst, src in zip(bufs[i][:2], (h_verts, h_faces)):
                    dst.copy_(src, non_blocking=True)
                geo_done[i].record(cs)
                bufs[i][2].copy_(h_ga, non_blocking=True)
                h2d_done[i].record(cs)

        e0.record(cs)
        upload(0)
        for k in range(n):
            i = k % NBUF
            if k + 1 < n:
                upload(k + 1)
            # the forward needs only the geometry; the backward waits for dL/dalpha as well;
            # alpha is final once the forward is done and goes out while the backward runs
            stream.wait_event(geo_done[i])
            dv, df, dg = bufs[i]
            flush.zero_()
            fwd_done = []

            def between():
                ev = torch.cuda.Event()
                ev.record(stream)
                fwd_done.append(ev)
                stream.wait_event(h2d_done[i])

            res = run(dv, df, dg, before_backward=between)
            done = torch.cuda.Event()
            done.record(stream)
            freed[i] = done
            with torch.cuda.stream(ds):
                for j, (h, d) in enumerate(zip(h_res, res)):
                    ds.wait_event(fwd_done[0] if j == 0 and fwd_done else done)
                    d.record_stream(ds)
                    h.copy_(d, non_blocking=True)
        e1.record(ds)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1)

    if args.e2e_steps > 0:
        e2e_step()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    serial_ms = e2e_serial(args.e2e_steps) if args.e2e_steps > 0 else 0.0
    if world > 1:
        dist.barrier()
    if args.e2e_steps > 0:
        e2e_pipelined(3)          # warm-up: the allocator caches the per-step output blocks
    e2e_ms = e2e_pipelined(args.e2e_steps) if args.e2e_steps > 0 else 0.0
    te = torch.tensor([e2e_ms, serial_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(te, op=dist.ReduceOp.MAX)
    e2e_value = tot_samples * args.e2e_steps / (float(te[0]) / 1e3) if args.e2e_steps > 0 else None
    h2d = h_verts.numel() * 4 + h_faces.numel() * 8 + h_ga.numel() * 4
    d2h = sum(h.numel() * 4 for h in h_res)

    # roofline of the dominant kernel (the fine pass: the pixel-face tests) and of the
    # epilogue (which writes the per-slot outputs); the stage times and launch counts are
    # totals over the steps of the second pass
    fine_ms, fine_n = stages["fine"]
    fine_s = fine_ms / 1e3 / args.steps
    epi_ms, epi_n = stages["epilogue"]
    epi_s = epi_ms / 1e3 / args.steps
    clk = clocks.summary()
    peaks = {}
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except (OSError, ValueError):
        pass
    sm_mhz_max = float(peaks.get("sm_max_mhz", 1965.0))
    peak_nominal = props.multi_processor_count * FP32_LANES_PER_SM * sm_mhz_max * 1e6 / 1e12   # T inst/s
    # the denominator is the FFMA issue rate measured on this device in this run (the peaks
    # file has no FP32 figure); unit counts x the maximum clock are reported beside it
    peak_alu = mr.measure_fp32_peak(dev) / 1e12
    hbm_peak = float(peaks.get("hbm_gbs", 6650.0))
    hbm_note = "of measured" if "hbm_gbs" in peaks else "of fallback"
    achieved_alu = samples * C_TEST / fine_s / 1e12
    npix = n_img * w.H * w.W
    fine_bytes = npix * 8 * w.K                      # the K winning face ids per pixel, written as pix_to_face
    epi_bytes = npix * (8 * w.K + 20 * w.K + (0 if hard else 4))   # ids in; zbuf, bary, dists(, alpha) out
    full_batch = args.images is None and args.config == 5
    roof = {"bound": "alu", "achieved": achieved_alu, "peak": peak_alu, "unit": "T FP32-inst/s",
            "frac": achieved_alu / peak_alu, "traffic": measured_traffic("k_fine") if full_batch else None,
            "kernel": "k_fine (stage-one fine pass: pixel-face tests and register top-K)",
            "ms_per_step": fine_s * 1e3, "launches_per_step": fine_n // args.steps,
            "samples_per_step": samples, "c_test": C_TEST,
            "peak_note": "of measured: FFMA-chain probe (mr_measure_fp32_peak) in this run",
            "peak_nominal": peak_nominal,
            "peak_nominal_note": f"{props.multi_processor_count} SMs x 128 FP32 lanes x {sm_mhz_max:.0f} MHz",
            "dense_tests_per_step": int(sum(int(n) for n in num)) * w.H * w.W,
            "hbm_bytes_per_step": fine_bytes,
            "a3a4": a3a4_roofline(samples, fine_s, epi_s, epi_bytes, peak_alu, hbm_peak, hbm_note),
            "epilogue": {"kernel": "k_epilogue (float64 outputs of the K winners + silhouette)",
                         "bound": "hbm", "ms_per_step": epi_s * 1e3, "bytes_per_step": epi_bytes,
                         "achieved": epi_bytes / epi_s / 1e9, "peak": hbm_peak, "unit": "GB/s",
                         "frac": epi_bytes / epi_s / 1e9 / hbm_peak, "peak_note": hbm_note,
                         "traffic": measured_traffic("k_epilogue") if full_batch else None}}

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dev_ms / args.steps, "higher_is_better": True,
            "scaling": "strong" if args.split else "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded icospheres and tori)",
            "config": workload_config(w, args), "mpix_per_s": mpix,
            "samples_per_step": tot_samples,
            "stages_ms_per_step": {k: v[0] / args.steps for k, v in stages.items() if v[1]},
            "stages_note": ("per-stage times from a second pass of the same steps with the library's CUDA events "
                            "around each stage on the launching stream; the timed steps run without them"),
            "roofline": roof,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": float(te[0]) / max(args.e2e_steps, 1), "pipelined": True,
                    "serial_ms_per_step": float(te[1]) / max(args.e2e_steps, 1),
                    "note": ("pinned host verts, faces in; the depth buffer out" if hard else
                             "pinned host verts, faces, dL/dalpha in; alpha and grad_verts out") + "; the copies of "
                            "step k+1 (in) and step k (out) overlap the compute of step k on two copy streams; a "
                            "step's forward waits for its geometry, its backward for its dL/dalpha"},
            "memory": memory,
            "gpu_launches": int(sum(v[1] * KERNELS_PER_STAGE.get(k, 1) for k, v in stages.items())),
            "clocks": clk}

    if args.no_shading or hard or args.split:   # the next rows run on the whole soft batch-5 workloads
        args.rows = ""
    rows = {}
    if "gouraud" in args.rows or "phong" in args.rows:
        rows.update(shading_step_timing(mr, torch, dev, stream, batch, verts, faces, first, num, flush, args, hbm_peak,
                                        hbm_note))
    if "points" in args.rows:
        rows["points_rgb"] = points_step_timing(mr, torch, dev, stream, flush, args, hbm_peak, hbm_note)
    if "knn" in args.rows:
        rows["knn"] = knn_step_timing(mr, torch, dev, stream, flush, args, peak_alu)
    if "subpixel" in args.rows:
        rows["subpixel_1024px"] = subpixel_step_timing(mr, torch, dev, stream, flush, args, peak_alu, hbm_peak,
                                                       hbm_note)
    if rows:
        line["next_rows"] = rows
        if rank == 0 and not args.no_cpu_baseline:
            for name, base in next_row_oracle_baselines(batch, args.rows).items():
                if name in rows:
                    rows[name]["cpu_baseline"] = base

    if rank == 0 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        rows, desc = oracle_sample(batch, ga_host)
        osamp = count_samples(batch, rows)
        tcpu = run_oracle(batch, ga_host, rows)
        line["cpu_baseline"] = {"value": osamp / tcpu, "unit": UNIT, "cores": oracle.default_threads(),
                                "kind": "oracle", "sample": desc, "seconds": tcpu}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()

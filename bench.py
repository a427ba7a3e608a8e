"""Benchmark of the forward NeRF render: one step = ray generation plus the full
coarse + fine render of one 800x800 frame (64 stratified + 128 inverse-CDF
samples per ray, 8x256 skip MLP with bf16 weights), all in libnerf's kernels.

Prints one JSON line (rank 0). `--impl reference` times the CPU oracle on the
same workload instead (a bounded sample of rays per step).

Extra lines (`--workload`):
  small                     200x200 coarse + fine with the 8x256 network in fp32
  small_tf32                the same with precision TF32 (layer GEMMs on the
                            tensor cores, three tf32 MMAs per product)
  tiny                      32x32, 64 stratified samples, a 4x64 fp32 network
  kilonerf, hashgrid        march renders of the two alternative scene functions
  hashgrid_bf16             the hash grid with its MLP in bf16 on the tensor cores
  sweep24                   24 cameras around the scene in one render call
  compact                   a 4x128 fp32 network on the CUDA-core MLP kernel
  compact_tf32              the same network with precision TF32
  train                     the training step (loss and both networks' gradients)
  hash_backward             the hash-grid encoding's backward (scatter-add)
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import nerf_inputs as S  # noqa: E402

WORKLOAD = "full"
METRIC = "rays/sec at 800x800 coarse+fine (64+128 samples/ray)"
UNIT = "rays/s"
SWEEP_FRAMES = 24                   # the novel-view video: 24 frames around the scene
TRAIN_BATCH = 4096                  # rays per training step (NeRF page, "7. Training loop")
MLP_FLOP_PER_ROW = 1186816          # algorithmic FLOPs of one 8x256 NeRF MLP evaluation


def mlp_flops_per_row(shape):
    return 2 * sum(n * k for name, n, k in shape.layer_shapes())


def mlp_label(wl):
    m = wl.mlp
    prec = "bf16" if wl.precision == S.PREC_BF16 else "fp32"
    skip = f" skip@{m.skip}" if m.skip >= 0 else ""
    return f"{m.D}x{m.W}{skip}, {prec} weights"


def rows_per_frame(wl):
    """MLP rows of one frame: the coarse samples, plus the fine pass's union."""
    return wl.n_rays * (wl.n_coarse + (wl.n_coarse + wl.n_fine if wl.n_fine else 0))


def config_json(wl, n_gpus, extra=None):
    c = {"workload": wl.name, "H": wl.H, "W": wl.W, "rays_per_frame": wl.n_rays,
         "n_coarse": wl.n_coarse, "n_fine": wl.n_fine, "mlp": mlp_label(wl),
         "mlp_rows_per_frame": rows_per_frame(wl),
         "parallelism": f"rays sharded, {n_gpus} independent frame(s) per step",
         "l2": "flushed between timed steps (256 MiB write)"}
    if extra:
        c.update(extra)
    return c


class ClockSampler:
    def __init__(self, index):
        self.proc = None
        self.index = index

    def __enter__(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            f = [x.strip() for x in ln.split(",")]
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def rank_camera(wl, rank):
    """Weak scaling: every rank renders one whole frame per step from its own
    camera (rank 0 renders the workload's camera). Rays never cross ranks."""
    if rank == 0:
        return wl.c2w()
    return S.look_at_c2w(*S.seeded_camera(wl.seed + 1000 * rank))


def max_over_ranks(value, dist, device):
    """Max over ranks of a per-rank device time (the only collective of the
    benchmark besides barriers; it is outside the timed region)."""
    if not dist:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rays_per_s(rays_per_rank_step, world, steps, max_ms):
    """Whole-job throughput: the rays all ranks rendered over the slowest rank's time."""
    return world * rays_per_rank_step * steps / (max_ms * 1e-3)


def cpu_baseline(wl, n_rays_sample, seed=123):
    """The oracle as it stands, on a bounded seeded sample of the frame's rays."""
    from oracle import nerf as onerf
    o, d = onerf.raygen(wl.H, wl.W, wl.focal, wl.c2w())
    ids = S.ray_subset(wl.n_rays, n_rays_sample, seed)
    cw, _ = S.nerf_weights(wl.mlp, wl.seed, 0, wl.sigma_scale, wl.precision)
    fw = S.nerf_weights(wl.mlp, wl.seed, 1, wl.sigma_scale, wl.precision)[0] if wl.n_fine else None
    t0 = time.perf_counter()
    onerf.render_nerf(wl, o[ids], d[ids], ids, cw, fw)
    dt = time.perf_counter() - t0
    return len(ids) / dt, dt, len(ids)


def n_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def run_reference(args, rank, world):
    wl = S.WORKLOADS[WORKLOAD]
    if rank != 0:
        return
    per_step = args.ref_rays
    for _ in range(args.warmup):
        cpu_baseline(wl, max(8, per_step // 8))
    times = []
    for k in range(args.steps):
        r, dt, n = cpu_baseline(wl, per_step, seed=1000 + k)
        times.append(dt)
    rays = per_step * args.steps
    value = rays / sum(times)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * sum(times) / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_json(wl, world, {"sample_rays_per_step": per_step}),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": n_cores(), "kind": "oracle",
                             "sample": f"{per_step} seeded rays of the frame per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def nerf_kernel_bytes(wl):
    """Algorithmic DRAM bytes per frame of the bandwidth-bound kernel classes of
    a NeRF render (each byte read or written once):
      composite  the last pass: raw (r, g, b, sigma) 16 B and, when the positions
                 are stored, t 4 B per sample; d 12 B in, rgb + depth + acc 20 B
                 out per ray
      resample   the coarse raw outputs 16 B per coarse sample and d 12 B in, the
                 sorted union 4 B per position out, per ray
      dir_bias   d 12 B in, W/2 fp32 out per ray, once per pass"""
    R, Nc, Nf = wl.n_rays, wl.n_coarse, wl.n_fine
    S_ = Nc + Nf
    passes = 2 if Nf else 1
    out = {"composite": R * ((S_ * 20 if Nf else Nc * 16) + 32),
           "dir_bias": passes * R * (12 + (wl.mlp.W // 2) * 4)}
    if Nf:
        out["resample"] = R * (Nc * 16 + 12 + S_ * 4)
    return out


def bandwidth_figures(kinds, bytes_per_frame, frames, hbm, peak_kind):
    """{class: achieved GB/s of its algorithmic bytes over its measured device
    time, and the fraction of the HBM copy peak}."""
    out = {}
    for k, nbytes in bytes_per_frame.items():
        ms, n = kinds.get(k, (0.0, 0))
        if n == 0 or ms <= 0:
            continue
        gbs = nbytes * frames / (ms * 1e-3) / 1e9
        out[k] = {"bytes_per_frame": nbytes, "ms_per_frame": ms / frames, "launches": n,
                  "achieved_gbs": gbs, "frac": gbs / hbm if hbm else None,
                  "peak_kind": f"HBM copy, {peak_kind}"}
    return out


NERF_METRICS = {
    "full": METRIC,
    "small": "rays/sec at 200x200 coarse+fine (64+128 samples/ray), 8x256 fp32 network",
    "small_tf32": "rays/sec at 200x200 coarse+fine (64+128 samples/ray), 8x256 network, fp32 "
                  "weights and I/O, layer products on the tensor cores (tf32 hi/lo, 3 passes)",
    "tiny": "rays/sec at 32x32, 64 stratified samples/ray, 4x64 fp32 network",
}


def run_nerf(args, rank, world, local_rank, key=WORKLOAD):
    """One step = ray generation + the whole render of one frame of workload `key`
    (full: the default bench line; small and tiny: the fp32 CUDA-core path)."""
    import torch
    import neural_radiance_field_b200 as nb
    from neural_radiance_field_b200 import build as nbuild
    nbuild.build()
    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    wl = S.WORKLOADS[key]
    if args.size:
        import dataclasses
        wl = dataclasses.replace(wl, H=args.size, W=args.size, focal=1.25 * args.size)
    bf16 = wl.precision == S.PREC_BF16
    c2w = rank_camera(wl, rank).ravel().tolist()
    cw, _ = S.nerf_weights(wl.mlp, wl.seed, 0, wl.sigma_scale, wl.precision)
    wdt = torch.bfloat16 if bf16 else torch.float32
    cwt = torch.from_numpy(cw).to(wdt).cuda()
    fwt = None
    if wl.n_fine:
        fw, _ = S.nerf_weights(wl.mlp, wl.seed, 1, wl.sigma_scale, wl.precision)
        fwt = torch.from_numpy(fw).to(wdt).cuda()
    R = wl.n_rays
    o = torch.empty(R, 3, device="cuda")
    d = torch.empty(R, 3, device="cuda")
    rgb = torch.empty(R, 3, device="cuda")
    dep = torch.empty(R, device="cuda")
    acc = torch.empty(R, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    m = wl.mlp
    rnd = nb.Renderer(D=m.D, W=m.W, skip=m.skip, sigma_act=wl.sigma_act, precision=wl.precision,
                      max_rays=R, max_samples=wl.n_coarse + wl.n_fine)
    p = rnd.params(coarse_w=cwt, fine_w=fwt, seed=wl.seed, perturb=1)
    stream = torch.cuda.current_stream()

    def step():
        nb.nerf_raygen(wl.H, wl.W, wl.focal, c2w, o, d)
        rnd.render(o, d, wl.near, wl.far, wl.n_coarse, wl.n_fine, p, rgb, dep, acc)

    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    torch.cuda.synchronize()
    rnd.sync_status()
    rnd.timing_enable(True)
    rnd.timing_read_kinds()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        for k in range(args.steps):
            flush.fill_(k & 0xFF)
            ev[k][0].record(stream)
            step()
            ev[k][1].record(stream)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    kinds = rnd.timing_read_kinds()
    mlp_ms, mlp_launches = kinds["network"]
    rnd.timing_enable(False)
    rnd.sync_status()
    tot_ms = max_over_ranks(sum(step_ms), dist, "cuda")

    # end to end through the host-buffer entry point (pinned host memory)
    oh, dh = o.cpu().pin_memory(), d.cpu().pin_memory()
    rgbh = torch.empty(R, 3).pin_memory()
    deph = torch.empty(R).pin_memory()
    acch = torch.empty(R).pin_memory()
    e2e_steps = max(1, min(args.steps, 5))
    rnd.render_host(oh, dh, wl.near, wl.far, wl.n_coarse, wl.n_fine, p, rgbh, deph, acch)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        rnd.render_host(oh, dh, wl.near, wl.far, wl.n_coarse, wl.n_fine, p, rgbh, deph, acch)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dist, "cuda")

    rows = rows_per_frame(wl)
    flop_row = mlp_flops_per_row(wl.mlp)
    passes = 2 if wl.n_fine else 1
    flops_launch_avg = flop_row * rows / passes            # coarse + fine launches per frame
    peaks, peak_kind = load_peaks()
    avg_launch_ms = mlp_ms / max(1, mlp_launches)
    achieved_tf = flops_launch_avg / (avg_launch_ms * 1e-3) / 1e12
    value = job_rays_per_s(R, world, args.steps, tot_ms)
    frame_tf = flop_row * rows * args.steps / (tot_ms * 1e-3) / 1e12
    clocks = clk.summary()
    if bf16:
        # The network kernel holds the top SM clock through a frame (see "clocks"),
        # so the burst cuBLAS figure is its ceiling; the power-capped sustained
        # figure is reported beside it.
        peak_tf = peaks.get("bf16_tflops")
        peak_sus = peaks.get("bf16_tflops_sustained", peak_tf)
        roofline = {"bound": "tensor", "kernel": "scene MLP (coarse and fine launches)",
                    "achieved": achieved_tf, "peak": peak_tf, "unit": "TFLOP/s",
                    "frac": achieved_tf / peak_tf, "peak_kind": f"bf16 burst, {peak_kind}",
                    "frac_of_sustained": achieved_tf / peak_sus,
                    "traffic": args.traffic_bytes or traffic_per_launch(flops_launch_avg),
                    "traffic_source": "--traffic-bytes" if args.traffic_bytes else TRAFFIC_SOURCE}
    elif wl.precision == S.PREC_TF32:
        # layer GEMMs on the tensor cores, three tf32 MMAs per product: the
        # roofline is the tf32 dense peak against the algorithmic FLOPs
        peak_tf = peaks.get("bf16_tflops") * TF32_PER_BF16
        roofline = {"bound": "tensor",
                    "kernel": "network pass: encoding, tensor-core row GEMMs (tf32 x3), heads",
                    "achieved": achieved_tf, "peak": peak_tf, "unit": "TFLOP/s",
                    "frac": achieved_tf / peak_tf,
                    "peak_kind": f"tf32 dense: bf16 {peak_kind} x 1.1 / 2.25 (nominal ratio)",
                    "frac_of_fp32_fma": achieved_tf / fp32_peak(clocks), "traffic": None}
    else:
        peak_tf = fp32_peak(clocks)
        roofline = {"bound": "alu", "kernel": f"mlp_fp32_kernel (CUDA-core MLP, W={wl.mlp.W})",
                    "achieved": achieved_tf, "peak": peak_tf, "unit": "TFLOP/s",
                    "frac": achieved_tf / peak_tf, "peak_kind": FP32_PEAK_NOTE, "traffic": None}
    roofline.update({"avg_launch_ms": avg_launch_ms, "flop_per_launch": flops_launch_avg,
                     # the same algorithmic FLOPs over the whole frame's time
                     # (sampling, compositing and resampling included)
                     "frame_achieved": frame_tf, "frame_frac": frame_tf / peak_tf})
    line = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            n_cpu = min(wl.n_rays, args.cpu_rays)
            rps, dt, n = cpu_baseline(wl, n_cpu)
            cpu = {"value": rps, "unit": UNIT, "cores": n_cores(), "kind": "oracle",
                   "sample": f"{n} seeded rays of the {wl.H}x{wl.W} frame, the whole oracle "
                             f"render of each ({dt:.1f} s)"}
        line = {
            "metric": NERF_METRICS[key], "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if bf16 else ("tf32x3" if wl.precision == S.PREC_TF32 else "f32"),
            "data": "synthetic (seeded camera, Xavier-init weights)",
            "config": config_json(wl, world),
            "sample_points_per_s": value * (wl.n_coarse + wl.n_fine),
            "mlp_rows_per_s": world * rows * args.steps / (tot_ms * 1e-3),
            "roofline": roofline,
            "bandwidth_kernels": bandwidth_figures(kinds, nerf_kernel_bytes(wl), args.steps,
                                                   peaks.get("hbm_gbs"), peak_kind),
            "cpu_baseline": cpu,
            "e2e": {"value": world * R / (e2e_ms * 1e-3), "unit": UNIT,
                    "h2d_bytes_per_step": R * 24, "d2h_bytes_per_step": R * 20},
            "gpu_launches": args.steps * nerf_launches_per_step(wl),
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    rnd.close()
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def nerf_launches_per_step(wl):
    """The library's kernels per NeRF step: ray generation; per pass the weight
    packing, the direction bias and the network; the resampling between passes;
    the final compositing. With precision TF32 the network of a pass is, per
    sub-batch of rays (the context's activation store holds 2^20 samples), the
    encoding, a weight split and a row GEMM per layer (D + 2 of them) and the
    heads."""
    passes = 2 if wl.n_fine else 1
    if wl.precision != S.PREC_TF32:
        return 1 + 3 * passes + (1 if wl.n_fine else 0) + 1
    fw_rows = min(wl.n_rays * (wl.n_coarse + wl.n_fine), 1 << 20)
    net = 0
    for s_pass in ([wl.n_coarse, wl.n_coarse + wl.n_fine] if wl.n_fine else [wl.n_coarse]):
        per = max(1, fw_rows // s_pass)
        n_sub = -(-wl.n_rays // per)
        # encoding and heads; a split and a row GEMM per tensor-core layer (the D
        # trunk layers and the feature layer; the direction layer when its W / 2
        # outputs are 128), one CUDA-core launch otherwise
        net += n_sub * (2 + 2 * (wl.mlp.D + 1) + (2 if wl.mlp.W == 256 else 1))
    return 1 + 2 * passes + net + (1 if wl.n_fine else 0) + 1


def fp32_peak(clocks):
    sm_mhz = clocks["sm_mhz"] or 1965.0
    return 148 * 128 * 2 * sm_mhz * 1e6 / 1e12


FP32_PEAK_NOTE = "fp32 FMA: 148 SMs x 128 lanes x 2 FLOP x SM clock"
# nominal dense tf32 / bf16 tensor rates of the part (1.1 and 2.25 PFLOP/s)
TF32_PER_BF16 = 1.1 / 2.25
# tensor-core FLOP the KiloNeRF kernel executes per point: three tf32 passes of
# the 64 (63 + padding) -> 32 and 32 -> 32 layers
KILO_MMA_FLOP_PER_POINT = 3 * 2 * (64 * 32 + 32 * 32)


def run_sweep(args, rank, world, local_rank):
    """One step = the rays of a 24-frame 360-degree orbit (one batched ray
    generation) rendered through ONE nerf_render call: 24 x 640,000 rays,
    coarse + fine, bf16 network (the novel-view video of the NeRF page,
    Section 3). An extra line; the headline is the single-frame workload."""
    import torch
    import neural_radiance_field_b200 as nb
    from neural_radiance_field_b200 import build as nbuild
    nbuild.build()
    torch.cuda.set_device(local_rank)
    wl = S.WORKLOADS[WORKLOAD]
    if args.size:
        import dataclasses
        wl = dataclasses.replace(wl, H=args.size, W=args.size, focal=1.25 * args.size)
    n_frames = SWEEP_FRAMES
    cams = [c.ravel().tolist() for c in S.orbit_c2ws(wl.seed, n_frames)]
    cw, _ = S.nerf_weights(wl.mlp, wl.seed, 0, wl.sigma_scale, wl.precision)
    fw, _ = S.nerf_weights(wl.mlp, wl.seed, 1, wl.sigma_scale, wl.precision)
    cwt = torch.from_numpy(cw).to(torch.bfloat16).cuda()
    fwt = torch.from_numpy(fw).to(torch.bfloat16).cuda()
    R = n_frames * wl.n_rays
    o = torch.empty(R, 3, device="cuda")
    d = torch.empty(R, 3, device="cuda")
    rgb = torch.empty(R, 3, device="cuda")
    dep = torch.empty(R, device="cuda")
    acc = torch.empty(R, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    rnd = nb.Renderer(precision=S.PREC_BF16, max_rays=R, max_samples=wl.n_coarse + wl.n_fine)
    p = rnd.params(coarse_w=cwt, fine_w=fwt, seed=wl.seed, perturb=1)
    stream = torch.cuda.current_stream()

    def step():
        nb.nerf_raygen_batch(wl.H, wl.W, wl.focal, cams, o, d)
        rnd.render(o, d, wl.near, wl.far, wl.n_coarse, wl.n_fine, p, rgb, dep, acc)

    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    torch.cuda.synchronize()
    rnd.sync_status()
    rnd.timing_enable(True)
    rnd.timing_read()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    with ClockSampler(local_rank) as clk:
        for k in range(args.steps):
            flush.fill_(k & 0xFF)
            ev[k][0].record(stream)
            step()
            ev[k][1].record(stream)
        torch.cuda.synchronize()
    tot_ms = sum(a.elapsed_time(b) for a, b in ev)
    mlp_ms, mlp_launches = rnd.timing_read()
    rnd.timing_enable(False)
    rnd.sync_status()
    rows = R * (2 * wl.n_coarse + wl.n_fine)
    flops_launch_avg = MLP_FLOP_PER_ROW * rows / 2
    peaks, peak_kind = load_peaks()
    peak_tf = peaks.get("bf16_tflops")
    peak_sus = peaks.get("bf16_tflops_sustained", peak_tf)
    avg_launch_ms = mlp_ms / max(1, mlp_launches)
    achieved_tf = flops_launch_avg / (avg_launch_ms * 1e-3) / 1e12
    line = {"metric": f"rays/sec, {n_frames}-frame 360-degree sweep at {wl.H}x{wl.W} coarse+fine "
                      f"({wl.n_coarse}+{wl.n_fine} samples/ray) in one render call",
            "value": R * args.steps / (tot_ms * 1e-3), "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded orbit cameras, Xavier-init weights)",
            "config": {"workload": f"sweep{n_frames}_{wl.name}", "frames": n_frames, "H": wl.H,
                       "W": wl.W, "rays_per_step": R, "n_coarse": wl.n_coarse, "n_fine": wl.n_fine,
                       "l2": "flushed between timed steps (256 MiB write)"},
            "frames_per_s": n_frames * args.steps / (tot_ms * 1e-3),
            "mlp_rows_per_s": rows * args.steps / (tot_ms * 1e-3),
            "roofline": {"bound": "tensor", "kernel": "scene MLP (coarse and fine launches)",
                         "achieved": achieved_tf, "peak": peak_tf, "unit": "TFLOP/s",
                         "frac": achieved_tf / peak_tf, "peak_kind": f"bf16 burst, {peak_kind}",
                         "frac_of_sustained": achieved_tf / peak_sus,
                         "traffic": traffic_per_launch(flops_launch_avg),
                         "traffic_source": TRAFFIC_SOURCE, "avg_launch_ms": avg_launch_ms,
                         "flop_per_launch": flops_launch_avg},
            "gpu_launches": args.steps * (2 + 7), "clocks": clk.summary()}
    print(json.dumps(line), flush=True)


def run_compact(args, rank, world, local_rank):
    """One step = ray generation + a coarse+fine render of the 800x800 frame with a
    compact fp32 network (D=4, W=128, skip after layer 1: a scene-specialised
    shape in the spirit of the NAS-NeRF page) on the CUDA-core MLP kernel, or with
    precision TF32 (`compact_tf32`: the layer GEMMs on the tensor cores). An
    extra line; the headline is the 8x256 bf16 workload."""
    import dataclasses
    import torch
    import neural_radiance_field_b200 as nb
    from neural_radiance_field_b200 import build as nbuild
    nbuild.build()
    torch.cuda.set_device(local_rank)
    shape = S.MLPShape(D=4, W=128, skip=1)
    tf32 = args.workload == "compact_tf32"
    prec = S.PREC_TF32 if tf32 else S.PREC_FP32
    wl = dataclasses.replace(S.WORKLOADS[WORKLOAD], mlp=shape, precision=prec)
    if args.size:
        wl = dataclasses.replace(wl, H=args.size, W=args.size, focal=1.25 * args.size)
    c2w = wl.c2w().ravel().tolist()
    cw, _ = S.nerf_weights(shape, wl.seed, 0, wl.sigma_scale, wl.precision)
    fw, _ = S.nerf_weights(shape, wl.seed, 1, wl.sigma_scale, wl.precision)
    cwt, fwt = torch.from_numpy(cw).cuda(), torch.from_numpy(fw).cuda()
    R = wl.n_rays
    o = torch.empty(R, 3, device="cuda")
    d = torch.empty(R, 3, device="cuda")
    rgb = torch.empty(R, 3, device="cuda")
    dep = torch.empty(R, device="cuda")
    acc = torch.empty(R, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    rnd = nb.Renderer(D=shape.D, W=shape.W, skip=shape.skip, precision=prec, max_rays=R,
                      max_samples=wl.n_coarse + wl.n_fine)
    p = rnd.params(coarse_w=cwt, fine_w=fwt, seed=wl.seed, perturb=1)
    stream = torch.cuda.current_stream()

    def step():
        nb.nerf_raygen(wl.H, wl.W, wl.focal, c2w, o, d)
        rnd.render(o, d, wl.near, wl.far, wl.n_coarse, wl.n_fine, p, rgb, dep, acc)

    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    torch.cuda.synchronize()
    rnd.sync_status()
    rnd.timing_enable(True)
    rnd.timing_read()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    with ClockSampler(local_rank) as clk:
        for k in range(args.steps):
            flush.fill_(k & 0xFF)
            ev[k][0].record(stream)
            step()
            ev[k][1].record(stream)
        torch.cuda.synchronize()
    tot_ms = sum(a.elapsed_time(b) for a, b in ev)
    mlp_ms, mlp_launches = rnd.timing_read()
    rnd.timing_enable(False)
    rnd.sync_status()
    flop_row = 2 * sum(n * k for _, n, k in shape.layer_shapes())
    rows = R * (2 * wl.n_coarse + wl.n_fine)
    clocks = clk.summary()
    sm_mhz = clocks["sm_mhz"] or 1965.0
    peak = 148 * 128 * 2 * sm_mhz * 1e6 / 1e12
    achieved = flop_row * rows * args.steps / (mlp_ms * 1e-3) / 1e12
    if tf32:
        peak_kind_tf = load_peaks()[1]
        roof = {"bound": "tensor", "kernel": "network pass: encoding, tensor-core row GEMMs (tf32 x3), heads",
                "peak": load_peaks()[0]["bf16_tflops"] * TF32_PER_BF16,
                "peak_kind": f"tf32 dense: bf16 {peak_kind_tf} x 1.1 / 2.25 (nominal ratio)",
                "frac_of_fp32_fma": achieved / peak}
    else:
        roof = {"bound": "alu", "kernel": "mlp_fp32_kernel (CUDA-core MLP, W=128)", "peak": peak,
                "peak_kind": FP32_PEAK_NOTE}
    line = {"metric": f"rays/sec at {wl.H}x{wl.W} coarse+fine ({wl.n_coarse}+{wl.n_fine} samples/ray), "
                      f"compact network D{shape.D} W{shape.W} skip@{shape.skip}, "
                      f"{'fp32 weights, layer GEMMs on the tensor cores (tf32 x3)' if tf32 else 'fp32'}",
            "value": R * args.steps / (tot_ms * 1e-3), "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "tf32x3" if tf32 else "f32",
            "data": "synthetic (seeded camera, Xavier-init weights)",
            "config": {"workload": f"compact_D{shape.D}W{shape.W}_{wl.H}x{wl.W}_{'tf32x3' if tf32 else 'fp32'}",
                       "mlp": f"{shape.D}x{shape.W} skip@{shape.skip}", "flop_per_row": flop_row,
                       "l2": "flushed between timed steps (256 MiB write)"},
            "mlp_rows_per_s": rows * args.steps / (tot_ms * 1e-3),
            "roofline": dict(roof, achieved=achieved, unit="TFLOP/s", frac=achieved / roof["peak"],
                             traffic=None, avg_launch_ms=mlp_ms / max(1, mlp_launches)),
            "gpu_launches": args.steps * nerf_launches_per_step(wl), "clocks": clocks}
    print(json.dumps(line), flush=True)


def run_train(args, rank, world, local_rank):
    """One step = the NeRF page's training step ("7. Training loop") on a batch of
    4096 rays drawn from the 800x800 frame: coarse + fine render of the 8x256
    network in fp32, loss = mse(coarse) + mse(fine) against seeded target colours,
    and the gradients of both networks (nerf_loss_grad). An extra line."""
    import dataclasses
    import torch
    import neural_radiance_field_b200 as nb
    from neural_radiance_field_b200 import build as nbuild
    nbuild.build()
    torch.cuda.set_device(local_rank)
    wl = dataclasses.replace(S.WORKLOADS[WORKLOAD], precision=S.PREC_FP32)
    B = args.batch or TRAIN_BATCH
    shape = wl.mlp
    o_all = torch.empty(wl.n_rays, 3, device="cuda")
    d_all = torch.empty(wl.n_rays, 3, device="cuda")
    nb.nerf_raygen(wl.H, wl.W, wl.focal, wl.c2w().ravel().tolist(), o_all, d_all)
    gen = torch.Generator(device="cpu").manual_seed(wl.seed)
    cw, _ = S.nerf_weights(shape, wl.seed, 0, wl.sigma_scale, S.PREC_FP32)
    fw, _ = S.nerf_weights(shape, wl.seed, 1, wl.sigma_scale, S.PREC_FP32)
    cwt, fwt = torch.from_numpy(cw).cuda(), torch.from_numpy(fw).cuda()
    n_batches = max(args.steps, args.warmup)
    idx = [torch.randperm(wl.n_rays, generator=gen)[:B].cuda() for _ in range(n_batches)]
    batches = [(o_all[i].contiguous(), d_all[i].contiguous()) for i in idx]
    targets = [torch.rand(B, 3, generator=gen).cuda() for _ in range(n_batches)]
    rnd = nb.Renderer(precision=S.PREC_FP32, max_rays=B, max_samples=wl.n_coarse + wl.n_fine)
    p = rnd.params(coarse_w=cwt, fine_w=fwt, seed=wl.seed, perturb=1)
    loss = torch.zeros(1, device="cuda")
    gc = torch.empty(cw.size, device="cuda")
    gf = torch.empty(fw.size, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step(k):
        o, d = batches[k]
        rnd.loss_grad(o, d, wl.near, wl.far, wl.n_coarse, wl.n_fine, p, targets[k], loss, gc, gf)

    for k in range(args.warmup):
        flush.fill_(1)
        step(k)
    torch.cuda.synchronize()
    rnd.sync_status()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    with ClockSampler(local_rank) as clk:
        for k in range(args.steps):
            flush.fill_(k & 0xFF)
            ev[k][0].record(stream)
            step(k)
            ev[k][1].record(stream)
        torch.cuda.synchronize()
    rnd.sync_status()
    tot_ms = sum(a.elapsed_time(b) for a, b in ev)
    # algorithmic FLOPs per MLP row: the forward, then the backward's weight
    # gradients (one multiply-add per weight and row) and input gradients (all
    # layers but the first, and not for the direction layer's gamma(d) columns)
    fwd = MLP_FLOP_PER_ROW
    bwd = fwd + (fwd - 2 * shape.W * shape.pos_ch - 2 * (shape.W // 2) * shape.dir_ch)
    rows = B * (2 * wl.n_coarse + wl.n_fine)
    clocks = clk.summary()
    sm_mhz = clocks["sm_mhz"] or 1965.0
    fma_peak = 148 * 128 * 2 * sm_mhz * 1e6 / 1e12
    peaks, pk = load_peaks()
    peak = peaks["bf16_tflops"] * TF32_PER_BF16
    tf32_kind = f"tf32 dense: bf16 {pk} x 1.1 / 2.25 (nominal ratio); algorithmic FLOPs, 3 MMA passes each"
    achieved = (fwd + bwd) * rows * args.steps / (tot_ms * 1e-3) / 1e12
    line = {"metric": f"training rays/sec, batches of {B} rays, {wl.H}x{wl.W} frame, coarse+fine "
                      f"({wl.n_coarse}+{wl.n_fine}), 8x256 fp32, loss + gradients of both networks",
            "value": B * args.steps / (tot_ms * 1e-3), "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded ray batches and target colours, Xavier-init weights)",
            "config": {"workload": f"train_batch{B}_nerf_800x800_fp32", "batch_rays": B,
                       "mlp": "8x256 skip@4, fp32", "flop_per_row_fwd_bwd": fwd + bwd,
                       "l2": "flushed between timed steps (256 MiB write)"},
            "loss_last_step": float(loss.item()),
            "roofline": {"bound": "tensor", "kernel": "whole training step (layer GEMMs on the "
                                                      "tensor cores in tf32 x3, heads on the CUDA cores)",
                         "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "peak_kind": tf32_kind,
                         "frac_of_fp32_fma": achieved / fma_peak, "traffic": None},
            # per pass: weight packing, direction bias, the forward (encoding, D + 2
            # layer GEMMs, heads), compositing backward, the backward (2 D + 9); a
            # weight split before each of the 2 D + 3 tensor-core row GEMMs, and a
            # second column tile for the skip layer's weight gradient; then the
            # resampling and the loss sum
            "gpu_launches": args.steps * (2 * ((shape.D + 6) + 1 + (2 * shape.D + 9) + (2 * shape.D + 3)
                                               + (1 if 0 <= shape.skip < shape.D - 1 else 0)) + 2),
            "clocks": clocks}
    print(json.dumps(line), flush=True)


def run_hash_backward(args, rank, world, local_rank):
    """One step = the hash-grid encoding's backward (the scatter-add that trains
    the grid) for 2^22 points drawn from the occupied voxels' region of the
    hash-grid workload, in both summation modes. An extra line."""
    import torch
    import neural_radiance_field_b200 as nb
    from neural_radiance_field_b200 import build as nbuild
    nbuild.build()
    torch.cuda.set_device(local_rank)
    n = 1 << 22
    gen = torch.Generator(device="cpu").manual_seed(5)
    x = (torch.rand(n, 3, generator=gen) * 3.0 - 1.5).cuda()
    g = torch.randn(n, 32, generator=gen).cuda()
    grad = torch.zeros(S.HASH_ENTRIES, 2, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    res = {}
    with ClockSampler(local_rank) as clk:
        for det in (False, True):
            for _ in range(args.warmup):
                nb.nerf_hash_encode_backward(x, g, grad, deterministic=det)
            torch.cuda.synchronize()
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
            for k in range(args.steps):
                flush.fill_(k & 0xFF)
                ev[k][0].record(stream)
                nb.nerf_hash_encode_backward(x, g, grad, deterministic=det)
                ev[k][1].record(stream)
            torch.cuda.synchronize()
            res[det] = sum(a.elapsed_time(b) for a, b in ev) / args.steps
    peaks, peak_kind = load_peaks()
    # algorithmic bytes per point: x (12 B) and d_feat (128 B) read, 16 levels x
    # 8 corners x 2 features of 4-byte read-modify-write in the gradient table
    bytes_pt = 12 + 128 + 16 * 8 * 2 * 4 * 2
    hbm = peaks.get("hbm_gbs")
    achieved = n * bytes_pt / (res[False] * 1e-3) / 1e9
    line = {"metric": "points/sec, hash-grid encoding backward (scatter-add into the tables), fp32 atomics",
            "value": n / (res[False] * 1e-3), "unit": "points/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": res[False], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": "hash_backward_4M_points", "points": n,
                       "table_rows": S.HASH_ENTRIES,
                       "l2": "flushed between timed steps (256 MiB write)"},
            "deterministic_mode": {"ms_per_step": res[True], "points_per_s": n / (res[True] * 1e-3),
                                   "summation": "int64 fixed point, bit-identical across runs"},
            "roofline": {"bound": "hbm", "kernel": "hash_bw_kernel (fp32 atomics)",
                         "achieved": achieved, "peak": hbm, "unit": "GB/s",
                         "frac": achieved / hbm if hbm else None,
                         "peak_kind": f"HBM copy, {peak_kind}; the 48.8 MB gradient table is "
                                      "L2-resident, so its atomics resolve in L2",
                         "traffic": None, "bytes_per_point": bytes_pt},
            "gpu_launches": args.steps, "clocks": clk.summary()}
    print(json.dumps(line), flush=True)


def march_kernel_bytes(wl, R, live, tc):
    """Algorithmic bytes per frame of the march kernel classes (each byte read or
    written once; `live` occupied candidates):
      march_mask       o, d 24 B in, 16 mask words and a count 68 B out, per ray
                       (plus one occupancy bit per candidate from the 256 KB grid)
      march_compact    count in and offset out 8 B, masks 64 B in, per ray; one
                       4 B live entry out per live candidate
      router           (KiloNeRF) live entry in, cell id out, cell id in, order
                       out: 16 B per live candidate
      network          (hash grid) 16 levels x 8 corners x 4 B of table gathers,
                       the live entry 4 B and the (r, g, b, sigma) 16 B out, per
                       live candidate
      march_composite  offset 4 B, d 12 B in, rgb + depth + acc 20 B out per ray;
                       live entry and (r, g, b, sigma) 20 B per live candidate"""
    out = {"march_mask": R * 92, "march_compact": R * 72 + live * 4,
           "march_composite": R * 36 + live * 20}
    if wl.model == "kilonerf":
        out["router"] = live * 16
    else:
        out["network"] = live * (512 + 20)
    return out


def march_cpu_baseline(wl, scene, n_rays_sample, seed=123):
    """The march oracle as it stands on a bounded seeded sample of the frame's rays."""
    from oracle import march as omarch
    from oracle import nerf as onerf
    o, d = onerf.raygen(wl.H, wl.W, wl.focal, wl.c2w())
    ids = S.ray_subset(wl.n_rays, n_rays_sample, seed)
    _, dense = S.occupancy_grid(wl.seed)
    if wl.model == "kilonerf":
        cells = scene
        ev = lambda idx, x, du: omarch.kilonerf_eval(cells, omarch.cell_id(x), x, du)
    else:
        from oracle import hashgrid as ohash
        grid = ohash.HashGrid3D()
        table, mlp = scene
        ev = lambda idx, x, du: omarch.hash_eval(grid, table, mlp, x, du)
    t0 = time.perf_counter()
    omarch.render_march(wl, o[ids], d[ids], dense, ev)
    dt = time.perf_counter() - t0
    return len(ids) / dt, dt, len(ids)


def run_march(args, rank, world, local_rank):
    """One step = ray generation + a full-frame march render of the KiloNeRF or
    hash-grid workload (occupancy skipping, scene function, compositing)."""
    import torch
    import neural_radiance_field_b200 as nb
    from neural_radiance_field_b200 import build as nbuild
    nbuild.build()
    torch.cuda.set_device(local_rank)
    tc = args.workload == "hashgrid_bf16"
    wl = S.WORKLOADS["hashgrid" if tc else args.workload]
    if args.size:
        import dataclasses
        wl = dataclasses.replace(wl, H=args.size, W=args.size, focal=1.25 * args.size)
    c2w = wl.c2w().ravel().tolist()
    R = wl.n_rays
    packed, _ = S.occupancy_grid(wl.seed)
    occ = torch.from_numpy(packed.view(np.int32)).cuda()
    if wl.model == "kilonerf":
        model = nb.NERF_MODEL_KILONERF
        cells_np = S.kilonerf_weights(wl.seed)
        cell_w = torch.from_numpy(cells_np).cuda()
        kw = dict(occupancy=occ, cell_w=cell_w)
        scene = cells_np
        flop_per_point, kname = 2 * 3249, "kilo_eval_kernel (per-cell tiny MLPs, 32-wide layers on the tensor cores in tf32 x3)"
    else:
        model = nb.NERF_MODEL_HASHGRID
        table_np = S.hashgrid_table(S.HashGridShape(), S.HASH_ENTRIES, wl.seed, 1e-4)
        table = torch.from_numpy(table_np.view(np.int16)).cuda()
        mlp_np = S.hash_mlp_weights(wl.seed)
        mlp = torch.from_numpy(mlp_np).cuda()
        kw = dict(occupancy=occ, hash_table=table, hash_mlp=mlp)
        scene = (table_np, mlp_np)
        flop_per_point = 2 * 15616
        kname = ("hash_tc_kernel (fp32 encoding, MLP on the tensor cores in bf16)" if tc
                 else "hash_eval_kernel (encoding + MLPs)")
    o = torch.empty(R, 3, device="cuda")
    d = torch.empty(R, 3, device="cuda")
    rgb = torch.empty(R, 3, device="cuda")
    dep = torch.empty(R, device="cuda")
    acc = torch.empty(R, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    rnd = nb.Renderer(model=model, max_rays=R, max_samples=wl.n_coarse,
                      precision=S.PREC_BF16 if tc else S.PREC_FP32)
    p = rnd.params(march_step=wl.march_step, ert_T=wl.ert_T, **kw)
    nb.nerf_raygen(wl.H, wl.W, wl.focal, c2w, o, d)
    cnt = torch.empty(R, dtype=torch.int32, device="cuda")
    nb.nerf_test_march(o, d, wl.near, wl.march_step, wl.n_coarse, occ, cnt)
    live = int(cnt.sum().item())          # occupied candidates (before termination)
    stream = torch.cuda.current_stream()

    def step():
        nb.nerf_raygen(wl.H, wl.W, wl.focal, c2w, o, d)
        rnd.render(o, d, wl.near, wl.far, wl.n_coarse, 0, p, rgb, dep, acc)

    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    torch.cuda.synchronize()
    rnd.sync_status()
    rnd.timing_enable(True)
    rnd.timing_read_kinds()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    with ClockSampler(local_rank) as clk:
        for k in range(args.steps):
            flush.fill_(k & 0xFF)
            ev[k][0].record(stream)
            step()
            ev[k][1].record(stream)
        torch.cuda.synchronize()
    tot_ms = sum(a.elapsed_time(b) for a, b in ev)
    kinds = rnd.timing_read_kinds()
    k_ms = kinds["network"][0]
    rnd.timing_enable(False)
    rnd.sync_status()

    # end to end through the host-buffer entry point (pinned host memory)
    oh, dh = o.cpu().pin_memory(), d.cpu().pin_memory()
    rgbh = torch.empty(R, 3).pin_memory()
    deph = torch.empty(R).pin_memory()
    acch = torch.empty(R).pin_memory()
    e2e_steps = max(1, min(args.steps, 5))
    rnd.render_host(oh, dh, wl.near, wl.far, wl.n_coarse, 0, p, rgbh, deph, acch)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        rnd.render_host(oh, dh, wl.near, wl.far, wl.n_coarse, 0, p, rgbh, deph, acch)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps

    clocks = clk.summary()
    peaks, pk = load_peaks()
    hbm = peaks.get("hbm_gbs")
    per_frame_k_ms = k_ms / args.steps
    achieved = live * flop_per_point / (per_frame_k_ms * 1e-3) / 1e12
    nbytes = march_kernel_bytes(wl, R, live, tc)
    if wl.model == "kilonerf":
        # the two 32-wide layers (6,080 of the 6,498 FLOP per point) run on the
        # tensor cores in tf32, three passes per product (hi*hi + hi*lo + lo*hi) for
        # fp32-level accuracy: the roofline is the tf32 dense peak (the bf16 figure
        # times the nominal tf32 / bf16 ratio 1.1 / 2.25); the fp32 FMA rate that
        # the CUDA-core version was measured against is reported beside it
        bf = peaks.get("bf16_tflops")
        peak = bf * TF32_PER_BF16 if bf else None
        roofline = {"bound": "tensor", "kernel": kname, "achieved": achieved, "peak": peak,
                    "unit": "TFLOP/s", "frac": achieved / peak if peak else None,
                    "peak_kind": f"tf32 dense: bf16 {pk} x 1.1 / 2.25 (nominal ratio)",
                    "traffic": None, "kernel_ms_per_frame": per_frame_k_ms,
                    "flop_per_point": flop_per_point,
                    "mma_flop_per_point": KILO_MMA_FLOP_PER_POINT,
                    "frac_of_fp32_fma": achieved / fp32_peak(clocks)}
    else:
        # the hash-grid scene kernel is bound by its 128 table gathers per point
        # (the 23.3 MiB table stays in L2): its roofline is the algorithmic gather
        # bytes against the HBM copy rate; the MLP's FLOP rate is reported beside it
        gbs = nbytes["network"] / (per_frame_k_ms * 1e-3) / 1e9
        roofline = {"bound": "hbm", "kernel": kname, "achieved": gbs, "peak": hbm,
                    "unit": "GB/s", "frac": gbs / hbm if hbm else None,
                    "peak_kind": f"HBM copy, {pk} (the table is L2-resident)",
                    "traffic": None, "kernel_ms_per_frame": per_frame_k_ms,
                    "bytes_per_point": 512 + 20, "mlp_tflops": achieved}
        if tc:
            bf = peaks.get("bf16_tflops")
            roofline["mlp_frac_of_bf16_burst"] = achieved / bf if bf else None
        else:
            roofline["mlp_frac_of_fp32_fma"] = achieved / fp32_peak(clocks)
    cpu = None
    if not args.no_cpu_baseline:
        rps, dt, n = march_cpu_baseline(wl, scene, args.march_cpu_rays)
        cpu = {"value": rps, "unit": UNIT, "cores": n_cores(), "kind": "oracle",
               "sample": f"{n} seeded rays of the {wl.H}x{wl.W} frame, the whole oracle march "
                         f"of each ({dt:.1f} s)"}
    line = {"metric": f"rays/sec, {wl.name} march render" + (", MLP in bf16 on the tensor cores" if tc else ""),
            "value": R * args.steps / (tot_ms * 1e-3),
            "unit": UNIT, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": tot_ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if tc else "f32", "data": "synthetic",
            "config": {"workload": wl.name + ("_bf16" if tc else ""), "H": wl.H, "W": wl.W,
                       "candidates": wl.n_coarse, "march_step": wl.march_step, "ert_T": wl.ert_T,
                       "occupied_candidates_per_frame": live,
                       "l2": "flushed between timed steps (256 MiB write)"},
            "sample_points_per_s": live * args.steps / (tot_ms * 1e-3),
            "roofline": roofline,
            "bandwidth_kernels": bandwidth_figures(kinds, nbytes, args.steps, hbm, pk),
            "cpu_baseline": cpu,
            "e2e": {"value": R / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": R * 24,
                    "d2h_bytes_per_step": R * 20},
            "gpu_launches": args.steps * march_launches_per_step(wl.model, R), "clocks": clocks}
    print(json.dumps(line), flush=True)
    rnd.close()


def march_launches_per_step(model, R):
    """The library's kernels per march step: ray generation, then per chunk of up
    to 2^19 rays the occupancy mask, a 3-kernel scan, the emit, the scene
    function (hash grid: 1 kernel; KiloNeRF: histogram, 3-kernel scan, scatter,
    work items, evaluation) and compositing."""
    chunks = -(-R // min(R, 1 << 19))
    per_chunk = 6 + (1 if model == "hashgrid" else 7)
    return 1 + chunks * per_chunk


# DRAM bytes (read + write) per MLP row of the scene-MLP kernel, from an ncu
# capture (dram__bytes_read.sum + dram__bytes_write.sum) of the fine launch of a
# 256x256 frame: 237.21 MB (87.59 MB read, 149.63 MB written) for 12,582,912
# rows. The traffic is the raw output and the sample positions, so it grows in
# proportion to the rows; it is scaled to the launch size here. Re-measure
# whenever the kernel changes.
TRAFFIC_B_PER_ROW = 237.21e6 / 12582912
TRAFFIC_SOURCE = ("ncu dram__bytes_read.sum + dram__bytes_write.sum of the fine launch at "
                  "256x256, scaled by rows to the average launch")


def traffic_per_launch(flops_launch_avg):
    return TRAFFIC_B_PER_ROW * flops_launch_avg / MLP_FLOP_PER_ROW


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-rays", type=int, default=1024)
    ap.add_argument("--ref-rays", type=int, default=128)
    ap.add_argument("--march-cpu-rays", type=int, default=256,
                    help="rays of the oracle's march sample (march workloads)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default=WORKLOAD,
                    choices=[WORKLOAD, "small", "small_tf32", "compact_tf32", "tiny", "kilonerf", "hashgrid", "hashgrid_bf16",
                             "sweep24", "compact", "train", "hash_backward"],
                    help="the benchmark workload (default) or a march workload (extra lines)")
    ap.add_argument("--traffic-bytes", type=float, default=0.0,
                    help="DRAM bytes per network launch from an ncu capture of this kernel")
    ap.add_argument("--batch", type=int, default=0,
                    help="rays per training step (train workload; default 4096)")
    ap.add_argument("--size", type=int, default=0,
                    help="render an SIZE x SIZE frame instead (profiling runs only)")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
    elif args.workload == "sweep24":
        run_sweep(args, rank, world, local_rank)
    elif args.workload in ("compact", "compact_tf32"):
        run_compact(args, rank, world, local_rank)
    elif args.workload == "train":
        run_train(args, rank, world, local_rank)
    elif args.workload == "hash_backward":
        run_hash_backward(args, rank, world, local_rank)
    elif args.workload in ("kilonerf", "hashgrid", "hashgrid_bf16"):
        run_march(args, rank, world, local_rank)
    else:
        run_nerf(args, rank, world, local_rank, args.workload)


if __name__ == "__main__":
    main()

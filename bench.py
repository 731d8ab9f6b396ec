"""Benchmark of the Wan-style video-VAE decoder hot path on B200.

One step = one decode of the Wan2.2-shaped decoder trunk (latents
[1, 48, 4, 44, 78] -> video [1, 3, 4, 704, 1248], bf16, random weights with the
trunk's shapes): conv_in, 8 residual blocks (norm + SiLU fused into the conv
epilogues, causal 3x3x3 convs, residual adds), 3 nearest-2x upsample convs and
norm_out + SiLU + head conv + pixel shuffle.  It runs every step of the hot
path; value = decoded frames/s over all ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--split replicas|rows]

Under torchrun each rank decodes its own replica by default (weak scaling);
with `--split rows` the ranks decode one video together, split by latent
rows with the halo rows exchanged over NCCL (strong scaling).  The timed
region is bracketed by a barrier and a device synchronise and its duration
is the max over ranks.  Besides the trunk the line carries the components:
norm-SiLU, the causal conv (direct and Winograd), the residual block, and
the 193-frame video of 49 latent frames streamed with temporal upsampling.
`--impl reference` times the CPU oracle instead (rank 0 only), one bounded
layer-shape sample per step.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "res-block conv TFLOP/s (% bf16 peak); norm-SiLU GB/s (% HBM); frames/s"
UNIT = "frames/s"
T, H, W = 4, 44, 78
WIDTHS = (512, 512, 256, 128)
WORKLOAD = ("Wan2.2-shaped decoder trunk: latents [1,48,4,44,78] -> video [1,3,4,704,1248]; "
            "conv_in, 4 stages of 2 res blocks (widths 512/512/256/128), 3 nearest-2x upsample "
            "convs, norm_out+SiLU+head conv + 2x2 pixel shuffle")
ZC = 48
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 512 << 20


# ------------------------------------------------------------------ workload
def trunk_layers(T=T, H=H, W=W, widths=WIDTHS, zc=ZC, executed=False, phase_form=False):
    """The trunk's launches in order with their dense FLOPs (all taps counted;
    the upsample convs at output resolution with 9 taps).  phase_form=True
    counts the upsample convs as four 2x2 phase convs on the low-res input
    (16/36 of dense: the least exact work).  executed=True gives the MMA FLOPs
    the kernels actually issue: the phase form, conv_in on 48 channels padded
    to 64, the head on 12 output channels padded to 16."""
    layers = [("layout", 0.0)]
    v = T * H * W
    layers.append(("conv_in", 2.0 * v * widths[0] * (64 if executed else zc) * 27))
    for s, c in enumerate(widths):
        vs = v * 4 ** s
        for b in range(2):
            layers.append((f"s{s}.b{b}.conv1", 2.0 * vs * c * c * 27))
            layers.append((f"s{s}.b{b}.conv2", 2.0 * vs * c * c * 27))
        if s + 1 < len(widths):
            up = 2.0 * vs * widths[s + 1] * c * 16 if (executed or phase_form) \
                else 2.0 * (4 * vs) * widths[s + 1] * c * 9
            layers.append((f"s{s}.up", up))
    v3 = v * 4 ** (len(widths) - 1)
    layers.append(("head", 2.0 * v3 * (16 if executed else 12) * widths[-1] * 27))
    return layers


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------ DRAM traffic
KERNEL_SOURCES = ("conv_tc.cu", "head_tc.cu", "api.cu", "internal.h", "ptx.cuh")
TRAFFIC_PROFILE = os.path.join(ROOT, "profiles", "conv_tc_trunk_dram_4x44x78.md")


def conv_source_hash() -> str:
    """Hash of the sources that decide what the conv kernel reads and writes."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "video_diffusion_vae_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def conv_traffic():
    """Mean DRAM bytes (read + write) per conv launch of a trunk step, from the
    committed ncu capture, or None when that capture was taken on other kernel
    sources (its `source_hash` line differs) or is missing."""
    try:
        kv = {}
        with open(TRAFFIC_PROFILE) as fh:
            for line in fh:
                if line.startswith("- ") and ":" in line:
                    k, v = line[2:].split(":", 1)
                    kv[k.strip()] = v.strip().strip("`")
        if kv.get("source_hash") != conv_source_hash():
            return None
        return float(kv["dram_bytes_per_conv_launch"])
    except (OSError, KeyError, ValueError):
        return None


# ------------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled while a region runs.

    NVML is polled every `period_s` from a thread (read-only queries), so even a
    timed region of a fraction of a second gets a dozen samples; without NVML,
    nvidia-smi at 100 ms.  Either way the first sample is taken before the
    region starts."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
               ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4),
               ("hw_power_brake_slowdown", 0x80))
    SMI_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                  "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index, period_s=0.02, nvml=None):
        self.idx = device_index
        self.period = period_s
        self.nvml = nvml          # a module with pynvml's interface (tests pass a fake)
        self.rows = []            # (sm_mhz, max_mhz, reason names)
        self.source = None
        self._stop = None
        self._thread = None
        self._proc = None
        self._path = None

    # ---- NVML
    def _handle(self, nv):
        try:
            import torch
            pr = torch.cuda.get_device_properties(self.idx)
            bus = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
            return nv.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.idx)

    def _sample(self, nv, h):
        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
        mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
        self.rows.append((float(sm), float(mx), [n for n, b in self.REASONS if bits & b]))

    def _poll(self, nv, h):
        while not self._stop.wait(self.period):
            try:
                self._sample(nv, h)
            except Exception:
                return

    def _start_nvml(self):
        import threading
        nv = self.nvml
        if nv is None:
            import pynvml as nv
        nv.nvmlInit()
        h = self._handle(nv)
        self._sample(nv, h)  # first sample before the region
        self._stop = threading.Event()
        self._thread = threading.Thread(target=self._poll, args=(nv, h), daemon=True)
        self._thread.start()
        self.source = "nvml"

    # ---- nvidia-smi
    def _start_smi(self):
        fd, self._path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self._proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.SMI_FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self._path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            os.unlink(self._path)
            raise
        t0 = time.time()
        while time.time() - t0 < 3.0 and os.path.getsize(self._path) == 0:
            time.sleep(0.02)
        self.source = "nvidia-smi"

    def _read_smi(self):
        names = [n for n, _ in self.REASONS[:4]]
        try:
            for line in open(self._path):
                f = [x.strip() for x in line.split(",")]
                if len(f) < 9 or not f[1].replace(".", "").isdigit():
                    continue
                mx = float(f[2]) if f[2].replace(".", "").isdigit() else float("nan")
                self.rows.append((float(f[1]), mx,
                                  [names[i] for i in range(4) if f[5 + i].lower() == "active"]))
        finally:
            os.unlink(self._path)

    def __enter__(self):
        try:
            self._start_nvml()
        except Exception:
            try:
                self._start_smi()
            except Exception:
                self._proc = None
        return self

    def __exit__(self, *a):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)
        if self._proc is not None:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except Exception:
                self._proc.kill()
            self._read_smi()

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [r[0] for r in self.rows]
        mx = [r[1] for r in self.rows if r[1] == r[1]]
        reasons = sorted({n for r in self.rows for n in r[2]})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.rows), "source": self.source}


# ----------------------------------------------------------- CPU baseline
ORACLE_CROP = 16


def oracle_layer_sample(crop=ORACLE_CROP, seed=1):
    """The CPU oracle timed on every distinct layer shape of the full workload.

    Each layer runs on a spatial crop of its own input: crop x crop voxels
    (crop/2 x crop/2 low-res voxels for the upsample convs, whose output is then
    crop x crop), all 4 frames, the layer's full channel width.  Its time is
    scaled by the layer's full output voxels over the crop's (the oracle's
    loops visit every tap of every output voxel, padded or not, so its work per
    output voxel does not depend on the position) and the layers are summed:
    conv_in, one residual block per stage (x 2 blocks), the three upsample
    convs and the head (norm_out + SiLU + conv + pixel shuffle).
    Returns (frames/s, seconds of oracle work, threads, per-layer detail)."""
    import torch
    from oracle import oracle as O
    from video_diffusion_vae_b200 import synth
    _, params = synth.trunk_input(T=T, H=2, W=2, seed=seed)
    g = torch.Generator().manual_seed(seed)
    c, ch = crop, crop // 2
    full_t, spent, detail = 0.0, 0.0, {}

    def run(name, fn, full_vox, crop_vox, count=1):
        nonlocal full_t, spent
        t0 = time.perf_counter()
        fn()
        dt = time.perf_counter() - t0
        spent += dt
        full_t += dt * full_vox / crop_vox * count
        detail[name] = round(dt * full_vox / crop_vox * count, 2)

    z = synth.normal(g, (ZC, T, c, c))
    run("conv_in", lambda: O.causal_conv3d(z, *params["conv_in"]), H * W, c * c)
    Hs, Ws = H, W
    for s, st in enumerate(params["stages"]):
        Cs = WIDTHS[s]
        x = synth.normal(g, (Cs, T, c, c))
        run(f"s{s}.resblock x2", lambda: O.resblock(x, st["blocks"][0]), Hs * Ws, c * c, 2)
        if st["up"] is not None:
            xl = synth.normal(g, (Cs, T, ch, ch))
            run(f"s{s}.up", lambda: O.upsample_conv(xl, *st["up"]), Hs * Ws, ch * ch)
            Hs, Ws = 2 * Hs, 2 * Ws
    hp = params["head"]
    xh = synth.normal(g, (WIDTHS[-1], T, c, c))
    run("head", lambda: O.head(xh, hp["gamma"], hp["beta"], hp["w"], hp["b"]), Hs * Ws, c * c)
    return T / full_t, spent, O.nthreads(), detail


def oracle_sample_text(crop, spent, reps):
    return (f"oracle (fp64 C, all host threads) on each distinct layer shape of the workload: "
            f"conv_in, one res block per stage, the 3 upsample convs and the head, each on a "
            f"{crop}x{crop}-voxel spatial crop of its input (4 frames, full channel width), "
            f"scaled per layer by full/crop output voxels and summed; {reps} sample(s), "
            f"{spent:.1f} s of oracle work")


def bench_config(world, split="replicas"):
    """The `config` object of the JSON line (both arms print the same one)."""
    if split == "rows":
        par = f"one decode split by latent rows over {world} GPU(s), NCCL halo exchange"
    else:
        par = f"replicas x{world}" if world > 1 else "single GPU"
    return {"workload": WORKLOAD,
            "parallelism": par,
            "l2": "flushed before every timed step, outside the step events (512 MiB written, "
                  "then read back: no dirty line of the flush left)",
            "trunk_dense_tflop_per_step": sum(f for _, f in trunk_layers()) / 1e12}


def cpu_baseline(reps=3):
    """Median of `reps` layer-shape samples (about 5 s each on 16 host threads)."""
    vals, spent, cores, detail = [], 0.0, 1, None
    for _ in range(reps):
        fps, dt, cores, detail = oracle_layer_sample()
        vals.append(fps)
        spent += dt
    v = statistics.median(vals)
    return {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": oracle_sample_text(ORACLE_CROP, spent, reps),
            "layer_s_full_size": detail, "full_step_s": T / v}


def run_reference(args, rank, world):
    """The reference arm: the CPU oracle, as it stands, on the host cores.  One
    step is one layer-shape sample of the workload (oracle_layer_sample), so
    `ms_per_step` is the sample's own duration; `value` is the full workload's
    frames/s that the sample measures (median over the timed steps)."""
    if rank != 0:
        return 0
    vals, secs, cores, spent = [], [], 1, 0.0
    for i in range(args.warmup + args.steps):
        fps, dt, cores, _ = oracle_layer_sample()
        if i >= args.warmup:
            vals.append(fps)
            secs.append(dt)
            spent += dt
    v = statistics.median(vals)
    sample = oracle_sample_text(ORACLE_CROP, spent, args.steps)
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.mean(secs) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) inputs, random weights with the trunk's shapes)",
        "config": bench_config(world),
        "step": "one layer-shape sample of the workload (see cpu_baseline.sample); "
                f"the full workload's step is {T / v:.0f} s at this rate",
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# -------------------------------------------------------------- components
def flush_l2(buf):
    """Evict L2 before a timed step: write a buffer larger than L2, then read it
    back, so that L2 holds none of the step's inputs and no dirty line of the
    flush (whose write-back would otherwise fall inside the timed step)."""
    buf.zero_()
    buf.sum()


def time_events(fn, reps, warm, flush):
    import torch
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        flush_l2(flush)
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record()
        fn()
        e.record()
        e.synchronize()
        ts.append(s.elapsed_time(e))
    return statistics.median(ts), min(ts)


def components(peaks, flush, reps=10):
    """Per-kernel figures of the metric on their own workloads: norm-SiLU GB/s on
    [512,4,88,156] / [256,4,176,312], the causal conv 512->512 on [512,4,88,156],
    and the res block 256->256 (and 256->128) on [256,4,176,312]."""
    import torch
    from video_diffusion_vae_b200 import binding as B
    from video_diffusion_vae_b200 import synth
    out = {}
    for shp in [(512, 4, 88, 156), (256, 4, 176, 312)]:
        x, g, b = synth.norm_silu_input(*shp)
        xd = x.permute(1, 2, 3, 0).contiguous().cuda().bfloat16()
        gd, bd = g.cuda(), b.cuda()
        y = torch.empty_like(xd)
        med, mn = time_events(lambda: B.norm_silu(xd, gd, bd, out=y), reps, 3, flush)
        gbs = 2 * xd.numel() * 2 / (med * 1e-3) / 1e9
        # Back to back over rotating buffers: the event clock ticks every ~2 us,
        # which is a tenth of one launch here, so time batches of launches; four
        # input/output pairs (> L2 together) make every launch read its input
        # from DRAM and write back the previous launches' outputs.
        nb = 4
        xs = [xd] + [xd.clone() for _ in range(nb - 1)]
        ys = [y] + [torch.empty_like(y) for _ in range(nb - 1)]
        batch = 20

        def run_batch():
            for i in range(batch):
                B.norm_silu(xs[i % nb], gd, bd, out=ys[i % nb])
        bmed, _ = time_events(run_batch, 5, 1, flush)
        per = bmed / batch
        gbs_b = 2 * xd.numel() * 2 / (per * 1e-3) / 1e9
        out[f"norm_silu_{'x'.join(map(str, shp))}"] = {
            "ms": per, "GB/s": gbs_b, "frac_hbm": gbs_b / peaks["hbm_gbs"], "frac_8TBs": gbs_b / 8000.0,
            "timing": f"median of 5 batches of {batch} launches over {nb} rotating input/output pairs",
            "single_launch_flushed": {"ms": med, "GB/s": gbs, "frac_hbm": gbs / peaks["hbm_gbs"]}}
        del xd, y, xs, ys
    x, w, b = synth.conv_input()
    pk = B.prepack_conv(w.cuda().bfloat16(), b.cuda())
    xd = x.permute(1, 2, 3, 0).contiguous().cuda().bfloat16()
    y = torch.empty_like(xd)
    med, mn = time_events(lambda: B.causal_conv3d(xd, pk, out=y), reps, 3, flush)
    fl = 2.0 * 512 * 512 * 27 * 4 * 88 * 156
    out["conv_512x512_4x88x156"] = {"ms": med, "TFLOP/s": fl / med / 1e9,
                                    "frac_bf16": fl / med / 1e9 / peaks["bf16_tflops"],
                                    "frac_2250": fl / med / 1e9 / 2250.0}
    # the same conv as Winograd F(2x2, 3x3) products (same box, same flush)
    pw = B.prepack_conv_winograd(w.cuda().bfloat16(), b.cuda())
    wsw = torch.empty(B.load().wvae_causal_conv3d_winograd_workspace_bytes(4, 88, 156, 512, 512),
                      dtype=torch.uint8, device="cuda")
    med, mn = time_events(lambda: B.causal_conv3d_winograd(xd, pw, out=y, workspace=wsw), reps, 3, flush)
    out["conv_512x512_4x88x156_winograd"] = {
        "ms": med, "TFLOP/s_dense_equiv": fl / med / 1e9,
        "frac_bf16_dense_equiv": fl / med / 1e9 / peaks["bf16_tflops"],
        "vs_direct": out["conv_512x512_4x88x156"]["ms"] / med}
    del xd, y, pk, pw, wsw
    # a 256-channel layer of the trunk's stage 2, direct and Winograd
    x, w, b = synth.conv_input(cin=256, cout=256, T=4, H=176, W=312, seed=0)
    xd = x.permute(1, 2, 3, 0).contiguous().cuda().bfloat16()
    y = torch.empty_like(xd)
    pk = B.prepack_conv(w.cuda().bfloat16(), b.cuda())
    pw = B.prepack_conv_winograd(w.cuda().bfloat16(), b.cuda())
    wsw = torch.empty(B.load().wvae_causal_conv3d_winograd_workspace_bytes(4, 176, 312, 256, 256),
                      dtype=torch.uint8, device="cuda")
    fl = 2.0 * 256 * 256 * 27 * 4 * 176 * 312
    md, _ = time_events(lambda: B.causal_conv3d(xd, pk, out=y), reps, 3, flush)
    mw, _ = time_events(lambda: B.causal_conv3d_winograd(xd, pw, out=y, workspace=wsw), reps, 3, flush)
    out["conv_256x256_4x176x312"] = {"ms": md, "TFLOP/s": fl / md / 1e9}
    out["conv_256x256_4x176x312_winograd"] = {"ms": mw, "TFLOP/s_dense_equiv": fl / mw / 1e9,
                                               "vs_direct": md / mw}
    del xd, y, pk, pw, wsw
    # the pages' video length: latents [1,48,49,44,78] -> 193 frames of 704 x 1248,
    # decoded in streaming chunks of 5 + 11 x 4 latent frames (temporal 2x steps,
    # causal caches carried between chunks)
    z49, p49 = synth.trunk_input(T=49, H=44, W=78, seed=2)
    tr49 = B.PackedTrunk(p49)
    zd49 = z49[None].cuda().bfloat16().contiguous()
    bounds = [0, 5] + [5 + 4 * k for k in range(1, 12)]
    zchunks = [zd49[:, :, a:b].contiguous() for a, b in zip(bounds, bounds[1:])]
    outs = [torch.empty((1, 3, B.video_frames(b - a, i > 0), 704, 1248), dtype=torch.bfloat16,
                        device="cuda") for i, (a, b) in enumerate(zip(bounds, bounds[1:]))]
    vs = B.VideoStream(tr49, 44, 78)
    wsv = torch.empty(tr49.video_workspace_bytes(5, 44, 78), dtype=torch.uint8, device="cuda")

    def decode_193():
        vs.started = False
        for zc, oc in zip(zchunks, outs):
            vs.decode(zc, out=oc, workspace=wsv)
    med, _ = time_events(decode_193, 3, 1, flush)
    nfr = sum(o.shape[2] for o in outs)
    assert nfr == 193
    out["video_193_frames_chunked"] = {
        "ms": med, "frames/s": nfr / (med * 1e-3),
        "workload": "latents [1,48,49,44,78] -> video [1,3,193,704,1248] (the trunk with its "
                    "temporal 2x steps), chunks of 5 + 11 x 4 latent frames"}
    del zd49, zchunks, outs, vs, wsv, tr49
    for cout in (256, 128):
        x, p = synth.resblock_input(cout=cout)
        blk = B.PackedResBlock(p)
        xd = x.permute(1, 2, 3, 0).contiguous().cuda().bfloat16()
        y = torch.empty((4, 176, 312, cout), dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(B.load().wvae_resblock_workspace_bytes(4, 176, 312, 256, cout, 0),
                         dtype=torch.uint8, device="cuda")
        med, mn = time_events(lambda: B.resblock(xd, blk, out=y, workspace=ws), reps, 3, flush)
        nv = 4 * 176 * 312
        fl = 2.0 * nv * 27 * (256 * cout + cout * cout) + (2.0 * nv * 256 * cout if cout != 256 else 0)
        out[f"resblock_256x{cout}_4x176x312"] = {"ms": med, "TFLOP/s": fl / med / 1e9,
                                                 "frac_bf16": fl / med / 1e9 / peaks["bf16_tflops"],
                                                 "frac_2250": fl / med / 1e9 / 2250.0}
        del xd, y, ws, blk
    return out


# ----------------------------------------------------- multi-rank timing
def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank number over all ranks (identity on one rank)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput(frames_per_step: int, steps: int, world: int, max_total_ms: float) -> float:
    """Whole-job frames/s: every rank decodes `steps` steps; time = slowest rank."""
    return frames_per_step * steps * world / (max_total_ms * 1e-3)


# ------------------------------------------------------------ profile cases
def profile_case(name: str, launches: int = 3) -> int:
    """Run one kernel workload `launches` times (for an ncu capture; no JSON line).
    conv512: causal conv 512->512 on [4,88,156]; norm512 / norm256: norm-SiLU on
    [512,4,88,156] / [256,4,176,312]; res256: res block 256->256 on [4,176,312];
    res128: res block 128->128 on [4,352,624] (the last stage's shape); wino512 /
    wino256: the Winograd conv 512->512 on [4,88,156] / 256->256 on [4,176,312];
    trunk: one trunk decode."""
    import torch
    from video_diffusion_vae_b200 import binding as B
    from video_diffusion_vae_b200 import synth
    torch.cuda.set_device(0)
    if name == "conv512":
        x, w, b = synth.conv_input()
        pk = B.prepack_conv(w.cuda().bfloat16(), b.cuda())
        xd = x.permute(1, 2, 3, 0).contiguous().cuda().bfloat16()
        fn = lambda: B.causal_conv3d(xd, pk)  # noqa: E731
    elif name in ("norm512", "norm256"):
        shp = (512, 4, 88, 156) if name == "norm512" else (256, 4, 176, 312)
        x, g, b = synth.norm_silu_input(*shp)
        xd = x.permute(1, 2, 3, 0).contiguous().cuda().bfloat16()
        gd, bd = g.cuda(), b.cuda()
        fn = lambda: B.norm_silu(xd, gd, bd)  # noqa: E731
    elif name == "res256":
        x, p = synth.resblock_input()
        blk = B.PackedResBlock(p)
        xd = x.permute(1, 2, 3, 0).contiguous().cuda().bfloat16()
        fn = lambda: B.resblock(xd, blk)  # noqa: E731
    elif name == "res128":
        x, p = synth.resblock_input(cin=128, cout=128, T=4, H=352, W=624)
        blk = B.PackedResBlock(p)
        xd = x.permute(1, 2, 3, 0).contiguous().cuda().bfloat16()
        fn = lambda: B.resblock(xd, blk)  # noqa: E731
    elif name in ("wino512", "wino256"):
        c, Hh, Ww = (512, 88, 156) if name == "wino512" else (256, 176, 312)
        x, w, b = synth.conv_input(cin=c, cout=c, T=4, H=Hh, W=Ww, seed=0)
        pw = B.prepack_conv_winograd(w.cuda().bfloat16(), b.cuda())
        xd = x.permute(1, 2, 3, 0).contiguous().cuda().bfloat16()
        fn = lambda: B.causal_conv3d_winograd(xd, pw)  # noqa: E731
    elif name == "trunk":
        z, params = synth.trunk_input()
        tr = B.PackedTrunk(params)
        zd = z[None].cuda().bfloat16().contiguous()
        fn = lambda: B.decode_trunk(zd, tr)  # noqa: E731
    else:
        raise SystemExit(f"unknown profile case {name}")
    for _ in range(launches):
        fn()
    torch.cuda.synchronize()
    assert B.device_error() == 0
    return 0


# ------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--split", default="replicas", choices=["replicas", "rows"],
                    help="replicas (default): one whole decode per GPU (weak scaling); rows: one "
                         "decode split by latent rows over the GPUs (strong scaling)")
    ap.add_argument("--no-components", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-case", default=None,
                    help="run one kernel workload for an ncu capture (conv512, norm512, norm256, "
                         "res256, res128, wino512, wino256, trunk) and exit")
    args = ap.parse_args()
    if args.profile_case:
        return profile_case(args.profile_case)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    args.warmup = max(args.warmup, 3)

    import torch
    import torch.distributed as dist
    from video_diffusion_vae_b200 import binding as B
    from video_diffusion_vae_b200 import synth

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=300))
    peaks, peak_kind = load_peaks()

    z, params = synth.trunk_input(T=T, H=H, W=W, seed=0)
    tr = B.PackedTrunk(params, device=dev)
    zd = z[None].to(dev, torch.bfloat16).contiguous()
    video = torch.empty((1, 3, T, 16 * H, 16 * W), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(tr.workspace_bytes(T, H, W), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    layers = trunk_layers()
    nl = B.trunk_launches()
    assert nl == len(layers)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * nl)] for _ in range(args.steps)]
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]

    rows = args.split == "rows"
    if rows:
        from video_diffusion_vae_b200 import shard
        dec = shard.RowSplitDecoder(tr, T, H, W, rank, world, device=dev)

    def step():
        if rows:
            dec.decode(zd)
        else:
            B.decode_trunk(zd, tr, out=video, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # ---- timed region: K steps, L2 flushed before each (outside the step events)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        t0 = time.perf_counter()
        for i in range(args.steps):
            flush_l2(flush)
            step_ev[i][0].record()
            step()
            step_ev[i][1].record()
        torch.cuda.synchronize()
        wall = time.perf_counter() - t0
    if world > 1:
        dist.barrier()
    step_ms = [a.elapsed_time(b) for a, b in step_ev]
    total_ms = sum(step_ms)
    max_total_ms = max_over_ranks(total_ms, dev)
    # replicas: every rank decodes; rows: the ranks decode one video together
    job_decodes = 1 if rows else world
    value = throughput(T, args.steps, job_decodes, max_total_ms)
    clocks = clk.summary()

    # ---- a second pass with events around every launch (the library records
    # them between its launches) for the per-launch durations; not in `value`
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush_l2(flush)
        B.decode_trunk(zd, tr, out=video, workspace=ws, events=ev[i])
    torch.cuda.synchronize()

    # per-launch durations -> the dominant kernel's (the tensor-core conv's)
    # share of a step; its time in the timed steps is that share of the timed
    # step (the events pass only apportions the step among its launches)
    per_layer = [[ev[i][2 * j].elapsed_time(ev[i][2 * j + 1]) for j in range(nl)] for i in range(args.steps)]
    conv_idx = [j for j, (name, _) in enumerate(layers) if name != "layout"]
    ev_conv_ms = statistics.mean(sum(per_layer[i][j] for j in conv_idx) for i in range(args.steps))
    ev_step_ms = statistics.mean(sum(per_layer[i]) for i in range(args.steps))
    conv_share = ev_conv_ms / ev_step_ms
    step_ms_timed = total_ms / args.steps            # this rank's timed step
    conv_launch_ms = conv_share * step_ms_timed / len(conv_idx)
    conv_flops = sum(layers[j][1] for j in conv_idx)
    exec_layers = trunk_layers(executed=True)
    phase_layers = trunk_layers(phase_form=True)
    conv_flops_exec = sum(exec_layers[j][1] for j in conv_idx)
    conv_flops_phase = sum(phase_layers[j][1] for j in conv_idx)
    per_launch_s = conv_launch_ms * 1e-3
    achieved = conv_flops / len(conv_idx) / per_launch_s / 1e12
    achieved_phase = conv_flops_phase / len(conv_idx) / per_launch_s / 1e12
    achieved_exec = conv_flops_exec / len(conv_idx) / per_launch_s / 1e12
    layer_ms = {layers[j][0]: statistics.mean(per_layer[i][j] for i in range(args.steps)) for j in range(nl)}

    # ---- e2e: every step copies its latents from pinned host memory and its
    # video back to pinned host memory; the copies run on their own streams
    # (one per direction, so the next step's input never queues behind the
    # previous video), double-buffered, so step i's video leaves while step
    # i+1 decodes (the way a serving loop runs).  No L2 flush here: a step's
    # working set (~1.3 GB of activations) is ten times L2.
    zh = z[None].to(torch.bfloat16).contiguous().pin_memory()
    vh = [torch.empty(video.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    zdb = [zd, torch.empty_like(zd)]
    vdb = [video, torch.empty_like(video)]
    comp_s = torch.cuda.current_stream()
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event(enable_timing=False)  # noqa: E731
    h2d_done, dec_done, d2h_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def e2e_steps(n):
        for i in range(n):
            b = i & 1
            if i >= 2:
                h2d_s.wait_event(dec_done[b])       # step i-2 has read zdb[b]
            with torch.cuda.stream(h2d_s):
                zdb[b].copy_(zh, non_blocking=True)
                h2d_done[b].record(h2d_s)
            comp_s.wait_event(h2d_done[b])
            if i >= 2:
                comp_s.wait_event(d2h_done[b])      # step i-2's video has left vdb[b]
            B.decode_trunk(zdb[b], tr, out=vdb[b], workspace=ws)
            dec_done[b].record(comp_s)
            d2h_s.wait_event(dec_done[b])
            with torch.cuda.stream(d2h_s):
                vh[b].copy_(vdb[b], non_blocking=True)
                d2h_done[b].record(d2h_s)

    def e2e_rows(n):
        # every rank copies the latents in; rank 0 copies the gathered video out
        for _ in range(n):
            zd.copy_(zh, non_blocking=True)
            v = dec.decode(zd)
            if v is not None:
                vh[0].copy_(v, non_blocking=True)

    run_e2e = e2e_rows if rows else e2e_steps
    run_e2e(3)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_start.record(comp_s)
    h2d_s.wait_stream(comp_s)  # the first input copy starts inside the timed region
    run_e2e(args.steps)
    d2h_s.wait_stream(comp_s)
    t_end.record(d2h_s)
    torch.cuda.synchronize()
    e2e_value = throughput(T, args.steps, job_decodes,
                           max_over_ranks(t_start.elapsed_time(t_end), dev))
    if rows:
        # the gathered video is the whole decode's
        if rank == 0:
            assert torch.equal(vh[0].cuda(), B.decode_trunk(zd, tr))
    else:
        assert torch.equal(vh[(args.steps - 1) & 1].cuda(), video)  # the copied-out result is the decode

    err = B.device_error()
    comp = None
    if rank == 0 and not args.no_components:
        del ws
        comp = components(peaks, flush)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline()

    if rank == 0:
        peak_t = peaks["bf16_tflops"]
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": max_total_ms / args.steps, "higher_is_better": True,
            "scaling": "strong" if rows else "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) latents, random weights with the trunk's shapes)",
            "config": bench_config(world, args.split),
            "tflops": sum(f for _, f in layers) * args.steps / (total_ms * 1e-3) / 1e12,
            "roofline": {"bound": "tensor",
                         "kernel": "the 21 conv launches of a step: conv_tc_kernel / conv_tc_staged_kernel x 20 (one body), head_tc_kernel x 1",
                         "achieved": achieved, "peak": peak_t, "unit": "TFLOP/s",
                         "frac": achieved / peak_t,
                         "peak_kind": f"{peak_kind} bf16 burst (sub-millisecond launches)",
                         "traffic": conv_traffic(), "traffic_unit": "bytes per launch (mean of the 21)",
                         "flops_per_launch": conv_flops / len(conv_idx),
                         "flop_count": "dense: every tap of the causal convs, the upsample convs "
                                       "at output resolution with 9 taps",
                         "achieved_phase_form": achieved_phase,
                         "frac_phase_form": achieved_phase / peak_t,
                         "achieved_executed": achieved_exec,
                         "frac_executed": achieved_exec / peak_t,
                         "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
                         "frac_of_2250": achieved / 2250.0,
                         "launch_ms": conv_launch_ms,
                         "conv_share_of_step": conv_share,
                         "launch_timing": "the convs' share of a step, from CUDA events around "
                                          "every launch in a second pass of the same steps, times "
                                          "the timed step's duration",
                         "events_pass_step_ms": ev_step_ms},
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": zh.numel() * 2,
                    "d2h_bytes_per_step": vh[0].numel() * 2,
                    "copies": "pinned host <-> device on one stream per direction, "
                              "double-buffered, overlapping the neighbouring steps' decodes; "
                              "no L2 flush"},
            "gpu_launches": nl * args.steps,
            "clocks": clocks,
            "wall_s_timed_region": wall,
            "layer_ms": layer_ms,
            "components": comp,
            "device_error_word": err,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

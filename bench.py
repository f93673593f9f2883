#!/usr/bin/env python
"""Throughput benchmark of the vision-to-language projector on B200.

One step = one whole pass of the bridge (placeholder index, geometry, LayerNorm,
GEMM1 with the merge-gather prologue, GEMM2 with the scatter epilogue, newline /
separator rows) over one batch of the chosen workload, through the C ABI. The line
also carries the projector backward (vlproj_backward, every gradient) timed the same
way on the same batch under "backward".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Prints ONE JSON line (rank 0). Timing: W untimed warm-up steps; then K steps, each
bracketed by CUDA events on the launching stream, with a 256 MiB write between steps
to flush L2 (outside the events); barrier + synchronize on both sides of the timed
region; max over ranks. Multi-GPU (torchrun): every rank projects its own replica
batch (weak scaling); there is no collective on the data path.

``--impl reference`` times the fp64 CPU oracle on the host cores instead (rank 0
only), on a bounded sample of the same workload per step.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "projected image tokens/s on 1 B200; % of dense BF16 tensor peak"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "stress"         # the largest single-GPU workload (262,144 tokens, 38.5 TFLOP per step)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# SM clock of the sustained cuBLAS figure when the peaks file gives none (the pool's
# earlier measurement settled near 1.4 PFLOP/s at about 1.3 GHz under the power cap)
SUSTAINED_PEAK_MHZ = 1300.0
# the sources that decide the GEMMs' DRAM traffic (kernel, its PTX, its launch and raster)
KERNEL_SOURCES = [os.path.join("vision_language_projector_b200", "csrc", f)
                  for f in ("gemm_sm100.cuh", "gelu_poly.cuh", "ptx.cuh", "host.cuh", "kernels_aux.cuh")]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.WORKLOADS))
    ap.add_argument("--images", type=int, default=0,
                    help="run the workload with this many images instead (sequences scaled to match; for "
                         "profiling captures of a smaller case); 0 = the workload's own count")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--backward-steps", type=int, default=5, help="timed vlproj_backward steps (0 = skip)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--raster-mb", type=int, default=0,
                    help="GEMM raster band budget in MB (vlproj_set_raster_budget); 0 = the library default")
    ap.add_argument("--tile-order", choices=("auto", "dynamic", "static"), default="auto",
                    help="GEMM tile order (vlproj_set_tile_order): the library's choice (default), every GEMM "
                         "from a counter, or fixed per CTA")
    ap.add_argument("--gather", default="auto", choices=["auto", "box", "im2col", "cpasync", "threads", "fused", "merged"],
                    help="GEMM1's merge-gather (vlproj_set_gather_mode); auto = the library's choice")
    return ap.parse_args()


# ----------------------------------------------------------------------------- helpers
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def peak_clock_mhz(peaks: dict, sustained: bool):
    """SM clock (MHz) under which the bf16 peak was measured, when the peaks file says."""
    for key in (("bf16_sustained_sm_mhz", "sustained_sm_mhz") if sustained else ("bf16_sm_mhz", "burst_sm_mhz")) + (
            "sm_mhz_median_under_load", "sm_mhz_median", "sm_mhz"):
        v = peaks.get(key)
        if isinstance(v, (int, float)) and v > 0:
            return float(v)
    clocks = peaks.get("clocks")
    if isinstance(clocks, dict):
        for key in ("sm_mhz_median_under_load", "median_sm_mhz", "sm_mhz_median", "sm_mhz"):
            v = clocks.get(key)
            if isinstance(v, (int, float)) and v > 0:
                return float(v)
    return None


def code_only(text: str) -> str:
    """The source without // comments, trailing blanks and empty lines: an edit of the
    comments alone keeps the stored DRAM counters valid."""
    out = []
    for line in text.splitlines():
        i = line.find("//")
        if i >= 0 and line.count('"', 0, i) % 2 == 0:
            line = line[:i]
        line = line.rstrip()
        if line:
            out.append(line)
    return "\n".join(out)


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), encoding="utf-8") as fh:
            h.update(code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def traffic_from_profiles(workload: str, kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if it was taken on
    the current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload, {}).get(kernel)
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


def workload_geometry(wl, seed):
    import vision_language_projector_b200 as vp
    hw = W.grid_hw(wl, seed)
    crop = W.spatial_crop(wl)
    cfg = vp.make_config(wl.k, wl.C, wl.N1, wl.N2, has_ln=wl.has_ln,
                         tile_tag=vp.TILE_2D if wl.tiled else vp.TILE_NONE)
    rows = vp.image_rows(cfg, hw, crop, wl.n_images)      # the library's own closed form
    return hw, crop, rows


def merged_tokens(wl, hw) -> int:
    k = wl.k
    return int(sum(((int(h) + k - 1) // k) * ((int(w) + k - 1) // k) for h, w in hw))


def flops_per_token(wl) -> int:
    return 2 * (wl.K1 * wl.N1 + wl.N1 * wl.N2)


class ClockSampler:
    """SM clock, power and throttle reasons of one GPU, polled through NVML every 5 ms on a
    background thread for as long as the timed region lasts (read-only queries)."""
    PERIOD_S = 0.005
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, device: int, enabled: bool = True):
        import threading
        self.samples = []
        self.thread = None
        self.smax = None
        if not enabled:
            return
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            prop = torch.cuda.get_device_properties(device)
            bus = f"{prop.pci_domain_id:08x}:{prop.pci_bus_id:02x}:{prop.pci_device_id:02x}.0"
            try:
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except pynvml.NVMLError:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device)
            self.nvml = pynvml
            self.smax = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            return
        self.stop_flag = threading.Event()
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def _run(self):
        n = self.nvml
        while not self.stop_flag.is_set():
            try:
                sm = n.nvmlDeviceGetClockInfo(self.h, n.NVML_CLOCK_SM)
                mask = n.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                pw = n.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                self.samples.append((sm, mask, pw))
            except Exception:
                pass
            self.stop_flag.wait(self.PERIOD_S)

    def stop(self):
        if self.thread is None:
            return None
        self.stop_flag.set()
        self.thread.join(timeout=5)
        if not self.samples:
            return None
        n = self.nvml
        reasons = sorted({name for _, mask, _ in self.samples for name, const in self.REASONS
                          if mask & getattr(n, const)})
        return {"sm_mhz": statistics.median(sm for sm, _, _ in self.samples), "sm_max_mhz": self.smax,
                "power_w_median": statistics.median(pw for _, _, pw in self.samples), "reasons": reasons,
                "samples": len(self.samples), "source": "NVML, 5 ms polling during the timed region"}


# ----------------------------------------------------------------------------- CPU oracle
def oracle_sample(wl, hw, crop, w, seed, budget_s: float, start_image: int = 0, max_images=None):
    """Time the fp64 oracle on whole images, in order from start_image, until budget_s is
    spent (at least one image). Returns (tokens, seconds, images)."""
    from oracle import projector as O
    params = O.params_f64(w)
    per = wl.views_per_image
    tokens, elapsed, n = 0, 0.0, 0
    img = start_image
    while True:
        views = list(range(img * per, (img + 1) * per))
        fe = W.features(wl, hw, seed, views=views, threads=1)
        offs = np.concatenate([[0], np.cumsum([int(hw[v, 0]) * int(hw[v, 1]) for v in views])])
        feats = [(fe[offs[i]:offs[i + 1]].astype(np.float64) if wl.feat_fp32 else
                  O.bf16_bits_to_f64(fe[offs[i]:offs[i + 1]])) for i in range(len(views))]
        vhw = [(int(hw[v, 0]), int(hw[v, 1])) for v in views]
        c = None if crop is None else (int(crop[img, 0]), int(crop[img, 1]))
        t0 = time.perf_counter()
        O.project_image(feats, vhw, wl.k, params, c, wl.ln_eps)
        elapsed += time.perf_counter() - t0
        tokens += sum(((h + wl.k - 1) // wl.k) * ((ww + wl.k - 1) // wl.k) for h, ww in vhw)
        n += 1
        img = (img + 1) % wl.n_images
        if elapsed >= budget_s or (max_images is not None and n >= max_images):
            break
    return tokens, elapsed, n


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        info = [i for i in threadpool_info() if i.get("user_api") == "blas"]
        if info:
            return int(max(i.get("num_threads", 1) for i in info))
    except Exception:
        pass
    return os.cpu_count() or 1


def pick_workload(args):
    """The named workload, or the same shapes with --images images (sequences scaled)."""
    wl = W.WORKLOADS[args.workload]
    if args.images and args.images != wl.n_images:
        seqs = max(1, -(-wl.B * args.images // wl.n_images))
        wl = dataclasses.replace(wl, n_images=args.images, B=seqs)
    return wl


def workload_config(args, wl, M: int, R: int) -> dict:
    """The workload keys of `config`, the same on both arms."""
    return {"workload": args.workload, "images": wl.n_images, "merged_tokens": M, "assembled_rows": R,
            "K1": wl.K1, "N1": wl.N1, "N2": wl.N2, "k": wl.k, "layernorm": wl.has_ln,
            "tiling": "2D" if wl.tiled else "none", "sequences": f"{wl.B}x{wl.S}"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    from oracle import projector as O
    wl = pick_workload(args)
    hw = W.grid_hw(wl, args.seed)
    crop = W.spatial_crop(wl)
    w = W.weights(wl, args.seed)
    # one step = the oracle on whole images of the workload, about a few seconds each
    budget = max(1.0, min(8.0, 150.0 / max(1, args.steps + args.warmup)))
    img = 0
    for _ in range(args.warmup):
        _, _, n = oracle_sample(wl, hw, crop, w, args.seed, budget, img, max_images=1)
        img = (img + n) % wl.n_images
    tok, sec = 0, 0.0
    for _ in range(args.steps):
        t, s, n = oracle_sample(wl, hw, crop, w, args.seed, budget, img)
        tok += t
        sec += s
        img = (img + n) % wl.n_images
    value = tok / sec
    M = sum(O.tokens_untiled(int(h_), int(w_), wl.k) for h_, w_ in hw)
    R = int(sum(O.image_rows(hw, wl.k, crop)))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * sec / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(workload_config(args, wl, M, R),
                       sample="whole images of the workload per step, fp64 numpy oracle on the host cores"),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": f"{tok} merged tokens over {args.steps} steps of whole images"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- GPU
def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    import torch.distributed as dist
    import vision_language_projector_b200 as vp

    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))

    wl = pick_workload(args)
    # data-parallel replicas: every rank holds the same weights and a batch of the same
    # shapes (geometry, placeholder layout), with feature values of its own
    seed = args.seed
    hw, crop, rows = workload_geometry(wl, seed)
    M = merged_tokens(wl, hw)
    M_all = M                              # the job's tokens: the sum over the ranks
    if world > 1:
        t = torch.tensor([float(M)], dtype=torch.float64, device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
        M_all = int(round(t.item()))
    wts = W.weights(wl, seed)
    feats_h = W.features(wl, hw, seed + rank, threads=min(16, os.cpu_count() or 1))
    ids_h = W.input_ids(wl, rows, seed)
    prefill_h = W.prefill_embeds(wl, ids_h, W.embed_table(wl, seed))

    def bf(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)

    def f32(a):
        return None if a is None else torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()

    proj = vp.Projector(wl.k, wl.C, wl.N1, wl.N2, bf(wts["W1"]), bf(wts["W2"]), f32(wts["b1"]), f32(wts["b2"]),
                        has_ln=wl.has_ln, ln_gamma=f32(wts["gamma"]), ln_beta=f32(wts["beta"]), ln_eps=wl.ln_eps,
                        feat_dtype=vp.FEAT_F32 if wl.feat_fp32 else vp.FEAT_BF16,
                        tile_tag=vp.TILE_2D if wl.tiled else vp.TILE_NONE)
    proj.set_gather_mode({"auto": vp.GATHER_AUTO, "box": vp.GATHER_BOX, "im2col": vp.GATHER_IM2COL,
                          "cpasync": vp.GATHER_CPASYNC, "threads": vp.GATHER_THREADS, "fused": vp.GATHER_FUSED,
                          "merged": vp.GATHER_MERGED}[args.gather])
    proj.set_raster_budget(args.raster_mb << 20)
    proj.set_tile_order({"static": vp.TILE_ORDER_STATIC, "auto": vp.TILE_ORDER_AUTO,
                         "dynamic": vp.TILE_ORDER_DYNAMIC}[args.tile_order])
    feats = f32(feats_h) if wl.feat_fp32 else bf(feats_h)
    ids = torch.from_numpy(ids_h).cuda()
    prefill = bf(prefill_h)
    out = prefill.clone()
    newline = bf(wts["newline"]) if wl.tiled else None
    sep = bf(wts["sep"]) if wl.tiled else None
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        proj.forward(feats, hw, crop, ids, W.IMAGE_TOKEN_ID, out, newline, sep, stream=stream, n_images=wl.n_images)

    # warm-up: every stage timed, to report per-stage times and pick the dominant kernel;
    # the timed steps then record events around that kernel only, so that stage events
    # do not separate the other kernels in the steps being measured
    proj.profile(True)
    proj.profile_stages(None)
    warm_acc = {}
    for _ in range(max(3, args.warmup)):
        step()
        for k_, v in proj.stage_ms().items():
            if v > 0.0:
                warm_acc.setdefault(k_, []).append(v)
    st = proj.status()
    if st != vp.OK:
        raise SystemExit(f"warm-up failed: {vp.strerror(st)}")
    # median over the warm-up steps: the first one also pays one-time setup (module loading,
    # kernel attributes) inside its stage events
    warm_avg = {k_: statistics.median(v) for k_, v in warm_acc.items()}
    dom = max(warm_avg, key=warm_avg.get)
    proj.profile_stages([dom])

    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local, not args.no_clocks)
    launches0 = proj.launch_count()
    step_ms, stage_acc = [], {}
    for _ in range(args.steps):
        flush.zero_()                      # L2 flush between steps, outside the events
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step()
        e1.record(stream)
        e1.synchronize()
        step_ms.append(e0.elapsed_time(e1))
        for k_, v in proj.stage_ms().items():
            if v > 0.0:                    # stages that ran in this step
                stage_acc.setdefault(k_, []).append(v)
    launches = proj.launch_count() - launches0
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clk = clocks.stop()
    st = proj.status()
    if st != vp.OK:
        raise SystemExit(f"timed steps failed: {vp.strerror(st)}")

    total_ms = float(sum(step_ms))
    if world > 1:
        t = torch.tensor([total_ms], dtype=torch.float64, device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
    value = M_all * args.steps / (total_ms / 1000.0)
    ms_per_step = total_ms / args.steps
    fl_tok = flops_per_token(wl)
    tflops = value * fl_tok / 1e12 / world

    # ---- roofline of the dominant kernel (largest average stage time in the warm-up),
    # its duration from the events around it in the timed steps
    peaks, peak_src = load_peaks()
    avg = {k_: statistics.mean(v) for k_, v in stage_acc.items()}
    sustained = total_ms > 2000.0
    peak_tf = peaks.get("bf16_tflops_sustained" if sustained else "bf16_tflops")
    if dom in ("gemm1", "gemm2"):
        fl = 2.0 * M * (wl.K1 * wl.N1 if dom == "gemm1" else wl.N1 * wl.N2)
        achieved = fl / (avg[dom] / 1000.0) / 1e12
        roof = {"kernel": dom, "bound": "tensor", "achieved": achieved, "peak": peak_tf, "unit": "TFLOP/s",
                "frac": achieved / peak_tf,
                "peak_source": f"{peak_src} bf16 {'sustained' if sustained else 'burst'}",
                "traffic": (traffic_from_profiles(args.workload, dom) if not args.images else None)}
    else:
        # algorithmic bytes of the memory-bound stages (what a perfect cache would move)
        n_ids = int(ids_h.shape[0])
        R = int(sum(rows))
        P = int(sum(int(h) * int(w_) for h, w_ in hw))
        feat_b = 4 if wl.feat_fp32 else 2
        n_special = R - M
        algo = {"index": 16 * n_ids + 4 * R,                      # ids read by count and compact, pos written
                "geometry": 12 * M,                              # pos read, rowdest + gather data written
                # features in; out: the merged bf16 A (fp32 features) or 8 B of statistics per patch
                "layernorm": P * wl.C * feat_b + (M * wl.K1 * 2 if wl.feat_fp32 else 8 * M * wl.k * wl.k),
                "special_rows": 4 * n_special * wl.N2}           # learned row read, placeholder row written
        b = algo.get(dom)
        achieved = None if b is None else b / (avg[dom] / 1000.0) / 1e9
        roof = {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": peaks.get("hbm_gbs"), "unit": "GB/s",
                "frac": None if achieved is None else achieved / peaks.get("hbm_gbs"),
                "peak_source": f"{peak_src} HBM copy", "traffic": (traffic_from_profiles(args.workload, dom) if not args.images else None),
                "algorithmic_bytes": b}

    # bytes per step: what the path must move (features in, image rows out, ids read) beside
    # what this implementation moves on top (the hidden activations written by GEMM1 and read
    # by GEMM2, per hidden layer; with a LayerNorm, the merged bf16 A written and read back)
    n_ids_step = int(ids_h.shape[0])
    R_step = int(sum(rows))
    P_step = int(sum(int(h) * int(w_) for h, w_ in hw))
    feat_b = 4 if wl.feat_fp32 else 2
    traffic_model = {
        "algorithmic_bytes": P_step * wl.C * feat_b + R_step * wl.N2 * 2 + 8 * n_ids_step,
        "hidden_round_trip_bytes": 2 * M * wl.N1 * 2,
        "merged_a_round_trip_bytes": 2 * M * wl.K1 * 2 if wl.feat_fp32 else 0,
        "layernorm_statistics_bytes": 2 * 8 * M * wl.k * wl.k if wl.has_ln and not wl.feat_fp32 else 0,
        "weights_bytes": 2 * (wl.N1 * wl.K1 + wl.N2 * wl.N1),
        "note": "per step and GPU; the hidden and merged-A round trips are implementation costs, not algorithmic",
    }
    # clock-normalised view of the dominant kernel: its FLOP per SM cycle at the median SM
    # clock seen in the timed region, against the same figure for the peak
    if clk and clk.get("sm_mhz") and roof.get("achieved"):
        mhz = float(clk["sm_mhz"])
        roof["sm_mhz"] = mhz
        roof["time_x_mhz"] = avg[dom] * mhz          # ms x MHz = thousands of SM cycles per launch
        pk_mhz = peak_clock_mhz(peaks, "sustained" in roof.get("peak_source", ""))
        if pk_mhz:
            roof["peak_sm_mhz"] = pk_mhz
            roof["frac_clock_normalised"] = roof["frac"] * pk_mhz / mhz
        if roof.get("bound") == "tensor":
            # the sustained peak scaled to this run's median clock: per-clock efficiency
            # against cuBLAS under the power cap (NVML clocks are 5 ms samples, a guide)
            s_mhz = peak_clock_mhz(peaks, True) or SUSTAINED_PEAK_MHZ
            s_tf = peaks.get("bf16_tflops_sustained")
            if s_tf:
                roof["per_clock_vs_sustained"] = roof["achieved"] / (s_tf * mhz / s_mhz)
                roof["per_clock_reference"] = f"bf16 sustained {s_tf} TFLOP/s at {s_mhz:.0f} MHz"

    # ---- end to end through the public API with host buffers: vlproj_project_host takes the
    # step's features from pinned host memory and returns the assembled rows of every image to
    # pinned host memory, its copies pipelined against the projection; the step ends when the
    # last rows have landed in host memory.
    e2e = None
    if args.e2e_steps > 0:
        R = int(sum(rows))
        feats_p = (torch.from_numpy(feats_h) if wl.feat_fp32 else torch.from_numpy(feats_h.view(np.int16))).pin_memory()
        rows_p = torch.empty((R, wl.N2), dtype=torch.int16).pin_memory()

        def e2e_step():
            proj.project_host(feats_p, hw, crop, rows_p, newline, sep, stream=stream, n_images=wl.n_images)

        proj.profile(False)            # no stage events inside the e2e steps: they report no stages

        e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e_ms = 0.0
        for _ in range(args.e2e_steps):
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            e2e_step()
            b.record(stream)
            b.synchronize()
            e_ms += a.elapsed_time(b)
        if world > 1:
            t = torch.tensor([e_ms], dtype=torch.float64, device="cuda")
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e_ms = float(t.item())
        st = proj.status()
        if st != vp.OK:
            raise SystemExit(f"e2e steps failed: {vp.strerror(st)}")
        io = [float(feats_p.numel() * feats_p.element_size()), float(rows_p.numel() * 2)]
        if world > 1:
            t = torch.tensor(io, dtype=torch.float64, device="cuda")
            dist.all_reduce(t, op=dist.ReduceOp.SUM)
            io = t.tolist()
        e2e = {"value": M_all * args.e2e_steps / (e_ms / 1000.0), "unit": UNIT,
               "h2d_bytes_per_step": int(io[0]), "d2h_bytes_per_step": int(io[1]), "steps": args.e2e_steps,
               "path": "vlproj_project_host: pinned host features in, every image's assembled rows out to "
                       "pinned host memory, copies pipelined against the projection in image chunks"}

    # ---- backward: every gradient of the projector for the same batch, timed like the forward
    bwd = None
    if args.backward_steps > 0:
        proj.profile(True)
        proj.profile_stages(None)
        gen = torch.Generator(device="cuda")
        gen.manual_seed(1000 + seed + rank)
        d_out = torch.randn((ids.numel(), wl.N2), device="cuda", generator=gen).to(torch.bfloat16)
        P = int(feats.shape[0])
        shapes = {"W1": (wl.N1, wl.K1), "b1": (wl.N1,), "W2": (wl.N2, wl.N1), "b2": (wl.N2,), "features": (P, wl.C)}
        if wl.has_ln:
            shapes.update(gamma=(wl.C,), beta=(wl.C,))
        if wl.tiled:
            shapes.update(newline=(wl.N2,), sep=(wl.N2,))
        grads = {n: torch.empty(sh, dtype=torch.float32, device="cuda") for n, sh in shapes.items()}

        from vision_language_projector_b200.shard import allreduce_gradients
        weight_grads = {n: t for n, t in grads.items() if n != "features"}

        def bstep():
            proj.backward(feats, hw, crop, ids, W.IMAGE_TOKEN_ID, d_out, grads, stream=stream, n_images=wl.n_images)
            if world > 1:
                # data-parallel training step: the ranks' weight gradients summed (one NCCL all-reduce)
                allreduce_gradients(weight_grads)

        for _ in range(3):
            bstep()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        b_ms, b_stage = [], {}
        for _ in range(args.backward_steps):
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            bstep()
            b.record(stream)
            b.synchronize()
            b_ms.append(a.elapsed_time(b))
            for k_, v in proj.stage_ms().items():
                if v > 0.0:
                    b_stage.setdefault(k_, []).append(v)
        bt = float(sum(b_ms))
        if world > 1:
            t = torch.tensor([bt], dtype=torch.float64, device="cuda")
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            bt = float(t.item())
        st = proj.status()
        if st != vp.OK:
            raise SystemExit(f"backward steps failed: {vp.strerror(st)}")
        b_step = bt / args.backward_steps
        b_flops = 2.0 * M_all * (3 * wl.K1 * wl.N1 + 2 * wl.N1 * wl.N2)       # whole job, per step
        b_tf = b_flops / world / (b_step / 1000.0) / 1e12
        b_peak = peaks.get("bf16_tflops_sustained" if bt > 2000.0 else "bf16_tflops")
        bwd = {"ms_per_step": b_step, "tflops_per_gpu": b_tf, "peak": b_peak,
               "frac_of_peak": b_tf / b_peak,
               "peak_source": f"{peak_src} bf16 {'sustained' if bt > 2000.0 else 'burst'}",
               "flops_per_step": b_flops, "steps": args.backward_steps, "gradients": sorted(shapes),
               "stage_ms": {k_: statistics.mean(v) for k_, v in b_stage.items()},
               "what": "vlproj_backward: GEMM1 recompute, dP, dW2, dW1, dA, LayerNorm backward, bias and "
                       "newline/separator sums; d_out ~N(0,1) bf16 on every id"
                       + ("; plus the all-reduce of the weight gradients over the ranks" if world > 1 else "")}
        del grads, d_out

    # ---- CPU oracle baseline (rank 0, one GPU only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tok, sec, n = oracle_sample(wl, hw, crop, wts, seed, args.cpu_seconds)
        cpu = {"value": tok / sec, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": f"{n} whole image(s) of the workload, {tok} merged tokens, fp64 numpy, {sec:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(workload_config(args, wl, M, int(sum(rows))), l2="flushed between steps (256 MiB write)",
                           gather=args.gather, raster_mb=args.raster_mb, tile_order=args.tile_order,
                           parallelism=f"replicas x{world}" if world > 1 else "single GPU"),
            "tflops_per_gpu": tflops,
            "pct_of_dense_bf16_peak": 100.0 * tflops / peaks.get("bf16_tflops"),
            "pct_of_datasheet_2250_tflops": 100.0 * tflops / 2250.0,
            "stage_ms": warm_avg,
            "stage_ms_note": "per stage, every stage timed, median over the warm-up steps; the timed steps time the dominant "
                             "kernel only",
            "roofline": roof,
            "traffic_model": traffic_model,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "backward": bwd,
            "gpu_launches": int(launches),
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    proj.close()
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

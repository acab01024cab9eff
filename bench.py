#!/usr/bin/env python
"""Throughput benchmark of the frame-causal sliding-window attention hot path.

One step = one pass of every stage of the path over one batch of synthetic
input, all inputs resident in HBM:
  * prefill   32 frames x 1004 tokens, 16 heads x 64, window 6 frames, 8 scale
              frames (schedule + tcgen05 attention)                  1.474 TFLOP
  * stream    8 consecutive frames of a 300-frame-style stream at steady state:
              append + evict on the device, split-KV attend over 8 scale + 64
              window frames (72 x 1004 keys), then the combine   8 x 0.297 TFLOP
  * band      Mistral-style token window: 32768 tokens, GQA 32/8, head_dim 128,
              W = 4096                                               2.062 TFLOP
  * decode    batch 64 at position 200000 against a 4096-slot rolling cache,
              GQA 32/8, head_dim 128 (1 GiB of K/V read)         64 tokens
Timed apart from the step and reported under ``parts`` as well: the whole
300-frame stream from an empty cache (fill included, frames/s and per-frame
latency percentiles), the whole 1000-frame stream with special-token retention
(and its last 8 frames apart), the non-keyframe attend, and the attention
prologue (with a RoPE
table and with the 3-D RoPE generated inside it).
``value`` is useful attention TFLOP/s over the whole step (visible query-key
pairs x 4 x head_dim per head; masked and padded work not counted).  Per-stage
throughput (TFLOP/s, frames/s, decode tokens/s and GB/s) is under ``parts``.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
For N > 1 launch under torchrun; each rank runs its own shard of independent
work (weak scaling, no collective on the data path).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "useful attn TFLOP/s & stream frames/s (% bf16 peak); decode tok/s (% HBM BW)"

# workload ------------------------------------------------------------------
PF = dict(F=32, P=1004, H=16, D=64, sws=6, nfpb=1, S=8)
ST = dict(P=1004, H=16, D=64, S=8, Wc=64, page=16, frames_per_step=8)
BD = dict(N=32768, Hq=32, Hkv=8, D=128, W=4096)
DC = dict(B=64, W=4096, Hq=32, Hkv=8, D=128, pos=200000)

CONFIG = {
    "workload": "frame-causal SWA hot path: prefill + streaming step + token-band GQA prefill + GQA decode",
    "prefill": "B=1, 32 frames x P=1004, C=1024 (16x64), sliding_window_size=6, num_frame_per_block=1, "
               "num_frame_for_scale=8, bf16, LayerNorm(x)@W inputs",
    "stream": "8 frames/step at steady state, P=1004, 16x64, 8 scale + 64 window frames, page 16, bf16",
    "band": "32768 tokens, GQA 32/8, head_dim 128, W=4096, bf16",
    "decode": "B=64, pos 200000 (slot 3392), 4096-slot rolling cache, GQA 32/8, head_dim 128, bf16",
    "l2": "no flush: every stage streams inputs larger than the 126 MB L2 (197 MB, 297 MB cache, "
          "403 MB, 1 GiB)",
}


def visible_frames(i, S, Wf):
    """Frames query frame i sees: scale frames plus the frame window (causal)."""
    lo = max(0, i - Wf + 1) if Wf > 0 else 0
    return min(S, i + 1) + (i + 1 - max(lo, min(S, i + 1)))


def flops_prefill():
    Wf = PF["sws"] * PF["nfpb"]
    pairs = sum(visible_frames(i, PF["S"], Wf) for i in range(PF["F"])) * PF["P"] ** 2
    return pairs * PF["H"] * 4 * PF["D"]


def flops_stream_frame():
    keys = (ST["S"] + ST["Wc"]) * ST["P"]
    return ST["P"] * keys * ST["H"] * 4 * ST["D"]


def flops_band():
    N, W = BD["N"], BD["W"]
    pairs = sum(min(t + 1, W) for t in range(N))
    return pairs * BD["Hq"] * 4 * BD["D"]


def flops_decode():
    return DC["B"] * DC["Hq"] * DC["W"] * 4 * DC["D"]


def decode_bytes():
    return 2 * DC["B"] * DC["W"] * DC["Hkv"] * DC["D"] * 2


def step_flops():
    return flops_prefill() + ST["frames_per_step"] * flops_stream_frame() + flops_band() + flops_decode()


# peaks -----------------------------------------------------------------------
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


KERNEL_SOURCES = {
    "attn": ("attn_tc.cu", "ptx.cuh", "tile_sched.h", "exp2_poly.cuh"),
    "decode": ("decode.cu", "decode_tc.cu", "ptx.cuh"),
}


def kernel_source_sha(kind="attn"):
    """Hash of the sources a kernel is built from: a recorded ncu traffic figure
    only applies while it matches."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kind]:
        with open(os.path.join(ROOT, "streaming_frame_causal_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_key):
    """DRAM bytes per launch from a committed ncu capture, if it was taken on
    the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(kernel_key)
    kind = "decode" if kernel_key.startswith("decode") else "attn"
    if not e or e.get("source_sha") != kernel_source_sha(kind):
        return None
    return e.get("bytes_per_launch")


# clocks ----------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"swa_clocks_{os.getpid()}_{gpu_index}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader",
                 "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1].split()[0]))
                    mx.append(float(parts[2].split()[0]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


def gpu_smi_id(torch, dev, fallback):
    """nvidia-smi -i accepts the GPU UUID, which survives CUDA_VISIBLE_DEVICES remapping."""
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(fallback)


# ---------------------------------------------------------------- multi-GPU plumbing
# The path shards into independent units (clips, streams, decode batches): every
# rank runs its own shard of the per-GPU workload with no collective on the data
# path (weak scaling).  Collectives appear only around the timed region: a
# barrier on entry and exit and a max over ranks of the device-timed elapsed time.
def shard_seed(rank: int) -> int:
    """Seed offset of a rank's shard: ranks draw disjoint synthetic inputs."""
    return 1000 * rank


def max_over_ranks(elapsed_ms: float, world: int, device) -> float:
    """Elapsed time of the slowest rank (all ranks must call it in the same order)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(elapsed_ms)], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(world: int, work_per_rank_step: float, steps: int, elapsed_ms: float) -> float:
    """Whole-job throughput in TFLOP/s: every rank's work over the slowest rank's time."""
    return world * work_per_rank_step * steps / (elapsed_ms * 1e-3) / 1e12


# ---------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import streaming_frame_causal_b200 as swa
    import synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    seed = shard_seed(rank)

    # ---- inputs (synthetic, seeded; shard = this rank's independent work)
    use = (lambda s: args.stage in ("all", s))
    g = torch.Generator(device=dev)
    g.manual_seed(seed + 2)
    pq = pk = pv = pout = bq = bk = bv = bout = dq = dkn = dvn = dkc = dvc = dout = dws = None
    if use("prefill"):
        pq, pk, pv = (t.to(dev) for t in synth.projected_qkv(seed=seed, F=PF["F"], P=PF["P"]))
        pout = torch.empty_like(pq)
    if use("band"):
        bq, bk, bv = (t.to(dev) for t in synth.band_qkv(seed=seed + 1))
        bout = torch.empty_like(bq)
    if use("decode"):
        dq = torch.randn(DC["B"], DC["Hq"], DC["D"], generator=g, device=dev).to(torch.bfloat16)
        dkn = torch.randn(DC["B"], DC["Hkv"], DC["D"], generator=g, device=dev).to(torch.bfloat16)
        dvn = torch.randn(DC["B"], DC["Hkv"], DC["D"], generator=g, device=dev).to(torch.bfloat16)
        dkc = torch.randn(DC["B"], DC["W"], DC["Hkv"], DC["D"], generator=g, device=dev).to(torch.bfloat16)
        dvc = torch.randn(DC["B"], DC["W"], DC["Hkv"], DC["D"], generator=g, device=dev).to(torch.bfloat16)
        dout = torch.empty_like(dq)
        dws = torch.empty(swa.swa_decode_workspace_bytes(DC["B"], DC["Hq"], DC["Hkv"], DC["D"], DC["W"]),
                          dtype=torch.uint8, device=dev)
    n_pool = 16
    frames, sout, cache = [], None, None
    state = {"frame": 0}
    if use("stream"):
        frames = [tuple(torch.randn(ST["P"], ST["H"], ST["D"], generator=g, device=dev).to(torch.bfloat16)
                        for _ in range(3)) for _ in range(n_pool)]
        sout = torch.empty(ST["P"], ST["H"], ST["D"], dtype=torch.bfloat16, device=dev)
        total_frames = ST["S"] + ST["Wc"] + (args.warmup + 2 * args.steps + 4) * ST["frames_per_step"]
        cache = swa.SwaStream(num_layers=1, heads=ST["H"], head_dim=ST["D"], P=ST["P"], scale_frames=ST["S"],
                              window_frames=ST["Wc"], page_tokens=ST["page"], max_frames=total_frames,
                              max_splits=12, device=dev)

    def stream_frame(fr=None, out=None):
        i = state["frame"]
        fq, fk, fv = frames[i % n_pool] if fr is None else fr
        cache.swa_stream_append_evict(0, i, fk, fv)
        cache.swa_stream_attend(0, i, fq, sout if out is None else out)
        state["frame"] = i + 1

    if use("stream"):
        # fill the cache to steady state (8 scale + 64 window frames), untimed
        for _ in range(ST["S"] + ST["Wc"]):
            stream_frame()

    def prefill(q=pq, k=pk, v=pv, out=pout):
        swa.swa_prefill(q, k, v, out, S=PF["F"], P=PF["P"], sliding_window_size=PF["sws"],
                        num_frame_per_block=PF["nfpb"], num_frame_for_scale=PF["S"])

    def band(q=bq, k=bk, v=bv, out=bout):
        swa.swa_band_prefill(q, k, v, out, window=BD["W"])

    def decode(q=dq, k_new=dkn, v_new=dvn, out=dout):
        swa.swa_decode(q, k_new, v_new, dkc, dvc, DC["pos"], out, workspace=dws)

    def stream_part(frame_evs=None):
        # frame_evs: events around each frame (append + attend) for
        # per-frame latency percentiles
        for j in range(ST["frames_per_step"]):
            if frame_evs is not None:
                frame_evs[j].record(stream)
            stream_frame()
        if frame_evs is not None:
            frame_evs[ST["frames_per_step"]].record(stream)

    all_parts = [("prefill", prefill), ("stream", stream_part), ("band", band), ("decode", decode)]
    parts = [(n, fn) for n, fn in all_parts if use(n)]

    def step(evs=None, frame_evs=None):
        for j, (name, fn) in enumerate(parts):
            if evs is not None:
                evs[j].record(stream)
            if name == "stream":
                fn(frame_evs)
            else:
                fn()
        if evs is not None:
            evs[len(parts)].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if swa.swa_device_error_check() != 0:
        raise RuntimeError("device error flag set during warm-up")

    # ---- device-timed region
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(gpu_smi_id(torch, dev, local_rank))
    clocks.start()
    time.sleep(0.25)
    part_ms = {name: 0.0 for name, _ in parts}
    launches0 = swa.swa_launch_count()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(parts) + 1)] for _ in range(args.steps)]
    fev = [[torch.cuda.Event(enable_timing=True) for _ in range(ST["frames_per_step"] + 1)]
           for _ in range(args.steps)] if use("stream") else [None] * args.steps
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for s in range(args.steps):
        step(ev[s], fev[s])
    end.record(stream)
    torch.cuda.synchronize()
    launches = swa.swa_launch_count() - launches0
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    elapsed_ms = start.elapsed_time(end)
    for s in range(args.steps):
        for j, (name, _) in enumerate(parts):
            part_ms[name] += ev[s][j].elapsed_time(ev[s][j + 1])
    if swa.swa_device_error_check() != 0:
        raise RuntimeError("device error flag set during the timed region")
    elapsed_ms = max_over_ranks(elapsed_ms, world, dev)
    ms_per_step = elapsed_ms / args.steps
    stage_flops = {"prefill": flops_prefill(), "stream": ST["frames_per_step"] * flops_stream_frame(),
                   "band": flops_band(), "decode": flops_decode()}
    flops = sum(stage_flops[n] for n, _ in parts)
    value = weak_scaling_value(world, flops, args.steps, elapsed_ms)

    peaks = measured_peaks()
    per = {k: v / args.steps for k, v in part_ms.items()}
    parts_out = {}
    if "prefill" in per:
        parts_out["prefill_tflops"] = flops_prefill() / (per["prefill"] * 1e-3) / 1e12
        parts_out["prefill_ms"] = per["prefill"]
        parts_out["prefill_frac_of_bf16"] = parts_out["prefill_tflops"] / peaks["bf16_tflops"]
        parts_out["prefill_frac_of_bf16_sustained"] = parts_out["prefill_tflops"] / peaks["bf16_tflops_sustained"]
    if "stream" in per:
        parts_out["stream_frames_per_s"] = ST["frames_per_step"] / (per["stream"] * 1e-3)
        parts_out["stream_ms_per_frame"] = per["stream"] / ST["frames_per_step"]
        parts_out["stream_tflops"] = stage_flops["stream"] / (per["stream"] * 1e-3) / 1e12
        parts_out["stream_frac_of_bf16"] = parts_out["stream_tflops"] / peaks["bf16_tflops"]
        parts_out["stream_frac_of_bf16_sustained"] = parts_out["stream_tflops"] / peaks["bf16_tflops_sustained"]
        lat = sorted(fev[s][j].elapsed_time(fev[s][j + 1]) for s in range(args.steps)
                     for j in range(ST["frames_per_step"]))
        parts_out["stream_frame_ms_p50"] = lat[len(lat) // 2]
        parts_out["stream_frame_ms_p99"] = lat[min(len(lat) - 1, (99 * len(lat)) // 100)]
    if "stream" in per and not args.no_extras:
        # the non-keyframe path at the same steady state (timed apart from the
        # step): the frame attends to the cache plus itself, nothing persists,
        # so its keys are 8 scale + 64 window + 1 frames
        tq, tk, tv = frames[0]
        nk_out = torch.empty_like(sout)
        for _ in range(3):
            cache.swa_stream_attend_transient(0, tq, tk, tv, nk_out)
        n_nk = 8
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n_nk):
            cache.swa_stream_attend_transient(0, tq, tk, tv, nk_out)
        e1.record(stream)
        torch.cuda.synchronize()
        nk_ms = e0.elapsed_time(e1) / n_nk
        nk_flops = flops_stream_frame() * (ST["S"] + ST["Wc"] + 1) / (ST["S"] + ST["Wc"])
        parts_out["stream_nonkey_ms_per_frame"] = nk_ms
        parts_out["stream_nonkey_frames_per_s"] = 1e3 / nk_ms
        parts_out["stream_nonkey_tflops"] = nk_flops / (nk_ms * 1e-3) / 1e12
        # the attention prologue of a streaming frame (norm1, qkv linear on the
        # tensor cores, q/k norms, RoPE), timed apart from the step
        Cm = ST["H"] * ST["D"]
        pin = {k: t.to(dev) for k, t in synth.prologue_inputs(seed=9, P=ST["P"], C=Cm, heads=ST["H"]).items()}
        pre_args = [pin[n] for n in ("ln_w", "ln_b", "w_qkv", "b_qkv", "qn_w", "qn_b", "kn_w", "kn_b", "rot")]
        pre_out = [torch.empty(ST["P"], ST["H"], ST["D"], dtype=torch.bfloat16, device=dev) for _ in range(3)]
        pre_ws = torch.empty_like(pin["x"])
        def pre():
            swa.swa_attn_pre(pin["x"], *pre_args, heads=ST["H"], q_out=pre_out[0], k_out=pre_out[1],
                             v_out=pre_out[2], xn_ws=pre_ws)
        for _ in range(3):
            pre()
        n_pre = 20
        # a GPU-side sleep first, so the host has queued all calls before the GPU
        # reaches them and the events time the kernels, not the Python call rate
        torch.cuda._sleep(50_000_000)
        e0.record(stream)
        for _ in range(n_pre):
            pre()
        e1.record(stream)
        torch.cuda.synchronize()
        pre_ms = e0.elapsed_time(e1) / n_pre
        parts_out["prologue_us"] = pre_ms * 1e3
        parts_out["prologue_qkv_tflops"] = 2.0 * ST["P"] * Cm * 3 * Cm / (pre_ms * 1e-3) / 1e12
        # the same prologue with the frame's 3-D RoPE generated inside it (no table)
        def pre3d():
            swa.swa_attn_pre_rope3d(pin["x"], *pre_args[:-1], heads=ST["H"], frame_idx=999, num_special=5,
                                    grid_w=27, q_out=pre_out[0], k_out=pre_out[1], v_out=pre_out[2], xn_ws=pre_ws)
        for _ in range(3):
            pre3d()
        torch.cuda._sleep(50_000_000)
        e0.record(stream)
        for _ in range(n_pre):
            pre3d()
        e1.record(stream)
        torch.cuda.synchronize()
        parts_out["prologue_rope3d_us"] = e0.elapsed_time(e1) / n_pre * 1e3
        parts_out.update(whole_streams(swa, torch, dev, stream, frames))
    if "band" in per:
        parts_out["band_tflops"] = flops_band() / (per["band"] * 1e-3) / 1e12
        parts_out["band_ms"] = per["band"]
        parts_out["band_frac_of_bf16"] = parts_out["band_tflops"] / peaks["bf16_tflops"]
        parts_out["band_frac_of_bf16_sustained"] = parts_out["band_tflops"] / peaks["bf16_tflops_sustained"]
    if "decode" in per:
        parts_out["decode_tok_per_s"] = DC["B"] / (per["decode"] * 1e-3)
        parts_out["decode_us"] = per["decode"] * 1e3
        parts_out["decode_gbs"] = decode_bytes() / (per["decode"] * 1e-3) / 1e9
        parts_out["decode_frac_of_hbm"] = parts_out["decode_gbs"] / peaks["hbm_gbs"]
        # the decode target is stated against about 8 TB/s of HBM3e bandwidth
        parts_out["decode_frac_of_8tbs"] = parts_out["decode_gbs"] / 8000.0

    # roofline of the dominant kernel: the kernel with the largest summed time in
    # the step.  attn_tc_kernel<64> runs the prefill launch and the eight
    # streaming attends; its launch duration is taken on the prefill launch, the
    # one launch of it that the step brackets alone with CUDA events (a streaming
    # attend shares its events with the append kernel), and on the
    # streaming stage only when the prefill stage is not run.
    cands = []
    if "band" in per:
        cands.append((per["band"], per["band"], "attn_tc_kernel<128> band 32768 tok GQA 32/8", flops_band(),
                      "attn_tc_band_32768_gqa32_8_d128", "tensor"))
    if "prefill" in per or "stream" in per:
        share = per.get("prefill", 0.0) + per.get("stream", 0.0)
        if "prefill" in per:
            cands.append((share, per["prefill"], "attn_tc_kernel<64>, prefill launch 32x1004 16x64",
                          flops_prefill(), "attn_tc_prefill_32x1004_h16_d64", "tensor"))
        else:
            cands.append((share, per["stream"], "attn_tc_kernel<64> stream attend + append, 8 frames",
                          stage_flops["stream"], "attn_tc_stream_72x1004_h16_d64", "tensor"))
    if "decode" in per:
        cands.append((per["decode"], per["decode"], "decode_tc_kernel<4> B64 W4096", decode_bytes(),
                      "decode_b64_w4096_gqa32_8_d128", "hbm"))
    _, kms, kname, kwork, tkey, bound = max(cands)
    if bound == "tensor":
        achieved = kwork / (kms * 1e-3) / 1e12
        # the dominant launch lasts about 2 ms at full clock inside a sub-second
        # timed region: the burst bf16 figure is its peak; the sustained one (a
        # seconds-long power-capped loop) is kept as a second reference
        roof = {"kernel": kname, "bound": "tensor", "achieved": achieved,
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"],
                "peak_note": f"{peaks['source']} burst bf16 peak",
                "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
                "traffic": recorded_traffic(tkey)}
    else:
        achieved = kwork / (kms * 1e-3) / 1e9
        roof = {"kernel": kname, "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "peak_note": f"{peaks['source']} HBM copy bandwidth",
                "traffic": recorded_traffic(tkey)}

    # ---- end to end through the public API: pinned host inputs -> device -> results back
    e2e = None if args.no_extras else run_e2e(args, swa, torch, dev, stream, parts, pq, pk, pv, pout, bq, bk,
                                               bv, bout, dq, dkn, dvn, dout, frames, sout, prefill, band, decode,
                                               stream_frame, world, dist, flops)

    out = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": CONFIG if args.stage == "all" else dict(CONFIG, stage_only=args.stage),
        "parts": parts_out, "roofline": roof, "e2e": e2e, "gpu_launches": int(launches),
        "clocks": clk,
    }
    return out


def stream_keys(i, S, Wc, P, specials=0):
    """Keys frame i attends to: retained full frames (scale + window) times P,
    plus the special tokens kept from evicted frames."""
    n_full = min(i + 1, S + Wc) if Wc > 0 else i + 1
    n_evicted = max(0, i + 1 - S - Wc) if Wc > 0 else 0
    return n_full * P + specials * n_evicted


def whole_streams(swa, torch, dev, stream, frames):
    """Two streams timed apart from the step, append + attend per frame:
    * the 300-frame stream from an empty cache (fill included): frames/s over
      all 300 frames and per-frame latency percentiles;
    * the 1000-frame stream that keeps the 5 special tokens of every evicted
      frame, from an empty cache: frames/s over all 1000 frames, per-frame
      latency percentiles, and the last 8 frames apart (76,928 keys at 999).
    Frame contents come from the pool of 16 synthetic frames."""
    out = {}
    P, H, D, S, Wc = ST["P"], ST["H"], ST["D"], ST["S"], ST["Wc"]
    sout = torch.empty(P, H, D, dtype=torch.bfloat16, device=dev)
    n_pool = len(frames)
    # ---- 300 frames, fill included
    F = 300
    cache = swa.SwaStream(num_layers=1, heads=H, head_dim=D, P=P, scale_frames=S, window_frames=Wc,
                          page_tokens=ST["page"], max_frames=F, max_splits=12, device=dev)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(F + 1)]
    torch.cuda._sleep(50_000_000)
    for i in range(F):
        fq, fk, fv = frames[i % n_pool]
        evs[i].record(stream)
        cache.swa_stream_append_evict(0, i, fk, fv)
        cache.swa_stream_attend(0, i, fq, sout)
    evs[F].record(stream)
    torch.cuda.synchronize()
    lat = sorted(evs[i].elapsed_time(evs[i + 1]) for i in range(F))
    total = evs[0].elapsed_time(evs[F])
    fl = sum(P * stream_keys(i, S, Wc, P) * H * 4 * D for i in range(F))
    out["stream300_frames_per_s"] = F / (total * 1e-3)
    out["stream300_tflops"] = fl / (total * 1e-3) / 1e12
    out["stream300_frame_ms_p50"] = lat[F // 2]
    out["stream300_frame_ms_p99"] = lat[min(F - 1, (99 * F) // 100)]
    cache.close()
    # ---- 1000 frames with special-token retention, fill included
    F = 1000
    cache = swa.SwaStream(num_layers=1, heads=H, head_dim=D, P=P, scale_frames=S, window_frames=Wc,
                          page_tokens=ST["page"], cross_frame_special=True, num_special=5, max_frames=F,
                          max_splits=12, device=dev)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(F + 1)]
    torch.cuda._sleep(50_000_000)
    for i in range(F):
        fq, fk, fv = frames[i % n_pool]
        evs[i].record(stream)
        cache.swa_stream_append_evict(0, i, fk, fv)
        cache.swa_stream_attend(0, i, fq, sout)
    evs[F].record(stream)
    torch.cuda.synchronize()
    lat = sorted(evs[i].elapsed_time(evs[i + 1]) for i in range(F))
    total = evs[0].elapsed_time(evs[F])
    fl_all = sum(P * stream_keys(i, S, Wc, P, 5) * H * 4 * D for i in range(F))
    out["stream1000_frames_per_s"] = F / (total * 1e-3)
    out["stream1000_tflops"] = fl_all / (total * 1e-3) / 1e12
    out["stream1000_frame_ms_p50"] = lat[F // 2]
    out["stream1000_frame_ms_p99"] = lat[min(F - 1, (99 * F) // 100)]
    t0 = F - 8
    ms = evs[t0].elapsed_time(evs[F])
    fl = sum(P * stream_keys(i, S, Wc, P, 5) * H * 4 * D for i in range(t0, F))
    out["stream1000_special_keys_at_999"] = stream_keys(F - 1, S, Wc, P, 5)
    out["stream1000_special_ms_per_frame"] = ms / (F - t0)
    out["stream1000_special_frames_per_s"] = (F - t0) / (ms * 1e-3)
    out["stream1000_special_tflops"] = fl / (ms * 1e-3) / 1e12
    cache.close()
    return out


def run_e2e(args, swa, torch, dev, stream, parts, pq, pk, pv, pout, bq, bk, bv, bout, dq, dkn, dvn, dout,
            frames, sout, prefill, band, decode, stream_frame, world, dist, flops):
    """The same step through the public API with every input copied from pinned
    host memory and every output copied back, inside the timed region.

    Steps are pipelined the way a serving loop would run them: inputs and
    outputs are double-buffered on the device, host-to-device copies run on one
    stream, the attention calls on the compute stream and the read-backs on a
    third, ordered by events, so step s+1's inputs arrive and step s-1's results
    leave while step s computes.  The timed region runs from the first input
    copy to the last read-back."""
    fps = ST["frames_per_step"]
    names = [n for n, _ in parts]
    fns = {"prefill": prefill, "band": band, "decode": decode}
    stage_io = {}
    if "prefill" in names:
        stage_io["prefill"] = ([pq, pk, pv], pout)
    if "band" in names:
        stage_io["band"] = ([bq, bk, bv], bout)
    if "decode" in names:
        stage_io["decode"] = ([dq, dkn, dvn], dout)
    use_stream = "stream" in names
    h_in = {n: [t.cpu().pin_memory() for t in ins] for n, (ins, _) in stage_io.items()}
    h_out = {n: torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for n, (_, o) in stage_io.items()}
    h_frames = [tuple(t.cpu().pin_memory() for t in frames[j]) for j in range(fps)] if use_stream else []
    h_sout = [torch.empty(sout.shape, dtype=sout.dtype, pin_memory=True) for _ in range(fps)] if use_stream else []
    d_in = [{n: [torch.empty_like(t) for t in ins] for n, (ins, _) in stage_io.items()} for _ in range(2)]
    d_out = [{n: torch.empty_like(o) for n, (_, o) in stage_io.items()} for _ in range(2)]
    d_frames = [[tuple(torch.empty_like(t) for t in frames[j]) for j in range(fps)] if use_stream else []
                for _ in range(2)]
    d_sout = [[torch.empty_like(sout) for _ in range(fps)] if use_stream else [] for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for ts in h_in.values() for t in ts) + sum(
        t.numel() * t.element_size() for fr in h_frames for t in fr)
    d2h = sum(t.numel() * t.element_size() for t in h_out.values()) + sum(
        t.numel() * t.element_size() for t in h_sout)

    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(s):
        k = s % 2
        with torch.cuda.stream(s_in):
            if s >= 2:
                s_in.wait_event(ev_comp[k])  # step s-2 no longer reads input set k
            for n, hs in h_in.items():
                for h, d in zip(hs, d_in[k][n]):
                    d.copy_(h, non_blocking=True)
            for j in range(len(h_frames)):
                for h, d in zip(h_frames[j], d_frames[k][j]):
                    d.copy_(h, non_blocking=True)
            ev_in[k].record(s_in)
        stream.wait_event(ev_in[k])
        if s >= 2:
            stream.wait_event(ev_out[k])  # step s-2's results in output set k were read back
        with torch.cuda.stream(stream):
            for name, _ in parts:
                if name == "stream":
                    for j in range(fps):
                        stream_frame(d_frames[k][j], d_sout[k][j])
                else:
                    fns[name](*d_in[k][name], d_out[k][name])
            ev_comp[k].record(stream)
        s_out.wait_event(ev_comp[k])
        with torch.cuda.stream(s_out):
            for n, h in h_out.items():
                h.copy_(d_out[k][n], non_blocking=True)
            for j in range(len(h_sout)):
                h_sout[j].copy_(d_sout[k][j], non_blocking=True)
            ev_out[k].record(s_out)

    steps = max(3, args.steps // 4)
    for s in range(2):
        e2e_step(s)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    for s in range(2, 2 + steps):
        e2e_step(s)
    b.record(s_out)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    ms = max_over_ranks(ms, world, dev)
    return {"value": weak_scaling_value(world, flops, steps, ms), "unit": "TFLOP/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": steps,
            "ms_per_step": ms / steps, "pipelined": "double-buffered inputs/outputs, copy-in / compute / "
                                                    "copy-out streams"}


# ---------------------------------------------------------------- oracle arm
def oracle_sample_setup():
    """Inputs for one bounded oracle sample of each stage (same shapes and
    distributions as the GPU workload, generated on the host)."""
    import numpy as np
    import torch

    import synth
    from oracle import attention as orc

    pq, pk, pv = synth.projected_qkv(seed=0, F=PF["F"], P=PF["P"])
    pre = tuple(x[:, :, :1].float().numpy() for x in (pq, pk, pv))  # one head, all tokens
    cache = orc.StreamCache(heads=1, head_dim=ST["D"], P=ST["P"], scale_frames=ST["S"],
                            window_frames=ST["Wc"], page_tokens=ST["page"])
    for i in range(ST["S"] + ST["Wc"]):
        _, k, v = synth.stream_frame(i, P=ST["P"], H=1, D=ST["D"])
        cache.append_evict(0, i, k.float().numpy(), v.float().numpy())
    n_band = BD["W"] + 127
    bq = synth.normal((1, n_band, 4, BD["D"]), 5).numpy()
    bk = synth.normal((1, n_band, 1, BD["D"]), 6).numpy()
    bv = synth.normal((1, n_band, 1, BD["D"]), 7).numpy()
    dq, dkn, dvn, dkc, dvc = (x.float().numpy() for x in synth.decode_inputs(seed=1, B=1))
    return {"orc": orc, "np": np, "synth": synth, "pre": pre, "cache": cache, "frame": ST["S"] + ST["Wc"],
            "band": (bq, bk, bv, n_band), "dec": (dq, dkn, dvn, dkc, dvc)}


def oracle_sample_step(ctx):
    """One bounded oracle sample: one query frame x one head of the prefill,
    one streaming frame (one head), 128 band rows x 4 heads, one decode
    sequence.  Returns the useful FLOPs it computed."""
    orc, np = ctx["orc"], ctx["np"]
    q, k, v = ctx["pre"]
    f = PF["F"] - 1
    rows = np.arange(f * PF["P"], (f + 1) * PF["P"])
    orc.prefill(q, k, v, P=PF["P"], scale_frames=PF["S"], sliding_window_size=PF["sws"],
                num_frame_per_block=PF["nfpb"], rows=rows)
    fl = PF["P"] * visible_frames(f, PF["S"], PF["sws"] * PF["nfpb"]) * PF["P"] * 4 * PF["D"]
    i = ctx["frame"]
    fq, fk, fv = ctx["synth"].stream_frame(i, P=ST["P"], H=1, D=ST["D"])
    ctx["cache"].append_evict(0, i, fk.float().numpy(), fv.float().numpy())
    ctx["cache"].attend(0, fq.float().numpy())
    ctx["frame"] = i + 1
    fl += ST["P"] * (ST["S"] + ST["Wc"]) * ST["P"] * 4 * ST["D"]
    bq, bk, bv, n = ctx["band"]
    rows = np.arange(n - 128, n)
    orc.band_attention(bq, bk, bv, BD["W"], rows=rows)
    fl += 128 * BD["W"] * 4 * BD["D"] * 4
    dq, dkn, dvn, dkc, dvc = ctx["dec"]
    orc.decode(dq, dkn, dvn, dkc, dvc, DC["pos"], DC["W"])
    fl += DC["Hq"] * DC["W"] * 4 * DC["D"]
    return fl


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline(budget_s=15.0):
    ctx = oracle_sample_setup()
    oracle_sample_step(ctx)  # warm
    t0 = time.perf_counter()
    fl, n = 0, 0
    while time.perf_counter() - t0 < budget_s or n == 0:
        fl += oracle_sample_step(ctx)
        n += 1
    dt = time.perf_counter() - t0
    return {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
            "sample": f"{n} samples in {dt:.1f} s; each = 1 query frame x 1 head of the prefill, 1 stream frame "
                      "x 1 head vs 72x1004 keys, 128 band rows x 4 heads x 4096 keys, 1 decode sequence "
                      "x 32 heads x 4096 slots; float64 NumPy oracle"}


def run_reference(args):
    ctx = oracle_sample_setup()
    for _ in range(args.warmup):
        oracle_sample_step(ctx)
    t0 = time.perf_counter()
    fl = 0
    for _ in range(args.steps):
        fl += oracle_sample_step(ctx)
    dt = time.perf_counter() - t0
    value = fl / dt / 1e12
    cores = cpu_cores()
    sample = ("each step = 1 query frame x 1 head of the prefill, 1 stream frame x 1 head vs 72x1004 keys, "
              "128 band rows x 4 heads x 4096 keys, 1 decode sequence x 32 heads; float64 NumPy oracle")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": CONFIG,
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--stage", choices=("all", "prefill", "stream", "band", "decode"), default="all",
                    help="time one stage only (for profiling); the reported value then covers that stage")
    ap.add_argument("--no-extras", action="store_true",
                    help="run the timed step only: skip the measurements taken apart from it (non-keyframe "
                         "attend, prologue, whole streams) and the end-to-end pass (for launch lists)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world:
        if world == 1 and args.gpus > 1:
            sys.exit("run --gpus N > 1 under torchrun (one process per GPU)")

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    import torch
    import torch.distributed as dist
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        out = run_ours(args, rank, world, local_rank)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline and args.stage == "all":
                out["cpu_baseline"] = cpu_baseline()
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

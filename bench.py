#!/usr/bin/env python
"""Benchmark of the ViT tower + 2x2 merge + projector forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload tower448|tower2016|attn65536|...]
    python bench.py --impl reference ...      # the fp64 CPU oracle on the host cores

One step = one forward of the whole path (patch unfold, patch embedding, 32 layers,
merge, projector) over one batch of synthetic input resident in HBM.  The timed region
is K steps, each bracketed by CUDA events on the launching stream, with an L2 flush
(a 512 MB write) between steps outside the events; barrier + synchronize on both sides;
the maximum over ranks is reported.  N > 1 runs independent replicas, one per GPU
(torchrun), each with its own batch: weak scaling, no collective in the data path.

Rank 0 prints one JSON line.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from vision_transformer_encoder_vit_b200 import replicas as REP  # noqa: E402
from vision_transformer_encoder_vit_b200 import synthetic as S  # noqa: E402

METRIC = "ViT tower images/s & tokens/s at 448²/2016²; attention+GEMM TFLOP/s vs BF16 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL_BF16_TFLOPS = 2250.0  # B200 dense bf16, the vendor's figure without sparsity


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


KERNEL_SOURCES = {"gemm": "gemm.cu", "attention": "attention.cu", "attention_backward": "attention_bwd.cu"}


def recorded_traffic(cls: str, workload_name: str):
    """Per-launch DRAM bytes of a kernel class from the committed ncu capture
    (profiles/traffic_<workload>.txt), or None if there is none for this workload or
    the kernel's sources changed since the capture."""
    import hashlib
    path = os.path.join(ROOT, "profiles", f"traffic_{workload_name}.txt")
    if not os.path.exists(path):
        return None
    csrc = os.path.join(ROOT, "vision_transformer_encoder_vit_b200", "csrc")
    data = open(os.path.join(csrc, KERNEL_SOURCES[cls]), "rb").read() + open(os.path.join(csrc, "ptx.cuh"), "rb").read()
    sha = hashlib.sha1(data).hexdigest()
    for line in open(path):
        f = line.split()
        if len(f) >= 8 and f[0] == "kernel_class" and f[1] == cls:
            return float(f[7]) if f[3] == sha else None
    return None


def workload(name: str) -> dict:
    """Shape of the benchmarked step."""
    if name in ("tower448", "tower2016"):
        cfg = S.get_config(name)
        t, gh, gw = S.token_grid(cfg)
        N = t * gh * gw
        return dict(kind="tower", name=name, cfg=cfg, batch=cfg["batch"], grid=(t, gh, gw), tokens=N,
                    desc=f"full tower (32 layers) + 2x2 merge + projector, {cfg['batch']} image(s) of "
                         f"{cfg['image'][0]}x{cfg['image'][1]}")
    if name == "varlen_mix":
        cfg = S.get_config("tower448")
        images = [(448, 448), (336, 448), (224, 224), (672, 672), (448, 224), (560, 560), (280, 392), (448, 448)]
        grids = [(1, h // cfg["patch"], w // cfg["patch"]) for h, w in images]
        return dict(kind="varlen", name=name, cfg=cfg, batch=len(images), images=images, grids=grids,
                    tokens=sum(g[1] * g[2] for g in grids),
                    desc="full tower + 2x2 merge + projector on one packed batch of 8 images of mixed sizes "
                         + ", ".join(f"{h}x{w}" for h, w in images))
    if name == "backward448":
        cfg = S.get_config("tower448")
        t, gh, gw = S.token_grid(cfg)
        return dict(kind="backward", name=name, cfg=cfg, batch=cfg["batch"], grid=(t, gh, gw), tokens=t * gh * gw,
                    desc=f"tower forward keeping every layer's input + backward to the pixels (32 layers), "
                         f"{cfg['batch']} images of 448x448")
    if name == "u8_672":
        cfg = dict(S.get_config("tower448"), image=(672, 672))
        sizes = [(1080, 1920), (768, 1024), (480, 640), (3024, 4032), (1200, 1600), (720, 1280), (2000, 3000),
                 (512, 512)]
        return dict(kind="u8", name=name, cfg=cfg, batch=len(sizes), sizes=sizes, grid=(1, 48, 48), tokens=48 * 48,
                    desc="decoded 8-bit images of 8 photo sizes (" + ", ".join(f"{h}x{w}" for h, w in sizes)
                         + ") resized on the GPU to 672x672 (bicubic, CLIP normalisation) + full tower + 2x2 merge"
                         " + projector")
    if name.startswith("video"):  # video<side>_f<frames>: 2 clips of that many square frames
        side, frames = (int(v) for v in name[5:].split("_f"))
        cfg = dict(S.get_config("tower448"), image=(side, side), batch=2)
        t, gh, gw = -(-frames // cfg["temporal_patch"]), side // cfg["patch"], side // cfg["patch"]
        return dict(kind="video", name=name, cfg=cfg, batch=2, frames=frames, grid=(t, gh, gw), tokens=t * gh * gw,
                    desc=f"full tower + 2x2 merge + projector, 2 clips of {frames} frames of {side}x{side} "
                         f"({t} temporal patches, {t * gh * gw} tokens per clip)")
    if name.startswith("attnbwd"):  # attnbwd<N>: the backward alone, 8 images of N tokens
        n = int(name[7:])
        return dict(kind="attn_bwd", name=name, batch=8, grid=None, tokens=n, heads=16, D=80,
                    desc=f"attention backward only (dq, dk, dv from q, k, v, dO; recomputed forward), "
                         f"8 images x 16 heads x 80, {n} tokens, no rotary embedding")
    if name.startswith("attn"):
        n = int(name[4:])
        side = int(round(n ** 0.5))
        return dict(kind="attn", name=name, batch=1, grid=(1, side, side), tokens=side * side, heads=16, D=80,
                    desc=f"attention only, 16 heads x 80, {side}x{side} tokens, 3D RoPE")
    raise SystemExit(f"unknown workload {name}")


def backward_flops(cfg: dict, N: int) -> float:
    """Algorithmic FLOPs of one image's tower forward plus its input-gradient backward:
    every linear layer's dX product costs what its forward costs; the attention backward
    is 5 products (S, dP, dV, dK, dQ) = 10 N^2 d; the score products it recomputes are
    not counted."""
    d, m = cfg["hidden"], cfg["mlp"]
    K0 = 3 * cfg["temporal_patch"] * cfg["patch"] ** 2
    L = cfg["layers"]
    gemm = 2 * N * K0 * d + L * 2 * N * d * (3 * d + d + 2 * m)
    return 2 * gemm + L * (4 + 10) * N * N * d


def tower_flops(cfg: dict, N: int) -> dict:
    """Algorithmic FLOPs of one image: 2MNK per GEMM, 4 N^2 d for attention."""
    d, m, P, Po = cfg["hidden"], cfg["mlp"], cfg["proj_hidden"], cfg["proj_out"]
    K0 = 3 * cfg["temporal_patch"] * cfg["patch"] ** 2
    L = cfg["layers"]
    gemm = 2 * N * K0 * d + L * 2 * N * d * (3 * d + d + 2 * m) + 2 * N * (d * P + P * P) + \
        2 * (N // 4) * (4 * P * P + P * Po)
    attn = L * 4 * N * N * d
    return dict(gemm=gemm, attn=attn, total=gemm + attn)


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples during the timed region (start before, stop after)."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict | None:
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append(dict(sm=float(f[1]), max=float(f[2]), power=float(f[3]),
                                 hw=f[5], hwt=f[6], swt=f[7], pcap=f[8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        loaded = [r for r in rows if r["power"] > 200] or rows
        reasons = set()
        for r in loaded:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded), "sm_max_mhz": max(r["max"] for r in rows),
                "samples": len(loaded), "reasons": sorted(reasons)}


# -------------------------------------------------------------- CPU oracle

_ORACLE_WEIGHTS: dict = {}


def oracle_threads() -> int:
    """Threads the oracle's numpy arithmetic runs on: the largest BLAS pool numpy has
    loaded (its matrix products dominate), else the host's logical CPUs."""
    try:
        from threadpoolctl import threadpool_info
        n = [p.get("num_threads") or 0 for p in threadpool_info() if p.get("user_api") == "blas"]
        if n and max(n) > 0:
            return int(max(n))
    except Exception:  # threadpoolctl missing or unable to inspect: fall back
        pass
    return os.cpu_count() or 1


def cpu_model() -> str:
    """The host CPU's model name (first entry of /proc/cpuinfo), or the platform's."""
    try:
        for line in open("/proc/cpuinfo"):
            if line.lower().startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or platform.machine()


def oracle_images_per_s(cfg: dict, budget_s: float = 15.0) -> dict:
    """Times the fp64 oracle on one image: patch embedding, as many layers as fit in the
    budget (at least one), and the projector; extrapolates to all layers.  The weights
    (4 layers and the projector) are generated once per configuration, outside the
    timed part."""
    from oracle import vit_ref as R
    key = json.dumps(cfg, sort_keys=True, default=str)
    if key not in _ORACLE_WEIGHTS:
        _ORACLE_WEIGHTS[key] = S.weights_f64(S.make_weights(cfg, layers=min(cfg["layers"], 4)))
    w = _ORACLE_WEIGHTS[key]
    px = S.make_pixels(cfg, batch=1)[0].astype(np.float64)
    t, gh, gw = S.token_grid(cfg)
    pos = R.positions_raster(t, gh, gw)
    t_sample = time.perf_counter()
    t0 = time.perf_counter()
    x = R.patch_embed(R.patch_unfold(px, cfg["patch"], cfg["temporal_patch"]), w["embeddings.proj.weight"],
                      w["embeddings.proj.bias"])
    t_embed = time.perf_counter() - t0
    layer_times = []
    start = time.perf_counter()
    i = 0
    while i < 4 and (i == 0 or time.perf_counter() - start < budget_s * 0.7):
        t0 = time.perf_counter()
        x = R.tower_layer(x, w, i, cfg, pos)
        layer_times.append(time.perf_counter() - t0)
        i += 1
    t0 = time.perf_counter()
    R.projector(x, w, cfg, t, gh, gw)
    t_proj = time.perf_counter() - t0
    per_image = t_embed + cfg["layers"] * statistics.mean(layer_times) + t_proj
    return dict(value=1.0 / per_image, unit="images/s", cores=oracle_threads(), cpu_model=cpu_model(), kind="oracle",
                timed_s=time.perf_counter() - t_sample,
                sample=f"one {cfg['image'][0]}x{cfg['image'][1]} image: patch embedding, {len(layer_times)} of "
                       f"{cfg['layers']} layers (mean layer time x {cfg['layers']}), projector; numpy float64",
                seconds=per_image)


def oracle_attention(wl: dict, budget_s: float = 15.0) -> dict:
    from oracle import vit_ref as R
    H, D, N = wl["heads"], wl["D"], wl["tokens"]
    rng = np.random.default_rng(3)
    q, k, v = (rng.standard_normal((H, N, D)) for _ in range(3))
    rows = np.arange(min(N, 256))
    t0 = time.perf_counter()
    n_heads = 0
    while n_heads < H and (n_heads == 0 or time.perf_counter() - t0 < budget_s):
        R.attention(q[n_heads:n_heads + 1], k[n_heads:n_heads + 1], v[n_heads:n_heads + 1], D ** -0.5, rows=rows)
        n_heads += 1
    dt = time.perf_counter() - t0
    per_call = dt / (n_heads * len(rows)) * N * H
    return dict(value=1.0 / per_call, unit="calls/s", cores=oracle_threads(), cpu_model=cpu_model(), kind="oracle",
                timed_s=dt,
                sample=f"{len(rows)} query rows x {n_heads} heads of the {N}-token attention, scaled to all rows "
                       f"and {H} heads", seconds=per_call)


# --------------------------------------------------------------- reference

def run_reference(args, wl):
    rank, _, _ = REP.rank_env()
    if rank != 0:
        return
    if wl["kind"] not in ("tower", "attn"):
        print(json.dumps(dict(impl="reference", unavailable=f"the oracle arm times the tower<side> and attn<N> "
                                                            f"workloads only, not {wl['kind']}")), flush=True)
        return

    def one_step():
        budget = args.ref_budget / max(args.steps, 1)
        return oracle_images_per_s(wl["cfg"], budget_s=budget) if wl["kind"] == "tower" else \
            oracle_attention(wl, budget_s=budget)

    for _ in range(args.warmup):  # untimed, each the same bounded sample as a timed step
        one_step()
    steps = [one_step() for _ in range(args.steps)]
    value = statistics.mean(s["value"] for s in steps)
    unit = steps[0]["unit"]
    line = dict(metric=METRIC, value=value, unit=unit, n_gpus=args.gpus, steps=args.steps, warmup=args.warmup,
                ms_per_step=1000.0 * statistics.mean(s["seconds"] for s in steps) *
                (wl["batch"] if wl["kind"] == "tower" else 1),
                higher_is_better=True, scaling="weak", vs_baseline=None, dtype="f64", data="synthetic",
                impl="reference",
                config=dict(workload=wl["name"], description=wl["desc"], global_batch=wl["batch"],
                            tokens_per_image=wl["tokens"]),
                cpu_baseline=dict(value=value, unit=unit, cores=steps[0]["cores"], cpu_model=steps[0]["cpu_model"],
                                  kind="oracle", sample=steps[0]["sample"]),
                # each step times a bounded sample and scales it to the whole workload:
                # ms_per_step is that extrapolation, timed_seconds what was actually timed
                extrapolated=True, timed_seconds=sum(s["timed_s"] for s in steps),
                e2e=dict(value=value, unit=unit, h2d_bytes_per_step=0, d2h_bytes_per_step=0))
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm

def _best_ms(torch, fn, stream, reps: int = 20, trials: int = 3) -> float:
    """Best of `trials` event-timed batches of `reps` back-to-back calls (warm L2), ms per call."""
    for _ in range(3):
        fn()
    best = float("inf")
    for _ in range(trials):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        best = min(best, a.elapsed_time(b) / reps)
    return best


def comparators(V, wl, dev, stream) -> dict:
    """Context only, never on the product path: the library's own kernels (vt_linear,
    vt_attention) against torch's on the same shapes, timed the same way (warm L2,
    back-to-back calls, best of three batches) after the benchmark's timed region.
    torch's linear is cuBLAS(Lt) with its bias epilogue; its attention is
    scaled_dot_product_attention on the flash and cuDNN backends, each where torch
    offers it for these shapes."""
    import torch
    import torch.nn.functional as F
    g = torch.Generator(device=dev).manual_seed(11)
    rows = []

    def rnd(*shape, scale=1.0):
        return (torch.randn(*shape, generator=g, device=dev, dtype=torch.float32) * scale).to(torch.bfloat16)

    def row(name, flops, ours, theirs: dict):
        t_o = _best_ms(torch, ours, stream)
        r = dict(op=name, ours_tflops=flops / t_o / 1e9, ours_us=1000 * t_o)
        for k, fn in theirs.items():
            try:
                t = _best_ms(torch, fn, stream)
                r[f"{k}_tflops"], r[f"{k}_us"] = flops / t / 1e9, 1000 * t
            except Exception as e:  # a backend torch does not offer for this shape
                r[f"{k}_tflops"], r[f"{k}_error"] = None, str(e).splitlines()[0][:120]
        rows.append(r)

    if wl["kind"] in ("tower", "varlen", "u8", "video", "backward"):
        cfg = wl["cfg"]
        d, m, P = cfg["hidden"], cfg["mlp"], cfg["proj_hidden"]
        M = wl["batch"] * wl["tokens"] if wl["kind"] != "varlen" else wl["tokens"]
        shapes = [("qkv", M, 3 * d, d, 0), ("o_proj", M, d, d, 0), ("fc1", M, m, d, 0), ("fc2", M, d, m, 0),
                  ("fc1+gelu_tanh", M, m, d, 1), ("proj_patch_fc2", M, P, P, 0),
                  ("proj_merge_fc1", M // 4, P, 4 * P, 0)]
        for name, Mr, Nr, Kr, act in shapes:
            A, W, bias = rnd(Mr, Kr), rnd(Nr, Kr, scale=0.02), rnd(Nr, scale=0.02)
            out = torch.empty((Mr, Nr), dtype=torch.bfloat16, device=dev)
            ours = (lambda A=A, W=W, bias=bias, out=out, Mr=Mr, Nr=Nr, Kr=Kr, act=act:
                    V.vt_linear(A, W, bias, None, out, Mr, Nr, Kr, act, stream))
            lib = ((lambda A=A, W=W, bias=bias: F.gelu(F.linear(A, W, bias), approximate="tanh")) if act else
                   (lambda A=A, W=W, bias=bias: F.linear(A, W, bias)))
            row(f"{name} [{Mr}x{Kr}]x[{Kr}x{Nr}]", 2.0 * Mr * Nr * Kr, ours,
                {"torch_cublas" + ("_plus_gelu_kernel" if act else ""): lib})
            del A, W, bias, out
    B = wl["batch"] if wl["kind"] not in ("attn", "varlen") else 1
    N = wl["tokens"] if wl["kind"] != "varlen" else 1024
    H, D = 16, 80
    q, k, v = rnd(B, H, N, D), rnd(B, H, N, D), rnd(B, H, N, D)
    o = torch.empty((B, N, H * D), dtype=torch.bfloat16, device=dev)
    wsb = V.vt_attention_workspace_bytes(B, H, N, D)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    from torch.nn.attention import SDPBackend, sdpa_kernel

    def sdpa(backend):
        def fn():
            with sdpa_kernel(backend):
                F.scaled_dot_product_attention(q, k, v, scale=D ** -0.5)
        return fn

    # ours: the kernel on operands in its layout (as the tower's QKV epilogue leaves
    # them: v transposed); "ours_with_prep" adds vt_attention's preparation pass.
    ld_vt = (N + 7) // 8 * 8  # the kernel's row pitch of v^T: a multiple of 8
    vt = torch.zeros((B, H, D, ld_vt), dtype=torch.bfloat16, device=dev)
    vt[..., :N] = v.transpose(-1, -2)
    row(f"attention non-causal B={B} H={H} N={N} D={D}", 4.0 * B * H * N * N * D,
        lambda: V.vt_attention_prepared(q, k, vt, ld_vt, o, B, H, N, D, D ** -0.5, stream),
        {"ours_with_prep": lambda: V.vt_attention(q, k, v, o, B, H, N, D, None, None, 10000.0, D ** -0.5, ws, wsb,
                                                  stream),
         "torch_sdpa_flash": sdpa(SDPBackend.FLASH_ATTENTION), "torch_sdpa_cudnn": sdpa(SDPBackend.CUDNN_ATTENTION)})
    return dict(method="warm L2, 20 back-to-back calls, best of 3 event-timed batches; context only",
                torch=torch.__version__, rows=rows)


def setup_step(wl, V, torch, dev, rank):
    """Synthetic inputs and buffers of one step of workload `wl` on this rank, and the
    launch of that step on a given stream.  Returns every local of the set-up (the
    end-to-end leg reuses the host buffers)."""
    import types
    B = wl["batch"]
    grid = wl.get("grid")
    N = wl["tokens"]
    extra_cfg = {}  # workload-specific config entries of the JSON line
    if wl["kind"] == "tower":
        cfg = wl["cfg"]
        tower = V.Tower(cfg, S.make_weights(cfg))
        px_host = torch.from_numpy(S.make_pixels(cfg, batch=B, seed=REP.replica_seed(cfg["seed"], rank))).pin_memory()
        px = px_host.to(dev)
        ws = tower.workspace(B, grid)
        out = torch.empty((B, N // 4, cfg["proj_out"]), dtype=torch.bfloat16, device=dev)

        def launch(s_):
            V.vt_forward(tower.h, px, grid, B, out, None, ws, ws.numel(), s_)

        flops = tower_flops(cfg, N)
        step_flops = B * flops["total"]
        units_per_step = B
        unit = "images/s"
    elif wl["kind"] == "varlen":
        cfg = wl["cfg"]
        tower = V.Tower(cfg, S.make_weights(cfg))
        pix = [S.make_pixels(dict(cfg, image=hw), batch=1, seed=REP.replica_seed(cfg["seed"], rank) + i)[0]
               for i, hw in enumerate(wl["images"])]
        px_host = torch.from_numpy(np.concatenate([a.ravel() for a in pix])).pin_memory()
        px = px_host.to(dev)
        grids = wl["grids"]
        ws_bytes = V.vt_workspace_bytes_varlen(tower.h, grids)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        out = torch.empty((N // 4, cfg["proj_out"]), dtype=torch.bfloat16, device=dev)

        def launch(s_):
            V.vt_forward_varlen(tower.h, px, grids, out, None, ws, ws_bytes, s_)

        step_flops = sum(tower_flops(cfg, g[1] * g[2])["total"] for g in grids)
        units_per_step = B
        unit = "images/s"
    elif wl["kind"] == "backward":
        cfg = wl["cfg"]
        tower = V.Tower(cfg, S.make_weights(cfg))
        V.vt_enable_backward(tower.h)
        px = torch.from_numpy(S.make_pixels(cfg, batch=B, seed=REP.replica_seed(cfg["seed"], rank))).to(dev)
        d_tower = torch.from_numpy(S.make_matrix((B, N, cfg["hidden"]), 9).view(np.int16)).view(
            torch.bfloat16).to(dev)
        saved_bytes, ws_bytes = V.vt_backward_bytes(tower.h, B, grid)
        saved = torch.empty(saved_bytes, dtype=torch.uint8, device=dev)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        tower_out = torch.empty((B, N, cfg["hidden"]), dtype=torch.bfloat16, device=dev)
        d_px = torch.empty_like(px)

        def launch(s_):
            V.vt_forward_saved(tower.h, px, grid, B, tower_out, saved, saved_bytes, ws, ws_bytes, s_)
            V.vt_backward(tower.h, saved, grid, B, d_tower, d_px, ws, ws_bytes, s_)

        step_flops = B * backward_flops(cfg, N)
        units_per_step = B
        unit = "images/s"
    elif wl["kind"] == "u8":
        cfg = wl["cfg"]
        tower = V.Tower(cfg, S.make_weights(cfg))
        images = S.make_images_u8(wl["sizes"], seed=REP.replica_seed(cfg["seed"], rank))
        img_host = torch.from_numpy(np.concatenate([im.ravel() for im in images])).pin_memory()
        img = img_host.to(dev)
        sizes = wl["sizes"]
        ws = tower.workspace(B, grid)
        out = torch.empty((B, N // 4, cfg["proj_out"]), dtype=torch.bfloat16, device=dev)

        def launch(s_):
            V.vt_forward_u8(tower.h, img, sizes, grid, out, None, ws, ws.numel(), stream=s_)

        step_flops = B * tower_flops(cfg, N)["total"]
        units_per_step = B
        unit = "images/s"
    elif wl["kind"] == "video":
        cfg = wl["cfg"]
        tower = V.Tower(cfg, S.make_weights(cfg))
        F = wl["frames"]
        px = torch.from_numpy(S.make_clips(cfg, F, batch=B, seed=REP.replica_seed(cfg["seed"], rank))).to(dev)
        ws = tower.workspace(B, grid)
        out = torch.empty((B, N // 4, cfg["proj_out"]), dtype=torch.bfloat16, device=dev)

        def launch(s_):
            V.vt_forward_video(tower.h, px, F, grid, B, out, None, ws, ws.numel(), s_)

        step_flops = B * tower_flops(cfg, N)["total"]
        units_per_step = B
        unit = "clips/s"
    elif wl["kind"] == "attn_bwd":
        H, D = wl["heads"], wl["D"]
        q, k, v = (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
                   for a in S.make_qkv(B, H, N, D, 3))
        dO = torch.from_numpy(S.make_matrix((B * N, H * D), 4).view(np.int16)).view(torch.bfloat16).to(dev)
        dqkv = torch.empty((B * N, 3 * H * D), dtype=torch.bfloat16, device=dev)
        ws_bytes = V.vt_attention_backward_workspace_bytes(B, H, N, D)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)

        def launch(s_):
            V.vt_attention_backward(q, k, v, dO, dqkv, B, H, N, D, D ** -0.5, ws, ws_bytes, s_)

        step_flops = 10.0 * B * H * N * N * D
        units_per_step = 1
        unit = "calls/s"
    else:
        H, D = wl["heads"], wl["D"]
        q, k, v = (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
                   for a in S.make_qkv(1, H, N, D, 3))
        pos = torch.from_numpy(
            np.stack(np.meshgrid(np.zeros(1), np.arange(grid[1]), np.arange(grid[2]), indexing="ij"), -1)
            .reshape(-1, 3).astype(np.int32)).to(dev)
        o = torch.empty((1, N, H * D), dtype=torch.bfloat16, device=dev)
        ws_bytes = V.vt_attention_workspace_bytes(1, H, N, D)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        # scratch of this call (linear in N) beside the f32 scores + bf16 probabilities
        # an untiled attention keeps per head: 6 N^2 bytes
        extra_cfg = dict(workspace_bytes=int(ws_bytes), untiled_score_buffers_bytes=6 * N * N)

        def launch(s_):
            V.vt_attention(q, k, v, o, 1, H, N, D, pos, (16, 32, 32), 10000.0, D ** -0.5, ws, ws_bytes, s_)

        step_flops = 4.0 * H * N * N * D
        units_per_step = 1
        unit = "calls/s"
    return types.SimpleNamespace(**locals())

def time_steps(args, ctx, V, torch, dist, dev, stream, world, local, steps, warmup, profile_steps):
    """Warm-up, optional CUDA graph of one step, then `steps` timed steps (CUDA events on
    the launching stream, L2 flushed between steps outside the events, clocks sampled,
    maximum over ranks), then `profile_steps` steps with every launch bracketed by
    events for the per-kernel-class times."""
    import types
    launch = ctx.launch

    def step():
        launch(stream)

    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)

    # warm-up (also compiles nothing: the library is prebuilt; first calls set kernel attributes)
    for _ in range(max(warmup, 3)):
        step()
    V.vt_check(stream)

    # optional CUDA graph of one step
    graph = None
    if not args.no_graph:
        try:
            g = torch.cuda.CUDAGraph()
            s2 = torch.cuda.Stream()
            s2.wait_stream(stream)
            with torch.cuda.stream(s2):
                with torch.cuda.graph(g, stream=s2):
                    launch(s2)
            stream.wait_stream(s2)
            g.replay()
            torch.cuda.synchronize()
            graph = g
        except Exception as e:  # capture is an optimisation; eager launches are the same kernels
            print(f"# graph capture failed, timing eager launches: {e}", file=sys.stderr)
            graph = None

    def timed_step():
        if graph is not None:
            graph.replay()
        else:
            step()

    # ---------------- timed region
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for i in range(steps):
        flush.fill_(i & 0xFF)
        starts[i].record(stream)
        timed_step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    V.vt_check(stream)
    ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
    ms = REP.max_over_ranks(ms, dev)
    ms_per_step = ms / steps
    value = REP.job_throughput(ctx.units_per_step, steps, ms, world)

    # ---------------- per-kernel-class times of one profiled step (events around each launch)
    V.vt_profile_begin(stream)
    for _ in range(profile_steps):
        flush.fill_(1)
        step()
    V.vt_profile_end(stream)
    prof = V.vt_profile_read()
    launches_per_step = sum(v["launches"] for v in prof.values()) / profile_steps
    return types.SimpleNamespace(value=value, ms=ms, ms_per_step=ms_per_step, prof=prof, graph=graph, clk=clk,
                                 launches_per_step=launches_per_step, flush=flush)


def summarize(prof, profile_steps, peaks, peaks_kind, wl_name):
    """Roofline of the dominant kernel class (against the measured burst bf16 peak: the
    kernels run inside steps of milliseconds to a tenth of a second, at burst clocks) and
    the per-class times of the profiled steps."""
    dom = max(("gemm", "attention", "attention_backward"), key=lambda c: prof[c]["ms"])
    p = prof[dom]
    achieved = p["flops"] / (p["ms"] / 1000.0) / 1e12 if p["ms"] > 0 else 0.0
    peak = peaks["bf16_tflops"]
    roofline = dict(bound="tensor", kernel={"gemm": "gemm_bf16_tcgen05 (all linear layers)",
                                            "attention": "attn_fwd_tcgen05",
                                            "attention_backward": "attn_bwd_dq + attn_bwd_dkdv"}[dom],
                    achieved=achieved, peak=peak, unit="TFLOP/s", frac=achieved / peak,
                    peak_source=f"{peaks_kind} bf16 burst",
                    frac_of_sustained=achieved / peaks["bf16_tflops_sustained"],
                    frac_of_nominal=achieved / NOMINAL_BF16_TFLOPS,
                    traffic=recorded_traffic(dom, {"tower448": "tower448_b8"}.get(wl_name, wl_name)),
                    traffic_unit="bytes per launch (ncu dram read + write)",
                    per_launch_flops=p["flops"] / max(p["launches"], 1),
                    avg_launch_us=1000.0 * p["ms"] / max(p["launches"], 1))
    classes = {k: dict(ms_per_step=v["ms"] / profile_steps,
                       launches_per_step=v["launches"] / profile_steps,
                       tflops=(v["flops"] / (v["ms"] / 1000.0) / 1e12) if v["ms"] > 0 and v["flops"] else None,
                       gbs=(v["bytes"] / (v["ms"] / 1000.0) / 1e9) if v["ms"] > 0 and v["bytes"] and
                       not v["flops"] else None)
               for k, v in prof.items() if v["launches"]}
    return roofline, classes


def run_gpu(args, wl):
    import torch
    import torch.distributed as dist

    rank, world, local = REP.rank_env()
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    from vision_transformer_encoder_vit_b200 import vt as V

    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    peaks, peaks_kind = load_peaks()
    ctx = setup_step(wl, V, torch, dev, rank)
    B, grid, N, unit = ctx.B, ctx.grid, ctx.N, ctx.unit
    tm = time_steps(args, ctx, V, torch, dist, dev, stream, world, local, args.steps, args.warmup,
                    args.profile_steps)
    value, ms, ms_per_step, prof, graph, clk = tm.value, tm.ms, tm.ms_per_step, tm.prof, tm.graph, tm.clk
    launches_per_step = tm.launches_per_step
    flush = tm.flush


    # ---------------- end to end through the C ABI with host buffers
    e2e = None
    # ---------------- end to end through the C ABI with host buffers
    e2e = None
    if wl["kind"] == "tower":
        # A serving pipeline: batches alternate between two streams, each with its own
        # workspace and pinned output, so one batch's copies overlap the other's forward.
        # Every step still copies its pixels in and its projected tokens out.
        wsb_h = V.vt_forward_host_workspace_bytes(ctx.tower.h, B, grid)
        ws_h = [torch.empty(wsb_h, dtype=torch.uint8, device=dev) for _ in range(2)]
        out_h = [torch.empty((B, N // 4, ctx.cfg["proj_out"]), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        streams = [stream, torch.cuda.Stream(device=dev)]
        for i in range(2):
            V.vt_forward_host(ctx.tower.h, ctx.px_host, grid, B, out_h[i], ws_h[i], wsb_h, streams[i])
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e_s = torch.cuda.Event(enable_timing=True)
        e_e = torch.cuda.Event(enable_timing=True)
        e_s.record(stream)
        streams[1].wait_event(e_s)
        for i in range(args.steps):
            V.vt_forward_host_async(ctx.tower.h, ctx.px_host, grid, B, out_h[i % 2], ws_h[i % 2], wsb_h, streams[i % 2])
        stream.wait_stream(streams[1])
        e_e.record(stream)
        torch.cuda.synchronize()
        e2e_ms = e_s.elapsed_time(e_e)
        e2e_ms = REP.max_over_ranks(e2e_ms, dev)
        e2e = dict(value=REP.job_throughput(B, args.steps, e2e_ms, world), unit=unit,
                   h2d_bytes_per_step=int(ctx.px_host.numel() * 4), d2h_bytes_per_step=int(out_h[0].numel() * 2),
                   api="vt_forward_host_async, two streams")
        del ws_h
    elif wl["kind"] == "u8":
        # decoded images from pinned host memory -> device, forward, projected tokens back;
        # batches alternate between two streams with their own buffers (serving pipeline)
        streams = [stream, torch.cuda.Stream(device=dev)]
        bufs = [(ctx.img, ctx.ws, ctx.out),
                (torch.empty_like(ctx.img), torch.empty_like(ctx.ws), torch.empty_like(ctx.out))]
        out_h = [torch.empty((B, N // 4, ctx.cfg["proj_out"]), dtype=torch.bfloat16).pin_memory() for _ in range(2)]

        def e2e_step(i):
            im, w_, o_ = bufs[i % 2]
            with torch.cuda.stream(streams[i % 2]):
                im.copy_(ctx.img_host, non_blocking=True)
                V.vt_forward_u8(ctx.tower.h, im, ctx.sizes, grid, o_, None, w_, w_.numel(), stream=streams[i % 2])
                out_h[i % 2].copy_(o_, non_blocking=True)

        e2e_step(0)
        e2e_step(1)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e_s = torch.cuda.Event(enable_timing=True)
        e_e = torch.cuda.Event(enable_timing=True)
        e_s.record(stream)
        streams[1].wait_event(e_s)
        for i in range(args.steps):
            e2e_step(i)
        stream.wait_stream(streams[1])
        e_e.record(stream)
        torch.cuda.synchronize()
        e2e_ms = REP.max_over_ranks(e_s.elapsed_time(e_e), dev)
        e2e = dict(value=REP.job_throughput(B, args.steps, e2e_ms, world), unit=unit,
                   h2d_bytes_per_step=int(ctx.img_host.numel()), d2h_bytes_per_step=int(out_h[0].numel() * 2),
                   api="vt_forward_u8 (+ host copies), two streams")

    # The second headline configuration: one 2016x2016 image (20736 tokens) through the
    # same path, timed the same way after the main workload (its buffers released).
    secondary = None
    if wl["name"] == "tower448" and args.secondary_steps > 0:
        wl2 = workload("tower2016")
        ctx2 = setup_step(wl2, V, torch, dev, rank)
        tm2 = time_steps(args, ctx2, V, torch, dist, dev, stream, world, local, args.secondary_steps, 3, 1)
        if rank == 0:
            roof2, classes2 = summarize(tm2.prof, 1, peaks, peaks_kind, wl2["name"])
            secondary = dict(workload=wl2["name"], description=wl2["desc"], value=tm2.value, unit=ctx2.unit,
                             steps=args.secondary_steps, warmup=3, ms_per_step=tm2.ms_per_step,
                             tokens_per_s=tm2.value * wl2["tokens"], output_tokens_per_s=tm2.value * wl2["tokens"] / 4,
                             tflops=world * ctx2.step_flops * args.secondary_steps / (tm2.ms / 1000.0) / 1e12,
                             launch="cuda graph" if tm2.graph else "eager", roofline=roof2, kernel_classes=classes2,
                             clocks=tm2.clk)
        del ctx2, tm2

    comp = comparators(V, wl, dev, stream) if args.comparators and rank == 0 else None

    if rank == 0:
        roofline, classes = summarize(prof, args.profile_steps, peaks, peaks_kind, wl["name"])
        cpu = None
        if world == 1 and not args.no_cpu_baseline and wl["kind"] in ("tower", "attn"):
            cpu = (oracle_images_per_s(ctx.cfg, args.cpu_budget) if wl["kind"] == "tower"
                   else oracle_attention(wl, args.cpu_budget))
            cpu = {k: cpu[k] for k in ("value", "unit", "cores", "cpu_model", "kind", "sample")}
        # tokens of one image (clip); a packed varlen batch reports its mean image
        per_unit = N / B if wl["kind"] == "varlen" else N
        line = dict(
            metric=METRIC, value=value, unit=unit, n_gpus=world, steps=args.steps, warmup=max(args.warmup, 3),
            ms_per_step=ms_per_step, higher_is_better=True, scaling="weak", vs_baseline=None, dtype="bf16",
            data="synthetic: seeded N(0,0.02) bf16 weights, U[0,1] ImageNet-normalised pixels",
            config=dict(workload=wl["name"], description=wl["desc"], per_gpu_batch=B, global_batch=B * world,
                        tokens_per_image=per_unit, merged_tokens_per_image=per_unit / 4,
                        l2="flushed (512 MB write) between timed steps", launch="cuda graph" if graph else "eager",
                        parallelism=f"replicas x{world}", **ctx.extra_cfg),
            tokens_per_s=value * per_unit if wl["kind"] not in ("attn", "attn_bwd") else None,
            output_tokens_per_s=value * per_unit / 4 if wl["kind"] not in ("attn", "attn_bwd") else None,
            tflops=world * ctx.step_flops * args.steps / (ms / 1000.0) / 1e12,
            roofline=roofline, kernel_classes=classes,
            cpu_baseline=cpu, e2e=e2e,
            gpu_launches=int(round(launches_per_step * args.steps)),
            clocks=clk,
        )
        if secondary is not None:
            line["secondary"] = secondary
        if comp is not None:
            line["comparators"] = comp
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="tower448")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-steps", type=int, default=2)
    ap.add_argument("--secondary-steps", type=int, default=5,
                    help="timed steps of the 2016x2016 configuration measured after tower448 (0: skip)")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--ref-budget", type=float, default=60.0)
    ap.add_argument("--comparators", action="store_true",
                    help="also time torch's cuBLAS linear and SDPA on the same shapes (context only)")
    args = ap.parse_args()
    wl = workload(args.workload)
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_gpu(args, wl)


if __name__ == "__main__":
    main()

"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds input generation only: the workload shapes, seeded random draws,
fp32 -> bf16 rounding of the draws and pixel normalisation.  It holds none of the
tower's arithmetic, and it imports neither the CUDA library nor the oracle.

Every tensor is drawn from ``numpy.random.default_rng(seed)`` in a fixed order
(``weight_names``), as float32, then rounded to bf16 with round-to-nearest-even.
The bf16 bit patterns (``uint16``) go to the GPU; their exact float64 values go to
the oracle, so both sides start from identical numbers.
"""
from __future__ import annotations

import copy

import numpy as np

# ImageNet channel statistics, used only to turn U[0,1] pixels into the normalised
# values the tower consumes.
IMAGENET_MEAN = (0.485, 0.456, 0.406)
IMAGENET_STD = (0.229, 0.224, 0.225)
# OpenAI CLIP image statistics (the "OpenAI CLIP mean/std" the preprocessing names).
CLIP_MEAN = (0.48145466, 0.4578275, 0.40821073)
CLIP_STD = (0.26862954, 0.26130258, 0.27577711)

_TOWER_BASE = dict(
    patch=14, temporal_patch=2, merge=2, rope_theta=10000.0, ln_eps=1e-6,
    gelu_tanh=True, proj_gelu_tanh=True, use_rope=True,
)

# Workloads.  Dimensions follow the MiniMax-M3 Vision model card (Architecture
# table: 32 layers, hidden 1280, 16 heads, MLP 5120, patch 14, Conv3d embed with
# temporal patch 2, 2x2 merge, projector 1280 -> 6144 -> 6144, 4 x 6144 -> 6144 -> 6144).
CONFIGS = {
    # Tiny tower: 2 layers, hidden 128, 4 heads of 32, 112x112 image -> 8x8 tokens.
    "tiny": dict(_TOWER_BASE, layers=2, hidden=128, heads=4, head_dim=32, mlp=512,
                 rope_sections=(8, 12, 12), proj_hidden=256, proj_out=256,
                 image=(112, 112), batch=1, seed=0),
    # One full-width tower layer on a 448x448 token grid (32x32 = 1024 tokens).
    "layer1280": dict(_TOWER_BASE, layers=1, hidden=1280, heads=16, head_dim=80,
                      mlp=5120, rope_sections=(16, 32, 32), proj_hidden=6144,
                      proj_out=6144, image=(448, 448), batch=1, seed=1),
    # Full tower + merge + projector, 8 images of 448x448.
    "tower448": dict(_TOWER_BASE, layers=32, hidden=1280, heads=16, head_dim=80,
                     mlp=5120, rope_sections=(16, 32, 32), proj_hidden=6144,
                     proj_out=6144, image=(448, 448), batch=8, seed=2),
    # Full tower + merge + projector, one 2016x2016 image (144x144 = 20736 tokens).
    "tower2016": dict(_TOWER_BASE, layers=32, hidden=1280, heads=16, head_dim=80,
                      mlp=5120, rope_sections=(16, 32, 32), proj_hidden=6144,
                      proj_out=6144, image=(2016, 2016), batch=1, seed=4),
}

# Attention-only sweep: 16 heads of 80, token grids 80x80, 128x128, 256x256.
ATTN_SWEEP = dict(heads=16, head_dim=80, grids=((80, 80), (128, 128), (256, 256)),
                  rope_sections=(16, 32, 32), rope_theta=10000.0, seed=3)


def get_config(name: str, **overrides) -> dict:
    cfg = copy.deepcopy(CONFIGS[name])
    cfg.update(overrides)
    return cfg


def token_grid(cfg: dict) -> tuple[int, int, int]:
    """(t, h, w) patch grid of one image of the workload."""
    H, W = cfg["image"]
    return 1, H // cfg["patch"], W // cfg["patch"]


# --------------------------------------------------------------------------- bf16

def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even); return uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + rounding) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact float64 value of bf16 bit patterns."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32)


# ------------------------------------------------------------------------ weights

def weight_names(cfg: dict) -> list[tuple[str, tuple[int, ...], str]]:
    """Tensor names, shapes and init kinds in draw order.

    Kinds: 'w' linear/conv weight, 'b' bias, 'g' LayerNorm scale, 'beta' LayerNorm shift.
    Linear weights are [out, in] (PyTorch convention); the patch embedding is the
    Conv3d weight [hidden, 3, temporal_patch, patch, patch].
    """
    d, m = cfg["hidden"], cfg["mlp"]
    p, tp = cfg["patch"], cfg["temporal_patch"]
    P, Po = cfg["proj_hidden"], cfg["proj_out"]
    mm = cfg["merge"] * cfg["merge"]
    out = [("embeddings.proj.weight", (d, 3, tp, p, p), "w"),
           ("embeddings.proj.bias", (d,), "b")]
    for i in range(cfg["layers"]):
        pre = f"layers.{i}."
        out += [
            (pre + "ln1.weight", (d,), "g"), (pre + "ln1.bias", (d,), "beta"),
            (pre + "attn.qkv.weight", (3 * d, d), "w"), (pre + "attn.qkv.bias", (3 * d,), "b"),
            (pre + "attn.o.weight", (d, d), "w"), (pre + "attn.o.bias", (d,), "b"),
            (pre + "ln2.weight", (d,), "g"), (pre + "ln2.bias", (d,), "beta"),
            (pre + "mlp.fc1.weight", (m, d), "w"), (pre + "mlp.fc1.bias", (m,), "b"),
            (pre + "mlp.fc2.weight", (d, m), "w"), (pre + "mlp.fc2.bias", (d,), "b"),
        ]
    out += [
        ("proj.patch_fc1.weight", (P, d), "w"), ("proj.patch_fc1.bias", (P,), "b"),
        ("proj.patch_fc2.weight", (P, P), "w"), ("proj.patch_fc2.bias", (P,), "b"),
        ("proj.merge_fc1.weight", (P, mm * P), "w"), ("proj.merge_fc1.bias", (P,), "b"),
        ("proj.merge_fc2.weight", (Po, P), "w"), ("proj.merge_fc2.bias", (Po,), "b"),
    ]
    return out


def make_weights(cfg: dict, seed: int | None = None, affine: bool = False,
                 layers: int | None = None) -> dict[str, np.ndarray]:
    """Seeded bf16 weights (uint16 bit arrays), keyed by name.

    Default init: weights N(0, 0.02), biases 0, LayerNorm scale 1 and shift 0.
    ``affine=True`` also draws biases N(0, 0.02), LayerNorm scale 1 + N(0, 0.1) and
    shift N(0, 0.02) from ``seed + 100`` so that the bias and affine paths carry
    non-trivial values.  ``layers`` limits how many tower layers are generated.
    """
    seed = cfg["seed"] if seed is None else seed
    c = dict(cfg)
    if layers is not None:
        c["layers"] = layers
    rng = np.random.default_rng(seed)
    rng_aff = np.random.default_rng(seed + 100)
    out = {}
    for name, shape, kind in weight_names(c):
        if kind == "w":
            v = rng.standard_normal(shape, dtype=np.float32) * np.float32(0.02)
        elif kind == "b":
            v = (rng_aff.standard_normal(shape, dtype=np.float32) * np.float32(0.02)
                 if affine else np.zeros(shape, np.float32))
        elif kind == "g":
            v = (np.float32(1) + rng_aff.standard_normal(shape, dtype=np.float32) * np.float32(0.1)
                 if affine else np.ones(shape, np.float32))
        else:
            v = (rng_aff.standard_normal(shape, dtype=np.float32) * np.float32(0.02)
                 if affine else np.zeros(shape, np.float32))
        out[name] = bf16_bits(v)
    return out


def weights_f64(w_bits: dict[str, np.ndarray]) -> dict[str, np.ndarray]:
    return {k: bf16_to_f64(v) for k, v in w_bits.items()}


# ------------------------------------------------------------------------ inputs

def make_pixels(cfg: dict, batch: int | None = None, seed: int | None = None,
                normalise: bool = True) -> np.ndarray:
    """Pixels U[0,1] as float32 [B, 3, H, W], optionally ImageNet-normalised."""
    seed = cfg["seed"] if seed is None else seed
    B = cfg["batch"] if batch is None else batch
    H, W = cfg["image"]
    rng = np.random.default_rng(seed + 1000)
    x = rng.random((B, 3, H, W), dtype=np.float32)
    if normalise:
        mean = np.asarray(IMAGENET_MEAN, np.float32)[None, :, None, None]
        std = np.asarray(IMAGENET_STD, np.float32)[None, :, None, None]
        x = (x - mean) / std
    return np.ascontiguousarray(x, dtype=np.float32)


def make_images_u8(sizes, seed: int = 0) -> list[np.ndarray]:
    """Decoded RGB images of the given (H, W) sizes as uint8 [H, W, 3]: a smooth random
    field (sum of low-frequency waves) plus uniform noise, clipped to 0..255, so both
    flat areas and edges occur."""
    rng = np.random.default_rng(seed + 2000)
    out = []
    for H, W in sizes:
        y = np.linspace(0.0, 1.0, H)[:, None, None]
        x = np.linspace(0.0, 1.0, W)[None, :, None]
        img = np.full((H, W, 3), 128.0)
        for _ in range(4):
            fy, fx = rng.uniform(0.5, 6.0, size=2)
            ph = rng.uniform(0, 2 * np.pi, size=3)[None, None, :]
            img += rng.uniform(20, 50) * np.sin(2 * np.pi * (fy * y + fx * x) + ph)
        img += rng.uniform(-40, 40, size=(H, W, 3))
        out.append(np.clip(np.rint(img), 0, 255).astype(np.uint8))
    return out


def make_clips(cfg: dict, frames: int, batch: int | None = None, seed: int | None = None) -> np.ndarray:
    """Clips of ``frames`` ImageNet-normalised U[0,1] frames, float32 [B, F, 3, H, W];
    the frames are independent draws (no motion model: every frame differs)."""
    seed = cfg["seed"] if seed is None else seed
    B = cfg["batch"] if batch is None else batch
    flat = make_pixels(cfg, batch=B * frames, seed=seed)
    return np.ascontiguousarray(flat.reshape(B, frames, *flat.shape[1:]))


def make_activations(rows: int, cols: int, seed: int) -> np.ndarray:
    """bf16 bits of N(0,1) activations [rows, cols]."""
    rng = np.random.default_rng(seed + 2000)
    return bf16_bits(rng.standard_normal((rows, cols), dtype=np.float32))


def make_qkv(B: int, H: int, N: int, D: int, seed: int) -> tuple[np.ndarray, ...]:
    """bf16 bits of N(0,1) q, k, v, each [B, H, N, D]."""
    rng = np.random.default_rng(seed + 3000)
    return tuple(bf16_bits(rng.standard_normal((B, H, N, D), dtype=np.float32))
                 for _ in range(3))


def make_matrix(shape: tuple[int, ...], seed: int, scale: float = 1.0) -> np.ndarray:
    """bf16 bits of N(0, scale^2) entries of the given shape."""
    rng = np.random.default_rng(seed + 4000)
    return bf16_bits(rng.standard_normal(shape, dtype=np.float32) * np.float32(scale))

"""Helpers shared by the GPU parity tests: moving bf16 bit arrays to and from the
device, and the comparison rules.

Tolerances (written here once, used by every parity test):
  * relative L2 error ||g - o||_2 / ||o||_2 <= 1e-2 for a tower layer output and for
    single kernels, <= 2e-2 for the final projected tokens;
  * element-wise |g - o| <= ELEM_RTOL * |o| + ELEM_ATOL * rms(o), a bound a few bf16
    half-ulps wide (bf16 keeps 8 significant bits, so rounding one result costs up to
    2^-9 relative), which catches a single wrong tile that an L2 norm could average away;
  * for outputs that crossed many bf16 layers (free-running towers), where single
    elements drift further than a few half-ulps, a relative L2 gate on every token row
    (assert_rows_close), which still catches a single wrong token or tile.
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch

from vision_transformer_encoder_vit_b200 import synthetic as S

REL_L2_LAYER = 1e-2
REL_L2_FINAL = 2e-2
ELEM_RTOL = 2.0 ** -5
ELEM_ATOL = 2.0 ** -5


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.cuda()


def dev_f32(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def host_f64(t: torch.Tensor) -> np.ndarray:
    torch.cuda.synchronize()
    bits = t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return S.bf16_to_f64(bits)


def host_bits(t: torch.Tensor) -> np.ndarray:
    torch.cuda.synchronize()
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def empty_bf16(*shape) -> torch.Tensor:
    return torch.empty(*shape, dtype=torch.bfloat16, device="cuda")


def rel_l2(g: np.ndarray, o: np.ndarray) -> float:
    g = np.asarray(g, np.float64)
    o = np.asarray(o, np.float64)
    return float(np.linalg.norm((g - o).ravel()) / max(np.linalg.norm(o.ravel()), 1e-300))


def report(what: str, **fields) -> None:
    """Appends one JSON line to $VT_PARITY_REPORT (if set): the measured errors."""
    path = os.environ.get("VT_PARITY_REPORT")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(dict(what=what, **fields)) + "\n")


def assert_close(g, o, rel=REL_L2_LAYER, rtol=ELEM_RTOL, atol=ELEM_ATOL, what=""):
    g = np.asarray(g, np.float64)
    o = np.asarray(o, np.float64)
    assert g.shape == o.shape, f"{what}: shape {g.shape} != {o.shape}"
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    r = rel_l2(g, o)
    rms_o = float(np.sqrt(np.mean(o ** 2))) if o.size else 0.0
    worst = float(np.max(np.abs(g - o) / (rtol * np.abs(o) + atol * rms_o + 1e-300))) if o.size else 0.0
    report(what, rel_l2=r, gate=rel, worst_elem_over_bound=worst)
    assert r <= rel, f"{what}: relative L2 error {r:.3e} > {rel:.1e}"
    rms = float(np.sqrt(np.mean(o ** 2))) if o.size else 0.0
    bound = rtol * np.abs(o) + atol * rms
    bad = np.abs(g - o) > bound
    if bad.any():
        idx = np.unravel_index(np.argmax(np.abs(g - o) - bound), g.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} elements outside the element-wise bound; worst at {idx}: "
                             f"got {g[idx]:.6g}, expected {o[idx]:.6g}")
    return r


def assert_rows_close(g, o, rel, rel_row, what=""):
    """Relative L2 over the whole tensor <= rel and over every row (last axis) <= rel_row;
    reports the worst row."""
    g = np.asarray(g, np.float64)
    o = np.asarray(o, np.float64)
    assert g.shape == o.shape, f"{what}: shape {g.shape} != {o.shape}"
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    r = rel_l2(g, o)
    g2 = g.reshape(-1, g.shape[-1])
    o2 = o.reshape(-1, o.shape[-1])
    per = np.linalg.norm(g2 - o2, axis=1) / np.maximum(np.linalg.norm(o2, axis=1), 1e-300)
    worst = int(np.argmax(per))
    report(what, rel_l2=r, gate=rel, worst_row=worst, worst_row_rel_l2=float(per[worst]), row_gate=rel_row)
    assert r <= rel, f"{what}: relative L2 error {r:.3e} > {rel:.1e}"
    assert per[worst] <= rel_row, f"{what}: row {worst} has relative L2 error {per[worst]:.3e} > {rel_row:.1e}"
    return r

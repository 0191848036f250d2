"""CPU tests of bench.py's host logic: the workload table and the algorithmic FLOP counts
that every reported TFLOP/s and roofline fraction divides by.

The expected totals are derived here from the layer list of the "MiniMax-M3 Vision"
model card (Architecture table), one product at a time, not by calling bench.py's
formula: 2 M N K per linear layer (patch embedding K = 3*2*14*14, QKV 3d, O d, fc1 m,
fc2 from m, projector 1280->6144->6144 per token and 24576->6144->6144 per merged token)
and 4 N^2 d per attention layer."""
import pytest

import bench
from vision_transformer_encoder_vit_b200 import synthetic as S


def _per_image_products(N, d=1280, m=5120, P=6144, layers=32):
    """(M, N_out, K) of every linear layer and the attention FLOPs of one image."""
    prods = [(N, d, 3 * 2 * 14 * 14)]                     # Conv3d patch embedding as a GEMM
    for _ in range(layers):
        prods += [(N, 3 * d, d), (N, d, d), (N, m, d), (N, d, m)]  # QKV, O, fc1, fc2
    prods += [(N, P, d), (N, P, P)]                       # per-token projector
    prods += [(N // 4, P, 4 * P), (N // 4, P, P)]         # merged projector
    gemm = sum(2.0 * a * b * c for a, b, c in prods)
    attn = layers * 4.0 * N * N * d
    return gemm, attn


@pytest.mark.parametrize("name,N", [("tower448", 1024), ("tower2016", 20736)])
def test_tower_flops_match_the_layer_list(name, N):
    cfg = S.get_config(name)
    f = bench.tower_flops(cfg, N)
    gemm, attn = _per_image_products(N)
    assert f["gemm"] == pytest.approx(gemm, rel=1e-12)
    assert f["attn"] == pytest.approx(attn, rel=1e-12)
    assert f["total"] == pytest.approx(gemm + attn, rel=1e-12)


def test_tower_flops_headline_totals():
    # 1.65 TFLOP per 448x448 image (attention about 10% of the 8-image batch's 13.2),
    # 100.45 TFLOP per 2016x2016 image (attention about 70%).
    f448 = bench.tower_flops(S.get_config("tower448"), 1024)
    f2016 = bench.tower_flops(S.get_config("tower2016"), 20736)
    assert f448["total"] / 1e12 == pytest.approx(1.654, abs=0.005)
    assert 8 * f448["total"] / 1e12 == pytest.approx(13.23, abs=0.03)
    assert f448["attn"] / f448["total"] == pytest.approx(0.104, abs=0.005)
    assert f2016["total"] / 1e12 == pytest.approx(100.45, abs=0.05)
    assert f2016["attn"] / f2016["total"] == pytest.approx(0.70, abs=0.01)


def test_backward_flops_count_forward_input_gradients_and_five_attention_products():
    cfg = S.get_config("tower448")
    N, d, L = 1024, 1280, 32
    gemm, _ = _per_image_products(N)
    # the tower only (no projector): patch embedding + 32 layers
    proj = 2.0 * N * (d * 6144 + 6144 * 6144) + 2.0 * (N // 4) * (4 * 6144 * 6144 + 6144 * 6144)
    tower_gemm = gemm - proj
    expect = 2 * tower_gemm + L * (4 + 10) * N * N * d
    assert bench.backward_flops(cfg, N) == pytest.approx(expect, rel=1e-12)


@pytest.mark.parametrize("name,kind,units", [
    ("tower448", "tower", 8), ("tower2016", "tower", 1), ("varlen_mix", "varlen", 8),
    ("backward448", "backward", 8), ("u8_672", "u8", 8), ("video448_f16", "video", 2),
    ("attn65536", "attn", 1), ("attn16384", "attn", 1), ("attnbwd1024", "attn_bwd", 8)])
def test_every_documented_workload_parses(name, kind, units):
    wl = bench.workload(name)
    assert wl["kind"] == kind and wl["name"] == name and wl["batch"] == units
    assert wl["tokens"] > 0 and wl["desc"]


def test_workload_token_counts():
    assert bench.workload("tower448")["tokens"] == 1024
    assert bench.workload("tower2016")["tokens"] == 20736
    assert bench.workload("u8_672")["tokens"] == 48 * 48
    v = bench.workload("video448_f16")
    assert v["grid"] == (8, 32, 32) and v["tokens"] == 8 * 1024
    mix = bench.workload("varlen_mix")
    assert mix["tokens"] == sum((h // 14) * (w // 14) for h, w in mix["images"])
    assert all(h % 28 == 0 and w % 28 == 0 for h, w in mix["images"])
    assert bench.workload("attn65536")["tokens"] == 256 * 256
    with pytest.raises(SystemExit):
        bench.workload("no_such_workload")


def test_cpu_baseline_reports_the_blas_threads():
    import os
    n = bench.oracle_threads()
    assert isinstance(n, int) and 1 <= n <= max(os.cpu_count() or 1, n)
    from threadpoolctl import threadpool_info
    blas = [p["num_threads"] for p in threadpool_info() if p.get("user_api") == "blas"]
    if blas:
        assert n == max(blas)

"""Per-kernel parity on the GPU, through the C ABI, against the fp64 oracle.

Sizes span several tiles and ragged tails; the bookkeeping kernels (patch unfold) are
compared bit for bit.
"""
import math

import numpy as np
import pytest
import torch

from oracle import vit_ref as R
from vision_transformer_encoder_vit_b200 import synthetic as S
from tests.gpu_util import assert_close, dev_bf16, dev_f32, empty_bf16, host_bits, host_f64

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from vision_transformer_encoder_vit_b200 import vt as V


# ------------------------------------------------------------------- GEMM

GEMM_CASES = [
    # M, N, K, bias, resid, act
    (128, 128, 64, False, False, 0),
    (64, 384, 128, True, False, 0),       # M below one tile
    (200, 136, 72, True, True, 0),        # ragged M, N, K
    (1024, 1280, 1280, True, True, 0),    # o-proj shape, 448 x 1 image
    (1000, 5120, 1280, True, False, 1),   # fc1 with GELU (tanh)
    (333, 1280, 5120, True, True, 0),     # fc2 with residual, long K
    (1024, 1280, 1176, True, False, 0),   # patch embedding, K = 1176 (partial K tile)
    (300, 256, 1024, True, False, 2),     # GELU (erf)
    (4096, 6144, 1280, True, False, 1),   # projector patch_fc1, many tiles
    (256, 6144, 24576, True, False, 1),   # projector merge_fc1, K = 24576
]


@pytest.mark.parametrize("M,N,K,use_bias,use_resid,act", GEMM_CASES)
def test_linear_parity(M, N, K, use_bias, use_resid, act):
    seed = M * 7 + N * 3 + K
    A = S.make_matrix((M, K), seed)
    W = S.make_matrix((N, K), seed + 1, scale=0.02 * 50 / math.sqrt(K))
    bias = S.make_matrix((N,), seed + 2, 0.1) if use_bias else None
    resid = S.make_matrix((M, N), seed + 3) if use_resid else None
    out = empty_bf16(M, N)
    dA, dW = dev_bf16(A), dev_bf16(W)
    dB = dev_bf16(bias) if use_bias else None
    dR = dev_bf16(resid) if use_resid else None
    V.vt_linear(dA, dW, dB, dR, out, M, N, K, act)
    V.vt_check()
    ref = S.bf16_to_f64(A) @ S.bf16_to_f64(W).T
    if use_bias:
        ref = ref + S.bf16_to_f64(bias)
    if act:
        ref = R.gelu(ref, tanh_form=(act == 1))
    if use_resid:
        ref = ref + S.bf16_to_f64(resid)
    assert_close(host_f64(out), ref, what=f"linear {M}x{N}x{K}")


# Shapes whose last round of CTA-pair tiles leaves most pairs idle with K >= 2048: the
# product shares out the K steps of those tiles and a second kernel sums the fp32
# partials (vt_linear_ws).  Ragged M, N and K (a partial K step) included.
SPLIT_CASES = [
    # M, N, K, bias, resid, act
    (1100, 1000, 4104, True, True, 0),
    (8192, 1280, 5120, True, True, 0),    # fc2 at 448 x 448 x 8
    (2048, 640, 2048, True, False, 1),    # GELU (tanh)
    (1024, 256, 8192, False, True, 2),    # GELU (erf), one column of tiles, 8 ranges
]


def _expected_split(M, N, K, sms):
    """K ranges per tile the library picks for 256-wide pair tiles (1: no split)."""
    pairs, tiles = sms // 2, -(-M // 256) * -(-N // 256)
    rem, nk = tiles % pairs, -(-K // 64)
    if M < 1024 or rem == 0 or 2 * rem > pairs or nk < 32:
        return 1
    return max(1, min(pairs // rem, nk // 8, 8))


@pytest.mark.parametrize("M,N,K,use_bias,use_resid,act", SPLIT_CASES)
def test_linear_split_k_tail(M, N, K, use_bias, use_resid, act):
    seed = M * 5 + N * 11 + K
    A = S.make_matrix((M, K), seed)
    W = S.make_matrix((N, K), seed + 1, scale=0.02 * 50 / math.sqrt(K))
    bias = S.make_matrix((N,), seed + 2, 0.1) if use_bias else None
    resid = S.make_matrix((M, N), seed + 3) if use_resid else None
    dA, dW = dev_bf16(A), dev_bf16(W)
    dB = dev_bf16(bias) if use_bias else None
    dR = dev_bf16(resid) if use_resid else None
    ws_bytes = V.vt_linear_workspace_bytes()
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    out = empty_bf16(M, N)
    V.vt_profile_begin()
    V.vt_linear_ws(dA, dW, dB, dR, out, M, N, K, act, ws, ws_bytes)
    V.vt_profile_end()
    prof = V.vt_profile_read()
    V.vt_check()
    split = _expected_split(M, N, K, torch.cuda.get_device_properties(0).multi_processor_count)
    assert split > 1, "the case should take the split-K path"
    assert prof["gemm"]["launches"] == 2  # the product and the tail sum
    # rows checked: all of them for small M, else a sample that includes the last tile
    rows = np.arange(M) if M <= 2048 else np.unique(np.concatenate(
        [np.random.default_rng(seed).choice(M, 256, replace=False), np.arange(M - 64, M)]))
    ref = S.bf16_to_f64(A)[rows] @ S.bf16_to_f64(W).T
    if use_bias:
        ref = ref + S.bf16_to_f64(bias)
    if act:
        ref = R.gelu(ref, tanh_form=(act == 1))
    if use_resid:
        ref = ref + S.bf16_to_f64(resid)[rows]
    got = host_f64(out)[rows]
    assert_close(got, ref, what=f"split-K linear {M}x{N}x{K}")
    # the same call again gives the same bits (fixed summation order)
    out2 = empty_bf16(M, N)
    V.vt_linear_ws(dA, dW, dB, dR, out2, M, N, K, act, ws, ws_bytes)
    assert torch.equal(out, out2)


def test_linear_large_a_ragged_column_tiles_fastest():
    # A above 48 MB and larger than W: the CTA pairs walk column tiles fastest.  Ragged M
    # (40 rows in the last 256-row tile), ragged N (232 columns in the last tile), a
    # partial K step; rows checked at a sample that includes the last tile.
    M, N, K = 9000, 1000, 4104
    A = S.make_matrix((M, K), 91)
    W = S.make_matrix((N, K), 92, scale=0.02 * 50 / math.sqrt(K))
    bias, resid = S.make_matrix((N,), 93, 0.1), S.make_matrix((M, N), 94)
    out = empty_bf16(M, N)
    V.vt_linear(dev_bf16(A), dev_bf16(W), dev_bf16(bias), dev_bf16(resid), out, M, N, K, 0)
    V.vt_check()
    rows = np.unique(np.concatenate([np.random.default_rng(95).choice(M, 256, replace=False), np.arange(M - 64, M)]))
    ref = S.bf16_to_f64(A)[rows] @ S.bf16_to_f64(W).T + S.bf16_to_f64(bias) + S.bf16_to_f64(resid)[rows]
    assert_close(host_f64(out)[rows], ref, what=f"linear {M}x{N}x{K}, column tiles fastest")


def test_linear_residual_in_place():
    M, N, K = 384, 512, 256
    A, W = S.make_matrix((M, K), 1), S.make_matrix((N, K), 2, 0.05)
    x = S.make_matrix((M, N), 3)
    dx = dev_bf16(x)
    V.vt_linear(dev_bf16(A), dev_bf16(W), None, dx, dx, M, N, K, 0)
    ref = S.bf16_to_f64(x) + S.bf16_to_f64(A) @ S.bf16_to_f64(W).T
    assert_close(host_f64(dx), ref, what="in-place residual")


def test_linear_rejects_bad_arguments():
    a = empty_bf16(16, 16)
    with pytest.raises(V.VtError) as e:
        V.vt_linear(a, a, None, None, a, 16, 12, 16, 0)
    assert e.value.name == "VT_ERR_INVALID_ARG"


# -------------------------------------------------------------- LayerNorm

@pytest.mark.parametrize("rows,cols", [(1, 1280), (1000, 1280), (77, 128), (50, 384), (9, 1024)])
def test_layernorm_parity(rows, cols):
    x = S.make_matrix((rows, cols), rows + cols, 2.0)
    g = S.make_matrix((cols,), 5, 0.3)
    g = S.bf16_bits(S.bf16_to_f32(g) + np.float32(1.0))
    b = S.make_matrix((cols,), 6, 0.1)
    y = empty_bf16(rows, cols)
    V.vt_layernorm(dev_bf16(x), dev_bf16(g), dev_bf16(b), y, rows, cols, 1e-6)
    ref = R.layer_norm(S.bf16_to_f64(x), S.bf16_to_f64(g), S.bf16_to_f64(b), 1e-6)
    assert_close(host_f64(y), ref, what=f"layernorm {rows}x{cols}")


# ----------------------------------------------------------- patch unfold

@pytest.mark.parametrize("B,H,W", [(1, 112, 112), (2, 56, 84), (1, 448, 448)])
@pytest.mark.parametrize("order", [0, 1])
def test_patch_unfold_is_exact(B, H, W, order):
    cfg = S.get_config("tiny", image=(H, W))
    px = S.make_pixels(cfg, batch=B)
    gh, gw = H // 14, W // 14
    out = empty_bf16(B * gh * gw, 1176)
    V.vt_patch_unfold(dev_f32(px), out, B, H, W, 14, 2, order)
    got = host_bits(out).reshape(B, gh * gw, 1176)
    for b in range(B):
        ref = R.patch_unfold(px[b].astype(np.float64), 14, 2)  # raster order, exact fp32 values
        if order == 1:
            ref = ref[R.block_order(1, gh, gw)]
        np.testing.assert_array_equal(got[b], S.bf16_bits(ref.astype(np.float32)))


# -------------------------------------------------------------- attention

def _attn_case(B, H, N, D, rope, seed, sections=None, grid=None, rows=None, t_axis=False):
    q, k, v = S.make_qkv(B, H, N, D, seed)
    dq, dk, dv = dev_bf16(q), dev_bf16(k), dev_bf16(v)
    o = empty_bf16(B, N, H * D)
    ws_bytes = V.vt_attention_workspace_bytes(B, H, N, D)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    pos = None
    if rope:
        if grid is None:
            pos = np.random.default_rng(seed).integers(0, 200, size=(N, 3)).astype(np.int32)
            if not t_axis:
                pos[:, 0] = 0
        else:
            pos = R.positions_raster(*grid).astype(np.int32)
        dpos = torch.from_numpy(pos).cuda()
    V.vt_attention(dq, dk, dv, o, B, H, N, D, dpos if rope else None, sections, 10000.0, D ** -0.5,
                   ws, ws_bytes)
    V.vt_check()
    got = host_f64(o).reshape(B, N, H, D)
    qf, kf, vf = (S.bf16_to_f64(t) for t in (q, k, v))
    for b in range(B):
        qb, kb = qf[b], kf[b]
        if rope:
            qb = R.apply_rope_3d(qb.transpose(1, 0, 2), pos, sections, 10000.0).transpose(1, 0, 2)
            kb = R.apply_rope_3d(kb.transpose(1, 0, 2), pos, sections, 10000.0).transpose(1, 0, 2)
        ref = R.attention(qb, kb, vf[b], D ** -0.5, rows=rows)
        g = got[b] if rows is None else got[b][rows]
        assert_close(g, ref, what=f"attention B{B} H{H} N{N} D{D} rope={rope} b={b}")


@pytest.mark.parametrize("N", [1, 5, 127, 128, 129, 300, 1024])
def test_attention_d80_ragged(N):
    _attn_case(1, 2, N, 80, False, N)


@pytest.mark.parametrize("N", [64, 200, 2304])
def test_attention_d32(N):
    _attn_case(2, 4, N, 32, True, N + 1, sections=(8, 12, 12))


# The preparation pass of vt_attention has three forms: a plain copy (no RoPE), the
# rotation of 16-byte channel chunks (every section a multiple of 16) and the rotation
# one channel pair at a time (other sections).  Ragged token counts leave a partial
# 32-token tile; positions include the t axis.
@pytest.mark.parametrize("B,H,N,D,sections", [
    (3, 5, 1001, 80, (16, 32, 32)),
    (1, 4, 250, 64, (16, 16, 32)),
    (2, 4, 777, 64, (16, 24, 24)),
    (2, 3, 517, 96, (32, 32, 32)),
    (1, 3, 333, 96, (32, 16, 48)),
    (1, 3, 45, 96, (24, 36, 36)),
    (2, 2, 70, 32, (0, 16, 16)),
    (1, 2, 300, 64, None),
    (1, 2, 301, 96, None),
])
def test_attention_prep_forms(B, H, N, D, sections):
    _attn_case(B, H, N, D, sections is not None, B * N + D, sections=sections, t_axis=True)


def test_attention_rope_raster_grid_448():
    _attn_case(2, 16, 1024, 80, True, 7, sections=(16, 32, 32), grid=(1, 32, 32))


def test_attention_large_values_rescale():
    # scaled-up q makes the running maximum jump between key tiles, exercising the
    # lazy rescale of O.
    B, H, N, D = 1, 2, 700, 80
    q, k, v = S.make_qkv(B, H, N, D, 11)
    q = S.bf16_bits(S.bf16_to_f32(q) * np.float32(6.0))
    k = S.bf16_bits(S.bf16_to_f32(k) * np.linspace(0.2, 3, N, dtype=np.float32)[None, None, :, None])
    o = empty_bf16(B, N, H * D)
    ws_bytes = V.vt_attention_workspace_bytes(B, H, N, D)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    V.vt_attention(dev_bf16(q), dev_bf16(k), dev_bf16(v), o, B, H, N, D, None, None, 0.0, D ** -0.5, ws, ws_bytes)
    ref = R.attention(S.bf16_to_f64(q)[0], S.bf16_to_f64(k)[0], S.bf16_to_f64(v)[0], D ** -0.5)
    assert_close(host_f64(o).reshape(N, H, D), ref, what="attention with rescales")


def test_attention_special_values():
    # V = 1 gives 1 everywhere; identical keys give the mean of V.
    B, H, N, D = 1, 2, 333, 80
    q, k, v = S.make_qkv(B, H, N, D, 12)
    ones = S.bf16_bits(np.ones((B, H, N, D), np.float32))
    o = empty_bf16(B, N, H * D)
    ws_bytes = V.vt_attention_workspace_bytes(B, H, N, D)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    V.vt_attention(dev_bf16(q), dev_bf16(k), dev_bf16(ones), o, B, H, N, D, None, None, 0.0, D ** -0.5, ws, ws_bytes)
    np.testing.assert_allclose(host_f64(o), 1.0, atol=2 ** -7)
    keq = np.broadcast_to(k[:, :, :1], k.shape).copy()
    V.vt_attention(dev_bf16(q), dev_bf16(keq), dev_bf16(v), o, B, H, N, D, None, None, 0.0, D ** -0.5, ws, ws_bytes)
    mean = S.bf16_to_f64(v)[0].mean(axis=1)  # [H, D]
    got = host_f64(o).reshape(N, H, D)
    assert_close(got, np.broadcast_to(mean[None], got.shape), what="equal keys")


@pytest.mark.parametrize("grid", [(1, 80, 80), (1, 128, 128), (1, 256, 256)])
def test_attention_sweep_sampled_rows(grid):
    # Attention-only sweep sizes (6400, 16384, 65536 tokens; 16 heads of 80; RoPE from
    # the (0, h, w) grid); the oracle evaluates a seeded sample of query rows.
    N = grid[1] * grid[2]
    rows = np.sort(np.random.default_rng(N).choice(N, size=96, replace=False))
    rows = np.concatenate([rows, [0, N - 1]])
    _attn_case(1, 16, N, 80, True, 3, sections=(16, 32, 32), grid=grid, rows=rows)


def test_attention_workspace_is_linear_in_tokens():
    sizes = [V.vt_attention_workspace_bytes(1, 16, n, 80) for n in (6400, 16384, 65536)]
    for n, s in zip((6400, 16384, 65536), sizes):
        assert s <= 3 * 16 * 80 * (n + 8) * 2 + 3 * 256
        assert s < 6 * n * n  # the pages' quadratic score + prob buffers

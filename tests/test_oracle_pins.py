"""Pins of the fp64 oracle against things other than itself.

Each test checks one oracle function against brute force, a library routine, a closed
form, an invariant of the mathematics, or a shape fact the pages print
(tests/golden/shape_facts.json).  The set is chosen so that a dropped term, a wrong
sign or index, or a transposed operand in the oracle fails at least one test.
CPU only.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import vit_ref as R
from vision_transformer_encoder_vit_b200 import synthetic as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "shape_facts.json")
torch.set_default_dtype(torch.float64)


def _rng(seed):
    return np.random.default_rng(seed)


# ------------------------------------------------------------------ attention

def _attention_brute(q, k, v, scale):
    """Scalar loops over (query i, key j, channel c) with math.exp; no numpy algebra."""
    H, N, D = q.shape
    Dv = v.shape[2]
    out = np.zeros((N, H, Dv))
    for h in range(H):
        for i in range(N):
            s = []
            for j in range(N):
                acc = 0.0
                for c in range(D):
                    acc += q[h, i, c] * k[h, j, c]
                s.append(acc * scale)
            mx = max(s)
            e = [math.exp(x - mx) for x in s]
            tot = sum(e)
            for c in range(Dv):
                acc = 0.0
                for j in range(N):
                    acc += e[j] / tot * v[h, j, c]
                out[i, h, c] = acc
    return out


@pytest.mark.parametrize("H,N,D", [(1, 1, 4), (2, 7, 5), (3, 17, 8), (1, 64, 6)])
def test_attention_matches_brute_force(H, N, D):
    r = _rng(N * 31 + D)
    q, k, v = (r.standard_normal((H, N, D)) for _ in range(3))
    scale = 1 / math.sqrt(D)
    np.testing.assert_allclose(R.attention(q, k, v, scale), _attention_brute(q, k, v, scale),
                               rtol=0, atol=1e-12)


def test_attention_brute_force_tiny_config_shape():
    # The tiny tower's attention shape: 4 heads of 32 over 64 tokens.
    r = _rng(5)
    q, k, v = (r.standard_normal((4, 64, 32)) * 0.5 for _ in range(3))
    np.testing.assert_allclose(R.attention(q, k, v, 32 ** -0.5),
                               _attention_brute(q, k, v, 32 ** -0.5), atol=1e-12, rtol=0)


def test_attention_matches_torch_sdpa():
    r = _rng(1)
    q, k, v = (r.standard_normal((4, 300, 80)) for _ in range(3))
    ref = F.scaled_dot_product_attention(torch.tensor(q), torch.tensor(k), torch.tensor(v))
    got = R.attention(q, k, v, 80 ** -0.5, row_block=37)
    np.testing.assert_allclose(got.transpose(1, 0, 2), ref.numpy(), atol=1e-12, rtol=0)


def test_attention_row_sample_equals_full():
    r = _rng(2)
    q, k, v = (r.standard_normal((2, 200, 16)) for _ in range(3))
    rows = np.array([0, 5, 199, 77])
    np.testing.assert_allclose(R.attention(q, k, v, 0.25, rows=rows),
                               R.attention(q, k, v, 0.25)[rows], atol=1e-14, rtol=0)


def test_softmax_rows_sum_to_one_and_nonnegative():
    r = _rng(3)
    p = R.attention_probs(r.standard_normal((50, 8)) * 4, r.standard_normal((90, 8)) * 4, 0.3)
    assert (p >= 0).all()
    np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-12, rtol=0)


def test_attention_special_cases():
    r = _rng(4)
    H, N, D = 2, 33, 8
    q, k, v = (r.standard_normal((H, N, D)) for _ in range(3))
    # a single key: every output row is that key's value
    o = R.attention(q, k[:, :1], v[:, :1], 0.5)
    np.testing.assert_allclose(o, np.broadcast_to(v[:, :1].transpose(1, 0, 2), o.shape), atol=1e-12)
    # all keys equal: uniform weights, output is the mean of the values
    keq = np.broadcast_to(k[:, :1], k.shape)
    o = R.attention(q, keq, v, 0.5)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=1)[None], o.shape), atol=1e-12)
    # V = 1 gives 1; a one-hot value column j reveals the probabilities of key j
    np.testing.assert_allclose(R.attention(q, k, np.ones_like(v), 0.5), 1.0, atol=1e-12)
    j = 11
    vj = np.zeros((H, N, 1))
    vj[:, j, 0] = 1.0
    o = R.attention(q, k, vj, 0.5)
    for h in range(H):
        np.testing.assert_allclose(o[:, h, 0], R.attention_probs(q[h], k[h], 0.5)[:, j], atol=1e-14)


def test_attention_is_noncausal():
    # The last key must influence the first query (no causal mask).
    r = _rng(6)
    q, k, v = (r.standard_normal((1, 10, 4)) for _ in range(3))
    v2 = v.copy()
    v2[0, -1] += 1.0
    assert abs(R.attention(q, k, v2, 0.5)[0] - R.attention(q, k, v, 0.5)[0]).max() > 1e-6


# ----------------------------------------------------------------------- RoPE

def test_rope_hand_values():
    # sections (8, 12, 12) of head_dim 32: channel 8 starts the h block (half 6),
    # channel 20 starts the w block (half 6), channel 0 the t block (half 4).
    sec, th = (8, 12, 12), 10000.0
    pos = np.array([[3, 1, 2]])
    cases = [  # (input channel, axis position, freq index j, block half, block offset)
        (8, 1, 0, 6, 8), (9, 1, 1, 6, 8), (20, 2, 0, 6, 20), (23, 2, 3, 6, 20), (1, 3, 1, 4, 0)]
    for ch, p, j, half, off in cases:
        x = np.zeros((1, 1, 32))
        x[0, 0, ch] = 1.0
        y = R.apply_rope_3d(x, pos, sec, th)[0, 0]
        block = 2 * half
        phi = p * th ** (-2.0 * j / block)
        exp = np.zeros(32)
        exp[ch] = math.cos(phi)
        exp[ch + half] = math.sin(phi)
        np.testing.assert_allclose(y, exp, atol=1e-15)
        # the second member of a pair turns the other way: e_b -> (-sin, cos)
        x = np.zeros((1, 1, 32))
        x[0, 0, ch + half] = 1.0
        y = R.apply_rope_3d(x, pos, sec, th)[0, 0]
        exp = np.zeros(32)
        exp[ch] = -math.sin(phi)
        exp[ch + half] = math.cos(phi)
        np.testing.assert_allclose(y, exp, atol=1e-15)


def test_rope_inv_freq_closed_form():
    np.testing.assert_allclose(R.rope_inv_freq(32, 10000.0)[[0, 1, 15]],
                               [1.0, 10000.0 ** (-1 / 16), 10000.0 ** (-15 / 16)], rtol=1e-15)


@pytest.mark.parametrize("sec,D", [((16, 32, 32), 80), ((8, 12, 12), 32)])
def test_rope_invariants(sec, D):
    r = _rng(D)
    N, H = 40, 3
    x = r.standard_normal((N, H, D))
    pos = np.stack([np.zeros(N, int), r.integers(0, 150, N), r.integers(0, 150, N)], 1)
    y = R.apply_rope_3d(x, pos, sec, 10000.0)
    # norm preserved per head vector
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-12)
    # position (0,0,0) is the identity
    np.testing.assert_array_equal(R.apply_rope_3d(x, np.zeros_like(pos), sec, 10000.0), x)
    # t = 0 leaves the t block unchanged
    np.testing.assert_array_equal(y[..., :sec[0]], x[..., :sec[0]])
    # q.k depends only on the position offset: shift all positions by (0, dh, dw)
    k = r.standard_normal((N, H, D))
    d1 = np.einsum("nhd,mhd->hnm", y, R.apply_rope_3d(k, pos, sec, 10000.0))
    shift = pos + np.array([0, 7, 13])
    d2 = np.einsum("nhd,mhd->hnm", R.apply_rope_3d(x, shift, sec, 10000.0),
                   R.apply_rope_3d(k, shift, sec, 10000.0))
    np.testing.assert_allclose(d1, d2, atol=1e-10)


def test_rope_positions_raster():
    p = R.positions_raster(1, 3, 4)
    assert p.shape == (12, 3)
    assert tuple(p[5]) == (0, 1, 1) and tuple(p[11]) == (0, 2, 3)


# ------------------------------------------------------ LayerNorm and GELU

def test_layer_norm_matches_torch_and_standardises():
    r = _rng(7)
    x = r.standard_normal((20, 1280)) * 3 + 1.5
    g, b = r.standard_normal(1280), r.standard_normal(1280)
    ref = F.layer_norm(torch.tensor(x), (1280,), torch.tensor(g), torch.tensor(b), eps=1e-6)
    np.testing.assert_allclose(R.layer_norm(x, g, b, 1e-6), ref.numpy(), atol=1e-12)
    z = R.layer_norm(x, np.ones(1280), np.zeros(1280), 1e-6)
    np.testing.assert_allclose(z.mean(axis=1), 0, atol=1e-12)
    np.testing.assert_allclose(z.var(axis=1), 1, atol=1e-6)


def test_gelu_matches_torch_and_identities():
    x = np.linspace(-8, 8, 1001)
    ref = F.gelu(torch.tensor(x), approximate="tanh").numpy()
    np.testing.assert_allclose(R.gelu(x, True), ref, atol=1e-14)
    np.testing.assert_allclose(R.gelu(x, False), F.gelu(torch.tensor(x)).numpy(), atol=1e-14)
    assert R.gelu(np.array([0.0]))[0] == 0.0
    np.testing.assert_allclose(R.gelu(x) - R.gelu(-x), x, atol=1e-14)


# ----------------------------------------------------------- patch embedding

@pytest.mark.parametrize("H,W", [(28, 56), (112, 112)])
def test_patch_embed_equals_conv3d(H, W):
    r = _rng(H + W)
    img = r.standard_normal((3, H, W))
    wt = r.standard_normal((24, 3, 2, 14, 14)) * 0.02
    bias = r.standard_normal(24)
    got = R.patch_embed(R.patch_unfold(img, 14, 2), wt, bias)  # [gh*gw, 24]
    clip = torch.tensor(np.stack([img, img], axis=1))[None]  # [1, 3, 2, H, W]: frame repeated
    ref = F.conv3d(clip, torch.tensor(wt), torch.tensor(bias), stride=(2, 14, 14))  # [1,24,1,gh,gw]
    ref = ref[0, :, 0].reshape(24, -1).T.numpy()
    np.testing.assert_allclose(got, ref, atol=1e-12)


@pytest.mark.parametrize("F", [1, 2, 3, 4])
def test_video_patch_embed_equals_conv3d(F):
    # A clip of F frames: Conv3d with temporal stride 2 over the frames, the last frame
    # repeated when F is odd (one image = a clip of one frame = its frame twice).
    r = _rng(40 + F)
    clip = r.standard_normal((F, 3, 28, 42))
    wt = r.standard_normal((12, 3, 2, 14, 14)) * 0.02
    bias = r.standard_normal(12)
    got = R.patch_embed(R.patch_unfold_video(clip, 14, 2), wt, bias)
    T = -(-F // 2)
    padded = np.concatenate([clip, np.repeat(clip[-1:], 2 * T - F, axis=0)], axis=0)  # [2T, 3, H, W]
    ref = F_conv3d(padded, wt, bias)  # [12, T, gh, gw]
    np.testing.assert_allclose(got, ref.reshape(12, -1).T, atol=1e-12)
    if F == 1:
        np.testing.assert_array_equal(R.patch_unfold_video(clip, 14, 2), R.patch_unfold(clip[0], 14, 2))


def F_conv3d(clip, wt, bias):
    x = torch.tensor(clip).permute(1, 0, 2, 3)[None]  # [1, 3, F, H, W]
    return F.conv3d(x, torch.tensor(wt), torch.tensor(bias), stride=(2, 14, 14))[0].numpy()


def test_video_forward_one_frame_equals_image_forward():
    cfg = S.get_config("tiny")
    w = S.weights_f64(S.make_weights(cfg, affine=True))
    px = S.make_pixels(cfg, batch=1).astype(np.float64)
    img = R.forward(px, w, cfg)
    vid = R.forward_video(px[:, None], w, cfg)
    np.testing.assert_allclose(vid["out"], img["out"], atol=1e-12)


def test_video_time_axis_matters_and_merges_within_slices():
    cfg = S.get_config("tiny", layers=1)
    w = S.weights_f64(S.make_weights(cfg, affine=True, layers=1))
    r = _rng(50)
    clip = r.standard_normal((1, 4, 3, 56, 56))
    res = R.forward_video(clip, w, cfg)
    assert res["tower"].shape == (1, 2 * 16, 128) and res["out"].shape == (1, 2 * 4, 256)
    # swapping the two temporal patches changes the result (RoPE's t block, attention
    # across time), so the time axis is not ignored
    swapped = np.concatenate([clip[:, 2:], clip[:, :2]], axis=1)
    assert abs(R.forward_video(swapped, w, cfg)["out"] - res["out"]).max() > 1e-6


def test_patch_unfold_layout():
    img = np.arange(3 * 28 * 42, dtype=np.float64).reshape(3, 28, 42)
    u = R.patch_unfold(img, 14, 2)
    assert u.shape == (6, 1176)
    # patch (h=1, w=2) is raster index 5; element (c=2, t=1, kh=3, kw=4)
    assert u[5, 2 * 392 + 1 * 196 + 3 * 14 + 4] == img[2, 14 + 3, 28 + 4]
    np.testing.assert_array_equal(u[:, :196], u[:, 196:392])  # repeated frame


# --------------------------------------------------------------------- merge

def test_merge_matches_brute_force_and_maps():
    t, h, w, C = 2, 4, 6, 3
    x = np.arange(t * h * w * C, dtype=np.float64).reshape(t * h * w, C)
    m = R.merge_2x2(x, t, h, w)
    assert m.shape == (t * h * w // 4, 4 * C)
    for tt in range(t):
        for i in range(h // 2):
            for j in range(w // 2):
                row = m[tt * (h // 2) * (w // 2) + i * (w // 2) + j]
                srcs = [(2 * i, 2 * j), (2 * i, 2 * j + 1), (2 * i + 1, 2 * j), (2 * i + 1, 2 * j + 1)]
                for a, (hh, ww) in enumerate(srcs):
                    np.testing.assert_array_equal(row[a * C:(a + 1) * C], x[tt * h * w + hh * w + ww])
    # the block order lists each merged group's members consecutively
    bo = R.block_order(t, h, w)
    np.testing.assert_array_equal(bo.reshape(-1, 4), R.merge_source_map(t, h, w))
    assert sorted(bo.tolist()) == list(range(t * h * w))


# ----------------------------------------------------------- layer, projector

def _layer_weights(cfg, seed, affine=True):
    return S.weights_f64(S.make_weights(cfg, seed=seed, affine=affine, layers=1))


def test_layer_without_rope_matches_torch_modules():
    cfg = S.get_config("tiny", use_rope=False)
    w = _layer_weights(cfg, 11)
    d, H = cfg["hidden"], cfg["heads"]
    r = _rng(12)
    x = r.standard_normal((64, d))
    mha = torch.nn.MultiheadAttention(d, H, bias=True, batch_first=True)
    ln1, ln2 = torch.nn.LayerNorm(d, eps=1e-6), torch.nn.LayerNorm(d, eps=1e-6)
    fc1, fc2 = torch.nn.Linear(d, cfg["mlp"]), torch.nn.Linear(cfg["mlp"], d)
    T = torch.tensor
    with torch.no_grad():
        mha.in_proj_weight.copy_(T(w["layers.0.attn.qkv.weight"]))
        mha.in_proj_bias.copy_(T(w["layers.0.attn.qkv.bias"]))
        mha.out_proj.weight.copy_(T(w["layers.0.attn.o.weight"]))
        mha.out_proj.bias.copy_(T(w["layers.0.attn.o.bias"]))
        for mod, nm in ((ln1, "ln1"), (ln2, "ln2")):
            mod.weight.copy_(T(w[f"layers.0.{nm}.weight"]))
            mod.bias.copy_(T(w[f"layers.0.{nm}.bias"]))
        for mod, nm in ((fc1, "fc1"), (fc2, "fc2")):
            mod.weight.copy_(T(w[f"layers.0.mlp.{nm}.weight"]))
            mod.bias.copy_(T(w[f"layers.0.mlp.{nm}.bias"]))
        xt = T(x)[None]
        a = ln1(xt)
        xt = xt + mha(a, a, a, need_weights=False)[0]
        xt = xt + fc2(F.gelu(fc1(ln2(xt)), approximate="tanh"))
    np.testing.assert_allclose(R.tower_layer(x, w, 0, cfg, None), xt[0].numpy(), atol=1e-11)


def test_layer_permutation_equivariance_and_translation_invariance():
    cfg = S.get_config("tiny")
    w = _layer_weights(cfg, 13)
    r = _rng(14)
    x = r.standard_normal((64, cfg["hidden"]))
    pos = R.positions_raster(1, 8, 8)
    perm = r.permutation(64)
    # RoPE off: permuting the tokens permutes the output
    y = R.tower_layer(x, w, 0, cfg, None)
    np.testing.assert_allclose(R.tower_layer(x[perm], w, 0, cfg, None), y[perm], atol=1e-12)
    # RoPE on: the same holds when positions travel with their tokens
    y = R.tower_layer(x, w, 0, cfg, pos)
    np.testing.assert_allclose(R.tower_layer(x[perm], w, 0, cfg, pos[perm]), y[perm], atol=1e-12)
    # RoPE makes attention depend on relative position only: a common shift of all
    # positions leaves the block's output unchanged (fails if v were rotated, or only
    # one of q, k)
    np.testing.assert_allclose(R.tower_layer(x, w, 0, cfg, pos + np.array([0, 5, 9])), y, atol=1e-10)
    # and RoPE is not a no-op
    assert abs(R.tower_layer(x, w, 0, cfg, None) - y).max() > 1e-6


def test_projector_matches_torch_modules():
    cfg = S.get_config("tiny")
    w = S.weights_f64(S.make_weights(cfg, seed=21, affine=True, layers=0))
    r = _rng(22)
    gh = gw = 4
    x = r.standard_normal((gh * gw, cfg["hidden"]))
    T = torch.tensor
    xt = T(x)
    y = F.linear(F.gelu(F.linear(xt, T(w["proj.patch_fc1.weight"]), T(w["proj.patch_fc1.bias"])),
                        approximate="tanh"),
                 T(w["proj.patch_fc2.weight"]), T(w["proj.patch_fc2.bias"]))
    # torch-side 2x2 grouping: [h, w, C] -> [h/2, 2, w/2, 2, C] -> [h/2, w/2, 2, 2, C]
    g = y.reshape(gh // 2, 2, gw // 2, 2, -1).permute(0, 2, 1, 3, 4).reshape(gh * gw // 4, -1)
    z = F.linear(F.gelu(F.linear(g, T(w["proj.merge_fc1.weight"]), T(w["proj.merge_fc1.bias"])),
                        approximate="tanh"),
                 T(w["proj.merge_fc2.weight"]), T(w["proj.merge_fc2.bias"]))
    np.testing.assert_allclose(R.projector(x, w, cfg, 1, gh, gw), z.numpy(), atol=1e-12)


def test_forward_is_order_independent_under_block_order():
    # The GPU keeps tokens in 2x2-block order; the tower output, permuted back, must
    # equal the raster-order tower, because positions travel with the tokens.
    cfg = S.get_config("tiny")
    w = S.weights_f64(S.make_weights(cfg, affine=True))
    px = S.make_pixels(cfg, batch=1).astype(np.float64)
    ref = R.forward(px, w, cfg)
    gh, gw = 8, 8
    bo = R.block_order(1, gh, gw)
    x = R.patch_embed(R.patch_unfold(px[0], 14, 2), w["embeddings.proj.weight"],
                      w["embeddings.proj.bias"])[bo]
    pos = R.positions_raster(1, gh, gw)[bo]
    for i in range(cfg["layers"]):
        x = R.tower_layer(x, w, i, cfg, pos)
    np.testing.assert_allclose(x, ref["tower"][0][bo], atol=1e-11)


# ------------------------------------------------------------- shape facts

def test_shape_facts_from_pages():
    facts = json.load(open(GOLDEN))
    for e in facts["images"]:
        g = R.token_grid(tuple(e["image"]), patch=facts["tower"]["patch"])
        assert (g["t"], g["h"], g["w"]) == tuple(e["grid"]), e["cite"]
        assert g["tokens"] == e["tokens"], e["cite"]
        if "merged_tokens" in e:
            assert g["merged"] == e["merged_tokens"], e["cite"]
    pj = facts["projector"]
    assert 4 * pj["hidden_size"] == pj["merged_hidden_size"]
    cfg = S.get_config("tower448")
    names = [n for n, _, _ in S.weight_names(cfg) if n.startswith("proj.")]
    assert len(names) == pj["tensors"]


def test_shape_facts_one_full_width_layer_448():
    # 448x448 -> 1024 tower tokens of 1280 -> 256 merged of 5120 -> 256 x 6144.
    facts = json.load(open(GOLDEN))["images"][0]
    cfg = S.get_config("tower448", layers=1)
    w = S.weights_f64(S.make_weights(cfg, layers=1))
    px = S.make_pixels(cfg, batch=1).astype(np.float64)
    res = R.forward(px, w, cfg)
    assert res["tower"].shape == (1, facts["tokens"], facts["tower_width"])
    assert res["merged"].shape == (1, facts["merged_tokens"], facts["merged_width"])
    assert res["out"].shape == (1, facts["merged_tokens"], facts["projected_width"])
    assert np.isfinite(res["out"]).all()


def test_tiny_shape_facts():
    cfg = S.get_config("tiny")
    w = S.weights_f64(S.make_weights(cfg))
    res = R.forward(S.make_pixels(cfg).astype(np.float64), w, cfg)
    assert res["tower"].shape == (1, 64, 128)
    assert res["merged"].shape == (1, 16, 512)
    assert res["out"].shape == (1, 16, 256)


def test_row_sampled_layer_and_projector_equal_full():
    cfg = S.get_config("tiny")
    w = S.weights_f64(S.make_weights(cfg, seed=31, affine=True, layers=1))
    x = _rng(32).standard_normal((64, cfg["hidden"]))
    pos = R.positions_raster(1, 8, 8)
    rows = np.array([0, 9, 33, 63])
    np.testing.assert_allclose(R.tower_layer_rows(x, w, 0, cfg, pos, rows),
                               R.tower_layer(x, w, 0, cfg, pos)[rows], atol=1e-12)
    np.testing.assert_allclose(R.tower_layer_rows(x, w, 0, cfg, None, rows),
                               R.tower_layer(x, w, 0, cfg, None)[rows], atol=1e-12)
    mrows = np.array([0, 5, 15])
    np.testing.assert_allclose(R.projector_rows(x, w, cfg, 1, 8, 8, mrows),
                               R.projector(x, w, cfg, 1, 8, 8)[mrows], atol=1e-12)


# -------------------------------------------------------------- preprocessing

def test_cubic_kernel_values_and_partition_of_unity():
    # Keys' kernel at a = -0.5, by hand: (a+2)|x|^3 - (a+3)|x|^2 + 1 on [0, 1],
    # a|x|^3 - 5a|x|^2 + 8a|x| - 4a on [1, 2)
    assert R.cubic_kernel(0.0) == 1.0
    for x in (1.0, -1.0, 2.0, -2.0, 2.5):
        assert R.cubic_kernel(x) == 0.0
    assert R.cubic_kernel(0.5) == pytest.approx(0.5625, abs=1e-15)
    assert R.cubic_kernel(-1.5) == pytest.approx(-0.0625, abs=1e-15)
    assert R.cubic_kernel(0.25) == pytest.approx(1.5 * 0.25 ** 3 - 2.5 * 0.25 ** 2 + 1, abs=1e-15)
    for x in _rng(40).uniform(0, 1, 7):  # the four taps around any point sum to 1
        assert sum(R.cubic_kernel(x + k) for k in (-2, -1, 0, 1)) == pytest.approx(1.0, abs=1e-14)


@pytest.mark.parametrize("src,dst", [((20, 30), (28, 42)), ((97, 61), (28, 28)), ((40, 13), (14, 56)),
                                     ((448, 336), (112, 84)), ((28, 28), (28, 28)), ((9, 300), (42, 14))])
def test_resize_equals_torch_antialiased_bicubic(src, dst):
    # torch's antialiased bicubic is an independent implementation of the same
    # resampling (a = -0.5, stretched kernel when shrinking, renormalised edge taps)
    img = _rng(41).uniform(0, 255, size=(*src, 3))
    got = R.resize_bicubic(img, *dst)
    ref = F.interpolate(torch.tensor(img).permute(2, 0, 1)[None], size=dst, mode="bicubic", antialias=True,
                        align_corners=False)[0].permute(1, 2, 0).numpy()
    np.testing.assert_allclose(got, ref, atol=1e-10)


def test_resize_identity_constant_and_linear():
    r = _rng(42)
    img = r.uniform(0, 255, size=(17, 23, 3))
    np.testing.assert_array_equal(R.resize_bicubic(img, 17, 23), img)  # same size: exact copy
    flat = np.full((31, 19, 3), 77.0)
    np.testing.assert_allclose(R.resize_bicubic(flat, 14, 42), 77.0, atol=1e-12)
    # upscaling reproduces a linear ramp away from the borders (cubic convolution is exact
    # on polynomials of degree < 3 when no tap is dropped)
    ramp = np.broadcast_to(np.arange(40.0)[None, :, None] * 3.0 + 5.0, (6, 40, 3)).copy()
    out = R.resize_bicubic(ramp, 6, 100)
    centres = (np.arange(100) + 0.5) * 40 / 100 - 0.5
    np.testing.assert_allclose(out[:, 5:-5, 0], np.broadcast_to(centres[5:-5] * 3.0 + 5.0, (6, 90)), atol=1e-10)


def test_preprocess_channel_order_and_statistics():
    img = np.zeros((14, 28, 3), dtype=np.uint8)
    img[..., 0], img[..., 1], img[..., 2] = 10, 128, 250
    out = R.preprocess(img, 28, 14, S.CLIP_MEAN, S.CLIP_STD)
    assert out.shape == (3, 28, 14)
    for c, v in enumerate((10, 128, 250)):
        np.testing.assert_allclose(out[c], (v / 255 - S.CLIP_MEAN[c]) / S.CLIP_STD[c], atol=1e-12)
    # a non-constant image: preprocess = normalise(torch resize) channel by channel
    img = S.make_images_u8([(50, 70)], seed=1)[0]
    ref = F.interpolate(torch.tensor(img, dtype=torch.float64).permute(2, 0, 1)[None], size=(28, 42),
                        mode="bicubic", antialias=True, align_corners=False)[0].numpy()
    ref = (ref / 255 - np.asarray(S.CLIP_MEAN)[:, None, None]) / np.asarray(S.CLIP_STD)[:, None, None]
    np.testing.assert_allclose(R.preprocess(img, 28, 42, S.CLIP_MEAN, S.CLIP_STD), ref, atol=1e-10)


# ------------------------------------------------------------------ backward

def _fd_directional(f, x, v, dy, eps=1e-5):
    """<dy, (f(x + eps v) - f(x - eps v)) / (2 eps)>: the directional derivative of
    the loss <dy, f(x)> along v, by central differences (error O(eps^2))."""
    return float(np.sum(dy * (f(x + eps * v) - f(x - eps * v))) / (2 * eps))


def test_layer_norm_and_gelu_backward_equal_autograd():
    r = _rng(50)
    x, dy, gamma = r.standard_normal((7, 40)), r.standard_normal((7, 40)), 1 + 0.1 * r.standard_normal(40)
    xt = torch.tensor(x, requires_grad=True)
    F.layer_norm(xt, (40,), torch.tensor(gamma), torch.tensor(0.1 * gamma), 1e-6).backward(torch.tensor(dy))
    np.testing.assert_allclose(R.layer_norm_backward(x, gamma, 1e-6, dy), xt.grad.numpy(), atol=1e-12)
    z = 3 * r.standard_normal((5, 33))
    dz = r.standard_normal((5, 33))
    for tanh_form, approx in ((True, "tanh"), (False, "none")):
        zt = torch.tensor(z, requires_grad=True)
        F.gelu(zt, approximate=approx).backward(torch.tensor(dz))
        np.testing.assert_allclose(R.gelu_backward(z, dz, tanh_form), zt.grad.numpy(), atol=1e-12)


def test_rope_backward_is_the_transpose():
    r = _rng(51)
    pos = R.positions_raster(2, 3, 5)
    x, y = r.standard_normal((30, 2, 80)), r.standard_normal((30, 2, 80))
    rx = R.apply_rope_3d(x, pos, (16, 32, 32), 1e4)
    # <R x, y> = <x, R^T y> and R^T R = I
    assert np.sum(rx * y) == pytest.approx(np.sum(x * R.rope_3d_backward(y, pos, (16, 32, 32), 1e4)), abs=1e-10)
    np.testing.assert_allclose(R.rope_3d_backward(rx, pos, (16, 32, 32), 1e4), x, atol=1e-12)


def test_attention_backward_equals_autograd_and_differences():
    r = _rng(52)
    n, N, D = 9, 13, 16
    q, k, v, do = r.standard_normal((n, D)), r.standard_normal((N, D)), r.standard_normal((N, D)), \
        r.standard_normal((n, D))
    scale = D ** -0.5
    dq, dk, dv = R.attention_backward(q, k, v, do, scale)
    qt, kt, vt = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    (torch.softmax(qt @ kt.T * scale, dim=1) @ vt).backward(torch.tensor(do))
    for got, ref in ((dq, qt.grad), (dk, kt.grad), (dv, vt.grad)):
        np.testing.assert_allclose(got, ref.numpy(), atol=1e-12)
    # and against central differences of the oracle's own forward, input by input
    f = lambda a, b, c: R.attention_probs(a, b, scale) @ c
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        vdir = r.standard_normal((q, k, v)[which].shape)
        args = [q, k, v]
        g = lambda z: f(*[z if i == which else args[i] for i in range(3)])
        assert _fd_directional(g, args[which], vdir, do) == pytest.approx(np.sum(grad * vdir), rel=1e-7)


def test_layer_backward_without_rope_equals_autograd_of_torch_modules():
    cfg = S.get_config("tiny", use_rope=False)
    w = _layer_weights(cfg, 53)
    d, H = cfg["hidden"], cfg["heads"]
    r = _rng(54)
    x, dy = r.standard_normal((24, d)), r.standard_normal((24, d))
    mha = torch.nn.MultiheadAttention(d, H, bias=True, batch_first=True)
    ln1, ln2 = torch.nn.LayerNorm(d, eps=1e-6), torch.nn.LayerNorm(d, eps=1e-6)
    fc1, fc2 = torch.nn.Linear(d, cfg["mlp"]), torch.nn.Linear(cfg["mlp"], d)
    T = torch.tensor
    with torch.no_grad():
        mha.in_proj_weight.copy_(T(w["layers.0.attn.qkv.weight"]))
        mha.in_proj_bias.copy_(T(w["layers.0.attn.qkv.bias"]))
        mha.out_proj.weight.copy_(T(w["layers.0.attn.o.weight"]))
        mha.out_proj.bias.copy_(T(w["layers.0.attn.o.bias"]))
        for mod, nm in ((ln1, "ln1"), (ln2, "ln2")):
            mod.weight.copy_(T(w[f"layers.0.{nm}.weight"]))
            mod.bias.copy_(T(w[f"layers.0.{nm}.bias"]))
        for mod, nm in ((fc1, "fc1"), (fc2, "fc2")):
            mod.weight.copy_(T(w[f"layers.0.mlp.{nm}.weight"]))
            mod.bias.copy_(T(w[f"layers.0.mlp.{nm}.bias"]))
    xt = T(x)[None].requires_grad_(True)
    a = ln1(xt)
    y = xt + mha(a, a, a, need_weights=False)[0]
    y = y + fc2(F.gelu(fc1(ln2(y)), approximate="tanh"))
    y.backward(T(dy)[None])
    np.testing.assert_allclose(R.tower_layer_backward(x, w, 0, cfg, None, dy), xt.grad[0].numpy(), atol=1e-11)


def test_layer_backward_with_rope_equals_central_differences():
    cfg = S.get_config("tiny")
    w = _layer_weights(cfg, 55)
    r = _rng(56)
    pos = R.positions_raster(1, 4, 6)
    x, dy = r.standard_normal((24, cfg["hidden"])), r.standard_normal((24, cfg["hidden"]))
    dx = R.tower_layer_backward(x, w, 0, cfg, pos, dy)
    for _ in range(3):
        vdir = r.standard_normal(x.shape)
        fd = _fd_directional(lambda z: R.tower_layer(z, w, 0, cfg, pos), x, vdir, dy)
        assert fd == pytest.approx(np.sum(dx * vdir), rel=1e-7)
    # the rotation matters: without it the gradient differs
    assert np.abs(R.tower_layer_backward(x, w, 0, cfg, None, dy) - dx).max() > 1e-3


def test_patch_fold_is_the_transpose_of_unfold():
    r = _rng(57)
    img, du = r.standard_normal((3, 28, 42)), r.standard_normal((6, 3 * 2 * 14 * 14))
    assert np.sum(R.patch_unfold(img, 14, 2) * du) == pytest.approx(np.sum(img * R.patch_fold(du, 28, 42)),
                                                                     abs=1e-10)


def test_tower_backward_equals_central_differences_on_pixels():
    cfg = dict(S.get_config("tiny"), image=(28, 56))
    w = S.weights_f64(S.make_weights(cfg, affine=True))
    r = _rng(58)
    px = r.standard_normal((1, 3, 28, 56))
    d_tower = r.standard_normal((1, 8, cfg["hidden"]))
    res = R.tower_backward(px, w, cfg, d_tower)
    np.testing.assert_allclose(res["tower"], R.forward(px, w, cfg)["tower"], atol=1e-12)
    for _ in range(2):
        vdir = r.standard_normal(px.shape)
        fd = _fd_directional(lambda z: R.forward(z, w, cfg)["tower"], px, vdir, d_tower)
        assert fd == pytest.approx(np.sum(res["d_pixels"] * vdir), rel=1e-6)

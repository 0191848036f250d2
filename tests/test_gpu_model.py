"""Tower-level parity on the GPU through the C ABI: patch embedding, single layers
(teacher-forced and free-running), merge + projector and the full forward, against the
fp64 oracle on the same seeded inputs.  Large images are checked on sampled outputs.
"""
import numpy as np
import pytest
import torch

from oracle import vit_ref as R
from vision_transformer_encoder_vit_b200 import synthetic as S
from tests.gpu_util import (REL_L2_FINAL, REL_L2_LAYER, assert_close, assert_rows_close, dev_bf16, dev_f32,
                            empty_bf16, host_bits, host_f64, rel_l2)

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from vision_transformer_encoder_vit_b200 import vt as V


def _tower(cfg, affine, layers=None):
    bits = S.make_weights(cfg, affine=affine, layers=layers)
    c = dict(cfg)
    if layers is not None:
        c["layers"] = layers
    return V.Tower(c, bits), S.weights_f64(bits), c


@pytest.mark.parametrize("affine", [False, True])
@pytest.mark.parametrize("B", [1, 2])
def test_tiny_forward(B, affine):
    cfg = S.get_config("tiny")
    tw, w, cfg = _tower(cfg, affine)
    px = S.make_pixels(cfg, batch=B)
    t, gh, gw = S.token_grid(cfg)
    grid = (t, gh, gw)
    N = gh * gw
    ws = tw.workspace(B, grid)
    out = empty_bf16(B, N // 4, cfg["proj_out"])
    tower = empty_bf16(B, N, cfg["hidden"])
    V.vt_forward(tw.h, dev_f32(px), grid, B, out, tower, ws, ws.numel())
    V.vt_check()
    ref = R.forward(px.astype(np.float64), w, cfg)
    assert_close(host_f64(tower), ref["tower"], rel=REL_L2_LAYER, what="tower output")
    assert_close(host_f64(out), ref["out"], rel=REL_L2_FINAL, what="projected tokens")
    tw.close()


@pytest.mark.parametrize("name", ["tiny", "layer1280"])
def test_layer_teacher_forced(name):
    cfg = S.get_config(name)
    tw, w, cfg = _tower(cfg, affine=True)
    t, gh, gw = S.token_grid(cfg)
    grid = (t, gh, gw)
    N = gh * gw
    B = 2
    x = S.make_activations(B * N, cfg["hidden"], cfg["seed"])
    xf = S.bf16_to_f64(x).reshape(B, N, -1)
    ws = tw.workspace(B, grid)
    pos = R.positions_raster(t, gh, gw)
    for i in range(cfg["layers"]):
        y = empty_bf16(B, N, cfg["hidden"])
        V.vt_tower_layer(tw.h, i, dev_bf16(x), y, grid, B, ws, ws.numel())
        got = host_f64(y)
        for b in range(B):
            ref = R.tower_layer(xf[b], w, i, cfg, pos)
            assert_close(got[b], ref, rel=REL_L2_LAYER, what=f"{name} layer {i} image {b}")
    tw.close()


def test_tiny_free_running_layers_and_projector():
    cfg = S.get_config("tiny")
    tw, w, cfg = _tower(cfg, affine=True)
    t, gh, gw = S.token_grid(cfg)
    grid = (t, gh, gw)
    N = gh * gw
    px = S.make_pixels(cfg, batch=1)
    ref = R.forward(px.astype(np.float64), w, cfg, keep_layers=True)
    ws = tw.workspace(1, grid)
    x = empty_bf16(1, N, cfg["hidden"])
    V.vt_patch_embed(tw.h, dev_f32(px), grid, 1, x, ws, ws.numel())
    assert_close(host_f64(x), ref["layer_in"][0], what="patch embedding")
    for i in range(cfg["layers"]):
        V.vt_tower_layer(tw.h, i, x, x, grid, 1, ws, ws.numel())
        assert_close(host_f64(x), ref["layer_out"][i], what=f"free-running layer {i}")
    out = empty_bf16(1, N // 4, cfg["proj_out"])
    V.vt_merge_project(tw.h, x, grid, 1, out, ws, ws.numel())
    assert_close(host_f64(out), ref["out"], rel=REL_L2_FINAL, what="merge + projector")
    tw.close()


def test_merge_project_teacher_forced():
    cfg = S.get_config("tiny", image=(224, 168))
    tw, w, cfg = _tower(cfg, affine=True, layers=0)
    t, gh, gw = S.token_grid(cfg)
    grid = (t, gh, gw)
    N = gh * gw
    x = S.make_activations(3 * N, cfg["hidden"], 9)
    ws = tw.workspace(3, grid)
    out = empty_bf16(3, N // 4, cfg["proj_out"])
    V.vt_merge_project(tw.h, dev_bf16(x), grid, 3, out, ws, ws.numel())
    got = host_f64(out)
    xf = S.bf16_to_f64(x).reshape(3, N, -1)
    for b in range(3):
        assert_close(got[b], R.projector(xf[b], w, cfg, t, gh, gw), rel=REL_L2_FINAL, what=f"projector {b}")
    tw.close()


def test_forward_host_matches_device_forward():
    cfg = S.get_config("tiny")
    tw, w, cfg = _tower(cfg, affine=True)
    B = 3
    t, gh, gw = S.token_grid(cfg)
    grid = (t, gh, gw)
    N = gh * gw
    px = S.make_pixels(cfg, batch=B)
    ws_bytes = V.vt_forward_host_workspace_bytes(tw.h, B, grid)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    host_px = torch.from_numpy(px).pin_memory()
    host_out = torch.empty((B, N // 4, cfg["proj_out"]), dtype=torch.bfloat16).pin_memory()
    V.vt_forward_host(tw.h, host_px, grid, B, host_out, ws, ws_bytes)
    dev_out = empty_bf16(B, N // 4, cfg["proj_out"])
    ws2 = tw.workspace(B, grid)
    V.vt_forward(tw.h, dev_f32(px), grid, B, dev_out, None, ws2, ws2.numel())
    np.testing.assert_array_equal(host_out.view(torch.int16).numpy(), host_bits(dev_out).view(np.int16))
    tw.close()


def test_forward_448_batch8_sampled_images():
    # The benchmark workload: 8 images of 448x448 through the 32-layer tower and the
    # projector, in the batch the benchmark launches; images 0 and 7 are compared with
    # the full fp64 oracle forward.  Gates: every layer teacher-forced (the oracle's
    # own layer input, rounded to bf16, through one GPU layer) <= 1e-2 with the element
    # bound; the free-running forward's projected tokens <= 2e-2 overall and <= 5e-2 on
    # every merged token; the free-running tower output after 32 bf16 layers <= 5e-2
    # overall and <= 1e-1 on every token.
    cfg = S.get_config("tower448")
    tw, w, cfg = _tower(cfg, affine=False)
    B = cfg["batch"]
    t, gh, gw = S.token_grid(cfg)
    grid = (t, gh, gw)
    N = gh * gw
    px = S.make_pixels(cfg, batch=B)
    ws = tw.workspace(B, grid)
    out = empty_bf16(B, N // 4, cfg["proj_out"])
    tower = empty_bf16(B, N, cfg["hidden"])
    V.vt_forward(tw.h, dev_f32(px), grid, B, out, tower, ws, ws.numel())
    V.vt_check()
    got_out, got_tower = host_f64(out), host_f64(tower)
    for b in (0, B - 1):
        ref = R.forward(px[b:b + 1].astype(np.float64), w, cfg, keep_layers=True)
        if b == 0:
            y = empty_bf16(1, N, cfg["hidden"])
            for i in range(cfg["layers"]):
                xin = dev_bf16(S.bf16_bits(ref["layer_in"][i][0].astype(np.float32)))
                V.vt_tower_layer(tw.h, i, xin, y, grid, 1, ws, ws.numel())
                assert_close(host_f64(y)[0], ref["layer_out"][i][0], rel=REL_L2_LAYER,
                             what=f"448 layer {i} teacher-forced")
        assert_rows_close(got_out[b], ref["out"][0], rel=REL_L2_FINAL, rel_row=5e-2,
                          what=f"448 projected image {b} (free-running)")
        assert_rows_close(got_tower[b], ref["tower"][0], rel=5e-2, rel_row=1e-1,
                          what=f"448 tower image {b} (free-running, 32 layers)")
    tw.close()


def test_forward_2016_sampled():
    # One 2016x2016 image (144x144 = 20736 tokens).  The full forward runs on the GPU;
    # the oracle checks (a) the patch embedding at sampled token rows, (b) layers 0, 10,
    # 20 and 31 teacher-forced: the GPU's own bf16 input of that layer (the layers run
    # one by one on the GPU) through the oracle's layer at sampled token rows (every key
    # and value from all 20736 tokens), against the GPU layer's output; (c) the
    # projector teacher-forced on the GPU tower output at sampled merged tokens.
    cfg = S.get_config("tower2016")
    tw, w, cfg = _tower(cfg, affine=False)
    t, gh, gw = S.token_grid(cfg)
    grid = (t, gh, gw)
    N = gh * gw
    px = S.make_pixels(cfg, batch=1)
    ws = tw.workspace(1, grid)
    out = empty_bf16(1, N // 4, cfg["proj_out"])
    tower = empty_bf16(1, N, cfg["hidden"])
    V.vt_forward(tw.h, dev_f32(px), grid, 1, out, tower, ws, ws.numel())
    V.vt_check()
    got_tower, got_out = host_f64(tower)[0], host_f64(out)[0]
    assert np.isfinite(got_tower).all() and np.isfinite(got_out).all()
    rng = np.random.default_rng(2016)
    # (a) patch embedding at sampled rows
    x = empty_bf16(1, N, cfg["hidden"])
    V.vt_patch_embed(tw.h, dev_f32(px), grid, 1, x, ws, ws.numel())
    rows = np.sort(rng.choice(N, size=64, replace=False))
    ref_pe = R.patch_embed(R.patch_unfold(px[0].astype(np.float64))[rows], w["embeddings.proj.weight"],
                           w["embeddings.proj.bias"])
    assert_close(host_f64(x)[0][rows], ref_pe, what="2016 patch embedding rows")
    # (b) layers spread over depth, teacher-forced at sampled rows
    pos = R.positions_raster(t, gh, gw)
    y = empty_bf16(1, N, cfg["hidden"])
    for i in range(cfg["layers"]):
        V.vt_tower_layer(tw.h, i, x, y, grid, 1, ws, ws.numel())
        if i in (0, 10, 20, cfg["layers"] - 1):
            rows = np.sort(rng.choice(N, size=48, replace=False))
            ref = R.tower_layer_rows(host_f64(x)[0], w, i, cfg, pos, rows)
            assert_close(host_f64(y)[0][rows], ref, what=f"2016 layer {i} rows (teacher-forced)")
        x, y = y, x
    # the layer-by-layer chain (raster token order) and the forward (2x2-block order)
    # round differently but compute the same tower: gated as a free-running tower
    assert_rows_close(host_f64(x)[0], got_tower, rel=5e-2, rel_row=1e-1,
                      what="2016 layer-by-layer chain vs forward tower")
    # (c) projector at sampled merged tokens, from the GPU tower output
    mrows = np.sort(rng.choice(N // 4, size=32, replace=False))
    ref_p = R.projector_rows(got_tower, w, cfg, t, gh, gw, mrows)
    assert_close(got_out[mrows], ref_p, rel=REL_L2_FINAL, what="2016 projector rows")
    tw.close()


def test_profile_counts_launches():
    cfg = S.get_config("tiny")
    tw, w, cfg = _tower(cfg, affine=False)
    t, gh, gw = S.token_grid(cfg)
    grid = (t, gh, gw)
    N = gh * gw
    ws = tw.workspace(1, grid)
    out = empty_bf16(1, N // 4, cfg["proj_out"])
    px = dev_f32(S.make_pixels(cfg, batch=1))
    V.vt_profile_begin()
    V.vt_forward(tw.h, px, grid, 1, out, None, ws, ws.numel())
    V.vt_profile_end()
    prof = V.vt_profile_read()
    L = cfg["layers"]
    assert prof["gemm"]["launches"] == 1 + 4 * L + 4
    assert prof["attention"]["launches"] == L
    assert prof["layernorm"]["launches"] == 2 * L
    assert prof["patch_unfold"]["launches"] == 1
    assert all(v["ms"] >= 0 for v in prof.values())
    tw.close()


def test_forward_rejects_small_workspace_and_bad_grid():
    cfg = S.get_config("tiny")
    tw, w, cfg = _tower(cfg, affine=False)
    ws = tw.workspace(1, (1, 8, 8))
    out = empty_bf16(16, 256)
    px = dev_f32(S.make_pixels(cfg, batch=1))
    with pytest.raises(V.VtError) as e:
        V.vt_forward(tw.h, px, (1, 8, 8), 1, out, None, ws, 1024)
    assert e.value.name == "VT_ERR_WORKSPACE"
    with pytest.raises(V.VtError) as e:
        V.vt_forward(tw.h, px, (1, 7, 8), 1, out, None, ws, ws.numel())
    assert e.value.name == "VT_ERR_SHAPE"
    V.vt_check()
    tw.close()


def test_host_forward_async_on_two_streams_matches_sync():
    cfg = S.get_config("tiny")
    bits = S.make_weights(cfg, affine=True)
    tw = V.Tower(cfg, bits)
    grid = (1, 8, 8)
    px = [torch.from_numpy(S.make_pixels(cfg, batch=2, seed=s)).pin_memory() for s in (1, 2)]
    wsb = V.vt_forward_host_workspace_bytes(tw.h, 2, grid)
    ws = [torch.empty(wsb, dtype=torch.uint8, device="cuda") for _ in range(2)]
    ref = [torch.empty((2, 16, cfg["proj_out"]), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    got = [torch.empty_like(r).pin_memory() for r in ref]
    for i in range(2):
        V.vt_forward_host(tw.h, px[i], grid, 2, ref[i], ws[i], wsb)
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    for i in range(2):
        V.vt_forward_host_async(tw.h, px[i], grid, 2, got[i], ws[i], wsb, streams[i])
    torch.cuda.synchronize()
    V.vt_check()
    for i in range(2):
        assert torch.equal(got[i].view(torch.int16), ref[i].view(torch.int16))
    tw.close()

"""Variable-resolution batches on the GPU: images of different sizes packed in one
vt_forward_varlen call, each compared with the fp64 oracle forward of that image alone
(tower output <= 1e-2, projected tokens <= 2e-2 relative L2)."""
import numpy as np
import pytest
import torch

from oracle import vit_ref as R
from vision_transformer_encoder_vit_b200 import synthetic as S
from tests.gpu_util import REL_L2_FINAL, REL_L2_LAYER, assert_close, empty_bf16, host_f64

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from vision_transformer_encoder_vit_b200 import vt as V


def _run(cfg, images, affine, layers=None):
    bits = S.make_weights(cfg, affine=affine, layers=layers)
    c = dict(cfg)
    if layers is not None:
        c["layers"] = layers
    tw = V.Tower(c, bits)
    w = S.weights_f64(bits)
    pix = [S.make_pixels(dict(c, image=hw), batch=1, seed=11 + i)[0] for i, hw in enumerate(images)]
    grids = [(1, hw[0] // 14, hw[1] // 14) for hw in images]
    ntok = [g[1] * g[2] for g in grids]
    packed = torch.from_numpy(np.concatenate([p.ravel() for p in pix])).cuda()
    ws_bytes = V.vt_workspace_bytes_varlen(tw.h, grids)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    out = empty_bf16(sum(ntok) // 4, c["proj_out"])
    tower = empty_bf16(sum(ntok), c["hidden"])
    V.vt_forward_varlen(tw.h, packed, grids, out, tower, ws, ws_bytes)
    V.vt_check()
    got_out, got_tower = host_f64(out), host_f64(tower)
    t0 = 0
    for i, (p, n) in enumerate(zip(pix, ntok)):
        ref = R.forward(p[None].astype(np.float64), w, c)
        assert_close(got_tower[t0:t0 + n], ref["tower"][0], rel=REL_L2_LAYER, what=f"varlen tower image {i}")
        assert_close(got_out[t0 // 4:(t0 + n) // 4], ref["out"][0], rel=REL_L2_FINAL,
                     what=f"varlen projected image {i}")
        t0 += n
    tw.close()


def test_varlen_tiny_mixed_sizes():
    _run(S.get_config("tiny"), [(112, 112), (56, 84), (28, 28), (140, 56), (252, 28)], affine=True)


def test_varlen_full_width_two_layers():
    # 1024 + 384 tokens: the packed rows cross CTA-pair tiles and image boundaries
    _run(S.get_config("tower448"), [(448, 448), (224, 336)], affine=False, layers=2)


def test_varlen_single_image_matches_uniform_forward():
    cfg = S.get_config("tiny")
    bits = S.make_weights(cfg, affine=True)
    tw = V.Tower(cfg, bits)
    px = S.make_pixels(cfg, batch=1)
    grid = (1, 8, 8)
    ws = tw.workspace(1, grid)
    out_u = empty_bf16(16, cfg["proj_out"])
    V.vt_forward(tw.h, torch.from_numpy(px).cuda(), grid, 1, out_u, None, ws, ws.numel())
    ws_v = torch.empty(V.vt_workspace_bytes_varlen(tw.h, [grid]), dtype=torch.uint8, device="cuda")
    out_v = empty_bf16(16, cfg["proj_out"])
    V.vt_forward_varlen(tw.h, torch.from_numpy(px).cuda(), [grid], out_v, None, ws_v, ws_v.numel())
    V.vt_check()
    np.testing.assert_array_equal(host_f64(out_v), host_f64(out_u)[0] if out_u.dim() == 3 else host_f64(out_u))
    tw.close()

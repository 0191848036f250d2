"""Guard bands around every buffer a call writes or reads: each workspace, output,
saved-activation buffer and input sits between two 4 KB bands filled with 0xA5, and
after the call both bands must still hold only 0xA5.  The inputs themselves must be
unchanged.  A kernel that writes one element past its buffer, or a workspace plan
smaller than what the launches touch, shows here even when the result still matches
the oracle.

The shapes are the ones where an extent is easiest to get wrong: grids that are odd
multiples of the 28-pixel merge unit (token counts that are not multiples of the
128-row tiles), a 2x2 grid (4 tokens), a 4096-token image, clips with a repeated last
frame, and a packed batch whose largest image comes last.
"""
import numpy as np
import pytest
import torch

from vision_transformer_encoder_vit_b200 import synthetic as S

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from vision_transformer_encoder_vit_b200 import vt as V

BAND = 4096
FILL = 0xA5


class Banded:
    """A device buffer of `nbytes` between two guard bands (the buffer starts 4096 bytes
    into the allocation, so it keeps the allocation's alignment)."""

    def __init__(self, nbytes: int, fill_body: bool = True):
        self.nbytes = int(nbytes)
        self.raw = torch.full((BAND + self.nbytes + BAND,), FILL, dtype=torch.uint8, device="cuda")
        self.body = self.raw[BAND:BAND + self.nbytes]
        if not fill_body:
            self.body.zero_()

    def typed(self, dtype, *shape):
        return self.body.view(dtype).view(*shape)

    def check(self, what: str):
        torch.cuda.synchronize()
        lo = self.raw[:BAND].cpu().numpy()
        hi = self.raw[BAND + self.nbytes:].cpu().numpy()
        for name, band in (("before", lo), ("after", hi)):
            bad = np.flatnonzero(band != FILL)
            assert bad.size == 0, f"{what}: {bad.size} bytes of the guard band {name} the buffer were written " \
                                  f"(first at band offset {int(bad[0])})"


def banded_from(array: np.ndarray) -> Banded:
    """An input buffer holding `array`'s bytes between guard bands."""
    a = np.ascontiguousarray(array)
    b = Banded(a.nbytes)
    b.body.copy_(torch.from_numpy(a.view(np.uint8).ravel()).cuda())
    return b


def unchanged(b: Banded, array: np.ndarray, what: str):
    b.check(what)
    got = b.body.cpu().numpy()
    assert np.array_equal(got, np.ascontiguousarray(array).view(np.uint8).ravel()), f"{what}: input was modified"


def _tower(name, layers=None, affine=True):
    cfg = S.get_config(name)
    bits = S.make_weights(cfg, affine=affine, layers=layers)
    if layers is not None:
        cfg = dict(cfg, layers=layers)
    return V.Tower(cfg, bits), cfg


@pytest.mark.parametrize("name,hw,B,layers", [
    ("tiny", (84, 140), 2, None),     # 6 x 10 grid, 60 tokens per image
    ("tiny", (28, 28), 3, None),      # 2 x 2 grid, 4 tokens per image
    ("tiny", (196, 252), 1, None),    # 14 x 18 grid, 252 tokens: two ragged 128-row tiles
    ("tower448", (896, 896), 1, 2),   # 64 x 64 = 4096 tokens at full width
])
def test_forward_guard_bands(name, hw, B, layers):
    tw, cfg = _tower(name, layers)
    grid = (1, hw[0] // 14, hw[1] // 14)
    N = grid[1] * grid[2]
    px = S.make_pixels(dict(cfg, image=hw), batch=B, seed=21)
    pin = banded_from(px)
    ws = Banded(V.vt_workspace_bytes(tw.h, B, grid))
    out = Banded(B * (N // 4) * cfg["proj_out"] * 2)
    tower = Banded(B * N * cfg["hidden"] * 2)
    V.vt_forward(tw.h, pin.typed(torch.float32, *px.shape), grid, B, out.typed(torch.bfloat16, B, N // 4, -1),
                 tower.typed(torch.bfloat16, B, N, -1), ws.body, ws.nbytes)
    V.vt_check()
    for b, what in ((ws, "workspace"), (out, "projected tokens"), (tower, "tower output")):
        b.check(f"vt_forward {name} {hw} x{B}: {what}")
    unchanged(pin, px, f"vt_forward {name} {hw}: pixels")
    assert np.isfinite(out.typed(torch.bfloat16, -1).float().cpu().numpy()).all()
    tw.close()


def test_forward_varlen_guard_bands():
    # the largest image last: its tokens end exactly at the end of the packed buffers
    tw, cfg = _tower("tiny")
    images = [(28, 28), (84, 56), (56, 140), (196, 168)]
    grids = [(1, h // 14, w // 14) for h, w in images]
    ntok = sum(g[1] * g[2] for g in grids)
    px = np.concatenate([S.make_pixels(dict(cfg, image=hw), batch=1, seed=30 + i)[0].ravel()
                         for i, hw in enumerate(images)])
    pin = banded_from(px)
    ws = Banded(V.vt_workspace_bytes_varlen(tw.h, grids))
    out = Banded((ntok // 4) * cfg["proj_out"] * 2)
    tower = Banded(ntok * cfg["hidden"] * 2)
    V.vt_forward_varlen(tw.h, pin.typed(torch.float32, -1), grids, out.typed(torch.bfloat16, ntok // 4, -1),
                        tower.typed(torch.bfloat16, ntok, -1), ws.body, ws.nbytes)
    V.vt_check()
    for b, what in ((ws, "workspace"), (out, "projected tokens"), (tower, "tower output")):
        b.check(f"vt_forward_varlen: {what}")
    unchanged(pin, px, "vt_forward_varlen: pixels")
    tw.close()


def test_forward_video_guard_bands():
    tw, cfg = _tower("tiny")
    F, hw, B = 3, (84, 56), 2  # 2 temporal patches, the last frame repeated
    c = dict(cfg, image=hw)
    clips = S.make_clips(c, F, batch=B, seed=40)
    grid = (-(-F // c["temporal_patch"]), hw[0] // 14, hw[1] // 14)
    N = grid[0] * grid[1] * grid[2]
    pin = banded_from(clips)
    ws = Banded(V.vt_workspace_bytes(tw.h, B, grid))
    out = Banded(B * (N // 4) * cfg["proj_out"] * 2)
    tower = Banded(B * N * cfg["hidden"] * 2)
    V.vt_forward_video(tw.h, pin.typed(torch.float32, *clips.shape), F, grid, B,
                       out.typed(torch.bfloat16, B, N // 4, -1), tower.typed(torch.bfloat16, B, N, -1), ws.body,
                       ws.nbytes)
    V.vt_check()
    for b, what in ((ws, "workspace"), (out, "projected tokens"), (tower, "tower output")):
        b.check(f"vt_forward_video: {what}")
    unchanged(pin, clips, "vt_forward_video: clips")
    tw.close()


def test_forward_u8_guard_bands():
    tw, cfg = _tower("tiny")
    sizes = [(37, 53), (200, 150), (84, 140)]
    images = S.make_images_u8(sizes, seed=50)
    raw = np.concatenate([im.ravel() for im in images])
    pin = banded_from(raw)
    grid, B = (1, 6, 10), len(sizes)
    N = grid[1] * grid[2]
    ws = Banded(V.vt_workspace_bytes(tw.h, B, grid))
    out = Banded(B * (N // 4) * cfg["proj_out"] * 2)
    V.vt_forward_u8(tw.h, pin.body, sizes, grid, out.typed(torch.bfloat16, B, N // 4, -1), None, ws.body, ws.nbytes)
    V.vt_check()
    ws.check("vt_forward_u8: workspace")
    out.check("vt_forward_u8: projected tokens")
    unchanged(pin, raw, "vt_forward_u8: images")
    tw.close()


@pytest.mark.parametrize("B,H,N,D", [(2, 3, 77, 80), (1, 2, 300, 32), (1, 16, 1024, 80)])
def test_attention_guard_bands(B, H, N, D):
    q, k, v = S.make_qkv(B, H, N, D, 60 + N)
    qb, kb, vb = banded_from(q), banded_from(k), banded_from(v)
    o = Banded(B * N * H * D * 2)
    ws = Banded(V.vt_attention_workspace_bytes(B, H, N, D))
    shape = (B, H, N, D)
    args = (qb.typed(torch.bfloat16, *shape), kb.typed(torch.bfloat16, *shape), vb.typed(torch.bfloat16, *shape))
    V.vt_attention(*args, o.typed(torch.bfloat16, B, N, H * D), B, H, N, D, None, None, 0.0, D ** -0.5, ws.body,
                   ws.nbytes)
    V.vt_check()
    ws.check(f"vt_attention {shape}: workspace")
    o.check(f"vt_attention {shape}: output")
    o2 = Banded(B * N * H * D * 2)
    V.vt_attention_static(*args, o2.typed(torch.bfloat16, B, N, H * D), B, H, N, D, None, None, 0.0, D ** -0.5)
    V.vt_check()
    o2.check(f"vt_attention_static {shape}: output")
    assert torch.equal(o.body, o2.body)
    for b, a, what in ((qb, q, "q"), (kb, k, "k"), (vb, v, "v")):
        unchanged(b, a, f"vt_attention {shape}: {what}")


def test_linear_split_k_guard_bands():
    # ragged split-K tail: 5 x 4 tiles of 256 on the pairs, K = 4104 (a partial K step)
    M, N, K = 1100, 1000, 4104
    A, W = S.make_matrix((M, K), 80), S.make_matrix((N, K), 81, 0.01)
    bias, resid = S.make_matrix((N,), 82, 0.1), S.make_matrix((M, N), 83)
    ab, wb, bb, rb = banded_from(A), banded_from(W), banded_from(bias), banded_from(resid)
    ws = Banded(V.vt_linear_workspace_bytes())
    out = Banded(M * N * 2)
    V.vt_linear_ws(ab.typed(torch.bfloat16, M, K), wb.typed(torch.bfloat16, N, K), bb.typed(torch.bfloat16, N),
                   rb.typed(torch.bfloat16, M, N), out.typed(torch.bfloat16, M, N), M, N, K, 0, ws.body, ws.nbytes)
    V.vt_check()
    ws.check("vt_linear_ws: split-K scratch")
    out.check("vt_linear_ws: output")
    for b, a, what in ((ab, A, "A"), (wb, W, "W"), (bb, bias, "bias"), (rb, resid, "resid")):
        unchanged(b, a, f"vt_linear_ws: {what}")


def test_backward_guard_bands():
    tw, cfg = _tower("tiny")
    V.vt_enable_backward(tw.h)
    hw, B = (84, 140), 2
    grid = (1, hw[0] // 14, hw[1] // 14)
    N = grid[1] * grid[2]
    px = S.make_pixels(dict(cfg, image=hw), batch=B, seed=70)
    d_tower = S.make_matrix((B, N, cfg["hidden"]), 71)
    pin, dtin = banded_from(px), banded_from(d_tower)
    saved_bytes, ws_bytes = V.vt_backward_bytes(tw.h, B, grid)
    saved, ws = Banded(saved_bytes), Banded(ws_bytes)
    tower = Banded(B * N * cfg["hidden"] * 2)
    dpx = Banded(px.nbytes)
    V.vt_forward_saved(tw.h, pin.typed(torch.float32, *px.shape), grid, B, tower.typed(torch.bfloat16, B, N, -1),
                       saved.body, saved.nbytes, ws.body, ws.nbytes)
    V.vt_backward(tw.h, saved.body, grid, B, dtin.typed(torch.bfloat16, B, N, -1),
                  dpx.typed(torch.float32, *px.shape), ws.body, ws.nbytes)
    V.vt_check()
    for b, what in ((saved, "saved activations"), (ws, "workspace"), (tower, "tower output"),
                    (dpx, "pixel gradient")):
        b.check(f"vt_forward_saved + vt_backward: {what}")
    unchanged(pin, px, "vt_forward_saved: pixels")
    unchanged(dtin, d_tower, "vt_backward: tower gradient")
    # the single-layer backward entry point, on its own workspace
    lws = Banded(V.vt_tower_layer_backward_bytes(tw.h, B, grid))
    x = S.make_matrix((B, N, cfg["hidden"]), 72)
    xin = banded_from(x)
    dx = Banded(B * N * cfg["hidden"] * 2)
    V.vt_tower_layer_backward(tw.h, 1, xin.typed(torch.bfloat16, B, N, -1), dtin.typed(torch.bfloat16, B, N, -1),
                              dx.typed(torch.bfloat16, B, N, -1), grid, B, lws.body, lws.nbytes)
    V.vt_check()
    lws.check("vt_tower_layer_backward: workspace")
    dx.check("vt_tower_layer_backward: dx")
    unchanged(xin, x, "vt_tower_layer_backward: x_in")
    tw.close()

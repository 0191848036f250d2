"""Video clips on the GPU: vt_forward_video on clips of F frames (T = ceil(F/2)
temporal patches, the last frame repeated when F is odd), compared with the fp64
oracle's forward_video (tower output <= 1e-2, projected tokens <= 2e-2 relative L2),
plus the exact reductions to the still-image path and the argument checks."""
import numpy as np
import pytest
import torch

from oracle import vit_ref as R
from vision_transformer_encoder_vit_b200 import synthetic as S
from tests.gpu_util import REL_L2_FINAL, REL_L2_LAYER, assert_close, empty_bf16, host_bits, host_f64

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from vision_transformer_encoder_vit_b200 import vt as V


def _forward_video(tw, c, clips):
    B, F, _, H, W = clips.shape
    grid = (-(-F // c["temporal_patch"]), H // c["patch"], W // c["patch"])
    N = grid[0] * grid[1] * grid[2]
    ws = tw.workspace(B, grid)
    out = empty_bf16(B, N // 4, c["proj_out"])
    tower = empty_bf16(B, N, c["hidden"])
    V.vt_forward_video(tw.h, torch.from_numpy(clips).cuda(), F, grid, B, out, tower, ws, ws.numel())
    V.vt_check()
    return out, tower


def _run(cfg, frames, hw, batch, affine, layers=None):
    bits = S.make_weights(cfg, affine=affine, layers=layers)
    c = dict(cfg, image=hw)
    if layers is not None:
        c["layers"] = layers
    tw = V.Tower(c, bits)
    clips = S.make_clips(c, frames, batch=batch, seed=5 + frames)
    out, tower = _forward_video(tw, c, clips)
    ref = R.forward_video(clips.astype(np.float64), S.weights_f64(bits), c)
    assert_close(host_f64(tower), ref["tower"], rel=REL_L2_LAYER, what=f"video tower F={frames} {hw}")
    assert_close(host_f64(out), ref["out"], rel=REL_L2_FINAL, what=f"video projected F={frames} {hw}")
    tw.close()


@pytest.mark.parametrize("frames,hw", [(3, (56, 84)), (4, (84, 56)), (5, (28, 56)), (2, (112, 112))])
def test_video_tiny_clips(frames, hw):
    # odd F repeats the last frame; T = 2 or 3 slices of the grid in one sequence
    _run(S.get_config("tiny"), frames, hw, batch=2, affine=True)


def test_video_full_width_two_layers():
    # 8 frames at 224^2: T = 4 slices of 16x16 patches, 1024 tokens per clip
    _run(S.get_config("tower448"), 8, (224, 224), batch=1, affine=False, layers=2)


def test_one_frame_clip_is_the_still_image_bit_for_bit():
    cfg = S.get_config("tiny")
    bits = S.make_weights(cfg, affine=True)
    tw = V.Tower(cfg, bits)
    px = S.make_pixels(cfg, batch=2)
    grid = (1, px.shape[2] // 14, px.shape[3] // 14)
    ws = tw.workspace(2, grid)
    out_i = empty_bf16(2, grid[1] * grid[2] // 4, cfg["proj_out"])
    V.vt_forward(tw.h, torch.from_numpy(px).cuda(), grid, 2, out_i, None, ws, ws.numel())
    for frames in (1, 2):  # one frame, or the frame given twice: the same Conv3d input
        clips = np.ascontiguousarray(np.repeat(px[:, None], frames, axis=1))
        out_v, _ = _forward_video(tw, cfg, clips)
        np.testing.assert_array_equal(host_bits(out_v), host_bits(out_i))
    tw.close()


def test_frame_count_must_match_grid():
    cfg = S.get_config("tiny")
    tw = V.Tower(cfg, S.make_weights(cfg, affine=True))
    clips = torch.zeros(1, 4, 3, 56, 56, device="cuda")
    ws = tw.workspace(1, (3, 4, 4))
    out = empty_bf16(1, 12, cfg["proj_out"])
    with pytest.raises(V.VtError) as e:
        V.vt_forward_video(tw.h, clips, 4, (3, 4, 4), 1, out, None, ws, ws.numel())
    assert e.value.name == "VT_ERR_SHAPE"
    with pytest.raises(V.VtError) as e:
        V.vt_forward(tw.h, clips, (2, 4, 4), 1, out, None, ws, ws.numel())
    assert e.value.name == "VT_ERR_SHAPE"
    with pytest.raises(V.VtError) as e:
        V.vt_forward_video(tw.h, clips, 0, (1, 4, 4), 1, out, None, ws, ws.numel())
    assert e.value.name == "VT_ERR_INVALID_ARG"
    tw.close()

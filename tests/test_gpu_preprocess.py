"""GPU preprocessing: decoded 8-bit images resized (bicubic), scaled and normalised on
the device, against the fp64 oracle's preprocess; and the fused forward from decoded
images against the forward from those pixels.

Tolerance of the pixels: the kernel sums at most 65 + 65 fp32 products of weights
(|w| <= 1, summing to 1) and 8-bit values, each rounding costing at most 2^-24
relative, so the resized value v (|v| < 400) is off by well under 130 * 400 * 2^-24
~= 3e-3; after /255 and /std (std >= 0.26) that is below 5e-5.  The test allows 1e-4.
"""
import numpy as np
import pytest
import torch

from oracle import vit_ref as R
from vision_transformer_encoder_vit_b200 import synthetic as S
from tests.gpu_util import REL_L2_FINAL, REL_L2_LAYER, assert_close, empty_bf16, host_bits, host_f64, report

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from vision_transformer_encoder_vit_b200 import vt as V

PIX_ATOL = 1e-4


def _dev_images(images):
    return torch.from_numpy(np.concatenate([im.ravel() for im in images])).cuda()


def _preprocess(h, images, grid, patch=14, mean=None, std=None):
    px = torch.empty((len(images), 3, grid[1] * patch, grid[2] * patch), dtype=torch.float32, device="cuda")
    V.vt_preprocess(h, _dev_images(images), [im.shape[:2] for im in images], grid, px, mean=mean, std=std)
    V.vt_check()
    return px


def _oracle_pixels(images, grid, patch=14, mean=S.CLIP_MEAN, std=S.CLIP_STD):
    return np.stack([R.preprocess(im, grid[1] * patch, grid[2] * patch, mean, std) for im in images])


@pytest.mark.parametrize("grid,sizes", [
    ((1, 4, 6), [(56, 84), (30, 41), (200, 333), (7, 5), (1, 1), (896, 1344)]),  # equal, up, down, 16x down
    ((1, 2, 2), [(28, 28), (27, 29), (448, 17)]),
    ((1, 48, 48), [(1080, 1920), (480, 640), (672, 672)]),                       # the pages' 672 x 672
])
def test_preprocess_equals_oracle(grid, sizes):
    cfg = S.get_config("tiny")
    h = V.vt_create(cfg)
    images = S.make_images_u8(sizes, seed=len(sizes))
    got = _preprocess(h, images, grid).cpu().numpy().astype(np.float64)
    ref = _oracle_pixels(images, grid)
    err = np.abs(got - ref).max()
    report("preprocess", grid=list(grid), sizes=[list(s) for s in sizes], max_abs=float(err))
    assert err <= PIX_ATOL, err
    V.vt_destroy(h)


def test_preprocess_custom_statistics_and_many_images():
    # 70 images: two launch tables (64 + 6), ImageNet statistics instead of CLIP's
    cfg = S.get_config("tiny")
    h = V.vt_create(cfg)
    r = np.random.default_rng(3)
    sizes = [(int(a), int(b)) for a, b in r.integers(3, 120, size=(70, 2))]
    images = S.make_images_u8(sizes, seed=9)
    grid = (1, 2, 4)
    got = _preprocess(h, images, grid, mean=S.IMAGENET_MEAN, std=S.IMAGENET_STD).cpu().numpy()
    ref = _oracle_pixels(images, grid, mean=S.IMAGENET_MEAN, std=S.IMAGENET_STD)
    assert np.abs(got - ref).max() <= PIX_ATOL
    V.vt_destroy(h)


def _forward_both(tw, cfg, images, grid):
    B = len(images)
    N = grid[1] * grid[2]
    ws = tw.workspace(B, grid)
    out_u8 = empty_bf16(B, N // 4, cfg["proj_out"])
    tower_u8 = empty_bf16(B, N, cfg["hidden"])
    V.vt_forward_u8(tw.h, _dev_images(images), [im.shape[:2] for im in images], grid, out_u8, tower_u8, ws,
                    ws.numel())
    px = _preprocess(tw.h, images, grid)
    out_px = empty_bf16(B, N // 4, cfg["proj_out"])
    V.vt_forward(tw.h, px, grid, B, out_px, None, ws, ws.numel())
    V.vt_check()
    return out_u8, tower_u8, out_px, px


def test_forward_from_decoded_images_tiny():
    cfg = S.get_config("tiny")
    bits = S.make_weights(cfg, affine=True)
    tw = V.Tower(cfg, bits)
    images = S.make_images_u8([(150, 90), (56, 56), (40, 70), (300, 300)], seed=4)
    grid = (1, 4, 4)
    out_u8, tower_u8, out_px, _ = _forward_both(tw, cfg, images, grid)
    # the fused path equals the two-step path bit for bit
    np.testing.assert_array_equal(host_bits(out_u8), host_bits(out_px))
    # and the oracle forward of the oracle's pixels
    ref = R.forward(_oracle_pixels(images, grid), S.weights_f64(bits), dict(cfg, image=(56, 56)))
    assert_close(host_f64(tower_u8), ref["tower"], rel=REL_L2_LAYER, what="u8 forward tower")
    assert_close(host_f64(out_u8), ref["out"], rel=REL_L2_FINAL, what="u8 forward projected")
    tw.close()


def test_forward_from_decoded_images_full_672():
    # full 32-layer tower at the pages' 672 x 672 preprocessing: fused path == two-step path
    cfg = dict(S.get_config("tower448"), image=(672, 672))
    tw = V.Tower(cfg, S.make_weights(cfg))
    images = S.make_images_u8([(1080, 1920), (480, 640)], seed=5)
    out_u8, _, out_px, px = _forward_both(tw, cfg, images, (1, 48, 48))
    np.testing.assert_array_equal(host_bits(out_u8), host_bits(out_px))
    assert np.abs(px.cpu().numpy() - _oracle_pixels(images, (1, 48, 48))).max() <= PIX_ATOL
    tw.close()

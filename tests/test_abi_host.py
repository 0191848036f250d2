"""Host-side checks of the C ABI that need no GPU: the library loads and exports every
symbol include/vt.h declares, configuration and argument checks return the documented
status codes, the workspace plan is affine in the token count, and the index maps
(2x2-block token order, RoPE positions, merge gather) equal the oracle's exactly.
"""
import os
import re

import numpy as np
import pytest

from oracle import vit_ref as R
from vision_transformer_encoder_vit_b200 import synthetic as S
from vision_transformer_encoder_vit_b200 import vt as V

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "vt.h")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^VT_API\s+[\w\s\*]+?\b(vt_\w+)\s*\(", text, flags=re.M)))


def test_every_declared_symbol_is_exported_and_bound():
    names = _declared()
    assert len(names) >= 20
    for n in names:
        assert hasattr(V.lib, n), f"{n} missing from libvt.so"
        assert n in V.EXPORTED, f"{n} has no binding"


def _status(e):
    return e.value.name


def test_create_validates_config():
    cfg = S.get_config("tower448")
    h = V.vt_create(cfg)
    V.vt_destroy(h)
    bad = [
        dict(heads=15),                      # heads * head_dim != hidden
        dict(rope_sections=(16, 32, 30)),    # does not sum to head_dim
        dict(rope_sections=(15, 33, 32)),    # odd section
        dict(mlp=0),
    ]
    for b in bad:
        with pytest.raises(V.VtError) as e:
            V.vt_create(dict(cfg, **b))
        assert _status(e) == "VT_ERR_INVALID_ARG", b
    for b in (dict(merge=3), dict(head_dim=64, heads=20, rope_sections=(16, 24, 24))):
        with pytest.raises(V.VtError) as e:
            V.vt_create(dict(cfg, **b))
        assert _status(e) == "VT_ERR_UNSUPPORTED", b


def test_forward_before_load_and_grid_errors():
    h = V.vt_create(S.get_config("tiny"))
    with pytest.raises(V.VtError) as e:
        V.vt_forward(h, 16, (1, 8, 8), 1, 16, None, 16, 1 << 20)
    assert _status(e) == "VT_ERR_NOT_LOADED"
    for grid, code in [((1, 7, 8), "VT_ERR_SHAPE"), ((4097, 8, 8), "VT_ERR_SHAPE"),
                       ((1, 8, 8194), "VT_ERR_SHAPE"), ((0, 8, 8), "VT_ERR_INVALID_ARG")]:
        with pytest.raises(V.VtError) as e:
            V.vt_workspace_bytes(h, 1, grid)
        assert _status(e) == code, grid
    with pytest.raises(V.VtError) as e:
        V.vt_workspace_bytes(h, 0, (1, 8, 8))
    assert _status(e) == "VT_ERR_INVALID_ARG"
    V.vt_destroy(h)


def test_load_weights_rejects_missing_names_without_touching_the_device():
    h = V.vt_create(S.get_config("tiny"))
    with pytest.raises(V.VtError) as e:
        V.vt_load_weights(h, {})
    assert _status(e) == "VT_ERR_WEIGHT"
    assert "embeddings.proj.weight" in str(e.value)
    V.vt_destroy(h)


def test_linear_and_attention_argument_checks():
    with pytest.raises(V.VtError) as e:
        V.vt_linear(16, 16, None, None, 16, 4, 12, 16, 0)  # N not a multiple of 8
    assert _status(e) == "VT_ERR_INVALID_ARG"
    with pytest.raises(V.VtError) as e:
        V.vt_linear(16, 16, None, None, 16, 4, 16, 16, 3)
    assert _status(e) == "VT_ERR_INVALID_ARG"
    with pytest.raises(V.VtError) as e:
        V.vt_attention_prepared(16, 16, 16, 8, 16, 1, 1, 8, 48, 0.1)
    assert _status(e) == "VT_ERR_UNSUPPORTED"
    with pytest.raises(V.VtError) as e:
        V.vt_attention_prepared(16, 16, 16, 4, 16, 1, 1, 8, 80, 0.1)  # ld_vt < N
    assert _status(e) == "VT_ERR_INVALID_ARG"
    with pytest.raises(V.VtError) as e:
        V.vt_attention(16, 16, 16, 16, 1, 2, 8, 80, 16, (16, 32, 30), 1e4, 0.1, 16, 1 << 30)
    assert _status(e) == "VT_ERR_INVALID_ARG"


@pytest.mark.parametrize("grid", [(1, 2, 2), (1, 4, 6), (1, 8, 8), (1, 32, 32), (1, 6, 2)])
def test_index_maps_equal_oracle(grid):
    order, pos, merge = V.vt_index_maps(grid)
    np.testing.assert_array_equal(np.asarray(order), R.block_order(*grid))
    np.testing.assert_array_equal(np.asarray(pos), R.positions_raster(*grid))
    np.testing.assert_array_equal(np.asarray(merge), R.merge_source_map(*grid))


def test_workspace_is_affine_in_tokens():
    cfg = S.get_config("tower448")
    h = V.vt_create(cfg)
    sizes = {}
    for side in (2, 4, 8, 16, 32, 64, 80, 128, 144, 256):
        sizes[side * side] = V.vt_workspace_bytes(h, 1, (1, side, side))
    ns = np.array(sorted(sizes))
    ws = np.array([sizes[n] for n in ns], dtype=np.float64)
    # fit ws = a + b * N on the large sizes; every size lies within the per-buffer
    # 256-byte rounding of that line (no N^2 term)
    b = (ws[-1] - ws[-3]) / (ns[-1] - ns[-3])
    a = ws[-1] - b * ns[-1]
    assert np.all(np.abs(ws - (a + b * ns)) <= 16 * 256), (a, b)
    # the constant part is the linear layers' split-K scratch: one 256 x 256 fp32 tile
    # per pair of SMs (the host falls back to 148 SMs without a device)
    assert 0 < a <= 74 * 256 * 256 * 4 + 16 * 256
    # per token: the residual stream x (2d bytes) plus the larger of the tower phase
    # (LN out, q, k, v^T, o: 5 x 2d, MLP hidden 2m) and the projector phase (two
    # P-wide activations and a quarter-row merged hidden: 2P + 2P + 2P/4)
    d, m, P = 1280, 5120, 6144
    assert b == pytest.approx(2 * d + max(5 * 2 * d + 2 * m, 2 * P + 2 * P + 2 * P / 4), rel=0.01)
    # the pages' untiled attention alone needs 6 N^2 bytes for scores + probabilities
    # (25.8 GB at 65536 tokens); the whole forward's workspace here is under 2 GB
    assert sizes[256 * 256] < 6 * (256 * 256) ** 2 / 10
    # batch scales the same way
    assert V.vt_workspace_bytes(h, 8, (1, 32, 32)) <= 8 * sizes[1024] + 16 * 256
    V.vt_destroy(h)


def test_varlen_workspace_and_argument_checks():
    cfg = S.get_config("tower448")
    h = V.vt_create(cfg)
    one = V.vt_workspace_bytes(h, 1, (1, 32, 32))
    assert V.vt_workspace_bytes_varlen(h, [(1, 32, 32)]) == one
    mixed = V.vt_workspace_bytes_varlen(h, [(1, 32, 32), (1, 16, 24), (1, 2, 2)])
    tokens = 1024 + 384 + 4
    # affine in the packed token count: the fixed split-K scratch plus 30208 bytes per token
    fixed = one - 30208 * 1024
    assert 0 < fixed <= 74 * 256 * 256 * 4 + 16 * 256
    assert one < mixed <= fixed + 30208 * tokens + 64 * 256
    with pytest.raises(V.VtError) as e:
        V.vt_workspace_bytes_varlen(h, [(1, 32, 32), (1, 15, 24)])
    assert _status(e) == "VT_ERR_SHAPE"
    with pytest.raises(V.VtError) as e:  # clips go through vt_forward_video
        V.vt_workspace_bytes_varlen(h, [(1, 32, 32), (2, 16, 24)])
    assert _status(e) == "VT_ERR_SHAPE"
    with pytest.raises(V.VtError) as e:
        V.vt_workspace_bytes_varlen(h, [(1, 2, 2)] * 65)
    assert _status(e) == "VT_ERR_INVALID_ARG"
    with pytest.raises(V.VtError) as e:
        V.vt_forward_varlen(h, 16, [(1, 2, 2)], 16, None, 16, 1 << 20)
    assert _status(e) == "VT_ERR_NOT_LOADED"
    V.vt_destroy(h)


def test_video_workspace_counts_every_temporal_patch():
    """A clip of grid (t, h, w) is one sequence of t*h*w tokens: its plan equals a still
    image of the same token count, and the still-image entry points refuse t > 1."""
    h = V.vt_create(S.get_config("tower448"))
    for t, gh, gw in [(2, 8, 8), (3, 16, 24), (8, 32, 32)]:
        assert V.vt_workspace_bytes(h, 2, (t, gh, gw)) == V.vt_workspace_bytes(h, 2, (1, gh, t * gw))
    with pytest.raises(V.VtError) as e:
        V.vt_forward_host_workspace_bytes(h, 1, (2, 8, 8))
    assert _status(e) == "VT_ERR_SHAPE"
    with pytest.raises(V.VtError) as e:
        V.vt_forward_video(h, 16, 4, (2, 8, 8), 1, 16, None, 16, 1 << 20)
    assert _status(e) == "VT_ERR_NOT_LOADED"
    V.vt_destroy(h)


def test_attention_workspace_linear():
    s1 = V.vt_attention_workspace_bytes(1, 16, 6400, 80)
    s2 = V.vt_attention_workspace_bytes(1, 16, 65536, 80)
    assert s1 == 3 * 16 * 80 * 6400 * 2
    assert s2 == 3 * 16 * 80 * 65536 * 2
    assert V.vt_attention_workspace_bytes(1, 1, 5, 80) == 3 * 80 * 8 * 2  # ragged N rounds to 8 columns


def test_last_error_message_is_thread_local_string():
    with pytest.raises(V.VtError):
        V.vt_linear(None, 16, None, None, 16, 4, 16, 16, 0)
    assert "NULL" in V.vt_last_error()


def test_preprocess_argument_checks_need_no_device():
    h = V.vt_create(S.get_config("tiny"))
    grid = (1, 4, 4)  # 56 x 56 target
    for src, code in [([(900, 56)], "VT_ERR_SHAPE"),       # more than 16x the target height
                      ([(56, 897)], "VT_ERR_SHAPE"),
                      ([(0, 56)], "VT_ERR_INVALID_ARG")]:
        with pytest.raises(V.VtError) as e:
            V.vt_preprocess(h, 16, src, grid, 16)
        assert _status(e) == code, src
    with pytest.raises(V.VtError) as e:
        V.vt_preprocess(h, 16, [(56, 56)], grid, 16, mean=(0.5, 0.5, 0.5), std=(0.2, 0.0, 0.2))
    assert _status(e) == "VT_ERR_INVALID_ARG"
    with pytest.raises(V.VtError) as e:
        V.vt_preprocess(h, 16, [(56, 56)], (2, 4, 4), 16)
    assert _status(e) == "VT_ERR_SHAPE"
    with pytest.raises(V.VtError) as e:
        V.vt_forward_u8(h, 16, [(56, 56)], grid, 16, None, 16, 1 << 20)
    assert _status(e) == "VT_ERR_NOT_LOADED"
    V.vt_destroy(h)


def test_backward_argument_checks_need_no_device():
    # v^T [B, H, D, ceil8(N)], the recomputed output [B*N, H*D], log-sum-exp and delta
    # [B*H, ceil64(N)] fp32: linear in N, no N^2 term
    assert V.vt_attention_backward_workspace_bytes(2, 16, 100, 80) == \
        (2 * 16 * 80 * 104 * 2 + 255) // 256 * 256 + (2 * 100 * 16 * 80 * 2 + 255) // 256 * 256 + \
        2 * ((2 * 16 * 128 * 4 + 255) // 256 * 256)
    for D, code in ((64, "VT_ERR_UNSUPPORTED"), (80, "VT_ERR_WORKSPACE")):
        with pytest.raises(V.VtError) as e:
            V.vt_attention_backward(16, 16, 16, 16, 16, 1, 2, 100, D, 0.1, 16, 1024)
        assert _status(e) == code
    with pytest.raises(V.VtError) as e:
        V.vt_layernorm_backward(16, 16, 16, 16, 16, 4, 1281, 1e-6)
    assert _status(e) == "VT_ERR_INVALID_ARG"
    h = V.vt_create(S.get_config("tower448"))
    saved, ws = V.vt_backward_bytes(h, 2, (1, 32, 32))
    # per layer: input, q, k, v^T, attention output, mid residual (6 x [M, 1280] bf16),
    # MLP pre-activation [M, 5120] bf16, log-sum-exp [B*H, 1024] fp32; M = 2048 tokens
    assert saved == 32 * (6 * 2048 * 1280 * 2 + 2048 * 5120 * 2 + 2 * 16 * 1024 * 4)
    assert ws >= V.vt_workspace_bytes(h, 2, (1, 32, 32))
    with pytest.raises(V.VtError) as e:
        V.vt_backward_bytes(h, 1, (2, 8, 8))
    assert _status(e) == "VT_ERR_SHAPE"
    with pytest.raises(V.VtError) as e:
        V.vt_enable_backward(h)
    assert _status(e) == "VT_ERR_NOT_LOADED"
    V.vt_destroy(h)


_TRACE_CALL = """
from vision_transformer_encoder_vit_b200 import vt as V
try:
    V.vt_linear(256, 512, None, None, 1024, 8, 16, 16, 0)
except V.VtError as e:
    print('status', e)
"""


def _cuda_visible():
    import torch
    return torch.cuda.is_available()


# Only on a machine without a CUDA device: the call passes the host checks with
# placeholder addresses and its launch then fails for want of a device, after the trace
# line is written.  Where a device exists the addresses would be real, so it is skipped.
@pytest.mark.skipif(_cuda_visible(), reason="placeholder addresses are only safe without a CUDA device")
def test_launch_trace_follows_vt_log():
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, VT_LOG="1")
    r = subprocess.run([sys.executable, "-c", _TRACE_CALL], cwd=root, env=env, capture_output=True, text=True,
                       timeout=120)
    assert "vt: launch gemm flops=4096 bytes=0" in r.stderr, r.stderr
    assert "VT_ERR_CUDA" in r.stdout
    for off in ("0", ""):
        env = dict(os.environ, VT_LOG=off)
        r = subprocess.run([sys.executable, "-c", _TRACE_CALL], cwd=root, env=env, capture_output=True, text=True,
                           timeout=120)
        assert "vt: launch" not in r.stderr


def test_static_attention_limit_is_exact_on_the_host():
    # vt_attention_static needs 3 * align256(B*H*D*ceil8(N)*2) bytes of its 32 MiB array.
    # The largest accepted single part is 11184640 bytes (43690 * 256): D = 80, one head,
    # N = 69904 tokens.  One token more rounds up to 69912 and must be rejected before
    # anything touches the device (so fake, aligned pointers are safe here).
    limit = V.vt_attention_static_max_bytes()
    assert limit == 32 << 20
    assert V.vt_attention_workspace_bytes(1, 1, 69904, 80) == 3 * 11184640 <= limit
    assert V.vt_attention_workspace_bytes(1, 1, 69905, 80) > limit
    fake = 1 << 20
    for N in (69905, 69912, 1 << 20):
        with pytest.raises(V.VtError) as e:
            V.vt_attention_static(fake, fake, fake, fake, 1, 1, N, 80, None, None, 0.0, 80 ** -0.5)
        assert _status(e) == "VT_ERR_WORKSPACE"
    # the row limit of the workspace entry point holds here too (B * H * N < 2^31)
    with pytest.raises(V.VtError) as e:
        V.vt_attention_static(fake, fake, fake, fake, 1 << 25, 1 << 25, 256, 32, None, None, 0.0, 32 ** -0.5)
    assert _status(e) == "VT_ERR_SHAPE"

"""vt_attention_static: attention for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc or give the library a workspace (for example a
plugin inside a host framework that owns every device allocation).  This entry point
keeps its scratch in a fixed array compiled into the library.  The test calls it
through the C ABI twice in a row and checks each result against vt_attention (the
entry point that takes a caller workspace) with the same tolerance as the other
attention parity tests.  The file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

from vision_transformer_encoder_vit_b200 import synthetic as S
from tests.gpu_util import assert_close, dev_bf16, empty_bf16, host_f64

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from vision_transformer_encoder_vit_b200 import vt as V


def _reference(q, k, v, B, H, N, D, pos, sections):
    o = empty_bf16(B, N, H * D)
    ws_bytes = V.vt_attention_workspace_bytes(B, H, N, D)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    V.vt_attention(q, k, v, o, B, H, N, D, pos, sections, 10000.0, D ** -0.5, ws, ws_bytes)
    return host_f64(o)


def test_static_scratch_attention_matches_workspace_attention_twice():
    cases = [
        (1, 16, 1024, 80, True),   # one 448x448 image's attention, 3D RoPE on a 32x32 grid
        (2, 4, 300, 32, False),    # a different shape second, so stale contents would show
    ]
    for B, H, N, D, rope in cases:
        q, k, v = (dev_bf16(a) for a in S.make_qkv(B, H, N, D, N + D))
        pos, sections = None, None
        if rope:
            side = int(round(N ** 0.5))
            grid = np.stack(np.meshgrid(np.zeros(1), np.arange(side), np.arange(side), indexing="ij"), -1)
            pos = torch.from_numpy(grid.reshape(-1, 3).astype(np.int32)).cuda()
            sections = (16, 32, 32)
        ref = _reference(q, k, v, B, H, N, D, pos, sections)
        for call in range(2):
            o = empty_bf16(B, N, H * D)
            o.fill_(float("nan"))
            V.vt_attention_static(q, k, v, o, B, H, N, D, pos, sections, 10000.0, D ** -0.5)
            V.vt_check()
            assert_close(host_f64(o), ref, what=f"static-scratch attention B{B} H{H} N{N} D{D} call {call}")


def test_static_scratch_rejects_oversized_problem():
    limit = V.vt_attention_static_max_bytes()
    assert limit == 32 << 20
    N = 16384  # 3 * 16 * 80 * 16384 * 2 bytes = 126 MB > 32 MiB
    q = empty_bf16(1, 16, 8, 80)  # never read: the size check fails first
    with pytest.raises(V.VtError) as e:
        V.vt_attention_static(q, q, q, q, 1, 16, N, 80, None, None, 0.0, 80 ** -0.5)
    assert e.value.name == "VT_ERR_WORKSPACE"


def test_static_scratch_accepts_the_exact_limit():
    # The largest problem the array holds: D = 80, one head, N = 69904 tokens, i.e.
    # 3 parts of 11184640 bytes (43690 * 256), within 32 MiB.  It runs and matches
    # vt_attention; one token more (69905, rounded up to 69912) is rejected.
    B, H, N, D = 1, 1, 69904, 80
    q, k, v = (dev_bf16(a) for a in S.make_qkv(B, H, N, D, 7))
    ref = _reference(q, k, v, B, H, N, D, None, None)
    o = empty_bf16(B, N, H * D)
    V.vt_attention_static(q, k, v, o, B, H, N, D, None, None, 0.0, D ** -0.5)
    V.vt_check()
    assert_close(host_f64(o), ref, what="static-scratch attention at the exact size limit")
    q1 = empty_bf16(B, H, N + 1, D)
    with pytest.raises(V.VtError) as e:
        V.vt_attention_static(q1, q1, q1, q1, B, H, N + 1, D, None, None, 0.0, D ** -0.5)
    assert e.value.name == "VT_ERR_WORKSPACE"

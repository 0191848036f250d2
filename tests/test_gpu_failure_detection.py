"""Failure detection on the GPU without a fault: a kernel wait that nothing can
satisfy gives up after its bound, the host reads VT_ERR_TIMEOUT through vt_check, the
error is cleared, and the context keeps working (a GEMM run afterwards is correct)."""
import time

import numpy as np
import pytest
import torch

from vision_transformer_encoder_vit_b200 import synthetic as S
from tests.gpu_util import assert_close, dev_bf16, empty_bf16, host_f64

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from vision_transformer_encoder_vit_b200 import vt as V


def test_wait_that_runs_out_is_reported_and_cleared():
    V.vt_check()  # nothing pending
    t0 = time.perf_counter()
    V.vt_selftest_wait_timeout()
    with pytest.raises(V.VtError) as e:
        V.vt_check()
    elapsed = time.perf_counter() - t0
    assert e.value.name == "VT_ERR_TIMEOUT"
    assert "self-test" in str(e.value)
    assert 0.5 < elapsed < 30.0  # the bound is 1 s of GPU global time
    V.vt_check()  # cleared
    # the context is still usable
    M, N, K = 256, 512, 128
    A, W = S.make_matrix((M, K), 1), S.make_matrix((N, K), 2, 0.05)
    out = empty_bf16(M, N)
    V.vt_linear(dev_bf16(A), dev_bf16(W), None, None, out, M, N, K, 0)
    V.vt_check()
    assert_close(host_f64(out), S.bf16_to_f64(A) @ S.bf16_to_f64(W).T, what="GEMM after a reported timeout")

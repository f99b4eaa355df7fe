"""Failure detection without a GPU fault: a kernel waits on a barrier that nothing
arrives on, through the bounded wait every pipelined kernel uses; it must give up,
latch ZDIT_ERR_DEVICE_TIMEOUT and leave the context usable."""
import numpy as np
import pytest
import torch

import stream_diffusion_transformer_s3_b200 as Z
from stream_diffusion_transformer_s3_b200 import synth
from _gpu import bf16, host, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()


def test_bounded_wait_times_out_and_context_survives():
    assert Z.zdit_device_status() == 0
    res = torch.zeros(1, dtype=torch.int32, device="cuda")
    Z.zdit_selftest_wait_timeout(res)
    assert Z.zdit_device_status() == -7  # ZDIT_ERR_DEVICE_TIMEOUT, latched then cleared
    assert int(res.item()) == 2          # the wait gave up (did not succeed)
    assert Z.zdit_device_status() == 0   # cleared
    # the context still runs the tensor-core path correctly
    rng = np.random.default_rng(0)
    A = synth.bf16_round(rng.standard_normal((300, 256), dtype=np.float32))
    B = synth.bf16_round(rng.standard_normal((512, 256), dtype=np.float32))
    out = torch.empty(300, 512, device="cuda")
    Z.zdit_gemm_bf16(bf16(A), bf16(B), out)
    assert Z.zdit_device_status() == 0
    ref = A.astype(np.float64) @ B.astype(np.float64).T
    assert np.linalg.norm(host(out) - ref) / np.linalg.norm(ref) < 1e-5

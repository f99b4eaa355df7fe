"""Stack-level parity on the GPU: zdit_stack_forward (embedders, noise and context
refiners, joint main blocks, final layer) against the oracle's stack_forward."""
import numpy as np
import pytest
import torch

import oracle as O
import stream_diffusion_transformer_s3_b200 as Z
from stream_diffusion_transformer_s3_b200 import synth
from _gpu import dev, dims_of, errors, host, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()


def run_stack(W, case, d, n_noise, n_ctx, n_main, cap_dim, flags=Z.F_ADALN | Z.F_SANDWICH_NORM):
    dims = dims_of(d)
    st = Z.DeviceStack(W, dims, n_noise, n_ctx, n_main, patch_dim=64, cap_dim=cap_dim, flags=flags)
    call = Z.StackCall(case["grid"], case["n_caps"], case["n_valids"], case["t"], dev(case["patches"]),
                       dev(case["caps"]))
    ws = torch.empty(Z.stack_workspace_bytes(st, call), dtype=torch.uint8, device="cuda")
    out = torch.full((len(case["n_caps"]), case["grid"][0] * case["grid"][1], 64), float("nan"), device="cuda")
    Z.zdit_stack_forward(st, call, out, ws)
    assert Z.zdit_device_status() == 0
    return host(out)


@pytest.mark.parametrize("n_caps,n_valids", [((64, 32), (45, 1)), ((32,), (0,))])
def test_small_stack_matches_oracle(n_caps, n_valids):
    d = synth.BlockDims(dim=256, n_heads=2, head_dim=128, ffn_hidden=384)
    W = synth.stack_weights(7, d, n_noise=1, n_context=1, n_main=2, cap_dim=128)
    case = synth.stack_case(7, 8, 8, list(n_caps), list(n_valids), [0.4] * len(n_caps), cap_dim=128)
    got = run_stack(W, case, d, 1, 1, 2, 128)
    ref = O.stack_forward(case, W, d)
    e = errors(got, ref)
    print("\nstack", e)
    assert e["rel_l2"] <= 2e-2, e


def test_full_width_stack_two_blocks_per_kind_256px():
    # full-width dims, 16x16 image grid, cond/uncond captions 64/32
    d = synth.FULL
    W = synth.stack_weights(3, d, n_noise=1, n_context=1, n_main=1)
    case = synth.stack_case(3, 16, 16, [64, 32], [45, 1], [0.25, 0.25])
    got = run_stack(W, case, d, 1, 1, 1, 2560)
    ref = O.stack_forward(case, W, d)
    e = errors(got, ref)
    print("\nstack full width", e)
    assert e["rel_l2"] <= 2e-2, e

"""zdit_block_forward_static: the block forward for callers that cannot allocate
device memory (a plugin whose host framework has reserved the GPU's memory for its
own pool, or a loop that must not pay cudaMalloc's device-wide synchronization).

Checks, through the C ABI on the GPU, that two calls in a row (sharing the library's
static scratch) give the same block output as zdit_block_forward with a caller
workspace, within the block-parity tolerance; that those two calls leave the device's
free memory unchanged (they allocate nothing); that a call of the most tokens the 40 MiB
scratch admits matches the workspace path too; and that a call too large for the scratch is
refused before any launch.  This file is collected last."""
import ctypes as C

import numpy as np
import pytest
import torch

import stream_diffusion_transformer_s3_b200 as Z
from stream_diffusion_transformer_s3_b200 import synth
from _gpu import N_ROUND_BLOCK, assert_parity, dev, dims_of, host, require_gpu, rope_tables

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()


def test_static_scratch_block_matches_workspace_block_twice():
    case = synth.config2(0)  # full width, cond/uncond 320 + 288 tokens (26.8 MiB of scratch)
    d = synth.FULL
    dims = dims_of(d)
    fl = Z.flags_of()
    w = Z.DeviceBlock(case["weights"])
    vl = Z.DeviceVarlen(case["cu_seqlens"])
    temb = dev(case["temb"])
    cs, sn = rope_tables(case["pos"], dims)

    x_ref = dev(case["x"])
    ws = torch.empty(Z.block_workspace_bytes(dims, fl, vl.total, 2), dtype=torch.uint8, device="cuda")
    Z.zdit_block_forward(dims, fl, w, vl, x_ref, temb, cs, sn, ws)
    assert Z.zdit_device_status() == 0
    ref = host(x_ref)

    # every device buffer of the measured calls exists before the free-memory reading;
    # one warm-up call loads the module that holds the scratch array
    x0 = dev(case["x"])
    xs = [torch.empty_like(x0) for _ in range(3)]
    xs[2].copy_(x0)
    Z.zdit_block_forward_static(dims, fl, w, vl, xs[2], temb, cs, sn)
    assert Z.zdit_device_status() == 0
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    for x in xs[:2]:  # the second call finds the first call's data in the scratch
        x.copy_(x0)
        Z.zdit_block_forward_static(dims, fl, w, vl, x, temb, cs, sn)
        assert Z.zdit_device_status() == 0
    torch.cuda.synchronize()
    free_after = torch.cuda.mem_get_info()[0]
    assert free_after == free_before, (free_before, free_after)
    for i, x in enumerate(xs[:2]):
        assert_parity(host(x), ref, TOL, base=case["x"], n_round=N_ROUND_BLOCK, label=f"static scratch, call {i + 1}")


def test_static_scratch_refuses_oversized_call():
    dims = Z.Dims()
    fl = Z.flags_of()
    T = 2048  # needs ~105 MiB of workspace at full width
    assert Z.block_workspace_bytes(dims, fl, T, 2) > (40 << 20)
    vl = Z.DeviceVarlen([0, 1024, T])
    cfg = dims.cfg(fl)
    wts = Z.BlockWeights(**{f: C.c_void_p(1 << 20) for f, _ in Z.BlockWeights._fields_})
    code = Z.lib().zdit_block_forward_static(C.byref(cfg), C.byref(wts), C.byref(vl.struct), C.c_void_p(1 << 20),
                                             C.c_void_p(1 << 20), C.c_void_p(1 << 20), C.c_void_p(1 << 20), None)
    assert code == -4  # ZDIT_ERR_WORKSPACE, nothing launched


def test_static_scratch_at_its_largest_admitted_size():
    # the most tokens whose workspace still fits the 40 MiB scratch at full width, in two branches
    dims = Z.Dims()
    fl = Z.flags_of()
    T = max(t for t in range(600, 1200) if Z.block_workspace_bytes(dims, fl, t, 2) <= (40 << 20))
    assert Z.block_workspace_bytes(dims, fl, T + 1, 2) > (40 << 20)
    d = synth.FULL
    n_img = 16 * 16
    lens = [T // 2, T - T // 2]
    rng = np.random.default_rng(0)
    x0 = (rng.standard_normal((T, d.dim)) * 3.0).astype(np.float32)
    cu = synth.cu_seqlens(lens)
    pos = np.concatenate([synth.branch_positions(16, 16, L - n_img)[:L] if L > n_img else
                          synth.branch_positions(16, 16, 0)[:L] for L in lens]).astype(np.int32)
    w = Z.DeviceBlock(synth.block_weights(0, 0, d))
    vl = Z.DeviceVarlen(cu)
    temb = dev(synth.randn(0, 9, (2, d.temb_dim)))
    cs, sn = rope_tables(pos, dims)
    x_ref = dev(x0)
    ws = torch.empty(Z.block_workspace_bytes(dims, fl, T, 2), dtype=torch.uint8, device="cuda")
    Z.zdit_block_forward(dims, fl, w, vl, x_ref, temb, cs, sn, ws)
    x = dev(x0)
    Z.zdit_block_forward_static(dims, fl, w, vl, x, temb, cs, sn)
    assert Z.zdit_device_status() == 0
    assert_parity(host(x), host(x_ref), TOL, base=x0, n_round=N_ROUND_BLOCK, label=f"static scratch, {T} tokens")

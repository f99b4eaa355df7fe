"""Parity at the full sizes of the 1024x1024 workload, in the launch configuration
bench.py times: one main block over the joint cond/uncond sequence (4224 + 4128
tokens, width 3840) checked on sampled rows against the oracle; the attention-only
sweep sizes checked on sampled query rows; the whole 34-block stack checked through
properties that hold at any size (branch isolation, determinism, finiteness) and, on request
(ZDIT_FULL_STACK_PARITY=1: the float64 oracle of the whole forward takes minutes of host
time), free-running against the oracle."""
import os

import numpy as np
import pytest
import torch

import oracle as O
import stream_diffusion_transformer_s3_b200 as Z
from stream_diffusion_transformer_s3_b200 import synth
from _gpu import BlockSource, LazyBlock, bf16, dev, errors, host, require_gpu, run_block_gpu, run_stack

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()


def _sample_rows(cu, extra_seed=0):
    rng = np.random.default_rng(extra_seed)
    rows = set()
    for b in range(len(cu) - 1):
        s, e = int(cu[b]), int(cu[b + 1])
        L = e - s
        for r in (0, 1, 127, 128, 255, 256, L - 129, L - 128, L - 33, L - 1):
            if 0 <= r < L:
                rows.add(s + r)
        rows.update((s + rng.integers(0, L, 4)).tolist())
    return np.array(sorted(rows))


def test_fullsize_main_block_sampled_rows():
    d = synth.FULL
    # image 64x64 grid, captions 128 (100 valid) and 32 (1 valid): T = 8352
    case = synth.block_case(21, d, 64, 64, [128, 32], [100, 1])
    got = run_block_gpu(case, d, O.Flags())
    rows = _sample_rows(case["cu_seqlens"])
    ref = O.block_forward_rows(case["x"], case["cu_seqlens"], case["pos"], case["temb"], case["weights"], d,
                               rows, O.Flags())
    x0 = case["x"][rows].astype(np.float64)
    e_upd = errors(got[rows] - x0, ref - x0)
    e_out = errors(got[rows], ref)
    print(f"\nfull-size block, {len(rows)} rows: update {e_upd}")
    assert e_upd["rel_l2"] <= TOL, e_upd
    assert e_out["rel_l2"] <= TOL, e_out


@pytest.mark.parametrize("n_img,n_cap", [(1024, 32), (4096, 128), (16384, 512)])
def test_attention_sweep_sampled_rows(n_img, n_cap):
    H = 30
    lengths = (n_img + n_cap, n_img + 32)  # cond, uncond (empty prompt pads to 32)
    c = synth.attention_case(5, H, 128, lengths)
    T = int(sum(lengths))
    vl = Z.DeviceVarlen(c["cu_seqlens"])
    o = torch.empty(T, H * 128, device="cuda", dtype=torch.bfloat16)
    Z.zdit_joint_attention(bf16(c["q"]), bf16(c["k"]), bf16(c["v"]), o, vl, H)
    assert Z.zdit_device_status() == 0
    got = host(o)
    rows = _sample_rows(c["cu_seqlens"], 1)
    cu = c["cu_seqlens"]
    ref = np.zeros((len(rows), H * 128))
    for i, r in enumerate(rows):
        b = int(np.searchsorted(cu, r, side="right") - 1)
        s, e = int(cu[b]), int(cu[b + 1])
        for h in range(H):
            sl = slice(h * 128, (h + 1) * 128)
            ref[i, sl] = O.softmax_attention(c["q"][r:r + 1, sl], c["k"][s:e, sl], c["v"][s:e, sl])[0]
    e = errors(got[rows], ref)
    print(f"\nattention {lengths}: {e}")
    assert e["rel_l2"] <= 1e-2, e


def _device_stack(seed=77):
    """34-block stack with seeded random weights generated on the device."""
    D, F, E = 3840, 10240, 256
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    bf = lambda *s: (torch.randn(*s, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    f32 = lambda *s: torch.randn(*s, generator=g, device="cuda") * 0.02
    nrm = lambda n: 1.0 + 0.1 * torch.randn(n, generator=g, device="cuda")
    kinds = ["noise"] * 2 + ["context"] * 2 + ["main"] * 30
    blocks = []
    for kind in kinds:
        t = {"w_qkv": bf(3 * D, D), "w_out": bf(D, D), "w_gate_up": bf(2 * F, D), "w_down": bf(D, F),
             "n_attn": nrm(D), "n_attn_post": nrm(D), "n_ffn": nrm(D), "n_ffn_post": nrm(D)}
        if kind != "context":
            t["w_ada"] = bf(4 * D, E)
            t["b_ada"] = f32(4 * D)
        blocks.append(Z.DeviceBlock.from_tensors(t))
    W = {"w_x": bf(D, 64), "b_x": f32(D), "w_capnorm": nrm(2560), "w_cap": bf(D, 2560), "b_cap": f32(D),
         "pad_vec": torch.randn(D, generator=g, device="cuda"), "w_t1": bf(E, E), "b_t1": f32(E),
         "w_t2": bf(E, E), "b_t2": f32(E), "w_fada": bf(D, E), "b_fada": f32(D), "w_final": bf(64, D),
         "b_final": f32(64)}
    return Z.DeviceStack(W, Z.Dims(), 2, 2, 30, patch_dim=64, cap_dim=2560, blocks=blocks)


def _run(stack, n_caps, n_valids, z, caps, t):
    call = Z.StackCall((64, 64), n_caps, n_valids, [t] * len(n_caps), z, caps, shared_patches=True)
    ws = torch.empty(Z.stack_workspace_bytes(stack, call), dtype=torch.uint8, device="cuda")
    out = torch.empty(len(n_caps), 4096, 64, device="cuda")
    Z.zdit_stack_forward(stack, call, out, ws)
    assert Z.zdit_device_status() == 0
    return out


def test_fullsize_stack_branch_isolation_and_determinism():
    stack = _device_stack()
    z = dev(synth.randn(42, 11, (4096, 64)))
    caps_c = synth.randn(42, 12, (100, 2560))
    caps_u = synth.randn(42, 13, (1, 2560))
    both = _run(stack, [128, 32], [100, 1], z, dev(np.concatenate([caps_c, caps_u])), 0.25)
    again = _run(stack, [128, 32], [100, 1], z, dev(np.concatenate([caps_c, caps_u])), 0.25)
    cond = _run(stack, [128], [100], z, dev(caps_c), 0.25)
    unc = _run(stack, [32], [1], z, dev(caps_u), 0.25)
    assert torch.isfinite(both).all()
    assert torch.equal(both, again), "stack forward is not deterministic"
    # branches never mix: each branch of the pair equals that branch run alone
    assert torch.equal(both[0], cond[0])
    assert torch.equal(both[1], unc[0])
    # the two branches differ (different captions)
    assert (both[0] - both[1]).abs().max().item() > 1e-3


@pytest.mark.skipif(os.environ.get("ZDIT_FULL_STACK_PARITY") != "1",
                    reason="the float64 oracle of the whole 1024x1024 forward takes ~7 min of host time")
def test_fullsize_stack_free_running():
    # the benchmarked workload end to end: 64x64 image grid per branch, captions 128 (100 valid)
    # and 32 (1 valid), 2 + 2 + 30 full-width blocks, embedders and final layer, against the
    # oracle's stack_forward on the same inputs
    d = synth.FULL
    seed = 31
    kinds = ["noise"] * 2 + ["context"] * 2 + ["main"] * 30
    W = synth.stack_weights(seed, d, blocks=False)
    src = BlockSource(seed, d, kinds)
    case = synth.stack_case(seed, 64, 64, [128, 32], [100, 1], [0.5, 0.5])
    ref = O.stack_forward(case, dict(W, blocks=[LazyBlock(src, i) for i in range(len(kinds))], block_kinds=kinds), d)
    got = run_stack(W, case, d, 2, 2, 30, 2560, blocks=src.device)
    e = errors(got, ref)
    print("\nstack 1024x1024, 34 blocks, free-running", e)
    assert e["rel_l2"] <= TOL, e

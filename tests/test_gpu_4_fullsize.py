"""Parity at the full sizes of the 1024x1024 workload, in the launch configuration
bench.py times: one main block over the joint cond/uncond sequence (4224 + 4128
tokens, width 3840) and one noise-refiner block over the image tokens of both branches
(2 x 4096 tokens) checked on sampled rows against the oracle (teacher-forced); the
attention-only sweep sizes checked on sampled query rows; the whole 34-block forward
free-running against the oracle's output of the same seeded inputs (stored by
tests/golden/make_stack_1024.py, since the float64 forward takes a quarter of an hour of
host time), and through properties that hold at any size (branch isolation,
determinism)."""
import os

import numpy as np
import pytest
import torch

import oracle as O
import stream_diffusion_transformer_s3_b200 as Z
from stream_diffusion_transformer_s3_b200 import synth
from _gpu import (N_ROUND_ATTN, N_ROUND_BLOCK, BlockSource, assert_parity, bf16, dev, host, require_gpu,
                  run_block_gpu, run_stack)

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
    assert_parity(got[rows], ref, TOL, base=x0, n_round=N_ROUND_BLOCK,
                  label=f"full-size main block, {len(rows)} sampled rows")


def test_fullsize_noise_refiner_block_sampled_rows():
    # a noise-refiner block at its real size: the image tokens of both branches (2 x 4096,
    # 64 x 64 grid each) as two segments, adaLN, image positions (n_cap_b + 1, h, w) with
    # the branches' caption lengths 128 and 32
    d = synth.FULL
    seed = 23
    n_img = 64 * 64
    cu = synth.cu_seqlens([n_img, n_img])
    pos = np.concatenate([synth.branch_positions(64, 64, c)[:n_img] for c in (128, 32)])
    case = {"x": synth.randn(seed, 1, (2 * n_img, d.dim)), "cu_seqlens": cu, "pos": pos,
            "temb": synth.randn(seed, 2, (2, d.temb_dim)), "weights": synth.block_weights(seed, 0, d)}
    got = run_block_gpu(case, d, O.Flags())
    rows = _sample_rows(cu, 2)
    ref = O.block_forward_rows(case["x"], cu, pos, case["temb"], case["weights"], d, rows, O.Flags())
    assert_parity(got[rows], ref, TOL, base=case["x"][rows].astype(np.float64), n_round=N_ROUND_BLOCK,
                  label=f"full-size noise-refiner block, {len(rows)} sampled rows")


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
    assert_parity(got[rows], ref, 1e-2, n_round=N_ROUND_ATTN, label=f"attention {lengths}, {len(rows)} sampled rows")


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


GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "stack_1024_seed31.npz")


def test_fullsize_stack_free_running():
    # the benchmarked workload end to end, free-running: 64x64 image grid per branch,
    # captions 128 (100 valid) and 32 (1 valid), 2 + 2 + 30 full-width blocks, embedders
    # and final layer, against the oracle's stack_forward of the same seeded inputs
    g = np.load(GOLDEN)
    seed = int(g["seed"])
    d = synth.FULL
    kinds = [str(k) for k in g["kinds"]]
    W = synth.stack_weights(seed, d, blocks=False)
    src = BlockSource(seed, d, kinds)
    for i in range(len(kinds)):  # draws each block once and uploads it
        src.host(i)
    case = synth.stack_case(seed, int(g["grid"][0]), int(g["grid"][1]), [int(c) for c in g["n_caps"]],
                            [int(v) for v in g["n_valids"]], [float(t) for t in g["t"]])
    got = run_stack(W, case, d, 2, 2, 30, 2560, blocks=src.device)
    ref = g["out"].astype(np.float64)
    assert_parity(got, ref, TOL, n_round=N_ROUND_BLOCK, label="1024x1024 forward, 34 blocks, free-running")

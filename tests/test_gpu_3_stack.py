"""Stack-level parity on the GPU: zdit_stack_forward (embedders, noise and context
refiners, joint main blocks, final layer) against the oracle's stack_forward."""
import pytest

import oracle as O
from stream_diffusion_transformer_s3_b200 import synth
from _gpu import N_ROUND_BLOCK, BlockSource, LazyBlock, assert_parity, require_gpu, run_stack

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()


@pytest.mark.parametrize("n_caps,n_valids", [((64, 32), (45, 1)), ((32,), (0,))])
def test_small_stack_matches_oracle(n_caps, n_valids):
    d = synth.BlockDims(dim=256, n_heads=2, head_dim=128, ffn_hidden=384)
    W = synth.stack_weights(7, d, n_noise=1, n_context=1, n_main=2, cap_dim=128)
    case = synth.stack_case(7, 8, 8, list(n_caps), list(n_valids), [0.4] * len(n_caps), cap_dim=128)
    got = run_stack(W, case, d, 1, 1, 2, 128)
    ref = O.stack_forward(case, W, d)
    assert_parity(got, ref, 2e-2, n_round=N_ROUND_BLOCK, label=f"stack {n_caps}")


def test_full_width_stack_two_blocks_per_kind_256px():
    # full-width dims, 16x16 image grid, cond/uncond captions 64/32
    d = synth.FULL
    W = synth.stack_weights(3, d, n_noise=1, n_context=1, n_main=1)
    case = synth.stack_case(3, 16, 16, [64, 32], [45, 1], [0.25, 0.25])
    got = run_stack(W, case, d, 1, 1, 1, 2560)
    ref = O.stack_forward(case, W, d)
    assert_parity(got, ref, 2e-2, n_round=N_ROUND_BLOCK, label="stack full width")


def test_full_width_full_depth_stack_256px():
    # the whole 34-block stack (2 noise refiners, 2 context refiners, 30 main blocks) at
    # full width, free-running from the embedders to the final layer, 16x16 image grid,
    # captions 64 / 32 (45 / 1 valid); the oracle runs first and each block it reads is
    # uploaded for the GPU on the way
    d = synth.FULL
    seed = 21
    kinds = ["noise"] * 2 + ["context"] * 2 + ["main"] * 30
    W = synth.stack_weights(seed, d, blocks=False)
    src = BlockSource(seed, d, kinds)
    case = synth.stack_case(seed, 16, 16, [64, 32], [45, 1], [0.6, 0.6])
    ref = O.stack_forward(case, dict(W, blocks=[LazyBlock(src, i) for i in range(len(kinds))], block_kinds=kinds), d)
    assert all(b is not None for b in src.device)
    got = run_stack(W, case, d, 2, 2, 30, 2560, blocks=src.device)
    # per-block bound 2e-2; the measured 34-block free-running error is 4.9e-3
    assert_parity(got, ref, 2e-2, n_round=N_ROUND_BLOCK, label="stack full width, 34 blocks")


def test_small_stack_three_branches():
    # three branches (e.g. two prompts and the empty one) in one call: the layout kernel, the
    # adaLN projections and the varlen attention over three segments
    d = synth.BlockDims(dim=256, n_heads=2, head_dim=128, ffn_hidden=384)
    W = synth.stack_weights(8, d, n_noise=1, n_context=1, n_main=2, cap_dim=128)
    case = synth.stack_case(8, 8, 8, [64, 32, 96], [45, 1, 70], [0.3, 0.3, 0.7], cap_dim=128)
    got = run_stack(W, case, d, 1, 1, 2, 128)
    ref = O.stack_forward(case, W, d)
    assert_parity(got, ref, 2e-2, n_round=N_ROUND_BLOCK, label="stack, three branches")


def test_small_stack_non_square_grid():
    # a 6 x 16 image grid (the stack takes image-token counts that are multiples of 32): the
    # image positions (h, w) and their RoPE axes, the patch-token order and the final layer's
    # image rows must all follow height and width, not a square
    d = synth.BlockDims(dim=256, n_heads=2, head_dim=128, ffn_hidden=384)
    W = synth.stack_weights(10, d, n_noise=1, n_context=1, n_main=2, cap_dim=128)
    case = synth.stack_case(10, 6, 16, [64, 32], [45, 1], [0.5, 0.5], cap_dim=128)
    got = run_stack(W, case, d, 1, 1, 2, 128)
    ref = O.stack_forward(case, W, d)
    assert_parity(got, ref, 2e-2, n_round=N_ROUND_BLOCK, label="stack, 6 x 16 grid")

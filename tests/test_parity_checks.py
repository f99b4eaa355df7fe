"""The parity checks used by the GPU tests must reject localized errors that one global
relative L2 norm lets through: one wrong token row of the 8352-token joint sequence, one
head's 128 columns lost in one row, one wrong element; and must pass results whose error
is the bf16 rounding noise of the path.  Runs on the CPU."""
import numpy as np
import pytest

import oracle as O
from stream_diffusion_transformer_s3_b200 import synth
from _parity import ParityError, assert_parity, parity_metrics

T, D = 8352, 3840  # the joint cond/uncond sequence of the 1024x1024 workload, model width


@pytest.fixture(scope="module")
def pair():
    rng = np.random.default_rng(3)
    ref = rng.standard_normal((T, D), dtype=np.float32)
    # rounding-level noise: relative 4e-3 per element, like a GPU block update
    got = ref + np.float32(4e-3) * rng.standard_normal((T, D), dtype=np.float32)
    return got, ref


def _global(got, ref):
    return float(np.linalg.norm((got - ref).astype(np.float64)) / np.linalg.norm(ref.astype(np.float64)))


def test_rounding_noise_passes(pair):
    got, ref = pair
    m = assert_parity(got, ref, 2e-2, label="noise")
    assert m["worst_elem_ratio"] < 0.5 and m["worst_row_rel"] < 6e-3


def test_one_wrong_row_of_8352_is_rejected(pair):
    got, ref = pair
    bad = got.copy()
    bad[4223] = np.random.default_rng(4).standard_normal(D)  # the last row of branch 0, unrelated values
    assert _global(bad, ref) < 2e-2  # the global norm alone would pass it
    with pytest.raises(ParityError, match="row 4223"):
        assert_parity(bad, ref, 2e-2, label="one row")


def test_one_head_lost_in_one_row_is_rejected(pair):
    got, ref = pair
    bad = got.copy()
    bad[8351, 7 * 128:8 * 128] = 0.0  # head 7 of the very last token
    assert _global(bad, ref) < 2e-2
    with pytest.raises(ParityError, match="row 8351"):
        assert_parity(bad, ref, 2e-2, label="one head")


def test_one_head_lost_in_one_query_tile_is_rejected(pair):
    got, ref = pair
    bad = got.copy()
    bad[4224:4224 + 128, 29 * 128:30 * 128] = 0.0  # the first query tile of branch 1, last head
    with pytest.raises(ParityError):
        assert_parity(bad, ref, 2e-2, label="one tile")


def test_one_wrong_element_is_rejected(pair):
    got, ref = pair
    bad = got.copy()
    bad[100, 200] += 0.5  # half the row's RMS
    assert _global(bad, ref) < 2e-2
    m = parity_metrics(bad, ref)
    assert m["worst_row_rel"] < 2e-2  # the row norm alone would pass it too
    with pytest.raises(ParityError, match=r"element \(100, 200\)"):
        assert_parity(bad, ref, 2e-2, label="one element")


def test_wrong_row_of_an_oracle_block_update_is_rejected():
    # a real oracle output (the tiny single block), perturbed at rounding level, then one
    # token's update made 10% too large: the output norm is dominated by the unchanged
    # input, so only the checks on the update catch it
    case = synth.config1(0)
    ref = O.block_forward(case["x"], case["cu_seqlens"], case["pos"], case["temb"], case["weights"], synth.TINY)
    x0 = case["x"].astype(np.float64)
    rng = np.random.default_rng(5)
    upd = ref - x0
    got = x0 + upd * (1.0 + 3e-3 * rng.standard_normal(upd.shape))
    assert_parity(got, ref, 2e-2, base=x0, label="oracle block")
    bad = got.copy()
    bad[40] = x0[40] + 1.1 * upd[40]
    assert _global(bad, ref) < 2e-2
    with pytest.raises(ParityError, match="row 40"):
        assert_parity(bad, ref, 2e-2, base=x0, label="oracle block, one token's update 10% large")


def test_non_finite_is_rejected():
    ref = np.ones((4, 8))
    got = ref.copy()
    got[2, 3] = np.nan
    with pytest.raises(ParityError, match="non-finite"):
        assert_parity(got, ref, 2e-2)

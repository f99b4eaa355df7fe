"""The stored expected output of the free-running 1024x1024 parity test
(tests/golden/stack_1024_seed31.npz, written by tests/golden/make_stack_1024.py, which
calls only the oracle and the seeded input generator) must belong to the inputs the
generator draws today: its recorded input digest is recomputed here.  Runs on the CPU."""
import os
import sys

import numpy as np

GOLDEN_DIR = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
sys.path.insert(0, GOLDEN_DIR)
import make_stack_1024 as M  # noqa: E402


def test_stored_stack_output_matches_the_generator():
    g = np.load(M.PATH)
    assert g["out"].shape == (2, 64 * 64, 64) and g["out"].dtype == np.float32
    assert np.all(np.isfinite(g["out"]))
    assert int(g["seed"]) == M.SEED
    assert tuple(g["grid"]) == M.GRID and tuple(g["n_caps"]) == M.N_CAPS
    assert tuple(g["n_valids"]) == M.N_VALIDS and tuple(g["t"]) == M.T_STEP
    assert [str(k) for k in g["kinds"]] == M.KINDS
    assert str(g["input_digest"]) == M.input_digest()

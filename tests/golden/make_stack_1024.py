"""Writes stack_1024_seed31.npz: the oracle's output of the benchmarked 1024x1024 DiT
forward, the expected value of the free-running full-size parity test.

The workload: a 64 x 64 patch grid per branch (latent 16 x 128 x 128 patchified 2 x 2),
captions padded to 128 (100 valid) and 32 (1 valid), t = 0.5 on both branches, 2 noise-
refiner + 2 context-refiner + 30 main full-width blocks (width 3840, 30 x 128 heads,
SwiGLU 10240), embedders and final layer, every weight and input drawn by the seeded
generator with seed 31.  Only oracle/ and the seeded input generator are called; the
float64 forward takes a quarter of an hour of host time, which is why its result is
stored instead of recomputed by the GPU test.

The file also holds a digest of the inputs the generator draws (patches, captions,
stack-level weights and every block's norm and adaLN-bias vectors), so a CPU test can
tell when the generator has changed and the stored output no longer belongs to it.

    python tests/golden/make_stack_1024.py
"""
from __future__ import annotations

import hashlib
import os
import sys
import time
from collections.abc import Mapping

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from stream_diffusion_transformer_s3_b200 import synth  # noqa: E402

SEED = 31
GRID = (64, 64)
N_CAPS = (128, 32)
N_VALIDS = (100, 1)
T_STEP = (0.5, 0.5)
KINDS = ["noise"] * 2 + ["context"] * 2 + ["main"] * 30
PATH = os.path.join(HERE, "stack_1024_seed31.npz")


def case():
    return synth.stack_case(SEED, GRID[0], GRID[1], list(N_CAPS), list(N_VALIDS), list(T_STEP))


def input_digest() -> str:
    """sha256 over the drawn inputs named in the module docstring, in a fixed order."""
    d = synth.FULL
    h = hashlib.sha256()
    c = case()
    for k in ("patches", "caps", "t"):
        h.update(np.ascontiguousarray(c[k], np.float32).tobytes())
    W = synth.stack_weights(SEED, d, blocks=False)
    for k in sorted(W):
        h.update(k.encode())
        h.update(np.ascontiguousarray(W[k], np.float32).tobytes())
    for i, kind in enumerate(KINDS):
        names = ["n_attn", "n_attn_post", "n_ffn", "n_ffn_post"] + (["b_ada"] if kind != "context" else [])
        for n in names:
            h.update(np.ascontiguousarray(synth.block_tensor(SEED, i, d, n), np.float32).tobytes())
    return h.hexdigest()


class _LazyBlocks(Mapping):
    """Block i's weights, drawn on first use; only the block being read is kept."""

    def __init__(self, i, cache):
        self.i, self.cache = i, cache
        self.names = ["w_qkv", "w_out", "w1", "w3", "w2", "n_attn", "n_attn_post", "n_ffn", "n_ffn_post"]
        if KINDS[i] != "context":
            self.names += ["w_ada", "b_ada"]

    def _w(self):
        if self.cache.get("i") != self.i:
            self.cache.clear()
            self.cache["i"] = self.i
            self.cache["w"] = synth.block_weights(SEED, self.i, synth.FULL, adaln=KINDS[self.i] != "context")
        return self.cache["w"]

    def __getitem__(self, name):
        if name not in self.names:
            raise KeyError(name)
        return self._w()[name]

    def __iter__(self):
        return iter(self.names)

    def __len__(self):
        return len(self.names)


def main():
    import oracle as O
    t0 = time.time()
    cache = {}
    W = dict(synth.stack_weights(SEED, synth.FULL, blocks=False),
             blocks=[_LazyBlocks(i, cache) for i in range(len(KINDS))], block_kinds=KINDS)
    out = O.stack_forward(case(), W, synth.FULL)
    np.savez_compressed(PATH, out=out.astype(np.float32), seed=SEED, grid=np.array(GRID),
                        n_caps=np.array(N_CAPS), n_valids=np.array(N_VALIDS), t=np.array(T_STEP),
                        kinds=np.array(KINDS), input_digest=input_digest())
    print(f"wrote {PATH}: out {out.shape}, |out| rms {np.sqrt(np.mean(out ** 2)):.4f}, {time.time() - t0:.0f} s")


if __name__ == "__main__":
    main()

"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module draws random numbers and lays out integer token metadata. It holds none
of the DiT's arithmetic: no norm, projection, rotation, attention or sampler step is
computed here. Both the CUDA path and the CPU oracle receive the arrays it returns.

Recipe (all draws are float32 ``standard_normal`` from NumPy's PCG64 seeded with
``SeedSequence([seed, tensor_id])``):

* GEMM weights: N(0, 0.02), rounded to bfloat16 with round-to-nearest-even.  The
  rounded values are what both sides compute with (the oracle widens them).
* adaLN / embedder / final-layer biases: N(0, 0.02) in float32.
* RMSNorm weights: 1 + 0.1 * N(0, 1) in float32 (non-trivial so a dropped or
  misplaced norm weight is visible in parity).
* learned caption pad vector: N(0, 1).
* residual stream x: N(0, 1); for the full-width block case the whole tensor is
  rescaled so that max |x| = 6.7e3 (the residual magnitude reported for the model
  in "Z-Image-Turbo port", section "fp16 does not work. bf16 does.").
* timestep embedding stand-in for block-level cases: N(0, 1) of width 256.
* caption features: N(0, 1) of width 2560.
* Q/K/V for the attention-only sweep: N(0, 1) rounded to bfloat16.

Token layout (a reading; the pages only fix that captions are padded to a multiple
of 32 with a learned pad token and that pads stay unmasked context, "Z-Image-Turbo
port", section "The three things that each cost a wrong image", item 3): every
branch b is one contiguous segment ``[image tokens | caption tokens]`` of length
``L_b = n_img_b + n_cap_b``; branches are packed back to back and described by
``cu_seqlens``.  Positions: caption token k has (k + 1, 0, 0); image token at grid
cell (h, w) has (n_cap_b + 1, h, w).
"""
from __future__ import annotations

import numpy as np

# Stable tensor ids: tensor_id = block_index * 64 + local id (blocks), or a fixed id
# (stack-level tensors, activations).
_BLOCK_TID = {
    "w_ada": 1, "b_ada": 2, "w_qkv": 3, "w_out": 4, "w1": 5, "w3": 6, "w2": 7,
    "n_attn": 8, "n_attn_post": 9, "n_ffn": 10, "n_ffn_post": 11, "n_q": 12, "n_k": 13,
}
_STACK_TID = {
    "w_x": 100001, "b_x": 100002, "w_capnorm": 100003, "w_cap": 100004, "b_cap": 100005,
    "pad_vec": 100006, "w_t1": 100007, "b_t1": 100008, "w_t2": 100009, "b_t2": 100010,
    "w_fada": 100011, "b_fada": 100012, "w_final": 100013, "b_final": 100014,
}
_ACT_TID = {"x": 200001, "temb": 200002, "caps": 200003, "patches": 200004,
            "q": 200005, "k": 200006, "v": 200007, "pad_row": 200008,
            "v_pos": 200009, "v_neg": 200010, "latent": 200011}


def randn(seed: int, tensor_id: int, shape, std: float = 1.0) -> np.ndarray:
    """float32 N(0, std^2) draws from PCG64 seeded by SeedSequence([seed, tensor_id])."""
    rng = np.random.default_rng(np.random.SeedSequence([int(seed), int(tensor_id)]))
    out = rng.standard_normal(size=tuple(int(s) for s in shape), dtype=np.float32)
    if std != 1.0:
        out *= np.float32(std)
    return out


def bf16_round(x: np.ndarray) -> np.ndarray:
    """float32 -> nearest bfloat16 value (ties to even), returned as float32.
    (uint32 arithmetic wraps like the truncation of a wider sum, so every input maps to
    the same bits as adding in 64 bits and keeping the low 32.)"""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u >> np.uint32(16)) & np.uint32(1)
    r += np.uint32(0x7FFF)
    r += u
    r &= np.uint32(0xFFFF0000)
    return r.view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) of float32 values that are already bf16-exact."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return (u >> 16).astype(np.uint16)


class BlockDims:
    def __init__(self, dim=3840, n_heads=30, head_dim=128, ffn_hidden=10240, temb_dim=256,
                 rope_axes=(32, 48, 48), rope_theta=10000.0, norm_eps=1e-5):
        self.dim, self.n_heads, self.head_dim = dim, n_heads, head_dim
        self.ffn_hidden, self.temb_dim = ffn_hidden, temb_dim
        self.rope_axes, self.rope_theta, self.norm_eps = tuple(rope_axes), rope_theta, norm_eps


TINY = BlockDims(dim=256, n_heads=2, head_dim=128, ffn_hidden=768)
FULL = BlockDims()


def block_weights(seed: int, block_index: int, d: BlockDims, adaln: bool = True,
                  qk_norm: bool = False) -> dict:
    """Weights of one block: GEMM weights bf16-valued float32, norms/biases float32.

    Shapes follow the linear-layer convention y = a @ W.T:
    w_qkv [3D, D] (rows q | k | v, head h at rows h*128 .. h*128+127 of each),
    w_out [D, D], w1 (gate) [F, D], w3 (up) [F, D], w2 [D, F], w_ada [4D, E], b_ada [4D].
    """
    names = ["w_qkv", "w_out", "w1", "w3", "w2", "n_attn", "n_attn_post", "n_ffn", "n_ffn_post"]
    if qk_norm:
        names += ["n_q", "n_k"]
    if adaln:
        names += ["w_ada", "b_ada"]
    return {n: block_tensor(seed, block_index, d, n) for n in names}


def block_tensor(seed: int, block_index: int, d: BlockDims, name: str) -> np.ndarray:
    """One tensor of block_weights(seed, block_index, d, ...), drawn on its own (each
    tensor has its own stream, so drawing one alone gives the same values)."""
    D, F, E, dh = d.dim, d.ffn_hidden, d.temb_dim, d.head_dim
    tid = block_index * 64 + _BLOCK_TID[name]
    gemm_shapes = {"w_qkv": (3 * D, D), "w_out": (D, D), "w1": (F, D), "w3": (F, D), "w2": (D, F),
                   "w_ada": (4 * D, E)}
    if name in gemm_shapes:
        return bf16_round(randn(seed, tid, gemm_shapes[name], 0.02))
    if name in ("n_attn", "n_attn_post", "n_ffn", "n_ffn_post"):
        return (1.0 + randn(seed, tid, (D,), 0.1)).astype(np.float32)
    if name in ("n_q", "n_k"):
        return (1.0 + randn(seed, tid, (dh,), 0.1)).astype(np.float32)
    if name == "b_ada":
        return randn(seed, tid, (4 * D,), 0.02)
    raise KeyError(name)


def stack_weights(seed: int, d: BlockDims, n_noise: int = 2, n_context: int = 2,
                  n_main: int = 30, patch_dim: int = 64, cap_dim: int = 2560,
                  qk_norm: bool = False, blocks: bool = True) -> dict:
    """All stack weights. Block order: noise refiners, context refiners, main blocks."""
    D, E = d.dim, d.temb_dim
    t = _STACK_TID
    g = lambda name, shape: bf16_round(randn(seed, t[name], shape, 0.02))
    b = lambda name, shape: randn(seed, t[name], shape, 0.02)
    w = {
        "w_x": g("w_x", (D, patch_dim)), "b_x": b("b_x", (D,)),
        "w_capnorm": (1.0 + randn(seed, t["w_capnorm"], (cap_dim,), 0.1)).astype(np.float32),
        "w_cap": g("w_cap", (D, cap_dim)), "b_cap": b("b_cap", (D,)),
        "pad_vec": randn(seed, t["pad_vec"], (D,)),
        "w_t1": g("w_t1", (E, E)), "b_t1": b("b_t1", (E,)),
        "w_t2": g("w_t2", (E, E)), "b_t2": b("b_t2", (E,)),
        "w_fada": g("w_fada", (D, E)), "b_fada": b("b_fada", (D,)),
        "w_final": g("w_final", (patch_dim, D)), "b_final": b("b_final", (patch_dim,)),
    }
    if blocks:
        kinds = ["noise"] * n_noise + ["context"] * n_context + ["main"] * n_main
        w["blocks"] = [block_weights(seed, i, d, adaln=(k != "context"), qk_norm=qk_norm)
                       for i, k in enumerate(kinds)]
        w["block_kinds"] = kinds
    return w


# ----------------------------------------------------------------------------- layout
def cu_seqlens(lengths) -> np.ndarray:
    out = np.zeros(len(lengths) + 1, dtype=np.int32)
    out[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return out


def branch_positions(grid_h: int, grid_w: int, n_cap: int) -> np.ndarray:
    """int32 [n_img + n_cap, 3] positions of one branch laid out [image | caption]."""
    hh, ww = np.meshgrid(np.arange(grid_h), np.arange(grid_w), indexing="ij")
    img = np.stack([np.full(grid_h * grid_w, n_cap + 1), hh.ravel(), ww.ravel()], axis=1)
    cap = np.stack([np.arange(1, n_cap + 1), np.zeros(n_cap, np.int64),
                    np.zeros(n_cap, np.int64)], axis=1)
    return np.concatenate([img, cap], axis=0).astype(np.int32)


def joint_positions(grid_h: int, grid_w: int, n_caps) -> np.ndarray:
    return np.concatenate([branch_positions(grid_h, grid_w, c) for c in n_caps], axis=0)


def block_case(seed: int, d: BlockDims, grid_h: int, grid_w: int, n_caps, n_valids,
               x_max: float | None = None, adaln: bool = True, qk_norm: bool = False) -> dict:
    """Inputs of one block call on a packed cond/uncond sequence.

    Caption rows at index >= n_valid of a branch hold one shared pad row (the learned
    pad token after embedding), so they are identical context rows.
    """
    D = d.dim
    n_img = grid_h * grid_w
    lens = [n_img + c for c in n_caps]
    T = int(sum(lens))
    x = randn(seed, _ACT_TID["x"], (T, D))
    pad_row = randn(seed, _ACT_TID["pad_row"], (D,))
    cu = cu_seqlens(lens)
    for b, (c, nv) in enumerate(zip(n_caps, n_valids)):
        start = cu[b] + n_img
        x[start + nv:start + c] = pad_row
    if x_max is not None:
        x *= np.float32(x_max / np.abs(x).max())
    case = {
        "x": x, "cu_seqlens": cu, "pos": joint_positions(grid_h, grid_w, n_caps),
        "temb": randn(seed, _ACT_TID["temb"], (len(n_caps), d.temb_dim)),
        "weights": block_weights(seed, 0, d, adaln=adaln, qk_norm=qk_norm),
        "grid": (grid_h, grid_w), "n_caps": list(n_caps), "n_valids": list(n_valids),
    }
    return case


def config1(seed: int = 0) -> dict:
    """Tiny single block: width 256, 2 heads x 128, FFN 768, 32 caption tokens of
    which the last 7 are pads, 64 image tokens on an 8x8 grid, batch 1."""
    return block_case(seed, TINY, 8, 8, [32], [25])


def config2(seed: int = 0) -> dict:
    """One full-width block at 256px: 16x16 image grid, cond/uncond pair with
    n_cap = 64 and 32 (n_valid 45 and 1), residual rescaled to max 6.7e3."""
    return block_case(seed, FULL, 16, 16, [64, 32], [45, 1], x_max=6.7e3)


def stack_case(seed: int, grid_h: int, grid_w: int, n_caps, n_valids, t, cap_dim=2560,
               patch_dim=64) -> dict:
    """Stack-level activations: patch tokens [B, n_img, 64], caption features
    [sum n_valid, cap_dim] (branches concatenated), timesteps t [B]."""
    B = len(n_caps)
    n_img = grid_h * grid_w
    return {
        "patches": randn(seed, _ACT_TID["patches"], (B, n_img, patch_dim)),
        "caps": randn(seed, _ACT_TID["caps"], (int(sum(n_valids)), cap_dim)),
        "n_caps": list(n_caps), "n_valids": list(n_valids), "grid": (grid_h, grid_w),
        "t": np.asarray(t, dtype=np.float32).reshape(B),
    }


def attention_case(seed: int, n_heads: int, head_dim: int, lengths) -> dict:
    """Attention-only inputs: bf16-valued Q, K, V [T, H*dh] and cu_seqlens."""
    T = int(sum(lengths))
    HD = n_heads * head_dim
    g = lambda name: bf16_round(randn(seed, _ACT_TID[name], (T, HD)))
    return {"q": g("q"), "k": g("k"), "v": g("v"), "cu_seqlens": cu_seqlens(lengths)}


def latent_noise(seed: int = 42, shape=(1, 16, 128, 128)) -> np.ndarray:
    return randn(seed, _ACT_TID["latent"], shape)


def velocity_pair(seed: int, n: int):
    return randn(seed, _ACT_TID["v_pos"], (n,)), randn(seed, _ACT_TID["v_neg"], (n,))

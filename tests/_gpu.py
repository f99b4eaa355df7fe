"""Shared helpers of the GPU parity tests (device marshalling and error metrics)."""
from collections.abc import Mapping

import numpy as np
import pytest
import torch

import stream_diffusion_transformer_s3_b200 as Z
from stream_diffusion_transformer_s3_b200 import synth


def require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    Z.lib()  # raises if the library is missing: no fallback


def dev(a, dtype=torch.float32):
    return torch.as_tensor(np.ascontiguousarray(a)).to(device="cuda", dtype=dtype).contiguous()


def bf16(a):
    return dev(np.asarray(a, np.float32), torch.bfloat16)


def host(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


from _parity import ParityError, assert_parity, parity_metrics  # noqa: F401  (re-exported)

# bf16 roundings on the block path, for the element bound of assert_parity: the
# operands a, q, k, v, P, o, a2, h and the stored projection outputs y (twice)
N_ROUND_BLOCK = 10
# attention alone: P before the PV product and the stored output
N_ROUND_ATTN = 2


def errors(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    diff = np.abs(got - ref)
    return {"rel_l2": float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)),
            "mean_abs": float(diff.mean()), "median_abs": float(np.median(diff)),
            "max_abs": float(diff.max())}


def rope_tables(pos, dims, stream=None):
    T = pos.shape[0]
    p = dev(pos.astype(np.int32), torch.int32)
    cs = torch.empty(T, dims.head_dim // 2, device="cuda")
    sn = torch.empty_like(cs)
    Z.zdit_rope_table(p, dims.rope_axes, dims.rope_theta, cs, sn, dims.head_dim)
    return cs, sn


def dims_of(d):
    return Z.Dims(dim=d.dim, n_heads=d.n_heads, head_dim=d.head_dim, ffn_hidden=d.ffn_hidden,
                  temb_dim=d.temb_dim, rope_axes=d.rope_axes, norm_eps=d.norm_eps,
                  rope_theta=d.rope_theta)


def run_block_gpu(case, d, flags):
    """Runs zdit_block_forward on a synth block case; returns the output rows."""
    dims = dims_of(d)
    fl = Z.flags_of(flags.adaln, flags.sandwich, flags.qk_norm, flags.tanh_gate)
    w = Z.DeviceBlock(case["weights"])
    vl = Z.DeviceVarlen(case["cu_seqlens"])
    x = dev(case["x"])
    temb = dev(case["temb"])
    cs, sn = rope_tables(case["pos"], dims)
    nbytes = Z.block_workspace_bytes(dims, fl, vl.total, len(case["cu_seqlens"]) - 1)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    Z.zdit_block_forward(dims, fl, w, vl, x, temb, cs, sn, ws)
    assert Z.zdit_device_status() == 0
    return host(x)


def run_stack(W, case, d, n_noise, n_ctx, n_main, cap_dim, flags=Z.F_ADALN | Z.F_SANDWICH_NORM, blocks=None):
    dims = dims_of(d)
    st = Z.DeviceStack(W, dims, n_noise, n_ctx, n_main, patch_dim=64, cap_dim=cap_dim, flags=flags, blocks=blocks)
    call = Z.StackCall(case["grid"], case["n_caps"], case["n_valids"], case["t"], dev(case["patches"]),
                       dev(case["caps"]))
    ws = torch.empty(Z.stack_workspace_bytes(st, call), dtype=torch.uint8, device="cuda")
    out = torch.full((len(case["n_caps"]), case["grid"][0] * case["grid"][1], 64), float("nan"), device="cuda")
    Z.zdit_stack_forward(st, call, out, ws)
    assert Z.zdit_device_status() == 0
    return host(out)


class BlockSource:
    """Draws each block's weights once: the first read of block i draws all its tensors,
    uploads them for the GPU and keeps the host copy only until another block is read, so
    the 34 full-width blocks (12 GB as bf16) never sit on the host at once."""

    def __init__(self, seed, d, kinds):
        self.seed, self.d, self.kinds = seed, d, kinds
        self.device = [None] * len(kinds)
        self.current = (None, None)

    def host(self, i):
        if self.current[0] != i:
            w = synth.block_weights(self.seed, i, self.d, adaln=self.kinds[i] != "context")
            if self.device[i] is None:
                self.device[i] = Z.DeviceBlock(w)
            self.current = (i, w)
        return self.current[1]


class LazyBlock(Mapping):
    """Block i's weights as the oracle reads them, drawn by a BlockSource on first use."""

    def __init__(self, source, i):
        self.source, self.i = source, i
        self.names = ["w_qkv", "w_out", "w1", "w3", "w2", "n_attn", "n_attn_post", "n_ffn", "n_ffn_post"]
        if source.kinds[i] != "context":
            self.names += ["w_ada", "b_ada"]

    def __getitem__(self, name):
        if name not in self.names:
            raise KeyError(name)
        return self.source.host(self.i)[name]

    def __iter__(self):
        return iter(self.names)

    def __len__(self):
        return len(self.names)

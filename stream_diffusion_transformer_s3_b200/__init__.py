"""B200-native hot path of the Z-Image-Turbo single-stream DiT (S3-DiT).

The compute lives in ``libzdit.so`` (hand-written sm_100a CUDA, C ABI declared in
``include/zdit.h``).  This module is the thin ctypes binding: it marshals torch
tensors (device memory, streams) into the C structs and calls the library under the
same names.  There is no fallback: if the library is missing or the device is not a
B200, calls raise.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass, field

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libzdit.so")
_lib = None

STATUS = {0: "ZDIT_OK", -1: "ZDIT_ERR_INVALID_ARG", -2: "ZDIT_ERR_SHAPE", -3: "ZDIT_ERR_ALIGNMENT",
          -4: "ZDIT_ERR_WORKSPACE", -5: "ZDIT_ERR_UNSUPPORTED", -6: "ZDIT_ERR_CUDA",
          -7: "ZDIT_ERR_DEVICE_TIMEOUT"}

F_ADALN, F_SANDWICH_NORM, F_QK_NORM, F_TANH_GATE = 1, 2, 4, 8


class ZditError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where} failed: {STATUS.get(code, code)}")
        self.code = code


# ----------------------------------------------------------------------- C structs
class BlockCfg(C.Structure):
    _fields_ = [("dim", C.c_int32), ("n_heads", C.c_int32), ("head_dim", C.c_int32),
                ("ffn_hidden", C.c_int32), ("temb_dim", C.c_int32), ("rope_axes", C.c_int32 * 3),
                ("norm_eps", C.c_float), ("rope_theta", C.c_float), ("flags", C.c_uint32)]


class BlockWeights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in (
        "w_ada", "b_ada", "w_qkv", "w_out", "w_gate_up", "w_down", "n_attn", "n_attn_post",
        "n_ffn", "n_ffn_post", "n_q", "n_k")]


class Varlen(C.Structure):
    _fields_ = [("batch", C.c_int32), ("cu_seqlens_dev", C.c_void_p),
                ("cu_seqlens_host", C.POINTER(C.c_int32))]


class StackCfg(C.Structure):
    _fields_ = [("block", BlockCfg), ("n_noise_refiner", C.c_int32), ("n_context_refiner", C.c_int32),
                ("n_main", C.c_int32), ("patch_dim", C.c_int32), ("cap_dim", C.c_int32),
                ("t_scale", C.c_float), ("final_eps", C.c_float)]


class StackWeights(C.Structure):
    _fields_ = [("blocks", C.POINTER(BlockWeights))] + [(n, C.c_void_p) for n in (
        "w_x", "b_x", "w_capnorm", "w_cap", "b_cap", "pad_vec", "w_t1", "b_t1", "w_t2", "b_t2",
        "w_fada", "b_fada", "w_final", "b_final")]


class StackInputs(C.Structure):
    _fields_ = [("batch", C.c_int32), ("grid_h", C.c_int32), ("grid_w", C.c_int32),
                ("n_cap", C.POINTER(C.c_int32)), ("n_valid", C.POINTER(C.c_int32)),
                ("patches", C.c_void_p), ("cap_feats", C.c_void_p), ("t", C.POINTER(C.c_float)),
                ("shared_patches", C.c_int32)]


class SampleCfg(C.Structure):
    _fields_ = [("n_steps", C.c_int32), ("guidance", C.c_float), ("cache_context", C.c_int32),
                ("dedup_noise", C.c_int32), ("use_graph", C.c_int32)]


class ProfileEntry(C.Structure):
    _fields_ = [("name", C.c_char * 40), ("launches", C.c_int32), ("total_ms", C.c_double),
                ("flops", C.c_double), ("bytes", C.c_double)]


_SIGS = {
    "zdit_profile_begin": (C.c_int, [C.c_int32]),
    "zdit_profile_end": (C.c_int, [C.POINTER(ProfileEntry), C.c_int32, C.POINTER(C.c_int32)]),
    "zdit_launch_count": (C.c_int64, []),
    "zdit_version": (C.c_int32, []),
    "zdit_status_string": (C.c_char_p, [C.c_int]),
    "zdit_block_workspace_bytes": (C.c_size_t, [C.POINTER(BlockCfg), C.c_int64, C.c_int32]),
    "zdit_block_forward": (C.c_int, [C.POINTER(BlockCfg), C.POINTER(BlockWeights), C.POINTER(Varlen),
                                     C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                     C.c_size_t, C.c_void_p]),
    "zdit_block_forward_static": (C.c_int, [C.POINTER(BlockCfg), C.POINTER(BlockWeights), C.POINTER(Varlen),
                                            C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]),
    "zdit_stack_workspace_bytes": (C.c_size_t, [C.POINTER(StackCfg), C.POINTER(StackInputs)]),
    "zdit_stack_forward": (C.c_int, [C.POINTER(StackCfg), C.POINTER(StackWeights), C.POINTER(StackInputs),
                                     C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]),
    "zdit_sample_workspace_bytes": (C.c_size_t, [C.POINTER(StackCfg), C.POINTER(StackInputs)]),
    "zdit_sample": (C.c_int, [C.POINTER(StackCfg), C.POINTER(StackWeights), C.POINTER(StackInputs),
                              C.POINTER(SampleCfg), C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]),
    "zdit_euler_cfg_step": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int64, C.c_float,
                                      C.c_float, C.c_float, C.c_void_p]),
    "zdit_sigma_schedule": (C.c_int, [C.c_int32, C.POINTER(C.c_float)]),
    "zdit_rope_table": (C.c_int, [C.c_void_p, C.c_int64, C.c_int32, C.POINTER(C.c_int32), C.c_float,
                                  C.c_void_p, C.c_void_p, C.c_void_p]),
    "zdit_joint_attention": (C.c_int, [C.c_void_p, C.c_int32, C.c_void_p, C.c_int32, C.c_void_p,
                                       C.c_int32, C.c_void_p, C.c_int32, C.POINTER(Varlen), C.c_int32,
                                       C.c_int32, C.c_void_p]),
    "zdit_adaln_project": (C.c_int, [C.POINTER(C.c_void_p), C.POINTER(C.c_void_p), C.POINTER(C.c_void_p),
                                     C.c_int32, C.c_void_p, C.c_int32, C.c_int32, C.c_int32, C.c_void_p]),
    "zdit_gemm_bf16": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int64, C.c_int64, C.c_int64,
                                 C.c_int64, C.c_void_p, C.c_void_p]),
    "zdit_patchify": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int32, C.c_int32, C.c_int32, C.c_void_p]),
    "zdit_unpatchify": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int32, C.c_int32, C.c_int32, C.c_void_p]),
    "zdit_device_status": (C.c_int, [C.c_void_p]),
    "zdit_selftest_wait_timeout": (C.c_int, [C.c_void_p, C.c_void_p]),
}


def lib():
    """Load libzdit.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libzdit.so not built ({LIB_PATH}); run "
                               "`python -m stream_diffusion_transformer_s3_b200.build`")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(code: int, where: str):
    if code != 0:
        raise ZditError(code, where)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


# ---------------------------------------------------------------- python-side config
@dataclass
class Dims:
    dim: int = 3840
    n_heads: int = 30
    head_dim: int = 128
    ffn_hidden: int = 10240
    temb_dim: int = 256
    rope_axes: tuple = (32, 48, 48)
    norm_eps: float = 1e-5
    rope_theta: float = 10000.0

    def cfg(self, flags: int) -> BlockCfg:
        c = BlockCfg()
        c.dim, c.n_heads, c.head_dim = self.dim, self.n_heads, self.head_dim
        c.ffn_hidden, c.temb_dim = self.ffn_hidden, self.temb_dim
        for i in range(3):
            c.rope_axes[i] = self.rope_axes[i]
        c.norm_eps, c.rope_theta, c.flags = self.norm_eps, self.rope_theta, flags
        return c


def flags_of(adaln=True, sandwich=True, qk_norm=False, tanh_gate=False) -> int:
    return (F_ADALN if adaln else 0) | (F_SANDWICH_NORM if sandwich else 0) | \
        (F_QK_NORM if qk_norm else 0) | (F_TANH_GATE if tanh_gate else 0)


class DeviceVarlen:
    """cu_seqlens on host and device, kept alive with the struct that points at them."""

    def __init__(self, cu_seqlens, device="cuda"):
        import torch
        cu = [int(v) for v in cu_seqlens]
        self.host = (C.c_int32 * len(cu))(*cu)
        self.dev = torch.tensor(cu, dtype=torch.int32, device=device)
        self.struct = Varlen(len(cu) - 1, C.c_void_p(self.dev.data_ptr()), self.host)
        self.total = cu[-1]


def interleave_gate_up(w1, w3):
    """[F, D] gate and up weights -> [2F, D] with 128-row blocks alternating
    (the w_gate_up layout declared in zdit.h).  Works on numpy arrays and tensors."""
    F = w1.shape[0]
    assert F % 128 == 0 and w3.shape == w1.shape
    if hasattr(w1, "reshape") and hasattr(w1, "dim"):  # torch
        import torch
        return torch.stack([w1.reshape(F // 128, 128, -1), w3.reshape(F // 128, 128, -1)], 1).reshape(2 * F, -1)
    import numpy as np
    return np.stack([w1.reshape(F // 128, 128, -1), w3.reshape(F // 128, 128, -1)], 1).reshape(2 * F, -1)


class DeviceBlock:
    """One block's weights in device memory (bf16 GEMM weights, fp32 norms/biases)."""

    def __init__(self, w: dict, device="cuda"):
        import torch
        bf = lambda a: torch.as_tensor(a, dtype=torch.float32).to(device=device, dtype=torch.bfloat16).contiguous()
        f32 = lambda a: torch.as_tensor(a, dtype=torch.float32).to(device).contiguous()
        self.t = {
            "w_qkv": bf(w["w_qkv"]), "w_out": bf(w["w_out"]),
            "w_gate_up": bf(interleave_gate_up(w["w1"], w["w3"])), "w_down": bf(w["w2"]),
        }
        for n in ("n_attn", "n_attn_post", "n_ffn", "n_ffn_post", "n_q", "n_k", "b_ada"):
            if n in w:
                self.t[n] = f32(w[n])
        if "w_ada" in w:
            self.t["w_ada"] = bf(w["w_ada"])
        self.struct = BlockWeights(**{n: (C.c_void_p(v.data_ptr())) for n, v in self.t.items()})

    @classmethod
    def from_tensors(cls, tensors: dict):
        self = cls.__new__(cls)
        self.t = dict(tensors)
        self.struct = BlockWeights(**{n: (C.c_void_p(v.data_ptr())) for n, v in self.t.items()})
        return self


# ------------------------------------------------------------------------ wrappers
def block_workspace_bytes(dims: Dims, flags: int, total_tokens: int, batch: int) -> int:
    c = dims.cfg(flags)
    return int(lib().zdit_block_workspace_bytes(C.byref(c), total_tokens, batch))


def zdit_block_forward(dims: Dims, flags: int, weights: DeviceBlock, varlen: DeviceVarlen, x, temb,
                       rope_cos, rope_sin, workspace, stream=None):
    c = dims.cfg(flags)
    code = lib().zdit_block_forward(C.byref(c), C.byref(weights.struct), C.byref(varlen.struct), _ptr(x),
                                    _ptr(temb), _ptr(rope_cos), _ptr(rope_sin), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream))
    _check(code, "zdit_block_forward")


def zdit_block_forward_static(dims: Dims, flags: int, weights: DeviceBlock, varlen: DeviceVarlen, x, temb,
                              rope_cos, rope_sin, stream=None):
    """zdit_block_forward with the library's static 40 MiB scratch as workspace: for
    callers that cannot allocate device memory.  Calls must not overlap on the GPU."""
    c = dims.cfg(flags)
    code = lib().zdit_block_forward_static(C.byref(c), C.byref(weights.struct), C.byref(varlen.struct), _ptr(x),
                                           _ptr(temb), _ptr(rope_cos), _ptr(rope_sin), _stream(stream))
    _check(code, "zdit_block_forward_static")


def zdit_rope_table(pos, rope_axes, theta, cos_out, sin_out, head_dim=128, stream=None):
    axes = (C.c_int32 * 3)(*rope_axes)
    _check(lib().zdit_rope_table(_ptr(pos), pos.shape[0], head_dim, axes, theta, _ptr(cos_out),
                                 _ptr(sin_out), _stream(stream)), "zdit_rope_table")


def zdit_joint_attention(q, k, v, o, varlen: DeviceVarlen, n_heads, head_dim=128, stream=None):
    _check(lib().zdit_joint_attention(_ptr(q), q.stride(0), _ptr(k), k.stride(0), _ptr(v), v.stride(0),
                                      _ptr(o), o.stride(0), C.byref(varlen.struct), n_heads, head_dim,
                                      _stream(stream)), "zdit_joint_attention")


def zdit_gemm_bf16(A, B, Cout, bias=None, stream=None):
    M, K = A.shape
    N = B.shape[0]
    _check(lib().zdit_gemm_bf16(_ptr(A), _ptr(B), _ptr(Cout), M, N, K, Cout.stride(0), _ptr(bias),
                                _stream(stream)), "zdit_gemm_bf16")


def zdit_adaln_project(w_ada, b_ada, out, temb, stream=None):
    """out[i] [B, rows] = temb [B, E] . w_ada[i]^T [E, rows] + b_ada[i] for every i, one launch
    (lists of device tensors: w_ada bf16 [rows, E], b_ada fp32 [rows] or None, out fp32 [B, rows])."""
    n = len(w_ada)
    rows, E = w_ada[0].shape
    ws = (C.c_void_p * n)(*[t.data_ptr() for t in w_ada])
    bs = (C.c_void_p * n)(*[(b.data_ptr() if b is not None else None) for b in b_ada])
    os_ = (C.c_void_p * n)(*[t.data_ptr() for t in out])
    _check(lib().zdit_adaln_project(ws, bs, os_, n, _ptr(temb), temb.shape[0], E, rows, _stream(stream)),
           "zdit_adaln_project")


def zdit_euler_cfg_step(x, v_pos, v_neg, g, sigma_cur, sigma_next, stream=None):
    _check(lib().zdit_euler_cfg_step(_ptr(x), _ptr(v_pos), _ptr(v_neg), x.numel(), g, sigma_cur,
                                     sigma_next, _stream(stream)), "zdit_euler_cfg_step")


def zdit_sigma_schedule(n_steps: int):
    buf = (C.c_float * (n_steps + 1))()
    _check(lib().zdit_sigma_schedule(n_steps, buf), "zdit_sigma_schedule")
    return list(buf)


def zdit_patchify(latent, tokens, stream=None):
    Cc, H2, W2 = latent.shape
    _check(lib().zdit_patchify(_ptr(latent), _ptr(tokens), Cc, H2, W2, _stream(stream)), "zdit_patchify")


def zdit_unpatchify(tokens, latent, stream=None):
    Cc, H2, W2 = latent.shape
    _check(lib().zdit_unpatchify(_ptr(tokens), _ptr(latent), Cc, H2, W2, _stream(stream)), "zdit_unpatchify")


def zdit_selftest_wait_timeout(result_dev, stream=None):
    _check(lib().zdit_selftest_wait_timeout(_ptr(result_dev), _stream(stream)), "zdit_selftest_wait_timeout")


def zdit_device_status(stream=None):
    return int(lib().zdit_device_status(_stream(stream)))


# ------------------------------------------------------------------------ stack
class DeviceStack:
    """All stack weights in device memory plus the C structs that point at them."""

    def __init__(self, W: dict, dims: Dims, n_noise: int, n_context: int, n_main: int,
                 patch_dim=64, cap_dim=2560, flags: int = F_ADALN | F_SANDWICH_NORM,
                 t_scale=1000.0, final_eps=1e-6, device="cuda", blocks=None):
        import torch
        bf = lambda a: torch.as_tensor(a, dtype=torch.float32).to(device=device, dtype=torch.bfloat16).contiguous()
        f32 = lambda a: torch.as_tensor(a, dtype=torch.float32).to(device).contiguous()
        self.dims, self.flags = dims, flags
        self.blocks = blocks if blocks is not None else [DeviceBlock(w, device) for w in W["blocks"]]
        assert len(self.blocks) == n_noise + n_context + n_main
        self.t = {}
        for n in ("w_x", "w_cap", "w_t1", "w_t2", "w_fada", "w_final"):
            self.t[n] = W[n] if hasattr(W[n], "data_ptr") else bf(W[n])
        for n in ("b_x", "w_capnorm", "b_cap", "pad_vec", "b_t1", "b_t2", "b_fada", "b_final"):
            self.t[n] = W[n] if hasattr(W[n], "data_ptr") else f32(W[n])
        self._barr = (BlockWeights * len(self.blocks))(*[b.struct for b in self.blocks])
        self.wstruct = StackWeights(C.cast(self._barr, C.POINTER(BlockWeights)),
                                    **{n: C.c_void_p(v.data_ptr()) for n, v in self.t.items()})
        self.cfg = StackCfg(dims.cfg(flags), n_noise, n_context, n_main, patch_dim, cap_dim, t_scale, final_eps)


class StackCall:
    """Inputs of one zdit_stack_forward call (host arrays kept alive)."""

    def __init__(self, grid, n_caps, n_valids, t, patches, cap_feats, shared_patches=False):
        B = len(n_caps)
        self.n_cap = (C.c_int32 * B)(*[int(v) for v in n_caps])
        self.n_valid = (C.c_int32 * B)(*[int(v) for v in n_valids])
        self.t = (C.c_float * B)(*[float(v) for v in t])
        self.patches, self.cap_feats = patches, cap_feats
        self.struct = StackInputs(B, int(grid[0]), int(grid[1]), self.n_cap, self.n_valid,
                                  C.c_void_p(patches.data_ptr()),
                                  C.c_void_p(cap_feats.data_ptr()) if cap_feats is not None else None,
                                  self.t, 1 if shared_patches else 0)

    def set_t(self, t):
        for i, v in enumerate(t):
            self.t[i] = float(v)


def stack_workspace_bytes(stack: DeviceStack, call: StackCall) -> int:
    return int(lib().zdit_stack_workspace_bytes(C.byref(stack.cfg), C.byref(call.struct)))


def zdit_stack_forward(stack: DeviceStack, call: StackCall, out, workspace, stream=None):
    _check(lib().zdit_stack_forward(C.byref(stack.cfg), C.byref(stack.wstruct), C.byref(call.struct),
                                    _ptr(out), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                    _stream(stream)), "zdit_stack_forward")


def zdit_profile_begin(max_records: int = 65536):
    _check(lib().zdit_profile_begin(max_records), "zdit_profile_begin")


def zdit_profile_end() -> dict:
    """{kernel kind: {launches, total_ms, flops, bytes}} of the launches recorded
    since zdit_profile_begin."""
    buf = (ProfileEntry * 32)()
    n = C.c_int32(0)
    _check(lib().zdit_profile_end(buf, 32, C.byref(n)), "zdit_profile_end")
    return {buf[i].name.decode(): {"launches": buf[i].launches, "total_ms": buf[i].total_ms,
                                   "flops": buf[i].flops, "bytes": buf[i].bytes} for i in range(n.value)}


def zdit_launch_count() -> int:
    return int(lib().zdit_launch_count())


def sample_workspace_bytes(stack: DeviceStack, call: StackCall) -> int:
    return int(lib().zdit_sample_workspace_bytes(C.byref(stack.cfg), C.byref(call.struct)))


def zdit_sample(stack: DeviceStack, call: StackCall, latent, workspace, n_steps=8, guidance=1.0,
                cache_context=True, dedup_noise=False, use_graph=False, stream=None):
    """In-place 8-step negated-CFG FlowMatchEuler sampling of `latent` [C, 2h, 2w].
    use_graph: capture the launch sequence as one CUDA graph and replay it on later calls
    with the same arguments."""
    sc = SampleCfg(n_steps, guidance, 1 if cache_context else 0, 1 if dedup_noise else 0, 1 if use_graph else 0)
    _check(lib().zdit_sample(C.byref(stack.cfg), C.byref(stack.wstruct), C.byref(call.struct), C.byref(sc),
                             _ptr(latent), _ptr(workspace), workspace.numel() * workspace.element_size(),
                             _stream(stream)), "zdit_sample")

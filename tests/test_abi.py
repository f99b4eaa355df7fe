"""CPU checks of the C-ABI library: it loads, exports every symbol the header
declares, and its host-side logic (validation, workspace sizing, the sigma schedule)
behaves as documented.  No call here reaches a GPU."""
import ctypes as C
import os
import re

import numpy as np

import oracle as O
import stream_diffusion_transformer_s3_b200 as Z

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "zdit.h")


def declared_symbols():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"ZDIT_API\s+[\w\s\*]+?\b(zdit_\w+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    L = Z.lib()
    names = declared_symbols()
    assert len(names) >= 14
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(Z._SIGS), "binding and header disagree"


def test_version_and_status_strings():
    L = Z.lib()
    assert L.zdit_version() == 200
    for code, name in Z.STATUS.items():
        assert L.zdit_status_string(code).decode() == name


def test_sigma_schedule_host_matches_oracle():
    for n in (1, 8, 50):
        got = np.array(Z.zdit_sigma_schedule(n), dtype=np.float64)
        np.testing.assert_allclose(got, O.sigma_schedule(n), rtol=1e-7, atol=1e-8)
        assert got[-1] == 0.0 and got[0] == 1.0
    assert Z.lib().zdit_sigma_schedule(0, (C.c_float * 2)()) == -1


def test_block_workspace_sizing():
    d = Z.Dims()
    f = Z.flags_of()
    small = Z.block_workspace_bytes(d, f, 608, 2)
    big = Z.block_workspace_bytes(d, f, 8352, 2)
    assert 0 < small < big
    # activations alone: a, o, y (bf16 D each) + qkv/h (bf16 max(3D, F)) per token
    per_tok = 3 * 2 * 3840 + 2 * 11520
    assert big >= 8352 * per_tok
    assert Z.block_workspace_bytes(Z.Dims(head_dim=64), f, 608, 2) == 0
    assert Z.block_workspace_bytes(d, f, 0, 2) == 0
    assert Z.block_workspace_bytes(d, f, 608, 9) == 0


def _fake(n=1 << 20):
    return C.c_void_p(n)


def test_block_forward_rejects_bad_arguments_before_launch():
    L = Z.lib()
    d = Z.Dims(dim=256, n_heads=2, ffn_hidden=768)
    cfg = d.cfg(Z.flags_of())
    w = Z.BlockWeights(**{f: _fake() for f, _ in Z.BlockWeights._fields_})
    cu = (C.c_int32 * 2)(0, 96)
    vl = Z.Varlen(1, _fake(), cu)
    args = lambda **k: dict(dict(cfg=C.byref(cfg), w=C.byref(w), vl=C.byref(vl), x=_fake(), temb=_fake(),
                                 rc=_fake(), rs=_fake(), ws=_fake(1 << 20), wsb=1 << 40), **k)
    call = lambda a: L.zdit_block_forward(a["cfg"], a["w"], a["vl"], a["x"], a["temb"], a["rc"], a["rs"],
                                          a["ws"], a["wsb"], None)
    assert call(args(x=None)) == -1
    bad = d.cfg(Z.flags_of())
    bad.head_dim = 64
    assert call(args(cfg=C.byref(bad))) == -2
    bad2 = d.cfg(Z.flags_of())
    bad2.rope_axes[0] = 30
    assert call(args(cfg=C.byref(bad2))) == -2
    wide = Z.Dims(dim=8448, n_heads=66, ffn_hidden=768).cfg(Z.flags_of())  # rows wider than 8192
    assert call(args(cfg=C.byref(wide))) == -2
    cu_bad = (C.c_int32 * 3)(0, 50, 40)
    vl_bad = Z.Varlen(2, _fake(), cu_bad)
    assert call(args(vl=C.byref(vl_bad))) == -2
    w_nul = Z.BlockWeights(**{f: _fake() for f, _ in Z.BlockWeights._fields_})
    w_nul.w_ada = None
    assert call(args(w=C.byref(w_nul))) == -1
    assert call(args(x=_fake((1 << 20) + 4))) == -3
    assert call(args(ws=_fake((1 << 20) + 64))) == -3


def test_stack_dims_validation():
    d = Z.Dims(dim=256, n_heads=2, ffn_hidden=768)
    cfg = Z.StackCfg(d.cfg(Z.flags_of()), 2, 2, 2, 64, 2560, 1000.0, 1e-6)
    n_cap = (C.c_int32 * 2)(64, 32)
    n_val = (C.c_int32 * 2)(45, 1)
    t = (C.c_float * 2)(0.5, 0.5)
    ok = Z.StackInputs(2, 8, 8, n_cap, n_val, _fake(), _fake(), t)
    L = Z.lib()
    assert L.zdit_stack_workspace_bytes(C.byref(cfg), C.byref(ok)) > 0
    n_cap_bad = (C.c_int32 * 2)(60, 32)   # caption length not a multiple of 32
    bad = Z.StackInputs(2, 8, 8, n_cap_bad, n_val, _fake(), _fake(), t)
    assert L.zdit_stack_workspace_bytes(C.byref(cfg), C.byref(bad)) == 0
    n_val_bad = (C.c_int32 * 2)(65, 1)    # more valid rows than caption slots
    bad = Z.StackInputs(2, 8, 8, n_cap, n_val_bad, _fake(), _fake(), t)
    assert L.zdit_stack_workspace_bytes(C.byref(cfg), C.byref(bad)) == 0
    odd_grid = Z.StackInputs(2, 5, 5, n_cap, n_val, _fake(), _fake(), t)   # 25 image tokens
    assert L.zdit_stack_workspace_bytes(C.byref(cfg), C.byref(odd_grid)) == 0
    wide_cap = Z.StackCfg(d.cfg(Z.flags_of()), 2, 2, 2, 64, 8256, 1000.0, 1e-6)  # caption width > 8192
    assert L.zdit_stack_workspace_bytes(C.byref(wide_cap), C.byref(ok)) == 0


def test_euler_rejects_null_and_misaligned():
    L = Z.lib()
    assert L.zdit_euler_cfg_step(None, _fake(), None, 16, 1.0, 1.0, 0.9, None) == -1
    assert L.zdit_euler_cfg_step(_fake((1 << 20) + 4), _fake(), None, 16, 1.0, 1.0, 0.9, None) == -3
    assert L.zdit_euler_cfg_step(_fake(), _fake(), None, 0, 1.0, 1.0, 0.9, None) == 0


def test_gate_up_interleave_layout():
    w1 = np.arange(256 * 3).reshape(256, 3)
    w3 = -np.arange(256 * 3).reshape(256, 3)
    g = Z.interleave_gate_up(w1, w3)
    assert g.shape == (512, 3)
    np.testing.assert_array_equal(g[0:128], w1[0:128])
    np.testing.assert_array_equal(g[128:256], w3[0:128])
    np.testing.assert_array_equal(g[256:384], w1[128:256])
    np.testing.assert_array_equal(g[384:512], w3[128:256])


def test_static_block_checks_match_workspace_block_order():
    # zdit_block_forward_static runs zdit_block_forward's checks, in the same order, before
    # its own size check: a call that zdit_block_forward rejects for a bad pointer or shape
    # is rejected with the same status, whatever its token count
    L = Z.lib()
    d = Z.Dims()
    cfg = d.cfg(Z.flags_of())
    w = Z.BlockWeights(**{f: _fake() for f, _ in Z.BlockWeights._fields_})
    cu = (C.c_int32 * 3)(0, 1024, 2048)  # far more tokens than the static scratch holds
    vl = Z.Varlen(2, _fake(), cu)
    stat = lambda w_=w, x=_fake(), vl_=vl: L.zdit_block_forward_static(C.byref(cfg), C.byref(w_), C.byref(vl_), x,
                                                                        _fake(), _fake(), _fake(), None)
    full = lambda w_=w, x=_fake(), vl_=vl: L.zdit_block_forward(C.byref(cfg), C.byref(w_), C.byref(vl_), x, _fake(),
                                                                 _fake(), _fake(), _fake(), 1 << 40, None)
    assert stat(x=None) == full(x=None) == -1
    assert stat(x=_fake((1 << 20) + 4)) == full(x=_fake((1 << 20) + 4)) == -3
    w_nul = Z.BlockWeights(**{f: _fake() for f, _ in Z.BlockWeights._fields_})
    w_nul.w_qkv = None
    assert stat(w_=w_nul) == full(w_=w_nul) == -1
    vl_bad = Z.Varlen(2, _fake(), (C.c_int32 * 3)(0, 1024, 1000))
    assert stat(vl_=vl_bad) == full(vl_=vl_bad) == -2


def test_adaln_project_rejects_bad_arguments_before_launch():
    L = Z.lib()
    arr = lambda *v: (C.c_void_p * len(v))(*v)
    ws, bs, os_ = arr(1 << 20, 1 << 21), arr(1 << 22, None), arr(1 << 23, 1 << 24)
    call = lambda w=ws, b=bs, o=os_, n=2, temb=_fake(), B=2, E=256, rows=15360: L.zdit_adaln_project(
        w, b, o, n, temb, B, E, rows, None)
    assert call(w=None) == -1
    assert call(temb=None) == -1
    assert call(w=arr(1 << 20, None)) == -1
    assert call(n=0) == -2
    assert call(B=9) == -2
    assert call(E=100) == -2          # not a multiple of 8
    assert call(E=2048) == -2         # wider than 1024
    assert call(rows=0) == -2
    assert call(w=arr(1 << 20, (1 << 21) + 8)) == -3   # weights must be 16-byte aligned
    assert call(temb=_fake((1 << 20) + 4)) == -3


def test_rope_table_rejects_bad_widths_before_launch():
    L = Z.lib()
    axes = lambda a, b, c: (C.c_int32 * 3)(a, b, c)
    call = lambda hd, ax: L.zdit_rope_table(_fake(), 16, hd, ax, 10000.0, _fake(), _fake(), None)
    assert call(128, axes(32, 48, 50)) == -2       # axes do not add up to the head width
    assert call(127, axes(31, 48, 48)) == -2       # odd head width
    assert call(2048, axes(512, 768, 768)) == -2   # wider than the 1024 the tables support
    assert L.zdit_rope_table(None, 16, 128, axes(32, 48, 48), 10000.0, _fake(), _fake(), None) == -1


def test_bench_names_a_bound_for_every_profiled_kernel_kind():
    # bench.py reports each kernel kind's fraction of the peak of its bound; every kind the
    # library's profiler records (the name table in prof.cu) must have one
    import re as _re
    import sys as _sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    _sys.path.insert(0, root)
    import bench
    src = open(os.path.join(root, "stream_diffusion_transformer_s3_b200", "csrc", "prof.cu")).read()
    table = src[src.index("{", src.index("const char*")):src.index("};", src.index("const char*"))]
    kinds = _re.findall(r'"(\w+)"', table)
    assert len(kinds) == 12
    assert set(kinds) == set(bench.KERNEL_BOUND)
    assert set(bench.KERNEL_BOUND.values()) <= {"tensor", "hbm", "latency"}

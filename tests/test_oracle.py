"""Pins of the CPU oracle against facts fixed by the pages and by mathematics.

Each test checks the oracle against something other than itself: a library routine
(torch, float64, CPU), a closed form, a value the pages print, an invariant, or a
brute-force computation on tiny inputs.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as O
from stream_diffusion_transformer_s3_b200 import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


def _t(a):
    return torch.from_numpy(np.asarray(a, np.float64))


# ------------------------------------------------------------------ elementary steps
def test_rms_norm_matches_torch():
    x = RNG.standard_normal((7, 96))
    w = RNG.standard_normal(96)
    ref = F.rms_norm(_t(x), (96,), weight=_t(w), eps=1e-5).numpy()
    np.testing.assert_allclose(O.rms_norm(x, w, 1e-5), ref, rtol=1e-13, atol=1e-13)


def test_layer_norm_matches_torch():
    x = RNG.standard_normal((5, 64)) * 3 + 2
    ref = F.layer_norm(_t(x), (64,), eps=1e-6).numpy()
    np.testing.assert_allclose(O.layer_norm_noaffine(x, 1e-6), ref, rtol=1e-12, atol=1e-12)


def test_silu_matches_torch():
    x = RNG.standard_normal(1000) * 8
    np.testing.assert_allclose(O.silu(x), F.silu(_t(x)).numpy(), rtol=1e-14, atol=1e-14)


# --------------------------------------------------------------------------- RoPE
def _rand_qk(T=11, H=3, dh=128):
    return RNG.standard_normal((T, H, dh))


def _rand_pos(T=11):
    return RNG.integers(0, 600, size=(T, 3))


def test_rope_preserves_pair_norms():
    x, pos = _rand_qk(), _rand_pos()
    y = O.rope_rotate(x, O.rope_angles(pos))
    nx = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    ny = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
    np.testing.assert_allclose(ny, nx, rtol=1e-12)


def test_rope_equals_complex_multiplication():
    # The real interleaved form equals (x_2i + i x_2i+1) * exp(i phi) ("bit-exact vs
    # the complex form", Core AI port, DiT row).
    x, pos = _rand_qk(), _rand_pos()
    phi = O.rope_angles(pos)
    z = (x[..., 0::2] + 1j * x[..., 1::2]) * np.exp(1j * phi)[:, None, :]
    ref = np.stack([z.real, z.imag], axis=-1).reshape(x.shape)
    np.testing.assert_allclose(O.rope_rotate(x, phi), ref, rtol=1e-12, atol=1e-12)


def test_rope_zero_position_is_identity():
    x = _rand_qk()
    y = O.rope_rotate(x, O.rope_angles(np.zeros((x.shape[0], 3), np.int64)))
    np.testing.assert_array_equal(y, x)


def test_rope_axis_assignment_and_frequencies():
    # Axis 0 drives pairs 0..15 (width 32), axis 1 pairs 16..39, axis 2 pairs 40..63.
    phi = O.rope_angles(np.array([[1, 0, 0], [0, 1, 0], [0, 0, 1]]))
    assert np.all(phi[0, :16] > 0) and np.all(phi[0, 16:] == 0)
    assert np.all(phi[1, 16:40] > 0) and np.all(phi[1, :16] == 0) and np.all(phi[1, 40:] == 0)
    assert np.all(phi[2, 40:] > 0) and np.all(phi[2, :40] == 0)
    # first pair of each axis turns one radian per position; last pair of axis 0
    # turns theta^(-30/32).
    assert phi[0, 0] == 1.0 and phi[1, 16] == 1.0 and phi[2, 40] == 1.0
    assert math.isclose(phi[0, 15], 10000.0 ** (-30.0 / 32.0), rel_tol=1e-14)
    assert math.isclose(phi[1, 39], 10000.0 ** (-46.0 / 48.0), rel_tol=1e-14)


def test_rope_relative_position_property():
    q = RNG.standard_normal((1, 1, 128))
    k = RNG.standard_normal((1, 1, 128))
    p, pk = np.array([[5, 9, 2]]), np.array([[1, 3, 7]])
    shift = np.array([[17, 4, 11]])

    def dot(pq, pk_):
        a = O.rope_rotate(q, O.rope_angles(pq))
        b = O.rope_rotate(k, O.rope_angles(pk_))
        return float((a * b).sum())

    assert math.isclose(dot(p, pk), dot(p + shift, pk + shift), rel_tol=1e-10)
    assert not math.isclose(dot(p, pk), dot(p + shift, pk), rel_tol=1e-6)


# ---------------------------------------------------------------------- attention
def test_attention_matches_torch_sdpa():
    T, H, dh = 40, 3, 128
    q, k, v = (RNG.standard_normal((T, H, dh)) for _ in range(3))
    cu = np.array([0, 40])
    ref = F.scaled_dot_product_attention(_t(q).transpose(0, 1), _t(k).transpose(0, 1),
                                         _t(v).transpose(0, 1)).transpose(0, 1).numpy()
    np.testing.assert_allclose(O.joint_attention(q, k, v, cu), ref, rtol=1e-11, atol=1e-12)


def test_attention_brute_force_loops():
    # tiny case with explicit scalar loops
    L, dh = 4, 8
    q, k, v = (RNG.standard_normal((L, dh)) for _ in range(3))
    out = np.zeros((L, dh))
    for i in range(L):
        logits = [sum(q[i, c] * k[j, c] for c in range(dh)) / math.sqrt(dh) for j in range(L)]
        m = max(logits)
        e = [math.exp(s - m) for s in logits]
        z = sum(e)
        for c in range(dh):
            out[i, c] = sum(e[j] / z * v[j, c] for j in range(L))
    np.testing.assert_allclose(O.softmax_attention(q, k, v), out, rtol=1e-12, atol=1e-13)


def test_attention_single_key_returns_value():
    q = RNG.standard_normal((5, 128))
    k, v = RNG.standard_normal((1, 128)), RNG.standard_normal((1, 128))
    np.testing.assert_allclose(O.softmax_attention(q, k, v), np.repeat(v, 5, 0), rtol=1e-14)


def test_attention_equal_keys_average_values():
    q = RNG.standard_normal((6, 128))
    k = np.repeat(RNG.standard_normal((1, 128)), 9, 0)
    v = RNG.standard_normal((9, 128))
    np.testing.assert_allclose(O.softmax_attention(q, k, v),
                               np.repeat(v.mean(0, keepdims=True), 6, 0), rtol=1e-12)


def test_attention_permutation_equivariant():
    T, H, dh = 30, 2, 128
    q, k, v = (RNG.standard_normal((T, H, dh)) for _ in range(3))
    perm = RNG.permutation(T)
    cu = np.array([0, T])
    a = O.joint_attention(q, k, v, cu)
    b = O.joint_attention(q[perm], k[perm], v[perm], cu)
    np.testing.assert_allclose(b, a[perm], rtol=1e-12, atol=1e-13)


def test_attention_branches_do_not_mix():
    H, dh = 2, 128
    q, k, v = (RNG.standard_normal((50, H, dh)) for _ in range(3))
    cu = np.array([0, 32, 50])
    both = O.joint_attention(q, k, v, cu)
    first = O.joint_attention(q[:32], k[:32], v[:32], np.array([0, 32]))
    second = O.joint_attention(q[32:], k[32:], v[32:], np.array([0, 18]))
    np.testing.assert_array_equal(both[:32], first)
    np.testing.assert_array_equal(both[32:], second)


def test_pad_tokens_are_unmasked_context():
    # n identical pad keys/values act as one key whose logit gains log(n) (closed form
    # of softmax over duplicated keys); masking or dropping them changes the output.
    dh, n_real, n_pad = 128, 25, 7
    q = RNG.standard_normal((3, dh))
    k_real, v_real = RNG.standard_normal((n_real, dh)), RNG.standard_normal((n_real, dh))
    k_pad, v_pad = RNG.standard_normal((1, dh)), RNG.standard_normal((1, dh))
    k = np.concatenate([k_real, np.repeat(k_pad, n_pad, 0)])
    v = np.concatenate([v_real, np.repeat(v_pad, n_pad, 0)])
    out = O.softmax_attention(q, k, v)
    logits = np.concatenate([q @ k_real.T, q @ k_pad.T], axis=1) / math.sqrt(dh)
    logits[:, -1] += math.log(n_pad)
    p = np.exp(logits - logits.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    ref = p @ np.concatenate([v_real, v_pad])
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)
    truncated = O.softmax_attention(q, k_real, v_real)
    assert np.abs(truncated - out).max() > 1e-3


# -------------------------------------------------------------------------- block
def _tiny_case(seed=3, adaln=True, qk_norm=False, n_caps=(32,), n_valids=(25,), grid=(4, 4)):
    d = synth.BlockDims(dim=256, n_heads=2, head_dim=128, ffn_hidden=384)
    case = synth.block_case(seed, d, grid[0], grid[1], list(n_caps), list(n_valids),
                            adaln=adaln, qk_norm=qk_norm)
    return d, case


def _run_block(d, case, flags=O.Flags(), w=None):
    return O.block_forward(case["x"], case["cu_seqlens"], case["pos"], case["temb"],
                           w if w is not None else case["weights"], d, flags)


def _torch_block(d, case, flags):
    """Independent composition from torch library routines (rms_norm, complex-form
    RoPE via view_as_complex, scaled_dot_product_attention, silu)."""
    w = {k: _t(v) for k, v in case["weights"].items()}
    x = _t(case["x"])
    T, D = x.shape
    H, dh = d.n_heads, d.head_dim
    cu = case["cu_seqlens"]
    temb = _t(case["temb"])
    if flags.adaln:
        mod = torch.nn.functional.linear(temb, w["w_ada"], w["b_ada"])
        s1, g1, s2, g2 = mod.chunk(4, dim=1)
        if flags.tanh_gate:  # only the two gate chunks pass through tanh; the scales do not
            g1, g2 = torch.tanh(g1), torch.tanh(g2)
    else:
        s1 = s2 = torch.zeros(len(cu) - 1, D, dtype=torch.float64)
        g1 = g2 = torch.ones(len(cu) - 1, D, dtype=torch.float64)
    seg = torch.repeat_interleave(torch.arange(len(cu) - 1), torch.from_numpy(np.diff(cu)))
    rms = lambda v, wt: F.rms_norm(v, (v.shape[-1],), weight=wt, eps=d.norm_eps)
    a = rms(x, w["n_attn"]) * (1 + s1[seg])
    wq, wk, wv = w["w_qkv"].split(D, dim=0)
    q, k, v = (F.linear(a, m).view(T, H, dh) for m in (wq, wk, wv))
    if flags.qk_norm:
        q, k = rms(q, w["n_q"]), rms(k, w["n_k"])
    # complex-form RoPE: angle of pair i from its axis
    pos = torch.from_numpy(case["pos"].astype(np.float64))
    freqs = []
    for ax, da in enumerate(d.rope_axes):
        inv = 1.0 / (d.rope_theta ** (torch.arange(0, da, 2, dtype=torch.float64) / da))
        freqs.append(torch.outer(pos[:, ax], inv))
    cis = torch.polar(torch.ones(T, dh // 2, dtype=torch.float64), torch.cat(freqs, 1))
    rot = lambda t_: torch.view_as_real(torch.view_as_complex(t_.reshape(T, H, dh // 2, 2))
                                        * cis[:, None, :]).reshape(T, H, dh)
    q, k = rot(q), rot(k)
    o = torch.zeros(T, H, dh, dtype=torch.float64)
    for b in range(len(cu) - 1):
        s, e = int(cu[b]), int(cu[b + 1])
        o[s:e] = F.scaled_dot_product_attention(q[s:e].transpose(0, 1), k[s:e].transpose(0, 1),
                                                v[s:e].transpose(0, 1)).transpose(0, 1)
    y = F.linear(o.reshape(T, D), w["w_out"])
    if flags.sandwich:
        y = rms(y, w["n_attn_post"])
    x = x + g1[seg] * y
    a = rms(x, w["n_ffn"]) * (1 + s2[seg])
    y = F.linear(F.silu(F.linear(a, w["w1"])) * F.linear(a, w["w3"]), w["w2"])
    if flags.sandwich:
        y = rms(y, w["n_ffn_post"])
    return (x + g2[seg] * y).numpy()


@pytest.mark.parametrize("flags", [O.Flags(), O.Flags(sandwich=False),
                                   O.Flags(qk_norm=True), O.Flags(adaln=False),
                                   O.Flags(tanh_gate=True), O.Flags(tanh_gate=True, sandwich=False)])
def test_block_matches_torch_composition(flags):
    d, case = _tiny_case(adaln=flags.adaln, qk_norm=flags.qk_norm, n_caps=(32, 64),
                         n_valids=(25, 40))
    np.testing.assert_allclose(_run_block(d, case, flags), _torch_block(d, case, flags),
                               rtol=1e-10, atol=1e-10)


def test_block_zero_adaln_is_identity():
    d, case = _tiny_case()
    w = dict(case["weights"])
    w["w_ada"] = np.zeros_like(w["w_ada"])
    w["b_ada"] = np.zeros_like(w["b_ada"])
    for flags in (O.Flags(), O.Flags(sandwich=False)):
        np.testing.assert_array_equal(_run_block(d, case, flags, w), case["x"].astype(np.float64))


def test_block_without_adaln_equals_unit_gate_zero_scale():
    d, case = _tiny_case()
    D = d.dim
    w = dict(case["weights"])
    w["w_ada"] = np.zeros_like(w["w_ada"])
    b = np.zeros(4 * D, np.float32)
    b[D:2 * D] = 1.0
    b[3 * D:] = 1.0
    w["b_ada"] = b
    a = _run_block(d, case, O.Flags(adaln=False))
    c = _run_block(d, case, O.Flags(adaln=True), w)
    np.testing.assert_allclose(a, c, rtol=1e-14, atol=1e-14)


def test_block_branches_independent():
    d, case = _tiny_case(n_caps=(32, 64), n_valids=(25, 40))
    both = _run_block(d, case)
    cu = case["cu_seqlens"]
    for b in range(2):
        s, e = cu[b], cu[b + 1]
        sub = dict(case, x=case["x"][s:e], pos=case["pos"][s:e], temb=case["temb"][b:b + 1],
                   cu_seqlens=np.array([0, e - s]))
        np.testing.assert_allclose(_run_block(d, sub), both[s:e], rtol=1e-12, atol=1e-12)


def test_block_rows_matches_full():
    d, case = _tiny_case(n_caps=(32, 64), n_valids=(25, 40), qk_norm=True)
    full = _run_block(d, case, O.Flags(qk_norm=True))
    rows = np.array([0, 5, 17, 47, 48, 50, 100, 111])
    part = O.block_forward_rows(case["x"], case["cu_seqlens"], case["pos"], case["temb"],
                                case["weights"], d, rows, O.Flags(qk_norm=True))
    np.testing.assert_allclose(part, full[rows], rtol=1e-12, atol=1e-12)


def test_image_axis0_rotation_cancels_in_image_only_attention():
    # In a noise-refiner block every image token shares axis-0 position n_cap + 1, so
    # that rotation cancels in q.k: the output does not depend on n_cap.
    d, case = _tiny_case(n_caps=(32,), n_valids=(32,))
    n_img = 16
    x = case["x"][:n_img]
    cu = np.array([0, n_img])
    outs = []
    for n_cap in (32, 128):
        pos = synth.branch_positions(4, 4, n_cap)[:n_img]
        outs.append(O.block_forward(x, cu, pos, case["temb"], case["weights"], d))
    np.testing.assert_allclose(outs[0], outs[1], rtol=1e-11, atol=1e-9)


def test_caption_pads_change_block_output_when_truncated():
    d, case = _tiny_case(n_caps=(32,), n_valids=(25,))
    full = _run_block(d, case)
    n_img = 16
    keep = n_img + 25
    sub = dict(case, x=case["x"][:keep], pos=case["pos"][:keep], cu_seqlens=np.array([0, keep]))
    trunc = _run_block(d, sub)
    assert np.abs(trunc[:n_img] - full[:n_img]).max() > 1e-3


# ---------------------------------------------------------------------- sampler
def test_sigma_schedule_golden_values():
    rows = [l.split() for l in open(os.path.join(GOLD, "sigma_schedule_8.txt"))
            if l.strip() and not l.startswith("#")]
    gold = np.array([float(Fraction(r[1])) for r in rows])
    np.testing.assert_allclose(O.sigma_schedule(8), gold, rtol=1e-15, atol=1e-16)


def test_sigma_schedule_equals_time_shift_form():
    # flow-matching time shift with factor 3: s t / (1 + (s - 1) t), t = 1 - u
    for n in (4, 8, 50):
        t = 1.0 - np.arange(n + 1) / n
        np.testing.assert_allclose(O.sigma_schedule(n), 3 * t / (1 + 2 * t), rtol=1e-14, atol=1e-16)
        s = O.sigma_schedule(n)
        assert s[0] == 1.0 and s[-1] == 0.0 and np.all(np.diff(s) < 0)


def test_negated_cfg_cases():
    p, n = RNG.standard_normal(100), RNG.standard_normal(100)
    np.testing.assert_array_equal(O.cfg_velocity(p, n, 0.0), -p)
    for g in (0.5, 1.0, 4.0):
        np.testing.assert_allclose(O.cfg_velocity(p, p, g), -p, rtol=0, atol=0)
    v0, v1, v3 = (O.cfg_velocity(p, n, g) for g in (0.0, 1.0, 3.0))
    np.testing.assert_allclose(v3, v0 + 3 * (v1 - v0), rtol=1e-13, atol=1e-13)
    # textbook form neg + g (pos - neg) differs: the sign and base branch both change
    np.testing.assert_allclose(O.cfg_velocity(p, n, 1.0), -(2 * p - n), rtol=1e-14)


def test_euler_constant_velocity_telescopes():
    x0 = RNG.standard_normal(64)
    v = RNG.standard_normal(64)
    s = O.sigma_schedule(8)
    x = x0
    for i in range(8):
        x = O.euler_step(x, v, s[i], s[i + 1])
    np.testing.assert_allclose(x, x0 - v, rtol=1e-13, atol=1e-13)


# ------------------------------------------------------------------- patchify
def test_patchify_golden_order():
    lat = np.zeros((2, 2, 4))
    for c in range(2):
        for y in range(2):
            for x in range(4):
                lat[c, y, x] = 100 * c + 10 * y + x
    rows = [list(map(float, l.split())) for l in open(os.path.join(GOLD, "patchify_tiny.txt"))
            if l.strip() and not l.startswith("#")]
    np.testing.assert_array_equal(O.patchify(lat), np.array(rows))


def test_patchify_round_trip():
    lat = RNG.standard_normal((16, 6, 10))
    tok = O.patchify(lat)
    assert tok.shape == (15, 64)
    np.testing.assert_array_equal(O.unpatchify(tok, 16, 3, 5), lat)


# -------------------------------------------------------------- stack and misc
def test_timestep_embedding_at_zero():
    w = {"w_t1": np.eye(256), "b_t1": np.zeros(256), "w_t2": np.eye(256), "b_t2": np.zeros(256)}
    emb = O.timestep_embedding(np.array([0.0]), w)
    np.testing.assert_allclose(emb[0, :128], O.silu(np.ones(128)), rtol=1e-15)
    np.testing.assert_allclose(emb[0, 128:], 0.0, atol=0)


def test_timestep_embedding_frequencies_at_nonzero_t():
    # Reading of the timestep embedding: the first half holds cos and the second half sin
    # of 1000 t times frequencies spaced geometrically from 1 down to 10000^(-127/128).
    # With identity MLP weights and zero biases the output is silu(embedding); the
    # expected values are written as a scalar loop with 10000 ** (-i / 128), another
    # expression than the oracle's exp(-ln(10000) i / half), so a divisor of (half - 1),
    # swapped cos / sin halves or a wrong time scale each fail here.
    w = {"w_t1": np.eye(256), "b_t1": np.zeros(256), "w_t2": np.eye(256), "b_t2": np.zeros(256)}
    t = 0.37
    emb = O.timestep_embedding(np.array([t]), w)[0]
    silu = lambda v: v / (1.0 + math.exp(-v))
    expect = [silu(math.cos(1000.0 * t * 10000.0 ** (-i / 128))) for i in range(128)]
    expect += [silu(math.sin(1000.0 * t * 10000.0 ** (-i / 128))) for i in range(128)]
    np.testing.assert_allclose(emb, np.array(expect), rtol=1e-12, atol=1e-12)
    # two entries worked by hand: i = 0 -> argument 370 rad; i = 64 -> 370 / 100 = 3.7 rad
    assert emb[0] == pytest.approx(silu(math.cos(370.0)), abs=1e-12)
    assert emb[128 + 64] == pytest.approx(silu(math.sin(3.7)), abs=1e-12)


def test_tanh_gate_touches_only_the_gate_chunks():
    # adaLN with the tanh-gate option: chunks (scale_attn, gate_attn, scale_ffn, gate_ffn);
    # only the gates pass through tanh.  Checked on a hand-set projection whose output
    # chunks are known: bias only, chunk c filled with the value c + 0.5.
    D, E = 4, 8
    w = {"w_ada": np.zeros((4 * D, E)), "b_ada": np.repeat(np.arange(4) + 0.5, D)}
    s1, g1, s2, g2 = O.adaln_vectors(np.ones((1, E)), w, D, O.Flags(tanh_gate=True))
    np.testing.assert_array_equal(s1, np.full((1, D), 0.5))
    np.testing.assert_allclose(g1, np.full((1, D), math.tanh(1.5)), rtol=1e-15)
    np.testing.assert_array_equal(s2, np.full((1, D), 2.5))
    np.testing.assert_allclose(g2, np.full((1, D), math.tanh(3.5)), rtol=1e-15)


def test_fp16_cannot_hold_projection_outputs():
    # out-projection / FFN outputs reach 3.1e5 (Core AI port, "fp16 does not work.
    # bf16 does."): beyond the fp16 maximum, inside the bf16 range.
    assert 3.1e5 > float(np.finfo(np.float16).max)
    assert float(synth.bf16_round(np.array([3.1e5], np.float32))[0]) == pytest.approx(3.1e5, rel=4e-3)


def test_parameter_count_near_6_15B():
    D, F_, E, H = 3840, 10240, 256, 30
    per_block = 3 * D * D + D * D + 3 * F_ * D + 4 * D
    ada = 4 * D * E + 4 * D
    blocks = 34 * per_block + 32 * ada
    embed = D * 64 + D + 2560 + D * 2560 + D + D + 2 * (E * E + E) + D * E + D + 64 * D + 64
    total = blocks + embed
    assert abs(total / 6.15e9 - 1) < 0.01


def test_stack_small_runs_and_pads_enter():
    d = synth.BlockDims(dim=256, n_heads=2, head_dim=128, ffn_hidden=384)
    W = synth.stack_weights(5, d, n_noise=1, n_context=1, n_main=1, cap_dim=64)
    case = synth.stack_case(5, 4, 4, [64, 32], [45, 1], [0.3, 0.3], cap_dim=64)
    out = O.stack_forward(case, W, d)
    assert out.shape == (2, 16, 64) and np.all(np.isfinite(out))
    # the uncond branch sees one valid caption row + 31 pad rows; changing the pad
    # vector changes its output
    W2 = dict(W, pad_vec=W["pad_vec"] + 1.0)
    out2 = O.stack_forward(case, W2, d)
    assert np.abs(out2[1] - out[1]).max() > 1e-6


def test_synth_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 3.0e38], np.float32)
    r = synth.bf16_round(x)
    assert r[0] == 1.0 and r[1] == 1.0 and r[2] == 1.0 + 2 ** -6 and r[3] == -2.5
    np.testing.assert_array_equal(
        r, torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy())


def _tiny_stack(seed=5, n_noise=1, n_context=1, n_main=1):
    d = synth.BlockDims(dim=256, n_heads=2, head_dim=128, ffn_hidden=384)
    W = synth.stack_weights(seed, d, n_noise=n_noise, n_context=n_context, n_main=n_main, cap_dim=64)
    case = synth.stack_case(seed, 4, 4, [64, 32], [45, 1], [0.3, 0.7], cap_dim=64)
    return d, W, case


def _zero_projections(wb):
    wb = dict(wb)
    for k in ("w_qkv", "w_out", "w1", "w3", "w2"):
        wb[k] = np.zeros_like(wb[k])
    return wb


def test_stack_with_zero_projections_is_embed_then_final_layer():
    # every block's projections zero => every block adds exactly 0 to its residual, so the
    # stack reduces to x-embed of the image rows followed by the final layer; the expected
    # value is composed here from torch float64 routines (Linear, LayerNorm, SiLU, cos/sin)
    d, W, case = _tiny_stack()
    Wz = dict(W, blocks=[_zero_projections(wb) for wb in W["blocks"]])
    out = O.stack_forward(case, Wz, d)
    t64 = lambda a: torch.as_tensor(np.asarray(a, np.float64))
    half = d.temb_dim // 2
    freqs = torch.exp(-math.log(10000.0) * torch.arange(half, dtype=torch.float64) / half)
    args = 1000.0 * t64(case["t"])[:, None] * freqs[None, :]
    emb = torch.cat([torch.cos(args), torch.sin(args)], dim=1)
    temb = torch.nn.functional.linear(torch.nn.functional.silu(
        torch.nn.functional.linear(emb, t64(W["w_t1"]), t64(W["b_t1"]))), t64(W["w_t2"]), t64(W["b_t2"]))
    for b in range(2):
        x = torch.nn.functional.linear(t64(case["patches"][b]), t64(W["w_x"]), t64(W["b_x"]))
        scale = torch.nn.functional.linear(temb[b], t64(W["w_fada"]), t64(W["b_fada"]))
        a = torch.nn.functional.layer_norm(x, (x.shape[-1],), eps=1e-6) * (1.0 + scale)
        ref = torch.nn.functional.linear(a, t64(W["w_final"]), t64(W["b_final"])).numpy()
        np.testing.assert_allclose(out[b], ref, rtol=1e-10, atol=1e-10)


def test_stack_branch_alone_equals_branch_in_pair():
    # branches never mix: the cond branch run alone gives the cond output of the pair
    d, W, case = _tiny_stack(seed=6)
    pair = O.stack_forward(case, W, d)
    alone = dict(case, patches=case["patches"][:1], caps=case["caps"][:45], n_caps=[64], n_valids=[45],
                 t=case["t"][:1])
    one = O.stack_forward(alone, W, d)
    np.testing.assert_allclose(one[0], pair[0], rtol=1e-12, atol=1e-12)


def test_captions_reach_the_image_only_through_main_blocks():
    # with the main blocks' projections zero, the image output does not depend on the
    # caption at all; with them live it does
    d, W, case = _tiny_stack(seed=8)
    kinds = W["block_kinds"]
    Wm = dict(W, blocks=[_zero_projections(wb) if k == "main" else wb for wb, k in zip(W["blocks"], kinds)])
    other = dict(case, caps=case["caps"] + 0.5)
    np.testing.assert_allclose(O.stack_forward(other, Wm, d), O.stack_forward(case, Wm, d), rtol=0, atol=0)
    assert np.abs(O.stack_forward(other, W, d) - O.stack_forward(case, W, d)).max() > 1e-6


# -------------------------------------------- stack and sampler against torch routines
def _torch_temb(t, W, dim):
    t64 = lambda a: torch.as_tensor(np.asarray(a, np.float64))
    half = dim // 2
    freqs = torch.exp(-math.log(10000.0) * torch.arange(half, dtype=torch.float64) / half)
    args = 1000.0 * t64(t).reshape(-1)[:, None] * freqs[None, :]
    emb = torch.cat([torch.cos(args), torch.sin(args)], dim=1)
    return F.linear(F.silu(F.linear(emb, t64(W["w_t1"]), t64(W["b_t1"]))), t64(W["w_t2"]), t64(W["b_t2"]))


def _torch_stack(d, W, case, flags=O.Flags()):
    """The whole forward composed from torch library routines: F.linear embedders,
    F.rms_norm caption norm, the blocks of _torch_block (rms_norm, complex-form RoPE,
    scaled_dot_product_attention, silu), F.layer_norm final layer; positions, packing and
    the block order are written here with torch indexing, not taken from the oracle."""
    t64 = lambda a: torch.as_tensor(np.asarray(a, np.float64))
    gh, gw = case["grid"]
    n_img = gh * gw
    n_caps, n_valids = list(case["n_caps"]), list(case["n_valids"])
    B = len(n_caps)
    temb = _torch_temb(case["t"], W, d.temb_dim)
    x_img = [F.linear(t64(case["patches"][b]), t64(W["w_x"]), t64(W["b_x"])) for b in range(B)]
    caps = t64(case["caps"])
    x_cap, off = [], 0
    for b in range(B):
        c = torch.empty(n_caps[b], d.dim, dtype=torch.float64)
        rows = caps[off:off + n_valids[b]]
        c[:n_valids[b]] = F.linear(F.rms_norm(rows, (rows.shape[1],), weight=t64(W["w_capnorm"]), eps=1e-5),
                                   t64(W["w_cap"]), t64(W["b_cap"]))
        c[n_valids[b]:] = t64(W["pad_vec"])
        x_cap.append(c)
        off += n_valids[b]
    hh, ww = torch.meshgrid(torch.arange(gh), torch.arange(gw), indexing="ij")
    img_pos = [torch.stack([torch.full((n_img,), n_caps[b] + 1), hh.reshape(-1), ww.reshape(-1)], 1)
               for b in range(B)]
    cap_pos = [torch.stack([torch.arange(1, n_caps[b] + 1), torch.zeros(n_caps[b], dtype=torch.long),
                            torch.zeros(n_caps[b], dtype=torch.long)], 1) for b in range(B)]
    cum = lambda lens: np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)

    def run(x, lens, pos, wb, fl):
        blk = {"weights": wb, "x": x.numpy(), "cu_seqlens": cum(lens), "pos": pos.numpy(),
               "temb": temb.numpy()}
        return torch.from_numpy(_torch_block(d, blk, fl))

    fl_ctx = O.Flags(adaln=False, sandwich=flags.sandwich, qk_norm=flags.qk_norm, tanh_gate=flags.tanh_gate)
    xi, xc = torch.cat(x_img), torch.cat(x_cap)
    for wb, kind in zip(W["blocks"], W["block_kinds"]):
        if kind == "noise":
            xi = run(xi, [n_img] * B, torch.cat(img_pos), wb, flags)
        elif kind == "context":
            xc = run(xc, n_caps, torch.cat(cap_pos), wb, fl_ctx)
    cap_cu = cum(n_caps)
    xj = torch.cat([torch.cat([xi[b * n_img:(b + 1) * n_img], xc[cap_cu[b]:cap_cu[b + 1]]]) for b in range(B)])
    pj = torch.cat([torch.cat([img_pos[b], cap_pos[b]]) for b in range(B)])
    lens = [n_img + c for c in n_caps]
    for wb, kind in zip(W["blocks"], W["block_kinds"]):
        if kind == "main":
            xj = run(xj, lens, pj, wb, flags)
    cu = cum(lens)
    out = []
    for b in range(B):
        x = xj[cu[b]:cu[b] + n_img]
        scale = F.linear(temb[b], t64(W["w_fada"]), t64(W["b_fada"]))
        a = F.layer_norm(x, (x.shape[-1],), eps=1e-6) * (1.0 + scale)
        out.append(F.linear(a, t64(W["w_final"]), t64(W["b_final"])))
    return torch.stack(out).numpy()


def test_stack_matches_torch_composition():
    d, W, case = _tiny_stack(seed=11, n_noise=2, n_context=2, n_main=2)
    np.testing.assert_allclose(O.stack_forward(case, W, d), _torch_stack(d, W, case), rtol=1e-9, atol=1e-9)


def test_stack_matches_torch_composition_qk_norm_no_sandwich():
    d = synth.BlockDims(dim=256, n_heads=2, head_dim=128, ffn_hidden=384)
    W = synth.stack_weights(12, d, n_noise=1, n_context=1, n_main=2, cap_dim=64, qk_norm=True)
    case = synth.stack_case(12, 4, 2, [32, 64], [1, 50], [0.9, 0.2], cap_dim=64)
    fl = O.Flags(sandwich=False, qk_norm=True)
    np.testing.assert_allclose(O.stack_forward(case, W, d, fl), _torch_stack(d, W, case, fl),
                               rtol=1e-9, atol=1e-9)


def test_sampler_matches_torch_composition():
    # the 8-step loop composed with torch: closed-form schedule, patchify by reshape /
    # permute, negated CFG and Euler with torch arithmetic, the forward of _torch_stack
    d, W, _ = _tiny_stack(seed=13)
    C, h, w = 16, 2, 3
    latent = synth.latent_noise(13, (C, 2 * h, 2 * w))
    caps_c = RNG.standard_normal((40, 64)).astype(np.float32)
    caps_u = RNG.standard_normal((1, 64)).astype(np.float32)
    cond = {"caps": caps_c, "n_cap": 64, "n_valid": 40}
    unc = {"caps": caps_u, "n_cap": 32, "n_valid": 1}
    g = 1.5
    got = O.sample(latent, cond, unc, W, d, g=g, n_steps=8)
    u = torch.arange(9, dtype=torch.float64) / 8
    sig = 3 * (1 - u) / (3 * (1 - u) + u)
    z = torch.as_tensor(latent, dtype=torch.float64).view(C, h, 2, w, 2).permute(1, 3, 2, 4, 0).reshape(h * w, 4 * C)
    for i in range(8):
        case = {"grid": (h, w), "patches": torch.stack([z, z]).numpy(),
                "caps": np.concatenate([caps_c, caps_u]), "n_caps": [64, 32], "n_valids": [40, 1],
                "t": np.array([1 - sig[i].item()] * 2)}
        out = torch.from_numpy(_torch_stack(d, W, case))
        v = -(out[0] + g * (out[0] - out[1]))
        z = z + (sig[i + 1] - sig[i]) * v
    ref = z.reshape(h, w, 2, 2, C).permute(4, 0, 2, 1, 3).reshape(C, 2 * h, 2 * w).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-9, atol=1e-9)

"""Kernel-level parity on the GPU: projection GEMM, joint attention, RoPE tables,
the fused negated-CFG Euler update and patchify, each against the CPU oracle (or a
float64 matrix product for the GEMM) on seeded inputs."""

import numpy as np
import pytest
import torch

import oracle as O
import stream_diffusion_transformer_s3_b200 as Z
from stream_diffusion_transformer_s3_b200 import synth
from _gpu import N_ROUND_ATTN, assert_parity, bf16, dev, host, require_gpu, rope_tables

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()


def gemm_tol(K):
    # fp32 accumulation of K products with random signs: relative error grows like
    # sqrt(K) ulp(1) = sqrt(K) * 2^-23 (tensor-core adds need not round to nearest)
    return 3.0 * np.sqrt(K) * 2.0 ** -23


@pytest.mark.parametrize("M,N,K", [
    (128, 256, 64),      # one tile
    (200, 512, 192),     # ragged M tail, 3 K slices
    (96, 64, 3840),      # N below the tile width (final-layer shape)
    (608, 3840, 3840),   # out-projection of the full-width cond/uncond pair
    (1000, 768, 256),    # several M tiles, ragged
    (33, 3840, 64),      # image-embedder shape, tiny M
])
def test_gemm_matches_float64_product(M, N, K):
    rng = np.random.default_rng(M * 7 + N + K)
    A = synth.bf16_round(rng.standard_normal((M, K), dtype=np.float32))
    B = synth.bf16_round(rng.standard_normal((N, K), dtype=np.float32) * 0.05)
    bias = rng.standard_normal(N).astype(np.float32)
    out = torch.full((M, N), float("nan"), device="cuda")
    Z.zdit_gemm_bf16(bf16(A), bf16(B), out, bias=dev(bias))
    assert Z.zdit_device_status() == 0
    ref = A.astype(np.float64) @ B.astype(np.float64).T + bias
    assert_parity(host(out), ref, gemm_tol(K), rtol=gemm_tol(K), label=f"gemm {M}x{N}x{K}")


def test_gemm_large_k_and_many_tiles():
    # the down-projection depth (K = 10240) over a few thousand rows
    rng = np.random.default_rng(5)
    M, N, K = 2100, 768, 10240
    A = synth.bf16_round(rng.standard_normal((M, K), dtype=np.float32))
    B = synth.bf16_round(rng.standard_normal((N, K), dtype=np.float32) * 0.02)
    out = torch.empty(M, N, device="cuda")
    Z.zdit_gemm_bf16(bf16(A), bf16(B), out)
    assert Z.zdit_device_status() == 0
    ref = A.astype(np.float64) @ B.astype(np.float64).T
    assert_parity(host(out), ref, gemm_tol(K), rtol=gemm_tol(K), label=f"gemm {M}x{N}x{K}")


@pytest.mark.parametrize("n_mat,B,rows,E", [
    (3, 2, 4 * 3840, 256),   # three blocks' adaLN projections at full width, cond/uncond
    (45, 8, 4 * 256, 256),   # more matrices than one launch holds, the largest batch
    (2, 1, 77, 1024),        # ragged rows (groups of 8 cut), four 256-column chunks
])
def test_adaln_project_matches_oracle(n_mat, B, rows, E):
    temb = synth.randn(8, 900, (B, E))
    ws = [synth.bf16_round(synth.randn(8, 901 + i, (rows, E), 0.02)) for i in range(n_mat)]
    bs = [synth.randn(8, 1001 + i, (rows,), 0.02) if i % 2 == 0 else None for i in range(n_mat)]
    outs = [torch.full((B, rows), float("nan"), device="cuda") for _ in range(n_mat)]
    Z.zdit_adaln_project([bf16(w) for w in ws], [dev(b) if b is not None else None for b in bs], outs, dev(temb))
    assert Z.zdit_device_status() == 0
    tol = 3.0 * np.sqrt(E) * 2.0 ** -23
    refs = []
    for i in range(n_mat):
        if rows % 4 == 0 and bs[i] is not None:
            # the oracle's adaLN step: four chunks (scale_attn, gate_attn, scale_ffn, gate_ffn)
            refs.append(np.concatenate(O.adaln_vectors(temb, {"w_ada": ws[i], "b_ada": bs[i]}, rows // 4, O.Flags()),
                                       axis=1))
        else:
            refs.append(temb.astype(np.float64) @ ws[i].astype(np.float64).T + (0.0 if bs[i] is None else bs[i]))
    # rows of the check: (matrix, branch)
    assert_parity(np.concatenate([host(o) for o in outs]), np.concatenate(refs), tol, rtol=tol,
                  label=f"adaLN projections, {n_mat} matrices x {B} branches x {rows}")


def _attn_case(lengths, H, seed=0):
    c = synth.attention_case(seed, H, 128, lengths)
    T = int(sum(lengths))
    q, k, v = (c[n].reshape(T, H, 128) for n in ("q", "k", "v"))
    return c, q, k, v


@pytest.mark.parametrize("lengths,H", [
    ((96,), 2),            # config-1 sequence
    ((320, 288), 4),       # config-2 lengths (cond 256+64, uncond 256+32)
    ((130, 33), 2),        # ragged: one full tile + 2 rows, and a short branch
    ((1, 127, 129), 3),    # single-token branch, one short of / one past a tile
    ((1056, 1056 + 96), 2),
])
def test_attention_matches_oracle(lengths, H):
    c, q, k, v = _attn_case(lengths, H)
    T = q.shape[0]
    vl = Z.DeviceVarlen(c["cu_seqlens"])
    o = torch.full((T, H * 128), float("nan"), device="cuda", dtype=torch.bfloat16)
    Z.zdit_joint_attention(bf16(c["q"]), bf16(c["k"]), bf16(c["v"]), o, vl, H)
    assert Z.zdit_device_status() == 0
    ref = O.joint_attention(q, k, v, c["cu_seqlens"]).reshape(T, H * 128)
    assert_parity(host(o), ref, 1e-2, n_round=N_ROUND_ATTN, label=f"attention {lengths} x {H}")


def test_attention_full_width_config5_small():
    # 30 heads x 128, image 1024 tokens + n_cap 128 cond / 32 uncond (attention sweep)
    lengths = (1024 + 128, 1024 + 32)
    c, q, k, v = _attn_case(lengths, 30, seed=3)
    T = q.shape[0]
    vl = Z.DeviceVarlen(c["cu_seqlens"])
    o = torch.empty(T, 30 * 128, device="cuda", dtype=torch.bfloat16)
    Z.zdit_joint_attention(bf16(c["q"]), bf16(c["k"]), bf16(c["v"]), o, vl, 30)
    assert Z.zdit_device_status() == 0
    ref = O.joint_attention(q, k, v, c["cu_seqlens"]).reshape(T, -1)
    assert_parity(host(o), ref, 1e-2, n_round=N_ROUND_ATTN, label="attention 1152/1056 x 30")


def test_attention_large_logits_move_reference_max():
    # keys growing along the sequence force the running max to move (O rescale path)
    rng = np.random.default_rng(9)
    L, H = 640, 1
    q = np.ones((L, H, 128), np.float32) * 0.5
    k = (rng.standard_normal((L, H, 128)) * 0.1 + np.linspace(0, 4, L)[:, None, None]).astype(np.float32)
    v = rng.standard_normal((L, H, 128)).astype(np.float32)
    q, k, v = (synth.bf16_round(a) for a in (q, k, v))
    vl = Z.DeviceVarlen([0, L])
    o = torch.empty(L, 128, device="cuda", dtype=torch.bfloat16)
    Z.zdit_joint_attention(bf16(q.reshape(L, -1)), bf16(k.reshape(L, -1)), bf16(v.reshape(L, -1)), o, vl, 1)
    assert Z.zdit_device_status() == 0
    ref = O.joint_attention(q, k, v, np.array([0, L])).reshape(L, -1)
    assert_parity(host(o), ref, 1e-2, n_round=N_ROUND_ATTN, label="attention, moving max")


def test_rope_table_matches_oracle():
    pos = synth.joint_positions(64, 64, [128, 32])
    dims = Z.Dims()
    cs, sn = rope_tables(pos, dims)
    phi = O.rope_angles(pos, dims.rope_axes, dims.rope_theta)
    np.testing.assert_allclose(host(cs), np.cos(phi), atol=2e-7, rtol=0)
    np.testing.assert_allclose(host(sn), np.sin(phi), atol=2e-7, rtol=0)


@pytest.mark.parametrize("n,g,with_neg", [(262144, 1.0, True), (1001, 4.0, True), (64, 0.0, False)])
def test_euler_cfg_matches_oracle(n, g, with_neg):
    vp, vn = synth.velocity_pair(1, n)
    x0 = synth.randn(2, 7, (n,))
    sig = O.sigma_schedule(8)
    x = dev(x0)
    Z.zdit_euler_cfg_step(x, dev(vp), dev(vn) if with_neg else None, g, float(sig[2]), float(sig[3]))
    assert Z.zdit_device_status() == 0
    v = O.cfg_velocity(vp, vn if with_neg else vp, g)
    ref = O.euler_step(x0, v, float(np.float32(sig[2])), float(np.float32(sig[3])))
    np.testing.assert_allclose(host(x), ref, rtol=1e-6, atol=1e-6)


def test_patchify_round_trip_non_square_latent():
    # 12 x 20 latent -> 6 x 10 token grid: a swapped height and width would reorder the tokens
    lat = synth.randn(43, 11, (16, 12, 20))
    t = torch.empty(6 * 10, 64, device="cuda")
    Z.zdit_patchify(dev(lat), t)
    np.testing.assert_array_equal(host(t), O.patchify(lat))
    back = torch.empty(16, 12, 20, device="cuda")
    Z.zdit_unpatchify(t, back)
    np.testing.assert_array_equal(host(back), lat)


def test_patchify_round_trip_matches_oracle():
    lat = synth.randn(42, 11, (16, 128, 128))
    t = torch.empty(64 * 64, 64, device="cuda")
    Z.zdit_patchify(dev(lat), t)
    np.testing.assert_array_equal(host(t), O.patchify(lat))
    back = torch.empty(16, 128, 128, device="cuda")
    Z.zdit_unpatchify(t, back)
    np.testing.assert_array_equal(host(back), lat)

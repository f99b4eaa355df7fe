"""CPU oracle for the Z-Image-Turbo single-stream DiT hot path.

TEST INFRASTRUCTURE ONLY.  This module is imported by the tests, by the package's
smoke check and by the benchmark's CPU-baseline leg; the product path (the CUDA
library and its Python binding) never imports, links or runs it.

Everything is plain NumPy in float64.  GEMM weights arrive as bfloat16 values (the
exact numbers the GPU multiplies) and are widened; activations are never rounded.
Library primitives used as steps: ``@`` (matrix product), ``exp``, ``cos``, ``sin``,
``tanh``, ``sqrt``.  There is no blocking, fusion or reordering: each function is the
textbook definition of its step, written in the order the pages give.

Sources (web pages, cited by title and section):
  [CoreAI]  "Z-Image-Turbo port - a 6B diffusion DiT on Core AI, and why it is
            Mac-only" (Core AI model zoo): table "Architecture -> export mapping"
            (DiT, Sampler rows), section "The three things that each cost a wrong
            image", section "fp16 does not work. bf16 does.", section "Hosting it
            from Swift" (patchify order, schedule closed form).
  [Jobs]    "Native creative jobs" (1Cat-vLLM design note), section "Recipes and
            precision".
  [Port]    "Z-Image Port Status" (FastVideo), section "Pinned Official Pipeline
            Context" (scheduler contract, defaults).

Readings where the pages are silent (each is also listed in the design notes):
  R1  Block: pre-norm RMSNorm with (1 + scale) modulation; optional RMSNorm of each
      projection output before its gated add ("sandwich", on by default); adaLN gives
      four D-wide chunks (scale_attn, gate_attn, scale_ffn, gate_ffn), no shift, no
      activation before the adaLN linear; identity gate unless tanh_gate is set.
  R2  RMSNorm eps 1e-5; final-layer LayerNorm (no affine) eps 1e-6.
  R3  No bias on QKV / out / FFN projections; biases on adaLN, embedders, final layer.
  R4  RoPE: pairs (2i, 2i+1) of each head; pair i < 16 rotates with position axis 0,
      16 <= i < 40 with axis 1, otherwise axis 2; frequency theta^(-2j/d_axis), j the
      pair index inside its axis, axis widths (32, 48, 48), theta 10000.
  R5  Timestep embedding: [cos | sin] of 1000 t times exp(-ln(10000) i / 128), i < 128,
      then Linear(256, 256) -> SiLU -> Linear(256, 256).
  R6  Final layer: LayerNorm_noaffine(x) * (1 + W_f temb + b_f), then Linear(D, 64).
  R7  The DiT is called with t = 1 - sigma.
  R8  Caption embed: RMSNorm over the caption width (weighted) then Linear + bias; the
      rows at index >= n_valid are replaced by the learned pad vector.
  R9  QK-norm (per-head RMSNorm of q and k before RoPE) is an option, off by default.

Pins: every function is checked in tests/test_oracle.py against library routines, brute
force, closed forms, invariants or values printed on the pages.  stack_forward and sample
(the pages print no output value for them) are checked against a composition of torch library
routines (F.linear, F.rms_norm, F.layer_norm, scaled_dot_product_attention, complex-form RoPE,
reshape/permute patchify) on tiny configurations; the block order, the packing and the
positions are written there independently, so a reading of the pages shared by both sides is
the one thing those tests cannot catch.  Stack-level invariants (zero projections reduce the
stack to embed + final layer, branch isolation, captions acting only through the main blocks)
and sampler invariants (schedule values, telescoping Euler steps, negated CFG cases) are pinned
as well.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

F64 = np.float64


@dataclass(frozen=True)
class Flags:
    adaln: bool = True
    sandwich: bool = True
    qk_norm: bool = False
    tanh_gate: bool = False


# ------------------------------------------------------------------ elementary steps
def rms_norm(v, w=None, eps: float = 1e-5):
    """v / sqrt(mean(v^2) + eps) over the last axis, times w if given (R1, R2)."""
    v = np.asarray(v, F64)
    out = v / np.sqrt(np.mean(v * v, axis=-1, keepdims=True) + eps)
    return out if w is None else out * np.asarray(w, F64)


def layer_norm_noaffine(v, eps: float = 1e-6):
    """(v - mean) / sqrt(var + eps) over the last axis (R6)."""
    v = np.asarray(v, F64)
    mu = v.mean(axis=-1, keepdims=True)
    var = ((v - mu) ** 2).mean(axis=-1, keepdims=True)
    return (v - mu) / np.sqrt(var + eps)


def silu(v):
    v = np.asarray(v, F64)
    return v / (1.0 + np.exp(-v))


def rope_angles(pos, axes=(32, 48, 48), theta: float = 10000.0):
    """Rotation angle of every pair: phi[t, i] = pos[t, axis(i)] * theta^(-2 j / d_axis).

    [CoreAI] "Architecture -> export mapping", DiT row: 3-axis RoPE fed with
    precomputed cos/sin.  Axis split and theta per R4.  Returns [T, sum(axes) / 2].
    """
    pos = np.asarray(pos, F64)
    cols = []
    for a, d_a in enumerate(axes):
        j = np.arange(d_a // 2, dtype=F64)
        omega = theta ** (-2.0 * j / d_a)
        cols.append(pos[:, a:a + 1] * omega[None, :])
    return np.concatenate(cols, axis=1)


def rope_rotate(x, phi):
    """Real interleaved RoPE: rotate each adjacent pair (x_2i, x_2i+1) by phi[t, i].

    x: [T, H, dh]; phi: [T, dh / 2].  [CoreAI] DiT row: the complex-form RoPE is
    replaced by a bit-exact real interleaved form.
    """
    x = np.asarray(x, F64)
    c = np.cos(phi)[:, None, :]
    s = np.sin(phi)[:, None, :]
    xe, xo = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = xe * c - xo * s
    out[..., 1::2] = xe * s + xo * c
    return out


def softmax_attention(q, k, v):
    """softmax(q k^T / sqrt(dh)) v for one head, no mask.  q [Lq, dh], k, v [L, dh]."""
    dh = q.shape[-1]
    s = (np.asarray(q, F64) @ np.asarray(k, F64).T) / math.sqrt(dh)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=1, keepdims=True)
    return p @ np.asarray(v, F64)


def joint_attention(q, k, v, cu_seqlens):
    """Attention of every branch segment over itself, heads independent, no mask.

    q, k, v: [T, H, dh]; cu_seqlens [B + 1].  Caption pad rows are ordinary context
    ([CoreAI] "The three things that each cost a wrong image", item 3); branches
    never attend to each other.
    """
    T, H, dh = q.shape
    out = np.zeros((T, H, dh), F64)
    for b in range(len(cu_seqlens) - 1):
        s, e = int(cu_seqlens[b]), int(cu_seqlens[b + 1])
        for h in range(H):
            out[s:e, h] = softmax_attention(q[s:e, h], k[s:e, h], v[s:e, h])
    return out


def branch_of_token(cu_seqlens):
    cu = np.asarray(cu_seqlens, np.int64)
    return np.repeat(np.arange(len(cu) - 1), np.diff(cu))


def adaln_vectors(temb, w, dim: int, flags: Flags):
    """(scale_attn, gate_attn, scale_ffn, gate_ffn), each [B, D] (R1).

    Without adaLN (the context refiner has none, [CoreAI] DiT row):
    scale = 0 and gate = 1.
    """
    B = np.asarray(temb).shape[0]
    if not flags.adaln:
        z, o = np.zeros((B, dim)), np.ones((B, dim))
        return z, o, z, o
    m = np.asarray(temb, F64) @ np.asarray(w["w_ada"], F64).T + np.asarray(w["b_ada"], F64)
    s1, g1, s2, g2 = (m[:, i * dim:(i + 1) * dim] for i in range(4))
    if flags.tanh_gate:
        g1, g2 = np.tanh(g1), np.tanh(g2)
    return s1, g1, s2, g2


# ------------------------------------------------------------------------- the block
def block_forward(x, cu_seqlens, pos, temb, w, d, flags: Flags = Flags(), trace=None):
    """One single-stream DiT block over a packed varlen sequence (float64).

    Order: adaLN vectors -> RMSNorm * (1 + scale) -> QKV projection -> (QK-norm) ->
    real RoPE -> joint attention -> output projection -> (sandwich norm) -> gated
    residual -> RMSNorm * (1 + scale) -> SwiGLU FFN -> (sandwich norm) -> gated
    residual.  [CoreAI] DiT row; [Jobs] "Recipes and precision" (FP32 range for
    projection outputs and SwiGLU gating before normalization, adaLN scaling,
    residual).  x [T, D]; temb [B, E]; pos [T, 3] integer positions.
    """
    x = np.asarray(x, F64)
    T, D = x.shape
    H, dh, eps = d.n_heads, d.head_dim, d.norm_eps
    bt = branch_of_token(cu_seqlens)
    s1, g1, s2, g2 = adaln_vectors(temb, w, D, flags)

    a = rms_norm(x, w["n_attn"], eps) * (1.0 + s1[bt])
    qkv = a @ np.asarray(w["w_qkv"], F64).T
    q = qkv[:, :D].reshape(T, H, dh)
    k = qkv[:, D:2 * D].reshape(T, H, dh)
    v = qkv[:, 2 * D:].reshape(T, H, dh)
    if flags.qk_norm:
        q = rms_norm(q, w["n_q"], eps)
        k = rms_norm(k, w["n_k"], eps)
    phi = rope_angles(pos, d.rope_axes, d.rope_theta)
    q = rope_rotate(q, phi)
    k = rope_rotate(k, phi)
    o = joint_attention(q, k, v, cu_seqlens).reshape(T, D)
    y = o @ np.asarray(w["w_out"], F64).T
    if flags.sandwich:
        y = rms_norm(y, w["n_attn_post"], eps)
    x1 = x + g1[bt] * y

    a2 = rms_norm(x1, w["n_ffn"], eps) * (1.0 + s2[bt])
    h = silu(a2 @ np.asarray(w["w1"], F64).T) * (a2 @ np.asarray(w["w3"], F64).T)
    y2 = h @ np.asarray(w["w2"], F64).T
    if flags.sandwich:
        y2 = rms_norm(y2, w["n_ffn_post"], eps)
    x2 = x1 + g2[bt] * y2
    if trace is not None:
        trace.update(q=q, k=k, v=v, attn=o, y_attn=y, x_mid=x1, h=h, y_ffn=y2)
    return x2


def block_forward_rows(x, cu_seqlens, pos, temb, w, d, rows, flags: Flags = Flags()):
    """block_forward restricted to the output rows `rows` (same definition).

    Keys and values of every token of the branches that the rows belong to are
    computed; queries, attention, projections and the FFN only for `rows`.  Used to
    check full-size GPU runs on a sample of tokens.
    """
    x = np.asarray(x, F64)
    T, D = x.shape
    H, dh, eps = d.n_heads, d.head_dim, d.norm_eps
    rows = np.asarray(rows, np.int64)
    bt = branch_of_token(cu_seqlens)
    s1, g1, s2, g2 = adaln_vectors(temb, w, D, flags)
    phi = rope_angles(pos, d.rope_axes, d.rope_theta)
    wqkv = np.asarray(w["w_qkv"], F64)
    out = np.zeros((len(rows), D))
    for b in sorted(set(bt[rows].tolist())):
        s, e = int(cu_seqlens[b]), int(cu_seqlens[b + 1])
        sel = np.nonzero(bt[rows] == b)[0]
        r = rows[sel]
        a_all = rms_norm(x[s:e], w["n_attn"], eps) * (1.0 + s1[b])
        kv = a_all @ wqkv[D:].T
        k = kv[:, :D].reshape(e - s, H, dh)
        v = kv[:, D:].reshape(e - s, H, dh)
        a_r = rms_norm(x[r], w["n_attn"], eps) * (1.0 + s1[b])
        q = (a_r @ wqkv[:D].T).reshape(len(r), H, dh)
        if flags.qk_norm:
            q = rms_norm(q, w["n_q"], eps)
            k = rms_norm(k, w["n_k"], eps)
        q = rope_rotate(q, phi[r])
        k = rope_rotate(k, phi[s:e])
        o = np.zeros((len(r), H, dh))
        for hh in range(H):
            o[:, hh] = softmax_attention(q[:, hh], k[:, hh], v[:, hh])
        y = o.reshape(len(r), D) @ np.asarray(w["w_out"], F64).T
        if flags.sandwich:
            y = rms_norm(y, w["n_attn_post"], eps)
        x1 = x[r] + g1[b] * y
        a2 = rms_norm(x1, w["n_ffn"], eps) * (1.0 + s2[b])
        hh_ = silu(a2 @ np.asarray(w["w1"], F64).T) * (a2 @ np.asarray(w["w3"], F64).T)
        y2 = hh_ @ np.asarray(w["w2"], F64).T
        if flags.sandwich:
            y2 = rms_norm(y2, w["n_ffn_post"], eps)
        out[sel] = x1 + g2[b] * y2
    return out


# ------------------------------------------------------------------------- the stack
def timestep_embedding(t, w, dim: int = 256, t_scale: float = 1000.0,
                       max_period: float = 10000.0):
    """temb = Linear(SiLU(Linear([cos | sin](t_scale * t * freqs)))) (R5)."""
    t = np.asarray(t, F64).reshape(-1)
    half = dim // 2
    freqs = np.exp(-math.log(max_period) * np.arange(half, dtype=F64) / half)
    args = t_scale * t[:, None] * freqs[None, :]
    emb = np.concatenate([np.cos(args), np.sin(args)], axis=1)
    h = silu(emb @ np.asarray(w["w_t1"], F64).T + np.asarray(w["b_t1"], F64))
    return h @ np.asarray(w["w_t2"], F64).T + np.asarray(w["b_t2"], F64)


def branch_positions(grid_h, grid_w, n_cap):
    """[image | caption] positions of one branch: caption k -> (k + 1, 0, 0), image
    cell (h, w) -> (n_cap + 1, h, w).  Each branch has its own caption RoPE
    ([CoreAI] "The three things...", item 3)."""
    pos = []
    for hh in range(grid_h):
        for ww in range(grid_w):
            pos.append((n_cap + 1, hh, ww))
    for kk in range(n_cap):
        pos.append((kk + 1, 0, 0))
    return np.asarray(pos, np.int64)


def caption_embed(caps, n_valid, n_cap, w, eps: float = 1e-5):
    """RMSNorm + Linear over valid caption rows, pad rows <- learned pad vector (R8;
    [CoreAI] "The three things...", item 3: pad to round_up(L, 32))."""
    D = np.asarray(w["b_cap"]).shape[0]
    out = np.empty((n_cap, D))
    if n_valid > 0:
        out[:n_valid] = (rms_norm(caps, w["w_capnorm"], eps) @ np.asarray(w["w_cap"], F64).T
                         + np.asarray(w["b_cap"], F64))
    out[n_valid:] = np.asarray(w["pad_vec"], F64)
    return out


def final_layer(x_img, temb_b, w):
    """LayerNorm_noaffine(x) * (1 + W_f temb + b_f) -> Linear(D, 64) (R6)."""
    scale = np.asarray(temb_b, F64) @ np.asarray(w["w_fada"], F64).T + np.asarray(w["b_fada"], F64)
    a = layer_norm_noaffine(x_img, 1e-6) * (1.0 + scale)
    return a @ np.asarray(w["w_final"], F64).T + np.asarray(w["b_final"], F64)


def stack_forward(case, W, d, flags: Flags = Flags(), trace=None):
    """Full DiT forward over a cond/uncond batch of branches.

    [CoreAI] DiT row: x-embed + cap-embed, 2 noise-refiner blocks (adaLN, image
    tokens only), 2 context-refiner blocks (no adaLN, caption only), 30 main blocks
    over the concatenated sequence, final layer.  The number of blocks of each kind
    is taken from W["block_kinds"].  Returns [B, n_img, patch_dim].
    """
    gh, gw = case["grid"]
    n_img = gh * gw
    n_caps, n_valids = case["n_caps"], case["n_valids"]
    B = len(n_caps)
    temb = timestep_embedding(case["t"], W, d.temb_dim)
    x_img = [np.asarray(case["patches"][b], F64) @ np.asarray(W["w_x"], F64).T
             + np.asarray(W["b_x"], F64) for b in range(B)]
    cap_off = np.concatenate([[0], np.cumsum(n_valids)]).astype(np.int64)
    x_cap = [caption_embed(case["caps"][cap_off[b]:cap_off[b + 1]], n_valids[b], n_caps[b], W)
             for b in range(B)]
    pos = [branch_positions(gh, gw, n_caps[b]) for b in range(B)]
    kinds = W["block_kinds"]
    flags_ctx = Flags(adaln=False, sandwich=flags.sandwich, qk_norm=flags.qk_norm,
                      tanh_gate=flags.tanh_gate)
    img_cu = np.arange(B + 1) * n_img
    cap_cu = np.concatenate([[0], np.cumsum(n_caps)])
    xi = np.concatenate(x_img, axis=0)
    xc = np.concatenate(x_cap, axis=0)
    pi = np.concatenate([p[:n_img] for p in pos], axis=0)
    pc = np.concatenate([p[n_img:] for p in pos], axis=0)
    for wb, kind in zip(W["blocks"], kinds):
        if kind == "noise":
            xi = block_forward(xi, img_cu, pi, temb, wb, d, flags)
        elif kind == "context":
            xc = block_forward(xc, cap_cu, pc, temb, wb, d, flags_ctx)
    xj = np.concatenate(
        [np.concatenate([xi[b * n_img:(b + 1) * n_img], xc[cap_cu[b]:cap_cu[b + 1]]], axis=0)
         for b in range(B)], axis=0)
    lens = [n_img + c for c in n_caps]
    cu = np.concatenate([[0], np.cumsum(lens)])
    pj = np.concatenate(pos, axis=0)
    for wb, kind in zip(W["blocks"], kinds):
        if kind == "main":
            xj = block_forward(xj, cu, pj, temb, wb, d, flags)
    out = np.stack([final_layer(xj[cu[b]:cu[b] + n_img], temb[b], W) for b in range(B)])
    if trace is not None:
        trace.update(temb=temb, x_joint=xj)
    return out


# ---------------------------------------------------------------------- the sampler
def sigma_schedule(n_steps: int = 8):
    """sigma_i = 3 (1 - u) / (3 (1 - u) + u), u = i / n_steps, i = 0..n_steps.

    [CoreAI] "Hosting it from Swift": closed form of the sampler schedule;
    [Port] scheduler contract: endpoint-preserving n + 1 points ending at 0.
    """
    u = np.arange(n_steps + 1, dtype=F64) / n_steps
    return 3.0 * (1.0 - u) / (3.0 * (1.0 - u) + u)


def cfg_velocity(v_pos, v_neg, g: float):
    """Negated classifier-free guidance: -(pos + g (pos - neg)).
    [CoreAI] "The three things...", item 2."""
    v_pos = np.asarray(v_pos, F64)
    v_neg = np.asarray(v_neg, F64)
    return -(v_pos + g * (v_pos - v_neg))


def euler_step(x, v, sigma_cur: float, sigma_next: float):
    """FlowMatchEuler update x + (sigma_next - sigma_cur) v ([CoreAI] Sampler row)."""
    return np.asarray(x, F64) + (sigma_next - sigma_cur) * np.asarray(v, F64)


def patchify(latent):
    """[C, 2h, 2w] latent -> [h*w, 4C] tokens, row-major over (h, w), feature
    f = (dy * 2 + dx) * C + c ([CoreAI] "Hosting it from Swift": patchify order)."""
    latent = np.asarray(latent)
    C, H2, W2 = latent.shape
    h, w = H2 // 2, W2 // 2
    out = np.empty((h * w, 4 * C), dtype=latent.dtype)
    for hi in range(h):
        for wi in range(w):
            for dy in range(2):
                for dx in range(2):
                    f0 = (dy * 2 + dx) * C
                    out[hi * w + wi, f0:f0 + C] = latent[:, 2 * hi + dy, 2 * wi + dx]
    return out


def unpatchify(tokens, C, h, w):
    tokens = np.asarray(tokens)
    out = np.empty((C, 2 * h, 2 * w), dtype=tokens.dtype)
    for hi in range(h):
        for wi in range(w):
            for dy in range(2):
                for dx in range(2):
                    f0 = (dy * 2 + dx) * C
                    out[:, 2 * hi + dy, 2 * wi + dx] = tokens[hi * w + wi, f0:f0 + C]
    return out


def sample(latent, cond, uncond, W, d, g: float = 1.0, n_steps: int = 8,
           flags: Flags = Flags()):
    """8-step FlowMatchEuler sampler with negated CFG on one latent [C, 2h, 2w].

    cond / uncond: dicts with "caps", "n_cap", "n_valid".  For each step i < n_steps
    the DiT is evaluated on both branches at t = 1 - sigma_i (R7); there is no call at
    the final sigma = 0 ([Port] scheduler contract).
    """
    C = latent.shape[0]
    gh, gw = latent.shape[1] // 2, latent.shape[2] // 2
    z = patchify(np.asarray(latent, F64))
    sig = sigma_schedule(n_steps)
    for i in range(n_steps):
        t = 1.0 - sig[i]
        case = {
            "grid": (gh, gw), "patches": np.stack([z, z]),
            "caps": np.concatenate([cond["caps"], uncond["caps"]], axis=0),
            "n_caps": [cond["n_cap"], uncond["n_cap"]],
            "n_valids": [cond["n_valid"], uncond["n_valid"]],
            "t": np.array([t, t]),
        }
        out = stack_forward(case, W, d, flags)
        v = cfg_velocity(out[0], out[1], g)
        z = euler_step(z, v, sig[i], sig[i + 1])
    return unpatchify(z, C, gh, gw)


def block_flops(T_lens, d):
    """Algorithmic FLOPs of one block: 2 * tokens * D * (3D + D + 2F + F) GEMMs plus
    4 * D * L^2 attention per branch (QK^T and PV)."""
    D, F = d.dim, d.ffn_hidden
    T = int(sum(T_lens))
    return 2 * T * D * (3 * D + D + 3 * F) + sum(4 * D * int(L) ** 2 for L in T_lens)

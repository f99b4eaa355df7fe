#!/usr/bin/env python
"""Benchmark of the Z-Image-Turbo single-stream DiT hot path on B200.

One step = one sampler step of the 1024x1024 workload: the 34-block DiT forward
(2 noise-refiner + 2 context-refiner + 30 main blocks + final layer) over the
cond/uncond pair (4096 image tokens each, captions padded to 128 and 32 tokens)
through zdit_stack_forward, then the fused negated-CFG FlowMatchEuler update
through zdit_euler_cfg_step.  Metric: DiT forward TFLOP/s (algorithmic FLOPs of the
forward / device time), with ms per step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (launched by torch.distributed.run) every rank runs an independent
replica (the DiT forward has no data-path exchange on one image; images are
independent), timings are the max over ranks, and `value` is the whole-job rate.
`--impl reference` times the CPU float64 oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

D, H, HD, F, E = 3840, 30, 128, 10240, 256
PATCH, CAP = 64, 2560
GRID = (64, 64)
N_CAPS, N_VALIDS = (128, 32), (100, 1)
KINDS = ["noise"] * 2 + ["context"] * 2 + ["main"] * 30
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
WORKLOAD = ("1024x1024 DiT forward, 34 blocks (2 noise-refiner + 2 context-refiner + 30 main + final), "
            "cond/uncond pair: 4096 image tokens each + captions 128 (100 valid) / 32 (1 valid), "
            "width 3840, 30x128 heads, SwiGLU 10240, then fused negated-CFG Euler update (g=1)")


def forward_flops() -> float:
    """Algorithmic FLOPs of one DiT forward of the benchmark workload."""
    n_img = GRID[0] * GRID[1]

    def block(lengths):
        T = sum(lengths)
        return 2.0 * T * D * (3 * D + D + 3 * F) + sum(4.0 * D * L * L for L in lengths)

    f = 2 * block([n_img] * 2) + 2 * block(list(N_CAPS)) + 30 * block([n_img + c for c in N_CAPS])
    f += 2.0 * 2 * n_img * PATCH * D + 2.0 * sum(N_VALIDS) * CAP * D + 2.0 * 2 * n_img * D * PATCH
    f += 32 * 2.0 * 2 * E * 4 * D + 2.0 * 2 * E * D
    return f


# DRAM bytes per launch of the dominant kernel (gate/up GEMM of a main block, 8352 x 20480
# x 3840), from one ncu capture of that kernel (dram__bytes_read.sum + dram__bytes_write.sum),
# valid for the GEMM sources with this hash only; any change to them makes the figure stale
# (reported null).
# The headline metric, shared by this implementation's line and the reference arm's.
METRIC = "DiT forward TFLOP/s (1024^2, 34-block step, bf16, 1 B200)"

NCU_TRAFFIC = {"kernel": "gemm_gate_up_swiglu", "bytes": 402328576 + 155948288, "src_hash": "d230e725b4f8169d"}


# What bounds each kernel kind of the library's profiler (its `kernels` table).
KERNEL_BOUND = {"gemm_qkv_rope": "tensor", "gemm_out_proj": "tensor", "gemm_gate_up_swiglu": "tensor",
                "gemm_down_proj": "tensor", "attention": "tensor", "residual_norm": "hbm",
                "norm_modulate": "hbm", "adaln_gemv": "hbm", "euler_cfg": "hbm",
                "gemm_embed_final": "latency", "rope_table": "latency", "misc": "latency"}


def gemm_src_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in ("gemm.cu", "ptx.cuh", "internal.h"):
        with open(os.path.join(ROOT, "stream_diffusion_transformer_s3_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def aggregate_ranks(ms, ms_e2e, flops, world, dist=None, device="cpu"):
    """Whole-job rates of `world` independent replicas: each rank ran the same work;
    the job time is the slowest rank's (max over ranks, through the process group)."""
    import torch
    if world > 1 and dist is not None:
        t = torch.tensor([ms, ms_e2e], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms, ms_e2e = float(t[0]), float(t[1])
    value = world * flops / (ms * 1e-3) / 1e12
    value_e2e = world * flops / (ms_e2e * 1e-3) / 1e12
    return ms, ms_e2e, value, value_e2e


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            return json.load(fh), "measured"
    return PEAKS_FALLBACK, "fallback"


# ------------------------------------------------------------------ clocks sampling
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.path = os.path.join("/tmp", f"zdit_clocks_{os.getpid()}.csv")
        self.proc = None
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", gpu_id, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ our arm
SAMPLER_WORKLOAD = ("1024x1024 image: 8-step FlowMatchEuler sampler with negated CFG (g=1) on the "
                    "cond/uncond pair, 34-block DiT, caption stream computed once (t-independent)")
BLOCK_WORKLOAD = ("one main DiT block of the 1024x1024 workload: joint cond/uncond sequence 4224 + 4128 "
                  "tokens, width 3840, 30x128 heads, SwiGLU 10240, adaLN + sandwich norm")


HBM_WORKLOAD = ("the HBM-bound small kernels of one 1024x1024 step at their real sizes: the adaLN projections "
                "of the 32 adaLN blocks in one launch (32 x bf16 [15360, 256], cond/uncond temb), the RoPE "
                "cos/sin tables of the joint sequence (8352 tokens x 64 pairs) and the fused negated-CFG Euler "
                "update of the 16 x 128 x 128 latent")


ATTN_SWEEP_IMG = (1024, 4096, 9216, 16384)
ATTN_SWEEP_CAP = (32, 128, 512)   # cond caption length; uncond 32
ATTN_SWEEP_LARGEST = (16384, (512, 32))
ATTN_WORKLOAD = ("joint attention alone: cond/uncond branches of 16384 image tokens + captions 512 / 32, "
                 "30 x 128 heads, Q/K/V N(0,1) bf16; sweep over image tokens {1024, 4096, 9216, 16384} x "
                 "cond caption {32, 128, 512}")


def attention_sweep(torch, Z, device, reps=3, per=10):
    """TFLOP/s of zdit_joint_attention over the image-token x caption-length grid (CUDA
    events around `per` back-to-back launches, median of `reps`, after 2 warm-up launches)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(7)
    out = {}
    for n_i in ATTN_SWEEP_IMG:
        for c in ATTN_SWEEP_CAP:
            lens = [n_i + c, n_i + 32]
            vl = Z.DeviceVarlen([0, lens[0], lens[0] + lens[1]], device=device)
            T = vl.total
            q, k, v = (torch.randn(T, H * HD, generator=g).to(device=device, dtype=torch.bfloat16)
                       for _ in range(3))
            o = torch.empty(T, H * HD, device=device, dtype=torch.bfloat16)
            for _ in range(2):
                Z.zdit_joint_attention(q, k, v, o, vl, H)
            times = []
            for _ in range(reps):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                for _ in range(per):
                    Z.zdit_joint_attention(q, k, v, o, vl, H)
                e1.record()
                torch.cuda.synchronize()
                times.append(e0.elapsed_time(e1) / per)
            ms = statistics.median(times)
            out[f"{n_i}+{c}/{n_i}+32"] = round(sum(4.0 * D * L * L for L in lens) / (ms * 1e-3) / 1e12, 1)
            del q, k, v, o
    return out


def build_block(torch, Z, device, seed=99):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    bf = lambda *s: (torch.randn(*s, generator=g, device=device) * 0.02).to(torch.bfloat16)
    nrm = lambda n: 1.0 + 0.1 * torch.randn(n, generator=g, device=device)
    t = {"w_qkv": bf(3 * D, D), "w_out": bf(D, D), "w_gate_up": bf(2 * F, D), "w_down": bf(D, F),
         "n_attn": nrm(D), "n_attn_post": nrm(D), "n_ffn": nrm(D), "n_ffn_post": nrm(D),
         "w_ada": bf(4 * D, E), "b_ada": torch.randn(4 * D, generator=g, device=device) * 0.02}
    return Z.DeviceBlock.from_tensors(t)


def build_model(torch, Z, device, seed=1234):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    bf = lambda *s: (torch.randn(*s, generator=g, device=device) * 0.02).to(torch.bfloat16)
    f32 = lambda *s: torch.randn(*s, generator=g, device=device) * 0.02
    nrm = lambda n: 1.0 + 0.1 * torch.randn(n, generator=g, device=device)
    blocks = []
    for kind in KINDS:
        t = {"w_qkv": bf(3 * D, D), "w_out": bf(D, D), "w_gate_up": bf(2 * F, D), "w_down": bf(D, F),
             "n_attn": nrm(D), "n_attn_post": nrm(D), "n_ffn": nrm(D), "n_ffn_post": nrm(D)}
        if kind != "context":
            t["w_ada"] = bf(4 * D, E)
            t["b_ada"] = f32(4 * D)
        blocks.append(Z.DeviceBlock.from_tensors(t))
    W = {"w_x": bf(D, PATCH), "b_x": f32(D), "w_capnorm": nrm(CAP), "w_cap": bf(D, CAP), "b_cap": f32(D),
         "pad_vec": torch.randn(D, generator=g, device=device), "w_t1": bf(E, E), "b_t1": f32(E),
         "w_t2": bf(E, E), "b_t2": f32(E), "w_fada": bf(D, E), "b_fada": f32(D), "w_final": bf(PATCH, D),
         "b_final": f32(PATCH)}
    dims = Z.Dims()
    return Z.DeviceStack(W, dims, 2, 2, 30, patch_dim=PATCH, cap_dim=CAP, blocks=blocks)


def run_ours(args):
    import torch
    import torch.distributed as dist
    import stream_diffusion_transformer_s3_b200 as Z

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=device)

    n_img = GRID[0] * GRID[1]
    g = torch.Generator(device="cpu")
    g.manual_seed(42)
    if args.workload == "stack":
        stack = build_model(torch, Z, device)
        # latent noise N(0, 1), 16 x 128 x 128, kept in patch-token layout [4096, 64]
        latent = torch.randn(16, 128, 128, generator=g).to(device)
        z = torch.empty(n_img, PATCH, device=device)
        Z.zdit_patchify(latent, z)
        caps = torch.randn(sum(N_VALIDS), CAP, generator=g).to(device)
        call = Z.StackCall(GRID, N_CAPS, N_VALIDS, [0.0, 0.0], z, caps, shared_patches=True)
        ws = torch.empty(Z.stack_workspace_bytes(stack, call), dtype=torch.uint8, device=device)
        out = torch.empty(2, n_img, PATCH, device=device)
        sig = Z.zdit_sigma_schedule(8)
        inputs = [z, caps]   # per-step inputs (e2e copies them in) ...
        result = z           # ... and the per-step result copied out
        flops = forward_flops()

        def step(i):
            s0, s1 = sig[i % 8], sig[i % 8 + 1]
            call.set_t([1.0 - s0, 1.0 - s0])
            Z.zdit_stack_forward(stack, call, out, ws)
            Z.zdit_euler_cfg_step(z, out[0], out[1], 1.0, s0, s1)
    elif args.workload == "attention":
        # joint attention alone at the largest size of the sweep: 16384 image tokens, caption
        # 512 (cond) / 32 (uncond), 30 heads x 128; Q, K, V N(0, 1) in bf16 (after RoPE)
        n_i, caps_ = ATTN_SWEEP_LARGEST
        lens = [n_i + caps_[0], n_i + caps_[1]]
        vl = Z.DeviceVarlen([0, lens[0], lens[0] + lens[1]], device=device)
        T = vl.total
        q, k, v = (torch.randn(T, H * HD, generator=g).to(device=device, dtype=torch.bfloat16) for _ in range(3))
        o = torch.empty(T, H * HD, device=device, dtype=torch.bfloat16)
        inputs, result = [q, k, v], o
        flops = sum(4.0 * D * L * L for L in lens)

        def step(i):
            Z.zdit_joint_attention(q, k, v, o, vl, H)
    elif args.workload == "sampler":
        # one 1024x1024 image: 8 sampler steps on the cond/uncond pair in one call
        stack = build_model(torch, Z, device)
        latent0 = torch.randn(16, 128, 128, generator=g).to(device)
        latent = latent0.clone()
        caps = torch.randn(sum(N_VALIDS), CAP, generator=g).to(device)
        call = Z.StackCall(GRID, N_CAPS, N_VALIDS, [0.0, 0.0], latent, caps)
        ws = torch.empty(Z.sample_workspace_bytes(stack, call), dtype=torch.uint8, device=device)
        inputs, result = [latent], latent
        n_img_ = GRID[0] * GRID[1]
        ctx_flops = 2 * (2.0 * sum(N_CAPS) * D * (3 * D + D + 3 * F) + sum(4.0 * D * c * c for c in N_CAPS))
        noise_flops = 2 * (2.0 * n_img_ * D * (3 * D + D + 3 * F) + 4.0 * D * n_img_ * n_img_)
        # executed work: 8 forwards, the caption stream once, the noise refiner once per
        # step for both branches unless deduplicated
        flops = 8 * forward_flops() - 7 * ctx_flops - (8 * noise_flops if args.dedup else 0)

        def step(i):
            latent.copy_(latent0)
            Z.zdit_sample(stack, call, latent, ws, n_steps=8, guidance=1.0, cache_context=True,
                          dedup_noise=args.dedup, use_graph=args.graph)
    elif args.workload == "hbm":
        # the small bandwidth-bound kernels of one step at their real sizes; the adaLN
        # weights (251.7 MB) exceed L2, the tables and the latent are the step's own sizes
        from stream_diffusion_transformer_s3_b200 import synth
        n_blk = sum(1 for k in KINDS if k != "context")
        w_ada = [(torch.randn(4 * D, E, generator=g) * 0.02).to(device=device, dtype=torch.bfloat16)
                 for _ in range(n_blk)]
        b_ada = [torch.randn(4 * D, generator=g).to(device) * 0.02 for _ in range(n_blk)]
        mods = [torch.empty(2, 4 * D, device=device) for _ in range(n_blk)]
        temb = torch.randn(2, E, generator=g).to(device)
        pos = torch.from_numpy(synth.joint_positions(GRID[0], GRID[1], list(N_CAPS))).to(device)
        T = pos.shape[0]
        cs = torch.empty(T, HD // 2, device=device)
        sn = torch.empty_like(cs)
        dims = Z.Dims()
        z = torch.randn(n_img, PATCH, generator=g).to(device)
        vel = torch.randn(2, n_img, PATCH, generator=g).to(device)
        sig = Z.zdit_sigma_schedule(8)
        inputs, result = [temb, z], z
        flops = 0.0
        hbm_bytes = (n_blk * (4 * D * E * 2 + 4 * D * 4 + 2 * 4 * D * 4) + T * (12 + 2 * 4 * HD // 2)
                     + n_img * PATCH * 16)

        def step(i):
            Z.zdit_adaln_project(w_ada, b_ada, mods, temb)
            Z.zdit_rope_table(pos, dims.rope_axes, dims.rope_theta, cs, sn)
            Z.zdit_euler_cfg_step(z, vel[0], vel[1], 1.0, sig[i % 8], sig[i % 8 + 1])
    else:
        # one main block of the workload: the joint cond/uncond sequence (4224 + 4128)
        from stream_diffusion_transformer_s3_b200 import synth
        blk = build_block(torch, Z, device)
        lens = [n_img + c for c in N_CAPS]
        vl = Z.DeviceVarlen([0, lens[0], lens[0] + lens[1]], device=device)
        T = vl.total
        x = torch.randn(T, D, generator=g).to(device)
        temb = torch.randn(2, E, generator=g).to(device)
        pos = torch.from_numpy(synth.joint_positions(GRID[0], GRID[1], list(N_CAPS))).to(device)
        cs = torch.empty(T, HD // 2, device=device)
        sn = torch.empty_like(cs)
        dims = Z.Dims()
        Z.zdit_rope_table(pos, dims.rope_axes, dims.rope_theta, cs, sn)
        fl = Z.flags_of()
        ws = torch.empty(Z.block_workspace_bytes(dims, fl, T, 2), dtype=torch.uint8, device=device)
        inputs, result = [x], x
        flops = 2.0 * T * D * (3 * D + D + 3 * F) + sum(4.0 * D * L * L for L in lens)

        def step(i):
            Z.zdit_block_forward(dims, fl, blk, vl, x, temb, cs, sn, ws)

    def barrier():
        if world > 1:
            dist.barrier()

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if Z.zdit_device_status() != 0:
        raise RuntimeError("device error during warm-up")

    uuid = str(torch.cuda.get_device_properties(device).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")
    time.sleep(0.3)
    stream = torch.cuda.current_stream()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = Z.zdit_launch_count()
    barrier()
    torch.cuda.synchronize()
    ev0.record(stream)
    for i in range(args.steps):
        step(args.warmup + i)
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    launches = Z.zdit_launch_count() - launches0
    clocks = sampler.stop()
    ms = ev0.elapsed_time(ev1) / args.steps
    if Z.zdit_device_status() != 0:
        raise RuntimeError("device error during the timed region")

    # Per-kernel durations: the same K steps again under the library's event profiler
    # (an event pair around every launch).  Kept out of the timed region above because
    # the events serialise the kernels that otherwise start early (programmatic launch,
    # residual rows started band by band).
    Z.zdit_profile_begin(65536)
    torch.cuda.synchronize()
    for i in range(args.steps):
        step(args.warmup + args.steps + i)
    torch.cuda.synchronize()
    kernels = Z.zdit_profile_end()
    if Z.zdit_device_status() != 0:
        raise RuntimeError("device error during the profiled pass")

    # end to end: pinned host inputs in, result out, every step
    h_in = [t.cpu().pin_memory() for t in inputs]
    h_out = torch.empty(result.shape, pin_memory=True)
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        for dst, src in zip(inputs, h_in):
            dst.copy_(src, non_blocking=True)
        step(i)
        h_out.copy_(result, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms_e2e = e0.elapsed_time(e1) / args.steps

    ms, ms_e2e, value, value_e2e = aggregate_ranks(ms, ms_e2e, flops, world, dist if world > 1 else None, device)

    peaks, peak_src = load_peaks()
    # A region that ran under the power cap (sw_power_cap seen in the clock samples) or
    # lasted a few seconds compares with the sustained GEMM peak (measured the same way,
    # a loop under the cap); a short uncapped region with the burst peak.
    capped = clocks is not None and "sw_power_cap" in clocks.get("reasons", [])
    sustained = capped or ms * args.steps > 3000.0
    peak_kind = "sustained" if sustained else "burst"
    peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    dom = max(kernels.items(), key=lambda kv: kv[1]["total_ms"]) if kernels else None
    roofline = None
    if dom is not None and args.workload == "hbm":
        name, k = dom
        achieved = k["bytes"] / (k["total_ms"] * 1e-3) / 1e9
        roofline = {"kernel": name, "bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                    "peak_source": f"{peak_src} copy bandwidth", "traffic": args.traffic,
                    "launches_per_step": k["launches"] / args.steps,
                    "ms_per_launch": k["total_ms"] / k["launches"],
                    "timing": "CUDA events around each launch, in a pass of the same steps right "
                              "after the timed one"}
    elif dom is not None:
        name, k = dom
        if k["flops"] > 0:
            achieved = k["flops"] / (k["total_ms"] * 1e-3) / 1e12
            roofline = {"kernel": name, "bound": "tensor", "achieved": round(achieved, 1), "peak": peak,
                        "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                        "peak_source": f"{peak_src} bf16 {peak_kind}",
                        "traffic": (args.traffic if args.traffic is not None else
                                    NCU_TRAFFIC["bytes"] if (name == NCU_TRAFFIC["kernel"] and
                                                             gemm_src_hash() == NCU_TRAFFIC["src_hash"]) else None),
                        "launches_per_step": k["launches"] / args.steps,
                        "ms_per_launch": k["total_ms"] / k["launches"],
                        "timing": "CUDA events around each launch, in a pass of the same steps right "
                                  "after the timed one"}
    kern_summary = {}
    total_k = sum(v["total_ms"] for v in kernels.values()) or 1.0
    for n, k in sorted(kernels.items(), key=lambda kv: -kv[1]["total_ms"]):
        row = {"launches": k["launches"], "ms_per_step": round(k["total_ms"] / args.steps, 3),
               "share": round(k["total_ms"] / total_k, 4)}
        if k["flops"] > 0:
            row["tflops"] = round(k["flops"] / (k["total_ms"] * 1e-3) / 1e12, 1)
        if k["bytes"] > 0:
            row["gbs"] = round(k["bytes"] / (k["total_ms"] * 1e-3) / 1e9, 1)
        # the bound of each kernel kind and its fraction of the matching measured peak (the
        # projections' and attention's bf16 peak as above; the row kernels' copy bandwidth)
        if n in KERNEL_BOUND:
            row["bound"] = KERNEL_BOUND[n]
            if KERNEL_BOUND[n] == "tensor" and "tflops" in row:
                row["frac"] = round(row["tflops"] / peak, 4)
            elif KERNEL_BOUND[n] == "hbm" and "gbs" in row:
                row["frac"] = round(row["gbs"] / peaks["hbm_gbs"], 4)
        kern_summary[n] = row

    if rank == 0:
        res = {
            "metric": METRIC,
            "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": {"stack": WORKLOAD, "block": BLOCK_WORKLOAD,
                                    "sampler": SAMPLER_WORKLOAD, "attention": ATTN_WORKLOAD,
                                    "hbm": HBM_WORKLOAD}[args.workload],
                       "global_batch": 2 * world, "seq_len": [n_img + c for c in N_CAPS],
                       "flops_per_forward": flops, "parallelism": f"replicas x{world}",
                       "l2": ("working set larger than L2 (12.3 GB of bf16 weights streamed per step)" if args.workload == "stack" else "working set larger than L2 (354 MB weights + 128 MB residual + 448 MB activations per block)"),
                       "frac_of_peak": round(value / world / peak, 4), "peak_kind": peak_kind},
            "roofline": roofline,
            "kernels": kern_summary,
            "gpu_launches": launches,
            "clocks": clocks,
            "e2e": {"value": round(value_e2e, 2), "unit": "TFLOP/s", "ms_per_step": round(ms_e2e, 3),
                    "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in h_in),
                    "d2h_bytes_per_step": h_out.numel() * h_out.element_size()},
        }
        if args.workload == "hbm":
            res["metric"] = "HBM-bound kernels of the 1024^2 step: algorithmic GB/s (1 B200)"
            res["value"] = round(world * hbm_bytes / (ms * 1e-3) / 1e9, 1)
            res["unit"] = "GB/s"
            res["dtype"] = "f32 / bf16 weights"
            res["config"]["bytes_per_step"] = hbm_bytes
            res["config"]["l2"] = ("adaLN weights (251.7 MB) larger than L2; the tables and the latent are the "
                                   "step's own few MB and stay L2-resident, as in the step")
            res["e2e"] = {"value": round(world * hbm_bytes / (ms_e2e * 1e-3) / 1e9, 1), "unit": "GB/s",
                          "ms_per_step": round(ms_e2e, 3), "h2d_bytes_per_step": res["e2e"]["h2d_bytes_per_step"],
                          "d2h_bytes_per_step": res["e2e"]["d2h_bytes_per_step"]}
            res["config"].pop("frac_of_peak", None)
        if args.workload == "block":
            res["metric"] = "DiT main-block forward TFLOP/s (1024^2 cond/uncond sequence, bf16, 1 B200)"
        if args.workload == "attention":
            res["metric"] = "joint attention TFLOP/s (30 x 128 heads, cond/uncond branches, bf16, 1 B200)"
            res["config"]["seq_len"] = [ATTN_SWEEP_LARGEST[0] + c for c in ATTN_SWEEP_LARGEST[1]]
            res["config"]["l2"] = "Q, K, V and O (1 GB) larger than L2"
            res["sweep"] = attention_sweep(torch, Z, device)
        if args.workload == "sampler":
            res["metric"] = "s per 1024^2 image, 8-step negated-CFG sampler (bf16, 1 B200)"
            res["value"] = round(ms / 1e3, 4)
            res["unit"] = "s/image"
            res["higher_is_better"] = False
            res["tflops"] = round(value, 2)
            res["e2e"] = {"value": round(ms_e2e / 1e3, 4), "unit": "s/image", "ms_per_step": round(ms_e2e, 3),
                          "h2d_bytes_per_step": res["e2e"]["h2d_bytes_per_step"],
                          "d2h_bytes_per_step": res["e2e"]["d2h_bytes_per_step"]}
            res["config"]["workload"] = (SAMPLER_WORKLOAD + (", noise refiner deduplicated across branches"
                                                             if args.dedup else "")
                                         + (", captured as one CUDA graph and replayed" if args.graph else ""))
        if world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = (cpu_baseline_attention() if args.workload == "attention"
                                   else cpu_baseline_hbm() if args.workload == "hbm"
                                   else cpu_baseline_block(seconds=None))
        print(json.dumps(res), flush=True)
    if world > 1:
        dist.destroy_process_group()


# ------------------------------------------------------------------ CPU oracle leg
def _oracle_sample():
    """One full-width main block of the workload on its uncond branch (L = 4128)."""
    import numpy as np
    from stream_diffusion_transformer_s3_b200 import synth
    case = synth.block_case(11, synth.FULL, GRID[0], GRID[1], [N_CAPS[1]], [N_VALIDS[1]])
    L = GRID[0] * GRID[1] + N_CAPS[1]
    flops = 2.0 * L * D * (3 * D + D + 3 * F) + 4.0 * D * L * L
    return case, flops


def _cores():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"), default=0)
        if n:
            return int(n)
    except Exception:
        pass
    return os.cpu_count()


def cpu_baseline_block(seconds=None):
    import oracle as O
    case, flops = _oracle_sample()
    t0 = time.perf_counter()
    O.block_forward(case["x"], case["cu_seqlens"], case["pos"], case["temb"], case["weights"],
                    __import__("stream_diffusion_transformer_s3_b200.synth", fromlist=["FULL"]).FULL)
    dt = time.perf_counter() - t0
    return {"value": round(flops / dt / 1e12, 5), "unit": "TFLOP/s", "cores": _cores(), "kind": "oracle",
            "sample": f"one full-width main block of the workload on its uncond branch (L=4128 tokens), "
                      f"NumPy float64 oracle, {dt:.1f} s"}


def cpu_baseline_hbm():
    """The oracle's steps behind the hbm workload on its full sizes: the adaLN vectors of the
    32 adaLN blocks, the rotary angles (cos / sin) of the joint sequence, the negated-CFG
    Euler update of the latent; algorithmic bytes of the GPU kernels over the oracle's time."""
    import numpy as np
    import oracle as O
    from stream_diffusion_transformer_s3_b200 import synth
    n_blk = sum(1 for k in KINDS if k != "context")
    temb = synth.randn(5, 1, (2, E))
    ws = [{"w_ada": synth.bf16_round(synth.randn(5, 10 + i, (4 * D, E), 0.02)), "b_ada": synth.randn(5, 100 + i, (4 * D,))}
          for i in range(n_blk)]
    pos = synth.joint_positions(GRID[0], GRID[1], list(N_CAPS))
    n = GRID[0] * GRID[1] * PATCH
    x, vp, vn = (synth.randn(5, 200 + i, (n,)) for i in range(3))
    t0 = time.perf_counter()
    for w in ws:
        O.adaln_vectors(temb, w, D, O.Flags())
    phi = O.rope_angles(pos)
    np.cos(phi), np.sin(phi)
    O.euler_step(x, O.cfg_velocity(vp, vn, 1.0), 1.0, 0.95)
    dt = time.perf_counter() - t0
    T = pos.shape[0]
    nbytes = n_blk * (4 * D * E * 2 + 4 * D * 4 + 2 * 4 * D * 4) + T * (12 + 2 * 4 * HD // 2) + n * 16
    return {"value": round(nbytes / dt / 1e9, 2), "unit": "GB/s", "cores": _cores(), "kind": "oracle",
            "sample": f"the whole hbm workload once (32 adaLN projections, the joint RoPE angles, one "
                      f"CFG-Euler update), NumPy float64 oracle, {dt:.2f} s"}


def cpu_baseline_attention():
    """The oracle's joint attention on a bounded sample of the attention workload: one head
    of the cond branch at 4096 + 512 tokens."""
    import numpy as np
    import oracle as O
    from stream_diffusion_transformer_s3_b200 import synth
    L = 4096 + 512
    q, k, v = (synth.bf16_round(synth.randn(11, i, (L, HD))).astype(np.float64) for i in range(3))
    t0 = time.perf_counter()
    O.softmax_attention(q, k, v)
    dt = time.perf_counter() - t0
    return {"value": round(4.0 * HD * L * L / dt / 1e12, 5), "unit": "TFLOP/s", "cores": _cores(),
            "kind": "oracle", "sample": f"one head of the cond branch at 4096 + 512 tokens, NumPy float64 "
                                        f"oracle, {dt:.1f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle as O
    from stream_diffusion_transformer_s3_b200 import synth
    case, flops = _oracle_sample()
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        O.block_forward(case["x"], case["cu_seqlens"], case["pos"], case["temb"], case["weights"], synth.FULL)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    sec = sum(times) / len(times)
    value = flops / sec / 1e12
    sample = ("each step: one full-width main block of the workload on its uncond branch (L=4128 tokens), "
              "NumPy float64 oracle on the host cores")
    res = {"metric": METRIC, "impl": "reference",
           "value": round(value, 5), "unit": "TFLOP/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(sec * 1e3, 1),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic", "config": {"workload": WORKLOAD, "sample": sample},
           "cpu_baseline": {"value": round(value, 5), "unit": "TFLOP/s", "cores": _cores(), "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": round(value, 5), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", choices=["stack", "block", "sampler", "attention", "hbm"], default="stack",
                    help="stack: the full DiT step (default); block: one main block (for kernel captures); "
                         "sampler: one whole 8-step image per step; attention: joint attention alone at "
                         "16384 image tokens, with a sweep over sequence lengths; hbm: the bandwidth-bound "
                         "small kernels of one step (adaLN projections, RoPE tables, CFG-Euler)")
    ap.add_argument("--graph", action="store_true",
                    help="sampler workload: the whole image as one captured CUDA graph, replayed")
    ap.add_argument("--dedup", action="store_true",
                    help="sampler workload: run the noise refiner once for both branches")
    ap.add_argument("--traffic", type=float, default=None,
                    help="dram bytes per launch of the dominant kernel from an ncu capture")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

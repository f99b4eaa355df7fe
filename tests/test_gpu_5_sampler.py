"""The 8-step FlowMatchEuler sampler with negated CFG driven through the public
calls (zdit_stack_forward on the cond/uncond pair, zdit_euler_cfg_step), at reduced
width so the oracle's float64 sampler finishes in seconds: latent 16 x 16 x 16
(8 x 8 patch grid), g = 1, endpoint-preserving 9-point schedule, no call at
sigma = 0."""
import pytest
import torch

import oracle as O
import stream_diffusion_transformer_s3_b200 as Z
from stream_diffusion_transformer_s3_b200 import synth
from _gpu import N_ROUND_BLOCK, assert_parity, dev, dims_of, host, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()


def _check(got_latent, ref_latent, label):
    # rows = patch tokens: the latents compared in the [h*w, 64] token layout
    assert_parity(O.patchify(got_latent), O.patchify(ref_latent), 2e-2, n_round=N_ROUND_BLOCK, label=label)


def test_eight_step_sampler_matches_oracle():
    d = synth.BlockDims(dim=256, n_heads=2, head_dim=128, ffn_hidden=384)
    W = synth.stack_weights(9, d, n_noise=2, n_context=2, n_main=2, cap_dim=128)
    latent = synth.latent_noise(42, (16, 16, 16))
    caps = synth.randn(9, 300, (46, 128))
    cond = {"caps": caps[:45], "n_cap": 64, "n_valid": 45}
    unc = {"caps": caps[45:], "n_cap": 32, "n_valid": 1}

    stack = Z.DeviceStack(W, dims_of(d), 2, 2, 2, patch_dim=64, cap_dim=128)
    z = torch.empty(64, 64, device="cuda")
    Z.zdit_patchify(dev(latent), z)
    call = Z.StackCall((8, 8), [64, 32], [45, 1], [0.0, 0.0], z, dev(caps), shared_patches=True)
    ws = torch.empty(Z.stack_workspace_bytes(stack, call), dtype=torch.uint8, device="cuda")
    out = torch.empty(2, 64, 64, device="cuda")
    sig = Z.zdit_sigma_schedule(8)
    calls = 0
    for i in range(8):
        call.set_t([1.0 - sig[i]] * 2)
        Z.zdit_stack_forward(stack, call, out, ws)
        calls += 1
        Z.zdit_euler_cfg_step(z, out[0], out[1], 1.0, sig[i], sig[i + 1])
    assert sig[8] == 0.0 and calls == 8
    result = torch.empty(16, 16, 16, device="cuda")
    Z.zdit_unpatchify(z, result)
    assert Z.zdit_device_status() == 0
    ref = O.sample(latent, cond, unc, W, d, g=1.0, n_steps=8)
    _check(host(result), ref, "sampler")


def _small_setup():
    d = synth.BlockDims(dim=256, n_heads=2, head_dim=128, ffn_hidden=384)
    W = synth.stack_weights(9, d, n_noise=2, n_context=2, n_main=2, cap_dim=128)
    latent = synth.latent_noise(42, (16, 16, 16))
    caps = synth.randn(9, 300, (46, 128))
    return d, W, latent, caps


@pytest.mark.parametrize("dedup", [False, True])
def test_sample_entry_point_matches_oracle(dedup):
    d, W, latent, caps = _small_setup()
    stack = Z.DeviceStack(W, dims_of(d), 2, 2, 2, patch_dim=64, cap_dim=128)
    call = Z.StackCall((8, 8), [64, 32], [45, 1], [0.0, 0.0], dev(caps), dev(caps))
    ws = torch.empty(Z.sample_workspace_bytes(stack, call), dtype=torch.uint8, device="cuda")
    lat = dev(latent)
    Z.zdit_sample(stack, call, lat, ws, n_steps=8, guidance=1.0, cache_context=True, dedup_noise=dedup)
    assert Z.zdit_device_status() == 0
    cond = {"caps": caps[:45], "n_cap": 64, "n_valid": 45}
    unc = {"caps": caps[45:], "n_cap": 32, "n_valid": 1}
    ref = O.sample(latent, cond, unc, W, d, g=1.0, n_steps=8)
    _check(host(lat), ref, f"zdit_sample dedup={dedup}")


def test_sample_non_square_latent():
    # latent 16 x 12 x 32 (6 x 16 patch grid) through the whole-image entry point
    d, W, _, caps = _small_setup()
    latent = synth.latent_noise(44, (16, 12, 32))
    stack = Z.DeviceStack(W, dims_of(d), 2, 2, 2, patch_dim=64, cap_dim=128)
    call = Z.StackCall((6, 16), [64, 32], [45, 1], [0.0, 0.0], dev(caps), dev(caps))
    ws = torch.empty(Z.sample_workspace_bytes(stack, call), dtype=torch.uint8, device="cuda")
    lat = dev(latent)
    Z.zdit_sample(stack, call, lat, ws, n_steps=8, guidance=1.0)
    assert Z.zdit_device_status() == 0
    cond = {"caps": caps[:45], "n_cap": 64, "n_valid": 45}
    unc = {"caps": caps[45:], "n_cap": 32, "n_valid": 1}
    ref = O.sample(latent, cond, unc, W, d, g=1.0, n_steps=8)
    _check(host(lat), ref, "zdit_sample, 6 x 16 grid")


def test_sample_single_branch_guidance_zero():
    d, W, latent, caps = _small_setup()
    stack = Z.DeviceStack(W, dims_of(d), 2, 2, 2, patch_dim=64, cap_dim=128)
    call = Z.StackCall((8, 8), [64], [45], [0.0], dev(caps), dev(caps[:45]))
    ws = torch.empty(Z.sample_workspace_bytes(stack, call), dtype=torch.uint8, device="cuda")
    lat = dev(latent)
    Z.zdit_sample(stack, call, lat, ws, n_steps=8, guidance=0.0)
    assert Z.zdit_device_status() == 0
    cond = {"caps": caps[:45], "n_cap": 64, "n_valid": 45}
    unc = {"caps": caps[45:], "n_cap": 32, "n_valid": 1}
    ref = O.sample(latent, cond, unc, W, d, g=0.0, n_steps=8)  # g = 0: v = -pos
    _check(host(lat), ref, "single branch, g = 0")


def test_sample_caching_is_bitwise_neutral():
    # the caption stream has no t dependence: computing it once equals recomputing it
    d, W, latent, caps = _small_setup()
    stack = Z.DeviceStack(W, dims_of(d), 2, 2, 2, patch_dim=64, cap_dim=128)
    call = Z.StackCall((8, 8), [64, 32], [45, 1], [0.0, 0.0], dev(caps), dev(caps))
    ws = torch.empty(Z.sample_workspace_bytes(stack, call), dtype=torch.uint8, device="cuda")
    a, b = dev(latent), dev(latent)
    Z.zdit_sample(stack, call, a, ws, cache_context=True)
    Z.zdit_sample(stack, call, b, ws, cache_context=False)
    assert Z.zdit_device_status() == 0
    assert torch.equal(a, b)


def test_sample_as_cuda_graph_is_bitwise_equal():
    # capture on the first call, replay on later ones; the replay reads the latent's new
    # contents through the same pointer
    d, W, latent, caps = _small_setup()
    stack = Z.DeviceStack(W, dims_of(d), 2, 2, 2, patch_dim=64, cap_dim=128)
    call = Z.StackCall((8, 8), [64, 32], [45, 1], [0.0, 0.0], dev(caps), dev(caps))
    ws = torch.empty(Z.sample_workspace_bytes(stack, call), dtype=torch.uint8, device="cuda")
    plain = dev(latent)
    Z.zdit_sample(stack, call, plain, ws, n_steps=8, guidance=1.0)
    lat = dev(latent)
    n0 = Z.zdit_launch_count()
    Z.zdit_sample(stack, call, lat, ws, n_steps=8, guidance=1.0, use_graph=True)    # capture + launch
    n1 = Z.zdit_launch_count()
    assert Z.zdit_device_status() == 0
    assert torch.equal(lat, plain)
    lat.copy_(dev(latent))
    Z.zdit_sample(stack, call, lat, ws, n_steps=8, guidance=1.0, use_graph=True)    # replay
    assert Z.zdit_device_status() == 0
    assert torch.equal(lat, plain)
    assert Z.zdit_launch_count() - n1 == n1 - n0 > 0
    other = dev(synth.latent_noise(43, (16, 16, 16)))
    ref_other = other.clone()
    Z.zdit_sample(stack, call, ref_other, ws, n_steps=8, guidance=1.0)
    lat.copy_(other)
    Z.zdit_sample(stack, call, lat, ws, n_steps=8, guidance=1.0, use_graph=True)    # replay, new noise
    assert torch.equal(lat, ref_other)


def test_base_recipe_fifty_steps_cfg_four():
    # the Base-model recipe ([Jobs] "Recipes and precision"): 50 steps, guidance 4, on the
    # same kernels; the schedule is the same closed form with u = i / 50
    d, W, latent, caps = _small_setup()
    stack = Z.DeviceStack(W, dims_of(d), 2, 2, 2, patch_dim=64, cap_dim=128)
    call = Z.StackCall((8, 8), [64, 32], [45, 1], [0.0, 0.0], dev(caps), dev(caps))
    ws = torch.empty(Z.sample_workspace_bytes(stack, call), dtype=torch.uint8, device="cuda")
    lat = dev(latent)
    Z.zdit_sample(stack, call, lat, ws, n_steps=50, guidance=4.0)
    assert Z.zdit_device_status() == 0
    cond = {"caps": caps[:45], "n_cap": 64, "n_valid": 45}
    unc = {"caps": caps[45:], "n_cap": 32, "n_valid": 1}
    ref = O.sample(latent, cond, unc, W, d, g=4.0, n_steps=50)
    _check(host(lat), ref, "base recipe")

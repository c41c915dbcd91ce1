"""Whole-forward parity of wan_dit_forward against the float64 oracle.

* one block + head at 192 tokens: every element, with the per-block error
  report (the residual stream after the patch embedding and after the block);
* the per-token-timestep variant (Wan2.2-5B widths, 48 channels);
* the 480p CFG-batch shapes (B = 2, L = 32760, launch configuration of the
  benchmark) with one block: sampled tokens against the oracle's row mode;
* the same shapes with all 30 blocks: properties that hold at any size
  (identical samples give identical outputs, run-to-run determinism, graph
  replay equals eager launches, finite values);
* argument validation and weight bookkeeping of the C ABI.
Tolerance on the velocity: relative L2 <= 2e-2 (bf16 storage, fp32
accumulation), the bound the method's precision policy allows.
"""
import pytest
import torch

from oracle import wan_oracle as O
from tests.gpu_common import DT, make_dit, need_gpu, rel_l2, to64, workload_inputs

pytestmark = pytest.mark.gpu

TOL = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def report(tag, errs):
    print(f"\n[{tag}] per-block rel-L2: " + " ".join(f"{e:.2e}" for e in errs))


def run_gpu(dit, lat, t, ctx):
    v = dit.forward(lat.cuda(), t.cuda(), ctx.cuda(), sync=True)
    return v.cpu()


def test_forward_one_block_192_tokens():
    cfg, W, lat, t, ctx = workload_inputs("wan1.3b-1blk-3x16x16")
    B, L, Lc = 1, O.token_count(*lat.shape[2:]), ctx.shape[1]
    dit = make_dit(cfg, B, L, Lc, W)
    dump = torch.zeros(cfg["num_blocks"] + 1, B * L, cfg["dim"], dtype=torch.bfloat16, device="cuda")
    dit.set_block_dump(dump)
    v_eager = run_gpu(dit, lat, t, ctx)
    dit.set_block_dump(None)
    ref, blocks = O.forward(lat.to(DT), t.to(DT), ctx.to(DT), to64(W), cfg, return_blocks=True)
    errs = [rel_l2(dump[i].cpu(), blocks[i].reshape(B * L, -1)) for i in range(len(blocks))]
    report("1 block, 192 tokens", errs)
    assert max(errs) < TOL
    err = rel_l2(v_eager, ref)
    print(f"velocity rel-L2 {err:.3e}")
    assert err < TOL
    # graph replay == eager launches, bit for bit, and run to run
    v_graph = run_gpu(dit, lat, t, ctx)
    v_graph2 = run_gpu(dit, lat, t, ctx)
    assert torch.equal(v_graph, v_eager)
    assert torch.equal(v_graph, v_graph2)
    assert dit.last_launch_count() > 0


def test_forward_host_io_matches_device_io():
    cfg, W, lat, t, ctx = workload_inputs("wan1.3b-1blk-3x16x16", seed=1)
    B, L, Lc = 1, O.token_count(*lat.shape[2:]), ctx.shape[1]
    dit = make_dit(cfg, B, L, Lc, W)
    v_dev = run_gpu(dit, lat, t, ctx)
    v_host = dit.forward(lat.pin_memory(), t.pin_memory(), ctx.pin_memory())
    dit.sync()
    assert not v_host.is_cuda
    assert torch.equal(v_host, v_dev)


def test_forward_per_token_timestep_5b_widths():
    from video_diffusion_transformer_dit_b200 import configs, synth
    cfg = configs.model_config("wan2.2-5b", num_blocks=1)
    shape = (1, 48, 3, 16, 16)
    L = O.token_count(*shape[2:])
    W = synth.make_weights(cfg, seed=3)
    lat = synth.make_latent(shape, seed=3)
    ctx = synth.make_context(1, 40, cfg["text_dim"], seed=3)
    t = synth.make_timestep_per_token(1, L, 64, seed=3)
    dit = make_dit(cfg, 1, L, 40, W)
    v = run_gpu(dit, lat, t, ctx)
    ref = O.forward(lat.to(DT), t.to(DT), ctx.to(DT), to64(W), cfg)
    err = rel_l2(v, ref)
    print(f"\nper-token 5B widths velocity rel-L2 {err:.3e}")
    assert err < TOL


def test_forward_480p_cfg_batch_one_block_sampled_rows():
    """B = 2, L = 32760 (81 frames 480x832), one block: sampled tokens of both
    samples against the oracle's row mode (keys/values over every token)."""
    cfg, W, lat, t, ctx = workload_inputs("wan1.3b-81f-480x832-cfg2", num_blocks=1)
    B, Cc, F, Hz, Wz = lat.shape
    L, Lc = O.token_count(F, Hz, Wz), ctx.shape[1]
    dit = make_dit(cfg, B, L, Lc, W)
    v = run_gpu(dit, lat, t, ctx)
    g = torch.Generator().manual_seed(0)
    rows = torch.cat([torch.tensor([0, 1, L // 2, L - 1]), torch.randint(0, L, (60,), generator=g)]).unique()
    o = O.forward(lat.to(DT), t.to(DT), ctx.to(DT), to64(W), cfg, rows=rows)
    idx = O.unpatch_index_map(Cc, F, Hz, Wz)[rows]
    got = v.reshape(B, -1)[:, idx]
    err = rel_l2(got, o)
    print(f"\n480p B=2 one block, {rows.numel()} sampled tokens rel-L2 {err:.3e}")
    assert err < TOL


def test_forward_480p_cfg_batch_30_blocks_properties():
    cfg, W, lat, t, ctx = workload_inputs("wan1.3b-81f-480x832-cfg2")
    B, Cc, F, Hz, Wz = lat.shape
    L, Lc = O.token_count(F, Hz, Wz), ctx.shape[1]
    dit = make_dit(cfg, B, L, Lc, W)
    ctx_same = ctx[:1].expand(B, -1, -1).contiguous()
    v1 = run_gpu(dit, lat, t, ctx_same)
    assert torch.isfinite(v1).all()
    assert torch.equal(v1[0], v1[1])            # identical samples, identical outputs
    v2 = run_gpu(dit, lat, t, ctx_same)
    assert torch.equal(v1, v2)                  # deterministic
    v3 = run_gpu(dit, lat, t, ctx)              # two contexts: the samples differ
    assert torch.isfinite(v3).all()
    assert not torch.equal(v3[0], v3[1])
    assert 0.1 < v3.std().item() < 10.0


# ------------------------------------------------------------------ C ABI bookkeeping
def test_abi_validation_and_missing_weights():
    from video_diffusion_transformer_dit_b200.binding import WanError
    cfg, W, lat, t, ctx = workload_inputs("wan1.3b-1blk-3x16x16", seed=2)
    L, Lc = O.token_count(*lat.shape[2:]), ctx.shape[1]
    dit = make_dit(cfg, 1, L, Lc)
    with pytest.raises(WanError) as e:
        dit.forward(lat.cuda(), t.cuda(), ctx.cuda())
    assert e.value.name == "WAN_ENOWEIGHTS"
    part = {k: v.cuda() for k, v in W.items() if k != "proj_out.bias"}
    dit.load_weights(part)
    n, names = dit.missing_weights()
    assert n == 1 and names == "proj_out.bias"
    with pytest.raises(WanError) as e:
        dit.forward(lat.cuda(), t.cuda(), ctx.cuda())
    assert e.value.name == "WAN_EMISSING_WEIGHT"
    with pytest.raises(WanError) as e:
        dit.load_weights({"blocks.7.attn1.to_q.weight": W["blocks.0.attn1.to_q.weight"].cuda()})
    assert e.value.name == "WAN_EUNEXPECTED_WEIGHT"
    with pytest.raises(WanError) as e:
        dit.load_weights({"proj_out.bias": torch.zeros(63, device="cuda")})
    assert e.value.name == "WAN_ESHAPE"
    dit.load_weights({"proj_out.bias": W["proj_out.bias"].cuda()})
    assert dit.missing_weights()[0] == 0
    # shapes beyond the workspace limits or odd grids are refused before any launch
    big = torch.zeros(1, 16, 4, 16, 16, device="cuda")
    with pytest.raises(WanError) as e:
        dit.forward(big, t.cuda(), ctx.cuda())
    assert e.value.name == "WAN_ESHAPE"
    odd = torch.zeros(1, 16, 3, 15, 16, device="cuda")
    with pytest.raises(WanError) as e:
        dit.forward(odd, t.cuda(), ctx.cuda())
    assert e.value.name == "WAN_ESHAPE"
    v = dit.forward(lat.cuda(), t.cuda(), ctx.cuda(), sync=True)
    assert torch.isfinite(v).all()


def _sampled_rows_case(cfg, shape, Lc, seed, per_token=False, n_rows=48):
    from video_diffusion_transformer_dit_b200 import synth
    B, Cc, F, Hz, Wz = shape
    L = O.token_count(F, Hz, Wz)
    W = synth.make_weights(cfg, seed=seed)
    lat = synth.make_latent(shape, seed=seed)
    ctx = synth.make_context(B, Lc, cfg["text_dim"], seed=seed)
    t = synth.make_timestep_per_token(B, L, (Hz // 2) * (Wz // 2), seed=seed) if per_token else \
        synth.make_timestep(B, 500.0)
    dit = make_dit(cfg, B, L, Lc, W)
    v = run_gpu(dit, lat, t, ctx)
    dit.close()
    g = torch.Generator().manual_seed(seed)
    rows = torch.cat([torch.tensor([0, L - 1]), torch.randint(0, L, (n_rows,), generator=g)]).unique()
    o = O.forward(lat.to(DT), t.to(DT), ctx.to(DT), to64(W), cfg, rows=rows)
    idx = O.unpatch_index_map(Cc, F, Hz, Wz)[rows]
    return rel_l2(v.reshape(B, -1)[:, idx], o), rows.numel()


def test_forward_14b_widths_one_block_sampled_rows():
    """Wan-14B widths (D 5120, 40 heads, FFN 13824, 512 text tokens), one block,
    81-frame 720x1280 spatial grid on 3 latent frames (10800 tokens)."""
    from video_diffusion_transformer_dit_b200 import configs
    cfg = configs.model_config("wan2.1-14b", num_blocks=1)
    err, n = _sampled_rows_case(cfg, (1, 16, 3, 90, 160), 512, seed=6)
    print(f"\n14B widths one block, {n} sampled tokens rel-L2 {err:.3e}")
    assert err < TOL


def test_forward_5b_per_token_full_shape_one_block_sampled_rows():
    """Wan2.2-5B shape at its full size (48 channels, 121 frames 704x1280 -> 27280
    tokens, 512 text tokens) with per-token timesteps, one block."""
    from video_diffusion_transformer_dit_b200 import configs
    cfg = configs.model_config("wan2.2-5b", num_blocks=1)
    err, n = _sampled_rows_case(cfg, (1, 48, 31, 44, 80), 512, seed=7, per_token=True)
    print(f"\n5B full shape per-token one block, {n} sampled tokens rel-L2 {err:.3e}")
    assert err < TOL


def test_forward_33f_352x640_all_30_blocks_full_oracle():
    """33 frames 352x640 (latent [1,16,9,44,80], 7920 tokens = 61 full 128-row
    tiles + a ragged 112), all 30 blocks, every element against the full float64
    oracle, with the per-block error report."""
    cfg, W, lat, t, ctx = workload_inputs("wan1.3b-33f-352x640")
    B, L, Lc = 1, O.token_count(*lat.shape[2:]), ctx.shape[1]
    dit = make_dit(cfg, B, L, Lc, W)
    dump = torch.zeros(cfg["num_blocks"] + 1, B * L, cfg["dim"], dtype=torch.bfloat16, device="cuda")
    dit.set_block_dump(dump)
    v = run_gpu(dit, lat, t, ctx)
    dump = dump.cpu()
    dit.close()
    ref, blocks = O.forward(lat.to(DT), t.to(DT), ctx.to(DT), to64(W), cfg, return_blocks=True)
    errs = [rel_l2(dump[i], blocks[i].reshape(B * L, -1)) for i in range(len(blocks))]
    report("33f 352x640, 30 blocks", errs)
    err = rel_l2(v, ref)
    print(f"velocity rel-L2 {err:.3e}")
    assert max(errs) < TOL
    assert err < TOL


# ---------------------------------------------------------------- I2V route and the expert switch

def _i2v_case(seed=0):
    from video_diffusion_transformer_dit_b200 import configs, synth
    w = configs.workload("wan-i2v-1blk-3x16x16")
    cfg = w["cfg"]
    B, Cc, F, Hz, Wz = w["latent"]
    W = synth.make_weights(cfg, seed=seed)
    lat = synth.make_latent(w["latent"], seed=seed)
    ctx = synth.make_context(B, w["text_len"], cfg["text_dim"], seed=seed)
    img = synth.make_image(B, w["image_len"], cfg["image_dim"], seed=seed)
    t = synth.make_timestep(B, w["timesteps"][0])
    return cfg, W, lat, t, ctx, img


def test_forward_i2v_one_block_against_oracle():
    """36-channel input (patch K 144, padded to the 64-wide K tile), 257 image
    tokens of width 1280 per sample, B = 2 with different images."""
    from video_diffusion_transformer_dit_b200.binding import WanDiT
    cfg, W, lat, t, ctx, img = _i2v_case()
    B, L, Lc, Li = lat.shape[0], O.token_count(*lat.shape[2:]), ctx.shape[1], img.shape[1]
    dit = WanDiT(cfg, max_batch=B, max_tokens=L, max_text=Lc, max_image=Li)
    dit.load_weights({k: v.cuda() for k, v in W.items()})
    assert dit.missing_weights()[0] == 0
    v = dit.forward(lat.cuda(), t.cuda(), ctx.cuda(), image=img.cuda(), sync=True).cpu()
    W64 = to64(W)
    ref = O.forward(lat.to(DT), t.to(DT), ctx.to(DT), W64, cfg, image=img.to(DT))
    err = rel_l2(v, ref)
    print(f"\n[I2V 1 block] velocity rel-L2 {err:.3e}")
    assert err < TOL
    # the image branch matters, and without image tokens the text branch alone runs
    v_txt = dit.forward(lat.cuda(), t.cuda(), ctx.cuda(), sync=True).cpu()
    ref_txt = O.forward(lat.to(DT), t.to(DT), ctx.to(DT), W64, cfg)
    assert rel_l2(v_txt, ref_txt) < TOL
    assert rel_l2(ref, ref_txt) > 5 * TOL             # ~0.26 for these synthetic weights
    # graph replay of the image plan is deterministic, host I/O equals device I/O
    v2 = dit.forward(lat.cuda(), t.cuda(), ctx.cuda(), image=img.cuda(), sync=True).cpu()
    assert torch.equal(v, v2)
    v_host = dit.forward(lat.pin_memory(), t.pin_memory(), ctx.pin_memory(), image=img.pin_memory())
    dit.sync()
    assert torch.equal(v_host, v)
    assert dit.flops(B, *lat.shape[2:], Lc, 0, Li) > dit.flops(B, *lat.shape[2:], Lc, 0)


def test_forward_image_argument_validation():
    from video_diffusion_transformer_dit_b200.binding import WanError
    cfg, W, lat, t, ctx, img = _i2v_case(seed=1)
    B, L, Lc = lat.shape[0], O.token_count(*lat.shape[2:]), ctx.shape[1]
    from video_diffusion_transformer_dit_b200.binding import WanDiT
    dit = WanDiT(cfg, max_batch=B, max_tokens=L, max_text=Lc, max_image=100)
    dit.load_weights({k: v.cuda() for k, v in W.items()})
    with pytest.raises(WanError) as e:                      # more image tokens than the workspace holds
        dit.forward(lat.cuda(), t.cuda(), ctx.cuda(), image=img.cuda())
    assert e.value.name == "WAN_ESHAPE"
    t2v_cfg, W2, lat2, t2, ctx2 = workload_inputs("wan1.3b-1blk-3x16x16")
    t2v = make_dit(t2v_cfg, 1, O.token_count(*lat2.shape[2:]), ctx2.shape[1], W2)
    with pytest.raises(WanError) as e:                      # a text-to-video model has no image branch
        t2v.forward(lat2.cuda(), t2.cuda(), ctx2.cuda(), image=img[:1, :10].cuda())
    assert e.value.name == "WAN_EINVAL"


def test_moe_expert_dispatch():
    """Two handles with different weights: each step runs on the expert its
    timestep selects, bit-identical to calling that expert directly."""
    from video_diffusion_transformer_dit_b200 import synth
    from video_diffusion_transformer_dit_b200.binding import WanMoE
    cfg, W_hi, lat, t, ctx = workload_inputs("wan1.3b-1blk-3x16x16", seed=4)
    W_lo = synth.make_weights(cfg, seed=5)
    L, Lc = O.token_count(*lat.shape[2:]), ctx.shape[1]
    hi, lo = make_dit(cfg, 1, L, Lc, W_hi), make_dit(cfg, 1, L, Lc, W_lo)
    moe = WanMoE(hi, lo, boundary=0.875, num_train_timesteps=1000)
    for tv, which in ((999.0, hi), (875.0, hi), (874.0, lo), (20.0, lo)):
        tt = torch.full((1,), tv)
        got = moe.forward(lat.cuda(), tt.cuda(), ctx.cuda(), sync=True).cpu()
        want = which.forward(lat.cuda(), tt.cuda(), ctx.cuda(), sync=True).cpu()
        assert torch.equal(got, want), tv
    ref_lo = O.forward(lat.to(DT), torch.full((1,), 20.0, dtype=DT), ctx.to(DT), to64(W_lo), cfg)
    assert rel_l2(moe.forward(lat.cuda(), torch.full((1,), 20.0).cuda(), ctx.cuda(), sync=True).cpu(), ref_lo) < TOL
    with pytest.raises(ValueError):                           # one timestep per step
        moe.expert(torch.tensor([900.0, 100.0]))


# ---------------------------------------------------------------- the 14B 720p and 5B per-token workloads at full size

def test_forward_14b_720p_full_grid_one_block_sampled_rows():
    """Wan-14B shape at its full 720p grid: latent [1,16,21,90,160] -> 75600
    tokens (the largest attention and GEMM M of the workloads: 591 query tiles
    of 128 per head), D 5120, 40 heads, FFN 13824, 512 text tokens, one block;
    rows 0 and L-1 plus 64 sampled tokens against the oracle's row mode."""
    from video_diffusion_transformer_dit_b200 import configs
    cfg = configs.model_config("wan2.1-14b", num_blocks=1)
    err, n = _sampled_rows_case(cfg, (1, 16, 21, 90, 160), 512, seed=8, n_rows=64)
    print(f"\n14B 720p full grid one block, {n} sampled tokens rel-L2 {err:.3e}")
    assert err < TOL


def _full_depth_properties(name, seed):
    """All blocks of a named workload with device-generated weights: finite,
    spread, run-to-run deterministic, graph replay bit-identical to eager
    launches."""
    from video_diffusion_transformer_dit_b200 import configs, synth
    from video_diffusion_transformer_dit_b200.binding import WAN_OPT_GRAPH, WanDiT
    w = configs.workload(name)
    cfg = w["cfg"]
    B, Cc, F, Hz, Wz = w["latent"]
    L, Lc = O.token_count(F, Hz, Wz), w["text_len"]
    dit = WanDiT(cfg, max_batch=B, max_tokens=L, max_text=Lc)
    W = synth.make_weights(cfg, seed=seed, device="cuda")
    dit.load_weights(W)
    del W
    torch.cuda.empty_cache()
    lat = synth.make_latent(w["latent"], seed=seed, device="cuda")
    ctx = synth.make_context(B, Lc, cfg["text_dim"], seed=seed, device="cuda")
    if w["timesteps"] == "per_token":
        t = synth.make_timestep_per_token(B, L, (Hz // 2) * (Wz // 2), seed=seed).cuda()
    else:
        t = synth.make_timestep(B, w["timesteps"][0]).cuda()
    v1 = dit.forward(lat, t, ctx, sync=True).cpu()
    v2 = dit.forward(lat, t, ctx, sync=True).cpu()
    dit.set_option(WAN_OPT_GRAPH, 0)
    v3 = dit.forward(lat, t, ctx, sync=True).cpu()
    launches = dit.last_launch_count()
    dit.close()
    assert torch.isfinite(v1).all()
    assert 0.05 < v1.std().item() < 20.0, v1.std().item()
    assert torch.equal(v1, v2)
    assert torch.equal(v1, v3)
    return launches


def test_forward_14b_720p_40_blocks_properties():
    """BASELINE config 3 at full depth and size (40 blocks, 75600 tokens, ~28 GB
    of bf16 weights): a float64 forward would be ~6500 TFLOP of host work, so the
    full depth is checked by properties that hold at any size; the one-block
    test above compares against the oracle."""
    n = _full_depth_properties("wan14b-81f-720x1280", seed=9)
    assert n > 10 * 40


def test_forward_5b_per_token_30_blocks_properties():
    """BASELINE config 4 at full depth and size: Wan2.2-5B shape, 48 channels,
    27280 tokens, per-token timesteps (first latent frame clean), 30 blocks."""
    n = _full_depth_properties("wan5b-121f-704x1280-pertoken", seed=10)
    assert n > 10 * 30


# ---------------------------------------------------------------- sampler step fused into proj_out (CFG + Euler)

def _cfg_case(name, seed, num_blocks=None):
    from video_diffusion_transformer_dit_b200 import configs, synth
    w = configs.workload(name)
    cfg = dict(w["cfg"])
    if num_blocks is not None:
        cfg["num_blocks"] = num_blocks
    _, Cc, F, Hz, Wz = w["latent"]
    Lc = w["text_len"]
    W = synth.make_weights(cfg, seed=seed)
    x = synth.make_latent((1, Cc, F, Hz, Wz), seed=seed)
    ctx = synth.make_context(2, Lc, cfg["text_dim"], seed=seed)      # conditional, unconditional
    return cfg, W, x, ctx


def test_forward_cfg_euler_one_block_against_oracle():
    """x_next = x + (sigma_next - sigma)(v_u + s (v_c - v_u)) with the two
    velocities of the B = 2 forward (same latent, conditional and unconditional
    context), one block + head, a step of the 50-step 480p schedule (shift 3)."""
    from video_diffusion_transformer_dit_b200 import binding as Bd
    cfg, W, x, ctx = _cfg_case("wan1.3b-1blk-3x16x16", seed=12)
    _, Cc, F, Hz, Wz = x.shape
    L, Lc = O.token_count(F, Hz, Wz), ctx.shape[1]
    sig = Bd.flow_sigmas(50, 3.0)
    i, s = 10, 5.0
    t = float(torch.tensor(sig[i] * 1000.0, dtype=torch.float32))
    dit = make_dit(cfg, 2, L, Lc, W)
    xn = dit.forward_cfg_euler(x.cuda(), t, ctx.cuda(), s, sig[i], sig[i + 1], sync=True).cpu()
    xd = x.to(DT)
    v = O.forward(xd.expand(2, -1, -1, -1, -1), torch.full((2,), t, dtype=DT), ctx.to(DT), to64(W), cfg)
    ref = O.euler_step(xd, sig[i], sig[i + 1], O.cfg_combine(v[1:2], v[0:1], s))
    ds = sig[i + 1] - sig[i]
    err = rel_l2((xn.to(DT) - xd) / ds, (ref - xd) / ds)          # the update carries the model output
    print(f"\n[CFG+Euler 1 block] update rel-L2 {err:.3e}")
    assert err < TOL
    # the unfused path (B = 2 forward, then the sampler-step op) gives the same bits
    vel = dit.forward(x.expand(2, -1, -1, -1, -1).contiguous().cuda(), torch.full((2,), t).cuda(), ctx.cuda(),
                      sync=True)
    out = torch.empty_like(x).cuda()
    Bd.op_cfg_euler(x.cuda(), vel[0:1].contiguous(), vel[1:2].contiguous(), s, sig[i], sig[i + 1], out)
    Bd.op_sync()
    assert torch.equal(out.cpu(), xn)
    # host buffers, and x_next aliasing x
    xh = dit.forward_cfg_euler(x.pin_memory(), t, ctx.pin_memory(), s, sig[i], sig[i + 1])
    dit.sync()
    assert torch.equal(xh, xn)
    xa = x.clone().cuda()
    dit.forward_cfg_euler(xa, t, ctx.cuda(), s, sig[i], sig[i + 1], x_next=xa, sync=True)
    assert torch.equal(xa.cpu(), xn)


def test_forward_cfg_euler_480p_30_blocks_matches_unfused():
    """The 480p CFG pair (L = 32760, 30 blocks): fused sampler step bit-identical
    to the B = 2 forward followed by the separate sampler-step kernel, at two
    steps of the schedule (the per-call scalars change without a new capture)."""
    from video_diffusion_transformer_dit_b200 import binding as Bd
    from video_diffusion_transformer_dit_b200 import synth
    cfg, _, x, ctx = _cfg_case("wan1.3b-81f-480x832-cfg2", seed=13, num_blocks=1)
    cfg["num_blocks"] = 30
    W = synth.make_weights(cfg, seed=13, device="cuda")
    _, Cc, F, Hz, Wz = x.shape
    L, Lc = O.token_count(F, Hz, Wz), ctx.shape[1]
    dit = make_dit(cfg, 2, L, Lc)
    dit.load_weights(W)
    del W
    sig = Bd.flow_sigmas(50, 3.0)
    xc, cc = x.cuda(), ctx.cuda()
    launches = None
    for i in (0, 37):
        t = float(torch.tensor(sig[i] * 1000.0, dtype=torch.float32))
        xn = dit.forward_cfg_euler(xc, t, cc, 5.0, sig[i], sig[i + 1], sync=True)
        launches = dit.last_launch_count()
        vel = dit.forward(xc.expand(2, -1, -1, -1, -1).contiguous(), torch.full((2,), t).cuda(), cc, sync=True)
        out = torch.empty_like(xc)
        Bd.op_cfg_euler(xc, vel[0:1].contiguous(), vel[1:2].contiguous(), 5.0, sig[i], sig[i + 1], out)
        Bd.op_sync()
        assert torch.isfinite(xn).all()
        assert torch.equal(out, xn), i
        assert not torch.equal(xn, xc)
    assert launches == dit.last_launch_count()

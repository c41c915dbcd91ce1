"""The Wan2.1 VAE decoder on the GPU against the float64 oracle (oracle/wan_vae.py).

* wan_op_conv3d, the implicit-GEMM causal convolution: the decoder's kernel
  shapes (3x3x3 with 0/1/2 cached frames, the (3,1,1) time_conv with its frame
  split, 1x1x1 shortcuts, 3x3 per-frame convolutions, conv_in's 16 channels,
  conv_out's 3), ragged spatial tiles, residual add;
* wan_vae_decode, the whole decoder with its frame loop and 33 frame caches,
  three latent frames (9 video frames) at the full channel widths, against the
  oracle's frame loop; host and device I/O; two samples with different latents.
Tolerance: relative L2 <= 1e-2 per convolution, <= 2e-2 for the decoded video
(bf16 activations through ~40 convolutions, fp32 accumulation).
"""
import pytest
import torch

from oracle import wan_vae as V
from tests.gpu_common import DT, need_gpu, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def B():
    from video_diffusion_transformer_dit_b200 import binding
    return binding


def pack(w):
    """[Co, Ci, kt, kh, kw] -> [Co_pad, taps * Cip] bf16, (tap, ci) order, zero padded."""
    Co, Ci, kt, kh, kw = w.shape
    cip = (Ci + 63) // 64 * 64
    co_pad = (Co + 63) // 64 * 64
    taps = kt * kh * kw
    out = torch.zeros(co_pad, taps, cip, dtype=torch.bfloat16)
    out[:Co, :, :Ci] = w.permute(0, 2, 3, 4, 1).reshape(Co, taps, Ci).to(torch.bfloat16)
    return out.reshape(co_pad, taps * cip)


CASES = [  # Ci, Co, kernel, T, H, W, cached frames, residual
    (384, 384, (3, 3, 3), 2, 13, 21, 2, False),
    (384, 384, (3, 3, 3), 1, 8, 16, 1, True),
    (96, 96, (3, 3, 3), 3, 24, 40, 0, True),
    (16, 384, (3, 3, 3), 1, 9, 11, 0, False),
    (96, 3, (3, 3, 3), 2, 17, 19, 2, False),
    (192, 384, (1, 1, 1), 2, 10, 10, 0, False),
    (192, 96, (1, 3, 3), 4, 12, 20, 0, False),
    (16, 16, (1, 1, 1), 1, 6, 8, 0, False),
]


@pytest.mark.parametrize("Ci,Co,kernel,T,H,W,nc,residual", CASES)
def test_conv3d_implicit_gemm_matches_oracle(Ci, Co, kernel, T, H, W, nc, residual):
    Bn = 2
    g = torch.Generator().manual_seed(Ci * 7 + Co + T + nc)
    kt, kh, kw = kernel
    x = torch.randn(Bn, Ci, T, H, W, generator=g).to(torch.bfloat16)
    w = (torch.randn(Co, Ci, kt, kh, kw, generator=g) / (Ci * kt * kh * kw) ** 0.5).to(torch.bfloat16)
    bias = torch.randn(Co, generator=g) * 0.1
    cache = torch.randn(Bn, Ci, nc, H, W, generator=g).to(torch.bfloat16) if nc else None
    ref = V.causal_conv3d(x.to(DT), w.to(DT), bias.to(DT), cache.to(DT) if nc else None)
    ldy = (Co + 7) // 8 * 8
    add = torch.randn(Bn, T, H, W, Co, generator=g).to(torch.bfloat16) if residual else None
    if residual:
        ref = ref + add.to(DT).permute(0, 4, 1, 2, 3)
    cl = lambda t: t.permute(0, 2, 3, 4, 1).contiguous().cuda()
    y = torch.full((Bn, T, H, W, ldy), float("nan"), dtype=torch.bfloat16, device="cuda")
    B().op_conv3d(cl(x), pack(w).cuda(), bias.cuda(), y, kernel, Co, cache=cl(cache) if nc else None,
                  add=add.cuda() if residual else None)
    B().op_sync()
    got = y[..., :Co].cpu().permute(0, 4, 1, 2, 3)
    err = rel_l2(got, ref)
    print(f"\n[conv {Ci}->{Co} {kernel} T{T} {H}x{W} cache {nc}{' +res' if residual else ''}] rel-L2 {err:.2e}")
    assert err < 1e-2


def test_conv3d_time_split_matches_oracle_upsampler():
    """time_conv (3,1,1) C -> 2C with the frame split of the time upsampler:
    channel half k of frame t becomes frame 2t + k (reading V4)."""
    Bn, C, T, H, W, nc = 1, 192, 2, 6, 10, 1
    g = torch.Generator().manual_seed(5)
    x = torch.randn(Bn, C, T, H, W, generator=g).to(torch.bfloat16)
    w = (torch.randn(2 * C, C, 3, 1, 1, generator=g) / (3 * C) ** 0.5).to(torch.bfloat16)
    bias = torch.randn(2 * C, generator=g) * 0.1
    cache = torch.randn(Bn, C, nc, H, W, generator=g).to(torch.bfloat16)
    y2 = V.causal_conv3d(x.to(DT), w.to(DT), bias.to(DT), cache.to(DT))
    ref = y2.reshape(Bn, 2, C, T, H, W).permute(0, 2, 3, 1, 4, 5).reshape(Bn, C, 2 * T, H, W)
    y = torch.empty(Bn, 2 * T, H, W, C, dtype=torch.bfloat16, device="cuda")
    cl = lambda t: t.permute(0, 2, 3, 4, 1).contiguous().cuda()
    B().op_conv3d(cl(x), pack(w).cuda(), bias.cuda(), y, (3, 1, 1), 2 * C, cache=cl(cache), time_split=True)
    B().op_sync()
    assert rel_l2(y.cpu().permute(0, 4, 1, 2, 3), ref) < 1e-2


def test_conv3d_argument_checks():
    x = torch.zeros(1, 1, 8, 8, 12, dtype=torch.bfloat16, device="cuda")        # Ci 12: not a multiple of 8
    w = torch.zeros(64, 27 * 64, dtype=torch.bfloat16, device="cuda")
    y = torch.zeros(1, 1, 8, 8, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(B().WanError) as e:
        B().op_conv3d(x, w, None, y, (3, 3, 3), 64)
    assert e.value.name == "WAN_ESHAPE"
    x = torch.zeros(1, 1, 8, 8, 16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(B().WanError):                                           # even kernel size
        B().op_conv3d(x, w, None, y, (2, 3, 3), 64)


def decoder_weights(seed=0):
    """Random decoder weights with fan-in scaling (activations stay O(1) through
    the residual blocks, the decoded video mostly inside the clamp)."""
    from video_diffusion_transformer_dit_b200 import synth
    return synth.make_vae_weights(seed=seed)


def test_vae_decode_matches_oracle_frame_loop():
    W = decoder_weights(3)
    g = torch.Generator().manual_seed(4)
    z = torch.randn(2, 16, 3, 6, 8, generator=g)
    vae = B().WanVAE(max_batch=2, max_h=6, max_w=10)
    vae.load_weights({k: v.cuda() for k, v in W.items()})
    assert vae.missing_weights()[0] == 0
    video = vae.decode(z.cuda(), sync=True).cpu()
    assert video.shape == (2, 3, 9, 48, 64)
    ref = V.decode(z.to(DT), {k: v.to(DT) for k, v in W.items()})
    err = rel_l2(video, ref)
    per_frame = [rel_l2(video[:, :, t], ref[:, :, t]) for t in range(9)]
    print(f"\n[VAE decode 3 latent frames 6x8 -> 9 x 48x64] rel-L2 {err:.2e}; per frame "
          + " ".join(f"{e:.1e}" for e in per_frame))
    assert err < 2e-2
    assert video.abs().max() <= 1.0
    # host buffers give the same bits; a second decode resets the caches
    vh = vae.decode(z.pin_memory())
    vae._check(B().lib().wan_vae_sync(vae._h, B()._stream(None)))
    assert torch.equal(vh, video)
    # the two samples are decoded independently
    v1 = vae.decode(z[1:].cuda(), sync=True).cpu()
    assert torch.equal(v1[0], video[1])


def test_vae_decode_argument_checks():
    vae = B().WanVAE(max_batch=1, max_h=4, max_w=4)
    with pytest.raises(B().WanError) as e:
        vae.decode(torch.zeros(1, 16, 2, 4, 4, device="cuda"))
    assert e.value.name == "WAN_EMISSING_WEIGHT"
    W = decoder_weights(5)
    vae.load_weights({k: v.cuda() for k, v in W.items()})
    with pytest.raises(B().WanError) as e:
        vae.decode(torch.zeros(1, 16, 2, 6, 4, device="cuda"))                 # larger than the workspace
    assert e.value.name == "WAN_ESHAPE"
    with pytest.raises(B().WanError) as e:
        vae.load_weights({"decoder.conv_out.weight": torch.zeros(3, 96, 3, 3, device="cuda")})
    assert e.value.name == "WAN_ESHAPE"

"""Pins of the float64 VAE-decoder oracle (oracle/wan_vae.py) against what the
pages print and what the mathematics fixes: the causal padding rule against a
library convolution, the frame-cache semantics against a whole-sequence
formulation written without the cache, the frame/size laws and the printed
per-chunk shapes, the channel schedule's convolution count, the upsampling
rule against the library's nearest-exact mode, the channel RMS norm and the
output clamp."""
import json
import os

import pytest
import torch
import torch.nn.functional as Fn

from oracle import wan_vae as V

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "shapes.json")))
VAE = GOLD["vae_decoder"]
DT = torch.float64


def rand_weights(base=8, seed=0, scale=0.3, z_dim=16):
    g = torch.Generator().manual_seed(seed)
    W = {}
    for k, s in V.param_shapes(z_dim=z_dim, base=base).items():
        W[k] = torch.randn(*s, generator=g, dtype=DT) * (scale if k.endswith("weight") else 0.1)
        if k.endswith(".gamma"):
            W[k] = 1.0 + 0.1 * W[k]
    return W


# ---------------------------------------------------------------- causal convolution

def test_causal_conv_is_a_library_conv_on_front_padded_frames():
    g = torch.Generator().manual_seed(1)
    x = torch.randn(2, 3, 5, 4, 6, generator=g, dtype=DT)
    w = torch.randn(4, 3, 3, 3, 3, generator=g, dtype=DT)
    b = torch.randn(4, generator=g, dtype=DT)
    xp = torch.cat([torch.zeros(2, 3, 2, 4, 6, dtype=DT), x], dim=2)          # 2 p_t zero frames before, none after
    ref = Fn.conv3d(xp, w, b, padding=(0, 1, 1))
    torch.testing.assert_close(V.causal_conv3d(x, w, b), ref, rtol=1e-13, atol=1e-13)
    # causality: a change at frame 3 leaves frames 0..2 of the output untouched
    x2 = x.clone()
    x2[:, :, 3] += 1.0
    d = (V.causal_conv3d(x2, w, b) - V.causal_conv3d(x, w, b)).abs().amax(dim=(0, 1, 3, 4))
    assert torch.all(d[:3] == 0) and torch.all(d[3:] > 0)


def test_cache_replaces_leading_zero_frames():
    g = torch.Generator().manual_seed(2)
    x = torch.randn(1, 3, 6, 4, 4, generator=g, dtype=DT)
    w = torch.randn(2, 3, 3, 3, 3, generator=g, dtype=DT)
    b = torch.randn(2, generator=g, dtype=DT)
    full = V.causal_conv3d(x, w, b)
    for cut in (1, 2, 4):
        a = V.causal_conv3d(x[:, :, :cut], w, b)
        cache = x[:, :, max(0, cut - V.CACHE_T):cut]                               # CACHE_T last frames
        rest = V.causal_conv3d(x[:, :, cut:], w, b, cache)
        torch.testing.assert_close(torch.cat([a, rest], dim=2), full, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------- layout facts the pages print

def test_decoder_has_the_printed_number_of_causal_convs_and_cache_depth():
    assert len(V.causal_conv_names()) == VAE["causal_convs"]
    assert V.CACHE_T == VAE["cache_t"]
    names = V.causal_conv_names()
    assert names[0] == "decoder.conv_in" and names[-1] == "decoder.conv_out"
    assert sum(n.endswith("time_conv") for n in names) == 2                        # two time upsamplings
    shapes = V.param_shapes()
    assert shapes["decoder.conv_in.weight"][:2] == (VAE["chunk_shapes"][0][1], VAE["z_dim"])
    assert shapes["decoder.conv_out.weight"][:2] == (3, VAE["chunk_shapes"][-1][1])


def test_per_chunk_shapes_follow_the_printed_ones():
    """Full channel widths, a small frame: the activations of a non-first latent
    frame after conv_in and after each up block have the printed channels and
    frame counts, and the printed spatial factors (1, 2, 4, 8, 8)."""
    W = rand_weights(base=96, scale=0.02)
    z = torch.randn(1, 16, 2, 2, 3, generator=torch.Generator().manual_seed(3), dtype=DT)
    trace = []
    V.decode(z, W, trace=trace)
    H0, W0 = VAE["chunk_shapes"][0][3], VAE["chunk_shapes"][0][4]
    for got, want in zip(trace[1], VAE["chunk_shapes"]):
        f = want[3] // H0
        assert tuple(got.shape) == (1, want[1], want[2], 2 * f, 3 * f), (tuple(got.shape), want)
        assert want[4] // W0 == f
    assert [tuple(t.shape)[2] for t in trace[0]] == [1, 1, 1, 1, 1]              # the first frame is not time-upsampled


@pytest.mark.parametrize("case", [c for c in GOLD["latent_law"] if c["z_dim"] == 16], ids=lambda c: str(c["video"]))
def test_frame_and_size_law_inverts_the_latent_law(case):
    T, H, Wd = case["latent"][2:]
    B, Cv, Tv, Hv, Wv = case["video"]
    assert 1 + 4 * (T - 1) == Tv and 8 * H == Hv and 8 * Wd == Wv
    W = rand_weights(base=8)
    z = torch.randn(1, 16, min(T, 3), 2, 3, dtype=DT)
    out = V.decode(z, W, base=8)
    assert out.shape == (1, 3, 1 + 4 * (z.shape[2] - 1), 16, 24)


def test_video_shape_of_the_480p_latent():
    B, C, T, H, Wd = VAE["latent"]
    assert [B, 3, 1 + 4 * (T - 1), 8 * H, 8 * Wd] == VAE["video"]


# ---------------------------------------------------------------- frame loop and whole sequence

@pytest.mark.parametrize("T", [1, 2, 4])
def test_frame_loop_with_cache_equals_whole_sequence(T):
    W = rand_weights(base=8, seed=4)
    z = torch.randn(2, 16, T, 3, 2, generator=torch.Generator().manual_seed(5), dtype=DT)
    a = V.decode(z, W, frame_loop=True, base=8)
    b = V.decode(z, W, frame_loop=False, base=8)
    torch.testing.assert_close(a, b, rtol=1e-11, atol=1e-12)


def test_later_latent_frames_do_not_change_earlier_video_frames():
    W = rand_weights(base=8, seed=6)
    z = torch.randn(1, 16, 3, 2, 2, generator=torch.Generator().manual_seed(7), dtype=DT)
    z2 = z.clone()
    z2[:, :, 2] += 1.0
    a, b = V.decode(z, W, base=8), V.decode(z2, W, base=8)
    torch.testing.assert_close(a[:, :, :5], b[:, :, :5], rtol=0, atol=0)         # video frames of latent frames 0, 1
    assert (a[:, :, 5:] - b[:, :, 5:]).abs().max() > 0


# ---------------------------------------------------------------- pieces

def test_nearest_upsampling_matches_library_nearest_exact():
    x = torch.randn(2, 3, 5, 7, dtype=DT)
    ref = Fn.interpolate(x, scale_factor=2.0, mode="nearest-exact")
    assert torch.equal(V.upsample_nearest2x(x), ref)


def test_channel_rms_norm():
    g = torch.Generator().manual_seed(8)
    x = torch.randn(2, 6, 3, 4, 5, generator=g, dtype=DT) * 3
    one, zero = torch.ones(6, dtype=DT), torch.zeros(6, dtype=DT)
    y = V.rms_norm_c(x, one, zero)
    torch.testing.assert_close((y * y).mean(dim=1), torch.ones(2, 3, 4, 5, dtype=DT), rtol=1e-10, atol=1e-10)
    torch.testing.assert_close(V.rms_norm_c(7.5 * x, one, zero), y, rtol=1e-12, atol=1e-12)
    gam, bet = torch.randn(6, generator=g, dtype=DT), torch.randn(6, generator=g, dtype=DT)
    torch.testing.assert_close(V.rms_norm_c(x, gam, bet), y * gam[None, :, None, None, None] + bet[None, :, None, None, None])


def test_mid_block_attention_is_uniform_without_queries():
    """With the query rows of to_qkv at zero every position attends uniformly, so
    the block adds proj(mean over positions of v) to every position."""
    n = "decoder.mid_block.attentions.0"
    C = 8 * 4                                                                       # mid-block width at base 8
    x = torch.randn(1, C, 2, 3, 4, generator=torch.Generator().manual_seed(10), dtype=DT)
    W = rand_weights(base=8, seed=9)
    W[n + ".to_qkv.weight"][:C] = 0
    W[n + ".to_qkv.bias"][:C] = 0
    out = V._attn(x, n, C, W)
    f = x.permute(0, 2, 1, 3, 4).reshape(2, C, 3, 4)
    h = V.rms_norm_c(f, W[n + ".norm.gamma"], W[n + ".norm.bias"])
    v = Fn.conv2d(h, W[n + ".to_qkv.weight"][2 * C:], W[n + ".to_qkv.bias"][2 * C:])
    vm = v.mean(dim=(2, 3), keepdim=True).expand_as(v)
    ref = f + Fn.conv2d(vm, W[n + ".proj.weight"], W[n + ".proj.bias"])
    torch.testing.assert_close(out, ref.reshape(1, 2, C, 3, 4).permute(0, 2, 1, 3, 4), rtol=1e-12, atol=1e-12)


def test_output_is_clamped():
    lo, hi = VAE["clamp"]
    W = rand_weights(base=8, seed=11, scale=1.5)
    out = V.decode(torch.randn(1, 16, 2, 2, 2, dtype=DT) * 3, W, base=8)
    assert out.min() >= lo and out.max() <= hi
    assert (out.abs() == 1.0).any()                                                 # the clamp is active here


def test_generator_table_matches_oracle_table():
    from video_diffusion_transformer_dit_b200 import synth
    assert synth.vae_param_shapes() == V.param_shapes()


"""Pins of the float64 oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: sizes the
pages print (``tests/golden/shapes.json``), brute-force loops on tiny inputs,
library routines that compute the same special case (Conv3d, LayerNorm,
RMSNorm, GELU, SiLU, scaled-dot-product attention, complex rotation), closed
forms and invariants.  They are chosen so a dropped term, a wrong sign or index
or a transposed operand anywhere in the oracle fails one of them.
"""
import json
import math
import os

import pytest
import torch
import torch.nn.functional as Fn

from oracle import wan_oracle as O
from video_diffusion_transformer_dit_b200 import configs, synth

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "shapes.json")))
DT = torch.float64


def tiny_cfg(**kw):
    cfg = dict(dim=24, heads=2, head_dim=12, ffn_dim=40, num_blocks=1, in_ch=4, out_ch=4,
               patch=(1, 2, 2), text_dim=16, freq_dim=8, eps=1e-6, rope_split=(4, 4, 4), rope_theta=10000.0)
    cfg.update(kw)
    return cfg


def rand_weights(cfg, seed=0, scale=0.3):
    g = torch.Generator().manual_seed(seed)
    W = {}
    for n, s in O.param_shapes(cfg).items():
        W[n] = torch.randn(*s, generator=g, dtype=DT) * scale
        if ".norm_q." in n or ".norm_k." in n or n.endswith("norm2.weight") or ".norm_added_k." in n:
            W[n] = 1.0 + W[n]
    return W


# ---------------------------------------------------------------- shapes

@pytest.mark.parametrize("case", GOLD["latent_law"], ids=lambda c: str(c["video"]))
def test_latent_shape_law(case):
    B, _, T, H, W = case["video"]
    got = O.latent_shape(B, T, H, W, z_dim=case["z_dim"], s_stride=case["s_stride"])
    assert list(got) == case["latent"]
    if "video_numel" in case:
        assert math.prod(case["video"]) == case["video_numel"]
    if "latent_numel" in case:
        assert math.prod(got) == case["latent_numel"]


def test_latent_shape_rejects_bad_frame_count():
    with pytest.raises(ValueError):
        O.latent_shape(1, 32, 480, 832)          # 32 is not 4n+1
    with pytest.raises(ValueError):
        O.latent_shape(1, 33, 484, 832)          # height not a multiple of 8


@pytest.mark.parametrize("case", GOLD["token_law"], ids=lambda c: str(c["tokens"]))
def test_token_law(case):
    F, Hz, Wz = case["latent_grid"]
    assert O.token_count(F, Hz, Wz) == case["tokens"]
    assert F * (Hz // 2) * (Wz // 2) == case["tokens"]
    assert [F, Hz // 2, Wz // 2] == case["grid"]
    idx = O.patch_index_map(2, F, Hz, Wz)
    assert idx.shape == (case["tokens"], 2 * 4)
    if "patch_out" in case:
        assert case["patch_out"][2:] == case["grid"]


def test_intermediate_shapes_480p():
    g = GOLD["intermediate_shapes_480p"]
    cfg = configs.model_config("wan2.1-1.3b", num_blocks=0)
    _, _, F, Hz, Wz = g["latent"]
    ang = O.rope_angles((F, Hz // 2, Wz // 2), cfg["rope_split"], cfg["rope_theta"])
    assert [1, 1] + list(ang.shape) == g["rope"]
    D = cfg["dim"]
    gen = torch.Generator().manual_seed(1)
    W = {n: torch.randn(*s, generator=gen, dtype=DT) * 0.02 for n, s in O.param_shapes(cfg).items()
         if n.startswith("condition_embedder.")}
    temb, tproj = O.time_embedding(torch.tensor([999.0]), W, cfg)
    assert list(temb.shape) == g["temb"]
    assert [1, tproj.shape[1] * tproj.shape[2]] == g["timestep_proj"]
    assert list(tproj.shape) == g["timestep_proj_unflattened"]
    ctx = O.text_embedding(torch.randn(1, g["text_len"], cfg["text_dim"], dtype=DT), W)
    assert list(ctx.shape) == g["context"]
    assert D == g["dim"]


# ---------------------------------------------------------------- patchify / unpatchify

def brute_patchify(lat, patch):
    B, C, F, H, W = lat.shape
    pt, ph, pw = patch
    Fp, Hp, Wp = F // pt, H // ph, W // pw
    X = torch.zeros(B, Fp * Hp * Wp, C * pt * ph * pw, dtype=lat.dtype)
    for b in range(B):
        for f in range(Fp):
            for i in range(Hp):
                for j in range(Wp):
                    l = (f * Hp + i) * Wp + j
                    k = 0
                    for c in range(C):
                        for kt in range(pt):
                            for kh in range(ph):
                                for kw in range(pw):
                                    X[b, l, k] = lat[b, c, f * pt + kt, i * ph + kh, j * pw + kw]
                                    k += 1
    return X


def brute_unpatchify(out, C, F, H, W, patch):
    B = out.shape[0]
    pt, ph, pw = patch
    Fp, Hp, Wp = F // pt, H // ph, W // pw
    vel = torch.full((B, C, F, H, W), float("nan"), dtype=out.dtype)
    for b in range(B):
        for f in range(Fp):
            for i in range(Hp):
                for j in range(Wp):
                    l = (f * Hp + i) * Wp + j
                    for kt in range(pt):
                        for kh in range(ph):
                            for kw in range(pw):
                                for c in range(C):
                                    kk = ((kt * ph + kh) * pw + kw) * C + c
                                    vel[b, c, f * pt + kt, i * ph + kh, j * pw + kw] = out[b, l, kk]
    return vel


@pytest.mark.parametrize("patch", [(1, 2, 2), (2, 2, 2)])
def test_patchify_matches_bruteforce(patch):
    lat = torch.randn(2, 3, 4, 4, 6, dtype=DT)
    assert torch.equal(O.patchify(lat, patch), brute_patchify(lat, patch))


@pytest.mark.parametrize("patch", [(1, 2, 2), (2, 2, 2)])
def test_unpatchify_matches_bruteforce(patch):
    C, F, H, W = 3, 4, 4, 6
    L = (F // patch[0]) * (H // patch[1]) * (W // patch[2])
    out = torch.randn(2, L, C * math.prod(patch), dtype=DT)
    ref = brute_unpatchify(out, C, F, H, W, patch)
    assert not torch.isnan(ref).any()
    assert torch.equal(O.unpatchify(out, C, F, H, W, patch), ref)


def test_patch_embed_is_conv3d():
    lat = torch.randn(2, 16, 3, 8, 10, dtype=DT)
    w = torch.randn(32, 16, 1, 2, 2, dtype=DT)
    b = torch.randn(32, dtype=DT)
    ref = Fn.conv3d(lat, w, b, stride=(1, 2, 2)).flatten(2).transpose(1, 2)
    torch.testing.assert_close(O.patch_embed(lat, w, b), ref, rtol=1e-12, atol=1e-12)


def test_patch_roundtrip_and_bijection():
    C, F, H, W = 16, 3, 16, 16
    lat = torch.randn(1, C, F, H, W, dtype=DT)
    X = O.patchify(lat)                                  # features (c, kh, kw)
    perm = X.reshape(1, -1, C, 4).transpose(2, 3).reshape(1, -1, 4 * C)   # -> (kh, kw, c)
    assert torch.equal(O.unpatchify(perm, C, F, H, W), lat)
    for idx in (O.patch_index_map(C, F, H, W), O.unpatch_index_map(C, F, H, W)):
        assert torch.equal(idx.reshape(-1).sort().values, torch.arange(C * F * H * W))


# ---------------------------------------------------------------- elementwise and norms

def test_activations_match_library():
    x = torch.linspace(-8, 8, 1001, dtype=DT)
    torch.testing.assert_close(O.gelu_tanh(x), Fn.gelu(x, approximate="tanh"), rtol=1e-13, atol=1e-13)
    torch.testing.assert_close(O.silu(x), Fn.silu(x), rtol=1e-13, atol=1e-13)


def test_layer_norm_matches_library_and_moments():
    x = torch.randn(5, 7, 96, dtype=DT) * 3 + 1
    g = torch.randn(96, dtype=DT)
    b = torch.randn(96, dtype=DT)
    eps = 1e-6
    torch.testing.assert_close(O.layer_norm(x, eps), Fn.layer_norm(x, (96,), eps=eps), rtol=1e-12, atol=1e-12)
    torch.testing.assert_close(O.layer_norm(x, eps, g, b), Fn.layer_norm(x, (96,), g, b, eps), rtol=1e-12, atol=1e-12)
    y = O.layer_norm(x, 0.5)
    v = x.var(-1, unbiased=False)
    torch.testing.assert_close(y.mean(-1), torch.zeros_like(v), atol=1e-12, rtol=0)
    torch.testing.assert_close(y.var(-1, unbiased=False), v / (v + 0.5), rtol=1e-12, atol=1e-12)


def test_rms_norm_matches_library_and_is_scale_free():
    x = torch.randn(4, 64, dtype=DT)
    g = torch.randn(64, dtype=DT)
    torch.testing.assert_close(O.rms_norm(x, 1e-6, g), Fn.rms_norm(x, (64,), g, 1e-6), rtol=1e-12, atol=1e-12)
    y = O.rms_norm(x, 0.0)
    torch.testing.assert_close((y * y).mean(-1), torch.ones(4, dtype=DT), rtol=1e-12, atol=1e-12)
    torch.testing.assert_close(O.rms_norm(7.0 * x, 0.0), y, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- sinusoid

def test_sinusoid_closed_forms():
    e0 = O.timestep_sinusoid(torch.tensor([0.0]), 256)
    assert torch.equal(e0[0, :128], torch.ones(128, dtype=DT))
    assert torch.equal(e0[0, 128:], torch.zeros(128, dtype=DT))
    t = torch.tensor([0.3, 17.0, 999.0])
    e = O.timestep_sinusoid(t, 256)
    torch.testing.assert_close(e[:, :128] ** 2 + e[:, 128:] ** 2, torch.ones(3, 128, dtype=DT))
    # frequency 0 is 1 rad per unit time; frequency 64 is base^-1/2 = 0.01
    torch.testing.assert_close(e[:, 0], torch.cos(t.to(DT)))
    torch.testing.assert_close(e[:, 128], torch.sin(t.to(DT)))
    torch.testing.assert_close(e[:, 128 + 64], torch.sin(0.01 * t.to(DT)))
    # geometric ladder: the angle ratio between neighbouring frequencies is constant
    ang = torch.atan2(e[0, 128:], e[0, :128])          # t = 0.3 keeps every angle below pi
    r = ang[1:] / ang[:-1]
    torch.testing.assert_close(r, torch.full_like(r, 10000.0 ** (-1 / 128)), rtol=1e-10, atol=0)


# ---------------------------------------------------------------- RoPE

def test_rope_identity_norm_and_unit_angles():
    split = (44, 42, 42)
    ang = O.rope_angles((3, 4, 5), split, 10000.0)
    assert ang.shape == (60, 64)
    assert torch.equal(ang[0], torch.zeros(64, dtype=DT))      # token (0,0,0) unrotated
    x = torch.randn(60, 3, 128, dtype=DT)
    y = O.rope_apply(x, ang)
    torch.testing.assert_close(y.norm(dim=-1), x.norm(dim=-1), rtol=1e-12, atol=1e-12)
    torch.testing.assert_close(y[0], x[0])
    # first pair of each axis turns by exactly one radian per unit of its own index
    tok = {"f": (1 * 4 + 0) * 5 + 0, "i": (0 * 4 + 1) * 5 + 0, "j": 1}
    e = torch.zeros(60, 1, 128, dtype=DT)
    for col in (0, 44, 86):
        e[:, 0, col] = 1.0
    y = O.rope_apply(e, ang)
    for name, col in (("f", 0), ("i", 44), ("j", 86)):
        l = tok[name]
        torch.testing.assert_close(y[l, 0, col:col + 2], torch.tensor([math.cos(1.0), math.sin(1.0)], dtype=DT))
    # last pair of the time axis turns by theta^(-42/44)
    l = tok["f"]
    assert abs(ang[l, 21] - 10000.0 ** (-42 / 44)) < 1e-15
    # other axes stay still when only f moves
    assert torch.equal(ang[l, 22:], torch.zeros(42, dtype=DT))


def test_rope_is_complex_rotation():
    ang = O.rope_angles((2, 3, 4), (4, 4, 4), 100.0)
    x = torch.randn(24, 2, 12, dtype=DT)
    z = torch.view_as_complex(x.reshape(24, 2, 6, 2).contiguous())
    ref = torch.view_as_real(z * torch.polar(torch.ones_like(ang), ang)[:, None, :]).reshape(24, 2, 12)
    torch.testing.assert_close(O.rope_apply(x, ang), ref, rtol=1e-12, atol=1e-12)


def test_rope_relative_position_invariance():
    split = (4, 4, 4)
    ang = O.rope_angles((6, 6, 6), split, 10000.0)
    q = torch.randn(1, 1, 12, dtype=DT)
    k = torch.randn(1, 1, 12, dtype=DT)

    def tok(f, i, j):
        return (f * 6 + i) * 6 + j

    def dot(m, n):
        return (O.rope_apply(q, ang[m:m + 1]) * O.rope_apply(k, ang[n:n + 1])).sum()

    base = dot(tok(1, 2, 0), tok(3, 1, 4))
    for s in ((1, 0, 0), (0, 2, 0), (0, 0, 1), (2, 3, 1)):
        shifted = dot(tok(1 + s[0], 2 + s[1], 0 + s[2]), tok(3 + s[0], 1 + s[1], 4 + s[2]))
        torch.testing.assert_close(shifted, base, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- attention

def brute_attention(q, k, v):
    B, Lq, h, d = q.shape
    Lk = k.shape[1]
    out = torch.zeros_like(q)
    for b in range(B):
        for hh in range(h):
            for i in range(Lq):
                w = [math.exp(sum(q[b, i, hh, t] * k[b, j, hh, t] for t in range(d)).item() / math.sqrt(d))
                     for j in range(Lk)]
                z = sum(w)
                for j in range(Lk):
                    out[b, i, hh] += w[j] / z * v[b, j, hh]
    return out


def test_attention_bruteforce_and_library():
    q, k, v = (torch.randn(2, n, 2, 8, dtype=DT) for n in (5, 7, 7))
    k = k[:, :7]
    got = O.attention(q, k, v)
    torch.testing.assert_close(got, brute_attention(q, k, v), rtol=1e-12, atol=1e-12)
    lib = Fn.scaled_dot_product_attention(q.transpose(1, 2), k.transpose(1, 2), v.transpose(1, 2)).transpose(1, 2)
    torch.testing.assert_close(got, lib, rtol=1e-12, atol=1e-12)
    # chunking the queries changes nothing
    torch.testing.assert_close(O.attention(q, k, v, chunk_elems=8), got, rtol=0, atol=0)


def test_attention_uniform_and_one_hot():
    v = torch.randn(1, 9, 1, 4, dtype=DT)
    k = torch.randn(1, 9, 1, 4, dtype=DT)
    out = O.attention(torch.zeros(1, 3, 1, 4, dtype=DT), k, v)
    torch.testing.assert_close(out, v.mean(1, keepdim=True).expand(1, 3, 1, 4))
    k2 = torch.zeros(1, 9, 1, 4, dtype=DT)
    k2[0, 6, 0, 0] = 1000.0
    q = torch.zeros(1, 1, 1, 4, dtype=DT)
    q[0, 0, 0, 0] = 1.0
    torch.testing.assert_close(O.attention(q, k2, v)[0, 0, 0], v[0, 6, 0])


# ---------------------------------------------------------------- block wiring probes

def probe_setup(cfg, L=6, Lc=3, seed=3):
    g = torch.Generator().manual_seed(seed)
    W = {n: torch.zeros(*s, dtype=DT) for n, s in O.param_shapes(cfg).items()}
    for n in W:
        if ".norm_q." in n or ".norm_k." in n or n.endswith("norm2.weight") or ".norm_added_k." in n:
            W[n] = torch.ones_like(W[n])
    D = cfg["dim"]
    x = torch.randn(1, L, D, generator=g, dtype=DT)
    ctx = torch.randn(1, Lc, D, generator=g, dtype=DT)
    mod = torch.randn(1, 1, 6, D, generator=g, dtype=DT) * 0.5
    ang = O.rope_angles((1, 2, 3), cfg["rope_split"], cfg["rope_theta"])
    return W, x, ctx, mod, ang, g


def test_block_gates_and_residuals():
    """Only output biases set: x + a*gate_msa + c + f*c_gate (rows 2 and 5 gate)."""
    cfg = tiny_cfg()
    W, x, ctx, mod, ang, g = probe_setup(cfg)
    D = cfg["dim"]
    a, c, f = (torch.randn(D, generator=g, dtype=DT) for _ in range(3))
    W["blocks.0.attn1.to_out.0.bias"] = a
    W["blocks.0.attn2.to_out.0.bias"] = c
    W["blocks.0.ffn.net.2.bias"] = f
    out = O.block_forward(x, ctx, mod, O.block_weights(W, 0), ang, cfg)
    ref = x + a * mod[:, :, 2] + c + f * mod[:, :, 5]
    torch.testing.assert_close(out, ref, rtol=1e-12, atol=1e-12)


def test_block_norm1_modulation():
    """q = k = 0 gives uniform attention; with v = out = identity the branch is
    the token mean of LN(x)*(1+scale)+shift (rows 0 and 1), gated by row 2."""
    cfg = tiny_cfg()
    W, x, ctx, mod, ang, _ = probe_setup(cfg)
    D = cfg["dim"]
    W["blocks.0.attn1.to_v.weight"] = torch.eye(D, dtype=DT)
    W["blocks.0.attn1.to_out.0.weight"] = torch.eye(D, dtype=DT)
    out = O.block_forward(x, ctx, mod, O.block_weights(W, 0), ang, cfg)
    y = Fn.layer_norm(x, (D,), eps=cfg["eps"]) * (1 + mod[:, :, 1]) + mod[:, :, 0]
    ref = x + y.mean(1, keepdim=True) * mod[:, :, 2]
    torch.testing.assert_close(out, ref, rtol=1e-12, atol=1e-12)


def test_block_ffn_modulation():
    """FFN branch alone: x + c_gate * GELU(LN(x)*(1+c_scale)+c_shift) (rows 3, 4, 5)."""
    cfg = tiny_cfg()
    W, x, ctx, mod, ang, _ = probe_setup(cfg)
    D, Fd = cfg["dim"], cfg["ffn_dim"]
    W["blocks.0.ffn.net.0.proj.weight"] = torch.eye(Fd, D, dtype=DT)
    W["blocks.0.ffn.net.2.weight"] = torch.eye(D, Fd, dtype=DT)
    out = O.block_forward(x, ctx, mod, O.block_weights(W, 0), ang, cfg)
    y = Fn.layer_norm(x, (D,), eps=cfg["eps"]) * (1 + mod[:, :, 4]) + mod[:, :, 3]
    ref = x + Fn.gelu(y, approximate="tanh") * mod[:, :, 5]
    torch.testing.assert_close(out, ref, rtol=1e-12, atol=1e-12)


def test_block_cross_attention_reads_context():
    """q = k = 0 in attn2: uniform over the context rows, so the branch adds
    Wo(Wv mean(ctx) + bv) + bo whatever the video tokens hold."""
    cfg = tiny_cfg()
    W, x, ctx, mod, ang, g = probe_setup(cfg)
    D = cfg["dim"]
    bv = torch.randn(D, generator=g, dtype=DT)
    W["blocks.0.attn2.to_v.weight"] = torch.eye(D, dtype=DT)
    W["blocks.0.attn2.to_v.bias"] = bv
    W["blocks.0.attn2.to_out.0.weight"] = torch.eye(D, dtype=DT) * 2.0
    out = O.block_forward(x, ctx, mod, O.block_weights(W, 0), ang, cfg)
    torch.testing.assert_close(out, x + 2.0 * (ctx.mean(1, keepdim=True) + bv), rtol=1e-12, atol=1e-12)


def test_block_norm2_is_affine_layernorm():
    """attn2 with identity projections: the queries are RMSNorm(LN2(x)) with
    the norm2 gain and bias, the keys RMSNorm(ctx) and the values ctx."""
    cfg = tiny_cfg()
    W, x, ctx, mod, ang, g = probe_setup(cfg, Lc=2)
    D = cfg["dim"]
    gam = 1 + torch.randn(D, generator=g, dtype=DT) * 0.3
    bet = torch.randn(D, generator=g, dtype=DT) * 0.3
    W["blocks.0.norm2.weight"] = gam
    W["blocks.0.norm2.bias"] = bet
    W["blocks.0.attn2.to_q.weight"] = torch.eye(D, dtype=DT)
    W["blocks.0.attn2.to_k.weight"] = torch.eye(D, dtype=DT)
    W["blocks.0.attn2.to_v.weight"] = torch.eye(D, dtype=DT)
    W["blocks.0.attn2.to_out.0.weight"] = torch.eye(D, dtype=DT)
    out = O.block_forward(x, ctx, mod, O.block_weights(W, 0), ang, cfg)
    yc = Fn.layer_norm(x, (D,), gam, bet, cfg["eps"])
    q = Fn.rms_norm(yc, (D,), eps=cfg["eps"]).reshape(1, -1, 2, 12).transpose(1, 2)
    k = Fn.rms_norm(ctx, (D,), eps=cfg["eps"]).reshape(1, -1, 2, 12).transpose(1, 2)
    v = ctx.reshape(1, -1, 2, 12).transpose(1, 2)
    att = Fn.scaled_dot_product_attention(q, k, v).transpose(1, 2).reshape(1, -1, D)
    torch.testing.assert_close(out, x + att, rtol=1e-12, atol=1e-12)


def test_qk_norm_spans_all_heads():
    """RMSNorm across heads keeps the 10:1 ratio between two heads' norms; a
    per-head norm would make it 1:1."""
    cfg = tiny_cfg()
    W, x, ctx, mod, ang, _ = probe_setup(cfg)
    D = cfg["dim"]
    wq = torch.eye(D, dtype=DT)
    wq[12:, 12:] *= 0.1
    Wb = O.block_weights(W, 0)
    Wb["attn1.to_q.weight"] = wq
    Wb["attn1.to_k.weight"] = torch.eye(D, dtype=DT)
    y = torch.ones(1, 6, D, dtype=DT)
    q, k, _ = O.self_attention_qkv(y, Wb, ang, cfg)
    r = q[..., 0, :].norm(dim=-1) / q[..., 1, :].norm(dim=-1)
    torch.testing.assert_close(r, torch.full_like(r, 10.0), rtol=1e-12, atol=0)
    total = (q.reshape(1, 6, D) ** 2).mean(-1)
    torch.testing.assert_close(total, torch.ones_like(total), rtol=1e-5, atol=0)


def test_self_attention_is_full_and_cross_attention_is_order_free():
    cfg = tiny_cfg()
    W = rand_weights(cfg, seed=5)
    Wb = O.block_weights(W, 0)
    g = torch.Generator().manual_seed(9)
    x = torch.randn(1, 6, 24, generator=g, dtype=DT)
    ctx = torch.randn(1, 3, 24, generator=g, dtype=DT)
    mod = torch.randn(1, 1, 6, 24, generator=g, dtype=DT) * 0.3
    ang = O.rope_angles((1, 2, 3), cfg["rope_split"], cfg["rope_theta"])
    out = O.block_forward(x, ctx, mod, Wb, ang, cfg)
    x2 = x.clone()
    x2[0, -1] += torch.randn(24, generator=g, dtype=DT)   # the last token reaches the first (no mask)
    assert (O.block_forward(x2, ctx, mod, Wb, ang, cfg)[0, 0] - out[0, 0]).abs().max() > 1e-6
    perm = torch.tensor([2, 0, 1])           # keys carry no position in cross-attention
    torch.testing.assert_close(O.block_forward(x, ctx[:, perm], mod, Wb, ang, cfg), out, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- whole forward

def tiny_forward_inputs(cfg, B=1, seed=11, F=2, Hz=4, Wz=6, Lc=3):
    g = torch.Generator().manual_seed(seed)
    lat = torch.randn(B, cfg["in_ch"], F, Hz, Wz, generator=g, dtype=DT)
    ctx = torch.randn(B, Lc, cfg["text_dim"], generator=g, dtype=DT)
    t = torch.full((B,), 500.0, dtype=DT)
    return lat, t, ctx


def test_forward_with_closed_gates_is_head_of_patch_embedding():
    cfg = tiny_cfg(num_blocks=2)
    W = rand_weights(cfg, seed=2)
    W["condition_embedder.time_proj.weight"].zero_()
    W["condition_embedder.time_proj.bias"].zero_()
    for i in range(2):
        W[f"blocks.{i}.scale_shift_table"][0, 2].zero_()
        W[f"blocks.{i}.scale_shift_table"][0, 5].zero_()
        W[f"blocks.{i}.attn2.to_out.0.weight"].zero_()
        W[f"blocks.{i}.attn2.to_out.0.bias"].zero_()
    lat, t, ctx = tiny_forward_inputs(cfg)
    vel, outs = O.forward(lat, t, ctx, W, cfg, return_blocks=True)
    assert len(outs) == 3
    torch.testing.assert_close(outs[2], outs[0], rtol=0, atol=0)
    x0 = Fn.conv3d(lat, W["patch_embedding.weight"], W["patch_embedding.bias"], stride=(1, 2, 2))
    x0 = x0.flatten(2).transpose(1, 2)
    torch.testing.assert_close(outs[0], x0, rtol=1e-12, atol=1e-12)
    temb, _ = O.time_embedding(t, W, cfg)
    o = O.head_forward(x0, temb, W, cfg)
    torch.testing.assert_close(vel, brute_unpatchify(o, 4, 2, 4, 6, (1, 2, 2)), rtol=1e-12, atol=1e-12)


def test_head_modulation_rows():
    """Head table row 0 shifts, row 1 scales: with proj_out = [I | 0] the output
    is LN(x)*(1+scale)+shift on the first columns."""
    cfg = tiny_cfg(num_blocks=0, out_ch=6)
    D = cfg["dim"]
    g = torch.Generator().manual_seed(4)
    x = torch.randn(2, 5, D, generator=g, dtype=DT)
    temb = torch.randn(2, D, generator=g, dtype=DT)
    sst = torch.randn(1, 2, D, generator=g, dtype=DT)
    W = {"scale_shift_table": sst, "proj_out.weight": torch.eye(24, D, dtype=DT),
         "proj_out.bias": torch.zeros(24, dtype=DT)}
    out = O.head_forward(x, temb, W, cfg)
    ref = Fn.layer_norm(x, (D,), eps=cfg["eps"]) * (1 + sst[0, 1] + temb[:, None]) + sst[0, 0] + temb[:, None]
    torch.testing.assert_close(out, ref[..., :24], rtol=1e-12, atol=1e-12)


def test_forward_invariances():
    cfg = tiny_cfg(num_blocks=2)
    W = rand_weights(cfg, seed=7)
    lat, t, ctx = tiny_forward_inputs(cfg, B=1)
    v1 = O.forward(lat, t, ctx, W, cfg)
    # context rows carry no order
    torch.testing.assert_close(O.forward(lat, t, ctx[:, [2, 0, 1]], W, cfg), v1, rtol=1e-11, atol=1e-12)
    # batch entries are independent
    lat2, t2, ctx2 = tiny_forward_inputs(cfg, B=1, seed=12)
    vb = O.forward(torch.cat([lat, lat2]), torch.cat([t, t2]), torch.cat([ctx, ctx2]), W, cfg)
    torch.testing.assert_close(vb[:1], v1, rtol=1e-12, atol=1e-13)
    torch.testing.assert_close(vb[1:], O.forward(lat2, t2, ctx2, W, cfg), rtol=1e-12, atol=1e-13)
    # a per-token timestep that is constant equals the per-sample one
    L = O.token_count(2, 4, 6)
    vt = O.forward(lat, t[:, None].expand(1, L).contiguous(), ctx, W, cfg)
    torch.testing.assert_close(vt, v1, rtol=1e-12, atol=1e-13)


def test_row_sampling_matches_full_forward():
    cfg = tiny_cfg(num_blocks=1)
    W = rand_weights(cfg, seed=8)
    lat, t, ctx = tiny_forward_inputs(cfg, B=2)
    vel = O.forward(lat, t, ctx, W, cfg)
    rows = torch.tensor([0, 3, 5])
    o = O.forward(lat, t, ctx, W, cfg, rows=rows)
    idx = O.unpatch_index_map(4, 2, 4, 6)[rows]
    torch.testing.assert_close(o, vel.reshape(2, -1)[:, idx], rtol=1e-12, atol=1e-13)
    # per-token timestep with row sampling
    L = O.token_count(2, 4, 6)
    tt = torch.rand(2, L, dtype=DT) * 1000
    vel = O.forward(lat, tt, ctx, W, cfg)
    o = O.forward(lat, tt, ctx, W, cfg, rows=rows)
    torch.testing.assert_close(o, vel.reshape(2, -1)[:, idx], rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- I2V route and MoE switch

@pytest.mark.parametrize("case", GOLD["i2v"]["input_channels"], ids=lambda c: str(c["z_dim"]))
def test_i2v_input_is_a_channel_concat(case):
    z, m = case["z_dim"], case["mask_channels"]
    g = torch.Generator().manual_seed(20)
    noisy = torch.randn(1, z, 3, 4, 4, generator=g, dtype=DT)
    cond = torch.randn(1, z, 3, 4, 4, generator=g, dtype=DT)
    mask = torch.randn(1, m, 3, 4, 4, generator=g, dtype=DT)
    x = O.i2v_input(noisy, cond, mask)
    assert x.shape == (1, case["in_ch"], 3, 4, 4)          # channel axis, frames unchanged
    assert torch.equal(x[:, :z], noisy) and torch.equal(x[:, z:2 * z], cond) and torch.equal(x[:, 2 * z:], mask)
    with pytest.raises(ValueError):
        O.i2v_input(noisy, cond, mask[:, :, :2])             # the mask must cover the same frames


def test_i2v_patch_features_and_image_table():
    pi, it = GOLD["i2v"]["patch_in"], GOLD["i2v"]["image_tokens"]
    cfg = configs.model_config("wan2.1-i2v-14b")
    assert cfg["in_ch"] * math.prod(cfg["patch"]) == pi["features"] and cfg["dim"] == pi["dim"]
    assert cfg["image_dim"] == it["width"]
    shapes = O.param_shapes(cfg)
    assert shapes["patch_embedding.weight"] == (pi["dim"], pi["in_ch"], *pi["patch"])
    assert shapes["condition_embedder.image_embedder.linear_1.weight"] == (cfg["dim"], it["width"])
    # the image branch adds exactly its embedder and two projections + one gain per block
    extra = O.param_count(cfg) - O.param_count(dict(cfg, image_dim=0, in_ch=36))
    D = cfg["dim"]
    assert extra == D * it["width"] + D + D * D + D + cfg["num_blocks"] * (2 * (D * D + D) + D)


def i2v_tiny():
    cfg = tiny_cfg(num_blocks=2, in_ch=9, image_dim=10)
    W = rand_weights(cfg, seed=21)
    g = torch.Generator().manual_seed(22)
    lat = torch.randn(2, 9, 2, 4, 6, generator=g, dtype=DT)
    ctx = torch.randn(2, 3, cfg["text_dim"], generator=g, dtype=DT)
    img = torch.randn(2, 5, 10, generator=g, dtype=DT)
    t = torch.full((2,), 700.0, dtype=DT)
    return cfg, W, lat, t, ctx, img


def test_i2v_image_branch_is_additive():
    """With the image value projection at zero the image attention outputs zero, so
    the I2V forward equals the forward without image tokens (same other weights)."""
    cfg, W, lat, t, ctx, img = i2v_tiny()
    v_img = O.forward(lat, t, ctx, W, cfg, image=img)
    v_txt = O.forward(lat, t, ctx, W, cfg)
    assert (v_img - v_txt).abs().max() > 1e-3                # the branch does something
    for i in range(2):
        W[f"blocks.{i}.attn2.add_v_proj.weight"].zero_()
        W[f"blocks.{i}.attn2.add_v_proj.bias"].zero_()
    torch.testing.assert_close(O.forward(lat, t, ctx, W, cfg, image=img), v_txt, rtol=1e-12, atol=1e-13)


def test_i2v_single_image_token_closed_form():
    """One image token: its softmax weight is 1, so the image attention returns its
    value row for every query; the block output follows by hand."""
    cfg, W, lat, t, ctx, img = i2v_tiny()
    Wb = O.block_weights(W, 0)
    g = torch.Generator().manual_seed(23)
    yc = torch.randn(2, 7, cfg["dim"], generator=g, dtype=DT)
    ctx_e = O.text_embedding(ctx, W)
    img_e = O.image_embedding(img[:, :1], W)
    got = O.cross_attention(yc, ctx_e, Wb, cfg, img_e)
    eps = cfg["eps"]
    q = O.rms_norm(O.linear(yc, Wb["attn2.to_q.weight"], Wb["attn2.to_q.bias"]), eps, Wb["attn2.norm_q.weight"])
    k = O.rms_norm(O.linear(ctx_e, Wb["attn2.to_k.weight"], Wb["attn2.to_k.bias"]), eps, Wb["attn2.norm_k.weight"])
    v = O.linear(ctx_e, Wb["attn2.to_v.weight"], Wb["attn2.to_v.bias"])
    hq = lambda z: z.reshape(z.shape[0], z.shape[1], cfg["heads"], cfg["head_dim"]).transpose(1, 2)
    o_txt = Fn.scaled_dot_product_attention(hq(q), hq(k), hq(v)).transpose(1, 2).reshape(q.shape)
    vi = O.linear(img_e, Wb["attn2.add_v_proj.weight"], Wb["attn2.add_v_proj.bias"])   # [2, 1, D]
    ref = O.linear(o_txt + vi, Wb["attn2.to_out.0.weight"], Wb["attn2.to_out.0.bias"])
    torch.testing.assert_close(got, ref, rtol=1e-11, atol=1e-12)


def test_i2v_image_tokens_carry_no_order_and_are_per_sample():
    cfg, W, lat, t, ctx, img = i2v_tiny()
    v = O.forward(lat, t, ctx, W, cfg, image=img)
    torch.testing.assert_close(O.forward(lat, t, ctx, W, cfg, image=img[:, [4, 2, 0, 1, 3]]), v,
                               rtol=1e-11, atol=1e-12)
    # sample 1's image does not reach sample 0
    img2 = img.clone()
    img2[1] = torch.randn(5, 10, dtype=DT)
    v2 = O.forward(lat, t, ctx, W, cfg, image=img2)
    torch.testing.assert_close(v2[0], v[0], rtol=0, atol=0)
    assert (v2[1] - v[1]).abs().max() > 1e-6


def test_image_embedding_is_two_linears_around_gelu():
    cfg, W, lat, t, ctx, img = i2v_tiny()
    p = "condition_embedder.image_embedder."
    h = Fn.linear(img, W[p + "linear_1.weight"], W[p + "linear_1.bias"])
    ref = Fn.linear(Fn.gelu(h, approximate="tanh"), W[p + "linear_2.weight"], W[p + "linear_2.bias"])
    torch.testing.assert_close(O.image_embedding(img, W), ref, rtol=1e-12, atol=1e-13)


def test_moe_expert_switch():
    assert "boundary * num_train_timesteps" in GOLD["moe_switch"]["rule"]
    # a sampling schedule runs t downwards: the high-noise expert first, then the low-noise one, never back
    ts = torch.linspace(999, 0, 50)
    experts = [O.moe_expert(float(t), 0.875) for t in ts]
    assert experts[0] == 0 and experts[-1] == 1
    assert experts == sorted(experts)                       # one switch, high -> low
    assert O.moe_expert(875.0, 0.875) == 0                  # the comparison includes the boundary
    assert O.moe_expert(874.999, 0.875) == 1
    assert O.moe_expert(900.0, 0.9, 1000) == 0 and O.moe_expert(899.0, 0.9, 1000) == 1
    assert O.moe_expert(90.0, 0.9, 100) == 0                # scales with num_train_timesteps


# ---------------------------------------------------------------- sizes and generator table

@pytest.mark.parametrize("case", GOLD["model_sizes"], ids=lambda c: c["model"])
def test_parameter_count_matches_model_size(case):
    n = O.param_count(configs.model_config(case["model"]))
    assert abs(n - case["approx_params"]) / case["approx_params"] <= case["rel_tol"], n


def test_generator_table_matches_oracle_table():
    for name in configs.MODELS:
        cfg = configs.model_config(name, num_blocks=2)
        assert synth.param_shapes(cfg) == O.param_shapes(cfg)


# ---------------------------------------------------------------- flow matching around the forward

def test_flow_matching_worked_example():
    g = GOLD["flow_example"]
    z, eps, s = (torch.tensor(g[k], dtype=DT) for k in ("z", "eps", "sigma"))
    x = O.flow_interpolate(z, eps, s)
    assert x.item() == g["x_sigma"]
    v = O.flow_target(z, eps)
    assert v.item() == g["v_target"]
    assert (g["v_pred"] - v.item()) ** 2 == g["sq_err"]
    x1 = O.euler_step(x, g["sigma"], g["sigma_next"], v)
    assert x1.item() == g["x_next"]
    x2 = O.euler_step(x1, g["sigma_next"], g["sigma_last"], v)
    assert x2.item() == g["x_last"] == g["z"]


def test_cfg_combine_endpoints():
    vu = torch.randn(10, dtype=DT)
    vc = torch.randn(10, dtype=DT)
    assert torch.equal(O.cfg_combine(vu, vc, 0.0), vu)
    torch.testing.assert_close(O.cfg_combine(vu, vc, 1.0), vc, rtol=0, atol=1e-15)
    torch.testing.assert_close(O.cfg_combine(vu, vc, 6.0), vu + 6.0 * (vc - vu))


# ---------------------------------------------------------------- conditioning MLPs against library layers

def test_text_embedding_is_two_linears_around_gelu():
    """R4 (config of the smallest case: Linear-GELU-Linear, GELU in its tanh
    form): the text path against torch's own linear and tanh-GELU layers."""
    cfg = tiny_cfg()
    W = rand_weights(cfg, seed=21)
    ctx = torch.randn(2, 5, cfg["text_dim"], generator=torch.Generator().manual_seed(22), dtype=DT)
    p = "condition_embedder.text_embedder."
    h = Fn.linear(ctx, W[p + "linear_1.weight"], W[p + "linear_1.bias"])
    ref = Fn.linear(Fn.gelu(h, approximate="tanh"), W[p + "linear_2.weight"], W[p + "linear_2.bias"])
    torch.testing.assert_close(O.text_embedding(ctx, W), ref, rtol=1e-12, atol=1e-13)
    # the activation matters at this scale: a dropped or exact-erf GELU would not match
    assert (Fn.linear(h, W[p + "linear_2.weight"], W[p + "linear_2.bias"]) - ref).abs().max() > 1e-3
    erf = Fn.linear(Fn.gelu(h), W[p + "linear_2.weight"], W[p + "linear_2.bias"])
    assert (erf - ref).abs().max() > 1e-6


def test_time_embedding_wiring():
    """R3: temb = L2(SiLU(L1(sinusoid(t)))), timestep_proj = Lp(SiLU(temb)) of
    width 6D, unflattened to [6, D] chunk by chunk -- against torch's linear and
    SiLU layers; the printed shapes temb (1, D), projection (1, 6D) -> (1, 6, D)
    are those of the 480p listing."""
    cfg = tiny_cfg()
    W = rand_weights(cfg, seed=23)
    D = cfg["dim"]
    t = torch.tensor([999.0, 500.0, 20.0], dtype=DT)
    p = "condition_embedder."
    e = O.timestep_sinusoid(t, cfg["freq_dim"])
    h = Fn.silu(Fn.linear(e, W[p + "time_embedder.linear_1.weight"], W[p + "time_embedder.linear_1.bias"]))
    temb_ref = Fn.linear(h, W[p + "time_embedder.linear_2.weight"], W[p + "time_embedder.linear_2.bias"])
    proj_ref = Fn.linear(Fn.silu(temb_ref), W[p + "time_proj.weight"], W[p + "time_proj.bias"])
    temb, proj = O.time_embedding(t, W, cfg)
    assert temb.shape == (3, D) and proj.shape == (3, 6, D)
    torch.testing.assert_close(temb, temb_ref, rtol=1e-12, atol=1e-13)
    for k in range(6):      # chunk k of the 6D projection is modulation row k
        torch.testing.assert_close(proj[:, k], proj_ref[:, k * D:(k + 1) * D], rtol=1e-12, atol=1e-13)
    # per-token timesteps [B, L] give per-token rows of the same map
    tt = torch.tensor([[0.0, 250.0], [999.0, 20.0]], dtype=DT)
    temb2, proj2 = O.time_embedding(tt, W, cfg)
    assert temb2.shape == (2, 2, D) and proj2.shape == (2, 2, 6, D)
    torch.testing.assert_close(temb2[1, 0], O.time_embedding(tt[1, :1], W, cfg)[0][0], rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- flow-shift schedule (reading R22)

def test_flow_shift_values_and_closed_forms():
    g = GOLD["flow_shift"]
    assert g["480p"] == 3.0 and g["720p"] == 5.0
    sig = torch.linspace(0, 1, 101, dtype=DT)
    for s in (g["480p"], g["720p"], 0.5, 1.7):
        y = O.flow_shift(sig, s)
        assert y[0].item() == 0.0 and y[-1].item() == 1.0              # endpoints stay
        assert bool((y[1:] > y[:-1]).all())                             # order of noise levels kept
        mid = sig[1:-1]
        ym = y[1:-1]
        torch.testing.assert_close(ym / (1 - ym), s * mid / (1 - mid), rtol=1e-12, atol=0)  # odds times s
        if s > 1:
            assert bool((ym > mid).all())                               # more of the run at high noise
    # the shift is a one-parameter group: applied twice it compounds (the pitfall the
    # pages warn of), the constructor's fixed 1 is neutral, and 1/s undoes s
    for a, b in ((3.0, 5.0), (2.0, 0.25)):
        torch.testing.assert_close(O.flow_shift(O.flow_shift(sig, a), b), O.flow_shift(sig, a * b),
                                   rtol=1e-12, atol=1e-15)
    torch.testing.assert_close(O.flow_shift(O.flow_shift(sig, g["constructor_shift"]), 3.0), O.flow_shift(sig, 3.0),
                               rtol=0, atol=1e-16)
    torch.testing.assert_close(O.flow_shift(O.flow_shift(sig, 5.0), 1 / 5.0), sig, rtol=1e-12, atol=1e-15)
    assert abs(O.flow_shift(0.5, 3.0).item() - 0.75) < 1e-15            # s / (1 + s) at the midpoint


def test_sampling_sigmas_and_timesteps():
    for steps in (1, 4, 50):
        torch.testing.assert_close(O.sampling_sigmas(steps, 1.0),
                                   torch.linspace(1, 0, steps + 1, dtype=DT), rtol=0, atol=1e-15)
    s = O.sampling_sigmas(50, 3.0)
    assert s.shape == (51,) and s[0].item() == 1.0 and s[-1].item() == 0.0
    assert bool((s[1:] < s[:-1]).all())
    ts = O.sampling_timesteps(50, 3.0)
    assert ts.shape == (50,) and ts[0].item() == 1000.0
    torch.testing.assert_close(ts, s[:50] * 1000)
    # the Euler walk over the schedule with the exact velocity lands on the data
    # (the worked example's straight path, at every step count and shift)
    z, eps = torch.tensor(2.0, dtype=DT), torch.tensor(10.0, dtype=DT)
    for steps, shift in ((4, 1.0), (7, 3.0), (30, 5.0)):
        sig = O.sampling_sigmas(steps, shift)
        x = O.flow_interpolate(z, eps, sig[0])
        for i in range(steps):
            x = O.euler_step(x, sig[i], sig[i + 1], O.flow_target(z, eps))
        assert abs(x.item() - 2.0) < 1e-12
    # a larger shift keeps more steps above the A14B switch point (the drift the pages warn of)
    hi = [int((O.sampling_timesteps(50, s) >= 875.0).sum()) for s in (1.0, 3.0, 5.0)]
    assert hi[0] < hi[1] < hi[2]

"""Seeded synthetic inputs and random-init weights for the Wan DiT forward.

This module only draws numbers: it holds none of the method's arithmetic, so
both the CUDA path and the float64 oracle can be fed from it.  Every tensor gets
its own generator seeded with ``seed * 2**31 + crc32(name)``, draws float32
N(0, 1), scales it and (for matrices, biases, latents and contexts) rounds it to
bf16 so the same bytes reach both sides.

Distributions (the synthetic workloads of the Wan shapes):
* every Linear / Conv3d weight and bias: N(0, 0.02), bf16 values;
* q/k RMSNorm gains and the norm2 gain: 1 + N(0, 0.02), float32;
* norm2 bias: N(0, 0.02), float32;
* block and head ``scale_shift_table``: N(0, 1) / sqrt(dim), float32;
* latent: N(0, 1) bf16 values held in float32; text context: N(0, 1) bf16;
* per-token timestep: 0 on the first latent frame, U[0, 1000) elsewhere.
"""
from __future__ import annotations

import math
import zlib
from typing import Dict, Tuple

import torch


def _gen(seed: int, name: str, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 2 ** 31 + zlib.crc32(name.encode())) % (2 ** 63))
    return g


def _randn(shape, seed, name, device):
    return torch.randn(*shape, generator=_gen(seed, name, device), device=device, dtype=torch.float32)


def param_shapes(cfg) -> Dict[str, Tuple[int, ...]]:
    """Names and shapes of every DiT parameter (diffusers-style names)."""
    D, Fd, C, Co = cfg["dim"], cfg["ffn_dim"], cfg["in_ch"], cfg["out_ch"]
    pt, ph, pw = cfg["patch"]
    s = {"patch_embedding.weight": (D, C, pt, ph, pw), "patch_embedding.bias": (D,)}
    ce = "condition_embedder."
    for n, (o, i) in (("time_embedder.linear_1", (D, cfg["freq_dim"])), ("time_embedder.linear_2", (D, D)),
                      ("time_proj", (6 * D, D)), ("text_embedder.linear_1", (D, cfg["text_dim"])),
                      ("text_embedder.linear_2", (D, D))):
        s[ce + n + ".weight"] = (o, i)
        s[ce + n + ".bias"] = (o,)
    for b in range(cfg["num_blocks"]):
        p = f"blocks.{b}."
        s[p + "scale_shift_table"] = (1, 6, D)
        for a in ("attn1", "attn2"):
            for n in ("to_q", "to_k", "to_v", "to_out.0"):
                s[p + f"{a}.{n}.weight"] = (D, D)
                s[p + f"{a}.{n}.bias"] = (D,)
            s[p + f"{a}.norm_q.weight"] = (D,)
            s[p + f"{a}.norm_k.weight"] = (D,)
        s[p + "norm2.weight"] = (D,)
        s[p + "norm2.bias"] = (D,)
        s[p + "ffn.net.0.proj.weight"] = (Fd, D)
        s[p + "ffn.net.0.proj.bias"] = (Fd,)
        s[p + "ffn.net.2.weight"] = (D, Fd)
        s[p + "ffn.net.2.bias"] = (D,)
        if cfg.get("image_dim", 0):  # image branch of the cross-attention (I2V)
            for n in ("add_k_proj", "add_v_proj"):
                s[p + f"attn2.{n}.weight"] = (D, D)
                s[p + f"attn2.{n}.bias"] = (D,)
            s[p + "attn2.norm_added_k.weight"] = (D,)
    if cfg.get("image_dim", 0):
        for n, (o, i) in (("image_embedder.linear_1", (D, cfg["image_dim"])), ("image_embedder.linear_2", (D, D))):
            s[ce + n + ".weight"] = (o, i)
            s[ce + n + ".bias"] = (o,)
    s["scale_shift_table"] = (1, 2, D)
    s["proj_out.weight"] = (Co * pt * ph * pw, D)
    s["proj_out.bias"] = (Co * pt * ph * pw,)
    return s


def weight_kind(name: str) -> str:
    if name.endswith("scale_shift_table"):
        return "table"
    if ".norm_q." in name or ".norm_k." in name or ".norm2.weight" in name or ".norm_added_k." in name:
        return "gain"
    if ".norm2.bias" in name:
        return "fp32bias"
    return "linear"


def make_weight(cfg, name, shape, seed=0, device="cpu") -> torch.Tensor:
    z = _randn(shape, seed, name, device)
    kind = weight_kind(name)
    if kind == "table":
        return z / math.sqrt(cfg["dim"])
    if kind == "gain":
        return 1.0 + 0.02 * z
    if kind == "fp32bias":
        return 0.02 * z
    return (0.02 * z).to(torch.bfloat16)


def make_weights(cfg, seed=0, device="cpu", blocks=None) -> Dict[str, torch.Tensor]:
    """All parameters (or those of the given block indices plus the shared
    ones).  Linear/Conv weights come back as bf16 tensors, the rest float32."""
    out = {}
    for name, shape in param_shapes(cfg).items():
        if blocks is not None and name.startswith("blocks."):
            if int(name.split(".")[1]) not in blocks:
                continue
        out[name] = make_weight(cfg, name, shape, seed, device)
    return out


def make_latent(shape, seed=0, device="cpu", same_across_batch=False) -> torch.Tensor:
    """Latent [B, C, F, Hz, Wz] float32 holding bf16 values of N(0, 1)."""
    if same_across_batch:
        one = _randn((1,) + tuple(shape[1:]), seed, "latent", device)
        z = one.expand(*shape).contiguous()
    else:
        z = _randn(shape, seed, "latent", device)
    return z.to(torch.bfloat16).to(torch.float32)


def make_context(B, Lc, text_dim, seed=0, device="cpu") -> torch.Tensor:
    """Text context [B, Lc, text_dim] bf16 of N(0, 1) (stands in for umT5 output)."""
    return _randn((B, Lc, text_dim), seed, "context", device).to(torch.bfloat16)


def make_image(B, Li, image_dim, seed=0, device="cpu") -> torch.Tensor:
    """Image tokens [B, Li, image_dim] bf16 of N(0, 1) (stands in for CLIP output)."""
    return _randn((B, Li, image_dim), seed, "image", device).to(torch.bfloat16)


def make_timestep(B, value) -> torch.Tensor:
    return torch.full((B,), float(value), dtype=torch.float32)


def make_timestep_per_token(B, L, tokens_first_frame, seed=0) -> torch.Tensor:
    """[B, L] float32: 0 on the first latent frame (a clean frame), U[0,1000) after."""
    g = _gen(seed, "timestep", "cpu")
    t = torch.rand(B, L, generator=g, dtype=torch.float32) * 1000.0
    t[:, :tokens_first_frame] = 0.0
    return t


# ---------------------------------------------------------------- Wan2.1 VAE decoder
VAE_DIMS = (384, 384, 384, 192, 96)    # conv_in width, then the up blocks' widths


def vae_param_shapes(z_dim: int = 16) -> Dict[str, Tuple[int, ...]]:
    """Names and shapes of the decoder parameters (post_quant_conv, conv_in, mid
    block, four up blocks of three residual blocks, upsamplers, head)."""
    s: Dict[str, Tuple[int, ...]] = {}

    def conv(n, cin, cout, k):
        s[n + ".weight"] = (cout, cin) + tuple(k)
        s[n + ".bias"] = (cout,)

    def norm(n, c):
        s[n + ".gamma"] = (c,)
        s[n + ".bias"] = (c,)

    def res(n, cin, cout):
        norm(n + ".norm1", cin)
        conv(n + ".conv1", cin, cout, (3, 3, 3))
        norm(n + ".norm2", cout)
        conv(n + ".conv2", cout, cout, (3, 3, 3))
        if cin != cout:
            conv(n + ".conv_shortcut", cin, cout, (1, 1, 1))

    d = VAE_DIMS
    conv("post_quant_conv", z_dim, z_dim, (1, 1, 1))
    conv("decoder.conv_in", z_dim, d[0], (3, 3, 3))
    res("decoder.mid_block.resnets.0", d[0], d[0])
    a = "decoder.mid_block.attentions.0"
    norm(a + ".norm", d[0])
    s[a + ".to_qkv.weight"] = (3 * d[0], d[0], 1, 1)
    s[a + ".to_qkv.bias"] = (3 * d[0],)
    s[a + ".proj.weight"] = (d[0], d[0], 1, 1)
    s[a + ".proj.bias"] = (d[0],)
    res("decoder.mid_block.resnets.1", d[0], d[0])
    for i in range(4):
        cin, cout = d[i] if i == 0 else d[i] // 2, d[i + 1]
        for r in range(3):
            res(f"decoder.up_blocks.{i}.resnets.{r}", cin if r == 0 else cout, cout)
        if i < 3:
            u = f"decoder.up_blocks.{i}.upsamplers.0"
            s[u + ".resample.1.weight"] = (cout // 2, cout, 3, 3)
            s[u + ".resample.1.bias"] = (cout // 2,)
            if i < 2:
                conv(u + ".time_conv", cout, 2 * cout, (3, 1, 1))
    norm("decoder.norm_out", d[4])
    conv("decoder.conv_out", d[4], 3, (3, 3, 3))
    return s


def make_vae_weights(seed=0, device="cpu") -> Dict[str, torch.Tensor]:
    """Random decoder parameters, float32: weights N(0, 1) / sqrt(fan_in) rounded
    to bf16 values, biases N(0, 0.1^2), norm gains 1 + N(0, 0.1^2)."""
    out = {}
    for name, shape in vae_param_shapes().items():
        z = _randn(shape, seed, name, device)
        if name.endswith(".weight"):
            fan = 1
            for v in shape[1:]:
                fan *= v
            out[name] = (z / math.sqrt(max(1, fan))).to(torch.bfloat16).to(torch.float32)
        elif name.endswith(".gamma"):
            out[name] = 1.0 + 0.1 * z
        else:
            out[name] = 0.1 * z
    return out


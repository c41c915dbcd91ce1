"""Plain float64 CPU oracle of the Wan2.1 VAE decoder (latent video -> pixels).

TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT PATH.  Only ``tests/`` may
import, call or execute this module.  It shares no code with the CUDA library.

Follows the decoder walk-through of [PSWP-WAN] (pswp.cn notes on diffusers
``WanPipeline``, sections "vae.decode", "WanDecoder3d", "WanCausalConv3d" and
"upsample blocks"), built from PyTorch CPU library primitives (conv3d, conv2d,
interpolate, matmul) in float64 with no intermediate rounding.  What the pages
fix:

* ``vae.decode``: a 1x1x1 ``post_quant_conv`` on the latent, then the decoder
  run latent frame by latent frame with a feature cache of the last
  ``CACHE_T = 2`` frames per causal convolution (33 of them for the Wan2.1
  VAE), the per-frame outputs concatenated on the time axis and clamped to
  [-1, 1];
* ``WanCausalConv3d``: zero padding of 2 p_t frames before and none after on
  the time axis, p_h / p_w on both sides spatially; with a cache the cached
  frames replace that many leading zero frames;
* ``WanDecoder3d``: conv_in (z_dim -> 384), mid block, four up blocks, RMS
  norm, SiLU, conv_out (96 -> 3), with the printed shapes of one non-first
  latent frame (1,384,1,60,104) -> (1,192,2,120,208) -> (1,192,4,240,416) ->
  (1,96,4,480,832) -> (1,96,4,480,832);
* up blocks: three residual blocks each (norm1, SiLU, conv1 3x3x3, norm2,
  dropout, conv2 3x3x3, shortcut 1x1x1 when the width changes), upsamplers
  ``upsample3d`` (time_conv (3,1,1) doubling the channels, then nearest-exact
  2x spatial and a 3x3 Conv2d halving them) for blocks 0 and 1,
  ``upsample2d`` (the spatial part only) for block 2, none for block 3.

Readings where the pages leave a step open (also in the design notes):

V1  RMS norm (WanRMS_norm, not printed): over the channel axis,
    x * rsqrt(mean_c x^2 + eps) * gamma + beta, eps 1e-12; gamma, beta per
    channel.
V2  mid block (not printed): residual block, single-head spatial attention per
    frame (RMS norm, 1x1 q/k/v projection, softmax over the H*W positions
    with scale 1/sqrt(C), 1x1 output projection, residual), residual block.
    The 33-convolution count of the pages fixes the two residual blocks.
V3  residual block order: h = conv1(SiLU(norm1(x))); h = conv2(SiLU(norm2(h)));
    out = h + shortcut(x) (dropout p = 0).
V4  time upsampling: time_conv maps C -> 2C channels per frame; channel half
    0 becomes frame 2t and half 1 frame 2t+1.  The first latent frame of the
    video is not time-upsampled (21 latent frames give 1 + 4 * 20 = 81 video
    frames, the frame law of the pages); the cache of time_conv starts
    after it.
V5  decoder head: RMS norm, SiLU, causal conv 96 -> 3 (3x3x3).

Parity unpinned: V1's eps and affine form, the mid-block attention (V2), the
block-internal order (V3) and the channel-half-to-frame assignment (V4); the
pins below fix everything the pages print (padding rule, cache semantics,
frame and size laws, channel schedule, convolution count, clamp).
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Tuple

import torch
import torch.nn.functional as Fn

DT = torch.float64
CACHE_T = 2

# Wan2.1 VAE decoder widths (conv_in output 384; up blocks 384 -> 192 -> 192 -> 96)
Z_DIM = 16
BASE = 96
DIM_MULT = (1, 2, 4, 4)


# --------------------------------------------------------------------------
# building blocks
# --------------------------------------------------------------------------

def causal_conv3d(x: torch.Tensor, w: torch.Tensor, b: torch.Tensor, cache: Optional[torch.Tensor] = None):
    """``WanCausalConv3d`` ([PSWP-WAN] "WanCausalConv3d"): kernel (kt, kh, kw),
    padding p = ((kt-1)/2, (kh-1)/2, (kw-1)/2); the input is padded with 2 p_t
    zero frames before (none after) and p_h, p_w on both spatial sides.  With a
    cache [B, C, c, H, W] the cached frames are put in front and replace c of
    the leading zero frames."""
    kt, kh, kw = w.shape[2:]
    pt, ph, pw = (kt - 1) // 2, (kh - 1) // 2, (kw - 1) // 2
    front = 2 * pt
    if cache is not None and front > 0:
        x = torch.cat([cache, x], dim=2)
        front -= cache.shape[2]
    x = Fn.pad(x, (pw, pw, ph, ph, front, 0))
    return Fn.conv3d(x, w, b)


def rms_norm_c(x: torch.Tensor, gamma: torch.Tensor, beta: torch.Tensor, eps: float = 1e-12) -> torch.Tensor:
    """Reading V1: RMS over the channel axis (dim 1), per-channel gain and bias."""
    shape = (1, -1) + (1,) * (x.dim() - 2)
    return x * torch.rsqrt((x * x).mean(dim=1, keepdim=True) + eps) * gamma.reshape(shape) + beta.reshape(shape)


def silu(x):
    return x * torch.sigmoid(x)


def upsample_nearest2x(x: torch.Tensor) -> torch.Tensor:
    """Nearest-exact 2x spatial upsampling of [N, C, H, W]: pixel (i, j) of the
    output takes input (i // 2, j // 2)."""
    N, C, H, W = x.shape
    i = torch.arange(2 * H) // 2
    j = torch.arange(2 * W) // 2
    return x[:, :, i][:, :, :, j]


# --------------------------------------------------------------------------
# parameter table
# --------------------------------------------------------------------------

def decoder_layout(z_dim: int = Z_DIM, base: int = BASE, mult=DIM_MULT):
    """Module list of the decoder in execution order.  Entries:
    ("conv", name, cin, cout, k) causal conv; ("res", name, cin, cout) residual
    block; ("attn", name, c) mid-block attention; ("up3d"|"up2d", name, c)
    upsampler; ("norm", name, c)."""
    dims = [base * m for m in (mult[-1],) + tuple(reversed(mult))]   # 384, 384, 384, 192, 96
    L = [("conv", "post_quant_conv", z_dim, z_dim, (1, 1, 1)), ("conv", "decoder.conv_in", z_dim, dims[0], (3, 3, 3)),
         ("res", "decoder.mid_block.resnets.0", dims[0], dims[0]), ("attn", "decoder.mid_block.attentions.0", dims[0]),
         ("res", "decoder.mid_block.resnets.1", dims[0], dims[0])]
    for i in range(len(mult)):
        cin, cout = dims[i], dims[i + 1]
        if i in (1, 2, 3):
            cin = cin // 2          # the previous upsampler halved the width
        for r in range(3):
            L.append(("res", f"decoder.up_blocks.{i}.resnets.{r}", cin if r == 0 else cout, cout))
        if i < len(mult) - 1:
            kind = "up3d" if i < 2 else "up2d"
            L.append((kind, f"decoder.up_blocks.{i}.upsamplers.0", cout))
    L += [("norm", "decoder.norm_out", dims[-1]), ("conv", "decoder.conv_out", dims[-1], 3, (3, 3, 3))]
    return L


def param_shapes(z_dim: int = Z_DIM, base: int = BASE, mult=DIM_MULT) -> Dict[str, Tuple[int, ...]]:
    s = {}

    def conv(n, cin, cout, k):
        s[n + ".weight"] = (cout, cin) + tuple(k)
        s[n + ".bias"] = (cout,)

    def norm(n, c):
        s[n + ".gamma"] = (c,)
        s[n + ".bias"] = (c,)

    for e in decoder_layout(z_dim, base, mult):
        kind, n = e[0], e[1]
        if kind == "conv":
            conv(n, e[2], e[3], e[4])
        elif kind == "res":
            cin, cout = e[2], e[3]
            norm(n + ".norm1", cin)
            conv(n + ".conv1", cin, cout, (3, 3, 3))
            norm(n + ".norm2", cout)
            conv(n + ".conv2", cout, cout, (3, 3, 3))
            if cin != cout:
                conv(n + ".conv_shortcut", cin, cout, (1, 1, 1))
        elif kind == "attn":
            c = e[2]
            norm(n + ".norm", c)
            s[n + ".to_qkv.weight"] = (3 * c, c, 1, 1)
            s[n + ".to_qkv.bias"] = (3 * c,)
            s[n + ".proj.weight"] = (c, c, 1, 1)
            s[n + ".proj.bias"] = (c,)
        elif kind in ("up3d", "up2d"):
            c = e[2]
            s[n + ".resample.1.weight"] = (c // 2, c, 3, 3)
            s[n + ".resample.1.bias"] = (c // 2,)
            if kind == "up3d":
                conv(n + ".time_conv", c, 2 * c, (3, 1, 1))
        elif kind == "norm":
            norm(n, e[2])
    return s


def causal_conv_names(z_dim: int = Z_DIM, base: int = BASE, mult=DIM_MULT) -> List[str]:
    """Names of the decoder's causal 3-D convolutions in cache order (the
    post_quant_conv runs outside the decoder and keeps no cache)."""
    out = []
    for e in decoder_layout(z_dim, base, mult):
        kind, n = e[0], e[1]
        if kind == "conv" and n != "post_quant_conv":
            out.append(n)
        elif kind == "res":
            out += [n + ".conv1", n + ".conv2"] + ([n + ".conv_shortcut"] if e[2] != e[3] else [])
        elif kind == "up3d":
            out.append(n + ".time_conv")
    return out


# --------------------------------------------------------------------------
# decoder, whole sequence or chunk by chunk with the frame cache
# --------------------------------------------------------------------------

class _Cache:
    """feat_cache of the pages: the last CACHE_T input frames of every causal
    convolution, filled in execution order."""

    def __init__(self, enabled: bool):
        self.enabled = enabled
        self.store: Dict[str, torch.Tensor] = {}

    def conv(self, name, x, W):
        w, b = W[name + ".weight"], W[name + ".bias"]
        if not self.enabled:
            return causal_conv3d(x, w, b)
        prev = self.store.get(name)
        keep = x[:, :, -CACHE_T:]
        if keep.shape[2] < CACHE_T and prev is not None:   # carry the last cached frame
            keep = torch.cat([prev[:, :, -1:], keep], dim=2)
        out = causal_conv3d(x, w, b, prev)
        self.store[name] = keep
        return out


def _res(x, n, cin, cout, W, cache):
    h = silu(rms_norm_c(x, W[n + ".norm1.gamma"], W[n + ".norm1.bias"]))
    h = cache.conv(n + ".conv1", h, W)
    h = silu(rms_norm_c(h, W[n + ".norm2.gamma"], W[n + ".norm2.bias"]))
    h = cache.conv(n + ".conv2", h, W)
    sc = cache.conv(n + ".conv_shortcut", x, W) if cin != cout else x
    return h + sc


def _attn(x, n, c, W):
    B, C, T, H, Wd = x.shape
    f = x.permute(0, 2, 1, 3, 4).reshape(B * T, C, H, Wd)
    h = rms_norm_c(f, W[n + ".norm.gamma"], W[n + ".norm.bias"])
    qkv = Fn.conv2d(h, W[n + ".to_qkv.weight"], W[n + ".to_qkv.bias"]).reshape(B * T, 3, C, H * Wd)
    q, k, v = qkv[:, 0].transpose(1, 2), qkv[:, 1].transpose(1, 2), qkv[:, 2].transpose(1, 2)   # [N, HW, C]
    s = (q @ k.transpose(1, 2)) / math.sqrt(C)
    p = torch.exp(s - s.amax(dim=-1, keepdim=True))
    o = (p / p.sum(dim=-1, keepdim=True)) @ v
    o = Fn.conv2d(o.transpose(1, 2).reshape(B * T, C, H, Wd), W[n + ".proj.weight"], W[n + ".proj.bias"])
    return (f + o).reshape(B, T, C, H, Wd).permute(0, 2, 1, 3, 4)


def _up(x, n, c, kind, W, cache, first):
    if kind == "up3d" and not first:
        # reading V4: C -> 2C channels per frame, halves interleaved into 2T frames
        y = cache.conv(n + ".time_conv", x, W)
        B, C2, T, H, Wd = y.shape
        y = y.reshape(B, 2, C2 // 2, T, H, Wd).permute(0, 2, 3, 1, 4, 5).reshape(B, C2 // 2, 2 * T, H, Wd)
        x = y
    elif kind == "up3d" and first and cache.enabled:
        cache.store.setdefault(n + ".time_conv", None)   # the cache of time_conv starts after the first frame
    B, C, T, H, Wd = x.shape
    f = x.permute(0, 2, 1, 3, 4).reshape(B * T, C, H, Wd)
    f = Fn.conv2d(upsample_nearest2x(f), W[n + ".resample.1.weight"], W[n + ".resample.1.bias"], padding=1)
    return f.reshape(B, T, C // 2, 2 * H, 2 * Wd).permute(0, 2, 1, 3, 4)


def _decoder(x, W, cache, first, layout, trace=None):
    """One chunk through the decoder; with ``trace`` (a list) the chunk's
    activation after conv_in and after every up block is appended."""
    for e in layout:
        kind, n = e[0], e[1]
        if n == "post_quant_conv":
            continue
        if kind == "conv":
            x = cache.conv(n, x, W)
        elif kind == "res":
            x = _res(x, n, e[2], e[3], W, cache)
        elif kind == "attn":
            x = _attn(x, n, e[2], W)
        elif kind in ("up3d", "up2d"):
            x = _up(x, n, e[2], kind, W, cache, first)
        elif kind == "norm":
            x = silu(rms_norm_c(x, W[n + ".gamma"], W[n + ".bias"]))   # reading V5: norm_out, SiLU, conv_out
        if trace is not None and (n == "decoder.conv_in" or _ends_up_block(layout, e)):
            trace.append(x)
    return x


def _ends_up_block(layout, e):
    """True for the last entry of an up block."""
    n = e[1]
    if not n.startswith("decoder.up_blocks."):
        return False
    i = layout.index(e)
    nxt = layout[i + 1][1] if i + 1 < len(layout) else ""
    return not nxt.startswith(".".join(n.split(".")[:3]) + ".")


def decode(z: torch.Tensor, W: Dict[str, torch.Tensor], frame_loop: bool = True, base: int = BASE,
           mult=DIM_MULT, trace: Optional[List[List[torch.Tensor]]] = None) -> torch.Tensor:
    """Latent [B, z_dim, T, H, W] -> video [B, 3, 1 + 4 (T - 1), 8 H, 8 W] in
    [-1, 1] ([PSWP-WAN] "vae.decode").  ``frame_loop`` runs the decoder one
    latent frame at a time with the CACHE_T feature cache, as the pages do;
    without it, the first latent frame and the remaining ones are decoded as
    two causal sequences (the cache carries exactly the causal context, so the
    two agree).  ``trace`` (frame loop only) receives, per latent frame, the
    activations after conv_in and after each up block."""
    layout = decoder_layout(z.shape[1], base, mult)
    x = causal_conv3d(z.to(DT), W["post_quant_conv.weight"], W["post_quant_conv.bias"])
    if frame_loop:
        cache = _Cache(True)
        outs = []
        for i in range(x.shape[2]):
            tr = [] if trace is not None else None
            outs.append(_decoder(x[:, :, i:i + 1], W, cache, i == 0, layout, tr))
            if trace is not None:
                trace.append(tr)
        out = torch.cat(outs, dim=2)
    else:
        out = _decode_sequence(x, W, layout)
    return out.clamp(-1.0, 1.0)


def _decode_sequence(x, W, layout):
    """Whole-sequence form of the frame loop, written without the cache: every
    causal convolution runs over all frames at its level at once, and each
    time upsampler keeps the first latent frame's output as one frame and runs
    time_conv causally over the frames after it (reading V4)."""
    def conv(n, h):
        return causal_conv3d(h, W[n + ".weight"], W[n + ".bias"])

    for e in layout:
        kind, n = e[0], e[1]
        if n == "post_quant_conv":
            continue
        if kind == "conv":
            x = conv(n, x)
        elif kind == "res":
            h = conv(n + ".conv1", silu(rms_norm_c(x, W[n + ".norm1.gamma"], W[n + ".norm1.bias"])))
            h = conv(n + ".conv2", silu(rms_norm_c(h, W[n + ".norm2.gamma"], W[n + ".norm2.bias"])))
            x = h + (conv(n + ".conv_shortcut", x) if e[2] != e[3] else x)
        elif kind == "attn":
            x = _attn(x, n, e[2], W)
        elif kind in ("up3d", "up2d"):
            if kind == "up3d" and x.shape[2] > 1:
                y = conv(n + ".time_conv", x[:, :, 1:])
                B, C2, T, H, Wd = y.shape
                y = y.reshape(B, 2, C2 // 2, T, H, Wd).permute(0, 2, 3, 1, 4, 5).reshape(B, C2 // 2, 2 * T, H, Wd)
                x = torch.cat([x[:, :, :1], y], dim=2)
            B, C, T, H, Wd = x.shape
            f = x.permute(0, 2, 1, 3, 4).reshape(B * T, C, H, Wd)
            f = Fn.conv2d(upsample_nearest2x(f), W[n + ".resample.1.weight"], W[n + ".resample.1.bias"], padding=1)
            x = f.reshape(B, T, C // 2, 2 * H, 2 * Wd).permute(0, 2, 1, 3, 4)
        elif kind == "norm":
            x = silu(rms_norm_c(x, W[n + ".gamma"], W[n + ".bias"]))
    return x

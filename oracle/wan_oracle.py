"""Plain float64 CPU oracle of one denoising-step forward of the Wan DiT.

TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT PATH.  Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference`` legs
of ``bench.py`` may import, call or execute anything under ``oracle/``.  The
CUDA library never calls back into this module and shares no code with it.

Every function follows the pages it cites, in float64, with no intermediate
rounding, built from PyTorch CPU library primitives (matmul, exp, sum, gather)
so a reader can check it against the pages by eye.  Page titles used in the
citations:

* [WAN21-GUIDE]  "【VLA与模仿学习】Wan2.1框架与训练源码导读" (CSDN) -- §3.1 latent
  shape law, §5.1 patchify and token law, §5.2 block order, §5.3 output head,
  §6.1/§6.3 flow-matching relations and worked example, §7 Euler step and CFG.
* [PSWP-WAN]     pswp.cn notes on diffusers ``WanPipeline`` (Wan2.1-T2V-1.3B,
  480p) -- sections "WanTransformer3DModel" (model forward listing with the
  printed intermediate shapes) and "WanTransformerBlock" (block forward listing,
  per-block ``scale_shift_table``).
* [ANIMATE-DIFF] "Diffusers 中 WanAnimateTransformer3DModel 深度解析" -- tables
  "配置参数全解" (qk_norm = rms_norm_across_heads, cross_attn_norm = True,
  freq_dim 256, eps 1e-6, attention_head_dim 128) and the forward pipeline
  section (RoPE per T/H/W axis, FP32 norm_out + scale-shift + proj_out,
  modules kept in FP32).
* [WOVR-README]  WoVR_Plus "Wan2.2 5B latent-ray + view-embedding" README --
  per-token timestep, VACE context shapes.

Readings taken where the pages leave a step open (the same list is in the
design notes of the repository):

R2  sinusoid: 128 frequencies omega_k = exp(-ln(1e4) k / 128), cos half first,
    timestep used raw (0..1000).
R3  time MLP: temb = L2(SiLU(L1(e))), tproj = Lp(SiLU(temb)) split 6 ways in the
    order shift, scale, gate, c_shift, c_scale, c_gate.
R4  text MLP: L2(GELU_tanh(L1(c))).
R5  q/k RMSNorm over the whole model width (all heads), gain of length D, used
    in self- and cross-attention; RoPE after the norm, self-attention only.
R6  norm2 is an affine LayerNorm; norm1, norm3, norm_out carry no affine.
R7  RoPE: head-dim split t/h/w, pairs (2k, 2k+1) interleaved, angle
    pos * theta^(-2k/d_axis), rotation (x0 c - x1 s, x0 s + x1 c).
R8  attention scale 1/sqrt(head_dim), no mask, heads are contiguous slices.
R10 GELU is the tanh form.
R11 token order (f, i, j) row-major, j fastest.
R12 patch feature order (c, kt, kh, kw), c slowest (Conv3d weight flatten).
R13 proj_out feature order (kt, kh, kw, c), c fastest (unpatchify reshape).
R14 per-token timestep: t of shape [B, L]; every modulation row per token.
R19 I2V image embedder: the CLIP tokens [B, Li, 1280] pass an MLP to the model
    width, taken in the text embedder's form L2(GELU_tanh(L1(c))) with L1
    1280 -> D and L2 D -> D.
R20 I2V image cross-attention: the image tokens (placed before the text tokens
    in the model forward) are split off again in every block and attended
    separately: own key/value projections, keys RMSNorm'd across heads like the
    text keys, the queries of the text cross-attention; the two attention
    outputs are summed before the shared output projection.
R21 MoE expert switch: with t decreasing over sampling, steps with
    t >= boundary * num_train_timesteps use the high-noise expert and the rest
    the low-noise expert; both forwards of a CFG step use the same expert.
R22 flow shift: the pages give only the value (3.0 at 480p, 5.0 at 720p) and
    where it acts (the scheduler's timestep set-up); taken as the usual
    flow-matching time shift sigma' = s sigma / (1 + (s - 1) sigma), which
    multiplies the noise odds sigma / (1 - sigma) by s, applied to the uniform
    ladder sigma_i = 1 - i / steps (i = 0 .. steps - 1) with a final 0, and
    timesteps t_i = sigma_i * num_train_timesteps.

Parity unpinned (conventions the pages do not fix, so no pin can tell a
right reading from a wrong one; the oracle and the CUDA path simply agree):
the choice of cos-before-sin and the 1e4 base of the sinusoid (R2), the
activation inside the time MLP (R3), the interleaved-pair RoPE layout and its
44/42/42 split (R7), the form of the image MLP (R19) and the projections and
norm of the image branch (R20), and the init/gain conventions of the synthetic
weights.
Everything else is pinned by ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Sequence, Tuple

import torch

DT = torch.float64

# --------------------------------------------------------------------------
# Shapes: latent law and token law
# --------------------------------------------------------------------------


def latent_shape(batch: int, frames: int, height: int, width: int,
                 z_dim: int = 16, t_stride: int = 4, s_stride: int = 8):
    """Video [B,3,T,H,W] -> latent [B,z,1+(T-1)/4,H/8,W/8] with T = 4n+1.

    [WAN21-GUIDE] §3.1 (shape law); [PSWP-WAN] "Wan-VAE compresses time 4x and
    height/width 8x" with ``(num_frames-1)//4+1`` latent frames.
    """
    if frames < 1 or (frames - 1) % t_stride != 0:
        raise ValueError(f"frame count {frames} is not {t_stride}n+1")
    if height % s_stride or width % s_stride:
        raise ValueError("height and width must be multiples of the spatial stride")
    return (batch, z_dim, 1 + (frames - 1) // t_stride, height // s_stride, width // s_stride)


def token_count(F: int, Hz: int, Wz: int, patch=(1, 2, 2)) -> int:
    """L = F * Hz/2 * Wz/2 tokens for a (1,2,2) patch ([WAN21-GUIDE] §5.1)."""
    pt, ph, pw = patch
    if F % pt or Hz % ph or Wz % pw:
        raise ValueError("latent grid is not divisible by the patch")
    return (F // pt) * (Hz // ph) * (Wz // pw)


# --------------------------------------------------------------------------
# Patchify / unpatchify as explicit index maps
# --------------------------------------------------------------------------


def _grid(F, Hz, Wz, patch):
    pt, ph, pw = patch
    return F // pt, Hz // ph, Wz // pw


def patch_index_map(C: int, F: int, Hz: int, Wz: int, patch=(1, 2, 2)) -> torch.Tensor:
    """idx[l, k] = flat index into one sample's latent [C,F,Hz,Wz] of patch
    feature k of token l.

    Token l = (f*H' + i)*W' + j (R11, the ``flatten(2)`` of the Conv3d output in
    [PSWP-WAN] "WanTransformer3DModel"); feature k = ((c*pt + kt)*ph + kh)*pw + kw
    (R12, the flattening of the Conv3d weight [D, C, pt, ph, pw]).
    """
    pt, ph, pw = patch
    Fp, Hp, Wp = _grid(F, Hz, Wz, patch)
    f = torch.arange(Fp).view(Fp, 1, 1, 1, 1, 1, 1)
    i = torch.arange(Hp).view(1, Hp, 1, 1, 1, 1, 1)
    j = torch.arange(Wp).view(1, 1, Wp, 1, 1, 1, 1)
    c = torch.arange(C).view(1, 1, 1, C, 1, 1, 1)
    kt = torch.arange(pt).view(1, 1, 1, 1, pt, 1, 1)
    kh = torch.arange(ph).view(1, 1, 1, 1, 1, ph, 1)
    kw = torch.arange(pw).view(1, 1, 1, 1, 1, 1, pw)
    flat = ((c * F + (f * pt + kt)) * Hz + (i * ph + kh)) * Wz + (j * pw + kw)
    return flat.reshape(Fp * Hp * Wp, C * pt * ph * pw)


def unpatch_index_map(C: int, F: int, Hz: int, Wz: int, patch=(1, 2, 2)) -> torch.Tensor:
    """idx[l, k'] = flat index into one sample's velocity [C,F,Hz,Wz] written by
    proj_out feature k' of token l, with k' = ((kt*ph + kh)*pw + kw)*C + c (R13:
    the reshape to (..., pt, ph, pw, C) before the permute in [PSWP-WAN]
    "WanTransformer3DModel", step 5 "Output norm, projection & unpatchify").
    """
    pt, ph, pw = patch
    Fp, Hp, Wp = _grid(F, Hz, Wz, patch)
    f = torch.arange(Fp).view(Fp, 1, 1, 1, 1, 1, 1)
    i = torch.arange(Hp).view(1, Hp, 1, 1, 1, 1, 1)
    j = torch.arange(Wp).view(1, 1, Wp, 1, 1, 1, 1)
    kt = torch.arange(pt).view(1, 1, 1, pt, 1, 1, 1)
    kh = torch.arange(ph).view(1, 1, 1, 1, ph, 1, 1)
    kw = torch.arange(pw).view(1, 1, 1, 1, 1, pw, 1)
    c = torch.arange(C).view(1, 1, 1, 1, 1, 1, C)
    flat = ((c * F + (f * pt + kt)) * Hz + (i * ph + kh)) * Wz + (j * pw + kw)
    return flat.reshape(Fp * Hp * Wp, pt * ph * pw * C)


def patchify(latent: torch.Tensor, patch=(1, 2, 2)) -> torch.Tensor:
    """[B,C,F,Hz,Wz] -> [B, L, C*pt*ph*pw] patch vectors (the Conv3d input view)."""
    B, C, F, Hz, Wz = latent.shape
    idx = patch_index_map(C, F, Hz, Wz, patch)
    return latent.reshape(B, -1)[:, idx]


def unpatchify(out: torch.Tensor, C: int, F: int, Hz: int, Wz: int, patch=(1, 2, 2)) -> torch.Tensor:
    """[B, L, pt*ph*pw*C] proj_out rows -> [B, C, F, Hz, Wz] velocity."""
    B = out.shape[0]
    idx = unpatch_index_map(C, F, Hz, Wz, patch)
    vel = torch.zeros(B, C * F * Hz * Wz, dtype=out.dtype)
    vel[:, idx.reshape(-1)] = out.reshape(B, -1)
    return vel.reshape(B, C, F, Hz, Wz)


def patch_embed(latent: torch.Tensor, weight: torch.Tensor, bias: torch.Tensor, patch=(1, 2, 2)) -> torch.Tensor:
    """``patch_embedding`` = Conv3d(kernel = stride = patch) followed by
    ``flatten(2).transpose(1, 2)`` ([PSWP-WAN] "WanTransformer3DModel";
    [WAN21-GUIDE] §5.1): a gather into patch vectors and one matmul."""
    D = weight.shape[0]
    X = patchify(latent.to(DT), patch)
    return X @ weight.to(DT).reshape(D, -1).T + bias.to(DT)


# --------------------------------------------------------------------------
# Elementwise pieces
# --------------------------------------------------------------------------


def silu(x):
    return x / (1.0 + torch.exp(-x))


def gelu_tanh(x):
    """GELU, tanh form (R10)."""
    return 0.5 * x * (1.0 + torch.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x * x * x)))


def linear(x, w, b=None):
    y = x @ w.to(DT).T
    if b is not None:
        y = y + b.to(DT)
    return y


def layer_norm(x, eps, gamma=None, beta=None):
    """LayerNorm over the last axis with the biased variance; optional affine."""
    mu = x.mean(-1, keepdim=True)
    var = ((x - mu) ** 2).mean(-1, keepdim=True)
    y = (x - mu) / torch.sqrt(var + eps)
    if gamma is not None:
        y = y * gamma.to(DT)
    if beta is not None:
        y = y + beta.to(DT)
    return y


def rms_norm(x, eps, gamma=None):
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * gamma."""
    y = x / torch.sqrt((x * x).mean(-1, keepdim=True) + eps)
    if gamma is not None:
        y = y * gamma.to(DT)
    return y


# --------------------------------------------------------------------------
# Conditioning: timestep sinusoid, time MLP, text MLP
# --------------------------------------------------------------------------


def timestep_sinusoid(t: torch.Tensor, dim: int = 256, base: float = 10000.0) -> torch.Tensor:
    """freq_dim = 256 sinusoidal timestep features ([ANIMATE-DIFF] config table),
    in reading R2: [cos(t*w_k), sin(t*w_k)], w_k = base^(-k/(dim/2))."""
    half = dim // 2
    k = torch.arange(half, dtype=DT)
    omega = torch.exp(-math.log(base) * k / half)
    arg = t.to(DT)[..., None] * omega
    return torch.cat([torch.cos(arg), torch.sin(arg)], dim=-1)


def time_embedding(t: torch.Tensor, W: Dict[str, torch.Tensor], cfg) -> Tuple[torch.Tensor, torch.Tensor]:
    """``condition_embedder`` time path: temb [..., D] and timestep_proj
    [..., 6, D] ([PSWP-WAN] "WanTransformer3DModel": temb (1,1536), projection
    (1,9216) unflattened to (1,6,1536)); reading R3."""
    p = "condition_embedder."
    e = timestep_sinusoid(t, cfg["freq_dim"])
    h = silu(linear(e, W[p + "time_embedder.linear_1.weight"], W[p + "time_embedder.linear_1.bias"]))
    temb = linear(h, W[p + "time_embedder.linear_2.weight"], W[p + "time_embedder.linear_2.bias"])
    proj = linear(silu(temb), W[p + "time_proj.weight"], W[p + "time_proj.bias"])
    return temb, proj.reshape(*proj.shape[:-1], 6, cfg["dim"])


def text_embedding(context: torch.Tensor, W: Dict[str, torch.Tensor]) -> torch.Tensor:
    """``condition_embedder`` text path: [B, Lc, 4096] -> [B, Lc, D] (R4)."""
    p = "condition_embedder.text_embedder."
    h = gelu_tanh(linear(context.to(DT), W[p + "linear_1.weight"], W[p + "linear_1.bias"]))
    return linear(h, W[p + "linear_2.weight"], W[p + "linear_2.bias"])


def image_embedding(image: torch.Tensor, W: Dict[str, torch.Tensor]) -> torch.Tensor:
    """I2V ``condition_embedder`` image path: CLIP tokens [B, Li, 1280] -> [B, Li, D]
    ([WAN21-GUIDE] §4 "T5与CLIP": 257 CLIP tokens of width 1280 projected to the
    model width by an MLP; [ANIMATE-DIFF] "配置参数全解": image_dim 1280 for the
    CLIP features; [PSWP-WAN] "WanTransformer3DModel": the image tokens come out
    of the condition embedder next to the text tokens).  Reading R19."""
    p = "condition_embedder.image_embedder."
    h = gelu_tanh(linear(image.to(DT), W[p + "linear_1.weight"], W[p + "linear_1.bias"]))
    return linear(h, W[p + "linear_2.weight"], W[p + "linear_2.bias"])


def i2v_input(noisy: torch.Tensor, cond: torch.Tensor, mask: torch.Tensor) -> torch.Tensor:
    """DiT input of the I2V route: noisy latent (z channels), first-frame
    condition latent (z channels) and known-frame mask (4 channels) joined on the
    channel axis, not the time axis: 2 z + 4 channels, 36 for z = 16
    ([WAN21-GUIDE] §4 table "I2V分量"; [ANIMATE-DIFF] "配置参数全解":
    in_channels 36 = 2 * latent_channels + 4)."""
    if not (noisy.shape[2:] == cond.shape[2:] == mask.shape[2:]) or mask.shape[1] != 4:
        raise ValueError("noisy, cond, mask must share (B, F, H, W); mask has 4 channels")
    return torch.cat([noisy, cond, mask], dim=1)


# --------------------------------------------------------------------------
# 3-axis rotary position embedding
# --------------------------------------------------------------------------


def rope_angles(grid: Sequence[int], split: Sequence[int], theta: float) -> torch.Tensor:
    """Angles [L, head_dim/2] of the T/H/W rotary embedding ([ANIMATE-DIFF]:
    separate 1-D rotary frequencies per axis, concatenated; [PSWP-WAN] prints
    the rope tensor (1,1,32760,64) for 64 pairs per token).  Pair k of axis a
    (width d_a) at position pos turns by pos * theta^(-2k/d_a) (R7)."""
    Fp, Hp, Wp = grid
    parts = []
    for n, (d_a, size, view) in enumerate(zip(split, (Fp, Hp, Wp),
                                              ((Fp, 1, 1), (1, Hp, 1), (1, 1, Wp)))):
        k = torch.arange(d_a // 2, dtype=DT)
        freq = theta ** (-2.0 * k / d_a)
        pos = torch.arange(size, dtype=DT).view(*view, 1)
        parts.append((pos * freq).expand(Fp, Hp, Wp, d_a // 2))
    return torch.cat(parts, dim=-1).reshape(Fp * Hp * Wp, -1)


def rope_apply(x: torch.Tensor, angles: torch.Tensor) -> torch.Tensor:
    """Rotate interleaved pairs of x [..., L, heads, head_dim] by angles [L, head_dim/2]."""
    x0 = x[..., 0::2]
    x1 = x[..., 1::2]
    c = torch.cos(angles)[:, None, :]
    s = torch.sin(angles)[:, None, :]
    out = torch.empty_like(x)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


# --------------------------------------------------------------------------
# Attention
# --------------------------------------------------------------------------


def attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, chunk_elems: int = 1 << 25) -> torch.Tensor:
    """softmax(q k^T / sqrt(d)) v per (batch, head), no mask (R8).

    q [B, Lq, h, d], k/v [B, Lk, h, d] -> [B, Lq, h, d].  The row maximum is
    subtracted before exp (softmax is invariant to it); queries are processed in
    chunks only to bound memory."""
    B, Lq, h, d = q.shape
    Lk = k.shape[1]
    scale = 1.0 / math.sqrt(d)
    qh = q.permute(0, 2, 1, 3)
    kh = k.permute(0, 2, 1, 3)
    vh = v.permute(0, 2, 1, 3)
    out = torch.empty(B, h, Lq, d, dtype=DT)
    step = max(1, chunk_elems // max(1, B * h * Lk))
    for s0 in range(0, Lq, step):
        s = (qh[:, :, s0:s0 + step] @ kh.transpose(-1, -2)) * scale
        s = s - s.max(dim=-1, keepdim=True).values
        p = torch.exp(s)
        out[:, :, s0:s0 + step] = (p @ vh) / p.sum(dim=-1, keepdim=True)
    return out.permute(0, 2, 1, 3)


# --------------------------------------------------------------------------
# Transformer block and head
# --------------------------------------------------------------------------


def _heads(x, cfg):
    return x.reshape(*x.shape[:-1], cfg["heads"], cfg["head_dim"])


def self_attention_qkv(y, Wb, angles, cfg, rows=None):
    """q, k, v of ``attn1``: projections, RMSNorm across heads (R5), RoPE on q, k."""
    eps = cfg["eps"]
    yq = y if rows is None else y[:, rows]
    q = rms_norm(linear(yq, Wb["attn1.to_q.weight"], Wb["attn1.to_q.bias"]), eps, Wb["attn1.norm_q.weight"])
    k = rms_norm(linear(y, Wb["attn1.to_k.weight"], Wb["attn1.to_k.bias"]), eps, Wb["attn1.norm_k.weight"])
    v = linear(y, Wb["attn1.to_v.weight"], Wb["attn1.to_v.bias"])
    qa = angles if rows is None else angles[rows]
    q = rope_apply(_heads(q, cfg), qa)
    k = rope_apply(_heads(k, cfg), angles)
    return q, k, _heads(v, cfg)


def self_attention(y, Wb, angles, cfg, rows=None):
    q, k, v = self_attention_qkv(y, Wb, angles, cfg, rows)
    o = attention(q, k, v).reshape(q.shape[0], q.shape[1], -1)
    return linear(o, Wb["attn1.to_out.0.weight"], Wb["attn1.to_out.0.bias"])


def cross_attention(yc, ctx, Wb, cfg, img=None):
    """``attn2``: queries from the video tokens, keys/values from the projected
    text context ([WAN21-GUIDE] §5.2), q/k RMSNorm across heads (R5), no RoPE.
    With ``img`` (I2V, [B, Li, D] embedded image tokens) a second, separately
    normalised attention over the image tokens is added before the output
    projection ([WAN21-GUIDE] §4 table: the CLIP condition takes its own image
    cross-attention; [ANIMATE-DIFF] "配置参数全解": an added key/value projection,
    and its architecture section: image embeddings joined in front of the text
    embeddings; reading R20)."""
    eps = cfg["eps"]
    q = rms_norm(linear(yc, Wb["attn2.to_q.weight"], Wb["attn2.to_q.bias"]), eps, Wb["attn2.norm_q.weight"])
    k = rms_norm(linear(ctx, Wb["attn2.to_k.weight"], Wb["attn2.to_k.bias"]), eps, Wb["attn2.norm_k.weight"])
    v = linear(ctx, Wb["attn2.to_v.weight"], Wb["attn2.to_v.bias"])
    o = attention(_heads(q, cfg), _heads(k, cfg), _heads(v, cfg)).reshape(q.shape)
    if img is not None:
        ki = rms_norm(linear(img, Wb["attn2.add_k_proj.weight"], Wb["attn2.add_k_proj.bias"]), eps,
                      Wb["attn2.norm_added_k.weight"])
        vi = linear(img, Wb["attn2.add_v_proj.weight"], Wb["attn2.add_v_proj.bias"])
        o = o + attention(_heads(q, cfg), _heads(ki, cfg), _heads(vi, cfg)).reshape(q.shape)
    return linear(o, Wb["attn2.to_out.0.weight"], Wb["attn2.to_out.0.bias"])


def feed_forward(y, Wb):
    h = gelu_tanh(linear(y, Wb["ffn.net.0.proj.weight"], Wb["ffn.net.0.proj.bias"]))
    return linear(h, Wb["ffn.net.2.weight"], Wb["ffn.net.2.bias"])


def block_forward(x, ctx, mod, Wb, angles, cfg, rows=None, img=None):
    """One ``WanTransformerBlock`` ([PSWP-WAN] "WanTransformerBlock"; order also
    in [WAN21-GUIDE] §5.2).

    x [B, L, D]; ctx [B, Lc, D]; mod [B, 1 or L, 6, D] = block table + shared
    timestep projection, in the order shift, scale, gate, c_shift, c_scale,
    c_gate.  With ``rows`` (a LongTensor of token indices) only those tokens'
    outputs are computed; keys and values still use every token.  ``img``: the
    embedded image tokens of the I2V route (R20), or None.
    """
    eps = cfg["eps"]
    shift, scale, gate, c_shift, c_scale, c_gate = (mod[:, :, n] for n in range(6))

    def sel(m):  # modulation rows matching the selected tokens
        return m if (rows is None or m.shape[1] == 1) else m[:, rows]

    # 1. self-attention with adaLN modulation and gated residual
    y = layer_norm(x, eps) * (1.0 + scale) + shift
    xr = x if rows is None else x[:, rows]
    xr = xr + self_attention(y, Wb, angles, cfg, rows) * sel(gate)
    # 2. cross-attention after the affine norm2, plain residual
    yc = layer_norm(xr, eps, Wb["norm2.weight"], Wb["norm2.bias"])
    xr = xr + cross_attention(yc, ctx, Wb, cfg, img)
    # 3. feed-forward with modulation and gated residual
    y = layer_norm(xr, eps) * (1.0 + sel(c_scale)) + sel(c_shift)
    return xr + feed_forward(y, Wb) * sel(c_gate)


def head_forward(x, temb, W, cfg):
    """Output head: (shift, scale) = head table + temb, FP32 LayerNorm without
    affine, modulation, proj_out ([PSWP-WAN] "WanTransformer3DModel" step 5;
    [ANIMATE-DIFF] "norm_out FP32 LayerNorm + scale-shift, then proj_out")."""
    sst = W["scale_shift_table"].to(DT).reshape(2, cfg["dim"])
    t = temb if temb.dim() == 3 else temb[:, None, :]
    shift = sst[0] + t
    scale = sst[1] + t
    z = layer_norm(x, cfg["eps"]) * (1.0 + scale) + shift
    return linear(z, W["proj_out.weight"], W["proj_out.bias"])


def block_weights(W, i):
    p = f"blocks.{i}."
    return {k[len(p):]: v for k, v in W.items() if k.startswith(p)}


def forward(latent, timestep, context, W, cfg, return_blocks: bool = False, rows=None, image=None):
    """Velocity of one denoising step: patchify, conditioning, N blocks, head,
    unpatchify ([PSWP-WAN] "WanTransformer3DModel").

    latent [B, C, F, Hz, Wz]; timestep [B] (or [B, L] per token, R14); context
    [B, Lc, text_dim].  Returns the velocity [B, C_out, F, Hz, Wz] and, with
    ``return_blocks``, the residual stream after the patch embedding and after
    every block.  With ``rows`` (one-block models only) the proj_out rows of
    those tokens are returned instead of the velocity.  ``image`` (I2V): CLIP
    tokens [B, Li, image_dim]; the forward listing of [PSWP-WAN] concatenates
    the embedded image tokens before the text tokens and every block splits them
    off again for the image attention (R20), so they are carried separately here.
    """
    B, C, F, Hz, Wz = latent.shape
    patch = tuple(cfg["patch"])
    grid = _grid(F, Hz, Wz, patch)
    x = patch_embed(latent, W["patch_embedding.weight"], W["patch_embedding.bias"], patch)
    temb, tproj = time_embedding(timestep, W, cfg)
    if tproj.dim() == 3:           # per-sample timestep: [B, 6, D] -> [B, 1, 6, D]
        tproj = tproj[:, None]
    ctx = text_embedding(context, W)
    img = image_embedding(image, W) if image is not None else None
    angles = rope_angles(grid, cfg["rope_split"], cfg["rope_theta"])
    outs = [x] if return_blocks else None
    nb = cfg["num_blocks"]
    if rows is not None and nb != 1:
        raise ValueError("row sampling needs a one-block model")
    for i in range(nb):
        Wb = block_weights(W, i)
        mod = Wb["scale_shift_table"].to(DT).reshape(1, 1, 6, cfg["dim"]) + tproj
        x = block_forward(x, ctx, mod, Wb, angles, cfg, rows, img)
        if return_blocks:
            outs.append(x)
    if rows is not None:
        t_rows = temb if temb.dim() == 2 else temb[:, rows]
        return head_forward(x, t_rows, W, cfg)
    o = head_forward(x, temb, W, cfg)
    vel = unpatchify(o, cfg["out_ch"], F, Hz, Wz, patch)
    return (vel, outs) if return_blocks else vel


# --------------------------------------------------------------------------
# Architecture table (parameter names and shapes)
# --------------------------------------------------------------------------


def param_shapes(cfg) -> Dict[str, Tuple[int, ...]]:
    """Parameter names and shapes of the DiT, diffusers-style names as printed in
    [PSWP-WAN] (patch_embedding, condition_embedder, blocks.i.{norm2, attn1,
    attn2, ffn, scale_shift_table}, norm_out, proj_out, scale_shift_table)."""
    D, Fd, C, Co = cfg["dim"], cfg["ffn_dim"], cfg["in_ch"], cfg["out_ch"]
    pt, ph, pw = cfg["patch"]
    td, fd = cfg["text_dim"], cfg["freq_dim"]
    s = {
        "patch_embedding.weight": (D, C, pt, ph, pw), "patch_embedding.bias": (D,),
        "condition_embedder.time_embedder.linear_1.weight": (D, fd),
        "condition_embedder.time_embedder.linear_1.bias": (D,),
        "condition_embedder.time_embedder.linear_2.weight": (D, D),
        "condition_embedder.time_embedder.linear_2.bias": (D,),
        "condition_embedder.time_proj.weight": (6 * D, D), "condition_embedder.time_proj.bias": (6 * D,),
        "condition_embedder.text_embedder.linear_1.weight": (D, td),
        "condition_embedder.text_embedder.linear_1.bias": (D,),
        "condition_embedder.text_embedder.linear_2.weight": (D, D),
        "condition_embedder.text_embedder.linear_2.bias": (D,),
    }
    for i in range(cfg["num_blocks"]):
        p = f"blocks.{i}."
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
        if cfg.get("image_dim", 0):
            for n in ("add_k_proj", "add_v_proj"):
                s[p + f"attn2.{n}.weight"] = (D, D)
                s[p + f"attn2.{n}.bias"] = (D,)
            s[p + "attn2.norm_added_k.weight"] = (D,)
    if cfg.get("image_dim", 0):
        s["condition_embedder.image_embedder.linear_1.weight"] = (D, cfg["image_dim"])
        s["condition_embedder.image_embedder.linear_1.bias"] = (D,)
        s["condition_embedder.image_embedder.linear_2.weight"] = (D, D)
        s["condition_embedder.image_embedder.linear_2.bias"] = (D,)
    s["scale_shift_table"] = (1, 2, D)
    s["proj_out.weight"] = (Co * pt * ph * pw, D)
    s["proj_out.bias"] = (Co * pt * ph * pw,)
    return s


def param_count(cfg) -> int:
    return sum(math.prod(v) for v in param_shapes(cfg).values())


# --------------------------------------------------------------------------
# Sampler pieces around the forward (flow matching)
# --------------------------------------------------------------------------


def flow_interpolate(z, eps, sigma):
    """x_sigma = (1 - sigma) z + sigma eps ([WAN21-GUIDE] §6.1)."""
    return (1.0 - sigma) * z + sigma * eps


def flow_target(z, eps):
    """Target velocity v* = eps - z ([WAN21-GUIDE] §6.1)."""
    return eps - z


def cfg_combine(v_uncond, v_cond, scale):
    """Classifier-free guidance v_u + s (v_c - v_u) ([WAN21-GUIDE] §7)."""
    return v_uncond + scale * (v_cond - v_uncond)


def moe_expert(t: float, boundary: float, num_train_timesteps: int = 1000) -> int:
    """Wan2.2 A14B expert for a sampling step: 0 = high-noise expert when
    t >= boundary * num_train_timesteps, else 1 = low-noise expert.  One expert
    serves a whole timestep, both CFG forwards included, and the switch compares
    the scheduler's timestep value with boundary * num_train_timesteps
    ([WAN22-PITFALLS] "一次生成会经过什么,又会在哪一步悄悄失败"); noise goes to the
    high-noise expert first and to the low-noise one after the threshold
    ([WAN21-GUIDE] §10.1).  Reading R21."""
    return 0 if float(t) >= float(boundary) * num_train_timesteps else 1


def euler_step(x, sigma, sigma_next, v):
    """x_next = x + (sigma_next - sigma) v ([WAN21-GUIDE] §7)."""
    return x + (sigma_next - sigma) * v


def flow_shift(sigma, shift: float):
    """Shifted noise level s sigma / (1 + (s - 1) sigma) (reading R22).  The
    shift value is set per resolution in the pipeline set-up of [PSWP-WAN]
    (flow_shift 3.0 at 480p, 5.0 at 720p) and takes effect where the scheduler
    builds its timesteps ([WAN22-PITFALLS] "shift 参数生效了两次,在两个地方")."""
    sigma = torch.as_tensor(sigma, dtype=DT)
    return shift * sigma / (1.0 + (shift - 1.0) * sigma)


def sampling_sigmas(steps: int, shift: float) -> torch.Tensor:
    """Noise levels of a `steps`-step sampling run, steps + 1 values from 1 down
    to a final 0: the uniform ladder 1 - i / steps (i < steps) shifted by
    flow_shift, then 0 for the last Euler update to land on (R22; the Euler
    update of [WAN21-GUIDE] §7 walks sigma to sigma_next)."""
    if steps < 1:
        raise ValueError("steps must be >= 1")
    ladder = 1.0 - torch.arange(steps, dtype=DT) / steps
    return torch.cat([flow_shift(ladder, shift), torch.zeros(1, dtype=DT)])


def sampling_timesteps(steps: int, shift: float, num_train_timesteps: int = 1000) -> torch.Tensor:
    """Timestep values the DiT (and the expert switch) sees: sigma * num_train_timesteps
    for the first `steps` noise levels (R22)."""
    return sampling_sigmas(steps, shift)[:steps] * num_train_timesteps

"""Shared helpers of the GPU parity tests (CUDA library vs the float64 oracle)."""
import math

import pytest
import torch

from oracle import wan_oracle as O
from video_diffusion_transformer_dit_b200 import configs, synth

DT = torch.float64


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def rel_l2(a, b) -> float:
    a = a.to(DT).cpu()
    b = b.to(DT).cpu()
    return (torch.linalg.vector_norm(a - b) / torch.linalg.vector_norm(b)).item()


def to64(W):
    return {k: v.to(DT) for k, v in W.items()}


def bf16_round(x):
    return x.to(torch.bfloat16).to(torch.float32)


def workload_inputs(name, seed=0, num_blocks=None, device="cpu"):
    """Seeded weights and inputs of a named workload (optionally fewer blocks)."""
    w = configs.workload(name)
    cfg = dict(w["cfg"])
    if num_blocks is not None:
        cfg["num_blocks"] = num_blocks
    B, Cc, F, Hz, Wz = w["latent"]
    W = synth.make_weights(cfg, seed=seed)
    lat = synth.make_latent(w["latent"], seed=seed, same_across_batch=w.get("same_latent", False))
    ctx = synth.make_context(B, w["text_len"], cfg["text_dim"], seed=seed)
    if w["timesteps"] == "per_token":
        L = O.token_count(F, Hz, Wz)
        t = synth.make_timestep_per_token(B, L, (Hz // 2) * (Wz // 2), seed=seed)
    else:
        t = synth.make_timestep(B, w["timesteps"][0])
    return cfg, W, lat, t, ctx


def make_dit(cfg, B, L, Lc, W=None):
    from video_diffusion_transformer_dit_b200.binding import WanDiT
    dit = WanDiT(cfg, max_batch=B, max_tokens=L, max_text=Lc)
    if W is not None:
        dit.load_weights({k: v.cuda() for k, v in W.items()})
    return dit

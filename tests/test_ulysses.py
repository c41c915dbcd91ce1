"""Ulysses sequence parallelism: the orchestration against the one-rank forward.

The host-side orchestration (``video_diffusion_transformer_dit_b200.ulysses``:
sharding with explicit padding, the two all-to-alls per block, the final sum)
is driven here with ranks that compute through the float64 oracle, so the
exchange layouts, the padding and the global RoPE / timestep positions are
checked on CPU:
* in one process (``LocalExchange``) for world sizes 1, 2, 3 and 4, with L not
  a multiple of the world size (the case the pages' uneven chunking gets
  wrong), per-sample and per-token timesteps;
* as two gloo processes (``DistExchange`` over torch.distributed), world size 2.
The CUDA ranks (``SpRank``) run the same orchestration in
``tests/test_gpu_ulysses.py``.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

from oracle import wan_oracle as O
from video_diffusion_transformer_dit_b200 import ulysses as U

DT = torch.float64


def tiny_cfg():
    return dict(dim=48, heads=4, head_dim=12, ffn_dim=40, num_blocks=2, in_ch=4, out_ch=4, patch=(1, 2, 2),
                text_dim=16, freq_dim=8, eps=1e-6, rope_split=(4, 4, 4), rope_theta=10000.0)


def rand_weights(cfg, seed=0, scale=0.3):
    g = torch.Generator().manual_seed(seed)
    W = {}
    for n, s in O.param_shapes(cfg).items():
        W[n] = torch.randn(*s, generator=g, dtype=DT) * scale
        if ".norm_q." in n or ".norm_k." in n or n.endswith("norm2.weight"):
            W[n] = 1.0 + W[n]
    return W


def inputs(cfg, B=2, F=3, Hz=6, Wz=6, Lc=5, per_token=False, seed=1):
    g = torch.Generator().manual_seed(seed)
    lat = torch.randn(B, cfg["in_ch"], F, Hz, Wz, generator=g, dtype=DT)
    ctx = torch.randn(B, Lc, cfg["text_dim"], generator=g, dtype=DT)
    L = F * (Hz // 2) * (Wz // 2)
    t = torch.rand(B, L, generator=g, dtype=DT) * 1000 if per_token else torch.tensor([999.0, 20.0][:B], dtype=DT)
    return lat, t, ctx


class OracleSpRank:
    """A rank whose shard runs through the float64 oracle, with the buffer
    layouts of the CUDA ranks (send [B, world, Ls, 3 hd], recv [B, Lp, 3 hd],
    out [B, Lp, hd], back [B, world, Ls, hd])."""

    def __init__(self, W, cfg, rank, world):
        self.W, self.cfg, self.rank, self.world = W, cfg, rank, world
        self.hl = cfg["heads"] // world
        self.hd = self.hl * cfg["head_dim"]

    def _pad_slice(self, a, dim=1, fill_last=False):
        """Tokens [tok0, tok0 + Ls) of a [B, L, ...] tensor padded to Lp tokens."""
        pad_shape = list(a.shape)
        pad_shape[dim] = self.Lp - self.L
        pad = a.narrow(dim, self.L - 1, 1).expand(*pad_shape) if fill_last else a.new_zeros(pad_shape)
        return torch.cat([a, pad], dim=dim).narrow(dim, self.tok0, self.Ls)

    def begin(self, latent, timestep, context):
        cfg, W = self.cfg, self.W
        B, C, F, Hz, Wz = latent.shape
        self.B, self.F, self.Hz, self.Wz = B, F, Hz, Wz
        self.L = O.token_count(F, Hz, Wz)
        self.Ls, self.Lp = U.shard(self.L, self.world)
        self.tok0 = self.rank * self.Ls
        x = O.patch_embed(latent, W["patch_embedding.weight"], W["patch_embedding.bias"])
        self.x = self._pad_slice(x)
        temb, tproj = O.time_embedding(timestep, W, cfg)
        if timestep.dim() == 2:          # per token: this shard's rows (padding rows copy the last token)
            self.temb, self.tproj = self._pad_slice(temb, fill_last=True), self._pad_slice(tproj, fill_last=True)
        else:
            self.temb, self.tproj = temb, tproj[:, None]
        self.ctx = O.text_embedding(context, W)
        ang = O.rope_angles((F, Hz // 2, Wz // 2), cfg["rope_split"], cfg["rope_theta"])
        self.angles = self._pad_slice(ang[None], fill_last=True)[0]

    def _mod(self, i):
        Wb = O.block_weights(self.W, i)
        return Wb, Wb["scale_shift_table"].to(DT).reshape(1, 1, 6, self.cfg["dim"]) + self.tproj

    def block_qkv(self, i):
        Wb, mod = self._mod(i)
        y = O.layer_norm(self.x, self.cfg["eps"]) * (1.0 + mod[:, :, 1]) + mod[:, :, 0]
        q, k, v = O.self_attention_qkv(y, Wb, self.angles, self.cfg)       # [B, Ls, heads, head_dim]
        parts = []
        for j in range(self.world):
            hs = slice(j * self.hl, (j + 1) * self.hl)
            parts.append(torch.cat([t[:, :, hs].reshape(self.B, self.Ls, self.hd) for t in (q, k, v)], dim=-1))
        return torch.stack(parts, dim=1)                                     # [B, world, Ls, 3 hd]

    def attention(self, recv):
        B, Lp, hd, hl = self.B, self.Lp, self.hd, self.hl
        q = recv[..., :hd].reshape(B, Lp, hl, -1)
        k = recv[:, :self.L, hd:2 * hd].reshape(B, self.L, hl, -1)         # padding is never a key
        v = recv[:, :self.L, 2 * hd:].reshape(B, self.L, hl, -1)
        return O.attention(q, k, v).reshape(B, Lp, hd)

    def block_finish(self, i, back):
        cfg = self.cfg
        Wb, mod = self._mod(i)
        o = back.permute(0, 2, 1, 3).reshape(self.B, self.Ls, cfg["dim"])  # head group j -> its columns
        x = self.x + O.linear(o, Wb["attn1.to_out.0.weight"], Wb["attn1.to_out.0.bias"]) * mod[:, :, 2]
        yc = O.layer_norm(x, cfg["eps"], Wb["norm2.weight"], Wb["norm2.bias"])
        x = x + O.cross_attention(yc, self.ctx, Wb, cfg)
        y = O.layer_norm(x, cfg["eps"]) * (1.0 + mod[:, :, 4]) + mod[:, :, 3]
        self.x = x + O.feed_forward(y, Wb) * mod[:, :, 5]

    def end(self):
        out = O.head_forward(self.x, self.temb, self.W, self.cfg)           # [B, Ls, 4 C]
        rows = out.new_zeros(self.B, self.Lp, out.shape[-1])
        rows[:, self.tok0:self.tok0 + self.Ls] = out
        return O.unpatchify(rows[:, :self.L], self.cfg["out_ch"], self.F, self.Hz, self.Wz)


def test_shard_pads_to_equal_shards():
    for L, world in ((75, 2), (27, 4), (32760, 8), (27280, 3), (7, 7), (5, 8)):
        Ls, Lp = U.shard(L, world)
        assert Lp == world * Ls and Lp >= L and Lp - L < world
    with pytest.raises(ValueError):
        U.shard(10, 0)


@pytest.mark.parametrize("world", [1, 2, 3, 4])
@pytest.mark.parametrize("per_token", [False, True])
def test_orchestration_in_one_process_matches_one_rank(world, per_token):
    cfg = tiny_cfg()
    if cfg["heads"] % world:
        cfg = dict(cfg, heads=6, dim=72, head_dim=12, rope_split=(4, 4, 4))
    W = rand_weights(cfg, seed=world)
    lat, t, ctx = inputs(cfg, per_token=per_token, seed=10 + world)        # L = 27 tokens
    ranks = [OracleSpRank(W, cfg, r, world) for r in range(world)]
    vel = U.sp_forward(ranks, U.LocalExchange(), lat, t, ctx, cfg["num_blocks"])[0]
    ref = O.forward(lat, t, ctx, W, cfg)
    torch.testing.assert_close(vel, ref, rtol=1e-10, atol=1e-11)
    if world > 1:   # every rank contributes only its own tokens
        parts = [r.end() for r in ranks]
        assert all(p.abs().sum() > 0 for p in parts)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gloo_rank(rank, world, port, per_token):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = tiny_cfg()
        W = rand_weights(cfg, seed=7)
        lat, t, ctx = inputs(cfg, Hz=10, Wz=6, per_token=per_token, seed=8)   # L = 45 tokens, one padding row
        vel = U.sp_forward([OracleSpRank(W, cfg, rank, world)], U.DistExchange(), lat, t, ctx, cfg["num_blocks"])[0]
        ref = O.forward(lat, t, ctx, W, cfg)
        torch.testing.assert_close(vel, ref, rtol=1e-10, atol=1e-11)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("per_token", [False, True])
def test_orchestration_over_gloo_world_2(per_token):
    mp.spawn(_gloo_rank, args=(2, _free_port(), per_token), nprocs=2, join=True)


def test_sp_rank_needs_heads_divisible_by_world():
    class FakeDit:
        cfg = dict(heads=12)
    with pytest.raises(ValueError):
        U.SpRank(FakeDit(), 0, 5)
    assert U.SpRank(FakeDit(), 1, 4).hd == 128 * 3

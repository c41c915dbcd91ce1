"""Ulysses sequence parallelism of the Wan DiT forward: host-side orchestration.

The pages describe it as two exchanges around every self-attention ("读完 Wan2.2
全部源码之后", section "显存和算力怎么分"): q, k and v are scattered along the
heads and gathered along the sequence by an all-to-all, each rank runs the
attention over the whole sequence for its share of the heads, and a second
all-to-all brings the outputs back to the ranks that own the tokens.  Every
other step of the forward is token-local and runs on the rank's shard.

The same pages name the failure of the reference split: ``torch.chunk`` makes
the last chunk shorter when L is not a multiple of the world size and the
per-rank RoPE frequencies then no longer match the tokens.  Here the sequence is
padded to ``world * Ls`` tokens (``shard``), every shard has Ls rows, padding
sits past the last real token, is never a key (the attention masks keys >= L)
and is dropped at the end; RoPE and per-token timesteps use global positions.

Roles:
* ``SpRank`` drives one rank's shard through the CUDA library's
  ``wan_dit_sp_*`` stages (argument marshalling only: the kernels do the work,
  torch allocates the exchange buffers);
* an exchange moves the buffers between ranks: ``DistExchange`` with
  ``torch.distributed`` (one rank per process: NCCL on GPUs, gloo on CPU),
  ``LocalExchange`` for several ranks driven from one process;
* ``sp_forward`` runs the stage sequence for a list of ranks in lockstep.

Any object with the ``SpRank`` methods can stand in for a rank (the tests drive
the float64 oracle through the same orchestration).
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

from . import binding as _b


def shard(L: int, world: int) -> Tuple[int, int]:
    """Tokens per shard Ls = ceil(L / world) and the padded length Lp = world * Ls."""
    if world < 1 or L < 1:
        raise ValueError("L and world must be positive")
    Ls = -(-L // world)
    return Ls, Ls * world


class SpRank:
    """One rank of a sequence-parallel forward on the CUDA library.

    Buffers (bf16 on the handle's device, hd = 128 * heads / world):
    send [B, world, Ls, 3 hd], out [B, Lp, hd]; the exchange supplies recv
    [B, Lp, 3 hd] and back [B, world, Ls, hd]."""

    def __init__(self, dit: "_b.WanDiT", rank: int, world: int):
        cfg = dit.cfg
        if cfg["heads"] % world:
            raise ValueError(f"heads ({cfg['heads']}) must be a multiple of the world size ({world})")
        self.dit, self.rank, self.world = dit, rank, world
        self.hd = 128 * cfg["heads"] // world

    def begin(self, latent, timestep, context, stream=None):
        import torch
        B, _, F, Hz, Wz = latent.shape
        self.B, self.shape = B, latent.shape
        self.L = F * (Hz // 2) * (Wz // 2)
        self.Ls, self.Lp = shard(self.L, self.world)
        dev = latent.device if latent.is_cuda else torch.device("cuda", torch.cuda.current_device())
        bf = torch.bfloat16
        self.send = torch.empty(B, self.world, self.Ls, 3 * self.hd, dtype=bf, device=dev)
        self.out = torch.empty(B, self.Lp, self.hd, dtype=bf, device=dev)
        self.vel = torch.empty(B, self.dit.cfg["out_ch"], F, Hz, Wz, device=dev)
        per_token = int(timestep.dim() == 2)
        self.dit._check(_b.lib().wan_dit_sp_begin(
            self.dit._h, _b._ptr(latent), _b._dtype_code(latent), B, F, Hz, Wz, _b._ptr(timestep), per_token,
            _b._ptr(context), context.shape[1], self.rank, self.world, int(latent.is_cuda), _b._stream(stream)))

    def block_qkv(self, i: int, stream=None):
        self.dit._check(_b.lib().wan_dit_sp_block_qkv(self.dit._h, i, _b._ptr(self.send), _b._stream(stream)))
        return self.send

    def attention(self, recv, stream=None):
        self.dit._check(_b.lib().wan_dit_sp_attention(self.dit._h, _b._ptr(recv), _b._ptr(self.out),
                                                      _b._stream(stream)))
        return self.out

    def block_finish(self, i: int, back, stream=None):
        self.dit._check(_b.lib().wan_dit_sp_block_finish(self.dit._h, i, _b._ptr(back), _b._stream(stream)))

    def end(self, stream=None):
        self.dit._check(_b.lib().wan_dit_sp_end(self.dit._h, _b._ptr(self.vel), 1, _b._stream(stream)))
        return self.vel


class LocalExchange:
    """Exchange for ranks driven from one process: rank r's receive slot j is
    rank j's send slot r (per sample), and the velocity reduction is a sum."""

    def all_to_all(self, sends: Sequence) -> List:
        world = len(sends)
        recvs = []
        for r in range(world):
            B, _, Ls, w = sends[r].shape
            recv = sends[r].new_empty(B, world, Ls, w)
            for j in range(world):
                recv[:, j].copy_(sends[j][:, r])
            recvs.append(recv.view(B, world * Ls, w))
        return recvs

    def all_reduce(self, tensors: Sequence) -> List:
        total = tensors[0].clone()
        for t in tensors[1:]:
            total += t.to(total.device)
        return [total for _ in tensors]


class DistExchange:
    """Exchange over torch.distributed, one rank per process (NCCL on GPUs,
    gloo on CPU): one all_to_all_single per sample and direction, so each
    peer's part is one contiguous slot of the send buffer."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group

    def all_to_all(self, sends: Sequence) -> List:
        (send,) = sends
        B, world, Ls, w = send.shape
        recv = send.new_empty(B, world, Ls, w)
        for b in range(B):
            self.dist.all_to_all_single(recv[b], send[b].contiguous(), group=self.group)
        return [recv.view(B, world * Ls, w)]

    def all_reduce(self, tensors: Sequence) -> List:
        (v,) = tensors
        self.dist.all_reduce(v, group=self.group)
        return [v]


def sp_forward(ranks: Sequence, exchange, latent, timestep, context, num_blocks: int):
    """Velocity of one denoising step with the sequence split across `ranks`
    (all of them, or this process's one), in lockstep: per block the q/k/v
    exchange, attention over the whole sequence, the exchange back; then the
    per-rank velocities (each holding its own tokens) summed."""
    for r in ranks:
        r.begin(latent, timestep, context)
    for i in range(num_blocks):
        recvs = exchange.all_to_all([r.block_qkv(i) for r in ranks])
        outs = [r.attention(x) for r, x in zip(ranks, recvs)]
        backs = exchange.all_to_all([o.view(o.shape[0], r.world, r.Ls, o.shape[-1]) for r, o in zip(ranks, outs)])
        for r, x in zip(ranks, backs):
            r.block_finish(i, x.view(x.shape[0], r.world, r.Ls, x.shape[-1]))
    return exchange.all_reduce([r.end() for r in ranks])


__all__ = ["shard", "SpRank", "LocalExchange", "DistExchange", "sp_forward"]

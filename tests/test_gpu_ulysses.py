"""Ulysses sequence parallelism on the CUDA library (one GPU).

Each rank is its own wan_dit handle driven through the wan_dit_sp_* stages by
the same orchestration as the CPU tests; the ranks share the one GPU and the
exchange copies their buffers in stream order (``LocalExchange``: no kernel of
one rank waits on another's), so world sizes 2 and 4 run here.  The summed
velocity is compared with the one-rank wan_dit_forward and with the float64
oracle.  L = 189 tokens is not a multiple of either world size (one and three
padding tokens).  Across GPUs the exchange is NCCL's all_to_all_single
(``DistExchange``), which this pool's one-GPU machines cannot measure.
"""
import pytest
import torch

from oracle import wan_oracle as O
from tests.gpu_common import DT, make_dit, need_gpu, rel_l2, to64

pytestmark = pytest.mark.gpu

TOL = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def _case(per_token, seed):
    from video_diffusion_transformer_dit_b200 import configs, synth
    cfg = configs.model_config("wan2.1-1.3b", num_blocks=2)
    shape = (2, 16, 3, 14, 18)
    L = O.token_count(*shape[2:])
    W = synth.make_weights(cfg, seed=seed)
    lat = synth.make_latent(shape, seed=seed)
    ctx = synth.make_context(2, 24, cfg["text_dim"], seed=seed)
    t = synth.make_timestep_per_token(2, L, 7 * 9, seed=seed) if per_token else torch.tensor([999.0, 500.0])
    return cfg, W, lat, t, ctx, L


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("per_token", [False, True])
def test_sequence_parallel_matches_one_rank_and_oracle(world, per_token):
    from video_diffusion_transformer_dit_b200 import ulysses as U
    cfg, W, lat, t, ctx, L = _case(per_token, seed=20 + world)
    Ls, Lp = U.shard(L, world)
    assert Lp > L
    Wd = {k: v.cuda() for k, v in W.items()}
    ranks = [U.SpRank(make_dit(cfg, 2, Ls, ctx.shape[1], Wd), r, world) for r in range(world)]
    vel = U.sp_forward(ranks, U.LocalExchange(), lat.cuda(), t.cuda(), ctx.cuda(), cfg["num_blocks"])[0]
    torch.cuda.synchronize()
    for r in ranks:
        r.dit.sync()
    one = make_dit(cfg, 2, L, ctx.shape[1], Wd)
    ref_gpu = one.forward(lat.cuda(), t.cuda(), ctx.cuda(), sync=True)
    err_gpu = rel_l2(vel, ref_gpu)
    ref = O.forward(lat.to(DT), t.to(DT), ctx.to(DT), to64(W), cfg)
    err = rel_l2(vel, ref)
    print(f"\n[Ulysses world {world}, per_token {per_token}] vs one rank {err_gpu:.2e}, vs oracle {err:.2e}")
    assert err_gpu < 1e-2
    assert err < TOL
    # a second forward through the same handles gives the same bits
    vel2 = U.sp_forward(ranks, U.LocalExchange(), lat.cuda(), t.cuda(), ctx.cuda(), cfg["num_blocks"])[0]
    assert torch.equal(vel, vel2)


def test_sequence_parallel_stage_order_is_checked():
    from video_diffusion_transformer_dit_b200 import ulysses as U
    from video_diffusion_transformer_dit_b200.binding import WanError
    cfg, W, lat, t, ctx, L = _case(False, seed=30)
    Ls, _ = U.shard(L, 2)
    r = U.SpRank(make_dit(cfg, 2, Ls, ctx.shape[1], {k: v.cuda() for k, v in W.items()}), 0, 2)
    r.send = torch.empty(2, 2, Ls, 3 * r.hd, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(WanError) as e:          # a block before sp_begin
        r.block_qkv(0)
    assert e.value.name == "WAN_EINVAL"
    r.begin(lat.cuda(), t.cuda(), ctx.cuda())
    with pytest.raises(WanError):               # blocks must come in order
        r.block_qkv(1)
    with pytest.raises(WanError):               # the head before the blocks
        r.end()
    small = make_dit(cfg, 2, Ls - 1, ctx.shape[1], {k: v.cuda() for k, v in W.items()})
    with pytest.raises(WanError) as e:          # shard larger than the workspace
        U.SpRank(small, 0, 2).begin(lat.cuda(), t.cuda(), ctx.cuda())
    assert e.value.name == "WAN_ESHAPE"

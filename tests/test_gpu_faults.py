"""Failure detection on the GPU without a GPU fault.

Every on-chip wait of the tcgen05 kernels has a time limit; when it runs out
the CTA records WAN_ETIMEOUT in a device word, drains its own copies, frees its
tensor memory and returns, so the context stays usable.  These tests make waits
run out on purpose -- a barrier nothing arrives on, and a forward whose wait
limit is zero -- then check the reported status and that the next forward with
the normal limit reproduces the reference output bit for bit.
"""
import pytest
import torch

from oracle import wan_oracle as O
from tests.gpu_common import make_dit, need_gpu, workload_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def test_wait_selftest_times_out_and_context_survives():
    from video_diffusion_transformer_dit_b200 import binding as Bd
    Bd.op_sync()
    Bd.op_wait_selftest(200_000)                       # 0.2 ms on a barrier nothing arrives on
    with pytest.raises(Bd.WanError) as e:
        Bd.op_sync()
    assert e.value.name == "WAN_ETIMEOUT"
    Bd.op_sync()                                       # flag cleared, context fine
    x = torch.ones(1024, device="cuda")
    out = torch.empty_like(x)
    Bd.op_cfg_euler(x, x, None, 1.0, 1.0, 0.5, out)
    Bd.op_sync()
    assert torch.equal(out.cpu(), torch.full((1024,), 0.5))


def test_forward_with_zero_wait_limit_reports_and_recovers():
    from video_diffusion_transformer_dit_b200.binding import WAN_OPT_WAIT_LIMIT_NS, WanError
    cfg, W, lat, t, ctx = workload_inputs("wan1.3b-1blk-3x16x16", seed=4)
    L, Lc = O.token_count(*lat.shape[2:]), ctx.shape[1]
    dit = make_dit(cfg, 1, L, Lc, W)
    ref = dit.forward(lat.cuda(), t.cuda(), ctx.cuda(), sync=True).cpu()
    # a limit of 0 gives up at the first probe that finds a barrier still open;
    # every forward has such waits (each TMA load takes time to land)
    dit.set_option(WAN_OPT_WAIT_LIMIT_NS, 0)
    seen = []
    for _ in range(3):
        dit.forward(lat.cuda(), t.cuda(), ctx.cuda())
        try:
            dit.sync()
            seen.append("WAN_OK")
        except WanError as e:
            seen.append(e.name)
    assert "WAN_ETIMEOUT" in seen, seen
    assert set(seen) <= {"WAN_ETIMEOUT", "WAN_OK"}, seen
    dit.set_option(WAN_OPT_WAIT_LIMIT_NS, 2_000_000_000)
    again = dit.forward(lat.cuda(), t.cuda(), ctx.cuda(), sync=True).cpu()
    assert torch.equal(again, ref)

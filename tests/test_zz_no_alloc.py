"""The allocation-free RMSNorm + RoPE entry point against the allocating one.

wan_op_rmsnorm_rope_noalloc serves callers that cannot allocate device memory
while they run (their own pool allocator owns HBM, or they cannot take the
synchronisation an allocation may cause).  It keeps its cos/sin table in a
fixed device array; this test calls it through the C ABI twice in a row, on
two different grids, and checks each result against wan_op_rmsnorm_rope on
the same input with the tolerance of the other kernel tests, checks one grid
against the float64 oracle directly, then checks that bad widths and strides
and a grid beyond the array's 1024 positions per axis are refused.  The file name
makes pytest collect it last.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu

TOL = 1e-2


def _rel_l2(a, b):
    a, b = a.double().cpu(), b.double().cpu()
    return (torch.linalg.vector_norm(a - b) / torch.linalg.vector_norm(b)).item()


@pytest.fixture(scope="module")
def B():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from video_diffusion_transformer_dit_b200 import binding
    binding.lib()
    return binding


def test_noalloc_matches_allocating_op_twice(B):
    D = 1536
    gain = (1 + 0.1 * torch.randn(D, generator=torch.Generator().manual_seed(1))).cuda()
    for call, (grid, batch) in enumerate((((3, 5, 7), 2), ((21, 30, 52), 1))):
        L = grid[0] * grid[1] * grid[2]
        x = torch.randn(batch * L, 3 * D, generator=torch.Generator().manual_seed(10 + call)).to(torch.bfloat16)
        ref = x.cuda()
        got = x.cuda()
        B.op_rmsnorm_rope(ref.data_ptr() + 2 * D, 3 * D, batch * L, D, 1e-6, gain, rope=True, grid=grid)
        B.op_rmsnorm_rope_noalloc(got.data_ptr() + 2 * D, 3 * D, batch * L, D, 1e-6, gain, rope=True, grid=grid)
        torch.cuda.synchronize()
        err = _rel_l2(got[:, D:2 * D], ref[:, D:2 * D])
        assert err < TOL, f"call {call}: rel-L2 {err}"
        assert torch.equal(got[:, :D].cpu(), x[:, :D]) and torch.equal(got[:, 2 * D:].cpu(), x[:, 2 * D:])


def test_noalloc_matches_oracle(B):
    """The fixed-array table path against the float64 oracle's RMSNorm across
    heads and 3-axis rotation directly (not only against the other CUDA op)."""
    from oracle import wan_oracle as O
    Fp, Hp, Wp = 3, 5, 7
    L, D = Fp * Hp * Wp, 1536
    x = torch.randn(2 * L, D, generator=torch.Generator().manual_seed(30)).to(torch.bfloat16)
    gain = 1 + 0.1 * torch.randn(D, generator=torch.Generator().manual_seed(31))
    got = x.cuda()
    B.op_rmsnorm_rope_noalloc(got.data_ptr(), D, 2 * L, D, 1e-6, gain.cuda(), rope=True, grid=(Fp, Hp, Wp))
    torch.cuda.synchronize()
    ref = O.rms_norm(x.double(), 1e-6, gain.double())
    ref = O.rope_apply(ref.reshape(2, L, 12, 128), O.rope_angles((Fp, Hp, Wp), (44, 42, 42), 10000.0))
    assert _rel_l2(got, ref.reshape(2 * L, D)) < TOL


def test_noalloc_rejects_bad_shapes_before_launch(B):
    D = 1536
    buf = torch.zeros(4, D, dtype=torch.bfloat16, device="cuda")
    gain = torch.ones(D, device="cuda")
    for args in ((D + 8, D), (D, D + 4), (D, D // 2)):       # width not a kernel width, odd stride, stride < D
        with pytest.raises(B.WanError) as e:
            B.op_rmsnorm_rope_noalloc(buf.data_ptr(), args[1], 4, args[0], 1e-6, gain, rope=True, grid=(1, 2, 2))
        assert e.value.name == "WAN_ESHAPE"


def test_noalloc_rejects_grid_beyond_table(B):
    D = 1536
    buf = torch.zeros(4, D, dtype=torch.bfloat16, device="cuda")
    gain = torch.ones(D, device="cuda")
    with pytest.raises(B.WanError) as e:
        B.op_rmsnorm_rope_noalloc(buf.data_ptr(), D, 4, D, 1e-6, gain, rope=True, grid=(1025, 1, 1))
    assert e.value.name == "WAN_ESHAPE"

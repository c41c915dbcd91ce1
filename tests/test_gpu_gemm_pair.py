"""The SM-pair GEMM (tcgen05 .cta_group::2, 256 x 256 tiles on clusters of two
CTAs) against the float64 oracle and against the single-SM GEMM.

The pair path takes GEMMs with N a multiple of 256 and M >= 512 and the bias,
GELU, gate * residual, residual and q/k-norm epilogues.  Shapes cover one K
step (K = 64) and 24 (K = 1536), ragged M where the odd CTA of the last pair
tile holds some valid rows (M = 1000) or none (M = 868: rows 896..1023 all past
the end), and the wide N of the QKV (4608) and FFN-up (8960) projections.
Every tile's accumulation runs over the same K slices in the same order on both
paths, so the two agree to fp32 rounding of the epilogue arithmetic.
"""
import pytest
import torch

from oracle import wan_oracle as O
from tests.gpu_common import DT, make_dit, need_gpu, rel_l2, workload_inputs

pytestmark = pytest.mark.gpu

TOL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()
    from video_diffusion_transformer_dit_b200 import binding
    binding.lib()
    yield
    binding.op_set_gemm_pair(True)
    binding.op_set_wait_limit_ns(2_000_000_000)


def B():
    from video_diffusion_transformer_dit_b200 import binding
    return binding


def _inputs(M, N, K, seed):
    g = torch.Generator().manual_seed(seed)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    W = (torch.randn(N, K, generator=g) * 0.05).to(torch.bfloat16)
    bias = torch.randn(N, generator=g)
    x = torch.randn(M, N, generator=g).to(torch.bfloat16)
    gates = torch.randn(2, N, generator=g) * 0.1
    return A, W, bias, x, gates


def _run(pair, epi, A, W, bias, x, gates, M, L):
    B().op_set_gemm_pair(pair)
    try:
        if epi in ("gate_residual", "residual"):
            out = x.cuda()
        else:
            out = torch.full((M, W.shape[0]), float("nan"), dtype=torch.bfloat16, device="cuda")
        kw = {}
        if epi == "gate_residual":
            kw = dict(gate1=gates.contiguous().cuda(), mod_div=L, mod_ld=W.shape[0])
        B().op_gemm(A.cuda(), W.cuda(), epi, out, bias=bias.cuda(), **kw)
        B().op_sync()
    finally:
        B().op_set_gemm_pair(True)
    return out.cpu()


def test_pair_clusters_available():
    n = B().op_gemm_pair_clusters()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    print(f"\n[SM-pair GEMM] {n} clusters of 2 on {sms} SMs")
    assert 0 < n <= sms // 2


@pytest.mark.parametrize("epi", ["bias", "bias_gelu", "gate_residual", "residual"])
@pytest.mark.parametrize("M,N,K", [(1000, 256, 64), (868, 1536, 1536), (2048, 4608, 1536), (600, 8960, 256)])
def test_pair_gemm_matches_oracle_and_single_sm(epi, M, N, K):
    A, W, bias, x, gates = _inputs(M, N, K, seed=M + N + K)
    L = (M + 1) // 2                          # two samples for the per-sample gate
    got = _run(True, epi, A, W, bias, x, gates, M, L)
    one = _run(False, epi, A, W, bias, x, gates, M, L)
    assert not torch.isnan(got.float()).any()
    lin = O.linear(A.to(DT), W.to(DT), bias.to(DT))
    if epi == "bias":
        ref = lin
    elif epi == "bias_gelu":
        ref = O.gelu_tanh(lin)
    elif epi == "residual":
        ref = x.to(DT) + lin
    else:
        gate = torch.cat([gates[0:1].to(DT).expand(L, N), gates[1:2].to(DT).expand(M - L, N)])
        ref = x.to(DT) + lin * gate
    err, err_one = rel_l2(got, ref), rel_l2(got, one)
    print(f"\n[pair {epi} {M}x{N}x{K}] vs oracle {err:.2e}, vs single-SM {err_one:.2e}, "
          f"identical {torch.equal(got, one)}")
    assert err < TOL
    assert err_one < 2e-3


@pytest.mark.parametrize("rope", [True, False])
def test_pair_qk_norm_epilogue(rope):
    """QKV projection with the q/k norm epilogue on SM pairs: B = 2 samples of
    L = 4*8*10 = 320 tokens (R = 640 rows, the last pair tile ragged), sums of
    squares and stored q/k/v against the oracle and the single-SM kernel."""
    Fp, Hp, Wp = 4, 8, 10
    L, Bn, D, h = Fp * Hp * Wp, 2, 1536, 12
    R = Bn * L
    g = torch.Generator().manual_seed(41)
    y = torch.randn(R, D, generator=g).to(torch.bfloat16)
    W = (0.02 * torch.randn(3 * D, D, generator=g)).to(torch.bfloat16)
    bias = 0.02 * torch.randn(3 * D, generator=g)
    gain = 1 + 0.1 * torch.randn(2 * D, generator=g)
    outs = {}
    for pair in (True, False):
        B().op_set_gemm_pair(pair)
        try:
            qkv = torch.full((R, 3 * D), float("nan"), dtype=torch.bfloat16, device="cuda")
            ssq = torch.full((R, 2 * h), float("nan"), device="cuda")
            B().op_gemm(y.cuda(), W.cuda(), "qk_norm", qkv, bias=bias.cuda(), gain=gain.cuda(), ssq=ssq,
                        norm_cols=2 * D, rope_grid=(Fp, Hp, Wp) if rope else None)
            B().op_sync()
        finally:
            B().op_set_gemm_pair(True)
        outs[pair] = (qkv.cpu(), ssq.cpu())
    lin = O.linear(y.to(DT), W.to(DT), bias.to(DT))
    ref_ssq = (lin[:, :2 * D] ** 2).reshape(R, 2 * h, 128).sum(-1)
    ang = O.rope_angles((Fp, Hp, Wp), (44, 42, 42), 10000.0)

    def rot(t):
        return O.rope_apply(t.reshape(Bn, L, h, 128), ang).reshape(R, D) if rope else t
    qkv, ssq = outs[True]
    assert rel_l2(ssq, ref_ssq) < 1e-4
    assert rel_l2(qkv[:, :D], rot(lin[:, :D] * gain[:D].to(DT))) < TOL
    assert rel_l2(qkv[:, D:2 * D], rot(lin[:, D:2 * D] * gain[D:].to(DT))) < TOL
    assert rel_l2(qkv[:, 2 * D:], lin[:, 2 * D:]) < TOL
    assert rel_l2(qkv, outs[False][0]) < 2e-3
    assert rel_l2(ssq, outs[False][1]) < 1e-5


def test_pair_gemm_zero_wait_limit_reports_and_recovers():
    """Waits that give up at the first open barrier, in both CTAs of every pair:
    the op reports WAN_ETIMEOUT (or finishes), and the next GEMM with the normal
    limit gives the reference bits."""
    M, N, K = 2048, 1536, 1536
    A, W, bias, x, gates = _inputs(M, N, K, seed=9)
    ref = _run(True, "bias", A, W, bias, x, gates, M, M)
    seen = []
    B().op_set_wait_limit_ns(0)
    try:
        for _ in range(3):
            out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
            B().op_gemm(A.cuda(), W.cuda(), "bias", out, bias=bias.cuda())
            try:
                B().op_sync()
                seen.append("WAN_OK")
            except B().WanError as e:
                seen.append(e.name)
    finally:
        B().op_set_wait_limit_ns(2_000_000_000)
    assert "WAN_ETIMEOUT" in seen, seen
    assert set(seen) <= {"WAN_ETIMEOUT", "WAN_OK"}, seen
    again = _run(True, "bias", A, W, bias, x, gates, M, M)
    assert torch.equal(again, ref)


def test_forward_pair_and_single_sm_gemms_agree():
    """A 2-block Wan-1.3B forward (B = 2, L = 9*12*12 = 1296 tokens, so every
    block GEMM has M = 2592) with the pair GEMMs and with single-SM GEMMs, both
    against the float64 oracle."""
    from video_diffusion_transformer_dit_b200.binding import WAN_OPT_GEMM_PAIR
    from video_diffusion_transformer_dit_b200 import configs, synth
    cfg = configs.model_config("wan2.1-1.3b", num_blocks=2)
    shape = (2, 16, 9, 24, 24)
    L = O.token_count(*shape[2:])
    W = synth.make_weights(cfg, seed=12)
    lat = synth.make_latent(shape, seed=12)
    ctx = synth.make_context(2, 40, cfg["text_dim"], seed=12)
    t = torch.tensor([900.0, 250.0])
    dit = make_dit(cfg, 2, L, 40, W)
    v_pair = dit.forward(lat.cuda(), t.cuda(), ctx.cuda(), sync=True).cpu()
    dit.set_option(WAN_OPT_GEMM_PAIR, 0)
    v_one = dit.forward(lat.cuda(), t.cuda(), ctx.cuda(), sync=True).cpu()
    dit.set_option(WAN_OPT_GEMM_PAIR, 1)
    v_again = dit.forward(lat.cuda(), t.cuda(), ctx.cuda(), sync=True).cpu()
    ref = O.forward(lat.to(DT), t.to(DT), ctx.to(DT), {k: v.to(DT) for k, v in W.items()}, cfg)
    e_pair, e_one = rel_l2(v_pair, ref), rel_l2(v_one, ref)
    print(f"\n[forward 2 blocks, L {L}] pair vs oracle {e_pair:.2e}, single-SM vs oracle {e_one:.2e}, "
          f"pair vs single {rel_l2(v_pair, v_one):.2e}")
    assert e_pair < 2e-2 and e_one < 2e-2
    assert torch.equal(v_again, v_pair)

"""Kernel-level parity: each CUDA kernel through the C ABI against the oracle.

Index maps (patchify / unpatchify) must match bit for bit; floating-point
kernels are compared by relative L2 error against float64 (bf16 storage with
fp32 accumulation: 1e-2 bounds a few bf16 roundings, 2^-9 each).
"""
import math

import pytest
import torch

from oracle import wan_oracle as O
from oracle import wan_vae as V
from tests.gpu_common import DT, bf16_round, need_gpu, rel_l2

pytestmark = pytest.mark.gpu

TOL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()
    from video_diffusion_transformer_dit_b200 import binding
    binding.lib()


def B():
    from video_diffusion_transformer_dit_b200 import binding
    return binding


# ------------------------------------------------------------------ index maps
@pytest.mark.parametrize("shape", [(1, 16, 3, 16, 16), (2, 16, 9, 44, 80), (1, 48, 2, 10, 6)])
def test_patchify_bit_exact(shape):
    lat = bf16_round(torch.randn(*shape))
    X = torch.empty(shape[0] * O.token_count(*shape[2:]), shape[1] * 4, dtype=torch.bfloat16, device="cuda")
    B().op_patchify(lat.cuda(), X)
    B().op_sync()
    ref = O.patchify(lat.to(DT)).reshape(X.shape)
    assert torch.equal(X.cpu().to(DT), ref)


def test_patchify_bf16_latent_bit_exact():
    lat = torch.randn(2, 16, 3, 8, 12).to(torch.bfloat16)
    X = torch.empty(2 * 3 * 4 * 6, 64, dtype=torch.bfloat16, device="cuda")
    B().op_patchify(lat.cuda(), X)
    B().op_sync()
    assert torch.equal(X.cpu().to(DT), O.patchify(lat.to(DT)).reshape(X.shape))


@pytest.mark.parametrize("shape", [(1, 16, 3, 16, 16), (2, 16, 21, 60, 104), (1, 48, 3, 44, 80)])
def test_unpatchify_bit_exact(shape):
    Bn, Cc, F, Hz, Wz = shape
    L = O.token_count(F, Hz, Wz)
    rows = torch.randn(Bn * L, 4 * Cc)
    vel = torch.full(shape, float("nan"), device="cuda")
    B().op_unpatchify(rows.cuda(), vel)
    B().op_sync()
    ref = O.unpatchify(rows.reshape(Bn, L, 4 * Cc).to(DT), Cc, F, Hz, Wz)
    assert torch.equal(vel.cpu().to(DT), ref)


# ------------------------------------------------------------------ GEMM
def _gemm_inputs(M, N, K, seed=0):
    g = torch.Generator().manual_seed(seed)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    W = (torch.randn(N, K, generator=g) * 0.05).to(torch.bfloat16)
    bias = torch.randn(N, generator=g)
    return A, W, bias


@pytest.mark.parametrize("M,N,K", [(300, 256, 192), (1000, 1536, 1536), (129, 128, 64), (77, 64, 256),
                                   (4100, 4608, 1536), (452, 9216, 1536)])
def test_gemm_bias(M, N, K):
    A, W, bias = _gemm_inputs(M, N, K)
    out = torch.zeros(M, N, dtype=torch.bfloat16, device="cuda")
    B().op_gemm(A.cuda(), W.cuda(), "bias", out, bias=bias.cuda())
    B().op_sync()
    ref = O.linear(A.to(DT), W.to(DT), bias.to(DT))
    assert rel_l2(out, ref) < TOL


def test_gemm_bias_gelu_and_f32():
    M, N, K = 333, 512, 320
    A, W, bias = _gemm_inputs(M, N, K, seed=1)
    out = torch.zeros(M, N, dtype=torch.bfloat16, device="cuda")
    B().op_gemm(A.cuda(), W.cuda(), "bias_gelu", out, bias=bias.cuda())
    out32 = torch.zeros(M, N, dtype=torch.float32, device="cuda")
    B().op_gemm(A.cuda(), W.cuda(), "bias_f32", out32, bias=bias.cuda())
    B().op_sync()
    lin = O.linear(A.to(DT), W.to(DT), bias.to(DT))
    assert rel_l2(out, O.gelu_tanh(lin)) < TOL
    assert rel_l2(out32, lin) < 1e-4


@pytest.mark.parametrize("per_token", [False, True])
def test_gemm_gate_residual(per_token):
    M, N, K, L = 400, 256, 256, 200          # two samples of 200 tokens
    A, W, bias = _gemm_inputs(M, N, K, seed=2)
    g = torch.Generator().manual_seed(3)
    x = torch.randn(M, N, generator=g).to(torch.bfloat16)
    sst = torch.randn(6, N, generator=g) * 0.1
    rows_mod = M if per_token else 2
    tproj = torch.randn(rows_mod, 6, N, generator=g) * 0.1
    xd = x.cuda()
    B().op_gemm(A.cuda(), W.cuda(), "gate_residual", xd, bias=bias.cuda(), gate0=sst[2].contiguous().cuda(),
                gate1=tproj[:, 2].contiguous().cuda(), mod_div=1 if per_token else L, mod_ld=N)
    B().op_sync()
    gate = sst[2].to(DT) + (tproj[:, 2].to(DT) if per_token else tproj[:, 2].to(DT).repeat_interleave(L, 0))
    ref = x.to(DT) + O.linear(A.to(DT), W.to(DT), bias.to(DT)) * gate
    assert rel_l2(xd, ref) < TOL


def test_gemm_gate_residual_single_gate_vector():
    # the per-sample form the forward uses: one precombined gate row per sample (gate0 absent),
    # and the table-only form (gate1 absent)
    M, N, K, L = 400, 256, 256, 200
    A, W, bias = _gemm_inputs(M, N, K, seed=6)
    g = torch.Generator().manual_seed(7)
    x = torch.randn(M, N, generator=g).to(torch.bfloat16)
    rows = torch.randn(2, 6, N, generator=g) * 0.1
    lin = O.linear(A.to(DT), W.to(DT), bias.to(DT))
    xd = x.cuda()
    B().op_gemm(A.cuda(), W.cuda(), "gate_residual", xd, bias=bias.cuda(), gate1=rows[:, 2].contiguous().cuda(),
                mod_div=L, mod_ld=N)
    B().op_sync()
    assert rel_l2(xd, x.to(DT) + lin * rows[:, 2].to(DT).repeat_interleave(L, 0)) < TOL
    xd = x.cuda()
    B().op_gemm(A.cuda(), W.cuda(), "gate_residual", xd, bias=bias.cuda(), gate0=rows[0, 5].contiguous().cuda())
    B().op_sync()
    assert rel_l2(xd, x.to(DT) + lin * rows[0, 5].to(DT)) < TOL
    with pytest.raises(B().WanError):
        B().op_gemm(A.cuda(), W.cuda(), "gate_residual", x.cuda(), bias=bias.cuda())


def test_gemm_residual():
    M, N, K = 260, 384, 128
    A, W, bias = _gemm_inputs(M, N, K, seed=4)
    x = torch.randn(M, N).to(torch.bfloat16)
    xd = x.cuda()
    B().op_gemm(A.cuda(), W.cuda(), "residual", xd, bias=bias.cuda())
    B().op_sync()
    ref = x.to(DT) + O.linear(A.to(DT), W.to(DT), bias.to(DT))
    assert rel_l2(xd, ref) < TOL


@pytest.mark.parametrize("shape", [(1, 16, 3, 16, 16), (2, 16, 5, 12, 20), (1, 48, 2, 8, 8)])
def test_gemm_unpatchify_epilogue(shape):
    Bn, Cc, F, Hz, Wz = shape
    L = O.token_count(F, Hz, Wz)
    M, N, K = Bn * L, 4 * Cc, 256
    A, W, bias = _gemm_inputs(M, N, K, seed=5)
    vel = torch.full(shape, float("nan"), device="cuda")
    B().op_gemm(A.cuda(), W.cuda(), "unpatchify", vel, bias=bias.cuda(), unpatch=(Cc, F, Hz, Wz))
    B().op_sync()
    o = O.linear(A.to(DT), W.to(DT), bias.to(DT)).reshape(Bn, L, N)
    ref = O.unpatchify(o, Cc, F, Hz, Wz)
    assert not torch.isnan(vel).any()
    assert rel_l2(vel, ref) < TOL


def test_gemm_rejects_bad_shapes():
    from video_diffusion_transformer_dit_b200.binding import WanError
    A = torch.zeros(64, 100, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(64, 100, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(WanError):
        B().op_gemm(A, W, "bias", out)


# ------------------------------------------------------------------ attention
@pytest.mark.parametrize("Bn,heads,Lq,Lk", [(1, 1, 128, 128), (2, 2, 300, 300), (2, 3, 200, 226),
                                            (1, 2, 1000, 32), (1, 1, 5, 700)])
def test_attention(Bn, heads, Lq, Lk):
    D = heads * 128
    g = torch.Generator().manual_seed(Lq * 7 + Lk)
    q = torch.randn(Bn * Lq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(Bn * Lk, D, generator=g).to(torch.bfloat16)
    v = torch.randn(Bn * Lk, D, generator=g).to(torch.bfloat16)
    o = torch.zeros(Bn * Lq, D, dtype=torch.bfloat16, device="cuda")
    B().op_attention(q.cuda(), k.cuda(), v.cuda(), o, Bn, heads, Lq, Lk)
    B().op_sync()
    ref = O.attention(q.to(DT).reshape(Bn, Lq, heads, 128), k.to(DT).reshape(Bn, Lk, heads, 128),
                      v.to(DT).reshape(Bn, Lk, heads, 128)).reshape(Bn * Lq, D)
    assert rel_l2(o, ref) < TOL


@pytest.mark.parametrize("Lk", [226, 300, 512])
def test_attention_units_walked_per_cta(Lk):
    """Short key sets (2, 3 or 4 key tiles) run with one CTA per SM walking
    256-query units; B = 2, 12 heads, Lq = 2000 (eight query blocks, the last
    ragged) give 192 units, so CTAs take one or two units and the barrier
    phases carry over between them; compared with the oracle per element and
    against a run whose units fit one per CTA (the first two heads alone)."""
    Bn, heads, Lq = 2, 12, 2000
    D = heads * 128
    g = torch.Generator().manual_seed(90 + Lk)
    q = torch.randn(Bn * Lq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(Bn * Lk, D, generator=g).to(torch.bfloat16)
    v = torch.randn(Bn * Lk, D, generator=g).to(torch.bfloat16)
    o = torch.full((Bn * Lq, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    B().op_attention(q.cuda(), k.cuda(), v.cuda(), o, Bn, heads, Lq, Lk)
    B().op_sync()
    ref = O.attention(q.to(DT).reshape(Bn, Lq, heads, 128), k.to(DT).reshape(Bn, Lk, heads, 128),
                      v.to(DT).reshape(Bn, Lk, heads, 128)).reshape(Bn * Lq, D)
    assert not torch.isnan(o.float()).any()
    assert rel_l2(o, ref) < TOL
    # two heads: 32 units, one per CTA; same per-row arithmetic, same bits
    o2 = torch.empty(Bn * Lq, 256, dtype=torch.bfloat16, device="cuda")
    B().op_attention(q[:, :256].contiguous().cuda(), k[:, :256].contiguous().cuda(), v[:, :256].contiguous().cuda(),
                     o2, Bn, 2, Lq, Lk)
    B().op_sync()
    assert torch.equal(o2.cpu(), o.cpu()[:, :256])


def test_attention_strided_qkv_buffer():
    """q, k, v as column slices of one [rows, 3D] buffer, as the forward uses them."""
    Bn, heads, L = 2, 2, 260
    D = heads * 128
    qkv = torch.randn(Bn * L, 3 * D).to(torch.bfloat16)
    d = qkv.cuda()
    o = torch.zeros(Bn * L, D, dtype=torch.bfloat16, device="cuda")
    base = d.data_ptr()
    B().op_attention_ptr(base, 3 * D, base + 2 * D, 3 * D, base + 4 * D, 3 * D, o.data_ptr(), D, Bn, heads, L, L)
    B().op_sync()
    t = qkv.to(DT).reshape(Bn, L, 3, heads, 128)
    ref = O.attention(t[:, :, 0], t[:, :, 1], t[:, :, 2]).reshape(Bn * L, D)
    assert rel_l2(o, ref) < TOL


def test_attention_large_logits_rescale():
    """Keys whose logits grow along the sequence force the running-max rescale."""
    Bn, heads, Lq, Lk = 1, 1, 128, 1024
    g = torch.Generator().manual_seed(11)
    q = torch.randn(Lq, 128, generator=g)
    k = torch.randn(Lk, 128, generator=g) * torch.linspace(0.1, 4.0, Lk)[:, None]
    v = torch.randn(Lk, 128, generator=g)
    q, k, v = (t.to(torch.bfloat16) for t in (q, k, v))
    o = torch.zeros(Lq, 128, dtype=torch.bfloat16, device="cuda")
    B().op_attention(q.cuda(), k.cuda(), v.cuda(), o, Bn, heads, Lq, Lk)
    B().op_sync()
    ref = O.attention(q.to(DT)[None, :, None], k.to(DT)[None, :, None], v.to(DT)[None, :, None])[0, :, 0]
    assert rel_l2(o, ref) < TOL


@pytest.mark.parametrize("Lq,Lk", [(1100, 777), (1300, 640), (513, 1000), (2048, 2056)])
def test_attention_sm_pairs_ragged(Lq, Lk):
    """Key sets longer than four tiles run on SM pairs (512 queries per cluster,
    each CTA holding 64-key halves of K and 64-column halves of V).  Lq = 1100
    leaves the last pair's odd CTA without a valid row, 1300 with some, 513 the
    even CTA with one; Lk = 777 and 2056 end in a tile whose odd-CTA key half is
    all padding.  B = 2, 3 heads against the oracle per element."""
    Bn, heads = 2, 3
    D = heads * 128
    g = torch.Generator().manual_seed(Lq + 3 * Lk)
    q = torch.randn(Bn * Lq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(Bn * Lk, D, generator=g).to(torch.bfloat16)
    v = torch.randn(Bn * Lk, D, generator=g).to(torch.bfloat16)
    o = torch.full((Bn * Lq, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    B().op_attention(q.cuda(), k.cuda(), v.cuda(), o, Bn, heads, Lq, Lk)
    B().op_sync()
    ref = O.attention(q.to(DT).reshape(Bn, Lq, heads, 128), k.to(DT).reshape(Bn, Lk, heads, 128),
                      v.to(DT).reshape(Bn, Lk, heads, 128)).reshape(Bn * Lq, D)
    assert not torch.isnan(o.float()).any()
    assert rel_l2(o, ref) < TOL


@pytest.mark.parametrize("Lk", [226, 1024])
def test_attention_rejects_misaligned_operands_before_launch(Lk):
    """A pointer off the 16-byte grid or a leading dimension that is not a
    multiple of 8 elements is WAN_ESHAPE, for the single-SM (226 keys) and the
    SM-pair (1024 keys) kernels alike, and nothing is written."""
    Bn, heads, Lq = 1, 2, 300
    D = heads * 128
    q = torch.randn(Bn * Lq + 1, D + 8).to(torch.bfloat16).cuda()
    kv = torch.randn(Bn * Lk + 1, D + 8).to(torch.bfloat16).cuda()
    o = torch.full((Bn * Lq + 1, D + 8), 7.0, dtype=torch.bfloat16, device="cuda")
    qp, kp, op = q.data_ptr(), kv.data_ptr(), o.data_ptr()
    ld = D + 8
    bad = [(qp + 2, ld, kp, ld, op, ld),          # q not 16-byte aligned
           (qp, ld, kp, ld, op + 2, ld),          # o not 16-byte aligned
           (qp, ld - 1, kp, ld, op, ld),          # ldq not a multiple of 8
           (qp, ld, kp, ld - 4, op, ld)]          # ldk not a multiple of 8
    for q_, ldq, k_, ldk, o_, ldo in bad:
        with pytest.raises(B().WanError) as e:
            B().op_attention_ptr(q_, ldq, k_, ldk, k_, ldk, o_, ldo, Bn, heads, Lq, Lk)
        assert e.value.name == "WAN_ESHAPE"
    B().op_sync()
    assert torch.all(o.cpu() == 7.0)


def test_attention_sm_pairs_zero_wait_limit_reports_and_recovers():
    """Waits that give up at the first open barrier in both CTAs of every pair:
    the op reports WAN_ETIMEOUT (or finishes), the pair drains its loads and
    MMAs, and the next run with the normal limit gives the reference bits."""
    Bn, heads, L = 1, 4, 2048
    D = heads * 128
    g = torch.Generator().manual_seed(5)
    q, k, v = (torch.randn(Bn * L, D, generator=g).to(torch.bfloat16).cuda() for _ in range(3))
    ref = torch.empty(Bn * L, D, dtype=torch.bfloat16, device="cuda")
    B().op_attention(q, k, v, ref, Bn, heads, L, L)
    B().op_sync()
    seen = []
    B().op_set_wait_limit_ns(0)
    try:
        for _ in range(3):
            o = torch.empty_like(ref)
            B().op_attention(q, k, v, o, Bn, heads, L, L)
            try:
                B().op_sync()
                seen.append("WAN_OK")
            except B().WanError as e:
                seen.append(e.name)
    finally:
        B().op_set_wait_limit_ns(2_000_000_000)
    assert "WAN_ETIMEOUT" in seen, seen
    assert set(seen) <= {"WAN_ETIMEOUT", "WAN_OK"}, seen
    again = torch.empty_like(ref)
    B().op_attention(q, k, v, again, Bn, heads, L, L)
    B().op_sync()
    assert torch.equal(again.cpu(), ref.cpu())


# ------------------------------------------------------------------ norms
@pytest.mark.parametrize("D", [1536, 3072, 5120])
def test_layernorm_modulated(D):
    rows, L = 600, 300
    g = torch.Generator().manual_seed(D)
    x = (torch.randn(rows, D, generator=g) * 2 + 0.5).to(torch.bfloat16)
    sst = torch.randn(6, D, generator=g) * 0.2
    tproj = torch.randn(2, 6, D, generator=g) * 0.2
    y = torch.zeros_like(x, device="cuda")
    tp = tproj.reshape(2, 6 * D).contiguous().cuda()
    s = sst.cuda()
    B().op_layernorm(x.cuda(), y, 1e-6, 0, shift0=s[0], shift1=tp[:, 0:D], scale0=s[1], scale1=tp[:, D:2 * D],
                     mod_div=L, mod_ld=6 * D)
    B().op_sync()
    shift = sst[0].to(DT) + tproj[:, 0].to(DT).repeat_interleave(L, 0)
    scale = sst[1].to(DT) + tproj[:, 1].to(DT).repeat_interleave(L, 0)
    ref = O.layer_norm(x.to(DT), 1e-6) * (1 + scale) + shift
    assert rel_l2(y, ref) < TOL


def test_layernorm_affine():
    rows, D = 333, 1536
    x = torch.randn(rows, D).to(torch.bfloat16)
    gam = 1 + torch.randn(D) * 0.1
    bet = torch.randn(D) * 0.1
    y = torch.zeros_like(x, device="cuda")
    B().op_layernorm(x.cuda(), y, 1e-6, 1, gamma=gam.cuda(), beta=bet.cuda())
    B().op_sync()
    assert rel_l2(y, O.layer_norm(x.to(DT), 1e-6, gam.to(DT), bet.to(DT))) < TOL


@pytest.mark.parametrize("D", [256, 1536])
def test_layernorm_row_walking_modes(D):
    """Enough rows (>= 8 warps per SM) for the kernel in which each warp walks
    consecutive rows with the modulation in registers: mode 2 (precombined
    per-sample scale / shift, the sample boundary 2123 falls inside a warp's
    rows) and mode 1 (affine); 4246 rows leave the last warp a ragged share."""
    rows, L = 4246, 2123
    g = torch.Generator().manual_seed(70 + D)
    x = (torch.randn(rows, D, generator=g) * 2 + 0.5).to(torch.bfloat16)
    scale1 = 1 + torch.randn(2, D, generator=g) * 0.2
    shift1 = torch.randn(2, D, generator=g) * 0.2
    tab = torch.zeros(2, 6 * D)
    tab[:, 0:D], tab[:, D:2 * D] = shift1, scale1
    tab = tab.cuda()
    y = torch.full((rows, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    B().op_layernorm(x.cuda(), y, 1e-6, 2, shift1=tab[:, 0:D], scale1=tab[:, D:2 * D], mod_div=L, mod_ld=6 * D)
    B().op_sync()
    ln = O.layer_norm(x.to(DT), 1e-6)
    ref = ln * scale1.to(DT).repeat_interleave(L, 0) + shift1.to(DT).repeat_interleave(L, 0)
    assert not torch.isnan(y.float()).any()
    assert rel_l2(y, ref) < TOL
    gam, bet = scale1[0].contiguous(), shift1[1].contiguous()
    y.fill_(float("nan"))
    B().op_layernorm(x.cuda(), y, 1e-6, 1, gamma=gam.cuda(), beta=bet.cuda())
    B().op_sync()
    assert not torch.isnan(y.float()).any()
    assert rel_l2(y, O.layer_norm(x.to(DT), 1e-6, gam.to(DT), bet.to(DT))) < TOL


@pytest.mark.parametrize("rope", [False, True])
def test_rmsnorm_rope(rope):
    Fp, Hp, Wp = 3, 5, 7
    L = Fp * Hp * Wp
    Bn, D = 2, 1536
    ld = 3 * D
    buf = torch.randn(Bn * L, ld).to(torch.bfloat16)
    gain = 1 + torch.randn(D) * 0.1
    d = buf.cuda()
    B().op_rmsnorm_rope(d.data_ptr() + 2 * D, ld, Bn * L, D, 1e-6, gain.cuda(), rope=rope, grid=(Fp, Hp, Wp))
    B().op_sync()
    seg = buf[:, D:2 * D].to(DT)
    ref = O.rms_norm(seg, 1e-6, gain.to(DT))
    if rope:
        ang = O.rope_angles((Fp, Hp, Wp), (44, 42, 42), 10000.0)
        ref = O.rope_apply(ref.reshape(Bn, L, 12, 128), ang).reshape(Bn * L, D)
    got = d.cpu()
    assert rel_l2(got[:, D:2 * D], ref) < TOL
    assert torch.equal(got[:, :D], buf[:, :D]) and torch.equal(got[:, 2 * D:], buf[:, 2 * D:])


# ------------------------------------------------------------------ q/k RMSNorm split across the QKV epilogue
@pytest.mark.parametrize("grid", [(3, 5, 9), (5, 12, 13)], ids=["L135", "L780"])
@pytest.mark.parametrize("rope", [True, False])
def test_qk_norm_epilogue_row_factors_and_attention(rope, grid):
    """The self-attention path with RMSNorm across heads in two parts: the QKV
    GEMM epilogue (gain, RoPE, per-head sums of squares), the key row factors in
    place, the query row factors inside the attention -- against the oracle's
    RMSNorm + RoPE + attention.  B = 2; L = 135 tokens (two key tiles, the
    single-SM kernel, a ragged second tile) and L = 780 (seven key tiles, the
    SM-pair kernel: the second pair's odd CTA holds 12 valid query rows)."""
    Fp, Hp, Wp = grid
    L, Bn, D, h, eps = Fp * Hp * Wp, 2, 1536, 12, 1e-6
    R = Bn * L
    g = torch.Generator().manual_seed(40)
    y = torch.randn(R, D, generator=g).to(torch.bfloat16)
    W = (0.02 * torch.randn(3 * D, D, generator=g)).to(torch.bfloat16)
    bias = 0.02 * torch.randn(3 * D, generator=g)
    gain = 1 + 0.1 * torch.randn(2 * D, generator=g)
    qkv = torch.empty(R, 3 * D, dtype=torch.bfloat16, device="cuda")
    ssq = torch.empty(R, 2 * h, device="cuda")
    B().op_gemm(y.cuda(), W.cuda(), "qk_norm", qkv, bias=bias.cuda(), gain=gain.cuda(), ssq=ssq, norm_cols=2 * D,
                rope_grid=(Fp, Hp, Wp) if rope else None)
    B().op_sync()
    lin = O.linear(y.to(DT), W.to(DT), bias.to(DT))
    ref_ssq = (lin[:, :2 * D] ** 2).reshape(R, 2 * h, 128).sum(-1)
    assert rel_l2(ssq.cpu(), ref_ssq) < 1e-4
    ang = O.rope_angles((Fp, Hp, Wp), (44, 42, 42), 10000.0)

    def rot(x):
        return O.rope_apply(x.reshape(Bn, L, h, 128), ang).reshape(R, D) if rope else x
    # stored q and k: gain * (acc + bias), rotated, not yet normalised; v plain
    stored = qkv.cpu()
    assert rel_l2(stored[:, :D], rot(lin[:, :D] * gain[:D].to(DT))) < TOL
    assert rel_l2(stored[:, 2 * D:], lin[:, 2 * D:]) < TOL
    base = qkv.data_ptr()
    B().op_rms_apply(base + 2 * D, 3 * D, R, D, ssq.data_ptr() + 4 * h, ssq.stride(0), h, eps)
    o = torch.empty(R, D, dtype=torch.bfloat16, device="cuda")
    B().op_attention_qnorm(base, 3 * D, base + 2 * D, 3 * D, base + 4 * D, 3 * D, o, Bn, h, L, L, ssq, h, eps)
    B().op_sync()
    q = rot(O.rms_norm(lin[:, :D], eps, gain[:D].to(DT)))
    k = rot(O.rms_norm(lin[:, D:2 * D], eps, gain[D:].to(DT)))
    assert rel_l2(qkv.cpu()[:, D:2 * D], k) < TOL                     # keys normalised in place
    ref = O.attention(q.reshape(Bn, L, h, 128), k.reshape(Bn, L, h, 128), lin[:, 2 * D:].reshape(Bn, L, h, 128))
    assert rel_l2(o.cpu(), ref.reshape(R, D)) < TOL


# ------------------------------------------------------------------ sampler step (CFG + Euler)
def test_cfg_euler_matches_oracle_and_worked_example():
    g = torch.Generator().manual_seed(21)
    shape = (1, 16, 21, 60, 104)
    x, vc, vu = (torch.randn(*shape, generator=g) for _ in range(3))
    out = torch.empty(shape, device="cuda")
    B().op_cfg_euler(x.cuda(), vc.cuda(), vu.cuda(), 6.0, 0.75, 0.5, out)
    B().op_sync()
    ref = O.euler_step(x.to(DT), 0.75, 0.5, O.cfg_combine(vu.to(DT), vc.to(DT), 6.0))
    assert rel_l2(out, ref) < 1e-6
    # the hand-worked example of the flow-matching section: x=8, v=8, sigma 0.75 -> 0.5 -> 0
    xs = torch.full((5,), 8.0, device="cuda")
    vs = torch.full((5,), 8.0, device="cuda")
    x1 = torch.empty_like(xs)
    B().op_cfg_euler(xs, vs, None, 1.0, 0.75, 0.5, x1)
    x2 = torch.empty_like(xs)
    B().op_cfg_euler(x1, vs, None, 1.0, 0.5, 0.0, x2)
    B().op_sync()
    assert torch.equal(x1.cpu(), torch.full((5,), 6.0)) and torch.equal(x2.cpu(), torch.full((5,), 2.0))


# ------------------------------------------------------------------ VAE decoder: causal Conv3d

@pytest.mark.parametrize("Ci,Co,kernel,T,nc", [(64, 128, (3, 3, 3), 3, 0), (16, 64, (3, 3, 3), 2, 2),
                                               (64, 128, (3, 1, 1), 4, 1), (32, 64, (1, 1, 1), 2, 0)])
def test_causal_conv3d_matches_oracle(Ci, Co, kernel, T, nc):
    """Channels-last causal Conv3d (gather + tcgen05 GEMM) against the oracle's
    WanCausalConv3d, with and without a cache of the frames before frame 0;
    Ci = 16 exercises the zero-padded K (432 -> 448)."""
    Bn, H, W = 2, 5, 7
    kt, kh, kw = kernel
    g = torch.Generator().manual_seed(Ci + Co + T + nc)
    x = torch.randn(Bn, Ci, T, H, W, generator=g).to(torch.bfloat16)
    w = (torch.randn(Co, Ci, kt, kh, kw, generator=g) * 0.05).to(torch.bfloat16)
    bias = torch.randn(Co, generator=g) * 0.1
    cache = torch.randn(Bn, Ci, nc, H, W, generator=g).to(torch.bfloat16) if nc else None
    ref = V.causal_conv3d(x.to(DT), w.to(DT), bias.to(DT), cache.to(DT) if nc else None)
    K = kt * kh * kw * Ci
    Kp = (K + 63) // 64 * 64
    wp = torch.zeros(Co, Kp, dtype=torch.bfloat16)
    wp[:, :K] = w.permute(0, 2, 3, 4, 1).reshape(Co, K)
    xd = x.permute(0, 2, 3, 4, 1).contiguous().cuda()
    cd = cache.permute(0, 2, 3, 4, 1).contiguous().cuda() if nc else None
    col = torch.empty(Bn * T * H * W * Kp, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(Bn, T, H, W, Co, dtype=torch.bfloat16, device="cuda")
    B_ = B()
    B_.op_causal_conv3d(xd, wp.cuda(), bias.cuda(), col, y, kernel, cache=cd)
    B_.op_sync()
    got = y.cpu().permute(0, 4, 1, 2, 3)
    assert rel_l2(got, ref) < TOL
    with pytest.raises(B_.WanError):                 # Co must be a multiple of 64
        B_.op_causal_conv3d(xd, wp[:32].contiguous().cuda(), None, col, y[..., :32].contiguous(), kernel, cache=cd)


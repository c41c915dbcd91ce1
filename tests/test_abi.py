"""Host-side checks of the C ABI that need no GPU: the library builds, loads,
exports every entry point include/*.h declares, and rejects configurations
the kernels do not cover before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from video_diffusion_transformer_dit_b200 import binding, build
    build.build()
    return binding.lib()


def declared_symbols():
    names = set()
    for h in ("wandit.h", "wandit_ops.h", "wanvae.h"):
        text = open(os.path.join(ROOT, "include", h)).read()
        names |= set(re.findall(r"WANDIT_API\s+[\w\s\*]+?\b(wan_\w+)\s*\(", text))
    return names


def test_every_declared_symbol_is_exported(lib):
    from video_diffusion_transformer_dit_b200 import binding
    names = declared_symbols()
    assert len(names) >= 20
    assert names == set(binding.SYMBOLS)
    for n in names:
        assert getattr(lib, n) is not None


def test_status_strings(lib):
    for code in range(11):
        s = lib.wan_status_string(code)
        assert s and s.decode() != "unknown status"


def test_create_rejects_unsupported_configs_without_a_device(lib):
    from video_diffusion_transformer_dit_b200 import binding, configs
    base = configs.model_config("wan2.1-1.3b")
    bad = [dict(base, head_dim=64, heads=24), dict(base, dim=1000), dict(base, patch=(2, 2, 2)),
           dict(base, rope_split=(44, 42, 40)), dict(base, ffn_dim=100)]
    for cfg in bad:
        c = binding.make_config(cfg, 1, 192, 32)
        h = ctypes.c_void_p()
        assert lib.wan_dit_create(ctypes.byref(c), 0, ctypes.byref(h)) == 10   # WAN_EUNSUPPORTED
        assert not h
    # image branch: width a multiple of 64, and a token limit with it
    i2v = configs.model_config("wan2.1-i2v-14b")
    for cfg, max_image in ((dict(i2v, image_dim=1000), 257), (i2v, 0)):
        c = binding.make_config(cfg, 1, 192, 32, max_image)
        h = ctypes.c_void_p()
        assert lib.wan_dit_create(ctypes.byref(c), 0, ctypes.byref(h)) == 10
        assert not h
    h = ctypes.c_void_p()
    assert lib.wan_dit_create(None, 0, ctypes.byref(h)) == 1                   # WAN_EINVAL


def test_moe_select_follows_the_switch_rule(lib):
    from oracle import wan_oracle as O
    from video_diffusion_transformer_dit_b200 import binding
    for boundary, n in ((0.875, 1000), (0.9, 1000), (0.5, 100)):
        for t in [0.0, 1.0, 87.4, 87.5, 450.0, 874.999, 875.0, 875.001, 899.9, 900.0, 999.0]:
            assert binding.moe_select(t, boundary, n) == O.moe_expert(t, boundary, n), (t, boundary, n)


def test_null_handle_calls_are_refused(lib):
    assert lib.wan_dit_forward(None, None, 0, 1, 1, 2, 2, None, 0, None, 1, None, 1, None) == 1
    assert lib.wan_dit_forward_image(None, None, 0, 1, 1, 2, 2, None, 0, None, 1, None, 0, None, 1, None) == 1
    assert lib.wan_dit_sync(None, None) == 1
    assert lib.wan_dit_last_launch_count(None) == 0
    assert lib.wan_dit_last_error(None) == b"null handle"


def test_attention_ops_reject_bad_arguments_before_the_device(lib):
    """Null pointers give WAN_EINVAL and impossible shapes WAN_ESHAPE, both
    before the op looks for a device (the checks run here without one)."""
    fake = ctypes.c_void_p(1 << 20)            # never dereferenced: every call below is refused first
    att, attq = lib.wan_op_attention, lib.wan_op_attention_qnorm
    assert att(None, 128, fake, 128, fake, 128, fake, 128, 1, 1, 128, 128, None) == 1
    assert att(fake, 128, fake, 128, fake, 128, None, 128, 1, 1, 128, 128, None) == 1
    for B, heads, Lq, Lk in ((-1, 1, 128, 128), (1, 0, 128, 128), (1, 1, -1, 128), (1, 1, 128, 0)):
        assert att(fake, 128, fake, 128, fake, 128, fake, 128, B, heads, Lq, Lk, None) == 2
    assert attq(fake, 128, fake, 128, fake, 128, fake, 128, 1, 1, 128, 128, None, 1, 1,
                ctypes.c_float(1e-6), None) == 1
    for ssq_ld, ngroups in ((1, 0), (1, 2)):
        assert attq(fake, 128, fake, 128, fake, 128, fake, 128, 1, 1, 128, 128, fake, ssq_ld, ngroups,
                    ctypes.c_float(1e-6), None) == 2


def test_flow_sigmas_match_oracle(lib):
    """The host-side sigma schedule against the oracle's reading R22."""
    import torch
    from oracle import wan_oracle as O
    from video_diffusion_transformer_dit_b200 import binding
    for steps, shift in ((1, 1.0), (4, 1.0), (50, 3.0), (40, 5.0), (30, 0.5)):
        got = torch.tensor(binding.flow_sigmas(steps, shift), dtype=torch.float64)
        torch.testing.assert_close(got, O.sampling_sigmas(steps, shift), rtol=1e-14, atol=1e-15)
    for steps, shift in ((0, 3.0), (10, 0.0), (10, -1.0)):
        with pytest.raises(binding.WanError):
            binding.flow_sigmas(steps, shift)

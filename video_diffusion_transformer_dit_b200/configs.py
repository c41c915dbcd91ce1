"""Model presets and the synthetic workloads of the Wan DiT forward.

Dimensions follow the model-size table of the Wan pages (Wan2.1 1.3B: width
1536, 30 blocks; 14B: width 5120, 40 blocks, 40 heads, FFN 13824; Wan2.2 5B:
width 3072, 30 blocks, 24 heads, 48 latent channels) and the diffusers config
defaults (head_dim 128, text_dim 4096, freq_dim 256, eps 1e-6, patch (1,2,2)).
Pure data: no arithmetic of the method lives here.
"""
from __future__ import annotations

import copy

_COMMON = dict(head_dim=128, patch=(1, 2, 2), text_dim=4096, freq_dim=256, eps=1e-6,
               rope_split=(44, 42, 42), rope_theta=10000.0, image_dim=0)

MODELS = {
    "wan2.1-1.3b": dict(dim=1536, heads=12, ffn_dim=8960, num_blocks=30, in_ch=16, out_ch=16, **_COMMON),
    "wan2.1-14b": dict(dim=5120, heads=40, ffn_dim=13824, num_blocks=40, in_ch=16, out_ch=16, **_COMMON),
    "wan2.2-5b": dict(dim=3072, heads=24, ffn_dim=14336, num_blocks=30, in_ch=48, out_ch=48, **_COMMON),
    # image-to-video route: 16 noisy + 16 condition + 4 mask channels in, CLIP image tokens of width 1280
    "wan2.1-i2v-14b": dict(dim=5120, heads=40, ffn_dim=13824, num_blocks=40, in_ch=36, out_ch=16,
                           **dict(_COMMON, image_dim=1280)),
}

# name -> (model, overrides, latent shape [B,C,F,Hz,Wz], text length, timesteps, notes)
WORKLOADS = {
    # one block + head, 192 tokens: the case the oracle finishes in seconds
    "wan1.3b-1blk-3x16x16": dict(model="wan2.1-1.3b", overrides=dict(num_blocks=1),
                                 latent=(1, 16, 3, 16, 16), text_len=32, timesteps=(500.0,)),
    # one block + head on a CFG pair, 720 tokens: self-attention and the block GEMMs on SM pairs
    # (the second 512-query pair ragged), still a case the oracle finishes in seconds
    "wan1.3b-1blk-5x24x24-cfg2": dict(model="wan2.1-1.3b", overrides=dict(num_blocks=1),
                                      latent=(2, 16, 5, 24, 24), text_len=32, timesteps=(500.0,),
                                      same_latent=True),
    # 33 frames 352x640 -> 7920 tokens, 30 blocks
    "wan1.3b-33f-352x640": dict(model="wan2.1-1.3b", overrides={},
                                latent=(1, 16, 9, 44, 80), text_len=226, timesteps=(999.0,)),
    # 81 frames 480x832 -> 32760 tokens, CFG batch 2 (same latent, two contexts)
    "wan1.3b-81f-480x832-cfg2": dict(model="wan2.1-1.3b", overrides={},
                                     latent=(2, 16, 21, 60, 104), text_len=226,
                                     timesteps=(999.0, 500.0, 20.0), same_latent=True),
    # 81 frames 720x1280 -> 75600 tokens, 14B shape
    "wan14b-81f-720x1280": dict(model="wan2.1-14b", overrides={},
                                latent=(1, 16, 21, 90, 160), text_len=512, timesteps=(500.0,)),
    # I2V at 1.3B widths, one block + head, 192 tokens, 257 image tokens (CFG-style batch of 2)
    "wan-i2v-1blk-3x16x16": dict(model="wan2.1-i2v-14b",
                                 overrides=dict(dim=1536, heads=12, ffn_dim=8960, num_blocks=1),
                                 latent=(2, 36, 3, 16, 16), text_len=32, image_len=257, timesteps=(500.0,)),
    # I2V route at Wan2.1-I2V-14B shapes, 81 frames 480x832 -> 32760 tokens, 257 image tokens
    "wan-i2v-14b-81f-480x832": dict(model="wan2.1-i2v-14b", overrides={},
                                    latent=(1, 36, 21, 60, 104), text_len=512, image_len=257, timesteps=(500.0,)),
    # Wan2.2-5B shape, 121 frames 704x1280 -> 27280 tokens, per-token timestep
    "wan5b-121f-704x1280-pertoken": dict(model="wan2.2-5b", overrides={},
                                         latent=(1, 48, 31, 44, 80), text_len=512, timesteps="per_token"),
}


def model_config(name: str, **overrides) -> dict:
    cfg = copy.deepcopy(MODELS[name])
    cfg.update(overrides)
    return cfg


def workload(name: str) -> dict:
    w = copy.deepcopy(WORKLOADS[name])
    w["cfg"] = model_config(w["model"], **w["overrides"])
    w["name"] = name
    return w

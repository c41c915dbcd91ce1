"""Benchmark of one Wan DiT denoising-step forward on B200 (sm_100a).

Default workload: Wan2.1-1.3B shapes at 480p, 81 frames -> latent
[2,16,21,60,104] (L = 32760 tokens, 30 blocks), CFG batch 2 (one latent, two
independent 226x4096 text contexts), random-init bf16 weights, timesteps
cycling through {999, 500, 20}.  A step is one wan_dit_forward (the whole hot
path).  `value` is whole-job tokens/s with inputs resident in HBM; `e2e` is the
same metric through the C ABI with host buffers (copies inside the timed
region).  Under torchrun every rank runs an independent replica (the forward
does not shard), timing is max over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

`--impl reference` times the float64 CPU oracle on a bounded sample of the
same workload (see cpu_sample()).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ms/denoise-step & tokens/s, Wan-1.3B-shape 480p; % of B200 bf16 TC peak"
DEFAULT_WORKLOAD = "wan1.3b-81f-480x832-cfg2"
SPEC_BF16_TFLOPS = 2250.0  # B200 dense bf16 tensor-core figure (no 2:4 sparsity)


def measured_traffic(kernel, source):
    """DRAM bytes per launch from the committed ncu capture, only while the kernel
    source is unchanged since the capture (else None)."""
    import hashlib
    try:
        rec = json.load(open(os.path.join(ROOT, "profiles", "roofline_traffic.json")))[kernel]
        sha = hashlib.sha256(open(os.path.join(ROOT, source), "rb").read()).hexdigest()
        return rec["dram_bytes_per_launch"] if sha == rec["source_sha256"] else None
    except (OSError, KeyError, ValueError):
        return None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples (200 ms) during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- CPU oracle sample
def cpu_sample(w, rows_small=128, rows_big=384, seed=0):
    """Time the float64 oracle on a bounded sample of the workload and scale it
    to one full denoising step.

    Sample: one block of the model (sample 0 of the batch) through the
    oracle's row mode at two query-row counts R1 < R2 (keys/values over all L
    tokens).  t(R) = a + b R fits the two timings; one full block is a + b L,
    one step is B * N * (a + b L).  Returns (tokens/s, seconds per step, description)."""
    import torch
    from oracle import wan_oracle as O
    from video_diffusion_transformer_dit_b200 import synth
    use_all_host_cores()
    cfg = dict(w["cfg"])
    B, Cc, F, Hz, Wz = w["latent"]
    L = O.token_count(F, Hz, Wz)
    cfg1 = dict(cfg, num_blocks=1)
    W = {k: v.double() for k, v in synth.make_weights(cfg1, seed=seed).items()}
    lat = synth.make_latent((1, Cc, F, Hz, Wz), seed=seed).double()
    ctx = synth.make_context(1, w["text_len"], cfg["text_dim"], seed=seed).double()
    t = torch.full((1,), 999.0, dtype=torch.float64)
    times = []
    for R in (rows_small, rows_big):
        rows = torch.linspace(0, L - 1, R).long()
        t0 = time.perf_counter()
        O.forward(lat, t, ctx, W, cfg1, rows=rows)
        times.append(time.perf_counter() - t0)
    b = max(0.0, (times[1] - times[0]) / (rows_big - rows_small))
    a = max(0.0, times[0] - b * rows_small)
    block_s = a + b * L
    step_s = B * cfg["num_blocks"] * block_s
    desc = (f"oracle row mode, 1 block x 1 sample at R={rows_small},{rows_big} query rows "
            f"({times[0]:.1f}s, {times[1]:.1f}s); step = B*N*(a+b*L), extrapolated")
    return B * L / step_s, step_s, desc, sum(times)


def use_all_host_cores():
    """Let torch's CPU kernels (the oracle's matmuls, BLAS underneath) use every
    core this process may run on."""
    import torch
    torch.set_num_threads(len(os.sched_getaffinity(0)))


def host_threads():
    """Cores this process may run on and the threads the oracle's CPU kernels used."""
    import torch
    return {"cores": len(os.sched_getaffinity(0)), "blas_threads": torch.get_num_threads()}


# ---------------------------------------------------------------- multi-rank plumbing
def reduce_max(values, device):
    """Max over ranks of per-rank timings (no-op in a single process)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return list(values)
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_tokens_per_s(world, batch, tokens, ms_per_step):
    """Every rank runs its own replica of the step: all ranks' tokens over the slowest rank's time."""
    return world * batch * tokens / (ms_per_step * 1e-3)


def arm_config(workload, world):
    """The `config` object both arms print for a workload."""
    from video_diffusion_transformer_dit_b200 import configs
    w = configs.workload(workload)
    cfg = w["cfg"]
    B, Cc, F, Hz, Wz = w["latent"]
    model = ("Wan2.1-T2V-1.3B shape" if "1.3b" in workload else
             "Wan2.1-I2V-14B shape" if "i2v-14b" in workload else cfg)
    extra = {"image_len": w["image_len"]} if w.get("image_len") else {}
    return {**extra, "workload": workload, "model": model,
            "global_batch": world * B, "seq_len": F * (Hz // 2) * (Wz // 2), "text_len": w["text_len"],
            "blocks": cfg["num_blocks"], "timesteps": w["timesteps"], "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2 (GBs of weights and activations per step); no flush"}


# ---------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from video_diffusion_transformer_dit_b200 import build, configs, synth
    from video_diffusion_transformer_dit_b200.binding import WAN_OPT_GEMM_PAIR, WAN_OPT_KERNEL_TIMING, WanDiT

    build.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = configs.workload(args.workload)
    cfg = w["cfg"]
    if args.blocks:
        cfg["num_blocks"] = args.blocks
    B, Cc, F, Hz, Wz = w["latent"]
    L = F * (Hz // 2) * (Wz // 2)
    Lc = w["text_len"]
    peaks = load_peaks()

    # random-init weights of the named shapes, generated on the device
    W = synth.make_weights(cfg, seed=args.seed, device=str(dev))
    lat = synth.make_latent(w["latent"], seed=args.seed, device=str(dev), same_across_batch=w.get("same_latent", False))
    ctx = synth.make_context(B, Lc, cfg["text_dim"], seed=args.seed, device=str(dev))
    if w["timesteps"] == "per_token":
        ts = [synth.make_timestep_per_token(B, L, (Hz // 2) * (Wz // 2), seed=args.seed).to(dev)]
    else:
        ts = [synth.make_timestep(B, v).to(dev) for v in w["timesteps"]]
    Li = w.get("image_len", 0)   # image tokens per sample (I2V workloads)
    img = synth.make_image(B, Li, cfg["image_dim"], seed=args.seed, device=str(dev)) if Li else None
    dit = WanDiT(cfg, max_batch=B, max_tokens=L, max_text=Lc, device=local_rank, max_image=max(Li, 1))
    dit.load_weights(W)
    dit.set_option(WAN_OPT_GEMM_PAIR, args.gemm_pair)
    del W
    torch.cuda.synchronize()
    vel = torch.empty(B, cfg["out_ch"], F, Hz, Wz, device=dev)
    stream = torch.cuda.current_stream()

    def step(k):
        dit.forward(lat, ts[k % len(ts)], ctx, velocity=vel, image=img)

    for k in range(args.warmup):
        step(k)
    dit.sync()

    dit.set_option(WAN_OPT_KERNEL_TIMING, 1)
    step(0)                      # capture the timed graph outside the timed region
    dit.sync()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for k in range(args.steps):
        step(k)
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    dit.sync()
    if world > 1:
        dist.barrier()
    ms = e0.elapsed_time(e1) / args.steps
    from video_diffusion_transformer_dit_b200.binding import BLOCK_GEMMS
    kt = {c: dit.kernel_time(c) for c in ("self_attention", "gemm", "cross_attention", "layernorm",
                                         "rmsnorm_rope", "patchify", "embedding") + BLOCK_GEMMS}
    gemm_parts = {c: kt.pop(c) for c in BLOCK_GEMMS}
    kt["gemm"] = (kt["gemm"][0] + sum(v[0] for v in gemm_parts.values()),
                  kt["gemm"][1] + sum(v[1] for v in gemm_parts.values()))
    launches = dit.last_launch_count()
    dit.set_option(WAN_OPT_KERNEL_TIMING, 0)

    # end to end through the C ABI with host buffers (pinned), copies inside the timed region
    lat_h = lat.cpu().pin_memory()
    ctx_h = ctx.cpu().pin_memory()
    ts_h = [t.cpu().pin_memory() for t in ts]
    img_h = img.cpu().pin_memory() if img is not None else None
    vel_h = torch.empty(vel.shape, dtype=torch.float32).pin_memory()
    for k in range(2):
        dit.forward(lat_h, ts_h[k % len(ts_h)], ctx_h, velocity=vel_h, image=img_h)
    dit.sync()
    if world > 1:
        dist.barrier()
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    e2e_steps = args.steps
    for k in range(e2e_steps):
        dit.forward(lat_h, ts_h[k % len(ts_h)], ctx_h, velocity=vel_h, image=img_h)
    e3.record(stream)
    dit.sync()
    ms_e2e = e2.elapsed_time(e3) / e2e_steps
    h2d = lat_h.numel() * lat_h.element_size() + ctx_h.numel() * ctx_h.element_size() + \
        ts_h[0].numel() * ts_h[0].element_size() + (img_h.numel() * img_h.element_size() if img_h is not None else 0)
    d2h = vel_h.numel() * vel_h.element_size()

    ms, ms_e2e = reduce_max([ms, ms_e2e], dev)

    flops = dit.flops(B, F, Hz, Wz, Lc, int(w["timesteps"] == "per_token"), Li)
    # dominant kernel: self-attention, 4 * L^2 * head_dim * heads * B flops per launch
    sa_ms, sa_n = kt["self_attention"]
    sa_flops = 4.0 * L * L * cfg["dim"] * B
    sa_avg_ms = sa_ms / max(1, sa_n)
    achieved = sa_flops / (sa_avg_ms * 1e-3) / 1e12 if sa_n else None
    peak = peaks["bf16_tflops_sustained"]
    result = {
        "metric": METRIC,
        "value": whole_job_tokens_per_s(world, B, L, ms),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic latents/contexts, random-init bf16 weights of the named shapes",
        "config": dict(arm_config(args.workload, world), **({"blocks": args.blocks} if args.blocks else {}),
                       **({} if args.gemm_pair else {"gemm_pair": 0})),
        "tflops_per_step": flops / 1e12,
        "achieved_tflops": flops / (ms * 1e-3) / 1e12,
        "tc_peak_frac": flops / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
        "tc_peak_frac_of": f"{peaks['source']} bf16 {peaks['bf16_tflops']} TFLOP/s (burst)",
        "tc_peak_frac_spec": flops / (ms * 1e-3) / 1e12 / SPEC_BF16_TFLOPS,
        "tc_peak_frac_spec_of": f"dense bf16 spec {SPEC_BF16_TFLOPS} TFLOP/s",
        "roofline": {"kernel": "self-attention (attn_pair_kernel)", "bound": "tensor", "achieved": achieved,
                     "peak": peak, "unit": "TFLOP/s", "frac": (achieved / peak) if achieved else None,
                     "peak_source": f"{peaks['source']} bf16_tflops_sustained (kernel timed inside a long step)",
                     "flops_per_launch": sa_flops, "avg_launch_ms": sa_avg_ms, "launches_per_step": sa_n,
                     # the committed ncu capture is of the default workload's self-attention launch
                     "traffic": measured_traffic("attn_pair_kernel",
                                                 "video_diffusion_transformer_dit_b200/csrc/attention.cu")
                     if args.workload == DEFAULT_WORKLOAD else None,
                     "traffic_unit": "DRAM bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)"},
        "kernel_ms_per_step": {c: v[0] for c, v in kt.items()},
        "gemm_ms_per_step": {c: v[0] for c, v in gemm_parts.items()},
        "e2e": {"value": whole_job_tokens_per_s(world, B, L, ms_e2e), "unit": "tokens/s", "ms_per_step": ms_e2e,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches * args.steps,
        "clocks": clk,
    }
    return result


# ---------------------------------------------------------------- single-kernel mode
KERNELS = ("self_attention", "cross_attention", "gemm_qkv", "gemm_qkv_norm", "gemm_o", "gemm_ffn_up", "gemm_ffn_down",
           "layernorm",
           "rmsnorm_rope", "vae_conv", "vae_decode")


def run_vae(args):
    """Time the Wan2.1 VAE decoder's implicit-GEMM convolution (384 -> 384,
    3x3x3, 2-frame cache, 2 frames at 120x208: the shape of up block 1 at 480p)
    or a whole decode of the 480p latent (21 frames 60x104 -> 81 frames
    480x832), random weights."""
    import torch
    from video_diffusion_transformer_dit_b200 import binding as Bd
    from video_diffusion_transformer_dit_b200 import build
    build.build()
    dev = "cuda"
    g = torch.Generator(device=dev).manual_seed(0)
    if args.kernel == "vae_conv":
        Ci = Co = 384
        T, H, W = 2, 120, 208
        x = torch.randn(1, T, H, W, Ci, generator=g, device=dev).to(torch.bfloat16)
        cache = torch.randn(1, 2, H, W, Ci, generator=g, device=dev).to(torch.bfloat16)
        w = (torch.randn(Co, 27 * Ci, generator=g, device=dev) * 0.02).to(torch.bfloat16)
        bias = torch.zeros(Co, device=dev)
        y = torch.empty(1, T, H, W, Co, dtype=torch.bfloat16, device=dev)
        fn = lambda: Bd.op_conv3d(x, w, bias, y, (3, 3, 3), Co, cache=cache)
        work, unit = 2.0 * T * H * W * Co * 27 * Ci, "TFLOP/s"
        sync = Bd.op_sync
    else:
        from video_diffusion_transformer_dit_b200 import synth
        vae = Bd.WanVAE(max_batch=1, max_h=60, max_w=104)
        vae.load_weights(synth.make_vae_weights(seed=0, device=dev))
        z = torch.randn(1, 16, 21, 60, 104, generator=g, device=dev)
        video = torch.empty(1, 3, 81, 480, 832, device=dev)
        fn = lambda: vae.decode(z, video=video)
        work, unit = 81.0, "frames/s"
        sync = lambda: vae._check(Bd.lib().wan_vae_sync(vae._h, Bd._stream(None)))
    for _ in range(args.warmup):
        fn()
    sync()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        fn()
    e1.record()
    sync()
    ms = e0.elapsed_time(e1) / args.steps
    rate = work / (ms * 1e-3) / (1e12 if unit == "TFLOP/s" else 1.0)
    out = {"kernel": args.kernel, "avg_ms": ms, "achieved": rate, "unit": unit, "launches": args.steps}
    if unit == "TFLOP/s":
        peaks = load_peaks()
        out.update(peak=peaks["bf16_tflops"], frac=rate / peaks["bf16_tflops"], peak_source=peaks["source"] + " (burst)")
    print(json.dumps(out))
    return 0


def run_kernel(args):
    """Time one kernel of the forward alone at the workload's shapes (synthetic
    operands on the device), K timed launches between CUDA events."""
    import torch
    from video_diffusion_transformer_dit_b200 import binding as Bd
    from video_diffusion_transformer_dit_b200 import build, configs
    build.build()
    Bd.op_set_gemm_pair(bool(args.gemm_pair))
    w = configs.workload(args.workload)
    cfg = w["cfg"]
    B, Cc, F, Hz, Wz = w["latent"]
    L, Lc, D, Fd, H = F * (Hz // 2) * (Wz // 2), w["text_len"], cfg["dim"], cfg["ffn_dim"], cfg["heads"]
    R = B * L
    dev = "cuda"
    g = torch.Generator(device=dev).manual_seed(0)

    def rnd(*shape, scale=1.0):
        return (torch.randn(*shape, generator=g, device=dev) * scale).to(torch.bfloat16)

    k = args.kernel
    if k in ("self_attention", "cross_attention"):
        Lk = L if k == "self_attention" else Lc
        qkv = rnd(R, 3 * D)
        kv = rnd(B * Lk, 2 * D)
        o = torch.empty(R, D, dtype=torch.bfloat16, device=dev)
        if k == "self_attention":
            base = qkv.data_ptr()
            fn = lambda: Bd.op_attention_ptr(base, 3 * D, base + 2 * D, 3 * D, base + 4 * D, 3 * D, o.data_ptr(), D,
                                             B, H, L, L)
        else:
            q = rnd(R, D)
            fn = lambda: Bd.op_attention_ptr(q.data_ptr(), D, kv.data_ptr(), 2 * D, kv.data_ptr() + 2 * D, 2 * D,
                                             o.data_ptr(), D, B, H, L, Lk)
        work, unit = 4.0 * L * Lk * D * B, "TFLOP/s"
    elif k.startswith("gemm"):
        N, K_, epi = {"gemm_qkv": (3 * D, D, "bias"), "gemm_qkv_norm": (3 * D, D, "bias"),
                      "gemm_o": (D, D, "gate_residual"),
                      "gemm_ffn_up": (Fd, D, "bias_gelu"), "gemm_ffn_down": (D, Fd, "gate_residual")}[k]
        A = rnd(R, K_)
        Wt = rnd(N, K_, scale=0.02)
        bias = torch.zeros(N, device=dev)
        out = rnd(R, N)
        gate0 = torch.full((N,), 0.1, device=dev)
        gate1 = torch.zeros(B, 6 * N, device=dev)
        fn = lambda: Bd.op_gemm(A, Wt, epi, out, bias=bias, gate0=gate0, gate1=gate1, mod_div=L, mod_ld=6 * N)
        if k == "gemm_qkv_norm":   # q/k gain, RoPE and per-head sums of squares in the epilogue
            gain = torch.ones(2 * D, device=dev)
            ssq = torch.empty(R, 2 * H, device=dev)
            fn = lambda: Bd.op_gemm(A, Wt, "qk_norm", out, bias=bias, gain=gain, ssq=ssq, norm_cols=2 * D,
                                    rope_grid=(F, Hz // 2, Wz // 2))
        work, unit = 2.0 * R * N * K_, "TFLOP/s"
    elif k == "layernorm":
        x = rnd(R, D)
        y = torch.empty_like(x)
        tp = torch.zeros(B, 6 * D, device=dev)
        # mode 2, the block LayerNorms: per-sample scale (1 + scale included) and shift rows
        fn = lambda: Bd.op_layernorm(x, y, 1e-6, 2, shift1=tp[:, 0:D], scale1=tp[:, D:2 * D], mod_div=L,
                                     mod_ld=6 * D)
        work, unit = 2.0 * R * D * 2, "GB/s"
    elif k == "rmsnorm_rope":
        qkv = rnd(R, 3 * D)
        gain = torch.ones(D, device=dev)
        fn = lambda: Bd.op_rmsnorm_rope(qkv.data_ptr(), 3 * D, R, D, 1e-6, gain, rope=True,
                                        grid=(F, Hz // 2, Wz // 2))
        work, unit = 2.0 * R * D * 2, "GB/s"
    else:
        raise SystemExit(f"unknown kernel {k}; one of {KERNELS}")
    for _ in range(args.warmup):
        fn()
    Bd.op_sync()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        fn()
    e1.record()
    Bd.op_sync()
    ms = e0.elapsed_time(e1) / args.steps
    rate = work / (ms * 1e-3) / (1e12 if unit == "TFLOP/s" else 1e9)
    peaks = load_peaks()
    peak = peaks["bf16_tflops"] if unit == "TFLOP/s" else peaks["hbm_gbs"]
    print(json.dumps({"kernel": k, "workload": args.workload, "avg_ms": ms, "achieved": rate, "unit": unit,
                      "peak": peak, "frac": rate / peak, "peak_source": peaks["source"] + " (burst)",
                      "work_per_launch": work, "launches": args.steps}))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=6)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--blocks", type=int, default=None,
                    help="profiling aid: run the workload's shapes with this many blocks (the line then says so "
                         "in config.blocks; not a measurement of the named model)")
    ap.add_argument("--kernel", choices=KERNELS, default=None,
                    help="time one kernel alone at the workload's shapes (profiling aid)")
    ap.add_argument("--gemm-pair", type=int, choices=[0, 1], default=1,
                    help="1: GEMMs with N a multiple of 256 on SM pairs (default); 0: single-SM tiles only")
    args = ap.parse_args()
    if args.kernel in ("vae_conv", "vae_decode"):
        return run_vae(args)
    if args.kernel:
        return run_kernel(args)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        from video_diffusion_transformer_dit_b200 import configs
        import torch
        w = configs.workload(args.workload)
        vals = []
        for k in range(args.warmup + args.steps):
            tok_s, step_s, desc, spent = cpu_sample(w)
            if k >= args.warmup:
                vals.append((tok_s, step_s))
        tok_s = sum(v[0] for v in vals) / len(vals)
        step_s = sum(v[1] for v in vals) / len(vals)
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": tok_s, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": arm_config(args.workload, world),
            "cpu_baseline": {"value": tok_s, "unit": "tokens/s", **host_threads(), "kind": "oracle", "sample": desc},
            "e2e": {"value": tok_s, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }))
        return 0

    import torch
    import torch.distributed as dist
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        res = run_ours(args, rank, world, local_rank)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                w = __import__("video_diffusion_transformer_dit_b200.configs", fromlist=["x"]).workload(args.workload)
                tok_s, step_s, desc, _ = cpu_sample(w)
                res["cpu_baseline"] = {"value": tok_s, "unit": "tokens/s", **host_threads(),
                                       "kind": "oracle", "sample": desc}
            print(json.dumps(res))
    finally:
        if world > 1:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

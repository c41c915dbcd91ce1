"""Thin ctypes binding of libwandit.so (include/wandit.h, include/wandit_ops.h).

Argument marshalling only: every step of the forward runs in the library's
CUDA kernels.  PyTorch tensors are passed by their ``data_ptr()``; streams by
``torch.cuda.current_stream().cuda_stream``.  Loading raises if the library has
not been built (``python -m video_diffusion_transformer_dit_b200.build``):
there is no fallback path.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Dict, Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libwandit.so")

WAN_STATUS = {0: "WAN_OK", 1: "WAN_EINVAL", 2: "WAN_ESHAPE", 3: "WAN_ENOMEM", 4: "WAN_ENOWEIGHTS",
              5: "WAN_EMISSING_WEIGHT", 6: "WAN_EUNEXPECTED_WEIGHT", 7: "WAN_ECUDA", 8: "WAN_ETIMEOUT",
              9: "WAN_EINTERNAL", 10: "WAN_EUNSUPPORTED"}
WAN_DTYPE_F32, WAN_DTYPE_BF16 = 0, 1
WAN_OPT_GRAPH, WAN_OPT_WAIT_LIMIT_NS, WAN_OPT_KERNEL_TIMING, WAN_OPT_GEMM_PAIR = 1, 2, 3, 4
KERNEL_CLASSES = {"patchify": 0, "gemm": 1, "self_attention": 2, "cross_attention": 3, "layernorm": 4,
                  "rmsnorm_rope": 5, "embedding": 6, "gemm_qkv": 7, "gemm_o": 8, "gemm_q2": 9, "gemm_o2": 10,
                  "gemm_ffn_up": 11, "gemm_ffn_down": 12}
BLOCK_GEMMS = ("gemm_qkv", "gemm_o", "gemm_q2", "gemm_o2", "gemm_ffn_up", "gemm_ffn_down")
EPI = {"bias": 0, "bias_gelu": 1, "gate_residual": 2, "residual": 3, "bias_f32": 4, "unpatchify": 5, "qk_norm": 8}

# every symbol include/*.h declares
SYMBOLS = ["wan_dit_create", "wan_dit_load_weights", "wan_dit_missing_weights", "wan_dit_forward", "wan_dit_sync",
           "wan_dit_set_block_dump", "wan_dit_set_option", "wan_dit_kernel_time", "wan_dit_last_launch_count",
           "wan_dit_flops", "wan_dit_forward_image", "wan_dit_flops_image", "wan_moe_select",
           "wan_dit_last_error", "wan_status_string", "wan_dit_destroy",
           "wan_op_gemm", "wan_op_attention", "wan_op_layernorm", "wan_op_rmsnorm_rope", "wan_op_patchify",
           "wan_op_unpatchify", "wan_op_sync", "wan_op_set_wait_limit_ns", "wan_op_rmsnorm_rope_noalloc", "wan_op_cfg_euler",
           "wan_op_wait_selftest", "wan_op_causal_conv3d", "wan_dit_forward_cfg_euler", "wan_flow_sigmas",
           "wan_op_attention_qnorm", "wan_op_rms_apply", "wan_dit_sp_begin", "wan_dit_sp_block_qkv",
           "wan_dit_sp_attention", "wan_dit_sp_block_finish", "wan_dit_sp_end",
           "wan_vae_create", "wan_vae_load_weights", "wan_vae_missing_weights", "wan_vae_decode", "wan_vae_sync",
           "wan_vae_last_error", "wan_vae_destroy", "wan_op_conv3d", "wan_op_set_gemm_pair", "wan_op_gemm_pair_clusters"]


class WanError(RuntimeError):
    def __init__(self, status: int, msg: str = ""):
        self.status = status
        self.name = WAN_STATUS.get(status, str(status))
        super().__init__(f"{self.name}: {msg}")


class wan_dit_config(C.Structure):
    _fields_ = [(n, C.c_int) for n in ("dim", "heads", "head_dim", "ffn_dim", "num_blocks", "in_ch", "out_ch",
                                        "patch_t", "patch_h", "patch_w", "text_dim", "freq_dim",
                                        "rope_t", "rope_h", "rope_w")] + \
              [("eps", C.c_float), ("rope_theta", C.c_float)] + \
              [(n, C.c_int) for n in ("max_batch", "max_tokens", "max_text", "image_dim", "max_image")]


class wan_epilogue(C.Structure):
    _fields_ = [("bias", C.c_void_p), ("out", C.c_void_p), ("ldo", C.c_int64), ("gate0", C.c_void_p),
                ("gate1", C.c_void_p), ("mod_div", C.c_int), ("mod_ld", C.c_int64),
                ("up_C", C.c_int), ("up_F", C.c_int), ("up_Hz", C.c_int), ("up_Wz", C.c_int),
                ("gain", C.c_void_p), ("ssq", C.c_void_p), ("ssq_ld", C.c_int64), ("norm_cols", C.c_int),
                ("rope", C.c_int), ("rope_F", C.c_int), ("rope_H", C.c_int), ("rope_W", C.c_int),
                ("rope_t", C.c_int), ("rope_h", C.c_int), ("rope_w", C.c_int), ("rope_theta", C.c_float)]


_lib = None


def lib() -> C.CDLL:
    """Load libwandit.so (once) and declare its signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise FileNotFoundError(f"{LIB_PATH} is missing: build it with "
                                "`python -m video_diffusion_transformer_dit_b200.build`")
    L = C.CDLL(LIB_PATH)
    P, I, I64, D, F = C.c_void_p, C.c_int, C.c_int64, C.c_double, C.c_float
    sig = {
        "wan_dit_create": (I, [C.POINTER(wan_dit_config), I, C.POINTER(P)]),
        "wan_dit_load_weights": (I, [P, I, C.POINTER(C.c_char_p), C.POINTER(P), C.POINTER(I),
                                     C.POINTER(C.POINTER(I64)), C.POINTER(I), I, P]),
        "wan_dit_missing_weights": (I, [P, C.c_char_p, I]),
        "wan_dit_forward": (I, [P, P, I, I, I, I, I, P, I, P, I, P, I, P]),
        "wan_dit_sync": (I, [P, P]),
        "wan_dit_set_block_dump": (I, [P, P]),
        "wan_dit_set_option": (I, [P, I, I64]),
        "wan_dit_kernel_time": (I, [P, I, C.POINTER(D), C.POINTER(I)]),
        "wan_dit_last_launch_count": (I, [P]),
        "wan_dit_flops": (D, [P, I, I, I, I, I, I]),
        "wan_dit_forward_image": (I, [P, P, I, I, I, I, I, P, I, P, I, P, I, P, I, P]),
        "wan_dit_flops_image": (D, [P, I, I, I, I, I, I, I]),
        "wan_moe_select": (I, [D, D, I]),
        "wan_dit_last_error": (C.c_char_p, [P]),
        "wan_status_string": (C.c_char_p, [I]),
        "wan_dit_destroy": (None, [P]),
        "wan_op_gemm": (I, [P, I64, P, I64, I, I, I, I, C.POINTER(wan_epilogue), P]),
        "wan_op_attention": (I, [P, I64, P, I64, P, I64, P, I64, I, I, I, I, P]),
        "wan_op_layernorm": (I, [P, P, I, I, F, I, P, P, P, P, P, P, I, I64, P]),
        "wan_op_rmsnorm_rope": (I, [P, I64, I, I, F, P, I, I, I, I, I, I, I, F, P]),
        "wan_op_rmsnorm_rope_noalloc": (I, [P, I64, I, I, F, P, I, I, I, I, I, I, I, F, P]),
        "wan_op_patchify": (I, [P, I, I, I, I, I, I, P, P]),
        "wan_op_unpatchify": (I, [P, I, I, I, I, I, P, P]),
        "wan_op_sync": (I, [P]),
        "wan_op_cfg_euler": (I, [P, P, P, F, F, F, I64, P, P]),
        "wan_op_wait_selftest": (I, [I64, P]),
        "wan_op_causal_conv3d": (I, [P, P, I, I, I, I, I, I, P, I64, P, I, I, I, I, P, I64, P, P]),
        "wan_op_set_wait_limit_ns": (None, [I64]),
        "wan_op_set_gemm_pair": (None, [I]),
        "wan_op_gemm_pair_clusters": (I, []),
        "wan_dit_forward_cfg_euler": (I, [P, P, I, I, I, F, P, I, F, F, F, P, I, P]),
        "wan_flow_sigmas": (I, [I, D, C.POINTER(D)]),
        "wan_op_attention_qnorm": (I, [P, I64, P, I64, P, I64, P, I64, I, I, I, I, P, I64, I, F, P]),
        "wan_op_rms_apply": (I, [P, I64, I, I, P, I64, I, F, P]),
        "wan_dit_sp_begin": (I, [P, P, I, I, I, I, I, P, I, P, I, I, I, I, P]),
        "wan_dit_sp_block_qkv": (I, [P, I, P, P]),
        "wan_dit_sp_attention": (I, [P, P, P, P]),
        "wan_dit_sp_block_finish": (I, [P, I, P, P]),
        "wan_dit_sp_end": (I, [P, P, I, P]),
        "wan_vae_create": (I, [I, I, I, I, C.POINTER(P)]),
        "wan_vae_load_weights": (I, [P, I, C.POINTER(C.c_char_p), C.POINTER(P), C.POINTER(I),
                                     C.POINTER(C.POINTER(I64)), C.POINTER(I), I, P]),
        "wan_vae_missing_weights": (I, [P, C.c_char_p, I]),
        "wan_vae_decode": (I, [P, P, I, I, I, I, P, I, P]),
        "wan_vae_sync": (I, [P, P]),
        "wan_vae_last_error": (C.c_char_p, [P]),
        "wan_vae_destroy": (None, [P]),
        "wan_op_conv3d": (I, [P, P, I, I, I, I, I, I, P, I64, P, I, I, I, I, I, P, I64, P, I64, I, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream=None) -> Optional[int]:
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    return torch.cuda.current_stream().cuda_stream


def _check(status: int, msg: str = ""):
    if status != 0:
        raise WanError(status, msg)


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float32:
        return WAN_DTYPE_F32
    if t.dtype == torch.bfloat16:
        return WAN_DTYPE_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def make_config(cfg: dict, max_batch: int, max_tokens: int, max_text: int, max_image: int = 0) -> wan_dit_config:
    c = wan_dit_config()
    for k in ("dim", "heads", "head_dim", "ffn_dim", "num_blocks", "in_ch", "out_ch", "text_dim", "freq_dim"):
        setattr(c, k, int(cfg[k]))
    c.patch_t, c.patch_h, c.patch_w = (int(v) for v in cfg["patch"])
    c.rope_t, c.rope_h, c.rope_w = (int(v) for v in cfg["rope_split"])
    c.eps = float(cfg["eps"])
    c.rope_theta = float(cfg["rope_theta"])
    c.max_batch, c.max_tokens, c.max_text = int(max_batch), int(max_tokens), int(max_text)
    c.image_dim = int(cfg.get("image_dim", 0))
    c.max_image = int(max_image) if c.image_dim else 0
    return c


class WanDiT:
    """Handle of ``wan_dit``: create / load_weights / forward / sync / destroy."""

    def __init__(self, cfg: dict, max_batch: int, max_tokens: int, max_text: int, device: int = 0,
                 max_image: int = 257):
        self.cfg = dict(cfg)
        self._h = C.c_void_p()
        c = make_config(cfg, max_batch, max_tokens, max_text, max_image)
        _check(lib().wan_dit_create(C.byref(c), int(device), C.byref(self._h)), "wan_dit_create")

    # -- lifetime
    def close(self):
        if self._h:
            lib().wan_dit_destroy(self._h)
            self._h = C.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def last_error(self) -> str:
        return lib().wan_dit_last_error(self._h).decode()

    def _check(self, status):
        if status != 0:
            raise WanError(status, self.last_error())

    # -- weights
    def load_weights(self, weights: Dict[str, "object"], stream=None):
        """Load a dict name -> torch tensor (f32 or bf16, CPU or CUDA, contiguous)."""
        items = list(weights.items())
        if not items:
            return
        on_dev = items[0][1].is_cuda
        keep = [t.contiguous() for _, t in items]
        if any(t.is_cuda != on_dev for t in keep):
            raise ValueError("all tensors of one load call must be on the same side (host or device)")
        n = len(items)
        names = (C.c_char_p * n)(*[k.encode() for k, _ in items])
        ptrs = (C.c_void_p * n)(*[t.data_ptr() for t in keep])
        dts = (C.c_int * n)(*[_dtype_code(t) for t in keep])
        shape_arrs = [(C.c_int64 * max(1, t.dim()))(*t.shape) for t in keep]
        shapes = (C.POINTER(C.c_int64) * n)(*[C.cast(a, C.POINTER(C.c_int64)) for a in shape_arrs])
        nd = (C.c_int * n)(*[t.dim() for t in keep])
        st = _stream(stream) if on_dev else None
        self._check(lib().wan_dit_load_weights(self._h, n, names, ptrs, dts, shapes, nd, int(on_dev), st))

    def missing_weights(self):
        buf = C.create_string_buffer(1 << 16)
        n = lib().wan_dit_missing_weights(self._h, buf, len(buf))
        return n, buf.value.decode()

    # -- forward
    def forward(self, latent, timestep, context, velocity=None, stream=None, sync=False, image=None):
        """latent [B,C,F,Hz,Wz] f32/bf16, timestep f32 [B] or [B,L], context bf16
        [B,Lc,text_dim], image (I2V models) bf16 [B,Li,image_dim] or None.  All
        CUDA tensors (device I/O) or all CPU tensors (host I/O, copies inside the
        call).  Returns the velocity tensor."""
        import torch
        B, Cin, F, Hz, Wz = latent.shape
        Lc = context.shape[1]
        per_token = int(timestep.dim() == 2)
        on_dev = latent.is_cuda
        if velocity is None:
            velocity = torch.empty(B, self.cfg["out_ch"], F, Hz, Wz, dtype=torch.float32, device=latent.device,
                                   pin_memory=not on_dev)
        st = _stream(stream)
        if image is None:
            self._check(lib().wan_dit_forward(self._h, _ptr(latent), _dtype_code(latent), B, F, Hz, Wz,
                                              _ptr(timestep), per_token, _ptr(context), Lc, _ptr(velocity),
                                              int(on_dev), st))
        else:
            self._check(lib().wan_dit_forward_image(self._h, _ptr(latent), _dtype_code(latent), B, F, Hz, Wz,
                                                    _ptr(timestep), per_token, _ptr(context), Lc, _ptr(image),
                                                    image.shape[1], _ptr(velocity), int(on_dev), st))
        if sync:
            self.sync(stream)
        return velocity

    def forward_cfg_euler(self, x, timestep: float, context, guidance: float, sigma: float, sigma_next: float,
                          x_next=None, stream=None, sync=False):
        """One fused sampler step of the CFG pair: x f32 [1,C,F,Hz,Wz], context bf16
        [2,Lc,text_dim] (conditional, unconditional).  Returns x_next (new tensor unless
        given; may be x itself).  CUDA tensors for device I/O, CPU tensors for host I/O."""
        import torch
        _, Cin, F, Hz, Wz = x.shape
        on_dev = x.is_cuda
        if x_next is None:
            x_next = torch.empty(x.shape, dtype=torch.float32, device=x.device, pin_memory=not on_dev)
        self._check(lib().wan_dit_forward_cfg_euler(self._h, _ptr(x), F, Hz, Wz, float(timestep), _ptr(context),
                                                    context.shape[1], float(guidance), float(sigma),
                                                    float(sigma_next), _ptr(x_next), int(on_dev), _stream(stream)))
        if sync:
            self.sync(stream)
        return x_next

    def sync(self, stream=None):
        self._check(lib().wan_dit_sync(self._h, _stream(stream)))

    def set_block_dump(self, dst):
        self._check(lib().wan_dit_set_block_dump(self._h, _ptr(dst)))

    def set_option(self, option: int, value: int):
        self._check(lib().wan_dit_set_option(self._h, option, int(value)))

    def kernel_time(self, kernel_class: str):
        """(total ms, launches) of one kernel class in the last timed forward."""
        ms, n = C.c_double(), C.c_int()
        self._check(lib().wan_dit_kernel_time(self._h, KERNEL_CLASSES[kernel_class], C.byref(ms), C.byref(n)))
        return ms.value, n.value

    def last_launch_count(self) -> int:
        return lib().wan_dit_last_launch_count(self._h)

    def flops(self, B, F, Hz, Wz, Lc, per_token=0, Li=0) -> float:
        return lib().wan_dit_flops_image(self._h, B, F, Hz, Wz, Lc, per_token, Li)


def flow_sigmas(steps: int, shift: float):
    """steps + 1 flow-shifted noise levels from 1 down to 0 (wan_flow_sigmas)."""
    out = (C.c_double * (steps + 1))()
    _check(lib().wan_flow_sigmas(int(steps), float(shift), out), "wan_flow_sigmas")
    return list(out)


def _weight_arrays(weights):
    """ctypes arrays of names, pointers, dtypes and shapes of a name -> tensor dict."""
    items = list(weights.items())
    on_dev = items[0][1].is_cuda
    keep = [t.contiguous() for _, t in items]
    if any(t.is_cuda != on_dev for t in keep):
        raise ValueError("all tensors of one load call must be on the same side (host or device)")
    n = len(items)
    names = (C.c_char_p * n)(*[k.encode() for k, _ in items])
    ptrs = (C.c_void_p * n)(*[t.data_ptr() for t in keep])
    dts = (C.c_int * n)(*[_dtype_code(t) for t in keep])
    shape_arrs = [(C.c_int64 * max(1, t.dim()))(*t.shape) for t in keep]
    shapes = (C.POINTER(C.c_int64) * n)(*[C.cast(a, C.POINTER(C.c_int64)) for a in shape_arrs])
    nd = (C.c_int * n)(*[t.dim() for t in keep])
    return n, names, ptrs, dts, shapes, nd, on_dev, (keep, shape_arrs)


class WanVAE:
    """Handle of ``wan_vae`` (include/wanvae.h): the Wan2.1 VAE decoder."""

    def __init__(self, max_batch: int, max_h: int, max_w: int, device: int = 0):
        self._h = C.c_void_p()
        _check(lib().wan_vae_create(int(device), int(max_batch), int(max_h), int(max_w), C.byref(self._h)),
               "wan_vae_create")

    def close(self):
        if self._h:
            lib().wan_vae_destroy(self._h)
            self._h = C.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _check(self, status):
        if status != 0:
            raise WanError(status, lib().wan_vae_last_error(self._h).decode())

    def load_weights(self, weights: Dict[str, "object"], stream=None):
        if not weights:
            return
        n, names, ptrs, dts, shapes, nd, on_dev, _keep = _weight_arrays(weights)
        self._check(lib().wan_vae_load_weights(self._h, n, names, ptrs, dts, shapes, nd, int(on_dev),
                                               _stream(stream) if on_dev else None))

    def missing_weights(self):
        buf = C.create_string_buffer(1 << 16)
        n = lib().wan_vae_missing_weights(self._h, buf, len(buf))
        return n, buf.value.decode()

    def decode(self, z, video=None, stream=None, sync=False):
        """z f32 [B, 16, T, H, W] (CUDA or CPU) -> video f32 [B, 3, 1 + 4 (T - 1), 8 H, 8 W]."""
        import torch
        B, _, T, H, W = z.shape
        on_dev = z.is_cuda
        if video is None:
            video = torch.empty(B, 3, 1 + 4 * (T - 1), 8 * H, 8 * W, dtype=torch.float32, device=z.device,
                                pin_memory=not on_dev)
        self._check(lib().wan_vae_decode(self._h, _ptr(z), B, T, H, W, _ptr(video), int(on_dev), _stream(stream)))
        if sync:
            self._check(lib().wan_vae_sync(self._h, _stream(stream)))
        return video


def op_conv3d(x, w_packed, bias, y, kernel, Co, cache=None, add=None, time_split=False, stream=None):
    """Implicit-GEMM causal Conv3d: x bf16 [B,T,H,W,Ci] (channels last), w_packed bf16
    [Co_pad, ldw] ((kt,kh,kw,ci) order, ci padded to a multiple of 64), y bf16 rows with
    channel stride y.shape[-1], cache [B,nc,H,W,Ci] or None, add residual or None."""
    B, T, H, W, Ci = x.shape
    kt, kh, kw = kernel
    nc = 0 if cache is None else cache.shape[1]
    _check(lib().wan_op_conv3d(_ptr(x), _ptr(cache), nc, B, T, H, W, Ci, _ptr(w_packed), w_packed.stride(0),
                               _ptr(bias), Co, w_packed.shape[0], kt, kh, kw, _ptr(y), y.shape[-1], _ptr(add),
                               0 if add is None else add.shape[-1], int(time_split), _stream(stream)), "wan_op_conv3d")


def moe_select(t: float, boundary: float, num_train_timesteps: int = 1000) -> int:
    """0 (high-noise expert) when t >= boundary * num_train_timesteps, else 1."""
    return lib().wan_moe_select(float(t), float(boundary), int(num_train_timesteps))


class WanMoE:
    """Two-expert route (Wan2.2 A14B): one ``WanDiT`` handle per expert and the
    timestep switch of ``wan_moe_select``; a step's forwards (both CFG branches)
    all run on the expert its timestep selects."""

    def __init__(self, high_noise: WanDiT, low_noise: WanDiT, boundary: float, num_train_timesteps: int = 1000):
        self.experts = (high_noise, low_noise)
        self.boundary = float(boundary)
        self.num_train_timesteps = int(num_train_timesteps)

    def expert(self, timestep) -> int:
        """Expert index of a per-sample timestep tensor [B] (all entries equal)."""
        t = timestep.detach().float().cpu()
        if t.dim() != 1 or not bool((t == t[0]).all()):
            raise ValueError("the expert switch takes one per-sample timestep shared by the batch")
        return moe_select(float(t[0]), self.boundary, self.num_train_timesteps)

    def forward(self, latent, timestep, context, **kw):
        return self.experts[self.expert(timestep)].forward(latent, timestep, context, **kw)


# ---------------------------------------------------------------- op-level wrappers
def op_gemm(A, W, epilogue: str, out, bias=None, gate0=None, gate1=None, mod_div=1, mod_ld=0,
            unpatch=(0, 0, 0, 0), M=None, stream=None, gain=None, ssq=None, norm_cols=0, rope_grid=None,
            rope_split=(44, 42, 42), rope_theta=10000.0):
    M = A.shape[0] if M is None else M
    N, K = W.shape
    rg = rope_grid or (0, 0, 0)
    e = wan_epilogue(bias=_ptr(bias), out=_ptr(out), ldo=(out.stride(0) if out.dim() == 2 else 0),
                     gate0=_ptr(gate0), gate1=_ptr(gate1), mod_div=mod_div, mod_ld=mod_ld,
                     up_C=unpatch[0], up_F=unpatch[1], up_Hz=unpatch[2], up_Wz=unpatch[3],
                     gain=_ptr(gain), ssq=_ptr(ssq), ssq_ld=(ssq.stride(0) if ssq is not None else 0),
                     norm_cols=norm_cols, rope=int(rope_grid is not None), rope_F=rg[0], rope_H=rg[1], rope_W=rg[2],
                     rope_t=rope_split[0], rope_h=rope_split[1], rope_w=rope_split[2], rope_theta=rope_theta)
    _check(lib().wan_op_gemm(_ptr(A), A.stride(0), _ptr(W), W.stride(0), M, N, K, EPI[epilogue], C.byref(e),
                             _stream(stream)), "wan_op_gemm")


def op_causal_conv3d(x, w_packed, bias, col, y, kernel, cache=None, stream=None):
    """x bf16 [B,T,H,W,Ci], w_packed bf16 [Co, ldw] ((kt,kh,kw,ci) order, zero padded
    to ldw), bias f32 [Co] or None, col bf16 workspace, y bf16 [B,T,H,W,Co],
    kernel (kt, kh, kw), cache bf16 [B,nc,H,W,Ci] or None (channels last)."""
    B, T, H, W, Ci = x.shape
    Co = w_packed.shape[0]
    kt, kh, kw = kernel
    nc = 0 if cache is None else cache.shape[1]
    _check(lib().wan_op_causal_conv3d(_ptr(x), _ptr(cache), nc, B, T, H, W, Ci, _ptr(w_packed), w_packed.stride(0),
                                      _ptr(bias), Co, kt, kh, kw, _ptr(col), col.numel(), _ptr(y), _stream(stream)),
           "wan_op_causal_conv3d")


def op_attention(q, k, v, o, B, heads, Lq, Lk, ldq=None, ldk=None, ldv=None, ldo=None, stream=None):
    _check(lib().wan_op_attention(_ptr(q), ldq or q.stride(0), _ptr(k), ldk or k.stride(0), _ptr(v),
                                  ldv or v.stride(0), _ptr(o), ldo or o.stride(0), B, heads, Lq, Lk,
                                  _stream(stream)), "wan_op_attention")


def op_attention_qnorm(q_ptr, ldq, k_ptr, ldk, v_ptr, ldv, o, B, heads, Lq, Lk, q_ssq, ngroups, eps, stream=None):
    """Attention with unnormalised queries scaled by their RMSNorm row factors."""
    _check(lib().wan_op_attention_qnorm(q_ptr, ldq, k_ptr, ldk, v_ptr, ldv, _ptr(o), o.stride(0), B, heads, Lq, Lk,
                                        _ptr(q_ssq), q_ssq.stride(0), ngroups, eps, _stream(stream)),
           "wan_op_attention_qnorm")


def op_rms_apply(buf_ptr, ld, rows, D, ssq_ptr, ssq_ld, ngroups, eps, stream=None):
    _check(lib().wan_op_rms_apply(buf_ptr, ld, rows, D, ssq_ptr, ssq_ld, ngroups, eps, _stream(stream)),
           "wan_op_rms_apply")


def op_attention_ptr(q, ldq, k, ldk, v, ldv, o, ldo, B, heads, Lq, Lk, stream=None):
    _check(lib().wan_op_attention(q, ldq, k, ldk, v, ldv, o, ldo, B, heads, Lq, Lk, _stream(stream)),
           "wan_op_attention")


def op_layernorm(x, y, eps, mode, gamma=None, beta=None, shift0=None, shift1=None, scale0=None, scale1=None,
                 mod_div=1, mod_ld=0, stream=None):
    rows, D = x.shape
    _check(lib().wan_op_layernorm(_ptr(x), _ptr(y), rows, D, eps, mode, _ptr(gamma), _ptr(beta), _ptr(shift0),
                                  _ptr(shift1), _ptr(scale0), _ptr(scale1), mod_div, mod_ld, _stream(stream)),
           "wan_op_layernorm")


def op_rmsnorm_rope(buf_ptr, ld, rows, D, eps, gain, rope=False, grid=(0, 0, 0), split=(44, 42, 42),
                    theta=10000.0, stream=None):
    _check(lib().wan_op_rmsnorm_rope(buf_ptr, ld, rows, D, eps, _ptr(gain), int(rope), grid[0], grid[1], grid[2],
                                     split[0], split[1], split[2], theta, _stream(stream)), "wan_op_rmsnorm_rope")


def op_rmsnorm_rope_noalloc(buf_ptr, ld, rows, D, eps, gain, rope=True, grid=(0, 0, 0), split=(44, 42, 42),
                            theta=10000.0, stream=None):
    """wan_op_rmsnorm_rope without any device allocation (fixed 1024-position table)."""
    _check(lib().wan_op_rmsnorm_rope_noalloc(buf_ptr, ld, rows, D, eps, _ptr(gain), int(rope), grid[0], grid[1],
                                             grid[2], split[0], split[1], split[2], theta, _stream(stream)),
           "wan_op_rmsnorm_rope_noalloc")


def op_patchify(latent, X, stream=None):
    B, Cc, F, Hz, Wz = latent.shape
    _check(lib().wan_op_patchify(_ptr(latent), _dtype_code(latent), B, Cc, F, Hz, Wz, _ptr(X), _stream(stream)),
           "wan_op_patchify")


def op_unpatchify(rows, vel, stream=None):
    B, Cc, F, Hz, Wz = vel.shape
    _check(lib().wan_op_unpatchify(_ptr(rows), B, Cc, F, Hz, Wz, _ptr(vel), _stream(stream)), "wan_op_unpatchify")


def op_cfg_euler(x, v_cond, v_uncond, guidance, sigma, sigma_next, out, stream=None):
    """out = x + (sigma_next - sigma) * (v_uncond + guidance * (v_cond - v_uncond)); f32 CUDA tensors."""
    _check(lib().wan_op_cfg_euler(_ptr(x), _ptr(v_cond), _ptr(v_uncond), guidance, sigma, sigma_next, x.numel(),
                                  _ptr(out), _stream(stream)), "wan_op_cfg_euler")


def op_wait_selftest(limit_ns, stream=None):
    _check(lib().wan_op_wait_selftest(int(limit_ns), _stream(stream)), "wan_op_wait_selftest")


def op_sync(stream=None):
    _check(lib().wan_op_sync(_stream(stream)), "wan_op_sync")


def op_set_wait_limit_ns(ns: int):
    lib().wan_op_set_wait_limit_ns(int(ns))


def op_set_gemm_pair(on: bool):
    """op_gemm on SM-pair (cta_group::2) tiles where it applies, or always single-SM."""
    lib().wan_op_set_gemm_pair(1 if on else 0)


def op_gemm_pair_clusters() -> int:
    """Two-CTA clusters the SM-pair GEMM runs with on this device (0: unavailable)."""
    n = lib().wan_op_gemm_pair_clusters()
    if n < 0:
        raise WanError(7, "wan_op_gemm_pair_clusters")
    return n

/*
 * wanvae.h -- C ABI of the Wan2.1 VAE decoder in libwandit.so (latent video
 * -> RGB frames) on one NVIDIA B200 (sm_100a).
 *
 * Follows the decoder walk-through of the pswp.cn notes on diffusers
 * WanPipeline (sections "vae.decode", "WanDecoder3d", "WanCausalConv3d" and
 * "upsample blocks"): a 1x1x1 post_quant_conv on the latent, then the decoder
 * run one latent frame at a time with a cache of the last 2 input frames of
 * every causal convolution (33 of them), the per-frame outputs joined on the
 * time axis and clamped to [-1, 1].  Decoder: conv_in (z_dim 16 -> 384), mid
 * block (residual block, single-head spatial attention, residual block), four
 * up blocks of three residual blocks each (widths 384, 384, 192, 96), time +
 * spatial upsampling after blocks 0 and 1 (time_conv (3,1,1) doubling the
 * channels into two frames, nearest 2x and a 3x3 conv halving them), spatial
 * only after block 2, then RMS norm, SiLU, conv_out (96 -> 3).
 * Readings where the pages are silent: channel RMS norm with gain and bias
 * (eps 1e-12); residual block h = conv2(SiLU(norm2(conv1(SiLU(norm1 x))))) +
 * shortcut(x); time_conv channel half k -> frame 2t + k; the first latent
 * frame is not time-upsampled (21 latent frames -> 81 video frames) and
 * time_conv's cache starts after it.
 *
 * On the GPU every convolution is an implicit GEMM on the tensor cores (the
 * causal taps gathered by 5-D TMA copies from channels-last activations or the
 * frame cache); the norms, the upsampling and the attention softmax are
 * bandwidth kernels; the attention products are the library's GEMMs.
 * Conventions as in wandit.h (status codes, last_error, stream as void*).
 */
#ifndef WANVAE_H
#define WANVAE_H

#include <stdint.h>
#include "wandit.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct wan_vae wan_vae; /* opaque handle */

/* Create a decoder on CUDA device `device` with workspace for latents of up to
 * max_batch x max_h x max_w (latent pixels; the video is 8x larger on each
 * side).  Synchronous.  WAN_ENOMEM if the workspace does not fit.            */
WANDIT_API wan_status wan_vae_create(int device, int max_batch, int max_h, int max_w, wan_vae** out);

/* Load named parameters (the diffusers AutoencoderKLWan decoder names:
 * post_quant_conv.*, decoder.conv_in.*, decoder.mid_block.{resnets.0|1,
 * attentions.0}.*, decoder.up_blocks.{i}.{resnets.{r}, upsamplers.0}.*,
 * decoder.norm_out.*, decoder.conv_out.*; norms carry .gamma and .bias).
 * Arguments as wan_dit_load_weights; the library repacks every convolution
 * into its K-major implicit-GEMM layout and synchronises `stream`.           */
WANDIT_API wan_status wan_vae_load_weights(wan_vae* v, int n, const char* const* names, const void* const* ptrs,
                                           const int* dtypes, const int64_t* const* shapes, const int* ndims,
                                           int ptrs_on_device, void* stream);

/* Names the decoder still expects (count; comma-separated list into buf). */
WANDIT_API int wan_vae_missing_weights(const wan_vae* v, char* buf, int len);

/* Decode a latent video.
 *   z      float [B, 16, T, H, W]   (T latent frames)
 *   video  float [B, 3, 1 + 4 (T - 1), 8 H, 8 W], values in [-1, 1]
 * Device pointers when io_on_device != 0, host pointers otherwise (copies in
 * stream order).  B <= max_batch, H <= max_h, W <= max_w.  Asynchronous on
 * `stream`; the frame loop issues every launch eagerly.                     */
WANDIT_API wan_status wan_vae_decode(wan_vae* v, const float* z, int B, int T, int H, int W, float* video,
                                     int io_on_device, void* stream);

/* Synchronise `stream`; WAN_ETIMEOUT if a kernel's bounded wait ran out.     */
WANDIT_API wan_status wan_vae_sync(wan_vae* v, void* stream);
WANDIT_API const char* wan_vae_last_error(const wan_vae* v);
WANDIT_API void wan_vae_destroy(wan_vae* v);

/* Causal 3-D convolution as an implicit GEMM (the decoder's convolutions,
 * exposed for kernel-level checks).  Channels-last bf16 device tensors:
 *   x      [B, T, H, W, Ci]; cache [B, nc, H, W, Ci] (the nc <= kt-1 frames
 *          right before frame 0) or NULL
 *   w      [Co_pad, ldw] bf16, row co = W[co, ci, it, ih, iw] in (it, ih, iw, ci)
 *          order with ci zero-padded to a multiple of 64 (ldw >= kt*kh*kw*Cip)
 *   bias   f32 [Co] or NULL
 *   y      [B, T, H, W, ldy] (time_split: [B, 2T, H, W, ldy])
 *   add    residual [B, T, H, W, ldadd] added before rounding, or NULL
 *   time_split != 0: Co = 2 C output channels, half k of frame t -> frame 2t + k
 * Requirements: Ci % 8 == 0, odd kernel sizes, Co_pad % 64 == 0.            */
WANDIT_API wan_status wan_op_conv3d(const void* x, const void* cache, int nc, int B, int T, int H, int W, int Ci,
                                    const void* w, int64_t ldw, const float* bias, int Co, int Co_pad, int kt, int kh,
                                    int kw, void* y, int64_t ldy, const void* add, int64_t ldadd, int time_split,
                                    void* stream);

#ifdef __cplusplus
}
#endif
#endif /* WANVAE_H */

/*
 * wandit.h -- C ABI of libwandit.so: one denoising-step forward of the Wan DiT
 * (Wan2.1 / Wan2.2 video diffusion transformer) on one NVIDIA B200 (sm_100a).
 *
 * The forward follows the diffusers WanTransformer3DModel / WanTransformerBlock
 * forward printed in the pswp.cn notes on WanPipeline (sections
 * "WanTransformer3DModel" and "WanTransformerBlock"):
 *   patchify by a (1,2,2) Conv3d into L = F * Hz/2 * Wz/2 tokens;
 *   sinusoidal timestep embedding -> temb and a shared 6-way modulation,
 *   plus a per-block scale_shift_table;
 *   N blocks of: modulated LayerNorm, self-attention with q/k RMSNorm across
 *   heads and 3-axis (T/H/W) RoPE, gated residual; affine LayerNorm,
 *   cross-attention to the projected text context, residual; modulated
 *   LayerNorm, GELU-tanh FFN, gated residual;
 *   FP32 output LayerNorm, scale-shift, proj_out and unpatchify -> velocity.
 * Configuration defaults come from the "配置参数全解" table of
 * "Diffusers 中 WanAnimateTransformer3DModel 深度解析" (head_dim 128, text_dim
 * 4096, freq_dim 256, eps 1e-6, qk_norm rms_norm_across_heads,
 * cross_attn_norm True) and the model-size table of
 * "【VLA与模仿学习】Wan2.1框架与训练源码导读" §10.
 *
 * Conventions for every entry point:
 *   - Pointers are plain addresses.  "device" pointers are CUDA device
 *     addresses on the handle's device; "host" pointers are CPU addresses
 *     (page-locked memory is recommended for speed, pageable works).
 *   - `stream` is a cudaStream_t passed as void*; NULL means the legacy default
 *     stream.  Calls are asynchronous on that stream unless stated otherwise.
 *   - The caller owns every buffer it passes; the library never frees them and
 *     never keeps a caller pointer past the call (it copies into its own
 *     staging buffers inside the stream order).
 *   - Every call returns a wan_status.  On failure nothing is launched for
 *     shape/argument errors; wan_dit_last_error() gives a one-line reason.
 *   - Kernels never wait forever: every on-chip wait has a time limit; when a
 *     limit runs out the kernel records WAN_ETIMEOUT in a device flag, drains
 *     its own copies, frees its tensor memory and returns.  wan_dit_sync()
 *     reports the flag.
 */
#ifndef WANDIT_H
#define WANDIT_H

#include <stdint.h>

#if defined(__GNUC__)
#define WANDIT_API __attribute__((visibility("default")))
#else
#define WANDIT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct wan_dit wan_dit; /* opaque handle */

typedef enum {
    WAN_OK = 0,
    WAN_EINVAL = 1,             /* null pointer or out-of-range argument       */
    WAN_ESHAPE = 2,             /* tensor shape does not fit the model/limits   */
    WAN_ENOMEM = 3,             /* device allocation failed at create/load      */
    WAN_ENOWEIGHTS = 4,         /* forward before any weights were loaded       */
    WAN_EMISSING_WEIGHT = 5,    /* a required parameter was never loaded        */
    WAN_EUNEXPECTED_WEIGHT = 6, /* a name the model does not have               */
    WAN_ECUDA = 7,              /* a CUDA runtime call failed                   */
    WAN_ETIMEOUT = 8,           /* a kernel's bounded on-chip wait ran out      */
    WAN_EINTERNAL = 9,
    WAN_EUNSUPPORTED = 10       /* valid config the kernels do not support      */
} wan_status;

enum { WAN_DTYPE_F32 = 0, WAN_DTYPE_BF16 = 1 };

/* Model dimensions and workspace limits.
 *   dim        model width D (multiple of 256), heads * head_dim == dim
 *   head_dim   must be 128 (attention_head_dim of every Wan model)
 *   ffn_dim    FFN hidden width (multiple of 64)
 *   num_blocks number of WanTransformerBlocks (30 for 1.3B/5B, 40 for 14B)
 *   in_ch/out_ch latent channels in and out (16 for the Wan2.1 VAE, 48 for
 *              Wan2.2-5B; in_ch 36 = 16 noisy + 16 condition + 4 mask channels
 *              for the I2V route, "I2V分量" table of the Wan2.1 source guide)
 *   patch_t/h/w patch size; only (1,2,2) is supported
 *   text_dim   context width (4096, umT5), multiple of 64
 *   freq_dim   timestep sinusoid width (256)
 *   rope_t/h/w head-dim split of the 3-axis RoPE (44/42/42), even, sum = head_dim
 *   eps        LayerNorm / RMSNorm epsilon (1e-6)
 *   rope_theta RoPE base (1e4)
 *   max_batch, max_tokens, max_text   workspace limits fixed at create
 *   image_dim  width of the image (CLIP) tokens of the I2V route (1280), a
 *              multiple of 64; 0 = no image branch (text-to-video models)
 *   max_image  workspace limit on image tokens per sample (257 for CLIP);
 *              ignored when image_dim is 0                                  */
typedef struct {
    int dim, heads, head_dim, ffn_dim, num_blocks;
    int in_ch, out_ch, patch_t, patch_h, patch_w;
    int text_dim, freq_dim;
    int rope_t, rope_h, rope_w;
    float eps, rope_theta;
    int max_batch, max_tokens, max_text;
    int image_dim, max_image;
} wan_dit_config;

/* Create a handle on CUDA device `device` and allocate its workspace for
 * max_batch * max_tokens tokens and max_batch * max_text context rows.
 * Synchronous.  Returns WAN_EUNSUPPORTED for dims the kernels do not cover,
 * WAN_ENOMEM if the workspace does not fit.  *out is NULL on failure.       */
WANDIT_API wan_status wan_dit_create(const wan_dit_config* cfg, int device, wan_dit** out);

/* Load (or replace) `n` named parameters.  Names and shapes are the
 * diffusers ones (patch_embedding.weight [D,C,1,2,2], condition_embedder.*,
 * blocks.{i}.{scale_shift_table, attn1.*, attn2.*, norm2.*, ffn.net.*},
 * scale_shift_table [1,2,D], proj_out.*).  ptrs[i] points at a dense
 * row-major tensor of dtype dtypes[i] (WAN_DTYPE_F32 or WAN_DTYPE_BF16) with
 * ndims[i] dimensions shapes[i][0..ndims[i]-1]; it is a device pointer when
 * ptrs_on_device != 0, else a host pointer.  The library converts and repacks
 * into its own layouts and synchronises `stream` before returning, so the
 * caller may free its buffers afterwards.  Unknown names give
 * WAN_EUNEXPECTED_WEIGHT and shape mismatches WAN_ESHAPE (the first offending
 * name is in last_error); the other names of the call are still loaded.     */
WANDIT_API wan_status wan_dit_load_weights(wan_dit* h, int n, const char* const* names,
                                const void* const* ptrs, const int* dtypes,
                                const int64_t* const* shapes, const int* ndims,
                                int ptrs_on_device, void* stream);

/* Number of parameters the model still expects; with buf != NULL writes a
 * comma-separated list of up to `len`-1 bytes of the missing names.         */
WANDIT_API int wan_dit_missing_weights(const wan_dit* h, char* buf, int len);

/* One denoising-step forward.
 *   latent    [B, in_ch, F, Hz, Wz], latent_dtype F32 or BF16
 *   timestep  float [B] (per_token = 0) or [B, L] (per_token = 1), L = F*Hz/2*Wz/2
 *   context   bf16 [B, Lc, text_dim]
 *   velocity  float [B, out_ch, F, Hz, Wz] (output; holds bf16-rounded values)
 * All four are device pointers when io_on_device != 0, host pointers
 * otherwise (then the host->device and device->host copies run inside the
 * call, in stream order; host buffers must stay valid until the stream
 * reaches the end of the call).  Hz and Wz must be even, B <= max_batch,
 * L <= max_tokens, Lc <= max_text.  The first call per shape builds and
 * captures the launch plan (synchronous); later calls replay it.           */
WANDIT_API wan_status wan_dit_forward(wan_dit* h, const void* latent, int latent_dtype,
                           int B, int F, int Hz, int Wz,
                           const float* timestep, int per_token,
                           const void* context, int Lc,
                           float* velocity, int io_on_device, void* stream);

/* The I2V forward (Wan2.1-I2V / Wan2.2-I2V route): as wan_dit_forward, with
 *   latent    [B, in_ch, F, Hz, Wz], in_ch = 36 for the I2V models: noisy
 *             latent, first-frame condition latent and known-frame mask joined
 *             on the channel axis
 *   image     bf16 [B, Li, image_dim] image tokens (CLIP, Li = 257), device or
 *             host pointer like the other buffers; 1 <= Li <= max_image
 * The image tokens pass the image embedder (two linears around GELU_tanh) and,
 * in every block, a separate attention with their own key/value projections
 * (blocks.{i}.attn2.add_k_proj / add_v_proj, keys RMSNorm'd across heads with
 * attn2.norm_added_k) whose output is added to the text attention output
 * before attn2.to_out (the model forward of the diffusers notes joins the
 * image tokens in front of the text tokens; the Wan2.1 guide's §4 gives the
 * CLIP condition its own image cross-attention).  image == NULL runs the text
 * branch alone.  WAN_EINVAL if the model has no image branch (image_dim 0). */
WANDIT_API wan_status wan_dit_forward_image(wan_dit* h, const void* latent, int latent_dtype,
                           int B, int F, int Hz, int Wz,
                           const float* timestep, int per_token,
                           const void* context, int Lc,
                           const void* image, int Li,
                           float* velocity, int io_on_device, void* stream);

/* One flow-matching sampler step of a classifier-free-guided run, fused into
 * the forward ("【VLA与模仿学习】Wan2.1框架与训练源码导读" §7: the CFG combination
 * v = v_u + s (v_c - v_u) of the conditional and unconditional predictions and
 * the Euler update x_next = x + (sigma_next - sigma) v; the flow-shifted noise
 * levels come from wan_flow_sigmas).  Runs the B = 2 forward of the same
 * latent with two contexts and, in the proj_out epilogue, combines each
 * token's two velocity rows (each rounded to bf16, as wan_dit_forward returns
 * them) and writes the updated latent -- the two velocities never reach memory.
 *   x         float [1, in_ch, F, Hz, Wz] sampler state (the latent)
 *   timestep  the DiT timestep of this step (both samples)
 *   context   bf16 [2, Lc, text_dim]: row block 0 the conditional prompt,
 *             row block 1 the unconditional (negative) prompt
 *   guidance  s; sigma, sigma_next: this step's and the next noise level
 *   x_next    float [1, out_ch, F, Hz, Wz] output; may alias x
 * x, context and x_next are device pointers when io_on_device != 0, else host
 * pointers (copies inside the call, in stream order).  The result equals
 * wan_dit_forward at B = 2 followed by wan_op_cfg_euler on its two halves, bit
 * for bit.  Needs in_ch == out_ch (WAN_EUNSUPPORTED otherwise, e.g. I2V) and
 * max_batch >= 2; other limits as wan_dit_forward.                          */
WANDIT_API wan_status wan_dit_forward_cfg_euler(wan_dit* h, const float* x, int F, int Hz, int Wz,
                           float timestep, const void* context, int Lc,
                           float guidance, float sigma, float sigma_next,
                           float* x_next, int io_on_device, void* stream);

/* Noise levels of a `steps`-step flow-matching run, steps + 1 doubles from 1
 * down to a final 0: the uniform ladder u_i = 1 - i/steps (i < steps) under
 * the flow shift  sigma = shift u / (1 + (shift - 1) u),  which multiplies the
 * noise odds u / (1 - u) by `shift` (the pswp.cn WanPipeline notes set
 * flow_shift 3.0 for 480p and 5.0 for 720p in the scheduler; "读完 Wan2.2 全部源码之后"
 * §"shift 参数生效了两次,在两个地方": it takes effect where the timesteps are
 * set).  The DiT timestep of step i is sigmas[i] * num_train_timesteps.  Pure
 * host function; WAN_EINVAL for steps < 1, shift <= 0 or sigmas == NULL.    */
WANDIT_API wan_status wan_flow_sigmas(int steps, double shift, double* sigmas);

/* Sequence-parallel (Ulysses) forward, one rank's part ("读完 Wan2.2 全部源码之后",
 * §"显存和算力怎么分": q, k, v are scattered along heads and gathered along the
 * sequence by an all-to-all, every rank runs attention over the whole
 * sequence for its heads, and a second all-to-all brings the outputs back).
 * The tokens are split into `world` shards of Ls = ceil(L / world) tokens;
 * rank r holds global tokens [r * Ls, (r + 1) * Ls), the last shard padded
 * past L.  Padding is explicit, so no shard is shorter than the others (the
 * uneven torch.chunk split those pages warn about cannot occur): padding
 * tokens never act as keys (the attention masks keys >= L) and their outputs
 * are dropped; RoPE and the timestep use each token's global position.
 * Everything except self-attention is token-local and runs on the shard.
 * The caller moves the exchange buffers between ranks (e.g. NCCL
 * all_to_all_single per sample); the library reads and writes only this
 * rank's device memory.  Call order per forward:
 *   sp_begin; for block i: sp_block_qkv(i) -> exchange -> sp_attention ->
 *   exchange back -> sp_block_finish(i); sp_end.
 * Layouts (bf16, device, hd = 128 * heads / world):
 *   send   [B][world][Ls][3][hd]  q, k, v of this shard, head group j in slot j
 *          (q and k RMSNorm'd across all heads and rotated)
 *   recv   [B][world][Ls][3][hd]  = [B][Lp][3 hd]: this rank's head group for
 *          every token of the padded sequence (Lp = world * Ls)
 *   out    [B][Lp][hd]            attention output of this rank's heads
 *   back   [B][world][Ls][hd]     slot j: head group j's output for this shard
 * sp_begin takes the whole latent, the whole timestep ([B] or [B, L]) and the
 * context, host or device like wan_dit_forward; it needs heads % world == 0,
 * Ls <= max_tokens (the workspace holds the shard) and a text-to-video model;
 * the first sp_begin of a latent size allocates device staging for the whole
 * latent and velocity (kept by the handle).  sp_end writes the full-size
 * velocity [B, out_ch, F, Hz, Wz] holding this shard's tokens and zeros
 * elsewhere: the sum over ranks is the velocity.  Calls are eager (no graph)
 * and asynchronous on `stream`; out-of-order calls return WAN_EINVAL.       */
WANDIT_API wan_status wan_dit_sp_begin(wan_dit* h, const void* latent, int latent_dtype,
                           int B, int F, int Hz, int Wz, const float* timestep, int per_token,
                           const void* context, int Lc, int rank, int world, int io_on_device, void* stream);
WANDIT_API wan_status wan_dit_sp_block_qkv(wan_dit* h, int block, void* send, void* stream);
WANDIT_API wan_status wan_dit_sp_attention(wan_dit* h, const void* recv, void* out, void* stream);
WANDIT_API wan_status wan_dit_sp_block_finish(wan_dit* h, int block, const void* back, void* stream);
WANDIT_API wan_status wan_dit_sp_end(wan_dit* h, float* velocity, int io_on_device, void* stream);

/* Expert of the Wan2.2 A14B two-expert route for one sampling step: 0 (the
 * high-noise expert) when t >= boundary * num_train_timesteps, else 1 (the
 * low-noise expert).  One expert runs the whole step, both CFG forwards
 * included ("读完 Wan2.2 全部源码之后", the sampling-loop section); the caller
 * keeps one handle per expert.  Pure host function.                         */
WANDIT_API int wan_moe_select(double t, double boundary, int num_train_timesteps);

/* Synchronise `stream` and report a kernel timeout recorded by any earlier
 * launch of this handle (WAN_ETIMEOUT, flag cleared) or a CUDA error.       */
WANDIT_API wan_status wan_dit_sync(wan_dit* h, void* stream);

/* Debug: with dst != NULL the next forwards (run without graph replay) copy
 * the residual stream after the patch embedding and after each block into the
 * device buffer dst = bf16 [num_blocks + 1, B, L, dim].  NULL turns it off. */
WANDIT_API wan_status wan_dit_set_block_dump(wan_dit* h, void* dst);

/* Options: WAN_OPT_GRAPH (1 = capture/replay the forward as a CUDA graph,
 * default 1), WAN_OPT_WAIT_LIMIT_NS (time limit of every on-chip wait,
 * default 2e9 ns; values below 1000 are for fault tests only),
 * WAN_OPT_KERNEL_TIMING (1 = record a CUDA event pair around every kernel of
 * the forward, read back with wan_dit_kernel_time; default 0),
 * WAN_OPT_GEMM_PAIR (1 = the block GEMMs with N a multiple of 256 run as
 * SM-pair tcgen05 GEMMs, 256 x 256 tiles on clusters of two CTAs; 0 = every
 * GEMM on single-SM 128-row tiles; default 1; same results either way up to
 * fp32 summation order).                                                   */
enum { WAN_OPT_GRAPH = 1, WAN_OPT_WAIT_LIMIT_NS = 2, WAN_OPT_KERNEL_TIMING = 3, WAN_OPT_GEMM_PAIR = 4 };

/* Kernel classes of the forward, for wan_dit_kernel_time().  WAN_KC_GEMM
 * covers the GEMMs outside the blocks (patch, timestep, text, cross K/V,
 * proj_out); the block GEMMs have a class each: q/k/v projection (with the
 * q/k RMSNorm epilogue), attention output, cross-attention query and output,
 * FFN up and down.                                                          */
enum {
    WAN_KC_PATCHIFY = 0, WAN_KC_GEMM = 1, WAN_KC_SELF_ATTENTION = 2, WAN_KC_CROSS_ATTENTION = 3,
    WAN_KC_LAYERNORM = 4, WAN_KC_RMSNORM_ROPE = 5, WAN_KC_EMBEDDING = 6,
    WAN_KC_GEMM_QKV = 7, WAN_KC_GEMM_O = 8, WAN_KC_GEMM_Q2 = 9, WAN_KC_GEMM_O2 = 10,
    WAN_KC_GEMM_FFN_UP = 11, WAN_KC_GEMM_FFN_DOWN = 12, WAN_KC_COUNT = 13
};

/* With WAN_OPT_KERNEL_TIMING on: total device time (ms) and number of
 * launches of kernel class `kc` in the most recent forward.  Synchronises the
 * forward's events (blocks until that forward has finished).               */
WANDIT_API wan_status wan_dit_kernel_time(wan_dit* h, int kc, double* total_ms, int* launches);
WANDIT_API wan_status wan_dit_set_option(wan_dit* h, int option, int64_t value);

/* Kernel launches issued by the most recent forward (a replayed graph counts
 * the kernels it holds).                                                   */
WANDIT_API int wan_dit_last_launch_count(const wan_dit* h);

/* Algorithmic FLOPs of one forward at the given shape (dense, no padding). */
WANDIT_API double wan_dit_flops(const wan_dit* h, int B, int F, int Hz, int Wz, int Lc, int per_token);
/* Same with Li image tokens per sample (I2V); Li = 0 equals wan_dit_flops. */
WANDIT_API double wan_dit_flops_image(const wan_dit* h, int B, int F, int Hz, int Wz, int Lc, int per_token, int Li);

WANDIT_API const char* wan_dit_last_error(const wan_dit* h);
WANDIT_API const char* wan_status_string(wan_status s);

/* Free the handle and everything it owns (synchronises its device). */
WANDIT_API void wan_dit_destroy(wan_dit* h);

#ifdef __cplusplus
}
#endif
#endif /* WANDIT_H */

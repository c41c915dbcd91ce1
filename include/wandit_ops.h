/*
 * wandit_ops.h -- kernel-level entry points of libwandit.so.
 *
 * These launch, one at a time, the same sm_100a kernels that wan_dit_forward()
 * strings together, so each step of the Wan DiT forward can be checked on its
 * own.  Citations name the page and section whose computation the kernel
 * performs (see wandit.h for the page list).  Conventions are those of
 * wandit.h: plain device pointers, `stream` is a cudaStream_t as void*, calls
 * are asynchronous, nothing is retained after the call, shape errors are
 * reported before any launch, and wan_op_sync() reports a kernel wait that ran
 * out of time.  All matrices are dense row-major with the given leading
 * dimension (in elements); bf16 means IEEE bfloat16, f32 means float.
 */
#ifndef WANDIT_OPS_H
#define WANDIT_OPS_H

#include <stdint.h>
#include "wandit.h"

#ifdef __cplusplus
extern "C" {
#endif

/* GEMM epilogues: out[r, c] for acc = sum_k A[r, k] * W[c, k] (fp32 in TMEM).
 *  WAN_EPI_BIAS          out bf16 = acc + bias[c]                       (every nn.Linear)
 *  WAN_EPI_BIAS_GELU     out bf16 = GELU_tanh(acc + bias[c])            (ffn.net.0 + activation;
 *                        text_embedder linear_1 + activation)
 *  WAN_EPI_GATE_RESIDUAL out bf16 = out + (acc + bias[c]) * gate(r, c)  (the gated residual
 *                        x + gate_msa * attn1(..) and x + c_gate_msa * ffn(..) of the pswp.cn
 *                        notes, section "WanTransformerBlock", added in fp32),
 *                        gate(r, c) = gate0[c] + gate1[(r / mod_div) * mod_ld + c]
 *  WAN_EPI_RESIDUAL      out bf16 = out + bf16(acc + bias[c])           (cross-attention residual)
 *  WAN_EPI_BIAS_F32      out f32  = acc + bias[c]
 *  WAN_EPI_UNPATCHIFY    velocity f32 = bf16(acc + bias[c]) scattered by the unpatchify map
 *                        (WanTransformer3DModel step 5); row r = b * L + token, column
 *                        c = ((kt * ph + kh) * pw + kw) * up_C + ch.
 *  WAN_EPI_QK_NORM       the q/k projection with "qk_norm = rms_norm_across_heads" split
 *                        in two: for c < norm_cols, out bf16 = gain[c] * (acc + bias[c]),
 *                        rotated by the 3-axis RoPE of token r % (rope_F*rope_H*rope_W)
 *                        when rope != 0, and ssq[r * ssq_ld + c / 128] = sum over the
 *                        128-column group of (acc + bias)^2 (fp32); columns >= norm_cols
 *                        get the bias epilogue.  The row factor rsqrt(sum / D + eps)
 *                        commutes with the gain and the rotation and is applied by
 *                        wan_op_rms_apply (keys) or wan_op_attention_qnorm (queries).
 *                        N % 256 == 0, norm_cols % 128 == 0.                            */
enum {
    WAN_EPI_BIAS = 0,
    WAN_EPI_BIAS_GELU = 1,
    WAN_EPI_GATE_RESIDUAL = 2,
    WAN_EPI_RESIDUAL = 3,
    WAN_EPI_BIAS_F32 = 4,
    WAN_EPI_UNPATCHIFY = 5,
    WAN_EPI_QK_NORM = 8
};

typedef struct {
    const float* bias;    /* [N] f32, or NULL for no bias                         */
    void* out;            /* output (bf16 or f32 per epilogue); read too for the
                             residual epilogues                                  */
    int64_t ldo;          /* row stride of out in elements                        */
    const float* gate0;   /* [N] f32 (gate epilogue), or NULL (read as 0)         */
    const float* gate1;   /* f32 rows of the per-sample / per-token modulation, or
                             NULL (read as 0); the gate epilogue needs at least
                             one of gate0, gate1 (else WAN_EINVAL)               */
    int mod_div;          /* modulation row = r / mod_div                         */
    int64_t mod_ld;       /* row stride of gate1 in elements                      */
    int up_C, up_F, up_Hz, up_Wz; /* unpatchify geometry, patch (1,2,2)           */
    /* WAN_EPI_QK_NORM only: */
    const float* gain;    /* [norm_cols] f32 RMSNorm gains                         */
    float* ssq;           /* f32 [M, ssq_ld] per-128-column sums of squares (output) */
    int64_t ssq_ld;       /* row stride of ssq, >= norm_cols / 128                  */
    int norm_cols;        /* leading columns that are normed                       */
    int rope;             /* 1: rotate the normed columns (RoPE), 0: no rotation     */
    int rope_F, rope_H, rope_W;   /* post-patch grid of the RoPE positions         */
    int rope_t, rope_h, rope_w;   /* head-dim split (even, sum 128)                */
    float rope_theta;     /* RoPE base                                             */
} wan_epilogue;

/* C = epilogue(A[M,K] . W[N,K]^T).  A, W bf16 device pointers, 16-byte aligned
 * rows (lda, ldw multiples of 8).  Requires K % 64 == 0 and N % 64 == 0; M is
 * arbitrary (ragged last tile masked).  tcgen05 MMA with TMEM accumulators fed
 * by TMA.                                                                   */
WANDIT_API wan_status wan_op_gemm(const void* A, int64_t lda, const void* W, int64_t ldw,
                       int M, int N, int K, int epilogue, const wan_epilogue* epi, void* stream);

/* Flash attention O = softmax(Q K^T / sqrt(128)) V per (batch, head), no mask
 * ("WanTransformerBlock" attn1 / attn2; bidirectional full attention,
 * 【VLA与模仿学习】Wan2.1框架与训练源码导读 §5.2).  Row (b, l) of Q/O starts at
 * q + (b * Lq + l) * ldq; of K/V at k + (b * Lk + l) * ldk; head h occupies
 * columns [128 h, 128 h + 128).  bf16 in/out, fp32 online softmax.  Key
 * rows past Lk in the last 128-key tile are masked.  Errors, reported before
 * any launch: WAN_EINVAL for a null pointer; WAN_ESHAPE for B < 0, heads <= 0,
 * Lq < 0, Lk <= 0, a leading dimension that is not a multiple of 8 elements,
 * or a pointer that is not 16-byte aligned.  B = 0 or Lq = 0 launches
 * nothing.  Up to four key tiles (Lk <= 512) run on one SM per CTA; longer
 * key sets run on SM pairs (clusters of two CTAs).                          */
WANDIT_API wan_status wan_op_attention(const void* q, int64_t ldq, const void* k, int64_t ldk,
                            const void* v, int64_t ldv, void* o, int64_t ldo,
                            int B, int heads, int Lq, int Lk, void* stream);

/* wan_op_attention with unnormalised queries: each query row (b, l) is first
 * multiplied by its RMSNorm factor rsqrt(sum_{g < ngroups} q_ssq[(b * Lq + l) *
 * ssq_ld + g] / (128 * heads) + eps), the sums of squares coming from the
 * WAN_EPI_QK_NORM epilogue (RMSNorm across heads: "qk_norm =
 * rms_norm_across_heads").  Same layouts and limits as wan_op_attention;
 * also WAN_EINVAL for a null q_ssq and WAN_ESHAPE for ngroups <= 0 or
 * ssq_ld < ngroups.                                                          */
WANDIT_API wan_status wan_op_attention_qnorm(const void* q, int64_t ldq, const void* k, int64_t ldk,
                            const void* v, int64_t ldv, void* o, int64_t ldo,
                            int B, int heads, int Lq, int Lk,
                            const float* q_ssq, int64_t ssq_ld, int ngroups, float eps, void* stream);

/* In-place row factor of the split RMSNorm: buf[r, 0:D) *= rsqrt(sum_{g <
 * ngroups} ssq[r * ssq_ld + g] / D + eps) for bf16 rows (row stride ld); the
 * key half of WAN_EPI_QK_NORM.  D as for wan_op_rmsnorm_rope.               */
WANDIT_API wan_status wan_op_rms_apply(void* buf, int64_t ld, int rows, int D, const float* ssq, int64_t ssq_ld,
                                       int ngroups, float eps, void* stream);

/* LayerNorm of bf16 rows x[rows, D] (fp32 statistics, biased variance, eps),
 * then either an affine (gamma, beta; mode 1: norm2) or the adaLN modulation
 * (mode 0: y = LN(x) * (1 + scale0[c] + scale1[m c]) + shift0[c] + shift1[m c],
 * m = r / mod_div, row stride mod_ld; norm_out), or the modulation with the
 * per-sample rows already combined (mode 2: y = LN(x) * scale1[m c] +
 * shift1[m c], scale1 holding 1 + scale; the forward's norm1/norm3, whose
 * rows come from the all-blocks modulation table).  D a multiple of 256;
 * WAN_EINVAL for another mode or a missing vector.  Output bf16.            */
WANDIT_API wan_status wan_op_layernorm(const void* x, void* y, int rows, int D, float eps, int mode,
                            const float* gamma, const float* beta,
                            const float* shift0, const float* shift1,
                            const float* scale0, const float* scale1,
                            int mod_div, int64_t mod_ld, void* stream);

/* In-place RMSNorm across all heads of bf16 row segments buf[r, 0:D] (row
 * stride ld), times gain[D] ("qk_norm = rms_norm_across_heads"), then, when
 * rope != 0, the 3-axis rotary embedding of token l = r % (Fp*Hp*Wp) at grid
 * position (f, i, j) (RoPE per T/H/W axis, pairs (2k, 2k+1) of each 128-wide
 * head, head-dim split rope_t/h/w, base theta).                             */
WANDIT_API wan_status wan_op_rmsnorm_rope(void* buf, int64_t ld, int rows, int D, float eps, const float* gain,
                               int rope, int Fp, int Hp, int Wp, int rope_t, int rope_h, int rope_w,
                               float theta, void* stream);

/* Allocation-free variant of wan_op_rmsnorm_rope (same arguments, same
 * result).  The pages have no counterpart: this exists for callers that must
 * not allocate device memory while they run -- serving stacks whose own pool
 * allocator holds (nearly) all of HBM, so a library cudaMalloc fails or breaks
 * their accounting, and latency-critical loops that cannot take the implicit
 * synchronisation cudaMalloc / cudaFree may cause.  wan_op_rmsnorm_rope
 * allocates its cos/sin table per call; this variant keeps it in a fixed
 * __device__ array of 1024 positions x 64 pairs (512 KiB) that every GPU
 * loading the library holds until the process exits, and calls no cudaMalloc,
 * cudaFree or other allocating routine.
 *  - Limit: Fp, Hp and Wp (post-patch grid) must each be <= 1024, the
 *    rope_max_seq_len of the Wan configs; larger grids, and D / ld outside
 *    the rules of wan_op_rmsnorm_rope, return WAN_ESHAPE before the array is
 *    touched or anything is launched.  A CUDA error already pending on the
 *    calling thread is returned as WAN_ECUDA, also before any launch (and
 *    left pending for the caller).
 *  - The first call on a device (with that device current) looks up the
 *    array's device address with cudaGetSymbolAddress and caches it; make
 *    that first call before any stream capture on the device.
 *  - Every call rewrites the part of the array it uses and all calls share
 *    it: calls that can overlap on the GPU (different streams without an
 *    ordering between them) race on the table and must be serialised.     */
WANDIT_API wan_status wan_op_rmsnorm_rope_noalloc(void* buf, int64_t ld, int rows, int D, float eps,
                                                  const float* gain, int rope, int Fp, int Hp, int Wp,
                                                  int rope_t, int rope_h, int rope_w, float theta,
                                                  void* stream);

/* Patchify gather: latent [B, C, F, Hz, Wz] (f32 or bf16) -> X bf16
 * [B * L, C * 4] with token order (f, i, j) and feature order (c, kh, kw) --
 * the input view of patch_embedding = Conv3d(k = s = (1,2,2)).               */
WANDIT_API wan_status wan_op_patchify(const void* latent, int latent_dtype, int B, int C, int F, int Hz, int Wz,
                           void* X, void* stream);

/* Unpatchify scatter: rows f32 [B * L, 4 * C] (feature order (kh, kw, c)) ->
 * velocity f32 [B, C, F, Hz, Wz]; the same index map the proj_out epilogue
 * uses.                                                                     */
WANDIT_API wan_status wan_op_unpatchify(const float* rows, int B, int C, int F, int Hz, int Wz,
                             float* velocity, void* stream);

/* Causal 3-D convolution of the Wan VAE decoder (pswp.cn WanPipeline notes,
 * "WanCausalConv3d": 2 p_t zero frames before the input and none after, p_h /
 * p_w zero rows / columns on both sides, p = (k - 1) / 2; with a cache of the
 * frames right before frame 0 those replace the leading zero frames, as in the
 * decoder's frame loop).  Channels-last bf16 tensors:
 *   x      [B, T, H, W, Ci]            input frames (device)
 *   cache  [B, nc, H, W, Ci] or NULL   the nc frames before frame 0 (nc <= kt - 1)
 *   w      [Co, ldw] bf16: row co holds W[co, :, it, ih, iw] in (it, ih, iw, ci)
 *          order, ci fastest, zero from kt*kh*kw*Ci up to ldw
 *   bias   f32 [Co] or NULL;  y  [B, T, H, W, Co] output (device)
 *   col    device workspace of at least B*T*H*W * ldw bf16 (the im2col rows)
 * kt, kh, kw odd; Ci % 8 == 0; Co % 64 == 0; ldw = kt*kh*kw*Ci rounded up to a
 * multiple of 64.  Runs as a gather into col plus the tcgen05 GEMM
 * y = col . w^T + bias.  Returns WAN_ESHAPE for sizes outside these rules.  */
WANDIT_API wan_status wan_op_causal_conv3d(const void* x, const void* cache, int nc, int B, int T, int H, int W,
                                           int Ci, const void* w, int64_t ldw, const float* bias, int Co, int kt,
                                           int kh, int kw, void* col, int64_t col_elems, void* y, void* stream);

/* One flow-matching sampler step with classifier-free guidance
 * ("【VLA与模仿学习】Wan2.1框架与训练源码导读" §7: CFG  v = v_uncond + s (v_cond - v_uncond),
 * Euler update  x_next = x + (sigma_next - sigma) v; §6.1 x_sigma = (1 - sigma) z + sigma eps).
 * x, v_cond, v_uncond, x_next: f32 device arrays of n elements, 16-byte aligned (x_next may
 * alias x).  v_uncond == NULL means no guidance (v = v_cond).  With the CFG batch of
 * wan_dit_forward (B = 2), v_cond / v_uncond are the two halves of its velocity output.   */
WANDIT_API wan_status wan_op_cfg_euler(const float* x, const float* v_cond, const float* v_uncond,
                                       float guidance, float sigma, float sigma_next, int64_t n,
                                       float* x_next, void* stream);

/* Self-test of the bounded on-chip waits every tcgen05 kernel uses: launches one
 * warp that waits on an mbarrier nothing arrives on, with a time limit of
 * `limit_ns` (clamped to [1 us, 1 s]).  The wait gives up, records the timeout in
 * the op error word and the kernel returns; wan_op_sync() then reports
 * WAN_ETIMEOUT and clears it.  Faults nothing and leaves the context usable.  */
WANDIT_API wan_status wan_op_wait_selftest(int64_t limit_ns, void* stream);

/* Synchronise `stream`; WAN_ETIMEOUT if an op kernel's bounded wait ran out
 * (flag cleared), WAN_ECUDA on a CUDA error.                                */
WANDIT_API wan_status wan_op_sync(void* stream);

/* Time limit in ns of every on-chip wait of the op kernels (default 2e9). */
WANDIT_API void wan_op_set_wait_limit_ns(int64_t ns);

/* wan_op_gemm on SM pairs where it applies (on != 0, the default: N a
 * multiple of 256, M >= 512, bias / GELU / gate-residual / residual / q-k
 * norm epilogues) or always on single-SM tiles (on == 0).                  */
WANDIT_API void wan_op_set_gemm_pair(int on);

/* Number of two-CTA clusters the SM-pair GEMM runs with on the current
 * device (0 if the device cannot co-schedule them; the GEMMs then use
 * single-SM tiles).  Initialises the op state of the device; -1 on a CUDA
 * error.                                                                   */
WANDIT_API int wan_op_gemm_pair_clusters(void);

#ifdef __cplusplus
}
#endif
#endif /* WANDIT_OPS_H */

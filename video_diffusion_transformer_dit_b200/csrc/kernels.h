// Host-side launch functions of the libwandit kernels (internal header).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace wan {

// Epilogue kinds of the tcgen05 GEMM (same numbering as WAN_EPI_* in wandit_ops.h).
enum EpiKind : int {
    EPI_BIAS = 0,
    EPI_BIAS_GELU = 1,
    EPI_GATE_RESIDUAL = 2,
    EPI_RESIDUAL = 3,
    EPI_BIAS_F32 = 4,
    EPI_UNPATCHIFY = 5,
    EPI_BIAS_SILU = 6,
    // CFG pair + Euler step in the proj_out epilogue: A holds the rows of two
    // samples (conditional rows [0, M), unconditional rows [pair_off, pair_off + M));
    // out = x_next scattered by the unpatchify map, x read at the same place
    EPI_CFG_EULER = 7,
    // q/k projection with RMSNorm across heads split in two: columns [0, norm_cols)
    // are stored as gain * acc (rotated by RoPE when rope.t != null) and each
    // 128-column group's sum of acc^2 goes to ssq[row * ssq_ld + group]; the
    // rsqrt(mean + eps) row factor is applied later (attention for q, a row
    // pass for k).  Columns past norm_cols get the plain bias epilogue.
    EPI_QK_NORM = 8
};

// RoPE tables: float2 (cos, sin) for each axis, [len_a][d_a/2], axes concatenated.
struct RopeTables {
    const float2* t;
    const float2* h;
    const float2* w;
    int Fp, Hp, Wp;
    int nt, nh, nw;   // pairs per axis
    int pair_major;   // 0: [len_a][pairs] (one row reads its pairs together);
                      // 1: [pairs][len_a] (consecutive tokens read neighbouring entries)
};

struct EpiParams {
    int kind;
    const float* bias;      // [N] or null
    void* out;              // bf16 / f32 output (read too for residual kinds)
    long long ldo;          // row stride of out (elements)
    const float* gate0;     // [N]
    const float* gate1;     // rows of modulation
    int mod_div;            // modulation row = r / mod_div
    long long mod_ld;       // row stride of gate1 (elements)
    int L, C, F, Hz, Wz;    // unpatchify: tokens per sample, channels, latent grid
    int pair_off;           // EPI_CFG_EULER: row offset of the unconditional rows in A
    const float* x;         // EPI_CFG_EULER: sampler state [C, F, Hz, Wz] f32
    const float* sched;     // EPI_CFG_EULER: device {guidance, sigma_next - sigma}
    int norm_cols;          // EPI_QK_NORM: columns that are RMS-normed (multiple of 128)
    const float* gain;      // EPI_QK_NORM: [norm_cols] RMSNorm gains
    float* ssq;             // EPI_QK_NORM: per-row sums of squares, one per 128-column group
    long long ssq_ld;       // EPI_QK_NORM: row stride of ssq (floats)
    int rope_L;             // EPI_QK_NORM: rows per sample (RoPE position = rope_tok0 + row % rope_L,
    int rope_tok0;          //   held at the grid's last token for padding rows past it)
    RopeTables rope;        // EPI_QK_NORM: rope.t == null for no rotation
    int up_rows, up_tok0;   // EPI_UNPATCHIFY: rows per sample (0: L) and the token of a sample's
                            //   first row; rows whose token is >= L (padding) are dropped
};

struct LaunchCtx {
    cudaStream_t stream;
    int* err;               // device error word
    uint64_t wait_limit_ns;
    int num_sms;
    int* launches;          // incremented per kernel launch (host counter), may be null
    int gemm_pair = 1;      // 1: large N % 256 == 0 GEMMs run on SM pairs (cta_group::2)
};

// Raise the dynamic shared-memory limit of the tcgen05 kernels (once per
// process and device; call outside stream capture).
cudaError_t init_kernel_attributes();
cudaError_t init_layernorm_attributes();  // part of init_kernel_attributes

// Tensor maps (TMA descriptors).
bool make_tmap_2d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint64_t ld_elems,
                  uint32_t box_inner, uint32_t box_outer);
bool make_tmap_3d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t d1, uint64_t d2, uint64_t ld1_elems,
                  uint64_t ld2_elems, uint32_t box_inner, uint32_t box1);

bool make_tmap_5d(CUtensorMap* m, const void* ptr, const uint64_t (&dims)[5], const uint64_t (&strides_elems)[4],
                  uint32_t box_inner, uint32_t box1, uint32_t box2);

// C = epi(A[M,K] . W[N,K]^T); returns a CUDA error (or cudaErrorInvalidValue
// for unsupported shapes).
// Two-CTA clusters the SM-pair GEMM runs with (0: not available); valid after
// init_kernel_attributes().
int gemm_pair_clusters();
cudaError_t launch_gemm(const void* A, long long lda, const void* W, long long ldw, int M, int N, int K,
                        const EpiParams& epi, const LaunchCtx& ctx);

// Row factors of an RMSNorm whose sums of squares were taken elsewhere (the
// EPI_QK_NORM epilogue): row r's factor is rsqrt(sum_{g < ngroups} ssq[r * ssq_ld + g] * inv_n + eps).
struct RowNorm {
    const float* ssq;       // null: no row factor
    long long ssq_ld;
    int ngroups;
    float inv_n, eps;
};

// Flash attention (bf16, head_dim 128).  With qn.ssq set, every query row is
// multiplied by its RMSNorm row factor (q stored unnormalised).
cudaError_t launch_attention(const void* q, long long ldq, const void* k, long long ldk, const void* v,
                             long long ldv, void* o, long long ldo, int B, int heads, int Lq, int Lk,
                             const LaunchCtx& ctx, const RowNorm& qn = RowNorm{nullptr, 0, 0, 0.f, 0.f});

// buf[r, 0:D) *= the RMSNorm row factor of rn (in place, bf16, one rounding).
cudaError_t launch_rms_apply(void* buf, long long ld, int rows, int D, const RowNorm& rn, const LaunchCtx& ctx);

// Per-sample modulation of every block: out[n][b][6][D] = sst[n] + tproj[b] (+1 on the scale rows).
cudaError_t launch_mod_combine(const float* sst, const float* tproj, float* out, int N, int B, int D,
                               const LaunchCtx& ctx);

// LayerNorm (+ modulation or affine); mode 0 modulation from table + rows, 1 affine,
// 2 precombined rows (scale1 = 1 + scale, shift1).
cudaError_t launch_layernorm(const void* x, void* y, int rows, int D, float eps, int mode, const float* gamma,
                             const float* beta, const float* shift0, const float* shift1, const float* scale0,
                             const float* scale1, int mod_div, long long mod_ld, const LaunchCtx& ctx);

#ifdef __CUDACC__
// (cos, sin) of pair p (0..63) of a 128-wide head at grid position (f, i, j):
// axis t for p < nt, h for p < nt + nh, else w.
__device__ __forceinline__ float2 rope_cs(const RopeTables& rt, int p, int f, int i, int j) {
    if (rt.pair_major) {
        if (p < rt.nt) return __ldg(rt.t + p * rt.Fp + f);
        p -= rt.nt;
        if (p < rt.nh) return __ldg(rt.h + p * rt.Hp + i);
        p -= rt.nh;
        return __ldg(rt.w + p * rt.Wp + j);
    }
    if (p < rt.nt) return __ldg(rt.t + f * rt.nt + p);
    p -= rt.nt;
    if (p < rt.nh) return __ldg(rt.h + i * rt.nh + p);
    p -= rt.nh;
    return __ldg(rt.w + j * rt.nw + p);
}
// Address of the (cos, sin) entry of pair p in pair-major tables, without
// branches (selects), so that a run of lookups can all be in flight at once.
__device__ __forceinline__ const float2* rope_entry_pm(const RopeTables& rt, int p, int f, int i, int j) {
    const float2* at_t = rt.t + p * rt.Fp + f;
    const float2* at_h = rt.h + (p - rt.nt) * rt.Hp + i;
    const float2* at_w = rt.w + (p - rt.nt - rt.nh) * rt.Wp + j;
    return p < rt.nt ? at_t : (p < rt.nt + rt.nh ? at_h : at_w);
}
#endif

// Row widths and strides the RMSNorm kernels take: D a supported multiple of
// 256 (up to 6144), ld a multiple of 8 elements and >= D.
bool rmsnorm_rope_shape_ok(int D, long long ld);

// In-place RMSNorm (+ RoPE) of nseg row segments (segment s at column
// s * seg_stride, gain gains + s * gain_stride).
cudaError_t launch_rmsnorm_rope(void* buf, long long ld, int rows, int D, float eps, const float* gains,
                                long long gain_stride, int nseg, long long seg_stride, const RopeTables* rope,
                                int rope_L, const LaunchCtx& ctx);

// X[b * rows + r] = patch of token tok0 + r of sample b (zero row when that token is >= L);
// ldx >= 4C: row stride of X, pad columns zeroed.  rows = 0 means rows = L, tok0 = 0.
cudaError_t launch_patchify(const void* latent, int latent_dtype, int B, int C, int F, int Hz, int Wz, void* X,
                            int ldx, const LaunchCtx& ctx, int tok0 = 0, int rows = 0);
// Implicit-GEMM causal Conv3d (tcgen05), channels last.  Epilogues:
//   CONV_EPI_BIAS        y[pix, co] = bf16(acc + bias[co])                          (co < Co)
//   CONV_EPI_ADD         y[pix, co] = bf16(acc + bias[co] + add[pix, co])           (residual)
//   CONV_EPI_TIME_SPLIT  Co = 2 csplit output channels of frame t go to frames 2t (co < csplit)
//                        and 2t + 1 (co >= csplit), channel co % csplit; y has 2T frames
enum ConvEpiKind : int { CONV_EPI_BIAS = 0, CONV_EPI_ADD = 1, CONV_EPI_TIME_SPLIT = 2 };
struct ConvEpi {
    int kind;
    const float* bias;          // [Co] or null
    __nv_bfloat16* y;           // output rows, channel stride ldy
    long long ldy;
    const __nv_bfloat16* add;   // CONV_EPI_ADD: rows of the residual, channel stride ldadd
    long long ldadd;
    int csplit;                 // CONV_EPI_TIME_SPLIT: channels per output frame
};
// x [B, T, H, W, Ci] bf16; cache [B, nc, H, W, Ci] (the nc frames right before
// frame 0) or null; w [Co_pad, ldw] bf16 with row co = W[co, ci, it, ih, iw] in
// (it, ih, iw, ci) order, ci padded to a multiple of 64 with zeros (ldw >=
// kt*kh*kw*ceil(Ci/64)*64); Co_pad a multiple of 64 (rows past Co are ignored).
// nc_cap: frame slots per sample in the cache buffer (its batch stride), >= nc.
cudaError_t launch_conv3d(const void* x, const void* cache, int nc, int B, int T, int H, int W, int Ci, const void* w,
                          long long ldw, int Co, int Co_pad, int kt, int kh, int kw, const ConvEpi& epi,
                          const LaunchCtx& ctx, int nc_cap = 0);
cudaError_t init_conv_attributes();

// Causal Conv3d im2col, channels last: col [B*T*H*W, Kp] bf16 (Kp >= kt*kh*kw*Ci, pad zeroed),
// cache [B, nc, H, W, Ci] (frames right before frame 0) or null.
cudaError_t launch_causal_im2col(const void* x, const void* cache, int nc, int B, int T, int H, int W, int Ci, int kt,
                                 int kh, int kw, void* col, int Kp, const LaunchCtx& ctx);
// Sequence-parallel exchange layouts for world size P (head group j = columns
// [j * D / P, (j + 1) * D / P) of each of q, k, v):
//   pack   qkv [B * Ls, 3D] -> send [B][P][Ls][3][D / P]
//   unpack back [B][P][Ls][D / P] -> o [B * Ls, D]
cudaError_t launch_sp_pack(const void* qkv, void* send, int B, int P, int Ls, int D, const LaunchCtx& ctx);
cudaError_t launch_sp_unpack(const void* back, void* o, int B, int P, int Ls, int D, const LaunchCtx& ctx);

// a[i] = bf16(a[i] + b[i]) for n bf16 values (n % 8 == 0, 16-byte aligned)
cudaError_t launch_add_bf16(void* a, const void* b, long long n, const LaunchCtx& ctx);
cudaError_t launch_unpatchify(const float* rows, int B, int C, int F, int Hz, int Wz, float* vel,
                              const LaunchCtx& ctx);

// out[b, n] = act_out(sum_k W[n, k] * act_in(x)[b, k] + bias[n]); W bf16 [N, K].
// act_in: 0 none, 1 SiLU, 2 timestep sinusoid of x[b, 0] (K = freq_dim);
// act_out: 0 none, 1 SiLU.
cudaError_t launch_gemv(const void* W, const float* bias, const float* x, long long ldx, float* out,
                        long long ldout, int B, int N, int K, int act_in, int act_out, const LaunchCtx& ctx);

// out[n, 0:dim] = [cos(t_n w_k), sin(t_n w_k)], w_k = 1e4^(-k / (dim/2)), bf16.
cudaError_t launch_sinusoid_bf16(const float* t, long long n, int dim, void* out, const LaunchCtx& ctx);

// out bf16 = SiLU(x f32), elementwise.
cudaError_t launch_silu_bf16(const float* x, void* out, long long n, const LaunchCtx& ctx);

// x_next = x + (sigma_next - sigma) * (v_uncond + guidance (v_cond - v_uncond)); v_uncond may be null.
cudaError_t launch_cfg_euler(const float* x, const float* v_cond, const float* v_uncond, float guidance, float sigma,
                             float sigma_next, long long n, float* x_next, const LaunchCtx& ctx);

// sched[0] = guidance, sched[1] = dsigma, t[0..nt) = t_value (one tiny kernel, stream ordered).
cudaError_t launch_set_sampler_scalars(float* sched, float guidance, float dsigma, float* t, int nt, float t_value,
                                       const LaunchCtx& ctx);

// One-warp kernel whose only mbarrier is never arrived on: exercises the bounded wait.
cudaError_t launch_wait_selftest(uint64_t limit_ns, const LaunchCtx& ctx);

// dst = convert(src), elementwise; dtypes 0 f32 / 1 bf16.
cudaError_t launch_convert(const void* src, int src_dtype, void* dst, int dst_dtype, long long n,
                           cudaStream_t stream);

}  // namespace wan

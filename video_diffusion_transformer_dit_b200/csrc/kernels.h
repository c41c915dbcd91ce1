// Host-side launch functions of the libwandit kernels (internal header).
#pragma once

#include <cuda.h>
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
    EPI_BIAS_SILU = 6
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
};

struct LaunchCtx {
    cudaStream_t stream;
    int* err;               // device error word
    uint64_t wait_limit_ns;
    int num_sms;
    int* launches;          // incremented per kernel launch (host counter), may be null
};

// Raise the dynamic shared-memory limit of the tcgen05 kernels (once per
// process and device; call outside stream capture).
cudaError_t init_kernel_attributes();

// Tensor maps (TMA descriptors).
bool make_tmap_2d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint64_t ld_elems,
                  uint32_t box_inner, uint32_t box_outer);
bool make_tmap_3d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t d1, uint64_t d2, uint64_t ld1_elems,
                  uint64_t ld2_elems, uint32_t box_inner, uint32_t box1);

// C = epi(A[M,K] . W[N,K]^T); returns a CUDA error (or cudaErrorInvalidValue
// for unsupported shapes).
cudaError_t launch_gemm(const void* A, long long lda, const void* W, long long ldw, int M, int N, int K,
                        const EpiParams& epi, const LaunchCtx& ctx);

// Flash attention (bf16, head_dim 128).
cudaError_t launch_attention(const void* q, long long ldq, const void* k, long long ldk, const void* v,
                             long long ldv, void* o, long long ldo, int B, int heads, int Lq, int Lk,
                             const LaunchCtx& ctx);

// Per-sample modulation of every block: out[n][b][6][D] = sst[n] + tproj[b] (+1 on the scale rows).
cudaError_t launch_mod_combine(const float* sst, const float* tproj, float* out, int N, int B, int D,
                               const LaunchCtx& ctx);

// LayerNorm (+ modulation or affine); mode 0 modulation from table + rows, 1 affine,
// 2 precombined rows (scale1 = 1 + scale, shift1).
cudaError_t launch_layernorm(const void* x, void* y, int rows, int D, float eps, int mode, const float* gamma,
                             const float* beta, const float* shift0, const float* shift1, const float* scale0,
                             const float* scale1, int mod_div, long long mod_ld, const LaunchCtx& ctx);

// RoPE tables: float2 (cos, sin) for each axis, [len_a][d_a/2], axes concatenated.
struct RopeTables {
    const float2* t;
    const float2* h;
    const float2* w;
    int Fp, Hp, Wp;
    int nt, nh, nw;   // pairs per axis
};

// Row widths and strides the RMSNorm kernels take: D a supported multiple of
// 256 (up to 6144), ld a multiple of 8 elements and >= D.
bool rmsnorm_rope_shape_ok(int D, long long ld);

// In-place RMSNorm (+ RoPE) of nseg row segments (segment s at column
// s * seg_stride, gain gains + s * gain_stride).
cudaError_t launch_rmsnorm_rope(void* buf, long long ld, int rows, int D, float eps, const float* gains,
                                long long gain_stride, int nseg, long long seg_stride, const RopeTables* rope,
                                int rope_L, const LaunchCtx& ctx);

cudaError_t launch_patchify(const void* latent, int latent_dtype, int B, int C, int F, int Hz, int Wz, void* X,
                            int ldx, const LaunchCtx& ctx);  // ldx >= 4C: row stride of X, pad columns zeroed
// Causal Conv3d im2col, channels last: col [B*T*H*W, Kp] bf16 (Kp >= kt*kh*kw*Ci, pad zeroed),
// cache [B, nc, H, W, Ci] (frames right before frame 0) or null.
cudaError_t launch_causal_im2col(const void* x, const void* cache, int nc, int B, int T, int H, int W, int Ci, int kt,
                                 int kh, int kw, void* col, int Kp, const LaunchCtx& ctx);
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

// One-warp kernel whose only mbarrier is never arrived on: exercises the bounded wait.
cudaError_t launch_wait_selftest(uint64_t limit_ns, const LaunchCtx& ctx);

// dst = convert(src), elementwise; dtypes 0 f32 / 1 bf16.
cudaError_t launch_convert(const void* src, int src_dtype, void* dst, int dst_dtype, long long n,
                           cudaStream_t stream);

}  // namespace wan

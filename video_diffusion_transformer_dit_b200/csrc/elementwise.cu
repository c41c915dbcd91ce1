// Bandwidth-bound kernels of the Wan DiT forward: LayerNorm with adaLN
// modulation or affine, RMSNorm across heads with the 3-axis RoPE rotation,
// the patchify gather, the unpatchify scatter (op-level), the small timestep
// MLP GEMVs and dtype conversion.  One warp per row, 16-byte vector accesses
// (8 bf16 per lane per step), fp32 statistics.
#include "common.cuh"
#include "kernels.h"

namespace wan {

// ------------------------------------------------------------------ helpers
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
    uint4 u = *reinterpret_cast<const uint4*>(p);
    float2 a = unpack_bf16(u.x), b = unpack_bf16(u.y), c = unpack_bf16(u.z), d = unpack_bf16(u.w);
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y; v[4] = c.x; v[5] = c.y; v[6] = d.x; v[7] = d.y;
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float (&v)[8]) {
    uint4 u = make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7]));
    *reinterpret_cast<uint4*>(p) = u;
}
__device__ __forceinline__ void load8f(const float* p, float (&v)[8]) {
    float4 a = __ldg(reinterpret_cast<const float4*>(p)), b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void unpack8(const uint4& u, float (&v)[8]) {
    const float2 a = unpack_bf16(u.x), b = unpack_bf16(u.y), c = unpack_bf16(u.z), d = unpack_bf16(u.w);
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y; v[4] = c.x; v[5] = c.y; v[6] = d.x; v[7] = d.y;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// ------------------------------------------------------------------ LayerNorm
// mode 0: y = LN(x) * (1 + scale0 + scale1[m]) + shift0 + shift1[m]
// mode 1: y = LN(x) * gamma + beta
// mode 2: y = LN(x) * scale1[m] + shift1[m]   (modulation precombined, 1 + scale included)
template <int NCH, int MODE>
__global__ void __launch_bounds__(256) layernorm_kernel(const __nv_bfloat16* __restrict__ x, __nv_bfloat16* __restrict__ y,
                                                        int rows, float eps, const float* gamma, const float* beta,
                                                        const float* shift0, const float* shift1, const float* scale0,
                                                        const float* scale1, int mod_div, long long mod_ld) {
    constexpr int D = NCH * 256;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * 8 + warp;
    if (row >= rows) return;
    const __nv_bfloat16* xr = x + (long long)row * D;
    uint4 u[NCH];  // the row stays packed (bf16) in registers between the passes
#pragma unroll
    for (int t = 0; t < NCH; ++t) u[t] = *reinterpret_cast<const uint4*>(xr + (t * 32 + lane) * 8);
    float s = 0.f;
#pragma unroll
    for (int t = 0; t < NCH; ++t) {
        float v[8];
        unpack8(u[t], v);
#pragma unroll
        for (int i = 0; i < 8; ++i) s += v[i];
    }
    const float mean = warp_sum(s) * (1.0f / D);
    float ss = 0.f;
#pragma unroll
    for (int t = 0; t < NCH; ++t) {
        float v[8];
        unpack8(u[t], v);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float d = v[i] - mean;
            ss += d * d;
        }
    }
    const float rstd = rsqrtf(warp_sum(ss) * (1.0f / D) + eps);
    const long long m = (long long)(row / mod_div) * mod_ld;
    __nv_bfloat16* yr = y + (long long)row * D;
#pragma unroll
    for (int t = 0; t < NCH; ++t) {
        const int c = (t * 32 + lane) * 8;
        float v[8], a[8], bb[8], o[8];
        unpack8(u[t], v);
        if (MODE == 2) {
            load8f(scale1 + m + c, a);
            load8f(shift1 + m + c, bb);
#pragma unroll
            for (int i = 0; i < 8; ++i) o[i] = (v[i] - mean) * rstd * a[i] + bb[i];
        } else if (MODE == 0) {
            float s1[8], h1[8];
            load8f(scale0 + c, a);
            load8f(shift0 + c, bb);
            load8f(scale1 + m + c, s1);
            load8f(shift1 + m + c, h1);
#pragma unroll
            for (int i = 0; i < 8; ++i) o[i] = (v[i] - mean) * rstd * (1.0f + a[i] + s1[i]) + (bb[i] + h1[i]);
        } else {
            load8f(gamma + c, a);
            load8f(beta + c, bb);
#pragma unroll
            for (int i = 0; i < 8; ++i) o[i] = (v[i] - mean) * rstd * a[i] + bb[i];
        }
        store8(yr + c, o);
    }
}

// LayerNorm modes 1 and 2 for D <= 1536, each warp walking `rpw` consecutive
// rows (a grid of one 256-thread CTA per SM).  The warp's columns of the
// modulation (or affine) vectors stay in registers and are reloaded only where
// the rows cross into the next sample, so per row only x and y move through L1
// (the per-row reload of 8 bytes of fp32 vectors per element made the
// one-row-per-warp kernel L1-bound).  Rows arrive through a ring of LN_RING
// shared-memory row buffers per warp, each filled by one bulk copy issued
// LN_RING rows ahead (bounded waits; no registers held for rows in flight).
constexpr int LN_RING = 4;
constexpr int LN_ROW_BYTES = 1536 * 2;
constexpr int LN_SMEM = 8 * LN_RING * LN_ROW_BYTES + 8 * LN_RING * 8 + 16;
template <int NCH, int MODE>
__global__ void __launch_bounds__(256, 1)
    layernorm_rows_kernel(const __nv_bfloat16* __restrict__ x, __nv_bfloat16* __restrict__ y, int rows, int rpw,
                          float eps, const float* gamma, const float* beta, const float* shift1,
                          const float* scale1, int mod_div, long long mod_ld, WaitCtl wc) {
    constexpr int D = NCH * 256;
    extern __shared__ __align__(128) uint8_t ln_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* ring = ln_smem + warp * LN_RING * LN_ROW_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(ln_smem + 8 * LN_RING * LN_ROW_BYTES) + warp * LN_RING;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(ln_smem + 8 * LN_RING * LN_ROW_BYTES + 8 * LN_RING * 8);
    if (threadIdx.x == 0) *abort_flag = 0;
    if (lane == 0) {
        for (int k = 0; k < LN_RING; ++k) mbar_init(bars + k, 1);
        fence_mbar_init();
    }
    __syncthreads();
    const int r0 = (blockIdx.x * 8 + warp) * rpw;
    const int r1 = min(r0 + rpw, rows);
    float ga[NCH][8], gb[NCH][8];  // y = (x - mean) * rstd * ga + gb on this lane's columns
    long long m_cur = -1;
    auto load_mod = [&](long long m) {
#pragma unroll
        for (int t = 0; t < NCH; ++t) {
            const int c = (t * 32 + lane) * 8;
            if (MODE == 2) {
                load8f(scale1 + m + c, ga[t]);
                load8f(shift1 + m + c, gb[t]);
            } else {
                load8f(gamma + c, ga[t]);
                load8f(beta + c, gb[t]);
            }
        }
    };
    auto fetch = [&](int row) {  // lane 0: the row into its ring slot
        const int k = (row - r0) % LN_RING;
        mbar_expect_tx(bars + k, D * 2);
        bulk_load(ring + k * LN_ROW_BYTES, x + (long long)row * D, D * 2, bars + k);
    };
    if (MODE == 1) load_mod(0);
    int issued = r0;  // rows whose copy has been issued: [r0, issued)
    if (lane == 0)
        for (; issued < r1 && issued < r0 + LN_RING; ++issued) fetch(issued);
    issued = __shfl_sync(0xffffffffu, issued, 0);
    int row = r0;
    for (; row < r1; ++row) {
        const int n = row - r0, k = n % LN_RING;
        if (!__all_sync(0xffffffffu, mbar_wait(bars + k, (n / LN_RING) & 1, abort_flag, wc))) break;
        uint4 u[NCH];
        const uint8_t* src = ring + k * LN_ROW_BYTES;
#pragma unroll
        for (int t = 0; t < NCH; ++t) u[t] = *reinterpret_cast<const uint4*>(src + (t * 32 + lane) * 16);
        __syncwarp();  // the slot is read: refill it with the row LN_RING ahead
        if (lane == 0 && issued < r1) {
            fence_proxy_async_smem();
            fetch(issued);
        }
        ++issued;
        if (MODE != 1) {
            const long long m = (long long)(row / mod_div) * mod_ld;
            if (m != m_cur) {
                load_mod(m);
                m_cur = m;
            }
        }
        float s = 0.f;
#pragma unroll
        for (int t = 0; t < NCH; ++t) {
            float v[8];
            unpack8(u[t], v);
#pragma unroll
            for (int i = 0; i < 8; ++i) s += v[i];
        }
        const float mean = warp_sum(s) * (1.0f / D);
        float ss = 0.f;
#pragma unroll
        for (int t = 0; t < NCH; ++t) {
            float v[8];
            unpack8(u[t], v);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float d = v[i] - mean;
                ss += d * d;
            }
        }
        const float rstd = rsqrtf(warp_sum(ss) * (1.0f / D) + eps);
        __nv_bfloat16* yr = y + (long long)row * D;
#pragma unroll
        for (int t = 0; t < NCH; ++t) {
            float v[8], o[8];
            unpack8(u[t], v);
#pragma unroll
            for (int i = 0; i < 8; ++i) o[i] = (v[i] - mean) * rstd * ga[t][i] + gb[t][i];
            store8(yr + (t * 32 + lane) * 8, o);
        }
    }
    // after a wait gave up, the copies in flight (rows from the one not waited for
    // up to the last issued, one per ring slot) land before the CTA exits
    if (row < r1 && lane == 0) {
        for (int rr = row; rr < min(issued, r1); ++rr) {
            const int n = rr - r0;
            mbar_drain(bars + n % LN_RING, (n / LN_RING) & 1, 200000000ull);
        }
    }
}

template <int NCH>
static cudaError_t set_ln_rows_attr() {
    cudaError_t e = cudaFuncSetAttribute(layernorm_rows_kernel<NCH, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, LN_SMEM);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(layernorm_rows_kernel<NCH, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, LN_SMEM);
    return e;
}

cudaError_t init_layernorm_attributes() {
    cudaError_t e = set_ln_rows_attr<1>();
    if (e == cudaSuccess) e = set_ln_rows_attr<2>();
    if (e == cudaSuccess) e = set_ln_rows_attr<3>();
    if (e == cudaSuccess) e = set_ln_rows_attr<4>();
    if (e == cudaSuccess) e = set_ln_rows_attr<6>();
    return e;
}

cudaError_t launch_layernorm(const void* x, void* y, int rows, int D, float eps, int mode, const float* gamma,
                             const float* beta, const float* shift0, const float* shift1, const float* scale0,
                             const float* scale1, int mod_div, long long mod_ld, const LaunchCtx& ctx) {
    if (rows <= 0) return cudaSuccess;
    if (D % 256) return cudaErrorInvalidValue;
    if (mod_div <= 0) mod_div = 1;
    dim3 grid((rows + 7) / 8);
    auto X = reinterpret_cast<const __nv_bfloat16*>(x);
    auto Y = reinterpret_cast<__nv_bfloat16*>(y);
    // rows walked per warp, modulation kept in registers (modes 1 and 2: mode 0
    // needs the vectors of two sources combined and would spill)
    if (D <= 1536 && mode != 0 && rows >= 8 * ctx.num_sms) {
        const int warps = 8 * ctx.num_sms;
        const int rpw = (rows + warps - 1) / warps;
        const int blocks = (rows + 8 * rpw - 1) / (8 * rpw);
        const WaitCtl wc{ctx.err, ctx.wait_limit_ns};
#define WAN_LN_ROWS(n)                                                                                            \
    case n:                                                                                                       \
        if (mode == 2)                                                                                            \
            layernorm_rows_kernel<n, 2><<<blocks, 256, LN_SMEM, ctx.stream>>>(X, Y, rows, rpw, eps, gamma, beta,   \
                                                                              shift1, scale1, mod_div, mod_ld, wc); \
        else                                                                                                      \
            layernorm_rows_kernel<n, 1><<<blocks, 256, LN_SMEM, ctx.stream>>>(X, Y, rows, rpw, eps, gamma, beta,   \
                                                                              shift1, scale1, mod_div, mod_ld, wc); \
        break;
        switch (D / 256) {
            WAN_LN_ROWS(1) WAN_LN_ROWS(2) WAN_LN_ROWS(3) WAN_LN_ROWS(4) WAN_LN_ROWS(6)
            default: return cudaErrorInvalidValue;
        }
#undef WAN_LN_ROWS
        if (ctx.launches) ++*ctx.launches;
        return cudaGetLastError();
    }
#define WAN_LN_CASE(n)                                                                                             \
    case n:                                                                                                        \
        if (mode == 2)                                                                                             \
            layernorm_kernel<n, 2><<<grid, 256, 0, ctx.stream>>>(X, Y, rows, eps, gamma, beta, shift0, shift1,      \
                                                                 scale0, scale1, mod_div, mod_ld);                 \
        else if (mode == 0)                                                                                        \
            layernorm_kernel<n, 0><<<grid, 256, 0, ctx.stream>>>(X, Y, rows, eps, gamma, beta, shift0, shift1,      \
                                                                 scale0, scale1, mod_div, mod_ld);                 \
        else                                                                                                       \
            layernorm_kernel<n, 1><<<grid, 256, 0, ctx.stream>>>(X, Y, rows, eps, gamma, beta, shift0, shift1,      \
                                                                 scale0, scale1, mod_div, mod_ld);                 \
        break;
    switch (D / 256) {
        WAN_LN_CASE(1) WAN_LN_CASE(2) WAN_LN_CASE(3) WAN_LN_CASE(4) WAN_LN_CASE(6) WAN_LN_CASE(8) WAN_LN_CASE(12)
        WAN_LN_CASE(16) WAN_LN_CASE(20) WAN_LN_CASE(24)
        default: return cudaErrorInvalidValue;
    }
#undef WAN_LN_CASE
    if (ctx.launches) ++*ctx.launches;
    return cudaGetLastError();
}

// ------------------------------------------------------------------ per-sample modulation, all blocks
// out[n][b][k][c] = sst[n][k][c] + tproj[b][k][c] + (k == 1 || k == 4 ? 1 : 0)
// (k: shift, scale, gate, c_shift, c_scale, c_gate; the "1 +" of the two scales folded in)
__global__ void mod_combine_kernel(const float* __restrict__ sst, const float* __restrict__ tproj, float* __restrict__ out,
                                   int N, int B, int D) {
    const long long total = (long long)N * B * 6 * D;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total; i += (long long)gridDim.x * blockDim.x) {
        const int c = i % D;
        const long long r = i / D;
        const int k = r % 6;
        const long long nb = r / 6;
        const int b = nb % B;
        const int n = nb / B;
        out[i] = sst[((long long)n * 6 + k) * D + c] + tproj[((long long)b * 6 + k) * D + c] + ((k == 1 || k == 4) ? 1.0f : 0.0f);
    }
}

cudaError_t launch_mod_combine(const float* sst, const float* tproj, float* out, int N, int B, int D,
                               const LaunchCtx& ctx) {
    const long long total = (long long)N * B * 6 * D;
    if (total <= 0) return cudaSuccess;
    long long g = (total + 255) / 256;
    if (g > ctx.num_sms * 8) g = ctx.num_sms * 8;
    mod_combine_kernel<<<(int)g, 256, 0, ctx.stream>>>(sst, tproj, out, N, B, D);
    if (ctx.launches) ++*ctx.launches;
    return cudaGetLastError();
}

// ------------------------------------------------------------------ RMSNorm across heads + RoPE

template <int NCH>
__global__ void __launch_bounds__(256) rmsnorm_rope_kernel(__nv_bfloat16* buf, long long ld, int rows, float eps,
                                                           const float* gains, long long gain_stride,
                                                           long long seg_stride, RopeTables rt, int use_rope,
                                                           int rope_L) {
    constexpr int D = NCH * 256;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * 8 + warp;
    if (row >= rows) return;
    const int seg = blockIdx.y;
    __nv_bfloat16* xr = buf + (long long)row * ld + seg * seg_stride;
    const float* g = gains + seg * gain_stride;
    float v[NCH][8];
    float ss = 0.f;
#pragma unroll
    for (int t = 0; t < NCH; ++t) {
        load8(xr + (t * 32 + lane) * 8, v[t]);
#pragma unroll
        for (int i = 0; i < 8; ++i) ss += v[t][i] * v[t][i];
    }
    const float rs = rsqrtf(warp_sum(ss) * (1.0f / D) + eps);
    int f = 0, ii = 0, jj = 0;
    if (use_rope) {
        const int l = row % rope_L;
        const int hw = rt.Hp * rt.Wp;
        f = l / hw;
        const int rem = l - f * hw;
        ii = rem / rt.Wp;
        jj = rem - ii * rt.Wp;
    }
#pragma unroll
    for (int t = 0; t < NCH; ++t) {
        const int c = (t * 32 + lane) * 8;
        float gg[8], o[8];
        load8f(g + c, gg);
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = v[t][i] * rs * gg[i];
        if (use_rope) {
            const int p0 = (c & 127) >> 1;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 cs = rope_cs(rt, p0 + k, f, ii, jj);
                const float a = o[2 * k], b = o[2 * k + 1];
                o[2 * k] = a * cs.x - b * cs.y;
                o[2 * k + 1] = a * cs.y + b * cs.x;
            }
        }
        store8(xr + c, o);
    }
}

// q and k of one token in one warp (the self-attention case): both rows are
// loaded before either reduction, and each cos/sin pair is fetched once for
// the two rotations.  q = buf[row, 0:D), k = buf[row, seg_stride:seg_stride+D).

template <int NCH>
__global__ void __launch_bounds__(256) rmsnorm_rope_qk_kernel(__nv_bfloat16* buf, long long ld, int rows, float eps,
                                                              const float* gains, long long gain_stride,
                                                              long long seg_stride, RopeTables rt, int rope_L) {
    constexpr int D = NCH * 256;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * 8 + warp;
    if (row >= rows) return;
    __nv_bfloat16* xq = buf + (long long)row * ld;
    __nv_bfloat16* xk = xq + seg_stride;
    uint4 uq[NCH], uk[NCH];
#pragma unroll
    for (int t = 0; t < NCH; ++t) {
        uq[t] = *reinterpret_cast<const uint4*>(xq + (t * 32 + lane) * 8);
        uk[t] = *reinterpret_cast<const uint4*>(xk + (t * 32 + lane) * 8);
    }
    const int l = row % rope_L;
    const int hw = rt.Hp * rt.Wp;
    const int f = l / hw;
    const int rem = l - f * hw;
    const int ii = rem / rt.Wp;
    const int jj = rem - ii * rt.Wp;
    float sq = 0.f, sk = 0.f;
#pragma unroll
    for (int t = 0; t < NCH; ++t) {
        float a[8], b[8];
        unpack8(uq[t], a);
        unpack8(uk[t], b);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            sq += a[i] * a[i];
            sk += b[i] * b[i];
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        sq += __shfl_xor_sync(0xffffffffu, sq, o);
        sk += __shfl_xor_sync(0xffffffffu, sk, o);
    }
    const float rq = rsqrtf(sq * (1.0f / D) + eps);
    const float rk = rsqrtf(sk * (1.0f / D) + eps);
#pragma unroll
    for (int t = 0; t < NCH; ++t) {
        const int c = (t * 32 + lane) * 8;
        float a[8], b[8], gq[8], gk[8];
        unpack8(uq[t], a);
        unpack8(uk[t], b);
        load8f(gains + c, gq);
        load8f(gains + gain_stride + c, gk);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            a[i] *= rq * gq[i];
            b[i] *= rk * gk[i];
        }
        const int p0 = (c & 127) >> 1;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 cs = rope_cs(rt, p0 + k, f, ii, jj);
            const float a0 = a[2 * k], a1 = a[2 * k + 1], b0 = b[2 * k], b1 = b[2 * k + 1];
            a[2 * k] = a0 * cs.x - a1 * cs.y;
            a[2 * k + 1] = a0 * cs.y + a1 * cs.x;
            b[2 * k] = b0 * cs.x - b1 * cs.y;
            b[2 * k + 1] = b0 * cs.y + b1 * cs.x;
        }
        store8(xq + c, a);
        store8(xk + c, b);
    }
}

bool rmsnorm_rope_shape_ok(int D, long long ld) {
    if (D <= 0 || D % 256 || ld % 8 || ld < D) return false;
    switch (D / 256) {
        case 1: case 2: case 3: case 4: case 6: case 8: case 12: case 16: case 20: case 24: return true;
        default: return false;
    }
}

cudaError_t launch_rmsnorm_rope(void* buf, long long ld, int rows, int D, float eps, const float* gains,
                                long long gain_stride, int nseg, long long seg_stride, const RopeTables* rope,
                                int rope_L, const LaunchCtx& ctx) {
    if (rows <= 0 || nseg <= 0) return cudaSuccess;
    if (!rmsnorm_rope_shape_ok(D, ld) || seg_stride % 8) return cudaErrorInvalidValue;
    RopeTables rt{};
    int use_rope = 0;
    if (rope) {
        rt = *rope;
        use_rope = 1;
        if (rope_L <= 0) return cudaErrorInvalidValue;
    } else {
        rope_L = 1;
    }
    auto Bp = reinterpret_cast<__nv_bfloat16*>(buf);
    if (use_rope && nseg == 2 && D <= 3072) {  // wider rows: two rows per warp would not fit in registers
#define WAN_RMS_QK_CASE(n)                                                                                     \
    case n:                                                                                                    \
        rmsnorm_rope_qk_kernel<n><<<(rows + 7) / 8, 256, 0, ctx.stream>>>(Bp, ld, rows, eps, gains, gain_stride, \
                                                                           seg_stride, rt, rope_L);            \
        break;
        switch (D / 256) {
            WAN_RMS_QK_CASE(1) WAN_RMS_QK_CASE(2) WAN_RMS_QK_CASE(3) WAN_RMS_QK_CASE(4) WAN_RMS_QK_CASE(6)
            WAN_RMS_QK_CASE(8) WAN_RMS_QK_CASE(12)
            default: return cudaErrorInvalidValue;
        }
#undef WAN_RMS_QK_CASE
        if (ctx.launches) ++*ctx.launches;
        return cudaGetLastError();
    }
    dim3 grid((rows + 7) / 8, nseg);
#define WAN_RMS_CASE(n)                                                                                           \
    case n:                                                                                                       \
        rmsnorm_rope_kernel<n><<<grid, 256, 0, ctx.stream>>>(Bp, ld, rows, eps, gains, gain_stride, seg_stride, rt, \
                                                             use_rope, rope_L);                                   \
        break;
    switch (D / 256) {
        WAN_RMS_CASE(1) WAN_RMS_CASE(2) WAN_RMS_CASE(3) WAN_RMS_CASE(4) WAN_RMS_CASE(6) WAN_RMS_CASE(8)
        WAN_RMS_CASE(12) WAN_RMS_CASE(16) WAN_RMS_CASE(20) WAN_RMS_CASE(24)
        default: return cudaErrorInvalidValue;
    }
#undef WAN_RMS_CASE
    if (ctx.launches) ++*ctx.launches;
    return cudaGetLastError();
}

// ------------------------------------------------------------------ RMSNorm row factor applied in place
// The sums of squares come from the q/k projection's epilogue; one warp per
// row, the row factor from the row's group sums (fixed order), 16-byte
// vectors, every load of the row issued before any store.
template <int NCH>
__global__ void __launch_bounds__(256) rms_apply_kernel(__nv_bfloat16* buf, long long ld, int rows, RowNorm rn) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * 8 + warp;
    if (row >= rows) return;
    __nv_bfloat16* xr = buf + (long long)row * ld;
    uint4 u[NCH];
#pragma unroll
    for (int t = 0; t < NCH; ++t) u[t] = *reinterpret_cast<const uint4*>(xr + (t * 32 + lane) * 8);
    const float* g = rn.ssq + (long long)row * rn.ssq_ld;
    float ss = 0.f;
    for (int k = 0; k < rn.ngroups; ++k) ss += __ldg(g + k);
    const float sc = rsqrtf(ss * rn.inv_n + rn.eps);
    const uint64_t sc2 = f2pack(sc, sc);
#pragma unroll
    for (int t = 0; t < NCH; ++t) {
        const uint32_t w[4] = {u[t].x, u[t].y, u[t].z, u[t].w};
        uint32_t o[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const float2 f = unpack_bf16(w[h]);
            float a, b;
            f2unpack(mul2(f2pack(f.x, f.y), sc2), a, b);
            o[h] = pack_bf16(a, b);
        }
        *reinterpret_cast<uint4*>(xr + (t * 32 + lane) * 8) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

cudaError_t launch_rms_apply(void* buf, long long ld, int rows, int D, const RowNorm& rn, const LaunchCtx& ctx) {
    if (rows <= 0) return cudaSuccess;
    if (!rn.ssq || rn.ngroups <= 0 || !rmsnorm_rope_shape_ok(D, ld) ||
        (reinterpret_cast<uintptr_t>(buf) & 15))
        return cudaErrorInvalidValue;
    auto Bp = reinterpret_cast<__nv_bfloat16*>(buf);
    const int grid = (rows + 7) / 8;
#define WAN_RMS_APPLY_CASE(n)                                                             \
    case n:                                                                               \
        rms_apply_kernel<n><<<grid, 256, 0, ctx.stream>>>(Bp, ld, rows, rn);              \
        break;
    switch (D / 256) {
        WAN_RMS_APPLY_CASE(1) WAN_RMS_APPLY_CASE(2) WAN_RMS_APPLY_CASE(3) WAN_RMS_APPLY_CASE(4)
        WAN_RMS_APPLY_CASE(6) WAN_RMS_APPLY_CASE(8) WAN_RMS_APPLY_CASE(12) WAN_RMS_APPLY_CASE(16)
        WAN_RMS_APPLY_CASE(20) WAN_RMS_APPLY_CASE(24)
        default: return cudaErrorInvalidValue;
    }
#undef WAN_RMS_APPLY_CASE
    if (ctx.launches) ++*ctx.launches;
    return cudaGetLastError();
}

// ------------------------------------------------------------------ sequence-parallel exchange layouts
// pack:   send[((b * P + j) * Ls + l) * 3hd + s * hd + c] = qkv[(b * Ls + l) * 3D + s * D + j * hd + c]
// unpack: o[(b * Ls + l) * D + j * hd + c]               = back[((b * P + j) * Ls + l) * hd + c]
// (s = q, k, v; hd = 128 * heads / P columns of head group j); 8 bf16 per thread step.
__global__ void sp_pack_kernel(const __nv_bfloat16* __restrict__ qkv, __nv_bfloat16* __restrict__ send, int B, int P,
                               int Ls, int D, int hd) {
    const int v8 = 3 * hd / 8;  // 16-byte vectors per packed row
    const long long total = (long long)B * P * Ls * v8;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int c8 = idx % v8;
        const long long rest = idx / v8;
        const int l = rest % Ls;
        const long long bj = rest / Ls;
        const int j = bj % P;
        const int b = bj / P;
        const int sidx = c8 / (hd / 8), cc = (c8 % (hd / 8)) * 8;
        const uint4 v = *reinterpret_cast<const uint4*>(qkv + ((long long)b * Ls + l) * 3 * D + (long long)sidx * D +
                                                        (long long)j * hd + cc);
        *reinterpret_cast<uint4*>(send + idx * 8) = v;
    }
}

__global__ void sp_unpack_kernel(const __nv_bfloat16* __restrict__ back, __nv_bfloat16* __restrict__ o, int B, int P,
                                 int Ls, int D, int hd) {
    const int v8 = hd / 8;
    const long long total = (long long)B * P * Ls * v8;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int c8 = idx % v8;
        const long long rest = idx / v8;
        const int l = rest % Ls;
        const long long bj = rest / Ls;
        const int j = bj % P;
        const int b = bj / P;
        const uint4 v = *reinterpret_cast<const uint4*>(back + idx * 8);
        *reinterpret_cast<uint4*>(o + ((long long)b * Ls + l) * D + (long long)j * hd + c8 * 8) = v;
    }
}

cudaError_t launch_sp_pack(const void* qkv, void* send, int B, int P, int Ls, int D, const LaunchCtx& ctx) {
    if (B <= 0 || Ls <= 0) return cudaSuccess;
    if (P <= 0 || D % P || (D / P) % 8 || ((reinterpret_cast<uintptr_t>(qkv) | reinterpret_cast<uintptr_t>(send)) & 15))
        return cudaErrorInvalidValue;
    const long long total = (long long)B * Ls * 3 * D / 8;
    long long g = (total + 255) / 256;
    if (g > ctx.num_sms * 16) g = ctx.num_sms * 16;
    sp_pack_kernel<<<(int)g, 256, 0, ctx.stream>>>(reinterpret_cast<const __nv_bfloat16*>(qkv),
                                                  reinterpret_cast<__nv_bfloat16*>(send), B, P, Ls, D, D / P);
    if (ctx.launches) ++*ctx.launches;
    return cudaGetLastError();
}

cudaError_t launch_sp_unpack(const void* back, void* o, int B, int P, int Ls, int D, const LaunchCtx& ctx) {
    if (B <= 0 || Ls <= 0) return cudaSuccess;
    if (P <= 0 || D % P || (D / P) % 8 || ((reinterpret_cast<uintptr_t>(back) | reinterpret_cast<uintptr_t>(o)) & 15))
        return cudaErrorInvalidValue;
    const long long total = (long long)B * Ls * D / 8;
    long long g = (total + 255) / 256;
    if (g > ctx.num_sms * 16) g = ctx.num_sms * 16;
    sp_unpack_kernel<<<(int)g, 256, 0, ctx.stream>>>(reinterpret_cast<const __nv_bfloat16*>(back),
                                                    reinterpret_cast<__nv_bfloat16*>(o), B, P, Ls, D, D / P);
    if (ctx.launches) ++*ctx.launches;
    return cudaGetLastError();
}

// ------------------------------------------------------------------ patchify / unpatchify
// X[b * L + (f * Hp + i) * Wp + j, c * 4 + kh * 2 + kw] = latent[b, c, f, 2i + kh, 2j + kw]
// for c < C; columns [4C, ldx) of every row are written as zeros (K padding of
// the patch GEMM when 4C is not a multiple of its K tile).
template <typename T>
__global__ void patchify_kernel(const T* __restrict__ lat, __nv_bfloat16* __restrict__ X, int B, int C, int F, int Hz,
                                int Wz, int ldx, int tok0, int rows) {
    const int Hp = Hz >> 1, Wp = Wz >> 1;
    const long long L = (long long)F * Hp * Wp;
    const int G = ldx >> 2;  // groups of 4 columns per row
    const long long total = (long long)B * rows * G;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int c = idx % G;
        const long long row = idx / G;
        uint2 u = make_uint2(0u, 0u);
        const int b = row / rows;
        const long long l = tok0 + (row - (long long)b * rows);
        if (c < C && l < L) {
            const int f = l / (Hp * Wp);
            const int rem = l - (long long)f * (Hp * Wp);
            const int i = rem / Wp, j = rem - (rem / Wp) * Wp;
            const T* src = lat + ((((long long)b * C + c) * F + f) * Hz + 2 * i) * Wz + 2 * j;
            float a = (float)src[0], bb = (float)src[1], cc = (float)src[Wz], d = (float)src[Wz + 1];
            u = make_uint2(pack_bf16(a, bb), pack_bf16(cc, d));
        }
        *reinterpret_cast<uint2*>(X + row * ldx + 4 * c) = u;
    }
}

cudaError_t launch_patchify(const void* latent, int latent_dtype, int B, int C, int F, int Hz, int Wz, void* X,
                            int ldx, const LaunchCtx& ctx, int tok0, int rows) {
    if (ldx < 4 * C || ldx % 4 || tok0 < 0 || rows < 0) return cudaErrorInvalidValue;
    if (rows == 0) {
        rows = F * (Hz / 2) * (Wz / 2);
        tok0 = 0;
    }
    const long long total = (long long)B * rows * (ldx / 4);
    if (total <= 0) return cudaSuccess;
    int grid = (int)((total + 255) / 256);
    if (grid > ctx.num_sms * 16) grid = ctx.num_sms * 16;
    if (latent_dtype == 0)
        patchify_kernel<float><<<grid, 256, 0, ctx.stream>>>(reinterpret_cast<const float*>(latent),
                                                              reinterpret_cast<__nv_bfloat16*>(X), B, C, F, Hz, Wz,
                                                              ldx, tok0, rows);
    else
        patchify_kernel<__nv_bfloat16><<<grid, 256, 0, ctx.stream>>>(reinterpret_cast<const __nv_bfloat16*>(latent),
                                                                      reinterpret_cast<__nv_bfloat16*>(X), B, C, F, Hz,
                                                                      Wz, ldx, tok0, rows);
    if (ctx.launches) ++*ctx.launches;
    return cudaGetLastError();
}

// ------------------------------------------------------------------ causal Conv3d im2col (channels last)
// col[row, k] for row = ((b * T + t) * H + h) * W + w and k = tap * Ci + c,
// tap = (it * kh + ih) * kw + iw: the input at frame t - (kt - 1) + it,
// row h - (kh - 1) / 2 + ih, column w - (kw - 1) / 2 + iw, channel c.  Frames
// before 0 come from the cache (its last frames sit right before frame 0),
// else zero; rows/columns outside the frame are zero; k in [taps * Ci, Kp) is
// zero padding.  8 channels (16 bytes) per thread step.
__global__ void causal_im2col_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ cache,
                                     int nc, int B, int T, int H, int W, int Ci, int kt, int kh, int kw,
                                     __nv_bfloat16* __restrict__ col, int Kp) {
    const int C8 = Ci >> 3, Kp8 = Kp >> 3;
    const long long K8 = (long long)kt * kh * kw * C8;
    const long long total = (long long)B * T * H * W * Kp8;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const long long row = idx / Kp8;
        const int k8 = (int)(idx - row * Kp8);
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (k8 < K8) {
            const int tap = k8 / C8, c8 = k8 - tap * C8;
            const int it = tap / (kh * kw), ih = (tap / kw) % kh, iw = tap % kw;
            const int w0 = (int)(row % W);
            const int h0 = (int)((row / W) % H);
            const int t0 = (int)((row / ((long long)W * H)) % T);
            const int b0 = (int)(row / ((long long)W * H * T));
            const int tt = t0 - (kt - 1) + it, hh = h0 - (kh - 1) / 2 + ih, ww = w0 - (kw - 1) / 2 + iw;
            if (hh >= 0 && hh < H && ww >= 0 && ww < W) {
                if (tt >= 0)
                    v = *reinterpret_cast<const uint4*>(x + ((((long long)b0 * T + tt) * H + hh) * W + ww) * Ci + c8 * 8);
                else if (cache && tt >= -nc)
                    v = *reinterpret_cast<const uint4*>(
                        cache + ((((long long)b0 * nc + (nc + tt)) * H + hh) * W + ww) * Ci + c8 * 8);
            }
        }
        *reinterpret_cast<uint4*>(col + row * Kp + (long long)k8 * 8) = v;
    }
}

cudaError_t launch_causal_im2col(const void* x, const void* cache, int nc, int B, int T, int H, int W, int Ci, int kt,
                                 int kh, int kw, void* col, int Kp, const LaunchCtx& ctx) {
    if (Ci % 8 || Kp % 8 || (long long)kt * kh * kw * Ci > Kp) return cudaErrorInvalidValue;
    const long long total = (long long)B * T * H * W * (Kp / 8);
    if (total <= 0) return cudaSuccess;
    long long g = (total + 255) / 256;
    if (g > ctx.num_sms * 16) g = ctx.num_sms * 16;
    causal_im2col_kernel<<<(int)g, 256, 0, ctx.stream>>>(reinterpret_cast<const __nv_bfloat16*>(x),
                                                        reinterpret_cast<const __nv_bfloat16*>(cache), nc, B, T, H, W,
                                                        Ci, kt, kh, kw, reinterpret_cast<__nv_bfloat16*>(col), Kp);
    if (ctx.launches) ++*ctx.launches;
    return cudaGetLastError();
}

// ------------------------------------------------------------------ a += b (bf16, fp32 sum, one rounding)
__global__ void add_bf16_kernel(__nv_bfloat16* __restrict__ a, const __nv_bfloat16* __restrict__ b, long long n8) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n8; i += (long long)gridDim.x * blockDim.x) {
        float x[8], y[8];
        load8(a + i * 8, x);
        load8(b + i * 8, y);
#pragma unroll
        for (int k = 0; k < 8; ++k) x[k] += y[k];
        store8(a + i * 8, x);
    }
}

cudaError_t launch_add_bf16(void* a, const void* b, long long n, const LaunchCtx& ctx) {
    if (n <= 0) return cudaSuccess;
    if (n % 8 || ((reinterpret_cast<uintptr_t>(a) | reinterpret_cast<uintptr_t>(b)) & 15)) return cudaErrorInvalidValue;
    const long long n8 = n / 8;
    long long g = (n8 + 255) / 256;
    if (g > ctx.num_sms * 16) g = ctx.num_sms * 16;
    add_bf16_kernel<<<(int)g, 256, 0, ctx.stream>>>(reinterpret_cast<__nv_bfloat16*>(a),
                                                   reinterpret_cast<const __nv_bfloat16*>(b), n8);
    if (ctx.launches) ++*ctx.launches;
    return cudaGetLastError();
}

// vel[b, ch, f, 2i + kh, 2j + kw] = rows[b * L + token, (kh * 2 + kw) * C + ch]
__global__ void unpatchify_kernel(const float* __restrict__ rows, float* __restrict__ vel, int B, int C, int F, int Hz,
                                  int Wz) {
    const int Hp = Hz >> 1, Wp = Wz >> 1;
    const long long L = (long long)F * Hp * Wp;
    const long long total = (long long)B * L * 4 * C;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int col = idx % (4 * C);
        const long long row = idx / (4 * C);
        const int b = row / L;
        const long long l = row - (long long)b * L;
        const int f = l / (Hp * Wp);
        const int rem = l - (long long)f * (Hp * Wp);
        const int i = rem / Wp, j = rem - (rem / Wp) * Wp;
        const int ch = col % C, s = col / C, kh = s >> 1, kw = s & 1;
        vel[((((long long)b * C + ch) * F + f) * Hz + 2 * i + kh) * Wz + 2 * j + kw] = rows[idx];
    }
}

cudaError_t launch_unpatchify(const float* rows, int B, int C, int F, int Hz, int Wz, float* vel,
                              const LaunchCtx& ctx) {
    const long long total = (long long)B * F * (Hz / 2) * (Wz / 2) * 4 * C;
    if (total <= 0) return cudaSuccess;
    int grid = (int)((total + 255) / 256);
    if (grid > ctx.num_sms * 16) grid = ctx.num_sms * 16;
    unpatchify_kernel<<<grid, 256, 0, ctx.stream>>>(rows, vel, B, C, F, Hz, Wz);
    if (ctx.launches) ++*ctx.launches;
    return cudaGetLastError();
}

// ------------------------------------------------------------------ small GEMV (timestep MLP)
// One warp per output column n, all B rows of x at once (B <= 8).
__global__ void __launch_bounds__(256) gemv_kernel(const __nv_bfloat16* __restrict__ W, const float* __restrict__ bias,
                                                   const float* __restrict__ x, long long ldx, float* __restrict__ out,
                                                   long long ldout, int B, int N, int K, int act_in, int act_out) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = blockIdx.x * 8 + warp;
    if (n >= N) return;
    float acc[8];
#pragma unroll
    for (int b = 0; b < 8; ++b) acc[b] = 0.f;
    const __nv_bfloat16* w = W + (long long)n * K;
    const int half = K / 2;
    for (int k0 = lane * 8; k0 < K; k0 += 256) {
        float wv[8];
        load8(w + k0, wv);
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            if (b >= B) break;
            float xv[8];
            if (act_in == 2) {
                // timestep sinusoid: [cos(t w_k), sin(t w_k)], w_k = 1e4^(-k / half), computed in double
                const double t = (double)x[b * ldx];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int k = k0 + i;
                    const int kk = k < half ? k : k - half;
                    const double w_k = exp(-9.210340371976184 * (double)kk / (double)half);  // ln(1e4)
                    xv[i] = (float)(k < half ? cos(t * w_k) : sin(t * w_k));
                }
            } else {
                load8f(x + b * ldx + k0, xv);
                if (act_in == 1) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) xv[i] = xv[i] / (1.0f + __expf(-xv[i]));
                }
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[b] = fmaf(wv[i], xv[i], acc[b]);
        }
    }
#pragma unroll
    for (int b = 0; b < 8; ++b) {
        if (b >= B) break;
        float s = warp_sum(acc[b]);
        if (lane == 0) {
            s += bias ? bias[n] : 0.f;
            if (act_out == 1) s = s / (1.0f + __expf(-s));
            out[b * ldout + n] = s;
        }
    }
}

cudaError_t launch_gemv(const void* W, const float* bias, const float* x, long long ldx, float* out, long long ldout,
                        int B, int N, int K, int act_in, int act_out, const LaunchCtx& ctx) {
    if (B <= 0 || N <= 0) return cudaSuccess;
    if (B > 8 || K % 8) return cudaErrorInvalidValue;
    gemv_kernel<<<(N + 7) / 8, 256, 0, ctx.stream>>>(reinterpret_cast<const __nv_bfloat16*>(W), bias, x, ldx, out,
                                                      ldout, B, N, K, act_in, act_out);
    if (ctx.launches) ++*ctx.launches;
    return cudaGetLastError();
}

// ------------------------------------------------------------------ per-token timestep features
__global__ void sinusoid_kernel(const float* __restrict__ t, long long n, int dim, __nv_bfloat16* __restrict__ out) {
    const int half = dim / 2;
    const long long total = n * dim;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const long long r = idx / dim;
        const int k = idx - r * dim;
        const int kk = k < half ? k : k - half;
        const double w_k = exp(-9.210340371976184 * (double)kk / (double)half);  // ln(1e4)
        const double a = (double)t[r] * w_k;
        out[idx] = __float2bfloat16_rn((float)(k < half ? cos(a) : sin(a)));
    }
}

cudaError_t launch_sinusoid_bf16(const float* t, long long n, int dim, void* out, const LaunchCtx& ctx) {
    if (n <= 0) return cudaSuccess;
    long long g = (n * dim + 255) / 256;
    if (g > ctx.num_sms * 16) g = ctx.num_sms * 16;
    sinusoid_kernel<<<(int)g, 256, 0, ctx.stream>>>(t, n, dim, reinterpret_cast<__nv_bfloat16*>(out));
    if (ctx.launches) ++*ctx.launches;
    return cudaGetLastError();
}

__global__ void silu_bf16_kernel(const float* __restrict__ x, __nv_bfloat16* __restrict__ out, long long n) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        const float v = x[i];
        out[i] = __float2bfloat16_rn(v / (1.0f + __expf(-v)));
    }
}

cudaError_t launch_silu_bf16(const float* x, void* out, long long n, const LaunchCtx& ctx) {
    if (n <= 0) return cudaSuccess;
    long long g = (n + 255) / 256;
    if (g > ctx.num_sms * 16) g = ctx.num_sms * 16;
    silu_bf16_kernel<<<(int)g, 256, 0, ctx.stream>>>(x, reinterpret_cast<__nv_bfloat16*>(out), n);
    if (ctx.launches) ++*ctx.launches;
    return cudaGetLastError();
}

// ------------------------------------------------------------------ flow-matching sampler step
// x_next = x + (sigma_next - sigma) * (v_u + s (v_c - v_u))   (v = v_c when v_u is null)
__global__ void cfg_euler_kernel(const float* __restrict__ x, const float* __restrict__ vc,
                                 const float* __restrict__ vu, float s, float dsigma, long long n,
                                 float* __restrict__ xn) {
    const long long n4 = n / 4;
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4; i += stride) {
        const float4 a = reinterpret_cast<const float4*>(x)[i];
        const float4 c = reinterpret_cast<const float4*>(vc)[i];
        float4 v = c;
        if (vu) {  // fused multiply-adds spelled out: the proj_out epilogue computes the same roundings
            const float4 u = reinterpret_cast<const float4*>(vu)[i];
            v = make_float4(__fmaf_rn(s, c.x - u.x, u.x), __fmaf_rn(s, c.y - u.y, u.y), __fmaf_rn(s, c.z - u.z, u.z),
                            __fmaf_rn(s, c.w - u.w, u.w));
        }
        reinterpret_cast<float4*>(xn)[i] = make_float4(__fmaf_rn(dsigma, v.x, a.x), __fmaf_rn(dsigma, v.y, a.y),
                                                       __fmaf_rn(dsigma, v.z, a.z), __fmaf_rn(dsigma, v.w, a.w));
    }
    for (long long i = n4 * 4 + blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += stride) {
        const float v = vu ? __fmaf_rn(s, vc[i] - vu[i], vu[i]) : vc[i];
        xn[i] = __fmaf_rn(dsigma, v, x[i]);
    }
}

cudaError_t launch_cfg_euler(const float* x, const float* v_cond, const float* v_uncond, float guidance, float sigma,
                             float sigma_next, long long n, float* x_next, const LaunchCtx& ctx) {
    if (n <= 0) return cudaSuccess;
    if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(v_cond) |
         reinterpret_cast<uintptr_t>(v_uncond) | reinterpret_cast<uintptr_t>(x_next)) & 15)
        return cudaErrorInvalidValue;
    long long g = (n / 4 + 255) / 256;
    if (g < 1) g = 1;
    if (g > ctx.num_sms * 8) g = ctx.num_sms * 8;
    cfg_euler_kernel<<<(int)g, 256, 0, ctx.stream>>>(x, v_cond, v_uncond, guidance, sigma_next - sigma, n, x_next);
    if (ctx.launches) ++*ctx.launches;
    return cudaGetLastError();
}

// ------------------------------------------------------------------ per-call sampler scalars
// sched = {guidance, sigma_next - sigma}; t[0..nt) = t_value.  Kernel arguments
// carry the values, so a captured forward reads them from device memory.
__global__ void set_sampler_scalars_kernel(float* sched, float guidance, float dsigma, float* t, int nt,
                                           float t_value) {
    const int i = threadIdx.x;
    if (i == 0) {
        sched[0] = guidance;
        sched[1] = dsigma;
    }
    for (int k = i; k < nt; k += blockDim.x) t[k] = t_value;
}

cudaError_t launch_set_sampler_scalars(float* sched, float guidance, float dsigma, float* t, int nt, float t_value,
                                       const LaunchCtx& ctx) {
    set_sampler_scalars_kernel<<<1, 32, 0, ctx.stream>>>(sched, guidance, dsigma, t, nt, t_value);
    if (ctx.launches) ++*ctx.launches;
    return cudaGetLastError();
}

// ------------------------------------------------------------------ bounded-wait self-test
// One warp waits on an mbarrier that nothing ever arrives on; the bounded wait
// gives up after limit_ns, raises the CTA's abort flag and records the timeout.
__global__ void wait_selftest_kernel(int* err, unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    WaitCtl wc{err, limit_ns};
    mbar_wait(&bar, 0, &abort_flag, wc);
}

cudaError_t launch_wait_selftest(uint64_t limit_ns, const LaunchCtx& ctx) {
    wait_selftest_kernel<<<1, 32, 0, ctx.stream>>>(ctx.err, limit_ns);
    if (ctx.launches) ++*ctx.launches;
    return cudaGetLastError();
}

// ------------------------------------------------------------------ dtype conversion
__global__ void convert_kernel(const void* src, int sd, void* dst, int dd, long long n) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        float v = sd == 0 ? reinterpret_cast<const float*>(src)[i]
                          : __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(src)[i]);
        if (dd == 0)
            reinterpret_cast<float*>(dst)[i] = v;
        else
            reinterpret_cast<__nv_bfloat16*>(dst)[i] = __float2bfloat16_rn(v);
    }
}

cudaError_t launch_convert(const void* src, int src_dtype, void* dst, int dst_dtype, long long n,
                           cudaStream_t stream) {
    if (n <= 0) return cudaSuccess;
    long long g = (n + 255) / 256;
    if (g > 4096) g = 4096;
    convert_kernel<<<(int)g, 256, 0, stream>>>(src, src_dtype, dst, dst_dtype, n);
    return cudaGetLastError();
}

}  // namespace wan

// Wan2.1 VAE decoder on the GPU: the C ABI of include/wanvae.h.
//
// The decoder walk-through of the pswp.cn WanPipeline notes ("vae.decode",
// "WanDecoder3d", "WanCausalConv3d", "upsample blocks"), run latent frame by
// latent frame with a 2-frame cache per causal convolution.  Activations are
// channels-last bf16 [B, T, H, W, C]; every convolution is the implicit-GEMM
// tcgen05 kernel of conv.cu (taps gathered by TMA from the activation or the
// frame cache), the mid-block attention is three library GEMMs around a row
// softmax, and the norms / upsampling / layout changes are bandwidth kernels
// below.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <initializer_list>
#include <map>
#include <set>
#include <string>
#include <vector>

#include "../../include/wanvae.h"
#include "common.cuh"
#include "kernels.h"

namespace wan {
namespace {

constexpr int Z_DIM = 16;
constexpr float NORM_EPS = 1e-12f;

// ------------------------------------------------------------------ bandwidth kernels
// Channel RMS norm of channels-last rows, y = x rsqrt(mean_c x^2 + eps) gamma + beta,
// then SiLU when asked.  LPP lanes per pixel (16 or 32), up to 2 16-byte vectors
// per lane (C <= 512), fp32 statistics.
template <int LPP>
__global__ void __launch_bounds__(256) chan_rmsnorm_kernel(const __nv_bfloat16* __restrict__ x, __nv_bfloat16* __restrict__ y,
                                                           long long P, int C, const float* __restrict__ g,
                                                           const float* __restrict__ beta, float eps, int silu) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long pix = ((long long)blockIdx.x * 8 + warp) * (32 / LPP) + lane / LPP;
    const int sub = lane % LPP;
    const int nv = C / 8;
    const bool live = pix < P;
    const __nv_bfloat16* xr = x + (live ? pix : 0) * C;
    uint4 u[2];
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int v = sub + k * LPP;
        u[k] = make_uint4(0u, 0u, 0u, 0u);
        if (live && v < nv) u[k] = *reinterpret_cast<const uint4*>(xr + v * 8);
        const uint32_t w[4] = {u[k].x, u[k].y, u[k].z, u[k].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = unpack_bf16(w[i]);
            ss += f.x * f.x + f.y * f.y;
        }
    }
#pragma unroll
    for (int o = LPP / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o, LPP);
    if (!live) return;
    const float rs = rsqrtf(ss / C + eps);
    __nv_bfloat16* yr = y + pix * C;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int v = sub + k * LPP;
        if (v >= nv) continue;
        const uint32_t w[4] = {u[k].x, u[k].y, u[k].z, u[k].w};
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = unpack_bf16(w[i]);
            const int c = v * 8 + 2 * i;
            float a = f.x * rs * __ldg(g + c) + __ldg(beta + c);
            float b = f.y * rs * __ldg(g + c + 1) + __ldg(beta + c + 1);
            if (silu) {
                a = a / (1.0f + __expf(-a));
                b = b / (1.0f + __expf(-b));
            }
            o[i] = pack_bf16(a, b);
        }
        *reinterpret_cast<uint4*>(yr + v * 8) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

cudaError_t launch_chan_rmsnorm(const void* x, void* y, long long P, int C, const float* g, const float* b, int silu,
                                const LaunchCtx& ctx) {
    if (P <= 0) return cudaSuccess;
    if (C % 8 || C > 512) return cudaErrorInvalidValue;
    const int lpp = (C / 8 <= 16) ? 16 : 32;
    const long long per_block = 8LL * (32 / lpp);
    const long long grid = (P + per_block - 1) / per_block;
    auto X = reinterpret_cast<const __nv_bfloat16*>(x);
    auto Y = reinterpret_cast<__nv_bfloat16*>(y);
    if (lpp == 16)
        chan_rmsnorm_kernel<16><<<(unsigned)grid, 256, 0, ctx.stream>>>(X, Y, P, C, g, b, NORM_EPS, silu);
    else
        chan_rmsnorm_kernel<32><<<(unsigned)grid, 256, 0, ctx.stream>>>(X, Y, P, C, g, b, NORM_EPS, silu);
    return cudaGetLastError();
}

// Nearest 2x spatial upsampling of channels-last frames: y[n, i, j] = x[n, i / 2, j / 2].
__global__ void upsample2x_kernel(const __nv_bfloat16* __restrict__ x, __nv_bfloat16* __restrict__ y, long long N, int H,
                                  int W, int C) {
    const int c8n = C / 8;
    const long long total = N * 2 * H * 2 * W * c8n;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int c8 = idx % c8n;
        long long r = idx / c8n;
        const int j = r % (2 * W);
        r /= 2 * W;
        const int i = r % (2 * H);
        const long long n = r / (2 * H);
        reinterpret_cast<uint4*>(y)[idx] =
            *reinterpret_cast<const uint4*>(x + (((n * H + i / 2) * W + j / 2) * C + c8 * 8));
    }
}

// Softmax of the first Lk columns of each fp32 row of S (scaled), written as bf16
// P with zeros past Lk up to ldp.  One block per row, three passes over the row.
__global__ void __launch_bounds__(256) softmax_rows_kernel(const float* __restrict__ S, long long lds, int Lk, float scale,
                                                           __nv_bfloat16* __restrict__ P, long long ldp) {
    __shared__ float red[32];
    const float* s = S + (long long)blockIdx.x * lds;
    __nv_bfloat16* pr = P + (long long)blockIdx.x * ldp;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    auto block_reduce = [&](float v, bool is_max) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float w = __shfl_xor_sync(0xffffffffu, v, o);
            v = is_max ? fmaxf(v, w) : v + w;
        }
        __syncthreads();
        if (lane == 0) red[warp] = v;
        __syncthreads();
        v = lane < (int)(blockDim.x >> 5) ? red[lane] : (is_max ? -INFINITY : 0.0f);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float w = __shfl_xor_sync(0xffffffffu, v, o);
            v = is_max ? fmaxf(v, w) : v + w;
        }
        return v;
    };
    float m = -INFINITY;
    for (int k = tid; k < Lk; k += blockDim.x) m = fmaxf(m, s[k] * scale);
    m = block_reduce(m, true);
    float sum = 0.f;
    for (int k = tid; k < Lk; k += blockDim.x) sum += expf(s[k] * scale - m);
    sum = block_reduce(sum, false);
    const float inv = 1.0f / sum;
    for (int k = tid; k < ldp; k += blockDim.x)
        pr[k] = __float2bfloat16_rn(k < Lk ? expf(s[k] * scale - m) * inv : 0.0f);
}

// vt[c, l] = v[l * ldv + c] for l < L, 0 for L <= l < Lp (32 x 32 tiles through shared memory).
__global__ void transpose_pad_kernel(const __nv_bfloat16* __restrict__ v, long long ldv, int L, int C,
                                     __nv_bfloat16* __restrict__ vt, int Lp) {
    __shared__ __nv_bfloat16 tile[32][33];
    const int l0 = blockIdx.x * 32, c0 = blockIdx.y * 32;
    for (int r = threadIdx.y; r < 32; r += blockDim.y) {
        const int l = l0 + r, c = c0 + threadIdx.x;
        tile[r][threadIdx.x] = (l < L && c < C) ? v[(long long)l * ldv + c] : __float2bfloat16_rn(0.0f);
    }
    __syncthreads();
    for (int r = threadIdx.y; r < 32; r += blockDim.y) {
        const int c = c0 + r, l = l0 + threadIdx.x;
        if (c < C && l < Lp) vt[(long long)c * Lp + l] = tile[threadIdx.x][r];
    }
}

// video[b, ch, t0 + t, h, w] = clamp(y[((b T + t) H + h) W + w, ch], -1, 1) for ch < 3.
__global__ void to_video_kernel(const __nv_bfloat16* __restrict__ y, long long ldy, int B, int T, int H, int W,
                                float* __restrict__ video, int Ttot, int t0) {
    const long long total = (long long)B * 3 * T * H * W;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int w = idx % W;
        long long r = idx / W;
        const int h = r % H;
        r /= H;
        const int t = r % T;
        r /= T;
        const int ch = r % 3;
        const int b = r / 3;
        const float v = __bfloat162float(y[((((long long)b * T + t) * H + h) * W + w) * ldy + ch]);
        video[((((long long)b * 3 + ch) * Ttot + t0 + t) * H + h) * W + w] = fminf(1.0f, fmaxf(-1.0f, v));
    }
}

// z [B, Cz, T, H, W] f32 -> channels-last bf16 [B, T, H, W, Cz].
__global__ void latent_to_cl_kernel(const float* __restrict__ z, __nv_bfloat16* __restrict__ out, int B, int Cz, int T,
                                    int H, int W) {
    const long long total = (long long)B * Cz * T * H * W;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int c = idx % Cz;
        long long r = idx / Cz;
        const int w = r % W;
        r /= W;
        const int h = r % H;
        r /= H;
        const int t = r % T;
        const int b = r / T;
        out[idx] = __float2bfloat16_rn(z[((((long long)b * Cz + c) * T + t) * H + h) * W + w]);
    }
}

// Repack one convolution weight W[Co, Ci, taps] (f32 or bf16) into the K-major
// implicit-GEMM layout out[co, tap * cip + ci] (out zeroed beforehand).
__global__ void pack_conv_weight_kernel(const void* __restrict__ in, int in_bf16, int Co, int Ci, int taps, int cip,
                                        __nv_bfloat16* __restrict__ out, long long ldw) {
    const long long total = (long long)Co * Ci * taps;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int tap = idx % taps;
        const long long r = idx / taps;
        const int ci = r % Ci;
        const int co = r / Ci;
        const float v = in_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(in)[idx])
                                : reinterpret_cast<const float*>(in)[idx];
        out[(long long)co * ldw + (long long)tap * cip + ci] = __float2bfloat16_rn(v);
    }
}

int grid_for(long long total, int sms) {
    long long g = (total + 255) / 256;
    if (g < 1) g = 1;
    if (g > (long long)sms * 16) g = (long long)sms * 16;
    return (int)g;
}

// ------------------------------------------------------------------ decoder description
enum Kind { K_CONV, K_RES, K_ATTN, K_UP3D, K_UP2D, K_NORM };
struct Entry {
    Kind kind;
    std::string name;
    int a, b;       // conv / res: cin, cout; attn / up / norm: channels
    int k;          // conv: kernel size (1 or 3, cubic)
    int scale;      // spatial scale of the level the entry runs at (1, 2, 4, 8)
};

// Module list in execution order: conv_in, mid block, four up blocks of three
// residual blocks (widths 384, 384, 192, 96), upsamplers after blocks 0, 1 (time
// + space) and 2 (space), head.
std::vector<Entry> decoder_layout() {
    const int dims[5] = {384, 384, 384, 192, 96};
    std::vector<Entry> L;
    L.push_back({K_CONV, "post_quant_conv", Z_DIM, Z_DIM, 1, 1});
    L.push_back({K_CONV, "decoder.conv_in", Z_DIM, dims[0], 3, 1});
    L.push_back({K_RES, "decoder.mid_block.resnets.0", dims[0], dims[0], 3, 1});
    L.push_back({K_ATTN, "decoder.mid_block.attentions.0", dims[0], dims[0], 1, 1});
    L.push_back({K_RES, "decoder.mid_block.resnets.1", dims[0], dims[0], 3, 1});
    int scale = 1;
    for (int i = 0; i < 4; ++i) {
        int cin = dims[i];
        const int cout = dims[i + 1];
        if (i > 0) cin /= 2;
        for (int r = 0; r < 3; ++r)
            L.push_back({K_RES, "decoder.up_blocks." + std::to_string(i) + ".resnets." + std::to_string(r),
                         r == 0 ? cin : cout, cout, 3, scale});
        if (i < 3) {
            L.push_back({i < 2 ? K_UP3D : K_UP2D, "decoder.up_blocks." + std::to_string(i) + ".upsamplers.0", cout, cout,
                         3, scale});
            scale *= 2;
        }
    }
    L.push_back({K_NORM, "decoder.norm_out", dims[4], dims[4], 1, scale});
    L.push_back({K_CONV, "decoder.conv_out", dims[4], 3, 3, scale});
    return L;
}

struct ConvW {
    __nv_bfloat16* w = nullptr;   // [co_pad, ldw]
    float* bias = nullptr;        // [co]
    int ci = 0, co = 0, co_pad = 0, kt = 1, kh = 1, kw = 1, cip = 0;
    long long ldw = 0;
    int scale = 1;                // spatial level (for the cache size)
    // frame cache (causal kernels with kt > 1)
    __nv_bfloat16* cache = nullptr;  // [max_batch, 2, H, W, ci]
    int nc = 0;
};
struct NormW {
    float* g = nullptr;
    float* b = nullptr;
    int c = 0;
};
struct Slot {
    int kind;        // 0 conv weight, 1 f32 vector
    std::string owner;
    std::vector<int64_t> shape;
};

}  // namespace
}  // namespace wan

struct wan_vae {
    int device = 0, num_sms = 148;
    int max_batch = 0, max_h = 0, max_w = 0;
    std::string err;
    std::vector<wan::Entry> layout;
    std::map<std::string, wan::ConvW> convs;
    std::map<std::string, wan::NormW> norms;
    std::map<std::string, wan::Slot> slots;
    std::set<std::string> loaded;
    std::vector<void*> allocs;
    // workspace
    __nv_bfloat16* buf[4] = {nullptr, nullptr, nullptr, nullptr};
    size_t buf_elems = 0;
    __nv_bfloat16 *zcl = nullptr, *pq = nullptr, *chunk = nullptr, *yout = nullptr;
    float* zstage = nullptr;
    float* vstage = nullptr;
    __nv_bfloat16 *qkv = nullptr, *P = nullptr, *vt = nullptr, *ao = nullptr;
    float* S = nullptr;
    int* d_err = nullptr;
};

namespace {
using namespace wan;

wan_status vfail(wan_vae* v, wan_status s, const std::string& m) {
    if (v) v->err = m;
    return s;
}
#define VCU(call, what)                                                                            \
    do {                                                                                           \
        cudaError_t e_ = (call);                                                                   \
        if (e_ != cudaSuccess) return vfail(v, WAN_ECUDA, std::string(what) + ": " + cudaGetErrorString(e_)); \
    } while (0)

void* vmalloc(wan_vae* v, size_t bytes) {
    void* p = nullptr;
    if (cudaMalloc(&p, bytes) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    cudaMemset(p, 0, bytes);
    v->allocs.push_back(p);
    return p;
}

void add_conv(wan_vae* v, const std::string& n, int ci, int co, int kt, int kh, int kw, int scale) {
    ConvW c;
    c.ci = ci;
    c.co = co;
    c.co_pad = (co + 63) / 64 * 64;
    c.kt = kt;
    c.kh = kh;
    c.kw = kw;
    c.cip = (ci + 63) / 64 * 64;
    c.ldw = (long long)kt * kh * kw * c.cip;
    c.scale = scale;
    v->convs[n] = c;
    std::vector<int64_t> ws = {co, ci};
    if (kt == 1 && n.find("resample") != std::string::npos) {
        ws.push_back(kh);
        ws.push_back(kw);
    } else if (n.find(".to_qkv") != std::string::npos || n.find(".proj") != std::string::npos) {
        ws.push_back(1);
        ws.push_back(1);
    } else {
        ws.push_back(kt);
        ws.push_back(kh);
        ws.push_back(kw);
    }
    v->slots[n + ".weight"] = Slot{0, n, ws};
    v->slots[n + ".bias"] = Slot{1, n, {co}};
}

void add_norm(wan_vae* v, const std::string& n, int c) {
    NormW w;
    w.c = c;
    v->norms[n] = w;
    v->slots[n + ".gamma"] = Slot{1, n, {c}};
    v->slots[n + ".bias"] = Slot{1, n, {c}};
}

wan_status build(wan_vae* v) {
    v->layout = decoder_layout();
    for (const Entry& e : v->layout) {
        switch (e.kind) {
            case K_CONV: add_conv(v, e.name, e.a, e.b, e.k, e.k, e.k, e.scale); break;
            case K_RES:
                add_norm(v, e.name + ".norm1", e.a);
                add_conv(v, e.name + ".conv1", e.a, e.b, 3, 3, 3, e.scale);
                add_norm(v, e.name + ".norm2", e.b);
                add_conv(v, e.name + ".conv2", e.b, e.b, 3, 3, 3, e.scale);
                if (e.a != e.b) add_conv(v, e.name + ".conv_shortcut", e.a, e.b, 1, 1, 1, e.scale);
                break;
            case K_ATTN:
                add_norm(v, e.name + ".norm", e.a);
                add_conv(v, e.name + ".to_qkv", e.a, 3 * e.a, 1, 1, 1, e.scale);
                add_conv(v, e.name + ".proj", e.a, e.a, 1, 1, 1, e.scale);
                break;
            case K_UP3D:
            case K_UP2D:
                add_conv(v, e.name + ".resample.1", e.a, e.a / 2, 1, 3, 3, e.scale * 2);
                if (e.kind == K_UP3D) add_conv(v, e.name + ".time_conv", e.a, 2 * e.a, 3, 1, 1, e.scale);
                break;
            case K_NORM: add_norm(v, e.name, e.a); break;
        }
    }
    // weights
    for (auto& kv : v->convs) {
        ConvW& c = kv.second;
        c.w = static_cast<__nv_bfloat16*>(vmalloc(v, (size_t)c.co_pad * c.ldw * 2));
        c.bias = static_cast<float*>(vmalloc(v, (size_t)c.co * 4));
        if (!c.w || !c.bias) return vfail(v, WAN_ENOMEM, "decoder weights");
        const bool causal = c.kt > 1 && kv.first != "post_quant_conv";
        if (causal) {
            const size_t el = (size_t)v->max_batch * 2 * (size_t)v->max_h * c.scale * v->max_w * c.scale * c.ci;
            c.cache = static_cast<__nv_bfloat16*>(vmalloc(v, el * 2));
            if (!c.cache) return vfail(v, WAN_ENOMEM, "frame caches");
        }
    }
    for (auto& kv : v->norms) {
        kv.second.g = static_cast<float*>(vmalloc(v, (size_t)kv.second.c * 4));
        kv.second.b = static_cast<float*>(vmalloc(v, (size_t)kv.second.c * 4));
        if (!kv.second.g || !kv.second.b) return vfail(v, WAN_ENOMEM, "decoder norms");
    }
    // activations: the largest is the upsampled input of the last upsampler's
    // convolution (4 frames at 8x, 192 channels); bound every tensor by it
    const size_t HW = (size_t)v->max_h * v->max_w;
    size_t mx = 0;
    for (const Entry& e : v->layout) {
        const size_t s2 = (size_t)e.scale * e.scale;
        const size_t frames = e.scale == 1 ? 1 : 4;
        mx = std::max(mx, frames * s2 * HW * std::max(e.a, e.b));
        if (e.kind == K_UP3D || e.kind == K_UP2D) mx = std::max(mx, (size_t)4 * 4 * s2 * HW * e.a);   // upsampled
        if (e.kind == K_UP3D) mx = std::max(mx, (size_t)2 * s2 * HW * 2 * e.a);
    }
    v->buf_elems = (size_t)v->max_batch * mx;
    for (int i = 0; i < 4; ++i) {
        v->buf[i] = static_cast<__nv_bfloat16*>(vmalloc(v, v->buf_elems * 2));
        if (!v->buf[i]) return vfail(v, WAN_ENOMEM, "decoder activations");
    }
    // latent staging, post-quant output, one chunk, the conv_out rows
    v->zstage = static_cast<float*>(vmalloc(v, (size_t)v->max_batch * Z_DIM * HW * 4));   // per frame, reused
    v->zcl = static_cast<__nv_bfloat16*>(vmalloc(v, (size_t)v->max_batch * HW * Z_DIM * 2));
    v->pq = static_cast<__nv_bfloat16*>(vmalloc(v, (size_t)v->max_batch * HW * Z_DIM * 2));
    v->chunk = v->pq;
    v->yout = static_cast<__nv_bfloat16*>(vmalloc(v, (size_t)v->max_batch * 4 * 64 * HW * 8 * 2));
    v->vstage = static_cast<float*>(vmalloc(v, (size_t)v->max_batch * 3 * 4 * 64 * HW * 4));
    // mid-block attention (latent level): qkv [Lp, 3C], S [L, Lp] f32, P [L, Lp], vt [C, Lp], out [L, C]
    const size_t L = HW, Lp = (HW + 63) / 64 * 64, C = 384;
    v->qkv = static_cast<__nv_bfloat16*>(vmalloc(v, Lp * 3 * C * 2));
    v->S = static_cast<float*>(vmalloc(v, L * Lp * 4));
    v->P = static_cast<__nv_bfloat16*>(vmalloc(v, L * Lp * 2));
    v->vt = static_cast<__nv_bfloat16*>(vmalloc(v, C * Lp * 2));
    v->ao = static_cast<__nv_bfloat16*>(vmalloc(v, L * C * 2));
    v->d_err = static_cast<int*>(vmalloc(v, sizeof(int)));
    if (!v->zstage || !v->zcl || !v->pq || !v->yout || !v->vstage || !v->qkv || !v->S || !v->P || !v->vt || !v->ao ||
        !v->d_err)
        return vfail(v, WAN_ENOMEM, "decoder workspace");
    return WAN_OK;
}

// ------------------------------------------------------------------ the frame loop
struct Run {
    wan_vae* v;
    LaunchCtx ctx;
    int B;
};

struct Act {  // a channels-last activation in one of the pool buffers
    int buf;
    int T, H, W, C;
};

int free_buf(std::initializer_list<int> used) {
    for (int i = 0; i < 4; ++i)
        if (std::find(used.begin(), used.end(), i) == used.end()) return i;
    return -1;
}

// One causal convolution of an activation (cache read and then updated).
cudaError_t conv(Run& r, ConvW& c, const __nv_bfloat16* x, int T, int H, int W, __nv_bfloat16* y, int epi_kind,
                 const __nv_bfloat16* add, long long ldy) {
    ConvEpi e{};
    e.kind = epi_kind;
    e.bias = c.bias;
    e.y = y;
    e.ldy = ldy;
    e.add = add;
    e.ldadd = c.co;
    e.csplit = epi_kind == CONV_EPI_TIME_SPLIT ? c.co / 2 : 0;
    const bool cached = c.cache != nullptr;
    cudaError_t err = launch_conv3d(x, cached && c.nc > 0 ? c.cache : nullptr, cached ? c.nc : 0, r.B, T, H, W, c.ci,
                                    c.w, c.ldw, c.co, c.co_pad, c.kt, c.kh, c.kw, e, r.ctx, 2);
    if (err != cudaSuccess || !cached) return err;
    // keep the last 2 input frames of [cache, x] (the cache was read above, in stream order)
    const size_t fb = (size_t)H * W * c.ci * 2;           // bytes per frame
    auto copy_frames = [&](void* dst, size_t dst_pitch, const void* src, size_t src_pitch) {
        return cudaMemcpy2DAsync(dst, dst_pitch, src, src_pitch, fb, r.B, cudaMemcpyDeviceToDevice, r.ctx.stream);
    };
    char* cc = reinterpret_cast<char*>(c.cache);
    const char* xc = reinterpret_cast<const char*>(x);
    if (T >= 2) {
        err = copy_frames(cc, 2 * fb, xc + (size_t)(T - 2) * fb, (size_t)T * fb);
        if (err == cudaSuccess) err = copy_frames(cc + fb, 2 * fb, xc + (size_t)(T - 1) * fb, (size_t)T * fb);
        c.nc = 2;
    } else if (c.nc >= 1) {
        if (c.nc == 2) err = copy_frames(cc, 2 * fb, cc + fb, 2 * fb);
        if (err == cudaSuccess) err = copy_frames(cc + fb, 2 * fb, xc, fb);
        c.nc = 2;
    } else {
        err = copy_frames(cc, 2 * fb, xc, fb);
        c.nc = 1;
    }
    return err;
}

cudaError_t norm(Run& r, const NormW& n, const __nv_bfloat16* x, __nv_bfloat16* y, long long pixels, int silu) {
    return launch_chan_rmsnorm(x, y, pixels, n.c, n.g, n.b, silu, r.ctx);
}

#define RTRY(x)                            \
    do {                                   \
        cudaError_t e_ = (x);              \
        if (e_ != cudaSuccess) return e_;  \
    } while (0)

// Residual block: h = conv1(SiLU(norm1 x)); out = conv2(SiLU(norm2 h)) + shortcut(x).
cudaError_t res_block(Run& r, const Entry& e, Act& a) {
    wan_vae* v = r.v;
    const long long pix = (long long)r.B * a.T * a.H * a.W;
    const int b1 = free_buf({a.buf}), b2 = free_buf({a.buf, b1});
    RTRY(norm(r, v->norms[e.name + ".norm1"], v->buf[a.buf], v->buf[b1], pix, 1));
    RTRY(conv(r, v->convs[e.name + ".conv1"], v->buf[b1], a.T, a.H, a.W, v->buf[b2], CONV_EPI_BIAS, nullptr, e.b));
    RTRY(norm(r, v->norms[e.name + ".norm2"], v->buf[b2], v->buf[b1], pix, 1));
    const __nv_bfloat16* sc = v->buf[a.buf];
    int b3 = -1;
    if (e.a != e.b) {
        b3 = free_buf({a.buf, b1, b2});
        RTRY(conv(r, v->convs[e.name + ".conv_shortcut"], v->buf[a.buf], a.T, a.H, a.W, v->buf[b3], CONV_EPI_BIAS,
                  nullptr, e.b));
        sc = v->buf[b3];
    }
    RTRY(conv(r, v->convs[e.name + ".conv2"], v->buf[b1], a.T, a.H, a.W, v->buf[b2], CONV_EPI_ADD, sc, e.b));
    a.buf = b2;
    a.C = e.b;
    return cudaSuccess;
}

// Mid-block attention, single head over the H W positions of each frame.
cudaError_t attn_block(Run& r, const Entry& e, Act& a) {
    wan_vae* v = r.v;
    const int C = e.a, L = a.H * a.W, Lp = (L + 63) / 64 * 64;
    const int bn = free_buf({a.buf});
    const long long pix = (long long)r.B * a.T * L;
    RTRY(norm(r, v->norms[e.name + ".norm"], v->buf[a.buf], v->buf[bn], pix, 0));
    const ConvW& wqkv = v->convs[e.name + ".to_qkv"];
    const ConvW& wp = v->convs[e.name + ".proj"];
    for (int f = 0; f < r.B * a.T; ++f) {
        __nv_bfloat16* xf = v->buf[a.buf] + (size_t)f * L * C;
        const __nv_bfloat16* hf = v->buf[bn] + (size_t)f * L * C;
        EpiParams p{};
        p.kind = EPI_BIAS;
        p.bias = wqkv.bias;
        p.out = v->qkv;
        p.ldo = 3LL * C;
        p.mod_div = 1;
        RTRY(launch_gemm(hf, C, wqkv.w, wqkv.ldw, L, 3 * C, C, p, r.ctx));   // rows L..Lp of qkv stay zero
        EpiParams ps{};
        ps.kind = EPI_BIAS_F32;
        ps.out = v->S;
        ps.ldo = Lp;
        ps.mod_div = 1;
        RTRY(launch_gemm(v->qkv, 3LL * C, v->qkv + C, 3LL * C, L, Lp, C, ps, r.ctx));
        softmax_rows_kernel<<<L, 256, 0, r.ctx.stream>>>(v->S, Lp, L, 1.0f / std::sqrt((float)C), v->P, Lp);
        RTRY(cudaGetLastError());
        dim3 tg((Lp + 31) / 32, (C + 31) / 32);
        transpose_pad_kernel<<<tg, dim3(32, 8), 0, r.ctx.stream>>>(v->qkv + 2 * C, 3LL * C, L, C, v->vt, Lp);
        RTRY(cudaGetLastError());
        EpiParams po{};
        po.kind = EPI_BIAS;
        po.out = v->ao;
        po.ldo = C;
        po.mod_div = 1;
        RTRY(launch_gemm(v->P, Lp, v->vt, Lp, L, C, Lp, po, r.ctx));
        EpiParams pr{};
        pr.kind = EPI_RESIDUAL;
        pr.bias = wp.bias;
        pr.out = xf;
        pr.ldo = C;
        pr.mod_div = 1;
        RTRY(launch_gemm(v->ao, C, wp.w, wp.ldw, L, C, C, pr, r.ctx));
    }
    return cudaSuccess;
}

// Upsampler: (time_conv into two frames per frame, except on the first latent
// frame) then nearest 2x and a 3x3 convolution halving the channels.
cudaError_t up_block(Run& r, const Entry& e, Act& a, bool first) {
    wan_vae* v = r.v;
    if (e.kind == K_UP3D && !first) {
        const int bt = free_buf({a.buf});
        RTRY(conv(r, v->convs[e.name + ".time_conv"], v->buf[a.buf], a.T, a.H, a.W, v->buf[bt], CONV_EPI_TIME_SPLIT,
                  nullptr, a.C));
        a.buf = bt;
        a.T *= 2;
    }
    const int bu = free_buf({a.buf}), bo = free_buf({a.buf, bu});
    const long long n = (long long)r.B * a.T;
    upsample2x_kernel<<<grid_for(n * 4 * a.H * a.W * a.C / 8, v->num_sms), 256, 0, r.ctx.stream>>>(
        v->buf[a.buf], v->buf[bu], n, a.H, a.W, a.C);
    RTRY(cudaGetLastError());
    a.H *= 2;
    a.W *= 2;
    ConvW& c = v->convs[e.name + ".resample.1"];
    // per-frame 3x3 convolution: frames are independent, so treat B * T as the batch
    const int Bsave = r.B;
    r.B = Bsave * a.T;
    cudaError_t err = conv(r, c, v->buf[bu], 1, a.H, a.W, v->buf[bo], CONV_EPI_BIAS, nullptr, c.co);
    r.B = Bsave;
    RTRY(err);
    a.buf = bo;
    a.C = c.co;
    return cudaSuccess;
}

// The decoder on one latent frame (chunk); returns the conv_out rows in v->yout.
cudaError_t decode_chunk(Run& r, const __nv_bfloat16* x, int H, int W, bool first, Act& out) {
    wan_vae* v = r.v;
    Act a{0, 1, H, W, Z_DIM};
    for (const Entry& e : v->layout) {
        if (e.name == "post_quant_conv") continue;
        switch (e.kind) {
            case K_CONV: {
                ConvW& c = v->convs[e.name];
                if (e.name == "decoder.conv_in") {
                    RTRY(conv(r, c, x, a.T, a.H, a.W, v->buf[0], CONV_EPI_BIAS, nullptr, c.co));
                    a = Act{0, a.T, a.H, a.W, c.co};
                } else {  // conv_out: 3 channels, rows of 8
                    RTRY(conv(r, c, v->buf[a.buf], a.T, a.H, a.W, v->yout, CONV_EPI_BIAS, nullptr, 8));
                    out = Act{-1, a.T, a.H, a.W, 3};
                }
                break;
            }
            case K_RES: RTRY(res_block(r, e, a)); break;
            case K_ATTN: RTRY(attn_block(r, e, a)); break;
            case K_UP3D:
            case K_UP2D: RTRY(up_block(r, e, a, first)); break;
            case K_NORM: {
                const int bn = free_buf({a.buf});
                RTRY(norm(r, v->norms[e.name], v->buf[a.buf], v->buf[bn], (long long)r.B * a.T * a.H * a.W, 1));
                a.buf = bn;
                break;
            }
        }
    }
    return cudaSuccess;
}

}  // namespace

extern "C" {

wan_status wan_vae_create(int device, int max_batch, int max_h, int max_w, wan_vae** out) {
    if (!out) return WAN_EINVAL;
    *out = nullptr;
    if (max_batch < 1 || max_h < 1 || max_w < 1) return WAN_EINVAL;
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) {
        cudaGetLastError();
        return WAN_ECUDA;
    }
    cudaSetDevice(device);
    if (init_kernel_attributes() != cudaSuccess) {
        cudaGetLastError();
        return WAN_ECUDA;
    }
    wan_vae* v = new wan_vae();
    v->device = device;
    v->max_batch = max_batch;
    v->max_h = max_h;
    v->max_w = max_w;
    cudaDeviceGetAttribute(&v->num_sms, cudaDevAttrMultiProcessorCount, device);
    wan_status s = build(v);
    if (s != WAN_OK) {
        wan_vae_destroy(v);
        return s;
    }
    cudaDeviceSynchronize();
    *out = v;
    return WAN_OK;
}

void wan_vae_destroy(wan_vae* v) {
    if (!v) return;
    cudaSetDevice(v->device);
    cudaDeviceSynchronize();
    for (void* p : v->allocs) cudaFree(p);
    delete v;
}

const char* wan_vae_last_error(const wan_vae* v) { return v ? v->err.c_str() : "null handle"; }

int wan_vae_missing_weights(const wan_vae* v, char* buf, int len) {
    if (!v) return -1;
    int missing = 0;
    std::string s;
    for (auto& kv : v->slots) {
        if (v->loaded.count(kv.first)) continue;
        ++missing;
        if (!s.empty()) s += ",";
        s += kv.first;
    }
    if (buf && len > 0) {
        std::strncpy(buf, s.c_str(), len - 1);
        buf[len - 1] = 0;
    }
    return missing;
}

wan_status wan_vae_load_weights(wan_vae* v, int n, const char* const* names, const void* const* ptrs, const int* dtypes,
                                const int64_t* const* shapes, const int* ndims, int ptrs_on_device, void* stream) {
    if (!v) return WAN_EINVAL;
    if (n < 0 || (n > 0 && (!names || !ptrs || !dtypes || !shapes || !ndims))) return vfail(v, WAN_EINVAL, "null arrays");
    cudaSetDevice(v->device);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    wan_status first = WAN_OK;
    void* tmp = nullptr;
    size_t tmp_bytes = 0;
    for (int i = 0; i < n; ++i) {
        if (!names[i] || !ptrs[i]) {
            if (first == WAN_OK) first = vfail(v, WAN_EINVAL, "null name or pointer");
            continue;
        }
        auto it = v->slots.find(names[i]);
        if (it == v->slots.end()) {
            if (first == WAN_OK) first = vfail(v, WAN_EUNEXPECTED_WEIGHT, std::string("unexpected weight ") + names[i]);
            continue;
        }
        const Slot& sl = it->second;
        bool ok = ndims[i] == (int)sl.shape.size() && shapes[i] && (dtypes[i] == WAN_DTYPE_F32 || dtypes[i] == WAN_DTYPE_BF16);
        long long numel = 1;
        for (int d = 0; ok && d < ndims[i]; ++d) {
            ok = shapes[i][d] == sl.shape[d];
            numel *= sl.shape[d];
        }
        if (!ok) {
            if (first == WAN_OK) first = vfail(v, WAN_ESHAPE, std::string("bad shape or dtype for ") + names[i]);
            continue;
        }
        const size_t bytes = (size_t)numel * (dtypes[i] == WAN_DTYPE_BF16 ? 2 : 4);
        const void* src = ptrs[i];
        if (!ptrs_on_device) {  // stage host data on the device
            if (bytes > tmp_bytes) {
                VCU(cudaStreamSynchronize(st), "weight staging");
                if (tmp) cudaFree(tmp);
                tmp = nullptr;
                VCU(cudaMalloc(&tmp, bytes), "weight staging allocation");
                tmp_bytes = bytes;
            }
            VCU(cudaMemcpyAsync(tmp, src, bytes, cudaMemcpyHostToDevice, st), "weight upload");
            src = tmp;
        }
        const std::string name = names[i];
        if (sl.kind == 0) {
            ConvW& c = v->convs[sl.owner];
            const int taps = c.kt * c.kh * c.kw;
            VCU(cudaMemsetAsync(c.w, 0, (size_t)c.co_pad * c.ldw * 2, st), "weight clear");
            pack_conv_weight_kernel<<<grid_for((long long)c.co * c.ci * taps, v->num_sms), 256, 0, st>>>(
                src, dtypes[i] == WAN_DTYPE_BF16, c.co, c.ci, taps, c.cip, c.w, c.ldw);
            VCU(cudaGetLastError(), "weight repack");
        } else {
            float* dst = nullptr;
            if (v->convs.count(sl.owner) && name.size() > 5 && name.compare(name.size() - 5, 5, ".bias") == 0 &&
                !v->norms.count(sl.owner))
                dst = v->convs[sl.owner].bias;
            else if (v->norms.count(sl.owner))
                dst = name.compare(name.size() - 6, 6, ".gamma") == 0 ? v->norms[sl.owner].g : v->norms[sl.owner].b;
            if (!dst) {
                if (first == WAN_OK) first = vfail(v, WAN_EINTERNAL, "no destination for " + name);
                continue;
            }
            if (dtypes[i] == WAN_DTYPE_F32)
                VCU(cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, st), "vector copy");
            else
                VCU(launch_convert(src, WAN_DTYPE_BF16, dst, WAN_DTYPE_F32, numel, st), "vector conversion");
        }
        if (!ptrs_on_device) VCU(cudaStreamSynchronize(st), "weight upload");
        v->loaded.insert(name);
    }
    VCU(cudaStreamSynchronize(st), "weight load");
    if (tmp) cudaFree(tmp);
    return first;
}

wan_status wan_vae_decode(wan_vae* v, const float* z, int B, int T, int H, int W, float* video, int io_on_device,
                          void* stream) {
    if (!v) return WAN_EINVAL;
    if (!z || !video) return vfail(v, WAN_EINVAL, "null input or output pointer");
    if (B < 1 || B > v->max_batch || T < 1 || H < 1 || W < 1 || H > v->max_h || W > v->max_w)
        return vfail(v, WAN_ESHAPE, "latent shape outside the workspace limits");
    if (v->loaded.size() != v->slots.size()) {
        char buf[256];
        const int m = wan_vae_missing_weights(v, buf, sizeof(buf));
        return vfail(v, WAN_EMISSING_WEIGHT, std::to_string(m) + " weights missing: " + buf);
    }
    cudaSetDevice(v->device);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    Run r{v, LaunchCtx{st, v->d_err, 2000000000ull, v->num_sms, nullptr}, B};
    for (auto& kv : v->convs) kv.second.nc = 0;   // a new video: empty caches
    const int Tv = 1 + 4 * (T - 1), Hv = 8 * H, Wv = 8 * W;
    const size_t HW = (size_t)H * W;
    const cudaMemcpyKind h2d = io_on_device ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice;
    ConvW& pq = v->convs["post_quant_conv"];
    for (int i = 0; i < T; ++i) {
        // latent frame i of every sample -> channels-last bf16, then post_quant_conv (1x1x1)
        VCU(cudaMemcpy2DAsync(v->zstage, HW * 4, z + (size_t)i * HW, (size_t)T * HW * 4, HW * 4, (size_t)B * Z_DIM, h2d, st),
            "latent copy");
        latent_to_cl_kernel<<<grid_for((long long)B * Z_DIM * HW, v->num_sms), 256, 0, st>>>(v->zstage, v->zcl, B, Z_DIM,
                                                                                              1, H, W);
        VCU(cudaGetLastError(), "latent layout");
        VCU(conv(r, pq, v->zcl, 1, H, W, v->chunk, CONV_EPI_BIAS, nullptr, Z_DIM), "post_quant_conv");
        Act out{};
        VCU(decode_chunk(r, v->chunk, H, W, i == 0, out), "decoder");
        const int t0 = i == 0 ? 0 : 1 + 4 * (i - 1);
        const long long total = (long long)B * 3 * out.T * out.H * out.W;
        float* dst = io_on_device ? video : v->vstage;
        const int tt0 = io_on_device ? t0 : 0;
        const int ttot = io_on_device ? Tv : out.T;
        to_video_kernel<<<grid_for(total, v->num_sms), 256, 0, st>>>(v->yout, 8, B, out.T, out.H, out.W, dst, ttot, tt0);
        VCU(cudaGetLastError(), "video layout");
        if (!io_on_device) {  // this chunk's frames into the host video [B, 3, Tv, Hv, Wv]
            const size_t fbytes = (size_t)out.T * Hv * Wv * 4;
            VCU(cudaMemcpy2DAsync(video + (size_t)t0 * Hv * Wv, (size_t)Tv * Hv * Wv * 4, v->vstage, fbytes, fbytes,
                                  (size_t)B * 3, cudaMemcpyDeviceToHost, st),
                "video copy");
            VCU(cudaStreamSynchronize(st), "video copy");   // the staging buffer is reused by the next chunk
        }
    }
    return WAN_OK;
}

wan_status wan_vae_sync(wan_vae* v, void* stream) {
    if (!v) return WAN_EINVAL;
    cudaSetDevice(v->device);
    VCU(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)), "stream synchronize");
    int flag = 0;
    VCU(cudaMemcpy(&flag, v->d_err, sizeof(int), cudaMemcpyDeviceToHost), "error word read");
    if (flag) {
        cudaMemset(v->d_err, 0, sizeof(int));
        return vfail(v, WAN_ETIMEOUT, "a kernel's on-chip wait ran out of time");
    }
    return WAN_OK;
}

}  // extern "C"

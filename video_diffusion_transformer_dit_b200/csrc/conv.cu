// Implicit-GEMM causal 3-D convolution on tcgen05 for the Wan VAE decoder
// (pswp.cn WanPipeline notes, "WanCausalConv3d": 2 p_t zero frames before the
// input and none after, p_h / p_w zero rows / columns on both sides; in the
// decoder's frame loop cached frames replace leading zero frames).
//
// y[b, t, h, w, co] = bias[co] + sum over taps (it, ih, iw) and channels ci of
//   x[b, t - (kt - 1) + it, h - (kh - 1) / 2 + ih, w - (kw - 1) / 2 + iw, ci] * W[co, ci, it, ih, iw]
// with frames before 0 taken from the cache (its last frames sit right before
// frame 0) and everything else outside the input zero.
//
// GEMM view: M = output pixels, N = output channels, K = taps x channels.  A
// tile is 256 output pixels of one frame (16 rows x 16 columns, two 128-row
// MMA halves sharing each weight tile); for the K block (tap, 64 channels) the
// producer loads the input patch shifted by the tap with ONE 5-D TMA copy
// straight from the channels-last input (or the cache), 64 channels x 16
// columns x 16 rows = two 128 x 64 K-major tiles with 128-byte swizzle, the
// layout the MMA reads.  Zero padding comes free: coordinates
// outside the tensor (negative ones included) read as zero.  No im2col matrix
// is ever written.  The rest is the persistent warp-specialised structure of
// the linear-layer GEMM: TMA producer warp, single-thread MMA issuer with two
// TMEM accumulators, 8 epilogue warps writing channels-last rows with the
// bias, an optional residual add, or the frame split of the decoder's time
// upsampler.
#include "common.cuh"
#include "kernels.h"

namespace wan {

struct ConvParams {
    int B, T, H, W, Ci, Co;
    int kt, kh, kw, nc;          // kernel; frames in the cache
    int cblocks, kblocks;        // 64-channel blocks per tap; taps * cblocks
    int ht, wt;                  // spatial tiles of 16 rows x 16 columns
    int num_m, num_n, num_tiles;
    ConvEpi epi;
    WaitCtl wc;
};

namespace cv {
constexpr int BM = 256, BK = 64, TH = 16, TW = 16;   // 256 pixels = two 128-row MMA halves
constexpr int HALF_BYTES = 128 * BK * 2;
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 64 + 32 * EPI_WARPS;
template <int BN>
struct Cfg {
    static constexpr int A_BYTES = BM * BK * 2;
    static constexpr int B_BYTES = BN * BK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int STAGES = (212992 / STAGE_BYTES) < 8 ? (212992 / STAGE_BYTES) : 8;
    static constexpr int ACC_COLS = 2 * BN;              // both halves of one accumulator set
    static constexpr int TMEM_COLS = 2 * ACC_COLS;       // double-buffered
    static_assert(TMEM_COLS <= 512, "tensor memory");
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
};
}  // namespace cv

// 32 accumulator columns [c, c + 32) of one output pixel.
__device__ __forceinline__ void conv_epilogue_chunk(const ConvParams& p, int b, int t, int h, int w, int c,
                                                    const uint32_t (&r)[32]) {
    const ConvEpi& e = p.epi;
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]) + (c + i < p.Co && e.bias ? __ldg(e.bias + c + i) : 0.0f);
    long long pix;
    int cc = c;
    if (e.kind == CONV_EPI_TIME_SPLIT) {  // channel half k of output channel co -> frame 2t + k, channel co % Csplit
        const int half = c / e.csplit;
        cc = c - half * e.csplit;
        pix = (((long long)b * 2 * p.T + 2 * t + half) * p.H + h) * p.W + w;
    } else {
        pix = (((long long)b * p.T + t) * p.H + h) * p.W + w;
    }
    __nv_bfloat16* dst = e.y + pix * e.ldy + cc;
    if (e.kind == CONV_EPI_ADD) {
        const __nv_bfloat16* a = e.add + ((((long long)b * p.T + t) * p.H + h) * p.W + w) * e.ldadd + c;
        if (c + 32 <= p.Co) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint4 u = *reinterpret_cast<const uint4*>(a + 8 * i);
                const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float2 f = unpack_bf16(uw[k]);
                    v[8 * i + 2 * k] += f.x;
                    v[8 * i + 2 * k + 1] += f.y;
                }
            }
        } else {
            for (int i = 0; i < 32 && c + i < p.Co; ++i) v[i] += __bfloat162float(a[i]);
        }
    }
    if (c + 32 <= p.Co) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            reinterpret_cast<uint4*>(dst)[i] =
                make_uint4(pack_bf16(v[8 * i], v[8 * i + 1]), pack_bf16(v[8 * i + 2], v[8 * i + 3]),
                           pack_bf16(v[8 * i + 4], v[8 * i + 5]), pack_bf16(v[8 * i + 6], v[8 * i + 7]));
    } else {
        for (int i = 0; i < 32 && c + i < p.Co; ++i) dst[i] = __float2bfloat16_rn(v[i]);
    }
}

template <int BN>
__global__ void __launch_bounds__(cv::THREADS, 1)
    conv3d_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmC,
                     const __grid_constant__ CUtensorMap tmW, const ConvParams p) {
    using C = cv::Cfg<BN>;
    constexpr int STAGES = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + STAGES * C::A_BYTES;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * C::STAGE_BYTES);
    uint64_t* empty = full + STAGES;
    uint64_t* tfull = empty + STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull + a, 1);
            mbar_init(tempty + a, cv::EPI_WARPS);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmX);
        if (p.nc > 0) tma_prefetch_desc(&tmC);
        tma_prefetch_desc(&tmW);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    uint32_t armed = 0, armed_par = 0;
    bool issued = false;

    // tile -> (m tile, n tile), n fastest: consecutive CTAs share one input patch in L2
    auto coords = [&](int tile, int& b, int& t, int& hb, int& wb, int& nb) {
        nb = tile % p.num_n;
        int m = tile / p.num_n;
        wb = m % p.wt;
        m /= p.wt;
        hb = m % p.ht;
        m /= p.ht;
        t = m % p.T;
        b = m / p.T;
    };

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer: one shifted input patch per (tap, 64 channels) ----------------
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            const int khw = p.kh * p.kw;
            for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
                int b, t, hb, wb, nb;
                coords(tile, b, t, hb, wb, nb);
                for (int kb = 0; kb < p.kblocks; ++kb) {
                    if (!mbar_wait(empty + stage, phase ^ 1, abort_flag, p.wc)) {
                        ok = false;
                        break;
                    }
                    const int tap = kb / p.cblocks, cb = kb - tap * p.cblocks;
                    const int it = tap / khw, rem = tap - it * khw;
                    const int ih = rem / p.kw, iw = rem - ih * p.kw;
                    const int tt = t - (p.kt - 1) + it;
                    const int hh = hb * cv::TH + ih - (p.kh - 1) / 2;
                    const int ww = wb * cv::TW + iw - (p.kw - 1) / 2;
                    mbar_expect_tx(full + stage, C::STAGE_BYTES);
                    uint8_t* a_dst = sA + stage * C::A_BYTES;
                    if (tt >= 0 || tt < -p.nc)   // a frame of x, or before the cache: frame -1 reads as zeros
                        tma_load_5d(a_dst, &tmX, full + stage, cb * cv::BK, ww, hh, tt >= 0 ? tt : -1, b);
                    else
                        tma_load_5d(a_dst, &tmC, full + stage, cb * cv::BK, ww, hh, p.nc + tt, b);
                    tma_load_2d(sB + stage * C::B_BYTES, &tmW, full + stage, kb * cv::BK, nb * BN);
                    armed |= 1u << stage;
                    armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer ----------------
            constexpr uint32_t IDESC = idesc_bf16(128, BN, false);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
                if (!mbar_wait(tempty + acc, acc_phase ^ 1, abort_flag, p.wc)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * C::ACC_COLS;
                for (int kb = 0; kb < p.kblocks; ++kb) {
                    if (!mbar_wait(full + stage, phase, abort_flag, p.wc)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sA + stage * C::A_BYTES);
                    const uint32_t b0 = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
                    for (int k = 0; k < cv::BK / 16; ++k) {
                        const uint64_t bd = sdesc_kmajor_sw128(b0 + 32 * k);
                        umma_bf16_ss(d_tmem, sdesc_kmajor_sw128(a0 + 32 * k), bd, IDESC, (kb | k) != 0);
                        umma_bf16_ss(d_tmem + BN, sdesc_kmajor_sw128(a0 + cv::HALF_BYTES + 32 * k), bd, IDESC,
                                     (kb | k) != 0);
                    }
                    issued = true;
                    umma_commit(empty + stage);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                umma_commit(tfull + acc);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1;
            }
        }
    } else {
        // ---------------- epilogue warps: TMEM lane = pixel of the 8 x 16 patch ----------------
        const int q = warp & 3;
        const int chalf = (warp - 2) >> 2;
        constexpr int CW = BN / 2;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
            int b, t, hb, wb, nb;
            coords(tile, b, t, hb, wb, nb);
            if (!__all_sync(0xffffffffu, mbar_wait(tfull + acc, acc_phase, abort_flag, p.wc))) break;
            tc_fence_after();
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                const int r = half * 128 + q * 32 + lane;
                const int h = hb * cv::TH + r / cv::TW, w = wb * cv::TW + r % cv::TW;
                const uint32_t taddr =
                    tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * C::ACC_COLS + half * BN;
#pragma unroll 1
                for (int c0 = chalf * CW; c0 < (chalf + 1) * CW; c0 += 32) {
                    uint32_t rr[32];
                    tmem_ld32(taddr + c0, rr);
                    tmem_ld_wait(rr);
                    const int c = nb * BN + c0;
                    if (h < p.H && w < p.W && c < p.Co) conv_epilogue_chunk(p, b, t, h, w, c, rr);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty + acc);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1;
        }
    }

    __syncthreads();
    if (*abort_flag && lane == 0) {
        // a wait gave up somewhere in the CTA: let this CTA's own loads and MMAs
        // land (bounded) before its shared and tensor memory are released
        if (warp == 0) {
            for (int s = 0; s < STAGES; ++s)
                if (armed & (1u << s)) mbar_drain(full + s, (armed_par >> s) & 1u, 200000000ull);
        } else if (warp == 1 && issued) {
            umma_commit(drain);
            mbar_drain(drain, 0, 200000000ull);
        }
    }
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

template <int BN>
static cudaError_t conv_attr() {
    return cudaFuncSetAttribute(conv3d_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                cv::Cfg<BN>::SMEM_BYTES);
}

cudaError_t init_conv_attributes() {
    cudaError_t e = conv_attr<128>();
    if (e == cudaSuccess) e = conv_attr<64>();
    return e;
}

cudaError_t launch_conv3d(const void* x, const void* cache, int nc, int B, int T, int H, int W, int Ci, const void* w,
                          long long ldw, int Co, int Co_pad, int kt, int kh, int kw, const ConvEpi& epi,
                          const LaunchCtx& ctx, int nc_cap) {
    if (nc_cap < nc) nc_cap = nc;
    if (B <= 0 || T <= 0 || H <= 0 || W <= 0) return cudaSuccess;
    if (Ci <= 0 || Ci % 8 || Co <= 0 || Co_pad < Co || Co_pad % 64 || kt <= 0 || kh <= 0 || kw <= 0 || !(kt & 1) ||
        !(kh & 1) || !(kw & 1) || nc < 0 || nc > kt - 1 || (nc > 0 && !cache) || !epi.y || epi.ldy % 8)
        return cudaErrorInvalidValue;
    const int cblocks = (Ci + 63) / 64;
    const long long K = (long long)kt * kh * kw * cblocks * 64;
    if (ldw < K || ldw % 8 || K > (1LL << 30)) return cudaErrorInvalidValue;
    if (epi.kind == CONV_EPI_ADD && (!epi.add || epi.ldadd % 8)) return cudaErrorInvalidValue;
    if (epi.kind == CONV_EPI_TIME_SPLIT && (epi.csplit <= 0 || Co != 2 * epi.csplit || epi.csplit % 32))
        return cudaErrorInvalidValue;
    if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(w) | reinterpret_cast<uintptr_t>(cache) |
         reinterpret_cast<uintptr_t>(epi.y) | reinterpret_cast<uintptr_t>(epi.add)) & 15)
        return cudaErrorInvalidValue;
    const int BN = (Co_pad % 128 == 0) ? 128 : 64;   // two halves x two buffers x BN <= 512 TMEM columns
    ConvParams p{};
    p.B = B; p.T = T; p.H = H; p.W = W; p.Ci = Ci; p.Co = Co;
    p.kt = kt; p.kh = kh; p.kw = kw; p.nc = nc;
    p.cblocks = cblocks;
    p.kblocks = kt * kh * kw * cblocks;
    p.ht = (H + cv::TH - 1) / cv::TH;
    p.wt = (W + cv::TW - 1) / cv::TW;
    p.num_m = B * T * p.ht * p.wt;
    p.num_n = Co_pad / BN;
    p.num_tiles = p.num_m * p.num_n;
    p.epi = epi;
    p.wc.err = ctx.err;
    p.wc.limit_ns = ctx.wait_limit_ns;
    // channels-last 5-D views [B][T][H][W][Ci]; the cache [B][nc][H][W][Ci]
    CUtensorMap tx, tc, tw;
    const uint64_t dx[5] = {(uint64_t)Ci, (uint64_t)W, (uint64_t)H, (uint64_t)T, (uint64_t)B};
    const uint64_t sx[4] = {(uint64_t)Ci, (uint64_t)W * Ci, (uint64_t)H * W * Ci, (uint64_t)T * H * W * Ci};
    if (!make_tmap_5d(&tx, x, dx, sx, 64, cv::TW, cv::TH)) return cudaErrorInvalidValue;
    if (nc > 0) {
        const uint64_t dc[5] = {(uint64_t)Ci, (uint64_t)W, (uint64_t)H, (uint64_t)nc, (uint64_t)B};
        const uint64_t sc[4] = {(uint64_t)Ci, (uint64_t)W * Ci, (uint64_t)H * W * Ci, (uint64_t)nc_cap * H * W * Ci};
        if (!make_tmap_5d(&tc, cache, dc, sc, 64, cv::TW, cv::TH)) return cudaErrorInvalidValue;
    } else {
        tc = tx;
    }
    if (!make_tmap_2d(&tw, w, (uint64_t)K, (uint64_t)Co_pad, (uint64_t)ldw, 64, BN)) return cudaErrorInvalidValue;
    const int grid = p.num_tiles < ctx.num_sms ? p.num_tiles : ctx.num_sms;
    if (BN == 128)
        conv3d_tc_kernel<128><<<grid, cv::THREADS, cv::Cfg<128>::SMEM_BYTES, ctx.stream>>>(tx, tc, tw, p);
    else
        conv3d_tc_kernel<64><<<grid, cv::THREADS, cv::Cfg<64>::SMEM_BYTES, ctx.stream>>>(tx, tc, tw, p);
    if (ctx.launches) ++*ctx.launches;
    return cudaGetLastError();
}

}  // namespace wan

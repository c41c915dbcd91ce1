// Flash attention on tcgen05 for the Wan DiT: O = softmax(Q K^T / sqrt(128)) V
// per (batch, head), no mask, head_dim 128, bf16 operands, fp32 softmax.
// Used for the self-attention over the L video tokens and the
// cross-attention to the Lc text tokens (ragged key tail masked).
//
// One CTA per (128-query tile, head, batch), 6 warps:
//   warp 0      TMA producer: the Q tile once, then K and V tiles of 128 keys
//               in two-slot rings (3-D tensor maps, rows past the sequence
//               read as zero);
//   warp 1      tensor-memory owner and MMA issuer: S_j = Q K_j^T into one of
//               two 128-column TMEM buffers, issued one tile ahead, and
//               O += P_j V_j into a third 128-column TMEM accumulator with V
//               as an MN-major operand;
//   warps 2..5  softmax, one query row per thread: tcgen05.ld of its S row,
//               running max / sum in fp32 (log2 domain, exp2), the new
//               probabilities written as bf16 into a swizzled shared tile P
//               for the next MMA.  O is rescaled in TMEM only when the row
//               maximum grows by more than 2^8 (the stale maximum is exact
//               because the final division uses the same running sum); the
//               last step divides by the sum and stores bf16 rows.
#include "common.cuh"
#include "kernels.h"

namespace wan {

struct AttnParams {
    int Lq, Lk, heads;
    __nv_bfloat16* o;
    long long ldo;
    float scale_log2;  // log2(e) / sqrt(head_dim)
    WaitCtl wc;
};

namespace attn {
constexpr int TILE_BYTES = 128 * 128 * 2;  // one 128 x 128 bf16 tile = two 64-column swizzled halves
constexpr int HALF_BYTES = 128 * 128;      // 128 rows x 128 bytes
constexpr int SQ = 0;
constexpr int SK = SQ + TILE_BYTES;          // 2 slots
constexpr int SV = SK + 2 * TILE_BYTES;      // 2 slots
constexpr int SP = SV + 2 * TILE_BYTES;      // 1 tile
constexpr int SBAR = SP + TILE_BYTES;
constexpr int SMEM_BYTES = SBAR + 256 + 1024;
constexpr float RESCALE_THRESHOLD = 8.0f;    // log2 units
}  // namespace attn

__global__ void __launch_bounds__(192, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
    using namespace attn;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SBAR);
    uint64_t* q_full = bars + 0;
    uint64_t* k_full = bars + 1;   // [2]
    uint64_t* k_empty = bars + 3;  // [2]
    uint64_t* v_full = bars + 5;   // [2]
    uint64_t* v_empty = bars + 7;  // [2]
    uint64_t* s_full = bars + 9;   // [2]
    uint64_t* s_empty = bars + 11; // [2]
    uint64_t* p_full = bars + 13;
    uint64_t* o_done = bars + 14;
    uint64_t* drain = bars + 15;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int q0 = qt * 128;
    const int nk = (p.Lk + 127) / 128;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(k_full + s, 1);
            mbar_init(k_empty + s, 1);
            mbar_init(v_full + s, 1);
            mbar_init(v_empty + s, 1);
            mbar_init(s_full + s, 1);
            mbar_init(s_empty + s, 4);
        }
        mbar_init(p_full, 4);
        mbar_init(o_done, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t TM_S0 = tmem, TM_O = tmem + 256;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- producer ----------------
            uint32_t armed = 0, armed_par = 0;  // bits: q=0, k slots 1..2, v slots 3..4
            bool ok = true;
            mbar_expect_tx(q_full, TILE_BYTES);
            tma_load_3d(smem + SQ, &tmQ, q_full, h * 128, q0, b);
            tma_load_3d(smem + SQ + HALF_BYTES, &tmQ, q_full, h * 128 + 64, q0, b);
            armed |= 1u;
            for (int j = 0; ok && j < nk; ++j) {
                const int s = j & 1;
                const uint32_t par = (j >> 1) & 1;
                if (!mbar_wait(k_empty + s, par ^ 1, abort_flag, p.wc)) { ok = false; break; }
                mbar_expect_tx(k_full + s, TILE_BYTES);
                tma_load_3d(smem + SK + s * TILE_BYTES, &tmK, k_full + s, h * 128, j * 128, b);
                tma_load_3d(smem + SK + s * TILE_BYTES + HALF_BYTES, &tmK, k_full + s, h * 128 + 64, j * 128, b);
                armed |= 2u << s;
                armed_par = (armed_par & ~(2u << s)) | (par << (1 + s));
                if (!mbar_wait(v_empty + s, par ^ 1, abort_flag, p.wc)) { ok = false; break; }
                mbar_expect_tx(v_full + s, TILE_BYTES);
                tma_load_3d(smem + SV + s * TILE_BYTES, &tmV, v_full + s, h * 128, j * 128, b);
                tma_load_3d(smem + SV + s * TILE_BYTES + HALF_BYTES, &tmV, v_full + s, h * 128 + 64, j * 128, b);
                armed |= 8u << s;
                armed_par = (armed_par & ~(8u << s)) | (par << (3 + s));
            }
            if (!ok) {
                mbar_drain(q_full, 0, 200000000ull);
                for (int s = 0; s < 2; ++s) {
                    if (armed & (2u << s)) mbar_drain(k_full + s, (armed_par >> (1 + s)) & 1, 200000000ull);
                    if (armed & (8u << s)) mbar_drain(v_full + s, (armed_par >> (3 + s)) & 1, 200000000ull);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer ----------------
            constexpr uint32_t ID_QK = idesc_bf16(128, 128, false);
            constexpr uint32_t ID_PV = idesc_bf16(128, 128, true);
            const uint32_t sq = smem_u32(smem + SQ);
            const uint32_t sp = smem_u32(smem + SP);
            bool ok = mbar_wait(q_full, 0, abort_flag, p.wc);
            bool issued = false;
            auto issue_s = [&](int j) -> bool {
                const int s = j & 1;
                if (!mbar_wait(k_full + s, (j >> 1) & 1, abort_flag, p.wc)) return false;
                if (j >= 2 && !mbar_wait(s_empty + s, ((j - 2) >> 1) & 1, abort_flag, p.wc)) return false;
                tc_fence_after();
                const uint32_t sk = smem_u32(smem + SK + s * TILE_BYTES);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
                    umma_bf16_ss(TM_S0 + s * 128, sdesc_kmajor_sw128(sq + off), sdesc_kmajor_sw128(sk + off), ID_QK,
                                 kk != 0);
                }
                issued = true;
                umma_commit(s_full + s);
                umma_commit(k_empty + s);
                return true;
            };
            if (ok) ok = issue_s(0);
            for (int j = 0; ok && j < nk; ++j) {
                if (j + 1 < nk && !issue_s(j + 1)) { ok = false; break; }
                const int s = j & 1;
                if (!mbar_wait(p_full, j & 1, abort_flag, p.wc)) { ok = false; break; }
                if (!mbar_wait(v_full + s, (j >> 1) & 1, abort_flag, p.wc)) { ok = false; break; }
                tc_fence_after();
                const uint32_t sv = smem_u32(smem + SV + s * TILE_BYTES);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    // P: K-major over keys; V: rows are keys, 64-wide d halves HALF_BYTES apart
                    const uint32_t poff = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
                    umma_bf16_ss(TM_O, sdesc_kmajor_sw128(sp + poff), sdesc_mnmajor_sw128(sv + kk * 2048, HALF_BYTES),
                                 ID_PV, (j | kk) != 0);
                }
                umma_commit(v_empty + s);
                umma_commit(o_done);
            }
            if (!ok && issued) {
                umma_commit(drain);
                mbar_drain(drain, 0, 200000000ull);
            }
        }
    } else {
        // ---------------- softmax / output warps ----------------
        const int qq = warp & 3;
        const int r = qq * 32 + lane;                     // row inside the tile == TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>(qq * 32) << 16;
        uint8_t* prow = smem + SP + r * 128;
        const int sw = r & 7;
        float m_run = -INFINITY, l_run = 0.0f;
        bool ok = true;
        for (int j = 0; j < nk; ++j) {
            const int s = j & 1;
            // every tcgen05.ld/st below is warp-collective: keep the warp's decisions uniform
            if (!__all_sync(0xffffffffu, mbar_wait(s_full + s, (j >> 1) & 1, abort_flag, p.wc))) { ok = false; break; }
            tc_fence_after();
            uint32_t sv[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(TM_S0 + lane_off + s * 128 + c * 32, sv[c]);
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld_wait(sv[c]);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(s_empty + s);

            const int valid = min(128, p.Lk - j * 128);
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    float x = __uint_as_float(sv[c][i]);
                    if (c * 32 + i >= valid) x = -INFINITY;
                    sv[c][i] = __float_as_uint(x);
                    mx = fmaxf(mx, x);
                }
            const float m_tile = mx * p.scale_log2;
            const float m_new = fmaxf(m_run, m_tile);
            const bool rescale = m_new > m_run + RESCALE_THRESHOLD;
            const float m_use = rescale ? m_new : m_run;
            float rowsum = 0.0f;
            uint32_t pk[64];
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    const float e0 = ex2_approx(fmaf(__uint_as_float(sv[c][i]), p.scale_log2, -m_use));
                    const float e1 = ex2_approx(fmaf(__uint_as_float(sv[c][i + 1]), p.scale_log2, -m_use));
                    rowsum += e0 + e1;
                    pk[c * 16 + i / 2] = pack_bf16(e0, e1);
                }
            // P buffer and O are free once P_{j-1} V_{j-1} has completed
            if (j > 0) {
                if (!__all_sync(0xffffffffu, mbar_wait(o_done, (j - 1) & 1, abort_flag, p.wc))) { ok = false; break; }
                tc_fence_after();
            }
            // alpha = 1 for rows that keep their maximum; 0 on the first tile
            const float alpha = rescale ? ex2_approx(m_run - m_use) : 1.0f;
            if (j > 0 && __any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t ov[32];
                    tmem_ld32(TM_O + lane_off + c * 32, ov);
                    tmem_ld_wait(ov);
#pragma unroll
                    for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
                    tmem_st32(TM_O + lane_off + c * 32, ov);
                }
                tmem_st_wait();
            }
            if (rescale) {
                l_run *= alpha;
                m_run = m_use;
            }
            l_run += rowsum;
            // P row -> shared memory, K-major with the 128-byte swizzle
#pragma unroll
            for (int ch = 0; ch < 16; ++ch) {
                const int half = ch >> 3, c16 = ch & 7;
                uint4 u = make_uint4(pk[ch * 4], pk[ch * 4 + 1], pk[ch * 4 + 2], pk[ch * 4 + 3]);
                *reinterpret_cast<uint4*>(prow + half * HALF_BYTES + ((c16 ^ sw) << 4)) = u;
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
        }
        if (ok && __all_sync(0xffffffffu, mbar_wait(o_done, (nk - 1) & 1, abort_flag, p.wc))) {
            tc_fence_after();
            const float inv = 1.0f / l_run;
            const int row = q0 + r;
            __nv_bfloat16* orow = p.o + ((long long)b * p.Lq + row) * p.ldo + h * 128;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t ov[32];
                tmem_ld32(TM_O + lane_off + c * 32, ov);
                tmem_ld_wait(ov);
                if (row < p.Lq) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        dst[i] = make_uint4(pack_bf16(__uint_as_float(ov[8 * i]) * inv, __uint_as_float(ov[8 * i + 1]) * inv),
                                            pack_bf16(__uint_as_float(ov[8 * i + 2]) * inv, __uint_as_float(ov[8 * i + 3]) * inv),
                                            pack_bf16(__uint_as_float(ov[8 * i + 4]) * inv, __uint_as_float(ov[8 * i + 5]) * inv),
                                            pack_bf16(__uint_as_float(ov[8 * i + 6]) * inv, __uint_as_float(ov[8 * i + 7]) * inv));
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

cudaError_t init_gemm_attributes();

cudaError_t init_kernel_attributes() {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, attn::SMEM_BYTES);
    if (e == cudaSuccess) e = init_gemm_attributes();
    return e;
}

cudaError_t launch_attention(const void* q, long long ldq, const void* k, long long ldk, const void* v,
                             long long ldv, void* o, long long ldo, int B, int heads, int Lq, int Lk,
                             const LaunchCtx& ctx) {
    if (B <= 0 || Lq <= 0) return cudaSuccess;
    if (Lk <= 0 || heads <= 0 || ldq % 8 || ldk % 8 || ldv % 8 || ldo % 8) return cudaErrorInvalidValue;
    if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v) |
         reinterpret_cast<uintptr_t>(o)) & 15)
        return cudaErrorInvalidValue;
    const uint64_t width = static_cast<uint64_t>(heads) * 128;
    CUtensorMap tq, tk, tv;
    if (!make_tmap_3d(&tq, q, width, Lq, B, ldq, (uint64_t)ldq * Lq, 64, 128)) return cudaErrorInvalidValue;
    if (!make_tmap_3d(&tk, k, width, Lk, B, ldk, (uint64_t)ldk * Lk, 64, 128)) return cudaErrorInvalidValue;
    if (!make_tmap_3d(&tv, v, width, Lk, B, ldv, (uint64_t)ldv * Lk, 64, 128)) return cudaErrorInvalidValue;
    AttnParams p;
    p.Lq = Lq;
    p.Lk = Lk;
    p.heads = heads;
    p.o = reinterpret_cast<__nv_bfloat16*>(o);
    p.ldo = ldo;
    p.scale_log2 = 1.4426950408889634f / sqrtf(128.0f);
    p.wc.err = ctx.err;
    p.wc.limit_ns = ctx.wait_limit_ns;
    dim3 grid((Lq + 127) / 128, heads, B);
    attn_tc_kernel<<<grid, 192, attn::SMEM_BYTES, ctx.stream>>>(tq, tk, tv, p);
    if (ctx.launches) ++*ctx.launches;
    return cudaGetLastError();
}

}  // namespace wan

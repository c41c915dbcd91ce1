// tcgen05 GEMM for every linear layer of the Wan DiT forward: C = epi(A . W^T)
// with A [M, K] activations and W [N, K] nn.Linear weights, both bf16 and
// K-major, fp32 accumulation in tensor memory.
//
// One persistent CTA per SM, 10 warps:
//   warp 0      TMA producer: 128 x 64 A tile and BN x 64 W tile per stage,
//               128-byte swizzle, STAGES-deep mbarrier ring;
//   warp 1      tensor-memory owner and MMA issuer (one thread): 4 x
//               tcgen05.mma (M=128, N=BN, K=16) per stage into one of two
//               TMEM accumulators (2 x BN columns), commit frees the stage;
//   warps 2..9  epilogue, two warps per TMEM lane quarter, each taking half of
//               the tile's columns: tcgen05.ld of 32 rows x 32 columns, fused
//               bias / GELU-tanh / gate * residual / unpatchify scatter, while
//               the MMA warp already accumulates the next tile in the other
//               TMEM buffer.
// Tiles are walked N-fastest (an A row block stays in L2 while its N tiles
// run) unless W is the larger operand, then M-fastest.
#include <cstdio>

#include "common.cuh"
#include "kernels.h"

namespace wan {

struct GemmParams {
    int M, N, K;
    int num_m, num_n, num_tiles;
    int m_fastest;
    EpiParams epi;
    WaitCtl wc;
};

// PAIR: two A tiles per stage (rows r and r + pair_off) against one W tile,
// two accumulators per tile (the CFG pair of EPI_CFG_EULER).
template <int BN, bool PAIR = false>
struct GemmCfg {
    static constexpr int BM = 128;
    static constexpr int BK = 64;
    static constexpr int NA = PAIR ? 2 : 1;
    static constexpr int A_BYTES = BM * BK * 2;
    static constexpr int B_BYTES = BN * BK * 2;
    static constexpr int STAGE_BYTES = NA * A_BYTES + B_BYTES;
    static constexpr int STAGES = (196608 / STAGE_BYTES) < 8 ? (196608 / STAGE_BYTES) : 8;
    static constexpr int TMEM_COLS = 2 * NA * BN;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
};

__device__ __forceinline__ void tile_coords(int tile, const GemmParams& p, int& mb, int& nb) {
    if (p.m_fastest) {
        mb = tile % p.num_m;
        nb = tile / p.num_m;
    } else {
        nb = tile % p.num_n;
        mb = tile / p.num_n;
    }
}

// Hot epilogues on packed fp32 pairs.  The accumulator columns arrive as 16
// pairs; bias, GELU, gate and residual run as f32x2 operations, which keeps
// the scalar FP32 pipe free for the MMA-issuing warp on the same SM
// sub-partitions (scalar FFMA traffic there slows tcgen05.mma issue).
// Where the four 16-byte words (8 bf16 each) of an epilogue chunk go: the
// row in global memory, or the row of an epilogue warp's shared-memory slab
// (128-byte swizzle: 16-byte chunk j of slab row r at chunk j ^ (r & 7)).
struct GlobalOut {
    uint4* p;
    __device__ __forceinline__ void put(int i, const uint4& w) const { p[i] = w; }
};
struct SlabOut {
    uint8_t* rowp;  // slab row (box base + r * 128)
    int j0, r7;     // first 16-byte chunk of the 32 columns, r & 7
    __device__ __forceinline__ void put(int i, const uint4& w) const {
        *reinterpret_cast<uint4*>(rowp + (((j0 + i) ^ r7) << 4)) = w;
    }
};
__device__ __forceinline__ GlobalOut global_out(const EpiParams& e, int row, int c) {
    return GlobalOut{reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(e.out) + (long long)row * e.ldo + c)};
}

// Residual rows of one 32-column chunk (4 x 16 B), loaded ahead of their use.
__device__ __forceinline__ void load_residual(const EpiParams& e, int row, int c, uint4 (&xu)[4]) {
    const uint4* xp = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(e.out) + (long long)row * e.ldo + c);
#pragma unroll
    for (int i = 0; i < 4; ++i) xu[i] = xp[i];
}

template <int KIND, class Out>
__device__ __forceinline__ void epilogue_chunk_f2(const EpiParams& e, int row, int c, const uint32_t (&r)[32],
                                                  const uint4 (&xu)[4], const Out& out) {
    uint64_t v2[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) v2[i] = f2pack(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
    if (e.bias) {
        const ulonglong2* b2 = reinterpret_cast<const ulonglong2*>(e.bias + c);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const ulonglong2 b = __ldg(b2 + i);
            v2[2 * i] = add2(v2[2 * i], b.x);
            v2[2 * i + 1] = add2(v2[2 * i + 1], b.y);
        }
    }
    if (KIND == EPI_BIAS || KIND == EPI_BIAS_GELU) {
        if (KIND == EPI_BIAS_GELU) {
#pragma unroll
            for (int i = 0; i < 16; ++i) v2[i] = gelu_tanh_f2(v2[i]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t w[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                float a, b;
                f2unpack(v2[4 * i + h], a, b);
                w[h] = pack_bf16(a, b);
            }
            out.put(i, make_uint4(w[0], w[1], w[2], w[3]));
        }
    } else {  // EPI_GATE_RESIDUAL, EPI_RESIDUAL: x (4 x 16 B) arrives preloaded
        const ulonglong2* g1 =
            e.gate1 ? reinterpret_cast<const ulonglong2*>(e.gate1 + (long long)(row / e.mod_div) * e.mod_ld + c) : nullptr;
        const ulonglong2* g0 = e.gate0 ? reinterpret_cast<const ulonglong2*>(e.gate0 + c) : nullptr;
#pragma unroll
        for (int i = 0; i < 4; ++i) {  // 8 columns: 16 B of x, 4 pairs of the gate
            uint64_t g2[4] = {0ull, 0ull, 0ull, 0ull};  // +0.0f pairs
            if (KIND == EPI_GATE_RESIDUAL) {
                if (g1) {
                    const ulonglong2 a0 = __ldg(g1 + 2 * i), a1 = __ldg(g1 + 2 * i + 1);
                    g2[0] = a0.x;
                    g2[1] = a0.y;
                    g2[2] = a1.x;
                    g2[3] = a1.y;
                }
                if (g0) {
                    const ulonglong2 a0 = __ldg(g0 + 2 * i), a1 = __ldg(g0 + 2 * i + 1);
                    g2[0] = add2(g2[0], a0.x);
                    g2[1] = add2(g2[1], a0.y);
                    g2[2] = add2(g2[2], a1.x);
                    g2[3] = add2(g2[3], a1.y);
                }
            }
            const uint32_t xw[4] = {xu[i].x, xu[i].y, xu[i].z, xu[i].w};
            uint32_t ow[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const float2 xf = unpack_bf16(xw[h]);
                const uint64_t x2 = f2pack(xf.x, xf.y);
                uint64_t o2;
                if (KIND == EPI_GATE_RESIDUAL) {
                    o2 = fma2(v2[4 * i + h], g2[h], x2);
                } else {  // the branch output is rounded to bf16 before the residual add
                    float a, b;
                    f2unpack(v2[4 * i + h], a, b);
                    const float2 ab = unpack_bf16(pack_bf16(a, b));
                    o2 = add2(x2, f2pack(ab.x, ab.y));
                }
                float a, b;
                f2unpack(o2, a, b);
                ow[h] = pack_bf16(a, b);
            }
            out.put(i, make_uint4(ow[0], ow[1], ow[2], ow[3]));
        }
    }
}

// Epilogue of 32 consecutive columns [c, c + 32) of one row (KIND fixed at compile time).
template <int KIND>
__device__ __forceinline__ void epilogue_chunk(const EpiParams& e, int row, int c, const uint32_t (&r)[32]) {
    if constexpr (KIND == EPI_BIAS || KIND == EPI_BIAS_GELU) {
        const uint4 none[4] = {};
        epilogue_chunk_f2<KIND>(e, row, c, r, none, global_out(e, row, c));
    } else {
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
    if (e.bias) {
        const float4* b4 = reinterpret_cast<const float4*>(e.bias + c);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float4 b = __ldg(b4 + i);
            v[4 * i] += b.x;
            v[4 * i + 1] += b.y;
            v[4 * i + 2] += b.z;
            v[4 * i + 3] += b.w;
        }
    }
    switch (KIND) {
        case EPI_BIAS:
        case EPI_BIAS_GELU:
        case EPI_BIAS_SILU: {
            if (KIND == EPI_BIAS_GELU) {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = gelu_tanh_f(v[i]);
            } else if (KIND == EPI_BIAS_SILU) {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = v[i] / (1.0f + __expf(-v[i]));
            }
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(e.out) + (long long)row * e.ldo + c);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint4 u;
                u.x = pack_bf16(v[8 * i], v[8 * i + 1]);
                u.y = pack_bf16(v[8 * i + 2], v[8 * i + 3]);
                u.z = pack_bf16(v[8 * i + 4], v[8 * i + 5]);
                u.w = pack_bf16(v[8 * i + 6], v[8 * i + 7]);
                dst[i] = u;
            }
            break;
        }
        case EPI_GATE_RESIDUAL:
        case EPI_RESIDUAL: {
            // issue every load of the chunk before any store: x (4 x 16 B) and the gate rows
            uint4* xp = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(e.out) + (long long)row * e.ldo + c);
            uint4 xu[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) xu[i] = xp[i];
            float g[32];
            if (KIND == EPI_GATE_RESIDUAL) {
#pragma unroll
                for (int i = 0; i < 32; ++i) g[i] = 0.0f;
                if (e.gate0) {
                    const float4* g0 = reinterpret_cast<const float4*>(e.gate0 + c);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float4 a = __ldg(g0 + i);
                        g[4 * i] = a.x;
                        g[4 * i + 1] = a.y;
                        g[4 * i + 2] = a.z;
                        g[4 * i + 3] = a.w;
                    }
                }
                if (e.gate1) {
                    const float4* g1 =
                        reinterpret_cast<const float4*>(e.gate1 + (long long)(row / e.mod_div) * e.mod_ld + c);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float4 a = __ldg(g1 + i);
                        g[4 * i] += a.x;
                        g[4 * i + 1] += a.y;
                        g[4 * i + 2] += a.z;
                        g[4 * i + 3] += a.w;
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t xw[4] = {xu[i].x, xu[i].y, xu[i].z, xu[i].w};
                uint32_t ow[4];
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const float2 xf = unpack_bf16(xw[h]);
                    const int cc = 8 * i + 2 * h;
                    if (KIND == EPI_GATE_RESIDUAL) {
                        ow[h] = pack_bf16(xf.x + v[cc] * g[cc], xf.y + v[cc + 1] * g[cc + 1]);
                    } else {
                        const float2 ab = unpack_bf16(pack_bf16(v[cc], v[cc + 1]));  // the branch output is bf16 first
                        ow[h] = pack_bf16(xf.x + ab.x, xf.y + ab.y);
                    }
                }
                xp[i] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
            }
            break;
        }
        case EPI_BIAS_F32: {
            float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(e.out) + (long long)row * e.ldo + c);
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            break;
        }
        case EPI_UNPATCHIFY: {
            // row = b * rows + r, token l = tok0 + r = (f * Hp + i) * Wp + j; column = (kh * 2 + kw) * C + ch
            const int Hp = e.Hz >> 1, Wp = e.Wz >> 1;
            const int rows = e.up_rows > 0 ? e.up_rows : e.L;
            const int b = row / rows;
            const int l = e.up_tok0 + (row - b * rows);
            if (l >= e.L) break;  // a padding row of a sequence shard
            const int f = l / (Hp * Wp);
            const int rem = l - f * (Hp * Wp);
            const int ii = rem / Wp;
            const int jj = rem - ii * Wp;
            float* vel = reinterpret_cast<float*>(e.out);
#pragma unroll
            for (int t = 0; t < 32; ++t) {
                const int col = c + t;
                const int ch = col % e.C;
                const int s = col / e.C;
                const int kh = s >> 1, kw = s & 1;
                const long long idx =
                    ((((long long)b * e.C + ch) * e.F + f) * e.Hz + (2 * ii + kh)) * e.Wz + (2 * jj + kw);
                vel[idx] = __bfloat162float(__float2bfloat16_rn(v[t]));
            }
            break;
        }
        default:
            break;
    }
    }
}

// EPI_QK_NORM on 32 consecutive columns [c, c + 32) of one row.  For normed
// columns the sum of squares of acc + bias is returned (fp32, before the
// gain) and the stored value is gain * (acc + bias), rotated pair by pair
// ((x0, x1) -> (x0 cos - x1 sin, x1 cos + x0 sin)) when RoPE is on; the row
// factor rsqrt(mean + eps) commutes with both and is applied later.  All of
// it on packed fp32 pairs, so the scalar FP32 pipe stays free for MMA issue.
// (frame, row, column) of the token of GEMM row `row` in the RoPE grid.
__device__ __forceinline__ void qk_position(const EpiParams& e, int row, int& f, int& ii, int& jj) {
    const int hw = e.rope.Hp * e.rope.Wp;
    const int l = min(e.rope_tok0 + row % e.rope_L, e.rope.Fp * hw - 1);
    f = l / hw;
    const int rem = l - f * hw;
    ii = rem / e.rope.Wp;
    jj = rem - ii * e.rope.Wp;
}

// RoPE (cos, sin) of the 16 rotation pairs of chunk K (32 columns) of a head,
// for the 22 / 21 / 21 pairs per axis of a 44 / 42 / 42 split: every pair's
// axis is fixed by the chunk, one multiply-add per table address.
template <int K>
__device__ __forceinline__ void qk_rope_load_fixed(const RopeTables& rt, int f, int ii, int jj, float2 (&cs)[16]) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int q = 16 * K + i;
        const float2* a = q < 22 ? rt.t + q * rt.Fp + f : (q < 43 ? rt.h + (q - 22) * rt.Hp + ii : rt.w + (q - 43) * rt.Wp + jj);
        cs[i] = __ldg(a);
    }
}

// RoPE (cos, sin) of the 16 rotation pairs of a 32-column chunk at token
// position (f, ii, jj), from the pair-major tables; loaded ahead of the chunk.
__device__ __forceinline__ void qk_rope_load(const EpiParams& e, int c, int f, int ii, int jj, float2 (&cs)[16]) {
    if (e.rope.nt == 22 && e.rope.nh == 21 && e.rope.nw == 21) {
        switch ((c & 127) >> 5) {
            case 0: qk_rope_load_fixed<0>(e.rope, f, ii, jj, cs); return;
            case 1: qk_rope_load_fixed<1>(e.rope, f, ii, jj, cs); return;
            case 2: qk_rope_load_fixed<2>(e.rope, f, ii, jj, cs); return;
            default: qk_rope_load_fixed<3>(e.rope, f, ii, jj, cs); return;
        }
    }
    const int p0 = (c & 127) >> 1;
#pragma unroll
    for (int i = 0; i < 16; ++i) cs[i] = __ldg(rope_entry_pm(e.rope, p0 + i, f, ii, jj));
}

template <class Out>
__device__ __forceinline__ float epilogue_qk_chunk(const EpiParams& e, int c, const uint32_t (&r)[32], bool normed,
                                                   const float2 (&cs)[16], const Out& out) {
    uint64_t v2[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) v2[i] = f2pack(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
    if (e.bias) {
        const ulonglong2* b2 = reinterpret_cast<const ulonglong2*>(e.bias + c);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const ulonglong2 b = __ldg(b2 + i);
            v2[2 * i] = add2(v2[2 * i], b.x);
            v2[2 * i + 1] = add2(v2[2 * i + 1], b.y);
        }
    }
    float ss = 0.0f;
    if (normed) {
        uint64_t s2 = 0ull;
#pragma unroll
        for (int i = 0; i < 16; ++i) s2 = fma2(v2[i], v2[i], s2);
        float sa, sb;
        f2unpack(s2, sa, sb);
        ss = sa + sb;
        const ulonglong2* g2 = reinterpret_cast<const ulonglong2*>(e.gain + c);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const ulonglong2 g = __ldg(g2 + i);
            v2[2 * i] = mul2(v2[2 * i], g.x);
            v2[2 * i + 1] = mul2(v2[2 * i + 1], g.y);
        }
        if (e.rope.t) {  // cs loaded by the caller ahead of the accumulator chunk
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float a, b;
                f2unpack(v2[i], a, b);
                v2[i] = fma2(v2[i], f2pack(cs[i].x, cs[i].x), mul2(f2pack(b, a), f2pack(-cs[i].y, cs[i].y)));
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t w[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            float a, b;
            f2unpack(v2[4 * i + h], a, b);
            w[h] = pack_bf16(a, b);
        }
        out.put(i, make_uint4(w[0], w[1], w[2], w[3]));
    }
    return ss;
}

// CFG + Euler on 32 consecutive columns [c, c + 32) of one token row: both
// velocities rounded to bf16 as proj_out's output is, then
// x_next = x + dsigma * (v_u + s (v_c - v_u)) at the unpatchify position.
__device__ __forceinline__ void epilogue_cfg_euler(const EpiParams& e, int row, int c, const uint32_t (&rc)[32],
                                                   const uint32_t (&ru)[32]) {
    const float s = __ldg(e.sched), dsig = __ldg(e.sched + 1);
    const int Hp = e.Hz >> 1, Wp = e.Wz >> 1;
    const int f = row / (Hp * Wp);
    const int rem = row - f * (Hp * Wp);
    const int ii = rem / Wp;
    const int jj = rem - ii * Wp;
    float* xn = reinterpret_cast<float*>(e.out);
#pragma unroll
    for (int t = 0; t < 32; ++t) {
        const int col = c + t;
        const int ch = col % e.C;
        const int sub = col / e.C;
        const int kh = sub >> 1, kw = sub & 1;
        const long long idx = (((long long)ch * e.F + f) * e.Hz + (2 * ii + kh)) * e.Wz + (2 * jj + kw);
        const float bias = e.bias ? __ldg(e.bias + col) : 0.0f;
        const float vc = __bfloat162float(__float2bfloat16_rn(__uint_as_float(rc[t]) + bias));
        const float vu = __bfloat162float(__float2bfloat16_rn(__uint_as_float(ru[t]) + bias));
        const float v = __fmaf_rn(s, vc - vu, vu);
        xn[idx] = __fmaf_rn(dsig, v, __ldg(e.x + idx));
    }
}

__host__ __device__ constexpr bool reads_residual(int kind) { return kind == EPI_GATE_RESIDUAL || kind == EPI_RESIDUAL; }
// SM-pair epilogues that go through a shared-memory slab per warp (TMA-loaded
// residual, TMA-stored results; 5 ring stages): the residual and q/k-norm
// kinds.  Bias and GELU keep 6 stages and store from registers (their long-K
// or wide-N mainloops gained nothing from the slab and lost a ring stage).
__host__ __device__ constexpr bool uses_slab(int kind) { return reads_residual(kind) || kind == EPI_QK_NORM; }

// Residual of the first chunk of an epilogue warp's share of tile (row, nb),
// loaded before the warp waits for the accumulator.
template <int BN, int KIND>
__device__ __forceinline__ void epilogue_prefetch(const GemmParams& p, int row, int nb, int chalf, uint4 (&x0)[4]) {
    if constexpr (reads_residual(KIND)) {
        if (row < p.M) load_residual(p.epi, row, nb * BN + chalf * (BN / 2), x0);
    }
}

// One epilogue warp's share of an accumulator tile: TMEM lanes of its quarter
// (rows `row`), columns [chalf * BN/2, (chalf + 1) * BN/2) of tile column `nb`.
// x0: the residual of its first chunk (residual epilogues).
template <int BN, int KIND, bool PAIR>
__device__ __forceinline__ void epilogue_tile(const GemmParams& p, int row, int nb, uint32_t taddr, int chalf,
                                              uint4 (&x0)[4]) {
    constexpr int CW = BN / 2;  // columns per epilogue warp
    if constexpr (reads_residual(KIND)) {
        // the residual of chunk k + 1 loads while chunk k is computed, through
        // two buffers (a buffer is reused only after its values are consumed)
        uint4 x1[4];
        auto chunk = [&](int k, uint4 (&use)[4], uint4 (&next)[4]) {
            const int c0 = chalf * CW + k * 32;
            if (k + 1 < CW / 32 && row < p.M) load_residual(p.epi, row, nb * BN + c0 + 32, next);
            uint32_t r[32];
            tmem_ld32(taddr + c0, r);
            tmem_ld_wait(r);
            if (row < p.M) epilogue_chunk_f2<KIND>(p.epi, row, nb * BN + c0, r, use, global_out(p.epi, row, nb * BN + c0));
        };
        chunk(0, x0, x1);
        if constexpr (CW / 32 > 1) chunk(1, x1, x0);
        if constexpr (CW / 32 > 2) chunk(2, x0, x1);
        if constexpr (CW / 32 > 3) chunk(3, x1, x0);
    } else if constexpr (KIND == EPI_QK_NORM) {
        // this warp's 128 columns are one head: its sum of squares is one ssq entry
        static_assert(BN == 256, "one 128-column group per epilogue warp");
        const int gcol = nb * BN + chalf * CW;
        const bool normed = gcol < p.epi.norm_cols;
        int f = 0, ii = 0, jj = 0;
        if (normed && p.epi.rope.t) qk_position(p.epi, row, f, ii, jj);
        float ss = 0.0f;
        // the RoPE entries of chunk k + 1 load while chunk k is read out of tensor
        // memory and computed (two buffers, each reused after its values are consumed)
        const bool rope = normed && p.epi.rope.t;
        float2 ca[16], cb[16];
        auto chunk = [&](int k, float2 (&use)[16], float2 (&next)[16]) {
            const int c0 = chalf * CW + k * 32;
            uint32_t r[32];
            tmem_ld32(taddr + c0, r);
            if (k + 1 < CW / 32 && rope) qk_rope_load(p.epi, nb * BN + c0 + 32, f, ii, jj, next);
            tmem_ld_wait(r);
            if (row < p.M) ss += epilogue_qk_chunk(p.epi, nb * BN + c0, r, normed, use, global_out(p.epi, row, nb * BN + c0));
        };
        if (rope) qk_rope_load(p.epi, nb * BN + chalf * CW, f, ii, jj, ca);
        chunk(0, ca, cb);
        chunk(1, cb, ca);
        chunk(2, ca, cb);
        chunk(3, cb, ca);
        if (normed && row < p.M) p.epi.ssq[(long long)row * p.epi.ssq_ld + gcol / 128] = ss;
    } else {
#pragma unroll 1
        for (int c0 = chalf * CW; c0 < (chalf + 1) * CW; c0 += 32) {
            uint32_t r[32];
            tmem_ld32(taddr + c0, r);
            tmem_ld_wait(r);
            if constexpr (PAIR) {
                uint32_t ru[32];
                tmem_ld32(taddr + BN + c0, ru);
                tmem_ld_wait(ru);
                if (row < p.M) epilogue_cfg_euler(p.epi, row, nb * BN + c0, r, ru);
            } else {
                if (row < p.M) epilogue_chunk<KIND>(p.epi, row, nb * BN + c0, r);
            }
        }
    }
}

constexpr int EPI_WARPS = 8;
constexpr int GEMM_THREADS = 64 + 32 * EPI_WARPS;

// SM-pair epilogue of one warp's share of a tile through its shared-memory
// slab: 32 rows (r = the thread's row in the slab) x 128 columns as two
// 64-column boxes with the 128-byte swizzle.  Residual kinds read x from the
// slab (TMA-loaded by the caller); every kind writes its bf16 results into the
// slab, which the caller then stores with TMA.
template <int KIND>
__device__ __forceinline__ void epilogue_tile_slab(const GemmParams& p, int row, int nb, uint32_t taddr, int chalf,
                                                   uint8_t* xs, int r) {
    constexpr int BN = 256, CW = 128;
    const int r7 = r & 7;
    auto slab = [&](int k) { return SlabOut{xs + (k >> 1) * (32 * 128) + r * 128, 4 * (k & 1), r7}; };
    if constexpr (KIND == EPI_QK_NORM) {
        const int gcol = nb * BN + chalf * CW;
        const bool normed = gcol < p.epi.norm_cols;
        int f = 0, ii = 0, jj = 0;
        if (normed && p.epi.rope.t) qk_position(p.epi, row, f, ii, jj);
        float ss = 0.0f;
        const bool rope = normed && p.epi.rope.t;
#pragma unroll 1
        for (int k = 0; k < CW / 32; ++k) {
            // the chunk's 16 RoPE entries load while its accumulator columns are read out
            const int c0 = chalf * CW + k * 32;
            uint32_t acc[32];
            float2 cs[16];
            tmem_ld32(taddr + c0, acc);
            if (rope) qk_rope_load(p.epi, nb * BN + c0, f, ii, jj, cs);
            tmem_ld_wait(acc);
            if (row < p.M) ss += epilogue_qk_chunk(p.epi, nb * BN + c0, acc, normed, cs, slab(k));
        }
        if (normed && row < p.M) p.epi.ssq[(long long)row * p.epi.ssq_ld + gcol / 128] = ss;
    } else {
#pragma unroll 1
        for (int k = 0; k < CW / 32; ++k) {
            const int c0 = chalf * CW + k * 32;
            uint32_t acc[32];
            tmem_ld32(taddr + c0, acc);
            uint4 xu[4] = {};
            if constexpr (reads_residual(KIND)) {
                const SlabOut s = slab(k);
#pragma unroll
                for (int i = 0; i < 4; ++i) xu[i] = *reinterpret_cast<const uint4*>(s.rowp + (((s.j0 + i) ^ r7) << 4));
            }
            tmem_ld_wait(acc);
            if (row < p.M) epilogue_chunk_f2<KIND>(p.epi, row, nb * BN + c0, acc, xu, slab(k));
        }
    }
}

template <int BN, int KIND>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const GemmParams p) {
    constexpr bool PAIR = KIND == EPI_CFG_EULER;
    using Cfg = GemmCfg<BN, PAIR>;
    constexpr int STAGES = Cfg::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;                                   // [STAGES][NA] A tiles
    uint8_t* sB = smem + STAGES * Cfg::NA * Cfg::A_BYTES;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * Cfg::STAGE_BYTES);
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
            mbar_init(tempty + a, EPI_WARPS);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int kblocks = p.K / Cfg::BK;
    // producer: stages with a load issued and the phase it completes; MMA issuer:
    // whether any MMA went out (both drained after an abort, before the CTA exits)
    uint32_t armed = 0, armed_par = 0;
    bool issued = false;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer ----------------
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
                int mb, nb;
                tile_coords(tile, p, mb, nb);
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(empty + stage, phase ^ 1, abort_flag, p.wc)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(full + stage, Cfg::STAGE_BYTES);
                    tma_load_2d(sA + stage * Cfg::NA * Cfg::A_BYTES, &tmA, full + stage, kb * Cfg::BK, mb * Cfg::BM);
                    if constexpr (PAIR)
                        tma_load_2d(sA + (stage * 2 + 1) * Cfg::A_BYTES, &tmA, full + stage, kb * Cfg::BK,
                                    p.epi.pair_off + mb * Cfg::BM);
                    tma_load_2d(sB + stage * Cfg::B_BYTES, &tmB, full + stage, kb * Cfg::BK, nb * BN);
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
            constexpr int ACC_COLS = Cfg::NA * BN;            // TMEM columns of one accumulator set
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
                const uint32_t d_tmem = tmem_base + acc * ACC_COLS;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(full + stage, phase, abort_flag, p.wc)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sA + stage * Cfg::NA * Cfg::A_BYTES);
                    const uint32_t b0 = smem_u32(sB + stage * Cfg::B_BYTES);
#pragma unroll
                    for (int k = 0; k < Cfg::BK / 16; ++k) {
                        umma_bf16_ss(d_tmem, sdesc_kmajor_sw128(a0 + 32 * k), sdesc_kmajor_sw128(b0 + 32 * k), IDESC,
                                     (kb | k) != 0);
                        if constexpr (PAIR)
                            umma_bf16_ss(d_tmem + BN, sdesc_kmajor_sw128(a0 + Cfg::A_BYTES + 32 * k),
                                         sdesc_kmajor_sw128(b0 + 32 * k), IDESC, (kb | k) != 0);
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
        // ---------------- epilogue warps ----------------
        const int q = warp & 3;                       // TMEM lane quarter this warp may access
        const int chalf = (warp - 2) >> 2;            // which half of the tile's columns
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
            int mb, nb;
            tile_coords(tile, p, mb, nb);
            const int row = mb * 128 + q * 32 + lane;
            uint4 x0[4];
            epilogue_prefetch<BN, KIND>(p, row, nb, chalf, x0);
            // tcgen05.ld is warp-collective: the whole warp takes the same branch
            if (!__all_sync(0xffffffffu, mbar_wait(tfull + acc, acc_phase, abort_flag, p.wc))) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * (Cfg::NA * BN);
            epilogue_tile<BN, KIND, PAIR>(p, row, nb, taddr, chalf, x0);
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
        tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
}

// ----------------------------------------------------------------------------
// SM-pair GEMM (tcgen05 .cta_group::2): a cluster of two CTAs computes a
// 256 x 256 tile; the even CTA issues one M = 256, N = 256, K = 16 MMA per
// 16-deep K slice.  Each CTA stages its own 128 A rows and its own 128-row half
// of the W tile (32 KB per 64-deep K step instead of the 48 KB a 128 x 256
// single-SM tile needs), and the tensor cores of the pair read both halves of
// W, which halves W's shared-memory and L2 traffic per SM.  Each CTA's tensor
// memory holds the accumulator rows of its own A rows (all 256 columns), so
// the epilogue is the single-SM one.
//
// Barriers sit at the same shared-memory offsets in both CTAs:
//   full[s]    even CTA: 1 arrival (its producer, announcing the bytes of both
//              CTAs' loads) + those bytes, which each CTA's loads deliver;
//   empty[s]   both: 1 arrival, the MMA commit multicast to the pair;
//   tfull[a]   both: 1 arrival, the MMA commit multicast to the pair;
//   tempty[a]  even CTA: 16 arrivals, the 8 epilogue warps of each CTA.
// All handshakes use CTA-scope acquire / release, also across the pair: the
// data they guard moves through the async proxy (TMA bytes counted on the
// barrier, MMA commits) or through tensor memory under tcgen05 fences, and a
// cluster-scope release would put a memory barrier into every K step.
// Teardown: both CTAs stop issuing, synchronise, and if either gave up a wait
// the even CTA completes every full[s] phase a load of either CTA went into
// and drains its MMAs before the pair synchronises again and frees its
// tensor memory.
// ----------------------------------------------------------------------------
namespace pair2 {
constexpr int BN = 256;
constexpr int HALF_BYTES = 128 * 64 * 2;      // one 128 x 64 bf16 operand tile
constexpr int STAGE_BYTES = 2 * HALF_BYTES;   // A rows + W half
constexpr int TMEM_COLS = 2 * BN;
constexpr int XSLAB_BYTES = 32 * 128 * 2;     // one epilogue warp's residual rows: 32 x 128 bf16
// Residual epilogues stage each warp's residual slab in shared memory (two
// 64-column TMA boxes, 128-byte swizzle), which leaves room for 5 ring stages.
template <bool STAGE_X>
struct Cfg {
    static constexpr int STAGES = STAGE_X ? 5 : 6;
    static constexpr int X_BYTES = STAGE_X ? EPI_WARPS * XSLAB_BYTES : 0;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + X_BYTES + 1024 + 256;
};
// loads a producer that issued n loads put into stage s
template <int STAGES>
__device__ __forceinline__ uint32_t loads_in_stage(uint32_t n, int s) {
    return n > (uint32_t)s ? (n - 1 - s) / STAGES + 1 : 0u;
}
}  // namespace pair2

// tmX (residual epilogues): the residual / output matrix, 64 x 32 boxes.
template <int KIND>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(GEMM_THREADS, 1)
    gemm_pair_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmX, const GemmParams p) {
    using namespace pair2;
    constexpr bool STAGE_X = uses_slab(KIND);
    constexpr int STAGES = Cfg<STAGE_X>::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;                          // [STAGES] this CTA's 128 A rows x 64
    uint8_t* sB = smem + STAGES * HALF_BYTES;    // [STAGES] this CTA's 128 W rows x 64
    uint8_t* sX = smem + STAGES * STAGE_BYTES;   // [EPI_WARPS] residual slabs (STAGE_X)
    uint64_t* full = reinterpret_cast<uint64_t*>(sX + Cfg<STAGE_X>::X_BYTES);
    uint64_t* empty = full + STAGES;
    uint64_t* tfull = empty + STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint64_t* xbar = drain + 1;                  // [EPI_WARPS] residual slab landed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(xbar + EPI_WARPS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile uint32_t* loads_issued = reinterpret_cast<volatile uint32_t*>(tmem_slot + 2);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();     // 0: the CTA that issues the MMAs
    const bool leader = rank == 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull + a, 1);
            mbar_init(tempty + a, 2 * EPI_WARPS);
        }
        mbar_init(drain, 1);
        for (int w = 0; w < EPI_WARPS; ++w) mbar_init(xbar + w, 1);
        *abort_flag = 0;
        *loads_issued = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if (STAGE_X) tma_prefetch_desc(&tmX);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();   // barriers initialised and tensor memory allocated in both CTAs
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int kblocks = p.K / 64;
    const int cid = static_cast<int>(cluster_id_x());
    const int ncl = static_cast<int>(num_clusters_x());
    uint32_t n_loads = 0;
    bool issued = false;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer (both CTAs) ----------------
            const uint32_t full0 = mapa_shared(smem_u32(full), 0);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = cid; ok && tile < p.num_tiles; tile += ncl) {
                int mb, nb;
                tile_coords(tile, p, mb, nb);
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(empty + stage, phase ^ 1, abort_flag, p.wc)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = full0 + 8u * stage;
                    if (leader) mbar_expect_tx(full + stage, 2 * STAGE_BYTES);
                    tma_load_2d_pair(sA + stage * HALF_BYTES, &tmA, fb, kb * 64, mb * 256 + rank * 128);
                    tma_load_2d_pair(sB + stage * HALF_BYTES, &tmB, fb, kb * 64, nb * BN + rank * 128);
                    ++n_loads;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            // the MMA commits that free this CTA's stages arrive here: wait for
            // the last of them so none lands after the CTA has exited
            for (int s = 0; ok && s < STAGES; ++s) {
                const uint32_t c = loads_in_stage<STAGES>(n_loads, s);
                if (c) ok = mbar_wait(empty + s, (c - 1) & 1u, abort_flag, p.wc);
            }
            *loads_issued = n_loads;
        }
    } else if (warp == 1) {
        if (leader && lane == 0) {
            // ---------------- MMA issuer (even CTA) ----------------
            constexpr uint32_t IDESC = idesc_bf16(256, BN, false);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int tile = cid; ok && tile < p.num_tiles; tile += ncl) {
                if (!mbar_wait(tempty + acc, acc_phase ^ 1, abort_flag, p.wc)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * BN;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(full + stage, phase, abort_flag, p.wc)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sA + stage * HALF_BYTES);
                    const uint32_t b0 = smem_u32(sB + stage * HALF_BYTES);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        umma_bf16_ss_pair(d_tmem, sdesc_kmajor_sw128(a0 + 32 * k), sdesc_kmajor_sw128(b0 + 32 * k),
                                          IDESC, (kb | k) != 0);
                    issued = true;
                    umma_commit_pair_mc(empty + stage, 0x3);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                umma_commit_pair_mc(tfull + acc, 0x3);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1;
            }
        }
    } else {
        // ---------------- epilogue warps (both CTAs) ----------------
        const int q = warp & 3;
        const int chalf = (warp - 2) >> 2;
        const uint32_t tempty0 = mapa_shared(smem_u32(tempty), 0);
        // each epilogue warp owns a slab of 32 rows x 128 columns: residual kinds
        // TMA-load the tile's x into it ahead of the accumulator (the next tile's as
        // soon as the current one has been stored), every kind writes its results
        // into it and stores them with TMA
        uint8_t* xs = sX + (warp - 2) * XSLAB_BYTES;
        uint64_t* xb = xbar + (warp - 2);
        uint32_t xpar = 0;
        bool xarmed = false, stored = false;
        auto slab_coords = [&](int tile, int& c0, int& r0) {
            int mb, nb;
            tile_coords(tile, p, mb, nb);
            r0 = mb * 256 + static_cast<int>(rank) * 128 + q * 32;
            c0 = nb * BN + chalf * 128;
        };
        auto load_x = [&](int tile) {
            int c0, r0;
            slab_coords(tile, c0, r0);
            if (lane == 0) {
                fence_proxy_async_smem();  // the slab's previous contents were read through the generic proxy
                mbar_expect_tx(xb, XSLAB_BYTES);
                tma_load_2d(xs, &tmX, xb, c0, r0);
                tma_load_2d(xs + XSLAB_BYTES / 2, &tmX, xb, c0 + 64, r0);
            }
            xarmed = true;
        };
        // the previous tile's store has read the slab (before it is rewritten)
        auto slab_free = [&]() {
            if (stored && lane == 0) bulk_wait_read_all();
            __syncwarp();
        };
        if (STAGE_X && reads_residual(KIND) && cid < p.num_tiles) load_x(cid);
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = cid; tile < p.num_tiles; tile += ncl) {
            int mb, nb;
            tile_coords(tile, p, mb, nb);
            const int row = mb * 256 + static_cast<int>(rank) * 128 + q * 32 + lane;
            if (!__all_sync(0xffffffffu, mbar_wait(tfull + acc, acc_phase, abort_flag, p.wc))) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN;
            if constexpr (!STAGE_X) {  // bias / GELU: results stored from registers
                uint4 x0[4];
                epilogue_tile<BN, KIND, false>(p, row, nb, taddr, chalf, x0);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(tempty0 + 8u * acc);
            } else {
                if constexpr (reads_residual(KIND)) {
                    if (!__all_sync(0xffffffffu, mbar_wait(xb, xpar, abort_flag, p.wc))) break;
                    xarmed = false;
                    xpar ^= 1;
                } else {
                    slab_free();
                }
                epilogue_tile_slab<KIND>(p, row, nb, taddr, chalf, xs, lane);
                tc_fence_before();
                fence_proxy_async_smem();  // the slab's results, written through the generic proxy, go out by TMA
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive_remote(tempty0 + 8u * acc);
                    int c0, r0;
                    slab_coords(tile, c0, r0);
                    tma_store_2d(&tmX, xs, c0, r0);
                    tma_store_2d(&tmX, xs + XSLAB_BYTES / 2, c0 + 64, r0);
                    bulk_commit();
                }
                stored = true;
                if (reads_residual(KIND) && tile + ncl < p.num_tiles) {
                    slab_free();
                    load_x(tile + ncl);
                }
            }
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1;
        }
        // stores complete and a slab load still in flight lands before the CTA's
        // shared memory is released
        if (stored && lane == 0) bulk_wait_all();
        if (xarmed && lane == 0) mbar_drain(xb, xpar, 200000000ull);
    }

    __syncthreads();
    cluster_sync_all();   // neither CTA issues another load, MMA or arrival
    const bool any_abort =
        *abort_flag != 0 || ld_shared_cluster_u32(mapa_shared(smem_u32((const void*)abort_flag), rank ^ 1u)) != 0;
    if (any_abort && leader && lane == 0) {
        if (warp == 0) {
            // every full[s] phase that a load of either CTA went into completes
            // once the loads issued into it have landed.  The two producers'
            // counts per stage differ by at most one (a load of phase j waits
            // for phase j - 1 to be consumed); where the odd CTA stopped first,
            // its bytes are counted as delivered, where the even CTA did, the
            // arrival it owed is made for the odd CTA's bytes alone
            const uint32_t n0 = *loads_issued;
            const uint32_t n1 = ld_shared_cluster_u32(mapa_shared(smem_u32((const void*)loads_issued), 1));
            for (int s = 0; s < STAGES; ++s) {
                const uint32_t c0 = loads_in_stage<STAGES>(n0, s), c1 = loads_in_stage<STAGES>(n1, s);
                const uint32_t c = c0 > c1 ? c0 : c1;
                if (!c) continue;
                if (c0 > c1) mbar_complete_tx(full + s, STAGE_BYTES);
                if (c1 > c0) mbar_expect_tx(full + s, STAGE_BYTES);
                mbar_drain(full + s, (c - 1) & 1u, 200000000ull);
            }
        } else if (warp == 1 && issued) {
            umma_commit_pair(drain);
            mbar_drain(drain, 0, 200000000ull);
        }
    }
    __syncthreads();
    cluster_sync_all();   // the pair's loads and MMAs have landed
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

template <int BN, int KIND>
static cudaError_t set_gemm_attr_one() {
    return cudaFuncSetAttribute(gemm_tc_kernel<BN, KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                GemmCfg<BN, KIND == EPI_CFG_EULER>::SMEM_BYTES);
}

template <int BN>
static cudaError_t set_gemm_attr() {
    cudaError_t e = set_gemm_attr_one<BN, EPI_BIAS>();
    if (e == cudaSuccess) e = set_gemm_attr_one<BN, EPI_BIAS_GELU>();
    if (e == cudaSuccess) e = set_gemm_attr_one<BN, EPI_GATE_RESIDUAL>();
    if (e == cudaSuccess) e = set_gemm_attr_one<BN, EPI_RESIDUAL>();
    if (e == cudaSuccess) e = set_gemm_attr_one<BN, EPI_BIAS_F32>();
    if (e == cudaSuccess) e = set_gemm_attr_one<BN, EPI_UNPATCHIFY>();
    if (e == cudaSuccess) e = set_gemm_attr_one<BN, EPI_BIAS_SILU>();
    return e;
}

// Clusters of two that fit on the device at once with one pair CTA per SM
// (0: the pair kernel is not used).
static int g_pair_clusters = 0;

template <int KIND>
static cudaError_t set_pair_attr_one() {
    return cudaFuncSetAttribute(gemm_pair_tc_kernel<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                pair2::Cfg<uses_slab(KIND)>::SMEM_BYTES);
}

static cudaError_t init_pair_gemm() {
    cudaError_t e = set_pair_attr_one<EPI_BIAS>();
    if (e == cudaSuccess) e = set_pair_attr_one<EPI_BIAS_GELU>();
    if (e == cudaSuccess) e = set_pair_attr_one<EPI_GATE_RESIDUAL>();
    if (e == cudaSuccess) e = set_pair_attr_one<EPI_RESIDUAL>();
    if (e == cudaSuccess) e = set_pair_attr_one<EPI_QK_NORM>();
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (sms / 2), 1, 1);
    cfg.blockDim = dim3(GEMM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = pair2::Cfg<false>::SMEM_BYTES;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_pair_tc_kernel<EPI_BIAS>, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
    }
    g_pair_clusters = n;
    return cudaSuccess;
}

int gemm_pair_clusters() { return g_pair_clusters; }

cudaError_t init_gemm_attributes() {
    cudaError_t e = init_pair_gemm();
    if (e == cudaSuccess) e = set_gemm_attr<256>();
    if (e == cudaSuccess) e = set_gemm_attr<128>();
    if (e == cudaSuccess) e = set_gemm_attr<64>();
    if (e == cudaSuccess) e = set_gemm_attr_one<64, EPI_CFG_EULER>();
    if (e == cudaSuccess) e = set_gemm_attr_one<256, EPI_QK_NORM>();
    return e;
}

template <int BN>
static cudaError_t launch_gemm_bn(const CUtensorMap& ta, const CUtensorMap& tb, const GemmParams& p,
                                  const LaunchCtx& ctx) {
    using Cfg = GemmCfg<BN>;
    const int grid = p.num_tiles < ctx.num_sms ? p.num_tiles : ctx.num_sms;
    if (p.epi.kind == EPI_CFG_EULER) {  // 64-column tiles only (proj_out: N = 4 * out_ch)
        if (BN != 64) return cudaErrorInvalidValue;
        gemm_tc_kernel<64, EPI_CFG_EULER><<<grid, GEMM_THREADS, GemmCfg<64, true>::SMEM_BYTES, ctx.stream>>>(ta, tb, p);
        if (ctx.launches) ++*ctx.launches;
        return cudaGetLastError();
    }
    if (p.epi.kind == EPI_QK_NORM) {  // 256-column tiles only: one head per epilogue warp
        if (BN != 256) return cudaErrorInvalidValue;
        gemm_tc_kernel<256, EPI_QK_NORM><<<grid, GEMM_THREADS, GemmCfg<256>::SMEM_BYTES, ctx.stream>>>(ta, tb, p);
        if (ctx.launches) ++*ctx.launches;
        return cudaGetLastError();
    }
    switch (p.epi.kind) {
#define WAN_GEMM_CASE(K)                                                                   \
    case K:                                                                                \
        gemm_tc_kernel<BN, K><<<grid, GEMM_THREADS, Cfg::SMEM_BYTES, ctx.stream>>>(ta, tb, p); \
        break;
        WAN_GEMM_CASE(EPI_BIAS)
        WAN_GEMM_CASE(EPI_BIAS_GELU)
        WAN_GEMM_CASE(EPI_GATE_RESIDUAL)
        WAN_GEMM_CASE(EPI_RESIDUAL)
        WAN_GEMM_CASE(EPI_BIAS_F32)
        WAN_GEMM_CASE(EPI_UNPATCHIFY)
        WAN_GEMM_CASE(EPI_BIAS_SILU)
#undef WAN_GEMM_CASE
        default:
            return cudaErrorInvalidValue;
    }
    if (ctx.launches) ++*ctx.launches;
    return cudaGetLastError();
}

cudaError_t launch_gemm(const void* A, long long lda, const void* W, long long ldw, int M, int N, int K,
                        const EpiParams& epi, const LaunchCtx& ctx) {
    if (M <= 0) return cudaSuccess;
    if (K <= 0 || K % 64 != 0 || N <= 0 || N % 64 != 0 || lda % 8 != 0 || ldw % 8 != 0)
        return cudaErrorInvalidValue;
    if ((reinterpret_cast<uintptr_t>(A) & 15) || (reinterpret_cast<uintptr_t>(W) & 15)) return cudaErrorInvalidValue;
    int BN = (N % 256 == 0) ? 256 : (N % 128 == 0) ? 128 : 64;
    const bool pair = epi.kind == EPI_CFG_EULER;
    if (pair) {
        BN = 64;
        if (epi.pair_off < M || !epi.x || !epi.sched || !epi.out) return cudaErrorInvalidValue;
    }
    if (epi.kind == EPI_QK_NORM) {  // the epilogue reads pair-major RoPE tables
        if ((epi.rope.t && !epi.rope.pair_major) ||
            N % 256 || epi.norm_cols < 0 || epi.norm_cols % 128 || epi.norm_cols > N || !epi.ssq ||
            (epi.norm_cols > 0 && !epi.gain) || epi.ssq_ld < epi.norm_cols / 128 || epi.ldo % 8 ||
            (epi.rope.t && epi.rope_L <= 0))
            return cudaErrorInvalidValue;
    }
    bool use_pair = ctx.gemm_pair && g_pair_clusters > 0 && BN == 256 && M >= 512 &&
                    (epi.kind == EPI_BIAS || epi.kind == EPI_BIAS_GELU || epi.kind == EPI_GATE_RESIDUAL ||
                     epi.kind == EPI_RESIDUAL || epi.kind == EPI_QK_NORM);
    // the pair epilogue loads residuals and stores results through TMA (32-row x
    // 64-column boxes of the bf16 output); an output TMA cannot describe (a
    // pointer or row stride off 16 bytes) takes the single-SM tiles instead
    CUtensorMap tx;
    if (use_pair && !make_tmap_2d(&tx, epi.out, (uint64_t)N, (uint64_t)M, (uint64_t)epi.ldo, 64, 32))
        use_pair = false;
    GemmParams p;
    p.M = M;
    p.N = N;
    p.K = K;
    p.num_m = use_pair ? (M + 255) / 256 : (M + 127) / 128;
    p.num_n = N / BN;
    p.num_tiles = p.num_m * p.num_n;
    // walk M fastest when the weight operand is the bigger one (few row blocks)
    p.m_fastest = ((long long)M < (long long)N) ? 1 : 0;
    p.epi = epi;
    if (p.epi.mod_div <= 0) p.epi.mod_div = 1;
    p.wc.err = ctx.err;
    p.wc.limit_ns = ctx.wait_limit_ns;
    CUtensorMap ta, tb;
    // the pair variant reads the second sample's rows [pair_off, pair_off + M) as well
    const uint64_t a_rows = pair ? (uint64_t)epi.pair_off + (uint64_t)M : (uint64_t)M;
    if (!make_tmap_2d(&ta, A, K, a_rows, lda, 64, 128)) return cudaErrorInvalidValue;
    if (!make_tmap_2d(&tb, W, K, N, ldw, 64, use_pair ? 128 : BN)) return cudaErrorInvalidValue;
    if (use_pair) {
        const int clusters = p.num_tiles < g_pair_clusters ? p.num_tiles : g_pair_clusters;
        switch (epi.kind) {
#define WAN_PAIR_CASE(K)                                                                                   \
    case K:                                                                                                \
        gemm_pair_tc_kernel<K><<<2 * clusters, GEMM_THREADS, pair2::Cfg<uses_slab(K)>::SMEM_BYTES,         \
                                 ctx.stream>>>(ta, tb, tx, p);                                             \
        break;
            WAN_PAIR_CASE(EPI_BIAS)
            WAN_PAIR_CASE(EPI_BIAS_GELU)
            WAN_PAIR_CASE(EPI_GATE_RESIDUAL)
            WAN_PAIR_CASE(EPI_RESIDUAL)
            WAN_PAIR_CASE(EPI_QK_NORM)
#undef WAN_PAIR_CASE
            default:
                return cudaErrorInvalidValue;
        }
        if (ctx.launches) ++*ctx.launches;
        return cudaGetLastError();
    }
    switch (BN) {
        case 256: return launch_gemm_bn<256>(ta, tb, p, ctx);
        case 128: return launch_gemm_bn<128>(ta, tb, p, ctx);
        default: return launch_gemm_bn<64>(ta, tb, p, ctx);
    }
}

}  // namespace wan

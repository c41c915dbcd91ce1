// Flash attention on tcgen05 for the Wan DiT: O = softmax(Q K^T / sqrt(128)) V
// per (batch, head), no mask, head_dim 128, bf16 operands, fp32 softmax.
// Two kernels:
//   attn_pair_kernel  the self-attention over the L video tokens: SM pairs
//                     (tcgen05 .cta_group::2), 512 queries per cluster, P in
//                     shared memory (described above the kernel);
//   attn_tc_kernel    short key sets (up to four 128-key tiles: the
//                     cross-attention to the Lc text tokens, ragged key tail
//                     masked), one SM per CTA, P in tensor memory.
//
// attn_tc_kernel.  Work unit: 256 queries (two 128-row tiles) of one (head,
// batch).  One CTA per SM walks units blockIdx.x, blockIdx.x + gridDim.x, ...,
// since a unit is only a few key tiles and the set-up (barriers, tensor
// memory, the first Q load) would otherwise be paid per unit.  Barrier phases
// run on over the units: Q once per unit (the next unit's Q loads as soon as
// the last S MMA of the current one has read Q), K / V / S / P once per key
// tile.  12 warps in three warpgroups; the first gives registers to the two
// softmax groups (104 / 192 / 192 per thread, 62464 of the 384 x 168 = 64512
// at launch):
//   warp 0      TMA producer: both Q tiles of a unit, then K and V tiles of 128
//               keys in two-slot rings (3-D tensor maps: rows past the
//               sequence read as zero);
//   warp 1      tensor-memory owner and MMA issuer.  Tensor memory holds
//               S0 | S1 | O0 | O1 (4 x 128 fp32 columns).  Per key tile j and
//               query tile t it issues S_t(j+1) for keys 64..127 as soon as
//               the softmax has read S_t(j), then P_t(j) V_j in two K = 64
//               halves (the first once the softmax has stored the
//               probabilities of keys 0..63), then S_t(j+1) for keys 0..63,
//               whose columns P_t(j) occupied;
//   warps 2..3  idle;
//   warps 4..7  softmax of tile 0, warps 8..11 softmax of tile 1 (one query
//               row per thread): tcgen05.ld of the S row, running max / sum in
//               fp32 (log2 domain), probabilities packed to bf16 and written
//               back with tcgen05.st over the S columns they came from (P
//               aliases S), read there by the P.V MMA as its A operand.  O is
//               rescaled in TMEM only when a row maximum grows by more than
//               2^8 (the stale maximum is exact because the final division
//               uses the same running sum); at the end each row is divided by
//               its sum and stored as bf16.
#include "common.cuh"
#include "kernels.h"

namespace wan {

struct AttnParams {
    int Lq, Lk, heads;
    int nqb, units;    // 256-row query blocks per (head, batch); nqb * heads * batch
    __nv_bfloat16* o;
    long long ldo;
    float scale_log2;  // log2(e) / sqrt(head_dim)
    RowNorm qn;        // RMSNorm row factors of unnormalised queries (qn.ssq null: none)
    WaitCtl wc;
};

namespace attn {
constexpr int TILE_BYTES = 128 * 128 * 2;  // one 128 x 128 bf16 tile = two 64-column swizzled halves
constexpr int HALF_BYTES = 128 * 128;      // 128 rows x 128 bytes
constexpr int KSTAGES = 2;                         // K ring slots (a third measured neutral)
constexpr int VSTAGES = 2;
constexpr int SQ = 0;                              // Q0 | Q1
constexpr int SK = SQ + 2 * TILE_BYTES;            // K ring
constexpr int SV = SK + KSTAGES * TILE_BYTES;      // V ring
constexpr int SBAR = SV + VSTAGES * TILE_BYTES;
constexpr int SMEM_BYTES = SBAR + 256 + 1024;
constexpr int THREADS = 384;
constexpr int REGS_LAUNCH = 168;   // 65536 / 384 rounded down to a multiple of 8
// warpgroup 0 (producer + MMA issuer) / warpgroups 1, 2 (softmax), measured in
// the 480p step: 88 / 208 spilled in the issuer (1-2 % slower than 96 / 200),
// 104 / 192 ran 0.8 % faster than 96 / 200 and level with 120 / 192, 112 / 184
// spills in the softmax
constexpr int REGS_CONTROL = 104;
constexpr int REGS_SOFTMAX = 192;
static_assert(128 * REGS_CONTROL + 256 * REGS_SOFTMAX <= THREADS * REGS_LAUNCH, "register split");
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units
// P.V of a key tile goes in two K = 64 halves, the first issued as soon as the
// softmax has stored the probabilities of keys 0..63 (measured at the 480p
// shape: two parts ~1210 TFLOP/s, four ~1035, one ~1060).
constexpr int PV_PARTS = 2;
}  // namespace attn

__global__ void __launch_bounds__(attn::THREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
    using namespace attn;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SBAR);
    uint64_t* q_full = bars + 0;
    uint64_t* q_empty = bars + 1;                // every S MMA of the unit has read Q
    uint64_t* k_full = bars + 2;                 // [KSTAGES]
    uint64_t* k_empty = k_full + KSTAGES;        // [KSTAGES]
    uint64_t* v_full = k_empty + KSTAGES;        // [VSTAGES]
    uint64_t* v_empty = v_full + VSTAGES;        // [VSTAGES]
    uint64_t* s_full = v_empty + VSTAGES;        // [2] per query tile
    uint64_t* p_part = s_full + 2;               // [2][PV_PARTS - 1] P columns of the first parts written
    uint64_t* p_full = p_part + 2 * (PV_PARTS - 1);  // [2]
    uint64_t* o_final = p_full + 2;              // [2]
    uint64_t* s_read = o_final + 2;              // [2] the softmax has read S_t (its upper key half may be rewritten)
    uint64_t* drain = s_read + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int nk = (p.Lk + 127) / 128;
    // unit u -> (query block, head, batch), query blocks fastest
    auto coords = [&](int u, int& q0, int& h, int& b) {
        q0 = (u % p.nqb) * 256;
        const int r = u / p.nqb;
        h = r % p.heads;
        b = r / p.heads;
    };

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int s = 0; s < KSTAGES; ++s) {
            mbar_init(k_full + s, 1);
            mbar_init(k_empty + s, 1);
        }
        for (int s = 0; s < VSTAGES; ++s) {
            mbar_init(v_full + s, 1);
            mbar_init(v_empty + s, 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(s_full + t, 1);
            for (int q = 0; q < PV_PARTS - 1; ++q) mbar_init(p_part + t * (PV_PARTS - 1) + q, 4);
            mbar_init(p_full + t, 4);
            mbar_init(o_final + t, 1);
            mbar_init(s_read + t, 4);
        }
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
    // producer: ring slots with a load issued and the phase it completes, and the
    // phase of the last Q load; MMA issuer: whether any MMA went out (both
    // drained after an abort, before exit)
    uint32_t karmed = 0, kpar = 0, varmed = 0, vpar = 0;
    int qpar = -1;
    bool issued = false;

    if (warp < 4) {
        regs_dealloc<REGS_CONTROL>();
    if (warp == 0) {
        if (lane == 0) {
            // ---------------- producer ----------------
            bool ok = true;
            int g = 0;  // key tiles loaded so far, over all units of this CTA
            for (int u = blockIdx.x, i = 0; ok && u < p.units; u += gridDim.x, ++i) {
            int q0, h, b;
            coords(u, q0, h, b);
            if (!mbar_wait(q_empty, (i & 1) ^ 1, abort_flag, p.wc)) { ok = false; break; }
            mbar_expect_tx(q_full, 2 * TILE_BYTES);
            for (int t = 0; t < 2; ++t) {
                tma_load_3d(smem + SQ + t * TILE_BYTES, &tmQ, q_full, h * 128, q0 + 128 * t, b);
                tma_load_3d(smem + SQ + t * TILE_BYTES + HALF_BYTES, &tmQ, q_full, h * 128 + 64, q0 + 128 * t, b);
            }
            qpar = i & 1;
            for (int j = 0; ok && j < nk; ++j, ++g) {
                const int ks = g % KSTAGES, vs = g % VSTAGES;
                const uint32_t kp = (g / KSTAGES) & 1, vp = (g / VSTAGES) & 1;
                if (!mbar_wait(k_empty + ks, kp ^ 1, abort_flag, p.wc)) { ok = false; break; }
                mbar_expect_tx(k_full + ks, TILE_BYTES);
                tma_load_3d(smem + SK + ks * TILE_BYTES, &tmK, k_full + ks, h * 128, j * 128, b);
                tma_load_3d(smem + SK + ks * TILE_BYTES + HALF_BYTES, &tmK, k_full + ks, h * 128 + 64, j * 128, b);
                karmed |= 1u << ks;
                kpar = (kpar & ~(1u << ks)) | (kp << ks);
                if (!mbar_wait(v_empty + vs, vp ^ 1, abort_flag, p.wc)) { ok = false; break; }
                mbar_expect_tx(v_full + vs, TILE_BYTES);
                tma_load_3d(smem + SV + vs * TILE_BYTES, &tmV, v_full + vs, h * 128, j * 128, b);
                tma_load_3d(smem + SV + vs * TILE_BYTES + HALF_BYTES, &tmV, v_full + vs, h * 128 + 64, j * 128, b);
                varmed |= 1u << vs;
                vpar = (vpar & ~(1u << vs)) | (vp << vs);
            }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        // The whole warp runs this loop (warp-uniform state); lane 0 waits on the
        // barriers, one elected lane issues each group of MMAs and its commits.
        // The issuing warp shares its SM sub-partition with two busy softmax
        // warps, so every instruction between MMAs is kept out of the loop:
        // descriptors are built once and moved by adding the offset (>> 4) to
        // their start-address field.
        constexpr uint32_t ID_QK = idesc_bf16(128, 128, false);
        constexpr uint32_t ID_QK64 = idesc_bf16(128, 64, false);
        constexpr uint32_t ID_PV = idesc_bf16(128, 128, true);
        const uint64_t dq = sdesc_kmajor_sw128(smem_u32(smem + SQ));
        const uint64_t dk = sdesc_kmajor_sw128(smem_u32(smem + SK));
        const uint64_t dv = sdesc_mnmajor_sw128(smem_u32(smem + SV), HALF_BYTES);
        auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
            int r = 1;
            if (lane == 0) r = mbar_wait(bar, parity, abort_flag, p.wc) ? 1 : 0;
            return __shfl_sync(0xffffffffu, r, 0) != 0;
        };
        // S_t(j) = Q_t K_j^T into TMEM columns [128 t, 128 t + 128); gj counts key
        // tiles over all units (ring slots and phases), the unit's last S also
        // releases Q for the next unit
        // part: S_ALL (all 128 keys; the unit's first key tile), S_HI (keys
        // 64..127 into columns 64..127, which P does not occupy: issued once the
        // softmax has read the previous S) or S_LO (keys 0..63 into columns
        // 0..63, after the P.V that reads P there; commits S_t)
        enum { S_ALL, S_HI, S_LO };
        auto issue_s = [&](int t, int gj, bool last, int part) -> bool {
            const int ks = gj % KSTAGES;
            if (t == 0 && part != S_LO && !wait(k_full + ks, (gj / KSTAGES) & 1)) return false;
            tc_fence_after();
            const uint64_t a = dq + (uint64_t)((t * TILE_BYTES) >> 4);
            const uint64_t b = dk + (uint64_t)((ks * TILE_BYTES + (part == S_HI ? 64 * 128 : 0)) >> 4);
            const uint32_t d = tmem + t * 128 + (part == S_HI ? 64 : 0);
            const uint32_t idesc = part == S_ALL ? ID_QK : ID_QK64;
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = ((kk >> 2) * HALF_BYTES + (kk & 3) * 32) >> 4;
                    umma_bf16_ss(d, a + off, b + off, idesc, kk != 0);
                }
                if (part != S_HI) {
                    umma_commit(s_full + t);
                    if (t == 1) umma_commit(k_empty + ks);
                    if (t == 1 && last) umma_commit(q_empty);
                }
            }
            __syncwarp();
            issued = true;
            return true;
        };
        // O_t += P_t(j) V_j, P_t read from the S_t columns (bf16 pairs), in
        // PV_PARTS parts over the keys, each issued as soon as the softmax has
        // stored its probabilities (p_part), the last after the whole row (p_full)
        // (j: the key tile inside the unit, gj: over all units)
        auto issue_pv = [&](int t, int gj, int j, int k0, int k1, uint64_t* bar) -> bool {
            const int vs = gj % VSTAGES;
            const bool last = k1 == 8;
            if (!wait(bar, gj & 1)) return false;
            if (t == 0 && k0 == 0 && !wait(v_full + vs, (gj / VSTAGES) & 1)) return false;
            tc_fence_after();
            const uint64_t b = dv + (uint64_t)((vs * TILE_BYTES) >> 4);
            const uint32_t acc0 = (j | k0) != 0;
            if (elect_one()) {
#pragma unroll
                for (int kk = k0; kk < k1; ++kk)
                    umma_bf16_ts(tmem + 256 + t * 128, tmem + t * 128 + kk * 8, b + ((kk * 2048) >> 4), ID_PV,
                                 kk == k0 ? acc0 : 1u);
                if (last) {
                    if (t == 1) umma_commit(v_empty + vs);
                    if (j == nk - 1) umma_commit(o_final + t);
                }
            }
            __syncwarp();
            return true;
        };
        auto issue_pv_all = [&](int t, int gj, int j) -> bool {
#pragma unroll
            for (int q = 0; q < PV_PARTS; ++q) {
                uint64_t* bar = q == PV_PARTS - 1 ? p_full + t : p_part + t * (PV_PARTS - 1) + q;
                if (!issue_pv(t, gj, j, q * 8 / PV_PARTS, (q + 1) * 8 / PV_PARTS, bar)) return false;
            }
            return true;
        };
        bool ok = true;
        int g = 0;  // first key tile of the unit, counted over all units
        for (int u = blockIdx.x, i = 0; ok && u < p.units; u += gridDim.x, ++i, g += nk) {
            ok = wait(q_full, i & 1) && issue_s(0, g, nk == 1, S_ALL) && issue_s(1, g, nk == 1, S_ALL);
            for (int j = 0; ok && j < nk; ++j) {
                const bool more = j + 1 < nk, last = j + 2 == nk;
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    // S_t(j + 1) for keys 64..127 as soon as the softmax has read S_t(j);
                    // keys 0..63 after P_t(j) V_j has read P_t(j) from those columns
                    if (more && !(wait(s_read + t, (g + j) & 1) && issue_s(t, g + j + 1, last, S_HI))) { ok = false; break; }
                    if (!issue_pv_all(t, g + j, j)) { ok = false; break; }
                    if (more && !issue_s(t, g + j + 1, last, S_LO)) { ok = false; break; }
                }
            }
        }
    }
    } else {
        regs_alloc<REGS_SOFTMAX>();
        // ---------------- softmax / output warps ----------------
        const int t = (warp - 4) >> 2;                   // query tile 0 or 1
        const int qq = warp & 3;                         // TMEM lane quarter
        const int r = qq * 32 + lane;                    // row inside the tile == TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>(qq * 32) << 16;
        const uint32_t TS = tmem + t * 128 + lane_off;   // S_t (and P_t)
        const uint32_t TO = tmem + 256 + t * 128 + lane_off;
        bool ok = true;
        int g = 0;  // first key tile of the unit, counted over all units
        for (int u = blockIdx.x, i = 0; ok && u < p.units; u += gridDim.x, ++i, g += nk) {
        int q0, h, b;
        coords(u, q0, h, b);
        // logits of this thread's query row in log2 units: S * scale_log2, times the
        // row's RMSNorm factor when the queries arrive unnormalised
        float row_scale = p.scale_log2;
        if (p.qn.ssq) {
            const int qrow = q0 + 128 * t + r;
            if (qrow < p.Lq) {
                const float* gs = p.qn.ssq + ((long long)b * p.Lq + qrow) * p.qn.ssq_ld;
                float ss = 0.f;
                for (int k = 0; k < p.qn.ngroups; ++k) ss += __ldg(gs + k);
                row_scale *= rsqrtf(ss * p.qn.inv_n + p.qn.eps);
            }
        }
        float m_run = -INFINITY, l_run = 0.0f;
        for (int j = 0; j < nk; ++j) {
            // all tcgen05.ld/st below are warp-collective: the warp's decisions stay uniform
            if (!__all_sync(0xffffffffu, mbar_wait(s_full + t, (g + j) & 1, abort_flag, p.wc))) { ok = false; break; }
            tc_fence_after();
            uint32_t sv[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(TS + c * 32, sv[c]);
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld_wait(sv[c]);
            {  // S_t(j) is in registers: the MMA may rewrite its upper key half
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(s_read + t);
            }

            const int valid = min(128, p.Lk - j * 128);
            if (valid < 128) {
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (c * 32 + i >= valid) sv[c][i] = __float_as_uint(-INFINITY);
            }
            // row maximum: eight independent 3-input max chains
            float mx[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const uint32_t* v = &sv[q >> 1][(q & 1) * 16];
                float a = fmaxf(__uint_as_float(v[0]), __uint_as_float(v[1]));
#pragma unroll
                for (int i = 2; i < 16; i += 2) a = max3f(a, __uint_as_float(v[i]), __uint_as_float(v[i + 1]));
                mx[q] = a;
            }
            const float m_tile =
                max3f(max3f(mx[0], mx[1], mx[2]), max3f(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) * row_scale;
            const float m_new = fmaxf(m_run, m_tile);
            const bool rescale = m_new > m_run + RESCALE_THRESHOLD;
            const float m_use = rescale ? m_new : m_run;
            // O_t is idle here (the commit of S_t(j) also covered P_t(j-1) V_{j-1}) and
            // must be rescaled before the first half of P_t(j) V_j is issued
            const float alpha = rescale ? ex2_approx(m_run - m_use) : 1.0f;  // 0 on the first tile
            if (j > 0 && __any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t ov[32];
                    tmem_ld32(TO + c * 32, ov);
                    tmem_ld_wait(ov);
#pragma unroll
                    for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
                    tmem_st32(TO + c * 32, ov);
                }
            }
            // probabilities on packed fp32 pairs, every exponential on the MUFU (scalar
            // FP32 work here would slow the MMA issue on the same sub-partitions);
            // each 32-column chunk is packed to bf16 and stored over its own S
            // columns (P_t = first 64 columns of S_t) at once
            uint64_t ps2[2] = {0ull, 0ull};
            const uint64_t scale2 = f2pack(row_scale, row_scale);
            const uint64_t negm2 = f2pack(-m_use, -m_use);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t pc[16];
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    const uint64_t x2 = fma2(f2pack(__uint_as_float(sv[c][i]), __uint_as_float(sv[c][i + 1])), scale2, negm2);
                    float x0, x1;
                    f2unpack(x2, x0, x1);
                    const float e0 = ex2_approx(x0), e1 = ex2_approx(x1);
                    ps2[(i >> 1) & 1] = add2(ps2[(i >> 1) & 1], f2pack(e0, e1));
                    pc[i / 2] = pack_bf16(e0, e1);
                }
                tmem_st16(TS + c * 16, pc);
                if (c < 3 && (c + 1) % (4 / PV_PARTS) == 0) {  // a part of P (and any O rescale) stored: its P.V may start
                    tmem_st_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(p_part + t * (PV_PARTS - 1) + (c + 1) / (4 / PV_PARTS) - 1);
                }
            }
            float ps[4];
            f2unpack(ps2[0], ps[0], ps[1]);
            f2unpack(ps2[1], ps[2], ps[3]);
            tmem_st_wait();
            if (rescale) {
                l_run *= alpha;
                m_run = m_use;
            }
            l_run += (ps[0] + ps[1]) + (ps[2] + ps[3]);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full + t);
        }
        if (!ok) break;
        // the unit's output: O_t / l once the last P.V of the unit has landed
        if (!__all_sync(0xffffffffu, mbar_wait(o_final + t, i & 1, abort_flag, p.wc))) { ok = false; break; }
        {
            tc_fence_after();
            const float inv = 1.0f / l_run;
            const int row = q0 + 128 * t + r;
            __nv_bfloat16* orow = p.o + ((long long)b * p.Lq + row) * p.ldo + h * 128;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t ov[32];
                tmem_ld32(TO + c * 32, ov);
                tmem_ld_wait(ov);
                if (row < p.Lq) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        dst[w] = make_uint4(pack_bf16(__uint_as_float(ov[8 * w]) * inv, __uint_as_float(ov[8 * w + 1]) * inv),
                                            pack_bf16(__uint_as_float(ov[8 * w + 2]) * inv, __uint_as_float(ov[8 * w + 3]) * inv),
                                            pack_bf16(__uint_as_float(ov[8 * w + 4]) * inv, __uint_as_float(ov[8 * w + 5]) * inv),
                                            pack_bf16(__uint_as_float(ov[8 * w + 6]) * inv, __uint_as_float(ov[8 * w + 7]) * inv));
                    }
                }
            }
        }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        // a wait gave up somewhere in the CTA: let this CTA's own loads and MMAs
        // land (bounded) before its shared and tensor memory are released
        if (warp == 0 && lane == 0) {
            if (qpar >= 0) mbar_drain(q_full, static_cast<uint32_t>(qpar), 200000000ull);
            for (int s = 0; s < KSTAGES; ++s)
                if (karmed & (1u << s)) mbar_drain(k_full + s, (kpar >> s) & 1, 200000000ull);
            for (int s = 0; s < VSTAGES; ++s)
                if (varmed & (1u << s)) mbar_drain(v_full + s, (vpar >> s) & 1, 200000000ull);
        } else if (warp == 1 && issued) {
            if (elect_one()) {  // the lane that issued the MMAs
                umma_commit(drain);
                mbar_drain(drain, 0, 200000000ull);
            }
            __syncwarp();
        }
    }
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ============================================================================
// Self-attention on SM pairs (tcgen05 .cta_group::2), P in shared memory.
//
// A cluster of two CTAs takes 512 queries of one (head, batch): each CTA two
// 128-row query tiles of its own 256 queries, S0 | S1 | O0 | O1 in its own
// tensor memory.  The even CTA issues every MMA of the pair:
//   S_t = Q_t K_j^T   M = 256 (128 query rows per SM), N = 128 keys, each
//                     CTA holding 64 of the tile's keys (both head-dim halves);
//   O_t += P_t V_j    M = 256, N = 128 head dims, each CTA holding 64 head-dim
//                     columns of the V tile for all 128 keys;
// so a K or V tile crosses into shared memory once per pair, half per SM.
// P_t is written by the softmax into shared memory (K-major, 128-byte
// swizzle) instead of over S_t: S_t(j+1) is issued as soon as the softmax of
// both SMs has read S_t(j) into registers and runs on the tensor core while the
// probabilities of S_t(j) are computed; P_t(j) V_j follows once both SMs have
// stored P_t(j).  The issuer takes the tiles one after the other (S_0(j+1),
// P_0 V, S_1(j+1), P_1 V), which lets the two query tiles settle half a key
// step apart, so one tile's exponentials overlap the other's MMAs.  The
// softmax computes the probabilities of keys 0..63 before it waits for
// P_t(j-1) V_{j-1} to finish, then stores them over P_t(j-1) (and rescales O_t
// when the maximum has grown past the threshold).
// Warps: 0 TMA producer (each CTA, its own halves), 1 tensor-memory owner (each
// CTA) and MMA issuer (even CTA), 2..3 idle, 4..11 softmax of tiles 0 / 1.
// ============================================================================
namespace attn2 {
constexpr int Q_TILE = 128 * 128 * 2;  // 128 query rows x 128 head dims: two 64-dim swizzled halves
constexpr int Q_HALF = 128 * 128;
constexpr int K_SLOT = 64 * 128 * 2;   // this CTA's 64 keys x 128 head dims: two 64-dim halves
constexpr int K_HALF = 64 * 128;
constexpr int V_SLOT = 128 * 64 * 2;   // 128 keys x this CTA's 64 head dims
constexpr int P_TILE = 128 * 128 * 2;  // 128 query rows x 128 keys: two 64-key halves
constexpr int P_HALF = 128 * 128;
constexpr int KST = 3, VST = 3;        // K / V ring slots
constexpr int SQ = 0;
constexpr int SK = SQ + 2 * Q_TILE;
constexpr int SV = SK + KST * K_SLOT;
constexpr int SP = SV + VST * V_SLOT;
constexpr int SBAR = SP + 2 * P_TILE;
constexpr int SMEM_BYTES = SBAR + 256 + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
// loads of a ring of `slots` slots that went into slot s after n loads
__device__ __forceinline__ uint32_t loads_in(uint32_t n, int s, int slots) {
    return n / slots + (static_cast<uint32_t>(s) < n % slots ? 1u : 0u);
}
}  // namespace attn2

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(attn::THREADS, 1)
    attn_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
    using namespace attn2;
    using attn::REGS_CONTROL;
    using attn::REGS_SOFTMAX;
    using attn::RESCALE_THRESHOLD;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SBAR);
    uint64_t* q_full = bars;                // even CTA: both CTAs' Q tiles landed
    uint64_t* k_full = bars + 1;            // [KST] even CTA: both halves of a K tile landed
    uint64_t* k_empty = k_full + KST;       // [KST] both CTAs: S_1 has read the K tile
    uint64_t* v_full = k_empty + KST;       // [VST] even CTA
    uint64_t* v_empty = v_full + VST;       // [VST] both CTAs: P_1 V has read the V tile
    uint64_t* s_full = v_empty + VST;       // [2] both CTAs: S_t in tensor memory
    uint64_t* s_read = s_full + 2;          // [2] even CTA: both SMs' softmax has read S_t
    uint64_t* p_full = s_read + 2;          // [2] even CTA: both SMs have stored P_t
    uint64_t* p_empty = p_full + 2;         // [2] both CTAs: P_t V has read P_t (O_t idle)
    uint64_t* o_final = p_empty + 2;        // [2] both CTAs: the last P_t V landed
    uint64_t* drain = o_final + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile uint32_t* kv_loads = reinterpret_cast<volatile uint32_t*>(tmem_slot + 2);  // [2] K, V tiles loaded

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();  // 0: the CTA that issues the MMAs
    const bool leader = rank == 0;
    const int nk = (p.Lk + 127) / 128;
    const int unit = static_cast<int>(cluster_id_x());
    const int q0 = (unit % p.nqb) * 512 + static_cast<int>(rank) * 256;
    const int h = (unit / p.nqb) % p.heads;
    const int b = unit / p.nqb / p.heads;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < KST; ++s) {
            mbar_init(k_full + s, 1);
            mbar_init(k_empty + s, 1);
        }
        for (int s = 0; s < VST; ++s) {
            mbar_init(v_full + s, 1);
            mbar_init(v_empty + s, 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(s_full + t, 1);
            mbar_init(s_read + t, 8);  // the four softmax warps of tile t in each CTA
            mbar_init(p_full + t, 8);
            mbar_init(p_empty + t, 1);
            mbar_init(o_final + t, 1);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        kv_loads[0] = kv_loads[1] = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();  // barriers initialised and tensor memory allocated in both CTAs
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool issued = false;

    if (warp < 4) {
        regs_dealloc<REGS_CONTROL>();
    if (warp == 0) {
        if (lane == 0) {
            // ---------------- producer (both CTAs) ----------------
            const uint32_t qf0 = mapa_shared(smem_u32(q_full), 0);
            const uint32_t kf0 = mapa_shared(smem_u32(k_full), 0);
            const uint32_t vf0 = mapa_shared(smem_u32(v_full), 0);
            if (leader) mbar_expect_tx(q_full, 4 * Q_TILE);
            for (int t = 0; t < 2; ++t) {
                tma_load_3d_pair(smem + SQ + t * Q_TILE, &tmQ, qf0, h * 128, q0 + 128 * t, b);
                tma_load_3d_pair(smem + SQ + t * Q_TILE + Q_HALF, &tmQ, qf0, h * 128 + 64, q0 + 128 * t, b);
            }
            uint32_t nkl = 0, nvl = 0;
            bool ok = true;
            for (int j = 0; j < nk; ++j) {
                const int ks = j % KST, vs = j % VST;
                if (!mbar_wait(k_empty + ks, ((j / KST) & 1) ^ 1, abort_flag, p.wc)) { ok = false; break; }
                if (leader) mbar_expect_tx(k_full + ks, 2 * K_SLOT);
                const int key0 = j * 128 + static_cast<int>(rank) * 64;
                tma_load_3d_pair(smem + SK + ks * K_SLOT, &tmK, kf0 + 8u * ks, h * 128, key0, b);
                tma_load_3d_pair(smem + SK + ks * K_SLOT + K_HALF, &tmK, kf0 + 8u * ks, h * 128 + 64, key0, b);
                ++nkl;
                if (!mbar_wait(v_empty + vs, ((j / VST) & 1) ^ 1, abort_flag, p.wc)) { ok = false; break; }
                if (leader) mbar_expect_tx(v_full + vs, 2 * V_SLOT);
                tma_load_3d_pair(smem + SV + vs * V_SLOT, &tmV, vf0 + 8u * vs, h * 128 + static_cast<int>(rank) * 64,
                                 j * 128, b);
                ++nvl;
            }
            // the MMA commits that free this CTA's slots arrive here: wait for the
            // last of them so none lands after the CTA has exited
            for (int s = 0; ok && s < KST; ++s) {
                const uint32_t c = loads_in(nkl, s, KST);
                if (c) ok = mbar_wait(k_empty + s, (c - 1) & 1u, abort_flag, p.wc);
            }
            for (int s = 0; ok && s < VST; ++s) {
                const uint32_t c = loads_in(nvl, s, VST);
                if (c) ok = mbar_wait(v_empty + s, (c - 1) & 1u, abort_flag, p.wc);
            }
            kv_loads[0] = nkl;
            kv_loads[1] = nvl;
        }
    } else if (warp == 1 && leader) {
        // ---------------- MMA issuer (even CTA) ----------------
        // the whole warp runs the loop; lane 0 waits, one elected lane issues
        constexpr uint32_t ID_QK = idesc_bf16(256, 128, false);
        constexpr uint32_t ID_PV = idesc_bf16(256, 128, true);
        const uint64_t dq = sdesc_kmajor_sw128(smem_u32(smem + SQ));
        const uint64_t dk = sdesc_kmajor_sw128(smem_u32(smem + SK));
        const uint64_t dv = sdesc_mnmajor_sw128(smem_u32(smem + SV), V_SLOT);  // one 64-column block per CTA
        const uint64_t dp = sdesc_kmajor_sw128(smem_u32(smem + SP));
        // the issuing thread spins on its barriers: a suspended wait woke up to ~1 us
        // after the phase completed, and every such delay is a tensor-core bubble
        auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
            int r = 1;
            if (lane == 0) r = mbar_spin(bar, parity, abort_flag, p.wc) ? 1 : 0;
            return __shfl_sync(0xffffffffu, r, 0) != 0;
        };
        // S_t(j) into tensor-memory columns [128 t, 128 t + 128) of both SMs
        auto issue_s = [&](int t, int j) -> bool {
            const int ks = j % KST;
            if (t == 0 && !wait(k_full + ks, (j / KST) & 1)) return false;
            tc_fence_after();
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t a = dq + (uint64_t)((t * Q_TILE + (kk >> 2) * Q_HALF + (kk & 3) * 32) >> 4);
                    const uint64_t bd = dk + (uint64_t)((ks * K_SLOT + (kk >> 2) * K_HALF + (kk & 3) * 32) >> 4);
                    umma_bf16_ss_pair(tmem + t * 128, a, bd, ID_QK, kk != 0);
                }
                umma_commit_pair_mc(s_full + t, 0x3);
                if (t == 1) umma_commit_pair_mc(k_empty + ks, 0x3);
            }
            __syncwarp();
            issued = true;
            return true;
        };
        // O_t += P_t(j) V_j once both SMs have stored P_t(j)
        auto issue_pv = [&](int t, int j) -> bool {
            const int vs = j % VST;
            if (!wait(p_full + t, j & 1)) return false;
            if (t == 0 && !wait(v_full + vs, (j / VST) & 1)) return false;
            tc_fence_after();
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t a = dp + (uint64_t)((t * P_TILE + (kk >> 2) * P_HALF + (kk & 3) * 32) >> 4);
                    const uint64_t bd = dv + (uint64_t)((vs * V_SLOT + kk * 2048) >> 4);
                    umma_bf16_ss_pair(tmem + 256 + t * 128, a, bd, ID_PV, (j | kk) != 0);
                }
                if (t == 1) umma_commit_pair_mc(v_empty + vs, 0x3);
                umma_commit_pair_mc(j + 1 < nk ? p_empty + t : o_final + t, 0x3);
            }
            __syncwarp();
            return true;
        };
        // per key tile, tile by tile: the next S as soon as the softmax has read the
        // current one, then P.V; the two query tiles settle half a step apart, so
        // one tile's exponentials overlap the other's MMAs
        bool ok = wait(q_full, 0) && issue_s(0, 0) && issue_s(1, 0);
        for (int j = 0; ok && j < nk; ++j) {
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                if (j + 1 < nk) ok = ok && wait(s_read + t, j & 1) && issue_s(t, j + 1);
                ok = ok && issue_pv(t, j);
            }
        }
    }
    } else {
        regs_alloc<REGS_SOFTMAX>();
        // ---------------- softmax / output warps (both CTAs) ----------------
        const int t = (warp - 4) >> 2;                  // query tile 0 or 1
        const int qq = warp & 3;                        // TMEM lane quarter
        const int r = qq * 32 + lane;                   // row inside the tile == TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>(qq * 32) << 16;
        const uint32_t TS = tmem + t * 128 + lane_off;
        const uint32_t TO = tmem + 256 + t * 128 + lane_off;
        const uint32_t prow = smem_u32(smem + SP + t * P_TILE + r * 128);  // row of P_t (128-byte swizzle: chunk ^ (r & 7))
        const int r7 = r & 7;
        const uint32_t s_read0 = mapa_shared(smem_u32(s_read + t), 0);
        const uint32_t p_full0 = mapa_shared(smem_u32(p_full + t), 0);
        float row_scale = p.scale_log2;
        if (p.qn.ssq) {
            const int qrow = q0 + 128 * t + r;
            if (qrow < p.Lq) {
                const float* gs = p.qn.ssq + ((long long)b * p.Lq + qrow) * p.qn.ssq_ld;
                float ss = 0.f;
                for (int k = 0; k < p.qn.ngroups; ++k) ss += __ldg(gs + k);
                row_scale *= rsqrtf(ss * p.qn.inv_n + p.qn.eps);
            }
        }
        float m_run = -INFINITY, l_run = 0.0f;
        bool ok = true;
        for (int j = 0; j < nk; ++j) {
            // tcgen05.ld/st are warp-collective: the warp's decisions stay uniform
            if (!__all_sync(0xffffffffu, mbar_wait(s_full + t, j & 1, abort_flag, p.wc))) { ok = false; break; }
            tc_fence_after();
            uint32_t sv[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(TS + c * 32, sv[c]);
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld_wait(sv[c]);
            // S_t(j) is in registers: the next S may overwrite its columns
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(s_read0);
            const int valid = min(128, p.Lk - j * 128);
            if (valid < 128) {
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (c * 32 + i >= valid) sv[c][i] = __float_as_uint(-INFINITY);
            }
            float mx[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const uint32_t* v = &sv[q >> 1][(q & 1) * 16];
                float a = fmaxf(__uint_as_float(v[0]), __uint_as_float(v[1]));
#pragma unroll
                for (int i = 2; i < 16; i += 2) a = max3f(a, __uint_as_float(v[i]), __uint_as_float(v[i + 1]));
                mx[q] = a;
            }
            const float m_tile =
                max3f(max3f(mx[0], mx[1], mx[2]), max3f(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) * row_scale;
            const float m_new = fmaxf(m_run, m_tile);
            const bool rescale = m_new > m_run + RESCALE_THRESHOLD;
            const float m_use = rescale ? m_new : m_run;
            const float alpha = rescale ? ex2_approx(m_run - m_use) : 1.0f;  // 0 on the first tile
            // probabilities on packed fp32 pairs, every exponential on the MUFU, packed
            // to bf16; keys 0..63 are computed while P_t(j-1) V_{j-1} may still be
            // reading P_t, each 32-key chunk stored as four 16-byte pieces of the row
            uint64_t ps2[2] = {0ull, 0ull};
            const uint64_t scale2 = f2pack(row_scale, row_scale);
            const uint64_t negm2 = f2pack(-m_use, -m_use);
            uint32_t pc[2][16];
            auto p_chunk = [&](int c, uint32_t (&out)[16]) {
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    const uint64_t x2 = fma2(f2pack(__uint_as_float(sv[c][i]), __uint_as_float(sv[c][i + 1])), scale2, negm2);
                    float x0, x1;
                    f2unpack(x2, x0, x1);
                    const float e0 = ex2_approx(x0), e1 = ex2_approx(x1);
                    ps2[(i >> 1) & 1] = add2(ps2[(i >> 1) & 1], f2pack(e0, e1));
                    out[i / 2] = pack_bf16(e0, e1);
                }
            };
            auto p_store = [&](int c, const uint32_t (&in)[16]) {
                const uint32_t half = prow + (c >> 1) * P_HALF;
#pragma unroll
                for (int w = 0; w < 4; ++w)
                    st_shared_v4(half + ((((c & 1) * 4 + w) ^ r7) << 4), in[4 * w], in[4 * w + 1], in[4 * w + 2],
                                 in[4 * w + 3]);
            };
            p_chunk(0, pc[0]);
            p_chunk(1, pc[1]);
            if (j > 0) {
                // P_t(j-1) V_{j-1} done: P_t may be overwritten and O_t is idle
                if (!__all_sync(0xffffffffu, mbar_wait(p_empty + t, (j - 1) & 1, abort_flag, p.wc))) { ok = false; break; }
                tc_fence_after();
                if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
                    for (int c = 0; c < 4; ++c) {
                        uint32_t ov[32];
                        tmem_ld32(TO + c * 32, ov);
                        tmem_ld_wait(ov);
#pragma unroll
                        for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
                        tmem_st32(TO + c * 32, ov);
                    }
                    tmem_st_wait();
                }
            }
            p_store(0, pc[0]);
            p_store(1, pc[1]);
            p_chunk(2, pc[0]);
            p_store(2, pc[0]);
            p_chunk(3, pc[1]);
            p_store(3, pc[1]);
            // P_t(j) (written through the generic proxy) goes to the tensor core
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(p_full0);
            float ps[4];
            f2unpack(ps2[0], ps[0], ps[1]);
            f2unpack(ps2[1], ps[2], ps[3]);
            if (rescale) {
                l_run *= alpha;
                m_run = m_use;
            }
            l_run += (ps[0] + ps[1]) + (ps[2] + ps[3]);
        }
        // the output: O_t / l once the last P_t V has landed
        if (ok && __all_sync(0xffffffffu, mbar_wait(o_final + t, 0, abort_flag, p.wc))) {
            tc_fence_after();
            const float inv = 1.0f / l_run;
            const int row = q0 + 128 * t + r;
            __nv_bfloat16* orow = p.o + ((long long)b * p.Lq + row) * p.ldo + h * 128;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t ov[32];
                tmem_ld32(TO + c * 32, ov);
                tmem_ld_wait(ov);
                if (row < p.Lq) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        dst[w] = make_uint4(pack_bf16(__uint_as_float(ov[8 * w]) * inv, __uint_as_float(ov[8 * w + 1]) * inv),
                                            pack_bf16(__uint_as_float(ov[8 * w + 2]) * inv, __uint_as_float(ov[8 * w + 3]) * inv),
                                            pack_bf16(__uint_as_float(ov[8 * w + 4]) * inv, __uint_as_float(ov[8 * w + 5]) * inv),
                                            pack_bf16(__uint_as_float(ov[8 * w + 6]) * inv, __uint_as_float(ov[8 * w + 7]) * inv));
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // neither CTA issues another load, MMA or arrival
    const bool any_abort =
        *abort_flag != 0 || ld_shared_cluster_u32(mapa_shared(smem_u32((const void*)abort_flag), rank ^ 1u)) != 0;
    if (any_abort && leader) {
        // let the pair's loads and MMAs land (bounded) before shared and tensor
        // memory are released.  Both CTAs always issue their Q loads.  Per ring
        // slot the two producers' load counts differ by at most one (both wait
        // for the same multicast releases): where the odd CTA stopped first its
        // bytes are counted as delivered, where the even CTA did, the arrival it
        // owed is made for the odd CTA's bytes alone
        if (warp == 0 && lane == 0) {
            mbar_drain(q_full, 0, 200000000ull);
            const uint32_t nk1 = ld_shared_cluster_u32(mapa_shared(smem_u32((const void*)kv_loads), 1));
            const uint32_t nv1 = ld_shared_cluster_u32(mapa_shared(smem_u32((const void*)(kv_loads + 1)), 1));
            auto drain_ring = [&](uint64_t* full, int slots, uint32_t bytes, uint32_t n0, uint32_t n1) {
                for (int s = 0; s < slots; ++s) {
                    const uint32_t c0 = loads_in(n0, s, slots), c1 = loads_in(n1, s, slots);
                    const uint32_t c = c0 > c1 ? c0 : c1;
                    if (!c) continue;
                    if (c0 > c1) mbar_complete_tx(full + s, bytes);
                    if (c1 > c0) mbar_expect_tx(full + s, bytes);
                    mbar_drain(full + s, (c - 1) & 1u, 200000000ull);
                }
            };
            drain_ring(k_full, KST, K_SLOT, kv_loads[0], nk1);
            drain_ring(v_full, VST, V_SLOT, kv_loads[1], nv1);
        } else if (warp == 1 && issued) {
            if (elect_one()) {  // the lane that issued the MMAs
                umma_commit_pair(drain);
                mbar_drain(drain, 0, 200000000ull);
            }
            __syncwarp();
        }
    }
    __syncthreads();
    cluster_sync_all();  // the pair's loads and MMAs have landed
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc_pair(tmem, 512);
    }
}

cudaError_t init_gemm_attributes();

cudaError_t init_kernel_attributes() {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, attn::SMEM_BYTES);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(attn_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, attn2::SMEM_BYTES);
    if (e == cudaSuccess) e = init_gemm_attributes();
    if (e == cudaSuccess) e = init_conv_attributes();
    if (e == cudaSuccess) e = init_layernorm_attributes();
    return e;
}

cudaError_t launch_attention(const void* q, long long ldq, const void* k, long long ldk, const void* v,
                             long long ldv, void* o, long long ldo, int B, int heads, int Lq, int Lk,
                             const LaunchCtx& ctx, const RowNorm& qn) {
    if (B <= 0 || Lq <= 0) return cudaSuccess;
    if (Lk <= 0 || heads <= 0 || ldq % 8 || ldk % 8 || ldv % 8 || ldo % 8) return cudaErrorInvalidValue;
    if (qn.ssq && (qn.ngroups <= 0 || qn.ssq_ld < qn.ngroups || !(qn.inv_n > 0.f))) return cudaErrorInvalidValue;
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
    p.nqb = (Lq + 255) / 256;
    p.units = p.nqb * heads * B;
    p.o = reinterpret_cast<__nv_bfloat16*>(o);
    p.ldo = ldo;
    p.scale_log2 = 1.4426950408889634f / sqrtf(128.0f);
    p.qn = qn;
    p.wc.err = ctx.err;
    p.wc.limit_ns = ctx.wait_limit_ns;
    // up to 4 key tiles (the text tokens of the cross-attention): one CTA per SM
    // walks 256-query units, the next S in two key halves; longer key sets (the
    // self-attention): SM pairs, 512 queries per cluster, P in shared memory
    const int nk = (Lk + 127) / 128;
    if (nk <= 4) {
        const int grid = p.units > ctx.num_sms ? ctx.num_sms : p.units;
        attn_tc_kernel<<<grid, attn::THREADS, attn::SMEM_BYTES, ctx.stream>>>(tq, tk, tv, p);
    } else {
        // each CTA of a pair loads 64-key halves of the K tiles
        CUtensorMap tk64;
        if (!make_tmap_3d(&tk64, k, width, Lk, B, ldk, (uint64_t)ldk * Lk, 64, 64)) return cudaErrorInvalidValue;
        p.nqb = (Lq + 511) / 512;
        p.units = p.nqb * heads * B;
        attn_pair_kernel<<<2 * p.units, attn::THREADS, attn2::SMEM_BYTES, ctx.stream>>>(tq, tk64, tv, p);
    }
    if (ctx.launches) ++*ctx.launches;
    return cudaGetLastError();
}

}  // namespace wan

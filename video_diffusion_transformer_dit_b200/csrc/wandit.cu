// libwandit host side: the C ABI of include/wandit.h and include/wandit_ops.h.
//
// A handle owns the repacked weights (one device allocation), a workspace sized
// at create from max_batch / max_tokens / max_text, a device error word and a
// cache of per-shape launch plans (RoPE tables + a captured CUDA graph).  The
// forward is the diffusers WanTransformer3DModel forward (pswp.cn notes on
// WanPipeline, sections "WanTransformer3DModel" and "WanTransformerBlock")
// expressed as launches of the sm_100a kernels in this directory.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <set>
#include <string>
#include <tuple>
#include <vector>

#include "../../include/wandit.h"
#include "../../include/wandit_ops.h"
#include "../../include/wanvae.h"
#include "kernels.h"

using wan::EpiParams;
using wan::LaunchCtx;

namespace {

constexpr uint64_t kDefaultWaitNs = 2000000000ull;

struct Slot {                  // where a named parameter lands
    void* dst;                 // device destination (inside the weight arena)
    int dst_dtype;             // WAN_DTYPE_*
    std::vector<int64_t> shape;
    long long numel;
};

struct BlockW {
    void *wqkv, *wo, *wq2, *wo2, *w1, *w2;          // bf16
    float *bqkv, *bo, *bq2, *bo2, *b1, *b2;         // f32 biases
    float *qk_gain;                                 // [2D]: norm_q | norm_k of attn1
    float *q2_gain;                                 // [D]: attn2.norm_q
    float *n2_g, *n2_b;                             // norm2 affine
    float *sst;                                     // [6D]
};

// CUDA-event pairs around every launch of one forward, tagged by kernel class.
struct KTimer {
    std::vector<cudaEvent_t> ev;
    std::vector<int> cls;
    int n = 0;
    cudaError_t ensure(int pairs) {
        while ((int)ev.size() < 2 * pairs) {
            cudaEvent_t e;
            cudaError_t r = cudaEventCreate(&e);
            if (r != cudaSuccess) return r;
            ev.push_back(e);
        }
        return cudaSuccess;
    }
    // External records become event nodes when the forward is captured into a graph.
    void begin(cudaStream_t s) { cudaEventRecordWithFlags(ev[2 * n], s, cudaEventRecordExternal); }
    void end(cudaStream_t s, int kc) {
        cudaEventRecordWithFlags(ev[2 * n + 1], s, cudaEventRecordExternal);
        if ((int)cls.size() <= n) cls.push_back(kc); else cls[n] = kc;
        ++n;
    }
    void destroy() {
        for (auto e : ev) cudaEventDestroy(e);
        ev.clear();
    }
};

struct Plan {
    cudaGraphExec_t exec = nullptr;         // plain replay
    cudaGraphExec_t exec_timed = nullptr;   // replay with the event pairs
    int launches = 0;
    float2* rope = nullptr;     // device tables: t | h | w
    wan::RopeTables rt{};
    KTimer timer;
    int timed_pairs = 0;        // pairs recorded by the most recent timed forward
};

using PlanKey = std::tuple<int, int, int, int, int, int, int, int, int, int, int, int>;

}  // namespace

struct wan_dit {
    wan_dit_config cfg{};
    int device = 0;
    int num_sms = 148;
    std::string err;
    // weights
    char* arena = nullptr;
    size_t arena_bytes = 0;
    std::map<std::string, Slot> slots;
    std::set<std::string> loaded;
    std::vector<BlockW> blocks;
    void *w_pe, *w_t1, *w_t2, *w_tp, *w_x1, *w_x2, *w_kv, *w_po;
    float *b_pe, *b_t1, *b_t2, *b_tp, *b_x1, *b_x2, *b_kv, *k2_gain, *sst_out, *b_po;
    int Kp = 0;           // patch GEMM K: 4 * in_ch rounded up to the 64-wide K tile
    void* w_pe_k;         // [D, Kp] patch weights as the GEMM reads them (== w_pe when Kp == 4 * in_ch)
    // image branch (image_dim > 0): embedder, all blocks' image K/V projections and key gains
    void *w_i1 = nullptr, *w_i2 = nullptr, *w_kvi = nullptr;
    float *b_i1 = nullptr, *b_i2 = nullptr, *b_kvi = nullptr, *ki_gain = nullptr;
    float* sst_all;       // [N, 6, D] block tables, contiguous
    // workspace
    char* ws = nullptr;
    size_t ws_bytes = 0;
    float* lat_stage;     // [R * in_ch * 4] f32 (or bf16 values)
    void* ctx_stage;      // bf16 [B * Lc, text_dim]
    float* t_stage;       // f32 [R]
    float* vel_stage;     // f32 [R * out_ch * 4]
    void *X, *x, *y, *qkv, *o, *qc, *u, *th, *ctx, *kv, *tsin, *tsilu;
    void *img_stage = nullptr, *ih = nullptr, *ictx = nullptr, *kvi = nullptr, *o2 = nullptr;  // image branch
    float *temb, *tproj, *th32;
    float* modc;          // [N, max_batch, 6, D] per-sample modulation of every block
    float* sched;         // {guidance, sigma_next - sigma} of the fused sampler step
    float* ssq;           // [R, 3 * heads] per-head sums of squares: self q | self k | cross q
    int* d_err = nullptr;
    // options / state
    bool use_graph = true;
    uint64_t wait_ns = kDefaultWaitNs;
    void* dump = nullptr;
    int last_launches = 0;
    cudaStream_t cap_stream = nullptr;
    std::map<PlanKey, Plan> plans;
    bool timing = false;
    bool gemm_pair = true;
    Plan* last_plan = nullptr;
    bool last_timed = false;
    // sequence-parallel forward in progress (between wan_dit_sp_begin and wan_dit_sp_end)
    bool sp_active = false;
    int sp_B = 0, sp_F = 0, sp_Hz = 0, sp_Wz = 0, sp_Lc = 0, sp_per_token = 0, sp_dtype = 0;
    int sp_rank = 0, sp_world = 0, sp_Ls = 0;
    // whole latent in and whole velocity out of a sequence-parallel forward (the
    // workspace holds only the shard's tokens); allocated by the first sp_begin of a size
    void* sp_lat = nullptr;
    size_t sp_lat_bytes = 0;
    float* sp_vel = nullptr;
    size_t sp_vel_bytes = 0;
    int sp_next_block = 0;
    int sp_phase = 0;     // 0: next call is sp_block_qkv, 1: sp_block_finish
};

namespace {

wan_status fail(wan_dit* h, wan_status s, const std::string& msg) {
    if (h) h->err = msg;
    return s;
}

wan_status cuda_fail(wan_dit* h, cudaError_t e, const char* what) {
    return fail(h, WAN_ECUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

#define WAN_CU(call, what)                          \
    do {                                            \
        cudaError_t e_ = (call);                    \
        if (e_ != cudaSuccess) return cuda_fail(h, e_, what); \
    } while (0)

#define WAN_CU_RET(call)                  \
    do {                                  \
        wan_status s_ = (call);           \
        if (s_ != WAN_OK) return s_;      \
    } while (0)

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ------------------------------------------------------------------ weight layout
bool valid_config(const wan_dit_config& c, std::string& why) {
    auto bad = [&](const char* m) { why = m; return false; };
    if (c.head_dim != 128) return bad("head_dim must be 128");
    if (c.dim <= 0 || c.dim % 256 != 0 || c.dim / 256 > 24) return bad("dim must be a multiple of 256 up to 6144");
    if (c.heads * c.head_dim != c.dim) return bad("heads * head_dim must equal dim");
    if (c.ffn_dim <= 0 || c.ffn_dim % 64) return bad("ffn_dim must be a positive multiple of 64");
    if (c.num_blocks <= 0) return bad("num_blocks must be positive");
    if (c.patch_t != 1 || c.patch_h != 2 || c.patch_w != 2) return bad("only patch (1,2,2) is supported");
    if (c.in_ch <= 0 || c.in_ch > 1024) return bad("in_ch must be 1..1024");
    if (c.out_ch <= 0 || (c.out_ch * 4) % 64) return bad("out_ch * 4 must be a multiple of 64");
    if (c.text_dim <= 0 || c.text_dim % 64) return bad("text_dim must be a positive multiple of 64");
    if (c.freq_dim <= 0 || c.freq_dim % 16) return bad("freq_dim must be a positive multiple of 16");
    if (c.rope_t % 2 || c.rope_h % 2 || c.rope_w % 2 || c.rope_t + c.rope_h + c.rope_w != c.head_dim)
        return bad("rope split must be even and sum to head_dim");
    if (!(c.eps > 0.f) || !(c.rope_theta > 0.f)) return bad("eps and rope_theta must be positive");
    if (c.max_batch <= 0 || c.max_batch > 8 || c.max_tokens <= 0 || c.max_text <= 0)
        return bad("max_batch must be 1..8; max_tokens, max_text positive");
    if (c.image_dim < 0 || c.image_dim % 64) return bad("image_dim must be 0 or a positive multiple of 64");
    if (c.image_dim > 0 && c.max_image <= 0) return bad("max_image must be positive with an image branch");
    return true;
}

void add_slot(wan_dit* h, const std::string& name, void* dst, int dt, std::vector<int64_t> shape) {
    long long n = 1;
    for (auto d : shape) n *= d;
    h->slots[name] = Slot{dst, dt, std::move(shape), n};
}

wan_status build_weights(wan_dit* h) {
    const auto& c = h->cfg;
    const long long D = c.dim, Fd = c.ffn_dim, N = c.num_blocks, P_in = c.in_ch * 4, P_out = c.out_ch * 4;
    const long long Kp = (P_in + 63) / 64 * 64, Di = c.image_dim;
    h->Kp = (int)Kp;
    // sizes in bytes
    size_t total = 0;
    auto sz = [&](long long n, int dt) { size_t b = align_up(n * (dt == WAN_DTYPE_BF16 ? 2 : 4), 256); total += b; return b; };
    sz(D * P_in, 1); sz(D, 0);
    if (Kp != P_in) sz(D * Kp, 1);
    if (Di > 0) {
        sz(D * Di, 1); sz(D, 0); sz(D * D, 1); sz(D, 0); sz(N * 2 * D * D, 1); sz(N * 2 * D, 0); sz(N * D, 0);
    }
    sz(D * c.freq_dim, 1); sz(D, 0); sz(D * D, 1); sz(D, 0); sz(6 * D * D, 1); sz(6 * D, 0);
    sz(D * c.text_dim, 1); sz(D, 0); sz(D * D, 1); sz(D, 0);
    sz(N * 2 * D * D, 1); sz(N * 2 * D, 0); sz(N * D, 0); sz(N * 6 * D, 0);
    for (int i = 0; i < N; ++i) {
        sz(3 * D * D, 1); sz(3 * D, 0); sz(D * D, 1); sz(D, 0); sz(D * D, 1); sz(D, 0); sz(D * D, 1); sz(D, 0);
        sz(Fd * D, 1); sz(Fd, 0); sz(D * Fd, 1); sz(D, 0); sz(2 * D, 0); sz(D, 0); sz(D, 0); sz(D, 0);
    }
    sz(2 * D, 0); sz(P_out * D, 1); sz(P_out, 0);
    h->arena_bytes = total;
    if (cudaMalloc(&h->arena, total) != cudaSuccess) {
        cudaGetLastError();
        return fail(h, WAN_ENOMEM, "cannot allocate " + std::to_string(total) + " bytes of weights");
    }
    cudaMemset(h->arena, 0, total);
    size_t off = 0;
    auto take = [&](long long n, int dt) {
        void* p = h->arena + off;
        off += align_up(n * (dt == WAN_DTYPE_BF16 ? 2 : 4), 256);
        return p;
    };
    h->w_pe = take(D * P_in, 1);
    h->b_pe = (float*)take(D, 0);
    add_slot(h, "patch_embedding.weight", h->w_pe, 1, {D, c.in_ch, c.patch_t, c.patch_h, c.patch_w});
    add_slot(h, "patch_embedding.bias", h->b_pe, 0, {D});
    h->w_pe_k = Kp != P_in ? take(D * Kp, 1) : h->w_pe;  // zero pad columns (arena is zeroed)
    const std::string ce = "condition_embedder.";
    h->w_t1 = take(D * c.freq_dim, 1); h->b_t1 = (float*)take(D, 0);
    h->w_t2 = take(D * D, 1); h->b_t2 = (float*)take(D, 0);
    h->w_tp = take(6 * D * D, 1); h->b_tp = (float*)take(6 * D, 0);
    add_slot(h, ce + "time_embedder.linear_1.weight", h->w_t1, 1, {D, c.freq_dim});
    add_slot(h, ce + "time_embedder.linear_1.bias", h->b_t1, 0, {D});
    add_slot(h, ce + "time_embedder.linear_2.weight", h->w_t2, 1, {D, D});
    add_slot(h, ce + "time_embedder.linear_2.bias", h->b_t2, 0, {D});
    add_slot(h, ce + "time_proj.weight", h->w_tp, 1, {6 * D, D});
    add_slot(h, ce + "time_proj.bias", h->b_tp, 0, {6 * D});
    h->w_x1 = take(D * c.text_dim, 1); h->b_x1 = (float*)take(D, 0);
    h->w_x2 = take(D * D, 1); h->b_x2 = (float*)take(D, 0);
    add_slot(h, ce + "text_embedder.linear_1.weight", h->w_x1, 1, {D, c.text_dim});
    add_slot(h, ce + "text_embedder.linear_1.bias", h->b_x1, 0, {D});
    add_slot(h, ce + "text_embedder.linear_2.weight", h->w_x2, 1, {D, D});
    add_slot(h, ce + "text_embedder.linear_2.bias", h->b_x2, 0, {D});
    // cross-attention keys/values of every block, one [N * 2D, D] matrix
    h->w_kv = take(N * 2 * D * D, 1);
    h->b_kv = (float*)take(N * 2 * D, 0);
    h->k2_gain = (float*)take(N * D, 0);
    h->sst_all = (float*)take(N * 6 * D, 0);
    if (Di > 0) {
        h->w_i1 = take(D * Di, 1); h->b_i1 = (float*)take(D, 0);
        h->w_i2 = take(D * D, 1); h->b_i2 = (float*)take(D, 0);
        h->w_kvi = take(N * 2 * D * D, 1);
        h->b_kvi = (float*)take(N * 2 * D, 0);
        h->ki_gain = (float*)take(N * D, 0);
        add_slot(h, ce + "image_embedder.linear_1.weight", h->w_i1, 1, {D, Di});
        add_slot(h, ce + "image_embedder.linear_1.bias", h->b_i1, 0, {D});
        add_slot(h, ce + "image_embedder.linear_2.weight", h->w_i2, 1, {D, D});
        add_slot(h, ce + "image_embedder.linear_2.bias", h->b_i2, 0, {D});
    }
    h->blocks.resize(N);
    for (int i = 0; i < N; ++i) {
        BlockW& b = h->blocks[i];
        const std::string p = "blocks." + std::to_string(i) + ".";
        b.wqkv = take(3 * D * D, 1); b.bqkv = (float*)take(3 * D, 0);
        b.wo = take(D * D, 1); b.bo = (float*)take(D, 0);
        b.wq2 = take(D * D, 1); b.bq2 = (float*)take(D, 0);
        b.wo2 = take(D * D, 1); b.bo2 = (float*)take(D, 0);
        b.w1 = take(Fd * D, 1); b.b1 = (float*)take(Fd, 0);
        b.w2 = take(D * Fd, 1); b.b2 = (float*)take(D, 0);
        b.qk_gain = (float*)take(2 * D, 0);
        b.q2_gain = (float*)take(D, 0);
        b.n2_g = (float*)take(D, 0);
        b.n2_b = (float*)take(D, 0);
        b.sst = h->sst_all + (long long)i * 6 * D;
        auto bf = [](void* base, long long elems) { return (void*)((char*)base + elems * 2); };
        auto f4 = [](float* base, long long elems) { return (void*)(base + elems); };
        add_slot(h, p + "scale_shift_table", b.sst, 0, {1, 6, D});
        add_slot(h, p + "attn1.to_q.weight", bf(b.wqkv, 0), 1, {D, D});
        add_slot(h, p + "attn1.to_k.weight", bf(b.wqkv, D * D), 1, {D, D});
        add_slot(h, p + "attn1.to_v.weight", bf(b.wqkv, 2 * D * D), 1, {D, D});
        add_slot(h, p + "attn1.to_q.bias", f4(b.bqkv, 0), 0, {D});
        add_slot(h, p + "attn1.to_k.bias", f4(b.bqkv, D), 0, {D});
        add_slot(h, p + "attn1.to_v.bias", f4(b.bqkv, 2 * D), 0, {D});
        add_slot(h, p + "attn1.to_out.0.weight", b.wo, 1, {D, D});
        add_slot(h, p + "attn1.to_out.0.bias", b.bo, 0, {D});
        add_slot(h, p + "attn1.norm_q.weight", f4(b.qk_gain, 0), 0, {D});
        add_slot(h, p + "attn1.norm_k.weight", f4(b.qk_gain, D), 0, {D});
        add_slot(h, p + "norm2.weight", b.n2_g, 0, {D});
        add_slot(h, p + "norm2.bias", b.n2_b, 0, {D});
        add_slot(h, p + "attn2.to_q.weight", b.wq2, 1, {D, D});
        add_slot(h, p + "attn2.to_q.bias", b.bq2, 0, {D});
        add_slot(h, p + "attn2.to_k.weight", bf(h->w_kv, (2LL * i) * D * D), 1, {D, D});
        add_slot(h, p + "attn2.to_v.weight", bf(h->w_kv, (2LL * i + 1) * D * D), 1, {D, D});
        add_slot(h, p + "attn2.to_k.bias", f4(h->b_kv, 2LL * i * D), 0, {D});
        add_slot(h, p + "attn2.to_v.bias", f4(h->b_kv, (2LL * i + 1) * D), 0, {D});
        add_slot(h, p + "attn2.to_out.0.weight", b.wo2, 1, {D, D});
        add_slot(h, p + "attn2.to_out.0.bias", b.bo2, 0, {D});
        add_slot(h, p + "attn2.norm_q.weight", b.q2_gain, 0, {D});
        add_slot(h, p + "attn2.norm_k.weight", f4(h->k2_gain, (long long)i * D), 0, {D});
        if (Di > 0) {  // image branch of attn2: K/V rows of all blocks in one matrix, like the text K/V
            add_slot(h, p + "attn2.add_k_proj.weight", bf(h->w_kvi, (2LL * i) * D * D), 1, {D, D});
            add_slot(h, p + "attn2.add_v_proj.weight", bf(h->w_kvi, (2LL * i + 1) * D * D), 1, {D, D});
            add_slot(h, p + "attn2.add_k_proj.bias", f4(h->b_kvi, 2LL * i * D), 0, {D});
            add_slot(h, p + "attn2.add_v_proj.bias", f4(h->b_kvi, (2LL * i + 1) * D), 0, {D});
            add_slot(h, p + "attn2.norm_added_k.weight", f4(h->ki_gain, (long long)i * D), 0, {D});
        }
        add_slot(h, p + "ffn.net.0.proj.weight", b.w1, 1, {Fd, D});
        add_slot(h, p + "ffn.net.0.proj.bias", b.b1, 0, {Fd});
        add_slot(h, p + "ffn.net.2.weight", b.w2, 1, {D, Fd});
        add_slot(h, p + "ffn.net.2.bias", b.b2, 0, {D});
    }
    h->sst_out = (float*)take(2 * D, 0);
    h->w_po = take(P_out * D, 1);
    h->b_po = (float*)take(P_out, 0);
    add_slot(h, "scale_shift_table", h->sst_out, 0, {1, 2, D});
    add_slot(h, "proj_out.weight", h->w_po, 1, {P_out, D});
    add_slot(h, "proj_out.bias", h->b_po, 0, {P_out});
    return WAN_OK;
}

wan_status build_workspace(wan_dit* h) {
    const auto& c = h->cfg;
    const long long R = (long long)c.max_batch * c.max_tokens;
    const long long Rc = (long long)c.max_batch * c.max_text;
    const long long D = c.dim, Fd = c.ffn_dim, N = c.num_blocks;
    const long long Pin = c.in_ch * 4, Pout = c.out_ch * 4, Kp = h->Kp;
    const long long Ri = c.image_dim > 0 ? (long long)c.max_batch * c.max_image : 0;
    struct Item { void** p; size_t bytes; };
    std::vector<Item> items = {
        {(void**)&h->lat_stage, (size_t)(R * Pin * 4)}, {&h->ctx_stage, (size_t)(Rc * c.text_dim * 2)},
        {(void**)&h->t_stage, (size_t)(R * 4)},        {(void**)&h->vel_stage, (size_t)(R * Pout * 4)},
        {&h->X, (size_t)(R * Kp * 2)},                 {&h->x, (size_t)(R * D * 2)},
        {&h->y, (size_t)(R * D * 2)},                  {&h->qkv, (size_t)(R * 3 * D * 2)},
        {&h->o, (size_t)(R * D * 2)},                  {&h->qc, (size_t)(R * D * 2)},
        {&h->u, (size_t)(R * Fd * 2)},                 {&h->th, (size_t)(Rc * D * 2)},
        {&h->ctx, (size_t)(Rc * D * 2)},               {&h->kv, (size_t)(Rc * N * 2 * D * 2)},
        {&h->tsin, (size_t)(R * c.freq_dim * 2)},      {&h->tsilu, (size_t)(R * D * 2)},
        {(void**)&h->temb, (size_t)(R * D * 4)},       {(void**)&h->tproj, (size_t)(R * 6 * D * 4)},
        {(void**)&h->th32, (size_t)(R * D * 4)},
        {(void**)&h->modc, (size_t)((long long)N * c.max_batch * 6 * D * 4)},
        {(void**)&h->sched, (size_t)64},
        {(void**)&h->ssq, (size_t)(R * 3 * c.heads * 4)},
    };
    if (Ri > 0) {
        items.push_back({&h->img_stage, (size_t)(Ri * c.image_dim * 2)});
        items.push_back({&h->ih, (size_t)(Ri * D * 2)});
        items.push_back({&h->ictx, (size_t)(Ri * D * 2)});
        items.push_back({&h->kvi, (size_t)(Ri * N * 2 * D * 2)});
        items.push_back({&h->o2, (size_t)(R * D * 2)});
    }
    size_t total = 0;
    for (auto& it : items) total += align_up(it.bytes, 1024);
    if (cudaMalloc(&h->ws, total) != cudaSuccess) {
        cudaGetLastError();
        return fail(h, WAN_ENOMEM, "cannot allocate " + std::to_string(total) + " bytes of workspace");
    }
    h->ws_bytes = total;
    size_t off = 0;
    for (auto& it : items) {
        *it.p = h->ws + off;
        off += align_up(it.bytes, 1024);
    }
    if (cudaMalloc(&h->d_err, sizeof(int)) != cudaSuccess) {
        cudaGetLastError();
        return fail(h, WAN_ENOMEM, "cannot allocate the error word");
    }
    cudaMemset(h->d_err, 0, sizeof(int));
    return WAN_OK;
}

// RoPE cos/sin tables per axis, computed in double on the host; entry (pos, k)
// at pos * pairs + k, or at k * len + pos when pair_major.
void rope_tables_host(const wan_dit_config& c, int Fp, int Hp, int Wp, std::vector<float2>& out, int& nt, int& nh,
                      int& nw, bool pair_major = false) {
    nt = c.rope_t / 2;
    nh = c.rope_h / 2;
    nw = c.rope_w / 2;
    out.clear();
    auto axis = [&](int len, int d_a) {
        const size_t base = out.size();
        out.resize(base + (size_t)len * (d_a / 2));
        for (int pos = 0; pos < len; ++pos)
            for (int k = 0; k < d_a / 2; ++k) {
                const double ang = pos * std::pow((double)c.rope_theta, -2.0 * k / d_a);
                const size_t at = pair_major ? (size_t)k * len + pos : (size_t)pos * (d_a / 2) + k;
                out[base + at] = make_float2((float)std::cos(ang), (float)std::sin(ang));
            }
    };
    axis(Fp, c.rope_t);
    axis(Hp, c.rope_h);
    axis(Wp, c.rope_w);
}

struct Shape {
    int B, F, Hz, Wz, Lc, per_token, lat_dtype, Li;  // Li: image tokens per sample, 0 without the image branch
    int cfg_euler;  // 1: B = 2 CFG pair whose proj_out epilogue writes the Euler-updated latent
    // sequence-parallel shard: this rank holds tokens [tok0, tok0 + Ls) of the
    // global sequence padded to world * Ls (tokens >= L are padding); world 0: whole sequence
    int tok0, Ls, world;
    int L() const { return F * (Hz / 2) * (Wz / 2); }
    int rows_per_sample() const { return world ? Ls : L(); }
};

#define TRY(x)                               \
    do {                                     \
        cudaError_t e_ = (x);                \
        if (e_ != cudaSuccess) return e_;    \
    } while (0)
#define TRYK(kc, x)                          \
    do {                                     \
        if (tm) tm->begin(ctx.stream);       \
        cudaError_t e_ = (x);                \
        if (e_ != cudaSuccess) return e_;    \
        if (tm) tm->end(ctx.stream, kc);     \
    } while (0)

EpiParams make_epi(int kind, const float* bias, void* out, long long ldo) {
    EpiParams p{};
    p.kind = kind;
    p.bias = bias;
    p.out = out;
    p.ldo = ldo;
    p.mod_div = 1;
    return p;
}

// RMSNorm row factors from the per-head sums of squares (row stride 3 heads):
// self-attention q | k, cross-attention q.
wan::RowNorm row_norm(const wan_dit* h, int which) {
    const auto& c = h->cfg;
    return wan::RowNorm{h->ssq + which * c.heads, 3LL * c.heads, c.heads, 1.0f / c.dim, c.eps};
}

// Patchify, patch GEMM, timestep embedding, text embedding and the cross K/V of
// every block (the part of the forward before the blocks).
cudaError_t issue_prologue(wan_dit* h, const Shape& s, const LaunchCtx& ctx, bool dump, KTimer* tm) {
    const auto& c = h->cfg;
    const int B = s.B, Lr = s.rows_per_sample(), Lc = s.Lc, D = c.dim, N = c.num_blocks;
    const int R = B * Lr, Rc = B * Lc;
    const long long D6 = 6LL * D;
    TRYK(WAN_KC_PATCHIFY, wan::launch_patchify(s.world ? h->sp_lat : h->lat_stage, s.lat_dtype, B, c.in_ch, s.F, s.Hz,
                                               s.Wz, h->X, h->Kp, ctx, s.world ? s.tok0 : 0, Lr));
    TRYK(WAN_KC_GEMM, wan::launch_gemm(h->X, h->Kp, h->w_pe_k, h->Kp, R, D, h->Kp,
                                       make_epi(wan::EPI_BIAS, h->b_pe, h->x, D), ctx));
    if (dump) TRY(cudaMemcpyAsync(h->dump, h->x, (size_t)R * D * 2, cudaMemcpyDeviceToDevice, ctx.stream));
    // ---- timestep embedding -> temb [B|R, D] f32, tproj [B|R, 6D] f32
    if (!s.per_token) {
        TRYK(WAN_KC_EMBEDDING, wan::launch_gemv(h->w_t1, h->b_t1, h->t_stage, 1, h->th32, D, B, D, c.freq_dim, 2, 1, ctx));
        TRYK(WAN_KC_EMBEDDING, wan::launch_gemv(h->w_t2, h->b_t2, h->th32, D, h->temb, D, B, D, D, 0, 0, ctx));
        TRYK(WAN_KC_EMBEDDING, wan::launch_gemv(h->w_tp, h->b_tp, h->temb, D, h->tproj, D6, B, 6 * D, D, 1, 0, ctx));
        TRYK(WAN_KC_EMBEDDING, wan::launch_mod_combine(h->sst_all, h->tproj, h->modc, N, B, D, ctx));
    } else {
        TRYK(WAN_KC_EMBEDDING, wan::launch_sinusoid_bf16(h->t_stage, R, c.freq_dim, h->tsin, ctx));
        TRYK(WAN_KC_GEMM, wan::launch_gemm(h->tsin, c.freq_dim, h->w_t1, c.freq_dim, R, D, c.freq_dim,
                                           make_epi(wan::EPI_BIAS_SILU, h->b_t1, h->y, D), ctx));
        TRYK(WAN_KC_GEMM, wan::launch_gemm(h->y, D, h->w_t2, D, R, D, D, make_epi(wan::EPI_BIAS_F32, h->b_t2, h->temb, D), ctx));
        TRYK(WAN_KC_EMBEDDING, wan::launch_silu_bf16(h->temb, h->tsilu, (long long)R * D, ctx));
        TRYK(WAN_KC_GEMM, wan::launch_gemm(h->tsilu, D, h->w_tp, D, R, 6 * D, D,
                                           make_epi(wan::EPI_BIAS_F32, h->b_tp, h->tproj, D6), ctx));
    }
    // ---- text embedding and the cross-attention keys/values of every block
    TRYK(WAN_KC_GEMM, wan::launch_gemm(h->ctx_stage, c.text_dim, h->w_x1, c.text_dim, Rc, D, c.text_dim,
                                       make_epi(wan::EPI_BIAS_GELU, h->b_x1, h->th, D), ctx));
    TRYK(WAN_KC_GEMM, wan::launch_gemm(h->th, D, h->w_x2, D, Rc, D, D, make_epi(wan::EPI_BIAS, h->b_x2, h->ctx, D), ctx));
    const long long ldkv = 2LL * N * D;
    TRYK(WAN_KC_GEMM, wan::launch_gemm(h->ctx, D, h->w_kv, D, Rc, (int)ldkv, D, make_epi(wan::EPI_BIAS, h->b_kv, h->kv, ldkv), ctx));
    TRYK(WAN_KC_RMSNORM_ROPE, wan::launch_rmsnorm_rope(h->kv, ldkv, Rc, D, c.eps, h->k2_gain, D, N, 2LL * D, nullptr, 0, ctx));
    // ---- image tokens (I2V): embedder (Linear, GELU_tanh, Linear), then every block's image K/V and key norm
    const int Ri = B * s.Li;
    if (s.Li > 0) {
        TRYK(WAN_KC_GEMM, wan::launch_gemm(h->img_stage, c.image_dim, h->w_i1, c.image_dim, Ri, D, c.image_dim,
                                           make_epi(wan::EPI_BIAS_GELU, h->b_i1, h->ih, D), ctx));
        TRYK(WAN_KC_GEMM, wan::launch_gemm(h->ih, D, h->w_i2, D, Ri, D, D, make_epi(wan::EPI_BIAS, h->b_i2, h->ictx, D), ctx));
        TRYK(WAN_KC_GEMM, wan::launch_gemm(h->ictx, D, h->w_kvi, D, Ri, (int)ldkv, D,
                                           make_epi(wan::EPI_BIAS, h->b_kvi, h->kvi, ldkv), ctx));
        TRYK(WAN_KC_RMSNORM_ROPE, wan::launch_rmsnorm_rope(h->kvi, ldkv, Ri, D, c.eps, h->ki_gain, D, N, 2LL * D, nullptr, 0,
                                                           ctx));
    }
    return cudaSuccess;
}

// Block i up to the self-attention: norm1 + modulation (shift row 0, scale row 1),
// the q, k, v projection with q and k RMSNorm'd across heads in two parts (the
// epilogue stores gain * RoPE(q), gain * RoPE(k) and each head's sum of
// squares; the key row factors are applied here in place, the query factors
// inside the attention -- or here too when the queries leave the GPU).
cudaError_t issue_block_pre(wan_dit* h, const Shape& s, const Plan& plan, int i, const LaunchCtx& ctx, KTimer* tm,
                            bool normalize_q) {
    const auto& c = h->cfg;
    const int B = s.B, Lr = s.rows_per_sample(), D = c.dim;
    const int R = B * Lr;
    const long long D6 = 6LL * D;
    const BlockW& w = h->blocks[i];
    const float* mc = h->modc + (long long)i * B * 6 * D;
    const int mod_div = s.per_token ? 1 : Lr;
    // per-sample: precombined rows of modc (1 + scale folded in); per-token: table + projection rows
    if (!s.per_token)
        TRYK(WAN_KC_LAYERNORM, wan::launch_layernorm(h->x, h->y, R, D, c.eps, 2, nullptr, nullptr, nullptr, mc,
                                                     nullptr, mc + D, mod_div, D6, ctx));
    else
        TRYK(WAN_KC_LAYERNORM, wan::launch_layernorm(h->x, h->y, R, D, c.eps, 0, nullptr, nullptr, w.sst, h->tproj,
                                                     w.sst + D, h->tproj + D, mod_div, D6, ctx));
    EpiParams p = make_epi(wan::EPI_QK_NORM, w.bqkv, h->qkv, 3LL * D);
    p.norm_cols = 2 * D;
    p.gain = w.qk_gain;
    p.ssq = h->ssq;
    p.ssq_ld = 3LL * c.heads;
    p.rope_L = Lr;
    p.rope_tok0 = s.world ? s.tok0 : 0;
    p.rope = plan.rt;
    TRYK(WAN_KC_GEMM_QKV, wan::launch_gemm(h->y, D, w.wqkv, D, R, 3 * D, D, p, ctx));
    char* qkv = reinterpret_cast<char*>(h->qkv);
    TRYK(WAN_KC_RMSNORM_ROPE, wan::launch_rms_apply(qkv + 2LL * D, 3LL * D, R, D, row_norm(h, 1), ctx));
    if (normalize_q) TRYK(WAN_KC_RMSNORM_ROPE, wan::launch_rms_apply(qkv, 3LL * D, R, D, row_norm(h, 0), ctx));
    return cudaSuccess;
}

// Block i after the self-attention, whose output (all heads) is in h->o: O
// projection + gated residual, affine norm2, cross-attention with its q
// RMSNorm split like the self-attention's, residual, norm3 + modulation,
// GELU-tanh FFN, gated residual.
cudaError_t issue_block_post(wan_dit* h, const Shape& s, int i, const LaunchCtx& ctx, KTimer* tm) {
    const auto& c = h->cfg;
    const int B = s.B, Lr = s.rows_per_sample(), Lc = s.Lc, D = c.dim, Fd = c.ffn_dim, N = c.num_blocks;
    const int R = B * Lr;
    const long long D6 = 6LL * D, ldkv = 2LL * N * D;
    const BlockW& w = h->blocks[i];
    const float* mc = h->modc + (long long)i * B * 6 * D;
    const int mod_div = s.per_token ? 1 : Lr;
    {
        EpiParams p = make_epi(wan::EPI_GATE_RESIDUAL, w.bo, h->x, D);
        p.gate0 = s.per_token ? w.sst + 2 * D : nullptr;
        p.gate1 = s.per_token ? h->tproj + 2 * D : mc + 2 * D;
        p.mod_div = mod_div;
        p.mod_ld = D6;
        TRYK(WAN_KC_GEMM_O, wan::launch_gemm(h->o, D, w.wo, D, R, D, D, p, ctx));
    }
    // 2. cross-attention: affine norm2, q projection + RMSNorm, attention to the context
    TRYK(WAN_KC_LAYERNORM, wan::launch_layernorm(h->x, h->y, R, D, c.eps, 1, w.n2_g, w.n2_b, nullptr, nullptr, nullptr,
                                                 nullptr, 1, 0, ctx));
    {
        EpiParams p = make_epi(wan::EPI_QK_NORM, w.bq2, h->qc, D);
        p.norm_cols = D;
        p.gain = w.q2_gain;
        p.ssq = h->ssq + 2 * c.heads;
        p.ssq_ld = 3LL * c.heads;
        TRYK(WAN_KC_GEMM_Q2, wan::launch_gemm(h->y, D, w.wq2, D, R, D, D, p, ctx));
    }
    const wan::RowNorm rn_qc = row_norm(h, 2);
    const char* kvb = reinterpret_cast<const char*>(h->kv) + 2LL * (2LL * i * D);
    TRYK(WAN_KC_CROSS_ATTENTION, wan::launch_attention(h->qc, D, kvb, ldkv, kvb + 2LL * D, ldkv, h->o, D, B, c.heads, Lr, Lc,
                                                       ctx, rn_qc));
    if (s.Li > 0) {  // image attention with the same queries, added before attn2.to_out
        const char* kvib = reinterpret_cast<const char*>(h->kvi) + 2LL * (2LL * i * D);
        TRYK(WAN_KC_CROSS_ATTENTION, wan::launch_attention(h->qc, D, kvib, ldkv, kvib + 2LL * D, ldkv, h->o2, D, B,
                                                           c.heads, Lr, s.Li, ctx, rn_qc));
        TRYK(WAN_KC_CROSS_ATTENTION, wan::launch_add_bf16(h->o, h->o2, (long long)R * D, ctx));
    }
    TRYK(WAN_KC_GEMM_O2, wan::launch_gemm(h->o, D, w.wo2, D, R, D, D, make_epi(wan::EPI_RESIDUAL, w.bo2, h->x, D), ctx));
    // 3. feed-forward: norm3 + modulation (shift row 3, scale row 4), GELU-tanh, gated residual (row 5)
    if (!s.per_token)
        TRYK(WAN_KC_LAYERNORM, wan::launch_layernorm(h->x, h->y, R, D, c.eps, 2, nullptr, nullptr, nullptr, mc + 3 * D,
                                                     nullptr, mc + 4 * D, mod_div, D6, ctx));
    else
        TRYK(WAN_KC_LAYERNORM, wan::launch_layernorm(h->x, h->y, R, D, c.eps, 0, nullptr, nullptr, w.sst + 3 * D,
                                                     h->tproj + 3 * D, w.sst + 4 * D, h->tproj + 4 * D, mod_div, D6,
                                                     ctx));
    TRYK(WAN_KC_GEMM_FFN_UP, wan::launch_gemm(h->y, D, w.w1, D, R, Fd, D, make_epi(wan::EPI_BIAS_GELU, w.b1, h->u, Fd), ctx));
    {
        EpiParams p = make_epi(wan::EPI_GATE_RESIDUAL, w.b2, h->x, D);
        p.gate0 = s.per_token ? w.sst + 5 * D : nullptr;
        p.gate1 = s.per_token ? h->tproj + 5 * D : mc + 5 * D;
        p.mod_div = mod_div;
        p.mod_ld = D6;
        TRYK(WAN_KC_GEMM_FFN_DOWN, wan::launch_gemm(h->u, Fd, w.w2, Fd, R, D, Fd, p, ctx));
    }
    return cudaSuccess;
}

// Output head: FP32 LayerNorm, (shift, scale) = head table + temb, proj_out with
// the unpatchify scatter (or the fused CFG + Euler step) in its epilogue.
cudaError_t issue_head(wan_dit* h, const Shape& s, const LaunchCtx& ctx, KTimer* tm) {
    const auto& c = h->cfg;
    const int B = s.B, L = s.L(), Lr = s.rows_per_sample(), D = c.dim;
    const int R = B * Lr;
    TRYK(WAN_KC_LAYERNORM, wan::launch_layernorm(h->x, h->y, R, D, c.eps, 0, nullptr, nullptr, h->sst_out, h->temb,
                                                 h->sst_out + D, h->temb, s.per_token ? 1 : Lr, D, ctx));
    EpiParams p = make_epi(s.cfg_euler ? wan::EPI_CFG_EULER : wan::EPI_UNPATCHIFY, h->b_po,
                           s.world ? h->sp_vel : h->vel_stage, 0);
    p.L = L;
    p.C = c.out_ch;
    p.F = s.F;
    p.Hz = s.Hz;
    p.Wz = s.Wz;
    p.up_rows = Lr;
    p.up_tok0 = s.world ? s.tok0 : 0;
    if (s.cfg_euler) {  // rows [0, L): conditional sample, [L, 2L): unconditional; x = sample 0's latent
        p.pair_off = L;
        p.x = h->lat_stage;
        p.sched = h->sched;
        TRYK(WAN_KC_GEMM, wan::launch_gemm(h->y, D, h->w_po, D, L, c.out_ch * 4, D, p, ctx));
    } else {
        TRYK(WAN_KC_GEMM, wan::launch_gemm(h->y, D, h->w_po, D, R, c.out_ch * 4, D, p, ctx));
    }
    return cudaSuccess;
}

// Issue every launch of one forward on ctx.stream (eager or under capture).
cudaError_t issue_forward(wan_dit* h, const Shape& s, const Plan& plan, const LaunchCtx& ctx, bool dump, KTimer* tm) {
    const auto& c = h->cfg;
    const int B = s.B, L = s.L(), D = c.dim, N = c.num_blocks;
    const int R = B * L;
    TRY(issue_prologue(h, s, ctx, dump, tm));
    char* qkv = reinterpret_cast<char*>(h->qkv);
    for (int i = 0; i < N; ++i) {
        TRY(issue_block_pre(h, s, plan, i, ctx, tm, false));
        TRYK(WAN_KC_SELF_ATTENTION, wan::launch_attention(qkv, 3LL * D, qkv + 2LL * D, 3LL * D, qkv + 4LL * D, 3LL * D, h->o,
                                                          D, B, c.heads, L, L, ctx, row_norm(h, 0)));
        TRY(issue_block_post(h, s, i, ctx, tm));
        if (dump)
            TRY(cudaMemcpyAsync(reinterpret_cast<char*>(h->dump) + (size_t)(i + 1) * R * D * 2, h->x, (size_t)R * D * 2,
                                cudaMemcpyDeviceToDevice, ctx.stream));
    }
    return issue_head(h, s, ctx, tm);
}
#undef TRY
#undef TRYK

wan_status ensure_plan(wan_dit* h, const Shape& s, Plan** out) {
    PlanKey key{s.B, s.F, s.Hz, s.Wz, s.Lc, s.per_token, s.lat_dtype, s.Li, s.cfg_euler, s.world, s.tok0, s.Ls};
    auto it = h->plans.find(key);
    if (it != h->plans.end()) {
        *out = &it->second;
        return WAN_OK;
    }
    Plan plan;
    std::vector<float2> tab;
    int nt, nh, nw;
    const int Fp = s.F, Hp = s.Hz / 2, Wp = s.Wz / 2;
    // the q/k projection epilogue reads the tables: pair-major, so the 32 tokens of
    // a warp read neighbouring entries
    rope_tables_host(h->cfg, Fp, Hp, Wp, tab, nt, nh, nw, true);
    WAN_CU(cudaMalloc(&plan.rope, tab.size() * sizeof(float2)), "rope table allocation");
    WAN_CU(cudaMemcpy(plan.rope, tab.data(), tab.size() * sizeof(float2), cudaMemcpyHostToDevice), "rope upload");
    plan.rt.t = plan.rope;
    plan.rt.h = plan.rope + (size_t)Fp * nt;
    plan.rt.w = plan.rt.h + (size_t)Hp * nh;
    plan.rt.Fp = Fp;
    plan.rt.Hp = Hp;
    plan.rt.Wp = Wp;
    plan.rt.nt = nt;
    plan.rt.nh = nh;
    plan.rt.nw = nw;
    plan.rt.pair_major = 1;
    auto res = h->plans.emplace(key, plan);
    *out = &res.first->second;
    return WAN_OK;
}

wan_status run_plan(wan_dit* h, const Shape& s, Plan* plan, cudaStream_t st);

LaunchCtx make_ctx(wan_dit* h, cudaStream_t st, int* counter) {
    LaunchCtx ctx;
    ctx.stream = st;
    ctx.err = h->d_err;
    ctx.wait_limit_ns = h->wait_ns;
    ctx.num_sms = h->num_sms;
    ctx.launches = counter;
    ctx.gemm_pair = h->gemm_pair ? 1 : 0;
    return ctx;
}

}  // namespace

// ====================================================================== C ABI
extern "C" {

const char* wan_status_string(wan_status s) {
    switch (s) {
        case WAN_OK: return "ok";
        case WAN_EINVAL: return "invalid argument";
        case WAN_ESHAPE: return "bad shape";
        case WAN_ENOMEM: return "out of device memory";
        case WAN_ENOWEIGHTS: return "no weights loaded";
        case WAN_EMISSING_WEIGHT: return "missing weight";
        case WAN_EUNEXPECTED_WEIGHT: return "unexpected weight";
        case WAN_ECUDA: return "CUDA error";
        case WAN_ETIMEOUT: return "kernel wait timed out";
        case WAN_EINTERNAL: return "internal error";
        case WAN_EUNSUPPORTED: return "unsupported configuration";
    }
    return "unknown status";
}

wan_status wan_dit_create(const wan_dit_config* cfg, int device, wan_dit** out) {
    if (!out) return WAN_EINVAL;
    *out = nullptr;
    if (!cfg) return WAN_EINVAL;
    std::string why;
    wan_dit* h = new wan_dit();
    h->cfg = *cfg;
    h->device = device;
    if (!valid_config(*cfg, why)) {
        delete h;
        return WAN_EUNSUPPORTED;
    }
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) {
        cudaGetLastError();
        delete h;
        return WAN_ECUDA;
    }
    cudaSetDevice(device);
    cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, device);
    if (wan::init_kernel_attributes() != cudaSuccess) {
        cudaGetLastError();
        delete h;
        return WAN_ECUDA;
    }
    wan_status s = build_weights(h);
    if (s == WAN_OK) s = build_workspace(h);
    if (s == WAN_OK && cudaStreamCreateWithFlags(&h->cap_stream, cudaStreamNonBlocking) != cudaSuccess) s = WAN_ECUDA;
    if (s != WAN_OK) {
        wan_dit_destroy(h);
        return s;
    }
    cudaDeviceSynchronize();
    *out = h;
    return WAN_OK;
}

void wan_dit_destroy(wan_dit* h) {
    if (!h) return;
    cudaSetDevice(h->device);
    cudaDeviceSynchronize();
    for (auto& kv : h->plans) {
        if (kv.second.exec) cudaGraphExecDestroy(kv.second.exec);
        if (kv.second.exec_timed) cudaGraphExecDestroy(kv.second.exec_timed);
        if (kv.second.rope) cudaFree(kv.second.rope);
        kv.second.timer.destroy();
    }
    if (h->cap_stream) cudaStreamDestroy(h->cap_stream);
    if (h->arena) cudaFree(h->arena);
    if (h->ws) cudaFree(h->ws);
    if (h->d_err) cudaFree(h->d_err);
    if (h->sp_lat) cudaFree(h->sp_lat);
    if (h->sp_vel) cudaFree(h->sp_vel);
    delete h;
}

const char* wan_dit_last_error(const wan_dit* h) { return h ? h->err.c_str() : "null handle"; }

int wan_dit_last_launch_count(const wan_dit* h) { return h ? h->last_launches : 0; }

wan_status wan_dit_load_weights(wan_dit* h, int n, const char* const* names, const void* const* ptrs,
                                const int* dtypes, const int64_t* const* shapes, const int* ndims, int ptrs_on_device,
                                void* stream) {
    if (!h) return WAN_EINVAL;
    if (n < 0 || (n > 0 && (!names || !ptrs || !dtypes || !shapes || !ndims))) return fail(h, WAN_EINVAL, "null arrays");
    cudaSetDevice(h->device);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    wan_status first = WAN_OK;
    void* tmp = nullptr;
    size_t tmp_bytes = 0;
    for (int i = 0; i < n; ++i) {
        if (!names[i] || !ptrs[i]) {
            if (first == WAN_OK) first = fail(h, WAN_EINVAL, "null name or pointer at index " + std::to_string(i));
            continue;
        }
        auto it = h->slots.find(names[i]);
        if (it == h->slots.end()) {
            if (first == WAN_OK) first = fail(h, WAN_EUNEXPECTED_WEIGHT, std::string("unexpected weight ") + names[i]);
            continue;
        }
        const Slot& sl = it->second;
        bool shape_ok = ndims[i] == (int)sl.shape.size() && shapes[i] != nullptr;
        for (int d = 0; shape_ok && d < ndims[i]; ++d) shape_ok = shapes[i][d] == sl.shape[d];
        if (!shape_ok || (dtypes[i] != WAN_DTYPE_F32 && dtypes[i] != WAN_DTYPE_BF16)) {
            if (first == WAN_OK) first = fail(h, WAN_ESHAPE, std::string("bad shape or dtype for ") + names[i]);
            continue;
        }
        const size_t src_bytes = sl.numel * (dtypes[i] == WAN_DTYPE_BF16 ? 2 : 4);
        const void* src = ptrs[i];
        if (!ptrs_on_device) {
            if (dtypes[i] == sl.dst_dtype) {
                WAN_CU(cudaMemcpyAsync(sl.dst, src, src_bytes, cudaMemcpyHostToDevice, st), "weight upload");
                h->loaded.insert(names[i]);
                continue;
            }
            if (src_bytes > tmp_bytes) {
                WAN_CU(cudaStreamSynchronize(st), "weight upload");
                if (tmp) cudaFree(tmp);
                tmp = nullptr;
                WAN_CU(cudaMalloc(&tmp, src_bytes), "weight staging allocation");
                tmp_bytes = src_bytes;
            }
            WAN_CU(cudaMemcpyAsync(tmp, src, src_bytes, cudaMemcpyHostToDevice, st), "weight upload");
            src = tmp;
        }
        if (dtypes[i] == sl.dst_dtype)
            WAN_CU(cudaMemcpyAsync(sl.dst, src, src_bytes, cudaMemcpyDeviceToDevice, st), "weight copy");
        else
            WAN_CU(wan::launch_convert(src, dtypes[i], sl.dst, sl.dst_dtype, sl.numel, st), "weight conversion");
        if (!ptrs_on_device) WAN_CU(cudaStreamSynchronize(st), "weight upload");
        h->loaded.insert(names[i]);
    }
    if (h->w_pe_k != h->w_pe && h->loaded.count("patch_embedding.weight")) {
        // [D, 4 * in_ch] -> [D, Kp]; the pad columns stay zero
        const size_t row = (size_t)h->cfg.in_ch * 4 * 2;
        WAN_CU(cudaMemcpy2DAsync(h->w_pe_k, (size_t)h->Kp * 2, h->w_pe, row, row, h->cfg.dim, cudaMemcpyDeviceToDevice,
                                 st),
               "patch weight repack");
    }
    WAN_CU(cudaStreamSynchronize(st), "weight load");
    if (tmp) cudaFree(tmp);
    return first;
}

int wan_dit_missing_weights(const wan_dit* h, char* buf, int len) {
    if (!h) return -1;
    int missing = 0;
    std::string s;
    for (auto& kv : h->slots) {
        if (h->loaded.count(kv.first)) continue;
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

wan_status wan_dit_set_block_dump(wan_dit* h, void* dst) {
    if (!h) return WAN_EINVAL;
    h->dump = dst;
    return WAN_OK;
}

wan_status wan_dit_set_option(wan_dit* h, int option, int64_t value) {
    if (!h) return WAN_EINVAL;
    if (option == WAN_OPT_GRAPH) {
        h->use_graph = value != 0;
        return WAN_OK;
    }
    if (option == WAN_OPT_WAIT_LIMIT_NS) {
        if (value < 0) return fail(h, WAN_EINVAL, "negative wait limit");
        h->wait_ns = (uint64_t)value;
        for (auto& kv : h->plans) {  // graphs hold the old limit
            if (kv.second.exec) cudaGraphExecDestroy(kv.second.exec);
            if (kv.second.exec_timed) cudaGraphExecDestroy(kv.second.exec_timed);
            kv.second.exec = kv.second.exec_timed = nullptr;
        }
        return WAN_OK;
    }
    if (option == WAN_OPT_KERNEL_TIMING) {
        h->timing = value != 0;
        return WAN_OK;
    }
    if (option == WAN_OPT_GEMM_PAIR) {
        h->gemm_pair = value != 0;
        for (auto& kv : h->plans) {  // graphs hold the old kernels
            if (kv.second.exec) cudaGraphExecDestroy(kv.second.exec);
            if (kv.second.exec_timed) cudaGraphExecDestroy(kv.second.exec_timed);
            kv.second.exec = kv.second.exec_timed = nullptr;
        }
        return WAN_OK;
    }
    return fail(h, WAN_EINVAL, "unknown option");
}

double wan_dit_flops(const wan_dit* h, int B, int F, int Hz, int Wz, int Lc, int per_token) {
    return wan_dit_flops_image(h, B, F, Hz, Wz, Lc, per_token, 0);
}

double wan_dit_flops_image(const wan_dit* h, int B, int F, int Hz, int Wz, int Lc, int per_token, int Li) {
    if (!h) return 0.0;
    const auto& c = h->cfg;
    const double L = (double)F * (Hz / 2) * (Wz / 2), D = c.dim, Fd = c.ffn_dim, N = c.num_blocks;
    const double Pin = c.in_ch * 4.0, Pout = c.out_ch * 4.0;
    double per_block = 2 * L * D * 6 * D + 4 * L * D * Fd + 4 * (double)Lc * D * D + 4 * L * L * D + 4 * L * Lc * D;
    double f = N * per_block + 2 * L * D * Pin + 2 * L * D * Pout + 2.0 * Lc * (c.text_dim * D + D * D);
    f += per_token ? 2 * L * (c.freq_dim * D + 7 * D * D) : 2 * (c.freq_dim * D + 7 * D * D);
    if (Li > 0 && c.image_dim > 0)  // image embedder, per block image K/V projections and image attention
        f += 2.0 * Li * ((double)c.image_dim * D + D * D) + N * (4.0 * Li * D * D + 4.0 * L * Li * D);
    return B * f;
}

int wan_moe_select(double t, double boundary, int num_train_timesteps) {
    return t >= boundary * (double)num_train_timesteps ? 0 : 1;
}

wan_status wan_dit_forward(wan_dit* h, const void* latent, int latent_dtype, int B, int F, int Hz, int Wz,
                           const float* timestep, int per_token, const void* context, int Lc, float* velocity,
                           int io_on_device, void* stream) {
    return wan_dit_forward_image(h, latent, latent_dtype, B, F, Hz, Wz, timestep, per_token, context, Lc, nullptr, 0,
                                 velocity, io_on_device, stream);
}

wan_status wan_dit_forward_image(wan_dit* h, const void* latent, int latent_dtype, int B, int F, int Hz, int Wz,
                                 const float* timestep, int per_token, const void* context, int Lc, const void* image,
                                 int Li, float* velocity, int io_on_device, void* stream) {
    if (!h) return WAN_EINVAL;
    if (!latent || !timestep || !context || !velocity) return fail(h, WAN_EINVAL, "null input or output pointer");
    if (image && h->cfg.image_dim <= 0) return fail(h, WAN_EINVAL, "image tokens given to a model without an image branch");
    if (!image) Li = 0;
    if (image && (Li < 1 || Li > h->cfg.max_image)) return fail(h, WAN_ESHAPE, "image token count outside 1..max_image");
    if (latent_dtype != WAN_DTYPE_F32 && latent_dtype != WAN_DTYPE_BF16) return fail(h, WAN_EINVAL, "latent dtype");
    const auto& c = h->cfg;
    if (B < 1 || B > c.max_batch) return fail(h, WAN_ESHAPE, "batch outside 1..max_batch");
    if (F < 1 || Hz < 2 || Wz < 2 || Hz % 2 || Wz % 2) return fail(h, WAN_ESHAPE, "latent grid must be F>=1, even Hz, Wz");
    const long long L = (long long)F * (Hz / 2) * (Wz / 2);
    if (L > c.max_tokens) return fail(h, WAN_ESHAPE, "token count exceeds max_tokens");
    if (Lc < 1 || Lc > c.max_text) return fail(h, WAN_ESHAPE, "context length outside 1..max_text");
    if (per_token != 0 && per_token != 1) return fail(h, WAN_EINVAL, "per_token must be 0 or 1");
    if (h->loaded.empty()) return fail(h, WAN_ENOWEIGHTS, "forward before load_weights");
    if (h->loaded.size() != h->slots.size()) {
        char buf[256];
        int m = wan_dit_missing_weights(h, buf, sizeof(buf));
        return fail(h, WAN_EMISSING_WEIGHT, std::to_string(m) + " weights missing: " + buf);
    }
    cudaSetDevice(h->device);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    Shape s{B, F, Hz, Wz, Lc, per_token, latent_dtype, Li, 0, 0, 0, 0};
    Plan* plan = nullptr;
    wan_status ps = ensure_plan(h, s, &plan);
    if (ps != WAN_OK) return ps;

    // inputs -> staging
    const cudaMemcpyKind h2d = io_on_device ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice;
    const size_t lat_bytes = (size_t)B * c.in_ch * F * Hz * Wz * (latent_dtype == WAN_DTYPE_F32 ? 4 : 2);
    WAN_CU(cudaMemcpyAsync(h->lat_stage, latent, lat_bytes, h2d, st), "latent copy");
    WAN_CU(cudaMemcpyAsync(h->t_stage, timestep, (size_t)(per_token ? B * L : B) * 4, h2d, st), "timestep copy");
    WAN_CU(cudaMemcpyAsync(h->ctx_stage, context, (size_t)B * Lc * c.text_dim * 2, h2d, st), "context copy");
    if (Li > 0) WAN_CU(cudaMemcpyAsync(h->img_stage, image, (size_t)B * Li * c.image_dim * 2, h2d, st), "image copy");

    WAN_CU_RET(run_plan(h, s, plan, st));
    const size_t vel_bytes = (size_t)B * c.out_ch * F * Hz * Wz * 4;
    WAN_CU(cudaMemcpyAsync(velocity, h->vel_stage, vel_bytes, io_on_device ? cudaMemcpyDeviceToDevice : cudaMemcpyDeviceToHost,
                           st),
           "velocity copy");
    return WAN_OK;
}

}  // extern "C"

namespace {
// Launch the forward of plan `plan` on `st` (graph replay, or eager launches
// when graphs are off or the block dump is on).  Inputs are already staged.
wan_status run_plan(wan_dit* h, const Shape& s, Plan* plan, cudaStream_t st) {
    const auto& c = h->cfg;
    const bool dump = h->dump != nullptr;
    const bool timed = h->timing;
    if (timed) WAN_CU(plan->timer.ensure(20 * c.num_blocks + 64), "timing events");
    KTimer* tm = timed ? &plan->timer : nullptr;
    if (tm) tm->n = 0;
    if (h->use_graph && !dump) {
        cudaGraphExec_t& exec = timed ? plan->exec_timed : plan->exec;
        if (!exec) {
            int count = 0;
            LaunchCtx ctx = make_ctx(h, h->cap_stream, &count);
            WAN_CU(cudaStreamBeginCapture(h->cap_stream, cudaStreamCaptureModeThreadLocal), "begin capture");
            cudaError_t e = issue_forward(h, s, *plan, ctx, false, tm);
            cudaGraph_t g = nullptr;
            cudaError_t e2 = cudaStreamEndCapture(h->cap_stream, &g);
            if (e != cudaSuccess) {
                if (g) cudaGraphDestroy(g);
                return cuda_fail(h, e, "forward launch (capture)");
            }
            if (e2 != cudaSuccess) return cuda_fail(h, e2, "end capture");
            cudaError_t e3 = cudaGraphInstantiate(&exec, g, 0);
            cudaGraphDestroy(g);
            if (e3 != cudaSuccess) return cuda_fail(h, e3, "graph instantiate");
            plan->launches = count;
            if (tm) plan->timed_pairs = tm->n;
        }
        WAN_CU(cudaGraphLaunch(exec, st), "graph launch");
        h->last_launches = plan->launches;
    } else {
        int count = 0;
        LaunchCtx ctx = make_ctx(h, st, &count);
        cudaError_t e = issue_forward(h, s, *plan, ctx, dump, tm);
        if (e != cudaSuccess) return cuda_fail(h, e, "forward launch");
        h->last_launches = count;
        if (tm) plan->timed_pairs = tm->n;
    }
    h->last_plan = plan;
    h->last_timed = timed;
    return WAN_OK;
}
}  // namespace

extern "C" {

wan_status wan_dit_forward_cfg_euler(wan_dit* h, const float* x, int F, int Hz, int Wz, float timestep,
                                     const void* context, int Lc, float guidance, float sigma, float sigma_next,
                                     float* x_next, int io_on_device, void* stream) {
    if (!h) return WAN_EINVAL;
    if (!x || !context || !x_next) return fail(h, WAN_EINVAL, "null input or output pointer");
    const auto& c = h->cfg;
    if (c.in_ch != c.out_ch) return fail(h, WAN_EUNSUPPORTED, "the sampler step needs in_ch == out_ch");
    if (c.max_batch < 2) return fail(h, WAN_ESHAPE, "the CFG pair needs max_batch >= 2");
    if (F < 1 || Hz < 2 || Wz < 2 || Hz % 2 || Wz % 2) return fail(h, WAN_ESHAPE, "latent grid must be F>=1, even Hz, Wz");
    const long long L = (long long)F * (Hz / 2) * (Wz / 2);
    if (L > c.max_tokens) return fail(h, WAN_ESHAPE, "token count exceeds max_tokens");
    if (Lc < 1 || Lc > c.max_text) return fail(h, WAN_ESHAPE, "context length outside 1..max_text");
    if (!std::isfinite(guidance) || !std::isfinite(sigma) || !std::isfinite(sigma_next) || !std::isfinite(timestep))
        return fail(h, WAN_EINVAL, "non-finite sampler scalar");
    if (h->loaded.empty()) return fail(h, WAN_ENOWEIGHTS, "forward before load_weights");
    if (h->loaded.size() != h->slots.size()) {
        char buf[256];
        int m = wan_dit_missing_weights(h, buf, sizeof(buf));
        return fail(h, WAN_EMISSING_WEIGHT, std::to_string(m) + " weights missing: " + buf);
    }
    cudaSetDevice(h->device);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    Shape s{2, F, Hz, Wz, Lc, 0, WAN_DTYPE_F32, 0, 1, 0, 0, 0};
    Plan* plan = nullptr;
    wan_status ps = ensure_plan(h, s, &plan);
    if (ps != WAN_OK) return ps;
    // the same latent for both samples; per-call scalars through a tiny kernel
    const cudaMemcpyKind h2d = io_on_device ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice;
    const size_t lat_bytes = (size_t)c.in_ch * F * Hz * Wz * 4;
    WAN_CU(cudaMemcpyAsync(h->lat_stage, x, lat_bytes, h2d, st), "latent copy");
    WAN_CU(cudaMemcpyAsync(reinterpret_cast<char*>(h->lat_stage) + lat_bytes, x, lat_bytes, h2d, st), "latent copy");
    WAN_CU(cudaMemcpyAsync(h->ctx_stage, context, (size_t)2 * Lc * c.text_dim * 2, h2d, st), "context copy");
    LaunchCtx sctx = make_ctx(h, st, nullptr);
    WAN_CU(wan::launch_set_sampler_scalars(h->sched, guidance, sigma_next - sigma, h->t_stage, 2, timestep, sctx),
           "sampler scalars");
    WAN_CU_RET(run_plan(h, s, plan, st));
    WAN_CU(cudaMemcpyAsync(x_next, h->vel_stage, lat_bytes, io_on_device ? cudaMemcpyDeviceToDevice : cudaMemcpyDeviceToHost,
                           st),
           "latent copy back");
    return WAN_OK;
}

// ---------------------------------------------------------------- sequence-parallel (Ulysses) stages
static Shape sp_shape(const wan_dit* h) {
    return Shape{h->sp_B, h->sp_F, h->sp_Hz, h->sp_Wz, h->sp_Lc, h->sp_per_token, h->sp_dtype, 0, 0,
                 h->sp_rank * h->sp_Ls, h->sp_Ls, h->sp_world};
}

wan_status wan_dit_sp_begin(wan_dit* h, const void* latent, int latent_dtype, int B, int F, int Hz, int Wz,
                            const float* timestep, int per_token, const void* context, int Lc, int rank, int world,
                            int io_on_device, void* stream) {
    if (!h) return WAN_EINVAL;
    if (!latent || !timestep || !context) return fail(h, WAN_EINVAL, "null input pointer");
    if (latent_dtype != WAN_DTYPE_F32 && latent_dtype != WAN_DTYPE_BF16) return fail(h, WAN_EINVAL, "latent dtype");
    const auto& c = h->cfg;
    if (world < 1 || rank < 0 || rank >= world) return fail(h, WAN_EINVAL, "rank outside 0..world-1");
    if (c.heads % world) return fail(h, WAN_ESHAPE, "heads must be a multiple of the world size");
    if (c.image_dim > 0) return fail(h, WAN_EUNSUPPORTED, "the sequence-parallel stages cover text-to-video models");
    if (B < 1 || B > c.max_batch) return fail(h, WAN_ESHAPE, "batch outside 1..max_batch");
    if (F < 1 || Hz < 2 || Wz < 2 || Hz % 2 || Wz % 2) return fail(h, WAN_ESHAPE, "latent grid must be F>=1, even Hz, Wz");
    if (Lc < 1 || Lc > c.max_text) return fail(h, WAN_ESHAPE, "context length outside 1..max_text");
    if (per_token != 0 && per_token != 1) return fail(h, WAN_EINVAL, "per_token must be 0 or 1");
    const long long L = (long long)F * (Hz / 2) * (Wz / 2);
    const long long Ls = (L + world - 1) / world;  // the sequence padded to world * Ls tokens
    if (Ls > c.max_tokens) return fail(h, WAN_ESHAPE, "shard tokens exceed max_tokens");
    if (h->loaded.empty()) return fail(h, WAN_ENOWEIGHTS, "forward before load_weights");
    if (h->loaded.size() != h->slots.size()) return fail(h, WAN_EMISSING_WEIGHT, "weights missing");
    cudaSetDevice(h->device);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    h->sp_B = B; h->sp_F = F; h->sp_Hz = Hz; h->sp_Wz = Wz; h->sp_Lc = Lc; h->sp_per_token = per_token;
    h->sp_dtype = latent_dtype; h->sp_rank = rank; h->sp_world = world; h->sp_Ls = (int)Ls;
    const Shape s = sp_shape(h);
    Plan* plan = nullptr;
    wan_status ps = ensure_plan(h, s, &plan);
    if (ps != WAN_OK) return ps;
    const cudaMemcpyKind h2d = io_on_device ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice;
    const size_t lat_bytes = (size_t)B * c.in_ch * F * Hz * Wz * (latent_dtype == WAN_DTYPE_F32 ? 4 : 2);
    const size_t vel_bytes = (size_t)B * c.out_ch * F * Hz * Wz * 4;
    if (lat_bytes > h->sp_lat_bytes) {
        if (h->sp_lat) cudaFree(h->sp_lat);
        h->sp_lat = nullptr;
        h->sp_lat_bytes = 0;
        WAN_CU(cudaMalloc(&h->sp_lat, lat_bytes), "sequence-parallel latent staging");
        h->sp_lat_bytes = lat_bytes;
    }
    if (vel_bytes > h->sp_vel_bytes) {
        if (h->sp_vel) cudaFree(h->sp_vel);
        h->sp_vel = nullptr;
        h->sp_vel_bytes = 0;
        WAN_CU(cudaMalloc(&h->sp_vel, vel_bytes), "sequence-parallel velocity staging");
        h->sp_vel_bytes = vel_bytes;
    }
    WAN_CU(cudaMemcpyAsync(h->sp_lat, latent, lat_bytes, h2d, st), "latent copy");
    if (per_token) {  // this shard's columns of the [B, L] timesteps; padding tokens get t = 0
        const long long tok0 = (long long)rank * Ls, n = std::max(0LL, std::min(Ls, L - tok0));
        WAN_CU(cudaMemsetAsync(h->t_stage, 0, (size_t)B * Ls * 4, st), "timestep clear");
        if (n > 0)
            WAN_CU(cudaMemcpy2DAsync(h->t_stage, (size_t)Ls * 4, timestep + tok0, (size_t)L * 4, (size_t)n * 4, B, h2d, st),
                   "timestep copy");
    } else {
        WAN_CU(cudaMemcpyAsync(h->t_stage, timestep, (size_t)B * 4, h2d, st), "timestep copy");
    }
    WAN_CU(cudaMemcpyAsync(h->ctx_stage, context, (size_t)B * Lc * c.text_dim * 2, h2d, st), "context copy");
    LaunchCtx ctx = make_ctx(h, st, nullptr);
    cudaError_t e = issue_prologue(h, s, ctx, false, nullptr);
    if (e != cudaSuccess) return cuda_fail(h, e, "sequence-parallel prologue");
    h->sp_active = true;
    h->sp_next_block = 0;
    h->sp_phase = 0;
    return WAN_OK;
}

wan_status wan_dit_sp_block_qkv(wan_dit* h, int block, void* send, void* stream) {
    if (!h) return WAN_EINVAL;
    if (!send) return fail(h, WAN_EINVAL, "null send buffer");
    if (!h->sp_active || block != h->sp_next_block || h->sp_phase != 0)
        return fail(h, WAN_EINVAL, "sp_block_qkv out of order (sp_begin, then per block qkv and finish)");
    cudaSetDevice(h->device);
    const Shape s = sp_shape(h);
    Plan* plan = nullptr;
    wan_status ps = ensure_plan(h, s, &plan);
    if (ps != WAN_OK) return ps;
    LaunchCtx ctx = make_ctx(h, reinterpret_cast<cudaStream_t>(stream), nullptr);
    cudaError_t e = issue_block_pre(h, s, *plan, block, ctx, nullptr, true);
    if (e == cudaSuccess) e = wan::launch_sp_pack(h->qkv, send, s.B, s.world, s.Ls, h->cfg.dim, ctx);
    if (e != cudaSuccess) return cuda_fail(h, e, "sequence-parallel block (q, k, v)");
    h->sp_phase = 1;
    return WAN_OK;
}

wan_status wan_dit_sp_attention(wan_dit* h, const void* recv, void* out, void* stream) {
    if (!h) return WAN_EINVAL;
    if (!recv || !out) return fail(h, WAN_EINVAL, "null exchange buffer");
    if (!h->sp_active || h->sp_phase != 1) return fail(h, WAN_EINVAL, "sp_attention outside a block");
    cudaSetDevice(h->device);
    const Shape s = sp_shape(h);
    const int hl = h->cfg.heads / s.world, hd = 128 * hl, Lp = s.Ls * s.world;
    LaunchCtx ctx = make_ctx(h, reinterpret_cast<cudaStream_t>(stream), nullptr);
    // queries: every (padded) token; keys: the L real tokens (padding sits past them).
    // One launch per sample: a sample's keys are L rows of a buffer whose samples are Lp rows apart.
    for (int b = 0; b < s.B; ++b) {
        const char* r = reinterpret_cast<const char*>(recv) + (size_t)b * Lp * 3 * hd * 2;
        char* o = reinterpret_cast<char*>(out) + (size_t)b * Lp * hd * 2;
        cudaError_t e = wan::launch_attention(r, 3LL * hd, r + 2LL * hd, 3LL * hd, r + 4LL * hd, 3LL * hd, o, hd, 1, hl,
                                              Lp, s.L(), ctx);
        if (e != cudaSuccess) return cuda_fail(h, e, "sequence-parallel attention");
    }
    return WAN_OK;
}

wan_status wan_dit_sp_block_finish(wan_dit* h, int block, const void* back, void* stream) {
    if (!h) return WAN_EINVAL;
    if (!back) return fail(h, WAN_EINVAL, "null exchange buffer");
    if (!h->sp_active || block != h->sp_next_block || h->sp_phase != 1)
        return fail(h, WAN_EINVAL, "sp_block_finish out of order");
    cudaSetDevice(h->device);
    const Shape s = sp_shape(h);
    LaunchCtx ctx = make_ctx(h, reinterpret_cast<cudaStream_t>(stream), nullptr);
    cudaError_t e = wan::launch_sp_unpack(back, h->o, s.B, s.world, s.Ls, h->cfg.dim, ctx);
    if (e == cudaSuccess) e = issue_block_post(h, s, block, ctx, nullptr);
    if (e != cudaSuccess) return cuda_fail(h, e, "sequence-parallel block (output side)");
    h->sp_phase = 0;
    h->sp_next_block = block + 1;
    return WAN_OK;
}

wan_status wan_dit_sp_end(wan_dit* h, float* velocity, int io_on_device, void* stream) {
    if (!h) return WAN_EINVAL;
    if (!velocity) return fail(h, WAN_EINVAL, "null output pointer");
    if (!h->sp_active || h->sp_phase != 0 || h->sp_next_block != h->cfg.num_blocks)
        return fail(h, WAN_EINVAL, "sp_end before every block finished");
    cudaSetDevice(h->device);
    const Shape s = sp_shape(h);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t vel_bytes = (size_t)s.B * h->cfg.out_ch * s.F * s.Hz * s.Wz * 4;
    WAN_CU(cudaMemsetAsync(h->sp_vel, 0, vel_bytes, st), "velocity clear");
    LaunchCtx ctx = make_ctx(h, st, nullptr);
    cudaError_t e = issue_head(h, s, ctx, nullptr);
    if (e != cudaSuccess) return cuda_fail(h, e, "sequence-parallel head");
    WAN_CU(cudaMemcpyAsync(velocity, h->sp_vel, vel_bytes, io_on_device ? cudaMemcpyDeviceToDevice : cudaMemcpyDeviceToHost,
                           st),
           "velocity copy");
    h->sp_active = false;
    return WAN_OK;
}

wan_status wan_flow_sigmas(int steps, double shift, double* sigmas) {
    if (!sigmas || steps < 1 || !(shift > 0.0) || !std::isfinite(shift)) return WAN_EINVAL;
    for (int i = 0; i < steps; ++i) {
        const double u = 1.0 - (double)i / steps;
        sigmas[i] = shift * u / (1.0 + (shift - 1.0) * u);
    }
    sigmas[steps] = 0.0;
    return WAN_OK;
}

wan_status wan_dit_kernel_time(wan_dit* h, int kc, double* total_ms, int* launches) {
    if (!h || !total_ms || !launches || kc < 0 || kc >= WAN_KC_COUNT) return WAN_EINVAL;
    *total_ms = 0.0;
    *launches = 0;
    if (!h->last_plan || !h->last_timed) return fail(h, WAN_EINVAL, "no timed forward yet");
    cudaSetDevice(h->device);
    KTimer& t = h->last_plan->timer;
    for (int i = 0; i < h->last_plan->timed_pairs; ++i) {
        if (t.cls[i] != kc) continue;
        WAN_CU(cudaEventSynchronize(t.ev[2 * i + 1]), "timing event");
        float ms = 0.f;
        WAN_CU(cudaEventElapsedTime(&ms, t.ev[2 * i], t.ev[2 * i + 1]), "timing event");
        *total_ms += ms;
        ++*launches;
    }
    return WAN_OK;
}

wan_status wan_dit_sync(wan_dit* h, void* stream) {
    if (!h) return WAN_EINVAL;
    cudaSetDevice(h->device);
    WAN_CU(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)), "stream synchronize");
    int flag = 0;
    WAN_CU(cudaMemcpy(&flag, h->d_err, sizeof(int), cudaMemcpyDeviceToHost), "error word read");
    if (flag) {
        cudaMemset(h->d_err, 0, sizeof(int));
        return fail(h, WAN_ETIMEOUT, "a kernel's on-chip wait ran out of time");
    }
    return WAN_OK;
}

// ====================================================================== op-level entry points
namespace {
struct OpState {
    int device = -1;
    int* d_err = nullptr;
    int num_sms = 148;
    uint64_t wait_ns = kDefaultWaitNs;
    int gemm_pair = 1;
};
std::mutex g_op_mu;
std::map<int, OpState> g_ops;

bool op_ctx(cudaStream_t st, LaunchCtx* ctx) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    std::lock_guard<std::mutex> lk(g_op_mu);
    OpState& s = g_ops[dev];
    if (!s.d_err) {
        if (cudaMalloc(&s.d_err, sizeof(int)) != cudaSuccess) return false;
        cudaMemset(s.d_err, 0, sizeof(int));
        cudaDeviceGetAttribute(&s.num_sms, cudaDevAttrMultiProcessorCount, dev);
        s.device = dev;
        if (wan::init_kernel_attributes() != cudaSuccess) return false;
    }
    ctx->stream = st;
    ctx->err = s.d_err;
    ctx->wait_limit_ns = s.wait_ns;
    ctx->num_sms = s.num_sms;
    ctx->launches = nullptr;
    ctx->gemm_pair = s.gemm_pair;
    return true;
}

wan_status op_status(cudaError_t e) {
    if (e == cudaSuccess) return WAN_OK;
    if (e == cudaErrorInvalidValue) return WAN_ESHAPE;
    return WAN_ECUDA;
}
}  // namespace

void wan_op_set_wait_limit_ns(int64_t ns) {
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lk(g_op_mu);
    g_ops[dev].wait_ns = ns < 0 ? 0 : (uint64_t)ns;
}

void wan_op_set_gemm_pair(int on) {
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lk(g_op_mu);
    g_ops[dev].gemm_pair = on ? 1 : 0;
}

int wan_op_gemm_pair_clusters(void) {
    LaunchCtx ctx;
    if (!op_ctx(nullptr, &ctx)) return -1;
    return wan::gemm_pair_clusters();
}

wan_status wan_op_sync(void* stream) {
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return WAN_ECUDA;
    LaunchCtx ctx;
    if (!op_ctx(nullptr, &ctx)) return WAN_ECUDA;
    int flag = 0;
    if (cudaMemcpy(&flag, ctx.err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return WAN_ECUDA;
    if (flag) {
        cudaMemset(ctx.err, 0, sizeof(int));
        return WAN_ETIMEOUT;
    }
    return WAN_OK;
}

wan_status wan_op_gemm(const void* A, int64_t lda, const void* W, int64_t ldw, int M, int N, int K, int epilogue,
                       const wan_epilogue* ep, void* stream) {
    if (!A || !W || !ep || !ep->out) return WAN_EINVAL;
    if ((epilogue < WAN_EPI_BIAS || epilogue > WAN_EPI_UNPATCHIFY) && epilogue != WAN_EPI_QK_NORM) return WAN_EINVAL;
    if (epilogue == WAN_EPI_GATE_RESIDUAL && !ep->gate0 && !ep->gate1) return WAN_EINVAL;
    if (M < 0) return WAN_ESHAPE;
    EpiParams p{};
    p.kind = epilogue;
    p.bias = ep->bias;
    p.out = ep->out;
    p.ldo = ep->ldo;
    p.gate0 = ep->gate0;
    p.gate1 = ep->gate1;
    p.mod_div = ep->mod_div > 0 ? ep->mod_div : 1;
    p.mod_ld = ep->mod_ld;
    if (epilogue == WAN_EPI_UNPATCHIFY) {
        if (ep->up_C <= 0 || ep->up_F <= 0 || ep->up_Hz % 2 || ep->up_Wz % 2 || N != 4 * ep->up_C) return WAN_ESHAPE;
        p.C = ep->up_C;
        p.F = ep->up_F;
        p.Hz = ep->up_Hz;
        p.Wz = ep->up_Wz;
        p.L = ep->up_F * (ep->up_Hz / 2) * (ep->up_Wz / 2);
        if (M % p.L) return WAN_ESHAPE;
    }
    float2* tab = nullptr;
    if (epilogue == WAN_EPI_QK_NORM) {
        if (!ep->ssq || (ep->norm_cols > 0 && !ep->gain)) return WAN_EINVAL;
        p.norm_cols = ep->norm_cols;
        p.gain = ep->gain;
        p.ssq = ep->ssq;
        p.ssq_ld = ep->ssq_ld;
        if (ep->rope) {
            if (ep->rope_F <= 0 || ep->rope_H <= 0 || ep->rope_W <= 0 || ep->rope_t % 2 || ep->rope_h % 2 ||
                ep->rope_w % 2 || ep->rope_t + ep->rope_h + ep->rope_w != 128 || !(ep->rope_theta > 0.f))
                return WAN_ESHAPE;
            if (N % 256 || ep->norm_cols % 128 || ep->norm_cols > N || ep->ssq_ld < ep->norm_cols / 128 ||
                ep->ldo % 8)
                return WAN_ESHAPE;
            wan_dit_config c{};
            c.rope_t = ep->rope_t;
            c.rope_h = ep->rope_h;
            c.rope_w = ep->rope_w;
            c.rope_theta = ep->rope_theta;
            std::vector<float2> host;
            int nt, nh, nw;
            rope_tables_host(c, ep->rope_F, ep->rope_H, ep->rope_W, host, nt, nh, nw, true);
            if (cudaMalloc(&tab, host.size() * sizeof(float2)) != cudaSuccess) {
                cudaGetLastError();
                return WAN_ENOMEM;
            }
            if (cudaMemcpy(tab, host.data(), host.size() * sizeof(float2), cudaMemcpyHostToDevice) != cudaSuccess) {
                cudaFree(tab);
                return WAN_ECUDA;
            }
            p.rope = wan::RopeTables{tab, tab + (size_t)ep->rope_F * nt, tab + (size_t)ep->rope_F * nt + (size_t)ep->rope_H * nh,
                                     ep->rope_F, ep->rope_H, ep->rope_W, nt, nh, nw, 1};
            p.rope_L = ep->rope_F * ep->rope_H * ep->rope_W;
        }
    }
    LaunchCtx ctx;
    if (!op_ctx(reinterpret_cast<cudaStream_t>(stream), &ctx)) {
        if (tab) cudaFree(tab);
        return WAN_ECUDA;
    }
    cudaError_t e = wan::launch_gemm(A, lda, W, ldw, M, N, K, p, ctx);
    if (tab) {  // the table is freed once the kernel that reads it has run
        cudaStreamSynchronize(ctx.stream);
        cudaFree(tab);
    }
    return op_status(e);
}

wan_status wan_op_attention_qnorm(const void* q, int64_t ldq, const void* k, int64_t ldk, const void* v, int64_t ldv,
                                  void* o, int64_t ldo, int B, int heads, int Lq, int Lk, const float* q_ssq,
                                  int64_t ssq_ld, int ngroups, float eps, void* stream) {
    if (!q || !k || !v || !o || !q_ssq) return WAN_EINVAL;
    if (B < 0 || heads <= 0 || Lq < 0 || Lk <= 0 || ngroups <= 0 || ssq_ld < ngroups) return WAN_ESHAPE;
    LaunchCtx ctx;
    if (!op_ctx(reinterpret_cast<cudaStream_t>(stream), &ctx)) return WAN_ECUDA;
    const wan::RowNorm rn{q_ssq, ssq_ld, ngroups, 1.0f / (128.0f * heads), eps};
    return op_status(wan::launch_attention(q, ldq, k, ldk, v, ldv, o, ldo, B, heads, Lq, Lk, ctx, rn));
}

wan_status wan_op_rms_apply(void* buf, int64_t ld, int rows, int D, const float* ssq, int64_t ssq_ld, int ngroups,
                            float eps, void* stream) {
    if (!buf || !ssq) return WAN_EINVAL;
    if (ngroups <= 0 || ssq_ld < ngroups || rows < 0 || D <= 0) return WAN_ESHAPE;
    LaunchCtx ctx;
    if (!op_ctx(reinterpret_cast<cudaStream_t>(stream), &ctx)) return WAN_ECUDA;
    const wan::RowNorm rn{ssq, ssq_ld, ngroups, 1.0f / D, eps};
    return op_status(wan::launch_rms_apply(buf, ld, rows, D, rn, ctx));
}

wan_status wan_op_attention(const void* q, int64_t ldq, const void* k, int64_t ldk, const void* v, int64_t ldv, void* o,
                            int64_t ldo, int B, int heads, int Lq, int Lk, void* stream) {
    if (!q || !k || !v || !o) return WAN_EINVAL;
    if (B < 0 || heads <= 0 || Lq < 0 || Lk <= 0) return WAN_ESHAPE;
    LaunchCtx ctx;
    if (!op_ctx(reinterpret_cast<cudaStream_t>(stream), &ctx)) return WAN_ECUDA;
    return op_status(wan::launch_attention(q, ldq, k, ldk, v, ldv, o, ldo, B, heads, Lq, Lk, ctx));
}

wan_status wan_op_layernorm(const void* x, void* y, int rows, int D, float eps, int mode, const float* gamma,
                            const float* beta, const float* shift0, const float* shift1, const float* scale0,
                            const float* scale1, int mod_div, int64_t mod_ld, void* stream) {
    if (!x || !y) return WAN_EINVAL;
    if (mode == 0 && (!shift0 || !shift1 || !scale0 || !scale1)) return WAN_EINVAL;
    if (mode == 1 && (!gamma || !beta)) return WAN_EINVAL;
    if (mode == 2 && (!shift1 || !scale1)) return WAN_EINVAL;
    if (mode != 0 && mode != 1 && mode != 2) return WAN_EINVAL;
    LaunchCtx ctx;
    if (!op_ctx(reinterpret_cast<cudaStream_t>(stream), &ctx)) return WAN_ECUDA;
    return op_status(
        wan::launch_layernorm(x, y, rows, D, eps, mode, gamma, beta, shift0, shift1, scale0, scale1, mod_div, mod_ld, ctx));
}

wan_status wan_op_rmsnorm_rope(void* buf, int64_t ld, int rows, int D, float eps, const float* gain, int rope, int Fp,
                               int Hp, int Wp, int rope_t, int rope_h, int rope_w, float theta, void* stream) {
    if (!buf || !gain) return WAN_EINVAL;
    LaunchCtx ctx;
    if (!op_ctx(reinterpret_cast<cudaStream_t>(stream), &ctx)) return WAN_ECUDA;
    if (!rope) return op_status(wan::launch_rmsnorm_rope(buf, ld, rows, D, eps, gain, 0, 1, 0, nullptr, 0, ctx));
    if (Fp <= 0 || Hp <= 0 || Wp <= 0 || rope_t % 2 || rope_h % 2 || rope_w % 2 || rope_t + rope_h + rope_w != 128)
        return WAN_ESHAPE;
    wan_dit_config c{};
    c.rope_t = rope_t;
    c.rope_h = rope_h;
    c.rope_w = rope_w;
    c.rope_theta = theta;
    std::vector<float2> tab;
    int nt, nh, nw;
    rope_tables_host(c, Fp, Hp, Wp, tab, nt, nh, nw);
    float2* d = nullptr;
    if (cudaMalloc(&d, tab.size() * sizeof(float2)) != cudaSuccess) {
        cudaGetLastError();
        return WAN_ENOMEM;
    }
    if (cudaMemcpy(d, tab.data(), tab.size() * sizeof(float2), cudaMemcpyHostToDevice) != cudaSuccess) {
        cudaFree(d);
        return WAN_ECUDA;
    }
    wan::RopeTables rt{d, d + (size_t)Fp * nt, d + (size_t)Fp * nt + (size_t)Hp * nh, Fp, Hp, Wp, nt, nh, nw, 0};
    cudaError_t e = wan::launch_rmsnorm_rope(buf, ld, rows, D, eps, gain, 0, 1, 0, &rt, Fp * Hp * Wp, ctx);
    cudaStreamSynchronize(ctx.stream);
    cudaFree(d);
    return op_status(e);
}

wan_status wan_op_wait_selftest(int64_t limit_ns, void* stream) {
    LaunchCtx ctx;
    if (!op_ctx(reinterpret_cast<cudaStream_t>(stream), &ctx)) return WAN_ECUDA;
    const uint64_t lim = limit_ns < 1000 ? 1000ull : (limit_ns > 1000000000 ? 1000000000ull : (uint64_t)limit_ns);
    return op_status(wan::launch_wait_selftest(lim, ctx));
}

wan_status wan_op_cfg_euler(const float* x, const float* v_cond, const float* v_uncond, float guidance, float sigma,
                            float sigma_next, int64_t n, float* x_next, void* stream) {
    if (!x || !v_cond || !x_next) return WAN_EINVAL;
    if (n < 0) return WAN_ESHAPE;
    LaunchCtx ctx;
    if (!op_ctx(reinterpret_cast<cudaStream_t>(stream), &ctx)) return WAN_ECUDA;
    return op_status(wan::launch_cfg_euler(x, v_cond, v_uncond, guidance, sigma, sigma_next, n, x_next, ctx));
}

wan_status wan_op_patchify(const void* latent, int latent_dtype, int B, int C, int F, int Hz, int Wz, void* X,
                           void* stream) {
    if (!latent || !X) return WAN_EINVAL;
    if (B < 0 || C <= 0 || F <= 0 || Hz % 2 || Wz % 2 || Hz <= 0 || Wz <= 0) return WAN_ESHAPE;
    LaunchCtx ctx;
    if (!op_ctx(reinterpret_cast<cudaStream_t>(stream), &ctx)) return WAN_ECUDA;
    return op_status(wan::launch_patchify(latent, latent_dtype, B, C, F, Hz, Wz, X, 4 * C, ctx));
}

wan_status wan_op_causal_conv3d(const void* x, const void* cache, int nc, int B, int T, int H, int W, int Ci,
                                const void* w, int64_t ldw, const float* bias, int Co, int kt, int kh, int kw, void* col,
                                int64_t col_elems, void* y, void* stream) {
    if (!x || !w || !col || !y) return WAN_EINVAL;
    if (B <= 0 || T <= 0 || H <= 0 || W <= 0 || Ci <= 0 || Co <= 0) return WAN_ESHAPE;
    if (kt <= 0 || kh <= 0 || kw <= 0 || !(kt & 1) || !(kh & 1) || !(kw & 1)) return WAN_ESHAPE;
    if (Ci % 8 || Co % 64 || nc < 0 || nc > kt - 1 || (nc > 0 && !cache)) return WAN_ESHAPE;
    const long long K = (long long)kt * kh * kw * Ci, Kp = (K + 63) / 64 * 64;
    if (ldw != Kp || Kp > (1LL << 30)) return WAN_ESHAPE;
    const long long M = (long long)B * T * H * W;
    if (M > (1LL << 31) - 1 || col_elems < M * Kp) return WAN_ESHAPE;
    if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(col) | reinterpret_cast<uintptr_t>(w) |
         reinterpret_cast<uintptr_t>(y) | reinterpret_cast<uintptr_t>(cache)) & 15)
        return WAN_EINVAL;
    LaunchCtx ctx;
    if (!op_ctx(reinterpret_cast<cudaStream_t>(stream), &ctx)) return WAN_ECUDA;
    cudaError_t e = wan::launch_causal_im2col(x, nc > 0 ? cache : nullptr, nc, B, T, H, W, Ci, kt, kh, kw, col, (int)Kp, ctx);
    if (e != cudaSuccess) return op_status(e);
    EpiParams p{};
    p.kind = wan::EPI_BIAS;
    p.bias = bias;
    p.out = y;
    p.ldo = Co;
    p.mod_div = 1;
    return op_status(wan::launch_gemm(col, Kp, w, Kp, (int)M, Co, (int)Kp, p, ctx));
}

wan_status wan_op_conv3d(const void* x, const void* cache, int nc, int B, int T, int H, int W, int Ci, const void* w,
                         int64_t ldw, const float* bias, int Co, int Co_pad, int kt, int kh, int kw, void* y, int64_t ldy,
                         const void* add, int64_t ldadd, int time_split, void* stream) {
    if (!x || !w || !y) return WAN_EINVAL;
    if (B <= 0 || T <= 0 || H <= 0 || W <= 0 || Ci <= 0 || Co <= 0) return WAN_ESHAPE;
    if (time_split && add) return WAN_EINVAL;
    wan::ConvEpi e{};
    e.kind = time_split ? wan::CONV_EPI_TIME_SPLIT : (add ? wan::CONV_EPI_ADD : wan::CONV_EPI_BIAS);
    e.bias = bias;
    e.y = reinterpret_cast<__nv_bfloat16*>(y);
    e.ldy = ldy;
    e.add = reinterpret_cast<const __nv_bfloat16*>(add);
    e.ldadd = ldadd;
    e.csplit = time_split ? Co / 2 : 0;
    LaunchCtx ctx;
    if (!op_ctx(reinterpret_cast<cudaStream_t>(stream), &ctx)) return WAN_ECUDA;
    return op_status(wan::launch_conv3d(x, cache, nc, B, T, H, W, Ci, w, ldw, Co, Co_pad, kt, kh, kw, e, ctx));
}

wan_status wan_op_unpatchify(const float* rows, int B, int C, int F, int Hz, int Wz, float* velocity, void* stream) {
    if (!rows || !velocity) return WAN_EINVAL;
    if (B < 0 || C <= 0 || F <= 0 || Hz % 2 || Wz % 2 || Hz <= 0 || Wz <= 0) return WAN_ESHAPE;
    LaunchCtx ctx;
    if (!op_ctx(reinterpret_cast<cudaStream_t>(stream), &ctx)) return WAN_ECUDA;
    return op_status(wan::launch_unpatchify(rows, B, C, F, Hz, Wz, velocity, ctx));
}

}  // extern "C"

// wan_op_rmsnorm_rope_noalloc: the RMSNorm-across-heads + 3-axis RoPE op with
// its cos/sin table in a fixed device array instead of a cudaMalloc'd buffer.
//
// For callers that must not allocate device memory while they run: serving
// stacks whose pool allocator owns (nearly) all of HBM, so an allocation from a
// library fails or breaks their accounting, and latency-critical loops that
// cannot afford the implicit synchronisation cudaMalloc / cudaFree may cause.
// The caller still passes the data buffer and the gain; the library neither
// allocates nor frees anything on this path.
//
// The table lives in g_rope_table, a file-scope __device__ array of
// kMaxRopePositions * 64 float2 (512 KiB) that every GPU loading this library
// keeps until the process exits.  Host code only knows a stand-in for that
// symbol, so the device address is fetched with cudaGetSymbolAddress once per
// device (on the first call made with that device current) and cached.
#include <cmath>
#include <mutex>

#include "../../include/wandit.h"
#include "../../include/wandit_ops.h"
#include "kernels.h"

namespace wan {
namespace {

// Positions per axis the table holds: the rope_max_seq_len of the Wan configs.
constexpr int kMaxRopePositions = 1024;
constexpr int kMaxPairs = 64;  // head_dim 128 -> 64 rotation pairs across the three axes
constexpr int kMaxDevices = 64;

__device__ __align__(256) float2 g_rope_table[kMaxRopePositions * kMaxPairs];

std::mutex g_mu;
float2* g_table_addr[kMaxDevices] = {};

// Device address of g_rope_table on the current device (set-up on first use).
float2* table_address() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_table_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_rope_table) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        g_table_addr[dev] = static_cast<float2*>(p);
    }
    return g_table_addr[dev];
}

// cos/sin of pos * theta^(-2k/d_a) for the three axes, written back to back
// (t | h | w), computed in double precision.
__global__ void fill_rope_table(float2* tab, int Fp, int Hp, int Wp, int dt, int dh, int dw, double log_theta) {
    const int nt = dt / 2, nh = dh / 2, nw = dw / 2;
    const int total = Fp * nt + Hp * nh + Wp * nw;
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < total; e += gridDim.x * blockDim.x) {
        int pos, k, d_a;
        if (e < Fp * nt) {
            pos = e / nt; k = e - pos * nt; d_a = dt;
        } else if (e < Fp * nt + Hp * nh) {
            const int x = e - Fp * nt;
            pos = x / nh; k = x - pos * nh; d_a = dh;
        } else {
            const int x = e - Fp * nt - Hp * nh;
            pos = x / nw; k = x - pos * nw; d_a = dw;
        }
        const double ang = pos * exp(-2.0 * k / d_a * log_theta);
        tab[e] = make_float2((float)cos(ang), (float)sin(ang));
    }
}

}  // namespace
}  // namespace wan

extern "C" wan_status wan_op_rmsnorm_rope_noalloc(void* buf, int64_t ld, int rows, int D, float eps, const float* gain,
                                                  int rope, int Fp, int Hp, int Wp, int rope_t, int rope_h, int rope_w,
                                                  float theta, void* stream) {
    using namespace wan;
    if (!buf || !gain) return WAN_EINVAL;
    // every shape check comes before the table is touched or anything is launched
    if (!rmsnorm_rope_shape_ok(D, ld)) return WAN_ESHAPE;
    if (rope && (Fp <= 0 || Hp <= 0 || Wp <= 0 || rope_t % 2 || rope_h % 2 || rope_w % 2 ||
                 rope_t + rope_h + rope_w != 128 || !(theta > 0.f)))
        return WAN_ESHAPE;
    // the fixed table holds kMaxRopePositions positions per axis
    if (rope && (Fp > kMaxRopePositions || Hp > kMaxRopePositions || Wp > kMaxRopePositions)) return WAN_ESHAPE;
    if (rows <= 0) return WAN_OK;
    // an error already pending on this thread is the caller's: report it, launch nothing
    if (cudaPeekAtLastError() != cudaSuccess) return WAN_ECUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess) return WAN_ECUDA;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    LaunchCtx ctx{st, nullptr, 0, sms, nullptr};
    if (!rope) {
        cudaError_t e = launch_rmsnorm_rope(buf, ld, rows, D, eps, gain, 0, 1, 0, nullptr, 0, ctx);
        return e == cudaSuccess ? WAN_OK : (e == cudaErrorInvalidValue ? WAN_ESHAPE : WAN_ECUDA);
    }
    float2* tab = table_address();
    if (!tab) return WAN_ECUDA;
    const int nt = rope_t / 2, nh = rope_h / 2, nw = rope_w / 2;
    const int total = Fp * nt + Hp * nh + Wp * nw;
    fill_rope_table<<<(total + 255) / 256, 256, 0, st>>>(tab, Fp, Hp, Wp, rope_t, rope_h, rope_w,
                                                         std::log((double)theta));
    if (cudaPeekAtLastError() != cudaSuccess) return WAN_ECUDA;
    RopeTables rt{tab, tab + (size_t)Fp * nt, tab + (size_t)Fp * nt + (size_t)Hp * nh, Fp, Hp, Wp, nt, nh, nw, 0};
    cudaError_t e = launch_rmsnorm_rope(buf, ld, rows, D, eps, gain, 0, 1, 0, &rt, Fp * Hp * Wp, ctx);
    return e == cudaSuccess ? WAN_OK : (e == cudaErrorInvalidValue ? WAN_ESHAPE : WAN_ECUDA);
}

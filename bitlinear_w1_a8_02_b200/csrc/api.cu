// C ABI of the BitLinear W1.58A8 library (declared in include/bitlinear.h).
//
// Each entry point validates its arguments on the host, carves its workspace,
// and launches kernels on the caller's stream. Nothing here allocates device
// memory, synchronises (except where the header says so) or lets a C++
// exception escape.
#include <bitlinear.h>

#include <atomic>

#include <cuda_runtime.h>

#include <algorithm>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

#define BL_API extern "C" __attribute__((visibility("default")))

namespace {

constexpr int64_t kMaxM = 65535;           // tokens per call (grid.y of the per-token kernels)
constexpr int64_t kMaxK = 262144;          // keeps the field-scaled int32 accumulators exact
constexpr int64_t kMaxN = int64_t(1) << 24;
constexpr size_t kWsAlign = 256;

inline size_t align_up(size_t v) { return (v + kWsAlign - 1) / kWsAlign * kWsAlign; }
inline bool aligned(const void* p, size_t a) { return (uintptr_t)p % a == 0; }

// Workspace carving -----------------------------------------------------------
// A tensor-core projection (M > 16) whose shape takes the stream-K split needs
// scratch for the pieces of split tiles; other shapes and the smaller paths do
// not. The split is decided, and the scratch sized, for 148 SMs without asking
// the device (workspace sizes are host-only arithmetic); a device with more SMs
// finds the scratch too small and keeps the data-parallel split.
constexpr int kStreamKSms = 148;
inline size_t sk_bytes(int64_t M, int64_t N, int64_t K) {
    return M > 16 && bl::gemm_use_stream_k(M, N, K, kStreamKSms)
               ? align_up(bl::gemm_sk_workspace_bytes(kStreamKSms))
               : 0;
}

struct ForwardWs {
    size_t xq, scale, xsum, sk, sk_bytes, total;
};
inline ForwardWs forward_ws(int64_t M, int64_t N, int64_t K) {
    ForwardWs w;
    w.xq = 0;
    w.scale = align_up((size_t)(M * K));
    w.xsum = w.scale + align_up((size_t)M * 4);
    w.sk = w.xsum + align_up((size_t)M * 4);
    w.sk_bytes = sk_bytes(M, N, K);
    w.total = w.sk + w.sk_bytes;
    return w;
}

struct FfnWs {
    size_t xq, scale, xsum, g, u, q2, s2, xsum2, sk, sk_bytes, total;
};
inline FfnWs ffn_ws(int64_t M, int64_t f, int64_t d) {
    FfnWs w;
    w.xq = 0;
    w.scale = align_up((size_t)(M * d));
    w.xsum = w.scale + align_up((size_t)M * 4);
    w.g = w.xsum + align_up((size_t)M * 4);
    w.u = w.g + align_up((size_t)(M * f) * 4);
    w.q2 = w.u + align_up((size_t)(M * f) * 4);
    w.s2 = w.q2 + align_up((size_t)(M * f));
    w.xsum2 = w.s2 + align_up((size_t)M * 4);
    w.sk = w.xsum2 + align_up((size_t)M * 4);
    // the down projection (M, d, f); gate and up with the split only on paths
    // without the fused gate + up launch
    w.sk_bytes = std::max(sk_bytes(M, d, f), sk_bytes(M, f, d));
    w.total = w.sk + w.sk_bytes;
    return w;
}

// Tensor-parallel FFN pieces. Up (sizes M, fl, d): codes of x, then g and u of
// the rank's fl columns (fp32). Down (sizes M, d, fl): codes of the rank's
// columns, their sums, and fp32 scratch for the projection's discarded dequantised
// output (only its int32 accumulators are kept).
struct TpUpWs {
    size_t xq, scale, xsum, g, u, sk, sk_bytes, total;
};
inline TpUpWs tp_up_ws(int64_t M, int64_t fl, int64_t d) {
    TpUpWs w;
    w.xq = 0;
    w.scale = align_up((size_t)(M * d));
    w.xsum = w.scale + align_up((size_t)M * 4);
    w.g = w.xsum + align_up((size_t)M * 4);
    w.u = w.g + align_up((size_t)(M * fl) * 4);
    w.sk = w.u + align_up((size_t)(M * fl) * 4);
    w.sk_bytes = sk_bytes(M, fl, d);
    w.total = w.sk + w.sk_bytes;
    return w;
}
struct TpDownWs {
    size_t q2, xsum2, y32, sk, sk_bytes, total;
};
inline TpDownWs tp_down_ws(int64_t M, int64_t d, int64_t fl) {
    TpDownWs w;
    w.q2 = 0;
    w.xsum2 = align_up((size_t)(M * fl));
    w.y32 = w.xsum2 + align_up((size_t)M * 4);
    w.sk = w.y32 + align_up((size_t)(M * d) * 4);
    w.sk_bytes = sk_bytes(M, d, fl);
    w.total = w.sk + w.sk_bytes;
    return w;
}

inline size_t pack_ws(int64_t N, int64_t K) {
    return align_up((size_t)bl::absmean_blocks(N * K) * sizeof(double));
}

// Device check: the kernels are built for sm_100a only.
bl_status check_device() {
    static int cached[64];  // 0 unknown, 1 ok, 2 unsupported
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
        cudaGetLastError();
        return BL_ERR_UNSUPPORTED;
    }
    if (dev < 64 && cached[dev]) return cached[dev] == 1 ? BL_OK : BL_ERR_UNSUPPORTED;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        cudaGetLastError();
        return BL_ERR_UNSUPPORTED;
    }
    const bool ok = (major == 10 && minor == 0);
    if (dev < 64) cached[dev] = ok ? 1 : 2;
    return ok ? BL_OK : BL_ERR_UNSUPPORTED;
}

inline bl_status cuda_status(cudaError_t e) { return e == cudaSuccess ? BL_OK : BL_ERR_CUDA; }

#define BL_TRY(expr)                                  \
    do {                                              \
        cudaError_t _e = (expr);                      \
        if (_e != cudaSuccess) return BL_ERR_CUDA;    \
    } while (0)

bl_status check_ws(const void* ws, size_t ws_bytes, size_t need) {
    if (need == 0) return BL_OK;
    if (!ws) return BL_ERR_NULL;
    if (!aligned(ws, kWsAlign)) return BL_ERR_ALIGN;
    if (ws_bytes < need) return BL_ERR_WORKSPACE;
    return BL_OK;
}

// Which kernel runs a projection, and the activation-code layout it reads.
enum class Path { GemvFast, GemvGeneric, GemmTc, GemvTc, GemvLut };

// Process-wide choice of the M <= 16 kernel (bitlinear_set_gemv_kernel).
std::atomic<int> g_gemv_kernel{BL_GEMV_AUTO};

// Automatic choice for M <= 16: the streamed dp4a / mma.sync GEMV. Measured on
// B200 with cold weights, the tensor-core GEMV is slower or equal at every
// shape and token count (its weight stream stays near 2.3 TB/s: each 512-code
// stage touches 128 rows), so it runs only when selected.
inline bool prefer_gemv_tc(int64_t, int64_t, int64_t) { return false; }

// `x` is the bf16 input the codes are made from (the fast quantiser reads it
// 16 bytes at a time); null when the codes come from the FFN glue kernel.
inline Path choose_path(const uint8_t* Wp, int64_t N, int64_t K, int64_t M, const void* xq,
                        const void* x) {
    if (x && !aligned(x, 16)) return Path::GemvGeneric;
    if (M > 16 && bl::gemm_tc_ok(N, K, Wp, xq)) return Path::GemmTc;
    if (bl::gemv_fast_ok(N, K) && aligned(Wp, 16)) {
        const int kind = g_gemv_kernel.load(std::memory_order_relaxed);
        const bool tc_ok = bl::gemv_tc_ok(N, K, M, Wp, xq);
        if (kind == BL_GEMV_TENSOR && tc_ok) return Path::GemvTc;
        if (kind == BL_GEMV_LUT && bl::gemv_lut_ok(N, K, M, Wp, xq)) return Path::GemvLut;
        if (kind == BL_GEMV_AUTO && tc_ok && prefer_gemv_tc(N, K, M)) return Path::GemvTc;
        return Path::GemvFast;
    }
    return Path::GemvGeneric;
}

inline int layout_of(Path p) {
    return (p == Path::GemmTc || p == Path::GemvTc) ? bl::XQ_G16T
           : p == Path::GemvFast                     ? bl::XQ_PLANES
                                                     : bl::XQ_NATURAL;  // generic and lookup-table kernels
}

// One BitLinear projection of already-quantised codes `xq` (in layout_of(path)).
bl_status project(Path path, const uint8_t* Wp, const float* gamma, int64_t N, int64_t K,
                  const int8_t* xq, const float* scale, const int32_t* xsum, int64_t M,
                  const bl::GemvOut& out, cudaStream_t s, void* sk_ws, size_t sk_ws_bytes) {
    switch (path) {
        case Path::GemmTc:
            return cuda_status(
                bl::launch_gemm_tc(Wp, gamma, N, K, xq, scale, xsum, M, out, s, sk_ws, sk_ws_bytes));
        case Path::GemvFast:
            return cuda_status(bl::launch_gemv(Wp, gamma, N, K, xq, scale, xsum, M, out, s));
        case Path::GemvTc:
            return cuda_status(bl::launch_gemv_tc(Wp, gamma, N, K, xq, scale, xsum, M, out, s));
        case Path::GemvLut:
            return cuda_status(bl::launch_gemv_lut(Wp, gamma, N, K, xq, scale, M, out, s));
        default:
            return cuda_status(bl::launch_gemv_generic(Wp, gamma, N, K, xq, scale, M, out, s));
    }
}

}  // namespace

// ----------------------------------------------------------------------------
BL_API const char* bitlinear_status_string(bl_status st) {
    switch (st) {
        case BL_OK: return "BL_OK";
        case BL_ERR_NULL: return "BL_ERR_NULL: a required pointer is NULL";
        case BL_ERR_SHAPE: return "BL_ERR_SHAPE: invalid or unsupported sizes";
        case BL_ERR_ALIGN: return "BL_ERR_ALIGN: misaligned pointer";
        case BL_ERR_DTYPE: return "BL_ERR_DTYPE: unknown dtype";
        case BL_ERR_WORKSPACE: return "BL_ERR_WORKSPACE: workspace too small";
        case BL_ERR_UNSUPPORTED: return "BL_ERR_UNSUPPORTED: needs an sm_100 (B200) device";
        case BL_ERR_CUDA: return "BL_ERR_CUDA: a CUDA call or launch failed";
        case BL_ERR_TIMEOUT: return "BL_ERR_TIMEOUT: a bounded wait in a kernel gave up";
        case BL_ERR_BAD_CODE: return "BL_ERR_BAD_CODE: packed weights hold the invalid code 3";
    }
    return "unknown bl_status";
}

BL_API int bitlinear_set_gemv_kernel(int kind) {
    if (kind < BL_GEMV_AUTO || kind > BL_GEMV_LUT) return -1;
    return g_gemv_kernel.exchange(kind);
}

BL_API size_t bitlinear_workspace_bytes(int op, int64_t M, int64_t N, int64_t K) {
    if (M < 0 || N < 0 || K < 0) return 0;
    switch (op) {
        case BL_OP_PACK: return pack_ws(N, K);
        case BL_OP_FORWARD: return forward_ws(M, N, K).total;
        case BL_OP_FFN: return ffn_ws(M, N, K).total;
        case BL_OP_VALIDATE: return kWsAlign;
        case BL_OP_FFN_TP_UP: return tp_up_ws(M, N, K).total;
        case BL_OP_FFN_TP_DOWN: return tp_down_ws(M, N, K).total;
        default: return 0;
    }
}

BL_API bl_status bitlinear_pack_weights(const void* W, int wdt, int64_t N, int64_t K, uint8_t* Wp,
                                        float* gamma, void* ws, size_t ws_bytes,
                                        bl_stream_t stream) {
    if (wdt != BL_BF16 && wdt != BL_FP32) return BL_ERR_DTYPE;
    if (N < 1 || K < 4 || K % 4 != 0 || N > kMaxN || K > kMaxK) return BL_ERR_SHAPE;
    if (!W || !Wp || !gamma) return BL_ERR_NULL;
    if (!aligned(W, 16) || !aligned(gamma, 4)) return BL_ERR_ALIGN;
    if (bl_status st = check_ws(ws, ws_bytes, pack_ws(N, K))) return st;
    if (bl_status st = check_device()) return st;
    cudaStream_t s = (cudaStream_t)stream;
    const bool fp32 = wdt == BL_FP32;
    BL_TRY(bl::launch_absmean(W, fp32, N * K, (double*)ws, gamma, s));
    BL_TRY(bl::launch_ternary_pack(W, fp32, N, K, gamma, Wp, s));
    return BL_OK;
}

BL_API bl_status bitlinear_pack_weights_rowwise(const void* W, int wdt, int64_t N, int64_t K, uint8_t* Wp,
                                                float* gammas, bl_stream_t stream) {
    if (wdt != BL_BF16 && wdt != BL_FP32) return BL_ERR_DTYPE;
    if (N < 1 || K < 4 || K % 4 != 0 || N > kMaxN || K > kMaxK) return BL_ERR_SHAPE;
    if (!W || !Wp || !gammas) return BL_ERR_NULL;
    if (!aligned(W, 16) || !aligned(gammas, 4)) return BL_ERR_ALIGN;
    if (bl_status st = check_device()) return st;
    cudaStream_t s = (cudaStream_t)stream;
    const bool fp32 = wdt == BL_FP32;
    BL_TRY(bl::launch_absmean_rows(W, fp32, N, K, gammas, s));
    BL_TRY(bl::launch_ternary_pack(W, fp32, N, K, gammas, Wp, s, true));
    return BL_OK;
}

BL_API bl_status bitlinear_quant_act(const uint16_t* x, int64_t M, int64_t K, int8_t* xq,
                                     float* scale, int32_t* xsum, bl_stream_t stream) {
    if (M < 0 || M > kMaxM || K < 4 || K % 4 != 0 || K > kMaxK) return BL_ERR_SHAPE;
    if (M == 0) return BL_OK;
    if (!x || !xq || !scale) return BL_ERR_NULL;
    if (!aligned(x, 2) || !aligned(scale, 4) || (xsum && !aligned(xsum, 4))) return BL_ERR_ALIGN;
    if (bl_status st = check_device()) return st;
    return cuda_status(
        bl::launch_act_quant(x, M, K, bl::XQ_NATURAL, xq, scale, xsum, (cudaStream_t)stream));
}

namespace {

// The forward behind bitlinear_forward and bitlinear_forward_ex: `out` carries
// the row segments (gamma holds one value per segment), `rmsnorm` quantises the
// unit-weight RMSNorm of x instead of x.
bl_status forward_impl(const uint8_t* Wp, const float* gamma, int64_t N, int64_t K, const uint16_t* x,
                       int64_t M, bool rmsnorm, bl::GemvOut out, void* ws, size_t ws_bytes,
                       cudaStream_t s) {
    const ForwardWs w = forward_ws(M, N, K);
    if (bl_status st = check_ws(ws, ws_bytes, w.total)) return st;
    if (bl_status st = check_device()) return st;
    char* base = (char*)ws;
    int8_t* xq = (int8_t*)(base + w.xq);
    float* scale = (float*)(base + w.scale);
    int32_t* xsum = (int32_t*)(base + w.xsum);

    Path path = choose_path(Wp, N, K, M, xq, x);
    // segment ends that do not fall on the fast paths' tiles take the generic kernel
    if ((path == Path::GemmTc && !bl::gemm_segments_ok(out, N)) ||
        ((path == Path::GemvFast || path == Path::GemvTc) && !bl::gemv_segments_ok(out, N)))
        path = Path::GemvGeneric;
    // one kernel (quantise + GEMV) up to 4 tokens where that beats the separate act-quant
    if (path == Path::GemvFast && bl::gemv_fused_ok(M, K) && bl::gemv_fused_pays(M, N, K))
        return cuda_status(bl::launch_gemv(Wp, gamma, N, K, nullptr, nullptr, nullptr, M, out, s, x, rmsnorm));
    BL_TRY(bl::launch_act_quant(x, M, K, layout_of(path), xq, scale, xsum, s, rmsnorm));
    return project(path, Wp, gamma, N, K, xq, scale, xsum, M, out, s, base + w.sk, w.sk_bytes);
}

bool forward_args_ok(int64_t N, int64_t K, int64_t M) {
    return M >= 0 && M <= kMaxM && N >= 0 && N <= kMaxN && K >= 4 && K % 4 == 0 && K <= kMaxK;
}

}  // namespace

BL_API bl_status bitlinear_forward(const uint8_t* Wp, const float* gamma, int64_t N, int64_t K,
                                   const uint16_t* x, int64_t M, const uint16_t* residual,
                                   uint16_t* y, int32_t* acc, void* ws, size_t ws_bytes,
                                   bl_stream_t stream) {
    if (!forward_args_ok(N, K, M)) return BL_ERR_SHAPE;
    if (M == 0 || N == 0) return BL_OK;
    if (!Wp || !gamma || !x || !y) return BL_ERR_NULL;
    if (!aligned(gamma, 4) || !aligned(x, 2) || !aligned(y, 2) || (residual && !aligned(residual, 2)) ||
        (acc && !aligned(acc, 4)))
        return BL_ERR_ALIGN;
    bl::GemvOut out;
    out.y = y;
    out.residual = residual;
    out.acc = acc;
    return forward_impl(Wp, gamma, N, K, x, M, false, out, ws, ws_bytes, (cudaStream_t)stream);
}

BL_API bl_status bitlinear_forward_ex(const uint8_t* Wp, const float* gammas, const int64_t* seg_rows,
                                      int32_t nseg, int64_t K, const uint16_t* x, int64_t M, int32_t rmsnorm,
                                      const uint16_t* residual, uint16_t* y, int32_t* acc, void* ws,
                                      size_t ws_bytes, bl_stream_t stream) {
    if (nseg < 1 || nseg > 4 || (rmsnorm != 0 && rmsnorm != 1)) return BL_ERR_SHAPE;
    if (!seg_rows) return BL_ERR_NULL;
    bl::GemvOut out;
    int64_t N = 0;
    for (int i = 0; i < nseg; ++i) {
        if (seg_rows[i] < 1) return BL_ERR_SHAPE;
        N += seg_rows[i];
        if (N > kMaxN) return BL_ERR_SHAPE;
        if (i < nseg - 1) out.seg_end[i] = (int)N;
    }
    if (!forward_args_ok(N, K, M)) return BL_ERR_SHAPE;
    if (M == 0) return BL_OK;
    if (!Wp || !gammas || !x || !y) return BL_ERR_NULL;
    if (!aligned(gammas, 4) || !aligned(x, 2) || !aligned(y, 2) || (residual && !aligned(residual, 2)) ||
        (acc && !aligned(acc, 4)))
        return BL_ERR_ALIGN;
    out.y = y;
    out.residual = residual;
    out.acc = acc;
    return forward_impl(Wp, gammas, N, K, x, M, rmsnorm != 0, out, ws, ws_bytes, (cudaStream_t)stream);
}

BL_API bl_status bitlinear_forward_rowwise(const uint8_t* Wp, const float* gammas, int64_t N, int64_t K,
                                           const uint16_t* x, int64_t M, const uint16_t* residual, uint16_t* y,
                                           int32_t* acc, void* ws, size_t ws_bytes, bl_stream_t stream) {
    if (!forward_args_ok(N, K, M)) return BL_ERR_SHAPE;
    if (M == 0 || N == 0) return BL_OK;
    if (!Wp || !gammas || !x || !y) return BL_ERR_NULL;
    if (!aligned(gammas, 4) || !aligned(x, 2) || !aligned(y, 2) || (residual && !aligned(residual, 2)) ||
        (acc && !aligned(acc, 4)))
        return BL_ERR_ALIGN;
    bl::GemvOut out;
    out.y = y;
    out.residual = residual;
    out.acc = acc;
    out.per_row = 1;
    return forward_impl(Wp, gammas, N, K, x, M, false, out, ws, ws_bytes, (cudaStream_t)stream);
}

BL_API bl_status bitlinear_ffn(const uint8_t* Wg, const float* gg, const uint8_t* Wu,
                               const float* gu, const uint8_t* Wd, const float* gd, int64_t d,
                               int64_t f, const uint16_t* x, int64_t M, const uint16_t* residual,
                               uint16_t* y, void* ws, size_t ws_bytes, bl_stream_t stream) {
    if (M < 0 || M > kMaxM || d < 4 || d % 4 != 0 || f < 4 || f % 4 != 0 || d > kMaxK ||
        f > kMaxK)
        return BL_ERR_SHAPE;
    if (M == 0) return BL_OK;
    if (!Wg || !gg || !Wu || !gu || !Wd || !gd || !x || !y) return BL_ERR_NULL;
    if (!aligned(gg, 4) || !aligned(gu, 4) || !aligned(gd, 4) || !aligned(x, 2) || !aligned(y, 2) ||
        (residual && !aligned(residual, 2)))
        return BL_ERR_ALIGN;
    const FfnWs w = ffn_ws(M, f, d);
    if (bl_status st = check_ws(ws, ws_bytes, w.total)) return st;
    if (bl_status st = check_device()) return st;
    cudaStream_t s = (cudaStream_t)stream;
    char* base = (char*)ws;
    int8_t* xq = (int8_t*)(base + w.xq);
    float* scale = (float*)(base + w.scale);
    int32_t* xsum = (int32_t*)(base + w.xsum);
    float* g = (float*)(base + w.g);
    float* u = (float*)(base + w.u);
    int8_t* q2 = (int8_t*)(base + w.q2);
    float* s2 = (float*)(base + w.s2);
    int32_t* xsum2 = (int32_t*)(base + w.xsum2);

    // gate and up share one quantisation of x, so they must share a path
    Path up = choose_path(Wg, f, d, M, xq, x);
    if (choose_path(Wu, f, d, M, xq, x) != up) up = Path::GemvGeneric;
    const Path down = choose_path(Wd, d, f, M, q2, nullptr);
    if (up == Path::GemvFast && down == Path::GemvFast && bl::gemv_fused_ok(M, d) &&
        bl::gemv_fused_ok(M, f)) {
        // Two kernels: gate+up streamed together with h and its per-tile partials
        // as output (h in the g slot, partials in the u slot), then the down
        // projection with the RMSNorm + requantisation folded into its prologue.
        const size_t nparts = (size_t)((f + 15) / 16);
        double* part_ss = (double*)u;
        float* part_max = (float*)((char*)u + align_up((size_t)M * nparts * sizeof(double)));
        BL_TRY(bl::launch_ffn_up_fused(Wg, gg, Wu, gu, f, d, x, M, g, part_ss, part_max, s));
        bl::GemvOut od;
        od.y = y;
        od.residual = residual;
        return cuda_status(bl::launch_ffn_down_fused(Wd, gd, d, f, g, part_ss, part_max, M, od, s));
    }
    if (up == Path::GemmTc) {
        // M > 16: gate and up in one tensor-core launch whose epilogue writes h (in
        // the g slot) and per-tile partials of sum h^2 and max |h| (in the u slot);
        // then the subln + requantisation from the partials, and the down projection.
        const int nparts = bl::gemm_dual_parts(f);
        bl::FfnUpOut fo;
        fo.h = g;
        fo.part_ss = (double*)u;
        fo.part_max = (float*)((char*)u + align_up((size_t)M * nparts * sizeof(double)));
        BL_TRY(bl::launch_act_quant(x, M, d, bl::XQ_G16T, xq, scale, xsum, s));
        BL_TRY(bl::launch_gemm_tc_dual(Wg, gg, Wu, gu, f, d, xq, scale, xsum, M, fo, s));
        BL_TRY(bl::launch_ffn_requant_parts(g, fo.part_ss, fo.part_max, nparts, M, f, layout_of(down), q2, s2, xsum2, s));
        bl::GemvOut od;
        od.y = y;
        od.residual = residual;
        return project(down, Wd, gd, d, f, q2, s2, xsum2, M, od, s, base + w.sk, w.sk_bytes);
    }
    bl::GemvOut og;
    og.y32 = g;
    bl::GemvOut ou;
    ou.y32 = u;
    if (up == Path::GemvFast && bl::gemv_fused_ok(M, d)) {
        BL_TRY(bl::launch_gemv(Wg, gg, f, d, nullptr, nullptr, nullptr, M, og, s, x));
        BL_TRY(bl::launch_gemv(Wu, gu, f, d, nullptr, nullptr, nullptr, M, ou, s, x));
    } else {
        BL_TRY(bl::launch_act_quant(x, M, d, layout_of(up), xq, scale, xsum, s));
        if (bl_status st = project(up, Wg, gg, f, d, xq, scale, xsum, M, og, s, base + w.sk, w.sk_bytes))
            return st;
        if (bl_status st = project(up, Wu, gu, f, d, xq, scale, xsum, M, ou, s, base + w.sk, w.sk_bytes))
            return st;
    }
    BL_TRY(bl::launch_ffn_finalise(g, u, M, f, layout_of(down), q2, s2, xsum2, s));
    bl::GemvOut od;
    od.y = y;
    od.residual = residual;
    return project(down, Wd, gd, d, f, q2, s2, xsum2, M, od, s, base + w.sk, w.sk_bytes);
}

BL_API bl_status bitlinear_validate_packed(const uint8_t* Wp, int64_t N, int64_t K,
                                           int64_t* bad_count, void* ws, size_t ws_bytes,
                                           bl_stream_t stream) {
    if (N < 0 || K < 0 || K % 4 != 0) return BL_ERR_SHAPE;
    if (bad_count) *bad_count = 0;
    if (N == 0 || K == 0) return BL_OK;
    if (!Wp) return BL_ERR_NULL;
    if (bl_status st = check_ws(ws, ws_bytes, kWsAlign)) return st;
    if (bl_status st = check_device()) return st;
    cudaStream_t s = (cudaStream_t)stream;
    unsigned long long* cnt = (unsigned long long*)ws;
    BL_TRY(cudaMemsetAsync(cnt, 0, sizeof(*cnt), s));
    BL_TRY(bl::launch_count_bad_codes(Wp, N * (K / 4), cnt, s));
    unsigned long long host = 0;
    BL_TRY(cudaMemcpyAsync(&host, cnt, sizeof(host), cudaMemcpyDeviceToHost, s));
    BL_TRY(cudaStreamSynchronize(s));
    if (bad_count) *bad_count = (int64_t)host;
    return host ? BL_ERR_BAD_CODE : BL_OK;
}

BL_API bl_status bitlinear_get_device_error(bl_stream_t stream) {
    if (bl_status st = check_device()) return st;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return BL_ERR_CUDA;
    if (cudaGetLastError() != cudaSuccess) return BL_ERR_CUDA;
    unsigned v = 0;
    if (bl::read_and_clear_device_error(&v) != cudaSuccess) return BL_ERR_CUDA;
    return v ? BL_ERR_TIMEOUT : BL_OK;
}

// ---------------------------------------------------------------- tensor-parallel pieces

BL_API bl_status bitlinear_absmean_sum(const void* W, int wdt, int64_t N, int64_t K, double* sum, void* ws,
                                       size_t ws_bytes, bl_stream_t stream) {
    if (wdt != BL_BF16 && wdt != BL_FP32) return BL_ERR_DTYPE;
    if (N < 1 || K < 4 || K % 4 != 0 || N > kMaxN || K > kMaxK) return BL_ERR_SHAPE;
    if (!W || !sum) return BL_ERR_NULL;
    if (!aligned(W, 16) || !aligned(sum, 8)) return BL_ERR_ALIGN;
    if (bl_status st = check_ws(ws, ws_bytes, pack_ws(N, K))) return st;
    if (bl_status st = check_device()) return st;
    return cuda_status(bl::launch_absmean_sum(W, wdt == BL_FP32, N * K, (double*)ws, sum, (cudaStream_t)stream));
}

BL_API bl_status bitlinear_pack_weights_global(const void* W, int wdt, int64_t N, int64_t K, const double* total_sum,
                                               int64_t total_count, uint8_t* Wp, float* gamma, bl_stream_t stream) {
    if (wdt != BL_BF16 && wdt != BL_FP32) return BL_ERR_DTYPE;
    if (N < 1 || K < 4 || K % 4 != 0 || N > kMaxN || K > kMaxK || total_count < N * K) return BL_ERR_SHAPE;
    if (!W || !total_sum || !Wp || !gamma) return BL_ERR_NULL;
    if (!aligned(W, 16) || !aligned(total_sum, 8) || !aligned(gamma, 4)) return BL_ERR_ALIGN;
    if (bl_status st = check_device()) return st;
    cudaStream_t s = (cudaStream_t)stream;
    BL_TRY(bl::launch_gamma_from_sum(total_sum, total_count, gamma, s));
    BL_TRY(bl::launch_ternary_pack(W, wdt == BL_FP32, N, K, gamma, Wp, s));
    return BL_OK;
}

BL_API bl_status bitlinear_ffn_tp_up(const uint8_t* Wg, const float* gg, const uint8_t* Wu, const float* gu,
                                     int64_t d, int64_t fl, const uint16_t* x, int64_t M, float* h, double* ss,
                                     float* hmax, void* ws, size_t ws_bytes, bl_stream_t stream) {
    if (M < 0 || M > kMaxM || d < 4 || d % 4 != 0 || fl < 4 || fl % 4 != 0 || d > kMaxK || fl > kMaxN)
        return BL_ERR_SHAPE;
    if (M == 0) return BL_OK;
    if (!Wg || !gg || !Wu || !gu || !x || !h || !ss || !hmax) return BL_ERR_NULL;
    if (!aligned(gg, 4) || !aligned(gu, 4) || !aligned(x, 2) || !aligned(h, 4) || !aligned(ss, 8) ||
        !aligned(hmax, 4))
        return BL_ERR_ALIGN;
    const TpUpWs w = tp_up_ws(M, fl, d);
    if (bl_status st = check_ws(ws, ws_bytes, w.total)) return st;
    if (bl_status st = check_device()) return st;
    cudaStream_t s = (cudaStream_t)stream;
    char* base = (char*)ws;
    int8_t* xq = (int8_t*)(base + w.xq);
    float* scale = (float*)(base + w.scale);
    int32_t* xsum = (int32_t*)(base + w.xsum);
    float* g = (float*)(base + w.g);
    float* u = (float*)(base + w.u);
    Path up = choose_path(Wg, fl, d, M, xq, x);  // gate and up share the codes, so a path
    if (choose_path(Wu, fl, d, M, xq, x) != up) up = Path::GemvGeneric;
    BL_TRY(bl::launch_act_quant(x, M, d, layout_of(up), xq, scale, xsum, s));
    bl::GemvOut og;
    og.y32 = g;
    bl::GemvOut ou;
    ou.y32 = u;
    if (bl_status st = project(up, Wg, gg, fl, d, xq, scale, xsum, M, og, s, base + w.sk, w.sk_bytes)) return st;
    if (bl_status st = project(up, Wu, gu, fl, d, xq, scale, xsum, M, ou, s, base + w.sk, w.sk_bytes)) return st;
    return cuda_status(bl::launch_ffn_tp_hstats(g, u, M, fl, h, ss, hmax, s));
}

BL_API bl_status bitlinear_ffn_tp_down(const uint8_t* Wd, int64_t d, int64_t fl, int64_t f_total, const float* h,
                                       int64_t M, const double* ss_all, const float* hmax_all, int32_t* acc,
                                       float* s2, void* ws, size_t ws_bytes, bl_stream_t stream) {
    if (M < 0 || M > kMaxM || d < 1 || d > kMaxN || fl < 4 || fl % 4 != 0 || fl > kMaxK || f_total < fl)
        return BL_ERR_SHAPE;
    if (M == 0) return BL_OK;
    if (!Wd || !h || !ss_all || !hmax_all || !acc || !s2) return BL_ERR_NULL;
    if (!aligned(h, 4) || !aligned(ss_all, 8) || !aligned(hmax_all, 4) || !aligned(acc, 4) || !aligned(s2, 4))
        return BL_ERR_ALIGN;
    const TpDownWs w = tp_down_ws(M, d, fl);
    if (bl_status st = check_ws(ws, ws_bytes, w.total)) return st;
    if (bl_status st = check_device()) return st;
    cudaStream_t s = (cudaStream_t)stream;
    char* base = (char*)ws;
    int8_t* q2 = (int8_t*)(base + w.q2);
    int32_t* xsum2 = (int32_t*)(base + w.xsum2);
    const Path down = choose_path(Wd, d, fl, M, q2, nullptr);
    BL_TRY(bl::launch_ffn_tp_requant(h, M, fl, f_total, ss_all, hmax_all, layout_of(down), q2, s2, xsum2, s));
    // the projection dequantises into scratch (s2 stands in for gamma there: that
    // output is discarded); the partial sums over the rank's columns go to acc
    bl::GemvOut od;
    od.y32 = (float*)(base + w.y32);
    od.acc = acc;
    return project(down, Wd, s2, d, fl, q2, s2, xsum2, M, od, s, base + w.sk, w.sk_bytes);
}

BL_API bl_status bitlinear_ffn_tp_finish(const int32_t* acc, const float* gd, const float* s2,
                                         const uint16_t* residual, uint16_t* y, int64_t M, int64_t d,
                                         bl_stream_t stream) {
    if (M < 0 || M > kMaxM || d < 0 || d > kMaxN) return BL_ERR_SHAPE;
    if (M == 0 || d == 0) return BL_OK;
    if (!acc || !gd || !s2 || !y) return BL_ERR_NULL;
    if (!aligned(acc, 4) || !aligned(gd, 4) || !aligned(s2, 4) || !aligned(y, 2) ||
        (residual && !aligned(residual, 2)))
        return BL_ERR_ALIGN;
    if (bl_status st = check_device()) return st;
    return cuda_status(bl::launch_ffn_tp_finish(acc, gd, s2, residual, y, M, d, (cudaStream_t)stream));
}

// bitlinear_forward_noalloc: the BitLinear forward for callers that cannot
// allocate device memory and have no workspace to hand over.
//
// Who needs it: code that runs inside a host program or engine which reserves
// all device memory up front and forbids allocation afterwards (a cudaMalloc
// there can fail, or implicitly synchronise the device in the middle of a
// latency-critical serving loop), and plain C callers that have no caching
// allocator to borrow a workspace from. The regular bitlinear_forward asks for
// a caller-owned workspace; this variant keeps its scratch in a fixed array of
// the library's own device memory instead.
//
// The scratch (activation codes, per-token scales and code sums, exactly what
// bitlinear_forward puts in its workspace) lives in `g_noalloc_scratch`, a
// file-scope device array of kNoallocScratchBytes bytes. Every GPU that loads
// the library holds one copy until the process exits. In host code the array's
// name is only a host-side stand-in, so the entry point asks the runtime for the
// device address (cudaGetSymbolAddress) once per device, on that device's first
// call, and passes that address to the kernels. The address is cached together
// with the id of the CUDA context it belongs to: after a cudaDeviceReset the
// module is loaded again in a new context, the ids differ, and the next call
// looks the address up again instead of passing a stale pointer.
//
// Kernels: the separate act-quant kernel (PLANES codes when the streamed GEMV
// runs, natural codes for the generic kernel), then the GEMV, for every M. This
// differs from bitlinear_forward, which fuses the quantisation into the GEMV for
// M <= 4 and runs the tensor-core GEMM for M > 16; all of these paths compute
// the same integers and the same bf16 bits.
//
// All calls on a device share the one array and it keeps whatever the last call
// wrote. Nothing in it has to start at zero: every byte a call reads was written
// earlier in the same call. Two calls that can run at the same time on the GPU
// (different streams, or host threads without ordering between them) race on
// the array and may corrupt each other's results.
#include <bitlinear.h>

#include <atomic>

#include <cuda.h>  // CUcontext, CUresult (types only)
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

#define BL_API extern "C" __attribute__((visibility("default")))

// 1 MiB: room for the codes of 16 tokens at K = 28672 (or M*K up to ~1 MB).
static constexpr size_t kNoallocScratchBytes = size_t(1) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;

// Per device: the scratch array's device address and the id of the context it
// was looked up in (0: not looked up yet).
struct ScratchSlot {
    std::atomic<unsigned long long> ctx_id{0};
    std::atomic<void*> addr{nullptr};
};
ScratchSlot g_scratch[kMaxDevices];

inline size_t up256(size_t v) { return (v + 255) / 256 * 256; }
inline bool is_aligned(const void* p, size_t a) { return (uintptr_t)p % a == 0; }

// Unique id of the calling thread's current CUDA context (driver API, reached
// through the runtime's entry-point query so the library needs no -lcuda).
bool current_context_id(unsigned long long* id) {
    using GetCurrentFn = CUresult (*)(CUcontext*);
    using GetIdFn = CUresult (*)(CUcontext, unsigned long long*);
    static GetCurrentFn get_current = nullptr;
    static GetIdFn get_id = nullptr;
    if (!get_current || !get_id) {
        void* p1 = nullptr;
        void* p2 = nullptr;
        cudaDriverEntryPointQueryResult q1, q2;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p1, cudaEnableDefault, &q1) != cudaSuccess ||
            q1 != cudaDriverEntryPointSuccess ||
            cudaGetDriverEntryPoint("cuCtxGetId", &p2, cudaEnableDefault, &q2) != cudaSuccess ||
            q2 != cudaDriverEntryPointSuccess) {
            cudaGetLastError();
            return false;
        }
        get_current = reinterpret_cast<GetCurrentFn>(p1);
        get_id = reinterpret_cast<GetIdFn>(p2);
    }
    CUcontext ctx = nullptr;
    return get_current(&ctx) == CUDA_SUCCESS && ctx && get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of this device's scratch array, looked up on the first call in
// each context of the device (with the device current: the caller has checked it).
bl_status scratch_address(int dev, void** out) {
    unsigned long long ctx = 0;
    if (!current_context_id(&ctx)) return BL_ERR_CUDA;
    ScratchSlot& slot = g_scratch[dev];
    void* p = slot.addr.load(std::memory_order_acquire);
    if (!p || slot.ctx_id.load(std::memory_order_acquire) != ctx) {
        p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return BL_ERR_CUDA;
        }
        slot.addr.store(p, std::memory_order_release);
        slot.ctx_id.store(ctx, std::memory_order_release);
    }
    *out = p;
    return BL_OK;
}

bl_status device_is_sm100(int* dev_out) {
    int dev = -1, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        cudaGetLastError();
        return BL_ERR_UNSUPPORTED;
    }
    *dev_out = dev;
    return (major == 10 && minor == 0) ? BL_OK : BL_ERR_UNSUPPORTED;
}

}  // namespace

BL_API bl_status bitlinear_forward_noalloc(const uint8_t* Wp, const float* gamma, int64_t N,
                                           int64_t K, const uint16_t* x, int64_t M,
                                           const uint16_t* residual, uint16_t* y, int32_t* acc,
                                           bl_stream_t stream) {
    if (M < 0 || M > 65535 || N < 0 || N > (int64_t(1) << 24) || K < 4 || K % 4 != 0 ||
        K > 262144)
        return BL_ERR_SHAPE;
    if (M == 0 || N == 0) return BL_OK;
    if (!Wp || !gamma || !x || !y) return BL_ERR_NULL;
    if (!is_aligned(gamma, 4) || !is_aligned(x, 2) || !is_aligned(y, 2) ||
        (residual && !is_aligned(residual, 2)) || (acc && !is_aligned(acc, 4)))
        return BL_ERR_ALIGN;
    // Scratch carving: codes, then scales, then code sums, each 256-byte aligned.
    const size_t off_scale = up256((size_t)(M * K));
    const size_t off_xsum = off_scale + up256((size_t)M * 4);
    const size_t need = off_xsum + up256((size_t)M * 4);
    if (need > kNoallocScratchBytes) return BL_ERR_WORKSPACE;
    int dev = -1;
    if (bl_status st = device_is_sm100(&dev)) return st;
    void* base = nullptr;
    if (bl_status st = scratch_address(dev, &base)) return st;

    cudaStream_t s = (cudaStream_t)stream;
    int8_t* xq = (int8_t*)base;
    float* scale = (float*)((char*)base + off_scale);
    int32_t* xsum = (int32_t*)((char*)base + off_xsum);
    // the streamed GEMV reads PLANES codes, which the quantiser writes only from a
    // 16-byte aligned x; any other x takes the generic kernel on natural codes
    const bool fast = bl::gemv_fast_ok(N, K) && is_aligned(Wp, 16) && is_aligned(x, 16);
    if (bl::launch_act_quant(x, M, K, fast ? bl::XQ_PLANES : bl::XQ_NATURAL, xq, scale, xsum, s) !=
        cudaSuccess)
        return BL_ERR_CUDA;
    bl::GemvOut out;
    out.y = y;
    out.residual = residual;
    out.acc = acc;
    const cudaError_t e =
        fast ? bl::launch_gemv(Wp, gamma, N, K, xq, scale, xsum, M, out, s)
             : bl::launch_gemv_generic(Wp, gamma, N, K, xq, scale, M, out, s);
    return e == cudaSuccess ? BL_OK : BL_ERR_CUDA;
}

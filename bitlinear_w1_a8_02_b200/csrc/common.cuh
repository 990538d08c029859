// Device helpers shared by the library's kernels (sm_100a).
//
// Every fp32 step of the BitLinear arithmetic is written with an explicit
// round-to-nearest intrinsic (__fmul_rn, __fadd_rn, __fdiv_rn, __fsqrt_rn) so
// that no multiply-add is fused and every division and square root is the IEEE
// one; the results are then unique bit patterns.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace bl {

constexpr float kWeightEps = 1e-5f;  // eps in W / (gamma + eps)
constexpr float kActEps = 1e-5f;     // floor on the per-token absmax
constexpr float kActRange = 127.0f;  // per-token scale maps absmax to 127
constexpr float kRmsEps = 1e-5f;     // subln RMSNorm eps

// Activation code layouts the quantiser can write.
//   NATURAL : xq[m][k], row-major (the exported layout).
//   PLANES  : four planes per token; plane i holds xq[m][4j+i] at byte j.
//             Plane i of token m starts at (4m + i) * K/4. Matches the i-th
//             2-bit field of every packed weight byte.
//   G16T    : row-major, each group of 16 codes stored transposed as 4x4 bytes:
//             position 16c + 4i + b holds xq[m][16c + 4b + i]. Matches a packed
//             32-bit word unpacked field by field.
enum XqLayout : int { XQ_NATURAL = 0, XQ_PLANES = 1, XQ_G16T = 2 };

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) { return __uint_as_float(h << 16); }

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// Quantise one value with scale s: clip(rint(x * s), -128, 127).
//
// Rounding by magic-number addition: for |v| < 2^22, fp32 v + 1.5 * 2^23 lies in
// [2^23, 2^24), where the spacing of fp32 values is exactly 1, so the IEEE
// round-to-nearest-even of that one addition is rint(v) (ties to even) and the
// integer sits in the low mantissa bits: bits(v + 1.5 * 2^23) = 0x4B400000 + rint(v).
// The per-token scale guarantees |x * s| <= 127 * (1 + 2^-23), so the bound holds
// and the clip to [-128, 127] can never bite; it stays for non-finite inputs.
// This avoids the reduced-rate float-to-int conversion pipe.
__device__ __forceinline__ int quant_code(float x, float s) {
    const float t = __fadd_rn(__fmul_rn(x, s), 12582912.0f);
    const int q = static_cast<int>(__float_as_uint(t)) - 0x4B400000;
    return min(max(q, -128), 127);
}

// Dequantise: y32 = float(acc) * (gamma / s).
__device__ __forceinline__ float dequant(int acc, float deq) { return __fmul_rn((float)acc, deq); }

template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Block-wide reductions for blockDim.x == 32 * NW. The combination order is
// fixed (warp butterfly, then warps in index order), so results are
// reproducible run to run. `scratch` holds NW values; result broadcast to all.
template <int NW, typename T>
__device__ __forceinline__ T block_sum(T v, T* scratch) {
    v = warp_sum(v);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0) scratch[w] = v;
    __syncthreads();
    T r = scratch[0];
#pragma unroll
    for (int i = 1; i < NW; ++i) r += scratch[i];
    return r;
}

template <int NW>
__device__ __forceinline__ float block_max(float v, float* scratch) {
    v = warp_max(v);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0) scratch[w] = v;
    __syncthreads();
    float r = scratch[0];
#pragma unroll
    for (int i = 1; i < NW; ++i) r = fmaxf(r, scratch[i]);
    return r;
}

// Streaming 16-byte load that skips L1 (each weight byte is read once).
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// 16-byte read-only load through L1 (activation codes, reused by many warps).
__device__ __forceinline__ uint4 ld_nc16(const void* p) {
    return __ldg(reinterpret_cast<const uint4*>(p));
}

// Programmatic dependent launch: the kernel may start while the previous kernel
// in the stream is still running; it must call griddepcontrol.wait before it
// reads anything that kernel may write and before its first global store.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

__device__ __forceinline__ void grid_dependency_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void grid_dependents_launch() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace bl

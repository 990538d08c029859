// Per-token absmax activation quantisation to int8.
//
// Paper card "BitNet b1.58 2B4T Technical Report", "Method Adaptation":
// activations of the linear projections are quantised per token to 8-bit
// integers with absmax. Reading of the unstated constants:
//   s_m = 127 / max(max_k |x[m,k]|, 1e-5)     IEEE fp32 division
//   xq  = clip(rint(x * s_m), -128, 127)       one fp32 multiply, ties to even
//   xsum_m = sum_k xq[m,k]
//
// One CTA per token. Pass 1 reduces the absmax (order-free, so exact); pass 2
// re-reads the row (an L1/L2 hit) and writes 16 codes per thread in the layout
// the consumer wants (see XqLayout).
//
// Optional unit-weight RMSNorm in front (the transformer block's pre-norm and
// the subln before the attention output projection; paper card "Method
// Adaptation": subln): pass 1 also sums x^2 in fp64 (each square of a bf16 value
// is exact in fp64, but with outlier channels the squares span more than 53 bits,
// so the sum depends on the order in its last bits; the fp32 r below differs from
// a sequential sum's only if the two fp64 sums straddle an fp32 rounding
// boundary), r = 1 / sqrtf(float(sum / K) + 1e-5), and the codes are those of
// fl(x * r) with s = 127 / max(fl(max |x| * r), 1e-5) (rounding is monotonic,
// so max |fl(x r)| = fl(max |x| r)).
#include "common.cuh"
#include "kernels.h"

namespace bl {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ float absmax8(uint4 v) {
    float a = fabsf(__uint_as_float(v.x << 16));
    a = fmaxf(a, fabsf(__uint_as_float(v.x & 0xffff0000u)));
    a = fmaxf(a, fabsf(__uint_as_float(v.y << 16)));
    a = fmaxf(a, fabsf(__uint_as_float(v.y & 0xffff0000u)));
    a = fmaxf(a, fabsf(__uint_as_float(v.z << 16)));
    a = fmaxf(a, fabsf(__uint_as_float(v.z & 0xffff0000u)));
    a = fmaxf(a, fabsf(__uint_as_float(v.w << 16)));
    a = fmaxf(a, fabsf(__uint_as_float(v.w & 0xffff0000u)));
    return a;
}

__device__ __forceinline__ void unpack8(uint4 v, float* f) {
    f[0] = __uint_as_float(v.x << 16);
    f[1] = __uint_as_float(v.x & 0xffff0000u);
    f[2] = __uint_as_float(v.y << 16);
    f[3] = __uint_as_float(v.y & 0xffff0000u);
    f[4] = __uint_as_float(v.z << 16);
    f[5] = __uint_as_float(v.z & 0xffff0000u);
    f[6] = __uint_as_float(v.w << 16);
    f[7] = __uint_as_float(v.w & 0xffff0000u);
}

// Vector path: K % 16 == 0, x and xq 16-byte aligned.
__device__ __forceinline__ double sumsq8(uint4 v) {
    float f[8];
    unpack8(v, f);
    double ss = 0.0;
#pragma unroll
    for (int e = 0; e < 8; ++e) ss = __fma_rn((double)f[e], (double)f[e], ss);
    return ss;
}

// r of the optional RMSNorm from the row's sum of squares (in fp64).
__device__ __forceinline__ float rms_factor(double ss, int K) {
    const float ms = __double2float_rn(__ddiv_rn(ss, (double)K));
    return __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, kRmsEps)));
}

template <int LAYOUT>
__global__ void __launch_bounds__(kThreads) act_quant_vec_kernel(const uint16_t* __restrict__ x,
                                                                  int K, int8_t* __restrict__ xq,
                                                                  float* __restrict__ scale,
                                                                  int32_t* __restrict__ xsum, int norm) {
    __shared__ float fscratch[kWarps];
    __shared__ int iscratch[kWarps];
    __shared__ double dscratch[kWarps];
    grid_dependency_wait();
    grid_dependents_launch();
    const int m = blockIdx.x;
    const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)m * K);
    const int nvec = K / 8;

    float amax = 0.0f;
    double ss = 0.0;
    for (int i = threadIdx.x; i < nvec; i += kThreads) {
        const uint4 v = xr[i];
        amax = fmaxf(amax, absmax8(v));
        if (norm) ss += sumsq8(v);
    }
    amax = block_max<kWarps>(amax, fscratch);
    float r = 1.0f;
    if (norm) {
        r = rms_factor(block_sum<kWarps>(ss, dscratch), K);
        amax = __fmul_rn(amax, r);
    }
    const float s = __fdiv_rn(kActRange, fmaxf(amax, kActEps));

    const int KB = K / 4;
    int sum = 0;
    for (int c = threadIdx.x; c < K / 16; c += kThreads) {
        float f[16];
        unpack8(xr[2 * c], f);
        unpack8(xr[2 * c + 1], f + 8);
        if (norm) {
#pragma unroll
            for (int e = 0; e < 16; ++e) f[e] = __fmul_rn(f[e], r);
        }
        int q[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            q[e] = quant_code(f[e], s);
            sum += q[e];
        }
        if (LAYOUT == XQ_NATURAL) {
            uint4 o;
            o.x = (q[0] & 255) | (q[1] & 255) << 8 | (q[2] & 255) << 16 | (unsigned)(q[3] & 255) << 24;
            o.y = (q[4] & 255) | (q[5] & 255) << 8 | (q[6] & 255) << 16 | (unsigned)(q[7] & 255) << 24;
            o.z = (q[8] & 255) | (q[9] & 255) << 8 | (q[10] & 255) << 16 | (unsigned)(q[11] & 255) << 24;
            o.w = (q[12] & 255) | (q[13] & 255) << 8 | (q[14] & 255) << 16 | (unsigned)(q[15] & 255) << 24;
            reinterpret_cast<uint4*>(xq + (size_t)m * K)[c] = o;
        } else {
            // word i holds codes 4b + i of the group, b = 0..3
            unsigned w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                w[i] = (q[i] & 255) | (q[4 + i] & 255) << 8 | (q[8 + i] & 255) << 16 |
                       (unsigned)(q[12 + i] & 255) << 24;
            if (LAYOUT == XQ_G16T) {
                reinterpret_cast<uint4*>(xq + (size_t)m * K)[c] = make_uint4(w[0], w[1], w[2], w[3]);
            } else {  // XQ_PLANES: byte j = 4c + b of plane i
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    reinterpret_cast<unsigned*>(xq + ((size_t)m * 4 + i) * KB)[c] = w[i];
            }
        }
    }
    sum = block_sum<kWarps>(sum, iscratch);
    if (threadIdx.x == 0) {
        scale[m] = s;
        if (xsum) xsum[m] = sum;
    }
}

// Scalar path for any K % 4 == 0 and any alignment; NATURAL layout only.
__global__ void __launch_bounds__(kThreads) act_quant_scalar_kernel(const uint16_t* __restrict__ x,
                                                                     int K, int8_t* __restrict__ xq,
                                                                     float* __restrict__ scale,
                                                                     int32_t* __restrict__ xsum, int norm) {
    __shared__ float fscratch[kWarps];
    __shared__ int iscratch[kWarps];
    __shared__ double dscratch[kWarps];
    grid_dependency_wait();
    grid_dependents_launch();
    const int m = blockIdx.x;
    const uint16_t* xr = x + (size_t)m * K;
    float amax = 0.0f;
    double ss = 0.0;
    for (int k = threadIdx.x; k < K; k += kThreads) {
        const float f = bf16_bits_to_f32(xr[k]);
        amax = fmaxf(amax, fabsf(f));
        if (norm) ss = __fma_rn((double)f, (double)f, ss);
    }
    amax = block_max<kWarps>(amax, fscratch);
    float r = 1.0f;
    if (norm) {
        r = rms_factor(block_sum<kWarps>(ss, dscratch), K);
        amax = __fmul_rn(amax, r);
    }
    const float s = __fdiv_rn(kActRange, fmaxf(amax, kActEps));
    int sum = 0;
    for (int k = threadIdx.x; k < K; k += kThreads) {
        const float f = bf16_bits_to_f32(xr[k]);
        const int q = quant_code(norm ? __fmul_rn(f, r) : f, s);
        xq[(size_t)m * K + k] = (int8_t)q;
        sum += q;
    }
    sum = block_sum<kWarps>(sum, iscratch);
    if (threadIdx.x == 0) {
        scale[m] = s;
        if (xsum) xsum[m] = sum;
    }
}

}  // namespace

cudaError_t launch_act_quant(const uint16_t* x, int64_t M, int64_t K, int layout, int8_t* xq,
                             float* scale, int32_t* xsum, cudaStream_t s, bool rmsnorm) {
    const int norm = rmsnorm ? 1 : 0;
    if (M == 0) return cudaSuccess;
    const bool vec = (K % 16 == 0) && ((uintptr_t)x % 16 == 0) && ((uintptr_t)xq % 16 == 0);
    if (!vec) {
        if (layout != XQ_NATURAL) return cudaErrorInvalidValue;
        return launch_pdl(act_quant_scalar_kernel, dim3((unsigned)M), dim3(kThreads), 0, s, x, (int)K,
                          xq, scale, xsum, norm);
    }
    if (layout == XQ_NATURAL)
        return launch_pdl(act_quant_vec_kernel<XQ_NATURAL>, dim3((unsigned)M), dim3(kThreads), 0, s, x,
                          (int)K, xq, scale, xsum, norm);
    if (layout == XQ_PLANES)
        return launch_pdl(act_quant_vec_kernel<XQ_PLANES>, dim3((unsigned)M), dim3(kThreads), 0, s, x,
                          (int)K, xq, scale, xsum, norm);
    return launch_pdl(act_quant_vec_kernel<XQ_G16T>, dim3((unsigned)M), dim3(kThreads), 0, s, x, (int)K,
                      xq, scale, xsum, norm);
}

}  // namespace bl

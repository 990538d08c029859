// FFN glue between the gate/up projections and the down projection.
//
// Fishai news digest of the 2B4T report (BitLinear list) and the paper card
// "BitNet b1.58 2B4T Technical Report", "Method Adaptation": ReLU^2 in the FFN
// sub-layer and subln sub-layer normalisation. Reading of the unstated order:
//   h  = (max(g, 0))^2 * u                  products rounded to fp32
//   r  = 1 / sqrtf(float(sum_j h_j^2 / f) + 1e-5)   sum and division in fp64
//   hn = h * r                              unit RMSNorm weight, no bias
//   q2, s2 = per-token absmax int8 quantisation of hn (as for x)
//
// One CTA per token; h is kept in shared memory between the passes.
#include "common.cuh"
#include "kernels.h"

namespace bl {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

template <int LAYOUT>
__global__ void __launch_bounds__(kThreads) ffn_finalise_kernel(const float* __restrict__ g,
                                                                 const float* __restrict__ u, int f,
                                                                 int8_t* __restrict__ q2,
                                                                 float* __restrict__ s2,
                                                                 int32_t* __restrict__ xsum2) {
    extern __shared__ float hs[];
    __shared__ double dscratch[kWarps];
    __shared__ float fscratch[kWarps];
    __shared__ int iscratch[kWarps];
    grid_dependency_wait();
    grid_dependents_launch();
    const int m = blockIdx.x;
    const float* gr = g + (size_t)m * f;
    const float* ur = u + (size_t)m * f;

    double ss = 0.0;
    for (int j = threadIdx.x; j < f; j += kThreads) {
        const float gv = gr[j];
        const float t = gv > 0.0f ? gv : 0.0f;
        const float h = __fmul_rn(__fmul_rn(t, t), ur[j]);
        hs[j] = h;
        ss = __dadd_rn(ss, __dmul_rn((double)h, (double)h));
    }
    ss = block_sum<kWarps>(ss, dscratch);
    const float ms = __double2float_rn(__ddiv_rn(ss, (double)f));
    const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, kRmsEps)));

    float amax = 0.0f;
    for (int j = threadIdx.x; j < f; j += kThreads) {
        const float hn = __fmul_rn(hs[j], r);
        hs[j] = hn;
        amax = fmaxf(amax, fabsf(hn));
    }
    amax = block_max<kWarps>(amax, fscratch);
    const float s = __fdiv_rn(kActRange, fmaxf(amax, kActEps));

    int sum = 0;
    if (LAYOUT == XQ_NATURAL) {
        for (int j = threadIdx.x; j < f; j += kThreads) {
            const int q = quant_code(hs[j], s);
            q2[(size_t)m * f + j] = (int8_t)q;
            sum += q;
        }
    } else {
        const int fb = f / 4;
        for (int c = threadIdx.x; c < f / 16; c += kThreads) {
            unsigned w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
            for (int b = 0; b < 4; ++b)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int q = quant_code(hs[16 * c + 4 * b + i], s);
                    sum += q;
                    w[i] |= (unsigned)(q & 255) << (8 * b);
                }
            if (LAYOUT == XQ_G16T) {
                reinterpret_cast<uint4*>(q2 + (size_t)m * f)[c] = make_uint4(w[0], w[1], w[2], w[3]);
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    reinterpret_cast<unsigned*>(q2 + ((size_t)m * 4 + i) * fb)[c] = w[i];
            }
        }
    }
    sum = block_sum<kWarps>(sum, iscratch);
    if (threadIdx.x == 0) {
        s2[m] = s;
        xsum2[m] = sum;
    }
}

template <int LAYOUT>
cudaError_t launch_fin(const float* g, const float* u, int64_t M, int64_t f, int8_t* q2, float* s2,
                       int32_t* xsum2, cudaStream_t s) {
    const size_t smem = (size_t)f * sizeof(float);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(ffn_finalise_kernel<LAYOUT>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    return launch_pdl(ffn_finalise_kernel<LAYOUT>, dim3((unsigned)M), dim3(kThreads), smem, s, g, u,
                      (int)f, q2, s2, xsum2);
}

}  // namespace

cudaError_t launch_ffn_finalise(const float* g, const float* u, int64_t M, int64_t f, int layout,
                                int8_t* q2, float* s2, int32_t* xsum2, cudaStream_t s) {
    if (M == 0) return cudaSuccess;
    if (layout != XQ_NATURAL && f % 16 != 0) return cudaErrorInvalidValue;
    if (layout == XQ_PLANES) return launch_fin<XQ_PLANES>(g, u, M, f, q2, s2, xsum2, s);
    if (layout == XQ_G16T) return launch_fin<XQ_G16T>(g, u, M, f, q2, s2, xsum2, s);
    return launch_fin<XQ_NATURAL>(g, u, M, f, q2, s2, xsum2, s);
}

}  // namespace bl

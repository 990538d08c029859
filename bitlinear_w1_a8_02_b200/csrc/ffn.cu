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
// Separate gate and up projections (ffn_finalise_kernel): one CTA per token, h
// kept in shared memory between its passes. After the fused gate+up GEMM (more
// than 16 tokens), whose epilogue writes h and per-tile partials of sum h^2 and
// max |h|, ffn_requant_parts_kernel reduces the partials and requantises.
//
// Tensor-parallel pieces (a rank owns fl of the f hidden columns; the pages give
// no distributed detail, this is the library's split): h with the rank's share
// of the per-token statistics sum h^2 and max |h|; the requantisation of the
// rank's columns once those statistics are summed / maximised over the ranks;
// and the dequantisation of the down projection's int32 accumulators once they
// are summed over the ranks.
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

// ---------------------------------------------------------------- tensor-parallel pieces
// A rank owns fl of the f hidden columns. Its h, and per token its share of the
// subln statistics: ss = sum_j h_j^2 (fp64, fixed order: thread strides, warp
// butterfly, warps in index order) and hmax = max_j |h_j|.
__global__ void __launch_bounds__(kThreads) ffn_tp_hstats_kernel(const float* __restrict__ g,
                                                                  const float* __restrict__ u, int fl,
                                                                  float* __restrict__ h, double* __restrict__ ss,
                                                                  float* __restrict__ hmax) {
    __shared__ double dscratch[kWarps];
    __shared__ float fscratch[kWarps];
    grid_dependency_wait();
    grid_dependents_launch();
    const int m = blockIdx.x;
    double acc = 0.0;
    float mx = 0.0f;
    for (int j = threadIdx.x; j < fl; j += kThreads) {
        const float gv = g[(size_t)m * fl + j];
        const float t = gv > 0.0f ? gv : 0.0f;
        const float hv = __fmul_rn(__fmul_rn(t, t), u[(size_t)m * fl + j]);
        h[(size_t)m * fl + j] = hv;
        acc = __dadd_rn(acc, __dmul_rn((double)hv, (double)hv));
        mx = fmaxf(mx, fabsf(hv));
    }
    acc = block_sum<kWarps>(acc, dscratch);
    mx = block_max<kWarps>(mx, fscratch);
    if (threadIdx.x == 0) {
        ss[m] = acc;
        hmax[m] = mx;
    }
}

// Requantisation of token m's fl columns from the statistics of the whole row
// (ss = sum h^2 over all f_total columns, hmax = max |h|):
// r = 1 / sqrtf(float(ss / f_total) + 1e-5), s2 = 127 / max(fl(hmax r), 1e-5)
// (the largest |fl(h_j r)| of the row: rounding is monotonic and r > 0); writes the
// codes of fl(h_j r) in LAYOUT, s2[m] and the codes' sum over the fl columns.
template <int LAYOUT>
__device__ __forceinline__ void requant_row(const float* __restrict__ h, int m, int fl, int64_t f_total, double ss,
                                            float hmax, int8_t* __restrict__ q2, float* __restrict__ s2,
                                            int32_t* __restrict__ xsum2, int* iscratch) {
    const float ms = __double2float_rn(__ddiv_rn(ss, (double)f_total));
    const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, kRmsEps)));
    const float s = __fdiv_rn(kActRange, fmaxf(__fmul_rn(hmax, r), kActEps));
    const float* hr = h + (size_t)m * fl;
    int sum = 0;
    if (LAYOUT == XQ_NATURAL) {
        for (int j = threadIdx.x; j < fl; j += kThreads) {
            const int q = quant_code(__fmul_rn(hr[j], r), s);
            q2[(size_t)m * fl + j] = (int8_t)q;
            sum += q;
        }
    } else {
        const int fb = fl / 4;
        for (int c = threadIdx.x; c < fl / 16; c += kThreads) {
            unsigned w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
            for (int b = 0; b < 4; ++b)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int q = quant_code(__fmul_rn(hr[16 * c + 4 * b + i], r), s);
                    sum += q;
                    w[i] |= (unsigned)(q & 255) << (8 * b);
                }
            if (LAYOUT == XQ_G16T) {
                reinterpret_cast<uint4*>(q2 + (size_t)m * fl)[c] = make_uint4(w[0], w[1], w[2], w[3]);
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) reinterpret_cast<unsigned*>(q2 + ((size_t)m * 4 + i) * fb)[c] = w[i];
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
__global__ void __launch_bounds__(kThreads) ffn_tp_requant_kernel(const float* __restrict__ h, int fl, int64_t f_total,
                                                                   const double* __restrict__ ss_all,
                                                                   const float* __restrict__ hmax_all,
                                                                   int8_t* __restrict__ q2, float* __restrict__ s2,
                                                                   int32_t* __restrict__ xsum2) {
    __shared__ int iscratch[kWarps];
    grid_dependency_wait();
    grid_dependents_launch();
    const int m = blockIdx.x;
    requant_row<LAYOUT>(h, m, fl, f_total, ss_all[m], hmax_all[m], q2, s2, xsum2, iscratch);
}

// The FFN's subln and requantisation after the fused gate+up GEMM: the token's
// per-tile partials of sum h^2 (fp64) and max |h| reduced in a fixed order
// (thread strides, warp butterfly, warps in index order), then requant_row.
template <int LAYOUT>
__global__ void __launch_bounds__(kThreads) ffn_requant_parts_kernel(const float* __restrict__ h,
                                                                      const double* __restrict__ part_ss,
                                                                      const float* __restrict__ part_max, int nparts,
                                                                      int f, int8_t* __restrict__ q2,
                                                                      float* __restrict__ s2,
                                                                      int32_t* __restrict__ xsum2) {
    __shared__ double dscratch[kWarps];
    __shared__ float fscratch[kWarps];
    __shared__ int iscratch[kWarps];
    grid_dependency_wait();
    grid_dependents_launch();
    const int m = blockIdx.x;
    double ss = 0.0;
    float mx = 0.0f;
    for (int p = threadIdx.x; p < nparts; p += kThreads) {
        ss = __dadd_rn(ss, part_ss[(size_t)m * nparts + p]);
        mx = fmaxf(mx, part_max[(size_t)m * nparts + p]);
    }
    ss = block_sum<kWarps>(ss, dscratch);
    mx = block_max<kWarps>(mx, fscratch);
    requant_row<LAYOUT>(h, m, f, f, ss, mx, q2, s2, xsum2, iscratch);
}

// y = bf16([residual +] float(acc) * (gd / s2)) on the accumulators summed over the ranks.
__global__ void __launch_bounds__(kThreads) ffn_tp_finish_kernel(const int32_t* __restrict__ acc,
                                                                  const float* __restrict__ gd,
                                                                  const float* __restrict__ s2,
                                                                  const uint16_t* __restrict__ residual,
                                                                  uint16_t* __restrict__ y, int64_t M, int64_t d) {
    grid_dependency_wait();
    const float gamma = *gd;
    const int64_t n = M * d;
    for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n; i += (int64_t)gridDim.x * kThreads) {
        const int64_t m = i / d;
        float v = dequant(acc[i], __fdiv_rn(gamma, s2[m]));
        if (residual) v = __fadd_rn(bf16_bits_to_f32(residual[i]), v);
        y[i] = f32_to_bf16_bits(v);
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

cudaError_t launch_ffn_tp_hstats(const float* g, const float* u, int64_t M, int64_t fl, float* h, double* ss,
                                 float* hmax, cudaStream_t s) {
    if (M == 0) return cudaSuccess;
    return launch_pdl(ffn_tp_hstats_kernel, dim3((unsigned)M), dim3(kThreads), 0, s, g, u, (int)fl, h, ss, hmax);
}

cudaError_t launch_ffn_tp_requant(const float* h, int64_t M, int64_t fl, int64_t f_total, const double* ss_all,
                                  const float* hmax_all, int layout, int8_t* q2, float* s2, int32_t* xsum2,
                                  cudaStream_t s) {
    if (M == 0) return cudaSuccess;
    if (layout != XQ_NATURAL && fl % 16 != 0) return cudaErrorInvalidValue;
    const dim3 g((unsigned)M), b(kThreads);
    if (layout == XQ_PLANES)
        return launch_pdl(ffn_tp_requant_kernel<XQ_PLANES>, g, b, 0, s, h, (int)fl, f_total, ss_all, hmax_all, q2, s2,
                          xsum2);
    if (layout == XQ_G16T)
        return launch_pdl(ffn_tp_requant_kernel<XQ_G16T>, g, b, 0, s, h, (int)fl, f_total, ss_all, hmax_all, q2, s2,
                          xsum2);
    return launch_pdl(ffn_tp_requant_kernel<XQ_NATURAL>, g, b, 0, s, h, (int)fl, f_total, ss_all, hmax_all, q2, s2,
                      xsum2);
}

cudaError_t launch_ffn_requant_parts(const float* h, const double* part_ss, const float* part_max, int nparts,
                                     int64_t M, int64_t f, int layout, int8_t* q2, float* s2, int32_t* xsum2,
                                     cudaStream_t s) {
    if (M == 0) return cudaSuccess;
    if (layout != XQ_NATURAL && f % 16 != 0) return cudaErrorInvalidValue;
    const dim3 g((unsigned)M), b(kThreads);
    if (layout == XQ_PLANES)
        return launch_pdl(ffn_requant_parts_kernel<XQ_PLANES>, g, b, 0, s, h, part_ss, part_max, nparts, (int)f, q2,
                          s2, xsum2);
    if (layout == XQ_G16T)
        return launch_pdl(ffn_requant_parts_kernel<XQ_G16T>, g, b, 0, s, h, part_ss, part_max, nparts, (int)f, q2, s2,
                          xsum2);
    return launch_pdl(ffn_requant_parts_kernel<XQ_NATURAL>, g, b, 0, s, h, part_ss, part_max, nparts, (int)f, q2, s2,
                      xsum2);
}

cudaError_t launch_ffn_tp_finish(const int32_t* acc, const float* gd, const float* s2, const uint16_t* residual,
                                 uint16_t* y, int64_t M, int64_t d, cudaStream_t s) {
    if (M == 0 || d == 0) return cudaSuccess;
    int64_t blocks = (M * d + kThreads - 1) / kThreads;
    if (blocks > 148 * 16) blocks = 148 * 16;
    return launch_pdl(ffn_tp_finish_kernel, dim3((unsigned)blocks), dim3(kThreads), 0, s, acc, gd, s2, residual, y,
                      M, d);
}

cudaError_t launch_ffn_finalise(const float* g, const float* u, int64_t M, int64_t f, int layout,
                                int8_t* q2, float* s2, int32_t* xsum2, cudaStream_t s) {
    if (M == 0) return cudaSuccess;
    if (layout != XQ_NATURAL && f % 16 != 0) return cudaErrorInvalidValue;
    if (layout == XQ_PLANES) return launch_fin<XQ_PLANES>(g, u, M, f, q2, s2, xsum2, s);
    if (layout == XQ_G16T) return launch_fin<XQ_G16T>(g, u, M, f, q2, s2, xsum2, s);
    return launch_fin<XQ_NATURAL>(g, u, M, f, q2, s2, xsum2, s);
}

}  // namespace bl

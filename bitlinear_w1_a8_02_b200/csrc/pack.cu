// Absmean ternary weight quantisation and packing (one-time work per weight).
//
// Paper card "BitNet b1.58 2B4T Technical Report", "Method Adaptation": weights
// quantised with absmean onto {-1, 0, +1}; four ternary weights stored in one
// 8-bit value in HBM.
//
//   gamma = fp32( sum |W| / (N*K) ), the sum and the division in fp64
//   q     = clip(rint(W / (gamma + 1e-5)), -1, 1), one IEEE fp32 division
//   byte j of row n = sum_i (q[n][4j+i] + 1) << 2i
// Per-row variant: gamma_n = fp32( sum_k |W[n, k]| / K ) (fp64 sum and division),
// and row n is ternarised with its own gamma_n.
#include "common.cuh"
#include "kernels.h"

namespace bl {
namespace {

constexpr int kPackThreads = 256;
constexpr int kAbsmeanMaxBlocks = 1184;  // 8 blocks per SM on 148 SMs

template <bool FP32>
__device__ __forceinline__ float load_w(const void* W, int64_t i) {
    if (FP32) return reinterpret_cast<const float*>(W)[i];
    return bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(W)[i]);
}

// Grid-stride fp64 sum of |W|; one partial per block, combined in a fixed order.
template <bool FP32>
__global__ void __launch_bounds__(kPackThreads) absmean_partial_kernel(const void* __restrict__ W,
                                                                       int64_t n,
                                                                       double* __restrict__ partial) {
    __shared__ double scratch[kPackThreads / 32];
    double acc = 0.0;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
        acc = __dadd_rn(acc, fabs((double)load_w<FP32>(W, i)));
    acc = block_sum<kPackThreads / 32>(acc, scratch);
    if (threadIdx.x == 0) partial[blockIdx.x] = acc;
}

// One warp: lane l sums partials l, l+32, ... in order; then a fixed butterfly.
__global__ void absmean_final_kernel(const double* __restrict__ partial, int nblocks, int64_t n,
                                     float* __restrict__ gamma) {
    double acc = 0.0;
    for (int i = threadIdx.x; i < nblocks; i += 32) acc = __dadd_rn(acc, partial[i]);
    acc = warp_sum(acc);
    if (threadIdx.x == 0) *gamma = __double2float_rn(__ddiv_rn(acc, (double)n));
}

// The fp64 sum itself (one shard's term of a per-tensor absmean split over ranks).
__global__ void absmean_sum_kernel(const double* __restrict__ partial, int nblocks, double* __restrict__ sum) {
    double acc = 0.0;
    for (int i = threadIdx.x; i < nblocks; i += 32) acc = __dadd_rn(acc, partial[i]);
    acc = warp_sum(acc);
    if (threadIdx.x == 0) *sum = acc;
}

// gamma of a whole tensor from the fp64 sum and the count of all its shards.
__global__ void gamma_from_sum_kernel(const double* __restrict__ total_sum, int64_t count,
                                      float* __restrict__ gamma) {
    *gamma = __double2float_rn(__ddiv_rn(*total_sum, (double)count));
}

// Per-row absmean: one CTA per row, fp64 sum in a fixed order (thread strides,
// warp butterfly, warps in index order).
template <bool FP32>
__global__ void __launch_bounds__(kPackThreads) absmean_rows_kernel(const void* __restrict__ W, int64_t K,
                                                                    float* __restrict__ gammas) {
    __shared__ double scratch[kPackThreads / 32];
    const int64_t row = blockIdx.x;
    double acc = 0.0;
    for (int64_t k = threadIdx.x; k < K; k += kPackThreads)
        acc = __dadd_rn(acc, fabs((double)load_w<FP32>(W, row * K + k)));
    acc = block_sum<kPackThreads / 32>(acc, scratch);
    if (threadIdx.x == 0) gammas[row] = __double2float_rn(__ddiv_rn(acc, (double)K));
}

// One packed byte (four weights) per thread. gamma: one value, or one per row
// (ROWS) for row-major bytes of KB per row.
template <bool FP32, bool ROWS>
__global__ void __launch_bounds__(kPackThreads) ternary_pack_kernel(const void* __restrict__ W,
                                                                    int64_t nbytes, int64_t KB,
                                                                    const float* __restrict__ gamma,
                                                                    uint8_t* __restrict__ Wp) {
    const float d0 = ROWS ? 0.0f : __fadd_rn(*gamma, kWeightEps);
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < nbytes; j += stride) {
        const float d = ROWS ? __fadd_rn(gamma[j / KB], kWeightEps) : d0;
        float w[4];
        if (FP32) {
            const float4 v = reinterpret_cast<const float4*>(W)[j];
            w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
        } else {
            const uint2 v = reinterpret_cast<const uint2*>(W)[j];
            w[0] = __uint_as_float(v.x << 16);
            w[1] = __uint_as_float(v.x & 0xffff0000u);
            w[2] = __uint_as_float(v.y << 16);
            w[3] = __uint_as_float(v.y & 0xffff0000u);
        }
        unsigned b = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float r = rintf(__fdiv_rn(w[i], d));
            r = fminf(fmaxf(r, -1.0f), 1.0f);
            b |= (unsigned)((int)r + 1) << (2 * i);
        }
        Wp[j] = (uint8_t)b;
    }
}

// Count 2-bit fields equal to 3 (the invalid code).
__global__ void __launch_bounds__(kPackThreads) count_bad_codes_kernel(const uint8_t* __restrict__ Wp,
                                                                       int64_t nbytes,
                                                                       unsigned long long* count) {
    __shared__ unsigned long long scratch[kPackThreads / 32];
    unsigned long long c = 0;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < nbytes; j += stride) {
        const unsigned b = Wp[j];
        c += __popc(b & (b >> 1) & 0x55u);
    }
    c = block_sum<kPackThreads / 32>(c, scratch);
    if (threadIdx.x == 0 && c) atomicAdd(count, c);
}

int grid_for(int64_t work, int cap) {
    int64_t g = (work + kPackThreads - 1) / kPackThreads;
    if (g > cap) g = cap;
    if (g < 1) g = 1;
    return (int)g;
}

}  // namespace

int absmean_blocks(int64_t n) { return grid_for(n, kAbsmeanMaxBlocks); }

cudaError_t launch_absmean(const void* W, bool fp32, int64_t n, double* partial, float* gamma,
                           cudaStream_t s) {
    const int g = absmean_blocks(n);
    if (fp32)
        absmean_partial_kernel<true><<<g, kPackThreads, 0, s>>>(W, n, partial);
    else
        absmean_partial_kernel<false><<<g, kPackThreads, 0, s>>>(W, n, partial);
    absmean_final_kernel<<<1, 32, 0, s>>>(partial, g, n, gamma);
    return cudaGetLastError();
}

cudaError_t launch_absmean_sum(const void* W, bool fp32, int64_t n, double* partial, double* sum, cudaStream_t s) {
    const int g = absmean_blocks(n);
    if (fp32)
        absmean_partial_kernel<true><<<g, kPackThreads, 0, s>>>(W, n, partial);
    else
        absmean_partial_kernel<false><<<g, kPackThreads, 0, s>>>(W, n, partial);
    absmean_sum_kernel<<<1, 32, 0, s>>>(partial, g, sum);
    return cudaGetLastError();
}

cudaError_t launch_gamma_from_sum(const double* total_sum, int64_t count, float* gamma, cudaStream_t s) {
    gamma_from_sum_kernel<<<1, 1, 0, s>>>(total_sum, count, gamma);
    return cudaGetLastError();
}

cudaError_t launch_ternary_pack(const void* W, bool fp32, int64_t N, int64_t K, const float* gamma,
                                uint8_t* Wp, cudaStream_t s, bool per_row) {
    const int64_t nbytes = N * (K / 4), KB = K / 4;
    const int g = grid_for(nbytes, 148 * 64);
    if (per_row) {
        if (fp32)
            ternary_pack_kernel<true, true><<<g, kPackThreads, 0, s>>>(W, nbytes, KB, gamma, Wp);
        else
            ternary_pack_kernel<false, true><<<g, kPackThreads, 0, s>>>(W, nbytes, KB, gamma, Wp);
    } else if (fp32) {
        ternary_pack_kernel<true, false><<<g, kPackThreads, 0, s>>>(W, nbytes, KB, gamma, Wp);
    } else {
        ternary_pack_kernel<false, false><<<g, kPackThreads, 0, s>>>(W, nbytes, KB, gamma, Wp);
    }
    return cudaGetLastError();
}

cudaError_t launch_absmean_rows(const void* W, bool fp32, int64_t N, int64_t K, float* gammas, cudaStream_t s) {
    if (fp32)
        absmean_rows_kernel<true><<<(unsigned)N, kPackThreads, 0, s>>>(W, K, gammas);
    else
        absmean_rows_kernel<false><<<(unsigned)N, kPackThreads, 0, s>>>(W, K, gammas);
    return cudaGetLastError();
}

cudaError_t launch_count_bad_codes(const uint8_t* Wp, int64_t nbytes, unsigned long long* count,
                                   cudaStream_t s) {
    const int g = grid_for(nbytes, 148 * 16);
    count_bad_codes_kernel<<<g, kPackThreads, 0, s>>>(Wp, nbytes, count);
    return cudaGetLastError();
}

}  // namespace bl

// Decode GEMV for M <= 16 tokens: acc[m, n] = sum_k Wq[n, k] * xq[m, k].
//
// Paper card "BitNet b1.58 2B4T Technical Report", "Method Adaptation": the
// packed int8 weights are loaded on chip, unpacked right before the matmul and
// multiplied with the int8 activations (pack-store-load-unpack-compute). Here
// the packed bytes stream from HBM straight into registers (16-byte loads that
// skip L1), are unpacked there with one AND per 4 codes, and feed int8 tensor-core
// MMAs (m16n8k32, u8 weights x s8 activations, int32 accumulators). Nothing of the
// weight is staged or re-read.
//
// Unpacking without shifts. A packed 32-bit word holds 16 codes c = q + 1; the
// i-th 2-bit field of its 4 bytes is (word & (0x03030303 << 2i)), i.e. the codes
// of k = 4j + i times 4^i. Each field i gets its own accumulator; at the end
// acc_u = A0 + A1/4 + A2/16 + A3/64 (each Ai is an exact multiple of 4^i) and
// acc = acc_u - sum_k xq (the +1 offset of the codes). The activation operand
// is laid out in PLANES (plane i holds xq[4j + i] at byte j), so a field of a
// weight word and a word of plane i cover the same k.
//
// Work split: one CTA per 16 output rows (and per group of 8*NT tokens); its 8
// warps split K in 64-byte column chunks; partial sums meet in shared memory and
// the dequantisation epilogue is fused.
#include "common.cuh"
#include "kernels.h"

namespace bl {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;
constexpr int kUnroll = 4;

__device__ __forceinline__ void mma_u8s8(int (&d)[4], unsigned a0, unsigned a1, unsigned a2,
                                         unsigned a3, unsigned b0, unsigned b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One 64-byte chunk column for one 16-row tile: wa is row g, wb row g+8 (16 B each
// per lane), xv[nt][i] the plane-i activation words of this lane's token.
template <int NT>
__device__ __forceinline__ void chunk_mma(int (&acc)[NT][4][4], const uint4& wa, const uint4& wb,
                                          const uint4 (&xv)[NT][4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const unsigned mask = 0x03030303u << (2 * i);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            mma_u8s8(acc[nt][i], wa.x & mask, wb.x & mask, wa.y & mask, wb.y & mask, xv[nt][i].x,
                     xv[nt][i].y);
            mma_u8s8(acc[nt][i], wa.z & mask, wb.z & mask, wa.w & mask, wb.w & mask, xv[nt][i].z,
                     xv[nt][i].w);
        }
    }
}

template <int NT>
__device__ __forceinline__ void load_x(uint4 (&xv)[NT][4], const int8_t* const (&xbase)[NT],
                                       const bool (&tv)[NT], int64_t KB, int off) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            xv[nt][i] = tv[nt] ? ld_nc16(xbase[nt] + i * KB + off) : make_uint4(0, 0, 0, 0);
    }
}

template <int NT>
__global__ void __launch_bounds__(kThreads) gemv_mma_kernel(
    const uint8_t* __restrict__ Wp, const float* __restrict__ gamma_p, int N, int KB,
    const int8_t* __restrict__ Xp, const float* __restrict__ scale, const int32_t* __restrict__ xsum,
    int M, GemvOut out) {
    constexpr int TOK = 8 * NT;
    __shared__ int red[kWarps][16][TOK];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int n0 = blockIdx.x * 16;
    const int tok0 = blockIdx.y * TOK;
    const int nchunks = KB >> 6;

    const int rowA = min(n0 + g, N - 1), rowB = min(n0 + g + 8, N - 1);
    const uint8_t* pA = Wp + (size_t)rowA * KB + 16 * t;
    const uint8_t* pB = Wp + (size_t)rowB * KB + 16 * t;

    const int8_t* xbase[NT];
    bool tv[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int tok = tok0 + 8 * nt + g;
        tv[nt] = tok < M;
        xbase[nt] = Xp + (size_t)(tv[nt] ? tok : 0) * 4 * KB + 16 * t;
    }

    int acc[NT][4][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[nt][i][e] = 0;

    int c = warp;
    for (; c + kWarps * (kUnroll - 1) < nchunks; c += kWarps * kUnroll) {
        uint4 wa[kUnroll], wb[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            wa[u] = ld_stream16(pA + 64 * (c + kWarps * u));
            wb[u] = ld_stream16(pB + 64 * (c + kWarps * u));
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            uint4 xv[NT][4];
            load_x<NT>(xv, xbase, tv, KB, 64 * (c + kWarps * u));
            chunk_mma<NT>(acc, wa[u], wb[u], xv);
        }
    }
    for (; c < nchunks; c += kWarps) {
        const uint4 wa = ld_stream16(pA + 64 * c), wb = ld_stream16(pB + 64 * c);
        uint4 xv[NT][4];
        load_x<NT>(xv, xbase, tv, KB, 64 * c);
        chunk_mma<NT>(acc, wa, wb, xv);
    }

    // Fold the four field accumulators; D element e sits at row g + 8*(e >> 1),
    // token 8*nt + 2t + (e & 1).
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int v = acc[nt][0][e] + (acc[nt][1][e] >> 2) + (acc[nt][2][e] >> 4) +
                          (acc[nt][3][e] >> 6);
            red[warp][g + 8 * (e >> 1)][8 * nt + 2 * t + (e & 1)] = v;
        }
    __syncthreads();

    const float gamma = *gamma_p;
    for (int idx = threadIdx.x; idx < 16 * TOK; idx += kThreads) {
        const int r = idx & 15, cl = idx >> 4;
        const int n = n0 + r, m = tok0 + cl;
        if (n >= N || m >= M) continue;
        int sum = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) sum += red[w][r][cl];
        const int a = sum - xsum[m];
        const float deq = __fdiv_rn(gamma, scale[m]);
        float v = dequant(a, deq);
        const size_t o = (size_t)m * N + n;
        if (out.y32) {
            out.y32[o] = v;
        } else {
            if (out.residual) v = __fadd_rn(bf16_bits_to_f32(out.residual[o]), v);
            out.y[o] = f32_to_bf16_bits(v);
        }
        if (out.acc) out.acc[o] = a;
    }
}

// Generic path: any K % 4 == 0, NATURAL codes. One warp per (row, token).
__global__ void __launch_bounds__(kThreads) gemv_generic_kernel(
    const uint8_t* __restrict__ Wp, const float* __restrict__ gamma_p, int N, int K,
    const int8_t* __restrict__ Xn, const float* __restrict__ scale, int M, GemvOut out) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = blockIdx.x * kWarps + warp;
    const int m = blockIdx.y;
    if (n >= N) return;
    const int KB = K / 4;
    const uint8_t* wr = Wp + (size_t)n * KB;
    const int8_t* xr = Xn + (size_t)m * K;
    int a = 0;
    for (int j = lane; j < KB; j += 32) {
        const unsigned b = wr[j];
#pragma unroll
        for (int i = 0; i < 4; ++i) a += ((int)((b >> (2 * i)) & 3u) - 1) * (int)xr[4 * j + i];
    }
    a = warp_sum(a);
    if (lane == 0) {
        const float deq = __fdiv_rn(*gamma_p, scale[m]);
        float v = dequant(a, deq);
        const size_t o = (size_t)m * N + n;
        if (out.y32) {
            out.y32[o] = v;
        } else {
            if (out.residual) v = __fadd_rn(bf16_bits_to_f32(out.residual[o]), v);
            out.y[o] = f32_to_bf16_bits(v);
        }
        if (out.acc) out.acc[o] = a;
    }
}

}  // namespace

bool gemv_fast_ok(int64_t N, int64_t K) { return N >= 1 && K % 256 == 0; }

cudaError_t launch_gemv(const uint8_t* Wp, const float* gamma, int64_t N, int64_t K,
                        const int8_t* Xp, const float* scale, const int32_t* xsum, int64_t M,
                        const GemvOut& out, cudaStream_t s) {
    if (M == 0 || N == 0) return cudaSuccess;
    const int KB = (int)(K / 4);
    const unsigned gx = (unsigned)((N + 15) / 16);
    if (M <= 8) {
        gemv_mma_kernel<1><<<dim3(gx, 1), kThreads, 0, s>>>(Wp, gamma, (int)N, KB, Xp, scale, xsum,
                                                            (int)M, out);
    } else {
        const unsigned gy = (unsigned)((M + 15) / 16);
        gemv_mma_kernel<2><<<dim3(gx, gy), kThreads, 0, s>>>(Wp, gamma, (int)N, KB, Xp, scale, xsum,
                                                             (int)M, out);
    }
    return cudaGetLastError();
}

cudaError_t launch_gemv_generic(const uint8_t* Wp, const float* gamma, int64_t N, int64_t K,
                                const int8_t* Xn, const float* scale, int64_t M,
                                const GemvOut& out, cudaStream_t s) {
    if (M == 0 || N == 0) return cudaSuccess;
    const dim3 grid((unsigned)((N + kWarps - 1) / kWarps), (unsigned)M);
    gemv_generic_kernel<<<grid, kThreads, 0, s>>>(Wp, gamma, (int)N, (int)K, Xn, scale, (int)M, out);
    return cudaGetLastError();
}

}  // namespace bl

// Lookup-table ternary GEMV for up to 16 tokens: acc[m, n] = sum_k Wq[n, k] * xq[m, k].
//
// The dignews article on the release, section 3 (bitnet.cpp): the CPU kernels
// follow T-MAC and replace multiplications by lookups in tables of precomputed
// partial sums of the activations, indexed by the packed weight bits, and are
// lossless. This is that method on the GPU, as a counterpart to the dp4a /
// mma.sync and tensor-core GEMVs:
//   table:  for each token, each 2-weight nibble position p of the packed row
//           (k = 2p, 2p + 1) and each 4-bit pattern e (codes c0 = e & 3,
//           c1 = e >> 2), T[p][e] = q(c0) xq[2p] + q(c1) xq[2p + 1] with
//           q(c) = c - 1 (code 3 is invalid and contributes 0); built once per
//           K segment per CTA and used by every row the CTA owns;
//   lookup: every packed byte costs two table reads per token (low and high
//           nibble) and two integer adds; no multiplications; the sum is exact.
// Layout in shared memory, int16 entries: [token][e][byte b of the word][word][half],
// where word index l of a segment is stored at column 128 (l / 128) + 32 (l % 4)
// + (l % 128) / 4. A lane holds words 4L .. 4L + 3 of a 128-word chunk (one
// 16-byte load), so when the 32 lanes look up their i-th word they read columns
// 32 i + L: 32 consecutive 32-bit words, one per bank, whatever the entries e.
//
// Work split: one CTA (16 warps) per range of rows; for each K segment the CTA
// builds the table of its (up to four) tokens, then each warp takes one row at a
// time, its lanes streaming 16-byte words. Up to four tokens per launch share
// the table (four tokens fill shared memory); more tokens take further launches,
// each streaming the weights again.
#include "common.cuh"
#include "kernels.h"

namespace bl {
namespace {

constexpr int LUT_THREADS = 512;
constexpr int LUT_WARPS = LUT_THREADS / 32;
constexpr int CHUNK = 128;            // words per lane-interleaved chunk (one 16-byte load per lane)
constexpr int PART_BYTES_MAX = 24 * 1024;

// table column of word l of a segment
__device__ __forceinline__ int lut_col(int l) { return (l & ~(CHUNK - 1)) + 32 * (l & 3) + ((l & (CHUNK - 1)) >> 2); }

__device__ __forceinline__ int tern(int c) { return c == 3 ? 0 : c - 1; }

template <int GT>
__global__ void __launch_bounds__(LUT_THREADS, 1)
    gemv_lut_kernel(const uint8_t* __restrict__ Wp, const float* __restrict__ gamma, int N, int K,
                    const int8_t* __restrict__ xq, const float* __restrict__ scale, int M, int m0,
                    int rows_per_cta, int seg_words, GemvOut out) {
    extern __shared__ __align__(16) uint8_t sm[];
    int16_t* lut = reinterpret_cast<int16_t*>(sm);  // [GT][16][4][seg_words][2]
    int32_t* part = reinterpret_cast<int32_t*>(sm + (size_t)GT * 16 * 4 * seg_words * 2 * sizeof(int16_t));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int W = K / 16;  // packed 32-bit words per row
    const int KB = K / 4;
    const int r0 = blockIdx.x * rows_per_cta, r1 = min(N, r0 + rows_per_cta);
    const int rows = r1 - r0;
    const int gt = min(GT, M - m0);
    const size_t ent_stride = (size_t)4 * seg_words * 2;  // int16 entries per pattern e

    grid_dependency_wait();
    for (int i = threadIdx.x; i < rows * GT; i += LUT_THREADS) part[i] = 0;

    for (int w0 = 0; w0 < W; w0 += seg_words) {
        const int sw = min(seg_words, W - w0);
        __syncthreads();  // the previous segment's lookups are done
        // table of this segment: one thread per (token, word, byte)
        for (int idx = threadIdx.x; idx < gt * sw * 4; idx += LUT_THREADS) {
            const int t = idx / (sw * 4), rem = idx - t * (sw * 4);
            const int l = rem >> 2, b = rem & 3;
            const int k = (w0 + l) * 16 + 4 * b;
            const uint32_t xw = *reinterpret_cast<const uint32_t*>(xq + (size_t)(m0 + t) * K + k);
            const int x[4] = {(int)(int8_t)(xw & 0xff), (int)(int8_t)((xw >> 8) & 0xff),
                              (int)(int8_t)((xw >> 16) & 0xff), (int)(int8_t)(xw >> 24)};
            int16_t* dst = lut + (size_t)t * 16 * ent_stride + ((size_t)b * seg_words + lut_col(l)) * 2;
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int q0 = tern(e & 3), q1 = tern(e >> 2);
                dst[e * ent_stride] = (int16_t)(q0 * x[0] + q1 * x[1]);
                dst[e * ent_stride + 1] = (int16_t)(q0 * x[2] + q1 * x[3]);
            }
        }
        __syncthreads();
        // rows: one warp per row, lanes over 16-byte words
        for (int r = r0 + warp; r < r1; r += LUT_WARPS) {
            const uint8_t* wrow = Wp + (size_t)r * KB + (size_t)w0 * 4;
            int acc[GT];
#pragma unroll
            for (int t = 0; t < GT; ++t) acc[t] = 0;
            for (int c = 0; c < sw; c += 4 * CHUNK) {
                uint4 wv[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {  // up to four chunks' loads in flight
                    const int l = c + u * CHUNK + 4 * lane;
                    wv[u] = l < sw ? ld_stream16(wrow + 4 * l) : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    if (c + u * CHUNK >= sw) break;
                    // lanes past the segment's last word have no table columns
                    if (c + u * CHUNK + 4 * lane >= sw) continue;
                    const uint32_t words[4] = {wv[u].x, wv[u].y, wv[u].z, wv[u].w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int col = c + u * CHUNK + 32 * i + lane;
#pragma unroll
                        for (int b = 0; b < 4; ++b) {
                            const uint32_t byte = (words[i] >> (8 * b)) & 0xffu;
                            const int16_t* base = lut + ((size_t)b * seg_words + col) * 2;
                            const int lo = (int)(byte & 15u), hi = (int)(byte >> 4);
#pragma unroll
                            for (int t = 0; t < GT; ++t) {
                                const int16_t* bt = base + (size_t)t * 16 * ent_stride;
                                acc[t] += (int)bt[lo * ent_stride] + (int)bt[hi * ent_stride + 1];
                            }
                        }
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < GT; ++t) {
                const int v = warp_sum(acc[t]);
                if (lane == 0) part[(r - r0) * GT + t] += v;
            }
        }
    }
    __syncthreads();
    // dequantising epilogue: thread per (row, token), rows fastest (coalesced stores)
    for (int idx = threadIdx.x; idx < rows * gt; idx += LUT_THREADS) {
        const int rr = idx % rows, t = idx / rows;
        const int n = r0 + rr, m = m0 + t;
        const int a = part[rr * GT + t];
        float y = dequant(a, __fdiv_rn(gamma[gamma_index(out, n)], scale[m]));
        const size_t o = (size_t)m * N + n;
        if (out.y32) {
            out.y32[o] = y;
        } else {
            if (out.residual) y = __fadd_rn(bf16_bits_to_f32(out.residual[o]), y);
            out.y[o] = f32_to_bf16_bits(y);
        }
        if (out.acc) out.acc[o] = a;
    }
}

int sm_count() {
    static int cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev < 64 && cached[dev]) return cached[dev];
    int n = 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n = 148;
    if (dev < 64) cached[dev] = n;
    return n;
}

template <int GT>
cudaError_t launch_gt(const uint8_t* Wp, const float* gamma, int64_t N, int64_t K, const int8_t* xq,
                      const float* scale, int64_t M, const GemvOut& out, cudaStream_t s) {
    // table words per segment: the table of GT tokens takes at most 192 KiB
    const int64_t W = K / 16;
    const int64_t seg_cap = (GT == 1 ? 768 : GT == 2 ? 384 : 128);
    const int64_t w_round = (W + CHUNK - 1) / CHUNK * CHUNK;
    const int seg_words = (int)(w_round < seg_cap ? w_round : seg_cap);
    const size_t lut_bytes = (size_t)GT * 16 * 4 * seg_words * 2 * sizeof(int16_t);
    int64_t rows = (N + sm_count() - 1) / sm_count();
    const int64_t rows_cap = PART_BYTES_MAX / (GT * 4);
    if (rows > rows_cap) rows = rows_cap;
    const unsigned grid = (unsigned)((N + rows - 1) / rows);
    const size_t smem = lut_bytes + (size_t)rows * GT * 4;
    auto kern = gemv_lut_kernel<GT>;
    static bool done[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64 || !done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        if (dev < 64) done[dev] = true;
    }
    for (int64_t m0 = 0; m0 < M; m0 += GT) {
        cudaError_t e = launch_pdl(kern, dim3(grid), dim3(LUT_THREADS), smem, s, Wp, gamma, (int)N, (int)K, xq, scale,
                                   (int)M, (int)m0, (int)rows, seg_words, out);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace

bool gemv_lut_ok(int64_t N, int64_t K, int64_t M, const void* Wp, const void* xq) {
    return N >= 1 && M >= 1 && M <= 16 && K % 256 == 0 && reinterpret_cast<uintptr_t>(Wp) % 16 == 0 &&
           reinterpret_cast<uintptr_t>(xq) % 4 == 0;
}

cudaError_t launch_gemv_lut(const uint8_t* Wp, const float* gamma, int64_t N, int64_t K, const int8_t* xq,
                            const float* scale, int64_t M, const GemvOut& out, cudaStream_t s) {
    if (M == 0 || N == 0) return cudaSuccess;
    if (!gemv_lut_ok(N, K, M, Wp, xq)) return cudaErrorInvalidValue;
    if (M == 1) return launch_gt<1>(Wp, gamma, N, K, xq, scale, M, out, s);
    if (M == 2) return launch_gt<2>(Wp, gamma, N, K, xq, scale, M, out, s);
    return launch_gt<4>(Wp, gamma, N, K, xq, scale, M, out, s);
}

}  // namespace bl

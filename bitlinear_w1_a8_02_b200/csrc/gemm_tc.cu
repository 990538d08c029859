// Prefill GEMM on the 5th-generation tensor cores (tcgen05, sm_100a):
//   acc[m, n] = sum_k Wq[n, k] * xq[m, k],   M > 16 tokens.
//
// Paper card "BitNet b1.58 2B4T Technical Report", "Method Adaptation": packed
// int8 weights are loaded into on-chip memory and unpacked right before the
// int8 matmul (pack-store-load-unpack-compute). On B200 this becomes:
//   TMA:     packed weight tile [BN rows x 32 bytes, BN = 256, or 128 / 64 when
//            wider tiles cannot fill the SMs] and activation-code tile
//            [128 tokens x 128 codes] -> shared memory (one mbarrier per stage);
//   unpack:  four warps turn every packed 32-bit word into 16 code bytes
//            (three shifts and four ANDs) and store them straight into the
//            128-byte-swizzled K-major operand layout the tensor core reads;
//   MMA:     one thread issues tcgen05.mma kind::i8 (A = codes s8, B = weight
//            codes u8 in {0,1,2}) into a 128 x BN int32 accumulator in TMEM;
//   epilogue: four more warps read TMEM (tcgen05.ld), subtract the code offset
//            (sum_k xq), dequantise and store bf16 / fp32 / int32, while the
//            next tile accumulates into the second TMEM accumulator.
// The activation codes are in the G16T layout (each 16-code group stored as a
// transposed 4x4 byte block), which is exactly the order a packed word unpacks
// into, so no byte shuffling is needed anywhere.
//
// Work split: data-parallel (each persistent CTA takes whole 128 x BN tiles) or,
// when the tiles would leave part of the last wave idle, stream-K: the k-blocks
// of all tiles, tile after tile, are cut into one contiguous range per CTA. A
// CTA whose range covers a whole tile finishes it as usual; a piece of a tile is
// written as raw int32 accumulators to a per-CTA slot of the workspace, and a
// second kernel sums the pieces of each split tile (int32, so in any order the
// same) and runs the same epilogue. No CTA ever waits for another.
//
// Every mbarrier wait is bounded (1 s); a wait that gives up sets the device
// error word (reported as BL_ERR_TIMEOUT), lets the CTA drain and returns.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace bl {
namespace {

constexpr int BM = 128;               // tokens per tile (TMEM lanes)
constexpr int BK = 128;               // codes per k-block (one 128-byte swizzle row)
constexpr int TSTAGES = 6;            // TMA ring: activation codes + packed weights
constexpr int USTAGES = 2;            // unpacked weight-code ring
constexpr int A_BYTES = BM * BK;      // 16 KiB activation codes
#ifndef BL_GEMM_UNPACK_WARPS
#define BL_GEMM_UNPACK_WARPS 4
#endif
constexpr int UNPACK_WARPS = BL_GEMM_UNPACK_WARPS;
constexpr int UNPACK_THREADS = 32 * UNPACK_WARPS;
constexpr int EPI_THREADS = 128;
constexpr int THREADS = 64 + UNPACK_THREADS + EPI_THREADS;  // TMA, MMA, unpack, epilogue warps
constexpr uint64_t WAIT_LIMIT_NS = 1000000000ull;
constexpr int NUM_BARS = 2 * TSTAGES + 2 * USTAGES + 4;

// Sizes that follow from the tile width BN (weight rows per tile = TMEM columns
// per accumulator): 256 normally, 128 or 64 when wider tiles cannot fill the SMs.
template <int BN>
struct TileCfg {
    static constexpr int P_BYTES = BN * BK / 4;  // packed weights per k-block
    static constexpr int U_BYTES = BN * BK;      // unpacked weight codes per k-block
    static constexpr int UNPACK_VEC = BN * BK / 4 / 16 / UNPACK_THREADS;  // 16-byte groups per thread
    static constexpr uint32_t TMEM_COLS = 2 * BN;  // two accumulators: epilogue of tile t overlaps t+1
    static constexpr size_t SMEM_BYTES =
        1024 /*alignment slack*/ + TSTAGES * (A_BYTES + P_BYTES) + USTAGES * U_BYTES + NUM_BARS * 8;
    static_assert(BN * BK / 4 / 16 % UNPACK_THREADS == 0, "unpack work must split evenly");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

__device__ __forceinline__ bool aligned16(const void* p) {
    return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

__device__ __forceinline__ void report_timeout(unsigned* err, int* abort_flag) {
    atomicOr(err, 1u);
    atomicExch(abort_flag, 1);
}

__device__ __forceinline__ bool aborted(const int* abort_flag) {
    return *reinterpret_cast<const volatile int*>(abort_flag) != 0;
}

// The (tile, k-block range) pieces one CTA works on, in order. Data-parallel:
// tiles c, c + G, ... whole. Stream-K: the units [U c / G, U (c + 1) / G) of the
// U = tiles x nkb k-blocks, tile-major.
template <bool SK>
struct WorkIter {
    int nkb, num_tiles, stride;
    int u, ue;  // stream-K: next unit, end of the range
    int tile;   // data-parallel: next tile
    __device__ WorkIter(int nkb_, int num_tiles_, int G, int c)
        : nkb(nkb_), num_tiles(num_tiles_), stride(G), u(0), ue(0), tile(c) {
        if (SK) {
            const long long U = (long long)num_tiles * nkb;
            u = (int)(U * c / G);
            ue = (int)(U * (c + 1) / G);
        }
    }
    __device__ bool next(int& t, int& kb0, int& kb1) {
        if (SK) {
            if (u >= ue) return false;
            t = u / nkb;
            kb0 = u - t * nkb;
            kb1 = min(nkb, kb0 + (ue - u));
            u += kb1 - kb0;
            return true;
        }
        if (tile >= num_tiles) return false;
        t = tile;
        kb0 = 0;
        kb1 = nkb;
        tile += stride;
        return true;
    }
};

// Per-row gamma variant: outputs nb .. nb + cnt - 1 of one row, each with
// deq = gamma[n] / s (one IEEE division per output, as the definition reads).
template <int CNT>
__device__ __forceinline__ void store_row_per_row_gamma(const uint32_t* v, int xs, float s, const float* gamma,
                                                        int nb, int N, size_t o, const GemvOut& out) {
#pragma unroll 4
    for (int j = 0; j < CNT; ++j) {
        if (nb + j >= N) break;
        const int a = static_cast<int>(v[j]) - xs;
        float f = dequant(a, __fdiv_rn(gamma[nb + j], s));
        if (out.y32) {
            out.y32[o + j] = f;
        } else {
            if (out.residual) f = __fadd_rn(bf16_bits_to_f32(out.residual[o + j]), f);
            out.y[o + j] = f32_to_bf16_bits(f);
        }
        if (out.acc) out.acc[o + j] = a;
    }
}

// Dequantise and store 32 consecutive outputs of one row (one TMEM load).
__device__ __forceinline__ void store_row_chunk(const uint32_t (&v)[32], int xs, float deq, int nb,
                                                int N, size_t o, const GemvOut& out, bool vec) {
    if (vec && nb + 32 <= N) {
        if (out.y32) {
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
                float4 f;
                f.x = dequant(static_cast<int>(v[j]) - xs, deq);
                f.y = dequant(static_cast<int>(v[j + 1]) - xs, deq);
                f.z = dequant(static_cast<int>(v[j + 2]) - xs, deq);
                f.w = dequant(static_cast<int>(v[j + 3]) - xs, deq);
                *reinterpret_cast<float4*>(out.y32 + o + j) = f;
            }
        } else {
#pragma unroll
            for (int j = 0; j < 32; j += 8) {
                uint4 r = make_uint4(0, 0, 0, 0);
                if (out.residual) r = *reinterpret_cast<const uint4*>(out.residual + o + j);
                const uint32_t rr[4] = {r.x, r.y, r.z, r.w};
                uint32_t pk[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float lo = dequant(static_cast<int>(v[j + 2 * e]) - xs, deq);
                    float hi = dequant(static_cast<int>(v[j + 2 * e + 1]) - xs, deq);
                    if (out.residual) {
                        lo = __fadd_rn(bf16_bits_to_f32(rr[e] & 0xffffu), lo);
                        hi = __fadd_rn(bf16_bits_to_f32(rr[e] >> 16), hi);
                    }
                    pk[e] = f32_to_bf16_bits(lo) | (static_cast<uint32_t>(f32_to_bf16_bits(hi)) << 16);
                }
                *reinterpret_cast<uint4*>(out.y + o + j) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
        }
        if (out.acc) {
#pragma unroll
            for (int j = 0; j < 32; j += 4)
                *reinterpret_cast<int4*>(out.acc + o + j) =
                    make_int4(static_cast<int>(v[j]) - xs, static_cast<int>(v[j + 1]) - xs,
                              static_cast<int>(v[j + 2]) - xs, static_cast<int>(v[j + 3]) - xs);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            if (nb + j >= N) break;
            const int a = static_cast<int>(v[j]) - xs;
            float f = dequant(a, deq);
            if (out.y32) {
                out.y32[o + j] = f;
            } else {
                if (out.residual) f = __fadd_rn(bf16_bits_to_f32(out.residual[o + j]), f);
                out.y[o + j] = f32_to_bf16_bits(f);
            }
            if (out.acc) out.acc[o + j] = a;
        }
    }
}

// Persistent CTAs walk the (m-tile, n-tile) grid with n fastest, so the CTAs in
// flight share activation tiles and the whole packed weight stays in L2.
// PR: one gamma per output row (the per-row variant); without it that code is
// compiled out of the epilogue.
// DUAL: the FFN's gate and up projections in one launch. Each 256-row weight
// tile holds 128 rows of the gate weight (tmB) and the same 128 rows of the up
// weight (tmB2); the epilogue forms h = max(g, 0)^2 * u of those 128 hidden
// columns and, per token, the tile's sum of h^2 (fp64, columns in order) and max
// |h| (FfnUpOut). Data-parallel tiles only.
template <int BN, bool SK, bool PR, bool DUAL = false>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmB2, int M, int N, int K, const float* __restrict__ gamma_p,
                   const float* __restrict__ scale, const int32_t* __restrict__ xsum, GemvOut out,
                   unsigned* err, uint32_t* __restrict__ partials, FfnUpOut up) {
    static_assert(!DUAL || (BN == 256 && !SK && !PR), "the gate+up tiles are 128 + 128 rows, data-parallel");
    constexpr int P_BYTES = TileCfg<BN>::P_BYTES;
    constexpr int U_BYTES = TileCfg<BN>::U_BYTES;
    constexpr int UNPACK_VEC = TileCfg<BN>::UNPACK_VEC;
    constexpr uint32_t TMEM_COLS = TileCfg<BN>::TMEM_COLS;
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;

    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* sA = smem;                         // TSTAGES x A_BYTES
    uint8_t* sU = sA + TSTAGES * A_BYTES;       // USTAGES x U_BYTES
    uint8_t* sP = sU + USTAGES * U_BYTES;       // TSTAGES x P_BYTES
    uint64_t* bars = reinterpret_cast<uint64_t*>(sP + TSTAGES * P_BYTES);
    auto bar = [&](int i) { return tc::smem_u32(bars + i); };
    auto tfull = [&](int s) { return bar(s); };                              // TMA landed
    auto tempty = [&](int s) { return bar(TSTAGES + s); };                   // MMA done with it
    auto ufull = [&](int u) { return bar(2 * TSTAGES + u); };                // unpacked
    auto uempty = [&](int u) { return bar(2 * TSTAGES + USTAGES + u); };     // MMA done with it
    auto afull = [&](int a) { return bar(2 * TSTAGES + 2 * USTAGES + a); };  // accumulator ready
    auto aempty = [&](int a) { return bar(2 * TSTAGES + 2 * USTAGES + 2 + a); };  // drained

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int TN = DUAL ? BN / 2 : BN;  // output columns per tile
    const int n_tiles = (N + TN - 1) / TN;
    const int num_tiles = n_tiles * ((M + BM - 1) / BM);
    const int nkb = (K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < TSTAGES; ++s) {
            tc::mbar_init(tfull(s), 1);
            tc::mbar_init(tempty(s), 1);
        }
        for (int u = 0; u < USTAGES; ++u) {
            tc::mbar_init(ufull(u), UNPACK_THREADS);
            tc::mbar_init(uempty(u), 1);
        }
        for (int a = 0; a < 2; ++a) {
            tc::mbar_init(afull(a), 1);
            tc::mbar_init(aempty(a), EPI_THREADS);
        }
        abort_sh = 0;
        tc::fence_mbar_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tc::smem_u32(&tmem_base_sh), TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = tmem_base_sh;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tc::prefetch_tmap(&tmA);
            tc::prefetch_tmap(&tmB);
            if (DUAL) tc::prefetch_tmap(&tmB2);
            uint32_t g = 0;
            WorkIter<SK> it(nkb, num_tiles, gridDim.x, blockIdx.x);
            int tile, kb0, kb1;
            while (!aborted(&abort_sh) && it.next(tile, kb0, kb1)) {
                const int m0 = (tile / n_tiles) * BM, n0 = (tile % n_tiles) * TN;
                for (int kb = kb0; kb < kb1; ++kb, ++g) {
                    const int s = g % TSTAGES;
                    if (g >= TSTAGES &&
                        !tc::mbar_wait(tempty(s), ((g / TSTAGES) - 1) & 1, WAIT_LIMIT_NS)) {
                        report_timeout(err, &abort_sh);
                        break;
                    }
                    tc::mbar_arrive_expect_tx(tfull(s), A_BYTES + P_BYTES);
                    tc::tma_load_2d(tc::smem_u32(sA + s * A_BYTES), &tmA, kb * BK, m0, tfull(s));
                    tc::tma_load_2d(tc::smem_u32(sP + s * P_BYTES), &tmB, kb * (BK / 4), n0, tfull(s));
                    if (DUAL)  // up rows into the second half of the weight tile
                        tc::tma_load_2d(tc::smem_u32(sP + s * P_BYTES + (BN / 2) * (BK / 4)), &tmB2, kb * (BK / 4), n0,
                                        tfull(s));
                }
            }
            if (aborted(&abort_sh)) {
                // let the copies still in flight land before the CTA exits
                const uint32_t first = g > TSTAGES ? g - TSTAGES : 0;
                for (uint32_t h = first; h < g; ++h)
                    tc::mbar_wait(tfull(h % TSTAGES), (h / TSTAGES) & 1, WAIT_LIMIT_NS);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = tc::idesc_i8_s8u8(BM, BN);
            uint32_t g = 0, t = 0;
            WorkIter<SK> it(nkb, num_tiles, gridDim.x, blockIdx.x);
            int tile, kb0, kb1;
            for (; !aborted(&abort_sh) && it.next(tile, kb0, kb1); ++t) {
                const int a = t & 1;
                if (t >= 2 && !tc::mbar_wait(aempty(a), ((t >> 1) - 1) & 1, WAIT_LIMIT_NS)) {
                    report_timeout(err, &abort_sh);
                    break;
                }
                tc::fence_after_sync();
                const uint32_t d = tmem + a * BN;
                bool ok = true;
                for (int kb = kb0; kb < kb1; ++kb, ++g) {
                    const int s = g % TSTAGES, u = g % USTAGES;
                    if (!tc::mbar_wait(ufull(u), (g / USTAGES) & 1, WAIT_LIMIT_NS) ||
                        !tc::mbar_wait(tfull(s), (g / TSTAGES) & 1, WAIT_LIMIT_NS)) {
                        report_timeout(err, &abort_sh);
                        ok = false;
                        break;
                    }
                    tc::fence_after_sync();
                    const uint64_t ad = tc::desc_kmajor_sw128(tc::smem_u32(sA + s * A_BYTES));
                    const uint64_t bd = tc::desc_kmajor_sw128(tc::smem_u32(sU + u * U_BYTES));
#pragma unroll
                    for (int kk = 0; kk < BK / 32; ++kk)  // 32 bytes of K per MMA: +2 in 16-byte units
                        tc::mma_i8(d, ad + 2 * kk, bd + 2 * kk, idesc, kb != kb0 || kk != 0);
                    tc::mma_commit(tempty(s));
                    tc::mma_commit(uempty(u));
                }
                if (!ok) break;
                tc::mma_commit(afull(a));
            }
        }
    } else if (warp < 2 + UNPACK_WARPS) {
        // ------------------------------------------------------------ unpack
        const int ut = threadIdx.x - 64;
        uint32_t g = 0;
        WorkIter<SK> it(nkb, num_tiles, gridDim.x, blockIdx.x);
        int tile, kb0, kb1;
        while (!aborted(&abort_sh) && it.next(tile, kb0, kb1)) {
            bool ok = true;
            for (int kb = kb0; kb < kb1; ++kb, ++g) {
                const int s = g % TSTAGES, u = g % USTAGES;
                if (!tc::mbar_wait(tfull(s), (g / TSTAGES) & 1, WAIT_LIMIT_NS) ||
                    (g >= USTAGES &&
                     !tc::mbar_wait(uempty(u), ((g / USTAGES) - 1) & 1, WAIT_LIMIT_NS))) {
                    report_timeout(err, &abort_sh);
                    ok = false;
                    break;
                }
                // Each thread owns UNPACK_VEC 16-byte groups of packed words; all of them are
                // loaded before any store so the shared-memory latencies overlap. Group q
                // holds words 4(q&1)..4(q&1)+3 of row q/2; the 16 codes of word j of row n
                // go to 16-byte chunk j of that row, at swizzle position j ^ (n % 8).
                const uint4* bp4 = reinterpret_cast<const uint4*>(sP + s * P_BYTES);
                uint8_t* bu = sU + u * U_BYTES;
                uint4 pw[UNPACK_VEC];
#pragma unroll
                for (int i = 0; i < UNPACK_VEC; ++i) pw[i] = bp4[ut + UNPACK_THREADS * i];
#pragma unroll
                for (int i = 0; i < UNPACK_VEC; ++i) {
                    const int qg = ut + UNPACK_THREADS * i;
                    const int n = qg >> 1, r = n & 7;
                    uint8_t* rowp = bu + (n >> 3) * 1024 + r * 128;
                    const uint32_t words[4] = {pw[i].x, pw[i].y, pw[i].z, pw[i].w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = 4 * (qg & 1) + e;
                        const uint32_t wd = words[e];
                        uint4 v;
                        v.x = wd & 0x03030303u;
                        v.y = (wd >> 2) & 0x03030303u;
                        v.z = (wd >> 4) & 0x03030303u;
                        v.w = (wd >> 6) & 0x03030303u;
                        *reinterpret_cast<uint4*>(rowp + ((j ^ r) << 4)) = v;
                    }
                }
                tc::fence_proxy_async_smem();
                tc::mbar_arrive(ufull(u));
            }
            if (!ok) break;
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;  // the TMEM lane quarter this warp may read
        const float gamma = *gamma_p;
        const bool vec = (N % 8 == 0) && aligned16(out.y) && aligned16(out.y32) &&
                         aligned16(out.residual) && aligned16(out.acc);
        uint32_t t = 0;
        WorkIter<SK> it(nkb, num_tiles, gridDim.x, blockIdx.x);
        int tile, kb0, kb1;
        for (; it.next(tile, kb0, kb1); ++t) {
            const int a = t & 1;
            bool ok = !aborted(&abort_sh) && tc::mbar_wait(afull(a), (t >> 1) & 1, WAIT_LIMIT_NS);
            if (!__all_sync(0xffffffffu, ok)) {  // tcgen05.ld below is warp-collective
                report_timeout(err, &abort_sh);
                break;
            }
            tc::fence_after_sync();
            const int m0 = (tile / n_tiles) * BM, n0 = (tile % n_tiles) * TN;
            const int m = m0 + q * 32 + lane;
            const bool mv = m < M;
            if constexpr (DUAL) {
                // h of this token's 128 hidden columns; gate in columns 0..127 of the
                // accumulator, up in 128..255
                const uint32_t tb = tmem + (static_cast<uint32_t>(q * 32) << 16) + a * BN;
                const float dg = mv ? __fdiv_rn(gamma, scale[m]) : 0.0f;
                const float du = mv ? __fdiv_rn(*up.gamma_u, scale[m]) : 0.0f;
                const int xs = mv ? xsum[m] : 0;
                double ss = 0.0;
                float mx = 0.0f;
#pragma unroll 1
                for (int c = 0; c < TN / 32; ++c) {
                    uint32_t vg[32], vu[32];
                    tc::tmem_ld_32x32(tb + c * 32, vg);
                    tc::tmem_ld_32x32(tb + TN + c * 32, vu);
                    tc::tmem_ld_wait();
                    const int nb = n0 + c * 32;
                    if (!mv || nb >= N) continue;
                    float hv[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float gv = dequant(static_cast<int>(vg[j]) - xs, dg);
                        const float uv = dequant(static_cast<int>(vu[j]) - xs, du);
                        const float t0 = gv > 0.0f ? gv : 0.0f;
                        hv[j] = __fmul_rn(__fmul_rn(t0, t0), uv);
                    }
                    const int cnt = min(32, N - nb);
                    float* hrow = up.h + (size_t)m * N + nb;
                    if (cnt == 32 && (N & 3) == 0) {  // 16-byte stores
#pragma unroll
                        for (int j = 0; j < 32; j += 4)
                            *reinterpret_cast<float4*>(hrow + j) = make_float4(hv[j], hv[j + 1], hv[j + 2], hv[j + 3]);
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (j < cnt) hrow[j] = hv[j];
                    }
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        if (j >= cnt) break;
                        ss = __dadd_rn(ss, __dmul_rn((double)hv[j], (double)hv[j]));
                        mx = fmaxf(mx, fabsf(hv[j]));
                    }
                }
                if (mv) {
                    up.part_ss[(size_t)m * n_tiles + (tile % n_tiles)] = ss;
                    up.part_max[(size_t)m * n_tiles + (tile % n_tiles)] = mx;
                }
                tc::fence_before_sync();
                tc::mbar_arrive(aempty(a));
                continue;
            }
            const bool whole = !SK || (kb0 == 0 && kb1 == nkb);
            // a piece of a split tile goes to slot 2c (the CTA's first piece) or 2c + 1,
            // column-major, so that the 32 rows of a warp store one 128-byte line
            uint32_t* slot = whole ? nullptr
                                   : partials + (size_t)(2 * blockIdx.x + (t == 0 ? 0 : 1)) * BM * BN +
                                         (q * 32 + lane);
            const float deq = mv && whole ? __fdiv_rn(gamma, scale[m]) : 0.0f;
            const int xs = mv && whole ? xsum[m] : 0;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t v[32];
                tc::tmem_ld_32x32(tmem + (static_cast<uint32_t>(q * 32) << 16) + a * BN + c * 32, v);
                tc::tmem_ld_wait();
                const int nb = n0 + c * 32;
                if (SK && !whole) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) slot[(size_t)(c * 32 + j) * BM] = v[j];
                } else if (PR && mv && nb < N) {
                    store_row_per_row_gamma<32>(v, xs, scale[m], gamma_p, nb, N, static_cast<size_t>(m) * N + nb, out);
                } else if (mv && nb < N) {
                    // row segments with their own gamma end on 32-column chunks
                    const int sgi = seg_of(out, nb);
                    const float dq = sgi == 0 ? deq : __fdiv_rn(gamma_p[sgi], scale[m]);
                    store_row_chunk(v, xs, dq, nb, N, static_cast<size_t>(m) * N + nb, out, vec);
                }
            }
            tc::fence_before_sync();
            tc::mbar_arrive(aempty(a));
        }
    }

    // ------------------------------------------------------------ teardown
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        if (lane == 0 && abort_sh) {
            // no MMA may still be writing TMEM when it is released
            tc::mma_commit(afull(0));
            tc::mbar_wait(afull(0), 0, WAIT_LIMIT_NS);
        }
        __syncwarp();
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, TMEM_COLS);
    }
}

// Dequantise and store 8 consecutive outputs of one row (stream-K fix-up).
__device__ __forceinline__ void store_row8(const uint32_t (&v)[8], int xs, float deq, int nb, int N, size_t o,
                                           const GemvOut& out, bool vec) {
    int a[8];
    float f[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        a[j] = static_cast<int>(v[j]) - xs;
        f[j] = dequant(a[j], deq);
    }
    if (vec && nb + 8 <= N) {
        if (out.y32) {
            *reinterpret_cast<float4*>(out.y32 + o) = make_float4(f[0], f[1], f[2], f[3]);
            *reinterpret_cast<float4*>(out.y32 + o + 4) = make_float4(f[4], f[5], f[6], f[7]);
        } else {
            uint4 r = make_uint4(0, 0, 0, 0);
            if (out.residual) r = *reinterpret_cast<const uint4*>(out.residual + o);
            const uint32_t rr[4] = {r.x, r.y, r.z, r.w};
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float lo = f[2 * e], hi = f[2 * e + 1];
                if (out.residual) {
                    lo = __fadd_rn(bf16_bits_to_f32(rr[e] & 0xffffu), lo);
                    hi = __fadd_rn(bf16_bits_to_f32(rr[e] >> 16), hi);
                }
                pk[e] = f32_to_bf16_bits(lo) | (static_cast<uint32_t>(f32_to_bf16_bits(hi)) << 16);
            }
            *reinterpret_cast<uint4*>(out.y + o) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        if (out.acc) {
            *reinterpret_cast<int4*>(out.acc + o) = make_int4(a[0], a[1], a[2], a[3]);
            *reinterpret_cast<int4*>(out.acc + o + 4) = make_int4(a[4], a[5], a[6], a[7]);
        }
        return;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        if (nb + j >= N) break;
        float v2 = f[j];
        if (out.y32) {
            out.y32[o + j] = v2;
        } else {
            if (out.residual) v2 = __fadd_rn(bf16_bits_to_f32(out.residual[o + j]), v2);
            out.y[o + j] = f32_to_bf16_bits(v2);
        }
        if (out.acc) out.acc[o + j] = a[j];
    }
}

// Stream-K fix-up: CTA (tile, 32-column chunk); a tile that one CTA finished
// returns at once, a split tile sums its pieces (slots of the CTAs whose ranges
// cover it) and runs the epilogue. Thread (quarter qd = tid / 128, row r = tid %
// 128) owns 8 columns of one row; the pieces are column-major, so each warp load
// reads one 128-byte line, and every piece's loads are in flight together.
template <int BN, bool PR>
__global__ void __launch_bounds__(512) gemm_sk_fixup_kernel(int M, int N, int K, int G,
                                                           const uint32_t* __restrict__ partials,
                                                           const float* __restrict__ gamma_p,
                                                           const float* __restrict__ scale,
                                                           const int32_t* __restrict__ xsum, GemvOut out) {
    grid_dependency_wait();
    const int n_tiles = (N + BN - 1) / BN;
    const int nkb = (K + BK - 1) / BK;
    const long long U = (long long)n_tiles * ((M + BM - 1) / BM) * nkb;
    const int tile = blockIdx.x;
    const long long t0 = (long long)tile * nkb, t1 = t0 + nkb;  // units of this tile
    // the CTA whose range [U c / G, U (c + 1) / G) holds unit u
    auto owner = [&](long long u) { return (int)(((u + 1) * G + U - 1) / U) - 1; };
    const int c_first = owner(t0), c_last = owner(t1 - 1);
    if (c_first == c_last) return;
    const int m0 = (tile / n_tiles) * BM, n0 = (tile % n_tiles) * BN;
    const int r = threadIdx.x & (BM - 1), qd = threadIdx.x / BM;
    const int m = m0 + r;
    const int col = blockIdx.y * 32 + qd * 8;  // first column of this thread inside the tile
    if (m >= M || n0 + col >= N) return;
    uint32_t v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = 0;
#pragma unroll 2
    for (int cta = c_first; cta <= c_last; ++cta) {
        const bool first_piece = (long long)(U * cta / G) >= t0;  // the range starts inside this tile
        const uint32_t* src =
            partials + (size_t)(2 * cta + (first_piece ? 0 : 1)) * BM * BN + (size_t)col * BM + r;
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] += src[(size_t)j * BM];
    }
    const bool vec = (N % 8 == 0) && aligned16(out.y) && aligned16(out.y32) && aligned16(out.residual) &&
                     aligned16(out.acc);
    if (PR) {
        store_row_per_row_gamma<8>(v, xsum[m], scale[m], gamma_p, n0 + col, N, static_cast<size_t>(m) * N + n0 + col,
                                   out);
        return;
    }
    store_row8(v, xsum[m], __fdiv_rn(gamma_p[seg_of(out, n0 + col)], scale[m]), n0 + col, N,
               static_cast<size_t>(m) * N + n0 + col, out, vec);
}

}  // namespace

// ---------------------------------------------------------------- host side
namespace {
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            cudaGetLastError();
    }
    return fn;
}
}  // namespace

bool make_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
              uint32_t box_cols, bool swizzle128) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool gemm_segments_ok(const GemvOut& out, int64_t N) {
    for (int i = 0; i < 3; ++i)
        if (out.seg_end[i] < N && out.seg_end[i] % 32 != 0) return false;
    return true;
}

bool gemm_tc_ok(int64_t N, int64_t K, const void* Wp, const void* xq) {
    return N >= 1 && K % 64 == 0 && reinterpret_cast<uintptr_t>(Wp) % 16 == 0 &&
           reinterpret_cast<uintptr_t>(xq) % 16 == 0;
}

namespace {
template <int BN, bool PR = false>
cudaError_t launch_bn(const uint8_t* Wp, const float* gamma, int64_t N, int64_t K, const int8_t* xq_g16t,
                      const float* scale, const int32_t* xsum, int64_t M, const GemvOut& out,
                      cudaStream_t s, int dev, int sms, uint32_t* partials) {
    constexpr size_t smem = TileCfg<BN>::SMEM_BYTES;
    CUtensorMap mapA, mapB;
    if (!make_map(&mapA, xq_g16t, (uint64_t)M, (uint64_t)K, BM, BK, true) ||
        !make_map(&mapB, Wp, (uint64_t)N, (uint64_t)(K / 4), BN, BK / 4, false))
        return cudaErrorInvalidValue;
    unsigned* err = nullptr;
    cudaError_t e = device_error_word(&err);
    if (e != cudaSuccess) return e;
    const bool sk = partials != nullptr;
    auto kern = sk ? gemm_tc_kernel<BN, true, PR> : gemm_tc_kernel<BN, false, PR>;
    static bool attr_set[64][2];
    if (dev >= 64 || !attr_set[dev][sk]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (dev < 64) attr_set[dev][sk] = true;
    }
    const int64_t tiles = ((N + BN - 1) / BN) * ((M + BM - 1) / BM);
    const int64_t units = tiles * ((K + BK - 1) / BK);
    const int64_t work = sk ? units : tiles;
    const unsigned grid = (unsigned)(work < sms ? work : sms);
    kern<<<grid, THREADS, smem, s>>>(mapA, mapB, mapB, (int)M, (int)N, (int)K, gamma, scale, xsum, out, err, partials,
                                     FfnUpOut());
    e = cudaGetLastError();
    if (e != cudaSuccess || !sk) return e;
    return launch_pdl(gemm_sk_fixup_kernel<BN, PR>, dim3((unsigned)tiles, BN / 32), dim3(512), 0, s, (int)M, (int)N,
                      (int)K, (int)grid, (const uint32_t*)partials, gamma, scale, xsum, out);
}
}  // namespace

cudaError_t launch_gemm_tc_dual(const uint8_t* Wg, const float* gg, const uint8_t* Wu, const float* gu, int64_t f,
                                int64_t d, const int8_t* xq_g16t, const float* scale, const int32_t* xsum, int64_t M,
                                const FfnUpOut& up, cudaStream_t s) {
    if (M == 0 || f == 0) return cudaSuccess;
    if (!gemm_tc_ok(f, d, Wg, xq_g16t) || !gemm_tc_ok(f, d, Wu, xq_g16t)) return cudaErrorInvalidValue;
    int dev = 0;
    cudaGetDevice(&dev);
    int sms = 148;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) sms = 148;
    constexpr int BN = 256;
    constexpr size_t smem = TileCfg<BN>::SMEM_BYTES;
    CUtensorMap mapA, mapG, mapU;
    if (!make_map(&mapA, xq_g16t, (uint64_t)M, (uint64_t)d, BM, BK, true) ||
        !make_map(&mapG, Wg, (uint64_t)f, (uint64_t)(d / 4), BN / 2, BK / 4, false) ||
        !make_map(&mapU, Wu, (uint64_t)f, (uint64_t)(d / 4), BN / 2, BK / 4, false))
        return cudaErrorInvalidValue;
    unsigned* err = nullptr;
    cudaError_t e = device_error_word(&err);
    if (e != cudaSuccess) return e;
    auto kern = gemm_tc_kernel<BN, false, false, true>;
    static bool attr_set[64];
    if (dev >= 64 || !attr_set[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (dev < 64) attr_set[dev] = true;
    }
    const int64_t tiles = ((f + BN / 2 - 1) / (BN / 2)) * ((M + BM - 1) / BM);
    const unsigned grid = (unsigned)(tiles < sms ? tiles : sms);
    FfnUpOut u = up;
    u.gamma_u = gu;
    kern<<<grid, THREADS, smem, s>>>(mapA, mapG, mapU, (int)M, (int)f, (int)d, gg, scale, xsum, GemvOut(), err,
                                     nullptr, u);
    return cudaGetLastError();
}

int gemm_dual_parts(int64_t f) { return (int)((f + 127) / 128); }

// Tile width: 256 weight rows per tile unless narrower tiles finish sooner. The
// estimate is waves x relative time of one tile; a narrower tile still loads the
// whole activation tile and pays the same per-k-block overheads, so on B200 a
// 128-row tile takes 0.68 and a 64-row tile 0.59 of a 256-row tile (measured).
namespace {
constexpr int kWidths[3] = {256, 128, 64};
constexpr double kTileCost[3] = {1.0, 0.68, 0.59};

// Estimated time (in 256-row tile times) and width of the best data-parallel plan.
double best_data_parallel(int64_t M, int64_t N, int sms, int* width) {
    const int64_t mt = (M + BM - 1) / BM;
    int best = 256;
    double best_time = 0.0;
    for (int i = 0; i < 3; ++i) {
        const int64_t tiles = mt * ((N + kWidths[i] - 1) / kWidths[i]);
        const double time = (double)((tiles + sms - 1) / sms) * kTileCost[i];
        if (i == 0 || time < best_time - 1e-9) {
            best = kWidths[i];
            best_time = time;
        }
    }
    *width = best;
    return best_time;
}
}  // namespace

int gemm_tc_tile_width(int64_t M, int64_t N, int sms) {
    int w = 256;
    best_data_parallel(M, N, sms, &w);
    return w;
}

size_t gemm_sk_workspace_bytes(int sms) { return (size_t)2 * sms * BM * 256 * sizeof(uint32_t); }


// Stream-K only where the best data-parallel plan leaves much of its last wave
// idle (under 70% of its CTA-slots busy), the tiles are long in K (at least 32
// k-blocks, so the pieces are large: each split tile costs a 128 KB write and
// read of int32 pieces plus the fix-up launch, which ate the gain on the other
// shapes measured: 2560 -> 6912 at M = 512, 6912 -> 2560 at M = 4096), and the
// plan stream-K actually runs (256-row tiles spread evenly over the SMs) is
// estimated faster than that data-parallel plan.
bool gemm_use_stream_k(int64_t M, int64_t N, int64_t K, int sms) {
    const int64_t mt = (M + BM - 1) / BM;
    int bn = 256;
    const double dp_time = best_data_parallel(M, N, sms, &bn);
    const int64_t dp_tiles = mt * ((N + bn - 1) / bn);
    const int64_t waves = (dp_tiles + sms - 1) / sms;
    const double busy = (double)dp_tiles / (double)(waves * sms);
    const double sk_time = (double)(mt * ((N + 255) / 256)) / (double)sms;
    return busy < 0.7 && (K + BK - 1) / BK >= 32 && sk_time < dp_time;
}

cudaError_t launch_gemm_tc(const uint8_t* Wp, const float* gamma, int64_t N, int64_t K,
                           const int8_t* xq_g16t, const float* scale, const int32_t* xsum, int64_t M,
                           const GemvOut& out, cudaStream_t s, void* sk_ws, size_t sk_ws_bytes) {
    if (M == 0 || N == 0) return cudaSuccess;
    int dev = 0;
    cudaGetDevice(&dev);
    static int num_sms[64];
    if (dev < 64 && !num_sms[dev]) {
        cudaError_t e = cudaDeviceGetAttribute(&num_sms[dev], cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
    }
    const int sms = dev < 64 ? num_sms[dev] : 148;
    const bool sk_ok = sk_ws && sk_ws_bytes >= gemm_sk_workspace_bytes(sms) && gemm_use_stream_k(M, N, K, sms);
    if (out.per_row)  // the per-row gamma variant runs 256-row tiles only
        return launch_bn<256, true>(Wp, gamma, N, K, xq_g16t, scale, xsum, M, out, s, dev, sms,
                                    sk_ok ? static_cast<uint32_t*>(sk_ws) : nullptr);
    if (sk_ok)
        return launch_bn<256>(Wp, gamma, N, K, xq_g16t, scale, xsum, M, out, s, dev, sms,
                              static_cast<uint32_t*>(sk_ws));
    switch (gemm_tc_tile_width(M, N, sms)) {
        case 64: return launch_bn<64>(Wp, gamma, N, K, xq_g16t, scale, xsum, M, out, s, dev, sms, nullptr);
        case 128: return launch_bn<128>(Wp, gamma, N, K, xq_g16t, scale, xsum, M, out, s, dev, sms, nullptr);
        default: return launch_bn<256>(Wp, gamma, N, K, xq_g16t, scale, xsum, M, out, s, dev, sms, nullptr);
    }
}

}  // namespace bl

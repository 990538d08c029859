// Tensor-core GEMV for up to 16 tokens: acc[m, n] = sum_k Wq[n, k] * xq[m, k].
//
// Paper card "BitNet b1.58 2B4T Technical Report", "Method Adaptation": packed
// int8 weights are loaded into on-chip memory, unpacked right before the int8
// matmul and multiplied with the int8 activations. Here the weights take the
// 128-row side of a 5th-generation tensor-core MMA and the few tokens its
// N = 8 or 16 side (the transposed product D[n, m] = A[n, k] B[m, k]), so a
// handful of tokens costs no more MMA issue than one:
//   TMA:     packed weight tile [128 rows x 128 bytes = 512 codes] (128-byte
//            swizzle) and the token codes [8 or 16 tokens x 128 codes] per
//            128-code block -> shared memory;
//   unpack:  four warps, one weight row per thread, read the row's 128 bytes
//            (conflict-free thanks to the swizzle), split every packed word into
//            its four 2-bit fields (code bytes 0..2) and write them straight into
//            tensor memory with tcgen05.st: 32 columns per 128 codes. The
//            unpacked weights never go through shared memory;
//   MMA:     one thread issues tcgen05.mma kind::i8 with A (unsigned codes) read
//            from tensor memory and B (signed activation codes) from shared
//            memory into 128 x N int32 accumulators in tensor memory. At N = 8 or
//            16 an MMA is short, so one accumulator would make every MMA wait for
//            the previous one's result; the K steps rotate over eight
//            accumulators instead, and the MMAs overlap in the tensor pipe;
//   epilogue: the same four warps read and sum the accumulators (tcgen05.ld),
//            subtract the code offset (sum_k xq), dequantise and store.
// The i-th field of packed word j of a row holds the codes of k = 16 j + 4 b + i
// (byte b); written to column 4 j + i, the A operand's K order is exactly the
// G16T order in which the act-quant kernel stores the token codes, so A and B
// agree without any byte shuffling.
//
// Work split: one CTA per (128-row tile, K range). When the tiles alone cannot
// fill the GPU, K is split across a cluster of up to 8 CTAs; every CTA but the
// first adds its int32 partial sums into the first CTA's shared memory with
// asynchronous remote adds (red.async ... complete_tx, counted on one mbarrier),
// and the first CTA runs the epilogue. No global scratch, no second kernel.
//
// Every mbarrier wait is bounded (1 s); a wait that gives up sets the device
// error word (reported as BL_ERR_TIMEOUT), the CTA stops issuing work, lets its
// copies and MMAs finish, writes nothing, and returns.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace bl {
namespace {

constexpr int WROWS = 128;                          // weight rows per tile: TMEM lanes, MMA M
constexpr int SUB = 128;                            // codes per TMEM A block (32 packed bytes per row)
constexpr int SUBS = 4;                             // A blocks fed by one shared-memory stage
constexpr int STAGE_CODES = SUB * SUBS;             // 512 codes = 128 packed bytes per row
constexpr int P_BYTES = WROWS * STAGE_CODES / 4;    // 16 KiB of packed weights per stage
constexpr int AS = 4;                               // TMEM A blocks in flight (32 columns each)
constexpr int ND = 8;                               // independent accumulators (summed at the end)
constexpr uint32_t D_COL = 32 * AS;                 // first TMEM column of the accumulators
constexpr uint32_t TMEM_COLS = 256;                 // A blocks + ND x 16 accumulator columns
constexpr int THREADS = 192;                        // TMA warp, MMA warp, 4 unpack / epilogue warps
constexpr int MAX_SPLIT = 8;                        // portable cluster size
constexpr uint64_t WAIT_NS = 1000000000ull;

template <int BNT>
struct TcCfg {
    static constexpr int B_BYTES = BNT * SUB;                 // token codes of one 128-code block
    static constexpr int TS = BNT == 8 ? 5 : 4;               // shared-memory stages (2 CTAs per SM)
    static constexpr int STAGE_BYTES = P_BYTES + SUBS * B_BYTES;
    static constexpr int RED_WORDS = WROWS * BNT;             // leader's reduction buffer
    static constexpr int NUM_BARS = 2 * TS + 2 * AS + 3;
    static constexpr size_t SMEM = 1024 + (size_t)TS * STAGE_BYTES + RED_WORDS * 4 + 16 + NUM_BARS * 8;
    static_assert(SMEM <= 113 * 1024, "two CTAs per SM");
    static_assert(D_COL + ND * BNT <= TMEM_COLS, "tensor memory budget");
};

struct TcArgs {
    int N, K, M;
    int split;             // CTAs per cluster: the K split of one tile
    const float* gamma;
    const float* scale;
    const int32_t* xsum;
    GemvOut out;
    unsigned* err;
};

__device__ __forceinline__ bool is_aborted(const int* flag) {
    return *reinterpret_cast<const volatile int*>(flag) != 0;
}

__device__ __forceinline__ void give_up(unsigned* err, int* flag) {
    atomicOr(err, 1u);
    atomicExch(flag, 1);
}

// Codes of 128-code block j of a stage that lie inside K (the last stage may hold fewer).
__device__ __forceinline__ int blocks_in_stage(int s, int K) {
    return min(SUBS, (K - s * STAGE_CODES) / SUB);
}

// XT: row segments with their own gamma or one gamma per row (the plain forward
// runs the instantiation without that code).
template <int BNT, bool XT>
__global__ void __launch_bounds__(THREADS, 2)
    gemv_tc_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                   const TcArgs a) {
    using C = TcCfg<BNT>;
    constexpr int TS = C::TS;
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;

    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* sP = smem;                                       // TS x P_BYTES (1024-aligned)
    uint8_t* sB = sP + TS * P_BYTES;                          // TS x SUBS x B_BYTES
    uint32_t* red = reinterpret_cast<uint32_t*>(sB + TS * SUBS * C::B_BYTES);  // [BNT][128]
    uint32_t* peer_abort = red + C::RED_WORDS;                // leader: sum of the peers' abort flags
    uint64_t* bars = reinterpret_cast<uint64_t*>(peer_abort + 4);
    auto bar = [&](int i) { return tc::smem_u32(bars + i); };
    auto tfull = [&](int s) { return bar(s); };                   // TMA landed
    auto tempty = [&](int s) { return bar(TS + s); };             // unpack warps and MMAs done with it
    auto afull = [&](int b) { return bar(2 * TS + b); };          // A block written to TMEM
    auto aempty = [&](int b) { return bar(2 * TS + AS + b); };    // MMAs done with the A block
    const uint32_t dfull = bar(2 * TS + 2 * AS);                  // accumulator final
    const uint32_t redfull = bar(2 * TS + 2 * AS + 1);            // leader: every peer's sums added
    const uint32_t drain = bar(2 * TS + 2 * AS + 2);              // teardown after an abort

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t S = (uint32_t)a.split;                         // CTAs per cluster (K split)
    const uint32_t rank = tc::cluster_ctarank();                  // = blockIdx.x % S
    const int n0 = (int)(blockIdx.x / S) * WROWS;
    const int K = a.K;
    const int nst = (K + STAGE_CODES - 1) / STAGE_CODES;
    const int st0 = (int)((long long)nst * rank / S), st1 = (int)((long long)nst * (rank + 1) / S);

    if (threadIdx.x == 0) {
        for (int s = 0; s < TS; ++s) {
            tc::mbar_init(tfull(s), 1);
            tc::mbar_init(tempty(s), 1 + 4);  // one MMA commit + one arrive per unpack warp
        }
        for (int b = 0; b < AS; ++b) {
            tc::mbar_init(afull(b), 128);
            tc::mbar_init(aempty(b), 1);
        }
        tc::mbar_init(dfull, 1);
        tc::mbar_init(redfull, 1);
        tc::mbar_init(drain, 1);
        abort_sh = 0;
        tc::fence_mbar_init();
    }
    if (rank == 0 && S > 1) {  // the peers add into the leader's buffer
        for (int i = threadIdx.x; i < C::RED_WORDS + 4; i += THREADS) red[i] = 0;
    }
    if (warp == 1) {
        tc::tmem_alloc(tc::smem_u32(&tmem_base_sh), TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (rank == 0 && S > 1 && threadIdx.x == 0)
        tc::mbar_arrive_expect_tx(redfull, (S - 1) * (uint32_t)(C::RED_WORDS * 4 + 4));
    // every CTA's barriers and the leader's zeroed buffer exist before any remote access
    tc::cluster_sync();
    grid_dependents_launch();
    const uint32_t tmem = tmem_base_sh;

    bool ok = true;  // this thread's role finished without giving up
    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tc::prefetch_tmap(&tmW);
            tc::prefetch_tmap(&tmX);
            // before the dependency wait only L2 prefetches of the weights run: they
            // write no shared memory, and L2 is the point of coherence
            for (int s = st0; s < st1 && s < st0 + TS; ++s) tc::tma_prefetch_2d(&tmW, s * (STAGE_CODES / 4), n0);
            grid_dependency_wait();
            uint32_t g = 0;
            for (int s = st0; s < st1; ++s, ++g) {
                const int stg = g % TS;
                if (g >= (uint32_t)TS && !tc::mbar_wait(tempty(stg), ((g / TS) - 1) & 1, WAIT_NS)) {
                    give_up(a.err, &abort_sh);
                    ok = false;
                    break;
                }
                if (is_aborted(&abort_sh)) {
                    ok = false;
                    break;
                }
                const int nb = blocks_in_stage(s, K);
                tc::mbar_arrive_expect_tx(tfull(stg), (uint32_t)(P_BYTES + nb * C::B_BYTES));
                tc::tma_load_2d(tc::smem_u32(sP + stg * P_BYTES), &tmW, s * (STAGE_CODES / 4), n0, tfull(stg));
                for (int j = 0; j < nb; ++j)
                    tc::tma_load_2d(tc::smem_u32(sB + (stg * SUBS + j) * C::B_BYTES), &tmX, s * STAGE_CODES + j * SUB,
                                    0, tfull(stg));
            }
            if (!ok) {
                // let the copies still in flight land before the CTA exits
                const uint32_t first = g > (uint32_t)TS ? g - TS : 0;
                for (uint32_t h = first; h < g; ++h) tc::mbar_wait(tfull(h % TS), (h / TS) & 1, WAIT_NS);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = tc::idesc_i8_u8s8(WROWS, BNT);
            uint32_t g = 0, h = 0;
            for (int s = st0; s < st1 && ok; ++s, ++g) {
                const int stg = g % TS;
                if (is_aborted(&abort_sh) || !tc::mbar_wait(tfull(stg), (g / TS) & 1, WAIT_NS)) {
                    give_up(a.err, &abort_sh);
                    ok = false;
                    break;
                }
                const int nb = blocks_in_stage(s, K);
                for (int j = 0; j < nb; ++j, ++h) {
                    const int ab = h % AS;
                    if (!tc::mbar_wait(afull(ab), (h / AS) & 1, WAIT_NS)) {
                        give_up(a.err, &abort_sh);
                        ok = false;
                        break;
                    }
                    tc::fence_after_sync();
                    const uint64_t bd = tc::desc_kmajor_sw128(tc::smem_u32(sB + (stg * SUBS + j) * C::B_BYTES));
                    // 32 codes per MMA (+2 in 16-byte units); K step kk of block h goes to
                    // accumulator 4 (h % 2) + kk, first written by block 0 or 1 (every
                    // CTA has at least two blocks: K % 256 == 0)
                    const uint32_t dh = tmem + D_COL + (uint32_t)((h & 1) * 4 * BNT);
#pragma unroll
                    for (int kk = 0; kk < SUB / 32; ++kk)
                        tc::mma_i8_tmem_a(dh + kk * BNT, tmem + 32 * ab + 8 * kk, bd + 2 * kk, idesc,
                                          h >= 2 ? 1u : 0u);
                    tc::mma_commit(aempty(ab));
                }
                if (!ok) break;
                tc::mma_commit(tempty(stg));
            }
            // arrives once every MMA issued above has completed (also after an abort)
            tc::mma_commit(dfull);
        }
    } else {
        // ------------------------------------------------------------ unpack
        const int q = warp & 3;  // the TMEM lane quarter this warp may access
        const int r = 32 * q + lane;
        const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
        uint32_t g = 0, h = 0;
        for (int s = st0; s < st1; ++s, ++g) {
            const int stg = g % TS;
            const bool got = !is_aborted(&abort_sh) && tc::mbar_wait(tfull(stg), (g / TS) & 1, WAIT_NS);
            if (!__all_sync(0xffffffffu, got)) {  // tcgen05.st below is warp-collective
                give_up(a.err, &abort_sh);
                ok = false;
                break;
            }
            // this row's 128 packed bytes: 16-byte chunk c sits at position c ^ (r % 8)
            const uint8_t* rowp = sP + stg * P_BYTES + r * 128;
            uint4 pk[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) pk[c] = *reinterpret_cast<const uint4*>(rowp + ((c ^ (r & 7)) << 4));
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(tempty(stg));
            const int nb = blocks_in_stage(s, K);
#pragma unroll
            for (int j = 0; j < SUBS; ++j) {
                if (j >= nb) break;
                const int ab = h % AS;
                const bool free_ = h < (uint32_t)AS || tc::mbar_wait(aempty(ab), ((h / AS) - 1) & 1, WAIT_NS);
                if (!__all_sync(0xffffffffu, free_)) {
                    give_up(a.err, &abort_sh);
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                const uint32_t words[8] = {pk[2 * j].x,     pk[2 * j].y,     pk[2 * j].z,     pk[2 * j].w,
                                           pk[2 * j + 1].x, pk[2 * j + 1].y, pk[2 * j + 1].z, pk[2 * j + 1].w};
                uint32_t v[32];
#pragma unroll
                for (int w = 0; w < 8; ++w)
#pragma unroll
                    for (int i = 0; i < 4; ++i) v[4 * w + i] = (words[w] >> (2 * i)) & 0x03030303u;
                tc::tmem_st_32x32(tmem + lane_base + 32 * ab, v);
                tc::tmem_st_wait();
                tc::fence_before_sync();
                tc::mbar_arrive(afull(ab));
                ++h;
            }
            if (!ok) break;
        }

        // ------------------------------------------------------------ epilogue
        grid_dependency_wait();  // scale, xsum and residual come from earlier kernels
        bool have = ok && tc::mbar_wait(dfull, 0, WAIT_NS);
        have = __all_sync(0xffffffffu, have) && !is_aborted(&abort_sh);
        uint32_t v[BNT];
#pragma unroll
        for (int c = 0; c < BNT; ++c) v[c] = 0;
        if (have) {
            tc::fence_after_sync();
            // the ND accumulators are ND x BNT consecutive columns; column j of a
            // 32-column load belongs to token j % BNT
#pragma unroll
            for (int c = 0; c < ND * BNT / 32; ++c) {
                uint32_t t[32];
                tc::tmem_ld_32x32(tmem + lane_base + D_COL + 32 * c, t);
                tc::tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j % BNT] += t[j];
            }
        } else if (ok) {
            give_up(a.err, &abort_sh);
        }
        if (rank != 0) {
            // add this CTA's partial sums into the leader's buffer; one thread also
            // adds this CTA's abort flag (every peer always sends the same bytes)
            const uint32_t rbase = tc::map_to_rank(tc::smem_u32(red), 0);
            const uint32_t rbar = tc::map_to_rank(redfull, 0);
#pragma unroll
            for (int c = 0; c < BNT; ++c) tc::red_add_remote(rbase + (uint32_t)(c * WROWS + r) * 4u, v[c], rbar);
            if (threadIdx.x == 64) {
                const uint32_t flag = (uint32_t)is_aborted(&abort_sh) | (have ? 0u : 1u);
                tc::red_add_remote(tc::map_to_rank(tc::smem_u32(peer_abort), 0), flag, rbar);
            }
        } else {
            bool all = have;
            if (S > 1) {
                const bool got = tc::mbar_wait(redfull, 0, WAIT_NS);
                if (!got) give_up(a.err, &abort_sh);
                all = all && got && *reinterpret_cast<volatile uint32_t*>(peer_abort) == 0;
                if (all) {
#pragma unroll
                    for (int c = 0; c < BNT; ++c) v[c] += red[c * WROWS + r];
                }
            }
            const int n = n0 + r;
            if (all && n < a.N) {
                const float gam = a.gamma[XT ? gamma_index(a.out, n) : 0];
#pragma unroll
                for (int m = 0; m < BNT; ++m) {
                    if (m >= a.M) break;
                    const int accv = static_cast<int>(v[m]) - a.xsum[m];
                    float y = dequant(accv, __fdiv_rn(gam, a.scale[m]));
                    const size_t o = (size_t)m * a.N + n;
                    if (a.out.y32) {
                        a.out.y32[o] = y;
                    } else {
                        if (a.out.residual) y = __fadd_rn(bf16_bits_to_f32(a.out.residual[o]), y);
                        a.out.y[o] = f32_to_bf16_bits(y);
                    }
                    if (a.out.acc) a.out.acc[o] = accv;
                }
            }
        }
    }

    // ------------------------------------------------------------ teardown
    tc::fence_before_sync();
    __syncthreads();
    // the peers stay resident until the leader has read their sums
    tc::cluster_sync();
    if (warp == 1) {
        if (lane == 0 && is_aborted(&abort_sh)) {
            // no MMA may still be writing TMEM when it is released
            tc::mma_commit(drain);
            tc::mbar_wait(drain, 0, WAIT_NS);
        }
        __syncwarp();
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, TMEM_COLS);
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

template <int BNT, bool XT>
cudaError_t launch_bnt(const CUtensorMap& mW, const CUtensorMap& mX, const TcArgs& a, int split, int n_tiles,
                       cudaStream_t s) {
    auto kern = gemv_tc_kernel<BNT, XT>;
    constexpr size_t smem = TcCfg<BNT>::SMEM;
    static bool done[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64 || !done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (dev < 64) done[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(split * n_tiles));  // cluster c = tile c, its CTAs split K
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)split;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, mW, mX, a);
}

}  // namespace

bool gemv_tc_ok(int64_t N, int64_t K, int64_t M, const void* Wp, const void* xq) {
    return N >= 1 && M >= 1 && M <= 16 && K % 256 == 0 && reinterpret_cast<uintptr_t>(Wp) % 16 == 0 &&
           reinterpret_cast<uintptr_t>(xq) % 16 == 0;
}

// K split: the split whose estimated time is shortest, where a CTA's time is its
// stages plus one stage of fixed cost, two CTAs share an SM, and waves of CTAs
// follow one another. Every CTA keeps at least one stage.
int gemv_tc_split(int64_t N, int64_t K, int sms) {
    const int64_t tiles = (N + WROWS - 1) / WROWS;
    const int64_t nst = (K + STAGE_CODES - 1) / STAGE_CODES;
    const int64_t slots = 2 * (int64_t)sms;
    int best = 1;
    double best_t = 0.0;
    for (int S = 1; S <= MAX_SPLIT && S <= nst; ++S) {
        const int64_t ctas = tiles * S;
        const int64_t waves = (ctas + slots - 1) / slots;
        const double t = (double)waves * ((double)((nst + S - 1) / S) + 1.0);
        if (S == 1 || t < best_t - 1e-9) {
            best = S;
            best_t = t;
        }
    }
    return best;
}

cudaError_t launch_gemv_tc(const uint8_t* Wp, const float* gamma, int64_t N, int64_t K,
                           const int8_t* xq_g16t, const float* scale, const int32_t* xsum, int64_t M,
                           const GemvOut& out, cudaStream_t s) {
    if (M == 0 || N == 0) return cudaSuccess;
    if (!gemv_tc_ok(N, K, M, Wp, xq_g16t)) return cudaErrorInvalidValue;
    const int bnt = M <= 8 ? 8 : 16;
    CUtensorMap mW, mX;
    if (!make_map(&mW, Wp, (uint64_t)N, (uint64_t)(K / 4), WROWS, STAGE_CODES / 4, true) ||
        !make_map(&mX, xq_g16t, (uint64_t)M, (uint64_t)K, (uint32_t)bnt, SUB, true))
        return cudaErrorInvalidValue;
    TcArgs a;
    a.N = (int)N;
    a.K = (int)K;
    a.M = (int)M;
    a.gamma = gamma;
    a.scale = scale;
    a.xsum = xsum;
    a.out = out;
    cudaError_t e = device_error_word(&a.err);
    if (e != cudaSuccess) return e;
    const int split = gemv_tc_split(N, K, sm_count());
    const int n_tiles = (int)((N + WROWS - 1) / WROWS);
    a.split = split;
    const bool xt = out.seg_end[0] < N || out.per_row;
    if (bnt == 8)
        return xt ? launch_bnt<8, true>(mW, mX, a, split, n_tiles, s) : launch_bnt<8, false>(mW, mX, a, split, n_tiles, s);
    return xt ? launch_bnt<16, true>(mW, mX, a, split, n_tiles, s) : launch_bnt<16, false>(mW, mX, a, split, n_tiles, s);
}

}  // namespace bl

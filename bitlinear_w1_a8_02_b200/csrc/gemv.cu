// Decode GEMV for M <= 16 tokens: acc[m, n] = sum_k Wq[n, k] * xq[m, k].
//
// Paper card "BitNet b1.58 2B4T Technical Report", "Method Adaptation": the
// packed int8 weights are loaded on chip, unpacked right before the matmul and
// multiplied with the int8 activations (pack-store-load-unpack-compute). Here a
// producer warp copies the packed rows with 1-D bulk copies (TMA engine) into a
// ring of shared-memory stages; eight consumer warps read them into registers,
// unpack there with one AND per 4 codes and feed int8 tensor-core MMAs
// (m16n8k32, u8 weights x s8 activations, int32 accumulators). Each weight byte
// is read from DRAM once.
//
// Unpacking without shifts. A packed 32-bit word holds 16 codes c = q + 1; the
// i-th 2-bit field of its 4 bytes is (word & (0x03030303 << 2i)), i.e. the codes
// of k = 4j + i times 4^i. Each field i gets its own accumulator; at the end
// acc_u = A0 + A1/4 + A2/16 + A3/64 (each Ai is an exact multiple of 4^i) and
// acc = acc_u - sum_k xq (the +1 offset of the codes). The activation operand
// is laid out in PLANES (plane i holds xq[4j + i] at byte j), so a field of a
// weight word and a word of plane i cover the same k.
//
// Work split: persistent CTAs walk units of 16 output rows x one K segment
// (at most 32 KiB of packed weights: 2 KiB of each row; a single token uses 8- or
// 4-row units for long rows or few row tiles); the 8 warps of a CTA split a unit
// in 64-byte column chunks, partial sums meet in shared memory and the
// dequantisation epilogue is fused. Before the dependency wait each CTA asks for
// its first tiles to be prefetched into L2, so DRAM already streams while the
// previous kernel ends.
//
// Single token (DP): an 8-column MMA would spend 7 columns on padding, so each
// thread instead owns 4 rows of the unit and every 64th packed word, and runs one
// dp4a per 2-bit field against the token's plane words, which the quantiser
// stores interleaved (the four plane words of a 16-code group side by side).
//
// Fused activation quantisation: when the codes of all M (<= 4) tokens fit in
// shared memory, each CTA quantises x itself (absmax per token, then PLANES codes
// into shared memory), so a forward call is one kernel. Where x fits in the
// threads' registers (one token; two or four tokens of short rows) it is read
// once and quantised from registers after one barrier; otherwise a two-pass loop
// reads it twice. Without fusion the codes come from the act-quant kernel
// through the workspace.
//
// Extended calls (XT): row segments with their own gamma (stacked projections),
// one gamma per row, and a unit-weight RMSNorm of x before the quantisation are
// compiled into separate instantiations; the plain forward's code stays as small
// as before (its prologue runs once per launch from a cold instruction cache).
//
// Programmatic dependent launch: before waiting for the previous kernel in the
// stream (griddepcontrol.wait) a CTA issues L2 prefetches of its weights, which
// cannot observe stale data (L2 is the point of coherence), sets up its barriers,
// and its producer copies the first kStages weight units into the ring. The
// packed weights are read-only to every kernel of the library, so a kernel that
// lets this one start early is not writing them; the public header states the
// same condition for a caller's own kernels. Every global load of other data and
// every store comes after the wait.
#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace bl {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;
constexpr int kUnroll = 4;
constexpr int kPrefetchAhead = 2;          // tiles of lookahead per CTA
constexpr int kFusedSmemLimit = 48 * 1024;  // codes of all tokens in shared memory
constexpr int kFusedMaxTokens = 4;          // beyond this the separate quantiser is faster
constexpr int kStages = 2;                  // shared-memory ring of streamed weight units (2 CTAs per SM)
constexpr int kMaxSegChunks = 32;           // 64-byte chunks of each row per 16-row unit (2 KiB)
constexpr uint64_t kWaitLimitNs = 1000000000ull;
constexpr size_t kMaxDynSmem = 200 * 1024;  // dynamic shared memory limit set on every instantiation


__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

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

// dp4a of the four 2-bit fields of a packed weight word (unsigned bytes code * 4^i)
// against the four plane words of one token (signed bytes), one accumulator per field.
__device__ __forceinline__ void dp4a_fields(int (&acc)[4], uint32_t w, const uint4& x) {
    const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
        asm("dp4a.u32.s32 %0, %1, %2, %0;" : "+r"(acc[i]) : "r"(w & (0x03030303u << (2 * i))), "r"(xw[i]));
}

// acc_u = A0 + A1 / 4 + A2 / 16 + A3 / 64; each Ai is an exact multiple of 4^i.
__device__ __forceinline__ int fold_fields(const int (&acc)[4]) {
    return acc[0] + (acc[1] >> 2) + (acc[2] >> 4) + (acc[3] >> 6);
}

struct GemvArgs {
    const uint8_t* Wp;
    const float* gamma;
    int N, KB, M;
    const uint16_t* x;     // bf16 input (fused quantisation)
    const int8_t* Xp;      // PLANES codes (not fused)
    const float* scale;    // [M] (not fused)
    const int32_t* xsum;   // [M] (not fused)
    GemvOut out;
    unsigned* err;         // device error word (bounded waits that give up)
    int norm;              // fused quantisation: unit-weight RMSNorm of x first
    int seg_chunks;        // 64-byte chunks per K segment of a streamed unit
    int unit_rows;         // rows per streamed unit: 16, or 8 / 4 for one token with long rows
    int rg_shift;          // one token: log2(threads per group of 4 rows) = log2(1024 / unit_rows)
    int pitch;             // shared-memory row pitch of a stage
    int codes_bytes;       // fused codes area at the start of dynamic shared memory
    // second weight stream (FFN up: Wp = gate, Wp2 = up; same rows, same codes)
    const uint8_t* Wp2;
    const float* gamma2;
    float* h;              // FFN up output: h = relu(g)^2 * u, [M, N] fp32
    double* part_ss;       // FFN up output: per (token, 16-row tile) sum of h^2
    float* part_max;       // FFN up output: per (token, 16-row tile) max |h|
    // FFN down input (SRC_H): h [M, K] fp32 and the per-tile partials of the up kernel
    const float* hin;
    const double* hin_ss;
    const float* hin_max;
    int hin_parts;         // tiles of the up projection (= ceil(K / 16))
};

// Where the activation codes of a streamed GEMV come from.
enum GemvSrc : int {
    SRC_CODES = 0,  // PLANES codes (+ scale, code sum) from the act-quant kernel
    SRC_X = 1,      // bf16 x, quantised per token inside the kernel
    SRC_H = 2,      // fp32 h of the FFN up kernel: subln RMSNorm + requant inside the kernel
};

// Named barrier of the eight consumer warps (the producer warp is not in it).
__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// Byte offset of plane i of token m in the fused shared-memory code buffer. The
// +64 per token keeps the tokens of one quarter-warp on different banks.
__device__ __forceinline__ int smem_plane_off(int m, int i, int KB) { return m * (4 * KB + 64) + i * KB; }

// Per-token quantisation inside the kernel. It runs once per launch from a cold
// instruction cache, so code size rather than arithmetic sets its latency: the
// loops stay rolled and each token costs one barrier.

__device__ __forceinline__ uint32_t bf16x2_max(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// max |x| over 16 bf16 values, returned as a bf16 bit pattern (sign bits cleared,
// so the patterns order like the values).
__device__ __forceinline__ uint32_t absmax16(uint4 v0, uint4 v1) {
    constexpr uint32_t k = 0x7fff7fffu;
    const uint32_t a = bf16x2_max(bf16x2_max(v0.x & k, v0.y & k), bf16x2_max(v0.z & k, v0.w & k));
    const uint32_t b = bf16x2_max(bf16x2_max(v1.x & k, v1.y & k), bf16x2_max(v1.z & k, v1.w & k));
    const uint32_t c = bf16x2_max(a, b);
    return max(c & 0xffffu, c >> 16);
}

// sum of the squares of 16 bf16 values in fp64 (each square is exact there)
__device__ __forceinline__ double sumsq16(uint4 v0, uint4 v1) {
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    double ss = 0.0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const double lo = (double)__uint_as_float(w[j] << 16), hi = (double)__uint_as_float(w[j] & 0xffff0000u);
        ss = __fma_rn(lo, lo, ss);
        ss = __fma_rn(hi, hi, ss);
    }
    return ss;
}

// PLANES codes of 16 consecutive elements k = 16 g + e with fp32 values f[e]:
// code rint(f s), taken from the low byte of fl(f s) + 1.5 * 2^23. The per-token
// scale keeps |f s| <= 127 (1 + 2^-23) for finite inputs, so the clip to
// [-128, 127] cannot bite and is left out. Plane i receives the codes of
// e = i, 4 + i, 8 + i, 12 + i as one word, stored at plane0 + i * KB, or, in the
// interleaved single-token layout (IL), the four plane words of group g side by
// side at plane0 = codes + 16 g. Returns the sum of the 16 codes.
template <bool IL>
__device__ __forceinline__ int quant_pack16(const float (&f)[16], float s, uint8_t* plane0, int KB) {
    uint32_t u[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) u[e] = __float_as_uint(__fadd_rn(__fmul_rn(f[e], s), 12582912.0f));
    uint32_t w[4];
    int sum = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        w[i] = __byte_perm(__byte_perm(u[i], u[4 + i], 0x0040), __byte_perm(u[8 + i], u[12 + i], 0x0040), 0x5410);
        sum = __dp4a(static_cast<int>(w[i]), 0x01010101, sum);
    }
    if (IL) {
        *reinterpret_cast<uint4*>(plane0) = make_uint4(w[0], w[1], w[2], w[3]);
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) *reinterpret_cast<uint32_t*>(plane0 + i * KB) = w[i];
    }
    return sum;
}

// Shared-memory address of the code words of 16-element group c of token m.
template <bool IL>
__device__ __forceinline__ uint8_t* group_codes(uint8_t* codes, int m, int c, int KB) {
    return IL ? codes + 16 * c : codes + smem_plane_off(m, 0, KB) + 4 * c;
}

// XT and norm: the codes of fl(x * r) (RMSNorm factor r)
template <bool IL, bool XT>
__device__ __forceinline__ int quant_bf16x16(uint4 v0, uint4 v1, float s, uint8_t* plane0, int KB, bool norm,
                                             float r) {
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    float f[16];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        f[2 * j] = __uint_as_float(w[j] << 16);
        f[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
    }
    if (XT && norm) {
#pragma unroll
        for (int e = 0; e < 16; ++e) f[e] = __fmul_rn(f[e], r);
    }
    return quant_pack16<IL>(f, s, plane0, KB);
}

// bf16 x [M, K] -> PLANES codes of each token in shared memory (consumer threads).
// Per token: absmax (warp reduction, one barrier), s = 127 / max(amax, eps),
// codes, and the code sum. Thread 0 records s and the dequantisation factors
// gamma / s. The first 16-element group of the next token is loaded while the
// current one is reduced.
// XT: the call may ask for the RMSNorm (a.norm); without it the norm code is
// compiled out (this prologue's size is its latency).
template <bool DUAL, bool IL, bool XT>
__device__ void fused_quantise(const GemvArgs& a, int KB, uint8_t* codes, uint32_t (*am_sh)[kWarps],
                               double (*ss_sh)[kWarps], float* s_sh, int* xs_sh, float* deq_sh,
                               float* deq2_sh) {
    const int M = a.M, groups = KB / 4;  // 16-element groups per token
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c0 = threadIdx.x;
    const uint4* xv = reinterpret_cast<const uint4*>(a.x);
    float gamma = 0.0f, gamma2 = 0.0f;
    if (threadIdx.x == 0) {
        gamma = *a.gamma;
        if (DUAL) gamma2 = *a.gamma2;
    }
    uint4 n0 = make_uint4(0, 0, 0, 0), n1 = n0;
    if (c0 < groups) {
        n0 = xv[2 * c0];
        n1 = xv[2 * c0 + 1];
    }
#pragma unroll 1
    for (int m = 0; m < M; ++m) {
        const uint4* xr = xv + (size_t)m * 2 * groups;
        const uint4 v0 = n0, v1 = n1;
        if (m + 1 < M && c0 < groups) {
            n0 = xr[2 * groups + 2 * c0];
            n1 = xr[2 * groups + 2 * c0 + 1];
        }
        uint32_t mx = absmax16(v0, v1);  // 0 when this thread has no group
        const bool norm = XT && a.norm;
        double ss = norm ? sumsq16(v0, v1) : 0.0;
#pragma unroll 1
        for (int c = c0 + kThreads; c < groups; c += kThreads) {
            const uint4 w0 = xr[2 * c], w1 = xr[2 * c + 1];
            mx = max(mx, absmax16(w0, w1));
            if (norm) ss += sumsq16(w0, w1);
        }
        mx = __reduce_max_sync(0xffffffffu, mx);
        if (norm) ss = warp_sum(ss);
        if (lane == 0) {
            am_sh[m][warp] = mx;
            if (XT) ss_sh[m][warp] = ss;
        }
        consumer_sync();
        uint32_t amb = am_sh[m][0];
#pragma unroll
        for (int w = 1; w < kWarps; ++w) amb = max(amb, am_sh[m][w]);
        float amax = __uint_as_float(amb << 16), r = 1.0f;
        if (norm) {  // unit-weight RMSNorm: max |fl(x r)| = fl(max |x| r)
            double tot = ss_sh[m][0];
#pragma unroll
            for (int w = 1; w < kWarps; ++w) tot += ss_sh[m][w];
            const float ms = __double2float_rn(__ddiv_rn(tot, (double)(4 * KB)));
            r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, kRmsEps)));
            amax = __fmul_rn(amax, r);
        }
        const float s = __fdiv_rn(kActRange, fmaxf(amax, kActEps));
        int sum = 0;
        if (c0 < groups) sum = quant_bf16x16<IL, XT>(v0, v1, s, group_codes<IL>(codes, m, c0, KB), KB, norm, r);
#pragma unroll 1
        for (int c = c0 + kThreads; c < groups; c += kThreads)
            sum += quant_bf16x16<IL, XT>(xr[2 * c], xr[2 * c + 1], s, group_codes<IL>(codes, m, c, KB), KB, norm,
                                         r);
        sum = __reduce_add_sync(0xffffffffu, sum);
        if (lane == 0) atomicAdd(&xs_sh[m], sum);
        if (threadIdx.x == 0) {
            s_sh[m] = s;
            deq_sh[m] = __fdiv_rn(gamma, s);
            if (DUAL) deq2_sh[m] = __fdiv_rn(gamma2, s);
        }
    }
}

// Up to MT tokens with G 16-element groups per thread and token (instantiations
// BIG = -1: four tokens, K <= 4096; BIG = -2: two tokens, K <= 8192): every
// token's groups are loaded at once, one named barrier serves the absmax (and
// RMSNorm sum) of all tokens, then each token is quantised from registers. Per
// token the reductions are those of fused_quantise (a thread's groups in order,
// then the warp, then the warps in order), so the codes and scales are the same
// bits.
template <bool DUAL, bool IL, bool XT, int MT, int G>
__device__ void fused_quantise_few(const GemvArgs& a, int KB, uint8_t* codes, uint32_t (*am_sh)[kWarps],
                                   double (*ss_sh)[kWarps], float* s_sh, int* xs_sh, float* deq_sh,
                                   float* deq2_sh) {
    const int M = a.M, groups = KB / 4;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c0 = threadIdx.x;
    const uint4* xv = reinterpret_cast<const uint4*>(a.x);
    float gamma = 0.0f, gamma2 = 0.0f;
    if (threadIdx.x == 0) {
        gamma = *a.gamma;
        if (DUAL) gamma2 = *a.gamma2;
    }
    const bool norm = XT && a.norm;
    uint4 v[MT][G][2];
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int i = 0; i < G; ++i) {
            const int c = c0 + i * kThreads;
            v[m][i][0] = v[m][i][1] = make_uint4(0u, 0u, 0u, 0u);
            if (m < M && c < groups) {
                v[m][i][0] = xv[(size_t)m * 2 * groups + 2 * c];
                v[m][i][1] = xv[(size_t)m * 2 * groups + 2 * c + 1];
            }
        }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        if (m >= M) break;
        uint32_t mx = 0;  // 0 when this thread has no group
        double ss = 0.0;
#pragma unroll
        for (int i = 0; i < G; ++i) {
            mx = max(mx, absmax16(v[m][i][0], v[m][i][1]));
            if (norm) ss += sumsq16(v[m][i][0], v[m][i][1]);
        }
        mx = __reduce_max_sync(0xffffffffu, mx);
        if (norm) ss = warp_sum(ss);
        if (lane == 0) {
            am_sh[m][warp] = mx;
            if (XT) ss_sh[m][warp] = ss;
        }
    }
    consumer_sync();
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        if (m >= M) break;
        uint32_t amb = am_sh[m][0];
#pragma unroll
        for (int w = 1; w < kWarps; ++w) amb = max(amb, am_sh[m][w]);
        float amax = __uint_as_float(amb << 16), r = 1.0f;
        if (norm) {  // unit-weight RMSNorm: max |fl(x r)| = fl(max |x| r)
            double tot = ss_sh[m][0];
#pragma unroll
            for (int w = 1; w < kWarps; ++w) tot += ss_sh[m][w];
            const float ms = __double2float_rn(__ddiv_rn(tot, (double)(4 * KB)));
            r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, kRmsEps)));
            amax = __fmul_rn(amax, r);
        }
        const float s = __fdiv_rn(kActRange, fmaxf(amax, kActEps));
        int sum = 0;
#pragma unroll
        for (int i = 0; i < G; ++i) {
            const int c = c0 + i * kThreads;
            if (c < groups)
                sum += quant_bf16x16<IL, XT>(v[m][i][0], v[m][i][1], s, group_codes<IL>(codes, m, c, KB), KB, norm, r);
        }
        sum = __reduce_add_sync(0xffffffffu, sum);
        if (lane == 0) atomicAdd(&xs_sh[m], sum);
        if (threadIdx.x == 0) {
            s_sh[m] = s;
            deq_sh[m] = __fdiv_rn(gamma, s);
            if (DUAL) deq2_sh[m] = __fdiv_rn(gamma2, s);
        }
    }
}

// One token (BIG = G instantiation): each thread loads all of its G 16-element
// groups at once (at most kBigGroups), keeps them in registers for the absmax and
// for the codes, so the token costs one round trip to L2 instead of one per group
// and pass. Codes in the interleaved single-token layout. DUAL: the FFN's gate
// and up projections share the codes; each gets its own gamma / s.
constexpr int kBigGroups = 8;

template <int G, bool DUAL>
__device__ void fused_quantise_big(const GemvArgs& a, int KB, uint8_t* codes, uint32_t* am_w, float* s_sh,
                                   int* xs_sh, float* deq_sh, float* deq2_sh) {
    const int groups = KB / 4;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint4* xv = reinterpret_cast<const uint4*>(a.x);
    const float gamma = threadIdx.x == 0 ? *a.gamma : 0.0f;
    const float gamma2 = DUAL && threadIdx.x == 0 ? *a.gamma2 : 0.0f;
    uint4 v[G][2];
#pragma unroll
    for (int i = 0; i < G; ++i) {
        const int c = threadIdx.x + i * kThreads;
        v[i][0] = v[i][1] = make_uint4(0u, 0u, 0u, 0u);
        if (c < groups) {
            v[i][0] = xv[2 * c];
            v[i][1] = xv[2 * c + 1];
        }
    }
    uint32_t mx = 0;  // zero groups (past the row) leave the maximum unchanged
#pragma unroll
    for (int i = 0; i < G; ++i) mx = max(mx, absmax16(v[i][0], v[i][1]));
    mx = __reduce_max_sync(0xffffffffu, mx);
    if (lane == 0) am_w[warp] = mx;
    consumer_sync();
    uint32_t amb = am_w[0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) amb = max(amb, am_w[w]);
    const float s = __fdiv_rn(kActRange, fmaxf(__uint_as_float(amb << 16), kActEps));
    int sum = 0;
#pragma unroll
    for (int i = 0; i < G; ++i) {
        const int c = threadIdx.x + i * kThreads;
        if (c < groups) sum += quant_bf16x16<true, false>(v[i][0], v[i][1], s, codes + 16 * c, KB, false, 1.0f);
    }
    sum = __reduce_add_sync(0xffffffffu, sum);
    if (lane == 0) atomicAdd(&xs_sh[0], sum);
    if (threadIdx.x == 0) {
        s_sh[0] = s;
        deq_sh[0] = __fdiv_rn(gamma, s);
        if (DUAL) deq2_sh[0] = __fdiv_rn(gamma2, s);
    }
}

// One token with f <= 8192 (the BIG = 2 instantiation of the down projection):
// the partials and this thread's two groups of h are requested together, so the
// token costs one round trip to L2 instead of one for the partials and one for
// h; the reductions are those of finalise_quantise, in the same order.
template <bool IL>
__device__ void finalise_quantise_one(const GemvArgs& a, int KB, uint8_t* codes, float* s_sh, int* xs_sh,
                                      float* r_sh, float* deq_sh) {
    const int f = 4 * KB, groups = KB / 4;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __shared__ double dred[kWarps];
    __shared__ float fred[kWarps];
    float gamma = 0.0f;
    if (threadIdx.x == 0) gamma = *a.gamma;
    const float4* hr = reinterpret_cast<const float4*>(a.hin);
    float4 h[2][4];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int c = threadIdx.x + i * kThreads;
#pragma unroll
        for (int q = 0; q < 4; ++q) h[i][q] = c < groups ? hr[4 * c + q] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    double ss = 0.0;
    float hmax = 0.0f;
#pragma unroll 1
    for (int p = threadIdx.x; p < a.hin_parts; p += kThreads) {
        ss = __dadd_rn(ss, a.hin_ss[p]);
        hmax = fmaxf(hmax, a.hin_max[p]);
    }
    ss = warp_sum(ss);
    hmax = warp_max(hmax);
    if (lane == 0) {
        dred[warp] = ss;
        fred[warp] = hmax;
    }
    consumer_sync();
    if (threadIdx.x == 0) {
        double tot = dred[0];
        float mx = fred[0];
#pragma unroll 1
        for (int w = 1; w < kWarps; ++w) {
            tot = __dadd_rn(tot, dred[w]);
            mx = fmaxf(mx, fred[w]);
        }
        const float ms = __double2float_rn(__ddiv_rn(tot, (double)f));
        const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, kRmsEps)));
        const float s = __fdiv_rn(kActRange, fmaxf(__fmul_rn(mx, r), kActEps));
        r_sh[0] = r;
        s_sh[0] = s;
        deq_sh[0] = __fdiv_rn(gamma, s);
    }
    consumer_sync();
    const float r = r_sh[0], s = s_sh[0];
    int sum = 0;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int c = threadIdx.x + i * kThreads;
        if (c < groups) {
            float v[16];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                v[4 * q] = __fmul_rn(h[i][q].x, r);
                v[4 * q + 1] = __fmul_rn(h[i][q].y, r);
                v[4 * q + 2] = __fmul_rn(h[i][q].z, r);
                v[4 * q + 3] = __fmul_rn(h[i][q].w, r);
            }
            sum += quant_pack16<IL>(v, s, group_codes<IL>(codes, 0, c, KB), KB);
        }
    }
    sum = __reduce_add_sync(0xffffffffu, sum);
    if (lane == 0) atomicAdd(&xs_sh[0], sum);
}

// FFN glue inside the down projection (consumer threads): per token,
// r = 1 / sqrtf(float(sum_j h_j^2 / f) + eps) from the up kernel's per-tile fp64
// partials (fixed order: thread strides, warp butterfly, warps in index order),
// s2 = 127 / max(max_j |h_j r|, eps) with max_j |fl(h_j r)| = fl(max_j |h_j| r)
// (rounding is monotonic, r > 0), then PLANES codes of fl(h_j r) into shared
// memory. Thread 0 records s2 and gamma / s2.
template <bool IL>
__device__ void finalise_quantise(const GemvArgs& a, int KB, uint8_t* codes, float* s_sh, int* xs_sh,
                                  float* r_sh, float* deq_sh) {
    const int f = 4 * KB;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __shared__ double dred[kFusedMaxTokens][kWarps];
    __shared__ float fred[kFusedMaxTokens][kWarps];
    float gamma = 0.0f;
    if (threadIdx.x < kFusedMaxTokens) gamma = *a.gamma;
    // every token's partials in one pass (their loads overlap), one barrier for all
#pragma unroll
    for (int m = 0; m < kFusedMaxTokens; ++m) {
        if (m >= a.M) break;
        double ss = 0.0;
        float hmax = 0.0f;
#pragma unroll 1
        for (int p = threadIdx.x; p < a.hin_parts; p += kThreads) {
            ss = __dadd_rn(ss, a.hin_ss[(size_t)m * a.hin_parts + p]);
            hmax = fmaxf(hmax, a.hin_max[(size_t)m * a.hin_parts + p]);
        }
        ss = warp_sum(ss);
        hmax = warp_max(hmax);
        if (lane == 0) {
            dred[m][warp] = ss;
            fred[m][warp] = hmax;
        }
    }
    consumer_sync();
    if (threadIdx.x < a.M && threadIdx.x < kFusedMaxTokens) {  // thread m: token m's r, s2 (warps in order)
        const int m = threadIdx.x;
        double tot = dred[m][0];
        float mx = fred[m][0];
#pragma unroll 1
        for (int w = 1; w < kWarps; ++w) {
            tot = __dadd_rn(tot, dred[m][w]);
            mx = fmaxf(mx, fred[m][w]);
        }
        const float ms = __double2float_rn(__ddiv_rn(tot, (double)f));
        const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, kRmsEps)));
        const float s = __fdiv_rn(kActRange, fmaxf(__fmul_rn(mx, r), kActEps));
        r_sh[m] = r;
        s_sh[m] = s;
        deq_sh[m] = __fdiv_rn(gamma, s);
    }
    consumer_sync();
    const int groups = KB / 4;
#pragma unroll 1
    for (int m = 0; m < a.M; ++m) {
        const float r = r_sh[m], s = s_sh[m];
        const float4* hr = reinterpret_cast<const float4*>(a.hin + (size_t)m * f);
        int sum = 0;
#pragma unroll 1
        for (int c = threadIdx.x; c < groups; c += kThreads) {
            float v[16];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 h4 = hr[4 * c + q];
                v[4 * q] = __fmul_rn(h4.x, r);
                v[4 * q + 1] = __fmul_rn(h4.y, r);
                v[4 * q + 2] = __fmul_rn(h4.z, r);
                v[4 * q + 3] = __fmul_rn(h4.w, r);
            }
            sum += quant_pack16<IL>(v, s, group_codes<IL>(codes, m, c, KB), KB);
        }
        sum = __reduce_add_sync(0xffffffffu, sum);
        if (lane == 0) atomicAdd(&xs_sh[m], sum);
    }
}

// 1-D bulk copy global -> this CTA's shared memory, completion counted on `bar`.
__device__ __forceinline__ void bulk_copy(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// The weight stream: a unit is one tile of unit_rows rows restricted to one K
// segment of at most 32 KiB (32 chunks of 64 bytes per row at 16 rows). The producer warp copies the unit's row
// segments into a ring of kStages shared-memory stages; the row pitch is
// congruent to 64 mod 128 bytes so rows g and g + 1 of a quarter-warp fall on
// different banks.
// XT: extended calls (row segments with their own gamma, RMSNorm of x); the
// plain forward runs the instantiation without that code.
// BIG: how x is quantised when the kernel does it (SRC_X). G > 0: one token from
// registers, G 16-element groups per thread (fused_quantise_big; with G = 8 the
// registers allow two CTAs per SM, otherwise three); -1: up to four tokens with
// K <= 4096, one group per thread and token, -2: two tokens with K <= 8192, two
// groups (fused_quantise_few); 0: the two-pass loop (fused_quantise).
// Units of the single-token path hold a.unit_rows rows (16, or 8 / 4 for rows
// longer than 2 KiB, so a unit stays a contiguous ~32 KiB and the tiles are fine
// enough to balance the CTAs; 8 also when 16-row tiles would leave SMs without
// one); every other path streams 16-row units.
template <int NT, int SRC, bool DUAL, bool DP, bool XT, int BIG = 0>
__global__ void __launch_bounds__(kThreads + 32, (NT == 1 && BIG <= 2) ? 3 : 2) gemv_mma_kernel(const GemvArgs a) {
    constexpr int TOK = 8 * NT;
    constexpr bool FUSED = SRC != SRC_CODES;
    static_assert(!DP || (FUSED && NT == 1), "the dp4a path reads one token's codes from shared memory");
    constexpr int NW = DUAL ? 2 : 1;  // weight streams
    extern __shared__ __align__(128) uint8_t dyn[];
    // per-tile partial sums of the warps; double-buffered for one token group
    // (tile t + 1 fills the other buffer while tile t's epilogue may still read
    // its own, so one named barrier per tile suffices)
    constexpr int RB = (NT == 1 && !DUAL) ? 2 : 1;
    __shared__ int red_buf[RB][kWarps][16][TOK];
    __shared__ int red2[DUAL ? kWarps : 1][16][TOK];
    __shared__ float s_sh[TOK];
    __shared__ int xs_sh[TOK];
    __shared__ uint32_t am_sh[TOK][kWarps];
    __shared__ double ss_sh[SRC == SRC_X && XT ? TOK : 1][kWarps];
    __shared__ float r_sh[TOK];
    __shared__ float deq_sh[TOK], deq2_sh[TOK];
    __shared__ int abort_sh;

    const int N = a.N, KB = a.KB;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int R = a.unit_rows;                         // rows per tile (16 except on the single-token path)
    const int ntiles = (N + R - 1) / R;
    const int nchunks = KB >> 6;
    const int cps = a.seg_chunks;                     // chunks per K segment
    const int nseg = (nchunks + cps - 1) / cps;
    const int pitch = a.pitch;
    const int tok0 = blockIdx.y * TOK;

    uint8_t* codes = dyn;                              // fused: PLANES codes of the M tokens
    uint8_t* stages = dyn + a.codes_bytes;             // kStages x NW x R rows x pitch
    const int stage_bytes = NW * R * pitch;
    uint64_t* bars = reinterpret_cast<uint64_t*>(stages + kStages * stage_bytes);
    auto full = [&](int st) { return tc::smem_u32(bars + st); };
    auto empty = [&](int st) { return tc::smem_u32(bars + kStages + st); };

    if (threadIdx.x == kThreads) {
        for (int st = 0; st < kStages; ++st) {
            tc::mbar_init(full(st), 1);
            tc::mbar_init(empty(st), kWarps);
        }
        abort_sh = 0;
        for (int m = 0; m < TOK; ++m) xs_sh[m] = 0;
        tc::fence_mbar_init();
        // L2 prefetch of the first tiles may run before the previous kernel ends
        for (int p = 0; p < kPrefetchAhead; ++p) {
            const int tile = blockIdx.x + p * gridDim.x;
            if (tile < ntiles) {
                const int n0 = tile * R;
                prefetch_l2(a.Wp + (size_t)n0 * KB, (uint32_t)(min(R, N - n0) * KB));
                if (DUAL) prefetch_l2(a.Wp2 + (size_t)n0 * KB, (uint32_t)(min(R, N - n0) * KB));
            }
        }
    }
    __syncthreads();
    grid_dependents_launch();

    if (warp == kWarps) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            uint32_t g = 0;
            bool stop = false;
            bool waited = false;
            for (int tile = blockIdx.x; tile < ntiles && !stop; tile += gridDim.x) {
                const int n0 = tile * R;
                const int rows = min(R, N - n0);
                for (int sg = 0; sg < nseg; ++sg, ++g) {
                    const int st = g % kStages;
                    if (g >= kStages &&
                        !tc::mbar_wait(empty(st), ((g / kStages) - 1) & 1, kWaitLimitNs)) {
                        atomicOr(a.err, 1u);
                        atomicExch(&abort_sh, 1);
                    }
                    if (*reinterpret_cast<volatile int*>(&abort_sh)) {
                        stop = true;
                        break;
                    }
                    const int c0 = sg * cps;
                    const uint32_t segb = (uint32_t)(min(cps, nchunks - c0) * 64);
                    tc::mbar_arrive_expect_tx(full(st), segb * rows * NW);
                    // The first kStages units are copied before the dependency wait: the
                    // packed weights are not written by a kernel that lets this one start
                    // early (the library's early-triggering kernels never write them),
                    // so the ring fills while the previous kernel finishes.
                    if (!waited && g >= (uint32_t)kStages) {
                        grid_dependency_wait();
                        waited = true;
                    }
                    const uint32_t dst = tc::smem_u32(stages + st * stage_bytes);
                    for (int r = 0; r < rows; ++r)
                        bulk_copy(dst + r * pitch, a.Wp + (size_t)(n0 + r) * KB + c0 * 64, segb, full(st));
                    if (DUAL)
                        for (int r = 0; r < rows; ++r)
                            bulk_copy(dst + (R + r) * pitch, a.Wp2 + (size_t)(n0 + r) * KB + c0 * 64, segb,
                                      full(st));
                }
            }
            if (stop) {
                // let the copies still in flight land before this warp exits
                const uint32_t first = g > (uint32_t)kStages ? g - kStages : 0;
                for (uint32_t h = first; h < g; ++h)
                    tc::mbar_wait(full(h % kStages), (h / kStages) & 1, kWaitLimitNs);
            }
            // otherwise every unit handed out was consumed: the consumers waited on
            // each full barrier, so no copy is in flight when this warp exits
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int g8 = lane >> 2, t = lane & 3;

    // this lane's activation operand: token 8*nt + g8 of the group. Lanes past the
    // last token read token 0's codes instead: they only feed output columns that
    // are never stored, and loading them costs less than zeroing registers.
    const uint8_t* xbase[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        int tok = tok0 + 8 * nt + g8;
        if (tok >= a.M) tok = 0;
        if (FUSED)
            xbase[nt] = codes + smem_plane_off(tok, 0, KB) + 16 * t;
        else
            xbase[nt] = reinterpret_cast<const uint8_t*>(a.Xp) + (size_t)tok * 4 * KB + 16 * t;
    }
    auto load_x = [&](uint4 (&xv)[NT][4], int off) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if (FUSED) {
                    xv[nt][i] = *reinterpret_cast<const uint4*>(xbase[nt] + i * KB + off);
                } else {
                    xv[nt][i] = ld_nc16(xbase[nt] + i * KB + off);
                }
            }
    };

    // An abort (a bounded wait that gave up) keeps every consumer warp on the same
    // sequence of named barriers: later waits are skipped and nothing is stored.
    auto aborted = [&]() { return *reinterpret_cast<volatile int*>(&abort_sh) != 0; };

    grid_dependency_wait();
    if (SRC == SRC_X) {
        if constexpr (BIG > 0)
            fused_quantise_big<BIG, DUAL>(a, KB, codes, am_sh[0], s_sh, xs_sh, deq_sh, deq2_sh);
        else if constexpr (BIG == -1)
            fused_quantise_few<DUAL, DP, XT, kFusedMaxTokens, 1>(a, KB, codes, am_sh, ss_sh, s_sh, xs_sh, deq_sh,
                                                                 deq2_sh);
        else if constexpr (BIG == -2)
            fused_quantise_few<DUAL, DP, XT, 2, 2>(a, KB, codes, am_sh, ss_sh, s_sh, xs_sh, deq_sh, deq2_sh);
        else
            fused_quantise<DUAL, DP, XT>(a, KB, codes, am_sh, ss_sh, s_sh, xs_sh, deq_sh, deq2_sh);
    } else if (SRC == SRC_H) {
        if constexpr (BIG > 0)
            finalise_quantise_one<DP>(a, KB, codes, s_sh, xs_sh, r_sh, deq_sh);
        else
            finalise_quantise<DP>(a, KB, codes, s_sh, xs_sh, r_sh, deq_sh);
    } else if (threadIdx.x < TOK && tok0 + (int)threadIdx.x < a.M) {
        const float s = a.scale[tok0 + threadIdx.x];
        s_sh[threadIdx.x] = s;
        xs_sh[threadIdx.x] = a.xsum[tok0 + threadIdx.x];
        deq_sh[threadIdx.x] = __fdiv_rn(*a.gamma, s);
    }
    consumer_sync();  // codes, code sums and dequantisation factors are ready

    uint32_t g = 0;
    int it = 0;  // tiles done by this CTA
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
        auto& red = red_buf[RB == 2 ? (it & 1) : 0];
        const int n0 = tile * R;
        if constexpr (DP) {
            // One token: thread (row group rg, lane tl of T = 1024 / R) owns rows
            // 4 rg .. 4 rg + 3 of the unit and its words j = tl, tl + T, ...; per word
            // one dp4a per field against the interleaved plane words of the token.
            const int rg = threadIdx.x >> a.rg_shift, tl = threadIdx.x & ((1 << a.rg_shift) - 1);
            const int tstride = 1 << a.rg_shift;
            int acc[4][4] = {}, acc2[DUAL ? 4 : 1][4] = {};
            for (int sg = 0; sg < nseg; ++sg, ++g) {
                const int st = g % kStages;
                if (aborted()) continue;
                if (!tc::mbar_wait(full(st), (g / kStages) & 1, kWaitLimitNs)) {
                    atomicOr(a.err, 1u);
                    atomicExch(&abort_sh, 1);
                    continue;
                }
                const int words = min(cps, nchunks - sg * cps) * 16;
                const uint8_t* wr = stages + st * stage_bytes + 4 * rg * pitch;
                const uint4* xw = reinterpret_cast<const uint4*>(codes) + sg * cps * 16;
#pragma unroll 2
                for (int j = tl; j < words; j += tstride) {
                    const uint4 xv = xw[j];
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const uint32_t w = *reinterpret_cast<const uint32_t*>(wr + r * pitch + 4 * j);
                        dp4a_fields(acc[r], w, xv);
                        if constexpr (DUAL) {
                            const uint32_t w2 = *reinterpret_cast<const uint32_t*>(wr + (R + r) * pitch + 4 * j);
                            dp4a_fields(acc2[r], w2, xv);
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(empty(st));
            }
            // fold the fields, sum the warp, and leave this warp's share of each of
            // the 16 rows (zero for rows of the other groups) as token 0's column
            int v[4], v2[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                v[r] = __reduce_add_sync(0xffffffffu, fold_fields(acc[r]));
                if constexpr (DUAL) v2[r] = __reduce_add_sync(0xffffffffu, fold_fields(acc2[r]));
            }
            if (lane < 16) {
                const bool mine = (lane >> 2) == rg;
                const int q = lane & 3;
                const int pick = q == 0 ? v[0] : q == 1 ? v[1] : q == 2 ? v[2] : v[3];
                red[warp][lane][0] = mine ? pick : 0;
                if constexpr (DUAL) {
                    const int pick2 = q == 0 ? v2[0] : q == 1 ? v2[1] : q == 2 ? v2[2] : v2[3];
                    red2[warp][lane][0] = mine ? pick2 : 0;
                }
            }
        } else {
            int acc[NT][4][4], acc2[NT][4][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[nt][i][e] = 0;
            if constexpr (DUAL) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int i = 0; i < 4; ++i)
#pragma unroll
                        for (int e = 0; e < 4; ++e) acc2[nt][i][e] = 0;
            }

            for (int sg = 0; sg < nseg; ++sg, ++g) {
                const int st = g % kStages;
                if (aborted()) continue;
                if (!tc::mbar_wait(full(st), (g / kStages) & 1, kWaitLimitNs)) {
                    atomicOr(a.err, 1u);
                    atomicExch(&abort_sh, 1);
                    continue;
                }
                const int c0 = sg * cps;
                const int segc = min(cps, nchunks - c0);
                const uint8_t* sa = stages + st * stage_bytes + g8 * pitch + 16 * t;
                const uint8_t* sb = sa + 8 * pitch;
#pragma unroll 2
                for (int u = 0; u < kUnroll; ++u) {
                    const int cl = warp + kWarps * u;
                    if (cl < segc) {
                        const uint4 wa = *reinterpret_cast<const uint4*>(sa + 64 * cl);
                        const uint4 wb = *reinterpret_cast<const uint4*>(sb + 64 * cl);
                        uint4 xv[NT][4];
                        load_x(xv, 64 * (c0 + cl));
                        chunk_mma<NT>(acc, wa, wb, xv);
                        if constexpr (DUAL) {
                            const uint4 wc = *reinterpret_cast<const uint4*>(sa + 16 * pitch + 64 * cl);
                            const uint4 wd = *reinterpret_cast<const uint4*>(sb + 16 * pitch + 64 * cl);
                            chunk_mma<NT>(acc2, wc, wd, xv);
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(empty(st));
            }

            // Fold the four field accumulators; D element e sits at row g8 + 8*(e >> 1),
            // token 8*nt + 2t + (e & 1).
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int v = acc[nt][0][e] + (acc[nt][1][e] >> 2) + (acc[nt][2][e] >> 4) +
                                  (acc[nt][3][e] >> 6);
                    red[warp][g8 + 8 * (e >> 1)][8 * nt + 2 * t + (e & 1)] = v;
                    if constexpr (DUAL) {
                        red2[warp][g8 + 8 * (e >> 1)][8 * nt + 2 * t + (e & 1)] =
                            acc2[nt][0][e] + (acc2[nt][1][e] >> 2) + (acc2[nt][2][e] >> 4) +
                            (acc2[nt][3][e] >> 6);
                    }
                }
        }
        consumer_sync();

        const bool store = !aborted();
        if constexpr (DUAL) {
            // FFN up epilogue: h = relu(g)^2 * u, plus the tile's per-token sum of
            // h^2 (fp64, fixed butterfly order over the 16 rows) and max |h|.
            for (int idx = threadIdx.x; idx < 16 * TOK; idx += kThreads) {
                const int r = idx & 15, cl = idx >> 4;
                const int n = n0 + r, m = tok0 + cl;
                const bool valid = n < N && m < a.M;
                float hv = 0.0f;
                if (valid) {
                    int sg = 0, su = 0;
#pragma unroll
                    for (int w = 0; w < kWarps; ++w) {
                        sg += red[w][r][cl];
                        su += red2[w][r][cl];
                    }
                    const float gv = dequant(sg - xs_sh[cl], deq_sh[cl]);
                    const float uv = dequant(su - xs_sh[cl], deq2_sh[cl]);
                    const float tv0 = gv > 0.0f ? gv : 0.0f;
                    hv = __fmul_rn(__fmul_rn(tv0, tv0), uv);
                    if (store) a.h[(size_t)m * N + n] = hv;
                }
                double ss = __dmul_rn((double)hv, (double)hv);
                float mx = fabsf(hv);
#pragma unroll
                for (int o = 8; o > 0; o >>= 1) {  // the 16 rows of a token are 16 adjacent lanes
                    ss = __dadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, o));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                }
                if (r == 0 && m < a.M && store) {
                    a.part_ss[(size_t)m * ntiles + tile] = ss;
                    a.part_max[(size_t)m * ntiles + tile] = mx;
                }
            }
        } else {
            for (int idx = threadIdx.x; idx < 16 * TOK; idx += kThreads) {
                const int r = idx & 15, cl = idx >> 4;
                const int n = n0 + r, m = tok0 + cl;
                if (r >= R || n >= N || m >= a.M) continue;
                int sum = 0;
#pragma unroll
                for (int w = 0; w < kWarps; ++w) sum += red[w][r][cl];
                const int accv = sum - xs_sh[cl];
                const int sgi = XT ? gamma_index(a.out, n) : 0;  // segments / rows with their own gamma
                float v = dequant(accv, sgi == 0 ? deq_sh[cl] : __fdiv_rn(a.gamma[sgi], s_sh[cl]));
                if (!store) continue;
                const size_t o = (size_t)m * N + n;
                if (a.out.y32) {
                    a.out.y32[o] = v;
                } else {
                    if (a.out.residual) v = __fadd_rn(bf16_bits_to_f32(a.out.residual[o]), v);
                    a.out.y[o] = f32_to_bf16_bits(v);
                }
                if (a.out.acc) a.out.acc[o] = accv;
            }
        }
        if (RB == 1) consumer_sync();  // the single buffer is reused by the next tile
    }
}

// Generic path: any K % 4 == 0, NATURAL codes. One warp per (row, token).
__global__ void __launch_bounds__(kThreads) gemv_generic_kernel(
    const uint8_t* __restrict__ Wp, const float* __restrict__ gamma_p, int N, int K,
    const int8_t* __restrict__ Xn, const float* __restrict__ scale, int M, GemvOut out) {
    grid_dependency_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = blockIdx.x * kWarps + warp;
    const int m = blockIdx.y;
    if (n >= N) return;
    const int KB = K / 4;
    const uint8_t* wr = Wp + (size_t)n * KB;
    const int8_t* xr = Xn + (size_t)m * K;
    int acc = 0;
    for (int j = lane; j < KB; j += 32) {
        const unsigned b = wr[j];
#pragma unroll
        for (int i = 0; i < 4; ++i) acc += ((int)((b >> (2 * i)) & 3u) - 1) * (int)xr[4 * j + i];
    }
    acc = warp_sum(acc);
    if (lane == 0) {
        const float deq = __fdiv_rn(gamma_p[gamma_index(out, n)], scale[m]);
        float v = dequant(acc, deq);
        const size_t o = (size_t)m * N + n;
        if (out.y32) {
            out.y32[o] = v;
        } else {
            if (out.residual) v = __fadd_rn(bf16_bits_to_f32(out.residual[o]), v);
            out.y[o] = f32_to_bf16_bits(v);
        }
        if (out.acc) out.acc[o] = acc;
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

template <int NT, int SRC, bool DUAL, bool DP = false, bool XT = false, int BIG = 0>
cudaError_t launch_variant(const GemvArgs& a, dim3 grid, size_t smem, cudaStream_t s) {
    auto kern = gemv_mma_kernel<NT, SRC, DUAL, DP, XT, BIG>;
    static bool done[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64 || !done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMaxDynSmem);
        if (e != cudaSuccess) return e;
        if (dev < 64) done[dev] = true;
    }
    return launch_pdl(kern, grid, dim3(kThreads + 32), smem, s, a);
}

// Codes in shared memory: a single token takes the dp4a path (the MMA path would
// spend 7 of its 8 token columns on padding).
template <int SRC, bool DUAL, bool XT = false>
cudaError_t launch_fused(const GemvArgs& a, dim3 grid, size_t smem, cudaStream_t s) {
    // K <= 4096 from x: the quantiser that loads every token's group at once
    if constexpr (SRC == SRC_X) {
        if (a.KB / 4 <= kThreads) {
            if (a.M == 1) return launch_variant<1, SRC, DUAL, true, XT, -1>(a, grid, smem, s);
            return launch_variant<1, SRC, DUAL, false, XT, -1>(a, grid, smem, s);
        }
        if (a.M <= 2 && a.KB / 4 <= 2 * kThreads) {  // two tokens, K <= 8192
            if (a.M == 1) return launch_variant<1, SRC, DUAL, true, XT, -2>(a, grid, smem, s);
            return launch_variant<1, SRC, DUAL, false, XT, -2>(a, grid, smem, s);
        }
    }
    if (a.M == 1) return launch_variant<1, SRC, DUAL, true, XT>(a, grid, smem, s);
    return launch_variant<1, SRC, DUAL, false, XT>(a, grid, smem, s);
}

// Segment plan, shared-memory size and grid of one streamed GEMV launch.
struct StreamPlan {
    size_t smem;
    unsigned grid_x;
};

// unit_rows: 16, or 8 / 4 for the single-token path (whose threads then cover
// one or two groups of four rows); a unit keeps at most 32 KiB of weights.
cudaError_t plan_stream(GemvArgs& a, int64_t N, int64_t K, int64_t M, int nw, bool codes_in_smem,
                        StreamPlan& p, int unit_rows = 16, int max_per_sm = 4) {
    cudaError_t e = device_error_word(&a.err);
    if (e != cudaSuccess) return e;
    a.unit_rows = unit_rows;
    a.rg_shift = unit_rows == 16 ? 6 : unit_rows == 8 ? 7 : 8;
    // K segments of at most kMaxSegChunks * 16 / unit_rows chunks, as even as possible
    const int max_seg = kMaxSegChunks * 16 / unit_rows;
    const int nchunks = (int)(K / 256);
    const int nseg = (nchunks + max_seg - 1) / max_seg;
    a.seg_chunks = (nchunks + nseg - 1) / nseg;
    const int segb = a.seg_chunks * 64;
    a.pitch = (segb % 128 == 0) ? segb + 64 : segb;  // rows g, g+1 on different banks
    a.codes_bytes = codes_in_smem ? (int)((M * (K + 64) + 127) / 128 * 128) : 0;
    p.smem = (size_t)a.codes_bytes + (size_t)kStages * nw * unit_rows * a.pitch + 2 * kStages * 8;
    const int ntiles = (int)((N + unit_rows - 1) / unit_rows);
    // as many CTAs per SM as shared memory allows (228 KiB per SM, static + reserve per CTA)
    int per_sm = (int)((228 * 1024) / (p.smem + 10 * 1024));
    per_sm = per_sm < 1 ? 1 : per_sm > max_per_sm ? max_per_sm : per_sm;
    const int cap = per_sm * sm_count();
    p.grid_x = (unsigned)(ntiles < cap ? ntiles : cap);
    // A grid that needs fewer CTAs per SM than fit: pad the shared memory so that
    // at most ceil(grid / SMs) of them fit on an SM, and the block scheduler
    // spreads the CTAs over more SMs (more SMs streaming) instead of stacking
    // them on a few. Only when the codes sit in shared memory: the kernels that
    // read them from global memory keep L1 for them (measured: 6912 -> 2560 at
    // 16 tokens slows down with the padding, the single-token calls speed up).
    const int want = (int)((p.grid_x + sm_count() - 1) / sm_count());
    if (codes_in_smem && want < per_sm) {
        size_t padded = (size_t)(228 * 1024) / (size_t)want - 10 * 1024;
        if (padded > kMaxDynSmem) padded = kMaxDynSmem;
        if (padded > p.smem) p.smem = padded;
    }
    return cudaSuccess;
}

GemvArgs base_args(const uint8_t* Wp, const float* gamma, int64_t N, int64_t K, int64_t M,
                   const GemvOut& out) {
    GemvArgs a = {};
    a.Wp = Wp;
    a.gamma = gamma;
    a.N = (int)N;
    a.KB = (int)(K / 4);
    a.M = (int)M;
    a.out = out;
    return a;
}

}  // namespace

bool gemv_fast_ok(int64_t N, int64_t K) { return N >= 1 && K % 256 == 0; }

bool gemv_segments_ok(const GemvOut& out, int64_t N) {
    for (int i = 0; i < 3; ++i)
        if (out.seg_end[i] < N && out.seg_end[i] % 16 != 0) return false;
    return true;
}

// The single kernel (quantise + GEMV) for the forward: every CTA quantises all M
// tokens, which costs more than the separate act-quant launch only for four
// tokens with K > 4096 on a grid of at most two 16-row tiles per SM (measured:
// 6912 -> 2560 at M = 4, 160 tiles: 6.90 us fused, 6.16 us with act-quant;
// 8192 -> 28672 at M = 4, 1792 tiles: 17.1 us fused, 22.7 us with it; two and
// three tokens are faster fused at 6912 -> 2560 too).
bool gemv_fused_pays(int64_t M, int64_t N, int64_t K) {
    return M <= 3 || K <= 4096 || (N + 15) / 16 > 2 * (int64_t)sm_count();
}

bool gemv_fused_ok(int64_t M, int64_t K) {
    return M >= 1 && M <= kFusedMaxTokens && (size_t)M * (K + 64) <= (size_t)kFusedSmemLimit;
}

cudaError_t launch_gemv(const uint8_t* Wp, const float* gamma, int64_t N, int64_t K,
                        const int8_t* Xp, const float* scale, const int32_t* xsum, int64_t M,
                        const GemvOut& out, cudaStream_t s, const uint16_t* x_fused, bool rmsnorm) {
    if (M == 0 || N == 0) return cudaSuccess;
    if (x_fused && !gemv_fused_ok(M, K)) return cudaErrorInvalidValue;
    if (!gemv_segments_ok(out, N)) return cudaErrorInvalidValue;
    GemvArgs a = base_args(Wp, gamma, N, K, M, out);
    a.x = x_fused;
    a.norm = (x_fused && rmsnorm) ? 1 : 0;
    a.Xp = Xp;
    a.scale = scale;
    a.xsum = xsum;
    const bool xt = a.norm || out.seg_end[0] < N || out.per_row;
    // One token: units of whole rows of up to 32 KiB (16, 8 or 4 rows), and for a
    // long row (8192 <= K <= 32768) the quantiser that keeps x in registers (its
    // register budget allows two CTAs per SM).
    const bool one = x_fused && M == 1;
    const int64_t KB = K / 4;
    // (8-row units also when 16-row tiles would leave SMs without one: 2560 -> 640
    // runs 80 CTAs instead of 40)
    const int unit_rows = one ? (KB <= 2048 ? ((N + 15) / 16 < sm_count() ? 8 : 16) : KB <= 4096 ? 8 : 4) : 16;
    const bool big = one && !xt && K / 16 <= (int64_t)kBigGroups * kThreads;
    StreamPlan p;
    // a token of at most 8192 codes needs two register groups per thread, which
    // leaves room for three CTAs per SM; longer tokens need eight (two CTAs)
    const bool big1 = big && K / 16 <= kThreads;
    const bool big2 = big && K / 16 <= 2 * kThreads;
    cudaError_t e = plan_stream(a, N, K, M, 1, x_fused != nullptr, p, unit_rows, big && !big2 ? 2 : 4);
    if (e != cudaSuccess) return e;
    const dim3 g1(p.grid_x, 1), g2(p.grid_x, (unsigned)((M + 15) / 16));
    if (xt) {
        if (x_fused) return launch_fused<SRC_X, false, true>(a, g1, p.smem, s);
        if (M <= 8) return launch_variant<1, SRC_CODES, false, false, true>(a, g1, p.smem, s);
        return launch_variant<2, SRC_CODES, false, false, true>(a, g2, p.smem, s);
    }
    if (big1) return launch_variant<1, SRC_X, false, true, false, 1>(a, g1, p.smem, s);
    if (big2) return launch_variant<1, SRC_X, false, true, false, 2>(a, g1, p.smem, s);
    if (big) return launch_variant<1, SRC_X, false, true, false, kBigGroups>(a, g1, p.smem, s);
    if (x_fused) return launch_fused<SRC_X, false>(a, g1, p.smem, s);
    if (M <= 8) return launch_variant<1, SRC_CODES, false>(a, g1, p.smem, s);
    return launch_variant<2, SRC_CODES, false>(a, g2, p.smem, s);
}

cudaError_t launch_ffn_up_fused(const uint8_t* Wg, const float* gg, const uint8_t* Wu, const float* gu,
                                int64_t f, int64_t d, const uint16_t* x, int64_t M, float* h,
                                double* part_ss, float* part_max, cudaStream_t s) {
    if (M == 0) return cudaSuccess;
    if (!gemv_fused_ok(M, d)) return cudaErrorInvalidValue;
    GemvArgs a = base_args(Wg, gg, f, d, M, GemvOut());
    a.x = x;
    a.Wp2 = Wu;
    a.gamma2 = gu;
    a.h = h;
    a.part_ss = part_ss;
    a.part_max = part_max;
    // one token: the register quantiser (one L2 round trip for x), as in launch_gemv
    const int groups = M == 1 && d / 16 <= (int64_t)kBigGroups * kThreads
                           ? (d / 16 <= kThreads ? 1 : d / 16 <= 2 * kThreads ? 2 : kBigGroups)
                           : 0;
    StreamPlan p;
    cudaError_t e = plan_stream(a, f, d, M, 2, true, p, 16, groups == kBigGroups ? 2 : 4);
    if (e != cudaSuccess) return e;
    const dim3 g1(p.grid_x, 1);
    if (groups == 1) return launch_variant<1, SRC_X, true, true, false, 1>(a, g1, p.smem, s);
    if (groups == 2) return launch_variant<1, SRC_X, true, true, false, 2>(a, g1, p.smem, s);
    if (groups == kBigGroups) return launch_variant<1, SRC_X, true, true, false, kBigGroups>(a, g1, p.smem, s);
    return launch_fused<SRC_X, true>(a, g1, p.smem, s);
}

cudaError_t launch_ffn_down_fused(const uint8_t* Wd, const float* gd, int64_t d, int64_t f,
                                  const float* h, const double* part_ss, const float* part_max,
                                  int64_t M, const GemvOut& out, cudaStream_t s) {
    if (M == 0) return cudaSuccess;
    if (!gemv_fused_ok(M, f)) return cudaErrorInvalidValue;
    GemvArgs a = base_args(Wd, gd, d, f, M, out);
    a.hin = h;
    a.hin_ss = part_ss;
    a.hin_max = part_max;
    a.hin_parts = (int)((f + 15) / 16);
    StreamPlan p;
    cudaError_t e = plan_stream(a, d, f, M, 1, true, p);
    if (e != cudaSuccess) return e;
    if (M == 1 && f / 16 <= 2 * kThreads)  // one token: partials and h in one round trip
        return launch_variant<1, SRC_H, false, true, false, 2>(a, dim3(p.grid_x, 1), p.smem, s);
    return launch_fused<SRC_H, false>(a, dim3(p.grid_x, 1), p.smem, s);
}

cudaError_t launch_gemv_generic(const uint8_t* Wp, const float* gamma, int64_t N, int64_t K,
                                const int8_t* Xn, const float* scale, int64_t M,
                                const GemvOut& out, cudaStream_t s) {
    if (M == 0 || N == 0) return cudaSuccess;
    const dim3 grid((unsigned)((N + kWarps - 1) / kWarps), (unsigned)M);
    return launch_pdl(gemv_generic_kernel, grid, dim3(kThreads), 0, s, Wp, gamma, (int)N, (int)K, Xn,
                      scale, (int)M, out);
}

}  // namespace bl

// Host-side launchers of the library's kernels (internal; the public
// interface is include/bitlinear.h). Each returns the cudaError_t of its launch.
#pragma once

#include <cuda.h>  // CUtensorMap (type only)
#include <cuda_runtime.h>
#include <stdint.h>

namespace bl {

// ---- weight packing (pack.cu)
// Per-block fp64 partial sums of |W| into partial[0 .. absmean_blocks(n)-1].
int absmean_blocks(int64_t n);
cudaError_t launch_absmean(const void* W, bool fp32, int64_t n, double* partial, float* gamma,
                           cudaStream_t s);
cudaError_t launch_ternary_pack(const void* W, bool fp32, int64_t N, int64_t K, const float* gamma,
                                uint8_t* Wp, cudaStream_t s, bool per_row = false);
// gammas[n] = fp32(sum_k |W[n, k]| / K) (per-row absmean variant)
cudaError_t launch_absmean_rows(const void* W, bool fp32, int64_t N, int64_t K, float* gammas, cudaStream_t s);
cudaError_t launch_count_bad_codes(const uint8_t* Wp, int64_t nbytes, unsigned long long* count,
                                   cudaStream_t s);

// fp64 sum of |W| of one shard (absmean term), and gamma = fp32(total / count)
cudaError_t launch_absmean_sum(const void* W, bool fp32, int64_t n, double* partial, double* sum, cudaStream_t s);
cudaError_t launch_gamma_from_sum(const double* total_sum, int64_t count, float* gamma, cudaStream_t s);

// ---- activation quantisation (actquant.cu); layout is an XqLayout
// rmsnorm: quantise fl(x * r), r = 1 / sqrtf(float(sum_k x^2 / K) + 1e-5) per token
// (unit-weight RMSNorm, sum in fp64), instead of x.
cudaError_t launch_act_quant(const uint16_t* x, int64_t M, int64_t K, int layout, int8_t* xq,
                             float* scale, int32_t* xsum, cudaStream_t s, bool rmsnorm = false);

// ---- decode GEMV (gemv.cu)
// Output modes: bf16 y (+ residual, + int32 acc dump) or fp32 dequantised y32.
struct GemvOut {
    uint16_t* y = nullptr;              // [M, N] bf16 bits
    const uint16_t* residual = nullptr; // [M, N] bf16 bits or null
    int32_t* acc = nullptr;             // [M, N] or null
    float* y32 = nullptr;               // [M, N] fp32 (used instead of y when set)
    // Row segments with their own gamma (weights stacked row-wise): output row n
    // uses gamma[seg_of(n)]; rows >= seg_end[i] lie past segment i. One segment by
    // default. The GEMV needs the ends on 16-row tiles, the GEMM on 32 columns.
    int seg_end[3] = {0x7fffffff, 0x7fffffff, 0x7fffffff};
    int per_row = 0;  // one gamma per output row (gamma[n]) instead of segments
};

__host__ __device__ __forceinline__ int seg_of(const GemvOut& o, int n) {
    return (n >= o.seg_end[0]) + (n >= o.seg_end[1]) + (n >= o.seg_end[2]);
}

// index into gamma of output row n
__host__ __device__ __forceinline__ int gamma_index(const GemvOut& o, int n) {
    return o.per_row ? n : seg_of(o, n);
}
// Requires K % 256 == 0 and 16-byte aligned Wp. Codes either come as PLANES
// layout Xp (+ scale, xsum) from the act-quant kernel, or, when x_fused is given
// (16-byte aligned bf16 x, gemv_fused_ok(M, K)), are computed inside the kernel.
bool gemv_fast_ok(int64_t N, int64_t K);
bool gemv_fused_ok(int64_t M, int64_t K);
// gemv_fused_ok and also faster than the separate act-quant launch for this shape
bool gemv_fused_pays(int64_t M, int64_t N, int64_t K);
bool gemv_segments_ok(const GemvOut& out, int64_t N);  // segment ends on 16-row tiles
cudaError_t launch_gemv(const uint8_t* Wp, const float* gamma, int64_t N, int64_t K,
                        const int8_t* Xp, const float* scale, const int32_t* xsum, int64_t M,
                        const GemvOut& out, cudaStream_t s, const uint16_t* x_fused = nullptr,
                        bool rmsnorm = false);  // fused quantisation of a unit-weight RMSNorm of x
// FFN sub-layer for M <= 4 tokens in two streamed kernels (K = d for the up
// projections, f for the down one; both multiples of 256, f + 64 codes per token
// in shared memory). up: h = relu(g)^2 * u [M, f] fp32 plus per (token, 16-row
// tile) partials sum h^2 (fp64) and max |h| [M, ceil(f/16)]; down: subln RMSNorm
// and requantisation of h from those partials, then the down projection.
cudaError_t launch_ffn_up_fused(const uint8_t* Wg, const float* gg, const uint8_t* Wu, const float* gu,
                                int64_t f, int64_t d, const uint16_t* x, int64_t M, float* h,
                                double* part_ss, float* part_max, cudaStream_t s);
cudaError_t launch_ffn_down_fused(const uint8_t* Wd, const float* gd, int64_t d, int64_t f,
                                  const float* h, const double* part_ss, const float* part_max,
                                  int64_t M, const GemvOut& out, cudaStream_t s);
// Any K % 4 == 0: NATURAL layout codes, one warp per output.
cudaError_t launch_gemv_generic(const uint8_t* Wp, const float* gamma, int64_t N, int64_t K,
                                const int8_t* Xn, const float* scale, int64_t M,
                                const GemvOut& out, cudaStream_t s);

// ---- prefill GEMM on tcgen05 tensor cores (gemm_tc.cu)
// xq_g16t: G16T layout codes for M tokens. Requires K % 64 == 0 and 16-byte
// aligned Wp and xq_g16t (TMA); any M, N (tails are zero-filled by the TMA).
bool gemm_tc_ok(int64_t N, int64_t K, const void* Wp, const void* xq);
bool gemm_segments_ok(const GemvOut& out, int64_t N);  // segment ends on 32-column chunks
int gemm_tc_tile_width(int64_t M, int64_t N, int sms);
// sk_ws / sk_ws_bytes: scratch for stream-K pieces (gemm_sk_workspace_bytes of the
// device's SM count); null or too small means the data-parallel split only.
cudaError_t launch_gemm_tc(const uint8_t* Wp, const float* gamma, int64_t N, int64_t K,
                           const int8_t* xq_g16t, const float* scale, const int32_t* xsum, int64_t M,
                           const GemvOut& out, cudaStream_t s, void* sk_ws = nullptr, size_t sk_ws_bytes = 0);
size_t gemm_sk_workspace_bytes(int sms);
// Whether launch_gemm_tc splits tiles across CTAs (stream-K) for this shape on
// `sms` SMs, given enough workspace.
bool gemm_use_stream_k(int64_t M, int64_t N, int64_t K, int sms);

// The FFN's gate and up projections in one tensor-core launch (M > 16): h =
// max(g, 0)^2 * u [M, f] fp32 and, per token and 128-column tile,
// part_ss = sum h^2 (fp64) and part_max = max |h| ([M, gemm_dual_parts(f)]).
struct FfnUpOut {
    float* h = nullptr;
    double* part_ss = nullptr;
    float* part_max = nullptr;
    const float* gamma_u = nullptr;  // gamma of the up weight (the gate's is the launch's gamma)
};
cudaError_t launch_gemm_tc_dual(const uint8_t* Wg, const float* gg, const uint8_t* Wu, const float* gu, int64_t f,
                                int64_t d, const int8_t* xq_g16t, const float* scale, const int32_t* xsum, int64_t M,
                                const FfnUpOut& up, cudaStream_t s);
int gemm_dual_parts(int64_t f);

// 2-D uint8 TMA tensor map over [rows, cols] (cols contiguous), box [box_rows,
// box_cols], optionally 128-byte swizzled; false when the driver refuses it.
bool make_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
              uint32_t box_cols, bool swizzle128);

// ---- tensor-core GEMV for up to 16 tokens (gemv_tc.cu)
// xq_g16t: G16T layout codes of M <= 16 tokens. Requires K % 256 == 0 and
// 16-byte aligned Wp and xq_g16t; any N.
bool gemv_tc_ok(int64_t N, int64_t K, int64_t M, const void* Wp, const void* xq);
cudaError_t launch_gemv_tc(const uint8_t* Wp, const float* gamma, int64_t N, int64_t K,
                           const int8_t* xq_g16t, const float* scale, const int32_t* xsum, int64_t M,
                           const GemvOut& out, cudaStream_t s);
// K-split of the tensor-core GEMV (CTAs per cluster) for a shape, >= 1.
int gemv_tc_split(int64_t N, int64_t K, int sms);

// ---- lookup-table GEMV for up to 16 tokens (gemv_lut.cu)
// xq: NATURAL layout codes (4-byte aligned). Requires K % 256 == 0 and a 16-byte
// aligned Wp; any N. Launches ceil(M / 4) times (four tokens per table).
bool gemv_lut_ok(int64_t N, int64_t K, int64_t M, const void* Wp, const void* xq);
cudaError_t launch_gemv_lut(const uint8_t* Wp, const float* gamma, int64_t N, int64_t K, const int8_t* xq,
                            const float* scale, int64_t M, const GemvOut& out, cudaStream_t s);

// ---- FFN glue (ffn.cu)
// h = relu(g)^2 * u; hn = subln(h); q2, s2, xsum2 = quant(hn) in `layout`.
cudaError_t launch_ffn_finalise(const float* g, const float* u, int64_t M, int64_t f, int layout,
                                int8_t* q2, float* s2, int32_t* xsum2, cudaStream_t s);

// tensor-parallel FFN pieces (ffn.cu): a rank owns fl of the f hidden columns
cudaError_t launch_ffn_tp_hstats(const float* g, const float* u, int64_t M, int64_t fl, float* h, double* ss,
                                 float* hmax, cudaStream_t s);
cudaError_t launch_ffn_tp_requant(const float* h, int64_t M, int64_t fl, int64_t f_total, const double* ss_all,
                                  const float* hmax_all, int layout, int8_t* q2, float* s2, int32_t* xsum2,
                                  cudaStream_t s);
// subln + requantisation of h from per-tile partials (sum h^2 fp64, max |h|),
// reduced in a fixed order per token; codes in `layout`.
cudaError_t launch_ffn_requant_parts(const float* h, const double* part_ss, const float* part_max, int nparts,
                                     int64_t M, int64_t f, int layout, int8_t* q2, float* s2, int32_t* xsum2,
                                     cudaStream_t s);
cudaError_t launch_ffn_tp_finish(const int32_t* acc, const float* gd, const float* s2, const uint16_t* residual,
                                 uint16_t* y, int64_t M, int64_t d, cudaStream_t s);

// ---- device error word: set by bounded waits inside kernels that give up.
// Address of the current device's word (for kernels), and a host read that
// also clears it.
cudaError_t device_error_word(unsigned int** ptr);
cudaError_t read_and_clear_device_error(unsigned int* value);

}  // namespace bl

/*
 * bitlinear.h -- C ABI of the B200 (sm_100a) BitLinear W1.58A8 library.
 *
 * The operation is the BitLinear forward of BitNet b1.58: ternary weights from
 * absmean quantisation packed four per byte, activations quantised per token to
 * int8 by absmax, an exact integer contraction, and a dequantisation to bf16.
 * Sources: "BitNet b1.58 2B4T Technical Report" paper card (ai-papers.xuzou.cn),
 * sections "Method Adaptation" (absmean ternary weights, per-token absmax int8
 * activations, subln, ReLU^2, no bias, four ternary weights per int8 value in
 * HBM, pack-store-load-unpack-compute kernel), "Compute Setup" (packed 1.58-bit
 * weights for inference, a custom W1.58A8 CUDA kernel) and "Bottleneck" (no
 * library kernel serves W1.58A8); the fishai news digest of the same report
 * (news.fishai.com.cn/news/3455510), list of the BitLinear layer's parts.
 *
 * Conventions shared by every call:
 *   - All tensor pointers are DEVICE pointers, allocated and owned by the caller.
 *     The library allocates no device memory in any call.
 *   - bf16 tensors are passed as their 16-bit patterns (uint16_t).
 *   - Matrices are row-major. W is [N, K] (out x in, as nn.Linear); x is [M, K];
 *     y and acc are [M, N].
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *     default stream). Arguments are validated on the host before anything is
 *     launched; on an error nothing is launched and the status says why.
 *   - No call synchronises the stream, except bitlinear_validate_packed and
 *     bitlinear_get_device_error, which say so.
 *   - No C++ exception crosses this boundary. A failed launch returns BL_ERR_CUDA.
 *   - Calls on different streams may overlap only if their workspaces differ.
 *   - Kernels launch with programmatic dependent launch: a call's kernel may start
 *     while the previous kernel in the stream finishes, and waits for it before
 *     reading its inputs x / h or writing anything. The packed weights (Wp, Wg,
 *     Wu, Wd) are the exception: the streamed GEMV starts copying them before that
 *     wait. So packed weights must not be written by the kernel just before the
 *     call in the same stream if that kernel triggers programmatic dependent launch
 *     early (the library's own kernels that do never write weights; the packing
 *     calls, host copies and ordinary kernels complete before a call starts).
 *
 * Packed weight format (this library's reading; the paper card, "Method
 * Adaptation", only fixes four ternary weights per 8-bit value): Wp is [N, K/4]
 * uint8, row-major. Byte j of row n holds weights k = 4j .. 4j+3; weight 4j+i
 * is stored in bits 2i..2i+1 as the code q+1 in {0, 1, 2} (q in {-1, 0, +1}).
 * Code 3 is invalid.
 *
 * Arithmetic (every step is one IEEE fp32 operation, round to nearest even, with
 * no fused multiply-add, unless noted):
 *   gamma = fp32( sum_{n,k} |W[n,k]| / (N*K) )      sum and division in fp64
 *   Wq    = clip(rint(W / (gamma + 1e-5)), -1, 1)
 *   s_m   = 127 / max(max_k |x[m,k]|, 1e-5)
 *   xq    = clip(rint(x * s_m), -128, 127)
 *   acc   = sum_k Wq[n,k] * xq[m,k]                 exact int32
 *   y     = bf16( float(acc) * (gamma / s_m) )      [+ float(residual) before bf16]
 */
#ifndef BITLINEAR_H
#define BITLINEAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, declared here so this header needs no CUDA headers. */
typedef struct CUstream_st* bl_stream_t;

typedef enum {
    BL_OK = 0,
    BL_ERR_NULL = 1,        /* a required pointer is NULL */
    BL_ERR_SHAPE = 2,       /* a size is negative, zero where it may not be, K % 4 != 0, or too large */
    BL_ERR_ALIGN = 3,       /* a pointer is not aligned as the call requires */
    BL_ERR_DTYPE = 4,       /* unknown bl_dtype */
    BL_ERR_WORKSPACE = 5,   /* workspace smaller than bitlinear_workspace_bytes() */
    BL_ERR_UNSUPPORTED = 6, /* valid arguments this build does not handle (e.g. no sm_100 device) */
    BL_ERR_CUDA = 7,        /* a CUDA call or launch failed */
    BL_ERR_TIMEOUT = 8,     /* a bounded wait inside a kernel gave up (see bitlinear_get_device_error) */
    BL_ERR_BAD_CODE = 9     /* packed weights hold the invalid code 3 */
} bl_status;

typedef enum { BL_BF16 = 0, BL_FP32 = 1 } bl_dtype;

/* Operation ids for bitlinear_workspace_bytes. */
typedef enum {
    BL_OP_PACK = 0,     /* sizes: N, K of the weight */
    BL_OP_FORWARD = 1,  /* sizes: M, N, K */
    BL_OP_FFN = 2,      /* sizes: M, N = f (hidden), K = d (model width) */
    BL_OP_VALIDATE = 3, /* sizes ignored */
    BL_OP_FFN_TP_UP = 4,    /* sizes: M, N = f_local (the rank's hidden columns), K = d */
    BL_OP_FFN_TP_DOWN = 5   /* sizes: M, N = d, K = f_local */
} bl_op;

/* Kernels for M <= 16 tokens (bitlinear_set_gemv_kernel). */
typedef enum {
    BL_GEMV_AUTO = 0,   /* the library picks per call (default) */
    BL_GEMV_STREAM = 1, /* streamed GEMV: dp4a (one token) / mma.sync (2..16 tokens) on registers */
    BL_GEMV_TENSOR = 2, /* tcgen05 GEMV: weights unpacked into tensor memory, tokens as the MMA's N */
    BL_GEMV_LUT = 3     /* lookup tables of activation partial sums indexed by packed weight nibbles
                           (the T-MAC method of the bitnet.cpp CPU kernels); four tokens per pass */
} bl_gemv_kernel;

/* Human-readable name of a status. Never NULL; host only. */
const char* bitlinear_status_string(bl_status status);

/* Bytes of workspace `op` needs for the given sizes (0 for an invalid op).
 * Host only, no CUDA call. The workspace must be 256-byte aligned. */
size_t bitlinear_workspace_bytes(int op, int64_t M, int64_t N, int64_t K);

/*
 * Absmean ternary quantisation and packing of one weight tensor (one-time work).
 * Paper card, "Method Adaptation": weights quantised with absmean onto {-1, 0, +1}
 * in the forward pass, four ternary weights packed into one 8-bit value in HBM.
 *
 *   W      [N, K] device, bf16 bits (wdt = BL_BF16) or fp32 (BL_FP32); 16-byte aligned
 *   N, K   N >= 1, K >= 4, K % 4 == 0, N*K < 2^40
 *   Wp     [N, K/4] device uint8 output (format above); 16-byte aligned
 *   gamma  [1] device fp32 output: mean |W| (the per-tensor absmean scale)
 *   ws     device workspace of bitlinear_workspace_bytes(BL_OP_PACK, 0, N, K) bytes
 * Deterministic: the fp64 sum runs in a fixed order for given N, K.
 */
bl_status bitlinear_pack_weights(const void* W, int wdt, int64_t N, int64_t K,
                                 uint8_t* Wp, float* gamma,
                                 void* ws, size_t ws_bytes, bl_stream_t stream);

/*
 * Per-token absmax quantisation of activations to int8.
 * Paper card, "Method Adaptation": activations quantised per token with absmax
 * to 8-bit integers.
 *
 *   x      [M, K] device bf16 bits; 16-byte aligned
 *   M, K   M >= 0 (M == 0 is a no-op), K >= 4, K % 4 == 0
 *   xq     [M, K] device int8 output, row-major; 16-byte aligned
 *   scale  [M] device fp32 output: s_m = 127 / max(absmax_m, 1e-5)
 *   xsum   [M] device int32 output: sum_k xq[m,k]; may be NULL
 */
bl_status bitlinear_quant_act(const uint16_t* x, int64_t M, int64_t K,
                              int8_t* xq, float* scale, int32_t* xsum, bl_stream_t stream);

/*
 * One BitLinear forward: quantise x per token, contract with the packed ternary
 * weights, dequantise to bf16. Dig news article on the release, section 2:
 * nn.Linear replaced by BitLinear; paper card, "Method Adaptation": packed int8
 * weights loaded to on-chip memory, unpacked right before the matmul, multiplied
 * with int8 activations. No bias.
 *
 *   Wp        [N, K/4] device packed weights; 16-byte aligned
 *   gamma     [1] device fp32 (as written by bitlinear_pack_weights)
 *   N, K      N >= 0, K >= 4, K % 4 == 0
 *   x         [M, K] device bf16 bits; 2-byte aligned (16-byte for the fast kernels)
 *   M         M >= 0; M == 0 or N == 0 launches nothing
 *   residual  [M, N] device bf16 bits added before the final rounding; may be NULL
 *   y         [M, N] device bf16 bits output; 4-byte aligned
 *   acc       [M, N] device int32 output of the exact accumulator; may be NULL
 *   ws        device workspace of bitlinear_workspace_bytes(BL_OP_FORWARD, M, N, K) bytes
 * Kernel choice: M <= 16 streams the packed weights once through a
 * bandwidth-bound GEMV (K % 256 == 0, Wp and x 16-byte aligned), quantising x
 * inside the same kernel for M <= 4 (not for four tokens with K > 4096 on small
 * N, where the separate quantisation is faster) when the codes of all M tokens
 * fit in 48 KiB (M * (K + 64) bytes); larger M runs the tensor-core GEMM (K % 64 == 0, same
 * alignment, any N), which for shapes whose tiles would leave most of the
 * last wave idle splits tiles across CTAs and keeps their partial sums in the
 * workspace (bitlinear_workspace_bytes includes that scratch only for such
 * shapes); other shapes take a generic kernel. Every path gives the same bits.
 */
bl_status bitlinear_forward(const uint8_t* Wp, const float* gamma, int64_t N, int64_t K,
                            const uint16_t* x, int64_t M, const uint16_t* residual,
                            uint16_t* y, int32_t* acc,
                            void* ws, size_t ws_bytes, bl_stream_t stream);

/*
 * Per-row absmean variant of bitlinear_pack_weights: one gamma per output row
 * instead of one per tensor (the paper card "BitNet b1.58 2B4T Technical
 * Report", "Method Adaptation", gives one absmean per weight tensor; this is the
 * finer-grained variant of that reading):
 *   gammas[n] = fp32( sum_k |W[n, k]| / K )     sum and division in fp64
 *   q[n, k]   = clip(rint(W[n, k] / (gammas[n] + 1e-5)), -1, 1)
 * and the same packed layout. Arguments as bitlinear_pack_weights, with
 * gammas [N] device fp32 (4-byte aligned) in place of gamma; no workspace.
 */
bl_status bitlinear_pack_weights_rowwise(const void* W, int wdt, int64_t N, int64_t K,
                                         uint8_t* Wp, float* gammas, bl_stream_t stream);

/*
 * bitlinear_forward with the per-row gammas of bitlinear_pack_weights_rowwise:
 *   y[m, n] = bf16([residual[m, n] +] float(acc[m, n]) * (gammas[n] / s_m))
 * Arguments, kernel choice and errors as bitlinear_forward, with gammas [N]
 * device fp32 in place of gamma; the same workspace.
 */
bl_status bitlinear_forward_rowwise(const uint8_t* Wp, const float* gammas, int64_t N, int64_t K,
                                    const uint16_t* x, int64_t M, const uint16_t* residual,
                                    uint16_t* y, int32_t* acc,
                                    void* ws, size_t ws_bytes, bl_stream_t stream);

/*
 * Several BitLinear projections of one input in one call, optionally after a
 * unit-weight RMSNorm of the input: the attention side of a BitNet b1.58 block
 * (paper card "BitNet b1.58 2B4T Technical Report", "Method Adaptation":
 * BitLinear replaces the linear layers, subln sub-layer normalisation; fishai
 * digest, BitLinear list). The query, key and value projections read the same
 * normalised x; the output projection reads the subln-normalised attention
 * output and adds the residual.
 *   y[m, n] = bf16([residual[m, n] +] float(acc[m, n]) * (gammas[seg(n)] / s_m))
 *   xq, s   = quant(rmsnorm ? x * r : x),  r = 1 / sqrtf(float(sum_k x^2 / K) + 1e-5)
 *             per token (sum in fp64; x * r kept in fp32 and quantised as in
 *             bitlinear_forward)
 * Arguments:
 *   Wp        [N, K/4] device: the packed rows of nseg weight matrices stacked
 *             row-wise (each packed by bitlinear_pack_weights; packed rows are
 *             independent, so stacking is a byte copy); N = sum of seg_rows
 *   gammas    [nseg] device fp32: gamma of each matrix, in the same order
 *   seg_rows  [nseg] host: rows of each matrix, each >= 1; 1 <= nseg <= 4
 *   K, x, M   as bitlinear_forward
 *   rmsnorm   0: quantise x; 1: quantise the unit-weight RMSNorm of x
 *   residual, y, acc   [M, N], as bitlinear_forward
 *   ws        device workspace of bitlinear_workspace_bytes(BL_OP_FORWARD, M, N, K)
 * Kernel choice as bitlinear_forward. Segment boundaries on multiples of 16 rows
 * keep the streamed GEMV (M <= 16) and on multiples of 32 the tensor-core GEMM;
 * other boundaries run the generic kernel. Errors: BL_ERR_SHAPE for nseg outside
 * 1..4, rmsnorm not 0 or 1, a segment without rows, or the bitlinear_forward
 * shape rules on N = sum of seg_rows; otherwise as bitlinear_forward.
 */
bl_status bitlinear_forward_ex(const uint8_t* Wp, const float* gammas, const int64_t* seg_rows,
                               int32_t nseg, int64_t K, const uint16_t* x, int64_t M,
                               int32_t rmsnorm, const uint16_t* residual, uint16_t* y,
                               int32_t* acc, void* ws, size_t ws_bytes, bl_stream_t stream);

/*
 * One FFN sub-layer of BitNet b1.58 (fishai digest: ReLU^2 in the FFN, subln;
 * paper card, "Method Adaptation": subln, ReLU^2 feed-forward, no bias):
 *   xq, s   = quant(x)                       x [M, d]
 *   g, u    = deq(Wg . xq), deq(Wu . xq)     fp32, [M, f]
 *   h       = max(g, 0)^2 * u
 *   hn      = h / sqrt(mean_j h^2 + 1e-5)    unit-weight RMSNorm; sum in fp64
 *   q2, s2  = quant(hn)
 *   y       = bf16(residual + deq(Wd . q2))  y [M, d]; residual may be NULL
 *   Wg, Wu  [f, d/4] packed; gg, gu [1] device fp32
 *   Wd      [d, f/4] packed; gd [1] device fp32
 *   d, f    multiples of 4
 *   ws      bitlinear_workspace_bytes(BL_OP_FFN, M, f, d) bytes
 * Alignment as bitlinear_forward.
 */
bl_status bitlinear_ffn(const uint8_t* Wg, const float* gg, const uint8_t* Wu, const float* gu,
                        const uint8_t* Wd, const float* gd, int64_t d, int64_t f,
                        const uint16_t* x, int64_t M, const uint16_t* residual, uint16_t* y,
                        void* ws, size_t ws_bytes, bl_stream_t stream);

/*
 * bitlinear_forward without a workspace, for callers that cannot allocate.
 * The pages have no counterpart of this call; it exists for deployment.
 *
 * Some callers cannot call cudaMalloc where they run a layer: a plugin inside an
 * engine that reserved all device memory at start-up and allows no allocation
 * afterwards, or a latency-critical loop in which an allocation would implicitly
 * synchronise the device. They may also have no workspace buffer to pass. This
 * call computes what bitlinear_forward computes, to the same integers and bf16
 * bits, but keeps its scratch in a fixed 1 MiB array inside the library's own
 * device memory, which every GPU that loads the library holds until the process
 * exits. It always runs the separate act-quant kernel and then the GEMV (the
 * streamed one when K % 256 == 0 and Wp and x are 16-byte aligned, else the
 * generic one), also for M > 16, where bitlinear_forward uses the tensor cores:
 * large M is correct but slow here.
 *
 *   Arguments as bitlinear_forward, minus ws / ws_bytes.
 *   Limit: the scratch must hold the activation codes plus two per-token words:
 *          round256(M*K) + 2*round256(4*M) <= 1048576 bytes (for example M <= 16 at
 *          K <= 28672). Larger sizes return BL_ERR_WORKSPACE and launch nothing.
 *   No call allocates device memory or calls an allocating library routine.
 *   The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress). After a cudaDeviceReset the next call on that
 *   device looks it up again.
 *   Every call on a device shares the one array, which keeps the last call's
 *   contents (nothing in it needs to start at zero). Calls that can overlap on
 *   the GPU (other streams, unordered host threads) race on it: order them.
 */
bl_status bitlinear_forward_noalloc(const uint8_t* Wp, const float* gamma, int64_t N, int64_t K,
                                    const uint16_t* x, int64_t M, const uint16_t* residual,
                                    uint16_t* y, int32_t* acc, bl_stream_t stream);

/*
 * Selects, for the whole process, which kernel the forward calls
 * (bitlinear_forward, _ex, _rowwise and the projections inside bitlinear_ffn)
 * use for M <= 16 tokens; the choice is read when a call launches its kernels.
 * It exists to compare the kernels and to pin one in deployment; every kernel
 * computes the same integers and bf16 bits. A kernel that cannot take a call's
 * shape or alignment (all need K % 256 == 0 and 16-byte aligned Wp and x)
 * leaves that call to the automatic choice. The paper card "BitNet b1.58 2B4T
 * Technical Report", "Method Adaptation", describes one GPU kernel, the
 * streamed and tensor-core GEMVs are this library's designs for B200, and the
 * lookup-table GEMV follows the bitnet.cpp CPU kernels (dignews article on the
 * release, section 3: lookup tables after T-MAC, lossless).
 *   kind   a bl_gemv_kernel value
 * Returns the previous selection, or -1 (and changes nothing) for an unknown kind.
 * Host only, no CUDA call.
 */
int bitlinear_set_gemv_kernel(int kind);

/*
 * Tensor-parallel pieces of the FFN sub-layer. The pages give no distributed
 * detail (paper card "BitNet b1.58 2B4T Technical Report", "Limits"); this is
 * the library's split of bitlinear_ffn over P ranks (one GPU each): rank r owns
 * f_local of the f hidden columns, i.e. those rows of the gate and up weights
 * and those columns of the down weight, packed with the gammas of the whole
 * tensors. Per layer, between the calls, the caller exchanges (NCCL over
 * NVLink, or any transport): the per-token sums ss (fp64, sum) and maxima hmax
 * (fp32, max) after bitlinear_ffn_tp_up, and the int32 accumulators (sum, exact
 * in any order) after bitlinear_ffn_tp_down. The result equals bitlinear_ffn on
 * the whole weights bit for bit, up to the order of the fp64 sum of the ranks'
 * ss (a different fp32 subln factor needs those sums to straddle an fp32
 * rounding boundary).
 *
 * Packing a shard: the per-tensor gamma of the paper card's absmean ("Method
 * Adaptation") is over the whole tensor, so each rank adds its fp64 sum of |W|
 * (bitlinear_absmean_sum, into a device double) to the others' and packs its
 * shard with that total (bitlinear_pack_weights_global).
 */

/* fp64 sum of |W| over one shard [N, K] of a weight tensor (bf16 or fp32, as
 * bitlinear_pack_weights), written to *sum (device, 8-byte aligned), in a fixed
 * order. ws: bitlinear_workspace_bytes(BL_OP_PACK, 0, N, K) bytes. */
bl_status bitlinear_absmean_sum(const void* W, int wdt, int64_t N, int64_t K, double* sum,
                                void* ws, size_t ws_bytes, bl_stream_t stream);

/* Pack one shard [N, K] with the gamma of the whole tensor:
 *   gamma = fp32(*total_sum / total_count)   (device double, fp64 division)
 * total_sum: the fp64 sum of |W| over every shard; total_count: the element count
 * of the whole tensor (>= N * K). Wp [N, K/4] and gamma [1] as bitlinear_pack_weights. */
bl_status bitlinear_pack_weights_global(const void* W, int wdt, int64_t N, int64_t K, const double* total_sum,
                                        int64_t total_count, uint8_t* Wp, float* gamma, bl_stream_t stream);

/* Rank-local first half of the FFN: xq, s = quant(x) (x [M, d] whole on every
 * rank); g, u = deq(Wg . xq), deq(Wu . xq) on the rank's f_local rows (fp32);
 * h = max(g, 0)^2 * u -> h [M, f_local] fp32 (device); per token the rank's share of
 * the subln statistics: ss[m] = sum_j h[m, j]^2 (fp64) and hmax[m] = max_j |h[m, j]|.
 *   Wg, Wu  [f_local, d/4] packed shard rows; gg, gu [1] device fp32 (whole-tensor gammas)
 *   ws      bitlinear_workspace_bytes(BL_OP_FFN_TP_UP, M, f_local, d) bytes */
bl_status bitlinear_ffn_tp_up(const uint8_t* Wg, const float* gg, const uint8_t* Wu, const float* gu,
                              int64_t d, int64_t f_local, const uint16_t* x, int64_t M, float* h, double* ss,
                              float* hmax, void* ws, size_t ws_bytes, bl_stream_t stream);

/* Rank-local second half, after ss and hmax are reduced over the ranks
 * (ss_all = sum, hmax_all = max; device, [M]):
 *   r  = 1 / sqrtf(float(ss_all / f_total) + 1e-5)
 *   s2 = 127 / max(fl(hmax_all * r), 1e-5)          -> s2 [M] device fp32
 *   q2 = clip(rint(fl(h * r) * s2))                  the rank's columns
 *   acc[m, n] = sum_{j in the rank's columns} Wd[n, j] q2[m, j]  -> acc [M, d] int32
 *   Wd  [d, f_local/4] packed shard columns (packed with the whole tensor's gamma)
 *   ws  bitlinear_workspace_bytes(BL_OP_FFN_TP_DOWN, M, d, f_local) bytes */
bl_status bitlinear_ffn_tp_down(const uint8_t* Wd, int64_t d, int64_t f_local, int64_t f_total, const float* h,
                                int64_t M, const double* ss_all, const float* hmax_all, int32_t* acc, float* s2,
                                void* ws, size_t ws_bytes, bl_stream_t stream);

/* After acc is summed over the ranks: y = bf16([residual +] float(acc) * (gd / s2)).
 *   acc [M, d] int32, s2 [M] fp32, gd [1] (whole-tensor gamma), residual [M, d] bf16
 *   (may be NULL), y [M, d] bf16; all device. No workspace. */
bl_status bitlinear_ffn_tp_finish(const int32_t* acc, const float* gd, const float* s2, const uint16_t* residual,
                                  uint16_t* y, int64_t M, int64_t d, bl_stream_t stream);

/*
 * Check packed weights for the invalid code 3. SYNCHRONISES `stream`.
 * Returns BL_OK when every code is valid, BL_ERR_BAD_CODE otherwise; the number
 * of invalid codes is written to *bad_count (host pointer, may be NULL).
 *   ws  bitlinear_workspace_bytes(BL_OP_VALIDATE, 0, 0, 0) bytes of device memory
 */
bl_status bitlinear_validate_packed(const uint8_t* Wp, int64_t N, int64_t K, int64_t* bad_count,
                                    void* ws, size_t ws_bytes, bl_stream_t stream);

/*
 * SYNCHRONISES `stream`, then reports BL_ERR_CUDA for a pending CUDA error, or
 * BL_ERR_TIMEOUT when a bounded wait inside one of this library's kernels gave up
 * since the last call on this device (the kernel that gave up wrote no output it
 * could not finish and returned); the timeout flag is cleared by this call.
 */
bl_status bitlinear_get_device_error(bl_stream_t stream);

/*
 * Self-test of the failure path (no counterpart in the method; it exists to
 * test this library's error reporting). Launches, on `stream`, one thread that
 * waits with the library's bounded mbarrier wait on a barrier nothing arrives
 * on; after limit_us microseconds (1 .. 2,000,000) the wait gives up, records a
 * timeout in the device error word and the kernel returns normally. The next
 * bitlinear_get_device_error on this device then reports BL_ERR_TIMEOUT (and
 * clears it). The GPU context stays usable. Returns the launch status.
 */
bl_status bitlinear_selftest_timeout(int64_t limit_us, bl_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* BITLINEAR_H */

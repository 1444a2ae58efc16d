/*
 * bitlinear.h — C ABI of libbitlinear.so, the BitNet b1.58 BitLinear W1.58·A8
 * matmul for NVIDIA B200 (sm_100a).
 *
 * The three calls follow the pages' statement of the layer: quantise the
 * weights once and cache them, quantise the activations on every forward,
 * multiply in integers, then dequantise and add the bias ("1.58-bit 大模型极限
 * 量化实战：从 BitNet 三值权重到单颗 CPU 跑起 100B 模型", chenxutan.com/d/5049.html,
 * §3.2 and §4.2).
 *
 * Conventions for every call:
 *  - Tensor pointers are DEVICE pointers owned by the caller; the library keeps
 *    none of them after the call returns and allocates no device memory.
 *  - Work is enqueued asynchronously on `stream` (NULL = the legacy default
 *    stream).  Outputs are valid once the stream reaches that point.
 *  - Every call returns a bitlinear_status and never throws or aborts.
 *    Argument errors are found on the host before anything is launched, and
 *    then no output is touched.  BL_ERR_CUDA reports a launch failure.
 *  - Calls are thread-safe; calls on one stream run in order.
 *  - Arithmetic is IEEE binary32 with round-to-nearest-even except where a
 *    call says otherwise; the integer path is exact.  Results are bit-for-bit
 *    reproducible for a given input, whatever the device's SM count.
 *  - The library runs only on compute capability 10.0 (B200); elsewhere calls
 *    return BL_ERR_ARCH.
 */
#ifndef BITLINEAR_H
#define BITLINEAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define BITLINEAR_API __attribute__((visibility("default")))
#else
#define BITLINEAR_API
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* bitlinear_stream_t;

typedef enum bitlinear_status {
    BL_OK = 0,
    BL_ERR_NULL = 1,      /* a required pointer is NULL */
    BL_ERR_SHAPE = 2,     /* a size is < 1 or above its stated maximum */
    BL_ERR_ALIGN = 3,     /* a pointer breaks its stated alignment */
    BL_ERR_DTYPE = 4,     /* unknown bitlinear_dtype */
    BL_ERR_WORKSPACE = 5, /* workspace NULL or smaller than required */
    BL_ERR_ARCH = 6,      /* current device is not compute capability 10.0 */
    BL_ERR_CUDA = 7,      /* the CUDA runtime reported an error */
    BL_ERR_COUNT = 8,     /* group count outside 1..BITLINEAR_MAX_GROUP */
    BL_ERR_TIMEOUT = 9,   /* a kernel's bounded wait expired (see bitlinear_device_error) */
    BL_ERR_FLAGS = 10     /* unknown flag bits */
} bitlinear_status;

typedef enum bitlinear_dtype {
    BL_F32 = 0,  /* IEEE binary32 */
    BL_BF16 = 1  /* bfloat16; widened exactly to binary32 before any arithmetic */
} bitlinear_dtype;

/* Largest K (input features) accepted; keeps every int32 accumulator exact. */
#define BITLINEAR_MAX_K ((int64_t)1 << 20)
/* Largest number of problems in one grouped call. */
#define BITLINEAR_MAX_GROUP 16

/* Bytes of one packed weight row: 16·ceil(K/64) (0 if K < 1).
 *
 * Packed weight layout ("W_packed", row-major [N][bitlinear_packed_row_bytes(K)]
 * uint8, 16-byte aligned): 2 bits per weight with codes 00/01/10 for the
 * ternary values -1/0/+1 (the pages' storage, chenxutan.com/d/5049.html §5.3);
 * row n holds output feature n, contiguous along the K input features.  The
 * row is read as little-endian 32-bit words of 16 weights each: weight
 * k = 16g + 4s + b lives in byte b of word g, bits 2s..2s+1.  So masking a word
 * with 0x03030303 << 2s yields the codes of weights 16g+4s .. 16g+4s+3 in the
 * four bytes, in order.  Weights k >= K are padding with code 01 (zero).  Code
 * 11 is never written by bitlinear_quantize_weights; a product over packed
 * data that contains it gives unspecified results. */
BITLINEAR_API size_t bitlinear_packed_row_bytes(int64_t K);

/* Device workspace bytes bitlinear_quantize_weights needs for an N×K matrix. */
BITLINEAR_API size_t bitlinear_quantize_weights_workspace_bytes(int64_t N, int64_t K);

/* Absmean ternary weight quantisation (chenxutan.com/d/5049.html §2.3, §4.1):
 *   α = mean(|W|) over the whole tensor, Ŵ = clip(round(W/α), -1, 1),
 * round = half to even, W/α one binary32 division (a NaN quotient, possible
 * only when α underflows to 0, gives the zero weight).  The sum of |W| is
 * exact; α = RN32(RN64(Σ|W| / (N·K))).
 *
 *   W          [N][K] row-major, `dtype`, aligned to its element size.
 *   W_packed   out: [N][bitlinear_packed_row_bytes(K)] uint8, 16-byte aligned.
 *   alpha      out: 1 float.
 *   workspace  device scratch of at least
 *              bitlinear_quantize_weights_workspace_bytes(N, K) bytes, 8-byte
 *              aligned; its contents are undefined afterwards.
 * Errors: BL_ERR_NULL, BL_ERR_SHAPE (N < 1, K < 1, K > BITLINEAR_MAX_K,
 * N·K > 2^40), BL_ERR_ALIGN, BL_ERR_DTYPE, BL_ERR_WORKSPACE, BL_ERR_ARCH,
 * BL_ERR_CUDA.  Non-finite weights give an undefined α. */
BITLINEAR_API bitlinear_status bitlinear_quantize_weights(const void* W, bitlinear_dtype dtype, int64_t N, int64_t K,
                                            uint8_t* W_packed, float* alpha, void* workspace,
                                            size_t workspace_bytes, bitlinear_stream_t stream);

/* bitlinear_quantize_weights without a workspace argument, for callers that
 * may not allocate device memory at all: a plugin running inside a host
 * application that owns the whole device-memory budget, or a latency-critical
 * loop in which cudaMalloc/cudaFree (which can synchronise the device) are
 * not allowed.  The pages have no counterpart: this is a packaging variant of
 * the same quantisation, with identical results.
 *
 * Its scratch (the partial sums of α) is a fixed 80 KiB array inside the
 * library that every GPU loading the library holds until the process exits;
 * the call allocates nothing.  Every call on a device shares that array and
 * overwrites what it reads, so calls that overlap on the GPU (e.g. on two
 * unordered streams) race and give wrong results; order them on one stream.
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) and so should come before any stream capture.  The
 * address is kept for the life of the process: resetting a device
 * (cudaDeviceReset) after that first call is not supported.
 * Arguments, layouts and errors are those of bitlinear_quantize_weights; the
 * maximum size is the same (N·K <= 2^40, K <= BITLINEAR_MAX_K), and larger
 * sizes return BL_ERR_SHAPE. */
BITLINEAR_API bitlinear_status bitlinear_quantize_weights_static(const void* W, bitlinear_dtype dtype, int64_t N,
                                                                 int64_t K, uint8_t* W_packed, float* alpha,
                                                                 bitlinear_stream_t stream);

/* Per-token absmax int8 activation quantisation (chenxutan.com/d/5049.html
 * §2.4, §4.1; per token as in nxmr.cn/news/148658 §3.2), for each row m:
 *   β_m = max_k |x[m][k]| + 1e-8   (binary32 add)
 *   x̃[m][k] = clip(round((x[m][k]·127) / β_m), -127, 127)
 * with the product and the quotient each rounded to binary32, half to even.
 *
 *   x     [M][K] row-major, `dtype`, aligned to its element size.
 *   x_q   out: [M][K] int8 row-major (row stride K).
 *   beta  out: [M] float.
 * Errors: BL_ERR_NULL, BL_ERR_SHAPE (M < 1, K < 1, K > BITLINEAR_MAX_K,
 * M > 2^31), BL_ERR_ALIGN, BL_ERR_DTYPE, BL_ERR_ARCH, BL_ERR_CUDA.  Non-finite
 * inputs give undefined results. */
BITLINEAR_API bitlinear_status bitlinear_quantize_act(const void* x, bitlinear_dtype dtype, int64_t M, int64_t K,
                                        int8_t* x_q, float* beta, bitlinear_stream_t stream);

/* Ternary product and dequantisation (chenxutan.com/d/5049.html §2.4–§2.5,
 * §4.2; add / subtract / skip as in nxmr.cn/news/148658 §3.3):
 *   acc[m][n] = Σ_k x̃[m][k]·Ŵ[n][k]                       (exact int32)
 *   s_m       = RN32( RN64( (double)α·(double)β_m / 127 ) )
 *   y[m][n]   = RN32( fp32(acc[m][n])·s_m )  (+ bias[n], binary32 add)
 *
 *   x_q, beta  from bitlinear_quantize_act ([M][K] int8, [M] float).
 *   W_packed, alpha  from bitlinear_quantize_weights for an N×K matrix;
 *              W_packed 16-byte aligned.
 *   bias       optional [N] float (NULL = no bias).
 *   y          out: [M][N] float row-major.
 *   acc_out    optional out: [M][N] int32 accumulators (NULL = not written).
 * Kernel choice is by shape only and never changes a result.
 * Errors: BL_ERR_NULL, BL_ERR_SHAPE (M, N, K < 1, K > BITLINEAR_MAX_K,
 * M or N > 2^31), BL_ERR_ALIGN, BL_ERR_ARCH, BL_ERR_CUDA. */
BITLINEAR_API bitlinear_status bitlinear_forward(const int8_t* x_q, const float* beta, int64_t M, int64_t K,
                                   const uint8_t* W_packed, const float* alpha, int64_t N,
                                   const float* bias, float* y, int32_t* acc_out,
                                   bitlinear_stream_t stream);

/* One problem of a grouped activation quantisation; fields as in
 * bitlinear_quantize_act. */
typedef struct bitlinear_act_problem {
    const void* x;
    int8_t* x_q;
    float* beta;
    int64_t M, K;
} bitlinear_act_problem;

/* bitlinear_quantize_act on `count` independent problems of one dtype in a
 * single launch (e.g. the several inputs of one transformer layer).
 * `problems` is a HOST array; it may be reused as soon as the call returns.
 * Errors: as bitlinear_quantize_act, plus BL_ERR_COUNT. */
BITLINEAR_API bitlinear_status bitlinear_quantize_act_grouped(const bitlinear_act_problem* problems, int count,
                                                bitlinear_dtype dtype, bitlinear_stream_t stream);

/* One problem of a grouped forward; fields as in bitlinear_forward.  Above
 * four tokens (and at three or four tokens when the call's weights total
 * 8 MB or more) all problems of a call share one tensor-core launch. */
typedef struct bitlinear_forward_problem {
    const int8_t* x_q;
    const float* beta;
    const uint8_t* W_packed;
    const float* alpha;
    const float* bias;
    float* y;
    int32_t* acc_out;
    int64_t M, N, K;
} bitlinear_forward_problem;

/* bitlinear_forward on `count` independent problems in a single launch, so
 * that the weight streams of several small matrices overlap (e.g. the seven
 * linears of one decoder layer).  `problems` is a HOST array.
 * Errors: as bitlinear_forward, plus BL_ERR_COUNT. */
BITLINEAR_API bitlinear_status bitlinear_forward_grouped(const bitlinear_forward_problem* problems, int count,
                                           bitlinear_stream_t stream);

/* One problem of a grouped linear (activation quantisation + forward);
 * fields as in bitlinear_quantize_act and bitlinear_forward.  x_q and beta are
 * outputs of the first step and inputs of the second. */
typedef struct bitlinear_linear_problem {
    const void* x;
    int8_t* x_q;
    float* beta;
    const uint8_t* W_packed;
    const float* alpha;
    const float* bias;
    float* y;
    int32_t* acc_out;
    int64_t M, N, K;
} bitlinear_linear_problem;

/* The BitLinear forward on cached weights (chenxutan.com/d/5049.html §3.2,
 * steps 2-4): bitlinear_quantize_act on x, then bitlinear_forward, with
 * identical results.  Both kernels use programmatic dependent launch: the
 * quantisation kernel waits for the work before it on `stream` before reading
 * x, and the product kernel starts streaming its weights as soon as the
 * quantisation kernel releases it, then waits for x̃ and β.  So consecutive
 * calls overlap each other's start-up and drain.
 * Errors: the union of both calls'. */
BITLINEAR_API bitlinear_status bitlinear_linear(const void* x, bitlinear_dtype dtype, int64_t M, int64_t K,
                                                const uint8_t* W_packed, const float* alpha, int64_t N,
                                                const float* bias, int8_t* x_q, float* beta, float* y,
                                                int32_t* acc_out, bitlinear_stream_t stream);

/* Flag for bitlinear_linear_grouped: the weights (W_packed, alpha) of this
 * call are not written by any work still running on the stream.  The product
 * kernel may then begin streaming weights while the work before the call is
 * still finishing (e.g. the previous layer's product), instead of after it. */
#define BL_LINEAR_WEIGHTS_STATIC 1u

/* Flag for bitlinear_linear_grouped: rotate each input x by the Hadamard
 * matrix of block bitlinear_hadamard_block(K) before quantising it (x_q and
 * beta then hold the rotated input's quantisation); the weights must have been
 * quantised from W·H/block.  Each K must have bitlinear_hadamard_block(K) > 1. */
#define BL_LINEAR_HADAMARD 2u

/* bitlinear_linear on `count` independent problems of one input dtype: one
 * grouped quantisation launch and one grouped product launch.  `problems` is a
 * HOST array.  flags: BL_LINEAR_WEIGHTS_STATIC and/or BL_LINEAR_HADAMARD.
 * With at most four tokens per problem (one token when rotated, K ≤ 24576) the
 * quantisation (and rotation) may instead run in the product kernel's prologue
 * (one launch; x_q and beta are still written),
 * when the problems fit it and the input rows are small next to the weights;
 * the environment variable BITLINEAR_LINEAR_FUSION=on|off forces the choice.
 * Results are identical either way.
 * Errors: as bitlinear_linear, plus BL_ERR_COUNT, BL_ERR_FLAGS. */
BITLINEAR_API bitlinear_status bitlinear_linear_grouped(const bitlinear_linear_problem* problems, int count,
                                                        bitlinear_dtype dtype, uint32_t flags,
                                                        bitlinear_stream_t stream);

/* Host-side input and output of one problem of bitlinear_linear_grouped_host. */
typedef struct bitlinear_host_io {
    const void* x_host; /* [M][K] `dtype`, HOST memory: copied into the problem's device x */
    float* y_host;      /* [M][N] float32, HOST memory: receives the problem's device y */
} bitlinear_host_io;

/* bitlinear_linear_grouped with the inputs and outputs in HOST memory (the
 * inference path of "1.58-bit 大模型极限量化实战", chenxutan.com/d/5049.html
 * §4.2, seen from a host program): enqueues on `stream` the copy of every
 * io[i].x_host into problems[i].x, the grouped linear, and the copy of every
 * problems[i].y into io[i].y_host.  The device buffers of `problems` are used
 * as by bitlinear_linear_grouped (x is overwritten by the copy).  Copies of
 * problems whose host and device buffers are both adjacent are merged into one
 * cudaMemcpyAsync, and a problem whose x (and x_host) repeats an earlier
 * problem's is copied once.  Host memory should be page-locked: with pageable
 * memory CUDA performs the copies synchronously.  The call returns once the
 * work is enqueued; y_host is valid after the stream reaches the end of it,
 * and neither host buffer may be modified before then.  `io` is a HOST array
 * of `count` entries.
 * Errors: as bitlinear_linear_grouped, plus BL_ERR_NULL (io or a host pointer
 * NULL) and BL_ERR_CUDA from a copy (work already enqueued stays enqueued). */
BITLINEAR_API bitlinear_status bitlinear_linear_grouped_host(const bitlinear_linear_problem* problems,
                                                             const bitlinear_host_io* io, int count,
                                                             bitlinear_dtype dtype, uint32_t flags,
                                                             bitlinear_stream_t stream);

/* One input of bitlinear_linear_block: x = a, or x = a + b added element-wise
 * in binary32 (round to nearest) when b is not NULL — the residual addition
 * that stays in floating point between BitLinear layers while every BitLinear
 * input is quantised on entry ("1.58-bit 大模型极限量化实战",
 * chenxutan.com/d/5049.html §6.1).  x is quantised exactly as by
 * bitlinear_quantize_act into x_q [M][K] and beta [M]; x_sum (nullable,
 * [M][K] float32) receives x itself.  a, b and x_sum are float32 [M][K]
 * row-major, 4-byte aligned; x_q as in bitlinear_quantize_act.
 * x_sum may be exactly a or exactly b (an in-place residual update h += y);
 * otherwise it must not overlap any a or b of the call (a partial overlap
 * gives undefined results).  When an x_sum overlaps an input, the call does
 * not take the single-launch fused form described below. */
typedef struct bitlinear_act_sum_problem {
    const float* a;
    const float* b;
    float* x_sum;
    int8_t* x_q;
    float* beta;
    int64_t M, K;
} bitlinear_act_sum_problem;

/* A block of linears that share quantised inputs (e.g. the q, k, v, gate and
 * up projections of one layer all reading quant(h)): one grouped quantisation
 * launch over the n_acts inputs, then one grouped product launch over the
 * n_fwd problems, each reading an x_q / beta written by the first step (or
 * any other), chained by programmatic dependent launch exactly as in
 * bitlinear_linear_grouped.  Either count may be 0, not both; each is at most
 * BITLINEAR_MAX_GROUP.  Both arrays are HOST arrays, reusable on return.
 * flags: 0 or BL_LINEAR_WEIGHTS_STATIC.  As in bitlinear_linear_grouped, with
 * at most four tokens the quantisation may run inside the product kernel when
 * every product reads one of this call's inputs and every input feeds one;
 * the first product of each input then writes its x_q, beta and x_sum.
 * Errors: as bitlinear_quantize_act (per input) and bitlinear_forward (per
 * problem), plus BL_ERR_COUNT and BL_ERR_FLAGS; nothing is launched then. */
BITLINEAR_API bitlinear_status bitlinear_linear_block(const bitlinear_act_sum_problem* acts, int n_acts,
                                                      const bitlinear_forward_problem* fwd, int n_fwd,
                                                      uint32_t flags, bitlinear_stream_t stream);

/* ---- Hadamard rotation before the absmax quantisation ("1.58-bit 大模型极限
 * 量化实战", chenxutan.com/d/5049.html §6.2: a few activation dimensions hold
 * large outliers that inflate β = max|x| and crush every other dimension; an
 * orthogonal Hadamard rotation of the activations first spreads them out).
 *
 * H is block-diagonal with Sylvester blocks of order `block` (a power of two
 * dividing K, at most BITLINEAR_MAX_HADAMARD_BLOCK): inside a block
 * out[j] = Σ_i x[i]·(-1)^popcount(i & j), unnormalised.  It is evaluated by
 * the butterfly network in binary32, stages h = 1, 2, 4, …, block/2 in that
 * order, each butterfly replacing the pair (i, i+h), i & h == 0, by
 * (a + b, a - b); so results are reproducible bit for bit.  The product is
 * unchanged when the weights take the same rotation scaled by 1/block:
 * (x·H)·(W·H/block)ᵀ = x·Wᵀ.  So a rotated layer quantises W' = W·H/block
 * (bitlinear_hadamard with scale 1/block, then bitlinear_quantize_weights)
 * and rotates x before bitlinear_quantize_act (bitlinear_quantize_act_hadamard,
 * or BL_LINEAR_HADAMARD on a linear call). */
#define BITLINEAR_MAX_HADAMARD_BLOCK 8192

/* The block a linear call flagged BL_LINEAR_HADAMARD uses: the largest power
 * of two dividing K, at most BITLINEAR_MAX_HADAMARD_BLOCK (0 if K < 1). */
BITLINEAR_API int64_t bitlinear_hadamard_block(int64_t K);

/* out[m][·] = (x[m][·]·H)·scale, each output one binary32 multiply by `scale`
 * after the last stage (scale 1 for activations, 1/block for weights).
 *   x    [M][K] row-major, `dtype`, aligned to its element size.
 *   out  [M][K] float32 (must not overlap x).
 * Errors: BL_ERR_NULL, BL_ERR_SHAPE (M, K < 1, K > BITLINEAR_MAX_K, M > 2^31,
 * block not a power of two dividing K or above the maximum), BL_ERR_ALIGN,
 * BL_ERR_DTYPE, BL_ERR_ARCH, BL_ERR_CUDA. */
BITLINEAR_API bitlinear_status bitlinear_hadamard(const void* x, bitlinear_dtype dtype, int64_t M, int64_t K,
                                                  int64_t block, float scale, float* out, bitlinear_stream_t stream);

/* bitlinear_quantize_act of x·H: β_m = max_k |(x·H)[m][k]| + 1e-8 and
 * x̃ = clip(round((x·H)·127/β), -127, 127), the rotated values never leaving
 * the chip.  Arguments as bitlinear_quantize_act plus `block`; errors as
 * bitlinear_hadamard. */
BITLINEAR_API bitlinear_status bitlinear_quantize_act_hadamard(const void* x, bitlinear_dtype dtype, int64_t M,
                                                               int64_t K, int64_t block, int8_t* x_q, float* beta,
                                                               bitlinear_stream_t stream);

/* ---- Finer scale granularity: one α per output row ("1.58 位大模型",
 * nxmr.cn/news/148658 §3.1, §4.2: alpha = mean(|w|) of each row) or per block
 * of `group` consecutive input features of a row (2kiu.com/news/4928193 §2.3,
 * §4.2: one scale per 128 elements, scale[C_out][C_in/128]).  `group` >= K
 * means one α per row; otherwise it must be a multiple of 64 (the page uses
 * 128); the last block of a row may be shorter.  alpha is [N][ceil(K/group)]
 * float32, each the exact mean of |W| over its group rounded once to binary64
 * and once to binary32 (as for the tensor). */

/* Absmean ternary quantisation with one α per group:
 * Ŵ[n][k] = clip(round(W[n][k] / α[n][k/group]), -1, 1), packed as for
 * bitlinear_quantize_weights.  Needs no workspace.
 * Errors: BL_ERR_NULL, BL_ERR_SHAPE (as bitlinear_quantize_weights, or group
 * < K and not a positive multiple of 64), BL_ERR_ALIGN, BL_ERR_DTYPE,
 * BL_ERR_ARCH, BL_ERR_CUDA. */
BITLINEAR_API bitlinear_status bitlinear_quantize_weights_scaled(const void* W, bitlinear_dtype dtype, int64_t N,
                                                                 int64_t K, int64_t group, uint8_t* W_packed,
                                                                 float* alpha, bitlinear_stream_t stream);

/* One problem of bitlinear_linear_scaled.  x (nullable): the input, quantised
 * into x_q and beta first as by bitlinear_quantize_act; when NULL, x_q and
 * beta are inputs.  acc_out (nullable) receives the int32 products and is
 * allowed only with one α per row (group >= K). */
typedef struct bitlinear_scaled_problem {
    const void* x;
    int8_t* x_q;
    float* beta;
    const uint8_t* W_packed;
    const float* alpha;
    const float* bias;
    float* y;
    int32_t* acc_out;
    int64_t M, N, K, group;
} bitlinear_scaled_problem;

/* The BitLinear forward with one α per group: for each group b of row n the
 * exact integer sum acc_b = Σ_{k in b} x̃[m][k]·Ŵ[n][k], S = Σ_b α[n][b]·acc_b,
 * y[m][n] = RN32( RN32(S)·RN32(RN64(β_m/127)) ) (+ bias[n]).  With one α per
 * row S = α_n·acc is exact; with several, S is summed in binary64 (each term
 * exact), in an order that may differ from a sequential sum in the last bits
 * of binary64.  `problems` is a HOST array; flags: 0 or
 * BL_LINEAR_WEIGHTS_STATIC.  CUDA cores: with one α per row and at most four
 * tokens (K a multiple of 16, x_q 16-byte aligned) the streaming GEMV of
 * bitlinear_linear_grouped with the row's α in its epilogue (one launch when
 * it can quantise x itself); otherwise a GEMV that streams the weights once
 * per four tokens (this variant is not the tensor-core path).
 * Errors: as bitlinear_linear_grouped, plus BL_ERR_SHAPE for a bad group or
 * acc_out with several α per row. */
BITLINEAR_API bitlinear_status bitlinear_linear_scaled(const bitlinear_scaled_problem* problems, int count,
                                                       bitlinear_dtype dtype, uint32_t flags,
                                                       bitlinear_stream_t stream);

/* ---- 4-bit activations ("BitNet CPU 实测", cf-1.com/news/5800143 §2.1: later
 * variants quantise the activations to 4 bits instead of 8).  The absmax rule
 * of bitlinear_quantize_act with the signed 4-bit range: β_m = max|x| + 1e-8,
 * x̃ = clip(round((x·7)/β_m), -7, 7), the product and the quotient each
 * rounded to binary32, half to even.  Storage ("x_q4"): [M][ceil(K/2)] bytes,
 * element k in byte k/2, the low nibble for even k, two's complement; the
 * high nibble of the last byte of an odd-K row is 0.  Dequantisation:
 * y = fp32(acc)·RN32(RN64(α·β/7)) (+ bias), one α for the tensor. */
BITLINEAR_API bitlinear_status bitlinear_quantize_act_a4(const void* x, bitlinear_dtype dtype, int64_t M, int64_t K,
                                                         uint8_t* x_q4, float* beta, bitlinear_stream_t stream);

/* acc[m][n] = Σ_k x̃[m][k]·Ŵ[n][k] (exact int32) on 4-bit activations, then
 * y = RN32(fp32(acc)·RN32(RN64(α·β_m/7))) (+ bias[n], binary32 add).
 * Arguments as bitlinear_forward with x_q4 in place of x_q.  CUDA cores, four
 * tokens per pass (this variant is not the tensor-core path). */
BITLINEAR_API bitlinear_status bitlinear_forward_a4(const uint8_t* x_q4, const float* beta, int64_t M, int64_t K,
                                                    const uint8_t* W_packed, const float* alpha, int64_t N,
                                                    const float* bias, float* y, int32_t* acc_out,
                                                    bitlinear_stream_t stream);

/* bitlinear_quantize_act_a4 then bitlinear_forward_a4 on `count` problems (one
 * grouped launch each, chained by programmatic dependent launch); the x_q field
 * of each problem is its x_q4 buffer.  flags: 0 or BL_LINEAR_WEIGHTS_STATIC.
 * Errors: as bitlinear_linear_grouped. */
BITLINEAR_API bitlinear_status bitlinear_linear_a4(const bitlinear_linear_problem* problems, int count,
                                                   bitlinear_dtype dtype, uint32_t flags, bitlinear_stream_t stream);

/* ---- Training with the straight-through estimator ("1.58-bit 大模型极限量化
 * 实战", chenxutan.com/d/5049.html §3.3, §4.2 training branch, §6.3;
 * "1.58 位大模型" nxmr.cn/news/148658 §3.4): the layer keeps latent float
 * weights W, quantises them afresh in every forward, and the backward passes
 * the gradient straight through both quantisers, except that a weight outside
 * the clip range (|W/α| > 1) gets no gradient; α and β are constants to it. */

/* Training forward: bitlinear_quantize_weights of the latent W [N][K]
 * (w_dtype) into W_packed and alpha, then bitlinear_linear of x [M][K]
 * (x_dtype) into x_q, beta and y, all on `stream` (the outputs the backward
 * needs are kept).  workspace as for bitlinear_quantize_weights.
 * Errors: the union of both calls'. */
BITLINEAR_API bitlinear_status bitlinear_train_forward(const void* W, bitlinear_dtype w_dtype, int64_t N, int64_t K,
                                                       const void* x, bitlinear_dtype x_dtype, int64_t M,
                                                       uint8_t* W_packed, float* alpha, int8_t* x_q, float* beta,
                                                       float* y, void* workspace, size_t workspace_bytes,
                                                       bitlinear_stream_t stream);

/* Backward for g = ∂L/∂y [M][N] float32:
 *   grad_x[m][k] = α·Σ_n g[m][n]·Ŵ[n][k]
 *   grad_W[n][k] = |RN32(W[n][k]/α)| <= 1 ? Σ_m RN32(g[m][n]·s_m)·x̃[m][k] : 0,
 *                  s_m = RN32(RN64(β_m/127))
 * from the forward's W_packed, alpha, x_q, beta and the latent W (w_dtype).
 * Float32 arithmetic: each output summed by one thread in index order with
 * fused multiply-adds, rounded once (grad_x then times α); a float64 sum
 * differs by at most the float32 summation bound.  grad_x [M][K] and grad_W
 * [N][K] float32 are each nullable (not computed).  CUDA cores.
 * Errors: BL_ERR_NULL, BL_ERR_SHAPE, BL_ERR_ALIGN, BL_ERR_DTYPE, BL_ERR_ARCH,
 * BL_ERR_CUDA. */
BITLINEAR_API bitlinear_status bitlinear_ste_backward(const float* g, int64_t M, int64_t N, int64_t K,
                                                      const uint8_t* W_packed, const float* alpha, const int8_t* x_q,
                                                      const float* beta, const void* W, bitlinear_dtype w_dtype,
                                                      float* grad_x, float* grad_W, bitlinear_stream_t stream);

/* Reads and clears the current device's error word, which a kernel sets when
 * one of its bounded waits expires (it then stops early and its outputs are
 * undefined).  Synchronous: call after the streams that ran the kernels have
 * been synchronised.  *code receives 0 or a bitlinear_status code; returns
 * BL_OK, BL_ERR_NULL or BL_ERR_CUDA. */
BITLINEAR_API bitlinear_status bitlinear_device_error(int* code);

/* Self-test of the timeout path: launches one CTA that waits on an mbarrier
 * nothing ever completes, for at most `polls` polls, after which it sets the
 * device error word to BL_ERR_TIMEOUT and returns.  No other state changes. */
BITLINEAR_API bitlinear_status bitlinear_selftest_timeout(uint32_t polls, bitlinear_stream_t stream);

/* Static description of a status code. */
BITLINEAR_API const char* bitlinear_status_string(bitlinear_status status);

/* ABI version: 100·major + minor (1.02 added bitlinear_linear_grouped_host). */
BITLINEAR_API int bitlinear_version(void);

#ifdef __cplusplus
}
#endif
#endif /* BITLINEAR_H */

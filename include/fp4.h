/*
 * fp4.h -- C ABI of libfp4: the 4-bit linear layer of FP4 LLM pre-training on B200
 * (sm_100a).
 *
 *   x (bf16) --rotate(H16/H32, along the contraction axis)--> fp32
 *            --microscale (MXFP4 | NVFP4)--> packed E2M1 codes + block scales
 *   A, B (FP4) --block-scaled tcgen05 GEMM, fp32 accumulate--> C (fp32 | bf16)
 *
 * Pages this follows (cited by title and section):
 *   gist.science, "기술 요약: MXFP4 를 활용한 대규모 언어 모델 사전 학습" (summary of
 *   arXiv 2605.09825): "방법론" (Methodology) item 2 (Fprop, Dgrad and Wgrad each in
 *   MXFP4), item 3 (deterministic 16x16 / 32x32 Hadamard rotations); "주요 기여 및
 *   발견" (Findings) sections 1-2 (Wgrad dominates the instability; deterministic
 *   H16 restores it).
 *   molayo1419.me, "Blackwell의 NVIDIA NVFP4, MaxText에서 JAX 학습 속도 1.8배 향상":
 *   "주요 사실" (Key facts) bullets 2 and 5 (two 4-bit values per byte; FP4 tensor
 *   cores on Blackwell).
 *
 * Conventions for every entry point
 *   - All data pointers are DEVICE pointers owned by the caller, 16-byte aligned.
 *     The library never allocates, frees or retains device memory.
 *   - Calls are asynchronous and ordered on `stream` (a cudaStream_t; NULL = legacy
 *     default stream). Arguments are validated on the host before anything is
 *     launched: a call that returns an error launched nothing.
 *   - Device-side failures (a pipeline wait that exceeded its time limit) do not
 *     trap: the kernel records them in a device status word and returns; read it
 *     with fp4_check_status().
 *   - Results are deterministic: the same inputs give bit-identical outputs on every
 *     run (fixed butterfly order, order-independent max reductions, no split-K).
 *
 * Data formats
 *   codes  : uint8 [R][C/2]; element 2i in the low nibble of byte i, 2i+1 in the high
 *            nibble; nibble = sign << 3 | E2M1 magnitude index
 *            (0, 0.5, 1, 1.5, 2, 3, 4, 6).
 *   scales : one byte per block of bs elements along C (bs = 32 MXFP4, 16 NVFP4):
 *            MXFP4 E8M0 (value 2^(byte-127)), NVFP4 UE4M3 (OCP E4M3, sign 0).
 *            Scale (r, kb), KB = C/bs, is stored at byte
 *              ((r/128)*KB4 + kb/4)*512 + (r%32)*16 + ((r%128)/32)*4 + kb%4,
 *            KB4 = ceil(KB/4): 128-row x 4-block atoms of 512 bytes, the order the
 *            tensor cores read them in. Padding bytes are written as zero.
 *   NVFP4 tensor scale : fp32 S = amax / (6*448) of the rotated tensor (S = 1 when
 *            amax is 0). Element value = e2m1 * ue4m3(scale byte) * S.
 */
#ifndef FP4_H_
#define FP4_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FP4_API __attribute__((visibility("default")))
#else
#define FP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream, declared here without CUDA headers. */
typedef struct CUstream_st *fp4_stream_t;

typedef enum {
    FP4_OK = 0,
    FP4_ERR_INVALID_ARG = 1,        /* bad enum value, NULL pointer, or a pointer that must be NULL */
    FP4_ERR_SHAPE = 2,              /* a size the kernels do not tile (see each call) */
    FP4_ERR_ALIGN = 3,              /* a data pointer not 16-byte aligned */
    FP4_ERR_UNSUPPORTED_DEVICE = 4, /* current device is not compute capability 10.x */
    FP4_ERR_CUDA = 5,               /* a CUDA runtime/driver call failed */
    FP4_ERR_TIMEOUT = 6,            /* a device-side pipeline wait gave up (fp4_check_status) */
    FP4_ERR_WORKSPACE = 7,          /* workspace NULL or smaller than required */
    FP4_ERR_BOUNDS = 8              /* a device-side range check failed (debug build only,
                                       see fp4_check_status) */
} fp4_status;

/* FP4_MXFP8 is the FP8 comparator the pages measure FP4 against (MXFP4 pre-training
 * summary, Methodology item 1: the FP8 baseline; Findings section 3: MXFP4 + H16 20%
 * faster per step than FP8). Elements are E4M3 (one byte each, codes [R][C]); each
 * block of 32 shares an E8M0 scale, e = floor(log2 amax) - 8 clamped to [-127, 127]
 * (amax 0 -> -127), and codes are E4M3_RNE_satfinite(v * 2^-e). Its scales use the
 * same layout as MXFP4. It has no tensor scale and no quantiser variants (the options
 * of fp4_quantize_opts). The GEMM is tcgen05.mma kind::mxf8f6f4 with block32 scales. */
typedef enum { FP4_MXFP4 = 0, FP4_NVFP4 = 1, FP4_MXFP8 = 2 } fp4_format;
typedef enum { FP4_AXIS_ROW = 0, FP4_AXIS_COL = 1 } fp4_axis;
typedef enum { FP4_OUT_F32 = 0, FP4_OUT_BF16 = 1 } fp4_out_dtype;
typedef enum { FP4_PASS_FPROP = 0, FP4_PASS_DGRAD = 1, FP4_PASS_WGRAD = 2 } fp4_pass;

/* Version of this ABI; bumped on any incompatible change. */
FP4_API int fp4_abi_version(void);

/* Bytes of a packed code matrix with R rows of C elements: R*C/2 (two 4-bit codes per
 * byte: NVFP4/MaxText page, Key facts bullet 2). */
FP4_API size_t fp4_codes_bytes(int64_t rows, int64_t cols);
/* Bytes of a code matrix of format fmt: R*C/2 (FP4 formats) or R*C (FP4_MXFP8). */
FP4_API size_t fp4_codes_bytes_fmt(int64_t rows, int64_t cols, fp4_format fmt);

/* Bytes of the scale matrix of an [R][C] code matrix in the atom layout above:
 * ceil(R/128)*128 * ceil(C/bs/4)*4 (one shared scale per block of bs elements: the
 * block scales of the NVFP4/MaxText page's first paragraph and of MXFP4 in the
 * pre-training summary, Methodology item 2). */
FP4_API size_t fp4_scales_bytes(int64_t rows, int64_t cols, fp4_format fmt);

/*
 * fp4_quantize -- rotate and quantise one bf16 matrix x[rows][cols] (row-major).
 *   Rotation: every aligned group of hadamard_n (0 = none, 16, 32) elements along the
 *   contraction axis is replaced by H*v/sqrt(n) (Sylvester H, fp32 butterfly with
 *   strides 1, 2, 4, ... in that order; the factor 1/sqrt(n) is RN_fp32(1/sqrt(n))).
 *   [MXFP4 pre-training summary, Methodology item 3.]
 *   axis = FP4_AXIS_ROW : groups and blocks run along each row;
 *                         codes [rows][cols/2], scales for an [rows][cols] matrix.
 *   axis = FP4_AXIS_COL : groups and blocks run down each column, output transposed;
 *                         codes [cols][rows/2], scales for a [cols][rows] matrix.
 *   MXFP4: per 32-block, e = floor(log2 amax) - 2 clamped to [-127,127] (amax 0 -> -127),
 *          scale byte e+127, code = E2M1_RNE_satfinite(v * 2^-e).
 *   NVFP4: S = amax_tensor/2688; per 16-block sb = E4M3_RNE_satfinite(bmax/(6*S)),
 *          code = E2M1_RNE_satfinite(v / (ue4m3(sb)*S)).
 *   tensor_scale: NVFP4 -> device float[2], written {S, amax}; slot [1] is also the
 *                 reduction cell of the amax pass. MXFP4 -> must be NULL.
 *   Shape: rows % 32 == 0 and cols % 32 == 0 (rows or cols 0: nothing is done).
 *   Launches: MXFP4 one kernel; NVFP4 a 4-byte memset, an amax kernel, a quantise kernel.
 */
FP4_API fp4_status fp4_quantize(const void *x_bf16, void *codes, void *scales, float *tensor_scale,
                        int64_t rows, int64_t cols, fp4_format fmt, int hadamard_n,
                        fp4_axis axis, fp4_stream_t stream);

/*
 * fp4_quantize_dual -- both layouts of fp4_quantize from ONE read of x: the row-wise
 * result (row_codes, row_scales) and the column-wise transposed one (col_codes,
 * col_scales), bit-identical to two separate fp4_quantize calls. Each activation and
 * gradient of a training step is needed in both: along its rows for Fprop / Dgrad and
 * along the token axis for Wgrad, the pass the pre-training summary finds most
 * sensitive to quantisation (Methodology item 2; Findings section 1).
 *   tensor_scale: NVFP4 -> device float[4], written {S_row, S_col, amax_row, amax_col}
 *                 (each layout is scaled by the amax of its own rotation).
 *                 MXFP4 -> must be NULL.
 *   Shape: as fp4_quantize.
 */
FP4_API fp4_status fp4_quantize_dual(const void *x_bf16, void *row_codes, void *row_scales,
                             void *col_codes, void *col_scales, float *tensor_scale,
                             int64_t rows, int64_t cols, fp4_format fmt, int hadamard_n,
                             fp4_stream_t stream);

/*
 * fp4_quantize_dual_batch -- fp4_quantize_dual of n tensors of one format and rotation,
 * grouped into as few launches as possible (up to four tensors per launch; a tensor
 * whose column-layout codes exceed 256 MB goes alone). Each item is exactly one
 * fp4_quantize_dual call: the outputs are bit-identical. A training step quantises the
 * activation, the weight and the upstream gradient of every projection in both layouts
 * (pre-training summary, Methodology item 2); one launch for all of them pays the
 * launch's fixed costs (start-up, pipeline fill and drain, the last partial wave of
 * tiles) once instead of three times.
 *   items: host array of n descriptions (read during the call only); tensor_scale as
 *          for fp4_quantize_dual (NVFP4: device float[4]; MXFP4 / MXFP8: NULL).
 *   Every item is validated before anything is launched; errors as fp4_quantize_dual.
 *   NVFP4: one memset per item, then one amax launch and one quantise launch per group.
 */
typedef struct fp4_quant_item {
    const void *x_bf16;
    void *row_codes;
    void *row_scales;
    void *col_codes;
    void *col_scales;
    float *tensor_scale;
    int64_t rows;
    int64_t cols;
} fp4_quant_item;

FP4_API fp4_status fp4_quantize_dual_batch(const fp4_quant_item *items, int n, fp4_format fmt,
                                           int hadamard_n, fp4_stream_t stream);

/*
 * Quantiser variants. The MXFP4 pre-training summary ("방법론" item 3 and "주요 기여
 * 및 발견" section 2) names two stabilisers, stochastic rounding and randomised
 * Hadamard rotations, which it tests and finds do not stabilise the full MXFP4
 * pipeline. Neither is specified further there. These options implement the plainest
 * deterministic-per-seed reading of each, plus a caller-supplied NVFP4 tensor amax.
 *
 * Random words: word(seed, index, stream) is word index%4 of Philox4x32-10 (Salmon et
 * al., SC 2011) with counter (index/4 low 32 bits, index/4 high 32 bits, stream, 0)
 * and key (seed low 32 bits, seed high 32 bits).
 *
 *   amax        NVFP4 only: a DEVICE float[1] (single layout) or float[2] {row, col}
 *               (dual). It holds the tensor amax T of the rotated values of each
 *               layout, supplied by the caller (e.g. from an earlier step), so the
 *               amax pass is skipped. S = T/2688 as usual, and T is copied into the
 *               amax slot(s) of tensor_scale. NULL = computed as in fp4_quantize.
 *               It must be NULL for MXFP4 and 4-byte aligned.
 *   stochastic  nonzero: each code's magnitude is rounded stochastically instead
 *               of to nearest. |q| >= 6 gives 6. Otherwise, with lo the E2M1
 *               magnitude below |q| and step the gap to the next one, the magnitude
 *               rounds up iff (w >> 8) * 2^-24 < (|q| - lo) / step, where
 *               w = word(sr_seed, i*C + c, 1 + axis) for element (i, c) of the
 *               quantised [R][C] matrix (axis 0 = ROW, 1 = COL). Block scales are
 *               unchanged. The NVFP4 quotient is the exact IEEE one.
 *   random_signs nonzero: before the rotation, the element at index j along the
 *               contraction axis (column j of the quantised [R][C] matrix) is
 *               negated when bit 31 of word(sign_seed, j, 0) is set. Both operands
 *               of one GEMM must use the same sign_seed; the product is then
 *               unchanged, as for the plain rotation. The NVFP4 amax pass applies
 *               the same signs.
 *   sr_seed, sign_seed  the keys of the two variants.
 * A NULL options pointer, or all fields zero, gives exactly fp4_quantize /
 * fp4_quantize_dual. Errors: as fp4_quantize; FP4_ERR_INVALID_ARG for an amax with
 * MXFP4, FP4_ERR_ALIGN for a misaligned amax.
 */
typedef struct fp4_quant_opts {
    const float *amax;
    int stochastic;
    int random_signs;
    uint64_t sr_seed;
    uint64_t sign_seed;
} fp4_quant_opts;

FP4_API fp4_status fp4_quantize_opts(const void *x_bf16, void *codes, void *scales,
                             float *tensor_scale, int64_t rows, int64_t cols, fp4_format fmt,
                             int hadamard_n, fp4_axis axis, const fp4_quant_opts *opts,
                             fp4_stream_t stream);
FP4_API fp4_status fp4_quantize_dual_opts(const void *x_bf16, void *row_codes, void *row_scales,
                                  void *col_codes, void *col_scales, float *tensor_scale,
                                  int64_t rows, int64_t cols, fp4_format fmt, int hadamard_n,
                                  const fp4_quant_opts *opts, fp4_stream_t stream);

/*
 * fp4_gemm -- C[M][N] = deq(A)[M][K] * deq(B)[N][K]^T with fp32 accumulation on the
 * sm_100a block-scaled tensor cores (tcgen05.mma kind::mxf4 / kind::mxf4nvf4).
 * [MXFP4 pre-training summary, Methodology item 2; NVFP4/MaxText page, Key facts 5.]
 *   A_codes [M][K/2], A_scales (layout above, M rows); B likewise with N rows; both
 *   quantised along K (fp4_quantize ROW of an [M][K] / [N][K] matrix, or COL of the
 *   transposed one).
 *   A_tensor_scale, B_tensor_scale: NVFP4 -> device float* to S of each operand; the
 *   epilogue multiplies by S_A*S_B (fp32). MXFP4 -> must be NULL.
 *   C: row-major [M][N], fp32 or bf16 (round-to-nearest-even of the fp32 result).
 *   Shape: M, N, K multiples of 32 (0 -> nothing is done).
 */
FP4_API fp4_status fp4_gemm(const void *A_codes, const void *A_scales, const float *A_tensor_scale,
                    const void *B_codes, const void *B_scales, const float *B_tensor_scale,
                    void *C, int64_t M, int64_t N, int64_t K, fp4_format fmt,
                    fp4_out_dtype out_dtype, fp4_stream_t stream);

/*
 * fp4_gemm_group -- up to FP4_GEMM_GROUP_MAX independent fp4_gemm calls of one format in
 * one launch: e.g. the Fprop, Dgrad and Wgrad GEMMs of one linear layer [MXFP4
 * pre-training summary, Methodology item 2: all three passes in FP4]. The persistent
 * CTA pairs walk the tiles of all problems as one sequence, so the last, partly filled
 * wave of one GEMM is completed with tiles of the next. Each problem's output is
 * bit-identical to the same fp4_gemm call.
 *   descs[n]: host array (read during the call only), 1 <= n <= FP4_GEMM_GROUP_MAX; each
 *     entry as the arguments of fp4_gemm. Problems with M or N zero are skipped.
 *   The problems must not overlap one another's outputs; they run in order of
 *   decreasing K, concurrently.
 *   Errors: FP4_ERR_INVALID_ARG for n out of range or a NULL descs; otherwise the first
 *   error of any entry as fp4_gemm reports it, and nothing is launched.
 */
#define FP4_GEMM_GROUP_MAX 3
typedef struct fp4_gemm_desc {
  const void *A_codes;
  const void *A_scales;
  const float *A_tensor_scale;
  const void *B_codes;
  const void *B_scales;
  const float *B_tensor_scale;
  void *C;
  int64_t M, N, K;
  fp4_out_dtype out_dtype;
} fp4_gemm_desc;
FP4_API fp4_status fp4_gemm_group(const fp4_gemm_desc *descs, int n, fp4_format fmt,
                                  fp4_stream_t stream);

/*
 * fp4_gemm_quant -- fp4_gemm with a bf16 output whose epilogue also quantises it for
 * the next layer: Q = the row-wise MXFP4 quantisation, with rotation q_hadamard_n
 * (0, 16, 32) along N, of Y = RN_bf16(C) -- bit-identical to
 * fp4_quantize(Y, ..., FP4_MXFP4, q_hadamard_n, FP4_AXIS_ROW) of the stored Y, without
 * reading Y back from memory. [Producer-fused quantisation: the rotated FP4 operand of
 * the next GEMM comes out of the previous one, with custom kernels fusing the
 * quantisation into the training step (NVFP4/MaxText pages: the JAX/MaxText section
 * on fused low-precision kernels); MXFP4 + H16 as the pre-training summary, Methodology
 * items 2-3.]
 *   A, B, tensor scales, fmt (FP4_MXFP4 or FP4_NVFP4 operands), M, N, K: as fp4_gemm.
 *   C: bf16 [M][N] output, or NULL to write only the quantised output.
 *   Q_codes [M][N/2] and Q_scales (fp4_scales_bytes(M, N, FP4_MXFP4) bytes, the atom
 *   layout above, padding written as zero): device, 16-byte aligned.
 *   Errors: FP4_ERR_INVALID_ARG for FP4_MXFP8 operands, a NULL Q buffer or another
 *   q_hadamard_n; otherwise as fp4_gemm.
 */
FP4_API fp4_status fp4_gemm_quant(const void *A_codes, const void *A_scales,
                                  const float *A_tensor_scale, const void *B_codes,
                                  const void *B_scales, const float *B_tensor_scale, void *C,
                                  void *Q_codes, void *Q_scales, int64_t M, int64_t N, int64_t K,
                                  fp4_format fmt, int q_hadamard_n, fp4_stream_t stream);

/*
 * fp4_gemm_group_quant -- fp4_gemm_group in which member q_index also quantises its
 * output in the epilogue, as fp4_gemm_quant does: Q = the row-wise MXFP4 quantisation,
 * rotation q_hadamard_n (0, 16, 32) along N, of Y = RN_bf16(C). The other members
 * store as in fp4_gemm_group; all run in one launch. [Producer-fused quantisation, as
 * fp4_gemm_quant; the layer's three GEMMs in one launch, as fp4_gemm_group.]
 *   descs, n, fmt: as fp4_gemm_group; member q_index has out_dtype FP4_OUT_BF16 and C a
 *   bf16 [M][N] output or NULL (only Q is written).
 *   Q_codes [M][N/2], Q_scales (fp4_scales_bytes(M, N, FP4_MXFP4) bytes): as
 *   fp4_gemm_quant.
 *   Errors: FP4_ERR_INVALID_ARG for q_index outside [0, n), FP4_ERR_INVALID_ARG as
 *   fp4_gemm_quant for the quantised member; otherwise as fp4_gemm_group. A quantised
 *   member with M or N zero is skipped like any other.
 */
FP4_API fp4_status fp4_gemm_group_quant(const fp4_gemm_desc *descs, int n, fp4_format fmt,
                                        int q_index, void *Q_codes, void *Q_scales,
                                        int q_hadamard_n, fp4_stream_t stream);

/*
 * The three passes of a linear layer Y = X W^T with X [M][K], W [N][K], dY [M][N],
 * each quantising its operands along its own contraction axis and multiplying them.
 * [MXFP4 pre-training summary, Methodology item 2: Fprop, Dgrad, Wgrad.]
 *   fprop: Y [M][N]  = Q_row(X) . Q_row(W)^T                  (contraction over K)
 *   dgrad: dX [M][K] = Q_row(dY) . Q_col(W)^T  (W along N)    (contraction over N)
 *   wgrad: dW [N][K] = Q_col(dY) . Q_col(X)^T  (along tokens) (contraction over M)
 * ws / ws_bytes: caller-owned device scratch of at least fp4_linear_workspace_size()
 * bytes; it receives the quantised operands (and NVFP4 tensor scales) in an
 * unspecified layout. Shape: M, N, K multiples of 32.
 */
FP4_API size_t fp4_linear_workspace_size(fp4_pass pass, int64_t M, int64_t N, int64_t K, fp4_format fmt);

FP4_API fp4_status fp4_linear_fprop(const void *X, const void *W, void *Y, int64_t M, int64_t N, int64_t K,
                            fp4_format fmt, int hadamard_n, fp4_out_dtype out_dtype, void *ws,
                            size_t ws_bytes, fp4_stream_t stream);
FP4_API fp4_status fp4_linear_dgrad(const void *dY, const void *W, void *dX, int64_t M, int64_t N,
                            int64_t K, fp4_format fmt, int hadamard_n, fp4_out_dtype out_dtype,
                            void *ws, size_t ws_bytes, fp4_stream_t stream);
FP4_API fp4_status fp4_linear_wgrad(const void *dY, const void *X, void *dW, int64_t M, int64_t N,
                            int64_t K, fp4_format fmt, int hadamard_n, fp4_out_dtype out_dtype,
                            void *ws, size_t ws_bytes, fp4_stream_t stream);

/*
 * fp4_linear_step -- the three passes above in two launches: the dual-layout
 * quantisation of X, W and dY from one read of each (one batched launch, as
 * fp4_quantize_dual_batch) and Fprop, Dgrad and Wgrad in one grouped launch (as
 * fp4_gemm_group). [MXFP4 pre-training summary, Methodology item 2: all three passes
 * in FP4.]
 *   X bf16 [M][K], W bf16 [N][K], dY bf16 [M][N]: device inputs.
 *   Y bf16 [M][N], dX bf16 [M][K], dW fp32 [N][K]: device outputs, equal bit for bit to
 *   fp4_linear_fprop / _dgrad (bf16 out) and fp4_linear_wgrad (fp32 out).
 *   ws / ws_bytes: caller-owned device scratch of at least
 *   fp4_linear_step_workspace_size() bytes, 16-byte aligned; it receives both layouts
 *   of the three quantised tensors (and NVFP4 tensor scales) in an unspecified layout.
 *   Shape: M, N, K multiples of 32 and of the block and rotation sizes; M, N or K zero
 *   launches nothing.
 *   Errors: FP4_ERR_WORKSPACE for a NULL or small workspace; otherwise as the
 *   quantisation and GEMM calls it makes, checked before anything is launched.
 */
FP4_API size_t fp4_linear_step_workspace_size(int64_t M, int64_t N, int64_t K, fp4_format fmt);
FP4_API fp4_status fp4_linear_step(const void *X, const void *W, const void *dY, void *Y,
                                   void *dX, void *dW, int64_t M, int64_t N, int64_t K,
                                   fp4_format fmt, int hadamard_n, void *ws, size_t ws_bytes,
                                   fp4_stream_t stream);

/*
 * fp4_linear_fprop_noalloc -- fp4_linear_fprop with library-owned scratch instead
 * of a caller workspace. The pages have no counterpart to this call; it exists for
 * callers that cannot allocate device memory: code running inside a host framework
 * that has already reserved the GPU's memory for its own allocator, plug-ins and
 * callbacks that are handed tensors but no allocator, and latency-critical loops
 * that must not call cudaMalloc (which can synchronise the whole device).
 *   Scratch: one static device array of FP4_NOALLOC_SCRATCH_BYTES (32 MiB) per GPU,
 *   reserved when the library's device code is loaded on that GPU and held until the
 *   process exits. The call allocates and frees nothing.
 *   Limit: if fp4_linear_workspace_size(FP4_PASS_FPROP, M, N, K, fmt) exceeds
 *   FP4_NOALLOC_SCRATCH_BYTES the call returns FP4_ERR_WORKSPACE and launches nothing.
 *   Set-up: the first call on each device looks the array's device address up (with
 *   that device current) and caches it; make that first call before any stream
 *   capture begins.
 *   Sharing: every call on a device uses the same array, which keeps the previous
 *   call's contents; each call re-zeroes what must start at zero. Calls whose GPU work
 *   can overlap (for example on two streams with no ordering between them) race on
 *   the array: order them on one stream or with events.
 *   Arguments, shapes, outputs and the other errors are those of fp4_linear_fprop.
 */
#define FP4_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
FP4_API fp4_status fp4_linear_fprop_noalloc(const void *X, const void *W, void *Y, int64_t M,
                                            int64_t N, int64_t K, fp4_format fmt, int hadamard_n,
                                            fp4_out_dtype out_dtype, fp4_stream_t stream);

/*
 * fp4_check_status -- synchronises `stream`, then returns and clears the device
 * status word of the current device: FP4_ERR_BOUNDS if a range check of the debug
 * build failed, else FP4_ERR_TIMEOUT if any kernel's bounded wait gave up since the
 * last check, FP4_ERR_CUDA if the synchronisation failed, else FP4_OK.
 *   Debug build (libfp4_debug.so, compiled with -DFP4_DEBUG_BOUNDS): every kernel
 *   range-checks its computed shared-memory offsets, TMEM columns, tile coordinates
 *   and global indices before use; a failed check skips that access (no trap) and
 *   sets the bit reported here. Same ABI and results as the release library.
 */
FP4_API fp4_status fp4_check_status(fp4_stream_t stream);

/*
 * fp4_selftest_timeout -- launches one tiny kernel that waits on a pipeline barrier
 * nobody arrives at, using the same bounded wait as the GEMM and quantise kernels,
 * with a limit of timeout_ns nanoseconds. It gives up, records FP4_ERR_TIMEOUT in
 * the status word and returns normally; no fault, no trap. Used to test the
 * failure-reporting path.
 */
FP4_API fp4_status fp4_selftest_timeout(uint64_t timeout_ns, fp4_stream_t stream);

/* Static English text for a status code. */
FP4_API const char *fp4_status_string(fp4_status s);

#ifdef __cplusplus
}
#endif

#endif /* FP4_H_ */

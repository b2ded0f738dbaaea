/*
 * fp4_oracle.c -- plain, slow, scalar CPU oracle for the 4-bit linear-layer path:
 *   deterministic block Hadamard rotation (H16 / H32) along the contraction axis
 *   -> microscaled FP4 quantisation (MXFP4 or NVFP4, E2M1 codes, two per byte)
 *   -> block-scaled FP4 GEMM, evaluated here in fp64 on the dequantised operands.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg may load this file. It shares no code, header, table or
 * constant with the CUDA library: every encoder below is written from the
 * format definitions, not from the kernels.
 *
 * Sources (web pages; cited by title and section):
 *   [MXFP4-PT]  gist.science, "기술 요약: MXFP4 를 활용한 대규모 언어 모델 사전 학습"
 *               (summary of arXiv 2605.09825).
 *               - "방법론" (Methodology), item 2: Fprop, Dgrad and Wgrad are each run
 *                 in MXFP4.
 *               - "방법론", item 3: deterministic Hadamard rotations with 16x16 (H16)
 *                 and 32x32 (H32) matrices.
 *               - "주요 기여 및 발견" (Findings) section 2: deterministic H16 restores
 *                 stability of the full MXFP4 pipeline.
 *   [NVFP4-MT]  molayo1419.me, "Blackwell의 NVIDIA NVFP4, MaxText에서 JAX 학습 속도 1.8배
 *               향상": "주요 사실" (Key facts), 2nd bullet: two 4-bit values are packed
 *               into one 8-bit register; body, first paragraph: a shared exponent keeps
 *               the dynamic range.
 *   The pages name the formats but do not spell out their numerics. The format
 *   definitions used here are: MXFP4 = 32-element blocks sharing one power-of-two
 *   E8M0 scale taken from the block amax, E2M1 elements {0, +-0.5, +-1, +-1.5, +-2,
 *   +-3, +-4, +-6} with round-to-nearest-even; NVFP4 = 16-element blocks with an
 *   E4M3 block scale under an fp32 per-tensor scale amax / (6 * 448).
 *
 * Readings where the pages are silent (each is a choice, listed with the others
 * in the design notes of the repository):
 *   R1  Rotation: Sylvester Hadamard, applied to each aligned group of hn elements
 *       along the contraction axis as an in-place butterfly with strides
 *       h = 1, 2, 4, ..., hn/2 in that order, each sum and difference rounded to
 *       fp32, then every element multiplied by c_hn = RN_fp32(1/sqrt(hn)).
 *       The rotated values stay fp32.
 *   R2  MX scale exponent e = floor(log2(amax)) - 2 (2 = largest E2M1 exponent),
 *       clamped to [-127, 127]; amax == 0 gives e = -127. Scale byte = e + 127.
 *   R3  MX element: q = v * 2^-e (fp32), code = E2M1_RNE_satfinite(q).
 *   R4  E2M1 rounding: nearest of the 8 magnitudes, ties to the even code,
 *       magnitudes above 6 saturate to 6, the sign bit of q is kept even when
 *       the magnitude rounds to zero.
 *   R5  NVFP4: T = max|v| over the whole rotated tensor, S = T / 2688 (fp32; S = 1
 *       when T == 0); per 16-block t = B / (6 * S) (two fp32 roundings),
 *       sb = E4M3_RNE_satfinite(t); d = decode(sb) * S (fp32); q = v / d (fp32
 *       division); sb == 0 gives signed zero codes.
 *   R6  Packing: element 2i in the low nibble of byte i, element 2i+1 in the high
 *       nibble; nibble = sign << 3 | magnitude index.
 *   R7  Scale layout: scale (r, kb) of a matrix with KB = cols / bs blocks per row
 *       lives at byte ((r/128) * KB4 + kb/4) * 512 + (r%32) * 16 + ((r%128)/32) * 4
 *       + kb%4, KB4 = ceil(KB/4); rows are padded to a multiple of 128 and KB to a
 *       multiple of 4; padding bytes are zero.
 *   R8  Column-wise ("COL") quantisation of x[R][C] quantises x^T: codes [C][R/2],
 *       scales laid out for a [C][R/bs] scale matrix.
 *
 * Variants the pages test and reject as stabilisers ([MXFP4-PT] "방법론" item 3,
 * "주요 기여 및 발견" section 2: stochastic rounding and randomised Hadamard
 * rotations both fail to stabilise the full MXFP4 pipeline). The pages give no
 * numerics for either; the readings below are the plainest deterministic-per-seed
 * ones. Random words come from Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel
 * random numbers: as easy as 1, 2, 3", SC 2011), written here from that definition:
 *   word(seed, index, stream) = Philox4x32-10(counter = (index/4 low 32 bits,
 *   index/4 high 32 bits, stream, 0), key = (seed low, seed high))[index % 4].
 *   R12 Stochastic rounding (replaces R4's nearest rounding of the magnitude): for
 *       |q| >= 6 the magnitude is 6; otherwise lo = the largest E2M1 magnitude <= |q|,
 *       hi = the next one, and the magnitude is hi when (w >> 8) * 2^-24 <
 *       (|q| - lo) / (hi - lo), else lo (both sides exact in fp32), with
 *       w = word(seed, i * C + c, 1 + layout) for element (i, c) of the quantised
 *       [R][C] matrix, layout 0 = ROW, 1 = COL. The sign is kept as in R4. Block
 *       scales are those of R2 / R5 unchanged.
 *   R13 Randomised Hadamard: before R1, the element at index j along the contraction
 *       axis (column j of the quantised [R][C] matrix) is negated when bit 31 of
 *       word(seed, j, 0) is set. Both GEMM operands of a pass use the same seed, so
 *       (X D H)(W D H)^T = X W^T as for the deterministic rotation. The NVFP4 tensor
 *       amax is taken after this rotation.
 *   R14 Caller-supplied NVFP4 tensor amax: R5 with T given instead of computed.
 *
 * FP8 comparator. The pages measure FP4 against an FP8 baseline ([MXFP4-PT]
 * "방법론" item 1: full FP8 training is the baseline; "주요 기여 및 발견" section 3:
 * MXFP4 + H16 is 20% faster per step than FP8) without saying which FP8 recipe.
 *   R15 MXFP8 = the MX rule with E4M3 elements: per 32-block e = floor(log2 amax) - 8
 *       (8 = largest E4M3 exponent, 448 = 1.75 * 2^8), clamped to [-127, 127], amax 0
 *       gives -127; code = E4M3_RNE_satfinite(v * 2^-e), one byte per element, codes
 *       [R][C]; scales as R7. The optional rotation is R1.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define FP4O_MXFP4 0
#define FP4O_NVFP4 1
#define FP4O_MXFP8 2 /* the FP8 comparator: E4M3 elements, E8M0 scale per 32 */
#define FP4O_ROW 0
#define FP4O_COL 1

/* ---------------------------------------------------------------- bit helpers */

static float bits_to_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t f32_to_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* bf16 -> fp32 is exact: the bf16 pattern is the upper half of the fp32 pattern. */
float fp4o_bf16_to_f32(uint16_t b) { return bits_to_f32((uint32_t)b << 16); }

/* ---------------------------------------------------------------- E2M1 */

/* The eight E2M1 magnitudes indexed by the 3-bit magnitude field (exponent bias 1,
 * one mantissa bit, subnormal 0.5). */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double fp4o_e2m1_decode(uint8_t nibble) {
    double m = E2M1_MAG[nibble & 7];
    return (nibble & 8) ? -m : m;
}

/* R4. The thresholds are the midpoints between neighbouring magnitudes; a value
 * exactly on a midpoint goes to the neighbour with the even magnitude index
 * (index parity = mantissa bit), so "<=" is used where the lower neighbour is
 * even and "<" where the upper one is. */
uint8_t fp4o_e2m1_encode(float q) {
    uint8_t sign = (f32_to_bits(q) >> 31) ? 8 : 0;
    float a = fabsf(q);
    uint8_t idx;
    if (a <= 0.25f)      idx = 0;  /* midpoint 0.25 between 0 (idx 0) and 0.5 (idx 1) */
    else if (a < 0.75f)  idx = 1;  /* midpoint 0.75 between 0.5 (idx 1) and 1 (idx 2) */
    else if (a <= 1.25f) idx = 2;  /* midpoint 1.25 between 1 (idx 2) and 1.5 (idx 3) */
    else if (a < 1.75f)  idx = 3;  /* midpoint 1.75 between 1.5 (idx 3) and 2 (idx 4) */
    else if (a <= 2.5f)  idx = 4;  /* midpoint 2.5 between 2 (idx 4) and 3 (idx 5) */
    else if (a < 3.5f)   idx = 5;  /* midpoint 3.5 between 3 (idx 5) and 4 (idx 6) */
    else if (a <= 5.0f)  idx = 6;  /* midpoint 5 between 4 (idx 6) and 6 (idx 7) */
    else                 idx = 7;  /* everything above saturates to 6 */
    return (uint8_t)(sign | idx);
}

/* ---------------------------------------------------------------- Philox4x32-10 */

/* One Philox round: two 32x32 -> 64-bit products of the even counter words with the
 * round multipliers; the high halves are mixed with the odd words and the key. */
void fp4o_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; round++) {
        uint64_t p0 = (uint64_t)0xD2511F53u * c0;
        uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        c0 = hi1 ^ c1 ^ k0;
        c1 = lo1;
        c2 = hi0 ^ c3 ^ k1;
        c3 = lo0;
        k0 += 0x9E3779B9u; /* Weyl key schedule */
        k1 += 0xBB67AE85u;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* word(seed, index, stream) of R12/R13. */
uint32_t fp4o_philox_word(uint64_t seed, uint64_t index, uint32_t stream) {
    uint64_t blk = index / 4;
    uint32_t ctr[4] = {(uint32_t)blk, (uint32_t)(blk >> 32), stream, 0};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t out[4];
    fp4o_philox4x32_10(ctr, key, out);
    return out[index % 4];
}

/* R12: stochastic E2M1 rounding of q with random word w. */
uint8_t fp4o_e2m1_encode_sr(float q, uint32_t w) {
    static const float mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
    uint8_t sign = (f32_to_bits(q) >> 31) ? 8 : 0;
    float a = fabsf(q);
    int idx;
    if (a >= 6.0f) {
        idx = 7;
    } else {
        int lo = 0;
        while (lo < 6 && mag[lo + 1] <= a) lo++;
        float p = (a - mag[lo]) / (mag[lo + 1] - mag[lo]);
        float u = (float)(w >> 8) * 0x1p-24f;
        idx = u < p ? lo + 1 : lo;
    }
    return (uint8_t)(sign | idx);
}

/* R13: 1 when the element at contraction index j is negated. */
int fp4o_rht_negate(uint64_t seed, int64_t j) {
    return (int)(fp4o_philox_word(seed, (uint64_t)j, 0) >> 31);
}

/* ---------------------------------------------------------------- E8M0 */

/* R2. floor(log2(amax)) is read exactly with frexp: amax = f * 2^ex, f in [0.5, 1),
 * so floor(log2(amax)) = ex - 1, also for subnormal amax. */
int fp4o_mx_scale_exponent(float amax) {
    if (!(amax > 0.0f)) return -127;
    int ex;
    (void)frexpf(amax, &ex);
    int e = (ex - 1) - 2;
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e;
}

double fp4o_e8m0_decode(uint8_t b) { return ldexp(1.0, (int)b - 127); }

/* ---------------------------------------------------------------- E4M3 (OCP FP8) */

/* E4M3: exponent bias 7, 3 mantissa bits, subnormals k * 2^-9 (k = 1..7), largest
 * finite 448 (code 0x7E), code 0x7F is NaN, no infinity. */
double fp4o_e4m3_decode(uint8_t c) {
    int s = (c >> 7) & 1, E = (c >> 3) & 15, m = c & 7;
    double v;
    if (E == 15 && m == 7) return NAN;
    if (E == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, E - 7);
    return s ? -v : v;
}

/* Round to nearest even with saturation to +-448. The code of a finite magnitude
 * is 8 * (E + 7) + m for normal values and k for subnormal ones, which is one
 * monotone integer scale, so rounding the mantissa step count with nearbyint
 * (round-half-even in the default rounding mode) and letting a carry flow into
 * the exponent gives the RNE code directly; an even step count is an even code. */
uint8_t fp4o_e4m3_encode(float t) {
    uint8_t sign = (f32_to_bits(t) >> 31) ? 0x80 : 0;
    double a = fabs((double)t);
    if (isnan(t)) return 0x7F;
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    long code;
    if (a < ldexp(1.0, -6)) {
        code = (long)nearbyint(a * 512.0);                 /* steps of 2^-9 */
    } else {
        int ex;
        double f = frexp(a, &ex);                          /* a = f * 2^ex, f in [0.5,1) */
        int E = ex - 1;                                    /* a in [2^E, 2^(E+1)) */
        long m = (long)nearbyint((ldexp(f, 1) - 1.0) * 8.0); /* 0..8 */
        code = 8L * (E + 7) + m;
    }
    if (code > 0x7E) code = 0x7E;
    return (uint8_t)(sign | (uint8_t)code);
}

/* ---------------------------------------------------------------- rotation (R1) */

#define FP4O_C32_BITS 0x3E3504F3u /* RN_fp32(1/sqrt(32)) */

float fp4o_hadamard_scale(int n) {
    if (n == 16) return 0.25f;
    if (n == 32) return bits_to_f32(FP4O_C32_BITS);
    return (float)(1.0 / sqrt((double)n));
}

/* In-place normalised fast Walsh-Hadamard transform of one group of n (a power of
 * two) fp32 values, Sylvester (natural) order, strides 1, 2, 4, ... in that order. */
void fp4o_fwht_f32(float *v, int n) {
    for (int h = 1; h < n; h <<= 1) {
        for (int i = 0; i < n; i++) {
            if ((i & h) == 0) {
                float a = v[i], b = v[i + h];
                v[i] = a + b;
                v[i + h] = a - b;
            }
        }
    }
    float c = fp4o_hadamard_scale(n);
    for (int i = 0; i < n; i++) v[i] = v[i] * c;
}

/* Rotate a bf16 matrix along its contraction axis. For axis ROW the groups run along
 * each row of x[rows][cols] and out is [rows][cols]; for axis COL they run down each
 * column and out is the transpose, [cols][rows] (R8). hn == 0 only widens. */
int fp4o_rotate_opt(const uint16_t *x, int64_t rows, int64_t cols, int hn, int axis, int rht,
                    uint64_t rht_seed, float *out);

int fp4o_rotate(const uint16_t *x, int64_t rows, int64_t cols, int hn, int axis, float *out) {
    return fp4o_rotate_opt(x, rows, cols, hn, axis, 0, 0, out);
}

/* As fp4o_rotate; with rht != 0 the random signs of R13 are applied first. */
int fp4o_rotate_opt(const uint16_t *x, int64_t rows, int64_t cols, int hn, int axis, int rht,
                    uint64_t rht_seed, float *out) {
    int64_t R = axis == FP4O_ROW ? rows : cols, C = axis == FP4O_ROW ? cols : rows;
    if (hn != 0 && (C % hn) != 0) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; r++)
        for (int64_t c = 0; c < C; c++)
            out[r * C + c] = fp4o_bf16_to_f32(axis == FP4O_ROW ? x[r * cols + c] : x[c * cols + r]);
    if (rht) {
#pragma omp parallel for schedule(static)
        for (int64_t c = 0; c < C; c++)
            if (fp4o_rht_negate(rht_seed, c))
                for (int64_t r = 0; r < R; r++) out[r * C + c] = -out[r * C + c];
    }
    if (hn != 0) {
#pragma omp parallel for schedule(static)
        for (int64_t r = 0; r < R; r++)
            for (int64_t g = 0; g < C; g += hn) fp4o_fwht_f32(out + r * C + g, hn);
    }
    return 0;
}

/* max |v| over the rotated matrix (the NVFP4 tensor amax of step 3), one row of the
 * rotated matrix at a time. */
float fp4o_rotated_amax_opt(const uint16_t *x, int64_t rows, int64_t cols, int hn, int axis,
                            int rht, uint64_t rht_seed);

float fp4o_rotated_amax(const uint16_t *x, int64_t rows, int64_t cols, int hn, int axis) {
    return fp4o_rotated_amax_opt(x, rows, cols, hn, axis, 0, 0);
}

float fp4o_rotated_amax_opt(const uint16_t *x, int64_t rows, int64_t cols, int hn, int axis,
                            int rht, uint64_t rht_seed) {
    int64_t R = axis == FP4O_ROW ? rows : cols, C = axis == FP4O_ROW ? cols : rows;
    float *v = (float *)malloc(sizeof(float) * (size_t)(C > 0 ? C : 1));
    float T = 0.0f;
    for (int64_t r = 0; r < R; r++) {
        for (int64_t c = 0; c < C; c++) {
            v[c] = fp4o_bf16_to_f32(axis == FP4O_ROW ? x[r * cols + c] : x[c * cols + r]);
            if (rht && fp4o_rht_negate(rht_seed, c)) v[c] = -v[c];
        }
        if (hn != 0)
            for (int64_t g = 0; g < C; g += hn) fp4o_fwht_f32(v + g, hn);
        for (int64_t c = 0; c < C; c++) T = fmaxf(T, fabsf(v[c]));
    }
    free(v);
    return T;
}

/* ---------------------------------------------------------------- scale layout (R7) */

int64_t fp4o_scale_layout_bytes(int64_t rows, int64_t kblocks) {
    int64_t rp = (rows + 127) / 128 * 128, kp = (kblocks + 3) / 4 * 4;
    return rp * kp;
}

int64_t fp4o_scale_offset(int64_t r, int64_t kb, int64_t kblocks) {
    int64_t kb4 = (kblocks + 3) / 4;
    return ((r / 128) * kb4 + kb / 4) * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (kb % 4);
}

/* ---------------------------------------------------------------- block quantisers */

/* MX block (R2, R3): bs values -> bs codes (one per byte, unpacked) and one E8M0 byte. */
/* w: NULL for nearest rounding (R4), else one random word per element (R12). */
static uint8_t encode_q(float q, const uint32_t *w, int i) {
    return w ? fp4o_e2m1_encode_sr(q, w[i]) : fp4o_e2m1_encode(q);
}

static void quantize_block_mx_w(const float *v, int bs, const uint32_t *w, uint8_t *codes,
                                uint8_t *scale_byte) {
    float amax = 0.0f;
    for (int i = 0; i < bs; i++) amax = fmaxf(amax, fabsf(v[i]));
    int e = fp4o_mx_scale_exponent(amax);
    float inv = (float)ldexp(1.0, -e); /* 2^-e, exact in fp32 for e in [-127, 127] */
    for (int i = 0; i < bs; i++) codes[i] = encode_q(v[i] * inv, w, i);
    *scale_byte = (uint8_t)(e + 127);
}

void fp4o_quantize_block_mx(const float *v, int bs, uint8_t *codes, uint8_t *scale_byte) {
    quantize_block_mx_w(v, bs, NULL, codes, scale_byte);
}

/* NV tensor scale (R5). */
float fp4o_nv_tensor_scale(float tensor_amax) {
    if (!(tensor_amax > 0.0f)) return 1.0f;
    return tensor_amax / 2688.0f;
}

/* NV block (R5): bs values -> bs codes and one UE4M3 byte, under tensor scale S. */
static void quantize_block_nv_w(const float *v, int bs, float S, const uint32_t *w,
                                uint8_t *codes, uint8_t *scale_byte) {
    float bmax = 0.0f;
    for (int i = 0; i < bs; i++) bmax = fmaxf(bmax, fabsf(v[i]));
    float six_s = 6.0f * S;
    float t = bmax / six_s;
    uint8_t sb = fp4o_e4m3_encode(t);
    float d = (float)fp4o_e4m3_decode(sb) * S; /* decode is exact in fp32; one rounding */
    for (int i = 0; i < bs; i++) {
        if (sb == 0) codes[i] = (f32_to_bits(v[i]) >> 31) ? 8 : 0;
        else codes[i] = encode_q(v[i] / d, w, i);
    }
    *scale_byte = sb;
}

void fp4o_quantize_block_nv(const float *v, int bs, float S, uint8_t *codes, uint8_t *scale_byte) {
    quantize_block_nv_w(v, bs, S, NULL, codes, scale_byte);
}

/* ---------------------------------------------------------------- tensor quantiser */

/* Quantise x[rows][cols] (bf16 bit patterns) along `axis`.
 *   codes:  [R][C/2] bytes, R x C = rows x cols (ROW) or cols x rows (COL)
 *   scales: fp4o_scale_layout_bytes(R, C/bs) bytes, written in layout R7
 *   nv_scale_out / nv_amax_out: NVFP4 only (may be NULL otherwise)
 * Returns 0, or -1 on a shape the format cannot block. */
int fp4o_quantize_ex(const uint16_t *x, int64_t rows, int64_t cols, int fmt, int hn, int axis,
                     const float *amax_in, uint8_t *codes, uint8_t *scales, float *nv_scale_out,
                     float *nv_amax_out);

int fp4o_quantize(const uint16_t *x, int64_t rows, int64_t cols, int fmt, int hn, int axis,
                  uint8_t *codes, uint8_t *scales, float *nv_scale_out, float *nv_amax_out) {
    return fp4o_quantize_ex(x, rows, cols, fmt, hn, axis, NULL, codes, scales, nv_scale_out,
                            nv_amax_out);
}

/* As fp4o_quantize; for NVFP4 a non-NULL amax_in supplies the tensor amax T of step 3
 * (the amax of the whole rotated tensor, when x is a slice of it: rows of a ROW
 * quantisation or columns of a COL one are quantised independently given T). */
int fp4o_quantize_opt(const uint16_t *x, int64_t rows, int64_t cols, int fmt, int hn, int axis,
                      const float *amax_in, int sr, uint64_t sr_seed, int rht, uint64_t rht_seed,
                      uint8_t *codes, uint8_t *scales, float *nv_scale_out, float *nv_amax_out);

int fp4o_quantize_ex(const uint16_t *x, int64_t rows, int64_t cols, int fmt, int hn, int axis,
                     const float *amax_in, uint8_t *codes, uint8_t *scales, float *nv_scale_out,
                     float *nv_amax_out) {
    return fp4o_quantize_opt(x, rows, cols, fmt, hn, axis, amax_in, 0, 0, 0, 0, codes, scales,
                             nv_scale_out, nv_amax_out);
}

/* As fp4o_quantize_ex, with the variants: sr != 0 rounds the codes stochastically
 * (R12, words keyed by sr_seed), rht != 0 applies the random signs of R13 (keyed by
 * rht_seed) before the rotation. */
int fp4o_quantize_opt(const uint16_t *x, int64_t rows, int64_t cols, int fmt, int hn, int axis,
                      const float *amax_in, int sr, uint64_t sr_seed, int rht, uint64_t rht_seed,
                      uint8_t *codes, uint8_t *scales, float *nv_scale_out, float *nv_amax_out) {
    int bs = fmt == FP4O_MXFP4 ? 32 : 16;
    int64_t R = axis == FP4O_ROW ? rows : cols, C = axis == FP4O_ROW ? cols : rows;
    if (C % bs != 0 || (hn != 0 && C % hn != 0) || C % 2 != 0) return -1;
    int64_t KB = C / bs;
    float *v = (float *)malloc(sizeof(float) * (size_t)(R * C > 0 ? R * C : 1));
    if (!v) return -2;
    /* steps 1-2: widen, rotate */
    fp4o_rotate_opt(x, rows, cols, hn, axis, rht, rht_seed, v);
    /* step 3 (NVFP4 only): tensor amax of the rotated values and the tensor scale */
    float S = 1.0f;
    if (fmt == FP4O_NVFP4) {
        float T = 0.0f;
        if (amax_in) {
            T = *amax_in;
        } else {
            /* a max is exact and order independent, so splitting it changes nothing */
#pragma omp parallel for schedule(static) reduction(max : T)
            for (int64_t i = 0; i < R * C; i++) T = fmaxf(T, fabsf(v[i]));
        }
        S = fp4o_nv_tensor_scale(T);
        if (nv_scale_out) *nv_scale_out = S;
        if (nv_amax_out) *nv_amax_out = T;
    }
    /* steps 4-5: block scales and codes; step 6: pack */
    memset(scales, 0, (size_t)fp4o_scale_layout_bytes(R, KB));
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; r++) {
        uint8_t blk[32];
        uint32_t w[32];
        for (int64_t kb = 0; kb < KB; kb++) {
            const float *bv = v + r * C + kb * bs;
            if (sr)
                for (int i = 0; i < bs; i++)
                    w[i] = fp4o_philox_word(sr_seed, (uint64_t)(r * C + kb * bs + i),
                                            1u + (uint32_t)axis);
            uint8_t sb;
            if (fmt == FP4O_MXFP4) quantize_block_mx_w(bv, bs, sr ? w : NULL, blk, &sb);
            else quantize_block_nv_w(bv, bs, S, sr ? w : NULL, blk, &sb);
            scales[fp4o_scale_offset(r, kb, KB)] = sb;
            for (int i = 0; i < bs; i += 2)
                codes[r * (C / 2) + (kb * bs + i) / 2] = (uint8_t)(blk[i] | (blk[i + 1] << 4));
        }
    }
    free(v);
    return 0;
}

/* R15: MXFP8 quantisation of x[rows][cols] along `axis`; codes [R][C] bytes. */
int fp4o_quantize_mxfp8(const uint16_t *x, int64_t rows, int64_t cols, int hn, int axis,
                        uint8_t *codes, uint8_t *scales) {
    int64_t R = axis == FP4O_ROW ? rows : cols, C = axis == FP4O_ROW ? cols : rows;
    if (C % 32 != 0 || (hn != 0 && C % hn != 0)) return -1;
    int64_t KB = C / 32;
    float *v = (float *)malloc(sizeof(float) * (size_t)(R * C > 0 ? R * C : 1));
    if (!v) return -2;
    fp4o_rotate(x, rows, cols, hn, axis, v);
    memset(scales, 0, (size_t)fp4o_scale_layout_bytes(R, KB));
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; r++) {
        for (int64_t kb = 0; kb < KB; kb++) {
            const float *bv = v + r * C + kb * 32;
            float amax = 0.0f;
            for (int i = 0; i < 32; i++) amax = fmaxf(amax, fabsf(bv[i]));
            int e = -127;
            if (amax > 0.0f) {
                int ex;
                frexp(amax, &ex);              /* amax = f * 2^ex, f in [0.5, 1) */
                e = ex - 1 - 8;
                if (e < -127) e = -127;
                if (e > 127) e = 127;
            }
            float inv = (float)ldexp(1.0, -e);
            for (int i = 0; i < 32; i++) codes[r * C + kb * 32 + i] = fp4o_e4m3_encode(bv[i] * inv);
            scales[fp4o_scale_offset(r, kb, KB)] = (uint8_t)(e + 127);
        }
    }
    free(v);
    return 0;
}

/* ---------------------------------------------------------------- dequantisation */

/* Value of element (r, c) of a quantised [R][C] matrix, exactly, in fp64. */
static double deq_elem(const uint8_t *codes, const uint8_t *scales, double S, int64_t C, int fmt,
                       int64_t r, int64_t c) {
    if (fmt == FP4O_MXFP8)
        return fp4o_e4m3_decode(codes[r * C + c]) *
               fp4o_e8m0_decode(scales[fp4o_scale_offset(r, c / 32, C / 32)]);
    int bs = fmt == FP4O_MXFP4 ? 32 : 16;
    int64_t KB = C / bs;
    uint8_t byte = codes[r * (C / 2) + c / 2];
    uint8_t nib = (c & 1) ? (byte >> 4) : (byte & 15);
    uint8_t sb = scales[fp4o_scale_offset(r, c / bs, KB)];
    double q = fp4o_e2m1_decode(nib);
    if (fmt == FP4O_MXFP4) return q * fp4o_e8m0_decode(sb);
    return q * fp4o_e4m3_decode(sb) * S;
}

void fp4o_dequantize(const uint8_t *codes, const uint8_t *scales, float tensor_scale, int64_t R,
                     int64_t C, int fmt, double *out) {
    double S = fmt == FP4O_NVFP4 ? (double)tensor_scale : 1.0;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; r++)
        for (int64_t c = 0; c < C; c++) out[r * C + c] = deq_elem(codes, scales, S, C, fmt, r, c);
}

/* ---------------------------------------------------------------- GEMM */

/* C[m][n] = sum_k A[m][k] * B[n][k] in fp64 (both operands K-major). */
void fp4o_gemm_f64(const double *A, const double *B, double *Cm, int64_t M, int64_t N, int64_t K) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; m++)
        for (int64_t n = 0; n < N; n++) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; k++) acc += A[m * K + k] * B[n * K + k];
            Cm[m * N + n] = acc;
        }
}

/* Selected entries of the block-scaled GEMM C = deq(A) * deq(B)^T, computed from the
 * quantised operands directly (A is [M][K], B is [N][K], both quantised along K). */
void fp4o_gemm_entries(const uint8_t *a_codes, const uint8_t *a_scales, float a_ts,
                       const uint8_t *b_codes, const uint8_t *b_scales, float b_ts, int64_t K,
                       int fmt, const int64_t *ms, const int64_t *ns, int64_t count, double *out) {
    double SA = fmt == FP4O_NVFP4 ? (double)a_ts : 1.0;
    double SB = fmt == FP4O_NVFP4 ? (double)b_ts : 1.0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < count; i++) {
        double acc = 0.0;
        for (int64_t k = 0; k < K; k++)
            acc += deq_elem(a_codes, a_scales, SA, K, fmt, ms[i], k) *
                   deq_elem(b_codes, b_scales, SB, K, fmt, ns[i], k);
        out[i] = acc;
    }
}

/* ---------------------------------------------------------------- array helpers */

void fp4o_e2m1_encode_array(const float *q, uint8_t *out, int64_t n) {
    for (int64_t i = 0; i < n; i++) out[i] = fp4o_e2m1_encode(q[i]);
}

void fp4o_e4m3_encode_array(const float *t, uint8_t *out, int64_t n) {
    for (int64_t i = 0; i < n; i++) out[i] = fp4o_e4m3_encode(t[i]);
}

void fp4o_mx_scale_exponent_array(const float *a, int32_t *out, int64_t n) {
    for (int64_t i = 0; i < n; i++) out[i] = fp4o_mx_scale_exponent(a[i]);
}

/* ---------------------------------------------------------------- threads */

/* Threads of the OpenMP build (the same source compiled with -fopenmp; the pragmas
 * above split independent rows, columns or entries and never a rounding step).
 * n > 0 sets the count; returns the count in use (1 in the serial build). */
int fp4o_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

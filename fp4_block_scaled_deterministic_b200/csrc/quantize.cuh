// quantize.cuh -- fused rotate + microscale-quantise kernel (and the NVFP4 amax pass).
//
// What it computes (gist.science summary of arXiv 2605.09825, Methodology items 2-3;
// molayo1419.me NVFP4/MaxText page, Key facts bullet 2):
//   x bf16 -> fp32 -> block Hadamard rotation of every aligned group of HN (0/16/32)
//   elements along the contraction axis (Sylvester H, butterfly strides 1,2,4,...,
//   each sum/difference rounded to fp32, then x RN_fp32(1/sqrt(HN)))
//   -> per block (32 MXFP4 / 16 NVFP4): scale from the block amax, E2M1 RNE codes,
//   two per byte (element 2i in the low nibble), scales in 128-row x 4-block atoms.
//   ROW: blocks run along rows, codes [R][C/2]. COL: blocks run down columns and the
//   output is transposed, codes [C][R/2] (the token-axis layout Wgrad needs).
//   DUAL: both from one read of x.
//
// Structure (two CTAs per SM, persistent): the input is cut into 128x128 bf16 tiles;
// a 2-stage TMA pipeline per CTA brings each tile into shared memory as two
// 128B-swizzled boxes of 128 rows x 64 columns. 256 threads then work from shared
// memory in jobs of two 32-element vectors held lane-wise in float2 registers:
//   ROW job = one row, 64 consecutive columns (two segments; 8 conflict-free 16-B reads);
//   COL job = two adjacent columns, 32 consecutive rows (32 conflict-free 4-B reads);
// the rotation runs in registers with packed fp32x2 arithmetic (its first stage fused
// into the bf16 widening), codes are staged in a 64B-swizzled [128][64 B] tile and
// written by a TMA store, scale atoms are assembled in shared memory (1-, 2- and 4-byte
// stores) and written by bulk copies. Staging is double-buffered so stores overlap the
// next tile.
//
// With H16 the rotation's x0.25 is a power of two and is applied per block, not per
// element, wherever that is exact: MXFP4 folds it into the E8M0 exponent, and the
// plain NVFP4 kernel into the block amax and the divisor (nv_block_x2, kQuarter).
//
// Also here: the MXFP8 comparator (E4M3 codes, one byte each, 128-byte code tiles,
// one CTA per SM); the EXT instances with the quantiser variants (random Hadamard
// signs, Philox-driven stochastic rounding); the BANDED instances, whose tile order
// suits tensors with very large column-layout outputs.
#pragma once

#include "common.cuh"

namespace fp4k {

enum { kModeRow = 1, kModeCol = 2, kModeDual = 3 };

constexpr int kQThreads = 256;
// Input pipeline depth and CTAs per SM: two tiles in flight per CTA, two CTAs per SM
// (one for MXFP8, whose 128-byte code tiles take more shared memory). One tile in
// flight at three CTAs per SM (70 KB each) was measured 6% slower for MXFP4.
__host__ __device__ constexpr int kQStagesOf(int fmt, bool ext) { return 2; }
constexpr int kQBoxBytes = 128 * 64 * 2;    // 128 rows x 64 bf16
constexpr int kQInBytes = 2 * kQBoxBytes;   // a 128 x 128 bf16 tile
constexpr int kQScaleBytes = 1024;          // up to two 512-byte atoms
// Staged code tile: 128 rows x 64 code bytes (FP4, 64B swizzle) or x 128 bytes (MXFP8,
// 128B swizzle). With the larger MXFP8 staging one CTA fits per SM.
__host__ __device__ constexpr int kQCodeBytesOf(int fmt) { return fmt == kFmtMX8 ? 128 * 128 : 128 * 64; }
__host__ __device__ constexpr int kQSmemBytesOf(int fmt, bool ext) {
  return 1024 /*align*/ + kQStagesOf(fmt, ext) * kQInBytes + 2 * 2 * kQCodeBytesOf(fmt) +
         2 * 2 * kQScaleBytes + 256 + 2048 /* random-sign masks, two tiles */;
}
__host__ __device__ constexpr int kQCtasPerSMOf(int fmt, bool ext) {
  return fmt == kFmtMX8 ? 1 : 2;
}

struct QuantArgs {
  int64_t rows, cols;
  int tiles_c, tiles_r, num_tiles;
  int band_c;  // tile order: see qtile_coords
  uint8_t* row_scales;   // ROW layout scales (scale matrix [rows][cols/bs])
  uint8_t* col_scales;   // COL layout scales (scale matrix [cols][rows/bs])
  int row_kb4, col_kb4;  // 512-byte atoms per 128-row block of each layout
  const float* amax_row; // NVFP4 quantise pass: tensor amax of each rotation
  const float* amax_col;
  float* s_row_out;      // NVFP4 quantise pass: tensor scales, written by CTA 0
  float* s_col_out;
  unsigned* amax_row_acc;  // NVFP4 amax pass: accumulators (bits of a non-negative float)
  unsigned* amax_col_acc;
  float* amax_row_copy;  // NVFP4 with a caller-supplied amax: CTA 0 copies it here
  float* amax_col_copy;
  int sr, rht;           // variant kernels: stochastic rounding, randomised Hadamard signs
  uint32_t sr_key[2], sign_key[2];
  uint64_t wait_limit_ns;
};

// One launch quantises up to kQMaxItems tensors (e.g. the X, W and dY of one projection
// of a training step), so that the launch's fixed costs -- start-up, pipeline fill,
// drain and the last partial wave of tiles -- are paid once. Tiles are numbered one
// tensor after the other (tensor k's first tile is tile0); each tensor has its own TMA
// maps and arguments. A single-tensor call is a batch of one.
constexpr int kQMaxItems = 4;
struct QuantItem {
  CUtensorMap in, rcodes, ccodes;
  QuantArgs a;
  int tile0;
};
struct QuantBatch {
  QuantItem item[kQMaxItems];
  int n, num_tiles;
};
// Tensor of global tile `tile`. NITEMS (a kernel template argument) is 1 for
// single-tensor launches, whose code then indexes item 0 at compile time.
template <int NITEMS>
__device__ __forceinline__ int batch_item(const QuantBatch& qb, int tile) {
  if constexpr (NITEMS == 1) return 0;
  int k = 0;
#pragma unroll
  for (int j = 1; j < NITEMS; ++j) k += (j < qb.n && tile >= qb.item[j].tile0) ? 1 : 0;
  return k;
}
// NVFP4 tensor scales of every tensor of the batch into s_S[2k] (row) and s_S[2k+1]
// (column layout): S = amax / 2688 (1 when amax is 0); CTA 0 also publishes them (and
// copies a caller-supplied amax). Thread 0 of each CTA calls this before its first barrier.
template <bool kRow, bool kCol, int NITEMS>
__device__ __forceinline__ void batch_tensor_scales(const QuantBatch& qb, float* s_S, bool publish) {
  const int n = NITEMS == 1 ? 1 : qb.n;
  for (int k = 0; k < n; ++k) {
    const QuantArgs& a = qb.item[k].a;
    float S_r = 1.0f, S_c = 1.0f;
    if constexpr (kRow) {
      const float T = *a.amax_row;
      S_r = T > 0.0f ? __fdiv_rn(T, 2688.0f) : 1.0f;
    }
    if constexpr (kCol) {
      const float T = *a.amax_col;
      S_c = T > 0.0f ? __fdiv_rn(T, 2688.0f) : 1.0f;
    }
    s_S[2 * k] = S_r;
    s_S[2 * k + 1] = S_c;
    if (publish) {
      if constexpr (kRow) *a.s_row_out = S_r;
      if constexpr (kCol) *a.s_col_out = S_c;
      if constexpr (kRow) if (a.amax_row_copy) *a.amax_row_copy = *a.amax_row;
      if constexpr (kCol) if (a.amax_col_copy) *a.amax_col_copy = *a.amax_col;
    }
  }
}

// Every unit of work ("job") is two independent 32-element vectors held lane-wise in
// float2 registers (.x = first vector, .y = second), so the butterflies, scalings and
// quotients use the packed fp32x2 instructions; each lane is rounded exactly as the
// scalar operation would be.
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  return __fadd2_rn(a, make_float2(-b.x, -b.y));  // a - b == a + (-b), same rounding
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 neg2(float2 a) { return make_float2(-a.x, -a.y); }

// Normalised block FWHT of both lanes: groups of HN along the 32 elements, butterfly
// strides 1, 2, 4, ... in that order, then x RN(1/sqrt(HN)).
template <int HN, bool kScale = true, int kFirst = 1>
__device__ __forceinline__ void fwht_x2(float2 (&p)[32]) {
  if constexpr (HN > 0) {
#pragma unroll
    for (int h = kFirst; h < HN; h <<= 1) {
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        if ((i & h) == 0) {
          const float2 a = p[i], b = p[i + h];
          p[i] = add2(a, b);
          p[i + h] = sub2(a, b);
        }
      }
    }
    // 0.25 = 1/sqrt(16) exactly; 0x3E3504F3 = fp32 nearest to 1/sqrt(32)
    if constexpr (kScale) {
      const float c = (HN == 16) ? 0.25f : __uint_as_float(0x3E3504F3u);
      const float2 c2 = make_float2(c, c);
#pragma unroll
      for (int i = 0; i < 32; ++i) p[i] = mul2(p[i], c2);
    }
  }
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// Max of N non-negative floats as a tree of three-input maxes (depth ~log3 N instead of
// a chain of N/2 dependent instructions; max is exact, so the order does not matter).
template <int N>
__device__ __forceinline__ float tree_max(const float* v) {
  if constexpr (N == 1) {
    return v[0];
  } else if constexpr (N == 2) {
    return fmaxf(v[0], v[1]);
  } else {
    constexpr int G = (N + 2) / 3;  // groups of three (the last may be shorter)
    float m[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      if (3 * g + 2 < N) m[g] = max3f(v[3 * g], v[3 * g + 1], v[3 * g + 2]);
      else if (3 * g + 1 < N) m[g] = fmaxf(v[3 * g], v[3 * g + 1]);
      else m[g] = v[3 * g];
    }
    return tree_max<G>(m);
  }
}
// max |x| over elements [B, B+N) of each lane.
template <int B, int N, int L>
__device__ __forceinline__ float2 amax_x2(const float2 (&p)[L]) {
  float ax[N], ay[N];
#pragma unroll
  for (int i = 0; i < N; ++i) {
    ax[i] = fabsf(p[B + i].x);
    ay[i] = fabsf(p[B + i].y);
  }
  return make_float2(tree_max<N>(ax), tree_max<N>(ay));
}

__device__ __forceinline__ uint32_t cvt8x(const float2 (&p)[32], int b) {
  const float v[8] = {p[b].x, p[b + 1].x, p[b + 2].x, p[b + 3].x,
                      p[b + 4].x, p[b + 5].x, p[b + 6].x, p[b + 7].x};
  return cvt_e2m1x8(v);
}
__device__ __forceinline__ uint32_t cvt8y(const float2 (&p)[32], int b) {
  const float v[8] = {p[b].y, p[b + 1].y, p[b + 2].y, p[b + 3].y,
                      p[b + 4].y, p[b + 5].y, p[b + 6].y, p[b + 7].y};
  return cvt_e2m1x8(v);
}

// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as 1, 2,
// 3", SC 2011): ten rounds of two 32x32->64-bit products mixed with the other counter
// words and the key, the key advanced by the two Weyl increments after each round.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    // one 32x32 -> 64-bit product each (both halves from one wide multiply)
    const uint64_t p0 = static_cast<uint64_t>(0xD2511F53u) * c.x;
    const uint64_t p1 = static_cast<uint64_t>(0xCD9E8D57u) * c.z;
    const uint32_t lo0 = static_cast<uint32_t>(p0), hi0 = static_cast<uint32_t>(p0 >> 32);
    const uint32_t lo1 = static_cast<uint32_t>(p1), hi1 = static_cast<uint32_t>(p1 >> 32);
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return c;
}
// The four random words of Philox block `blk` (elements 4*blk .. 4*blk+3) of a stream.
__device__ __forceinline__ uint4 philox_block(uint64_t blk, uint32_t stream, const uint32_t (&key)[2]) {
  return philox4x32_10(make_uint4(static_cast<uint32_t>(blk), static_cast<uint32_t>(blk >> 32),
                                  stream, 0u),
                       key[0], key[1]);
}

// Stochastic E2M1 rounding of q with random word w: |q| >= 6 gives 6; otherwise the
// magnitude rounds up from the E2M1 value lo below |q| to the next one with probability
// p = (|q| - lo) / step, taken as (w >> 8) * 2^-24 < p. |q| - lo is exact (lo >= |q|/2
// or lo = 0) and step is a power of two, so p is exact; the sign is kept.
__device__ __forceinline__ uint32_t e2m1_sr(float q, uint32_t w) {
  const float a = fabsf(q);
  uint32_t lo;
  float base, inv_step;
  if (a < 2.0f) {
    lo = static_cast<uint32_t>(a * 2.0f);  // 0, 0.5, 1, 1.5
    base = static_cast<float>(lo) * 0.5f;
    inv_step = 2.0f;
  } else if (a < 4.0f) {
    const float f = floorf(a);             // 2, 3
    lo = static_cast<uint32_t>(f) + 2u;
    base = f;
    inv_step = 1.0f;
  } else {
    lo = 6u;                               // 4
    base = 4.0f;
    inv_step = 0.5f;
  }
  const float pr = __fmul_rn(__fsub_rn(a, base), inv_step);
  const float u = static_cast<float>(w >> 8) * 0x1p-24f;
  const uint32_t idx = a >= 6.0f ? 7u : lo + (u < pr ? 1u : 0u);
  return ((__float_as_uint(q) >> 31) << 3) | idx;
}

// Conversion of a job's quotients (two lanes of 32) to packed codes.
struct RneCodes {
  static constexpr bool kExactQuotient = false;
  __device__ __forceinline__ void operator()(const float2 (&p)[32], uint4& cx, uint4& cy) const {
    cx = make_uint4(cvt8x(p, 0), cvt8x(p, 8), cvt8x(p, 16), cvt8x(p, 24));
    cy = make_uint4(cvt8y(p, 0), cvt8y(p, 8), cvt8y(p, 16), cvt8y(p, 24));
  }
};
// Stochastic rounding: element i of lane x (y) draws word i of the lane's run of Philox
// blocks starting at blk_x (blk_y). The quotient must be the exact one.
struct SrCodes {
  static constexpr bool kExactQuotient = true;
  uint64_t blk_x, blk_y;
  uint32_t stream;
  const uint32_t* key;
  __device__ __forceinline__ void operator()(const float2 (&p)[32], uint4& cx, uint4& cy) const {
    uint32_t wx[8], wy[8];
    const uint32_t k[2] = {key[0], key[1]};
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      const uint4 rx = philox_block(blk_x + g, stream, k);
      const uint4 ry = philox_block(blk_y + g, stream, k);
      const uint32_t ux[4] = {rx.x, rx.y, rx.z, rx.w}, uy[4] = {ry.x, ry.y, ry.z, ry.w};
      uint32_t bx = 0, by = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        bx |= e2m1_sr(p[4 * g + j].x, ux[j]) << (4 * j);
        by |= e2m1_sr(p[4 * g + j].y, uy[j]) << (4 * j);
      }
      wx[g] = bx;
      wy[g] = by;
    }
    cx = make_uint4(wx[0] | (wx[1] << 16), wx[2] | (wx[3] << 16), wx[4] | (wx[5] << 16),
                    wx[6] | (wx[7] << 16));
    cy = make_uint4(wy[0] | (wy[1] << 16), wy[2] | (wy[3] << 16), wy[4] | (wy[5] << 16),
                    wy[6] | (wy[7] << 16));
  }
};

// Encoded job: 16 code bytes per lane and its scale bytes (MXFP4: byte 0; NVFP4: bytes
// 0 and 1 for the two 16-element blocks).
struct Enc {
  uint4 cx, cy;
  uint32_t sx, sy;  // scale bytes, lowest byte first
};

// MXFP4 block of 32 per lane: byte = max(biased exponent of amax - 2, 0), i.e. the byte of
// e = floor(log2 amax) - 2 clamped at -127 (zero and subnormal amax give 0); codes of
// v * 2^-e, 2^-e = 2^(127 - byte) built from its bit pattern (byte <= 252).
template <class Codes = RneCodes>
__device__ __forceinline__ Enc mx_encode_x2(float2 (&p)[32], const Codes& codes = Codes()) {
  const float2 am = amax_x2<0, 32>(p);
  const uint32_t ex = (__float_as_uint(am.x) >> 23) & 0xFFu;
  const uint32_t ey = (__float_as_uint(am.y) >> 23) & 0xFFu;
  const uint32_t bx = ex > 2u ? ex - 2u : 0u, by = ey > 2u ? ey - 2u : 0u;
  const float2 inv = make_float2(__uint_as_float((254u - bx) << 23), __uint_as_float((254u - by) << 23));
#pragma unroll
  for (int i = 0; i < 32; ++i) p[i] = mul2(p[i], inv);
  Enc e;
  codes(p, e.cx, e.cy);
  e.sx = bx;
  e.sy = by;
  return e;
}

// MXFP4 after an H16 butterfly whose final x0.25 has NOT been applied: the exact x0.25 is
// folded into the power-of-two scale, q = v * 2^(-e-2), with e taken from amax*0.25
// (byte = biased exponent of amax - 4). This equals the two-step RN(RN(v*0.25) * 2^-e)
// whenever the block amax is >= 2^-100: v*0.25 is then exact unless |v| < 2^-124, and
// such an element lands below 2^-20 either way (code 0, sign kept). Smaller blocks
// take the two-step path.
template <class Codes = RneCodes>
__device__ __forceinline__ Enc mx_encode_x2_h16fold(float2 (&p)[32], const Codes& codes = Codes()) {
  const float2 am = amax_x2<0, 32>(p);
  if (am.x >= 0x1p-100f && am.y >= 0x1p-100f) {
    const uint32_t bx = ((__float_as_uint(am.x) >> 23) & 0xFFu) - 4u;
    const uint32_t by = ((__float_as_uint(am.y) >> 23) & 0xFFu) - 4u;
    const float2 inv = make_float2(__uint_as_float((252u - bx) << 23), __uint_as_float((252u - by) << 23));
#pragma unroll
    for (int i = 0; i < 32; ++i) p[i] = mul2(p[i], inv);
    Enc e;
    codes(p, e.cx, e.cy);
    e.sx = bx;
    e.sy = by;
    return e;
  }
  const float2 q = make_float2(0.25f, 0.25f);
#pragma unroll
  for (int i = 0; i < 32; ++i) p[i] = mul2(p[i], q);
  return mx_encode_x2(p, codes);
}

// NVFP4 block of 16 per lane under tensor scale S (six_s = 6*S, rounded once):
// byte = UE4M3_RNE_satfinite(bmax / six_s), d = ue4m3(byte) * S, codes of the fp32
// quotient RN(v / d); a zero byte gives signed zeros.
// The quotient comes from y = RN(1/d) by two FMA correction steps: q0 = RN(v*y), which
// can be just over one ulp from v/d; q1 = RN(q0 + RN(v - q0*d)*y), which is faithful;
// then, with the residual r = v - q1*d exact as one FMA, q = RN(q1 + r*y) is the
// correctly rounded quotient RN(v/d) (the last step is Markstein's, "Computation of
// elementary functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1),
// 1990; Muller et al., Handbook of Floating-Point Arithmetic, the FMA-based division
// section). That needs d and the reciprocal away from underflow and overflow: with
// 2^-100 <= d <= 2^100 a residual can underflow only when |v/d| < 2^-3, whose code is a
// signed zero either way. The residual is formed negated, n = RN(q*d - v), and each step
// adds (-n)*y: round-to-nearest is odd, so every nonzero value is the one above, and the
// zero sums that can arise keep v's sign (-0 / d stays -0) with no sign copy. Blocks
// with a zero scale, a d outside that range or a non-finite element are divided exactly.
//
// kQuarter: p holds w = 4v, the H16 butterflies without their x0.25. Round-to-nearest
// is monotonic and odd, so the block amax of v is RN(amax|w| / 4), one multiply per
// block. Where v = w/4 exactly (|w| >= 2^-124), v/d = w/(4d) with 4d exact, so the
// quotient is taken from w and d' = 4d, in the same range check: the same number
// wherever the sequence is exact, and below 2^-3 a signed zero code either way.
// Smaller elements have |v/d| and |w/d'| below 2^-22 (d' >= 2^-100): both encode as
// the signed zero of w's sign. Blocks off the fast path scale by 0.25 first and go on
// exactly as before.
template <int b, bool kExact = false, int L = 32, bool kQuarter = false>
__device__ __forceinline__ void nv_block_x2(float2 (&p)[L], float S, float six_s,
                                            uint32_t& sbx, uint32_t& sby) {
  float2 bm = amax_x2<b, 16>(p);
  if constexpr (kQuarter) bm = make_float2(__fmul_rn(bm.x, 0.25f), __fmul_rn(bm.y, 0.25f));
  sbx = cvt_e4m3(__fdiv_rn(bm.x, six_s));
  sby = cvt_e4m3(__fdiv_rn(bm.y, six_s));
  const float dx = __fmul_rn(e4m3_to_f32(sbx), S), dy = __fmul_rn(e4m3_to_f32(sby), S);
  // the divisor of the values held: d, or 4d for kQuarter (exact, or infinite and so
  // off the fast path)
  const float ex = kQuarter ? __fmul_rn(dx, 4.0f) : dx;
  const float ey = kQuarter ? __fmul_rn(dy, 4.0f) : dy;
  const bool fast = !kExact && ex >= 0x1p-100f && ey >= 0x1p-100f && ex <= 0x1p100f &&
                    ey <= 0x1p100f && bm.x <= 3.0e38f && bm.y <= 3.0e38f;
  if (fast) {
    const float2 y2 = make_float2(__frcp_rn(ex), __frcp_rn(ey));
    const float2 e2 = make_float2(ex, ey);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float2 v = p[b + i];
      const float2 q0 = mul2(v, y2);
      const float2 q1 = __ffma2_rn(neg2(__ffma2_rn(q0, e2, neg2(v))), y2, q0);  // faithful
      p[b + i] = __ffma2_rn(neg2(__ffma2_rn(q1, e2, neg2(v))), y2, q1);           // RN(v/d)
    }
    return;
  }
  // A zero block scale gives zeros that keep the sign of the element itself (the
  // quotient by d = 0 is an infinity, or a NaN for a zero element).
  const bool zx = sbx == 0u, zy = sby == 0u;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float2 v = kQuarter ? mul2(p[b + i], make_float2(0.25f, 0.25f)) : p[b + i];
    p[b + i] = make_float2(zx ? __uint_as_float(__float_as_uint(v.x) & 0x80000000u)
                              : __fdiv_rn(v.x, dx),
                           zy ? __uint_as_float(__float_as_uint(v.y) & 0x80000000u)
                              : __fdiv_rn(v.y, dy));
  }
}

// (Stochastic rounding needs the exact quotient, not only its side of each threshold.)
template <class Codes = RneCodes>
__device__ __forceinline__ Enc nv_encode_x2(float2 (&p)[32], float S, float six_s,
                                            const Codes& codes = Codes()) {
  uint32_t x0, y0, x1, y1;
  nv_block_x2<0, Codes::kExactQuotient>(p, S, six_s, x0, y0);
  nv_block_x2<16, Codes::kExactQuotient>(p, S, six_s, x1, y1);
  Enc e;
  codes(p, e.cx, e.cy);
  e.sx = x0 | (x1 << 8);
  e.sy = y0 | (y1 << 8);
  return e;
}

template <int FMT, bool kFold, class Codes = RneCodes>
__device__ __forceinline__ Enc encode_x2(float2 (&p)[32], float S, float six_s,
                                         const Codes& codes = Codes()) {
  if constexpr (FMT == kFmtMX && kFold) return mx_encode_x2_h16fold(p, codes);
  else if constexpr (FMT == kFmtMX) return mx_encode_x2(p, codes);
  else return nv_encode_x2(p, S, six_s, codes);
}

// Four fp32 -> E4M3 (RNE, saturating to +-448) in one word, v0 in the low byte.
__device__ __forceinline__ uint32_t cvt_e4m3x4(float v0, float v1, float v2, float v3) {
  uint32_t out;
  asm("{\n\t.reg .b16 lo, hi;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
      "mov.b32 %0, {lo, hi};\n\t}"
      : "=r"(out)
      : "f"(v0), "f"(v1), "f"(v2), "f"(v3));
  return out;
}

// MXFP8 job: 32 E4M3 code bytes per lane (two 16-byte chunks) and one scale byte.
struct Enc8 {
  uint4 cx[2], cy[2];
  uint32_t sx, sy;
};
// MXFP8 block of 32 per lane: byte = max(biased exponent of amax - 8, 0), i.e. the byte of
// e = floor(log2 amax) - 8 clamped at -127 (8 = largest E4M3 exponent); codes
// E4M3_RNE_satfinite(v * 2^-e), 2^-e = 2^(127 - byte) built from its bit pattern.
__device__ __forceinline__ Enc8 mx8_encode_x2(float2 (&p)[32]) {
  const float2 am = amax_x2<0, 32>(p);
  const uint32_t ex = (__float_as_uint(am.x) >> 23) & 0xFFu;
  const uint32_t ey = (__float_as_uint(am.y) >> 23) & 0xFFu;
  const uint32_t bx = ex > 8u ? ex - 8u : 0u, by = ey > 8u ? ey - 8u : 0u;
  const float2 inv = make_float2(__uint_as_float((254u - bx) << 23), __uint_as_float((254u - by) << 23));
#pragma unroll
  for (int i = 0; i < 32; ++i) p[i] = mul2(p[i], inv);
  uint32_t wx[8], wy[8];
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    wx[g] = cvt_e4m3x4(p[4 * g].x, p[4 * g + 1].x, p[4 * g + 2].x, p[4 * g + 3].x);
    wy[g] = cvt_e4m3x4(p[4 * g].y, p[4 * g + 1].y, p[4 * g + 2].y, p[4 * g + 3].y);
  }
  Enc8 e;
  e.cx[0] = make_uint4(wx[0], wx[1], wx[2], wx[3]);
  e.cx[1] = make_uint4(wx[4], wx[5], wx[6], wx[7]);
  e.cy[0] = make_uint4(wy[0], wy[1], wy[2], wy[3]);
  e.cy[1] = make_uint4(wy[4], wy[5], wy[6], wy[7]);
  e.sx = bx;
  e.sy = by;
  return e;
}

// Offset of scale (row r of the 128-row atom block, block kb of the tile) in a staged
// scale tile of one or two atoms: atom kb/4, then (r%32)*16 + (r/32)*4 + kb%4.
__device__ __forceinline__ int atom_off(int r, int kb) {
  return (kb >> 2) * 512 + (r & 31) * 16 + (r >> 5) * 4 + (kb & 3);
}
// Staged code tile [128 rows][64 B], 64-byte swizzle: 16-byte chunk q of row r.
__device__ __forceinline__ uint8_t* code_chunk(uint8_t* tile, int r, int q) {
  return tile + r * 64 + ((q ^ ((r >> 1) & 3)) << 4);
}
// Staged MXFP8 code tile [128 rows][128 B], 128-byte swizzle: 16-byte chunk q of row r.
__device__ __forceinline__ uint8_t* code_chunk8(uint8_t* tile, int r, int q) {
  return tile + r * 128 + ((q ^ (r & 7)) << 4);
}
// Debug-build range checks of the offsets into the staged tiles (always true otherwise):
// 16-byte code chunk q of tile row r (nq chunks per row), `bytes` scale bytes at
// atom_off(r, kb), and the base of a ROW job (row r of box b) or a COL job (column pair
// w of box b, rows 32s .. 32s+31) of the input tile.
__device__ __forceinline__ bool code_ok(int r, int q, int nq) {
  return FP4_IN_BOUNDS(r >= 0 && r < 128 && q >= 0 && q < nq);
}
__device__ __forceinline__ bool scale_ok(int r, int kb, int bytes) {
  return FP4_IN_BOUNDS(r >= 0 && r < 128 && kb >= 0 && atom_off(r, kb) + bytes <= kQScaleBytes);
}
__device__ __forceinline__ bool row_job_ok(int r, int b) {
  return FP4_IN_BOUNDS(r >= 0 && r < 128 && b >= 0 && b * kQBoxBytes + r * 128 + 128 <= kQInBytes);
}
__device__ __forceinline__ bool col_job_ok(int b, int w, int s) {
  return FP4_IN_BOUNDS(b >= 0 && b < 2 && w >= 0 && w < 32 && s >= 0 && s < 4);
}

// ROW job: tile row r, box b (columns 64b .. 64b+63) = segments 2b (lane x) and 2b+1
// (lane y); 8 conflict-free 16-byte reads of the 128B-swizzled box row.
// Random signs as XOR masks on the raw bf16x2 words: cm[q] flips the two columns of
// column pair q of the tile (bits 15 and 31), rm[r] both halves of tile row r.
__device__ __forceinline__ uint4 xor4(uint4 a, uint4 m) {
  return make_uint4(a.x ^ m.x, a.y ^ m.y, a.z ^ m.z, a.w ^ m.w);
}

template <bool kSigns = false>
__device__ __forceinline__ void load_row_job(const uint8_t* in, int r, int b, float2 (&p)[32],
                                             const uint32_t* cm = nullptr) {
  if (!row_job_ok(r, b)) {
#pragma unroll
    for (int i = 0; i < 32; ++i) p[i] = make_float2(0.0f, 0.0f);
    return;
  }
  const uint8_t* rowp = in + b * kQBoxBytes + r * 128;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 wx = *reinterpret_cast<const uint4*>(rowp + ((i ^ (r & 7)) << 4));
    uint4 wy = *reinterpret_cast<const uint4*>(rowp + (((4 + i) ^ (r & 7)) << 4));
    if constexpr (kSigns) {  // pairs 32b + 4i .. (lane x) and 32b + 16 + 4i .. (lane y)
      wx = xor4(wx, *reinterpret_cast<const uint4*>(cm + 32 * b + 4 * i));
      wy = xor4(wy, *reinterpret_cast<const uint4*>(cm + 32 * b + 16 + 4 * i));
    }
    p[8 * i + 0] = make_float2(bf16lo(wx.x), bf16lo(wy.x));
    p[8 * i + 1] = make_float2(bf16hi(wx.x), bf16hi(wy.x));
    p[8 * i + 2] = make_float2(bf16lo(wx.y), bf16lo(wy.y));
    p[8 * i + 3] = make_float2(bf16hi(wx.y), bf16hi(wy.y));
    p[8 * i + 4] = make_float2(bf16lo(wx.z), bf16lo(wy.z));
    p[8 * i + 5] = make_float2(bf16hi(wx.z), bf16hi(wy.z));
    p[8 * i + 6] = make_float2(bf16lo(wx.w), bf16lo(wy.w));
    p[8 * i + 7] = make_float2(bf16hi(wx.w), bf16hi(wy.w));
  }
}
// COL job: tile columns c = 64b + 2w (lane x) and c + 1 (lane y), rows 32s .. 32s+31;
// 32 conflict-free 4-byte reads.
template <bool kSigns = false>
__device__ __forceinline__ void load_col_job(const uint8_t* in, int b, int w, int s,
                                             float2 (&p)[32], const uint32_t* rm = nullptr) {
  if (!col_job_ok(b, w, s)) {
#pragma unroll
    for (int i = 0; i < 32; ++i) p[i] = make_float2(0.0f, 0.0f);
    return;
  }
  const uint8_t* boxp = in + b * kQBoxBytes;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int r = 32 * s + i;
    uint32_t v = *reinterpret_cast<const uint32_t*>(boxp + r * 128 +
                                                    (((w >> 2) ^ (r & 7)) << 4) + ((w & 3) << 2));
    if constexpr (kSigns) v ^= rm[r];
    p[i] = make_float2(bf16lo(v), bf16hi(v));
  }
}

// bf16 (low or high half of w) + c in fp32 with one rounding; the widening is exact, so
// this is RN_fp32(widen(bf16) + c), the stride-1 butterfly of the rotation, issued on
// the FMA pipe instead of widening on the integer pipe first.
__device__ __forceinline__ float add_lo(uint32_t w, float c) {
  float d;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tadd.rn.f32.bf16 %0, l, %2;\n\t}"
      : "=f"(d) : "r"(w), "f"(c));
  return d;
}
__device__ __forceinline__ float add_hi(uint32_t w, float c) {
  float d;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tadd.rn.f32.bf16 %0, h, %2;\n\t}"
      : "=f"(d) : "r"(w), "f"(c));
  return d;
}
// Stride-1 butterfly of two bf16 values u (element 2k) and v (element 2k+1) given as
// the bf16 u and the widened v: (u + v, u - v), each rounded once.
__device__ __forceinline__ void bfly1_lo(uint32_t wu, float v, float& s, float& d) {
  s = add_lo(wu, v);
  d = add_lo(wu, -v);
}
__device__ __forceinline__ void bfly1_hi(uint32_t wu, float v, float& s, float& d) {
  s = add_hi(wu, v);
  d = add_hi(wu, -v);
}

// ROW job with the first (stride-1) butterfly fused into the widening: elements 2k and
// 2k+1 of a lane are the low and high halves of one 32-bit word.
template <bool kSigns = false>
__device__ __forceinline__ void load_row_job_bfly1(const uint8_t* in, int r, int b,
                                                   float2 (&p)[32], const uint32_t* cm = nullptr) {
  if (!row_job_ok(r, b)) {
#pragma unroll
    for (int i = 0; i < 32; ++i) p[i] = make_float2(0.0f, 0.0f);
    return;
  }
  const uint8_t* rowp = in + b * kQBoxBytes + r * 128;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 wx = *reinterpret_cast<const uint4*>(rowp + ((i ^ (r & 7)) << 4));
    uint4 wy = *reinterpret_cast<const uint4*>(rowp + (((4 + i) ^ (r & 7)) << 4));
    if constexpr (kSigns) {
      wx = xor4(wx, *reinterpret_cast<const uint4*>(cm + 32 * b + 4 * i));
      wy = xor4(wy, *reinterpret_cast<const uint4*>(cm + 32 * b + 16 + 4 * i));
    }
    const uint32_t ax[4] = {wx.x, wx.y, wx.z, wx.w}, ay[4] = {wy.x, wy.y, wy.z, wy.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float sx, dx, sy, dy;
      bfly1_lo(ax[k], add_hi(ax[k], -0.0f), sx, dx);  // x + (-0) widens exactly
      bfly1_lo(ay[k], add_hi(ay[k], -0.0f), sy, dy);
      p[8 * i + 2 * k] = make_float2(sx, sy);
      p[8 * i + 2 * k + 1] = make_float2(dx, dy);
    }
  }
}
// COL job with the first butterfly fused: elements i and i+1 are consecutive rows, lane x
// the low halves (column c) and lane y the high halves (column c+1) of the two words.
template <bool kSigns = false>
__device__ __forceinline__ void load_col_job_bfly1(const uint8_t* in, int b, int w, int s,
                                                   float2 (&p)[32], const uint32_t* rm = nullptr) {
  if (!col_job_ok(b, w, s)) {
#pragma unroll
    for (int i = 0; i < 32; ++i) p[i] = make_float2(0.0f, 0.0f);
    return;
  }
  const uint8_t* boxp = in + b * kQBoxBytes;
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    const int r0 = 32 * s + i, r1 = r0 + 1;
    uint32_t v0 = *reinterpret_cast<const uint32_t*>(boxp + r0 * 128 +
                                                     (((w >> 2) ^ (r0 & 7)) << 4) + ((w & 3) << 2));
    uint32_t v1 = *reinterpret_cast<const uint32_t*>(boxp + r1 * 128 +
                                                     (((w >> 2) ^ (r1 & 7)) << 4) + ((w & 3) << 2));
    if constexpr (kSigns) {
      v0 ^= rm[r0];
      v1 ^= rm[r1];
    }
    float sx, dx, sy, dy;
    bfly1_lo(v0, add_lo(v1, -0.0f), sx, dx);
    bfly1_hi(v0, add_hi(v1, -0.0f), sy, dy);
    p[i] = make_float2(sx, sy);
    p[i + 1] = make_float2(dx, dy);
  }
}

// Tile order. Row-major (tile column fastest) keeps the input rows of the tiles in
// flight long and sequential, which is best while the column-layout (transposed)
// codes, written 64 bytes per output row per tile, can still be merged in L2. For
// tensors whose column-layout codes far exceed L2 the host launches the BANDED kernels:
// bands of a.band_c tile columns (32; 16 for the MXFP4 column layout alone) with the
// tile column fastest inside a band. With 32, the tiles in flight cover about nine tile
// rows of one band, and each column-layout row receives a 576-byte run instead of
// scattered 64-byte pieces.
template <bool BANDED>
__device__ __forceinline__ void qtile_coords(int tile, const QuantArgs& a, int& tr, int& tc) {
  if constexpr (!BANDED) {
    tr = tile / a.tiles_c;
    tc = tile - tr * a.tiles_c;
    return;
  }
  const int first = tile / (a.band_c * a.tiles_r) * a.band_c;
  const int width = min(a.band_c, a.tiles_c - first);
  const int r = tile - first * a.tiles_r;
  tc = first + r % width;
  tr = r / width;
}

// EXT kernels also implement the variants selected at run time by a.rht (random +-1
// signs along the contraction axis before the rotation) and a.sr (stochastic rounding).
template <int FMT, int HN, int MODE, bool AMAX, bool EXT = false, bool BANDED = false,
          int NITEMS = 1>
__global__ void __launch_bounds__(kQThreads, kQCtasPerSMOf(FMT, EXT))
    quantize_kernel(const __grid_constant__ QuantBatch qb) {
  constexpr bool kRow = (MODE & kModeRow) != 0;
  constexpr bool kCol = (MODE & kModeCol) != 0;
  // MXFP4 + H16 quantise pass: the rotation's x0.25 is folded into the block scale
  constexpr bool kFoldH16 = FMT == kFmtMX && HN == 16 && !AMAX;
  // variants come one tensor per launch
  const bool rht = EXT && qb.item[0].a.rht != 0, sr = EXT && qb.item[0].a.sr != 0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* s_in = smem;
  constexpr int kQStages = kQStagesOf(FMT, EXT);
  uint8_t* s_rcode = s_in + kQStages * kQInBytes;
  constexpr int kCodeBytes = kQCodeBytesOf(FMT);
  uint8_t* s_ccode = s_rcode + 2 * kCodeBytes;
  uint8_t* s_rsc = s_ccode + 2 * kCodeBytes;
  uint8_t* s_csc = s_rsc + 2 * kQScaleBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(s_csc + 2 * kQScaleBytes);
  // per-tensor amax accumulators of the amax pass (bits of non-negative floats) and
  // NVFP4 tensor scales {row, col} of the batch's tensors
  unsigned* s_amax = reinterpret_cast<unsigned*>(full + kQStages);  // [kQMaxItems][2]
  float* s_S = reinterpret_cast<float*>(s_amax + 2 * kQMaxItems);   // [kQMaxItems][2]
  // random-sign XOR masks of a tile, double-buffered by tile parity: 64 column-pair
  // words (ROW jobs) and 128 row words (COL jobs) per buffer; 16-byte aligned
  uint32_t* s_masks = reinterpret_cast<uint32_t*>(
      (reinterpret_cast<uintptr_t>(s_S + 2 * kQMaxItems) + 15) & ~static_cast<uintptr_t>(15));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bid = blockIdx.x, nctas = gridDim.x;
  const int my_tiles = bid < qb.num_tiles ? (qb.num_tiles - bid + nctas - 1) / nctas : 0;

  // Signs of a tile's 128 columns (warp 0) and 128 rows (warp 1) into mask buffer `buf`:
  // Philox block (tile start)/4 + lane holds the words of indices 4*lane .. 4*lane+3.
  auto write_masks = [&](int tile, int buf) {
    const QuantItem& I = qb.item[batch_item<NITEMS>(qb, tile)];
    const QuantArgs& a = I.a;
    int tr, tc;
    qtile_coords<BANDED>(tile - I.tile0, a, tr, tc);
    uint32_t* cm = s_masks + 192 * buf;
    if (kRow && warp == 0) {
      const uint4 w = philox_block(static_cast<uint64_t>(tc) * 32u + lane, 0u, a.sign_key);
      // column pairs 2*lane (columns 4*lane, +1) and 2*lane+1 (columns 4*lane+2, +3)
      *reinterpret_cast<uint2*>(cm + 2 * lane) =
          make_uint2(((w.x >> 31) << 15) | (w.y & 0x80000000u),
                     ((w.z >> 31) << 15) | (w.w & 0x80000000u));
    }
    if (kCol && warp == 1) {
      const uint4 w = philox_block(static_cast<uint64_t>(tr) * 32u + lane, 0u, a.sign_key);
      *reinterpret_cast<uint4*>(cm + 64 + 4 * lane) =
          make_uint4((w.x >> 31) * 0x80008000u, (w.y >> 31) * 0x80008000u,
                     (w.z >> 31) * 0x80008000u, (w.w >> 31) * 0x80008000u);
    }
  };
  if (tid == 0) {
    for (int k = 0; k < (NITEMS == 1 ? 1 : qb.n); ++k) tma_prefetch_desc(&qb.item[k].in);
    for (int s = 0; s < kQStages; ++s) mbar_init(&full[s], 1);
    for (int k = 0; k < 2 * kQMaxItems; ++k) s_amax[k] = 0u;
    if constexpr (FMT == kFmtNV && !AMAX) batch_tensor_scales<kRow, kCol, NITEMS>(qb, s_S, bid == 0);
    mbar_fence_init();
  }
  if (rht && my_tiles > 0) write_masks(bid, 0);
  __syncthreads();

  auto issue_load = [&](int stage, int tile) {
    const QuantItem& I = qb.item[batch_item<NITEMS>(qb, tile)];
    int tr, tc;
    qtile_coords<BANDED>(tile - I.tile0, I.a, tr, tc);
    uint8_t* dst = s_in + stage * kQInBytes;
    if (!FP4_IN_BOUNDS(tile < qb.num_tiles && tr >= 0 && tr < I.a.tiles_r && tc >= 0 &&
                       tc < I.a.tiles_c)) {
      tr = 0;  // an in-range tile: the barrier still gets its bytes and nothing hangs
      tc = 0;
    }
    if (!FP4_IN_BOUNDS(stage >= 0 && stage < kQStages)) return;  // the bounded waits report it
    mbar_arrive_expect_tx(&full[stage], kQInBytes);
    tma_load_2d(dst, &I.in, &full[stage], tc * 128, tr * 128);
    tma_load_2d(dst + kQBoxBytes, &I.in, &full[stage], tc * 128 + 64, tr * 128);
  };
  if (tid == 0) {
    const int pro = my_tiles < kQStages ? my_tiles : kQStages;
    for (int s = 0; s < pro; ++s) issue_load(s, bid + s * nctas);
  }

  // Work split of one 128x128 tile over the 256 threads:
  //   ROW job : row tid%128, box tid/128
  //   COL job : column pair tid%64, segment tid/64
  // A thread takes its ROW job (ROW, DUAL) and its COL job (COL, DUAL), so in the dual
  // pass every warp carries the same instruction mix and reaches the barriers together.
  const int row_r = tid & 127;
  const int col_pair = tid & 63, col_b = col_pair >> 5, col_w = col_pair & 31;
  const int col_c = 64 * col_b + 2 * col_w;

  float amax_r = 0.0f, amax_c = 0.0f;
  // Every tensor of a batch has the same wait limit.
  const uint64_t wait_ns = qb.item[0].a.wait_limit_ns;
  for (int it = 0; it < my_tiles; ++it) {
    const int tile = bid + it * nctas;
    // The tile's tensor and coordinates are resolved where they are used: in the jobs
    // only by the variants (always one tensor per launch, so item 0) and NVFP4 (its
    // tensor scales), and after the tile's barrier by the threads that store or publish.
    // Kept live through the jobs, they cost the batched instances registers and time.
    const QuantArgs& a = qb.item[0].a;
    int tr = 0, tc = 0;
    if constexpr (EXT) qtile_coords<BANDED>(tile - qb.item[0].tile0, a, tr, tc);
    float S_r = 1.0f, S_c = 1.0f;  // NVFP4 tensor scales of this tile's tensor
    if constexpr (FMT == kFmtNV && !AMAX) {
      const int item = batch_item<NITEMS>(qb, tile);
      S_r = s_S[2 * item];
      S_c = s_S[2 * item + 1];
    }
    const float six_r = __fmul_rn(6.0f, S_r), six_c = __fmul_rn(6.0f, S_c);
    const int st = it % kQStages, ob = it & 1;
    // One barrier per tile (at its end). The next tile's signs go to the other mask
    // buffer, whose readers (the tile before this one) finished before the last barrier.
    if (rht && it + 1 < my_tiles) write_masks(tile + nctas, (it + 1) & 1);
    const uint32_t* s_cmask = s_masks + 192 * (it & 1);
    const uint32_t* s_rmask = s_cmask + 64;
    // A wait that runs out is acted on at the barrier below, together: the jobs then
    // read stale (never faulting) shared memory, and nothing of this tile is stored.
    const bool ok = mbar_wait(&full[st], static_cast<uint32_t>((it / kQStages) & 1), wait_ns);
    const uint8_t* in = s_in + st * kQInBytes;
    uint8_t* rcode = s_rcode + ob * kCodeBytes;
    uint8_t* ccode = s_ccode + ob * kCodeBytes;
    uint8_t* rsc = s_rsc + ob * kQScaleBytes;
    uint8_t* csc = s_csc + ob * kQScaleBytes;

    if constexpr (kRow) {
      const int b = tid >> 7;
      {
        float2 p[32];
        // the stride-1 butterfly is fused into the widening; random signs (EXT) are
        // XORed into the raw bf16 words before it
        constexpr bool kFuse1 = HN > 0;
        if (rht) {
          if constexpr (kFuse1) load_row_job_bfly1<true>(in, row_r, b, p, s_cmask);
          else load_row_job<true>(in, row_r, b, p, s_cmask);
        } else {
          if constexpr (kFuse1) load_row_job_bfly1(in, row_r, b, p);
          else load_row_job(in, row_r, b, p);
        }
        fwht_x2<HN, !kFoldH16, kFuse1 ? 2 : 1>(p);
        if constexpr (AMAX) {
          const float2 m = amax_x2<0, 32>(p);
          amax_r = max3f(amax_r, m.x, m.y);
        } else if constexpr (FMT == kFmtMX8) {
          const Enc8 e = mx8_encode_x2(p);  // lane x: bytes 64b .. +31, lane y: 64b+32 .. +63
          if (code_ok(row_r, 4 * b + 3, 8)) {
            *reinterpret_cast<uint4*>(code_chunk8(rcode, row_r, 4 * b)) = e.cx[0];
            *reinterpret_cast<uint4*>(code_chunk8(rcode, row_r, 4 * b + 1)) = e.cx[1];
            *reinterpret_cast<uint4*>(code_chunk8(rcode, row_r, 4 * b + 2)) = e.cy[0];
            *reinterpret_cast<uint4*>(code_chunk8(rcode, row_r, 4 * b + 3)) = e.cy[1];
          }
          if (scale_ok(row_r, 2 * b, 2))
            *reinterpret_cast<uint16_t*>(rsc + atom_off(row_r, 2 * b)) =
                static_cast<uint16_t>(e.sx | (e.sy << 8));
        } else {
          Enc e;
          if (sr) {
            // element (row, column) of the ROW-layout matrix: word of index row*cols + column
            const uint64_t f = (static_cast<uint64_t>(tr) * 128 + row_r) * static_cast<uint64_t>(a.cols) +
                               static_cast<uint64_t>(tc) * 128 + 64 * b;
            const SrCodes codes{f >> 2, (f >> 2) + 8, 1u, a.sr_key};
            e = encode_x2<FMT, kFoldH16>(p, S_r, six_r, codes);
          } else {
            e = encode_x2<FMT, kFoldH16>(p, S_r, six_r);
          }
          if (code_ok(row_r, 2 * b + 1, 4)) {
            *reinterpret_cast<uint4*>(code_chunk(rcode, row_r, 2 * b)) = e.cx;
            *reinterpret_cast<uint4*>(code_chunk(rcode, row_r, 2 * b + 1)) = e.cy;
          }
          if constexpr (FMT == kFmtMX) {  // blocks 2b, 2b+1 of this row: adjacent bytes
            if (scale_ok(row_r, 2 * b, 2))
              *reinterpret_cast<uint16_t*>(rsc + atom_off(row_r, 2 * b)) =
                  static_cast<uint16_t>(e.sx | (e.sy << 8));
          } else {  // blocks 4b .. 4b+3: one 4-byte group of atom b
            if (scale_ok(row_r, 4 * b, 4))
              *reinterpret_cast<uint32_t*>(rsc + atom_off(row_r, 4 * b)) = e.sx | (e.sy << 16);
          }
        }
      }
    }
    if constexpr (kCol) {
      const int s = tid >> 6;
      {
        float2 p[32];
        constexpr bool kFuse1 = HN > 0;
        if (rht) {
          if constexpr (kFuse1) load_col_job_bfly1<true>(in, col_b, col_w, s, p, s_rmask);
          else load_col_job<true>(in, col_b, col_w, s, p, s_rmask);
        } else {
          if constexpr (kFuse1) load_col_job_bfly1(in, col_b, col_w, s, p);
          else load_col_job(in, col_b, col_w, s, p);
        }
        fwht_x2<HN, !kFoldH16, kFuse1 ? 2 : 1>(p);
        if constexpr (AMAX) {
          const float2 m = amax_x2<0, 32>(p);
          amax_c = max3f(amax_c, m.x, m.y);
        } else if constexpr (FMT == kFmtMX8) {
          const Enc8 e = mx8_encode_x2(p);  // column c (x) and c+1 (y): rows 32s .. 32s+31
          if (code_ok(col_c + 1, 2 * s + 1, 8)) {
            *reinterpret_cast<uint4*>(code_chunk8(ccode, col_c, 2 * s)) = e.cx[0];
            *reinterpret_cast<uint4*>(code_chunk8(ccode, col_c, 2 * s + 1)) = e.cx[1];
            *reinterpret_cast<uint4*>(code_chunk8(ccode, col_c + 1, 2 * s)) = e.cy[0];
            *reinterpret_cast<uint4*>(code_chunk8(ccode, col_c + 1, 2 * s + 1)) = e.cy[1];
          }
          if (scale_ok(col_c + 1, s, 1)) {
            csc[atom_off(col_c, s)] = static_cast<uint8_t>(e.sx);
            csc[atom_off(col_c + 1, s)] = static_cast<uint8_t>(e.sy);
          }
        } else {
          Enc e;
          if (sr) {
            // element (column, row) of the COL-layout matrix: word of index column*rows + row
            const uint64_t c0 = static_cast<uint64_t>(tc) * 128 + col_c;
            const uint64_t r0 = static_cast<uint64_t>(tr) * 128 + 32 * s;
            const uint64_t fx = c0 * static_cast<uint64_t>(a.rows) + r0;
            const uint64_t fy = fx + static_cast<uint64_t>(a.rows);
            const SrCodes codes{fx >> 2, fy >> 2, 2u, a.sr_key};
            e = encode_x2<FMT, kFoldH16>(p, S_c, six_c, codes);
          } else {
            e = encode_x2<FMT, kFoldH16>(p, S_c, six_c);
          }
          if (code_ok(col_c + 1, s, 4)) {
            *reinterpret_cast<uint4*>(code_chunk(ccode, col_c, s)) = e.cx;
            *reinterpret_cast<uint4*>(code_chunk(ccode, col_c + 1, s)) = e.cy;
          }
          // block kb of segment s: s (MXFP4, one byte) or 2s, 2s+1 (NVFP4, two bytes)
          if constexpr (FMT == kFmtMX) {
            if (scale_ok(col_c + 1, s, 1)) {
              csc[atom_off(col_c, s)] = static_cast<uint8_t>(e.sx);
              csc[atom_off(col_c + 1, s)] = static_cast<uint8_t>(e.sy);
            }
          } else if (scale_ok(col_c + 1, 2 * s, 2)) {
            *reinterpret_cast<uint16_t*>(csc + atom_off(col_c, 2 * s)) = static_cast<uint16_t>(e.sx);
            *reinterpret_cast<uint16_t*>(csc + atom_off(col_c + 1, 2 * s)) = static_cast<uint16_t>(e.sy);
          }
        }
      }
    }

    if constexpr (!AMAX) {
      fence_proxy_async_smem();
      // The next tile writes staging buffer ob^1, which the stores issued after the last
      // barrier are reading: wait for those reads before this barrier releases it.
      if (tid == 0) bulk_wait_read<0>();
    } else {
      // this tile's amax into its tensor's accumulator (a max: exact in any order)
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        amax_r = fmaxf(amax_r, __shfl_xor_sync(0xffffffffu, amax_r, o));
        amax_c = fmaxf(amax_c, __shfl_xor_sync(0xffffffffu, amax_c, o));
      }
      if (lane == 0) {
        const int item = batch_item<NITEMS>(qb, tile);
        if constexpr (kRow) atomicMax(&s_amax[2 * item], __float_as_uint(amax_r));
        if constexpr (kCol) atomicMax(&s_amax[2 * item + 1], __float_as_uint(amax_c));
      }
      amax_r = 0.0f;
      amax_c = 0.0f;
    }
    if (__syncthreads_or(!ok)) break;  // give up together; the status word says why
    if (tid == 0) {
      if constexpr (!AMAX) {
        const int item = batch_item<NITEMS>(qb, tile);
        const QuantItem& I = qb.item[item];
        const QuantArgs& a = I.a;
        qtile_coords<BANDED>(tile - I.tile0, a, tr, tc);
        constexpr int kAtomsPerTile = (FMT == kFmtNV) ? 2 : 1;
        constexpr int kTileCodeBytes = FMT == kFmtMX8 ? 128 : 64;  // code bytes per tile row
        const bool tile_ok = FP4_IN_BOUNDS(tr >= 0 && tr < a.tiles_r && tc >= 0 && tc < a.tiles_c);
        if constexpr (kRow) {
          const int first = tc * kAtomsPerTile;
          const int n = (a.row_kb4 - first) < kAtomsPerTile ? (a.row_kb4 - first) : kAtomsPerTile;
          if (tile_ok) tma_store_2d(&I.rcodes, rcode, tc * kTileCodeBytes, tr * 128);
          if (tile_ok && FP4_IN_BOUNDS(n > 0 && first + n <= a.row_kb4))
            bulk_store(a.row_scales + (static_cast<int64_t>(tr) * a.row_kb4 + first) * 512, rsc,
                       static_cast<uint32_t>(n * 512));
        }
        if constexpr (kCol) {
          const int first = tr * kAtomsPerTile;
          const int n = (a.col_kb4 - first) < kAtomsPerTile ? (a.col_kb4 - first) : kAtomsPerTile;
          if (tile_ok) tma_store_2d(&I.ccodes, ccode, tr * kTileCodeBytes, tc * 128);
          if (tile_ok && FP4_IN_BOUNDS(n > 0 && first + n <= a.col_kb4))
            bulk_store(a.col_scales + (static_cast<int64_t>(tc) * a.col_kb4 + first) * 512, csc,
                       static_cast<uint32_t>(n * 512));
        }
        bulk_commit();
      }
      if (it + kQStages < my_tiles) issue_load(st, tile + kQStages * nctas);
    }
  }
  if constexpr (!AMAX) {
    if (tid == 0) bulk_wait<0>();
  } else {
    __syncthreads();
    if (tid == 0) {
      // non-negative floats order like their bit patterns: max is exact and
      // independent of the order in which CTAs arrive
      for (int k = 0; k < (NITEMS == 1 ? 1 : qb.n); ++k) {
        if constexpr (kRow) atomicMax(qb.item[k].a.amax_row_acc, s_amax[2 * k]);
        if constexpr (kCol) atomicMax(qb.item[k].a.amax_col_acc, s_amax[2 * k + 1]);
      }
    }
  }
}


// ====================================================================================
// quantize_wide_kernel: the plain MXFP4 / NVFP4 quantiser (no variant) with twice the
// warps per SM. The same tiles, TMA pipeline, staging and stores as quantize_kernel, but
// 512 threads per CTA whose jobs hold 32 values (32 registers) instead of 64, so two
// CTAs of 16 warps fit per SM: the ALU and FMA pipes, not warp latency, then set the
// pace. Per 128x128 tile every thread takes
//   one ROW job : row t%128, columns 32q .. 32q+31 (q = t/128) -- one MX block or two NV
//                 blocks -- as 16 pairs (v[2k], v[2k+1]), so strides >= 2 of the
//                 butterfly and the scaling are packed fp32x2 ops;
//   one COL job : columns c, c+1 (lanes x, y) of 16 consecutive rows; lanes 0-15 and
//                 16-31 of a warp hold the two 16-row halves of the same 32-row MX
//                 block, whose amax (and the H32 stride-16 butterfly) they complete
//                 with one warp shuffle.
// The arithmetic of every value is the one quantize_kernel (and the oracle) performs.
constexpr int kQWThreads = 512;
constexpr int kQWSmemBytes = 1024 + 2 * kQInBytes + 2 * 2 * kQCodeBytesOf(kFmtMX) +
                             2 * 2 * kQScaleBytes + 256;

// ROW job loader: row r, columns 32q .. 32q+31 as pairs q2[k] = (v[2k], v[2k+1]); with
// kFuse1 the stride-1 butterfly is done here (q2[k] = (v[2k] + v[2k+1], v[2k] - v[2k+1])).
template <bool kFuse1>
__device__ __forceinline__ void load_row_v(const uint8_t* in, int r, int q, float2 (&q2)[16]) {
  if (!FP4_IN_BOUNDS(r >= 0 && r < 128 && q >= 0 && q < 4)) {
#pragma unroll
    for (int i = 0; i < 16; ++i) q2[i] = make_float2(0.0f, 0.0f);
    return;
  }
  const uint8_t* rowp = in + (q >> 1) * kQBoxBytes + r * 128;
  const int cb = (q & 1) * 4;  // first 16-byte chunk of the 32 columns in the box row
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint4 w = *reinterpret_cast<const uint4*>(rowp + (((cb + j) ^ (r & 7)) << 4));
    const uint32_t a[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if constexpr (kFuse1) {
        float sm, df;
        bfly1_lo(a[k], add_hi(a[k], -0.0f), sm, df);
        q2[4 * j + k] = make_float2(sm, df);
      } else {
        q2[4 * j + k] = make_float2(bf16lo(a[k]), bf16hi(a[k]));
      }
    }
  }
}

// COL job loader: columns 2*cp, 2*cp+1 of the tile (lanes x, y), rows r0 .. r0+15
// (r0 a multiple of 16), p[i] = row r0+i; kFuse1 as for the ROW job.
template <bool kFuse1>
__device__ __forceinline__ void load_col_v(const uint8_t* in, int cp, int r0, float2 (&p)[16]) {
  if (!FP4_IN_BOUNDS(cp >= 0 && cp < 64 && r0 >= 0 && r0 + 16 <= 128 && (r0 & 15) == 0)) {
#pragma unroll
    for (int i = 0; i < 16; ++i) p[i] = make_float2(0.0f, 0.0f);
    return;
  }
  const int wc = cp & 31;
  const uint8_t* colp = in + (cp >> 5) * kQBoxBytes + r0 * 128 + ((wc & 3) << 2);
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    // rows r0+i, r0+i+1: (r0 + i) & 7 == i & 7, a compile-time swizzle per step
    const uint32_t v0 = *reinterpret_cast<const uint32_t*>(colp + i * 128 + (((wc >> 2) ^ (i & 7)) << 4));
    const uint32_t v1 =
        *reinterpret_cast<const uint32_t*>(colp + (i + 1) * 128 + (((wc >> 2) ^ ((i + 1) & 7)) << 4));
    if constexpr (kFuse1) {
      float sx, dx, sy, dy;
      bfly1_lo(v0, add_lo(v1, -0.0f), sx, dx);
      bfly1_hi(v0, add_hi(v1, -0.0f), sy, dy);
      p[i] = make_float2(sx, sy);
      p[i + 1] = make_float2(dx, dy);
    } else {
      p[i] = make_float2(bf16lo(v0), bf16hi(v0));
      p[i + 1] = make_float2(bf16lo(v1), bf16hi(v1));
    }
  }
}

// Rotation stages after the fused stride-1 stage, and the final x c (unless folded).
// ROW: strides 2 .. HN/2 pair q2[j] with q2[j + h/2] (both values of a pair share bit h).
template <int HN, bool kScale>
__device__ __forceinline__ void fwht_row_v(float2 (&q2)[16]) {
  if constexpr (HN > 0) {
#pragma unroll
    for (int h = 2; h < HN; h <<= 1) {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if ((j & (h >> 1)) == 0) {
          const float2 a = q2[j], b = q2[j + (h >> 1)];
          q2[j] = add2(a, b);
          q2[j + (h >> 1)] = sub2(a, b);
        }
      }
    }
    if constexpr (kScale) {
      const float c = (HN == 16) ? 0.25f : __uint_as_float(0x3E3504F3u);
      const float2 c2 = make_float2(c, c);
#pragma unroll
      for (int i = 0; i < 16; ++i) q2[i] = mul2(q2[i], c2);
    }
  }
}
// COL: strides 2 .. 8 inside the 16 rows; for H32 the stride-16 stage pairs row i of the
// lower half-warp (a) with row i of the upper one (b): lower keeps a + b, upper a - b.
template <int HN, bool kScale>
__device__ __forceinline__ void fwht_col_v(float2 (&p)[16], bool upper) {
  if constexpr (HN > 0) {
#pragma unroll
    for (int h = 2; h < HN && h < 16; h <<= 1) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        if ((i & h) == 0) {
          const float2 a = p[i], b = p[i + h];
          p[i] = add2(a, b);
          p[i + h] = sub2(a, b);
        }
      }
    }
    if constexpr (HN == 32) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float2 o = make_float2(__shfl_xor_sync(0xffffffffu, p[i].x, 16),
                                     __shfl_xor_sync(0xffffffffu, p[i].y, 16));
        // lower: p + o; upper: o + (-p) = o - p, each rounded once
        const float2 x = upper ? o : p[i];
        const float2 y = upper ? make_float2(-p[i].x, -p[i].y) : o;
        p[i] = add2(x, y);
      }
    }
    if constexpr (kScale) {
      const float c = (HN == 16) ? 0.25f : __uint_as_float(0x3E3504F3u);
      const float2 c2 = make_float2(c, c);
#pragma unroll
      for (int i = 0; i < 16; ++i) p[i] = mul2(p[i], c2);
    }
  }
}

// MX scale byte and multiplier 2^-e from a block amax (R2), with the H16 fold when kFold:
// byte = biased exponent of amax - 4 and the multiplier takes the x0.25 along
// (valid when amax >= 2^-100, else *two_step is set and the caller multiplies by 0.25
// first and uses the plain rule).
__device__ __forceinline__ uint32_t mx_byte(float amax) {
  const uint32_t e = (__float_as_uint(amax) >> 23) & 0xFFu;
  return e > 2u ? e - 2u : 0u;
}
__device__ __forceinline__ float mx_inv(uint32_t byte) { return __uint_as_float((254u - byte) << 23); }

// Codes of 16 pairs (v[2k] low nibble, v[2k+1] high) as four words, byte k = pair k.
__device__ __forceinline__ uint4 codes_row16(const float2 (&q2)[16]) {
  uint32_t w[4];
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const float v[8] = {q2[4 * m].x,     q2[4 * m].y,     q2[4 * m + 1].x, q2[4 * m + 1].y,
                        q2[4 * m + 2].x, q2[4 * m + 2].y, q2[4 * m + 3].x, q2[4 * m + 3].y};
    w[m] = cvt_e2m1x8(v);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}
// Codes of one lane of 16 consecutive entries (8 bytes).
__device__ __forceinline__ uint2 codes_col16x(const float2 (&p)[16]) {
  const float a[8] = {p[0].x, p[1].x, p[2].x, p[3].x, p[4].x, p[5].x, p[6].x, p[7].x};
  const float b[8] = {p[8].x, p[9].x, p[10].x, p[11].x, p[12].x, p[13].x, p[14].x, p[15].x};
  return make_uint2(cvt_e2m1x8(a), cvt_e2m1x8(b));
}
__device__ __forceinline__ uint2 codes_col16y(const float2 (&p)[16]) {
  const float a[8] = {p[0].y, p[1].y, p[2].y, p[3].y, p[4].y, p[5].y, p[6].y, p[7].y};
  const float b[8] = {p[8].y, p[9].y, p[10].y, p[11].y, p[12].y, p[13].y, p[14].y, p[15].y};
  return make_uint2(cvt_e2m1x8(a), cvt_e2m1x8(b));
}

// NVFP4 block of 16 values held as 8 pairs q2[B .. B+8) (ROW job): scale byte, and the
// pairs replaced by their quotients RN(v/d) (or signed zeros); the arithmetic of
// nv_block_x2 (the correction step, else exact division), kQuarter included.
template <int B, bool kQuarter = false>
__device__ __forceinline__ uint32_t nv_block_row_v(float2 (&q2)[16], float S, float six_s) {
  float a[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    a[2 * i] = fabsf(q2[B + i].x);
    a[2 * i + 1] = fabsf(q2[B + i].y);
  }
  float bm = tree_max<16>(a);
  if constexpr (kQuarter) bm = __fmul_rn(bm, 0.25f);
  const uint32_t sb = cvt_e4m3(__fdiv_rn(bm, six_s));
  const float d = __fmul_rn(e4m3_to_f32(sb), S);
  const float e = kQuarter ? __fmul_rn(d, 4.0f) : d;  // the divisor of the values held
  if (e >= 0x1p-100f && e <= 0x1p100f && bm <= 3.0e38f) {  // the correction step
    const float y = __frcp_rn(e);
    const float2 y2 = make_float2(y, y), e2 = make_float2(e, e);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 v = q2[B + i];
      const float2 q0 = mul2(v, y2);
      const float2 q1 = __ffma2_rn(neg2(__ffma2_rn(q0, e2, neg2(v))), y2, q0);  // faithful
      q2[B + i] = __ffma2_rn(neg2(__ffma2_rn(q1, e2, neg2(v))), y2, q1);          // RN(v/d)
    }
  } else if (sb == 0u) {  // a zero block scale: zeros that keep the sign of each element
#pragma unroll
    for (int i = 0; i < 8; ++i)
      q2[B + i] = make_float2(__uint_as_float(__float_as_uint(q2[B + i].x) & 0x80000000u),
                              __uint_as_float(__float_as_uint(q2[B + i].y) & 0x80000000u));
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 v = kQuarter ? mul2(q2[B + i], make_float2(0.25f, 0.25f)) : q2[B + i];
      q2[B + i] = make_float2(__fdiv_rn(v.x, d), __fdiv_rn(v.y, d));
    }
  }
  return sb;
}

template <int FMT, int HN, int MODE, bool AMAX, bool BANDED = false, int NITEMS = 1>
__global__ void __launch_bounds__(kQWThreads, 2)
    quantize_wide_kernel(const __grid_constant__ QuantBatch qb) {
  static_assert(FMT == kFmtMX || FMT == kFmtNV, "FP4 formats only");
  constexpr bool kRow = (MODE & kModeRow) != 0;
  constexpr bool kCol = (MODE & kModeCol) != 0;
  constexpr bool kFold = FMT == kFmtMX && HN == 16 && !AMAX;
  // NVFP4 + H16: the rotation's x0.25 is applied per block (to its amax and divisor),
  // not per element; the amax pass applies it once to each published tile amax
  constexpr bool kQuarter = FMT == kFmtNV && HN == 16;
  constexpr bool kScale = !kFold && !kQuarter;
  constexpr bool kFuse1 = HN > 0;
  constexpr int kStages = 2;
  constexpr int kCodeBytes = kQCodeBytesOf(FMT);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* s_in = smem;
  uint8_t* s_rcode = s_in + kStages * kQInBytes;
  uint8_t* s_ccode = s_rcode + 2 * kCodeBytes;
  uint8_t* s_rsc = s_ccode + 2 * kCodeBytes;
  uint8_t* s_csc = s_rsc + 2 * kQScaleBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(s_csc + 2 * kQScaleBytes);
  unsigned* s_amax = reinterpret_cast<unsigned*>(full + kStages);  // [kQMaxItems][2]
  float* s_S = reinterpret_cast<float*>(s_amax + 2 * kQMaxItems);   // [kQMaxItems][2]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bid = blockIdx.x, nctas = gridDim.x;
  const int my_tiles = bid < qb.num_tiles ? (qb.num_tiles - bid + nctas - 1) / nctas : 0;

  if (tid == 0) {
    for (int k = 0; k < (NITEMS == 1 ? 1 : qb.n); ++k) tma_prefetch_desc(&qb.item[k].in);
    for (int st = 0; st < kStages; ++st) mbar_init(&full[st], 1);
    for (int k = 0; k < 2 * kQMaxItems; ++k) s_amax[k] = 0u;
    if constexpr (FMT == kFmtNV && !AMAX) batch_tensor_scales<kRow, kCol, NITEMS>(qb, s_S, bid == 0);
    mbar_fence_init();
  }
  __syncthreads();

  auto issue_load = [&](int stage, int tile) {
    const QuantItem& I = qb.item[batch_item<NITEMS>(qb, tile)];
    int tr, tc;
    qtile_coords<BANDED>(tile - I.tile0, I.a, tr, tc);
    uint8_t* dst = s_in + stage * kQInBytes;
    if (!FP4_IN_BOUNDS(tile < qb.num_tiles && tr >= 0 && tr < I.a.tiles_r && tc >= 0 &&
                       tc < I.a.tiles_c)) {
      tr = 0;
      tc = 0;
    }
    if (!FP4_IN_BOUNDS(stage >= 0 && stage < kStages)) return;
    mbar_arrive_expect_tx(&full[stage], kQInBytes);
    tma_load_2d(dst, &I.in, &full[stage], tc * 128, tr * 128);
    tma_load_2d(dst + kQBoxBytes, &I.in, &full[stage], tc * 128 + 64, tr * 128);
  };
  if (tid == 0) {
    const int pro = my_tiles < kStages ? my_tiles : kStages;
    for (int st = 0; st < pro; ++st) issue_load(st, bid + st * nctas);
  }

  // job coordinates (fixed for the kernel)
  const int row_r = tid & 127, row_q = tid >> 7;
  const int col_cp = (warp & 3) * 16 + (lane & 15);  // column pair 0 .. 63
  const int col_s = warp >> 2;                        // 32-row block 0 .. 3
  const bool col_upper = lane >= 16;                  // rows 16 .. 31 of the block
  const int col_r0 = 32 * col_s + (col_upper ? 16 : 0);
  const int col_c = 2 * col_cp;

  float amax_r = 0.0f, amax_c = 0.0f;
  // Every tensor of a batch has the same wait limit.
  const uint64_t wait_ns = qb.item[0].a.wait_limit_ns;
  for (int it = 0; it < my_tiles; ++it) {
    const int tile = bid + it * nctas;
    // The jobs need only the NVFP4 tensor scales of the tile's tensor, read where each
    // job uses them; its arguments and coordinates are resolved after the tile's
    // barrier, by the threads that store or publish (kept live through the jobs they
    // cost registers and spills).
    const int item = (FMT == kFmtNV && !AMAX) ? batch_item<NITEMS>(qb, tile) : 0;
    const int st = it % kStages, ob = it & 1;
    const bool ok = mbar_wait(&full[st], static_cast<uint32_t>((it / kStages) & 1), wait_ns);
    const uint8_t* in = s_in + st * kQInBytes;
    uint8_t* rcode = s_rcode + ob * kCodeBytes;
    uint8_t* ccode = s_ccode + ob * kCodeBytes;
    uint8_t* rsc = s_rsc + ob * kQScaleBytes;
    uint8_t* csc = s_csc + ob * kQScaleBytes;

    if constexpr (kRow) {
      float2 q2[16];
      load_row_v<kFuse1>(in, row_r, row_q, q2);
      fwht_row_v<HN, kScale>(q2);
      if constexpr (AMAX) {
        float v[32];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          v[2 * i] = fabsf(q2[i].x);
          v[2 * i + 1] = fabsf(q2[i].y);
        }
        amax_r = fmaxf(amax_r, tree_max<32>(v));
      } else if constexpr (FMT == kFmtMX) {
        float v[32];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          v[2 * i] = fabsf(q2[i].x);
          v[2 * i + 1] = fabsf(q2[i].y);
        }
        const float am = tree_max<32>(v);
        uint32_t byte;
        float inv;
        if (kFold && am >= 0x1p-100f) {  // the x0.25 of H16 folded into the scale
          byte = ((__float_as_uint(am) >> 23) & 0xFFu) - 4u;
          inv = __uint_as_float((252u - byte) << 23);
        } else {
          if constexpr (kFold) {  // tiny block: the two-step rule
            const float2 c2 = make_float2(0.25f, 0.25f);
#pragma unroll
            for (int i = 0; i < 16; ++i) q2[i] = mul2(q2[i], c2);
            byte = mx_byte(__fmul_rn(am, 0.25f));
          } else {
            byte = mx_byte(am);
          }
          inv = mx_inv(byte);
        }
        const float2 inv2 = make_float2(inv, inv);
#pragma unroll
        for (int i = 0; i < 16; ++i) q2[i] = mul2(q2[i], inv2);
        if (code_ok(row_r, row_q, 4))
          *reinterpret_cast<uint4*>(code_chunk(rcode, row_r, row_q)) = codes_row16(q2);
        if (scale_ok(row_r, row_q, 1)) rsc[atom_off(row_r, row_q)] = static_cast<uint8_t>(byte);
      } else {  // NVFP4: blocks 2q and 2q+1
        const float S_r = s_S[2 * item], six_r = __fmul_rn(6.0f, S_r);
        const uint32_t b0 = nv_block_row_v<0, kQuarter>(q2, S_r, six_r);
        const uint32_t b1 = nv_block_row_v<8, kQuarter>(q2, S_r, six_r);
        if (code_ok(row_r, row_q, 4))
          *reinterpret_cast<uint4*>(code_chunk(rcode, row_r, row_q)) = codes_row16(q2);
        if (scale_ok(row_r, 2 * row_q, 2))
          *reinterpret_cast<uint16_t*>(rsc + atom_off(row_r, 2 * row_q)) =
              static_cast<uint16_t>(b0 | (b1 << 8));
      }
    }
    if constexpr (kCol) {
      float2 p[16];
      load_col_v<kFuse1>(in, col_cp, col_r0, p);
      fwht_col_v<HN, kScale>(p, col_upper);
      if constexpr (AMAX) {
        const float2 m = amax_x2<0, 16>(p);
        amax_c = max3f(amax_c, m.x, m.y);
      } else if constexpr (FMT == kFmtMX) {
        float2 m = amax_x2<0, 16>(p);  // this half's 16 rows, then the other half's
        m.x = fmaxf(m.x, __shfl_xor_sync(0xffffffffu, m.x, 16));
        m.y = fmaxf(m.y, __shfl_xor_sync(0xffffffffu, m.y, 16));
        uint32_t bx, by;
        float2 inv;
        if (kFold && m.x >= 0x1p-100f && m.y >= 0x1p-100f) {
          bx = ((__float_as_uint(m.x) >> 23) & 0xFFu) - 4u;
          by = ((__float_as_uint(m.y) >> 23) & 0xFFu) - 4u;
          inv = make_float2(__uint_as_float((252u - bx) << 23), __uint_as_float((252u - by) << 23));
        } else {
          if constexpr (kFold) {
            const float2 c2 = make_float2(0.25f, 0.25f);
#pragma unroll
            for (int i = 0; i < 16; ++i) p[i] = mul2(p[i], c2);
            bx = mx_byte(__fmul_rn(m.x, 0.25f));
            by = mx_byte(__fmul_rn(m.y, 0.25f));
          } else {
            bx = mx_byte(m.x);
            by = mx_byte(m.y);
          }
          inv = make_float2(mx_inv(bx), mx_inv(by));
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) p[i] = mul2(p[i], inv);
        if (code_ok(col_c + 1, col_s, 4)) {
          *reinterpret_cast<uint2*>(code_chunk(ccode, col_c, col_s) + (col_upper ? 8 : 0)) =
              codes_col16x(p);
          *reinterpret_cast<uint2*>(code_chunk(ccode, col_c + 1, col_s) + (col_upper ? 8 : 0)) =
              codes_col16y(p);
        }
        if (!col_upper && scale_ok(col_c + 1, col_s, 1)) {
          csc[atom_off(col_c, col_s)] = static_cast<uint8_t>(bx);
          csc[atom_off(col_c + 1, col_s)] = static_cast<uint8_t>(by);
        }
      } else {  // NVFP4: the 16 rows are one block per column
        const float S_c = s_S[2 * item + 1], six_c = __fmul_rn(6.0f, S_c);
        uint32_t sbx, sby;
        nv_block_x2<0, false, 16, kQuarter>(p, S_c, six_c, sbx, sby);
        if (code_ok(col_c + 1, col_s, 4)) {
          *reinterpret_cast<uint2*>(code_chunk(ccode, col_c, col_s) + (col_upper ? 8 : 0)) =
              codes_col16x(p);
          *reinterpret_cast<uint2*>(code_chunk(ccode, col_c + 1, col_s) + (col_upper ? 8 : 0)) =
              codes_col16y(p);
        }
        const int kb = 2 * col_s + (col_upper ? 1 : 0);
        if (scale_ok(col_c + 1, kb, 1)) {
          csc[atom_off(col_c, kb)] = static_cast<uint8_t>(sbx);
          csc[atom_off(col_c + 1, kb)] = static_cast<uint8_t>(sby);
        }
      }
    }

    if constexpr (!AMAX) {
      fence_proxy_async_smem();
      if (tid == 0) bulk_wait_read<0>();  // staging ob^1 free before the barrier releases it
    } else {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        amax_r = fmaxf(amax_r, __shfl_xor_sync(0xffffffffu, amax_r, o));
        amax_c = fmaxf(amax_c, __shfl_xor_sync(0xffffffffu, amax_c, o));
      }
      if (lane == 0) {
        const int k = batch_item<NITEMS>(qb, tile);
        // max |RN(w/4)| = RN(max |w| / 4): rounding is monotonic and odd
        if constexpr (kQuarter) {
          amax_r = __fmul_rn(amax_r, 0.25f);
          amax_c = __fmul_rn(amax_c, 0.25f);
        }
        if constexpr (kRow) atomicMax(&s_amax[2 * k], __float_as_uint(amax_r));
        if constexpr (kCol) atomicMax(&s_amax[2 * k + 1], __float_as_uint(amax_c));
      }
      amax_r = 0.0f;
      amax_c = 0.0f;
    }
    if (__syncthreads_or(!ok)) break;  // give up together; the status word says why
    if (tid == 0) {
      if constexpr (!AMAX) {
        const QuantItem& I = qb.item[batch_item<NITEMS>(qb, tile)];
        const QuantArgs& a = I.a;
        int tr, tc;
        qtile_coords<BANDED>(tile - I.tile0, a, tr, tc);
        constexpr int kAtomsPerTile = (FMT == kFmtNV) ? 2 : 1;
        const bool tile_ok = FP4_IN_BOUNDS(tr >= 0 && tr < a.tiles_r && tc >= 0 && tc < a.tiles_c);
        if constexpr (kRow) {
          const int first = tc * kAtomsPerTile;
          const int n = (a.row_kb4 - first) < kAtomsPerTile ? (a.row_kb4 - first) : kAtomsPerTile;
          if (tile_ok) tma_store_2d(&I.rcodes, rcode, tc * 64, tr * 128);
          if (tile_ok && FP4_IN_BOUNDS(n > 0 && first + n <= a.row_kb4))
            bulk_store(a.row_scales + (static_cast<int64_t>(tr) * a.row_kb4 + first) * 512, rsc,
                       static_cast<uint32_t>(n * 512));
        }
        if constexpr (kCol) {
          const int first = tr * kAtomsPerTile;
          const int n = (a.col_kb4 - first) < kAtomsPerTile ? (a.col_kb4 - first) : kAtomsPerTile;
          if (tile_ok) tma_store_2d(&I.ccodes, ccode, tr * 64, tc * 128);
          if (tile_ok && FP4_IN_BOUNDS(n > 0 && first + n <= a.col_kb4))
            bulk_store(a.col_scales + (static_cast<int64_t>(tc) * a.col_kb4 + first) * 512, csc,
                       static_cast<uint32_t>(n * 512));
        }
        bulk_commit();
      }
      if (it + kStages < my_tiles) issue_load(st, tile + kStages * nctas);
    }
  }
  if constexpr (!AMAX) {
    if (tid == 0) bulk_wait<0>();
  } else {
    __syncthreads();
    if (tid == 0) {
      for (int k = 0; k < (NITEMS == 1 ? 1 : qb.n); ++k) {
        if constexpr (kRow) atomicMax(qb.item[k].a.amax_row_acc, s_amax[2 * k]);
        if constexpr (kCol) atomicMax(qb.item[k].a.amax_col_acc, s_amax[2 * k + 1]);
      }
    }
  }
}

}  // namespace fp4k

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
// Structure (one CTA per SM, persistent): the input is cut into 128x128 bf16 tiles;
// a 3-stage TMA pipeline brings each tile into shared memory as two 128B-swizzled
// boxes of 128 rows x 64 columns. 256 threads then work from shared memory:
//   ROW job  = one row, 32 consecutive columns (4 x 16-byte conflict-free reads);
//   COL job  = two adjacent columns, 32 consecutive rows (32 x 4-byte reads);
// the rotation runs entirely in registers, codes are staged in a 64B-swizzled
// [128][64 B] tile and written by a TMA store, scale atoms are assembled in shared
// memory and written by bulk copies. Staging is double-buffered so stores overlap
// the next tile.
#pragma once

#include "common.cuh"

namespace fp4k {

enum { kModeRow = 1, kModeCol = 2, kModeDual = 3 };

constexpr int kQThreads = 256;
constexpr int kQStages = 3;
constexpr int kQBoxBytes = 128 * 64 * 2;    // 128 rows x 64 bf16
constexpr int kQInBytes = 2 * kQBoxBytes;   // a 128 x 128 bf16 tile
constexpr int kQCodeBytes = 128 * 64;       // 128 rows x 64 code bytes
constexpr int kQScaleBytes = 1024;          // up to two 512-byte atoms
constexpr int kQSmemBytes = 1024 /*align*/ + kQStages * kQInBytes + 2 * 2 * kQCodeBytes +
                            2 * 2 * kQScaleBytes + 256;

struct QuantArgs {
  int64_t rows, cols;
  int tiles_c, num_tiles;
  uint8_t* row_scales;   // ROW layout scales (scale matrix [rows][cols/bs])
  uint8_t* col_scales;   // COL layout scales (scale matrix [cols][rows/bs])
  int row_kb4, col_kb4;  // 512-byte atoms per 128-row block of each layout
  const float* amax_row; // NVFP4 quantise pass: tensor amax of each rotation
  const float* amax_col;
  float* s_row_out;      // NVFP4 quantise pass: tensor scales, written by CTA 0
  float* s_col_out;
  unsigned* amax_row_acc;  // NVFP4 amax pass: accumulators (bits of a non-negative float)
  unsigned* amax_col_acc;
  uint64_t wait_limit_ns;
};

// Normalised block FWHT of 32 registers holding 32/HN independent groups.
template <int HN>
__device__ __forceinline__ void fwht32(float (&v)[32]) {
  if constexpr (HN > 0) {
#pragma unroll
    for (int h = 1; h < HN; h <<= 1) {
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        if ((i & h) == 0) {
          const float a = v[i], b = v[i + h];
          v[i] = __fadd_rn(a, b);
          v[i + h] = __fsub_rn(a, b);
        }
      }
    }
    // 0.25 = 1/sqrt(16) exactly; 0x3E3504F3 = fp32 nearest to 1/sqrt(32)
    const float c = (HN == 16) ? 0.25f : __uint_as_float(0x3E3504F3u);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __fmul_rn(v[i], c);
  }
}

__device__ __forceinline__ float amax_of(const float* v, int n) {
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < n; ++i) m = fmaxf(m, fabsf(v[i]));
  return m;
}

// MXFP4 block of 32: E8M0 byte = max(biased exponent of amax - 2, 0), i.e. the byte of
// e = floor(log2 amax) - 2 clamped at -127 (zero and subnormal amax give 0); codes of
// v * 2^-e. 2^-e = 2^(127 - byte) is built from its bit pattern (byte <= 252).
__device__ __forceinline__ uint32_t mx_encode32(float (&v)[32], uint4& codes) {
  const float amax = amax_of(v, 32);
  const uint32_t ex = (__float_as_uint(amax) >> 23) & 0xFFu;
  const uint32_t sb = ex > 2u ? ex - 2u : 0u;
  const float inv = __uint_as_float((254u - sb) << 23);
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __fmul_rn(v[i], inv);
  codes.x = cvt_e2m1x8(v + 0);
  codes.y = cvt_e2m1x8(v + 8);
  codes.z = cvt_e2m1x8(v + 16);
  codes.w = cvt_e2m1x8(v + 24);
  return sb;
}

// NVFP4 block of 16 under tensor scale S (six_s = 6*S, rounded once):
// byte = UE4M3_RNE_satfinite(bmax / six_s), d = ue4m3(byte) * S, codes of v / d;
// a zero byte gives signed zeros.
__device__ __forceinline__ uint32_t nv_encode16(float* v, float S, float six_s, uint32_t& c0,
                                                uint32_t& c1) {
  const float bmax = amax_of(v, 16);
  const uint32_t sb = cvt_e4m3(__fdiv_rn(bmax, six_s));
  if (sb == 0u) {
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(__float_as_uint(v[i]) & 0x80000000u);
  } else {
    const float d = __fmul_rn(e4m3_to_f32(sb), S);
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __fdiv_rn(v[i], d);
  }
  c0 = cvt_e2m1x8(v);
  c1 = cvt_e2m1x8(v + 8);
  return sb;
}

// Offset of scale (row-in-atom-block r, block kb within the tile's atoms) in a staged
// scale tile holding one or two atoms: atom = kb/4, then (r%32)*16 + (r/32)*4 + kb%4.
__device__ __forceinline__ int atom_off(int r, int kb) {
  return (kb >> 2) * 512 + (r & 31) * 16 + (r >> 5) * 4 + (kb & 3);
}

// Encode 32 rotated values (one ROW segment or one COL column segment) into 16 code
// bytes at code_dst and their scale byte(s) into the staged atom(s).
template <int FMT>
__device__ __forceinline__ void encode32(float (&v)[32], uint8_t* code_dst, uint8_t* sc_tile,
                                         int r, int seg, float S, float six_s) {
  uint4 codes;
  if constexpr (FMT == kFmtMX) {
    const uint32_t sb = mx_encode32(v, codes);
    sc_tile[atom_off(r, seg)] = static_cast<uint8_t>(sb);
  } else {
    const uint32_t s0 = nv_encode16(v, S, six_s, codes.x, codes.y);
    const uint32_t s1 = nv_encode16(v + 16, S, six_s, codes.z, codes.w);
    sc_tile[atom_off(r, 2 * seg)] = static_cast<uint8_t>(s0);
    sc_tile[atom_off(r, 2 * seg + 1)] = static_cast<uint8_t>(s1);
  }
  *reinterpret_cast<uint4*>(code_dst) = codes;
}

template <int FMT, int HN, int MODE, bool AMAX>
__global__ void __launch_bounds__(kQThreads, 1)
    quantize_kernel(const __grid_constant__ CUtensorMap tm_in,
                    const __grid_constant__ CUtensorMap tm_rcodes,
                    const __grid_constant__ CUtensorMap tm_ccodes, const QuantArgs a) {
  constexpr bool kRow = (MODE & kModeRow) != 0;
  constexpr bool kCol = (MODE & kModeCol) != 0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* s_in = smem;
  uint8_t* s_rcode = s_in + kQStages * kQInBytes;
  uint8_t* s_ccode = s_rcode + 2 * kQCodeBytes;
  uint8_t* s_rsc = s_ccode + 2 * kQCodeBytes;
  uint8_t* s_csc = s_rsc + 2 * kQScaleBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(s_csc + 2 * kQScaleBytes);
  float* s_red = reinterpret_cast<float*>(full + kQStages);  // [8 warps][2]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bid = blockIdx.x, nctas = gridDim.x;
  const int my_tiles = bid < a.num_tiles ? (a.num_tiles - bid + nctas - 1) / nctas : 0;

  if (tid == 0) {
    tma_prefetch_desc(&tm_in);
    for (int s = 0; s < kQStages; ++s) mbar_init(&full[s], 1);
    mbar_fence_init();
  }
  __syncthreads();

  // NVFP4 tensor scales of the quantise pass: S = amax / 2688 (1 when amax is 0).
  float S_r = 1.0f, S_c = 1.0f;
  if constexpr (FMT == kFmtNV && !AMAX) {
    if constexpr (kRow) {
      const float T = *a.amax_row;
      S_r = T > 0.0f ? __fdiv_rn(T, 2688.0f) : 1.0f;
    }
    if constexpr (kCol) {
      const float T = *a.amax_col;
      S_c = T > 0.0f ? __fdiv_rn(T, 2688.0f) : 1.0f;
    }
    if (bid == 0 && tid == 0) {
      if constexpr (kRow) *a.s_row_out = S_r;
      if constexpr (kCol) *a.s_col_out = S_c;
    }
  }
  const float six_r = __fmul_rn(6.0f, S_r), six_c = __fmul_rn(6.0f, S_c);

  auto issue_load = [&](int stage, int tile) {
    const int tr = tile / a.tiles_c, tc = tile - tr * a.tiles_c;
    uint8_t* dst = s_in + stage * kQInBytes;
    mbar_arrive_expect_tx(&full[stage], kQInBytes);
    tma_load_2d(dst, &tm_in, &full[stage], tc * 128, tr * 128);
    tma_load_2d(dst + kQBoxBytes, &tm_in, &full[stage], tc * 128 + 64, tr * 128);
  };
  if (tid == 0) {
    const int pro = my_tiles < kQStages ? my_tiles : kQStages;
    for (int s = 0; s < pro; ++s) issue_load(s, bid + s * nctas);
  }

  float amax_r = 0.0f, amax_c = 0.0f;
  for (int it = 0; it < my_tiles; ++it) {
    const int tile = bid + it * nctas;
    const int tr = tile / a.tiles_c, tc = tile - tr * a.tiles_c;
    const int st = it % kQStages, ob = it & 1;
    const bool ok = mbar_wait(&full[st], static_cast<uint32_t>((it / kQStages) & 1), a.wait_limit_ns);
    if (__syncthreads_or(!ok)) break;  // give up together; the status word says why
    const uint8_t* in = s_in + st * kQInBytes;

    if constexpr (kRow) {
      // ROW jobs: row r of the tile, 32-column segments seg = 2*(warp/4) + j
      const int r = 32 * (warp & 3) + lane;
#pragma unroll 1
      for (int j = 0; j < 2; ++j) {
        const int seg = 2 * (warp >> 2) + j;
        const uint8_t* rowp = in + (seg >> 1) * kQBoxBytes + r * 128;
        float v[32];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int chunk = (seg & 1) * 4 + i;
          const uint4 w = *reinterpret_cast<const uint4*>(rowp + ((chunk ^ (r & 7)) << 4));
          v[8 * i + 0] = bf16lo(w.x); v[8 * i + 1] = bf16hi(w.x);
          v[8 * i + 2] = bf16lo(w.y); v[8 * i + 3] = bf16hi(w.y);
          v[8 * i + 4] = bf16lo(w.z); v[8 * i + 5] = bf16hi(w.z);
          v[8 * i + 6] = bf16lo(w.w); v[8 * i + 7] = bf16hi(w.w);
        }
        fwht32<HN>(v);
        if constexpr (AMAX) {
          amax_r = fmaxf(amax_r, amax_of(v, 32));
        } else {
          uint8_t* cdst = s_rcode + ob * kQCodeBytes + r * 64 + ((seg ^ ((r >> 1) & 3)) << 4);
          encode32<FMT>(v, cdst, s_rsc + ob * kQScaleBytes, r, seg, S_r, six_r);
        }
      }
    }
    if constexpr (kCol) {
      // COL jobs: box b = warp%2 (tile columns 64b..64b+63), rows 32*seg..32*seg+31,
      // lane -> tile columns c = 64b + 2*lane and c + 1
      const int b = warp & 1, seg = warp >> 1;
      const uint8_t* boxp = in + b * kQBoxBytes;
      float v0[32], v1[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int r = 32 * seg + i;
        const uint32_t w = *reinterpret_cast<const uint32_t*>(
            boxp + r * 128 + ((((lane >> 2) ^ (r & 7))) << 4) + ((lane & 3) << 2));
        v0[i] = bf16lo(w);
        v1[i] = bf16hi(w);
      }
      fwht32<HN>(v0);
      fwht32<HN>(v1);
      if constexpr (AMAX) {
        amax_c = fmaxf(amax_c, fmaxf(amax_of(v0, 32), amax_of(v1, 32)));
      } else {
        const int c = 64 * b + 2 * lane;
        uint8_t* ctile = s_ccode + ob * kQCodeBytes;
        uint8_t* stile = s_csc + ob * kQScaleBytes;
        encode32<FMT>(v0, ctile + c * 64 + ((seg ^ ((c >> 1) & 3)) << 4), stile, c, seg, S_c,
                      six_c);
        encode32<FMT>(v1, ctile + (c + 1) * 64 + ((seg ^ (((c + 1) >> 1) & 3)) << 4), stile,
                      c + 1, seg, S_c, six_c);
      }
    }

    if constexpr (!AMAX) fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      if constexpr (!AMAX) {
        constexpr int kAtomsPerTile = (FMT == kFmtMX) ? 1 : 2;
        if constexpr (kRow) {
          tma_store_2d(&tm_rcodes, s_rcode + ob * kQCodeBytes, tc * 64, tr * 128);
          const int first = tc * kAtomsPerTile;
          const int n = (a.row_kb4 - first) < kAtomsPerTile ? (a.row_kb4 - first) : kAtomsPerTile;
          bulk_store(a.row_scales + (static_cast<int64_t>(tr) * a.row_kb4 + first) * 512,
                     s_rsc + ob * kQScaleBytes, static_cast<uint32_t>(n * 512));
        }
        if constexpr (kCol) {
          tma_store_2d(&tm_ccodes, s_ccode + ob * kQCodeBytes, tr * 64, tc * 128);
          const int first = tr * kAtomsPerTile;
          const int n = (a.col_kb4 - first) < kAtomsPerTile ? (a.col_kb4 - first) : kAtomsPerTile;
          bulk_store(a.col_scales + (static_cast<int64_t>(tc) * a.col_kb4 + first) * 512,
                     s_csc + ob * kQScaleBytes, static_cast<uint32_t>(n * 512));
        }
        bulk_commit();
      }
      if (it + kQStages < my_tiles) issue_load(st, tile + kQStages * nctas);
      if constexpr (!AMAX) bulk_wait_read<1>();
    }
    __syncthreads();
  }
  if constexpr (!AMAX) {
    if (tid == 0) bulk_wait<0>();
  } else {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      amax_r = fmaxf(amax_r, __shfl_xor_sync(0xffffffffu, amax_r, o));
      amax_c = fmaxf(amax_c, __shfl_xor_sync(0xffffffffu, amax_c, o));
    }
    if (lane == 0) {
      s_red[2 * warp] = amax_r;
      s_red[2 * warp + 1] = amax_c;
    }
    __syncthreads();
    if (tid == 0) {
      float mr = 0.0f, mc = 0.0f;
      for (int w = 0; w < kQThreads / 32; ++w) {
        mr = fmaxf(mr, s_red[2 * w]);
        mc = fmaxf(mc, s_red[2 * w + 1]);
      }
      // non-negative floats order like their bit patterns: max is exact and
      // independent of the order in which CTAs arrive
      if constexpr (kRow) atomicMax(a.amax_row_acc, __float_as_uint(mr));
      if constexpr (kCol) atomicMax(a.amax_col_acc, __float_as_uint(mc));
    }
  }
}

}  // namespace fp4k

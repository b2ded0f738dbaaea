// gemm.cuh -- block-scaled FP4 GEMM on the sm_100a tensor cores.
//
//   C[M][N] = sum_k deq(A)[m][k] * deq(B)[n][k]   (both operands K-major, E2M1 packed)
//
// with deq = e2m1 * 2^(byte-127) (MXFP4, 32-element blocks) or e2m1 * ue4m3(byte)
// (NVFP4, 16-element blocks; the fp32 tensor scales S_A * S_B are applied in the
// epilogue), or e4m3 * 2^(byte-127) for the MXFP8 comparator (one byte per element).
// Accumulation is fp32 in tensor memory. [gist.science summary of arXiv
// 2605.09825, Methodology item 2 (all three GEMM passes in FP4); molayo1419.me
// NVFP4/MaxText page, Key facts bullet 5 (FP4 tensor cores on Blackwell).]
//
// Two kernels share the MMA issue loop (Issuer) and the epilogue (store_row_segment):
// gemm_fp4_pair_kernel (CTA pairs, cta_group::2, 256x256 tiles; every M > 128, all
// MXFP8, and groups of GEMMs run in one launch, GemmGroup) and gemm_fp4_kernel (one
// CTA, 128x256 tiles; FP4 with M <= 128), the latter described here:
//
// Design (one CTA per SM, persistent over 128x256 output tiles, K in slabs of 256):
//   warp 0   : TMA producer. Per slab it loads A 128x128 B, B 256x128 B (128B swizzle)
//              and the matching 512-byte scale atoms into a 4-stage ring.
//   warp 1   : allocates 512 TMEM columns; per slab, once the stage has landed, copies
//              its scale atoms smem -> TMEM (tcgen05.cp 32x128b.warpx4) into the slab's
//              ring slot and issues its 4 MMAs of 128x256x64 (tcgen05.mma kind::mxf4 /
//              kind::mxf4nvf4) behind them, in order, then commits the stage back to
//              the producer; after the last slab it commits the accumulator to the
//              epilogue (Issuer::run).
//   The producer and MMA roles run their loops on all 32 lanes (waits and the
//   abort flag combined by votes, so control flow and descriptors stay warp-uniform);
//   one lane chosen by elect.sync issues each TMA copy and tcgen05 instruction.
//   warps 2-9: epilogue. Each warp owns one 32-lane quarter of TMEM and one half of
//              the 256 columns: it pulls its 32x128 fp32 block into registers,
//              releases the accumulator (so the next tile's MMAs start), then scales
//              and stores fp32 or bf16 rows to global memory.
// TMEM columns: [0,256) accumulator, then a ring of 4 scale-factor regions (one per
// slab in flight, so a slab's scale copies never wait for the previous slab's MMAs).
// No cluster multicast anywhere. Every wait is bounded (status word on expiry).
#pragma once

#include "common.cuh"
#include "quantize.cuh"

namespace fp4k {

constexpr int kGBM = 128, kGBN = 256, kGBK = 256;  // tile M, tile N, K elements per slab
constexpr int kGStages = 4;
constexpr int kGThreads = 320;
constexpr int kGABytes = kGBM * kGBK / 2;  // 16 KB
constexpr int kGBBytes = kGBN * kGBK / 2;  // 32 KB

template <int FMT>
struct GemmCfg {
  static constexpr int kBlock = FMT == kFmtMX ? 32 : 16;
  static constexpr int kAtoms = kGBK / (4 * kBlock);  // scale atoms per 128 rows per slab
  static constexpr int kSFABytes = kAtoms * 512;
  static constexpr int kSFBBytes = 2 * kAtoms * 512;
  static constexpr int kStageBytes = kGABytes + kGBBytes + kSFABytes + kSFBBytes;
  // Scale factors of consecutive slabs go to a ring of kSFBufs TMEM regions so that a
  // slab's smem->TMEM copies never overwrite columns the previous slab's MMAs still read.
  static constexpr int kSFCols = 12 * kAtoms;  // 4*kAtoms (A) + 8*kAtoms (B) per slab
  static constexpr int kSFBufs = 4;
  static constexpr int kTmemSF = 256;
  static constexpr int kSmemBytes = 1024 + kGStages * kStageBytes + 256;
};

struct GemmArgs {
  int M, N, K;
  int tiles_m, tiles_n, num_tiles, k_tiles;
  int band, band_n;  // tile order: see tile_coords
  int c_v8;          // output 32-byte aligned: 32-byte stores
  void* C;           // output; may be null when the epilogue quantises it (fp4_gemm_quant)
  const float* sa;  // NVFP4 tensor scales (device), or null
  const float* sb;
  uint64_t wait_limit_ns;
  // Fused output quantisation (gemm_fp4_pair_kernel with QHN >= 0): row-wise MXFP4
  // codes [M][N/2] and scales (128-row x 4-block atoms, q_kb4 atoms per 128 rows) of
  // RN_bf16(C); rows [M, m_pad) get zero scale bytes (the layout's padding).
  uint8_t* q_codes;
  uint8_t* q_scales;
  int q_kb4, m_pad;
};

// Output tile order. Tiles are numbered in bands of g.band tile rows (g.band_n == 0) or
// tile columns (g.band_n == 1), the banded index running fastest inside a band. The
// operand panels of the banded dimension are then reused by every tile of the band while
// they sit in L2, and the other operand's panels are streamed once per band; the host
// picks the orientation and width from the operand sizes.
__device__ __forceinline__ void tile_coords(int tile, const GemmArgs& g, int& tm, int& tn) {
  const int banded = g.band_n ? g.tiles_n : g.tiles_m;
  const int other = g.band_n ? g.tiles_m : g.tiles_n;
  const int first = tile / (g.band * other) * g.band;
  const int width = min(g.band, banded - first);
  const int r = tile - first * other;
  const int a = first + r % width, b = r / width;
  tm = g.band_n ? b : a;
  tn = g.band_n ? a : b;
  if (!FP4_IN_BOUNDS(tm >= 0 && tm < g.tiles_m && tn >= 0 && tn < g.tiles_n)) {
    tm = 0;  // debug build: an in-range tile keeps every pipeline count intact
    tn = 0;
  }
}

// A group of GEMMs run by one launch of the pair kernel (fp4_gemm_group): their tiles
// form one sequence, problem 0's first, that the persistent CTA pairs walk, so the last
// wave of one GEMM is filled with tiles of the next. Each problem keeps its own tensor
// maps, tile order, K and output type. A single GEMM is a group of one.
constexpr int kGMaxProblems = 3;
struct alignas(64) GemmProblem {
  CUtensorMap a, b, sa, sb;  // operand codes and scales
  CUtensorMap c;             // the output, for the fp32 epilogue's TMA stores
  GemmArgs g;
  int tile0;                 // index of the problem's first tile in the group
  int out_bf16;              // epilogue output: bf16 (1) or fp32 (0)
};
struct GemmGroup {
  GemmProblem p[kGMaxProblems];
  int n;          // problems in use
  int num_tiles;  // tiles of all problems
};

// Problem of a tile of the group (problems are few: a linear scan).
__device__ __forceinline__ int group_problem(const GemmGroup& grp, int tile) {
  int q = 0;
#pragma unroll
  for (int i = 1; i < kGMaxProblems; ++i)
    if (i < grp.n && tile >= grp.p[i].tile0) q = i;
  return q;
}

// Tile schedules the issue threads walk: how many tiles, and how many K slabs a tile has.
struct ArgsSched {  // one GEMM (the one-CTA kernel)
  const GemmArgs& g;
  __device__ __forceinline__ int num_tiles() const { return g.num_tiles; }
  __device__ __forceinline__ int k_tiles(int) const { return g.k_tiles; }
  __device__ __forceinline__ uint64_t wait_ns() const { return g.wait_limit_ns; }
};
struct GroupSched {  // a group (the pair kernel)
  const GemmGroup& grp;
  __device__ __forceinline__ int num_tiles() const { return grp.num_tiles; }
  __device__ __forceinline__ int k_tiles(int tile) const {
    return grp.p[group_problem(grp, tile)].g.k_tiles;
  }
  __device__ __forceinline__ uint64_t wait_ns() const { return grp.p[0].g.wait_limit_ns; }
};

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of 128 bytes,
// 8-row groups 1024 bytes apart (SBO), sm_100 descriptor version 1.
__device__ __forceinline__ uint64_t desc_kmajor_sw128(uint32_t saddr) {
  uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(1) << 16;            // leading byte offset (unused here), 16 B
  d |= static_cast<uint64_t>(1024 >> 4) << 32;    // stride byte offset
  d |= static_cast<uint64_t>(1) << 46;            // version
  d |= static_cast<uint64_t>(2) << 61;            // SWIZZLE_128B
  return d;
}
// Descriptor of one 512-byte scale atom as a 32-row x 16-byte matrix (no swizzle;
// 8-row core matrices of 128 bytes stacked 128 bytes apart).
__device__ __forceinline__ uint64_t desc_sf_atom(uint32_t saddr) {
  uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(128 >> 4) << 16;
  d |= static_cast<uint64_t>(128 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  return d;
}
// Instruction descriptor of the block-scaled MMA: E2M1 x E2M1, both K-major,
// N = 256, M = 128, scale type UE8M0 (MXFP4) or UE4M3 (NVFP4), dense K = 64.
template <int FMT>
__device__ __forceinline__ constexpr uint32_t idesc_fp4() {
  return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(kGBN >> 3) << 17) |
         ((FMT == kFmtMX ? 1u : 0u) << 23) | (static_cast<uint32_t>(kGBM >> 4) << 24);
}


// Instruction descriptor of the pair MMA: as idesc_fp4 with M = 256.
// Operand formats [7,10) and [10,13): E2M1 = 1 for the mxf4 kinds, E4M3 = 0 for
// kind::mxf8f6f4; scale type [23]: UE8M0 (MX formats) or UE4M3 (NVFP4).
template <int FMT>
__device__ __forceinline__ constexpr uint32_t idesc_fp4_pair() {
  constexpr uint32_t ab = FMT == kFmtMX8 ? 0u : 1u;
  return (ab << 7) | (ab << 10) | (static_cast<uint32_t>(256 >> 3) << 17) |
         ((FMT == kFmtNV ? 0u : 1u) << 23) | (static_cast<uint32_t>(256 >> 4) << 24);
}


// ---------------------------------------------------------------- MMA issuer
// The issuing thread walks the K slabs of its tiles with a cursor: the slab's pipeline
// stage and phase, the shared-memory descriptors of its A, B and scale tiles, and the
// TMEM ring slot of its scale factors. Stepping the descriptors only adds to their
// start-address field (+2 per 32 bytes of K inside a 128-byte row, +1024 per 16 KB
// sub-tile, +32 per 512-byte scale atom), which never carries out of the field.
struct SlabCursor {
  int stage;
  uint32_t phase;
  uint64_t dA, dB, dSA, dSB;
  uint32_t t_sf, slot;
};

template <int FMT, bool PAIR, int SLAB_K, int STAGES, int A_BYTES, int B_BYTES, int SFA_BYTES,
          int SFB_BYTES, int SF_COLS, int SF_BUFS>
struct Issuer {
  static constexpr int kAtoms = SLAB_K / (4 * (FMT == kFmtNV ? 16 : 32));
  static constexpr int kMMAs = SLAB_K / (FMT == kFmtMX8 ? 32 : 64);  // K per MMA: 32 B of codes
  static constexpr int kCopies = 3 * kAtoms;  // A atoms, then B atoms of row blocks 0 and 1

  __device__ __forceinline__ static void step(SlabCursor& c, const SlabCursor& base) {
    if (++c.stage == STAGES) {
      c.stage = 0;
      c.phase ^= 1u;
      c.dA = base.dA; c.dB = base.dB; c.dSA = base.dSA; c.dSB = base.dSB;
    } else {
      c.dA += A_BYTES >> 4; c.dB += B_BYTES >> 4;
      c.dSA += SFA_BYTES >> 4; c.dSB += SFB_BYTES >> 4;
    }
    if (++c.slot == SF_BUFS) {
      c.slot = 0;
      c.t_sf = base.t_sf;
    } else {
      c.t_sf += SF_COLS;
    }
  }
  // Scale-factor copies [lo, hi) of a slab into its TMEM ring slot (t_sfb = t_sfa + 4*atoms).
  template <int LO, int HI>
  __device__ __forceinline__ static void copies(const SlabCursor& c) {
#pragma unroll
    for (int i = LO; i < HI; ++i) {
      uint32_t t;
      uint64_t d;
      if (i < kAtoms) {
        t = c.t_sf + 4 * i;
        d = c.dSA + 32 * i;
      } else {
        const int rb = (i - kAtoms) / kAtoms, at = (i - kAtoms) % kAtoms;
        t = c.t_sf + 4 * kAtoms + 8 * at + 4 * rb;
        d = c.dSB + rb * (kAtoms * 32) + 32 * at;
      }
      if (!FP4_IN_BOUNDS((t & 0xFFFFu) + 4u <= 512u)) continue;  // TMEM columns of the copy
      if constexpr (PAIR) tc_cp_32x128b_warpx4_pair(t, d);
      else tc_cp_32x128b_warpx4(t, d);
    }
  }
  // MMA j of a slab: code bytes [32j, 32j+32) of each row (K elements [64j, 64j+64) of
  // FP4, [32j, 32j+32) of FP8).
  __device__ __forceinline__ static void mma(const SlabCursor& c, uint32_t tmem_acc, int j,
                                             bool first) {
    // MXFP4: two MMAs share one atom column, bytes {0,1} then {2,3} (scale id 0 / 2);
    // NVFP4: one atom column per MMA, all four bytes (scale id 0);
    // MXFP8: four MMAs share one atom column, one byte each (scale id 0..3).
    const int at = FMT == kFmtMX ? (j >> 1) : FMT == kFmtNV ? j : (j >> 2);
    const uint32_t id = FMT == kFmtMX    ? static_cast<uint32_t>((j & 1) * 2)
                        : FMT == kFmtMX8 ? static_cast<uint32_t>(j & 3)
                                         : 0u;
    const uint32_t tsfa = (c.t_sf + 4 * at) | (id << 30);
    const uint32_t tsfb = (c.t_sf + 4 * kAtoms + 8 * at) | (id << 30);
    constexpr uint32_t kIdesc = PAIR ? idesc_fp4_pair<FMT>() : idesc_fp4<FMT>();
    const uint32_t idesc = kIdesc | (id << 29) | (id << 4);
    const uint64_t koff = (j >> 2) * (128 * 128 >> 4) + 2 * (j & 3);
    const uint32_t acc = first ? 0u : 1u;
    if (!FP4_IN_BOUNDS((c.t_sf & 0xFFFFu) + SF_COLS <= 512u && (tmem_acc & 0xFFFFu) + 256u <= 512u))
      return;  // TMEM columns of the scale slot or the accumulator
    if constexpr (PAIR)
      tc_mma_fp4_pair<FMT>(tmem_acc, c.dA + koff, c.dB + koff, idesc, tsfa, tsfb, acc);
    else
      tc_mma_fp4<FMT == kFmtMX>(tmem_acc, c.dA + koff, c.dB + koff, idesc, tsfa, tsfb, acc);
  }
  template <int J>
  __device__ __forceinline__ static void slab_mmas(const SlabCursor& c, uint32_t tmem_acc,
                                                   bool first_slab) {
    if constexpr (J < kMMAs) {
      mma(c, tmem_acc, J, first_slab && J == 0);
      slab_mmas<J + 1>(c, tmem_acc, first_slab);
    }
  }
  __device__ __forceinline__ static void commit(uint64_t* bar) {
    if constexpr (PAIR) tc_commit_pair_mc(bar, 0x3);
    else tc_commit(bar);
  }

  __device__ __forceinline__ static SlabCursor make_base(uint32_t tmem, uint8_t* sA, uint8_t* sB,
                                                         uint8_t* sSFA, uint8_t* sSFB) {
    SlabCursor b;
    b.stage = 0;
    b.phase = 0;
    b.dA = desc_kmajor_sw128(smem_u32(sA));
    b.dB = desc_kmajor_sw128(smem_u32(sB));
    b.dSA = desc_sf_atom(smem_u32(sSFA));
    b.dSB = desc_sf_atom(smem_u32(sSFB));
    b.t_sf = tmem + 256;
    b.slot = 0;
    return b;
  }

  // A slab's scale copies go to its TMEM ring slot, issued in order before its MMAs by
  // the same warp. A slot is rewritten only once the slab SF_BUFS later has its stage,
  // whose load waited for the MMAs of the slab STAGES back to complete; SF_BUFS >= STAGES
  // makes those the slot's previous readers (or later ones), so no slot is overwritten
  // while an MMA may still read it.
  static_assert(SF_BUFS >= STAGES, "scale ring must cover the stage ring");

  // Runs all tiles of this CTA (or CTA pair): tiles first, first+stride, ... < num_tiles.
  template <class Sched>
  __device__ static void run(uint32_t tmem, uint8_t* sA, uint8_t* sB, uint8_t* sSFA,
                             uint8_t* sSFB, uint64_t* full, uint64_t* empty, uint64_t* acc_full,
                             uint64_t* acc_empty, volatile int* abort_flag, int first,
                             int stride, const Sched& sc) {
    SlabCursor base = make_base(tmem, sA, sB, sSFA, sSFB);
    SlabCursor cur = base;
    const int nt = sc.num_tiles();
    const int my_tiles = first < nt ? (nt - first + stride - 1) / stride : 0;
    uint32_t acc_phase = 0;
    for (int t = 0; t < my_tiles; ++t) {
      if (!mbar_wait_warp(acc_empty, acc_phase ^ 1u, sc.wait_ns()) || flag_set_warp(abort_flag)) {
        *abort_flag = 1;
        return;
      }
      tc_fence_after();
      const int kts = sc.k_tiles(first + t * stride);
      for (int kt = 0; kt < kts; ++kt) {
        // Each slab: wait for its stage, copy its scales into its TMEM ring slot, issue its
        // MMAs back to back, then release the stage. (Spreading the next slab's copies
        // between this slab's MMAs was measured to be slower.)
        if (!mbar_wait_warp(&full[cur.stage], cur.phase, sc.wait_ns())) {
          *abort_flag = 1;
          return;
        }
        if (elect_one_sync()) {
          copies<0, kCopies>(cur);
          slab_mmas<0>(cur, tmem, kt == 0);
          commit(&empty[cur.stage]);
        }
        __syncwarp();
        step(cur, base);
      }
      if (elect_one_sync()) commit(acc_full);
      __syncwarp();
      acc_phase ^= 1u;
    }
  }
};

// 32-byte global store (one full L2 sector per thread); the address must be 32-byte aligned.
__device__ __forceinline__ void st_global_v8(void* p, const uint32_t (&w)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(w[0]),
               "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

// Two fp32 values -> one word of two bf16 (RN), the first in the low half.
__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Scale (NVFP4) and store one thread's row segment of 128 accumulator columns:
// output row m, columns [n0, n0 + 128), skipping rows >= M and 32-column chunks >= N.
// Each store writes 32 bytes when the output is 32-byte aligned (g.c_v8; rows then are
// too, N being a multiple of 32), else 16 bytes.
template <int FMT, int OUT_BF16>
__device__ __forceinline__ void store_row_segment(const uint32_t (&r)[128], int m, int n0,
                                                  const GemmArgs& g, float alpha) {
  if (m >= g.M) return;
  auto val = [&](int i) {
    const float x = __uint_as_float(r[i]);
    return FMT == kFmtNV ? __fmul_rn(x, alpha) : x;
  };
  if constexpr (OUT_BF16) {
    __nv_bfloat16* crow = static_cast<__nv_bfloat16*>(g.C) + static_cast<int64_t>(m) * g.N + n0;
    auto pack = [&](int i) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(val(i), val(i + 1));
      return *reinterpret_cast<const uint32_t*>(&h);
    };
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if (n0 + 32 * c < g.N) {
        if (g.c_v8) {
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            uint32_t w[8];
#pragma unroll
            for (int p = 0; p < 8; ++p) w[p] = pack(32 * c + 16 * i + 2 * p);
            st_global_v8(crow + 32 * c + 16 * i, w);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int b = 32 * c + 8 * i;
            *reinterpret_cast<uint4*>(crow + b) =
                make_uint4(pack(b), pack(b + 2), pack(b + 4), pack(b + 6));
          }
        }
      }
    }
  } else {
    float* crow = static_cast<float*>(g.C) + static_cast<int64_t>(m) * g.N + n0;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if (n0 + 32 * c < g.N) {
        if (g.c_v8) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint32_t w[8];
#pragma unroll
            for (int p = 0; p < 8; ++p) w[p] = __float_as_uint(val(32 * c + 8 * i + p));
            st_global_v8(crow + 32 * c + 8 * i, w);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int b = 32 * c + 4 * i;
            *reinterpret_cast<float4*>(crow + b) = make_float4(val(b), val(b + 1), val(b + 2), val(b + 3));
          }
        }
      }
    }
  }
}

// Epilogue of the pair kernel for fp32 outputs: one warp's 32-row x 128-column block
// (rows row0 ... row0 + 31, lane i holding row row0 + i in r) leaves the SM through TMA
// stores instead of per-thread global stores. Chunk by chunk (16 bf16 or 8 fp32 columns,
// 32 bytes a row) the lanes write their rows into the warp's 1 KB staging buffer and
// lane 0 issues one bulk tensor store of the 32 x 32-byte box; the TMA drops rows >= M
// and columns >= N. Measured on the Llama layer's Wgrad GEMMs: +3 to +6% over 32-byte
// global stores from registers; bf16 outputs (half the bytes) gained nothing and keep
// store_row_segment.
template <int FMT, int OUT_BF16>
__device__ __forceinline__ void store_segment_tma(const uint32_t (&r)[128], uint8_t* stg,
                                                  const CUtensorMap* tmC, int row0, int n0,
                                                  const GemmArgs& g, float alpha, int lane) {
  constexpr int kCols = OUT_BF16 ? 16 : 8;  // columns of one 32-byte row chunk
  constexpr int kChunks = 128 / kCols;
  if (row0 >= g.M) return;  // the warp's whole block lies beyond M
  auto val = [&](int i) {
    const float x = __uint_as_float(r[i]);
    return FMT == kFmtNV ? __fmul_rn(x, alpha) : x;
  };
#pragma unroll
  for (int ch = 0; ch < kChunks; ++ch) {
    const int c0 = n0 + ch * kCols;
    if (c0 >= g.N) break;  // the rest of the block lies beyond N
    uint32_t w[8];
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      if constexpr (OUT_BF16)
        w[p] = pack2_bf16(val(ch * kCols + 2 * p), val(ch * kCols + 2 * p + 1));
      else
        w[p] = __float_as_uint(val(ch * kCols + p));
    }
    // the previous chunk's store has finished reading the buffer
    if (lane == 0) bulk_wait_read<0>();
    __syncwarp();
    uint4* sp = reinterpret_cast<uint4*>(stg + lane * 32);
    sp[0] = make_uint4(w[0], w[1], w[2], w[3]);
    sp[1] = make_uint4(w[4], w[5], w[6], w[7]);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(tmC, stg, c0, row0);
      bulk_commit();
    }
  }
}

// Epilogue with the output quantised for the next layer, row-wise along N (the next
// contraction axis): the thread's 128 accumulator columns of row m are rounded to bf16
// (the layer output Y, stored when g.C is set), widened back exactly, rotated in groups
// of QHN consecutive columns and quantised to MXFP4 in four 32-column blocks -- the
// quantiser's own ROW-job arithmetic (fused first butterfly, H16 scale fold), so the
// codes and scales equal a separate quantisation of the stored bf16 Y. Columns >= N
// are not stored; their scale bytes, in the same 4-byte word, are the layout's padding
// and come out zero because those accumulator columns are zero (B rows >= N are
// zero-filled by TMA).
template <int FMT, int QHN>
__device__ __forceinline__ void store_row_segment_quant(const uint32_t (&r)[128], int m, int n0,
                                                        const GemmArgs& g, float alpha) {
  // A segment wholly beyond N owns no output column and no scale byte (its scale word
  // would fall into the next atom).
  if (n0 >= g.N) return;
  const int64_t sc_off = (static_cast<int64_t>(m >> 7) * g.q_kb4 + (n0 >> 7)) * 512 +
                         (m & 31) * 16 + ((m & 127) >> 5) * 4;
  const int64_t sc_bytes = static_cast<int64_t>(g.m_pad) * g.q_kb4 * 4;
  if (m >= g.M) {  // rows [M, m_pad): the layout's zero padding; rows beyond: nothing
    if (m < g.m_pad && FP4_IN_BOUNDS(sc_off + 4 <= sc_bytes))
      *reinterpret_cast<uint32_t*>(g.q_scales + sc_off) = 0u;
    return;
  }
  if (!FP4_IN_BOUNDS(m >= 0 && n0 >= 0 && (n0 & 127) == 0 && sc_off + 4 <= sc_bytes)) return;
  uint32_t w[64];  // bf16x2 words: w[k] holds columns 2k (low half) and 2k+1 (high half)
#pragma unroll
  for (int k = 0; k < 64; ++k) {
    float x0 = __uint_as_float(r[2 * k]), x1 = __uint_as_float(r[2 * k + 1]);
    if constexpr (FMT == kFmtNV) {
      x0 = __fmul_rn(x0, alpha);
      x1 = __fmul_rn(x1, alpha);
    }
    const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
    w[k] = *reinterpret_cast<const uint32_t*>(&h);
  }
  if (g.C) {
    __nv_bfloat16* crow = static_cast<__nv_bfloat16*>(g.C) + static_cast<int64_t>(m) * g.N + n0;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if (n0 + 32 * c < g.N) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          *reinterpret_cast<uint4*>(crow + 32 * c + 8 * i) =
              make_uint4(w[16 * c + 4 * i], w[16 * c + 4 * i + 1], w[16 * c + 4 * i + 2],
                         w[16 * c + 4 * i + 3]);
      }
    }
  }
  constexpr bool kFold = QHN == 16;  // MXFP4 + H16: the x0.25 goes into the scale
  constexpr bool kFuse1 = QHN > 0;   // first butterfly fused into the widening
  uint8_t* qrow = g.q_codes + static_cast<int64_t>(m) * (g.N >> 1) + (n0 >> 1);
  uint32_t sbytes = 0;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    // lane x = columns 64*half + 0..31, lane y = 64*half + 32..63 (words wx, wy)
    float2 p[32];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const uint32_t wx = w[32 * half + k], wy = w[32 * half + 16 + k];
      if constexpr (kFuse1) {
        float sx, dx, sy, dy;
        bfly1_lo(wx, add_hi(wx, -0.0f), sx, dx);
        bfly1_lo(wy, add_hi(wy, -0.0f), sy, dy);
        p[2 * k] = make_float2(sx, sy);
        p[2 * k + 1] = make_float2(dx, dy);
      } else {
        p[2 * k] = make_float2(bf16lo(wx), bf16lo(wy));
        p[2 * k + 1] = make_float2(bf16hi(wx), bf16hi(wy));
      }
    }
    fwht_x2<QHN, !kFold, kFuse1 ? 2 : 1>(p);
    const Enc e = encode_x2<kFmtMX, kFold>(p, 1.0f, 6.0f);
    if (n0 + 64 * half < g.N) *reinterpret_cast<uint4*>(qrow + 32 * half) = e.cx;
    if (n0 + 64 * half + 32 < g.N) *reinterpret_cast<uint4*>(qrow + 32 * half + 16) = e.cy;
    sbytes |= (e.sx | (e.sy << 8)) << (16 * half);
  }
  *reinterpret_cast<uint32_t*>(g.q_scales + sc_off) = sbytes;
}

// Threads of the one-CTA kernel: warp 0 loads, warp 1 issues each slab's scale copies
// and MMAs (Issuer::run), warps 2-9 drain the accumulator.
constexpr int kGSingleThreads = kGThreads;

template <int FMT, int OUT_BF16>
__global__ void __launch_bounds__(kGSingleThreads, 1)
    gemm_fp4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmSFA,
                    const __grid_constant__ CUtensorMap tmSFB, const GemmArgs g) {
  using Cfg = GemmCfg<FMT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + kGStages * kGABytes;
  uint8_t* sSFA = sB + kGStages * kGBBytes;
  uint8_t* sSFB = sSFA + kGStages * Cfg::kSFABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sSFB + kGStages * Cfg::kSFBBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + kGStages;
  uint64_t* acc_full = bars + 2 * kGStages;
  uint64_t* acc_empty = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  static_assert((2 * kGStages + 2) * 8 + 8 <= 256, "barrier area");
  using SingleIssuer = Issuer<FMT, false, kGBK, kGStages, kGABytes, kGBBytes, Cfg::kSFABytes,
                              Cfg::kSFBBytes, Cfg::kSFCols, Cfg::kSFBufs>;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmSFA);
    tma_prefetch_desc(&tmSFB);
    for (int s = 0; s < kGStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 8);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    {
      // ------------------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      for (int tile = blockIdx.x; tile < g.num_tiles && !flag_set_warp(abort_flag);
           tile += gridDim.x) {
        int tm, tn;
        tile_coords(tile, g, tm, tn);
        bool ok = true;
        for (int kt = 0; kt < g.k_tiles; ++kt) {
          if (!mbar_wait_warp(&empty[stage], phase ^ 1u, g.wait_limit_ns)) {
            ok = false;
            break;
          }
          if (elect_one_sync()) {
            mbar_arrive_expect_tx(&full[stage], Cfg::kStageBytes);
            tma_load_2d(sA + stage * kGABytes, &tmA, &full[stage], kt * (kGBK / 2), tm * kGBM);
            tma_load_2d(sB + stage * kGBBytes, &tmB, &full[stage], kt * (kGBK / 2), tn * kGBN);
            tma_load_2d(sSFA + stage * Cfg::kSFABytes, &tmSFA, &full[stage],
                        kt * Cfg::kAtoms * 64, tm);
            tma_load_2d(sSFB + stage * Cfg::kSFBBytes, &tmSFB, &full[stage],
                        kt * Cfg::kAtoms * 64, tn * 2);
          }
          __syncwarp();
          if (++stage == kGStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) {
          *abort_flag = 1;
          break;
        }
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------- scale copies + MMAs
    SingleIssuer::run(tmem, sA, sB, sSFA, sSFB, full, empty, acc_full, acc_empty, abort_flag,
                      blockIdx.x, gridDim.x, ArgsSched{g});
  } else {
    // -------------------------------------------------------------- epilogue
    const int ew = warp - 2;
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int half = ew >> 2;      // accumulator columns [128*half, 128*half + 128)
    float alpha = 1.0f;
    if constexpr (FMT == kFmtNV) alpha = __fmul_rn(*g.sa, *g.sb);
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < g.num_tiles && !*abort_flag; tile += gridDim.x) {
      int tm, tn;
      tile_coords(tile, g, tm, tn);
      if (!mbar_wait(acc_full, acc_phase, g.wait_limit_ns)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      uint32_t r[128];
      tmem_ld_32x32b_x128(tmem + (static_cast<uint32_t>(32 * quarter) << 16) + 128 * half, r);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
      acc_phase ^= 1u;

      store_row_segment<FMT, OUT_BF16>(r, tm * kGBM + 32 * quarter + lane, tn * kGBN + 128 * half,
                                       g, alpha);
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}


// ====================================================================================
// CTA-pair variant (cta_group::2): a cluster of two CTAs on two SMs computes a 256x256
// output tile. Each CTA stages its own 128 rows of A and its own 128-row half of B
// (plus the scales of all 256 B rows, which both tensor cores need), so each SM pulls
// a third less operand data per flop from L2 than the single-CTA kernel, and the
// smaller stages allow a deeper ring. CTA rank 0 of the pair (the leader) issues the
// pair-wide MMAs; both CTAs load through TMA into their own shared memory with the
// transfers counted on the leader's barrier, and both drain their own half of the
// accumulator (rows 128*rank ... +128, all 256 columns) from their own TMEM.
// Roles: warp 0 of both CTAs loads; in the leader, warp 1 issues each slab's scale
// copies and then its MMAs (Issuer::run); warps 2-9 of both CTAs run the epilogue.
// The loads carry no multicast; only the tcgen05.commit arrivals are multicast to the
// two CTAs of the pair.
template <int FMT>
struct PairCfg {
  static constexpr int kBlock = FMT == kFmtNV ? 16 : 32;
  // K per stage: 256 for MXFP4 (4 MMAs per barrier wait and commit, 6 stages) and NVFP4
  // (5 stages), 256 for MXFP8 (the same 256 code bytes per row as 512 K of MXFP4, 8 MMAs
  // of K = 32; 3 stages). The mainloop is bound by how long a stage stays occupied (load
  // latency + MMAs), not by barrier waits: six 35 KB MXFP4 stages keep the same bytes in
  // flight as three 70 KB ones but free each after 512 MMA cycles instead of 1024
  // (measured 5165 -> 5396 TFLOP/s over the Llama layer's GEMMs).
  static constexpr int kSlabK = 256;
  static constexpr int kRowBytes = FMT == kFmtMX8 ? kSlabK : kSlabK / 2;  // code bytes/row
  static constexpr int kSub = kRowBytes / 128;       // 128-byte-wide swizzled sub-tiles
  static constexpr int kAtoms = kSlabK / (4 * kBlock);
  static constexpr int kABytes = 128 * kRowBytes;    // this CTA's 128 rows of A
  static constexpr int kBBytes = 128 * kRowBytes;    // this CTA's 128-row half of B
  static constexpr int kSFABytes = kAtoms * 512;     // scales of this CTA's A rows
  static constexpr int kSFBBytes = 2 * kAtoms * 512; // scales of all 256 B rows
  static constexpr int kStageBytes = kABytes + kBBytes + kSFABytes + kSFBBytes;
  static constexpr int kStages = FMT == kFmtNV ? 5 : (FMT == kFmtMX ? 6 : 3);
  // Every format issues a slab's scale copies from the MMA warp, in order before its MMAs
  // (Issuer::run). With the issuing roles run as whole warps the issue is cheap; copy
  // warps of their own, handing each slab to the MMA warp through a barrier, measured
  // slower (the Llama layer's GEMMs: MXFP4 -2.0%, NVFP4 -5.4%).
  static constexpr int kThreads = kGThreads;
  static constexpr int kSFCols = 12 * kAtoms;
  // At least one ring slot per stage (the ring's reuse rule, Issuer): 5 x 48 columns for
  // NVFP4, 6 x 24 for MXFP4, 4 x 24 for MXFP8, after the 256 accumulator columns.
  static constexpr int kSFBufs = kStages > 4 ? kStages : 4;
  static constexpr int kTmemSF = 256;
  static_assert(kTmemSF + kSFBufs * kSFCols <= 512, "TMEM columns");
  // 1 KB of output staging per epilogue warp (store_segment_tma, fp32 outputs) after the
  // barriers.
  static constexpr int kStagingBytes = 8 * 1024;
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + 256 + kStagingBytes;
};


// The kernel runs a group of GEMMs (one problem for fp4_gemm); each tile's problem gives
// its operand maps, coordinates, K, output type and (NVFP4) tensor scales.
// QHN >= 0: the epilogue of the group's member with q_codes set also quantises its
// output (store_row_segment_quant, rotation QHN along N); the other members store as
// usual.
template <int FMT, int QHN = -1>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfg<FMT>::kThreads, 1)
    gemm_fp4_pair_kernel(const __grid_constant__ GemmGroup grp) {
  using Cfg = PairCfg<FMT>;
  constexpr int S = Cfg::kStages;
  using PairIssuer = Issuer<FMT, true, Cfg::kSlabK, S, Cfg::kABytes, Cfg::kBBytes,
                            Cfg::kSFABytes, Cfg::kSFBBytes, Cfg::kSFCols, Cfg::kSFBufs>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + S * Cfg::kABytes;
  uint8_t* sSFA = sB + S * Cfg::kBBytes;
  uint8_t* sSFB = sSFA + S * Cfg::kSFABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sSFB + S * Cfg::kSFBBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* acc_full = bars + 2 * S;
  uint64_t* acc_empty = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  static_assert((2 * S + 2) * 8 + 8 <= 256, "barrier area");
  uint8_t* s_stage_out = reinterpret_cast<uint8_t*>(bars) + 256;  // [8 warps][1 KB]
  const GroupSched sched{grp};
  const uint64_t wait_ns = grp.p[0].g.wait_limit_ns;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int q = 0; q < grp.n; ++q) {
      tma_prefetch_desc(&grp.p[q].a);
      tma_prefetch_desc(&grp.p[q].b);
      tma_prefetch_desc(&grp.p[q].sa);
      tma_prefetch_desc(&grp.p[q].sb);
      if (QHN < 0 && !grp.p[q].out_bf16) tma_prefetch_desc(&grp.p[q].c);
    }
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 16);  // 8 epilogue warps in each CTA of the pair
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t leader_full = mapa_shared(smem_u32(full), 0);
  const uint32_t leader_acc_empty = mapa_shared(smem_u32(acc_empty), 0);

  if (warp == 0) {
    {
      // ------------------------------------------------------------ TMA producer (both CTAs)
      int stage = 0;
      uint32_t phase = 0;
      for (int tile = pair; tile < grp.num_tiles && !flag_set_warp(abort_flag); tile += npairs) {
        const GemmProblem& P = grp.p[group_problem(grp, tile)];
        int tm, tn;
        tile_coords(tile - P.tile0, P.g, tm, tn);
        bool ok = true;
        for (int kt = 0; kt < P.g.k_tiles; ++kt) {
          if (!mbar_wait_warp(&empty[stage], phase ^ 1u, wait_ns)) {
            ok = false;
            break;
          }
          if (elect_one_sync()) {
            if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * Cfg::kStageBytes);
            const uint32_t bar = leader_full + 8u * stage;
#pragma unroll
            for (int sub = 0; sub < Cfg::kSub; ++sub) {
              const int kx = kt * Cfg::kRowBytes + 128 * sub;
              tma_load_2d_pair(sA + stage * Cfg::kABytes + sub * 16384, &P.a, bar, kx,
                               tm * 256 + 128 * static_cast<int>(rank));
              tma_load_2d_pair(sB + stage * Cfg::kBBytes + sub * 16384, &P.b, bar, kx,
                               tn * 256 + 128 * static_cast<int>(rank));
            }
            tma_load_2d_pair(sSFA + stage * Cfg::kSFABytes, &P.sa, bar, kt * Cfg::kAtoms * 64,
                             2 * tm + static_cast<int>(rank));
            tma_load_2d_pair(sSFB + stage * Cfg::kSFBBytes, &P.sb, bar, kt * Cfg::kAtoms * 64,
                             2 * tn);
          }
          __syncwarp();
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        if (!ok) {
          *abort_flag = 1;
          break;
        }
      }
    }
  } else if (warp == 1) {
    if (rank == 0) {
      // ------------------------------------------------------ scale copies + MMAs (leader)
      PairIssuer::run(tmem, sA, sB, sSFA, sSFB, full, empty, acc_full, acc_empty, abort_flag,
                      pair, npairs, sched);
    }
  } else {
    // -------------------------------------------------------------- epilogue (both CTAs)
    const int ew = warp - 2;
    const int quarter = warp & 3;
    const int half = ew >> 2;
    uint32_t acc_phase = 0;
    for (int tile = pair; tile < grp.num_tiles && !*abort_flag; tile += npairs) {
      const GemmProblem& P = grp.p[group_problem(grp, tile)];
      int tm, tn;
      tile_coords(tile - P.tile0, P.g, tm, tn);
      float alpha = 1.0f;
      if constexpr (FMT == kFmtNV) alpha = __fmul_rn(*P.g.sa, *P.g.sb);
      if (!mbar_wait(acc_full, acc_phase, wait_ns)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      uint32_t r[128];
      tmem_ld_32x32b_x128(tmem + (static_cast<uint32_t>(32 * quarter) << 16) + 128 * half, r);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      // CTA-scope release: a cluster-scope release here would first wait for this thread's
      // earlier global stores (the previous tile's output) and stall the leader's MMAs by
      // about a microsecond per tile.
      if (lane == 0) mbar_arrive_cluster_cta_release(leader_acc_empty);
      acc_phase ^= 1u;
      const int row0 = tm * 256 + 128 * static_cast<int>(rank) + 32 * quarter;
      const int n0 = tn * kGBN + 128 * half;
      if constexpr (QHN >= 0) {
        if (P.g.q_codes != nullptr) {  // the group's member whose output is quantised too
          store_row_segment_quant<FMT, QHN>(r, row0 + lane, n0, P.g, alpha);
          continue;
        }
      }
      if (P.out_bf16)
        store_row_segment<FMT, 1>(r, row0 + lane, n0, P.g, alpha);
      else  // fp32: through TMA stores (store_segment_tma)
        store_segment_tma<FMT, 0>(r, s_stage_out + 1024 * ew, &P.c, row0, n0, P.g, alpha, lane);
    }
    // every store of this warp has completed before the CTA (and its staging) goes away
    if (lane == 0) bulk_wait<0>();
    __syncwarp();
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace fp4k

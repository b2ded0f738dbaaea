// gemm.cuh -- block-scaled FP4 GEMM on the sm_100a tensor cores.
//
//   C[M][N] = sum_k deq(A)[m][k] * deq(B)[n][k]   (both operands K-major, E2M1 packed)
//
// with deq = e2m1 * 2^(byte-127) (MXFP4, 32-element blocks) or e2m1 * ue4m3(byte)
// (NVFP4, 16-element blocks; the fp32 tensor scales S_A * S_B are applied in the
// epilogue). Accumulation is fp32 in tensor memory. [gist.science summary of arXiv
// 2605.09825, Methodology item 2 (all three GEMM passes in FP4); molayo1419.me
// NVFP4/MaxText page, Key facts bullet 5 (FP4 tensor cores on Blackwell).]
//
// Design (one CTA per SM, persistent over 128x256 output tiles, K in slabs of 256):
//   warp 0   : TMA producer. Per slab it loads A 128x128 B, B 256x128 B (128B swizzle)
//              and the matching 512-byte scale atoms into a 4-stage ring.
//   warp 1   : allocates 512 TMEM columns; one thread copies the slab's scale atoms
//              smem -> TMEM (tcgen05.cp 32x128b.warpx4) and issues 4 MMAs of
//              128x256x64 (tcgen05.mma kind::mxf4 / kind::mxf4nvf4), then commits
//              the stage back to the producer; after the last slab it commits the
//              accumulator to the epilogue.
//   warps 2-9: epilogue. Each warp owns one 32-lane quarter of TMEM and one half of
//              the 256 columns: it pulls its 32x128 fp32 block into registers,
//              releases the accumulator (so the next tile's MMAs start), then scales
//              and stores fp32 or bf16 rows to global memory.
// TMEM columns: [0,256) accumulator, then the scale factors of the current slab.
// No cluster multicast anywhere. Every wait is bounded (status word on expiry).
#pragma once

#include "common.cuh"

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
  static constexpr int kTmemSFA = 256;
  static constexpr int kTmemSFB = 256 + 4 * kAtoms;
  static constexpr int kSmemBytes = 1024 + kGStages * kStageBytes + 256;
};

struct GemmArgs {
  int M, N, K;
  int tiles_m, tiles_n, num_tiles, k_tiles;
  void* C;
  const float* sa;  // NVFP4 tensor scales (device), or null
  const float* sb;
  uint64_t wait_limit_ns;
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

template <int FMT, int OUT_BF16>
__global__ void __launch_bounds__(kGThreads, 1)
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
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      for (int tile = blockIdx.x; tile < g.num_tiles && !*abort_flag; tile += gridDim.x) {
        const int tm = tile % g.tiles_m, tn = tile / g.tiles_m;
        for (int kt = 0; kt < g.k_tiles; ++kt) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, g.wait_limit_ns) || *abort_flag) {
            *abort_flag = 1;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], Cfg::kStageBytes);
          tma_load_2d(sA + stage * kGABytes, &tmA, &full[stage], kt * (kGBK / 2), tm * kGBM);
          tma_load_2d(sB + stage * kGBBytes, &tmB, &full[stage], kt * (kGBK / 2), tn * kGBN);
          tma_load_2d(sSFA + stage * Cfg::kSFABytes, &tmSFA, &full[stage], kt * Cfg::kAtoms * 64,
                      tm);
          tma_load_2d(sSFB + stage * Cfg::kSFBBytes, &tmSFB, &full[stage], kt * Cfg::kAtoms * 64,
                      tn * 2);
          if (++stage == kGStages) { stage = 0; phase ^= 1u; }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      for (int tile = blockIdx.x; tile < g.num_tiles && !*abort_flag; tile += gridDim.x) {
        if (!mbar_wait(acc_empty, acc_phase ^ 1u, g.wait_limit_ns)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        bool ok = true;
        for (int kt = 0; kt < g.k_tiles; ++kt) {
          if (!mbar_wait(&full[stage], phase, g.wait_limit_ns) || *abort_flag) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + stage * kGABytes);
          const uint32_t b_base = smem_u32(sB + stage * kGBBytes);
          const uint32_t sfa = smem_u32(sSFA + stage * Cfg::kSFABytes);
          const uint32_t sfb = smem_u32(sSFB + stage * Cfg::kSFBBytes);
#pragma unroll
          for (int at = 0; at < Cfg::kAtoms; ++at)
            tc_cp_32x128b_warpx4(tmem + Cfg::kTmemSFA + 4 * at, desc_sf_atom(sfa + 512 * at));
#pragma unroll
          for (int rb = 0; rb < 2; ++rb)
#pragma unroll
            for (int at = 0; at < Cfg::kAtoms; ++at)
              tc_cp_32x128b_warpx4(tmem + Cfg::kTmemSFB + 8 * at + 4 * rb,
                                   desc_sf_atom(sfb + rb * Cfg::kSFABytes + 512 * at));
#pragma unroll
          for (int j = 0; j < kGBK / 64; ++j) {
            // MXFP4: two MMAs share one atom column, bytes {0,1} then {2,3} (scale id 0/2);
            // NVFP4: one atom column per MMA, all four bytes (scale id 0).
            const int at = FMT == kFmtMX ? (j >> 1) : j;
            const uint32_t id = FMT == kFmtMX ? static_cast<uint32_t>((j & 1) * 2) : 0u;
            const uint32_t tsfa = (tmem + Cfg::kTmemSFA + 4 * at) | (id << 30);
            const uint32_t tsfb = (tmem + Cfg::kTmemSFB + 8 * at) | (id << 30);
            const uint32_t idesc = idesc_fp4<FMT>() | (id << 29) | (id << 4);
            tc_mma_fp4<FMT == kFmtMX>(tmem, desc_kmajor_sw128(a_base + 32 * j),
                                      desc_kmajor_sw128(b_base + 32 * j), idesc, tsfa, tsfb,
                                      (kt | j) != 0 ? 1u : 0u);
          }
          tc_commit(&empty[stage]);
          if (++stage == kGStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(acc_full);
        acc_phase ^= 1u;
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int ew = warp - 2;
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int half = ew >> 2;      // accumulator columns [128*half, 128*half + 128)
    float alpha = 1.0f;
    if constexpr (FMT == kFmtNV) alpha = __fmul_rn(*g.sa, *g.sb);
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < g.num_tiles && !*abort_flag; tile += gridDim.x) {
      const int tm = tile % g.tiles_m, tn = tile / g.tiles_m;
      if (!mbar_wait(acc_full, acc_phase, g.wait_limit_ns)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      uint32_t r[4][32];
      const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * quarter) << 16) + 128 * half;
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(taddr + 32 * c, r[c]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
      acc_phase ^= 1u;

      const int m = tm * kGBM + 32 * quarter + lane;
      const int n0 = tn * kGBN + 128 * half;
      if (m < g.M) {
        if constexpr (OUT_BF16) {
          __nv_bfloat16* crow = static_cast<__nv_bfloat16*>(g.C) + static_cast<int64_t>(m) * g.N + n0;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            if (n0 + 32 * c < g.N) {
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                uint32_t w[4];
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                  float x0 = __uint_as_float(r[c][8 * i + 2 * p]);
                  float x1 = __uint_as_float(r[c][8 * i + 2 * p + 1]);
                  if constexpr (FMT == kFmtNV) { x0 = __fmul_rn(x0, alpha); x1 = __fmul_rn(x1, alpha); }
                  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
                  w[p] = *reinterpret_cast<const uint32_t*>(&h);
                }
                *reinterpret_cast<uint4*>(crow + 32 * c + 8 * i) = make_uint4(w[0], w[1], w[2], w[3]);
              }
            }
          }
        } else {
          float* crow = static_cast<float*>(g.C) + static_cast<int64_t>(m) * g.N + n0;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            if (n0 + 32 * c < g.N) {
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                float4 o;
                o.x = __uint_as_float(r[c][4 * i + 0]);
                o.y = __uint_as_float(r[c][4 * i + 1]);
                o.z = __uint_as_float(r[c][4 * i + 2]);
                o.w = __uint_as_float(r[c][4 * i + 3]);
                if constexpr (FMT == kFmtNV) {
                  o.x = __fmul_rn(o.x, alpha); o.y = __fmul_rn(o.y, alpha);
                  o.z = __fmul_rn(o.z, alpha); o.w = __fmul_rn(o.w, alpha);
                }
                *reinterpret_cast<float4*>(crow + 32 * c + 4 * i) = o;
              }
            }
          }
        }
      }
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

}  // namespace fp4k

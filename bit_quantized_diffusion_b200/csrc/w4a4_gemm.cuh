// w4a4_gemm.cuh -- steps a5..a6: the NVFP4 4-bit GEMM on tcgen05 block-scaled
// MMA (kind::mxf4nvf4, one UE4M3 scale per 16 along K), with the low-rank
// up-projection (x_hat L1) L2 and the bias accumulated into the same
// tensor-memory accumulator, so the 16-bit branch never round-trips HBM
// (Nunchaku README, "Engine design" (b): up projection and 4-bit compute share
// the output).
//
// Persistent kernel: one CTA per SM walks 128 x 256 output tiles. Warp roles
// (14 warps):
//   warp 0      TMA producer: A/B code tiles [rows x 128 B] with 128-byte swizzle,
//               A/B scale atoms by plain bulk copies, L2 chunks [32 x 256] bf16;
//               runs ahead across tiles through a 3-stage ring
//   warp 1      tensor-memory owner and MMA issuer (one thread)
//   warps 2-5   low-rank staging: xl1 (float32) as bf16 hi + lo operand tiles
//               for the up-projection MMAs
// Each tile is a sequence of ring slots: K/256 FP4 slots, then ceil(r/32)
// low-rank slots holding an L2 chunk (by TMA) and the matching xl1 hi/lo tiles
// (by the staging warps). Every slot's "full" barrier counts the producer and
// the four staging warps, so both kinds of slot flow through one pipeline.
//   warps 6-13  epilogue, two warps per tensor-memory lane quadrant (one per
//               128-column half): accumulator -> + bias -> bf16 / f32 -> swizzled
//               shared-memory staging -> TMA store (coalesced, asynchronous)
// Two 256-column accumulators share tensor memory with a 64-column overlap
// ([0, 256) and [192, 448)); scale factors sit in [448, 496). The epilogue
// drains the overlapped columns of a tile first and releases them, so the next
// tile's MMAs start while the rest of the tile is still being stored.
#pragma once

#include "sm100.cuh"

namespace svdq {

constexpr int kGmThreads = 448;
constexpr int kGmEpiWarps = 8;
constexpr int kGmStageOut = 4096;                // epilogue staging bytes per warp
constexpr int kGmBM = 128, kGmBN = 256;
constexpr int kGmBKBytes = 128;  // 256 FP4 values per row per stage
constexpr int kGmAStage = kGmBM * kGmBKBytes;   // 16 KB
constexpr int kGmBStage = kGmBN * kGmBKBytes;   // 32 KB
constexpr int kGmSfaStage = 4 * 512;            // 4 atoms (one per 64-wide K block)
constexpr int kGmSfbStage = 2 * 4 * 512;        // 2 row blocks x 4 atoms
constexpr int kGmStageBytes = kGmAStage + kGmBStage + kGmSfaStage + kGmSfbStage;  // 54 KB
constexpr int kGmStages = 3;
constexpr int kGmLrK = 32;                                // low-rank K per ring slot
constexpr int kGmLrBTile = kGmLrK * kGmBN * 2;            // 16 KB, slot offset 0
constexpr int kGmLrATile = kGmBM * kGmLrK * 2;            // 8 KB per bf16 tile (hi, lo)
// tensor-memory columns
constexpr uint32_t kTmAcc1 = 192, kTmOverlap = 64, kTmSfa = 448, kTmSfb = 464, kTmCols = 512;

struct GemmParams {
  int M, N, K, r;
  int tiles_m, tiles;
  const uint8_t* a_scales;
  const uint8_t* w_scales;
  const float* xl1;
  const __nv_bfloat16* bias;
  void* Y;
  int ldy;
  int out_f32;
  uint32_t* status;
};

struct GmSmem {
  uint32_t ring, out, bias, bars, tmem_slot, total;
};

__host__ __device__ constexpr GmSmem gm_smem_layout() {
  GmSmem s{};
  s.ring = 0;
  s.out = kGmStages * kGmStageBytes;         // 1024-aligned (54 KB multiples)
  s.bias = s.out + kGmEpiWarps * kGmStageOut;  // 128 floats per epilogue warp
  s.bars = s.bias + kGmEpiWarps * 128 * 4;
  s.tmem_slot = s.bars + 8 * (2 * kGmStages + 2);
  s.total = s.tmem_slot + 16;
  return s;
}

constexpr size_t kGmSmemBytes = gm_smem_layout().total + 1024;

__global__ void __launch_bounds__(kGmThreads, 1)
    w4a4_nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tm_a,
                           const __grid_constant__ CUtensorMap tm_b,
                           const __grid_constant__ CUtensorMap tm_l2,
                           const __grid_constant__ CUtensorMap tm_y, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  constexpr GmSmem L = gm_smem_layout();
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  const int kblocks = p.K / 64;                      // 64-wide scale atoms along K
  const int ktiles = (kblocks + 3) / 4;
  const int lr_chunks = p.r / kGmLrK + ((p.r % kGmLrK) ? 1 : 0);
  // this CTA's tiles: blockIdx.x, blockIdx.x + gridDim.x, ...; M fastest
  const int my_tiles = p.tiles > static_cast<int>(blockIdx.x)
                           ? (p.tiles - 1 - static_cast<int>(blockIdx.x)) / gridDim.x + 1
                           : 0;
  auto tile_mn = [&](int i, int& m0, int& n0) {
    const int t = blockIdx.x + i * gridDim.x;
    m0 = (t % p.tiles_m) * kGmBM;
    n0 = (t / p.tiles_m) * kGmBN;
  };

  auto stage = [&](int s) { return sbase + L.ring + s * kGmStageBytes; };
  auto a_st = [&](int s) { return stage(s); };
  auto b_st = [&](int s) { return stage(s) + kGmAStage; };
  auto sfa_st = [&](int s) { return stage(s) + kGmAStage + kGmBStage; };
  auto sfb_st = [&](int s) { return sfa_st(s) + kGmSfaStage; };
  auto bar_full = [&](int s) { return sbase + L.bars + 8 * s; };
  auto bar_empty = [&](int s) { return sbase + L.bars + 8 * (kGmStages + s); };
  const uint32_t bar_acc_full = sbase + L.bars + 8 * (2 * kGmStages);
  const uint32_t bar_acc_free = bar_acc_full + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.tmem_slot);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGmStages; ++s) {
      mbar_init(bar_full(s), 1 + 4);  // producer (with tx) + 4 staging warps
      mbar_init(bar_empty(s), 1);
    }
    mbar_init(bar_acc_full, 1);
    mbar_init(bar_acc_free, kGmEpiWarps);
    fence_barrier_init();
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    prefetch_tmap(&tm_y);
    if (p.r > 0) prefetch_tmap(&tm_l2);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      bool ok = true;
      int kt_global = 0;
      for (int i = 0; i < my_tiles && ok; ++i) {
        int m0, n0;
        tile_mn(i, m0, n0);
        const int n_tile = min(kGmBN, p.N - n0);
        const int n_sfb = n_tile > 128 ? 2 : 1;
        const int mb = m0 / 128;
        for (int kt = 0; kt < ktiles + lr_chunks && ok; ++kt, ++kt_global) {
          const int s = kt_global % kGmStages;
          ok = mbar_wait(bar_empty(s), ((kt_global / kGmStages) & 1) ^ 1, p.status);
          if (!ok) break;
          if (kt < ktiles) {
            const int nkb = min(4, kblocks - 4 * kt);
            mbar_arrive_expect_tx(bar_full(s), kGmAStage + kGmBStage + nkb * 512 * (1 + n_sfb));
            tma_load_2d(a_st(s), &tm_a, bar_full(s), kt * kGmBKBytes, m0);
            tma_load_2d(b_st(s), &tm_b, bar_full(s), kt * kGmBKBytes, n0);
            bulk_load(sfa_st(s), p.a_scales + (static_cast<size_t>(mb) * kblocks + 4 * kt) * 512,
                      nkb * 512, bar_full(s));
            for (int j = 0; j < n_sfb; ++j)
              bulk_load(sfb_st(s) + j * 2048,
                        p.w_scales + (static_cast<size_t>(n0 / 128 + j) * kblocks + 4 * kt) * 512,
                        nkb * 512, bar_full(s));
          } else {
            // low-rank slot: L2 rows [32 c, 32 c + 32) x columns [n0, n0 + 256),
            // four 64-wide boxes (rows past r read as zero)
            const int c = kt - ktiles;
            mbar_arrive_expect_tx(bar_full(s), kGmLrBTile);
            for (int nb = 0; nb < 4; ++nb)
              tma_load_2d(stage(s) + nb * (kGmLrK * 128), &tm_l2, bar_full(s), n0 + nb * 64,
                          c * kGmLrK);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      bool ok = true;
      const uint32_t id_lr = idesc_bf16_f32(128, kGmBN, false, true);
      int kt_global = 0;
      for (int i = 0; i < my_tiles && ok; ++i) {
        int m0, n0;
        tile_mn(i, m0, n0);
        const int n_tile = min(kGmBN, p.N - n0);
        const int n_sfb = n_tile > 128 ? 2 : 1;
        const uint32_t acc = tmem + ((i & 1) ? kTmAcc1 : 0u);
        // the previous tile's epilogue has drained the overlapped columns
        if (i > 0) {
          ok = mbar_wait(bar_acc_free, (i - 1) & 1, p.status);
          if (!ok) break;
        }
        tc_fence_after();
        const uint32_t id_fp4 = idesc_nvfp4(128, n_tile);
        for (int kt = 0; kt < ktiles + lr_chunks && ok; ++kt, ++kt_global) {
          const int s = kt_global % kGmStages;
          ok = mbar_wait(bar_full(s), (kt_global / kGmStages) & 1, p.status);
          if (!ok) break;
          tc_fence_after();
          if (kt < ktiles) {
            const int nkb = min(4, kblocks - 4 * kt);
            for (int kb = 0; kb < nkb; ++kb) {
              tc_cp_32x128b_warpx4(tmem + kTmSfa + 4 * kb,
                                   smem_desc(sfa_st(s) + kb * 512, 128, 128, kSwizzleNone));
              for (int j = 0; j < n_sfb; ++j)
                tc_cp_32x128b_warpx4(tmem + kTmSfb + 8 * kb + 4 * j,
                                     smem_desc(sfb_st(s) + j * 2048 + kb * 512, 128, 128,
                                               kSwizzleNone));
            }
            for (int kb = 0; kb < nkb; ++kb) {
              const uint64_t ad = smem_desc(a_st(s) + kb * 32, 16, 1024, kSwizzle128B);
              const uint64_t bd = smem_desc(b_st(s) + kb * 32, 16, 1024, kSwizzle128B);
              mma_nvfp4(acc, ad, bd, id_fp4, tmem + kTmSfa + 4 * kb, tmem + kTmSfb + 8 * kb,
                        (kt > 0 || kb > 0) ? 1u : 0u);
            }
          } else {
            // low-rank slot: B = L2 chunk (MN-major, 128-byte swizzle; 64-wide N
            // blocks 4096 B apart = LBO, 8-deep K groups 1024 B apart = SBO);
            // A = xl1 hi / lo (no-swizzle K-major: K-adjacent core matrices 128 B
            // apart = LBO, 8-row groups 512 B apart = SBO)
            const uint32_t a_hi = stage(s) + kGmLrBTile, a_lo = a_hi + kGmLrATile;
#pragma unroll
            for (int kk = 0; kk < kGmLrK / 16; ++kk) {
              const uint64_t bd = smem_desc(stage(s) + kk * 2048, kGmLrK * 128, 1024, kSwizzle128B);
              mma_f16(acc, smem_desc(a_hi + kk * 256, 128, 512, kSwizzleNone), bd, id_lr, 1u);
              mma_f16(acc, smem_desc(a_lo + kk * 256, 128, 512, kSwizzleNone), bd, id_lr, 1u);
            }
          }
          tc_commit(bar_empty(s));
        }
        tc_commit(bar_acc_full);
      }
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ low-rank staging
    const int quad = warp & 3;
    const int trow = quad * 32 + lane;
    bool ok = true;
    int kt_global = 0;
    for (int i = 0; i < my_tiles && ok; ++i) {
      int m0, n0;
      tile_mn(i, m0, n0);
      const int m = m0 + trow;
      for (int kt = 0; kt < ktiles + lr_chunks && ok; ++kt, ++kt_global) {
        const int s = kt_global % kGmStages;
        float v[kGmLrK];
        const int c = kt - ktiles;
        if (c >= 0) {
          // load before waiting: the global read overlaps the wait for the slot
          const float4* src = reinterpret_cast<const float4*>(p.xl1 + static_cast<size_t>(m) * p.r +
                                                              c * kGmLrK);
#pragma unroll
          for (int j = 0; j < kGmLrK / 4; ++j) {
            // rows past M and columns past r (r % 32 == 16) contribute zeros
            const float4 f = (m < p.M && c * kGmLrK + 4 * j < p.r) ? __ldg(src + j)
                                                                   : make_float4(0.f, 0.f, 0.f, 0.f);
            v[4 * j] = f.x; v[4 * j + 1] = f.y; v[4 * j + 2] = f.z; v[4 * j + 3] = f.w;
          }
        }
        ok = mbar_wait(bar_empty(s), ((kt_global / kGmStages) & 1) ^ 1, p.status);
        if (!ok) break;
        if (c >= 0) {
          const uint32_t a_hi = stage(s) + kGmLrBTile, a_lo = a_hi + kGmLrATile;
#pragma unroll
          for (int cm = 0; cm < kGmLrK / 8; ++cm) {
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float x0 = v[8 * cm + 2 * j], x1 = v[8 * cm + 2 * j + 1];
              const __nv_bfloat162 hb = __floats2bfloat162_rn(x0, x1);
              const float2 hf = __bfloat1622float2(hb);
              const __nv_bfloat162 lb = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
              hi[j] = *reinterpret_cast<const uint32_t*>(&hb);
              lo[j] = *reinterpret_cast<const uint32_t*>(&lb);
            }
            const uint32_t off = (trow >> 3) * 512 + cm * 128 + (trow & 7) * 16;
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a_hi + off), "r"(hi[0]),
                         "r"(hi[1]), "r"(hi[2]), "r"(hi[3])
                         : "memory");
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a_lo + off), "r"(lo[0]),
                         "r"(lo[1]), "r"(lo[2]), "r"(lo[3])
                         : "memory");
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_full(s));
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Each warp owns 4 of the tile's eight 32-column sub-tiles for its lane
    // quadrant. The two sub-tiles shared with the other accumulator ([192, 256)
    // of buffer 0, [0, 64) of buffer 1) come first, one in each half's warps, so
    // the next tile's MMAs are let in after a single tensor-memory load per warp.
    const int quad = warp & 3;          // tensor-memory lanes 32 quad .. 32 quad + 31
    const int half = (warp - 6) >> 2;   // 0 or 1
    const uint32_t out_buf = sbase + L.out + (warp - 6) * kGmStageOut;
    float* bias_s = reinterpret_cast<float*>(smem + L.bias) + (warp - 6) * 128;  // [4][32]
    bool ok = true;
    int stores = 0;
    for (int i = 0; i < my_tiles && ok; ++i) {
      int m0, n0;
      tile_mn(i, m0, n0);
      const int n_tile = min(kGmBN, p.N - n0);
      const bool odd = i & 1;
      const uint32_t t_row = tmem + (odd ? kTmAcc1 : 0u) + (static_cast<uint32_t>(quad * 32) << 16);
      // sub-tile order: the overlapped one, then three of the six others
      int sub_col[4];
      const int ovl = odd ? 0 : kGmBN - kTmOverlap;   // first overlapped column
      sub_col[0] = ovl + 32 * half;
      const int other0 = odd ? kTmOverlap : 0;        // first non-overlapped column
      for (int t = 0; t < 3; ++t) sub_col[1 + t] = other0 + 32 * (3 * half + t);
      // bias for this warp's sub-tiles, fetched before the accumulator is ready
      __syncwarp();
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int n = n0 + sub_col[t] + lane;
        bias_s[t * 32 + lane] = (p.bias != nullptr && n < p.N) ? __bfloat162float(p.bias[n]) : 0.0f;
      }
      __syncwarp();
      ok = mbar_wait(bar_acc_full, i & 1, p.status);
      if (!ok) break;
      tc_fence_after();
      for (int t = 0; t < 4; ++t) {
        const int j0 = sub_col[t];
        uint32_t acc[32];
        tmem_ld32(t_row + j0, acc);
        tmem_ld_wait();
        if (t == 0) {
          // this warp's overlapped columns are in registers: let the next tile's MMAs in
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_acc_free);
        }
        if (j0 >= n_tile) continue;  // warp-uniform
        float y[32];
        const float4* bv = reinterpret_cast<const float4*>(bias_s + t * 32);
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) {
          const float4 b = bv[q4];
          y[4 * q4 + 0] = __uint_as_float(acc[4 * q4 + 0]) + b.x;
          y[4 * q4 + 1] = __uint_as_float(acc[4 * q4 + 1]) + b.y;
          y[4 * q4 + 2] = __uint_as_float(acc[4 * q4 + 2]) + b.z;
          y[4 * q4 + 3] = __uint_as_float(acc[4 * q4 + 3]) + b.w;
        }
        // stage the warp's 32 x 32 sub-tile in the TMA store's swizzled layout
        uint32_t buf;
        if (p.out_f32) {
          buf = out_buf;  // one 4 KB buffer, rows of 128 B, 128-byte swizzle
          if (lane == 0) bulk_wait_read<0>();
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 8; ++c)
            asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(
                             buf + lane * 128 + ((c ^ (lane & 7)) << 4)),
                         "f"(y[4 * c]), "f"(y[4 * c + 1]), "f"(y[4 * c + 2]), "f"(y[4 * c + 3])
                         : "memory");
        } else {
          buf = out_buf + (stores & 1) * 2048;  // two 2 KB buffers, rows of 64 B, 64-byte swizzle
          if (lane == 0) bulk_wait_read<1>();
          __syncwarp();
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const __nv_bfloat162 b = __floats2bfloat162_rn(y[2 * j], y[2 * j + 1]);
            pk[j] = *reinterpret_cast<const uint32_t*>(&b);
          }
#pragma unroll
          for (int c = 0; c < 4; ++c)
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                             buf + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4)),
                         "r"(pk[4 * c]), "r"(pk[4 * c + 1]), "r"(pk[4 * c + 2]), "r"(pk[4 * c + 3])
                         : "memory");
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tm_y, buf, n0 + j0, m0 + quad * 32);
          bulk_commit();
        }
        ++stores;
      }
    }
    if (lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmCols);
  }
}

}  // namespace svdq

// w4a4_gemm.cuh -- steps a5..a6: the NVFP4 4-bit GEMM on tcgen05 block-scaled
// MMA (kind::mxf4nvf4, one UE4M3 scale per 16 along K), with the low-rank
// up-projection (x_hat L1) L2 and the bias accumulated into the same
// tensor-memory accumulator, so the 16-bit branch never round-trips HBM
// (Nunchaku README, "Engine design" (b): up projection and 4-bit compute share
// the output).
//
// Persistent kernel: one CTA per SM walks 128 x 256 output tiles. Warp roles
// (10 warps):
//   warp 0     TMA producer: A/B code tiles [rows x 128 B] with 128-byte swizzle,
//              A/B scale atoms by plain bulk copies, L2 chunks [32 x 256] bf16;
//              runs ahead across tiles through a 3-stage ring
//   warp 1     tensor-memory owner and MMA issuer (one thread)
//   warps 2-5  low-rank staging: xl1 (float32) of the next tile as bf16 hi + lo
//              operand tiles for the up-projection MMAs
//   warps 6-9  epilogue: accumulator -> + bias -> bf16 / f32 -> global memory
// Two 256-column accumulators share tensor memory with a 64-column overlap
// ([0, 256) and [192, 448)); scale factors sit in [448, 496). The epilogue
// drains the overlapped columns of a tile first and releases them, so the next
// tile's MMAs start while the rest of the tile is still being stored.
#pragma once

#include "sm100.cuh"

namespace svdq {

constexpr int kGmThreads = 320;
constexpr int kGmBM = 128, kGmBN = 256;
constexpr int kGmBKBytes = 128;  // 256 FP4 values per row per stage
constexpr int kGmAStage = kGmBM * kGmBKBytes;   // 16 KB
constexpr int kGmBStage = kGmBN * kGmBKBytes;   // 32 KB
constexpr int kGmSfaStage = 4 * 512;            // 4 atoms (one per 64-wide K block)
constexpr int kGmSfbStage = 2 * 4 * 512;        // 2 row blocks x 4 atoms
constexpr int kGmStageBytes = kGmAStage + kGmBStage + kGmSfaStage + kGmSfbStage;  // 54 KB
constexpr int kGmStages = 3;
constexpr int kGmLrK = 32;                                // low-rank K per chunk
constexpr int kGmLrATile = kGmBM * kGmLrK * 2;            // 8 KB per bf16 tile
constexpr int kGmLrBTile = kGmLrK * kGmBN * 2;            // 16 KB
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
  uint32_t ring, lr_a, lr_b, bars, tmem_slot, total;
};

__host__ __device__ constexpr GmSmem gm_smem_layout() {
  GmSmem s{};
  s.ring = 0;
  s.lr_b = kGmStages * kGmStageBytes;        // 1024-aligned (54 KB multiples)
  s.lr_a = s.lr_b + kGmLrBTile;
  s.bars = s.lr_a + 2 * kGmLrATile;
  s.tmem_slot = s.bars + 8 * (2 * kGmStages + 4);
  s.total = s.tmem_slot + 16;
  return s;
}

constexpr size_t kGmSmemBytes = gm_smem_layout().total + 1024;

__global__ void __launch_bounds__(kGmThreads, 1)
    w4a4_nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tm_a,
                           const __grid_constant__ CUtensorMap tm_b,
                           const __grid_constant__ CUtensorMap tm_l2, const GemmParams p) {
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
  const uint32_t bar_lr_full = sbase + L.bars + 8 * (2 * kGmStages);
  const uint32_t bar_lr_empty = bar_lr_full + 8;
  const uint32_t bar_acc_full = bar_lr_full + 16;
  const uint32_t bar_acc_free = bar_lr_full + 24;
  const uint32_t lr_b = sbase + L.lr_b;
  const uint32_t lr_hi = sbase + L.lr_a, lr_lo = lr_hi + kGmLrATile;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.tmem_slot);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGmStages; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_empty(s), 1);
    }
    mbar_init(bar_lr_full, 1 + 4);  // producer (with tx) + 4 staging warps
    mbar_init(bar_lr_empty, 1);
    mbar_init(bar_acc_full, 1);
    mbar_init(bar_acc_free, 4);     // 4 epilogue warps
    fence_barrier_init();
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
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
      int kt_global = 0, lr_global = 0;
      for (int i = 0; i < my_tiles && ok; ++i) {
        int m0, n0;
        tile_mn(i, m0, n0);
        const int n_tile = min(kGmBN, p.N - n0);
        const int n_sfb = n_tile > 128 ? 2 : 1;
        for (int c = 0; c < lr_chunks && ok; ++c, ++lr_global) {
          ok = mbar_wait(bar_lr_empty, (lr_global & 1) ^ 1, p.status);
          if (!ok) break;
          mbar_arrive_expect_tx(bar_lr_full, kGmLrBTile);
          for (int nb = 0; nb < 4; ++nb)
            tma_load_2d(lr_b + nb * 4096, &tm_l2, bar_lr_full, n0 + nb * 64, c * kGmLrK);
        }
        const int mb = m0 / 128;
        for (int kt = 0; kt < ktiles && ok; ++kt, ++kt_global) {
          const int s = kt_global % kGmStages;
          ok = mbar_wait(bar_empty(s), ((kt_global / kGmStages) & 1) ^ 1, p.status);
          if (!ok) break;
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
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      bool ok = true;
      const uint32_t id_lr = idesc_bf16_f32(128, kGmBN, false, true);
      int kt_global = 0, lr_global = 0;
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
        for (int c = 0; c < lr_chunks && ok; ++c, ++lr_global) {
          ok = mbar_wait(bar_lr_full, lr_global & 1, p.status);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kGmLrK / 16; ++kk) {
            // A (xl1 hi/lo): no-swizzle K-major, LBO 128 B (next 8 K), SBO 512 B (next 8 rows)
            const uint64_t ah = smem_desc(lr_hi + kk * 256, 128, 512, kSwizzleNone);
            const uint64_t al = smem_desc(lr_lo + kk * 256, 128, 512, kSwizzleNone);
            // B (L2 chunk): MN-major, 128-byte swizzle; 64-wide N blocks 4096 B apart
            // (LBO), 8-deep K groups 1024 B apart (SBO); 16 K = 2048 B.
            const uint64_t bd = smem_desc(lr_b + kk * 2048, 4096, 1024, kSwizzle128B);
            mma_f16(acc, ah, bd, id_lr, (c > 0 || kk > 0) ? 1u : 0u);
            mma_f16(acc, al, bd, id_lr, 1u);
          }
          tc_commit(bar_lr_empty);
        }
        const uint32_t id_fp4 = idesc_nvfp4(128, n_tile);
        for (int kt = 0; kt < ktiles && ok; ++kt, ++kt_global) {
          const int s = kt_global % kGmStages;
          ok = mbar_wait(bar_full(s), (kt_global / kGmStages) & 1, p.status);
          if (!ok) break;
          tc_fence_after();
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
                      (lr_chunks > 0 || kt > 0 || kb > 0) ? 1u : 0u);
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
    int lr_global = 0;
    for (int i = 0; i < my_tiles && ok; ++i) {
      int m0, n0;
      tile_mn(i, m0, n0);
      const int m = m0 + trow;
      for (int c = 0; c < lr_chunks && ok; ++c, ++lr_global) {
        // load before waiting: the global read overlaps the wait for the buffer
        float v[kGmLrK];
        const float4* src = reinterpret_cast<const float4*>(p.xl1 + static_cast<size_t>(m) * p.r +
                                                            c * kGmLrK);
#pragma unroll
        for (int j = 0; j < kGmLrK / 4; ++j) {
          // rows past M and columns past r (r % 32 == 16) contribute zeros
          const float4 f = (m < p.M && c * kGmLrK + 4 * j < p.r) ? __ldg(src + j)
                                                                 : make_float4(0.f, 0.f, 0.f, 0.f);
          v[4 * j] = f.x; v[4 * j + 1] = f.y; v[4 * j + 2] = f.z; v[4 * j + 3] = f.w;
        }
        ok = mbar_wait(bar_lr_empty, (lr_global & 1) ^ 1, p.status);
        if (!ok) break;
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
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(lr_hi + off), "r"(hi[0]),
                       "r"(hi[1]), "r"(hi[2]), "r"(hi[3])
                       : "memory");
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(lr_lo + off), "r"(lo[0]),
                       "r"(lo[1]), "r"(lo[2]), "r"(lo[3])
                       : "memory");
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_lr_full);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;
    const int trow = quad * 32 + lane;
    bool ok = true;
    for (int i = 0; i < my_tiles && ok; ++i) {
      int m0, n0;
      tile_mn(i, m0, n0);
      const int n_tile = min(kGmBN, p.N - n0);
      const int m = m0 + trow;
      const bool odd = i & 1;
      const uint32_t t_row = tmem + (odd ? kTmAcc1 : 0u) + (static_cast<uint32_t>(quad * 32) << 16);
      ok = mbar_wait(bar_acc_full, i & 1, p.status);
      if (!ok) break;
      tc_fence_after();
      // columns of this tile, in 16-wide chunks, starting with the 64 columns
      // shared with the other accumulator: [192, 256) of buffer 0, [0, 64) of buffer 1
      const int first = odd ? 0 : kGmBN - kTmOverlap;
      for (int step = 0; step < kGmBN / 16; ++step) {
        const int j0 = (first + step * 16) % kGmBN;
        uint32_t acc[16];
        tmem_ld16(t_row + j0, acc);
        tmem_ld_wait();
        if (step == kTmOverlap / 16 - 1) {
          // the overlapped columns are in registers: let the next tile's MMAs in
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_acc_free);
        }
        if (m >= p.M || j0 >= n_tile) continue;
        float y[16];
        const uint4* bsrc = reinterpret_cast<const uint4*>(p.bias + n0 + j0);
        if (p.bias != nullptr) {
          const uint4 b0 = __ldg(bsrc), b1 = __ldg(bsrc + 1);
          const uint32_t bw[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            y[2 * j] = __uint_as_float(acc[2 * j]) + __uint_as_float(bw[j] << 16);
            y[2 * j + 1] = __uint_as_float(acc[2 * j + 1]) + __uint_as_float(bw[j] & 0xFFFF0000u);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) y[j] = __uint_as_float(acc[j]);
        }
        if (p.out_f32) {
          float* dst = reinterpret_cast<float*>(p.Y) + static_cast<size_t>(m) * p.ldy + n0 + j0;
#pragma unroll
          for (int j = 0; j < 4; ++j)
            reinterpret_cast<float4*>(dst)[j] =
                make_float4(y[4 * j], y[4 * j + 1], y[4 * j + 2], y[4 * j + 3]);
        } else {
          uint32_t pk[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const __nv_bfloat162 b = __floats2bfloat162_rn(y[2 * j], y[2 * j + 1]);
            pk[j] = *reinterpret_cast<const uint32_t*>(&b);
          }
          __nv_bfloat16* dst =
              reinterpret_cast<__nv_bfloat16*>(p.Y) + static_cast<size_t>(m) * p.ldy + n0 + j0;
          reinterpret_cast<uint4*>(dst)[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          reinterpret_cast<uint4*>(dst)[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmCols);
  }
}

}  // namespace svdq

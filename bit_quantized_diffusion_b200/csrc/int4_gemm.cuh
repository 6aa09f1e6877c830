// int4_gemm.cuh -- steps a5..a6 for the INT4 format: symmetric int4 codes with
// one FP16 scale per 64 values along K, for both the activations and the
// residual weights (Diffusers blog, "quantization_config": svdq_w4a4 with
// precision int4, group_size 64), plus the low-rank up-projection and bias:
//
//   Y[m,n] = sum_g sa[m,g] sw[n,g] P_g[m,n] + sum_j xl1[m,j] L2[j,n] + bias[n]
//   P_g[m,n] = sum_{k in group g} qa[m,k] qw[n,k]
//
// sm_100a has no 4-bit integer MMA, and every group's partial product carries
// its own pair of FP16 scales, so the tensor cores produce one group at a time
// and the CUDA cores apply the scales:
//  - Tiled INT4 codes are sign-magnitude nibbles. A converter turns each into
//    the byte sign<<7 | magnitude, which is the E4M3 subnormal magnitude/512, so
//    kind::f8f6f4 computes P_g / 2^18 exactly in float32 (every product and
//    partial sum is a small multiple of 2^-18). The 2^18 is folded into the
//    weight scale.
//  - P_g goes to one of four 128-column tensor-memory buffers; rescale warps
//    read it and accumulate acc += sa * ((2^18 sw) * P) in float32 registers.
//  - The low-rank product (x_hat L1) L2 runs as bf16 hi/lo MMAs (kind::f16) into
//    a buffer of its own that the rescale warps add unscaled.
// The converter permutes K inside every 8-code word (even codes, then odd
// codes) the same way for A and B, which leaves each dot product unchanged.
//
// Persistent kernel, one CTA per SM, 128 x 128 output tiles, M fastest.
// Warp roles (14 warps):
//   warp 0      TMA producer: packed A/B codes [128 rows x 64 B] and the FP16
//               scales of both operands, two groups (K = 128) per stage
//   warp 1      tensor-memory owner and MMA issuer (one thread)
//   warps 2-5   converters: codes -> E4M3 operand tiles (128-byte swizzle) and
//               scales -> float32 scale ring; for a low-rank slot, the L2 chunk
//               by TMA and xl1 as bf16 hi + lo operand tiles
//   warps 6-13  rescale and epilogue, two per tensor-memory lane quadrant, 64
//               columns each: float32 accumulators in registers, + bias, bf16
//               or float32 stores straight to global memory
#pragma once

#include "sm100.cuh"

namespace svdq {

constexpr int kI4Threads = 448;
constexpr int kI4BM = 128, kI4BN = 128;
constexpr int kI4PackOp = 128 * 64;                        // packed codes, 128 K, one operand
constexpr int kI4PackScales = 2 * 128 * 2;                 // fp16 [2 groups][128 rows]
constexpr int kI4PackStage = 2 * kI4PackOp + 2 * kI4PackScales;  // 17 KB
constexpr int kI4PackStages = 4;
constexpr int kI4ExpOp = 128 * 128;                        // E4M3 operand tile, 128 K
constexpr int kI4ExpStage = 2 * kI4ExpOp;                  // 32 KB
constexpr int kI4ExpStages = 3;
constexpr int kI4PBufs = 4;                                // tensor-memory partial buffers
constexpr int kI4ScRing = 16;                              // groups of scales in flight
constexpr int kI4ScEntry = 2 * 128 * 4;                    // sa, 2^18 sw as float32
constexpr int kI4LrK = 32;                                 // low-rank K per slot
constexpr int kI4LrHi = 8192, kI4LrLo = 16384;             // xl1 planes inside a slot
constexpr uint32_t kI4OffExp = 0;
constexpr uint32_t kI4OffPack = kI4OffExp + kI4ExpStages * kI4ExpStage;
constexpr uint32_t kI4OffSc = kI4OffPack + kI4PackStages * kI4PackStage;
constexpr uint32_t kI4OffBias = kI4OffSc + kI4ScRing * kI4ScEntry;
constexpr uint32_t kI4OffBars = kI4OffBias + 8 * 64 * 4;
constexpr int kI4NumBars = 2 * kI4PackStages + 2 * kI4ExpStages + 2 * kI4PBufs + 2 * kI4ScRing;
constexpr uint32_t kI4OffTmem = kI4OffBars + 8 * kI4NumBars;
constexpr size_t kI4SmemBytes = kI4OffTmem + 16 + 1024;
static_assert(kI4PackStage % 1024 == 0 && kI4ExpStage % 1024 == 0, "1024-byte aligned stages");
static_assert(kI4LrLo + 128 * kI4LrK * 2 <= kI4ExpStage, "a low-rank slot fits in a stage");

struct I4Params {
  int M, N, K, r;
  int tiles_m, tiles;
  const float* xl1;
  const __nv_bfloat16* bias;
  void* Y;
  int ldy;
  int out_f32;
  uint32_t* status;
};

// The low nibble of each byte of w, a sign-magnitude code, as an E4M3 byte:
// sign to bit 7, magnitude to bits 0..2.
__device__ __forceinline__ uint32_t i4_even_e4m3(uint32_t w) {
  return (w & 0x07070707u) | ((w << 4) & 0x80808080u);
}
// The same for the high nibble of each byte of w.
__device__ __forceinline__ uint32_t i4_odd_e4m3(uint32_t w) {
  return ((w >> 4) & 0x07070707u) | (w & 0x80808080u);
}

// 14 warps: four of them share one of the SM's four 16K-register partitions,
// which caps the kernel at 128 registers per thread.
__global__ void __launch_bounds__(kI4Threads, 1)
    w4a4_int4_gemm_kernel(const __grid_constant__ CUtensorMap tm_a,
                          const __grid_constant__ CUtensorMap tm_b,
                          const __grid_constant__ CUtensorMap tm_sa,
                          const __grid_constant__ CUtensorMap tm_sw,
                          const __grid_constant__ CUtensorMap tm_l2, const I4Params p) {
  constexpr int NP = kI4PackStages, NE = kI4ExpStages, NB = kI4PBufs, NSC = kI4ScRing;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  const int G = p.K / 64;                                // scale groups along K
  const int kslots = (G + 1) / 2;                        // packed stages per tile
  const int lr_chunks = (p.r + kI4LrK - 1) / kI4LrK;     // low-rank slots per tile
  const int my_tiles =
      p.tiles > static_cast<int>(blockIdx.x) ? (p.tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  auto tile_mn = [&](int i, int& m0, int& n0) {
    const int t = blockIdx.x + i * gridDim.x;
    m0 = (t % p.tiles_m) * kI4BM;
    n0 = (t / p.tiles_m) * kI4BN;
  };
  auto pk = [&](int s) { return sbase + kI4OffPack + s * kI4PackStage; };
  auto ex = [&](int s) { return sbase + kI4OffExp + s * kI4ExpStage; };
  auto bar = [&](int i) { return sbase + kI4OffBars + 8 * i; };
  auto pk_full = [&](int s) { return bar(s); };
  auto pk_empty = [&](int s) { return bar(NP + s); };
  auto ex_full = [&](int s) { return bar(2 * NP + s); };
  auto ex_empty = [&](int s) { return bar(2 * NP + NE + s); };
  auto p_full = [&](int b) { return bar(2 * NP + 2 * NE + b); };
  auto p_free = [&](int b) { return bar(2 * NP + 2 * NE + NB + b); };
  auto sc_full = [&](int e) { return bar(2 * NP + 2 * NE + 2 * NB + e); };
  auto sc_empty = [&](int e) { return bar(2 * NP + 2 * NE + 2 * NB + NSC + e); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kI4OffTmem);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NP; ++s) {
      mbar_init(pk_full(s), 1);    // producer (with tx)
      mbar_init(pk_empty(s), 4);   // converter warps
    }
    for (int s = 0; s < NE; ++s) {
      mbar_init(ex_full(s), 4);    // converter warps (+ tx of a low-rank slot's L2 chunk)
      mbar_init(ex_empty(s), 1);   // MMA commit
    }
    for (int b = 0; b < NB; ++b) {
      mbar_init(p_full(b), 1);     // MMA commit
      mbar_init(p_free(b), 8);     // rescale warps
    }
    for (int e = 0; e < NSC; ++e) {
      mbar_init(sc_full(e), 4);    // converter warps
      mbar_init(sc_empty(e), 8);   // rescale warps
    }
    fence_barrier_init();
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    prefetch_tmap(&tm_sa);
    prefetch_tmap(&tm_sw);
    if (p.r > 0) prefetch_tmap(&tm_l2);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  cta_sync_converged();
  grid_dep_wait();  // the prologue above touches no global memory the previous grid may write
  grid_dep_launch();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      bool ok = true;
      int jp = 0;
      for (int i = 0; i < my_tiles && ok; ++i) {
        int m0, n0;
        tile_mn(i, m0, n0);
        for (int ks = 0; ks < kslots && ok; ++ks, ++jp) {
          const int s = jp % NP;
          ok = mbar_wait(pk_empty(s), ((jp / NP) & 1) ^ 1, p.status);
          if (!ok) break;
          // out-of-range rows, K bytes and groups arrive as zeros (full box bytes)
          mbar_arrive_expect_tx(pk_full(s), kI4PackStage);
          tma_load_2d(pk(s), &tm_a, pk_full(s), ks * 64, m0);
          tma_load_2d(pk(s) + kI4PackOp, &tm_b, pk_full(s), ks * 64, n0);
          tma_load_2d(pk(s) + 2 * kI4PackOp, &tm_sa, pk_full(s), m0, 2 * ks);
          tma_load_2d(pk(s) + 2 * kI4PackOp + kI4PackScales, &tm_sw, pk_full(s), n0, 2 * ks);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      bool ok = true;
      const uint32_t id8 = idesc_e4m3_f32(kI4BM, kI4BN);
      const uint32_t id16 = idesc_bf16_f32(kI4BM, kI4BN, false, true);
      int je = 0, pg = 0;
      for (int i = 0; i < my_tiles && ok; ++i) {
        for (int sl = 0; sl < kslots + lr_chunks && ok; ++sl, ++je) {
          const int s = je % NE;
          ok = mbar_wait(ex_full(s), (je / NE) & 1, p.status);
          if (!ok) break;
          tc_fence_after();
          const bool lr = sl >= kslots;
          const int ngroups = lr ? 1 : min(2, G - 2 * sl);
          for (int h = 0; h < ngroups && ok; ++h, ++pg) {
            const int b = pg % NB;
            ok = mbar_wait(p_free(b), ((pg / NB) & 1) ^ 1, p.status);
            if (!ok) break;
            tc_fence_after();
            const uint32_t d = tmem + b * 128;
            if (!lr) {
              // one group = 64 bytes of each 128-byte row = two K = 32 MMAs
#pragma unroll
              for (int kk = 0; kk < 2; ++kk) {
                const uint64_t ad = smem_desc(ex(s) + 64 * h + 32 * kk, 16, 1024, kSwizzle128B);
                const uint64_t bd =
                    smem_desc(ex(s) + kI4ExpOp + 64 * h + 32 * kk, 16, 1024, kSwizzle128B);
                mma_f8f6f4(d, ad, bd, id8, kk);
              }
            } else {
              // B = L2 chunk (MN-major, 128-byte swizzle: 64-wide N blocks 4096 B
              // apart = LBO, 8-deep K groups 1024 B apart = SBO); A = xl1 hi / lo
              // (no-swizzle K-major: K-adjacent core matrices 128 B apart = LBO,
              // 8-row groups 512 B apart = SBO)
#pragma unroll
              for (int kk = 0; kk < kI4LrK / 16; ++kk) {
                const uint64_t bd = smem_desc(ex(s) + kk * 2048, kI4LrK * 128, 1024, kSwizzle128B);
                const uint64_t ah = smem_desc(ex(s) + kI4LrHi + kk * 256, 128, 512, kSwizzleNone);
                const uint64_t al = smem_desc(ex(s) + kI4LrLo + kk * 256, 128, 512, kSwizzleNone);
                mma_f16(d, ah, bd, id16, kk);
                mma_f16(d, al, bd, id16, 1u);
              }
            }
            tc_commit(p_full(b));
          }
          tc_commit(ex_empty(s));
        }
      }
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ converters
    const int ct = threadIdx.x - 64;  // 0..127
    bool ok = true;
    int jp = 0, je = 0, jg = 0;
    for (int i = 0; i < my_tiles && ok; ++i) {
      int m0, n0;
      tile_mn(i, m0, n0);
      for (int sl = 0; sl < kslots + lr_chunks && ok; ++sl, ++je) {
        const int s = je % NE;
        if (sl < kslots) {
          const int ps = jp % NP;
          ok = mbar_wait(pk_full(ps), (jp / NP) & 1, p.status) &&
               mbar_wait(ex_empty(s), ((je / NE) & 1) ^ 1, p.status);
          if (!ok) break;
          const uint8_t* src = smem + (pk(ps) - sbase);
          // 2 operands x 128 rows x 4 chunks of 16 packed bytes; each chunk
          // becomes 32 E4M3 bytes = two 16-byte units of the swizzled row
#pragma unroll 4
          for (int t = 0; t < 8; ++t) {
            const int item = ct + 128 * t;
            const int op = item >> 9;
            const int row = (item >> 2) & 127;
            const int c = item & 3;
            const uint4 w = *reinterpret_cast<const uint4*>(src + op * kI4PackOp + row * 64 + c * 16);
            const uint32_t rowp = ex(s) + op * kI4ExpOp + row * 128;
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                             rowp + (((2 * c) ^ (row & 7)) << 4)),
                         "r"(i4_even_e4m3(w.x)), "r"(i4_odd_e4m3(w.x)), "r"(i4_even_e4m3(w.y)),
                         "r"(i4_odd_e4m3(w.y))
                         : "memory");
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                             rowp + (((2 * c + 1) ^ (row & 7)) << 4)),
                         "r"(i4_even_e4m3(w.z)), "r"(i4_odd_e4m3(w.z)), "r"(i4_even_e4m3(w.w)),
                         "r"(i4_odd_e4m3(w.w))
                         : "memory");
          }
          // the slot's scales as float32, the weight's times 2^18 (exact)
          const int ngroups = min(2, G - 2 * sl);
          const __half* sa = reinterpret_cast<const __half*>(src + 2 * kI4PackOp);
          const __half* sw = reinterpret_cast<const __half*>(src + 2 * kI4PackOp + kI4PackScales);
          for (int h = 0; h < ngroups && ok; ++h, ++jg) {
            const int e = jg % NSC;
            ok = mbar_wait(sc_empty(e), ((jg / NSC) & 1) ^ 1, p.status);
            if (!ok) break;
            float* ring = reinterpret_cast<float*>(smem + kI4OffSc + e * kI4ScEntry);
            ring[ct] = __half2float(sa[h * 128 + ct]);
            ring[128 + ct] = __half2float(sw[h * 128 + ct]) * 262144.0f;
            __syncwarp();
            if (lane == 0) mbar_arrive(sc_full(e));
          }
          if (!ok) break;
          fence_proxy_async_smem();  // generic writes -> tensor-core reads
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(ex_full(s));
            mbar_arrive(pk_empty(ps));
          }
          ++jp;
        } else {
          ok = mbar_wait(ex_empty(s), ((je / NE) & 1) ^ 1, p.status);
          if (!ok) break;
          const int c = sl - kslots;
          if (ct == 0) {
            // rows past r and columns past N arrive as zeros (full box bytes)
            mbar_expect_tx(ex_full(s), kI4LrK * kI4BN * 2);
            for (int nb = 0; nb < kI4BN / 64; ++nb)
              tma_load_2d(ex(s) + nb * 4096, &tm_l2, ex_full(s), n0 + nb * 64, c * kI4LrK);
          }
          // xl1 row m0 + ct, columns 32c..32c+31, as bf16 hi + lo
          const int m = m0 + ct;
          float v[kI4LrK];
          const float4* srcx =
              reinterpret_cast<const float4*>(p.xl1 + static_cast<size_t>(m) * p.r + c * kI4LrK);
#pragma unroll
          for (int j = 0; j < kI4LrK / 4; ++j) {
            const float4 f = (m < p.M && c * kI4LrK + 4 * j < p.r) ? __ldg(srcx + j)
                                                                   : make_float4(0.f, 0.f, 0.f, 0.f);
            v[4 * j] = f.x;
            v[4 * j + 1] = f.y;
            v[4 * j + 2] = f.z;
            v[4 * j + 3] = f.w;
          }
#pragma unroll
          for (int cm = 0; cm < kI4LrK / 8; ++cm) {
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
            const uint32_t off = (ct >> 3) * 512 + cm * 128 + (ct & 7) * 16;
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(ex(s) + kI4LrHi + off),
                         "r"(hi[0]), "r"(hi[1]), "r"(hi[2]), "r"(hi[3])
                         : "memory");
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(ex(s) + kI4LrLo + off),
                         "r"(lo[0]), "r"(lo[1]), "r"(lo[2]), "r"(lo[3])
                         : "memory");
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(ex_full(s));
        }
      }
    }
  } else {
    // ------------------------------------------------------------ rescale + epilogue
    const int quad = warp & 3;          // tensor-memory lanes 32 quad .. 32 quad + 31
    const int half = (warp - 6) >> 2;   // columns 64 half .. 64 half + 63 of the tile
    const int row = quad * 32 + lane;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quad * 32) << 16) + half * 64;
    float* bias_s = reinterpret_cast<float*>(smem + kI4OffBias) + (warp - 6) * 64;
    bool ok = true;
    int pg = 0, jg = 0;
    for (int i = 0; i < my_tiles && ok; ++i) {
      int m0, n0;
      tile_mn(i, m0, n0);
      __syncwarp();
      for (int c = lane; c < 64; c += 32) {
        const int n = n0 + half * 64 + c;
        bias_s[c] = (p.bias != nullptr && n < p.N) ? __bfloat162float(p.bias[n]) : 0.0f;
      }
      __syncwarp();
      uint64_t acc[32];  // 64 float32 accumulators as pairs
#pragma unroll
      for (int q = 0; q < 32; ++q) acc[q] = 0ull;
      for (int g = 0; g < G + lr_chunks && ok; ++g, ++pg) {
        const int b = pg % NB;
        ok = mbar_wait(p_full(b), (pg / NB) & 1, p.status);
        if (!ok) break;
        tc_fence_after();
        if (g < G) {
          const int e = jg % NSC;
          ok = mbar_wait(sc_full(e), (jg / NSC) & 1, p.status);
          if (!ok) break;
          const float* ring = reinterpret_cast<const float*>(smem + kI4OffSc + e * kI4ScEntry);
          const float sa = ring[row];
          const uint64_t sa2 = f2_pack(sa, sa);
          const float4* sw4 = reinterpret_cast<const float4*>(ring + 128 + half * 64);
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t v[16];
            tmem_ld16(t_lane + b * 128 + cc * 16, v);
            tmem_ld_wait();
            if (cc == 3) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(p_free(b));
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float4 w = sw4[cc * 4 + q];
              const uint64_t p0 = f2_pack(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]));
              const uint64_t p1 =
                  f2_pack(__uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
              acc[cc * 8 + 2 * q] = f2_fma(f2_mul(p0, f2_pack(w.x, w.y)), sa2, acc[cc * 8 + 2 * q]);
              acc[cc * 8 + 2 * q + 1] =
                  f2_fma(f2_mul(p1, f2_pack(w.z, w.w)), sa2, acc[cc * 8 + 2 * q + 1]);
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(sc_empty(e));
          ++jg;
        } else {
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t v[16];
            tmem_ld16(t_lane + b * 128 + cc * 16, v);
            tmem_ld_wait();
            if (cc == 3) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(p_free(b));
            }
#pragma unroll
            for (int q = 0; q < 8; ++q)
              acc[cc * 8 + q] =
                  f2_add(acc[cc * 8 + q],
                         f2_pack(__uint_as_float(v[2 * q]), __uint_as_float(v[2 * q + 1])));
          }
        }
      }
      if (!ok) break;
      // epilogue: + bias, then this thread's 64 columns of row m
      const int m = m0 + row;
      if (m < p.M) {
        const int nbase = n0 + half * 64;
        if (p.out_f32) {
          float* y = static_cast<float*>(p.Y) + static_cast<size_t>(m) * p.ldy + nbase;
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            if (nbase + 4 * q >= p.N) break;
            const float2 a = f2_unpack(acc[2 * q]), c = f2_unpack(acc[2 * q + 1]);
            *reinterpret_cast<float4*>(y + 4 * q) =
                make_float4(a.x + bias_s[4 * q], a.y + bias_s[4 * q + 1], c.x + bias_s[4 * q + 2],
                            c.y + bias_s[4 * q + 3]);
          }
        } else {
          __nv_bfloat16* y = static_cast<__nv_bfloat16*>(p.Y) + static_cast<size_t>(m) * p.ldy + nbase;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            if (nbase + 8 * q >= p.N) break;
            uint32_t pk4[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float2 a = f2_unpack(acc[4 * q + j]);
              const __nv_bfloat162 bb = __floats2bfloat162_rn(a.x + bias_s[8 * q + 2 * j],
                                                              a.y + bias_s[8 * q + 2 * j + 1]);
              pk4[j] = *reinterpret_cast<const uint32_t*>(&bb);
            }
            *reinterpret_cast<uint4*>(y + 8 * q) = make_uint4(pk4[0], pk4[1], pk4[2], pk4[3]);
          }
        }
      }
    }
  }

  tc_fence_before();
  cta_sync_converged();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace svdq

// int4_gemm.cuh -- steps a5..a6 for the INT4 format: symmetric int4 codes with
// one FP16 scale per 64 values along K, for both the activations and the
// residual weights (Diffusers blog, "quantization_config": svdq_w4a4 with
// precision int4, group_size 64), plus the low-rank up-projection and bias:
//
//   Y[m,n] = sum_k (sa[m,g(k)] qa[m,k]) (sw[n,g(k)] qw[n,k]) + sum_j xl1[m,j] L2[j,n] + bias[n]
//
// Every 64-wide group carries its own pair of scales, so an integer MMA would
// need one float multiply-add per output element per group on the CUDA cores.
// Instead the operands are dequantized on their way into shared memory: each
// code becomes the FP16 value fp16(s q), one rounding (relative error at most
// 2^-12), and one FP16 x FP16 -> FP32 tensor-core GEMM (tcgen05 kind::f16)
// accumulates all of K in tensor memory. With power-of-two scales the products
// are exact and so is the result; otherwise the rounding stays orders of
// magnitude inside the output tolerance. |s q| must stay within FP16's range
// (65504), i.e. a group's absolute maximum below about 65504.
//
// Tiled INT4 codes are two's complement nibbles, even K in the low nibble. A
// nibble u = q & 15 gives the FP16 pattern 0x6400 | (u ^ 8) = 1032 + q exactly,
// so a pair of codes dequantizes with one byte select, one mask, one FP16
// subtract and one FP16 multiply.
//
// Persistent kernel. A cluster of two CTAs on two SMs computes 256 x 256 output
// tiles with cta_group::2 MMAs: each CTA dequantizes its own 128 rows of A and
// 128 of the tile's 256 B rows, and each CTA's tensor memory accumulates its 128
// rows. The kernel is launched in pairs only (kPair): a lone CTA's converters
// would fill only half of the 256 B rows its N = 256 MMAs read.
// Two disjoint 256-column accumulators (no scale factors live in tensor
// memory) let the next tile's MMAs run while the epilogue drains the last one.
//
// Warp roles per CTA (22 warps):
//   warp 0      TMA producer: packed A and B codes [128 rows x 32 B] and their
//               FP16 scales [128] for one group per packed-ring stage
//   warp 1      tensor-memory owner; in the leader CTA also the MMA issuer
//   warps 2-17  converters: packed ring -> FP16 operand ring (128-byte swizzle,
//               half a row per thread: the dequantization's dependent steps need
//               many warps to hide them); for a low-rank slot, the L2 chunk by
//               TMA and xl1 as bf16 hi + lo operand tiles
//   warps 18-21 epilogue, one warp per tensor-memory lane quadrant (it is idle
//               for most of a tile): accumulator -> + bias -> bf16 / f32 ->
//               swizzled shared memory -> TMA store
#pragma once

#include "sm100.cuh"

namespace svdq {

constexpr int kI4Threads = 704;
constexpr int kI4CvtWarps = 16;
constexpr int kI4EpiWarps = 4;
constexpr int kI4BM = 128, kI4BN = 256;               // rows per CTA, columns per tile
constexpr int kI4PkOp = 128 * 32;                     // one operand's packed codes, one group
constexpr int kI4PkStage = 2 * kI4PkOp + 2 * 128 * 2; // A, B codes; A, B FP16 scales: 8.5 KB
constexpr int kI4PkStages = 4;
constexpr int kI4OpTile = 128 * 128;                  // 128 rows x 64 FP16 (128-byte rows)
constexpr int kI4OpStage = 2 * kI4OpTile;             // A tile, then this CTA's B rows: 32 KB
constexpr int kI4OpStages = 4;
constexpr int kI4LrK = 32;                            // low-rank K per slot
constexpr int kI4LrATile = 128 * kI4LrK * 2;          // 8 KB per bf16 tile (hi, lo)
constexpr int kI4StageOut = 4096;                     // epilogue staging bytes per warp
constexpr uint32_t kI4OffOp = 0;
constexpr uint32_t kI4OffPk = kI4OffOp + kI4OpStages * kI4OpStage;
constexpr uint32_t kI4OffOut = (kI4OffPk + kI4PkStages * kI4PkStage + 1023) / 1024 * 1024;
constexpr uint32_t kI4OffBias = kI4OffOut + kI4EpiWarps * kI4StageOut;
constexpr uint32_t kI4OffBars = kI4OffBias + kI4EpiWarps * 256 * 4;
constexpr int kI4NumBars = 2 * kI4PkStages + 2 * kI4OpStages + 4;
constexpr uint32_t kI4OffTmemSlot = kI4OffBars + 8 * kI4NumBars;
constexpr size_t kI4SmemBytes = kI4OffTmemSlot + 16 + 1024;  // + alignment slack
static_assert(kI4OffPk % 1024 == 0 && kI4PkStage % 128 == 0, "stage alignment");
static_assert(kI4OffOut % 1024 == 0, "staging alignment");
static_assert(kI4OpTile + 2 * kI4LrATile <= kI4OpStage, "a low-rank slot fits in a stage");

struct I4Params {
  int M, N, K, r;
  int tiles_m, tiles;      // tiles of kCtas * 128 rows x 256 columns, M fastest
  const float* xl1;
  const __nv_bfloat16* bias;
  int out_f32;
  uint32_t* status;
};

// Instruction descriptor, kind::f16 with FP16 A and B, f32 accumulate.
__host__ __device__ constexpr uint32_t idesc_f16_f32(uint32_t M, uint32_t N, bool a_mn_major,
                                                     bool b_mn_major) {
  return (1u << 4)                               // D format: f32
         | ((a_mn_major ? 1u : 0u) << 15)        // A major
         | ((b_mn_major ? 1u : 0u) << 16)        // B major
         | ((N >> 3) << 17)                      // N / 8
         | ((M >> 4) << 24);                     // M / 16
}

// Eight two's complement INT4 codes (code i in bits 4i..4i+3) times an FP16
// scale: four FP16 pairs, pair j = (code 2j, code 2j + 1), each fp16(s q).
__device__ __forceinline__ void int4x8_dequant(uint32_t w, __half2 s2, uint32_t (&out)[4]) {
  const uint32_t ev = w & 0x0F0F0F0Fu;          // codes 0, 2, 4, 6 in bytes 0..3
  const uint32_t od = (w >> 4) & 0x0F0F0F0Fu;   // codes 1, 3, 5, 7
  const __half2 bias2 = __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408));
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    // bytes (even j, -, odd j, -); the mask keeps the two nibbles, the xor
    // turns them into 0x6400 | (u ^ 8)
    uint32_t t;
    asm("prmt.b32 %0, %1, %2, %3;"
        : "=r"(t)
        : "r"(ev), "r"(od), "r"(j | (j << 4) | ((4 + j) << 8) | ((4 + j) << 12)));
    t = (t & 0x000F000Fu) ^ 0x64086408u;
    const __half2 v = __hsub2(*reinterpret_cast<const __half2*>(&t), bias2);  // q, exact
    const __half2 r = __hmul2(v, s2);
    out[j] = *reinterpret_cast<const uint32_t*>(&r);
  }
}

// 22 warps: up to six share one of the SM's four 16K-register partitions, which
// caps the kernel at 80 registers per thread.
template <bool kPair>
__global__ void __maxnreg__(80)
    w4a4_int4_gemm_kernel(const __grid_constant__ CUtensorMap tm_a,
                          const __grid_constant__ CUtensorMap tm_b,
                          const __grid_constant__ CUtensorMap tm_sa,
                          const __grid_constant__ CUtensorMap tm_sw,
                          const __grid_constant__ CUtensorMap tm_l2,
                          const __grid_constant__ CUtensorMap tm_y, const I4Params p) {
  constexpr int kCtas = kPair ? 2 : 1;
  static_assert(kPair, "CTA pairs only: a lone CTA's converters fill 128 of the tile's 256 B rows");
  constexpr int NP = kI4PkStages, NO = kI4OpStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = kPair ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;

  const int G = p.K / 64;
  const int lr_chunks = (p.r + kI4LrK - 1) / kI4LrK;
  const int slots = G + lr_chunks;                   // operand-ring slots per tile
  const int unit = blockIdx.x / kCtas;
  const int units = gridDim.x / kCtas;
  const int my_tiles = p.tiles > unit ? (p.tiles - 1 - unit) / units + 1 : 0;
  auto tile_mn = [&](int i, int& m0, int& n0) {
    const int t = unit + i * units;
    m0 = (t % p.tiles_m) * (kI4BM * kCtas);
    n0 = (t / p.tiles_m) * kI4BN;
  };

  auto op_st = [&](int s) { return sbase + kI4OffOp + s * kI4OpStage; };
  auto pk_st = [&](int s) { return sbase + kI4OffPk + s * kI4PkStage; };
  const uint32_t bars = sbase + kI4OffBars;
  auto pk_full = [&](int s) { return bars + 8 * s; };
  auto pk_empty = [&](int s) { return bars + 8 * (NP + s); };
  auto op_full = [&](int s) { return bars + 8 * (2 * NP + s); };       // the leader's counts
  auto op_empty = [&](int s) { return bars + 8 * (2 * NP + NO + s); };
  auto acc_full = [&](int b) { return bars + 8 * (2 * NP + 2 * NO + b); };
  auto acc_free = [&](int b) { return bars + 8 * (2 * NP + 2 * NO + 2 + b); };  // the leader's
  auto lead = [&](uint32_t a) { return kPair ? map_peer_smem(a, 0) : a; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kI4OffTmemSlot);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NP; ++s) {
      mbar_init(pk_full(s), 1);                   // this CTA's producer (with tx)
      mbar_init(pk_empty(s), kI4CvtWarps);        // this CTA's converters
    }
    for (int s = 0; s < NO; ++s) {
      mbar_init(op_full(s), kI4CvtWarps * kCtas);  // both CTAs' converters (+ L2 tx)
      mbar_init(op_empty(s), 1);                   // the MMA commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full(b), 1);
      mbar_init(acc_free(b), kI4EpiWarps * kCtas);
    }
    fence_barrier_init();
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    prefetch_tmap(&tm_sa);
    prefetch_tmap(&tm_sw);
    prefetch_tmap(&tm_y);
    if (p.r > 0) prefetch_tmap(&tm_l2);
  }
  if (warp == 1) {
    if (kPair) {
      tmem_alloc_pair(smem_u32(tmem_slot), 512);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_slot), 512);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if (kPair) cluster_sync_converged(); else cta_sync_converged();  // barriers initialised in both CTAs
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
        const int mrow = m0 + kI4BM * static_cast<int>(rank);
        const int nrow = n0 + kI4BM * static_cast<int>(rank);
        for (int g = 0; g < G && ok; ++g, ++jp) {
          const int s = jp % NP;
          ok = mbar_wait(pk_empty(s), ((jp / NP) & 1) ^ 1, p.status);
          if (!ok) break;
          const uint32_t dst = pk_st(s);
          mbar_arrive_expect_tx(pk_full(s), kI4PkStage);
          tma_load_2d(dst, &tm_a, pk_full(s), g * 32, mrow);
          tma_load_2d(dst + kI4PkOp, &tm_b, pk_full(s), g * 32, nrow);
          tma_load_2d(dst + 2 * kI4PkOp, &tm_sa, pk_full(s), mrow, g);
          tma_load_2d(dst + 2 * kI4PkOp + 256, &tm_sw, pk_full(s), nrow, g);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (leader && elect_one()) {
      bool ok = true;
      const uint32_t mma_m = kI4BM * kCtas;
      const uint32_t id_lr = idesc_bf16_f32(mma_m, kI4BN, false, true);
      const uint32_t id_op = idesc_f16_f32(mma_m, kI4BN, false, false);
      int jo = 0;
      for (int i = 0; i < my_tiles && ok; ++i) {
        const int b = i & 1, u = i >> 1;  // the u-th use of accumulator b
        const uint32_t acc = tmem + b * 256;
        if (u > 0) {
          ok = mbar_wait(acc_free(b), (u - 1) & 1, p.status);
          if (!ok) break;
        }
        tc_fence_after();
        for (int kt = 0; kt < slots && ok; ++kt, ++jo) {
          const int s = jo % NO;
          ok = mbar_wait(op_full(s), (jo / NO) & 1, p.status);
          if (!ok) break;
          tc_fence_after();
          const uint32_t st = op_st(s);
          if (kt < G) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              // 16 K = 32 B of each 128-byte swizzled row
              const uint64_t ad = smem_desc(st + kk * 32, 16, 1024, kSwizzle128B);
              const uint64_t bd = smem_desc(st + kI4OpTile + kk * 32, 16, 1024, kSwizzle128B);
              const uint32_t accum = (kt > 0 || kk > 0) ? 1u : 0u;
              if (kPair) mma_f16_pair(acc, ad, bd, id_op, accum);
              else mma_f16(acc, ad, bd, id_op, accum);
            }
          } else {
            // low-rank slot: B = L2 chunk (MN-major, 128-byte swizzle; 64-wide N
            // blocks 4096 B apart = LBO, 8-deep K groups 1024 B apart = SBO);
            // A = xl1 hi / lo (no-swizzle K-major: K-adjacent core matrices 128 B
            // apart = LBO, 8-row groups 512 B apart = SBO)
            const uint32_t a_hi = st + kI4OpTile, a_lo = a_hi + kI4LrATile;
#pragma unroll
            for (int kk = 0; kk < kI4LrK / 16; ++kk) {
              const uint64_t bd = smem_desc(st + kk * 2048, kI4LrK * 128, 1024, kSwizzle128B);
              const uint64_t ah = smem_desc(a_hi + kk * 256, 128, 512, kSwizzleNone);
              const uint64_t al = smem_desc(a_lo + kk * 256, 128, 512, kSwizzleNone);
              const uint32_t accum = (kt > 0 || kk > 0) ? 1u : 0u;
              if (kPair) {
                mma_f16_pair(acc, ah, bd, id_lr, accum);
                mma_f16_pair(acc, al, bd, id_lr, 1u);
              } else {
                mma_f16(acc, ah, bd, id_lr, accum);
                mma_f16(acc, al, bd, id_lr, 1u);
              }
            }
          }
          if (kPair) tc_commit_pair(op_empty(s), 0x3);
          else tc_commit(op_empty(s));
        }
        if (kPair) tc_commit_pair(acc_full(b), 0x3);
        else tc_commit(acc_full(b));
      }
    }
  } else if (warp < 2 + kI4CvtWarps) {
    // ------------------------------------------------------------ converters
    const int ct = threadIdx.x - 64;           // 0..511
    const int op = (ct >> 7) & 1;              // 0: an A row, 1: a B row
    const int row = ct & 127;
    const int hk = ct >> 8;                    // which 32 of the row's 64 K
    bool ok = true;
    int jp = 0, jo = 0;
    for (int i = 0; i < my_tiles && ok; ++i) {
      int m0, n0;
      tile_mn(i, m0, n0);
      const int m = m0 + kI4BM * static_cast<int>(rank) + row;  // this thread's A row
      const int nrow = n0 + kI4BM * static_cast<int>(rank);
      for (int kt = 0; kt < slots && ok; ++kt, ++jo) {
        const int s = jo % NO;
        const uint32_t st = op_st(s);
        if (kt < G) {
          const int ps = jp % NP;
          ok = mbar_wait(pk_full(ps), (jp / NP) & 1, p.status) &&
               mbar_wait(op_empty(s), ((jo / NO) & 1) ^ 1, p.status);
          if (!ok) break;
          const uint32_t src = pk_st(ps) + op * kI4PkOp + row * 32 + hk * 16;
          const uint4 c0 = lds_u4(src);
          uint16_t sc;
          asm volatile("ld.shared.u16 %0, [%1];"
                       : "=h"(sc)
                       : "r"(pk_st(ps) + 2 * kI4PkOp + op * 256 + row * 2));
          const __half2 s2 = __halves2half2(__ushort_as_half(sc), __ushort_as_half(sc));
          // this thread's 32 FP16 values: 16-byte chunk c = codes 8c .. 8c + 7
          const uint32_t rowp = st + op * kI4OpTile + row * 128;
          const uint32_t w[4] = {c0.x, c0.y, c0.z, c0.w};
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            const int c = 4 * hk + cc;
            uint32_t o[4];
            int4x8_dequant(w[cc], s2, o);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                             rowp + ((c ^ (row & 7)) << 4)),
                         "r"(o[0]), "r"(o[1]), "r"(o[2]), "r"(o[3])
                         : "memory");
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(pk_empty(ps));
            // The leader's pair MMA reads this CTA's rows through this SM's own
            // tensor core from this CTA's shared memory: the writes above are
            // ordered for it by the proxy fence and a CTA-scope release.
            if (kPair) mbar_arrive_remote(lead(op_full(s)));
            else mbar_arrive(op_full(s));
          }
          ++jp;
        } else {
          // low-rank slot: the A-row threads stage xl1 (loaded before the wait,
          // so the global read overlaps it); one thread brings this CTA's L2 chunk
          const int c = kt - G;
          float v[kI4LrK];
          const bool stager = op == 0 && hk == 0;  // one thread per A row
          if (stager) {
            const float4* srcx =
                reinterpret_cast<const float4*>(p.xl1 + static_cast<size_t>(m) * p.r + c * kI4LrK);
#pragma unroll
            for (int j = 0; j < kI4LrK / 4; ++j) {
              // rows past M and columns past r (r % 32 == 16) contribute zeros
              const float4 f = (m < p.M && c * kI4LrK + 4 * j < p.r)
                                   ? __ldg(srcx + j)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
              v[4 * j] = f.x; v[4 * j + 1] = f.y; v[4 * j + 2] = f.z; v[4 * j + 3] = f.w;
            }
          }
          ok = mbar_wait(op_empty(s), ((jo / NO) & 1) ^ 1, p.status);
          if (!ok) break;
          if (ct == 128) {
            // L2 rows [32 c, 32 c + 32) x this CTA's 128 columns as two 64-wide
            // boxes (rows past r read as zero); the leader expects both CTAs' bytes
            const uint32_t fb = lead(op_full(s));
            if (leader) mbar_expect_tx(op_full(s), kCtas * kI4LrK * 128 * 2);
            for (int nb = 0; nb < 2; ++nb) {
              if (kPair)
                tma_load_2d_pair(st + nb * (kI4LrK * 128), &tm_l2, fb, nrow + nb * 64, c * kI4LrK);
              else
                tma_load_2d(st + nb * (kI4LrK * 128), &tm_l2, fb, nrow + nb * 64, c * kI4LrK);
            }
          }
          if (stager) {
            const uint32_t a_hi = st + kI4OpTile, a_lo = a_hi + kI4LrATile;
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
              const uint32_t off = (row >> 3) * 512 + cm * 128 + (row & 7) * 16;
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
          if (lane == 0) {
            if (kPair) mbar_arrive_remote(lead(op_full(s)));
            else mbar_arrive(op_full(s));
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Each warp owns the eight 32-column sub-tiles of its lane quadrant.
    const int ew = warp - 2 - kI4CvtWarps;   // 0..3
    const int quad = warp & 3;               // tensor-memory lanes 32 quad .. 32 quad + 31
    const uint32_t out_buf = sbase + kI4OffOut + ew * kI4StageOut;
    float* bias_s = reinterpret_cast<float*>(smem + kI4OffBias) + ew * 256;  // [8][32]
    bool ok = true;
    int stores = 0;
    for (int i = 0; i < my_tiles && ok; ++i) {
      int m0, n0;
      tile_mn(i, m0, n0);
      const int mrow = m0 + kI4BM * static_cast<int>(rank);
      const int b = i & 1, u = i >> 1;
      const uint32_t t_row = tmem + b * 256 + (static_cast<uint32_t>(quad * 32) << 16);
      // bias for this warp's sub-tiles, fetched before the accumulator is ready
      __syncwarp();
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const int n = n0 + 32 * t + lane;
        bias_s[t * 32 + lane] = (p.bias != nullptr && n < p.N) ? __bfloat162float(p.bias[n]) : 0.0f;
      }
      __syncwarp();
      ok = mbar_wait(acc_full(b), u & 1, p.status);
      if (!ok) break;
      tc_fence_after();
      for (int t = 0; t < 8; ++t) {
        const int j0 = 32 * t;
        uint32_t acc[32];
        tmem_ld32(t_row + j0, acc);
        tmem_ld_wait();
        if (t == 7) {
          // the warp's whole slice is in registers: the accumulator is free
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if (kPair) mbar_arrive_remote(lead(acc_free(b)));  // hands over no memory contents
            else mbar_arrive(acc_free(b));
          }
        }
        if (n0 + j0 >= p.N || mrow >= p.M) continue;  // warp-uniform
        float y[32];
        const float4* bv = reinterpret_cast<const float4*>(bias_s + t * 32);
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) {
          const float4 bb = bv[q4];
          y[4 * q4 + 0] = __uint_as_float(acc[4 * q4 + 0]) + bb.x;
          y[4 * q4 + 1] = __uint_as_float(acc[4 * q4 + 1]) + bb.y;
          y[4 * q4 + 2] = __uint_as_float(acc[4 * q4 + 2]) + bb.z;
          y[4 * q4 + 3] = __uint_as_float(acc[4 * q4 + 3]) + bb.w;
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
            const __nv_bfloat162 bb = __floats2bfloat162_rn(y[2 * j], y[2 * j + 1]);
            pk[j] = *reinterpret_cast<const uint32_t*>(&bb);
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
          tma_store_2d(&tm_y, buf, n0 + j0, mrow + quad * 32);
          bulk_commit();
        }
        ++stores;
      }
    }
    if (lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  // both CTAs' tensor memory is written by the leader's MMAs: release it only
  // once every warp of the pair is done
  if (kPair) cluster_sync_converged(); else cta_sync_converged();
  if (warp == 1) {
    tc_fence_after();
    if (kPair) tmem_dealloc_pair(tmem, 512);
    else tmem_dealloc(tmem, 512);
  }
}

}  // namespace svdq

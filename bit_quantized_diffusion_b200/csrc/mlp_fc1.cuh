// mlp_fc1.cuh -- the first half of the fused MLP (Diffusers blog, "From
// SVDQuant to Nunchaku Lite": the original engine runs GELU/MLP as one fused
// path): fc1's NVFP4 GEMM with its low-rank branch and bias, and in its
// epilogue GELU, fc2's smoothing and fc2's steps a2..a4, so the [M, N1] hidden
// activation never reaches HBM in 16 bits:
//
//   y1     = Q(X1_hat) Q(R1)^T + xl1_1 L2_1 + bias1                (tensor memory, float32)
//   h_hat  = RN32(RN32(GELU_tanh(RN32(y1))) * smooth_inv2[n])      (epilogue, float32; GELU as
//            y / (1 + exp(-2u)), which equals its tanh form 0.5 y (1 + tanh(u)), to a few ulps)
//   codes2, scales2 = NVFP4 of h_hat, groups of 16 along N1         (fc2's tiled layouts)
//   xl1_2  = h_hat L1_2                                            (tensor cores, float32)
//
// The down-projection xl1_2 sums over all of N1, so it runs on the tensor
// cores: the epilogue writes each tile's h_hat as a bf16 hi + lo pair (to
// about 2^-17 relative) into a shared-memory operand, and the MMA issuer adds
// h_hat_hi L1_2 + h_hat_lo L1_2 into a tensor-memory accumulator of r2 columns
// that stays there across all the tiles of a unit. A unit is one 256-row block
// and a contiguous range of N1 tiles; at its end the epilogue writes the
// unit's partial sum [256, r2] to one slice of the caller's working space, and
// a second kernel adds the slices in order (as the quantizer's K split does).
//
// Layout of the work: CTA pairs (cta_group::2), tiles of 256 rows x 128
// columns (each CTA stages its 128 rows of A and 64 of the tile's 128 B rows).
// Tensor memory per CTA: two 128-column fc1 accumulators (tile i uses i % 2),
// the xl1_2 accumulator (128 columns), four 32-column scale-factor buffers (the
// quadrant warps may fill a buffer once the MMAs four 4-bit slots back are done).
// Ring slots of a unit, in order: for each tile its K/256 FP4 slots and
// ceil(r1/32) low-rank slots, then (from the second tile on) the xl1_2 slot of
// the previous tile (L1_2^T's [r2/2 x 128] slice per CTA); after the last tile
// the xl1_2 slot of that tile. The previous tile's xl1_2 MMAs are issued after
// this tile's fc1 MMAs, so the epilogue has a whole tile's time to form h_hat.
//
// Warp roles per CTA (14 warps): warp 0 TMA producer; warp 1 tensor-memory
// owner and (leader) MMA issuer; warps 2-5 scale factors by tcgen05.st and the
// low-rank operand staging (as in the NVFP4 GEMM); warps 6-13 epilogue, two
// per lane quadrant, 64 columns each.
#pragma once

#include "quantize_act.cuh"
#include "sm100.cuh"

namespace svdq {

constexpr int kMlThreads = 448;
constexpr int kMlBM = 128;                         // rows per CTA (a pair's tile: 256)
constexpr int kMlBN = 128;                         // fc1 columns per tile
constexpr int kMlBRows = kMlBN / 2;                // B rows staged per CTA
constexpr int kMlAStage = kMlBM * 128;             // 16 KB
constexpr int kMlBStage = kMlBRows * 128;          // 8 KB
constexpr int kMlSfaStage = 4 * 512;               // 4 atoms (one per 64-wide K block)
constexpr int kMlSfbStage = 4 * 512;               // one 128-row atom per K block
constexpr int kMlStageBytes = kMlAStage + kMlBStage + kMlSfaStage + kMlSfbStage;  // 28 KB
constexpr int kMlStages = 4;
constexpr int kMlLrK = 32;                         // fc1 low-rank K per slot
constexpr int kMlLrBTile = kMlLrK * kMlBRows * 2;  // L2_1 chunk [32 x 64] bf16
constexpr int kMlR2Max = 128;
constexpr uint32_t kMlRing = 0;
constexpr uint32_t kMlHhat = kMlStages * kMlStageBytes;            // [hi, lo][2 K chunks][128 x 128 B]
constexpr uint32_t kMlHhatPlane = 2 * kMlBM * 128;                 // 32 KB
constexpr uint32_t kMlStaging = kMlHhat + 2 * kMlHhatPlane;        // bias1, smooth_inv2 per epilogue warp
constexpr uint32_t kMlBars = kMlStaging + 8 * 2 * 64 * 4;
// full, empty, ready, sf landed per stage; acc full, acc free x2; sf full, sf free x4;
// hhat full, hhat free; xl1_2 full, xl1_2 free
constexpr int kMlSfBufs = 4;                      // scale-factor buffers in tensor memory
constexpr uint32_t kMlTmemSlot = kMlBars + 8 * (4 * kMlStages + 4 + 2 * kMlSfBufs + 4);
constexpr size_t kMlSmemBytes = kMlTmemSlot + 16 + 1024;
// tensor-memory columns
constexpr uint32_t kMlTmAcc = 0, kMlTmXl1 = 256, kMlTmSf = 384, kMlTmSfBuf = 32, kMlTmCols = 512;
static_assert(kMlTmSf + kMlSfBufs * kMlTmSfBuf <= kMlTmCols, "tensor-memory layout");
static_assert(kMlStageBytes % 1024 == 0, "stages stay 1024-byte aligned");
static_assert(kMlLrBTile + 2 * kMlBM * kMlLrK * 2 <= kMlStageBytes, "a low-rank slot fits in a stage");
static_assert(2 * (kMlR2Max / 2) * 128 <= kMlStageBytes, "an xl1_2 slot fits in a stage");

struct MlpParams {
  int M, N1, K1, r1, r2;
  int row_blocks;          // 256-row blocks
  int ntn;                 // 128-column tiles of N1
  int tps;                 // tiles per unit (the last unit of a row block may have fewer)
  int nsplit;              // units per row block
  int units;
  const __nv_bfloat16* bias1;
  const float* smooth_inv2;  // [N1] or null (1)
  uint8_t* codes2;           // [M, N1 / 2]
  uint8_t* scales2;          // atoms [(rows / 128)][N1 / 64][512]
  float* xl1_part;           // [nsplit][M][r2]
  float* hhat;               // [M][N1] float32, or null
  uint32_t* status;
};

// GELU of two values: 0.5 y (1 + tanh(u)), u = sqrt(2/pi) (y + 0.044715 y^3), in
// float32 through the identity 1 + tanh(u) = 2 / (1 + exp(-2u)), i.e. GELU =
// y / (1 + exp(-2u)): one exponential and one division per value (a few float32
// ulps), the polynomial on paired float32 instructions. The form has no
// cancellation; exp's argument is capped at 80 (finite in float32), where GELU
// is 0 to float32 precision already.
__device__ __forceinline__ float2 gelu_tanh2(float2 y) {
  const float2 yy = __fmul2_rn(y, y);
  const float2 a = __fmul2_rn(y, make_float2(0.044715f, 0.044715f));
  const float2 t = __ffma2_rn(a, yy, y);                                         // y + 0.044715 y^3
  const float2 m = __fmul2_rn(t, make_float2(-1.5957691216057308f, -1.5957691216057308f));  // -2u
  const float dx = 1.0f + __expf(fminf(m.x, 80.0f)), dy = 1.0f + __expf(fminf(m.y, 80.0f));
  return make_float2(__fdividef(y.x, dx), __fdividef(y.y, dy));
}

__global__ void __launch_bounds__(kMlThreads, 1)
    w4a4_mlp_fc1_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                        const __grid_constant__ CUtensorMap tm_sfa, const __grid_constant__ CUtensorMap tm_sfb,
                        const __grid_constant__ CUtensorMap tm_l2, const __grid_constant__ CUtensorMap tm_xl1,
                        const __grid_constant__ CUtensorMap tm_l1t, const MlpParams p) {
  constexpr int NS = kMlStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  const int kblocks = p.K1 / 64;
  const int ktiles = (kblocks + 3) / 4;
  const int lr_chunks = (p.r1 + kMlLrK - 1) / kMlLrK;
  const bool x2 = p.r2 > 0;
  const int pair_id = blockIdx.x / 2;
  const int npairs = gridDim.x / 2;
  // unit u: row block u % row_blocks, tiles [tps (u / row_blocks), ...) of N1
  auto unit_tiles = [&](int u, int& rb, int& t0, int& nt) {
    rb = u % p.row_blocks;
    t0 = (u / p.row_blocks) * p.tps;
    nt = min(p.tps, p.ntn - t0);
  };

  auto stage = [&](int s) { return sbase + kMlRing + s * kMlStageBytes; };
  auto a_st = [&](int s) { return stage(s); };
  auto b_st = [&](int s) { return stage(s) + kMlAStage; };
  auto sfa_st = [&](int s) { return stage(s) + kMlAStage + kMlBStage; };
  auto sfb_st = [&](int s) { return sfa_st(s) + kMlSfaStage; };
  auto bar_full = [&](int s) { return sbase + kMlBars + 8 * s; };
  auto bar_empty = [&](int s) { return sbase + kMlBars + 8 * (NS + s); };
  auto bar_ready = [&](int s) { return sbase + kMlBars + 8 * (2 * NS + s); };
  auto bar_sf_landed = [&](int s) { return sbase + kMlBars + 8 * (3 * NS + s); };
  const uint32_t bar0 = sbase + kMlBars + 8 * (4 * NS);
  auto bar_acc_full = [&](int a) { return bar0 + 8 * a; };
  auto bar_acc_free = [&](int a) { return bar0 + 16 + 8 * a; };
  auto bar_sf_full = [&](int b) { return bar0 + 32 + 8 * b; };
  auto bar_sf_free = [&](int b) { return bar0 + 32 + 8 * kMlSfBufs + 8 * b; };
  const uint32_t bar_hh_full = bar0 + 32 + 16 * kMlSfBufs, bar_hh_free = bar_hh_full + 8;
  const uint32_t bar_x2_full = bar_hh_full + 16, bar_x2_free = bar_hh_full + 24;
  auto lead = [&](uint32_t a) { return map_peer_smem(a, 0); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kMlTmemSlot);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_ready(s), 4 * 2);
      mbar_init(bar_empty(s), 1);
      mbar_init(bar_sf_landed(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar_acc_full(a), 1);
      mbar_init(bar_acc_free(a), 8 * 2);
    }
    for (int b = 0; b < kMlSfBufs; ++b) {
      mbar_init(bar_sf_full(b), 4 * 2);
      mbar_init(bar_sf_free(b), 1);
    }
    mbar_init(bar_hh_full, 8 * 2);
    mbar_init(bar_hh_free, 1);
    mbar_init(bar_x2_full, 1);
    mbar_init(bar_x2_free, 8 * 2);
    fence_barrier_init();
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    prefetch_tmap(&tm_sfa);
    prefetch_tmap(&tm_sfb);
    if (p.r1 > 0) {
      prefetch_tmap(&tm_l2);
      prefetch_tmap(&tm_xl1);
    }
    if (x2) prefetch_tmap(&tm_l1t);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), kMlTmCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_converged();
  grid_dep_wait();
  grid_dep_launch();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      bool ok = true;
      int sg = 0;  // ring slots so far
      auto next_slot = [&](int& s) {
        s = sg % NS;
        ok = mbar_wait(bar_empty(s), ((sg / NS) & 1) ^ 1, p.status);
        ++sg;
        return ok;
      };
      for (int u = pair_id; u < p.units && ok; u += npairs) {
        int rb, t0, nt;
        unit_tiles(u, rb, t0, nt);
        const int mrow = rb * 2 * kMlBM + kMlBM * static_cast<int>(rank);
        for (int i = 0; i <= nt && ok; ++i) {
          if (i < nt) {
            const int n0 = (t0 + i) * kMlBN;
            const int nrow = n0 + kMlBRows * static_cast<int>(rank);
            for (int kt = 0; kt < ktiles + lr_chunks && ok; ++kt) {
              int s;
              if (!next_slot(s)) break;
              const uint32_t fb = lead(bar_full(s));
              const uint32_t sl = bar_sf_landed(s);
              if (kt < ktiles) {
                if (leader) mbar_arrive_expect_tx(bar_full(s), 2 * (kMlAStage + kMlBStage));
                tma_load_2d_pair(a_st(s), &tm_a, fb, kt * 128, mrow);
                tma_load_2d_pair(b_st(s), &tm_b, fb, kt * 128, nrow);
                mbar_arrive_expect_tx(sl, kMlSfaStage + kMlSfbStage);
                tma_load_2d(sfa_st(s), &tm_sfa, sl, 0, ((mrow / 128) * kblocks + 4 * kt) * 2);
                tma_load_2d(sfb_st(s), &tm_sfb, sl, 0, ((n0 / 128) * kblocks + 4 * kt) * 2);
              } else {
                const int c = kt - ktiles;
                mbar_arrive_expect_tx(sl, kMlBM * kMlLrK * 4);
                tma_load_2d(stage(s) + kMlLrBTile, &tm_xl1, sl, c * kMlLrK, mrow);
                if (leader) mbar_arrive_expect_tx(bar_full(s), 2 * kMlLrBTile);
                tma_load_2d_pair(stage(s), &tm_l2, fb, nrow, c * kMlLrK);
              }
            }
          }
          if (x2 && i > 0 && ok) {
            // the previous tile's L1_2^T slice: this CTA's r2 / 2 ranks x 128 columns
            int s;
            if (!next_slot(s)) break;
            const int n0 = (t0 + i - 1) * kMlBN;
            const int rrow = (p.r2 / 2) * static_cast<int>(rank);
            if (leader) mbar_arrive_expect_tx(bar_full(s), 2 * 2 * (p.r2 / 2) * 128);
            for (int c = 0; c < 2; ++c)
              tma_load_2d_pair(stage(s) + c * (p.r2 / 2) * 128, &tm_l1t, lead(bar_full(s)), n0 + 64 * c, rrow);
            mbar_arrive(bar_sf_landed(s));  // nothing for the quadrant warps: keeps the phases in step
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (leader && elect_one()) {
      bool ok = true;
      const uint32_t id_fp4 = idesc_nvfp4(2 * kMlBM, kMlBN);
      const uint32_t id_lr = idesc_bf16_f32(2 * kMlBM, kMlBN, false, true);
      const uint32_t id_x2 = idesc_bf16_f32(2 * kMlBM, static_cast<uint32_t>(x2 ? p.r2 : 16), false, false);
      const uint64_t a_desc0 = smem_desc(a_st(0), 16, 1024, kSwizzle128B);
      const uint64_t b_desc0 = smem_desc(b_st(0), 16, 1024, kSwizzle128B);
      constexpr uint64_t kStageStep = static_cast<uint64_t>(kMlStageBytes >> 4);
      int sg = 0, fp4 = 0, gt = 0, uc = 0, xs = 0;  // slots, 4-bit slots, tiles, units, xl1_2 slots
      uint32_t lr_uses = 0;
      auto take = [&](int& s) {
        s = sg % NS;
        ok = mbar_wait(bar_full(s), (sg / NS) & 1, p.status);
        ++sg;
        if (ok) tc_fence_after();
        return ok;
      };
      for (int u = pair_id; u < p.units && ok; u += npairs, ++uc) {
        int rb, t0, nt;
        unit_tiles(u, rb, t0, nt);
        for (int i = 0; i <= nt && ok; ++i) {
          if (i < nt) {
            const int a = gt & 1;
            const uint32_t acc = tmem + kMlTmAcc + 128u * static_cast<uint32_t>(a);
            if (gt >= 2) {
              ok = mbar_wait(bar_acc_free(a), ((gt >> 1) - 1) & 1, p.status);
              if (!ok) break;
              tc_fence_after();
            }
            for (int kt = 0; kt < ktiles + lr_chunks && ok; ++kt) {
              int s;
              if (!take(s)) break;
              if (kt < ktiles) {
                const uint32_t buf = static_cast<uint32_t>(fp4 % kMlSfBufs);
                ok = mbar_wait(bar_sf_full(buf), (fp4 / kMlSfBufs) & 1, p.status);
                if (!ok) break;
                tc_fence_after();
                const uint32_t sfa = tmem + kMlTmSf + kMlTmSfBuf * buf, sfb = sfa + 16;
                const uint64_t ad = a_desc0 + kStageStep * static_cast<uint64_t>(s);
                const uint64_t bd = b_desc0 + kStageStep * static_cast<uint64_t>(s);
                const int nkb = min(4, kblocks - 4 * kt);
                for (int kb = 0; kb < nkb; ++kb)
                  mma_nvfp4_pair(acc, ad + 2 * kb, bd + 2 * kb, id_fp4, sfa + 4 * kb, sfb + 4 * kb,
                                 (kt > 0 || kb > 0) ? 1u : 0u);
                tc_commit_pair(bar_sf_free(buf), 0x3);
                ++fp4;
              } else {
                ok = mbar_wait(bar_ready(s), (lr_uses >> s) & 1u, p.status);
                lr_uses ^= 1u << s;
                if (!ok) break;
                tc_fence_after();
                const uint32_t a_lr = stage(s) + kMlLrBTile;
#pragma unroll
                for (int kk = 0; kk < kMlLrK / 16; ++kk) {
                  const uint64_t bd = smem_desc(stage(s) + kk * 2048, kMlLrK * 128, 1024, kSwizzle128B);
                  const uint64_t ah = smem_desc(a_lr + kk * 256, 128, 1024, kSwizzleNone);
                  const uint64_t al = smem_desc(a_lr + 512 + kk * 256, 128, 1024, kSwizzleNone);
                  mma_f16_pair(acc, ah, bd, id_lr, 1u);
                  mma_f16_pair(acc, al, bd, id_lr, 1u);
                }
              }
              tc_commit_pair(bar_empty(s), 0x3);
            }
            if (!ok) break;
            tc_commit_pair(bar_acc_full(a), 0x3);
            ++gt;
          }
          if (x2 && i > 0) {
            // xl1_2 += h_hat(tile i - 1) L1_2[tile i - 1 columns, :]
            int s;
            if (!take(s)) break;
            ok = mbar_wait(bar_hh_full, xs & 1, p.status);
            if (ok && i == 1 && uc > 0) ok = mbar_wait(bar_x2_free, (uc - 1) & 1, p.status);
            if (!ok) break;
            tc_fence_after();
            const uint32_t x2acc = tmem + kMlTmXl1;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint32_t ha = sbase + kMlHhat + c * (kMlBM * 128) + kk * 32;
                const uint64_t ah = smem_desc(ha, 16, 1024, kSwizzle128B);
                const uint64_t al = smem_desc(ha + kMlHhatPlane, 16, 1024, kSwizzle128B);
                const uint64_t bd = smem_desc(stage(s) + c * (p.r2 / 2) * 128 + kk * 32, 16, 1024, kSwizzle128B);
                mma_f16_pair(x2acc, ah, bd, id_x2, (i > 1 || c > 0 || kk > 0) ? 1u : 0u);
                mma_f16_pair(x2acc, al, bd, id_x2, 1u);
              }
            }
            tc_commit_pair(bar_empty(s), 0x3);
            tc_commit_pair(bar_hh_free, 0x3);
            if (i == nt) tc_commit_pair(bar_x2_full, 0x3);
            ++xs;
          }
        }
      }
    }
  } else if (warp < 6) {
    // ---------------------------------------- scale factors and low-rank staging
    const int quad = warp & 3;
    const int trow = quad * 32 + lane;
    const uint32_t sf_lanes = tmem + kMlTmSf + (static_cast<uint32_t>(quad * 32) << 16);
    bool ok = true;
    int sg = 0, fp4 = 0;
    auto wait_slot = [&](int& s) {
      s = sg % NS;
      ok = mbar_wait(bar_empty(s), ((sg / NS) & 1) ^ 1, p.status) &&
           mbar_wait(bar_sf_landed(s), (sg / NS) & 1, p.status);
      ++sg;
      ok = __all_sync(0xffffffffu, ok);
      return ok;
    };
    for (int u = pair_id; u < p.units && ok; u += npairs) {
      int rb, t0, nt;
      unit_tiles(u, rb, t0, nt);
      for (int i = 0; i <= nt && ok; ++i) {
        if (i < nt) {
          for (int kt = 0; kt < ktiles && ok; ++kt, ++fp4) {
            int s;
            if (!wait_slot(s)) break;
            const int buf = fp4 % kMlSfBufs;
            uint32_t sa[16], sbv[16];
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
              const uint4 a = lds_u4(sfa_st(s) + kb * 512 + lane * 16);
              sa[4 * kb] = a.x; sa[4 * kb + 1] = a.y; sa[4 * kb + 2] = a.z; sa[4 * kb + 3] = a.w;
              const uint4 b = lds_u4(sfb_st(s) + kb * 512 + lane * 16);
              sbv[4 * kb] = b.x; sbv[4 * kb + 1] = b.y; sbv[4 * kb + 2] = b.z; sbv[4 * kb + 3] = b.w;
            }
            ok = fp4 < kMlSfBufs || mbar_wait(bar_sf_free(buf), ((fp4 / kMlSfBufs) - 1) & 1, p.status);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            const uint32_t dst = sf_lanes + kMlTmSfBuf * static_cast<uint32_t>(buf);
            tmem_st16(dst, sa);
            tmem_st16(dst + 16, sbv);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(lead(bar_sf_full(buf)));
          }
          for (int c = 0; c < lr_chunks && ok; ++c) {
            int s;
            if (!wait_slot(s)) break;
            // this lane's row of the float32 xl1_1 chunk -> bf16 hi + lo operand rows
            const uint32_t lr = stage(s) + kMlLrBTile;
            float v[kMlLrK];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float4 f = lds_f4(lr + trow * 128 + ((q ^ (trow & 7)) << 4));
              v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
            }
            __syncwarp();
#pragma unroll
            for (int cm = 0; cm < kMlLrK / 8; ++cm) {
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
              const uint32_t off = (trow >> 3) * 1024 + cm * 128 + (trow & 7) * 16;
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(lr + off), "r"(hi[0]),
                           "r"(hi[1]), "r"(hi[2]), "r"(hi[3])
                           : "memory");
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(lr + off + 512), "r"(lo[0]),
                           "r"(lo[1]), "r"(lo[2]), "r"(lo[3])
                           : "memory");
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(lead(bar_ready(s)));
          }
        }
        if (x2 && i > 0 && ok) {
          int s;
          wait_slot(s);  // the xl1_2 slot: nothing to stage, but its phases are waited in order
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;
    const int half = (warp - 6) >> 2;   // columns 64 half .. + 63 of the tile
    float* stg = reinterpret_cast<float*>(smem + kMlStaging) + (warp - 6) * 128;  // bias [64], smooth [64]
    bool ok = true;
    int gt = 0, uc = 0;
    const int N1 = p.N1;
    for (int u = pair_id; u < p.units && ok; u += npairs, ++uc) {
      int rb, t0, nt;
      unit_tiles(u, rb, t0, nt);
      const int mrow = rb * 2 * kMlBM + kMlBM * static_cast<int>(rank);
      const int m = mrow + quad * 32 + lane;  // this lane's row
      const bool m_ok = m < p.M;
      for (int i = 0; i < nt && ok; ++i, ++gt) {
        const int n0 = (t0 + i) * kMlBN;
        const int a = gt & 1;
        // this warp's 64 columns of bias1 and smooth_inv2, before the accumulator is ready
        __syncwarp();
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const int n = n0 + 64 * half + 32 * t + lane;
          stg[32 * t + lane] = p.bias1 != nullptr ? __bfloat162float(p.bias1[n]) : 0.0f;
          stg[64 + 32 * t + lane] = p.smooth_inv2 != nullptr ? p.smooth_inv2[n] : 1.0f;
        }
        __syncwarp();
        ok = mbar_wait(bar_acc_full(a), (gt >> 1) & 1, p.status);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const uint32_t t_row = tmem + kMlTmAcc + 128u * static_cast<uint32_t>(a) +
                               (static_cast<uint32_t>(quad * 32) << 16) + 64u * static_cast<uint32_t>(half);
        // the previous tile's xl1_2 MMAs have read the h_hat operand
        if (x2 && gt > 0) {
          ok = mbar_wait(bar_hh_free, (gt - 1) & 1, p.status);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
        }
#pragma unroll 1
        for (int t = 0; t < 2; ++t) {
          const int j0 = 64 * half + 32 * t;  // column of the tile
          uint32_t acc[32];
          tmem_ld32(t_row + 32 * t, acc);
          tmem_ld_wait();
          if (t == 1) {
            // the warp's columns of this accumulator are in registers: the MMAs of
            // the tile after next may use it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(lead(bar_acc_free(a)));
          }
          float hv[32];
#pragma unroll
          for (int q = 0; q < 32; q += 2) {
            const float2 b = *reinterpret_cast<const float2*>(stg + 32 * t + q);
            const float2 sm = *reinterpret_cast<const float2*>(stg + 64 + 32 * t + q);
            const float2 y = __fadd2_rn(make_float2(__uint_as_float(acc[q]), __uint_as_float(acc[q + 1])), b);
            const float2 h = __fmul2_rn(gelu_tanh2(y), sm);
            hv[q] = m_ok ? h.x : 0.0f;
            hv[q + 1] = m_ok ? h.y : 0.0f;
          }
          if (p.hhat != nullptr && m_ok) {
            float4* dst = reinterpret_cast<float4*>(p.hhat + static_cast<size_t>(m) * N1 + n0 + j0);
#pragma unroll
            for (int q = 0; q < 8; ++q) dst[q] = make_float4(hv[4 * q], hv[4 * q + 1], hv[4 * q + 2], hv[4 * q + 3]);
          }
          // fc2's NVFP4 codes and scales: two groups of 16
          uint32_t code[4], sc[2];
#pragma unroll
          for (int g = 0; g < 2; ++g) {
            float2 pv[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) pv[q] = make_float2(hv[16 * g + 2 * q], hv[16 * g + 2 * q + 1]);
            const float amax = absmax16(pv);
            sc[g] = e4m3_code(div_by_const_rn<6>(amax));
            const float sv = e4m3_value(sc[g]);
            const float rcp = sv != 0.0f ? __frcp_rn(sv) : 0.0f;
            float2 y0[4], y1[4];
            const float2 rcp2 = make_float2(rcp, rcp);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              y0[q] = __fmul2_rn(pv[q], rcp2);
              y1[q] = __fmul2_rn(pv[4 + q], rcp2);
            }
            code[2 * g] = sv != 0.0f ? e2m1x8(y0) : 0u;
            code[2 * g + 1] = sv != 0.0f ? e2m1x8(y1) : 0u;
          }
          const int n = n0 + j0;  // fc2's K position of this lane's first value
          if (m_ok)
            *reinterpret_cast<uint4*>(p.codes2 + static_cast<size_t>(m) * (N1 / 2) + n / 2) =
                make_uint4(code[0], code[1], code[2], code[3]);
          if (m < (p.M + 127) / 128 * 128) {
            // scale bytes of groups n / 16, n / 16 + 1 of row m (zero for the padding rows past M)
            const size_t atom = static_cast<size_t>(m / 128) * (N1 / 64) + n / 64;
            const uint16_t pair = m_ok ? static_cast<uint16_t>(sc[0] | (sc[1] << 8)) : 0;
            *reinterpret_cast<uint16_t*>(p.scales2 + atom * 512 + (m & 31) * 16 + ((m & 127) >> 5) * 4 +
                                         ((n >> 4) & 3)) = pair;
          }
          if (x2) {
            // h_hat as bf16 hi + lo into the xl1_2 operand: K-major, 128-byte swizzle,
            // row = this lane's row of the CTA, K = tile column
            const int row = quad * 32 + lane;
            const uint32_t cbase = sbase + kMlHhat + (j0 >> 6) * (kMlBM * 128) + row * 128;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              uint32_t hi[4], lo[4];
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const float2 x = make_float2(hv[8 * cc + 2 * j], hv[8 * cc + 2 * j + 1]);
                const __nv_bfloat162 hb = __floats2bfloat162_rn(x.x, x.y);
                const float2 r = __fadd2_rn(x, make_float2(-__bfloat162float(hb.x), -__bfloat162float(hb.y)));
                const __nv_bfloat162 lb = __floats2bfloat162_rn(r.x, r.y);
                hi[j] = *reinterpret_cast<const uint32_t*>(&hb);
                lo[j] = *reinterpret_cast<const uint32_t*>(&lb);
              }
              const uint32_t chunk = static_cast<uint32_t>((((j0 & 63) >> 3) + cc) ^ (row & 7)) << 4;
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(cbase + chunk), "r"(hi[0]),
                           "r"(hi[1]), "r"(hi[2]), "r"(hi[3])
                           : "memory");
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(cbase + kMlHhatPlane + chunk),
                           "r"(lo[0]), "r"(lo[1]), "r"(lo[2]), "r"(lo[3])
                           : "memory");
            }
          }
        }
        if (x2) {
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive_remote(lead(bar_hh_full));
        }
      }
      if (!ok || !x2) continue;
      // the unit's partial xl1_2 [its rows, r2] -> slice u / row_blocks of the working space
      ok = mbar_wait(bar_x2_full, uc & 1, p.status);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int split = u / p.row_blocks;
      float* dst = p.xl1_part + (static_cast<size_t>(split) * p.M + (m_ok ? m : 0)) * p.r2;
      for (int c = 64 * half; c < 64 * half + 64 && c < p.r2; c += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + kMlTmXl1 + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(c), v);
        tmem_ld_wait();
        if (m_ok) {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            reinterpret_cast<float4*>(dst + c)[q] =
                make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                            __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(lead(bar_x2_free));
    }
  }

  tc_fence_before();
  cluster_sync_converged();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kMlTmCols);
  }
}

}  // namespace svdq

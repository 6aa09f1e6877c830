// w4a4_gemm.cuh -- steps a5..a6: the NVFP4 4-bit GEMM on tcgen05 block-scaled
// MMA (kind::mxf4nvf4, one UE4M3 scale per 16 along K), with the low-rank
// up-projection (x_hat L1) L2 and the bias accumulated into the same
// tensor-memory accumulator, so the 16-bit branch never round-trips HBM
// (Nunchaku README, "Engine design" (b): up projection and 4-bit compute share
// the output).
//
// Persistent kernel. In pair mode (kPair) a cluster of two CTAs on two SMs
// computes 256 x 256 output tiles with cta_group::2 MMAs: each CTA stages its
// own 128 rows of A and its own 128 of the tile's 256 B rows, the pair's tensor
// cores exchange the B halves, and each CTA's tensor memory accumulates its 128
// rows. Per CTA that halves the B traffic and the B shared memory of a stage,
// which buys a 4-stage ring. Without kPair one CTA computes 128 x 256 tiles.
//
// Warp roles per CTA (14 warps):
//   warp 0      TMA producer: A/B code tiles [rows x 128 B] with 128-byte swizzle,
//               A/B scale atoms, L2 chunks [32 x 128 or 256] bf16; runs ahead
//               across tiles through the ring
//   warp 1      tensor-memory owner; in the leader CTA also the MMA issuer (one
//               thread)
//   warps 2-5   one per tensor-memory lane quadrant: place each 4-bit slot's
//               scale factors in tensor memory (tcgen05.st), and stage xl1
//               (float32) as bf16 hi + lo operand tiles for the low-rank slots
//   warps 6-13  epilogue, two warps per tensor-memory lane quadrant: accumulator
//               -> + bias -> bf16 / f32 -> swizzled shared memory -> TMA store
// Each tile is a sequence of ring slots: K/256 FP4 slots, then ceil(r/32)
// low-rank slots holding an L2 chunk and the matching xl1 chunk [128 rows x 32]
// float32 (both by TMA), which the quadrant warps turn in place into the bf16
// hi + lo operand (each warp's 32 rows read and write the same 4 KB). A slot's "full" barrier (the leader's) counts the
// leader's producer, whose expected bytes cover both CTAs' loads; a low-rank
// slot's operand tiles are announced on the slot's "ready" barrier (the
// leader's) by every staging warp of the pair; the MMA commit frees the slot
// in both CTAs.
// Scale factors: copying them into tensor memory with tcgen05.cp puts the copies
// in the MMA issuer's queue, and they run serialised with the MMAs (three 512-byte
// copies per 64-wide K block nearly double the time of its MMA). Instead the four
// quadrant warps write them with tcgen05.st, which runs beside the MMAs: each warp
// reads the slot's scale atoms from shared memory (each CTA loads its own copy,
// announced on its own "sf landed" barrier) and stores the 32-lane pattern into
// its own lane quadrant (every quadrant holds the same 32 lanes, the layout
// tcgen05.cp .32x128b.warpx4 would produce). Two 48-column scale buffers
// alternate between 4-bit slots: "sf full" (the leader's, counting every quadrant
// warp of the pair) lets the MMA issuer in, "sf free" (committed after the slot's
// MMAs) lets the warps refill the buffer. The MMA issuer is one thread whose
// instruction latency paces the tensor pipe, so its loop is kept lean: operand
// descriptors are built once and advanced by constant offsets.
// Tensor-memory columns: two 256-column accumulators overlapping by 96 columns
// ([0, 256) and [160, 416)), the two scale buffers in [416, 512). The epilogue
// drains the overlapped columns of a tile first and releases them, so the next
// tile's MMAs start while the rest of the tile is still being stored.
//
// Fused QKV epilogue (kQkNorm; Diffusers blog, the fused QKV section: one to_qkv
// linear whose output is Q, then K, then V, each head of Q and K normalised by
// norm_q / norm_k and then rotated by the rotary embedding, in one fused call).
// Heads are 128 columns, so a 256-column tile holds two whole heads. Each row's
// head is split between the quadrant's two epilogue warps: each warp sums the
// squares of its columns of each head (y = alpha acc + bias in float32), the two
// trade their partial sums through shared memory behind a per-quadrant
// mbarrier, and each then scales its columns by rsqrt(mean + eps) and the head's
// weight and turns adjacent pairs (2i, 2i+1) by the row's angle i. The angle
// tables are angle-major ([64, M]): a lane holds one row, so for each angle the
// warp's 32 rows read one contiguous 128-byte run (row-major tables would cost
// a cache line per lane and load). Overlapped sub-tiles are released after
// their first load as usual and kept in registers; the others are read from
// tensor memory twice. V heads take the plain path.
#pragma once

#include "sm100.cuh"

namespace svdq {

constexpr int kGmThreads = 448;
constexpr int kGmEpiWarps = 8;
constexpr int kGmStageOut = 4096;                // epilogue staging bytes per warp
constexpr int kGmBM = 128, kGmBN = 256;          // rows per CTA, columns per tile
constexpr int kGmBKBytes = 128;                  // 256 FP4 values per row per stage
constexpr int kGmAStage = kGmBM * kGmBKBytes;    // 16 KB
constexpr int kGmSfaStage = 4 * 512;             // 4 atoms (one per 64-wide K block)
constexpr int kGmSfbStage = 2 * 4 * 512;         // 2 row blocks x 4 atoms
constexpr int kGmLrK = 32;                       // low-rank K per ring slot
constexpr int kGmLrATile = kGmBM * kGmLrK * 2;   // 8 KB per bf16 tile (hi, lo)
// tensor-memory columns: accumulators at 0 and kTmAcc1 (kTmOverlap shared); scale
// buffer b at kTmSf + kTmSfBuf b: 16 columns of A scales (4 per K block), then 32 of
// B scales (8 per K block: two 128-row atoms of 4)
constexpr uint32_t kTmAcc1 = 160, kTmOverlap = 96, kTmSf = 416, kTmSfBuf = 48, kTmCols = 512;
static_assert(kTmAcc1 + 256 <= kTmSf && kTmSf + 2 * kTmSfBuf <= kTmCols, "tensor-memory layout");
static_assert(256 - kTmOverlap == kTmAcc1, "the accumulators overlap by kTmOverlap columns");

template <bool kPair, bool kQkNorm = false>
struct GmCfg {
  static constexpr int kCtas = kPair ? 2 : 1;
  static constexpr int kBRows = kGmBN / kCtas;                // B rows staged per CTA
  static constexpr int kBStage = kBRows * kGmBKBytes;
  static constexpr int kStageBytes = kGmAStage + kBStage + kGmSfaStage + kGmSfbStage;
  static constexpr int kStages = kPair ? 4 : 3;
  static constexpr int kLrBTile = kGmLrK * kBRows * 2;        // L2 chunk, slot offset 0
  static constexpr uint32_t kOut = kStages * kStageBytes;     // 1024-aligned
  static constexpr uint32_t kBias = kOut + kGmEpiWarps * kGmStageOut;
  static constexpr uint32_t kBars = kBias + kGmEpiWarps * 128 * 4;
  // full, empty, ready, sf landed per stage; acc full, acc free; sf full, sf free per buffer
  static constexpr uint32_t kTmemSlot = kBars + 8 * (4 * kStages + 2 + 2 * 2);
  // fused QKV epilogue only: head weights per epilogue warp [4][32] float32, the
  // partial sums of squares [2 phases][4 quadrants][2 warps][2 heads][32 rows],
  // one exchange barrier per quadrant, and a 32 x 32 float32 sub-tile parked by
  // each of the first half's four epilogue warps
  static constexpr uint32_t kGamma = kTmemSlot + 16;
  static constexpr uint32_t kRed = kGamma + kGmEpiWarps * 128 * 4;
  static constexpr uint32_t kNormBars = kRed + 2 * 4 * 2 * 2 * 32 * 4;
  static constexpr uint32_t kPark = kNormBars + 4 * 8;
  static constexpr size_t kSmemBytes = (kQkNorm ? kPark + 4 * 4096 : kTmemSlot + 16) + 1024;
  static_assert(kStageBytes % 1024 == 0, "stages must stay 1024-byte aligned");
  static_assert(kLrBTile + 2 * kGmLrATile <= kStageBytes, "a low-rank slot fits in a stage");
};

struct GemmParams {
  int M, N, K, r;
  int tiles_m, tiles;      // tiles of kCtas * 128 rows x 256 columns
  const __nv_bfloat16* bias;
  // two-level NVFP4: the activation and weight tensor scales s_t (device), or null;
  // Y = RN32(s_a s_w) * (4-bit product) + xl1 L2 + bias
  const float* a_tscale;
  const float* w_tscale;
  int out_f32;
  uint32_t* status;
  // fused QKV epilogue (kQkNorm): q_heads heads of 128 columns each of Q and K
  // (columns [0, 128 q_heads) and [128 q_heads, 256 q_heads)); head weights
  // [128] bf16 or null (1); rotation tables cos, sin [64, M] float32 (angle-major) or null
  int q_heads;
  float eps;
  const __nv_bfloat16* norm_q;
  const __nv_bfloat16* norm_k;
  const float* rope_cos;
  const float* rope_sin;
};

template <bool kPair, bool kQkNorm = false>
__global__ void __launch_bounds__(kGmThreads, 1)
    w4a4_nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tm_a,
                           const __grid_constant__ CUtensorMap tm_b,
                           const __grid_constant__ CUtensorMap tm_sfa,
                           const __grid_constant__ CUtensorMap tm_sfb,
                           const __grid_constant__ CUtensorMap tm_l2,
                           const __grid_constant__ CUtensorMap tm_xl1,
                           const __grid_constant__ CUtensorMap tm_y, const GemmParams p) {
  using Cfg = GmCfg<kPair, kQkNorm>;
  constexpr int NS = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = kPair ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;

  const int kblocks = p.K / 64;                      // 64-wide scale atoms along K
  const int ktiles = (kblocks + 3) / 4;
  const int lr_chunks = (p.r + kGmLrK - 1) / kGmLrK;
  const int slots = ktiles + lr_chunks;              // ring slots per tile
  const int unit = blockIdx.x / Cfg::kCtas;          // this CTA (pair)'s scheduling unit
  const int units = gridDim.x / Cfg::kCtas;
  // this unit's tiles: unit, unit + units, ...; M fastest
  const int my_tiles = p.tiles > unit ? (p.tiles - 1 - unit) / units + 1 : 0;
  auto tile_mn = [&](int i, int& m0, int& n0) {
    const int t = unit + i * units;
    m0 = (t % p.tiles_m) * (kGmBM * Cfg::kCtas);
    n0 = (t / p.tiles_m) * kGmBN;
  };

  auto stage = [&](int s) { return sbase + s * Cfg::kStageBytes; };
  auto a_st = [&](int s) { return stage(s); };
  auto b_st = [&](int s) { return stage(s) + kGmAStage; };
  auto sfa_st = [&](int s) { return stage(s) + kGmAStage + Cfg::kBStage; };
  auto sfb_st = [&](int s) { return sfa_st(s) + kGmSfaStage; };
  auto bar_full = [&](int s) { return sbase + Cfg::kBars + 8 * s; };
  auto bar_empty = [&](int s) { return sbase + Cfg::kBars + 8 * (NS + s); };
  auto bar_ready = [&](int s) { return sbase + Cfg::kBars + 8 * (2 * NS + s); };
  auto bar_sf_landed = [&](int s) { return sbase + Cfg::kBars + 8 * (3 * NS + s); };
  const uint32_t bar_acc_full = sbase + Cfg::kBars + 8 * (4 * NS);
  const uint32_t bar_acc_free = bar_acc_full + 8;
  auto bar_sf_full = [&](int b) { return bar_acc_full + 16 + 8 * b; };
  auto bar_sf_free = [&](int b) { return bar_acc_full + 32 + 8 * b; };
  // the leader's copies of the pipeline barriers, as seen from this CTA
  auto lead = [&](uint32_t a) { return kPair ? map_peer_smem(a, 0) : a; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::kTmemSlot);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar_full(s), 1);                  // leader producer (with tx)
      mbar_init(bar_ready(s), 4 * Cfg::kCtas);    // staging warps of a low-rank slot
      mbar_init(bar_empty(s), 1);
      mbar_init(bar_sf_landed(s), 1);             // this CTA's producer (with tx)
    }
    mbar_init(bar_acc_full, 1);
    mbar_init(bar_acc_free, kGmEpiWarps * Cfg::kCtas);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_sf_full(b), 4 * Cfg::kCtas);  // quadrant warps of the pair
      mbar_init(bar_sf_free(b), 1);               // MMA commit
    }
    if constexpr (kQkNorm)
      for (int q = 0; q < 4; ++q) mbar_init(sbase + Cfg::kNormBars + 8 * q, 2);  // a quadrant's two epilogue warps
    fence_barrier_init();
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    prefetch_tmap(&tm_sfa);
    prefetch_tmap(&tm_sfb);
    prefetch_tmap(&tm_y);
    if (p.r > 0) {
      prefetch_tmap(&tm_l2);
      prefetch_tmap(&tm_xl1);
    }
  }
  if (warp == 1) {
    if (kPair) {
      tmem_alloc_pair(smem_u32(tmem_slot), kTmCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_slot), kTmCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if (kPair) cluster_sync_converged(); else cta_sync_converged();  // barriers initialised in both CTAs
  // everything above touches no global memory the previous grid may write
  grid_dep_wait();
  grid_dep_launch();
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
        const int mrow = m0 + kGmBM * static_cast<int>(rank);        // this CTA's A rows
        const int nrow = n0 + Cfg::kBRows * static_cast<int>(rank);  // this CTA's B rows
        for (int kt = 0; kt < slots && ok; ++kt, ++kt_global) {
          const int s = kt_global % NS;
          ok = mbar_wait(bar_empty(s), ((kt_global / NS) & 1) ^ 1, p.status);
          if (!ok) break;
          const uint32_t fb = lead(bar_full(s));
          auto load = [&](uint32_t dst, const CUtensorMap* m, int c0, int c1) {
            if (kPair) tma_load_2d_pair(dst, m, fb, c0, c1);
            else tma_load_2d(dst, m, fb, c0, c1);
          };
          if (kt < ktiles) {
            if (leader)
              mbar_arrive_expect_tx(bar_full(s), Cfg::kCtas * (kGmAStage + Cfg::kBStage));
            load(a_st(s), &tm_a, kt * kGmBKBytes, mrow);
            load(b_st(s), &tm_b, kt * kGmBKBytes, nrow);
            // scale atoms, viewed as rows of 256 B (4 atoms = 8 rows): this CTA's
            // own copy, for its quadrant warps, on its own barrier
            const uint32_t sl = bar_sf_landed(s);
            mbar_arrive_expect_tx(sl, kGmSfaStage + kGmSfbStage);
            tma_load_2d(sfa_st(s), &tm_sfa, sl, 0, ((mrow / 128) * kblocks + 4 * kt) * 2);
            for (int j = 0; j < 2; ++j)
              tma_load_2d(sfb_st(s) + j * 2048, &tm_sfb, sl, 0, ((n0 / 128 + j) * kblocks + 4 * kt) * 2);
          } else {
            // low-rank slot: xl1 rows of this CTA x columns [32 c, 32 c + 32), float32
            // with 128-byte swizzle (rows past M and columns past r read as zero), on
            // this CTA's own barrier for its quadrant warps
            const int c = kt - ktiles;
            const uint32_t sl = bar_sf_landed(s);
            mbar_arrive_expect_tx(sl, kGmBM * kGmLrK * 4);
            tma_load_2d(stage(s) + Cfg::kLrBTile, &tm_xl1, sl, c * kGmLrK, mrow);
            // L2 rows [32 c, 32 c + 32) x this CTA's columns, 64-wide boxes (rows
            // past r read as zero)
            if (leader) mbar_arrive_expect_tx(bar_full(s), kGmLrK * kGmBN * 2);
            for (int nb = 0; nb < Cfg::kBRows / 64; ++nb)
              load(stage(s) + nb * (kGmLrK * 128), &tm_l2, nrow + nb * 64, c * kGmLrK);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (leader && elect_one()) {
      bool ok = true;
      const uint32_t mma_m = kGmBM * Cfg::kCtas;
      const uint32_t id_lr = idesc_bf16_f32(mma_m, kGmBN, false, true);
      const uint32_t id_fp4 = idesc_nvfp4(mma_m, kGmBN);
      int kt_global = 0;
      int fp4 = 0;           // 4-bit slots issued so far: fp4 & 1 is the scale buffer
      // operand descriptors of ring stage 0; stage s is kStageBytes further (>> 4)
      const uint64_t a_desc0 = smem_desc(a_st(0), 16, 1024, kSwizzle128B);
      const uint64_t b_desc0 = smem_desc(b_st(0), 16, 1024, kSwizzle128B);
      constexpr uint64_t kStageStep = static_cast<uint64_t>(Cfg::kStageBytes >> 4);
      uint32_t lr_uses = 0;  // bit s: parity of the low-rank uses of ring slot s so far
      for (int i = 0; i < my_tiles && ok; ++i) {
        const uint32_t acc = tmem + ((i & 1) ? kTmAcc1 : 0u);
        // the previous tile's epilogues (both CTAs) drained the overlapped columns
        if (i > 0) {
          ok = mbar_wait(bar_acc_free, (i - 1) & 1, p.status);
          if (!ok) break;
        }
        tc_fence_after();
        for (int kt = 0; kt < slots && ok; ++kt, ++kt_global) {
          const int s = kt_global % NS;
          ok = mbar_wait(bar_full(s), (kt_global / NS) & 1, p.status);
          if (!ok) break;
          tc_fence_after();
          if (kt < ktiles) {
            // this slot's scale factors are in tensor memory (both CTAs)
            const uint32_t buf = static_cast<uint32_t>(fp4 & 1);
            ok = mbar_wait(bar_sf_full(buf), (fp4 >> 1) & 1, p.status);
            if (!ok) break;
            tc_fence_after();
            const uint32_t sfa = tmem + kTmSf + kTmSfBuf * buf, sfb = sfa + 16;
            const uint64_t ad = a_desc0 + kStageStep * static_cast<uint64_t>(s);
            const uint64_t bd = b_desc0 + kStageStep * static_cast<uint64_t>(s);
            const uint32_t acc0 = kt > 0 ? 1u : 0u;
            // K block kb starts 32 bytes (2 in descriptor units) further along the row
            if (kblocks - 4 * kt >= 4) {
              if (kPair) {
                mma_nvfp4_pair(acc, ad, bd, id_fp4, sfa, sfb, acc0);
                mma_nvfp4_pair(acc, ad + 2, bd + 2, id_fp4, sfa + 4, sfb + 8, 1u);
                mma_nvfp4_pair(acc, ad + 4, bd + 4, id_fp4, sfa + 8, sfb + 16, 1u);
                mma_nvfp4_pair(acc, ad + 6, bd + 6, id_fp4, sfa + 12, sfb + 24, 1u);
              } else {
                mma_nvfp4(acc, ad, bd, id_fp4, sfa, sfb, acc0);
                mma_nvfp4(acc, ad + 2, bd + 2, id_fp4, sfa + 4, sfb + 8, 1u);
                mma_nvfp4(acc, ad + 4, bd + 4, id_fp4, sfa + 8, sfb + 16, 1u);
                mma_nvfp4(acc, ad + 6, bd + 6, id_fp4, sfa + 12, sfb + 24, 1u);
              }
            } else {
              const int nkb = kblocks - 4 * kt;
              for (int kb = 0; kb < nkb; ++kb) {
                const uint32_t accum = (kt > 0 || kb > 0) ? 1u : 0u;
                if (kPair)
                  mma_nvfp4_pair(acc, ad + 2 * kb, bd + 2 * kb, id_fp4, sfa + 4 * kb, sfb + 8 * kb, accum);
                else
                  mma_nvfp4(acc, ad + 2 * kb, bd + 2 * kb, id_fp4, sfa + 4 * kb, sfb + 8 * kb, accum);
              }
            }
            // the scale buffer is free once this slot's MMAs are done
            if (kPair) tc_commit_pair(bar_sf_free(buf), 0x3);
            else tc_commit(bar_sf_free(buf));
            ++fp4;
          } else {
            ok = mbar_wait(bar_ready(s), (lr_uses >> s) & 1u, p.status);
            lr_uses ^= 1u << s;
            if (!ok) break;
            tc_fence_after();
            // low-rank slot: B = L2 chunk (MN-major, 128-byte swizzle; 64-wide N
            // blocks 4096 B apart = LBO, 8-deep K groups 1024 B apart = SBO);
            // A = xl1 hi / lo (no-swizzle K-major: K-adjacent core matrices 128 B
            // apart = LBO; each 8-row group holds 512 B of hi, then 512 B of lo, so
            // groups are 1024 B apart = SBO)
            const uint32_t a_lr = stage(s) + Cfg::kLrBTile;
#pragma unroll
            for (int kk = 0; kk < kGmLrK / 16; ++kk) {
              const uint64_t bd = smem_desc(stage(s) + kk * 2048, kGmLrK * 128, 1024, kSwizzle128B);
              const uint64_t ah = smem_desc(a_lr + kk * 256, 128, 1024, kSwizzleNone);
              const uint64_t al = smem_desc(a_lr + 512 + kk * 256, 128, 1024, kSwizzleNone);
              if (kPair) {
                mma_f16_pair(acc, ah, bd, id_lr, 1u);
                mma_f16_pair(acc, al, bd, id_lr, 1u);
              } else {
                mma_f16(acc, ah, bd, id_lr, 1u);
                mma_f16(acc, al, bd, id_lr, 1u);
              }
            }
          }
          if (kPair) tc_commit_pair(bar_empty(s), 0x3);
          else tc_commit(bar_empty(s));
        }
        if (kPair) tc_commit_pair(bar_acc_full, 0x3);
        else tc_commit(bar_acc_full);
      }
    }
  } else if (warp < 6) {
    // ---------------------------------------- scale factors and low-rank staging
    const int quad = warp & 3;
    const int trow = quad * 32 + lane;
    const uint32_t sf_lanes = tmem + kTmSf + (static_cast<uint32_t>(quad * 32) << 16);
    // two-level NVFP4: the low-rank branch shares the accumulator that the epilogue
    // multiplies by alpha, so xl1 enters divided by it
    const float alpha_inv =
        p.a_tscale != nullptr ? __frcp_rn(__fmul_rn(p.a_tscale[0], p.w_tscale[0])) : 1.0f;
    bool ok = true;
    int kt_global = 0;
    int fp4 = 0;  // 4-bit slots handled so far: fp4 & 1 is the scale buffer
    for (int i = 0; i < my_tiles && ok; ++i) {
      // 4-bit slots: place the scale factors. The slot's "empty" phases are still
      // waited in order: a parity wait is only meaningful one phase at a time, so
      // skipping ahead could pass a phase that has not come yet.
      for (int kt = 0; kt < ktiles && ok; ++kt, ++kt_global, ++fp4) {
        const int s = kt_global % NS;
        const int buf = fp4 & 1;
        ok = mbar_wait(bar_empty(s), ((kt_global / NS) & 1) ^ 1, p.status) &&
             mbar_wait(bar_sf_landed(s), (kt_global / NS) & 1, p.status);
        // lane l: the 16 bytes at l * 16 of each scale atom (rows l, l + 32, l + 64,
        // l + 96 of its 128-row block, 4 scales each) -> 4 columns per atom; read
        // before waiting for the buffer
        uint32_t sa[16], sbv[32];
        if (ok) {
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {
            const uint4 a = lds_u4(sfa_st(s) + kb * 512 + lane * 16);
            sa[4 * kb] = a.x; sa[4 * kb + 1] = a.y; sa[4 * kb + 2] = a.z; sa[4 * kb + 3] = a.w;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const uint4 v = lds_u4(sfb_st(s) + j * 2048 + kb * 512 + lane * 16);
              sbv[8 * kb + 4 * j] = v.x; sbv[8 * kb + 4 * j + 1] = v.y;
              sbv[8 * kb + 4 * j + 2] = v.z; sbv[8 * kb + 4 * j + 3] = v.w;
            }
          }
        }
        ok = ok && (fp4 < 2 || mbar_wait(bar_sf_free(buf), ((fp4 >> 1) - 1) & 1, p.status));
        ok = __all_sync(0xffffffffu, ok);  // tcgen05.st below needs the whole warp
        if (!ok) break;
        tc_fence_after();
        const uint32_t dst = sf_lanes + kTmSfBuf * static_cast<uint32_t>(buf);
        tmem_st16(dst, sa);
        tmem_st32(dst + 16, sbv);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          // the pair's MMAs read this CTA's scale columns through this SM's own
          // tensor core: the completed stores are ordered for them by the fence
          // and a CTA-scope release, as for the low-rank operand tiles
          if (kPair) mbar_arrive_remote(lead(bar_sf_full(buf)));
          else mbar_arrive(bar_sf_full(buf));
        }
      }
      for (int c = 0; c < lr_chunks && ok; ++c, ++kt_global) {
        const int s = kt_global % NS;
        ok = mbar_wait(bar_empty(s), ((kt_global / NS) & 1) ^ 1, p.status) &&
             mbar_wait(bar_sf_landed(s), (kt_global / NS) & 1, p.status);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        // this lane's row of the float32 chunk (128 B, 16-byte units swizzled by row % 8)
        const uint32_t lr = stage(s) + Cfg::kLrBTile;
        float v[kGmLrK];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 f = lds_f4(lr + trow * 128 + ((q ^ (trow & 7)) << 4));
          v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
        }
        __syncwarp();  // the warp's 4 KB is read before any lane overwrites it
#pragma unroll
        for (int q = 0; q < kGmLrK; ++q) v[q] = __fmul_rn(v[q], alpha_inv);  // exact when 1
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
        if (lane == 0) {
          // The leader's pair MMA reads this CTA's rows through this SM's own
          // tensor core from this CTA's shared memory: the writes above are
          // ordered for it by the proxy fence and a CTA-scope release.
          if (kPair) mbar_arrive_remote(lead(bar_ready(s)));
          else mbar_arrive(bar_ready(s));
        }
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
    const uint32_t out_buf = sbase + Cfg::kOut + (warp - 6) * kGmStageOut;
    float* bias_s = reinterpret_cast<float*>(smem + Cfg::kBias) + (warp - 6) * 128;  // [4][32]
    const uint32_t free_bar = lead(bar_acc_free);
    bool ok = true;
    int stores = 0;
    const float alpha = p.a_tscale != nullptr ? __fmul_rn(p.a_tscale[0], p.w_tscale[0]) : 1.0f;
    // stage the warp's 32 x 32 sub-tile (its rows, columns n0 + j0 ..) in the TMA
    // store's swizzled layout and store it
    auto store_sub = [&](const float (&y)[32], int n0, int j0, int mrow) {
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
        tma_store_2d(&tm_y, buf, n0 + j0, mrow + quad * 32);
        bulk_commit();
      }
      ++stores;
    };
    // y = alpha * acc + bias for one sub-tile, one rounding (alpha = 1 without
    // tensor scales: the plain sum); with two-level scales the accumulator holds
    // the 4-bit product and the low-rank term divided by alpha
    auto finish = [&](const uint32_t (&acc)[32], int t, float (&y)[32]) {
      const float4* bv = reinterpret_cast<const float4*>(bias_s + t * 32);
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4) {
        const float4 b = bv[q4];
        y[4 * q4 + 0] = __fmaf_rn(__uint_as_float(acc[4 * q4 + 0]), alpha, b.x);
        y[4 * q4 + 1] = __fmaf_rn(__uint_as_float(acc[4 * q4 + 1]), alpha, b.y);
        y[4 * q4 + 2] = __fmaf_rn(__uint_as_float(acc[4 * q4 + 2]), alpha, b.z);
        y[4 * q4 + 3] = __fmaf_rn(__uint_as_float(acc[4 * q4 + 3]), alpha, b.w);
      }
    };
    int nt = 0;  // fused-norm tiles so far: the phase of this quadrant's exchange barrier
    for (int i = 0; i < my_tiles && ok; ++i) {
      int m0, n0;
      tile_mn(i, m0, n0);
      const int mrow = m0 + kGmBM * static_cast<int>(rank);
      const bool odd = i & 1;
      const uint32_t t_row = tmem + (odd ? kTmAcc1 : 0u) + (static_cast<uint32_t>(quad * 32) << 16);
      // sub-tile order: the overlapped ones first (two in the first half's warps,
      // one in the second's), then the five others
      int sub_col[4];
      const int ovl = odd ? 0 : kGmBN - kTmOverlap;   // first overlapped column
      const int other0 = odd ? kTmOverlap : 0;        // first non-overlapped column
      if (half == 0) {
        sub_col[0] = ovl;
        sub_col[1] = ovl + 64;
        sub_col[2] = other0;
        sub_col[3] = other0 + 32;
      } else {
        sub_col[0] = ovl + 32;
        sub_col[1] = other0 + 64;
        sub_col[2] = other0 + 96;
        sub_col[3] = other0 + 128;
      }
      const bool norm_tile = kQkNorm && n0 < 256 * p.q_heads;  // holds a Q or K head
      // bias (and head weights) for this warp's sub-tiles, fetched before the
      // accumulator is ready
      __syncwarp();
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int n = n0 + sub_col[t] + lane;
        bias_s[t * 32 + lane] = (p.bias != nullptr && n < p.N) ? __bfloat162float(p.bias[n]) : 0.0f;
      }
      if constexpr (kQkNorm) {
        if (norm_tile) {
          float* gamma_s = reinterpret_cast<float*>(smem + Cfg::kGamma) + (warp - 6) * 128;
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int g = n0 / 128 + (sub_col[t] >> 7);  // global head
            const __nv_bfloat16* w =
                g < p.q_heads ? p.norm_q : (g < 2 * p.q_heads ? p.norm_k : nullptr);
            gamma_s[t * 32 + lane] = w != nullptr ? __bfloat162float(w[(sub_col[t] & 127) + lane]) : 1.0f;
          }
        }
      }
      __syncwarp();
      ok = mbar_wait(bar_acc_full, i & 1, p.status);
      if (!ok) break;
      tc_fence_after();
      if constexpr (kQkNorm) {
        if (norm_tile) {
          // The overlapped sub-tiles are released once read: the first stays in
          // registers, the first half's second is parked, as y, in shared memory.
          uint32_t h0[32];
          const uint32_t park = sbase + Cfg::kPark + quad * 4096;  // first-half warps only
          float ss0 = 0.0f, ss1 = 0.0f;  // the row's sums of squares over this warp's columns of either head
          auto add_sq = [&](const float (&y)[32], int t) {
            float sq = 0.0f;
#pragma unroll
            for (int q = 0; q < 32; ++q) sq = __fmaf_rn(y[q], y[q], sq);
            if (sub_col[t] < 128) ss0 += sq;
            else ss1 += sq;
          };
          if (half == 0) {
            // the second overlapped sub-tile first: to y, into the sums, parked
            uint32_t h1[32];
            tmem_ld32(t_row + sub_col[1], h1);
            tmem_ld_wait();
            if (mrow < p.M) {
              float y[32];
              finish(h1, 1, y);
              add_sq(y, 1);
#pragma unroll
              for (int c = 0; c < 8; ++c)
                asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(
                                 park + lane * 128 + ((c ^ (lane & 7)) << 4)),
                             "f"(y[4 * c]), "f"(y[4 * c + 1]), "f"(y[4 * c + 2]), "f"(y[4 * c + 3])
                             : "memory");
            }
          }
          tmem_ld32(t_row + sub_col[0], h0);
          tmem_ld_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if (kPair) mbar_arrive_remote(free_bar);
            else mbar_arrive(free_bar);
          }
          if (mrow >= p.M) continue;  // the same for both warps of the quadrant
          // pass 1: the rest of the sums of squares
          {
            float y[32];
            finish(h0, 0, y);
            add_sq(y, 0);
          }
#pragma unroll
          for (int t = 1; t < 4; ++t) {
            if (t == 1 && half == 0) continue;
            uint32_t acc[32];
            tmem_ld32(t_row + sub_col[t], acc);
            tmem_ld_wait();
            float y[32];
            finish(acc, t, y);
            add_sq(y, t);
          }
          // trade the partial sums with the quadrant's other warp (two phases of
          // slots: a warp can be at most one tile ahead of its partner)
          float* red = reinterpret_cast<float*>(smem + Cfg::kRed);
          float* mine = red + (((nt & 1) * 4 + quad) * 2 + half) * 64;
          const float* theirs = red + (((nt & 1) * 4 + quad) * 2 + (half ^ 1)) * 64;
          mine[lane] = ss0;
          mine[32 + lane] = ss1;
          __syncwarp();
          const uint32_t xbar = sbase + Cfg::kNormBars + 8 * quad;
          if (lane == 0) mbar_arrive(xbar);
          ok = mbar_wait(xbar, nt & 1, p.status);
          ++nt;
          if (!ok) break;
          const float rs0 = rsqrtf(__fmaf_rn(ss0 + theirs[lane], 1.0f / 128.0f, p.eps));
          const float rs1 = rsqrtf(__fmaf_rn(ss1 + theirs[32 + lane], 1.0f / 128.0f, p.eps));
          // pass 2: scale, weight, rotate, store. src 0: h0; 1: the parked y; 2: tensor memory
          const float* gamma_s = reinterpret_cast<const float*>(smem + Cfg::kGamma) + (warp - 6) * 128;
          const int m = mrow + quad * 32 + lane;
          const int tcol = m < p.M ? m : 0;  // the row's place in the tables; rows past M: any valid row
          auto emit = [&](int t, int src) {
            const int j0 = sub_col[t];
            float y[32];
            if (src == 0) {
              finish(h0, t, y);
            } else if (src == 1) {
#pragma unroll
              for (int c = 0; c < 8; ++c)
                asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                             : "=f"(y[4 * c]), "=f"(y[4 * c + 1]), "=f"(y[4 * c + 2]), "=f"(y[4 * c + 3])
                             : "r"(park + lane * 128 + ((c ^ (lane & 7)) << 4))
                             : "memory");
            } else {
              uint32_t acc[32];
              tmem_ld32(t_row + j0, acc);
              tmem_ld_wait();
              finish(acc, t, y);
            }
            if (n0 / 128 + (j0 >> 7) < 2 * p.q_heads) {
              // paired float32 instructions; each lane rounds as the scalar form would
              const float rs = j0 < 128 ? rs0 : rs1;
              const float2 rs2 = make_float2(rs, rs);
              const float4* gv = reinterpret_cast<const float4*>(gamma_s + t * 32);
#pragma unroll
              for (int q4 = 0; q4 < 8; ++q4) {
                const float4 w = gv[q4];
                const float2 lo = __fmul2_rn(__fmul2_rn(make_float2(y[4 * q4 + 0], y[4 * q4 + 1]), rs2),
                                             make_float2(w.x, w.y));
                const float2 hi = __fmul2_rn(__fmul2_rn(make_float2(y[4 * q4 + 2], y[4 * q4 + 3]), rs2),
                                             make_float2(w.z, w.w));
                y[4 * q4 + 0] = lo.x;
                y[4 * q4 + 1] = lo.y;
                y[4 * q4 + 2] = hi.x;
                y[4 * q4 + 3] = hi.y;
              }
              if (p.rope_cos != nullptr) {
                // the sub-tile's 16 pairs are angles a0 .. a0 + 15 of the row, a0 = (j0 mod
                // 128) / 2; the tables are angle-major, so for each angle the warp's 32
                // consecutive rows are one contiguous 128-byte run
                const size_t a0 = static_cast<size_t>((j0 & 127) >> 1) * p.M + tcol;
                const size_t am = static_cast<size_t>(p.M);
                // (x, z) -> (x c - RN(z s), z c + RN(x s)): the products (-z s, x s) as one
                // paired multiply, then one paired fused multiply-add
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                  const float c = __ldg(p.rope_cos + a0 + i * am), sn = __ldg(p.rope_sin + a0 + i * am);
                  const float2 zx = __fmul2_rn(make_float2(y[2 * i + 1], y[2 * i]), make_float2(-sn, sn));
                  const float2 r = __ffma2_rn(make_float2(y[2 * i], y[2 * i + 1]), make_float2(c, c), zx);
                  y[2 * i] = r.x;
                  y[2 * i + 1] = r.y;
                }
              }
            }
            if (n0 + j0 >= p.N) return;
            store_sub(y, n0, j0, mrow);
          };
          emit(0, 0);
          emit(1, half == 0 ? 1 : 2);
          emit(2, 2);
          emit(3, 2);
          continue;
        }
      }
      uint32_t acc_next[32];  // the first half's second overlapped sub-tile
      for (int t = 0; t < 4; ++t) {
        const int j0 = sub_col[t];
        uint32_t acc[32];
        if (t == 1 && half == 0) {
#pragma unroll
          for (int q = 0; q < 32; ++q) acc[q] = acc_next[q];
        } else {
          tmem_ld32(t_row + j0, acc);
          if (t == 0 && half == 0) tmem_ld32(t_row + sub_col[1], acc_next);
          tmem_ld_wait();
        }
        if (t == 0) {
          // this warp's overlapped columns are in registers: let the next tile's MMAs in
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if (kPair) mbar_arrive_remote(free_bar);  // hands over no memory contents
            else mbar_arrive(free_bar);
          }
        }
        if (n0 + j0 >= p.N || mrow >= p.M) continue;  // warp-uniform
        float y[32];
        finish(acc, t, y);
        store_sub(y, n0, j0, mrow);
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
    if (kPair) tmem_dealloc_pair(tmem, kTmCols);
    else tmem_dealloc(tmem, kTmCols);
  }
}

}  // namespace svdq

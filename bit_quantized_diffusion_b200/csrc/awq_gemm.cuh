// awq_gemm.cuh -- step a7 on the tensor cores: the AWQ W4A16 linear for any
// token count (Diffusers blog, "From SVDQuant to Nunchaku Lite": awq_w4a16,
// int4 weights with a bf16 scale and zero point per 64 values along K, 16-bit
// activations, on the memory-bound modulation projections).
//
//   Y[m,n] = sum_g s[n,g] * D_g[n,m] + bias[n],   D_g[n,m] = sum_{k in g} (q[n,k] - z[n,g]) X[m,k]
//
// The integer part q - z lies in [-15, 15], so it is exact in bf16, and every
// product (q - z) X is exact in float32: the tensor core forms D_g for one
// 64-wide group at a time (kind::f16, float32 accumulate) into its own
// tensor-memory buffer, and the epilogue warps apply the group's scale with
// one float32 multiply-add per output, keeping the running sum in registers.
// The weights therefore enter the MMA as they are (no bf16 rounding of
// (q - z) s), and the converters do one byte select and one bf16 subtraction
// per pair of weights.
//
// Orientation: the MMA's M side is 128 weight rows (tensor-memory lanes) and
// its N side the token tile (16..128 tokens, tensor-memory columns), so a
// handful of tokens costs no padding beyond 16. One CTA per SM, persistent
// over (token tile, 128-row weight tile) pairs; each tile streams its rows'
// weights once.
//
// Weights are read in the fragment order of svdq_pack(AWQ) (the layout the
// small-M GEMV reads): per 16-row block and 64-wide group, 32 lanes x 16 bytes,
// lane (r0, t) holding rows r0 and r0 + 8, columns 2t, 2t + 1, 2t + 8, 2t + 9
// of each of the group's four 16-wide K steps. A converter warp takes a whole
// block: lane l reads lane l's 16 bytes (one conflict-free 16-byte load per
// lane) and writes its 32 weights as 4-byte bf16 pairs straight to their
// places in the A tile (128-byte swizzle, K-major), which is conflict-free too.
//
// Each group's partial sums get a tensor-memory buffer of their own, from a ring
// of 512 / tb buffers (16 at up to 32 tokens), so the tensor core can run that
// many groups ahead of the epilogue. The scales reach the epilogue through
// shared memory: the converters copy the group's 128 scales into a ring of 16
// slots, each announced on its own barrier and refilled once the epilogue has
// read it. The MMA issuer, the converters and the epilogue poll their barriers.
//
// Warp roles (26 warps):
//   warp 0       TMA producer: per group the 8 blocks' fragment words (4 KB),
//                their (s, z) pairs (512 B) and the X tile [T x 64] bf16
//                (128-byte swizzle, tokens past M read as zero)
//   warp 1       tensor-memory owner and MMA issuer (one thread)
//   warps 2-9    converters: codes -> bf16 (q - z) into the A tile, one
//                16-row block per warp per group; the group's scales
//   warps 10-25  epilogue: four per lane quadrant, each 32 (or 16) token columns
#pragma once

#include "sm100.cuh"

namespace svdq {

constexpr int kAgConvWarps = 8;
constexpr int kAgEpiWarps = 16;
constexpr int kAgThreads = 32 * (2 + kAgConvWarps + kAgEpiWarps);  // 832
constexpr int kAgRows = 128;                 // weight rows per tile (MMA M)
constexpr int kAgMaxT = 128;                 // tokens per tile (MMA N)
constexpr int kAgMaxBufs = 16;               // tensor-memory group buffers: 512 / tb of them
constexpr int kAgSlots = 16;                 // scale slots (a ring of its own)
constexpr int kAgATile = kAgRows * 128;      // bf16 [128 x 64], 16 KB
constexpr int kAgQBytes = 8 * 512;           // fragment words of 8 blocks
constexpr int kAgSzBytes = 8 * 64;           // (s, z) of 8 blocks
constexpr int kAgMaxStages = 8;

struct AgParams {
  int M, N, K;
  int T;               // token tile width: a multiple of 16, <= kAgMaxT
  int tb;              // tensor-memory columns per group buffer (32, 64 or 128)
  int nbuf;            // tensor-memory group buffers: 512 / tb
  int stages;
  int tiles_m, tiles;  // token tiles, all tiles (token tile fastest)
  const uint32_t* sz;  // (s, z) pairs in svdq_pack(AWQ) order, for the epilogue's scales
  const __nv_bfloat16* bias;
  __nv_bfloat16* Y;
  uint32_t* status;
};

// stage: A tile, X tile, fragment words, (s, z); 1024-byte aligned
__host__ __device__ constexpr uint32_t ag_stage_bytes(int T) {
  return (static_cast<uint32_t>(kAgATile + T * 128 + kAgQBytes + kAgSzBytes) + 1023u) / 1024u * 1024u;
}
__host__ __device__ constexpr uint32_t ag_bars_off(int T, int stages) {
  return static_cast<uint32_t>(stages) * ag_stage_bytes(T);
}
// barriers: full, ready, empty per stage; full, free, scales per buffer; then
// full, free per tensor-memory buffer; full, free per scale slot; then the
// tensor-memory slot (16 bytes) and the scale slots [kAgSlots][128] float32
__host__ __device__ constexpr uint32_t ag_svec_off(int T, int stages) {
  return ag_bars_off(T, stages) + 8 * (3 * stages + 2 * kAgMaxBufs + 2 * kAgSlots) + 16;
}
__host__ __device__ constexpr size_t ag_smem_bytes(int T, int stages) {
  return ag_svec_off(T, stages) + kAgSlots * kAgRows * 4 + 1024;
}

__device__ __forceinline__ uint32_t ag_prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// bf16x2 a - b, each half rounded to nearest (exact here: small integers)
__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// tm_q: qweight as [N/16 blocks][K/64 groups][64 x 8 bytes], box {64, 1, 8};
// tm_sz: (s, z) as [N/16][K/64][8 x 8 bytes], box {8, 1, 8}; tm_x: X [M, K]
// bf16, box {64, T}, 128-byte swizzle.
__global__ void __launch_bounds__(kAgThreads, 1)
    awq_gemm_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_sz,
                    const __grid_constant__ CUtensorMap tm_x, const AgParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int NS = p.stages, T = p.T;
  const int G = p.K / 64;
  const uint32_t SB = ag_stage_bytes(T);
  const int my_tiles = p.tiles > static_cast<int>(blockIdx.x)
                           ? (p.tiles - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                           : 0;
  auto tile_of = [&](int i, int& m0, int& n0) {
    const int t = static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x);
    m0 = (t % p.tiles_m) * kAgMaxT;
    n0 = (t / p.tiles_m) * kAgRows;
  };
  auto a_st = [&](int s) { return sbase + s * SB; };
  auto x_st = [&](int s) { return a_st(s) + kAgATile; };
  auto q_st = [&](int s) { return x_st(s) + T * 128; };
  auto sz_st = [&](int s) { return q_st(s) + kAgQBytes; };
  const uint32_t bars = sbase + ag_bars_off(T, NS);
  auto bar_full = [&](int s) { return bars + 8 * s; };              // producer (with tx)
  auto bar_ready = [&](int s) { return bars + 8 * (NS + s); };      // converters
  auto bar_empty = [&](int s) { return bars + 8 * (2 * NS + s); };  // MMA commit
  auto bar_dfull = [&](int b) { return bars + 8 * (3 * NS + b); };  // MMA commit
  auto bar_dfree = [&](int b) { return bars + 8 * (3 * NS + kAgMaxBufs + b); };  // epilogue warps
  auto bar_sfull = [&](int q) { return bars + 8 * (3 * NS + 2 * kAgMaxBufs + q); };  // converters
  auto bar_sfree = [&](int q) { return bars + 8 * (3 * NS + 2 * kAgMaxBufs + kAgSlots + q); };  // epilogue
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + ag_svec_off(T, NS) - 16);
  float* svec = reinterpret_cast<float*>(smem + ag_svec_off(T, NS));  // [kAgSlots][128] scales
  const int NB = p.nbuf;  // tensor-memory buffers of tb columns
  const int nslices = (T + 31) / 32;  // epilogue column slices of 32 (the last may hold 16)

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_ready(s), kAgConvWarps);
      mbar_init(bar_empty(s), 1);
    }
    for (int b = 0; b < NB; ++b) {
      mbar_init(bar_dfull(b), 1);
      mbar_init(bar_dfree(b), 4 * nslices);
    }
    for (int q = 0; q < kAgSlots; ++q) {
      mbar_init(bar_sfull(q), kAgConvWarps);
      mbar_init(bar_sfree(q), 4 * nslices);
    }
    fence_barrier_init();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_sz);
    prefetch_tmap(&tm_x);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), static_cast<uint32_t>(NB * p.tb));
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
      int gc = 0;  // groups issued so far (all tiles)
      for (int i = 0; i < my_tiles && ok; ++i) {
        int m0, n0;
        tile_of(i, m0, n0);
        for (int g = 0; g < G; ++g, ++gc) {
          const int s = gc % NS;
          ok = mbar_wait(bar_empty(s), ((gc / NS) & 1) ^ 1, p.status);
          if (!ok) break;
          mbar_arrive_expect_tx(bar_full(s), kAgQBytes + kAgSzBytes + T * 128);
          tma_load_3d(q_st(s), &tm_q, bar_full(s), 0, g, n0 / 16);
          tma_load_3d(sz_st(s), &tm_sz, bar_full(s), 0, g, n0 / 16);
          tma_load_2d(x_st(s), &tm_x, bar_full(s), g * 64, m0);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      bool ok = true;
      const uint32_t idesc = idesc_bf16_f32(kAgRows, static_cast<uint32_t>(T), false, false);
      int gc = 0;
      for (int i = 0; i < my_tiles && ok; ++i) {
        for (int g = 0; g < G; ++g, ++gc) {
          const int s = gc % NS, b = gc % NB;
          const uint32_t ph = (gc / NS) & 1;
          ok = mbar_wait_poll(bar_full(s), ph, p.status) && mbar_wait_poll(bar_ready(s), ph, p.status);
          // the epilogue has read this buffer's previous group
          if (ok && gc >= NB) ok = mbar_wait_poll(bar_dfree(b), ((gc / NB) - 1) & 1, p.status);
          if (!ok) break;
          tc_fence_after();
          const uint32_t d = tmem + static_cast<uint32_t>(b * p.tb);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            // 16 K = 32 bytes of each 128-byte swizzled row of the A (weights) and B (X) tiles
            const uint64_t ad = smem_desc(a_st(s) + kk * 32, 16, 1024, kSwizzle128B);
            const uint64_t bd = smem_desc(x_st(s) + kk * 32, 16, 1024, kSwizzle128B);
            mma_f16(d, ad, bd, idesc, kk > 0 ? 1u : 0u);
          }
          tc_commit(bar_empty(s));
          tc_commit(bar_dfull(b));
        }
      }
    }
  } else if (warp < 2 + kAgConvWarps) {
    // ------------------------------------------------------------ converters
    // Warp cw converts block cw of each group. Lane l = 4 r0 + t holds fragment
    // lane l's word for each K step ks: nibbles 8j + 4h of it are row r0 + 8h's
    // codes of columns 2t, 2t + 8, 2t + 1, 2t + 9 (j = 0..3). The lane's eight
    // destinations (K step, low or high half of the step) are fixed offsets in
    // the A tile, computed once; row r0 + 8 is 1024 bytes further.
    const int cw = warp - 2;
    const int r0 = lane >> 2, t = lane & 3;
    const uint32_t c43 = 0x43434343u;
    uint32_t aoff[8];
#pragma unroll
    for (int c = 0; c < 8; ++c)
      aoff[c] = static_cast<uint32_t>((16 * cw + r0) * 128 + t * 4) + (static_cast<uint32_t>(c ^ r0) << 4);
    bool ok = true;
    int gc = 0;
    for (int i = 0; i < my_tiles && ok; ++i) {
      for (int g = 0; g < G; ++g, ++gc) {
        const int s = gc % NS, bb = gc % kAgSlots;
        ok = mbar_wait_poll(bar_full(s), (gc / NS) & 1, p.status);
        // the epilogue has read this slot's previous scales
        if (ok && gc >= kAgSlots) ok = mbar_wait_poll(bar_sfree(bb), ((gc / kAgSlots) - 1) & 1, p.status);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        const uint4 w = lds_u4(q_st(s) + cw * 512 + lane * 16);
        const uint32_t sz0 = lds_u32(sz_st(s) + cw * 64 + r0 * 4);        // row r0
        const uint32_t sz8 = lds_u32(sz_st(s) + cw * 64 + (r0 + 8) * 4);  // row r0 + 8
        if (t == 0) {
          svec[bb * kAgRows + 16 * cw + r0] = __uint_as_float(sz0 << 16);
          svec[bb * kAgRows + 16 * cw + r0 + 8] = __uint_as_float(sz8 << 16);
        }
        // 128 + z as bf16 pairs: z is an integer 0..15, so bf16(128 + z) = 0x4300 + z
        const uint32_t z0 = static_cast<uint32_t>(__uint_as_float(sz0 & 0xFFFF0000u));
        const uint32_t z8 = static_cast<uint32_t>(__uint_as_float(sz8 & 0xFFFF0000u));
        const uint32_t zb0 = (0x4300u + z0) * 0x10001u, zb8 = (0x4300u + z8) * 0x10001u;
        const uint32_t words[4] = {w.x, w.y, w.z, w.w};
        const uint32_t ab = a_st(s);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint32_t e0 = words[ks] & 0x0F0F0F0Fu, e8 = (words[ks] >> 4) & 0x0F0F0F0Fu;
          // columns (2t, 2t + 1) in chunk 2 ks, (2t + 8, 2t + 9) in chunk 2 ks + 1
          const uint32_t lo = ab + aoff[2 * ks], hi = ab + aoff[2 * ks + 1];
          asm volatile("st.shared.b32 [%0], %1;" ::"r"(lo), "r"(bf16x2_sub(ag_prmt(e0, c43, 0x4240u), zb0)) : "memory");
          asm volatile("st.shared.b32 [%0], %1;" ::"r"(hi), "r"(bf16x2_sub(ag_prmt(e0, c43, 0x4341u), zb0)) : "memory");
          asm volatile("st.shared.b32 [%0+1024], %1;" ::"r"(lo), "r"(bf16x2_sub(ag_prmt(e8, c43, 0x4240u), zb8)) : "memory");
          asm volatile("st.shared.b32 [%0+1024], %1;" ::"r"(hi), "r"(bf16x2_sub(ag_prmt(e8, c43, 0x4341u), zb8)) : "memory");
        }
        fence_proxy_async_smem();  // the A tile is read by the tensor core (async proxy)
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar_ready(s));
          mbar_arrive(bar_sfull(bb));
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2 - kAgConvWarps;  // 0..15
    const int quad = warp & 3;                // tensor-memory lanes 32 quad .. + 31
    const int slice = ew >> 2;                // token columns 32 slice .. + 31
    const int ncol = T - 32 * slice < 32 ? T - 32 * slice : 32;  // 16 or 32 (or <= 0: idle)
    if (ncol > 0) {
      bool ok = true;
      int gc = 0;
      for (int i = 0; i < my_tiles && ok; ++i) {
        int m0, n0;
        tile_of(i, m0, n0);
        const int n = n0 + quad * 32 + lane;  // this lane's weight row
        const bool n_ok = n < p.N;
        float acc[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[j] = 0.0f;
        for (int g = 0; g < G; ++g, ++gc) {
          const int b = gc % NB, q = gc % kAgSlots;
          ok = mbar_wait_poll(bar_sfull(q), (gc / kAgSlots) & 1, p.status);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          const float sc = svec[q * kAgRows + quad * 32 + lane];  // this row's scale of group g
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_sfree(q));
          ok = mbar_wait_poll(bar_dfull(b), (gc / NB) & 1, p.status);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
          const uint32_t ta = tmem + static_cast<uint32_t>(b * p.tb + 32 * slice) +
                              (static_cast<uint32_t>(quad * 32) << 16);
          // the slice's columns, 16 at a time (the running sums hold 32 registers)
          uint32_t d[16];
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            if (half == 1 && ncol != 32) break;
            asm volatile(
                "tcgen05.ld.sync.aligned.32x32b.x16.b32"
                " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
                : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3]), "=r"(d[4]), "=r"(d[5]),
                  "=r"(d[6]), "=r"(d[7]), "=r"(d[8]), "=r"(d[9]), "=r"(d[10]), "=r"(d[11]),
                  "=r"(d[12]), "=r"(d[13]), "=r"(d[14]), "=r"(d[15])
                : "r"(ta + 16 * half));
            tmem_ld_wait();
            if (half == 1 || ncol != 32) {
              // the warp's columns of this buffer are in registers: the MMA may reuse it
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(bar_dfree(b));
            }
#pragma unroll
            for (int j = 0; j < 16; ++j)
              acc[16 * half + j] = __fmaf_rn(sc, __uint_as_float(d[j]), acc[16 * half + j]);
          }
        }
        if (!ok) break;
        // Y[m0 + 32 slice + j, n] for this lane's row: a warp writes 64 contiguous bytes per token
        if (n_ok) {
          const float bv = p.bias != nullptr ? __bfloat162float(p.bias[n]) : 0.0f;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int m = m0 + 32 * slice + j;
            if (j < ncol && m < p.M) p.Y[static_cast<size_t>(m) * p.N + n] = __float2bfloat16_rn(acc[j] + bv);
          }
        }
      }
    }
  }

  tc_fence_before();
  cta_sync_converged();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, static_cast<uint32_t>(NB * p.tb));
  }
}

}  // namespace svdq

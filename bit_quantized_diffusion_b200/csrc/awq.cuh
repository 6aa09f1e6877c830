// awq.cuh -- step a7: the AWQ W4A16 linear for small M (adaptive-norm modulation
// projections; Diffusers blog, "From SVDQuant to Nunchaku Lite": awq_w4a16 keeps
// 16-bit activations with 4-bit weights on these memory-bound layers).
//
//   Y[m,n] = sum_g s[n,g] * sum_{k in g} X[m,k] (q[n,k] - z[n,g]) + bias[n]
//          = sum_g s[n,g] * ( sum_{k in g} X[m,k] (128 + q[n,k]) - (128 + z[n,g]) xs[m,g] )
//
// with xs[m,g] = sum_{k in g} X[m,k]. The kernel is bound by streaming the
// 4-bit weights from HBM; its multiply-adds run on the warp-level tensor-core
// MMA (m16n8k16, bf16 in, f32 accumulate) with a 16-row weight block as the A
// operand and the (at most 8) tokens of a block as the N side: at M = 4 the
// 226 M multiply-adds would cost more on the CUDA cores than the 28 MB weight
// stream takes at full HBM speed.
//
// Weights arrive in "fragment order" (see svdq_pack): for a 16-row block and a
// 64-wide group each lane reads one 16-byte word holding exactly its A
// fragments for the group's four K=16 steps. A nibble pair OR-ed into the
// bf16 pattern 0x4300 is the exact bf16 pair (128 + q), so the dequantization
// is one mask per pair; the zero point enters once per group through xs.
//
// Each warp owns a contiguous run of groups of one 16-row block; its weights
// and (scale, zero) pairs are two contiguous byte ranges, fetched by bulk
// copies into shared memory so that every load of the CTA is in flight at once.
// X is staged in shared memory once per CTA, rows 16 bytes longer than K so the
// B-fragment reads of the 8 token rows fall in distinct banks.
#pragma once

#include "sm100.cuh"

namespace svdq {

constexpr int kAwqParts = 8;                 // warps sharing one 16-row block (K split)
constexpr int kAwqBlocksPerCta = 2;          // 16-row blocks per CTA
constexpr int kAwqWarps = kAwqParts * kAwqBlocksPerCta;
constexpr int kAwqThreads = 32 * kAwqWarps;  // 512
constexpr int kAwqBatch = 6;                 // groups per warp per bulk copy
constexpr int kAwqGroupBytes = 512 + 64;     // fragment words + (s, z) pairs of 16 rows
constexpr int kAwqMaxM = 64;

struct AwqParams {
  int M, N, K;
  const __nv_bfloat16* X;
  const uint4* qweight;   // fragment order
  const uint32_t* sz;     // (s, z) bf16 pairs
  const __nv_bfloat16* bias;
  __nv_bfloat16* Y;
  uint32_t* status;
};

// dynamic shared memory: weight staging per warp, X rows, per-group token sums, barriers
__host__ __device__ constexpr size_t awq_stage_bytes() {
  return static_cast<size_t>(kAwqWarps) * kAwqBatch * kAwqGroupBytes;
}
__host__ __device__ constexpr size_t awq_xrow_bytes(int K) { return static_cast<size_t>(K) * 2 + 16; }
__host__ __device__ constexpr size_t awq_smem_bytes(int M, int K) {
  return awq_stage_bytes() + static_cast<size_t>(M + 1) * awq_xrow_bytes(K) +
         static_cast<size_t>((M + 7) / 8) * 8 * (K / 64) * 4 + kAwqWarps * 8 + 128;
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32"
      " {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int kMB>  // number of 8-token blocks (1 or 2; the host splits larger M)
__global__ void __launch_bounds__(kAwqThreads, 2) awq_gemv_kernel(const AwqParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                             ~uintptr_t(127));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int blk = blockIdx.x * kAwqBlocksPerCta + warp / kAwqParts;  // 16-row block
  const int part = warp % kAwqParts;
  const int G = p.K / 64;
  const int g_begin = part * G / kAwqParts, g_end = (part + 1) * G / kAwqParts;
  const int nblocks = (p.N + 15) / 16;
  const int r0 = lane >> 2, c0 = 2 * (lane & 3);

  uint8_t* wbuf = smem + static_cast<size_t>(warp) * kAwqBatch * kAwqGroupBytes;
  const size_t xrow_bytes = awq_xrow_bytes(p.K);
  uint8_t* xsm = smem + awq_stage_bytes();  // [M + 1][K + 8] bf16, row M all zero
  float* xs = reinterpret_cast<float*>(xsm + static_cast<size_t>(p.M + 1) * xrow_bytes);  // [kMB*8][G]
  const uint32_t bar = smem_u32(xs + kMB * 8 * G) + warp * 8;

  if (lane == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  // stage X in shared memory, plus one zero row that padding tokens read
  for (int t = threadIdx.x; t < (p.M + 1) * (p.K / 8); t += kAwqThreads) {
    const int m = t / (p.K / 8), c = t % (p.K / 8);
    *reinterpret_cast<uint4*>(xsm + m * xrow_bytes + c * 16) =
        m < p.M ? __ldg(reinterpret_cast<const uint4*>(p.X + static_cast<size_t>(m) * p.K) + c)
                : make_uint4(0u, 0u, 0u, 0u);
  }
  __syncthreads();
  // per-group token sums xs[m][g] (rows >= M are zero)
  for (int t = threadIdx.x; t < kMB * 8 * G; t += kAwqThreads) {
    const int m = t / G, g = t % G;
    float sum = 0.0f;
    if (m < p.M) {
      const uint4* xp = reinterpret_cast<const uint4*>(xsm + m * xrow_bytes + g * 128);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint4 v = xp[j];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
          sum += __uint_as_float(w[e] << 16) + __uint_as_float(w[e] & 0xFFFF0000u);
      }
    }
    xs[t] = sum;
  }
  __syncthreads();

  float acc[kMB][4];
#pragma unroll
  for (int b = 0; b < kMB; ++b)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[b][j] = 0.0f;

  if (blk < nblocks) {
    // token rows this lane feeds as the B operand (rows >= M read the zero row)
    const uint32_t* xrow[kMB];
#pragma unroll
    for (int b = 0; b < kMB; ++b) {
      const int m = b * 8 + r0;
      xrow[b] = reinterpret_cast<const uint32_t*>(xsm + (m < p.M ? m : p.M) * xrow_bytes) + c0 / 2;
    }
    uint32_t phase = 0;
    for (int g0 = g_begin; g0 < g_end; g0 += kAwqBatch) {
      const int ng = min(kAwqBatch, g_end - g0);
      if (lane == 0) {
        // one bulk copy each for the run's fragment words and its (s, z) pairs
        mbar_arrive_expect_tx(bar, ng * kAwqGroupBytes);
        bulk_load(smem_u32(wbuf), p.qweight + (static_cast<size_t>(blk) * G + g0) * 32, ng * 512,
                  bar);
        bulk_load(smem_u32(wbuf) + kAwqBatch * 512, p.sz + (static_cast<size_t>(blk) * G + g0) * 16,
                  ng * 64, bar);
      }
      if (!mbar_wait(bar, phase, p.status)) break;
      phase ^= 1;
      const uint4* wq = reinterpret_cast<const uint4*>(wbuf) + lane;
      const uint32_t* szs = reinterpret_cast<const uint32_t*>(wbuf + kAwqBatch * 512) + r0;
#pragma unroll
      for (int j = 0; j < kAwqBatch; ++j) {
        if (j < ng) {
          const int g = g0 + j;
          const uint4 w = wq[j * 32];
          const uint32_t sz0 = szs[j * 16], sz8 = szs[j * 16 + 8];
          float part_acc[kMB][4];
#pragma unroll
          for (int b = 0; b < kMB; ++b)
#pragma unroll
            for (int e = 0; e < 4; ++e) part_acc[b][e] = 0.0f;
          const uint32_t words[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            uint32_t a[4];
#pragma unroll
            for (int pr = 0; pr < 4; ++pr)
              a[pr] = ((words[ks] >> (4 * pr)) & 0x000F000Fu) | 0x43004300u;  // bf16 (128 + q) pairs
            const int kw = (g * 64 + ks * 16) / 2;  // 32-bit word index of the fragment
#pragma unroll
            for (int b = 0; b < kMB; ++b) mma_bf16_16816(part_acc[b], a, xrow[b][kw], xrow[b][kw + 4]);
          }
          const float s0 = __uint_as_float(sz0 << 16), s8 = __uint_as_float(sz8 << 16);
          const float z0 = __uint_as_float(sz0 & 0xFFFF0000u) + 128.0f;
          const float z8 = __uint_as_float(sz8 & 0xFFFF0000u) + 128.0f;
#pragma unroll
          for (int b = 0; b < kMB; ++b) {
            const float xs0 = xs[(b * 8 + c0) * G + g], xs1 = xs[(b * 8 + c0 + 1) * G + g];
            acc[b][0] = fmaf(fmaf(-z0, xs0, part_acc[b][0]), s0, acc[b][0]);
            acc[b][1] = fmaf(fmaf(-z0, xs1, part_acc[b][1]), s0, acc[b][1]);
            acc[b][2] = fmaf(fmaf(-z8, xs0, part_acc[b][2]), s8, acc[b][2]);
            acc[b][3] = fmaf(fmaf(-z8, xs1, part_acc[b][3]), s8, acc[b][3]);
          }
        }
      }
      __syncwarp();  // every lane is done with the staging buffer before it is refilled
    }
  }
  // the first warp of each block adds the other K parts (in a fixed order) and
  // writes Y, one 8-token block at a time, through the (now idle) staging memory
  float* red = reinterpret_cast<float*>(smem);  // [kAwqWarps][32][4]
#pragma unroll
  for (int b = 0; b < kMB; ++b) {
    __syncthreads();
#pragma unroll
    for (int j = 0; j < 4; ++j) red[(warp * 32 + lane) * 4 + j] = acc[b][j];
    __syncthreads();
    if (part == 0 && blk < nblocks) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float v = red[(warp * 32 + lane) * 4 + j];
#pragma unroll
        for (int q = 1; q < kAwqParts; ++q) v += red[((warp + q) * 32 + lane) * 4 + j];
        const int n = blk * 16 + r0 + ((j & 2) ? 8 : 0);
        const int m = b * 8 + c0 + (j & 1);
        if (n < p.N && m < p.M) {
          const float bb = p.bias != nullptr ? __bfloat162float(p.bias[n]) : 0.0f;
          p.Y[static_cast<size_t>(m) * p.N + n] = __float2bfloat16_rn(v + bb);
        }
      }
    }
  }
}

}  // namespace svdq

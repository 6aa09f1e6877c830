// awq.cuh -- step a7: the AWQ W4A16 linear for small M (adaptive-norm modulation
// projections; Diffusers blog, "From SVDQuant to Nunchaku Lite": awq_w4a16 keeps
// 16-bit activations with 4-bit weights on these memory-bound layers).
//
//   Y[m,n] = sum_g s[n,g] * sum_{k in g} X[m,k] (q[n,k] - z[n,g]) + bias[n]
//
// The kernel is bound by streaming the 4-bit weights from HBM. Its
// multiply-adds run on the warp-level tensor-core MMA (m16n8k16, bf16 in, f32
// accumulate) with the weight tile as the 16-row A operand and the (at most 8)
// tokens as the N side: at M = 4, 226 M multiply-adds would otherwise cost more
// time on the CUDA cores than the 28 MB weight stream takes at full HBM speed.
//
// Weights arrive in "fragment order" (see svdq_pack): for a 16-row block and a
// 64-wide group each lane loads one 16-byte word that holds exactly its A
// fragments for the group's four K=16 steps. A nibble pair becomes a bf16 pair
// 128 + q by OR-ing it into the exponent pattern 0x4300, and subtracting the
// bf16 pair 128 + z gives q - z exactly. Each group's partial sums are scaled
// by s in float32 and added to the running float32 result.
#pragma once

#include "sm100.cuh"

namespace svdq {

constexpr int kAwqParts = 4;                 // warps sharing one 16-row block (K split)
constexpr int kAwqBlocksPerCta = 4;          // 16-row blocks per CTA
constexpr int kAwqThreads = 32 * kAwqParts * kAwqBlocksPerCta;  // 512
// groups whose weights are loaded before use (fewer when more tokens need registers)
__host__ __device__ constexpr int awq_batch(int mb) { return mb <= 2 ? 12 : (mb <= 4 ? 6 : 3); }
constexpr int kAwqMaxM = 64;

struct AwqParams {
  int M, N, K;
  const __nv_bfloat16* X;
  const uint4* qweight;   // fragment order
  const uint32_t* sz;     // (s, z) bf16 pairs
  const __nv_bfloat16* bias;
  __nv_bfloat16* Y;
};

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32"
      " {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int kMB>  // number of 8-token blocks (1..8)
__global__ void __launch_bounds__(kAwqThreads) awq_gemv_kernel(const AwqParams p) {
  __shared__ float red[kAwqThreads / 32][32][4];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int blk = blockIdx.x * kAwqBlocksPerCta + warp / kAwqParts;  // 16-row block
  const int part = warp % kAwqParts;
  const int G = p.K / 64;
  const int g_begin = part * G / kAwqParts, g_end = (part + 1) * G / kAwqParts;
  const int nblocks = (p.N + 15) / 16;
  const int r0 = lane >> 2, c0 = 2 * (lane & 3);

  float acc[kMB][4];
#pragma unroll
  for (int b = 0; b < kMB; ++b)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[b][j] = 0.0f;

  if (blk < nblocks) {
    const uint4* wq = p.qweight + static_cast<size_t>(blk) * G * 32 + lane;
    const uint32_t* szp = p.sz + static_cast<size_t>(blk) * G * 16;
    // token rows this lane feeds as the B operand (rows >= M read row 0, results dropped)
    const __nv_bfloat16* xrow[kMB];
#pragma unroll
    for (int b = 0; b < kMB; ++b) {
      const int m = b * 8 + r0;
      xrow[b] = p.X + static_cast<size_t>(m < p.M ? m : 0) * p.K + c0;
    }
    constexpr int kAwqBatch = awq_batch(kMB);
    for (int g0 = g_begin; g0 < g_end; g0 += kAwqBatch) {
      // issue every weight load of the batch first: the HBM latency is paid once
      uint4 w[kAwqBatch];
      uint32_t sz0[kAwqBatch], sz8[kAwqBatch];
#pragma unroll
      for (int j = 0; j < kAwqBatch; ++j) {
        if (g0 + j < g_end) {
          w[j] = __ldg(wq + static_cast<size_t>(g0 + j) * 32);
          sz0[j] = __ldg(szp + (g0 + j) * 16 + r0);
          sz8[j] = __ldg(szp + (g0 + j) * 16 + r0 + 8);
        }
      }
#pragma unroll
      for (int j = 0; j < kAwqBatch; ++j) {
        if (g0 + j >= g_end) break;
        const int g = g0 + j;
        // bf16 pairs (128 + z) for rows r0 and r0 + 8
        const float zf0 = __uint_as_float(sz0[j] & 0xFFFF0000u) + 128.0f;
        const float zf8 = __uint_as_float(sz8[j] & 0xFFFF0000u) + 128.0f;
        const __nv_bfloat162 zz0 = __floats2bfloat162_rn(zf0, zf0);
        const __nv_bfloat162 zz8 = __floats2bfloat162_rn(zf8, zf8);
        const float s0 = __uint_as_float(sz0[j] << 16), s8 = __uint_as_float(sz8[j] << 16);
        float part_acc[kMB][4];
#pragma unroll
        for (int b = 0; b < kMB; ++b)
#pragma unroll
          for (int e = 0; e < 4; ++e) part_acc[b][e] = 0.0f;
        const uint32_t words[4] = {w[j].x, w[j].y, w[j].z, w[j].w};
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          uint32_t a[4];
#pragma unroll
          for (int pr = 0; pr < 4; ++pr) {
            const uint32_t bits = ((words[ks] >> (4 * pr)) & 0x000F000Fu) | 0x43004300u;
            __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&bits);
            v = __hsub2(v, (pr & 1) ? zz8 : zz0);
            a[pr] = *reinterpret_cast<const uint32_t*>(&v);
          }
          const int k = g * 64 + ks * 16;
#pragma unroll
          for (int b = 0; b < kMB; ++b) {
            const uint32_t b0 = __ldg(reinterpret_cast<const uint32_t*>(xrow[b] + k));
            const uint32_t b1 = __ldg(reinterpret_cast<const uint32_t*>(xrow[b] + k + 8));
            mma_bf16_16816(part_acc[b], a, b0, b1);
          }
        }
#pragma unroll
        for (int b = 0; b < kMB; ++b) {
          acc[b][0] = fmaf(part_acc[b][0], s0, acc[b][0]);
          acc[b][1] = fmaf(part_acc[b][1], s0, acc[b][1]);
          acc[b][2] = fmaf(part_acc[b][2], s8, acc[b][2]);
          acc[b][3] = fmaf(part_acc[b][3], s8, acc[b][3]);
        }
      }
    }
  }
  // the first warp of each block adds the other K parts (in a fixed order) and
  // writes Y, one 8-token block at a time through shared memory
#pragma unroll
  for (int b = 0; b < kMB; ++b) {
    if (b > 0) __syncthreads();
#pragma unroll
    for (int j = 0; j < 4; ++j) red[warp][lane][j] = acc[b][j];
    __syncthreads();
    if (part == 0 && blk < nblocks) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float v = red[warp][lane][j];
#pragma unroll
        for (int q = 1; q < kAwqParts; ++q) v += red[warp + q][lane][j];
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

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
// Persistent: one CTA per SM owns a contiguous run of 16-row blocks and takes
// them BPR at a time ("rounds"; BPR = 1, 2, 4 or 8, chosen by the host so the
// sixteen consumer warps have work). Each block of a round gets 16 / BPR
// consumer warps. A ring stage holds one slice of K for all the round's blocks,
// 4 groups per warp, so every warp handles exactly four groups per stage (all
// loads first, then two MMA chains per group). A producer warp fills each stage
// with two tiled TMA copies (fragment-ordered weights and (s, z) pairs, as 3-D
// boxes over blocks x groups), starting at kernel entry, while the consumers stage X in
// shared memory in B-fragment order, summing each group's tokens (xs) on the way. Each warp
// keeps its block's partial sum in registers for the whole round; at the end of
// the round the block's first warp adds the block's partials in warp order and
// writes Y.
#pragma once

#include "sm100.cuh"

namespace svdq {

constexpr int kAwqConsumers = 16;                         // consumer warps
constexpr int kAwqThreads = 32 * (kAwqConsumers + 1);     // + the producer warp
constexpr int kAwqWarpGroups = 4;                         // groups per warp per ring stage
constexpr int kAwqGroupBytes = 512 + 64;                  // fragment words + (s, z) of 16 rows
constexpr int kAwqMaxStages = 4;
constexpr int kAwqMaxM = 64;

struct AwqParams {
  int M, N, K;
  int stages;             // ring depth (2..4)
  int bpr;                // blocks per round: 1, 2, 4 or 8
  const __nv_bfloat16* X;
  const uint4* qweight;   // fragment order
  const uint32_t* sz;     // (s, z) bf16 pairs
  const __nv_bfloat16* bias;
  __nv_bfloat16* Y;
  uint32_t* status;
};

// dynamic shared memory: ring, X rows, token sums, partial sums, barriers.
// A stage holds kAwqConsumers * kAwqWarpGroups groups (for any blocks per round).
__host__ __device__ constexpr size_t awq_stage_bytes() {
  return static_cast<size_t>(kAwqConsumers) * kAwqWarpGroups * kAwqGroupBytes;  // 27 KB
}
__host__ __device__ constexpr size_t awq_xrow_bytes(int K) { return static_cast<size_t>(K) * 2 + 16; }
// Row stride of the token sums xs (floats): the group count rounded up to
// 4 (mod 32), so the tokens 0, 2, 4, 6 a lane quad reads hit different banks.
__host__ __device__ constexpr int awq_xs_ld(int K) { return (K / 64 + 27) / 32 * 32 + 4; }
__host__ __device__ constexpr size_t awq_fixed_bytes(int M, int K, int kMB) {
  return static_cast<size_t>(M + 1) * awq_xrow_bytes(K) +               // X
         static_cast<size_t>(kMB) * 8 * awq_xs_ld(K) * 4 +               // xs
         static_cast<size_t>(kAwqConsumers) * 32 * 4 * kMB * 4 +        // partial sums
         8 * 2 * kAwqMaxStages + 128;                                   // barriers, alignment
}
__host__ __device__ constexpr size_t awq_smem_bytes(int M, int K, int kMB, int stages) {
  return static_cast<size_t>(stages) * awq_stage_bytes() + awq_fixed_bytes(M, K, kMB);
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32"
      " {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// The same with a zero accumulator: the first K step of a chain.
__device__ __forceinline__ void mma_bf16_16816_z(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                                 uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32"
      " {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%10, %10, %10, %10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.0f));
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ float ldsf(uint32_t addr) { return __uint_as_float(lds32(addr)); }
// The same with a compile-time byte offset folded into the instruction.
template <int kOff>
__device__ __forceinline__ uint4 lds128o(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4+%5];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr), "n"(kOff));
  return v;
}
template <int kOff>
__device__ __forceinline__ uint32_t lds32o(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1+%2];" : "=r"(v) : "r"(addr), "n"(kOff));
  return v;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// One fragment word (nibble s = bits 4s..4s+3) -> the four bf16 pairs
// (128 + q[s], 128 + q[s + 4]), s = 0..3: even nibbles are gathered into the
// bytes of `ev`, odd ones into `od`, and each pair is two byte selects next to
// the exponent byte 0x43.
__device__ __forceinline__ void awq_dequant_word(uint32_t w, uint32_t (&a)[4]) {
  const uint32_t ev = w & 0x0F0F0F0Fu;
  const uint32_t od = (w >> 4) & 0x0F0F0F0Fu;
  const uint32_t e43 = 0x43434343u;
  a[0] = prmt(ev, e43, 0x4240u);  // nibbles 0, 4
  a[1] = prmt(od, e43, 0x4240u);  // nibbles 1, 5
  a[2] = prmt(ev, e43, 0x4341u);  // nibbles 2, 6
  a[3] = prmt(od, e43, 0x4341u);  // nibbles 3, 7
}

// kN consecutive 64-wide groups of one warp: all shared-memory loads first,
// then the groups' MMA chains (two per group: K steps 0, 1 and 2, 3)
// interleaved, then the per-group scale and zero point.
//   wp   this lane's first fragment word          (+512 per group)
//   szp  (s, z) of row r0 of the first group        (+64 per group, row r0 + 8 at +32)
//   xa   this lane's X fragment runs, xo the first group's offset in them (+128 per group)
//   xsp  xs[c0][first group]                        (+4 per group, token c0 + 1 at +4 xs_ld)
template <int kMB, int kN>  // kN <= 4
__device__ __forceinline__ void awq_groups(uint32_t wp, uint32_t szp, const uint32_t (&xa)[kMB],
                                           uint32_t xo, uint32_t xsp, int xs_ld, float (&acc)[kMB][4]) {
  uint4 w[kN], xl[kN][kMB][2];
  uint32_t sz0[kN], sz8[kN];
  float xs0[kN][kMB], xs1[kN][kMB];
  uint32_t xb[kMB], xs0a[kMB], xs1a[kMB];
#pragma unroll
  for (int mb = 0; mb < kMB; ++mb) {
    xb[mb] = xa[mb] + xo;
    xs0a[mb] = xsp + mb * 8 * xs_ld * 4;
    xs1a[mb] = xs0a[mb] + xs_ld * 4;
  }
#pragma unroll
  for (int u = 0; u < kN; ++u) {
    // u is a compile-time constant here: every offset below is an immediate
    switch (u) {
#define SVDQ_AWQ_LOADS(U)                                                        \
  case U:                                                                        \
    w[U] = lds128o<(U) * 512>(wp);                                               \
    sz0[U] = lds32o<(U) * 64>(szp);                                              \
    sz8[U] = lds32o<(U) * 64 + 32>(szp);                                         \
    for (int mb = 0; mb < kMB; ++mb) {                                           \
      xl[U][mb][0] = lds128o<(U) * 128>(xb[mb]);                                 \
      xl[U][mb][1] = lds128o<(U) * 128 + 16>(xb[mb]);                            \
      xs0[U][mb] = __uint_as_float(lds32o<(U) * 4>(xs0a[mb]));                   \
      xs1[U][mb] = __uint_as_float(lds32o<(U) * 4>(xs1a[mb]));                   \
    }                                                                            \
    break;
      SVDQ_AWQ_LOADS(0)
      SVDQ_AWQ_LOADS(1)
      SVDQ_AWQ_LOADS(2)
      SVDQ_AWQ_LOADS(3)
#undef SVDQ_AWQ_LOADS
    }
  }
  float pc[kN][2][kMB][4];
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
    for (int u = 0; u < kN; ++u) {
      const uint32_t word = ks == 0 ? w[u].x : ks == 1 ? w[u].y : ks == 2 ? w[u].z : w[u].w;
      uint32_t a[4];
      awq_dequant_word(word, a);  // bf16 (128 + q) pairs
#pragma unroll
      for (int mb = 0; mb < kMB; ++mb) {
        const uint4& x = xl[u][mb][ks >> 1];
        if (ks < 2)
          mma_bf16_16816_z(pc[u][ks & 1][mb], a, (ks & 1) ? x.z : x.x, (ks & 1) ? x.w : x.y);
        else
          mma_bf16_16816(pc[u][ks & 1][mb], a, (ks & 1) ? x.z : x.x, (ks & 1) ? x.w : x.y);
      }
    }
  }
#pragma unroll
  for (int u = 0; u < kN; ++u) {
    const float s0 = __uint_as_float(sz0[u] << 16), s8 = __uint_as_float(sz8[u] << 16);
    const float z0 = __uint_as_float(sz0[u] & 0xFFFF0000u) + 128.0f;
    const float z8 = __uint_as_float(sz8[u] & 0xFFFF0000u) + 128.0f;
#pragma unroll
    for (int mb = 0; mb < kMB; ++mb) {
      acc[mb][0] = fmaf(fmaf(-z0, xs0[u][mb], pc[u][0][mb][0] + pc[u][1][mb][0]), s0, acc[mb][0]);
      acc[mb][1] = fmaf(fmaf(-z0, xs1[u][mb], pc[u][0][mb][1] + pc[u][1][mb][1]), s0, acc[mb][1]);
      acc[mb][2] = fmaf(fmaf(-z8, xs0[u][mb], pc[u][0][mb][2] + pc[u][1][mb][2]), s8, acc[mb][2]);
      acc[mb][3] = fmaf(fmaf(-z8, xs1[u][mb], pc[u][0][mb][3] + pc[u][1][mb][3]), s8, acc[mb][3]);
    }
  }
}

// tm_q: qweight as [N/16 blocks][K/64 groups][64 x 8 bytes]; tm_sz: (s, z) pairs as
// [N/16][K/64][8 x 8 bytes]: one box {64 or 8, GSK, BPR} is one stage's slice of
// the round's blocks (rows past N and groups past K arrive as zeros).
template <int kMB>  // number of 8-token blocks (1 or 2; the host splits larger M)
__global__ void __launch_bounds__(kAwqThreads, 1)
    awq_gemv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_sz,
                    const AwqParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                             ~uintptr_t(127));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int G = p.K / 64;
  const int BPR = p.bpr;                               // blocks per round
  const int WPB = kAwqConsumers / BPR;                 // warps per block
  const int GSK = kAwqWarpGroups * WPB;                // groups per block per stage
  const int nst = (G + GSK - 1) / GSK;                 // ring stages per round
  const int NS = p.stages;
  const size_t SB = awq_stage_bytes();
  const uint32_t sz_off = static_cast<uint32_t>(BPR) * GSK * 512;  // (s, z) part of a stage
  const int nblocks = (p.N + 15) / 16;
  const int b_begin = static_cast<int>(static_cast<long long>(blockIdx.x) * nblocks / gridDim.x);
  const int b_end = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * nblocks / gridDim.x);
  const int nrounds = (b_end - b_begin + BPR - 1) / BPR;
  const int r0 = lane >> 2, c0 = 2 * (lane & 3);

  uint8_t* ring = smem;
  const size_t xrow_bytes = awq_xrow_bytes(p.K);
  uint8_t* xsm = ring + NS * SB;  // [M + 1][K + 8] bf16, row M all zero
  float* xs = reinterpret_cast<float*>(xsm + static_cast<size_t>(p.M + 1) * xrow_bytes);  // [kMB*8][xs_ld]
  const int xs_ld = awq_xs_ld(p.K);
  float* red = xs + kMB * 8 * xs_ld;                 // [consumers][32][4 kMB]
  const uint32_t bars = (smem_u32(red + kAwqConsumers * 32 * 4 * kMB) + 7) & ~7u;
  auto full = [&](int s) { return bars + 8 * s; };
  auto empty = [&](int s) { return bars + 8 * (kAwqMaxStages + s); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), kAwqConsumers);
    }
    fence_barrier_init();
  }
  cta_sync_converged();
  grid_dep_launch();

  if (warp == kAwqConsumers) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      grid_dep_wait();
      int it = 0;
      bool ok = true;
      for (int rr = 0; rr < nrounds && ok; ++rr) {
        const int bb = b_begin + rr * BPR;
        for (int t = 0; t < nst && ok; ++t, ++it) {
          const int s = it % NS;
          // the producer is not on the critical path: it waits suspended
          ok = mbar_wait(empty(s), ((it / NS) & 1) ^ 1, p.status, kWaitLimitNs, 2000u);
          if (!ok) break;
          const uint32_t dst = smem_u32(ring + s * SB);
          // two tiled copies fill the stage; their boxes count in full
          mbar_arrive_expect_tx(full(s), BPR * GSK * kAwqGroupBytes);
          tma_load_3d(dst, &tm_q, full(s), 0, t * GSK, bb);
          tma_load_3d(dst + sz_off, &tm_sz, full(s), 0, t * GSK, bb);
        }
      }
    }
    return;  // the consumers synchronise among themselves from here on
  }

  // -------------------------------------------------------------- consumers
  constexpr int kCT = kAwqConsumers * 32;
  grid_dep_wait();  // X and Y may be the previous grid's
  // X in shared memory, plus one zero row that padding tokens read. Source
  // 16-byte unit c of a row holds words 4h..4h+3 (h = c % 2) of K step
  // ks = (c / 2) % 4 of group c / 8; word 4h + t goes to lane quad t's run.
  // Thread tid owns unit columns c = tid, tid + 512, ... (every thread takes
  // every pass, so the shuffles below see full warps); its rows' loads are
  // issued four at a time before their stores, so their latencies overlap.
  // The eight units of a group sit in eight consecutive lanes: their sums,
  // combined by a fixed xor tree, give the token sums xs[m][g].
  const int U = p.K / 8;  // 16-byte units per row (a multiple of 8)
  for (int c0 = 0; c0 < U; c0 += kCT) {
    const int c = c0 + threadIdx.x;
    const bool has = c < U;
    const int ks = (c >> 1) & 3, h = c & 1;
    const uint4* src = reinterpret_cast<const uint4*>(p.X) + c;
    uint8_t* dst = xsm + (c >> 3) * 128;
    for (int m0 = 0; m0 <= p.M; m0 += 4) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        v[u] = has && m0 + u < p.M ? __ldg(src + static_cast<size_t>(m0 + u) * U) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int m = m0 + u;
        if (m > p.M) break;
        if (has) {
          uint32_t* grp = reinterpret_cast<uint32_t*>(dst + m * xrow_bytes);
          grp[0 * 8 + ks * 2 + h] = v[u].x;
          grp[1 * 8 + ks * 2 + h] = v[u].y;
          grp[2 * 8 + ks * 2 + h] = v[u].z;
          grp[3 * 8 + ks * 2 + h] = v[u].w;
        }
        if (m < p.M) {
          const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
          float e[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) e[j] = __uint_as_float(w[j] << 16) + __uint_as_float(w[j] & 0xFFFF0000u);
          float sum = (e[0] + e[1]) + (e[2] + e[3]);
          sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 1);
          sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 2);
          sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 4);
          if (has && (c & 7) == 0) xs[m * xs_ld + (c >> 3)] = sum;
        }
      }
    }
  }
  // token rows M .. 8 kMB - 1 are padding: their sums are zero
  for (int i = threadIdx.x; i < (kMB * 8 - p.M) * G; i += kCT) {
    const int m = p.M + i / G, g = i - (i / G) * G;
    xs[m * xs_ld + g] = 0.0f;
  }
  __syncwarp();
  asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory");

  // this lane's B-fragment runs: token rows r0 (+ 8 mb), lane quad t = lane % 4
  // (rows >= M read the zero row)
  uint32_t xa[kMB];
#pragma unroll
  for (int mb = 0; mb < kMB; ++mb) {
    const int m = mb * 8 + r0;
    xa[mb] = smem_u32(xsm) + (m < p.M ? m : p.M) * static_cast<uint32_t>(xrow_bytes) + (lane & 3) * 32;
  }
  const uint32_t xs_a = smem_u32(xs) + c0 * xs_ld * 4;  // xs[c0][0]
  const int jslot = warp / WPB, part = warp % WPB;  // this warp's block slot and K share
  bool ok = true;
  int s = 0;          // ring slot
  uint32_t ph = 0;    // its phase parity
  for (int rr = 0; rr < nrounds; ++rr) {
    const int b = b_begin + rr * BPR + jslot;
    const bool active = b < b_end;
    float acc[kMB][4];
#pragma unroll
    for (int mb = 0; mb < kMB; ++mb)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[mb][j] = 0.0f;
    for (int t = 0; t < nst; ++t) {
      if (ok) ok = mbar_wait_poll(full(s), ph, p.status);
      const int g0 = t * GSK, n = min(GSK, G - g0);
      // a full stage gives every warp kAwqWarpGroups groups; only a last, partial
      // stage needs the general split
      const int lo = n == GSK ? part * kAwqWarpGroups : part * n / WPB;
      const int hi = n == GSK ? lo + kAwqWarpGroups : (part + 1) * n / WPB;
      const uint32_t st = smem_u32(ring + s * SB);
      const uint32_t wp = st + jslot * GSK * 512 + lo * 512 + lane * 16;     // fragment word
      const uint32_t szp = st + sz_off + jslot * GSK * 64 + lo * 64 + r0 * 4;  // (s, z) of row r0
      const uint32_t xo = (g0 + lo) * 128;                                    // X run offset
      const uint32_t xsp = xs_a + (g0 + lo) * 4;                              // xs[c0][g]
      if (ok && active) {
        if (hi - lo == kAwqWarpGroups) {
          awq_groups<kMB, kAwqWarpGroups>(wp, szp, xa, xo, xsp, xs_ld, acc);
        } else {
          for (int j = 0; j < hi - lo; ++j)
            awq_groups<kMB, 1>(wp + j * 512, szp + j * 64, xa, xo + j * 128, xsp + j * 4, xs_ld, acc);
        }
      }
      __syncwarp();  // every lane is done with the stage before it is released
      if (lane == 0) mbar_arrive(empty(s));
      if (++s == NS) {
        s = 0;
        ph ^= 1u;
      }
    }
    // the block's partial sums (one per K share), added in share order by share 0
#pragma unroll
    for (int mb = 0; mb < kMB; ++mb)
      *reinterpret_cast<float4*>(red + ((warp * 32 + lane) * kMB + mb) * 4) =
          make_float4(acc[mb][0], acc[mb][1], acc[mb][2], acc[mb][3]);
    __syncwarp();
    asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory");
    if (part == 0 && active && ok) {
#pragma unroll
      for (int mb = 0; mb < kMB; ++mb) {
        float4 v = *reinterpret_cast<const float4*>(red + ((warp * 32 + lane) * kMB + mb) * 4);
        for (int q = 1; q < WPB; ++q) {
          const float4 u =
              *reinterpret_cast<const float4*>(red + (((warp + q) * 32 + lane) * kMB + mb) * 4);
          v.x += u.x;
          v.y += u.y;
          v.z += u.z;
          v.w += u.w;
        }
        const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int n = b * 16 + r0 + ((j & 2) ? 8 : 0);
          const int m = mb * 8 + c0 + (j & 1);
          if (n < p.N && m < p.M) {
            const float bb = p.bias != nullptr ? __bfloat162float(p.bias[n]) : 0.0f;
            p.Y[static_cast<size_t>(m) * p.N + n] = __float2bfloat16_rn(vv[j] + bb);
          }
        }
      }
    }
    __syncwarp();
    asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory");  // red is free for the next round
  }
}

}  // namespace svdq

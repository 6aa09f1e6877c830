// quantize_act.cuh -- steps a1..a4 of the SVDQuant layer in one pass over X:
// smoothing, group scale, 4-bit quantization + packing, and the rank-r
// down-projection on the tensor cores (Nunchaku README, "Engine design" (b):
// the down projection and the quantizer share their input).
//
// The down-projection reads the raw bf16 X tile that TMA brought in for the
// quantizer: x_hat L1 = X (diag(smooth_inv) L1), and the smoothed factor
// L1s = diag(smooth_inv) L1 comes pre-split into two bf16 planes (hi + lo, see
// svdq_pack_lowrank), so two kind::f16 MMAs per K step give the product to
// about 2^-17 relative, accumulated in float32 in tensor memory. The quantizer
// threads therefore only read X and write codes and scales.
//
// One CTA per SM (a kernel that allocates tensor memory runs one CTA per SM)
// owns 128 rows and a contiguous range of 64-column chunks of X: the grid
// splits K into S = svdq_xl1_splits(M, K, r) ranges so that the row blocks times
// S fill the SMs. Each split writes its own partial down-projection (split 0
// into xl1, the others into working space), so no CTA waits for another; a
// small kernel then adds the S partials in split order into xl1.
//
// A ring stage holds two 64-column sub-chunks (when shared memory allows; one
// for large r). Warp roles (18 warps):
//   warp 0      TMA producer: per sub-chunk the X tile [128 x 64] bf16 (128-byte
//               swizzle), the L1s hi and lo tiles [r x 64] bf16, 64 smooth_inv
//   warp 1      tensor-memory owner and MMA issuer (one thread)
//   warps 2..17 quantizers; quantizer w takes sub-chunk w / 8 of a stage, rows
//               16 (w % 8) .. + 15; lane l handles row 16 (w % 8) + l % 16 and
//               columns 32 (l / 16) .. + 31 of the sub-chunk: two NVFP4 groups, or
//               half an INT4 group (the other half is lane l ^ 16); the float32
//               arithmetic runs on paired (float2) instructions
#pragma once

#include "sm100.cuh"

namespace svdq {

constexpr int kQaWarps = 18;
constexpr int kQaThreads = kQaWarps * 32;
constexpr int kQaQuantWarps = 16;
constexpr int kQaChunk = 64;                        // columns per sub-chunk
constexpr int kQaXStageBytes = 128 * kQaChunk * 2;  // 16 KB
constexpr int kQaSmoothBytes = kQaChunk * 4;        // 256 B
constexpr int kQaSmTarget = 148;                    // B200 SMs: the K split fills them

// Number of K splits (partial down-projections) for an M x K activation: the
// largest power of two <= 8 that keeps (row blocks x splits) within the SMs.
__host__ __device__ inline int qa_splits(int M, int K) {
  const int row_blocks = (M + 127) / 128;
  const int kc_total = K / kQaChunk;
  int s = 1;
  while (s * 2 <= 8 && s * 2 <= kc_total && row_blocks * s * 2 <= kQaSmTarget) s *= 2;
  return s;
}

struct QuantActParams {
  int M, K, r;
  int ksplit;      // K ranges (grid.x); split ks writes xl1[ks]
  int stages;      // ring depth
  int spc;         // sub-chunks per stage (1 or 2)
  int m_pad;       // M rounded up to 128
  const float* smooth_inv;
  const float* tensor_scale;  // NVFP4 two-level: [s_t, RN32(1 / s_t)] on the device, or null
  uint8_t* codes;
  uint8_t* scales;
  float* xl1;      // split 0 (and, after the reduction, the sum): [M][r]
  float* xl1_rest; // splits 1 .. ksplit - 1: [ksplit - 1][M][r]
  uint32_t* status;
};

struct QaSmem {
  // byte offsets from the 1024-aligned dynamic shared memory base
  uint32_t ring, sub_bytes, stage_bytes, l1_off, sm_off, table, bars, tmem_slot;
};

__host__ __device__ inline QaSmem qa_smem_layout(int r, int stages, int spc) {
  QaSmem s;
  s.ring = 0;
  s.l1_off = kQaXStageBytes;                       // hi plane, then lo plane
  s.sm_off = kQaXStageBytes + 2 * r * 128;         // smooth_inv chunk
  s.sub_bytes = (s.sm_off + kQaSmoothBytes + 1023) / 1024 * 1024;
  s.stage_bytes = spc * s.sub_bytes;
  s.table = s.ring + stages * s.stage_bytes;       // E4M3 (value, reciprocal) x 128
  s.bars = s.table + 128 * 8;
  s.tmem_slot = s.bars + 8 * (2 * stages + 1);
  return s;
}

__host__ inline size_t qa_smem_bytes(int r, int stages, int spc) {
  QaSmem s = qa_smem_layout(r, stages, spc);
  return s.tmem_slot + 16 + 1024;  // + alignment slack
}

// RN32(a / b) for a >= 0 and the constant divisors b = 6 (NVFP4) and 7 (INT4):
// one multiply by c = RN32(1 / b), the exact remainder a - q0 b in one FMA, and
// one correction q0 + rem c rounded once (Markstein's correction step for a
// division by a known divisor). For these two divisors this equals the IEEE
// quotient for every float32 a whose quotient is normal (checked exhaustively
// binade by binade on the CPU); where the quotient underflows, both are far
// below the smallest E4M3 / FP16 scale and give scale code 0.
template <int kB>
__device__ __forceinline__ float div_by_const_rn(float a) {
  static_assert(kB == 6 || kB == 7, "verified divisors only");
  const float c = __uint_as_float(kB == 6 ? 0x3e2aaaabu : 0x3e124925u);  // RN32(1 / b)
  const float q0 = __fmul_rn(a, c);
  const float rem = __fmaf_rn(-q0, static_cast<float>(kB), a);
  return __fmaf_rn(rem, c, q0);
}

// max(a, b, c) of three float32 values in one instruction
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Largest magnitude of 8 float pairs, as a tree of three-input maxima.
__device__ __forceinline__ float absmax16(const float2* v) {
  const float a = max3f(fabsf(v[0].x), fabsf(v[0].y), fabsf(v[1].x));
  const float b = max3f(fabsf(v[1].y), fabsf(v[2].x), fabsf(v[2].y));
  const float c = max3f(fabsf(v[3].x), fabsf(v[3].y), fabsf(v[4].x));
  const float d = max3f(fabsf(v[4].y), fabsf(v[5].x), fabsf(v[5].y));
  const float e = max3f(fabsf(v[6].x), fabsf(v[6].y), fabsf(v[7].x));
  return fmaxf(max3f(a, b, c), max3f(d, e, fabsf(v[7].y)));
}

template <int kFmt>  // 0: NVFP4 (E2M1, UE4M3 per 16), 1: INT4 (FP16 per 64)
__global__ void __launch_bounds__(kQaThreads, 1)
    quantize_act_kernel(const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_l1, const QuantActParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const QaSmem L = qa_smem_layout(p.r, p.stages, p.spc);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int NS = p.stages;
  const int r = p.r;
  const bool smoothing = p.smooth_inv != nullptr;

  const int ks = blockIdx.x;
  const int rb = blockIdx.y;
  const int kc_total = p.K / kQaChunk;
  const int kc0 = ks * kc_total / p.ksplit;
  const int kc1 = (ks + 1) * kc_total / p.ksplit;
  const int nchunks = kc1 - kc0;
  const int nstage = (nchunks + p.spc - 1) / p.spc;  // ring uses of this CTA

  auto bar_full = [&](int s) { return sbase + L.bars + 8 * s; };
  auto bar_empty = [&](int s) { return sbase + L.bars + 8 * (NS + s); };
  const uint32_t bar_acc = sbase + L.bars + 8 * (2 * NS);
  auto x_stage = [&](int s) { return sbase + L.ring + s * L.stage_bytes; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.tmem_slot);
  const uint32_t tmem_cols = r <= 32 ? 32 : (r <= 64 ? 64 : (r <= 128 ? 128 : 256));
  float2* table = reinterpret_cast<float2*>(smem + L.table);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar_full(s), 1);
      // the quantizer warps finish reading X, and the MMAs finish reading X and L1s
      mbar_init(bar_empty(s), kQaQuantWarps + (r > 0 ? 1 : 0));
    }
    mbar_init(bar_acc, 1);
    fence_barrier_init();
    prefetch_tmap(&tm_x);
    if (r > 0) prefetch_tmap(&tm_l1);
  }
  if (kFmt == 0 && threadIdx.x >= 64 && threadIdx.x < 64 + 128) {
    // every E4M3 scale code: its value and correctly rounded float32 reciprocal
    const uint32_t c = threadIdx.x - 64;
    const float v = c < 0x7F ? e4m3_value(c) : 0.0f;
    table[c] = make_float2(v, v != 0.0f ? __frcp_rn(v) : 0.0f);
  }
  if (warp == 1 && r > 0) {
    tmem_alloc(smem_u32(tmem_slot), tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  cta_sync_converged();
  grid_dep_wait();  // the prologue above touches no global memory the previous grid may write
  grid_dep_launch();
  tc_fence_after();
  const uint32_t tmem_base = r > 0 ? *tmem_slot : 0;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (elect_one()) {
      const uint32_t sub_tx = kQaXStageBytes + 2 * r * 128 + (smoothing ? kQaSmoothBytes : 0);
      for (int i = 0; i < nstage; ++i) {
        const int s = i % NS;
        if (!mbar_wait(bar_empty(s), ((i / NS) & 1) ^ 1, p.status)) break;
        const int nsub = min(p.spc, nchunks - i * p.spc);
        mbar_arrive_expect_tx(bar_full(s), nsub * sub_tx);
        for (int u = 0; u < nsub; ++u) {
          const int kc = kc0 + i * p.spc + u;
          const uint32_t base = x_stage(s) + u * L.sub_bytes;
          tma_load_2d(base, &tm_x, bar_full(s), kc * kQaChunk, rb * 128);
          if (r > 0) {
            tma_load_2d(base + L.l1_off, &tm_l1, bar_full(s), kc * kQaChunk, 0);
            tma_load_2d(base + L.l1_off + r * 128, &tm_l1, bar_full(s), kc * kQaChunk, r);
          }
          if (smoothing)
            bulk_load(base + L.sm_off, p.smooth_inv + kc * kQaChunk, kQaSmoothBytes, bar_full(s));
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (r > 0 && elect_one()) {
      const uint32_t idesc = idesc_bf16_f32(128, r, false, false);
      for (int i = 0; i < nstage; ++i) {
        const int s = i % NS;
        if (!mbar_wait(bar_full(s), (i / NS) & 1, p.status)) break;
        tc_fence_after();
        const int nsub = min(p.spc, nchunks - i * p.spc);
        for (int u = 0; u < nsub; ++u) {
          const uint32_t base = x_stage(s) + u * L.sub_bytes;
#pragma unroll
          for (int kk = 0; kk < kQaChunk / 16; ++kk) {
            // A: the X tile, 128 rows x 128 B, 128-byte swizzle; 16 K = 32 B
            const uint64_t ad = smem_desc(base + kk * 32, 16, 1024, kSwizzle128B);
            // B: L1s hi / lo planes, r rows x 128 B each, 128-byte swizzle
            const uint64_t bh = smem_desc(base + L.l1_off + kk * 32, 16, 1024, kSwizzle128B);
            const uint64_t bl = smem_desc(base + L.l1_off + r * 128 + kk * 32, 16, 1024, kSwizzle128B);
            mma_f16(tmem_base, ad, bh, idesc, (i > 0 || u > 0 || kk > 0) ? 1u : 0u);
            mma_f16(tmem_base, ad, bl, idesc, 1u);
          }
        }
        tc_commit(bar_empty(s));
      }
      tc_commit(bar_acc);
    }
  } else {
    // ---------------------------------------------------------------- quantizers
    const int qw = warp - 2;
    const int sub = p.spc == 2 ? qw >> 3 : 0;     // which sub-chunk of a stage
    const bool active = p.spc == 2 || qw < 8;    // one sub-chunk per stage: warps 0..7 quantize
    const int row = (qw & 7) * 16 + (lane & 15);
    const int half = lane >> 4;  // which 32 columns of the sub-chunk
    const int m = rb * 128 + row;
    const bool row_ok = m < p.M;
    uint8_t* const code_row = p.codes + static_cast<size_t>(m) * (p.K / 2) + half * 16;
    const uint32_t table_u32 = sbase + L.table;
    // two-level NVFP4: the smoothed values are quantized as x_hat * RN32(1 / s_t)
    const bool two_level = kFmt == 0 && p.tensor_scale != nullptr;
    const float t_inv = two_level ? p.tensor_scale[1] : 1.0f;
    bool ok = true;
    int s = 0;        // ring slot of stage i
    uint32_t ph = 0;  // its phase parity
    for (int i = 0; i < nstage; ++i) {
      const int slot = s;
      ok = mbar_wait(bar_full(slot), ph, p.status);
      if (!ok) break;
      if (++s == NS) {
        s = 0;
        ph ^= 1u;
      }
      const int kc = kc0 + i * p.spc + sub;
      if (!active || kc >= kc1) {
        // nothing of this stage for this warp
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_empty(slot));
        continue;
      }
      const uint32_t sub_base = x_stage(slot) + sub * L.sub_bytes;
      // -- 32 bf16 of this row from the 128B-swizzled X tile, as 16 float pairs
      float2 xv[16];
      {
        const uint32_t rowbase = sub_base + row * 128;
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const int c = 4 * half + h;
          const uint4 v = lds_u4(rowbase + ((c ^ (row & 7)) << 4));
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int j = 0; j < 4; ++j)
            xv[4 * h + j] = make_float2(__uint_as_float(w[j] << 16), __uint_as_float(w[j] & 0xFFFF0000u));
        }
      }
      // -- a1: smoothing, one float32 multiply per element
      if (smoothing) {
        const uint32_t sp = sub_base + L.sm_off + 128 * half;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 sv = lds_f4(sp + 16 * j);
          xv[2 * j] = __fmul2_rn(xv[2 * j], make_float2(sv.x, sv.y));
          xv[2 * j + 1] = __fmul2_rn(xv[2 * j + 1], make_float2(sv.z, sv.w));
        }
      }
      // this warp no longer reads the stage's shared memory
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_empty(slot));
      if (two_level) {
        const float2 t2 = make_float2(t_inv, t_inv);
#pragma unroll
        for (int j = 0; j < 16; ++j) xv[j] = __fmul2_rn(xv[j], t2);
      }
      // -- a2 + a3: group scale and codes
      uint32_t code[4];
      if (kFmt == 0) {
        uint32_t sc[2];
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          const float amax = absmax16(xv + 8 * g);
          sc[g] = e4m3_code(div_by_const_rn<6>(amax));
          const float2 vr = lds_f2(table_u32 + 8 * sc[g]);  // (decoded scale, its reciprocal)
          const float2 rcp2 = make_float2(vr.y, vr.y);
          float2 y0[4], y1[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            y0[j] = __fmul2_rn(xv[8 * g + j], rcp2);
            y1[j] = __fmul2_rn(xv[8 * g + 4 + j], rcp2);
          }
          const bool live = vr.x != 0.0f;  // a zero scale stores zero codes
          code[2 * g] = live ? e2m1x8(y0) : 0u;
          code[2 * g + 1] = live ? e2m1x8(y1) : 0u;
        }
        // the row's four scale bytes: groups 2 half, 2 half + 1 here, the others in lane ^ 16
        const uint32_t mine = sc[0] | (sc[1] << 8);
        const uint32_t other = __shfl_xor_sync(0xffffffffu, mine, 16);
        if (half == 0) {
          const uint32_t word = mine | (other << 16);
          const size_t atom = static_cast<size_t>(rb) * kc_total + kc;
          *reinterpret_cast<uint32_t*>(p.scales + atom * 512 + (row & 31) * 16 + (row >> 5) * 4) = word;
        }
      } else {
        float amax = fmaxf(absmax16(xv), absmax16(xv + 8));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 16));
        const __half hs = __float2half_rn(div_by_const_rn<7>(amax));
        const float sval = __half2float(hs);
#pragma unroll
        for (int w = 0; w < 4; ++w) code[w] = 0u;
        if (sval != 0.0f) {
          const float rcp = __frcp_rn(sval);
          const float2 rcp2 = make_float2(rcp, rcp);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float2 q = __fmul2_rn(xv[j], rcp2);
            const float qq[2] = {q.x, q.y};
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              int v = __float2int_rn(qq[e]);
              v = max(-7, min(7, v));
              const uint32_t nib = static_cast<uint32_t>(v) & 15u;  // two's complement nibble
              code[j >> 2] |= nib << (4 * (2 * (j & 3) + e));
            }
          }
        }
        if (half == 0)
          reinterpret_cast<__half*>(p.scales)[static_cast<size_t>(kc) * p.m_pad + rb * 128 + row] = hs;
      }
      if (row_ok)
        *reinterpret_cast<uint4*>(code_row + kc * 32) = make_uint4(code[0], code[1], code[2], code[3]);
    }
    // ------------------------------------------------------------ xl1 epilogue
    // this split's partial down-projection of the CTA's 128 rows
    if (r > 0 && ok && mbar_wait(bar_acc, 0, p.status)) {
      tc_fence_after();
      const int quad = warp & 3;         // tensor-memory lanes this warp may read
      const int part = (warp - 2) >> 2;  // which quarter of the r columns
      const int trow = quad * 32 + lane;
      const int ncol = r / 4, c_begin = part * ncol;
      const int tm = rb * 128 + trow;
      float* dst = (ks == 0 ? p.xl1 : p.xl1_rest + static_cast<size_t>(ks - 1) * p.M * r) +
                   static_cast<size_t>(tm) * r;
      for (int c = c_begin; c < c_begin + ncol; c += 4) {
        uint32_t v[4];
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
                     : "r"(tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + c));
        tmem_ld_wait();
        if (tm < p.M)
          *reinterpret_cast<float4*>(dst + c) =
              make_float4(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]),
                          __uint_as_float(v[3]));
      }
    }
  }

  tc_fence_before();
  cta_sync_converged();
  if (warp == 1 && r > 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

// The K splits' partial down-projections, added in split order into split 0:
// xl1 = ((xl1 + rest[0]) + ...) + rest[S-2]; n4 float4 per split.
__global__ void xl1_reduce_kernel(float4* xl1, const float4* rest, int splits, size_t n4) {
  grid_dep_wait();
  grid_dep_launch();
  for (size_t t = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; t < n4;
       t += static_cast<size_t>(gridDim.x) * blockDim.x) {
    float4 v = xl1[t];
    for (int sp = 1; sp < splits; ++sp) {
      const float4 u = rest[(sp - 1) * n4 + t];
      v.x += u.x;
      v.y += u.y;
      v.z += u.z;
      v.w += u.w;
    }
    xl1[t] = v;
  }
}

// Largest |RN32(x * smooth_inv)| of an M x K bf16 tensor, accumulated into *amax_bits
// (which holds float32 bits and starts at zero: non-negative floats order like
// their bit patterns, so an integer atomic max is exact). Units of 8 columns.
__global__ void tensor_absmax_kernel(const __nv_bfloat16* X, int ldx, const float* smooth_inv,
                                     int M, int K, uint32_t* amax_bits) {
  grid_dep_wait();
  grid_dep_launch();
  const int k8 = K / 8;
  const size_t units = static_cast<size_t>(M) * k8;
  float m = 0.0f;
#pragma unroll 4
  for (size_t u = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; u < units;
       u += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int row = static_cast<int>(u / k8), c = static_cast<int>(u % k8) * 8;
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(X + static_cast<size_t>(row) * ldx + c));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float sm[8] = {1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f};
    if (smooth_inv != nullptr) {
      const float4 s0 = __ldg(reinterpret_cast<const float4*>(smooth_inv + c));
      const float4 s1 = __ldg(reinterpret_cast<const float4*>(smooth_inv + c + 4));
      sm[0] = s0.x; sm[1] = s0.y; sm[2] = s0.z; sm[3] = s0.w;
      sm[4] = s1.x; sm[5] = s1.y; sm[6] = s1.z; sm[7] = s1.w;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float a = __fmul_rn(__uint_as_float(w[j] << 16), sm[2 * j]);  // exact when 1
      const float b = __fmul_rn(__uint_as_float(w[j] & 0xFFFF0000u), sm[2 * j + 1]);
      m = fmaxf(m, fmaxf(fabsf(a), fabsf(b)));
    }
  }
  uint32_t bits = __float_as_uint(m);
  bits = __reduce_max_sync(0xffffffffu, bits);
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, bits);
}

// scale[0] = s_t = RN32(amax / (6 * 448)) if that is a normal float32, else 1;
// scale[1] = RN32(1 / s_t). scale[0] holds the absolute maximum's bits on entry.
__global__ void tensor_scale_finalize_kernel(float* scale) {
  grid_dep_wait();
  grid_dep_launch();
  const float amax = __uint_as_float(*reinterpret_cast<const uint32_t*>(scale));
  float st = __fdiv_rn(amax, 2688.0f);
  if (!(st >= 1.17549435e-38f)) st = 1.0f;  // 2^-126, the smallest normal float32
  scale[0] = st;
  scale[1] = __frcp_rn(st);
}

// L1s = diag(smooth_inv) L1 as two bf16 planes [2][r][K] (hi, lo): hi = RN_bf16(v),
// lo = RN_bf16(v - hi), v = RN32(smooth_inv[k] * L1[k][j]).
__global__ void pack_lowrank_kernel(const __nv_bfloat16* L1, const float* smooth_inv,
                                    __nv_bfloat16* L1s, int K, int r) {
  const size_t total = static_cast<size_t>(K) * r;
  for (size_t t = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int j = static_cast<int>(t / K), k = static_cast<int>(t % K);
    float v = __bfloat162float(L1[static_cast<size_t>(k) * r + j]);
    if (smooth_inv != nullptr) v = __fmul_rn(v, smooth_inv[k]);
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    const __nv_bfloat16 lo = __float2bfloat16_rn(__fsub_rn(v, __bfloat162float(hi)));
    L1s[t] = hi;
    L1s[total + t] = lo;
  }
}

}  // namespace svdq

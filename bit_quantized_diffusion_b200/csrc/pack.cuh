// pack.cuh -- conversion between plain and tiled storage of quantized operands.
// Each kernel computes one output element per thread from the index formulas of
// the layouts declared in svdq.h (gathers on pack, the inverse on unpack).
#pragma once

#include "sm100.cuh"

namespace svdq {

__device__ __forceinline__ size_t nvfp4_scale_offset(int m, int j, int K) {
  const size_t atom = static_cast<size_t>(m / 128) * (K / 64) + j / 4;
  return atom * 512 + (m % 32) * 16 + ((m % 128) / 32) * 4 + (j % 4);
}

// tiled[t] <- plain[m, j] for every byte t of the atom layout (padding rows -> 0)
__global__ void pack_nvfp4_scales_kernel(const uint8_t* plain, uint8_t* tiled, int rows, int K) {
  const int J = K / 16;
  const size_t total = static_cast<size_t>((rows + 127) / 128) * 128 * J;
  for (size_t t = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t atom = t / 512;
    const int within = static_cast<int>(t % 512);
    const int kb_per_row = K / 64;
    const int mb = static_cast<int>(atom / kb_per_row), kb = static_cast<int>(atom % kb_per_row);
    const int m = mb * 128 + (within % 16) / 4 * 32 + within / 16;
    const int j = kb * 4 + within % 4;
    tiled[t] = m < rows ? plain[static_cast<size_t>(m) * J + j] : 0;
  }
}

__global__ void unpack_nvfp4_scales_kernel(const uint8_t* tiled, uint8_t* plain, int rows, int K) {
  const int J = K / 16;
  const size_t total = static_cast<size_t>(rows) * J;
  for (size_t t = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int m = static_cast<int>(t / J), j = static_cast<int>(t % J);
    plain[t] = tiled[nvfp4_scale_offset(m, j, K)];
  }
}

// INT4 scales: plain fp16 [rows, K/64] <-> group-major [K/64][rows padded to 128]
__global__ void pack_int4_scales_kernel(const uint16_t* plain, uint16_t* tiled, int rows, int K) {
  const int G = K / 64, rp = (rows + 127) / 128 * 128;
  const size_t total = static_cast<size_t>(G) * rp;
  for (size_t t = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int g = static_cast<int>(t / rp), m = static_cast<int>(t % rp);
    tiled[t] = m < rows ? plain[static_cast<size_t>(m) * G + g] : 0;
  }
}

__global__ void unpack_int4_scales_kernel(const uint16_t* tiled, uint16_t* plain, int rows, int K) {
  const int G = K / 64, rp = (rows + 127) / 128 * 128;
  const size_t total = static_cast<size_t>(rows) * G;
  for (size_t t = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int m = static_cast<int>(t / G), g = static_cast<int>(t % G);
    plain[t] = tiled[static_cast<size_t>(g) * rp + m];
  }
}

__global__ void copy_bytes_kernel(const uint4* src, uint4* dst, size_t n16) {
  for (size_t t = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; t < n16;
       t += static_cast<size_t>(gridDim.x) * blockDim.x)
    dst[t] = src[t];
}

// AWQ qweight: nibble slot s of word j of lane t in (block b, group g)
__device__ __constant__ int kAwqSlotRow[8] = {0, 8, 0, 8, 0, 8, 0, 8};
__device__ __constant__ int kAwqSlotCol[8] = {0, 0, 8, 8, 1, 1, 9, 9};

__global__ void pack_awq_qweight_kernel(const uint8_t* plain, uint32_t* tiled, int N, int K) {
  const int G = K / 64, NB = (N + 15) / 16;
  const size_t total = static_cast<size_t>(NB) * G * 32 * 4;  // words
  for (size_t t = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int j = static_cast<int>(t % 4);
    const int lane = static_cast<int>((t / 4) % 32);
    const size_t bg = t / 128;
    const int g = static_cast<int>(bg % G), b = static_cast<int>(bg / G);
    const int r0 = lane / 4, c0 = 2 * (lane % 4);
    uint32_t w = 0;
    for (int s = 0; s < 8; ++s) {
      const int n = b * 16 + r0 + kAwqSlotRow[s];
      const int k = g * 64 + 16 * j + c0 + kAwqSlotCol[s];
      uint32_t v = 0;
      if (n < N) {
        const uint8_t byte = plain[static_cast<size_t>(n) * (K / 2) + k / 2];
        v = (k & 1) ? (byte >> 4) : (byte & 0xF);
      }
      w |= v << (4 * s);
    }
    tiled[t] = w;
  }
}

// one thread per plain byte (two nibbles)
__global__ void unpack_awq_qweight_kernel(const uint32_t* tiled, uint8_t* plain, int N, int K) {
  const int G = K / 64;
  const size_t total = static_cast<size_t>(N) * (K / 2);
  for (size_t t = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int n = static_cast<int>(t / (K / 2));
    uint32_t out = 0;
    for (int h = 0; h < 2; ++h) {
      const int k = static_cast<int>(t % (K / 2)) * 2 + h;
      const int b = n / 16, rr = n % 16, g = k / 64, kk = k % 64;
      const int j = kk / 16, kc = kk % 16;
      // find the lane and slot holding (rr, kc): rows rr = r0 (+8), cols c0 (+1, +8, +9)
      const int r0 = rr % 8, hi_row = rr / 8;
      const int c0 = (kc % 8) / 2 * 2, dc = kc - c0;  // dc in {0, 1, 8, 9}
      const int lane = r0 * 4 + c0 / 2;
      int slot = 0;
      for (int s = 0; s < 8; ++s)
        if (kAwqSlotRow[s] == 8 * hi_row && kAwqSlotCol[s] == dc) slot = s;
      const uint32_t w = tiled[((static_cast<size_t>(b) * G + g) * 32 + lane) * 4 + j];
      out |= ((w >> (4 * slot)) & 0xFu) << (4 * h);
    }
    plain[t] = static_cast<uint8_t>(out);
  }
}

// (s, z) bf16 pairs: plain s, z [N, K/64] <-> [N/16][K/64][16][2]
__global__ void pack_awq_sz_kernel(const uint16_t* s, const uint16_t* z, uint32_t* tiled, int N,
                                   int K) {
  const int G = K / 64, NB = (N + 15) / 16;
  const size_t total = static_cast<size_t>(NB) * G * 16;
  for (size_t t = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int rr = static_cast<int>(t % 16);
    const size_t bg = t / 16;
    const int g = static_cast<int>(bg % G), b = static_cast<int>(bg / G);
    const int n = b * 16 + rr;
    uint32_t v = 0;
    if (n < N) {
      const size_t i = static_cast<size_t>(n) * G + g;
      v = static_cast<uint32_t>(s[i]) | (static_cast<uint32_t>(z[i]) << 16);
    }
    tiled[t] = v;
  }
}

__global__ void unpack_awq_sz_kernel(const uint32_t* tiled, uint16_t* s, uint16_t* z, int N,
                                     int K) {
  const int G = K / 64;
  const size_t total = static_cast<size_t>(N) * G;
  for (size_t t = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int n = static_cast<int>(t / G), g = static_cast<int>(t % G);
    const uint32_t v = tiled[((static_cast<size_t>(n / 16)) * G + g) * 16 + n % 16];
    s[t] = static_cast<uint16_t>(v & 0xFFFFu);
    z[t] = static_cast<uint16_t>(v >> 16);
  }
}

// Diagnostics: wait on a barrier nobody arrives at; the bounded wait runs out.
__global__ void debug_wait_timeout_kernel(uint32_t* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(b, 0, status, limit_ns);
  cta_sync_converged();
}

}  // namespace svdq

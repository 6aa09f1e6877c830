// svdq.cu -- the C ABI of include/svdq.h: argument checks, tensor-map
// construction, launch configuration and the device status word.
// All kernels live in this one translation unit.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <utility>

#include "../../include/svdq.h"
#include "awq.cuh"
#include "awq_gemm.cuh"
#include "int4_gemm.cuh"
#include "mlp_fc1.cuh"
#include "pack.cuh"
#include "prep.cuh"
#include "quantize_act.cuh"
#include "w4a4_gemm.cuh"

namespace {

using namespace svdq;

__device__ uint32_t g_svdq_status;

// Working space of svdq_quantize_act_noalloc: the partial down-projections of
// K splits 1 .. S-1, (S - 1) * M * r floats at most kXl1ScratchFloats (8 MiB).
// Nothing in it needs to start at zero (each call writes every element it
// reads); two such calls in flight at the same time race on it.
constexpr size_t kXl1ScratchFloats = size_t(1) << 21;
static __device__ __align__(256) float g_xl1_scratch[kXl1ScratchFloats];

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  int num_sms = 0;
  int gemm_pairs = 0;  // co-resident clusters of the CTA-pair NVFP4 GEMM
  int int4_pairs = 0;  // the same for the INT4 GEMM
  int mlp_pairs = 0;   // the same for the fused MLP's fc1
  int gemm_pair_mode = -1;  // -1: by shape; SVDQ_GEMM_PAIR=0/1 forces single-CTA / CTA-pair tiles
  uint32_t* status = nullptr;
  float* xl1_scratch = nullptr;  // device address of g_xl1_scratch
  bool pdl = true;  // programmatic dependent launch of the hot-path kernels (SVDQ_PDL=0: off)
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

// Launch a hot-path kernel. With programmatic dependent launch the grid may be
// scheduled while the previous grid in the stream is finishing: every such
// kernel runs grid_dep_wait before its first global access, so stream order
// holds, and only its launch and prologue overlap the previous grid's tail.
// cluster_x > 1 launches clusters of that many CTAs.
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(const DeviceInfo* d, void (*kern)(KArgs...), dim3 grid, dim3 block,
                          size_t smem, cudaStream_t stream, int cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  if (d->pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Per-device set-up (status word address, SM count, kernel attributes), done
// once per device with that device current.
svdq_status device_setup(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SVDQ_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    if (g_encode == nullptr) {
      cudaDriverEntryPointQueryResult q;
      void* fn = nullptr;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        return SVDQ_ERR_CUDA;
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    void* st = nullptr;
    if (cudaGetSymbolAddress(&st, g_svdq_status) != cudaSuccess) return SVDQ_ERR_CUDA;
    void* scratch = nullptr;  // this device's copy (the device is current here)
    if (cudaGetSymbolAddress(&scratch, g_xl1_scratch) != cudaSuccess) return SVDQ_ERR_CUDA;
    if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return SVDQ_ERR_CUDA;
    const int max_smem = 232448;
    if (cudaFuncSetAttribute(quantize_act_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             max_smem) != cudaSuccess ||
        cudaFuncSetAttribute(quantize_act_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             max_smem) != cudaSuccess ||
        cudaFuncSetAttribute(w4a4_nvfp4_gemm_kernel<false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(GmCfg<false>::kSmemBytes)) != cudaSuccess ||
        cudaFuncSetAttribute(w4a4_nvfp4_gemm_kernel<true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(GmCfg<true>::kSmemBytes)) != cudaSuccess ||
        cudaFuncSetAttribute(w4a4_nvfp4_gemm_kernel<false, true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(GmCfg<false, true>::kSmemBytes)) != cudaSuccess ||
        cudaFuncSetAttribute(w4a4_nvfp4_gemm_kernel<true, true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(GmCfg<true, true>::kSmemBytes)) != cudaSuccess)
      return SVDQ_ERR_CUDA;
    if (cudaFuncSetAttribute(w4a4_int4_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kI4SmemBytes)) != cudaSuccess ||
        cudaFuncSetAttribute(w4a4_mlp_fc1_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kMlSmemBytes)) != cudaSuccess)
      return SVDQ_ERR_CUDA;
    // all of the SM's unified L1/shared storage as shared memory, so that the
    // occupancy the host code plans for (e.g. two quantizer CTAs per SM) is real
    for (const void* f : {reinterpret_cast<const void*>(quantize_act_kernel<0>),
                          reinterpret_cast<const void*>(quantize_act_kernel<1>),
                          reinterpret_cast<const void*>(w4a4_nvfp4_gemm_kernel<false>),
                          reinterpret_cast<const void*>(w4a4_nvfp4_gemm_kernel<true>),
                          reinterpret_cast<const void*>(w4a4_nvfp4_gemm_kernel<false, true>),
                          reinterpret_cast<const void*>(w4a4_nvfp4_gemm_kernel<true, true>),
                          reinterpret_cast<const void*>(w4a4_int4_gemm_kernel<true>),
                          reinterpret_cast<const void*>(awq_gemm_kernel),
                          reinterpret_cast<const void*>(w4a4_mlp_fc1_kernel),
                          reinterpret_cast<const void*>(awq_gemv_kernel<1>),
                          reinterpret_cast<const void*>(awq_gemv_kernel<2>)})
      if (cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared) != cudaSuccess)
        return SVDQ_ERR_CUDA;
    if (cudaFuncSetAttribute(awq_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             max_smem) != cudaSuccess ||
        cudaFuncSetAttribute(awq_gemv_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             max_smem) != cudaSuccess ||
        cudaFuncSetAttribute(awq_gemv_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             max_smem) != cudaSuccess)
      return SVDQ_ERR_CUDA;
    {
      // how many 2-CTA clusters of the pair GEMM can be resident at once (a
      // persistent grid larger than that would run its last clusters late)
      auto pairs = [&](auto kern, int threads, size_t smem) {
        cudaLaunchConfig_t q = {};
        q.gridDim = dim3(2 * (d.num_sms / 2), 1, 1);
        q.blockDim = dim3(threads, 1, 1);
        q.dynamicSmemBytes = smem;
        cudaLaunchAttribute a[1];
        a[0].id = cudaLaunchAttributeClusterDimension;
        a[0].val.clusterDim.x = 2;
        a[0].val.clusterDim.y = 1;
        a[0].val.clusterDim.z = 1;
        q.attrs = a;
        q.numAttrs = 1;
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, kern, &q) != cudaSuccess || clusters <= 0) {
          (void)cudaGetLastError();
          clusters = d.num_sms / 2;
        }
        return clusters < d.num_sms / 2 ? clusters : d.num_sms / 2;
      };
      d.gemm_pairs = pairs(w4a4_nvfp4_gemm_kernel<true>, kGmThreads, GmCfg<true>::kSmemBytes);
      d.int4_pairs = pairs(w4a4_int4_gemm_kernel<true>, kI4Threads, kI4SmemBytes);
      d.mlp_pairs = pairs(w4a4_mlp_fc1_kernel, kMlThreads, kMlSmemBytes);
      if (std::getenv("SVDQ_DEBUG") != nullptr)
        std::fprintf(stderr, "svdq: %d SMs, %d / %d co-resident NVFP4 / INT4 GEMM CTA pairs\n",
                     d.num_sms, d.gemm_pairs, d.int4_pairs);
    }
    if (const char* e = std::getenv("SVDQ_GEMM_PAIR")) d.gemm_pair_mode = std::atoi(e) != 0;
    if (const char* e = std::getenv("SVDQ_PDL")) d.pdl = std::atoi(e) != 0;
    d.status = static_cast<uint32_t*>(st);
    d.xl1_scratch = static_cast<float*>(scratch);
    d.ready = true;
  }
  *out = &d;
  return SVDQ_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

bool debug_on() { return std::getenv("SVDQ_DEBUG") != nullptr; }

svdq_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess && debug_on()) std::fprintf(stderr, "svdq: launch failed: %s\n", cudaGetErrorString(e));
  return e == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA;
}

bool make_tmap_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* ptr, uint64_t inner,
                  uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                  CUtensorMapSwizzle swz) {
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS && debug_on())
    std::fprintf(stderr, "svdq: tensor map (dims %llu x %llu, box %u x %u) failed: %d\n",
                 static_cast<unsigned long long>(inner), static_cast<unsigned long long>(outer),
                 box_inner, box_outer, static_cast<int>(r));
  return r == CUDA_SUCCESS;
}

// A 3-D map over [outer][mid][inner] 8-byte elements, rows contiguous, for
// unswizzled boxes {inner, box_mid, box_outer} (the inner dimension whole).
bool make_tmap_3d_u64(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t mid, uint64_t outer,
                      uint32_t box_mid, uint32_t box_outer) {
  const cuuint64_t dims[3] = {inner, mid, outer};
  const cuuint64_t strides[2] = {inner * 8, inner * 8 * mid};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(inner), box_mid, box_outer};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT64, 3, const_cast<void*>(ptr), dims,
                              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS && debug_on())
    std::fprintf(stderr, "svdq: 3-d tensor map (%llu x %llu x %llu) failed: %d\n",
                 static_cast<unsigned long long>(inner), static_cast<unsigned long long>(mid),
                 static_cast<unsigned long long>(outer), static_cast<int>(r));
  return r == CUDA_SUCCESS;
}

bool rank_ok(int r) { return r == 0 || (r % 16 == 0 && r >= 16 && r <= 256); }

size_t pad128(int rows) { return (static_cast<size_t>(rows) + 127) / 128 * 128; }

unsigned grid_for(size_t n, unsigned threads) {
  size_t b = (n + threads - 1) / threads;
  if (b < 1) b = 1;
  if (b > 65535u * 8u) b = 65535u * 8u;
  return static_cast<unsigned>(b);
}

// INT4 W4A4 GEMM (w4a4_int4_gemm_kernel): packed codes [rows, K/2] as one-group
// boxes [128 rows x 32 B], group-major FP16 scales [K/64][rows padded to 128]
// as one-group boxes [128], Y as 32 x 32 TMA-store boxes. Always CTA pairs, at
// any M: each CTA's converters fill 128 of a tile's 256 weight rows, so one CTA
// alone would leave half of the tile's B operand unfilled. Rows of a pair's tile
// past M read as zeros (TMA fill) and are clipped by the TMA store.
svdq_status launch_int4_gemm(const DeviceInfo* d, int M, int N, int K, int r, const void* a_codes,
                             const void* a_scales, const float* xl1, const void* w_codes,
                             const void* w_scales, const void* L2, const void* bias, void* Y,
                             int ldy, svdq_out out, cudaStream_t stream) {
  const int ctas = 2;
  CUtensorMap tm_a, tm_b, tm_sa, tm_sw, tm_l2, tm_y;
  const uint64_t G = static_cast<uint64_t>(K / 64);
  if (!make_tmap_2d(&tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_codes, K / 2, M, K / 2, 32, kI4BM,
                    CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tmap_2d(&tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_codes, K / 2, N, K / 2, 32, kI4BM,
                    CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tmap_2d(&tm_sa, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, a_scales, pad128(M), G, pad128(M) * 2,
                    128, 1, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tmap_2d(&tm_sw, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, w_scales, pad128(N), G, pad128(N) * 2,
                    128, 1, CU_TENSOR_MAP_SWIZZLE_NONE))
    return SVDQ_ERR_CUDA;
  if (r > 0) {
    if (!make_tmap_2d(&tm_l2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L2, N, r,
                      static_cast<uint64_t>(N) * 2, 64, kI4LrK, CU_TENSOR_MAP_SWIZZLE_128B))
      return SVDQ_ERR_CUDA;
  } else {
    tm_l2 = tm_a;
  }
  // output: 32 x 32 boxes, bf16 rows of 64 B (64-byte swizzle) or f32 rows of 128 B
  const bool f32 = out == SVDQ_OUT_F32;
  const int esz = f32 ? 4 : 2;
  if (!make_tmap_2d(&tm_y, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                    Y, N, M, static_cast<uint64_t>(ldy) * esz, 32, 32,
                    f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B))
    return SVDQ_ERR_CUDA;
  I4Params p;
  p.M = M;
  p.N = N;
  p.K = K;
  p.r = r;
  p.xl1 = xl1;
  p.bias = static_cast<const __nv_bfloat16*>(bias);
  p.out_f32 = f32;
  p.status = d->status;
  p.tiles_m = (M + kI4BM * ctas - 1) / (kI4BM * ctas);
  p.tiles = p.tiles_m * ((N + kI4BN - 1) / kI4BN);
  const int units = p.tiles < d->int4_pairs ? p.tiles : d->int4_pairs;
  const cudaError_t e = launch_kernel(d, w4a4_int4_gemm_kernel<true>, dim3(units * 2), dim3(kI4Threads),
                                      kI4SmemBytes, stream, 2, tm_a, tm_b, tm_sa, tm_sw, tm_l2, tm_y, p);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return SVDQ_ERR_CUDA;
  }
  return launch_status();
}

// AWQ W4A16 on the tensor cores (awq_gemm_kernel): token tiles of T = M rounded
// up to 16 (at most 128), 128 weight rows per tile, one persistent CTA per SM;
// weights and (s, z) in the fragment order of svdq_pack(AWQ).
svdq_status launch_awq_gemm(const DeviceInfo* d, int M, int N, int K, const void* X,
                            const void* qweight, const void* sz, const void* bias, void* Y,
                            cudaStream_t stream) {
  const int T = M >= kAgMaxT ? kAgMaxT : (M + 15) / 16 * 16;
  const int tb = T <= 32 ? 32 : (T <= 64 ? 64 : 128);
  int stages = kAgMaxStages;
  while (stages > 2 && ag_smem_bytes(T, stages) > 232448) --stages;
  const int G = K / 64, nblocks = (N + 15) / 16;
  CUtensorMap tm_q, tm_sz, tm_x;
  if (!make_tmap_3d_u64(&tm_q, qweight, 64, G, nblocks, 1, 8) ||
      !make_tmap_3d_u64(&tm_sz, sz, 8, G, nblocks, 1, 8) ||
      !make_tmap_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, K, M, static_cast<uint64_t>(K) * 2, 64,
                    T, CU_TENSOR_MAP_SWIZZLE_128B))
    return SVDQ_ERR_CUDA;
  AgParams p;
  p.M = M;
  p.N = N;
  p.K = K;
  p.T = T;
  p.tb = tb;
  p.nbuf = 512 / tb;
  p.stages = stages;
  p.tiles_m = (M + kAgMaxT - 1) / kAgMaxT;
  p.tiles = p.tiles_m * ((N + kAgRows - 1) / kAgRows);
  p.sz = static_cast<const uint32_t*>(sz);
  p.bias = static_cast<const __nv_bfloat16*>(bias);
  p.Y = static_cast<__nv_bfloat16*>(Y);
  p.status = d->status;
  const int grid = p.tiles < d->num_sms ? p.tiles : d->num_sms;
  if (debug_on())
    std::fprintf(stderr, "awq_w4a16_linear (tensor cores): M=%d N=%d K=%d T=%d stages=%d tiles=%d grid=%d\n",
                 M, N, K, T, stages, p.tiles, grid);
  if (launch_kernel(d, awq_gemm_kernel, dim3(grid), dim3(kAgThreads), ag_smem_bytes(T, stages), stream, 1,
                    tm_q, tm_sz, tm_x, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return SVDQ_ERR_CUDA;
  }
  return launch_status();
}

svdq_status quantize_act_impl(svdq_format format, int M, int K, int r, const void* X, int ldx,
                              const float* smooth_inv, const void* L1s, void* codes, void* scales,
                              float* xl1, bool static_rest, svdq_stream_t stream,
                              const float* tensor_scale = nullptr) {
  if (format != SVDQ_NVFP4_G16 && format != SVDQ_INT4_G64) return SVDQ_ERR_INVALID_ARG;
  if (tensor_scale != nullptr && format != SVDQ_NVFP4_G16) return SVDQ_ERR_INVALID_ARG;
  if (tensor_scale != nullptr && (reinterpret_cast<uintptr_t>(tensor_scale) & 7u))
    return SVDQ_ERR_ALIGNMENT;
  if (M < 1 || K < 64 || K % 64 || !rank_ok(r) || ldx < K) return SVDQ_ERR_INVALID_ARG;
  if (X == nullptr || codes == nullptr || scales == nullptr) return SVDQ_ERR_INVALID_ARG;
  if ((r > 0) != (L1s != nullptr) || (r > 0) != (xl1 != nullptr)) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(codes) || !aligned16(scales) || ldx % 8 ||
      (smooth_inv && !aligned16(smooth_inv)) || (L1s && !aligned16(L1s)) ||
      (xl1 && !aligned16(xl1)))
    return SVDQ_ERR_ALIGNMENT;
  DeviceInfo* d = nullptr;
  if (svdq_status st = device_setup(&d); st != SVDQ_OK) return st;

  CUtensorMap tm_x, tm_l1;
  if (!make_tmap_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, K, M, static_cast<uint64_t>(ldx) * 2,
                    64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
    return SVDQ_ERR_CUDA;
  if (r > 0) {
    if (!make_tmap_2d(&tm_l1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L1s, K, 2 * r,
                      static_cast<uint64_t>(K) * 2, 64, r, CU_TENSOR_MAP_SWIZZLE_128B))
      return SVDQ_ERR_CUDA;
  } else {
    tm_l1 = tm_x;  // unused
  }

  const int row_blocks = (M + 127) / 128;
  // One CTA per SM (the kernel allocates tensor memory), K split into
  // qa_splits(M, K) ranges; ring stages of two 64-column sub-chunks where at
  // least two such stages fit, else of one.
  const int ksplit = qa_splits(M, K);
  const size_t budget = 227 * 1024;
  int spc = 0, stages = 0;
  for (int c = 2; c >= 1 && stages == 0; --c)
    for (int st = 8; st >= 2 && stages == 0; --st)
      if (qa_smem_bytes(r, st, c) <= budget) {
        spc = c;
        stages = st;
      }
  if (stages == 0) return SVDQ_ERR_UNSUPPORTED;
  const size_t smem_bytes = qa_smem_bytes(r, stages, spc);
  auto kern = format == SVDQ_NVFP4_G16 ? quantize_act_kernel<0> : quantize_act_kernel<1>;
  if (debug_on())
    std::fprintf(stderr,
                 "svdq_quantize_act: M=%d K=%d r=%d stages=%d x %d sub-chunks ksplit=%d grid=%d "
                 "smem=%zu\n",
                 M, K, r, stages, spc, ksplit, ksplit * row_blocks, smem_bytes);

  QuantActParams p;
  p.M = M;
  p.K = K;
  p.r = r;
  p.ksplit = ksplit;
  p.stages = stages;
  p.spc = spc;
  p.m_pad = static_cast<int>(pad128(M));
  p.smooth_inv = smooth_inv;
  p.tensor_scale = tensor_scale;
  p.codes = static_cast<uint8_t*>(codes);
  p.scales = static_cast<uint8_t*>(scales);
  // splits 1 .. S-1: the rest of the caller's buffer, or the library's static
  // working space (svdq_quantize_act_noalloc)
  const size_t rest_floats = static_cast<size_t>(ksplit - 1) * M * r;
  if (static_rest && r > 0 && rest_floats > kXl1ScratchFloats) {
    if (debug_on())
      std::fprintf(stderr,
                   "svdq_quantize_act_noalloc: needs %zu floats of working space, the static "
                   "array holds %zu\n",
                   rest_floats, kXl1ScratchFloats);
    return SVDQ_ERR_UNSUPPORTED;
  }
  p.xl1 = xl1;
  p.xl1_rest = r > 0 ? (static_rest ? d->xl1_scratch : xl1 + static_cast<size_t>(M) * r) : nullptr;
  p.status = d->status;
  const cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (launch_kernel(d, kern, dim3(ksplit, row_blocks, 1), dim3(kQaThreads), smem_bytes, cs, 1, tm_x,
                    tm_l1, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return SVDQ_ERR_CUDA;
  }
  if (r > 0 && ksplit > 1) {
    // xl1[0] += xl1[1] + ... + xl1[S-1], in order
    const size_t n4 = static_cast<size_t>(M) * r / 4;
    if (launch_kernel(d, xl1_reduce_kernel, dim3(grid_for(n4, 256)), dim3(256), 0, cs, 1,
                      reinterpret_cast<float4*>(xl1), reinterpret_cast<const float4*>(p.xl1_rest),
                      ksplit, n4) != cudaSuccess) {
      (void)cudaGetLastError();
      return SVDQ_ERR_CUDA;
    }
  }
  return launch_status();
}

}  // namespace

extern "C" {

const char* svdq_status_str(svdq_status s) {
  switch (s) {
    case SVDQ_OK: return "ok";
    case SVDQ_ERR_INVALID_ARG: return "invalid argument";
    case SVDQ_ERR_ALIGNMENT: return "pointer or leading dimension not 16-byte aligned";
    case SVDQ_ERR_UNSUPPORTED: return "unsupported by this build";
    case SVDQ_ERR_CUDA: return "CUDA error";
    case SVDQ_ERR_TIMEOUT: return "a kernel's bounded wait ran out";
  }
  return "unknown status";
}

int svdq_version(void) { return 100; }

size_t svdq_codes_bytes(svdq_format f, int rows, int K) {
  if ((f != SVDQ_NVFP4_G16 && f != SVDQ_INT4_G64) || rows < 1 || K < 64 || K % 64) return 0;
  return static_cast<size_t>(rows) * (K / 2);
}

size_t svdq_scales_bytes(svdq_format f, int rows, int K) {
  if (rows < 1 || K < 64 || K % 64) return 0;
  if (f == SVDQ_NVFP4_G16) return pad128(rows) * (K / 16);
  if (f == SVDQ_INT4_G64) return pad128(rows) * (K / 64) * 2;
  return 0;
}

size_t awq_qweight_bytes(int N, int K) {
  if (N < 1 || K < 64 || K % 64) return 0;
  return (static_cast<size_t>(N) + 15) / 16 * 16 * (K / 2);
}

size_t awq_sz_bytes(int N, int K) {
  if (N < 1 || K < 64 || K % 64) return 0;
  return (static_cast<size_t>(N) + 15) / 16 * 16 * (K / 64) * 4;
}

int svdq_xl1_splits(int M, int K, int r) {
  if (M < 1 || K < 64 || K % 64 || !rank_ok(r)) return 0;
  return r == 0 ? 1 : qa_splits(M, K);
}

svdq_status svdq_quantize_act(svdq_format format, int M, int K, int r, const void* X, int ldx,
                              const float* smooth_inv, const void* L1s, void* codes,
                              void* scales, float* xl1, svdq_stream_t stream) {
  return quantize_act_impl(format, M, K, r, X, ldx, smooth_inv, L1s, codes, scales, xl1, false,
                           stream);
}

svdq_status svdq_quantize_act_noalloc(svdq_format format, int M, int K, int r, const void* X,
                                      int ldx, const float* smooth_inv, const void* L1s,
                                      void* codes, void* scales, float* xl1,
                                      svdq_stream_t stream) {
  return quantize_act_impl(format, M, K, r, X, ldx, smooth_inv, L1s, codes, scales, xl1, true,
                           stream);
}

}  // extern "C"

namespace {

// the fused QKV epilogue's arguments (svdq_w4a4_linear_qkv_norm_rope)
struct QkNormArgs {
  int q_heads;
  float eps;
  const void* norm_q;
  const void* norm_k;
  const float* rope_cos;
  const float* rope_sin;
};

svdq_status w4a4_linear_impl(svdq_format format, int M, int N, int K, int r, const void* a_codes,
                             const void* a_scales, const float* xl1, const void* w_codes,
                             const void* w_scales, const void* L2, const void* bias, void* Y,
                             int ldy, svdq_out out, svdq_stream_t stream, const float* a_tscale,
                             const float* w_tscale, const QkNormArgs* qk = nullptr) {
  if (format != SVDQ_NVFP4_G16 && format != SVDQ_INT4_G64) return SVDQ_ERR_INVALID_ARG;
  if ((a_tscale != nullptr) != (w_tscale != nullptr)) return SVDQ_ERR_INVALID_ARG;
  if (a_tscale != nullptr && format != SVDQ_NVFP4_G16) return SVDQ_ERR_INVALID_ARG;
  if (a_tscale != nullptr && ((reinterpret_cast<uintptr_t>(a_tscale) & 3u) ||
                              (reinterpret_cast<uintptr_t>(w_tscale) & 3u)))
    return SVDQ_ERR_ALIGNMENT;
  if (out != SVDQ_OUT_BF16 && out != SVDQ_OUT_F32) return SVDQ_ERR_INVALID_ARG;
  if (M < 1 || N < 16 || N % 16 || K < 64 || K % 64 || !rank_ok(r) || ldy < N)
    return SVDQ_ERR_INVALID_ARG;
  if (!a_codes || !a_scales || !w_codes || !w_scales || !Y) return SVDQ_ERR_INVALID_ARG;
  if ((r > 0) != (xl1 != nullptr) || (r > 0) != (L2 != nullptr)) return SVDQ_ERR_INVALID_ARG;
  const int esz = out == SVDQ_OUT_F32 ? 4 : 2;
  if (!aligned16(a_codes) || !aligned16(a_scales) || !aligned16(w_codes) || !aligned16(w_scales) ||
      !aligned16(Y) || (xl1 && !aligned16(xl1)) || (L2 && !aligned16(L2)) ||
      (bias && !aligned16(bias)) || (static_cast<size_t>(ldy) * esz) % 16)
    return SVDQ_ERR_ALIGNMENT;
  if (qk != nullptr && format != SVDQ_NVFP4_G16) return SVDQ_ERR_UNSUPPORTED;
  DeviceInfo* d = nullptr;
  if (svdq_status st = device_setup(&d); st != SVDQ_OK) return st;
  if (format == SVDQ_INT4_G64)
    return launch_int4_gemm(d, M, N, K, r, a_codes, a_scales, xl1, w_codes, w_scales, L2, bias, Y,
                            ldy, out, static_cast<cudaStream_t>(stream));

  // CTA pairs (cta_group::2, 256-row tiles): each CTA stages half of B, so a
  // pair moves a third less operand data per MMA than two single CTAs; measured
  // on B200 they are faster at every shape once the pair's cross-CTA arrivals
  // use CTA-scope release (QKV 70.3 vs 75.0 us, fc1 r=128 115.8 vs 122.1 us).
  const bool pair_auto = true;
  const bool pair = (d->gemm_pair_mode < 0 ? pair_auto : d->gemm_pair_mode != 0) && M > kGmBM;
  const int ctas = pair ? 2 : 1;
  const int b_rows = kGmBN / ctas;
  CUtensorMap tm_a, tm_b, tm_sfa, tm_sfb, tm_l2, tm_xl1, tm_y;
  const uint64_t kb = static_cast<uint64_t>(K / 64);
  if (!make_tmap_2d(&tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_codes, K / 2, M, K / 2, kGmBKBytes,
                    kGmBM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_codes, K / 2, N, K / 2, kGmBKBytes,
                    b_rows, CU_TENSOR_MAP_SWIZZLE_128B) ||
      // scale atoms as rows of 256 B (two rows per 512-byte atom), 8 rows = 4 atoms per box
      !make_tmap_2d(&tm_sfa, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_scales, 256, pad128(M) / 128 * kb * 2,
                    256, 256, 8, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tmap_2d(&tm_sfb, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_scales, 256, pad128(N) / 128 * kb * 2,
                    256, 256, 8, CU_TENSOR_MAP_SWIZZLE_NONE))
    return SVDQ_ERR_CUDA;
  if (r > 0) {
    // xl1 [M, r] float32 in chunks of 32 columns x 128 rows, 128-byte swizzle
    if (!make_tmap_2d(&tm_l2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L2, N, r,
                      static_cast<uint64_t>(N) * 2, 64, kGmLrK, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_2d(&tm_xl1, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, xl1, r, M,
                      static_cast<uint64_t>(r) * 4, kGmLrK, kGmBM, CU_TENSOR_MAP_SWIZZLE_128B))
      return SVDQ_ERR_CUDA;
  } else {
    tm_l2 = tm_a;
    tm_xl1 = tm_a;
  }
  // output: 32 x 32 boxes, bf16 rows of 64 B (64-byte swizzle) or f32 rows of 128 B
  const bool f32 = out == SVDQ_OUT_F32;
  if (!make_tmap_2d(&tm_y, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                    Y, N, M, static_cast<uint64_t>(ldy) * esz, 32, 32,
                    f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B))
    return SVDQ_ERR_CUDA;
  GemmParams p;
  p.M = M;
  p.N = N;
  p.K = K;
  p.r = r;
  p.bias = static_cast<const __nv_bfloat16*>(bias);
  p.a_tscale = a_tscale;
  p.w_tscale = w_tscale;
  p.out_f32 = f32;
  p.status = d->status;
  p.q_heads = qk != nullptr ? qk->q_heads : 0;
  p.eps = qk != nullptr ? qk->eps : 0.0f;
  p.norm_q = qk != nullptr ? static_cast<const __nv_bfloat16*>(qk->norm_q) : nullptr;
  p.norm_k = qk != nullptr ? static_cast<const __nv_bfloat16*>(qk->norm_k) : nullptr;
  p.rope_cos = qk != nullptr ? qk->rope_cos : nullptr;
  p.rope_sin = qk != nullptr ? qk->rope_sin : nullptr;
  p.tiles_m = (M + kGmBM * ctas - 1) / (kGmBM * ctas);
  p.tiles = p.tiles_m * ((N + kGmBN - 1) / kGmBN);
  const int max_units = pair ? d->gemm_pairs : d->num_sms;
  const int units = p.tiles < max_units ? p.tiles : max_units;
  const cudaStream_t cs = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (qk != nullptr)
    e = pair ? launch_kernel(d, w4a4_nvfp4_gemm_kernel<true, true>, dim3(units * 2), dim3(kGmThreads),
                             GmCfg<true, true>::kSmemBytes, cs, 2, tm_a, tm_b, tm_sfa, tm_sfb, tm_l2,
                             tm_xl1, tm_y, p)
             : launch_kernel(d, w4a4_nvfp4_gemm_kernel<false, true>, dim3(units), dim3(kGmThreads),
                             GmCfg<false, true>::kSmemBytes, cs, 1, tm_a, tm_b, tm_sfa, tm_sfb, tm_l2,
                             tm_xl1, tm_y, p);
  else
    e = pair ? launch_kernel(d, w4a4_nvfp4_gemm_kernel<true>, dim3(units * 2), dim3(kGmThreads),
                             GmCfg<true>::kSmemBytes, cs, 2, tm_a, tm_b, tm_sfa, tm_sfb, tm_l2, tm_xl1,
                             tm_y, p)
             : launch_kernel(d, w4a4_nvfp4_gemm_kernel<false>, dim3(units), dim3(kGmThreads),
                             GmCfg<false>::kSmemBytes, cs, 1, tm_a, tm_b, tm_sfa, tm_sfb, tm_l2, tm_xl1,
                             tm_y, p);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return SVDQ_ERR_CUDA;
  }
  return launch_status();
}

}  // namespace

extern "C" {

svdq_status svdq_w4a4_linear(svdq_format format, int M, int N, int K, int r, const void* a_codes,
                             const void* a_scales, const float* xl1, const void* w_codes,
                             const void* w_scales, const void* L2, const void* bias, void* Y,
                             int ldy, svdq_out out, svdq_stream_t stream) {
  return w4a4_linear_impl(format, M, N, K, r, a_codes, a_scales, xl1, w_codes, w_scales, L2, bias,
                          Y, ldy, out, stream, nullptr, nullptr);
}

svdq_status svdq_w4a4_linear_two_level(int M, int N, int K, int r, const void* a_codes,
                                       const void* a_scales, const float* a_tensor_scale,
                                       const float* xl1, const void* w_codes, const void* w_scales,
                                       const float* w_tensor_scale, const void* L2, const void* bias,
                                       void* Y, int ldy, svdq_out out, svdq_stream_t stream) {
  if (a_tensor_scale == nullptr || w_tensor_scale == nullptr) return SVDQ_ERR_INVALID_ARG;
  return w4a4_linear_impl(SVDQ_NVFP4_G16, M, N, K, r, a_codes, a_scales, xl1, w_codes, w_scales,
                          L2, bias, Y, ldy, out, stream, a_tensor_scale, w_tensor_scale);
}

svdq_status svdq_w4a4_linear_qkv_norm_rope(int M, int N, int K, int r, const void* a_codes,
                                           const void* a_scales, const float* xl1,
                                           const void* w_codes, const void* w_scales, const void* L2,
                                           const void* bias, const void* norm_q, const void* norm_k,
                                           float eps, const float* rope_cos, const float* rope_sin,
                                           void* Y, int ldy, svdq_out out, svdq_stream_t stream) {
  if (N < 384 || N % 384 || !(eps >= 0.0f) || eps > 3.0e38f) return SVDQ_ERR_INVALID_ARG;
  if ((rope_cos != nullptr) != (rope_sin != nullptr)) return SVDQ_ERR_INVALID_ARG;
  if ((rope_cos && (!aligned4(rope_cos) || !aligned4(rope_sin))) ||
      (reinterpret_cast<uintptr_t>(norm_q) & 1u) || (reinterpret_cast<uintptr_t>(norm_k) & 1u))
    return SVDQ_ERR_ALIGNMENT;
  const QkNormArgs qk{N / 384, eps, norm_q, norm_k, rope_cos, rope_sin};
  return w4a4_linear_impl(SVDQ_NVFP4_G16, M, N, K, r, a_codes, a_scales, xl1, w_codes, w_scales,
                          L2, bias, Y, ldy, out, stream, nullptr, nullptr, &qk);
}

int svdq_mlp_splits(int M, int N1) {
  if (M < 1 || N1 < kMlBN || N1 % kMlBN) return 0;
  DeviceInfo* d = nullptr;
  if (device_setup(&d) != SVDQ_OK) return 0;
  const int row_blocks = (M + 2 * kMlBM - 1) / (2 * kMlBM), ntn = N1 / kMlBN;
  int nsplit = d->mlp_pairs / row_blocks;
  if (nsplit < 1) nsplit = 1;
  if (nsplit > 8) nsplit = 8;
  if (nsplit > ntn) nsplit = ntn;
  const int tps = (ntn + nsplit - 1) / nsplit;
  return (ntn + tps - 1) / tps;
}

svdq_status svdq_mlp_fc1(int M, int N1, int K1, int r1, int r2, const void* a_codes, const void* a_scales,
                         const float* xl1_1, const void* w_codes, const void* w_scales, const void* L2_1,
                         const void* bias1, const float* smooth_inv2, const void* L1t_2, void* codes2,
                         void* scales2, float* xl1_2, float* hhat, svdq_stream_t stream) {
  if (M < 1 || N1 < kMlBN || N1 % kMlBN || K1 < 64 || K1 % 64 || !rank_ok(r1)) return SVDQ_ERR_INVALID_ARG;
  if (r2 < 0 || r2 > kMlR2Max || r2 % 32) return SVDQ_ERR_INVALID_ARG;
  if (!a_codes || !a_scales || !w_codes || !w_scales || !codes2 || !scales2) return SVDQ_ERR_INVALID_ARG;
  if ((r1 > 0) != (xl1_1 != nullptr) || (r1 > 0) != (L2_1 != nullptr)) return SVDQ_ERR_INVALID_ARG;
  if ((r2 > 0) != (L1t_2 != nullptr) || (r2 > 0) != (xl1_2 != nullptr)) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(a_codes) || !aligned16(a_scales) || !aligned16(w_codes) || !aligned16(w_scales) ||
      !aligned16(codes2) || !aligned16(scales2) || (xl1_1 && !aligned16(xl1_1)) || (L2_1 && !aligned16(L2_1)) ||
      (L1t_2 && !aligned16(L1t_2)) || (xl1_2 && !aligned16(xl1_2)) || (hhat && !aligned16(hhat)) ||
      (smooth_inv2 && (reinterpret_cast<uintptr_t>(smooth_inv2) & 3u)) ||
      (bias1 && (reinterpret_cast<uintptr_t>(bias1) & 1u)))
    return SVDQ_ERR_ALIGNMENT;
  DeviceInfo* d = nullptr;
  if (svdq_status st = device_setup(&d); st != SVDQ_OK) return st;
  const uint64_t kb = static_cast<uint64_t>(K1 / 64);
  CUtensorMap tm_a, tm_b, tm_sfa, tm_sfb, tm_l2, tm_xl1, tm_l1t;
  if (!make_tmap_2d(&tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_codes, K1 / 2, M, K1 / 2, 128, kMlBM,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_codes, K1 / 2, N1, K1 / 2, 128, kMlBRows,
                    CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tm_sfa, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_scales, 256, pad128(M) / 128 * kb * 2, 256, 256,
                    8, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tmap_2d(&tm_sfb, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_scales, 256, pad128(N1) / 128 * kb * 2, 256,
                    256, 8, CU_TENSOR_MAP_SWIZZLE_NONE))
    return SVDQ_ERR_CUDA;
  if (r1 > 0) {
    if (!make_tmap_2d(&tm_l2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L2_1, N1, r1, static_cast<uint64_t>(N1) * 2,
                      64, kMlLrK, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_2d(&tm_xl1, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, xl1_1, r1, M, static_cast<uint64_t>(r1) * 4,
                      kMlLrK, kMlBM, CU_TENSOR_MAP_SWIZZLE_128B))
      return SVDQ_ERR_CUDA;
  } else {
    tm_l2 = tm_a;
    tm_xl1 = tm_a;
  }
  if (r2 > 0) {
    // L1_2^T [r2, N1] bf16: 64-column boxes of this CTA's r2 / 2 ranks
    if (!make_tmap_2d(&tm_l1t, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L1t_2, N1, r2, static_cast<uint64_t>(N1) * 2,
                      64, r2 / 2, CU_TENSOR_MAP_SWIZZLE_128B))
      return SVDQ_ERR_CUDA;
  } else {
    tm_l1t = tm_a;
  }
  MlpParams p;
  p.M = M;
  p.N1 = N1;
  p.K1 = K1;
  p.r1 = r1;
  p.r2 = r2;
  p.row_blocks = (M + 2 * kMlBM - 1) / (2 * kMlBM);
  p.ntn = N1 / kMlBN;
  p.nsplit = svdq_mlp_splits(M, N1);
  p.tps = (p.ntn + p.nsplit - 1) / p.nsplit;
  p.units = p.row_blocks * p.nsplit;
  p.bias1 = static_cast<const __nv_bfloat16*>(bias1);
  p.smooth_inv2 = smooth_inv2;
  p.codes2 = static_cast<uint8_t*>(codes2);
  p.scales2 = static_cast<uint8_t*>(scales2);
  p.xl1_part = xl1_2;
  p.hhat = hhat;
  p.status = d->status;
  const int pairs = p.units < d->mlp_pairs ? p.units : d->mlp_pairs;
  const cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (debug_on())
    std::fprintf(stderr, "svdq_mlp_fc1: M=%d N1=%d K1=%d r1=%d r2=%d units=%d (splits %d, %d tiles each) pairs=%d\n",
                 M, N1, K1, r1, r2, p.units, p.nsplit, p.tps, pairs);
  if (launch_kernel(d, w4a4_mlp_fc1_kernel, dim3(2 * pairs), dim3(kMlThreads), kMlSmemBytes, cs, 2, tm_a, tm_b,
                    tm_sfa, tm_sfb, tm_l2, tm_xl1, tm_l1t, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return SVDQ_ERR_CUDA;
  }
  if (r2 > 0 && p.nsplit > 1) {
    // xl1_2[0] += xl1_2[1] + ... in order
    const size_t n4 = static_cast<size_t>(M) * r2 / 4;
    if (launch_kernel(d, xl1_reduce_kernel, dim3(grid_for(n4, 256)), dim3(256), 0, cs, 1,
                      reinterpret_cast<float4*>(xl1_2), reinterpret_cast<const float4*>(xl1_2 + static_cast<size_t>(M) * r2),
                      p.nsplit, n4) != cudaSuccess) {
      (void)cudaGetLastError();
      return SVDQ_ERR_CUDA;
    }
  }
  return launch_status();
}

svdq_status svdq_tensor_scale(int M, int K, const void* X, int ldx, const float* smooth_inv,
                              float* scale, svdq_stream_t stream) {
  if (M < 1 || K < 64 || K % 64 || ldx < K || ldx % 8 || !X || !scale) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X) || (reinterpret_cast<uintptr_t>(scale) & 7u) ||
      (smooth_inv && !aligned16(smooth_inv)))
    return SVDQ_ERR_ALIGNMENT;
  DeviceInfo* d = nullptr;
  if (svdq_status st = device_setup(&d); st != SVDQ_OK) return st;
  const cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(scale, 0, sizeof(float), cs) != cudaSuccess) {
    (void)cudaGetLastError();
    return SVDQ_ERR_CUDA;
  }
  const size_t units = static_cast<size_t>(M) * (K / 8);
  unsigned grid = grid_for(units, 256);
  if (grid > static_cast<unsigned>(4 * d->num_sms)) grid = 4 * d->num_sms;
  if (launch_kernel(d, tensor_absmax_kernel, dim3(grid), dim3(256), 0, cs, 1,
                    static_cast<const __nv_bfloat16*>(X), ldx, smooth_inv, M, K,
                    reinterpret_cast<uint32_t*>(scale)) != cudaSuccess ||
      launch_kernel(d, tensor_scale_finalize_kernel, dim3(1), dim3(1), 0, cs, 1, scale) !=
          cudaSuccess) {
    (void)cudaGetLastError();
    return SVDQ_ERR_CUDA;
  }
  return launch_status();
}

svdq_status svdq_quantize_act_two_level(int M, int K, int r, const void* X, int ldx,
                                        const float* smooth_inv, const float* tensor_scale,
                                        const void* L1s, void* codes, void* scales, float* xl1,
                                        svdq_stream_t stream) {
  if (tensor_scale == nullptr) return SVDQ_ERR_INVALID_ARG;
  return quantize_act_impl(SVDQ_NVFP4_G16, M, K, r, X, ldx, smooth_inv, L1s, codes, scales, xl1,
                           false, stream, tensor_scale);
}

svdq_status awq_w4a16_linear(int M, int N, int K, int group, const void* X, const void* qweight,
                             const void* sz, const void* bias, void* Y, svdq_stream_t stream) {
  if (group != 64 || M < 1 || N < 1 || K < 64 || K % 64) return SVDQ_ERR_INVALID_ARG;
  if (!X || !qweight || !sz || !Y) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(qweight) || !aligned16(sz) || !aligned16(Y) ||
      (bias && (reinterpret_cast<uintptr_t>(bias) & 1)))
    return SVDQ_ERR_ALIGNMENT;
  DeviceInfo* d = nullptr;
  if (svdq_status st = device_setup(&d); st != SVDQ_OK) return st;
  // the path by M; SVDQ_AWQ_PATH=0 / 1 forces the GEMV / the tensor-core GEMM (read per call)
  const char* force = std::getenv("SVDQ_AWQ_PATH");
  const bool gemm = force != nullptr ? std::atoi(force) != 0 : M > kAwqMaxM;
  if (gemm) return launch_awq_gemm(d, M, N, K, X, qweight, sz, bias, Y, static_cast<cudaStream_t>(stream));
  if (M > kAwqMaxM) return SVDQ_ERR_UNSUPPORTED;  // the GEMV was forced
  // tokens per launch: at most 16 (two 8-token MMA blocks), and as many X rows
  // as fit in shared memory beside a weight ring of at least two stages
  const size_t smem_cap = 232448;
  auto fits = [&](int mc, int stages) {
    return awq_smem_bytes(mc, K, mc > 8 ? 2 : 1, stages) <= smem_cap;
  };
  int mc = M < 16 ? M : 16;
  while (mc > 1 && !fits(mc, 2)) --mc;
  if (!fits(mc, 2)) return SVDQ_ERR_UNSUPPORTED;
  const int nblocks = (N + 15) / 16;
  // one persistent CTA per SM, each streaming a contiguous run of 16-row blocks,
  // taken bpr at a time: the smallest power of two (<= 8) covering its blocks
  const int grid = nblocks < d->num_sms ? nblocks : d->num_sms;
  const int per_cta = (nblocks + grid - 1) / grid;
  int bpr = 1;
  while (bpr < per_cta && bpr < 8) bpr *= 2;
  // the stage boxes: weights [blocks][groups][64 x 8 B], (s, z) [blocks][groups][8 x 8 B]
  const int G = K / 64, wpb = kAwqConsumers / bpr, gsk = kAwqWarpGroups * wpb;
  CUtensorMap tm_q, tm_sz;
  if (!make_tmap_3d_u64(&tm_q, qweight, 64, G, nblocks, gsk, bpr) ||
      !make_tmap_3d_u64(&tm_sz, sz, 8, G, nblocks, gsk, bpr))
    return SVDQ_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  for (int m0 = 0; m0 < M; m0 += mc) {
    const int mm = M - m0 < mc ? M - m0 : mc;
    const int kmb = mm > 8 ? 2 : 1;
    int stages = kAwqMaxStages;
    while (stages > 2 && awq_smem_bytes(mm, K, kmb, stages) > smem_cap) --stages;
    AwqParams p;
    p.M = mm;
    p.N = N;
    p.K = K;
    p.stages = stages;
    p.bpr = bpr;
    p.X = static_cast<const __nv_bfloat16*>(X) + static_cast<size_t>(m0) * K;
    p.qweight = static_cast<const uint4*>(qweight);
    p.sz = static_cast<const uint32_t*>(sz);
    p.bias = static_cast<const __nv_bfloat16*>(bias);
    p.Y = static_cast<__nv_bfloat16*>(Y) + static_cast<size_t>(m0) * N;
    p.status = d->status;
    const size_t smem = awq_smem_bytes(mm, K, kmb, stages);
    const cudaError_t e =
        kmb == 1 ? launch_kernel(d, awq_gemv_kernel<1>, dim3(grid), dim3(kAwqThreads), smem, s, 1,
                                 tm_q, tm_sz, p)
                 : launch_kernel(d, awq_gemv_kernel<2>, dim3(grid), dim3(kAwqThreads), smem, s, 1,
                                 tm_q, tm_sz, p);
    if (e != cudaSuccess) {
      (void)cudaGetLastError();
      return SVDQ_ERR_CUDA;
    }
  }
  return launch_status();
}

svdq_status svdq_pack(svdq_pack_kind kind, svdq_format format, int rows, int K,
                      const void* plain_codes, const void* plain_scales, const void* plain_zeros,
                      void* tiled_codes, void* tiled_scales, svdq_stream_t stream) {
  if (rows < 1 || K < 64 || K % 64) return SVDQ_ERR_INVALID_ARG;
  if (!plain_codes || !plain_scales || !tiled_codes || !tiled_scales) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(plain_codes) || !aligned16(tiled_codes) || !aligned16(tiled_scales) ||
      (reinterpret_cast<uintptr_t>(plain_scales) & 1))
    return SVDQ_ERR_ALIGNMENT;
  if (kind != SVDQ_PACK_ACT && kind != SVDQ_PACK_WEIGHT && kind != SVDQ_PACK_AWQ)
    return SVDQ_ERR_INVALID_ARG;
  if (kind == SVDQ_PACK_AWQ) {
    if (plain_zeros == nullptr || (reinterpret_cast<uintptr_t>(plain_zeros) & 1)) return SVDQ_ERR_INVALID_ARG;
  } else if (plain_zeros != nullptr || (format != SVDQ_NVFP4_G16 && format != SVDQ_INT4_G64)) {
    return SVDQ_ERR_INVALID_ARG;
  }
  DeviceInfo* d = nullptr;
  if (svdq_status st = device_setup(&d); st != SVDQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const unsigned T = 256;
  if (kind == SVDQ_PACK_ACT || kind == SVDQ_PACK_WEIGHT) {
    if (plain_zeros != nullptr) return SVDQ_ERR_INVALID_ARG;
    if (format != SVDQ_NVFP4_G16 && format != SVDQ_INT4_G64) return SVDQ_ERR_INVALID_ARG;
    const size_t n16 = static_cast<size_t>(rows) * (K / 2) / 16;
    // the tiled codes of both formats are the plain bytes
    copy_bytes_kernel<<<grid_for(n16, T), T, 0, s>>>(static_cast<const uint4*>(plain_codes),
                                                     static_cast<uint4*>(tiled_codes), n16);
    if (format == SVDQ_NVFP4_G16) {
      const size_t n = pad128(rows) * (K / 16);
      pack_nvfp4_scales_kernel<<<grid_for(n, T), T, 0, s>>>(
          static_cast<const uint8_t*>(plain_scales), static_cast<uint8_t*>(tiled_scales), rows, K);
    } else {
      const size_t n = pad128(rows) * (K / 64);
      pack_int4_scales_kernel<<<grid_for(n, T), T, 0, s>>>(
          static_cast<const uint16_t*>(plain_scales), static_cast<uint16_t*>(tiled_scales), rows,
          K);
    }
    return launch_status();
  }
  if (kind == SVDQ_PACK_AWQ) {
    if (plain_zeros == nullptr || (reinterpret_cast<uintptr_t>(plain_zeros) & 1))
      return SVDQ_ERR_INVALID_ARG;
    const size_t nw = (static_cast<size_t>(rows) + 15) / 16 * (K / 64) * 128;
    pack_awq_qweight_kernel<<<grid_for(nw, T), T, 0, s>>>(
        static_cast<const uint8_t*>(plain_codes), static_cast<uint32_t*>(tiled_codes), rows, K);
    const size_t ns = (static_cast<size_t>(rows) + 15) / 16 * (K / 64) * 16;
    pack_awq_sz_kernel<<<grid_for(ns, T), T, 0, s>>>(
        static_cast<const uint16_t*>(plain_scales), static_cast<const uint16_t*>(plain_zeros),
        static_cast<uint32_t*>(tiled_scales), rows, K);
    return launch_status();
  }
  return SVDQ_ERR_INVALID_ARG;
}

svdq_status svdq_unpack(svdq_pack_kind kind, svdq_format format, int rows, int K,
                        const void* tiled_codes, const void* tiled_scales, void* plain_codes,
                        void* plain_scales, void* plain_zeros, svdq_stream_t stream) {
  if (rows < 1 || K < 64 || K % 64) return SVDQ_ERR_INVALID_ARG;
  if (!plain_codes || !plain_scales || !tiled_codes || !tiled_scales) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(plain_codes) || !aligned16(tiled_codes) || !aligned16(tiled_scales) ||
      (reinterpret_cast<uintptr_t>(plain_scales) & 1))
    return SVDQ_ERR_ALIGNMENT;
  if (kind != SVDQ_PACK_ACT && kind != SVDQ_PACK_WEIGHT && kind != SVDQ_PACK_AWQ)
    return SVDQ_ERR_INVALID_ARG;
  if (kind == SVDQ_PACK_AWQ) {
    if (plain_zeros == nullptr || (reinterpret_cast<uintptr_t>(plain_zeros) & 1)) return SVDQ_ERR_INVALID_ARG;
  } else if (plain_zeros != nullptr || (format != SVDQ_NVFP4_G16 && format != SVDQ_INT4_G64)) {
    return SVDQ_ERR_INVALID_ARG;
  }
  DeviceInfo* d = nullptr;
  if (svdq_status st = device_setup(&d); st != SVDQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const unsigned T = 256;
  if (kind == SVDQ_PACK_ACT || kind == SVDQ_PACK_WEIGHT) {
    if (plain_zeros != nullptr) return SVDQ_ERR_INVALID_ARG;
    if (format != SVDQ_NVFP4_G16 && format != SVDQ_INT4_G64) return SVDQ_ERR_INVALID_ARG;
    const size_t n16 = static_cast<size_t>(rows) * (K / 2) / 16;
    copy_bytes_kernel<<<grid_for(n16, T), T, 0, s>>>(static_cast<const uint4*>(tiled_codes),
                                                     static_cast<uint4*>(plain_codes), n16);
    if (format == SVDQ_NVFP4_G16) {
      const size_t n = static_cast<size_t>(rows) * (K / 16);
      unpack_nvfp4_scales_kernel<<<grid_for(n, T), T, 0, s>>>(
          static_cast<const uint8_t*>(tiled_scales), static_cast<uint8_t*>(plain_scales), rows, K);
    } else {
      const size_t n = static_cast<size_t>(rows) * (K / 64);
      unpack_int4_scales_kernel<<<grid_for(n, T), T, 0, s>>>(
          static_cast<const uint16_t*>(tiled_scales), static_cast<uint16_t*>(plain_scales), rows,
          K);
    }
    return launch_status();
  }
  if (kind == SVDQ_PACK_AWQ) {
    if (plain_zeros == nullptr || (reinterpret_cast<uintptr_t>(plain_zeros) & 1))
      return SVDQ_ERR_INVALID_ARG;
    const size_t nb = static_cast<size_t>(rows) * (K / 2);
    unpack_awq_qweight_kernel<<<grid_for(nb, T), T, 0, s>>>(
        static_cast<const uint32_t*>(tiled_codes), static_cast<uint8_t*>(plain_codes), rows, K);
    const size_t ns = static_cast<size_t>(rows) * (K / 64);
    unpack_awq_sz_kernel<<<grid_for(ns, T), T, 0, s>>>(
        static_cast<const uint32_t*>(tiled_scales), static_cast<uint16_t*>(plain_scales),
        static_cast<uint16_t*>(plain_zeros), rows, K);
    return launch_status();
  }
  return SVDQ_ERR_INVALID_ARG;
}

svdq_status svdq_pack_lowrank(int K, int r, const void* L1, const float* smooth_inv, void* L1s,
                              svdq_stream_t stream) {
  if (K < 64 || K % 64 || r < 16 || r > 256 || r % 16 || !L1 || !L1s) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(L1) || !aligned16(L1s) || (smooth_inv && !aligned16(smooth_inv)))
    return SVDQ_ERR_ALIGNMENT;
  DeviceInfo* d = nullptr;
  if (svdq_status st = device_setup(&d); st != SVDQ_OK) return st;
  const size_t n = static_cast<size_t>(K) * r;
  pack_lowrank_kernel<<<grid_for(n, 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(L1), smooth_inv, static_cast<__nv_bfloat16*>(L1s), K, r);
  return launch_status();
}

svdq_status svdq_column_absmax(int rows, int K, const void* A, int lda, float* absmax,
                               svdq_stream_t stream) {
  if (rows < 1 || K < 8 || K % 8 || lda < K || lda % 8 || !A || !absmax) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(A) || (reinterpret_cast<uintptr_t>(absmax) & 3u)) return SVDQ_ERR_ALIGNMENT;
  DeviceInfo* d = nullptr;
  if (svdq_status st = device_setup(&d); st != SVDQ_OK) return st;
  const cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(absmax, 0, static_cast<size_t>(K) * sizeof(float), cs) != cudaSuccess) {
    (void)cudaGetLastError();
    return SVDQ_ERR_CUDA;
  }
  // at least one thread per 8 columns; the rows are split among the rest
  const size_t units = static_cast<size_t>(K / 8);
  unsigned grid = grid_for(units * static_cast<size_t>(rows), 256);
  if (grid > static_cast<unsigned>(4 * d->num_sms)) grid = 4 * d->num_sms;
  const unsigned min_grid = static_cast<unsigned>((units + 255) / 256);
  if (grid < min_grid) grid = min_grid;
  column_absmax_kernel<<<grid, 256, 0, cs>>>(static_cast<const uint16_t*>(A), rows, K, lda,
                                             reinterpret_cast<uint32_t*>(absmax));
  return launch_status();
}

svdq_status svdq_smoothing(int N, int K, const float* x_absmax, const void* W, float* smooth_inv,
                           svdq_stream_t stream) {
  if (N < 1 || K < 8 || K % 8 || !x_absmax || !W || !smooth_inv) return SVDQ_ERR_INVALID_ARG;
  if (svdq_status st = svdq_column_absmax(N, K, W, K, smooth_inv, stream); st != SVDQ_OK) return st;
  smoothing_kernel<<<(K + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(x_absmax, smooth_inv, K);
  return launch_status();
}

svdq_status svdq_lowrank_factors(int N, int K, int r, const double* U, int ldu, const double* S,
                                 const double* Vh, int ldvh, void* L1, void* L2, svdq_stream_t stream) {
  if (N < 1 || K < 1 || r < 1 || r > N || r > K || ldu < r || ldvh < K) return SVDQ_ERR_INVALID_ARG;
  if (!U || !S || !Vh || !L1 || !L2) return SVDQ_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(U) & 7u) || (reinterpret_cast<uintptr_t>(S) & 7u) ||
      (reinterpret_cast<uintptr_t>(Vh) & 7u) || (reinterpret_cast<uintptr_t>(L1) & 1u) ||
      (reinterpret_cast<uintptr_t>(L2) & 1u))
    return SVDQ_ERR_ALIGNMENT;
  DeviceInfo* d = nullptr;
  if (svdq_status st = device_setup(&d); st != SVDQ_OK) return st;
  const size_t total = static_cast<size_t>(K) * r + static_cast<size_t>(r) * N;
  lowrank_factors_kernel<<<grid_for(total, 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      U, ldu, S, Vh, ldvh, static_cast<uint16_t*>(L1), static_cast<uint16_t*>(L2), N, K, r);
  return launch_status();
}

svdq_status svdq_residual(int N, int K, int r, const void* W, const float* smooth_inv, const void* L1,
                          const void* L2, void* R, svdq_stream_t stream) {
  if (N < 1 || K < 1 || r < 0 || r > 4096 || !W || !smooth_inv || !R) return SVDQ_ERR_INVALID_ARG;
  if ((r > 0) != (L1 != nullptr) || (r > 0) != (L2 != nullptr)) return SVDQ_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(W) & 1u) || (reinterpret_cast<uintptr_t>(R) & 1u) ||
      (reinterpret_cast<uintptr_t>(smooth_inv) & 3u) || (reinterpret_cast<uintptr_t>(L1) & 1u) ||
      (reinterpret_cast<uintptr_t>(L2) & 1u))
    return SVDQ_ERR_ALIGNMENT;
  DeviceInfo* d = nullptr;
  if (svdq_status st = device_setup(&d); st != SVDQ_OK) return st;
  const dim3 grid((K + kResTile - 1) / kResTile, (N + kResTile - 1) / kResTile);
  residual_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint16_t*>(W), smooth_inv, static_cast<const uint16_t*>(L1),
      static_cast<const uint16_t*>(L2), static_cast<uint16_t*>(R), N, K, r);
  return launch_status();
}

svdq_status awq_quantize_weight(int N, int K, const void* W, void* qweight, void* sz,
                                svdq_stream_t stream) {
  if (N < 1 || K < 64 || K % 64 || !W || !qweight || !sz) return SVDQ_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(W) & 1u) || !aligned16(qweight) || !aligned16(sz))
    return SVDQ_ERR_ALIGNMENT;
  DeviceInfo* d = nullptr;
  if (svdq_status st = device_setup(&d); st != SVDQ_OK) return st;
  const size_t blocks = static_cast<size_t>((N + 15) / 16) * (K / 64);
  if (blocks > 0x7FFFFFFFull) return SVDQ_ERR_UNSUPPORTED;
  awq_quantize_kernel<<<static_cast<unsigned>(blocks), 128, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint16_t*>(W), N, K, static_cast<uint32_t*>(qweight), static_cast<uint32_t*>(sz));
  return launch_status();
}

svdq_status svdq_check_device_status(svdq_stream_t stream) {
  DeviceInfo* d = nullptr;
  if (svdq_status st = device_setup(&d); st != SVDQ_OK) return st;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    (void)cudaGetLastError();
    return SVDQ_ERR_CUDA;
  }
  uint32_t v = 0;
  if (cudaMemcpyFromSymbol(&v, g_svdq_status, sizeof(v)) != cudaSuccess) return SVDQ_ERR_CUDA;
  if (v != 0) {
    const uint32_t zero = 0;
    if (cudaMemcpyToSymbol(g_svdq_status, &zero, sizeof(zero)) != cudaSuccess)
      return SVDQ_ERR_CUDA;
  }
  return (v & kStatusTimeout) ? SVDQ_ERR_TIMEOUT : SVDQ_OK;
}

svdq_status svdq_debug_wait_timeout(int limit_us, svdq_stream_t stream) {
  if (limit_us < 1 || limit_us > 1000000) return SVDQ_ERR_INVALID_ARG;
  DeviceInfo* d = nullptr;
  if (svdq_status st = device_setup(&d); st != SVDQ_OK) return st;
  debug_wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      d->status, static_cast<uint64_t>(limit_us) * 1000ull);
  return launch_status();
}

}  // extern "C"

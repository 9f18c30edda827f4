// Host side of the tcgen05 GEMM engine: TMA descriptor encoding, tile-width
// choice and dispatch to the kernel instantiations.
#include <mutex>

#include "gemm2.cuh"
#include "kernels.h"

namespace asr {

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

constexpr int kSlotRows[kGemmSlots] = {256, 128, 240, 64, 160, 120};

template <int BN>
constexpr int stages_for() {
  return BN >= 192 ? 4 : (BN > 128 ? 5 : (BN == 128 ? 6 : 8));
}

template <int BN, bool G, int EPI, int KIND>
cudaError_t run(const CUtensorMap* a, const CUtensorMap& b, const CUtensorMap& o, const GemmParams& p, int grid, cudaStream_t st) {
  using S = GemmShape<BN, stages_for<BN>(), G>;
  void (*k)(CUtensorMap, CUtensorMap, CUtensorMap, GemmParams);
  if constexpr (KIND == KIND_F16)
    k = gemm_f16_tc_kernel<BN, S::STAGES, G, EPI>;
  else
    k = gemm_bf16_tc_kernel<BN, S::STAGES, G, EPI>;
  cudaError_t err = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM_BYTES);
  if (err != cudaSuccess) return err;
  return launch_pdl(k, dim3(grid), dim3(S::THREADS), S::SMEM_BYTES, st, a ? *a : b, b, o, p);
}

template <int BN, int EPI>
cudaError_t run_tf32(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& o, const GemmParams& p, int grid,
                     cudaStream_t st) {
  using S = GemmShape<BN, stages_for<BN>(), false, KIND_TF32>;
  auto k = gemm_tf32_tc_kernel<BN, S::STAGES, EPI>;
  cudaError_t err = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM_BYTES);
  if (err != cudaSuccess) return err;
  return launch_pdl(k, dim3(grid), dim3(S::THREADS), S::SMEM_BYTES, st, a, b, o, p);
}

// tf32 epilogues: every output is fp32.
template <int BN>
cudaError_t run_tf32_epi(int epi, const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& o, const GemmParams& p,
                         int grid, cudaStream_t st) {
  switch (epi) {
    case EPI_OUT_F32: return run_tf32<BN, EPI_OUT_F32>(a, b, o, p, grid, st);
    case EPI_OUT_F32 | EPI_GELU: return run_tf32<BN, EPI_OUT_F32 | EPI_GELU>(a, b, o, p, grid, st);
    case EPI_RESID: return run_tf32<BN, EPI_RESID>(a, b, o, p, grid, st);
    case EPI_OUT_F32 | EPI_PE: return run_tf32<BN, EPI_OUT_F32 | EPI_PE>(a, b, o, p, grid, st);
    case EPI_OUT_F32 | EPI_SWIGLU: return run_tf32<BN, EPI_OUT_F32 | EPI_SWIGLU>(a, b, o, p, grid, st);
    case EPI_GELU | EPI_OUT_F32 | EPI_PE: return run_tf32<BN, EPI_GELU | EPI_OUT_F32 | EPI_PE>(a, b, o, p, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

template <int BN, int KIND>
cudaError_t run_tma(int epi, const CUtensorMap* a, const CUtensorMap& b, const CUtensorMap& o, const GemmParams& p, int grid,
                    cudaStream_t st) {
  switch (epi) {
    case 0: return run<BN, false, 0, KIND>(a, b, o, p, grid, st);
    case EPI_GELU: return run<BN, false, EPI_GELU, KIND>(a, b, o, p, grid, st);
    case EPI_OUT_F32: return run<BN, false, EPI_OUT_F32, KIND>(a, b, o, p, grid, st);
    case EPI_RESID: return run<BN, false, EPI_RESID, KIND>(a, b, o, p, grid, st);
    case EPI_OUT_F32 | EPI_PE: return run<BN, false, EPI_OUT_F32 | EPI_PE, KIND>(a, b, o, p, grid, st);
    case EPI_SWIGLU: return run<BN, false, EPI_SWIGLU, KIND>(a, b, o, p, grid, st);
    case EPI_GELU | EPI_OUT_F32 | EPI_PE: return run<BN, false, EPI_GELU | EPI_OUT_F32 | EPI_PE, KIND>(a, b, o, p, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

// 240-wide tiles only serve the convolutions (N = 480).
template <int KIND>
cudaError_t run_tma240(int epi, const CUtensorMap* a, const CUtensorMap& b, const CUtensorMap& o, const GemmParams& p, int grid,
                       cudaStream_t st) {
  switch (epi) {
    case EPI_GELU: return run<240, false, EPI_GELU, KIND>(a, b, o, p, grid, st);
    case EPI_GELU | EPI_OUT_F32 | EPI_PE: return run<240, false, EPI_GELU | EPI_OUT_F32 | EPI_PE, KIND>(a, b, o, p, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

template <int BN, int KIND>
cudaError_t run_gather(int epi, const CUtensorMap& b, const CUtensorMap& o, const GemmParams& p, int grid, cudaStream_t st) {
  switch (epi) {
    case EPI_GELU: return run<BN, true, EPI_GELU, KIND>(nullptr, b, o, p, grid, st);
    case EPI_GELU | EPI_OUT_F32 | EPI_PE: return run<BN, true, EPI_GELU | EPI_OUT_F32 | EPI_PE, KIND>(nullptr, b, o, p, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

// KP = 2: stages of two k-blocks (3-D maps), three of them in the same
// shared memory as six single-k-block stages.
template <int BN, int EPI, int KIND, int KP = 1>
cudaError_t run2(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& o, const GemmParams& p, int grid, cudaStream_t st) {
  using S = Gemm2Shape<BN, KP == 2 ? 3 : 6, gemm2_epi_warps<EPI>(), gemm2_nbuf<BN>(), KP>;
  void (*k)(CUtensorMap, CUtensorMap, CUtensorMap, GemmParams);
  if constexpr (KIND == KIND_F16)
    k = gemm_f16_tc2_kernel<BN, S::STAGES, EPI, KP>;
  else
    k = gemm_bf16_tc2_kernel<BN, S::STAGES, EPI, KP>;
  cudaError_t err = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM_BYTES);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(S::THREADS, 1, 1);
  cfg.dynamicSmemBytes = S::SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, k, a, b, o, p);
}

template <int BN, int KIND>
cudaError_t run2_epi(int epi, const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& o, const GemmParams& p, int grid,
                     cudaStream_t st) {
  switch (epi) {
    case 0: return run2<BN, 0, KIND>(a, b, o, p, grid, st);
    case EPI_GELU: return run2<BN, EPI_GELU, KIND>(a, b, o, p, grid, st);
    case EPI_OUT_F32: return run2<BN, EPI_OUT_F32, KIND>(a, b, o, p, grid, st);
    case EPI_RESID: return run2<BN, EPI_RESID, KIND>(a, b, o, p, grid, st);
    case EPI_OUT_F32 | EPI_PE: return run2<BN, EPI_OUT_F32 | EPI_PE, KIND>(a, b, o, p, grid, st);
    case EPI_SWIGLU: return run2<BN, EPI_SWIGLU, KIND>(a, b, o, p, grid, st);
    case EPI_GELU | EPI_OUT_F32 | EPI_PE: return run2<BN, EPI_GELU | EPI_OUT_F32 | EPI_PE, KIND>(a, b, o, p, grid, st);
    default: return cudaErrorInvalidValue;
  }
}
// 256-wide pair tiles with two-k-block stages (plain A, K % 128 == 0).
template <int KIND>
cudaError_t run2_kp2(int epi, const CUtensorMap& a3, const CUtensorMap& b3, const CUtensorMap& o, const GemmParams& p,
                     int grid, cudaStream_t st) {
  switch (epi) {
    case 0: return run2<256, 0, KIND, 2>(a3, b3, o, p, grid, st);
    case EPI_GELU: return run2<256, EPI_GELU, KIND, 2>(a3, b3, o, p, grid, st);
    case EPI_OUT_F32: return run2<256, EPI_OUT_F32, KIND, 2>(a3, b3, o, p, grid, st);
    case EPI_RESID: return run2<256, EPI_RESID, KIND, 2>(a3, b3, o, p, grid, st);
    case EPI_OUT_F32 | EPI_PE: return run2<256, EPI_OUT_F32 | EPI_PE, KIND, 2>(a3, b3, o, p, grid, st);
    case EPI_SWIGLU: return run2<256, EPI_SWIGLU, KIND, 2>(a3, b3, o, p, grid, st);
    default: return cudaErrorInvalidValue;
  }
}
template <int KIND>
cudaError_t run2_kp2_ln(const CUtensorMap& a3, const CUtensorMap& b3, const GemmParams& p, int grid, cudaStream_t st) {
  return run2<256, EPI_RESID | EPI_LN, KIND, 2>(a3, b3, b3, p, grid, st);
}

template <int KIND>
cudaError_t run2_240(int epi, const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& o, const GemmParams& p, int grid,
                     cudaStream_t st) {
  switch (epi) {
    case EPI_GELU: return run2<240, EPI_GELU, KIND>(a, b, o, p, grid, st);
    case EPI_GELU | EPI_OUT_F32 | EPI_PE: return run2<240, EPI_GELU | EPI_OUT_F32 | EPI_PE, KIND>(a, b, o, p, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

// CTA pairs that can be resident at once: 148 SMs do not always pair up
// into 74 clusters of two, and stream-K needs every pair of its grid
// resident (an owner waits for the next pair's first piece).  Queried once
// per device for the largest pair configuration (one CTA per SM).
// Stream-K only from 40 k-blocks: in the 16 x 30 s forward it takes fc2
// (80 k-blocks) from 2.45 to 2.39 ms per step, and at 20 it would also take
// the out-projection, which it slows (1.00 to 1.10 ms).
constexpr int kStreamKMinKBlocks = 40;

int resident_pairs(int num_sms) {
  static std::mutex mu;
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(mu);
  if (dev >= 0 && dev < 64 && cache[dev] > 0) return cache[dev];
  using S = Gemm2Shape<256, 6, gemm2_epi_warps<EPI_RESID>(), gemm2_nbuf<256>()>;
  auto k = gemm_bf16_tc2_kernel<256, 6, EPI_RESID>;
  int n = 0;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM_BYTES) == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(num_sms, 1, 1);
    cfg.blockDim = dim3(S::THREADS, 1, 1);
    cfg.dynamicSmemBytes = S::SMEM_BYTES;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, reinterpret_cast<const void*>(k), &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();
  if (n <= 0 || n > num_sms / 2) n = num_sms / 2;
  if (dev >= 0 && dev < 64) cache[dev] = n;
  return n;
}

}  // namespace

int gemm_bn_slot(int bn) {
  for (int i = 0; i < kGemmSlots; ++i)
    if (kSlotRows[i] == bn) return i;
  return -1;
}

bool make_tmap_bf16(CUtensorMap* map, const void* ptr, unsigned long long rows, unsigned long long cols,
                    unsigned long long row_stride_elems, unsigned int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || !ptr || (reinterpret_cast<uintptr_t>(ptr) & 15) || (row_stride_elems * 2) % 16 || rows == 0 ||
      cols == 0 || box_rows == 0 || box_rows > 256)
    return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_stride_elems * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_convbox(CUtensorMap* map, const void* ptr, int C, int F_in, int T_in, int n_img, int F_out, int sf,
                       int TR, int st, int kind) {
  EncodeTiledFn fn = encode_fn();
  const cuuint64_t esz = kind == KIND_TF32 ? 4 : 2;
  if (!fn || !ptr || (reinterpret_cast<uintptr_t>(ptr) & 15) || (C * esz) % 16 || F_out * sf > 256 || TR * st > 256 ||
      F_out * TR != 128 || sf < 1 || sf > 8 || st < 1 || st > 8)
    return false;
  cuuint64_t dims[4] = {(cuuint64_t)C, (cuuint64_t)F_in, (cuuint64_t)T_in, (cuuint64_t)n_img};
  cuuint64_t strides[3] = {(cuuint64_t)C * esz, (cuuint64_t)F_in * C * esz, (cuuint64_t)T_in * F_in * C * esz};
  cuuint32_t box[4] = {(cuuint32_t)kind_row_elems(kind), (cuuint32_t)(F_out * sf), (cuuint32_t)(TR * st), 1};
  cuuint32_t es[4] = {1, (cuuint32_t)sf, (cuuint32_t)st, 1};
  return fn(map, kind == KIND_TF32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
            const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_out(CUtensorMap* map, const void* ptr, unsigned long long rows, unsigned long long cols,
                   unsigned long long row_stride_elems, bool f32) {
  EncodeTiledFn fn = encode_fn();
  const unsigned long long es = f32 ? 4 : 2;
  if (!fn || !ptr || (reinterpret_cast<uintptr_t>(ptr) & 15) || (row_stride_elems * es) % 16 || rows == 0 || cols == 0)
    return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_stride_elems * es};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr),
            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_convphase(CUtensorMap* map, const void* ptr, int C, int F_h, int T_h, int n_planes, int F_out, int TR,
                         int kind) {
  EncodeTiledFn fn = encode_fn();
  const cuuint64_t esz = kind == KIND_TF32 ? 4 : 2;
  if (!fn || !ptr || (reinterpret_cast<uintptr_t>(ptr) & 15) || (C * esz) % 16 || F_out > 256 || TR > 256 ||
      F_out * TR != 128)
    return false;
  cuuint64_t dims[4] = {(cuuint64_t)C, (cuuint64_t)F_h, (cuuint64_t)T_h, (cuuint64_t)n_planes};
  cuuint64_t strides[3] = {(cuuint64_t)C * esz, (cuuint64_t)F_h * C * esz, (cuuint64_t)T_h * F_h * C * esz};
  cuuint32_t box[4] = {(cuuint32_t)kind_row_elems(kind), (cuuint32_t)F_out, (cuuint32_t)TR, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(map, kind == KIND_TF32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
            const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_f32(CUtensorMap* map, const void* ptr, unsigned long long rows, unsigned long long cols,
                   unsigned long long row_stride_elems, unsigned int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || !ptr || (reinterpret_cast<uintptr_t>(ptr) & 15) || (row_stride_elems * 4) % 16 || rows == 0 ||
      cols == 0 || box_rows == 0 || box_rows > 256)
    return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_stride_elems * 4};
  cuuint32_t box[2] = {32, box_rows};  // one 128-byte swizzled row of 32 fp32
  cuuint32_t es[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_act(int kind, CUtensorMap* map, const void* ptr, unsigned long long rows, unsigned long long cols,
                   unsigned long long row_stride_elems, unsigned int box_rows) {
  return kind == KIND_TF32 ? make_tmap_f32(map, ptr, rows, cols, row_stride_elems, box_rows)
                           : make_tmap_bf16(map, ptr, rows, cols, row_stride_elems, box_rows);
}

bool make_tmap_3d16(CUtensorMap* map, const void* ptr, unsigned long long rows, unsigned long long cols,
                    unsigned long long row_stride_elems, unsigned int box_rows, int kind) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || !ptr || kind == KIND_TF32 || (reinterpret_cast<uintptr_t>(ptr) & 15) || (row_stride_elems * 2) % 16 ||
      rows == 0 || cols % 128 || box_rows == 0 || box_rows > 256)
    return false;
  cuuint64_t dims[3] = {64, rows, cols / 64};
  cuuint64_t strides[2] = {row_stride_elems * 2, 128};
  cuuint32_t box[3] = {64, box_rows, 2};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(map, kind == KIND_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
            const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_weight_maps(GemmB& w) {
  w.has3 = w.kind != KIND_TF32 && w.K % 128 == 0 && make_tmap_3d16(&w.map3, w.ptr, w.N, w.K, w.K, 128, w.kind);
  for (int i = 0; i < kGemmSlots; ++i)
    if (!make_tmap_act(w.kind, &w.map[i], w.ptr, w.N, w.K, w.K, kSlotRows[i])) return false;
  return true;
}

int gemm_pick_bn_tf32(int M, int N, int num_sms) {
  // one-SM tiles of 256, 128 or 64 columns: fewest waves, then the wider tile
  if (N <= 64) return 64;
  int best = 256;
  long long best_cost = -1;
  for (int bn : {256, 128}) {
    const long long tiles = (long long)((M + 127) / 128) * ((N + bn - 1) / bn);
    const long long cost = (tiles + num_sms - 1) / num_sms * (bn + 32);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = bn;
    }
  }
  return best;
}

int gemm_pick_bn(int M, int N, int num_sms, bool gather) {
  if (gather && N % 240 == 0 && N % 256 != 0 && N <= 480) return 240;
  if (N <= 64) return 64;
  // Estimated cost = waves x per-tile time.  A CTA pair computes a 256 x bn
  // tile in about the time one SM needs for 128 x bn (the same per-SM MMA
  // rate), slightly faster on long K thanks to its deeper pipeline.
  long long best_cost = -1;
  int best = 256;
  auto consider = [&](int bn, bool pair) {
    const long long mb = pair ? (M + 255) / 256 : (M + 127) / 128;
    const long long units = pair ? num_sms / 2 : num_sms;
    const long long tiles = mb * ((N + bn - 1) / bn);
    const long long waves = (tiles + units - 1) / units;
    const long long cost = waves * (bn + 32) * (pair ? 93 : 100);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = pair ? -bn : bn;
    }
  };
  consider(256, false);
  if (!gather && N % 160 == 0) consider(160, false);
  consider(128, false);
  if (!gather && M > 128) {
    consider(256, true);
    consider(128, true);
  }
  return best;
}

int gemm_pick_bn_conv(int n_sub, int N, int num_sms) {
  // Convolution N is 480 (two 240-wide tiles) or d_model; pairs take two
  // 128-row sub-tiles at once.
  const int bn = (N % 240 == 0 && N % 256 != 0 && N <= 480) ? 240 : (N <= 64 ? 64 : (N % 256 == 0 ? 256 : 128));
  if (bn == 64) return 64;
  const long long nb = (N + bn - 1) / bn;
  const long long w1 = ((long long)n_sub * nb + num_sms - 1) / num_sms;
  const long long w2 = (((long long)n_sub + 1) / 2 * nb + num_sms / 2 - 1) / (num_sms / 2);
  return (w2 * 93 <= w1 * 100) ? -bn : bn;
}

template <int KIND>
cudaError_t launch16(const CUtensorMap* a_map, const GemmB& w, GemmParams p, int epi, int bn, int num_sms,
                     cudaStream_t st, const CUtensorMap* out_map, const CUtensorMap* a_map3) {
  p.out_tma = (out_map != nullptr && !(epi & (EPI_PE | EPI_SWIGLU))) ? 1 : 0;
  if (epi & EPI_LN) {
    // Residual + LayerNorm: 256-wide pair tiles with two-k-block stages,
    // whole tiles in n-fast order (the epilogue waits on the row block's
    // other n-tiles), N a multiple of 32, and at least as many resident
    // pairs as n-tiles per row block.  Both outputs by plain stores.
    const int n_blocks = (w.N + 255) / 256;
    if (epi != (EPI_RESID | EPI_LN) || !a_map || !a_map3 || !w.has3 || p.conv_box || w.K % 128 || w.N % 32 ||
        p.ldo % 8 || !p.ln_gamma || !p.ln_beta || !p.ln_count || !p.ln_part || !p.ln_h || p.M <= 0 ||
        resident_pairs(num_sms) < n_blocks)
      return cudaErrorInvalidValue;
    p.out_tma = 0;
    p.k_full = 1;
    p.n_fast = 1;
    p.sk = 0;
    p.N = w.N;
    p.K = w.K;
    p.m_blocks = (p.M + 255) / 256;
    p.n_blocks = n_blocks;
    p.k_blocks = p.K / 128;
    p.num_tiles = p.m_blocks * p.n_blocks;
    p.ln_parts = 2 * n_blocks;  // two epilogue warps per lane quarter and n-tile
    const int grid = 2 * std::min(p.num_tiles, resident_pairs(num_sms));
    return run2_kp2_ln<KIND>(*a_map3, w.map3, p, grid, st);
  }
  // Whole four-step k-blocks everywhere when A and B both come by TMA: the
  // steps past K (or past a tap's channels) multiply the zeros that the TMA
  // fills outside the tensors and that pad the conv weights, and issuing
  // them costs less than a test per k-block.  The cp.async gather leaves
  // those bytes unwritten, so it keeps the partial steps.
  p.k_full = a_map != nullptr ? 1 : 0;
  // Tile order: the tiles running at once share the larger operand, so it
  // crosses from DRAM once and is re-read from L2 (and the TMA latency the
  // stage ring has to cover is the L2's, not the DRAM's).  A (M x K) is the
  // larger when M > N; convolutions always re-read their gathered A.
  p.n_fast = (p.conv_box || a_map == nullptr || p.M > w.N) ? 1 : 0;
  if (bn < 0) {
    // CTA-pair kernel: 256 x |bn| tiles, each CTA stages |bn|/2 rows of B.
    const int w2 = -bn;
    const int slot2 = gemm_bn_slot(w2 / 2);
    if (!a_map || slot2 < 0 || p.M <= 0 || (w2 != 256 && w2 != 128 && w2 != 240)) return cudaErrorInvalidValue;
    p.N = w.N;
    p.K = w.K;
    p.m_blocks = p.conv_box ? (p.cb.n_sub + 1) / 2 : (p.M + 255) / 256;
    p.n_blocks = (p.N + w2 - 1) / w2;
    // Two k-blocks per stage (3-D copies) for plain 256-wide tiles when the
    // caller gave the 3-D map of A and K is a whole number of stages.
    const bool kp2 = a_map3 && w.has3 && w2 == 256 && !p.conv_box && p.K % 128 == 0 &&
                     (epi == 0 || epi == EPI_GELU || epi == EPI_OUT_F32 || epi == EPI_RESID ||
                      epi == (EPI_OUT_F32 | EPI_PE) || epi == EPI_SWIGLU);
    p.k_blocks = kp2 ? p.K / 128 : (p.K + 63) / 64;
    p.num_tiles = p.m_blocks * p.n_blocks;
    const int pairs = std::min(p.num_tiles, resident_pairs(num_sms));
    const int grid = 2 * pairs;
    // Stream-K when the caller gave the flags, the epilogue is the residual
    // add, whole tiles would leave a ragged last wave, and K is long enough
    // (>= 40 k-blocks) for a split piece to outlast an epilogue (about 3 us):
    // with short K the extra epilogues of the split tiles cost more than the
    // balanced last wave saves.  (Its units are stages.)
    p.sk = (p.sk_flags && epi == EPI_RESID && !p.conv_box && (p.K + 63) / 64 >= kStreamKMinKBlocks &&
            p.num_tiles > pairs && p.num_tiles % pairs != 0)
               ? 1
               : 0;
    if (kp2)
      return run2_kp2<KIND>(epi, *a_map3, w.map3, p.out_tma ? *out_map : w.map3, p, grid, st);
    if (w2 == 240) return run2_240<KIND>(epi, *a_map, w.map[slot2], p.out_tma ? *out_map : w.map[slot2], p, grid, st);
    const CUtensorMap& o2 = p.out_tma ? *out_map : w.map[slot2];
    return w2 == 256 ? run2_epi<256, KIND>(epi, *a_map, w.map[slot2], o2, p, grid, st)
                     : run2_epi<128, KIND>(epi, *a_map, w.map[slot2], o2, p, grid, st);
  }
  const int slot = gemm_bn_slot(bn);
  if (slot < 0 || p.M <= 0) return cudaErrorInvalidValue;
  p.sk = 0;  // the one-SM kernel runs whole tiles
  p.N = w.N;
  p.K = w.K;
  p.m_blocks = p.conv_box ? p.cb.n_sub : (p.M + 127) / 128;
  p.n_blocks = (p.N + bn - 1) / bn;
  p.k_blocks = (p.K + 63) / 64;
  p.num_tiles = p.m_blocks * p.n_blocks;
  const int grid = p.num_tiles < num_sms ? p.num_tiles : num_sms;
  const CUtensorMap& b = w.map[slot];
  const CUtensorMap& o = p.out_tma ? *out_map : b;
  const bool gather = (a_map == nullptr);
  if (gather) {
    switch (bn) {
      case 256: return run_gather<256, KIND>(epi, b, o, p, grid, st);
      case 240: return run_gather<240, KIND>(epi, b, o, p, grid, st);
      case 128: return run_gather<128, KIND>(epi, b, o, p, grid, st);
      case 64: return run_gather<64, KIND>(epi, b, o, p, grid, st);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (bn) {
    case 256: return run_tma<256, KIND>(epi, a_map, b, o, p, grid, st);
    case 240: return run_tma240<KIND>(epi, a_map, b, o, p, grid, st);
    case 160: return run_tma<160, KIND>(epi, a_map, b, o, p, grid, st);
    case 128: return run_tma<128, KIND>(epi, a_map, b, o, p, grid, st);
    case 64: return run_tma<64, KIND>(epi, a_map, b, o, p, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

bool gemm_ln_supported(const GemmB& w, int num_sms) {
  return w.kind != KIND_TF32 && w.has3 && w.K % 128 == 0 && w.N % 32 == 0 && w.N > 0 &&
         resident_pairs(num_sms) >= (w.N + 255) / 256;
}

cudaError_t launch_gemm(const CUtensorMap* a_map, const GemmB& w, GemmParams p, int epi, int bn, int num_sms,
                        cudaStream_t st, const CUtensorMap* out_map, const CUtensorMap* a_map3) {
  if (w.kind == KIND_BF16) return launch16<KIND_BF16>(a_map, w, p, epi, bn, num_sms, st, out_map, a_map3);
  if (w.kind == KIND_F16) return launch16<KIND_F16>(a_map, w, p, epi, bn, num_sms, st, out_map, a_map3);
  // fp32 operands: one-SM tiles only (the CTA-pair kernel takes 16-bit
  // operands), no gather mode, no LayerNorm epilogue
  if (epi & EPI_LN) return cudaErrorInvalidValue;
  p.out_tma = (out_map != nullptr && !(epi & (EPI_PE | EPI_SWIGLU))) ? 1 : 0;
  p.n_fast = (p.conv_box || p.M > w.N) ? 1 : 0;
  p.k_full = 1;  // A and B by TMA (see launch16)
  const int slot = gemm_bn_slot(bn);
  if (bn < 0 || slot < 0 || p.M <= 0 || !a_map) return cudaErrorInvalidValue;
  p.sk = 0;
  p.N = w.N;
  p.K = w.K;
  p.m_blocks = p.conv_box ? p.cb.n_sub : (p.M + 127) / 128;
  p.n_blocks = (p.N + bn - 1) / bn;
  p.k_blocks = (p.K + 31) / 32;
  p.num_tiles = p.m_blocks * p.n_blocks;
  const int grid = p.num_tiles < num_sms ? p.num_tiles : num_sms;
  const CUtensorMap& b = w.map[slot];
  const CUtensorMap& o = p.out_tma ? *out_map : b;
  switch (bn) {
    case 256: return run_tf32_epi<256>(epi, *a_map, b, o, p, grid, st);
    case 128: return run_tf32_epi<128>(epi, *a_map, b, o, p, grid, st);
    case 64: return run_tf32_epi<64>(epi, *a_map, b, o, p, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace asr

// Per-layer kernels other than the GEMMs and the attention: LayerNorm and
// small helpers (window offsets, variable-length descriptors, conversions,
// the device GELU, the bounded-wait probe).  Attention runs on the tcgen05
// kernels of attn_tc.cu (segments of at most 128 tokens) and attn_fa.cu
// (longer segments).
#include "kernels.h"

namespace asr {

// ------------------------------------------------------------ LayerNorm
// One warp per row, V float4 per lane (D = 128 V), the whole row held in
// registers: every load of the row is issued at once (one memory round trip
// per row), then the statistics, then the normalised row is written from the
// registers.  The statistics take one pass in shifted form: with
// K = x[row][0],
//   mean = K + S1 / D,  var = S2 / D - (S1 / D)^2,
//   S1 = sum (x - K),   S2 = sum (x - K)^2,
// which keeps the cancellation at the scale of the row's spread (|x - K|
// is a few standard deviations), not of its mean.
// The grid is one wave of resident blocks (four warps each); a warp takes
// rows gw, gw + W, ... and copies its next row into its shared-memory
// buffer (cp.async) while it normalises the current one, so rows past the
// first wave do not pay a second memory round trip.  Gamma and beta are
// staged in shared memory once per block, before the dependency wait (they
// are weights, not the previous kernel's output).

template <int V, int OUT>
__global__ void __launch_bounds__(128) layer_norm_kernel(const float* __restrict__ x, const float* __restrict__ g,
                                                         const float* __restrict__ b, long long M, float eps,
                                                         void* __restrict__ y) {
  constexpr int D = V * 128;
  extern __shared__ float4 ln_smem[];
  float4* g4 = ln_smem;                 // [D / 4]
  float4* b4 = ln_smem + D / 4;         // [D / 4]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float4* buf = ln_smem + 2 * (D / 4) + warp * (D / 4);  // this warp's row buffer
  for (int i = threadIdx.x; i < D / 4; i += 128) {
    g4[i] = __ldg(reinterpret_cast<const float4*>(g) + i);
    b4[i] = __ldg(reinterpret_cast<const float4*>(b) + i);
  }
  __syncthreads();
  pdl_wait();
  pdl_trigger();
  const long long W = gridDim.x * 4LL;
  long long row = blockIdx.x * 4LL + warp;
  auto fetch = [&](long long r) {
    const float4* xr = reinterpret_cast<const float4*>(x + r * D);
#pragma unroll
    for (int i = 0; i < V; ++i) cp_async_16_zfill(buf + lane + 32 * i, xr + lane + 32 * i, true);
    cp_async_commit();
  };
  if (row < M) fetch(row);
  for (; row < M; row += W) {
    // each lane reads back exactly the 16-byte chunks it copied
    cp_async_wait<0>();
    float4 v[V];
#pragma unroll
    for (int i = 0; i < V; ++i) v[i] = buf[lane + 32 * i];
    if (row + W < M) fetch(row + W);
    const float K = __shfl_sync(0xffffffffu, v[0].x, 0);  // x[row][0]
    float s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int i = 0; i < V; ++i) {
      const float a = v[i].x - K, bb = v[i].y - K, c = v[i].z - K, d = v[i].w - K;
      s1 += (a + bb) + (c + d);
      s2 += (a * a + bb * bb) + (c * c + d * d);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      s1 += __shfl_xor_sync(0xffffffffu, s1, o);
      s2 += __shfl_xor_sync(0xffffffffu, s2, o);
    }
    const float m1 = s1 * (1.0f / D);
    const float mean = K + m1;
    const float var = fmaxf(s2 * (1.0f / D) - m1 * m1, 0.0f);
    const float rstd = rsqrtf(var + eps);
#pragma unroll
    for (int i = 0; i < V; ++i) {
      const int c4 = lane + 32 * i;
      const float4 gg = g4[c4], bv = b4[c4];
      const float o0 = (v[i].x - mean) * rstd * gg.x + bv.x;
      const float o1 = (v[i].y - mean) * rstd * gg.y + bv.y;
      const float o2 = (v[i].z - mean) * rstd * gg.z + bv.z;
      const float o3 = (v[i].w - mean) * rstd * gg.w + bv.w;
      if (OUT == KIND_TF32) {
        reinterpret_cast<float4*>(reinterpret_cast<float*>(y) + row * D)[c4] = make_float4(o0, o1, o2, o3);
      } else {
        const uint2 w2 = make_uint2(pack2_16<OUT>(o0, o1), pack2_16<OUT>(o2, o3));
        reinterpret_cast<uint2*>(reinterpret_cast<bf16*>(y) + row * D)[c4] = w2;
      }
    }
  }
}

// Single-wave form, for row counts that fit the SMs at once (at d = 1280
// up to 44 rows per SM: four blocks of 11 warps, 220 KB of row buffers):
// one row per warp, copied into the warp's shared-memory buffer (cp.async)
// and read from there twice, statistics then output, so a thread holds none
// of the row across the two passes; every row's load is in flight at once
// instead of the two rounds of the register form.  Same arithmetic, in the
// same order, as layer_norm_kernel.
constexpr int kLnWaveWarps = 11;
template <int V, int OUT>
__global__ void __launch_bounds__(32 * kLnWaveWarps, 4) layer_norm_wave_kernel(const float* __restrict__ x, const float* __restrict__ g,
                                                              const float* __restrict__ b, long long M, float eps,
                                                              void* __restrict__ y) {
  constexpr int D = V * 128;
  extern __shared__ float4 ln_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float4* buf = ln_smem + warp * (D / 4);
  const long long row = (long long)blockIdx.x * kLnWaveWarps + warp;
  pdl_wait();
  pdl_trigger();
  if (row >= M) return;
  const float4* xr = reinterpret_cast<const float4*>(x + row * D);
#pragma unroll
  for (int i = 0; i < V; ++i) cp_async_16_zfill(buf + lane + 32 * i, xr + lane + 32 * i, true);
  cp_async_commit();
  cp_async_wait<0>();
  // each lane reads back exactly the 16-byte chunks it copied
  const float K = __shfl_sync(0xffffffffu, buf[lane].x, 0);  // x[row][0]
  float s1 = 0.f, s2 = 0.f;
#pragma unroll 2
  for (int i = 0; i < V; ++i) {
    const float4 v = buf[lane + 32 * i];
    const float a = v.x - K, bb = v.y - K, c = v.z - K, d = v.w - K;
    s1 += (a + bb) + (c + d);
    s2 += (a * a + bb * bb) + (c * c + d * d);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s1 += __shfl_xor_sync(0xffffffffu, s1, o);
    s2 += __shfl_xor_sync(0xffffffffu, s2, o);
  }
  const float m1 = s1 * (1.0f / D);
  const float mean = K + m1;
  const float var = fmaxf(s2 * (1.0f / D) - m1 * m1, 0.0f);
  const float rstd = rsqrtf(var + eps);
#pragma unroll 2
  for (int i = 0; i < V; ++i) {
    const int c4 = lane + 32 * i;
    const float4 v = buf[c4];
    const float4 gg = __ldg(reinterpret_cast<const float4*>(g) + c4), bv = __ldg(reinterpret_cast<const float4*>(b) + c4);
    const float o0 = (v.x - mean) * rstd * gg.x + bv.x;
    const float o1 = (v.y - mean) * rstd * gg.y + bv.y;
    const float o2 = (v.z - mean) * rstd * gg.z + bv.z;
    const float o3 = (v.w - mean) * rstd * gg.w + bv.w;
    if (OUT == KIND_TF32) {
      reinterpret_cast<float4*>(reinterpret_cast<float*>(y) + row * D)[c4] = make_float4(o0, o1, o2, o3);
    } else {
      const uint2 w2 = make_uint2(pack2_16<OUT>(o0, o1), pack2_16<OUT>(o2, o3));
      reinterpret_cast<uint2*>(reinterpret_cast<bf16*>(y) + row * D)[c4] = w2;
    }
  }
}

template <int V, int OUT>
static cudaError_t ln_launch(const float* x, const float* g, const float* b, long long M, float eps, void* y,
                             cudaStream_t st) {
  {
    // single-wave form when every row fits in flight at once
    constexpr int WSMEM = kLnWaveWarps * V * 128 * 4;  // one row buffer per warp
    static int wave_per_sm[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (wave_per_sm[dev] == 0) {
      cudaError_t e =
          cudaFuncSetAttribute(layer_norm_wave_kernel<V, OUT>, cudaFuncAttributeMaxDynamicSharedMemorySize, WSMEM);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(layer_norm_wave_kernel<V, OUT>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
      int n = 0;
      if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, layer_norm_wave_kernel<V, OUT>, 32 * kLnWaveWarps, WSMEM);
      if (e != cudaSuccess) return e;
      wave_per_sm[dev] = n > 0 ? n : -1;
    }
    int sms = 0;
    cudaError_t e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const long long need = (M + kLnWaveWarps - 1) / kLnWaveWarps;
    if (wave_per_sm[dev] > 0 && need <= (long long)sms * wave_per_sm[dev])
      return launch_pdl(layer_norm_wave_kernel<V, OUT>, dim3(static_cast<unsigned>(need)), dim3(32 * kLnWaveWarps),
                        WSMEM, st, x, g, b, M, eps, y);
  }
  constexpr int SMEM = (2 + 4) * V * 128 * 4;  // gamma, beta, four row buffers
  static int per_sm[64] = {0};                  // resident blocks per SM, per device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (per_sm[dev] == 0) {
    cudaError_t e = cudaFuncSetAttribute(layer_norm_kernel<V, OUT>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(layer_norm_kernel<V, OUT>, cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared);
    int n = 0;
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, layer_norm_kernel<V, OUT>, 128, SMEM);
    if (e != cudaSuccess) return e;
    per_sm[dev] = n > 0 ? n : 1;
  }
  int sms = 0;
  cudaError_t e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const long long need = (M + 3) / 4;
  const long long wave = (long long)sms * per_sm[dev];
  const unsigned blocks = static_cast<unsigned>(need < wave ? need : wave);
  return launch_pdl(layer_norm_kernel<V, OUT>, dim3(blocks), dim3(128), SMEM, st, x, g, b, M, eps, y);
}

template <int OUT>
static cudaError_t ln_dispatch(int V, const float* x, const float* g, const float* b, long long M, float eps, void* y,
                               cudaStream_t st) {
  switch (V) {
#define ASR_LN_CASE(n) \
  case n: return ln_launch<n, OUT>(x, g, b, M, eps, y, st);
    ASR_LN_CASE(1) ASR_LN_CASE(2) ASR_LN_CASE(3) ASR_LN_CASE(4) ASR_LN_CASE(5) ASR_LN_CASE(6) ASR_LN_CASE(7)
    ASR_LN_CASE(8) ASR_LN_CASE(9) ASR_LN_CASE(10) ASR_LN_CASE(11) ASR_LN_CASE(12) ASR_LN_CASE(13)
    ASR_LN_CASE(14) ASR_LN_CASE(15) ASR_LN_CASE(16)
#undef ASR_LN_CASE
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_layer_norm(const float* x, const float* g, const float* b, long long M, int D, float eps, void* y,
                              int out_kind, cudaStream_t st) {
  if (D % 128 || D > 2048 || M <= 0) return cudaErrorInvalidValue;
  switch (out_kind) {
    case KIND_TF32: return ln_dispatch<KIND_TF32>(D / 128, x, g, b, M, eps, y, st);
    case KIND_F16: return ln_dispatch<KIND_F16>(D / 128, x, g, b, M, eps, y, st);
    default: return ln_dispatch<KIND_BF16>(D / 128, x, g, b, M, eps, y, st);
  }
}

// ------------------------------------------------------------ helpers
__global__ void fill_windows_kernel(int* cu, int batch, int tpc, int window, int nw) {
  pdl_wait();
  pdl_trigger();
  const int total = batch * nw;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i <= total; i += gridDim.x * blockDim.x) {
    if (i == total) {
      cu[i] = batch * tpc;
    } else {
      const int b = i / nw, j = i - b * nw;
      cu[i] = b * tpc + min(j * window, tpc);
    }
  }
}

cudaError_t launch_fill_windows(int* cu, int batch, int tokens_per_clip, int window, int n_win_per_clip,
                                cudaStream_t st) {
  const int total = batch * n_win_per_clip + 1;
  return launch_pdl(fill_windows_kernel, dim3((total + 255) / 256), dim3(256), 0, st, cu, batch, tokens_per_clip, window,
                    n_win_per_clip);
}

__global__ void varlen_fill_kernel(const VarClipBatch vb, int chunk_frames, int window, int t3, MelClip* __restrict__ mc,
                                   ChunkDesc* __restrict__ cd, int* __restrict__ cu, int last, int n_win, int n_tokens) {
  pdl_wait();
  pdl_trigger();
  const VarClip& v = vb.c[blockIdx.x];
  const int clip = vb.first + blockIdx.x;
  if (threadIdx.x == 0) {
    MelClip m;
    m.s_off = v.s_off;
    m.n = v.n;
    m.f_off = v.f_off;
    m.frames = v.frames;
    m.g_off = v.g_off;
    m.left = v.left;
    mc[clip] = m;
  }
  for (int q = threadIdx.x; q < v.chunks; q += blockDim.x) {
    ChunkDesc c;
    c.clip = clip;
    c.frame0 = q * chunk_frames;
    c.nvalid = min(chunk_frames, v.frames - q * chunk_frames);
    c.tok_dst = v.tok_off + q * t3;
    cd[v.chunk_off + q] = c;
  }
  const int w = window ? window : v.tokens;
  for (int j = threadIdx.x; j < v.wins; j += blockDim.x) cu[v.win_off + j] = v.tok_off + j * w;
  if (last && blockIdx.x == gridDim.x - 1 && threadIdx.x == 0) cu[n_win] = n_tokens;
}

cudaError_t launch_varlen_fill(const VarClipBatch& vb, int chunk_frames, int window, int t3, MelClip* mc,
                               ChunkDesc* cd, int* cu, int last, int n_win, int n_tokens, cudaStream_t st) {
  if (vb.count <= 0 || vb.count > kVarClipsPerLaunch) return cudaErrorInvalidValue;
  return launch_pdl(varlen_fill_kernel, dim3(vb.count), dim3(128), 0, st, vb, chunk_frames, window, t3, mc, cd, cu,
                    last, n_win, n_tokens);
}

__global__ void bf16_to_f32_kernel(const uint16_t* __restrict__ in, float* __restrict__ out, long long n, int f16) {
  pdl_wait();
  pdl_trigger();
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
    out[i] = f16 ? __half2float(__ushort_as_half(in[i])) : __bfloat162float(__ushort_as_bfloat16(in[i]));
}

cudaError_t launch_bf16_to_f32(const void* in, float* out, long long n, bool f16, cudaStream_t st) {
  const int blocks = static_cast<int>(std::min<long long>((n + 255) / 256, 148LL * 32));
  return launch_pdl(bf16_to_f32_kernel, dim3(blocks), dim3(256), 0, st, static_cast<const uint16_t*>(in), out, n,
                    f16 ? 1 : 0);
}

__global__ void gelu_kernel(const float* __restrict__ x, float* __restrict__ y, long long n) {
  pdl_wait();
  pdl_trigger();
  // pairs through the packed form used by the GEMM epilogues and the stem; an
  // odd last element through the scalar form
  const long long np = n / 2;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < np; i += (long long)gridDim.x * blockDim.x) {
    const float2 g = gelu_erf2(make_float2(x[2 * i], x[2 * i + 1]));
    y[2 * i] = g.x;
    y[2 * i + 1] = g.y;
  }
  if ((n & 1) && blockIdx.x == 0 && threadIdx.x == 0) y[n - 1] = gelu_erf(x[n - 1]);
}

cudaError_t launch_gelu(const float* x, float* y, long long n, cudaStream_t st) {
  const int blocks = static_cast<int>(std::min<long long>((n + 255) / 256, 148LL * 32));
  return launch_pdl(gelu_kernel, dim3(blocks), dim3(256), 0, st, x, y, n);
}

// A barrier that nothing ever completes, waited on with the same bounded wait
// as the GEMM pipeline: the wait gives up after limit_ns and records a status.
__global__ void wait_probe_kernel(unsigned long long limit_ns, int* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait_bounded(&bar, 0, limit_ns, status, DEV_TIMEOUT_PROBE);
  __syncthreads();
}

cudaError_t launch_wait_probe(unsigned long long limit_ns, int* status, cudaStream_t st) {
  wait_probe_kernel<<<1, 32, 0, st>>>(limit_ns, status);
  return cudaGetLastError();
}

}  // namespace asr

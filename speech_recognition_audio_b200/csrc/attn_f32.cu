// Attention in fp32 on the CUDA cores, for the fp32 (tf32-GEMM) path of
// geometries whose weights are fp32 ("MOSS-Transcribe-preview-2B-GGUF",
// Architecture "Audio encoder": windowed, block-diagonal attention; the
// whisper-style variant attends over whole clips): for each segment
// [cu[j], cu[j+1]) and head h, softmax(Q K^T / 8) V in fp32 arithmetic.
//
// One block of 128 threads per (segment, head, 128-query tile); each thread
// owns one query row (q and its output accumulator in registers).  Keys and
// values come through shared memory in tiles of 32 keys; per tile the
// thread computes its 32 scores, and the online softmax rescales the
// accumulator once per tile when the running maximum grows.
#include "kernels.h"

namespace asr {

namespace {
constexpr int AF_KT = 32;   // keys per tile
}

__global__ void __launch_bounds__(128) attention_f32_kernel(const float* __restrict__ qkv, const int* __restrict__ cu,
                                                            int H, float* __restrict__ out) {
  __shared__ float ks[AF_KT][64];
  __shared__ float vs[AF_KT][64];
  pdl_wait();
  pdl_trigger();
  const int seg = blockIdx.x, h = blockIdx.y;
  const int s0 = cu[seg], L = cu[seg + 1] - s0;
  const int q0 = blockIdx.z * 128;
  if (q0 >= L) return;
  const int tid = threadIdx.x;
  const long long ld = 3LL * H * 64;
  const int qi = q0 + tid;
  const bool live = qi < L;
  float q[64], o[64];
  const float* qrow = qkv + (long long)(s0 + (live ? qi : 0)) * ld + h * 64;
#pragma unroll
  for (int c = 0; c < 64; c += 4) {
    const float4 v = *reinterpret_cast<const float4*>(qrow + c);
    q[c] = v.x * 0.125f; q[c + 1] = v.y * 0.125f; q[c + 2] = v.z * 0.125f; q[c + 3] = v.w * 0.125f;
  }
#pragma unroll
  for (int c = 0; c < 64; ++c) o[c] = 0.f;
  float m = -INFINITY, l = 0.f;
  for (int k0 = 0; k0 < L; k0 += AF_KT) {
    const int kn = min(AF_KT, L - k0);
    __syncthreads();
    for (int i = tid; i < AF_KT * 16; i += 128) {
      const int r = i >> 4, c = (i & 15) * 4;
      float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), vv = kv;
      if (r < kn) {
        const float* base = qkv + (long long)(s0 + k0 + r) * ld;
        kv = *reinterpret_cast<const float4*>(base + (H + h) * 64 + c);
        vv = *reinterpret_cast<const float4*>(base + (2 * H + h) * 64 + c);
      }
      *reinterpret_cast<float4*>(&ks[r][c]) = kv;
      *reinterpret_cast<float4*>(&vs[r][c]) = vv;
    }
    __syncthreads();
    float sc[AF_KT];
    float mt = -INFINITY;
#pragma unroll
    for (int k = 0; k < AF_KT; ++k) {
      float a = 0.f;
#pragma unroll
      for (int c = 0; c < 64; ++c) a = fmaf(q[c], ks[k][c], a);
      sc[k] = k < kn ? a : -INFINITY;
      mt = fmaxf(mt, sc[k]);
    }
    const float mn = fmaxf(m, mt);
    const float corr = expf(m - mn);  // 0 on the first tile (m = -inf)
    l *= corr;
#pragma unroll
    for (int c = 0; c < 64; ++c) o[c] *= corr;
    m = mn;
#pragma unroll
    for (int k = 0; k < AF_KT; ++k) {
      const float pk = expf(sc[k] - m);
      l += pk;
#pragma unroll
      for (int c = 0; c < 64; ++c) o[c] = fmaf(pk, vs[k][c], o[c]);
    }
  }
  if (live) {
    const float inv = 1.0f / l;
    float* orow = out + (long long)(s0 + qi) * (H * 64) + h * 64;
#pragma unroll
    for (int c = 0; c < 64; c += 4)
      *reinterpret_cast<float4*>(orow + c) = make_float4(o[c] * inv, o[c + 1] * inv, o[c + 2] * inv, o[c + 3] * inv);
  }
}

cudaError_t launch_attention_f32(const float* qkv, const int* cu, int n_seg, int max_seg, int H, float* out,
                                 cudaStream_t st) {
  if (n_seg <= 0 || max_seg <= 0 || H <= 0) return cudaErrorInvalidValue;
  dim3 grid(n_seg, H, (max_seg + 127) / 128);
  return launch_pdl(attention_f32_kernel, grid, dim3(128), 0, st, qkv, cu, H, out);
}

}  // namespace asr

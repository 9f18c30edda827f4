// First convolution of the chunked Conv2D stem ("MOSS-Transcribe-preview-2B-
// GGUF", Architecture "Conv front-end": 3 x Conv2D stride 2, 1 -> 480).
// With one input channel its contraction length is 9, so it runs on the CUDA
// cores: each block stages a normalised, zero-padded patch of one chunk's
// log-mel in shared memory, and each thread produces 8 output channels of a
// (time, frequency) position (bias + GELU) as one 16-byte store.  The log-mel normalisation
// (clamp at clip max - 8, then (x + 4) / 4) is applied while staging.
// Output layout: [chunk, T1, F1, C] bf16 (channels innermost), the input
// layout of the implicit-GEMM conv2.
#include "kernels.h"

namespace asr {

namespace {
constexpr int TB = 10;         // output time rows per block
constexpr int MAXM = 128;      // mel-bin capacity
constexpr int THREADS = 256;
}  // namespace

// Block: groups = C/8 channel groups x PL position lanes.  Each thread keeps
// the 9 taps of its 8 channels (and their biases) in registers and walks the
// positions of its lane, so the inner loop reads only the (broadcast) patch
// from shared memory.
__global__ void __launch_bounds__(THREADS)
    conv1_chunked_kernel(const float* __restrict__ mel_raw, const unsigned int* __restrict__ clip_max, int n_mels,
                         int n_frames, int chunk_frames, int chunks_per_clip, const float* __restrict__ w,
                         const float* __restrict__ bias, int C, bf16* __restrict__ out) {
  __shared__ float patch[(2 * TB + 1) * (MAXM + 2)];
  pdl_wait();
  pdl_trigger();
  const int chunk = blockIdx.x;
  const int b = chunk / chunks_per_clip;
  const int q = chunk - b * chunks_per_clip;
  const int T1 = (chunk_frames - 1) / 2 + 1;
  const int F1 = (n_mels - 1) / 2 + 1;
  const int t0 = blockIdx.y * TB;
  const int nt = min(TB, T1 - t0);
  const int PW = n_mels + 2;
  const float mfloor = ordered_to_float(clip_max[b]) - 8.0f;
  const float* src = mel_raw + (long long)b * n_mels * n_frames + (long long)q * chunk_frames;

  // patch row j holds chunk-local time 2*t0 - 1 + j; column c holds mel bin c - 1.
  const int rows = 2 * nt + 1;
  for (int i = threadIdx.x; i < rows * PW; i += blockDim.x) {
    const int j = i / PW, c = i - j * PW;
    const int t = 2 * t0 - 1 + j, m = c - 1;
    float v = 0.f;
    if (t >= 0 && t < chunk_frames && m >= 0 && m < n_mels)
      v = (fmaxf(src[(long long)m * n_frames + t], mfloor) + 4.0f) * 0.25f;
    patch[i] = v;
  }
  const int groups = C / 8;
  const int cg = threadIdx.x % groups;
  const int lane_p = threadIdx.x / groups;
  const int PL = blockDim.x / groups;
  float wr[9][8], br[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    br[i] = bias ? __ldg(bias + cg * 8 + i) : 0.f;
#pragma unroll
    for (int k = 0; k < 9; ++k) wr[k][i] = __ldg(w + (cg * 8 + i) * 9 + k);
  }
  __syncthreads();
  if (lane_p >= PL) return;

  const int npos = nt * F1;
  for (int pos = lane_p; pos < npos; pos += PL) {
    const int tl = pos / F1, fo = pos - tl * F1;
    float in[9];
#pragma unroll
    for (int kh = 0; kh < 3; ++kh)
#pragma unroll
      for (int kw = 0; kw < 3; ++kw) in[kh * 3 + kw] = patch[(2 * tl + kw) * PW + 2 * fo + kh];
    alignas(16) __nv_bfloat162 r[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float a0 = br[2 * i], a1 = br[2 * i + 1];
#pragma unroll
      for (int k = 0; k < 9; ++k) {
        a0 = fmaf(wr[k][2 * i], in[k], a0);
        a1 = fmaf(wr[k][2 * i + 1], in[k], a1);
      }
      r[i] = __floats2bfloat162_rn(gelu_erf(a0), gelu_erf(a1));
    }
    bf16* dst = out + (((long long)chunk * T1 + t0 + tl) * F1 + fo) * C + cg * 8;
    *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<uint4*>(r);
  }
}

cudaError_t launch_conv1_chunked(const float* mel_raw, const unsigned int* clip_max, int batch, int n_mels,
                                 int n_frames, int chunk_frames, const float* w, const float* b, int C, bf16* out,
                                 cudaStream_t st) {
  if (C > 512 || n_mels > MAXM || C % 8) return cudaErrorInvalidValue;
  const int chunks_per_clip = n_frames / chunk_frames;
  const int T1 = (chunk_frames - 1) / 2 + 1;
  dim3 grid(batch * chunks_per_clip, (T1 + TB - 1) / TB);
  const int groups = C / 8;
  const int threads = groups * std::max(1, THREADS / groups);
  return launch_pdl(conv1_chunked_kernel, grid, dim3(threads), 0, st, mel_raw, clip_max, n_mels, n_frames, chunk_frames,
                    chunks_per_clip, w, b, C, out);
}

}  // namespace asr

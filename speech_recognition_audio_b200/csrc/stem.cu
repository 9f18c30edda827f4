// First convolution of the chunked Conv2D stem ("MOSS-Transcribe-preview-2B-
// GGUF", Architecture "Conv front-end": 3 x Conv2D stride 2, 1 -> 480).
// With one input channel its contraction length is 9, so it runs on the CUDA
// cores; its cost is the bias + GELU of every output (16 x 30 s of audio give
// 737 M of them) and the bf16 write of the result.
//
// Persistent blocks walk work units of C1_TB output time rows of one chunk.
// Each thread keeps the 9 taps of 8 output channels (and their biases) in
// registers as channel pairs and computes two channels per packed fp32
// instruction (f32x2 FMA, GELU in pairs).  The input patch of a unit - the
// normalised, zero-padded log-mel rows it reads - sits in shared memory with
// every value duplicated ({v, v}) so that one 8-byte load gives the packed
// operand; the next unit's patch is fetched into registers while the current
// one is computed (two patch buffers, one barrier per unit).  The log-mel
// normalisation (clamp at clip max - 8, then (x + 4) / 4) is applied while
// staging.  Output layout: [chunk, T1, F1, C] bf16 (channels innermost), or
// (phase mode, T1 and F1 even) the chunk's four parity planes
// [chunk][t % 2][f % 2][T1 / 2][F1 / 2][C], so that every tap of the stride-2
// conv2 reads consecutive rows of one plane as a dense TMA box; each thread
// stores 16 bytes.
#include "kernels.h"

namespace asr {

namespace {
constexpr int C1_TB = 5;                    // output time rows per work unit
constexpr int C1_THREADS = 480;             // block size limit
constexpr int C1_MAXM = 128;                // mel-bin capacity
constexpr int C1_PW = C1_MAXM + 2;          // patch row pitch (zero column on each side)
constexpr int C1_ROWS = 2 * C1_TB + 1;      // patch rows of a full unit
constexpr int C1_PATCH = C1_ROWS * C1_PW;   // float2 entries per buffer
constexpr int C1_PF = 8;                    // patch values a thread fetches per unit
}  // namespace

struct Conv1Args {
  const float* mel_raw;
  const unsigned int* clip_max;
  int n_mels, n_frames, chunk_frames, chunks_per_clip, T1, F1, units_per_chunk, n_units;
  const float* w;
  const float* bias;
  int C;
  int phase;  // 1 = parity-plane output
  bf16* out;
};

// Fetch the patch values of unit u owned by this thread: element e of the
// (rows x PW) patch, time row fastest (consecutive threads read consecutive
// frames of one mel bin).
__device__ __forceinline__ void conv1_fetch(const Conv1Args& a, int u, float (&pf)[C1_PF]) {
  const int chunk = u / a.units_per_chunk;
  const int t0 = (u - chunk * a.units_per_chunk) * C1_TB;
  const int rows = 2 * min(C1_TB, a.T1 - t0) + 1;
  const int b = chunk / a.chunks_per_clip;
  const int q = chunk - b * a.chunks_per_clip;
  const float mfloor = ordered_to_float(a.clip_max[b]) - 8.0f;
  const float* src = a.mel_raw + (long long)b * a.n_mels * a.n_frames + (long long)q * a.chunk_frames;
  const int n = rows * (a.n_mels + 2);
#pragma unroll
  for (int k = 0; k < C1_PF; ++k) {
    const int e = threadIdx.x + k * blockDim.x;
    float v = 0.f;
    if (e < n) {
      const int c = e / rows, j = e - c * rows;
      const int t = 2 * t0 - 1 + j, m = c - 1;
      if (t >= 0 && t < a.chunk_frames && m >= 0 && m < a.n_mels)
        v = (fmaxf(__ldg(src + (long long)m * a.n_frames + t), mfloor) + 4.0f) * 0.25f;
    }
    pf[k] = v;
  }
}

__device__ __forceinline__ void conv1_stage(const Conv1Args& a, int u, const float (&pf)[C1_PF], float2* buf) {
  const int chunk = u / a.units_per_chunk;
  const int t0 = (u - chunk * a.units_per_chunk) * C1_TB;
  const int rows = 2 * min(C1_TB, a.T1 - t0) + 1;
  const int n = rows * (a.n_mels + 2);
#pragma unroll
  for (int k = 0; k < C1_PF; ++k) {
    const int e = threadIdx.x + k * blockDim.x;
    if (e < n) {
      const int c = e / rows, j = e - c * rows;
      buf[j * C1_PW + c] = make_float2(pf[k], pf[k]);
    }
  }
}

__global__ void __launch_bounds__(C1_THREADS, 1) conv1_chunked_kernel(const Conv1Args a) {
  __shared__ float2 patch[2][C1_PATCH];
  const int groups = a.C / 8;
  const int PL = blockDim.x / groups;  // position lanes; blockDim.x == groups * PL
  const int cg = threadIdx.x % groups;
  const int lane_p = threadIdx.x / groups;

  // weights are constants of the model: load them before the dependency wait
  float2 wr[9][4], br[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    br[i] = a.bias ? make_float2(__ldg(a.bias + cg * 8 + 2 * i), __ldg(a.bias + cg * 8 + 2 * i + 1))
                   : make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < 9; ++k)
      wr[k][i] = make_float2(__ldg(a.w + (cg * 8 + 2 * i) * 9 + k), __ldg(a.w + (cg * 8 + 2 * i + 1) * 9 + k));
  }
  pdl_wait();
  pdl_trigger();

  float pf[C1_PF];
  int u = blockIdx.x;
  if (u < a.n_units) {
    conv1_fetch(a, u, pf);
    conv1_stage(a, u, pf, patch[0]);
  }
  __syncthreads();
  int cur = 0;
  for (; u < a.n_units; u += gridDim.x) {
    const int un = u + gridDim.x;
    if (un < a.n_units) conv1_fetch(a, un, pf);  // in flight while this unit computes

    const int chunk = u / a.units_per_chunk;
    const int t0 = (u - chunk * a.units_per_chunk) * C1_TB;
    const int npos = min(C1_TB, a.T1 - t0) * a.F1;
    const float2* buf = patch[cur];
    bf16* obase = a.out + ((long long)chunk * a.T1 + t0) * a.F1 * a.C + cg * 8;
    bf16* pbase = a.out + (long long)chunk * a.T1 * a.F1 * a.C + cg * 8;  // the chunk's four parity planes
    if (lane_p < PL) {
      for (int pos = lane_p; pos < npos; pos += PL) {
        const int tl = pos / a.F1, fo = pos - tl * a.F1;
        float2 acc[4] = {br[0], br[1], br[2], br[3]};
#pragma unroll
        for (int kh = 0; kh < 3; ++kh)
#pragma unroll
          for (int kw = 0; kw < 3; ++kw) {
            // tap (kh, kw): frequency 2 fo + kh - 1, time 2 t + kw - 1 (patch offsets +1)
            const float2 x = buf[(2 * tl + kw) * C1_PW + 2 * fo + kh];
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[i] = fma2(wr[kh * 3 + kw][i], x, acc[i]);
          }
        alignas(16) __nv_bfloat162 r[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 g = gelu_erf2(acc[i]);
          r[i] = __floats2bfloat162_rn(g.x, g.y);
        }
        bf16* dst;
        if (a.phase) {
          const int t = t0 + tl;
          const int plane = (t & 1) * 2 + (fo & 1);
          dst = pbase + (((long long)plane * (a.T1 >> 1) + (t >> 1)) * (a.F1 >> 1) + (fo >> 1)) * a.C;
        } else {
          dst = obase + (long long)pos * a.C;
        }
        *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<uint4*>(r);
      }
    }
    if (un < a.n_units) conv1_stage(a, un, pf, patch[cur ^ 1]);
    __syncthreads();
    cur ^= 1;
  }
}

cudaError_t launch_conv1_chunked(const float* mel_raw, const unsigned int* clip_max, int batch, int n_mels,
                                 int n_frames, int chunk_frames, const float* w, const float* b, int C, bf16* out,
                                 int phase, cudaStream_t st) {
  if (n_mels > C1_MAXM || C % 8 || C / 8 > C1_THREADS) return cudaErrorInvalidValue;
  Conv1Args a;
  a.mel_raw = mel_raw;
  a.clip_max = clip_max;
  a.n_mels = n_mels;
  a.n_frames = n_frames;
  a.chunk_frames = chunk_frames;
  a.chunks_per_clip = n_frames / chunk_frames;
  a.T1 = (chunk_frames - 1) / 2 + 1;
  a.F1 = (n_mels - 1) / 2 + 1;
  a.units_per_chunk = (a.T1 + C1_TB - 1) / C1_TB;
  a.n_units = batch * a.chunks_per_clip * a.units_per_chunk;
  a.w = w;
  a.bias = b;
  a.C = C;
  a.out = out;
  a.phase = phase ? 1 : 0;
  if (a.phase && (a.T1 % 2 || a.F1 % 2)) return cudaErrorInvalidValue;
  const int groups = C / 8;
  const int threads = groups * (C1_THREADS / groups);
  // every patch value of a unit has an owner: threads * C1_PF >= rows * pitch
  if (threads * C1_PF < C1_ROWS * (n_mels + 2)) return cudaErrorInvalidValue;
  if (a.n_units == 0) return cudaSuccess;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int grid = std::min(a.n_units, sms);
  return launch_pdl(conv1_chunked_kernel, dim3(grid), dim3(threads), 0, st, a);
}

}  // namespace asr

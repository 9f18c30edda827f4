// First convolution of the chunked Conv2D stem ("MOSS-Transcribe-preview-2B-
// GGUF", Architecture "Conv front-end": 3 x Conv2D stride 2, 1 -> 480).
//
// With one input channel the convolution's contraction length is 9.  It
// runs as a tcgen05 GEMM (output positions x channels, K = 9 taps padded to
// 16, the remaining 48 columns of the 64-wide k-block filled with zeros by
// the TMA), so the CUDA cores spend their cycles on the bias + GELU epilogue
// of the 737 M outputs of a 16 x 30 s batch rather than on the taps.  This
// file builds the GEMM's A operand: for every output position the 9
// normalised log-mel values its 3 x 3 window reads (clamp at the clip
// maximum - 8, then (x + 4) / 4; zero outside the chunk), as bf16, in rows
// of 16.
//
// Row order (layout): 0 plain [chunk][T1][F1]; 1 (T1 and F1 even) the
// chunk's four parity planes [chunk][t % 2][f % 2][T1 / 2][F1 / 2], so the
// GEMM's output rows land in the layout the stride-2 conv2 reads as dense
// TMA boxes; 2 (packed) the planes over all chunks,
// [t % 2][f % 2][chunk][S2][F1 / 2] with S2 = T1 / 2 + 1: the last row of
// every chunk is a zero row (A row zero here; the GEMM writes its output
// row as zero).  Threads run along time within a plane row so that the mel
// reads (frames contiguous) are coalesced; each thread writes one 32-byte
// row.
#include "kernels.h"

namespace asr {

template <int OUTK>
__global__ void __launch_bounds__(256) conv1_im2col_kernel(const float* __restrict__ mel_raw,
                                                           const unsigned int* __restrict__ clip_max, int n_mels,
                                                           int n_frames, int chunk_frames, int chunks_per_clip,
                                                           int T1, int F1, long long rows, int phase,
                                                           long long n_chunks, const ChunkDesc* __restrict__ cd,
                                                           const MelClip* __restrict__ mc, void* __restrict__ a_out) {
  pdl_wait();
  pdl_trigger();
  const long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (i >= rows) return;
  // thread index -> (chunk, plane, f, t) with t fastest (t < TS; t = TP is
  // the packed layout's zero row)
  const int TP = phase ? T1 / 2 : T1, FP = phase ? F1 / 2 : F1, TS = phase == 2 ? TP + 1 : TP;
  const int t = static_cast<int>(i % TS);
  long long rest = i / TS;
  const int f = static_cast<int>(rest % FP);
  rest /= FP;
  int plane;
  long long chunk;
  if (phase == 2) {
    chunk = rest % n_chunks;
    plane = static_cast<int>(rest / n_chunks);
  } else {
    plane = phase ? static_cast<int>(rest % 4) : 0;
    chunk = phase ? rest / 4 : rest;
  }
  // output row: [chunk][plane][T][F] (plain: [chunk][T1][F1]; packed:
  // [plane][chunk][S2][F])
  const long long row = phase == 2 ? ((plane * n_chunks + chunk) * (long long)TS + t) * FP + f
                                   : (chunk * (phase ? 4 : 1) + plane) * (long long)TP * FP + (long long)t * FP + f;
  if (t >= TP) {
    if constexpr (OUTK == KIND_TF32) {
      float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a_out) + row * 16);
#pragma unroll
      for (int k = 0; k < 4; ++k) dst[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    } else {
      uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(a_out) + row * 16);
      dst[0] = dst[1] = make_uint4(0, 0, 0, 0);
    }
    return;
  }
  const int t1 = phase ? 2 * t + (plane >> 1) : t;
  const int f1 = phase ? 2 * f + (plane & 1) : f;
  int b, F, valid;
  const float* src;
  if (cd) {
    // variable-length batch: the chunk's clip, first frame and valid frames
    const ChunkDesc c = cd[chunk];
    b = c.clip;
    F = mc[b].frames;
    valid = c.nvalid;
    src = mel_raw + (long long)n_mels * mc[b].f_off + c.frame0;
  } else {
    b = static_cast<int>(chunk / chunks_per_clip);
    const int q = static_cast<int>(chunk - (long long)b * chunks_per_clip);
    F = n_frames;
    valid = chunk_frames;
    src = mel_raw + (long long)b * n_mels * n_frames + (long long)q * chunk_frames;
  }
  const float mfloor = ordered_to_float(clip_max[b]) - 8.0f;
  float v[16];
#pragma unroll
  for (int kh = 0; kh < 3; ++kh)
#pragma unroll
    for (int kw = 0; kw < 3; ++kw) {
      // tap (kh, kw): frequency 2 f1 + kh - 1, time 2 t1 + kw - 1; frames
      // past the chunk's valid ones are the convolution's zero padding
      const int m = 2 * f1 + kh - 1, tt = 2 * t1 + kw - 1;
      float x = 0.f;
      if (m >= 0 && m < n_mels && tt >= 0 && tt < valid)
        x = (fmaxf(__ldg(src + (long long)m * F + tt), mfloor) + 4.0f) * 0.25f;
      v[kh * 3 + kw] = x;
    }
#pragma unroll
  for (int k = 9; k < 16; ++k) v[k] = 0.f;
  if constexpr (OUTK == KIND_TF32) {
    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a_out) + row * 16);
#pragma unroll
    for (int k = 0; k < 4; ++k) dst[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
  } else {
    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(a_out) + row * 16);
    dst[0] = pack8_16<OUTK>(v);
    dst[1] = pack8_16<OUTK>(v + 8);
  }
}

// a: rows of the kind's element type (bf16, f16, or fp32 for KIND_TF32).
template <int OUTK>
static cudaError_t im2col_launch(const float* mel_raw, const unsigned int* clip_max, int n_mels, int n_frames,
                                 int chunk_frames, int chunks_per_clip, int T1, int F1, long long rows, int phase,
                                 long long n_chunks, const ChunkDesc* cd, const MelClip* mc, void* a, cudaStream_t st) {
  const unsigned blocks = static_cast<unsigned>((rows + 255) / 256);
  return launch_pdl(conv1_im2col_kernel<OUTK>, dim3(blocks), dim3(256), 0, st, mel_raw, clip_max, n_mels, n_frames,
                    chunk_frames, chunks_per_clip, T1, F1, rows, phase, n_chunks, cd, mc, a);
}

static cudaError_t im2col_kind(int kind, const float* mel_raw, const unsigned int* clip_max, int n_mels, int n_frames,
                               int chunk_frames, int chunks_per_clip, int T1, int F1, long long rows, int phase,
                               long long n_chunks, const ChunkDesc* cd, const MelClip* mc, void* a, cudaStream_t st) {
  switch (kind) {
    case KIND_TF32: return im2col_launch<KIND_TF32>(mel_raw, clip_max, n_mels, n_frames, chunk_frames, chunks_per_clip,
                                                    T1, F1, rows, phase, n_chunks, cd, mc, a, st);
    case KIND_F16: return im2col_launch<KIND_F16>(mel_raw, clip_max, n_mels, n_frames, chunk_frames, chunks_per_clip,
                                                  T1, F1, rows, phase, n_chunks, cd, mc, a, st);
    default: return im2col_launch<KIND_BF16>(mel_raw, clip_max, n_mels, n_frames, chunk_frames, chunks_per_clip, T1,
                                             F1, rows, phase, n_chunks, cd, mc, a, st);
  }
}

// Rows of the A operand (= conv1 output positions) in a layout.
static long long im2col_rows(long long chunks, int T1, int F1, int phase) {
  return phase == 2 ? 4LL * chunks * (T1 / 2 + 1) * (F1 / 2) : chunks * T1 * F1;
}

cudaError_t launch_conv1_im2col(const float* mel_raw, const unsigned int* clip_max, int batch, int n_mels,
                                int n_frames, int chunk_frames, int phase, void* a, int kind, cudaStream_t st) {
  const int T1 = (chunk_frames - 1) / 2 + 1, F1 = (n_mels - 1) / 2 + 1;
  if (phase < 0 || phase > 2 || (phase && (T1 % 2 || F1 % 2))) return cudaErrorInvalidValue;
  const int chunks_per_clip = n_frames / chunk_frames;
  const long long chunks = (long long)batch * chunks_per_clip;
  const long long rows = im2col_rows(chunks, T1, F1, phase);
  if (rows == 0) return cudaSuccess;
  return im2col_kind(kind, mel_raw, clip_max, n_mels, n_frames, chunk_frames, chunks_per_clip, T1, F1, rows, phase,
                     chunks, nullptr, nullptr, a, st);
}

cudaError_t launch_conv1_im2col_varlen(const float* mel_raw, const unsigned int* clip_max, int n_chunks, int n_mels,
                                       int chunk_frames, int phase, const ChunkDesc* cd, const MelClip* mc, void* a,
                                       int kind, cudaStream_t st) {
  const int T1 = (chunk_frames - 1) / 2 + 1, F1 = (n_mels - 1) / 2 + 1;
  if (phase < 0 || phase > 2 || (phase && (T1 % 2 || F1 % 2))) return cudaErrorInvalidValue;
  const long long rows = im2col_rows(n_chunks, T1, F1, phase);
  if (rows == 0) return cudaSuccess;
  return im2col_kind(kind, mel_raw, clip_max, n_mels, 0, chunk_frames, 1, T1, F1, rows, phase, n_chunks, cd, mc, a, st);
}

// ---------------------------------------------------------- short chunks
// A chunk with fewer than chunk_frames valid frames is computed in the
// layout of a whole one.  Its conv1 / conv2 output rows at or past the short
// chunk's own output length are zeroed, so that the next convolution reads
// zero padding there exactly as it would at the end of the short input
// (rows before that length only read valid inputs or that padding).
// level 1: conv1 output (length ceil(L / 2)), level 2: conv2 output
// (ceil(ceil(L / 2) / 2)).  One block per chunk; whole chunks return at once.
// (act: elements of `es` bytes, 2 or 4; C * es a multiple of 16.)
__global__ void mask_short_chunks_kernel(uint8_t* __restrict__ act, const ChunkDesc* __restrict__ cd, int chunk_frames,
                                         int level, int T, int F, int C, int layout, int S2, int n_chunks, int es) {
  pdl_wait();
  pdl_trigger();
  const int c = blockIdx.x;
  const int L = cd[c].nvalid;
  if (L >= chunk_frames) return;
  int tv = (L + 1) / 2;
  if (level == 2) tv = (tv + 1) / 2;
  if (tv >= T) return;
  const uint4 z = make_uint4(0, 0, 0, 0);
  if (layout == 0 || (layout == 2 && level == 2)) {
    // rows [tv, T) of the chunk's [T][F][C] block are contiguous (packed
    // conv2 output: the chunk's block starts at row c * S2)
    const long long r0 = (layout == 2 ? (long long)c * S2 : (long long)c * T) + tv;
    uint4* p = reinterpret_cast<uint4*>(act + r0 * F * C * es);
    const long long n16 = (long long)(T - tv) * F * C * es / 16;
    for (long long j = threadIdx.x; j < n16; j += blockDim.x) p[j] = z;
  } else {
    // parity planes: plane (pt, pf) holds t = 2 th + pt, TH = T / 2 rows of
    // the chunk, [chunk][4][TH] (layout 1) or [4][chunk][S2] (layout 2)
    const int TH = T / 2, FH = F / 2;
    for (int pl = 0; pl < 4; ++pl) {
      const int pt = pl >> 1;
      const int th0 = tv - pt <= 0 ? 0 : (tv - pt + 1) / 2;
      if (th0 >= TH) continue;
      const long long r0 = layout == 2 ? ((long long)pl * n_chunks + c) * S2 + th0 : ((long long)c * 4 + pl) * TH + th0;
      uint4* p = reinterpret_cast<uint4*>(act + r0 * FH * C * es);
      const long long n16 = (long long)(TH - th0) * FH * C * es / 16;
      for (long long j = threadIdx.x; j < n16; j += blockDim.x) p[j] = z;
    }
  }
}

cudaError_t launch_mask_short_chunks(void* act, const ChunkDesc* cd, int n_chunks, int chunk_frames, int level, int T,
                                     int F, int C, int layout, int S2, int es, cudaStream_t st) {
  if (n_chunks <= 0) return cudaSuccess;
  if ((C * es) % 16 || layout < 0 || layout > 2 || (layout == 1 && (T % 2 || F % 2)) ||
      (layout == 2 && level == 1 && (T % 2 || F % 2 || S2 != T / 2 + 1)) || (layout == 2 && level == 2 && S2 != T + 1))
    return cudaErrorInvalidValue;
  return launch_pdl(mask_short_chunks_kernel, dim3(n_chunks), dim3(256), 0, st, static_cast<uint8_t*>(act), cd,
                    chunk_frames, level, T, F, C, layout, S2, n_chunks, es);
}

// Valid tokens of every chunk, from the padded conv_out rows [chunk][t3] to
// the packed token rows of their clips (one warp per padded row).
__global__ void compact_tokens_kernel(const float* __restrict__ xpad, float* __restrict__ x,
                                      const ChunkDesc* __restrict__ cd, long long rows, int t3, int d) {
  pdl_wait();
  pdl_trigger();
  const long long r = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= rows) return;
  const int lane = threadIdx.x & 31;
  const long long c = r / t3;
  const int j = static_cast<int>(r - c * t3);
  const ChunkDesc dsc = cd[c];
  const int L = dsc.nvalid;
  const int tv = ((((L + 1) / 2) + 1) / 2 + 1) / 2;  // ceil(ceil(ceil(L / 2) / 2) / 2)
  if (j >= tv) return;
  const float4* s = reinterpret_cast<const float4*>(xpad + r * d);
  float4* o = reinterpret_cast<float4*>(x + (long long)(dsc.tok_dst + j) * d);
  for (int k = lane; k < d / 4; k += 32) o[k] = s[k];
}

cudaError_t launch_compact_tokens(const float* xpad, float* x, const ChunkDesc* cd, int n_chunks, int t3, int d,
                                  cudaStream_t st) {
  const long long rows = (long long)n_chunks * t3;
  if (rows <= 0) return cudaSuccess;
  if (d % 4) return cudaErrorInvalidValue;
  return launch_pdl(compact_tokens_kernel, dim3(static_cast<unsigned>((rows + 7) / 8)), dim3(256), 0, st, xpad, x, cd,
                    rows, t3, d);
}

}  // namespace asr

// Log-mel front-end kernel ("MOSS-Transcribe-preview-2B-GGUF", Architecture
// "Audio" row: 16 kHz, n_fft=400, hop=160, 128 mel bins matching
// WhisperFeatureExtractor; Non-obvious gotchas: trailing STFT frame dropped).
//
// One block processes FB consecutive frames of one clip:
//   1. the PCM span of those frames (reflect-padded at the clip edges) is
//      staged in shared memory with coalesced loads;
//   2. each windowed 400-sample real frame is packed into a 200-point complex
//      sequence z[m] = x[2m] + i x[2m+1] and transformed by a mixed-radix
//      FFT, 200 = 8 x 25 = 8 x 5 x 5 (one radix-8 pass with twiddles, two
//      radix-5 passes), all in fp32 in shared memory;
//   3. the 201 one-sided bins of the real 400-point DFT are recovered from
//      Z[k] and Z[200-k], squared (power);
//   4. the sparse Slaney filterbank (<= ~16 taps per filter) gives the mel
//      energies, then log10(max(., 1e-10)) is written to [B, n_mels, F];
//   5. the block's maximum goes to the clip's max with one atomicMax on an
//      order-preserving integer encoding.
// The clamp at (max - 8) and the (x + 4) / 4 scaling need the clip maximum,
// so consumers apply them when they read the mel (conv stem, transpose, tap).
#include "kernels.h"

namespace asr {

namespace {

constexpr int FB = 8;         // frames per block
constexpr int NFFT = 400, HOP = 160, NC = 200, NBIN = 201;
constexpr int SPAN = (FB - 1) * HOP + NFFT;
constexpr int THREADS = 128;

__device__ __forceinline__ float2 cmul(float2 a, float2 b) {
  return make_float2(a.x * b.x - a.y * b.y, a.x * b.y + a.y * b.x);
}
__device__ __forceinline__ float2 cadd(float2 a, float2 b) { return make_float2(a.x + b.x, a.y + b.y); }
__device__ __forceinline__ float2 csub(float2 a, float2 b) { return make_float2(a.x - b.x, a.y - b.y); }
// -i * a
__device__ __forceinline__ float2 mul_mi(float2 a) { return make_float2(a.y, -a.x); }

// Forward 8-point DFT (exp(-2 pi i k n / 8)) in registers.
__device__ __forceinline__ void dft8(float2* x) {
  const float r = 0.70710678118654752f;
  float2 a0 = cadd(x[0], x[4]), a1 = csub(x[0], x[4]);
  float2 a2 = cadd(x[2], x[6]), a3 = csub(x[2], x[6]);
  float2 a4 = cadd(x[1], x[5]), a5 = csub(x[1], x[5]);
  float2 a6 = cadd(x[3], x[7]), a7 = csub(x[3], x[7]);
  float2 e0 = cadd(a0, a2), e2 = csub(a0, a2), e1 = cadd(a1, mul_mi(a3)), e3 = csub(a1, mul_mi(a3));
  float2 o0 = cadd(a4, a6), o2 = csub(a4, a6), o1 = cadd(a5, mul_mi(a7)), o3 = csub(a5, mul_mi(a7));
  // twiddles W8^k = exp(-i pi k / 4)
  float2 t1 = make_float2(r * (o1.x + o1.y), r * (o1.y - o1.x));   // o1 * (r - i r)
  float2 t2 = mul_mi(o2);                                         // o2 * (-i)
  float2 t3 = make_float2(r * (o3.y - o3.x), -r * (o3.x + o3.y));  // o3 * (-r - i r)
  x[0] = cadd(e0, o0); x[4] = csub(e0, o0);
  x[1] = cadd(e1, t1); x[5] = csub(e1, t1);
  x[2] = cadd(e2, t2); x[6] = csub(e2, t2);
  x[3] = cadd(e3, t3); x[7] = csub(e3, t3);
}

// Forward 5-point DFT using the conjugate-pair symmetry of the kernel.
__device__ __forceinline__ void dft5(float2* x) {
  const float c1 = 0.30901699437494742f, c2 = -0.80901699437494742f;
  const float s1 = 0.95105651629515357f, s2 = 0.58778525229247313f;
  float2 sa = cadd(x[1], x[4]), da = csub(x[1], x[4]);
  float2 sb = cadd(x[2], x[3]), db = csub(x[2], x[3]);
  float2 x0 = x[0];
  float2 p1 = make_float2(x0.x + c1 * sa.x + c2 * sb.x, x0.y + c1 * sa.y + c2 * sb.y);
  float2 p2 = make_float2(x0.x + c2 * sa.x + c1 * sb.x, x0.y + c2 * sa.y + c1 * sb.y);
  float2 q1 = make_float2(s1 * da.x + s2 * db.x, s1 * da.y + s2 * db.y);  // X1 = p1 - i q1, X4 = p1 + i q1
  float2 q2 = make_float2(s2 * da.x - s1 * db.x, s2 * da.y - s1 * db.y);  // X2 = p2 - i q2, X3 = p2 + i q2
  x[0] = make_float2(x0.x + sa.x + sb.x, x0.y + sa.y + sb.y);
  x[1] = make_float2(p1.x + q1.y, p1.y - q1.x);
  x[4] = make_float2(p1.x - q1.y, p1.y + q1.x);
  x[2] = make_float2(p2.x + q2.y, p2.y - q2.x);
  x[3] = make_float2(p2.x - q2.y, p2.y + q2.x);
}

}  // namespace

__global__ void __launch_bounds__(THREADS) log_mel_kernel(const float* __restrict__ pcm, long long n_samples,
                                                          int n_frames, int n_mels, const MelTables* __restrict__ tab,
                                                          float* __restrict__ mel, unsigned int* __restrict__ clip_max) {
  __shared__ float xs[SPAN];
  __shared__ float2 buf0[FB * NC];
  __shared__ float2 buf1[FB * NC];
  __shared__ float2 w200[NC];
  __shared__ float2 w400[NBIN];
  __shared__ float hann[NFFT];
  __shared__ float red[THREADS / 32];

  pdl_wait();
  pdl_trigger();
  const int groups_per_clip = (n_frames + FB - 1) / FB;
  const int b = blockIdx.x / groups_per_clip;
  const int f0 = (blockIdx.x - b * groups_per_clip) * FB;
  const int nf = min(FB, n_frames - f0);
  const float* x = pcm + (long long)b * n_samples;
  const int tid = threadIdx.x;

  for (int i = tid; i < NC; i += THREADS) w200[i] = tab->w200[i];
  for (int i = tid; i < NBIN; i += THREADS) w400[i] = tab->w400[i];
  for (int i = tid; i < NFFT; i += THREADS) hann[i] = tab->hann[i];
  // Padded sample j of frame f is original index f*HOP + j - NFFT/2, reflected.
  const long long base = (long long)f0 * HOP - NFFT / 2;
  const int span = (nf - 1) * HOP + NFFT;
  for (int j = tid; j < span; j += THREADS) {
    long long i = base + j;
    if (i < 0) i = -i;
    if (i >= n_samples) i = 2 * (n_samples - 1) - i;
    xs[j] = __ldg(x + i);
  }
  __syncthreads();

  // Pass A: for each frame r and n2 < 25: 8-point DFT over n1 of
  // z[25 n1 + n2], times W200^(n2 k1); stored k1-major: buf0[r][k1*25 + n2].
  for (int task = tid; task < nf * 25; task += THREADS) {
    const int r = task / 25, n2 = task - r * 25;
    const float* xr = xs + r * HOP;
    float2 v[8];
#pragma unroll
    for (int n1 = 0; n1 < 8; ++n1) {
      const int m = 25 * n1 + n2;
      v[n1] = make_float2(xr[2 * m] * hann[2 * m], xr[2 * m + 1] * hann[2 * m + 1]);
    }
    dft8(v);
#pragma unroll
    for (int k1 = 0; k1 < 8; ++k1) buf0[r * NC + k1 * 25 + n2] = k1 ? cmul(v[k1], w200[n2 * k1]) : v[0];
  }
  __syncthreads();
  // Pass B1: for each (r, k1, b): 5-point DFT over a of buf0[r][k1*25 + 5a + b],
  // times W25^(b c) = W200^(8 b c); stored buf1[r][k1*25 + 5c + b].
  for (int task = tid; task < nf * 40; task += THREADS) {
    const int r = task / 40, rem = task - r * 40, k1 = rem / 5, bb = rem - k1 * 5;
    float2 v[5];
    const float2* src = buf0 + r * NC + k1 * 25 + bb;
#pragma unroll
    for (int a = 0; a < 5; ++a) v[a] = src[5 * a];
    dft5(v);
    float2* dst = buf1 + r * NC + k1 * 25 + bb;
#pragma unroll
    for (int c = 0; c < 5; ++c) dst[5 * c] = c ? cmul(v[c], w200[8 * bb * c]) : v[0];
  }
  __syncthreads();
  // Pass B2: for each (r, k1, c): 5-point DFT over b of buf1[r][k1*25 + 5c + b];
  // output d is Z[k1 + 8 (c + 5 d)], stored in natural order in buf0.
  for (int task = tid; task < nf * 40; task += THREADS) {
    const int r = task / 40, rem = task - r * 40, k1 = rem / 5, c = rem - k1 * 5;
    float2 v[5];
    const float2* src = buf1 + r * NC + k1 * 25 + 5 * c;
#pragma unroll
    for (int bb = 0; bb < 5; ++bb) v[bb] = src[bb];
    dft5(v);
#pragma unroll
    for (int d = 0; d < 5; ++d) buf0[r * NC + k1 + 8 * (c + 5 * d)] = v[d];
  }
  __syncthreads();
  // Real 400-point spectrum: X[k] = E[k] + W400^k O[k] with
  // E = (Z[k] + conj Z[200-k]) / 2, O = -i (Z[k] - conj Z[200-k]) / 2; power.
  float* pw = reinterpret_cast<float*>(buf1);  // [FB][NBIN]
  for (int task = tid; task < nf * NBIN; task += THREADS) {
    const int r = task / NBIN, k = task - r * NBIN;
    const float2 zk = buf0[r * NC + (k == NC ? 0 : k)];
    const float2 zc0 = buf0[r * NC + (k == 0 ? 0 : NC - k)];
    const float2 zc = make_float2(zc0.x, -zc0.y);
    const float2 e = make_float2(0.5f * (zk.x + zc.x), 0.5f * (zk.y + zc.y));
    const float2 o = mul_mi(make_float2(0.5f * (zk.x - zc.x), 0.5f * (zk.y - zc.y)));
    const float2 xk = cadd(e, cmul(w400[k], o));
    pw[r * NBIN + k] = xk.x * xk.x + xk.y * xk.y;
  }
  __syncthreads();
  // Mel filterbank, log10, store; frames fastest for coalesced stores.
  float lmax = -INFINITY;
  float* out = mel + (long long)b * n_mels * n_frames;
  for (int task = tid; task < n_mels * FB; task += THREADS) {
    const int m = task / FB, r = task - m * FB;
    if (r < nf) {
      const int st = tab->fstart[m], cnt = tab->fcount[m], off = tab->foff[m];
      float acc = 0.f;
      for (int j = 0; j < cnt; ++j) acc = fmaf(tab->fw[off + j], pw[r * NBIN + st + j], acc);
      const float l = log10f(fmaxf(acc, 1e-10f));
      out[(long long)m * n_frames + f0 + r] = l;
      lmax = fmaxf(lmax, l);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
  if ((tid & 31) == 0) red[tid >> 5] = lmax;
  __syncthreads();
  if (tid == 0) {
    float mx = red[0];
    for (int i = 1; i < THREADS / 32; ++i) mx = fmaxf(mx, red[i]);
    atomicMax(clip_max + b, float_to_ordered(mx));
  }
}

// Normalised log-mel in [B, n_mels, F] fp32: (max(L, m - 8) + 4) / 4.
__global__ void mel_normalize_kernel(const float* __restrict__ raw, const unsigned int* __restrict__ clip_max,
                                     long long per_clip, int batch, float* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  const long long total = per_clip * batch;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int b = static_cast<int>(i / per_clip);
    const float m = ordered_to_float(clip_max[b]);
    out[i] = (fmaxf(raw[i], m - 8.0f) + 4.0f) * 0.25f;
  }
}

// Normalise and transpose to time-major bf16 [B, F, n_mels] (input of the
// Conv1D stem's implicit GEMM).
__global__ void mel_normalize_transpose_kernel(const float* __restrict__ raw, const unsigned int* __restrict__ clip_max,
                                               int n_mels, int n_frames, bf16* __restrict__ out) {
  __shared__ float tile[32][33];
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.z;
  const int f0 = blockIdx.x * 32, m0 = blockIdx.y * 32;
  const float mx = ordered_to_float(clip_max[b]) - 8.0f;
  const float* src = raw + (long long)b * n_mels * n_frames;
  for (int j = threadIdx.y; j < 32; j += blockDim.y) {
    const int m = m0 + j, f = f0 + threadIdx.x;
    if (m < n_mels && f < n_frames) tile[j][threadIdx.x] = (fmaxf(src[(long long)m * n_frames + f], mx) + 4.0f) * 0.25f;
  }
  __syncthreads();
  bf16* dst = out + (long long)b * n_frames * n_mels;
  for (int j = threadIdx.y; j < 32; j += blockDim.y) {
    const int f = f0 + j, m = m0 + threadIdx.x;
    if (m < n_mels && f < n_frames) dst[(long long)f * n_mels + m] = __float2bfloat16_rn(tile[threadIdx.x][j]);
  }
}

cudaError_t launch_log_mel(const float* pcm, long long n_samples, int batch, int n_mels, const MelTables* tab,
                           float* mel_raw, unsigned int* clip_max, cudaStream_t st) {
  const int n_frames = static_cast<int>(n_samples / HOP);
  const int groups = (n_frames + FB - 1) / FB;
  return launch_pdl(log_mel_kernel, dim3(groups * batch), dim3(THREADS), 0, st, pcm, n_samples, n_frames, n_mels, tab,
                    mel_raw, clip_max);
}

cudaError_t launch_mel_normalize(const float* raw, const unsigned int* clip_max, long long per_clip, int batch,
                                 float* out, cudaStream_t st) {
  const long long total = per_clip * batch;
  const int blocks = static_cast<int>(std::min<long long>((total + 255) / 256, 148LL * 16));
  return launch_pdl(mel_normalize_kernel, dim3(blocks), dim3(256), 0, st, raw, clip_max, per_clip, batch, out);
}

cudaError_t launch_mel_normalize_transpose(const float* raw, const unsigned int* clip_max, int batch, int n_mels,
                                           int n_frames, bf16* out, cudaStream_t st) {
  dim3 grid((n_frames + 31) / 32, (n_mels + 31) / 32, batch);
  return launch_pdl(mel_normalize_transpose_kernel, grid, dim3(32, 8), 0, st, raw, clip_max, n_mels, n_frames, out);
}

}  // namespace asr

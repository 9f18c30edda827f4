// Log-mel front-end ("MOSS-Transcribe-preview-2B-GGUF", Architecture "Audio"
// row: 16 kHz, n_fft=400, hop=160, 128 mel bins matching
// WhisperFeatureExtractor; Non-obvious gotchas: trailing STFT frame dropped,
// n_samples / hop frames).
//
// Tables (mel_tables_kernel): twiddles, the periodic Hann window and the
// sparse Slaney filterbank are computed on the device, in double precision
// and rounded once to float, into a MelTables buffer the caller provides.
// Every log-mel entry point builds its tables with this one kernel, so they
// all see identical tables and no host-to-device copy is needed.
//
// Log-mel (log_mel_kernel): a persistent grid, two 256-thread blocks per SM;
// a block takes groups of G = 32 consecutive frames of one clip in turn.
//   1. The PCM span of the next group (reflect-padded at the clip edges) is
//      copied into shared memory with cp.async while the current group is
//      transformed (double buffer).
//   2. Each frame belongs to 8 threads (an octet, 4 frames per warp).  The
//      windowed 400-sample real frame is packed as 200 complex points
//      z[m] = x[2m] + i x[2m+1]; with m = 8 n2 + t, thread t computes the
//      25-point DFT over n2 in registers (5 x 5) and multiplies by the
//      twiddles W200^(t k2).  A radix-8 pass over t (through the warp's
//      shared buffer, XOR-swizzled so that neither side conflicts) gives
//      Z[k2 + 25 k1], the 200-point DFT.
//   3. The real 400-point spectrum follows from Z[k] and Z[200-k] in pairs:
//      X[k] = E + W400^k O and conj X[200-k] = E - W400^k O with
//      E = (Z[k] + conj Z[200-k]) / 2, O = -i (Z[k] - conj Z[200-k]) / 2;
//      the 201 powers |X|^2 replace Z in the buffer.
//   4. The filterbank's taps (filter-major) are split over the octet in
//      eight runs of whole filters with about equal tap counts; each thread
//      walks its run with one fixed loop, emitting log10(max(sum, 1e-10))
//      at each filter's last tap; the block writes the [n_mels][32] tile with
//      coalesced row stores; the group's maximum goes to its clip with one
//      atomicMax on an order-preserving integer encoding.
// Only warp-level synchronisation separates the transform steps; three
// block barriers per group order the shared PCM span and the output tile.
// The clamp at (max - 8) and the (x + 4) / 4 scaling need the clip maximum,
// so consumers apply them when they read the mel (conv stem, transpose, tap).
#include "kernels.h"

namespace asr {

namespace {

constexpr int NFFT = 400, HOP = 160, NC = 200, NBIN = 201;
constexpr int G = 32;                               // frames per group
constexpr int SPAN_MAX = (G - 1) * HOP + NFFT;      // 5360 samples
constexpr int THREADS = 256;                        // 8 warps x 4 octets
constexpr int STAGE_PITCH = G + 1;                  // output tile row pitch (floats)

// Shared-memory layout of log_mel_kernel (bytes).
constexpr int SM_SPAN = 0;                                  // float [2][SPAN_MAX]
constexpr int SM_FFT = SM_SPAN + 2 * SPAN_MAX * 4;          // float2 [G][NC]
constexpr int SM_TW = SM_FFT + G * NC * 8;                  // float2 [25][8]: W200^(t k2)
constexpr int SM_W25 = SM_TW + 25 * 8 * 8;                  // float2 [25]: W25^j
constexpr int SM_W400 = SM_W25 + 26 * 8;                    // float2 [201 + 1]
constexpr int SM_HANN = SM_W400 + 202 * 8;                  // float2 [200]: (w[2m], w[2m+1])
constexpr int SM_TPART = SM_HANN + NC * 8;                  // int [9] (+ pad)
constexpr int SM_TCODE = SM_TPART + 16 * 4;                 // int [kMelMaxWeights]
constexpr int SM_FW = SM_TCODE + kMelMaxWeights * 4;        // float [kMelMaxWeights]
constexpr int SM_RED = SM_FW + kMelMaxWeights * 4;          // float [8]
constexpr int SM_BYTES = SM_RED + 8 * 4;
static_assert(128 * STAGE_PITCH <= SPAN_MAX, "the output tile fits in one PCM span buffer");
static_assert(2 * (SM_BYTES + 1024) <= 228 * 1024, "two blocks per SM");

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

// Forward 5-point DFT of (a0..a4), using the conjugate-pair symmetry of the
// kernel: X1 = p1 - i q1, X4 = p1 + i q1, X2 = p2 - i q2, X3 = p2 + i q2.
__device__ __forceinline__ void dft5(float2& a0, float2& a1, float2& a2, float2& a3, float2& a4) {
  const float c1 = 0.30901699437494742f, c2 = -0.80901699437494742f;   // cos(2 pi / 5), cos(4 pi / 5)
  const float s1 = 0.95105651629515357f, s2 = 0.58778525229247313f;    // sin(2 pi / 5), sin(4 pi / 5)
  const float2 sa = cadd(a1, a4), da = csub(a1, a4);
  const float2 sb = cadd(a2, a3), db = csub(a2, a3);
  const float2 x0 = a0;
  const float2 p1 = make_float2(x0.x + c1 * sa.x + c2 * sb.x, x0.y + c1 * sa.y + c2 * sb.y);
  const float2 p2 = make_float2(x0.x + c2 * sa.x + c1 * sb.x, x0.y + c2 * sa.y + c1 * sb.y);
  const float2 q1 = make_float2(s1 * da.x + s2 * db.x, s1 * da.y + s2 * db.y);
  const float2 q2 = make_float2(s2 * da.x - s1 * db.x, s2 * da.y - s1 * db.y);
  a0 = make_float2(x0.x + sa.x + sb.x, x0.y + sa.y + sb.y);
  a1 = make_float2(p1.x + q1.y, p1.y - q1.x);
  a4 = make_float2(p1.x - q1.y, p1.y + q1.x);
  a2 = make_float2(p2.x + q2.y, p2.y - q2.x);
  a3 = make_float2(p2.x - q2.y, p2.y + q2.x);
}

__device__ __forceinline__ void cp_async_4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

// Group g -> its clip, first frame and frame count, and the clip's PCM and
// mel bases.  Uniform batches use arithmetic; variable-length batches carry
// per-clip descriptors and are searched by group offset.
struct GroupLoc {
  const float* x;       // clip PCM
  long long n;          // clip samples
  float* out;           // clip mel [n_mels][F]
  int F, f0, nf, clip;
  int left;             // real samples before x
};

__device__ __forceinline__ GroupLoc locate(const MelArgs& a, int g) {
  GroupLoc L;
  if (!a.clips) {
    const int gpc = (a.n_frames + G - 1) / G;
    L.clip = g / gpc;
    L.f0 = (g - L.clip * gpc) * G;
    L.F = a.n_frames;
    L.n = a.n_samples;
    L.x = a.pcm + (long long)L.clip * a.n_samples;
    L.out = a.mel + (long long)L.clip * a.n_mels * a.n_frames;
    L.left = 0;
  } else {
    int lo = 0, hi = a.batch - 1;  // last clip whose first group is <= g
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (a.clips[mid].g_off <= g) lo = mid; else hi = mid - 1;
    }
    const MelClip& c = a.clips[lo];
    L.clip = lo;
    L.f0 = (g - c.g_off) * G;
    L.F = c.frames;
    L.n = c.n;
    L.x = a.pcm + c.s_off;
    L.out = a.mel + (long long)a.n_mels * c.f_off;
    L.left = c.left;
  }
  L.nf = min(G, L.F - L.f0);
  return L;
}

__device__ __forceinline__ void cp_async_16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

// Issue the cp.async copies of group g's reflect-padded PCM span: 16-byte
// copies when the span lies inside the clip (or its real history) and is
// 16-byte aligned (every span is a multiple of 8 samples), else 4-byte
// copies with the reflection.
__device__ __forceinline__ void stage_span(const MelArgs& a, int g, float* dst, int tid) {
  const GroupLoc L = locate(a, g);
  const long long base = (long long)L.f0 * HOP - NFFT / 2;
  const int span = (L.nf - 1) * HOP + NFFT;
  const float* src = L.x + base;
  if (base >= -(long long)L.left && base + span <= L.n && (reinterpret_cast<uintptr_t>(src) & 15) == 0) {
    for (int j = tid; j < span / 4; j += THREADS) cp_async_16(dst + 4 * j, src + 4 * j);
  } else {
    for (int j = tid; j < span; j += THREADS) {
      long long i = base + j;
      if (i < -(long long)L.left) i = -i;      // reflect at the start of the audio
      if (i >= L.n) i = 2 * (L.n - 1) - i;     // and at its end
      cp_async_4(dst + j, L.x + i);
    }
  }
  cp_async_commit();
}

}  // namespace

// ---------------------------------------------------------------- tables
// One block.  Slaney mel scale (3 f / 200 below 1 kHz, 15 + 27 ln(f / 1000)
// / ln 6.4 above); n_mels + 2 points uniform in mel over 0..8 kHz; filter m
// is the triangle from point m up to m + 1 and down to m + 2 at the bin
// frequencies 40 k Hz, scaled by 2 / (f_{m+2} - f_m); its non-zero run is
// stored as (first bin, count, offset into fw).
__global__ void __launch_bounds__(256) mel_tables_kernel(int n_mels, MelTables* __restrict__ t) {
  __shared__ double fpts[130];
  __shared__ int cnt[128], first[128];
  pdl_wait();
  pdl_trigger();
  const int tid = threadIdx.x;
  for (int j = tid; j < NC; j += blockDim.x) {
    double s, c;
    sincospi(2.0 * j / NC, &s, &c);
    t->w200[j] = make_float2((float)c, (float)-s);
  }
  for (int k = tid; k <= NC; k += blockDim.x) {
    double s, c;
    sincospi(2.0 * k / NFFT, &s, &c);
    t->w400[k] = make_float2((float)c, (float)-s);
  }
  for (int n = tid; n < NFFT; n += blockDim.x) t->hann[n] = (float)(0.5 - 0.5 * cospi(2.0 * n / NFFT));
  const double ln64 = log(6.4);
  const double mmax = 15.0 + 27.0 * log(8.0) / ln64;  // mel of 8 kHz (above 1 kHz)
  for (int i = tid; i < n_mels + 2; i += blockDim.x) {
    const double m = mmax * i / (n_mels + 1);
    fpts[i] = m < 15.0 ? 200.0 * m / 3.0 : 1000.0 * exp((m - 15.0) * ln64 / 27.0);
  }
  __syncthreads();
  auto weight = [&](int m, int k) {
    const double lo = fpts[m], ce = fpts[m + 1], hi = fpts[m + 2];
    const double f = 40.0 * k;
    return fmax(0.0, fmin((f - lo) / (ce - lo), (hi - f) / (hi - ce))) * (2.0 / (hi - lo));
  };
  if (tid < n_mels) {
    int f = -1, c = 0;
    for (int k = 0; k <= NC; ++k) {
      if (weight(tid, k) > 0.0) {
        if (f < 0) f = k;
        ++c;
      } else if (f >= 0) {
        break;
      }
    }
    first[tid] = f < 0 ? 0 : f;
    cnt[tid] = c;
  }
  __syncthreads();
  if (tid == 0) {
    int off = 0;
    for (int m = 0; m < n_mels; ++m) {
      t->fstart[m] = first[m];
      t->fcount[m] = min(max(cnt[m], 1), kMelMaxWeights - off);  // an empty filter keeps one zero tap
      t->foff[m] = off;
      off += t->fcount[m];
    }
    for (int m = n_mels; m < 128; ++m) t->fstart[m] = t->fcount[m] = t->foff[m] = 0;
    // thread split: cut at the first filter start at or after each eighth of the taps
    t->tpart[0] = 0;
    int m = 0;
    for (int q = 1; q < 8; ++q) {
      const int target = (q * off) / 8;
      while (m < n_mels && t->foff[m] < target) ++m;
      t->tpart[q] = m < n_mels ? t->foff[m] : off;
    }
    t->tpart[8] = off;
  }
  __syncthreads();
  if (tid < n_mels) {
    const int st = t->fstart[tid], c = t->fcount[tid], o = t->foff[tid];
    for (int j = 0; j < c; ++j) {
      t->fw[o + j] = cnt[tid] ? (float)weight(tid, st + j) : 0.0f;
      t->tcode[o + j] = (st + j) | ((j == c - 1) << 8) | (tid << 9);
    }
  }
}

// ---------------------------------------------------------------- log-mel
__global__ void __launch_bounds__(THREADS, 2) log_mel_kernel(const MelArgs a, const MelTables* __restrict__ tab) {
  extern __shared__ __align__(16) uint8_t smem[];
  float* span = reinterpret_cast<float*>(smem + SM_SPAN);
  float2* fft = reinterpret_cast<float2*>(smem + SM_FFT);
  float2* tw = reinterpret_cast<float2*>(smem + SM_TW);
  float2* w25 = reinterpret_cast<float2*>(smem + SM_W25);
  float2* w400 = reinterpret_cast<float2*>(smem + SM_W400);
  float2* hann2 = reinterpret_cast<float2*>(smem + SM_HANN);
  int* tpart = reinterpret_cast<int*>(smem + SM_TPART);
  int* tcode = reinterpret_cast<int*>(smem + SM_TCODE);
  float* fw = reinterpret_cast<float*>(smem + SM_FW);
  float* red = reinterpret_cast<float*>(smem + SM_RED);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t = lane & 7;                 // thread within the frame's octet
  const int r = warp * 4 + (lane >> 3);   // frame slot of this octet in the group
  pdl_wait();
  pdl_trigger();

  // Tables into shared memory, once per block.
  for (int i = tid; i < 25 * 8; i += THREADS) {
    const int k2 = i >> 3, tt = i & 7;
    tw[i] = tab->w200[tt * k2];           // W200^(t k2), t k2 <= 168
  }
  for (int i = tid; i < 25; i += THREADS) w25[i] = tab->w200[8 * i];
  for (int i = tid; i < NBIN; i += THREADS) w400[i] = tab->w400[i];
  for (int i = tid; i < NC; i += THREADS) hann2[i] = make_float2(tab->hann[2 * i], tab->hann[2 * i + 1]);
  if (tid < 9) tpart[tid] = tab->tpart[tid];
  for (int i = tid; i < kMelMaxWeights; i += THREADS) {
    fw[i] = tab->fw[i];
    tcode[i] = tab->tcode[i];
  }

  int g = blockIdx.x;
  int buf = 0;
  if (g < a.n_groups) stage_span(a, g, span, tid);
  for (; g < a.n_groups; g += gridDim.x, buf ^= 1) {
    const GroupLoc L = locate(a, g);
    float* cur = span + buf * SPAN_MAX;
    cp_async_wait_all();
    __syncthreads();                                       // (A) span and tables visible
    if (g + (int)gridDim.x < a.n_groups) stage_span(a, g + gridDim.x, span + (buf ^ 1) * SPAN_MAX, tid);

    float2* fb = fft + r * NC;                             // this frame's buffer (200 complex)
    // ---- 25-point DFTs over n2 (m = 8 n2 + t), then W200^(t k2)
    {
      const float2* xs = reinterpret_cast<const float2*>(cur + r * HOP);
      float2 z[25];
#pragma unroll
      for (int n2 = 0; n2 < 25; ++n2) {
        const float2 v = xs[8 * n2 + t], h = hann2[8 * n2 + t];
        z[n2] = make_float2(v.x * h.x, v.y * h.y);
      }
      // n2 = 5 a + b: 5-point DFTs over a (result c stored where a was)
#pragma unroll
      for (int b = 0; b < 5; ++b) dft5(z[b], z[5 + b], z[10 + b], z[15 + b], z[20 + b]);
      // inner twiddles W25^(b c)
#pragma unroll
      for (int c = 1; c < 5; ++c)
#pragma unroll
        for (int b = 1; b < 5; ++b) z[5 * c + b] = cmul(z[5 * c + b], w25[b * c]);
      // 5-point DFTs over b: slot 5 c + d holds Z[c + 5 d]
#pragma unroll
      for (int c = 0; c < 5; ++c) dft5(z[5 * c], z[5 * c + 1], z[5 * c + 2], z[5 * c + 3], z[5 * c + 4]);
      // row k2 of the [25][8] buffer, column t swizzled by k2 & 7
#pragma unroll
      for (int c = 0; c < 5; ++c)
#pragma unroll
        for (int d = 0; d < 5; ++d) {
          const int k2 = c + 5 * d;
          const float2 v = k2 ? cmul(z[5 * c + d], tw[k2 * 8 + t]) : z[5 * c + d];
          fb[k2 * 8 + (t ^ (k2 & 7))] = v;
        }
    }
    __syncwarp();
    // ---- 8-point DFTs over t: task k2 = t + 8 j gives Z[k2 + 25 k1]
    {
      float2 y[4][8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int k2 = t + 8 * j;
        if (k2 < 25) {
#pragma unroll
          for (int s = 0; s < 8; ++s) y[j][s] = fb[k2 * 8 + (s ^ (k2 & 7))];
          dft8(y[j]);
        }
      }
      __syncwarp();
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int k2 = t + 8 * j;
        if (k2 < 25) {
#pragma unroll
          for (int k1 = 0; k1 < 8; ++k1) fb[k2 + 25 * k1] = y[j][k1];
        }
      }
    }
    __syncwarp();
    // ---- real 400-point spectrum: powers of bins k and 200 - k, in pairs
    float* pw = reinterpret_cast<float*>(fb);              // 201 powers replace Z
    {
      float p0[13], p1[13];
#pragma unroll
      for (int j = 0; j < 13; ++j) {
        const int k = t + 8 * j;
        if (k <= 100) {
          const float2 zk = fb[k];
          const float2 zm = fb[k ? NC - k : 0];
          const float2 e = make_float2(0.5f * (zk.x + zm.x), 0.5f * (zk.y - zm.y));
          const float2 o = mul_mi(make_float2(0.5f * (zk.x - zm.x), 0.5f * (zk.y + zm.y)));
          const float2 wo = cmul(w400[k], o);
          const float2 xa = cadd(e, wo), xb = csub(e, wo);   // X[k], conj X[400 - k] = X[200 - k]*
          p0[j] = xa.x * xa.x + xa.y * xa.y;
          p1[j] = xb.x * xb.x + xb.y * xb.y;
        }
      }
      __syncwarp();
#pragma unroll
      for (int j = 0; j < 13; ++j) {
        const int k = t + 8 * j;
        if (k <= 100) {
          pw[k] = p0[j];
          pw[NC - k] = p1[j];                                // k = 100 writes the same value twice
        }
      }
    }
    __syncwarp();
    __syncthreads();                                       // (B) every warp is done with the PCM span
    // ---- filterbank, log10, into the output tile [n_mels][G] (in the PCM span buffer)
    float* tile = cur;
    float lmax = -INFINITY;
    {
      // this thread's share of the taps: whole filters, in order
      const int j1 = tpart[t + 1];
      float acc = 0.f;
      for (int j = tpart[t]; j < j1; ++j) {
        const int c = tcode[j];
        acc = fmaf(fw[j], pw[c & 255], acc);
        if (c & 256) {
          const float l = __log10f(fmaxf(acc, 1e-10f));
          tile[(c >> 9) * STAGE_PITCH + r] = l;
          if (r < L.nf) lmax = fmaxf(lmax, l);
          acc = 0.f;
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
    if (lane == 0) red[warp] = lmax;
    __syncthreads();                                       // (C) tile complete
    for (int m = warp; m < a.n_mels; m += THREADS / 32)
      if (lane < L.nf) L.out[(long long)m * L.F + L.f0 + lane] = tile[m * STAGE_PITCH + lane];
    if (tid == 0) {
      float mx = red[0];
#pragma unroll
      for (int i = 1; i < THREADS / 32; ++i) mx = fmaxf(mx, red[i]);
      atomicMax(a.clip_max + L.clip, float_to_ordered(mx));
    }
  }
  cp_async_wait_all();
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
template <int OUTK>
__global__ void mel_normalize_transpose_kernel(const float* __restrict__ raw, const unsigned int* __restrict__ clip_max,
                                               int n_mels, int n_frames, void* __restrict__ out) {
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
  const long long base = (long long)b * n_frames * n_mels;
  for (int j = threadIdx.y; j < 32; j += blockDim.y) {
    const int f = f0 + j, m = m0 + threadIdx.x;
    if (m < n_mels && f < n_frames) {
      const long long i = base + (long long)f * n_mels + m;
      const float v = tile[threadIdx.x][j];
      if constexpr (OUTK == KIND_TF32)
        static_cast<float*>(out)[i] = v;
      else if constexpr (OUTK == KIND_F16)
        static_cast<__half*>(out)[i] = __float2half_rn(v);
      else
        static_cast<bf16*>(out)[i] = __float2bfloat16_rn(v);
    }
  }
}

cudaError_t launch_mel_tables(int n_mels, MelTables* tab, cudaStream_t st) {
  if (n_mels <= 0 || n_mels > 128 || !tab) return cudaErrorInvalidValue;
  return launch_pdl(mel_tables_kernel, dim3(1), dim3(256), 0, st, n_mels, tab);
}

static int sm_count_current() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

int mel_groups(long long n_frames) { return static_cast<int>((n_frames + G - 1) / G); }

cudaError_t launch_log_mel(const MelArgs& args, const MelTables* tab, cudaStream_t st) {
  if (args.n_groups <= 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(log_mel_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SM_BYTES);
  // Two blocks per SM need ~213 KB: ask for the whole shared-memory carveout.
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(log_mel_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  const int blocks = std::min(args.n_groups, 2 * sm_count_current());
  return launch_pdl(log_mel_kernel, dim3(blocks), dim3(THREADS), SM_BYTES, st, args, tab);
}

cudaError_t launch_log_mel(const float* pcm, long long n_samples, int batch, int n_mels, const MelTables* tab,
                           float* mel_raw, unsigned int* clip_max, cudaStream_t st) {
  MelArgs a = {};
  a.pcm = pcm;
  a.mel = mel_raw;
  a.clip_max = clip_max;
  a.n_mels = n_mels;
  a.batch = batch;
  a.n_samples = n_samples;
  a.n_frames = static_cast<int>(n_samples / HOP);
  a.n_groups = mel_groups(a.n_frames) * batch;
  a.clips = nullptr;
  return launch_log_mel(a, tab, st);
}

cudaError_t launch_mel_normalize(const float* raw, const unsigned int* clip_max, long long per_clip, int batch,
                                 float* out, cudaStream_t st) {
  const long long total = per_clip * batch;
  const int blocks = static_cast<int>(std::min<long long>((total + 255) / 256, 148LL * 16));
  return launch_pdl(mel_normalize_kernel, dim3(blocks), dim3(256), 0, st, raw, clip_max, per_clip, batch, out);
}

cudaError_t launch_mel_normalize_transpose(const float* raw, const unsigned int* clip_max, int batch, int n_mels,
                                           int n_frames, void* out, int kind, cudaStream_t st) {
  dim3 grid((n_frames + 31) / 32, (n_mels + 31) / 32, batch);
  switch (kind) {
    case KIND_TF32:
      return launch_pdl(mel_normalize_transpose_kernel<KIND_TF32>, grid, dim3(32, 8), 0, st, raw, clip_max, n_mels,
                        n_frames, out);
    case KIND_F16:
      return launch_pdl(mel_normalize_transpose_kernel<KIND_F16>, grid, dim3(32, 8), 0, st, raw, clip_max, n_mels,
                        n_frames, out);
    default:
      return launch_pdl(mel_normalize_transpose_kernel<KIND_BF16>, grid, dim3(32, 8), 0, st, raw, clip_max, n_mels,
                        n_frames, out);
  }
}

}  // namespace asr

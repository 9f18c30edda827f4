// Per-layer kernels other than the GEMMs: LayerNorm, windowed / full
// attention, and small helpers.
//
// Attention ("MOSS-Transcribe-preview-2B-GGUF", Architecture "Audio encoder":
// windowed, block-diagonal attention; the whisper-small variant attends over
// the whole clip): segments are given by cumulative offsets and only a
// segment's own keys are visited, so the block-diagonal structure costs
// nothing.  Segments of at most 128 tokens run on the tcgen05 kernel of
// attn_tc.cu.  Longer ones (the whisper-small variant's 1500-frame clips) run
// here: QK^T and PV on bf16 tensor cores (mma.sync m16n8k16, fp32
// accumulate), a flash-style kernel with one block per (64-query tile,
// segment, head) and an online softmax over 64-key tiles in fp32 registers,
// keys past the segment end masked to -inf, scale 1/sqrt(64).
#include "kernels.h"

namespace asr {

// ------------------------------------------------------------ LayerNorm
// One warp per row, V float4 per lane (D = 128 V).  The statistics take one
// pass over the row in shifted form: with K = x[row][0],
//   mean = K + S1 / D,  var = S2 / D - (S1 / D)^2,
//   S1 = sum (x - K),   S2 = sum (x - K)^2,
// which keeps the cancellation at the scale of the row's spread (|x - K|
// is a few standard deviations), not of its mean.  The second pass re-reads
// the row (L1 / L2 hits) to normalise and store, so no thread holds a whole
// row and every row of a 6240 x 1280 residual stream is in flight at once
// (one wave of warps instead of two).

// Read-only 16-byte load that the compiler may not merge with another load
// of the same address (the second pass must re-read, not keep the row).
__device__ __forceinline__ float4 ldg_f4_nomerge(const float4* p) {
  float4 v;
  asm volatile("ld.global.nc.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "l"(p));
  return v;
}

template <int V, bool OUT_F32>
__global__ void __launch_bounds__(256, 6) layer_norm_kernel(const float* __restrict__ x, const float* __restrict__ g,
                                                            const float* __restrict__ b, long long M, float eps,
                                                            void* __restrict__ y) {
  pdl_wait();
  pdl_trigger();
  const long long row = blockIdx.x * 8LL + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  constexpr int D = V * 128;
  // 16-byte loads in flight per lane: the statistics pass keeps up to 5 in
  // flight (the row arrives in two round trips), the normalising pass 2
  // (its re-reads hit L1, and it also holds gamma and beta).
  constexpr int U1 = V % 5 == 0 ? 5 : (V % 4 == 0 ? 4 : (V % 3 == 0 ? 3 : (V % 2 == 0 ? 2 : 1)));
  constexpr int U = V % 2 == 0 ? 2 : 1;
  // (at most 6 blocks of 256 threads per SM fit 42 registers per thread:
  // 48 row-warps per SM, 7104 rows in flight on 148 SMs)
  const float4* xr = reinterpret_cast<const float4*>(x + row * D);
  const float K = __ldg(x + row * D);
  float s1 = 0.f, s2 = 0.f;
#pragma unroll 1
  for (int i0 = 0; i0 < V; i0 += U1) {
    float4 v[U1];
#pragma unroll
    for (int u = 0; u < U1; ++u) v[u] = ldg_f4_nomerge(xr + lane + 32 * (i0 + u));
#pragma unroll
    for (int u = 0; u < U1; ++u) {
      const float a = v[u].x - K, bb = v[u].y - K, c = v[u].z - K, d = v[u].w - K;
      s1 += (a + bb) + (c + d);
      s2 += (a * a + bb * bb) + (c * c + d * d);
    }
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
  const float4* g4 = reinterpret_cast<const float4*>(g);
  const float4* b4 = reinterpret_cast<const float4*>(b);
#pragma unroll 1
  for (int i0 = 0; i0 < V; i0 += U) {
    float4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) v[u] = ldg_f4_nomerge(xr + lane + 32 * (i0 + u));
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c4 = lane + 32 * (i0 + u);
      const float4 gg = __ldg(g4 + c4), bv = __ldg(b4 + c4);
      const float o0 = (v[u].x - mean) * rstd * gg.x + bv.x;
      const float o1 = (v[u].y - mean) * rstd * gg.y + bv.y;
      const float o2 = (v[u].z - mean) * rstd * gg.z + bv.z;
      const float o3 = (v[u].w - mean) * rstd * gg.w + bv.w;
      if (OUT_F32) {
        reinterpret_cast<float4*>(reinterpret_cast<float*>(y) + row * D)[c4] = make_float4(o0, o1, o2, o3);
      } else {
        __nv_bfloat162 p0 = __floats2bfloat162_rn(o0, o1), p1 = __floats2bfloat162_rn(o2, o3);
        uint2 w2;
        w2.x = *reinterpret_cast<uint32_t*>(&p0);
        w2.y = *reinterpret_cast<uint32_t*>(&p1);
        reinterpret_cast<uint2*>(reinterpret_cast<bf16*>(y) + row * D)[c4] = w2;
      }
    }
  }
}

template <bool F32>
static cudaError_t ln_dispatch(int V, const float* x, const float* g, const float* b, long long M, float eps, void* y,
                               cudaStream_t st) {
  const unsigned blocks = static_cast<unsigned>((M + 7) / 8);
  switch (V) {
#define ASR_LN_CASE(n) \
  case n: {                                                                                  \
    cudaError_t e_ = launch_pdl(layer_norm_kernel<n, F32>, dim3(blocks), dim3(256), 0, st, x, g, b, M, eps, y); \
    if (e_ != cudaSuccess) return e_;                                                        \
    break;                                                                                   \
  }
    ASR_LN_CASE(1) ASR_LN_CASE(2) ASR_LN_CASE(3) ASR_LN_CASE(4) ASR_LN_CASE(5) ASR_LN_CASE(6) ASR_LN_CASE(7)
    ASR_LN_CASE(8) ASR_LN_CASE(9) ASR_LN_CASE(10) ASR_LN_CASE(11) ASR_LN_CASE(12) ASR_LN_CASE(13)
    ASR_LN_CASE(14) ASR_LN_CASE(15) ASR_LN_CASE(16)
#undef ASR_LN_CASE
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_layer_norm(const float* x, const float* g, const float* b, long long M, int D, float eps, void* y,
                              bool out_f32, cudaStream_t st) {
  if (D % 128 || D > 2048 || M <= 0) return cudaErrorInvalidValue;
  return out_f32 ? ln_dispatch<true>(D / 128, x, g, b, M, eps, y, st) : ln_dispatch<false>(D / 128, x, g, b, M, eps, y, st);
}

// ------------------------------------------------------------ attention
namespace {
constexpr int BQ = 64, BKV = 64, HD = 64, LDS = HD + 8;

__device__ __forceinline__ void ldsm_x4(uint32_t* r, const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t* r, const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void mma_bf16_16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
// Copy a 64-row x 64-col bf16 tile (rows >= valid are zero-filled).
__device__ __forceinline__ void load_tile(bf16* dst, const bf16* src, long long ld, int valid, int tid) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int c = tid + 128 * i;  // 512 chunks of 16 bytes
    const int r = c >> 3, k = (c & 7) * 8;
    const bool v = r < valid;
    cp_async_16_zfill(dst + r * LDS + k, v ? src + r * ld + k : src, v);
  }
}
}  // namespace

__global__ void __launch_bounds__(128) attention_kernel(const bf16* __restrict__ qkv, const int* __restrict__ cu, int H,
                                                        bf16* __restrict__ out) {
  __shared__ __align__(16) bf16 Qs[BQ * LDS];
  __shared__ __align__(16) bf16 Ks[2][BKV * LDS];
  __shared__ __align__(16) bf16 Vs[2][BKV * LDS];
  pdl_wait();
  pdl_trigger();
  const int seg = blockIdx.y, h = blockIdx.z;
  const int s0 = cu[seg], L = cu[seg + 1] - s0;
  const int q0 = blockIdx.x * BQ;
  if (q0 >= L) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long ld = 3LL * H * HD;
  const bf16* qbase = qkv + (long long)(s0 + q0) * ld + h * HD;
  const bf16* kbase = qkv + (long long)s0 * ld + (H + h) * HD;
  const bf16* vbase = qkv + (long long)s0 * ld + (2 * H + h) * HD;
  const int n_kv = (L + BKV - 1) / BKV;

  load_tile(Qs, qbase, ld, L - q0, tid);
  load_tile(Ks[0], kbase, ld, L, tid);
  load_tile(Vs[0], vbase, ld, L, tid);
  cp_async_commit();

  const float sl2 = 0.125f * 1.4426950408889634f;  // (1/sqrt(64)) * log2(e)
  float o[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
  uint32_t qf[4][4];
  const int g = lane >> 2, t4 = lane & 3;

  for (int j = 0; j < n_kv; ++j) {
    const int cur = j & 1;
    if (j + 1 < n_kv) {
      load_tile(Ks[cur ^ 1], kbase + (long long)(j + 1) * BKV * ld, ld, L - (j + 1) * BKV, tid);
      load_tile(Vs[cur ^ 1], vbase + (long long)(j + 1) * BKV * ld, ld, L - (j + 1) * BKV, tid);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (j == 0) {
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        ldsm_x4(qf[ks], Qs + (warp * 16 + (lane & 15)) * LDS + ks * 16 + (lane >> 4) * 8);
    }
    // S = Q K^T for this warp's 16 rows x 64 keys.
    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
    const bf16* Kt = Ks[cur];
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        uint32_t kb[4];
        ldsm_x4(kb, Kt + (16 * p + (lane & 7) + (lane >> 4) * 8) * LDS + ks * 16 + ((lane >> 3) & 1) * 8);
        mma_bf16_16816(s[2 * p], qf[ks], kb[0], kb[1]);
        mma_bf16_16816(s[2 * p + 1], qf[ks], kb[2], kb[3]);
      }
    }
    // Mask keys past the segment end; online softmax (base-2, pre-scaled).
    const int kv0 = j * BKV;
    float mnew[2] = {mrow[0], mrow[1]};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = kv0 + nt * 8 + 2 * t4 + (e & 1);
        float v = s[nt][e] * sl2;
        if (key >= L) v = -INFINITY;
        s[nt][e] = v;
        mnew[e >> 1] = fmaxf(mnew[e >> 1], v);
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mnew[r] = fmaxf(mnew[r], __shfl_xor_sync(0xffffffffu, mnew[r], 1));
      mnew[r] = fmaxf(mnew[r], __shfl_xor_sync(0xffffffffu, mnew[r], 2));
    }
    float corr[2], psum[2] = {0.f, 0.f};
#pragma unroll
    for (int r = 0; r < 2; ++r) corr[r] = exp2f(mrow[r] - mnew[r]);
    uint32_t pf[4][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const float p0 = exp2f(s[nt][0] - mnew[0]), p1 = exp2f(s[nt][1] - mnew[0]);
      const float p2 = exp2f(s[nt][2] - mnew[1]), p3 = exp2f(s[nt][3] - mnew[1]);
      psum[0] += p0 + p1;
      psum[1] += p2 + p3;
      pf[nt >> 1][(nt & 1) * 2 + 0] = pack_bf16(p0, p1);
      pf[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16(p2, p3);
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      psum[r] += __shfl_xor_sync(0xffffffffu, psum[r], 1);
      psum[r] += __shfl_xor_sync(0xffffffffu, psum[r], 2);
      lrow[r] = lrow[r] * corr[r] + psum[r];
      mrow[r] = mnew[r];
    }
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      o[nt][0] *= corr[0]; o[nt][1] *= corr[0];
      o[nt][2] *= corr[1]; o[nt][3] *= corr[1];
    }
    // O += P V
    const bf16* Vt = Vs[cur];
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      // A fragment of P for keys 16ks..16ks+15: (a0,a1) from n-tile 2ks, (a2,a3) from 2ks+1.
      uint32_t a[4] = {pf[ks][0], pf[ks][1], pf[ks][2], pf[ks][3]};
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        uint32_t vb[4];
        ldsm_x4_t(vb, Vt + (16 * ks + (lane & 7) + ((lane >> 3) & 1) * 8) * LDS + 16 * p + (lane >> 4) * 8);
        mma_bf16_16816(o[2 * p], a, vb[0], vb[1]);
        mma_bf16_16816(o[2 * p + 1], a, vb[2], vb[3]);
      }
    }
    __syncthreads();
  }
  // Normalise and store rows inside the segment.
  const float inv0 = 1.f / lrow[0], inv1 = 1.f / lrow[1];
  const int r0 = q0 + warp * 16 + g, r1 = r0 + 8;
  bf16* ob = out + (long long)s0 * (H * HD) + h * HD;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    const int col = nt * 8 + 2 * t4;
    if (r0 < L)
      *reinterpret_cast<uint32_t*>(ob + (long long)r0 * (H * HD) + col) = pack_bf16(o[nt][0] * inv0, o[nt][1] * inv0);
    if (r1 < L)
      *reinterpret_cast<uint32_t*>(ob + (long long)r1 * (H * HD) + col) = pack_bf16(o[nt][2] * inv1, o[nt][3] * inv1);
  }
}

cudaError_t launch_attention(const bf16* qkv, const int* cu, int n_seg, int max_seg, int H, bf16* out,
                             cudaStream_t st) {
  if (n_seg <= 0 || max_seg <= 0 || H <= 0) return cudaErrorInvalidValue;
  dim3 grid((max_seg + BQ - 1) / BQ, n_seg, H);
  return launch_pdl(attention_kernel, grid, dim3(128), 0, st, qkv, cu, H, out);
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

__global__ void bf16_to_f32_kernel(const bf16* __restrict__ in, float* __restrict__ out, long long n) {
  pdl_wait();
  pdl_trigger();
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
    out[i] = __bfloat162float(in[i]);
}

cudaError_t launch_bf16_to_f32(const bf16* in, float* out, long long n, cudaStream_t st) {
  const int blocks = static_cast<int>(std::min<long long>((n + 255) / 256, 148LL * 32));
  return launch_pdl(bf16_to_f32_kernel, dim3(blocks), dim3(256), 0, st, in, out, n);
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

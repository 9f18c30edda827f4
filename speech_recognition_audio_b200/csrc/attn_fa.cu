// Attention over long segments on the tcgen05 tensor cores: the full
// (unwindowed) attention of the whisper-small variant ("CrisperWhisper ->
// ONNX", What this exports instead: whisper-small geometry; Results: 1500
// encoder frames per 30 s window), and any segment longer than the 128
// tokens the one-tile kernel of attn_tc.cu takes.
//
// One CTA per (128-query tile, segment, head), 10 warps:
//   warp 8  TMA producer: Q once, then K_j (one buffer, reloaded once S_j
//           has read it) and V_j (two buffers, so V_{j+1} arrives while the
//           softmax and P V of tile j run);
//   warp 9  MMA issuer: S = Q K_j^T (M=128, N=128, K=64) into tensor memory,
//           issued for tile j+1 as soon as the softmax has read S_j, then
//           O += P_j V_j (M=128, N=64, K=128) with O kept in tensor memory;
//   warps 0-7  softmax: warps w and w+4 share the 32 query rows of TMEM lane
//           quarter w % 4 and take keys [64 h, 64 h + 64) of every tile and
//           O columns [32 h, 32 h + 32), h = w / 4; the two halves of a row
//           exchange their maxima and, at the end, their sums through shared
//           memory at a named barrier of the warp pair.  Online softmax in
//           base 2 with the scale 1/sqrt(64) folded into one FMA into
//           ex2.approx; the running maximum used for the exponentials moves
//           only when a tile's maximum exceeds it by more than 8 (then O and
//           the row sums are rescaled by 2^(old - new)), so probabilities
//           stay <= 256 and most tiles need no rescale.  P (bf16 or f16, the
//           operands' type) goes to shared memory as the A operand of the
//           next MMA; at the end each thread divides its 32 O columns by the
//           row sum and stores them.
// Tensor memory: S in columns 0..127, O in 128..191 (256 allocated: two
// CTAs per SM).  Shared memory: Q (16 KB), K (16 KB), V (2 x 16 KB), P
// (32 KB).  Every wait is bounded; tensor memory is freed after all MMAs
// have completed.
#include "kernels.h"

namespace asr {

namespace {
constexpr int FA_THREADS = 320;
// K and V ring slots (16 KB each): V double-buffered (measured 504 against
// 535 us per whisper-small launch with K double-buffered instead; both
// double-buffered do not fit two CTAs per SM, and one CTA per SM, or two
// query tiles per CTA sharing the rings, measured slower)
constexpr int FA_KB = 1, FA_VB = 2;
constexpr int FA_SQ = 0, FA_SK = 16384, FA_SV = FA_SK + FA_KB * 16384, FA_SP = FA_SV + FA_VB * 16384;  // P: two 64-key halves
constexpr int FA_TILES = FA_SP + 32768;
constexpr int FA_RED = FA_TILES;                 // float [2 tiles][2 halves][128 rows] row maxima, then sums
constexpr int FA_BARS = FA_RED + 2 * 2 * 128 * 4;
constexpr int FA_SMEM = 1024 + FA_BARS + 256;
constexpr int FA_TMEM_COLS = 256;
constexpr int FA_O_COL = 128;
constexpr float FA_RESCALE_LOG2 = 8.0f;

enum { B_Q = 0, B_KF0, B_KF1, B_KE0, B_KE1, B_VF0, B_VF1, B_VE0, B_VE1, B_SF, B_SFREE, B_PF, B_OD, B_DRAIN, B_COUNT };
static_assert(FA_KB <= 2 && FA_VB <= 2, "barrier table");

// Named barrier of the two softmax warps of one TMEM lane quarter (ids 1-4).
__device__ __forceinline__ void pair_sync(int q) { asm volatile("bar.sync %0, 64;" ::"r"(1 + q) : "memory"); }
}  // namespace

template <int KIND>
__global__ void __launch_bounds__(FA_THREADS, 2) attention_fa_kernel(const __grid_constant__ CUtensorMap tm_qkv,
                                                                     const int* __restrict__ cu, int H,
                                                                     bf16* __restrict__ out, int* status,
                                                                     unsigned long long limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* red = reinterpret_cast<float*>(sm + FA_RED);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + FA_BARS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + B_COUNT);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qt = blockIdx.x, seg = blockIdx.y, h = blockIdx.z;

  if (tid == 0) {
    for (int i = 0; i < B_COUNT; ++i) mbar_init(&bar[i], (i == B_SFREE || i == B_PF) ? 8 : 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_qkv);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, FA_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();
  pdl_trigger();

  const int s0 = cu[seg], L = cu[seg + 1] - s0;
  const int q0 = qt * 128;
  const int nk = (L + 127) / 128;
  if (q0 < L) {
    if (warp == 8) {
      // ------------------------------------------------ TMA producer
      if (lane == 0) {
        bool ok = true;
        int issued_k = 0, issued_v = 0;
        mbar_arrive_expect_tx(&bar[B_Q], 16384);
        tma_load_2d(sm + FA_SQ, &tm_qkv, &bar[B_Q], h * 64, s0 + q0);
        for (int j = 0; j < nk && ok; ++j) {
          // K_j into ring slot j % KB once S_{j-KB} has read it
          const int kb = j % FA_KB;
          if (j >= FA_KB && !(ok = mbar_wait_bounded(&bar[B_KE0 + kb], (j / FA_KB - 1) & 1, limit_ns, status,
                                                     DEV_TIMEOUT_PRODUCER)))
            break;
          mbar_arrive_expect_tx(&bar[B_KF0 + kb], 16384);
          tma_load_2d(sm + FA_SK + kb * 16384, &tm_qkv, &bar[B_KF0 + kb], (H + h) * 64, s0 + j * 128);
          ++issued_k;
          // V_j into ring slot j % VB once P_{j-VB} V_{j-VB} has read it
          const int vb = j % FA_VB;
          if (j >= FA_VB && !(ok = mbar_wait_bounded(&bar[B_VE0 + vb], (j / FA_VB - 1) & 1, limit_ns, status,
                                                     DEV_TIMEOUT_PRODUCER)))
            break;
          mbar_arrive_expect_tx(&bar[B_VF0 + vb], 16384);
          tma_load_2d(sm + FA_SV + vb * 16384, &tm_qkv, &bar[B_VF0 + vb], (2 * H + h) * 64, s0 + j * 128);
          ++issued_v;
        }
        // every issued load lands before the CTA exits
        mbar_wait_bounded(&bar[B_Q], 0, kDrainLimitNs, nullptr, 0);
        for (int j = issued_k - FA_KB < 0 ? 0 : issued_k - FA_KB; j < issued_k; ++j)
          mbar_wait_bounded(&bar[B_KF0 + j % FA_KB], (j / FA_KB) & 1, kDrainLimitNs, nullptr, 0);
        for (int j = issued_v - FA_VB < 0 ? 0 : issued_v - FA_VB; j < issued_v; ++j)
          mbar_wait_bounded(&bar[B_VF0 + j % FA_VB], (j / FA_VB) & 1, kDrainLimitNs, nullptr, 0);
      }
    } else if (warp == 9) {
      // ------------------------------------------------ MMA issuer
      if (lane == 0) {
        const uint32_t idesc_s = idesc_kind_f32(KIND, 128, 128);
        const uint32_t idesc_o = idesc_kind_f32(KIND, 128, 64) | (1u << 16);  // B = V, MN-major
        const uint64_t qd = sw128_kmajor_desc(smem_u32(sm + FA_SQ));
        auto issue_s = [&](int j) {
          const uint64_t kd = sw128_kmajor_desc(smem_u32(sm + FA_SK + (j % FA_KB) * 16384));
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 4; ++k) tc_mma_bf16(tmem, qd + 2 * k, kd + 2 * k, idesc_s, k > 0 ? 1u : 0u);
          tc_commit(&bar[B_SF]);
          tc_commit(&bar[B_KE0 + j % FA_KB]);
        };
        bool ok = mbar_wait_bounded(&bar[B_Q], 0, limit_ns, status, DEV_TIMEOUT_MMA) &&
                  mbar_wait_bounded(&bar[B_KF0], 0, limit_ns, status, DEV_TIMEOUT_MMA);
        if (ok) issue_s(0);
        for (int j = 0; j < nk && ok; ++j) {
          if (j + 1 < nk) {
            // S for the next tile once its K has landed and the softmax has read S_j
            ok = mbar_wait_bounded(&bar[B_KF0 + (j + 1) % FA_KB], ((j + 1) / FA_KB) & 1, limit_ns, status, DEV_TIMEOUT_MMA) &&
                 mbar_wait_bounded(&bar[B_SFREE], j & 1, limit_ns, status, DEV_TIMEOUT_MMA);
            if (!ok) break;
            issue_s(j + 1);
          }
          ok = mbar_wait_bounded(&bar[B_PF], j & 1, limit_ns, status, DEV_TIMEOUT_MMA) &&
               mbar_wait_bounded(&bar[B_VF0 + j % FA_VB], (j / FA_VB) & 1, limit_ns, status, DEV_TIMEOUT_MMA);
          if (!ok) break;
          tc_fence_after();
          const uint64_t vd = sw128_mnmajor_desc(smem_u32(sm + FA_SV + (j % FA_VB) * 16384));
#pragma unroll
          for (int kb = 0; kb < 2; ++kb) {
            const uint64_t pd = sw128_kmajor_desc(smem_u32(sm + FA_SP + kb * 16384));
#pragma unroll
            for (int k = 0; k < 4; ++k)
              tc_mma_bf16(tmem + FA_O_COL, pd + 2 * k, vd + (uint64_t)((kb * 4 + k) * 128), idesc_o,
                          (j > 0 || kb > 0 || k > 0) ? 1u : 0u);
          }
          tc_commit(&bar[B_OD]);
          tc_commit(&bar[B_VE0 + j % FA_VB]);
        }
        // all issued MMAs complete before tensor memory is released
        tc_commit(&bar[B_DRAIN]);
        mbar_wait_bounded(&bar[B_DRAIN], 0, kDrainLimitNs, nullptr, 0);
      }
    } else {
      // ------------------------------------------------ softmax (warps 0-7)
      const int q = warp & 3, hh = warp >> 2;            // lane quarter, key / O-column half
      const int row = q * 32 + lane;
      const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16);
      const float sl2 = 0.125f * 1.4426950408889634f;  // (1 / sqrt(64)) log2(e)
      float m_used = -INFINITY, lsum = 0.f;
      bool ok = true;
      // Every tile runs through both pair barriers even after a failed wait
      // (ok stays false and later waits are skipped), so the two warps of a
      // pair always meet the same number of barriers.
      for (int j = 0; j < nk; ++j) {
        ok = __all_sync(0xffffffffu, ok && mbar_wait_bounded(&bar[B_SF], j & 1, limit_ns, status, DEV_TIMEOUT_EPILOGUE));
        tc_fence_after();
        float sv[64];
#pragma unroll
        for (int c = 0; c < 64; c += 16) tmem_ld16(trow + hh * 64 + c, sv + c);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[B_SFREE]);
        const int kv = min(128, L - j * 128) - hh * 64;  // valid keys of this half (may be <= 0)
        // half-row maximum of the raw scores (four chains; only a partial
        // half needs the per-key mask)
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        if (kv >= 64) {
#pragma unroll
          for (int c = 0; c < 64; ++c) m4[c & 3] = fmaxf(m4[c & 3], sv[c]);
        } else {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c < kv) m4[c & 3] = fmaxf(m4[c & 3], sv[c]);
        }
        float* rbuf = red + (j & 1) * 256;
        rbuf[hh * 128 + row] = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        pair_sync(q);
        // the scale is positive: max(s) * scale = max(s * scale)
        float mt = fmaxf(rbuf[row], rbuf[128 + row]);
        mt = ok ? mt * sl2 : 0.f;
        const bool grow = j > 0 && mt > m_used + FA_RESCALE_LOG2;
        const float corr = grow ? ex2_approx(m_used - mt) : 1.0f;
        if (j == 0 || grow) m_used = mt;
        // p = 2^((s - m) / 8 log2 e) as one FMA into ex2.approx, while the
        // previous tile's P V may still run
        const float nm = -m_used;
        // whole 16-key chunks as packed pair FMAs and packed sums; per-key
        // masks only in the chunk that holds the segment's end; chunks past
        // it stay zero (uniform tests)
        const float2 sl2v = make_float2(sl2, sl2), nmv = make_float2(nm, nm);
        float2 s2[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) s2[i] = make_float2(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < 64; c += 16) {
          if (c + 16 <= kv && ok) {
#pragma unroll
            for (int i = c; i < c + 16; i += 2) {
              const float2 a = fma2(make_float2(sv[i], sv[i + 1]), sl2v, nmv);
              sv[i] = ex2_approx(a.x);
              sv[i + 1] = ex2_approx(a.y);
              s2[(i >> 1) & 3] = add2(s2[(i >> 1) & 3], make_float2(sv[i], sv[i + 1]));
            }
          } else if (c < kv && ok) {
#pragma unroll
            for (int i = c; i < c + 16; ++i) {
              sv[i] = (i < kv) ? ex2_approx(fmaf(sv[i], sl2, nm)) : 0.f;
              s2[(i >> 1) & 3].x += sv[i];
            }
          } else {
#pragma unroll
            for (int i = c; i < c + 16; ++i) sv[i] = 0.f;
          }
        }
        lsum = lsum * corr + (((s2[0].x + s2[0].y) + (s2[1].x + s2[1].y)) + ((s2[2].x + s2[2].y) + (s2[3].x + s2[3].y)));
        // P_j may overwrite P_{j-1} and O may be rescaled once O_{j-1} is complete
        if (j > 0) ok = __all_sync(0xffffffffu, ok && mbar_wait_bounded(&bar[B_OD], (j - 1) & 1, limit_ns, status,
                                                                        DEV_TIMEOUT_EPILOGUE));
        tc_fence_after();
        // this half's 64 keys of the P row: one 128-byte row of P block hh,
        // 16-byte chunks swizzled by (row & 7)
        uint4* prow = reinterpret_cast<uint4*>(sm + FA_SP + hh * 16384 + row * 128);
#pragma unroll
        for (int c = 0; c < 8; ++c) prow[c ^ (row & 7)] = pack8_16<KIND>(sv + c * 8);
        if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
          for (int c = 0; c < 32; c += 16) {
            float ov[16];
            tmem_ld16(trow + FA_O_COL + hh * 32 + c, ov);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) ov[i] *= corr;
            tmem_st16(trow + FA_O_COL + hh * 32 + c, ov);
          }
          tmem_st_wait();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[B_PF]);
      }
      // epilogue: the row sum from both halves, then this half's O columns / sum
      const bool got = ok && mbar_wait_bounded(&bar[B_OD], (nk - 1) & 1, limit_ns, status, DEV_TIMEOUT_EPILOGUE);
      tc_fence_after();
      float* sbuf = red + (nk & 1) * 256;  // the buffer the last tile did not use
      sbuf[hh * 128 + row] = lsum;
      pair_sync(q);
      const float tot = sbuf[row] + sbuf[128 + row];
      float ov[32];
#pragma unroll
      for (int c = 0; c < 32; c += 16) tmem_ld16(trow + FA_O_COL + hh * 32 + c, ov + c);
      tmem_ld_wait();
      const float inv = (got && tot > 0.f) ? 1.0f / tot : 0.f;
      if (q0 + row < L) {
        uint4* dst = reinterpret_cast<uint4*>(out + (long long)(s0 + q0 + row) * (H * 64) + h * 64 + hh * 32);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float t8[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) t8[i] = ov[8 * c + i] * inv;
          dst[c] = pack8_16<KIND>(t8);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, FA_TMEM_COLS);
}

template <int KIND>
static cudaError_t launch_fa(const CUtensorMap& tm_qkv, const int* cu, int n_seg, int max_seg, int H, bf16* out,
                             int* status, unsigned long long limit_ns, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(attention_fa_kernel<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize, FA_SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attention_fa_kernel<KIND>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  dim3 grid((max_seg + 127) / 128, n_seg, H);
  return launch_pdl(attention_fa_kernel<KIND>, grid, dim3(FA_THREADS), FA_SMEM, st, tm_qkv, cu, H, out, status, limit_ns);
}

// out: bf16, or f16 with f16 != 0.
cudaError_t launch_attention_fa(const CUtensorMap& tm_qkv, const int* cu, int n_seg, int max_seg, int H, void* out,
                                int* status, unsigned long long limit_ns, bool f16, cudaStream_t st) {
  if (n_seg <= 0 || max_seg <= 0 || H <= 0) return cudaErrorInvalidValue;
  bf16* o = static_cast<bf16*>(out);
  return f16 ? launch_fa<KIND_F16>(tm_qkv, cu, n_seg, max_seg, H, o, status, limit_ns, st)
             : launch_fa<KIND_BF16>(tm_qkv, cu, n_seg, max_seg, H, o, status, limit_ns, st);
}

}  // namespace asr

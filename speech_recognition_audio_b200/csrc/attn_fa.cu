// Attention over long segments on the tcgen05 tensor cores: the full
// (unwindowed) attention of the whisper-small variant ("CrisperWhisper ->
// ONNX", What this exports instead: whisper-small geometry; Results: 1500
// encoder frames per 30 s window), and any segment longer than the 128
// tokens the one-tile kernel of attn_tc.cu takes.
//
// One CTA per (128-query tile, segment, head), 6 warps:
//   warp 4  TMA producer: Q once, then K_j and V_j (128 keys x 64 dims, one
//           buffer each) as soon as the previous tile's MMA has read them;
//   warp 5  MMA issuer: S = Q K_j^T (M=128, N=128, K=64) into tensor memory,
//           issued for tile j+1 while the softmax of tile j runs, then
//           O += P_j V_j (M=128, N=64, K=128) with O kept in tensor memory;
//   warps 0-3  softmax, one query row per thread: load the row of S, mask
//           keys past the segment, online softmax in base 2 with the scale
//           1/sqrt(64) folded in.  The running maximum used for the
//           exponentials moves only when a tile's maximum exceeds it by
//           more than 8 (then O and the row sum are rescaled by
//           2^(old - new)), so probabilities stay <= 256 and most tiles need
//           no rescale.  P (bf16 or f16, the operands' type) goes to shared
//           memory as the A operand of the next MMA; at the end each thread
//           divides its O row by its sum and stores it.
// Tensor memory: S in columns 0..127, O in 128..191 (256 allocated: two
// CTAs per SM).  Shared memory: Q, K, V (16 KB each), P (32 KB).  Every wait
// is bounded; tensor memory is freed after all MMAs have completed.
#include "kernels.h"

namespace asr {

namespace {
constexpr int FA_THREADS = 192;
constexpr int FA_SQ = 0, FA_SK = 16384, FA_SV = 32768, FA_SP = 49152;  // P: two 64-key halves of 16 KB
constexpr int FA_TILES = 81920;
constexpr int FA_BARS = FA_TILES;                                    // 10 barriers + TMEM slot
constexpr int FA_SMEM = 1024 + FA_TILES + 128;
constexpr int FA_TMEM_COLS = 256;
constexpr int FA_O_COL = 128;
constexpr float FA_RESCALE_LOG2 = 8.0f;

enum { B_Q = 0, B_KF, B_KE, B_VF, B_VE, B_SF, B_SFREE, B_PF, B_OD, B_DRAIN, B_COUNT };

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15]))
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
}  // namespace

template <int KIND>
__global__ void __launch_bounds__(FA_THREADS, 2) attention_fa_kernel(const __grid_constant__ CUtensorMap tm_qkv,
                                                                     const int* __restrict__ cu, int H,
                                                                     bf16* __restrict__ out, int* status,
                                                                     unsigned long long limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + FA_BARS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + B_COUNT);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qt = blockIdx.x, seg = blockIdx.y, h = blockIdx.z;

  if (tid == 0) {
    mbar_init(&bar[B_Q], 1);
    mbar_init(&bar[B_KF], 1);
    mbar_init(&bar[B_KE], 1);
    mbar_init(&bar[B_VF], 1);
    mbar_init(&bar[B_VE], 1);
    mbar_init(&bar[B_SF], 1);
    mbar_init(&bar[B_SFREE], 4);
    mbar_init(&bar[B_PF], 4);
    mbar_init(&bar[B_OD], 1);
    mbar_init(&bar[B_DRAIN], 1);
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
    if (warp == 4) {
      // ------------------------------------------------ TMA producer
      if (lane == 0) {
        bool ok = true;
        int issued_k = 0, issued_v = 0;
        mbar_arrive_expect_tx(&bar[B_Q], 16384);
        tma_load_2d(sm + FA_SQ, &tm_qkv, &bar[B_Q], h * 64, s0 + q0);
        for (int j = 0; j < nk && ok; ++j) {
          if (j > 0 && !(ok = mbar_wait_bounded(&bar[B_KE], (j - 1) & 1, limit_ns, status, DEV_TIMEOUT_PRODUCER))) break;
          mbar_arrive_expect_tx(&bar[B_KF], 16384);
          tma_load_2d(sm + FA_SK, &tm_qkv, &bar[B_KF], (H + h) * 64, s0 + j * 128);
          ++issued_k;
          if (j > 0 && !(ok = mbar_wait_bounded(&bar[B_VE], (j - 1) & 1, limit_ns, status, DEV_TIMEOUT_PRODUCER))) break;
          mbar_arrive_expect_tx(&bar[B_VF], 16384);
          tma_load_2d(sm + FA_SV, &tm_qkv, &bar[B_VF], (2 * H + h) * 64, s0 + j * 128);
          ++issued_v;
        }
        // every issued load lands before the CTA exits
        mbar_wait_bounded(&bar[B_Q], 0, kDrainLimitNs, nullptr, 0);
        if (issued_k) mbar_wait_bounded(&bar[B_KF], (issued_k - 1) & 1, kDrainLimitNs, nullptr, 0);
        if (issued_v) mbar_wait_bounded(&bar[B_VF], (issued_v - 1) & 1, kDrainLimitNs, nullptr, 0);
      }
    } else if (warp == 5) {
      // ------------------------------------------------ MMA issuer
      if (lane == 0) {
        const uint32_t idesc_s = idesc_kind_f32(KIND, 128, 128);
        const uint32_t idesc_o = idesc_kind_f32(KIND, 128, 64) | (1u << 16);  // B = V, MN-major
        const uint64_t qd = sw128_kmajor_desc(smem_u32(sm + FA_SQ));
        const uint64_t kd = sw128_kmajor_desc(smem_u32(sm + FA_SK));
        const uint64_t vd = sw128_mnmajor_desc(smem_u32(sm + FA_SV));
        bool ok = mbar_wait_bounded(&bar[B_Q], 0, limit_ns, status, DEV_TIMEOUT_MMA) &&
                  mbar_wait_bounded(&bar[B_KF], 0, limit_ns, status, DEV_TIMEOUT_MMA);
        if (ok) {
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 4; ++k) tc_mma_bf16(tmem, qd + 2 * k, kd + 2 * k, idesc_s, k > 0 ? 1u : 0u);
          tc_commit(&bar[B_SF]);
          tc_commit(&bar[B_KE]);
        }
        for (int j = 0; j < nk && ok; ++j) {
          if (j + 1 < nk) {
            // S for the next tile once its K has landed and the softmax has read S_j
            ok = mbar_wait_bounded(&bar[B_KF], (j + 1) & 1, limit_ns, status, DEV_TIMEOUT_MMA) &&
                 mbar_wait_bounded(&bar[B_SFREE], j & 1, limit_ns, status, DEV_TIMEOUT_MMA);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 4; ++k) tc_mma_bf16(tmem, qd + 2 * k, kd + 2 * k, idesc_s, k > 0 ? 1u : 0u);
            tc_commit(&bar[B_SF]);
            tc_commit(&bar[B_KE]);
          }
          ok = mbar_wait_bounded(&bar[B_PF], j & 1, limit_ns, status, DEV_TIMEOUT_MMA) &&
               mbar_wait_bounded(&bar[B_VF], j & 1, limit_ns, status, DEV_TIMEOUT_MMA);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kb = 0; kb < 2; ++kb) {
            const uint64_t pd = sw128_kmajor_desc(smem_u32(sm + FA_SP + kb * 16384));
#pragma unroll
            for (int k = 0; k < 4; ++k)
              tc_mma_bf16(tmem + FA_O_COL, pd + 2 * k, vd + (uint64_t)((kb * 4 + k) * 128), idesc_o,
                          (j > 0 || kb > 0 || k > 0) ? 1u : 0u);
          }
          tc_commit(&bar[B_OD]);
          tc_commit(&bar[B_VE]);
        }
        // all issued MMAs complete before tensor memory is released
        tc_commit(&bar[B_DRAIN]);
        mbar_wait_bounded(&bar[B_DRAIN], 0, kDrainLimitNs, nullptr, 0);
      }
    } else {
      // ------------------------------------------------ softmax (warps 0-3)
      const int row = warp * 32 + lane;
      const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);
      const float sl2 = 0.125f * 1.4426950408889634f;  // (1 / sqrt(64)) log2(e)
      float m_used = -INFINITY, lsum = 0.f;
      bool ok = true;
      for (int j = 0; j < nk; ++j) {
        ok = mbar_wait_bounded(&bar[B_SF], j & 1, limit_ns, status, DEV_TIMEOUT_EPILOGUE);
        tc_fence_after();
        float sv[128];
#pragma unroll
        for (int c = 0; c < 128; c += 16) tmem_ld16(trow + c, sv + c);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[B_SFREE]);
        const int kv = min(128, L - j * 128);  // valid keys in this tile (>= 1)
        // tile maximum of the raw scores (four chains; only a partial last
        // tile needs the per-key mask); the scale is positive, so
        // max(s) * scale = max(s * scale)
        float m8[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) m8[i] = -INFINITY;
        if (kv == 128) {
#pragma unroll
          for (int c = 0; c < 128; ++c) m8[c & 3] = fmaxf(m8[c & 3], sv[c]);
        } else {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c < kv) m8[c & 3] = fmaxf(m8[c & 3], sv[c]);
        }
        float mt = fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3]));
        mt = ok ? mt * sl2 : 0.f;
        // P_j may overwrite P_{j-1} and O may be rescaled once O_{j-1} is complete
        if (j > 0) ok = mbar_wait_bounded(&bar[B_OD], (j - 1) & 1, limit_ns, status, DEV_TIMEOUT_EPILOGUE) && ok;
        tc_fence_after();
        const bool grow = mt > m_used + FA_RESCALE_LOG2;
        if (j == 0) {
          m_used = mt;
        } else if (__any_sync(0xffffffffu, grow)) {
          const float corr = grow ? ex2_approx(m_used - mt) : 1.0f;
          if (grow) {
            m_used = mt;
            lsum *= corr;
          }
#pragma unroll
          for (int c = 0; c < 64; c += 16) {
            float ov[16];
            tmem_ld16(trow + FA_O_COL + c, ov);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) ov[i] *= corr;
            tmem_st16(trow + FA_O_COL + c, ov);
          }
          tmem_st_wait();
        }
        // p = 2^((s - m) / 8 log2 e) as one FMA into ex2.approx
        const float nm = -m_used;
        float s8[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) s8[i] = 0.f;
#pragma unroll
        for (int c = 0; c < 128; c += 16) {
          if (c < kv && ok) {  // uniform: 16-key chunks wholly past the segment stay zero
#pragma unroll
            for (int i = c; i < c + 16; ++i) {
              sv[i] = (i < kv) ? ex2_approx(fmaf(sv[i], sl2, nm)) : 0.f;
              s8[i & 3] += sv[i];
            }
          } else {
#pragma unroll
            for (int i = c; i < c + 16; ++i) sv[i] = 0.f;
          }
        }
        lsum += (s8[0] + s8[1]) + (s8[2] + s8[3]);
        // P row into two 64-key halves, 16-byte chunks swizzled by (row & 7)
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
          uint4* prow = reinterpret_cast<uint4*>(sm + FA_SP + kb * 16384 + row * 128);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            prow[c ^ (row & 7)] = pack8_16<KIND>(sv + kb * 64 + c * 8);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[B_PF]);
        if (!ok) break;
      }
      // epilogue: O / sum
      const bool got = ok && mbar_wait_bounded(&bar[B_OD], (nk - 1) & 1, limit_ns, status, DEV_TIMEOUT_EPILOGUE);
      tc_fence_after();
      float ov[64];
#pragma unroll
      for (int c = 0; c < 64; c += 16) tmem_ld16(trow + FA_O_COL + c, ov + c);
      tmem_ld_wait();
      const float inv = (got && lsum > 0.f) ? 1.0f / lsum : 0.f;
      if (q0 + row < L) {
        uint4* dst = reinterpret_cast<uint4*>(out + (long long)(s0 + q0 + row) * (H * 64) + h * 64);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
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

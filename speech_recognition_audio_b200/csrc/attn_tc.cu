// Windowed attention on the tcgen05 tensor cores, for segments of at most
// 128 tokens (the 104-token windows of "MOSS-Transcribe-preview-2B-GGUF",
// Architecture "Audio encoder": windowed, block-diagonal attention).
//
// One CTA (4 warps) per (segment, head):
//   - thread 0 TMA-loads Q and K of the head as 128-row boxes starting at the
//     segment's first token (rows past the segment belong to the next
//     segment or lie outside the tensor: their scores are masked and their
//     probabilities are zero);
//   - V comes by TMA too (keys x dims) and serves as the MN-major B operand
//     of P V (rows past the segment meet zero probabilities);
//   - S = Q K^T: tcgen05.mma M=128 N=128 K=64 into tensor memory;
//   - each thread owns one query row: tcgen05.ld of its 128 scores, the
//     maximum over keys < L, then exp2 of (s - max) / 8 log2 e as one FMA
//     into ex2.approx (packed pair FMAs over whole 16-key chunks, per-key
//     masks only in the chunk that holds L) and the sum, in independent
//     chains;
//     P (bf16, or f16 for f16 operands) is written row-major, swizzled, over
//     the Q and K tiles as the A operand of the next MMA;
//   - O = P V: tcgen05.mma M=128 N=64 K=128 into S's tensor-memory columns;
//   48 KB of shared memory and 128 TMEM columns per block: 4 blocks per SM.
//   - each thread scales its output row by 1 / sum and stores 128 bytes.
// Every barrier wait is bounded (status word); tensor memory is freed after
// all MMAs have completed.
#include "kernels.h"

namespace asr {

namespace {
constexpr int AT_THREADS = 128;
// smem: Q and K (16 KB each), later overwritten by P (2 x 16 KB); V (16 KB)
constexpr int SQ = 0, SK = 16384, SP = 0, SV = 32768;
constexpr int AT_SMEM = 1024 + 49152 + 64;  // tiles + barriers + TMEM slot
constexpr int AT_TMEM_COLS = 128;           // S (128 columns), then O (64) in the same columns
}  // namespace

template <int KIND>
__global__ void __launch_bounds__(AT_THREADS, 3) attention_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv,
                                                                   const bf16* __restrict__ qkv,
                                                                   const int* __restrict__ cu, int H,
                                                                   bf16* __restrict__ out, int* status,
                                                                   unsigned long long limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + 49152);
  uint64_t* bar_qk = bars;
  uint64_t* bar_s = bars + 1;
  uint64_t* bar_o = bars + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int seg = blockIdx.x, h = blockIdx.y;

  if (tid == 0) {
    mbar_init(bar_qk, 1);
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_qkv);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, AT_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();
  pdl_trigger();

  const int s0 = cu[seg], L = cu[seg + 1] - s0;
  bool ok = true;
  if (tid == 0) {
    mbar_arrive_expect_tx(bar_qk, 3 * 16384);
    tma_load_2d(sm + SQ, &tm_qkv, bar_qk, h * 64, s0);
    tma_load_2d(sm + SK, &tm_qkv, bar_qk, (H + h) * 64, s0);
    tma_load_2d(sm + SV, &tm_qkv, bar_qk, (2 * H + h) * 64, s0);  // keys x dims: the MN-major B of P V
  }
  // S = Q K^T
  if (tid == 0) {
    ok = mbar_wait_bounded(bar_qk, 0, limit_ns, status, DEV_TIMEOUT_MMA);
    if (ok) {
      tc_fence_after();
      const uint32_t idesc = idesc_kind_f32(KIND, 128, 128);
      const uint64_t ad = sw128_kmajor_desc(smem_u32(sm + SQ)), bd = sw128_kmajor_desc(smem_u32(sm + SK));
#pragma unroll
      for (int k = 0; k < 4; ++k) tc_mma_bf16(tmem, ad + 2 * k, bd + 2 * k, idesc, k > 0 ? 1u : 0u);
    }
    tc_commit(bar_s);
  }
  // softmax of this thread's row
  float rsum = 1.f;
  {
    const bool got = mbar_wait_bounded(bar_s, 0, limit_ns, status, DEV_TIMEOUT_EPILOGUE);
    tc_fence_after();
    const int row = warp * 32 + lane;
    const uint32_t taddr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    float sv[128];
#pragma unroll
    for (int c = 0; c < 128; c += 16) tmem_ld16(taddr + c, sv + c);
    tmem_ld_wait();
    const float sl2 = 0.125f * 1.4426950408889634f;
    // row maximum over keys < L (four independent chains; only the 16-key
    // chunk that holds L needs a per-key mask)
    float m8[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) m8[i] = -INFINITY;
#pragma unroll
    for (int c = 0; c < 128; c += 16) {
      if (c + 16 <= L) {
#pragma unroll
        for (int j = 0; j < 16; ++j) m8[j & 3] = fmaxf(m8[j & 3], sv[c + j]);
      } else if (c < L) {
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (c + j < L) m8[j & 3] = fmaxf(m8[j & 3], sv[c + j]);
      }
    }
    float mx = fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3]));
    // exp2((s - max) / 8 log2 e) as one FMA into ex2; the scale is positive,
    // so max(s) * scale = max(s * scale)
    const float nm = got ? -mx * sl2 : 0.f;
    // whole 16-key chunks: the argument as a packed pair FMA, the sum in
    // four packed chains; the chunk that holds L masks per key; chunks past
    // the segment stay zero (all tests are uniform across the block)
    const float2 sl2v = make_float2(sl2, sl2), nmv = make_float2(nm, nm);
    float2 s2[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) s2[i] = make_float2(0.f, 0.f);
#pragma unroll
    for (int c = 0; c < 128; c += 16) {
      if (c + 16 <= L && got) {
#pragma unroll
        for (int j = c; j < c + 16; j += 2) {
          const float2 a = fma2(make_float2(sv[j], sv[j + 1]), sl2v, nmv);
          sv[j] = ex2_approx(a.x);
          sv[j + 1] = ex2_approx(a.y);
          s2[(j >> 1) & 3] = add2(s2[(j >> 1) & 3], make_float2(sv[j], sv[j + 1]));
        }
      } else if (c < L && got) {
#pragma unroll
        for (int j = c; j < c + 16; ++j) {
          sv[j] = (j < L) ? ex2_approx(fmaf(sv[j], sl2, nm)) : 0.f;
          s2[(j >> 1) & 3].x += sv[j];
        }
      } else {
#pragma unroll
        for (int j = c; j < c + 16; ++j) sv[j] = 0.f;
      }
    }
    const float s = ((s2[0].x + s2[0].y) + (s2[1].x + s2[1].y)) + ((s2[2].x + s2[2].y) + (s2[3].x + s2[3].y));
    rsum = s > 0.f ? 1.f / s : 0.f;
    // P overwrites Q and K: every thread has passed bar_s, so the MMA that
    // read them is complete.
    __syncthreads();
    fence_proxy_async_smem();
    // P row into two 64-key blocks, 16-byte chunks swizzled by (row & 7)
#pragma unroll
    for (int kb = 0; kb < 2; ++kb) {
      uint4* prow = reinterpret_cast<uint4*>(sm + SP + kb * 16384 + row * 128);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        prow[c ^ (row & 7)] = pack8_16<KIND>(sv + kb * 64 + c * 8);
      }
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  // O = P V
  if (tid == 0) {
    tc_fence_after();
    if (ok) {
      // B = V stored keys x dims (dims contiguous): MN-major, 128-byte swizzle,
      // 8-key groups 1024 bytes apart; each K=16 step advances 16 keys (2048 B).
      const uint32_t idesc = idesc_kind_f32(KIND, 128, 64) | (1u << 16);
      const uint64_t bd0 = sw128_mnmajor_desc(smem_u32(sm + SV));
#pragma unroll
      for (int kb = 0; kb < 2; ++kb) {
        const uint64_t ad = sw128_kmajor_desc(smem_u32(sm + SP + kb * 16384));
#pragma unroll
        for (int k = 0; k < 4; ++k)
          tc_mma_bf16(tmem, ad + 2 * k, bd0 + (uint64_t)((kb * 4 + k) * 128), idesc, (kb > 0 || k > 0) ? 1u : 0u);
      }
    }
    tc_commit(bar_o);
  }
  {
    mbar_wait_bounded(bar_o, 0, limit_ns, status, DEV_TIMEOUT_EPILOGUE);
    tc_fence_after();
    const int row = warp * 32 + lane;
    const uint32_t taddr = tmem + (static_cast<uint32_t>(warp * 32) << 16);  // O reuses S's columns
    float ov[64];
#pragma unroll
    for (int c = 0; c < 64; c += 16) tmem_ld16(taddr + c, ov + c);
    tmem_ld_wait();
    if (row < L) {
      uint4* dst = reinterpret_cast<uint4*>(out + (long long)(s0 + row) * (H * 64) + h * 64);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float t8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) t8[i] = ov[8 * c + i] * rsum;
        dst[c] = pack8_16<KIND>(t8);
      }
    }
  }
  // Both MMA groups have completed (bar_o covers all of thread 0's MMAs); after
  // a failed wait the Q/K loads may still be in flight: let them land.
  if (tid == 0 && !ok) mbar_wait_bounded(bar_qk, 0, kDrainLimitNs, nullptr, 0);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, AT_TMEM_COLS);
}

bool make_tmap_qkv(CUtensorMap* map, const void* qkv, long long T, int H) {
  return make_tmap_bf16(map, qkv, (unsigned long long)T, 3ULL * H * 64, 3ULL * H * 64, 128);
}

template <int KIND>
static cudaError_t launch_tc(const CUtensorMap& tm_qkv, const bf16* qkv, const int* cu, int n_seg, int H, bf16* out,
                             int* status, unsigned long long limit_ns, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(attention_tc_kernel<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize, AT_SMEM);
  // Ask for the whole shared-memory carveout: without it the driver picked a
  // 164 KB configuration (3 blocks per SM, 2.7 waves for 1200 blocks).
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attention_tc_kernel<KIND>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  return launch_pdl(attention_tc_kernel<KIND>, dim3(n_seg, H), dim3(AT_THREADS), AT_SMEM, st, tm_qkv, qkv, cu, H, out,
                    status, limit_ns);
}

// qkv / out: bf16, or f16 with f16 != 0 (the bytes pass through TMA as they are).
cudaError_t launch_attention_tc(const CUtensorMap& tm_qkv, const void* qkv, const int* cu, int n_seg, int H, void* out,
                                int* status, unsigned long long limit_ns, bool f16, cudaStream_t st) {
  const bf16* q = static_cast<const bf16*>(qkv);
  bf16* o = static_cast<bf16*>(out);
  return f16 ? launch_tc<KIND_F16>(tm_qkv, q, cu, n_seg, H, o, status, limit_ns, st)
             : launch_tc<KIND_BF16>(tm_qkv, q, cu, n_seg, H, o, status, limit_ns, st);
}

}  // namespace asr

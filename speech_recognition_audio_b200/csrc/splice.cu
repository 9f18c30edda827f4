// Audio injection ("MOSS-Transcribe-preview-2B-GGUF", Architecture table,
// "Audio injection" and "Prompt" rows): the LLM's input embeddings for a
// tokenised prompt are the token embeddings, except at the audio placeholder
// positions, whose rows are replaced, in order, by the adapter's output
// frames.
//
// Two kernels:
//   splice_rank_kernel   one block: exclusive count of placeholders before
//                        each position (the frame that position receives)
//                        and the total, checked against the frame count;
//   splice_gather_kernel one warp per output row: 16-byte copies of the
//                        token's table row, or the frame converted to the
//                        output type (round to nearest even).
// Ids outside [0, vocab) and a placeholder count that differs from the
// frame count are reported in the status word; the affected rows are zero.
#include "kernels.h"

namespace asr {

namespace {

constexpr int RANK_THREADS = 1024;

__device__ __forceinline__ float load_elem(const void* base, long long i, int dtype) {
  if (dtype == SPLICE_F32) return reinterpret_cast<const float*>(base)[i];
  if (dtype == SPLICE_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[i]);
  return __half2float(reinterpret_cast<const __half*>(base)[i]);
}
__device__ __forceinline__ void store_elem(void* base, long long i, int dtype, float v) {
  if (dtype == SPLICE_F32) reinterpret_cast<float*>(base)[i] = v;
  else if (dtype == SPLICE_BF16) reinterpret_cast<__nv_bfloat16*>(base)[i] = __float2bfloat16_rn(v);
  else reinterpret_cast<__half*>(base)[i] = __float2half_rn(v);
}

}  // namespace

// Exclusive placeholder count per position, in chunks of 1024 with a carry.
__global__ void __launch_bounds__(RANK_THREADS) splice_rank_kernel(const int* __restrict__ ids, long long n_ids,
                                                                   int placeholder, long long n_frames,
                                                                   int* __restrict__ rank, int* __restrict__ status) {
  __shared__ int warp_sums[RANK_THREADS / 32];
  __shared__ long long carry;
  pdl_wait();
  pdl_trigger();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (long long base = 0; base < n_ids; base += RANK_THREADS) {
    const long long i = base + tid;
    const int flag = (i < n_ids && ids[i] == placeholder) ? 1 : 0;
    // inclusive scan within the warp, then over the warp totals
    int v = flag;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    if (lane == 31) warp_sums[warp] = v;
    __syncthreads();
    if (warp == 0) {
      int w = warp_sums[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      warp_sums[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    const long long before = carry + (warp ? warp_sums[warp - 1] : 0) + (v - flag);
    if (i < n_ids) rank[i] = flag ? static_cast<int>(before) : -1;
    __syncthreads();
    if (tid == 0) carry += warp_sums[RANK_THREADS / 32 - 1];
    __syncthreads();
  }
  if (tid == 0 && carry != n_frames) atomicCAS(status, 0, SPLICE_E_COUNT);
}

__global__ void __launch_bounds__(256) splice_gather_kernel(const int* __restrict__ ids, const int* __restrict__ rank,
                                                            long long n_ids, const void* __restrict__ table, int vocab,
                                                            int table_dtype, const float* __restrict__ frames,
                                                            long long n_frames, int D, void* __restrict__ out,
                                                            int out_dtype, int* __restrict__ status) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long row = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5); row < n_ids; row += warps) {
    const int rk = rank[row];
    const long long o = row * D;
    if (rk >= 0) {
      const bool ok = rk < n_frames;
      if (!ok && lane == 0) atomicCAS(status, 0, SPLICE_E_COUNT);
      const float* f = frames + (long long)rk * D;
      for (int c = lane; c < D; c += 32) store_elem(out, o + c, out_dtype, ok ? f[c] : 0.0f);
      continue;
    }
    const int id = ids[row];
    if (id < 0 || id >= vocab) {
      if (lane == 0) atomicCAS(status, 0, SPLICE_E_ID);
      for (int c = lane; c < D; c += 32) store_elem(out, o + c, out_dtype, 0.0f);
      continue;
    }
    const int es = table_dtype == SPLICE_F32 ? 4 : 2;
    const char* src = reinterpret_cast<const char*>(table) + (long long)id * D * es;
    if (table_dtype == out_dtype && ((long long)D * es) % 16 == 0 &&
        (reinterpret_cast<uintptr_t>(table) & 15) == 0 && (reinterpret_cast<uintptr_t>(out) & 15) == 0) {
      // same type: the row is copied bit for bit, 16 bytes per lane
      const uint4* s4 = reinterpret_cast<const uint4*>(src);
      uint4* d4 = reinterpret_cast<uint4*>(reinterpret_cast<char*>(out) + o * es);
      for (int c = lane; c < D * es / 16; c += 32) d4[c] = s4[c];
    } else {
      for (int c = lane; c < D; c += 32) store_elem(out, o + c, out_dtype, load_elem(table, (long long)id * D + c, table_dtype));
    }
  }
}

cudaError_t launch_splice(const int* ids, long long n_ids, int placeholder, const void* table, int vocab,
                          int table_dtype, const float* frames, long long n_frames, int D, void* out, int out_dtype,
                          int* rank, int* status, int num_sms, cudaStream_t st) {
  cudaError_t e = launch_pdl(splice_rank_kernel, dim3(1), dim3(RANK_THREADS), 0, st, ids, n_ids, placeholder, n_frames,
                             rank, status);
  if (e != cudaSuccess) return e;
  const long long blocks = std::min<long long>((n_ids + 7) / 8, 4LL * num_sms);
  return launch_pdl(splice_gather_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, ids,
                    static_cast<const int*>(rank), n_ids, table, vocab, table_dtype, frames, n_frames, D, out,
                    out_dtype, status);
}

}  // namespace asr

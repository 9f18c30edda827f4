// tcgen05 GEMM engine for sm_100a: D[M,N] = A[M,K] * B[N,K]^T, bf16 inputs,
// fp32 accumulation in tensor memory, fused epilogues.
//
// Every dense contraction of the encoder runs here: the conv stem as an
// implicit GEMM (A gathered from the NHWC activation by cp.async warps), the
// conv_out projection with the sinusoidal positions, the QKV / output / FFN
// projections of each pre-LN layer with bias, GELU and residual epilogues,
// and the head and SwiGLU adapter projections ("MOSS-Transcribe-preview-2B-
// GGUF", Architecture table: "Audio encoder", "Conv front-end", "Encoder
// head", "Adapter" rows).
//
// Structure (one persistent CTA per SM, static round-robin over 128 x BN
// output tiles):
//   warp 0      TMA producer: B tiles (and A tiles when A is a plain matrix)
//               into a STAGES-deep ring of 128-byte-swizzled smem buffers.
//   warp 1      allocates tensor memory; lane 0 issues tcgen05.mma
//               (M=128, N=BN, K=16) and commits to the ring's "empty"
//               barriers and, per tile, to an accumulator "full" barrier.
//   warps 2-9   epilogue: tcgen05.ld the accumulator (a warp may only read
//               the 32 TMEM lanes of its quarter, warp % 4; two warps share
//               each quarter and take alternate 32-column groups), apply
//               bias / GELU / SwiGLU, transpose through a per-warp shared
//               buffer, add positions / the residual and store with
//               coalesced accesses, release the accumulator.  Two
//               accumulators in TMEM let the epilogue of tile i overlap the
//               MMAs of tile i+1.
//   warps 10-17 (implicit-GEMM mode only) gather the A tile with 16-byte
//               cp.async (zero fill for padding and tails) into the same
//               swizzled layout; each thread's copies arrive on the stage's
//               full barrier when they land (cp.async.mbarrier.arrive.noinc),
//               and the MMA thread fences the async proxy before reading.
// All waits are bounded (globaltimer); a role that gives up records a status
// code, and the CTA drains its in-flight copies and MMAs before freeing
// tensor memory and exiting.
#pragma once

#include "common.cuh"

namespace asr {

// EPI_LN (with EPI_RESID, CTA-pair tiles): the residual update is followed
// by the LayerNorm of the updated rows, written as a second 16-bit output.
enum : int { EPI_GELU = 1, EPI_OUT_F32 = 2, EPI_RESID = 4, EPI_PE = 8, EPI_SWIGLU = 16, EPI_LN = 32 };

struct ConvGather {
  const bf16* x;  // activation [n_img, T_in, F_in, C] (C innermost)
  int T_in, F_in, C;
  int T_out, F_out;
  int st, sf;     // strides along T and F
  int kt, kf;     // kernel extents
  int pt, pf;     // zero padding
};

// Convolution A operand read by TMA as strided boxes: the activation is
// [n_img, T_in, F_in, C] (C innermost) and a 128-row tile is TR output
// t-rows x all F_out columns of one image; for each tap and 64-channel block
// one 4-D box {64, F_out * sf, TR * st, 1} with element strides {1, sf, st, 1}
// lands the 128 x 64 A tile (zero fill outside the image = the padding).
//
// Phase mode (phase = 1, strides 2 along T and F): the activation is stored
// as its four parity planes [n_img][t % 2][f % 2][T_in / 2][F_in / 2][C], so
// the input rows a tap reads for consecutive outputs are consecutive in
// one plane and each box is dense ({64, F_out, TR, 1}, no element strides).
struct ConvBox {
  int TR, F_out, T_out;   // output rows per tile, output geometry
  int tiles_per_img;      // ceil(T_out / TR)
  int n_sub;              // n_img * tiles_per_img 128-row sub-tiles
  int st, sf, pt, pf;     // strides and padding along T and F
  int kf, CB;             // taps along F, 64-channel blocks per tap
  int phase;              // 1 = parity-plane input (see above)
  int k16_last;           // K=16 MMA steps holding channels in a tap's last 64-channel block
};

struct GemmParams {
  int M, N, K;
  int m_blocks, n_blocks, k_blocks, num_tiles;
  void* out;
  long long ldo;          // output row stride in elements
  const float* bias;      // [N] or null
  const float* pe;        // [pe_period, N] or null
  int pe_period;
  ConvGather g;
  int* status;
  unsigned long long limit_ns;
  int n_fast;             // tile order: 1 = the n-blocks of an m-block run back to back
  int conv_box;           // 1 = A is a ConvBox (4-D strided TMA), rows mapped per image
  ConvBox cb;
  int out_tma;            // 1 = the kernel's output tensor map is valid (TMA store epilogue)
  // Stream-K (CTA-pair kernel, residual epilogue): the num_tiles x k_blocks
  // (tile, k-block) units are cut into equal contiguous ranges, one per CTA
  // pair, so that no pair idles in a partial last wave.  A tile split
  // between two pairs is a trailing piece (the first piece of the later
  // pair: its partial sum goes into the residual stream, then one flag per
  // epilogue warp is raised) and a leading piece (the owner, which adds the
  // bias: it waits for the flag before its own residual update), so every
  // element sees the same additions in the same order on every run.
  int sk;
  int* sk_flags;          // [pairs][2 CTAs][8 warps], zero before the launch
  int k_full;             // 1 = every k-block holds four whole MMA steps (set by the launcher)
  // Output rows r with r % zero_period >= zero_from are written as zeros
  // (the padding rows of a packed convolution layout); zero_period 0 = none.
  int zero_period, zero_from;
  // Residual + LayerNorm epilogue (EPI_LN): gamma, beta [N] and epsilon of
  // the norm, its 16-bit output ln_h [M][ldo]; ln_part holds ln_parts
  // partial statistics {count, mean, M2, 0} per row, [part][M] (one per
  // epilogue warp and n-tile covering the row), ln_count one arrival counter
  // per 32-row group: zero before the first launch on the buffer, each
  // launch adds ln_parts to every group's count, and ln_epoch is the number
  // of launches on the buffer before this one.
  const float* ln_gamma;
  const float* ln_beta;
  float ln_eps;
  int ln_parts;
  int* ln_count;
  float* ln_part;
  void* ln_h;
  int ln_epoch;
};

template <bool B>
struct BoolTag {
  static constexpr bool value = B;
};

// Kinds of work piece: a whole tile, the trailing k-blocks of a split tile
// (partial sum added to the residual stream first, without bias), or the
// leading k-blocks of a split tile (adds bias and its sum once the trailing
// piece's update has landed).
enum : int { PIECE_FULL = 0, PIECE_PARTIAL = 1, PIECE_OWNER = 2 };

// The sequence of (tile, k-block range) pieces of one scheduling unit (a CTA
// pair): tiles unit, unit + n_units, ... whole, or under stream-K the unit
// range [total * unit / n_units, total * (unit + 1) / n_units) of the
// row-major (tile, k-block) order.  With num_tiles >= n_units every range
// spans at least one tile's k-blocks, so a tile is split at most once:
// its trailing part is the first piece of unit + 1.
struct PieceIter {
  long long u, u_end;
  int t, step;
  __device__ __forceinline__ PieceIter(const GemmParams& p, int unit, int n_units) : u(0), u_end(0), t(unit), step(n_units) {
    if (p.sk) {
      const long long total = (long long)p.num_tiles * p.k_blocks;
      u = total * unit / n_units;
      u_end = total * (unit + 1) / n_units;
    }
  }
  __device__ __forceinline__ bool next(const GemmParams& p, int& tile, int& kb0, int& kb1) {
    if (!p.sk) {
      if (t >= p.num_tiles) return false;
      tile = t;
      kb0 = 0;
      kb1 = p.k_blocks;
      t += step;
      return true;
    }
    if (u >= u_end) return false;
    tile = static_cast<int>(u / p.k_blocks);
    kb0 = static_cast<int>(u - (long long)tile * p.k_blocks);
    const long long left = u_end - u;
    kb1 = left < p.k_blocks - kb0 ? kb0 + static_cast<int>(left) : p.k_blocks;
    u += kb1 - kb0;
    return true;
  }
};
__device__ __forceinline__ int piece_kind(const GemmParams& p, int kb0, int kb1) {
  return kb0 > 0 ? PIECE_PARTIAL : (kb1 < p.k_blocks ? PIECE_OWNER : PIECE_FULL);
}

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_gpu(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Orders this thread's global accesses of the async proxy (bulk tensor
// copies) with its generic-proxy accesses, in both directions.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
// Wait (one thread) until *flag != 0, for at most limit_ns; gives up early
// when the status word already holds an error.
static __device__ __noinline__ bool flag_wait_bounded(const int* flag, uint64_t limit_ns, int* status, int code) {
  if (ld_acquire_gpu(flag) != 0) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0;; ++it) {
    __nanosleep(64);
    if (ld_acquire_gpu(flag) != 0) return true;
    if ((it & 15) == 15) {
      if (globaltimer_ns() - t0 > limit_ns) {
        if (status) atomicCAS(status, 0, code);
        return false;
      }
      if (status && *reinterpret_cast<volatile int*>(status) != 0) return false;
    }
  }
}

// Wait (one thread) until *count >= target, for at most limit_ns; gives up
// early when the status word already holds an error.
static __device__ __noinline__ bool count_wait_bounded(const int* count, int target, uint64_t limit_ns, int* status,
                                                       int code) {
  if (ld_acquire_gpu(count) >= target) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0;; ++it) {
    __nanosleep(32);
    if (ld_acquire_gpu(count) >= target) return true;
    if ((it & 15) == 15) {
      if (globaltimer_ns() - t0 > limit_ns) {
        if (status) atomicCAS(status, 0, code);
        return false;
      }
      if (status && *reinterpret_cast<volatile int*>(status) != 0) return false;
    }
  }
}
__device__ __forceinline__ void red_add_release_gpu(int* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ float4 ld_relaxed_gpu_f4(const float* p) {
  float4 v;
  asm volatile("ld.relaxed.gpu.global.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p)
               : "memory");
  return v;
}

// Output rows covered by 128-row sub-tile u: [first, last) (conv-box mode
// maps a sub-tile to TR output t-rows of one image; rows past the image end
// are padding).  Plain mode: rows u*128 .. u*128+127 clipped at M.
__device__ __forceinline__ void subtile_rows(const GemmParams& p, int u, int& first, int& last) {
  if (p.conv_box) {
    const ConvBox& c = p.cb;
    if (u >= c.n_sub) {
      first = last = 0;
      return;
    }
    const int img = u / c.tiles_per_img, tb = u - img * c.tiles_per_img;
    const int rows = min(c.TR, c.T_out - tb * c.TR) * c.F_out;
    first = img * c.T_out * c.F_out + tb * c.TR * c.F_out;
    last = first + rows;
  } else {
    first = u * 128;
    last = min(first + 128, p.M);
  }
}

// TMA coordinates of the A tile of sub-tile u at k-block kb (conv-box mode).
__device__ __forceinline__ void convbox_coords(const GemmParams& p, int u, int kb, int& c0, int& f0, int& t0, int& img,
                                               int BK = 64) {
  const ConvBox& c = p.cb;
  const int uu = u < c.n_sub ? u : c.n_sub - 1;  // past the end: any valid box, rows are masked
  img = uu / c.tiles_per_img;
  const int tb = uu - img * c.tiles_per_img;
  const int tap = kb / c.CB;
  const int cbk = kb - tap * c.CB;
  const int dt = tap / c.kf, df = tap - dt * c.kf;
  c0 = cbk * BK;
  if (c.phase) {
    // input index 2 o + d - p lies in plane (d - p) & 1 at o + ((d - p) >> 1)
    const int at = dt - c.pt, af = df - c.pf;
    f0 = af >> 1;
    t0 = tb * c.TR + (at >> 1);
    img = img * 4 + (at & 1) * 2 + (af & 1);
  } else {
    f0 = df - c.pf;
    t0 = tb * c.TR * c.st + dt - c.pt;
  }
  if (u >= c.n_sub) t0 = 1 << 20;  // entirely outside: zero tile
}

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1, int c2,
                                            int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

// Tile t -> (m block, n block).  With n_fast the tiles that share A rows run
// on neighbouring CTAs at the same time, so A (the gathered activation of a
// convolution) is fetched from DRAM once and re-read from L2.
__device__ __forceinline__ void tile_coords(const GemmParams& p, int t, int& mb, int& nb) {
  if (p.n_fast) {
    nb = t % p.n_blocks;
    mb = t / p.n_blocks;
  } else {
    mb = t % p.m_blocks;
    nb = t / p.m_blocks;
  }
}

static constexpr unsigned long long kDrainLimitNs = 200ull * 1000 * 1000;

// K=16 MMA steps of k-block kb that hold non-zero operands: 4, except in a
// k-block past the end of K (plain mode) or in the last channel block of a
// tap when the channel count is not a multiple of 64 (conv-box mode), whose
// zero-padded tail the MMA can skip.
// (BK elements per k-block, 4 MMA steps of BK / 4.)
__device__ __forceinline__ int k16_steps(const GemmParams& p, int kb, int BK = 64) {
  if (p.conv_box) return (kb % p.cb.CB == p.cb.CB - 1) ? p.cb.k16_last : 4;
  const int rem = p.K - kb * BK;
  const int ks = BK / 4;
  return rem >= BK ? 4 : (rem + ks - 1) / ks;
}

template <int BN_, int STAGES_, bool GATHER_, int KIND_ = KIND_BF16>
struct GemmShape {
  static constexpr int KIND = KIND_;
  static constexpr int BM = 128, BN = BN_, BK = kind_row_elems(KIND_), STAGES = STAGES_;
  static constexpr bool GATHER = GATHER_;
  static constexpr int A_BYTES = BM * 128;   // 128-byte rows of BK elements
  static constexpr int B_BYTES = BN * 128;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int ACC_COLS = (BN + 31) / 32 * 32;
  static constexpr int TMEM_COLS =
      2 * ACC_COLS <= 32 ? 32 : 2 * ACC_COLS <= 64 ? 64 : 2 * ACC_COLS <= 128 ? 128 : 2 * ACC_COLS <= 256 ? 256 : 512;
  static constexpr int EPI_WARPS = 8;   // two per TMEM lane quarter, columns split between them
  static constexpr int GATHER_WARPS = GATHER ? 8 : 0;
  static constexpr int THREADS = 32 * (2 + EPI_WARPS + GATHER_WARPS);
  static constexpr int EPI_BUF_BYTES = EPI_WARPS * 4096;   // per-warp transpose buffers
  static constexpr int BAR_BYTES = 8 * (2 * STAGES + 5) + 16;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + EPI_BUF_BYTES + BAR_BYTES;
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N for M=128");
  static_assert(2 * ACC_COLS <= 512, "two accumulators must fit in TMEM");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
  static_assert(!(GATHER_ && KIND_ == KIND_TF32), "the cp.async gather stages 16-bit operands");
};

// Epilogue warps: four per TMEM lane quarter share the accumulator columns
// with 8 warps as two column parts (32-column groups part, part + 2, ...),
// with 16 warps as four (part, part + 4, ...); `cstride` = 32 x parts.
//
// Residual epilogues read 128 x BN fp32 values per tile; issuing L2
// prefetches for the tile's rows before waiting for the accumulator moves that
// DRAM latency under the tile's MMAs.  Each thread prefetches the 128-byte
// lines of its own row in the 32-column groups its warp will handle.
__device__ __forceinline__ void epilogue_prefetch_l2(const GemmParams& p, int t, int half, int q, int lane, int BN,
                                                     int BM, int rank_rows, int cstride = 64) {
  int mb, nb;
  tile_coords(p, t, mb, nb);
  const int m0 = mb * BM + rank_rows;
  const int n0 = nb * BN;
  const int row = m0 + 32 * q + lane;
  if (row >= p.M) return;
  const float* base = reinterpret_cast<const float*>(p.out) + (long long)row * p.ldo + n0;
  for (int c = half * 32; c < BN && n0 + c < p.N; c += cstride)
    asm volatile("prefetch.global.L2 [%0];" ::"l"(base + c) : "memory");
}

// TMA stores from shared memory (bulk-group completion).  The tensor map
// covers the output [rows, cols]; the box is 32 x 32 with the 128-byte
// (fp32) or 64-byte (bf16) swizzle that the epilogue buffer is written in.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}
// out[box] += smem (fp32 add performed at L2): the residual update.
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* map, const void* src, int x, int y) {
  asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Shared-memory sources of this thread's bulk stores may be overwritten.
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// All but the most recent of this thread's bulk stores have read their source.
__device__ __forceinline__ void bulk_wait_read1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
// This thread's bulk stores have completed (written to global memory).
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Bias of the tile's columns for one epilogue warp, loaded before the
// accumulator is ready: lane l holds bias[n0 + c_j + l] for the warp's
// column groups c_j = 32 half + cstride j (the epilogue broadcasts it by
// shuffle).
__device__ __forceinline__ void load_bias(const GemmParams& p, int n0, int BN, int half, int lane, float* breg,
                                          int cstride = 64) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int c = half * 32 + cstride * j;
    const int n = n0 + c + lane;
    breg[j] = (p.bias && c < BN && c + lane < BN && n < p.N) ? __ldg(p.bias + n) : 0.0f;
  }
}

// Epilogue of one warp: its 32 TMEM lanes (tile rows row0..row0+31) over the
// 32-column groups g = half, half + 2, ... of a BN-wide accumulator.
//   phase A (one thread per row): tcgen05.ld 32 columns, add the bias, apply
//     GELU or SwiGLU, and write the row into the warp's 4 KB shared buffer
//     (fp32, or bf16 for bf16 outputs; 16-byte chunks XOR-swizzled by row:
//     the 128-byte / 64-byte swizzle of the TMA store, which also keeps
//     the row-wise writes free of bank conflicts);
//   store: one lane issues a TMA store of the 32 x 32 box (plain outputs) or
//     a TMA reduce-add into the fp32 residual stream, so the warp never
//     waits on global memory; the buffer is reused once the bulk copy has
//     read it.
//   phase B (fallback, threads along columns) for positions, SwiGLU, conv
//     sub-tiles whose 32 rows are not all valid, and 16-column tails: read
//     the buffer back so that a warp instruction covers whole 128-byte
//     (fp32) or 64-byte (bf16) row segments, add positions with coalesced
//     loads, and store with coalesced 16-byte (fp32) or 8-byte (bf16)
//     stores.
//   Stream-K pieces (residual epilogue only): PIECE_PARTIAL adds its raw
//     accumulator (no bias) to the residual stream; the caller orders the
//     owner's update after it.
//   Staging: NBUF buffers of BUFB bytes per warp, used in turn (gcount
//     counts the warp's groups across tiles), so with two a group's smem
//     writes overlap the previous group's store and two stores per warp are
//     in flight.
template <int EPI, int KIND = KIND_BF16, int NBUF = 1, int BUFB = 4096>
__device__ __forceinline__ void epilogue_warp(const GemmParams& p, const CUtensorMap* tm_out, uint32_t tb, int row0,
                                              int mlimit, int n0, int BN, int half, int lane, uint8_t* wbase,
                                              const float* breg, int kind = PIECE_FULL, int cstride = 64,
                                              int* gcount = nullptr) {
  constexpr bool F32 = (EPI & (EPI_OUT_F32 | EPI_RESID)) != 0;
  constexpr bool SWI = (EPI & EPI_SWIGLU) != 0;  // with F32: fp32 outputs, stored per row
  constexpr bool TMA_OK = (EPI & (EPI_PE | EPI_SWIGLU)) == 0;
  if (row0 >= mlimit) return;  // no valid row in this quarter (warp-uniform)
  // A 32-row box may be stored whole when all its rows belong to this
  // sub-tile, or when the rows past the end lie past M (the TMA clips them).
  const bool rows_ok = TMA_OK && p.out_tma && (mlimit - row0 >= 32 || mlimit >= p.M);
  // 16-byte aligned bias: vector loads of each group's biases (else the
  // per-lane values loaded before the accumulator wait, broadcast by shuffle)
  const bool bias_vec = (reinterpret_cast<uintptr_t>(p.bias) & 15) == 0;
  // this lane's row is a zero (padding) row of a packed convolution layout
  const bool zero_row = p.zero_period && (row0 + lane) % p.zero_period >= p.zero_from;
  int j = 0;
#pragma unroll 1
  for (int c = half * 32; c < BN; c += cstride, ++j) {
    const int n = n0 + c;
    if (n >= p.N) break;                                  // warp-uniform
    const int w = (BN - c < 32 || p.N - n < 32) ? 16 : 32;  // valid columns in this group (N % 16 == 0)
    const bool use_tma = rows_ok && BN - c >= 32;
    float v[32];
    if (BN - c >= 32)
      tmem_ld32(tb + c, v);
    else
      tmem_ld16(tb + c, v);
    tmem_ld_wait();
    // ---- phase A
    if (p.bias && kind != PIECE_PARTIAL) {
      if (bias_vec) {
        // the group's biases: the same address in every lane (broadcast loads)
        const float4* b4 = reinterpret_cast<const float4*>(p.bias + n);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          if (4 * k < w) {
            const float4 b = __ldg(b4 + k);
            const float2 lo = add2(make_float2(v[4 * k], v[4 * k + 1]), make_float2(b.x, b.y));
            const float2 hi = add2(make_float2(v[4 * k + 2], v[4 * k + 3]), make_float2(b.z, b.w));
            v[4 * k] = lo.x;
            v[4 * k + 1] = lo.y;
            v[4 * k + 2] = hi.x;
            v[4 * k + 3] = hi.y;
          }
        }
      } else {
        const float bj = breg[j];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] += __shfl_sync(0xffffffffu, bj, i);
      }
    }
    if (zero_row) {
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = 0.f;  // GELU(0) = 0: the row stays zero
    }
    if (SWI && F32) {
      // gate = columns c..c+15, up = c+16..c+31 -> 16 fp32 outputs of this row
      const int row = row0 + lane;
      if (row < mlimit) {
        float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + (long long)row * p.ldo + (n >> 1));
#pragma unroll
        for (int k = 0; k < 4; ++k)
          dst[k] = make_float4(silu(v[4 * k]) * v[16 + 4 * k], silu(v[4 * k + 1]) * v[17 + 4 * k],
                               silu(v[4 * k + 2]) * v[18 + 4 * k], silu(v[4 * k + 3]) * v[19 + 4 * k]);
      }
      continue;
    }
    // This group's buffer, which may still be the source of the bulk store
    // issued from it NBUF groups ago.
    uint8_t* wbuf = wbase;
    if (NBUF == 2) {
      wbuf += (*gcount & 1) * BUFB;
      ++*gcount;
    }
    if (lane == 0) {
      if (NBUF == 2)
        bulk_wait_read1();
      else
        bulk_wait_read0();
    }
    __syncwarp();
    if (SWI) {
      // gate = columns c..c+15, up = c+16..c+31 -> 16 bf16 outputs (2 chunks).
      uint4* row = reinterpret_cast<uint4*>(wbuf + lane * 64);
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        uint32_t r[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int jj = 8 * k + 2 * i;
          r[i] = pack2_16<KIND>(silu(v[jj]) * v[16 + jj], silu(v[jj + 1]) * v[17 + jj]);
        }
        row[k ^ ((lane >> 1) & 3)] = make_uint4(r[0], r[1], r[2], r[3]);
      }
    } else {
      if (EPI & EPI_GELU) {
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float2 g = gelu_erf2(make_float2(v[i], v[i + 1]));
          v[i] = g.x;
          v[i + 1] = g.y;
        }
      }
      if (F32) {
        float4* row = reinterpret_cast<float4*>(wbuf + lane * 128);
#pragma unroll
        for (int k = 0; k < 8; ++k) row[k ^ (lane & 7)] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
      } else {
        uint4* row = reinterpret_cast<uint4*>(wbuf + lane * 64);
#pragma unroll
        for (int k = 0; k < 4; ++k) row[k ^ ((lane >> 1) & 3)] = pack8_16<KIND>(v + 8 * k);
      }
    }
    if (use_tma) {
      fence_proxy_async_smem();  // make this lane's smem writes visible to the bulk copy
      __syncwarp();
      if (lane == 0) {
        if (EPI & EPI_RESID)
          tma_reduce_add_2d(tm_out, wbuf, n, row0);
        else
          tma_store_2d(tm_out, wbuf, n, row0);
        bulk_commit();
      }
      continue;
    }
    __syncwarp();
    // ---- phase B
    if (F32) {
      // 8 threads per row (float4 each), 4 rows per instruction, 8 passes.
      const int k = lane & 7;
      const int nc = n + 4 * k;
      const bool col_ok = 4 * k < w;
      float4 pre[8];
      if (EPI & (EPI_RESID | EPI_PE)) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = (lane >> 3) + 4 * i;
          const int row = row0 + r;
          if (col_ok && row < mlimit) {
            if (EPI & EPI_RESID)
              pre[i] = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p.out) + (long long)row * p.ldo + nc);
            else
              pre[i] = __ldg(reinterpret_cast<const float4*>(p.pe + (long long)(row % p.pe_period) * p.N + nc));
          }
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = (lane >> 3) + 4 * i;
        const int row = row0 + r;
        float4 x = reinterpret_cast<const float4*>(wbuf + r * 128)[k ^ (r & 7)];
        if (col_ok && row < mlimit) {
          if (EPI & (EPI_RESID | EPI_PE)) {
            x.x += pre[i].x; x.y += pre[i].y; x.z += pre[i].z; x.w += pre[i].w;
          }
          *reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + (long long)row * p.ldo + nc) = x;
        }
      }
    } else {
      // bf16: outputs per row = w (or w/2 for SwiGLU); 4 per thread (8 bytes).
      const int wo = SWI ? w / 2 : w;
      const int tpr = wo / 4;           // threads per row: 8 or 4 (or 2)
      const int rpi = 32 / tpr;         // rows per pass
      const int k4 = lane % tpr;        // which 4-column piece
      const int rr = lane / tpr;
      const long long ncol = SWI ? (n >> 1) + 4 * k4 : n + 4 * k4;
#pragma unroll 1
      for (int r = rr; r < 32; r += rpi) {
        const int row = row0 + r;
        const uint2* src = reinterpret_cast<const uint2*>(wbuf + r * 64);
        const int chunk = (k4 >> 1) ^ ((r >> 1) & 3);
        const uint2 val = src[2 * chunk + (k4 & 1)];
        if (row < mlimit) *reinterpret_cast<uint2*>(reinterpret_cast<bf16*>(p.out) + (long long)row * p.ldo + ncol) = val;
      }
    }
    __syncwarp();
  }
}

template <int BN, int STAGES, bool GATHER, int EPI, int KIND>
__device__ __forceinline__ void gemm_tc_body(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmOut,
                                             const GemmParams& p) {
  using S = GemmShape<BN, STAGES, GATHER, KIND>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * S::A_BYTES;
  uint8_t* sEpi = smem + STAGES * S::STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sEpi + S::EPI_BUF_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* tfull = bars + 2 * STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], GATHER ? 1 + 32 * S::GATHER_WARPS : 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], S::EPI_WARPS);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmB);
    if (!GATHER) tma_prefetch_desc(&tmA);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, S::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
        int mb, nb;
        tile_coords(p, t, mb, nb);
        const int m0 = mb * S::BM;
        const int n0 = nb * BN;
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait_bounded(&empty[s], ph ^ 1, p.limit_ns, p.status, DEV_TIMEOUT_PRODUCER)) {
            ok = false;
            break;
          }
          if (GATHER) {
            mbar_arrive_expect_tx(&full[s], S::B_BYTES);
          } else {
            mbar_arrive_expect_tx(&full[s], S::A_BYTES + S::B_BYTES);
            if (p.conv_box) {
              int c0, f0, t0, img;
              convbox_coords(p, mb, kb, c0, f0, t0, img, S::BK);
              tma_load_4d(sA + s * S::A_BYTES, &tmA, &full[s], c0, f0, t0, img);
            } else {
              tma_load_2d(sA + s * S::A_BYTES, &tmA, &full[s], kb * S::BK, m0);
            }
          }
          tma_load_2d(sB + s * S::B_BYTES, &tmB, &full[s], kb * S::BK, n0);
          ++it;
        }
      }
      // Drain: every issued load must have landed before the CTA exits.
      if (!GATHER) {
        for (int s = 0; s < STAGES; ++s) {
          if (it > s) {
            const int last = s + ((it - 1 - s) / STAGES) * STAGES;
            mbar_wait_bounded(&full[s], (last / STAGES) & 1, kDrainLimitNs, nullptr, 0);
          }
        }
      } else {
        // Gather mode: full[] also needs the gather warps' arrivals, which
        // may be missing after a failure; the bound covers that case.
        for (int s = 0; s < STAGES; ++s) {
          if (it > s) {
            const int last = s + ((it - 1 - s) / STAGES) * STAGES;
            if (!ok || *reinterpret_cast<volatile int*>(p.status) != 0)
              mbar_wait_bounded(&full[s], (last / STAGES) & 1, kDrainLimitNs / 20, nullptr, 0);
            else
              mbar_wait_bounded(&full[s], (last / STAGES) & 1, kDrainLimitNs, nullptr, 0);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_kind_f32(KIND, S::BM, BN);
      int it = 0, tl = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x, ++tl) {
        const int a = tl & 1;
        const uint32_t aph = (tl >> 1) & 1;
        if (!mbar_wait_bounded(&tempty[a], aph ^ 1, p.limit_ns, p.status, DEV_TIMEOUT_MMA)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + a * S::ACC_COLS;
        // The k-loop in two versions: every k-block whole (four MMA steps
        // issued as one sequence, no per-block test: a test in the loop
        // measured about 8 % of the MMA rate), or with partial k-blocks.
        auto kloop = [&](auto full_tag) {
          constexpr bool FULL = decltype(full_tag)::value;
          for (int kb = 0; kb < p.k_blocks; ++kb) {
            const int s = it % STAGES;
            const uint32_t ph = (it / STAGES) & 1;
            if (!mbar_wait_bounded(&full[s], ph, p.limit_ns, p.status, DEV_TIMEOUT_MMA)) {
              ok = false;
              break;
            }
            // cp.async wrote the A tile through the generic proxy; order those
            // writes (observed through the barrier) before the MMA's reads.
            if (GATHER) fence_proxy_async_smem();
            tc_fence_after();
            const uint64_t ad = sw128_kmajor_desc(smem_u32(sA + s * S::A_BYTES));
            const uint64_t bd = sw128_kmajor_desc(smem_u32(sB + s * S::B_BYTES));
            // each step: 32 bytes of K (16 bf16 or 8 tf32 elements)
            if (FULL) {
              if (KIND == KIND_TF32)
                tc_mma4_tf32(d_tmem, ad, bd, idesc, kb > 0 ? 1u : 0u);
              else
                tc_mma4_bf16(d_tmem, ad, bd, idesc, kb > 0 ? 1u : 0u);
            } else {
              const int ks = k16_steps(p, kb, S::BK);
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                if (k < ks) {
                  if (KIND == KIND_TF32)
                    tc_mma_tf32(d_tmem, ad + 2 * k, bd + 2 * k, idesc, (kb > 0 || k > 0) ? 1u : 0u);
                  else
                    tc_mma_bf16(d_tmem, ad + 2 * k, bd + 2 * k, idesc, (kb > 0 || k > 0) ? 1u : 0u);
                }
              }
            }
            tc_commit(&empty[s]);
            ++it;
          }
        };
        if (p.k_full)
          kloop(BoolTag<true>{});
        else
          kloop(BoolTag<false>{});
        if (!ok) break;
        tc_commit(&tfull[a]);
      }
      // Drain: all issued MMAs complete before tensor memory is released.
      tc_commit(drain);
      mbar_wait_bounded(drain, 0, kDrainLimitNs, nullptr, 0);
    }
  } else if (warp < 2 + S::EPI_WARPS) {
    // ------------------------------------------------ epilogue
    const int q = warp & 3;                   // TMEM lane quarter this warp may access
    const int half = (warp - 2) / 4;          // which alternate column chunks it takes
    const int rank_rows = 0;
    int tl = 0;
    for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x, ++tl) {
      const int a = tl & 1;
      const uint32_t aph = (tl >> 1) & 1;
      int mb, nb;
      tile_coords(p, t, mb, nb);
      const int n0 = nb * BN;
      if (EPI & EPI_RESID) epilogue_prefetch_l2(p, t, half, q, lane, BN, S::BM, rank_rows);
      float breg[4];
      load_bias(p, n0, BN, half, lane, breg);
      if (!mbar_wait_bounded(&tfull[a], aph, p.limit_ns, p.status, DEV_TIMEOUT_EPILOGUE)) break;
      tc_fence_after();
      int r_first, r_last;
      subtile_rows(p, mb, r_first, r_last);
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + a * S::ACC_COLS;
      epilogue_warp<EPI, KIND>(p, &tmOut, tb, r_first + 32 * q, r_last, n0, BN, half, lane, sEpi + (warp - 2) * 4096, breg);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[a]);
    }
    if (lane == 0) bulk_wait0();  // bulk stores complete before the CTA exits
  } else if (GATHER) {
    // ------------------------------------------------ implicit-GEMM gather
    constexpr int RSTEP = (S::GATHER_WARPS > 0 ? S::GATHER_WARPS : 1) * 4;  // rows per pass (8 threads per row)
    constexpr int NR = 128 / RSTEP;                         // passes over the 128-row tile
    const int gt = threadIdx.x - 32 * (2 + S::EPI_WARPS);
    const int chunk = gt & 7;                               // 16-byte chunk of a 128-byte row
    const int rsub = gt >> 3;                               // rows rsub + RSTEP * i
    const ConvGather& g = p.g;
    const int per_img = g.T_out * g.F_out;
    int it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
      int mb, nb;
      tile_coords(p, t, mb, nb);
      const int m0 = mb * S::BM;
      const bf16* rbase[NR];
      int tb[NR], fb[NR];
      bool rv[NR];
#pragma unroll
      for (int i = 0; i < NR; ++i) {
        const int m = m0 + rsub + RSTEP * i;
        rv[i] = m < p.M;
        const int mm = rv[i] ? m : 0;
        const int img = mm / per_img;
        const int rem = mm - img * per_img;
        const int to = rem / g.F_out;
        const int fo = rem - to * g.F_out;
        tb[i] = to * g.st - g.pt;
        fb[i] = fo * g.sf - g.pf;
        rbase[i] = g.x + (long long)img * g.T_in * g.F_in * g.C;
      }
      for (int kb = 0; kb < p.k_blocks; ++kb) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (!mbar_wait_bounded(&empty[s], ph ^ 1, p.limit_ns, p.status, DEV_TIMEOUT_GATHER)) {
          ok = false;
          break;
        }
        const int k = kb * S::BK + chunk * 8;
        const bool kv = k < p.K;
        const int tap = kv ? k / g.C : 0;
        const int c = k - tap * g.C;
        const int dt = tap / g.kf;
        const int df = tap - dt * g.kf;
        uint8_t* dst_stage = sA + s * S::A_BYTES;
#pragma unroll
        for (int i = 0; i < NR; ++i) {
          const int row = rsub + RSTEP * i;
          const int ti = tb[i] + dt;
          const int fi = fb[i] + df;
          const bool valid = kv && rv[i] && ti >= 0 && ti < g.T_in && fi >= 0 && fi < g.F_in;
          const bf16* src = valid ? rbase[i] + ((long long)(ti * g.F_in + fi) * g.C + c) : g.x;
          uint8_t* dst = dst_stage + row * 128 + ((chunk ^ (row & 7)) << 4);
          cp_async_16_zfill(dst, src, valid);
        }
        // The barrier completes this thread's share when its copies land.
        cp_async_arrive_noinc(&full[s]);
        ++it;
      }
    }
    cp_async_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, S::TMEM_COLS);
}

// bf16 operands (kind::f16).
template <int BN, int STAGES, bool GATHER, int EPI>
__global__ void __launch_bounds__(GemmShape<BN, STAGES, GATHER>::THREADS, 1)
    gemm_bf16_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmOut, const GemmParams p) {
  gemm_tc_body<BN, STAGES, GATHER, EPI, KIND_BF16>(tmA, tmB, tmOut, p);
}

// f16 operands (kind::f16).
template <int BN, int STAGES, bool GATHER, int EPI>
__global__ void __launch_bounds__(GemmShape<BN, STAGES, GATHER>::THREADS, 1)
    gemm_f16_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmOut, const GemmParams p) {
  gemm_tc_body<BN, STAGES, GATHER, EPI, KIND_F16>(tmA, tmB, tmOut, p);
}

// fp32 operands in memory, multiplied as tf32 (kind::tf32), fp32 accumulate.
template <int BN, int STAGES, int EPI>
__global__ void __launch_bounds__(GemmShape<BN, STAGES, false, KIND_TF32>::THREADS, 1)
    gemm_tf32_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmOut, const GemmParams p) {
  gemm_tc_body<BN, STAGES, false, EPI, KIND_TF32>(tmA, tmB, tmOut, p);
}

}  // namespace asr

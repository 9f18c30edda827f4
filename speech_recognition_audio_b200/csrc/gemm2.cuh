// Two-SM variant of the tcgen05 GEMM engine: a CTA pair (cluster of 2)
// computes 256 x BN output tiles with tcgen05.mma.cta_group::2 (M = 256).
//
// Each CTA of the pair stages its own 128 rows of A and its own BN/2 rows of
// B (plain TMA loads, no multicast); the tensor cores of the pair exchange
// the B halves, so every SM fetches a third less operand data per FLOP than
// the one-SM 128 x BN tile, and each 32 KB stage covers twice the FLOPs of a
// one-SM 48 KB stage, which is what hides L2 / HBM latency.  Accumulators:
// each CTA's tensor memory holds its 128 rows x BN columns, twice (double
// buffered).
//
// Roles (per CTA, 320 threads):
//   warp 0  lane 0: TMA producer.  Both CTAs load into their own smem and
//           signal the LEADER's full barrier (mapa to CTA rank 0); the leader
//           arms it with the byte count of both halves.
//   warp 1  allocates tensor memory (cta_group::2, both CTAs); in the leader,
//           lane 0 issues the MMAs and commits, multicast to both CTAs, to
//           the stage's empty barriers and the accumulator full barriers.
//   warps 2-9  epilogue on the CTA's own TMEM rows; releases the accumulator
//           with a remote arrive on the leader's accumulator-empty barrier.
// Every wait is bounded; both CTAs meet at a cluster barrier before tensor
// memory is freed.
#pragma once

#include "gemm.cuh"

namespace asr {

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// TMA load into this CTA's smem, completion (bytes) reported to the barrier
// at `bar_cluster_addr` (a shared::cluster address, here the leader's).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster_addr, int x,
                                                 int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster_addr), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tma_load_4d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster_addr, int c0,
                                                 int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, "
      "%6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster_addr), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
// 3-D box {64 elements, rows, 2 k-blocks} of a [rows][K] matrix viewed as
// {64, rows, K / 64}: two 64-element k-blocks of `rows` rows in one copy,
// landing as two consecutive canonical 128-byte-row tiles.
__device__ __forceinline__ void tma_load_3d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster_addr, int c0,
                                                 int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster_addr), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_mma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                 uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// The four K = 16 steps of a 64-element k-block as one sequence (see
// tc_mma4_bf16), CTA-pair form.
__device__ __forceinline__ void tc_mma4_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                  uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %5, %6, %3, 1;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %7, %8, %3, 1;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %9, %10, %3, 1;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "l"(adesc + 2), "l"(bdesc + 2), "l"(adesc + 4),
      "l"(bdesc + 4), "l"(adesc + 6), "l"(bdesc + 6)
      : "memory");
}
// Arrive (once each) on the barrier at the same offset in every CTA of `mask`
// when the pair's previously issued MMAs complete.
__device__ __forceinline__ void tc_commit_pair_mc(uint64_t* bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(mask)
      : "memory");
}

// EPIW_: epilogue warps, 8 or 16 (16 only for bf16 outputs, whose 32 x 32
// staging box takes 2 KB); NBUF_: staging buffers per epilogue warp, used in
// turn (two let a warp fill the next box while the previous TMA store still
// reads its buffer).  The staging area is 32 KB per buffer.
// KP_: 64-element k-blocks per pipeline stage.  With 2 each operand's stage
// comes in one 3-D copy (the per-copy cost of the TMA, not its bytes, bounds
// 128-row boxes: 0.27 us per k-block with one copy per k-block and operand,
// 0.19 us with one per two, measured without MMAs).
template <int BN_, int STAGES_, int EPIW_ = 8, int NBUF_ = 1, int KP_ = 1>
struct Gemm2Shape {
  static constexpr int BM = 256, BN = BN_, BK = 64, STAGES = STAGES_, KP = KP_;
  static constexpr int A_BYTES = 128 * BK * 2 * KP;        // this CTA's half of A
  static constexpr int B_BYTES = (BN / 2) * BK * 2 * KP;   // this CTA's half of B
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TX_BYTES = 2 * STAGE_BYTES;    // both CTAs, counted on the leader
  static constexpr int ACC_COLS = (BN + 31) / 32 * 32;
  static constexpr int TMEM_COLS = 2 * ACC_COLS <= 64 ? 64 : 2 * ACC_COLS <= 128 ? 128 : 2 * ACC_COLS <= 256 ? 256 : 512;
  static constexpr int EPI_WARPS = EPIW_;
  static constexpr int THREADS = 32 * (2 + EPI_WARPS);
  static constexpr int BOXB = EPI_WARPS == 16 ? 2048 : 4096;  // one 32 x 32 output box (bf16 / fp32)
  static constexpr int NBUF = NBUF_;                          // staging buffers per epilogue warp
  static constexpr int WBUF = NBUF * BOXB;                    // staging bytes per epilogue warp
  static constexpr int CSTRIDE = 32 * (EPI_WARPS / 4);       // column stride of a warp's groups
  static constexpr int EPI_BUF_BYTES = EPI_WARPS * WBUF;
  static constexpr int BAR_BYTES = 8 * (2 * STAGES + 5) + 16;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + EPI_BUF_BYTES + BAR_BYTES;
  static_assert(BN % 16 == 0 && (BN / 2) % 8 == 0 && BN >= 64 && BN <= 256, "UMMA N for M=256; B halves of 8-row atoms");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
  static_assert(EPI_WARPS == 8 || EPI_WARPS == 16, "two or four column parts per lane quarter");
};

// Staging buffers per epilogue warp: tiles of 192 columns and more keep six
// 32 KB pipeline stages with one buffer (measured: a second buffer at the
// cost of a stage made the residual GEMMs 2-6 % slower and the others no
// faster); narrower tiles have room for both.
template <int BN>
constexpr int gemm2_nbuf() {
  return BN >= 192 ? 1 : 2;
}

// Epilogue warps of an instance: 16 for the bias + GELU bf16 epilogue (the
// GELU's arithmetic is the epilogue's cost; with 8 warps it is latency-bound,
// and it is the whole cost of the K = 16 conv1 GEMM), 8 otherwise.
template <int EPI>
constexpr int gemm2_epi_warps() {
  return EPI == EPI_GELU ? 16 : 8;
}

// Residual + LayerNorm epilogue (EPI_RESID | EPI_LN; whole tiles of plain
// GEMMs, BN = 256, N a multiple of 32, the n-tiles of a row block back to
// back).
//
// One warp: 32 rows (one per lane) over the four 32-column groups
// c = 32 half + 64 j of the accumulator, with a 4 KB shared buffer in which
// 32 x 32 blocks are transposed between the row-per-lane layout of tensor
// memory and coalesced global accesses (8 lanes per 128-byte row segment of
// fp32, 4 per 64-byte segment of 16-bit values; 16-byte chunks XOR-swizzled
// by row, which keeps both access patterns free of bank conflicts).
//   pass 1, per group: the old residual block (loaded two groups ahead, the
//     first two before the accumulator is ready) is transposed into the
//     lanes; each lane forms x_new = x + (acc + bias) for its row (the
//     additions of the plain residual epilogue, so the stream is the same
//     bit for bit), writes it back into tensor memory and accumulates
//     shifted sums (shift = the row's first value here);
//   publish: the warp's partial statistics {count, mean, M2} of each row go
//     to p.ln_part [part][row], then one release reduction-add (lane 0, after
//     the warp barrier) on the 32-row group's counter;
//   x pass: x_new from tensor memory, transposed, stored (coalesced) into
//     the residual stream, while the other tiles of the rows publish;
//   wait (bounded) until every warp of every n-tile covering these rows has
//     added to the counter: it then holds (p.ln_epoch + 1) * p.ln_parts;
//   merge: each lane folds its row's partials in one pass with the pairwise
//     update of Chan, Golub and LeVeque (mean and M2 of a union from those
//     of its parts), var = M2 / N;
//   pass 3: h = (x_new - mean) / sqrt(var + eps) * gamma + beta from tensor
//     memory, in 16 bits, transposed and stored (coalesced) into p.ln_h.
// No wait cycle: under the persistent whole-tile schedule a tile's epilogue
// waits only on the other n-tiles of its row block, whose indices are within
// n_blocks of its own; each of those is processed by a resident pair after a
// tile at least n_pairs (>= n_blocks) lower, and every warp publishes
// before it waits.
constexpr int kLnGroups = 4;  // 32-column groups of a warp (BN = 256, two warps per lane quarter)

// Old residual block of rows row0.. (< mlimit) and columns n..n+31 in the
// coalesced layout: lane l holds row row0 + l / 8 + 4 i, columns n + 4 (l % 8).
__device__ __forceinline__ void ln_load_x(const GemmParams& p, int row0, int mlimit, int n, int lane, float4* pre) {
  const float* base = reinterpret_cast<const float*>(p.out) + n + 4 * (lane & 7);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int row = row0 + (lane >> 3) + 4 * i;
    pre[i] = row < mlimit ? *reinterpret_cast<const float4*>(base + (long long)row * p.ldo) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

template <int KIND>
__device__ __forceinline__ void epilogue_warp_resid_ln(const GemmParams& p, uint32_t tb, int row0, int mlimit, int n0,
                                                       int half, int lane, uint8_t* wbuf, int part,
                                                       float4 (&pre)[2][8]) {
  if (row0 >= mlimit) return;  // no valid row: nobody waits on this group (warp-uniform)
  const int row = row0 + lane;
  const bool valid = row < mlimit;
  float4* wrow = reinterpret_cast<float4*>(wbuf + lane * 128);  // this lane's fp32 row of the block
  float K = 0.f;
  float2 s1 = make_float2(0.f, 0.f), s2 = make_float2(0.f, 0.f);
  int cnt = 0;
#pragma unroll
  for (int j = 0; j < kLnGroups; ++j) {
    const int n = n0 + half * 32 + 64 * j;
    if (n >= p.N) break;  // warp-uniform
    float v[32];
    tmem_ld16(tb + n - n0, v);
    tmem_ld16(tb + n - n0 + 16, v + 16);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = (lane >> 3) + 4 * i;
      reinterpret_cast<float4*>(wbuf + r * 128)[(lane & 7) ^ (r & 7)] = pre[j & 1][i];
    }
    if (j + 2 < kLnGroups && n + 128 < p.N) ln_load_x(p, row0, mlimit, n + 128, lane, pre[j & 1]);
    __syncwarp();
    tmem_ld_wait();
    const float4* b4 = p.bias ? reinterpret_cast<const float4*>(p.bias + n) : nullptr;  // same address in every lane
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float4 o = wrow[k ^ (lane & 7)];
      const float4 bq = b4 ? __ldg(b4 + k) : make_float4(0.f, 0.f, 0.f, 0.f);
      // x_new = x + (acc + bias), the plain residual epilogue's additions
      const float2 lo = add2(make_float2(o.x, o.y), add2(make_float2(v[4 * k], v[4 * k + 1]), make_float2(bq.x, bq.y)));
      const float2 hi =
          add2(make_float2(o.z, o.w), add2(make_float2(v[4 * k + 2], v[4 * k + 3]), make_float2(bq.z, bq.w)));
      v[4 * k] = lo.x;
      v[4 * k + 1] = lo.y;
      v[4 * k + 2] = hi.x;
      v[4 * k + 3] = hi.y;
    }
    __syncwarp();  // the block is read before the next group overwrites it
    if (j == 0) K = v[0];
    const float2 nk = make_float2(-K, -K);
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      const float2 dv = add2(make_float2(v[i], v[i + 1]), nk);
      s1 = add2(s1, dv);
      s2 = fma2(dv, dv, s2);
    }
    cnt += 32;
    tmem_st16(tb + n - n0, v);
    tmem_st16(tb + n - n0 + 16, v + 16);
  }
  // publish this warp's partial statistics of its rows
  {
    const float inv = cnt ? 1.0f / static_cast<float>(cnt) : 0.f;
    const float t1 = s1.x + s1.y, t2 = s2.x + s2.y;
    const float mu = K + t1 * inv;
    const float m2 = fmaxf(t2 - t1 * t1 * inv, 0.f);
    if (valid)
      *reinterpret_cast<float4*>(p.ln_part + ((long long)part * p.M + row) * 4) =
          make_float4(static_cast<float>(cnt), mu, m2, 0.f);
  }
  __syncwarp();  // orders the lanes' partials before lane 0's release
  int* counter = p.ln_count + row0 / 32;
  if (lane == 0) red_add_release_gpu(counter, 1);
  tmem_st_wait();
  // x pass: the updated rows into the residual stream
  float* xo = reinterpret_cast<float*>(p.out) + 4 * (lane & 7);
#pragma unroll
  for (int j = 0; j < kLnGroups; ++j) {
    const int n = n0 + half * 32 + 64 * j;
    if (n >= p.N) break;
    float v[32];
    tmem_ld16(tb + n - n0, v);
    tmem_ld16(tb + n - n0 + 16, v + 16);
    tmem_ld_wait();
#pragma unroll
    for (int k = 0; k < 8; ++k) wrow[k ^ (lane & 7)] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = (lane >> 3) + 4 * i;
      const float4 o = reinterpret_cast<const float4*>(wbuf + r * 128)[(lane & 7) ^ (r & 7)];
      if (row0 + r < mlimit) *reinterpret_cast<float4*>(xo + (long long)(row0 + r) * p.ldo + n) = o;
    }
    __syncwarp();
  }
  // every warp of this launch covering these rows has added once: the
  // counter (zero before the forward) reaches (epoch + 1) * parts
  if (lane == 0) count_wait_bounded(counter, (p.ln_epoch + 1) * p.ln_parts, p.limit_ns, p.status, DEV_TIMEOUT_EPILOGUE);
  __syncwarp();
  (void)ld_acquire_gpu(counter);  // every lane: the partials below come after the arrivals
  float mean = 0.f, rstd = 0.f;
  if (valid) {
    const float4* pr = reinterpret_cast<const float4*>(p.ln_part) + row;
    float nt = 0.f, m2 = 0.f;
    for (int i0 = 0; i0 < p.ln_parts; i0 += 8) {
      float4 q[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) q[i] = i0 + i < p.ln_parts ? __ldcg(pr + (long long)(i0 + i) * p.M) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (q[i].x > 0.f) {
          const float nn = nt + q[i].x;
          const float dm = q[i].y - mean;
          const float wb = __fdividef(q[i].x, nn);
          mean = fmaf(dm, wb, mean);
          m2 += q[i].z + dm * dm * nt * wb;
          nt = nn;
        }
    }
    rstd = rsqrtf(fmaxf(m2 / nt, 0.f) + p.ln_eps);
  }
  // pass 3: the normalised rows, 16-bit (64-byte row segments in the buffer)
  uint16_t* ho = reinterpret_cast<uint16_t*>(p.ln_h) + 8 * (lane & 3);
  const float2 nm = make_float2(-mean, -mean), rs = make_float2(rstd, rstd);
#pragma unroll
  for (int j = 0; j < kLnGroups; ++j) {
    const int n = n0 + half * 32 + 64 * j;
    if (n >= p.N) break;
    float v[32];
    tmem_ld16(tb + n - n0, v);
    tmem_ld16(tb + n - n0 + 16, v + 16);
    tmem_ld_wait();
    const float4* g4 = reinterpret_cast<const float4*>(p.ln_gamma + n);
    const float4* b4 = reinterpret_cast<const float4*>(p.ln_beta + n);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float4 g = __ldg(g4 + k), b = __ldg(b4 + k);
      const float2 lo = fma2(add2(make_float2(v[4 * k], v[4 * k + 1]), nm), mul2(rs, make_float2(g.x, g.y)),
                             make_float2(b.x, b.y));
      const float2 hi = fma2(add2(make_float2(v[4 * k + 2], v[4 * k + 3]), nm), mul2(rs, make_float2(g.z, g.w)),
                             make_float2(b.z, b.w));
      v[4 * k] = lo.x;
      v[4 * k + 1] = lo.y;
      v[4 * k + 2] = hi.x;
      v[4 * k + 3] = hi.y;
    }
    uint4* hrow = reinterpret_cast<uint4*>(wbuf + lane * 64);
#pragma unroll
    for (int k = 0; k < 4; ++k) hrow[k ^ ((lane >> 1) & 3)] = pack8_16<KIND>(v + 8 * k);
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = (lane >> 2) + 8 * i;
      const uint4 o = reinterpret_cast<const uint4*>(wbuf + r * 64)[(lane & 3) ^ ((r >> 1) & 3)];
      if (row0 + r < mlimit) *reinterpret_cast<uint4*>(ho + (long long)(row0 + r) * p.ldo + n) = o;
    }
    __syncwarp();
  }
}

template <int BN, int STAGES, int EPI, int KIND, int KP = 1>
__device__ __forceinline__ void gemm_tc2_body(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmOut,
                                              const GemmParams& p) {
  // KP == 2: tmA / tmB are 3-D maps, p.k_blocks counts two-k-block stages
  using S = Gemm2Shape<BN, STAGES, gemm2_epi_warps<EPI>(), gemm2_nbuf<BN>(), KP>;
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
  const uint32_t rank = cluster_ctarank();  // 0 = leader
  const int pair = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);   // leader: its own arrive.expect_tx (+ both CTAs' bytes)
      mbar_init(&empty[s], 1);  // one multicast commit per stage use
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * S::EPI_WARPS);  // leader: epilogue warps of both CTAs
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, S::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // barriers of both CTAs initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      const uint32_t full_leader0 = mapa_shared(smem_u32(&full[0]), 0);
      int it = 0;
      bool ok = true;
      PieceIter pi(p, pair, n_pairs);
      int t, kb0, kb1;
      while (ok && pi.next(p, t, kb0, kb1)) {
        int mb, nb;
        tile_coords(p, t, mb, nb);
        const int u = 2 * mb + static_cast<int>(rank);  // this CTA's 128-row sub-tile
        const int m0 = u * 128;
        const int n0 = nb * BN + static_cast<int>(rank) * (BN / 2);
        for (int kb = kb0; kb < kb1; ++kb) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait_bounded(&empty[s], ph ^ 1, p.limit_ns, p.status, DEV_TIMEOUT_PRODUCER)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&full[s], S::TX_BYTES);
          const uint32_t fb = full_leader0 + 8u * s;
          if constexpr (KP == 2) {
            tma_load_3d_pair(sA + s * S::A_BYTES, &tmA, fb, 0, m0, 2 * kb);
            tma_load_3d_pair(sB + s * S::B_BYTES, &tmB, fb, 0, n0, 2 * kb);
          } else {
            if (p.conv_box) {
              int c0, f0, t0, img;
              convbox_coords(p, u, kb, c0, f0, t0, img);
              tma_load_4d_pair(sA + s * S::A_BYTES, &tmA, fb, c0, f0, t0, img);
            } else {
              tma_load_2d_pair(sA + s * S::A_BYTES, &tmA, fb, kb * S::BK, m0);
            }
            tma_load_2d_pair(sB + s * S::B_BYTES, &tmB, fb, kb * S::BK, n0);
          }
          ++it;
        }
      }
      // Drain (leader sees both CTAs' bytes on its full barriers).
      if (rank == 0) {
        for (int s = 0; s < STAGES; ++s) {
          if (it > s) {
            const int last = s + ((it - 1 - s) / STAGES) * STAGES;
            mbar_wait_bounded(&full[s], (last / STAGES) & 1, kDrainLimitNs, nullptr, 0);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      const uint32_t idesc = idesc_kind_f32(KIND, S::BM, BN);
      int it = 0, tl = 0;
      bool ok = true;
      PieceIter pi(p, pair, n_pairs);
      int t, kb0, kb1;
      for (; ok && pi.next(p, t, kb0, kb1); ++tl) {
        const int a = tl & 1;
        const uint32_t aph = (tl >> 1) & 1;
        if (!mbar_wait_bounded(&tempty[a], aph ^ 1, p.limit_ns, p.status, DEV_TIMEOUT_MMA)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + a * S::ACC_COLS;
        // Two versions of the k-loop (see the one-SM kernel): whole k-blocks
        // only, or with partial ones.
        auto kloop = [&](auto full_tag) {
          constexpr bool FULL = decltype(full_tag)::value;
          for (int kb = kb0; kb < kb1; ++kb) {
            const int s = it % STAGES;
            const uint32_t ph = (it / STAGES) & 1;
            if (!mbar_wait_bounded(&full[s], ph, p.limit_ns, p.status, DEV_TIMEOUT_MMA)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t ad = sw128_kmajor_desc(smem_u32(sA + s * S::A_BYTES));
            const uint64_t bd = sw128_kmajor_desc(smem_u32(sB + s * S::B_BYTES));
            if (FULL) {
              // k-block j of the stage: A tile at +16 KB j, B tile at +(BN/2) x 128 B j
#pragma unroll
              for (int j = 0; j < KP; ++j)
                tc_mma4_bf16_pair(d_tmem, ad + (uint64_t)(j * (128 * 128 >> 4)), bd + (uint64_t)(j * ((BN / 2) * 128 >> 4)),
                                  idesc, (kb > kb0 || j > 0) ? 1u : 0u);
            } else {
              const int ks = k16_steps(p, kb);
#pragma unroll
              for (int k = 0; k < S::BK / 16; ++k)
                if (k < ks) tc_mma_bf16_pair(d_tmem, ad + 2 * k, bd + 2 * k, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
            }
            tc_commit_pair_mc(&empty[s], 0x3);
            ++it;
          }
        };
        if (p.k_full)
          kloop(BoolTag<true>{});
        else
          kloop(BoolTag<false>{});
        if (!ok) break;
        tc_commit_pair_mc(&tfull[a], 0x3);
      }
      tc_commit_pair_mc(drain, 0x1);
      mbar_wait_bounded(drain, 0, kDrainLimitNs, nullptr, 0);
    }
  } else {
    // epilogue: this CTA's 128 rows of the 256-row tile
    const int q = warp & 3;
    const int half = (warp - 2) / 4;  // column part (0..EPI_WARPS/4 - 1)
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&tempty[0]), 0);
    const int rank_rows = static_cast<int>(rank) * 128;
    const int ew = warp - 2;
    int tl = 0, groups = 0;
    PieceIter pi(p, pair, n_pairs);
    int t, kb0, kb1;
    for (; pi.next(p, t, kb0, kb1); ++tl) {
      const int a = tl & 1;
      const uint32_t aph = (tl >> 1) & 1;
      const int kind = piece_kind(p, kb0, kb1);
      int mb, nb;
      tile_coords(p, t, mb, nb);
      const int n0 = nb * BN;
      if ((EPI & EPI_RESID) && kind != PIECE_PARTIAL)
        epilogue_prefetch_l2(p, t, half, q, lane, BN, S::BM, rank_rows, S::CSTRIDE);
      float breg[4];
      load_bias(p, n0, BN, half, lane, breg, S::CSTRIDE);
      int r_first, r_last;
      subtile_rows(p, 2 * mb + static_cast<int>(rank), r_first, r_last);
      float4 pre[2][(EPI & EPI_LN) ? 8 : 1];  // LayerNorm epilogue: the first two groups' old rows
      if constexpr ((EPI & EPI_LN) != 0) {
        static_assert(BN == 256 && S::EPI_WARPS == 8, "LayerNorm epilogue: four groups per warp");
        const int row0 = r_first + 32 * q;
        for (int j = 0; j < 2; ++j)
          if (row0 < r_last && n0 + half * 32 + 64 * j < p.N) ln_load_x(p, row0, r_last, n0 + half * 32 + 64 * j, lane, pre[j]);
      }
      if (!mbar_wait_bounded(&tfull[a], aph, p.limit_ns, p.status, DEV_TIMEOUT_EPILOGUE)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + a * S::ACC_COLS;
      // Flag of this warp's rows and columns: the trailing piece of a split
      // tile is the first piece of the next pair, so it uses that pair's slot.
      const int slot = kind == PIECE_PARTIAL ? pair : pair + 1;
      int* flag = kind == PIECE_FULL ? nullptr : p.sk_flags + (slot * 2 + static_cast<int>(rank)) * S::EPI_WARPS + ew;
      bool have = true;
      if (kind == PIECE_OWNER) {
        if (lane == 0) {
          have = flag_wait_bounded(flag, p.limit_ns, p.status, DEV_TIMEOUT_EPILOGUE);
          fence_proxy_async_global();  // the bulk reduces below come after the trailing piece's
          // one split per flag and launch: clear it for the next launch (which
          // starts after this grid has completed)
          if (have) *flag = 0;
        }
        have = __shfl_sync(0xffffffffu, have, 0);
      }
      if constexpr ((EPI & EPI_LN) != 0)
        epilogue_warp_resid_ln<KIND>(p, tb, r_first + 32 * q, r_last, n0, half, lane, sEpi + ew * S::WBUF,
                                     nb * 2 + half, pre);
      else if (have)
        epilogue_warp<EPI, KIND, S::NBUF, S::BOXB>(p, &tmOut, tb, r_first + 32 * q, r_last, n0, BN, half, lane,
                                                   sEpi + ew * S::WBUF, breg, kind, S::CSTRIDE, &groups);
      tc_fence_before();
      __syncwarp();
      if (kind == PIECE_PARTIAL && lane == 0) {
        bulk_wait0();                 // this warp's bulk reduces have been performed
        fence_proxy_async_global();
        __threadfence();
        st_release_gpu(flag, 1);
      }
      if (lane == 0) mbar_arrive_cluster(tempty_leader0 + 8u * a);
    }
    if (lane == 0) bulk_wait0();  // bulk stores complete before the CTA exits
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the pair's MMAs are drained before either CTA frees TMEM
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, S::TMEM_COLS);
}

// bf16 and f16 operands (kind::f16), CTA pairs.
template <int BN, int STAGES, int EPI, int KP = 1>
__global__ void __launch_bounds__(Gemm2Shape<BN, STAGES, gemm2_epi_warps<EPI>(), gemm2_nbuf<BN>(), KP>::THREADS, 1)
    gemm_bf16_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                         const __grid_constant__ CUtensorMap tmOut, const GemmParams p) {
  gemm_tc2_body<BN, STAGES, EPI, KIND_BF16, KP>(tmA, tmB, tmOut, p);
}
template <int BN, int STAGES, int EPI, int KP = 1>
__global__ void __launch_bounds__(Gemm2Shape<BN, STAGES, gemm2_epi_warps<EPI>(), gemm2_nbuf<BN>(), KP>::THREADS, 1)
    gemm_f16_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmOut, const GemmParams p) {
  gemm_tc2_body<BN, STAGES, EPI, KIND_F16, KP>(tmA, tmB, tmOut, p);
}

}  // namespace asr

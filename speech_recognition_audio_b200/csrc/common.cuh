// Device helpers shared by the sm_100a kernels: PTX wrappers for mbarriers,
// TMA tiled loads, tcgen05 (UMMA / tensor memory) and bounded waits.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace asr {

typedef __nv_bfloat16 bf16;

// Device status codes written to the forward's status word.
enum : int { DEV_OK = 0, DEV_TIMEOUT_PRODUCER = 1, DEV_TIMEOUT_MMA = 2, DEV_TIMEOUT_EPILOGUE = 3,
             DEV_TIMEOUT_GATHER = 4, DEV_TIMEOUT_DRAIN = 5, DEV_TIMEOUT_PROBE = 6 };

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------- programmatic dependent launch
// Kernels are launched with programmatic stream serialisation: a kernel may
// start (prologue: barrier init, tensor-memory allocation, descriptor
// prefetch) while its predecessor is still finishing.  pdl_wait() blocks
// until the predecessor grid has completed and its memory is visible; every
// kernel calls it before its first global-memory access.  pdl_trigger() lets
// the successor begin launching; it still waits for this grid to complete.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(addr), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait until the barrier phase of the given parity has completed, for at most
// limit_ns of device time.  Also gives up early when the shared status word
// already holds an error (another role or block gave up).  On giving up it
// records `code` in *status and returns false.
static __device__ __noinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                               int* status, int code) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0;; ++it) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(a, parity)) return true;
    const uint64_t now = globaltimer_ns();
    if (now - t0 > limit_ns) {
      if (status) atomicCAS(status, 0, code);
      return false;
    }
    if (status && (it & 15) == 15 && *reinterpret_cast<volatile int*>(status) != 0) return false;
  }
}

// --------------------------------------------------------------- TMA loads
// 2-D tiled bulk tensor load into this CTA's shared memory, completing on
// `bar` (complete_tx).  No multicast.  x = innermost coordinate (elements).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------------------- cp.async
__device__ __forceinline__ void cp_async_16_zfill(void* dst, const void* src, bool valid) {
  const uint32_t n = valid ? 16u : 0u;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(n) : "memory");
}
// Arrive on `bar` once all of this thread's previously issued cp.async
// copies have completed; the barrier's expected count already includes
// this arrival (.noinc), and the issuing thread does not wait.
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive once on `bar` when all previously issued tcgen05.mma of this thread complete.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// The four K = 16 steps of one 64-element (128-byte) k-block in one asm
// statement: descriptors advance by 32 bytes (2 in the >> 4 address field)
// per step; the first step accumulates if `accumulate` != 0, the others
// always.  Issuing the steps of a whole k-block back to back, with no
// per-step guard between them, keeps the tensor pipe fed (per-step guarded
// issue measured about 10 % slower).
__device__ __forceinline__ void tc_mma4_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %5, %6, %3, 1;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %7, %8, %3, 1;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %9, %10, %3, 1;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "l"(adesc + 2), "l"(bdesc + 2), "l"(adesc + 4),
      "l"(bdesc + 4), "l"(adesc + 6), "l"(bdesc + 6)
      : "memory");
}
__device__ __forceinline__ void tc_mma4_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %5, %6, %3, 1;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %7, %8, %3, 1;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %9, %10, %3, 1;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "l"(adesc + 2), "l"(bdesc + 2), "l"(adesc + 4),
      "l"(bdesc + 4), "l"(adesc + 6), "l"(bdesc + 6)
      : "memory");
}
// 32 lanes x 32 bit, 16 consecutive columns starting at taddr (lane field = warp's quarter).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
// 32 lanes x 32 bit, 32 consecutive columns starting at taddr.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
      "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// 32 lanes x 32 bit, 16 consecutive columns written from v (lane field = warp's quarter).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15]))
      : "memory");
}
// This thread's tcgen05.st writes have completed.
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor for a K-major operand tile stored in the
// canonical 128-byte-swizzle layout (8-row x 128-byte atoms, 1024 bytes per
// atom, atoms stacked along M/N).  Fields: start address >> 4 (bits 0-13),
// leading byte offset (unused for swizzled K-major, 1), stride byte offset
// 1024 >> 4 (bits 32-45), descriptor version 1 (bits 46-47), swizzle mode
// 128B = 2 (bits 61-63).
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(1u) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// Descriptor of an MN-major operand tile in the 128-byte-swizzle layout:
// each K index is a 128-byte row of 64 bf16 MN elements, 8 rows form a
// 1024-byte swizzle atom and atoms follow along K (stride byte offset 1024);
// one atom wide along MN (leading byte offset unused).
__device__ __forceinline__ uint64_t sw128_mnmajor_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(1u) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// Instruction descriptor, kind::f16 with bf16 A/B, fp32 D, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// Operand kinds of the GEMM engine: bf16 (kind::f16), tf32 (kind::tf32,
// fp32 operands in memory, the tensor core reading their tf32 part), f16
// (kind::f16).  A 128-byte swizzled row holds 64 16-bit or 32 fp32 elements,
// and one MMA step takes 32 bytes of K: 16 or 8 elements.
enum : int { KIND_BF16 = 0, KIND_TF32 = 1, KIND_F16 = 2 };
__host__ __device__ constexpr int kind_row_elems(int kind) { return kind == KIND_TF32 ? 32 : 64; }
// Instruction descriptor of a kind: fp32 D, A and B K-major; A/B format
// fields (bits 7-9, 10-12): kind::f16 F16 = 0, BF16 = 1; kind::tf32 TF32 = 2.
__host__ __device__ constexpr uint32_t idesc_kind_f32(int kind, int M, int N) {
  return (1u << 4) | (kind == KIND_TF32 ? (2u << 7) | (2u << 10) : kind == KIND_F16 ? 0u : (1u << 7) | (1u << 10)) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}
// Two fp32 values rounded to nearest-even into a packed pair of the kind's
// 16-bit type (f16 for KIND_F16, else bf16), low half first.
template <int KIND>
__device__ __forceinline__ uint32_t pack2_16(float a, float b) {
  if constexpr (KIND == KIND_F16) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  } else {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
}
// Eight fp32 values as one 16-byte chunk of the kind's 16-bit type.
template <int KIND>
__device__ __forceinline__ uint4 pack8_16(const float* v) {
  return make_uint4(pack2_16<KIND>(v[0], v[1]), pack2_16<KIND>(v[2], v[3]), pack2_16<KIND>(v[4], v[5]),
                    pack2_16<KIND>(v[6], v[7]));
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::tf32 (fp32 operands, fp32 accumulate).
__device__ __forceinline__ void tc_mma_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// ---------------------------------------------------------------- math
// Packed fp32 pair arithmetic (the f32x2 instructions of sm_100): one
// instruction issues two IEEE fp32 operations with the usual rounding.
__device__ __forceinline__ unsigned long long f2_bits(float2 v) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(v.x), "f"(v.y));
  return r;
}
__device__ __forceinline__ float2 bits_f2(unsigned long long r) {
  float2 v;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(v.x), "=f"(v.y) : "l"(r));
  return v;
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(f2_bits(a)), "l"(f2_bits(b)), "l"(f2_bits(c)));
  return bits_f2(d);
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2_bits(a)), "l"(f2_bits(b)));
  return bits_f2(d);
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  unsigned long long d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2_bits(a)), "l"(f2_bits(b)));
  return bits_f2(d);
}
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// GELU(x) = x Phi(x) in the tanh form of Hendrycks & Gimpel (2016):
//   GELU(x) ~ 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))),
// which differs from the exact x Phi(x) by at most 4.8e-4 (near |x| = 2.7;
// below the rounding of a bf16 output there, 2^-9 |GELU|).  tanh comes from
// the hardware tanh.approx.f32 (relative error <= 2^-10.98), adding at most
// 2.5e-4 |x|.  Per pair of values: 4 packed fp32 operations and 2 tanh.
__device__ __forceinline__ float tanh_approx(float x) {
  float r;
  asm("tanh.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
// 2^x from the hardware ex2.approx.ftz.f32 (relative error ~2^-22; inputs
// below the normal range give 0, -inf gives 0).
__device__ __forceinline__ float ex2_approx(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
namespace gelu_tanh {
constexpr float k0 = 0.7978845608028654f;               // sqrt(2 / pi)
constexpr float k1 = 0.7978845608028654f * 0.044715f;   // sqrt(2 / pi) * 0.044715
}  // namespace gelu_tanh

__device__ __forceinline__ float2 gelu_erf2(float2 x) {
  using namespace gelu_tanh;
  const float2 u = mul2(x, fma2(mul2(x, x), make_float2(k1, k1), make_float2(k0, k0)));
  const float2 t = make_float2(tanh_approx(u.x), tanh_approx(u.y));
  const float2 h = mul2(x, make_float2(0.5f, 0.5f));
  return fma2(h, t, h);
}

__device__ __forceinline__ float gelu_erf(float x) {
  using namespace gelu_tanh;
  const float u = x * fmaf(x * x, k1, k0);
  const float h = 0.5f * x;
  return fmaf(h, tanh_approx(u), h);
}
__device__ __forceinline__ float silu(float x) { return x / (1.0f + __expf(-x)); }

// Order-preserving map of a float to an unsigned int (for atomicMax).
__device__ __forceinline__ unsigned int float_to_ordered(float f) {
  unsigned int u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float ordered_to_float(unsigned int u) {
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u);
}

}  // namespace asr

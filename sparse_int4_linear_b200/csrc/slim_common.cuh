// Shared device helpers for libslim (sm_100a): mbarrier + bulk-copy PTX
// wrappers, warp-level tensor-core MMAs, and the int4 -> bf16 decode.
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "slim.h"

namespace slim {

// One decode-stream chunk = 16 rows x 256 K of packed weights:
//   [0, 512)     lane-major 16-byte words, value words of MMA steps 0..3
//   [512, 1024)  value words of MMA steps 4..7
//   [1024, 1536) metadata words (each lane holds the 4 steps it supplies)
//   [1536, 1600) fp16 scales: 8 bytes per row pair (g, g + 8), g = 0..7, as
//                (group 0 row g, group 0 row g+8, group 1 row g, group 1
//                row g+8), so the lanes of MMA row group g read theirs with
//                one 8-byte load
constexpr int kDecChunk = 1600;

// Index (in fp16 units from byte 1536) of the scale of 128-group gg (0, 1)
// of the chunk and tile row rr (0..15).
__host__ __device__ __forceinline__ int scale_slot(int gg, int rr) { return (rr & 7) * 4 + gg * 2 + (rr >> 3); }
constexpr uint32_t kLayerMagic = 0x534c694du;  // "SLiM"

// Bounded waits give up after this many SM clock cycles (~1 s at 2 GHz).
constexpr long long kWaitBudgetCycles = 2000000000ll;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void record_status(int32_t* status, int32_t code) {
  if (status) atomicCAS(status, 0, code);
}

// Index check of the debug build: true when `ok`; otherwise records
// SLIM_ERR_BOUNDS and returns false, and the caller skips the access.  The
// release build returns true and the condition is compiled away.
#ifdef SLIM_DEBUG
__device__ __forceinline__ bool dcheck(bool ok, int32_t* status) {
  if (!ok) record_status(status, SLIM_ERR_BOUNDS);
  return ok;
}
#else
__device__ __forceinline__ bool dcheck(bool, int32_t*) { return true; }
#endif

// ------------------------------------------------------------ mbarrier / bulk copy
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
// 1-D bulk copy global -> this CTA's shared memory, completion on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Wait for phase `parity` of `bar`; false if it did not complete in budget.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitBudgetCycles) return false;
  }
  return true;
}
// After a wait gave up: wait, until `deadline` (clock64), for phase `parity`
// of `bar` to complete, so that a bulk copy this thread issued lands before
// the CTA exits (its destination is the CTA's own shared memory).  Returns
// at once for a phase that has completed.
__device__ __forceinline__ void drain_phase(uint64_t* bar, uint32_t parity, long long deadline) {
  while (!mbar_try_wait(bar, parity) && clock64() < deadline) {
  }
}

// Order this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (bulk copy) writes to the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------ shared loads
__device__ __forceinline__ uint4 lds128(const void* p) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(smem_u32(p)));
  return v;
}
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}

__device__ __forceinline__ void ldmatrix_x2(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(smem_u32(p)));
  r[2] = r[3] = 0u;
}

// The same loads on 32-bit shared-memory addresses (no generic-to-shared
// conversion per access in hot loops).
__device__ __forceinline__ uint4 lds128_s(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds16_s(uint32_t a) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ void ldmatrix_x4_s(uint32_t (&r)[4], uint32_t a) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a));
}
// The same with a constant byte offset folded into the instruction's
// address (no integer add per load in an unrolled loop).
template <int OFF>
__device__ __forceinline__ void ldmatrix_x4_so(uint32_t (&r)[4], uint32_t a) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4+%5];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a), "n"(OFF));
}
template <int OFF>
__device__ __forceinline__ uint4 lds128_so(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4+%5];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a),
               "n"(OFF));
  return v;
}
template <int OFF>
__device__ __forceinline__ void lds64_so(uint32_t a, uint32_t& x, uint32_t& y) {
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2+%3];" : "=r"(x), "=r"(y) : "r"(a), "n"(OFF));
}
__device__ __forceinline__ bool mbar_try_wait_s(uint32_t a, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(a), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_s(uint32_t a, uint32_t parity) {
  if (mbar_try_wait_s(a, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait_s(a, parity)) {
    if (clock64() - t0 > kWaitBudgetCycles) return false;
  }
  return true;
}

// ------------------------------------------------------------ warp MMAs
// Structured-sparse m16n8k32 bf16 -> fp32.  A is 16 x 32 with 2 of every 4
// k kept (8 bf16 per lane); `e` holds the 2-bit positions; F selects which
// thread pair of each quad supplies `e` (0: lanes t=0,1; 1: lanes t=2,3).
template <int F>
__device__ __forceinline__ void mma_sp_16832(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[4],
                                             uint32_t e) {
  asm(
      "mma.sp::ordered_metadata.sync.aligned.m16n8k32.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9,%10,%11}, {%0,%1,%2,%3}, %12, %13;\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]), "r"(b[2]), "r"(b[3]), "r"(e),
        "n"(F));
}
// Dense m16n8k16 bf16 -> fp32.
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint4& a, uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b0), "r"(b1));
}

// ------------------------------------------------------------ int4 decode
// A value word holds 4 pairs of biased nibbles u = q + 8: pair p has its
// first value at bits [4p, 4p+4) and its second at [16+4p, 20+4p).  The
// bf16 with bits 0x4300 | u is exactly 128 + u, so subtracting 136 gives q
// exactly.
__device__ __forceinline__ void decode_word(uint32_t w, uint32_t (&a)[4]) {
  const __nv_bfloat162 bias = __halves2bfloat162(__ushort_as_bfloat16(0x4308), __ushort_as_bfloat16(0x4308));
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    uint32_t x = ((w >> (4 * p)) & 0x000F000Fu) | 0x43004300u;
    __nv_bfloat162 v = __hsub2(*reinterpret_cast<__nv_bfloat162*>(&x), bias);
    a[p] = *reinterpret_cast<uint32_t*>(&v);
  }
}

// fp16 bits -> fp32 with integer operations and one multiply: the 15 low
// bits shifted into place give the fp32 whose value is 2^-112 times the fp16
// value (for subnormal fp16 too, as an fp32 subnormal), and scaling by 2^112
// is exact.  Keeps the conversion off the special-function pipe.
__device__ __forceinline__ float f16_bits_to_f32(uint32_t h) {
  return __uint_as_float(((h & 0x7fffu) << 13) | ((h & 0x8000u) << 16)) * 0x1p112f;
}

// The same for a non-negative fp16 (the packed scales: fp16 of amax / 7),
// whose sign bit is clear: one shift and one multiply.
__device__ __forceinline__ float f16_nonneg_bits_to_f32(uint32_t h) {
  return __uint_as_float(h << 13) * 0x1p112f;
}

// ------------------------------------------------------------ global flags
__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_u32(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Tag of one launch of the single-launch decode kernel, carried in the high
// half of the 64-bit words it leaves in a workspace (seq = the workspace's
// launch count).  Tags lie in [0x7F800001, 0x7FBFFFFE]: read as the high
// half of a word of fp32 data that is an fp32 NaN, of bf16 or fp16 data a
// +Inf or a NaN, of tensor-core metadata words an invalid 2:4 position
// pair.  So no word that any kernel of the library writes from finite data
// (T tiles, weight images, fp32 partial sums) can look like a current tag,
// whatever layer or path used the workspace before; consecutive launches
// differ, and a tag repeats only after 2^22 - 2 launches.
__host__ __device__ __forceinline__ uint32_t launch_tag(uint32_t seq) { return 0x7F800001u + seq % 0x3FFFFEu; }

// 64-bit words read and written as single accesses (a value and its tag
// arrive together).
__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// ------------------------------------------------------------ programmatic dependent launch
// Let the next kernel on the stream start launching (it still waits for this
// grid's completion before reading what this grid writes).
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// Wait until every grid this one depends on has completed and its memory is
// visible; a no-op when the kernel was launched without such a dependency.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// ------------------------------------------------------------ 4-bit adapters
// Layouts of the adapter factors quantized to 4 bits (symmetric, fp16 scale
// per 128 entries along the reduction dimension).  Both hold the A operand
// of the dense m16n8k16 MMA in fragment order, as the bf16 layouts Lf / Rf
// do, with every bf16 replaced by a biased nibble u = q + 8 that
// decode_word() expands: one 32-bit word per lane per 16 x 16 step.
//   Lq  A = L^T [rl16 rows][K]: block (jt, kg) of 16 adapter columns x 128 K
//       at (jt * K/128 + kg) * kLqBlock: 8 steps x 32 lanes x 4 bytes, then
//       the 16 columns' fp16 scales (slot frag_scale_slot(row)).
//   Rq  A = R^T [N16 rows][r16]: row tile rt at rt * rq_tile_bytes(): JS =
//       r16/16 steps x 32 lanes x 4 bytes, then per 128-group of r the 16
//       rows' fp16 scales (32 bytes a group, slots as for Lq).
constexpr int kLqBlock = 8 * 128 + 32;
__host__ __device__ __forceinline__ int rq_groups(int r) { return (r + 127) / 128; }
__host__ __device__ __forceinline__ int rq_tile_bytes(int r16, int r) { return r16 / 16 * 128 + rq_groups(r) * 32; }
// Element (row, k) of a 16 x 16 step: lane (row % 8) * 4 + (k % 8) / 2 holds
// it, in register (row / 8) + 2 (k / 8), first (even k) or second half.
__host__ __device__ __forceinline__ int frag_lane(int row, int k) { return (row & 7) * 4 + ((k & 7) >> 1); }
__host__ __device__ __forceinline__ int frag_shift(int row, int k) {
  return 4 * ((row >> 3) + 2 * (k >> 3)) + 16 * (k & 1);
}
// Scales of rows g and g + 8 share one 32-bit word (g low, g + 8 high).
__host__ __device__ __forceinline__ int frag_scale_slot(int row) { return 2 * (row & 7) + (row >> 3); }

// Byte offset of bf16 element (row, col) in a K-major operand tile of
// `rows` rows stored as 128-byte-swizzled atoms: each atom holds 64 columns
// (128 bytes) of every row, 8-row groups of 1024 bytes, and the 16-byte
// chunk index of a row is XORed with (row % 8).  This is the layout the
// tensor cores read through a SWIZZLE_128B shared-memory descriptor and the
// layout a SWIZZLE_128B tensor copy writes; atoms must be 1024-byte aligned.
__host__ __device__ __forceinline__ uint32_t sw128_offset(int row, int col, int rows) {
  const int atom = col >> 6, c = col & 63;
  return (uint32_t)(atom * rows * 128 + (row >> 3) * 1024 + (row & 7) * 128 +
                    ((((c * 2) >> 4) ^ (row & 7)) << 4) + ((c * 2) & 15));
}

}  // namespace slim

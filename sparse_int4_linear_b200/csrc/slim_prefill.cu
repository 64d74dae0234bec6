// Tensor-core prefill forward for M > 16 tokens (sm_100a, tcgen05).
//
// Many tokens reuse every weight, so this path is compute-bound (thesis
// §2.5.1 "The Compute-Bound Regimes: Training and Prefill") and the 2:4
// structure is exploited by the sparse tensor cores, which skip the pruned
// products (§2.2.3 "Sparse Tensor Core Acceleration").
//
// After T = X L, a pre-dequantization pass and one of two MMA kernels:
//   k_predequant  packed decode stream -> per (128 rows x 128 K) tile a
//                 16 KB image of bf16(q * s) in the 128-byte-swizzled layout
//                 of the sparse MMA's A operand, and a 2 KB image of the 2:4
//                 metadata words in tensor-memory lane order (bandwidth-bound;
//                 each weight is expanded once per call, not once per token
//                 tile);
//   k_prefill2    a cluster of two CTAs on an SM pair = 512 layer rows x TT
//                 tokens (TT up to 240): tcgen05.mma.sp.cta_group::2 with
//                 M = 256 takes 128 rows and TT/2 tokens from each CTA, so each
//                 SM stores and reads half of the X tile;
//   k_prefill     one CTA = 128 or 256 layer rows x 64 to 192 tokens:
//                 tcgen05.mma.sp.kind::f16 per 128-row half sharing one X tile.
// Both MMA kernels keep fp32 accumulators in tensor memory, load X by TMA
// (SWIZZLE_128B) and the images by bulk or tensor copies, move metadata into
// tensor memory with tcgen05.cp, run the adapter R^T T^T as dense tcgen05.mma
// stages ahead of the sparse ones in the same rings, and end with a bf16
// epilogue staged through shared memory.  The tile is picked per call from
// how the CTAs fill the SMs.
// T = X L itself runs first on the tensor cores (k_tgemm): 128 tokens x
// r per CTA, K split over a cluster, partial sums added in rank order through
// distributed shared memory, written straight into the swizzled T tiles.
#include <cooperative_groups.h>
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include "slim_common.cuh"
#include "slim_internal.h"

namespace slim {
namespace {

constexpr int TILE_ROWS = 128;                 // rows per image tile / per MMA
constexpr int kImgA = TILE_ROWS * 64 * 2;      // 16 KB: one swizzled atom of 128 rows x 64 values
constexpr int kImgM = TILE_ROWS * 16;          // 2 KB: 128 lanes x 4 metadata words
constexpr int kImg = kImgA + kImgM;            // per (128-row tile, 128-K group)
constexpr int kRowBytes = 1024;                // byte buffers seen by a tensor map as rows of 128 u64
constexpr int kImgRows = kImg / kRowBytes;     // 18 rows per image
static_assert(kImg % kRowBytes == 0 && kImgA % kRowBytes == 0, "images and atoms are whole tensor-map rows");
constexpr int kTmemCols = 512;
constexpr int kAccCol = 0;                     // half h accumulator at h * TT
constexpr int kThreads = 320;

// CTA tile: NH 128-row halves (256 or 128 rows) x TT tokens (the MMA's N:
// 192, 128 or 64), picked per call by how the tiles fill the SMs.  The X
// ring holds 96 KB and the A ring 108 KB for every shape.
template <int TT_, int NH_>
struct PfCfg {
  static constexpr int TT = TT_;
  static constexpr int NH = NH_;
  static constexpr int kCtaRows = NH_ * TILE_ROWS;
  static constexpr int kXStage = TT_ * 128;              // TT tokens x 64 K bf16, one swizzled atom
  static constexpr int NX = 96 * 1024 / kXStage;         // X stages of 64 K
  static constexpr int kAStage = NH_ * kImg;             // images of the CTA's halves, 128 K
  static constexpr int NA = NH_ == 2 ? 3 : 6;            // A stages
  static constexpr int kOffX = 0;
  static constexpr int kOffA = kOffX + NX * kXStage;     // 96 KB
  static constexpr int kOffBar = kOffA + NA * kAStage;   // + 108 KB
  // x_full x_empty [NX], a_full a_empty [NA], acc_full
  static constexpr int kNumBars = 2 * NX + 2 * NA + 1;
  static constexpr int kSmemBytes = kOffBar + kNumBars * 8 + 16 + 1024;
  static constexpr int kMetaCol = NH_ * TT_;             // half h, slot a, step jl at kMetaCol + (h * NA + a) * 4 + jl
  static_assert(kAStage >= NH_ * kImgA, "an adapter stage (R^T atoms of the CTA's halves) fits an A slot");
  static_assert(TT_ <= kPrefillMaxTile, "T workspace is sized for tiles of at most kPrefillMaxTile tokens");
};

struct PrefillParams {
  const uint8_t* img;     // dequantized images, [4 * ceil(N/512)][K/128][kImg]
  const uint8_t* Rp;      // pre-swizzled R^T, 128-row tiles of r64 columns
  const uint8_t* Tswz;    // T tiles of TT tokens x r64 columns, swizzled
  uint16_t* Y;
  int M, N, K, r16;
  int n_groups;                         // fused linears (T tiles hold n_groups * r64 columns)
  int group_end[SLIM_MAX_GROUPS];       // rows of fused linear g end at group_end[g]
  int32_t* status;
};

// ------------------------------------------------------------ tcgen05 / TMA wrappers
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  // K-major, 128-byte swizzle: start >> 4, LBO 16 B (unused), SBO 1024 B
  // between 8-row groups, descriptor version 1, layout type 2.
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
__device__ __forceinline__ void mma_sp(uint32_t d, uint64_t a, uint64_t b, uint32_t e, uint32_t idesc, int acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.sp.cta_group::1.kind::f16 [%0], %1, %2, [%3], %5, {%6, %6, %6, %6}, p;\n}\n" ::"r"(d),
      "l"(a), "l"(b), "r"(e), "r"(acc), "r"(idesc), "r"(0u)
      : "memory");
}
__device__ __forceinline__ void mma_dense(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, int acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %3, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %4, {%5, %5, %5, %5}, p;\n}\n" ::"r"(d),
      "l"(a), "l"(b), "r"(acc), "r"(idesc), "r"(0u)
      : "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
// Shared-memory descriptor of the metadata image: 128 rows of 16 bytes (no
// swizzle, K-major: rows 16 B apart inside an 8-row core matrix, core
// matrices 128 B apart), the source of a 128-lane x 128-bit tensor-memory copy.
__device__ __forceinline__ uint64_t meta_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(128 >> 4) << 16) | ((uint64_t)(128 >> 4) << 32) |
         ((uint64_t)1 << 46);
}
// Copy 128 lanes x 4 words from shared memory into tensor memory columns
// [taddr, taddr + 4): ordered before the MMAs this thread issues after it.
__device__ __forceinline__ void tc_cp_meta(uint32_t taddr, uint64_t desc) {
  asm volatile("tcgen05.cp.cta_group::1.128x128b [%0], %1;" ::"r"(taddr), "l"(desc) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Named barrier 1 of the 256 epilogue threads that also returns the OR of
// `v` over them.
__device__ __forceinline__ bool epi_bar_or(bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, 1, 256, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

// Bounded wait that gives up at once when another role has already given up.
__device__ __forceinline__ bool pwait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitBudgetCycles) {
      *abort_flag = 1;
      return false;
    }
  }
  return true;
}

// ---------------------------------------------------------------- pre-dequant
// Grid (K/128 groups, 128-row tiles incl. padding up to a multiple of 2), 128
// threads.  Source: the group's half of 8 decode-stream chunks (16-row tiles
// x 256 K).  Thread slot (row tile m2, chunk lane l) expands one 16-byte value
// word-set: pairs (v0, v1) of rows g / g+8 for blocks t / t+4 of 4 MMA steps.
// Launched as a dependent of T = X L (when there is an adapter), which signals
// right after its own grid-dependency wait: the images of the previous call
// are then no longer read, so this kernel writes them at once and waits for
// T = X L only at its end, so that the main kernel (which waits for this one)
// sees T.  Without an adapter it waits first (`wait_first`).
__global__ void __launch_bounds__(128) k_predequant(const uint8_t* __restrict__ dec, int NKB, int NRT, int S,
                                                    uint8_t* __restrict__ img, int wait_first) {
  if (wait_first) pdl_wait();
  __shared__ __align__(1024) uint8_t at[kImgA];
  const int s = blockIdx.x, tile = blockIdx.y;
  const int G = s & 1, kb = s >> 1;
  const int tg = threadIdx.x;
  const int rt0 = tile * 8;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int li = tg + half * 128;
    const int m2 = li >> 5, l = li & 31, g = l >> 2, t = l & 3;
    const bool valid = rt0 + m2 < NRT;
    const uint8_t* ch = dec + ((size_t)(rt0 + m2) * NKB + kb) * kDecChunk;
    uint4 vw = make_uint4(0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u);
    float s_lo = 0.f, s_hi = 0.f;
    if (valid) {
      vw = __ldg(reinterpret_cast<const uint4*>(ch + G * 512 + l * 16));
      const __half* sc = reinterpret_cast<const __half*>(ch + 1536);
      s_lo = __half2float(sc[scale_slot(G, g)]);
      s_hi = __half2float(sc[scale_slot(G, g + 8)]);
    }
    const uint32_t words[4] = {vw.x, vw.y, vw.z, vw.w};
#pragma unroll
    for (int jl = 0; jl < 4; ++jl) {
      const uint32_t w = words[jl];
#pragma unroll
      for (int pr = 0; pr < 4; ++pr) {
        const int row = 16 * m2 + g + 8 * (pr & 1);
        const int cc = 16 * jl + 2 * (t + 4 * (pr >> 1));
        const float sv = (pr & 1) ? s_hi : s_lo;
        const float f0 = (float)((int)((w >> (4 * pr)) & 15u) - 8) * sv;
        const float f1 = (float)((int)((w >> (16 + 4 * pr)) & 15u) - 8) * sv;
        *reinterpret_cast<__nv_bfloat162*>(at + sw128_offset(row, cc, 128)) = __floats2bfloat162_rn(f0, f1);
      }
    }
  }
  // Metadata words of lane L = tg for the 4 MMA steps of this group.
  uint8_t* out = img + ((size_t)tile * S + s) * kImg;
  {
    const int L = tg, mm2 = L >> 4, mp = (L >> 3) & 1, mm0 = L & 7;
    const bool valid = rt0 + mm2 < NRT;
    const uint8_t* ch = dec + ((size_t)(rt0 + mm2) * NKB + kb) * kDecChunk;
    uint32_t e[4];
#pragma unroll
    for (int jl = 0; jl < 4; ++jl) {
      const int j = 4 * G + jl;
      const int owner = mm0 * 4 + (j & 1) * 2 + mp;
      e[jl] = valid ? __ldg(reinterpret_cast<const uint32_t*>(ch + 1024 + owner * 16 + (j >> 1) * 4)) : 0x44444444u;
    }
    *reinterpret_cast<uint4*>(out + kImgA + L * 16) = make_uint4(e[0], e[1], e[2], e[3]);
  }
  __syncthreads();
  for (int i = tg; i < kImgA / 16; i += 128)
    reinterpret_cast<uint4*>(out)[i] = reinterpret_cast<const uint4*>(at)[i];
  pdl_wait();
}

// ---------------------------------------------------------------- main kernel
// Warp roles (320 threads):
//   warps 0-7  the epilogue (warps 0-3: rows 0-127, 4-7: rows 128-255)
//   warp 8     producer: A/metadata images (bulk copies), X tiles (TMA),
//              then the adapter tiles
//   warp 9     tensor-memory allocation and the single-thread issue of the
//              metadata copies into tensor memory and of the MMAs
template <int TT_, int NH_>
__global__ void __launch_bounds__(kThreads, 1) k_prefill(const __grid_constant__ CUtensorMap tmap_x,
                                                         const PrefillParams p) {
  using C = PfCfg<TT_, NH_>;
  constexpr int TT = C::TT, NH = C::NH, NX = C::NX, NA = C::NA, kXStage = C::kXStage, kAStage = C::kAStage;
  constexpr int kOffX = C::kOffX, kOffA = C::kOffA, kCtaRows = C::kCtaRows;
  constexpr int kOffBar = C::kOffBar, kNumBars = C::kNumBars, kMetaCol = C::kMetaCol;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* xs = smem + kOffX;
  uint8_t* as = smem + kOffA;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* x_full = bars;
  uint64_t* x_empty = bars + NX;
  uint64_t* a_full = bars + 2 * NX;
  uint64_t* a_empty = a_full + NA;
  uint64_t* acc_full = a_empty + NA;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(bars + kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + kNumBars) + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = p.K / 128;                      // A stages (128 K)
  const int t0 = blockIdx.x * TT;            // token tile (fastest: CTAs of a row pair share its images in L2)
  const int rp = blockIdx.y;                  // block of NH 128-row image tiles
  const int r64 = ceil_div(p.r16, 64) * 64;
  // Pipeline stages: first the adapter, one 64-column atom of T R per stage
  // (R^T atoms of the CTA's halves in an A slot, the T atom in an X slot),
  // then the K groups of 128 (images of the halves, two X slots).
  const int NAD = r64 / 64;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NX; ++i) {
      mbar_init(x_full + i, 1);
      mbar_init(x_empty + i, 1);
    }
    for (int i = 0; i < NA; ++i) {
      mbar_init(a_full + i, 1);
      mbar_init(a_empty + i, 1);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32((const void*)tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_x)) : "memory");
      // The images and T were written by the previous kernels on the stream.
      pdl_wait();
      const uint8_t* img0 = p.img + (size_t)(NH * rp) * S * kImg;
      const uint8_t* rp0 = p.Rp + (size_t)(NH * rp) * r64 * 256;
      // Debug build: the row block's image and R^T tiles lie inside their buffers
      // (4 * ceil(N/512) tiles of 128 rows), and the T tiles of this token tile exist.
      if (!dcheck((NH * rp + NH) * 128 <= ceil_div(p.N, 512) * 512 && t0 < p.M, p.status)) *abort_flag = 1;
      // T columns of this row block's fused linear: atoms [grp * r64/64, ...)
      int grp = 0;
      while (grp + 1 < p.n_groups && rp * kCtaRows >= p.group_end[grp]) ++grp;
      const uint8_t* tt = p.Tswz + (size_t)blockIdx.x * p.n_groups * r64 * (TT * 2) + (size_t)grp * (r64 / 64) * kXStage;
      int xs_i = 0;   // X slots filled so far
      int a_iss = 0;  // A slots filled so far
      for (int u = 0; u < NAD + S; ++u) {
        const int a = u % NA;
        if (!pwait(a_empty + a, ((u / NA) & 1) ^ 1, abort_flag)) break;
        ++a_iss;
        if (u < NAD) {
          mbar_expect_tx(a_full + a, NH * kImgA);
#pragma unroll
          for (int h = 0; h < NH; ++h)
            bulk_g2s(as + a * kAStage + h * kImgA, rp0 + (size_t)h * r64 * 256 + (size_t)u * kImgA, kImgA, a_full + a);
        } else {
          const int s = u - NAD;
          mbar_expect_tx(a_full + a, NH * kImg);
#pragma unroll
          for (int h = 0; h < NH; ++h)
            bulk_g2s(as + a * kAStage + h * kImg, img0 + ((size_t)h * S + s) * kImg, kImg, a_full + a);
        }
        bool ok = true;
        for (int x = 0; x < (u < NAD ? 1 : 2); ++x, ++xs_i) {
          const int xi = xs_i % NX;
          if (!pwait(x_empty + xi, ((xs_i / NX) & 1) ^ 1, abort_flag)) { ok = false; break; }
          mbar_expect_tx(x_full + xi, kXStage);
          if (u < NAD)
            bulk_g2s(xs + xi * kXStage, tt + (size_t)u * kXStage, kXStage, x_full + xi);
          else
            tma_load_2d(xs + xi * kXStage, &tmap_x, (2 * (u - NAD) + x) * 64, t0, x_full + xi);
        }
        if (!ok) break;
      }
      if (*abort_flag) {
        // Let the copies still in flight land before the CTA exits.
        const long long deadline = clock64() + kWaitBudgetCycles;
        for (int j = max(0, a_iss - NA); j < a_iss; ++j) drain_phase(a_full + j % NA, (j / NA) & 1, deadline);
        for (int j = max(0, xs_i - NX); j < xs_i; ++j) drain_phase(x_full + j % NX, (j / NX) & 1, deadline);
      }
    }
  } else if (warp == 9) {
    // ---------------------------------------------------------------- MMA issue
    if (lane == 0) {
      const uint32_t idesc_sp = (1u << 2) | (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(TT >> 3) << 17) |
                                ((uint32_t)(TILE_ROWS >> 4) << 24);
      const uint32_t idesc_dn = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(TT >> 3) << 17) |
                                ((uint32_t)(TILE_ROWS >> 4) << 24);
      const uint32_t xs_a = smem_u32(xs), as_a = smem_u32(as);
      int xs_i = 0;
      for (int u = 0; u < NAD + S; ++u) {
        const int a = u % NA;
        if (!pwait(a_full + a, (u / NA) & 1, abort_flag)) break;
        tc_fence_after();
        bool ok = true;
        if (u < NAD) {
          // T R for adapter columns 64u ... (whole 16-column steps only).
          const int xi = xs_i % NX;
          if (!pwait(x_full + xi, (xs_i / NX) & 1, abort_flag)) break;
          tc_fence_after();
          const int kks = min(4, (p.r16 - 64 * u) / 16);
          for (int kk = 0; kk < kks; ++kk) {
            const uint64_t bd = sw128_desc(xs_a + xi * kXStage + kk * 32);
#pragma unroll
            for (int h = 0; h < NH; ++h)
              mma_dense(tmem + kAccCol + h * TT, sw128_desc(as_a + a * kAStage + h * kImgA + kk * 32), bd, idesc_dn,
                        (u | kk) != 0);
          }
          tc_commit(x_empty + xi);
          ++xs_i;
        } else {
          const int s = u - NAD;
          // This stage's metadata words (all row halves) into their tensor-
          // memory slots; the slot was last read by the MMAs NA stages ago,
          // which completed before the slot was reloaded.
#pragma unroll
          for (int h = 0; h < NH; ++h)
            tc_cp_meta(tmem + (uint32_t)(kMetaCol + (h * NA + a) * 4),
                       meta_desc(as_a + a * kAStage + h * kImg + kImgA));
          for (int x = 0; x < 2; ++x, ++xs_i) {
            const int xi = xs_i % NX;
            if (!pwait(x_full + xi, (xs_i / NX) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
              const int jl = 2 * x + k2;
              const uint64_t bd = sw128_desc(xs_a + xi * kXStage + k2 * 64);
#pragma unroll
              for (int h = 0; h < NH; ++h) {
                const uint64_t ad = sw128_desc(as_a + a * kAStage + h * kImg + jl * 32);
                const uint32_t mcol = kMetaCol + (h * NA + a) * 4 + jl;
                mma_sp(tmem + kAccCol + h * TT, ad, bd, tmem + (mcol & ~1u), idesc_sp | (mcol & 1u),
                       NAD > 0 || (s | jl) != 0);
              }
            }
            tc_commit(x_empty + xi);
          }
        }
        if (!ok) break;
        tc_commit(a_empty + a);
      }
      tc_commit(acc_full);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int h = warp >> 2;                  // row half
    const int wq = warp & 3;                  // tensor-memory lane quarter
    const int L = wq * 32 + lane;
    // The MMA thread commits acc_full whether or not its loop completed, so
    // this wait also guarantees that no MMA is in flight when tensor memory
    // is freed.
    const bool acc_ok = mbar_wait(acc_full, 0);
    tc_fence_after();
    pdl_launch_dependents();
    pdl_wait();   // Y may still be in use by earlier work on the stream
    // Accumulators -> bf16 tile [token][row] in the (free) X ring, then
    // coalesced row-major stores of Y.  The named barrier is reached by all
    // 256 epilogue threads whatever happened before it.
    uint16_t* stage = reinterpret_cast<uint16_t*>(xs);
    // Warp-uniform: the tensor-memory loads below are .sync.aligned.
    const bool stage_ok = __all_sync(0xffffffffu, acc_ok && !*abort_flag);
    if (stage_ok && h < NH) {
      const int rloc = h * TILE_ROWS + L;
      for (int c0 = 0; c0 < TT; c0 += 32) {
        uint32_t v[32];
        const uint32_t taddr = tmem + ((uint32_t)(wq * 32) << 16) + (uint32_t)(kAccCol + h * TT + c0);
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
            "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
              "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
              "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),
              "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]),
              "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
            : "r"(taddr)
            : "memory");
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
        for (int c = 0; c < 32; ++c)
          stage[(c0 + c) * kCtaRows + rloc] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[c])));
      }
    }
    // One decision for the tile: stored as zeros if any wait gave up.
    const bool bad = epi_bar_or(!stage_ok);
    if (bad && threadIdx.x == 0) record_status(p.status, SLIM_ERR_TIMEOUT);
    {
      const int n0 = rp * kCtaRows;
      const int ntok = min(TT, p.M - t0);
      const int tid = threadIdx.x;   // 0..255
      if ((p.N & 7) == 0 && n0 + kCtaRows <= p.N) {
        for (int i = tid; i < ntok * (kCtaRows / 8); i += 256) {
          const int tk = i / (kCtaRows / 8), c8 = i % (kCtaRows / 8);
          if (!dcheck(t0 + tk < p.M, p.status)) continue;
          *reinterpret_cast<uint4*>(p.Y + (size_t)(t0 + tk) * p.N + n0 + c8 * 8) =
              bad ? make_uint4(0u, 0u, 0u, 0u) : *reinterpret_cast<const uint4*>(stage + tk * kCtaRows + c8 * 8);
        }
      } else {
        for (int i = tid; i < ntok * kCtaRows; i += 256) {
          const int tk = i / kCtaRows, rr = i % kCtaRows;
          if (n0 + rr < p.N) p.Y[(size_t)(t0 + tk) * p.N + n0 + rr] = bad ? (uint16_t)0 : stage[tk * kCtaRows + rr];
        }
      }
    }
  }
  if (*abort_flag && threadIdx.x == 0) record_status(p.status, SLIM_ERR_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// ---------------------------------------------------------------- 2-SM kernel
// A cluster of two CTAs on an SM pair computes 512 rows x TT tokens with
// tcgen05.mma(.sp).cta_group::2.  Each M = 256 MMA takes 128 rows from each
// CTA and half of the TT tokens from each, so for the same MMA work per SM
// every CTA stores and reads half the X tile the one-SM kernel does (its
// shared-memory traffic, which bounds the one-SM kernel, drops by a third).
// Rank 0 issues every tensor-core instruction for both CTAs; its commits
// arrive on the barriers of both CTAs (multicast).  Each CTA loads its own
// rows and tokens with its own tensor copies, and the copies of both CTAs
// complete on rank 0's stage barriers (.cta_group::2 form), whose expected
// byte count rank 0 sets for the pair: no thread relays a stage.  The
// adapter product T R runs first, as ordinary stages of the same rings.
//   warps 0-7  epilogue of this CTA's 256 rows (two 128-row blocks)
//   warp 8     producer: R^T and this CTA's half of T, then its images and
//              its half of X
//   warp 9     tensor-memory allocation (both CTAs); MMA issue (rank 0)
template <int TT_>
struct Pf2Cfg {
  static constexpr int TT = TT_;
  static constexpr int TH = TT_ / 2;                     // tokens this CTA holds
  static constexpr int kXStage = TH * 128;               // TH tokens x 64 K bf16, one swizzled atom
  static constexpr int NX = TT_ <= 192 ? 96 * 1024 / kXStage : 7;   // X stages of 64 K
  static constexpr int kAStage = 2 * kImg;               // this CTA's two 128-row tiles, 128 K
  static constexpr int NA = 3;
  static constexpr int kOffX = 0;
  static constexpr int kOffA = kOffX + NX * kXStage;     // 96 KB
  static constexpr int kOffBar = kOffA + NA * kAStage;   // + 108 KB
  static_assert(TT_ % 16 == 0 && TT_ <= 240, "MMA N of the pair: a multiple of 16; 2 TT + 24 tensor-memory columns");
  static_assert(TT_ <= kPrefillMaxTile, "T workspace is sized for tiles of at most kPrefillMaxTile tokens");
  static_assert(TT_ * 512 <= kOffBar, "epilogue staging exceeds the rings");
  static_assert(kAStage >= 2 * kImgA, "an adapter stage (R^T atoms of both row groups) fits an A slot");
  // x_full x_empty [NX], a_full a_empty [NA], acc_full
  static constexpr int kNumBars = 2 * NX + 2 * NA + 1;
  static constexpr int kSmemBytes = kOffBar + kNumBars * 8 + 16 + 1024;
  static constexpr int kMetaCol = 2 * TT_;               // group h, slot a, step jl at kMetaCol + (h * NA + a) * 4 + jl
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ void mma_sp2(uint32_t d, uint64_t a, uint64_t b, uint32_t e, uint32_t idesc, int acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.sp.cta_group::2.kind::f16 [%0], %1, %2, [%3], %5, {%6, %6, %6, %6, %6, %6, %6, %6}, p;\n}\n" ::"r"(d),
      "l"(a), "l"(b), "r"(e), "r"(acc), "r"(idesc), "r"(0u)
      : "memory");
}
__device__ __forceinline__ void mma_dense2(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, int acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %3, 0;\n"
      " tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %4, {%5, %5, %5, %5, %5, %5, %5, %5}, p;\n}\n" ::"r"(d),
      "l"(a), "l"(b), "r"(acc), "r"(idesc), "r"(0u)
      : "memory");
}
// Tensor copy into this CTA's shared memory that completes on a barrier of
// either CTA of the pair (bar: a shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
  return a;
}
__device__ __forceinline__ void tc_cp_meta2(uint32_t taddr, uint64_t desc) {
  asm volatile("tcgen05.cp.cta_group::2.128x128b [%0], %1;" ::"r"(taddr), "l"(desc) : "memory");
}
// Arrive (when the tensor-core work issued so far is done) on the barrier at
// this shared-memory offset in both CTAs of the pair.
__device__ __forceinline__ void tc_commit2(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"((uint16_t)3)
      : "memory");
}
// Same, to the barriers of the CTAs in `mask` only.
__device__ __forceinline__ void tc_commit2_mask(uint64_t* bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(mask)
      : "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

template <int TT_>
__global__ void __launch_bounds__(kThreads, 1) k_prefill2(const __grid_constant__ CUtensorMap tmap_x,
                                                          const __grid_constant__ CUtensorMap tmap_img,
                                                          const __grid_constant__ CUtensorMap tmap_rp,
                                                          const __grid_constant__ CUtensorMap tmap_t,
                                                          const PrefillParams p) {
  using C = Pf2Cfg<TT_>;
  constexpr int TT = C::TT, TH = C::TH, NX = C::NX, NA = C::NA, kXStage = C::kXStage, kAStage = C::kAStage;
  constexpr int kOffX = C::kOffX, kOffA = C::kOffA, kOffBar = C::kOffBar, kNumBars = C::kNumBars;
  constexpr int kMetaCol = C::kMetaCol;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* xs = smem + kOffX;
  uint8_t* as = smem + kOffA;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* x_full = bars;        // rank 0's count both CTAs' copies
  uint64_t* x_empty = x_full + NX;
  uint64_t* a_full = x_empty + NX;
  uint64_t* a_empty = a_full + NA;
  uint64_t* acc_full = a_empty + NA;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(bars + kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + kNumBars) + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int S = p.K / 128;
  const int ptile = blockIdx.x >> 1;                   // the pair's token tile
  const int t0 = ptile * TT;                           // the pair's first token
  const int pb = blockIdx.y;                           // 512-row block
  const int r64 = ceil_div(p.r16, 64) * 64;
  // Pipeline stages: first the adapter, one 64-column atom of T R per stage
  // (R^T atoms of both row groups in an A slot, this CTA's half of the T
  // atom in an X slot), then the K groups of 128 (two images, two X slots).
  const int NAD = r64 / 64;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) mbar_init(bars + i, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32((const void*)tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  // Both CTAs' barriers are initialised and tensor memory allocated before any
  // remote arrive or pair-wide tensor-core instruction.
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_x)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_img)) : "memory");
      if (NAD > 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_rp)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_t)) : "memory");
      }
      pdl_wait();   // images and T were written by the previous kernels on the stream
      // All sources are read as rows of kRowBytes: images (group h reads tile
      // pb*4 + 2h + rank), R^T of those tiles, and this CTA's half of the
      // pair's T tile for the fused linear that owns rows pb*512...
      const int img_row0 = (pb * 4 + (int)rank) * S * kImgRows;
      int grp = 0;
      while (grp + 1 < p.n_groups && pb * 512 >= p.group_end[grp]) ++grp;
      const int t_row0 = (int)(((size_t)ptile * p.n_groups * r64 * (TT * 2) + (size_t)grp * (r64 / 64) * (TT * 128) +
                                (size_t)rank * TH * 128) / kRowBytes);
      const uint32_t a_full0 = cluster_addr(a_full, 0), x_full0 = cluster_addr(x_full, 0);
      int xs_i = 0;   // X slots filled so far
      int a_iss = 0;  // A slots filled so far
      for (int u = 0; u < NAD + S; ++u) {
        const int a = u % NA;
        if (!pwait(a_empty + a, ((u / NA) & 1) ^ 1, abort_flag)) break;
        ++a_iss;
        const int nx = u < NAD ? 1 : 2;
        if (u < NAD) {
          if (rank == 0) mbar_expect_tx(a_full + a, 2 * 2 * kImgA);
#pragma unroll
          for (int h = 0; h < 2; ++h)
            tma_load_2d_pair(as + a * kAStage + h * kImgA, &tmap_rp, 0,
                             (pb * 4 + 2 * h + (int)rank) * (r64 / 4) + u * (kImgA / kRowBytes), a_full0 + 8u * (uint32_t)a);
        } else {
          const int s = u - NAD;
          if (rank == 0) mbar_expect_tx(a_full + a, 2 * 2 * kImg);
#pragma unroll
          for (int h = 0; h < 2; ++h)
            tma_load_2d_pair(as + a * kAStage + h * kImg, &tmap_img, 0, img_row0 + (2 * h * S + s) * kImgRows,
                             a_full0 + 8u * (uint32_t)a);
        }
        bool ok = true;
        for (int x = 0; x < nx; ++x, ++xs_i) {
          const int xi = xs_i % NX;
          if (!pwait(x_empty + xi, ((xs_i / NX) & 1) ^ 1, abort_flag)) { ok = false; break; }
          if (rank == 0) mbar_expect_tx(x_full + xi, 2 * kXStage);
          if (u < NAD)
            tma_load_2d_pair(xs + xi * kXStage, &tmap_t, 0, t_row0 + u * (TT * 128 / kRowBytes),
                             x_full0 + 8u * (uint32_t)xi);
          else
            tma_load_2d_pair(xs + xi * kXStage, &tmap_x, (2 * (u - NAD) + x) * 64, t0 + (int)rank * TH,
                             x_full0 + 8u * (uint32_t)xi);
        }
        if (!ok) break;
      }
      if (*abort_flag) {
        // Let the copies still in flight land before the pair exits.  Rank
        // 0's barriers count the bytes of both CTAs' copies of the stages it
        // armed; rank 1 cannot wait on them and gives its own copies a fixed
        // grace period instead.
        const long long t_start = clock64();
        const long long deadline = t_start + kWaitBudgetCycles;
        if (rank == 0) {
          for (int j = max(0, a_iss - NA); j < a_iss; ++j) drain_phase(a_full + j % NA, (j / NA) & 1, deadline);
          for (int j = max(0, xs_i - NX); j < xs_i; ++j) drain_phase(x_full + j % NX, (j / NX) & 1, deadline);
        } else {
          while (clock64() - t_start < 200000) {
          }
        }
      }
    }
  } else if (warp == 9) {
    if (lane == 0 && rank == 0) {
      // ---------------------------------------------------------------- MMA issue (both CTAs)
      const uint32_t idesc_sp = (1u << 2) | (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(TT >> 3) << 17) |
                                ((uint32_t)(256 >> 4) << 24);
      const uint32_t idesc_dn = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(TT >> 3) << 17) |
                                ((uint32_t)(256 >> 4) << 24);
      const uint32_t xs_a = smem_u32(xs), as_a = smem_u32(as);
      int xs_i = 0;
      bool complete = false;
      for (int u = 0; u < NAD + S; ++u) {
        const int a = u % NA;
        if (!pwait(a_full + a, (u / NA) & 1, abort_flag)) break;
        tc_fence_after();
        bool ok = true;
        if (u < NAD) {
          // T R for adapter columns 64u ... (whole 16-column steps only).
          const int xi = xs_i % NX;
          if (!pwait(x_full + xi, (xs_i / NX) & 1, abort_flag)) break;
          tc_fence_after();
          const int kks = min(4, (p.r16 - 64 * u) / 16);
          for (int kk = 0; kk < kks; ++kk) {
            const uint64_t bd = sw128_desc(xs_a + xi * kXStage + kk * 32);
#pragma unroll
            for (int h = 0; h < 2; ++h)
              mma_dense2(tmem + kAccCol + h * TT, sw128_desc(as_a + a * kAStage + h * kImgA + kk * 32), bd, idesc_dn,
                         (u | kk) != 0);
          }
          tc_commit2(x_empty + xi);
          ++xs_i;
        } else {
          const int s = u - NAD;
#pragma unroll
          for (int h = 0; h < 2; ++h)
            tc_cp_meta2(tmem + (uint32_t)(kMetaCol + (h * NA + a) * 4), meta_desc(as_a + a * kAStage + h * kImg + kImgA));
          for (int x = 0; x < 2; ++x, ++xs_i) {
            const int xi = xs_i % NX;
            if (!pwait(x_full + xi, (xs_i / NX) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
              const int jl = 2 * x + k2;
              const uint64_t bd = sw128_desc(xs_a + xi * kXStage + k2 * 64);
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const uint64_t ad = sw128_desc(as_a + a * kAStage + h * kImg + jl * 32);
                const uint32_t mcol = kMetaCol + (h * NA + a) * 4 + jl;
                mma_sp2(tmem + kAccCol + h * TT, ad, bd, tmem + (mcol & ~1u), idesc_sp | (mcol & 1u),
                        NAD > 0 || (s | jl) != 0);
              }
            }
            tc_commit2(x_empty + xi);
          }
        }
        if (!ok) break;
        tc_commit2(a_empty + a);
        complete = u + 1 == NAD + S;
      }
      // Always arrives on this CTA's barrier (its epilogue waits for the MMAs
      // in flight before tensor memory is freed); on the peer's only when the
      // accumulators are complete, so that after a give-up the peer's own
      // bounded wait fails and it stores zeros.
      tc_commit2_mask(acc_full, complete ? 3 : 1);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int h = warp >> 2;                  // MMA row group
    const int wq = warp & 3;                  // tensor-memory lane quarter
    const int L = wq * 32 + lane;
    // Rank 0 (which issues the MMAs) always gets acc_full, so its wait also
    // guarantees that no MMA is in flight when the pair frees tensor memory
    // (rank 1 frees only after the closing cluster barrier).  Rank 1 gets it
    // only for complete accumulators.
    const bool acc_ok = rank == 0 ? mbar_wait(acc_full, 0) : pwait(acc_full, 0, abort_flag);
    tc_fence_after();
    pdl_launch_dependents();
    pdl_wait();   // Y may still be in use by earlier work on the stream
    // Accumulators -> bf16 tile [token][local row] in the (free) rings; local
    // row h * 128 + L is global row pb * 512 + h * 256 + rank * 128 + L.
    uint16_t* stage = reinterpret_cast<uint16_t*>(xs);
    const bool stage_ok = __all_sync(0xffffffffu, acc_ok && !*abort_flag);
    if (stage_ok) {
      const int rloc = h * TILE_ROWS + L;
      for (int c0 = 0; c0 < TT; c0 += 32) {
        uint32_t v[32];
        const uint32_t taddr = tmem + ((uint32_t)(wq * 32) << 16) + (uint32_t)(kAccCol + h * TT + c0);
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
            "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
              "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
              "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),
              "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]),
              "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
            : "r"(taddr)
            : "memory");
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if (TT % 32 == 0 || c0 + c < TT)
            stage[(c0 + c) * 256 + rloc] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[c])));
      }
    }
    // One decision for this CTA's tile: stored as zeros if any wait gave up.
    const bool bad = epi_bar_or(!stage_ok);
    if (bad && threadIdx.x == 0) record_status(p.status, SLIM_ERR_TIMEOUT);
    {
      const int ntok = min(TT, p.M - t0);
      const int tid = threadIdx.x;   // 0..255
      for (int i = tid; i < ntok * 32; i += 256) {
        const int tk = i >> 5, c8 = i & 31;                  // 8 local rows c8*8 .. +7
        const int lr = c8 * 8;
        const int n = pb * 512 + (lr >> 7) * 256 + (int)rank * 128 + (lr & 127);
        const uint16_t* src = stage + tk * 256 + lr;
        uint16_t* dst = p.Y + (size_t)(t0 + tk) * p.N + n;
        if (!dcheck(t0 + tk < p.M && n < ceil_div(p.N, 512) * 512, p.status)) continue;
        if ((p.N & 7) == 0 && n + 8 <= p.N) {
          *reinterpret_cast<uint4*>(dst) = bad ? make_uint4(0u, 0u, 0u, 0u) : *reinterpret_cast<const uint4*>(src);
        } else {
          for (int q = 0; q < 8; ++q)
            if (n + q < p.N) dst[q] = bad ? (uint16_t)0 : src[q];
        }
      }
    }
  }
  if (*abort_flag && threadIdx.x == 0) record_status(p.status, SLIM_ERR_TIMEOUT);
  tc_fence_before();
  __syncwarp();
  __syncthreads();
  // Neither CTA leaves while the other may still touch its shared or tensor
  // memory (the rank-0 MMAs are complete: both epilogues waited for them).
  cluster_sync_all();
  if (warp == 9) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// ---------------------------------------------------------------- T = X L
constexpr int TG_TOK = 128;                  // tokens per CTA (MMA M)
constexpr int TG_NST_MIN = 4;                // stages of 64 K: at least, and as many as fit
constexpr int TG_NST_MAX = 6;                //   in TG_SMEM_BUDGET (more bytes in flight per CTA)
constexpr int TG_SMEM_BUDGET = 200 * 1024;
constexpr int TG_XST = TG_TOK * 128;         // 16 KB X tile per stage
constexpr int TG_THREADS = 192;              // warp 0 producer, warp 1 MMA, warps 2-5 epilogue

constexpr int TG_COLS = 256;                 // most T columns per CTA (MMA N limit)
struct TgParams {
  const uint8_t* Lp;      // L^T images, [K/64][rl16 rows x 128 B]
  uint16_t* Tswz;         // output: tiles of `tt` tokens x (n_groups x r64) columns, swizzled
  int M, K, tt;
  int cwmax;              // T columns per CTA: 256, or 128 when the grid would leave most SMs idle
  int rl16;               // T columns (all fused linears); this CTA: [blockIdx.z * cwmax, + cw)
  int r16, r64, n_groups; // per fused linear: columns, padded to whole 64-column atoms
  int32_t* status;
};

__host__ __device__ inline int tg_lstage(int cw) { return cw * 128; }
// The fp32 partial sums [TG_TOK][cw + 4] reuse the rings: the L rings hold
// TG_TOK x cw floats exactly, the X rings the padding.
static_assert(TG_NST_MIN * 128 >= TG_TOK * 4 && TG_NST_MIN * TG_XST >= TG_TOK * 4 * 4, "partial sums fit the rings");
__host__ __device__ inline int tg_stages(int cw) {
  int n = TG_SMEM_BUDGET / (TG_XST + tg_lstage(cw));
  return n < TG_NST_MIN ? TG_NST_MIN : n > TG_NST_MAX ? TG_NST_MAX : n;
}
__host__ __device__ inline int tg_smem(int cw) {
  const int nst = tg_stages(cw);
  return nst * (TG_XST + tg_lstage(cw)) + (2 * nst + 1) * 8 + 16 + 1024;
}
__host__ __device__ inline int tg_tmem_cols(int r16) {
  int c = 32;
  while (c < r16) c <<= 1;
  return c;
}

__global__ void __launch_bounds__(TG_THREADS, 1) k_tgemm(const __grid_constant__ CUtensorMap tmap_x,
                                                         const TgParams p) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int c0 = blockIdx.z * p.cwmax;                // this CTA's T columns [c0, c0 + cw)
  const int cw = min(p.cwmax, p.rl16 - c0);
  const int lst = tg_lstage(cw);
  uint8_t* xs = smem;
  const int NST = tg_stages(cw);
  uint8_t* ls = smem + NST * TG_XST;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + NST * (TG_XST + lst));
  uint64_t* full = bars;
  uint64_t* empty = bars + NST;
  uint64_t* acc_full = bars + 2 * NST;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(bars + 2 * NST + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * NST + 1) + 1;
  float* red = reinterpret_cast<float*>(smem);           // [128][cw + 4] fp32, reuses the rings after the K loop

  const int S = gridDim.x, rank = blockIdx.x, tile = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KS = p.K / 64;
  const int k0 = (int)((long long)rank * KS / S), k1 = (int)((long long)(rank + 1) * KS / S);
  const int ncols = tg_tmem_cols(cw);

  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, 1);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32((const void*)tmem_slot)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      pdl_wait();   // X may have been written by the previous kernel
      // The previous call has completed: the weight-image pass of this call
      // may start now (it does not read T).
      pdl_launch_dependents();
      int iss = 0;    // stages filled so far
      for (int i = k0; i < k1; ++i) {
        const int it = i - k0, st = it % NST;
        if (!pwait(empty + st, ((it / NST) & 1) ^ 1, abort_flag)) break;
        if (!dcheck(i < p.K / 64, p.status)) break;
        mbar_expect_tx(full + st, (uint32_t)(TG_XST + lst));
        tma_load_2d(xs + st * TG_XST, &tmap_x, i * 64, tile * TG_TOK, full + st);
        bulk_g2s(ls + st * lst, p.Lp + ((size_t)i * p.rl16 + c0) * 128, (uint32_t)lst, full + st);
        ++iss;
      }
      if (*abort_flag) {
        // Let the copies still in flight land before the CTA exits.
        const long long deadline = clock64() + kWaitBudgetCycles;
        for (int j = max(0, iss - NST); j < iss; ++j) drain_phase(full + j % NST, (j / NST) & 1, deadline);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(cw >> 3) << 17) |
                             ((uint32_t)(TG_TOK >> 4) << 24);
      const uint32_t xa = smem_u32(xs), la = smem_u32(ls);
      for (int i = k0; i < k1; ++i) {
        const int it = i - k0, st = it % NST;
        if (!pwait(full + st, (it / NST) & 1, abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_dense(tmem, sw128_desc(xa + st * TG_XST + kk * 32), sw128_desc(la + st * lst + kk * 32), idesc,
                    (it | kk) != 0);
        tc_commit(empty + st);
      }
      tc_commit(acc_full);
    }
  } else {
    // Accumulator rows (tokens) of this warp's lane quarter -> red[tok][j].
    // (The MMA thread commits acc_full whether or not its loop completed, so
    // no MMA is in flight once this wait returns.)
    const int wq = warp & 3;
    const bool ok = mbar_wait(acc_full, 0);
    if (!ok && lane == 0) *abort_flag = 1;
    tc_fence_after();
    if (ok) {
      for (int cc = 0; cc < cw; cc += 16) {
        uint32_t v[16];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
              "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
              "=r"(v[15])
            : "r"(tmem + ((uint32_t)(wq * 32) << 16) + (uint32_t)cc)
            : "memory");
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        // Rows padded by 4 floats: a quarter-warp's 16-byte stores hit 8 distinct bank groups.
        float4* rr = reinterpret_cast<float4*>(red + (size_t)(wq * 32 + lane) * (cw + 4) + cc);
#pragma unroll
        for (int c = 0; c < 4; ++c)
          rr[c] = make_float4(__uint_as_float(v[4 * c]), __uint_as_float(v[4 * c + 1]), __uint_as_float(v[4 * c + 2]),
                              __uint_as_float(v[4 * c + 3]));
      }
    }
  }
  if (*abort_flag && threadIdx.x == 0) record_status(p.status, SLIM_ERR_TIMEOUT);
  tc_fence_before();
  cluster.sync();
  // Rank c adds rows [c*128/S, (c+1)*128/S) over the ranks, in rank order,
  // 8 consecutive columns per thread (16-byte bf16 stores; all ranks' loads
  // are issued before they are added).  If a wait of any rank gave up, T is
  // written as bf16 NaN, so the outputs that use it can never look valid.
  bool bad = false;
  for (int q = 0; q < S; ++q) bad = bad || *cluster.map_shared_rank(const_cast<int*>(abort_flag), q) != 0;
  {
    const int r0 = rank * TG_TOK / S, r1 = (rank + 1) * TG_TOK / S;
    const int per_row = cw / 8;
    const int E = (r1 - r0) * per_row;
    const size_t tile_bytes = (size_t)p.n_groups * p.r64 * 2 * p.tt;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      const int row = r0 + e / per_row, j = (e % per_row) * 8;
      const size_t off = (size_t)row * (cw + 4) + j;
      float4 a[8], b[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (q < S) {
          const float4* src = reinterpret_cast<const float4*>(cluster.map_shared_rank(red, q) + off);
          a[q] = src[0];
          b[q] = src[1];
        }
      }
      float sum[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (q < S) {
          sum[0] += a[q].x; sum[1] += a[q].y; sum[2] += a[q].z; sum[3] += a[q].w;
          sum[4] += b[q].x; sum[5] += b[q].y; sum[6] += b[q].z; sum[7] += b[q].w;
        }
      }
      const int tok = tile * TG_TOK + row;
      if (tok < p.M) {
        // 8 columns form one 16-byte swizzle chunk of the T tile row; T
        // column c of fused linear c / r16 sits at (c / r16) * r64 + c % r16.
        const int cg = c0 + j, col = (cg / p.r16) * p.r64 + cg % p.r16;
        __nv_bfloat162 o[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) o[c] = __floats2bfloat162_rn(sum[2 * c], sum[2 * c + 1]);
        if (bad) {
#pragma unroll
          for (int c = 0; c < 4; ++c) o[c] = __halves2bfloat162(__ushort_as_bfloat16(0x7FC0), __ushort_as_bfloat16(0x7FC0));
        }
        *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(p.Tswz) + (size_t)(tok / p.tt) * tile_bytes +
                                  sw128_offset(tok % p.tt, col, p.tt)) = *reinterpret_cast<uint4*>(o);
      }
    }
  }
  cluster.sync();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols) : "memory");
  }
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

}  // namespace

// Clusters of S CTAs of k_tgemm (dynamic shared memory smem) that fit on the
// current device at once; cached per (device, S, smem).
int tg_max_clusters(cudaLaunchConfig_t cfg, int S, int smem) {
  static std::mutex mu;
  static std::map<std::pair<int, std::pair<int, int>>, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find({dev, {S, smem}});
  if (it != cache.end()) return it->second;
  cfg.stream = nullptr;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, k_tgemm, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    n = 0;
  }
  cache[{dev, {S, smem}}] = n;
  return n;
}

cudaError_t launch_tgemm(const slim_layer& L, const uint16_t* X, int M, uint16_t* Tswz, cudaStream_t s) {
  NvtxRange nv("prefill: T = X L (k_tgemm)");
  auto encode = tensor_map_encoder();
  if (!encode) return cudaErrorNotSupported;
  CUtensorMap tmap;
  const cuuint64_t dims[2] = {(cuuint64_t)L.K, (cuuint64_t)M};
  const cuuint64_t strides[1] = {(cuuint64_t)L.K * 2};
  const cuuint32_t box[2] = {64, TG_TOK};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(X), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  TgParams p;
  p.Lp = reinterpret_cast<const uint8_t*>(L.Lp);
  p.Tswz = Tswz;
  p.M = M;
  p.K = L.K;
  p.rl16 = L.rl16;
  p.r16 = L.r16;
  p.r64 = ceil_div(L.r16, 64) * 64;
  p.n_groups = L.n_groups;
  p.tt = prefill_tokens_per_tile(L, M);
  p.status = L.status;
  const int KS = L.K / 64;
  // 128 columns per CTA instead of 256 when the 256-column grid, even with
  // the largest K split, would hold fewer CTAs than half the SMs (few
  // tokens, as at M = 512): twice the CTAs, each with half the MMA width.
  const int nsm = num_sms();
  p.cwmax = (L.rl16 > 128 && ceil_div(M, TG_TOK) * ceil_div(L.rl16, TG_COLS) * 8 < nsm / 2) ? 128 : TG_COLS;
  // Largest split of K (cluster size, any of 1..8) that keeps >= 4 K steps
  // per CTA and lets every cluster of the grid be resident at once: a cluster
  // left for a second wave doubles the kernel's time.
  const int smem = tg_smem(std::min(p.cwmax, L.rl16));
  {
    cudaError_t e = ensure_func_attrs(reinterpret_cast<const void*>(k_tgemm), (size_t)smem);
    if (e != cudaSuccess) return e;
  }
  const int clusters = ceil_div(M, TG_TOK) * ceil_div(L.rl16, p.cwmax);
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(TG_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  int S = 8;
  for (; S > 1; --S) {
    if (KS / S < 4) continue;
    cfg.gridDim = dim3(S, ceil_div(M, TG_TOK), ceil_div(L.rl16, p.cwmax));
    attr[1].val.clusterDim.x = S;
    cfg.numAttrs = 2;
    if (clusters <= tg_max_clusters(cfg, S, smem)) break;
  }
  cfg.gridDim = dim3(S, ceil_div(M, TG_TOK), ceil_div(L.rl16, p.cwmax));
  attr[1].val.clusterDim.x = S;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, k_tgemm, tmap, p);
}

// CTA tile whose waves of CTAs (one per SM) finish first.  A CTA's time is
// modelled as 128-row halves x (tokens + 264) units: measured on B200, a
// 128-token CTA takes 0.86 of a 192-token one (pipeline fill and epilogue do
// not shrink with the tile).  Among the one-SM tiles a tie keeps the earlier
// (larger) one.
//
// The 2-SM kernel (pairs of 512 rows; each CTA holds two halves) serves
// layers whose fused linears start on 512-row boundaries, for M >= 256, when
// it costs strictly less than the best one-SM tile.
struct PrefillTile {
  int TT, NH;
  bool two_sm;
};
PrefillTile prefill_tile(const slim_layer& L, int M) {
  const Tuning tn = tuning();
  bool pair_ok = M >= 256 && !tn.prefill_1sm;
  for (int g = 0; g + 1 < L.n_groups; ++g) pair_ok = pair_ok && L.group_end[g] % 512 == 0;
  if (tn.prefill_tile) {   // forced tile, for tuning and tests
    if (tn.prefill_pair && pair_ok) return {tn.prefill_tt, 2, true};
    if (!tn.prefill_pair) return {tn.prefill_tt, tn.prefill_nh, false};
  }
  // Cost of a tile: waves of CTAs x per-CTA time, the latter ~ rows x (TT +
  // 264) (the constant is the per-CTA fixed cost, in token-equivalents,
  // fitted on the measured kernels).  A pair CTA holds 256 rows like a
  // two-half CTA; on a tie the one-SM kernel wins (it measured faster).
  const long long nsm = num_sms();
  const PrefillTile cand[4] = {{192, 2, false}, {128, 2, false}, {128, 1, false}, {64, 1, false}};
  PrefillTile best = cand[0];
  long long best_cost = -1;
  for (const PrefillTile& c : cand) {
    const long long ctas = (long long)ceil_div(L.N, c.NH * TILE_ROWS) * ceil_div(M, c.TT);
    const long long cost = (ctas + nsm - 1) / nsm * c.NH * (c.TT + 264);
    if (best_cost < 0 || cost < best_cost) {
      best = c;
      best_cost = cost;
    }
  }
  if (pair_ok)
    for (int tt : {240, 224, 192, 128}) {
      const long long ctas = 2LL * ceil_div(L.N, 512) * ceil_div(M, tt);
      const long long cost = (ctas + nsm - 1) / nsm * 2 * (tt + 264);
      if (cost < best_cost) {
        best = {tt, 2, true};
        best_cost = cost;
      }
    }
  return best;
}

int prefill_tokens_per_tile(const slim_layer& L, int M) { return prefill_tile(L, M).TT; }

// Images of 128-row tiles, padded to whole 512-row blocks (the 2-SM tile).
size_t prefill_image_bytes(int N, int K) { return (size_t)ceil_div(N, 512) * 4 * (K / 128) * kImg; }

namespace {

template <int TT, int NH>
cudaError_t launch_prefill_tt(const slim_layer& L, const uint16_t* X, int M, uint16_t* Y, const uint16_t* Tswz,
                              uint8_t* img, cudaStream_t s) {
  auto encode = tensor_map_encoder();
  if (!encode) return cudaErrorNotSupported;
  using C = PfCfg<TT, NH>;
  CUtensorMap tmap;
  const cuuint64_t dims[2] = {(cuuint64_t)L.K, (cuuint64_t)M};
  const cuuint64_t strides[1] = {(cuuint64_t)L.K * 2};
  const cuuint32_t box[2] = {64, TT};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(X), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  PrefillParams p;
  p.img = img;
  p.Rp = reinterpret_cast<const uint8_t*>(L.Rp);
  p.Tswz = reinterpret_cast<const uint8_t*>(Tswz);
  p.Y = Y;
  p.M = M;
  p.N = L.N;
  p.K = L.K;
  p.r16 = L.r16;
  p.n_groups = L.n_groups;
  for (int g = 0; g < SLIM_MAX_GROUPS; ++g) p.group_end[g] = L.group_end[g];
  p.status = L.status;
  {
    cudaError_t e = ensure_func_attrs(reinterpret_cast<const void*>(k_prefill<TT, NH>), C::kSmemBytes);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ceil_div(M, TT), ceil_div(L.N, C::kCtaRows));   // token tiles fastest
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_prefill<TT, NH>, tmap, p);
}

// A byte buffer as a 2-D tensor of kRowBytes rows (u64 elements), boxes of
// box_rows whole rows, no swizzle: a box lands in shared memory as the same bytes.
CUresult encode_rows(PFN_cuTensorMapEncodeTiled_v12000 encode, CUtensorMap* map, void* base, size_t bytes, int box_rows) {
  const cuuint64_t dims[2] = {kRowBytes / 8, (cuuint64_t)(bytes / kRowBytes)};
  const cuuint64_t strides[1] = {kRowBytes};
  const cuuint32_t box[2] = {kRowBytes / 8, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT64, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

template <int TT>
cudaError_t launch_prefill2_tt(const slim_layer& L, const uint16_t* X, int M, uint16_t* Y, const uint16_t* Tswz,
                               uint8_t* img, cudaStream_t s) {
  auto encode = tensor_map_encoder();
  if (!encode) return cudaErrorNotSupported;
  using C = Pf2Cfg<TT>;
  CUtensorMap tmap, tmap_img, tmap_rp, tmap_t;
  const cuuint64_t dims[2] = {(cuuint64_t)L.K, (cuuint64_t)M};
  const cuuint64_t strides[1] = {(cuuint64_t)L.K * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)C::TH};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(X), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  // The images, R^T and T, byte for byte, as rows of kRowBytes: one box is
  // one image, one R^T atom of a 128-row tile, or half of a T atom.
  if (encode_rows(encode, &tmap_img, img, prefill_image_bytes(L.N, L.K), kImgRows) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  std::memset(&tmap_rp, 0, sizeof(tmap_rp));
  std::memset(&tmap_t, 0, sizeof(tmap_t));
  if (L.r16 > 0) {
    const int r64 = ceil_div(L.r16, 64) * 64;
    const size_t rp_bytes = (size_t)ceil_div(L.N, 512) * 512 * r64 * 2;
    const size_t t_bytes = (size_t)ceil_div(M, TT) * L.n_groups * r64 * 2 * TT;
    if (encode_rows(encode, &tmap_rp, const_cast<uint16_t*>(L.Rp), rp_bytes, kImgA / kRowBytes) != CUDA_SUCCESS ||
        encode_rows(encode, &tmap_t, const_cast<uint16_t*>(Tswz), t_bytes, C::TH * 128 / kRowBytes) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  PrefillParams p;
  p.img = img;
  p.Rp = reinterpret_cast<const uint8_t*>(L.Rp);
  p.Tswz = reinterpret_cast<const uint8_t*>(Tswz);
  p.Y = Y;
  p.M = M;
  p.N = L.N;
  p.K = L.K;
  p.r16 = L.r16;
  p.n_groups = L.n_groups;
  for (int g = 0; g < SLIM_MAX_GROUPS; ++g) p.group_end[g] = L.group_end[g];
  p.status = L.status;
  {
    cudaError_t e = ensure_func_attrs(reinterpret_cast<const void*>(k_prefill2<TT>), C::kSmemBytes);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * ceil_div(M, TT), ceil_div(L.N, 512));   // CTA pairs along x, token tiles fastest
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, k_prefill2<TT>, tmap, tmap_img, tmap_rp, tmap_t, p);
}

}  // namespace

cudaError_t launch_prefill(const slim_layer& L, const uint16_t* X, int M, uint16_t* Y, const uint16_t* Tswz,
                           uint8_t* img, cudaStream_t s) {
  const int S = L.K / 128;
  {
    NvtxRange nv("prefill: weight images (k_predequant)");
    // Dequantized images (4 * ceil(N/512) tiles of 128 rows, padded with zeros).
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(S, ceil_div(L.N, 512) * 4);
    cfg.blockDim = dim3(128);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, k_predequant, L.dec, L.n_kblocks, L.n_row_tiles, S, img,
                                       L.r16 > 0 ? 0 : 1);
    if (e != cudaSuccess) return e;
  }
  NvtxRange nv("prefill: sparse MMA, adapter T R and epilogue (k_prefill / k_prefill2)");
  const PrefillTile t = prefill_tile(L, M);
  if (t.two_sm) {
    if (t.TT == 128) return launch_prefill2_tt<128>(L, X, M, Y, Tswz, img, s);
    if (t.TT == 192) return launch_prefill2_tt<192>(L, X, M, Y, Tswz, img, s);
    if (t.TT == 224) return launch_prefill2_tt<224>(L, X, M, Y, Tswz, img, s);
    return launch_prefill2_tt<240>(L, X, M, Y, Tswz, img, s);
  }
  if (t.NH == 1) {
    if (t.TT == 64) return launch_prefill_tt<64, 1>(L, X, M, Y, Tswz, img, s);
    return launch_prefill_tt<128, 1>(L, X, M, Y, Tswz, img, s);
  }
  if (t.TT == 128) return launch_prefill_tt<128, 2>(L, X, M, Y, Tswz, img, s);
  return launch_prefill_tt<192, 2>(L, X, M, Y, Tswz, img, s);
}

}  // namespace slim

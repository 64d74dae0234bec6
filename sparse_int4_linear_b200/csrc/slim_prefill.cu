// Tensor-core prefill forward for M > 16 tokens (sm_100a, tcgen05).
//
// Many tokens reuse every weight, so this path is compute-bound (thesis
// §2.5.1 "The Compute-Bound Regimes: Training and Prefill") and the 2:4
// structure is exploited by the sparse tensor cores, which skip the pruned
// products (§2.2.3 "Sparse Tensor Core Acceleration").
//
// One CTA computes a 128-row (layer outputs) x 128-token tile of
//   Y^T = W_eff X^T + R^T T^T          (T = X L, computed beforehand)
// with tcgen05.mma.sp.kind::f16: A = the compressed weight tile (bf16 values
// q * s, 64 per row per 128 logical K, 128-byte-swizzled shared memory),
// its 2-bit position metadata in tensor memory, B = the X tile
// (128-byte-swizzled, loaded by TMA), fp32 accumulator in tensor memory.
// The adapter is added as r/16 extra dense MMAs into the same accumulator.
//
// Warp roles (320 threads):
//   warps 0-3, 4-7   dequant groups 0 and 1 (stages of even / odd 128-K
//                    groups): packed chunk -> bf16(q * s) into the A tile,
//                    metadata -> tensor memory; later the epilogue
//   warp 8           producer: bulk copies of the packed decode-stream
//                    chunks, TMA tensor loads of X, then the adapter tiles
//   warp 9           tensor-memory allocation and the single-thread MMA issue
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "slim_common.cuh"
#include "slim_internal.h"

namespace slim {
namespace {

constexpr int BNR = 128;                     // layer rows per CTA (MMA M)
constexpr int BTK = 128;                     // tokens per CTA (MMA N)
constexpr int NSTAGE = 4;                    // 128-K pipeline stages
constexpr int NDEC = 2;                      // packed-stream ring units (256 K each)
constexpr int kXStage = BTK * 128 * 2;       // 32 KB: 2 swizzled atoms of 128 tokens x 64 K
constexpr int kAStage = BNR * 64 * 2;        // 16 KB: 1 swizzled atom of 128 rows x 64 values
constexpr int kDecUnit = 8 * kDecChunk;      // 12.8 KB: 8 row tiles x 256 K
constexpr int kTmemCols = 256;
constexpr int kAccCol = 0;
constexpr int kMetaCol = 128;                // NSTAGE x 4 columns of metadata
constexpr int kThreads = 320;

constexpr int kOffX = 0;
constexpr int kOffA = kOffX + NSTAGE * kXStage;          // 128 KB
constexpr int kOffDec = kOffA + NSTAGE * kAStage;        // 192 KB
constexpr int kOffBar = kOffDec + NDEC * kDecUnit;       // + 25.6 KB
// barriers: x_full[4] a_full[4] st_empty[4] dec_full[2] dec_empty[2] main_done ad_full acc_full
constexpr int kNumBars = 3 * NSTAGE + 2 * NDEC + 3;
constexpr int kSmemBytes = kOffBar + kNumBars * 8 + 16 + 1024;   // + words, + alignment slack

struct PrefillParams {
  const uint8_t* dec;
  const uint8_t* Rp;      // pre-swizzled R^T tiles
  const uint8_t* Tswz;    // pre-swizzled T tiles (workspace)
  uint16_t* Y;
  int M, N, K, NKB, NRT, r16;
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
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
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

__global__ void __launch_bounds__(kThreads, 1) k_prefill(const __grid_constant__ CUtensorMap tmap_x,
                                                         const PrefillParams p) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the swizzled operand tiles
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* xs = smem + kOffX;
  uint8_t* as = smem + kOffA;
  uint8_t* ds = smem + kOffDec;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* x_full = bars;
  uint64_t* a_full = bars + NSTAGE;
  uint64_t* st_empty = bars + 2 * NSTAGE;
  uint64_t* dec_full = bars + 3 * NSTAGE;
  uint64_t* dec_empty = dec_full + NDEC;
  uint64_t* main_done = dec_empty + NDEC;
  uint64_t* ad_full = main_done + 1;
  uint64_t* acc_full = ad_full + 1;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(bars + kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + kNumBars) + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rt0 = blockIdx.x * 8;                 // first 16-row tile of this CTA
  const int n0 = blockIdx.x * BNR, t0 = blockIdx.y * BTK;
  const int S = p.K / 128;                        // 128-K stages
  const int r64 = ceil_div(p.r16, 64) * 64;
  const uint32_t ad_bytes = (uint32_t)r64 * 256u;  // one 128-row (or 128-token) adapter tile

  if (threadIdx.x == 0) {
    for (int i = 0; i < NSTAGE; ++i) {
      mbar_init(x_full + i, 1);
      mbar_init(a_full + i, 128);
      mbar_init(st_empty + i, 1);
    }
    for (int i = 0; i < NDEC; ++i) {
      mbar_init(dec_full + i, 1);
      mbar_init(dec_empty + i, 256);
    }
    mbar_init(main_done, 1);
    mbar_init(ad_full, 1);
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
      bool waited = false;
      for (int s = 0; s < S; ++s) {
        if ((s & 1) == 0) {
          const int u = s >> 1, slot = u % NDEC;
          if (!pwait(dec_empty + slot, ((u / NDEC) & 1) ^ 1, abort_flag)) break;
          int nvalid = 0;
          for (int m2 = 0; m2 < 8; ++m2) nvalid += (rt0 + m2 < p.NRT);
          mbar_expect_tx(dec_full + slot, (uint32_t)nvalid * kDecChunk);
          for (int m2 = 0; m2 < 8; ++m2)
            if (rt0 + m2 < p.NRT)
              bulk_g2s(ds + slot * kDecUnit + m2 * kDecChunk, p.dec + ((size_t)(rt0 + m2) * p.NKB + u) * kDecChunk,
                       kDecChunk, dec_full + slot);
        }
        if (!waited) {  // X (and later T) may be written by the previous kernel
          pdl_wait();
          waited = true;
        }
        const int st = s % NSTAGE;
        if (!pwait(st_empty + st, ((s / NSTAGE) & 1) ^ 1, abort_flag)) break;
        mbar_expect_tx(x_full + st, kXStage);
        tma_load_2d(xs + st * kXStage, &tmap_x, s * 128, t0, x_full + st);
        tma_load_2d(xs + st * kXStage + kXStage / 2, &tmap_x, s * 128 + 64, t0, x_full + st);
      }
      if (p.r16 > 0 && pwait(main_done, 0, abort_flag)) {
        // The ring buffers are free: adapter operands R^T (A) and T (B).
        mbar_expect_tx(ad_full, 2 * ad_bytes);
        bulk_g2s(as, p.Rp + (size_t)blockIdx.x * ad_bytes, ad_bytes, ad_full);
        bulk_g2s(xs, p.Tswz + (size_t)blockIdx.y * ad_bytes, ad_bytes, ad_full);
      }
    }
  } else if (warp == 9) {
    // ---------------------------------------------------------------- MMA issue
    if (lane == 0) {
      const uint32_t idesc_sp = (1u << 2) | (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BTK >> 3) << 17) |
                                ((uint32_t)(BNR >> 4) << 24);
      const uint32_t idesc_dn = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BTK >> 3) << 17) |
                                ((uint32_t)(BNR >> 4) << 24);
      const uint32_t xs_a = smem_u32(xs), as_a = smem_u32(as);
      bool ok = true;
      for (int s = 0; s < S && ok; ++s) {
        const int st = s % NSTAGE;
        const uint32_t par = (s / NSTAGE) & 1;
        if (!pwait(x_full + st, par, abort_flag) || !pwait(a_full + st, par, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int jl = 0; jl < 4; ++jl) {
          const uint64_t ad = sw128_desc(as_a + st * kAStage + jl * 32);
          const uint64_t bd = sw128_desc(xs_a + st * kXStage + (jl >> 1) * (kXStage / 2) + (jl & 1) * 64);
          const uint32_t mcol = kMetaCol + st * 4 + jl;
          mma_sp(tmem + kAccCol, ad, bd, tmem + (mcol & ~1u), idesc_sp | (mcol & 1u), (s | jl) != 0);
        }
        tc_commit(st_empty + st);
      }
      if (ok && p.r16 > 0) {
        tc_commit(main_done);
        if (pwait(ad_full, 0, abort_flag)) {
          tc_fence_after();
          for (int kk = 0; kk < p.r16 / 16; ++kk) {
            const uint64_t ad = sw128_desc(as_a + (kk >> 2) * kAStage + (kk & 3) * 32);
            const uint64_t bd = sw128_desc(xs_a + (kk >> 2) * (kXStage / 2) + (kk & 3) * 32);
            mma_dense(tmem + kAccCol, ad, bd, idesc_dn, 1);
          }
        }
      }
      tc_commit(acc_full);
    }
  } else {
    // ---------------------------------------------------------------- dequant
    const int G = warp >> 2;                 // group: even / odd stages
    const int tg = threadIdx.x & 127;        // thread in group
    const int wq = warp & 3;                 // tensor-memory lane quarter
    const int L = wq * 32 + lane;            // this thread's metadata lane
    const int mm2 = L >> 4, mp = (L >> 3) & 1, mm0 = L & 7;
    for (int u = 0;; ++u) {
      const int s = 2 * u + G;
      if (s >= S) break;
      const int slot = u % NDEC, st = s % NSTAGE;
      if (!pwait(dec_full + slot, (u / NDEC) & 1, abort_flag)) break;
      if (!pwait(st_empty + st, ((s / NSTAGE) & 1) ^ 1, abort_flag)) break;
      const uint8_t* unit = ds + slot * kDecUnit;
      uint8_t* at = as + st * kAStage;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int li = tg + half * 128;       // (row tile, lane) slot of the unit
        const int m2 = li >> 5, l = li & 31, g = l >> 2, t = l & 3;
        const bool valid = rt0 + m2 < p.NRT;
        const uint8_t* ch = unit + m2 * kDecChunk;
        const uint4 vw = valid ? lds128(ch + G * 512 + l * 16) : make_uint4(0x88888888u, 0x88888888u, 0x88888888u,
                                                                           0x88888888u);
        const __half* sc = reinterpret_cast<const __half*>(ch + 1536);
        const float s_lo = valid ? __half2float(sc[G * 16 + g]) : 0.f;
        const float s_hi = valid ? __half2float(sc[G * 16 + g + 8]) : 0.f;
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
            const __nv_bfloat162 v = __floats2bfloat162_rn(f0, f1);
            *reinterpret_cast<__nv_bfloat162*>(at + sw128_offset(row, cc, 128)) = v;
          }
        }
      }
      // Metadata of this stage's 4 MMA steps -> tensor memory lane L.
      {
        const bool valid = rt0 + mm2 < p.NRT;
        const uint8_t* ch = unit + mm2 * kDecChunk;
        uint32_t e[4];
#pragma unroll
        for (int jl = 0; jl < 4; ++jl) {
          const int j = 4 * G + jl;
          const int owner = mm0 * 4 + (j & 1) * 2 + mp;
          e[jl] = valid ? *reinterpret_cast<const uint32_t*>(ch + 1024 + owner * 16 + (j >> 1) * 4) : 0x44444444u;
        }
        const uint32_t taddr = tmem + ((uint32_t)(wq * 32) << 16) + (uint32_t)(kMetaCol + st * 4);
        asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(e[0]),
                     "r"(e[1]), "r"(e[2]), "r"(e[3])
                     : "memory");
      }
      fence_proxy_async_smem();
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      tc_fence_before();
      mbar_arrive(a_full + st);
      mbar_arrive(dec_empty + slot);
    }
    // ---------------------------------------------------------------- epilogue
    const bool acc_ok = pwait(acc_full, 0, abort_flag);
    tc_fence_after();
    pdl_launch_dependents();
    pdl_wait();
    if (acc_ok && !*abort_flag) {
      const int row = n0 + wq * 32 + lane;
      for (int c0 = G * 64; c0 < G * 64 + 64; c0 += 32) {
        uint32_t v[32];
        const uint32_t taddr = tmem + ((uint32_t)(wq * 32) << 16) + (uint32_t)(kAccCol + c0);
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
        if (row < p.N) {
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int tok = t0 + c0 + c;
            if (tok < p.M)
              p.Y[(size_t)tok * p.N + row] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[c])));
          }
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

cudaError_t launch_prefill(const slim_layer& L, const uint16_t* X, int M, uint16_t* Y, const uint16_t* Tswz,
                           cudaStream_t s) {
  auto encode = tensor_map_encoder();
  if (!encode) return cudaErrorNotSupported;
  CUtensorMap tmap;
  const cuuint64_t dims[2] = {(cuuint64_t)L.K, (cuuint64_t)M};
  const cuuint64_t strides[1] = {(cuuint64_t)L.K * 2};
  const cuuint32_t box[2] = {64, BTK};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(X), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  PrefillParams p;
  p.dec = L.dec;
  p.Rp = reinterpret_cast<const uint8_t*>(L.Rp);
  p.Tswz = reinterpret_cast<const uint8_t*>(Tswz);
  p.Y = Y;
  p.M = M;
  p.N = L.N;
  p.K = L.K;
  p.NKB = L.n_kblocks;
  p.NRT = L.n_row_tiles;
  p.r16 = L.r16;
  p.status = L.status;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(k_prefill, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ceil_div(L.N, BNR), ceil_div(M, BTK));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_prefill, tmap, p);
}

}  // namespace slim

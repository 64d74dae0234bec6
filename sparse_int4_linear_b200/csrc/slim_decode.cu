// Token-parallel forward kernels built on warp-level tensor-core MMAs.
//
//   k_adapter_down : T = X L                    (dense m16n8k16)
//   k_decode       : Y = X W_eff^T + T R        (structured-sparse m16n8k32
//                    for the int4 2:4 weight, dense m16n8k16 for T R)
//
// Decoding a few tokens is memory-bound: the weight is loaded once and used
// for one small matrix product (thesis §2.5.2 "The Memory-Bound Regime:
// Inference Decoding"), so the packed 4-bit weight is streamed with bulk
// copies into shared memory while the sparse tensor cores select the
// matching activations from the 2-bit metadata (§2.2.3).  The adapter is a
// separate path added to the same fp32 accumulators, never merged into the
// sparse weight (§4, lazy low-rank adapters).
//
// Work split: CTA (rank, rg, tt) owns W_ROWS row tiles of 16 output rows
// (row group rg), a contiguous range of 256-wide K blocks (its rank in a
// cluster that spans K), and 16 tokens (tile tt).  The cluster's partial
// sums are added in rank order through distributed shared memory, so the
// result does not depend on timing.
#include <cooperative_groups.h>

#include "slim_common.cuh"
#include "slim_internal.h"

namespace cg = cooperative_groups;

namespace slim {
namespace {

constexpr int kDecodeStages = 4;   // bulk-copy ring depth per warp

struct DecodeParams {
  const uint16_t* X;
  uint16_t* Y;
  const uint8_t* dec;
  const uint4* Rf;
  const uint16_t* T;
  int M, K, N, NRT, NKB, r16;
  int seg_kb_max;      // largest K-block count of any rank
  int32_t* status;
};

// ---------------------------------------------------------------- T = X L
// Grid (S, r16/16, ceil(M/16)), cluster (S, 1, 1), 4 warps.  The K/16 steps
// are split over S x 4 warps; warp partials are added in the CTA, CTA
// partials in rank order across the cluster.
template <int NT>
__global__ void __launch_bounds__(128) k_adapter_down(const uint16_t* __restrict__ X, int M, int K,
                                                      const uint4* __restrict__ Lf, int r16,
                                                      uint16_t* __restrict__ T) {
  cg::cluster_group cluster = cg::this_cluster();
  __shared__ float red[4][256];
  __shared__ float part[256];
  const int S = gridDim.x, rank = blockIdx.x;
  const int jt = blockIdx.y, tt = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int KS = K / 16;
  const int nsplit = S * 4, sidx = rank * 4 + warp;
  const int ks0 = (int)((long long)sidx * KS / nsplit), ks1 = (int)((long long)(sidx + 1) * KS / nsplit);
  const int tok0 = tt * 16;
  const int Mt = min(16, M - tok0);

  float acc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
  const uint4* la = Lf + ((size_t)jt * KS) * 32 + lane;
  const uint16_t* xr[NT];
  bool tv[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int tok = nt * 8 + g;
    tv[nt] = tok < Mt;
    xr[nt] = X + (size_t)(tok0 + (tv[nt] ? tok : 0)) * K + 2 * t;
  }
#pragma unroll 4
  for (int ks = ks0; ks < ks1; ++ks) {
    const uint4 a = __ldg(la + (size_t)ks * 32);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      uint32_t b0 = 0, b1 = 0;
      if (tv[nt]) {
        b0 = __ldg(reinterpret_cast<const uint32_t*>(xr[nt] + ks * 16));
        b1 = __ldg(reinterpret_cast<const uint32_t*>(xr[nt] + ks * 16 + 8));
      }
      mma_16816(acc[nt], a, b0, b1);
    }
  }
  // element e = tok * 16 + row
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int tk = nt * 8 + 2 * t;
    red[warp][tk * 16 + g] = acc[nt][0];
    red[warp][(tk + 1) * 16 + g] = acc[nt][1];
    red[warp][tk * 16 + g + 8] = acc[nt][2];
    red[warp][(tk + 1) * 16 + g + 8] = acc[nt][3];
  }
  if (NT == 1) {
    for (int e = lane; e < 128; e += 32) red[warp][128 + e] = 0.f;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < 256; e += 128) part[e] = red[0][e] + red[1][e] + red[2][e] + red[3][e];
  cluster.sync();
  const int e0 = rank * 256 / S, e1 = (rank + 1) * 256 / S;
  for (int e = e0 + (int)threadIdx.x; e < e1; e += 128) {
    float s = 0.f;
    for (int q = 0; q < S; ++q) s += cluster.map_shared_rank(part, q)[e];
    const int tok = e >> 4, row = e & 15;
    T[(size_t)(tok0 + tok) * r16 + jt * 16 + row] = __bfloat16_as_ushort(__float2bfloat16_rn(s));
  }
  cluster.sync();
}

// ---------------------------------------------------------------- main product
template <int NT, int WR>
__global__ void __launch_bounds__(WR * 32) k_decode(const DecodeParams p) {
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ __align__(128) uint8_t smem[];
  const int S = gridDim.x, rank = blockIdx.x;
  const int rg = blockIdx.y, tt = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;

  const int kb0 = (int)((long long)rank * p.NKB / S), kb1 = (int)((long long)(rank + 1) * p.NKB / S);
  const int nkb = kb1 - kb0;
  const int kstart = kb0 * 256, kend = min(kb1 * 256, p.K);
  const int xrow = p.seg_kb_max * 256 + 8;      // padded row (elements) of the staged X
  const int tok0 = tt * 16;
  const int Mt = min(16, p.M - tok0);
  const int xrows = min(Mt, NT * 8);
  const int rt = rg * WR + warp;
  const bool active = rt < p.NRT;

  uint16_t* Xs = reinterpret_cast<uint16_t*>(smem);
  uint8_t* ring = smem + (size_t)NT * 8 * xrow * 2;
  float* red = reinterpret_cast<float*>(ring + (size_t)WR * kDecodeStages * kDecChunk);
  uint64_t* bars = reinterpret_cast<uint64_t*>(red + 16 * 16 * WR);
  uint64_t* xbar = bars + WR * kDecodeStages;

  if (threadIdx.x == 0) {
    for (int i = 0; i < WR * kDecodeStages + 1; ++i) mbar_init(bars + i, 1);
    fence_mbar_init();
  }
  // Zero the staged-X columns past K (the padded tail of the last K block).
  const int tail0 = kend - kstart, tail1 = nkb * 256;
  for (int i = threadIdx.x; i < xrows * (tail1 - tail0); i += blockDim.x) {
    const int tk = i / (tail1 - tail0), k = tail0 + i % (tail1 - tail0);
    Xs[tk * xrow + k] = 0;
  }
  __syncthreads();

  if (threadIdx.x == 0 && xrows > 0) {
    const uint32_t bytes = (uint32_t)(kend - kstart) * 2u;
    mbar_expect_tx(xbar, bytes * xrows);
    for (int tk = 0; tk < xrows; ++tk)
      bulk_g2s(Xs + tk * xrow, p.X + (size_t)(tok0 + tk) * p.K + kstart, bytes, xbar);
  }
  uint8_t* wring = ring + (size_t)warp * kDecodeStages * kDecChunk;
  uint64_t* wbar = bars + warp * kDecodeStages;
  const uint8_t* src = p.dec + ((size_t)rt * p.NKB + kb0) * kDecChunk;
  if (active && lane == 0) {
    for (int s = 0; s < kDecodeStages && s < nkb; ++s) {
      mbar_expect_tx(wbar + s, kDecChunk);
      bulk_g2s(wring + s * kDecChunk, src + (size_t)s * kDecChunk, kDecChunk, wbar + s);
    }
  }

  bool ok = true;
  if (xrows > 0) ok = mbar_wait(xbar, 0);

  float acc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;

  if (active && ok) {
    for (int i = 0; i < nkb; ++i) {
      const int s = i % kDecodeStages;
      if (!mbar_wait(wbar + s, (i / kDecodeStages) & 1)) { ok = false; break; }
      const uint8_t* st = wring + s * kDecChunk;
      const uint4 v0 = lds128(st + lane * 16);
      const uint4 v1 = lds128(st + 512 + lane * 16);
      const uint4 ev = lds128(st + 1024 + lane * 16);
      const __half* sc = reinterpret_cast<const __half*>(st + 1536);
      const float sg[2][2] = {{__half2float(sc[g]), __half2float(sc[g + 8])},
                              {__half2float(sc[16 + g]), __half2float(sc[16 + g + 8])}};
      const uint32_t vw[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
      const uint32_t ew[4] = {ev.x, ev.y, ev.z, ev.w};
      const uint16_t* xk = Xs + (lane & 7) * xrow + i * 256 + (lane >> 3) * 8;
#pragma unroll
      for (int grp = 0; grp < 2; ++grp) {
        float part[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) part[nt][0] = part[nt][1] = part[nt][2] = part[nt][3] = 0.f;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int j = grp * 4 + jj;
          uint32_t a[4];
          decode_word(vw[j], a);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            uint32_t b[4];
            ldmatrix_x4(b, xk + nt * 8 * xrow + 32 * j);
            if (j & 1) mma_sp_16832<1>(part[nt], a, b, ew[j >> 1]);
            else       mma_sp_16832<0>(part[nt], a, b, ew[j >> 1]);
          }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          acc[nt][0] = fmaf(sg[grp][0], part[nt][0], acc[nt][0]);
          acc[nt][1] = fmaf(sg[grp][0], part[nt][1], acc[nt][1]);
          acc[nt][2] = fmaf(sg[grp][1], part[nt][2], acc[nt][2]);
          acc[nt][3] = fmaf(sg[grp][1], part[nt][3], acc[nt][3]);
        }
      }
      __syncwarp();
      if (lane == 0 && i + kDecodeStages < nkb) {
        fence_proxy_async_smem();
        mbar_expect_tx(wbar + s, kDecChunk);
        bulk_g2s(wring + s * kDecChunk, src + (size_t)(i + kDecodeStages) * kDecChunk, kDecChunk, wbar + s);
      }
    }
  }
  if (!ok && lane == 0) record_status(p.status, SLIM_ERR_TIMEOUT);

  // Adapter up-projection for this row tile, done by one rank of the cluster:
  // acc[n][tok] += sum_j R^T[n][j] T[tok][j].
  if (active && p.r16 > 0 && (warp % S) == rank) {
    const int JS = p.r16 / 16;
    const uint4* ra = p.Rf + ((size_t)rt * JS) * 32 + lane;
    for (int js = 0; js < JS; ++js) {
      const uint4 a = __ldg(ra + (size_t)js * 32);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint16_t* tr = p.T + (size_t)(tok0 + nt * 8 + g) * p.r16 + js * 16 + 2 * t;
        const uint32_t b0 = __ldg(reinterpret_cast<const uint32_t*>(tr));
        const uint32_t b1 = __ldg(reinterpret_cast<const uint32_t*>(tr + 8));
        mma_16816(acc[nt], a, b0, b1);
      }
    }
  }

  // Partial tile -> shared memory as [token][row of the group].
  const int RW = 16 * WR;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int tk = nt * 8 + 2 * t;
    const int row = warp * 16 + g;
    red[tk * RW + row] = acc[nt][0];
    red[(tk + 1) * RW + row] = acc[nt][1];
    red[tk * RW + row + 8] = acc[nt][2];
    red[(tk + 1) * RW + row + 8] = acc[nt][3];
  }
  cluster.sync();

  // Rank c adds the cluster's partials for its share of (token, row pair)
  // and stores bf16.
  const int P = Mt * (RW / 2);
  const int pb = (int)((long long)rank * P / S), pe = (int)((long long)(rank + 1) * P / S);
  const bool even_n = (p.N & 1) == 0;
  for (int q = pb + (int)threadIdx.x; q < pe; q += blockDim.x) {
    const int tk = q / (RW / 2), rp = q % (RW / 2);
    const int row = rp * 2;
    const int n = rg * RW + row;
    if (n >= p.N) continue;
    float y0 = 0.f, y1 = 0.f;
    for (int c = 0; c < S; ++c) {
      const float2 v = *reinterpret_cast<const float2*>(cluster.map_shared_rank(red, c) + tk * RW + row);
      y0 += v.x;
      y1 += v.y;
    }
    uint16_t* yp = p.Y + (size_t)(tok0 + tk) * p.N + n;
    if (even_n) {
      *reinterpret_cast<__nv_bfloat162*>(yp) = __floats2bfloat162_rn(y0, y1);
    } else {
      yp[0] = __bfloat16_as_ushort(__float2bfloat16_rn(y0));
      if (n + 1 < p.N) yp[1] = __bfloat16_as_ushort(__float2bfloat16_rn(y1));
    }
  }
  cluster.sync();
}

size_t decode_smem_bytes(int NT, int WR, int seg_kb_max) {
  const size_t xrow = (size_t)seg_kb_max * 256 + 8;
  return (size_t)NT * 8 * xrow * 2 + (size_t)WR * kDecodeStages * kDecChunk + 16 * 16 * WR * 4 +
         (WR * kDecodeStages + 1) * 8;
}

template <typename Kern>
cudaError_t launch_cluster(Kern kern, dim3 grid, dim3 block, size_t smem, int cluster_x, cudaStream_t s,
                           const DecodeParams& p) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster_x;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

template <int NT, int WR>
cudaError_t run_decode(const DecodeParams& p, int S, int n_rg, int n_tt, cudaStream_t s) {
  auto kern = k_decode<NT, WR>;
  const size_t smem = decode_smem_bytes(NT, WR, p.seg_kb_max);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (S > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  return launch_cluster(kern, dim3(S, n_rg, n_tt), dim3(WR * 32), smem, S, s, p);
}

}  // namespace

int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

cudaError_t launch_adapter_down(const slim_layer& L, const uint16_t* X, int M, uint16_t* T, cudaStream_t s) {
  const int KS = L.K / 16;
  const int n_tt = ceil_div(M, 16);
  int S = 8;
  while (S > 1 && S * 4 > KS) S >>= 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(S, L.r16 / 16, n_tt);
  cfg.blockDim = dim3(128);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const uint4* Lf = reinterpret_cast<const uint4*>(L.Lf);
  if (M <= 8) return cudaLaunchKernelEx(&cfg, k_adapter_down<1>, X, M, L.K, Lf, L.r16, T);
  return cudaLaunchKernelEx(&cfg, k_adapter_down<2>, X, M, L.K, Lf, L.r16, T);
}

cudaError_t launch_decode(const slim_layer& L, const uint16_t* X, int M, uint16_t* Y, const uint16_t* T,
                          cudaStream_t s) {
  constexpr int WR = 4;
  const int n_tt = ceil_div(M, 16);
  const int n_rg = ceil_div(L.n_row_tiles, WR);
  const int NT = (M <= 8) ? 1 : 2;
  // Cluster size S (the K split): enough CTAs for ~2 per SM, at most 8
  // (16 when the staged X slice would not fit), never more than K blocks.
  const int target = 2 * num_sms();
  int S = 1;
  while (S < 8 && S < L.n_kblocks && (long long)S * n_rg * n_tt < target) S <<= 1;
  const int max_seg_kb = (NT == 1) ? 16 : 8;   // staged X <= 64 KB
  while (S < 16 && S < L.n_kblocks && ceil_div(L.n_kblocks, S) > max_seg_kb) S = (S < 8) ? S * 2 : 16;
  S = std::min(S, L.n_kblocks);
  DecodeParams p;
  p.X = X;
  p.Y = Y;
  p.dec = L.dec;
  p.Rf = reinterpret_cast<const uint4*>(L.Rf);
  p.T = T;
  p.M = M;
  p.K = L.K;
  p.N = L.N;
  p.NRT = L.n_row_tiles;
  p.NKB = L.n_kblocks;
  p.r16 = L.r16;
  p.seg_kb_max = ceil_div(L.n_kblocks, S);
  p.status = L.status;
  if (NT == 1) return run_decode<1, WR>(p, S, n_rg, n_tt, s);
  return run_decode<2, WR>(p, S, n_rg, n_tt, s);
}

}  // namespace slim

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
// Both kernels are launched with programmatic dependent launch: each one
// lets the next kernel on the stream start launching right away, and bulk-
// loads its share of the packed layer (constant data) before it waits for
// the previous kernel to finish.  Everything that earlier work may have
// written (X, T, the workspace, Y) is touched only after that wait.
//
// Work split: a CTA owns a set of 16-row tiles (one per warp), a contiguous
// range of K (its rank in a cluster that spans K), and up to 16 tokens.  The
// cluster's partial sums are added in rank order through distributed shared
// memory, so results do not depend on timing.
#include <cooperative_groups.h>

#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <map>
#include <mutex>
#include <utility>

#include "slim_common.cuh"
#include "slim_internal.h"

namespace cg = cooperative_groups;

namespace slim {
namespace {

constexpr int kMaxStages = 8;      // bulk-copy ring depth per warp (decode)
constexpr int kAdStages = 4;       // ring depth per warp (adapter down)
constexpr int kAdChunkSteps = 8;   // K/16 steps per adapter ring chunk (4 KB)

// B operand of a dense m16n8k16 MMA for NT 8-token tiles staged row-major in
// shared memory (row stride `ld` elements): ldmatrix matrices 0/1 = tokens
// 0-7, k 0-7 / 8-15; matrices 2/3 (NT == 2) = tokens 8-15.
template <int NT>
__device__ __forceinline__ void load_b16(uint32_t (&b)[4], const uint16_t* base, int ld, int lane) {
  const uint16_t* a = base + ((lane & 7) + ((lane >> 4) & 1) * 8 * (NT - 1)) * ld + ((lane >> 3) & 1) * 8;
  if (NT == 2) ldmatrix_x4(b, a);
  else ldmatrix_x2(b, a);
}

// ---------------------------------------------------------------- T = X L
// Grid (S, ceil(r16/64), ceil(M/16)), cluster (S, 1, 1), 4 warps; warp w owns
// 16 adapter columns j.  Rank c covers K/16 steps [c*KS/S, (c+1)*KS/S); the
// packed L^T fragments of that range stream through a per-warp ring, X is
// staged once per CTA.  Rank partials are added in rank order.
struct AdParams {
  const uint16_t* X;
  const uint4* Lf;
  uint16_t* T;
  int M, K, r16;
  int xrow;            // staged X row length (elements), padded
  int32_t* status;
};

// bf16 NaN: what a T element is written as when a wait it depends on gave up
// (so every output of Y that uses it is NaN, never a plausible value).
constexpr uint16_t kBf16NaN = 0x7FC0;

template <int NT>
__global__ void __launch_bounds__(128) k_adapter_down(const AdParams p) {
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ __align__(128) uint8_t smem[];
  const int S = gridDim.x, rank = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int JT = p.r16 / 16;
  const int jt = blockIdx.y * 4 + warp;
  const bool active = jt < JT;
  const int tt = blockIdx.z, tok0 = tt * 16;
  const int Mt = min(16, p.M - tok0);
  const int xrows = min(Mt, NT * 8);
  const int KS = p.K / 16;
  const int ks0 = (int)((long long)rank * KS / S), ks1 = (int)((long long)(rank + 1) * KS / S);
  const int nks = ks1 - ks0;
  const int nch = ceil_div(nks, kAdChunkSteps);

  uint16_t* Xs = reinterpret_cast<uint16_t*>(smem);
  uint8_t* ring = smem + (size_t)NT * 8 * p.xrow * 2;
  float* part = reinterpret_cast<float*>(ring + 4 * kAdStages * kAdChunkSteps * 512);
  uint64_t* bars = reinterpret_cast<uint64_t*>(part + 4 * 256);
  int* cta_bad = reinterpret_cast<int*>(bars + 4 * kAdStages + 1);   // some wait of this CTA gave up
  uint8_t* wring = ring + warp * kAdStages * kAdChunkSteps * 512;
  uint64_t* wbar = bars + warp * kAdStages;
  const uint8_t* src = reinterpret_cast<const uint8_t*>(p.Lf + ((size_t)jt * KS + ks0) * 32);
  const bool src_ok = dcheck(!active || (ks1 <= KS && tok0 < p.M), p.status);

  if (threadIdx.x == 0) {
    for (int i = 0; i < 4 * kAdStages + 1; ++i) mbar_init(bars + i, 1);
    *cta_bad = 0;
    fence_mbar_init();
  }
  __syncthreads();
  auto issue = [&](int c) {  // chunk c of this warp's K range -> stage c % kAdStages
    if (!src_ok) return;
    const int s0 = c * kAdChunkSteps;
    const uint32_t bytes = (uint32_t)min(kAdChunkSteps, nks - s0) * 512u;
    uint64_t* b = wbar + c % kAdStages;
    mbar_expect_tx(b, bytes);
    bulk_g2s(wring + (c % kAdStages) * kAdChunkSteps * 512, src + (size_t)s0 * 512, bytes, b);
  };
  // The packed adapter is constant: start loading it before the wait.
  if (active && lane == 0)
    for (int c = 0; c < kAdStages && c < nch; ++c) issue(c);
  pdl_wait();
  // The main-product kernel that follows may start loading its weights now;
  // it still waits for this grid before reading T.
  pdl_launch_dependents();
  // X slice with plain loads (not queued behind the bulk copies above).
  {
    const int per_row = nks * 2;   // uint4 per staged row
    for (int i = threadIdx.x; i < xrows * per_row; i += blockDim.x) {
      const int tk = i / per_row, c8 = i % per_row;
      const uint4 v = __ldcg(reinterpret_cast<const uint4*>(p.X + (size_t)(tok0 + tk) * p.K + ks0 * 16) + c8);
      *reinterpret_cast<uint4*>(Xs + tk * p.xrow + c8 * 8) = v;
    }
  }
  __syncthreads();
  bool ok = true;
  float acc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
  if (active && ok) {
    for (int c = 0; c < nch; ++c) {
      const int st = c % kAdStages;
      if (!mbar_wait(wbar + st, (c / kAdStages) & 1)) {
        ok = false;
        // Let the copies issued ahead of the failed wait land first.
        if (lane == 0) {
          const long long deadline = clock64() + kWaitBudgetCycles;
          for (int cc = c; cc < nch && cc < c + kAdStages; ++cc)
            drain_phase(wbar + cc % kAdStages, (cc / kAdStages) & 1, deadline);
        }
        break;
      }
      const uint8_t* lp = wring + st * kAdChunkSteps * 512 + lane * 16;
      const int s0 = c * kAdChunkSteps, s1 = min(nks, s0 + kAdChunkSteps);
      for (int s = s0; s < s1; ++s) {
        const uint4 a = lds128(lp + (s - s0) * 512);
        uint32_t b[4];
        load_b16<NT>(b, Xs + s * 16, p.xrow, lane);
        mma_16816(acc[0], a, b[0], b[1]);
        if (NT == 2) mma_16816(acc[NT - 1], a, b[2], b[3]);
      }
      __syncwarp();
      if (lane == 0 && c + kAdStages < nch) {
        fence_proxy_async_smem();
        issue(c + kAdStages);
      }
    }
  }
  if (!ok && lane == 0) {
    *cta_bad = 1;
    record_status(p.status, SLIM_ERR_TIMEOUT);
  }
  float* wp = part + warp * 256;  // element (tok, row) at tok * 16 + row
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int t = lane & 3, g = lane >> 2;
    const int tk = nt * 8 + 2 * t;
    wp[tk * 16 + g] = acc[nt][0];
    wp[(tk + 1) * 16 + g] = acc[nt][1];
    wp[tk * 16 + g + 8] = acc[nt][2];
    wp[(tk + 1) * 16 + g + 8] = acc[nt][3];
  }
  cluster.sync();
  bool bad = false;
  for (int q = 0; q < S; ++q) bad = bad || *cluster.map_shared_rank(cta_bad, q) != 0;
  const int E = 4 * 16 * 16;
  const int e0 = (int)((long long)rank * E / S), e1 = (int)((long long)(rank + 1) * E / S);
  for (int e = e0 + (int)threadIdx.x; e < e1; e += blockDim.x) {
    const int w = e >> 8, tok = (e >> 4) & 15, row = e & 15;
    const int j = (blockIdx.y * 4 + w) * 16 + row;
    if (j >= p.r16 || tok >= NT * 8) continue;
    if (!dcheck(tok0 + tok < ceil_div(p.M, 16) * 16, p.status)) continue;
    float s = 0.f;
    for (int q = 0; q < S; ++q) s += cluster.map_shared_rank(part, q)[e];
    p.T[(size_t)(tok0 + tok) * p.r16 + j] = bad ? kBf16NaN : __bfloat16_as_ushort(__float2bfloat16_rn(s));
  }
  cluster.sync();
}

// ---------------------------------------------------------------- main product
// CTA = WR row tiles x KW K-warps: warp (wr, kw) multiplies row tile
// rg*WR + wr over the kw-th share of the CTA's K blocks.  The CTA's K range
// is its rank's share when a cluster of S CTAs splits K (S > 1), else all of
// K.  Partials are added in a fixed order: over kw in shared memory, then
// over ranks through distributed shared memory.
struct DecodeParams {
  const uint16_t* X;
  uint16_t* Y;
  const uint8_t* dec;
  const uint4* Rf;
  const uint16_t* T;
  int M, K, N, NRT, NKB;
  int r16;             // adapter rank of each fused linear (R^T tiles)
  int rl16;            // adapter columns of T over all fused linears
  int n_groups;
  int group_end_rt[SLIM_MAX_GROUPS];
  int seg_kb_max;      // largest K-block count of any rank
  int nst;             // ring stages per warp (<= kMaxStages)
  int ad_slots;        // adapter row tiles per CTA rank: ceil(WR / S)
  int xrows_alloc;     // staged token rows: min(16, M)
  int32_t* status;
};

struct DecodeSmem {
  size_t xs, ring, rs, ts, red, bars, flag, total;
};

__host__ __device__ inline DecodeSmem decode_smem(int WR, int KW, int seg_kb_max, int nst, int ad_slots,
                                                  int r16, int rl16, int xrows_alloc) {
  DecodeSmem m;
  size_t off = 0;
  m.xs = off;   off += (size_t)xrows_alloc * (seg_kb_max * 256 + 8) * 2;
  m.ring = off; off += (size_t)WR * KW * nst * kDecChunk;
  m.rs = off;   off += (size_t)ad_slots * (r16 / 16) * 512;
  m.ts = off;   off += (rl16 > 0) ? (size_t)xrows_alloc * (rl16 + 8) * 2 : 0;
  off = (off + 15) / 16 * 16;
  m.red = off;  off += (size_t)KW * 16 * 16 * WR * 4;
  m.bars = off; off += (size_t)(WR * KW * nst + ad_slots + 1) * 8;
  m.flag = off; off += 16;
  m.total = off;
  return m;
}

template <int NT, int WR, int KW>
__global__ void __launch_bounds__(WR * KW * 32) k_decode(const DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int S = gridDim.x, rank = blockIdx.x;
  const int rg = blockIdx.y, tt = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wr = warp % WR, kw = warp / WR;
  const int g = lane >> 2, t = lane & 3;
  const int nst = p.nst;

  const int kb0 = (int)((long long)rank * p.NKB / S), kb1 = (int)((long long)(rank + 1) * p.NKB / S);
  const int nkb = kb1 - kb0;
  const int kstart = kb0 * 256, kend = min(kb1 * 256, p.K);
  const int wkb0 = kw * nkb / KW, wkb1 = (kw + 1) * nkb / KW;   // this warp's blocks (CTA-relative)
  const int xrow = p.seg_kb_max * 256 + 8;
  const int trow = p.rl16 + 8;
  const int tok0 = tt * 16;
  const int Mt = min(16, p.M - tok0);
  const int xrows = min(Mt, NT * 8);
  const int rt = rg * WR + wr;
  const bool active = rt < p.NRT;
  const bool adapter_here = active && kw == 0 && p.r16 > 0 && (wr % S) == rank;
  const int JS = p.r16 / 16;

  const DecodeSmem L = decode_smem(WR, KW, p.seg_kb_max, nst, p.ad_slots, p.r16, p.rl16, p.xrows_alloc);
  uint16_t* Xs = reinterpret_cast<uint16_t*>(smem + L.xs);
  uint8_t* wring = smem + L.ring + (size_t)warp * nst * kDecChunk;
  uint8_t* Rs = smem + L.rs + (size_t)(wr / S) * JS * 512;
  uint16_t* Ts = reinterpret_cast<uint16_t*>(smem + L.ts);
  float* red = reinterpret_cast<float*>(smem + L.red);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* wbar = bars + warp * nst;
  uint64_t* rbar = bars + WR * KW * nst + wr / S;
  int* cta_bad = reinterpret_cast<int*>(smem + L.flag);   // some wait of this CTA gave up

  if (threadIdx.x == 0) {
    for (int i = 0; i < WR * KW * nst + p.ad_slots + 1; ++i) mbar_init(bars + i, 1);
    *cta_bad = 0;
    fence_mbar_init();
  }
  // Zero the staged-X columns past K (the padded tail of the last K block);
  // the bulk copies below write only columns [0, kend - kstart).
  const int tail0 = kend - kstart, tail1 = nkb * 256;
  for (int i = threadIdx.x; i < xrows * (tail1 - tail0); i += blockDim.x) {
    const int tk = i / (tail1 - tail0), k = tail0 + i % (tail1 - tail0);
    Xs[tk * xrow + k] = 0;
  }
  __syncthreads();

  // The packed layer is constant: start streaming it before the wait.
  const int nmine = wkb1 - wkb0;
  const uint8_t* src = p.dec + ((size_t)rt * p.NKB + kb0 + wkb0) * kDecChunk;
  const bool src_ok = dcheck(!active || (rt < p.NRT && kb1 <= p.NKB), p.status);
  if (active && lane == 0 && src_ok) {
    for (int s = 0; s < nst && s < nmine; ++s) {
      mbar_expect_tx(wbar + s, kDecChunk);
      bulk_g2s(wring + s * kDecChunk, src + (size_t)s * kDecChunk, kDecChunk, wbar + s);
    }
    if (adapter_here) {
      mbar_expect_tx(rbar, (uint32_t)JS * 512u);
      bulk_g2s(Rs, p.Rf + (size_t)rt * JS * 32, (uint32_t)JS * 512u, rbar);
    }
  }
  pdl_wait();
  // X slice and T rows with plain loads (not queued behind the bulk copies).
  {
    const int per_row = (kend - kstart) / 8;
    for (int i = threadIdx.x; i < xrows * per_row; i += blockDim.x) {
      const int tk = i / per_row, c8 = i % per_row;
      if (!dcheck(tok0 + tk < p.M && kstart + c8 * 8 + 8 <= p.K, p.status)) continue;
      const uint4 v = __ldcg(reinterpret_cast<const uint4*>(p.X + (size_t)(tok0 + tk) * p.K + kstart) + c8);
      *reinterpret_cast<uint4*>(Xs + tk * xrow + c8 * 8) = v;
    }
    const int t_row = p.rl16 / 8;
    for (int i = threadIdx.x; i < xrows * t_row; i += blockDim.x) {
      const int tk = i / t_row, c8 = i % t_row;
      if (!dcheck(tok0 + tk < ceil_div(p.M, 16) * 16, p.status)) continue;
      const uint4 v = __ldcg(reinterpret_cast<const uint4*>(p.T + (size_t)(tok0 + tk) * p.rl16) + c8);
      *reinterpret_cast<uint4*>(Ts + tk * trow + c8 * 8) = v;
    }
  }
  __syncthreads();
  bool ok = true;

  float acc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;

  // ldmatrix rows are tokens; rows past the staged ones repeat the last
  // staged row (their products land in output columns that are not stored).
  const int last = max(xrows - 1, 0);
  const uint16_t* xk0 = Xs + min(lane & 7, last) * xrow + (lane >> 3) * 8;
  const uint16_t* xk1 = Xs + min(8 + (lane & 7), last) * xrow + (lane >> 3) * 8;

  if (active && ok) {
    for (int i = 0; i < nmine; ++i) {
      const int s = i % nst;
      if (!mbar_wait(wbar + s, (i / nst) & 1)) {
        ok = false;
        // Let the copies issued ahead of the failed wait (and this warp's
        // R^T tiles) land first.
        if (lane == 0) {
          const long long deadline = clock64() + kWaitBudgetCycles;
          for (int ii = i; ii < nmine && ii < i + nst; ++ii) drain_phase(wbar + ii % nst, (ii / nst) & 1, deadline);
          if (adapter_here) drain_phase(rbar, 0, deadline);
        }
        break;
      }
      const uint8_t* st = wring + s * kDecChunk;
      const uint4 v0 = lds128(st + lane * 16);
      const uint4 v1 = lds128(st + 512 + lane * 16);
      const uint4 ev = lds128(st + 1024 + lane * 16);
      const __half* sc = reinterpret_cast<const __half*>(st + 1536);
      const float sg[2][2] = {{__half2float(sc[scale_slot(0, g)]), __half2float(sc[scale_slot(0, g + 8)])},
                              {__half2float(sc[scale_slot(1, g)]), __half2float(sc[scale_slot(1, g + 8)])}};
      const uint32_t vw[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
      const uint32_t ew[4] = {ev.x, ev.y, ev.z, ev.w};
      const int kcol = (wkb0 + i) * 256;
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
            ldmatrix_x4(b, (nt == 0 ? xk0 : xk1) + kcol + 32 * j);
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
      if (src_ok && lane == 0 && i + nst < nmine) {
        fence_proxy_async_smem();
        mbar_expect_tx(wbar + s, kDecChunk);
        bulk_g2s(wring + s * kDecChunk, src + (size_t)(i + nst) * kDecChunk, kDecChunk, wbar + s);
      }
    }
  }

  // The heavy part is done: let the next kernel start loading its constants.
  pdl_launch_dependents();

  // Adapter up-projection for this row tile, by one warp of one rank:
  // acc[n][tok] += sum_j R^T[n][j] T[tok][j].
  if (adapter_here && ok) {
    if (!mbar_wait(rbar, 0)) {
      ok = false;   // (the wait itself bounded the copy's time in flight)
    } else {
      const uint16_t* tb = Ts + ((lane & 7) + ((lane >> 4) & 1) * 8 * (NT - 1)) * trow + ((lane >> 3) & 1) * 8;
      if (NT == 2) tb = Ts + min((lane & 7) + ((lane >> 4) & 1) * 8, last) * trow + ((lane >> 3) & 1) * 8;
      else tb = Ts + min(lane & 7, last) * trow + ((lane >> 3) & 1) * 8;
      // this row tile's fused linear owns T columns [grp * r16, (grp+1) * r16)
      int grp = 0;
      while (grp + 1 < p.n_groups && rt >= p.group_end_rt[grp]) ++grp;
      tb += grp * p.r16;
      for (int js = 0; js < JS; ++js) {
        const uint4 a = lds128(Rs + js * 512 + lane * 16);
        uint32_t b[4];
        if (NT == 2) ldmatrix_x4(b, tb + js * 16);
        else ldmatrix_x2(b, tb + js * 16);
        mma_16816(acc[0], a, b[0], b[1]);
        if (NT == 2) mma_16816(acc[NT - 1], a, b[2], b[3]);
      }
    }
  }
  if (!ok && lane == 0) {
    *cta_bad = 1;
    record_status(p.status, SLIM_ERR_TIMEOUT);
  }

  // Partial tile -> shared memory as [kw][token][row of the group].
  const int RW = 16 * WR;
  float* myred = red + (size_t)kw * 16 * RW;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int tk = nt * 8 + 2 * t;
    const int row = wr * 16 + g;
    myred[tk * RW + row] = acc[nt][0];
    myred[(tk + 1) * RW + row] = acc[nt][1];
    myred[tk * RW + row + 8] = acc[nt][2];
    myred[(tk + 1) * RW + row + 8] = acc[nt][3];
  }
  if (S > 1) cg::this_cluster().sync();
  else __syncthreads();

  // Rank c adds the partials (ranks in order, then K-warps in order) for its
  // share of (token, row pair) and stores bf16; zeros if a wait of any rank
  // gave up.
  bool bad = false;
  for (int c = 0; c < S; ++c)
    bad = bad || *((S > 1) ? cg::this_cluster().map_shared_rank(cta_bad, c) : cta_bad) != 0;
  const int P = Mt * (RW / 2);
  const int pb = (int)((long long)rank * P / S), pe = (int)((long long)(rank + 1) * P / S);
  const bool even_n = (p.N & 1) == 0;
  for (int q = pb + (int)threadIdx.x; q < pe; q += blockDim.x) {
    const int tk = q / (RW / 2), rp = q % (RW / 2);
    const int row = rp * 2;
    const int n = rg * RW + row;
    if (n >= p.N) continue;
    float y0 = 0.f, y1 = 0.f;
    for (int c = 0; c < S && !bad; ++c) {
      const float* rc = (S > 1) ? cg::this_cluster().map_shared_rank(red, c) : red;
      for (int w = 0; w < KW; ++w) {
        const float2 v = *reinterpret_cast<const float2*>(rc + (size_t)w * 16 * RW + tk * RW + row);
        y0 += v.x;
        y1 += v.y;
      }
    }
    uint16_t* yp = p.Y + (size_t)(tok0 + tk) * p.N + n;
    if (!dcheck(tok0 + tk < p.M && n < p.N, p.status)) continue;
    if (even_n) {
      *reinterpret_cast<__nv_bfloat162*>(yp) = __floats2bfloat162_rn(y0, y1);
    } else {
      yp[0] = __bfloat16_as_ushort(__float2bfloat16_rn(y0));
      if (n + 1 < p.N) yp[1] = __bfloat16_as_ushort(__float2bfloat16_rn(y1));
    }
  }
  if (S > 1) cg::this_cluster().sync();
}

template <typename... Args>
cudaError_t launch_ex(void (*kern)(Args...), dim3 grid, dim3 block, size_t smem, int cluster_x, cudaStream_t s,
                      const typename std::remove_reference<Args>::type&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int na = 0;
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  if (cluster_x > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = cluster_x;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// Per-kernel attributes, set once per process for the largest request seen.
template <typename Kern>
cudaError_t prepare(Kern kern, size_t smem, int cluster_x) {
  return ensure_func_attrs(reinterpret_cast<const void*>(kern), smem, cluster_x > 8);
}

template <int NT, int WR, int KW>
cudaError_t run_decode(DecodeParams p, int S, int n_rg, int n_tt, cudaStream_t s) {
  auto kern = k_decode<NT, WR, KW>;
  // ring depth: all of a warp's K blocks when they fit, else kMaxStages
  p.nst = std::min(kMaxStages, ceil_div(p.seg_kb_max, KW));
  p.ad_slots = p.r16 > 0 ? ceil_div(WR, S) : 0;
  auto bytes = [&]() {
    return decode_smem(WR, KW, p.seg_kb_max, p.nst, p.ad_slots, p.r16, p.rl16, p.xrows_alloc).total;
  };
  size_t smem = bytes();
  while (smem > 200 * 1024 && p.nst > 2) {
    --p.nst;
    smem = bytes();
  }
  cudaError_t e = prepare(kern, smem, S);
  if (e != cudaSuccess) return e;
  return launch_ex(kern, dim3(S, n_rg, n_tt), dim3(WR * KW * 32), smem, S, s, p);
}

template <int NT>
cudaError_t run_adapter(const AdParams& p, int S, int n_jg, int n_tt, cudaStream_t s) {
  auto kern = k_adapter_down<NT>;
  const size_t smem = (size_t)NT * 8 * p.xrow * 2 + 4 * kAdStages * kAdChunkSteps * 512 + 4 * 256 * 4 +
                      (4 * kAdStages + 1) * 8 + 16;
  cudaError_t e = prepare(kern, smem, S);
  if (e != cudaSuccess) return e;
  return launch_ex(kern, dim3(S, n_jg, n_tt), dim3(128), smem, S, s, p);
}

// Optional tuning override "WR,KW,S": row tiles per CTA, K-warps per row
// tile, K-split cluster size.
bool decode_override(int& wr, int& kw, int& s) {
  const Tuning t = tuning();
  if (!t.decode_cfg || t.dec_wr == 0) return false;
  wr = t.dec_wr;
  kw = t.dec_kw;
  s = t.dec_s;
  return true;
}

template <int NT>
cudaError_t dispatch_decode(const DecodeParams& p, int WR, int KW, int S, int n_rg, int n_tt, cudaStream_t s) {
  if (WR == 1 && KW == 8) return run_decode<NT, 1, 8>(p, S, n_rg, n_tt, s);
  if (WR == 1 && KW == 4) return run_decode<NT, 1, 4>(p, S, n_rg, n_tt, s);
  if (WR == 2 && KW == 4) return run_decode<NT, 2, 4>(p, S, n_rg, n_tt, s);
  if (WR == 4 && KW == 2) return run_decode<NT, 4, 2>(p, S, n_rg, n_tt, s);
  if (WR == 8 && KW == 1) return run_decode<NT, 8, 1>(p, S, n_rg, n_tt, s);
  return run_decode<NT, 4, 1>(p, S, n_rg, n_tt, s);
}

}  // namespace

// The failure path of every device wait, on its own: one thread waits, with
// the same clock budget as the forward's waits, on a barrier that nothing
// completes; the wait gives up and the kernel records SLIM_ERR_TIMEOUT.
__global__ void k_wait_probe(int32_t* status, long long budget_cycles) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    const long long t0 = clock64();
    bool done = false;
    while (!(done = mbar_try_wait(&bar, 0)))
      if (clock64() - t0 > budget_cycles) break;
    if (!done) record_status(status, SLIM_ERR_TIMEOUT);
  }
}

cudaError_t launch_wait_probe(int32_t* status, int wait_us, cudaStream_t s) {
  int dev = 0, khz = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&khz, cudaDevAttrClockRate, dev);
  if (e != cudaSuccess) return e;
  const long long cycles = std::min<long long>((long long)wait_us * khz / 1000, kWaitBudgetCycles);
  k_wait_probe<<<1, 32, 0, s>>>(status, cycles);
  return cudaGetLastError();
}

cudaError_t ensure_func_attrs(const void* func, size_t smem, bool nonportable_cluster) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, std::pair<size_t, bool>> done;   // (kernel, device) -> set
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  std::pair<size_t, bool>& d = done[{func, dev}];
  if (smem > d.first) {
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    d.first = smem;
  }
  if (nonportable_cluster && !d.second) {
    e = cudaFuncSetAttribute(func, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    d.second = true;
  }
  return cudaSuccess;
}

cudaError_t launch_adapter_down(const slim_layer& L, const uint16_t* X, int M, uint16_t* T, cudaStream_t s) {
  NvtxRange nv("decode: T = X L (k_adapter_down)");
  const int KS = L.K / 16;
  const int n_tt = ceil_div(M, 16);
  const int n_jg = ceil_div(L.rl16 / 16, 4);
  // K split: up to 16 ranks, at least 16 K/16-steps each.
  int S = 16;
  while (S > 1 && S * 16 > KS) S >>= 1;
  AdParams p;
  p.X = X;
  p.Lf = reinterpret_cast<const uint4*>(L.Lf);
  p.T = T;
  p.M = M;
  p.K = L.K;
  p.r16 = L.rl16;   // T columns of all fused linears
  p.xrow = ceil_div(KS, S) * 16 + 8;
  p.status = L.status;
  if (M <= 8) return run_adapter<1>(p, S, n_jg, n_tt, s);
  return run_adapter<2>(p, S, n_jg, n_tt, s);
}

cudaError_t launch_decode(const slim_layer& L, const uint16_t* X, int M, uint16_t* Y, const uint16_t* T,
                          cudaStream_t s) {
  NvtxRange nv("decode: sparse product, adapter T R and epilogue (k_decode)");
  const int n_tt = ceil_div(M, 16);
  const int NT = (M <= 8) ? 1 : 2;
  const int xrows_alloc = std::min(16, M);
  // Staged X slice budget (bytes): keeps two CTAs per SM.
  const size_t x_budget = 64 * 1024;
  int WR = 1, KW = 8, S = 1;
  if (!decode_override(WR, KW, S)) {
    const int target = num_sms();
    if ((size_t)xrows_alloc * L.n_kblocks * 512 <= x_budget) {
      // One row tile per CTA, 8 warps splitting K: no cluster when there are
      // enough row tiles.
      WR = 1;
      KW = 8;
      S = 1;
      while (S < 8 && S < L.n_kblocks && (long long)S * L.n_row_tiles * n_tt < target) S <<= 1;
    } else {
      // The X slice must be split along K: 4 row tiles per CTA share it.
      WR = 4;
      KW = 1;
      S = 2;
      while (S < 16 && S < L.n_kblocks &&
             ((size_t)xrows_alloc * ceil_div(L.n_kblocks, S) * 512 > x_budget ||
              (long long)S * ceil_div(L.n_row_tiles, WR) * n_tt < 2 * target))
        S = (S < 8) ? S * 2 : 16;
    }
  }
  S = std::max(1, std::min(S, L.n_kblocks));
  const int n_rg = ceil_div(L.n_row_tiles, WR);
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
  p.rl16 = L.rl16;
  p.n_groups = L.n_groups;
  for (int gi = 0; gi < SLIM_MAX_GROUPS; ++gi) p.group_end_rt[gi] = ceil_div(L.group_end[gi], 16);
  p.seg_kb_max = ceil_div(L.n_kblocks, S);
  p.nst = 0;
  p.ad_slots = 0;
  p.xrows_alloc = xrows_alloc;
  p.status = L.status;
  if (NT == 1) return dispatch_decode<1>(p, WR, KW, S, n_rg, n_tt, s);
  return dispatch_decode<2>(p, WR, KW, S, n_rg, n_tt, s);
}

size_t forward_ctl_bytes(int r16) {
  return r16 > 0 ? ((size_t)4 * (2 + 2 * (r16 / 16)) + 255) / 256 * 256 : 0;
}

static size_t t_region(int r16, int M) { return ((size_t)ceil_div(M, 16) * 16 * r16 * 2 + 255) / 256 * 256; }

// The tensor-core prefill path serves M > 16 when T = X L of all fused
// linears has at most 1024 columns.
static bool use_prefill(int rl16, int M, bool allow) {
  return allow && M > 16 && rl16 <= 1024 && !tuning().no_prefill;
}

static size_t a1k(size_t x) { return (x + 1023) / 1024 * 1024; }

// T for the prefill path: swizzled tiles of TT tokens x (fused linears x
// ceil(r16/64)) atoms.  Sized for M + kPrefillMaxTile - 1 tokens, the most
// any tile width pads M to, so that the size grows with M whatever tile
// width a smaller M picks (a workspace sized for M serves every M' <= M).
static size_t t_swz_region(const slim_layer& L, int M) {
  return (size_t)(M + kPrefillMaxTile - 1) * L.n_groups * ceil_div(L.r16, 64) * 64 * 2;
}

// The single-launch streaming kernel serves M <= 16 whenever its plan fits
// the device and its workspace fits `ws_limit`.
static bool use_stream(const slim_layer& L, int M, size_t ws_limit) {
  if (M > 16 || tuning().decode_cfg) return false;
  if (!stream_supported(L, M)) return false;
  return stream_workspace_bytes(L, M) <= ws_limit;
}

namespace {

enum class Path { kNone, kPrefill, kStream, kPair };

struct ForwardPlan {
  Path path = Path::kNone;
  size_t ws = 0;        // workspace of a call with exactly M tokens
  size_t ws_upto = 0;   // the most any call with M' <= M tokens needs
  int launches = 0;
};

ForwardPlan forward_plan_uncached(const slim_layer& L, int M, bool allow_prefill, size_t ws_limit) {
  ForwardPlan f;
  if (M <= 0) return f;
  if (use_prefill(L.rl16, M, allow_prefill)) {
    f.path = Path::kPrefill;
    f.ws = a1k(forward_ctl_bytes(L.r16)) + a1k(t_swz_region(L, M)) + prefill_image_bytes(L.N, L.K);
    f.launches = (L.r16 > 0 ? 1 : 0) + 2;   // [X L] + dequant + main
  } else if (use_stream(L, M, ws_limit)) {
    f.path = Path::kStream;
    f.ws = stream_workspace_bytes(L, M);
    f.launches = 1;
  } else {
    f.path = Path::kPair;
    f.ws = L.r16 == 0 ? 0 : forward_ctl_bytes(L.r16) + t_region(L.rl16, M);
    f.launches = (L.r16 > 0 ? 1 : 0) + 1;   // [X L] + main
  }
  return f;
}

// Plans are computed once per (device, tuning, layer shape, M, path limits).
ForwardPlan forward_plan(const slim_layer& L, int M, bool allow_prefill, size_t ws_limit) {
  static PlanCache<19, ForwardPlan> cache;
  const Tuning tn = tuning();
  const long long lim = ws_limit == SIZE_MAX ? -1 : (long long)ws_limit;
  return cache.get({current_device(), (long long)tn.generation, L.K, L.N, L.r16, L.rl16, L.n_groups, M, L.adapter_bits,
                    allow_prefill ? 1 : 0, lim, L.group_end[0], L.group_end[1], L.group_end[2], L.group_end[3],
                    L.group_end[4], L.group_end[5], L.group_end[6], L.group_end[7]},
                   [&] {
                     ForwardPlan f = forward_plan_uncached(L, M, allow_prefill, ws_limit);
                     // A workspace sized for M serves every smaller M: small M
                     // on the single-launch kernel can need more than a larger M.
                     f.ws_upto = f.ws;
                     for (int m = 1; m <= std::min(M - 1, 16); ++m)
                       f.ws_upto = std::max(f.ws_upto, forward_plan_uncached(L, m, allow_prefill, ws_limit).ws);
                     return f;
                   });
}

}  // namespace

size_t forward_workspace_bytes(const slim_layer& L, int M, bool allow_prefill, size_t ws_limit) {
  return forward_plan(L, M, allow_prefill, ws_limit).ws;
}

size_t forward_workspace_bytes_upto(const slim_layer& L, int M, bool allow_prefill, size_t ws_limit) {
  return forward_plan(L, M, allow_prefill, ws_limit).ws_upto;
}

int forward_launches(const slim_layer& L, int M, bool allow_prefill, size_t ws_limit) {
  return forward_plan(L, M, allow_prefill, ws_limit).launches;
}

cudaError_t launch_forward(const slim_layer& L, const uint16_t* X, int M, uint16_t* Y, void* ws, bool allow_prefill,
                           size_t ws_limit, cudaStream_t s) {
  uint8_t* wb = static_cast<uint8_t*>(ws);
  const Path path = forward_plan(L, M, allow_prefill, ws_limit).path;
  if (path == Path::kNone) return cudaSuccess;
  if (path == Path::kPrefill) {
    uint16_t* Tz = L.r16 > 0 ? reinterpret_cast<uint16_t*>(wb + a1k(forward_ctl_bytes(L.r16))) : nullptr;
    uint8_t* img = wb + a1k(forward_ctl_bytes(L.r16)) + (L.r16 > 0 ? a1k(t_swz_region(L, M)) : 0);
    cudaError_t e = cudaSuccess;
    if (L.r16 > 0) e = launch_tgemm(L, X, M, Tz, s);
    if (e != cudaSuccess) return e;
    return launch_prefill(L, X, M, Y, Tz, img, s);
  }
  if (path == Path::kStream) return launch_stream(L, X, M, Y, ws, s);
  // Token-tiled pair: T = X L, then the main product with T R folded in.
  // (The control block at the start of this workspace is not used here.)
  uint16_t* T = L.r16 > 0 ? reinterpret_cast<uint16_t*>(wb + forward_ctl_bytes(L.r16)) : nullptr;
  cudaError_t e;
  if (L.r16 > 0) {
    e = launch_adapter_down(L, X, M, T, s);
    if (e != cudaSuccess) return e;
  }
  return launch_decode(L, X, M, Y, T, s);
}

}  // namespace slim

// Single-launch decode forward for M <= 16 tokens (sm_100a).
//
// Decoding is memory-bound: every packed weight byte is used for one small
// matrix product (thesis §2.5.2 "The Memory-Bound Regime: Inference
// Decoding").  The layer is therefore streamed once, with the copy engines
// kept busy from the first to the last byte, and everything else of the call
// - the adapter's X L, its (X L) R, the cross-warp and cross-panel sums - is
// folded into the same launch so that a chain of calls pays one grid hand-off
// per call.
//
// Work split.  A unit is (K panel p, 16-row tile rt); units are numbered
// panel-major and every CTA owns a contiguous, balanced range of them (a
// persistent grid of at most one CTA per SM).  Each of the 8 main warps takes
// the same 1/8 of every unit's K blocks and streams its 1600-byte packed
// chunks through its own ring of bulk copies, across unit boundaries, so the
// ring never drains while the CTA has work.  The sparse int4 product uses
// mma.sp m16n8k32 (§2.2.3 "Sparse Tensor Core Acceleration"): the 2-bit
// metadata selects the matching activations on the tensor cores.
//
// The adapter (§4, lazy low-rank adapters: never merged into the sparse
// weight) runs on one more warp per CTA: CTA i < JT*SA computes the partial
// T[:, 16 jt .. 16 jt + 15] = X L over the sa-th of SA K ranges and writes
// it to the workspace as 64-bit words that carry the fp32 value and the
// launch's tag (see the control block below), so a reader needs no flag:
// a word with the current tag is the current value.  After its stream,
// every CTA reads the JT*SA partials it needs, adds them in sa order into a
// bf16 T in shared memory and adds R^T T^T to its finished units.  With more
// than one K panel, the panel partials of a row tile meet in the workspace
// and the last one to arrive adds them in panel order.  Every sum has a
// fixed order, so results do not depend on timing.
//
// Control block (start of the workspace, zero before first use): [0]
// sequence number, [1] finished CTAs (rewound to zero by the launch that
// raised it), then one 64-bit arrival word per row tile (launch tag << 32 |
// count).  The last CTA to finish advances the sequence number.  Every word
// this kernel relies on carries the launch's tag (launch_tag(): a bit range
// that no finite data written by any kernel of the library can produce), so
// whatever another layer or another path left in the workspace is never
// mistaken for a value of this launch; only words [0] and [1] must be left
// alone by the other paths, which start their data 256 bytes in.
//
// Failure: if a bounded wait of a CTA gives up, the CTA records
// SLIM_ERR_TIMEOUT and stores zeros for the units it finishes; a CTA whose
// panel partial is part of another CTA's row tile marks the tile's arrival
// word, and that tile is stored as zeros too.
//
// Whole-grid residency is required (CTAs wait for words written by other
// CTAs of the same grid): the host launches at most one CTA per SM, with at
// most one CTA's worth of shared memory.  Every CTA signals the next launch
// once its adapter warp has published its slice (right after the grid
// dependency wait when it has none), so the next grid can start, and
// prefetch its constant data, only once every CTA of this grid is resident;
// its CTAs then wait for this grid with one thread each while the rest of
// their threads sit on a barrier, taking no issue slots from this grid.
#include <algorithm>
#include <cstdlib>

#include "slim_common.cuh"
#include "slim_internal.h"

namespace slim {
namespace {

// Main warps per CTA: 8 (two CTAs of this kernel fit on an SM, so the next
// launch can start while this one finishes) or 16 (more warps to hide the
// latency of long streams).
constexpr int kMaxStagesS = 8;
constexpr int kMaxTCols = 1024;            // adapter columns of T over all fused linears
constexpr int kCtlRtWord = 4;             // 32-bit word index of the first row-tile arrival word
constexpr uint32_t kRtPoison = 0x80000000u; // arrival-word flag: a partial of this row tile is missing
constexpr int kMaxLLLoads = 16;            // tagged partial words in flight per thread
constexpr size_t kSmemLimit = 220 * 1024;
constexpr size_t kRsBudget = 32 * 1024;    // R^T tiles prefetched into shared memory up to this size
constexpr int kAdStageSteps = 8;           // K/16 steps per adapter ring stage (4 KB of packed L^T)
constexpr int kMaxAdStages = 8;

struct StreamParams {
  const uint16_t* X;
  uint16_t* Y;
  const uint8_t* dec;
  const uint4* Rf;
  const uint4* Lf;
  unsigned long long* part_ll;   // [JT][SA][256] tagged X L partials: fp32 bits | launch_tag(seq) << 32
  float* part_main;     // [NRT][P][256] (P > 1)
  uint32_t* ctl;
  int M, K, N, NRT, NKB;
  int r16;              // adapter rank of each fused linear, rounded up to 16 (R^T tiles)
  int rl16;             // adapter columns of T = X L over all fused linears
  int n_groups;
  int group_end_rt[SLIM_MAX_GROUPS];   // row tiles of fused linear g end at group_end_rt[g]
  int P, KP, U;         // K panels, K blocks per panel, units = P * NRT
  int SA;               // adapter K splits
  int nst;              // ring stages per main warp
  int nbuf;             // staged X panels (1 or 2)
  int units_max;        // most units any CTA owns
  int rs_smem;          // R^T tiles of the CTA's units prefetched into shared memory
  int nls;              // adapter ring stages
  int early;            // signal the next launch before the wait (not only after the stream)
  int32_t* status;
  long long t_wait;     // budget (SM cycles) of each wait for a T partial
  uint32_t tag_skew;    // 0; test aid: readers of T partials expect launch_tag(seq + tag_skew)
};

struct StreamSmem {
  size_t xs, ring, red, res, ts, rs, ls, bars, total;
};

__host__ __device__ inline size_t a16(size_t x) { return (x + 15) / 16 * 16; }

// Shared memory: staged X panels, the main warps' chunk rings, the cross-warp
// sum buffers, per-unit results (one K panel only; with several panels the
// unit partials go to the workspace), T, the R^T tiles of the CTA's units,
// the adapter ring, mbarriers.
__host__ __device__ inline StreamSmem stream_smem(int NT, int MW, int xrows, int KP, int nbuf, int nst,
                                                  int units_max, int r16, int rl16, int rs_smem, int nls) {
  const int RSZ = NT * 8 * 16;
  StreamSmem m;
  size_t off = 0;
  m.xs = off;   off = a16(off + (size_t)nbuf * xrows * (KP * 256 + 8) * 2);
  m.ring = off; off = a16(off + (size_t)MW * nst * kDecChunk);
  m.red = off;  off = a16(off + (size_t)2 * MW * RSZ * 4);
  m.res = off;  off = a16(off + (nbuf == 1 ? (size_t)units_max * RSZ * 4 : 0));
  m.ts = off;   off = a16(off + (rl16 > 0 ? (size_t)16 * (rl16 + 8) * 2 : 0));
  m.rs = off;   off = a16(off + (rs_smem ? (size_t)units_max * (r16 / 16) * 512 : 0));
  m.ls = off;   off = a16(off + (size_t)nls * kAdStageSteps * 512);
  m.bars = off; off += (size_t)(MW * nst + nls + 2) * 8 + 16 + 4 * MW;
  m.total = off;
  return m;
}

// Barrier 2: every thread of the CTA (main warps and adapter warp, reached
// from their own code paths).
template <int MW>
__device__ __forceinline__ void bar_all() {
  asm volatile("bar.sync 2, %0;" ::"n"((MW + 1) * 32) : "memory");
}
template <int MW>
__device__ __forceinline__ void bar_main() {
  asm volatile("bar.sync 1, %0;" ::"n"(MW * 32) : "memory");
}
// Barrier of the main warps that also returns the AND of `v` over them.
template <int MW>
__device__ __forceinline__ bool bar_main_and(bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, 1, %2, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(MW * 32)
      : "memory");
  return r != 0;
}

// Position in a main warp's chunk sequence (chunk i goes to ring slot
// i % nst, phase (i / nst) & 1) of chunk `k_in_unit` of unit u, for a CTA
// whose units start at u0.  Used only after a give-up, so kept out of line.
__device__ __noinline__ int chunk_index(int u0, int u, int k_in_unit, int NRT, int KP, int NKB, int warp,
                                        int log2mw) {
  int n = 0;
  for (int v = u0; v < u; ++v) {
    const int pk0 = (v / NRT) * KP;
    const int nk = min(KP, NKB - pk0);
    n += (((warp + 1) * nk) >> log2mw) - ((warp * nk) >> log2mw);
  }
  return n + k_in_unit;
}

template <int NT, int MW>
__global__ void __launch_bounds__((MW + 1) * 32, MW == 8 ? 2 : 1) k_stream(const StreamParams p) {
  constexpr int kMainWarps = MW;
  constexpr int kLog2MW = MW == 8 ? 3 : 4;
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int RSZ = NT * 8 * 16;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int G = gridDim.x, cta = blockIdx.x;
  const int xrows = min(p.M, NT * 8);
  const int last = xrows - 1;
  const int JT = p.rl16 / 16;      // T column tiles (all fused linears)
  const int JS = p.r16 / 16;       // R^T tiles of one row tile
  const int nst = p.nst;
  const int xrow = p.KP * 256 + 8;
  const int trow = p.rl16 + 8;
  const int u0 = (int)((long long)cta * p.U / G), u1 = (int)((long long)(cta + 1) * p.U / G);
  const int nunits = u1 - u0;
  const int p_first = nunits > 0 ? u0 / p.NRT : 0;
  const int p_last = nunits > 0 ? (u1 - 1) / p.NRT : -1;

  const StreamSmem L =
      stream_smem(NT, MW, xrows, p.KP, p.nbuf, nst, p.units_max, p.r16, p.rl16, p.rs_smem, p.nls);
  uint16_t* Xs = reinterpret_cast<uint16_t*>(smem + L.xs);
  uint8_t* ring = smem + L.ring;
  float* red = reinterpret_cast<float*>(smem + L.red);
  float* res = reinterpret_cast<float*>(smem + L.res);
  uint16_t* Ts = reinterpret_cast<uint16_t*>(smem + L.ts);
  uint8_t* Rs = smem + L.rs;
  uint8_t* Ls = smem + L.ls;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* lbar = bars + kMainWarps * nst;    // [nls] adapter ring
  uint64_t* rbar = lbar + p.nls;               // R^T tiles
  uint64_t* xbar = rbar + 1;                   // X staged (main threads arrive)
  volatile uint32_t* sh = reinterpret_cast<volatile uint32_t*>(xbar + 1);   // [0] seq, [1] T ready
  int* fail_at = const_cast<int*>(reinterpret_cast<volatile int*>(sh + 4));   // [main warp] (after a give-up)

  if (threadIdx.x == 0) {
    for (int i = 0; i < kMainWarps * nst + p.nls + 1; ++i) mbar_init(bars + i, 1);
    mbar_init(xbar, kMainWarps * 32);
    fence_mbar_init();
  }
  // Zero the staged-X columns past K (the padded tail of the last K block).
  for (int b = 0; b < p.nbuf; ++b) {
    const int pb = p_first + b;
    if (pb > p_last) break;
    const int kstart = pb * p.KP * 256;
    const int ncols = min(p.KP * 256, p.K - kstart);
    const int pad = min(p.KP, p.NKB - pb * p.KP) * 256 - ncols;
    for (int i = threadIdx.x; i < xrows * pad; i += blockDim.x)
      Xs[(size_t)b * xrows * xrow + (i / pad) * xrow + ncols + i % pad] = 0;
  }
  __syncthreads();

  if (warp < kMainWarps) {
    // ------------------------------------------------------------ main warps
    // Cursor over this warp's chunks: unit u = (panel pp, row tile rt), the
    // warp's K blocks [lo, hi) of that panel, k the current one.  Advanced
    // incrementally: no division on the per-chunk path.
    struct Cursor {
      int u, rt, pp, lo, hi, k;
    };
    auto set_range = [&](Cursor& c) {
      const int pk0 = c.pp * p.KP;
      const int nk = min(p.KP, p.NKB - pk0);
      c.lo = pk0 + ((warp * nk) >> kLog2MW);
      c.hi = pk0 + (((warp + 1) * nk) >> kLog2MW);
      c.k = c.lo;
    };
    auto next_unit = [&](Cursor& c) {
      ++c.u;
      if (++c.rt == p.NRT) {
        c.rt = 0;
        ++c.pp;
      }
      set_range(c);
    };
    auto start = [&](Cursor& c) {
      c.u = u0;
      c.rt = u0 % p.NRT;
      c.pp = u0 / p.NRT;
      set_range(c);
    };
    Cursor pc;   // producer: next chunk to copy, kept past empty ranges
    start(pc);
    auto settle = [&]() {
      while (pc.u < u1 && pc.k >= pc.hi) next_unit(pc);
    };
    settle();
    uint8_t* wring = ring + (size_t)warp * nst * kDecChunk;
    uint64_t* wbar = bars + warp * nst;
    auto issue = [&](int s) {
      const uint8_t* src = p.dec + ((size_t)pc.rt * p.NKB + pc.k) * kDecChunk;
      mbar_expect_tx(wbar + s, kDecChunk);
      bulk_g2s(wring + s * kDecChunk, src, kDecChunk, wbar + s);
    };
    auto seq_index = [&](int u, int k, int lo) {
      return chunk_index(u0, u, k - lo, p.NRT, p.KP, p.NKB, warp, kLog2MW);
    };
    // The packed layer is constant: start streaming it before the wait.
    for (int s = 0; s < nst && pc.u < u1; ++s) {
      if (lane == 0) issue(s);
      ++pc.k;
      settle();
    }
    // One thread waits for the previous grid; the others block on the
    // barrier, where they take no issue slots from the grid still running
    // on this SM.
    if (p.early) pdl_launch_dependents();
    if (threadIdx.x == 0) pdl_wait();
    bar_all<MW>();
    if (threadIdx.x == 0) sh[0] = JT > 0 ? *reinterpret_cast<volatile uint32_t*>(p.ctl) : 0u;
    // X panels with plain loads (not queued behind the bulk copies above).
    for (int b = 0; b < p.nbuf; ++b) {
      const int pb = p_first + b;
      if (pb > p_last) break;
      const int kstart = pb * p.KP * 256;
      const int per_row = min(p.KP * 256, p.K - kstart) / 8;
      for (int i = threadIdx.x; i < xrows * per_row; i += kMainWarps * 32) {
        const int tk = i / per_row, c8 = i % per_row;
        const uint4 v = __ldcg(reinterpret_cast<const uint4*>(p.X + (size_t)tk * p.K + kstart) + c8);
        *reinterpret_cast<uint4*>(Xs + (size_t)b * xrows * xrow + tk * xrow + c8 * 8) = v;
      }
    }
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(xbar)) : "memory");
    bar_main<MW>();
    const uint32_t seq = sh[0];

    bool ok = true;
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
    Cursor cc;   // consumer
    start(cc);
    int st = 0, buf = 0;
    uint32_t ph = 0;
    const uint32_t ring_s = smem_u32(wring), bar_s = smem_u32(wbar);
    const uint32_t xs_s = smem_u32(Xs);
    for (int uu = 0; uu < nunits; ++uu) {
      if (uu > 0) next_unit(cc);
      const int pk0 = cc.pp * p.KP;
      // ldmatrix rows are tokens; rows past the staged ones repeat the last
      // staged row (their products land in outputs that are not stored).
      const uint32_t xb = xs_s + (uint32_t)((cc.pp - p_first) * xrows * xrow) * 2u;
      const uint32_t xk0 = xb + (uint32_t)(min(lane & 7, last) * xrow + (lane >> 3) * 8) * 2u;
      const uint32_t xk1 = xb + (uint32_t)(min(8 + (lane & 7), last) * xrow + (lane >> 3) * 8) * 2u;
      for (int kb = cc.lo; kb < cc.hi; ++kb) {
        if (ok) {
          ok = __all_sync(0xffffffffu, mbar_wait_s(bar_s + st * 8, ph));
          if (!ok && lane == 0) fail_at[warp] = seq_index(cc.u, kb, cc.lo);   // first chunk not consumed
        }
        if (ok) {
          const uint32_t sp = ring_s + st * kDecChunk;
          const uint4 v0 = lds128_s(sp + lane * 16);
          const uint4 v1 = lds128_s(sp + 512 + lane * 16);
          const uint4 ev = lds128_s(sp + 1024 + lane * 16);
          // scales [group][row] as fp16, non-negative by construction
          const float sg[2][2] = {{f16_nonneg_bits_to_f32(lds16_s(sp + 1536 + 2 * g)),
                                   f16_nonneg_bits_to_f32(lds16_s(sp + 1536 + 2 * (g + 8)))},
                                  {f16_nonneg_bits_to_f32(lds16_s(sp + 1568 + 2 * g)),
                                   f16_nonneg_bits_to_f32(lds16_s(sp + 1568 + 2 * (g + 8)))}};
          const uint32_t vw[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
          const uint32_t ew[4] = {ev.x, ev.y, ev.z, ev.w};
          const uint32_t kofs = (uint32_t)(kb - pk0) * 512u;   // 256 bf16 per K block
          // Per scale group two accumulator sets (even / odd MMA step), so
          // the tensor-core chain of a group is two MMAs long, not four.
#pragma unroll
          for (int grp = 0; grp < 2; ++grp) {
            float part[2][NT][4];
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) part[h][nt][0] = part[h][nt][1] = part[h][nt][2] = part[h][nt][3] = 0.f;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              const int j = grp * 4 + jj;
              uint32_t a[4];
              decode_word(vw[j], a);
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                uint32_t b[4];
                ldmatrix_x4_s(b, (nt == 0 ? xk0 : xk1) + kofs + 64 * j);
                if (j & 1) mma_sp_16832<1>(part[jj & 1][nt], a, b, ew[j >> 1]);
                else       mma_sp_16832<0>(part[jj & 1][nt], a, b, ew[j >> 1]);
              }
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              acc[nt][0] = fmaf(sg[grp][0], part[0][nt][0] + part[1][nt][0], acc[nt][0]);
              acc[nt][1] = fmaf(sg[grp][0], part[0][nt][1] + part[1][nt][1], acc[nt][1]);
              acc[nt][2] = fmaf(sg[grp][1], part[0][nt][2] + part[1][nt][2], acc[nt][2]);
              acc[nt][3] = fmaf(sg[grp][1], part[0][nt][3] + part[1][nt][3], acc[nt][3]);
            }
          }
        }
        __syncwarp();
        if (ok && pc.u < u1) {
          if (lane == 0) {
            fence_proxy_async_smem();
            issue(st);
          }
          ++pc.k;
          settle();
        }
        if (++st == nst) {
          st = 0;
          ph ^= 1u;
        }
      }
      // Unit done: warp partial -> red[buf][warp] as [token][row]; warp
      // uu % 8 adds the 8 partials in warp order into res[uu] (one K panel)
      // or into the unit's panel partial in the workspace.
      float* myred = red + (size_t)(buf * kMainWarps + warp) * RSZ;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int tk = nt * 8 + 2 * t;
        myred[tk * 16 + g] = acc[nt][0];
        myred[(tk + 1) * 16 + g] = acc[nt][1];
        myred[tk * 16 + g + 8] = acc[nt][2];
        myred[(tk + 1) * 16 + g + 8] = acc[nt][3];
        acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
      }
      bar_main<MW>();
      if (warp == uu % kMainWarps) {
        float* dst = p.P == 1 ? res + (size_t)uu * RSZ : p.part_main + ((size_t)cc.rt * p.P + cc.pp) * 256;
        for (int e = lane; e < xrows * 16; e += 32) {
          float s = 0.f;
#pragma unroll
          for (int w = 0; w < kMainWarps; ++w) s += red[(size_t)(buf * kMainWarps + w) * RSZ + e];
          dst[e] = s;
        }
      }
      buf ^= 1;
    }
    if (!ok && lane == 0) {
      // Let the copies issued and not consumed land before the CTA exits.
      const long long deadline = clock64() + kWaitBudgetCycles;
      const int n_issued = pc.u < u1 ? seq_index(pc.u, pc.k, pc.lo) : seq_index(u1, 0, 0);
      for (int i = fail_at[warp]; i < n_issued; ++i) drain_phase(wbar + i % nst, (i / nst) & 1, deadline);
    }

    // Adapter: T[tok][16 jt + j] = sum over sa, in order, of the tagged
    // partials of this launch, rounded to bf16 into shared memory.  Each
    // thread owns whole outputs, so the order is fixed.
    const uint32_t tag = launch_tag(seq);
    const uint32_t ttag = launch_tag(seq + p.tag_skew);   // == tag outside the failure-path test
    bool tready = true;
    if (JT > 0) {
      const int n_out = JT * xrows * 16;
      for (int o = threadIdx.x; o < n_out; o += kMainWarps * 32) {
        const int jt = o / (xrows * 16), e = o % (xrows * 16);
        const unsigned long long* src = p.part_ll + (size_t)jt * p.SA * 256 + e;
        float sum = 0.f;
        for (int q0 = 0; q0 < p.SA; q0 += kMaxLLLoads) {
          unsigned long long v[kMaxLLLoads];
#pragma unroll
          for (int q = 0; q < kMaxLLLoads; ++q)
            if (q0 + q < p.SA) v[q] = ld_relaxed_u64(src + (size_t)(q0 + q) * 256);
#pragma unroll
          for (int q = 0; q < kMaxLLLoads; ++q) {
            if (q0 + q < p.SA) {
              if (tready && (uint32_t)(v[q] >> 32) != ttag) {
                const long long c0 = clock64();
                do {
                  v[q] = ld_relaxed_u64(src + (size_t)(q0 + q) * 256);
                  if (clock64() - c0 > p.t_wait) break;
                } while ((uint32_t)(v[q] >> 32) != ttag);
                if ((uint32_t)(v[q] >> 32) != ttag) tready = false;
              }
              sum += __uint_as_float((uint32_t)v[q]);
            }
          }
        }
        Ts[(e >> 4) * trow + jt * 16 + (e & 15)] = __bfloat16_as_ushort(__float2bfloat16_rn(sum));
      }
    }
    // One decision for the whole CTA: every wait of its main warps (their
    // streams, the T partials, the R^T tiles) completed.  Otherwise its
    // outputs are stored as zeros.
    bool good = ok && tready;
    if (JT > 0 && p.rs_smem && nunits > 0) good = mbar_wait(rbar, 0) && good;   // waited for even after a give-up
    good = bar_main_and<MW>(good);   // also orders the T writes above before the reads below
    if (!good && threadIdx.x == 0) record_status(p.status, SLIM_ERR_TIMEOUT);
    const bool rs_ok = JT > 0 && good;

    // Finish units: (panel sum) + R^T T^T + bf16 store.  Warp w takes units
    // w, w + 8, ...
    unsigned long long* rt_word = reinterpret_cast<unsigned long long*>(p.ctl + kCtlRtWord);
    for (int uu = warp; uu < nunits; uu += kMainWarps) {
      const int u = u0 + uu, rt = u % p.NRT;
      // One K panel: the unit result is in res.  Several: this warp wrote
      // the unit's panel partial at the end of the unit; the last of the
      // row tile's P partials to arrive adds them in panel order (into this
      // warp's sum buffer, free now).  The arrival word counts this launch's
      // arrivals: a word with an older tag counts as zero.
      float* ru = p.P == 1 ? res + (size_t)uu * RSZ : red + (size_t)warp * RSZ;
      bool store = good;
      if (p.P > 1) {
        __threadfence();
        __syncwarp();
        uint32_t lastp = 0, poisoned = 0;
        if (lane == 0) {
          unsigned long long* w = rt_word + rt;
          unsigned long long old = ld_relaxed_u64(w);
          uint32_t cnt;
          while (true) {
            cnt = (uint32_t)(old >> 32) == tag ? (uint32_t)old : 0u;
            const uint32_t nc = ((cnt & ~kRtPoison) + 1u) | (cnt & kRtPoison) | (good ? 0u : kRtPoison);
            const unsigned long long prev = atomicCAS(w, old, ((unsigned long long)tag << 32) | nc);
            if (prev == old) {
              cnt = nc;
              break;
            }
            old = prev;
          }
          lastp = (cnt & ~kRtPoison) == (uint32_t)p.P ? 1u : 0u;
          poisoned = (cnt & kRtPoison) ? 1u : 0u;
        }
        lastp = __shfl_sync(0xffffffffu, lastp, 0);
        poisoned = __shfl_sync(0xffffffffu, poisoned, 0);
        if (!lastp) continue;
        store = store && !poisoned;
        __threadfence();
        for (int e = lane; e < xrows * 16; e += 32) {
          float s = 0.f;
          for (int q = 0; q < p.P; ++q) s += __ldcg(p.part_main + ((size_t)rt * p.P + q) * 256 + e);
          ru[e] = s;
        }
        __syncwarp();
      }
      if (!store) {
        for (int e = lane; e < xrows * 16; e += 32) ru[e] = 0.f;
        __syncwarp();
      } else if (rs_ok) {
        float a4[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int tk = nt * 8 + 2 * t;
          a4[nt][0] = tk < xrows ? ru[tk * 16 + g] : 0.f;
          a4[nt][1] = tk + 1 < xrows ? ru[(tk + 1) * 16 + g] : 0.f;
          a4[nt][2] = tk < xrows ? ru[tk * 16 + g + 8] : 0.f;
          a4[nt][3] = tk + 1 < xrows ? ru[(tk + 1) * 16 + g + 8] : 0.f;
        }
        // This row tile's fused linear owns T columns [grp * r16, (grp+1) * r16).
        int grp = 0;
        while (grp + 1 < p.n_groups && rt >= p.group_end_rt[grp]) ++grp;
        const uint16_t* tb = (NT == 2) ? Ts + min((lane & 7) + ((lane >> 4) & 1) * 8, last) * trow
                                       : Ts + min(lane & 7, last) * trow;
        tb += ((lane >> 3) & 1) * 8 + grp * p.r16;
        for (int js0 = 0; js0 < JS; js0 += 8) {
          uint4 af[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            if (js0 + q < JS) {
              af[q] = p.rs_smem ? lds128(Rs + ((size_t)uu * JS + js0 + q) * 512 + lane * 16)
                                : __ldg(p.Rf + ((size_t)rt * JS + js0 + q) * 32 + lane);
            }
          }
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            if (js0 + q < JS) {
              uint32_t b[4];
              if (NT == 2) ldmatrix_x4(b, tb + (js0 + q) * 16);
              else ldmatrix_x2(b, tb + (js0 + q) * 16);
              mma_16816(a4[0], af[q], b[0], b[1]);
              if (NT == 2) mma_16816(a4[NT - 1], af[q], b[2], b[3]);
            }
          }
        }
        __syncwarp();
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int tk = nt * 8 + 2 * t;
          if (tk < xrows) {
            ru[tk * 16 + g] = a4[nt][0];
            ru[tk * 16 + g + 8] = a4[nt][2];
          }
          if (tk + 1 < xrows) {
            ru[(tk + 1) * 16 + g] = a4[nt][1];
            ru[(tk + 1) * 16 + g + 8] = a4[nt][3];
          }
        }
        __syncwarp();
      }
      const bool even_n = (p.N & 1) == 0;
      for (int q = lane; q < xrows * 8; q += 32) {
        const int tk = q >> 3, row = (q & 7) * 2;
        const int n = rt * 16 + row;
        if (n >= p.N) continue;
        const float y0 = ru[tk * 16 + row], y1 = ru[tk * 16 + row + 1];
        uint16_t* yp = p.Y + (size_t)tk * p.N + n;
        if (even_n) {
          *reinterpret_cast<__nv_bfloat162*>(yp) = __floats2bfloat162_rn(y0, y1);
        } else {
          yp[0] = __bfloat16_as_ushort(__float2bfloat16_rn(y0));
          if (n + 1 < p.N) yp[1] = __bfloat16_as_ushort(__float2bfloat16_rn(y1));
        }
      }
      __syncwarp();   // ru is reused by this warp's next unit
    }
  } else {
    // ------------------------------------------------------------ adapter warp
    const int item = cta;
    const bool has_item = JT > 0 && item < JT * p.SA;
    const int KS = p.K / 16;
    const int jt = has_item ? item / p.SA : 0, sa = has_item ? item % p.SA : 0;
    const int s0 = (int)((long long)sa * KS / p.SA), s1 = has_item ? (int)((long long)(sa + 1) * KS / p.SA) : s0;
    const int nlc = ceil_div(s1 - s0, kAdStageSteps);   // ring chunks of this item
    const uint8_t* lsrc = reinterpret_cast<const uint8_t*>(p.Lf + ((size_t)jt * KS + s0) * 32);
    auto lissue = [&](int c) {
      const int st = c % p.nls;
      const uint32_t bytes = (uint32_t)min(kAdStageSteps, s1 - s0 - c * kAdStageSteps) * 512u;
      mbar_expect_tx(lbar + st, bytes);
      bulk_g2s(Ls + (size_t)st * kAdStageSteps * 512, lsrc + (size_t)c * kAdStageSteps * 512, bytes, lbar + st);
    };
    // Constant data before the wait: the item's packed L^T, the R^T tiles.
    if (lane == 0) {
      for (int c = 0; c < p.nls && c < nlc; ++c) lissue(c);
      if (JT > 0 && p.rs_smem && nunits > 0) {
        mbar_expect_tx(rbar, (uint32_t)nunits * JS * 512u);
        for (int uu = 0; uu < nunits; ++uu)
          bulk_g2s(Rs + (size_t)uu * JS * 512, p.Rf + (size_t)((u0 + uu) % p.NRT) * JS * 32, (uint32_t)JS * 512u,
                   rbar);
      }
    }
    if (p.early) pdl_launch_dependents();
    bar_all<MW>();   // the previous grid has completed (thread 0 waited)
    if (has_item) {
      const uint32_t seq = *reinterpret_cast<volatile uint32_t*>(p.ctl);
      float acc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
      // A = L^T fragments (16 columns j x 16 k).  B = X: from the staged
      // panel when there is a single one (it covers all of K), else read
      // from global memory in the m16n8k16 B-fragment layout.
      const bool xs_ok = p.P == 1;
      bool ok = !xs_ok || mbar_wait(xbar, 0);
      const int xr = NT == 2 ? min((lane & 7) + ((lane >> 4) & 1) * 8, last) : min(lane & 7, last);
      const uint16_t* xsb = Xs + xr * xrow + ((lane >> 3) & 1) * 8;
      const uint16_t* xa = p.X + (size_t)min(g, last) * p.K + 2 * t;
      const uint16_t* xc = p.X + (size_t)min(8 + g, last) * p.K + 2 * t;
      int fail_c = 0;   // first chunk whose wait gave up
      for (int c = 0; c < nlc; ++c) {
        const int st = c % p.nls;
        if (ok) ok = mbar_wait(lbar + st, (c / p.nls) & 1);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) {
          fail_c = c;
          break;
        }
        const int sb = s0 + c * kAdStageSteps;
        const int n = min(kAdStageSteps, s1 - sb);
        uint32_t bx[kAdStageSteps][4];
        if (!xs_ok) {
#pragma unroll
          for (int q = 0; q < kAdStageSteps; ++q) {
            if (q < n) {
              const int k0 = (sb + q) * 16;
              bx[q][0] = __ldcg(reinterpret_cast<const unsigned int*>(xa + k0));
              bx[q][1] = __ldcg(reinterpret_cast<const unsigned int*>(xa + k0 + 8));
              if (NT == 2) {
                bx[q][2] = __ldcg(reinterpret_cast<const unsigned int*>(xc + k0));
                bx[q][3] = __ldcg(reinterpret_cast<const unsigned int*>(xc + k0 + 8));
              }
            }
          }
        }
#pragma unroll
        for (int q = 0; q < kAdStageSteps; ++q) {
          if (q < n) {
            const uint4 a = lds128(Ls + ((size_t)st * kAdStageSteps + q) * 512 + lane * 16);
            uint32_t b[4];
            if (xs_ok) {
              if (NT == 2) ldmatrix_x4(b, xsb + (sb + q) * 16);
              else ldmatrix_x2(b, xsb + (sb + q) * 16);
            } else {
              b[0] = bx[q][0];
              b[1] = bx[q][1];
              b[2] = bx[q][2];
              b[3] = bx[q][3];
            }
            mma_16816(acc[0], a, b[0], b[1]);
            if (NT == 2) mma_16816(acc[NT - 1], a, b[2], b[3]);
          }
        }
        __syncwarp();
        if (lane == 0 && c + p.nls < nlc) {
          fence_proxy_async_smem();
          lissue(c + p.nls);
        }
      }
      if (!ok && lane == 0) {
        record_status(p.status, SLIM_ERR_TIMEOUT);
        // Let the copies issued ahead of the failed wait land first.
        const long long deadline = clock64() + kWaitBudgetCycles;
        for (int c = fail_c; c < nlc && c < fail_c + p.nls; ++c) drain_phase(lbar + c % p.nls, (c / p.nls) & 1, deadline);
      }
      if (ok) {
        // Partial tile [token][column] -> workspace as tagged words.
        unsigned long long* mine = p.part_ll + ((size_t)jt * p.SA + sa) * 256;
        const unsigned long long tag = (unsigned long long)launch_tag(seq) << 32;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int tk = nt * 8 + 2 * t;
          if (tk < xrows) {
            st_relaxed_u64(mine + tk * 16 + g, tag | __float_as_uint(acc[nt][0]));
            st_relaxed_u64(mine + tk * 16 + g + 8, tag | __float_as_uint(acc[nt][2]));
          }
          if (tk + 1 < xrows) {
            st_relaxed_u64(mine + (tk + 1) * 16 + g, tag | __float_as_uint(acc[nt][1]));
            st_relaxed_u64(mine + (tk + 1) * 16 + g + 8, tag | __float_as_uint(acc[nt][3]));
          }
        }
      }
    }
    // This CTA's slice is published: let the next launch start loading its
    // constants.
    pdl_launch_dependents();
  }

  if (JT == 0) return;
  // The last CTA to finish advances the sequence word for the next launch.
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t seq = sh[0];
    __threadfence();
    const uint32_t fin = atomicAdd(p.ctl + 1, 1u);
    if (fin == (uint32_t)G - 1u) {
      p.ctl[1] = 0u;
      p.ctl[0] = seq + 1u;
      __threadfence();
    }
  }
}

// ------------------------------------------------------------ host planning
struct StreamPlan {
  bool ok = false;
  int NT = 1, MW = 8, P = 1, KP = 1, U = 0, G = 0, units_max = 0, nst = 1, nbuf = 1, SA = 1, rs_smem = 0, nls = 0;
  bool ad_prefetched = true;   // every adapter item's L^T slice fits the ring (no copies after the wait)
  size_t smem = 0;
};

StreamPlan plan_stream_mw(const slim_layer& L, int M, int MW);

// Main warps per CTA: 8 while a CTA streams few chunks (two CTAs fit on an
// SM, so the next launch overlaps this one's tail), 16 for long streams
// (more warps to hide the latency of the per-chunk work).
StreamPlan plan_stream_uncached(const slim_layer& L, int M, const Tuning& tn) {
  if (M < 1 || M > 16 || L.rl16 > kMaxTCols || tn.no_stream) return StreamPlan();
  int MW = (long long)ceil_div(L.n_row_tiles, num_sms()) * L.n_kblocks >= 128 ? 16 : 8;
  if (tn.stream_warps) MW = tn.stream_warps;
  StreamPlan pl = plan_stream_mw(L, M, MW);
  if (!pl.ok) pl = plan_stream_mw(L, M, 24 - MW);
  // Two token tiles with an adapter slice that does not fit its ring: the
  // slice's refills queue behind the weight stream and the adapter becomes
  // the critical path unless the stream is long; the token-tiled pair is
  // faster there.
  if (pl.ok && pl.NT == 2 && !pl.ad_prefetched && (long long)pl.units_max * pl.KP < 128) pl.ok = false;
  return pl;
}

// Plans depend on the layer's shape, M, the device and the tuning knobs;
// each is computed once.
StreamPlan plan_stream(const slim_layer& L, int M) {
  static PlanCache<7, StreamPlan> cache;
  const Tuning tn = tuning();
  return cache.get({current_device(), (long long)tn.generation, L.K, L.N, L.r16, L.rl16, M},
                   [&] { return plan_stream_uncached(L, M, tn); });
}

StreamPlan plan_stream_mw(const slim_layer& L, int M, int MW) {
  StreamPlan pl;
  const int NT = M <= 8 ? 1 : 2;
  const int xrows = std::min(M, NT * 8);
  const int JT = L.rl16 / 16;
  const int nsm = num_sms();
  if (JT > nsm) return pl;
  // Fewest K panels first (each extra panel adds a partial per row tile);
  // within a panel count, the deepest rings that fit.
  for (int Pwant = 1; Pwant <= L.n_kblocks; ++Pwant) {
    const int KP = ceil_div(L.n_kblocks, Pwant);
    const int P = ceil_div(L.n_kblocks, KP);
    if (P > 1 && L.r16 == 0) return pl;   // panel partials need a workspace; r = 0 has none
    if (P > 1 && P > Pwant) continue;
    const int U = P * L.n_row_tiles;
    const int per = ceil_div(U, nsm);
    const int G = ceil_div(U, per);
    if (P > 1 && per > L.n_row_tiles) continue;   // a CTA's units then span at most two panels
    const int nbuf = P == 1 ? 1 : 2;
    const int nst_max = std::max(1, std::min(kMaxStagesS, per * ceil_div(KP, MW)));
    // Adapter K splits: enough items for the grid, few enough that every
    // CTA reads at most 16 tagged partial words per thread (see the kernel).
    const int SA = JT > 0 ? std::max(1, std::min({G / JT, L.K / 16, std::max(1, 64 / xrows)})) : 1;
    const int nls_max = JT > 0 ? std::min(kMaxAdStages, ceil_div(ceil_div(L.K / 16, SA), kAdStageSteps)) : 0;
    const int rs_fit = (JT > 0 && (size_t)per * (L.r16 / 16) * 512 <= kRsBudget) ? 1 : 0;
    for (int rs_smem = rs_fit; rs_smem >= 0; --rs_smem) {
      for (int nst = nst_max; nst >= std::min(nst_max, 3); --nst) {
        for (int nls = nls_max; nls >= std::min(nls_max, 2); nls = (nls > 2 ? nls / 2 : nls - 1)) {
          const size_t smem = stream_smem(NT, MW, xrows, KP, nbuf, nst, per, L.r16, L.rl16, rs_smem, nls).total;
          if (smem > kSmemLimit) continue;
          // At most one CTA per SM and one CTA's worth of shared memory: the
          // whole grid fits on the device at once.
          pl.ok = true;
          pl.NT = NT;
          pl.MW = MW;
          pl.P = P;
          pl.KP = KP;
          pl.U = U;
          pl.G = G;
          pl.units_max = per;
          pl.nst = nst;
          pl.nbuf = nbuf;
          pl.SA = SA;
          pl.rs_smem = rs_smem;
          pl.nls = nls;
          pl.ad_prefetched = JT == 0 || nls * kAdStageSteps >= ceil_div(L.K / 16, SA);
          pl.smem = smem;
          return pl;
        }
      }
    }
  }
  return pl;
}

template <int NT, int MW>
cudaError_t set_smem(size_t smem) {
  return ensure_func_attrs(reinterpret_cast<const void*>(k_stream<NT, MW>), smem);
}

template <int NT, int MW>
cudaError_t run(cudaLaunchConfig_t& cfg, size_t smem, const StreamParams& p) {
  cudaError_t e = set_smem<NT, MW>(smem);
  if (e != cudaSuccess) return e;
  return cudaLaunchKernelEx(&cfg, k_stream<NT, MW>, p);
}

size_t a256(size_t x) { return (x + 255) / 256 * 256; }

struct StreamWs {
  size_t ctl, part_ll, part_main, total;
};

StreamWs stream_ws(const slim_layer& L, const StreamPlan& pl) {
  StreamWs w;
  const int JT = L.rl16 / 16;
  const bool need_ctl = JT > 0 || pl.P > 1;
  size_t off = 0;
  w.ctl = off;       off += need_ctl ? a256((size_t)4 * kCtlRtWord + (pl.P > 1 ? (size_t)8 * L.n_row_tiles : 0)) : 0;
  w.part_ll = off;   off += JT > 0 ? a256((size_t)JT * pl.SA * 256 * 8) : 0;
  w.part_main = off; off += pl.P > 1 ? a256((size_t)L.n_row_tiles * pl.P * 256 * 4) : 0;
  w.total = off;
  return w;
}

}  // namespace

size_t stream_workspace_bytes(const slim_layer& L, int M) {
  const StreamPlan pl = plan_stream(L, M);
  return pl.ok ? stream_ws(L, pl).total : 0;
}

bool stream_supported(const slim_layer& L, int M) { return plan_stream(L, M).ok; }

cudaError_t launch_stream(const slim_layer& L, const uint16_t* X, int M, uint16_t* Y, void* ws, cudaStream_t s) {
  return launch_stream_ex(L, X, M, Y, ws, kWaitBudgetCycles, 0u, s);
}

cudaError_t launch_stream_ex(const slim_layer& L, const uint16_t* X, int M, uint16_t* Y, void* ws,
                             long long t_wait_cycles, uint32_t tag_skew, cudaStream_t s) {
  const StreamPlan pl = plan_stream(L, M);
  if (!pl.ok) return cudaErrorNotSupported;
  const StreamWs w = stream_ws(L, pl);
  uint8_t* wb = static_cast<uint8_t*>(ws);
  StreamParams p;
  p.X = X;
  p.Y = Y;
  p.dec = L.dec;
  p.Rf = reinterpret_cast<const uint4*>(L.Rf);
  p.Lf = reinterpret_cast<const uint4*>(L.Lf);
  p.part_ll = L.r16 > 0 ? reinterpret_cast<unsigned long long*>(wb + w.part_ll) : nullptr;
  p.part_main = pl.P > 1 ? reinterpret_cast<float*>(wb + w.part_main) : nullptr;
  p.ctl = (L.r16 > 0 || pl.P > 1) ? reinterpret_cast<uint32_t*>(wb + w.ctl) : nullptr;
  p.M = M;
  p.K = L.K;
  p.N = L.N;
  p.NRT = L.n_row_tiles;
  p.NKB = L.n_kblocks;
  p.r16 = L.r16;
  p.rl16 = L.rl16;
  p.n_groups = L.n_groups;
  for (int g = 0; g < SLIM_MAX_GROUPS; ++g) p.group_end_rt[g] = ceil_div(L.group_end[g], 16);
  p.P = pl.P;
  p.KP = pl.KP;
  p.U = pl.U;
  p.SA = pl.SA;
  p.nst = pl.nst;
  p.nbuf = pl.nbuf;
  p.units_max = pl.units_max;
  p.rs_smem = pl.rs_smem;
  p.nls = pl.nls;
  p.early = tuning().pdl_early ? 1 : 0;
  p.status = L.status;
  p.t_wait = t_wait_cycles;
  p.tag_skew = tag_skew;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.G);
  cfg.blockDim = dim3((pl.MW + 1) * 32);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return pl.MW == 8 ? (pl.NT == 1 ? run<1, 8>(cfg, pl.smem, p) : run<2, 8>(cfg, pl.smem, p))
                    : (pl.NT == 1 ? run<1, 16>(cfg, pl.smem, p) : run<2, 16>(cfg, pl.smem, p));
}

}  // namespace slim

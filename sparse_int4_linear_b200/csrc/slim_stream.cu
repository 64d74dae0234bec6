// Single-launch decode forward for M <= 16 tokens (sm_100a).
//
// Decoding is memory-bound: every packed weight byte is used for one small
// matrix product (thesis §2.5.2 "The Memory-Bound Regime: Inference
// Decoding").  The layer is therefore streamed once, with the copy engines
// kept busy from the first to the last byte, and everything else of the call
// - the adapter's X L, its (X L) R, the sums across K - is folded into the
// same launch so that a chain of calls pays one grid hand-off per call.
//
// Work split (stream-K).  The packed layer is a grid of 1600-byte chunks
// (16-row tile rt x 256-K block kb).  K is cut into P panels, as few as let
// the panel of X (the tokens x the panel's K) sit in shared memory: P = 1
// whenever the whole X fits.  Panel p gets a share of the CTAs (at most one
// per SM) in proportion to its chunks; inside a panel the chunks are ordered
// row tile by row tile, K block by K block, and every main warp of those
// CTAs takes one contiguous, balanced range of them.  A warp streams its
// range through its own ring of bulk copies and keeps the 16 x tokens
// partial of the current row tile in registers; when its range leaves a row
// tile it writes that partial (a "segment") to the workspace.  There is no
// barrier and no cross-warp reduction in the streaming loop.  The sparse
// int4 product uses mma.sp m16n8k32 (§2.2.3 "Sparse Tensor Core
// Acceleration"): the 2-bit metadata selects the matching activations on
// the tensor cores.
//
// A row tile is finished by the warp holding its first chunk (in panel
// rt % P): where that warp's range ends inside the tile, the rest of the
// tile belongs to the next warp, which wrote its segment at the start of its
// stream, so the finisher (the last writer in time) rarely waits.  Segments
// are written as 64-bit words that carry the fp32 value and the launch's
// tag, like the adapter partials below: the finisher reads every segment of
// its tile, waiting (bounded) on each word until it carries the current tag,
// adds them in slot order, adds R^T T^T (the adapter) and stores bf16 Y (in
// 8-warp CTAs and with two token tiles it sums its first tile's segments and
// copies that tile's R^T into its idle ring before it waits for T).  No
// atomics on the data path, no barrier between the main warps; every sum has
// a fixed order, so results do not depend on timing.
//
// The adapter (§4, lazy low-rank adapters: never merged into the sparse
// weight) runs on NA = 1 or 2 more warps per CTA (2 when L and R are a large
// share of the layer's bytes).  Each panel's K range is cut into SAp slices
// and the JT*SAp items (jt, slice) of a panel go to the adapter warps of
// that panel's CTAs, so an item reads X from the CTA's staged panel: the item computes
// the partial T[:, 16 jt .. 16 jt + 15] = X L over its slice and writes it
// to the workspace as 64-bit words that carry the fp32 value and the
// launch's tag (see the control block below), so a reader needs no flag: a
// word with the current tag is the current value.  The first panel-0 items
// of column tile jt (one per 32 elements of the tile) then add its SA = P *
// SAp partials in slice order and publish T[:, jt] the same way.  Each CTA's
// main warps gather T into shared memory (bf16) cooperatively as their
// streams end.
//
// Control block (start of the workspace, zero before first use): [0]
// sequence number, [1] finished CTAs (rewound to zero by the launch that
// raised it).  The last CTA to finish advances the sequence number.  Every word
// this kernel relies on carries the launch's tag (launch_tag(): a bit range
// that no finite data written by any kernel of the library can produce), so
// whatever another layer or another path left in the workspace is never
// mistaken for a value of this launch; only words [0] and [1] must be left
// alone by the other paths, which start their data 256 bytes in.
//
// Failure: if a bounded wait of a CTA gives up, the CTA records
// SLIM_ERR_TIMEOUT, lets its copies in flight land, and stores zeros for the
// tiles it finishes; a warp whose stream gave up writes its segments with a
// signalling-NaN payload (kPoison, which no arithmetic produces), and a
// tile with such a segment is stored as zeros too.
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

constexpr int kMaxStagesS = 8;
constexpr int kMaxTCols = 1024;            // adapter columns of T over all fused linears
constexpr int kMaxLLLoads = 12;            // tagged partial words in flight per thread
constexpr int kGatherLoads = 4;            // T words per lane of one unit of the cooperative T gather
constexpr size_t kSmemLimit = 220 * 1024;
constexpr size_t kSmemPair = 110 * 1024;   // two CTAs per SM fit: the next launch starts beside this one
constexpr int kAdStageSteps = 8;           // K/16 steps per adapter ring stage (4 KB of bf16 L^T)
constexpr int kAdQBlocks = 4;              // 128-K blocks per adapter ring stage with 4-bit L^T (4.1 KB)
constexpr int kMaxAdStages = 8;
constexpr int kMaxPanels = 32;
constexpr uint32_t kPoison = 0x7FA00000u;   // segment value of a warp whose stream gave up (a signalling NaN)
// Ring stages a main warp fills before the grid-dependency wait.  More would
// put so many bytes in flight that the X panel, loaded right after the wait,
// queues behind them; the rest of the ring is filled once X is staged.
constexpr int kPreStages = 2;
constexpr int kRuBytes = 16 * 16 * 4;           // a finisher's segment sums (16 tokens x 16 rows, fp32) at the ring's start

struct StreamParams {
  const uint16_t* X;
  uint16_t* Y;
  const uint8_t* dec;
  const uint4* Rf;
  const uint4* Lf;
  const uint8_t* Rq;             // 4-bit adapter layouts (used when aq)
  const uint8_t* Lq;
  int aq;                        // 1: the adapter factors are 4-bit (Lq, Rq), else bf16 (Lf, Rf); the kernel's AQ
  int rqt, ngr;                  // bytes of one Rq row tile; 128-groups of r
  unsigned long long* part_ll;   // [JT][SA][256] tagged X L partials: fp32 bits | launch_tag(seq) << 32
  unsigned long long* t_fin;     // [JT][256] tagged T = X L (the partials added; part_ll itself when SA == 1)
  unsigned long long* part;      // [NRT][segmax][xrows * 16] tagged segment partials: fp32 bits | tag << 32
  uint32_t* ctl;                 // [0] sequence number, [1] finished CTAs
  int M, K, N, NRT, NKB;
  int r16;              // adapter rank of each fused linear, rounded up to 16 (R^T tiles)
  int rl16;             // adapter columns of T = X L over all fused linears
  int n_groups;
  int group_end_rt[SLIM_MAX_GROUPS];   // row tiles of fused linear g end at group_end_rt[g]
  int P, KP;            // K panels, K blocks per panel (the last panel may have fewer)
  int segmax;           // segment slots per row tile
  int SA, SAp;          // adapter K slices in all, per panel (SA = P * SAp)
  int nst;              // ring stages per main warp
  int nls;              // adapter ring stages
  int early;            // signal the next launch before the wait (not only after the stream)
  int cta0[kMaxPanels + 1];   // panel p is served by CTAs [cta0[p], cta0[p + 1])
  int32_t* status;
  long long t_wait;     // budget (SM cycles) of each wait for a T partial
  uint32_t tag_skew;    // 0; test aid: readers of T partials expect launch_tag(seq + tag_skew)
};

// The chunks of panel pn: every row tile, K blocks [pn * KP, pn * KP + kp).
struct PanelShape {
  int kb0, kp;          // first K block, K blocks
  long long C;          // chunks
  int W;                // warps with work (each has at least one chunk)
};

__host__ __device__ inline PanelShape panel_shape(int NRT, int NKB, int KP, int MW, const int* cta0, int pn) {
  PanelShape s;
  s.kb0 = pn * KP;
  s.kp = min(KP, NKB - s.kb0);
  s.C = (long long)NRT * s.kp;
  const long long w = (long long)(cta0[pn + 1] - cta0[pn]) * MW;
  s.W = (int)(w < s.C ? w : s.C);
  return s;
}
// Warp lw's chunk range of a panel starts at chunk_start(lw).
__host__ __device__ inline long long chunk_start(const PanelShape& s, int lw) { return (long long)lw * s.C / s.W; }
// The warp whose range holds chunk f.
__host__ __device__ inline int warp_of(const PanelShape& s, long long f) {
  return (int)(((f + 1) * s.W - 1) / s.C);
}
// Slot (ordinal) of warp lw's segment of row tile rt of panel pn among all
// segments of the tile (panels in order, warps in order), and their count.
__host__ __device__ inline int2 segment_slot(int NRT, int NKB, int KP, int MW, int P, const int* cta0, int rt,
                                             int pn, int lw) {
  int before = 0, total = 0;
  for (int q = 0; q < P; ++q) {
    const PanelShape s = panel_shape(NRT, NKB, KP, MW, cta0, q);
    const int lo = warp_of(s, (long long)rt * s.kp), hi = warp_of(s, (long long)rt * s.kp + s.kp - 1);
    if (q < pn) before += hi - lo + 1;
    if (q == pn) before += lw - lo;
    total += hi - lo + 1;
  }
  return make_int2(before, total);
}

struct StreamSmem {
  size_t xs, ring, ts, ls, bars, total;
};

__host__ __device__ inline size_t a16(size_t x) { return (x + 15) / 16 * 16; }

// Bytes of one row tile's R^T (bf16 fragments, or 4-bit ones with scales)
// and of one adapter ring stage.
__host__ __device__ inline int r_tile_bytes(int aq, int r16, int rqt) { return aq ? rqt : r16 / 16 * 512; }
__host__ __device__ inline int ad_stage_bytes(int aq) { return aq ? kAdQBlocks * kLqBlock : kAdStageSteps * 512; }

// Shared memory: the staged X panel, the main warps' chunk rings, T, the
// adapter warps' rings, mbarriers and a few words (the sequence number, the
// T gather's counters, each main warp's give-up point).
__host__ __device__ inline StreamSmem stream_smem(int MW, int NA, int xrows, int KP, int nst, int rl16, int nls,
                                                  int ls_stage) {
  StreamSmem m;
  size_t off = 0;
  m.xs = off;   off = a16(off + (size_t)xrows * (KP * 256 + 8) * 2);
  m.ring = off; off = a16(off + (size_t)MW * nst * kDecChunk);
  m.ts = off;   off = a16(off + (rl16 > 0 ? (size_t)16 * (rl16 + 8) * 2 : 0));
  m.ls = off;   off = a16(off + (size_t)NA * nls * ls_stage);
  m.bars = off; off += (size_t)(MW * nst + NA * nls + 1) * 8 + 16 + 4 * MW;
  m.total = off;
  return m;
}

// Barrier of the main warps and the adapter warps (every thread of the CTA).
template <int TW>
__device__ __forceinline__ void bar_all() {
  asm volatile("bar.sync 2, %0;" ::"n"(TW * 32) : "memory");
}
__device__ __forceinline__ void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }
// 16-byte asynchronous global -> shared copies (completion by wait_all).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// X fragments of MMA step j (0..7) of a K block: 64 bytes apart; j is a
// constant once the callers' loops are unrolled, so the switch folds away.
__device__ __forceinline__ void ldmatrix_x4_step(uint32_t (&b)[4], uint32_t a, int j) {
  switch (j) {
    case 0: ldmatrix_x4_so<0>(b, a); break;
    case 1: ldmatrix_x4_so<64>(b, a); break;
    case 2: ldmatrix_x4_so<128>(b, a); break;
    case 3: ldmatrix_x4_so<192>(b, a); break;
    case 4: ldmatrix_x4_so<256>(b, a); break;
    case 5: ldmatrix_x4_so<320>(b, a); break;
    case 6: ldmatrix_x4_so<384>(b, a); break;
    default: ldmatrix_x4_so<448>(b, a); break;
  }
}

// Out of line: the slot search runs once per row tile a warp leaves.
__device__ __noinline__ int2 slot_of(const StreamParams* p, int MW, int rt, int pn, int lw) {
  return segment_slot(p->NRT, p->NKB, p->KP, MW, p->P, p->cta0, rt, pn, lw);
}

// MW main warps + NA adapter warps = 8 or 16 warps, a multiple of the four
// warp schedulers, so the register file splits evenly (up to 128 registers
// a thread; with 17 warps the limit drops to 96).
template <int NT, int MW, int NA, bool AQ>
__global__ void __launch_bounds__((MW + NA) * 32, MW + NA == 8 ? 2 : 1)
    k_stream(const __grid_constant__ StreamParams p) {
  constexpr int kMainWarps = MW;
  constexpr int TW = MW + NA;
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int G = gridDim.x, cta = blockIdx.x;
  const int xrows = min(p.M, NT * 8);
  const int last = xrows - 1;
  const int E = xrows * 16;        // outputs of one row tile
  const int JT = p.rl16 / 16;      // T column tiles (all fused linears)
  const int JS = p.r16 / 16;       // R^T tiles of one row tile
  const int nst = p.nst;
  const int xrow = p.KP * 256 + 8;
  const int trow = p.rl16 + 8;
  int pn = 0;
  while (pn + 1 < p.P && cta >= p.cta0[pn + 1]) ++pn;
  const PanelShape ps = panel_shape(p.NRT, p.NKB, p.KP, MW, p.cta0, pn);

  // R^T of one row tile (bf16 or 4-bit fragments): its bytes and the
  // global address of row tile rt's (recomputed where used: fewer live
  // registers across the stream).
  auto rtile = [&]() { return r_tile_bytes(AQ, p.r16, p.rqt); };
  auto rtile_src = [&](int rt) {
    return (AQ ? p.Rq : reinterpret_cast<const uint8_t*>(p.Rf)) + (size_t)rt * rtile();
  };
  const int ls_stage = ad_stage_bytes(AQ);
  const StreamSmem L = stream_smem(MW, NA, xrows, p.KP, nst, p.rl16, p.nls, ls_stage);
  uint16_t* Xs = reinterpret_cast<uint16_t*>(smem + L.xs);
  uint8_t* ring = smem + L.ring;
  uint16_t* Ts = reinterpret_cast<uint16_t*>(smem + L.ts);
  uint8_t* Ls_all = smem + L.ls;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* lbar_all = bars + kMainWarps * nst;  // [NA][nls] adapter rings
  uint64_t* xbar = lbar_all + NA * p.nls;        // X staged
  volatile uint32_t* sh = reinterpret_cast<volatile uint32_t*>(xbar + 1);   // [0] seq
  int* tctl = const_cast<int*>(reinterpret_cast<volatile int*>(sh + 1));  // T gather: [0] next unit, [1] units done, [2] a word gave up
  int* fail_at = const_cast<int*>(reinterpret_cast<volatile int*>(sh + 4));   // [main warp] (after a give-up)

  if (threadIdx.x == 0) {
    for (int i = 0; i < kMainWarps * nst + NA * p.nls; ++i) mbar_init(bars + i, 1);
    mbar_init(xbar, 1);
    tctl[0] = tctl[1] = tctl[2] = 0;
    fence_mbar_init();
  }
  // T = X L into Ts (bf16, [token][column]), gathered cooperatively: units
  // of 32 x kGatherLoads elements of the reduced, tagged T words, handed out
  // by tctl[0] to the main warps as their streams end (busy-polling warps
  // would take issue slots from the warps still streaming, so the adapter
  // warps, done early, do not take part); tctl[1] counts the units written,
  // tctl[2] is set when a word never got this launch's tag (the finishers
  // then store zeros).
  const int n_el = JT * E;
  const int n_units = ceil_div(n_el, 32 * kGatherLoads);
  auto gather_t = [&](uint32_t ttag) {
    for (;;) {
      int u = 0;
      if (lane == 0) u = atomicAdd(tctl, 1);
      u = __shfl_sync(0xffffffffu, u, 0);
      if (u >= n_units) break;
      const int base = u * 32 * kGatherLoads;
      unsigned long long v[kGatherLoads];
#pragma unroll
      for (int i = 0; i < kGatherLoads; ++i) {
        const int o = base + i * 32 + lane;
        v[i] = o < n_el && dcheck(o / E < JT, p.status) ? ld_relaxed_u64(p.t_fin + (size_t)(o / E) * 256 + o % E)
                                                         : 0ull;
      }
      // Words not yet current are polled again together (one round trip a
      // poll), within the wait budget.
      bool gok = true;
      const long long c0 = clock64();
      for (;;) {
        bool stale = false;
#pragma unroll
        for (int i = 0; i < kGatherLoads; ++i)
          stale = stale || (base + i * 32 + lane < n_el && (uint32_t)(v[i] >> 32) != ttag);
        if (!stale) break;
        if (clock64() - c0 > p.t_wait) {
          gok = false;
          break;
        }
#pragma unroll
        for (int i = 0; i < kGatherLoads; ++i) {
          const int o = base + i * 32 + lane;
          if (o < n_el && (uint32_t)(v[i] >> 32) != ttag) v[i] = ld_relaxed_u64(p.t_fin + (size_t)(o / E) * 256 + o % E);
        }
      }
#pragma unroll
      for (int i = 0; i < kGatherLoads; ++i) {
        const int o = base + i * 32 + lane;
        if (o < n_el) {
          const int jt = o / E, e = o - jt * E;
          Ts[(e >> 4) * trow + jt * 16 + (e & 15)] =
              __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float((uint32_t)v[i])));
        }
      }
      gok = __all_sync(0xffffffffu, gok);
      if (lane == 0) {
        if (!gok) {
          tctl[2] = 1;
          record_status(p.status, SLIM_ERR_TIMEOUT);
        }
        __threadfence_block();
        atomicAdd(tctl + 1, 1);
      }
      __syncwarp();
    }
  };
  // Wait (bounded) until every unit of T is in Ts; false if T is not usable.
  auto wait_t = [&]() -> bool {
    int done = 1;
    if (lane == 0) {
      const long long c0 = clock64();
      while (*reinterpret_cast<volatile int*>(tctl + 1) < n_units) {
        if (clock64() - c0 > kWaitBudgetCycles) {
          done = 0;
          record_status(p.status, SLIM_ERR_TIMEOUT);
          break;
        }
      }
      __threadfence_block();
    }
    done = __shfl_sync(0xffffffffu, done, 0);
    __syncwarp();
    return done != 0 && *reinterpret_cast<volatile int*>(tctl + 2) == 0;
  };
  // Zero the staged-X columns past K (the padded tail of the last K block).
  {
    const int ncols = min(ps.kp * 256, p.K - ps.kb0 * 256);
    const int pad = ps.kp * 256 - ncols;
    for (int i = threadIdx.x; i < xrows * pad; i += blockDim.x) Xs[(i / pad) * xrow + ncols + i % pad] = 0;
  }
  __syncthreads();

  if (warp < kMainWarps) {
    // ------------------------------------------------------------ main warps
    const int lw = (cta - p.cta0[pn]) * kMainWarps + warp;   // warp index within the panel
    const bool has_work = lw < ps.W;
    const long long f0 = has_work ? chunk_start(ps, lw) : 0, f1 = has_work ? chunk_start(ps, lw + 1) : 0;
    const int rt_a = has_work ? (int)(f0 / ps.kp) : 0;
    const int kb_a = has_work ? (int)(f0 - (long long)rt_a * ps.kp) : 0;   // first K block of the first tile
    uint8_t* wring = ring + (size_t)warp * nst * kDecChunk;
    uint64_t* wbar = bars + warp * nst;
    // Producer cursor: next chunk to copy, as (row tile, K block in panel).
    const int nch = (int)(f1 - f0);   // chunks of this warp's range
    int ni = 0;                        // chunks issued
    int rt_i = rt_a, kb_i = kb_a;
    const uint8_t* src_i = p.dec + ((size_t)rt_a * p.NKB + ps.kb0 + kb_a) * kDecChunk;
    const size_t tile_step = (size_t)(p.NKB - ps.kp + 1) * kDecChunk;   // from a tile's last chunk to the next tile's first
    auto issue = [&](int s) {
      if (!dcheck(rt_i < p.NRT && ps.kb0 + kb_i < p.NKB, p.status)) return;
      mbar_expect_tx(wbar + s, kDecChunk);
      bulk_g2s(wring + s * kDecChunk, src_i, kDecChunk, wbar + s);
    };
    auto advance_i = [&]() {
      ++ni;
      if (++kb_i == ps.kp) {
        kb_i = 0;
        ++rt_i;
        src_i += tile_step;
      } else {
        src_i += kDecChunk;
      }
    };
    // The packed layer is constant: start streaming it before the wait.
    const int npre = min(nst, kPreStages);
    for (int s = 0; s < npre && ni < nch; ++s) {
      if (lane == 0) issue(s);
      advance_i();
    }
    // Row tiles this warp finishes: those of panel rt % P (panel 0 with one
    // panel) whose first chunk in that panel lies in this warp's range,
    // rt_f .. rt_z (every other panel rt % P).  That warp writes its segment
    // of the tile last in time: where its range ends inside the tile, the
    // next warp (holding the rest of the tile) wrote its segment at the start
    // of its stream; so the finisher rarely waits.  The R^T of these tiles is
    // warmed in L2 when the stream is a ring's depth from its end (before the
    // wait for a short stream): early enough to be on chip for the finishing,
    // late enough to stay out of the way of X and the first chunks.
    const int rt_z = has_work ? (int)((f1 - 1) / ps.kp) : -1;
    const int rt_f = has_work ? rt_a + (kb_a != 0 ? 1 : 0) : 0;
    auto finishes = [&](int rt) { return p.P == 1 || rt % p.P == pn; };
    auto warm_rt = [&]() {
      if (JT == 0) return;
      for (int rt = rt_f; rt <= rt_z; ++rt)
        if (finishes(rt))
          for (int o = lane * 128; o < rtile(); o += 32 * 128) prefetch_l2(rtile_src(rt) + o);
    };
    const bool warm_early = nch <= nst;
    const int n_warm = nch - nst;   // chunks consumed when the R^T is warmed
    if (warm_early) warm_rt();
    // One thread waits for the previous grid and issues the X panel at once
    // (one bulk copy per token row, completing on xbar), ahead of the rest of
    // the ring; the others block on the barrier, where they take no issue
    // slots from the grid still running on this SM.
    if (p.early) pdl_launch_dependents();
    if (threadIdx.x == 0) {
      pdl_wait();
      if (dcheck(xrows <= p.M && ps.kb0 < p.NKB, p.status)) {
        const uint32_t row_bytes = (uint32_t)min(ps.kp * 256, p.K - ps.kb0 * 256) * 2u;
        mbar_expect_tx(xbar, row_bytes * (uint32_t)xrows);
        for (int tk = 0; tk < xrows; ++tk)
          bulk_g2s(Xs + tk * xrow, p.X + (size_t)tk * p.K + ps.kb0 * 256, row_bytes, xbar);
      }
      sh[0] = *reinterpret_cast<volatile uint32_t*>(p.ctl);
    }
    bar_all<TW>();
    // The rest of the ring.
    for (int s = npre; s < nst && ni < nch; ++s) {
      if (lane == 0) issue(s);
      advance_i();
    }
    const bool x_ok = mbar_wait(xbar, 0);
    asm volatile("bar.sync 1, %0;" ::"n"(MW * 32) : "memory");
    const uint32_t seq = sh[0];
    const uint32_t tag = launch_tag(seq);

    bool ok = __all_sync(0xffffffffu, x_ok);
    if (!ok && lane == 0) fail_at[warp] = 0;
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
    int st = 0;
    uint32_t ph = 0;
    const uint32_t ring_s = smem_u32(wring), bar_s = smem_u32(wbar);
    const uint32_t xs_s = smem_u32(Xs);
    // ldmatrix rows are tokens; rows past the staged ones repeat the last
    // staged row (their products land in outputs that are not stored).
    const uint32_t xk0 = xs_s + (uint32_t)(min(lane & 7, last) * xrow + (lane >> 3) * 8) * 2u;
    const uint32_t xk1 = xs_s + (uint32_t)(min(8 + (lane & 7), last) * xrow + (lane >> 3) * 8) * 2u;
    const uint32_t ring_l = ring_s + lane * 16, ring_g = ring_s + 1536 + 8 * g;   // this lane's words of stage 0
    int rt_c = rt_a, kb_c = kb_a;
    uint32_t kofs = (uint32_t)kb_a * 512u;   // X column offset of the chunk's K block (256 bf16 per block)
    for (int n = 0; n < nch; ++n) {
      if (!warm_early && n == n_warm) warm_rt();
      if (ok) {
        ok = __all_sync(0xffffffffu, mbar_wait_s(bar_s + st * 8, ph));
        if (!ok && lane == 0) fail_at[warp] = n;   // first chunk not consumed
      }
      if (ok) {
        const uint32_t so = (uint32_t)st * kDecChunk;
        const uint4 v0 = lds128_so<0>(ring_l + so);
        const uint4 v1 = lds128_so<512>(ring_l + so);
        const uint4 ev = lds128_so<1024>(ring_l + so);
        // fp16 scales (non-negative) of rows g and g+8 for the chunk's two 128-groups
        uint32_t sw0, sw1;
        lds64_so<0>(ring_g + so, sw0, sw1);
        const float sg[2][2] = {{f16_nonneg_bits_to_f32(sw0 & 0xFFFFu), f16_nonneg_bits_to_f32(sw0 >> 16)},
                                {f16_nonneg_bits_to_f32(sw1 & 0xFFFFu), f16_nonneg_bits_to_f32(sw1 >> 16)}};
        const uint32_t vw[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        const uint32_t ew[4] = {ev.x, ev.y, ev.z, ev.w};
        const uint32_t xa0 = xk0 + kofs, xa1 = xk1 + kofs;
        // One tensor-core chain per scale group; the two groups are
        // independent, so their MMAs interleave.
        float part[2][NT][4];
#pragma unroll
        for (int grp = 0; grp < 2; ++grp)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            part[grp][nt][0] = part[grp][nt][1] = part[grp][nt][2] = part[grp][nt][3] = 0.f;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
#pragma unroll
          for (int grp = 0; grp < 2; ++grp) {
            const int j = grp * 4 + jj;
            uint32_t a[4];
            decode_word(vw[j], a);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              uint32_t b[4];
              ldmatrix_x4_step(b, nt == 0 ? xa0 : xa1, j);
              if (j & 1) mma_sp_16832<1>(part[grp][nt], a, b, ew[j >> 1]);
              else       mma_sp_16832<0>(part[grp][nt], a, b, ew[j >> 1]);
            }
          }
        }
#pragma unroll
        for (int grp = 0; grp < 2; ++grp)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            acc[nt][0] = fmaf(sg[grp][0], part[grp][nt][0], acc[nt][0]);
            acc[nt][1] = fmaf(sg[grp][0], part[grp][nt][1], acc[nt][1]);
            acc[nt][2] = fmaf(sg[grp][1], part[grp][nt][2], acc[nt][2]);
            acc[nt][3] = fmaf(sg[grp][1], part[grp][nt][3], acc[nt][3]);
          }
      }
      __syncwarp();
      if (ok && ni < nch) {
        if (lane == 0) {
          fence_proxy_async_smem();
          issue(st);
        }
        advance_i();
      }
      if (++st == nst) {
        st = 0;
        ph ^= 1u;
      }
      // Leaving a row tile (or the range): its partial is one segment, kept
      // in the workspace at its slot among the tile's segments.
      if (kb_c + 1 == ps.kp || n + 1 == nch) {
        const bool whole = p.P == 1 && kb_c + 1 == ps.kp && (rt_c != rt_a || kb_a == 0);
        const int slot = whole ? 0 : slot_of(&p, MW, rt_c, pn, lw).x;
        unsigned long long* dst = p.part + ((size_t)rt_c * p.segmax + slot) * E;
        const unsigned long long tg = (unsigned long long)tag << 32;
        const bool in_ws = dcheck(rt_c < p.NRT && slot < p.segmax, p.status);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int tk = nt * 8 + 2 * t;
          if (!ok) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = __uint_as_float(kPoison);
          if (in_ws && tk < xrows) {
            st_relaxed_u64(dst + tk * 16 + g, tg | __float_as_uint(acc[nt][0]));
            st_relaxed_u64(dst + tk * 16 + g + 8, tg | __float_as_uint(acc[nt][2]));
          }
          if (in_ws && tk + 1 < xrows) {
            st_relaxed_u64(dst + (tk + 1) * 16 + g, tg | __float_as_uint(acc[nt][1]));
            st_relaxed_u64(dst + (tk + 1) * 16 + g + 8, tg | __float_as_uint(acc[nt][3]));
          }
          acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
        }
      }
      if (++kb_c == ps.kp) {
        kb_c = 0;
        kofs = 0;
        ++rt_c;
      } else {
        kofs += 512u;
      }
    }
    if (!ok && lane == 0) {
      record_status(p.status, SLIM_ERR_TIMEOUT);
      // Let the copies issued and not consumed land before the CTA exits.
      const long long deadline = clock64() + kWaitBudgetCycles;
      for (int i = fail_at[warp]; i < ni; ++i) drain_phase(wbar + i % nst, (i / nst) & 1, deadline);
    }
    __syncwarp();   // the ring is idle from here on (ru, R^T fragments)
    // T = X L in shared memory (bf16), gathered cooperatively by the main
    // warps as their streams end (gather_t); then this warp finishes its row
    // tiles: every segment of the tile (slot order, each word waited for,
    // bounded, until it carries this launch's tag), plus T R^T, stored as
    // bf16.  A tile with a segment of a stream that gave up, a segment that
    // never arrived or a T that could not be gathered is stored as zeros.
    //
    // Sum of a tile's segments in slot order, element e = lane + 32 k per
    // lane (into ru, this warp's idle ring); words (k, segment) in flight
    // together, the ones not yet current polled again together.  False when
    // the tile is skipped (a slot count out of bounds, debug builds only).
    float* ru = reinterpret_cast<float*>(wring);
    auto sum_segments = [&](int rt, bool& seg_ok, bool& poisoned) -> bool {
      const int nseg = slot_of(&p, MW, rt, 0, 0).y;
      if (!dcheck(nseg <= p.segmax, p.status)) return false;
      const unsigned long long* src = p.part + (size_t)rt * p.segmax * E;
      seg_ok = true;
      poisoned = false;
      const int nw = (lane < E ? (E - lane + 31) / 32 : 0) * nseg;
      int ke = lane, kq = 0;   // element and segment of the next word to load
      int se = lane, sq = 0;   // ... and of the next word to add
      float run = 0.f;
      for (int w0 = 0; w0 < nw; w0 += kMaxLLLoads) {
        unsigned long long v[kMaxLLLoads];
#pragma unroll
        for (int i2 = 0; i2 < kMaxLLLoads; ++i2) {
          if (w0 + i2 < nw) {
            v[i2] = ld_relaxed_u64(src + kq * E + ke);
            if (++kq == nseg) {
              kq = 0;
              ke += 32;
            }
          }
        }
        const long long c0 = clock64();
        while (seg_ok) {
          bool stale = false;
#pragma unroll
          for (int i2 = 0; i2 < kMaxLLLoads; ++i2)
            stale = stale || (w0 + i2 < nw && (uint32_t)(v[i2] >> 32) != tag);
          if (!stale) break;
          if (clock64() - c0 > kWaitBudgetCycles) {
            seg_ok = false;
            break;
          }
#pragma unroll
          for (int i2 = 0; i2 < kMaxLLLoads; ++i2) {
            const int w = w0 + i2;   // word w: segment w % nseg of element lane + 32 (w / nseg)
            if (w < nw && (uint32_t)(v[i2] >> 32) != tag)
              v[i2] = ld_relaxed_u64(src + (w % nseg) * E + lane + 32 * (w / nseg));
          }
        }
#pragma unroll
        for (int i2 = 0; i2 < kMaxLLLoads; ++i2) {
          if (w0 + i2 < nw) {
            poisoned = poisoned || (uint32_t)v[i2] == kPoison;
            run += __uint_as_float((uint32_t)v[i2]);
            if (++sq == nseg) {
              ru[se] = run;
              run = 0.f;
              sq = 0;
              se += 32;
            }
          }
        }
      }
      seg_ok = __all_sync(0xffffffffu, seg_ok);
      poisoned = __any_sync(0xffffffffu, poisoned);
      if (!seg_ok && lane == 0) record_status(p.status, SLIM_ERR_TIMEOUT);
      return true;
    };
    // With two token tiles, or in 8-warp CTAs, the first tile this warp
    // finishes has its segments summed, and (bf16 R^T) its R^T fragments
    // copied into this warp's idle ring behind ru, before T is waited for:
    // its segments are in place by the end of this warp's stream as a rule
    // and its R^T is warm in L2, so once T is in shared memory only T R^T and
    // the store are left.  (Measured on the 70B shapes: 70B down at 16 tokens
    // 64.9 -> 60.6 us, k at one token 14.3 -> 13.2 us; in 16-warp CTAs at one
    // token, where T is ready before the streams end, 70B gate took 1.8 us
    // longer, so there the T gather still comes first.)
    constexpr bool kPresum = NT == 2 || TW == 8;
    int rt_pre = -1;
    for (int rt = rt_f; kPresum && JT > 0 && rt <= rt_z; ++rt)
      if (finishes(rt)) {
        rt_pre = rt;
        break;
      }
    const uint32_t rfs = ring_s + kRuBytes + lane * 16;   // this lane's fragment of step 0
    int pre_js = 0;                                        // column steps copied
    bool pre_valid = false, pre_ok = true, pre_pois = false;
    if (rt_pre >= 0 && dcheck(rt_pre < p.NRT, p.status)) {
      if (!AQ) {
        pre_js = min(JS, (nst * kDecChunk - kRuBytes) / 512);
        const uint8_t* rf = rtile_src(rt_pre) + lane * 16;
        for (int q = 0; q < pre_js; ++q) cp_async16(rfs + q * 512, rf + q * 512);
        cp_async_commit();
      }
      pre_valid = sum_segments(rt_pre, pre_ok, pre_pois);
    }
    if (JT > 0) gather_t(launch_tag(seq + p.tag_skew));   // == tag outside the failure-path test
    const bool t_good = JT == 0 || wait_t();
    if (pre_js > 0) cp_async_wait_all();   // each lane reads back only its own fragments
    for (int rt = rt_f; rt <= rt_z; ++rt) {
      if (!finishes(rt)) continue;
      if (!dcheck(rt < p.NRT, p.status)) continue;
      const bool pre = rt == rt_pre;
      bool seg_ok = pre_ok, poisoned = pre_pois;
      if (pre ? !pre_valid : !sum_segments(rt, seg_ok, poisoned)) continue;
      const uint8_t* rtg = rtile_src(rt);
      const bool store = seg_ok && !poisoned && t_good;
      if (!store)
        for (int e = lane; e < E; e += 32) ru[e] = 0.f;
      __syncwarp();
      float a4[NT][4];
      if (store && JT > 0) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int tk = nt * 8 + 2 * t;
          a4[nt][0] = tk < xrows ? ru[tk * 16 + g] : 0.f;
          a4[nt][1] = tk + 1 < xrows ? ru[(tk + 1) * 16 + g] : 0.f;
          a4[nt][2] = tk < xrows ? ru[tk * 16 + g + 8] : 0.f;
          a4[nt][3] = tk + 1 < xrows ? ru[(tk + 1) * 16 + g + 8] : 0.f;
        }
      }
      if (store && JT > 0) {
        // This row tile's fused linear owns T columns [grp * r16, (grp+1) * r16).
        int grp = 0;
        while (grp + 1 < p.n_groups && rt >= p.group_end_rt[grp]) ++grp;
        const uint16_t* tb = (NT == 2) ? Ts + min((lane & 7) + ((lane >> 4) & 1) * 8, last) * trow
                                       : Ts + min(lane & 7, last) * trow;
        tb += ((lane >> 3) & 1) * 8 + grp * p.r16;
        if (AQ) {
          // 4-bit R^T: per 128-group of r, the group's steps into a
          // separate accumulator, then scaled per output row (rows g and
          // g + 8 of the tile) into the tile's sums.
          for (int gr = 0; gr < p.ngr; ++gr) {
            const int js0 = gr * 8, jn = min(8, JS - js0);
            uint32_t wv[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
              if (q < jn) wv[q] = __ldg(reinterpret_cast<const uint32_t*>(rtg) + (js0 + q) * 32 + lane);
            const uint32_t sw = __ldg(reinterpret_cast<const uint32_t*>(rtg + JS * 128 + gr * 32) + g);
            float tq[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) tq[nt][0] = tq[nt][1] = tq[nt][2] = tq[nt][3] = 0.f;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              if (q < jn) {
                uint32_t a[4], b[4];
                decode_word(wv[q], a);
                const uint4 af = make_uint4(a[0], a[1], a[2], a[3]);
                if (NT == 2) ldmatrix_x4(b, tb + (js0 + q) * 16);
                else ldmatrix_x2(b, tb + (js0 + q) * 16);
                mma_16816(tq[0], af, b[0], b[1]);
                if (NT == 2) mma_16816(tq[NT - 1], af, b[2], b[3]);
              }
            }
            const float s_lo = f16_nonneg_bits_to_f32(sw & 0xFFFFu), s_hi = f16_nonneg_bits_to_f32(sw >> 16);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              a4[nt][0] = fmaf(s_lo, tq[nt][0], a4[nt][0]);
              a4[nt][1] = fmaf(s_lo, tq[nt][1], a4[nt][1]);
              a4[nt][2] = fmaf(s_hi, tq[nt][2], a4[nt][2]);
              a4[nt][3] = fmaf(s_hi, tq[nt][3], a4[nt][3]);
            }
          }
        } else {
          // Steps below ncp are in the ring (the first tile), the rest in L2.
          const int ncp = pre ? pre_js : 0;
          const uint4* rf = reinterpret_cast<const uint4*>(rtg);
          for (int js0 = 0; js0 < JS; js0 += 8) {
            uint4 af[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
              if (js0 + q < JS) af[q] = js0 + q < ncp ? lds128_s(rfs + (js0 + q) * 512) : __ldg(rf + (js0 + q) * 32 + lane);
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
        }
      }
      if (store && JT > 0) {
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
      __syncwarp();   // ru is reused for this warp's next tile
    }
  } else {
    // ------------------------------------------------------------ adapter warps
    // Item (jt, slice) of this CTA's panel: a range of the panel's K.
    const int aw = warp - kMainWarps;
    uint64_t* lbar = lbar_all + aw * p.nls;
    uint8_t* Ls = Ls_all + (size_t)aw * p.nls * ls_stage;
    const int item = (cta - p.cta0[pn]) * NA + aw;
    const bool has_item = JT > 0 && item < JT * p.SAp;
    const int KS = p.K / 16;
    const int jt = has_item ? item / p.SAp : 0, sl = has_item ? item % p.SAp : 0;
    const int ps0 = ps.kb0 * 16, ps1 = min((ps.kb0 + ps.kp) * 16, KS);
    const int sa = pn * p.SAp + sl;   // slot of the partial among the SA of column tile jt
    // The panel's K in units: K/16 steps of bf16 L^T (512 bytes each), or
    // 128-K blocks of 4-bit L^T (kLqBlock bytes, 8 steps, one scale group);
    // the item takes units [u0, u1), a ring stage holds ups of them.
    const int spu = AQ ? 8 : 1;
    const int ubytes = AQ ? kLqBlock : 512;
    const int ups = AQ ? kAdQBlocks : kAdStageSteps;
    const int pu0 = ps0 / spu, pu1 = ceil_div(ps1, spu);   // K is a multiple of 128: both exact
    const int u0 = pu0 + (int)((long long)sl * (pu1 - pu0) / p.SAp);
    const int u1 = has_item ? pu0 + (int)((long long)(sl + 1) * (pu1 - pu0) / p.SAp) : u0;
    const int s0 = u0 * spu;                   // first K/16 step
    const bool item_ok = dcheck(!has_item || (jt < JT && u1 * spu <= KS && sa < p.SA), p.status);
    const int nlc = item_ok ? ceil_div(u1 - u0, ups) : 0;   // ring chunks of this item
    const uint8_t* lsrc = AQ ? p.Lq + ((size_t)jt * (p.K / SLIM_GROUP) + u0) * kLqBlock
                               : reinterpret_cast<const uint8_t*>(p.Lf + ((size_t)jt * KS + u0) * 32);
    auto lissue = [&](int c) {
      const int st = c % p.nls;
      const uint32_t bytes = (uint32_t)min(ups, u1 - u0 - c * ups) * (uint32_t)ubytes;
      mbar_expect_tx(lbar + st, bytes);
      bulk_g2s(Ls + (size_t)st * ls_stage, lsrc + (size_t)c * ups * ubytes, bytes, lbar + st);
    };
    // Constant data before the wait: the item's packed L^T.
    if (lane == 0)
      for (int c = 0; c < p.nls && c < nlc; ++c) lissue(c);
    if (p.early) pdl_launch_dependents();
    bar_all<TW>();   // the previous grid has completed (thread 0 waited)
    if (has_item) {
      const uint32_t seq = *reinterpret_cast<volatile uint32_t*>(p.ctl);
      // Two accumulator chains (even and odd steps), added at the end: the
      // tensor-core chain of a stage is half as long.
      float acc[2][NT][4];
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) acc[h][nt][0] = acc[h][nt][1] = acc[h][nt][2] = acc[h][nt][3] = 0.f;
      // A = L^T fragments (16 columns j x 16 k).  B = X from the CTA's
      // staged panel (the item's steps lie in it).
      bool ok = mbar_wait(xbar, 0);
      const int xr = NT == 2 ? min((lane & 7) + ((lane >> 4) & 1) * 8, last) : min(lane & 7, last);
      const uint16_t* xsb = Xs + xr * xrow + ((lane >> 3) & 1) * 8 - ps0 * 16;   // indexed by absolute step
      int fail_c = 0;   // first chunk whose wait gave up
      for (int c = 0; c < nlc; ++c) {
        const int st = c % p.nls;
        if (ok) ok = mbar_wait(lbar + st, (c / p.nls) & 1);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) {
          fail_c = c;
          break;
        }
        const int n = min(ups, u1 - u0 - c * ups);   // units in this stage
        const uint8_t* sbase = Ls + (size_t)st * ls_stage;
        if (AQ) {
          // One scale group per block: its 8 steps into two short chains,
          // then scaled per adapter column (rows g and g + 8 of the tile).
#pragma unroll 1
          for (int qb = 0; qb < kAdQBlocks; ++qb) {
            if (qb < n) {
              const uint8_t* blk = sbase + qb * kLqBlock;
              const int sb = s0 + (c * kAdQBlocks + qb) * 8;
              float tq[2][NT][4];
#pragma unroll
              for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) tq[h][nt][0] = tq[h][nt][1] = tq[h][nt][2] = tq[h][nt][3] = 0.f;
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                uint32_t a[4], b[4];
                decode_word(*reinterpret_cast<const uint32_t*>(blk + (q * 32 + lane) * 4), a);
                const uint4 af = make_uint4(a[0], a[1], a[2], a[3]);
                if (NT == 2) ldmatrix_x4(b, xsb + (sb + q) * 16);
                else ldmatrix_x2(b, xsb + (sb + q) * 16);
                mma_16816(tq[q & 1][0], af, b[0], b[1]);
                if (NT == 2) mma_16816(tq[q & 1][NT - 1], af, b[2], b[3]);
              }
              const uint32_t sw = *reinterpret_cast<const uint32_t*>(blk + 1024 + 4 * g);
              const float s_lo = f16_nonneg_bits_to_f32(sw & 0xFFFFu), s_hi = f16_nonneg_bits_to_f32(sw >> 16);
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                acc[0][nt][0] = fmaf(s_lo, tq[0][nt][0] + tq[1][nt][0], acc[0][nt][0]);
                acc[0][nt][1] = fmaf(s_lo, tq[0][nt][1] + tq[1][nt][1], acc[0][nt][1]);
                acc[0][nt][2] = fmaf(s_hi, tq[0][nt][2] + tq[1][nt][2], acc[0][nt][2]);
                acc[0][nt][3] = fmaf(s_hi, tq[0][nt][3] + tq[1][nt][3], acc[0][nt][3]);
              }
            }
          }
        } else {
          const int sb = s0 + c * kAdStageSteps;
#pragma unroll
          for (int q = 0; q < kAdStageSteps; ++q) {
            if (q < n) {
              const uint4 a = lds128(sbase + (size_t)q * 512 + lane * 16);
              uint32_t b[4];
              if (NT == 2) ldmatrix_x4(b, xsb + (sb + q) * 16);
              else ldmatrix_x2(b, xsb + (sb + q) * 16);
              mma_16816(acc[q & 1][0], a, b[0], b[1]);
              if (NT == 2) mma_16816(acc[q & 1][NT - 1], a, b[2], b[3]);
            }
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
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[0][nt][i] += acc[1][nt][i];
        unsigned long long* mine = p.part_ll + ((size_t)jt * p.SA + sa) * 256;
        const unsigned long long tg = (unsigned long long)launch_tag(seq) << 32;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int tk = nt * 8 + 2 * t;
          if (tk < xrows) {
            st_relaxed_u64(mine + tk * 16 + g, tg | __float_as_uint(acc[0][nt][0]));
            st_relaxed_u64(mine + tk * 16 + g + 8, tg | __float_as_uint(acc[0][nt][2]));
          }
          if (tk + 1 < xrows) {
            st_relaxed_u64(mine + (tk + 1) * 16 + g, tg | __float_as_uint(acc[0][nt][1]));
            st_relaxed_u64(mine + (tk + 1) * 16 + g + 8, tg | __float_as_uint(acc[0][nt][3]));
          }
        }
      }
    }
    // The first NR panel-0 items of column tile jt add its SA partials in
    // slice order and publish T[:, jt] (with SA == 1 its partial is T): item
    // (jt, 0, sl) the elements [sl E / NR, (sl + 1) E / NR), one reducer per
    // 32 elements (a reducer spins until the partials arrive, so no more
    // warps than the work needs).  Words not yet current are polled again
    // together.
    const int NR = min(p.SAp, ceil_div(E, 32));
    if (has_item && pn == 0 && sl < NR && p.SA > 1) {
      const uint32_t seq = *reinterpret_cast<volatile uint32_t*>(p.ctl);
      const uint32_t tag = launch_tag(seq);
      const unsigned long long tg = (unsigned long long)tag << 32;
      const unsigned long long* src = p.part_ll + (size_t)jt * p.SA * 256;
      const int e0 = sl * E / NR, e1 = (sl + 1) * E / NR;
      bool rok = true;
      const int nw = (lane < e1 - e0 ? (e1 - e0 - lane + 31) / 32 : 0) * p.SA;
      int ke = e0 + lane, kq = 0, se = e0 + lane, sq = 0;
      float run = 0.f;
      for (int w0 = 0; w0 < nw; w0 += kMaxLLLoads) {
        unsigned long long v[kMaxLLLoads];
#pragma unroll
        for (int i = 0; i < kMaxLLLoads; ++i) {
          if (w0 + i < nw) {
            v[i] = ld_relaxed_u64(src + (size_t)kq * 256 + ke);
            if (++kq == p.SA) {
              kq = 0;
              ke += 32;
            }
          }
        }
        const long long c0 = clock64();
        while (rok) {
          bool stale = false;
#pragma unroll
          for (int i = 0; i < kMaxLLLoads; ++i) stale = stale || (w0 + i < nw && (uint32_t)(v[i] >> 32) != tag);
          if (!stale) break;
          if (clock64() - c0 > kWaitBudgetCycles) {
            rok = false;
            break;
          }
#pragma unroll
          for (int i = 0; i < kMaxLLLoads; ++i) {
            const int w = w0 + i;   // word w: partial w % SA of element e0 + lane + 32 (w / SA)
            if (w < nw && (uint32_t)(v[i] >> 32) != tag)
              v[i] = ld_relaxed_u64(src + (size_t)(w % p.SA) * 256 + e0 + lane + 32 * (w / p.SA));
          }
        }
#pragma unroll
        for (int i = 0; i < kMaxLLLoads; ++i) {
          if (w0 + i < nw) {
            run += __uint_as_float((uint32_t)v[i]);
            if (++sq == p.SA) {
              if (rok) st_relaxed_u64(p.t_fin + (size_t)jt * 256 + se, tg | __float_as_uint(run));
              run = 0.f;
              sq = 0;
              se += 32;
            }
          }
        }
      }
      if (!rok) record_status(p.status, SLIM_ERR_TIMEOUT);
    }
    // This CTA's slice is published: let the next launch start loading its
    // constants.
    pdl_launch_dependents();
  }

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
  int NT = 1, MW = 7, NA = 1, P = 1, KP = 1, G = 0, nst = 1, SA = 1, SAp = 1, nls = 0, segmax = 1;
  int cta0[kMaxPanels + 1] = {};
  size_t smem = 0;
};

int plan_segmax(const slim_layer& L, int MW, int P, int KP, const int* cta0) {
  int best = 1;
  for (int rt = 0; rt < L.n_row_tiles; ++rt)
    best = std::max(best, segment_slot(L.n_row_tiles, L.n_kblocks, KP, MW, P, cta0, rt, 0, 0).y);
  return best;
}

// CTAs per panel in proportion to the panel's chunks (at least one each).
void split_ctas(int P, int KP, int NKB, int G, int* cta0) {
  cta0[0] = 0;
  for (int q = 1; q < P; ++q) {
    const long long before = std::min((long long)q * KP, (long long)NKB);
    int c = (int)((before * G + NKB / 2) / NKB);
    c = std::max(c, cta0[q - 1] + 1);
    c = std::min(c, G - (P - q));
    cta0[q] = c;
  }
  cta0[P] = G;
}

StreamPlan plan_stream_mw(const slim_layer& L, int M, int MW, int NA) {
  StreamPlan pl;
  const int NT = M <= 8 ? 1 : 2;
  const int xrows = std::min(M, NT * 8);
  const int JT = L.rl16 / 16;
  const int nsm = num_sms();
  const long long chunks = (long long)L.n_row_tiles * L.n_kblocks;
  // CTAs: one per SM, fewer when there are not 2 chunks per main warp.
  const int G = (int)std::max<long long>(1, std::min<long long>(nsm, chunks / (2 * MW)));
  const size_t limit = MW + NA == 8 ? kSmemPair : kSmemLimit;
  const int aq = L.adapter_bits == 4 ? 1 : 0;
  // Fewest K panels that fit (each extra panel adds segments to every row
  // tile); then the deepest rings.
  const int nst_min = MW + NA == 16 ? 2 : 3;
  for (int Pw = 1; Pw <= std::min(L.n_kblocks, kMaxPanels); ++Pw) {
    const int KP = ceil_div(L.n_kblocks, Pw);
    const int P = ceil_div(L.n_kblocks, KP);
    if (P != Pw) continue;
    if (P > G) break;
    int cta0[kMaxPanels + 1] = {};
    split_ctas(P, KP, L.n_kblocks, G, cta0);
    int nc_min = G;
    for (int q = 0; q < P; ++q) nc_min = std::min(nc_min, cta0[q + 1] - cta0[q]);
    // Adapter slices per panel: every item on its own adapter warp of the
    // panel, at most 16 partials per T element in all, at least 8 K steps a
    // slice.
    if (JT > nc_min * NA) continue;
    const int SAp = JT > 0 ? std::max(1, std::min({nc_min * NA / JT, std::max(1, 16 / P), KP * 16 / 8})) : 1;
    const int nls_max =
        JT > 0 ? std::min(kMaxAdStages, aq ? ceil_div(ceil_div(KP * 2, SAp), kAdQBlocks)
                                           : ceil_div(ceil_div(KP * 16, SAp), kAdStageSteps))
               : 0;
    const int nls_min = std::min(nls_max, 4);
    for (int nst = kMaxStagesS; nst >= nst_min; --nst) {
      for (int nls = nls_max; nls >= nls_min; --nls) {
        const size_t smem = stream_smem(MW, NA, xrows, KP, nst, L.rl16, nls, ad_stage_bytes(aq)).total;
        if (smem > limit) continue;
        pl.ok = true;
        pl.NT = NT;
        pl.MW = MW;
        pl.NA = NA;
        pl.P = P;
        pl.KP = KP;
        pl.G = G;
        pl.nst = nst;
        pl.SAp = SAp;
        pl.SA = P * SAp;
        pl.nls = nls;
        pl.smem = smem;
        std::copy(cta0, cta0 + kMaxPanels + 1, pl.cta0);
        pl.segmax = plan_segmax(L, MW, P, KP, pl.cta0);
        return pl;
      }
    }
  }
  return pl;
}

StreamPlan plan_stream_uncached(const slim_layer& L, int M, const Tuning& tn) {
  if (M < 1 || M > 16 || L.rl16 > kMaxTCols || tn.no_stream) return StreamPlan();
  if (L.rl16 / 16 > num_sms()) return StreamPlan();
  // CTAs of 16 warps for long streams (latency hiding), 8 when the stream is
  // short (two CTAs fit on an SM, so the next launch overlaps this one's
  // end), unless 8-warp CTAs would need more K panels.  Two of them adapter
  // warps when L and R are at least a quarter of the packed weight's bytes.
  const long long chunks = (long long)L.n_row_tiles * L.n_kblocks;
  const double wbytes = (double)L.N * L.K * 25.0 / 64.0;
  const double abytes = L.adapter_bits == 4
                            ? (double)(L.rl16 / 16) * (L.K / SLIM_GROUP) * kLqBlock +
                                  (double)L.n_row_tiles * rq_tile_bytes(L.r16, L.r)
                            : 2.0 * L.K * L.rl16 + 2.0 * L.r16 * L.N;
  const int NA = L.rl16 > 0 && abytes >= 0.25 * wbytes ? 2 : 1;
  // Layers of 2048 up to 64 chunks per SM with an adapter (LLaMA-2-70B k and
  // v, 7B q_proj: 8 MB) spend most of a single-launch call on its fixed costs
  // (the cross-CTA T reduction, finishing); the token-tiled pair measured
  // faster (bf16 adapters, 70B k: 11.6 against 13.4 us at one token, 12.8
  // against 15.1 at four; 7B q_proj: 9.7 against 11.4; 4-bit adapters, 70B
  // k: 11.9 against 13.0, 15.5 against 17.9 at eight; 7B q_proj: 9.5 against
  // 11.5, 15.1 against 17.6 at sixteen).  A forced warp count keeps the
  // single-launch kernel.
  if (!tn.stream_warps && L.rl16 > 0 && chunks >= 2048 && chunks < (long long)num_sms() * 64) return StreamPlan();
  int TW = chunks >= (long long)num_sms() * 64 ? 16 : 8;
  if (tn.stream_warps) TW = tn.stream_warps == 16 ? 16 : 8;
  StreamPlan pl = plan_stream_mw(L, M, TW - NA, NA);
  if (!tn.stream_warps) {
    const StreamPlan alt = plan_stream_mw(L, M, 24 - TW - NA, NA);
    if (alt.ok && (!pl.ok || (TW == 8 && alt.P < pl.P && pl.P > 2))) pl = alt;
  }
  // A short stream of two token tiles cut into many segments per row tile:
  // the finishing reads outweigh the stream, and the token-tiled pair of
  // kernels is faster (measured on the 7B q_proj and 70B k/v shapes).
  if (pl.ok && pl.NT == 2 && pl.segmax > 8 && chunks < (long long)num_sms() * 64) return StreamPlan();
  return pl;
}

// Plans depend on the layer's shape, M, the device and the tuning knobs;
// each is computed once.
StreamPlan plan_stream(const slim_layer& L, int M) {
  static PlanCache<8, StreamPlan> cache;
  const Tuning tn = tuning();
  return cache.get({current_device(), (long long)tn.generation, L.K, L.N, L.r16, L.rl16, M, L.adapter_bits},
                   [&] { return plan_stream_uncached(L, M, tn); });
}

template <int NT, int MW, int NA, bool AQ>
cudaError_t run(cudaLaunchConfig_t& cfg, size_t smem, const StreamParams& p) {
  cudaError_t e = ensure_func_attrs(reinterpret_cast<const void*>(k_stream<NT, MW, NA, AQ>), smem);
  if (e != cudaSuccess) return e;
  return cudaLaunchKernelEx(&cfg, k_stream<NT, MW, NA, AQ>, p);
}

template <int NT, bool AQ>
cudaError_t run_nt(cudaLaunchConfig_t& cfg, const StreamPlan& pl, const StreamParams& p) {
  if (pl.MW == 7) return run<NT, 7, 1, AQ>(cfg, pl.smem, p);
  if (pl.MW == 6) return run<NT, 6, 2, AQ>(cfg, pl.smem, p);
  if (pl.MW == 15) return run<NT, 15, 1, AQ>(cfg, pl.smem, p);
  return run<NT, 14, 2, AQ>(cfg, pl.smem, p);
}

size_t a256(size_t x) { return (x + 255) / 256 * 256; }

struct StreamWs {
  size_t ctl, part_ll, t_fin, part, total;
};

// Workspace: the control block (256 bytes), the adapter's tagged partials
// and the tagged T they add up to, the tagged segment partials.
StreamWs stream_ws(const slim_layer& L, const StreamPlan& pl, int M) {
  StreamWs w;
  const int JT = L.rl16 / 16;
  const int xrows = std::min(M, pl.NT * 8);
  size_t off = 0;
  w.ctl = off;      off += 256;
  w.part_ll = off;  off += JT > 0 ? a256((size_t)JT * pl.SA * 256 * 8) : 0;
  w.t_fin = off;    off += JT > 0 && pl.SA > 1 ? a256((size_t)JT * 256 * 8) : 0;
  w.part = off;     off += a256((size_t)L.n_row_tiles * pl.segmax * xrows * 16 * 8);
  w.total = off;
  return w;
}

}  // namespace

size_t stream_workspace_bytes(const slim_layer& L, int M) {
  const StreamPlan pl = plan_stream(L, M);
  return pl.ok ? stream_ws(L, pl, M).total : 0;
}

bool stream_supported(const slim_layer& L, int M) { return plan_stream(L, M).ok; }

cudaError_t launch_stream(const slim_layer& L, const uint16_t* X, int M, uint16_t* Y, void* ws, cudaStream_t s) {
  return launch_stream_ex(L, X, M, Y, ws, kWaitBudgetCycles, 0u, s);
}

cudaError_t launch_stream_ex(const slim_layer& L, const uint16_t* X, int M, uint16_t* Y, void* ws,
                             long long t_wait_cycles, uint32_t tag_skew, cudaStream_t s) {
  NvtxRange nv("decode: stream, adapter, finishing and epilogue in one launch (k_stream)");
  const StreamPlan pl = plan_stream(L, M);
  if (!pl.ok) return cudaErrorNotSupported;
  const StreamWs w = stream_ws(L, pl, M);
  uint8_t* wb = static_cast<uint8_t*>(ws);
  StreamParams p;
  p.X = X;
  p.Y = Y;
  p.dec = L.dec;
  p.Rf = reinterpret_cast<const uint4*>(L.Rf);
  p.Lf = reinterpret_cast<const uint4*>(L.Lf);
  p.aq = L.adapter_bits == 4 ? 1 : 0;
  p.Rq = L.Rq;
  p.Lq = L.Lq;
  p.rqt = L.r16 ? rq_tile_bytes(L.r16, L.r) : 0;
  p.ngr = rq_groups(L.r);
  p.part_ll = L.r16 > 0 ? reinterpret_cast<unsigned long long*>(wb + w.part_ll) : nullptr;
  p.t_fin = L.r16 > 0 ? reinterpret_cast<unsigned long long*>(wb + (pl.SA > 1 ? w.t_fin : w.part_ll)) : nullptr;
  p.part = reinterpret_cast<unsigned long long*>(wb + w.part);
  p.ctl = reinterpret_cast<uint32_t*>(wb + w.ctl);
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
  p.segmax = pl.segmax;
  p.SA = pl.SA;
  p.SAp = pl.SAp;
  p.nst = pl.nst;
  p.nls = pl.nls;
  p.early = tuning().pdl_early ? 1 : 0;
  for (int q = 0; q <= kMaxPanels; ++q) p.cta0[q] = pl.cta0[q];
  p.status = L.status;
  p.t_wait = t_wait_cycles;
  p.tag_skew = tag_skew;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.G);
  cfg.blockDim = dim3((pl.MW + pl.NA) * 32);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (p.aq) return pl.NT == 1 ? run_nt<1, true>(cfg, pl, p) : run_nt<2, true>(cfg, pl, p);
  return pl.NT == 1 ? run_nt<1, false>(cfg, pl, p) : run_nt<2, false>(cfg, pl, p);
}

}  // namespace slim

// Packing kernels: dense bf16 W -> canonical (vals, meta, scales) + the
// decode-stream layout, and the adapter L, R -> tensor-core fragment order.
//
// SLiM pipeline (thesis "Compression Trinity", Fig. 7.1 caption): step 1
// quantizes W with a symmetric quantizer, step 2 prunes the *quantized*
// weights.  Quantization is 4-bit, weight-only, group size 128 (summary page,
// paragraph on the reported setups); 2:4 runs along the reduction dimension
// K and is stored as packed values plus position metadata (§2.2.3 "Sparse
// Tensor Core Acceleration").
#include "slim_common.cuh"
#include "slim_internal.h"

namespace slim {
namespace {

// One CTA per decode chunk (16 rows x 256 K).  Warp w quantizes row w % 16 of
// 128-group w / 16: lane l owns the four consecutive weights 4l..4l+3 of the
// group (one 2:4 block).
__global__ void __launch_bounds__(1024) k_pack(const uint16_t* __restrict__ W, int K, int N,
                                               uint8_t* __restrict__ vals, uint8_t* __restrict__ meta,
                                               uint16_t* __restrict__ scales, uint8_t* __restrict__ dec,
                                               int n_kblocks, int32_t* status) {
  __shared__ uint32_t chunk[kDecChunk / 4];
  const int kb = blockIdx.x, rt = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rr = warp & 15, gg = warp >> 4;
  const int n = rt * 16 + rr;
  const int G = K / SLIM_GROUP;
  const int g = kb * 2 + gg;
  for (int i = threadIdx.x; i < kDecChunk / 4; i += blockDim.x) chunk[i] = 0u;
  __syncthreads();

  const bool valid = (n < N) && (g < G);
  float w[4] = {0.f, 0.f, 0.f, 0.f};
  if (valid) {
    const uint2 raw = *reinterpret_cast<const uint2*>(W + (size_t)n * K + (size_t)g * SLIM_GROUP + lane * 4);
    w[0] = __uint_as_float(raw.x << 16);
    w[1] = __uint_as_float(raw.x & 0xFFFF0000u);
    w[2] = __uint_as_float(raw.y << 16);
    w[3] = __uint_as_float(raw.y & 0xFFFF0000u);
  }
  // Group abs-max (exact in any order) and the NaN check fmaxf would hide.
  float amax = fmaxf(fmaxf(fabsf(w[0]), fabsf(w[1])), fmaxf(fabsf(w[2]), fabsf(w[3])));
  const bool nan4 = isnan(w[0]) || isnan(w[1]) || isnan(w[2]) || isnan(w[3]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const bool any_nan = __any_sync(0xffffffffu, nan4);

  // s = fp16_rn(amax / 7) in IEEE fp32 (correctly rounded division).
  const float s32 = __fdiv_rn(amax, 7.0f);
  const __half s16 = __float2half_rn(s32);
  const float sf = __half2float(s16);
  const bool bad = any_nan || isinf(sf);
  if (valid && bad && lane == 0) record_status(status, SLIM_ERR_RANGE);

  int q[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (!valid || bad || sf == 0.f) {
      q[i] = 0;
    } else {
      float t = rintf(__fdiv_rn(w[i], sf));  // round half to even
      t = fminf(fmaxf(t, -7.f), 7.f);
      q[i] = static_cast<int>(t);
    }
  }
  // 2:4: keep the pair with the largest |q| sum, first pair (lexicographic)
  // on ties.
  const int a0 = abs(q[0]), a1 = abs(q[1]), a2 = abs(q[2]), a3 = abs(q[3]);
  int i0 = 0, i1 = 1, best = a0 + a1;
  if (a0 + a2 > best) { best = a0 + a2; i0 = 0; i1 = 2; }
  if (a0 + a3 > best) { best = a0 + a3; i0 = 0; i1 = 3; }
  if (a1 + a2 > best) { best = a1 + a2; i0 = 1; i1 = 2; }
  if (a1 + a3 > best) { best = a1 + a3; i0 = 1; i1 = 3; }
  if (a2 + a3 > best) { best = a2 + a3; i0 = 2; i1 = 3; }
  const int v0 = q[i0], v1 = q[i1];
  const uint32_t nib = static_cast<uint32_t>(i0 | (i1 << 2));

  // Canonical format.
  if (valid) {
    vals[(size_t)n * (K / 4) + (size_t)g * 32 + lane] = static_cast<uint8_t>((v0 & 0xF) | ((v1 & 0xF) << 4));
  }
  const uint32_t nib_hi = __shfl_down_sync(0xffffffffu, nib, 1);
  if (valid && !(lane & 1)) {
    meta[(size_t)n * (K / 8) + (size_t)g * 16 + (lane >> 1)] = static_cast<uint8_t>(nib | (nib_hi << 4));
  }
  const uint16_t s_bits = (valid && !bad) ? __half_as_ushort(s16) : static_cast<uint16_t>(0);
  if (valid && lane == 0) scales[(size_t)n * G + g] = s_bits;

  // Decode-stream chunk.  Chunk index within the 256-K block: cc = 0..63;
  // MMA step j = cc / 8 covers 32 K; within the step, block u = cc % 8.
  const int cc = gg * 32 + lane;
  const int j = cc >> 3, u = cc & 7;
  const int half = u >> 2, c = u & 3;     // A fragment: blocks 0-3 -> regs a0/a1, 4-7 -> a2/a3
  const int hi_row = rr >> 3;             // rows 8..15 of the tile use the odd registers
  const int frag_lane = (rr & 7) * 4 + c;
  const int p = half * 2 + hi_row;
  const uint32_t u0 = static_cast<uint32_t>((v0 + 8) & 0xF), u1 = static_cast<uint32_t>((v1 + 8) & 0xF);
  atomicOr(&chunk[(j >> 2) * 128 + frag_lane * 4 + (j & 3)], (u0 << (4 * p)) | (u1 << (16 + 4 * p)));
  // Metadata: for step j, the thread pair 2*(j&1) + {0,1} of each quad
  // supplies it; pair member `half` holds blocks 4*half..4*half+3 for rows
  // g (low 16 bits) and g+8 (high 16 bits).
  const int owner = (rr & 7) * 4 + (j & 1) * 2 + half;
  atomicOr(&chunk[256 + owner * 4 + (j >> 1)], nib << (hi_row * 16 + 4 * c));
  if (lane == 0) {
    const int si = scale_slot(gg, rr);
    atomicOr(&chunk[384 + (si >> 1)], static_cast<uint32_t>(s_bits) << ((si & 1) * 16));
  }
  __syncthreads();
  uint32_t* out = reinterpret_cast<uint32_t*>(dec + ((size_t)rt * n_kblocks + kb) * kDecChunk);
  for (int i = threadIdx.x; i < kDecChunk / 4; i += blockDim.x) out[i] = chunk[i];
}

// Adapter column c of T = X L (0 <= c < G * r16) is column c % r16 of
// linear c / r16's factor, i.e. column (c / r16) * r + c % r16 of the
// caller's L [K][G * r]; -1 for the zero padding between r and r16.
__device__ __forceinline__ int l_column(int c, int r, int r16) {
  const int g = c / r16, j = c % r16;
  return j < r ? g * r + j : -1;
}

// ------------------------------------------------------------ 4-bit adapters
// Quantized SLiM quantizes the low-rank adapters too (thesis §7.4.3
// "Low-rank adapter quantization"; Tables E.13 / E.14 captions).  The
// weights' quantizer is applied to each factor along its reduction
// dimension: L [K][G r] per column over 128 consecutive k, R [r][N] per
// column over 128 consecutive j (the last group shorter when r % 128 != 0),
// with the same IEEE fp32 steps as k_pack.
struct AdapterShape {
  int K, N, r, r16, G;
  int KG;        // K / 128
  int JT;        // rl16 / 16
  int JS;        // r16 / 16
  int NRT;       // ceil(N / 16)
  int ngr;       // 128-groups of r
  int rqt;       // bytes of one Rq row tile
};

AdapterShape adapter_shape(const slim_layer& L) {
  AdapterShape a;
  a.K = L.K;
  a.N = L.N;
  a.r = L.r;
  a.r16 = L.r16;
  a.G = L.n_groups;
  a.KG = L.K / SLIM_GROUP;
  a.JT = L.rl16 / 16;
  a.JS = L.r16 / 16;
  a.NRT = L.n_row_tiles;
  a.ngr = rq_groups(L.r);
  a.rqt = L.r16 ? rq_tile_bytes(L.r16, L.r) : 0;
  return a;
}

// q = clip(rint(v / s), -7, 7) as k_pack computes it; 0 for a zero or
// non-finite scale and for a NaN value (the pack then reports a range error).
__device__ __forceinline__ int quant4(float v, uint16_t s_bits) {
  const float sf = __half2float(__ushort_as_half(s_bits));
  if (sf == 0.f || isinf(sf) || isnan(v)) return 0;
  const float t = fminf(fmaxf(rintf(__fdiv_rn(v, sf)), -7.f), 7.f);
  return static_cast<int>(t);
}

// One thread per (column c of L^T, 128-group of K) and per (row n of R^T,
// 128-group of r): the group's fp16 scale into its slot of Lq / Rq.
__global__ void k_quant_adapter_scales(const uint16_t* __restrict__ Lsrc, const uint16_t* __restrict__ Rsrc,
                                       AdapterShape a, uint8_t* __restrict__ Lq, uint8_t* __restrict__ Rq,
                                       int32_t* status) {
  const int rl16 = a.JT * 16;
  const size_t nL = (size_t)rl16 * a.KG, nR = (size_t)a.NRT * 16 * a.ngr;
  const size_t tid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (tid >= nL + nR) return;
  float amax = 0.f;
  bool nan = false;
  uint16_t* slot;
  if (tid < nL) {
    const int c = static_cast<int>(tid % rl16), kg = static_cast<int>(tid / rl16);
    const int lc = l_column(c, a.r, a.r16);
    if (lc >= 0)
      for (int k = kg * SLIM_GROUP; k < (kg + 1) * SLIM_GROUP; ++k) {
        const float v = __uint_as_float(static_cast<uint32_t>(Lsrc[(size_t)k * a.G * a.r + lc]) << 16);
        nan = nan || isnan(v);
        amax = fmaxf(amax, fabsf(v));
      }
    slot = reinterpret_cast<uint16_t*>(Lq + ((size_t)(c >> 4) * a.KG + kg) * kLqBlock + 1024) +
           frag_scale_slot(c & 15);
  } else {
    const size_t i = tid - nL;
    const int n = static_cast<int>(i % ((size_t)a.NRT * 16)), gr = static_cast<int>(i / ((size_t)a.NRT * 16));
    if (n < a.N)
      for (int j = gr * SLIM_GROUP; j < min((gr + 1) * SLIM_GROUP, a.r); ++j) {
        const float v = __uint_as_float(static_cast<uint32_t>(Rsrc[(size_t)j * a.N + n]) << 16);
        nan = nan || isnan(v);
        amax = fmaxf(amax, fabsf(v));
      }
    slot = reinterpret_cast<uint16_t*>(Rq + (size_t)(n >> 4) * a.rqt + a.JS * 128 + gr * 32) +
           frag_scale_slot(n & 15);
  }
  const __half s16 = __float2half_rn(__fdiv_rn(amax, 7.0f));
  if (nan || isinf(__half2float(s16))) record_status(status, SLIM_ERR_RANGE);
  *slot = __half_as_ushort(s16);
}

// One thread per fragment word (8 nibbles) of Lq and of Rq; the scales are
// already in place.
__global__ void k_quant_adapter_words(const uint16_t* __restrict__ Lsrc, const uint16_t* __restrict__ Rsrc,
                                      AdapterShape a, uint8_t* __restrict__ Lq, uint8_t* __restrict__ Rq) {
  const size_t nL = (size_t)a.JT * a.KG * 8 * 32, nR = (size_t)a.NRT * a.JS * 32;
  const size_t tid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (tid >= nL + nR) return;
  const int lane = static_cast<int>(tid & 31), g = lane >> 2, t = lane & 3;
  uint32_t word = 0;
  if (tid < nL) {
    const int step = static_cast<int>((tid >> 5) & 7);
    const size_t blk = tid >> 8;
    const int jt = static_cast<int>(blk / a.KG), kg = static_cast<int>(blk % a.KG);
    uint8_t* base = Lq + blk * kLqBlock;
    const uint16_t* sc = reinterpret_cast<const uint16_t*>(base + 1024);
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int row = g + 8 * (p & 1), kl = 2 * t + 8 * (p >> 1) + e;
        const int lc = l_column(jt * 16 + row, a.r, a.r16);
        const int k = kg * SLIM_GROUP + step * 16 + kl;
        const float v = lc >= 0 ? __uint_as_float(static_cast<uint32_t>(Lsrc[(size_t)k * a.G * a.r + lc]) << 16)
                                : 0.f;
        const int q = quant4(v, sc[frag_scale_slot(row)]);
        word |= static_cast<uint32_t>(q + 8) << frag_shift(row, kl);
      }
    reinterpret_cast<uint32_t*>(base)[step * 32 + lane] = word;
  } else {
    const size_t i = tid - nL;
    const size_t ts = i >> 5;
    const int rt = static_cast<int>(ts / a.JS), js = static_cast<int>(ts % a.JS);
    uint8_t* tile = Rq + (size_t)rt * a.rqt;
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int row = g + 8 * (p & 1), kl = 2 * t + 8 * (p >> 1) + e;
        const int n = rt * 16 + row, j = js * 16 + kl;
        const float v = (n < a.N && j < a.r)
                            ? __uint_as_float(static_cast<uint32_t>(Rsrc[(size_t)j * a.N + n]) << 16)
                            : 0.f;
        const uint16_t* sc = reinterpret_cast<const uint16_t*>(tile + a.JS * 128 + (j >> 7) * 32);
        const int q = quant4(v, sc[frag_scale_slot(row)]);
        word |= static_cast<uint32_t>(q + 8) << frag_shift(row, kl);
      }
    reinterpret_cast<uint32_t*>(tile)[js * 32 + lane] = word;
  }
}

// q and the bf16 bits of q * s (exact in fp32, then rounded to nearest
// even) of one element of Lq (column c of L^T, k) or of Rq (row n of R^T, j).
__device__ __forceinline__ int lq_q(const uint8_t* Lq, int KG, int c, int k) {
  const uint8_t* blk = Lq + ((size_t)(c >> 4) * KG + (k >> 7)) * kLqBlock;
  const int row = c & 15, kl = k & 15;
  const uint32_t w = reinterpret_cast<const uint32_t*>(blk)[((k & 127) >> 4) * 32 + frag_lane(row, kl)];
  return static_cast<int>((w >> frag_shift(row, kl)) & 15u) - 8;
}
__device__ __forceinline__ uint16_t lq_s(const uint8_t* Lq, int KG, int c, int k) {
  const uint8_t* blk = Lq + ((size_t)(c >> 4) * KG + (k >> 7)) * kLqBlock;
  return reinterpret_cast<const uint16_t*>(blk + 1024)[frag_scale_slot(c & 15)];
}
__device__ __forceinline__ int rq_q(const uint8_t* Rq, int rqt, int n, int j) {
  const uint8_t* tile = Rq + (size_t)(n >> 4) * rqt;
  const int row = n & 15, kl = j & 15;
  const uint32_t w = reinterpret_cast<const uint32_t*>(tile)[(j >> 4) * 32 + frag_lane(row, kl)];
  return static_cast<int>((w >> frag_shift(row, kl)) & 15u) - 8;
}
__device__ __forceinline__ uint16_t rq_s(const uint8_t* Rq, int rqt, int JS, int n, int j) {
  const uint8_t* tile = Rq + (size_t)(n >> 4) * rqt;
  return reinterpret_cast<const uint16_t*>(tile + JS * 128 + (j >> 7) * 32)[frag_scale_slot(n & 15)];
}
__device__ __forceinline__ uint16_t dequant_bf16(int q, uint16_t s_bits) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(static_cast<float>(q) * __half2float(__ushort_as_half(s_bits))));
}

// The adapter values the bf16 layouts hold: the caller's L and R, or (with
// Lq / Rq set) the dequantized 4-bit factors.
struct AdapterSrc {
  const uint16_t* L;
  const uint16_t* R;
  const uint8_t* Lq;   // NULL: bf16 adapters
  const uint8_t* Rq;
  int N, lstride, KG, JS, rqt;
  // L[k][lc], lc the caller's column of adapter column c.
  __device__ __forceinline__ uint16_t l(int k, int c, int lc) const {
    return Lq ? dequant_bf16(lq_q(Lq, KG, c, k), lq_s(Lq, KG, c, k)) : L[(size_t)k * lstride + lc];
  }
  // R[j][n] (j < r, n < N).
  __device__ __forceinline__ uint16_t rv(int j, int n) const {
    return Rq ? dequant_bf16(rq_q(Rq, rqt, n, j), rq_s(Rq, rqt, JS, n, j)) : R[(size_t)j * N + n];
  }
};

AdapterSrc adapter_src(const slim_layer& L, const uint16_t* Lsrc, const uint16_t* Rsrc) {
  AdapterSrc a;
  a.L = Lsrc;
  a.R = Rsrc;
  const bool q4 = L.adapter_bits == 4;
  a.Lq = q4 ? L.Lq : nullptr;
  a.Rq = q4 ? L.Rq : nullptr;
  a.N = L.N;
  a.lstride = L.n_groups * L.r;
  a.KG = L.K / SLIM_GROUP;
  a.JS = L.r16 / 16;
  a.rqt = L.r16 ? rq_tile_bytes(L.r16, L.r) : 0;
  return a;
}

// Test aid: the 4-bit layouts back to q_L [K][G r], s_L [K/128][G r],
// q_R [r][N], s_R [ceil(r/128)][N].  One thread per output element.
__global__ void k_unpack_adapters(AdapterShape a, const uint8_t* __restrict__ Lq, const uint8_t* __restrict__ Rq,
                                  int8_t* __restrict__ qL, uint16_t* __restrict__ sL, int8_t* __restrict__ qR,
                                  uint16_t* __restrict__ sR) {
  const size_t gr_ = (size_t)a.G * a.r;
  const size_t n0 = (size_t)a.K * gr_, n1 = n0 + (size_t)a.KG * gr_, n2 = n1 + (size_t)a.r * a.N,
               n3 = n2 + (size_t)a.ngr * a.N;
  const size_t tid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (tid >= n3) return;
  if (tid < n1) {
    const bool sc = tid >= n0;
    const size_t i = sc ? tid - n0 : tid;
    const int lc = static_cast<int>(i % gr_), kk = static_cast<int>(i / gr_);
    const int c = (lc / a.r) * a.r16 + lc % a.r;
    if (sc) sL[i] = lq_s(Lq, a.KG, c, kk * SLIM_GROUP);
    else qL[i] = static_cast<int8_t>(lq_q(Lq, a.KG, c, kk));
  } else {
    const bool sc = tid >= n2;
    const size_t i = sc ? tid - n2 : tid - n1;
    const int n = static_cast<int>(i % a.N), jj = static_cast<int>(i / a.N);
    if (sc) sR[i] = rq_s(Rq, a.rqt, a.JS, n, jj * SLIM_GROUP);
    else qR[i] = static_cast<int8_t>(rq_q(Rq, a.rqt, n, jj));
  }
}

// Adapter layouts for the dense m16n8k16 A operand (16 rows x 16 k per
// fragment, lane (g, t) holds rows g / g+8 at k = 2t, 2t+1 and 2t+8, 2t+9):
//   Lf: A = L^T  [rl16 rows][K], tile (jt, ks) at ((jt * K/16 + ks) * 32 + lane) * 4 words;
//   Rf: A = R^T  [N16 rows][r16], tile (rt, js) at ((rt * r16/16 + js) * 32 + lane) * 4 words.
// Rows or columns beyond r / N are zero.  L has G * r columns (G fused
// linears side by side), R has N columns.
__global__ void k_pack_adapter(AdapterSrc src, int K, int N, int r, int r16, int G, uint32_t* __restrict__ Lf,
                               uint32_t* __restrict__ Rf) {
  const int rl16 = G * r16;
  const size_t nL = (size_t)rl16 * K / 2;
  const size_t nR = (size_t)ceil_div(N, 16) * 16 * r16 / 2;
  const size_t tid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (tid >= nL + nR) return;
  const bool isL = tid < nL;
  const size_t idx = isL ? tid : tid - nL;
  const int reg = static_cast<int>(idx & 3);
  const int lane = static_cast<int>((idx >> 2) & 31);
  const size_t tile = idx >> 7;
  const int g = lane >> 2, t = lane & 3;
  const int row_off = g + ((reg & 1) ? 8 : 0);
  const int col_off = 2 * t + ((reg & 2) ? 8 : 0);
  uint32_t lo = 0, hi = 0;
  if (isL) {
    const int KS = K / 16;
    const int jt = static_cast<int>(tile / KS), ks = static_cast<int>(tile % KS);
    const int jrow = jt * 16 + row_off, k = ks * 16 + col_off;  // A[j][k] = L[k][j]
    const int lc = l_column(jrow, r, r16);
    if (lc >= 0) {
      lo = src.l(k, jrow, lc);
      hi = src.l(k + 1, jrow, lc);
    }
    Lf[idx] = lo | (hi << 16);
  } else {
    const int JS = r16 / 16;
    const int rt = static_cast<int>(tile / JS), js = static_cast<int>(tile % JS);
    const int n = rt * 16 + row_off, jj = js * 16 + col_off;  // A[n][j] = R[j][n]
    if (n < N) {
      if (jj < r) lo = src.rv(jj, n);
      if (jj + 1 < r) hi = src.rv(jj + 1, n);
    }
    Rf[idx] = lo | (hi << 16);
  }
}

// Expand the decode stream back to dense q and scales (test aid).  One
// thread per (row, 4-block).
__global__ void k_unpack_dec(const uint8_t* __restrict__ dec, int K, int N, int n_kblocks,
                             int8_t* __restrict__ q, uint16_t* __restrict__ scales) {
  const size_t tid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t nblk = (size_t)N * (K / 4);
  if (tid >= nblk) return;
  const int n = static_cast<int>(tid / (K / 4));
  const int blk = static_cast<int>(tid % (K / 4));  // 4-block index along K
  const int rt = n / 16, rr = n % 16;
  const int kb = blk / 64, cc = blk % 64;
  const uint32_t* ch = reinterpret_cast<const uint32_t*>(dec + ((size_t)rt * n_kblocks + kb) * kDecChunk);
  const int j = cc >> 3, u = cc & 7, half = u >> 2, c = u & 3, hi_row = rr >> 3;
  const int p = half * 2 + hi_row;
  const uint32_t w = ch[(j >> 2) * 128 + ((rr & 7) * 4 + c) * 4 + (j & 3)];
  const int v0 = static_cast<int>((w >> (4 * p)) & 0xF) - 8;
  const int v1 = static_cast<int>((w >> (16 + 4 * p)) & 0xF) - 8;
  const int owner = (rr & 7) * 4 + (j & 1) * 2 + half;
  const uint32_t nib = (ch[256 + owner * 4 + (j >> 1)] >> (hi_row * 16 + 4 * c)) & 0xF;
  const int i0 = nib & 3, i1 = nib >> 2;
  char4 out = make_char4(0, 0, 0, 0);
  int8_t* o = reinterpret_cast<int8_t*>(&out);
  o[i0] = static_cast<int8_t>(v0);
  o[i1] = static_cast<int8_t>(v1);
  *reinterpret_cast<char4*>(q + (size_t)n * K + (size_t)blk * 4) = out;
  if ((blk & 31) == 0) {
    const int gg = (blk / 32) & 1;
    const int si = scale_slot(gg, rr);
    const uint32_t sw = ch[384 + (si >> 1)];
    scales[(size_t)n * (K / SLIM_GROUP) + blk / 32] = static_cast<uint16_t>(sw >> ((si & 1) * 16));
  }
}

// R^T image for the prefill kernel's adapter MMA: 128-row tiles, each
// ceil(r16/64) swizzled atoms of 128 rows x 64 columns (see sw128_offset).
__global__ void k_pack_rp(AdapterSrc src, int N, int r, int r64, uint16_t* __restrict__ Rp, size_t total) {
  const size_t tid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (tid >= total) return;
  const int j = static_cast<int>(tid % r64);
  const size_t n = tid / r64;
  const size_t tile = n / 128;
  const int row = static_cast<int>(n % 128);
  const uint16_t v = (n < (size_t)N && j < r) ? src.rv(j, static_cast<int>(n)) : static_cast<uint16_t>(0);
  uint8_t* base = reinterpret_cast<uint8_t*>(Rp) + tile * (size_t)r64 * 256;
  *reinterpret_cast<uint16_t*>(base + sw128_offset(row, j, 128)) = v;
}

// L^T images for the prefill path's X L: one 128-byte-swizzled atom of rl16
// rows x 64 K per 64-K block (see sw128_offset).
__global__ void k_pack_lp(AdapterSrc src, int K, int r, int r16, int G, uint16_t* __restrict__ Lp, size_t total) {
  const size_t tid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (tid >= total) return;
  const int rl16 = G * r16;
  const int j = static_cast<int>(tid % rl16);
  const size_t k = tid / rl16;
  const int lc = l_column(j, r, r16);
  const uint16_t v = lc >= 0 ? src.l(static_cast<int>(k), j, lc) : static_cast<uint16_t>(0);
  uint8_t* base = reinterpret_cast<uint8_t*>(Lp) + (k / 64) * (size_t)rl16 * 128;
  *reinterpret_cast<uint16_t*>(base + sw128_offset(j, static_cast<int>(k % 64), rl16)) = v;
}

// Empty kernel launched last by slim_pack.  slim_linear's kernels may start
// (and read the packed layer) while the kernel just before them is still
// running; this normally launched kernel starts only after the packing
// kernels have completed, so whatever follows it sees a finished layer.
__global__ void k_pack_done() {}

}  // namespace

cudaError_t launch_pack_done(cudaStream_t s) {
  k_pack_done<<<1, 32, 0, s>>>();
  return cudaGetLastError();
}

cudaError_t launch_pack(const slim_layer& L, const uint16_t* W, cudaStream_t s) {
  NvtxRange nv("pack: quantize, 2:4 prune, canonical bytes and decode stream (k_pack)");
  dim3 grid(L.n_kblocks, L.n_row_tiles);
  k_pack<<<grid, 1024, 0, s>>>(W, L.K, L.N, L.vals, L.meta, L.scales, L.dec, L.n_kblocks, L.status);
  return cudaGetLastError();
}

cudaError_t launch_pack_adapter(const slim_layer& L, const uint16_t* Lsrc, const uint16_t* Rsrc,
                                cudaStream_t s) {
  if (L.r == 0) return cudaSuccess;
  NvtxRange nv("pack: adapter fragments (k_pack_adapter)");
  const size_t total = (size_t)L.rl16 * L.K / 2 + (size_t)L.n_row_tiles * 16 * L.r16 / 2;
  const int threads = 256;
  const size_t blocks = (total + threads - 1) / threads;
  k_pack_adapter<<<static_cast<unsigned>(blocks), threads, 0, s>>>(adapter_src(L, Lsrc, Rsrc), L.K, L.N, L.r,
                                                                    L.r16, L.n_groups,
                                                                    reinterpret_cast<uint32_t*>(L.Lf),
                                                                    reinterpret_cast<uint32_t*>(L.Rf));
  return cudaGetLastError();
}

cudaError_t launch_pack_rp(const slim_layer& L, const uint16_t* Rsrc, cudaStream_t s) {
  if (L.r == 0) return cudaSuccess;
  NvtxRange nv("pack: R^T operand images (k_pack_rp)");
  const int r64 = ceil_div(L.r16, 64) * 64;
  const size_t total = (size_t)ceil_div(L.N, 512) * 512 * r64;
  const int threads = 256;
  k_pack_rp<<<static_cast<unsigned>((total + threads - 1) / threads), threads, 0, s>>>(
      adapter_src(L, nullptr, Rsrc), L.N, L.r, r64, L.Rp, total);
  return cudaGetLastError();
}

cudaError_t launch_pack_lp(const slim_layer& L, const uint16_t* Lsrc, cudaStream_t s) {
  if (L.r == 0) return cudaSuccess;
  NvtxRange nv("pack: L^T operand images (k_pack_lp)");
  const size_t total = (size_t)L.K * L.rl16;
  const int threads = 256;
  k_pack_lp<<<static_cast<unsigned>((total + threads - 1) / threads), threads, 0, s>>>(
      adapter_src(L, Lsrc, nullptr), L.K, L.r, L.r16, L.n_groups, L.Lp, total);
  return cudaGetLastError();
}

cudaError_t launch_quant_adapter(const slim_layer& L, const uint16_t* Lsrc, const uint16_t* Rsrc, cudaStream_t s) {
  if (L.r == 0) return cudaSuccess;
  NvtxRange nv("pack: 4-bit adapter quantization (k_quant_adapter_scales, k_quant_adapter_words)");
  const AdapterShape a = adapter_shape(L);
  const int threads = 256;
  const size_t ns = (size_t)a.JT * 16 * a.KG + (size_t)a.NRT * 16 * a.ngr;
  k_quant_adapter_scales<<<static_cast<unsigned>((ns + threads - 1) / threads), threads, 0, s>>>(Lsrc, Rsrc, a, L.Lq,
                                                                                                 L.Rq, L.status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t nw = (size_t)a.JT * a.KG * 256 + (size_t)a.NRT * a.JS * 32;
  k_quant_adapter_words<<<static_cast<unsigned>((nw + threads - 1) / threads), threads, 0, s>>>(Lsrc, Rsrc, a, L.Lq,
                                                                                                L.Rq);
  return cudaGetLastError();
}

cudaError_t launch_unpack_adapters(const slim_layer& L, int8_t* qL, uint16_t* sL, int8_t* qR, uint16_t* sR,
                                   cudaStream_t s) {
  const AdapterShape a = adapter_shape(L);
  const size_t gr = (size_t)a.G * a.r;
  const size_t total = (size_t)a.K * gr + (size_t)a.KG * gr + (size_t)a.r * a.N + (size_t)a.ngr * a.N;
  const int threads = 256;
  k_unpack_adapters<<<static_cast<unsigned>((total + threads - 1) / threads), threads, 0, s>>>(a, L.Lq, L.Rq, qL, sL,
                                                                                               qR, sR);
  return cudaGetLastError();
}

cudaError_t launch_unpack_dec(const slim_layer& L, int8_t* q, uint16_t* scales, cudaStream_t s) {
  const size_t total = (size_t)L.N * (L.K / 4);
  const int threads = 256;
  const size_t blocks = (total + threads - 1) / threads;
  k_unpack_dec<<<static_cast<unsigned>(blocks), threads, 0, s>>>(L.dec, L.K, L.N, L.n_kblocks, q, scales);
  return cudaGetLastError();
}

}  // namespace slim

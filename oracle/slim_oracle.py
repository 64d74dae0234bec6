"""CPU oracle for the SLiM-style compressed linear layer (test infrastructure).

This module is TEST INFRASTRUCTURE. Only the test-suite, the package's smoke
check and the benchmark's CPU-baseline leg may import it. The product path
(the CUDA library and its Python binding) never imports it, and it imports
nothing from the product package.

It restates, plainly and slowly, what the compressed layer computes:

    Y = X . (dequant(Wq) (.) M_2:4)^T + (X . L) . R

Sources (the thesis "Compression Trinity: Exploring Sparsity, Quantization,
and Low-Rank Approximations for LLM Compression", arXiv:2608.24070, and a
summary page of it):

* Fig. 7.1 caption (SLiM pipeline): weights are first quantized with a
  *symmetric* quantizer, then the *quantized* weights are sparsified by a
  pruning method, then low-rank adapters L, R are added.
* developinglight.com study page, paragraph on the reported setups: SLiM
  uses 4-bit weight-only quantization with group size 128.
* §2.6 "The Compression Trinity as a Solution Framework": quantization is
  applied per group.
* §2.2.3 "Sparse Tensor Core Acceleration": in every contiguous block of 4
  elements along the reduction dimension at least 2 are zero; the non-zeros
  are stored packed, with small metadata indices giving their positions.
* §2.1 "The Transformer Bottleneck: Linear Layers": W is d_out x d_in and the
  forward pass is Y = X W^T.
* §1.2.3 "Low-rank Approximations": W ~ L R with thin factors; §4 (SLoPe,
  lazy low-rank adapters): the adapter product is kept as a separate
  computational path, never added into the sparse weight.

Readings where the pages are silent (each is listed in the design notes):

* scale rule: abs-max per group (the "Group AbsMax" baseline of Table 7.1),
  s = fp16(amax / 7) computed in IEEE fp32 and rounded to nearest-even;
  quantization divides by the *rounded* fp16 scale;
* integer range [-7, 7]; rounding half-to-even, then clip;
* an all-zero group (or a scale that rounds to 0 in fp16) gives q = 0 and a
  stored scale of 0; a scale that is Inf/NaN in fp16 is a range error;
* pruning key |q| (equal to |q.s| within a group); keep the pair (i0 < i1)
  with the largest |q[i0]| + |q[i1]|, ties to the lexicographically smallest
  pair; exactly two kept slots per group of 4, possibly holding zeros;
* quantized adapters (§7.4.3 "Low-rank adapter quantization", named in the
  table of contents; Tables E.13 / E.14 captions say only that Quantized SLiM
  quantizes the adapters too): the weights' quantizer, 4-bit symmetric
  abs-max with fp16 scales, in groups of 128 along each factor's reduction
  dimension (K for L, r for R, the last group shorter when r % 128 != 0);
* 8-bit inputs (W4A8, named by the captions of Tables E.2 / E.5; oracle only,
  not on the CUDA path): symmetric abs-max per token at 8 bits with an fp32
  scale, the integer group sums scaled by the weight group's and the token's
  scales, the adapter on the same dequantized input;
* hybrid tiles (PATCH, Chapter 6 summary; oracle only, not on the CUDA path):
  128 x 128 tiles, each dense or 2:4 by an input flag, quantize first, then
  prune inside the 2:4 tiles only;
* canonical byte format (a C-ABI contract of this library, not of the pages):
  vals[n][K/4]  one byte per group of 4: (v0 & 0xF) | (v1 & 0xF) << 4,
                4-bit two's complement, v0 at i0 and v1 at i1;
  meta[n][K/8]  one nibble per group: i0 | i1 << 2, even group in the low
                nibble;
  scales[n][K/128] IEEE fp16 bit patterns.

All quantization arithmetic is numpy float32 (correctly rounded IEEE ops);
the forward is float64.  Parity of the worked-example values is unpinned by
the pages (they print none); the pins are brute force, closed forms and
invariants in tests/test_oracle_*.py.
"""
from __future__ import annotations

import numpy as np

GROUP = 128
QMAX = 7

# The six ways to keep two of four positions, in lexicographic order.
PAIRS = ((0, 1), (0, 2), (0, 3), (1, 2), (1, 3), (2, 3))


class OracleRangeError(ValueError):
    """A group's fp16 scale is not finite (NaN/Inf input or fp16 overflow)."""


# ---------------------------------------------------------------- bf16 inputs
def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float32."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(bits).astype(np.float64)


# ---------------------------------------------------------------- step 1
def quantize(W32: np.ndarray, group: int = GROUP):
    """Symmetric per-group 4-bit quantization (SLiM pipeline step 1).

    Fig. 7.1 caption (symmetric quantizer), summary page (4-bit, g=128),
    §2.6 (per-group).  Returns (q int8 [N][K], scale fp16 [N][K/group]).
    """
    W32 = np.asarray(W32, dtype=np.float32)
    N, K = W32.shape
    if K % group:
        raise ValueError("K must be a multiple of the group size")
    G = K // group
    Wg = W32.reshape(N, G, group)
    amax = np.max(np.abs(Wg), axis=2)                       # float32, exact
    s32 = np.divide(amax, np.float32(QMAX), dtype=np.float32)  # IEEE fp32 division
    with np.errstate(over="ignore", invalid="ignore"):
        s16 = s32.astype(np.float16)                         # round to nearest even
    if not np.all(np.isfinite(s16)):
        raise OracleRangeError("fp16 group scale is not finite")
    sf = s16.astype(np.float32)
    q = np.zeros((N, G, group), dtype=np.int8)
    nz = sf != 0
    if np.any(nz):
        ratio = np.divide(Wg[nz], sf[nz][:, None], dtype=np.float32)  # IEEE fp32 division
        q[nz] = np.clip(np.rint(ratio), -QMAX, QMAX).astype(np.int8)  # half-to-even, then clip
    return q.reshape(N, K), s16


# ---------------------------------------------------------------- step 2
def prune_2of4(q: np.ndarray):
    """2:4 magnitude pruning of the quantized weights (SLiM step 2).

    §2.2.3: blocks of 4 consecutive elements along the reduction dimension
    (K).  Keeps the pair (i0 < i1) with the largest |q[i0]| + |q[i1]|; ties go
    to the first pair in lexicographic order.  Returns (i0, i1) as int8
    arrays of shape [N][K/4].
    """
    q = np.asarray(q, dtype=np.int8)
    N, K = q.shape
    a = np.abs(q.reshape(N, K // 4, 4).astype(np.int32))
    scores = np.stack([a[..., i] + a[..., j] for (i, j) in PAIRS], axis=-1)
    best = np.argmax(scores, axis=-1)                        # first maximum wins
    pairs = np.array(PAIRS, dtype=np.int8)
    return pairs[best, 0], pairs[best, 1]


def mask_from_pairs(i0: np.ndarray, i1: np.ndarray) -> np.ndarray:
    """Boolean keep-mask [N][K] from the kept positions."""
    N, G4 = i0.shape
    m = np.zeros((N, G4, 4), dtype=bool)
    rows = np.arange(N)[:, None]
    cols = np.arange(G4)[None, :]
    m[rows, cols, i0] = True
    m[rows, cols, i1] = True
    return m.reshape(N, G4 * 4)


# ---------------------------------------------------------------- step 3
def pack(q: np.ndarray, i0: np.ndarray, i1: np.ndarray):
    """Pack kept values and their positions into the canonical byte format."""
    N, K = q.shape
    qg = q.reshape(N, K // 4, 4)
    rows = np.arange(N)[:, None]
    cols = np.arange(K // 4)[None, :]
    v0 = qg[rows, cols, i0].astype(np.int32)
    v1 = qg[rows, cols, i1].astype(np.int32)
    vals = ((v0 & 0xF) | ((v1 & 0xF) << 4)).astype(np.uint8)
    nib = (i0.astype(np.int32) | (i1.astype(np.int32) << 2))
    meta = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    return vals, meta


def pack_layer(W_bits: np.ndarray, group: int = GROUP):
    """bf16 weight bits [N][K] -> canonical (vals, meta, scale_bits)."""
    W32 = bf16_bits_to_f32(W_bits)
    q, s16 = quantize(W32, group)
    i0, i1 = prune_2of4(q)
    vals, meta = pack(q, i0, i1)
    return vals, meta, s16.view(np.uint16)


# ---------------------------------------------------------------- unpack
def unpack(vals: np.ndarray, meta: np.ndarray) -> np.ndarray:
    """Canonical bytes -> dense int8 q [N][K] with zeros at pruned positions."""
    vals = np.asarray(vals, dtype=np.uint8)
    meta = np.asarray(meta, dtype=np.uint8)
    N, G4 = vals.shape
    n0 = (vals & 0xF).astype(np.int32)
    n1 = (vals >> 4).astype(np.int32)
    v0 = np.where(n0 >= 8, n0 - 16, n0)
    v1 = np.where(n1 >= 8, n1 - 16, n1)
    nib = np.empty((N, G4), dtype=np.int32)
    nib[:, 0::2] = meta & 0xF
    nib[:, 1::2] = meta >> 4
    i0 = nib & 3
    i1 = (nib >> 2) & 3
    out = np.zeros((N, G4, 4), dtype=np.int8)
    rows = np.arange(N)[:, None]
    cols = np.arange(G4)[None, :]
    out[rows, cols, i0] = v0
    out[rows, cols, i1] = v1   # i1 != i0 in every valid encoding
    return out.reshape(N, G4 * 4)


def effective_weight(vals, meta, scale_bits, group: int = GROUP) -> np.ndarray:
    """W_eff[n,k] = s[n, k // group] * q[n,k] in float64 (pruned -> 0)."""
    q = unpack(vals, meta).astype(np.float64)
    s = np.asarray(scale_bits, dtype=np.uint16).view(np.float16).astype(np.float64)
    return q * np.repeat(s, group, axis=1)


# ---------------------------------------------------------------- forward
def forward(vals, meta, scale_bits, L_bits, R_bits, X_bits, group: int = GROUP) -> np.ndarray:
    """Y = X W_eff^T + (X L) R in float64.

    §2.1 (Y = X W^T with W of shape d_out x d_in); the adapter product is a
    separate path added to the sparse product (§4, lazy low-rank adapters),
    never merged into W_eff.  L is [K][r], R is [r][N]; r = 0 drops the term.
    """
    W_eff = effective_weight(vals, meta, scale_bits, group)
    X = bf16_bits_to_f64(X_bits)
    Y = X @ W_eff.T
    if L_bits is not None and np.asarray(L_bits).size:
        L = bf16_bits_to_f64(L_bits)
        R = bf16_bits_to_f64(R_bits)
        Y = Y + (X @ L) @ R
    return Y


def adapter_down(L_bits, X_bits) -> np.ndarray:
    """T = X L in float64 (the adapter's first contraction)."""
    return bf16_bits_to_f64(X_bits) @ bf16_bits_to_f64(L_bits)


# ---------------------------------------------------------------- quantized adapters
def quantize_along_rows(F32: np.ndarray, group: int = GROUP):
    """quantize() of each row of F32 [rows][n] in groups of `group`
    consecutive entries, the last group shorter when n % group != 0.

    The short group is padded with zeros before quantize(): a zero changes
    neither the group's abs-max nor any other entry's q, and its own q is 0.
    Returns (q int8 [rows][n], scale fp16 [rows][ceil(n / group)]).
    """
    F32 = np.asarray(F32, dtype=np.float32)
    rows, n = F32.shape
    ng = -(-n // group)
    padded = np.zeros((rows, ng * group), dtype=np.float32)
    padded[:, :n] = F32
    q, s16 = quantize(padded, group)
    return q[:, :n], s16


def quantize_adapters(L_bits, R_bits, group: int = GROUP):
    """Quantized SLiM: the low-rank adapters are quantized too.

    Thesis §7.4.3 "Low-rank adapter quantization" (table of contents) and
    the captions of Tables E.13 / E.14 ("In Quantized SLIM, the low-rank
    adapters are also quantized") say that it is done, not how.  Reading:
    the weights' own quantizer (step 1 above: symmetric abs-max, 4-bit,
    fp16 scales) applied to each factor in groups of `group` along the
    factor's reduction dimension:
      L [K][r]: column j, groups of 128 consecutive k (T = X L sums over k);
      R [r][N]: column n, groups of 128 consecutive j (Y += T R sums over j),
                the last group shorter when r % 128 != 0.
    Returns (qL int8 [K][r], sL fp16 [K/128][r], qR int8 [r][N],
    sR fp16 [ceil(r/128)][N]).
    """
    L32 = bf16_bits_to_f32(L_bits)
    R32 = bf16_bits_to_f32(R_bits)
    qLt, sLt = quantize_along_rows(L32.T, group)
    qRt, sRt = quantize_along_rows(R32.T, group)
    return qLt.T, sLt.T, qRt.T, sRt.T


def dequantize_adapter(q, s16, group: int = GROUP) -> np.ndarray:
    """F[i][c] = s[i // group][c] * q[i][c] in float64 (i: reduction index)."""
    q = np.asarray(q).astype(np.float64)
    s = np.asarray(s16, dtype=np.float16).astype(np.float64)
    return q * np.repeat(s, group, axis=0)[: q.shape[0]]


def forward_quantized_adapters(vals, meta, scale_bits, L_bits, R_bits, X_bits, group: int = GROUP) -> np.ndarray:
    """Y = X W_eff^T + (X L^) R^ in float64, L^ and R^ the dequantized
    quantize_adapters() factors (the same lazy parallel path as forward())."""
    W_eff = effective_weight(vals, meta, scale_bits, group)
    X = bf16_bits_to_f64(X_bits)
    Y = X @ W_eff.T
    if L_bits is not None and np.asarray(L_bits).size:
        qL, sL, qR, sR = quantize_adapters(L_bits, R_bits, group)
        Y = Y + (X @ dequantize_adapter(qL, sL, group)) @ dequantize_adapter(qR, sR, group)
    return Y


# ---------------------------------------------------------------- W4A8 (8-bit inputs)
# Oracle only: the CUDA path does not implement this setting.
QMAX8 = 127


def quantize_activations(X_bits):
    """8-bit input quantization of the W4A8 setting.

    The captions of Tables E.2 / E.5 name "4-bit weight and 8-bit input
    quantization"; the pages give no activation quantizer.  Reading: the
    weights' symmetric abs-max rule at 8 bits, one scale per token (row of
    X): s = fp32(amax / 127) in IEEE fp32 (a per-token scale is computed at
    run time, not stored, so it stays fp32), q = clip(rint(x / s), -127,
    127) with the fp32 quotient rounded half-to-even; an all-zero row gives
    q = 0 and s = 0; a non-finite scale is a range error.  Returns
    (q int8 [M][K], s float32 [M]).
    """
    X = bf16_bits_to_f32(X_bits)
    if X.ndim != 2:
        raise ValueError("X must be [M][K]")
    amax = np.max(np.abs(X), axis=1) if X.shape[1] else np.zeros(X.shape[0], np.float32)
    with np.errstate(over="ignore", invalid="ignore"):
        s = np.divide(amax, np.float32(QMAX8), dtype=np.float32)
    if not np.all(np.isfinite(s)):
        raise OracleRangeError("per-token input scale is not finite")
    q = np.zeros(X.shape, dtype=np.int8)
    nz = s != 0
    if np.any(nz):
        ratio = np.divide(X[nz], s[nz][:, None], dtype=np.float32)
        q[nz] = np.clip(np.rint(ratio), -QMAX8, QMAX8).astype(np.int8)
    return q, s


def forward_w4a8(vals, meta, scale_bits, L_bits, R_bits, X_bits, group: int = GROUP) -> np.ndarray:
    """Y for 4-bit weights and 8-bit inputs, in the order an integer tensor
    core computes it: per token m, output n and weight group g the exact
    integer sum D[m,n,g] = sum over k in g of q_x[m,k] q_w[n,k], then
    Y[m,n] = s_x[m] sum_g s_w[n,g] D[m,n,g] in float64, plus the adapter on
    the same (dequantized) input, (X^ L) R with X^ = s_x q_x (the layer's
    input is quantized once, and the adapter is the lazy parallel path of
    forward()).  Reading of Tables E.2 / E.5 as in quantize_activations().
    """
    qw = unpack(vals, meta).astype(np.int64)
    N, K = qw.shape
    if K % group:
        raise ValueError("K must be a multiple of the group size")
    G = K // group
    sw = np.asarray(scale_bits, dtype=np.uint16).view(np.float16).astype(np.float64)
    qx, sx = quantize_activations(X_bits)
    M = qx.shape[0]
    D = np.einsum("mgk,ngk->mng", qx.astype(np.int64).reshape(M, G, group), qw.reshape(N, G, group))
    Y = sx.astype(np.float64)[:, None] * np.sum(D.astype(np.float64) * sw[None, :, :], axis=2)
    if L_bits is not None and np.asarray(L_bits).size:
        Xh = qx.astype(np.float64) * sx.astype(np.float64)[:, None]
        Y = Y + (Xh @ bf16_bits_to_f64(L_bits)) @ bf16_bits_to_f64(R_bits)
    return Y


# ---------------------------------------------------------------- hybrid tiles (PATCH)
# Oracle only: the CUDA path does not implement this setting.
HYBRID_TILE = 128


def hybrid_effective_weight(W_bits, sparse_tiles, tile: int = HYBRID_TILE, group: int = GROUP) -> np.ndarray:
    """W_eff of a hybrid dense / 2:4 layer in float64.

    Chapter 6 (PATCH) summary: the weight matrix is cut into tiles and each
    tile is either dense or 2:4 sparse (a learned mask, so between 0 % and
    50 % of the weights are pruned), composable with SLiM's quantization and
    adapters.  The pages give neither the tile size nor how the choice is
    stored.  Reading: square tiles of `tile` rows x `tile` K (128, one
    quantization group wide), the per-tile choice an input (sparse_tiles
    [ceil(N/tile)][K/tile], True = 2:4; the learning of the mask is
    training, out of scope); the weights are quantized first as in SLiM
    (step 1), then 2:4-pruned (step 2) inside the sparse tiles only; dense
    tiles keep every quantized value.
    """
    W32 = bf16_bits_to_f32(W_bits)
    N, K = W32.shape
    if K % tile or tile % 4:
        raise ValueError("K must be a multiple of the tile, the tile of 4")
    sparse_tiles = np.asarray(sparse_tiles, dtype=bool)
    if sparse_tiles.shape != (-(-N // tile), K // tile):
        raise ValueError("one flag per (row tile, K tile)")
    q, s16 = quantize(W32, group)
    i0, i1 = prune_2of4(q)
    keep = mask_from_pairs(i0, i1)
    flags = np.repeat(np.repeat(sparse_tiles, tile, axis=0)[:N], tile, axis=1)
    qh = np.where(flags & ~keep, 0, q).astype(np.float64)
    return qh * np.repeat(s16.astype(np.float64), group, axis=1)


def forward_hybrid(W_bits, sparse_tiles, L_bits, R_bits, X_bits, tile: int = HYBRID_TILE,
                   group: int = GROUP) -> np.ndarray:
    """Y = X W_eff^T + (X L) R with the hybrid W_eff (the adapter is the lazy
    parallel path of forward())."""
    X = bf16_bits_to_f64(X_bits)
    Y = X @ hybrid_effective_weight(W_bits, sparse_tiles, tile, group).T
    if L_bits is not None and np.asarray(L_bits).size:
        Y = Y + (X @ bf16_bits_to_f64(L_bits)) @ bf16_bits_to_f64(R_bits)
    return Y


# ---------------------------------------------------------------- acceptance
REL_FRO_TOL = 5e-3
MAX_ABS_TOL = 2e-2


def errors(Y, Y_ref):
    """(relative Frobenius error, max-abs error / max|Y_ref|)."""
    Y = np.asarray(Y, dtype=np.float64)
    Y_ref = np.asarray(Y_ref, dtype=np.float64)
    den = np.linalg.norm(Y_ref)
    amax = np.max(np.abs(Y_ref)) if Y_ref.size else 0.0
    rel = np.linalg.norm(Y - Y_ref) / den if den > 0 else float(np.linalg.norm(Y - Y_ref))
    mab = np.max(np.abs(Y - Y_ref)) / amax if amax > 0 else (float(np.max(np.abs(Y))) if Y.size else 0.0)
    return float(rel), float(mab)


def within_tolerance(Y, Y_ref) -> bool:
    rel, mab = errors(Y, Y_ref)
    return rel <= REL_FRO_TOL and mab <= MAX_ABS_TOL


# ---------------------------------------------------------------- sizes
def canonical_bytes(N: int, K: int, group: int = GROUP) -> int:
    """vals + meta + scales: 0.25 + 0.125 bytes per weight + 2 bytes per group."""
    return N * K // 4 + N * K // 8 + 2 * N * (K // group)

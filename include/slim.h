/*
 * slim.h — C ABI of libslim: the jointly compressed linear layer
 *
 *     Y = X · (dequant(Wq) ⊙ M_2:4)^T + (X · L) · R
 *
 * on one NVIDIA B200 (sm_100a).
 *
 * Where each part of the operation comes from (thesis "Compression Trinity:
 * Exploring Sparsity, Quantization, and Low-Rank Approximations for LLM
 * Compression", arXiv:2608.24070, and a summary page of it):
 *   - SLiM pipeline, Fig. 7.1 caption: symmetric quantization of W first,
 *     then pruning of the *quantized* weights, then low-rank adapters L, R.
 *   - developinglight.com study page, paragraph on the reported setups:
 *     4-bit weight-only quantization, group size 128.
 *   - §2.2.3 "Sparse Tensor Core Acceleration": 2:4 sparsity along the
 *     reduction dimension, non-zeros stored packed with position metadata.
 *   - §2.1 "The Transformer Bottleneck: Linear Layers": W is d_out × d_in and
 *     the forward pass is Y = X W^T.
 *   - §1.2.3 "Low-rank Approximations" and §4 (lazy low-rank adapters): the
 *     adapter is a thin product kept as its own path, never merged into W.
 *
 * Shapes and dtypes.  K = d_in (reduction), N = d_out, r = adapter rank,
 * group = 128 (the only supported value).  Every matrix is row-major:
 *   W [N][K] bf16, L [K][r] bf16, R [r][N] bf16, X [M][K] bf16, Y [M][N] bf16.
 * bf16 and fp16 values are passed as their uint16_t bit patterns.
 *
 * Memory.  Every pointer is DEVICE memory unless its name ends in _host.
 * The library never allocates device memory: the caller owns every buffer
 * (the packed layer, the workspace, inputs and outputs).  Device pointers
 * must be 16-byte aligned.  `stream` is a cudaStream_t passed as void*
 * (NULL = the legacy default stream).  All calls are asynchronous on
 * `stream` unless stated otherwise, and none synchronizes the device.
 *
 * Errors.  Calls return a slim_status.  Argument errors are detected on the
 * host before anything is launched.  Errors found on the device (a
 * non-finite or overflowing fp16 group scale during packing, a bounded wait
 * that gave up) are recorded in the layer's sticky device status word and
 * returned by slim_sync_status().  A failed CUDA call returns SLIM_ERR_CUDA
 * (from every entry point, slim_linear_noalloc included);
 * slim_last_cuda_error() gives the cudaError_t value of the calling host
 * thread's last failure.
 *
 * Bounded waits.  Every wait inside a kernel gives up after about one second
 * of SM clock.  The kernel then records SLIM_ERR_TIMEOUT and never leaves a
 * plausible-looking partial result: the output tiles it owns are written as
 * zeros, and an adapter product X·L it could not finish is written as NaN,
 * so the outputs that use it are NaN.  Treat the whole Y of a call after
 * which slim_sync_status() reports SLIM_ERR_TIMEOUT as invalid.
 *
 * Debug build.  libslim_debug.so (built with -DSLIM_DEBUG) checks the index
 * arithmetic of the kernels' global-memory accesses (chunk, tile, segment,
 * adapter-column and output indices against the layer's and workspace's
 * extents).  A failed check records SLIM_ERR_BOUNDS in the status word and
 * the access is skipped (a skipped copy then ends in a bounded wait), so a
 * bad index never reads or writes outside its buffer.  The release build
 * compiles the checks away.  Host calls are wrapped in NVTX ranges (pack,
 * adapter quantization, each kernel launch) in both builds.
 *
 * Thread safety.  Calls on different layers, or on one layer from one host
 * thread, are safe.  Concurrent slim_linear calls on one layer are safe if
 * they use different workspaces.
 *
 * Concurrency with other kernels.  Where M <= 16 runs as one launch (see
 * slim_linear_launches), the forward is one grid of at most one CTA per SM
 * whose CTAs wait for words written by other CTAs of the same grid, so it
 * needs all of its CTAs resident at once.  Kernels running
 * concurrently on other streams can hold SMs and delay that; a call delayed
 * beyond the wait budget fails as described above (zeros, SLIM_ERR_TIMEOUT).
 * Results never depend on timing otherwise.
 */
#ifndef SLIM_H_
#define SLIM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SLIM_GROUP 128
#define SLIM_ABI_VERSION 3
/* Most linears one packed layer can fuse (see slim_grouped_layer_init). */
#define SLIM_MAX_GROUPS 8

typedef enum slim_status {
  SLIM_OK = 0,
  SLIM_ERR_ARG = -1,         /* null pointer, negative size, bad enum */
  SLIM_ERR_ALIGN = -2,       /* a pointer is not 16-byte aligned */
  SLIM_ERR_SHAPE = -3,       /* K not a multiple of 128, group != 128, N < 1, r < 0, too large */
  SLIM_ERR_WORKSPACE = -4,   /* workspace missing or smaller than slim_workspace_bytes() */
  SLIM_ERR_RANGE = -5,       /* device: NaN/Inf weight or fp16 group-scale overflow */
  SLIM_ERR_TIMEOUT = -6,     /* device: a bounded wait inside a kernel gave up */
  SLIM_ERR_CUDA = -7,        /* a CUDA runtime call failed */
  SLIM_ERR_UNSUPPORTED = -8, /* device is not sm_100 */
  SLIM_ERR_STATE = -9,       /* layer descriptor not initialised by slim_layer_init */
  SLIM_ERR_BOUNDS = -10      /* device, debug build only: a kernel's index check failed */
} slim_status;

/*
 * Packed layer descriptor.  A plain struct filled by slim_layer_init(); the
 * pointers all point into ONE caller-owned device buffer of
 * slim_layer_bytes() bytes.  Treat the fields as read-only.
 *
 * Canonical packed format (the library's interchange format, bit-exact with
 * the CPU oracle):
 *   vals   [N][K/4]   one byte per group of 4 consecutive K elements:
 *                     (v0 & 0xF) | (v1 & 0xF) << 4, 4-bit two's complement,
 *                     v0 the kept value at position i0, v1 at i1 (i0 < i1);
 *   meta   [N][K/8]   one nibble per group of 4: i0 | i1 << 2; the even
 *                     group of a pair sits in the low nibble;
 *   scales [N][K/128] fp16 bit patterns, one per row and 128-group.
 * Derived layouts (byte permutations of the same information that the
 * kernels stream; their format is internal and may change between versions):
 *   dec    decode-kernel stream, [ceil(N/16)][ceil(K/256)][1600 B];
 *   Lf, Rf the adapter L and R in tensor-core fragment order (bf16);
 *   Rp     R^T in 128-row tiles, in the 128-byte-swizzled shared-memory
 *          image the prefill kernel's tensor-core operand uses (bf16);
 *   Lp     L^T as 128-byte-swizzled images of 64 K each (bf16), the operand
 *          of the prefill path's X·L;
 *   Lq, Rq L^T and R^T as 4-bit tensor-core fragments with their fp16
 *          scales (written only when adapter_bits == 4).
 */
typedef struct slim_layer {
  uint32_t magic;            /* set by slim_layer_init */
  int32_t K, N, r, group;    /* N: all rows; r: the adapter rank of each fused linear */
  int32_t r16;               /* r rounded up to a multiple of 16 */
  int32_t n_groups;          /* linears fused in this layer (1 for a plain layer) */
  int32_t group_end[SLIM_MAX_GROUPS];  /* group g owns rows [group_end[g-1], group_end[g]) */
  int32_t rl16;              /* n_groups * r16: adapter columns of T = X L */
  int32_t n_row_tiles;       /* ceil(N/16) */
  int32_t n_kblocks;         /* ceil(K/256) */
  void* base;                /* the caller's device buffer */
  size_t bytes;
  uint8_t* vals;
  uint8_t* meta;
  uint16_t* scales;
  uint8_t* dec;
  uint16_t* Lf;              /* NULL when r == 0 */
  uint16_t* Rf;              /* NULL when r == 0 */
  uint16_t* Rp;              /* NULL when r == 0 */
  uint16_t* Lp;              /* NULL when r == 0 */
  int32_t* status;           /* sticky device status word (0 = ok) */
  uint8_t* Lq;               /* 4-bit adapter layouts; NULL when r == 0 */
  uint8_t* Rq;
  int32_t adapter_bits;      /* 16 (bf16 adapters, the default) or 4; see slim_layer_set_adapter_bits */
} slim_layer;

/* Host-only.  Bytes of device memory a packed layer of this shape needs
 * (0 on a bad shape). */
size_t slim_layer_bytes(int K, int N, int r, int group);

/* Host-only.  A grouped layer fuses G <= SLIM_MAX_GROUPS linears that read
 * the same X (for example the q, k and v projections, or gate and up):
 *   W stacks their rows, [N_0 + ... + N_{G-1}][K];
 *   L puts their adapter factors side by side, [K][G*r] (linear g's L in
 *     columns [g*r, (g+1)*r));
 *   R puts theirs side by side along N, [r][N];
 * and output row n of linear g is X W_g^T + (X L_g) R_g, exactly what G
 * separate layers compute.  Every N_g but the last must be a multiple of 256
 * (the prefill tile); all use the same r.  This is not in the thesis: it
 * packs several of its compressed linears into one call so that a decoder
 * block pays one launch per group of linears that share an input.
 * slim_layer_bytes / slim_layer_init are the G = 1 case. */
size_t slim_grouped_layer_bytes(int K, int G, const int32_t* N_list, int r, int group);
slim_status slim_grouped_layer_init(slim_layer* layer, int K, int G, const int32_t* N_list, int r, int group,
                                    void* dev_buf, size_t bytes, void* stream);

/* Host-only.  Carves `dev_buf` (device memory, >= slim_layer_bytes(),
 * 1024-byte aligned) into the layer's sub-buffers and fills `layer`.  Clears
 * the device status word with an asynchronous memset on `stream`. */
slim_status slim_layer_init(slim_layer* layer, int K, int N, int r, int group,
                            void* dev_buf, size_t bytes, void* stream);

/* Pack a dense layer (SLiM steps: quantize, 2:4-prune the quantized weights,
 * pack; the adapter is copied into the kernels' layouts).
 *   W [N][K] bf16 (device), L [K][r] bf16, R [r][N] bf16 (device; both NULL
 *   iff r == 0).  For a grouped layer L is [K][G*r] (see
 *   slim_grouped_layer_init).
 * Per row n and 128-group g, in IEEE fp32: amax = max|W|, s = fp16_rn(amax/7)
 * (stored), q = clip(rint(W / s), -7, 7) (q = 0 when s == 0); per 4-group
 * keep the pair i0 < i1 with the largest |q[i0]| + |q[i1]| (ties to the first
 * pair in lexicographic order).  A NaN/Inf weight or an fp16 scale overflow
 * sets SLIM_ERR_RANGE in the device status word.  Deterministic: the same
 * input always gives the same bytes. */
slim_status slim_pack(const slim_layer* layer, const uint16_t* W, const uint16_t* L,
                      const uint16_t* R, void* stream);

/* Host-only.  Choose how slim_pack stores the adapter of an initialised
 * layer: bits = 16 (bf16 L and R, the default after slim_layer_init) or 4
 * ("Quantized SLiM", in which the low-rank adapters are quantized too:
 * thesis §7.4.3 "Low-rank adapter quantization" and the captions of Tables
 * E.13 / E.14).  With 4, slim_pack quantizes L and R with the weights'
 * quantizer: per column of L and 128 consecutive k, and per column of R and
 * 128 consecutive j (the last group shorter when r % 128 != 0), in IEEE
 * fp32 amax = max|v|, s = fp16_rn(amax / 7), q = clip(rint(v / s), -7, 7)
 * (q = 0 when s == 0); a NaN/Inf value or an fp16 scale overflow sets
 * SLIM_ERR_RANGE.  The forward then computes X·W_eff^T + (X·L^)·R^ with
 * L^ = q_L·s_L and R^ = q_R·s_R: the single-launch decode kernel (M <= 16)
 * streams the 4-bit factors (about a quarter of the bf16 adapter bytes),
 * the other kernels read bf16 images of L^ and R^ (each q·s rounded to
 * bf16).  Takes effect at the next slim_pack, which must follow before the
 * next forward.  Errors: SLIM_ERR_STATE (descriptor), SLIM_ERR_ARG (bits
 * other than 4 or 16). */
slim_status slim_layer_set_adapter_bits(slim_layer* layer, int bits);

/* Test aid: expand the 4-bit adapter layouts of a layer packed with
 * adapter_bits == 4 back into q_L int8 [K][G*r], s_L fp16 [K/128][G*r],
 * q_R int8 [r][N] and s_R fp16 [ceil(r/128)][N] (device), so they can be
 * compared with the oracle's quantization.  Errors: SLIM_ERR_STATE
 * (descriptor, or adapters not 4-bit, or r == 0), SLIM_ERR_ARG, SLIM_ERR_ALIGN
 * (every pointer 16-byte aligned). */
slim_status slim_unpack_adapters(const slim_layer* layer, int8_t* qL, uint16_t* sL, int8_t* qR,
                                 uint16_t* sR, void* stream);

/* Host-only.  Device workspace bytes slim_linear needs for any M' <= M
 * tokens: a workspace sized for M serves every smaller M (the size never
 * decreases with M; it is 0 when r == 0 and M <= 16).  The workspace holds a
 * small control block, the adapter's T = X·L and fp32 partial sums (for
 * M <= 16: of X·L slices and, for long K, of K panels), or, for M > 16, T and
 * the dequantized weight tiles of the tensor-core path (needed with r == 0
 * too).  Zero-fill it once before its first use (for example
 * with cudaMemsetAsync); every call leaves it ready for the next call,
 * whatever layer that call is for.  Calls that may overlap on the GPU need
 * separate workspaces. */
size_t slim_workspace_bytes(const slim_layer* layer, int M);

/* Forward: Y[M][N] = X[M][K] · W_eff^T + (X · L) · R, bf16 in and out, fp32
 * accumulation.  X and Y are device pointers and must not overlap.  M == 0
 * is a no-op.  The workspace (device, >= slim_workspace_bytes(layer, M),
 * zero-filled before its first use) is scratch for the adapter and partial
 * sums.  For M <= 16 one kernel streams the packed layer and computes the
 * adapter in the same launch (at most one CTA per SM, all resident at once),
 * except for layers of about 8 MB (2048 up to 64 x SMs 16-row x 256-K chunks,
 * with an adapter) and shapes whose single-launch plan does not fit, which
 * take two token-tiled kernels (X·L, then the main product); for M > 16 the
 * tensor-core path runs (see slim_linear_launches).  Results
 * are deterministic: every sum is taken in a fixed order.
 * Overlap: the kernels are launched with programmatic dependent launch, so
 * they may start while the previous kernel on `stream` is still running and
 * read the (constant) packed layer before it finishes; X, the workspace and
 * Y are touched only after it has completed.  So the kernel immediately
 * before slim_linear on `stream` must not write the packed layer
 * (slim_pack ends with an empty kernel for this reason). */
slim_status slim_linear(const slim_layer* layer, const uint16_t* X, int M, uint16_t* Y,
                        void* workspace, size_t ws_bytes, void* stream);

/* Host-only.  Number of kernels one slim_linear call launches for M tokens
 * on the current device (0 for M == 0, -1 for an invalid descriptor or
 * M < 0).  Not part of the thesis: it lets callers size CUDA graphs and
 * count launches. */
int slim_linear_launches(const slim_layer* layer, int M);

/* Host-only.  Device workspace bytes slim_linear_host needs: the
 * slim_linear workspace plus device staging for X and Y. */
size_t slim_host_workspace_bytes(const slim_layer* layer, int M);

/* Forward on HOST buffers: copies X_host (M×K bf16, ideally pinned) to the
 * device, runs slim_linear, copies Y back to Y_host (M×N bf16) and waits for
 * `stream` to finish.  Synchronous. */
slim_status slim_linear_host(const slim_layer* layer, const uint16_t* X_host, int M,
                             uint16_t* Y_host, void* workspace, size_t ws_bytes, void* stream);

/* slim_linear_host without the wait: enqueues on `stream` the copy of X_host
 * to the device staging area in `workspace`, the forward and the copy of Y
 * back to Y_host, then returns.  X_host must stay unmodified and Y_host
 * unread until the stream has passed this call (cudaStreamSynchronize or an
 * event); with pageable host memory CUDA may copy synchronously.  Calls on
 * one stream may share one workspace; calls on different streams need their
 * own.  Same arguments, sizes and errors as slim_linear_host. */
slim_status slim_linear_host_async(const slim_layer* layer, const uint16_t* X_host, int M,
                                   uint16_t* Y_host, void* workspace, size_t ws_bytes, void* stream);

/* Test aid for the failure path of the kernels' waits.  Launches one
 * thread that waits, with the same bounded wait the forward's kernels use,
 * on a barrier that nothing completes, for about `wait_us` microseconds of
 * SM clock (capped at the forward's wait budget, about one second); the
 * wait gives up and records SLIM_ERR_TIMEOUT in the layer's status word, as
 * a kernel of the forward would.  slim_sync_status() then returns that code
 * and clears it; the CUDA context stays usable.  Asynchronous on `stream`.
 * Errors: SLIM_ERR_STATE (descriptor), SLIM_ERR_ARG (wait_us < 0). */
slim_status slim_test_wait_timeout(const slim_layer* layer, int wait_us, void* stream);

/* Test aid for the store-on-timeout rule of the single-launch decode kernel
 * (M <= 16 tokens, r > 0, a layer and M that slim_linear_launches() reports
 * as one launch).  Runs that kernel exactly as slim_linear would, except
 * that its CTAs wait, for about `wait_us` microseconds of SM clock each, for
 * adapter partial sums tagged for the NEXT launch, which no CTA writes: every
 * such wait gives up, every output tile is written as zeros and
 * SLIM_ERR_TIMEOUT is recorded in the layer's status word.  The workspace
 * must be one slim_linear could use for this M; it is left ready for the
 * next call.  Errors: SLIM_ERR_ARG (M outside 1..16, r == 0, wait_us < 0),
 * SLIM_ERR_UNSUPPORTED (this shape and M do not use the single-launch
 * kernel), SLIM_ERR_WORKSPACE, SLIM_ERR_ALIGN, SLIM_ERR_STATE. */
slim_status slim_test_stream_timeout(const slim_layer* layer, const uint16_t* X, int M, uint16_t* Y,
                                     void* workspace, size_t ws_bytes, int wait_us, void* stream);

/* Test aid: expand the DECODE stream layout back into dense int8 q [N][K]
 * (zeros at pruned positions) and fp16 scales [N][K/128] (device), so the
 * derived layout can be checked against the canonical one. */
slim_status slim_unpack_dec(const slim_layer* layer, int8_t* q_dense, uint16_t* scales,
                            void* stream);

/* Forward for callers that cannot allocate device memory.  This entry point
 * has no counterpart in the thesis; it exists for callers that own no
 * allocator or must not call one (a plugin inside an inference engine whose
 * device memory is planned up front, code where cudaMalloc is not allowed or
 * would synchronize the device) and so cannot hand slim_linear its
 * workspace.  It computes exactly what slim_linear computes, with the
 * adapter's X·L scratch kept in a fixed array inside the library:
 *   - the array holds SLIM_NOALLOC_SCRATCH_BYTES bytes on every GPU that
 *     loads the library, until the process exits;
 *   - M <= 16 runs on the single-launch decode kernel when its workspace
 *     fits the array, every other M on the token-tiled decode kernels (the
 *     tensor-core prefill path needs a workspace for dequantized weights
 *     that would not fit); the token-tiled kernels need a 256-byte control
 *     block plus ceil(M/16)·16 · r16 · 2 bytes for the adapter's X·L (r16 =
 *     r rounded up to 16); a larger request returns SLIM_ERR_WORKSPACE and
 *     launches nothing (M <= 1008 at r = 128, M <= 496 at r = 256);
 *   - every call on a device shares the one array and leaves its contents
 *     behind; the control block starts at zero (the array is zero when the
 *     library loads) and every call leaves it ready for the next one; calls
 *     that overlap on the GPU (other streams, other host threads) race on
 *     the array, so keep them ordered;
 *   - the first call on each device looks up the array's device address
 *     with that device current; make that first call before any stream
 *     capture.
 * It allocates nothing: no cudaMalloc, no cudaFree, no allocating library
 * routine.  X, Y, M and `stream` are as for slim_linear. */
#define SLIM_NOALLOC_SCRATCH_BYTES (256u * 1024u)
slim_status slim_linear_noalloc(const slim_layer* layer, const uint16_t* X, int M, uint16_t* Y,
                                void* stream);

/* Host-only, synchronizing.  Waits for `stream`, returns the sticky device
 * status (SLIM_OK, SLIM_ERR_RANGE or SLIM_ERR_TIMEOUT) and clears it. */
slim_status slim_sync_status(const slim_layer* layer, void* stream);

/* Host-only.  The library reads its tuning variables (SLIM_NO_STREAM,
 * SLIM_STREAM_WARPS, SLIM_PDL_EARLY, SLIM_DECODE_CFG, SLIM_NO_PREFILL,
 * SLIM_PREFILL_1SM, SLIM_PREFILL_TILE: which kernels and tiles a call
 * uses, for tuning and tests) from the environment once, at its first call,
 * and plans every (layer shape, M) once.  This re-reads them and makes the
 * following calls plan again.  Not to be called while another host thread
 * is inside the library. */
void slim_tuning_reload(void);

/* Host-only. */
const char* slim_status_string(slim_status s);
int slim_last_cuda_error(void);
int slim_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SLIM_H_ */

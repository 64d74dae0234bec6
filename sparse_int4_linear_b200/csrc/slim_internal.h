// Internal launch wrappers shared by the host API (not part of the C ABI).
#pragma once
#include <cuda_runtime.h>
#include <cstdint>
#include <cstddef>

#include "slim.h"

namespace slim {

cudaError_t launch_pack(const slim_layer& L, const uint16_t* W, cudaStream_t s);
cudaError_t launch_pack_adapter(const slim_layer& L, const uint16_t* Lsrc, const uint16_t* Rsrc,
                                cudaStream_t s);
cudaError_t launch_pack_done(cudaStream_t s);
cudaError_t launch_unpack_dec(const slim_layer& L, int8_t* q, uint16_t* scales, cudaStream_t s);

// Adapter down-projection T = X L into `T` (bf16 [ceil(M/16)*16][r16]).
cudaError_t launch_adapter_down(const slim_layer& L, const uint16_t* X, int M, uint16_t* T,
                                cudaStream_t s);
// Sparse int4 main product plus the adapter up-projection, bf16 Y.
cudaError_t launch_decode(const slim_layer& L, const uint16_t* X, int M, uint16_t* Y, const uint16_t* T,
                          cudaStream_t s);

// The forward: tensor-core prefill (M > 16, when allowed), the single-launch
// streaming decode (M <= 16, when its plan fits and its workspace fits
// `ws_limit`), else the token-tiled adapter-down + decode pair.  `ws` must be
// zero-filled before its first use (the streaming kernel keeps a control
// block at its start).
size_t forward_ctl_bytes(int r16);
// `allow_prefill` false keeps M > 16 on the token-tiled decode kernels (no
// dequantized-image workspace).
size_t forward_workspace_bytes(const slim_layer& L, int M, bool allow_prefill, size_t ws_limit = SIZE_MAX);
cudaError_t launch_forward(const slim_layer& L, const uint16_t* X, int M, uint16_t* Y, void* ws, bool allow_prefill,
                           size_t ws_limit, cudaStream_t s);

// Kernels one launch_forward call launches.
int forward_launches(const slim_layer& L, int M, bool allow_prefill, size_t ws_limit = SIZE_MAX);

// Single-launch streaming decode (M <= 16).
bool stream_supported(const slim_layer& L, int M);
size_t stream_workspace_bytes(const slim_layer& L, int M);
cudaError_t launch_stream(const slim_layer& L, const uint16_t* X, int M, uint16_t* Y, void* ws, cudaStream_t s);

// Bytes of the pre-swizzled R^T image: 128-row tiles x ceil(r16/64) atoms,
// padded to whole 512-row blocks (the largest prefill CTA-pair tile).
inline size_t rp_bytes(int N, int r16) {
  return r16 > 0 ? (size_t)((N + 511) / 512) * 4 * 128 * (size_t)((r16 + 63) / 64) * 64 * 2 : 0;
}
cudaError_t launch_pack_rp(const slim_layer& L, const uint16_t* Rsrc, cudaStream_t s);
cudaError_t launch_pack_lp(const slim_layer& L, const uint16_t* Lsrc, cudaStream_t s);
// T = X L on the tensor cores into the prefill kernel's swizzled T tiles.
cudaError_t launch_tgemm(const slim_layer& L, const uint16_t* X, int M, uint16_t* Tswz, cudaStream_t s);

// Tensor-core prefill forward (M > 16): the dequantized weight images go to
// `img` (prefill_image_bytes(N, K) bytes of workspace).
int prefill_tokens_per_tile(const slim_layer& L, int M);
constexpr int kPrefillMaxTile = 240;   // widest token tile of the prefill kernels
size_t prefill_image_bytes(int N, int K);
cudaError_t launch_prefill(const slim_layer& L, const uint16_t* X, int M, uint16_t* Y, const uint16_t* Tswz,
                           uint8_t* img, cudaStream_t s);

// Number of SMs of the current device (cached).
int num_sms();
// Test aid: a one-thread wait on a barrier nothing completes, bounded by
// about wait_us of SM clock (at most the forward's wait budget); records
// SLIM_ERR_TIMEOUT in `status`.
cudaError_t launch_wait_probe(int32_t* status, int wait_us, cudaStream_t s);
// Raise `func`'s dynamic shared-memory limit to at least `smem` bytes (and
// allow cluster sizes above 8 when asked) on the current device.  Function
// attributes belong to a (kernel, device); what was set is remembered per
// pair under a lock, so concurrent first calls from several host threads,
// or one thread driving several GPUs, each get them set.
cudaError_t ensure_func_attrs(const void* func, size_t smem, bool nonportable_cluster = false);

}  // namespace slim

// Internal launch wrappers shared by the host API (not part of the C ABI).
#pragma once
#include <cuda_runtime.h>
#include <cstdint>

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

// The forward (dispatch between the fused single-launch decode kernel and
// the adapter-down + decode pair).  `ws` holds a control block followed by
// T; it must be zero-filled before its first use.
size_t forward_ctl_bytes(int r16);
size_t forward_workspace_bytes(int r16, int M);
cudaError_t launch_forward(const slim_layer& L, const uint16_t* X, int M, uint16_t* Y, void* ws, cudaStream_t s);

// Bytes of the pre-swizzled R^T image (128-row tiles x ceil(r16/64) atoms).
inline size_t rp_bytes(int N, int r16) {
  return r16 > 0 ? (size_t)((N + 127) / 128) * 128 * (size_t)((r16 + 63) / 64) * 64 * 2 : 0;
}
cudaError_t launch_pack_rp(const slim_layer& L, const uint16_t* Rsrc, cudaStream_t s);

// Adapter down-projection into the swizzled B-operand image used by the
// prefill kernel: 128-token tiles x ceil(r16/64) atoms.
cudaError_t launch_adapter_down_swz(const slim_layer& L, const uint16_t* X, int M, uint16_t* Tswz,
                                    cudaStream_t s);
// Tensor-core prefill forward (M > 16).
cudaError_t launch_prefill(const slim_layer& L, const uint16_t* X, int M, uint16_t* Y, const uint16_t* Tswz,
                           cudaStream_t s);

// Number of SMs of the current device (cached).
int num_sms();

}  // namespace slim

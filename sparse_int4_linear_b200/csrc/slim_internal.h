// Internal launch wrappers shared by the host API (not part of the C ABI).
#pragma once
#include <cuda_runtime.h>
#include <array>
#include <cstdint>
#include <cstddef>
#include <map>
#include <shared_mutex>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "slim.h"

namespace slim {

// An NVTX range over a scope of host code (a call, a pack step, a kernel
// launch); a no-op unless a profiler is attached.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Tuning knobs, read from the environment at the library's first call and
// again by slim_tuning_reload():
//   SLIM_NO_STREAM      M <= 16 never uses the single-launch kernel
//   SLIM_STREAM_WARPS   8 or 16 main warps in the single-launch kernel
//   SLIM_PDL_EARLY      the single-launch kernel signals the next launch early
//   SLIM_DECODE_CFG     "WR,KW,S" forces the token-tiled decode kernel's split
//   SLIM_NO_PREFILL     M > 16 stays on the token-tiled decode kernels
//   SLIM_PREFILL_1SM    the prefill path never uses SM pairs
//   SLIM_PREFILL_TILE   "halves,tokens" or "pair,tokens" forces a prefill tile
struct Tuning {
  bool no_stream = false, no_prefill = false, prefill_1sm = false, pdl_early = false;
  int stream_warps = 0;                      // 0: chosen per call
  bool decode_cfg = false;
  int dec_wr = 0, dec_kw = 0, dec_s = 0;
  bool prefill_tile = false, prefill_pair = false;
  int prefill_nh = 0, prefill_tt = 0;
  unsigned generation = 0;                   // bumped by every reload; part of every plan-cache key
};
Tuning tuning();
void reload_tuning();

// Thread-safe memo of host-side plans.  Keys hold the device, the tuning
// generation and every input the plan depends on.
template <size_t N, class V>
class PlanCache {
 public:
  using Key = std::array<long long, N>;
  template <class F>
  V get(const Key& k, F&& make) {
    {
      std::shared_lock<std::shared_mutex> lock(mu_);
      auto it = map_.find(k);
      if (it != map_.end()) return it->second;
    }
    V v = make();
    std::unique_lock<std::shared_mutex> lock(mu_);
    map_.emplace(k, v);
    return v;
  }

 private:
  std::shared_mutex mu_;
  std::map<Key, V> map_;
};

// The calling thread's current CUDA device (-1 if it cannot be read).
int current_device();
// Record a failed CUDA call for slim_last_cuda_error() (per host thread).
void set_last_cuda_error(cudaError_t e);
int last_cuda_error();

cudaError_t launch_pack(const slim_layer& L, const uint16_t* W, cudaStream_t s);
cudaError_t launch_pack_adapter(const slim_layer& L, const uint16_t* Lsrc, const uint16_t* Rsrc,
                                cudaStream_t s);
cudaError_t launch_pack_done(cudaStream_t s);
// 4-bit adapters (layer.adapter_bits == 4): quantize L and R into Lq / Rq.
// The bf16 layouts (Lf, Rf, Rp, Lp) packed after it then hold the
// dequantized values.
cudaError_t launch_quant_adapter(const slim_layer& L, const uint16_t* Lsrc, const uint16_t* Rsrc, cudaStream_t s);
cudaError_t launch_unpack_adapters(const slim_layer& L, int8_t* qL, uint16_t* sL, int8_t* qR, uint16_t* sR,
                                   cudaStream_t s);
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
// The most forward_workspace_bytes gives for any M' in [1, M].
size_t forward_workspace_bytes_upto(const slim_layer& L, int M, bool allow_prefill, size_t ws_limit = SIZE_MAX);
cudaError_t launch_forward(const slim_layer& L, const uint16_t* X, int M, uint16_t* Y, void* ws, bool allow_prefill,
                           size_t ws_limit, cudaStream_t s);

// Kernels one launch_forward call launches.
int forward_launches(const slim_layer& L, int M, bool allow_prefill, size_t ws_limit = SIZE_MAX);

// Single-launch streaming decode (M <= 16).
bool stream_supported(const slim_layer& L, int M);
size_t stream_workspace_bytes(const slim_layer& L, int M);
cudaError_t launch_stream(const slim_layer& L, const uint16_t* X, int M, uint16_t* Y, void* ws, cudaStream_t s);
// The same with the budget of the waits for T partials in SM cycles, and
// readers that expect the tag of launch seq + tag_skew (a test aid: with
// tag_skew = 1 no CTA writes what they wait for, so every wait gives up).
cudaError_t launch_stream_ex(const slim_layer& L, const uint16_t* X, int M, uint16_t* Y, void* ws,
                             long long t_wait_cycles, uint32_t tag_skew, cudaStream_t s);

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

// Number of SMs of the current device (cached per device).
int num_sms();
// Compute-capability major of the current device (cached per device; -1 on error).
int device_cc_major();
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

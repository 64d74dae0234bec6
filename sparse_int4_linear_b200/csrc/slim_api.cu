// Host side of the C ABI declared in include/slim.h: argument checks, the
// packed-layer memory map, dispatch, and status reporting.
#include <algorithm>
#include <cstring>

#include "slim_common.cuh"
#include "slim_internal.h"

namespace {

slim_status cuda_fail(cudaError_t e) {
  slim::set_last_cuda_error(e);
  return SLIM_ERR_CUDA;
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Packed-layer memory map (offsets into one buffer, each 256-byte aligned).
struct LayerMap {
  size_t vals, meta, scales, dec, Lf, Rf, Rp, Lp, Lq, Rq, status, total;
};

bool shape_ok(int K, int N, int r, int group) {
  if (group != SLIM_GROUP) return false;
  if (K <= 0 || K % SLIM_GROUP != 0 || N <= 0 || r < 0) return false;
  if (K > (1 << 20) || N > (1 << 20) || r > 4096) return false;
  return true;
}

// Group row counts: 1..SLIM_MAX_GROUPS positive counts, all but the last a
// multiple of 256; total N and the adapter columns within the limits.
bool groups_ok(int K, int G, const int32_t* N_list, int r, int group, int* N_out) {
  if (G < 1 || G > SLIM_MAX_GROUPS || !N_list) return false;
  long long N = 0;
  for (int g = 0; g < G; ++g) {
    if (N_list[g] <= 0) return false;
    if (g + 1 < G && N_list[g] % 256 != 0) return false;
    N += N_list[g];
  }
  if (N > (1 << 20) || (long long)G * slim::ceil_div(r, 16) * 16 > 4096) return false;
  if (!shape_ok(K, (int)N, r, group)) return false;
  *N_out = (int)N;
  return true;
}

// rl16: adapter columns of T over all groups (G * r16).
LayerMap layer_map(int K, int N, int r, int rl16) {
  const size_t nrt = (size_t)slim::ceil_div(N, 16), nkb = (size_t)slim::ceil_div(K, 256);
  const size_t r16 = (size_t)slim::ceil_div(r, 16) * 16;
  LayerMap m;
  size_t off = 0;
  m.vals = off;   off = align_up(off + (size_t)N * K / 4, 256);
  m.meta = off;   off = align_up(off + (size_t)N * K / 8, 256);
  m.scales = off; off = align_up(off + (size_t)N * (K / SLIM_GROUP) * 2, 256);
  m.dec = off;    off = align_up(off + nrt * nkb * slim::kDecChunk, 1024);
  m.Lf = off;     off = align_up(off + (size_t)rl16 * K * 2, 256);
  m.Rf = off;     off = align_up(off + nrt * 16 * r16 * 2, 256);
  m.Rp = off;     off = align_up(off + slim::rp_bytes(N, (int)r16), 1024);
  m.Lp = off;     off = align_up(off + (size_t)K * rl16 * 2, 1024);
  m.Lq = off;     off = align_up(off + (size_t)(rl16 / 16) * (K / SLIM_GROUP) * slim::kLqBlock, 256);
  m.Rq = off;     off = align_up(off + nrt * (r16 ? slim::rq_tile_bytes((int)r16, r) : 0), 256);
  m.status = off; off = align_up(off + 16, 256);
  m.total = off;
  return m;
}

bool layer_ok(const slim_layer* L) {
  return L && L->magic == slim::kLayerMagic && L->base && L->status;
}

// Exact workspace need of one call with M tokens.
size_t t_bytes(const slim_layer* L, int M) { return slim::forward_workspace_bytes(*L, M, true); }
// What slim_workspace_bytes reports: enough for every M' <= M (the decode
// paths of small M can need more than a larger M does).
size_t t_bytes_upto(const slim_layer* L, int M) { return slim::forward_workspace_bytes_upto(*L, M, true); }

// The current device must be an sm_100 part (checked once per device).
slim_status check_device() {
  const int major = slim::device_cc_major();
  if (major < 0) return SLIM_ERR_CUDA;
  return major == 10 ? SLIM_OK : SLIM_ERR_UNSUPPORTED;
}

}  // namespace

extern "C" {

size_t slim_grouped_layer_bytes(int K, int G, const int32_t* N_list, int r, int group) {
  int N = 0;
  if (!groups_ok(K, G, N_list, r, group, &N)) return 0;
  return layer_map(K, N, r, G * slim::ceil_div(r, 16) * 16).total;
}

size_t slim_layer_bytes(int K, int N, int r, int group) {
  const int32_t n[1] = {N};
  return slim_grouped_layer_bytes(K, 1, n, r, group);
}

slim_status slim_grouped_layer_init(slim_layer* layer, int K, int G, const int32_t* N_list, int r, int group,
                                    void* dev_buf, size_t bytes, void* stream) {
  if (!layer || !dev_buf) return SLIM_ERR_ARG;
  int N = 0;
  if (!groups_ok(K, G, N_list, r, group, &N)) return SLIM_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(dev_buf) & 1023u) != 0) return SLIM_ERR_ALIGN;
  const int r16 = slim::ceil_div(r, 16) * 16;
  const LayerMap m = layer_map(K, N, r, G * r16);
  if (bytes < m.total) return SLIM_ERR_WORKSPACE;
  uint8_t* b = static_cast<uint8_t*>(dev_buf);
  std::memset(layer, 0, sizeof(*layer));
  layer->K = K;
  layer->N = N;
  layer->r = r;
  layer->group = group;
  layer->r16 = r16;
  layer->n_groups = G;
  int end = 0;
  for (int g = 0; g < SLIM_MAX_GROUPS; ++g) {
    if (g < G) end += N_list[g];
    layer->group_end[g] = end;
  }
  layer->rl16 = G * r16;
  layer->n_row_tiles = slim::ceil_div(N, 16);
  layer->n_kblocks = slim::ceil_div(K, 256);
  layer->base = dev_buf;
  layer->bytes = bytes;
  layer->vals = b + m.vals;
  layer->meta = b + m.meta;
  layer->scales = reinterpret_cast<uint16_t*>(b + m.scales);
  layer->dec = b + m.dec;
  layer->Lf = r ? reinterpret_cast<uint16_t*>(b + m.Lf) : nullptr;
  layer->Rf = r ? reinterpret_cast<uint16_t*>(b + m.Rf) : nullptr;
  layer->Rp = r ? reinterpret_cast<uint16_t*>(b + m.Rp) : nullptr;
  layer->Lp = r ? reinterpret_cast<uint16_t*>(b + m.Lp) : nullptr;
  layer->status = reinterpret_cast<int32_t*>(b + m.status);
  layer->Lq = r ? b + m.Lq : nullptr;
  layer->Rq = r ? b + m.Rq : nullptr;
  layer->adapter_bits = 16;
  layer->magic = slim::kLayerMagic;
  cudaError_t e = cudaMemsetAsync(layer->status, 0, sizeof(int32_t), static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return SLIM_OK;
}

slim_status slim_layer_init(slim_layer* layer, int K, int N, int r, int group, void* dev_buf, size_t bytes,
                            void* stream) {
  const int32_t n[1] = {N};
  if (!layer || !dev_buf) return SLIM_ERR_ARG;
  return slim_grouped_layer_init(layer, K, 1, n, r, group, dev_buf, bytes, stream);
}

slim_status slim_pack(const slim_layer* layer, const uint16_t* W, const uint16_t* L, const uint16_t* R,
                      void* stream) {
  slim::NvtxRange nv("slim_pack");
  if (!layer_ok(layer)) return SLIM_ERR_STATE;
  if (!W) return SLIM_ERR_ARG;
  if ((layer->r > 0) != (L != nullptr) || (layer->r > 0) != (R != nullptr)) return SLIM_ERR_ARG;
  if (!aligned16(W) || (L && !aligned16(L)) || (R && !aligned16(R))) return SLIM_ERR_ALIGN;
  slim_status st = check_device();
  if (st != SLIM_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = slim::launch_pack(*layer, W, s);
  if (e != cudaSuccess) return cuda_fail(e);
  if (layer->adapter_bits == 4) {
    e = slim::launch_quant_adapter(*layer, L, R, s);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  e = slim::launch_pack_adapter(*layer, L, R, s);
  if (e != cudaSuccess) return cuda_fail(e);
  e = slim::launch_pack_rp(*layer, R, s);
  if (e != cudaSuccess) return cuda_fail(e);
  e = slim::launch_pack_lp(*layer, L, s);
  if (e != cudaSuccess) return cuda_fail(e);
  e = slim::launch_pack_done(s);
  if (e != cudaSuccess) return cuda_fail(e);
  return SLIM_OK;
}

slim_status slim_layer_set_adapter_bits(slim_layer* layer, int bits) {
  if (!layer_ok(layer)) return SLIM_ERR_STATE;
  if (bits != 4 && bits != 16) return SLIM_ERR_ARG;
  layer->adapter_bits = bits;
  return SLIM_OK;
}

slim_status slim_unpack_adapters(const slim_layer* layer, int8_t* qL, uint16_t* sL, int8_t* qR, uint16_t* sR,
                                 void* stream) {
  if (!layer_ok(layer) || layer->adapter_bits != 4 || layer->r == 0) return SLIM_ERR_STATE;
  if (!qL || !sL || !qR || !sR) return SLIM_ERR_ARG;
  if (!aligned16(qL) || !aligned16(sL) || !aligned16(qR) || !aligned16(sR)) return SLIM_ERR_ALIGN;
  slim_status st = check_device();
  if (st != SLIM_OK) return st;
  cudaError_t e = slim::launch_unpack_adapters(*layer, qL, sL, qR, sR, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return SLIM_OK;
}

size_t slim_workspace_bytes(const slim_layer* layer, int M) {
  if (!layer_ok(layer) || M < 0) return 0;
  return t_bytes_upto(layer, M);
}

slim_status slim_linear(const slim_layer* layer, const uint16_t* X, int M, uint16_t* Y, void* workspace,
                        size_t ws_bytes, void* stream) {
  slim::NvtxRange nv("slim_linear");
  if (!layer_ok(layer)) return SLIM_ERR_STATE;
  if (M < 0) return SLIM_ERR_ARG;
  if (M == 0) return SLIM_OK;
  if (!X || !Y) return SLIM_ERR_ARG;
  if (!aligned16(X) || !aligned16(Y)) return SLIM_ERR_ALIGN;
  const size_t need = t_bytes(layer, M);
  if (need > 0 && (!workspace || ws_bytes < need)) return SLIM_ERR_WORKSPACE;
  if (workspace && !aligned16(workspace)) return SLIM_ERR_ALIGN;
  {
    const uintptr_t x0 = reinterpret_cast<uintptr_t>(X), x1 = x0 + (size_t)M * layer->K * 2;
    const uintptr_t y0 = reinterpret_cast<uintptr_t>(Y), y1 = y0 + (size_t)M * layer->N * 2;
    if (x0 < y1 && y0 < x1) return SLIM_ERR_ARG;  // X and Y overlap
  }
  slim_status st = check_device();
  if (st != SLIM_OK) return st;
  cudaError_t e = slim::launch_forward(*layer, X, M, Y, workspace, true, SIZE_MAX, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return SLIM_OK;
}

size_t slim_host_workspace_bytes(const slim_layer* layer, int M) {
  if (!layer_ok(layer) || M < 0) return 0;
  return t_bytes_upto(layer, M) + align_up((size_t)M * layer->K * 2, 256) + align_up((size_t)M * layer->N * 2, 256);
}

slim_status slim_linear_host(const slim_layer* layer, const uint16_t* X_host, int M, uint16_t* Y_host,
                             void* workspace, size_t ws_bytes, void* stream) {
  slim_status st = slim_linear_host_async(layer, X_host, M, Y_host, workspace, ws_bytes, stream);
  if (st != SLIM_OK || M == 0) return st;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return SLIM_OK;
}

slim_status slim_linear_host_async(const slim_layer* layer, const uint16_t* X_host, int M, uint16_t* Y_host,
                                   void* workspace, size_t ws_bytes, void* stream) {
  slim::NvtxRange nv("slim_linear_host_async");
  if (!layer_ok(layer)) return SLIM_ERR_STATE;
  if (M < 0) return SLIM_ERR_ARG;
  if (M == 0) return SLIM_OK;
  if (!X_host || !Y_host || !workspace) return SLIM_ERR_ARG;
  if (!aligned16(workspace)) return SLIM_ERR_ALIGN;
  const size_t tb = t_bytes_upto(layer, M);
  const size_t xb = (size_t)M * layer->K * 2, yb = (size_t)M * layer->N * 2;
  if (ws_bytes < slim_host_workspace_bytes(layer, M)) return SLIM_ERR_WORKSPACE;
  uint8_t* w = static_cast<uint8_t*>(workspace);
  uint16_t* Xd = reinterpret_cast<uint16_t*>(w + tb);
  uint16_t* Yd = reinterpret_cast<uint16_t*>(w + tb + align_up(xb, 256));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(Xd, X_host, xb, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return cuda_fail(e);
  slim_status st = slim_linear(layer, Xd, M, Yd, tb ? w : nullptr, tb, stream);
  if (st != SLIM_OK) return st;
  e = cudaMemcpyAsync(Y_host, Yd, yb, cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return cuda_fail(e);
  return SLIM_OK;
}

slim_status slim_test_wait_timeout(const slim_layer* layer, int wait_us, void* stream) {
  if (!layer_ok(layer)) return SLIM_ERR_STATE;
  if (wait_us < 0) return SLIM_ERR_ARG;
  slim_status st = check_device();
  if (st != SLIM_OK) return st;
  cudaError_t e = slim::launch_wait_probe(layer->status, wait_us, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return SLIM_OK;
}

slim_status slim_test_stream_timeout(const slim_layer* layer, const uint16_t* X, int M, uint16_t* Y,
                                     void* workspace, size_t ws_bytes, int wait_us, void* stream) {
  if (!layer_ok(layer)) return SLIM_ERR_STATE;
  if (M < 1 || M > 16 || !X || !Y || wait_us < 0 || layer->r16 == 0) return SLIM_ERR_ARG;
  if (!aligned16(X) || !aligned16(Y) || !aligned16(workspace)) return SLIM_ERR_ALIGN;
  slim_status st = check_device();
  if (st != SLIM_OK) return st;
  if (!slim::stream_supported(*layer, M)) return SLIM_ERR_UNSUPPORTED;
  const size_t need = slim::stream_workspace_bytes(*layer, M);
  if (!workspace || ws_bytes < need) return SLIM_ERR_WORKSPACE;
  int dev = slim::current_device(), khz = 0;
  cudaError_t e = cudaDeviceGetAttribute(&khz, cudaDevAttrClockRate, dev);
  if (e != cudaSuccess) return cuda_fail(e);
  const long long cycles = std::min<long long>((long long)wait_us * khz / 1000, slim::kWaitBudgetCycles);
  e = slim::launch_stream_ex(*layer, X, M, Y, workspace, cycles, 1u, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return SLIM_OK;
}

slim_status slim_unpack_dec(const slim_layer* layer, int8_t* q_dense, uint16_t* scales, void* stream) {
  if (!layer_ok(layer)) return SLIM_ERR_STATE;
  if (!q_dense || !scales) return SLIM_ERR_ARG;
  if (!aligned16(q_dense) || !aligned16(scales)) return SLIM_ERR_ALIGN;
  slim_status st = check_device();
  if (st != SLIM_OK) return st;
  cudaError_t e = slim::launch_unpack_dec(*layer, q_dense, scales, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return SLIM_OK;
}

slim_status slim_sync_status(const slim_layer* layer, void* stream) {
  if (!layer_ok(layer)) return SLIM_ERR_STATE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t h = 0;
  cudaError_t e = cudaMemcpyAsync(&h, layer->status, sizeof(h), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(layer->status, 0, sizeof(int32_t), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e);
  return static_cast<slim_status>(h);
}

const char* slim_status_string(slim_status s) {
  switch (s) {
    case SLIM_OK: return "ok";
    case SLIM_ERR_ARG: return "invalid argument";
    case SLIM_ERR_ALIGN: return "pointer not 16-byte aligned";
    case SLIM_ERR_SHAPE: return "unsupported shape (K % 128, group, N, r)";
    case SLIM_ERR_WORKSPACE: return "buffer or workspace too small";
    case SLIM_ERR_RANGE: return "non-finite weight or fp16 group-scale overflow";
    case SLIM_ERR_TIMEOUT: return "a bounded wait in a kernel gave up";
    case SLIM_ERR_CUDA: return "CUDA runtime error";
    case SLIM_ERR_UNSUPPORTED: return "device is not sm_100";
    case SLIM_ERR_STATE: return "layer descriptor not initialised";
    case SLIM_ERR_BOUNDS: return "a kernel index check failed (debug build)";
  }
  return "unknown status";
}

int slim_linear_launches(const slim_layer* layer, int M) {
  if (!layer_ok(layer) || M < 0) return -1;
  return slim::forward_launches(*layer, M, true);
}

int slim_last_cuda_error(void) { return slim::last_cuda_error(); }

void slim_tuning_reload(void) { slim::reload_tuning(); }

int slim_abi_version(void) { return SLIM_ABI_VERSION; }

}  // extern "C"

// Host-side state shared by every entry point: the tuning knobs, per-device
// attributes, and the last failed CUDA call.
#include <atomic>
#include <cstdio>
#include <cstdlib>

#include "slim_common.cuh"
#include "slim_internal.h"

namespace slim {
namespace {

constexpr int kMaxDevices = 64;

std::mutex g_tuning_mu;
Tuning g_tuning;
bool g_tuning_read = false;

Tuning read_env(unsigned generation) {
  Tuning t;
  t.generation = generation;
  t.no_stream = std::getenv("SLIM_NO_STREAM") != nullptr;
  t.no_prefill = std::getenv("SLIM_NO_PREFILL") != nullptr;
  t.prefill_1sm = std::getenv("SLIM_PREFILL_1SM") != nullptr;
  t.pdl_early = std::getenv("SLIM_PDL_EARLY") != nullptr;
  if (const char* v = std::getenv("SLIM_STREAM_WARPS")) t.stream_warps = std::atoi(v) == 16 ? 16 : 8;
  if (const char* v = std::getenv("SLIM_DECODE_CFG")) {
    int a = 0, b = 0, c = 0;
    const bool known_split = std::sscanf(v, "%d,%d,%d", &a, &b, &c) == 3 &&
                             ((a == 1 && b == 8) || (a == 2 && b == 4) || (a == 4 && (b == 1 || b == 2)) ||
                              (a == 8 && b == 1) || (a == 1 && b == 4)) &&
                             c >= 1 && c <= 16;
    // Any value, valid or not, keeps M <= 16 off the single-launch kernel.
    t.decode_cfg = true;
    if (known_split) {
      t.dec_wr = a;
      t.dec_kw = b;
      t.dec_s = c;
    }
  }
  if (const char* v = std::getenv("SLIM_PREFILL_TILE")) {
    int nh = 0, tt = 0;
    if (std::sscanf(v, "pair,%d", &tt) == 1 && (tt == 128 || tt == 192 || tt == 224 || tt == 240)) {
      t.prefill_tile = t.prefill_pair = true;
      t.prefill_tt = tt;
    } else if (std::sscanf(v, "%d,%d", &nh, &tt) == 2 && (nh == 1 || nh == 2) && (tt == 64 || tt == 128 || tt == 192)) {
      t.prefill_tile = true;
      t.prefill_nh = nh;
      t.prefill_tt = tt;
    }
  }
  return t;
}

thread_local int g_last_cuda_error = 0;

std::atomic<int> g_sms[kMaxDevices];
std::atomic<int> g_major[kMaxDevices];

}  // namespace

Tuning tuning() {
  std::lock_guard<std::mutex> lock(g_tuning_mu);
  if (!g_tuning_read) {
    g_tuning = read_env(0);
    g_tuning_read = true;
  }
  return g_tuning;
}

void reload_tuning() {
  std::lock_guard<std::mutex> lock(g_tuning_mu);
  g_tuning = read_env(g_tuning_read ? g_tuning.generation + 1 : 0);
  g_tuning_read = true;
}

int current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}

int num_sms() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return 148;
  int n = g_sms[dev].load(std::memory_order_relaxed);
  if (n <= 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    g_sms[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

int device_cc_major() {
  const int dev = current_device();
  if (dev < 0) return -1;
  if (dev >= kMaxDevices) {
    int major = -1;
    return cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) == cudaSuccess ? major : -1;
  }
  int major = g_major[dev].load(std::memory_order_relaxed);
  if (major <= 0) {
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return -1;
    g_major[dev].store(major, std::memory_order_relaxed);
  }
  return major;
}

void set_last_cuda_error(cudaError_t e) { g_last_cuda_error = static_cast<int>(e); }

int last_cuda_error() { return g_last_cuda_error; }

}  // namespace slim

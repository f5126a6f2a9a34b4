// Host-side entry points that launch nothing: status strings, sizes, device
// checks.
#include <cuda_runtime.h>

#include <atomic>

#include "qoq.h"
#include "qoq_internal.h"

namespace qoq {

namespace {
constexpr int kMaxDevices = 64;
// 0 = unknown, 1 = supported, 2 = unsupported
std::atomic<int> g_dev_ok[kMaxDevices];
std::atomic<int> g_dev_sms[kMaxDevices];
}  // namespace

int check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return QOQ_ERR_CUDA;
  }
  if (dev >= 0 && dev < kMaxDevices) {
    const int v = g_dev_ok[dev].load(std::memory_order_relaxed);
    if (v == 1) return QOQ_OK;
    if (v == 2) return QOQ_ERR_UNSUPPORTED;
  }
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
    cudaGetLastError();
    return QOQ_ERR_CUDA;
  }
  const bool ok = (major == 10 && minor == 0);
  if (dev >= 0 && dev < kMaxDevices) g_dev_ok[dev].store(ok ? 1 : 2, std::memory_order_relaxed);
  return ok ? QOQ_OK : QOQ_ERR_UNSUPPORTED;
}

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return 148;
  }
  if (dev >= 0 && dev < kMaxDevices) {
    const int v = g_dev_sms[dev].load(std::memory_order_relaxed);
    if (v > 0) return v;
  }
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      sms <= 0) {
    cudaGetLastError();
    return 148;
  }
  if (dev >= 0 && dev < kMaxDevices) g_dev_sms[dev].store(sms, std::memory_order_relaxed);
  return sms;
}

int launch_status() {
  return cudaGetLastError() == cudaSuccess ? QOQ_OK : QOQ_ERR_CUDA;
}

}  // namespace qoq

extern "C" const char* qoq_status_str(int status) {
  switch (status) {
    case QOQ_OK: return "ok";
    case QOQ_ERR_INVALID_ARG: return "invalid argument (pointer, shape or alignment)";
    case QOQ_ERR_UNSUPPORTED: return "unsupported (device, group size or problem size)";
    case QOQ_ERR_CUDA: return "CUDA runtime or driver error";
    case QOQ_ERR_WORKSPACE: return "split-K workspace too small for the launch plan";
    default: return "unknown status";
  }
}

extern "C" int qoq_version(void) { return 1; }

extern "C" int qoq_protective_range(void) { return qoq::kProtectiveRange; }

extern "C" size_t qoq_packed_block_bytes(int group) { return qoq::block_bytes(group); }

extern "C" size_t qoq_packed_weight_bytes(int N, int K, int group) {
  if (qoq::check_weight_shape(N, K, group) != QOQ_OK) return 0;
  const size_t blocks = static_cast<size_t>(N / qoq::kTileN) * static_cast<size_t>(K / qoq::kTileK);
  return blocks * qoq::block_bytes(group);
}

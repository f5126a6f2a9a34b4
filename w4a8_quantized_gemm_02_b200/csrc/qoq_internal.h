// Host-side helpers shared by the library's translation units.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "qoq.h"

namespace qoq {

constexpr int kTileN = 128;       // output channels per weight block / MMA M
constexpr int kTileK = 128;       // input channels per weight block (one swizzle row)
constexpr int kCodesBytes = kTileN * kTileK / 2;   // 8192
constexpr int kMaxK = 133120;     // 127 * 127 * K < 2^31
constexpr int kProtectiveRange = 119;

inline bool aligned16(const void* p) {
  return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline size_t block_bytes(int group) {
  if (group != 64 && group != 128) return 0;
  const int gpt = kTileK / group;                  // groups per block row
  return static_cast<size_t>(kCodesBytes) + static_cast<size_t>(gpt) * (128 + 64);
}

// Shape checks common to every weight entry point.
inline int check_weight_shape(int N, int K, int group) {
  if (group != 64 && group != 128) return QOQ_ERR_UNSUPPORTED;
  if (N <= 0 || K <= 0) return QOQ_ERR_INVALID_ARG;
  if (N % kTileN != 0 || K % kTileK != 0 || K % group != 0) return QOQ_ERR_INVALID_ARG;
  if (K > kMaxK) return QOQ_ERR_UNSUPPORTED;
  return QOQ_OK;
}

// The current device must be compute capability 10.0 (sm_100a code only).
int check_device();
// Number of SMs of the current device (cached per device; 148 if unknown).
int sm_count();
// cudaGetLastError -> status.
int launch_status();

// The CUDA-core GEMV for one to four tokens (qoq_gemv.cu): same integer
// product and epilogue as the tensor-core GEMM.  Launched as a programmatic
// dependent; with w_dep_wait == 0 its first weight loads may precede the
// preceding grid's completion.
struct GemvArgs {
  const uint8_t* packed;
  const int8_t* X8;
  const __half* sx;
  const __half* s1;
  __half* Y;        // FP16 output, or
  int32_t* acc;     // the INT32 accumulators (exactly one of the two)
  int M, N, K, group, blk_bytes, w_dep_wait;
  int ks, kt_per;           // K split into ks ranges of kt_per k-tiles
  int stages;               // copy-ring slots per warp: 2 or 4
  uint32_t* ws_count;       // ks > 1: an arrival counter per 32 channels (zero between calls)
  int32_t* ws_acc;          // ks > 1: [split][M][N] INT32 partial sums
};
constexpr int kGemvMaxTokens = 4;
constexpr size_t kGemvMaxSmem = 227 * 1024;   // the opt-in maximum per block on sm_100
size_t gemv_smem_bytes(int M, int K, int stages);
int launch_gemv(const GemvArgs& a, cudaStream_t s);

// The GEMM launcher shared by the entry points.  The kernel may start while
// the preceding kernel on the stream is still running (programmatic
// dependent launch): it sets up right away and waits for that grid before
// reading X8 / sx, writing anything, and (unless
// `weights_independent`: the preceding kernel cannot have written the
// weights) before copying weights.  With `clear_counters` the workspace's
// arrival counters are zeroed on the stream before the kernel, when the
// plan splits K (after every argument check, so a rejected call enqueues
// nothing).
int gemm_impl(const int8_t* X8, const void* sx, const void* packed, const void* s1, int M, int N,
              int K, int group, void* Y, int32_t* acc, int tok_req, int splits_req, void* ws,
              size_t ws_bytes, void* stream, bool weights_independent, bool clear_counters);

// Launch the per-token activation quantizer (no argument checks).  With
// `pdl` it may start while the preceding kernel on the stream drains; it
// waits for that grid before touching memory.
// `smooth` (FP16[K] or nullptr): divide each value by its channel's
// smoothing factor before quantizing.
int launch_act_quant(const void* X, int M, int K, int8_t* X8, void* sx, void* stream, bool pdl,
                     const void* smooth);

}  // namespace qoq

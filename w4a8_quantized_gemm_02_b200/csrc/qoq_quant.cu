// Quantization kernels: per-token INT8 activations (online), progressive
// group quantization of the weights into the packed block format (offline),
// packing of given codes and the debug unpacker.
//
// Method: "QServe: W4A8KV4 Quantization and System Co-design for Efficient
// LLM Serving" -- Methods, 1) Algorithm: QoQ (progressive group quantization:
// per-channel INT8 with FP16 scales, then UINT4 per group) and 2) System:
// QServe (protective range; "subtraction after multiplication").
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "qoq.h"
#include "qoq_actq.cuh"
#include "qoq_device.cuh"
#include "qoq_internal.h"

namespace qoq {
namespace {

// Per-input-channel smoothing of eight FP16 values (the k-th value by the
// k-th factor): times the factor for weights (one rounding of the exact
// product), divided by it for activations (binary32 quotient, then FP16).
template <bool kDivide>
__device__ __forceinline__ uint4 smooth8(uint4 v, uint4 f) {
  __half2* h = reinterpret_cast<__half2*>(&v);
  const __half2* g = reinterpret_cast<const __half2*>(&f);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 x = __half22float2(h[j]);
    const float2 y = __half22float2(g[j]);
    h[j] = kDivide ? __floats2half2_rn(__fdiv_rn(x.x, y.x), __fdiv_rn(x.y, y.y))
                   : __floats2half2_rn(__fmul_rn(x.x, y.x), __fmul_rn(x.y, y.y));
  }
  return v;
}

// Packed row n of a weight -> its row in the caller's matrix.  Plain
// weights: n.  A fused gate_up weight of 2I rows (gate rows 0 .. I-1, up
// rows I .. 2I-1, gate_up_i = I): every 128-row tile t holds gate rows
// 64t .. 64t+63 in its rows 0..63 and the up rows of the same channels in
// rows 64..127, so one tile of the GEMM holds both halves of 64 outputs.
__device__ __forceinline__ int source_row(int n, int gate_up_i) {
  if (gate_up_i == 0) return n;
  const int t = n >> 7, r = n & 127;
  return r < 64 ? 64 * t + r : gate_up_i + 64 * t + (r - 64);
}

// Exact round-half-even of a / b for b > 0.
__device__ __forceinline__ int div_rne(int a, int b) {
  int q = a / b;
  int r = a - q * b;
  int ar = r < 0 ? -r : r;
  if (2 * ar > b || (2 * ar == b && (q & 1))) q += (a < 0) ? -1 : 1;
  return q;
}

// kWarps warps per CTA, kWarpsPerRow of them share a row (1: a warp per row;
// kWarps: a CTA per row).  Each thread keeps up to kRegVec 16-byte vectors of
// its row in registers (one pass over global memory); longer rows are read
// twice.  Few vectors per thread keep the register count low, so that many
// CTAs share an SM and many loads are in flight.
template <int kWarps, int kWarpsPerRow, int kRegVec, bool kSmooth>
__global__ void __launch_bounds__(32 * kWarps)
act_quant_kernel(const __half* __restrict__ X, int M, int K, int8_t* __restrict__ X8,
                 __half* __restrict__ sx, const __half* __restrict__ smooth) {
  // Launched as a programmatic dependent of the previous kernel on the stream
  // (qoq_w4a8_linear), this CTA may start while that kernel drains: nothing
  // is read or written before that grid has completed and its writes are
  // visible.  Without the launch attribute the wait returns at once.
  grid_dependency_wait();
  // the GEMM that consumes X8 may start its weight prologue right away
  grid_launch_dependents();
  __shared__ float red[kWarps];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr int kRows = kWarps / kWarpsPerRow;
  const int m = blockIdx.x * kRows + warp / kWarpsPerRow;
  const int t = (warp % kWarpsPerRow) * 32 + lane;   // thread index within the row
  constexpr int kT = 32 * kWarpsPerRow;              // threads per row
  const bool active = m < M;
  const uint4* row = reinterpret_cast<const uint4*>(X + static_cast<size_t>(active ? m : 0) * K);
  uint2* out = reinterpret_cast<uint2*>(X8 + static_cast<size_t>(active ? m : 0) * K);
  const int nvec = active ? K / 8 : 0;
  const bool in_regs = K / 8 <= kT * kRegVec;
  // smoothed activations: each value divided by its channel's factor first
  const uint4* sv = reinterpret_cast<const uint4*>(smooth);
  auto load = [&](int i) {
    uint4 x = __ldg(row + i);
    if constexpr (kSmooth) x = smooth8<true>(x, __ldg(sv + i));
    return x;
  };
  uint4 v[kRegVec];
  __half2 hmax = __float2half2_rn(0.0f);
  if (in_regs) {
#pragma unroll
    for (int u = 0; u < kRegVec; ++u) {
      const int i = t + kT * u;
      if (i < nvec) v[u] = load(i);
    }
#pragma unroll
    for (int u = 0; u < kRegVec; ++u)
      if (t + kT * u < nvec) hmax = absmax8(v[u], hmax);
  } else {
    for (int i0 = 0; i0 < nvec; i0 += kT * 8) {
      uint4 w[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + t + kT * u;
        if (i < nvec) w[u] = load(i);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (i0 + t + kT * u < nvec) hmax = absmax8(w[u], hmax);
    }
  }
  float amax = fmaxf(__low2float(hmax), __high2float(hmax));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (kWarpsPerRow > 1) {
    if (lane == 0) red[warp] = amax;
    __syncthreads();
    amax = 0.0f;
#pragma unroll
    for (int w = 0; w < kWarpsPerRow; ++w)
      amax = fmaxf(amax, red[(warp / kWarpsPerRow) * kWarpsPerRow + w]);
  }
  if (!active) return;
  const __half s = scale_from_absmax(amax, 127.0f);
  if (t == 0) sx[m] = s;
  const float sf = __half2float(s);
  const float rcp = __frcp_rn(sf);
  const float half_sf = 0.5f * sf;
  const bool clamp = sf < 6.103515625e-05f;   // subnormal FP16 scale (below 2^-14)
  if (in_regs) {
    if (!clamp) {
#pragma unroll
      for (int u = 0; u < kRegVec; ++u) {
        const int i = t + kT * u;
        if (i < nvec) out[i] = quantize8<false>(v[u], sf, rcp, half_sf);
      }
    } else {
#pragma unroll
      for (int u = 0; u < kRegVec; ++u) {
        const int i = t + kT * u;
        if (i < nvec) out[i] = quantize8<true>(v[u], sf, rcp, half_sf);
      }
    }
  } else {
    if (!clamp) {
      for (int i = t; i < nvec; i += kT) out[i] = quantize8<false>(load(i), sf, rcp, half_sf);
    } else {
      for (int i = t; i < nvec; i += kT) out[i] = quantize8<true>(load(i), sf, rcp, half_sf);
    }
  }
}

// ---------------------------------------------------------------------------
// Level 1 scale: one warp per output channel.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
row_scale_kernel(const __half* __restrict__ W, int N, int K, __half* __restrict__ s1,
                 const __half* __restrict__ smooth, int gate_up_i) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= N) return;
  const uint4* row =
      reinterpret_cast<const uint4*>(W + static_cast<size_t>(source_row(warp, gate_up_i)) * K);
  float amax = 0.0f;
  for (int i = lane; i < K / 8; i += 32) {
    uint4 v = __ldg(row + i);
    if (smooth) v = smooth8<false>(v, __ldg(reinterpret_cast<const uint4*>(smooth) + i));
    const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float2 f = __half22float2(h[j]);
      amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (lane == 0) s1[warp] = scale_from_absmax(amax, static_cast<float>(kProtectiveRange));
}

// ---------------------------------------------------------------------------
// Level 2 + pack: one CTA of 128 threads per (n-tile, k-tile) block; thread r
// owns output channel n0 + r.  The FP16 tile is staged through shared memory
// (rows padded by 16 bytes so that a thread per row reads without bank
// conflicts).
// ---------------------------------------------------------------------------
constexpr int kPackRowBytes = kTileK * 2 + 16;   // 272

__device__ __forceinline__ int level1_code(float w, float s1f) {
  int v = __float2int_rn(__fdiv_rn(w, s1f));
  return max(-kProtectiveRange, min(kProtectiveRange, v));
}

__global__ void __launch_bounds__(128)
pack_weights_kernel(const __half* __restrict__ W, int K, int group,
                    const __half* __restrict__ s1, uint8_t* __restrict__ packed,
                    int blk_bytes, const __half* __restrict__ smooth, int gate_up_i) {
  __shared__ __align__(16) uint8_t tile[kTileN * kPackRowBytes];
  const int kt = blockIdx.x, nt = blockIdx.y;
  const int n0 = nt * kTileN, k0 = kt * kTileK;
  const int r = threadIdx.x;
  // coalesced staging: 128 rows x 256 bytes = 2048 chunks of 16 bytes
  for (int c = threadIdx.x; c < kTileN * 16; c += 128) {
    const int row = c >> 4, col = c & 15;
    uint4 v = __ldg(reinterpret_cast<const uint4*>(
                        W + static_cast<size_t>(source_row(n0 + row, gate_up_i)) * K + k0) + col);
    if (smooth) v = smooth8<false>(v, __ldg(reinterpret_cast<const uint4*>(smooth + k0) + col));
    *reinterpret_cast<uint4*>(tile + row * kPackRowBytes + col * 16) = v;
  }
  __syncthreads();

  const float s1f = __half2float(s1[n0 + r]);
  const __half* my = reinterpret_cast<const __half*>(tile + r * kPackRowBytes);
  const int gpt = kTileK / group;
  uint8_t* blk = packed + static_cast<size_t>(nt * (K / kTileK) + kt) * blk_bytes;

  int s2g[2] = {1, 1}, zg[2] = {0, 0};
  for (int gl = 0; gl < gpt; ++gl) {
    int mn = 0, mx = 0;
    for (int i = 0; i < group; ++i) {
      const int v = level1_code(__half2float(my[gl * group + i]), s1f);
      mn = min(mn, v);
      mx = max(mx, v);
    }
    const int s2 = max(1, (mx - mn + 14) / 15);
    s2g[gl] = s2;
    zg[gl] = div_rne(-mn, s2);
  }

  // codes: word w of chunk j covers k = 32j + 8w .. +7
#pragma unroll 1
  for (int j = 0; j < 4; ++j) {
    uint32_t words[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int kb = 32 * j + 8 * w;
      const int gl = kb / group;
      uint32_t word = 0;
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        const int v = level1_code(__half2float(my[kb + b]), s1f);
        const int q = max(0, min(15, div_rne(v, s2g[gl]) + zg[gl]));
        const int lane = b & 3, hi = b >> 2;
        word |= static_cast<uint32_t>(q) << (8 * lane + 4 * hi);
      }
      words[w] = word;
    }
    *reinterpret_cast<uint4*>(blk + (j * kTileN + r) * 16) =
        make_uint4(words[0], words[1], words[2], words[3]);
  }
  // metadata
  for (int gl = 0; gl < gpt; ++gl) {
    blk[kCodesBytes + gl * kTileN + r] = static_cast<uint8_t>(s2g[gl]);
    const int zo = __shfl_xor_sync(0xffffffffu, zg[gl], 1);
    if ((r & 1) == 0) {
      blk[kCodesBytes + gpt * kTileN + gl * 64 + (r >> 1)] =
          static_cast<uint8_t>((zg[gl] & 15) | ((zo & 15) << 4));
    }
  }
}

// ---------------------------------------------------------------------------
// Pack given canonical codes (one CTA of 128 threads per block).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128)
pack_codes_kernel(const uint8_t* __restrict__ q, const int8_t* __restrict__ s2,
                  const uint8_t* __restrict__ z, int K, int group,
                  uint8_t* __restrict__ packed, int blk_bytes) {
  const int kt = blockIdx.x, nt = blockIdx.y, r = threadIdx.x;
  const int n = nt * kTileN + r, k0 = kt * kTileK;
  const int gpt = kTileK / group, ng = K / group;
  uint8_t* blk = packed + static_cast<size_t>(nt * (K / kTileK) + kt) * blk_bytes;
  const uint8_t* qrow = q + static_cast<size_t>(n) * K + k0;
  for (int j = 0; j < 4; ++j) {
    uint32_t words[4];
    for (int w = 0; w < 4; ++w) {
      uint32_t word = 0;
      for (int b = 0; b < 8; ++b) {
        const uint32_t c = qrow[32 * j + 8 * w + b] & 15u;
        word |= c << (8 * (b & 3) + 4 * (b >> 2));
      }
      words[w] = word;
    }
    *reinterpret_cast<uint4*>(blk + (j * kTileN + r) * 16) =
        make_uint4(words[0], words[1], words[2], words[3]);
  }
  for (int gl = 0; gl < gpt; ++gl) {
    const int g = kt * gpt + gl;
    blk[kCodesBytes + gl * kTileN + r] = static_cast<uint8_t>(s2[static_cast<size_t>(n) * ng + g]);
    const int zv = z[static_cast<size_t>(n) * ng + g] & 15;
    const int zo = __shfl_xor_sync(0xffffffffu, zv, 1);
    if ((r & 1) == 0) {
      blk[kCodesBytes + gpt * kTileN + gl * 64 + (r >> 1)] =
          static_cast<uint8_t>(zv | (zo << 4));
    }
  }
}

// ---------------------------------------------------------------------------
// Smoothing factors: per input channel k, the largest |X| of the calibration
// batch (ax) and the largest |W| (aw), then s = fp16(clamp(sqrt(ax / aw),
// 2^-14, 2^14)) in binary32 (1 where a maximum is 0).  A CTA of 256 threads
// takes 32 channels; its 8 row lanes stride the rows.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
smooth_factors_kernel(const __half* __restrict__ Xc, int Mc, const __half* __restrict__ W, int N,
                      int K, __half* __restrict__ s) {
  __shared__ float red[2][8][32];
  const int c = threadIdx.x & 31, rl = threadIdx.x >> 5;
  const int k = blockIdx.x * 32 + c;
  float ax = 0.0f, aw = 0.0f;
  if (k < K) {
    for (int m = rl; m < Mc; m += 8) ax = fmaxf(ax, fabsf(__half2float(Xc[static_cast<size_t>(m) * K + k])));
    for (int n = rl; n < N; n += 8) aw = fmaxf(aw, fabsf(__half2float(W[static_cast<size_t>(n) * K + k])));
  }
  red[0][rl][c] = ax;
  red[1][rl][c] = aw;
  __syncthreads();
  if (rl != 0 || k >= K) return;
#pragma unroll
  for (int i = 1; i < 8; ++i) {
    ax = fmaxf(ax, red[0][i][c]);
    aw = fmaxf(aw, red[1][i][c]);
  }
  if (ax == 0.0f || aw == 0.0f) {
    s[k] = __ushort_as_half(0x3c00);
    return;
  }
  const float r = fminf(fmaxf(__fsqrt_rn(__fdiv_rn(ax, aw)), 0x1p-14f), 0x1p14f);
  s[k] = __float2half_rn(r);
}

// ---------------------------------------------------------------------------
// Debug unpacker: canonical q / s2 / z and dq via the GEMM's byte-lane path.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128)
unpack_kernel(const uint8_t* __restrict__ packed, int K, int group, uint8_t* __restrict__ q,
              int8_t* __restrict__ s2o, uint8_t* __restrict__ zo, int8_t* __restrict__ dq,
              int blk_bytes) {
  const int kt = blockIdx.x, nt = blockIdx.y, r = threadIdx.x;
  const int n = nt * kTileN + r, k0 = kt * kTileK;
  const int gpt = kTileK / group, ng = K / group;
  const uint8_t* blk = packed + static_cast<size_t>(nt * (K / kTileK) + kt) * blk_bytes;
  uint32_t s2v[2], zv[2], bias[2];
  for (int gl = 0; gl < gpt; ++gl) {
    s2v[gl] = static_cast<uint32_t>(static_cast<int8_t>(blk[kCodesBytes + gl * kTileN + r]));
    const uint32_t zb = blk[kCodesBytes + gpt * kTileN + gl * 64 + (r >> 1)];
    zv[gl] = (r & 1) ? (zb >> 4) : (zb & 15u);
    bias[gl] = dq_bias(zv[gl], s2v[gl]);
    const int g = kt * gpt + gl;
    if (s2o) s2o[static_cast<size_t>(n) * ng + g] = static_cast<int8_t>(s2v[gl]);
    if (zo) zo[static_cast<size_t>(n) * ng + g] = static_cast<uint8_t>(zv[gl]);
  }
  for (int j = 0; j < 4; ++j) {
    const uint4 v = *reinterpret_cast<const uint4*>(blk + (j * kTileN + r) * 16);
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
    for (int w = 0; w < 4; ++w) {
      const int kb = 32 * j + 8 * w;
      const int gl = kb / group;
      const uint32_t lo = lo_codes(w4[w]), hi = hi_codes(w4[w]);
      const size_t base = static_cast<size_t>(n) * K + k0 + kb;
      if (q) {
        *reinterpret_cast<uint32_t*>(q + base) = lo;
        *reinterpret_cast<uint32_t*>(q + base + 4) = hi;
      }
      if (dq) {
        *reinterpret_cast<uint32_t*>(dq + base) = dq_lanes(lo, s2v[gl], bias[gl]);
        *reinterpret_cast<uint32_t*>(dq + base + 4) = dq_lanes(hi, s2v[gl], bias[gl]);
      }
    }
  }
}

}  // namespace
}  // namespace qoq

using namespace qoq;

namespace qoq {
template <int kWarps, int kWarpsPerRow, int kRegVec>
int launch_aq(const __half* X, int M, int K, int8_t* X8, __half* sx, cudaStream_t st, bool pdl,
              const __half* smooth) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(M), 1, 1);
  cfg.blockDim = dim3(32 * kWarps, 1, 1);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  cudaError_t e = smooth
      ? cudaLaunchKernelEx(&cfg, act_quant_kernel<kWarps, kWarpsPerRow, kRegVec, true>, X, M, K, X8,
                           sx, smooth)
      : cudaLaunchKernelEx(&cfg, act_quant_kernel<kWarps, kWarpsPerRow, kRegVec, false>, X, M, K,
                           X8, sx, smooth);
  return e == cudaSuccess ? QOQ_OK : QOQ_ERR_CUDA;
}

int launch_act_quant(const void* X, int M, int K, int8_t* X8, void* sx, void* stream, bool pdl,
                     const void* smooth) {
  const __half* sm = static_cast<const __half*>(smooth);
  const __half* Xh = static_cast<const __half*>(X);
  __half* sxh = static_cast<__half*>(sx);
  cudaStream_t st = as_stream(stream);
  const int nvec = K / 8;
  // one row per CTA in every variant
  if (M <= 2 * sm_count()) {
    // few rows: 8 warps per row keep many loads in flight per row
    return launch_aq<8, 8, 16>(Xh, M, K, X8, sxh, st, pdl, sm);
  }
  if (nvec <= 128 * 4) {
    // many rows: a CTA of 4 warps per row holding 4 vectors per thread
    return launch_aq<4, 4, 4>(Xh, M, K, X8, sxh, st, pdl, sm);
  }
  if (nvec <= 256 * 4) return launch_aq<8, 8, 4>(Xh, M, K, X8, sxh, st, pdl, sm);
  if (nvec <= 256 * 8) return launch_aq<8, 8, 8>(Xh, M, K, X8, sxh, st, pdl, sm);
  return launch_aq<8, 8, 16>(Xh, M, K, X8, sxh, st, pdl, sm);
}
}  // namespace qoq

extern "C" int qoq_quantize_act_per_token(const void* X, int M, int K, int8_t* X8, void* sx,
                                          void* stream) {
  if (!X || !X8 || !sx) return QOQ_ERR_INVALID_ARG;
  if (M <= 0 || K <= 0 || K % 8 != 0) return QOQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(X8) || !aligned16(sx)) return QOQ_ERR_INVALID_ARG;
  if (int st = check_device()) return st;
  return launch_act_quant(X, M, K, X8, sx, stream, false, nullptr);
}

extern "C" int qoq_quantize_act_per_token_smoothed(const void* X, const void* smooth, int M, int K,
                                                   int8_t* X8, void* sx, void* stream) {
  if (!X || !smooth || !X8 || !sx) return QOQ_ERR_INVALID_ARG;
  if (M <= 0 || K <= 0 || K % 8 != 0) return QOQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(smooth) || !aligned16(X8) || !aligned16(sx))
    return QOQ_ERR_INVALID_ARG;
  if (int st = check_device()) return st;
  return launch_act_quant(X, M, K, X8, sx, stream, false, smooth);
}

extern "C" int qoq_smooth_factors(const void* Xcal, int Mc, const void* W, int N, int K,
                                  void* smooth, void* stream) {
  if (!Xcal || !W || !smooth) return QOQ_ERR_INVALID_ARG;
  if (Mc <= 0 || N <= 0 || K <= 0) return QOQ_ERR_INVALID_ARG;
  if (int st = check_device()) return st;
  smooth_factors_kernel<<<(K + 31) / 32, 256, 0, as_stream(stream)>>>(
      static_cast<const __half*>(Xcal), Mc, static_cast<const __half*>(W), N, K,
      static_cast<__half*>(smooth));
  return launch_status();
}

namespace qoq {
namespace {
int quantize_weights_impl(const void* W, const void* smooth, int N, int K, int group,
                          void* packed, void* s1, void* stream, int gate_up_i) {
  if (!W || !packed || !s1) return QOQ_ERR_INVALID_ARG;
  if (int st = check_weight_shape(N, K, group)) return st;
  if (!aligned16(W) || !aligned16(packed) || !aligned16(s1) || (smooth && !aligned16(smooth)))
    return QOQ_ERR_INVALID_ARG;
  if (int st = check_device()) return st;
  cudaStream_t s = as_stream(stream);
  const __half* Wh = static_cast<const __half*>(W);
  const __half* sm = static_cast<const __half*>(smooth);
  __half* s1h = static_cast<__half*>(s1);
  row_scale_kernel<<<(N + 7) / 8, 256, 0, s>>>(Wh, N, K, s1h, sm, gate_up_i);
  if (int st = launch_status()) return st;
  dim3 grid(K / kTileK, N / kTileN);
  pack_weights_kernel<<<grid, 128, 0, s>>>(Wh, K, group, s1h, static_cast<uint8_t*>(packed),
                                           static_cast<int>(block_bytes(group)), sm, gate_up_i);
  return launch_status();
}
}  // namespace
}  // namespace qoq

extern "C" int qoq_quantize_weights(const void* W, int N, int K, int group, void* packed,
                                    void* s1, void* stream) {
  return quantize_weights_impl(W, nullptr, N, K, group, packed, s1, stream, 0);
}

extern "C" int qoq_quantize_weights_gate_up(const void* W, int I, int K, int group, void* packed,
                                            void* s1, void* stream) {
  if (I <= 0 || I % 64 != 0) return QOQ_ERR_INVALID_ARG;
  return quantize_weights_impl(W, nullptr, 2 * I, K, group, packed, s1, stream, I);
}

extern "C" int qoq_quantize_weights_smoothed(const void* W, const void* smooth, int N, int K,
                                             int group, void* packed, void* s1, void* stream) {
  if (!smooth) return QOQ_ERR_INVALID_ARG;
  return quantize_weights_impl(W, smooth, N, K, group, packed, s1, stream, 0);
}

extern "C" int qoq_pack_codes(const uint8_t* q, const int8_t* s2, const uint8_t* z, int N,
                              int K, int group, void* packed, void* stream) {
  if (!q || !s2 || !z || !packed) return QOQ_ERR_INVALID_ARG;
  if (int st = check_weight_shape(N, K, group)) return st;
  if (!aligned16(packed)) return QOQ_ERR_INVALID_ARG;
  if (int st = check_device()) return st;
  dim3 grid(K / kTileK, N / kTileN);
  pack_codes_kernel<<<grid, 128, 0, as_stream(stream)>>>(
      q, s2, z, K, group, static_cast<uint8_t*>(packed), static_cast<int>(block_bytes(group)));
  return launch_status();
}

extern "C" int qoq_unpack_weights(const void* packed, int N, int K, int group, uint8_t* q,
                                  int8_t* s2, uint8_t* z, int8_t* dq, void* stream) {
  if (!packed) return QOQ_ERR_INVALID_ARG;
  if (int st = check_weight_shape(N, K, group)) return st;
  if (!aligned16(packed) || (q && !aligned16(q)) || (dq && !aligned16(dq)))
    return QOQ_ERR_INVALID_ARG;
  if (int st = check_device()) return st;
  dim3 grid(K / kTileK, N / kTileN);
  unpack_kernel<<<grid, 128, 0, as_stream(stream)>>>(static_cast<const uint8_t*>(packed), K,
                                                     group, q, s2, z, dq,
                                                     static_cast<int>(block_bytes(group)));
  return launch_status();
}

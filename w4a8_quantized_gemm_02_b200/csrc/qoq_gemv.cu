// W4A8 GEMV for a few tokens (decode): the same integer product and epilogue
// as the tensor-core GEMM, on the CUDA cores.
//
// Method: "QServe: W4A8KV4 Quantization and System Co-design for Efficient
// LLM Serving" -- Methods 1) Algorithm: QoQ (per-channel INT8 first level,
// per-group UINT4 second level) and 2) System: QServe (register-level
// dequantization, dq = q*s2 - z*s2, the FP16 scaling once after K).
//
// With one to four tokens the product is a matrix-vector product: every
// weight is used by at most four multiply-adds, so the work is the stream of
// packed weights through the SM, and a 128 x TOK tensor-core tile would carry
// over 97% padding.  Here lane l of a warp owns channel 32 c + l of its CTA's
// 32 channels.  A CTA covers 32 channels over one of ks ranges of K; its
// eight warps take every eighth k-tile of the range.  Each warp streams its
// k-tiles through its own ring of S shared-memory slots with asynchronous
// 16-byte copies (per k-tile every lane copies its row's four code chunks,
// the warp 512 contiguous bytes per chunk, and six lanes the group scales and
// zero points), so S k-tiles per warp are in flight while one is multiplied.
// S is 2, or 4 for long K ranges (measured on B200: the deeper ring holds
// more bytes in flight, the shallower one more CTAs per SM).  The multiply
// turns four codes into four INT8 weights per 32-bit multiply-add (the same
// byte-lane arithmetic as the GEMM) and multiplies them with the tokens' INT8
// codes four at a time (dp4a, exact INT32).  The warps' sums are added in shared memory.  With ks > 1
// each CTA stores its INT32 partial sums in the workspace and counts its
// arrival at its 32 channels (acquire-release at GPU scope); the last arrival
// adds the ks slices.  Warp 0 of the CTA holding the whole sum applies
// Y = fp16(float(acc) * (sx * s1)), the GEMM's epilogue, bit for bit.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "qoq.h"
#include "qoq_device.cuh"
#include "qoq_internal.h"

namespace qoq {
namespace {

constexpr int kGemvWarps = 8;
constexpr int kGemvRows = 32;          // channels per CTA (one per lane)
// A ring slot: the 32 rows' code chunks (chunk j of lane l at 512 j + 16 l),
// then s2 of up to two groups ([group][row], 32 bytes each) and their zero
// points ([group][row / 2], two nibbles per byte, 16 bytes each).
constexpr int kSlotCodes = 4 * 512;
constexpr int kSlotS2 = kSlotCodes;
constexpr int kSlotZ = kSlotCodes + 64;
constexpr int kSlotBytes = kSlotCodes + 64 + 32;
constexpr size_t ring_bytes(int S) { return static_cast<size_t>(kGemvWarps) * S * kSlotBytes; }

// One k-tile of one row in registers: four 16-byte chunks of codes (chunk j
// holds codes 32 j .. 32 j + 31) and the group scale / bias of its one or
// two groups.
struct GemvTile {
  uint4 c[4];
  uint32_t s2[2], bias[2];
};

// Copy one k-tile of the CTA's 32 rows (rows rr0 .. rr0 + 31 of the packed
// block blk) into a ring slot.  Every source is 16-byte aligned: blocks are
// multiples of 16 bytes, rr0 is a multiple of 32.
__device__ __forceinline__ void gemv_issue(const uint8_t* blk, int rr0, int gpt, int lane,
                                           uint32_t slot) {
  const uint8_t* src = blk + (rr0 + lane) * 16;
#pragma unroll
  for (int j = 0; j < 4; ++j) cp_async16(slot + j * 512 + lane * 16, src + j * 2048);
  const uint8_t* scl = blk + kCodesBytes;
  if (lane < 2 * gpt) {            // s2 of group lane / 2, half lane % 2
    const int g = lane >> 1, h = lane & 1;
    cp_async16(slot + kSlotS2 + g * 32 + h * 16, scl + g * 128 + rr0 + h * 16);
  } else if (lane < 3 * gpt) {     // the zero points of group lane - 2 gpt
    const int g = lane - 2 * gpt;
    cp_async16(slot + kSlotZ + g * 16, scl + gpt * 128 + g * 64 + (rr0 >> 1));
  }
}

// This lane's row of a landed slot into registers.
__device__ __forceinline__ void gemv_read(const uint8_t* slot, int lane, int gpt, GemvTile& t) {
#pragma unroll
  for (int j = 0; j < 4; ++j) t.c[j] = *reinterpret_cast<const uint4*>(slot + j * 512 + lane * 16);
#pragma unroll
  for (int g = 0; g < 2; ++g) {
    const int gg = g < gpt ? g : 0;          // one group: both entries alike
    const uint32_t s2 = slot[kSlotS2 + gg * 32 + lane];
    const uint32_t zb = slot[kSlotZ + gg * 16 + (lane >> 1)];
    const uint32_t z = (lane & 1) ? (zb >> 4) : (zb & 15u);
    t.s2[g] = s2;
    t.bias[g] = dq_bias(z, s2);
  }
}

template <int MT>
__device__ __forceinline__ void gemv_accumulate(const GemvTile& t, int gpt, const int8_t* xs, int K,
                                                int k0, int (&acc)[MT]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    // the second group of a block of group 64 covers chunks 2 and 3; a
    // select rather than an index keeps the tile in registers
    const bool g1 = gpt == 2 && j >= 2;
    const uint32_t s2 = g1 ? t.s2[1] : t.s2[0];
    const uint32_t bias = g1 ? t.bias[1] : t.bias[0];
    const uint32_t w[4] = {t.c[j].x, t.c[j].y, t.c[j].z, t.c[j].w};
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      // the 32 token codes of chunk j: words 0..7 (word 2 q + 0: the low
      // nibbles' codes of chunk word q, word 2 q + 1: the high nibbles')
      const uint4 xa = *reinterpret_cast<const uint4*>(xs + m * K + k0 + 32 * j);
      const uint4 xb = *reinterpret_cast<const uint4*>(xs + m * K + k0 + 32 * j + 16);
      const int x[8] = {static_cast<int>(xa.x), static_cast<int>(xa.y), static_cast<int>(xa.z),
                        static_cast<int>(xa.w), static_cast<int>(xb.x), static_cast<int>(xb.y),
                        static_cast<int>(xb.z), static_cast<int>(xb.w)};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int lo = static_cast<int>(dq_lanes(lo_codes(w[q]), s2, bias));
        const int hi = static_cast<int>(dq_lanes(hi_codes(w[q]), s2, bias));
        acc[m] = __dp4a(lo, x[2 * q], acc[m]);
        acc[m] = __dp4a(hi, x[2 * q + 1], acc[m]);
      }
    }
  }
}

template <int MT, int S>
__global__ void __launch_bounds__(32 * kGemvWarps)
w4a8_gemv_kernel(const GemvArgs a) {
  extern __shared__ __align__(16) uint8_t gsm[];
  constexpr size_t kRing = ring_bytes(S);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* ring = gsm + static_cast<size_t>(warp) * S * kSlotBytes;            // this warp's
  int8_t* xs = reinterpret_cast<int8_t*>(gsm + kRing);                         // [MT][K]
  int* red = reinterpret_cast<int*>(gsm + kRing + ((MT * a.K + 15) & ~15));    // [warps][MT][32]
  const int grp = blockIdx.x / a.ks, split = blockIdx.x - grp * a.ks;
  const int r = grp * kGemvRows + lane;                                       // output channel
  const int nt = r >> 7, rr0 = (grp * kGemvRows) & 127;
  const int kt_total = a.K / kTileK;
  const int gpt = kTileK / a.group;
  const uint8_t* wrow = a.packed + static_cast<size_t>(nt) * kt_total * a.blk_bytes;

  // this warp's k-tiles: kt0, kt0 + 8, ... below kt_end
  const int kt0 = split * a.kt_per + warp;
  const int kt_end = min(kt_total, (split + 1) * a.kt_per);
  const int n = kt0 < kt_end ? (kt_end - kt0 + kGemvWarps - 1) / kGemvWarps : 0;
  // k-tile i goes to slot i mod S; one commit group per k-tile
  // index, empty past the end, keeps the group count uniform
  auto issue = [&](int i) {
    if (i < n)
      gemv_issue(wrow + static_cast<size_t>(kt0 + i * kGemvWarps) * a.blk_bytes, rr0, gpt, lane,
                 smem_u32(ring + (i % S) * kSlotBytes));
    cp_async_commit();
  };

  // The first k-tiles' weights may be read before the preceding grid
  // completes when that grid cannot have written them (programmatic
  // dependent launch); everything else waits for it.
  if (!a.w_dep_wait) {
#pragma unroll
    for (int i = 0; i < S; ++i) issue(i);
  }
  grid_dependency_wait();
  if (a.w_dep_wait) {
#pragma unroll
    for (int i = 0; i < S; ++i) issue(i);
  }
  // the tokens' codes, M x K bytes, into shared memory
  {
    const uint4* src = reinterpret_cast<const uint4*>(a.X8);
    uint4* dst = reinterpret_cast<uint4*>(xs);
    const int n16 = MT * a.K / 16;
    for (int i = threadIdx.x; i < n16; i += blockDim.x) dst[i] = __ldg(src + i);
  }
  __syncthreads();
  grid_launch_dependents();

  int acc[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) acc[m] = 0;
  for (int i = 0; i < n; ++i) {
    // groups 0 .. i have landed (S + i committed so far); the
    // warp-wide sync makes the scales other lanes copied visible, and the
    // second one keeps the slot's refill behind every lane's read
    cp_async_wait<S - 1>();
    __syncwarp();
    GemvTile t;
    gemv_read(ring + (i % S) * kSlotBytes, lane, gpt, t);
    __syncwarp();
    issue(i + S);
    gemv_accumulate<MT>(t, gpt, xs, a.K, (kt0 + i * kGemvWarps) * kTileK, acc);
  }
  cp_async_wait<0>();
#pragma unroll
  for (int m = 0; m < MT; ++m) red[(warp * MT + m) * 32 + lane] = acc[m];
  __syncthreads();
  if (warp != 0) return;
  int tot[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    tot[m] = 0;
#pragma unroll
    for (int w = 0; w < kGemvWarps; ++w) tot[m] += red[(w * MT + m) * 32 + lane];
  }
  if (a.ks > 1) {
    // publish this split's sums, count the arrival; the last one adds all
    int32_t* mine = a.ws_acc + static_cast<size_t>(split) * MT * a.N;
#pragma unroll
    for (int m = 0; m < MT; ++m) __stcg(mine + static_cast<size_t>(m) * a.N + r, tot[m]);
    __syncwarp();
    uint32_t last = 0;
    if (lane == 0) {
      uint32_t old;
      asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
                   : "=r"(old)
                   : "l"(a.ws_count + grp)
                   : "memory");
      last = old == static_cast<uint32_t>(a.ks - 1);
      if (last) a.ws_count[grp] = 0u;
    }
    __syncwarp();
    if (!__shfl_sync(0xffffffffu, last, 0)) return;
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      int sum = 0;
      for (int q = 0; q < a.ks; ++q)
        sum += __ldcg(a.ws_acc + (static_cast<size_t>(q) * MT + m) * a.N + r);
      tot[m] = sum;
    }
  }
  {
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const int s = tot[m];
      if (m < a.M) {
        if (a.Y) {
          const float scale = __fmul_rn(__half2float(a.sx[m]), __half2float(a.s1[r]));
          a.Y[static_cast<size_t>(m) * a.N + r] =
              __float2half_rn(__fmul_rn(static_cast<float>(s), scale));
        } else {
          a.acc[static_cast<size_t>(m) * a.N + r] = s;
        }
      }
    }
  }
}

template <int MT, int S>
int launch_mt(const GemvArgs& a, cudaStream_t s) {
  const size_t smem = gemv_smem_bytes(MT, a.K, S);
  static int configured_mask = 0;   // one bit per device id < 31
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QOQ_ERR_CUDA;
  const int bit = dev < 31 ? (1 << dev) : 0;
  if (!bit || !(__atomic_load_n(&configured_mask, __ATOMIC_ACQUIRE) & bit)) {
    if (cudaFuncSetAttribute(w4a8_gemv_kernel<MT, S>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kGemvMaxSmem)) != cudaSuccess)
      return QOQ_ERR_CUDA;
    if (bit) __atomic_fetch_or(&configured_mask, bit, __ATOMIC_RELEASE);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.N / kGemvRows * a.ks), 1, 1);
  cfg.blockDim = dim3(32 * kGemvWarps, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, w4a8_gemv_kernel<MT, S>, a) != cudaSuccess) return QOQ_ERR_CUDA;
  return QOQ_OK;
}

template <int MT>
int launch_stages(const GemvArgs& a, cudaStream_t s) {
  return a.stages == 4 ? launch_mt<MT, 4>(a, s) : launch_mt<MT, 2>(a, s);
}

}  // namespace

size_t gemv_smem_bytes(int M, int K, int stages) {
  return ring_bytes(stages) + ((static_cast<size_t>(M) * K + 15) & ~static_cast<size_t>(15)) +
         static_cast<size_t>(kGemvWarps) * M * 32 * sizeof(int);
}

int launch_gemv(const GemvArgs& a, cudaStream_t s) {
  switch (a.M) {
    case 1: return launch_stages<1>(a, s);
    case 2: return launch_stages<2>(a, s);
    case 3: return launch_stages<3>(a, s);
    default: return launch_stages<4>(a, s);
  }
}

}  // namespace qoq

// W4A8 GEMM for sm_100a: Y[m, n] = fp16((sum_k X8[m,k] * dq[n,k]) * sx[m] * s1[n]).
//
// Method: "QServe: W4A8KV4 Quantization and System Co-design for Efficient
// LLM Serving" -- Methods, 1) Algorithm: QoQ (all GEMMs on INT8 tensor cores
// after progressive group quantization) and 2) System: QServe (UINT4 -> INT8
// with register-level parallelism, "subtraction after multiplication");
// Background (per-group W4A4 dequantizes INT32 partial sums in its main loop,
// this kernel scales once, after the whole K reduction).
//
// One CTA computes a 128-channel x TOK-token output tile over a range of K.
// The weights are the MMA's M operand and the tokens its N operand, so a
// single decode token still fills the 128-row tensor-core tile.
//   warp 0      TMA producer: one bulk copy of the packed weight block and one
//               tensor-map copy of the X8 tile (128-byte swizzle) per k-tile,
//               into a ring of shared-memory stages;
//   warp 1      owns tensor memory and issues tcgen05.mma.kind::i8 (M = 128,
//               N = TOK, K = 32 per instruction, 4 per k-tile) with the INT8
//               weights read from tensor memory and X8 from shared memory,
//               INT32 accumulators in tensor memory;
//   warps 2..9  two dequantizing warpgroups taking alternate k-tiles: each
//               thread turns one weight row of the UINT4 block into INT8 (four
//               byte lanes per 32-bit multiply-add) and writes the 128-byte
//               row into tensor memory with one tcgen05.st; afterwards the
//               same warps run the epilogue.
// When K is split over several CTAs, each writes its INT32 partial tile to the
// caller's workspace and the last one to arrive (an arrival counter per output
// tile) adds them up exactly and runs the epilogue.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "qoq.h"
#include "qoq_device.cuh"
#include "qoq_internal.h"

namespace qoq {

__device__ unsigned int g_error_word = 0;

namespace {

constexpr int kThreads = 320;        // 10 warps
constexpr int kEpiThreads = 256;     // warps 2..9
constexpr int kRawStageBytes = 8576; // largest packed block (group 64), 16-byte multiple
constexpr int kSmemPerSm = 233472;   // 228 KiB of shared memory per SM
// The workspace starts with a fixed region of arrival counters (one word per
// output tile), so that counter words never share memory with the partial
// sums of a launch of another shape.
constexpr int kMaxCounterTiles = 4096;
constexpr size_t kCounterBytes = kMaxCounterTiles * 4;

template <int TOK>
struct Cfg {
  static constexpr int kStages = TOK <= 32 ? 8 : (TOK <= 64 ? 6 : 4);
  static constexpr int kDqStages = 4;
  static constexpr int kXBytes = TOK * kTileK;
  static constexpr int kOffX = 0;
  static constexpr int kOffRaw = kOffX + kStages * kXBytes;
  static constexpr int kOffSx = kOffRaw + kStages * kRawStageBytes;
  static constexpr int kOffBar = kOffSx + ((TOK * 4 + 15) / 16) * 16;
  static constexpr int kNumBars = 2 * kStages + 2 * kDqStages + 1;
  static constexpr int kOffMisc = kOffBar + 8 * kNumBars;
  static constexpr int kSmemUsed = kOffMisc + 16 + 1024;   // + base alignment slack
  // tensor memory: A operand stages at columns 32 d, the accumulator after them
  static constexpr int kTmemA = 0;
  static constexpr int kTmemD = 32 * kDqStages;
  static constexpr int kTmemCols = (kTmemD + TOK <= 256) ? 256 : 512;
  // Never more CTAs on an SM than tensor memory holds: request enough shared
  // memory that one more CTA cannot fit, so tcgen05.alloc never has to wait.
  static constexpr int kCtasPerSm = 512 / kTmemCols;
  static constexpr int kSmemFloor = kSmemPerSm / (kCtasPerSm + 1);
  static constexpr int kSmemBytes = kSmemUsed > kSmemFloor ? kSmemUsed : kSmemFloor;
  // epilogue slot: the INT32 tile as [token column][row], in the X ring
  static constexpr int kSlotBytes = kTileN * TOK * 4;
  static_assert(kOffRaw % 1024 == 0 && kXBytes % 1024 == 0, "swizzled tiles need 1 KiB alignment");
  static_assert(kOffBar % 8 == 0, "mbarriers need 8-byte alignment");
  static_assert(kSlotBytes <= kStages * kXBytes, "epilogue slot must fit in the X ring");
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
  static_assert(kTmemD + TOK <= kTmemCols, "tensor memory");
};

struct GemmArgs {
  const uint8_t* packed;
  const __half* sx;
  const __half* s1;
  __half* Y;
  int32_t* acc;
  int32_t* ws_part;     // [m_tile][split][TOK][N] partial sums (splits > 1)
  uint32_t* ws_count;   // [m_tile][n_tile] arrival counters (fixed region, zero between launches)
  int M, N, K, group;
  int splits;
  int blk_bytes;
};

// Bounded wait that ignores the abort flag: used only to drain work already
// in flight before a CTA tears down.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      atomicOr(&g_error_word, kErrProducer);
      return;
    }
  }
}

__device__ __forceinline__ void epi_bar() {
  asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
}

__device__ __forceinline__ uint4 add4(uint4 a, uint4 b) {
  return make_uint4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

__device__ __forceinline__ uint4 ld_cg_v4(const int32_t* p) {
  return __ldcg(reinterpret_cast<const uint4*>(p));
}

// Register this CTA's arrival at its output tile (one thread, after the
// CTA's partial tile is written and a fence made it visible).  The counter
// counts the arrivals of the current launch; the last of `splits` arrivals
// resets it to zero, so the counter region returns to zero after every
// launch that completes.
__device__ __forceinline__ bool arrive_last(uint32_t* ctr, int splits) {
  const uint32_t old = atomicAdd(ctr, 1u);
  if (old >= static_cast<uint32_t>(splits)) atomicOr(&g_error_word, kErrCounter);
  const bool last = old == static_cast<uint32_t>(splits - 1);
  if (last) atomicExch(ctr, 0u);
  return last;
}

template <int TOK>
__global__ void __launch_bounds__(kThreads, 1)
w4a8_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const GemmArgs args) {
  using C = Cfg<TOK>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t base = (raw_base + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw_base);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int splits = args.splits;
  const int nt = blockIdx.x / splits;
  const int split = blockIdx.x - nt * splits;
  const int mt = blockIdx.y;
  const int m0 = mt * TOK;
  const int kt_total = args.K / kTileK;
  const int kt_begin = (split * kt_total) / splits;
  const int num_kt = ((split + 1) * kt_total) / splits - kt_begin;

  const uint32_t bar_full = base + C::kOffBar;
  const uint32_t bar_empty = bar_full + 8 * C::kStages;
  const uint32_t bar_dqfull = bar_empty + 8 * C::kStages;
  const uint32_t bar_dqempty = bar_dqfull + 8 * C::kDqStages;
  const uint32_t bar_acc = bar_dqempty + 8 * C::kDqStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + C::kOffMisc + 4);
  volatile uint32_t* last_flag = reinterpret_cast<volatile uint32_t*>(smem + C::kOffMisc + 8);
  float* sx_s = reinterpret_cast<float*>(smem + C::kOffSx);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    for (int d = 0; d < C::kDqStages; ++d) {
      mbar_init(bar_dqfull + 8 * d, 4);
      mbar_init(bar_dqempty + 8 * d, 1);
    }
    mbar_init(bar_acc, 1);
    *abort_flag = 0u;
    *last_flag = 0u;
    fence_mbar_init();
    prefetch_tensormap(&tmap_x);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      const uint64_t policy = l2_policy_evict_first();
      const uint8_t* src =
          args.packed + (static_cast<size_t>(nt) * kt_total + kt_begin) * args.blk_bytes;
      const uint32_t tx = static_cast<uint32_t>(args.blk_bytes + C::kXBytes);
      const int pre = num_kt < C::kStages ? num_kt : C::kStages;
      // the weight stream does not depend on the preceding grid: start it
      // before waiting for the activations
      for (int i = 0; i < pre; ++i) {
        mbar_arrive_expect_tx(bar_full + 8 * i, tx);
        bulk_load(base + C::kOffRaw + i * kRawStageBytes, src + static_cast<size_t>(i) * args.blk_bytes,
                  static_cast<uint32_t>(args.blk_bytes), bar_full + 8 * i, policy);
      }
      grid_dependency_wait();
      for (int i = 0; i < pre; ++i)
        tma_load_2d(base + C::kOffX + i * C::kXBytes, &tmap_x, (kt_begin + i) * kTileK, m0,
                    bar_full + 8 * i);
      int i = pre;
      for (; i < num_kt; ++i) {
        const int s = i % C::kStages;
        if (!mbar_wait(bar_empty + 8 * s, ((i / C::kStages) & 1) ^ 1, abort_flag, &g_error_word,
                       kErrProducer))
          break;
        mbar_arrive_expect_tx(bar_full + 8 * s, tx);
        bulk_load(base + C::kOffRaw + s * kRawStageBytes, src + static_cast<size_t>(i) * args.blk_bytes,
                  static_cast<uint32_t>(args.blk_bytes), bar_full + 8 * s, policy);
        tma_load_2d(base + C::kOffX + s * C::kXBytes, &tmap_x, (kt_begin + i) * kTileK, m0,
                    bar_full + 8 * s);
      }
      if (i < num_kt) {
        // aborted: the copies already issued must land before the CTA exits
        for (int j = (i > C::kStages ? i - C::kStages : 0); j < i; ++j)
          drain_wait(bar_full + 8 * (j % C::kStages), (j / C::kStages) & 1);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(kTileN, TOK);
      const uint32_t d_tmem = tmem + C::kTmemD;
      for (int i = 0; i < num_kt; ++i) {
        const int s = i % C::kStages, d = i % C::kDqStages;
        if (!mbar_wait(bar_full + 8 * s, (i / C::kStages) & 1, abort_flag, &g_error_word, kErrMma))
          break;
        if (!mbar_wait(bar_dqfull + 8 * d, (i / C::kDqStages) & 1, abort_flag, &g_error_word,
                       kErrMma))
          break;
        tc_fence_after_sync();
        const uint32_t a_tmem = tmem + C::kTmemA + 32 * d;
        const uint32_t b_addr = base + C::kOffX + s * C::kXBytes;
#pragma unroll
        for (int kk = 0; kk < kTileK / 32; ++kk) {
          // K = 32 bytes per instruction: 8 tensor-memory columns of A, 32
          // bytes along the swizzled rows of B
          mma_i8_ts(d_tmem, a_tmem + 8 * kk, smem_desc_sw128(b_addr + kk * 32), idesc,
                    (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar_empty + 8 * s);     // X tile and raw block of stage s are free
        mma_commit(bar_dqempty + 8 * d);   // A stage d is free
      }
      mma_commit(bar_acc);                 // accumulator complete (or aborted)
      drain_wait(bar_acc, 0);              // no MMA in flight past this point
    }
  } else {
    // ---------------------------------------------------------------- dequantizers
    const int wg = (warp - 2) >> 2;        // warpgroup: even or odd k-tiles
    const int q4 = warp & 3;               // tensor-memory lane quarter of this warp
    const int r = q4 * 32 + lane;          // weight row (output channel) within the tile
    const uint32_t row_tmem = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const int gpt = kTileK / args.group;
    for (int i = wg; i < num_kt; i += 2) {
      const int s = i % C::kStages, d = i % C::kDqStages;
      if (!mbar_wait(bar_full + 8 * s, (i / C::kStages) & 1, abort_flag, &g_error_word,
                     kErrDequant)) {
        ok = false;
        break;
      }
      if (i >= C::kDqStages &&
          !mbar_wait(bar_dqempty + 8 * d, ((i / C::kDqStages) & 1) ^ 1, abort_flag, &g_error_word,
                     kErrDequant)) {
        ok = false;
        break;
      }
      const uint8_t* blk = smem + C::kOffRaw + s * kRawStageBytes;
      uint32_t s2v[2], bias[2];
#pragma unroll
      for (int gl = 0; gl < 2; ++gl) {
        if (gl < gpt) {
          s2v[gl] = blk[kCodesBytes + gl * kTileN + r];
          const uint32_t zb = blk[kCodesBytes + gpt * kTileN + gl * 64 + (r >> 1)];
          const uint32_t zv = (r & 1) ? (zb >> 4) : (zb & 15u);
          bias[gl] = dq_bias(zv, s2v[gl]);
        } else {
          s2v[gl] = s2v[0];
          bias[gl] = bias[0];
        }
      }
      uint32_t out[32];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 w = *reinterpret_cast<const uint4*>(blk + (j * kTileN + r) * 16);
        const int gl = (gpt == 2) ? (j >> 1) : 0;
        const uint32_t sv = s2v[gl], bv = bias[gl];
        out[8 * j + 0] = dq_lanes(lo_codes(w.x), sv, bv);
        out[8 * j + 1] = dq_lanes(hi_codes(w.x), sv, bv);
        out[8 * j + 2] = dq_lanes(lo_codes(w.y), sv, bv);
        out[8 * j + 3] = dq_lanes(hi_codes(w.y), sv, bv);
        out[8 * j + 4] = dq_lanes(lo_codes(w.z), sv, bv);
        out[8 * j + 5] = dq_lanes(hi_codes(w.z), sv, bv);
        out[8 * j + 6] = dq_lanes(lo_codes(w.w), sv, bv);
        out[8 * j + 7] = dq_lanes(hi_codes(w.w), sv, bv);
      }
      // one 128-byte row of the INT8 A operand: column c holds K bytes 4c..4c+3
      tmem_st_32x32b_x32(row_tmem + C::kTmemA + 32 * d, out);
      tmem_st_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_dqfull + 8 * d);
    }
  }

  // ------------------------------------------------------------------ epilogue
  // 1) accumulator -> slot [token column][row] (INT32) in the X ring
  uint32_t* slot = reinterpret_cast<uint32_t*>(smem + C::kOffX);
  const bool epi = warp >= 2;
  const int et = threadIdx.x - 64;         // epilogue thread 0..255
  if (epi) {
    const int wg = (warp - 2) >> 2;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const bool have = ok && mbar_wait(bar_acc, 0, abort_flag, &g_error_word, kErrEpilogue);
    tc_fence_after_sync();
    if (__all_sync(0xffffffffu, have && (*abort_flag == 0u))) {
      const uint32_t t_row = tmem + C::kTmemD + (static_cast<uint32_t>(q4 * 32) << 16);
#pragma unroll 1
      for (int c0 = 16 * wg; c0 < TOK; c0 += 32) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(t_row + c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) slot[(c0 + j) * kTileN + r] = v[j];
      }
    }
    if (args.Y) {
      grid_dependency_wait();   // sx comes from the preceding grid under PDL
      for (int c = et; c < TOK; c += kEpiThreads) {
        const int m = m0 + c;
        sx_s[c] = m < args.M ? __half2float(args.sx[m]) : 0.0f;
      }
    }
    epi_bar();
  }

  // 2) thread et owns rows 8*(et%16) .. +7 and token columns c = et/16 (mod 16)
  const int M = args.M, N = args.N;
  const int r8 = 8 * (et & 15);
  const int n = nt * kTileN + r8;
  const int c_first = et >> 4;
  int c_end = M - m0;
  if (c_end > TOK) c_end = TOK;
  if (epi && splits > 1) {
    // publish this split's partial tile, then count the arrival: the
    // barrier orders every thread's stores before thread 0's fence, and the
    // fence is cumulative (release); the last arrival fences again (acquire)
    // before the barrier that releases the readers
    int32_t* part = args.ws_part + (static_cast<size_t>(mt * splits + split) * TOK) * N + n;
    for (int c = c_first; c < c_end; c += 16) {
      const uint4* sv = reinterpret_cast<const uint4*>(slot + c * kTileN + r8);
      uint4* dst = reinterpret_cast<uint4*>(part + static_cast<size_t>(c) * N);
      __stcg(dst, sv[0]);
      __stcg(dst + 1, sv[1]);
    }
    epi_bar();
    if (et == 0) {
      __threadfence();
      const bool last = arrive_last(args.ws_count + mt * (N / kTileN) + nt, splits);
      if (last) __threadfence();
      *last_flag = last ? 1u : 0u;
    }
    epi_bar();
  }
  const bool writer = epi && (*abort_flag == 0u) && (splits == 1 || *last_flag != 0u);
  if (writer) {
    float s1o[8];
    if (args.Y) {
      const uint4 sv = *reinterpret_cast<const uint4*>(args.s1 + n);
      const __half2* h = reinterpret_cast<const __half2*>(&sv);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __half22float2(h[j]);
        s1o[2 * j] = f.x;
        s1o[2 * j + 1] = f.y;
      }
    }
    const int32_t* parts = args.ws_part + (static_cast<size_t>(mt * splits) * TOK) * N + n;
#pragma unroll 2
    for (int c = c_first; c < c_end; c += 16) {
      const uint4* sv = reinterpret_cast<const uint4*>(slot + c * kTileN + r8);
      uint4 v0 = sv[0], v1 = sv[1];
      for (int q = 0; q < splits; ++q) {
        if (q == split) continue;
        const int32_t* p = parts + (static_cast<size_t>(q) * TOK + c) * N;
        v0 = add4(v0, ld_cg_v4(p));
        v1 = add4(v1, ld_cg_v4(p + 4));
      }
      const size_t o = static_cast<size_t>(m0 + c) * N + n;
      if (args.acc) {
        reinterpret_cast<uint4*>(args.acc + o)[0] = v0;
        reinterpret_cast<uint4*>(args.acc + o)[1] = v1;
      } else {
        const float sxf = sx_s[c];
        const int32_t a[8] = {static_cast<int32_t>(v0.x), static_cast<int32_t>(v0.y),
                              static_cast<int32_t>(v0.z), static_cast<int32_t>(v0.w),
                              static_cast<int32_t>(v1.x), static_cast<int32_t>(v1.y),
                              static_cast<int32_t>(v1.z), static_cast<int32_t>(v1.w)};
        uint32_t pk[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const __half2 y = __floats2half2_rn(
              __fmul_rn(static_cast<float>(a[2 * j]), __fmul_rn(sxf, s1o[2 * j])),
              __fmul_rn(static_cast<float>(a[2 * j + 1]), __fmul_rn(sxf, s1o[2 * j + 1])));
          pk[j] = *reinterpret_cast<const uint32_t*>(&y);
        }
        *reinterpret_cast<uint4*>(args.Y + o) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
    }
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ----------------------------------------------------------------------------
// Host side
// ----------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

struct Plan {
  int tok, splits, m_tiles, n_tiles, stages;
};

bool splittable(const Plan& p) {
  return static_cast<long>(p.m_tiles) * p.n_tiles <= kMaxCounterTiles;
}

int stages_for(int tok) { return tok <= 32 ? 8 : (tok <= 64 ? 6 : 4); }

bool valid_tok(int t) { return t == 16 || t == 32 || t == 64 || t == 128 || t == 256; }

int auto_tok(int M) { return M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128; }

int ctas_per_sm(int tok) { return tok <= 128 ? 2 : 1; }

int auto_splits(int tiles, int kt, int tok) {
  const long slots = static_cast<long>(sm_count()) * ctas_per_sm(tok);
  int best_s = 1;
  if (tiles >= slots) return 1;
  double best = 0.0;
  for (int s = 1; s <= 8 && s <= kt; ++s) {
    if (s > 1 && kt / s < 4) break;
    const long ctas = static_cast<long>(tiles) * s;
    const long waves = (ctas + slots - 1) / slots;
    const double eff = static_cast<double>(ctas) / static_cast<double>(waves * slots);
    if (eff > best + 1e-9) {
      best = eff;
      best_s = s;
    }
  }
  return best_s;
}

Plan make_plan(int M, int N, int K, int tok_req, int splits_req) {
  Plan p;
  p.n_tiles = N / kTileN;
  const int kt = K / kTileK;
  p.tok = tok_req ? tok_req : auto_tok(M);
  p.m_tiles = (M + p.tok - 1) / p.tok;
  p.stages = stages_for(p.tok);
  p.splits = splits_req ? splits_req : auto_splits(p.n_tiles * p.m_tiles, kt, p.tok);
  if (!splits_req && !splittable(p)) p.splits = 1;
  return p;
}

size_t ws_bytes_for(const Plan& p, int N) {
  if (p.splits <= 1) return 0;
  const size_t part = static_cast<size_t>(p.m_tiles) * p.splits * p.tok * N * 4;
  return kCounterBytes + part;
}

template <int TOK>
int launch_tok(const CUtensorMap& map, const GemmArgs& a, const Plan& p, cudaStream_t stream,
               bool pdl) {
  using C = Cfg<TOK>;
  static int configured_mask = 0;   // one bit per device id < 31
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QOQ_ERR_CUDA;
  const int bit = dev < 31 ? (1 << dev) : 0;
  if (!bit || !(__atomic_load_n(&configured_mask, __ATOMIC_ACQUIRE) & bit)) {
    if (cudaFuncSetAttribute(w4a8_gemm_kernel<TOK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kSmemBytes) != cudaSuccess)
      return QOQ_ERR_CUDA;
    if (bit) __atomic_fetch_or(&configured_mask, bit, __ATOMIC_RELEASE);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(p.n_tiles * p.splits), static_cast<unsigned>(p.m_tiles), 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  if (cudaLaunchKernelEx(&cfg, w4a8_gemm_kernel<TOK>, map, a) != cudaSuccess) return QOQ_ERR_CUDA;
  return QOQ_OK;
}

}  // namespace

int gemm_impl(const int8_t* X8, const void* sx, const void* packed, const void* s1, int M, int N,
              int K, int group, void* Y, int32_t* acc, int tok_req, int splits_req, void* ws,
              size_t ws_bytes, void* stream, bool pdl) {
  if (!X8 || !packed) return QOQ_ERR_INVALID_ARG;
  if ((Y == nullptr) == (acc == nullptr)) return QOQ_ERR_INVALID_ARG;
  if (Y && (!sx || !s1)) return QOQ_ERR_INVALID_ARG;
  if (M <= 0) return QOQ_ERR_INVALID_ARG;
  if (int st = check_weight_shape(N, K, group)) return st;
  if (!aligned16(X8) || !aligned16(packed) || (Y && !aligned16(Y)) || (acc && !aligned16(acc)) ||
      (sx && !aligned16(sx)) || (s1 && !aligned16(s1)) || (ws && !aligned16(ws)))
    return QOQ_ERR_INVALID_ARG;
  if (tok_req && !valid_tok(tok_req)) return QOQ_ERR_INVALID_ARG;
  if (splits_req && (splits_req < 1 || splits_req > 8 || splits_req > K / kTileK))
    return QOQ_ERR_INVALID_ARG;

  Plan p = make_plan(M, N, K, tok_req, splits_req);
  if (p.m_tiles > 65535) return QOQ_ERR_UNSUPPORTED;
  if (p.splits > 1 && !splittable(p)) {
    if (splits_req) return QOQ_ERR_UNSUPPORTED;
    p.splits = 1;
  }
  if (p.splits > 1 && (ws == nullptr || ws_bytes < ws_bytes_for(p, N))) {
    if (splits_req) return QOQ_ERR_INVALID_ARG;   // explicit split needs its workspace
    p.splits = 1;                                  // auto plan: do not split K
  }
  if (int st = check_device()) return st;
  EncodeTiledFn enc = encode_fn();
  if (!enc) return QOQ_ERR_CUDA;

  CUtensorMap map;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kTileK), static_cast<cuuint32_t>(p.tok)};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(X8), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return QOQ_ERR_CUDA;

  GemmArgs a;
  a.packed = static_cast<const uint8_t*>(packed);
  a.sx = static_cast<const __half*>(sx);
  a.s1 = static_cast<const __half*>(s1);
  a.Y = static_cast<__half*>(Y);
  a.acc = acc;
  a.ws_part = nullptr;
  a.ws_count = nullptr;
  if (p.splits > 1) {
    a.ws_count = static_cast<uint32_t*>(ws);
    a.ws_part = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + kCounterBytes);
  }
  a.M = M;
  a.N = N;
  a.K = K;
  a.group = group;
  a.splits = p.splits;
  a.blk_bytes = static_cast<int>(block_bytes(group));

  cudaStream_t s = as_stream(stream);
  switch (p.tok) {
    case 16: return launch_tok<16>(map, a, p, s, pdl);
    case 32: return launch_tok<32>(map, a, p, s, pdl);
    case 64: return launch_tok<64>(map, a, p, s, pdl);
    case 128: return launch_tok<128>(map, a, p, s, pdl);
    default: return launch_tok<256>(map, a, p, s, pdl);
  }
}

size_t gemm_ws_bytes(int M, int N, int K, int tok_req, int splits_req) {
  const Plan p = make_plan(M, N, K, tok_req, splits_req);
  if (!splittable(p)) return 0;
  return ws_bytes_for(p, N);
}

}  // namespace qoq

using namespace qoq;

extern "C" size_t qoq_gemm_workspace_bytes(int M, int N, int K, int group) {
  if (M <= 0 || check_weight_shape(N, K, group) != QOQ_OK) return 0;
  return gemm_ws_bytes(M, N, K, 0, 0);
}

extern "C" size_t qoq_gemm_workspace_bytes_config(int M, int N, int K, int group, int tok_tile,
                                                  int splits) {
  if (M <= 0 || check_weight_shape(N, K, group) != QOQ_OK) return 0;
  if (tok_tile && !valid_tok(tok_tile)) return 0;
  if (splits < 0 || splits > 8 || splits > K / kTileK) return 0;
  return gemm_ws_bytes(M, N, K, tok_tile, splits);
}

extern "C" int qoq_w4a8_gemm(const int8_t* X8, const void* sx, const void* packed, const void* s1,
                             int M, int N, int K, int group, void* Y, void* ws, size_t ws_bytes,
                             void* stream) {
  if (!Y) return QOQ_ERR_INVALID_ARG;
  return gemm_impl(X8, sx, packed, s1, M, N, K, group, Y, nullptr, 0, 0, ws, ws_bytes, stream,
                   false);
}

extern "C" int qoq_w4a8_gemm_i32(const int8_t* X8, const void* packed, int M, int N, int K,
                                 int group, int32_t* acc, void* ws, size_t ws_bytes,
                                 void* stream) {
  if (!acc) return QOQ_ERR_INVALID_ARG;
  return gemm_impl(X8, nullptr, packed, nullptr, M, N, K, group, nullptr, acc, 0, 0, ws, ws_bytes,
                   stream, false);
}

extern "C" int qoq_w4a8_gemm_config(const int8_t* X8, const void* sx, const void* packed,
                                    const void* s1, int M, int N, int K, int group, void* Y,
                                    int32_t* acc, int tok_tile, int splits, void* ws,
                                    size_t ws_bytes, void* stream) {
  return gemm_impl(X8, sx, packed, s1, M, N, K, group, Y, acc, tok_tile, splits, ws, ws_bytes,
                   stream, false);
}

extern "C" int qoq_w4a8_linear(const void* X, int M, int K, const void* packed, const void* s1,
                               int N, int group, int8_t* X8, void* sx, void* Y, void* ws,
                               size_t ws_bytes, void* stream) {
  if (!X || !X8 || !sx || !Y || !packed || !s1) return QOQ_ERR_INVALID_ARG;
  if (M <= 0) return QOQ_ERR_INVALID_ARG;
  if (int st = check_weight_shape(N, K, group)) return st;
  if (!aligned16(X) || !aligned16(X8) || !aligned16(sx) || !aligned16(Y) || !aligned16(packed) ||
      !aligned16(s1) || (ws && !aligned16(ws)))
    return QOQ_ERR_INVALID_ARG;
  if (int st = check_device()) return st;
  if (int st = launch_act_quant(X, M, K, X8, sx, stream)) return st;
  // both kernels are this library's: the GEMM reads nothing the quantizer
  // writes before its grid-dependency wait, so it may overlap its tail
  return gemm_impl(X8, sx, packed, s1, M, N, K, group, Y, nullptr, 0, 0, ws, ws_bytes, stream,
                   true);
}

extern "C" int qoq_gemm_plan(int M, int N, int K, int group, int* tok_tile, int* splits, int* ctas,
                             int* stages) {
  if (M <= 0) return QOQ_ERR_INVALID_ARG;
  if (int st = check_weight_shape(N, K, group)) return st;
  const Plan p = make_plan(M, N, K, 0, 0);
  if (tok_tile) *tok_tile = p.tok;
  if (splits) *splits = p.splits;
  if (ctas) *ctas = p.n_tiles * p.m_tiles * p.splits;
  if (stages) *stages = p.stages;
  return QOQ_OK;
}

extern "C" int qoq_device_error(unsigned int* value, int clear) {
  if (!value) return QOQ_ERR_INVALID_ARG;
  if (int st = check_device()) return st;
  if (cudaMemcpyFromSymbol(value, g_error_word, sizeof(unsigned int)) != cudaSuccess)
    return QOQ_ERR_CUDA;
  if (clear) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(unsigned int)) != cudaSuccess)
      return QOQ_ERR_CUDA;
  }
  return QOQ_OK;
}

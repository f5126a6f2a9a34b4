// W4A8 GEMM for sm_100a: Y[m, n] = fp16((sum_k X8[m,k] * dq[n,k]) * sx[m] * s1[n]).
//
// Method: "QServe: W4A8KV4 Quantization and System Co-design for Efficient
// LLM Serving" -- Methods, 1) Algorithm: QoQ (all GEMMs on INT8 tensor cores
// after progressive group quantization) and 2) System: QServe (UINT4 -> INT8
// with register-level parallelism, "subtraction after multiplication");
// Background (per-group W4A4 dequantizes INT32 partial sums in its main loop,
// this kernel scales once, after the whole K reduction).
//
// Persistent kernel, one CTA per SM.  A work unit is a 128-channel x
// TOK-token output tile over a range of K (the weights are the MMA's M operand
// and the tokens its N operand, so one decode token still fills the 128-row
// tensor-core tile).  Units are ordered channel-tile major, token tile next,
// K split innermost, so the CTAs running at the same time share weight blocks
// through L2 and every weight byte comes from HBM about once.  A pipeline
// stage covers two k-tiles of 128 for token tiles up to 128, one for the
// wider tiles (176, 192, 256).
//   warp 0       X producer: tensor-map copies of the X8 tiles (128-byte
//                swizzle) into the X ring, refilled when the stage's MMAs
//                completed;
//   last warp    W producer: one bulk copy of the stage's packed weight
//                blocks into the weight ring, refilled as soon as the
//                dequantizers hold the blocks in registers, so the weight
//                stream runs ahead of the MMAs;
//   warp 1       owns tensor memory and issues tcgen05.mma.kind::i8 (M = 128,
//                N = TOK, K = 32 per instruction) with the INT8 weights read
//                from tensor memory and X8 from shared memory, into one of two
//                INT32 accumulators in tensor memory (double buffered); one
//                commit per stage frees its X8 tiles and A columns;
//   warps 2..     three or four dequantizing warpgroups (four for token
//                tiles up to 64) taking stages in turn: each
//                thread turns one weight row of the UINT4 blocks into INT8
//                (four byte lanes per 32-bit multiply-add) and writes one
//                128-byte row per k-tile into the stage's tensor-memory
//                columns with tcgen05.st;
//   next 4 warps epilogue: tcgen05.ld of a finished accumulator, one FP32
//                scale per element, a transpose through shared memory and
//                16-byte stores, overlapping the next unit's main loop.
// When K is split, each epilogue warp writes its 32-channel slice of the INT32
// partial tile to the caller's workspace, and the last warp to arrive at a
// slice (an arrival counter per slice) adds the slices up exactly and runs
// the scaling.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "qoq.h"
#include "qoq_actq.cuh"
#include "qoq_device.cuh"
#include "qoq_internal.h"

namespace qoq {

__device__ unsigned int g_error_word = 0;

namespace {

constexpr int kRawStageBytes = 8576;             // largest packed block (group 64)
constexpr int kTmemCols = 512;
constexpr int kStageBytesEpi = 32 * 16 * 4;      // per epilogue warp: 16 columns x 32 rows
// The workspace starts with a fixed region of arrival counters, so that
// counter words never share memory with the partial sums of a launch of
// another shape.  Each epilogue warp counts the arrivals at its own 32-channel
// slice of an output tile, so a tile has four counters.
constexpr int kSlicesPerTile = 4;
constexpr int kMaxCounterTiles = 1024;
constexpr size_t kCounterBytes = kMaxCounterTiles * kSlicesPerTile * 4;
// A GEMM quantizes its own activations when its token rows (FP16) fit this
// shared-memory staging area: every CTA copies them in, computes each row's
// scale and writes the INT8 tiles of its K range straight into its X ring.
constexpr int kMaxFusedRowBytes = 48 * 1024;

template <int TOK, bool kCluster = false, bool kFuseX = false>
struct Cfg {
  // One ring of kStages stages.  A stage covers kNB consecutive k-tiles of
  // 128 (the last stage of a unit may cover fewer): their X8 tiles and packed
  // weight blocks in shared memory, and the dequantized INT8 weights in tensor
  // memory columns kACols s .. kACols s + kACols - 1.  Two k-tiles per stage
  // halve the per-stage work of the single-warp producer and MMA loops, whose
  // wait / issue / commit sequence costs about as much as the MMAs of one
  // 128 x 128 x 128 k-tile.  kAcc accumulators of TOK columns let the
  // epilogue of one unit overlap the main loop of the next.
  // Warp layout: producers and MMA (warps 0, 1), kDqGroups dequantizing
  // warpgroups, four epilogue warps, the weight producer last.  Small token
  // tiles (decode) are limited by how fast one CTA dequantizes its share of
  // the weights, so they get four warpgroups; from 128 tokens on the SM's
  // issue slots are the limit and three warpgroups run faster.
  static constexpr int kDqGroups = TOK <= 64 ? 4 : 3;
  static constexpr int kWarpEpi0 = 2 + 4 * kDqGroups;        // first epilogue warp
  static constexpr int kWarpW = kWarpEpi0 + 4;               // weight producer warp
  static constexpr int kThreads = 32 * (kWarpW + 1);
  static constexpr int kNB = TOK <= 128 ? 2 : 1;
  static constexpr int kXBytes = TOK * kTileK;                // one 128-byte-wide X8 tile
  static constexpr int kStageX = kNB * kXBytes;
  static constexpr int kStageRaw = kNB * kRawStageBytes;
  static constexpr int kStages = TOK <= 32 ? 7 : TOK == 64 ? 6 : TOK == 176 ? 5 : 4;
  // The weight ring may be deeper than the X ring: its slots are small and
  // its consumers (the dequantizers) have the longest latency.  It must not
  // be shallower (see the parity note at the dequantizers' waits).
  static constexpr int kWStages = TOK <= 64 ? kStages : TOK == 128 ? 5 : TOK == 256 ? 8 : 10;
  static_assert(kWStages >= kStages, "weight ring at least as deep as the X ring");
  // a dequantizer's A-slot wait is exact only if its own previous stage
  // (g - kDqGroups) already implied the slot's older phase
  static_assert(kStages >= kDqGroups, "at least as many stages as dequantizing warpgroups");
  static constexpr int kAcc = TOK <= 192 ? 2 : 1;
  static constexpr int kACols = 32 * kNB;                     // tensor-memory columns of A per stage
  // Tensor-memory columns: up to 128 tokens the A slots come first and the
  // accumulators after them (at a multiple of TOK); for the wide token tiles
  // of 176 and 192 the two accumulators come first (at columns 0 and TOK)
  // and the A slots after them, at a multiple of 32.
  static constexpr bool kAccFirst = TOK == 176 || TOK == 192;
  static constexpr int kTmemA = kAccFirst ? kAcc * TOK : 0;
  static constexpr int kTmemD =
      kAccFirst ? 0 : ((kStages * kACols + TOK - 1) / TOK) * TOK;   // accumulators
  static constexpr int kOffX = 0;
  static constexpr int kOffRaw = kOffX + kStages * kStageX;
  static constexpr int kOffEpi = kOffRaw + kWStages * kStageRaw;
  static constexpr int kOffSx = kOffEpi + 4 * kStageBytesEpi;          // 4 warps x TOK floats
  static constexpr int kOffBar = kOffSx + 4 * TOK * 4;
  // The kernel variant that splits K across a cluster (token tiles up to 32)
  // has eight more barriers and the leader CTA's reduction buffer, which
  // receives the INT32 partial tiles of the other CTAs:
  // [slot = rank - 1][epilogue warp][token][32 channels].
  static constexpr int kRedBars = kCluster ? 8 : 0;
  // The variant that quantizes its own activations has one more barrier (its
  // token rows landed), the FP16 rows and each row's scale and reciprocal.
  static constexpr int kFuseBars = kFuseX ? 2 : 0;
  static constexpr int kNumBars = 3 * kStages + 2 * kWStages + 2 * kAcc + 1 + kRedBars + kFuseBars;
  static constexpr int kOffMisc = kOffBar + 8 * kNumBars;
  static constexpr int kMaxClusterSplit = !kCluster ? 1 : TOK <= 16 ? 8 : TOK <= 32 ? 3 : 1;
  static constexpr int kRedSlotBytes = kTileN * TOK * 4;
  static constexpr int kOffRed = ((kOffMisc + 32 + 127) / 128) * 128;
  static constexpr int kRedBytes = (kMaxClusterSplit - 1) * kRedSlotBytes;
  static constexpr int kOffXrow = kOffRed + kRedBytes;
  static constexpr int kOffSxq = kOffXrow + (kFuseX ? kMaxFusedRowBytes : 0);
  static constexpr int kSmemBytes = kOffSxq + (kFuseX ? TOK * 8 : 0) + 1024;   // + alignment slack
  static_assert(!kFuseX || (TOK == 16 && !kCluster), "own activations: 16-token tiles");
  static_assert(kOffXrow % 128 == 0, "bulk copy destination alignment");
  static_assert(!kCluster || TOK <= 32, "K split across a cluster for token tiles up to 32");
  static_assert(kOffRaw % 1024 == 0 && kXBytes % 1024 == 0, "swizzled tiles need 1 KiB alignment");
  static_assert(kOffBar % 8 == 0, "mbarriers need 8-byte alignment");
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
  static_assert(kTmemD + kAcc * TOK <= kTmemCols, "tensor memory");
  static_assert(kAccFirst ? kTmemA + kACols * kStages <= kTmemCols
                          : kTmemA + kACols * kStages <= kTmemD,
                "tensor memory A stages");
  static_assert(kTmemA % 32 == 0 && kTmemD % TOK == 0, "tensor memory alignment");
  static_assert(kStageRaw % 16 == 0, "bulk copies need 16-byte alignment");
};

struct GemmArgs {
  const uint8_t* packed;
  const __half* sx;
  const __half* s1;
  __half* Y;
  int32_t* acc;
  int32_t* ws_part;     // [m_tile][split][TOK][N] partial sums (splits > 1)
  uint32_t* ws_count;   // [m_tile][n_tile] arrival counters (zero between launches)
  int M, N, K, group;
  int splits;
  int m_tiles, n_tiles;
  int units;            // n_tiles * m_tiles * splits
  int blk_bytes;
  float rcp_splits;     // 1 / splits and 1 / m_tiles, rounded (for small_div)
  float rcp_mtiles;
  int w_dep_wait;       // the weight producer waits for the preceding grid (it may
                        // have written the weights) before its first copy
  int cs;               // K split across a cluster of cs CTAs (1: none); then
                        // splits == cs and the split partials never leave the
                        // cluster (no workspace)
  // The GEMM that quantizes its own activations (X != nullptr): every CTA
  // copies the M FP16 token rows of X into shared memory, computes their
  // scales and quantizes the tiles it multiplies; the CTAs of the first
  // channel tile also write X8 (the tiles of their K range) and CTA 0 writes
  // sx, so the caller sees the same X8 / sx as from the stand-alone quantizer.
  const __half* X;
  int8_t* X8;
};

struct Unit {
  int nt, mt, split, kt_begin, num_kt;
};

// n / d for 0 <= n < 2^22 and d >= 1 without an integer division: the
// binary32 product n * rn(1/d), truncated, is within one of the quotient (its
// relative error is below 2^-22), and the remainder check corrects it.
__device__ __forceinline__ int small_div(int n, int d, float rcp_d) {
  int q = static_cast<int>(__fmul_rz(static_cast<float>(n), rcp_d));
  const int r = n - q * d;
  if (r < 0) {
    --q;
  } else if (r >= d) {
    ++q;
  }
  return q;
}

__device__ __forceinline__ Unit unit_of(const GemmArgs& a, int u, int kt_total) {
  Unit w;
  int rest = u;
  if (a.splits == 1) {
    w.split = 0;
    w.kt_begin = 0;
    w.num_kt = kt_total;
  } else {
    rest = small_div(u, a.splits, a.rcp_splits);
    w.split = u - rest * a.splits;
    w.kt_begin = small_div(w.split * kt_total, a.splits, a.rcp_splits);
    w.num_kt = small_div((w.split + 1) * kt_total, a.splits, a.rcp_splits) - w.kt_begin;
  }
  w.nt = small_div(rest, a.m_tiles, a.rcp_mtiles);
  w.mt = rest - w.nt * a.m_tiles;
  return w;
}

// Bounded wait that ignores the abort flag: used only to drain work already
// in flight before a CTA tears down.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return;
  const long long t0 = sm_clock();
  while (!mbar_try_wait_sleep(bar, parity, kSuspendHintNs)) {
    if (sm_clock() - t0 > kWaitLimitCycles) {
      atomicOr(&g_error_word, kErrProducer);
      return;
    }
  }
}

// Register one warp's arrival at its slice of an output tile (lane 0, after
// the warp's partial slice is written and a warp barrier ordered the lanes'
// stores before this thread).  The add has acquire-release semantics at GPU
// scope: it releases those stores (cumulatively) to the last arrival and, for
// the last arrival, acquires the stores of the others, in one round trip.
// The counter counts the arrivals of the current launch; the last of `splits`
// arrivals resets it to zero, so the counter region returns to zero after
// every launch that completes.
__device__ __forceinline__ bool arrive_last(uint32_t* ctr, int splits) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
               : "=r"(old)
               : "l"(ctr)
               : "memory");
  if (old >= static_cast<uint32_t>(splits)) atomicOr(&g_error_word, kErrCounter);
  const bool last = old == static_cast<uint32_t>(splits - 1);
  if (last) atomicExch(ctr, 0u);
  return last;
}

// One weight row of one packed block in registers: its 64 code bytes and
// the group scale / dequantization bias of its (one or two) groups.
struct RowBlock {
  uint4 v[4];
  uint32_t s2v[2], bias[2];
};

__device__ __forceinline__ void load_row_block(const uint8_t* blk, int r, int gpt, RowBlock& rb) {
#pragma unroll
  for (int gl = 0; gl < 2; ++gl) {
    if (gl < gpt) {
      rb.s2v[gl] = blk[kCodesBytes + gl * kTileN + r];
      const uint32_t zb = blk[kCodesBytes + gpt * kTileN + gl * 64 + (r >> 1)];
      const uint32_t zv = (r & 1) ? (zb >> 4) : (zb & 15u);
      rb.bias[gl] = dq_bias(zv, rb.s2v[gl]);
    } else {
      rb.s2v[gl] = rb.s2v[0];
      rb.bias[gl] = rb.bias[0];
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) rb.v[j] = *reinterpret_cast<const uint4*>(blk + (j * kTileN + r) * 16);
}

// Four byte lanes per 32-bit op into INT8 and one 128-byte row into tensor
// memory at `taddr`: column c holds K bytes 4c..4c+3.  The source registers
// are read at issue; the caller waits for the stores once per stage.
__device__ __forceinline__ void dequant_store_row_block(const RowBlock& rb, int gpt,
                                                        uint32_t taddr) {
  uint32_t out[32];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    // second group of the block (group 64) for the last two 32-byte chunks;
    // a select rather than an index keeps the struct in registers
    const bool g1 = gpt == 2 && j >= 2;
    const uint32_t sv = g1 ? rb.s2v[1] : rb.s2v[0];
    const uint32_t bv = g1 ? rb.bias[1] : rb.bias[0];
    out[8 * j + 0] = dq_lanes(lo_codes(rb.v[j].x), sv, bv);
    out[8 * j + 1] = dq_lanes(hi_codes(rb.v[j].x), sv, bv);
    out[8 * j + 2] = dq_lanes(lo_codes(rb.v[j].y), sv, bv);
    out[8 * j + 3] = dq_lanes(hi_codes(rb.v[j].y), sv, bv);
    out[8 * j + 4] = dq_lanes(lo_codes(rb.v[j].z), sv, bv);
    out[8 * j + 5] = dq_lanes(hi_codes(rb.v[j].z), sv, bv);
    out[8 * j + 6] = dq_lanes(lo_codes(rb.v[j].w), sv, bv);
    out[8 * j + 7] = dq_lanes(hi_codes(rb.v[j].w), sv, bv);
  }
  tmem_st_32x32b_x32(taddr, out);
}

// The weight producer's walk over its units' stages, resumable: run() with
// `prologue` issues stages until the weight ring is full and never waits;
// without, it continues to the end, waiting for free slots.  The whole warp
// runs it; one elected lane issues each bulk copy.
struct WeightStream {
  int u, i;
  uint32_t g;
  Unit w;
  const uint8_t* src;
  uint64_t policy;

  __device__ __forceinline__ void load_unit(const GemmArgs& a, int kt_total) {
    w = unit_of(a, u, kt_total);
    src = a.packed + (static_cast<size_t>(w.nt) * kt_total + w.kt_begin) * a.blk_bytes;
    i = 0;
  }

  __device__ __forceinline__ void begin(const GemmArgs& a, int kt_total) {
    policy = l2_policy_evict_first();
    g = 0;
    u = blockIdx.x;
    i = 0;
    if (u < a.units) load_unit(a, kt_total);
  }

  template <class C>
  __device__ __forceinline__ bool run(const GemmArgs& a, uint32_t base, uint32_t bar_wfull,
                                      uint32_t bar_wempty, volatile uint32_t* abort_flag,
                                      bool prologue) {
    constexpr int SW = C::kWStages;
    const int kt_total = a.K / kTileK;
    while (u < a.units) {
      const int nsteps = (w.num_kt + C::kNB - 1) / C::kNB;
      if (i >= nsteps) {
        u += gridDim.x;
        if (u >= a.units) break;
        load_unit(a, kt_total);
        continue;
      }
      const int sw = g % SW;
      if (g >= SW) {
        if (prologue) return true;
        if (!__all_sync(0xffffffffu, mbar_wait(bar_wempty + 8 * sw, ((g / SW) & 1) ^ 1,
                                               abort_flag, &g_error_word, kErrProducer)))
          return false;
      }
      if (elect_one()) {
        const int nb = min(C::kNB, w.num_kt - i * C::kNB);
        mbar_arrive_expect_tx(bar_wfull + 8 * sw, static_cast<uint32_t>(nb * a.blk_bytes));
        bulk_load(base + C::kOffRaw + sw * C::kStageRaw,
                  src + static_cast<size_t>(i * C::kNB) * a.blk_bytes,
                  static_cast<uint32_t>(nb * a.blk_bytes), bar_wfull + 8 * sw, policy);
      }
      __syncwarp();
      ++i;
      ++g;
    }
    return true;
  }
};

// kGateUp: the weight is a fused gate_up projection packed with
// qoq_quantize_weights_gate_up (tile rows 0..63 gate, 64..127 up of the same
// 64 channels); the epilogue writes H = fp16(silu(gate) * up), M x (N / 2),
// instead of Y.
template <int TOK, bool kCluster, bool kFuseX, bool kGateUp>
__global__ void __launch_bounds__(Cfg<TOK>::kThreads, 1)
w4a8_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const GemmArgs args) {
  using C = Cfg<TOK, kCluster, kFuseX>;
  static_assert(!kGateUp || (!kCluster && !kFuseX), "gate_up: no cluster split, X8 given");
  constexpr int S = C::kStages;
  // a launch with less shared memory than this layout needs does nothing
  // (every thread returns before any barrier) and records the mistake
  if (dynamic_smem_bytes() < static_cast<uint32_t>(C::kSmemBytes)) {
    if (threadIdx.x == 0) atomicOr(&g_error_word, kErrLaunch);
    return;
  }
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t base = (raw_base + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw_base);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int kt_total = args.K / kTileK;

  // Two rings of S slots, both indexed by the running stage g (slot g % S):
  //   X ring     xfull[s]: the X8 tiles of stage g landed (X producer);
  //              empty[s]: the MMAs of stage g completed, which frees both the
  //              X8 tiles and the tensor-memory A columns of slot s;
  //   weight ring wfull[s]: the packed blocks of stage g landed (W producer);
  //              wempty[s]: the dequantizers copied them into registers.
  // dqfull[s]: A operand of stage g written and its X8 tiles landed (the MMA
  // warp waits on this one barrier).  The weight ring is released as soon as
  // the blocks are in registers, so the weight stream runs ahead of the MMAs
  // and the weight copy overlaps the previous stages' dequantization.
  constexpr int SW = C::kWStages;
  const uint32_t bar_xfull = base + C::kOffBar;
  const uint32_t bar_empty = bar_xfull + 8 * S;
  const uint32_t bar_dqfull = bar_empty + 8 * S;
  const uint32_t bar_wfull = bar_dqfull + 8 * S;
  const uint32_t bar_wempty = bar_wfull + 8 * SW;
  const uint32_t bar_accfull = bar_wempty + 8 * SW;
  const uint32_t bar_accempty = bar_accfull + 8 * C::kAcc;
  const uint32_t bar_drain = bar_accempty + 8 * C::kAcc;
  // K split across a cluster: red_full[q] (leader CTA) counts the other
  // CTAs' partial slices of epilogue warp q; red_free[q] (every other CTA)
  // completes when the leader has added them up and the buffer may be
  // written again.
  const uint32_t bar_red_full = bar_drain + 8;
  const uint32_t bar_red_free = bar_red_full + 8 * 4;
  // own activations: the FP16 token rows landed in shared memory; this CTA
  // has written X8 (the X producer waits for this one)
  const uint32_t bar_xrow = bar_drain + 8 + 8 * C::kRedBars;
  const uint32_t bar_x8 = bar_xrow + 8;
  const int cs = kCluster ? args.cs : 1;
  const uint32_t crank = cs > 1 ? cluster_ctarank() : 0u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + C::kOffMisc + 4);

  if (warp == 0) {
    // the barriers are contiguous from bar_xfull: xfull, empty, dqfull (S
    // each), wfull, wempty (SW each), accfull, accempty (kAcc each), drain;
    // dqfull, wempty and accempty count the four warps of a warpgroup; the
    // lanes of warp 0 initialize all but the weight ring's, which the weight
    // producer initializes itself
    for (int i = lane; i < C::kNumBars - C::kRedBars - C::kFuseBars; i += 32) {
      const int acc0 = 3 * S + 2 * SW;
      if (i >= 3 * S && i < acc0) continue;
      const bool four = (i >= 2 * S && i < 3 * S) ||
                        (i >= acc0 + C::kAcc && i < acc0 + 2 * C::kAcc);
      mbar_init(bar_xfull + 8 * i, four ? 4u : 1u);
    }
    if (kCluster) {
      if (lane < 4) mbar_init(bar_red_full + 8 * lane, cs > 1 ? static_cast<uint32_t>(cs - 1) : 1u);
      else if (lane < 8) mbar_init(bar_red_free + 8 * (lane - 4), 1u);
    }
    if (kFuseX && lane < 2) mbar_init(bar_xrow + 8 * lane, 1u);
    if (lane == 0) {
      *abort_flag = 0u;
      prefetch_tensormap(&tmap_x);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  // The weight producer starts the weight stream before the start-up
  // barrier: its own barriers, then (once the preceding grid completed, if
  // that grid may have written the weights) the first SW stages of bulk
  // copies, all without waiting for a free slot.
  WeightStream wstream;
  if (warp == C::kWarpW) {
    for (int i = lane; i < 2 * SW; i += 32) mbar_init(bar_wfull + 8 * i, i < SW ? 1u : 4u);
    fence_mbar_init();
    __syncwarp();
    wstream.begin(args, kt_total);
    if (args.w_dep_wait) grid_dependency_wait();
    wstream.run<C>(args, base, bar_wfull, bar_wempty, abort_flag, /*prologue=*/true);
  }
  tc_fence_before_sync();
  __syncthreads();
  // the leader's reduction barriers must be initialized before another CTA
  // of the cluster arrives on them
  if (cs > 1) cluster_sync_all();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // -------------------------------------------------------------- X producer
    // The whole warp runs the loop and waits; one elected lane issues copies.
    uint32_t g = 0;              // running stage index of this CTA
    bool aborted = false;
    grid_dependency_wait();      // X8 comes from the preceding grid under PDL
    if constexpr (kFuseX) {
      // own activations: X8 is written by this CTA's epilogue warps first;
      // the copies below read it through the async proxy
      aborted = !__all_sync(0xffffffffu, mbar_wait(bar_x8, 0, abort_flag, &g_error_word,
                                                    kErrProducer));
      fence_proxy_async_global();
    }
    for (int u = blockIdx.x; u < args.units && !aborted; u += gridDim.x) {
      const Unit w = unit_of(args, u, kt_total);
      const int m0 = w.mt * TOK;
      const int nsteps = (w.num_kt + C::kNB - 1) / C::kNB;
      for (int i = 0; i < nsteps; ++i, ++g) {
        const int s = g % S;
        if (g >= S && !__all_sync(0xffffffffu, mbar_wait(bar_empty + 8 * s, ((g / S) & 1) ^ 1,
                                                         abort_flag, &g_error_word,
                                                         kErrProducer))) {
          aborted = true;
          break;
        }
        if (elect_one()) {
          const int nb = min(C::kNB, w.num_kt - i * C::kNB);
          mbar_arrive_expect_tx(bar_xfull + 8 * s, static_cast<uint32_t>(nb * C::kXBytes));
          for (int q = 0; q < nb; ++q)
            tma_load_2d(base + C::kOffX + s * C::kStageX + q * C::kXBytes, &tmap_x,
                        (w.kt_begin + i * C::kNB + q) * kTileK, m0, bar_xfull + 8 * s);
        }
        __syncwarp();
      }
    }
    // the copies already issued must land before the CTA exits, also when
    // another role gave up a wait after this loop had issued its last stage
    // (on the normal path they have all landed and every test passes at once)
    for (uint32_t j = (g > S ? g - S : 0); j < g; ++j)
      drain_wait(bar_xfull + 8 * (j % S), (j / S) & 1);
    (void)aborted;
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    // The whole warp runs the loop and waits; one elected lane issues each
    // tcgen05.mma / tcgen05.commit.
    constexpr uint32_t idesc = idesc_i8(kTileN, TOK);
    uint32_t g = 0;
    int lt = 0;
    bool aborted = false;
    for (int u = blockIdx.x; u < args.units && !aborted; u += gridDim.x, ++lt) {
      const Unit w = unit_of(args, u, kt_total);
      const int b = lt % C::kAcc;
      if (lt >= C::kAcc &&
          !__all_sync(0xffffffffu, mbar_wait(bar_accempty + 8 * b, ((lt / C::kAcc) & 1) ^ 1,
                                             abort_flag, &g_error_word, kErrMma)))
        break;
      tc_fence_after_sync();
      const uint32_t d_tmem = tmem + C::kTmemD + b * TOK;
      const int nsteps = (w.num_kt + C::kNB - 1) / C::kNB;
      for (int i = 0; i < nsteps; ++i, ++g) {
        const int s = g % S;
        if (!__all_sync(0xffffffffu, mbar_wait(bar_dqfull + 8 * s, (g / S) & 1, abort_flag,
                                               &g_error_word, kErrMma))) {
          aborted = true;
          break;
        }
        tc_fence_after_sync();
        if (elect_one()) {
          const int nb = min(C::kNB, w.num_kt - i * C::kNB);
          const uint32_t a_tmem = tmem + C::kTmemA + C::kACols * s;
          const uint32_t b_addr = base + C::kOffX + s * C::kStageX;
#pragma unroll
          for (int q = 0; q < C::kNB; ++q) {
            if (q < nb) {
#pragma unroll
              for (int kk = 0; kk < kTileK / 32; ++kk) {
                // K = 32 bytes per instruction: 8 tensor-memory columns of A,
                // 32 bytes along the swizzled rows of B
                mma_i8_ts(d_tmem, a_tmem + 32 * q + 8 * kk,
                          smem_desc_sw128(b_addr + q * C::kXBytes + kk * 32), idesc,
                          (i > 0 || q > 0 || kk > 0) ? 1u : 0u);
              }
            }
          }
          mma_commit(bar_empty + 8 * s);     // stage s is free once these MMAs complete
        }
        __syncwarp();
      }
      if (!aborted && elect_one()) mma_commit(bar_accfull + 8 * b);   // accumulator b is complete
      __syncwarp();
    }
    if (elect_one()) mma_commit(bar_drain);
    __syncwarp();
    drain_wait(bar_drain, 0);                // no MMA in flight past this point
  } else if (warp < C::kWarpEpi0) {
    // ---------------------------------------------------------------- dequantizers
    constexpr int kDqGroups = C::kDqGroups;
    const int wg = (warp - 2) >> 2;         // 0 .. kDqGroups-1: takes stages g = wg (mod kDqGroups)
    const int q4 = warp & 3;                // tensor-memory lane quarter of this warp
    const int r = q4 * 32 + lane;           // weight row (output channel) within the tile
    const uint32_t row_tmem = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const int gpt = kTileK / args.group;
    uint32_t g0 = 0;                        // running stage index of the unit's first stage
    bool aborted = false;

    for (int u = blockIdx.x; u < args.units && !aborted; u += gridDim.x) {
      const Unit w = unit_of(args, u, kt_total);
      const int nsteps = (w.num_kt + C::kNB - 1) / C::kNB;
      // this warpgroup's first stage of the unit, then every kDqGroups-th
      int i = static_cast<int>((static_cast<uint32_t>(wg) + kDqGroups - g0 % kDqGroups) %
                               kDqGroups);
      for (; i < nsteps; i += kDqGroups) {
        const uint32_t g = g0 + i;
        const int s = g % S;
        const uint32_t ph = (g / S) & 1;
        const int sw = g % SW;
        const uint32_t phw = (g / SW) & 1;
        // A parity wait is only exact while the barrier has completed the
        // phase before the awaited one.  This warpgroup first waits for the
        // A columns of slot s (the MMAs of stage g - S completed, in order):
        // those MMAs read the dequantized weights of every stage up to
        // g - S, and the weight slot's previous phase belongs to stage
        // g - SW <= g - S, so it has completed before its parity is tested
        // below.
        if (g >= S && !mbar_wait(bar_empty + 8 * s, ph ^ 1, abort_flag, &g_error_word,
                                 kErrDequant)) {
          aborted = true;
          break;
        }
        tc_fence_after_sync();
        if (!mbar_wait(bar_wfull + 8 * sw, phw, abort_flag, &g_error_word, kErrDequant)) {
          aborted = true;
          break;
        }
        const int nb = min(C::kNB, w.num_kt - i * C::kNB);
        const uint8_t* stage_raw = smem + C::kOffRaw + sw * C::kStageRaw;
        const uint32_t a_cols = row_tmem + C::kTmemA + C::kACols * s;
        if constexpr (C::kDqGroups == 3) {
          // every block of the stage into registers first, so the weight slot
          // is released as early as possible
          RowBlock rb[C::kNB];
#pragma unroll
          for (int q = 0; q < C::kNB; ++q)
            if (q < nb) load_row_block(stage_raw + q * args.blk_bytes, r, gpt, rb[q]);
          // the weight slot may be refilled once every lane has read it (the
          // arrive releases this warp's reads, ordered by the warp barrier)
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_wempty + 8 * sw);
#pragma unroll
          for (int q = 0; q < C::kNB; ++q)
            if (q < nb) dequant_store_row_block(rb[q], gpt, a_cols + 32 * q);
        } else {
          // four warpgroups leave fewer registers per thread: one block at a
          // time, the weight slot released after the last block's loads
#pragma unroll
          for (int q = 0; q < C::kNB; ++q) {
            if (q < nb) {
              RowBlock rb;
              load_row_block(stage_raw + q * args.blk_bytes, r, gpt, rb);
              if (q == nb - 1) {
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_wempty + 8 * sw);
              }
              dequant_store_row_block(rb, gpt, a_cols + 32 * q);
            }
          }
        }
        tmem_st_wait();
        // the MMAs of the stage also read its X8 tiles: the MMA warp waits on
        // dqfull alone
        if (!mbar_wait(bar_xfull + 8 * s, ph, abort_flag, &g_error_word, kErrDequant)) {
          aborted = true;
          break;
        }
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_dqfull + 8 * s);
      }
      g0 += static_cast<uint32_t>(nsteps);
    }
  } else if (warp < C::kWarpW) {
    // ---------------------------------------------------------------- epilogue
    const int q4 = warp & 3;                // tensor-memory lane quarter
    const int ew = warp - C::kWarpEpi0;     // 0..3
    const int r = q4 * 32 + lane;           // output channel within the tile
    const int M = args.M, N = args.N;
    uint8_t* stage = smem + C::kOffEpi + ew * kStageBytesEpi;   // [16 columns][32 rows] x 4 B
    float* sx_w = reinterpret_cast<float*>(smem + C::kOffSx) + ew * TOK;
    // transposed read of the staging buffer: lane reads column c = lane / 2,
    // rows 16 * (lane & 1) .. +15 of this warp's 32-row slice
    const int tc = lane >> 1, th = lane & 1;
    uint32_t gu_seq = 0;                    // gate_up: chunks handed over so far
    grid_dependency_wait();                 // sx comes from the preceding grid under PDL
    // Own activations, before the first accumulator can be ready: the M FP16
    // token rows (contiguous, M*K*2 bytes) in one bulk copy, each row's scale
    // as the stand-alone quantizer computes it (CTA 0 writes sx), then all of
    // X8 written with the same codes by every CTA (identical bytes), and the
    // X producer released.
    float* sxq = reinterpret_cast<float*>(smem + C::kOffSxq);   // [row] scale, reciprocal
    bool sx_ok = true;
    if constexpr (kFuseX) {
      const int t = ew * 32 + lane;
      const uint32_t bytes = static_cast<uint32_t>(M) * static_cast<uint32_t>(args.K) * 2u;
      if (t == 0) {
        mbar_arrive_expect_tx(bar_xrow, bytes);
        bulk_load_plain(base + C::kOffXrow, args.X, bytes, bar_xrow);
      }
      sx_ok = __all_sync(0xffffffffu, mbar_wait(bar_xrow, 0, abort_flag, &g_error_word,
                                                 kErrEpilogue));
      const uint4* rv = reinterpret_cast<const uint4*>(smem + C::kOffXrow);
      const int vpr = args.K / 8;                     // 16-byte vectors per row
      if (sx_ok) {
        for (int m = ew; m < M; m += 4) {
          __half2 hmax = __float2half2_rn(0.0f);
          for (int i = lane; i < vpr; i += 32) hmax = absmax8(rv[m * vpr + i], hmax);
          float amax = fmaxf(__low2float(hmax), __high2float(hmax));
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
          if (lane == 0) {
            const __half sh = scale_from_absmax(amax, 127.0f);
            const float sf = __half2float(sh);
            sxq[2 * m] = sf;
            sxq[2 * m + 1] = __frcp_rn(sf);
            if (blockIdx.x == 0) const_cast<__half*>(args.sx)[m] = sh;
          }
        }
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (sx_ok) {
        uint2* x8 = reinterpret_cast<uint2*>(args.X8);
        for (int v = t; v < M * vpr; v += 128) {
          const int m = v / vpr;
          const float sf = sxq[2 * m], rcp = sxq[2 * m + 1];
          x8[v] = sf < 6.103515625e-05f ? quantize8<true>(rv[v], sf, rcp, 0.5f * sf)
                                        : quantize8<false>(rv[v], sf, rcp, 0.5f * sf);
        }
        // the tensor copies of this CTA's X producer read these stores
        fence_proxy_async_global();
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (t == 0 && sx_ok) mbar_arrive(bar_x8);
    }
    int lt = 0;
    for (int u = blockIdx.x; u < args.units && sx_ok; u += gridDim.x, ++lt) {
      const Unit w = unit_of(args, u, kt_total);
      const int b = lt % C::kAcc;
      const int m0 = w.mt * TOK;
      const int nrow0 = w.nt * kTileN + q4 * 32;   // first channel of this warp's slice
      int c_end = M - m0;
      if (c_end > TOK) c_end = TOK;
      // the scales do not depend on the accumulator: fetch them while the
      // main loop of this unit is still running
      float s1r = 0.0f;
      if (args.Y) {
        s1r = __half2float(args.s1[w.nt * kTileN + r]);
        for (int c = lane; c < TOK; c += 32)
          sx_w[c] = (m0 + c < M) ? (kFuseX ? sxq[2 * (m0 + c)] : __half2float(args.sx[m0 + c]))
                                 : 0.0f;
        __syncwarp();
      }
      bool ok = mbar_wait(bar_accfull + 8 * b, (lt / C::kAcc) & 1, abort_flag,
                          &g_error_word, kErrEpilogue);
      if constexpr (kGateUp) {
        // the four warps meet at a named barrier in every chunk below: they
        // decide together whether to run this unit, so that all or none of
        // them reach each barrier (every wait before this one is bounded)
        ok = named_barrier_and(3, 128, ok && *abort_flag == 0u);
      }
      if (!__all_sync(0xffffffffu, ok)) break;
      // At this CTA's last accumulator a kernel launched after this one as
      // its programmatic dependent may be scheduled: it waits for this grid
      // to complete before it touches memory this grid uses, so only its
      // launch and set-up overlap this tail.
      if (u + static_cast<int>(gridDim.x) >= args.units) grid_launch_dependents();
      tc_fence_after_sync();
      const uint32_t t_acc = tmem + C::kTmemD + b * TOK + (static_cast<uint32_t>(q4 * 32) << 16);
      const int splits = args.splits;
      bool write_out = true;
      bool red_ok = true;
      if (cs > 1 && crank != 0) {
        // K split across the cluster, not the leader: once the leader has
        // added up the previous unit's slices, write this warp's INT32 slice
        // into the leader's reduction buffer and arrive on its barrier
        if (lt > 0) red_ok = mbar_wait_cluster(bar_red_free + 8 * q4, (lt - 1) & 1, abort_flag,
                                                &g_error_word, kErrEpilogue);
        red_ok = __all_sync(0xffffffffu, red_ok);
        if (red_ok) {
          const uint32_t dst = map_to_rank(
              base + C::kOffRed + ((crank - 1) * 4 + q4) * (TOK * 128), 0u) + lane * 4;
          for (int c0 = 0; c0 < c_end; c0 += 16) {
            uint32_t v[16];
            tmem_ld_32x32b_x16(t_acc + c0, v);
            tmem_ld_wait(v);
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (c0 + j < c_end) st_cluster_u32(dst + (c0 + j) * 128, v[j]);
          }
          // every lane's stores are ordered before lane 0's release
          asm volatile("fence.acq_rel.cluster;" ::: "memory");
          __syncwarp();
          if (lane == 0) mbar_arrive_remote(map_to_rank(bar_red_full + 8 * q4, 0u));
        }
        write_out = false;
      } else if (cs > 1) {
        // the leader: wait for the other CTAs' slices of this unit
        red_ok = __all_sync(0xffffffffu, mbar_wait_cluster(bar_red_full + 8 * q4, lt & 1,
                                                           abort_flag, &g_error_word,
                                                           kErrEpilogue));
        if (!red_ok) write_out = false;
      } else if (splits > 1) {
        // publish this unit's partial tile (INT32, [token][channel]) ...
        int32_t* part = args.ws_part + (static_cast<size_t>(w.mt * splits + w.split) * TOK) * N;
        for (int c0 = 0; c0 < c_end; c0 += 16) {
          uint32_t v[16];
          tmem_ld_32x32b_x16(t_acc + c0, v);
          tmem_ld_wait(v);
          uint32_t* st = reinterpret_cast<uint32_t*>(stage);
#pragma unroll
          for (int j = 0; j < 16; ++j) st[j * 32 + lane] = v[j];
          __syncwarp();
          if (c0 + tc < c_end) {
            const uint4* src = reinterpret_cast<const uint4*>(st + tc * 32 + 16 * th);
            uint4* dst = reinterpret_cast<uint4*>(part + static_cast<size_t>(c0 + tc) * N + nrow0 +
                                                  16 * th);
#pragma unroll
            for (int e = 0; e < 4; ++e) __stcg(dst + e, src[e]);
          }
          __syncwarp();
        }
        // ... then count this warp's arrival at its slice.  The warp barrier
        // orders the lanes' stores before lane 0's release, and the second
        // warp barrier orders the lanes' reads of the other partials after
        // the last arrival's acquire.
        __syncwarp();
        bool last = false;
        if (lane == 0) {
          last = arrive_last(
              args.ws_count + (w.mt * args.n_tiles + w.nt) * kSlicesPerTile + q4, splits);
        }
        __syncwarp();
        write_out = __shfl_sync(0xffffffffu, last ? 1 : 0, 0) != 0;
      }
      if (write_out && (kGateUp || *abort_flag == 0u)) {
        const int32_t* parts = args.ws_part + (static_cast<size_t>(w.mt * splits) * TOK) * N;
        // software-pipelined over 16-column chunks: the next chunk's load
        // from tensor memory is in flight while this chunk is scaled and
        // stored
        uint32_t v[16], vn[16];
        tmem_ld_32x32b_x16(t_acc, vn);
        for (int c0 = 0; c0 < c_end; c0 += 16) {
          tmem_ld_wait(vn);
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = vn[j];
          // (the gate_up epilogue issues it once this chunk's outputs are in
          // its staging buffer, which keeps its registers within the
          // launch's budget)
          if (!kGateUp && c0 + 16 < c_end) tmem_ld_32x32b_x16(t_acc + c0 + 16, vn);
          if (cs > 1) {
            // add the cluster's slices from this CTA's reduction buffer
            for (int q = 0; q < cs - 1; ++q) {
              const uint32_t* rp = reinterpret_cast<const uint32_t*>(
                  smem + C::kOffRed + (q * 4 + q4) * (TOK * 128) + lane * 4);
#pragma unroll
              for (int j = 0; j < 16; ++j)
                if (c0 + j < c_end) v[j] += rp[(c0 + j) * 32];
            }
          } else if (TOK > 32 && splits > 1) {
            // wide token tiles (an explicit split): the other splits'
            // partials one after another (a batched version in this
            // instance measured 3% slower at 4096 tokens, unsplit)
            for (int q = 0; q < splits; ++q) {
              if (q == w.split) continue;
              const int32_t* p = parts + (static_cast<size_t>(q) * TOK + c0) * N + nrow0 + lane;
#pragma unroll
              for (int j = 0; j < 16; ++j)
                if (c0 + j < c_end) v[j] += static_cast<uint32_t>(__ldcg(p + static_cast<size_t>(j) * N));
            }
          } else if (splits > 1) {
            // decode tiles: add the other splits' partials of this chunk's
            // tokens, taken
            // as a list of (split, token) pairs, 16 pairs per batch: the
            // batch's loads are unconditional (a pair past the end of the
            // list reads the last split's row again and is not added), so
            // all 16 are in flight together and a batch costs one L2 round
            // trip.  The sums collect in the warp's staging buffer, each
            // lane in its own column.
            const int cnt = c_end - c0 < 16 ? c_end - c0 : 16;
            uint32_t* st = reinterpret_cast<uint32_t*>(stage);
#pragma unroll
            for (int j = 0; j < 16; ++j) st[j * 32 + lane] = v[j];
            int q = 0, jj = 0;
            while (q < splits) {
              uint32_t t[16];
              int qb[16], jb[16];
#pragma unroll
              for (int b = 0; b < 16; ++b) {
                qb[b] = q;
                jb[b] = jj;
                const int qc = q < splits ? q : splits - 1;
                t[b] = static_cast<uint32_t>(
                    __ldcg(parts + (static_cast<size_t>(qc) * TOK + c0 + jj) * N + nrow0 + lane));
                jj = jj + 1 == cnt ? 0 : jj + 1;
                q = jj == 0 ? q + 1 : q;
              }
#pragma unroll
              for (int b = 0; b < 16; ++b)
                if (qb[b] < splits && qb[b] != w.split) st[jb[b] * 32 + lane] += t[b];
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = st[j * 32 + lane];
          }
          if (args.acc) {
            uint32_t* st = reinterpret_cast<uint32_t*>(stage);
#pragma unroll
            for (int j = 0; j < 16; ++j) st[j * 32 + lane] = v[j];
            __syncwarp();
            if (c0 + tc < c_end) {
              const uint4* src = reinterpret_cast<const uint4*>(st + tc * 32 + 16 * th);
              uint4* dst = reinterpret_cast<uint4*>(args.acc + static_cast<size_t>(m0 + c0 + tc) * N +
                                                    nrow0 + 16 * th);
#pragma unroll
              for (int e = 0; e < 4; ++e) dst[e] = src[e];
            }
          } else if constexpr (kGateUp) {
            // Every warp's 16 outputs of the chunk in FP16, [column][row], go
            // to half h of its staging buffer (h alternates chunk by chunk,
            // across units too, so a half is written again only after every
            // warp has finished reading it: they all passed the barrier of
            // the chunk in between).  The four warps pass the same barriers:
            // they agreed at the unit's start to run its chunks.  Then all four warps form
            // silu(gate) * up: warp q4 takes the gate rows of lane quarter
            // q4 & 1 (their up rows are quarter (q4 & 1) + 2) for token
            // columns 8 (q4 >> 1) .. +7, writes the products over the gate
            // values it read and stores them to H.
            const int hb = static_cast<int>(gu_seq & 1u);
            __half* st = reinterpret_cast<__half*>(stage) + hb * 512;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float scale = __fmul_rn(sx_w[c0 + j], s1r);
              st[j * 32 + lane] =
                  __float2half_rn(__fmul_rn(static_cast<float>(static_cast<int32_t>(v[j])), scale));
            }
            if (c0 + 16 < c_end) tmem_ld_32x32b_x16(t_acc + c0 + 16, vn);
            asm volatile("bar.sync 2, 128;" ::: "memory");
            ++gu_seq;
            const int gq = q4 & 1, jb = 8 * (q4 >> 1);
            __half* gs = reinterpret_cast<__half*>(
                             smem + C::kOffEpi + ((gq - C::kWarpEpi0) & 3) * kStageBytesEpi) +
                         hb * 512;
            const __half* us = reinterpret_cast<const __half*>(
                                   smem + C::kOffEpi + ((gq + 2 - C::kWarpEpi0) & 3) * kStageBytesEpi) +
                               hb * 512;
#pragma unroll
            for (int j = jb; j < jb + 8; ++j) {
              const float g = __half2float(gs[j * 32 + lane]);
              const float u = __half2float(us[j * 32 + lane]);
              gs[j * 32 + lane] = __float2half_rn(__fmul_rn(__fdividef(g, 1.0f + __expf(-g)), u));
            }
            __syncwarp();
            // lane: token column jb + lane / 4, channels 8 (lane & 3) .. +7
            const int tq = jb + (lane >> 2), tp = lane & 3;
            if (c0 + tq < c_end) {
              *reinterpret_cast<uint4*>(args.Y + static_cast<size_t>(m0 + c0 + tq) * (N / 2) +
                                        w.nt * 64 + gq * 32 + 8 * tp) =
                  *reinterpret_cast<const uint4*>(gs + tq * 32 + 8 * tp);
            }
          } else {
            __half* st = reinterpret_cast<__half*>(stage);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float scale = __fmul_rn(sx_w[c0 + j], s1r);
              st[j * 32 + lane] =
                  __float2half_rn(__fmul_rn(static_cast<float>(static_cast<int32_t>(v[j])), scale));
            }
            __syncwarp();
            if (c0 + tc < c_end) {
              const uint4* src = reinterpret_cast<const uint4*>(st + tc * 32 + 16 * th);
              uint4* dst = reinterpret_cast<uint4*>(args.Y + static_cast<size_t>(m0 + c0 + tc) * N +
                                                    nrow0 + 16 * th);
              dst[0] = src[0];
              dst[1] = src[1];
            }
          }
          __syncwarp();
        }
      }
      if (cs > 1 && crank == 0 && red_ok && u + static_cast<int>(gridDim.x) < args.units) {
        // the slices are added up: the other CTAs may write the next unit's
        __syncwarp();
        if (lane == 0)
          for (int r = 1; r < cs; ++r)
            mbar_arrive_remote(map_to_rank(bar_red_free + 8 * q4, static_cast<uint32_t>(r)));
      }
      if (!red_ok) break;
      // the accumulator may be overwritten by the unit after next
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_accempty + 8 * b);
    }
    if constexpr (kFuseX) {
      // the row copy must land before the CTA exits, also if its wait gave up
      if (!sx_ok && ew == 0) drain_wait(bar_xrow, 0);
    }
  } else {
    // -------------------------------------------------------------- W producer
    // The stages after the prologue, waiting for free slots.
    wstream.run<C>(args, base, bar_wfull, bar_wempty, abort_flag, /*prologue=*/false);
    // every copy issued lands before the CTA exits, also when another role
    // gave up a wait after this loop had issued its last stage (on the
    // normal path they have all landed and every test passes at once)
    const uint32_t g = wstream.g;
    for (uint32_t j = (g > SW ? g - SW : 0); j < g; ++j)
      drain_wait(bar_wfull + 8 * (j % SW), (j / SW) & 1);
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before_sync();
  __syncthreads();
  // no CTA of the cluster leaves while another may still access its shared
  // memory (every thread of every CTA reaches this point on every path)
  if (cs > 1) cluster_sync_all();

  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
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
  int tok, splits, m_tiles, n_tiles, stages, units, grid;
  int cs;   // K split across a cluster of cs CTAs (1: split through the workspace, or none)
  bool gemv = false;   // one to four tokens on the CUDA cores (qoq_gemv.cu): tok = 0
  int rows = 0;        // the GEMV's tokens
};

// Largest K split a cluster can reduce in the leader's shared memory.
int max_cluster_split(int tok) { return tok <= 16 ? 8 : tok <= 32 ? 3 : 1; }

template <int TOK, bool kCluster, bool kFuseX, bool kGateUp>
__global__ void __launch_bounds__(Cfg<TOK>::kThreads, 1)
w4a8_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const GemmArgs args);

template <int TOK>
int query_active_clusters(int cs) {
  using C = Cfg<TOK, true>;
  if (cudaFuncSetAttribute(w4a8_gemm_kernel<TOK, true, false, false>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
          cudaSuccess ||
      cudaFuncSetAttribute(w4a8_gemm_kernel<TOK, true, false, false>,
                           cudaFuncAttributeNonPortableClusterSizeAllowed, 0) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(cs * 64), 1, 1);
  cfg.blockDim = dim3(C::kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(cs);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, w4a8_gemm_kernel<TOK, true, false, false>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

// Clusters of cs CTAs of the `tok` kernel that can be resident at once on the
// current device (one CTA per SM), cached per device; without a device (or
// if the query fails) the SM count divided by cs.
int active_clusters(int tok, int cs) {
  const int sms = sm_count();
  if (cs <= 1) return sms;
  constexpr int kDev = 16;
  static std::atomic<int> cache[kDev][2][9];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return sms / cs;
  }
  const int ti = tok <= 16 ? 0 : 1;
  if (dev >= 0 && dev < kDev) {
    const int v = cache[dev][ti][cs].load(std::memory_order_relaxed);
    if (v > 0) return v;
  }
  int n = tok <= 16 ? query_active_clusters<16>(cs) : query_active_clusters<32>(cs);
  if (n <= 0) n = sms / cs;
  if (n > sms / cs) n = sms / cs;
  if (dev >= 0 && dev < kDev) cache[dev][ti][cs].store(n, std::memory_order_relaxed);
  return n;
}

bool splittable(const Plan& p) {
  return static_cast<long>(p.m_tiles) * p.n_tiles <= kMaxCounterTiles;   // one counter per slice
}

int stages_for(int tok) { return tok <= 32 ? 7 : tok == 64 ? 6 : tok == 176 ? 5 : 4; }

// Token tiles a caller may request; 1 asks for the CUDA-core GEMV.
bool valid_tok(int t) {
  return t == 1 || t == 16 || t == 32 || t == 64 || t == 128 || t == 176 || t == 192 || t == 256;
}

// The CUDA-core GEMV's copy ring: 4 slots per warp when each warp has at
// least 16 k-tiles of its K range (and the larger ring fits beside the token
// rows), else 2.  On B200 the deeper ring made Qwen1.5-72B down (K = 24576,
// 24 k-tiles per warp) 18% faster and the layers with 4 to 8 k-tiles per
// warp 9-17% slower (fewer CTAs per SM).
int gemv_ring(int M, int K, int kt_per) {
  const bool long_k = (kt_per + 7) / 8 >= 16;
  return long_k && gemv_smem_bytes(M, K, 4) <= kGemvMaxSmem ? 4 : 2;
}

bool gemv_fits(int M, int K, int stages) {
  return M <= kGemvMaxTokens && gemv_smem_bytes(M, K, stages) <= kGemvMaxSmem;
}

// For two to four tokens, GEMV or tensor cores: modelled launch times in us
// against the packed weight megabytes, fitted to back-to-back launches on
// B200 over the six Llama-3-8B and Qwen1.5-72B layers (the GEMV at one and
// four tokens, the 16-token tensor-core tile).  The GEMV turns
// compute-bound as tokens are added; the tensor-core kernel costs the same
// for one to sixteen tokens but has the larger fixed cost.  One token always
// takes the GEMV; two to four take it when its modelled time is at least 5%
// lower (the per-layer slopes scatter around the fit).
bool gemv_preferred(int M, int N, int K) {
  if (M == 1) return true;
  const double mb = static_cast<double>(N) * K * 0.5e-6;
  const double t_gemv = 3.4 + 0.27 * M + (0.122 + 0.034 * M) * mb;
  const double t_mma = 6.2 + 0.169 * mb;
  return t_gemv < 0.95 * t_mma;
}

// Token tile for a shape.  Up to 32 tokens the smallest tile that holds M; up
// to 64 two 32-token tiles when they fit one round of units, else one of 64.
// Beyond that the choice is between 128 (two k-tiles per pipeline stage) and
// the wide tiles 176 / 192 (one k-tile per stage, so more control work per
// K but fewer output tiles): the cost of a shape is the number of rounds of
// units over the SMs times the time a unit takes per k-tile, measured on B200
// with every SM busy as about 277, 363 and 377 ns for 128, 176 and 192 tokens
// (Llama-3-8B QKV at 4096 tokens; the wide tiles gained from the deeper
// weight ring).
int auto_tok(int M, int n_tiles) {
  const long sms = sm_count();
  if (M <= 16) return 16;
  if (M <= 32) return 32;
  if (M <= 64) {
    // two 32-token tiles run on twice the SMs as long as they fit one round
    return static_cast<long>((M + 31) / 32) * n_tiles <= sms ? 32 : 64;
  }
  const int cand[3] = {128, 176, 192};
  const double per_kt[3] = {277.0, 363.0, 377.0};
  int best = 128;
  double best_cost = 1e30;
  for (int i = 0; i < 3; ++i) {
    const long units = static_cast<long>((M + cand[i] - 1) / cand[i]) * n_tiles;
    const long rounds = (units + sms - 1) / sms;
    const double cost = static_cast<double>(rounds) * per_kt[i];
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = cand[i];
    }
  }
  return best;
}

// Cost model for the number of K splits of a decode plan: units are spread
// over the CTAs, a unit costs its k-tiles plus a fixed overhead (pipeline
// fill and epilogue), a split unit a little more.  A split is added up either
// inside a cluster (through the leader CTA's shared memory, up to
// max_cluster_split CTAs) or through the workspace in L2 (partial slices
// written, the last arrival reading the others back).  Measured on B200 with
// 16-token tiles: up to four tokens the workspace split is the faster of the
// two (its tail is one L2 round trip per batch of 16 partial rows, and a
// cluster waits for all of its SMs to be free); with more tokens the cluster
// split is, while a 16-token Llama QKV tile (32 k-tiles) ran fastest unsplit
// through the workspace.  32-token tiles ran faster unsplit than split across
// a cluster (K = N = 2048 and 4096), so the planner keeps clusters for 16.
int auto_splits(int tiles, int kt, int tok, int M, bool* cluster_out) {
  *cluster_out = false;
  if (tok > 32) return 1;
  const int tokens = M < tok ? M : tok;
  const bool cluster_ok = tokens > 4 && tok <= 16;
  const bool l2_ok = tokens <= 4 || kt >= 64;
  const long sms = sm_count();
  int best_s = 1;
  double best = 1e30;
  for (int s = 1; s <= 8 && s <= kt; ++s) {
    if (s > 1 && kt / s < 2) break;
    const bool cluster = s > 1 && cluster_ok && s <= max_cluster_split(tok);
    if (s > 1 && !cluster && (!l2_ok || static_cast<long>(tiles) * s > 4L * sms)) continue;
    const long slots = cluster ? static_cast<long>(active_clusters(tok, s)) * s : sms;
    const long units = static_cast<long>(tiles) * s;
    const long rounds = (units + slots - 1) / slots;
    const double ovh = s == 1 ? 0.0 : cluster ? 1.0 : 2.0;
    const double cost = static_cast<double>(rounds) * (static_cast<double>(kt) / s + 3.0 + ovh);
    if (cost < best - 1e-9) {
      best = cost;
      best_s = s;
      *cluster_out = cluster;
    }
  }
  return best_s;
}

void finish_plan(Plan& p) {
  if (p.gemv) return;   // a CTA per 32 channels, set by make_plan
  p.units = p.n_tiles * p.m_tiles * p.splits;
  const int sms = sm_count();
  if (p.cs > 1) {
    // whole clusters, each taking the splits of one output tile
    const int tiles = p.n_tiles * p.m_tiles;
    const int ncl = active_clusters(p.tok, p.cs);
    p.grid = (tiles < ncl ? tiles : ncl) * p.cs;
  } else {
    p.grid = p.units < sms ? p.units : sms;
  }
}

Plan make_plan(int M, int N, int K, int tok_req, int splits_req) {
  Plan p;
  p.n_tiles = N / kTileN;
  const int kt = K / kTileK;
  const bool want_gemv =
      tok_req == 1 || (!tok_req && !splits_req && M <= kGemvMaxTokens && gemv_preferred(M, N, K));
  if (want_gemv) {
    // a matrix-vector product: the packed weights streamed through the CUDA
    // cores.  K is split only when fewer than half the SMs would get a CTA
    // (the partial sums go through the workspace and the last arrival adds
    // them; with the copy rings every split measured slower on the six
    // Llama-3-8B / Qwen1.5-72B layers), each warp keeping two k-tiles.
    const long groups = N / 32;
    long ks = splits_req;
    if (!ks) {
      const long sms = sm_count();
      ks = 2 * groups < sms ? (sms + groups - 1) / groups : 1;
      const long cap = kt / (2 * 8) > 1 ? kt / (2 * 8) : 1;
      if (ks > cap) ks = cap;
    }
    const int stages = gemv_ring(M, K, (kt + static_cast<int>(ks) - 1) / static_cast<int>(ks));
    // an explicit request that cannot run is refused by gemm_prepare; the
    // automatic plan takes the tensor cores instead
    if (tok_req == 1 || gemv_fits(M, K, stages)) {
      p.gemv = true;
      p.rows = M;
      p.tok = 0;
      p.cs = 1;
      p.m_tiles = 1;
      p.stages = stages;
      p.splits = static_cast<int>(ks);
      p.units = p.grid = static_cast<int>(groups * ks);
      return p;
    }
  }
  p.tok = tok_req ? tok_req : auto_tok(M, p.n_tiles);
  p.m_tiles = (M + p.tok - 1) / p.tok;
  p.stages = stages_for(p.tok);
  if (splits_req) {
    // an explicit split runs on a cluster whenever the tile's kernel can
    // reduce it there
    p.splits = splits_req;
    p.cs = (p.splits > 1 && p.splits <= max_cluster_split(p.tok)) ? p.splits : 1;
  } else {
    bool cluster = false;
    p.splits = auto_splits(p.n_tiles * p.m_tiles, kt, p.tok, M, &cluster);
    p.cs = cluster ? p.splits : 1;
  }
  if (!splits_req && p.cs == 1 && !splittable(p)) p.splits = 1;
  finish_plan(p);
  return p;
}

size_t ws_bytes_for(const Plan& p, int N) {
  if (p.splits <= 1 || p.cs > 1) return 0;   // a cluster split needs no workspace
  if (p.gemv)   // a slice of INT32 sums per split
    return kCounterBytes + static_cast<size_t>(p.splits) * p.rows * N * 4;
  const size_t part = static_cast<size_t>(p.m_tiles) * p.splits * p.tok * N * 4;
  return kCounterBytes + part;
}

template <int TOK, bool kCluster, bool kFuseX, bool kGateUp = false>
int launch_kernel(const CUtensorMap& map, const GemmArgs& a, const Plan& p, cudaStream_t stream,
               bool pdl) {
  // the same layout as the kernel instance (its shared-memory size)
  using C = Cfg<TOK, kCluster, kFuseX>;
  static int configured_mask = 0;   // one bit per device id < 31
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QOQ_ERR_CUDA;
  const int bit = dev < 31 ? (1 << dev) : 0;
  if (!bit || !(__atomic_load_n(&configured_mask, __ATOMIC_ACQUIRE) & bit)) {
    if (cudaFuncSetAttribute(w4a8_gemm_kernel<TOK, kCluster, kFuseX, kGateUp>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kSmemBytes) != cudaSuccess)
      return QOQ_ERR_CUDA;
    if (bit) __atomic_fetch_or(&configured_mask, bit, __ATOMIC_RELEASE);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(p.grid), 1, 1);
  cfg.blockDim = dim3(C::kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (p.cs > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = static_cast<unsigned>(p.cs);
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  if (cudaLaunchKernelEx(&cfg, w4a8_gemm_kernel<TOK, kCluster, kFuseX, kGateUp>, map, a) != cudaSuccess) return QOQ_ERR_CUDA;
  return QOQ_OK;
}

// The cluster variant of the kernel for token tiles up to 32 when the plan
// splits K across a cluster, the plain one otherwise.
template <int TOK>
int launch_tok(const CUtensorMap& map, const GemmArgs& a, const Plan& p, cudaStream_t stream,
               bool pdl, bool gate_up) {
  if constexpr (TOK <= 128 && TOK != 176) {
    if (gate_up) return launch_kernel<TOK, false, false, true>(map, a, p, stream, pdl);
  }
  const bool fuse = a.X != nullptr;
  if constexpr (TOK <= 32) {
    if (p.cs > 1) return launch_kernel<TOK, true, false>(map, a, p, stream, pdl);
  }
  if constexpr (TOK == 16) {
    if (fuse) return launch_kernel<TOK, false, true>(map, a, p, stream, pdl);
  }
  return launch_kernel<TOK, false, false>(map, a, p, stream, pdl);
}

// Everything one GEMM launch needs, built and checked before anything is
// enqueued: the plan, the X8 tensor map and the kernel arguments.
struct GemmLaunch {
  Plan p;
  CUtensorMap map;
  GemmArgs a;
  GemvArgs g;             // the plan is a GEMV (p.gemv)
  bool gate_up = false;   // the epilogue writes silu(gate) * up (kGateUp kernel)
};

// Validate the arguments, pick the plan and encode the tensor map.  Calls no
// CUDA API that enqueues work.
int gemm_prepare(const int8_t* X8, const void* sx, const void* packed, const void* s1, int M,
                 int N, int K, int group, void* Y, int32_t* acc, int tok_req, int splits_req,
                 void* ws, size_t ws_bytes, GemmLaunch& L) {
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
  if (p.gemv && !gemv_fits(M, K, p.stages)) return QOQ_ERR_UNSUPPORTED;
  // the kernel divides unit indices below 2^22 by multiplication (small_div)
  if (static_cast<long>(p.n_tiles) * p.m_tiles * p.splits >= (1L << 22)) return QOQ_ERR_UNSUPPORTED;
  if (p.splits > 1 && p.cs == 1 && !splittable(p)) {
    if (splits_req) return QOQ_ERR_UNSUPPORTED;
    p.splits = 1;
  }
  if (p.splits > 1 && p.cs == 1 && (ws == nullptr || ws_bytes < ws_bytes_for(p, N))) {
    // an explicit split needs its workspace; so does the automatic plan,
    // unless the caller passed none (an explicit request not to split K)
    if (splits_req || ws != nullptr) return QOQ_ERR_WORKSPACE;
    p.splits = 1;
  }
  finish_plan(p);
  if (int st = check_device()) return st;
  if (p.gemv) {
    p.units = p.grid = (N / 32) * p.splits;   // the split may have been dropped above
    GemvArgs& g = L.g;
    g.packed = static_cast<const uint8_t*>(packed);
    g.X8 = X8;
    g.sx = static_cast<const __half*>(sx);
    g.s1 = static_cast<const __half*>(s1);
    g.Y = static_cast<__half*>(Y);
    g.acc = acc;
    g.M = M;
    g.N = N;
    g.K = K;
    g.group = group;
    g.blk_bytes = static_cast<int>(block_bytes(group));
    g.w_dep_wait = 1;
    g.ks = p.splits;
    g.kt_per = (K / kTileK + p.splits - 1) / p.splits;
    g.stages = gemv_ring(M, K, g.kt_per);   // the split may have been dropped above
    g.ws_count = nullptr;
    g.ws_acc = nullptr;
    if (p.splits > 1) {
      g.ws_count = static_cast<uint32_t*>(ws);
      g.ws_acc = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + kCounterBytes);
    }
    L.p = p;
    return QOQ_OK;
  }
  EncodeTiledFn enc = encode_fn();
  if (!enc) return QOQ_ERR_CUDA;

  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kTileK), static_cast<cuuint32_t>(p.tok)};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(&L.map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(X8), dims, strides, box,
          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return QOQ_ERR_CUDA;

  GemmArgs& a = L.a;
  a.packed = static_cast<const uint8_t*>(packed);
  a.sx = static_cast<const __half*>(sx);
  a.s1 = static_cast<const __half*>(s1);
  a.Y = static_cast<__half*>(Y);
  a.acc = acc;
  a.ws_part = nullptr;
  a.ws_count = nullptr;
  if (p.splits > 1 && p.cs == 1) {
    a.ws_count = static_cast<uint32_t*>(ws);
    a.ws_part = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + kCounterBytes);
  }
  a.cs = p.cs;
  a.X = nullptr;
  a.X8 = nullptr;
  a.M = M;
  a.N = N;
  a.K = K;
  a.group = group;
  a.splits = p.splits;
  a.m_tiles = p.m_tiles;
  a.n_tiles = p.n_tiles;
  a.units = p.units;
  a.blk_bytes = static_cast<int>(block_bytes(group));
  a.rcp_splits = 1.0f / static_cast<float>(p.splits);
  a.rcp_mtiles = 1.0f / static_cast<float>(p.m_tiles);
  a.w_dep_wait = 1;
  L.p = p;
  return QOQ_OK;
}

// Enqueue a prepared launch.  With `clear_counters` the workspace's arrival
// counters are zeroed on the stream first when the plan splits K.  Every
// launch may start as a programmatic dependent of the preceding kernel: the
// kernel touches nothing that kernel may write before its grid-dependency
// waits.  `weights_independent` says the preceding kernel does not
// write the weights (the library's own quantizer), so the weight stream
// need not wait for it.
int gemm_launch(GemmLaunch L, void* stream, bool weights_independent, bool clear_counters) {
  cudaStream_t s = as_stream(stream);
  const bool pdl = true;
  if (L.p.gemv) {
    L.g.w_dep_wait = weights_independent ? 0 : 1;
    if (clear_counters && L.g.ws_count != nullptr &&
        cudaMemsetAsync(L.g.ws_count, 0, kCounterBytes, s) != cudaSuccess)
      return QOQ_ERR_CUDA;
    return launch_gemv(L.g, s);
  }
  L.a.w_dep_wait = weights_independent ? 0 : 1;
  if (clear_counters && L.a.ws_count != nullptr &&
      cudaMemsetAsync(L.a.ws_count, 0, kCounterBytes, s) != cudaSuccess)
    return QOQ_ERR_CUDA;
  switch (L.p.tok) {
    case 16: return launch_tok<16>(L.map, L.a, L.p, s, pdl, L.gate_up);
    case 32: return launch_tok<32>(L.map, L.a, L.p, s, pdl, L.gate_up);
    case 64: return launch_tok<64>(L.map, L.a, L.p, s, pdl, L.gate_up);
    case 128: return launch_tok<128>(L.map, L.a, L.p, s, pdl, L.gate_up);
    case 176: return launch_tok<176>(L.map, L.a, L.p, s, pdl, L.gate_up);
    case 192: return launch_tok<192>(L.map, L.a, L.p, s, pdl, L.gate_up);
    default: return launch_tok<256>(L.map, L.a, L.p, s, pdl, L.gate_up);
  }
}


}  // namespace

int gemm_impl(const int8_t* X8, const void* sx, const void* packed, const void* s1, int M, int N,
              int K, int group, void* Y, int32_t* acc, int tok_req, int splits_req, void* ws,
              size_t ws_bytes, void* stream, bool weights_independent, bool clear_counters) {
  GemmLaunch L;
  if (int st = gemm_prepare(X8, sx, packed, s1, M, N, K, group, Y, acc, tok_req, splits_req, ws,
                            ws_bytes, L))
    return st;
  return gemm_launch(L, stream, weights_independent, clear_counters);
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
                   false, false);
}

// ---------------------------------------------------------------------------
// qoq_w4a8_gemm_static_ws: the same GEMM for callers that may not allocate
// device memory at all (e.g. code running inside a caching allocator's own
// hooks, or a runtime whose memory is fully reserved up front).  The K-split
// workspace is a fixed array in this module's device memory instead of a
// caller buffer: every call on a device shares it.
// ---------------------------------------------------------------------------
namespace qoq {
namespace {

constexpr size_t kStaticWsBytes = QOQ_STATIC_WS_BYTES;
static_assert(kStaticWsBytes > kCounterBytes, "static workspace smaller than its counter region");

static __device__ __align__(256) uint8_t g_static_ws[kStaticWsBytes];

constexpr int kMaxStaticWsDevices = 64;
std::mutex g_static_ws_mutex;
void* g_static_ws_ptr[kMaxStaticWsDevices] = {};

// Device address of g_static_ws on the current device, looked up once per
// device (the first call on a device loads this module there if needed).
int static_ws_ptr(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QOQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxStaticWsDevices) return QOQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_static_ws_mutex);
  if (!g_static_ws_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess || p == nullptr) return QOQ_ERR_CUDA;
    g_static_ws_ptr[dev] = p;
  }
  *out = g_static_ws_ptr[dev];
  return QOQ_OK;
}

}  // namespace
}  // namespace qoq

extern "C" int qoq_w4a8_gemm_static_ws(const int8_t* X8, const void* sx, const void* packed,
                                       const void* s1, int M, int N, int K, int group, void* Y,
                                       void* stream) {
  if (!X8 || !sx || !packed || !s1 || !Y) return QOQ_ERR_INVALID_ARG;
  if (M <= 0) return QOQ_ERR_INVALID_ARG;
  if (int st = check_weight_shape(N, K, group)) return st;
  if (!aligned16(X8) || !aligned16(sx) || !aligned16(packed) || !aligned16(s1) || !aligned16(Y))
    return QOQ_ERR_INVALID_ARG;
  const size_t need = gemm_ws_bytes(M, N, K, 0, 0);
  if (need > kStaticWsBytes) return QOQ_ERR_UNSUPPORTED;   // larger than the fixed array
  if (int st = check_device()) return st;
  void* ws = nullptr;
  if (int st = static_ws_ptr(&ws)) return st;
  // The arrival counters must start at zero: a completed call leaves them so,
  // but the array keeps whatever an interrupted earlier call left.  The GEMM
  // launcher clears them on `stream` after its own checks, only when K is
  // split, so a rejected call enqueues nothing.
  return gemm_impl(X8, sx, packed, s1, M, N, K, group, Y, nullptr, 0, 0, ws, kStaticWsBytes,
                   stream, false, true);
}

extern "C" int qoq_w4a8_gemm_i32(const int8_t* X8, const void* packed, int M, int N, int K,
                                 int group, int32_t* acc, void* ws, size_t ws_bytes,
                                 void* stream) {
  if (!acc) return QOQ_ERR_INVALID_ARG;
  return gemm_impl(X8, nullptr, packed, nullptr, M, N, K, group, nullptr, acc, 0, 0, ws, ws_bytes,
                   stream, false, false);
}

extern "C" int qoq_w4a8_gemm_config(const int8_t* X8, const void* sx, const void* packed,
                                    const void* s1, int M, int N, int K, int group, void* Y,
                                    int32_t* acc, int tok_tile, int splits, void* ws,
                                    size_t ws_bytes, void* stream) {
  return gemm_impl(X8, sx, packed, s1, M, N, K, group, Y, acc, tok_tile, splits, ws, ws_bytes,
                   stream, false, false);
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
  // every check of the GEMM runs before the quantizer is launched
  GemmLaunch L;
  if (int st = gemm_prepare(X8, sx, packed, s1, M, N, K, group, Y, nullptr, 0, 0, ws, ws_bytes, L))
    return st;
  // For few rows the quantizer may start while the preceding kernel on the
  // stream drains (it waits for that grid before touching memory); this hides
  // its launch latency.  For many rows that overlap measured slower on B200,
  // so the quantizer is then an ordinary launch.
  const bool aq_pdl = M <= 2 * sm_count();
  if (int st = launch_act_quant(X, M, K, X8, sx, stream, aq_pdl, nullptr)) return st;
  // both kernels are this library's: the GEMM reads nothing the quantizer
  // writes before its grid-dependency wait, so it may overlap its tail
  return gemm_launch(L, stream, /*weights_independent=*/true, false);
}

extern "C" int qoq_w4a8_linear_fused(const void* X, int M, int K, const void* packed,
                                     const void* s1, int N, int group, int8_t* X8, void* sx,
                                     void* Y, void* ws, size_t ws_bytes, void* stream) {
  if (!X || !X8 || !sx || !Y || !packed || !s1) return QOQ_ERR_INVALID_ARG;
  if (M <= 0) return QOQ_ERR_INVALID_ARG;
  if (int st = check_weight_shape(N, K, group)) return st;
  if (!aligned16(X) || !aligned16(X8) || !aligned16(sx) || !aligned16(Y) || !aligned16(packed) ||
      !aligned16(s1) || (ws && !aligned16(ws)))
    return QOQ_ERR_INVALID_ARG;
  if (static_cast<long>(M) * K * 2 > static_cast<long>(kMaxFusedRowBytes))
    return QOQ_ERR_UNSUPPORTED;
  GemmLaunch L;
  // the kernel's own 16-token tile also where the automatic plan would take
  // the CUDA-core GEMV (one to four tokens)
  const int tok = M <= kGemvMaxTokens ? 16 : 0;
  if (int st = gemm_prepare(X8, sx, packed, s1, M, N, K, group, Y, nullptr, tok, 0, ws, ws_bytes, L))
    return st;
  if (L.p.tok != 16 || L.p.cs != 1) return QOQ_ERR_UNSUPPORTED;
  // One kernel: every CTA copies the FP16 token rows into shared memory,
  // computes their scales and writes X8 (identical bytes from every CTA)
  // before its X producer reads it; CTA 0 writes sx.  The preceding kernel
  // is the caller's, so the weight stream waits for it too.
  L.a.X = static_cast<const __half*>(X);
  L.a.X8 = X8;
  return gemm_launch(L, stream, /*weights_independent=*/false, false);
}

extern "C" int qoq_w4a8_gate_up_silu(const int8_t* X8, const void* sx, const void* packed,
                                     const void* s1, int M, int I, int K, int group, void* H,
                                     int8_t* H8, void* sh, void* stream) {
  if (!X8 || !sx || !packed || !s1 || !H || !H8 || !sh) return QOQ_ERR_INVALID_ARG;
  if (M <= 0 || I <= 0 || I % 64 != 0) return QOQ_ERR_INVALID_ARG;
  if (!aligned16(H) || !aligned16(H8) || !aligned16(sh)) return QOQ_ERR_INVALID_ARG;
  // K is not split (each CTA's epilogue needs the whole sum of both halves)
  // and the token tile is one the gate_up epilogue is built for
  int tok = 0;
  if (M > 64) tok = 128;
  GemmLaunch L;
  if (int st = gemm_prepare(X8, sx, packed, s1, M, 2 * I, K, group, H, nullptr, tok, 1, nullptr,
                            0, L))
    return st;
  L.gate_up = true;
  if (int st = gemm_launch(L, stream, /*weights_independent=*/false, false)) return st;
  // the per-token INT8 quantization of H for the down projection, launched
  // as the GEMM's programmatic dependent (it waits for the GEMM to complete)
  return launch_act_quant(H, M, I, H8, sh, stream, true, nullptr);
}

extern "C" int qoq_gemm_plan(int M, int N, int K, int group, int* tok_tile, int* splits, int* ctas,
                             int* stages) {
  if (M <= 0) return QOQ_ERR_INVALID_ARG;
  if (int st = check_weight_shape(N, K, group)) return st;
  const Plan p = make_plan(M, N, K, 0, 0);
  if (tok_tile) *tok_tile = p.tok;
  if (splits) *splits = p.splits;
  if (ctas) *ctas = p.grid;
  if (stages) *stages = p.stages;
  return QOQ_OK;
}

namespace qoq {
namespace {
// One warp waits, with the library's bounded wait, on an mbarrier that
// nothing ever arrives at: the wait gives up after its SM-clock limit (about
// two seconds), records kErrSelfTest in the error word and the kernel returns.
__global__ void __launch_bounds__(32, 1) wait_timeout_selftest_kernel() {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t abort_word;
  volatile uint32_t* abort_flag = &abort_word;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_word = 0u;
    fence_mbar_init();
  }
  __syncwarp();
  mbar_wait(smem_u32(&bar), 0, abort_flag, &g_error_word, kErrSelfTest);
}
}  // namespace
}  // namespace qoq

extern "C" int qoq_selftest_wait_timeout(void* stream) {
  if (int st = check_device()) return st;
  wait_timeout_selftest_kernel<<<1, 32, 0, as_stream(stream)>>>();
  return launch_status();
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

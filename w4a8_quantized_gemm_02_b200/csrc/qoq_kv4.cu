// 4-bit KV cache and the decode attention over it.
//
// Method: "QServe: Cuantificación W4A8KV4 y Co-diseño del Sistema para un
// Servicio Eficiente de LLM", abstract (W4A8KV4: a 4-bit KV cache) and
// "QServe: W4A8KV4 Quantization and System Co-design for Efficient LLM
// Serving" (velog notes), Insight (the fused attention is made memory-bound,
// so that the 4-bit cache turns into speed).  The pages fix no cache format;
// the one here: every (token, KV head) vector x of 128 FP16 values is
// quantized on its own to UINT4 codes q with an FP16 scale s and an FP16
// offset m (the vector's minimum), x^ = s q + m, with
// s = fp16((max - min) / 15) and q = clamp(rne((x - min) / s), 0, 15) in
// IEEE binary32 (q = 0 when s = 0).
//
// Decode attention, one query token per sequence: query head h reads KV head
// h / g (g = Hq / Hkv, grouped-query attention); score_t = q . k^_t / sqrt(d)
// over the sequence's first L_b tokens; out = softmax(score) . v^.
//
// The attention never dequantizes a vector.  With k^ = s q + m,
//     q_h . k^_t = s_t (q_h . c_t) + m_t Q_h,     Q_h = sum_i q_h,i,
//     sum_t p_t v^_t = sum_t (p_t s_t) c_t + sum_t p_t m_t,
// so the tensor cores multiply the raw codes c, which are exact FP16
// numbers, by FP16 queries (and by the FP16 weights p s) and accumulate in
// FP32 (mma.sync m16n8k16: exact products, FP32 sums).  The codes are the
// 16-row operand: S^T = C_K Q^T (16 tokens x 8 heads) and O^T += C_V^T P^T
// (16 dimensions x 8 heads), so one MMA covers 16 tokens or 16 dimensions
// and up to 8 query heads of a KV head, and the probabilities move from the
// S^T accumulator to the P^T operand with one 8x8 transpose (movmatrix) per
// half.  Each code becomes FP16 by masking its nibble into the low bits of a
// half: the bits 0x000c are the subnormal c * 2^-24, so a shift and an AND
// make two operands, and the factor 2^24 goes back onto the FP32 sums.  The
// tensor cores keep the arithmetic below the memory time, which CUDA-core
// FP32 would not at 4 query heads per KV head (512 multiply-adds per 136
// cache bytes).
//
// Layouts (per (batch, KV head) pair, L tokens, L a multiple of 16): the K
// and the V codes of a block of 16 tokens are 1024 bytes each, 32 runs of
// 32 bytes, run r = 4 gid + tig holding eight 32-bit words; word w, nibble
// p (bits 4p..4p+3), j = p & 3, e = p >> 2 holds
//  - K: token gid + 8 (j & 1), dimension 16 w + 2 tig + e + 8 (j >> 1)
//  - V: token 2 tig + e + 8 (j >> 1), dimension 16 w + gid + 8 (j & 1)
// (the A fragments of the two products for lane r: it loads its 32 bytes).
// Scales: four FP16 per token, (s_K, m_K, s_V, m_V).
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>

#include <type_traits>

#include "qoq.h"
#include "qoq_device.cuh"
#include "qoq_internal.h"

namespace qoq {
namespace {

constexpr int kHeadDim = 128;
constexpr int kWarpsPerCta = 4;
constexpr int kRingStages = 4;       // per warp: blocks of 16 tokens in flight
// a partial result per head: max, sum, two unused words, 128 outputs (the
// outputs start 16-byte aligned)
constexpr int kPartFloats = 4 + kHeadDim;

// ---------------------------------------------------------------------------
// Quantization
// ---------------------------------------------------------------------------

struct Quant4 {
  __half s, m;
  float sf, mn;
};

// Scale and offset of the warp's vector from each lane's four values.
__device__ __forceinline__ Quant4 kv4_params(const float (&x)[4]) {
  float mn = fminf(fminf(x[0], x[1]), fminf(x[2], x[3]));
  float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  Quant4 r;
  r.s = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), 15.0f));
  r.sf = __half2float(r.s);
  r.mn = mn;
  r.m = mn == 0.0f ? __float2half_rn(0.0f) : __float2half_rn(mn);   // exact: mn is an FP16 value
  return r;
}

__device__ __forceinline__ int kv4_code(float x, const Quant4& p) {
  if (!(p.sf > 0.0f)) return 0;
  const int c = __float2int_rn(__fdiv_rn(__fsub_rn(x, p.mn), p.sf));
  return c < 0 ? 0 : (c > 15 ? 15 : c);
}

// Nibble positions of a block's codes: the (token, dimension) of word w
// (0..7) of run r (0..31), nibble p, for K and for V.
__device__ __forceinline__ void k_slot(int r, int w, int p, int& tok, int& dim) {
  const int gid = r >> 2, tig = r & 3, j = p & 3, e = p >> 2;
  tok = gid + 8 * (j & 1);
  dim = 16 * w + 2 * tig + e + 8 * (j >> 1);
}
__device__ __forceinline__ void v_slot(int r, int w, int p, int& tok, int& dim) {
  const int gid = r >> 2, tig = r & 3, j = p & 3, e = p >> 2;
  tok = 2 * tig + e + 8 * (j >> 1);
  dim = 16 * w + gid + 8 * (j & 1);
}

// One CTA per 16-token block of one (batch, KV head) pair; warp tau quantizes
// token 16 blk + tau (K and V) when it lies in [t0, t0 + T).  A block's codes
// interleave its 16 tokens, so the CTA gathers them in shared memory and
// writes the block's 2 x 1024 bytes, keeping the nibbles of the tokens
// outside the range from the existing block.
__global__ void __launch_bounds__(512)
kv4_quant_kernel(const __half* __restrict__ K, const __half* __restrict__ V, int Hkv, int T, int L,
                 int t0, uint8_t* __restrict__ kc, uint8_t* __restrict__ vc,
                 __half* __restrict__ sc) {
  __shared__ uint8_t codes[2][16][kHeadDim];
  __shared__ uint32_t covered;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;                        // b * Hkv + hk
  const int blk = t0 / 16 + blockIdx.x;
  const int t = blk * 16 + warp;                     // cache position of this warp's token
  const bool mine = t >= t0 && t < t0 + T;
  if (threadIdx.x == 0) covered = 0u;
  __syncthreads();
  if (mine) {
    if (lane == 0) atomicOr(&covered, 1u << warp);
    const size_t src = (static_cast<size_t>(bh) * T + (t - t0)) * kHeadDim + 4 * lane;
    float xk[4], xv[4];
    {
      const uint2 rk = *reinterpret_cast<const uint2*>(K + src);
      const uint2 rv = *reinterpret_cast<const uint2*>(V + src);
      const __half2* hk = reinterpret_cast<const __half2*>(&rk);
      const __half2* hv = reinterpret_cast<const __half2*>(&rv);
      const float2 k0 = __half22float2(hk[0]), k1 = __half22float2(hk[1]);
      const float2 v0 = __half22float2(hv[0]), v1 = __half22float2(hv[1]);
      xk[0] = k0.x; xk[1] = k0.y; xk[2] = k1.x; xk[3] = k1.y;
      xv[0] = v0.x; xv[1] = v0.y; xv[2] = v1.x; xv[3] = v1.y;
    }
    const Quant4 pk = kv4_params(xk);
    const Quant4 pv = kv4_params(xv);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      codes[0][warp][4 * lane + u] = static_cast<uint8_t>(kv4_code(xk[u], pk));
      codes[1][warp][4 * lane + u] = static_cast<uint8_t>(kv4_code(xv[u], pv));
    }
    if (lane == 0) {
      __half2 h[2] = {__halves2half2(pk.s, pk.m), __halves2half2(pv.s, pv.m)};
      *reinterpret_cast<uint2*>(sc + (static_cast<size_t>(bh) * L + t) * 4) =
          *reinterpret_cast<const uint2*>(h);
    }
  }
  __syncthreads();
  // thread k builds word w = k % 8 of run r = (k / 8) % 32 of the K block
  // (k < 256) or the V block (k >= 256)
  const int k = threadIdx.x;
  const int which = k >> 8, r = (k >> 3) & 31, w = k & 7;
  uint8_t* base = which ? vc : kc;
  uint32_t* dst =
      reinterpret_cast<uint32_t*>(base + (static_cast<size_t>(bh) * (L / 16) + blk) * 1024) +
      (k & 255);
  const uint32_t cov = covered;
  uint32_t word = cov == 0xffffu ? 0u : *dst;
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    int tok, dim;
    if (which) v_slot(r, w, p, tok, dim);
    else k_slot(r, w, p, tok, dim);
    if (cov & (1u << tok)) {
      word &= ~(0xfu << (4 * p));
      word |= static_cast<uint32_t>(codes[which][tok][dim]) << (4 * p);
    }
  }
  *dst = word;
}

// ---------------------------------------------------------------------------
// Decode attention
// ---------------------------------------------------------------------------

__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 8x8 transpose of 16-bit elements across the warp: lane 4 r + c holds row r,
// columns 2c and 2c + 1, before and after.
__device__ __forceinline__ uint32_t transpose8x8(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// Codes enter the tensor cores as FP16 subnormals: the pairs masked from
// bits 0..3 of each half are c * 2^-24, those masked from bits 4..7 are
// c * 2^-20 (no shift needed).  In both products the latter land on rows 8..15
// of the 16-row operand (tokens gid + 8 of S^T, dimensions gid + 8 of O^T),
// so each accumulator row has one factor: kRowScale0 for rows 0..7,
// kRowScale1 for rows 8..15.  With kCodesAsSubnormals false the codes are
// made exact normal FP16 integers instead (0x6400 | c is 1024 + c, minus
// 1024) and both factors are 1.
constexpr bool kCodesAsSubnormals = true;
constexpr float kRowScale0 = kCodesAsSubnormals ? 16777216.0f : 1.0f;
constexpr float kRowScale1 = kCodesAsSubnormals ? 1048576.0f : 1.0f;

// Two codes (nibbles j and j + 4 of `word`) as an FP16 pair.
__device__ __forceinline__ uint32_t codes_h2(uint32_t word, int j) {
  const uint32_t m = (word >> (4 * j)) & 0x000f000fu;
  if constexpr (kCodesAsSubnormals) {
    return m;
  } else {
    const uint32_t n = m | 0x64006400u;
    const __half2 h = __hsub2(*reinterpret_cast<const __half2*>(&n), __float2half2_rn(1024.0f));
    return *reinterpret_cast<const uint32_t*>(&h);
  }
}

// The A fragment (16 rows x 16 k) held in one word of a run: one shift and
// four masks.  The pairs j = 1 and 3 (rows 8..15) stay at c * 2^-20.
__device__ __forceinline__ void a_frag(uint32_t word, uint32_t (&a)[4]) {
  if constexpr (kCodesAsSubnormals) {
    const uint32_t hi = word >> 8;
    a[0] = word & 0x000f000fu;
    a[1] = word & 0x00f000f0u;
    a[2] = hi & 0x000f000fu;
    a[3] = hi & 0x00f000f0u;
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j) a[j] = codes_h2(word, j);
  }
}

// 2^x by the SFU's approximation (relative error ~2^-22, far inside the
// attention's tolerance); 2^-inf = 0.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// reductions over the 8 lanes that share lane % 4 (the 8 token rows of S^T)
__device__ __forceinline__ float rows_max(float v) {
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
  return fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
}
__device__ __forceinline__ float rows_sum(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 4);
  v += __shfl_xor_sync(0xffffffffu, v, 8);
  return v + __shfl_xor_sync(0xffffffffu, v, 16);
}

// Per warp and stage: the block's K codes (1024 bytes), V codes (1024) and
// scales (128).  Each copy instruction of the warp moves 512 contiguous bytes
// (lane l: bytes 16 l .. +15 of the half), so every L2 sector is requested
// once; the 16-byte chunk c of a code block goes to slot
// c ^ ((c >> 3) & 1), which lets lane l read chunks 2l and 2l + 1 (its run)
// without bank conflicts.
constexpr int kStageBytes = 1024 + 1024 + 128;

__device__ __forceinline__ int chunk_slot(int c) { return c ^ ((c >> 3) & 1); }

// Grid (nsplit, B * Hkv), four warps.  CTA sigma covers the 16-token blocks
// [sigma * bps, (sigma + 1) * bps) of its pair, warp w every fourth of them
// from w on.  Each warp keeps, for heads 2 tig and 2 tig + 1 of the group (g
// <= 8), the running maximum (log2 units), the sum of 2^(score - max), the
// offset term sum p m_V, and O^T in 8 accumulator tiles; at the end the four
// warps' results are merged in shared memory and the CTA leaves one partial
// result per head: ws[pair][sigma][head] = (max, sum, 128 outputs), or, when
// it covers the whole sequence (nsplit = 1), the output itself.
__global__ void __launch_bounds__(32 * kWarpsPerCta)
kv4_decode_kernel(const __half* __restrict__ Q, const uint8_t* __restrict__ kc,
                  const uint8_t* __restrict__ vc, const __half* __restrict__ sc,
                  const int* __restrict__ seqlen, int Hq, int Hkv, int L, int g, int bps,
                  float* __restrict__ ws, __half* __restrict__ out) {
  __shared__ __align__(16) uint8_t smem[kWarpsPerCta * kRingStages * kStageBytes];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int bh = blockIdx.y;
  const int b = bh / Hkv, hk = bh - b * Hkv;
  int Lb = seqlen[b];
  Lb = Lb < 0 ? 0 : (Lb > L ? L : Lb);
  const int nblk = (Lb + 15) >> 4;
  const int blk0 = blockIdx.x * bps + warp;
  int blk1 = (blockIdx.x + 1) * bps;
  blk1 = blk1 < nblk ? blk1 : nblk;
  const int niter = blk0 < blk1 ? (blk1 - blk0 + kWarpsPerCta - 1) / kWarpsPerCta : 0;

  // the next block to copy (pointers advance by kWarpsPerCta blocks a copy):
  // lane l moves chunks l and 32 + l of the K and of the V block, and lanes
  // 0..7 the eight 16-byte chunks of the block's scales
  const uint8_t* kp = kc + (static_cast<size_t>(bh) * (L / 16) + blk0) * 1024 + 16 * lane;
  const uint8_t* vp = vc + (static_cast<size_t>(bh) * (L / 16) + blk0) * 1024 + 16 * lane;
  const uint8_t* sp =
      reinterpret_cast<const uint8_t*>(sc + (static_cast<size_t>(bh) * L + 16 * blk0) * 4) +
      16 * (lane & 7);
  uint8_t* wring = smem + warp * kRingStages * kStageBytes;
  const uint32_t ring0 = static_cast<uint32_t>(__cvta_generic_to_shared(wring));
  const uint32_t s_lo = 16 * chunk_slot(lane), s_hi = 16 * chunk_slot(32 + lane);
  auto issue = [&](int it) {
    if (it < niter) {
      const uint32_t dst = ring0 + (it % kRingStages) * kStageBytes;
      cp_async16(dst + s_lo, kp);
      cp_async16(dst + s_hi, kp + 512);
      cp_async16(dst + 1024 + s_lo, vp);
      cp_async16(dst + 1024 + s_hi, vp + 512);
      if (lane < 8) cp_async16(dst + 2048 + 16 * lane, sp);
      kp += kWarpsPerCta * 1024;
      vp += kWarpsPerCta * 1024;
      sp += kWarpsPerCta * 16 * 8;
    }
    cp_async_commit();   // an empty group past the end keeps the counting uniform
  };
#pragma unroll
  for (int it = 0; it < kRingStages - 1; ++it) issue(it);

  // Q^T as B fragments (k = dimensions, n = head gid; zero past g) and the
  // row sums Q_h of heads 2 tig and 2 tig + 1
  const bool qrow = gid < g;
  const __half* q = Q + (static_cast<size_t>(b) * Hq + hk * g + gid) * kHeadDim;
  uint32_t qb[8][2];
  float qs = 0.0f;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const int d0 = 16 * ks + 2 * tig;
    qb[ks][0] = qrow ? *reinterpret_cast<const uint32_t*>(q + d0) : 0u;
    qb[ks][1] = qrow ? *reinterpret_cast<const uint32_t*>(q + d0 + 8) : 0u;
    const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&qb[ks][0]));
    const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&qb[ks][1]));
    qs += (f0.x + f0.y) + (f1.x + f1.y);
  }
  qs += __shfl_xor_sync(0xffffffffu, qs, 1);
  qs += __shfl_xor_sync(0xffffffffu, qs, 2);                    // Q_gid in lanes 4 gid ..
  // scores in log2 units: (q . k^) * log2(e) / sqrt(128)
  const float kScale = 1.4426950408889634f / 11.313708498984761f;
  const float qh[2] = {__shfl_sync(0xffffffffu, qs, 8 * tig) * kScale,       // Q of head 2 tig
                       __shfl_sync(0xffffffffu, qs, 8 * tig + 4) * kScale};  // and 2 tig + 1
  float acc[8][4];
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.0f;
  float mrun[2] = {-INFINITY, -INFINITY}, lsum[2] = {0.0f, 0.0f}, msum[2] = {0.0f, 0.0f};

  for (int it = 0; it < niter; ++it) {
    // the block's copies landed (this lane's), then the whole warp's
    cp_async_wait<kRingStages - 2>();
    __syncwarp();
    const int blk = blk0 + it * kWarpsPerCta;
    const uint8_t* stage = wring + (it % kRingStages) * kStageBytes;
    const uint4 kq0 = *reinterpret_cast<const uint4*>(stage + 16 * chunk_slot(2 * lane));
    const uint4 kq1 = *reinterpret_cast<const uint4*>(stage + 16 * chunk_slot(2 * lane + 1));
    const uint4 vq0 = *reinterpret_cast<const uint4*>(stage + 1024 + 16 * chunk_slot(2 * lane));
    const uint4 vq1 = *reinterpret_cast<const uint4*>(stage + 1024 + 16 * chunk_slot(2 * lane + 1));
    uint4 sq;
    *reinterpret_cast<uint2*>(&sq.x) = *reinterpret_cast<const uint2*>(stage + 2048 + 8 * gid);
    *reinterpret_cast<uint2*>(&sq.z) = *reinterpret_cast<const uint2*>(stage + 2048 + 64 + 8 * gid);
    // every lane has read the stage before any lane copies into it again
    __syncwarp();
    issue(it + kRingStages - 1);

    // the block's work; only a block that reaches past the sequence's end
    // masks its tokens (kMasked), the others skip the selects
    auto step = [&](auto masked) {
      constexpr bool kMasked = decltype(masked)::value;
      // S^T = C_K Q^T: rows tokens (gid, gid + 8), columns heads (2 tig, +1)
      // (two accumulators, even and odd k-steps, halve the dependent chain)
      float s[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      {
        float s2[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        const uint32_t wk[8] = {kq0.x, kq0.y, kq0.z, kq0.w, kq1.x, kq1.y, kq1.z, kq1.w};
#pragma unroll
        for (int ks = 0; ks < 8; ks += 2) {
          uint32_t a[4], a2[4];
          a_frag(wk[ks], a);
          a_frag(wk[ks + 1], a2);
          mma_16816(s, a, qb[ks][0], qb[ks][1]);
          mma_16816(s2, a2, qb[ks + 1][0], qb[ks + 1][1]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) s[i] += s2[i];
      }
      // scales of tokens gid (first 8 bytes) and gid + 8
      const __half* hs = reinterpret_cast<const __half*>(&sq);
      float skt[2], mkt[2], svt[2], mvt[2];
      bool valid[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        // row r of S^T is token gid + 8 r: its codes carry 1 / kRowScale<r>
        skt[r] = __half2float(hs[4 * r + 0]) * ((r ? kRowScale1 : kRowScale0) * kScale);
        mkt[r] = __half2float(hs[4 * r + 1]);
        svt[r] = __half2float(hs[4 * r + 2]);
        mvt[r] = __half2float(hs[4 * r + 3]);
        valid[r] = !kMasked || blk * 16 + gid + 8 * r < Lb;
      }
      float bm[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int r = 0; r < 2; ++r) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const float v =
              !kMasked || valid[r] ? skt[r] * s[2 * r + c] + mkt[r] * qh[c] : -INFINITY;
          s[2 * r + c] = v;
          bm[c] = fmaxf(bm[c], v);
        }
      }
      float al[2];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const float mn = fmaxf(mrun[c], rows_max(bm[c]));
        al[c] = mn == -INFINITY ? 1.0f : fast_exp2(mrun[c] - mn);
        mrun[c] = mn;
        lsum[c] *= al[c];
        msum[c] *= al[c];
      }
      if (al[0] != 1.0f || al[1] != 1.0f) {
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          acc[mt][0] *= al[0];
          acc[mt][1] *= al[1];
          acc[mt][2] *= al[0];
          acc[mt][3] *= al[1];
        }
      }
      // the weights w = p s_V (a token past the length has p = 0 and scales
      // that were never written: its terms are left out, not multiplied by 0)
      float wt[4];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const float p = mrun[c] == -INFINITY ? 0.0f : fast_exp2(s[2 * r + c] - mrun[c]);
          lsum[c] += p;
          if constexpr (kMasked) {
            wt[2 * r + c] = valid[r] ? p * svt[r] : 0.0f;
            msum[c] += valid[r] ? p * mvt[r] : 0.0f;
          } else {
            wt[2 * r + c] = p * svt[r];
            msum[c] += p * mvt[r];
          }
        }
      }
      // P^T as the B fragment, in an FP16 high part and the FP16 rest
      const uint32_t top = pack_h2(wt[0], wt[1]), bot = pack_h2(wt[2], wt[3]);
      const float2 ft = __half22float2(*reinterpret_cast<const __half2*>(&top));
      const float2 fb = __half22float2(*reinterpret_cast<const __half2*>(&bot));
      const uint32_t b0h = transpose8x8(top), b1h = transpose8x8(bot);
      const uint32_t b0l = transpose8x8(pack_h2(wt[0] - ft.x, wt[1] - ft.y));
      const uint32_t b1l = transpose8x8(pack_h2(wt[2] - fb.x, wt[3] - fb.y));
      // O^T += C_V^T P^T, dimension tile mt from V word mt
      const uint32_t wv[8] = {vq0.x, vq0.y, vq0.z, vq0.w, vq1.x, vq1.y, vq1.z, vq1.w};
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        uint32_t a[4];
        a_frag(wv[mt], a);
        mma_16816(acc[mt], a, b0h, b1h);
        mma_16816(acc[mt], a, b0l, b1l);
      }
    };
    if (blk * 16 + 16 <= Lb) step(std::false_type{});
    else step(std::true_type{});
  }
  cp_async_wait<0>();
  __syncthreads();   // the ring becomes the merge area

  // per warp and head: max, sum, 128 outputs (sum p s_V c + sum p m_V)
  float* mrg = reinterpret_cast<float*>(smem);     // [warp][8 heads][kPartFloats]
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    const int h = 2 * tig + c;
    const float l = rows_sum(lsum[c]);
    const float mo = rows_sum(msum[c]);
    float* row = mrg + (warp * 8 + h) * kPartFloats;
    if (gid == 0) {
      row[0] = mrun[c];
      row[1] = l;
    }
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      row[4 + 16 * mt + gid] = acc[mt][c] * kRowScale0 + mo;
      row[4 + 16 * mt + gid + 8] = acc[mt][2 + c] * kRowScale1 + mo;
    }
  }
  __syncthreads();
  // thread i of the CTA merges head i / 16's dimensions 8 (i % 16) .. +7
  {
    const int h = threadIdx.x >> 4, d0 = 8 * (threadIdx.x & 15);
    if (h < g) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kWarpsPerCta; ++w) M = fmaxf(M, mrg[(w * 8 + h) * kPartFloats]);
      float f[kWarpsPerCta];
      float den = 0.0f;
#pragma unroll
      for (int w = 0; w < kWarpsPerCta; ++w) {
        const float* row = mrg + (w * 8 + h) * kPartFloats;
        f[w] = M == -INFINITY ? 0.0f : exp2f(row[0] - M);
        den += f[w] * row[1];
      }
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        v[u] = 0.0f;
#pragma unroll
        for (int w = 0; w < kWarpsPerCta; ++w)
          v[u] += f[w] == 0.0f ? 0.0f : f[w] * mrg[(w * 8 + h) * kPartFloats + 4 + d0 + u];
      }
      if (gridDim.x == 1) {
        // the whole sequence in this CTA: the output directly
        __half2 o[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          o[u] = __floats2half2_rn(den > 0.0f ? __fdiv_rn(v[2 * u], den) : 0.0f,
                                   den > 0.0f ? __fdiv_rn(v[2 * u + 1], den) : 0.0f);
        *reinterpret_cast<uint4*>(out + (static_cast<size_t>(b) * Hq + hk * g + h) * kHeadDim +
                                  d0) = *reinterpret_cast<const uint4*>(o);
      } else {
        float* part =
            ws + ((static_cast<size_t>(bh) * gridDim.x + blockIdx.x) * g + h) * kPartFloats;
        if ((threadIdx.x & 15) == 0) {
          part[0] = M;
          part[1] = den;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) part[4 + d0 + u] = v[u];
      }
    }
  }
}

// out[b][h] from the partial results of the nsplit CTAs of its pair: eight
// warps take every eighth split, a lane four dimensions, and the warps'
// sums are added in shared memory.
__global__ void __launch_bounds__(256)
kv4_combine_kernel(const float* __restrict__ ws, int Hq, int Hkv, int g, int nsplit,
                   __half* __restrict__ out) {
  __shared__ float red_m[8];
  __shared__ float4 red_num[8][32];
  __shared__ float red_den[8];
  const int bq = blockIdx.x;                 // b * Hq + h
  const int b = bq / Hq, h = bq - b * Hq;
  const int hk = h / g, r = h - hk * g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* base = ws + ((static_cast<size_t>(b) * Hkv + hk) * nsplit * g + r) * kPartFloats;
  const size_t stride = static_cast<size_t>(g) * kPartFloats;
  float M = -INFINITY;
  for (int p = threadIdx.x; p < nsplit; p += blockDim.x) M = fmaxf(M, base[p * stride]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if (lane == 0) red_m[warp] = M;
  __syncthreads();
  M = red_m[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) M = fmaxf(M, red_m[w]);
  float4 num = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  float den = 0.0f;
  if (M != -INFINITY) {
#pragma unroll 4
    for (int p = warp; p < nsplit; p += 8) {
      const float* pp = base + p * stride;
      const float mp = pp[0];
      if (mp == -INFINITY) continue;
      const float f = exp2f(mp - M);
      den += f * pp[1];
      const float4 a = *reinterpret_cast<const float4*>(pp + 4 + 4 * lane);
      num.x += f * a.x;
      num.y += f * a.y;
      num.z += f * a.z;
      num.w += f * a.w;
    }
  }
  red_num[warp][lane] = num;
  if (lane == 0) red_den[warp] = den;
  __syncthreads();
  if (warp == 0) {
    float4 n = red_num[0][lane];
    float d = red_den[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) {
      const float4 a = red_num[w][lane];
      n.x += a.x;
      n.y += a.y;
      n.z += a.z;
      n.w += a.w;
      d += red_den[w];
    }
    __half2 o[2];
    o[0] = __floats2half2_rn(d > 0.0f ? __fdiv_rn(n.x, d) : 0.0f,
                             d > 0.0f ? __fdiv_rn(n.y, d) : 0.0f);
    o[1] = __floats2half2_rn(d > 0.0f ? __fdiv_rn(n.z, d) : 0.0f,
                             d > 0.0f ? __fdiv_rn(n.w, d) : 0.0f);
    *reinterpret_cast<uint2*>(out + static_cast<size_t>(bq) * kHeadDim + 4 * lane) =
        *reinterpret_cast<const uint2*>(o);
  }
}

struct AttnPlan {
  int nsplit, bps;
};



// Splits of the sequence axis: about four waves of CTAs (four resident per
// SM), each warp keeping at least eight blocks of 16 tokens (fewer, longer
// CTAs measured faster than more, shorter ones), at most 64 splits (the
// merge reads every split).
AttnPlan attn_plan(int B, int Hkv, int L) {
  const long pairs = static_cast<long>(B) * Hkv;
  const int nblk = L / 16;
  const long want = 4L * 4 * sm_count();
  long ns = (want + pairs - 1) / pairs;
  long cap = nblk / (8 * kWarpsPerCta);
  if (cap > 64) cap = 64;
  if (ns > cap) ns = cap;
  if (ns < 1) ns = 1;
  AttnPlan p;
  p.bps = static_cast<int>((nblk + ns - 1) / ns);
  p.nsplit = (nblk + p.bps - 1) / p.bps;
  return p;
}

int check_kv_shape(int B, int Hkv, int L, int d) {
  if (B <= 0 || Hkv <= 0 || L <= 0) return QOQ_ERR_INVALID_ARG;
  if (d != kHeadDim || L % 16 != 0) return QOQ_ERR_UNSUPPORTED;
  if (static_cast<long>(B) * Hkv > 65535) return QOQ_ERR_UNSUPPORTED;   // grid rows
  return QOQ_OK;
}

}  // namespace
}  // namespace qoq

using namespace qoq;

extern "C" int qoq_kv4_cache_bytes(int B, int Hkv, int L, int d, size_t* k_bytes, size_t* v_bytes,
                                   size_t* scale_bytes) {
  if (int st = check_kv_shape(B, Hkv, L, d)) return st;
  const size_t tokens = static_cast<size_t>(B) * Hkv * L;
  if (k_bytes) *k_bytes = tokens / 16 * 1024;
  if (v_bytes) *v_bytes = tokens / 16 * 1024;
  if (scale_bytes) *scale_bytes = tokens * 8;
  return QOQ_OK;
}

extern "C" int qoq_kv4_quantize(const void* K, const void* V, int B, int Hkv, int T, int d, int L,
                                int t0, uint8_t* k_codes, uint8_t* v_codes, void* scales,
                                void* stream) {
  if (!K || !V || !k_codes || !v_codes || !scales) return QOQ_ERR_INVALID_ARG;
  if (int st = check_kv_shape(B, Hkv, L, d)) return st;
  if (T <= 0 || t0 < 0 || static_cast<long>(t0) + T > L) return QOQ_ERR_INVALID_ARG;
  if (!aligned16(K) || !aligned16(V) || !aligned16(k_codes) || !aligned16(v_codes) ||
      !aligned16(scales))
    return QOQ_ERR_INVALID_ARG;
  if (int st = check_device()) return st;
  const int nblk = (t0 + T - 1) / 16 - t0 / 16 + 1;
  dim3 grid(static_cast<unsigned>(nblk), static_cast<unsigned>(B * Hkv));
  kv4_quant_kernel<<<grid, 512, 0, as_stream(stream)>>>(
      static_cast<const __half*>(K), static_cast<const __half*>(V), Hkv, T, L, t0, k_codes,
      v_codes, static_cast<__half*>(scales));
  return launch_status();
}

extern "C" size_t qoq_kv4_attention_workspace_bytes(int B, int Hq, int Hkv, int L, int d) {
  if (check_kv_shape(B, Hkv, L, d) || Hq <= 0 || Hq % Hkv != 0 || Hq / Hkv > 8) return 0;
  const AttnPlan p = attn_plan(B, Hkv, L);
  return static_cast<size_t>(B) * Hkv * p.nsplit * (Hq / Hkv) * kPartFloats * sizeof(float);
}

extern "C" int qoq_kv4_decode_attention(const void* Q, const uint8_t* k_codes,
                                        const uint8_t* v_codes, const void* scales,
                                        const int* seqlen, int B, int Hq, int Hkv, int L, int d,
                                        void* out, void* ws, size_t ws_bytes, void* stream) {
  if (!Q || !k_codes || !v_codes || !scales || !seqlen || !out) return QOQ_ERR_INVALID_ARG;
  if (int st = check_kv_shape(B, Hkv, L, d)) return st;
  if (Hq <= 0 || Hq % Hkv != 0) return QOQ_ERR_INVALID_ARG;
  if (Hq / Hkv > 8) return QOQ_ERR_UNSUPPORTED;
  if (!aligned16(Q) || !aligned16(k_codes) || !aligned16(v_codes) || !aligned16(scales) ||
      !aligned16(out) || (reinterpret_cast<uintptr_t>(seqlen) & 3u))
    return QOQ_ERR_INVALID_ARG;
  const size_t need = qoq_kv4_attention_workspace_bytes(B, Hq, Hkv, L, d);
  if (ws == nullptr || ws_bytes < need || !aligned16(ws)) return QOQ_ERR_WORKSPACE;
  if (int st = check_device()) return st;
  const AttnPlan p = attn_plan(B, Hkv, L);
  const int g = Hq / Hkv;
  cudaStream_t s = as_stream(stream);
  dim3 grid(static_cast<unsigned>(p.nsplit), static_cast<unsigned>(B * Hkv));
  float* parts = static_cast<float*>(ws);
  kv4_decode_kernel<<<grid, 32 * kWarpsPerCta, 0, s>>>(
      static_cast<const __half*>(Q), k_codes, v_codes, static_cast<const __half*>(scales), seqlen,
      Hq, Hkv, L, g, p.bps, parts, static_cast<__half*>(out));
  if (int st = launch_status()) return st;
  if (p.nsplit > 1) {
    kv4_combine_kernel<<<B * Hq, 256, 0, s>>>(parts, Hq, Hkv, g, p.nsplit,
                                              static_cast<__half*>(out));
    return launch_status();
  }
  return QOQ_OK;
}

// Stage 1 kernels: block mean pooling, pooled scores + cumulative-energy
// selection, and the per-head tile order.
//
// Stage 1 of the two-stage filter in the SpargeAttn abstract predicts the
// attention map cheaply; the kept set per query block is the one the DynSparse
// article ("Training-free sparse attention based on cumulative energy
// filtering") describes: a fixed recall of attention energy, i.e. a per-row
// threshold derived from the cumulative energy.
#pragma once

#include <climits>

#include <cuda_fp8.h>

#include "sa_device.cuh"

namespace sa {

// Shared memory of the pairing kernel for Nb blocks per head without the bitsets:
// the sort keys of the blocks and of the tiles (powers of two), the pairs, the
// order, the matching state and the scan scratch.
__host__ __device__ inline int pair_base_smem_bytes(int Nb) {
  int p = 2, p2 = 2;
  while (p < Nb) p <<= 1;
  const int Tq = (Nb + 1) / 2;
  while (p2 < Tq) p2 <<= 1;
  return (p + p2) * 8 + (2 * Tq + 4 * Nb + 34) * 4;
}
// The pairing keeps the kept-set bitsets, regrouped by sorted position, in shared
// memory when they fit beside the rest (up to about 1,180 blocks per head), else in
// global memory (the plan workspace's bitsT region).
__host__ __device__ inline bool pair_bits_in_smem(int Nb) {
  return pair_base_smem_bytes(Nb) + Nb * ((Nb + 31) / 32) * 4 <= 227 * 1024;
}

// The pooled scores are computed in strips of 128 query blocks of one head
// (pooled_scores_tc_kernel) into a buffer of whole strips, then selected
// (select_kernel); the plan runs strip batches until every strip is done. The
// buffer holds at most kPlanScoreBytes (or, in a fixed scratch, what is left),
// and at least one strip.
constexpr size_t kPlanScoreBytes = 64ull << 20;
constexpr int kStripRows = 128;
__host__ __device__ inline int score_ld(int Nb) { return (Nb + 31) & ~31; }   // floats per score row
inline size_t score_strip_bytes(int Nb) { return static_cast<size_t>(kStripRows) * score_ld(Nb) * sizeof(float); }

// Byte offsets of the plan workspace: pooled Q and K (fp32 [B,H,Nb,d]), then per
// query block a 64-bit MinHash sort key and the kept set as a bitset of W words;
// when the pairing's copy of the bitsets does not fit in shared memory, that copy,
// word-major by sorted position ([B,H][W][Nb]); last the score strips (fp32
// [strips][128][score_ld(Nb)]). score_cap bounds the strips' bytes (at least one
// strip is always counted).
struct PlanWorkspace {
  size_t qp, kp, sig, bits, bitsT, scores, total;
  int W, strips, strips_per_batch;
};
inline PlanWorkspace plan_workspace(long long BH, int Nb, int D, size_t score_cap = kPlanScoreBytes) {
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  PlanWorkspace w;
  w.W = (Nb + 31) / 32;
  const size_t pooled = al(static_cast<size_t>(BH) * Nb * D * sizeof(float));
  const size_t bitset = al(static_cast<size_t>(BH) * Nb * w.W * sizeof(uint32_t));
  w.qp = 0;
  w.kp = pooled;
  w.sig = 2 * pooled;
  w.bits = w.sig + al(static_cast<size_t>(BH) * Nb * sizeof(unsigned long long));
  w.bitsT = w.bits + bitset;
  w.scores = w.bitsT + (pair_bits_in_smem(Nb) ? 0 : bitset);
  const long long strips = BH * ((Nb + kStripRows - 1) / kStripRows);
  const size_t sb = score_strip_bytes(Nb);
  long long fit = static_cast<long long>(score_cap / sb);
  fit = fit < 1 ? 1 : (fit > strips ? strips : fit);
  w.strips = static_cast<int>(strips);
  w.strips_per_batch = static_cast<int>(fit);
  w.total = w.scores + al(static_cast<size_t>(fit) * sb);
  return w;
}

// MurmurHash3's 32-bit finaliser (a published bijective mixer): MinHash of kept sets.
static __device__ __forceinline__ uint32_t mix32(uint32_t x) {
  // MurmurHash3's 32-bit finaliser (a published bijective mixer).
  x ^= x >> 16;
  x *= 0x85ebca6bu;
  x ^= x >> 13;
  x *= 0xc2b2ae35u;
  x ^= x >> 16;
  return x;
}

// ----------------------------------------------------------------------------
// Pool: Xp[bh, i, :] = mean of X[bh, 64 i : min(N, 64 i + 64), :], fp32.
// One CTA per (block, head) and per tensor (blockIdx.y: 0 = Q, 1 = K). Each
// thread loads 16-byte vectors (8 bf16) of a row; D/8 threads cover a row, so a
// warp reads whole rows contiguously. Partial sums meet in shared memory.
// HBM-bound: it is the one full pass over Q and K on the predictor side.
// With Q8 (and K8, qs, ks) given, the same pass also quantizes the block for the
// quantized-score forward, [B,H,N,d] bytes and [B,H,Nb] fp32 scales (scale 1,
// codes 0 for an all-zero block). qfmt = kScoreE4M3: FP8 E4M3, scale = amax / 448,
// codes = x * (448 / amax) rounded to nearest even and saturated; qfmt =
// kScoreI8: signed INT8, scale = amax / 127, codes = x * (127 / amax) rounded to
// the nearest integer, ties to even (|code| <= 127).
template <int D>
__global__ void __launch_bounds__(256) pool_kernel(const __nv_bfloat16* __restrict__ Q,
                                                   const __nv_bfloat16* __restrict__ K,
                                                   float* __restrict__ Qp, float* __restrict__ Kp,
                                                   int N, int Nb, uint8_t* __restrict__ Q8 = nullptr,
                                                   uint8_t* __restrict__ K8 = nullptr,
                                                   float* __restrict__ qs = nullptr,
                                                   float* __restrict__ ks = nullptr, int qfmt = kScoreE4M3) {
  constexpr int LPR = D / 8;          // threads per row
  constexpr int RPP = 256 / LPR;      // rows per pass
  __shared__ float part[RPP][D];
  __shared__ float wmax[8];
  const long long g = blockIdx.x;     // (bh, i) flattened
  const long long bh = g / Nb;
  const int i = static_cast<int>(g - bh * Nb);
  const __nv_bfloat16* src = (blockIdx.y == 0 ? Q : K) + (bh * N + static_cast<long long>(i) * kBlock) * D;
  float* dst = (blockIdx.y == 0 ? Qp : Kp) + g * D;
  const int rows = min(kBlock, N - i * kBlock);
  const int r0 = threadIdx.x / LPR;
  const int c8 = (threadIdx.x % LPR) * 8;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  // every load of the thread first (all in flight at once), then the sums
  constexpr int kPasses = kBlock / RPP;
  uint4 u[kPasses];
#pragma unroll
  for (int p = 0; p < kPasses; ++p) {
    const int r = r0 + p * RPP;
    u[p] = (r < rows) ? __ldg(reinterpret_cast<const uint4*>(src + static_cast<long long>(r) * D + c8))
                      : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int p = 0; p < kPasses; ++p) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u[p]);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h[e]);
      acc[2 * e] += f.x;
      acc[2 * e + 1] += f.y;
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[r0][c8 + e] = acc[e];
  uint8_t* q8 = (Q8 == nullptr) ? nullptr : (blockIdx.y == 0 ? Q8 : K8);
  float amax = 0.f;
  if (q8) {
    // largest |x| of the block (tail rows loaded as zeros)
#pragma unroll
    for (int p = 0; p < kPasses; ++p) {
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u[p]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h[e]);
        amax = fmax3(amax, fabsf(f.x), fabsf(f.y));
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = amax;
  }
  __syncthreads();
  if (threadIdx.x < D) {
    float s = 0.f;
#pragma unroll
    for (int r = 0; r < RPP; ++r) s += part[r][threadIdx.x];
    dst[threadIdx.x] = s / static_cast<float>(rows);
  }
  if (q8) {
    amax = fmax3(fmax3(wmax[0], wmax[1], wmax[2]), fmax3(wmax[3], wmax[4], wmax[5]), fmaxf(wmax[6], wmax[7]));
    const float qmax = qfmt == kScoreI8 ? 127.f : 448.f;
    const float inv = amax > 0.f ? qmax / amax : 0.f;
    if (threadIdx.x == 0) (blockIdx.y == 0 ? qs : ks)[g] = amax > 0.f ? amax / qmax : 1.f;
    uint8_t* dst8 = q8 + (bh * N + static_cast<long long>(i) * kBlock) * D;
#pragma unroll
    for (int p = 0; p < kPasses; ++p) {
      const int r = r0 + p * RPP;
      if (r < rows) {
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u[p]);
        uint32_t w[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float2 f0 = __bfloat1622float2(h[2 * e]), f1 = __bfloat1622float2(h[2 * e + 1]);
          if (qfmt == kScoreI8) {
            const float y[4] = {f0.x * inv, f0.y * inv, f1.x * inv, f1.y * inv};
            uint32_t b = 0;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int c = max(-127, min(127, __float2int_rn(y[q])));   // nearest, ties to even
              b |= (static_cast<uint32_t>(c) & 0xFFu) << (8 * q);
            }
            w[e] = b;
          } else {
            const uint32_t lo =
                __nv_cvt_float2_to_fp8x2(make_float2(f0.x * inv, f0.y * inv), __NV_SATFINITE, __NV_E4M3);
            const uint32_t hi =
                __nv_cvt_float2_to_fp8x2(make_float2(f1.x * inv, f1.y * inv), __NV_SATFINITE, __NV_E4M3);
            w[e] = lo | (hi << 16);
          }
        }
        *reinterpret_cast<uint2*>(dst8 + static_cast<long long>(r) * D + c8) = make_uint2(w[0], w[1]);
      }
    }
  }
}

// Ascending bitonic sort of 64 64-bit keys held two per lane by one warp: lane l
// holds elements 2l (v[0]) and 2l+1 (v[1]). Stages with partner distance 1 stay in
// the lane; longer ones exchange with lane l ^ (distance / 2).
static __device__ __forceinline__ void warp_bitonic_sort64(unsigned long long (&v)[2], int lane) {
#pragma unroll
  for (int k = 2; k <= 64; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j == 1) {
        const bool up = ((2 * lane) & k) == 0;
        const unsigned long long a = v[0], b = v[1];
        v[0] = up ? min(a, b) : max(a, b);
        v[1] = up ? max(a, b) : min(a, b);
      } else {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int i = 2 * lane + h;
          const unsigned long long o = __shfl_xor_sync(0xffffffffu, v[h], j >> 1);
          const bool up = (i & k) == 0, lower = (i & j) == 0;
          v[h] = (lower == up) ? min(v[h], o) : max(v[h], o);
        }
      }
    }
  }
}

// In-place ascending sort of n64 <= 64 (a power of two) 64-bit keys in shared
// memory by one warp (the caller synchronises afterwards).
static __device__ void warp_sort_keys(unsigned long long* keys, int n64, int lane) {
  unsigned long long v[2];
  v[0] = (2 * lane < n64) ? keys[2 * lane] : ~0ull;
  v[1] = (2 * lane + 1 < n64) ? keys[2 * lane + 1] : ~0ull;
  warp_bitonic_sort64(v, lane);
  if (2 * lane < n64) keys[2 * lane] = v[0];
  if (2 * lane + 1 < n64) keys[2 * lane + 1] = v[1];
}

// Selection of one row of at most 64 blocks by one warp, the sorted-prefix rule
// itself: e_j = exp(L_j - max) sorted descending (ties: lower j first), prefix sums
// in that order, and the kept set is the shortest prefix whose sum reaches tau times
// the total (every e_j > 0 when tau >= 1). Same outputs as select_row.
static __device__ __forceinline__ void select_row_sorted64(const float* row, int Nb, int i, long long bh,
                                                           float tau, int lane, uint8_t* __restrict__ mask,
                                                           int* __restrict__ count, int* __restrict__ idx,
                                                           unsigned long long* sig_out, uint32_t* brow) {
  const unsigned FULL = 0xffffffffu;
  const float LOG2E = 1.4426950408889634f;
  const int j0 = 2 * lane, j1 = 2 * lane + 1;
  const float x0 = (j0 < Nb) ? row[j0] : -INFINITY, x1 = (j1 < Nb) ? row[j1] : -INFINITY;
  float m = fmaxf(x0, x1);
#pragma unroll
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, o));
  // keys sorted ascending = e descending, then j ascending: ~((e bits << 32) | (0xffff - j))
  auto key = [&](float x, int j) -> unsigned long long {
    const float e = (j < Nb) ? ex2((x - m) * LOG2E) : 0.f;
    return ~((static_cast<unsigned long long>(__float_as_uint(e)) << 32) | static_cast<uint32_t>(0xffff - j));
  };
  unsigned long long v[2] = {key(x0, j0), key(x1, j1)};
  warp_bitonic_sort64(v, lane);
  // sorted positions 2*lane, 2*lane+1: their e and block index
  const unsigned long long u0 = ~v[0], u1 = ~v[1];
  const float e0 = __uint_as_float(static_cast<uint32_t>(u0 >> 32));
  const float e1 = __uint_as_float(static_cast<uint32_t>(u1 >> 32));
  const int s0 = 0xffff - static_cast<int>(u0 & 0xffffu), s1 = 0xffff - static_cast<int>(u1 & 0xffffu);
  // inclusive prefix sums in sorted order
  const float pair = e0 + e1;
  float inc = pair;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float y = __shfl_up_sync(FULL, inc, o);
    if (lane >= o) inc += y;
  }
  const float c1 = inc, c0 = inc - pair + e0;
  const float total = __shfl_sync(FULL, inc, 31);
  bool k0, k1;
  if (tau >= 1.f) {
    k0 = e0 > 0.f;
    k1 = e1 > 0.f;
  } else {
    const float T = tau * total;
    const unsigned b0 = __ballot_sync(FULL, c0 >= T), b1 = __ballot_sync(FULL, c1 >= T);
    const int r0 = b0 ? 2 * (__ffs(b0) - 1) : 1 << 30, r1 = b1 ? 2 * (__ffs(b1) - 1) + 1 : 1 << 30;
    const int rstar = min(r0, r1);                  // last kept sorted position
    k0 = 2 * lane <= rstar;
    k1 = 2 * lane + 1 <= rstar;
  }
  unsigned long long kept = (k0 ? 1ull << s0 : 0ull) | (k1 ? 1ull << s1 : 0ull);
#pragma unroll
  for (int o = 16; o; o >>= 1) kept |= __shfl_xor_sync(FULL, kept, o);
  // emit mask, ascending idx, count, MinHash key and bitset
  uint8_t* mrow = mask + (bh * Nb + i) * static_cast<long long>(Nb);
  int* irow = idx ? idx + (bh * Nb + i) * static_cast<long long>(Nb) : nullptr;
  uint32_t h1 = 0xffffffffu, h2 = 0xffffffffu;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int j = 32 * half + lane;
    if (j < Nb) {
      const bool keep = (kept >> j) & 1ull;
      mrow[j] = keep ? 1 : 0;
      if (keep) {
        if (irow) irow[__popcll(kept & ((1ull << j) - 1ull))] = j;
        h1 = min(h1, mix32(static_cast<uint32_t>(j) ^ 0x9e3779b9u));
        h2 = min(h2, mix32(static_cast<uint32_t>(j) + 0x7f4a7c15u));
      }
    }
  }
  if (sig_out) {
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      h1 = min(h1, __shfl_xor_sync(FULL, h1, o));
      h2 = min(h2, __shfl_xor_sync(FULL, h2, o));
    }
  }
  if (lane == 0) {
    count[bh * Nb + i] = __popcll(kept);
    if (brow) {
      brow[0] = static_cast<uint32_t>(kept);
      if (Nb > 32) brow[1] = static_cast<uint32_t>(kept >> 32);
    }
    if (sig_out)
      *sig_out = (static_cast<unsigned long long>(h1) << 32) | (static_cast<unsigned long long>(h2 & 0xffffu) << 16) |
                 static_cast<unsigned long long>(i);
  }
}

// Selection of one row by one warp (phase 2 of the score kernels): e_j = exp(L_j -
// max) in place of the scores, the cut-off e* by an IEEE bit-pattern search (a
// bisection, or 8-way with kEightWay), then the mask row, the ascending kept list,
// count[bh*Nb + i], the MinHash sort key of the kept set (*sig_out) and its bitset
// (brow, ceil(Nb/32) words) for the pairing. sig_out and brow may be null.
// One lane's part of sum{e_j : bits(e_j) >= key} over a row of non-negative values:
// the lane's elements j = lane + 32 t go to four partial sums by t mod 4 (so four
// independent shared-memory loads and additions are in flight instead of one
// chain), combined as (p0 + p1) + (p2 + p3). Every such sum of a row is formed in
// this same order, with +0 for the elements below key, so sums over nested sets
// are ordered like the sets (rounded addition of non-negative terms is monotone).
static __device__ __forceinline__ float lane_sum_ge(const float* row, int Nb, int lane, uint32_t key) {
  float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
  int j = lane;
  for (; j + 96 < Nb; j += 128) {
    const float e0 = row[j], e1 = row[j + 32], e2 = row[j + 64], e3 = row[j + 96];
    p0 += (__float_as_uint(e0) >= key) ? e0 : 0.f;
    p1 += (__float_as_uint(e1) >= key) ? e1 : 0.f;
    p2 += (__float_as_uint(e2) >= key) ? e2 : 0.f;
    p3 += (__float_as_uint(e3) >= key) ? e3 : 0.f;
  }
  if (j < Nb) p0 += (__float_as_uint(row[j]) >= key) ? row[j] : 0.f;
  if (j + 32 < Nb) p1 += (__float_as_uint(row[j + 32]) >= key) ? row[j + 32] : 0.f;
  if (j + 64 < Nb) p2 += (__float_as_uint(row[j + 64]) >= key) ? row[j + 64] : 0.f;
  return (p0 + p1) + (p2 + p3);
}

// lane_sum_ge, plus how many of the lane's elements have bits >= key.
static __device__ __forceinline__ float lane_sum_count_ge(const float* row, int Nb, int lane, uint32_t key, int& n) {
  float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
  int n0 = 0, n1 = 0, n2 = 0, n3 = 0;
  int j = lane;
  for (; j + 96 < Nb; j += 128) {
    const float e0 = row[j], e1 = row[j + 32], e2 = row[j + 64], e3 = row[j + 96];
    const bool g0 = __float_as_uint(e0) >= key, g1 = __float_as_uint(e1) >= key;
    const bool g2 = __float_as_uint(e2) >= key, g3 = __float_as_uint(e3) >= key;
    p0 += g0 ? e0 : 0.f;
    p1 += g1 ? e1 : 0.f;
    p2 += g2 ? e2 : 0.f;
    p3 += g3 ? e3 : 0.f;
    n0 += g0;
    n1 += g1;
    n2 += g2;
    n3 += g3;
  }
  if (j < Nb && __float_as_uint(row[j]) >= key) {
    p0 += row[j];
    ++n0;
  }
  if (j + 32 < Nb && __float_as_uint(row[j + 32]) >= key) {
    p1 += row[j + 32];
    ++n1;
  }
  if (j + 64 < Nb && __float_as_uint(row[j + 64]) >= key) {
    p2 += row[j + 64];
    ++n2;
  }
  n = (n0 + n1) + (n2 + n3);
  return (p0 + p1) + (p2 + p3);
}

template <bool kEightWay>
static __device__ __forceinline__ void select_row(float* row, int Nb, int i, long long bh, float tau, int lane,
                                                  uint8_t* __restrict__ mask, int* __restrict__ count,
                                                  int* __restrict__ idx, unsigned long long* sig_out,
                                                  uint32_t* brow) {
  const unsigned FULL = 0xffffffffu;
  const float LOG2E = 1.4426950408889634f;
  float m = -INFINITY;
  {
    float m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
    int j = lane;
    for (; j + 96 < Nb; j += 128) {
      m = fmaxf(m, row[j]);
      m1 = fmaxf(m1, row[j + 32]);
      m2 = fmaxf(m2, row[j + 64]);
      m3 = fmaxf(m3, row[j + 96]);
    }
    for (; j < Nb; j += 32) m = fmaxf(m, row[j]);
    m = fmaxf(fmaxf(m, m1), fmaxf(m2, m3));
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, o));
  // e_j in place; the row max maps to exactly 1.
  float tot = 0.f;
  uint32_t kmax = 0;
  if constexpr (kEightWay) {
    for (int j = lane; j < Nb; j += 32) {
      const float e = ex2((row[j] - m) * LOG2E);
      row[j] = e;
      tot += e;
      kmax = max(kmax, __float_as_uint(e));
    }
  } else {
    uint32_t k1 = 0, k2 = 0, k3 = 0;
    int j = lane;
    for (; j + 96 < Nb; j += 128) {
      const float e0 = ex2((row[j] - m) * LOG2E), e1 = ex2((row[j + 32] - m) * LOG2E);
      const float e2 = ex2((row[j + 64] - m) * LOG2E), e3 = ex2((row[j + 96] - m) * LOG2E);
      row[j] = e0;
      row[j + 32] = e1;
      row[j + 64] = e2;
      row[j + 96] = e3;
      kmax = max(kmax, __float_as_uint(e0));
      k1 = max(k1, __float_as_uint(e1));
      k2 = max(k2, __float_as_uint(e2));
      k3 = max(k3, __float_as_uint(e3));
    }
    for (; j < Nb; j += 32) {
      const float e = ex2((row[j] - m) * LOG2E);
      row[j] = e;
      kmax = max(kmax, __float_as_uint(e));
    }
    kmax = max(max(kmax, k1), max(k2, k3));
    __syncwarp();
    tot = lane_sum_ge(row, Nb, lane, 0u);          // the total, formed like every probe sum
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    tot += __shfl_xor_sync(FULL, tot, o);
    kmax = max(kmax, __shfl_xor_sync(FULL, kmax, o));
  }
  __syncwarp();
  uint32_t K;          // key (bit pattern) of the cut-off value e*
  int need_ties;       // how many ties at e* are kept (lowest indices first)
  if (tau >= 1.f) {
    K = 1u;            // every block with e_j > 0 (finite score) is kept
    need_ties = 0x7fffffff;
  } else {
    const float T = tau * tot;
    uint32_t lo = 0u, hi = kmax + 1u;   // S(lo) >= T > S(hi)
    // bisection only: the numbers of elements with bits >= lo and >= hi, and S(hi).
    // Once exactly one element lies in [lo, hi), S is constant on [lo, its bits]
    // and on (its bits, hi], so its bits are the largest key with S >= T, the key
    // the search would end on: it stops there.
    int c_lo = Nb, c_hi = 0;
    float s_hi = 0.f;
    bool single = false;
    while (hi - lo > 1u) {
      if constexpr (kEightWay) {
        // 7 probes split [lo, hi) into 8 parts; the last one is above lo once hi - lo >= 2
        const uint32_t span = hi - lo;
        uint32_t pr[7];
        float ps[7];
#pragma unroll
        for (int t = 0; t < 7; ++t) {
          pr[t] = lo + static_cast<uint32_t>((static_cast<unsigned long long>(span) * (t + 1)) >> 3);
          ps[t] = 0.f;
        }
        for (int j = lane; j < Nb; j += 32) {
          const float e = row[j];
          const uint32_t u = __float_as_uint(e);
#pragma unroll
          for (int t = 0; t < 7; ++t) ps[t] += (u >= pr[t]) ? e : 0.f;
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
#pragma unroll
          for (int t = 0; t < 7; ++t) ps[t] += __shfl_xor_sync(FULL, ps[t], o);
        }
        uint32_t nlo = lo, nhi = hi;
#pragma unroll
        for (int t = 0; t < 7; ++t) {
          if (ps[t] >= T) nlo = max(nlo, pr[t]);
          else nhi = min(nhi, pr[t]);
        }
        lo = nlo;
        hi = nhi;
      } else {
        if (c_lo - c_hi == 1) {
          single = true;
          break;
        }
        const uint32_t mid = lo + ((hi - lo) >> 1);
        int c;
        float s = lane_sum_count_ge(row, Nb, lane, mid, c);
#pragma unroll
        for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(FULL, s, o);
        c = __reduce_add_sync(FULL, c);
        if (s >= T) {
          lo = mid;
          c_lo = c;
        } else {
          hi = mid;
          c_hi = c;
          s_hi = s;
        }
      }
    }
    K = lo;
    float sgt = 0.f;
    int nties = 0;
    if (single) {
      // the one element in [lo, hi): its bits are the cut-off; S(hi) was formed like
      // every probe, over the elements above it
      uint32_t u = 0u;
      for (int j = lane; j < Nb; j += 32) {
        const uint32_t kj = __float_as_uint(row[j]);
        if (kj >= lo && kj < hi) u = kj;
      }
      K = __reduce_max_sync(FULL, u);
      sgt = s_hi;
      nties = 1;
    } else if constexpr (kEightWay) {
      for (int j = lane; j < Nb; j += 32) {
        const uint32_t kj = __float_as_uint(row[j]);
        sgt += (kj > K) ? row[j] : 0.f;
        nties += (kj == K);
      }
    } else {
      sgt = lane_sum_ge(row, Nb, lane, K + 1u);     // the values above e*, formed like the probes
      int n1 = 0, n2 = 0, n3 = 0;
      int j = lane;
      for (; j + 96 < Nb; j += 128) {
        nties += __float_as_uint(row[j]) == K;
        n1 += __float_as_uint(row[j + 32]) == K;
        n2 += __float_as_uint(row[j + 64]) == K;
        n3 += __float_as_uint(row[j + 96]) == K;
      }
      for (; j < Nb; j += 32) nties += __float_as_uint(row[j]) == K;
      nties += (n1 + n2) + n3;
    }
    if (!single) {   // the lanes' parts (the single case has the totals already)
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        sgt += __shfl_xor_sync(FULL, sgt, o);
        nties += __shfl_xor_sync(FULL, nties, o);
      }
    }
    const float eK = __uint_as_float(K);
    float acc = sgt;
    need_ties = 0;
    do {
      acc += eK;
      ++need_ties;
    } while (acc < T && need_ties < nties);
  }
  // emit mask, ascending idx, count
  uint8_t* mrow = mask + (bh * Nb + i) * static_cast<long long>(Nb);
  int* irow = idx ? idx + (bh * Nb + i) * static_cast<long long>(Nb) : nullptr;
  uint32_t s1 = 0xffffffffu, s2 = 0xffffffffu;  // MinHash signatures of the kept set
  int kept = 0, ties_seen = 0;
  for (int jb = 0; jb < Nb; jb += 32) {
    const int j = jb + lane;
    uint32_t kj = 0u;
    if (j < Nb) kj = __float_as_uint(row[j]);
    const bool tie = (j < Nb) && (kj == K);
    const unsigned tb = __ballot_sync(FULL, tie);
    const int my_tie_rank = ties_seen + __popc(tb & ((1u << lane) - 1u));
    const bool keep = (j < Nb) && (kj > K || (tie && my_tie_rank < need_ties));
    ties_seen += __popc(tb);
    const unsigned kb = __ballot_sync(FULL, keep);
    if (j < Nb) mrow[j] = keep ? 1 : 0;
    if (irow && keep) irow[kept + __popc(kb & ((1u << lane) - 1u))] = j;
    if (brow && lane == 0) brow[jb >> 5] = kb;
    if (keep) {
      s1 = min(s1, mix32(static_cast<uint32_t>(j) ^ 0x9e3779b9u));
      s2 = min(s2, mix32(static_cast<uint32_t>(j) + 0x7f4a7c15u));
    }
    kept += __popc(kb);
  }
  if (sig_out) {
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      s1 = min(s1, __shfl_xor_sync(FULL, s1, o));
      s2 = min(s2, __shfl_xor_sync(FULL, s2, o));
    }
  }
  if (lane == 0) {
    count[bh * Nb + i] = kept;
    if (sig_out)
      *sig_out = (static_cast<unsigned long long>(s1) << 32) | (static_cast<unsigned long long>(s2 & 0xffffu) << 16) |
                 static_cast<unsigned long long>(i);
  }
}

// ----------------------------------------------------------------------------
// Pooled scores. One CTA = a 128 x 128 tile of
//   L[i][j] = scale * <Qp_i, Kp_j>   (-inf for causal j > i)
// of one head: query blocks 128 rt .. of strip (bh, rt), key blocks 128 ct ...
// Every L[i][j] is one fp32 FMA chain over k = 0 .. D-1 in order, then the scale:
// fp32 accumulation matters here, since the kept set near tau moves with the
// scores' rounding (tcgen05 kind::tf32 with an exact three-way split of the
// operands was measured at about ten times the error of these chains: its fp32
// accumulation is coarser). With kT = 128, thread t (of 256) owns the 8 x 8
// outputs rows 8 (t / 16) .., columns 8 (t % 16) ..; heads of at most 64 blocks take
// kT = 64 tiles (4 x 4 outputs per thread), which gives the same chains. The
// operands pass through shared memory transposed (k-major) in 16-k slices, the next
// slice loading into registers while the current one is used. The tile is stored
// into the strip buffer scores[blockIdx.y][row][j] (row stride score_ld(Nb)). Grid
// (ceil(Nb/kT) column tiles, strips of the batch), 256 threads.
template <int D, int kT = 128>
__global__ void __launch_bounds__(256, 2) pooled_scores_kernel(const float* __restrict__ Qp,
                                                               const float* __restrict__ Kp, int Nb, float scale,
                                                               int causal, int strip0, float* __restrict__ scores) {
  static_assert(kT == 128 || kT == 64, "tile of 128 or 64 blocks");
  constexpr int kK = 16;                       // k per slice
  constexpr int kO = kT / 16;                  // outputs per thread along each side
  constexpr int kV = kT / 64;                  // float4 loads per operand and slice per thread
  __shared__ __align__(16) float As[2][kK][kT];
  __shared__ __align__(16) float Bs[2][kK][kT];
  const int t = threadIdx.x, tx = t & 15, ty = t >> 4;
  const int nrt = (Nb + 127) / 128;
  const int strip = strip0 + static_cast<int>(blockIdx.y);
  const int bh = strip / nrt, rt = strip - bh * nrt, ct = static_cast<int>(blockIdx.x);
  // kT = 64 serves heads of at most 64 blocks: one row tile (rt = 0) and one column tile
  const float* qa = Qp + (static_cast<long long>(bh) * Nb + 128 * rt) * D;
  const float* kb = Kp + (static_cast<long long>(bh) * Nb + kT * ct) * D;
  const int nq = min(kT, Nb - 128 * rt), nk = min(kT, Nb - kT * ct);
  // loads of a slice: thread t reads row t / (256 / kT) of both operands, kV float4s
  // of k from 4 kV (t % (256 / kT)); zeros past the head's last block
  const int lr = t / (256 / kT), lk = (t % (256 / kT)) * 4 * kV;
  float4 ra[kV], rb[kV];
  auto fetch = [&](int k0) {
#pragma unroll
    for (int u = 0; u < kV; ++u) {
      ra[u] = lr < nq ? __ldg(reinterpret_cast<const float4*>(qa + static_cast<long long>(lr) * D + k0 + lk) + u)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
      rb[u] = lr < nk ? __ldg(reinterpret_cast<const float4*>(kb + static_cast<long long>(lr) * D + k0 + lk) + u)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  auto stash = [&](int buf) {                  // transposed: [k][row]
#pragma unroll
    for (int u = 0; u < kV; ++u) {
      const float a4[4] = {ra[u].x, ra[u].y, ra[u].z, ra[u].w};
      const float b4[4] = {rb[u].x, rb[u].y, rb[u].z, rb[u].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        As[buf][lk + 4 * u + e][lr] = a4[e];
        Bs[buf][lk + 4 * u + e][lr] = b4[e];
      }
    }
  };
  float acc[kO][kO];
#pragma unroll
  for (int r = 0; r < kO; ++r)
#pragma unroll
    for (int c = 0; c < kO; ++c) acc[r][c] = 0.f;
  fetch(0);
  stash(0);
  __syncthreads();
  for (int s = 0; s < D / kK; ++s) {
    const int buf = s & 1;
    if (s + 1 < D / kK) fetch((s + 1) * kK);   // in flight during this slice's FMAs
#pragma unroll
    for (int kk = 0; kk < kK; ++kk) {
      float av[kO], bv[kO];
#pragma unroll
      for (int h = 0; h < kO / 4; ++h) {
        const float4 a = *reinterpret_cast<const float4*>(&As[buf][kk][kO * ty + 4 * h]);
        const float4 b = *reinterpret_cast<const float4*>(&Bs[buf][kk][kO * tx + 4 * h]);
        av[4 * h] = a.x;
        av[4 * h + 1] = a.y;
        av[4 * h + 2] = a.z;
        av[4 * h + 3] = a.w;
        bv[4 * h] = b.x;
        bv[4 * h + 1] = b.y;
        bv[4 * h + 2] = b.z;
        bv[4 * h + 3] = b.w;
      }
#pragma unroll
      for (int r = 0; r < kO; ++r)
#pragma unroll
        for (int c = 0; c < kO; ++c) acc[r][c] = fmaf(av[r], bv[c], acc[r][c]);
    }
    if (s + 1 < D / kK) {
      stash(buf ^ 1);                          // the other buffer was last read a slice ago
      __syncthreads();
    }
  }
  const int ld = score_ld(Nb);
#pragma unroll
  for (int r = 0; r < kO; ++r) {
    const int row = kO * ty + r, i = 128 * rt + row;
    if (i >= Nb) break;
    const int j0 = kT * ct + kO * tx;
    float* dst = scores + (static_cast<long long>(blockIdx.y) * 128 + row) * ld + j0;
    float v[kO];
#pragma unroll
    for (int c = 0; c < kO; ++c) {
      v[c] = acc[r][c] * scale;
      if (causal && j0 + c > i) v[c] = -INFINITY;
    }
    if (j0 + kO <= Nb) {
#pragma unroll
      for (int h = 0; h < kO / 4; ++h)
        reinterpret_cast<float4*>(dst)[h] = make_float4(v[4 * h], v[4 * h + 1], v[4 * h + 2], v[4 * h + 3]);
    } else {
#pragma unroll
      for (int c = 0; c < kO; ++c)
        if (j0 + c < Nb) dst[c] = v[c];
    }
  }
}

// Selection of 4 query blocks per CTA from the score strips, one warp per row
// (phase 2 below): rows 4 blockIdx.x .. of strip strip0 + blockIdx.y, copied from
// the strip buffer into shared memory (the search reads a row many times). Rows
// of up to 256 blocks take the 8-way search, up to 64 the sorted prefix. Grid
// (32, strips of the batch), 128 threads, 16 score_ld(Nb) bytes of shared memory.
// tau is the recall threshold of every head, or tau_bh[b*H + h] per head when
// tau_bh is given.
//
// Selection (one warp per row): e_j = exp(L_j - max), T = tau * sum e. The kept
// set is {j : e_j > e*} plus the lowest-index ties at e* needed to reach T, where
// e* is the largest value with sum_{e_j >= e*} e_j >= T. e* is found by searching
// the IEEE bit pattern of e (monotone for non-negative floats): a bisection that
// stops once one element lies between its bounds, or for short rows an 8-way
// search (7 probes per step, about 10 steps instead of 30, where the steps'
// shuffle latency dominates). Every probe sums in the same fixed order, so the
// kept set does not depend on the search path.
template <bool kShort>
__global__ void __launch_bounds__(128) select_kernel(const float* __restrict__ scores, int Nb, int strip0, float tau,
                                                     const float* __restrict__ tau_bh, uint8_t* __restrict__ mask,
                                                     int* __restrict__ count, int* __restrict__ idx,
                                                     unsigned long long* __restrict__ sig,
                                                     uint32_t* __restrict__ bits) {
  extern __shared__ __align__(16) float Lrows[];   // [4][ld]
  const int ld = score_ld(Nb);
  const int nrt = (Nb + 127) / 128;
  const int strip = strip0 + static_cast<int>(blockIdx.y);
  const long long bh = strip / nrt;
  const int rt = strip - static_cast<int>(bh) * nrt;
  const int r0 = 4 * static_cast<int>(blockIdx.x);          // first row within the strip
  if (128 * rt + r0 >= Nb) return;
  const float4* src = reinterpret_cast<const float4*>(scores + (static_cast<long long>(blockIdx.y) * 128 + r0) * ld);
  for (int x = threadIdx.x; x < ld; x += 128) reinterpret_cast<float4*>(Lrows)[x] = src[x];   // 4 rows
  __syncthreads();
  // the head's own tau when one is given per (b, h); an invalid one (not in (0, 1])
  // is recorded in the device error word and the head keeps every block
  if (tau_bh) {
    tau = tau_bh[bh];
    if (!(tau > 0.f && tau <= 1.f)) {
      if (threadIdx.x == 0) atomicOr(&g_dev_error, DEVERR_VALUE);
      tau = 1.f;
    }
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = 128 * rt + r0 + warp;
  if (i >= Nb) return;
  uint32_t* brow = bits ? bits + (bh * Nb + i) * static_cast<long long>((Nb + 31) / 32) : nullptr;
  unsigned long long* srow = sig ? sig + bh * Nb + i : nullptr;
  if (kShort && Nb <= 64)
    select_row_sorted64(Lrows + warp * ld, Nb, i, bh, tau, lane, mask, count, idx, srow, brow);
  else
    select_row<kShort>(Lrows + warp * ld, Nb, i, bh, tau, lane, mask, count, idx, srow, brow);
}

// Dynamic shared memory of select_kernel for Nb blocks per head.
inline int select_smem_bytes(int Nb) { return 4 * score_ld(Nb) * static_cast<int>(sizeof(float)); }


// ----------------------------------------------------------------------------
// Query-tile pairing and order. A 128-row query tile holds two 64-row query
// blocks of one head and walks the union of their kept lists, so its cost is the
// union size. Adjacent blocks of a video raster often keep disjoint key blocks
// (their partners are in the neighbouring frame), so the pairs are chosen from
// the masks. Query blocks are sorted by two MinHash signatures of their kept sets
// (equal sets sort together). Then, in rounds, every unpaired block picks the
// unpaired block within kPairWindow places of it in that order whose kept set
// matches best (overlap minus symmetric difference; ties to the nearer, then the
// earlier block), and blocks that pick each other are paired; after
// kPairRounds rounds, or a round without a new pair, the rest are paired in
// order. Every block of a head is examined at once, so a round costs one pass.
// The pairs of a head are then ordered by decreasing union size (longest first).
// When the bitsets do not fit in shared
// memory and consecutive blocks of the sorted order are paired directly.
// Output: work[2*r], work[2*r+1] = global query-block ids (bh*Nb + i) of the r-th
// tile (second -1 if the head has an odd block count).
constexpr int kPairWindow = 16;
constexpr int kPairRounds = 6;
// Heads per interleaved group of the tile order: as many as have their K and V
// together within half of L2 (64 MB), at least one.
inline int order_group_heads(long long BH, int N, int D) {
  const long long kv_bytes = 2ll * N * D * 2;
  const long long g = (64ll << 20) / kv_bytes;
  return static_cast<int>(g < 1 ? 1 : (g > BH ? BH : g));
}


// In-place ascending bitonic sort of n64 (a power of two) 64-bit keys in shared memory.
static __device__ void block_bitonic_sort(unsigned long long* keys, int n64) {
  for (int k = 2; k <= n64; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int t = threadIdx.x; t < n64 / 2; t += blockDim.x) {
        const int lo = 2 * j * (t / j) + (t % j);
        const int hi = lo + j;
        const bool up = ((lo & k) == 0);
        const unsigned long long a = keys[lo], b = keys[hi];
        if ((a > b) == up) {
          keys[lo] = b;
          keys[hi] = a;
        }
      }
      __syncthreads();
    }
  }
}

// Exclusive prefix sum of v over the threads of the block (any multiple of 32
// threads up to 1024); every thread must call it. *total receives the sum.
// sbuf: 33 ints of shared memory. Without kTrailingSync the caller must pass a
// __syncthreads before sbuf is written again.
template <bool kTrailingSync = true>
static __device__ int block_exclusive_scan(int v, int* sbuf, int* total) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sbuf[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = (lane < nw) ? sbuf[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < nw) sbuf[lane] = w;            // inclusive warp totals
    if (lane == 31) sbuf[32] = w;
  }
  __syncthreads();
  const int excl = x - v + (warp > 0 ? sbuf[warp - 1] : 0);
  *total = sbuf[32];
  if (kTrailingSync) __syncthreads();         // sbuf may be reused right after
  return excl;
}

// Heads are laid out in groups of G consecutive heads (the last group may be
// smaller); within a group, tile rank r of the group's u-th head goes to position
// group_start + r * group_size + u. The CTAs running at one time then take the
// longest tiles of every head of the group first, while the group's K and V
// (chosen by the host to fit in L2) stay resident.
// Pairs and orders the query blocks of head bh (see above); called by every
// thread of the CTA. keys: shared memory for P 64-bit keys whose first Nb entries
// hold the blocks' MinHash sort keys; bits_rows: the kept-set bitsets, row-major
// [Nb][ceil(Nb/32)], in global or shared memory; psm: the rest of the shared
// memory (pair_order_smem_bytes minus the keys). BH heads in all.
static __device__ void pair_and_order(unsigned long long* keys, const uint32_t* bits_rows,
                                      const int* __restrict__ count, int Nb, int Tq, int G, long long bh,
                                      long long BH, int* __restrict__ work, unsigned char* psm,
                                      uint32_t* bits_by_pos) {
  const int P = 1 << (32 - __clz(max(Nb, 2) - 1));   // next power of two >= Nb
  const int P2 = 1 << (32 - __clz(max(Tq, 2) - 1));
  // bitsets by sorted position: in shared memory when they fit, else in the global
  // bits_by_pos region ([W][Nb] of this head)
  const bool in_smem = pair_bits_in_smem(Nb);
  const bool match = in_smem || bits_by_pos != nullptr;
  const int W = (Nb + 31) / 32;                       // bitset words per row
  unsigned long long* keys2 = reinterpret_cast<unsigned long long*>(psm);      // [P2]
  int* pa = reinterpret_cast<int*>(keys2 + P2);                                  // [Tq]
  int* pb = pa + Tq;                                                             // [Tq]
  int* order = pb + Tq;                                                          // [Nb] position -> block
  int* alive = order + Nb;                                                       // [Nb] unpaired positions, ascending
  int* best = alive + Nb;                                                        // [Nb] pick of a position
  int* partner = best + Nb;                                                      // [Nb] -1 while unpaired
  int* sbuf = partner + Nb;                                                      // [34] scan scratch
  uint32_t* bitsT = in_smem ? reinterpret_cast<uint32_t*>(sbuf + 34)  // [W][Nb] by position
                           : bits_by_pos;
  const int* cnt = count + bh * Nb;

  // 1. sort the MinHash keys
  for (int i = threadIdx.x; i < Nb; i += blockDim.x) partner[i] = -1;
  for (int i = Nb + threadIdx.x; i < P; i += blockDim.x) keys[i] = ~0ull;
  __syncthreads();
  if (P <= 64) {
    if (threadIdx.x < 32) warp_sort_keys(keys, P, threadIdx.x);
    __syncthreads();
  } else {
    block_bitonic_sort(keys, P);
  }
  for (int p = threadIdx.x; p < Nb; p += blockDim.x) {
    order[p] = static_cast<int>(keys[p] & 0xffffu);
    alive[p] = p;
  }
  __syncthreads();

  // 2. pairs (as sorted positions in pa/pb) and their costs (union sizes, or count
  //    sums without bitsets)
  if (match) {
    // kept-set bitsets, word-major by sorted position: neighbouring candidates are
    // neighbouring addresses (shared memory, or this head's global region; the
    // barrier makes the CTA's global writes visible to its own later reads)
    for (int x = threadIdx.x; x < Nb * W; x += blockDim.x) {
      const int p = x / W, w = x - p * W;
      bitsT[static_cast<long long>(w) * Nb + p] = bits_rows[static_cast<long long>(order[p]) * W + w];
    }
    __syncthreads();
    // one warp per alive position, one lane per candidate (the 16 alive positions
    // on each side)
    int na = Nb;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    for (int round = 0; round < kPairRounds; ++round) {
      const int t = threadIdx.x;
      for (int a = warp; a < na; a += nwarps) {
        const int me = alive[a];
        const int d = lane < kPairWindow ? lane - kPairWindow : lane - kPairWindow + 1;   // -16..-1, 1..16
        const int q = a + d;
        const bool ok = q >= 0 && q < na;
        const int cpos = ok ? alive[q] : -1;
        int sc = INT_MIN;
        if (ok) {
          sc = 0;
#pragma unroll 4
          for (int w = 0; w < W; ++w) {
            const uint32_t x = bitsT[static_cast<long long>(w) * Nb + me];
            const uint32_t y = bitsT[static_cast<long long>(w) * Nb + cpos];
            sc += __popc(x & y) - __popc(x ^ y);
          }
        }
        // warp argmax of (score, -distance, -offset): ties to the nearer, then the
        // earlier. One 64-bit key per lane (score + 4096 in the high word, distinct
        // offsets below it, the candidate in the low bits); 0 = no candidate.
        unsigned long long kb = 0ull;
        if (ok)
          kb = (static_cast<unsigned long long>(sc + 4096) << 32) |
               (static_cast<unsigned long long>(16 - abs(d)) << 24) |
               (static_cast<unsigned long long>(16 - d) << 16) | static_cast<unsigned long long>(cpos);
#pragma unroll
        for (int o = 16; o; o >>= 1) kb = max(kb, __shfl_xor_sync(0xffffffffu, kb, o));
        if (lane == 0) best[me] = kb ? static_cast<int>(kb & 0xffffu) : -1;
      }
      __syncthreads();
      // mutual picks pair up, and the unpaired positions are compacted in place,
      // blockDim.x positions at a time: thread t alone reads and writes
      // partner[alive[base + t]], and an entry only ever moves to a lower index, so
      // a chunk's writes never reach entries still to be read
      int nna = 0;
      for (int base = 0; base < na; base += blockDim.x) {
        const int me = (base + t < na) ? alive[base + t] : -1;
        if (me >= 0) {
          const int c = best[me];
          if (c >= 0 && best[c] == me) partner[me] = c;
        }
        const bool stay = me >= 0 && partner[me] < 0;
        int tot = 0;
        const int at = block_exclusive_scan(stay ? 1 : 0, sbuf, &tot);   // its barriers order reads and writes
        if (stay) alive[nna + at] = me;
        nna += tot;
      }
      __syncthreads();
      if (nna == na) break;
      na = nna;
    }
    // matched pairs, numbered by the position of their earlier block, then the
    // unpaired blocks two by two in order
    int nm = 0;
    for (int p0 = 0; p0 < Nb; p0 += blockDim.x) {
      const int p = p0 + threadIdx.x;
      const int c = (p < Nb) ? partner[p] : -1;
      const bool first = c > p;
      int tot = 0;
      const int j = nm + block_exclusive_scan(first ? 1 : 0, sbuf, &tot);
      if (first) {
        pa[j] = p;
        pb[j] = c;
      }
      nm += tot;
    }
    for (int q = 2 * threadIdx.x; q < na; q += 2 * blockDim.x) {
      pa[nm + q / 2] = alive[q];
      pb[nm + q / 2] = (q + 1 < na) ? alive[q + 1] : -1;
    }
    __syncthreads();
    for (int p = threadIdx.x; p < Tq; p += blockDim.x) {
      const int a = pa[p], b = pb[p];
      int c = 0;
      for (int w = 0; w < W; ++w)
        c += __popc(bitsT[static_cast<long long>(w) * Nb + a] |
                    (b >= 0 ? bitsT[static_cast<long long>(w) * Nb + b] : 0u));
      keys2[p] = (static_cast<unsigned long long>(0xffffffu - static_cast<uint32_t>(c)) << 32) |
                 static_cast<unsigned long long>(p);
    }
  } else {
    for (int p = threadIdx.x; p < Tq; p += blockDim.x) {
      const int a = 2 * p, b = (2 * p + 1 < Nb) ? 2 * p + 1 : -1;
      pa[p] = a;
      pb[p] = b;
      const int c = cnt[order[a]] + (b >= 0 ? cnt[order[b]] : 0);
      keys2[p] = (static_cast<unsigned long long>(0xffffffu - static_cast<uint32_t>(c)) << 32) |
                 static_cast<unsigned long long>(p);
    }
  }
  __syncthreads();
  for (int p = Tq + threadIdx.x; p < P2; p += blockDim.x) keys2[p] = ~0ull;
  __syncthreads();
  // 3. longest first, then write the global query-block ids
  if (P2 <= 64) {
    if (threadIdx.x < 32) warp_sort_keys(keys2, P2, threadIdx.x);
    __syncthreads();
  } else {
    block_bitonic_sort(keys2, P2);
  }
  const long long g0 = (bh / G) * G;                                  // first head of the group
  const long long gsize = min(static_cast<long long>(G), BH - g0);
  const long long u = bh - g0;
  for (int r = threadIdx.x; r < Tq; r += blockDim.x) {
    const int p = static_cast<int>(keys2[r] & 0xffffffffu);
    const int a = order[pa[p]], b = pb[p] >= 0 ? order[pb[p]] : -1;
    const long long pos = g0 * Tq + static_cast<long long>(r) * gsize + u;
    work[2 * pos] = static_cast<int>(bh * Nb + a);
    work[2 * pos + 1] = b >= 0 ? static_cast<int>(bh * Nb + b) : -1;
  }
}

// One CTA per head: MinHash keys and bitsets from the selection kernel. bitsT_g
// (the plan workspace's bitsT region, [BH][W][Nb]) is needed above
// blocks per head whose bitsets do not fit in shared memory; without it such heads
// pair consecutive blocks
// of the sorted order.
static __global__ void __launch_bounds__(1024) pair_order_kernel(const unsigned long long* __restrict__ sig,
                                                                 const uint32_t* __restrict__ bits_g,
                                                                 const int* __restrict__ count, int Nb,
                                                                 int Tq, int G, int* __restrict__ work,
                                                                 uint32_t* __restrict__ bitsT_g) {
  extern __shared__ __align__(16) unsigned char psm[];
  const int P = 1 << (32 - __clz(max(Nb, 2) - 1));
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(psm);
  const long long bh = blockIdx.x;
  const long long words = static_cast<long long>(Nb) * ((Nb + 31) / 32);
  for (int i = threadIdx.x; i < Nb; i += blockDim.x) keys[i] = sig[bh * Nb + i];
  pair_and_order(keys, bits_g + bh * words, count, Nb, Tq, G, bh, gridDim.x, work,
                 psm + P * sizeof(unsigned long long),
                 (!pair_bits_in_smem(Nb) && bitsT_g != nullptr) ? bitsT_g + bh * words : nullptr);
}

// Shared memory of pair_order_kernel for Nb blocks per head.
inline int pair_order_smem_bytes(int Nb) {
  int bytes = pair_base_smem_bytes(Nb);
  if (pair_bits_in_smem(Nb)) bytes += Nb * ((Nb + 31) / 32) * 4;
  return bytes;
}

// Threads of pair_order_kernel: a warp per query block in the matching rounds,
// and at least one thread per block of the alive list.
inline int pair_order_threads(int /*Nb*/) { return 1024; }

}  // namespace sa

// Interaction clustering: k-means of one side's tokens (queries or keys) under
// the other side's Gram metric, and the token reordering that follows it.
//
// The iCATS abstract clusters query and key tokens by their dot-product
// interaction rather than by feature similarity, and reduces the objective to a
// quadratic form. Replacing a token x by a centroid c changes its score with
// every token y of the other side by (x - c).y; the sum of the squares is
// (x - c)^T G (x - c) with G = sum_y y y^T (gram_tc_kernel and gram_reduce_kernel,
// on the tensor cores with fp32 accumulation). Dropping the term x^T G x, which is
// the same for every centroid, the nearest centroid is the argmin over c of
// c^T G c - 2 x . (G c). So each Lloyd iteration is: w_c = G c and b_c = c . w_c
// per centroid (cluster_prep_kernel), an argmin over all centroids per token (a
// tensor-core product of the bf16 tokens with the w_c split into bf16 high and
// low parts that keeps each token's four best, cluster_assign_tc_kernel, then
// their exact fp32 scores, cluster_rescore_kernel), and the mean of each
// cluster's tokens (cluster_centroid_kernel). The clusters start at the 64-token
// block means (the pooling kernel), so zero iterations reproduce the plain blocks.
//
// The reordering is a stable sort of the tokens by cluster: a per-head
// exclusive scan of the cluster sizes gives each cluster's first position, and
// each cluster's tokens follow in token order. Clusters are packed back to back,
// so the tail of one shares a 64-token block with the head of the next (the
// abstract's tail merging, with no padding at all).
//
// Each iteration: cluster_prep_kernel (w_c, b_c, their bf16 operand rows; clears
// the sizes), cluster_assign_tc_kernel and cluster_rescore_kernel (argmin; counts
// the sizes), cluster_offsets_kernel (each cluster's first position), the stable
// order (cluster_chunk_count_kernel, cluster_chunk_scan_kernel,
// cluster_order_kernel) and cluster_centroid_kernel (each cluster's mean, summed
// over its tokens in token order through the order just built; the last
// iteration skips it unless the centroids are returned). Everything is
// deterministic: every fp32 sum runs in a fixed order, the sizes are integer
// counts, and argmin ties go to the lowest cluster index.
#pragma once

#include "sa_device.cuh"

namespace sa {

// Tokens per partial Gram matrix: at most 592 CTAs over all heads (four per SM,
// one wave), at least 512 tokens each, a multiple of 32.
inline int gram_chunk(long long BH, int N) {
  const long long want_splits = BH >= 592 ? 1 : 592 / BH;
  long long chunk = (N + want_splits - 1) / want_splits;
  chunk = chunk < 512 ? 512 : chunk;
  return static_cast<int>((chunk + 31) / 32 * 32);
}

// Tokens per chunk of the stable order: at most 64 chunks per head, at least
// 1024 tokens each, a multiple of 32.
inline int order_chunk(int N) {
  int n = (N + 1023) / 1024;
  n = n > 64 ? 64 : n;
  const int L = (N + n - 1) / n;
  return (L + 31) / 32 * 32;
}

// Byte offsets of the clustering workspace: partial Gram matrices, the Gram
// matrix, centroids, w_c = G c, b_c, cluster sizes, first positions, the
// assignment (when the caller does not want it back), the tensor-core operand
// rows of the centroids (bf16 [B*H][C][2D + 64], see cluster_prep_kernel), four
// candidate clusters per token, and per (chunk, cluster) token counts, then
// first positions, of the stable order.
struct ClusterWorkspace {
  size_t gpart, gram, cent, w, b, cnt, off, assign, w16, cand, chunks, total;
  int splits, chunk, C, order_len, order_chunks;
};
inline ClusterWorkspace cluster_workspace(long long BH, int N, int D) {
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  ClusterWorkspace w;
  w.C = (N + kBlock - 1) / kBlock;
  w.chunk = gram_chunk(BH, N);
  w.splits = (N + w.chunk - 1) / w.chunk;
  w.order_len = order_chunk(N);
  w.order_chunks = (N + w.order_len - 1) / w.order_len;
  const size_t dd = static_cast<size_t>(D) * D * sizeof(float);
  const size_t cd = static_cast<size_t>(BH) * w.C * D * sizeof(float);
  const size_t c4 = static_cast<size_t>(BH) * w.C * sizeof(int);
  w.gpart = 0;
  w.gram = al(static_cast<size_t>(BH) * w.splits * dd);
  w.cent = w.gram + al(static_cast<size_t>(BH) * dd);
  w.w = w.cent + al(cd);
  w.b = w.w + al(cd);
  w.cnt = w.b + al(c4);
  w.off = w.cnt + al(c4);
  w.assign = w.off + al(c4);
  w.w16 = w.assign + al(static_cast<size_t>(BH) * N * sizeof(int));
  w.cand = w.w16 + al(static_cast<size_t>(BH) * w.C * (2 * D + 64) * 2);
  w.chunks = w.cand + al(static_cast<size_t>(BH) * N * 4 * sizeof(int));
  w.total = w.chunks + al(static_cast<size_t>(BH) * w.order_chunks * w.C * sizeof(int));
  return w;
}

// Partial Gram matrix sum_t y_t y_t^T over one chunk of `chunk` tokens of one
// head on the tensor cores. Grid (chunks, B*H), 128 threads. Per 64-token tile the
// threads write Y^T (feature rows, token columns: the token is the contraction
// index) into a 128-byte-swizzled K-major shared tile, 2 bytes at a time (lane =
// token, so a warp's stores fall in 16 distinct banks); the one tile is both
// operands of four K = 16 steps of tcgen05.mma (M = 128 feature rows, N = D
// feature columns, fp32 accumulate in TMEM across the whole chunk). Rows D..127 of
// the tile stay zero when D = 64. Two tiles alternate: a tile is rewritten once
// the MMAs that read it two tiles earlier have completed, and the next tile's
// loads are in flight while the current one is written. The accumulator goes to
// part[bh][split] (fp32 D x D).
template <int D>
struct GramTcCfg {
  static constexpr int kTok = 64;                      // tokens per tile (one 128-byte row)
  static constexpr int kTileBytes = 128 * 128;         // 128 feature rows x 64 tokens, bf16
  static constexpr int kSmemBytes = 2 * kTileBytes + 1024 + 64;
  static constexpr uint32_t kTmemCols = D;             // N = D fp32 columns
  static constexpr uint32_t kIdesc = idesc_bf16_f32(128, D, false);
};

template <int D>
__global__ void __launch_bounds__(128, 4) gram_tc_kernel(const __nv_bfloat16* __restrict__ Y, float* __restrict__ part,
                                                      int N, int splits, int chunk) {
  using Cf = GramTcCfg<D>;
  constexpr int kOct = D / 8;                          // 16-byte feature groups of a token
  constexpr int kUnits = 2 * kOct;                     // (32-token half, feature group) pairs per tile
  extern __shared__ uint8_t gsm_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gsm_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* done = reinterpret_cast<uint64_t*>(base + 2 * Cf::kTileBytes);   // [2]: MMAs of a tile completed
  volatile int* abort_flag = reinterpret_cast<volatile int*>(done + 2);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(done + 3);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long bh = blockIdx.y;
  const int s = blockIdx.x;
  const int t0 = s * chunk, t1 = min(N, t0 + chunk);
  const int ntile = t1 > t0 ? (t1 - t0 + Cf::kTok - 1) / Cf::kTok : 0;

  for (int x = threadIdx.x; x < 2 * Cf::kTileBytes / 16; x += 128)
    reinterpret_cast<uint4*>(base)[x] = make_uint4(0u, 0u, 0u, 0u);
  if (threadIdx.x == 0) {
    mbar_init(&done[0], 1);
    mbar_init(&done[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(tmem_holder, Cf::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const __nv_bfloat16* src = Y + bh * static_cast<long long>(N) * D;

  // this warp's units of a tile: 32 consecutive tokens (one per lane) x 8 features
  auto load_tile = [&](int j, uint4 (&u)[kUnits / 4]) {
    const int tt = t0 + j * Cf::kTok;
#pragma unroll
    for (int q = 0; q < kUnits / 4; ++q) {
      const int unit = warp + 4 * q, half = unit / kOct, oct = unit % kOct;
      const int t = tt + 32 * half + lane;
      u[q] = (j < ntile && t < t1) ? __ldg(reinterpret_cast<const uint4*>(src + static_cast<long long>(t) * D) + oct)
                                    : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  bool ok = true;
  uint4 u[kUnits / 4];
  load_tile(0, u);
  for (int j = 0; j < ntile; ++j) {
    const int buf = j & 1;
    uint4 un[kUnits / 4];
    load_tile(j + 1, un);                            // in flight while tile j is written
    if (j >= 2) {   // the MMAs of tile j - 2 (the last readers of this buffer) are done
      const bool w = mbar_wait(&done[buf], static_cast<uint32_t>((j - 2) >> 1) & 1u, abort_flag);
      if (!__syncthreads_and(w)) {
        ok = false;
        break;
      }
      tc_fence_after();
    }
    uint8_t* tile = base + buf * Cf::kTileBytes;
#pragma unroll
    for (int q = 0; q < kUnits / 4; ++q) {
      const int unit = warp + 4 * q, half = unit / kOct, oct = unit % kOct;
      const int kl = 32 * half + lane;                 // token within the tile = K index
      const uint16_t* h = reinterpret_cast<const uint16_t*>(&u[q]);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int row = 8 * oct + e;                   // feature = M (and N) index
        *reinterpret_cast<uint16_t*>(tile + row * 128 + ((((kl >> 3) ^ (row & 7))) << 4) + (kl & 7) * 2) = h[e];
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) {
      tc_fence_after();
      const uint32_t ta = smem_u32(tile);
#pragma unroll
      for (int kk = 0; kk < Cf::kTok / 16; ++kk) {
        const uint64_t d = sdesc_sw128(ta + kk * 32, 16, 1024);
        tc_mma_ss(tmem_base, d, d, Cf::kIdesc, (j > 0 || kk > 0) ? 1u : 0u);
      }
      tc_commit(&done[buf]);
    }
#pragma unroll
    for (int q = 0; q < kUnits / 4; ++q) u[q] = un[q];
  }
  // the last commit covers every MMA of the chunk
  if (ok && ntile > 0) {
    const int jl = ntile - 1;
    ok = __syncthreads_and(mbar_wait(&done[jl & 1], static_cast<uint32_t>(jl >> 1) & 1u, abort_flag));
  }
  tc_fence_after();
  float* out = part + (bh * splits + s) * static_cast<long long>(D) * D;
  const int row = warp * 32 + lane;                    // TMEM lane = feature row
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {
    float v[32];
    tmem_ld32(tmem_base + (static_cast<uint32_t>(warp * 32) << 16) + c * 32, v);
    tmem_wait_ld();
    pin32(v);
    if (row < D) {
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        // a chunk without tokens, or a wait that gave up, contributes zeros
        const bool use = ok && ntile > 0;
        *reinterpret_cast<float4*>(out + row * D + c * 32 + e) =
            make_float4(use ? v[e] : 0.f, use ? v[e + 1] : 0.f, use ? v[e + 2] : 0.f, use ? v[e + 3] : 0.f);
      }
    }
  }
  if (!ok) atomicOr(&g_dev_error, DEVERR_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cf::kTmemCols);
  }
}

// G[bh] = sum over the chunks, in chunk order. Grid (D*D/256, B*H), 256 threads.
template <int D>
__global__ void __launch_bounds__(256) gram_reduce_kernel(const float* __restrict__ part, float* __restrict__ G,
                                                          int splits) {
  const long long bh = blockIdx.y;
  const int e = blockIdx.x * 256 + threadIdx.x;
  float s = 0.f;
  for (int k = 0; k < splits; ++k) s += part[(bh * splits + k) * static_cast<long long>(D) * D + e];
  G[bh * D * D + e] = s;
}

// assign[bh, t] = t / 64 (every token in its own block's cluster) and
// cnt[bh, c] = the block's size. One thread per token.
__global__ void __launch_bounds__(256) cluster_init_assign_kernel(int* __restrict__ assign, int* __restrict__ cnt,
                                                                  int N, int C, long long total) {
  const long long x = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x;
  if (x < total) assign[x] = static_cast<int>(x % N) / kBlock;
  if (x < total / N * C) {
    const int c = static_cast<int>(x % C);
    cnt[x] = min(kBlock, N - c * kBlock);
  }
}

// w_c = G c and b_c = c . w_c for 16 centroids of one head per CTA, and their
// sizes cleared for the assignment to count. Grid
// (ceil(C/16), B*H), D threads: thread i forms component i (G is symmetric, so
// it reads column i of G as row i, and a warp reads G row by row).
//
// W16 (bf16 [B*H][C][2D + 64]) receives each centroid's tensor-core operand row
// for the assignment: v = -2 w_c as two bf16 parts, hi = bf16(v) in columns
// [0, D) and lo = bf16(v - hi) in [D, 2D) (together 16 significant bits), then
// b_c the same way (b_hi in column 2D, b_lo in 2D + 1) and zeros.
template <int D>
__global__ void __launch_bounds__(D) cluster_prep_kernel(const float* __restrict__ G, const float* __restrict__ cent,
                                                         float* __restrict__ W, float* __restrict__ bvec,
                                                         int* __restrict__ cnt, int C,
                                                         __nv_bfloat16* __restrict__ W16) {
  constexpr int kCl = 16;
  __shared__ float cs[kCl][D];
  __shared__ float red[kCl][D / 32];
  __shared__ float bsh[kCl];
  const long long bh = blockIdx.y;
  const int c0 = blockIdx.x * kCl;
  const int ncl = min(kCl, C - c0);
  const int i = threadIdx.x, lane = i & 31, warp = i >> 5;
#pragma unroll
  for (int c = 0; c < kCl; ++c) cs[c][i] = c < ncl ? cent[(bh * C + c0 + c) * D + i] : 0.f;
  __syncthreads();
  float acc[kCl];
#pragma unroll
  for (int c = 0; c < kCl; ++c) acc[c] = 0.f;
  const float* g = G + bh * D * D;
  for (int j = 0; j < D; ++j) {
    const float gji = g[j * D + i];
#pragma unroll
    for (int c = 0; c < kCl; ++c) acc[c] = fmaf(gji, cs[c][j], acc[c]);
  }
#pragma unroll
  for (int c = 0; c < kCl; ++c) {
    if (c < ncl) {
      W[(bh * C + c0 + c) * D + i] = acc[c];
      const float v = -2.f * acc[c];
      const __nv_bfloat16 hi = __float2bfloat16_rn(v);
      W16[(bh * C + c0 + c) * (2 * D + 64) + i] = hi;
      W16[(bh * C + c0 + c) * (2 * D + 64) + D + i] = __float2bfloat16_rn(v - __bfloat162float(hi));
    }
    float v = cs[c][i] * acc[c];
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[c][warp] = v;
  }
  __syncthreads();
  if (i < ncl) {
    float b = 0.f;
#pragma unroll
    for (int w = 0; w < D / 32; ++w) b += red[i][w];
    bvec[bh * C + c0 + i] = b;
    bsh[i] = b;
    cnt[bh * C + c0 + i] = 0;   // counted again by the assignment
  }
  __syncthreads();
  // the bias columns of the operand rows: b_hi, b_lo, then zeros
  for (int x = i; x < ncl * 64; x += D) {
    const int c = x >> 6, k = x & 63;
    const float b = bsh[c];
    const __nv_bfloat16 hi = __float2bfloat16_rn(b);
    __nv_bfloat16 v = __float2bfloat16_rn(0.f);
    if (k == 0) v = hi;
    if (k == 1) v = __float2bfloat16_rn(b - __bfloat162float(hi));
    W16[(bh * C + c0 + c) * (2 * D + 64) + 2 * D + k] = v;
  }
}

// ----------------------------------------------------------------------------
// Tensor-core assignment: the four nearest centroids of every token by a bf16
// product on the tensor cores, then the exact argmin among those four in fp32
// (cluster_rescore_kernel). One CTA = 256 tokens of one head, two halves of 128
// (the M = 128 of tcgen05.mma); per tile of 64 centroids
//   D_h[token][c] = x . hi_c + x . lo_c + 1 . b_hi_c + 1 . b_lo_c
// (kind::f16, fp32 accumulate in TMEM; hi + lo = -2 w_c to 16 significant bits,
// so the product is off by about 2^-17 of |x| |w_c| rather than bf16's 2^-9) with
// the tokens as the A operand in TMEM (written once from registers, so the MMAs
// read only the centroid tile from shared memory) and the centroid tile's rows
// from cluster_prep_kernel as B (TMA, one 4-D box per tile with the low part and
// the bias chunk): D / 16 K-steps of the tokens against the high part, D / 16
// against the low part, then one K-step of a block of TMEM columns whose rows
// start with two ones against the rows' bias columns. Both halves use each centroid tile, so a tile crosses L2 once per 256
// tokens. Warp 16 (one thread) issues the loads; warps 17 and 18 (one thread
// each) issue the MMAs of half 0 and half 1: a single issuing thread waits about
// as long per MMA as a 128 x 64 x 16 product takes at half the math rate, two keep
// the tensor pipe busy. Warps 0-15 are the epilogue:
// warp w reads TMEM lanes 32 (w % 4) .. (its 32 tokens) of half (w / 4) % 2 and
// the 32 columns of column half w / 8 of each tile and keeps each token's four
// smallest values with their centroids in registers; the two
// column halves merge at the end. A lane marks the values below its token's
// current fourth best in a bit mask, parks the 32 values in its own shared-memory
// row, and offers only the marked ones, so a warp pays for its busiest lane's
// entries (after the first tile a few at most) rather than for every value that
// any lane needs. Two TMEM buffers per half keep
// the tensor cores and the epilogue overlapped; a CTA visits the centroid tiles
// starting from the one that holds its tokens' first clusters (visit_tile), so
// the four best settle in the first tile. The split product still moves the
// argmin where two distances agree to about 1e-5; its four best contained the
// fp32 argmin for every token measured (inputs whose distances crowd within 1e-4
// of each other included, where bf16 alone needed sixteen), and the re-score
// restores it exactly.
template <int D>
struct ClusterTcCfg {
  static constexpr int kCh = D / 64;                   // 128-byte column chunks of a row
  static constexpr int kTok = 256;                     // tokens per CTA: two halves of 128
  static constexpr int kCt = 64;                       // centroids per tile (N of the MMA)
  static constexpr int kChunkBytes = kCt * 128;        // 8 KB: one column chunk of a tile
  static constexpr int kWStage = (2 * kCh + 1) * kChunkBytes;   // high, low and bias chunks
  static constexpr int kStages = D == 128 ? 3 : 5;
  static constexpr int kEpiWarps = 16;                 // 4 lane quadrants x 2 halves x 2 column halves
  static constexpr int kLoadWarp = kEpiWarps;          // TMA
  static constexpr int kMmaWarp = kEpiWarps + 1;       // + h: the MMAs of half h; warp kMmaWarp owns TMEM
  static constexpr int kThreads = (kEpiWarps + 3) * 32;
  static constexpr int oW = 0;
  static constexpr int oMerge = oW + kStages * kWStage;     // [2 halves][128 tokens][4 values, 4 centroids]
  static constexpr int kParkStride = 36;               // floats per lane row (144 B: 16-byte stores conflict-free)
  static constexpr int oPark = oMerge + 2 * 128 * 8 * 4;    // [16 warps][32 lanes][36] fp32
  static constexpr int oBar = oPark + kEpiWarps * 32 * kParkStride * 4;
  static constexpr int kSmemBytes = oBar + 256 + 1024;
  // TMEM columns: accumulator (buffer b, half h) at 64 (2 b + h); the tokens of
  // half h (bf16 pairs, D / 2 columns) at kColX + (D / 2) h; the ones block (its
  // first column two bf16 ones, then zeros) at kColOnes
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColX = 256;
  static constexpr uint32_t kColOnes = 384;
  static constexpr uint32_t kIdesc = idesc_bf16_f32(128, kCt, false);
};

// A token's four smallest values so far, ascending, with their centroids.
struct Top4 {
  float b0, b1, b2, b3;
  int i0, i1, i2, i3;
  __device__ __forceinline__ void init() {
    b0 = b1 = b2 = b3 = INFINITY;
    i0 = i1 = i2 = i3 = 0x7fffffff;
  }
  // x enters if it is smaller than the fourth best; it goes after the values it
  // equals. Every new entry is a select of the old ones (no data-dependent
  // branches beyond the entry test), so the state stays in registers.
  __device__ __forceinline__ void offer(float x, int c) {
    if (x < b3) {
      const bool l2 = x < b2, l1 = x < b1, l0 = x < b0;
      b3 = l2 ? b2 : x;
      i3 = l2 ? i2 : c;
      b2 = l1 ? b1 : (l2 ? x : b2);
      i2 = l1 ? i1 : (l2 ? c : i2);
      b1 = l0 ? b0 : (l1 ? x : b1);
      i1 = l0 ? i0 : (l1 ? c : i1);
      b0 = l0 ? x : b0;
      i0 = l0 ? c : i0;
    }
  }
};

// The k-th centroid tile a CTA visits: its own tile tt0 first (the clusters its
// tokens started in), then alternately the next one up and the next one down
// (odd k up, even k down) while both sides last, then the rest of the longer
// side, so a token's nearest clusters come early and the four best settle at once.
static __device__ __forceinline__ int visit_tile(int k, int tt0, int nt) {
  const int up = nt - 1 - tt0, m = min(up, tt0);
  if (k <= 2 * m) return (k & 1) ? tt0 + (k + 1) / 2 : tt0 - k / 2;
  return up > tt0 ? tt0 + k - m : tt0 - (k - m);
}

template <int D>
__global__ void __launch_bounds__(ClusterTcCfg<D>::kThreads, 1)
    cluster_assign_tc_kernel(const __nv_bfloat16* __restrict__ X, const __grid_constant__ CUtensorMap tmW, int N,
                             int C, int* __restrict__ cand) {
  using Cf = ClusterTcCfg<D>;
  extern __shared__ uint8_t tsm_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tsm_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sW = base + Cf::oW;
  float* sMerge = reinterpret_cast<float*>(base + Cf::oMerge);
  float* sPark = reinterpret_cast<float*>(base + Cf::oPark);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + Cf::oBar);
  uint64_t* wfull = bars;                      // [kStages]
  uint64_t* wempty = bars + 6;                 // [kStages], one arrival per half's MMAs
  uint64_t* dfull = bars + 12;                 // [half][buffer]
  uint64_t* dempty = bars + 16;                // [half][buffer], one arrival per epilogue warp of the half
  uint64_t* drain = bars + 20;                 // [half]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 22);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 23);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long bh = blockIdx.y;
  const int t0 = blockIdx.x * Cf::kTok;
  const int ntiles = (C + Cf::kCt - 1) / Cf::kCt;
  // the centroid tile holding the first cluster of this CTA's tokens (64 per cluster)
  const int tt0 = min(ntiles - 1, t0 / (kBlock * Cf::kCt));

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cf::kStages; ++s) {
      mbar_init(&wfull[s], 1);
      mbar_init(&wempty[s], 2);
    }
    for (int b = 0; b < 4; ++b) {
      mbar_init(&dfull[b], 1);
      mbar_init(&dempty[b], Cf::kEpiWarps / 2);
    }
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == Cf::kMmaWarp) tmem_alloc(tmem_holder, Cf::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // the tokens into TMEM: warp w < 8 writes lanes 32 (w % 4) .. of half w / 4, one
  // token per lane, its bf16 row as D / 2 packed columns (zeros past N)
  if (warp < 8) {
    const int quad = warp & 3, h = warp >> 2;
    const int tok = t0 + 128 * h + 32 * quad + lane;
    const uint4* src = reinterpret_cast<const uint4*>(X + (bh * N + min(tok, N - 1)) * static_cast<long long>(D));
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      uint32_t r[32];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint4 u = tok < N ? __ldg(src + 8 * c + q) : make_uint4(0u, 0u, 0u, 0u);
        r[4 * q] = u.x;
        r[4 * q + 1] = u.y;
        r[4 * q + 2] = u.z;
        r[4 * q + 3] = u.w;
      }
      tmem_st32u(tmem_base + (static_cast<uint32_t>(32 * quad) << 16) + Cf::kColX + (D / 2) * h + 32 * c, r);
    }
    if (h == 0) {   // the ones block, for this warp's lanes
      uint32_t r[32];
#pragma unroll
      for (int q = 0; q < 32; ++q) r[q] = q == 0 ? 0x3F803F80u : 0u;   // two bf16 ones
      tmem_st32u(tmem_base + (static_cast<uint32_t>(32 * quad) << 16) + Cf::kColOnes, r);
    }
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp == Cf::kLoadWarp) {
    // ------------------------------------------------------------ loads
    if (lane == 0) {
      tma_prefetch_desc(&tmW);
      int nw = 0;
      for (int t = 0; t < ntiles; ++t) {
        const int s = t % Cf::kStages;
        // the stage's previous tile (t - kStages) is read by both halves' MMAs
        if (t >= Cf::kStages &&
            !mbar_wait(&wempty[s], static_cast<uint32_t>((t - Cf::kStages) / Cf::kStages) & 1u, abort_flag))
          break;
        mbar_expect_tx(&wfull[s], Cf::kWStage);
        tma_load_4d(sW + s * Cf::kWStage, &tmW, 0, visit_tile(t, tt0, ntiles) * Cf::kCt, 0, static_cast<int>(bh),
                    &wfull[s]);
        ++nw;
      }
      for (int k = max(0, nw - Cf::kStages); k < nw; ++k)   // no copy outlives the CTA
        mbar_wait_drain(&wfull[k % Cf::kStages], static_cast<uint32_t>(k / Cf::kStages) & 1u);
    }
  } else if (warp > Cf::kLoadWarp) {
    // ------------------------------------------------------------ the MMAs of half h
    const int h = warp - Cf::kMmaWarp;
    if (lane == 0) {
      const uint32_t wa = smem_u32(sW);
      const uint32_t aX = tmem_base + Cf::kColX + (D / 2) * h;
      for (int t = 0; t < ntiles; ++t) {
        const int s = t % Cf::kStages, buf = t & 1;
        if (!mbar_wait(&wfull[s], static_cast<uint32_t>(t / Cf::kStages) & 1u, abort_flag)) break;
        if (t >= 2 && !mbar_wait(&dempty[2 * h + buf], static_cast<uint32_t>((t >> 1) - 1) & 1u, abort_flag))
          break;
        tc_fence_after();
        const uint32_t wb = wa + s * Cf::kWStage;
        const uint32_t dD = tmem_base + Cf::kCt * (2 * buf + h);
#pragma unroll
        for (int kk = 0; kk < 2 * (D / 16); ++kk) {   // the high part, then the low part
          const int k = kk % (D / 16);
          tc_mma_ts(dD, aX + k * 8,
                    sdesc_sw128(wb + (kk >> 2) * Cf::kChunkBytes + (kk & 3) * 32, 16, 1024), Cf::kIdesc,
                    kk > 0 ? 1u : 0u);
        }
        // the bias: the ones block against the first K-step of the rows' bias chunk
        tc_mma_ts(dD, tmem_base + Cf::kColOnes, sdesc_sw128(wb + 2 * Cf::kCh * Cf::kChunkBytes, 16, 1024),
                  Cf::kIdesc, 1u);
        tc_commit(&dfull[2 * h + buf]);
        tc_commit(&wempty[s]);
      }
      tc_commit(&drain[h]);
      mbar_wait_drain(&drain[h], 0u);
    }
  } else {
    // ------------------------------------------------------------ epilogue: the four best
    const int quad = warp & 3, h = (warp >> 2) & 1, cq = warp >> 3;
    const int row = quad * 32 + lane;          // token of the half == TMEM lane
    const uint32_t lane_bits = static_cast<uint32_t>(quad * 32) << 16;
    float* park = sPark + (warp * 32 + lane) * Cf::kParkStride;
    Top4 st;
    st.init();
    bool alive = true;
    for (int t = 0; t < ntiles; ++t) {
      const int buf = t & 1;
      const int c0 = visit_tile(t, tt0, ntiles) * Cf::kCt + cq * 32;
      const int ncol = C - c0;                 // < 32 in the last tile: columns past C read zero rows
      if (!warp_wait(&dfull[2 * h + buf], static_cast<uint32_t>(t >> 1) & 1u, abort_flag)) {
        alive = false;
        break;
      }
      tc_fence_after();
      float v[32];
      tmem_ld32(tmem_base + lane_bits + Cf::kCt * (2 * buf + h) + cq * 32, v);
      tmem_wait_ld();
      pin32(v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&dempty[2 * h + buf]);   // the buffer may take tile t + 2
      if (ncol < 32) {
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (e >= ncol) v[e] = INFINITY;
      }
      // 8-column groups whose minimum is below the fourth best, then their values
      uint32_t gm = 0;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const float* w = v + 8 * g;
        const float m = fmin3(fmin3(w[0], w[1], w[2]), fmin3(w[3], w[4], w[5]), fminf(w[6], w[7]));
        gm |= (m < st.b3 ? 1u : 0u) << g;
      }
      if (__any_sync(0xffffffffu, gm != 0u)) {
        uint32_t pend = 0;                     // the values that may enter
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          if (gm & (1u << g)) {
            const float* w = v + 8 * g;
#pragma unroll
            for (int e = 0; e < 8; ++e) pend |= (w[e] < st.b3 ? 1u : 0u) << (8 * g + e);
            reinterpret_cast<float4*>(park)[2 * g] = make_float4(w[0], w[1], w[2], w[3]);
            reinterpret_cast<float4*>(park)[2 * g + 1] = make_float4(w[4], w[5], w[6], w[7]);
          }
        }
        while (pend) {                         // this lane's own row: no exchange between lanes
          const int e0 = __ffs(pend) - 1;      // two entries per pass: their loads overlap
          pend &= pend - 1;
          const int e1 = pend ? __ffs(pend) - 1 : e0;
          pend &= pend - 1;
          const float x0 = park[e0], x1 = park[e1];
          st.offer(x0, c0 + e0);
          if (e1 != e0) st.offer(x1, c0 + e1);
        }
      }
    }
    // the column halves of a token merge: half 1 hands its four to half 0
    if (cq == 1) {
      float* m = sMerge + (h * 128 + row) * 8;
      m[0] = st.b0;
      m[1] = st.b1;
      m[2] = st.b2;
      m[3] = st.b3;
      m[4] = __int_as_float(st.i0);
      m[5] = __int_as_float(st.i1);
      m[6] = __int_as_float(st.i2);
      m[7] = __int_as_float(st.i3);
    }
    asm volatile("bar.sync 1, %0;" ::"n"(Cf::kEpiWarps * 32) : "memory");   // the epilogue warps
    const int tok = t0 + 128 * h + row;
    if (cq == 0 && tok < N) {
      const float* m = sMerge + (h * 128 + row) * 8;
#pragma unroll
      for (int q = 0; q < 4; ++q) st.offer(m[q], __float_as_int(m[4 + q]));
      // a wait that gave up anywhere leaves this token's candidates unwritten
      if (alive && !*abort_flag) {
        int4 o;
        o.x = st.i0;
        o.y = st.i1;
        o.z = st.i2;
        o.w = st.i3;
        *reinterpret_cast<int4*>(cand + (bh * N + tok) * 4) = o;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == Cf::kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cf::kTmemCols);
  }
}

// The exact argmin among a token's four candidates: b_c - 2 x . w_c in fp32
// (x the bf16 token, w_c and b_c from cluster_prep_kernel), ties to the lowest
// c; the winner is counted into its cluster's size. A candidate outside [0, C)
// (a head with fewer than four clusters) is skipped. A warp per token: lane l
// holds components [D/32 l, D/32 (l+1)) of x and of the four rows (coalesced
// loads, all issued before the arithmetic), and the four partial dot products are
// summed across the warp. Grid (ceil(N / 64), B*H), 256 threads, 8 tokens per warp.
template <int D>
__global__ void __launch_bounds__(256) cluster_rescore_kernel(const __nv_bfloat16* __restrict__ X,
                                                              const float* __restrict__ W,
                                                              const float* __restrict__ bvec,
                                                              const int* __restrict__ cand,
                                                              int* __restrict__ assign, int* __restrict__ cnt, int N,
                                                              int C) {
  constexpr int E = D / 32;                    // components per lane: 4 or 2
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long bh = blockIdx.y;
  for (int k = 0; k < 8; ++k) {
    const int tok = blockIdx.x * 64 + warp * 8 + k;
    if (tok >= N) return;
    const long long r = bh * N + tok;
    const int4 cd = *reinterpret_cast<const int4*>(cand + r * 4);
    const int cs[4] = {cd.x, cd.y, cd.z, cd.w};
    float x[E];
    if constexpr (E == 4) {
      const uint2 u = __ldg(reinterpret_cast<const uint2*>(X + r * D) + lane);
      x[0] = __uint_as_float(u.x << 16);
      x[1] = __uint_as_float(u.x & 0xffff0000u);
      x[2] = __uint_as_float(u.y << 16);
      x[3] = __uint_as_float(u.y & 0xffff0000u);
    } else {
      const uint32_t u = __ldg(reinterpret_cast<const uint32_t*>(X + r * D) + lane);
      x[0] = __uint_as_float(u << 16);
      x[1] = __uint_as_float(u & 0xffff0000u);
    }
    float wv[4][E];
    float bq[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const bool ok = cs[q] >= 0 && cs[q] < C;
      const long long row = bh * C + (ok ? cs[q] : 0);
      if constexpr (E == 4) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(W + row * D) + lane);
        wv[q][0] = v.x;
        wv[q][1] = v.y;
        wv[q][2] = v.z;
        wv[q][3] = v.w;
      } else {
        const float2 v = __ldg(reinterpret_cast<const float2*>(W + row * D) + lane);
        wv[q][0] = v.x;
        wv[q][1] = v.y;
      }
      bq[q] = __ldg(bvec + row);
    }
    float best = INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) dot = fmaf(x[e], wv[q][e], dot);
#pragma unroll
      for (int o = 16; o; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      const float sc = bq[q] - 2.f * dot;
      const int c = cs[q];
      if (c >= 0 && c < C && (sc < best || (sc == best && c < bi))) {
        best = sc;
        bi = c;
      }
    }
    // a NaN score never compares smaller: a token whose every candidate scores NaN
    // keeps no cluster, which the range check turns into cluster 0 and an error bit
    if (lane == 0) {
      if (bi < 0 || bi >= C) {
        atomicOr(&g_dev_error, DEVERR_VALUE);
        bi = 0;
      }
      assign[r] = bi;
      atomicAdd(&cnt[bh * C + bi], 1);
    }
  }
}

// The stable order, a counting sort in three steps over chunks of L tokens of a
// head (order_chunk): the tokens of cluster c go to perm[off[c] ..] in token order.
//
// Step 1: part[bh][j][c] = the number of chunk j's tokens in cluster c. Grid
// (chunks, B*H), 256 threads, a shared-memory histogram of C counts (a warp's
// lanes with the same cluster add once, through match_any). A cluster index
// outside [0, C) is not counted; it sets the range bit of the device error word.
__global__ void __launch_bounds__(256) cluster_chunk_count_kernel(const int* __restrict__ assign,
                                                                  int* __restrict__ part, int N, int C, int L) {
  extern __shared__ int hist[];
  const long long bh = blockIdx.y;
  const int j = blockIdx.x, lane = threadIdx.x & 31;
  const int t0 = j * L, t1 = min(N, t0 + L);
  for (int c = threadIdx.x; c < C; c += 256) hist[c] = 0;
  __syncthreads();
  for (int tb = t0; tb < t1; tb += 256) {
    const int t = tb + threadIdx.x;
    int c = t < t1 ? assign[bh * N + t] : -1;
    if (t < t1 && (c < 0 || c >= C)) {
      atomicOr(&g_dev_error, DEVERR_RANGE);
      c = -1;
    }
    const unsigned peers = __match_any_sync(0xffffffffu, c);
    if (c >= 0 && lane == __ffs(peers) - 1) atomicAdd(&hist[c], __popc(peers));
  }
  __syncthreads();
  for (int c = threadIdx.x; c < C; c += 256) part[(bh * gridDim.x + j) * C + c] = hist[c];
}

// Step 2: part[bh][j][c] becomes the first position of chunk j's tokens of
// cluster c: off[c] plus the counts of the earlier chunks. Grid (ceil(C/256),
// B*H), a thread per cluster walking the chunks in order.
__global__ void __launch_bounds__(256) cluster_chunk_scan_kernel(const int* __restrict__ off, int* __restrict__ part,
                                                                 int C, int chunks) {
  const long long bh = blockIdx.y;
  const int c = blockIdx.x * 256 + threadIdx.x;
  if (c >= C) return;
  int run = off[bh * C + c];
  int* col = part + bh * chunks * static_cast<long long>(C) + c;
  for (int j0 = 0; j0 < chunks; j0 += 16) {   // 16 loads in flight, then their stores
    int v[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) v[q] = j0 + q < chunks ? col[static_cast<long long>(j0 + q) * C] : 0;
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      if (j0 + q < chunks) col[static_cast<long long>(j0 + q) * C] = run;
      run += v[q];
    }
  }
}

// Step 3: one warp per chunk places its tokens 32 at a time, in token order: a
// token's position is its cluster's next free position in the chunk (a
// shared-memory copy of step 2's column) plus its rank among the lanes with the
// same cluster (match_any); the group's highest lane then advances the position.
// Grid (chunks, B*H), 32 threads, C ints of shared memory. A position outside
// [0, N) (inconsistent sizes) is not written; it sets the range bit.
__global__ void __launch_bounds__(32) cluster_order_kernel(const int* __restrict__ assign,
                                                           const int* __restrict__ part, int* __restrict__ perm,
                                                           int N, int C, int L) {
  extern __shared__ int next[];
  const long long bh = blockIdx.y;
  const int j = blockIdx.x, lane = threadIdx.x;
  const int t0 = j * L, t1 = min(N, t0 + L);
  const int* col = part + (bh * gridDim.x + j) * C;
  for (int c = lane; c < C; c += 32) next[c] = col[c];
  __syncwarp();
  const unsigned below = (1u << lane) - 1u;
  for (int tb = t0; tb < t1; tb += 32) {
    const int t = tb + lane;
    int c = t < t1 ? assign[bh * N + t] : -1;
    if (c >= C) c = -1;                        // counted as an error in step 1
    const unsigned peers = __match_any_sync(0xffffffffu, c);
    if (c >= 0) {
      const int pos = next[c] + __popc(peers & below);
      if (pos >= 0 && pos < N)
        perm[bh * N + pos] = t;
      else
        atomicOr(&g_dev_error, DEVERR_RANGE);
    }
    __syncwarp();
    if (c >= 0 && lane == 31 - __clz(peers)) next[c] += __popc(peers);
    __syncwarp();
  }
}

// Each cluster's mean, one warp per cluster: its tokens in token order are
// perm[off[c] .. off[c] + cnt[c]), summed in that order (fp32), each lane owning
// D/32 dimensions. An empty cluster keeps its centroid. Grid (ceil(C/8), B*H),
// 256 threads.
template <int D>
__global__ void __launch_bounds__(256) cluster_centroid_kernel(const __nv_bfloat16* __restrict__ X,
                                                               const int* __restrict__ perm,
                                                               const int* __restrict__ off,
                                                               const int* __restrict__ cnt, float* __restrict__ cent,
                                                               int N, int C) {
  constexpr int PL = D / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long bh = blockIdx.y;
  const int c = blockIdx.x * 8 + warp;
  if (c >= C) return;
  const int n = cnt[bh * C + c];
  if (n == 0) return;
  const int* p = perm + bh * N + off[bh * C + c];
  float acc[PL];
#pragma unroll
  for (int e = 0; e < PL; ++e) acc[e] = 0.f;
  // four members' loads in flight at a time, added in token order
  for (int r = 0; r < n; r += 4) {
    float v[4][PL];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (r + u < n) {
        const __nv_bfloat16* row = X + (bh * N + p[r + u]) * static_cast<long long>(D) + lane * PL;
        if constexpr (PL == 4) {
          const uint2 w = *reinterpret_cast<const uint2*>(row);
          const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.x));
          const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.y));
          v[u][0] = f0.x;
          v[u][1] = f0.y;
          v[u][2] = f1.x;
          v[u][3] = f1.y;
        } else {
          static_assert(PL == 2, "d must be 64 or 128");
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(row));
          v[u][0] = f.x;
          v[u][1] = f.y;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (r + u < n) {
#pragma unroll
        for (int e = 0; e < PL; ++e) acc[e] += v[u][e];
      }
    }
  }
#pragma unroll
  for (int e = 0; e < PL; ++e) cent[(bh * C + c) * static_cast<long long>(D) + lane * PL + e] = acc[e] / n;
}

// off[bh, c] = sum of cnt[bh, c'] over c' < c: one CTA of 1024 threads per head,
// 4 consecutive clusters per thread (C <= 4096).
__global__ void __launch_bounds__(1024) cluster_offsets_kernel(const int* __restrict__ cnt, int* __restrict__ off,
                                                               int C) {
  __shared__ int sbuf[33];
  const long long bh = blockIdx.x;
  const int c0 = threadIdx.x * 4;
  int v[4], local = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    v[e] = (c0 + e < C) ? cnt[bh * C + c0 + e] : 0;
    local += v[e];
  }
  // exclusive scan of `local` over the block
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int x = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sbuf[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = sbuf[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    sbuf[lane] = w;   // inclusive warp totals
  }
  __syncthreads();
  int run = x - local + (warp > 0 ? sbuf[warp - 1] : 0);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    if (c0 + e < C) off[bh * C + c0 + e] = run;
    run += v[e];
  }
}

// Row moves of [B,H,N,D] bf16 tensors by a per-head permutation: gather
// dst[bh, p] = src[bh, perm[bh, p]], or (inverse) scatter dst[bh, perm[bh, p]] =
// src[bh, p]. Grid (ceil(N * D / 8 / 1024), B*H), four 16-byte vectors per
// thread (the index within a head fits 32 bits). A perm entry outside [0, N) moves nothing
// and sets the range bit of the device error word.
template <int D>
__global__ void __launch_bounds__(256) permute_rows_kernel(const __nv_bfloat16* __restrict__ src,
                                                           const int* __restrict__ perm, __nv_bfloat16* __restrict__ dst,
                                                           int N, int inverse) {
  constexpr int V = D / 8;   // 16-byte vectors per row
  constexpr int kU = 4;      // vectors per thread, 256 apart: all loads issue before the stores
  const long long bh = blockIdx.y;
  const int base = blockIdx.x * 256 * kU + threadIdx.x;
  uint4 val[kU];
  long long to[kU];
#pragma unroll
  for (int u = 0; u < kU; ++u) {
    const int x = base + u * 256;
    to[u] = -1;
    if (x < N * V) {
      const int r = x / V, v = x % V;
      const int p = __ldg(perm + bh * N + r);
      if (p < 0 || p >= N) {
        if (v == 0) atomicOr(&g_dev_error, DEVERR_RANGE);
      } else {
        const long long from = bh * N + (inverse ? r : p);
        to[u] = (bh * N + (inverse ? p : r)) * V + v;
        val[u] = __ldg(reinterpret_cast<const uint4*>(src + from * D) + v);
      }
    }
  }
#pragma unroll
  for (int u = 0; u < kU; ++u)
    if (to[u] >= 0) reinterpret_cast<uint4*>(dst)[to[u]] = val[u];
}

}  // namespace sa

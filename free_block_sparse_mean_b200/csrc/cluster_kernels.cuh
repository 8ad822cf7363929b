// Interaction clustering: k-means of one side's tokens (queries or keys) under
// the other side's Gram metric, and the token reordering that follows it.
//
// The iCATS abstract clusters query and key tokens by their dot-product
// interaction rather than by feature similarity, and reduces the objective to a
// quadratic form. Replacing a token x by a centroid c changes its score with
// every token y of the other side by (x - c).y; the sum of the squares is
// (x - c)^T G (x - c) with G = sum_y y y^T. Dropping the term x^T G x, which is
// the same for every centroid, the nearest centroid is the argmin over c of
// c^T G c - 2 x . (G c). So each Lloyd iteration is: w_c = G c and b_c = c . w_c
// per centroid (cluster_prep_kernel), an argmin over all centroids per token (a
// bf16 tensor-core product of the tokens with the w_c that keeps each token's four
// best, cluster_assign_tc_kernel, then their exact fp32 scores,
// cluster_rescore_kernel), and the mean of each cluster's tokens
// (cluster_centroid_kernel). The
// clusters start at the 64-token block means (the pooling kernel), so zero
// iterations reproduce the plain blocks.
//
// The reordering is a stable sort of the tokens by cluster: a per-head
// exclusive scan of the cluster sizes gives each cluster's first position, and
// each cluster's tokens follow in token order. Clusters are packed back to back,
// so the tail of one shares a 64-token block with the head of the next (the
// abstract's "tail merging", with no padding at all).
//
// Each iteration: cluster_prep_kernel (w_c, b_c, their bf16 operand rows; clears
// the sizes), cluster_assign_tc_kernel and cluster_rescore_kernel (argmin; counts
// the sizes), cluster_offsets_kernel (each
// cluster's first position), cluster_order_kernel (the stable order) and
// cluster_centroid_kernel (each cluster's mean, summed over its tokens in token
// order through the order just built). Everything is deterministic: every fp32
// sum runs in a fixed order, the sizes are integer counts, and argmin ties go to
// the lowest cluster index.
#pragma once

#include "sa_device.cuh"

namespace sa {

// Tokens per partial Gram matrix: about 600 CTAs over all heads, at least 512
// tokens each, a multiple of 32.
inline int gram_chunk(long long BH, int N) {
  const long long want_splits = (600 + BH - 1) / BH;
  long long chunk = (N + want_splits - 1) / want_splits;
  chunk = chunk < 512 ? 512 : chunk;
  return static_cast<int>((chunk + 31) / 32 * 32);
}

// Byte offsets of the clustering workspace: partial Gram matrices, the Gram
// matrix, centroids, w_c = G c, b_c, cluster sizes, first positions, the
// assignment (when the caller does not want it back), the tensor-core operand
// rows of the centroids (bf16 [B*H][C][D + 64], see cluster_prep_kernel) and four
// candidate clusters per token.
struct ClusterWorkspace {
  size_t gpart, gram, cent, w, b, cnt, off, assign, w16, cand, total;
  int splits, chunk, C;
};
inline ClusterWorkspace cluster_workspace(long long BH, int N, int D) {
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  ClusterWorkspace w;
  w.C = (N + kBlock - 1) / kBlock;
  w.chunk = gram_chunk(BH, N);
  w.splits = (N + w.chunk - 1) / w.chunk;
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
  w.cand = w.w16 + al(static_cast<size_t>(BH) * w.C * (D + 64) * 2);
  w.total = w.cand + al(static_cast<size_t>(BH) * N * 4 * sizeof(int));
  return w;
}

// Partial Gram matrix sum_t y_t y_t^T over one chunk of `chunk` tokens of one
// head, fp32, tokens in order. Grid (chunks, B*H), 256 threads; thread (r, c) of
// a 16 x 16 grid owns the T x T entries rows T r .., columns T c .. (T = D/16).
template <int D>
__global__ void __launch_bounds__(256) gram_partial_kernel(const __nv_bfloat16* __restrict__ Y,
                                                           float* __restrict__ part, int N, int splits, int chunk) {
  constexpr int T = D / 16;
  constexpr int kTok = 32;
  __shared__ __align__(16) float ys[kTok][D];
  const long long bh = blockIdx.y;
  const int s = blockIdx.x;
  const int t0 = s * chunk, t1 = min(N, t0 + chunk);
  const int ri = (threadIdx.x >> 4) * T, ci = (threadIdx.x & 15) * T;
  float acc[T][T];
#pragma unroll
  for (int i = 0; i < T; ++i)
#pragma unroll
    for (int j = 0; j < T; ++j) acc[i][j] = 0.f;
  const __nv_bfloat16* src = Y + bh * static_cast<long long>(N) * D;
  for (int t = t0; t < t1; t += kTok) {
    const int n = min(kTok, t1 - t);
    __syncthreads();   // the previous rows are consumed
    for (int x = threadIdx.x; x < kTok * D / 8; x += 256) {
      const int r = x / (D / 8), c8 = (x % (D / 8)) * 8;
      uint4 u = make_uint4(0u, 0u, 0u, 0u);
      if (r < n) u = __ldg(reinterpret_cast<const uint4*>(src + static_cast<long long>(t + r) * D + c8));
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h[e]);
        ys[r][c8 + 2 * e] = f.x;
        ys[r][c8 + 2 * e + 1] = f.y;
      }
    }
    __syncthreads();
    for (int r = 0; r < n; ++r) {
      float a[T], b[T];
#pragma unroll
      for (int i = 0; i < T; ++i) {
        a[i] = ys[r][ri + i];
        b[i] = ys[r][ci + i];
      }
#pragma unroll
      for (int i = 0; i < T; ++i)
#pragma unroll
        for (int j = 0; j < T; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
  }
  float* out = part + (bh * splits + s) * static_cast<long long>(D) * D;
#pragma unroll
  for (int i = 0; i < T; ++i)
#pragma unroll
    for (int j = 0; j < T; ++j) out[(ri + i) * D + ci + j] = acc[i][j];
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
// W16 (bf16 [B*H][C][D + 64]) receives each centroid's tensor-core operand row for
// the assignment: -2 w_c in columns [0, D), then b_c as the sum of two bf16 values
// (b_hi = bf16(b_c) in column D, b_lo = bf16(b_c - b_hi) in column D + 1) and zeros.
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
      W16[(bh * C + c0 + c) * (D + 64) + i] = __float2bfloat16_rn(-2.f * acc[c]);
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
    W16[(bh * C + c0 + c) * (D + 64) + D + k] = v;
  }
}

// ----------------------------------------------------------------------------
// Tensor-core assignment: the four nearest centroids of every token by a bf16
// product on the tensor cores, then the exact argmin among those four in fp32
// (cluster_rescore_kernel). One CTA = 128 tokens of one head:
//   D[token][c] = x . (-2 w_c) + 1 . b_hi_c + 1 . b_lo_c
// (tcgen05.mma kind::f16, fp32 accumulate in TMEM), over tiles of 128 centroids:
// D / 16 K-steps of the token tile (TMA'd once) against the centroid tile's bf16
// rows from cluster_prep_kernel, plus one K-step of a constant tile whose rows
// start with two ones against the rows' bias columns. Warp 4 (one thread) loads
// and issues; warps 0-3 (thread = token = TMEM lane) keep each token's four
// smallest D values with their centroids (ties to the lower centroid) in
// registers. Two TMEM buffers of 128 columns and three centroid-tile stages keep
// the tensor cores and the epilogue overlapped.
// The bf16 product moves the argmin for a fraction of a percent of the tokens;
// the four best of the product contain the fp32 argmin (measured on the
// workloads' inputs), and the re-score restores it exactly.
template <int D>
struct ClusterTcCfg {
  static constexpr int kCh = D / 64;                   // 128-byte column chunks of a row
  static constexpr int kTile = 128;                    // tokens per CTA, centroids per tile
  static constexpr int kChunkBytes = kTile * 128;      // 16 KB: one column chunk of a tile
  static constexpr int kStages = 3;
  static constexpr int kWStage = (kCh + 1) * kChunkBytes;   // centroid rows + bias chunk
  static constexpr int oX = 0;
  static constexpr int oOnes = oX + kCh * kChunkBytes;
  static constexpr int oW = oOnes + kChunkBytes;
  static constexpr int oBar = oW + kStages * kWStage;
  static constexpr int kSmemBytes = oBar + 128 + 1024;
  static constexpr uint32_t kTmemCols = 256;
  static constexpr uint32_t kIdesc = idesc_bf16_f32(128, 128, false);
};

// A token's four smallest scores so far, ascending, with their centroids (the
// epilogue's state, touched only when a score may enter).
struct Top4 {
  float b[4];
  int i[4];
};

// Offers the scores x[e] of centroids c0 + e (e < lim) in ascending centroid order;
// a score enters if it is smaller than the fourth best (so a tie keeps the earlier
// centroid). Returns the new fourth best. Not inlined: the insertion code then
// exists once, and the epilogue's hot path stays small.
static __device__ __noinline__ float top4_offer8(Top4* st, float x0, float x1, float x2, float x3, float x4,
                                                 float x5, float x6, float x7, int c0, int lim) {
  const float xs[8] = {x0, x1, x2, x3, x4, x5, x6, x7};
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float x = xs[e];
    if (e < lim && x < st->b[3]) {
      int p = 3;
      while (p > 0 && x < st->b[p - 1]) {
        st->b[p] = st->b[p - 1];
        st->i[p] = st->i[p - 1];
        --p;
      }
      st->b[p] = x;
      st->i[p] = c0 + e;
    }
  }
  return st->b[3];
}

template <int D>
__global__ void __launch_bounds__(160, 1)
    cluster_assign_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                             int N, int C, int* __restrict__ cand) {
  using Cf = ClusterTcCfg<D>;
  extern __shared__ uint8_t tsm_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tsm_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sX = base + Cf::oX;
  uint8_t* sOnes = base + Cf::oOnes;
  uint8_t* sW = base + Cf::oW;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + Cf::oBar);
  uint64_t* wfull = bars;                      // [3]
  uint64_t* wempty = bars + 3;                 // [3]
  uint64_t* dfull = bars + 6;                  // [2]
  uint64_t* dempty = bars + 8;                 // [2], 4 arrivals
  uint64_t* xfull = bars + 10;
  uint64_t* drain = bars + 11;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 12);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 13);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long bh = blockIdx.y;
  const int t0 = blockIdx.x * Cf::kTile;
  const int ntiles = (C + Cf::kTile - 1) / Cf::kTile;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cf::kStages; ++s) {
      mbar_init(&wfull[s], 1);
      mbar_init(&wempty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&dfull[b], 1);
      mbar_init(&dempty[b], 4);
    }
    mbar_init(xfull, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // the constant tile: row r holds ones in columns 0 and 1 (16-byte chunk 0 of the
  // row, which the 128-byte swizzle stores at chunk (r & 7)), zeros elsewhere
  for (int x = threadIdx.x; x < Cf::kChunkBytes / 16; x += blockDim.x)
    reinterpret_cast<uint4*>(sOnes)[x] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  if (threadIdx.x < Cf::kTile) {
    const int r = threadIdx.x;
    const uint32_t one2 = 0x3F803F80u;         // two bf16 ones
    *reinterpret_cast<uint32_t*>(sOnes + r * 128 + (r & 7) * 16) = one2;
  }
  fence_proxy_async_smem();                    // generic-proxy writes -> the tensor cores' reads
  if (warp == 4) tmem_alloc(tmem_holder, Cf::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 4) {
    // ------------------------------------------------------------ loads and MMAs
    if (lane == 0) {
      tma_prefetch_desc(&tmX);
      tma_prefetch_desc(&tmW);
      mbar_expect_tx(xfull, Cf::kCh * Cf::kChunkBytes);
      for (int c = 0; c < Cf::kCh; ++c)
        tma_load_3d(sX + c * Cf::kChunkBytes, &tmX, c * 64, t0, static_cast<int>(bh), xfull);
      auto load_w = [&](int t) {
        const int s = t % Cf::kStages;
        mbar_expect_tx(&wfull[s], Cf::kWStage);
        for (int c = 0; c <= Cf::kCh; ++c)
          tma_load_3d(sW + s * Cf::kWStage + c * Cf::kChunkBytes, &tmW, c * 64, t * Cf::kTile,
                      static_cast<int>(bh), &wfull[s]);
      };
      int nw = 0;
      for (; nw < Cf::kStages && nw < ntiles; ++nw) load_w(nw);
      const uint32_t xa = smem_u32(sX), oa = smem_u32(sOnes), wa = smem_u32(sW);
      bool ok = mbar_wait(xfull, 0u, abort_flag);
      for (int t = 0; ok && t < ntiles; ++t) {
        const int s = t % Cf::kStages, buf = t & 1;
        if (!mbar_wait(&wfull[s], static_cast<uint32_t>(t / Cf::kStages) & 1u, abort_flag)) break;
        if (t >= 2 && !mbar_wait(&dempty[buf], static_cast<uint32_t>((t >> 1) - 1) & 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t dD = tmem_base + buf * 128;
        const uint32_t wb = wa + s * Cf::kWStage;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * Cf::kChunkBytes + (kk & 3) * 32;
          tc_mma_ss(dD, sdesc_sw128(xa + off, 16, 1024), sdesc_sw128(wb + off, 16, 1024), Cf::kIdesc,
                    kk > 0 ? 1u : 0u);
        }
        // the bias: the ones tile's first K-step against the rows' bias columns
        tc_mma_ss(dD, sdesc_sw128(oa, 16, 1024), sdesc_sw128(wb + Cf::kCh * Cf::kChunkBytes, 16, 1024), Cf::kIdesc,
                  1u);
        tc_commit(&dfull[buf]);
        tc_commit(&wempty[s]);
        if (t + Cf::kStages < ntiles) {
          if (!mbar_wait(&wempty[s], static_cast<uint32_t>(t / Cf::kStages) & 1u, abort_flag)) break;
          load_w(t + Cf::kStages);
          ++nw;
        }
      }
      tc_commit(drain);
      mbar_wait_drain(drain, 0u);
      mbar_wait_drain(xfull, 0u);
      for (int k = max(0, nw - Cf::kStages); k < nw; ++k)
        mbar_wait_drain(&wfull[k % Cf::kStages], static_cast<uint32_t>(k / Cf::kStages) & 1u);
    }
  } else {
    // ------------------------------------------------------------ epilogue: the four best
    const int row = warp * 32 + lane;          // token of the tile == TMEM lane
    const uint32_t lane_bits = static_cast<uint32_t>(warp * 32) << 16;
    Top4 st;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      st.b[q] = INFINITY;
      st.i[q] = 0x7fffffff;
    }
    float b3 = INFINITY;                       // st.b[3], in a register for the hot path
    bool alive = true;
    for (int t = 0; t < ntiles; ++t) {
      const int buf = t & 1;
      if (!warp_wait(&dfull[buf], static_cast<uint32_t>(t >> 1) & 1u, abort_flag)) {
        alive = false;
        break;
      }
      tc_fence_after();
      float v[128];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        tmem_ld32(tmem_base + lane_bits + buf * 128 + q * 32, *reinterpret_cast<float(*)[32]>(&v[32 * q]));
      tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < 4; ++q) pin32(*reinterpret_cast<float(*)[32]>(&v[32 * q]));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&dempty[buf]);   // the buffer may take tile t + 2
      const int c0 = t * Cf::kTile;
      const int ncol = min(Cf::kTile, C - c0);
      const bool partial = ncol < Cf::kTile;   // the last tile: columns past C read zero rows
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float* w = v + 32 * q;
        float m8[4];
#pragma unroll
        for (int g = 0; g < 4; ++g)
          m8[g] = fminf(fminf(fminf(w[8 * g], w[8 * g + 1]), fminf(w[8 * g + 2], w[8 * g + 3])),
                        fminf(fminf(w[8 * g + 4], w[8 * g + 5]), fminf(w[8 * g + 6], w[8 * g + 7])));
        if (partial || fminf(fminf(m8[0], m8[1]), fminf(m8[2], m8[3])) < b3) {
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int cb = 32 * q + 8 * g;
            if (cb < ncol && (partial || m8[g] < b3))
              b3 = top4_offer8(&st, w[8 * g], w[8 * g + 1], w[8 * g + 2], w[8 * g + 3], w[8 * g + 4],
                               w[8 * g + 5], w[8 * g + 6], w[8 * g + 7], c0 + cb, ncol - cb);
          }
        }
      }
    }
    const int tok = t0 + row;
    if (alive && tok < N) {
      int4 o;
      o.x = st.i[0];
      o.y = st.i[1];
      o.z = st.i[2];
      o.w = st.i[3];
      *reinterpret_cast<int4*>(cand + (bh * N + tok) * 4) = o;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cf::kTmemCols);
  }
}

// The exact argmin among a token's four candidates: b_c - 2 x . w_c in fp32
// (x the bf16 token, w_c and b_c from cluster_prep_kernel), ties to the lowest c;
// the winner is counted into its cluster's size. A candidate outside [0, C) (a
// head with fewer than four clusters) is skipped. One thread per token.
template <int D>
__global__ void __launch_bounds__(256) cluster_rescore_kernel(const __nv_bfloat16* __restrict__ X,
                                                              const float* __restrict__ W,
                                                              const float* __restrict__ bvec,
                                                              const int* __restrict__ cand,
                                                              int* __restrict__ assign, int* __restrict__ cnt, int N,
                                                              int C) {
  const long long bh = blockIdx.y;
  const int tok = blockIdx.x * 256 + threadIdx.x;
  if (tok >= N) return;
  float x[D];
  const uint4* src = reinterpret_cast<const uint4*>(X + (bh * N + tok) * static_cast<long long>(D));
#pragma unroll
  for (int q = 0; q < D / 8; ++q) {
    const uint4 u = __ldg(src + q);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h[e]);
      x[8 * q + 2 * e] = f.x;
      x[8 * q + 2 * e + 1] = f.y;
    }
  }
  const int4 cd = *reinterpret_cast<const int4*>(cand + (bh * N + tok) * 4);
  const int cs[4] = {cd.x, cd.y, cd.z, cd.w};
  float best = INFINITY;
  int bi = 0x7fffffff;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int c = cs[q];
    if (c < 0 || c >= C) continue;
    const float4* w = reinterpret_cast<const float4*>(W + (bh * C + c) * static_cast<long long>(D));
    float dot = 0.f;
#pragma unroll
    for (int k = 0; k < D / 4; ++k) {
      const float4 wv = __ldg(w + k);
      dot = fmaf(x[4 * k], wv.x, dot);
      dot = fmaf(x[4 * k + 1], wv.y, dot);
      dot = fmaf(x[4 * k + 2], wv.z, dot);
      dot = fmaf(x[4 * k + 3], wv.w, dot);
    }
    const float sc = bvec[bh * C + c] - 2.f * dot;
    if (sc < best || (sc == best && c < bi)) {
      best = sc;
      bi = c;
    }
  }
  // a NaN score never compares smaller: a token whose every candidate scores NaN
  // keeps no cluster, which the range check turns into cluster 0 and an error bit
  if (bi < 0 || bi >= C) {
    atomicOr(&g_dev_error, DEVERR_VALUE);
    bi = 0;
  }
  assign[bh * N + tok] = bi;
  atomicAdd(&cnt[bh * C + bi], 1);
}

// Clusters per CTA of cluster_order_kernel.
constexpr int kOrderClusters = 64;

// The stable order: the tokens of cluster c go to perm[off[c] ..] in token
// order. One CTA per 64 clusters of a head scans the head's assignment 256
// tokens at a time; a token's place among its cluster's tokens of those 256 is
// its rank among the lanes of its warp with the same cluster (match_any) plus
// the counts of the earlier warps. Grid (ceil(C/64), B*H), 256 threads.
__global__ void __launch_bounds__(256) cluster_order_kernel(const int* __restrict__ assign,
                                                            const int* __restrict__ off, int* __restrict__ perm,
                                                            int N, int C) {
  __shared__ int scnt[kOrderClusters];          // tokens placed so far per cluster
  __shared__ int wcnt[8][kOrderClusters];       // per warp, current 256 tokens
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long bh = blockIdx.y;
  const int c0 = blockIdx.x * kOrderClusters;
  const int ncl = min(kOrderClusters, C - c0);
  const int* a = assign + bh * N;
  if (threadIdx.x < kOrderClusters) scnt[threadIdx.x] = 0;
  for (int t0 = 0; t0 < N; t0 += 256) {
    const int t = t0 + threadIdx.x;
    const int c = (t < N) ? a[t] - c0 : -1;
    const bool mine = c >= 0 && c < ncl;
    for (int e = threadIdx.x; e < 8 * kOrderClusters; e += 256) (&wcnt[0][0])[e] = 0;
    __syncthreads();
    const unsigned in = __ballot_sync(0xffffffffu, mine);
    unsigned peers = 0u;
    if (mine) {
      peers = __match_any_sync(in, c);
      if ((peers & ((1u << lane) - 1u)) == 0u) wcnt[warp][c] = __popc(peers);   // lowest lane of the group
    }
    __syncthreads();
    if (mine) {
      int rank = scnt[c] + __popc(peers & ((1u << lane) - 1u));
      for (int w = 0; w < warp; ++w) rank += wcnt[w][c];
      perm[bh * N + off[bh * C + c0 + c] + rank] = t;
    }
    __syncthreads();
    if (threadIdx.x < kOrderClusters) {
      int add = 0;
      for (int w = 0; w < 8; ++w) add += wcnt[w][threadIdx.x];
      scnt[threadIdx.x] += add;
    }
    __syncthreads();   // wcnt is read above before the next 256 clear it
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
// src[bh, p]. One thread per 16 bytes. A perm entry outside [0, N) moves
// nothing and sets the range bit of the device error word.
template <int D>
__global__ void __launch_bounds__(256) permute_rows_kernel(const __nv_bfloat16* __restrict__ src,
                                                           const int* __restrict__ perm, __nv_bfloat16* __restrict__ dst,
                                                           int N, long long rows, int inverse) {
  constexpr int V = D / 8;   // 16-byte vectors per row
  const long long x = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x;
  if (x >= rows * V) return;
  const long long r = x / V;
  const int v = static_cast<int>(x - r * V);
  const long long bh = r / N;
  const int p = perm[r];
  if (p < 0 || p >= N) {
    if (v == 0) atomicOr(&g_dev_error, DEVERR_RANGE);
    return;
  }
  const long long other = bh * N + p;
  const long long from = inverse ? r : other, to = inverse ? other : r;
  reinterpret_cast<uint4*>(dst + to * D)[v] = __ldg(reinterpret_cast<const uint4*>(src + from * D) + v);
}

}  // namespace sa

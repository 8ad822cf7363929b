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
// per centroid (cluster_prep_kernel), an argmin over all centroids per token
// (cluster_assign_kernel, a register-tiled fp32 product of the tokens with the
// w_c), and the mean of each cluster's tokens (cluster_centroid_kernel). The
// clusters start at the 64-token block means (the pooling kernel), so zero
// iterations reproduce the plain blocks.
//
// The reordering is a stable sort of the tokens by cluster: a per-head
// exclusive scan of the cluster sizes gives each cluster's first position, and
// each cluster's tokens follow in token order. Clusters are packed back to back,
// so the tail of one shares a 64-token block with the head of the next (the
// abstract's "tail merging", with no padding at all).
//
// Each iteration: cluster_prep_kernel (w_c, b_c; clears the sizes),
// cluster_assign_kernel (argmin; counts the sizes), cluster_offsets_kernel (each
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
// matrix, centroids, w_c = G c, b_c, cluster sizes, first positions, and the
// assignment (when the caller does not want it back).
struct ClusterWorkspace {
  size_t gpart, gram, cent, w, b, cnt, off, assign, total;
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
  w.total = w.assign + al(static_cast<size_t>(BH) * N * sizeof(int));
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
template <int D>
__global__ void __launch_bounds__(D) cluster_prep_kernel(const float* __restrict__ G, const float* __restrict__ cent,
                                                         float* __restrict__ W, float* __restrict__ bvec,
                                                         int* __restrict__ cnt, int C) {
  constexpr int kCl = 16;
  __shared__ float cs[kCl][D];
  __shared__ float red[kCl][D / 32];
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
    if (c < ncl) W[(bh * C + c0 + c) * D + i] = acc[c];
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
    cnt[bh * C + c0 + i] = 0;   // counted again by the assignment
  }
}

// Shared memory of cluster_assign_kernel: 64 tokens and 64 w_c, both D x 64 fp32.
template <int D>
constexpr int cluster_assign_smem_bytes() {
  return 2 * D * 64 * static_cast<int>(sizeof(float));
}

// Nearest centroid of 64 tokens of one head: argmin over c of b_c - 2 x . w_c,
// fp32, ties to the lowest c. Grid (ceil(N/64), B*H), 256 threads. Tokens and
// w_c sit in shared memory dimension-major, so a thread's 4 tokens and 4
// centroids are one 16-byte read each per dimension; thread (tg, cg) forms the
// 4 x 4 products of tokens 4 tg .. and centroids 4 cg .. of each chunk of 64
// centroids and keeps its 4 running minima; the 16 threads of a token group
// then meet in shared memory, and the winner is counted into its cluster's size.
template <int D>
__global__ void __launch_bounds__(256) cluster_assign_kernel(const __nv_bfloat16* __restrict__ X,
                                                             const float* __restrict__ W,
                                                             const float* __restrict__ bvec, int* __restrict__ assign,
                                                             int* __restrict__ cnt, int N, int C) {
  extern __shared__ __align__(16) float csm[];
  float* xs = csm;            // [D][64]: xs[k * 64 + token]
  float* ws = csm + D * 64;   // [D][64]: ws[k * 64 + centroid of the chunk]
  __shared__ float bs[64];
  __shared__ float rsc[16][64];
  __shared__ int ridx[16][64];
  const long long bh = blockIdx.y;
  const int t0 = blockIdx.x * 64;
  const int nt = min(64, N - t0);
  const __nv_bfloat16* src = X + (bh * N + t0) * static_cast<long long>(D);
  for (int x = threadIdx.x; x < 64 * D / 8; x += 256) {
    const int r = x & 63, c8 = (x >> 6) * 8;
    uint4 u = make_uint4(0u, 0u, 0u, 0u);
    if (r < nt) u = __ldg(reinterpret_cast<const uint4*>(src + static_cast<long long>(r) * D + c8));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h[e]);
      xs[(c8 + 2 * e) * 64 + r] = f.x;
      xs[(c8 + 2 * e + 1) * 64 + r] = f.y;
    }
  }
  const int tg = threadIdx.x & 15, cg = threadIdx.x >> 4;
  float best[4];
  int bidx[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    best[i] = INFINITY;
    bidx[i] = 0x7fffffff;
  }
  const float* wsrc = W + bh * static_cast<long long>(C) * D;
  for (int cc = 0; cc < C; cc += 64) {
    const int ncc = min(64, C - cc);
    __syncthreads();   // the previous chunk is consumed (and, the first time, xs is written)
    for (int x = threadIdx.x; x < 64 * D / 4; x += 256) {
      const int c = x & 63, k4 = (x >> 6) * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c < ncc) v = __ldg(reinterpret_cast<const float4*>(wsrc + static_cast<long long>(cc + c) * D + k4));
      ws[(k4 + 0) * 64 + c] = v.x;
      ws[(k4 + 1) * 64 + c] = v.y;
      ws[(k4 + 2) * 64 + c] = v.z;
      ws[(k4 + 3) * 64 + c] = v.w;
    }
    if (threadIdx.x < 64) bs[threadIdx.x] = threadIdx.x < ncc ? bvec[bh * C + cc + threadIdx.x] : 0.f;
    __syncthreads();
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 8
    for (int k = 0; k < D; ++k) {
      const float4 xv = *reinterpret_cast<const float4*>(&xs[k * 64 + 4 * tg]);
      const float4 wv = *reinterpret_cast<const float4*>(&ws[k * 64 + 4 * cg]);
      const float xa[4] = {xv.x, xv.y, xv.z, xv.w};
      const float wa[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(xa[i], wa[j], acc[i][j]);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int cl = 4 * cg + j;
      if (cl < ncc) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float sc = bs[cl] - 2.f * acc[i][j];
          if (sc < best[i]) {       // centroids arrive in ascending order: ties keep the first
            best[i] = sc;
            bidx[i] = cc + cl;
          }
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    rsc[cg][4 * tg + i] = best[i];
    ridx[cg][4 * tg + i] = bidx[i];
  }
  __syncthreads();
  if (threadIdx.x < nt) {
    float b = rsc[0][threadIdx.x];
    int bi = ridx[0][threadIdx.x];
    for (int g = 1; g < 16; ++g) {
      const float v = rsc[g][threadIdx.x];
      const int vi = ridx[g][threadIdx.x];
      if (v < b || (v == b && vi < bi)) {
        b = v;
        bi = vi;
      }
    }
    // a NaN score never compares smaller: a token whose every score is NaN keeps
    // no cluster, which the range check below turns into cluster 0 and an error bit
    if (bi < 0 || bi >= C) {
      atomicOr(&g_dev_error, DEVERR_VALUE);
      bi = 0;
    }
    assign[bh * N + t0 + threadIdx.x] = bi;
    atomicAdd(&cnt[bh * C + bi], 1);
  }
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

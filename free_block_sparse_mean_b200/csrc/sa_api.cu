// C ABI of the block-sparse attention library: argument checks, workspace
// layout, TMA descriptors and launches. The kernels are in plan_kernels.cuh,
// fwd_kernel.cuh and cluster_kernels.cuh; the stage-1 launch sequence is in
// plan_launch.cuh, shared with the allocation-free entry point (sa_noalloc.cu,
// the library's second translation unit).
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <algorithm>
#include <cstring>
#include <mutex>

#include "../../include/sparse_attn.h"
#include "fwd_kernel.cuh"
#include "plan_kernels.cuh"
#include "plan_launch.cuh"
#include "cluster_kernels.cuh"

namespace {

inline int64_t num_blocks(const sa_shape& s) { return (static_cast<int64_t>(s.N) + 63) / 64; }


bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

sa_status check_shape(const sa_shape& s) {
  if (s.B < 1 || s.H < 1 || s.N < 1) return SA_ERR_INVALID_ARG;
  if (s.block != 64) return SA_ERR_UNSUPPORTED;
  if (s.d != 64 && s.d != 128) return SA_ERR_UNSUPPORTED;
  if (num_blocks(s) > sa::kMaxNb) return SA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(s.B) * s.H > 65535) return SA_ERR_UNSUPPORTED;
  return SA_OK;
}


// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// [B*H, N, d] bf16 viewed as a 3-D tensor {d, N, B*H}; box {64, rows, 1}, 128B swizzle.
// Rows past N of a head read as zero (out-of-bounds fill), never the next head.
bool make_map(CUtensorMap* map, const void* ptr, const sa_shape& s, int box_rows) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(s.d), static_cast<cuuint64_t>(s.N),
                        static_cast<cuuint64_t>(s.B) * s.H};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(s.d) * 2, static_cast<cuuint64_t>(s.N) * s.d * 2};
  cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(box_rows), 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// [B*H, N, d] bf16 viewed as a 4-D tensor {64 elements, N rows, d/64 chunks, B*H}
// (row stride 2d bytes, chunk stride 128 bytes): one box {64, 64, d/64, 1} is a
// whole 64-row block, landing in shared memory as [chunk][row][128 B] with the
// 128B swizzle, one TMA instruction per block. Rows past N of a head read as zero
// (out-of-bounds fill), never the next head.
bool make_block_map(CUtensorMap* map, const void* ptr, const sa_shape& s) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[4] = {64u, static_cast<cuuint64_t>(s.N), static_cast<cuuint64_t>(s.d / 64),
                        static_cast<cuuint64_t>(s.B) * s.H};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(s.d) * 2, 128u, static_cast<cuuint64_t>(s.N) * s.d * 2};
  cuuint32_t box[4] = {64u, 64u, static_cast<cuuint32_t>(s.d / 64), 1u};
  cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// FP8 codes [B*H, N, d] (d bytes per row) as a 3-D tensor {d, N, B*H}; box
// {d = 128, 64 rows, 1}, 128B swizzle: one load per 64-row block.
bool make_map8(CUtensorMap* map, const void* ptr, const sa_shape& s) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(s.d), static_cast<cuuint64_t>(s.N),
                        static_cast<cuuint64_t>(s.B) * s.H};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(s.d), static_cast<cuuint64_t>(s.N) * s.d};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(s.d), 64u, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// kRecall: the P.V filter is the recall test with budget = 1 - recall (lambda unused).
template <int D, int kQ = sa::kScoreBF16, bool kRecall = false>
sa_status launch_fwd(const sa_shape& s, const void* Q, const void* K, const void* V, const uint8_t* mask,
                     const int32_t* work, float lambda, float scale, int causal, void* O, int64_t* stats,
                     cudaStream_t st, const float* qscale = nullptr, const float* kscale = nullptr,
                     float budget = 0.f, uint8_t* decisions = nullptr) {
  using Cfg = sa::FwdCfg<D, kQ>;
  const int Nb = static_cast<int>(num_blocks(s));
  const int Tq = (Nb + 1) / 2;
  const long long tiles = static_cast<long long>(s.B) * s.H * Tq;
  if (tiles > 0x7fffffffLL) return SA_ERR_UNSUPPORTED;
  CUtensorMap mq, mk, mv;
  if (Cfg::kF8) {
    if (!make_map8(&mq, Q, s) || !make_map8(&mk, K, s)) return SA_ERR_CUDA;
  } else {
    if (!make_map(&mq, Q, s, 64) || !make_block_map(&mk, K, s)) return SA_ERR_CUDA;
  }
  if (!make_block_map(&mv, V, s)) return SA_ERR_CUDA;
  if (stats && cudaMemsetAsync(stats, 0, 4 * sizeof(int64_t), st) != cudaSuccess) return SA_ERR_CUDA;
  const float LOG2E = 1.4426950408889634f;
  const int lam_on = kRecall ? 1 : (std::isinf(lambda) && lambda < 0 ? 0 : 1);
  auto kern = sa::fwd_kernel<D, kQ, kRecall>;
  if (sa::set_smem(kern, Cfg::kSmemBytes) != SA_OK) return SA_ERR_CUDA;
  kern<<<static_cast<unsigned>(tiles), Cfg::kThreads, Cfg::kSmemBytes, st>>>(
      mq, mk, mv, mask, work, static_cast<__nv_bfloat16*>(O), s.N, Nb, Tq, tiles,
      static_cast<long long>(s.B) * s.H * Nb, scale * LOG2E,
      (lam_on && !kRecall) ? lambda * LOG2E : 0.f, lam_on, budget, causal,
      reinterpret_cast<unsigned long long*>(stats), qscale, kscale, decisions);
  if (cudaGetLastError() != cudaSuccess) return SA_ERR_CUDA;
  return SA_OK;
}

// The centroids' bf16 operand rows [B*H][C][2D + 64] as a 4-D tensor {64
// elements, C rows, D/32 + 1 chunks, B*H} (row stride 2(2D + 64) bytes, chunk
// stride 128 bytes): one box {64, 64, D/32 + 1, 1} is a 64-centroid tile with its
// high, low and bias chunks, landing as [chunk][row][128 B] with the 128B
// swizzle. Rows past C read as zero.
bool make_w16_map(CUtensorMap* map, const void* ptr, long long BH, int C, int D) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[4] = {64u, static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(D / 32 + 1),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(2 * D + 64) * 2, 128u,
                           static_cast<cuuint64_t>(C) * (2 * D + 64) * 2};
  cuuint32_t box[4] = {64u, 64u, static_cast<cuuint32_t>(D / 32 + 1), 1u};
  cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Interaction clustering of X under the Gram metric of Y (see cluster_kernels.cuh).
template <int D>
sa_status launch_cluster(const sa_shape& s, const void* X, const void* Y, int iters, int32_t* assign_out,
                         int32_t* perm, float* cent_out, void* ws, cudaStream_t st) {
  const int N = s.N;
  const long long BH = static_cast<long long>(s.B) * s.H;
  const sa::ClusterWorkspace L = sa::cluster_workspace(BH, N, D);
  const int C = L.C;
  char* wsb = static_cast<char*>(ws);
  float* gpart = reinterpret_cast<float*>(wsb + L.gpart);
  float* G = reinterpret_cast<float*>(wsb + L.gram);
  float* cent = reinterpret_cast<float*>(wsb + L.cent);
  float* W = reinterpret_cast<float*>(wsb + L.w);
  float* bvec = reinterpret_cast<float*>(wsb + L.b);
  int* cnt = reinterpret_cast<int*>(wsb + L.cnt);
  int* off = reinterpret_cast<int*>(wsb + L.off);
  int* assign = assign_out ? assign_out : reinterpret_cast<int*>(wsb + L.assign);
  auto* w16 = reinterpret_cast<__nv_bfloat16*>(wsb + L.w16);
  int* cand = reinterpret_cast<int*>(wsb + L.cand);
  const auto* x = static_cast<const __nv_bfloat16*>(X);
  const auto* y = static_cast<const __nv_bfloat16*>(Y);
  const unsigned by = static_cast<unsigned>(BH);
  if (sa::set_smem(sa::gram_tc_kernel<D>, sa::GramTcCfg<D>::kSmemBytes) != SA_OK) return SA_ERR_CUDA;
  sa::gram_tc_kernel<D><<<dim3(L.splits, by), 128, sa::GramTcCfg<D>::kSmemBytes, st>>>(y, gpart, N, L.splits, L.chunk);
  sa::gram_reduce_kernel<D><<<dim3(D * D / 256, by), 256, 0, st>>>(gpart, G, L.splits);
  // the block means (the pooling kernel, queries half only) and every token in its block
  sa::pool_kernel<D><<<dim3(static_cast<unsigned>(BH * C), 1), 256, 0, st>>>(x, x, cent, nullptr, N, C);
  const long long total = BH * N;
  sa::cluster_init_assign_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, st>>>(assign, cnt, N, C,
                                                                                               total);
  if (cudaGetLastError() != cudaSuccess) return SA_ERR_CUDA;
  using TC = sa::ClusterTcCfg<D>;
  if (sa::set_smem(sa::cluster_assign_tc_kernel<D>, TC::kSmemBytes) != SA_OK) return SA_ERR_CUDA;
  CUtensorMap mw;
  if (iters > 0 && !make_w16_map(&mw, w16, BH, C, D)) return SA_ERR_CUDA;
  int* part = reinterpret_cast<int*>(wsb + L.chunks);
  const dim3 chunk_grid(static_cast<unsigned>(L.order_chunks), by);
  const size_t hist_bytes = static_cast<size_t>(C) * sizeof(int);
  // the stable order of the current assignment (cnt holds the sizes)
  auto order = [&]() {
    sa::cluster_chunk_count_kernel<<<chunk_grid, 256, hist_bytes, st>>>(assign, part, N, C, L.order_len);
    sa::cluster_offsets_kernel<<<by, 1024, 0, st>>>(cnt, off, C);
    sa::cluster_chunk_scan_kernel<<<dim3((C + 255) / 256, by), 256, 0, st>>>(off, part, C, L.order_chunks);
    sa::cluster_order_kernel<<<chunk_grid, 32, hist_bytes, st>>>(assign, part, perm, N, C, L.order_len);
  };
  const dim3 cent_grid((C + 7) / 8, by);
  for (int it = 0; it < iters; ++it) {
    sa::cluster_prep_kernel<D><<<dim3((C + 15) / 16, by), D, 0, st>>>(G, cent, W, bvec, cnt, C, w16);
    sa::cluster_assign_tc_kernel<D><<<dim3((N + TC::kTok - 1) / TC::kTok, by), TC::kThreads, TC::kSmemBytes, st>>>(
        x, mw, N, C, cand);
    sa::cluster_rescore_kernel<D><<<dim3((N + 63) / 64, by), 256, 0, st>>>(x, W, bvec, cand, assign, cnt, N, C);
    order();
    // the means of the new clusters: the next iteration's centroids, or the output
    if (it + 1 < iters || cent_out)
      sa::cluster_centroid_kernel<D><<<cent_grid, 256, 0, st>>>(x, perm, off, cnt, cent, N, C);
    if (cudaGetLastError() != cudaSuccess) return SA_ERR_CUDA;
  }
  if (iters == 0) order();   // the plain blocks: identity order, block means from the pooling kernel
  if (cudaGetLastError() != cudaSuccess) return SA_ERR_CUDA;
  if (cent_out && cudaMemcpyAsync(cent_out, cent, static_cast<size_t>(BH) * C * D * sizeof(float),
                                  cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return SA_ERR_CUDA;
  return SA_OK;
}

}  // namespace

namespace sa {
cudaError_t take_noalloc_device_error(cudaStream_t st, unsigned int* out);   // sa_noalloc.cu

// Exercises the device-side failure path: one warp waits on an mbarrier whose
// phase nothing completes, through the same bounded wait the pipelines use, with
// a short limit. The wait gives up, records DEVERR_TIMEOUT in the error word and
// the kernel returns normally.
__global__ void __launch_bounds__(32) wait_timeout_selftest_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) mbar_wait_slow(&bar, 0u, &abort_flag, limit_ns);   // nothing arrives
  __syncwarp();
}
}  // namespace sa

extern "C" {

size_t sparse_attn_plan_workspace_size(sa_shape s) {
  if (check_shape(s) != SA_OK) return 0;
  return sa::plan_workspace(static_cast<long long>(s.B) * s.H, static_cast<int>(num_blocks(s)), s.d).total;
}

int64_t sparse_attn_num_tiles(sa_shape s) {
  if (check_shape(s) != SA_OK) return 0;
  return static_cast<int64_t>(s.B) * s.H * ((num_blocks(s) + 1) / 2);
}

sa_status sparse_attn_plan(const void* Q, const void* K, sa_shape s, float tau, float scale, int32_t causal,
                           uint8_t* mask, int32_t* count, int32_t* idx, int32_t* work, void* workspace,
                           size_t workspace_bytes, void* stream) {
  if (!Q || !K || !mask || !count) return SA_ERR_INVALID_ARG;
  const sa_status sh = check_shape(s);
  if (sh != SA_OK) return sh;
  if (!(tau > 0.f && tau <= 1.f)) return SA_ERR_INVALID_ARG;  // also rejects NaN
  if (!(std::isfinite(scale) && scale > 0.f)) return SA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K)) return SA_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      workspace_bytes < sparse_attn_plan_workspace_size(s))
    return SA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (s.d == 64)
    return sa::launch_plan<64>(s, Q, K, tau, nullptr, scale, causal != 0, mask, count, idx, work, workspace, st);
  return sa::launch_plan<128>(s, Q, K, tau, nullptr, scale, causal != 0, mask, count, idx, work, workspace, st);
}

sa_status sparse_attn_plan_heads(const void* Q, const void* K, sa_shape s, const float* tau, float scale,
                                 int32_t causal, uint8_t* mask, int32_t* count, int32_t* idx, int32_t* work,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  if (!Q || !K || !tau || !mask || !count) return SA_ERR_INVALID_ARG;
  const sa_status sh = check_shape(s);
  if (sh != SA_OK) return sh;
  if (!(std::isfinite(scale) && scale > 0.f)) return SA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || (reinterpret_cast<uintptr_t>(tau) & 3u) != 0) return SA_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      workspace_bytes < sparse_attn_plan_workspace_size(s))
    return SA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (s.d == 64)
    return sa::launch_plan<64>(s, Q, K, 1.f, tau, scale, causal != 0, mask, count, idx, work, workspace, st);
  return sa::launch_plan<128>(s, Q, K, 1.f, tau, scale, causal != 0, mask, count, idx, work, workspace, st);
}

sa_status sparse_attn_fwd(const void* Q, const void* K, const void* V, sa_shape s, const uint8_t* mask,
                          const int32_t* work, float lambda, float scale, int32_t causal, void* O,
                          int64_t* stats, void* stream) {
  if (!Q || !K || !V || !mask || !O) return SA_ERR_INVALID_ARG;
  const sa_status sh = check_shape(s);
  if (sh != SA_OK) return sh;
  if (std::isnan(lambda) || (std::isinf(lambda) && lambda > 0)) return SA_ERR_INVALID_ARG;
  if (!(std::isfinite(scale) && scale > 0.f)) return SA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return SA_ERR_INVALID_ARG;
  if (stats && (reinterpret_cast<uintptr_t>(stats) & 7u) != 0) return SA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (s.d == 64) return launch_fwd<64>(s, Q, K, V, mask, work, lambda, scale, causal != 0, O, stats, st);
  return launch_fwd<128>(s, Q, K, V, mask, work, lambda, scale, causal != 0, O, stats, st);
}

sa_status sparse_attn_fwd_recall(const void* Q, const void* K, const void* V, sa_shape s, const uint8_t* mask,
                                 const int32_t* work, float recall, float scale, int32_t causal, void* O,
                                 int64_t* stats, void* stream) {
  if (!Q || !K || !V || !mask || !O) return SA_ERR_INVALID_ARG;
  const sa_status sh = check_shape(s);
  if (sh != SA_OK) return sh;
  if (!(recall > 0.f && recall <= 1.f)) return SA_ERR_INVALID_ARG;  // also rejects NaN
  if (!(std::isfinite(scale) && scale > 0.f)) return SA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return SA_ERR_INVALID_ARG;
  if (stats && (reinterpret_cast<uintptr_t>(stats) & 7u) != 0) return SA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const float budget = 1.f - recall;
  if (s.d == 64)
    return launch_fwd<64, sa::kScoreBF16, true>(s, Q, K, V, mask, work, 0.f, scale, causal != 0, O, stats, st, nullptr,
                                       nullptr, budget);
  return launch_fwd<128, sa::kScoreBF16, true>(s, Q, K, V, mask, work, 0.f, scale, causal != 0, O, stats, st, nullptr,
                                      nullptr, budget);
}

sa_status sparse_attn_fwd_decisions(const void* Q, const void* K, const void* V, sa_shape s,
                                    const uint8_t* mask, const int32_t* work, int32_t filter, float value,
                                    float scale, int32_t causal, void* O, int64_t* stats, uint8_t* decisions,
                                    void* stream) {
  if (!Q || !K || !V || !mask || !O || !decisions) return SA_ERR_INVALID_ARG;
  const sa_status sh = check_shape(s);
  if (sh != SA_OK) return sh;
  if (filter == SA_FILTER_LAMBDA) {
    if (std::isnan(value) || (std::isinf(value) && value > 0)) return SA_ERR_INVALID_ARG;
  } else if (filter == SA_FILTER_RECALL) {
    if (!(value > 0.f && value <= 1.f)) return SA_ERR_INVALID_ARG;
  } else {
    return SA_ERR_INVALID_ARG;
  }
  if (!(std::isfinite(scale) && scale > 0.f)) return SA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return SA_ERR_INVALID_ARG;
  if (stats && (reinterpret_cast<uintptr_t>(stats) & 7u) != 0) return SA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool c = causal != 0;
  if (filter == SA_FILTER_RECALL) {
    const float budget = 1.f - value;
    if (s.d == 64)
      return launch_fwd<64, sa::kScoreBF16, true>(s, Q, K, V, mask, work, 0.f, scale, c, O, stats, st, nullptr, nullptr,
                                         budget, decisions);
    return launch_fwd<128, sa::kScoreBF16, true>(s, Q, K, V, mask, work, 0.f, scale, c, O, stats, st, nullptr, nullptr,
                                        budget, decisions);
  }
  if (s.d == 64)
    return launch_fwd<64>(s, Q, K, V, mask, work, value, scale, c, O, stats, st, nullptr, nullptr, 0.f, decisions);
  return launch_fwd<128>(s, Q, K, V, mask, work, value, scale, c, O, stats, st, nullptr, nullptr, 0.f, decisions);
}

// ---------------------------------------------------------------- host-buffer call
namespace {
// Device workspace of sparse_attn_host: Q, K, V, O copies, mask, count, work, the
// plan scratch of the largest head group, and with FP8 scores their codes and scales.
struct HostWorkspace {
  size_t q, k, v, o, mask, count, work, plan, q8, k8, qs, ks, total;
};
HostWorkspace host_workspace(const sa_shape& s, int chunks, bool fp8) {
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t BH = static_cast<size_t>(s.B) * s.H;
  const size_t Nb = static_cast<size_t>(num_blocks(s)), Tq = (Nb + 1) / 2;
  const size_t act = BH * s.N * s.d * 2;
  const long long group = (static_cast<long long>(BH) + chunks - 1) / chunks;
  HostWorkspace w{};
  size_t o = 0;
  w.q = o; o += al(act);
  w.k = o; o += al(act);
  w.v = o; o += al(act);
  w.o = o; o += al(act);
  w.mask = o; o += al(BH * Nb * Nb);
  w.count = o; o += al(BH * Nb * 4);
  w.work = o; o += al(2 * BH * Tq * 4);
  w.plan = o; o += al(sa::plan_workspace(group, static_cast<int>(Nb), s.d).total);
  if (fp8) {
    w.q8 = o; o += al(act / 2);
    w.k8 = o; o += al(act / 2);
    w.qs = o; o += al(BH * Nb * 4);
    w.ks = o; o += al(BH * Nb * 4);
  }
  w.total = o;
  return w;
}
}  // namespace

size_t sparse_attn_host_workspace_size(sa_shape s, int32_t chunks, int32_t flags) {
  if (check_shape(s) != SA_OK || chunks < 1) return 0;
  const long long BH = static_cast<long long>(s.B) * s.H;
  return host_workspace(s, static_cast<int>(std::min<long long>(chunks, BH)),
                        (flags & (SA_HOST_FP8_SCORES | SA_HOST_INT8_SCORES)) != 0)
      .total;
}

sa_status sparse_attn_host(const void* Qh, const void* Kh, const void* Vh, sa_shape s, float tau,
                           const float* tau_heads, int32_t filter, float value, float scale, int32_t causal,
                           int32_t flags, void* Oh, void* workspace,
                           size_t workspace_bytes, int32_t chunks, void* stream, void* copy_in_stream,
                           void* copy_out_stream) {
  if (!Qh || !Kh || !Vh || !Oh) return SA_ERR_INVALID_ARG;
  const sa_status sh = check_shape(s);
  if (sh != SA_OK) return sh;
  const bool fp8 = (flags & SA_HOST_FP8_SCORES) != 0, i8 = (flags & SA_HOST_INT8_SCORES) != 0;
  if ((flags & ~(SA_HOST_FP8_SCORES | SA_HOST_INT8_SCORES)) != 0 || (fp8 && i8) || chunks < 1)
    return SA_ERR_INVALID_ARG;
  const bool q8 = fp8 || i8;                       // 8-bit score codes
  if (tau_heads ? (reinterpret_cast<uintptr_t>(tau_heads) & 3u) != 0 : !(tau > 0.f && tau <= 1.f))
    return SA_ERR_INVALID_ARG;
  if (!(std::isfinite(scale) && scale > 0.f)) return SA_ERR_INVALID_ARG;
  if (filter == SA_FILTER_LAMBDA) {
    if (std::isnan(value) || (std::isinf(value) && value > 0)) return SA_ERR_INVALID_ARG;
  } else if (filter == SA_FILTER_RECALL) {
    if (!(value > 0.f && value <= 1.f) || q8) return SA_ERR_INVALID_ARG;
  } else {
    return SA_ERR_INVALID_ARG;
  }
  if (q8 && s.d != 128) return SA_ERR_UNSUPPORTED;
  const long long BH = static_cast<long long>(s.B) * s.H;
  const int nch = static_cast<int>(std::min<long long>(chunks, BH));
  const HostWorkspace L = host_workspace(s, nch, q8);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || workspace_bytes < L.total)
    return SA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaStream_t cin = copy_in_stream ? static_cast<cudaStream_t>(copy_in_stream) : st;
  cudaStream_t cout = copy_out_stream ? static_cast<cudaStream_t>(copy_out_stream) : st;
  char* ws = static_cast<char*>(workspace);
  const int Nb = static_cast<int>(num_blocks(s)), Tq = (Nb + 1) / 2;
  const size_t row_bytes = static_cast<size_t>(s.N) * s.d * 2;   // one head of Q, K, V or O

  // Events order the three streams; each is released at the end of the call
  // (the runtime keeps it alive until its recorded work has completed).
  cudaEvent_t start = nullptr, finish = nullptr;
  cudaEvent_t ev[2 * 64] = {};
  const int nev = 2 * std::min(nch, 64);
  sa_status rc = SA_OK;
  auto ok = [&](cudaError_t e) {
    if (e != cudaSuccess && rc == SA_OK) rc = SA_ERR_CUDA;
    return e == cudaSuccess;
  };
  if (!ok(cudaEventCreateWithFlags(&start, cudaEventDisableTiming)) ||
      !ok(cudaEventCreateWithFlags(&finish, cudaEventDisableTiming)))
    goto done;
  for (int i = 0; i < nev; ++i)
    if (!ok(cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming))) goto done;
  // the copies may only overwrite the workspace once earlier work on `stream` is done
  if (!ok(cudaEventRecord(start, st)) || !ok(cudaStreamWaitEvent(cin, start, 0)) ||
      !ok(cudaStreamWaitEvent(cout, start, 0)))
    goto done;
  for (int c = 0; c < nch && rc == SA_OK; ++c) {
    const long long lo = BH * c / nch, hi = BH * (c + 1) / nch;
    if (hi == lo) continue;
    cudaEvent_t in_ready = ev[2 * (c % 64)], out_ready = ev[2 * (c % 64) + 1];
    const size_t off = static_cast<size_t>(lo) * row_bytes, bytes = static_cast<size_t>(hi - lo) * row_bytes;
    if (!ok(cudaMemcpyAsync(ws + L.q + off, static_cast<const char*>(Qh) + off, bytes, cudaMemcpyHostToDevice, cin)) ||
        !ok(cudaMemcpyAsync(ws + L.k + off, static_cast<const char*>(Kh) + off, bytes, cudaMemcpyHostToDevice, cin)) ||
        !ok(cudaMemcpyAsync(ws + L.v + off, static_cast<const char*>(Vh) + off, bytes, cudaMemcpyHostToDevice, cin)) ||
        !ok(cudaEventRecord(in_ready, cin)) || !ok(cudaStreamWaitEvent(st, in_ready, 0)))
      break;
    const sa_shape g{1, static_cast<int32_t>(hi - lo), s.N, s.d, 64};
    const void* q = ws + L.q + off;
    const void* k = ws + L.k + off;
    const void* v = ws + L.v + off;
    void* o = ws + L.o + off;
    uint8_t* mask = reinterpret_cast<uint8_t*>(ws + L.mask) + static_cast<size_t>(lo) * Nb * Nb;
    int32_t* count = reinterpret_cast<int32_t*>(ws + L.count) + static_cast<size_t>(lo) * Nb;
    int32_t* work = reinterpret_cast<int32_t*>(ws + L.work) + static_cast<size_t>(2) * lo * Tq;
    void* pws = ws + L.plan;
    const float* tg = tau_heads ? tau_heads + lo : nullptr;   // this group's per-head thresholds
    sa_status r;
    if (q8) {
      uint8_t* c8q = reinterpret_cast<uint8_t*>(ws + L.q8) + off / 2;
      uint8_t* c8k = reinterpret_cast<uint8_t*>(ws + L.k8) + off / 2;
      float* qs = reinterpret_cast<float*>(ws + L.qs) + static_cast<size_t>(lo) * Nb;
      float* ks = reinterpret_cast<float*>(ws + L.ks) + static_cast<size_t>(lo) * Nb;
      r = sa::launch_plan<128>(g, q, k, tau, tg, scale, causal != 0, mask, count, nullptr, work, pws, st, c8q, c8k,
                               qs, ks, i8 ? sa::kScoreI8 : sa::kScoreE4M3);
      if (r == SA_OK)
        r = i8 ? launch_fwd<128, sa::kScoreI8>(g, c8q, c8k, v, mask, work, value, scale, causal != 0, o, nullptr, st,
                                               qs, ks)
               : launch_fwd<128, sa::kScoreE4M3>(g, c8q, c8k, v, mask, work, value, scale, causal != 0, o, nullptr,
                                                 st, qs, ks);
    } else {
      r = s.d == 64 ? sa::launch_plan<64>(g, q, k, tau, tg, scale, causal != 0, mask, count, nullptr, work, pws, st)
                    : sa::launch_plan<128>(g, q, k, tau, tg, scale, causal != 0, mask, count, nullptr, work, pws,
                                           st);
      if (r == SA_OK) {
        if (filter == SA_FILTER_RECALL)
          r = s.d == 64 ? launch_fwd<64, sa::kScoreBF16, true>(g, q, k, v, mask, work, 0.f, scale, causal != 0, o, nullptr,
                                                      st, nullptr, nullptr, 1.f - value)
                        : launch_fwd<128, sa::kScoreBF16, true>(g, q, k, v, mask, work, 0.f, scale, causal != 0, o, nullptr,
                                                       st, nullptr, nullptr, 1.f - value);
        else
          r = s.d == 64 ? launch_fwd<64>(g, q, k, v, mask, work, value, scale, causal != 0, o, nullptr, st)
                        : launch_fwd<128>(g, q, k, v, mask, work, value, scale, causal != 0, o, nullptr, st);
      }
    }
    if (r != SA_OK) {
      rc = r;
      break;
    }
    if (!ok(cudaEventRecord(out_ready, st)) || !ok(cudaStreamWaitEvent(cout, out_ready, 0)) ||
        !ok(cudaMemcpyAsync(static_cast<char*>(Oh) + off, ws + L.o + off, bytes, cudaMemcpyDeviceToHost, cout)))
      break;
  }
  // `stream` completes only once the last copy back has
  if (rc == SA_OK) {
    ok(cudaEventRecord(finish, cout));
    ok(cudaStreamWaitEvent(st, finish, 0));
  }
done:
  for (int i = 0; i < nev; ++i)
    if (ev[i]) cudaEventDestroy(ev[i]);
  if (start) cudaEventDestroy(start);
  if (finish) cudaEventDestroy(finish);
  return rc;
}

size_t sparse_attn_cluster_workspace_size(sa_shape s) {
  if (check_shape(s) != SA_OK) return 0;
  return sa::cluster_workspace(static_cast<long long>(s.B) * s.H, s.N, s.d).total;
}

sa_status sparse_attn_cluster(const void* X, const void* Y, sa_shape s, int32_t iters, int32_t* assign,
                              int32_t* perm, float* centroids, void* workspace, size_t workspace_bytes,
                              void* stream) {
  if (!X || !Y || !perm) return SA_ERR_INVALID_ARG;
  const sa_status sh = check_shape(s);
  if (sh != SA_OK) return sh;
  if (iters < 0 || iters > 64) return SA_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Y) || (reinterpret_cast<uintptr_t>(perm) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(assign) & 3u) != 0 || (reinterpret_cast<uintptr_t>(centroids) & 3u) != 0)
    return SA_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      workspace_bytes < sparse_attn_cluster_workspace_size(s))
    return SA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (s.d == 64) return launch_cluster<64>(s, X, Y, iters, assign, perm, centroids, workspace, st);
  return launch_cluster<128>(s, X, Y, iters, assign, perm, centroids, workspace, st);
}

sa_status sparse_attn_permute_rows(const void* src, const int32_t* perm, sa_shape s, int32_t inverse, void* dst,
                                   void* stream) {
  if (!src || !perm || !dst || src == dst) return SA_ERR_INVALID_ARG;
  const sa_status sh = check_shape(s);
  if (sh != SA_OK) return sh;
  if (!aligned16(src) || !aligned16(dst) || (reinterpret_cast<uintptr_t>(perm) & 3u) != 0)
    return SA_ERR_INVALID_ARG;
  const dim3 grid(static_cast<unsigned>((static_cast<long long>(s.N) * (s.d / 8) + 1023) / 1024),
                  static_cast<unsigned>(static_cast<long long>(s.B) * s.H));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const auto* x = static_cast<const __nv_bfloat16*>(src);
  auto* y = static_cast<__nv_bfloat16*>(dst);
  if (s.d == 64)
    sa::permute_rows_kernel<64><<<grid, 256, 0, st>>>(x, perm, y, s.N, inverse != 0);
  else
    sa::permute_rows_kernel<128><<<grid, 256, 0, st>>>(x, perm, y, s.N, inverse != 0);
  if (cudaGetLastError() != cudaSuccess) return SA_ERR_CUDA;
  return SA_OK;
}

const char* sparse_attn_status_string(sa_status st) {
  switch (st) {
    case SA_OK: return "SA_OK";
    case SA_ERR_INVALID_ARG: return "SA_ERR_INVALID_ARG: null pointer, bad size or value, or misaligned pointer";
    case SA_ERR_UNSUPPORTED: return "SA_ERR_UNSUPPORTED: d must be 64 or 128, block 64, Nb <= 4096, B*H <= 65535";
    case SA_ERR_WORKSPACE: return "SA_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case SA_ERR_CUDA: return "SA_ERR_CUDA: a CUDA call or kernel launch failed";
    case SA_ERR_DEVICE_CHECK: return "SA_ERR_DEVICE_CHECK: a device-side check fired";
  }
  return "unknown sa_status";
}

sa_status sparse_attn_plan_q8(const void* Q, const void* K, sa_shape s, float tau, float scale, int32_t causal,
                              uint8_t* mask, int32_t* count, int32_t* idx, int32_t* work, void* Q8, void* K8,
                              float* qscale, float* kscale, void* workspace, size_t workspace_bytes,
                              void* stream) {
  if (!Q || !K || !mask || !count || !Q8 || !K8 || !qscale || !kscale) return SA_ERR_INVALID_ARG;
  const sa_status sh = check_shape(s);
  if (sh != SA_OK) return sh;
  if (s.d != 128) return SA_ERR_UNSUPPORTED;
  if (!(tau > 0.f && tau <= 1.f)) return SA_ERR_INVALID_ARG;
  if (!(std::isfinite(scale) && scale > 0.f)) return SA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(Q8) || !aligned16(K8) ||
      (reinterpret_cast<uintptr_t>(qscale) & 3u) != 0 || (reinterpret_cast<uintptr_t>(kscale) & 3u) != 0)
    return SA_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      workspace_bytes < sparse_attn_plan_workspace_size(s))
    return SA_ERR_WORKSPACE;
  return sa::launch_plan<128>(s, Q, K, tau, nullptr, scale, causal != 0, mask, count, idx, work, workspace,
                          static_cast<cudaStream_t>(stream), static_cast<uint8_t*>(Q8), static_cast<uint8_t*>(K8),
                          qscale, kscale);
}

sa_status sparse_attn_fwd_q8(const void* Q8, const void* K8, const float* qscale, const float* kscale,
                             const void* V, sa_shape s, const uint8_t* mask, const int32_t* work, float lambda,
                             float scale, int32_t causal, void* O, int64_t* stats, void* stream) {
  if (!Q8 || !K8 || !qscale || !kscale || !V || !mask || !O) return SA_ERR_INVALID_ARG;
  const sa_status sh = check_shape(s);
  if (sh != SA_OK) return sh;
  if (s.d != 128) return SA_ERR_UNSUPPORTED;
  if (std::isnan(lambda) || (std::isinf(lambda) && lambda > 0)) return SA_ERR_INVALID_ARG;
  if (!(std::isfinite(scale) && scale > 0.f)) return SA_ERR_INVALID_ARG;
  if (!aligned16(Q8) || !aligned16(K8) || !aligned16(V) || !aligned16(O) ||
      (reinterpret_cast<uintptr_t>(qscale) & 3u) != 0 || (reinterpret_cast<uintptr_t>(kscale) & 3u) != 0)
    return SA_ERR_INVALID_ARG;
  if (stats && (reinterpret_cast<uintptr_t>(stats) & 7u) != 0) return SA_ERR_INVALID_ARG;
  return launch_fwd<128, sa::kScoreE4M3>(s, Q8, K8, V, mask, work, lambda, scale, causal != 0, O, stats,
                               static_cast<cudaStream_t>(stream), qscale, kscale);
}

sa_status sparse_attn_plan_i8(const void* Q, const void* K, sa_shape s, float tau, float scale, int32_t causal,
                              uint8_t* mask, int32_t* count, int32_t* idx, int32_t* work, void* Q8, void* K8,
                              float* qscale, float* kscale, void* workspace, size_t workspace_bytes,
                              void* stream) {
  if (!Q || !K || !mask || !count || !Q8 || !K8 || !qscale || !kscale) return SA_ERR_INVALID_ARG;
  const sa_status sh = check_shape(s);
  if (sh != SA_OK) return sh;
  if (s.d != 128) return SA_ERR_UNSUPPORTED;
  if (!(tau > 0.f && tau <= 1.f)) return SA_ERR_INVALID_ARG;
  if (!(std::isfinite(scale) && scale > 0.f)) return SA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(Q8) || !aligned16(K8) ||
      (reinterpret_cast<uintptr_t>(qscale) & 3u) != 0 || (reinterpret_cast<uintptr_t>(kscale) & 3u) != 0)
    return SA_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      workspace_bytes < sparse_attn_plan_workspace_size(s))
    return SA_ERR_WORKSPACE;
  return sa::launch_plan<128>(s, Q, K, tau, nullptr, scale, causal != 0, mask, count, idx, work, workspace,
                          static_cast<cudaStream_t>(stream), static_cast<uint8_t*>(Q8), static_cast<uint8_t*>(K8),
                          qscale, kscale, sa::kScoreI8);
}

sa_status sparse_attn_fwd_i8(const void* Q8, const void* K8, const float* qscale, const float* kscale,
                             const void* V, sa_shape s, const uint8_t* mask, const int32_t* work, float lambda,
                             float scale, int32_t causal, void* O, int64_t* stats, void* stream) {
  if (!Q8 || !K8 || !qscale || !kscale || !V || !mask || !O) return SA_ERR_INVALID_ARG;
  const sa_status sh = check_shape(s);
  if (sh != SA_OK) return sh;
  if (s.d != 128) return SA_ERR_UNSUPPORTED;
  if (std::isnan(lambda) || (std::isinf(lambda) && lambda > 0)) return SA_ERR_INVALID_ARG;
  if (!(std::isfinite(scale) && scale > 0.f)) return SA_ERR_INVALID_ARG;
  if (!aligned16(Q8) || !aligned16(K8) || !aligned16(V) || !aligned16(O) ||
      (reinterpret_cast<uintptr_t>(qscale) & 3u) != 0 || (reinterpret_cast<uintptr_t>(kscale) & 3u) != 0)
    return SA_ERR_INVALID_ARG;
  if (stats && (reinterpret_cast<uintptr_t>(stats) & 7u) != 0) return SA_ERR_INVALID_ARG;
  return launch_fwd<128, sa::kScoreI8>(s, Q8, K8, V, mask, work, lambda, scale, causal != 0, O, stats,
                               static_cast<cudaStream_t>(stream), qscale, kscale);
}

sa_status sparse_attn_selftest_wait_timeout(uint32_t limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 4000000) return SA_ERR_INVALID_ARG;
  sa::wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<unsigned long long>(limit_us) * 1000ull);
  if (cudaGetLastError() != cudaSuccess) return SA_ERR_CUDA;
  return SA_OK;
}

sa_status sparse_attn_device_error(void* stream, int32_t* code) {
  if (!code) return SA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbolAsync(&v, sa::g_dev_error, sizeof(v), 0, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return SA_ERR_CUDA;
  if (cudaMemcpyToSymbolAsync(sa::g_dev_error, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, st) !=
      cudaSuccess)
    return SA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return SA_ERR_CUDA;
  unsigned int w = 0;   // the other translation unit's word (see sa_noalloc.cu)
  if (sa::take_noalloc_device_error(st, &w) != cudaSuccess) return SA_ERR_CUDA;
  *code = static_cast<int32_t>(v | w);
  return SA_OK;
}

}  // extern "C"

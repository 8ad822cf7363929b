// Host-side launch sequence of stage 1 (pool -> pooled scores + selection ->
// tile order), shared by the workspace entry points (sa_api.cu) and the
// allocation-free one (sa_noalloc.cu): both pass a scratch region laid out by
// plan_workspace and get the same kernels, grid shapes and shared-memory sizes.
#pragma once

#include <mutex>

#include "../../include/sparse_attn.h"
#include "plan_kernels.cuh"

namespace sa {

// Raises a kernel's dynamic shared-memory limit (the attribute belongs to the
// current device's context; the mutex keeps concurrent first calls orderly).
template <typename F>
inline sa_status set_smem(F* kernel, int bytes) {
  static std::mutex mu;
  std::lock_guard<std::mutex> lk(mu);
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return SA_ERR_CUDA;
  return SA_OK;
}

// Stage 1 on the stream: pool Q and K (and, with Q8 given, write their 8-bit
// codes in format qfmt and per-block scales), the pooled scores and the cumulative-energy selection
// (mask, count, optional idx), then, with `work` given, the tile pairs and their
// order. `scratch` holds plan_workspace(B*H, Nb, D).total bytes, 256-byte aligned.
// tau_bh, when given, is a device array of one threshold per (b, h) that replaces tau.
template <int D>
sa_status launch_plan(const sa_shape& s, const void* Q, const void* K, float tau, const float* tau_bh,
                      float scale, int causal, uint8_t* mask, int32_t* count, int32_t* idx, int32_t* work,
                      void* scratch, cudaStream_t st, uint8_t* Q8 = nullptr, uint8_t* K8 = nullptr,
                      float* qscale = nullptr, float* kscale = nullptr, int qfmt = kScoreE4M3) {
  const int Nb = static_cast<int>((static_cast<int64_t>(s.N) + 63) / 64);
  const long long BH = static_cast<long long>(s.B) * s.H;
  const PlanWorkspace L = plan_workspace(BH, Nb, D);
  char* wsb = static_cast<char*>(scratch);
  float* Qp = reinterpret_cast<float*>(wsb + L.qp);
  float* Kp = reinterpret_cast<float*>(wsb + L.kp);
  unsigned long long* sig = reinterpret_cast<unsigned long long*>(wsb + L.sig);
  uint32_t* bits = reinterpret_cast<uint32_t*>(wsb + L.bits);
  uint32_t* bitsT = pair_bits_in_smem(Nb) ? nullptr : reinterpret_cast<uint32_t*>(wsb + L.bitsT);
  pool_kernel<D><<<dim3(static_cast<unsigned>(BH * Nb), 2), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(Q), static_cast<const __nv_bfloat16*>(K), Qp, Kp, s.N, Nb, Q8, K8, qscale,
      kscale, qfmt);
  if (cudaGetLastError() != cudaSuccess) return SA_ERR_CUDA;

  // R query blocks per CTA: 4 for short heads so that the grid still fills the GPU.
  auto launch_ss = [&](auto kern, int R, int NT) -> sa_status {
    const int smem = R == 4 ? score_select_smem_bytes<D, 4>(Nb)
                            : (R == 8 ? score_select_smem_bytes<D, 8>(Nb) : score_select_smem_bytes<D, 16>(Nb));
    if (set_smem(kern, smem) != SA_OK) return SA_ERR_CUDA;
    kern<<<dim3((Nb + R - 1) / R, static_cast<unsigned>(BH)), NT, smem, st>>>(Qp, Kp, Nb, scale, causal, tau,
                                                                               tau_bh, mask, count, idx, sig, bits);
    return SA_OK;
  };
  sa_status ls;
  if (Nb <= 256)
    ls = launch_ss(score_select_kernel<D, 4, 128>, 4, 128);
  else if (Nb <= 1536)
    ls = launch_ss(score_select_kernel<D, 16, 256>, 16, 256);
  else if (Nb <= 3000)   // 16 warps: a row per warp in the selection, two-pass score rows
    ls = launch_ss(score_select_kernel<D, 16, 512>, 16, 512);
  else
    ls = launch_ss(score_select_kernel<D, 8, 256>, 8, 256);
  if (ls != SA_OK) return ls;
  if (cudaGetLastError() != cudaSuccess) return SA_ERR_CUDA;

  if (work) {
    const int Tq = (Nb + 1) / 2;
    const int smem = pair_order_smem_bytes(Nb);
    if (set_smem(pair_order_kernel, smem) != SA_OK) return SA_ERR_CUDA;
    const int G = order_group_heads(BH, s.N, D);
    pair_order_kernel<<<static_cast<unsigned>(BH), pair_order_threads(Nb), smem, st>>>(sig, bits, count, Nb, Tq,
                                                                                     G, work, bitsT);
    if (cudaGetLastError() != cudaSuccess) return SA_ERR_CUDA;
  }
  return SA_OK;
}

}  // namespace sa

// Host-side launch sequence of stage 1 (pool -> pooled scores -> selection ->
// tile order), shared by the workspace entry points (sa_api.cu) and the
// allocation-free one (sa_noalloc.cu): both pass a scratch region laid out by
// plan_workspace and get the same kernels and arithmetic (only the number of
// score strips per batch may differ, which changes no result).
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
// codes in format qfmt and per-block scales), the pooled scores in batches of
// 128-block strips (pooled_scores_kernel) each followed by their selection
// (mask, count, optional idx), then, with `work` given, the tile pairs and their
// order. `scratch` holds plan_workspace(B*H, Nb, D, score_cap).total bytes,
// 256-byte aligned. tau_bh, when given, is a device array of one threshold per
// (b, h) that replaces tau.
template <int D>
sa_status launch_plan(const sa_shape& s, const void* Q, const void* K, float tau, const float* tau_bh,
                      float scale, int causal, uint8_t* mask, int32_t* count, int32_t* idx, int32_t* work,
                      void* scratch, cudaStream_t st, uint8_t* Q8 = nullptr, uint8_t* K8 = nullptr,
                      float* qscale = nullptr, float* kscale = nullptr, int qfmt = kScoreE4M3,
                      size_t score_cap = kPlanScoreBytes) {
  const int Nb = static_cast<int>((static_cast<int64_t>(s.N) + 63) / 64);
  const long long BH = static_cast<long long>(s.B) * s.H;
  const PlanWorkspace L = plan_workspace(BH, Nb, D, score_cap);
  char* wsb = static_cast<char*>(scratch);
  float* Qp = reinterpret_cast<float*>(wsb + L.qp);
  float* Kp = reinterpret_cast<float*>(wsb + L.kp);
  unsigned long long* sig = reinterpret_cast<unsigned long long*>(wsb + L.sig);
  uint32_t* bits = reinterpret_cast<uint32_t*>(wsb + L.bits);
  uint32_t* bitsT = pair_bits_in_smem(Nb) ? nullptr : reinterpret_cast<uint32_t*>(wsb + L.bitsT);
  float* scores = reinterpret_cast<float*>(wsb + L.scores);
  pool_kernel<D><<<dim3(static_cast<unsigned>(BH * Nb), 2), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(Q), static_cast<const __nv_bfloat16*>(K), Qp, Kp, s.N, Nb, Q8, K8, qscale,
      kscale, qfmt);
  if (cudaGetLastError() != cudaSuccess) return SA_ERR_CUDA;

  const bool shortrows = Nb <= 256;
  const int ssm = select_smem_bytes(Nb);
  if (set_smem(shortrows ? select_kernel<true> : select_kernel<false>, ssm) != SA_OK) return SA_ERR_CUDA;
  const unsigned nct = static_cast<unsigned>((Nb + 127) / 128);
  for (int s0 = 0; s0 < L.strips; s0 += L.strips_per_batch) {
    const unsigned ns = static_cast<unsigned>(min(L.strips_per_batch, L.strips - s0));
    if (Nb <= 64)   // one 64-block tile per head
      pooled_scores_kernel<D, 64><<<dim3(1, ns), 256, 0, st>>>(Qp, Kp, Nb, scale, causal, s0, scores);
    else
      pooled_scores_kernel<D, 128><<<dim3(nct, ns), 256, 0, st>>>(Qp, Kp, Nb, scale, causal, s0, scores);
    if (shortrows)
      select_kernel<true><<<dim3(32, ns), 128, ssm, st>>>(scores, Nb, s0, tau, tau_bh, mask, count, idx, sig, bits);
    else
      select_kernel<false><<<dim3(32, ns), 128, ssm, st>>>(scores, Nb, s0, tau, tau_bh, mask, count, idx, sig,
                                                           bits);
    if (cudaGetLastError() != cudaSuccess) return SA_ERR_CUDA;
  }

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

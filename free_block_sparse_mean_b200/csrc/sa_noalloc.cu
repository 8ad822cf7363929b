// sparse_attn_plan_noalloc: the plan call for callers that cannot allocate device
// memory.
//
// Some hosts cannot give this library a workspace. Examples: an inference
// runtime that reserves its whole device-memory budget at start-up and hands
// out nothing afterwards; a plugin whose host process owns the allocator and
// gives the plugin none; a latency-critical path where a cudaMalloc, which can
// synchronise the device or fail once memory is fragmented, is not acceptable.
// This entry point needs no workspace: the pooled Q and K live in a fixed
// array of device memory that is part of the loaded library.
//
// Scratch: kNoAllocScratchBytes = 32 MiB, a file-scope __device__ array. Every
// GPU that loads the library holds it until the process exits. A call needs the
// same bytes as sparse_attn_plan_workspace_size: the pooled Q and K
// (2 * B*H*ceil(N/64)*d*4 bytes) plus, per query block, an 8-byte sort key and a
// ceil(Nb/32)-word bitset of its kept set (for example H=24, d=128 fits up to
// N = 75,776). Larger calls are rejected with SA_ERR_WORKSPACE before
// anything runs.
//
// Every call shares the one array, and the array keeps the last call's
// contents. The kernels write every scratch byte they later read, so nothing
// has to start at zero. Calls whose work overlaps on the GPU (on two streams,
// or from two host threads) race on the array and give wrong masks: order them
// on one stream or otherwise serialise them.
//
// The first call on each device looks up the array's device address with
// cudaGetSymbolAddress (in host code the array's name is only a host-side
// stand-in, not a device address) and caches it for that device; make that
// first call before any stream capture on the device.
#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/sparse_attn.h"
#include "plan_kernels.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_plan_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};


// Device address of the scratch array on the current device (set up once per device).
sa_status scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_plan_scratch) != cudaSuccess || p == nullptr) return SA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return SA_OK;
}

template <int D>
sa_status launch_plan_noalloc(const sa_shape& s, const void* Q, const void* K, float tau, float scale,
                              int causal, uint8_t* mask, int32_t* count, int32_t* idx, int32_t* work,
                              void* scratch, cudaStream_t st) {
  const int Nb = static_cast<int>((static_cast<int64_t>(s.N) + 63) / 64);
  const long long BH = static_cast<long long>(s.B) * s.H;
  const sa::PlanWorkspace L = sa::plan_workspace(BH, Nb, D);
  char* wsb = static_cast<char*>(scratch);
  float* Qp = reinterpret_cast<float*>(wsb + L.qp);
  float* Kp = reinterpret_cast<float*>(wsb + L.kp);
  unsigned long long* sig = reinterpret_cast<unsigned long long*>(wsb + L.sig);
  uint32_t* bits = reinterpret_cast<uint32_t*>(wsb + L.bits);
  sa::pool_kernel<D><<<dim3(static_cast<unsigned>(BH * Nb), 2), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(Q), static_cast<const __nv_bfloat16*>(K), Qp, Kp, s.N, Nb);
  if (cudaGetLastError() != cudaSuccess) return SA_ERR_CUDA;
  // Small heads: 4 query blocks per CTA so the grid still fills the GPU.
  auto launch_ss = [&](auto kern, int R, int NT) -> sa_status {
    const int smem = R == 4 ? sa::score_select_smem_bytes<D, 4>(Nb)
                            : (R == 8 ? sa::score_select_smem_bytes<D, 8>(Nb) : sa::score_select_smem_bytes<D, 16>(Nb));
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return SA_ERR_CUDA;
    kern<<<dim3((Nb + R - 1) / R, static_cast<unsigned>(BH)), NT, smem, st>>>(Qp, Kp, Nb, scale, causal, tau,
                                                                               nullptr, mask, count, idx, sig, bits);
    return SA_OK;
  };
  sa_status ls;
  if (Nb <= 256)
    ls = launch_ss(sa::score_select_kernel<D, 4, 128>, 4, 128);
  else if (Nb <= 3000)
    ls = launch_ss(sa::score_select_kernel<D, 16, 256>, 16, 256);
  else
    ls = launch_ss(sa::score_select_kernel<D, 8, 256>, 8, 256);
  if (ls != SA_OK) return ls;
  if (cudaGetLastError() != cudaSuccess) return SA_ERR_CUDA;
  if (work) {
    const int Tq = (Nb + 1) / 2;
    const int smem = sa::pair_order_smem_bytes(Nb);
    if (cudaFuncSetAttribute(sa::pair_order_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return SA_ERR_CUDA;
    sa::pair_order_kernel<<<static_cast<unsigned>(BH), sa::pair_order_threads(Nb), smem, st>>>(
        sig, bits, count, Nb, Tq, sa::order_group_heads(BH, s.N, D), work);
    if (cudaGetLastError() != cudaSuccess) return SA_ERR_CUDA;
  }
  return SA_OK;
}

}  // namespace

namespace sa {
// Reads and clears this translation unit's copy of the device error word. The
// plan kernels are templates instantiated here and in the main translation unit;
// a launch may run either unit's copy, and each copy reports into its own unit's
// word, so sparse_attn_device_error reads both.
cudaError_t take_noalloc_device_error(cudaStream_t st, unsigned int* out) {
  unsigned int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_dev_error, sizeof(*out), 0, cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return e;
  e = cudaMemcpyToSymbolAsync(g_dev_error, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return e;
  return cudaStreamSynchronize(st);
}
}  // namespace sa

extern "C" sa_status sparse_attn_plan_noalloc(const void* Q, const void* K, sa_shape s, float tau, float scale,
                                              int32_t causal, uint8_t* mask, int32_t* count, int32_t* idx,
                                              int32_t* work, void* stream) {
  if (!Q || !K || !mask || !count) return SA_ERR_INVALID_ARG;
  if (s.B < 1 || s.H < 1 || s.N < 1) return SA_ERR_INVALID_ARG;
  if (s.block != 64 || (s.d != 64 && s.d != 128)) return SA_ERR_UNSUPPORTED;
  if ((static_cast<int64_t>(s.N) + 63) / 64 > sa::kMaxNb) return SA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(s.B) * s.H > 65535) return SA_ERR_UNSUPPORTED;
  if (!(tau > 0.f && tau <= 1.f)) return SA_ERR_INVALID_ARG;
  if (!(std::isfinite(scale) && scale > 0.f)) return SA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(Q) & 15u) || (reinterpret_cast<uintptr_t>(K) & 15u)) return SA_ERR_INVALID_ARG;
  const sa::PlanWorkspace need = sa::plan_workspace(static_cast<long long>(s.B) * s.H,
                                                    static_cast<int>((static_cast<int64_t>(s.N) + 63) / 64), s.d);
  if (need.total > kNoAllocScratchBytes) return SA_ERR_WORKSPACE;  // beyond the fixed scratch
  void* scratch = nullptr;
  const sa_status got = scratch_for_current_device(&scratch);
  if (got != SA_OK) return got;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (s.d == 64)
    return launch_plan_noalloc<64>(s, Q, K, tau, scale, causal != 0, mask, count, idx, work, scratch, st);
  return launch_plan_noalloc<128>(s, Q, K, tau, scale, causal != 0, mask, count, idx, work, scratch, st);
}

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
// fixed regions of sparse_attn_plan_workspace_size (the pooled Q and K,
// 2 * B*H*ceil(N/64)*d*4 bytes, plus, per query block, an 8-byte sort key and a
// ceil(Nb/32)-word bitset of its kept set, and, above about 1,200 blocks per
// head, the pairing's copy of the bitsets) and room for at least one strip of
// pooled scores (128 rows of ceil(Nb/32)*32 floats); the strips take whatever is
// left (for example H=24, d=128 fits up to N = 74,432). Larger calls are rejected
// with SA_ERR_WORKSPACE before anything runs.
//
// Every call shares the one array, and the array keeps the last call's
// contents. The kernels write every scratch byte they later read, so nothing
// has to start at zero. Calls whose work overlaps on the GPU (on two streams,
// or from two host threads) race on the array and give wrong masks: order them
// on one stream or otherwise serialise them.
//
// Each call made outside stream capture looks up the array's device address on
// the current device with cudaGetSymbolAddress (in host code the array's name is
// only a host-side stand-in, not a device address) and remembers it for that
// device; a call made while its stream is being captured uses the remembered
// address. So make the first call on a device before any stream capture on it
// (a first call inside a capture returns SA_ERR_CUDA).
#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/sparse_attn.h"
#include "plan_launch.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_plan_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device. A call made outside
// stream capture looks the address up again (cheap), so a context that was torn
// down and re-created, e.g. after cudaDeviceReset, gets the array's new address;
// a call made while `st` is being captured uses the address cached by the last
// call outside capture, since a lookup could load the module inside the capture.
sa_status scratch_for_current_device(cudaStream_t st, void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SA_ERR_CUDA;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cap) != cudaSuccess) return SA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (cap == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_plan_scratch) != cudaSuccess || p == nullptr) return SA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  } else if (!g_scratch_ptr[dev]) {
    return SA_ERR_CUDA;   // first call on this device inside a capture: no address yet
  }
  *out = g_scratch_ptr[dev];
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
  // the fixed regions and one score strip must fit; the strips then take the rest
  const long long BH = static_cast<long long>(s.B) * s.H;
  const int Nb = static_cast<int>((static_cast<int64_t>(s.N) + 63) / 64);
  const sa::PlanWorkspace least = sa::plan_workspace(BH, Nb, s.d, 0);
  if (least.total > kNoAllocScratchBytes) return SA_ERR_WORKSPACE;  // beyond the fixed scratch
  const size_t score_cap = kNoAllocScratchBytes - least.scores;
  void* scratch = nullptr;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const sa_status got = scratch_for_current_device(st, &scratch);
  if (got != SA_OK) return got;
  if (s.d == 64)
    return sa::launch_plan<64>(s, Q, K, tau, nullptr, scale, causal != 0, mask, count, idx, work, scratch, st,
                               nullptr, nullptr, nullptr, nullptr, sa::kScoreE4M3, score_cap);
  return sa::launch_plan<128>(s, Q, K, tau, nullptr, scale, causal != 0, mask, count, idx, work, scratch, st,
                              nullptr, nullptr, nullptr, nullptr, sa::kScoreE4M3, score_cap);
}

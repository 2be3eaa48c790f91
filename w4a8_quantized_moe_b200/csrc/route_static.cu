// route_static.cu - w4a8_moe_route_permute_noalloc: routing + permutation for
// callers that cannot allocate device memory.
//
// Some callers may not call cudaMalloc or any allocating routine at the point
// where they route tokens: runtimes and plugin interfaces that hand a kernel
// only its pre-planned input and output buffers and no scratch, and
// latency-critical paths whose device memory budget is fixed up front.  This
// entry point takes only inputs and outputs; its
// scratch (per-block expert histograms, their scanned bases and the GEMM tile
// prefix) lives in the file-scope device array below, which every device that
// loads the library holds until the process exits.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <mutex>

#include "../../include/w4a8.h"
#include "internal.h"

namespace w4a8 {
const char* set_last_error(const char* msg);
}

namespace {

// Capacity: ceil(T / 256) * E <= kTableEntries (e.g. T = 65536 with E = 256,
// or T = 16384 with E = 1024).
constexpr int64_t kTableEntries = 65536;
constexpr int64_t kScratchInts = 2 * kTableEntries + (w4a8::kMaxExperts + 1);

// 2 * 65536 + 1025 int32 = 528,388 bytes of device memory per device.
static __device__ __align__(256) int32_t g_route_scratch[kScratchInts];

std::mutex g_mu;
int32_t* g_scratch_ptr[64] = {};

// Device address of g_route_scratch on the current device.  In host code the
// array's name is only a host-side stand-in; the kernels need the address the
// runtime reports for the current device, looked up once per device and kept
// for the life of the process.  cudaDeviceReset discards the device's copy of
// the array, so the kept address is stale afterwards: a process that resets a
// device must not call w4a8_moe_route_permute_noalloc on it again.
w4a8_status scratch_for_current_device(int32_t** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) {
    w4a8::set_last_error(cudaGetErrorString(err));
    return W4A8_ERR_CUDA;
  }
  if (dev < 0 || dev >= 64) {
    w4a8::set_last_error("device ordinal above 63 is not supported by the static scratch");
    return W4A8_ERR_INVALID_ARG;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_route_scratch);
    if (err != cudaSuccess || !p) {
      w4a8::set_last_error(err != cudaSuccess ? cudaGetErrorString(err)
                                              : "cudaGetSymbolAddress returned NULL");
      return W4A8_ERR_CUDA;
    }
    g_scratch_ptr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_scratch_ptr[dev];
  return W4A8_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" W4A8_API w4a8_status w4a8_moe_route_permute_noalloc(
    const float* logits, int64_t T, int32_t E, int32_t k, int32_t* topk_ids, float* topk_w,
    int32_t* expert_offsets, int32_t* sorted_token_ids, int32_t* row_of, void* stream) {
  if (T < 0) {
    w4a8::set_last_error("T < 0");
    return W4A8_ERR_INVALID_ARG;
  }
  if (E < 1 || E > w4a8::kMaxExperts || k < 1 || k > E || k > w4a8::kMaxTopK) {
    w4a8::set_last_error("need 1 <= E <= 1024 and 1 <= k <= min(E, 32)");
    return W4A8_ERR_UNSUPPORTED_SHAPE;
  }
  const int64_t entries = w4a8::route_blocks(T) * static_cast<int64_t>(E);
  if (entries > kTableEntries) {
    static thread_local char msg[256];
    snprintf(msg, sizeof(msg),
             "T = %lld, E = %d needs %lld scratch entries per table; the static scratch holds "
             "%lld (ceil(T / 256) * E <= %lld); use w4a8_moe_route_permute with a workspace",
             static_cast<long long>(T), E, static_cast<long long>(entries),
             static_cast<long long>(kTableEntries), static_cast<long long>(kTableEntries));
    w4a8::set_last_error(msg);
    return W4A8_ERR_UNSUPPORTED_SHAPE;
  }
  if (!expert_offsets || (T > 0 && (!logits || !topk_ids || !topk_w || !sorted_token_ids ||
                                    !row_of))) {
    w4a8::set_last_error("NULL pointer argument");
    return W4A8_ERR_INVALID_ARG;
  }
  for (const void* p : {static_cast<const void*>(logits), static_cast<const void*>(topk_ids),
                        static_cast<const void*>(topk_w), static_cast<const void*>(expert_offsets),
                        static_cast<const void*>(sorted_token_ids),
                        static_cast<const void*>(row_of)})
    if (!aligned16(p)) {
      w4a8::set_last_error("pointers must be 16-byte aligned");
      return W4A8_ERR_INVALID_ARG;
    }
  int major = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
    w4a8::set_last_error("cannot query the current device");
    return W4A8_ERR_CUDA;
  }
  if (major != 10) {
    w4a8::set_last_error("this library is built for sm_100a (compute capability 10.x)");
    return W4A8_ERR_UNSUPPORTED_ARCH;
  }
  int32_t* scratch = nullptr;
  if (w4a8_status st = scratch_for_current_device(&scratch)) return st;
  // The histograms are zeroed inside launch_route on `stream`; the bases and
  // the tile prefix are fully rewritten before they are read.
  cudaError_t err = w4a8::launch_route(logits, T, E, k, topk_ids, topk_w, expert_offsets,
                                       sorted_token_ids, row_of, scratch, scratch + kTableEntries,
                                       scratch + 2 * kTableEntries, w4a8::kTileNPrefill,
                                       nullptr, static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) {
    w4a8::set_last_error(cudaGetErrorString(err));
    return W4A8_ERR_CUDA;
  }
  return W4A8_OK;
}
